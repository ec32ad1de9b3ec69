"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Packed codes, scales and superblock records must be byte-identical to the
oracle's, rq_dequant bit-identical (RWKV-7 G1 1.5B int4 model card: kernel
output is bit-identical to the offline dequantization), and y within the
stated tolerance: relative L2 error <= 5e-3 and per element
|y - y_ref| <= 1e-2 * sum_k |x_k| |w_hat_k|, against the oracle's fp64 sums.
Inputs come from the seeded generators; the oracle never sees a CUDA result
as an input.
"""
import numpy as np
import pytest
import torch

import headroom
import oracle
import weight_only_quantized_rq_b200 as rq
from weight_only_quantized_rq_b200 import workloads as wl

pytestmark = pytest.mark.gpu

GROUP = {"w4g64": 64, "w8g16": 16, "w4sb32": 32}


@pytest.fixture(scope="module", autouse=True)
def _setup():
    from weight_only_quantized_rq_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    yield
    assert rq.rq_device_status() == 0


# ------------------------------------------------------------ helpers ------
def to_dev(a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()


def scales_used(fmt, K, N):
    return 0 if fmt == "w4sb32" else N * (K // GROUP[fmt]) * 2


def gpu_planes(p, fmt, K, N):
    codes = p.codes.cpu().numpy()
    if p.scales is None:
        return codes.reshape(N, -1), None
    raw = p.scales.cpu().numpy()
    used = scales_used(fmt, K, N)
    assert not raw[used:].any(), "scale-plane padding must be zero"
    return codes.reshape(N, -1), raw[:used].view(np.uint16).reshape(N, -1)


def upload(fmt, K, N, codes, scales):
    """A Packed matrix whose planes hold the ORACLE's bytes."""
    p = rq.alloc_packed(fmt, K, N)
    p.codes.copy_(torch.from_numpy(np.ascontiguousarray(codes).reshape(-1)))
    if p.scales is not None:
        p.scales.zero_()
        raw = np.ascontiguousarray(scales).view(np.uint8).reshape(-1)
        p.scales[: raw.size].copy_(torch.from_numpy(raw))
    return p


def make_x(seed, M, K, a=None):
    x = wl.random_x(seed, M, K, a)
    return x, wl.bf16_bits(x)


check_y = headroom.check_y


# --------------------------------------------------------- quantize-pack ---
PACK_CASES = [
    # fmt, K, N, act recipe, n_cand, (t_lo, t_hi), outliers
    ("w4g64", 64, 1, None, 1, (0.7, 1.0), False),
    ("w4g64", 768, 45, "ch5", 1, (1.0, 1.0), False),
    ("w4g64", 2048, 37, "ch1202", 64, (0.7, 1.0), False),
    ("w4g64", 320, 9, "rand", 7, (0.5, 1.2), True),
    ("w4g64", 1024, 16, None, 256, (0.7, 1.0), False),
    ("w8g16", 2048, 29, None, 64, (0.7, 1.0), True),
    ("w8g16", 64, 3, "rand", 33, (0.6, 1.0), False),
    ("w8g16", 4096, 5, "eight", 64, (0.7, 1.0), True),
    ("w4sb32", 2560, 19, "eight", 64, (0.7, 1.0), False),
    ("w4sb32", 256, 3, None, 1, (1.0, 1.0), False),
    ("w4sb32", 1024, 11, "rand", 40, (0.5, 1.1), True),
]


def act_for(recipe, K, seed):
    if recipe is None:
        return None
    if recipe == "ch5":
        a = np.ones(K, np.float32); a[5] = 2500.0; return a
    if recipe == "ch1202":
        a = np.ones(K, np.float32); a[1202 % K] = 2500.0; return a
    if recipe == "eight":
        return wl.random_act_sq(seed, K, massive=8, energy=15631.0)
    rng = np.random.default_rng(seed)
    return (rng.random(K) * 3).astype(np.float32)


def weights_for(seed, N, K, outliers):
    W = wl.random_matrix(seed, N, K).numpy()
    if outliers:
        rng = np.random.default_rng(seed + 1)
        idx = rng.choice(N * K, size=max(1, N * K // 1000), replace=False)
        W.reshape(-1)[idx] *= 10.0
    return W


@pytest.mark.parametrize("case", range(len(PACK_CASES)))
def test_quantize_pack_bytes_match_oracle(case):
    fmt, K, N, recipe, n, (lo, hi), out = PACK_CASES[case]
    W = weights_for(100 + case, N, K, out)
    a = act_for(recipe, K, 200 + case)
    oc, osc = oracle.pack(fmt, W, a, n_cand=n, t_lo=lo, t_hi=hi)
    p = rq.rq_quantize_pack(to_dev(W), fmt, to_dev(a), n, lo, hi)
    gc, gsc = gpu_planes(p, fmt, K, N)
    assert np.array_equal(gc, oc.reshape(N, -1))
    if osc is not None:
        assert np.array_equal(gsc, osc)
    # the dequant export is bit-identical to the oracle's dequantization
    wd = rq.rq_dequant(p).cpu().numpy()
    assert np.array_equal(wd.view(np.uint32), oracle.dequant(fmt, K, N, oc, osc).view(np.uint32))


def test_quantize_pack_deterministic_and_in_bounds():
    fmt, K, N = "w4g64", 2048, 33
    W = to_dev(wl.random_matrix(7, N, K).numpy())
    p1 = rq.rq_quantize_pack(W, fmt)
    # a guard band around both planes must stay untouched
    cb, sb = rq.rq_packed_size(fmt, K, N)
    big_c = torch.full((cb + 512,), 0xA5, dtype=torch.uint8, device="cuda")
    big_s = torch.full((sb + 512,), 0x5A, dtype=torch.uint8, device="cuda")
    p2 = rq.Packed(p1.fmt, K, N, big_c[256:256 + cb], big_s[256:256 + sb])
    rq.rq_quantize_pack(W, fmt, out=p2)
    torch.cuda.synchronize()
    assert torch.equal(p1.codes, p2.codes) and torch.equal(p1.scales, p2.scales)
    for buf, v, n in ((big_c, 0xA5, cb), (big_s, 0x5A, sb)):
        assert bool((buf[:256] == v).all()) and bool((buf[256 + n:] == v).all())


def test_all_zero_and_tiny_groups():
    K, N = 256, 4
    W = np.zeros((N, K), np.float32)
    W[1, :64] = 7 * 2.0 ** -24          # every candidate rounds to the same fp16 subnormal
    W[2, ::3] = 1e-30                   # underflows to a zero scale
    W[3] = wl.random_matrix(3, 1, K).numpy()
    for fmt in ("w4g64", "w8g16", "w4sb32"):
        oc, osc = oracle.pack(fmt, W, None, n_cand=64)
        p = rq.rq_quantize_pack(to_dev(W), fmt)
        gc, gsc = gpu_planes(p, fmt, K, N)
        assert np.array_equal(gc, oc.reshape(N, -1))
        if osc is not None:
            assert np.array_equal(gsc, osc)


# -------------------------------------------------------------- product ----
WGEMM_CASES = [
    # fmt, K, N, M
    ("w4g64", 2048, 2048, 1),
    ("w4g64", 2048, 300, 1),
    ("w4g64", 768, 768, 1),
    ("w4g64", 8192, 130, 1),
    ("w4g64", 64, 5, 1),
    ("w4g64", 320, 77, 3),
    ("w4g64", 2048, 257, 2),
    ("w4g64", 2048, 129, 4),
    ("w4g64", 1024, 200, 5),
    ("w4g64", 4096, 96, 8),
    ("w4g64", 2048, 64, 17),
    ("w4g64", 2048, 64, 32),
    ("w4g64", 1024, 40, 64),
    ("w4g64", 512, 24, 128),
    ("w4g64", 16384, 40, 1),
    ("w4g64", 32768, 8, 1),
    ("w8g16", 2048, 2048, 1),
    ("w8g16", 2048, 111, 2),
    ("w8g16", 4096, 64, 4),
    ("w8g16", 448, 33, 8),
    ("w8g16", 1024, 16, 128),
    ("w4sb32", 2560, 2560, 1),
    ("w4sb32", 10240, 72, 1),
    ("w4sb32", 2560, 99, 8),
    ("w4sb32", 256, 7, 32),
    ("w4sb32", 768, 33, 3),
    # M >= 33: int4 g64 and int8 g16 on the tensor-core prefill kernel
    ("w4g64", 2048, 300, 33),
    ("w4g64", 4096, 257, 64),
    ("w4g64", 768, 130, 100),
    ("w4g64", 64, 5, 128),
    ("w4g64", 320, 77, 48),
    ("w4g64", 16384, 40, 128),
    ("w8g16", 4096, 200, 64),
    ("w8g16", 2048, 129, 128),
    ("w8g16", 448, 33, 80),
    # superblock records on the tensor-core kernel (M >= 3)
    ("w4sb32", 512, 40, 64),
    ("w4sb32", 2560, 300, 16),
    ("w4sb32", 10240, 130, 128),
    # more tiles than SMs: persistent CTAs take two tiles (double-buffered accumulator)
    ("w4g64", 512, 20000, 16),
    ("w8g16", 256, 19500, 8),
    # K split over a cluster with a half stage at the end of K (int4 scale windows)
    ("w4g64", 832, 200, 24),
    ("w8g16", 832, 130, 40),
]


@pytest.mark.parametrize("case", range(len(WGEMM_CASES)))
def test_wgemm_matches_oracle(case):
    fmt, K, N, M = WGEMM_CASES[case]
    W = wl.random_matrix(300 + case, N, K).numpy()
    a = wl.random_act_sq(400 + case, K, massive=2)
    oc, osc = oracle.pack(fmt, W, a, n_cand=8)
    p = upload(fmt, K, N, oc, osc)
    x, xb = make_x(500 + case, M, K, a)
    y = rq.rq_wgemm(x.cuda(), p).cpu().numpy()
    y_ref = oracle.wgemm(fmt, xb, K, N, oc, osc)
    check_y(y, y_ref, xb, oracle.dequant(fmt, K, N, oc, osc), fmt)


@pytest.mark.parametrize("fmt,unit", [("w4g64", 2.0 ** -6), ("w8g16", 2.0 ** -10)])
@pytest.mark.parametrize("M", [1, 3, 8, 64, 128])
def test_wgemm_exact_integer_products(fmt, unit, M):
    """w = q 2^-e and small-integer x: every partial sum is an integer
    multiple of 2^-e below 2^24, so the fp32 result must be exact."""
    G, qmax = GROUP[fmt], oracle.QMAX[fmt]
    rng = np.random.default_rng(17)
    K, N = 2048, 100
    q = rng.integers(-qmax, qmax + 1, size=(N, K))
    q.reshape(N, K // G, G)[:, :, 0] = qmax
    W = (q * unit).astype(np.float32)
    p = rq.rq_quantize_pack(to_dev(W), fmt, None, 1, 1.0, 1.0)
    xi = rng.integers(-8, 9, size=(M, K))
    x = torch.from_numpy(xi.astype(np.float32)).to(torch.bfloat16)
    y = rq.rq_wgemm(x.cuda(), p).cpu().numpy().astype(np.float64)
    assert np.array_equal(y, (xi @ q.T).astype(np.float64) * unit)


def test_wgemm_exact_superblock():
    """Superblock weights c (q - 8) 2^-12 need up to 9 significant bits: exact
    in the fp32 GEMV path (M <= 2); the tensor-core path (M >= 3) rounds w_hat
    to bf16 and is covered by the tolerance cases."""
    rng = np.random.default_rng(23)
    N, K, M = 50, 1024, 2
    q = rng.integers(0, 16, size=(N, K))
    qg = q.reshape(N, K // 32, 32)
    qg[:, :, 0], qg[:, :, 1] = 0, 15
    c = rng.integers(1, 64, size=(N, K // 32))
    c.reshape(N, -1, 8)[:, :, 0] = 63
    W = (c.repeat(32, axis=1) * (q - 8) * 2.0 ** -12).astype(np.float32)
    p = rq.rq_quantize_pack(to_dev(W), "w4sb32")
    assert np.array_equal(rq.rq_dequant(p).cpu().numpy(), W)
    xi = rng.integers(-8, 9, size=(M, K))
    x = torch.from_numpy(xi.astype(np.float32)).to(torch.bfloat16)
    y = rq.rq_wgemm(x.cuda(), p).cpu().numpy().astype(np.float64)
    want = (xi[:, None, :] * (c.repeat(32, axis=1) * (q - 8))[None]).sum(-1) * 2.0 ** -12
    assert np.array_equal(y, want)


def test_wgemm_guard_band_and_repeatability():
    fmt, K, N, M = "w4g64", 2048, 333, 2
    W = wl.random_matrix(5, N, K).numpy()
    p = rq.rq_quantize_pack(to_dev(W), fmt)
    x, _ = make_x(6, M, K)
    xd = x.cuda()
    big = torch.full((M * N + 2048,), float("nan"), device="cuda")
    y = big[1024:1024 + M * N].view(M, N)
    rq.rq_wgemm(xd, p, y)
    y2 = rq.rq_wgemm(xd, p)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    assert bool(torch.isnan(big[:1024]).all()) and bool(torch.isnan(big[1024 + M * N:]).all())


# ------------------------------------------- full sizes, sampled outputs ----
def _full_size_check(widx, layer_sample=1, rows_per_matrix=48, Ms=None):
    w = wl.WORKLOADS[widx]
    rng = np.random.default_rng(1000 + widx)
    for j, layer, m in w.matrices():
        if layer >= layer_sample:
            break
        W = wl.weights(w, j, m)
        a = wl.act_sq(w, m.K)
        p = rq.rq_quantize_pack(W.cuda(), m.fmt, to_dev(a) if m.n_cand > 1 else None, m.n_cand,
                                0.7 if m.n_cand > 1 else 1.0, 1.0)
        rows = np.sort(rng.choice(m.N, size=min(rows_per_matrix, m.N), replace=False)).astype(np.int32)
        rows[-1] = m.N - 1
        Wr = W.numpy()[rows]
        oc, osc = oracle.pack(m.fmt, Wr, a if m.n_cand > 1 else None, n_cand=m.n_cand,
                              t_lo=0.7 if m.n_cand > 1 else 1.0, t_hi=1.0)
        gc, gsc = gpu_planes(p, m.fmt, m.K, m.N)
        assert np.array_equal(gc[rows], oc.reshape(len(rows), -1)), (m.name, "codes")
        if osc is not None:
            assert np.array_equal(gsc[rows], osc), (m.name, "scales")
        for M in (Ms or w.Ms):
            x = wl.activations(w, j, m.K, M)
            xb = wl.bf16_bits(x)
            y = rq.rq_wgemm(x.cuda(), p).cpu().numpy()
            y_ref = oracle.wgemm(m.fmt, xb, m.K, len(rows), oc, osc)
            check_y(y[:, rows], y_ref, xb, oracle.dequant(m.fmt, m.K, len(rows), oc, osc), m.fmt)
        del p


@pytest.mark.parametrize("widx", [0, 1, 2, 3, 4])
def test_full_size_workloads_sampled(widx):
    _full_size_check(widx)


# --------------------------------------------------------------- batches ---
@pytest.mark.parametrize("fmt,shapes,M", [
    ("w4g64", [(2048, 2048), (2048, 8192), (8192, 2048), (768, 5), (2048, 1)], 1),
    ("w4g64", [(1024, 300), (1024, 64), (4096, 77)], 2),
    ("w8g16", [(2048, 130), (4096, 33), (448, 9)], 1),
    ("w4sb32", [(2560, 200), (10240, 40), (256, 3)], 3),
    ("w4sb32", [(2560, 2560), (2560, 1000), (10240, 77)], 32),
    ("w4g64", [(2048, 300), (4096, 129), (64, 7)], 64),
    ("w8g16", [(1024, 257), (448, 5)], 128),
    ("w4g64", [(512, 9000), (1024, 12000), (320, 3)], 32),
    ("w8g16", [(256, 4000), (512, 300), (2048, 16000)], 4),
])
def test_wgemm_batch_matches_oracle(fmt, shapes, M):
    """One launch over products of different shapes equals the oracle per
    product; outputs are written only inside each y (guard bands)."""
    xs, ws, ys, refs = [], [], [], []
    bigs = []
    for i, (K, N) in enumerate(shapes):
        W = wl.random_matrix(700 + i, N, K).numpy()
        oc, osc = oracle.pack(fmt, W, None, n_cand=4)
        p = upload(fmt, K, N, oc, osc)
        x, xb = make_x(800 + i, M, K)
        big = torch.full((M * N + 512,), float("nan"), device="cuda")
        xs.append(x.cuda())
        ws.append(p)
        ys.append(big[256:256 + M * N].view(M, N))
        bigs.append((big, M * N))
        refs.append((oracle.wgemm(fmt, xb, K, N, oc, osc), xb, oracle.dequant(fmt, K, N, oc, osc)))
    rq.rq_wgemm_batch(xs, ws, ys)
    torch.cuda.synchronize()
    for y, (y_ref, xb, wd), (big, n) in zip(ys, refs, bigs):
        check_y(y.cpu().numpy(), y_ref, xb, wd, fmt)
        assert bool(torch.isnan(big[:256]).all()) and bool(torch.isnan(big[256 + n:]).all())


def test_wgemm_batch_equals_single_calls():
    """The batched launch gives bit-identical outputs to one call per item
    (each row's sum is formed by the same lanes in the same order)."""
    fmt, M = "w4g64", 1
    shapes = [(2048, 2048)] * 3 + [(2048, 8192), (8192, 2048)]
    xs, ws = [], []
    for i, (K, N) in enumerate(shapes):
        ws.append(rq.rq_quantize_pack(wl.random_matrix(900 + i, N, K).cuda(), fmt))
        xs.append(make_x(950 + i, M, K)[0].cuda())
    ys = [torch.empty(M, w.N, device="cuda") for w in ws]
    rq.rq_wgemm_batch(xs, ws, ys)
    singles = [rq.rq_wgemm(x, w) for x, w in zip(xs, ws)]
    torch.cuda.synchronize()
    for a, b in zip(ys, singles):
        assert torch.equal(a, b)


# ------------------------------------------------------------ bf16 output ---
@pytest.mark.parametrize("fmt,K,N,M", [
    ("w4g64", 2048, 300, 1),       # register path
    ("w8g16", 2048, 129, 2),
    ("w4sb32", 2560, 77, 1),
    ("w8g64", 1024, 64, 2),
    ("w4g64", 2048, 300, 16),      # tensor-core epilogue
    ("w8g16", 448, 33, 128),
    ("w4sb32", 2560, 300, 8),
    ("w5sb32", 2560, 99, 1),
    ("w6g16", 768, 200, 5),
    ("w4g64", 4096, 200, 24),      # K split over a cluster (rank-order DSMEM reduction)
    ("w4g64", 4096, 203, 40),      # the same with N % 4 != 0 (element stores)
])
def test_wgemm_bf16_output_is_the_rounded_fp32(fmt, K, N, M):
    """The bf16-output epilogue writes exactly the fp32 result rounded to
    nearest even, and nothing outside y."""
    W = wl.random_matrix(3100 + K + N, N, K).cuda()
    p = rq.rq_quantize_pack(W, fmt, None, 8)
    x, _ = make_x(3200 + M, M, K)
    xd = x.cuda()
    y32 = rq.rq_wgemm(xd, p)
    big = torch.full((M * N + 512,), float("nan"), dtype=torch.bfloat16, device="cuda")
    y16 = big[256:256 + M * N].view(M, N)
    rq.rq_wgemm(xd, p, y16)
    torch.cuda.synchronize()
    assert torch.equal(y16.view(torch.int16), y32.to(torch.bfloat16).view(torch.int16))
    assert bool(torch.isnan(big[:256]).all()) and bool(torch.isnan(big[256 + M * N:]).all())


@pytest.mark.parametrize("fmt,M", [("w4g64", 1), ("w4g64", 16), ("w8g16", 4)])
def test_wgemm_batch_bf16_output(fmt, M):
    """r/k/v-style batch (three 2048^2 products) with bf16 outputs."""
    xs, ws, y32s, y16s = [], [], [], []
    for i in range(3):
        ws.append(rq.rq_quantize_pack(wl.random_matrix(3300 + i, 2048, 2048).cuda(), fmt, None, 4))
        xs.append(make_x(3400 + i, M, 2048)[0].cuda())
        y32s.append(torch.empty(M, 2048, device="cuda"))
        y16s.append(torch.empty(M, 2048, dtype=torch.bfloat16, device="cuda"))
    rq.rq_wgemm_batch(xs, ws, y32s)
    rq.rq_wgemm_batch(xs, ws, y16s)
    torch.cuda.synchronize()
    for a, b in zip(y16s, y32s):
        assert torch.equal(a.view(torch.int16), b.to(torch.bfloat16).view(torch.int16))
