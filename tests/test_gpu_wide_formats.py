"""Parity of the preset variants between the CUDA path and the CPU oracle:
the 5- and 6-bit asymmetric superblock formats (the COMPRESSION preset's wider
matrices: ffn.key and head in 5 bits, embedding and LoRA branches in 6;
rwkv-quant article, "Two presets and six sizes"), the 6-bit symmetric group-16
format (the REDUCTION preset's channel-mix) and the int8 group-64 tier
(RWKV-7 G1 1.5B int4 model card, "Accuracy warning").

Packed bytes must be identical to the oracle's, rq_dequant bit-identical, and
y within the tolerance of the other formats. The 5- and 6-bit formats have no
register-path kernel: every M, 1 included, runs on the tensor-core kernel
(w_hat rounded once to bf16). int8 g64 runs on the register path at M <= 2
(exact fp32 w_hat; an exact integer-product case checks it) and on the tensor
cores above.
"""
import numpy as np
import pytest
import torch

import headroom
import oracle
import weight_only_quantized_rq_b200 as rq
from weight_only_quantized_rq_b200 import workloads as wl

pytestmark = pytest.mark.gpu

WIDE = ("w5sb32", "w6sb32")
SYM = ("w6g16", "w8g64")


@pytest.fixture(scope="module", autouse=True)
def _setup():
    from weight_only_quantized_rq_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    yield
    assert rq.rq_device_status() == 0


def to_dev(a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()


def upload(fmt, K, N, codes, scales=None):
    p = rq.alloc_packed(fmt, K, N)
    assert (p.scales is None) == (scales is None)
    p.codes.copy_(torch.from_numpy(np.ascontiguousarray(codes).reshape(-1)))
    if scales is not None:
        p.scales.zero_()
        raw = np.ascontiguousarray(scales).view(np.uint8).reshape(-1)
        p.scales[: raw.size].copy_(torch.from_numpy(raw))
    return p


def gpu_scales(p, K, N, fmt):
    raw = p.scales.cpu().numpy()
    used = N * (K // oracle.GROUP[fmt]) * 2
    assert not raw[used:].any(), "scale-plane padding must be zero"
    return raw[:used].view(np.uint16).reshape(N, -1)


check_y = headroom.check_y


def weights_for(seed, N, K, outliers):
    W = wl.random_matrix(seed, N, K).numpy()
    if outliers:
        rng = np.random.default_rng(seed + 1)
        idx = rng.choice(N * K, size=max(1, N * K // 1000), replace=False)
        W.reshape(-1)[idx] *= 10.0
    return W


# --------------------------------------------------------- quantize-pack ---
PACK_CASES = [
    # K, N, act recipe, n_cand, (t_lo, t_hi), outliers
    (2560, 19, "eight", 64, (0.7, 1.0), False),
    (256, 3, None, 1, (1.0, 1.0), False),
    (1024, 11, "rand", 40, (0.5, 1.1), True),
    (4096, 7, "eight", 256, (0.7, 1.0), True),
]


def act_for(recipe, K, seed):
    if recipe is None:
        return None
    if recipe == "eight":
        return wl.random_act_sq(seed, K, massive=8, energy=15631.0)
    rng = np.random.default_rng(seed)
    return (rng.random(K) * 3).astype(np.float32)


@pytest.mark.parametrize("fmt", WIDE)
@pytest.mark.parametrize("case", range(len(PACK_CASES)))
def test_pack_records_match_oracle(fmt, case):
    K, N, recipe, n, (lo, hi), out = PACK_CASES[case]
    W = weights_for(1100 + case, N, K, out)
    a = act_for(recipe, K, 1200 + case)
    oc, osc = oracle.pack(fmt, W, a, n_cand=n, t_lo=lo, t_hi=hi)
    assert osc is None
    p = rq.rq_quantize_pack(to_dev(W), fmt, to_dev(a), n, lo, hi)
    assert p.scales is None
    assert np.array_equal(p.codes.cpu().numpy().reshape(N, -1), oc.reshape(N, -1))
    wd = rq.rq_dequant(p).cpu().numpy()
    assert np.array_equal(wd.view(np.uint32), oracle.dequant(fmt, K, N, oc, None).view(np.uint32))


@pytest.mark.parametrize("fmt", WIDE)
def test_all_zero_and_tiny_groups(fmt):
    K, N = 512, 4
    W = np.zeros((N, K), np.float32)
    W[1, :64] = 7 * 2.0 ** -24
    W[2, ::3] = 1e-30
    W[3] = wl.random_matrix(3, 1, K).numpy()
    oc, _ = oracle.pack(fmt, W, None, n_cand=64)
    p = rq.rq_quantize_pack(to_dev(W), fmt)
    assert np.array_equal(p.codes.cpu().numpy().reshape(N, -1), oc.reshape(N, -1))


@pytest.mark.parametrize("fmt,bits", [("w5sb32", 5), ("w6sb32", 6)])
def test_dequant_exact_representable(fmt, bits):
    """Weights c (q - 2^(b-1)) 2^-12 with every code of [0, 2^b - 1] used and
    the largest c = 63 in every superblock are represented exactly, so the
    export returns W itself: the high-bit plane is read at every position."""
    rng = np.random.default_rng(29 + bits)
    L = (1 << bits) - 1
    N, K = 24, 1024
    q = rng.integers(0, L + 1, size=(N, K))
    qg = q.reshape(N, K // 32, 32)
    qg[:, :, 0], qg[:, :, 1] = 0, L
    c = rng.integers(1, 64, size=(N, K // 32))
    c.reshape(N, -1, 8)[:, :, 0] = 63
    W = (c.repeat(32, axis=1) * (q - (1 << (bits - 1))) * 2.0 ** -12).astype(np.float32)
    p = rq.rq_quantize_pack(to_dev(W), fmt)
    oc, _ = oracle.pack(fmt, W, None, n_cand=64)
    assert np.array_equal(p.codes.cpu().numpy().reshape(N, -1), oc.reshape(N, -1))
    assert np.array_equal(rq.rq_dequant(p).cpu().numpy(), W)


# -------------------------------------------------------------- product ----
WGEMM_CASES = [
    # K, N, M
    (2560, 2560, 1),       # 2.9B ffn.key width in, one decode row
    (2560, 300, 2),
    (256, 7, 3),
    (768, 33, 5),
    (4096, 129, 8),
    (2560, 257, 16),
    (10240, 130, 32),
    (512, 40, 64),
    (1024, 200, 100),
    (2560, 99, 128),
    (512, 20000, 16),      # more tiles than SMs
    (768, 200, 24),        # K split over a cluster
]


@pytest.mark.parametrize("fmt", WIDE)
@pytest.mark.parametrize("case", range(len(WGEMM_CASES)))
def test_wgemm_matches_oracle(fmt, case):
    K, N, M = WGEMM_CASES[case]
    W = wl.random_matrix(1300 + case, N, K).numpy()
    a = wl.random_act_sq(1400 + case, K, massive=2)
    oc, _ = oracle.pack(fmt, W, a, n_cand=8)
    p = upload(fmt, K, N, oc)
    x = wl.random_x(1500 + case, M, K, a)
    xb = wl.bf16_bits(x)
    y = rq.rq_wgemm(x.cuda(), p).cpu().numpy()
    check_y(y, oracle.wgemm(fmt, xb, K, N, oc, None), xb, oracle.dequant(fmt, K, N, oc, None), fmt)


@pytest.mark.parametrize("fmt,shapes,M", [
    ("w5sb32", [(2560, 10240), (2560, 65), (256, 3)], 1),
    ("w6sb32", [(2560, 200), (10240, 40), (512, 3)], 7),
    ("w5sb32", [(4096, 300), (1024, 1000)], 64),
])
def test_wgemm_batch_matches_oracle(fmt, shapes, M):
    xs, ws, ys, refs, bigs = [], [], [], [], []
    for i, (K, N) in enumerate(shapes):
        W = wl.random_matrix(1600 + i, N, K).numpy()
        oc, _ = oracle.pack(fmt, W, None, n_cand=4)
        x = wl.random_x(1700 + i, M, K)
        xb = wl.bf16_bits(x)
        big = torch.full((M * N + 512,), float("nan"), device="cuda")
        xs.append(x.cuda())
        ws.append(upload(fmt, K, N, oc))
        ys.append(big[256:256 + M * N].view(M, N))
        bigs.append((big, M * N))
        refs.append((oracle.wgemm(fmt, xb, K, N, oc, None), xb, oracle.dequant(fmt, K, N, oc, None)))
    rq.rq_wgemm_batch(xs, ws, ys)
    torch.cuda.synchronize()
    for y, (y_ref, xb, wd), (big, n) in zip(ys, refs, bigs):
        check_y(y.cpu().numpy(), y_ref, xb, wd, fmt)
        assert bool(torch.isnan(big[:256]).all()) and bool(torch.isnan(big[256 + n:]).all())


@pytest.mark.parametrize("fmt", WIDE)
def test_full_size_head_sampled(fmt):
    """The 2.9B head (2560 -> 65536, 5 bits in the COMPRESSION preset) at
    full size: sampled rows against the oracle, M = 1 and 16."""
    K, N = 2560, 65536
    W = wl.random_matrix(1800, N, K)
    a = wl.random_act_sq(1801, K, massive=8, energy=15631.0)
    p = rq.rq_quantize_pack(W.cuda(), fmt, to_dev(a), 64)
    rng = np.random.default_rng(1802)
    rows = np.sort(rng.choice(N, size=40, replace=False)).astype(np.int32)
    rows[-1] = N - 1
    oc, _ = oracle.pack(fmt, W.numpy()[rows], a, n_cand=64)
    assert np.array_equal(p.codes.cpu().numpy().reshape(N, -1)[rows], oc.reshape(len(rows), -1))
    for M in (1, 16):
        x = wl.random_x(1803 + M, M, K, a)
        xb = wl.bf16_bits(x)
        y = rq.rq_wgemm(x.cuda(), p).cpu().numpy()
        check_y(y[:, rows], oracle.wgemm(fmt, xb, K, len(rows), oc, None), xb,
                oracle.dequant(fmt, K, len(rows), oc, None), fmt)


# --------------------------------------- symmetric 6-bit g16 and int8 g64 ---
SYM_PACK_CASES = [
    # K, N, act recipe, n_cand, (t_lo, t_hi), outliers
    (64, 1, None, 1, (1.0, 1.0), False),
    (2048, 37, "eight", 64, (0.7, 1.0), False),
    (320, 9, "rand", 7, (0.5, 1.2), True),
    (4096, 5, "eight", 256, (0.7, 1.0), True),
]


@pytest.mark.parametrize("fmt", SYM)
@pytest.mark.parametrize("case", range(len(SYM_PACK_CASES)))
def test_sym_pack_matches_oracle(fmt, case):
    K, N, recipe, n, (lo, hi), out = SYM_PACK_CASES[case]
    W = weights_for(2100 + case, N, K, out)
    a = act_for(recipe, K, 2200 + case)
    oc, osc = oracle.pack(fmt, W, a, n_cand=n, t_lo=lo, t_hi=hi)
    p = rq.rq_quantize_pack(to_dev(W), fmt, to_dev(a), n, lo, hi)
    assert np.array_equal(p.codes.cpu().numpy().reshape(N, -1), oc.reshape(N, -1))
    assert np.array_equal(gpu_scales(p, K, N, fmt), osc)
    wd = rq.rq_dequant(p).cpu().numpy()
    assert np.array_equal(wd.view(np.uint32), oracle.dequant(fmt, K, N, oc, osc).view(np.uint32))


SYM_WGEMM_CASES = [
    # K, N, M
    (2048, 2048, 1),
    (2048, 300, 2),
    (320, 77, 3),
    (4096, 129, 8),
    (768, 200, 16),
    (2048, 64, 32),
    (1024, 40, 64),
    (512, 24, 128),
    (832, 130, 40),        # half stage at the end of K
    (256, 19500, 8),       # more tiles than SMs
    (8192, 40, 1),
]


@pytest.mark.parametrize("fmt", SYM)
@pytest.mark.parametrize("case", range(len(SYM_WGEMM_CASES)))
def test_sym_wgemm_matches_oracle(fmt, case):
    K, N, M = SYM_WGEMM_CASES[case]
    W = wl.random_matrix(2300 + case, N, K).numpy()
    a = wl.random_act_sq(2400 + case, K, massive=2)
    oc, osc = oracle.pack(fmt, W, a, n_cand=8)
    p = upload(fmt, K, N, oc, osc)
    x = wl.random_x(2500 + case, M, K, a)
    xb = wl.bf16_bits(x)
    y = rq.rq_wgemm(x.cuda(), p).cpu().numpy()
    check_y(y, oracle.wgemm(fmt, xb, K, N, oc, osc), xb, oracle.dequant(fmt, K, N, oc, osc), fmt)


@pytest.mark.parametrize("M", [1, 2])
def test_w8g64_exact_integer_products(M):
    """int8 g64 at M <= 2 (register path, exact fp32 w_hat): w = q 2^-10 with
    each group's absmax at 127 and small-integer x give exact sums."""
    rng = np.random.default_rng(41)
    K, N = 2048, 100
    q = rng.integers(-127, 128, size=(N, K))
    q.reshape(N, K // 64, 64)[:, :, 0] = 127
    W = (q * 2.0 ** -10).astype(np.float32)
    p = rq.rq_quantize_pack(to_dev(W), "w8g64", None, 1, 1.0, 1.0)
    xi = rng.integers(-8, 9, size=(M, K))
    x = torch.from_numpy(xi.astype(np.float32)).to(torch.bfloat16)
    y = rq.rq_wgemm(x.cuda(), p).cpu().numpy().astype(np.float64)
    assert np.array_equal(y, (xi @ q.T).astype(np.float64) * 2.0 ** -10)


@pytest.mark.parametrize("fmt,shapes,M", [
    ("w8g64", [(2048, 2048), (2048, 8192), (768, 5)], 1),
    ("w6g16", [(2048, 300), (4096, 129), (64, 7)], 2),
    ("w8g64", [(1024, 257), (448, 5)], 64),
])
def test_sym_wgemm_batch_matches_oracle(fmt, shapes, M):
    xs, ws, ys, refs = [], [], [], []
    for i, (K, N) in enumerate(shapes):
        W = wl.random_matrix(2600 + i, N, K).numpy()
        oc, osc = oracle.pack(fmt, W, None, n_cand=4)
        x = wl.random_x(2700 + i, M, K)
        xb = wl.bf16_bits(x)
        xs.append(x.cuda())
        ws.append(upload(fmt, K, N, oc, osc))
        ys.append(torch.empty(M, N, device="cuda"))
        refs.append((oracle.wgemm(fmt, xb, K, N, oc, osc), xb, oracle.dequant(fmt, K, N, oc, osc)))
    rq.rq_wgemm_batch(xs, ws, ys)
    torch.cuda.synchronize()
    for y, (y_ref, xb, wd) in zip(ys, refs):
        check_y(y.cpu().numpy(), y_ref, xb, wd, fmt)
