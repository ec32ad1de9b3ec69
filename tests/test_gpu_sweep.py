"""Every activation-row count and exact products on every kernel path.

- Every M in 1..128 on one small, ragged shape per format against the
  oracle (each M sets the tensor-core kernel's padded N, the x rows copied,
  the number of MMA-issuing warps and accumulators and the x box; the
  register GEMV covers M <= 2).
- Exact integer products: weights q * 2^-e whose every product with small
  integer activations, and every partial sum, is exact, so the fp32 outputs
  must equal the integer result exactly on every path (the RWKV-7 G1 1.5B
  int4 model card's "bit-identical to the offline dequantization" holds there
  in the strongest form). For the 5- and 6-bit superblock formats the records
  are written by hand from the format's definition (power-of-two group scales
  and a min of exactly half the code range, so every w_hat has at most six
  significant bits) and decoded by the oracle to check the encoding.
"""
import numpy as np
import pytest
import torch

import headroom
import oracle
import weight_only_quantized_rq_b200 as rq
from weight_only_quantized_rq_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ALL = ("w4g64", "w8g16", "w8g64", "w6g16", "w4sb32", "w5sb32", "w6sb32")


@pytest.fixture(scope="module", autouse=True)
def _setup():
    from weight_only_quantized_rq_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    yield
    assert rq.rq_device_status() == 0


def upload(fmt, K, N, codes, scales=None):
    p = rq.alloc_packed(fmt, K, N)
    p.codes.copy_(torch.from_numpy(np.ascontiguousarray(codes).reshape(-1)))
    if p.scales is not None:
        p.scales.zero_()
        raw = np.ascontiguousarray(scales).view(np.uint8).reshape(-1)
        p.scales[: raw.size].copy_(torch.from_numpy(raw))
    return p


@pytest.mark.parametrize("fmt", ALL)
def test_every_m_from_1_to_128(fmt):
    K = 512 if fmt.endswith("sb32") else 448          # 448: a half stage at the end of K
    N = 200                                           # two tiles, the second ragged
    W = wl.random_matrix(3100 + ALL.index(fmt), N, K).numpy()
    a = wl.random_act_sq(3200, K, massive=2)
    oc, osc = oracle.pack(fmt, W, a, n_cand=4)
    p = upload(fmt, K, N, oc, osc)
    x = wl.random_x(3300, 128, K, a)
    xb = wl.bf16_bits(x)
    y_ref = oracle.wgemm(fmt, xb, K, N, oc, osc)      # row m of y depends on row m of x only
    w_hat = oracle.dequant(fmt, K, N, oc, osc)
    xd = x.cuda()
    for M in range(1, 129):
        y = rq.rq_wgemm(xd[:M], p).cpu().numpy()
        headroom.check_y(y, y_ref[:M], xb[:M], w_hat, fmt)


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 13, 16, 17, 24, 31, 32, 33, 64, 100, 128])
def test_w4g64_exact_integer_products_every_path(M):
    rng = np.random.default_rng(3400 + M)
    K, N, unit = 1088, 150, 2.0 ** -6                 # 1088: 4.25 stages of 256
    q = rng.integers(-7, 8, size=(N, K))
    q.reshape(N, K // 64, 64)[:, :, 0] = 7
    W = (q * unit).astype(np.float32)
    p = rq.rq_quantize_pack(torch.from_numpy(W).cuda(), "w4g64", None, 1, 1.0, 1.0)
    xi = rng.integers(-8, 9, size=(M, K))
    x = torch.from_numpy(xi.astype(np.float32)).to(torch.bfloat16)
    y = rq.rq_wgemm(x.cuda(), p).cpu().numpy().astype(np.float64)
    assert np.array_equal(y, (xi @ q.T).astype(np.float64) * unit)


@pytest.mark.parametrize("M", [1, 2, 7, 16])
def test_w6g16_exact_integer_products(M):
    rng = np.random.default_rng(3500 + M)
    K, N, unit = 1024, 90, 2.0 ** -8
    q = rng.integers(-31, 32, size=(N, K))
    q.reshape(N, K // 16, 16)[:, :, 3] = -31          # |q| = 31 in every group: scale = unit exactly
    W = (q * unit).astype(np.float32)
    p = rq.rq_quantize_pack(torch.from_numpy(W).cuda(), "w6g16", None, 1, 1.0, 1.0)
    assert np.array_equal(rq.rq_dequant(p).cpu().numpy(), W)
    xi = rng.integers(-8, 9, size=(M, K))
    x = torch.from_numpy(xi.astype(np.float32)).to(torch.bfloat16)
    y = rq.rq_wgemm(x.cuda(), p).cpu().numpy().astype(np.float64)
    assert np.array_equal(y, (xi @ q.T).astype(np.float64) * unit)


def sb_records(bits, d_exp, sc, q):
    """Superblock records (the format's byte layout) for fp16 d = 2^d_exp,
    dmin = 2^(bits - 1) d, 6-bit sc_j = m_j = sc[n, blk, j] and codes q
    [N][K]: w_hat = d sc_j (q - 2^(bits - 1))."""
    N, K = q.shape
    rec = {4: 144, 5: 176, 6: 208}[bits]
    out = np.zeros((N, K // 256, rec), np.uint8)
    d = np.float16(2.0 ** d_exp)
    dmin = np.float16(2.0 ** (d_exp + bits - 1))
    for n in range(N):
        for b in range(K // 256):
            r = out[n, b]
            r[0:2] = np.frombuffer(d.tobytes(), np.uint8)
            r[2:4] = np.frombuffer(dmin.tobytes(), np.uint8)
            bitstr = 0
            for j in range(8):
                bitstr |= int(sc[n, b, j]) << (6 * j)
                bitstr |= int(sc[n, b, j]) << (48 + 6 * j)
            r[4:16] = np.frombuffer(bitstr.to_bytes(12, "little"), np.uint8)
            qq = q[n, 256 * b:256 * (b + 1)]
            lo = qq & 15
            r[16:144] = (lo[0::2] | (lo[1::2] << 4)).astype(np.uint8)
            up = qq >> 4
            if bits == 5:
                r[144:176] = np.packbits(up.astype(np.uint8), bitorder="little")
            elif bits == 6:
                r[144:208] = (up[0::4] | (up[1::4] << 2) | (up[2::4] << 4) | (up[3::4] << 6)).astype(np.uint8)
    return out


@pytest.mark.parametrize("fmt,bits", [("w4sb32", 4), ("w5sb32", 5), ("w6sb32", 6)])
@pytest.mark.parametrize("M", [1, 2, 5, 16, 40])
def test_superblock_exact_integer_products(fmt, bits, M):
    rng = np.random.default_rng(3600 + bits * 7 + M)
    K, N, h = 768, 70, 1 << (bits - 1)
    q = rng.integers(0, 1 << bits, size=(N, K))
    sc = (1 << rng.integers(0, 6, size=(N, K // 256, 8))).astype(np.int64)   # 1 .. 32
    codes = sb_records(bits, -12, sc, q)
    S = sc.reshape(N, -1).repeat(32, axis=1).astype(np.float64) * 2.0 ** -12
    want_w = S * (q - h)
    assert np.array_equal(oracle.dequant(fmt, K, N, codes, None).astype(np.float64), want_w)
    p = upload(fmt, K, N, codes)
    assert np.array_equal(rq.rq_dequant(p).cpu().numpy().astype(np.float64), want_w)
    xi = rng.integers(-8, 9, size=(M, K))
    x = torch.from_numpy(xi.astype(np.float32)).to(torch.bfloat16)
    y = rq.rq_wgemm(x.cuda(), p).cpu().numpy().astype(np.float64)
    want = (xi[:, None, :] * (sc.reshape(N, -1).repeat(32, axis=1) * (q - h))[None]).sum(-1) * 2.0 ** -12
    assert np.array_equal(y, want)
