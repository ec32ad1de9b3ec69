"""The on-device E[x^2] statistic (rq_act_sumsq / rq_act_finalize) against
the oracle, which sums each channel's squares one row at a time in ascending
row order (the statistic's definition: rwkv-quant article, "Two presets and
six sizes", the mean of x_k^2 over the calibration rows).

The device adds the same exact fp64 squares in another fixed order, so the
sums may differ by fp64 rounding only. Bound (derived from the arithmetic):
any order of n additions of non-negative terms is within (n - 1) 2^-53 of
the exact sum relative to it, so the two sides are within 2 (R + 1) 2^-53 of
each other. Where every partial sum is exact (constant rows, small integers,
small multiples of a power of two) they must agree bit for bit, and so must
E[x^2] and the codes packed from it.
"""
import numpy as np
import pytest
import torch

import oracle
import weight_only_quantized_rq_b200 as rq
from weight_only_quantized_rq_b200 import workloads as wl

pytestmark = pytest.mark.gpu

U53 = 2.0 ** -53


@pytest.fixture(scope="module", autouse=True)
def _setup():
    from weight_only_quantized_rq_b200 import build
    build.build()
    oracle.build()
    torch.cuda.set_device(0)
    yield
    assert rq.rq_device_status() == 0


def calib(seed, R, K, massive=None):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(R, K, generator=g)
    if massive is not None:
        x[:, massive] *= 50.0
    return x.to(torch.bfloat16)


def calib_exact(seed, R, K, massive=None):
    """Rows of small multiples of 2^-3 (|x| < 32, at most 8 significant bits,
    so exact in bf16); every partial sum of their squares is a multiple of
    2^-6 below 2^53 * 2^-6, hence exact in fp64 in any order."""
    rng = np.random.default_rng(seed)
    x = rng.integers(-255, 256, size=(R, K)).astype(np.float32) / 8.0
    if massive is not None:
        x[:, massive] *= 32.0
    return torch.from_numpy(x).to(torch.bfloat16)


def check_sums(s_dev, s_ref, rows):
    tol = 2.0 * (rows + 1) * U53
    err = np.abs(s_dev - s_ref)
    assert np.all(err <= tol * np.abs(s_ref)), float(np.max(err / np.maximum(np.abs(s_ref), 1e-300)))
    return float(np.max(err / np.maximum(np.abs(s_ref), 1e-300)))


def check_act(a_dev, a_ref):
    """fp32(sum / rows) of two sums that differ by fp64 rounding: at most one
    fp32 unit in the last place apart."""
    ulp = np.spacing(np.abs(a_ref).astype(np.float32))
    assert np.all(np.abs(a_dev.astype(np.float64) - a_ref.astype(np.float64)) <= ulp)


@pytest.mark.parametrize("R,K", [(1, 5), (7, 64), (8, 130), (9, 65), (31, 72), (33, 4095), (1000, 2048),
                                 (4097, 768), (5000, 4096), (3, 20000), (70000, 64)])
def test_sumsq_and_finalize_within_rounding(R, K):
    x = calib(100 + R + K, R, K, massive=min(5, K - 1))
    xb = wl.bf16_bits(x)
    s = rq.rq_act_sumsq(x.cuda())
    a = rq.rq_act_finalize(s, R)
    torch.cuda.synchronize()
    s_ref = oracle.act_sumsq(xb)
    check_sums(s.cpu().numpy(), s_ref, R)
    check_act(a.cpu().numpy(), oracle.act_finalize(s_ref, R))
    # the device order is fixed: a second call gives the same bits
    s2 = rq.rq_act_sumsq(x.cuda())
    assert np.array_equal(s2.cpu().numpy().view(np.uint64), s.cpu().numpy().view(np.uint64))


@pytest.mark.parametrize("R,K", [(1, 8), (64, 64), (777, 136), (4096, 2048), (9, 67)])
def test_sumsq_exact_when_partial_sums_are_exact(R, K):
    x = calib_exact(300 + R + K, R, K, massive=min(7, K - 1))
    s = rq.rq_act_sumsq(x.cuda())
    a = rq.rq_act_finalize(s, R)
    torch.cuda.synchronize()
    s_ref = oracle.act_sumsq(wl.bf16_bits(x))
    assert np.array_equal(s.cpu().numpy().view(np.uint64), s_ref.view(np.uint64))
    assert np.array_equal(a.cpu().numpy().view(np.uint32), oracle.act_finalize(s_ref, R).view(np.uint32))


def test_constant_rows_give_the_exact_square():
    R, K = 1000, 24
    c = np.linspace(-3.0, 3.0, K).astype(np.float32)
    x = torch.from_numpy(np.tile(c, (R, 1))).to(torch.bfloat16)
    cb = x[0].float().numpy().astype(np.float64)
    a = rq.rq_act_finalize(rq.rq_act_sumsq(x.cuda()), R)
    assert np.array_equal(a.cpu().numpy(), (cb ** 2).astype(np.float32))


def test_sumsq_accumulates_batches():
    K = 2048
    batches = [calib(7 + i, R, K, massive=1202) for i, R in enumerate((300, 1, 4096))]
    s = None
    s_ref = None
    for x in batches:
        s = rq.rq_act_sumsq(x.cuda(), s)
        s_ref = oracle.act_sumsq(wl.bf16_bits(x), s_ref)
    rows = sum(x.shape[0] for x in batches)
    a = rq.rq_act_finalize(s, rows)
    torch.cuda.synchronize()
    check_sums(s.cpu().numpy(), s_ref, rows)
    check_act(a.cpu().numpy(), oracle.act_finalize(s_ref, rows))


def test_guard_band_and_padding():
    """Only sum_sq[0:K] is touched."""
    R, K = 100, 70
    x = calib(9, R, K).cuda()
    big = torch.full((K + 64,), 7.0, dtype=torch.float64, device="cuda")
    s = big[32:32 + K]
    s.zero_()
    rq.rq_act_sumsq(x, s)
    torch.cuda.synchronize()
    assert bool((big[:32] == 7.0).all()) and bool((big[32 + K:] == 7.0).all())


@pytest.mark.parametrize("fmt", ["w4g64", "w8g16", "w4sb32", "w5sb32", "w6sb32", "w8g64", "w6g16"])
def test_calibrate_then_pack_matches_oracle_chain(fmt):
    """Device statistic -> device pack gives the codes of oracle statistic ->
    oracle pack: the whole calibration path stays on the GPU. The rows are
    small multiples of 2^-3 (with a massive channel), so both statistics are
    exact and the packs must agree byte for byte."""
    sb = fmt.endswith("sb32")
    K, N, R = 2560 if sb else 2048, 48, 512
    x = calib_exact(11, R, K, massive=517 if sb else 1202)
    W = wl.random_matrix(12, N, K)
    a_dev = rq.rq_act_finalize(rq.rq_act_sumsq(x.cuda()), R)
    p = rq.rq_quantize_pack(W.cuda(), fmt, a_dev, 64)
    a_ref = oracle.act_finalize(oracle.act_sumsq(wl.bf16_bits(x)), R)
    oc, osc = oracle.pack(fmt, W.numpy(), a_ref, n_cand=64)
    assert np.array_equal(a_dev.cpu().numpy(), a_ref)
    assert np.array_equal(p.codes.cpu().numpy().reshape(N, -1), oc.reshape(N, -1))
    if osc is not None:
        used = N * (K // oracle.GROUP[fmt]) * 2
        assert np.array_equal(p.scales.cpu().numpy()[:used].view(np.uint16).reshape(N, -1), osc)
