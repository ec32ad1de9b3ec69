"""The on-device E[x^2] statistic (rq_act_sumsq / rq_act_finalize) against
the oracle: bit-identical fp64 running sums and fp32 E[x^2] (both sides sum
in the same fixed order: 64 contiguous row chunks, rows ascending within a
chunk, chunks ascending; squares of bf16 values are exact in fp64), batch
accumulation, and the calibrate-then-pack chain producing the same codes as
the oracle's chain."""
import numpy as np
import pytest
import torch

import oracle
import weight_only_quantized_rq_b200 as rq
from weight_only_quantized_rq_b200 import workloads as wl

pytestmark = pytest.mark.gpu


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


@pytest.mark.parametrize("R,K", [(1, 5), (7, 64), (8, 130), (9, 65), (1000, 2048), (4097, 768), (33, 4095),
                                 (5000, 4096), (3, 20000)])
def test_sumsq_and_finalize_bit_identical(R, K):
    x = calib(100 + R + K, R, K, massive=min(5, K - 1))
    xb = wl.bf16_bits(x)
    s = rq.rq_act_sumsq(x.cuda())
    a = rq.rq_act_finalize(s, R)
    torch.cuda.synchronize()
    s_ref = oracle.act_sumsq(xb)
    assert np.array_equal(s.cpu().numpy().view(np.uint64), s_ref.view(np.uint64))
    assert np.array_equal(a.cpu().numpy().view(np.uint32), oracle.act_finalize(s_ref, R).view(np.uint32))


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
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(a.cpu().numpy(), oracle.act_finalize(s_ref, rows))


def test_guard_band_and_padding():
    """Only sum_sq[0:K] is touched; rows of a strided x are not needed."""
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
    oracle pack: the whole calibration path stays on the GPU."""
    sb = fmt.endswith("sb32")
    K, N, R = 2560 if sb else 2048, 48, 512
    x = calib(11, R, K, massive=517 if sb else 1202)
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
