"""GPTQ on the preset's grid (rwkv-quant article, "Calibration leakage and
honest measurements"; RWKV-7 G1 1.5B int4 model card: symmetric int4 group
64, GPTQ-calibrated) on the GPU against the CPU oracle.

- The Hessian is bit-identical (exact fp64 products summed in ascending rows).
- The factor U is compared with the oracle's (numpy's LAPACK steps) to a
  relative 1e-8: the two use different summation orders.
- Given the oracle's U, the column loop's codes and scales are byte-identical
  (the same fp64 operations in the same order).
- The whole device chain (Hessian -> U -> codes) against the whole oracle
  chain may differ only where an fp64 difference in U moves a weight across a
  rounding boundary: at most 0.1 % of the values (1 % for the superblock
  formats, whose header covers 256 values), and the output error
  tr((W - W_hat) H (W - W_hat)^T) within 1 %.
"""
import numpy as np
import pytest
import torch

import oracle
import weight_only_quantized_rq_b200 as rq
from weight_only_quantized_rq_b200 import workloads as wl

pytestmark = pytest.mark.gpu

SYM = ("w4g64", "w8g16", "w8g64", "w6g16")
# GPTQ into the superblock formats follows the same tests below


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


def calib_x(seed, R, K, rank=None):
    """Correlated bf16 calibration rows: a low-rank mix plus noise."""
    rng = np.random.default_rng(seed)
    r = rank or max(4, K // 8)
    x = rng.standard_normal((R, r)) @ rng.standard_normal((r, K)) + 0.1 * rng.standard_normal((R, K))
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)


def scales_of(p, fmt, K, N):
    used = N * (K // oracle.GROUP[fmt]) * 2
    raw = p.scales.cpu().numpy()
    assert not raw[used:].any()
    return raw[:used].view(np.uint16).reshape(N, -1)


@pytest.mark.parametrize("R,K", [(1, 64), (300, 200), (517, 320), (64, 1)])
def test_hessian_bit_exact(R, K):
    x = calib_x(81 + R, R, K)
    xb = wl.bf16_bits(x)
    H = rq.rq_hessian_accum(x.cuda())
    H = rq.rq_hessian_accum(x.cuda(), H)                       # a second batch accumulates
    ref = oracle.hessian_accum(xb, oracle.hessian_accum(xb))
    assert np.array_equal(H.cpu().numpy(), ref)


@pytest.mark.parametrize("K,dead_ch", [(64, None), (256, 17), (333, 0), (1024, 1023)])
def test_prepare_matches_oracle(K, dead_ch):
    x = calib_x(90 + K, 4 * K, K)
    if dead_ch is not None:
        x[:, dead_ch] = 0
    Hd = rq.rq_hessian_accum(x.cuda())
    U, dead = rq.rq_gptq_prepare(Hd, 0.01)
    Ur, deadr = oracle.gptq_prepare(oracle.hessian_accum(wl.bf16_bits(x)), 0.01)
    Ug = U.cpu().numpy()
    assert np.array_equal(dead.cpu().numpy(), deadr)
    assert np.count_nonzero(np.tril(Ug, -1)) == 0
    assert np.all(np.isfinite(Ug))
    assert np.max(np.abs(Ug - Ur)) <= 1e-8 * np.max(np.abs(Ur))


def test_prepare_flags_a_non_positive_pivot():
    """-I with no damping has no Cholesky factor: the device status word
    gets the pivot bit (no fault, NaNs in U)."""
    K = 64
    H = -torch.eye(K, dtype=torch.float64, device="cuda")
    rq.rq_gptq_prepare(H, 0.0)
    word = rq.rq_device_status()
    assert word == 32


@pytest.mark.parametrize("fmt", SYM)
@pytest.mark.parametrize("K,N,act", [(256, 37, False), (1024, 9, True), (128, 300, True)])
def test_gptq_pack_bit_exact_given_U(fmt, K, N, act):
    x = calib_x(100 + K + N, 3 * K, K)
    x[:, 5] = 0                                                # a dead channel
    H = oracle.hessian_accum(wl.bf16_bits(x))
    U, dead = oracle.gptq_prepare(H, 0.01)
    a = (np.diag(H) / (3 * K)).astype(np.float32) + np.float32(1e-3) if act else None
    W = wl.random_matrix(110 + K, N, K).numpy()
    oc, osc = oracle.gptq_pack(fmt, W, U, dead, a, n_cand=32)
    p = rq.rq_gptq_quantize_pack(to_dev(W), fmt, to_dev(U), to_dev(dead), to_dev(a), 32)
    assert np.array_equal(p.codes.cpu().numpy().reshape(N, -1), oc.reshape(N, -1))
    assert np.array_equal(scales_of(p, fmt, K, N), osc)


@pytest.mark.parametrize("fmt", ["w4sb32", "w5sb32", "w6sb32"])
@pytest.mark.parametrize("K,N,act", [(512, 21, True), (1024, 5, False)])
def test_gptq_sb_pack_bit_exact_given_U(fmt, K, N, act):
    """Superblock formats: headers, low nibbles and high-bit planes."""
    x = calib_x(140 + K + N, 3 * K, K)
    x[:, 300] = 0
    H = oracle.hessian_accum(wl.bf16_bits(x))
    U, dead = oracle.gptq_prepare(H, 0.01)
    a = (np.diag(H) / (3 * K)).astype(np.float32) + np.float32(1e-3) if act else None
    W = wl.random_matrix(150 + K, N, K).numpy()
    oc, _ = oracle.gptq_pack(fmt, W, U, dead, a, n_cand=32)
    p = rq.rq_gptq_quantize_pack(to_dev(W), fmt, to_dev(U), to_dev(dead), to_dev(a), 32)
    assert p.scales is None
    assert np.array_equal(p.codes.cpu().numpy().reshape(N, -1), oc.reshape(N, -1))


@pytest.mark.parametrize("fmt", ["w4g64", "w8g16", "w4sb32"])
def test_gptq_device_chain(fmt):
    K, N, R = 512, 64, 2048
    x = calib_x(120, R, K)
    H = rq.rq_hessian_accum(x.cuda())
    U, dead = rq.rq_gptq_prepare(H)
    a = rq.rq_act_finalize(rq.rq_act_sumsq(x.cuda()), R)
    W = wl.random_matrix(121, N, K)
    p = rq.rq_gptq_quantize_pack(W.cuda(), fmt, U, dead, a, 64)
    Hn = oracle.hessian_accum(wl.bf16_bits(x))
    Ur, deadr = oracle.gptq_prepare(Hn)
    ar = oracle.act_finalize(oracle.act_sumsq(wl.bf16_bits(x)), R)
    oc, osc = oracle.gptq_pack(fmt, W.numpy(), Ur, deadr, ar, n_cand=64)
    Wg = rq.rq_dequant(p).cpu().numpy().astype(np.float64)
    Wo = oracle.dequant(fmt, K, N, oc, osc).astype(np.float64)
    mism = np.count_nonzero(Wg != Wo)
    # a flipped superblock header changes up to 256 values at once
    assert mism <= (1e-2 if fmt.endswith("sb32") else 1e-3) * N * K, mism
    def out_err(Wh):
        D = W.numpy().astype(np.float64) - Wh
        return float(np.einsum("nk,kl,nl->", D, Hn, D))
    assert abs(out_err(Wg) - out_err(Wo)) <= 0.01 * out_err(Wo)


def test_gptq_full_width_sampled_rows():
    """The 1.5B o_proj width (2048 -> 2048) at full size on the GPU; sampled
    rows against the oracle given the same U."""
    K, N, R = 2048, 2048, 4096
    x = calib_x(130, R, K, rank=256)
    Hn = oracle.hessian_accum(wl.bf16_bits(x))
    Ur, deadr = oracle.gptq_prepare(Hn)
    W = wl.random_matrix(131, N, K)
    p = rq.rq_gptq_quantize_pack(W.cuda(), "w4g64", to_dev(Ur), to_dev(deadr), None, 64)
    rows = np.sort(np.random.default_rng(132).choice(N, 24, replace=False))
    rows[-1] = N - 1
    oc, osc = oracle.gptq_pack("w4g64", W.numpy()[rows], Ur, deadr, None, n_cand=64)
    assert np.array_equal(p.codes.cpu().numpy().reshape(N, -1)[rows], oc.reshape(len(rows), -1))
    assert np.array_equal(scales_of(p, "w4g64", K, N)[rows], osc)
