"""Bounded device waits run out without a fault and leave the context usable.

The testing hook rq_test_hooks(wait_ns, 1) makes the threads that issue the
weight copies issue none, so every wait for a copy runs out after wait_ns
(1 ms here). Each kernel path must then finish on its own, report
RQ_ERR_DEVICE_TIMEOUT through the device status word (no trap, no fault),
and the next ordinary call on the same stream must give correct results.
Nothing here faults or hangs a GPU: the waits are bounded and nothing is left
in flight when a CTA gives up.
"""
import numpy as np
import pytest
import torch

import headroom
import oracle
import weight_only_quantized_rq_b200 as rq
from weight_only_quantized_rq_b200 import workloads as wl

pytestmark = pytest.mark.gpu

WAIT_BITS = 0x1F          # copy, slot, commit, TMEM and staged-x waits


@pytest.fixture(scope="module", autouse=True)
def _setup():
    from weight_only_quantized_rq_b200 import build
    build.build()
    oracle.build()
    torch.cuda.set_device(0)
    yield
    rq.rq_test_hooks(0, 0)
    assert rq.rq_device_status() == 0


@pytest.mark.parametrize("fmt,M,K,kernel", [
    ("w4g64", 1, 1024, "register GEMV"),
    ("w4g64", 1, 8192, "register GEMV with rows split over k-slice warps"),
    ("w8g16", 2, 4096, "register GEMV with rows split over k-slice warps"),
    ("w4g64", 8, 1024, "tensor-core kernel"),
    ("w8g16", 8, 1024, "tensor-core kernel"),
    ("w5sb32", 1, 1024, "tensor-core kernel"),
    ("w4g64", 64, 1024, "tensor-core kernel"),
])
def test_waits_run_out_then_the_next_call_is_correct(fmt, M, K, kernel):
    N = 700
    W = wl.random_matrix(3700, N, K).numpy()
    oc, osc = oracle.pack(fmt, W, None, n_cand=1, t_lo=1.0, t_hi=1.0)
    p = rq.alloc_packed(fmt, K, N)
    p.codes.copy_(torch.from_numpy(np.ascontiguousarray(oc).reshape(-1)))
    if p.scales is not None:
        p.scales.zero_()
        raw = np.ascontiguousarray(osc).view(np.uint8).reshape(-1)
        p.scales[: raw.size].copy_(torch.from_numpy(raw))
    x = wl.random_x(3701, M, K)
    xb = wl.bf16_bits(x)
    xd = x.cuda()
    assert rq.rq_device_status() == 0
    try:
        rq.rq_test_hooks(1_000_000, 1)                 # 1 ms, no copies
        rq.rq_wgemm(xd, p)
        word = rq.rq_device_status()                   # synchronizes; the call has finished
    finally:
        rq.rq_test_hooks(0, 0)
    assert word & WAIT_BITS, f"{kernel}: no wait gave up (status {word})"
    assert rq.rq_device_status() == 0                  # the read above cleared the word
    y = rq.rq_wgemm(xd, p).cpu().numpy()
    headroom.check_y(y, oracle.wgemm(fmt, xb, K, N, oc, osc), xb, oracle.dequant(fmt, K, N, oc, osc), fmt)
    assert rq.rq_device_status() == 0


def test_hook_rejects_bad_values():
    for args in ((-1, 0), (61_000_000_000, 0), (0, 2)):
        with pytest.raises(rq.RqError):
            rq.rq_test_hooks(*args)
