"""The C ABI without a GPU: librq.so loads, exports every function that
include/rq.h declares, reports the packed sizes the header defines, and
rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

import weight_only_quantized_rq_b200 as rq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from weight_only_quantized_rq_b200 import build
    build.build()
    return rq.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "rq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(rq_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 8, names
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/rq.h but not exported"
    assert set(rq.EXPORTS) <= set(names)


def test_version_and_status_strings(L):
    assert rq.rq_version() >= 100
    for s in range(7):
        assert rq.rq_status_string(s)
    assert rq.rq_status_string(99) == "unknown status"
    assert rq.rq_status_string(0) == "ok"


@pytest.mark.parametrize("fmt,K,N,codes,scales", [
    ("w4g64", 2048, 2048, 2048 * 1024, 2048 * 32 * 2),
    ("w8g16", 2048, 2048, 2048 * 2048, 2048 * 128 * 2),
    ("w4sb32", 2560, 2560, 2560 * 10 * 144, 0),
    ("w5sb32", 2560, 2560, 2560 * 10 * 176, 0),
    ("w6sb32", 256, 3, 3 * 208, 0),
    ("w8g64", 2048, 5, 5 * 2048, 5 * 32 * 2),
    ("w6g16", 320, 3, 3 * 5 * 48, 128),     # 3 rows x 20 scales x 2 B = 120, padded to 128
    ("w4g64", 768, 3, 3 * 384, 80),        # 3 rows x 12 scales x 2 B = 72, padded to 80
])
def test_packed_size(L, fmt, K, N, codes, scales):
    cb, sb = rq.rq_packed_size(fmt, K, N)
    assert cb == codes
    G = {"w4g64": 64, "w8g64": 64, "w8g16": 16, "w6g16": 16}.get(fmt)
    raw = N * (K // G) * 2 if G else 0
    assert sb == (raw + 15) // 16 * 16
    assert sb == scales


def test_bits_per_weight(L):
    K = N = 4096
    for fmt, bpw in [("w4g64", 4.25), ("w8g16", 9.0), ("w4sb32", 4.5), ("w5sb32", 5.5), ("w6sb32", 6.5),
                     ("w8g64", 8.25), ("w6g16", 7.0)]:
        cb, sb = rq.rq_packed_size(fmt, K, N)
        assert (cb + sb) * 8 / (K * N) == bpw


@pytest.mark.parametrize("fmt,K,N", [("w4g64", 96, 4), ("w4sb32", 320, 4), ("w8g16", 65536, 4),
                                     ("w5sb32", 320, 4), ("w6sb32", 64, 4), ("w4g64", 2048, 0),
                                     ("w8g64", 96, 4), ("w6g16", 32, 4),
                                     ("w4g64", 32, 1), (8, 2048, 2), (0, 2048, 2)])
def test_packed_size_rejects(L, fmt, K, N):
    f = rq.fmt_id(fmt)
    assert L.rq_packed_size(f, K, N, None, None) == 0


def _desc(fmt, K, N, codes=0x10000, scales=0x20000, reserved=0):
    return rq.RqPacked(rq.fmt_id(fmt), K, N, reserved, codes, scales)


A = ctypes.c_void_p(0x40000)     # aligned fake device address (never dereferenced)
U = ctypes.c_void_p(0x40008)     # misaligned


def test_wgemm_validation(L):
    d = _desc("w4g64", 2048, 256)
    st = ctypes.c_void_p(0)
    assert L.rq_wgemm(None, 1, 2048, 256, ctypes.byref(d), A, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_wgemm(A, 0, 2048, 256, ctypes.byref(d), A, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_wgemm(A, 129, 2048, 256, ctypes.byref(d), A, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_wgemm(A, 1, 1024, 256, ctypes.byref(d), A, st) == rq.RQ_ERR_FORMAT_MISMATCH
    assert L.rq_wgemm(A, 1, 2048, 255, ctypes.byref(d), A, st) == rq.RQ_ERR_FORMAT_MISMATCH
    assert L.rq_wgemm(U, 1, 2048, 256, ctypes.byref(d), A, st) == rq.RQ_ERR_MISALIGNED
    assert L.rq_wgemm(A, 1, 2048, 256, ctypes.byref(d), U, st) == rq.RQ_ERR_MISALIGNED
    bad = _desc("w4g64", 2048, 256, codes=0x10004)
    assert L.rq_wgemm(A, 1, 2048, 256, ctypes.byref(bad), A, st) == rq.RQ_ERR_MISALIGNED
    nos = _desc("w4g64", 2048, 256, scales=0)
    assert L.rq_wgemm(A, 1, 2048, 256, ctypes.byref(nos), A, st) == rq.RQ_ERR_INVALID_ARG
    for f in ("w4sb32", "w5sb32", "w6sb32"):   # superblock formats carry no scales plane
        sb = _desc(f, 2048, 256)
        assert L.rq_wgemm(A, 1, 2048, 256, ctypes.byref(sb), A, st) == rq.RQ_ERR_FORMAT_MISMATCH
    res = _desc("w4g64", 2048, 256, reserved=1)
    assert L.rq_wgemm(A, 1, 2048, 256, ctypes.byref(res), A, st) == rq.RQ_ERR_FORMAT_MISMATCH
    odd = _desc("w4g64", 2080, 256)
    assert L.rq_wgemm(A, 1, 2080, 256, ctypes.byref(odd), A, st) == rq.RQ_ERR_UNSUPPORTED_SHAPE
    assert L.rq_wgemm(A, 1, 2048, 256, None, A, st) == rq.RQ_ERR_INVALID_ARG


def test_quantize_pack_validation(L):
    d = _desc("w8g16", 2048, 64)
    st = ctypes.c_void_p(0)
    S = rq.RqSearch
    assert L.rq_quantize_pack(None, 2048, 64, None, None, ctypes.byref(d), st) == rq.RQ_ERR_INVALID_ARG
    for bad in [S(0, 0.7, 1.0), S(257, 0.7, 1.0), S(64, 0.0, 1.0), S(64, 0.9, 0.8), S(64, 0.7, 5.0),
                S(64, float("nan"), 1.0)]:
        assert L.rq_quantize_pack(A, 2048, 64, None, ctypes.byref(bad), ctypes.byref(d), st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_quantize_pack(U, 2048, 64, None, None, ctypes.byref(d), st) == rq.RQ_ERR_MISALIGNED
    assert L.rq_quantize_pack(A, 2048, 64, U, None, ctypes.byref(d), st) == rq.RQ_ERR_MISALIGNED
    assert L.rq_quantize_pack(A, 4096, 64, None, None, ctypes.byref(d), st) == rq.RQ_ERR_FORMAT_MISMATCH


def test_gptq_validation(L):
    st = ctypes.c_void_p(0)
    B = ctypes.c_void_p(0x80000)        # a second aligned fake device address
    assert L.rq_hessian_accum(None, 8, 64, A, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_hessian_accum(A, 0, 64, B, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_hessian_accum(A, 8, 32769, B, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_hessian_accum(U, 8, 64, B, st) == rq.RQ_ERR_MISALIGNED
    assert L.rq_gptq_prepare(A, 64, 0.01, None, B, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_gptq_prepare(A, 16385, 0.01, B, B, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_gptq_prepare(A, 64, -1.0, B, B, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_gptq_prepare(A, 64, float("nan"), B, B, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_gptq_prepare(A, 64, 0.01, A, B, st) == rq.RQ_ERR_INVALID_ARG       # U overlaps H
    assert L.rq_gptq_prepare(U, 64, 0.01, B, B, st) == rq.RQ_ERR_MISALIGNED
    d = _desc("w4g64", 2048, 64)
    assert L.rq_gptq_quantize_pack(A, 2048, 64, None, B, None, None, ctypes.byref(d), st) == rq.RQ_ERR_INVALID_ARG
    sb = _desc("w4sb32", 2048, 64)                          # superblock descriptor with a scales plane
    assert L.rq_gptq_quantize_pack(A, 2048, 64, B, B, None, None, ctypes.byref(sb), st) == rq.RQ_ERR_FORMAT_MISMATCH
    assert L.rq_gptq_quantize_pack(A, 2048, 64, B, B, U, None, ctypes.byref(d), st) == rq.RQ_ERR_MISALIGNED
    wide = _desc("w4g64", 32768, 4)
    assert L.rq_gptq_quantize_pack(A, 32768, 4, B, B, None, None, ctypes.byref(wide), st) == rq.RQ_ERR_UNSUPPORTED_SHAPE
    assert L.rq_gptq_quantize_pack(A, 1024, 64, B, B, None, None, ctypes.byref(d), st) == rq.RQ_ERR_FORMAT_MISMATCH
    assert L.rq_gptq_quantize_pack(U, 2048, 64, B, B, None, None, ctypes.byref(d), st) == rq.RQ_ERR_MISALIGNED
    assert rq.rq_status_string(rq.RQ_ERR_NOT_POSITIVE_DEFINITE) != "unknown status"


def test_wgemm_out_validation(L):
    d = _desc("w4g64", 2048, 256)
    st = ctypes.c_void_p(0)
    assert L.rq_wgemm_out(A, 1, 2048, 256, ctypes.byref(d), A, 2, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_wgemm_out(A, 1, 2048, 256, ctypes.byref(d), A, -1, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_wgemm_out(A, 1, 2048, 256, ctypes.byref(d), U, rq.RQ_OUT_BF16, st) == rq.RQ_ERR_MISALIGNED
    item = rq.RqWgemmItem(0x40000, ctypes.pointer(d), 0x40000)
    arr = (rq.RqWgemmItem * 1)(item)
    assert L.rq_wgemm_batch_out(arr, 1, 1, 3, st) == rq.RQ_ERR_INVALID_ARG


def test_dequant_validation(L):
    st = ctypes.c_void_p(0)
    d = _desc("w4sb32", 512, 8, scales=0)
    assert L.rq_dequant(ctypes.byref(d), None, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_dequant(ctypes.byref(d), U, st) == rq.RQ_ERR_MISALIGNED
    assert L.rq_dequant(None, A, st) == rq.RQ_ERR_INVALID_ARG
    for f in ("w4sb32", "w5sb32", "w6sb32"):
        bad = _desc(f, 320, 8, scales=0)
        assert L.rq_dequant(ctypes.byref(bad), A, st) == rq.RQ_ERR_UNSUPPORTED_SHAPE


def test_binding_raises_without_library(monkeypatch, tmp_path):
    """The binding has no fallback: a missing library is an error."""
    monkeypatch.setattr(rq, "_L", None)
    monkeypatch.setattr(rq, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(ImportError):
        rq.rq_version()


def test_wgemm_batch_validation(L):
    st = ctypes.c_void_p(0)
    d1 = _desc("w4g64", 2048, 256)
    d2 = _desc("w8g16", 2048, 256)
    Items = rq.RqWgemmItem * 2
    good = Items(rq.RqWgemmItem(0x40000, ctypes.pointer(d1), 0x50000),
                 rq.RqWgemmItem(0x60000, ctypes.pointer(d1), 0x70000))
    assert L.rq_wgemm_batch(None, 1, 1, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_wgemm_batch(good, 0, 1, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_wgemm_batch(good, 161, 1, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_wgemm_batch(good, 2, 0, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_wgemm_batch(good, 2, 129, st) == rq.RQ_ERR_INVALID_ARG
    mixed = Items(rq.RqWgemmItem(0x40000, ctypes.pointer(d1), 0x50000),
                  rq.RqWgemmItem(0x60000, ctypes.pointer(d2), 0x70000))
    assert L.rq_wgemm_batch(mixed, 2, 1, st) == rq.RQ_ERR_FORMAT_MISMATCH
    mis = Items(rq.RqWgemmItem(0x40000, ctypes.pointer(d1), 0x50000),
                rq.RqWgemmItem(0x60008, ctypes.pointer(d1), 0x70000))
    assert L.rq_wgemm_batch(mis, 2, 1, st) == rq.RQ_ERR_MISALIGNED
    nul = Items(rq.RqWgemmItem(0x40000, ctypes.pointer(d1), 0x50000),
                rq.RqWgemmItem(0x60000, None, 0x70000))
    assert L.rq_wgemm_batch(nul, 2, 1, st) == rq.RQ_ERR_INVALID_ARG


def test_act_stats_validation(L):
    """The E[x^2] calls reject bad arguments on the host (nothing launched)."""
    A, U, st = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 20) + 8), None
    assert L.rq_act_sumsq(None, 4, 64, A, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_act_sumsq(A, 4, 64, None, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_act_sumsq(A, 0, 64, A, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_act_sumsq(A, 4, 0, A, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_act_sumsq(A, (1 << 24) + 1, 64, A, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_act_sumsq(U, 4, 64, A, st) == rq.RQ_ERR_MISALIGNED
    assert L.rq_act_sumsq(A, 4, 64, U, st) == rq.RQ_ERR_MISALIGNED
    assert L.rq_act_finalize(None, 64, 4, A, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_act_finalize(A, 64, 0, A, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_act_finalize(A, 0, 4, A, st) == rq.RQ_ERR_INVALID_ARG
    assert L.rq_act_finalize(A, 64, 4, U, st) == rq.RQ_ERR_MISALIGNED
