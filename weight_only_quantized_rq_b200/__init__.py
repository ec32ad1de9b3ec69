"""Python binding of librq (include/rq.h): weight-only group-quantized matrix
products for RWKV-7 on B200.

This module only marshals arguments: it passes torch tensors' device pointers
and the current CUDA stream to the C ABI. PyTorch provides device memory and
streams; every step of the computation runs in librq's CUDA kernels. There is
no fallback: if librq.so is missing, every call raises.

Formats (see include/rq.h): ``RQ_W4_SYM_G64`` (symmetric int4, group 64),
``RQ_W8_SYM_G16`` / ``RQ_W8_SYM_G64`` (symmetric int8, group 16 / 64),
``RQ_W6_SYM_G16`` (symmetric 6-bit, group 16), ``RQ_W4_ASYM_SB32``,
``RQ_W5_ASYM_SB32``, ``RQ_W6_ASYM_SB32`` (asymmetric 4-, 5-, 6-bit superblocks
of 8 groups of 32). The strings "w4g64", "w8g16", "w8g64", "w6g16", "w4sb32",
"w5sb32", "w6sb32" are accepted wherever a format is expected.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librq.so")

RQ_OK = 0
RQ_ERR_INVALID_ARG = 1
RQ_ERR_UNSUPPORTED_SHAPE = 2
RQ_ERR_FORMAT_MISMATCH = 3
RQ_ERR_MISALIGNED = 4
RQ_ERR_CUDA = 5
RQ_ERR_DEVICE_TIMEOUT = 6
RQ_ERR_NOT_POSITIVE_DEFINITE = 7

RQ_OUT_F32 = 0
RQ_OUT_BF16 = 1

RQ_W4_SYM_G64 = 1
RQ_W8_SYM_G16 = 2
RQ_W4_ASYM_SB32 = 3
RQ_W5_ASYM_SB32 = 4
RQ_W6_ASYM_SB32 = 5
RQ_W8_SYM_G64 = 6
RQ_W6_SYM_G16 = 7
FORMAT_IDS = {"w4g64": RQ_W4_SYM_G64, "w8g16": RQ_W8_SYM_G16, "w4sb32": RQ_W4_ASYM_SB32,
              "w5sb32": RQ_W5_ASYM_SB32, "w6sb32": RQ_W6_ASYM_SB32, "w8g64": RQ_W8_SYM_G64,
              "w6g16": RQ_W6_SYM_G16}
SB_FORMATS = (RQ_W4_ASYM_SB32, RQ_W5_ASYM_SB32, RQ_W6_ASYM_SB32)
EXPORTS = ("rq_packed_size", "rq_quantize_pack", "rq_wgemm", "rq_wgemm_batch", "rq_wgemm_out", "rq_wgemm_batch_out",
           "rq_dequant",
           "rq_act_sumsq", "rq_act_finalize", "rq_hessian_accum", "rq_gptq_prepare", "rq_gptq_quantize_pack",
           "rq_status_string", "rq_last_cuda_error", "rq_device_status", "rq_test_hooks", "rq_version")
MAX_BATCH = 160
TC_MIN_M = 3         # activation rows from which int4/int8/4-bit superblock products run on the tensor cores
                     # (5- and 6-bit products run there at every M)
TC_MAX_ITEMS = 96    # products per tensor-core launch (larger batches take several)


def tc_path(fmt, M: int) -> bool:
    """Whether products of this format at M activation rows run on the
    tensor-core kernel (else on the register-path GEMV)."""
    f = fmt_id(fmt)
    if f in (RQ_W5_ASYM_SB32, RQ_W6_ASYM_SB32, RQ_W6_SYM_G16):
        return True
    return M >= TC_MIN_M


class RqSearch(ctypes.Structure):
    _fields_ = [("n_cand", ctypes.c_int), ("t_lo", ctypes.c_float), ("t_hi", ctypes.c_float)]


class RqPacked(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int), ("K", ctypes.c_int), ("N", ctypes.c_int), ("reserved", ctypes.c_int),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class RqWgemmItem(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("w", ctypes.POINTER(RqPacked)), ("y", ctypes.c_void_p)]


class RqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {rq_status_string(status)} (status {status})"
        if status == RQ_ERR_CUDA:
            msg += f", cudaError {_lib().rq_last_cuda_error()}"
        super().__init__(msg)


_L = None


def _lib() -> ctypes.CDLL:
    """Load librq.so (built in-tree). Raises if it is absent: there is no
    other implementation to fall back to."""
    global _L
    if _L is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"librq.so is not built ({LIB_PATH}); run "
                              "`python -m weight_only_quantized_rq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I = ctypes.c_void_p, ctypes.c_int
        L.rq_packed_size.argtypes = [I, I, I, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]
        L.rq_packed_size.restype = ctypes.c_size_t
        L.rq_quantize_pack.argtypes = [P, I, I, P, ctypes.POINTER(RqSearch), ctypes.POINTER(RqPacked), P]
        L.rq_quantize_pack.restype = I
        L.rq_wgemm.argtypes = [P, I, I, I, ctypes.POINTER(RqPacked), P, P]
        L.rq_wgemm.restype = I
        L.rq_wgemm_batch.argtypes = [ctypes.POINTER(RqWgemmItem), I, I, P]
        L.rq_wgemm_batch.restype = I
        L.rq_wgemm_out.argtypes = [P, I, I, I, ctypes.POINTER(RqPacked), P, I, P]
        L.rq_wgemm_out.restype = I
        L.rq_wgemm_batch_out.argtypes = [ctypes.POINTER(RqWgemmItem), I, I, I, P]
        L.rq_wgemm_batch_out.restype = I
        L.rq_dequant.argtypes = [ctypes.POINTER(RqPacked), P, P]
        L.rq_dequant.restype = I
        L.rq_act_sumsq.argtypes = [P, I, I, P, P]
        L.rq_act_sumsq.restype = I
        L.rq_act_finalize.argtypes = [P, I, ctypes.c_longlong, P, P]
        L.rq_act_finalize.restype = I
        L.rq_hessian_accum.argtypes = [P, I, I, P, P]
        L.rq_hessian_accum.restype = I
        L.rq_gptq_prepare.argtypes = [P, I, ctypes.c_double, P, P, P]
        L.rq_gptq_prepare.restype = I
        L.rq_gptq_quantize_pack.argtypes = [P, I, I, P, P, P, ctypes.POINTER(RqSearch), ctypes.POINTER(RqPacked), P]
        L.rq_gptq_quantize_pack.restype = I
        L.rq_status_string.argtypes = [I]
        L.rq_status_string.restype = ctypes.c_char_p
        L.rq_last_cuda_error.argtypes = []
        L.rq_last_cuda_error.restype = I
        L.rq_device_status.argtypes = [P, ctypes.POINTER(I)]
        L.rq_device_status.restype = I
        L.rq_test_hooks.argtypes = [ctypes.c_longlong, I]
        L.rq_test_hooks.restype = I
        L.rq_version.argtypes = []
        L.rq_version.restype = I
        _L = L
    return _L


def lib() -> ctypes.CDLL:
    return _lib()


def fmt_id(fmt) -> int:
    return FORMAT_IDS[fmt] if isinstance(fmt, str) else int(fmt)


def _stream(stream=None) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _check(status: int, where: str) -> None:
    if status != RQ_OK:
        raise RqError(status, where)


# ------------------------------------------------------------------ calls --
def rq_status_string(status: int) -> str:
    return _lib().rq_status_string(int(status)).decode()


def rq_version() -> int:
    return _lib().rq_version()


def rq_packed_size(fmt, K: int, N: int) -> tuple[int, int]:
    """(codes_bytes, scales_bytes); raises for an unsupported shape."""
    cb, sb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    tot = _lib().rq_packed_size(fmt_id(fmt), int(K), int(N), ctypes.byref(cb), ctypes.byref(sb))
    if tot == 0:
        raise RqError(RQ_ERR_UNSUPPORTED_SHAPE, "rq_packed_size")
    return cb.value, sb.value


@dataclass
class Packed:
    """A packed matrix: the descriptor fields plus the two device planes
    (uint8 tensors that own the memory)."""
    fmt: int
    K: int
    N: int
    codes: torch.Tensor
    scales: torch.Tensor | None

    def desc(self) -> RqPacked:
        return RqPacked(self.fmt, self.K, self.N, 0, self.codes.data_ptr(),
                        None if self.scales is None else self.scales.data_ptr())

    @property
    def nbytes(self) -> int:
        return self.codes.numel() + (0 if self.scales is None else self.scales.numel())


def alloc_packed(fmt, K: int, N: int, device=None) -> Packed:
    f = fmt_id(fmt)
    cb, sb = rq_packed_size(f, K, N)
    dev = torch.device("cuda") if device is None else torch.device(device)
    codes = torch.empty(cb, dtype=torch.uint8, device=dev)
    scales = torch.empty(sb, dtype=torch.uint8, device=dev) if sb else None
    return Packed(f, int(K), int(N), codes, scales)


def rq_quantize_pack(W: torch.Tensor, fmt, act_sq: torch.Tensor | None = None, n_cand: int = 64,
                     t_lo: float = 0.7, t_hi: float = 1.0, out: Packed | None = None, stream=None) -> Packed:
    """Quantize and pack W (fp32 [N][K], CUDA). Returns the Packed matrix."""
    N, K = W.shape
    if out is None:
        out = alloc_packed(fmt, K, N, W.device)
    sr = RqSearch(int(n_cand), float(t_lo), float(t_hi))
    d = out.desc()
    _check(_lib().rq_quantize_pack(_ptr(W), int(K), int(N), _ptr(act_sq), ctypes.byref(sr), ctypes.byref(d),
                                   _stream(stream)), "rq_quantize_pack")
    return out


def _out_type(dtype) -> int:
    if dtype == torch.float32:
        return RQ_OUT_F32
    if dtype == torch.bfloat16:
        return RQ_OUT_BF16
    raise ValueError("y must be float32 or bfloat16")


def rq_wgemm(x: torch.Tensor, w: Packed, y: torch.Tensor | None = None, stream=None,
             out_dtype=torch.float32) -> torch.Tensor:
    """y = x @ w_hat.T with x bf16 [M][K] and y [M][N] (CUDA tensors), y fp32
    or bf16 (the fp32 result rounded once; by y's dtype, else out_dtype)."""
    M, K = x.shape
    if y is None:
        y = torch.empty(M, w.N, dtype=out_dtype, device=x.device)
    d = w.desc()
    _check(_lib().rq_wgemm_out(_ptr(x), int(M), int(K), int(w.N), ctypes.byref(d), _ptr(y), _out_type(y.dtype),
                               _stream(stream)), "rq_wgemm_out")
    return y


class WgemmBatch:
    """A prepared batch for rq_wgemm_batch: the ctypes item array is built
    once (so repeated calls and CUDA-graph capture pay no marshalling)."""

    def __init__(self, xs, ws, ys):
        if not (len(xs) == len(ws) == len(ys)) or not 1 <= len(xs) <= MAX_BATCH:
            raise ValueError("need 1..160 items with one x, w, y each")
        self.M = int(xs[0].shape[0])
        self._keep = (list(xs), list(ws), list(ys))
        self._descs = [w.desc() for w in ws]
        self._items = (RqWgemmItem * len(xs))()
        self.out = _out_type(ys[0].dtype)
        for i, (x, d, y) in enumerate(zip(xs, self._descs, ys)):
            if int(x.shape[0]) != self.M:
                raise ValueError("every item must have the same M")
            if _out_type(y.dtype) != self.out:
                raise ValueError("every y must have the same dtype")
            self._items[i] = RqWgemmItem(x.data_ptr(), ctypes.pointer(d), y.data_ptr())
        self.count = len(xs)

    def __call__(self, stream=None):
        _check(_lib().rq_wgemm_batch_out(self._items, self.count, self.M, self.out, _stream(stream)),
               "rq_wgemm_batch_out")


def rq_wgemm_batch(xs, ws, ys, stream=None) -> None:
    """Independent products ys[i] = xs[i] @ w_hat_i.T in one launch."""
    WgemmBatch(xs, ws, ys)(stream)


def rq_dequant(w: Packed, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """w_hat as fp32 [N][K] (CUDA)."""
    if out is None:
        out = torch.empty(w.N, w.K, dtype=torch.float32, device=w.codes.device)
    d = w.desc()
    _check(_lib().rq_dequant(ctypes.byref(d), _ptr(out), _stream(stream)), "rq_dequant")
    return out


def rq_act_sumsq(x: torch.Tensor, sum_sq: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Add sum_r x[r][k]^2 (x bf16 [R][K] on the GPU) into the fp64 running
    sums sum_sq[K] (created as zeros when None) and return them."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 [R][K] tensor")
    R, K = int(x.shape[0]), int(x.shape[1])
    if sum_sq is None:
        sum_sq = torch.zeros(K, dtype=torch.float64, device=x.device)
    _check(_lib().rq_act_sumsq(_ptr(x), R, K, _ptr(sum_sq), _stream(stream)), "rq_act_sumsq")
    return sum_sq


def rq_act_finalize(sum_sq: torch.Tensor, rows: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """E[x^2] = fp32(sum_sq / rows), the act_sq that rq_quantize_pack takes."""
    K = int(sum_sq.shape[0])
    if out is None:
        out = torch.empty(K, dtype=torch.float32, device=sum_sq.device)
    _check(_lib().rq_act_finalize(_ptr(sum_sq), K, int(rows), _ptr(out), _stream(stream)), "rq_act_finalize")
    return out


def rq_hessian_accum(x: torch.Tensor, H: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """H += x^T x (x bf16 [R][K] on the GPU; H fp64 [K][K], created as zeros
    when None), each element summed in ascending row order. Returns H."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 [R][K] tensor")
    R, K = int(x.shape[0]), int(x.shape[1])
    if H is None:
        H = torch.zeros(K, K, dtype=torch.float64, device=x.device)
    _check(_lib().rq_hessian_accum(_ptr(x), R, K, _ptr(H), _stream(stream)), "rq_hessian_accum")
    return H


def rq_gptq_prepare(H: torch.Tensor, damp: float = 0.01, U: torch.Tensor | None = None,
                    dead: torch.Tensor | None = None, stream=None):
    """The upper Cholesky factor U of the damped inverse Hessian and the dead
    channel flags (H fp64 [K][K] on the GPU). Returns (U, dead)."""
    K = int(H.shape[0])
    if U is None:
        U = torch.empty(K, K, dtype=torch.float64, device=H.device)
    if dead is None:
        dead = torch.empty(K, dtype=torch.uint8, device=H.device)
    _check(_lib().rq_gptq_prepare(_ptr(H), K, float(damp), _ptr(U), _ptr(dead), _stream(stream)), "rq_gptq_prepare")
    return U, dead


def rq_gptq_quantize_pack(W: torch.Tensor, fmt, U: torch.Tensor, dead: torch.Tensor,
                          act_sq: torch.Tensor | None = None, n_cand: int = 64, t_lo: float = 0.7, t_hi: float = 1.0,
                          out: Packed | None = None, stream=None) -> Packed:
    """GPTQ on the preset's grid: quantize W (fp32 [N][K], CUDA) into any
    format with the factor of rq_gptq_prepare. Returns the Packed matrix (same
    planes as rq_quantize_pack)."""
    N, K = W.shape
    if out is None:
        out = alloc_packed(fmt, K, N, W.device)
    sr = RqSearch(int(n_cand), float(t_lo), float(t_hi))
    d = out.desc()
    _check(_lib().rq_gptq_quantize_pack(_ptr(W), int(K), int(N), _ptr(U), _ptr(dead), _ptr(act_sq), ctypes.byref(sr),
                                        ctypes.byref(d), _stream(stream)), "rq_gptq_quantize_pack")
    return out


def rq_device_status(stream=None) -> int:
    """Read and clear the device status word (synchronizes the stream)."""
    word = ctypes.c_int(0)
    st = _lib().rq_device_status(_stream(stream), ctypes.byref(word))
    if st not in (RQ_OK, RQ_ERR_DEVICE_TIMEOUT, RQ_ERR_NOT_POSITIVE_DEFINITE):
        raise RqError(st, "rq_device_status")
    return word.value


def rq_test_hooks(wait_ns: int = 0, flags: int = 0) -> None:
    """Testing hook: the bound of every device wait (0 = the default 2 s)
    and flags (1 = issue no weight copies, so the waits run out)."""
    _check(_lib().rq_test_hooks(int(wait_ns), int(flags)), "rq_test_hooks")


# short aliases
quantize_pack = rq_quantize_pack
wgemm = rq_wgemm
wgemm_batch = rq_wgemm_batch
dequant = rq_dequant
packed_size = rq_packed_size
