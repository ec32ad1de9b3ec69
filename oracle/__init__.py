"""CPU oracle for weight-only group quantization (RTN and E[x^2]-weighted
search), packing, exact dequantization, the fp64 product and the activation
statistic E[x^2].

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The product library
(``weight_only_quantized_rq_b200``) shares no code with it and never calls it.

The arithmetic lives in ``rq_oracle.c`` (plain C loops, IEEE fp32/fp64, no
contraction, no fast-math); this module only compiles it and marshals numpy
arrays. Formats are named by strings here: ``"w4g64"`` (symmetric int4, group
64), ``"w8g16"`` / ``"w8g64"`` (symmetric int8, group 16 / 64), ``"w6g16"``
(symmetric 6-bit, group 16), ``"w4sb32"`` / ``"w5sb32"`` / ``"w6sb32"``
(asymmetric 4-, 5-, 6-bit superblocks of 8 groups of 32).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rq_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_SO = os.path.join(_OUT_DIR, "librq_oracle.so")

FORMATS = {"w4g64": 1, "w8g16": 2, "w4sb32": 3, "w5sb32": 4, "w6sb32": 5, "w8g64": 6, "w6g16": 7}
GROUP = {"w4g64": 64, "w8g16": 16, "w4sb32": 32, "w5sb32": 32, "w6sb32": 32, "w8g64": 64, "w6g16": 16}
SB_BITS = {"w4sb32": 4, "w5sb32": 5, "w6sb32": 6}
SB_BYTES = {"w4sb32": 144, "w5sb32": 176, "w6sb32": 208}
QMAX = {"w4g64": 7, "w8g16": 127, "w8g64": 127, "w6g16": 31}

_P = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/librq_oracle.so``."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    if (not force and os.path.exists(_SO)
            and os.path.getmtime(_SO) >= os.path.getmtime(_SRC)):
        return _SO
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fopenmp", "-fPIC", "-shared", _SRC, "-o", _SO + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(_SO + ".tmp", _SO)
    return _SO


_lib = None


def _bind(L: ctypes.CDLL) -> ctypes.CDLL:
    L.orc_f32_to_f16.argtypes = [_f]
    L.orc_f32_to_f16.restype = ctypes.c_uint16
    L.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
    L.orc_f16_to_f32.restype = _f
    L.orc_f32_to_f16_n.argtypes = [_P, _P, ctypes.c_long]
    L.orc_f32_to_f16_n.restype = None
    L.orc_f16_to_f32_n.argtypes = [_P, _P, ctypes.c_long]
    L.orc_f16_to_f32_n.restype = None
    L.orc_grid.argtypes = [_i, _f, _f, _P]
    L.orc_grid.restype = None
    L.orc_sym_group.argtypes = [_P, _P, _i, _i, _P, _i, _P, _P, _P]
    L.orc_sym_group.restype = _i
    L.orc_asym_group.argtypes = [_P, _P, _i, _P, _i, _i, _P, _P, _P]
    L.orc_asym_group.restype = _i
    L.orc_sb_finish.argtypes = [_P, _P, _P, _i, _P]
    L.orc_sb_finish.restype = None
    L.orc_sb_field.argtypes = [_P, _i, _i]
    L.orc_sb_field.restype = _i
    L.orc_pack_sym.argtypes = [_P, _i, _i, _P, _i, _i, _f, _f, _P, _P]
    L.orc_pack_sym.restype = None
    L.orc_pack_sb32.argtypes = [_P, _i, _i, _P, _i, _f, _f, _i, _P]
    L.orc_pack_sb32.restype = None
    L.orc_dequant.argtypes = [_i, _i, _i, _P, _P, _P]
    L.orc_dequant.restype = None
    L.orc_wgemm.argtypes = [_i, _P, _i, _i, _i, _P, _P, _P, _i, _P]
    L.orc_wgemm.restype = None
    L.orc_act_sumsq.argtypes = [_P, _i, _i, _P]
    L.orc_act_sumsq.restype = None
    L.orc_act_finalize.argtypes = [_P, _i, ctypes.c_longlong, _P]
    L.orc_act_finalize.restype = None
    L.orc_hessian_accum.argtypes = [_P, _i, _i, _P]
    L.orc_hessian_accum.restype = None
    L.orc_gptq_pack_sym.argtypes = [_P, _i, _i, _P, _P, _P, _i, _i, _f, _f, _P, _P]
    L.orc_gptq_pack_sym.restype = None
    L.orc_gptq_pack_sb.argtypes = [_P, _i, _i, _P, _P, _P, _i, _f, _f, _i, _P]
    L.orc_gptq_pack_sb.restype = None
    L.orc_threads.argtypes = []
    L.orc_threads.restype = _i
    L.orc_set_threads.argtypes = [_i]
    L.orc_set_threads.restype = None
    return L


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(_SO))
    return _lib


def compile_variant(src_text: str, out_so: str) -> None:
    """Compile C source text with the oracle's flags (used by the mutation
    test to plant mistakes in a copy, never by the product)."""
    src = out_so + ".c"
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                    "-fopenmp", "-fPIC", "-shared", src, "-o", out_so, "-lm"], check=True)


def swap_library(path: str | None):
    """Bind the module to the library at ``path`` (None: the real oracle).
    Returns the previously bound library handle."""
    global _lib
    prev = _lib
    _lib = None if path is None else _bind(ctypes.CDLL(path))
    return prev


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def threads() -> int:
    return lib().orc_threads()


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


# ---------------------------------------------------------------- numbers ---
def f32_to_f16_bits(v) -> np.ndarray:
    """IEEE binary16 bits of each fp32 value (round to nearest even)."""
    v = _c(v, np.float32).ravel()
    out = np.zeros(v.size, dtype=np.uint16)
    lib().orc_f32_to_f16_n(_ptr(v), _ptr(out), v.size)
    return out


def f16_bits_to_f32(h) -> np.ndarray:
    h = _c(h, np.uint16).ravel()
    out = np.zeros(h.size, dtype=np.float32)
    lib().orc_f16_to_f32_n(_ptr(h), _ptr(out), h.size)
    return out


def grid(n: int, t_lo: float = 0.7, t_hi: float = 1.0) -> np.ndarray:
    t = np.zeros(n, dtype=np.float32)
    lib().orc_grid(n, t_lo, t_hi, _ptr(t))
    return t


# ----------------------------------------------------------------- groups ---
def sym_group(w, a, qmax: int, n: int = 64, t_lo: float = 0.7, t_hi: float = 1.0):
    """Search one symmetric group. Returns (index, fp16 scale bits, codes, losses)."""
    w = _c(w, np.float32)
    a = None if a is None else _c(a, np.float32)
    t = grid(n, t_lo, t_hi)
    s = np.zeros(1, dtype=np.uint16)
    q = np.zeros(w.size, dtype=np.int8)
    losses = np.zeros(n, dtype=np.float64)
    idx = lib().orc_sym_group(_ptr(w), _ptr(a), w.size, qmax, _ptr(t), n, _ptr(s), _ptr(q), _ptr(losses))
    return idx, int(s[0]), q, losses


def asym_group(w, a, n: int = 64, t_lo: float = 0.7, t_hi: float = 1.0, bits: int = 4):
    """Search one asymmetric group of `bits`-bit codes. Returns (index, S*, M*, losses)."""
    w = _c(w, np.float32)
    a = None if a is None else _c(a, np.float32)
    t = grid(n, t_lo, t_hi)
    S = np.zeros(1, dtype=np.float32)
    M = np.zeros(1, dtype=np.float32)
    losses = np.zeros(n, dtype=np.float64)
    idx = lib().orc_asym_group(_ptr(w), _ptr(a), w.size, _ptr(t), n, bits, _ptr(S), _ptr(M), _ptr(losses))
    return idx, float(S[0]), float(M[0]), losses


def sb_finish(w256, S_star, M_star, bits: int = 4) -> np.ndarray:
    """The superblock record (144 / 176 / 208 bytes for 4 / 5 / 6 bits) for
    256 weights and 8 searched (S*, M*)."""
    w = _c(w256, np.float32)
    S = _c(S_star, np.float32)
    M = _c(M_star, np.float32)
    blk = np.zeros(16 + 128 + (bits - 4) * 32, dtype=np.uint8)
    lib().orc_sb_finish(_ptr(w), _ptr(S), _ptr(M), bits, _ptr(blk))
    return blk


def sb_field(blk, which: int, j: int) -> int:
    blk = _c(blk, np.uint8)
    return lib().orc_sb_field(_ptr(blk), which, j)


# ---------------------------------------------------------------- matrices --
def packed_shapes(fmt: str, K: int, N: int):
    """(codes shape, codes dtype, scales shape or None)."""
    if fmt == "w4g64":
        return (N, K // 2), np.uint8, (N, K // 64)
    if fmt == "w8g16":
        return (N, K), np.uint8, (N, K // 16)
    if fmt == "w8g64":
        return (N, K), np.uint8, (N, K // 64)
    if fmt == "w6g16":
        return (N, K // 64 * 48), np.uint8, (N, K // 16)
    if fmt in SB_BYTES:
        return (N, (K // 256) * SB_BYTES[fmt]), np.uint8, None
    raise ValueError(fmt)


def pack(fmt: str, W, act_sq=None, n_cand: int = 64, t_lo: float = 0.7, t_hi: float = 1.0):
    """Quantize and pack W [N][K] fp32. Returns (codes, scales or None)."""
    W = _c(W, np.float32)
    N, K = W.shape
    a = None if act_sq is None else _c(act_sq, np.float32)
    cshape, cdt, sshape = packed_shapes(fmt, K, N)
    codes = np.zeros(cshape, dtype=cdt)
    if fmt in SB_BITS:
        lib().orc_pack_sb32(_ptr(W), K, N, _ptr(a), n_cand, t_lo, t_hi, SB_BITS[fmt], _ptr(codes))
        return codes, None
    scales = np.zeros(sshape, dtype=np.uint16)
    lib().orc_pack_sym(_ptr(W), K, N, _ptr(a), FORMATS[fmt], n_cand, t_lo, t_hi,
                       _ptr(codes), _ptr(scales))
    return codes, scales


def dequant(fmt: str, K: int, N: int, codes, scales) -> np.ndarray:
    codes = _c(codes, np.uint8)
    scales = None if scales is None else _c(scales, np.uint16)
    out = np.zeros((N, K), dtype=np.float32)
    lib().orc_dequant(FORMATS[fmt], K, N, _ptr(codes), _ptr(scales), _ptr(out))
    return out


def wgemm(fmt: str, x_bf16_bits, K: int, N: int, codes, scales, rows=None) -> np.ndarray:
    """fp64 y[M][len(rows)] = x @ w_hat[rows].T, ascending-k sums.

    ``x_bf16_bits`` is the raw bf16 bit pattern of x, uint16 [M][K]."""
    x = _c(x_bf16_bits, np.uint16)
    M = x.shape[0]
    codes = _c(codes, np.uint8)
    scales = None if scales is None else _c(scales, np.uint16)
    r = None if rows is None else _c(rows, np.int32)
    nr = N if r is None else r.size
    y = np.zeros((M, nr), dtype=np.float64)
    lib().orc_wgemm(FORMATS[fmt], _ptr(x), M, K, N, _ptr(codes), _ptr(scales), _ptr(r), nr, _ptr(y))
    return y


def act_sumsq(x_bf16_bits, sum_sq=None) -> np.ndarray:
    """Running per-channel sums of x^2 over the rows of x (raw bf16 bits,
    uint16 [R][K]) added into ``sum_sq`` (fp64 [K], zeros when None): each
    channel's squares are added to its running sum one row at a time, rows
    ascending, in fp64."""
    x = _c(x_bf16_bits, np.uint16)
    R, K = x.shape
    out = np.zeros(K, dtype=np.float64) if sum_sq is None else np.array(sum_sq, dtype=np.float64, copy=True)
    lib().orc_act_sumsq(_ptr(x), R, K, _ptr(out))
    return out


def act_finalize(sum_sq, rows: int) -> np.ndarray:
    """E[x^2] = fp32(sum_sq / rows)."""
    s = _c(sum_sq, np.float64)
    out = np.zeros(s.size, dtype=np.float32)
    lib().orc_act_finalize(_ptr(s), s.size, int(rows), _ptr(out))
    return out


# --------------------------------------------------------------------- GPTQ --
def hessian_accum(x_bf16_bits, H=None) -> np.ndarray:
    """H += x^T x (fp64 [K][K]) over the bf16 rows x [R][K], every element
    summed in ascending row order."""
    x = _c(x_bf16_bits, np.uint16)
    R, K = x.shape
    out = np.zeros((K, K), np.float64) if H is None else _c(H, np.float64).copy()
    lib().orc_hessian_accum(_ptr(x), R, K, _ptr(out))
    return out


def gptq_prepare(H, damp: float = 0.01):
    """The factor GPTQ's column loop needs (Frantar et al. 2022): columns with
    H_kk == 0 are dead (H_kk := 1, their weights are zeroed); the diagonal is
    damped by damp * mean(diag H); U = the upper Cholesky factor of H^-1,
    computed as in the method's description: Cholesky of H, the inverse from
    it, Cholesky of the inverse. numpy's LAPACK routines are the library
    steps. Returns (U fp64 [K][K] upper, dead uint8 [K])."""
    H = np.array(H, dtype=np.float64, copy=True)
    K = H.shape[0]
    d = np.diag(H).copy()
    dead = d == 0.0
    H[np.arange(K)[dead], np.arange(K)[dead]] = 1.0
    lam = damp * np.mean(np.diag(H))
    H[np.arange(K), np.arange(K)] += lam
    L = np.linalg.cholesky(H)
    Linv = np.linalg.inv(L)
    Hinv = Linv.T @ Linv
    U = np.linalg.cholesky(Hinv).T
    return np.ascontiguousarray(np.triu(U)), dead.astype(np.uint8)


def gptq_pack(fmt: str, W, U, dead, act_sq=None, n_cand: int = 64, t_lo: float = 0.7, t_hi: float = 1.0):
    """GPTQ on the preset's grid; the same planes as pack(). Returns
    (codes, scales or None)."""
    W = _c(W, np.float32)
    N, K = W.shape
    U = _c(U, np.float64)
    dead = _c(dead, np.uint8)
    a = None if act_sq is None else _c(act_sq, np.float32)
    cshape, cdt, sshape = packed_shapes(fmt, K, N)
    codes = np.zeros(cshape, dtype=cdt)
    if fmt in SB_BITS:
        lib().orc_gptq_pack_sb(_ptr(W), K, N, _ptr(U), _ptr(dead), _ptr(a), n_cand, t_lo, t_hi, SB_BITS[fmt],
                               _ptr(codes))
        return codes, None
    scales = np.zeros(sshape, dtype=np.uint16)
    lib().orc_gptq_pack_sym(_ptr(W), K, N, _ptr(U), _ptr(dead), _ptr(a), FORMATS[fmt], n_cand, t_lo, t_hi,
                            _ptr(codes), _ptr(scales))
    return codes, scales
