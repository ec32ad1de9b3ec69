"""Pins for the CPU oracle.

Every test here checks the oracle against something other than itself: exact
rational brute force on tiny groups, closed-form bounds, invariants of the
method, constructions whose exact result is known in integers, a library
routine the computation reduces to, and sizes the pages print
(tests/golden/format_sizes.json). The pages are the rwkv-quant article
("Two presets and six sizes", "Where 2.9B breaks") and the RWKV-7 G1 1.5B int4
model card ("Format & loading", summary paragraph).
"""
import json
import os
from fractions import Fraction as Fr

import numpy as np
import pytest

GOLD = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------ helpers ------
def nearest_int_even(v: Fr) -> int:
    """Exact nearest integer, ties to even."""
    f = v.numerator // v.denominator
    r = v - f
    if r > Fr(1, 2):
        return f + 1
    if r < Fr(1, 2):
        return f
    return f if f % 2 == 0 else f + 1


def near_half(v: Fr, tol=Fr(1, 1 << 18)) -> bool:
    """True when v is within tol (relative) of a half-integer, where an fp32
    quotient rounded before rint may legitimately round the other way."""
    f = v.numerator // v.denominator
    return abs((v - f) - Fr(1, 2)) <= tol * max(1, abs(v))


def f16(x) -> np.float32:
    """numpy's IEEE round-to-nearest-even binary16 conversion, back to fp32."""
    return np.float32(np.float16(np.float32(x)))


def grid_exact(n, lo=0.7, hi=1.0):
    return [Fr(float(np.float32(lo))) + (Fr(float(np.float32(hi))) - Fr(float(np.float32(lo)))) * i / (n - 1)
            for i in range(n)]


# ------------------------------------------------------ number formats -----
def test_f16_round_trip_every_half(orc):
    h = np.arange(65536, dtype=np.uint16)
    f = h.view(np.float16).astype(np.float32)
    fin = np.isfinite(f)
    got = orc.f16_bits_to_f32(h)
    assert np.array_equal(got[fin].view(np.uint32), f[fin].view(np.uint32))
    assert np.array_equal(orc.f32_to_f16_bits(f[fin]), h[fin])
    inf = np.isinf(f)
    assert np.array_equal(got[inf], f[inf])


def test_f16_midpoints_and_random_match_numpy(orc):
    # exact midpoints between neighbouring finite halves: ties must go to even
    h = np.arange(0, 0x7bff, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)  # exact in fp32
    vals = np.concatenate([mid, -mid])
    assert np.array_equal(orc.f32_to_f16_bits(vals), vals.astype(np.float16).view(np.uint16))
    # random fp32 values spanning the subnormal, normal and overflow ranges
    rng = np.random.default_rng(7)
    e = rng.integers(-30, 18, size=400_000)
    m = rng.random(400_000) + 1.0
    v = (np.ldexp(m, e) * rng.choice([-1.0, 1.0], size=e.size)).astype(np.float32)
    bits = rng.integers(0, 2**32, size=400_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    v = np.concatenate([v, bits[~np.isnan(bits)]])
    with np.errstate(over="ignore"):
        want = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(orc.f32_to_f16_bits(v), want)


# ------------------------------------------------------------- grid --------
def test_grid_is_uniform_and_spans_the_range(orc):
    """64 candidates over [0.7, 1.0] x absmax/qmax, both ends included, each
    within half an fp32 ulp of the exact uniform point."""
    t = orc.grid(64, 0.7, 1.0)
    assert t.size == 64 and t[0] == np.float32(0.7) and t[-1] == np.float32(1.0)
    assert np.all(np.diff(t) > 0)
    for ti, ex in zip(t, grid_exact(64)):
        ulp = np.spacing(np.float32(ti))
        assert abs(Fr(float(ti)) - ex) <= Fr(float(ulp)) / 2
    assert list(orc.grid(1, 0.7, 1.0)) == [1.0]


# ------------------------------------------- symmetric search, brute force --
def brute_sym(w, a, qmax, t):
    """Exhaustive exact-rational search over the candidate scales.
    Candidate s_i = fp16(fp32(t_i) * fp32(absmax / qmax)) via numpy; for each
    element the code is the exact nearest integer in [-qmax, qmax]."""
    absmax = np.float32(np.max(np.abs(w)))
    base = np.float32(absmax / np.float32(qmax))
    losses, codes = [], []
    for ti in t:
        s = Fr(float(f16(np.float32(ti) * base)))
        qs = []
        L = Fr(0)
        for wk, ak in zip(w, a):
            if s == 0:
                q = 0
            else:
                q = max(-qmax, min(qmax, nearest_int_even(Fr(float(wk)) / s)))
            qs.append(q)
            L += Fr(float(ak)) * (Fr(float(wk)) - q * s) ** 2
        losses.append(L)
        codes.append(qs)
    best = min(range(len(t)), key=lambda i: (losses[i], i))
    return best, losses, codes


def sym_cases():
    rng = np.random.default_rng(11)
    cases = []
    for G, qmax in [(4, 7), (16, 127), (16, 7), (64, 7)]:
        for rep in range(6 if G < 64 else 3):
            w = (rng.standard_normal(G) * 0.02).astype(np.float32)
            if rep % 3 == 1:
                w[rng.integers(G)] *= 10.0             # an outlier
            if rep % 3 == 2:
                w[rng.integers(G)] = 0.0
            a = np.ones(G, dtype=np.float32)
            if rep % 2 == 1:
                a[rng.integers(G)] = 2500.0            # a massive channel
            if rep == 4:
                a = rng.random(G).astype(np.float32)
            cases.append((w, a, qmax))
    return cases


@pytest.mark.parametrize("case", range(len(sym_cases())))
def test_sym_search_matches_exact_brute_force(orc, case):
    w, a, qmax = sym_cases()[case]
    t = orc.grid(64)
    idx, sbits, q, _ = orc.sym_group(w, a, qmax, 64)
    bidx, bl, bq = brute_sym(w, a, qmax, t)
    if idx != bidx:
        # only a near-tie (relative 1e-12) may be resolved differently by fp64
        assert abs(bl[idx] - bl[bidx]) <= Fr(1, 10**12) * max(bl[bidx], Fr(1, 10**30))
    s = Fr(float(np.array([sbits], dtype=np.uint16).view(np.float16)[0]))
    # the stored scale is the candidate's fp16 value
    absmax = np.float32(np.max(np.abs(w)))
    assert s == Fr(float(f16(np.float32(t[idx]) * np.float32(absmax / np.float32(qmax)))))
    for k, (wk, qk) in enumerate(zip(w, q)):
        if s != 0 and near_half(Fr(float(wk)) / s):
            continue
        assert qk == bq[idx][k]


def test_sym_ties_pick_lowest_index(orc):
    t = orc.grid(64)
    rng = np.random.default_rng(3)
    w = (rng.standard_normal(16) * 0.02).astype(np.float32)
    # all a_k = 0: every loss is 0
    idx, _, _, losses = orc.sym_group(w, np.zeros(16, np.float32), 127, 64)
    assert idx == 0 and np.all(losses == 0)
    # all-zero group: zero scale, zero codes, index 0
    idx, s, q, _ = orc.sym_group(np.zeros(64, np.float32), None, 7, 64)
    assert idx == 0 and s == 0 and not q.any()
    # every candidate rounds to the same fp16 subnormal: equal losses, index 0
    w = np.full(64, 7 * 2.0 ** -24, dtype=np.float32)
    idx, s, _, losses = orc.sym_group(w, None, 7, 64)
    assert idx == 0 and np.all(losses == losses[0]) and s == 1
    assert len(t) == 64


# ---------------------------------------------------- RTN closed form ------
@pytest.mark.parametrize("fmt", ["w4g64", "w8g16", "w8g64", "w6g16"])
def test_rtn_error_at_most_half_scale(orc, fmt):
    """RTN (one candidate, t = 1): no code clamps, every element is within
    s/2 of its dequantized value, and each group's absmax maps to +-qmax."""
    G, qmax = orc.GROUP[fmt], orc.QMAX[fmt]
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((8, 512)) * 0.02).astype(np.float32)
    W[0, :7] *= 30
    codes, scales = orc.pack(fmt, W, None, n_cand=1)
    Wd = orc.dequant(fmt, 512, 8, codes, scales)
    s = orc.f16_bits_to_f32(scales).reshape(8, -1).repeat(G, axis=1)
    err = np.abs(W.astype(np.float64) - Wd.astype(np.float64))
    assert np.all(err <= s.astype(np.float64) * (0.5 + qmax * 2.0 ** -23))
    q = np.round(Wd.astype(np.float64) / np.where(s == 0, 1, s)).astype(int)
    g = np.abs(W).reshape(8, -1, G).argmax(axis=2)
    qg = q.reshape(8, -1, G)
    for n in range(8):
        for j in range(qg.shape[1]):
            assert abs(qg[n, j, g[n, j]]) == qmax


# ----------------------------------------------------------- invariants ----
@pytest.mark.parametrize("fmt", ["w4g64", "w8g16", "w8g64", "w6g16"])
def test_sym_invariants(orc, fmt):
    G = orc.GROUP[fmt]
    rng = np.random.default_rng(9)
    W = (rng.standard_normal((4, 256)) * 0.02).astype(np.float32)
    a = np.ones(256, np.float32)
    a[17] = 2500.0
    c0, s0 = orc.pack(fmt, W, a)
    q0 = orc.dequant(fmt, 256, 4, c0, s0)
    # W -> -W: codes negate, scales unchanged
    c1, s1 = orc.pack(fmt, -W, a)
    assert np.array_equal(s1, s0)
    assert np.array_equal(orc.dequant(fmt, 256, 4, c1, s1), -q0)
    # W -> 2^e W: same codes, scales x 2^e, while every scale stays an fp16
    # normal (below 2^-14 the fp16 grid is coarser and the invariant is void)
    for e in {"w4g64": (-3, 2), "w6g16": (-2, 2)}.get(fmt, (1, 3)):
        sc = np.ldexp(orc.f16_bits_to_f32(s0), e)
        assert np.all(sc >= 2.0 ** -14) and np.all(sc <= 60000.0)
        c2, s2 = orc.pack(fmt, np.ldexp(W, e).astype(np.float32), a)
        assert np.array_equal(c2, c0)
        assert np.array_equal(orc.f16_bits_to_f32(s2), sc)
    # a -> 4a: same choice
    c3, s3 = orc.pack(fmt, W, 4 * a)
    assert np.array_equal(c3, c0) and np.array_equal(s3, s0)
    # permuting whole groups (with their a) permutes the output groups
    perm = rng.permutation(256 // G)
    Wp = W.reshape(4, -1, G)[:, perm].reshape(4, 256)
    ap = a.reshape(-1, G)[perm].reshape(256)
    c4, s4 = orc.pack(fmt, Wp, ap)
    assert np.array_equal(s4, s0[:, perm])
    assert np.array_equal(orc.dequant(fmt, 256, 4, c4, s4), q0.reshape(4, -1, G)[:, perm].reshape(4, 256))


def test_sb32_invariants(orc):
    rng = np.random.default_rng(21)
    W = (rng.standard_normal((3, 512)) * 0.02).astype(np.float32)
    a = np.ones(512, np.float32)
    a[300] = 15631.0
    c0, _ = orc.pack("w4sb32", W, a)
    blk0 = c0.reshape(3, 2, 144)
    for e in (1, 3):
        c1, _ = orc.pack("w4sb32", np.ldexp(W, e).astype(np.float32), a)
        blk1 = c1.reshape(3, 2, 144)
        assert np.array_equal(blk1[..., 4:], blk0[..., 4:])
        d0 = blk0[..., :4].copy().view(np.uint16)
        d1 = blk1[..., :4].copy().view(np.uint16)
        assert np.array_equal(orc.f16_bits_to_f32(d1), np.ldexp(orc.f16_bits_to_f32(d0), e))
    c2, _ = orc.pack("w4sb32", W, 8 * a)
    assert np.array_equal(c2, c0)


# ------------------------------------------- exact integer constructions ---
def designed_sym(rng, N, K, G, qmax, unit):
    q = rng.integers(-qmax, qmax + 1, size=(N, K))
    qg = q.reshape(N, K // G, G)
    qg[:, :, 0] = qmax * rng.choice([-1, 1], size=qg.shape[:2])   # absmax = qmax*unit
    return q, (q * unit).astype(np.float32)


@pytest.mark.parametrize("fmt,unit", [("w4g64", 2.0 ** -6), ("w8g16", 2.0 ** -10), ("w8g64", 2.0 ** -10),
                                      ("w6g16", 2.0 ** -8)])
@pytest.mark.parametrize("n_cand", [1, 64])
def test_exact_products_sym(orc, fmt, unit, n_cand):
    """w = q * 2^-e with each group's absmax at qmax * 2^-e: the scale is 2^-e
    exactly, codes come back exactly, and with small-integer x the product is
    an exact multiple of 2^-e known in integer arithmetic."""
    G, qmax = orc.GROUP[fmt], orc.QMAX[fmt]
    rng = np.random.default_rng(31)
    N, K, M = 24, 256, 3
    q, W = designed_sym(rng, N, K, G, qmax, unit)
    a = np.ones(K, np.float32)
    a[5] = 2500.0
    codes, scales = orc.pack(fmt, W, a, n_cand=n_cand)
    assert np.all(orc.f16_bits_to_f32(scales) == np.float32(unit))
    assert np.array_equal(orc.dequant(fmt, K, N, codes, scales), W)
    xi = rng.integers(-8, 9, size=(M, K))
    xb = (xi.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    y = orc.wgemm(fmt, xb, K, N, codes, scales)
    assert np.array_equal(y, (xi @ q.T).astype(np.float64) * unit)


def test_w6g16_bytes_follow_the_layout(orc):
    """The 6-bit symmetric codes, read back from the bytes by the layout's
    definition (per 64 weights: 32 bytes of low nibbles, even j in the low
    half of byte j/2; then bits 4..5 of u_j at bits 2 (j % 4) of byte
    32 + j/4), are u = q + 32 for weights built as q * 2^-8 with every
    group's absmax at 31 * 2^-8."""
    rng = np.random.default_rng(37)
    N, K = 6, 320
    q, W = designed_sym(rng, N, K, 16, 31, 2.0 ** -8)
    codes, scales = orc.pack("w6g16", W, None, n_cand=1)
    assert codes.shape == (N, K // 64 * 48)
    assert np.all(orc.f16_bits_to_f32(scales) == np.float32(2.0 ** -8))
    u = np.zeros((N, K), dtype=np.int64)
    for n in range(N):
        for k in range(K):
            ch = codes[n, (k // 64) * 48:(k // 64) * 48 + 48].astype(np.int64)
            j = k % 64
            lo = (ch[j // 2] >> (4 * (j % 2))) & 15
            hi = (ch[32 + j // 4] >> (2 * (j % 4))) & 3
            u[n, k] = lo + 16 * hi
    assert np.array_equal(u, q + 32)


def test_sym_bits_per_weight(orc):
    """Stored bits per weight: codes plus one fp16 scale per group."""
    K = N = 4096
    for fmt, bpw in [("w4g64", 4.25), ("w8g16", 9.0), ("w8g64", 8.25), ("w6g16", 7.0)]:
        assert packed_bytes(orc, fmt, K, N) * 8 / (K * N) == bpw


def test_exact_products_sb32(orc):
    """w = S_j (q - 8) with S_j = c_j 2^-12 (c_j <= 63, one group per
    superblock at 63) and codes spanning 0..15: the search's t = 1 candidate
    is exact, d = 2^-12 and dmin = 2^-9 exactly, sc_j = m_j = c_j, and the
    weights and the product come back exactly."""
    rng = np.random.default_rng(41)
    N, K, M = 6, 512, 2
    q = rng.integers(0, 16, size=(N, K))
    qg = q.reshape(N, K // 32, 32)
    qg[:, :, 0] = 0
    qg[:, :, 1] = 15
    c = rng.integers(1, 64, size=(N, K // 32))
    c.reshape(N, -1, 8)[:, :, 3] = 63
    S = c.repeat(32, axis=1).astype(np.float64) * 2.0 ** -12
    W = (S * (q - 8)).astype(np.float32)
    assert np.array_equal(W.astype(np.float64), S * (q - 8))
    codes, _ = orc.pack("w4sb32", W, None, n_cand=64)
    blk = codes.reshape(N, K // 256, 144)
    assert np.all(blk[..., 0:2].copy().view(np.uint16) == np.float16(2.0 ** -12).view(np.uint16))
    assert np.all(blk[..., 2:4].copy().view(np.uint16) == np.float16(2.0 ** -9).view(np.uint16))
    assert np.array_equal(orc.dequant("w4sb32", K, N, codes, None), W)
    xi = rng.integers(-8, 9, size=(M, K))
    xb = (xi.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    y = orc.wgemm("w4sb32", xb, K, N, codes, None)
    want = (xi[:, None, :] * (c.repeat(32, axis=1) * (q - 8))[None]).sum(-1) * 2.0 ** -12
    assert np.array_equal(y, want.astype(np.float64))


@pytest.mark.parametrize("fmt,bits", [("w5sb32", 5), ("w6sb32", 6)])
def test_exact_products_sb_wide(orc, fmt, bits):
    """5- and 6-bit superblocks: w = S_j (q - 2^(bits-1)) with S_j = c_j 2^-12
    (c_j <= 63, one group per superblock at 63) and codes spanning
    0..2^bits - 1: the t = 1 candidate is exact, d = 2^-12, dmin =
    2^(bits-13), sc_j = m_j = c_j, and weights and product come back exactly."""
    rng = np.random.default_rng(42 + bits)
    L, h = (1 << bits) - 1, 1 << (bits - 1)
    N, K, M = 5, 512, 2
    q = rng.integers(0, L + 1, size=(N, K))
    qg = q.reshape(N, K // 32, 32)
    qg[:, :, 0] = 0
    qg[:, :, 1] = L
    c = rng.integers(1, 64, size=(N, K // 32))
    c.reshape(N, -1, 8)[:, :, 5] = 63
    S = c.repeat(32, axis=1).astype(np.float64) * 2.0 ** -12
    W = (S * (q - h)).astype(np.float32)
    assert np.array_equal(W.astype(np.float64), S * (q - h))
    codes, _ = orc.pack(fmt, W, None, n_cand=64)
    blk = codes.reshape(N, K // 256, orc.SB_BYTES[fmt])
    assert np.all(blk[..., 0:2].copy().view(np.uint16) == np.float16(2.0 ** -12).view(np.uint16))
    assert np.all(blk[..., 2:4].copy().view(np.uint16) == np.float16(2.0 ** (bits - 13)).view(np.uint16))
    assert np.array_equal(orc.dequant(fmt, K, N, codes, None), W)
    # the stored codes decode to q: low nibbles plus the high-bit plane
    lo = np.stack([blk[..., 16:144] & 15, blk[..., 16:144] >> 4], -1).reshape(N, K // 256, 256)
    plane = blk[..., 144:]
    if bits == 5:
        up = np.unpackbits(plane, axis=-1, bitorder="little").reshape(N, K // 256, 256)
    else:
        up = np.stack([(plane >> (2 * i)) & 3 for i in range(4)], -1).reshape(N, K // 256, 256)
    assert np.array_equal((lo | (up << 4)).reshape(N, K), q)
    xi = rng.integers(-8, 9, size=(M, K))
    xb = (xi.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    y = orc.wgemm(fmt, xb, K, N, codes, None)
    want = (xi[:, None, :] * (c.repeat(32, axis=1) * (q - h))[None]).sum(-1) * 2.0 ** -12
    assert np.array_equal(y, want.astype(np.float64))


# ---------------------------------------- superblock fields, brute force ---
def test_sb_fields_and_codes_brute_force(orc):
    rng = np.random.default_rng(51)
    for rep in range(6):
        w = (rng.standard_normal(256) * 0.02).astype(np.float32)
        if rep == 1:
            w[:32] = np.abs(w[:32])                   # a group with lo = 0
        if rep == 2:
            w[32:64] = -np.abs(w[32:64])              # a group with hi = 0
        if rep == 3:
            w[64:96] = 0.0                            # an all-zero group
        a = np.ones(256, np.float32)
        a[rng.integers(256)] = 15631.0
        SM = [orc.asym_group(w[32 * j:32 * j + 32], a[32 * j:32 * j + 32], 64)[1:3] for j in range(8)]
        S_star = np.array([s for s, _ in SM], np.float32)
        M_star = np.array([m for _, m in SM], np.float32)
        blk = orc.sb_finish(w, S_star, M_star)
        d = f16(np.float32(S_star.max()) / np.float32(63))
        dm = f16(np.float32(M_star.max()) / np.float32(63))
        assert blk[0:2].copy().view(np.float16)[0] == np.float16(d)
        assert blk[2:4].copy().view(np.float16)[0] == np.float16(dm)
        bits = np.unpackbits(blk[4:16], bitorder="little")
        for j in range(8):
            sc = int((bits[6 * j:6 * j + 6] * (1 << np.arange(6))).sum())
            mc = int((bits[48 + 6 * j:54 + 6 * j] * (1 << np.arange(6))).sum())
            assert sc == orc.sb_field(blk, 0, j) and mc == orc.sb_field(blk, 1, j)
            want_sc = 0 if d == 0 else max(0, min(63, nearest_int_even(Fr(float(S_star[j])) / Fr(float(d)))))
            want_mc = 0 if dm == 0 else max(0, min(63, nearest_int_even(Fr(float(M_star[j])) / Fr(float(dm)))))
            assert (sc, mc) == (want_sc, want_mc)
            Sj, Mj = Fr(float(d)) * sc, Fr(float(dm)) * mc
            for k in range(32):
                kk = 32 * j + k
                qk = (blk[16 + kk // 2] >> (4 * (kk & 1))) & 0xF
                if Sj == 0:
                    assert qk == 0
                    continue
                v = (Fr(float(w[kk])) + Mj) / Sj
                if near_half(v):
                    continue
                assert qk == max(0, min(15, nearest_int_even(v)))


def brute_asym(w, a, t, levels=15):
    """Exact-rational loss of every candidate of the asymmetric reading
    (shrink [min(0,min w), max(0,max w)] about its midpoint by t_i; the step
    S = 2r/15 and offset M = max(0, r - mid) formed with numpy fp32 ops),
    codes the exact nearest integer in [0, 15]."""
    lo = np.float32(min(0.0, float(w.min())))
    hi = np.float32(max(0.0, float(w.max())))
    half = np.float32((hi - lo) * np.float32(0.5))
    mid = np.float32((hi + lo) * np.float32(0.5))
    out = []
    for ti in t:
        r = np.float32(np.float32(ti) * half)
        S = np.float32(np.float32(2.0) * r / np.float32(levels))
        loi = np.float32(mid - r)
        M = np.float32(-loi) if loi < 0 else np.float32(0.0)
        L = Fr(0)
        for wk, ak in zip(w, a):
            if S == 0:
                q = 0
            else:
                q = max(0, min(levels, nearest_int_even((Fr(float(wk)) + Fr(float(M))) / Fr(float(S)))))
            wh = Fr(float(np.float32(np.float32(q) * S) - M))
            L += Fr(float(ak)) * (Fr(float(wk)) - wh) ** 2
        out.append((L, float(S), float(M)))
    return out


@pytest.mark.parametrize("bits", [4, 5, 6])
@pytest.mark.parametrize("seed", range(6))
def test_asym_search_matches_exact_brute_force(orc, seed, bits):
    rng = np.random.default_rng(100 + seed)
    w = (rng.standard_normal(32) * 0.02).astype(np.float32)
    if seed == 1:
        w = np.abs(w)
    if seed == 2:
        w[3] *= 12
    a = np.ones(32, np.float32)
    if seed % 2:
        a[rng.integers(32)] = 15631.0
    t = orc.grid(64)
    idx, S, M, _ = orc.asym_group(w, a, 64, bits=bits)
    bl = brute_asym(w, a, t, (1 << bits) - 1)
    bidx = min(range(64), key=lambda i: (bl[i][0], i))
    if idx != bidx:
        assert abs(bl[idx][0] - bl[bidx][0]) <= Fr(1, 10**12) * bl[bidx][0]
    assert (S, M) == (bl[idx][1], bl[idx][2])


@pytest.mark.parametrize("bits", [4, 5, 6])
def test_asym_t1_covers_the_group_range(orc, bits):
    """With the single candidate t = 1 the representable range [-M, L S - M]
    (L = 2^bits - 1) covers [min(0, min w), max(0, max w)] and every weight is
    within S/2 (plus fp32 rounding) of its dequantized value."""
    rng = np.random.default_rng(61)
    L = (1 << bits) - 1
    for rep in range(50):
        w = (rng.standard_normal(32) * 0.02 * (1 + rep)).astype(np.float32)
        _, S, M, _ = orc.asym_group(w, None, 1, bits=bits)
        lo, hi = min(0.0, float(w.min())), max(0.0, float(w.max()))
        assert -M <= lo * (1 - 1e-6) + 1e-12 and L * S - M >= hi * (1 - 1e-6) - 1e-12
        for wk in w:
            q = max(0, min(L, round((float(wk) + M) / S)))
            assert abs(float(wk) - (S * q - M)) <= S / 2 * (1 + 1e-5)


# ------------------------------------------------ reduction to a library ----
@pytest.mark.parametrize("fmt", ["w4g64", "w8g16", "w4sb32", "w8g64", "w6g16", "w5sb32"])
def test_product_matches_numpy_matmul(orc, fmt):
    rng = np.random.default_rng(71)
    N, K, M = 40, 768, 5
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    codes, scales = orc.pack(fmt, W, None, n_cand=8)
    Wd = orc.dequant(fmt, K, N, codes, scales).astype(np.float64)
    x = rng.standard_normal((M, K)).astype(np.float32)
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    xf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    y = orc.wgemm(fmt, xb, K, N, codes, scales)
    ref = xf @ Wd.T
    bound = 1e-13 * (np.abs(xf) @ np.abs(Wd).T) + 1e-300
    assert np.all(np.abs(y - ref) <= bound)
    rows = np.array([39, 0, 7], dtype=np.int32)
    assert np.array_equal(orc.wgemm(fmt, xb, K, N, codes, scales, rows=rows), y[:, rows])


# ---------------------------------------------------- the pages' sizes -----
def packed_bytes(orc, fmt, K, N):
    cs, _, ss = orc.packed_shapes(fmt, K, N)
    return cs[0] * cs[1] + (0 if ss is None else 2 * ss[0] * ss[1])


def test_format_sizes_match_the_pages(orc):
    g = json.load(open(os.path.join(GOLD, "format_sizes.json")))
    c = g["w4sb32_o_proj_bf16_delta"]
    delta = c["K"] * c["N"] * 2 - packed_bytes(orc, "w4sb32", c["K"], c["N"])
    assert round(delta / 1e6, c["decimals"]) == c["delta_MB"]
    c = g["w4sb32_all_o_proj_plus_bits"]
    per_bit = c["layers"] * c["K"] * c["N"] / 8
    assert round(per_bit / 1e6, 1) == c["plus_1bit_MB"]
    assert round(2 * per_bit / 1e6, 1) == c["plus_2bit_MB"]
    # the 5- and 6-bit superblock records carry exactly those deltas
    base = packed_bytes(orc, "w4sb32", c["K"], c["N"])
    d5 = c["layers"] * (packed_bytes(orc, "w5sb32", c["K"], c["N"]) - base)
    d6 = c["layers"] * (packed_bytes(orc, "w6sb32", c["K"], c["N"]) - base)
    assert round(d5 / 1e6, c["decimals"]) == c["plus_1bit_MB"]
    assert round(d6 / 1e6, c["decimals"]) == c["plus_2bit_MB"]
    c = g["w4sb32_first_o_proj_range"]
    for C in c["widths"]:
        d = C * C * 2 - packed_bytes(orc, "w4sb32", C, C)
        assert c["lo_MB"] <= d / 1e6 <= c["hi_MB"]
    c = g["w4g64_checkpoint_1p5b"]
    C, L, V = c["C"], c["layers"], c["vocab"]
    proj = [(C, C)] * 4 + [(C, 4 * C), (4 * C, C)]
    fp16 = L * sum(k * n for k, n in proj) * 2 + 2 * V * C * 2
    int4 = L * sum(packed_bytes(orc, "w4g64", k, n) for k, n in proj) + 2 * V * C * 2
    assert abs(fp16 / 1e9 - c["fp16_GB"]) <= c["rel_tol"] * c["fp16_GB"]
    assert abs(int4 / 1e9 - c["int4_GB"]) <= c["rel_tol"] * c["int4_GB"]


# ----------------------------------------------------- E[x^2] statistic ---
def _bf16_bits(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


@pytest.mark.parametrize("R", [1, 3, 64, 65, 128, 1000])
def test_act_stats_constant_rows(orc, R):
    """Rows all equal to c (exact in bf16): E[x^2] = c^2 exactly."""
    K = 5
    c = np.array([1.5, -2.0, 0.0, 3.25, -0.125], np.float32)
    x = np.tile(c, (R, 1))
    got = orc.act_finalize(orc.act_sumsq(_bf16_bits(x)), R)
    assert np.array_equal(got, (c.astype(np.float64) ** 2).astype(np.float32))


def test_act_stats_integer_rows_exact(orc):
    """Small-integer activations: every partial sum is an exact integer in
    fp64, so the result is the integer sum of squares over R, rounded once."""
    rng = np.random.default_rng(31)
    R, K = 4097, 67
    xi = rng.integers(-40, 41, size=(R, K))
    s = orc.act_sumsq(_bf16_bits(xi.astype(np.float32)))
    assert np.array_equal(s, (xi.astype(np.int64) ** 2).sum(0).astype(np.float64))
    assert np.array_equal(orc.act_finalize(s, R), ((xi.astype(np.int64) ** 2).sum(0) / R).astype(np.float32))


def test_act_stats_match_numpy_and_accumulate(orc):
    """Random bf16 activations with a massive channel: the fp64 sums agree
    with numpy's to 1e-12, and two batches accumulate to the one-shot sum."""
    rng = np.random.default_rng(32)
    R, K = 1000, 96
    x = rng.standard_normal((R, K)).astype(np.float32)
    x[:, 7] *= 50.0
    b = _bf16_bits(x)
    xf = (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = (xf ** 2).sum(0)
    s = orc.act_sumsq(b)
    assert np.allclose(s, ref, rtol=1e-12, atol=0)
    s2 = orc.act_sumsq(b[600:], orc.act_sumsq(b[:600]))
    assert np.allclose(s2, ref, rtol=1e-12, atol=0)
    a = orc.act_finalize(s, R)
    assert np.allclose(a, (ref / R).astype(np.float32), rtol=1e-6, atol=0)
    assert int(np.argmax(a)) == 7


# ------------------------------------------------------------------ GPTQ ---
def test_hessian_accum_exact_integers(orc):
    """Small-integer bf16 rows: every product and sum is an exact integer, so
    H must equal the integer x^T x, and two calls accumulate."""
    rng = np.random.default_rng(61)
    x = rng.integers(-9, 10, size=(37, 24))
    xb = _bf16_bits(x.astype(np.float32))
    H = orc.hessian_accum(xb)
    assert np.array_equal(H, (x.T @ x).astype(np.float64))
    H2 = orc.hessian_accum(xb[20:], orc.hessian_accum(xb[:20]))
    assert np.array_equal(H2, H)


def _sym_codes_np(w32, sf, qmax):
    if sf == 0.0:
        return np.zeros_like(w32, dtype=np.int64)
    v = (w32 / np.float32(sf)).astype(np.float32)
    return np.rint(np.clip(v, -qmax, qmax)).astype(np.int64)


def _gptq_by_obs(orc, fmt, W, H, a, n_cand, damp=0.01):
    """GPTQ written a second way: after quantizing column k, the not yet
    quantized columns F = k+1.. move by the optimal-brain-surgeon update
    computed from the damped Hessian restricted to {k} u F (an explicit
    inverse of that block; no Cholesky factor)."""
    G, qmax = orc.GROUP[fmt], orc.QMAX[fmt]
    N, K = W.shape
    Hd = np.array(H, dtype=np.float64, copy=True)
    dead = np.diag(Hd) == 0
    Hd[dead, dead] = 1.0
    Hd[np.arange(K), np.arange(K)] += damp * np.mean(np.diag(Hd))
    codes = np.zeros((N, K), np.int64)
    scales = np.zeros((N, K // G), np.uint16)
    for n in range(N):
        w = W[n].astype(np.float64)
        w[dead] = 0.0
        for g in range(K // G):
            k0 = g * G
            _, s, _, _ = orc.sym_group(w[k0:k0 + G].astype(np.float32), None if a is None else a[k0:k0 + G],
                                       qmax, n_cand)
            scales[n, g] = s
            sf = float(orc.f16_bits_to_f32(np.array([s], np.uint16))[0])
            for k in range(k0, k0 + G):
                q = int(_sym_codes_np(np.array([w[k]], np.float32), sf, qmax)[0])
                codes[n, k] = q
                e = w[k] - float(np.float32(q) * np.float32(sf))
                Hinv = np.linalg.inv(Hd[k:, k:])
                w[k:] -= e * Hinv[:, 0] / Hinv[0, 0]
    return codes, scales


@pytest.mark.parametrize("fmt", ["w4g64", "w8g16", "w6g16"])
def test_gptq_matches_sequential_obs(orc, fmt):
    rng = np.random.default_rng(67)
    N, K, R = 3, 128, 400
    mix = rng.standard_normal((K, K)) * 0.3 + np.eye(K)       # correlated channels
    x = (rng.standard_normal((R, K)) @ mix).astype(np.float32)
    xb = _bf16_bits(x)
    H = orc.hessian_accum(xb)
    a = (np.diag(H) / R).astype(np.float32)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    U, dead = orc.gptq_prepare(H)
    codes, scales = orc.gptq_pack(fmt, W, U, dead, a, n_cand=16)
    q_ref, s_ref = _gptq_by_obs(orc, fmt, W, H, a, 16)
    assert np.array_equal(scales, s_ref)
    wd = orc.dequant(fmt, K, N, codes, scales).astype(np.float64)
    sf = orc.f16_bits_to_f32(s_ref).reshape(N, -1).astype(np.float64).repeat(orc.GROUP[fmt], axis=1)
    assert np.array_equal(wd, q_ref * sf)


@pytest.mark.parametrize("fmt", ["w4g64", "w8g64"])
def test_gptq_diagonal_hessian_is_the_preset_pack(orc, fmt):
    """Uncorrelated channels (diagonal H): U is diagonal, no column moves, and
    GPTQ gives the preset pack's bytes; a dead channel's weights become 0."""
    rng = np.random.default_rng(71)
    N, K = 5, 256
    d = rng.random(K) * 3 + 0.5
    d[7] = 0.0                                               # a channel that never fires
    H = np.diag(d)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    a = rng.random(K).astype(np.float32) + 0.1
    U, dead = orc.gptq_prepare(H)
    assert np.count_nonzero(np.triu(U, 1)) == 0 and dead[7] == 1 and dead.sum() == 1
    c1, s1 = orc.gptq_pack(fmt, W, U, dead, a, n_cand=32)
    W0 = W.copy()
    W0[:, 7] = 0.0
    c0, s0 = orc.pack(fmt, W0, a, n_cand=32)
    assert np.array_equal(c1, c0) and np.array_equal(s1, s0)


def test_gptq_lowers_the_output_error(orc):
    """On strongly correlated inputs GPTQ's output error
    tr((W - W_hat) H (W - W_hat)^T) is well below the per-group search's."""
    rng = np.random.default_rng(73)
    N, K, R = 16, 256, 600
    basis = rng.standard_normal((24, K))
    x = (rng.standard_normal((R, 24)) @ basis + 0.05 * rng.standard_normal((R, K))).astype(np.float32)
    H = orc.hessian_accum(_bf16_bits(x))
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    U, dead = orc.gptq_prepare(H)
    cg, sg = orc.gptq_pack("w4g64", W, U, dead, None, n_cand=1)
    cr, sr = orc.pack("w4g64", W, None, n_cand=1)
    def out_err(c, s):
        D = W.astype(np.float64) - orc.dequant("w4g64", K, N, c, s).astype(np.float64)
        return float(np.einsum("nk,kl,nl->", D, H, D))
    assert out_err(cg, sg) < 0.7 * out_err(cr, sr)


def _gptq_sb_by_obs(orc, fmt, W, H, a, n_cand, damp=0.01):
    """Superblock GPTQ written the second way (explicit inverse of the
    trailing Hessian block): returns w_hat [N][K] and the records' headers."""
    bits = orc.SB_BITS[fmt]
    L = (1 << bits) - 1
    N, K = W.shape
    Hd = np.array(H, dtype=np.float64, copy=True)
    dead = np.diag(Hd) == 0
    Hd[dead, dead] = 1.0
    Hd[np.arange(K), np.arange(K)] += damp * np.mean(np.diag(Hd))
    what = np.zeros((N, K), np.float64)
    headers = np.zeros((N, K // 256, 16), np.uint8)
    for n in range(N):
        w = W[n].astype(np.float64)
        w[dead] = 0.0
        for b in range(K // 256):
            k0 = 256 * b
            wsb = w[k0:k0 + 256].astype(np.float32)
            S = np.zeros(8, np.float32)
            M = np.zeros(8, np.float32)
            for j in range(8):
                _, S[j], M[j], _ = orc.asym_group(wsb[32 * j:32 * j + 32],
                                                  None if a is None else a[k0 + 32 * j:k0 + 32 * j + 32],
                                                  n_cand, bits=bits)
            blk = orc.sb_finish(wsb, S, M, bits)
            headers[n, b] = blk[:16]
            d, dm = orc.f16_bits_to_f32(blk[:4].copy().view(np.uint16))
            for i in range(256):
                k = k0 + i
                Sj = np.float32(d * np.float32(orc.sb_field(blk, 0, i // 32)))
                Mj = np.float32(dm * np.float32(orc.sb_field(blk, 1, i // 32)))
                if Sj == 0:
                    q = 0
                else:
                    v = np.float32(np.float32(np.float32(w[k]) + Mj) / Sj)
                    q = int(np.rint(np.clip(v, np.float32(0), np.float32(L))))
                wq = float(np.float32(np.float32(np.float32(q) * Sj) - Mj))
                what[n, k] = wq
                e = w[k] - wq
                Hinv = np.linalg.inv(Hd[k:, k:])
                w[k:] -= e * Hinv[:, 0] / Hinv[0, 0]
    return what, headers


@pytest.mark.parametrize("fmt", ["w4sb32", "w5sb32", "w6sb32"])
def test_gptq_sb_matches_sequential_obs(orc, fmt):
    rng = np.random.default_rng(79)
    N, K, R = 2, 512, 900
    mix = rng.standard_normal((K, K)) * 0.2 + np.eye(K)
    x = (rng.standard_normal((R, K)) @ mix).astype(np.float32)
    H = orc.hessian_accum(_bf16_bits(x))
    a = (np.diag(H) / R).astype(np.float32)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    U, dead = orc.gptq_prepare(H)
    codes, _ = orc.gptq_pack(fmt, W, U, dead, a, n_cand=16)
    what, headers = _gptq_sb_by_obs(orc, fmt, W, H, a, 16)
    rs = orc.SB_BYTES[fmt]
    assert np.array_equal(codes.reshape(N, K // 256, rs)[:, :, :16], headers)
    assert np.array_equal(orc.dequant(fmt, K, N, codes, None).astype(np.float64), what)


@pytest.mark.parametrize("fmt", ["w4sb32", "w6sb32"])
def test_gptq_sb_diagonal_hessian_is_the_preset_pack(orc, fmt):
    rng = np.random.default_rng(83)
    N, K = 3, 512
    d = rng.random(K) * 3 + 0.5
    d[300] = 0.0
    U, dead = orc.gptq_prepare(np.diag(d))
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    a = rng.random(K).astype(np.float32) + 0.1
    c1, _ = orc.gptq_pack(fmt, W, U, dead, a, n_cand=32)
    W0 = W.copy()
    W0[:, 300] = 0.0
    c0, _ = orc.pack(fmt, W0, a, n_cand=32)
    assert np.array_equal(c1, c0)
