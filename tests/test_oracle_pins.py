"""Pins for the CPU oracle: what the pages and the mathematics fix, checked by
means other than re-running the oracle's own formulas.

  * exhaustive brute-force nearest-grid search (ties to the even code) for E2M1,
  * torch's float8_e4m3fn cast (a library routine) and brute force for E4M3,
  * closed-form tie points, grid membership, the per-element error bound,
  * brute-force quantization of tiny tensors (searches, not format rounding),
  * round trips of grid-valued blocks, zero tensors, storage-ratio closed forms,
  * one-hot products and a float64 library matmul for the GEMMs.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_gemm_quantize_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_facts.json")))

# E2M1 magnitudes in code order (1 sign, 2 exponent, 1 mantissa bit): the set a
# 1-2-1 binary float can hold.  The test below checks it against the page.
E2M1_GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]

# All E4M3FN values, decoded by torch (library routine).
_E4M3_ALL = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
E4M3_POS = [(c, _E4M3_ALL[c]) for c in range(0x7F)]      # codes 0x00..0x7E, non-negative finite


def brute_e2m1(q: float) -> int:
    """Nearest E2M1 magnitude by exhaustive search, ties to the even code,
    sign copied from q; |q| above 6 clips to 6."""
    m = abs(Fraction(float(q)))
    best, bestd = None, None
    for c, v in enumerate(E2M1_GRID):
        d = abs(m - Fraction(v))
        if bestd is None or d < bestd or (d == bestd and c % 2 == 0):
            best, bestd = c, d
    sign = 8 if np.signbit(q) else 0
    return sign | best


def brute_e4m3(v: float) -> int:
    """Nearest non-negative finite E4M3 value by search, ties to the even code,
    saturating at 448."""
    m = Fraction(float(v))
    best, bestd = None, None
    for c, val in E4M3_POS:
        d = abs(m - Fraction(val))
        if bestd is None or d < bestd or (d == bestd and c % 2 == 0):
            best, bestd = c, d
    return best


# ------------------------------------------------------------------ E2M1
def test_e2m1_bit_split_and_grid_against_page():
    vals = [oracle.e2m1_decode(c) for c in range(16)]
    bits = GOLD["e2m1_bits"]["value"]
    assert bits["sign"] + bits["exponent"] + bits["mantissa"] == 4
    assert len(vals) == 2 ** 4
    listed = set(GOLD["e2m1_listed_magnitudes"]["value"])
    mags = sorted({abs(v) for v in vals})
    # every non-zero magnitude of the format is on the page's list
    assert set(m for m in mags if m != 0) <= listed
    # 8 distinct magnitudes, sign bit is bit 3, max is the clip value
    assert len(mags) == 8
    assert max(mags) == GOLD["clip_range"]["value"][1]
    for c in range(8):
        assert vals[c + 8] == -vals[c]
    assert [abs(v) for v in vals[:8]] == E2M1_GRID


def test_e2m1_encode_exhaustive_bf16_patterns():
    """Every bf16 bit pattern read as a quotient q: oracle == brute force."""
    pats = np.arange(65536, dtype=np.uint32)
    qs = (pats << 16).view(np.float32)
    L = oracle.lib()
    for q in qs:
        if np.isnan(q):
            continue
        got = L.oracle_e2m1_encode(float(q))
        if np.isinf(q):
            assert got == (15 if q < 0 else 7)
            continue
        assert got == brute_e2m1(q), (q, got)


def test_e2m1_encode_fp32_near_thresholds():
    """fp32 values within a few ulps of every rounding threshold and grid point."""
    L = oracle.lib()
    pts = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for p in pts:
        base = int(np.array([p], np.float32).view(np.uint32)[0])
        for d in range(-6, 7):
            q = np.array([base + d], np.uint32).view(np.float32)[0]
            for sq in (q, -q):
                assert L.oracle_e2m1_encode(float(sq)) == brute_e2m1(sq), sq


def test_e2m1_tie_points_closed_form():
    # midpoints go to the even code: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    expect = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for t, v in expect.items():
        assert oracle.e2m1_decode(oracle.e2m1_encode(t)) == v
        assert oracle.e2m1_decode(oracle.e2m1_encode(-t)) == -v
    # clipping to [-6, 6]
    assert oracle.e2m1_decode(oracle.e2m1_encode(6.375)) == 6.0
    assert oracle.e2m1_decode(oracle.e2m1_encode(-1e30)) == -6.0
    # sign of zero results follows x
    assert oracle.e2m1_encode(-0.1) == 0x8
    assert oracle.e2m1_encode(0.1) == 0x0


# ------------------------------------------------------------------ E4M3
def test_e4m3_decode_matches_library_cast():
    for c in range(256):
        o = oracle.e4m3_decode(c)
        t = _E4M3_ALL[c]
        if np.isnan(t):
            assert np.isnan(o)
        else:
            assert o == t, c


def test_e4m3_roundtrip_all_finite_codes():
    for c, v in E4M3_POS:
        assert oracle.e4m3_encode(v) == c


def test_e4m3_encode_vs_library_and_brute_force():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        np.exp(rng.uniform(np.log(2.0 ** -12), np.log(440.0), 4000)),
        # midpoints between neighbours (ties) and one ulp either side
        [(E4M3_POS[i][1] + E4M3_POS[i + 1][1]) / 2 for i in range(len(E4M3_POS) - 1)],
    ]).astype(np.float32)
    more = []
    for v in vals[-(len(E4M3_POS) - 1):]:
        u = int(np.array([v], np.float32).view(np.uint32)[0])
        more += [np.array([u - 1], np.uint32).view(np.float32)[0], np.array([u + 1], np.uint32).view(np.float32)[0]]
    vals = np.concatenate([vals, np.array(more, np.float32)])
    lib_codes = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for v, lc in zip(vals, lib_codes):
        oc = oracle.e4m3_encode(v)
        assert oc == brute_e4m3(v), v
        if v <= 448.0:
            assert oc == lc, (v, oc, lc)


def test_e4m3_saturates():
    for v in (448.0, 460.0, 464.0, 480.0, 1e6, 3.0e38, float("inf")):
        assert oracle.e4m3_encode(v) == 0x7E
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_encode(2.0 ** -10) == 0       # tie between 0 and 2^-9 -> even (0)
    assert oracle.e4m3_encode(1.5 * 2.0 ** -10) == 1


# ------------------------------------------------------------------ bf16
def test_bf16_rounding_vs_search():
    rng = np.random.default_rng(1)
    # doubles with up to 30 significant bits, like the exact dequantized products
    m = rng.integers(1 << 29, 1 << 30, 3000).astype(np.float64)
    e = rng.integers(-150, 100, 3000)
    vals = np.ldexp(m, e - 29) * rng.choice([-1.0, 1.0], 3000)
    allbf = (np.arange(0x7F81, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)
    for v in vals:
        got = oracle.bf16_from_double(v)
        a = Fraction(abs(v))
        # search the two positive bf16 neighbours of |v|
        f = np.float32(abs(v))
        u = int(np.array([f], np.float32).view(np.uint32)[0] >> 16)
        cands = [c for c in (u - 1, u, u + 1, u + 2) if 0 <= c < 0x7F81]
        best = min(cands, key=lambda c: (abs(a - Fraction(float(allbf[c]))), c % 2))
        if np.signbit(v):
            best |= 0x8000
        assert got == best, v


# ------------------------------------------------------------------ SF layout
def test_sf_offset_bijection_and_hand_values():
    rows, k = 256, 128
    kb = k // 16
    seen = set()
    for r in range(rows):
        for c in range(kb):
            seen.add(oracle.sf_offset(r, c, kb))
    assert seen == set(range(oracle.sf_bytes(rows, k)))
    # hand-derived: atom = 128 rows x 4 blocks = 512 bytes, line r%32, word (r%128)/32, byte c%4
    assert oracle.sf_offset(0, 0, kb) == 0
    assert oracle.sf_offset(0, 1, kb) == 1
    assert oracle.sf_offset(1, 0, kb) == 16
    assert oracle.sf_offset(32, 0, kb) == 4
    assert oracle.sf_offset(127, 3, kb) == 31 * 16 + 3 * 4 + 3
    assert oracle.sf_offset(0, 4, kb) == 512
    assert oracle.sf_offset(128, 0, kb) == 2 * 512
    assert oracle.sf_bytes(600, 4096) == 640 * 256


def test_sf_matrix_helper_agrees_with_offset():
    rows, k = 300, 192
    rng = np.random.default_rng(2)
    sf = rng.integers(0, 256, oracle.sf_bytes(rows, k)).astype(np.uint8)
    mat = oracle.sf_matrix(sf, rows, k)
    for r in range(0, rows, 7):
        for c in range(k // 16):
            assert mat[r, c] == sf[oracle.sf_offset(r, c, k // 16)]


# ------------------------------------------------------------------ quantize
def brute_quantize(xf32: np.ndarray, scale=None):
    """Quantize by searches: g from amax, sf by nearest-E4M3 search, codes by
    nearest-E2M1 search, every product/quotient a single fp32 rounding."""
    rows, k = xf32.shape
    f = np.float32
    if scale is None:
        amax = f(np.max(np.abs(xf32))) if xf32.size else f(0)
        g = f(amax / f(2688.0))
    else:
        g = f(scale)
    d = f(f(6.0) * g)
    codes = np.zeros((rows, k), np.uint8)
    sfm = np.zeros((rows, k // 16), np.uint8)
    for r in range(rows):
        for c in range(k // 16):
            blk = xf32[r, 16 * c:16 * c + 16]
            ab = f(np.max(np.abs(blk)))
            sfc = brute_e4m3(f(ab / d)) if d > 0 else 0
            sfm[r, c] = sfc
            s = f(f(_E4M3_ALL[sfc]) * g)
            for i in range(16):
                codes[r, 16 * c + i] = brute_e2m1(f(blk[i] / s)) if s != 0 else 0
    return codes, sfm, g


@pytest.mark.parametrize("case", range(10))
def test_quantize_vs_brute_force_tiny(case):
    rng = np.random.default_rng(100 + case)
    rows, k = [(1, 64), (3, 64), (2, 128), (5, 64), (4, 192)][case % 5]
    x = rng.standard_normal((rows, k)).astype(np.float32)
    if case % 3 == 1:
        x *= np.exp(rng.uniform(-8, 8, (rows, 1))).astype(np.float32)   # wide dynamic range
    if case % 4 == 2:
        x[:, rng.integers(0, k, 3)] = 0.0
        x[0, :16] = 0.0                                                  # an all-zero block
    if case % 5 == 3:
        x[1, 5] = -0.0
        x[2, 7] = -1e-6                                                  # negative -> code 0x8
    xb = torch.from_numpy(x).to(torch.bfloat16)
    xf = xb.float().numpy()
    scale = None if case < 7 else float(np.float32(np.max(np.abs(xf)) / 2000.0))
    codes, sf, g = oracle.quantize(xb, scale)
    bc, bsf, bg = brute_quantize(xf, scale)
    assert np.float32(g) == bg
    assert np.array_equal(oracle.unpack_codes(codes), bc)
    assert np.array_equal(oracle.sf_matrix(sf, rows, k), bsf)


def _grid_checks(xb, codes, sf, g):
    """grid membership and the half-spacing error bound, per element."""
    xf = xb.float().numpy().astype(np.float64)
    rows, k = xf.shape
    deq = oracle.dequantize(codes, sf, g, "f64")
    sfm = oracle.sf_matrix(sf, rows, k)
    s = np.repeat(_E4M3_ALL[sfm], 16, axis=1) * np.float64(np.float32(g))
    s32 = np.repeat(np.float32(_E4M3_ALL[sfm]) * np.float32(g), 16, axis=1).astype(np.float64)
    nz = s32 > 0
    ratio = np.where(nz, deq / np.where(nz, s, 1.0), 0.0)
    grid = set(E2M1_GRID) | {-v for v in E2M1_GRID}
    assert set(np.unique(ratio)) <= grid
    # error bound: spacing of the grid interval that holds |q|
    q = np.abs(xf) / np.where(nz, s32, 1.0)
    spacing = np.where(q < 2, 0.5, np.where(q < 4, 1.0, 2.0))
    err = np.abs(xf - deq)
    # |x - code*s| <= s*spacing/2 inside the grid, |x| - 6s when clipped; the
    # fp32 quotient and the fp32 scale each add at most 2^-23 relative to |x|.
    bound = np.where(q <= 6, s * spacing / 2, np.abs(xf) - 6 * s)
    assert np.all(~nz | (err <= bound + 2.0 ** -21 * np.abs(xf)))
    return deq


@pytest.mark.parametrize("dist", ["normal", "student_t3", "outlier", "token_scaled"])
def test_quantize_grid_membership_and_error_bound(dist):
    xb = synth.random_bf16((256, 1024), seed=7, dist=dist)
    codes, sf, g = oracle.quantize(xb)
    _grid_checks(xb, codes, sf, g)


def test_block_scale_never_exceeds_e4m3_range_and_scale_relation():
    xb = synth.random_bf16((128, 512), seed=8, dist="student_t3")
    codes, sf, g = oracle.quantize(xb)
    amax = np.float32(np.max(np.abs(xb.float().numpy())))
    assert g == np.float32(amax / np.float32(2688.0))
    sfm = oracle.sf_matrix(sf, 128, 512)
    assert sfm.max() <= 0x7E
    # the largest block scale is the one of the block holding amax: E4M3(amax / (6 g)) ~ 448
    assert _E4M3_ALL[sfm.max()] == 448.0


def test_grid_valued_blocks_round_trip_exactly():
    """Blocks of grid values times 2^m, with a power-of-two tensor scale, come
    back unchanged: s = 2^m exactly, so every quotient is on the grid."""
    rng = np.random.default_rng(3)
    rows, k = 8, 128
    vals = np.array(E2M1_GRID + [-v for v in E2M1_GRID[1:]], np.float64)
    x = rng.choice(vals, (rows, k))
    m = rng.integers(-12, 1, (rows, k // 16))     # block scale 2^(m+8) stays in E4M3 range
    for r in range(rows):
        for c in range(k // 16):
            x[r, 16 * c] = 6.0                       # block amax = 6 * 2^m
            x[r, 16 * c:16 * c + 16] *= 2.0 ** m[r, c]
    xb = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(xb.float().numpy(), x.astype(np.float32))
    codes, sf, g = oracle.quantize(xb, scale=2.0 ** -8)
    deq = oracle.dequantize(codes, sf, g, "f64")
    assert np.array_equal(deq, x)


def test_zero_tensor():
    xb = torch.zeros(130, 64, dtype=torch.bfloat16)
    codes, sf, g = oracle.quantize(xb)
    assert g == 0.0 and not codes.any() and not sf.any()
    assert not oracle.dequantize(codes, sf, g, "f64").any()


def test_storage_ratios_from_page():
    rows, k = 4096, 4096
    total = rows * k // 2 + oracle.sf_bytes(rows, k) + 4
    bits = total * 8 / (rows * k)
    assert abs(bits - 4.5) < 1e-5
    assert round(16 / bits, 1) == GOLD["memory_reduction_vs_fp16"]["value"] + 0.1 or \
        abs(16 / bits - GOLD["memory_reduction_vs_fp16"]["value"]) < 0.1
    assert abs(8 / bits - GOLD["memory_reduction_vs_fp8"]["value"]) < 0.05
    assert 16 / (8 / GOLD["packed_codes_per_byte"]["value"]) == GOLD["packed_memory_reduction_vs_fp16"]["value"]


def test_relative_error_next_to_page_bound():
    """Lemma III.2 states eps = 2^-3.  The tensor-level relative error on
    Gaussian and heavy-tailed inputs stays below it (the per-element worst case
    of the format does not, see the design notes)."""
    eps = GOLD["eps_fp4"]["value"]
    for dist in ("normal", "student_t3"):
        xb = synth.random_bf16((512, 1024), seed=9, dist=dist)
        codes, sf, g = oracle.quantize(xb)
        deq = oracle.dequantize(codes, sf, g, "f64")
        xf = xb.float().numpy().astype(np.float64)
        rel = np.linalg.norm(xf - deq) / np.linalg.norm(xf)
        assert rel < eps, (dist, rel)


# ------------------------------------------------------------------ dequantize
def test_dequantize_roundings():
    xb = synth.random_bf16((64, 256), seed=10, dist="student_t3")
    codes, sf, g = oracle.quantize(xb)
    d64 = oracle.dequantize(codes, sf, g, "f64")
    d32 = oracle.dequantize(codes, sf, g, "f32")
    db = oracle.dequantize(codes, sf, g, "bf16")
    assert np.array_equal(d32, d64.astype(np.float32))            # library double->float (RNE)
    for v, b in zip(d64.ravel()[:4000], db.ravel()[:4000]):
        assert b == oracle.bf16_from_double(v)


# ------------------------------------------------------------------ GEMM
def _zero_operand(rows, k):
    return np.zeros((rows, k // 2), np.uint8), np.zeros(oracle.sf_bytes(rows, k), np.uint8)


@pytest.mark.parametrize("m0,n0,k0", [(0, 0, 0), (5, 3, 17), (127, 130, 63), (64, 255, 100)])
def test_gemm_one_hot(m0, n0, k0):
    M, N, K = 128, 256, 128
    ac, asf = _zero_operand(M, K)
    bc, bsf = _zero_operand(N, K)
    ca, cb = 0x3, 0xB           # 1.5 and -1.5
    ac[m0, k0 // 2] = ca << (4 * (k0 & 1))
    bc[n0, k0 // 2] = cb << (4 * (k0 & 1))
    asf[oracle.sf_offset(m0, k0 // 16, K // 16)] = 0x40     # 2.0
    bsf[oracle.sf_offset(n0, k0 // 16, K // 16)] = 0x30     # 0.5
    ga, gb = 0.25, 3.0
    y = oracle.gemm_w4a4(ac, asf, ga, bc, bsf, gb)
    expect = np.zeros((M, N))
    expect[m0, n0] = ga * gb * (1.5 * 2.0) * (-1.5 * 0.5)
    assert np.array_equal(y, expect)
    # mismatched k positions give zero everywhere
    bc2, _ = _zero_operand(N, K)
    k1 = (k0 + 1) % K
    bc2[n0, k1 // 2] = cb << (4 * (k1 & 1))
    bsf2 = bsf.copy()
    bsf2[oracle.sf_offset(n0, k1 // 16, K // 16)] = 0x30
    assert not oracle.gemm_w4a4(ac, asf, ga, bc2, bsf2, gb).any()


def test_gemm_vs_library_matmul():
    x = synth.random_bf16((96, 320), seed=11, dist="outlier")
    w = synth.random_bf16((160, 320), seed=12, scale=0.02)
    ac, asf, ga = oracle.quantize(x)
    bc, bsf, gb = oracle.quantize(w)
    y = oracle.gemm_w4a4(ac, asf, ga, bc, bsf, gb)
    da = torch.from_numpy(oracle.dequantize(ac, asf, ga, "f64"))
    db = torch.from_numpy(oracle.dequantize(bc, bsf, gb, "f64"))
    ref = (da @ db.T).numpy()
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # single-element and row-slice entry points agree with the full product
    assert oracle.gemm_w4a4_at(ac, asf, ga, bc, bsf, gb, 17, 33) == pytest.approx(y[17, 33], rel=1e-13, abs=1e-300)
    assert np.allclose(oracle.gemm_w4a4(ac, asf, ga, bc, bsf, gb, rows=slice(10, 20)), y[10:20], rtol=1e-13)


def test_gemm_w4a16_vs_library_matmul():
    x = synth.random_bf16((64, 256), seed=13)
    w = synth.random_bf16((96, 256), seed=14, scale=0.015)
    wc, wsf, gw = oracle.quantize(w)
    y = oracle.gemm_w4a16(x, wc, wsf, gw)
    dw = torch.from_numpy(oracle.dequantize(wc, wsf, gw, "f64"))
    ref = (x.double() @ dw.T).numpy()
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    xb = oracle.bf16_bits(x)
    assert oracle.gemm_w4a16_at(xb, wc, wsf, gw, 5, 7) == pytest.approx(y[5, 7], rel=1e-13)


# ------------------------------------------------------------------ QAT fake quantization
def bf16_by_search(v: Fraction) -> int:
    """bf16 bits of the nearest bf16 value to an exact rational (ties to the
    even pattern), by searching the neighbours of its float32 conversion."""
    a = abs(v)
    f = np.float32(float(a))
    u = int(np.array([f], np.float32).view(np.uint32)[0] >> 16)
    cands = [c for c in (u - 1, u, u + 1, u + 2) if 0 <= c < 0x7F80]
    val = lambda c: Fraction(float((np.array([c << 16], np.uint32)).view(np.float32)[0]))
    best = min(cands, key=lambda c: (abs(a - val(c)), c % 2))
    return best


def brute_fake_quantize(xf32: np.ndarray, scale=None):
    """Fake quantization by searches: the brute-force codes and scales, each
    value e2m1 * e4m3 * g formed as an exact rational and rounded to bf16 by
    search, the clip mask by exact rational comparison |x| > 6 s."""
    codes, sfm, g = brute_quantize(xf32, scale)
    rows, k = xf32.shape
    y = np.zeros((rows, k), np.uint16)
    clip = np.zeros((rows, k), bool)
    for r in range(rows):
        for j in range(k):
            c = int(codes[r, j])
            dec = Fraction(float(_E4M3_ALL[sfm[r, j // 16]]))
            mag = Fraction(E2M1_GRID[c & 7]) * dec * Fraction(float(g))
            b = bf16_by_search(mag)
            y[r, j] = b | (0x8000 if c & 8 else 0)
            s = np.float32(np.float32(_E4M3_ALL[sfm[r, j // 16]]) * g)
            clip[r, j] = s > 0 and abs(Fraction(float(xf32[r, j]))) > 6 * Fraction(float(s))
    return y, clip, g


def unpack_mask(m: np.ndarray, k: int) -> np.ndarray:
    return np.unpackbits(m, axis=1, bitorder="little")[:, :k].astype(bool)


@pytest.mark.parametrize("case", range(8))
def test_fake_quantize_vs_brute_force_tiny(case):
    rng = np.random.default_rng(200 + case)
    rows, k = [(2, 64), (3, 128), (1, 192), (4, 64)][case % 4]
    x = rng.standard_normal((rows, k)).astype(np.float32)
    if case % 3 == 1:
        x *= np.exp(rng.uniform(-9, 9, (rows, 1))).astype(np.float32)   # E4M3 subnormal scales
    if case % 4 == 3:
        x[0, :16] = 0.0
        x[1, 3] = -1e-7
    xb = torch.from_numpy(x).to(torch.bfloat16)
    xf = xb.float().numpy()
    amax = float(np.max(np.abs(xf)))
    # a static scale: from the data (None), the data's own, or too small (clips)
    scale = [None, None, float(np.float32(amax / 2688.0)), float(np.float32(amax / 20000.0))][case % 4]
    y, m, g = oracle.fake_quantize(xb, scale)
    by, bclip, bg = brute_fake_quantize(xf, scale)
    assert np.float32(g) == bg
    assert np.array_equal(y, by)
    assert np.array_equal(unpack_mask(m, k), bclip)
    y32, _, _ = oracle.fake_quantize(xb, scale, out="f32")
    # f32 output: the same exact products, rounded by numpy's double -> float cast
    codes, sf, _ = oracle.quantize(xb, scale)
    assert np.array_equal(y32, oracle.dequantize(codes, sf, g, "f64").astype(np.float32))


def test_fake_quantize_saturating_elements_closed_form():
    """With a tensor scale g = 2^-e too small for the data, every element with
    |x| > 2688 g lies in a block whose E4M3 scale saturates at 448, so it clips
    to exactly +-2688 g (exact in bf16) and is marked; elements below stay
    within half a grid spacing."""
    xb = synth.random_bf16((128, 256), seed=21, dist="student_t3")
    xf = xb.float().numpy().astype(np.float64)
    amax = np.max(np.abs(xf))
    e = int(np.ceil(np.log2(2688.0 / amax))) + 3          # 2688 g = amax / 8 .. amax / 4
    g = 2.0 ** -e
    y, m, gg = oracle.fake_quantize(xb, g)
    assert gg == np.float32(g)
    yf = oracle.bf16_to_f32(y).astype(np.float64)
    big = np.abs(xf) > 2688.0 * g
    assert big.sum() > 100
    assert np.array_equal(yf[big], np.sign(xf[big]) * 2688.0 * g)
    clip = unpack_mask(m, 256)
    assert np.all(clip[big])
    assert not np.any(clip[np.abs(xf) <= 2688.0 * g] & (np.abs(yf[np.abs(xf) <= 2688.0 * g]) == 0))


@pytest.mark.parametrize("dist", ["normal", "student_t3", "token_scaled"])
def test_fake_quantize_idempotent_under_fixed_scale(dist):
    """Q(Q(x)) == Q(x) with the tensor scale held fixed: the output already
    lies on the grid its own block scales define (a dropped factor, a swapped
    sign or a wrong rounding would move it)."""
    xb = synth.random_bf16((256, 512), seed=22, dist=dist)
    _, _, g = oracle.fake_quantize(xb)
    y1, _, _ = oracle.fake_quantize(xb, float(g))
    y2, _, _ = oracle.fake_quantize(y1.view(np.uint16).reshape(256, 512), float(g))
    assert np.array_equal(y1, y2)


def test_fake_quantize_zero_cases():
    z = torch.zeros(130, 64, dtype=torch.bfloat16)
    y, m, g = oracle.fake_quantize(z)
    assert g == 0.0 and not y.any() and not m.any()
    # a zero tensor scale: every block scale is 0, every value flushes to +0, nothing clips
    xb = synth.random_bf16((64, 128), seed=23, dist="normal")
    y, m, _ = oracle.fake_quantize(xb, 0.0)
    assert not y.any() and not m.any()


def test_fake_quantize_unclipped_elements_within_half_spacing():
    """Where the mask is clear, |x - y| is at most half the grid spacing at
    |x / s| (plus the bf16 rounding of y); where it is set, |y| is the block's
    largest grid value 6 s."""
    xb = synth.random_bf16((256, 1024), seed=24, dist="outlier")
    y, m, g = oracle.fake_quantize(xb)
    xf = xb.float().numpy().astype(np.float64)
    yf = oracle.bf16_to_f32(y).astype(np.float64)
    codes, sf, _ = oracle.quantize(xb)
    sfm = oracle.sf_matrix(sf, 256, 1024)
    s32 = np.repeat(np.float32(_E4M3_ALL[sfm]) * np.float32(g), 16, axis=1).astype(np.float64)
    clip = unpack_mask(m, 1024)
    q = np.abs(xf) / np.where(s32 > 0, s32, 1.0)
    spacing = np.where(q < 2, 0.5, np.where(q < 4, 1.0, 2.0))
    ok = ~clip & (s32 > 0)
    assert np.all(np.abs(xf - yf)[ok] <= (s32 * spacing / 2 + 2.0 ** -8 * np.abs(yf) + 2.0 ** -21 * np.abs(xf))[ok])
    assert np.all(np.abs(np.abs(yf[clip]) - 6 * s32[clip]) <= 2.0 ** -8 * 6 * s32[clip])
    assert np.all(q[clip] > 6)


def test_ste_backward_closed_form():
    rng = np.random.default_rng(25)
    rows, k = 96, 256
    m = rng.integers(0, 256, (rows, k // 8)).astype(np.uint8)
    keep = ~unpack_mask(m, k)
    g32 = rng.standard_normal((rows, k)).astype(np.float32)
    out = oracle.ste_backward(g32, m)
    assert np.array_equal(out, np.where(keep, g32, np.float32(0.0)))
    assert not np.signbit(out[~keep]).any()
    gb = rng.integers(0, 1 << 16, (rows, k)).astype(np.uint16)
    out = oracle.ste_backward(gb, m)
    assert np.array_equal(out, np.where(keep, gb, np.uint16(0)))


def test_fake_quantize_grid_valued_input_is_a_fixed_point():
    """Grid values times 2^m per block with g = 2^-8: s = 2^m exactly, every
    value comes back unchanged, and the block maxima (|x| = 6 s exactly, on
    clip's boundary) are not marked as clipped."""
    rng = np.random.default_rng(26)
    rows, k = 8, 128
    vals = np.array(E2M1_GRID + [-v for v in E2M1_GRID[1:]], np.float64)
    x = rng.choice(vals, (rows, k))
    m = rng.integers(-12, 1, (rows, k // 16))
    for r in range(rows):
        for c in range(k // 16):
            x[r, 16 * c] = -6.0 if (r + c) % 2 else 6.0
            x[r, 16 * c:16 * c + 16] *= 2.0 ** m[r, c]
    xb = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    y, mask, _ = oracle.fake_quantize(xb, 2.0 ** -8)
    assert np.array_equal(oracle.bf16_to_f32(y).astype(np.float64), x)
    assert not mask.any()


# ------------------------------------------------------------------ epilogue activation
def test_gelu_tanh_against_library_and_identities():
    """The tanh-form GELU: torch's float64 implementation (a library routine),
    the identity g(v) - g(-v) = v (the tanh term is odd), the erf form within
    1e-3, and the limits."""
    import math
    rng = np.random.default_rng(30)
    v = np.concatenate([rng.standard_normal(4000) * 3, np.linspace(-12, 12, 2001), [0.0, 1e-30, -1e-30]])
    g = oracle.gelu_tanh(v)
    ref = torch.nn.functional.gelu(torch.from_numpy(v), approximate="tanh").numpy()
    assert np.max(np.abs(g - ref)) <= 1e-14 * np.maximum(1.0, np.abs(v)).max()
    assert np.max(np.abs(g - oracle.gelu_tanh(-v) - v)) <= 1e-13
    erf = np.array([0.5 * x * (1 + math.erf(x / math.sqrt(2))) for x in v])
    assert np.max(np.abs(g - erf)) < 1e-3
    assert oracle.gelu_tanh(0.0) == 0.0
    assert oracle.gelu_tanh(40.0) == 40.0 and oracle.gelu_tanh(-40.0) == 0.0


# ------------------------------------------------------------------ MXFP4
def brute_mx(xf32: np.ndarray):
    """MX quantization by searches: the block exponent s is the integer with
    4 * 2^s <= max|x| < 8 * 2^s (searched, clamped to [-127, 127]; -127 for an
    all-zero block), codes by the nearest-grid search of x / 2^s."""
    rows, k = xf32.shape
    codes = np.zeros((rows, k), np.uint8)
    exps = np.zeros((rows, k // 32), np.int64)
    for r in range(rows):
        for c in range(k // 32):
            blk = [Fraction(float(v)) for v in xf32[r, 32 * c:32 * c + 32]]
            amax = max(abs(v) for v in blk)
            s = -127
            if amax > 0:
                s = next(t for t in range(-160, 160) if 4 * Fraction(2) ** t <= amax < 8 * Fraction(2) ** t)
                s = min(max(s, -127), 127)
            exps[r, c] = s
            for i, v in enumerate(blk):
                q = v / Fraction(2) ** s
                code = brute_e2m1(float(q))
                if v == 0 and np.signbit(xf32[r, 32 * c + i]):
                    code |= 8
                codes[r, 32 * c + i] = code
    return codes, exps


@pytest.mark.parametrize("case", range(6))
def test_mx_quantize_vs_brute_force_tiny(case):
    rng = np.random.default_rng(300 + case)
    rows, k = [(1, 128), (3, 128), (2, 256)][case % 3]
    x = rng.standard_normal((rows, k)).astype(np.float32)
    x *= np.exp2(rng.uniform(-30, 30, (rows, k // 32))).repeat(32, axis=1).astype(np.float32)
    if case == 4:
        x[0, :32] = 0.0
        x[0, 3] = -0.0
    if case == 5:
        x[1, 32:64] = (rng.standard_normal(32) * 2.0 ** -128).astype(np.float32)   # bf16 subnormals:
        x[0, 64:96] = np.float32(2.0 ** -133)                                      # exponent clamps at -127
    xb = torch.from_numpy(x).to(torch.bfloat16)
    xf = xb.float().numpy()
    codes, sf = oracle.mx_quantize(xb)
    bc, be = brute_mx(xf)
    assert np.array_equal(oracle.unpack_codes(codes), bc)
    assert np.array_equal(oracle.mx_sf_matrix(sf, rows, k).astype(np.int64) - 127, be)


def test_mx_grid_membership_error_bound_and_fixed_points():
    xb = synth.random_bf16((256, 1024), seed=31, dist="outlier")
    codes, sf = oracle.mx_quantize(xb)
    xf = xb.float().numpy().astype(np.float64)
    deq = oracle.mx_dequantize(codes, sf)
    X = np.exp2(oracle.mx_sf_matrix(sf, 256, 1024).astype(np.float64) - 127).repeat(32, axis=1)
    grid = set(E2M1_GRID) | {-v for v in E2M1_GRID}
    assert set(np.unique(deq / X)) <= grid
    q = np.abs(xf) / X
    spacing = np.where(q < 2, 0.5, np.where(q < 4, 1.0, 2.0))
    bound = np.where(q <= 6, X * spacing / 2, np.abs(xf) - 6 * X)
    assert np.all(np.abs(xf - deq) <= bound)
    assert q.max() < 8 and (q > 6).any()                       # the block maximum can clip (8 > 6)
    # grid values times 2^m whose block maximum is 4 or 6 come back unchanged
    rng = np.random.default_rng(32)
    vals = np.array(E2M1_GRID + [-v for v in E2M1_GRID[1:]])
    g = rng.choice(vals, (8, 256))
    g[:, ::32] = rng.choice([4.0, -6.0, 6.0], (8, 8))
    g *= np.exp2(rng.integers(-20, 20, (8, 8))).repeat(32, axis=1)
    gb = torch.from_numpy(g.astype(np.float32)).to(torch.bfloat16)
    c2, s2 = oracle.mx_quantize(gb)
    assert np.array_equal(oracle.mx_dequantize(c2, s2), g)


def test_mx_zero_tensor_and_gemm_vs_library_matmul():
    codes, sf = oracle.mx_quantize(torch.zeros(130, 128, dtype=torch.bfloat16))
    assert not codes.any() and not oracle.mx_sf_matrix(sf, 130, 128).any()
    x = synth.random_bf16((64, 384), seed=33, dist="student_t3")
    w = synth.random_bf16((48, 384), seed=34, dist="normal", scale=0.02)
    ac, asf = oracle.mx_quantize(x)
    bc, bsf = oracle.mx_quantize(w)
    y = oracle.mx_gemm(ac, asf, bc, bsf)
    ref = torch.from_numpy(oracle.mx_dequantize(ac, asf)) @ torch.from_numpy(oracle.mx_dequantize(bc, bsf)).T
    assert np.allclose(y, ref.numpy(), rtol=1e-12, atol=1e-12 * np.abs(y).max())
    assert np.array_equal(oracle.mx_gemm(ac, asf, bc, bsf, rows=slice(5, 9)), y[5:9])


# ------------------------------------------------------------------ adaptive block size (Alg. 1, Eq. 9)
def brute_block_quantize(xf32: np.ndarray, block: int, g: np.float32):
    """Per `block` values: the E4M3 scale by search, codes by nearest-grid
    search, the dequantized value e2m1 * e4m3 * g as an exact rational."""
    rows, k = xf32.shape
    f = np.float32
    d = f(f(6.0) * g)
    codes = np.zeros((rows, k), np.uint8)
    scales = np.zeros((rows, k // block), np.uint8)
    deq = np.zeros((rows, k), object)
    for r in range(rows):
        for c in range(k // block):
            blk = xf32[r, block * c:block * c + block]
            ab = f(np.max(np.abs(blk)))
            sfc = brute_e4m3(f(ab / d)) if d > 0 else 0
            scales[r, c] = sfc
            s = f(f(_E4M3_ALL[sfc]) * g)
            for i in range(block):
                code = brute_e2m1(f(blk[i] / s)) if s != 0 else 0
                codes[r, block * c + i] = code
                mag = Fraction(E2M1_GRID[code & 7]) * Fraction(float(_E4M3_ALL[sfc])) * Fraction(float(g))
                deq[r, block * c + i] = -mag if code & 8 else mag
    return codes, scales, deq


def test_quantize_block_16_is_quantize_and_larger_blocks_vs_brute_force():
    xb = synth.random_bf16((130, 256), seed=40, dist="outlier")
    c16, s16, g16 = oracle.quantize_block(xb, 16)
    c, s, g = oracle.quantize(xb)
    assert g16 == g and np.array_equal(c16, c) and np.array_equal(s16, s)
    rng = np.random.default_rng(41)
    x = (rng.standard_normal((3, 128)) * np.exp2(rng.uniform(-6, 6, (3, 1)))).astype(np.float32)
    xt = torch.from_numpy(x).to(torch.bfloat16)
    xf = xt.float().numpy()
    for block in (32, 64):
        codes, sf, g = oracle.quantize_block(xt, block)
        bc, bs, _ = brute_block_quantize(xf, block, np.float32(g))
        assert np.array_equal(oracle.unpack_codes(codes), bc)
        # each block scale repeated in its block/16 slots of the block-16 layout
        assert np.array_equal(oracle.sf_matrix(sf, 3, 128), np.repeat(bs, block // 16, axis=1))


def test_block_size_errors_vs_brute_force_and_dequantized_quantization():
    rng = np.random.default_rng(42)
    x = (rng.standard_normal((2, 64)) * np.exp2(rng.uniform(-4, 4, (2, 64)))).astype(np.float32)
    xt = torch.from_numpy(x).to(torch.bfloat16)
    xf = xt.float().numpy()
    g = oracle.tensor_scale(xt)
    err, ss = oracle.block_size_errors(xt, g)
    assert ss == pytest.approx(float(np.sum(xf.astype(np.float64) ** 2)), rel=1e-15)
    for i, b in enumerate(oracle.BLOCK_SIZES):
        _, _, deq = brute_block_quantize(xf, b, np.float32(g))
        exact = sum((Fraction(float(v)) - q) ** 2 for v, q in zip(xf.ravel(), deq.ravel()))
        assert err[i] == pytest.approx(float(exact), rel=1e-12), b
    # on a larger tensor: blocks 16 / 32 / 64 match the dequantized block quantization
    xb = synth.random_bf16((64, 512), seed=43, dist="student_t3")
    g = oracle.tensor_scale(xb)
    err, _ = oracle.block_size_errors(xb, g)
    xd = xb.float().numpy().astype(np.float64)
    for i, b in ((4, 16), (5, 32), (6, 64)):
        c, s, gg = oracle.quantize_block(xb, b, float(g))
        assert err[i] == pytest.approx(float(np.sum((xd - oracle.dequantize(c, s, gg)) ** 2)), rel=1e-12)


def test_select_block_size_limits():
    xb = synth.random_bf16((64, 256), seed=44, dist="student_t3")
    err, ss = oracle.block_size_errors(xb, oracle.tensor_scale(xb))
    rel = err / ss
    assert oracle.select_block_size(err, ss, 0.0) == oracle.BLOCK_SIZES[int(np.argmin(rel))]
    assert oracle.select_block_size(err, ss, 1e6) == 64
    # hand case: only 8 and 16 differ and memory decides at lambda = 1
    e = np.array([1.0, 1.0, 1.0, 0.10, 0.10, 1.0, 1.0]) * 100.0
    assert oracle.select_block_size(e, 100.0, 0.0) == 8                 # first minimum
    assert oracle.select_block_size(e, 100.0, 1.0) == 16                # 4 + 8/16 < 4 + 8/8
    # Memory is normalised by Memory(1) = 12 bits: errors 0.10 (b = 8) and 0.15
    # (b = 16) against memory terms lambda * 5/12 and lambda * 4.5/12
    e = np.array([1.0, 1.0, 1.0, 0.10, 0.15, 1.0, 1.0]) * 100.0
    assert oracle.select_block_size(e, 100.0, 1.0) == 8                 # 0.5167 < 0.525
    assert oracle.select_block_size(e, 100.0, 2.0) == 16                # 0.9333 > 0.9


# ------------------------------------------------------------------ attention (Eq. 10)
def _attn_operands(H, Lq, Lk, d, seed):
    q = oracle.quantize(synth.random_bf16((H * Lq, d), seed=seed, dist="normal"))
    k = oracle.quantize(synth.random_bf16((H * Lk, d), seed=seed + 1, dist="normal"))
    v = oracle.quantize(synth.random_bf16((H * Lk, d), seed=seed + 2, dist="student_t3"))
    return q, k, v


def test_attention_vs_library_and_identities():
    H, Lq, Lk, d = 2, 40, 96, 64
    q, k, v = _attn_operands(H, Lq, Lk, d, 60)
    s_head = np.array([1.0, 3.5])
    qd = oracle.dequantize(*q).reshape(H, Lq, d)
    kd = oracle.dequantize(*k).reshape(H, Lk, d)
    vd = oracle.dequantize(*v).reshape(H, Lk, d)
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(qd), torch.from_numpy(kd),
                                                           torch.from_numpy(vd)).numpy()
    for h in range(H):
        o = oracle.attention(q, k, v, s_head, H, Lq, Lk, d, h)
        assert np.allclose(o, ref[h], rtol=1e-12, atol=1e-12 * np.abs(vd).max())
        # the per-head term is a constant shift of every logit of the head
        o1 = oracle.attention(q, k, v, np.ones(H), H, Lq, Lk, d, h)
        assert np.allclose(o, o1, rtol=1e-12, atol=1e-12 * np.abs(vd).max())
        assert np.array_equal(oracle.attention(q, k, v, s_head, H, Lq, Lk, d, h, rows=slice(7, 11)), o[7:11])
    # rows of p sum to one: with a constant V the output is that constant
    ones = oracle.quantize(torch.ones(H * Lk, d, dtype=torch.bfloat16))
    c = oracle.dequantize(*ones)[0, 0]
    o = oracle.attention(q, k, ones, s_head, H, Lq, Lk, d, 1)
    assert np.allclose(o, c, rtol=1e-14)


def test_attention_one_hot_selects_the_matching_key():
    """Q row i a large multiple of K row (3 i mod Lk) (logit 512 against 0):
    the output is V of that key."""
    H, Lq, Lk, d = 1, 16, 64, 64
    eye = torch.zeros(Lk, d)
    for j in range(Lk):
        eye[j, j] = 1.0
    kq = oracle.quantize(eye.bfloat16())
    qx = torch.zeros(Lq, d)
    for i in range(Lq):
        qx[i, (3 * i) % Lk] = 4096.0
    q = oracle.quantize(qx.bfloat16())
    v = oracle.quantize(synth.random_bf16((Lk, d), seed=61, dist="normal"))
    o = oracle.attention(q, kq, v, np.ones(1), H, Lq, Lk, d, 0)
    vd = oracle.dequantize(*v)
    for i in range(Lq):
        assert np.allclose(o[i], vd[(3 * i) % Lk], rtol=1e-12, atol=1e-12)


def _tensor_scale_bf16_strided(bits: np.ndarray, k: int) -> np.float32:
    """Call the oracle's bf16 tensor scale on the first k columns of a wider
    row-major buffer (row stride = the buffer's width)."""
    bits = np.ascontiguousarray(bits, np.uint16)
    rows, ld = bits.shape
    return np.float32(oracle.lib().oracle_tensor_scale_bf16(bits.ctypes.data, rows, k, ld))


def _numpy_scale(bits: np.ndarray) -> np.float32:
    """Independent value: numpy's float32 max |x| over the bf16 values, then
    one IEEE float32 division by 6 * 448 (RFC, Motivation: one FP32 scale per
    tensor; the tensor maximum maps onto 2688)."""
    f = (bits.astype(np.uint32) << 16).view(np.float32)
    return np.float32(np.max(np.abs(f))) / np.float32(2688.0) if f.size else np.float32(0.0)


def test_tensor_scale_bf16_pinned_by_numpy():
    rng = np.random.default_rng(11)
    # bf16 bits by truncation of float32 (the test only needs some bf16 values)
    f32 = lambda a: (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    # strided views: padding columns beyond k hold a value larger than any inside
    for rows, k, ld in [(7, 64, 80), (130, 256, 264), (1, 1024, 1024)]:
        x = f32(rng.standard_normal((rows, ld)) * 3.0)
        x[:, k:] = f32(1e30)
        inner = x[:, :k]
        got = _tensor_scale_bf16_strided(x, k)
        assert got.view(np.uint32) == _numpy_scale(inner).view(np.uint32)
        # the maximum is in the last row and column
        y = x.copy()
        y[-1, k - 1] = f32(-1e4)
        top = (np.uint32(y[-1, k - 1] & 0x7FFF) << 16).view(np.float32)
        assert _tensor_scale_bf16_strided(y, k) == _numpy_scale(y[:, :k]) == top / np.float32(2688.0)
    # a negative maximum magnitude
    x = f32([[-5.0] + [1.0] * 63])
    assert _tensor_scale_bf16_strided(x, 64) == np.float32(5.0) / np.float32(2688.0)
    # -0 everywhere, +0 everywhere: g = +0
    for z in (0x8000, 0x0000):
        g = _tensor_scale_bf16_strided(np.full((3, 64), z, np.uint16), 64)
        assert g == 0 and not np.signbit(g)
    # bf16 subnormals: amax itself subnormal, quotient rounded (or flushed) by IEEE float32 rules
    for top in (0x0001, 0x0007, 0x007F, 0x0080):
        x = np.zeros((2, 64), np.uint16)
        x[1, 5] = top
        x[0, 3] = 0x8000 | max(top - 1, 0)
        assert _tensor_scale_bf16_strided(x, 64).view(np.uint32) == _numpy_scale(x).view(np.uint32)
    # every finite bf16 magnitude as the maximum of a small tensor (sampled)
    for b in range(0, 0x7F80, 97):
        x = np.zeros((1, 64), np.uint16)
        x[0, 63] = b | 0x8000
        assert _tensor_scale_bf16_strided(x, 64).view(np.uint32) == _numpy_scale(x).view(np.uint32)


# ---------------------------------------------------------------- LayerNorm (fused producer)
def _ln_inputs(rows, k, seed, dist, groups):
    x = synth.random_bf16((rows, k), seed=seed, dist=dist)
    rng = np.random.default_rng(seed)
    gamma = (1.0 + 0.5 * rng.standard_normal((groups, k))).astype(np.float32)
    beta = (0.3 * rng.standard_normal((groups, k))).astype(np.float32)
    return x, gamma, beta


def _ln_library(x, gamma, beta, rows_per_group, eps):
    """torch's float64 layer_norm (library routine), one group of rows at a time."""
    xf = torch.from_numpy(oracle.bf16_to_f32(oracle.bf16_bits(x)).astype(np.float64))
    rows, k = xf.shape
    out = torch.empty_like(xf)
    for r0 in range(0, rows, rows_per_group or rows):
        r1 = min(rows, r0 + (rows_per_group or rows))
        gi = r0 // rows_per_group if rows_per_group else 0
        w = None if gamma is None else torch.from_numpy(gamma[gi].astype(np.float64))
        b = None if beta is None else torch.from_numpy(beta[gi].astype(np.float64))
        out[r0:r1] = torch.nn.functional.layer_norm(xf[r0:r1], (k,), w, b, eps)
    return out.numpy(), xf.numpy()


@pytest.mark.parametrize("rows,k,dist,groups,affine", [(37, 1152, "outlier", 5, True), (8, 3072, "token_scaled", 2, True),
                                                        (16, 256, "student_t3", 1, False), (3, 5120, "normal", 3, True)])
def test_layernorm_vs_library(rows, k, dist, groups, affine):
    x, gamma, beta = _ln_inputs(rows, k, rows + k, dist, groups)
    rpg = -(-rows // groups)
    g, b = (gamma, beta) if affine else (None, None)
    y = oracle.layernorm(x, g, b, rpg if affine else 0, 1e-6)
    ref, xf = _ln_library(x, g, b, rpg if affine else 0, 1e-6)
    mu = xf.mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(xf.var(axis=1, keepdims=True) + 1e-6)
    gam = np.repeat(g, rpg, axis=0)[:rows].astype(np.float64) if affine else 1.0
    bet = np.repeat(b, rpg, axis=0)[:rows].astype(np.float64) if affine else 0.0
    # FP32 normalisation: a few roundings of |x - mu| rstd |gamma|, of the
    # rounded mean and of the shift
    tol = 2.0 ** -20 * ((np.abs(xf - mu) + np.abs(mu)) * rstd * np.abs(gam) + np.abs(bet)) + 1e-30
    assert np.all(np.abs(y.astype(np.float64) - ref) <= tol)


def test_layernorm_rows_are_standardized_and_constant_rows_give_beta():
    x = synth.random_bf16((64, 1152), seed=9, dist="token_scaled")
    y = oracle.layernorm(x).astype(np.float64)
    xf = oracle.bf16_to_f32(oracle.bf16_bits(x)).astype(np.float64)
    v = xf.var(axis=1)
    assert np.all(np.abs(y.mean(axis=1)) <= 1e-6)
    assert np.all(np.abs(y.var(axis=1) - v / (v + 1e-6)) <= 1e-5)
    # a constant row normalises to exact zeros, so the output is beta itself
    c = np.full((2, 256), 0x4049, np.uint16)                      # bf16 3.140625
    beta = np.linspace(-1, 1, 256, dtype=np.float32)[None, :]
    gamma = np.full((1, 256), 2.5, np.float32)
    yc = oracle.layernorm(c, gamma, beta, 2, 1e-6)
    assert np.array_equal(yc, np.repeat(beta, 2, axis=0))


def test_layernorm_groups_match_rows_taken_one_group_at_a_time():
    x, gamma, beta = _ln_inputs(12, 512, 4, "outlier", 3)
    y = oracle.layernorm(x, gamma, beta, 4, 1e-6)
    for gi in range(3):
        yi = oracle.layernorm(x[4 * gi:4 * gi + 4], gamma[gi], beta[gi], 0, 1e-6)
        assert np.array_equal(y[4 * gi:4 * gi + 4], yi)


def test_layernorm_quantize_is_quantize_of_the_layernorm():
    x, gamma, beta = _ln_inputs(130, 1152, 5, "student_t3", 1)
    c, s, g = oracle.layernorm_quantize(x, gamma, beta, 0, 1e-6)
    c2, s2, g2 = oracle.quantize(oracle.layernorm(x, gamma, beta, 0, 1e-6))
    assert g == g2 and np.array_equal(c, c2) and np.array_equal(s, s2)
