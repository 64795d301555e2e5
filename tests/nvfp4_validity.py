"""Complete validity check of an NVFP4 tensor produced from values known only
within a tolerance (the fused NVFP4 output of a GEMM epilogue, whose FP32
accumulation order is not fixed).

The quantizer ("NVFP4-DiT" README, Definition III.1, with the two-level scaling
of "[RFC]: NVFP4 Quantization Support for Diffusion Models", Motivation) is
monotone at every step:

  block scale   sf = E4M3_rne(rn(a_b / rn(6 g))),  a_b = max |y'| over 16 values
  element code  c  = E2M1_rne(rn(y' / s)),         s = rn(e4m3(sf) * g)

where y' is the kernel's FP32 value of an element, known to lie within t of the
oracle's FP64 value v.  So a GPU output is a correct rounding of SOME admissible
y' exactly when

  * per block: sf lies between the codes of the smallest and the largest
    admissible block maximum, and
  * per element: with the GPU's own s, the decoded code lies between the
    decoded codes of rn(v - t) / s and rn(v + t) / s, and a signed zero has a
    sign some admissible y' can have.

Both bounds are taken with the oracle's own codecs (``oracle.e4m3_encode``,
``oracle.e2m1_encode``), never with the CUDA library.  A code one grid step off,
or a scale byte one E4M3 step off, fails unless the tolerance interval itself
straddles a rounding boundary.
"""
from __future__ import annotations

import numpy as np

import oracle

_E2M1 = np.array([oracle.e2m1_decode(c) for c in range(16)], np.float64)
_e2m1_enc = np.frompyfunc(lambda q: oracle.e2m1_encode(float(q)), 1, 1)
_e4m3_enc = np.frompyfunc(lambda r: oracle.e4m3_encode(float(r)), 1, 1)
_E4M3 = np.array([oracle.e4m3_decode(c) for c in range(0x7F)] + [np.nan], np.float64)


def nvfp4_rounding_violations(codes: np.ndarray, sfm: np.ndarray, g_y: float, v: np.ndarray,
                              t: np.ndarray) -> dict:
    """Return the violations of the check above as index arrays.

    codes [M, N/2] uint8 and sfm [M, N/16] (the scale bytes gathered out of the
    tensor-core layout by ``oracle.sf_matrix``) are the tensor under test, g_y
    its FP32 tensor scale, v [M, N] the FP64 values it should encode, and t
    (broadcastable to v, >= 0) how far the producer's FP32 values may be from v.
    Keys: 'scale' -> (row, block) pairs, 'code' -> (row, col) pairs.
    """
    v = np.asarray(v, np.float64)
    M, N = v.shape
    kb = N // 16
    t = np.broadcast_to(np.asarray(t, np.float64), v.shape)
    g = np.float32(g_y)
    d = np.float32(6.0) * g

    # ---- block scales: the range of admissible block maxima
    lo_mag = np.maximum(np.abs(v) - t, 0.0)
    hi_mag = np.abs(v) + t
    a_lo = lo_mag.reshape(M, kb, 16).max(axis=2).astype(np.float32)
    a_hi = hi_mag.reshape(M, kb, 16).max(axis=2).astype(np.float32)
    sfm = np.asarray(sfm).astype(np.int64)
    if d > 0:
        with np.errstate(over="ignore"):
            sf_lo = _e4m3_enc(a_lo / d).astype(np.int64)
            sf_hi = _e4m3_enc(a_hi / d).astype(np.int64)
    else:
        sf_lo = sf_hi = np.zeros_like(sfm)
    bad_sf = (sfm < sf_lo) | (sfm > sf_hi) | (sfm >= 0x7F)

    # ---- element codes, divided by the GPU's own block scale
    s = (_E4M3[np.minimum(sfm, 0x7F)].astype(np.float32) * g).astype(np.float32)
    s_el = np.repeat(s, 16, axis=1)
    nib = oracle.unpack_codes(codes).astype(np.int64)
    val = _E2M1[nib]
    y_lo = (v - t).astype(np.float32)
    y_hi = (v + t).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        q_lo = np.where(s_el > 0, y_lo / s_el, 0.0).astype(np.float32)
        q_hi = np.where(s_el > 0, y_hi / s_el, 0.0).astype(np.float32)
    c_lo = _E2M1[_e2m1_enc(q_lo).astype(np.int64)]
    c_hi = _E2M1[_e2m1_enc(q_hi).astype(np.int64)]
    bad = (val < c_lo) | (val > c_hi)
    # signed zeros: 0x8 needs an admissible value <= 0, 0x0 one >= 0
    bad |= (nib == 8) & (y_lo > 0)
    bad |= (nib == 0) & (y_hi < 0)
    # a zero scale quantizes everything to code 0x0
    bad |= (s_el == 0) & (nib != 0)
    return {"scale": np.argwhere(bad_sf), "code": np.argwhere(bad)}


def assert_valid_nvfp4_rounding(codes, sfm, g_y, v, t) -> None:
    viol = nvfp4_rounding_violations(codes, sfm, g_y, v, t)
    ns, nc = len(viol["scale"]), len(viol["code"])
    assert ns == 0 and nc == 0, (
        f"{ns} scale bytes and {nc} codes are no valid rounding within the tolerance; "
        f"first scale (row, block) {viol['scale'][:3].tolist()}, first code (row, col) {viol['code'][:3].tolist()}")
