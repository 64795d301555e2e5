"""CPU oracle for NVFP4 two-level quantization and the FP4 GEMMs.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product library never links or calls it, and it shares no code
with the CUDA path.

The arithmetic lives in ``nvfp4_oracle.c`` (plain C, one rounding per
operation, double-precision sums).  This module only moves numpy arrays in and
out of it.  Each wrapper names the passage it follows; see the C file header
for the readings taken where the pages are silent.

Parity status per function:
  e2m1_encode / e2m1_decode, e4m3_encode / e4m3_decode  -- pinned (exhaustive
      brute force, library FP8 cast, closed-form tie points)
  quantize                                              -- pinned (brute force
      on tiny inputs, grid membership, error bound, special cases)
  sf_offset                                             -- pinned (bijection,
      hand-derived offsets; the layout itself is the tensor core's, confirmed
      on the GPU by one-hot products)
  dequantize                                            -- pinned (exact
      products, round-trip of grid-valued blocks)
  gemm_w4a4 / gemm_w4a16                                -- pinned (one-hot
      products, float64 library matmul of the dequantized operands)
  fake_quantize                                         -- pinned (brute force
      on tiny inputs, idempotence under a fixed tensor scale, the closed form
      of saturating elements)
  ste_backward                                          -- pinned (closed form
      through numpy's bit unpacking)
  mx_quantize / mx_dequantize / mx_gemm                 -- pinned (brute-force
      exponent and nearest-grid searches on tiny inputs, grid membership and
      the error bound, power-of-two fixed points, a float64 library matmul)
  quantize_block / block_size_errors / select_block_size -- pinned (block 16
      equals quantize, brute force for blocks 32 and 64, errors against the
      dequantized oracle quantization and brute force, Eq. 9 limits)
  attention                                             -- pinned (float64
      library attention of the dequantized operands, rows of p summing to
      one, invariance under the per-head term, a one-hot case)
  layernorm / layernorm_quantize                        -- pinned (torch's
      float64 layer_norm within the FP32 rounding of the normalisation,
      zero-mean / unit-variance rows, constant rows, the per-group affine
      against explicit rows, planted mistakes; the quantization is quantize)
  gelu_tanh                                             -- pinned (torch's
      float64 tanh-form GELU, the odd-part identity g(v) - g(-v) = v, the erf
      form within 1e-3, limits)
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

_i64 = ctypes.c_int64
_f32 = ctypes.c_float
_p = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint]
        L.oracle_e2m1_decode.restype = ctypes.c_double
        L.oracle_e2m1_encode.argtypes = [_f32]
        L.oracle_e2m1_encode.restype = ctypes.c_uint
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_encode.argtypes = [_f32]
        L.oracle_e4m3_encode.restype = ctypes.c_uint
        L.oracle_bf16_from_double.argtypes = [ctypes.c_double]
        L.oracle_bf16_from_double.restype = ctypes.c_uint16
        L.oracle_sf_bytes.argtypes = [_i64, _i64]
        L.oracle_sf_bytes.restype = _i64
        L.oracle_sf_offset.argtypes = [_i64, _i64, _i64]
        L.oracle_sf_offset.restype = _i64
        L.oracle_tensor_scale_f32.argtypes = [_p, _i64, _i64, _i64]
        L.oracle_tensor_scale_f32.restype = _f32
        L.oracle_tensor_scale_bf16.argtypes = [_p, _i64, _i64, _i64]
        L.oracle_tensor_scale_bf16.restype = _f32
        for name in ("oracle_quantize_f32", "oracle_quantize_bf16"):
            fn = getattr(L, name)
            fn.argtypes = [_p, _i64, _i64, _i64, ctypes.c_int, _p, _p, _p]
            fn.restype = None
        for name in ("oracle_dequantize_f64", "oracle_dequantize_f32", "oracle_dequantize_bf16"):
            fn = getattr(L, name)
            fn.argtypes = [_p, _p, _f32, _i64, _i64, _p]
            fn.restype = None
        L.oracle_gemm_w4a4_rows.argtypes = [_p, _p, _f32, _p, _p, _f32, _i64, _i64, _i64, _i64, _i64, _p]
        L.oracle_gemm_w4a4_rows.restype = None
        L.oracle_gemm_w4a4_at.argtypes = [_p, _p, _f32, _p, _p, _f32, _i64, _i64, _i64]
        L.oracle_gemm_w4a4_at.restype = ctypes.c_double
        L.oracle_gemm_w4a16_rows.argtypes = [_p, _p, _p, _f32, _i64, _i64, _i64, _i64, _i64, _p]
        L.oracle_gemm_w4a16_rows.restype = None
        L.oracle_gemm_w4a16_at.argtypes = [_p, _p, _p, _f32, _i64, _i64, _i64]
        L.oracle_gemm_w4a16_at.restype = ctypes.c_double
        L.oracle_fake_quantize_bf16.argtypes = [_p, _i64, _i64, _i64, ctypes.c_int, _p, ctypes.c_int, _p, _p]
        L.oracle_fake_quantize_bf16.restype = None
        L.oracle_ste_backward.argtypes = [_p, _p, _i64, _i64, ctypes.c_int, _p]
        L.oracle_ste_backward.restype = None
        L.oracle_mx_sf_bytes.argtypes = [_i64, _i64]
        L.oracle_mx_sf_bytes.restype = _i64
        L.oracle_mx_quantize_bf16.argtypes = [_p, _i64, _i64, _i64, _p, _p]
        L.oracle_mx_quantize_bf16.restype = None
        L.oracle_mx_dequantize_f64.argtypes = [_p, _p, _i64, _i64, _p]
        L.oracle_mx_dequantize_f64.restype = None
        L.oracle_mx_gemm_rows.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64, _i64, _p]
        L.oracle_mx_gemm_rows.restype = None
        L.oracle_quantize_block_bf16.argtypes = [_p, _i64, _i64, _i64, ctypes.c_int, ctypes.c_int, _p, _p, _p]
        L.oracle_quantize_block_bf16.restype = None
        L.oracle_block_size_errors.argtypes = [_p, _i64, _i64, _i64, _f32, _p, _p]
        L.oracle_block_size_errors.restype = None
        L.oracle_select_block_size.argtypes = [_p, ctypes.c_double, ctypes.c_double]
        L.oracle_select_block_size.restype = ctypes.c_int
        L.oracle_attention_rows.argtypes = [_p, _p, _f32, _p, _p, _f32, _p, _p, _f32, _i64, _i64, _i64, _p, _i64,
                                            _i64, _i64, _p]
        L.oracle_attention_rows.restype = None
        L.oracle_layernorm_f32.argtypes = [_p, _i64, _i64, _i64, _p, _p, _i64, ctypes.c_double, _p]
        L.oracle_layernorm_f32.restype = None
        L.oracle_gelu_tanh.argtypes = [ctypes.c_double]
        L.oracle_gelu_tanh.restype = ctypes.c_double
        L.oracle_gelu_tanh_array.argtypes = [_p, _i64, _p]
        L.oracle_gelu_tanh_array.restype = None
        _LIB = L
    return _LIB


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


# ---------------------------------------------------------------- codecs
def e2m1_decode(code: int) -> float:
    """Value of a 4-bit E2M1 code (1 sign, 2 exponent, 1 mantissa bit;
    NVFP4-DiT README, Definition III.1)."""
    return lib().oracle_e2m1_decode(int(code))


def e2m1_encode(q: float) -> int:
    """RNE of an FP32 quotient onto E2M1, clipped to [-6, 6]."""
    return lib().oracle_e2m1_encode(float(np.float32(q)))


def e4m3_decode(code: int) -> float:
    """Value of an E4M3FN byte (NaN for S.1111.111)."""
    return lib().oracle_e4m3_decode(int(code))


def e4m3_encode(v: float) -> int:
    """RNE of a non-negative FP32 value onto E4M3FN, saturating at 448."""
    return lib().oracle_e4m3_encode(float(np.float32(v)))


def bf16_from_double(v: float) -> int:
    return int(lib().oracle_bf16_from_double(float(v)))


def sf_bytes(rows: int, k: int) -> int:
    return int(lib().oracle_sf_bytes(rows, k))


def sf_offset(r: int, c: int, kb: int) -> int:
    return int(lib().oracle_sf_offset(r, c, kb))


# ---------------------------------------------------------------- tensors
def bf16_bits(x) -> np.ndarray:
    """uint16 view of a bf16 torch tensor (CPU) or pass-through of uint16."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def quantize(x, scale: float | None = None):
    """Two-level NVFP4 quantization (NVFP4-DiT README, Definition III.1, with the
    RFC's two-level scaling).  ``x`` is a bf16 torch tensor, a uint16 array of
    bf16 bits, or a float32 array, shape [rows, k].  Returns (codes uint8
    [rows, k/2], sf uint8 [sf_bytes], g float32)."""
    L = lib()
    if isinstance(x, np.ndarray) and x.dtype == np.float32:
        xa = np.ascontiguousarray(x)
        fn = L.oracle_quantize_f32
    else:
        xa = bf16_bits(x)
        fn = L.oracle_quantize_bf16
    rows, k = xa.shape
    assert k % 64 == 0
    codes = np.zeros((rows, k // 2), np.uint8)
    sf = np.zeros(sf_bytes(rows, k), np.uint8)
    g = np.zeros(1, np.float32)
    if scale is not None:
        g[0] = np.float32(scale)
    fn(_ptr(xa), rows, k, k, 1 if scale is not None else 0, _ptr(g), _ptr(codes), _ptr(sf))
    return codes, sf, np.float32(g[0])


def dequantize(codes: np.ndarray, sf: np.ndarray, g: float, out: str = "f64") -> np.ndarray:
    """v = (e2m1(code) * dec(sf)) * g, exact in double; 'f32' / 'bf16' round it
    once (RNE).  'bf16' returns uint16 bits."""
    L = lib()
    codes = np.ascontiguousarray(codes, np.uint8)
    sf = np.ascontiguousarray(sf, np.uint8)
    rows, kh = codes.shape
    k = kh * 2
    if out == "f64":
        y = np.empty((rows, k), np.float64)
        L.oracle_dequantize_f64(_ptr(codes), _ptr(sf), float(g), rows, k, _ptr(y))
    elif out == "f32":
        y = np.empty((rows, k), np.float32)
        L.oracle_dequantize_f32(_ptr(codes), _ptr(sf), float(g), rows, k, _ptr(y))
    elif out == "bf16":
        y = np.empty((rows, k), np.uint16)
        L.oracle_dequantize_bf16(_ptr(codes), _ptr(sf), float(g), rows, k, _ptr(y))
    else:
        raise ValueError(out)
    return y


def gemm_w4a4(a_codes, a_sf, g_a, b_codes, b_sf, g_b, rows: slice | None = None) -> np.ndarray:
    """Y = g_a g_b sum_k a^ b^ in double, Y = A B^T (A [M,K], B [N,K])."""
    L = lib()
    a_codes = np.ascontiguousarray(a_codes, np.uint8)
    b_codes = np.ascontiguousarray(b_codes, np.uint8)
    a_sf = np.ascontiguousarray(a_sf, np.uint8)
    b_sf = np.ascontiguousarray(b_sf, np.uint8)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = b_codes.shape[0]
    assert b_codes.shape[1] * 2 == K
    m0, m1 = (0, M) if rows is None else (rows.start or 0, rows.stop)
    y = np.empty((m1 - m0, N), np.float64)
    L.oracle_gemm_w4a4_rows(_ptr(a_codes), _ptr(a_sf), float(g_a), _ptr(b_codes), _ptr(b_sf),
                            float(g_b), M, N, K, m0, m1 - m0, _ptr(y))
    return y


def gemm_w4a4_at(a_codes, a_sf, g_a, b_codes, b_sf, g_b, m: int, n: int) -> float:
    L = lib()
    K = a_codes.shape[1] * 2
    return L.oracle_gemm_w4a4_at(_ptr(a_codes), _ptr(a_sf), float(g_a), _ptr(b_codes),
                                 _ptr(b_sf), float(g_b), K, int(m), int(n))


def gemm_w4a16(x, w_codes, w_sf, g_w, rows: slice | None = None) -> np.ndarray:
    """Y = g_w sum_k x w^ in double (bf16 activations, NVFP4 weights)."""
    L = lib()
    xb = bf16_bits(x)
    w_codes = np.ascontiguousarray(w_codes, np.uint8)
    w_sf = np.ascontiguousarray(w_sf, np.uint8)
    M, K = xb.shape
    N = w_codes.shape[0]
    m0, m1 = (0, M) if rows is None else (rows.start or 0, rows.stop)
    y = np.empty((m1 - m0, N), np.float64)
    L.oracle_gemm_w4a16_rows(_ptr(xb), _ptr(w_codes), _ptr(w_sf), float(g_w), M, N, K, m0,
                             m1 - m0, _ptr(y))
    return y


def gemm_w4a16_at(x_bits: np.ndarray, w_codes, w_sf, g_w, m: int, n: int) -> float:
    L = lib()
    K = x_bits.shape[1]
    return L.oracle_gemm_w4a16_at(_ptr(x_bits), _ptr(w_codes), _ptr(w_sf), float(g_w), K,
                                  int(m), int(n))


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """[rows, k/2] bytes -> [rows, k] nibbles (element 2j from the low nibble)."""
    lo = codes & 0x0F
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)


def sf_matrix(sf: np.ndarray, rows: int, k: int) -> np.ndarray:
    """Gather the scale bytes into a [rows, k/16] matrix through sf_offset."""
    kb = k // 16
    r = np.arange(rows)[:, None]
    c = np.arange(kb)[None, :]
    off = ((r // 128) * (kb // 4) + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
    return sf[off]


def tensor_scale(x) -> np.float32:
    """g = amax(|x|) / 2688 in IEEE single (the tensor-level scale of the RFC's
    two-level scaling)."""
    L = lib()
    if isinstance(x, np.ndarray) and x.dtype == np.float32:
        xa = np.ascontiguousarray(x)
        rows, k = xa.shape
        return np.float32(L.oracle_tensor_scale_f32(_ptr(xa), rows, k, k))
    xb = bf16_bits(x)
    rows, k = xb.shape
    return np.float32(L.oracle_tensor_scale_bf16(_ptr(xb), rows, k, k))


# ---------------------------------------------------------------- LayerNorm
def layernorm(x, gamma=None, beta=None, rows_per_group: int = 0, eps: float = 1e-6) -> np.ndarray:
    """LayerNorm over the last axis of a bf16 tensor with an optional affine per
    group of rows (the DiT pre-norm and its adaLN modulation; a reading, the
    pages do not define it): double statistics in index order, FP32
    normalisation, one rounding per operation.  gamma / beta: float32
    [groups, k] or [k].  Returns float32 [rows, k]."""
    L = lib()
    xb = bf16_bits(x)
    rows, k = xb.shape
    g = None if gamma is None else np.ascontiguousarray(np.asarray(gamma, np.float32).reshape(-1, k))
    b = None if beta is None else np.ascontiguousarray(np.asarray(beta, np.float32).reshape(-1, k))
    y = np.empty((rows, k), np.float32)
    L.oracle_layernorm_f32(_ptr(xb), rows, k, k, None if g is None else _ptr(g), None if b is None else _ptr(b),
                           int(rows_per_group), float(eps), _ptr(y))
    return y


def layernorm_quantize(x, gamma=None, beta=None, rows_per_group: int = 0, eps: float = 1e-6,
                       scale: float | None = None):
    """NVFP4 quantization (``quantize``) of the FP32 LayerNorm output: the
    fused producer's result.  Returns (codes, sf, g)."""
    return quantize(layernorm(x, gamma, beta, rows_per_group, eps), scale)


# ---------------------------------------------------------------- QAT
def fake_quantize(x, scale: float | None = None, out: str = "bf16", mask: bool = True):
    """Fake quantization for QAT (NVFP4-DiT README, Definition III.1, and
    Methodology 2's straight-through estimator): y = e2m1(code) * dec(sf) * g
    rounded once to bf16 (uint16 bits) or f32, with the codes and scales of
    ``quantize``; the clip mask marks s > 0 and |x| > 6 s, packed 8 elements
    per byte (element j of a row: bit j % 8 of byte j / 8).  Returns
    (y, mask or None, g)."""
    L = lib()
    xb = bf16_bits(x)
    rows, k = xb.shape
    assert k % 64 == 0
    y = np.empty((rows, k), np.float32 if out == "f32" else np.uint16)
    m = np.zeros((rows, k // 8), np.uint8) if mask else None
    g = np.zeros(1, np.float32)
    if scale is not None:
        g[0] = np.float32(scale)
    L.oracle_fake_quantize_bf16(_ptr(xb), rows, k, k, 1 if scale is not None else 0, _ptr(g),
                                1 if out == "f32" else 0, _ptr(y), _ptr(m) if m is not None else None)
    return y, m, np.float32(g[0])


def ste_backward(grad_y: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """Straight-through estimator backward with the clip mask: grad_y where
    the element was not clipped, +0 where it was.  ``grad_y`` is uint16 bf16
    bits or float32, shape [rows, k]."""
    L = lib()
    gy = np.ascontiguousarray(grad_y)
    assert gy.dtype in (np.uint16, np.float32)
    m = np.ascontiguousarray(mask, np.uint8)
    rows, k = gy.shape
    assert m.shape == (rows, k // 8)
    gx = np.empty_like(gy)
    L.oracle_ste_backward(_ptr(gy), _ptr(m), rows, k, gy.dtype.itemsize, _ptr(gx))
    return gx


# ---------------------------------------------------------------- epilogue activation
def gelu_tanh(v):
    """GELU, tanh form, in double (the fused GEMM epilogue's activation; the
    pages name none, a reading).  Scalar or float64 array."""
    L = lib()
    if np.isscalar(v):
        return float(L.oracle_gelu_tanh(float(v)))
    a = np.ascontiguousarray(v, np.float64)
    out = np.empty_like(a)
    L.oracle_gelu_tanh_array(_ptr(a), a.size, _ptr(out))
    return out


# ---------------------------------------------------------------- MXFP4
def mx_sf_bytes(rows: int, k: int) -> int:
    return int(lib().oracle_mx_sf_bytes(rows, k))


def mx_quantize(x):
    """MXFP4 (OCP MX reading): E2M1 codes [rows, k/2] and E8M0 block-32 scales
    in the tensor-core layout (k % 128 == 0)."""
    L = lib()
    xb = bf16_bits(x)
    rows, k = xb.shape
    assert k % 128 == 0
    codes = np.zeros((rows, k // 2), np.uint8)
    sf = np.zeros(mx_sf_bytes(rows, k), np.uint8)
    L.oracle_mx_quantize_bf16(_ptr(xb), rows, k, k, _ptr(codes), _ptr(sf))
    return codes, sf


def mx_dequantize(codes: np.ndarray, sf: np.ndarray) -> np.ndarray:
    L = lib()
    codes = np.ascontiguousarray(codes, np.uint8)
    sf = np.ascontiguousarray(sf, np.uint8)
    rows, kh = codes.shape
    out = np.empty((rows, kh * 2), np.float64)
    L.oracle_mx_dequantize_f64(_ptr(codes), _ptr(sf), rows, kh * 2, _ptr(out))
    return out


def mx_gemm(a_codes, a_sf, b_codes, b_sf, rows: slice | None = None) -> np.ndarray:
    """Y = A B^T of two MXFP4 operands, in double."""
    L = lib()
    a_codes = np.ascontiguousarray(a_codes, np.uint8)
    b_codes = np.ascontiguousarray(b_codes, np.uint8)
    a_sf = np.ascontiguousarray(a_sf, np.uint8)
    b_sf = np.ascontiguousarray(b_sf, np.uint8)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = b_codes.shape[0]
    m0, m1 = (0, M) if rows is None else (rows.start or 0, rows.stop)
    y = np.empty((m1 - m0, N), np.float64)
    L.oracle_mx_gemm_rows(_ptr(a_codes), _ptr(a_sf), _ptr(b_codes), _ptr(b_sf), N, K, m0, m1 - m0, _ptr(y))
    return y


def mx_sf_matrix(sf: np.ndarray, rows: int, k: int) -> np.ndarray:
    """The E8M0 bytes as a [rows, k/32] matrix."""
    kb = k // 32
    r = np.arange(rows)[:, None]
    c = np.arange(kb)[None, :]
    off = ((r // 128) * (kb // 4) + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
    return sf[off]


# ---------------------------------------------------------------- adaptive block size
BLOCK_SIZES = (1, 2, 4, 8, 16, 32, 64)


def quantize_block(x, block: int, scale: float | None = None):
    """NVFP4 with `block` values per E4M3 scale (16, 32 or 64), scales repeated
    into the block-16 layout.  Returns (codes, sf, g)."""
    L = lib()
    xb = bf16_bits(x)
    rows, k = xb.shape
    assert block in (16, 32, 64) and k % 64 == 0
    codes = np.zeros((rows, k // 2), np.uint8)
    sf = np.zeros(sf_bytes(rows, k), np.uint8)
    g = np.zeros(1, np.float32)
    if scale is not None:
        g[0] = np.float32(scale)
    L.oracle_quantize_block_bf16(_ptr(xb), rows, k, k, block, 1 if scale is not None else 0, _ptr(g),
                                 _ptr(codes), _ptr(sf))
    return codes, sf, np.float32(g[0])


def block_size_errors(x, g: float):
    """Squared quantization errors for b = 1, 2, ..., 64 (Eq. 9's Error before
    normalisation) and the sum of squares of x."""
    L = lib()
    xb = bf16_bits(x)
    rows, k = xb.shape
    err = np.zeros(7, np.float64)
    ss = np.zeros(1, np.float64)
    L.oracle_block_size_errors(_ptr(xb), rows, k, k, float(g), _ptr(err), _ptr(ss))
    return err, float(ss[0])


def select_block_size(err, sumsq: float, lam: float) -> int:
    """Eq. 9: argmin_b Error(b) / sum x^2 + lambda (4 + 8/b) / 12."""
    e = np.ascontiguousarray(err, np.float64)
    return int(lib().oracle_select_block_size(_ptr(e), float(sumsq), float(lam)))


# ---------------------------------------------------------------- attention
def attention(q, k, v, s_head, H: int, Lq: int, Lk: int, d: int, h: int, rows: slice | None = None) -> np.ndarray:
    """O of head h (Eq. 10 over NVFP4 Q, K, V; q/k/v = (codes, sf, g) of
    [H*Lq, d] / [H*Lk, d] tensors), query rows `rows` (all by default), in
    double."""
    L = lib()
    (qc, qs, gq), (kc, ks, gk), (vc, vs, gv) = q, k, v
    qc, qs, kc, ks, vc, vs = (np.ascontiguousarray(a, np.uint8) for a in (qc, qs, kc, ks, vc, vs))
    sh = np.ascontiguousarray(s_head, np.float64)
    q0, q1 = (0, Lq) if rows is None else (rows.start or 0, rows.stop)
    out = np.empty((q1 - q0, d), np.float64)
    L.oracle_attention_rows(_ptr(qc), _ptr(qs), float(gq), _ptr(kc), _ptr(ks), float(gk), _ptr(vc), _ptr(vs),
                            float(gv), Lq, Lk, d, _ptr(sh), h, q0, q1 - q0, _ptr(out))
    return out
