"""NVFP4 two-level quantization and block-scaled FP4 GEMMs for B200 (sm_100a).

Python binding of the C ABI in include/nvfp4.h.  Every function below only
marshals torch tensors into pointers and sizes and calls the library of the
same name; all arithmetic runs in the CUDA kernels.  torch supplies device
memory and streams.  Every tensor must live on the current CUDA device (the
library launches there; nothing here switches devices), and the default stream
argument is that device's current torch stream.

Low-level (same names and argument order as the C calls):
    nvfp4_sf_bytes, nvfp4_quantize_workspace_bytes, nvfp4_quantize,
    nvfp4_quantize_noalloc, nvfp4_layernorm_quantize, nvfp4_quantize_block, nvfp4_block_size_errors, nvfp4_select_block_size,
    nvfp4_dequantize, nvfp4_fake_quantize, nvfp4_ste_backward,
    nvfp4_gemm_w4a4, nvfp4_gemm_w4a4_grouped, nvfp4_gemm_w4a16, nvfp4_mx_sf_bytes, nvfp4_mx_quantize,
    nvfp4_mx_dequantize, nvfp4_mx_gemm, nvfp4_attention, nvfp4_attention_workspace_bytes, nvfp4_launch_count
Convenience (allocate outputs with torch, then call the above):
    NVFP4Tensor, quantize, layernorm_quantize, dequantize, gemm_w4a4, gemm_w4a4_nvfp4_out, gemm_w4a4_grouped,
    gemm_w4a16,
    fake_quantize, ste_backward, FakeQuantizeSTE (autograd: the two kernels),
    MXTensor, mx_quantize, mx_dequantize, mx_gemm, quantize_block, block_size_errors, select_block_size,
    attention
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from ._lib import MAX_GROUP, NVFP4Error, NVFP4GemmProblem, check, lib  # noqa: F401

NVFP4_DTYPE_BF16 = 0
NVFP4_DTYPE_F32 = 1
NVFP4_SCALE_GIVEN = 1
NVFP4_ACT_NONE = 0
NVFP4_ACT_GELU_TANH = 1

_DT = {torch.bfloat16: NVFP4_DTYPE_BF16, torch.float32: NVFP4_DTYPE_F32}


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


# ----------------------------------------------------------------- C ABI
def nvfp4_sf_bytes(rows: int, k: int) -> int:
    return int(lib().nvfp4_sf_bytes(rows, k))


def nvfp4_quantize_workspace_bytes(rows: int, k: int) -> int:
    return int(lib().nvfp4_quantize_workspace_bytes(rows, k))


def nvfp4_launch_count() -> int:
    return int(lib().nvfp4_launch_count())


def nvfp4_shutdown() -> None:
    lib().nvfp4_shutdown()


def nvfp4_debug_wait_timeout(dev_status, limit_us: int, stream=None) -> None:
    """Check of the failure detection: one warp waits, with the library's
    bounded wait, on a barrier nothing arrives at, gives up after limit_us and
    writes NVFP4_ERR_TIMEOUT to dev_status (a zeroed device int32)."""
    st = lib().nvfp4_debug_wait_timeout(_ptr(dev_status), limit_us, _stream(stream))
    check(st, "nvfp4_debug_wait_timeout")


def nvfp4_quantize(x, rows, k, ld_x, codes, sf, tensor_scale, flags=0, workspace=None,
                   workspace_bytes=0, dev_status=None, stream=None) -> None:
    st = lib().nvfp4_quantize(_ptr(x), rows, k, ld_x, _ptr(codes), _ptr(sf), _ptr(tensor_scale),
                              flags, _ptr(workspace), workspace_bytes, _ptr(dev_status), _stream(stream))
    check(st, "nvfp4_quantize")


def nvfp4_layernorm_quantize(x, rows, k, ld_x, gamma, beta, rows_per_group, eps, codes, sf, tensor_scale, flags=0,
                             workspace=None, workspace_bytes=0, dev_status=None, stream=None) -> None:
    st = lib().nvfp4_layernorm_quantize(_ptr(x), rows, k, ld_x, _ptr(gamma), _ptr(beta), rows_per_group, float(eps),
                                        _ptr(codes), _ptr(sf), _ptr(tensor_scale), flags, _ptr(workspace),
                                        workspace_bytes, _ptr(dev_status), _stream(stream))
    check(st, "nvfp4_layernorm_quantize")


def nvfp4_quantize_noalloc(x, rows, k, ld_x, codes, sf, tensor_scale, flags=0, dev_status=None,
                           stream=None) -> None:
    """nvfp4_quantize without a workspace argument, for callers that cannot
    allocate device memory (the amax scratch is a fixed device array inside the
    library; overlapping calls race, see include/nvfp4.h)."""
    st = lib().nvfp4_quantize_noalloc(_ptr(x), rows, k, ld_x, _ptr(codes), _ptr(sf), _ptr(tensor_scale), flags,
                                      _ptr(dev_status), _stream(stream))
    check(st, "nvfp4_quantize_noalloc")


def nvfp4_quantize_block(x, rows, k, ld_x, block, codes, sf, tensor_scale, flags=0, workspace=None,
                         workspace_bytes=0, dev_status=None, stream=None) -> None:
    st = lib().nvfp4_quantize_block(_ptr(x), rows, k, ld_x, block, _ptr(codes), _ptr(sf), _ptr(tensor_scale), flags,
                                    _ptr(workspace), workspace_bytes, _ptr(dev_status), _stream(stream))
    check(st, "nvfp4_quantize_block")


def nvfp4_block_size_errors(x, rows, k, ld_x, tensor_scale, errors, stream=None) -> None:
    check(lib().nvfp4_block_size_errors(_ptr(x), rows, k, ld_x, _ptr(tensor_scale), _ptr(errors), _stream(stream)),
          "nvfp4_block_size_errors")


def nvfp4_select_block_size(errors_host, lam: float) -> int:
    """Eq. 9 on a host sequence of 8 doubles (the device errors copied back)."""
    arr = (ctypes.c_double * 8)(*[float(v) for v in errors_host])
    return int(lib().nvfp4_select_block_size(ctypes.addressof(arr), float(lam)))


def nvfp4_dequantize(codes, sf, tensor_scale, rows, k, out, out_dtype, stream=None) -> None:
    st = lib().nvfp4_dequantize(_ptr(codes), _ptr(sf), _ptr(tensor_scale), rows, k, _ptr(out),
                                out_dtype, _stream(stream))
    check(st, "nvfp4_dequantize")


def nvfp4_fake_quantize(x, rows, k, ld_x, y, y_dtype, clip_mask, tensor_scale, flags=0, workspace=None,
                        workspace_bytes=0, dev_status=None, stream=None) -> None:
    st = lib().nvfp4_fake_quantize(_ptr(x), rows, k, ld_x, _ptr(y), y_dtype, _ptr(clip_mask), _ptr(tensor_scale),
                                   flags, _ptr(workspace), workspace_bytes, _ptr(dev_status), _stream(stream))
    check(st, "nvfp4_fake_quantize")


def nvfp4_ste_backward(grad_y, clip_mask, rows, k, dtype, grad_x, stream=None) -> None:
    st = lib().nvfp4_ste_backward(_ptr(grad_y), _ptr(clip_mask), rows, k, dtype, _ptr(grad_x), _stream(stream))
    check(st, "nvfp4_ste_backward")


def nvfp4_gemm_w4a4(a_codes, a_sf, a_scale, b_codes, b_sf, b_scale, M, N, K, y=None,
                    y_dtype=NVFP4_DTYPE_BF16, y_codes=None, y_sf=None, y_scale=None, y_amax=None,
                    act=0, dev_status=None, stream=None) -> None:
    st = lib().nvfp4_gemm_w4a4(_ptr(a_codes), _ptr(a_sf), _ptr(a_scale), _ptr(b_codes), _ptr(b_sf),
                               _ptr(b_scale), M, N, K, _ptr(y), y_dtype, _ptr(y_codes), _ptr(y_sf),
                               _ptr(y_scale), _ptr(y_amax), act, _ptr(dev_status), _stream(stream))
    check(st, "nvfp4_gemm_w4a4")


def nvfp4_gemm_w4a4_grouped(problems, y_dtype=NVFP4_DTYPE_BF16, dev_status=None, stream=None) -> None:
    """``problems``: a list of dicts with the fields of nvfp4_gemm_problem
    (tensors or None for the pointers, ints for M, N, K)."""
    arr = (NVFP4GemmProblem * len(problems))()
    for i, d in enumerate(problems):
        for name, _ in NVFP4GemmProblem._fields_:
            v = d.get(name)
            setattr(arr[i], name, int(v or 0) if name in ("M", "N", "K", "act") else _ptr(v))
    st = lib().nvfp4_gemm_w4a4_grouped(ctypes.addressof(arr), len(problems), y_dtype, _ptr(dev_status),
                                       _stream(stream))
    check(st, "nvfp4_gemm_w4a4_grouped")


def nvfp4_mx_sf_bytes(rows: int, k: int) -> int:
    return int(lib().nvfp4_mx_sf_bytes(rows, k))


def nvfp4_mx_quantize(x, rows, k, ld_x, codes, sf, stream=None) -> None:
    check(lib().nvfp4_mx_quantize(_ptr(x), rows, k, ld_x, _ptr(codes), _ptr(sf), _stream(stream)),
          "nvfp4_mx_quantize")


def nvfp4_mx_dequantize(codes, sf, rows, k, out, out_dtype, stream=None) -> None:
    check(lib().nvfp4_mx_dequantize(_ptr(codes), _ptr(sf), rows, k, _ptr(out), out_dtype, _stream(stream)),
          "nvfp4_mx_dequantize")


def nvfp4_mx_gemm(a_codes, a_sf, b_codes, b_sf, M, N, K, y, y_dtype=NVFP4_DTYPE_BF16, act=0, dev_status=None,
                  stream=None) -> None:
    check(lib().nvfp4_mx_gemm(_ptr(a_codes), _ptr(a_sf), _ptr(b_codes), _ptr(b_sf), M, N, K, _ptr(y), y_dtype, act,
                              _ptr(dev_status), _stream(stream)), "nvfp4_mx_gemm")


def nvfp4_attention_workspace_bytes(H: int, Lk: int, d: int) -> int:
    return int(lib().nvfp4_attention_workspace_bytes(H, Lk, d))


def nvfp4_attention(q_codes, q_sf, q_scale, k_codes, k_sf, k_scale, v_codes, v_sf, v_scale, s_head, H, Lq, Lk, d,
                    out, workspace, workspace_bytes, dev_status=None, stream=None) -> None:
    check(lib().nvfp4_attention(_ptr(q_codes), _ptr(q_sf), _ptr(q_scale), _ptr(k_codes), _ptr(k_sf), _ptr(k_scale),
                                _ptr(v_codes), _ptr(v_sf), _ptr(v_scale), _ptr(s_head), H, Lq, Lk, d, _ptr(out),
                                _ptr(workspace), workspace_bytes, _ptr(dev_status), _stream(stream)),
          "nvfp4_attention")


def nvfp4_gemm_w4a16(x, w_codes, w_sf, w_scale, M, N, K, y, y_dtype=NVFP4_DTYPE_BF16,
                     dev_status=None, stream=None) -> None:
    st = lib().nvfp4_gemm_w4a16(_ptr(x), _ptr(w_codes), _ptr(w_sf), _ptr(w_scale), M, N, K, _ptr(y),
                                y_dtype, _ptr(dev_status), _stream(stream))
    check(st, "nvfp4_gemm_w4a16")


# ----------------------------------------------------------------- convenience
@dataclass
class NVFP4Tensor:
    """codes [rows, k/2] uint8, sf [sf_bytes] uint8 (tensor-core layout),
    scale [1] float32 -- all on one CUDA device."""
    codes: torch.Tensor
    sf: torch.Tensor
    scale: torch.Tensor
    rows: int
    k: int

    @staticmethod
    def empty(rows: int, k: int, device) -> "NVFP4Tensor":
        return NVFP4Tensor(torch.empty(rows, k // 2, dtype=torch.uint8, device=device),
                           torch.empty(max(nvfp4_sf_bytes(rows, k), 16), dtype=torch.uint8, device=device),
                           torch.zeros(1, dtype=torch.float32, device=device), rows, k)


def quantize(x: torch.Tensor, scale: torch.Tensor | float | None = None, out: NVFP4Tensor | None = None,
             workspace: torch.Tensor | None = None, dev_status=None, stream=None) -> NVFP4Tensor:
    """Quantize a bf16 [rows, k] CUDA tensor.  ``scale`` given -> used as the
    tensor scale g; otherwise g = amax / 2688 is computed on the device."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, k = x.shape
    q = out if out is not None else NVFP4Tensor.empty(rows, k, x.device)
    flags = 0
    if scale is not None:
        if isinstance(scale, torch.Tensor):
            q.scale.copy_(scale.reshape(1).to(torch.float32))
        else:
            q.scale.fill_(float(scale))
        flags = NVFP4_SCALE_GIVEN
    wsb = nvfp4_quantize_workspace_bytes(rows, k)
    if flags == 0 and workspace is None:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=x.device)
    nvfp4_quantize(x, rows, k, x.stride(0), q.codes, q.sf, q.scale, flags,
                   workspace if flags == 0 else None, wsb if flags == 0 else 0, dev_status, stream)
    return q


def layernorm_quantize(x: torch.Tensor, gamma: torch.Tensor | None = None, beta: torch.Tensor | None = None,
                       rows_per_group: int = 0, eps: float = 1e-6, scale: torch.Tensor | float | None = None,
                       out: NVFP4Tensor | None = None, workspace: torch.Tensor | None = None, dev_status=None,
                       stream=None) -> NVFP4Tensor:
    """LayerNorm of a bf16 [rows, k] CUDA tensor (optional FP32 affine per
    group of rows_per_group rows: gamma / beta [groups, k]) emitted directly as
    NVFP4.  ``scale`` given -> the tensor scale; otherwise the largest |y| / 2688."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, k = x.shape
    for t in (gamma, beta):
        assert t is None or (t.dtype == torch.float32 and t.is_contiguous() and t.shape[-1] == k)
    q = out if out is not None else NVFP4Tensor.empty(rows, k, x.device)
    flags = 0
    if scale is not None:
        if isinstance(scale, torch.Tensor):
            q.scale.copy_(scale.reshape(1).to(torch.float32))
        else:
            q.scale.fill_(float(scale))
        flags = NVFP4_SCALE_GIVEN
    wsb = nvfp4_quantize_workspace_bytes(rows, k)
    if flags == 0 and workspace is None:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=x.device)
    nvfp4_layernorm_quantize(x, rows, k, x.stride(0), gamma, beta, rows_per_group, eps, q.codes, q.sf, q.scale, flags,
                             workspace if flags == 0 else None, wsb if flags == 0 else 0, dev_status, stream)
    return q


def dequantize(q: NVFP4Tensor, dtype=torch.bfloat16, stream=None) -> torch.Tensor:
    out = torch.empty(q.rows, q.k, dtype=dtype, device=q.codes.device)
    nvfp4_dequantize(q.codes, q.sf, q.scale, q.rows, q.k, out, _DT[dtype], stream)
    return out


def gemm_w4a4(a: NVFP4Tensor, b: NVFP4Tensor, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
              act=NVFP4_ACT_NONE, dev_status=None, stream=None) -> torch.Tensor:
    """Y = act(A B^T), A [M,K] activations, B [N,K] weights, both NVFP4."""
    assert a.k == b.k
    y = out if out is not None else torch.empty(a.rows, b.rows, dtype=out_dtype, device=a.codes.device)
    nvfp4_gemm_w4a4(a.codes, a.sf, a.scale, b.codes, b.sf, b.scale, a.rows, b.rows, a.k, y=y,
                    y_dtype=_DT[y.dtype], act=act, dev_status=dev_status, stream=stream)
    return y


def gemm_w4a4_nvfp4_out(a: NVFP4Tensor, b: NVFP4Tensor, y_scale: torch.Tensor, y_amax: torch.Tensor | None = None,
                        out: NVFP4Tensor | None = None, act=NVFP4_ACT_NONE, dev_status=None,
                        stream=None) -> NVFP4Tensor:
    """act(Y = A B^T) emitted directly as NVFP4 with the caller's tensor scale."""
    q = out if out is not None else NVFP4Tensor.empty(a.rows, b.rows, a.codes.device)
    q.scale.copy_(y_scale.reshape(1))
    nvfp4_gemm_w4a4(a.codes, a.sf, a.scale, b.codes, b.sf, b.scale, a.rows, b.rows, a.k,
                    y_codes=q.codes, y_sf=q.sf, y_scale=q.scale, y_amax=y_amax, act=act, dev_status=dev_status,
                    stream=stream)
    return q


def gemm_w4a4_grouped(pairs, out_dtype=torch.bfloat16, act=NVFP4_ACT_NONE, dev_status=None, stream=None) -> list:
    """Y_i = A_i B_i^T for up to MAX_GROUP independent (A_i, B_i) NVFP4 pairs in
    one launch; returns the outputs in order."""
    ys, probs = [], []
    for a, b in pairs:
        assert a.k == b.k
        y = torch.empty(a.rows, b.rows, dtype=out_dtype, device=a.codes.device)
        ys.append(y)
        probs.append(dict(a_codes=a.codes, a_sf=a.sf, a_scale=a.scale, b_codes=b.codes, b_sf=b.sf,
                          b_scale=b.scale, M=a.rows, N=b.rows, K=a.k, y=y, act=act))
    nvfp4_gemm_w4a4_grouped(probs, _DT[out_dtype], dev_status, stream)
    return ys


def gemm_w4a16(x: torch.Tensor, w: NVFP4Tensor, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
               dev_status=None, stream=None) -> torch.Tensor:
    """Y = X W^T, X bf16 [M,K], W NVFP4 [N,K]."""
    assert x.dtype == torch.bfloat16 and x.is_contiguous() and x.shape[1] == w.k
    y = out if out is not None else torch.empty(x.shape[0], w.rows, dtype=out_dtype, device=x.device)
    nvfp4_gemm_w4a16(x, w.codes, w.sf, w.scale, x.shape[0], w.rows, w.k, y, _DT[y.dtype], dev_status, stream)
    return y


# ----------------------------------------------------------------- QAT
def fake_quantize(x: torch.Tensor, scale: torch.Tensor | float | None = None, out_dtype=torch.bfloat16,
                  clip_mask: bool = True, workspace: torch.Tensor | None = None, dev_status=None, stream=None):
    """Fake-quantize a bf16 [rows, k] CUDA tensor: returns (y, mask, scale) with
    y = the NVFP4 value of each element (bf16 or f32), mask the packed clip
    bits ([rows, k/8] uint8, None unless ``clip_mask``) and scale the tensor
    scale used (computed on the device unless given)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, k = x.shape
    y = torch.empty(rows, k, dtype=out_dtype, device=x.device)
    m = torch.empty(rows, k // 8, dtype=torch.uint8, device=x.device) if clip_mask else None
    g = torch.zeros(1, dtype=torch.float32, device=x.device)
    flags = 0
    if scale is not None:
        if isinstance(scale, torch.Tensor):
            g.copy_(scale.reshape(1).to(torch.float32))
        else:
            g.fill_(float(scale))
        flags = NVFP4_SCALE_GIVEN
    wsb = nvfp4_quantize_workspace_bytes(rows, k)
    if flags == 0 and workspace is None:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=x.device)
    nvfp4_fake_quantize(x, rows, k, x.stride(0), y, _DT[out_dtype], m, g, flags,
                        workspace if flags == 0 else None, wsb if flags == 0 else 0, dev_status, stream)
    return y, m, g


def ste_backward(grad_y: torch.Tensor, clip_mask: torch.Tensor, out: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """grad_y where the clip mask is clear, +0 where set (``out`` may be grad_y)."""
    assert grad_y.dim() == 2 and grad_y.is_contiguous() and grad_y.dtype in _DT
    rows, k = grad_y.shape
    gx = out if out is not None else torch.empty_like(grad_y)
    nvfp4_ste_backward(grad_y, clip_mask, rows, k, _DT[grad_y.dtype], gx, stream)
    return gx


class FakeQuantizeSTE(torch.autograd.Function):
    """Autograd wrapper of the two kernels: forward = nvfp4_fake_quantize,
    backward = nvfp4_ste_backward with the forward's clip mask (masked=True)
    or the identity (masked=False, the plain straight-through estimator)."""

    @staticmethod
    def forward(ctx, x, scale=None, masked=True):
        y, m, _ = fake_quantize(x, scale, clip_mask=masked)
        ctx.save_for_backward(*([m] if masked else []))
        ctx.masked = masked
        return y

    @staticmethod
    def backward(ctx, grad_y):
        if not ctx.masked:
            return grad_y, None, None
        (m,) = ctx.saved_tensors
        return ste_backward(grad_y.contiguous(), m), None, None


# ----------------------------------------------------------------- MX variant
@dataclass
class MXTensor:
    """codes [rows, k/2] uint8, sf [mx_sf_bytes] uint8 (E8M0, block 32)."""
    codes: torch.Tensor
    sf: torch.Tensor
    rows: int
    k: int

    @staticmethod
    def empty(rows: int, k: int, device) -> "MXTensor":
        return MXTensor(torch.empty(rows, k // 2, dtype=torch.uint8, device=device),
                        torch.empty(max(nvfp4_mx_sf_bytes(rows, k), 16), dtype=torch.uint8, device=device), rows, k)


def mx_quantize(x: torch.Tensor, out: MXTensor | None = None, stream=None) -> MXTensor:
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, k = x.shape
    q = out if out is not None else MXTensor.empty(rows, k, x.device)
    nvfp4_mx_quantize(x, rows, k, x.stride(0), q.codes, q.sf, stream)
    return q


def mx_dequantize(q: MXTensor, dtype=torch.bfloat16, stream=None) -> torch.Tensor:
    out = torch.empty(q.rows, q.k, dtype=dtype, device=q.codes.device)
    nvfp4_mx_dequantize(q.codes, q.sf, q.rows, q.k, out, _DT[dtype], stream)
    return out


def mx_gemm(a: MXTensor, b: MXTensor, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
            act=NVFP4_ACT_NONE, dev_status=None, stream=None) -> torch.Tensor:
    assert a.k == b.k
    y = out if out is not None else torch.empty(a.rows, b.rows, dtype=out_dtype, device=a.codes.device)
    nvfp4_mx_gemm(a.codes, a.sf, b.codes, b.sf, a.rows, b.rows, a.k, y, _DT[y.dtype], act, dev_status, stream)
    return y


# ----------------------------------------------------------------- block size (Algorithm 1 / Eq. 9)
def quantize_block(x: torch.Tensor, block: int, scale: torch.Tensor | float | None = None,
                   out: NVFP4Tensor | None = None, workspace: torch.Tensor | None = None, dev_status=None,
                   stream=None) -> NVFP4Tensor:
    """quantize() with `block` (16, 32, 64) values per scale; scales repeated in
    the block-16 layout, so gemm_w4a4 takes the result as it is."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, k = x.shape
    q = out if out is not None else NVFP4Tensor.empty(rows, k, x.device)
    flags = 0
    if scale is not None:
        if isinstance(scale, torch.Tensor):
            q.scale.copy_(scale.reshape(1).to(torch.float32))
        else:
            q.scale.fill_(float(scale))
        flags = NVFP4_SCALE_GIVEN
    wsb = nvfp4_quantize_workspace_bytes(rows, k)
    if flags == 0 and workspace is None:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=x.device)
    nvfp4_quantize_block(x, rows, k, x.stride(0), block, q.codes, q.sf, q.scale, flags,
                         workspace if flags == 0 else None, wsb if flags == 0 else 0, dev_status, stream)
    return q


def block_size_errors(x: torch.Tensor, tensor_scale: torch.Tensor, stream=None) -> torch.Tensor:
    """Device float64 [8]: squared errors for b = 1, 2, ..., 64 and sum x^2."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    errors = torch.empty(8, dtype=torch.float64, device=x.device)
    nvfp4_block_size_errors(x, x.shape[0], x.shape[1], x.stride(0), tensor_scale, errors, stream)
    return errors


def select_block_size(x: torch.Tensor, lam: float, tensor_scale: torch.Tensor | None = None) -> int:
    """Algorithm 1 / Eq. 9 for one tensor: errors on the device, the argmin on
    the host (one 64-byte copy)."""
    if tensor_scale is None:
        tensor_scale = quantize(x).scale
    return nvfp4_select_block_size(block_size_errors(x, tensor_scale).cpu().tolist(), lam)


# ----------------------------------------------------------------- attention (Eq. 10)
def attention(q: NVFP4Tensor, k: NVFP4Tensor, v: NVFP4Tensor, H: int, s_head: torch.Tensor | None = None,
              out: torch.Tensor | None = None, workspace: torch.Tensor | None = None, dev_status=None,
              stream=None) -> torch.Tensor:
    """softmax(Q K^T / sqrt(d) + log s_head) V per head over NVFP4 Q [H*Lq, d],
    K and V [H*Lk, d] (d = 128); returns bf16 [H*Lq, d]."""
    d = q.k
    Lq, Lk = q.rows // H, k.rows // H
    o = out if out is not None else torch.empty(q.rows, d, dtype=torch.bfloat16, device=q.codes.device)
    wsb = nvfp4_attention_workspace_bytes(H, Lk, d)
    if workspace is None:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=q.codes.device)
    nvfp4_attention(q.codes, q.sf, q.scale, k.codes, k.sf, k.scale, v.codes, v.sf, v.scale, s_head, H, Lq, Lk, d, o,
                    workspace, wsb, dev_status, stream)
    return o
