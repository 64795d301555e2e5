"""Attention over NVFP4 Q, K, V (Eq. 10) on the GPU vs the CPU oracle.

The oracle computes softmax(q^ k^T / sqrt(d) + log s_head) v^ in double from
the exact element values.  The kernel's deviations: P rounded to bf16 (2^-9
relative per element), the softmax sum taken over the unrounded values, FP32
accumulation, exp2 from the hardware approximation, and the bf16 output; so
per element |O - O_ref| <= 3e-3 max|v^| + 5e-3 |O_ref| (head-wise max)."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_gemm_quantize_b200 as nv
from nvfp4_w4a4_gemm_quantize_b200 import synth

pytestmark = pytest.mark.gpu

D = 128


def _upload(t):
    codes, sf, g = t
    q = nv.NVFP4Tensor.empty(codes.shape[0], codes.shape[1] * 2, "cuda")
    q.codes.copy_(torch.from_numpy(codes))
    q.sf[: sf.size].copy_(torch.from_numpy(sf))
    q.scale.fill_(float(g))
    return q


def _check(q, k, v, H, Lq, Lk, s_head=None, rows=None):
    Q, K, V = _upload(q), _upload(k), _upload(v)
    sh = torch.tensor(s_head, dtype=torch.float32, device="cuda") if s_head is not None else None
    o = nv.attention(Q, K, V, H, s_head=sh).float().cpu().numpy()
    vmax = np.abs(oracle.dequantize(*v)).reshape(H, Lk, D).max(axis=(1, 2))
    shd = np.asarray(s_head if s_head is not None else np.ones(H), np.float64)
    for h in range(H):
        sel = slice(None) if rows is None else rows
        ref = oracle.attention(q, k, v, shd, H, Lq, Lk, D, h, rows=sel if rows is not None else None)
        got = o[h * Lq:(h + 1) * Lq][sel]
        err = np.abs(got.astype(np.float64) - ref)
        assert np.all(err <= 3e-3 * vmax[h] + 5e-3 * np.abs(ref)), (h, float(err.max()))
    return o


def test_attention_small_all_rows(cuda_ok):
    H, Lq, Lk = 2, 128, 256
    q = oracle.quantize(synth.random_bf16((H * Lq, D), seed=70, dist="normal"))
    k = oracle.quantize(synth.random_bf16((H * Lk, D), seed=71, dist="normal"))
    v = oracle.quantize(synth.random_bf16((H * Lk, D), seed=72, dist="student_t3"))
    o1 = _check(q, k, v, H, Lq, Lk)
    # the per-head term shifts a head's logits by a constant: the same output
    o2 = _check(q, k, v, H, Lq, Lk, s_head=[0.25, 7.0])
    assert np.max(np.abs(o1 - o2)) <= 4e-3 * np.abs(o1).max()


def test_attention_sharp_rows_across_tiles(cuda_ok):
    """Queries aligned with one key each, the keys spread over all key tiles
    (the running maximum jumps late and early): the online rescaling."""
    H, Lq, Lk = 1, 256, 1024
    rng = np.random.default_rng(73)
    kx = rng.standard_normal((Lk, D)).astype(np.float32)
    qx = np.zeros((Lq, D), np.float32)
    for i in range(Lq):
        qx[i] = 3.0 * kx[(7 * i + 100) % Lk] + 0.1 * rng.standard_normal(D).astype(np.float32)
    q = oracle.quantize(torch.from_numpy(qx).bfloat16())
    k = oracle.quantize(torch.from_numpy(kx).bfloat16())
    v = oracle.quantize(synth.random_bf16((Lk, D), seed=74, dist="normal"))
    _check(q, k, v, H, Lq, Lk)


def test_attention_larger_sampled_rows_gpu_quantized(cuda_ok):
    """GPU-quantized operands (bit-exact with the oracle's quantization, as the
    quantize tests show), several heads, sampled query rows."""
    H, Lq, Lk = 4, 512, 1024
    xq = synth.random_bf16((H * Lq, D), seed=75, dist="token_scaled")
    xk = synth.random_bf16((H * Lk, D), seed=76, dist="normal")
    xv = synth.random_bf16((H * Lk, D), seed=77, dist="outlier")
    Q, K, V = nv.quantize(xq.cuda()), nv.quantize(xk.cuda()), nv.quantize(xv.cuda())
    o = nv.attention(Q, K, V, H).float().cpu().numpy()
    q, k, v = oracle.quantize(xq), oracle.quantize(xk), oracle.quantize(xv)
    vmax = np.abs(oracle.dequantize(*v)).reshape(H, Lk, D).max(axis=(1, 2))
    rows = np.array([0, 1, 127, 128, 300, 511])
    for h in range(H):
        for r in rows:
            ref = oracle.attention(q, k, v, np.ones(H), H, Lq, Lk, D, h, rows=slice(int(r), int(r) + 1))[0]
            err = np.abs(o[h * Lq + r].astype(np.float64) - ref)
            assert np.all(err <= 3e-3 * vmax[h] + 5e-3 * np.abs(ref))
