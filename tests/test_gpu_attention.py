"""Attention over NVFP4 Q, K, V (Eq. 10) on the GPU vs the CPU oracle.

The oracle computes softmax(q^ k^T / sqrt(d) + log s_head) v^ in double from
the exact element values.  The kernel's deviations: P rounded to f16 (up to 2^-11
relative per element for P >= 2^-14 of the running reference, an absolute 2^-25 below
it), the softmax sum taken over the unrounded values, FP32
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


@pytest.mark.parametrize("tiles", ["2", "1"])
def test_attention_sharp_rows_across_tiles(cuda_ok, monkeypatch, tiles):
    """Queries aligned with one key each, the keys spread over all key tiles
    (the running maximum jumps late and early): the online rescaling.  Two
    query tiles per CTA (the default for an even number of tiles) and one
    (NVFP4_ATTN_TILES=1, the kernel of odd tile counts)."""
    monkeypatch.setenv("NVFP4_ATTN_TILES", tiles)
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


def _sampled_heads(xq, xk, xv, H, Lq, Lk, heads, rows, s_head=None):
    """The kernel on the whole tensors (GPU-quantized) against the oracle on
    the sampled heads' slices, quantized with the whole tensors' scales."""
    Q, K, V = nv.quantize(xq.cuda()), nv.quantize(xk.cuda()), nv.quantize(xv.cuda())
    sh_dev = torch.tensor(s_head, dtype=torch.float32, device="cuda") if s_head is not None else None
    o = nv.attention(Q, K, V, H, s_head=sh_dev)
    torch.cuda.synchronize()
    gq, gk, gv = (oracle.tensor_scale(x) for x in (xq, xk, xv))
    for h in heads:
        q = oracle.quantize(xq[h * Lq:(h + 1) * Lq], gq)
        k = oracle.quantize(xk[h * Lk:(h + 1) * Lk], gk)
        v = oracle.quantize(xv[h * Lk:(h + 1) * Lk], gv)
        vmax = np.abs(oracle.dequantize(*v)).max()
        sh = np.array([1.0 if s_head is None else s_head[h]])
        got = o[h * Lq:(h + 1) * Lq].float().cpu().numpy()
        for r in rows:
            ref = oracle.attention(q, k, v, sh, 1, Lq, Lk, D, 0, rows=slice(int(r), int(r) + 1))[0]
            err = np.abs(got[r].astype(np.float64) - ref)
            assert np.all(err <= 3e-3 * vmax + 5e-3 * np.abs(ref)), (h, r, float(err.max()))


# "fused": the two-tile kernel decodes V itself, each work item a share of its
# head's rows, two rounds ahead; "prepass": a separate V decode kernel first.
DECODE = ["fused", "prepass"]


@pytest.fixture
def decode(request, monkeypatch):
    if request.param == "prepass":
        monkeypatch.setenv("NVFP4_ATTN_DECODE", "prepass")
    return request.param


@pytest.mark.parametrize("decode", DECODE, indirect=True)
def test_attention_several_items_per_cta(cuda_ok, decode):
    """More work items (head, 256-query pair of tiles) than SMs: each
    persistent CTA takes several, over different heads with different s_head;
    ring slots and barrier phases run on across the item boundaries, and a
    head's items fall in two rounds."""
    H, Lq, Lk = 24, 2048, 512
    xq = synth.random_bf16((H * Lq, D), seed=78, dist="token_scaled")
    xk = synth.random_bf16((H * Lk, D), seed=79, dist="normal")
    xv = synth.random_bf16((H * Lk, D), seed=80, dist="student_t3")
    s_head = [0.5 + 0.25 * h for h in range(H)]
    _sampled_heads(xq, xk, xv, H, Lq, Lk, heads=(0, 9, 10, 18, 23), rows=(0, 129, 1151, 2047), s_head=s_head)


@pytest.mark.parametrize("decode", DECODE, indirect=True)
def test_attention_full_size_sampled(cuda_ok, decode):
    """The video DiT's spatial attention as timed: 384 heads x 2048 tokens,
    d = 128 (3072 work items on the persistent grid), sampled heads and rows."""
    H, L = 384, 2048
    xs = [synth.random_bf16((H * L, D), seed=90 + i, dist="normal") for i in range(3)]
    _sampled_heads(*xs, H, L, L, heads=(0, 147, 148, 295, 383), rows=(0, 777, 2047))


def test_attention_decode_parts_with_empty_shares(cuda_ok):
    """24 work items per head over 128 keys: shares of ceil(128 / 24) = 6 rows,
    the last two empty; 480 items, so shares are also decoded two rounds ahead
    in the kernel's main loop -- empty ones must still be marked done."""
    H, Lq, Lk = 20, 6144, 128
    xq = synth.random_bf16((H * Lq, D), seed=81, dist="normal")
    xk = synth.random_bf16((H * Lk, D), seed=82, dist="normal")
    xv = synth.random_bf16((H * Lk, D), seed=83, dist="outlier")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    Q, K, V = nv.quantize(xq.cuda()), nv.quantize(xk.cuda()), nv.quantize(xv.cuda())
    nv.attention(Q, K, V, H, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    _sampled_heads(xq, xk, xv, H, Lq, Lk, heads=(0, 7, 19), rows=(0, 3001, 6143))


def test_attention_more_items_per_head_than_slots(cuda_ok):
    """33 work items per head (Lq = 8448): more than the 32 decode slots of a
    head, so the library decodes V in a separate pass first; the two-tile
    kernel then reads it as when it decodes V itself."""
    H, Lq, Lk = 2, 8448, 256
    xq = synth.random_bf16((H * Lq, D), seed=84, dist="normal")
    xk = synth.random_bf16((H * Lk, D), seed=85, dist="normal")
    xv = synth.random_bf16((H * Lk, D), seed=86, dist="student_t3")
    _sampled_heads(xq, xk, xv, H, Lq, Lk, heads=(0, 1), rows=(0, 4321, 8447))
