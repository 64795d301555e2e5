"""Grouped W4A4 launch vs the CPU oracle.

Several independent problems run in one persistent launch; each output must
meet the same tolerances as a single call (2e-3 normalised for bf16, 1e-5 for
FP32), be bit-identical to the single call of the same kernel (N % 256 != 0:
same tiles, same accumulation order), and, for the NVFP4-emitting epilogue
with exactly representable products, match the oracle's codes bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_gemm_quantize_b200 as nv
from nvfp4_w4a4_gemm_quantize_b200 import synth

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-3
TOL_F32 = 1e-5


def upload(codes, sf, g, rows, k) -> nv.NVFP4Tensor:
    q = nv.NVFP4Tensor.empty(rows, k, "cuda")
    q.codes.copy_(torch.from_numpy(np.ascontiguousarray(codes)))
    q.sf[: sf.size].copy_(torch.from_numpy(sf))
    q.scale.fill_(float(g))
    return q


def norm_err(y_gpu, y_ref, a_deq, b_deq):
    na = np.linalg.norm(a_deq, axis=1)[:, None]
    nb = np.linalg.norm(b_deq, axis=1)[None, :]
    den = na * nb
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    return float(np.max(np.where(den > 0, err / np.where(den > 0, den, 1.0), err)))


def _operands(M, N, K, seed, dist="student_t3"):
    x = synth.random_bf16((M, K), seed=seed, dist=dist)
    w = synth.random_bf16((N, K), seed=seed + 1, dist="normal", scale=0.02)
    ac, asf, ga = oracle.quantize(x)
    bc, bsf, gb = oracle.quantize(w)
    return (ac, asf, ga), (bc, bsf, gb)


@pytest.mark.parametrize("out_dtype,tol", [(torch.bfloat16, TOL_BF16), (torch.float32, TOL_F32)])
def test_grouped_matches_oracle_and_single_calls(cuda_ok, out_dtype, tol):
    shapes = [(300, 384, 1152), (128, 256, 256), (77, 1152, 4096), (1, 136, 64), (513, 648, 320)]
    ops = [_operands(M, N, K, 40 + i) for i, (M, N, K) in enumerate(shapes)]
    pairs = [(upload(*a, M, K), upload(*b, N, K)) for (a, b), (M, N, K) in zip(ops, shapes)]
    ys = nv.gemm_w4a4_grouped(pairs, out_dtype=out_dtype)
    singles = [nv.gemm_w4a4(A, B, out_dtype=out_dtype) for A, B in pairs]
    torch.cuda.synchronize()
    for (a, b), (M, N, K), y, y1 in zip(ops, shapes, ys, singles):
        yref = oracle.gemm_w4a4(*a, *b)
        e = norm_err(y.float().cpu().numpy(), yref, oracle.dequantize(*a), oracle.dequantize(*b))
        assert e <= tol, ((M, N, K), e)
        if N % 256 != 0:                           # the single call runs the same kernel
            assert torch.equal(y.view(torch.int16) if out_dtype == torch.bfloat16 else y.view(torch.int32),
                               y1.view(torch.int16) if out_dtype == torch.bfloat16 else y1.view(torch.int32))


def test_grouped_pixart_block_projections(cuda_ok):
    """One PixArt-1024 block's independent projections in one launch: the
    image-token QKV (M 8192, K 1152, N 3456) and the text-token cross-attention
    K and V (M 600, K 4096, N 1152); sampled full rows vs the oracle."""
    names = ("qkv", "xattn_k", "xattn_v")
    data, pairs = [], []
    for name in names:
        x, w = synth.layer_tensors("pixart1024", name, device="cpu")
        ac, asf, ga = oracle.quantize(x)
        bc, bsf, gb = oracle.quantize(w)
        data.append(((ac, asf, ga), (bc, bsf, gb)))
        pairs.append((upload(ac, asf, ga, *x.shape), upload(bc, bsf, gb, *w.shape)))
    ys = nv.gemm_w4a4_grouped(pairs)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    for (a, b), y in zip(data, ys):
        M = a[0].shape[0]
        rows = np.array(sorted({0, 127, 128, M - 1} | set(int(r) for r in rng.integers(0, M, 12))))
        yref = np.concatenate([oracle.gemm_w4a4(*a, *b, rows=slice(int(r), int(r) + 1)) for r in rows])
        adeq = oracle.dequantize(*a)[rows]
        assert norm_err(y.float().cpu().numpy()[rows], yref, adeq, oracle.dequantize(*b)) <= TOL_BF16


def _exact_operands(rows, K, seed):
    """Codes with scale 1.0 everywhere: every partial sum is exact in FP32."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, (rows, K // 2)).astype(np.uint8)
    sf = np.zeros(oracle.sf_bytes(rows, K), np.uint8)
    for r in range(rows):
        for c in range(K // 16):
            sf[oracle.sf_offset(r, c, K // 16)] = 0x38
    return codes, sf


def test_grouped_nvfp4_epilogue_bit_exact_and_amax_per_problem(cuda_ok):
    shapes = [(256, 192, 1024), (300, 128, 256), (130, 320, 512)]
    probs, expect = [], []
    for i, (M, N, K) in enumerate(shapes):
        ac, asf = _exact_operands(M, K, 10 + i)
        bc, bsf = _exact_operands(N, K, 20 + i)
        ga, gb = 0.5, 0.25 * (i + 1)
        yref = oracle.gemm_w4a4(ac, asf, ga, bc, bsf, gb).astype(np.float32)
        gy = float(np.float32(np.abs(yref).max() / 2688.0 * 0.8))
        oc, osf, _ = oracle.quantize(yref, scale=gy)
        A, B = upload(ac, asf, ga, M, K), upload(bc, bsf, gb, N, K)
        q = nv.NVFP4Tensor.empty(M, N, "cuda")
        q.scale.fill_(gy)
        amax = torch.zeros(1, dtype=torch.float32, device="cuda")
        probs.append(dict(a_codes=A.codes, a_sf=A.sf, a_scale=A.scale, b_codes=B.codes, b_sf=B.sf,
                          b_scale=B.scale, M=M, N=N, K=K, y_codes=q.codes, y_sf=q.sf, y_scale=q.scale,
                          y_amax=amax))
        expect.append((oc, osf, np.abs(yref).max(), q, amax, (A, B)))
    nv.nvfp4_gemm_w4a4_grouped(probs)
    torch.cuda.synchronize()
    for oc, osf, am, q, amax, _ in expect:
        assert np.array_equal(q.codes.cpu().numpy(), oc)
        assert np.array_equal(q.sf.cpu().numpy()[: osf.size], osf)
        assert amax.item() == am


def test_grouped_skips_empty_problems_and_group_of_one(cuda_ok):
    (a, b) = _operands(200, 384, 512, 60)
    A, B = upload(*a, 200, 512), upload(*b, 384, 512)
    E = nv.NVFP4Tensor.empty(0, 512, "cuda")
    y = torch.empty(200, 384, dtype=torch.bfloat16, device="cuda")
    probs = [dict(a_codes=E.codes, a_sf=E.sf, a_scale=E.scale, b_codes=B.codes, b_sf=B.sf, b_scale=B.scale,
                  M=0, N=384, K=512, y=y),
             dict(a_codes=A.codes, a_sf=A.sf, a_scale=A.scale, b_codes=B.codes, b_sf=B.sf, b_scale=B.scale,
                  M=200, N=384, K=512, y=y)]
    n0 = nv.nvfp4_launch_count()
    nv.nvfp4_gemm_w4a4_grouped(probs)
    assert nv.nvfp4_launch_count() - n0 == 1
    y1 = nv.gemm_w4a4(A, B)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y1.view(torch.int16))
    n0 = nv.nvfp4_launch_count()
    nv.nvfp4_gemm_w4a4_grouped(probs[:1])           # only an empty problem: nothing launched
    assert nv.nvfp4_launch_count() == n0


PAIR_GROUPS = {256: [(300, 512, 1152), (128, 256, 256), (77, 768, 4096), (513, 256, 320)],
               192: [(300, 384, 1152), (128, 192, 256), (77, 1152, 4096), (513, 576, 320)]}


@pytest.mark.parametrize("bn", [256, 192])
@pytest.mark.parametrize("out_dtype,tol", [(torch.bfloat16, TOL_BF16), (torch.float32, TOL_F32)])
def test_grouped_on_the_pair_kernel(cuda_ok, monkeypatch, bn, out_dtype, tol):
    """A group whose every N allows one pair tile width runs on the CTA-pair
    kernel (forced here: the shapes are small); each output meets the oracle's
    tolerance and equals the single pair-kernel call bit for bit (same tiles,
    same accumulation order)."""
    monkeypatch.setenv("NVFP4_GEMM_KERNEL", "pair")
    monkeypatch.setenv("NVFP4_PAIR_TILE_N", str(bn))
    shapes = PAIR_GROUPS[bn]
    ops = [_operands(M, N, K, 140 + i) for i, (M, N, K) in enumerate(shapes)]
    pairs = [(upload(*a, M, K), upload(*b, N, K)) for (a, b), (M, N, K) in zip(ops, shapes)]
    ys = nv.gemm_w4a4_grouped(pairs, out_dtype=out_dtype)
    singles = [nv.gemm_w4a4(A, B, out_dtype=out_dtype) for A, B in pairs]
    torch.cuda.synchronize()
    view = torch.int16 if out_dtype == torch.bfloat16 else torch.int32
    for (a, b), (M, N, K), y, y1 in zip(ops, shapes, ys, singles):
        yref = oracle.gemm_w4a4(*a, *b)
        e = norm_err(y.float().cpu().numpy(), yref, oracle.dequantize(*a), oracle.dequantize(*b))
        assert e <= tol, ((M, N, K), e)
        assert torch.equal(y.view(view), y1.view(view))


def test_grouped_pair_kernel_nvfp4_epilogue_bit_exact_and_amax_per_problem(cuda_ok, monkeypatch):
    monkeypatch.setenv("NVFP4_GEMM_KERNEL", "pair")
    shapes = [(256, 384, 1024), (300, 192, 256), (130, 576, 512)]
    probs, expect = [], []
    for i, (M, N, K) in enumerate(shapes):
        ac, asf = _exact_operands(M, K, 30 + i)
        bc, bsf = _exact_operands(N, K, 40 + i)
        ga, gb = 0.5, 0.25 * (i + 1)
        yref = oracle.gemm_w4a4(ac, asf, ga, bc, bsf, gb).astype(np.float32)
        gy = float(np.float32(np.abs(yref).max() / 2688.0 * 0.8))
        oc, osf, _ = oracle.quantize(yref, scale=gy)
        A, B = upload(ac, asf, ga, M, K), upload(bc, bsf, gb, N, K)
        q = nv.NVFP4Tensor.empty(M, N, "cuda")
        q.scale.fill_(gy)
        amax = torch.zeros(1, dtype=torch.float32, device="cuda")
        probs.append(dict(a_codes=A.codes, a_sf=A.sf, a_scale=A.scale, b_codes=B.codes, b_sf=B.sf,
                          b_scale=B.scale, M=M, N=N, K=K, y_codes=q.codes, y_sf=q.sf, y_scale=q.scale,
                          y_amax=amax))
        expect.append((oc, osf, np.abs(yref).max(), q, amax))
    nv.nvfp4_gemm_w4a4_grouped(probs)
    torch.cuda.synchronize()
    for oc, osf, am, q, amax in expect:
        assert np.array_equal(q.codes.cpu().numpy(), oc)
        assert np.array_equal(q.sf.cpu().numpy()[: osf.size], osf)
        assert amax.item() == am
