"""W4A4 GEMM with the GELU epilogue (act = NVFP4_ACT_GELU_TANH) vs the CPU
oracle: y = GELU(alpha * acc), in bf16, FP32 or as the next layer's NVFP4
codes.

The kernel's GELU uses the hardware tanh approximation (relative error about
2^-11 in tanh), so values are compared against the oracle's double-precision
GELU of its FP64 product within a bound built from three parts:
  * the GEMM's own tolerance (1e-5 of |row(A^)| |row(B^)| for FP32
    accumulation), times 1.13, the largest slope of GELU;
  * the activation: |0.5 v| * 2^-11 * |tanh|, bounded here by 2^-10 |v|;
  * the output rounding (bf16: 2^-9 relative).  The NVFP4 output must be the
    exact rounding of some value within that bound of the oracle's GELU
    (tests/nvfp4_validity.py: per block scale byte and per element code).
With exactly representable products the accumulation term vanishes and the
comparison isolates the activation."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_gemm_quantize_b200 as nv
from nvfp4_w4a4_gemm_quantize_b200 import synth
from nvfp4_validity import assert_valid_nvfp4_rounding
from gemm_kernels import KERNELS, select_kernel

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
GELU_SLOPE = 1.13
ACT_ERR = 2.0 ** -10


def upload(codes, sf, g, rows, k) -> nv.NVFP4Tensor:
    q = nv.NVFP4Tensor.empty(rows, k, "cuda")
    q.codes.copy_(torch.from_numpy(np.ascontiguousarray(codes)))
    q.sf[: sf.size].copy_(torch.from_numpy(sf))
    q.scale.fill_(float(g))
    return q


def _operands(M, N, K, seed):
    x = synth.random_bf16((M, K), seed=seed, dist="student_t3")
    w = synth.random_bf16((N, K), seed=seed + 1, dist="normal", scale=0.02)
    return oracle.quantize(x), oracle.quantize(w)


def _den(a, b):
    na = np.linalg.norm(oracle.dequantize(*a), axis=1)[:, None]
    nb = np.linalg.norm(oracle.dequantize(*b), axis=1)[None, :]
    return na * nb


SHAPES = [(300, 512, 1152), (256, 256, 256), (300, 384, 512), (130, 1152, 4096), (300, 576, 512)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("kernel", KERNELS)
def test_gelu_epilogue_values(cuda_ok, monkeypatch, kernel, M, N, K, out_dtype):
    select_kernel(monkeypatch, kernel, N)
    a, b = _operands(M, N, K, 70 + M + N)
    A, B = upload(*a, M, K), upload(*b, N, K)
    y = nv.gemm_w4a4(A, B, out_dtype=out_dtype, act=nv.NVFP4_ACT_GELU_TANH)
    torch.cuda.synchronize()
    v = oracle.gemm_w4a4(*a, *b)
    g = oracle.gelu_tanh(v)
    bound = GELU_SLOPE * TOL_F32 * _den(a, b) + ACT_ERR * np.abs(v) + 1e-30
    if out_dtype == torch.bfloat16:
        bound = bound + 2.0 ** -8 * np.abs(g)
    err = np.abs(y.float().cpu().numpy().astype(np.float64) - g)
    assert np.all(err <= bound), float(np.max(err / bound))
    # the activation really ran: negative inputs are squashed (GELU >= -0.17)
    neg = v < -0.5
    assert neg.any() and np.all(np.abs(y.float().cpu().numpy()[neg]) < 0.2)


def _exact_operands(rows, K, seed):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, (rows, K // 2)).astype(np.uint8)
    sf = np.zeros(oracle.sf_bytes(rows, K), np.uint8)
    for r in range(rows):
        for c in range(K // 16):
            sf[oracle.sf_offset(r, c, K // 16)] = 0x38
    return codes, sf


@pytest.mark.parametrize("M,N,K", [(256, 512, 256), (200, 320, 512)])
def test_gelu_epilogue_exact_products_isolate_the_activation(cuda_ok, M, N, K):
    ac, asf = _exact_operands(M, K, 3)
    bc, bsf = _exact_operands(N, K, 4)
    ga, gb = 2.0 ** -4, 2.0 ** -3                       # v = acc / 128: spans GELU's curved part
    A, B = upload(ac, asf, ga, M, K), upload(bc, bsf, gb, N, K)
    y = nv.gemm_w4a4(A, B, out_dtype=torch.float32, act=nv.NVFP4_ACT_GELU_TANH).cpu().numpy()
    v = oracle.gemm_w4a4(ac, asf, ga, bc, bsf, gb)
    g = oracle.gelu_tanh(v)
    assert np.all(np.abs(y - g) <= ACT_ERR * np.abs(v) + 1e-30)
    assert np.abs(v).max() > 4 and (np.abs(v) < 1).mean() > 0.1


@pytest.mark.parametrize("M,N,K", [(300, 512, 1152), (300, 384, 512), (300, 576, 512)])
@pytest.mark.parametrize("kernel", KERNELS)
def test_gelu_nvfp4_epilogue_is_a_valid_rounding(cuda_ok, monkeypatch, kernel, M, N, K):
    select_kernel(monkeypatch, kernel, N)
    """MLP fc1 with the next layer's input emitted directly: decoded codes are a
    valid NVFP4 rounding of GELU(y), and y_amax is the largest |GELU(y)|."""
    a, b = _operands(M, N, K, 90 + N)
    A, B = upload(*a, M, K), upload(*b, N, K)
    v = oracle.gemm_w4a4(*a, *b)
    g = oracle.gelu_tanh(v)
    gy = float(np.float32(np.abs(g).max() / 2688.0))
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    q = nv.gemm_w4a4_nvfp4_out(A, B, torch.tensor([gy], device="cuda"), y_amax=amax, act=nv.NVFP4_ACT_GELU_TANH)
    deq = nv.dequantize(q, torch.float32).cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    val = GELU_SLOPE * TOL_F32 * _den(a, b) + ACT_ERR * np.abs(v)
    assert_valid_nvfp4_rounding(q.codes.cpu().numpy(), oracle.sf_matrix(q.sf.cpu().numpy(), M, N), gy, g, val)
    assert np.all(np.abs(deq - g) <= np.repeat((np.abs(g) + val).reshape(M, N // 16, 16).max(axis=2)
                                               * (1 + 2.0 ** -4) / 6.0, 16, axis=1) + val)
    assert abs(amax.item() - np.abs(g).max()) <= val.max() + 1e-6 * np.abs(g).max()


def test_gelu_in_a_grouped_launch(cuda_ok):
    shapes = [(300, 384, 512), (77, 1152, 1152)]
    ops = [_operands(M, N, K, 110 + i) for i, (M, N, K) in enumerate(shapes)]
    pairs = [(upload(*a, M, K), upload(*b, N, K)) for (a, b), (M, N, K) in zip(ops, shapes)]
    ys = nv.gemm_w4a4_grouped(pairs, out_dtype=torch.float32, act=nv.NVFP4_ACT_GELU_TANH)
    torch.cuda.synchronize()
    for (a, b), y in zip(ops, ys):
        v = oracle.gemm_w4a4(*a, *b)
        bound = GELU_SLOPE * TOL_F32 * _den(a, b) + ACT_ERR * np.abs(v) + 1e-30
        assert np.all(np.abs(y.cpu().numpy() - oracle.gelu_tanh(v)) <= bound)
