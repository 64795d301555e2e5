"""The MX variant (E2M1 in blocks of 32, E8M0 scales) on the GPU vs the CPU
oracle: quantization and dequantization bit for bit, the block32 MMA within
the GEMM tolerances (2e-3 normalised for bf16, 1e-5 for FP32), and one-hot
products that pin the scale layout and the byte id of the second K = 64 step
of each scale word."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_gemm_quantize_b200 as nv
from nvfp4_w4a4_gemm_quantize_b200 import synth
from gemm_kernels import KERNELS, select_kernel

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-3, torch.float32: 1e-5}


def _gpu_mx(xb, ld=None):
    rows, k = xb.shape
    if ld is not None and ld != k:
        big = torch.zeros(rows, ld, dtype=torch.bfloat16)
        big[:, :k] = xb
        xg = big.cuda()[:, :k]
    else:
        xg = xb.cuda()
    q = nv.mx_quantize(xg)
    torch.cuda.synchronize()
    return q, q.codes.cpu().numpy(), q.sf.cpu().numpy()[: oracle.mx_sf_bytes(rows, k)]


def _check(xb, ld=None):
    q, codes, sf = _gpu_mx(xb, ld)
    oc, osf = oracle.mx_quantize(xb)
    assert np.array_equal(codes, oc), np.argwhere(codes != oc)[:3]
    assert np.array_equal(sf, osf)
    return q, oc, osf


def test_mx_quantize_every_finite_bf16_pattern(cuda_ok):
    pats = np.arange(65536, dtype=np.uint32)
    pats = pats[((pats >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    rng = np.random.default_rng(0)
    for order in range(3):
        p = pats.copy()
        rng.shuffle(p) if order else None
        n = ((len(p) + 127) // 128) * 128
        full = np.zeros(n, np.uint16)
        full[: len(p)] = p
        _check(torch.from_numpy(full.view(np.int16).reshape(-1, 128)).view(torch.bfloat16))


@pytest.mark.parametrize("rows,k,ld,dist", [
    (1, 128, 128, "normal"), (127, 256, 264, "student_t3"), (130, 384, 384, "outlier"),
    (600, 4096, 4096, "token_scaled"), (257, 1152, 1160, "normal"),
])
def test_mx_quantize_shapes(cuda_ok, rows, k, ld, dist):
    _check(synth.random_bf16((rows, k), seed=rows + k, dist=dist), ld=ld)


def test_mx_quantize_wide_range_and_dequantize(cuda_ok):
    rng = np.random.default_rng(4)
    x = rng.standard_normal((300, 512)).astype(np.float32)
    x *= np.exp2(rng.uniform(-60, 60, (300, 16))).repeat(32, axis=1).astype(np.float32)
    x[0, :32] = 0.0
    x[1, 32:64] = (rng.standard_normal(32) * 2.0 ** -128).astype(np.float32)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    q, oc, osf = _check(xb)
    ref = oracle.mx_dequantize(oc, osf)
    d32 = nv.mx_dequantize(q, torch.float32).cpu().numpy()
    d16 = nv.mx_dequantize(q, torch.bfloat16).float().cpu().numpy()
    assert np.array_equal(d32.astype(np.float64), ref)
    assert np.array_equal(d16.astype(np.float64), ref)


def _upload(codes, sf, rows, k):
    q = nv.MXTensor.empty(rows, k, "cuda")
    q.codes.copy_(torch.from_numpy(np.ascontiguousarray(codes)))
    q.sf[: sf.size].copy_(torch.from_numpy(sf))
    return q


@pytest.mark.parametrize("m0,n0,k0", [(0, 0, 0), (5, 3, 17), (127, 130, 70), (64, 255, 100), (130, 7, 300),
                                       (1, 2, 255)])
def test_mx_gemm_one_hot(cuda_ok, m0, n0, k0):
    M, N, K = 256, 384, 384
    kb = K // 32
    ac = np.zeros((M, K // 2), np.uint8)
    bc = np.zeros((N, K // 2), np.uint8)
    ac[m0, k0 // 2] = 0x5 << (4 * (k0 & 1))             # 3.0
    bc[n0, k0 // 2] = 0xB << (4 * (k0 & 1))             # -1.5
    asf = np.full(oracle.mx_sf_bytes(M, K), 127, np.uint8)
    bsf = np.full(oracle.mx_sf_bytes(N, K), 127, np.uint8)
    asf[oracle.sf_offset(m0, k0 // 32, kb)] = 127 + 3
    bsf[oracle.sf_offset(n0, k0 // 32, kb)] = 127 - 2
    y = nv.mx_gemm(_upload(ac, asf, M, K), _upload(bc, bsf, N, K), out_dtype=torch.float32).cpu().numpy()
    expect = np.zeros((M, N))
    expect[m0, n0] = 3.0 * -1.5 * 2.0 ** 3 * 2.0 ** -2
    assert np.array_equal(y, expect)
    assert np.array_equal(oracle.mx_gemm(ac, asf, bc, bsf), expect)


@pytest.mark.parametrize("m0,n0,k0", [(0, 0, 0), (200, 300, 600), (383, 511, 639), (129, 129, 129),
                                       (255, 256, 383), (130, 7, 300), (10, 200, 64)])
@pytest.mark.parametrize("N,kernel", [(512, "pair256"), (576, "pair192")])
def test_mx_gemm_one_hot_pair_kernel(cuda_ok, monkeypatch, N, kernel, m0, n0, k0):
    """CTA-pair kernels (N = 512: 256-wide tiles; N = 576: 192-wide tiles,
    the second one starting half-way into a scale atom): one nonzero product
    lands in the right output, also in the second CTA's rows, the second B
    half and the last, half-filled K stage."""
    select_kernel(monkeypatch, kernel, N)
    M, K = 384, 640
    kb = K // 32
    ac = np.zeros((M, K // 2), np.uint8)
    bc = np.zeros((N, K // 2), np.uint8)
    ac[m0, k0 // 2] = 0x5 << (4 * (k0 & 1))             # 3.0
    bc[n0, k0 // 2] = 0xB << (4 * (k0 & 1))             # -1.5
    asf = np.full(oracle.mx_sf_bytes(M, K), 127, np.uint8)
    bsf = np.full(oracle.mx_sf_bytes(N, K), 127, np.uint8)
    asf[oracle.sf_offset(m0, k0 // 32, kb)] = 127 + 5
    bsf[oracle.sf_offset(n0, k0 // 32, kb)] = 127 - 7
    y = nv.mx_gemm(_upload(ac, asf, M, K), _upload(bc, bsf, N, K), out_dtype=torch.float32).cpu().numpy()
    expect = np.zeros((M, N))
    expect[m0, n0] = 3.0 * -1.5 * 2.0 ** 5 * 2.0 ** -7
    assert np.array_equal(y, expect)
    assert np.array_equal(oracle.mx_gemm(ac, asf, bc, bsf), expect)


# every kernel the shape allows (tests/gemm_kernels.py); K = 640 and 1152 end
# in a half stage (one MX scale atom)
@pytest.mark.parametrize("M,N,K", [(300, 384, 1152), (128, 256, 256), (77, 1152, 640), (513, 136, 384),
                                   (300, 512, 1152), (513, 768, 640), (64, 256, 384)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("kernel", KERNELS)
def test_mx_gemm_vs_oracle(cuda_ok, monkeypatch, kernel, M, N, K, out_dtype):
    select_kernel(monkeypatch, kernel, N)
    x = synth.random_bf16((M, K), seed=M + K, dist="student_t3")
    w = synth.random_bf16((N, K), seed=N + K, dist="normal", scale=0.02)
    ac, asf = oracle.mx_quantize(x)
    bc, bsf = oracle.mx_quantize(w)
    y = nv.mx_gemm(_upload(ac, asf, M, K), _upload(bc, bsf, N, K), out_dtype=out_dtype).float().cpu().numpy()
    ref = oracle.mx_gemm(ac, asf, bc, bsf)
    den = (np.linalg.norm(oracle.mx_dequantize(ac, asf), axis=1)[:, None]
           * np.linalg.norm(oracle.mx_dequantize(bc, bsf), axis=1)[None, :])
    err = np.abs(y.astype(np.float64) - ref)
    assert np.max(err / np.where(den > 0, den, 1.0)) <= TOL[out_dtype]


def test_mx_gemm_with_gpu_quantized_operands_and_gelu(cuda_ok):
    x = synth.random_bf16((256, 1024), seed=5, dist="outlier")
    w = synth.random_bf16((512, 1024), seed=6, dist="normal", scale=0.02)
    A, W = _check(x)[0], _check(w)[0]
    ac, asf = oracle.mx_quantize(x)
    bc, bsf = oracle.mx_quantize(w)
    v = oracle.mx_gemm(ac, asf, bc, bsf)
    y = nv.mx_gemm(A, W, out_dtype=torch.float32, act=nv.NVFP4_ACT_GELU_TANH).cpu().numpy()
    den = (np.linalg.norm(oracle.mx_dequantize(ac, asf), axis=1)[:, None]
           * np.linalg.norm(oracle.mx_dequantize(bc, bsf), axis=1)[None, :])
    bound = 1.13 * 1e-5 * den + 2.0 ** -10 * np.abs(v) + 1e-30
    assert np.all(np.abs(y - oracle.gelu_tanh(v)) <= bound)
