"""GPU W4A4 GEMM vs the CPU oracle.

The oracle's operands are its own quantization of the seeded bf16 tensors;
the GPU GEMM reads the same codes (uploaded, or produced by the GPU quantizer
whose bit-exactness is asserted on the same rows).  Tolerances:
  bf16 output   max |Y - Y_ref| / (|row_m(A^)| |row_n(B^)|) <= 2e-3
                (bf16 rounding alone contributes up to 2^-9 = 1.95e-3)
  FP32 output   the same ratio <= 1e-5 (FP32 accumulation order only)
  NVFP4 output  bit-exact where the FP32 accumulation is exact; otherwise every
                scale byte and code is the exact rounding of some FP32 value
                within the FP32 tolerance (tests/nvfp4_validity.py).
"""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_gemm_quantize_b200 as nv
from nvfp4_w4a4_gemm_quantize_b200 import synth
from nvfp4_validity import assert_valid_nvfp4_rounding
from gemm_kernels import KERNELS, select_kernel

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


def run_and_compare(x, w, out_dtype):
    M, K = x.shape
    N = w.shape[0]
    ac, asf, ga = oracle.quantize(x)
    bc, bsf, gb = oracle.quantize(w)
    A = upload(ac, asf, ga, M, K)
    B = upload(bc, bsf, gb, N, K)
    y = nv.gemm_w4a4(A, B, out_dtype=out_dtype)
    torch.cuda.synchronize()
    yref = oracle.gemm_w4a4(ac, asf, ga, bc, bsf, gb)
    e = norm_err(y.float().cpu().numpy(), yref, oracle.dequantize(ac, asf, ga), oracle.dequantize(bc, bsf, gb))
    return e


def _one_hot_operands(rows, K, positions, code, sfbyte):
    c = np.zeros((rows, K // 2), np.uint8)
    sf = np.zeros(oracle.sf_bytes(rows, K), np.uint8)
    for r, k in positions:
        c[r, k // 2] |= code << (4 * (k & 1))
        sf[oracle.sf_offset(r, k // 16, K // 16)] = sfbyte
    return c, sf


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (300, 384, 1152), (256, 512, 320), (300, 576, 256),
                                   (520, 768, 512)])
def test_one_hot_pins_nibble_order_and_scale_layout(cuda_ok, monkeypatch, kernel, M, N, K):
    """Row m of A has one non-zero at k_a(m), row n of B one at k_b(n); Y[m,n]
    is the single product when k_a(m) == k_b(n) and exactly 0 otherwise.
    N = 576 and 768 give 192-wide tiles that start half-way into a 128-row
    scale atom (odd tiles)."""
    select_kernel(monkeypatch, kernel, N)
    rng = np.random.default_rng(M + N + K)
    ka = rng.integers(0, K, M)
    kb = rng.integers(0, K, N)
    kb[: min(N, M)] = ka[: min(N, M)]          # guarantee matches on the diagonal
    ac, asf = _one_hot_operands(M, K, list(enumerate(ka)), 0x5, 0x40)    # 3.0 * 2.0
    bc, bsf = _one_hot_operands(N, K, list(enumerate(kb)), 0xB, 0x30)    # -1.5 * 0.5
    A = upload(ac, asf, 0.25, M, K)
    B = upload(bc, bsf, 4.0, N, K)
    y = nv.gemm_w4a4(A, B, out_dtype=torch.float32).cpu().numpy()
    ref = oracle.gemm_w4a4(ac, asf, 0.25, bc, bsf, 4.0)
    assert np.array_equal(y.astype(np.float64), ref)
    assert (ref != 0).sum() >= min(M, N)


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (1, 256, 64), (200, 384, 320), (300, 1152, 1152),
                                   (257, 512, 4608), (600, 1152, 4096), (129, 128, 192), (64, 640, 1024),
                                   (700, 960, 704)])
@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("kernel", KERNELS)
def test_random_shapes_vs_oracle(cuda_ok, monkeypatch, kernel, M, N, K, out):
    select_kernel(monkeypatch, kernel, N)
    x = synth.random_bf16((M, K), seed=M * 7 + K, dist="outlier")
    w = synth.random_bf16((N, K), seed=N * 13 + K, scale=0.02)
    e = run_and_compare(x, w, out)
    assert e <= (TOL_BF16 if out == torch.bfloat16 else TOL_F32), e


def test_pr1_full(cuda_ok):
    x, w = synth.layer_tensors("pr1", "linear")
    assert run_and_compare(x, w, torch.bfloat16) <= TOL_BF16
    assert run_and_compare(x, w, torch.float32) <= TOL_F32


def _sample(n, rng, k=56):
    s = {0, 1, 126, 127, 128, 129, 255, 256, n // 2, n - 2, n - 1}
    s |= set(int(v) for v in rng.integers(0, n, k))
    return np.array(sorted(r for r in s if 0 <= r < n))


WORKLOAD_LAYERS = [(w, l.name) for w in ("dit_xl2", "pixart1024", "video_dit") for l in synth.WORKLOADS[w].layers]


@pytest.mark.parametrize("workload,layer", WORKLOAD_LAYERS)
def test_workload_layer_full_size_sampled(cuda_ok, workload, layer):
    """The launch configuration the benchmark times, on the full layer: GPU
    quantize + GEMM; the oracle quantizes sampled rows of X and W with the
    tensor scales it computes over the whole tensors and forms those entries."""
    x, w = synth.layer_tensors(workload, layer, device="cuda")
    M, K = x.shape
    N = w.shape[0]
    A = nv.quantize(x)
    B = nv.quantize(w)
    y = nv.gemm_w4a4(A, B)
    torch.cuda.synchronize()
    rng = np.random.default_rng(11)
    ms, ns = _sample(M, rng), _sample(N, rng)
    xc, wc = x.cpu(), w.cpu()
    ga, gb = oracle.tensor_scale(xc), oracle.tensor_scale(wc)
    assert np.float32(A.scale.item()) == ga and np.float32(B.scale.item()) == gb
    ac, asf, _ = oracle.quantize(xc[torch.from_numpy(ms)], scale=float(ga))
    bc, bsf, _ = oracle.quantize(wc[torch.from_numpy(ns)], scale=float(gb))
    # the GPU operands on those rows are the oracle's, bit for bit
    assert np.array_equal(A.codes.cpu().numpy()[ms], ac)
    assert np.array_equal(B.codes.cpu().numpy()[ns], bc)
    assert np.array_equal(oracle.sf_matrix(A.sf.cpu().numpy(), M, K)[ms], oracle.sf_matrix(asf, len(ms), K))
    assert np.array_equal(oracle.sf_matrix(B.sf.cpu().numpy(), N, K)[ns], oracle.sf_matrix(bsf, len(ns), K))
    yref = oracle.gemm_w4a4(ac, asf, ga, bc, bsf, gb)
    yg = y.float().cpu().numpy()[np.ix_(ms, ns)]
    e = norm_err(yg, yref, oracle.dequantize(ac, asf, ga), oracle.dequantize(bc, bsf, gb))
    assert e <= TOL_BF16, e
    assert torch.isfinite(y).all()


def _exact_operands(rows, K, seed):
    """Codes with scale byte 1.0 everywhere: every product is a multiple of
    1/4 and every partial sum stays exactly representable in FP32 for
    K <= 4096, so any accumulation order gives the exact value."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, (rows, K // 2)).astype(np.uint8)
    sf = np.zeros(oracle.sf_bytes(rows, K), np.uint8)
    for r in range(rows):
        for c in range(K // 16):
            sf[oracle.sf_offset(r, c, K // 16)] = 0x38
    return codes, sf


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("M,N,K", [(256, 256, 1024), (300, 384, 4096), (128, 1152, 256), (260, 768, 512)])
def test_nvfp4_epilogue_bit_exact(cuda_ok, monkeypatch, kernel, M, N, K):
    select_kernel(monkeypatch, kernel, N)
    ac, asf = _exact_operands(M, K, 1)
    bc, bsf = _exact_operands(N, K, 2)
    ga, gb = 0.5, 0.25
    A, B = upload(ac, asf, ga, M, K), upload(bc, bsf, gb, N, K)
    yref = oracle.gemm_w4a4(ac, asf, ga, bc, bsf, gb)
    y32 = nv.gemm_w4a4(A, B, out_dtype=torch.float32).cpu().numpy()
    assert np.array_equal(y32.astype(np.float64), yref)           # accumulation is exact here
    yref32 = yref.astype(np.float32)
    gy = float(np.float32(np.abs(yref32).max() / 2688.0 * 0.8))    # a scale that also clips
    oc, osf, _ = oracle.quantize(yref32, scale=gy)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    q = nv.gemm_w4a4_nvfp4_out(A, B, torch.tensor([gy], device="cuda"), y_amax=amax)
    torch.cuda.synchronize()
    assert np.array_equal(q.codes.cpu().numpy(), oc)
    assert np.array_equal(q.sf.cpu().numpy()[: osf.size], osf)
    assert amax.item() == np.abs(yref32).max()


@pytest.mark.parametrize("kernel", KERNELS)
def test_nvfp4_epilogue_random_data_is_a_valid_rounding(cuda_ok, monkeypatch, kernel):
    """Random operands: the accumulation order is not fixed, so the codes are
    not unique; every scale byte and code must be the exact rounding of SOME
    FP32 value within the FP32 tolerance of the oracle's FP64 product
    (tests/nvfp4_validity.py: a code one grid step or a scale byte one E4M3
    step off fails)."""
    x, w = synth.layer_tensors("dit_xl2", "fc1", device="cpu")
    M, K = x.shape
    N = w.shape[0]
    select_kernel(monkeypatch, kernel, N)
    ac, asf, ga = oracle.quantize(x)
    bc, bsf, gb = oracle.quantize(w)
    rows = np.array([0, 1, 127, 128, 1000, 2047])
    yref = np.concatenate([oracle.gemm_w4a4(ac, asf, ga, bc, bsf, gb, rows=slice(int(r), int(r) + 1))
                           for r in rows])
    gy = float(np.float32(np.abs(yref).max() / 2688.0))
    A, B = upload(ac, asf, ga, M, K), upload(bc, bsf, gb, N, K)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    q = nv.gemm_w4a4_nvfp4_out(A, B, torch.tensor([gy], device="cuda"), y_amax=amax)
    torch.cuda.synchronize()
    ar, asr, _ = oracle.quantize(x[torch.from_numpy(rows)], scale=float(ga))
    na = np.linalg.norm(oracle.dequantize(ar, asr, ga), axis=1)
    nb = np.linalg.norm(oracle.dequantize(bc, bsf, gb), axis=1)
    tol = TOL_F32 * na[:, None] * nb[None, :]
    codes = q.codes.cpu().numpy()[rows]
    sfm = oracle.sf_matrix(q.sf.cpu().numpy(), M, N)[rows]
    assert_valid_nvfp4_rounding(codes, sfm, gy, yref, tol)
    # the observed amax is the largest FP32 value: within the tolerance of the oracle's
    full = oracle.gemm_w4a4(ac, asf, ga, bc, bsf, gb, rows=slice(0, 256))
    assert amax.item() >= np.abs(full).max() - TOL_F32 * na.max() * nb.max()


def test_dev_status_stays_zero_and_m_zero_noop(cuda_ok):
    x = synth.random_bf16((256, 512), seed=3).cuda()
    w = synth.random_bf16((256, 512), seed=4).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    A, B = nv.quantize(x), nv.quantize(w)
    nv.gemm_w4a4(A, B, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    e = nv.NVFP4Tensor.empty(0, 512, "cuda")
    y = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    nv.gemm_w4a4(e, B, out=y)
