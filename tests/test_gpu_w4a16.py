"""GPU W4A16 GEMM (bf16 activations x NVFP4 weights, dequantization fused in
the mainloop) vs the CPU oracle.

The oracle's weight operand is its own quantization of the seeded bf16
weights; activations are the seeded bf16 tensors.  Bound: the FP32
accumulation within 1e-5 of |row(x)| |row(w^)|; a bf16 output may add its own
rounding, at most 2^-8 of the exact |y| (round to nearest with an 8-bit
significand) -- which a heavy-tailed row can bring close to |x| |w^| itself."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_gemm_quantize_b200 as nv
from nvfp4_w4a4_gemm_quantize_b200 import synth

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
BF16_ROUND = 2.0 ** -8


def upload(codes, sf, g, rows, k) -> nv.NVFP4Tensor:
    q = nv.NVFP4Tensor.empty(rows, k, "cuda")
    q.codes.copy_(torch.from_numpy(np.ascontiguousarray(codes)))
    q.sf[: sf.size].copy_(torch.from_numpy(sf))
    q.scale.fill_(float(g))
    return q


def norm_err(y, yref, xd, wd, rounding=0.0):
    """Largest |y - yref| beyond `rounding` |yref|, over |row(x)| |row(w)|."""
    den = np.linalg.norm(xd, axis=1)[:, None] * np.linalg.norm(wd, axis=1)[None, :]
    err = np.maximum(np.abs(y.astype(np.float64) - yref) - rounding * np.abs(yref), 0.0)
    return float(np.max(np.where(den > 0, err / np.where(den > 0, den, 1.0), err)))


# "single": one CTA per 256 x 256 tile; "pair": CTA pairs on 512 x 256 tiles;
# "auto": the library's choice (pairs once their tiles fill half the SMs).
KERNELS = ["auto", "single", "pair"]


@pytest.fixture
def kernel(request, monkeypatch):
    if request.param != "auto":
        monkeypatch.setenv("NVFP4_W4A16_KERNEL", request.param)
    return request.param


@pytest.mark.parametrize("kernel", ["single", "pair"], indirect=True)
def test_one_hot_pins_dequant_layout(cuda_ok, kernel):
    M, N, K = 128, 256, 128
    rng = np.random.default_rng(5)
    wc = np.zeros((N, K // 2), np.uint8)
    wsf = np.zeros(oracle.sf_bytes(N, K), np.uint8)
    kk = rng.integers(0, K, N)
    for n in range(N):
        k = int(kk[n])
        wc[n, k // 2] |= (0x5 if n % 2 else 0xB) << (4 * (k & 1))    # 3.0 or -1.5
        wsf[oracle.sf_offset(n, k // 16, K // 16)] = 0x40 if n % 3 else 0x30
    x = torch.zeros(M, K, dtype=torch.bfloat16)
    for m in range(M):
        x[m, (m * 7) % K] = 1.0 + (m % 5)
    W = upload(wc, wsf, 0.25, N, K)
    y = nv.gemm_w4a16(x.cuda(), W, out_dtype=torch.float32).cpu().numpy()
    ref = oracle.gemm_w4a16(x, wc, wsf, 0.25)
    assert np.array_equal(y.astype(np.float64), ref)
    assert (ref != 0).sum() > 0


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (1, 256, 128), (200, 384, 320), (300, 512, 1152), (257, 256, 4608),
                                   (1100, 776, 640), (1536, 1024, 256)])
@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("kernel", KERNELS, indirect=True)
def test_random_shapes_vs_oracle(cuda_ok, M, N, K, out, kernel):
    x = synth.random_bf16((M, K), seed=M + 3 * K, dist="student_t3")
    w = synth.random_bf16((N, K), seed=N + 5 * K, scale=0.015)
    wc, wsf, gw = oracle.quantize(w)
    W = upload(wc, wsf, gw, N, K)
    y = nv.gemm_w4a16(x.cuda(), W, out_dtype=out)
    torch.cuda.synchronize()
    yref = oracle.gemm_w4a16(x, wc, wsf, gw)
    e = norm_err(y.float().cpu().numpy(), yref, x.float().numpy(), oracle.dequantize(wc, wsf, gw),
                 BF16_ROUND if out == torch.bfloat16 else 0.0)
    assert e <= TOL_F32, e


@pytest.mark.parametrize("layer", ["fc1", "fc2"])
@pytest.mark.parametrize("kernel", ["auto", "single"], indirect=True)
def test_w4a16_workload_full_size_sampled(cuda_ok, layer, kernel):
    """The weights-only workload at full size (M=16384): GPU quantize of the
    weights + fused-dequant GEMM; the oracle quantizes sampled weight rows with
    the tensor scale it computes over the whole weight and forms those entries."""
    x, w = synth.layer_tensors("w4a16", layer, device="cuda")
    M, K = x.shape
    N = w.shape[0]
    W = nv.quantize(w)
    y = nv.gemm_w4a16(x, W)
    torch.cuda.synchronize()
    rng = np.random.default_rng(13)
    ms = np.array(sorted({0, 1, 127, 128, M - 1, M // 2} | set(int(v) for v in rng.integers(0, M, 50))))
    ns = np.array(sorted({0, 1, 255, 256, N - 1} | set(int(v) for v in rng.integers(0, N, 50))))
    wcpu = w.cpu()
    gw = oracle.tensor_scale(wcpu)
    assert np.float32(W.scale.item()) == gw
    wc, wsf, _ = oracle.quantize(wcpu[torch.from_numpy(ns)], scale=float(gw))
    assert np.array_equal(W.codes.cpu().numpy()[ns], wc)
    xs = x.cpu()[torch.from_numpy(ms)]
    yref = oracle.gemm_w4a16(xs, wc, wsf, gw)
    yg = y.float().cpu().numpy()[np.ix_(ms, ns)]
    e = norm_err(yg, yref, xs.float().numpy(), oracle.dequantize(wc, wsf, gw), BF16_ROUND)
    assert e <= TOL_F32, e
