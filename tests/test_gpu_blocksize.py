"""Block size per layer (Algorithm 1 / Eq. 9) on the GPU vs the CPU oracle:
quantization with 32 or 64 values per scale bit for bit, the product of
such operands within the GEMM tolerance, the per-candidate squared errors to
a relative 1e-6 (the kernel rounds each element difference once in FP32),
and the selected block size equal to the oracle's unless the two best
objectives are within that tolerance."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_gemm_quantize_b200 as nv
from nvfp4_w4a4_gemm_quantize_b200 import synth

pytestmark = pytest.mark.gpu


def _to_gpu(xb, ld=None):
    rows, k = xb.shape
    if ld is not None and ld != k:
        big = torch.zeros(rows, ld, dtype=torch.bfloat16)
        big[:, :k] = xb
        return big.cuda()[:, :k]
    return xb.cuda()


def _check_block(xb, block, scale=None, ld=None):
    rows, k = xb.shape
    q = nv.quantize_block(_to_gpu(xb, ld), block, scale=scale)
    torch.cuda.synchronize()
    oc, osf, og = oracle.quantize_block(xb, block, scale)
    assert np.float32(q.scale.item()) == og
    assert np.array_equal(q.codes.cpu().numpy(), oc)
    assert np.array_equal(q.sf.cpu().numpy()[: osf.size], osf)
    return q, (oc, osf, og)


@pytest.mark.parametrize("block", [32, 64])
def test_quantize_block_every_finite_pattern(cuda_ok, block):
    pats = np.arange(65536, dtype=np.uint32)
    pats = pats[((pats >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    np.random.default_rng(block).shuffle(pats)
    n = ((len(pats) + 255) // 256) * 256
    full = np.zeros(n, np.uint16)
    full[: len(pats)] = pats
    x = torch.from_numpy(full.view(np.int16).reshape(-1, 256)).view(torch.bfloat16)
    _check_block(x, block)
    _check_block(x, block, scale=1e-3)


@pytest.mark.parametrize("block", [32, 64])
@pytest.mark.parametrize("rows,k,ld,dist", [(1, 64, 64, "normal"), (129, 320, 328, "outlier"),
                                            (600, 4096, 4096, "student_t3"), (257, 1152, 1152, "token_scaled")])
def test_quantize_block_shapes(cuda_ok, block, rows, k, ld, dist):
    x = synth.random_bf16((rows, k), seed=rows + k + block, dist=dist)
    _check_block(x, block, ld=ld)
    _check_block(x, block, scale=float(oracle.tensor_scale(x)) * 0.5, ld=ld)


def test_gemm_of_block_64_operands(cuda_ok):
    x = synth.random_bf16((300, 1152), seed=7, dist="student_t3")
    w = synth.random_bf16((512, 1152), seed=8, dist="normal", scale=0.02)
    A, (ac, asf, ga) = _check_block(x, 64)
    W, (bc, bsf, gb) = _check_block(w, 64)
    y = nv.gemm_w4a4(A, W, out_dtype=torch.float32).cpu().numpy()
    ref = oracle.gemm_w4a4(ac, asf, ga, bc, bsf, gb)
    den = (np.linalg.norm(oracle.dequantize(ac, asf, ga), axis=1)[:, None]
           * np.linalg.norm(oracle.dequantize(bc, bsf, gb), axis=1)[None, :])
    assert np.max(np.abs(y - ref) / den) <= 1e-5


def _errors_match(xb, g):
    gpu = nv.block_size_errors(xb.cuda(), torch.tensor([g], device="cuda")).cpu().numpy()
    err, ss = oracle.block_size_errors(xb, g)
    assert gpu[7] == pytest.approx(ss, rel=1e-12)
    assert np.all(np.abs(gpu[:7] - err) <= 1e-6 * err + 1e-300)
    return gpu, err, ss


@pytest.mark.parametrize("dist", ["normal", "student_t3", "outlier", "token_scaled"])
def test_block_size_errors_and_selection(cuda_ok, dist):
    xb = synth.random_bf16((384, 1024), seed=11, dist=dist)
    g = float(oracle.tensor_scale(xb))
    gpu, err, ss = _errors_match(xb, g)
    for lam in (0.0, 1e-3, 1e-2, 3e-2, 0.1, 1.0):
        want = oracle.select_block_size(err, ss, lam)
        got = nv.nvfp4_select_block_size(gpu.tolist(), lam)
        obj = err / ss + lam * (4 + 8 / np.array(oracle.BLOCK_SIZES)) / 12
        best2 = np.sort(obj)[:2]
        assert got == want or best2[1] - best2[0] <= 1e-6 * best2[0]


def test_block_size_errors_zero_tensor_and_ragged_rows(cuda_ok):
    z = torch.zeros(130, 128, dtype=torch.bfloat16)
    gpu = nv.block_size_errors(z.cuda(), torch.zeros(1, device="cuda")).cpu().numpy()
    assert not gpu.any()
    _errors_match(synth.random_bf16((131, 192), seed=12, dist="outlier"), 0.01)


def test_block_size_errors_full_size_rows(cuda_ok):
    """The video fc2 input: errors over the full tensor on the GPU; parity on
    row slices (the errors are sums over rows; g from the whole tensor)."""
    x, = synth.layer_tensors("video_dit", "fc2", device="cuda", want=("x",))
    g = nv.quantize(x).scale
    full = nv.block_size_errors(x, g).cpu().numpy()
    assert np.all(full[:7] > 0) and np.all(np.diff(full[:7]) > 0)      # coarser blocks: larger error
    xc = x.cpu()
    for r0 in (0, 16000, 32768 - 96):
        _errors_match(xc[r0:r0 + 96], float(g.item()))


def test_one_workspace_across_output_kinds(cuda_ok):
    """Consecutive one-kernel calls of different kinds (codes, fake-quantized
    values, 64-value blocks) on the same workspace: each call's per-CTA slots
    carry a number no other call in the process used, so a large maximum left
    by one call is never taken for the next call's."""
    ws = torch.empty(nv.nvfp4_quantize_workspace_bytes(256, 512), dtype=torch.uint8, device="cuda")
    big = synth.random_bf16((256, 512), seed=50, dist="normal", scale=1000.0)
    small = synth.random_bf16((256, 512), seed=51, dist="normal")
    for _ in range(3):
        for xb in (big, small):
            q = nv.quantize(xb.cuda(), workspace=ws)
            y, m, g = nv.fake_quantize(xb.cuda(), workspace=ws)
            qb = nv.quantize_block(xb.cuda(), 64, workspace=ws)
            torch.cuda.synchronize()
            og = oracle.tensor_scale(xb)
            assert np.float32(q.scale.item()) == og and np.float32(g.item()) == og
            assert np.float32(qb.scale.item()) == og
            oc, osf, _ = oracle.quantize_block(xb, 64)
            assert np.array_equal(qb.codes.cpu().numpy(), oc)
            oy, om, _ = oracle.fake_quantize(xb)
            assert np.array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), oy)
