"""GPU fake quantization and straight-through-estimator backward vs the CPU
oracle, bit for bit.

Inputs (tensors, scales, gradients and clip masks given to the backward) are
seeded; the oracle sees only those inputs, never a value produced on the GPU.
Values (bf16 and f32), clip masks and the tensor scale must be identical."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_gemm_quantize_b200 as nv
from nvfp4_w4a4_gemm_quantize_b200 import synth

pytestmark = pytest.mark.gpu


def _to_gpu(xb_cpu: torch.Tensor, ld=None) -> torch.Tensor:
    rows, k = xb_cpu.shape
    if ld is not None and ld != k:
        big = torch.zeros(rows, ld, dtype=torch.bfloat16)
        big[:, :k] = xb_cpu
        return big.cuda()[:, :k]
    return xb_cpu.cuda()


def _bits(t: torch.Tensor) -> np.ndarray:
    t = t.cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy().view(np.uint32)


def _first_diff(a, b):
    bad = np.argwhere(a != b)[:3]
    return [(tuple(i), hex(int(a[tuple(i)])), hex(int(b[tuple(i)]))) for i in bad]


def _check(xb_cpu, scale=None, ld=None, out_dtype=torch.bfloat16):
    xg = _to_gpu(xb_cpu, ld)
    y, m, g = nv.fake_quantize(xg, scale, out_dtype=out_dtype)
    torch.cuda.synchronize()
    oy, om, og = oracle.fake_quantize(xb_cpu, scale, out="f32" if out_dtype == torch.float32 else "bf16")
    assert np.float32(g.item()) == og
    gy = _bits(y)
    oyb = oy.view(np.uint32) if out_dtype == torch.float32 else oy
    assert np.array_equal(gy, oyb), _first_diff(gy, oyb)
    gm = m.cpu().numpy()
    assert np.array_equal(gm, om), _first_diff(gm, om)
    return gm


def _all_finite_bf16(seed=0):
    pats = np.arange(65536, dtype=np.uint32)
    exp = (pats >> 7) & 0xFF
    pats = pats[exp != 0xFF].astype(np.uint16)
    rng = np.random.default_rng(seed)
    rng.shuffle(pats)
    n = ((len(pats) + 255) // 256) * 256
    full = np.zeros(n, np.uint16)
    full[: len(pats)] = pats
    return torch.from_numpy(full.view(np.int16).reshape(-1, 256)).view(torch.bfloat16)


def test_fake_quantize_every_finite_bf16_pattern(cuda_ok):
    """Every finite bf16 value, with the data's own scale and with given
    scales from 2^-140 (block scales so small that the products fall below
    FP32's normal range) to 1e30 (every element clipped to 6 * 448 g)."""
    x = _all_finite_bf16()
    _check(x)
    _check(x, out_dtype=torch.float32)
    for g in (2.0 ** -140, 1e-30, 2.0 ** -20, 1e-3, 0.37, 1.0, 3.0e3, 2.0 ** 60, 1e30):
        _check(x, scale=g)
        _check(x, scale=g, out_dtype=torch.float32)


def test_fake_quantize_grid_range_and_tiny_tensors(cuda_ok):
    """Every bf16 mantissa at exponents that span the E2M1 range, and the
    same blocks scaled down to 2^-120 (block scales below 2^-118: the
    exactly-rounded slow path)."""
    rng = np.random.default_rng(2)
    mant = np.arange(128, dtype=np.uint16)
    for e in list(range(120, 136)) + [8, 12, 20]:
        pats = (np.uint16(e) << 7 | mant)
        sign = rng.integers(0, 2, pats.size).astype(np.uint16) << 15
        vals = np.tile(pats | sign, 32)
        rng.shuffle(vals)
        x = torch.from_numpy(vals.view(np.int16).reshape(-1, 256)).view(torch.bfloat16)
        _check(x)
        _check(x, scale=float(np.float32(2.0 ** (e - 127) / 2688.0 * rng.uniform(0.5, 2.0))))


@pytest.mark.parametrize("rows,k,ld,dist", [
    (1, 64, 64, "normal"), (127, 64, 64, "student_t3"), (129, 192, 200, "outlier"),
    (600, 4096, 4096, "student_t3"), (300, 320, 328, "token_scaled"), (257, 1152, 1152, "outlier"),
    (64, 4608, 4616, "normal"),
])
def test_fake_quantize_shapes(cuda_ok, rows, k, ld, dist):
    x = synth.random_bf16((rows, k), seed=rows * 17 + k, dist=dist)
    _check(x, ld=ld)
    _check(x, ld=ld, out_dtype=torch.float32)
    # a static scale 8x too small: the large elements clip and are marked
    m = _check(x, scale=float(oracle.tensor_scale(x)) / 8, ld=ld)
    assert m.any()


def test_fake_quantize_wide_dynamic_range(cuda_ok):
    """Rows spread over 2^-20 .. 2^20: small blocks get subnormal E4M3 scales,
    whose coarse rounding clips elements even with the data's own scale."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((512, 256)).astype(np.float32)
    x *= np.exp2(rng.uniform(-20, 20, (512, 1))).astype(np.float32)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    m = _check(xb)
    assert m.any()


def test_fake_quantize_zero_single_and_empty(cuda_ok):
    z = torch.zeros(130, 128, dtype=torch.bfloat16)
    _check(z)
    one = z.clone()
    one[129, 77] = -3.0
    _check(one)
    _check(synth.random_bf16((64, 128), seed=4, dist="normal"), scale=0.0)     # zero scale: all +0, no clip
    x = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    g = torch.full((1,), 5.0, device="cuda")
    ws = torch.empty(nv.nvfp4_quantize_workspace_bytes(0, 64), dtype=torch.uint8, device="cuda")
    nv.nvfp4_fake_quantize(x, 0, 64, 64, y, nv.NVFP4_DTYPE_BF16, None, g, 0, ws, ws.numel())
    torch.cuda.synchronize()
    assert g.item() == 0.0


def test_fake_quantize_without_mask_and_agrees_with_quantize_dequantize(cuda_ok):
    x = synth.random_bf16((384, 1024), seed=5, dist="student_t3").cuda()
    y1, m, g = nv.fake_quantize(x)
    y2, none, g2 = nv.fake_quantize(x, clip_mask=False)
    q = nv.quantize(x)
    d = nv.dequantize(q)
    torch.cuda.synchronize()
    assert none is None and torch.equal(g, g2) and torch.equal(g, q.scale)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(y1.view(torch.int16), d.view(torch.int16))


@pytest.mark.parametrize("workload,layer", [("video_dit", "fc1"), ("video_dit", "fc2")])
def test_fake_quantize_full_size_sampled_rows(cuda_ok, workload, layer):
    """Full-size activations and weights fake-quantized on the GPU; the
    oracle computes g over the whole tensor and fake-quantizes sampled rows
    with it."""
    x, w = synth.layer_tensors(workload, layer, device="cuda")
    for t in (x, w):
        rows, k = t.shape
        y, m, g = nv.fake_quantize(t)
        torch.cuda.synchronize()
        tc = t.cpu()
        og = oracle.tensor_scale(tc)
        assert np.float32(g.item()) == og
        rng = np.random.default_rng(8)
        sel = np.array(sorted({0, 1, 127, 128, rows - 1, rows // 2} | set(int(v) for v in rng.integers(0, rows, 40))))
        oy, om, _ = oracle.fake_quantize(tc[torch.from_numpy(sel)], scale=float(og))
        assert np.array_equal(_bits(y)[sel], oy)
        assert np.array_equal(m.cpu().numpy()[sel], om)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,k", [(1, 16), (3, 48), (129, 320), (1000, 4096)])
def test_ste_backward_matches_oracle(cuda_ok, dtype, rows, k):
    rng = np.random.default_rng(rows + k)
    mask = rng.integers(0, 256, (rows, k // 8)).astype(np.uint8)
    mask[0, 0] = 0xFF
    g = rng.standard_normal((rows, k)).astype(np.float32)
    gt = torch.from_numpy(g).to(dtype)
    og = _bits(gt) if dtype == torch.bfloat16 else gt.numpy().copy()
    expect = oracle.ste_backward(og, mask)
    gx = nv.ste_backward(gt.cuda(), torch.from_numpy(mask).cuda())
    torch.cuda.synchronize()
    exp_bits = expect if dtype == torch.bfloat16 else expect.view(np.uint32)
    assert np.array_equal(_bits(gx), exp_bits)
    # in place
    gi = gt.cuda()
    nv.ste_backward(gi, torch.from_numpy(mask).cuda(), out=gi)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(gi), exp_bits)


def test_autograd_forward_backward(cuda_ok):
    """FakeQuantizeSTE: forward values and clip mask from the kernels, the
    backward masks the incoming gradient with the forward's mask; the plain
    estimator passes it through untouched."""
    xb = synth.random_bf16((256, 512), seed=11, dist="outlier")
    g = float(oracle.tensor_scale(xb)) / 4                 # some elements clip
    oy, om, _ = oracle.fake_quantize(xb, g)
    rng = np.random.default_rng(12)
    gy = torch.from_numpy(rng.standard_normal((256, 512)).astype(np.float32)).bfloat16()
    expect = oracle.ste_backward(_bits(gy), om)
    x = xb.cuda().requires_grad_(True)
    y = nv.FakeQuantizeSTE.apply(x, g, True)
    y.backward(gy.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(_bits(y.detach()), oy)
    assert np.array_equal(_bits(x.grad), expect)
    assert om.any()
    x2 = xb.cuda().requires_grad_(True)
    nv.FakeQuantizeSTE.apply(x2, g, False).backward(gy.cuda())
    torch.cuda.synchronize()
    assert torch.equal(x2.grad.cpu().view(torch.int16), gy.view(torch.int16))
