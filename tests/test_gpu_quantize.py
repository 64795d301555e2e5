"""GPU quantize / dequantize vs the CPU oracle, bit for bit.

Inputs are seeded bf16 tensors; the oracle sees only those inputs (never a
value produced on the GPU).  Codes, scale bytes and the tensor scale must be
identical."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_gemm_quantize_b200 as nv
from nvfp4_w4a4_gemm_quantize_b200 import synth

pytestmark = pytest.mark.gpu


def _gpu_quantize(xb_cpu: torch.Tensor, scale=None, ld=None):
    rows, k = xb_cpu.shape
    if ld is not None and ld != k:
        big = torch.zeros(rows, ld, dtype=torch.bfloat16)
        big[:, :k] = xb_cpu
        xg = big.cuda()[:, :k]
    else:
        xg = xb_cpu.cuda()
    q = nv.quantize(xg, scale=scale)
    torch.cuda.synchronize()
    return q.codes.cpu().numpy(), q.sf.cpu().numpy()[: oracle.sf_bytes(rows, k)], np.float32(q.scale.item())


def _check(xb_cpu, scale=None, ld=None):
    codes, sf, g = _gpu_quantize(xb_cpu, scale, ld)
    oc, osf, og = oracle.quantize(xb_cpu, scale)
    assert g == og, (g, og)
    if not np.array_equal(codes, oc):
        bad = np.argwhere(codes != oc)[:5]
        raise AssertionError(f"codes differ at {bad.tolist()}: gpu {codes[tuple(bad[0])]:02x} oracle {oc[tuple(bad[0])]:02x}")
    assert np.array_equal(sf, osf)


def _all_finite_bf16(seed=0):
    pats = np.arange(65536, dtype=np.uint32)
    exp = (pats >> 7) & 0xFF
    pats = pats[exp != 0xFF].astype(np.uint16)          # drop inf / NaN
    rng = np.random.default_rng(seed)
    rng.shuffle(pats)
    n = ((len(pats) + 255) // 256) * 256
    full = np.zeros(n, np.uint16)
    full[: len(pats)] = pats
    return torch.from_numpy(full.view(np.int16).reshape(-1, 256)).view(torch.bfloat16)


def test_quantize_every_finite_bf16_pattern(cuda_ok):
    x = _all_finite_bf16()
    _check(x)                                            # g from the data
    for g in (2.0 ** -140, 1e-30, 2.0 ** -20, 1e-3, 0.37, 1.0, 3.0e3, 2.0 ** 60, 1e30):
        _check(x, scale=g)


def test_quantize_every_pattern_scaled_into_grid_range(cuda_ok):
    """Every bf16 mantissa at exponents that put x/s across the whole E2M1
    range, in blocks whose scales vary: exercises every rounding midpoint."""
    rng = np.random.default_rng(1)
    mant = np.arange(128, dtype=np.uint16)
    for e in range(120, 136):
        pats = (np.uint16(e) << 7 | mant)
        sign = rng.integers(0, 2, pats.size).astype(np.uint16) << 15
        vals = np.tile(pats | sign, 64)
        rng.shuffle(vals)
        x = torch.from_numpy(vals.view(np.int16).reshape(-1, 256)).view(torch.bfloat16)
        _check(x)
        _check(x, scale=float(np.float32(2.0 ** (e - 127) / 2688.0 * rng.uniform(0.5, 2.0))))


def test_quantize_exact_ties_with_power_of_two_scales(cuda_ok):
    """x / s exactly on each rounding midpoint (s a power of two), and one bf16
    ulp either side: ties must go to the even code."""
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 1.5, 3.0, 6.0, 5.5], np.float32)
    rows = []
    for m in mids:
        b = torch.tensor([m]).bfloat16().view(torch.int16).item() & 0xFFFF
        for d in (-1, 0, 1):
            rows.append((b + d) & 0xFFFF)
    vals = np.array(rows, np.uint16)
    blocks = []
    for sgn in (0, 0x8000):
        for e in (-12, -8, -3, 0):
            blk = np.zeros(16, np.uint16)
            blk[0] = (torch.tensor([6.0 * 2.0 ** e]).bfloat16().view(torch.int16).item() & 0xFFFF)
            for i, v in enumerate(vals):
                f = torch.tensor([v], dtype=torch.int16).view(torch.bfloat16).float().item() * 2.0 ** e
                blk[1 + (i % 15)] = (torch.tensor([f]).bfloat16().view(torch.int16).item() & 0xFFFF) | sgn
                if i % 15 == 14 or i == len(vals) - 1:
                    blocks.append(blk.copy())
    arr = np.concatenate(blocks)
    arr = np.concatenate([arr, np.zeros((-arr.size) % 256, np.uint16)])
    x = torch.from_numpy(arr.view(np.int16).reshape(-1, 256)).view(torch.bfloat16)
    _check(x, scale=2.0 ** -8)          # s = e4m3(2^(e+8)) * 2^-8 = 2^e exactly


@pytest.mark.parametrize("rows,k,ld,dist", [
    (1, 64, 64, "normal"), (127, 64, 64, "student_t3"), (129, 192, 200, "outlier"),
    (600, 4096, 4096, "student_t3"), (300, 320, 328, "token_scaled"), (128, 256, 256, "normal"),
    (257, 1152, 1152, "outlier"), (64, 4608, 4616, "normal"),
])
def test_quantize_shapes(cuda_ok, rows, k, ld, dist):
    x = synth.random_bf16((rows, k), seed=rows * 31 + k, dist=dist)
    _check(x, ld=ld)
    _check(x, scale=float(oracle.tensor_scale(x)) * 0.75, ld=ld)


@pytest.mark.parametrize("rows,k,ld", [(129, 192, 200), (600, 4096, 4096), (4096, 3072, 3072)])
def test_streamed_one_kernel_form(cuda_ok, monkeypatch, rows, k, ld):
    """The one-kernel form that streams the tiles through a ring of shared-memory
    buffers by TMA (the default for fake quantization; for codes a switch,
    NVFP4_QUANT_ONE_KERNEL=stream) gives the same codes, scales and tensor
    scale.  4096 x 3072 is 384 tiles over one CTA per SM: up to three tiles a
    CTA, so each CTA's six loads wrap its three-buffer ring."""
    x = synth.random_bf16((rows, k), seed=rows + 7 * k, dist="student_t3")
    monkeypatch.setenv("NVFP4_QUANT_ONE_KERNEL", "stream")
    _check(x, ld=ld)


def test_quantize_zero_single_and_empty(cuda_ok):
    z = torch.zeros(130, 128, dtype=torch.bfloat16)
    codes, sf, g = _gpu_quantize(z)
    assert g == 0 and not codes.any() and not sf.any()
    one = z.clone()
    one[129, 77] = -3.0
    _check(one)
    # rows == 0: g = 0 written, nothing else touched
    x = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    q = nv.NVFP4Tensor.empty(0, 64, "cuda")
    q.scale.fill_(5.0)
    ws = torch.empty(nv.nvfp4_quantize_workspace_bytes(0, 64), dtype=torch.uint8, device="cuda")
    nv.nvfp4_quantize(x, 0, 64, 64, q.codes, q.sf, q.scale, 0, ws, ws.numel())
    torch.cuda.synchronize()
    assert q.scale.item() == 0.0


def test_dynamic_and_given_scale_agree(cuda_ok):
    x = synth.random_bf16((256, 512), seed=5, dist="student_t3").cuda()
    q1 = nv.quantize(x)
    q2 = nv.quantize(x, scale=q1.scale.clone())
    torch.cuda.synchronize()
    assert torch.equal(q1.codes, q2.codes) and torch.equal(q1.sf, q2.sf)


@pytest.mark.parametrize("workload", ["pr1", "dit_xl2", "pixart1024"])
def test_quantize_workload_tensors_full(cuda_ok, workload):
    for layer in synth.WORKLOADS[workload].layers:
        x, w = synth.layer_tensors(workload, layer.name, device="cpu")
        _check(x)
        _check(w)


def _rows_sample(n, rng, extra=()):
    base = {0, 1, 126, 127, 128, 129, n - 1, n - 2, n // 2}
    base |= set(int(v) for v in rng.integers(0, n, 48))
    base |= set(extra)
    return np.array(sorted(r for r in base if 0 <= r < n))


@pytest.mark.parametrize("workload,layer", [("video_dit", "qkv"), ("video_dit", "fc1"), ("video_dit", "fc2"),
                                            ("w4a16", "fc2")])
def test_quantize_full_size_sampled_rows(cuda_ok, workload, layer):
    """Full-size activations quantized on the GPU; the oracle computes g over
    the whole tensor and quantizes sampled rows with it."""
    x, = synth.layer_tensors(workload, layer, device="cuda", want=("x",))
    rows, k = x.shape
    q = nv.quantize(x)
    torch.cuda.synchronize()
    xc = x.cpu()
    g = oracle.tensor_scale(xc)
    assert np.float32(q.scale.item()) == g
    rng = np.random.default_rng(7)
    sel = _rows_sample(rows, rng)
    oc, osf, _ = oracle.quantize(xc[torch.from_numpy(sel)], scale=float(g))
    gc = q.codes.cpu().numpy()[sel]
    assert np.array_equal(gc, oc)
    gsf = oracle.sf_matrix(q.sf.cpu().numpy(), rows, k)[sel]
    assert np.array_equal(gsf, oracle.sf_matrix(osf, len(sel), k))


def test_dequantize_matches_oracle(cuda_ok):
    x = synth.random_bf16((300, 512), seed=9, dist="student_t3")
    oc, osf, og = oracle.quantize(x)
    q = nv.NVFP4Tensor.empty(300, 512, "cuda")
    q.codes.copy_(torch.from_numpy(oc))
    q.sf[: osf.size].copy_(torch.from_numpy(osf))
    q.scale.fill_(float(og))
    d32 = nv.dequantize(q, torch.float32).cpu().numpy()
    d16 = nv.dequantize(q, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(d32.view(np.uint32), oracle.dequantize(oc, osf, og, "f32").view(np.uint32))
    assert np.array_equal(d16, oracle.dequantize(oc, osf, og, "bf16"))
