"""nvfp4_quantize_noalloc against nvfp4_quantize, through the C ABI.

The allocation-free entry point exists for callers that cannot allocate
device memory -- a plugin whose host application owns every device buffer, a
server that allocates nothing after start-up, a caller with no CUDA allocator
binding.  It must give exactly what the workspace entry point gives (codes,
scale bytes and tensor scale, bit for bit: the quantize tests' tolerance), on
two calls in a row, since both calls share one scratch array inside the
library.  This file is collected last and needs nothing from the other tests.
"""

import numpy as np
import pytest
import torch

from nvfp4_w4a4_gemm_quantize_b200 import _lib, synth

pytestmark = pytest.mark.gpu


def _quantize_both(L, x: torch.Tensor, given_scale=None):
    rows, k = x.shape
    sfb = L.nvfp4_sf_bytes(rows, k)
    st = torch.cuda.current_stream().cuda_stream
    flags = 1 if given_scale is not None else 0
    out = []
    for which in ("workspace", "noalloc"):
        codes = torch.full((rows, k // 2), 0xAA, dtype=torch.uint8, device="cuda")
        sf = torch.full((sfb,), 0xAA, dtype=torch.uint8, device="cuda")
        scale = torch.tensor([given_scale if given_scale is not None else -1.0], dtype=torch.float32, device="cuda")
        if which == "workspace":
            wsb = L.nvfp4_quantize_workspace_bytes(rows, k)
            ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
            rc = L.nvfp4_quantize(x.data_ptr(), rows, k, x.stride(0), codes.data_ptr(), sf.data_ptr(),
                                  scale.data_ptr(), flags, ws.data_ptr() if flags == 0 else None,
                                  wsb if flags == 0 else 0, None, st)
        else:
            rc = L.nvfp4_quantize_noalloc(x.data_ptr(), rows, k, x.stride(0), codes.data_ptr(), sf.data_ptr(),
                                          scale.data_ptr(), flags, None, st)
        assert rc == 0, (which, rc)
        torch.cuda.synchronize()
        out.append((codes.cpu().numpy(), sf.cpu().numpy(), scale.item()))
    return out


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(cuda_ok):
    L = _lib.lib()
    cases = [((2048, 4608), 31, "student_t3"),      # first call on this device
             ((600, 4096), 32, "outlier"),          # second call: leftover scratch from the first
             ((32768, 3072), 33, "token_scaled")]   # a full-size activation
    for (shape, seed, dist) in cases:
        x = synth.random_bf16(shape, seed=seed, dist=dist, device="cuda")
        (c0, s0, g0), (c1, s1, g1) = _quantize_both(L, x)
        assert np.float32(g0) == np.float32(g1)
        assert np.array_equal(c0, c1)
        assert np.array_equal(s0, s1)
    # after nvfp4_shutdown() the scratch address is looked up again: still the same results
    L.nvfp4_shutdown()
    x = synth.random_bf16((1024, 2048), seed=35, dist="student_t3", device="cuda")
    (c0, s0, g0), (c1, s1, g1) = _quantize_both(L, x)
    assert np.float32(g0) == np.float32(g1) and np.array_equal(c0, c1) and np.array_equal(s0, s1)
    # with a caller-given tensor scale (no scratch involved) the two agree too
    x = synth.random_bf16((256, 512), seed=34, device="cuda")
    (c0, s0, g0), (c1, s1, g1) = _quantize_both(L, x, given_scale=1e-3)
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1) and g0 == g1


def test_noalloc_rejects_bad_arguments_before_launch(cuda_ok):
    L = _lib.lib()
    A, B, C = 0x10000, 0x20000, 0x30000
    assert L.nvfp4_quantize_noalloc(A, 128, 96, 96, B, C, A, 0, None, None) == 2       # k % 64
    assert L.nvfp4_quantize_noalloc(A + 2, 128, 256, 256, B, C, A, 0, None, None) == 3  # misaligned
    assert L.nvfp4_quantize_noalloc(A, 128, 256, 256, B, C, None, 0, None, None) == 1   # no scale
