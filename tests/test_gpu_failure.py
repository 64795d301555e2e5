"""Failure detection on the GPU without a GPU fault.

* A bounded device-side wait that runs out (one warp waiting on a barrier
  that nothing arrives at) returns NVFP4_ERR_TIMEOUT through dev_status, and
  the context stays usable: a quantization right after it is still exact.
* The amax pass flags Inf / NaN inputs with NVFP4_ERR_NONFINITE (inputs must
  be finite; the flag says the contract was broken) and leaves a finite input
  unflagged.
"""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_gemm_quantize_b200 as nv
from nvfp4_w4a4_gemm_quantize_b200 import synth

pytestmark = pytest.mark.gpu

TIMEOUT, NONFINITE = 6, 8


def test_bounded_wait_reports_timeout_and_context_survives(cuda_ok):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_debug_wait_timeout(status, 200_000)          # 0.2 s
    torch.cuda.synchronize()
    assert int(status.item()) == TIMEOUT
    # the context still works, and exactly
    x = synth.random_bf16((256, 512), seed=41)
    q = nv.quantize(x.cuda())
    torch.cuda.synchronize()
    codes, sf, g = oracle.quantize(x)
    assert np.float32(q.scale.item()) == g
    assert np.array_equal(q.codes.cpu().numpy(), codes)
    assert np.array_equal(q.sf.cpu().numpy()[: sf.size], sf)


@pytest.mark.parametrize("bad", [float("inf"), float("-inf"), float("nan")])
def test_amax_pass_flags_nonfinite_input(cuda_ok, bad):
    x = synth.random_bf16((300, 1024), seed=42, device="cuda")
    x[123, 517] = bad
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.quantize(x, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == NONFINITE


def test_finite_input_is_not_flagged(cuda_ok):
    x = synth.random_bf16((300, 1024), seed=43, dist="outlier", device="cuda")
    x[5, 7] = 3.0e38            # large but finite (bf16 max is about 3.39e38)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.quantize(x, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_first_error_stays(cuda_ok):
    status = torch.full((1,), TIMEOUT, dtype=torch.int32, device="cuda")
    x = synth.random_bf16((128, 256), seed=44, device="cuda")
    x[0, 0] = float("nan")
    nv.quantize(x, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == TIMEOUT
