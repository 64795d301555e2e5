"""Fused LayerNorm -> NVFP4 producer (nvfp4_layernorm_quantize) vs the CPU
oracle (oracle.layernorm_quantize): codes, scale bytes and the tensor scale
bit for bit.

Both sides form the row statistics in double and normalise with the same FP32
operations; the kernel adds a row in another order than the oracle's index
order.  Each test first checks on its inputs that the FP32 statistics do not
depend on that order (index-order and correctly rounded sums give the same
FP32 mean and 1/std), so a mismatch can only come from the kernel."""
import math

import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_gemm_quantize_b200 as nv
from nvfp4_w4a4_gemm_quantize_b200 import synth

pytestmark = pytest.mark.gpu


def _stats_order_free(x, eps=1e-6) -> bool:
    """The FP32 mean and 1/std of every row come out the same from index-order
    double sums (the oracle's) and from correctly rounded ones (math.fsum):
    the order in which the kernel adds a row then cannot change them."""
    xf = oracle.bf16_to_f32(oracle.bf16_bits(x)).astype(np.float64)
    k = xf.shape[1]

    def stats(s1, s2):
        mu = s1 / k
        var = max(s2 / k - mu * mu, 0.0)
        return np.float32(mu), np.float32(1.0 / math.sqrt(var + eps))

    seq1 = np.cumsum(xf, axis=1)[:, -1]
    seq2 = np.cumsum(xf * xf, axis=1)[:, -1]
    return all(stats(seq1[r], seq2[r]) == stats(math.fsum(xf[r]), math.fsum(xf[r] * xf[r]))
               for r in range(xf.shape[0]))


def _affine(groups, k, seed):
    rng = np.random.default_rng(seed)
    gamma = (1.0 + 0.3 * rng.standard_normal((groups, k))).astype(np.float32)
    beta = (0.2 * rng.standard_normal((groups, k))).astype(np.float32)
    return gamma, beta


def _run(x, gamma, beta, rpg, eps, scale=None):
    g = None if gamma is None else torch.from_numpy(gamma).cuda()
    b = None if beta is None else torch.from_numpy(beta).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = nv.layernorm_quantize(x.cuda(), g, b, rpg, eps, scale=scale, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return q


def _compare(q, x, gamma, beta, rpg, eps, scale=None):
    rows, k = x.shape
    c, sf, gs = oracle.layernorm_quantize(x, gamma, beta, rpg, eps, scale)
    assert np.float32(q.scale.item()) == gs
    assert np.array_equal(q.codes.cpu().numpy(), c)
    assert np.array_equal(q.sf.cpu().numpy()[: sf.size], sf)


@pytest.mark.parametrize("rows,k,dist,groups", [(37, 1152, "outlier", 3), (300, 3072, "token_scaled", 0),
                                                (130, 256, "student_t3", 1), (1, 64, "normal", 1),
                                                (513, 5120, "normal", 2)])
@pytest.mark.parametrize("given", [False, True])
def test_layernorm_quantize_bit_exact(cuda_ok, rows, k, dist, groups, given):
    x = synth.random_bf16((rows, k), seed=rows + k, dist=dist)
    assert _stats_order_free(x)
    gamma, beta = _affine(groups, k, rows) if groups else (None, None)
    rpg = -(-rows // groups) if groups else 0
    scale = 2.0 ** -9 if given else None
    q = _run(x, gamma, beta, rpg, 1e-6, scale)
    _compare(q, x, gamma, beta, rpg, 1e-6, scale)


def test_layernorm_quantize_pixart_block_input_full(cuda_ok):
    """PixArt-1024's block input (8192 tokens x 1152, two samples of 4096
    tokens, each with its own adaLN shift and scale), data-derived scale,
    every row compared."""
    x = synth.random_bf16((8192, 1152), seed=21, dist="student_t3")
    assert _stats_order_free(x)
    gamma, beta = _affine(2, 1152, 21)
    q = _run(x, gamma, beta, 4096, 1e-6)
    _compare(q, x, gamma, beta, 4096, 1e-6)


def test_layernorm_quantize_video_block_input_sampled(cuda_ok):
    """The video block input (32768 x 3072) in the benchmark's launch
    configuration: tensor scale from the whole tensor, codes and scales on
    sampled rows (the oracle quantizes those rows with that scale)."""
    x = synth.random_bf16((32768, 3072), seed=22, dist="token_scaled")
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 32767], rng.integers(0, 32768, 60)]))
    xs = x[torch.from_numpy(rows)]
    assert _stats_order_free(xs)
    q = _run(x, None, None, 0, 1e-6)
    g = np.float32(np.abs(oracle.layernorm(x)).max() / np.float32(2688.0))
    assert np.float32(q.scale.item()) == g
    c, sf, _ = oracle.layernorm_quantize(xs, scale=float(g))
    assert np.array_equal(q.codes.cpu().numpy()[rows], c)
    assert np.array_equal(oracle.sf_matrix(q.sf.cpu().numpy(), 32768, 3072)[rows], oracle.sf_matrix(sf, len(rows), 3072))


def test_layernorm_quantize_edges(cuda_ok):
    # no rows: the data-derived scale is 0
    e = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    q = nv.layernorm_quantize(e)
    torch.cuda.synchronize()
    assert q.scale.item() == 0.0
    # padding rows of the scale layout are written as zeros
    x = synth.random_bf16((200, 512), seed=3)
    out = nv.NVFP4Tensor.empty(200, 512, "cuda")
    out.sf.fill_(0xAB)
    nv.layernorm_quantize(x.cuda(), out=out)
    torch.cuda.synchronize()
    sfm = oracle.sf_matrix(out.sf.cpu().numpy(), 256, 512)
    assert np.all(sfm[200:] == 0)
    # eps must be positive
    with pytest.raises(nv.NVFP4Error):
        nv.layernorm_quantize(x.cuda(), eps=0.0)
    # an Inf in the input is reported
    xi = x.clone()
    xi[7, 9] = float("inf")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.layernorm_quantize(xi.cuda(), dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 8                                   # NVFP4_ERR_NONFINITE
