"""The NVFP4 validity check used on the fused GEMM epilogue's output
(tests/nvfp4_validity.py) is itself checked here, on the CPU: the oracle's own
quantization of values it knows exactly passes, and planted mistakes -- a code
one grid step off, a flipped sign, a scale byte one E4M3 step off -- fail it.
A tolerance that straddles a rounding boundary admits both neighbours."""
import numpy as np
import pytest

import oracle
from nvfp4_validity import nvfp4_rounding_violations

M, N = 24, 256


def _case(seed):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((M, N)) * np.exp(rng.uniform(-2, 2, (M, 1)))
    y32 = v.astype(np.float32)
    gy = float(np.float32(np.abs(y32).max() / 2688.0 * 0.9))     # a scale that also clips
    codes, sf, _ = oracle.quantize(y32, scale=gy)
    t = np.abs(v - y32.astype(np.float64)) + 1e-12 * np.abs(v).max()
    return v, t, codes, oracle.sf_matrix(sf, M, N), gy


def _set_nibble(codes, r, c, nib):
    b = int(codes[r, c // 2])
    sh = 4 * (c & 1)
    codes[r, c // 2] = (b & (0xFF ^ (0xF << sh))) | (nib << sh)


@pytest.mark.parametrize("seed", [0, 1])
def test_exact_quantization_passes(seed):
    v, t, codes, sfm, gy = _case(seed)
    viol = nvfp4_rounding_violations(codes, sfm, gy, v, t)
    assert len(viol["scale"]) == 0 and len(viol["code"]) == 0


def test_code_one_grid_step_off_fails():
    v, t, codes, sfm, gy = _case(2)
    rng = np.random.default_rng(7)
    nib = oracle.unpack_codes(codes)
    for _ in range(60):
        r, c = int(rng.integers(M)), int(rng.integers(N))
        mag, sign = int(nib[r, c]) & 7, int(nib[r, c]) & 8
        step = 1 if mag == 0 else (-1 if mag == 7 else int(rng.choice([-1, 1])))
        bad = codes.copy()
        _set_nibble(bad, r, c, sign | (mag + step))
        viol = nvfp4_rounding_violations(bad, sfm, gy, v, t)
        assert [r, c] in viol["code"].tolist()


def test_sign_flip_fails():
    v, t, codes, sfm, gy = _case(3)
    nib = oracle.unpack_codes(codes)
    rs, cs = np.nonzero(nib & 7)
    for r, c in list(zip(rs, cs))[:40]:
        bad = codes.copy()
        _set_nibble(bad, int(r), int(c), int(nib[r, c]) ^ 8)
        assert [int(r), int(c)] in nvfp4_rounding_violations(bad, sfm, gy, v, t)["code"].tolist()


def test_scale_byte_one_step_off_fails():
    v, t, codes, sfm, gy = _case(4)
    rng = np.random.default_rng(8)
    for _ in range(60):
        r, b = int(rng.integers(M)), int(rng.integers(N // 16))
        bad = sfm.astype(np.int64)
        bad[r, b] = bad[r, b] + (1 if bad[r, b] == 0 or rng.integers(2) else -1)
        assert [r, b] in nvfp4_rounding_violations(codes, bad, gy, v, t)["scale"].tolist()


def test_tolerance_across_a_tie_admits_both_neighbours():
    # one block whose maximum fixes a power-of-two scale, so the quotients are exact
    g = np.float32(2.0 ** -8)
    v = np.zeros((1, 64))
    v[0, 0] = 6.0 * 0.5                 # a_b / (6 g) = 128: sf exact, s = 128 g = 0.5
    v[0, 1] = 2.5 * 0.5                 # quotient 2.5: the tie between codes 2 and 3 (values 2, 3 -> RNE 2)
    codes, sf, _ = oracle.quantize(v.astype(np.float32), scale=float(g))
    sfm = oracle.sf_matrix(sf, 1, 64)
    t = np.full(v.shape, 1e-3)
    assert len(nvfp4_rounding_violations(codes, sfm, g, v, t)["code"]) == 0
    alt = codes.copy()
    _set_nibble(alt, 0, 1, 0x5)         # 3.0: the value just above the tie, admissible within t
    assert len(nvfp4_rounding_violations(alt, sfm, g, v, t)["code"]) == 0
    assert len(nvfp4_rounding_violations(alt, sfm, g, v, np.zeros_like(t))["code"]) == 1
