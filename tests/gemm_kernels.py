"""Which W4A4 kernel a GPU test runs on.

The library picks the kernel from the shape: the CTA-pair kernel (256 x 192
tiles when N % 192 == 0, else 256 x 256 when N % 256 == 0) when the problem
has enough pair tiles to fill the GPU, else the single-CTA kernel.  Small
test shapes would therefore never reach the pair kernels, so tests force the
choice through the two variables the library reads at every launch
(NVFP4_GEMM_KERNEL = pair | single, NVFP4_PAIR_TILE_N = 192 | 256).
"""
import pytest

KERNELS = ["auto", "pair192", "pair256", "single"]


def select_kernel(monkeypatch, kernel: str, N: int) -> None:
    if kernel == "auto":
        return
    if kernel == "single":
        monkeypatch.setenv("NVFP4_GEMM_KERNEL", "single")
        return
    bn = 192 if kernel == "pair192" else 256
    if N % bn:
        pytest.skip(f"N = {N} is no multiple of {bn}")
    monkeypatch.setenv("NVFP4_GEMM_KERNEL", "pair")
    monkeypatch.setenv("NVFP4_PAIR_TILE_N", str(bn))
