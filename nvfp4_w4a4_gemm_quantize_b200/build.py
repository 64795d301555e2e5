"""Build the CUDA library libnvfp4.so in-tree for sm_100a with nvcc."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libnvfp4.so")
SOURCES = ["api.cu", "quantize.cu", "quantize_noalloc.cu", "layernorm.cu", "mx.cu", "blocksize.cu", "attn.cu", "gemm_w4a4.cu",
           "gemm_w4a4_2sm.cu", "gemm_w4a16.cu"]
HEADERS = ["ptx.cuh", "quant_math.cuh", "epilogue.cuh", "internal.h", "gemm.h", "tmap.h"]
INCLUDE = os.path.join(os.path.dirname(HERE), "include", "nvfp4.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v" if os.environ.get("NVFP4_PTXAS_VERBOSE") else "-O3",
    "--expt-relaxed-constexpr",
]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [INCLUDE, __file__]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["nvcc", *NVCC_FLAGS, *[os.path.join(CSRC, s) for s in SOURCES], "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed building libnvfp4.so")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
