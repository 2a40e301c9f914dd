"""Build and run dequant_rate.cu (the CUDA-core MXFP4 -> bf16 dequantisation rate per SM).

    python -m block_scaled_moe_softmax_b200.probes.dequant_rate

Compiles the program for sm_100a into the package's _build folder and runs it on the
current GPU; prints elements per clock per SM for two conversions.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
BUILD = os.path.join(os.path.dirname(HERE), "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def build() -> str:
    os.makedirs(BUILD, exist_ok=True)
    exe = os.path.join(BUILD, "dequant_rate")
    src = os.path.join(HERE, "dequant_rate.cu")
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", src, "-o", exe],
                   check=True)
    return exe


if __name__ == "__main__":
    sys.exit(subprocess.run([build()]).returncode)
