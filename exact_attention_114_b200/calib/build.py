"""Build the calibration microbenchmarks (roofline denominators and the
co-running-load measurements quoted for the kernels) into calib/_build/.

    python exact_attention_114_b200/calib/build.py      # then run e.g. calib/_build/load_bench

mma_bench   cycles per tcgen05.mma (kind::f16, M = 128, K = 16) for N = 64 / 128 / 256, SS and TS operands
mufu_bench  MUFU ex2 results per clock per SM for f32, f16x2 and bf16x2
load_bench  the forward kernel's MMA sequence while other warps run MUFU, FMA, ALU or TMEM load/store work
softmax_pass_bench  the backward's P / dS pass of one query step alone on one SM, and with pieces left out
convert_bench  ex2 against the e4m3 / bf16 conversions (shared pipe or not), and an arithmetic e4m3 conversion
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "csrc")
OUT = os.path.join(HERE, "_build")
BENCHES = ("mma_bench", "mufu_bench", "load_bench", "softmax_pass_bench", "convert_bench")


def build() -> list:
    if __package__:
        from ..build import nvcc
    else:  # run as a script
        sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
        from exact_attention_114_b200.build import nvcc
    os.makedirs(OUT, exist_ok=True)
    outs = []
    for b in BENCHES:
        exe = os.path.join(OUT, b)
        src = os.path.join(HERE, b + ".cu")
        if not (os.path.exists(exe) and os.path.getmtime(exe) >= os.path.getmtime(src)):
            subprocess.run([nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                            "-I", CSRC, "-o", exe, src], check=True)
        outs.append(exe)
    return outs


if __name__ == "__main__":
    print("\n".join(build()))
