"""Build the test-only probe library tests/gpu_probes/libbq_probes.so (sm_100a)."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from dequantization_bq_quantize_b200 import _build as libbuild  # noqa: E402

SRC = os.path.join(HERE, "bq_probes.cu")
LIB = os.path.join(HERE, "libbq_probes.so")


def build(force=False):
    deps = [SRC] + libbuild.DEPS
    if not force and os.path.exists(LIB) and all(os.path.getmtime(d) <= os.path.getmtime(LIB)
                                                 for d in deps):
        return LIB
    cmd = [libbuild.nvcc(), *libbuild.NVCC_FLAGS, "-I", libbuild.INCLUDE, "-I", libbuild.CSRC,
           SRC, "-o", LIB]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
