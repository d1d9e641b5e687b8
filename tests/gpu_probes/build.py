"""Build the test-only CUDA libraries under tests/gpu_probes (sm_100a):

- libbq_probes.so: the probes of bq_probes.cu (exact arithmetic, search,
  bounded waits, programmatic-dependent-launch ordering);
- libbq_testhooks.so: the library's own sources built with a 2 ms wait limit
  and the test hook that makes a producer skip one tile's copy, for the tests
  of the fault path.  libbq.so itself never has the hook.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from dequantization_bq_quantize_b200 import _build as libbuild  # noqa: E402

SRC = os.path.join(HERE, "bq_probes.cu")
LIB = os.path.join(HERE, "libbq_probes.so")
HOOKS_LIB = os.path.join(HERE, "libbq_testhooks.so")
HOOKS_FLAGS = ["-DBQ_TEST_HOOKS", "-DBQ_WAIT_LIMIT_NS=2000000ull"]


def _stale(target, deps):
    return not os.path.exists(target) or any(os.path.getmtime(d) > os.path.getmtime(target)
                                             for d in deps)


def build(force=False):
    deps = [SRC] + libbuild.DEPS
    if force or _stale(LIB, deps):
        cmd = [libbuild.nvcc(), *libbuild.NVCC_FLAGS, "-I", libbuild.INCLUDE, "-I", libbuild.CSRC,
               SRC, "-o", LIB]
        subprocess.run(cmd, check=True)
    return LIB


def build_hooks(force=False):
    if force or _stale(HOOKS_LIB, libbuild.DEPS):
        cmd = [libbuild.nvcc(), *libbuild.NVCC_FLAGS, *HOOKS_FLAGS, "-I", libbuild.INCLUDE, "-I",
               libbuild.CSRC, *libbuild.SOURCES, "-o", HOOKS_LIB]
        subprocess.run(cmd, check=True)
    return HOOKS_LIB


if __name__ == "__main__":
    print(build(force=True))
    print(build_hooks(force=True))
