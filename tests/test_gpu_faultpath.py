"""The give-up path of the bounded waits, in the pipelined kernels themselves.

Every mbarrier wait of the quantize and streaming dequantize kernels gives up
after a time limit, sets a bit of the device fault word and leaves the kernel,
so that a lost copy cannot hang the GPU.  These tests use a test-only build of
the library's own sources (tests/gpu_probes/libbq_testhooks.so: a 2 ms limit
and a hook that makes the producer skip one tile's copy; libbq.so has
neither).  The skipped copy is the only thing that goes wrong - there is no
invalid memory access - and the tests check that the call returns, that the
kernel leaves within a few limits, that the fault word names the waits that
gave up, that reading it with reset clears it, and that the same context then
computes the oracle's results.
"""
import ctypes
import os
import sys
import time

import numpy as np
import pytest
import torch

import dequantization_bq_quantize_b200 as bq
import oracle
from bq_inputs import codebooks, synth

from gpu_util import np_bits

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

NF4 = codebooks.nf4()


@pytest.fixture(scope="module")
def H():
    sys.path.insert(0, os.path.join(os.path.dirname(__file__), "gpu_probes"))
    import build as pbuild
    L = ctypes.CDLL(pbuild.build_hooks())
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    L.bq_quantize_blockwise.argtypes = [vp, i32, i64, i32, vp, i32, vp, vp, vp]
    L.bq_dequantize_blockwise.argtypes = [vp, vp, i64, i32, vp, i32, vp, i32, vp]
    L.bq_device_fault.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
    L.bq_test_skip_tile.argtypes = [i64]
    for f in ("bq_quantize_blockwise", "bq_dequantize_blockwise", "bq_device_fault",
              "bq_test_skip_tile"):
        getattr(L, f).restype = ctypes.c_int
    yield L
    L.bq_test_skip_tile(-1)


def _fault(L, reset):
    v = ctypes.c_uint32(0)
    assert L.bq_device_fault(ctypes.byref(v), 1 if reset else 0) == 0
    return v.value


# At least 8 tiles per CTA for either kernel on 148 SMs (quantize: 2 CTAs
# per SM and 8192 bf16 elements per tile; streaming dequantize: 3 CTAs per
# SM, 8192 elements per tile), so the producer of the CTA whose tile is
# skipped reaches the stage its consumers never freed and its own wait runs
# out too
N = 4 * 148 * 8 * 8192
SKIP = 2 * 4 * 148


@pytest.mark.parametrize("bs,name", [(64, "nf4"), (4096, "nf4"), (4096, "dyn8")])
def test_quantize_consumer_and_producer_waits_give_up(H, bs, name):
    """Blocksize 64: the consumers' shuffle-tree form; blocksize 4096: the
    statistics-warp forms (two statistics warps for NF4, one for dyn8),
    whose statistics warps wait on the skipped tile as well."""
    table = codebooks.get(name)
    x = synth.normal(N, "bf16", seed=31, std=0.02)
    xd = x.cuda()
    code = torch.from_numpy(table).cuda()
    a = torch.empty(N // bs, device="cuda")
    q = torch.empty(N // 2 if table.size == 16 else N, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    _fault(H, True)
    assert H.bq_test_skip_tile(SKIP) == bq.BQ_OK
    t0 = time.perf_counter()
    assert H.bq_quantize_blockwise(xd.data_ptr(), bq.BQ_BF16, N, bs, code.data_ptr(), table.size,
                                   a.data_ptr(), q.data_ptr(), 0) == bq.BQ_OK
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    f = _fault(H, True)
    assert f & 1, f"consumer wait did not give up (fault word {f:#x})"
    assert f & 2, f"producer wait did not give up (fault word {f:#x})"
    assert f & ~3 == 0, f"unexpected fault bits {f:#x}"
    assert elapsed < 1.0, f"the kernel took {elapsed:.3f} s to leave"
    assert _fault(H, False) == 0, "reset did not clear the fault word"
    # the context is healthy: without the hook the same call gives the oracle's result
    assert H.bq_test_skip_tile(-1) == bq.BQ_OK
    assert H.bq_quantize_blockwise(xd.data_ptr(), bq.BQ_BF16, N, bs, code.data_ptr(), table.size,
                                   a.data_ptr(), q.data_ptr(), 0) == bq.BQ_OK
    torch.cuda.synchronize()
    assert _fault(H, True) == 0
    oa, oq = oracle.quantize_blockwise_threaded(np_bits(x), "bf16", bs, table,
                                                oracle.host_threads())
    assert np.array_equal(a.cpu().numpy(), oa) and np.array_equal(q.cpu().numpy(), oq)


def test_streaming_dequantize_waits_give_up(H):
    x = synth.normal(N, "bf16", seed=32, std=0.02)
    oa, oq = oracle.quantize_blockwise_threaded(np_bits(x), "bf16", 64, NF4,
                                                oracle.host_threads())
    a, q = torch.from_numpy(oa).cuda(), torch.from_numpy(oq).cuda()
    code = torch.from_numpy(NF4).cuda()
    y = torch.empty(N, dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    _fault(H, True)
    assert H.bq_test_skip_tile(SKIP) == bq.BQ_OK
    t0 = time.perf_counter()
    assert H.bq_dequantize_blockwise(q.data_ptr(), a.data_ptr(), N, 64, code.data_ptr(), 16,
                                     y.data_ptr(), bq.BQ_BF16, 0) == bq.BQ_OK
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    f = _fault(H, True)
    assert f & 4, f"consumer wait did not give up (fault word {f:#x})"
    assert f & 8, f"producer wait did not give up (fault word {f:#x})"
    assert f & ~12 == 0, f"unexpected fault bits {f:#x}"
    assert elapsed < 1.0, f"the kernel took {elapsed:.3f} s to leave"
    assert _fault(H, False) == 0
    assert H.bq_test_skip_tile(-1) == bq.BQ_OK
    assert H.bq_dequantize_blockwise(q.data_ptr(), a.data_ptr(), N, 64, code.data_ptr(), 16,
                                     y.data_ptr(), bq.BQ_BF16, 0) == bq.BQ_OK
    torch.cuda.synchronize()
    assert _fault(H, True) == 0
    want = oracle.dequantize_blockwise_threaded(oq, oa, N, 64, NF4, "bf16", oracle.host_threads())
    assert np.array_equal(np_bits(y.cpu()), want)


def test_product_library_has_no_test_hook():
    assert not hasattr(bq.lib(), "bq_test_skip_tile")
