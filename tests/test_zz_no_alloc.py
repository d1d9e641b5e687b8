"""The allocation-free entry point bq_quantize_blockwise_nested_noalloc.

Some callers cannot allocate device memory (a plug-in whose host framework
owns every device buffer and hands it only inputs and outputs).  For them the
library keeps the fp32 first-level statistics of the compressed-statistics
quantization in a fixed device array of its own instead of a caller buffer.
This checks, through the C ABI, that two calls in a row give exactly the
outputs of bq_quantize_blockwise_nested (the entry point that takes a caller
buffer): the first call at the array's maximum size, the second smaller and of
another element type, so that it runs over what the first left in the array.

The file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import dequantization_bq_quantize_b200 as bq
from bq_inputs import codebooks, synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DT_CODE = {"f32": bq.BQ_F32, "f16": bq.BQ_F16, "bf16": bq.BQ_BF16}


def _outputs(n, bs, bs2, entries, dev):
    nb = (n + bs - 1) // bs
    out = torch.full((bq.code_bytes(n, entries),), 0xA5, dtype=torch.uint8, device=dev)
    absmax2 = torch.full(((nb + bs2 - 1) // bs2,), -1.0, dtype=torch.float32, device=dev)
    qabsmax = torch.full((nb,), 0xA5, dtype=torch.uint8, device=dev)
    return out, absmax2, qabsmax


def _both(x, dtype, bs, bs2, code, code2, stream):
    """(no-alloc outputs, outputs of the entry point with a caller buffer)."""
    n = x.numel()
    dev = x.device
    got = _outputs(n, bs, bs2, code.numel(), dev)
    st = bq.bq_quantize_blockwise_nested_noalloc(
        x.data_ptr(), DT_CODE[dtype], n, bs, code.data_ptr(), code.numel(), code2.data_ptr(), 256,
        bs2, got[0].data_ptr(), got[1].data_ptr(), got[2].data_ptr(), stream)
    assert st == bq.BQ_OK, (st, bq.bq_last_cuda_error())
    want = _outputs(n, bs, bs2, code.numel(), dev)
    absmax = torch.empty((n + bs - 1) // bs, dtype=torch.float32, device=dev)
    st = bq.bq_quantize_blockwise_nested(
        x.data_ptr(), DT_CODE[dtype], n, bs, code.data_ptr(), code.numel(), code2.data_ptr(), 256,
        bs2, absmax.data_ptr(), want[0].data_ptr(), want[1].data_ptr(), want[2].data_ptr(), stream)
    assert st == bq.BQ_OK, (st, bq.bq_last_cuda_error())
    return got, want


def test_noalloc_matches_nested_on_two_calls_in_a_row():
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream().cuda_stream
    nf4 = torch.from_numpy(codebooks.nf4()).to(dev)
    dyn8 = torch.from_numpy(codebooks.dynamic8()).to(dev)
    bq.bq_device_fault(reset=True)

    # call 1: the largest input the array allows (2^20 blocks of 64 bf16)
    n1, bs1, bs2_1 = bq.BQ_NOALLOC_MAX_BLOCKS * 64, 64, 256
    x1 = synth.with_zero_block(synth.normal(n1, "bf16", seed=41, std=0.02), bs1).to(dev)
    got1, want1 = _both(x1, "bf16", bs1, bs2_1, nf4, dyn8, stream)
    # call 2, straight after on the same stream: fewer blocks, fp32, other
    # block sizes, 8-bit element codes
    n2, bs2, bs2_2 = 300 * 256 + 37, 256, 64
    x2 = synth.with_zero_block(synth.normal(n2, "f32", seed=42), bs2).to(dev)
    got2, want2 = _both(x2, "f32", bs2, bs2_2, dyn8, dyn8, stream)
    torch.cuda.synchronize()

    for got, want in ((got1, want1), (got2, want2)):
        for name, g, w in zip(("codes", "absmax2", "qabsmax"), got, want):
            assert torch.equal(g.view(torch.uint8), w.view(torch.uint8)), name
    assert bq.bq_device_fault(reset=True) == 0

    # one block beyond the array is refused before anything is launched
    n3 = (bq.BQ_NOALLOC_MAX_BLOCKS + 1) * 32
    sentinel = _outputs(64, 32, 32, 16, dev)
    st = bq.bq_quantize_blockwise_nested_noalloc(
        x1.data_ptr(), bq.BQ_BF16, n3, 32, nf4.data_ptr(), 16, dyn8.data_ptr(), 256, 256,
        sentinel[0].data_ptr(), sentinel[1].data_ptr(), sentinel[2].data_ptr(), stream)
    assert st == bq.BQ_ERR_INVALID_ARG
    assert "BQ_NOALLOC_MAX_BLOCKS" in bq.bq_last_cuda_error()
    torch.cuda.synchronize()
    assert bool((sentinel[0] == 0xA5).all()) and bool((sentinel[2] == 0xA5).all())
