"""The sharded path through the library itself: every rank's range of whole
blocks (dequantization_bq_quantize_b200.shard) is quantized, dequantized or
decoded by its own calls with pointer offsets into the whole input, into its
own output buffers; the gathered (concatenated) outputs must equal the
oracle's result for the whole tensor.  The ranks are independent launches on
one GPU - no kernel waits on another - standing in for one process per GPU,
where the same calls run on each rank's device.
"""
import numpy as np
import pytest
import torch

import dequantization_bq_quantize_b200 as bq
import oracle
from bq_inputs import codebooks, synth
from dequantization_bq_quantize_b200 import shard

from gpu_util import np_bits

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

EB = {"f32": 4, "f16": 2, "bf16": 2}
DT = {"f32": bq.BQ_F32, "f16": bq.BQ_F16, "bf16": bq.BQ_BF16}


def _ok(st):
    assert st == bq.BQ_OK, (st, bq.bq_last_cuda_error())


@pytest.mark.parametrize("world", [2, 3, 8])
@pytest.mark.parametrize("name,dtype,bs", [("nf4", "bf16", 64), ("dyn8", "f32", 256),
                                           ("fp4", "f16", 4096)])
def test_sharded_quantize_dequantize_equals_oracle(world, name, dtype, bs):
    table = codebooks.get(name)
    code = torch.from_numpy(table).cuda()
    x_cpu = synth.sweep(dtype, bs, seed=60 + world)
    n = x_cpu.numel()
    x = x_cpu.cuda()
    eb = EB[dtype]
    absmax, codes, ys = [], [], []
    for lo, hi in shard.block_ranges(n, bs, world):
        m = hi - lo
        a0, na, c0, nc = shard.shard_offsets(lo, hi, bs, table.size)
        a = torch.empty(na, dtype=torch.float32, device="cuda")
        q = torch.empty(nc, dtype=torch.uint8, device="cuda")
        y = torch.empty(m, dtype=x.dtype, device="cuda")
        _ok(bq.bq_quantize_blockwise(x.data_ptr() + lo * eb, DT[dtype], m, bs, code.data_ptr(),
                                     table.size, a.data_ptr(), q.data_ptr(), 0))
        _ok(bq.bq_dequantize_blockwise(q.data_ptr(), a.data_ptr(), m, bs, code.data_ptr(),
                                       table.size, y.data_ptr(), DT[dtype], 0))
        absmax.append(a)
        codes.append(q)
        ys.append(y)
    torch.cuda.synchronize()
    xh = np_bits(x_cpu)
    oa, oq = oracle.quantize_blockwise_threaded(xh, dtype, bs, table, oracle.host_threads())
    oy = oracle.dequantize_blockwise_threaded(oq, oa, n, bs, table, dtype, oracle.host_threads())
    assert np.array_equal(torch.cat(absmax).cpu().numpy().view(np.uint32), oa.view(np.uint32))
    assert np.array_equal(torch.cat(codes).cpu().numpy(), oq)
    assert np.array_equal(np_bits(torch.cat(ys).cpu()), oy)
    assert bq.bq_device_fault() == 0


@pytest.mark.parametrize("world", [2, 8])
@pytest.mark.parametrize("kind", ["q4_0", "q8_0", "q6_k"])
def test_sharded_gguf_equals_oracle(world, kind):
    per, bb = bq.GGUF_TYPES[kind]
    nblk = 4096 * 14336 // per + 3
    blocks = synth.gguf_blocks(nblk, kind, seed=61)
    bd = torch.from_numpy(blocks.reshape(-1)).cuda()
    fn = getattr(bq, "bq_dequant_" + kind)
    parts = []
    for b0, b1 in shard.gguf_ranges(nblk, world):
        y = torch.empty((b1 - b0) * per, dtype=torch.bfloat16, device="cuda")
        _ok(fn(bd.data_ptr() + b0 * bb, b1 - b0, y.data_ptr(), bq.BQ_BF16, 0))
        parts.append(y)
    torch.cuda.synchronize()
    assert np.array_equal(np_bits(torch.cat(parts).cpu()), oracle.dequant_gguf(kind, blocks, "bf16"))
    assert bq.bq_device_fault() == 0
