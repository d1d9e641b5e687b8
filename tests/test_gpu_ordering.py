"""Stream ordering: every entry point sees what earlier work on the caller's
stream wrote ("bitsandbytes PR #2052", Reproduced failure: a producer on
PyTorch's current stream and blockwise quantization on the legacy default
stream read stale data for direct General8, compressed-statistics General8,
direct NF4 and compressed-statistics NF4).

Each case fills an input on a non-blocking stream after a device-side delay of
tens of milliseconds and calls the entry point at once.  On the caller's stream
the result must equal the oracle's for the final input; the control makes the
same call on the legacy default stream, which does not wait for that stream,
and must see the stale input (so the case can tell the two apart).

The late-writer cases go further: the codebook is written by a kernel that is
still running when the library's kernel starts under programmatic dependent
launch.
"""
import ctypes
import os
import sys

import numpy as np
import pytest
import torch

import dequantization_bq_quantize_b200 as bq
import oracle
from bq_inputs import codebooks, synth

from gpu_util import np_bits

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

TABLES = {name: codebooks.get(name) for name in ("nf4", "fp4", "dyn8")}
N, BS, BS2 = 1 << 20, 64, 256
DELAY_CYCLES = 50_000_000  # torch.cuda._sleep: a bounded spin, tens of ms


@pytest.fixture(autouse=True)
def _no_fault():
    bq.bq_device_fault(reset=True)
    yield
    assert bq.bq_device_fault(reset=True) == 0, "a kernel gave up waiting (fault word set)"


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _input(dtype="bf16", n=N, seed=5):
    return np_bits(synth.with_zero_block(synth.normal(n, dtype, seed), BS))


def _late(pairs, call, on_callers_stream):
    """On a fresh non-blocking stream: delay, copy each (dst, final) pair,
    then call(stream handle) - the caller's stream, or the legacy stream."""
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        torch.cuda._sleep(DELAY_CYCLES)
        for dst, final in pairs:
            dst.copy_(final)
        call(s.cuda_stream if on_callers_stream else 0)
    torch.cuda.synchronize()


def _ok(st):
    assert st == bq.BQ_OK, (st, bq.bq_last_cuda_error())


# --------------------------------------------------------------- cases ----

def case_quantize(name):
    table = TABLES[name]
    xh = _input()
    want = oracle.quantize_blockwise(xh, "bf16", BS, table)

    def run(on_callers_stream):
        final = dev(xh.view(np.int16))
        x = torch.zeros_like(final)
        code = dev(table)
        a = torch.empty(N // BS, device="cuda")
        q = torch.empty(bq.code_bytes(N, table.size), dtype=torch.uint8, device="cuda")
        _late([(x, final)], lambda st: _ok(bq.bq_quantize_blockwise(
            x.data_ptr(), bq.BQ_BF16, N, BS, code.data_ptr(), table.size, a.data_ptr(),
            q.data_ptr(), st)), on_callers_stream)
        return np.array_equal(a.cpu().numpy(), want[0]) and np.array_equal(q.cpu().numpy(), want[1])
    return run


def case_quantize_nested(name):
    table, dyn = TABLES[name], TABLES["dyn8"]
    xh = _input()
    oa, oq = oracle.quantize_blockwise(xh, "bf16", BS, table)
    oa2, oqa = oracle.quantize_blockwise(oa, "f32", BS2, dyn)

    def run(on_callers_stream):
        final = dev(xh.view(np.int16))
        x = torch.zeros_like(final)
        c1, c2 = dev(table), dev(dyn)
        nb = N // BS
        a = torch.empty(nb, device="cuda")
        q = torch.empty(bq.code_bytes(N, table.size), dtype=torch.uint8, device="cuda")
        a2 = torch.empty(nb // BS2, device="cuda")
        qa = torch.empty(nb, dtype=torch.uint8, device="cuda")
        _late([(x, final)], lambda st: _ok(bq.bq_quantize_blockwise_nested(
            x.data_ptr(), bq.BQ_BF16, N, BS, c1.data_ptr(), table.size, c2.data_ptr(), 256, BS2,
            a.data_ptr(), q.data_ptr(), a2.data_ptr(), qa.data_ptr(), st)), on_callers_stream)
        return (np.array_equal(q.cpu().numpy(), oq) and np.array_equal(qa.cpu().numpy(), oqa)
                and np.array_equal(a2.cpu().numpy(), oa2))
    return run


def case_dequantize():
    table = TABLES["nf4"]
    oa, oq = oracle.quantize_blockwise(_input(), "bf16", BS, table)
    want = oracle.dequantize_blockwise(oq, oa, N, BS, table, "bf16")

    def run(on_callers_stream):
        fq, fa = dev(oq), dev(oa)
        q, a = torch.zeros_like(fq), torch.zeros_like(fa)
        code = dev(table)
        y = torch.empty(N, dtype=torch.bfloat16, device="cuda")
        _late([(q, fq), (a, fa)], lambda st: _ok(bq.bq_dequantize_blockwise(
            q.data_ptr(), a.data_ptr(), N, BS, code.data_ptr(), 16, y.data_ptr(), bq.BQ_BF16,
            st)), on_callers_stream)
        return np.array_equal(np_bits(y), want)
    return run


def case_dequantize_nested():
    table, dyn = TABLES["nf4"], TABLES["dyn8"]
    oa, oq = oracle.quantize_blockwise(_input(), "bf16", BS, table)
    oa2, oqa = oracle.quantize_blockwise(oa, "f32", BS2, dyn)
    want = oracle.dequantize_blockwise(
        oq, oracle.dequantize_blockwise(oqa, oa2, oa.size, BS2, dyn, "f32"), N, BS, table, "bf16")

    def run(on_callers_stream):
        fq, fqa, fa2 = dev(oq), dev(oqa), dev(oa2)
        q, qa, a2 = torch.zeros_like(fq), torch.zeros_like(fqa), torch.zeros_like(fa2)
        c1, c2 = dev(table), dev(dyn)
        y = torch.empty(N, dtype=torch.bfloat16, device="cuda")
        _late([(q, fq), (qa, fqa), (a2, fa2)], lambda st: _ok(bq.bq_dequantize_blockwise_nested(
            q.data_ptr(), qa.data_ptr(), a2.data_ptr(), N, BS, c1.data_ptr(), 16, c2.data_ptr(),
            256, BS2, y.data_ptr(), bq.BQ_BF16, st)), on_callers_stream)
        return np.array_equal(np_bits(y), want)
    return run


def case_gguf(kind):
    nblk = 1 << 15
    blocks = synth.gguf_blocks(nblk, kind, seed=6)
    per = bq.GGUF_TYPES[kind][0]
    want = oracle.dequant_gguf(kind, blocks, "bf16")

    def run(on_callers_stream):
        fb = dev(blocks.reshape(-1))
        b = torch.zeros_like(fb)
        y = torch.empty(per * nblk, dtype=torch.bfloat16, device="cuda")
        fn = getattr(bq, "bq_dequant_" + kind)
        _late([(b, fb)], lambda st: _ok(fn(b.data_ptr(), nblk, y.data_ptr(), bq.BQ_BF16, st)),
              on_callers_stream)
        return np.array_equal(np_bits(y), want)
    return run


def case_encode(kind):
    xh = np_bits(synth.normal(N, "bf16", seed=9, std=0.02))
    want = oracle.quantize_gguf(kind, xh, "bf16").reshape(-1)

    def run(on_callers_stream):
        final = dev(xh.view(np.int16))
        x = torch.zeros_like(final)
        out = torch.empty(want.size, dtype=torch.uint8, device="cuda")
        fn = getattr(bq, "bq_quantize_" + kind)
        _late([(x, final)], lambda st: _ok(fn(x.data_ptr(), bq.BQ_BF16, N, out.data_ptr(), st)),
              on_callers_stream)
        return np.array_equal(out.cpu().numpy(), want)
    return run


def case_host_pipeline():
    """The host pipeline's device-side input, the codebook, is written late on
    stream0; the call's second stream must wait for it too."""
    table = TABLES["nf4"]
    xh = _input(n=N + 4096 + 17)
    n = xh.size
    want = oracle.quantize_blockwise(xh, "bf16", BS, table)
    xpin = torch.from_numpy(xh.view(np.int16)).pin_memory()
    chunk = 1 << 17

    def run(on_callers_stream):
        final = dev(table)
        code = torch.zeros_like(final)
        a = torch.empty((n + BS - 1) // BS, device="cuda")
        q = torch.empty(bq.code_bytes(n, 16), dtype=torch.uint8, device="cuda")
        staging = torch.empty(2 * chunk * 2, dtype=torch.uint8, device="cuda")
        side = torch.cuda.Stream()
        _late([(code, final)], lambda st: _ok(bq.bq_quantize_blockwise_host(
            xpin.data_ptr(), bq.BQ_BF16, n, BS, code.data_ptr(), 16, None, 0, 0, a.data_ptr(),
            q.data_ptr(), None, None, staging.data_ptr(), staging.numel(), chunk, st,
            side.cuda_stream)), on_callers_stream)
        return np.array_equal(a.cpu().numpy(), want[0]) and np.array_equal(q.cpu().numpy(), want[1])
    return run


CASES = {
    "quantize_nf4": lambda: case_quantize("nf4"),
    "quantize_dyn8": lambda: case_quantize("dyn8"),
    "nested_nf4": lambda: case_quantize_nested("nf4"),
    "nested_dyn8": lambda: case_quantize_nested("dyn8"),
    "dequantize": case_dequantize,
    "dequantize_nested": case_dequantize_nested,
    "gguf_q4_0": lambda: case_gguf("q4_0"),
    "gguf_q6_k": lambda: case_gguf("q6_k"),
    "encode_q8_0": lambda: case_encode("q8_0"),
    "encode_q4_0": lambda: case_encode("q4_0"),
    "host_pipeline": case_host_pipeline,
}


@pytest.mark.parametrize("case", list(CASES))
def test_respects_callers_stream(case):
    """On the caller's stream the entry point sees the final input."""
    assert CASES[case]()(True)


@pytest.mark.parametrize("case", list(CASES))
def test_ordering_control_on_legacy_stream(case):
    """Control: the same sequence on the legacy default stream reads stale
    input, so the case above can tell the two apart."""
    assert not CASES[case]()(False)


# ------------------------------------------------- codebook written late ----

@pytest.fixture(scope="module")
def probes():
    sys.path.insert(0, os.path.join(os.path.dirname(__file__), "gpu_probes"))
    import build as pbuild
    L = ctypes.CDLL(pbuild.build())
    vp = ctypes.c_void_p
    L.probe_late_write.argtypes = [vp, vp, ctypes.c_int, ctypes.c_ulonglong, vp]
    L.probe_early_read.argtypes = [vp, ctypes.c_int, vp, vp]
    return L


SPIN_NS = 20_000_000  # the late writer spins 20 ms before writing
# The first launch of a kernel in a process loads its module and does not
# overlap the kernel before it, so every sequence below runs once as a
# warm-up (short spin) before the checked run.
WARM_NS = 100_000
_STREAMS = []


def _pdl_stream():
    """A fresh non-blocking stream (kept alive for the session) for the
    dependent-launch sequences."""
    _STREAMS.append(torch.cuda.Stream())
    return _STREAMS[-1].cuda_stream


def test_late_writer_opens_a_window(probes):
    """Control: a kernel launched after the late writer under programmatic
    dependent launch reads the old codebook before its wait and the new one
    after it, so the tests below do exercise a codebook that changes under a
    running quantize kernel."""
    old, new = dev(TABLES["fp4"]), dev(TABLES["nf4"])
    assert old[1].item() != new[1].item()
    out = torch.zeros(2, device="cuda")
    s = _pdl_stream()
    scratch = torch.zeros(16, device="cuda")
    for dst, spin in ((scratch, WARM_NS), (old, SPIN_NS)):
        torch.cuda.synchronize()
        assert probes.probe_late_write(dst.data_ptr(), new.data_ptr(), 16, spin, s) == 0
        assert probes.probe_early_read(dst.data_ptr(), 1, out.data_ptr(), s) == 0
    torch.cuda.synchronize()
    assert out[0].item() == TABLES["fp4"][1] and out[1].item() == TABLES["nf4"][1]


@pytest.mark.parametrize("old_name,new_name", [("fp4", "nf4"), ("nf4", "fp4"),
                                               ("lin256", "dyn8")])
@pytest.mark.parametrize("between", [0, 1, 2], ids=["direct", "one_call_between",
                                                     "two_calls_between"])
def test_codebook_written_by_a_running_kernel(probes, old_name, new_name, between):
    """The codebook is rewritten by a kernel that is still running when the
    quantize kernel starts (directly before it, or with one or two library
    calls in between on the same stream): the quantize kernel must use the
    new table."""
    tables = dict(TABLES, lin256=np.linspace(-1, 1, 256).astype(np.float32))
    old, new = tables[old_name], tables[new_name]
    xh = _input(n=3 * 8192 * 8 + 5 * BS + 7, seed=12)
    n = xh.size
    want = oracle.quantize_blockwise(xh, "bf16", BS, new)
    x = dev(xh.view(np.int16))
    code, src = dev(old), dev(new)
    a = torch.empty((n + BS - 1) // BS, device="cuda")
    q = torch.empty(bq.code_bytes(n, new.size), dtype=torch.uint8, device="cuda")
    # library calls in between: dequantizations of unrelated buffers
    fq = torch.zeros(8192, dtype=torch.uint8, device="cuda")
    fa = torch.ones(8192 * 2 // BS, device="cuda")
    fy = torch.empty(8192 * 2, dtype=torch.bfloat16, device="cuda")
    other = dev(TABLES["nf4"])
    s = _pdl_stream()
    warm = dev(new)
    for table, spin in ((warm, WARM_NS), (code, SPIN_NS)):
        torch.cuda.synchronize()
        assert probes.probe_late_write(table.data_ptr(), src.data_ptr(), new.size, spin, s) == 0
        for _ in range(between):
            _ok(bq.bq_dequantize_blockwise(fq.data_ptr(), fa.data_ptr(), fy.numel(), BS,
                                           other.data_ptr(), 16, fy.data_ptr(), bq.BQ_BF16, s))
        _ok(bq.bq_quantize_blockwise(x.data_ptr(), bq.BQ_BF16, n, BS, table.data_ptr(), new.size,
                                     a.data_ptr(), q.data_ptr(), s))
    torch.cuda.synchronize()
    assert np.array_equal(a.cpu().numpy(), want[0])
    assert np.array_equal(q.cpu().numpy(), want[1])


def test_codebook_produced_by_the_preceding_library_call(probes):
    """The codebook is the output of the dequantization launched just before
    the quantization on the same stream (its last 16 fp32 outputs decode to
    the NF4 table), with a late writer ahead of both so that the quantize
    kernel starts while the codebook is still being produced."""
    nf4 = TABLES["nf4"]
    m = 1 << 22                       # dequantized elements, the last 16 form the table
    # codes: all zero, except the last 16 elements which take codes 0..15
    q = np.zeros(m // 2, np.uint8)
    q[-8:] = np.array([(2 * i) << 4 | (2 * i + 1) for i in range(8)], np.uint8)
    amax = np.ones(m // 32, np.float32)
    qd, ad, c16 = dev(q), dev(amax), dev(nf4)
    y = torch.full((m,), 7.0, device="cuda")          # fp32 output; table = y[-16:]
    xh = _input(n=8192 * 16 + 3 * BS, seed=13)
    n = xh.size
    want = oracle.quantize_blockwise(xh, "bf16", BS, nf4)
    x = dev(xh.view(np.int16))
    a = torch.empty((n + BS - 1) // BS, device="cuda")
    out = torch.empty(bq.code_bytes(n, 16), dtype=torch.uint8, device="cuda")
    junk, fill = torch.zeros(16, device="cuda"), torch.zeros(16, device="cuda")
    s = _pdl_stream()
    code_ptr = y.data_ptr() + 4 * (m - 16)
    for spin in (WARM_NS, SPIN_NS):
        torch.cuda.synchronize()
        y.fill_(7.0)
        torch.cuda.synchronize()
        assert probes.probe_late_write(junk.data_ptr(), fill.data_ptr(), 16, spin, s) == 0
        _ok(bq.bq_dequantize_blockwise(qd.data_ptr(), ad.data_ptr(), m, 32, c16.data_ptr(), 16,
                                       y.data_ptr(), bq.BQ_F32, s))
        _ok(bq.bq_quantize_blockwise(x.data_ptr(), bq.BQ_BF16, n, BS, code_ptr, 16, a.data_ptr(),
                                     out.data_ptr(), s))
    torch.cuda.synchronize()
    assert np.array_equal(y[-16:].cpu().numpy(), nf4)
    assert np.array_equal(a.cpu().numpy(), want[0])
    assert np.array_equal(out.cpu().numpy(), want[1])
