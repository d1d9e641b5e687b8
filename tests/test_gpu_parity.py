"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Codes, packed bytes and absmax must match bit for bit; dequantized values
must match exactly (the contract allows 1 ulp for bf16/fp16; the kernels do the
same single product and rounding, so exact equality is asserted).
"""
import ctypes

import numpy as np
import pytest
import torch

import dequantization_bq_quantize_b200 as bq
import oracle
from bq_inputs import codebooks, synth

from gpu_util import Guarded, device_copy, np_bits

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DT_CODE = {"f32": bq.BQ_F32, "f16": bq.BQ_F16, "bf16": bq.BQ_BF16}
EB = {"f32": 4, "f16": 2, "bf16": 2}
TABLES = {name: codebooks.get(name) for name in ("nf4", "fp4", "dyn8")}
BLOCKSIZES = [32, 64, 128, 256, 512, 1024, 2048, 4096]


@pytest.fixture(autouse=True)
def _no_fault():
    bq.bq_device_fault(reset=True)
    yield
    assert bq.bq_device_fault(reset=True) == 0, "a kernel gave up waiting (fault word set)"


def code_dev(table):
    return torch.from_numpy(np.ascontiguousarray(table, np.float32)).cuda()


def gpu_quantize(x_np, dtype, bs, table, x_offset=0, out_offset=0, stream=0):
    """Quantize host array x_np (oracle conventions) on the GPU through the
    C ABI; returns (absmax, codes) as numpy plus guard status."""
    n = x_np.size
    xt, xp = device_copy(x_np, x_offset)
    code = code_dev(table)
    nb = (n + bs - 1) // bs
    amax = Guarded(4 * nb)
    out = Guarded(oracle.code_bytes(n, table.size), out_offset)
    st = bq.bq_quantize_blockwise(xp, DT_CODE[dtype], n, bs, code.data_ptr(), table.size,
                                  amax.ptr, out.ptr, stream)
    assert st == bq.BQ_OK, (st, bq.bq_last_cuda_error())
    torch.cuda.synchronize()
    assert amax.guards_intact() and out.guards_intact()
    return amax.host().view(np.float32), out.host(), (xt, code)


def gpu_dequantize(q_np, amax_np, n, bs, table, ydtype, y_offset=0, q_offset=0):
    qt, qp = device_copy(q_np, q_offset)
    at, ap = device_copy(amax_np)
    code = code_dev(table)
    y = Guarded(EB[ydtype] * n, y_offset)
    st = bq.bq_dequantize_blockwise(qp, ap, n, bs, code.data_ptr(), table.size, y.ptr,
                                    DT_CODE[ydtype], 0)
    assert st == bq.BQ_OK, (st, bq.bq_last_cuda_error())
    torch.cuda.synchronize()
    assert y.guards_intact()
    h = y.host()
    return h.view(np.float32) if ydtype == "f32" else h.view(np.uint16)


def check_quant(x_np, dtype, bs, name, **kw):
    table = TABLES[name]
    ga, go, _ = gpu_quantize(x_np, dtype, bs, table, **kw)
    oa, oo = oracle.quantize_blockwise(x_np, dtype, bs, table)
    assert np.array_equal(ga.view(np.uint32), oa.view(np.uint32)), "absmax differs"
    bad = np.nonzero(go != oo)[0]
    assert bad.size == 0, f"{bad.size} code bytes differ, first at {bad[:5]}: gpu {go[bad[:5]]} oracle {oo[bad[:5]]}"
    return oa, oo


def check_dequant(q, amax, n, bs, name, ydtype, **kw):
    table = TABLES[name]
    gy = gpu_dequantize(q, amax, n, bs, table, ydtype, **kw)
    oy = oracle.dequantize_blockwise(q, amax, n, bs, table, ydtype)
    bad = np.nonzero(gy.view(np.uint32 if ydtype == "f32" else np.uint16) !=
                     oy.view(np.uint32 if ydtype == "f32" else np.uint16))[0]
    assert bad.size == 0, f"{bad.size} dequantized values differ, first at {bad[:5]}"


def small_input(n, dtype, bs, seed):
    """N(0,1) with one all-zero block, a block of outliers, exact table values."""
    x = synth.normal(n, dtype, seed).float()
    nb = (n + bs - 1) // bs
    if nb > 2:
        x[(nb // 2) * bs: min(n, (nb // 2 + 1) * bs)] = 0
        x[bs: 2 * bs] *= 50.0
    return np_bits(x.to(synth.TORCH_DTYPES[dtype]))


# ------------------------------------------------------------ small sweep --

@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("name", ["nf4", "fp4", "dyn8"])
@pytest.mark.parametrize("bs", BLOCKSIZES)
def test_quantize_dequantize_parity_small(dtype, name, bs):
    # several 16 KiB tiles plus a ragged tail of whole and partial blocks
    n = 5 * 8192 + 3 * bs + 37 if dtype != "f32" else 9 * 4096 + 3 * bs + 37
    x = small_input(n, dtype, bs, seed=bs + 7 * len(name))
    oa, oo = check_quant(x, dtype, bs, name)
    for ydtype in ("f32", "bf16", "f16"):
        check_dequant(oo, oa, n, bs, name, ydtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("name", ["nf4", "dyn8"])
def test_edge_sizes(dtype, name):
    for bs in (32, 64, 4096):
        for n in (1, 2, 3, 31, 32, 33, bs - 1, bs, bs + 1, 2 * bs + 37):
            x = small_input(n, dtype, bs, seed=n)
            oa, oo = check_quant(x, dtype, bs, name)
            check_dequant(oo, oa, n, bs, name, dtype)


@pytest.mark.parametrize("name", ["nf4", "dyn8"])
def test_unaligned_pointers(name):
    n, bs = 3 * 8192 + 101, 64
    x = small_input(n, "bf16", bs, seed=3)
    for x_off, o_off in ((2, 0), (0, 1), (6, 3), (16, 8)):
        check_quant(x, "bf16", bs, name, x_offset=x_off, out_offset=o_off)
    oa, oo = oracle.quantize_blockwise(x, "bf16", bs, TABLES[name])
    for y_off, q_off in ((2, 0), (0, 1), (8, 2)):
        check_dequant(oo, oa, n, bs, name, "bf16", y_offset=y_off, q_offset=q_off)


def test_special_values_and_ties():
    """Exact codebook values, midpoints between entries and their neighbours,
    tiny and huge magnitudes (the IEEE-division fallback), fp32."""
    rng = np.random.default_rng(11)
    for name in ("nf4", "fp4", "dyn8"):
        t = TABLES[name].astype(np.float64)
        mids = ((t[:-1] + t[1:]) / 2).astype(np.float32)
        vals = np.concatenate([t.astype(np.float32), mids, np.nextafter(mids, np.float32(2)),
                               np.nextafter(mids, np.float32(-2))])
        bs = 64
        blocks = []
        for scale in (1.0, 3.0, 1e-30, 1e30, 2.0 ** -126, 7.25):
            v = (vals * np.float32(scale)).astype(np.float32)
            for k in range(0, v.size, bs - 1):
                blk = np.zeros(bs, np.float32)
                part = v[k:k + bs - 1]
                blk[:part.size] = part
                blk[bs - 1] = np.float32(scale)            # absmax = scale
                blocks.append(blk)
        # blocks with a huge dynamic range: |x| far below absmax * 2^-40
        for _ in range(8):
            blk = (rng.standard_normal(bs) * np.exp(rng.uniform(-80, 0, bs))).astype(np.float32)
            blk[0] = 1.0
            blocks.append(blk)
        x = np.concatenate(blocks)
        oa, oo = check_quant(x, "f32", bs, name)
        check_dequant(oo, oa, x.size, bs, name, "f32")


def test_unsorted_and_tight_tables():
    """Tables the fast search does not accept: unsorted (plain scan) and
    tightly spaced (bisection or scan) still give the rule's result."""
    n, bs = 2 * 8192 + 77, 64
    x = small_input(n, "bf16", bs, seed=21)
    rng = np.random.default_rng(2)
    perm = TABLES["nf4"][rng.permutation(16)]
    tight = np.sort(np.concatenate([np.linspace(-1, 1, 15), [1e-7]])).astype(np.float32)
    dup = np.sort(np.concatenate([TABLES["nf4"][:12], [0.5, 0.5, 0.5, 1.0]])).astype(np.float32)
    lin256 = np.linspace(-1, 1, 256).astype(np.float32)
    for table in (perm, tight, dup, lin256):
        ga, go, _ = gpu_quantize(x, "bf16", bs, table)
        oa, oo = oracle.quantize_blockwise(x, "bf16", bs, table)
        assert np.array_equal(ga, oa) and np.array_equal(go, oo)


def test_zero_length_and_bad_arguments():
    code = code_dev(TABLES["nf4"])
    amax = torch.empty(4, device="cuda")
    out = torch.empty(64, dtype=torch.uint8, device="cuda")
    x = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    assert bq.bq_quantize_blockwise(x.data_ptr(), bq.BQ_BF16, 0, 64, code.data_ptr(), 16,
                                    amax.data_ptr(), out.data_ptr(), 0) == bq.BQ_OK
    assert bq.bq_quantize_blockwise(x.data_ptr(), bq.BQ_BF16, 64, 48, code.data_ptr(), 16,
                                    amax.data_ptr(), out.data_ptr(), 0) == bq.BQ_ERR_INVALID_ARG
    assert bq.bq_quantize_blockwise(x.data_ptr() + 1, bq.BQ_BF16, 64, 64, code.data_ptr(), 16,
                                    amax.data_ptr(), out.data_ptr(), 0) == bq.BQ_ERR_INVALID_ARG
    assert bq.bq_dequant_q8_0(0, 5, out.data_ptr(), bq.BQ_BF16, 0) == bq.BQ_ERR_INVALID_ARG


# ------------------------------------------------------------------ GGUF --

@pytest.mark.parametrize("kind", list(bq.GGUF_TYPES))
@pytest.mark.parametrize("ydtype", ["bf16", "f16", "f32"])
def test_gguf_parity(kind, ydtype):
    """Every output of every block, bit for bit, on random blocks: sizes that
    span many warp steps (the 4096 x 14336 matrix among them), partial steps,
    single blocks, and streams at byte offsets 1, 2 and 16."""
    per, bb = bq.GGUF_TYPES[kind]
    fn = getattr(bq, "bq_dequant_" + kind)
    odd = 1 if kind != "bf16" else 2      # bf16 data must be 2-byte aligned
    for nblk, off in ((4096, 0), (4096 * 14336 // per, 0), (1, 0), (7, 0), (8, 0), (9, 0),
                      (1000 + 3, 0), (1003, 2), (517, odd), (64, 16)):
        blocks = synth.gguf_blocks(nblk, kind, seed=4 + nblk)
        bt, bp = device_copy(blocks, off)
        y = Guarded(EB[ydtype] * per * nblk)
        assert fn(bp, nblk, y.ptr, DT_CODE[ydtype], 0) == bq.BQ_OK
        torch.cuda.synchronize()
        assert y.guards_intact()
        got = y.host().view(np.float32 if ydtype == "f32" else np.uint16)
        want = oracle.dequant_gguf(kind, blocks, ydtype)
        assert np.array_equal(got, want), (kind, nblk, off)


def test_gguf_hand_blocks_on_gpu():
    import test_oracle_pins as pins
    for kind, blk, expect in pins._load_hand_blocks():
        per, bb = bq.GGUF_TYPES[kind]
        fn = getattr(bq, "bq_dequant_" + kind)
        bt, bp = device_copy(blk)
        y = Guarded(4 * expect.size)
        assert fn(bp, blk.size // bb, y.ptr, bq.BQ_F32, 0) == bq.BQ_OK
        torch.cuda.synchronize()
        assert np.array_equal(y.host().view(np.uint32), expect.view(np.uint32)), kind


def test_gguf_torch_helpers():
    """The torch-level helpers: output sizes, default dtype and whole-block check."""
    for kind, (per, bb) in bq.GGUF_TYPES.items():
        blocks = synth.gguf_blocks(33, kind, seed=77)
        t = torch.from_numpy(blocks.reshape(-1)).cuda()
        y = bq.dequant_gguf(kind, t)
        assert y.dtype == torch.bfloat16 and y.numel() == 33 * per
        want = oracle.dequant_gguf(kind, blocks, "bf16")
        assert np.array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), want)
        with pytest.raises(ValueError):
            bq.dequant_gguf(kind, t[:-1])


# --------------------------------------------------------- GGUF encoders --

def _encode_input(nblk, dtype, seed, special=False):
    """N(0, 0.02) blocks, with every 7th block rounded to a grid of 1/64
    (ties on |x| and exact halves after scaling), every 11th all zeros
    (every 22nd starting with -0) and every 17th (from the 4th) drawn from
    {+-0.5, 0.25, -0.125, 0} (ties between +amax and -amax).  `special` adds blocks with inf, -inf,
    NaN, fp32/bf16 subnormals and magnitudes whose scale reciprocal
    overflows."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(nblk, 32, generator=g).mul_(0.02)
    x[::7] = torch.round(x[::7] * 64) / 64
    x[::11] = 0.0
    x[::22, 0] = -0.0
    # every 17th block: values from {+-0.5, 0.25, -0.125, 0}, so the largest
    # magnitude occurs with both signs, in random order
    pick = torch.randint(0, 5, (x[3::17].shape[0], 32), generator=g)
    x[3::17] = torch.tensor([0.5, -0.5, 0.25, -0.125, 0.0])[pick]
    if special:
        x[1::13, 3] = float("inf")
        x[2::13, 5] = -float("inf")
        x[3::13, 0] = float("nan")
        x[4::13, :] = float("nan")
        x[5::13, :] *= 2.0 ** -120           # d subnormal, 1/d overflows
        x[6::13, 9] = 2.0 ** -133            # bf16-representable subnormal maximum ...
        x[6::13, :9] = 0.0
        x[6::13, 10:] = 0.0
        x[7::13, :] = torch.tensor(1e-40)    # fp32 subnormal everywhere
        x[8::13, 4] = 65504.0 * 4            # beyond fp16 range: d overflows fp16
    return x.reshape(-1).to(synth.TORCH_DTYPES[dtype])


@pytest.mark.parametrize("kind", ["q8_0", "q4_0"])
@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
def test_gguf_encode_parity(kind, dtype):
    """Every byte of every block against the oracle: many warp steps (the
    4096 x 14336 matrix among them), partial steps, single blocks, inputs at
    element offsets that break 16-byte alignment, outputs at byte offsets."""
    bb = bq.GGUF_TYPES[kind][1]
    fn = getattr(bq, "bq_quantize_" + kind)
    for nblk, xoff, ooff in ((4096, 0, 0), (4096 * 14336 // 32, 0, 0), (1, 0, 0), (31, 0, 0),
                             (32, 0, 0), (33, 0, 0), (1003, 1, 3), (517, 0, 1), (64, 8, 16),
                             (200, 3, 0)):
        x = _encode_input(nblk, dtype, seed=nblk + xoff)
        xh = np_bits(x)
        xt, xp = device_copy(xh, xoff * EB[dtype])
        out = Guarded(nblk * bb, offset=ooff)
        assert fn(xp, DT_CODE[dtype], 32 * nblk, out.ptr, 0) == bq.BQ_OK
        torch.cuda.synchronize()
        assert out.guards_intact()
        want = oracle.quantize_gguf(kind, xh, dtype).reshape(-1)
        got = out.host()
        assert np.array_equal(got, want), (kind, dtype, nblk, xoff, ooff,
                                           int(np.nonzero(got != want)[0][0]) // bb)


@pytest.mark.parametrize("kind", ["q8_0", "q4_0"])
@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
def test_gguf_encode_special_values(kind, dtype):
    """Non-finite and subnormal inputs: the clamps give the same defined
    bytes on both sides."""
    nblk = 13 * 40
    x = _encode_input(nblk, dtype, seed=99, special=True)
    xh = np_bits(x)
    blocks = bq.quantize_gguf(kind, x.cuda())
    want = oracle.quantize_gguf(kind, xh, dtype).reshape(-1)
    assert np.array_equal(blocks.cpu().numpy(), want)


def test_gguf_encode_hand_blocks_and_round_trip():
    import test_oracle_pins as pins
    for kind, blk, x in pins._load_encode_blocks():
        for dt in ("f32", "f16", "bf16"):
            t = torch.from_numpy(x).to(synth.TORCH_DTYPES[dt]).cuda()
            assert np.array_equal(bq.quantize_gguf(kind, t).cpu().numpy(), blk), (kind, dt)
    # encode -> decode on the device equals the oracle's encode -> decode
    x = _encode_input(4096, "bf16", seed=5).cuda()
    for kind in ("q8_0", "q4_0"):
        y = bq.dequant_gguf(kind, bq.quantize_gguf(kind, x))
        want = oracle.dequant_gguf(kind, oracle.quantize_gguf(kind, np_bits(x), "bf16"), "bf16")
        assert np.array_equal(np_bits(y), want)


def test_gguf_encode_rejects_bad_arguments():
    x = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(2 * 34, dtype=torch.uint8, device="cuda")
    E = bq.BQ_ERR_INVALID_ARG
    assert bq.bq_quantize_q8_0(x.data_ptr(), bq.BQ_BF16, 63, out.data_ptr(), 0) == E
    assert bq.bq_quantize_q4_0(x.data_ptr() + 1, bq.BQ_BF16, 32, out.data_ptr(), 0) == E
    with pytest.raises(ValueError):
        bq.quantize_gguf("q8_0", x[:40])
    with pytest.raises(ValueError):
        bq.quantize_gguf("q4_k", x)
    assert bq.bq_device_fault() == 0


# ------------------------------------------------------ full-size configs --

THREADS = oracle.host_threads()


def _bits(a):
    """Raw bit patterns, so that -0 / +0 and NaN payloads count as different."""
    a = np.ascontiguousarray(a)
    return a.view({4: np.uint32, 2: np.uint16, 1: np.uint8}[a.itemsize])


def _assert_same(what, got, want):
    g, w = _bits(got), _bits(want)
    assert g.shape == w.shape, (what, g.shape, w.shape)
    bad = np.flatnonzero(g != w)
    assert bad.size == 0, f"{what}: {bad.size} of {g.size} differ, first at {bad[:5]}"


def _run_full(x_cpu, dtype, bs, name):
    """Full-size run through the torch helpers (the launch configuration the
    benchmark times), then EVERY absmax, code byte and dequantized value
    against the oracle (driven over disjoint block ranges on all host
    threads; blocks are independent, so that is the single call's result)."""
    table = TABLES[name]
    code = code_dev(table)
    n = x_cpu.numel()
    x = x_cpu.cuda()
    amax, q = bq.quantize_blockwise(x, code, bs)
    y = bq.dequantize_blockwise(q, amax, n, bs, code, dtype=x.dtype)
    torch.cuda.synchronize()
    ah, qh, yh = amax.cpu().numpy(), q.cpu().numpy(), np_bits(y.cpu())
    del x, amax, q, y
    xh = np_bits(x_cpu)
    oa, oq = oracle.quantize_blockwise_threaded(xh, dtype, bs, table, THREADS)
    _assert_same("absmax", ah, oa)
    _assert_same("codes", qh, oq)
    oy = oracle.dequantize_blockwise_threaded(oq, oa, n, bs, table, dtype, THREADS)
    _assert_same("dequantized", yh, oy)


def test_config_small_fp32_nf4_full():
    """n = 65536 fp32 N(0,1), NF4, blocksize 64: every byte against the oracle."""
    x = np_bits(synth.normal(synth.SMALL_N, "f32", 0))
    oa, oo = check_quant(x, "f32", 64, "nf4")
    check_dequant(oo, oa, x.size, 64, "nf4", "f32")


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("name", ["nf4", "fp4", "dyn8"])
def test_config_sweep_full(dtype, name):
    """The 45-cell sweep at n = 8388608 + 37 with one all-zero block: every
    output of every cell (dequantized to the cell's input dtype)."""
    for i, bs in enumerate((32, 64, 256, 1024, 4096)):
        cell = ["f16", "bf16", "f32"].index(dtype) * 15 + ["nf4", "fp4", "dyn8"].index(name) * 5 + i
        x = synth.sweep(dtype, bs, seed=1 + cell)
        _run_full(x, dtype, bs, name)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("name", ["nf4", "dyn8"])
def test_wide_blocks_ring_wrap_full(dtype, name):
    """Blocks wider than a warp of quantize threads (fp16 / bf16 blocksize
    2048 and 4096, fp32 blocksize 1024 to 4096: absmax from the statistics
    warp) and the streaming dequantization's blocksize-4096 form (each warp
    reads its scale), at n = 2^25 + 37: about 14 tiles per CTA, so every ring
    and its mbarrier phases wrap several times.  Every output against the
    oracle."""
    for i, bs in enumerate((1024, 2048, 4096)):
        x = synth.sweep(dtype, bs, seed=500 + i, n=(1 << 25) + 37)
        _run_full(x, dtype, bs, name)


def test_config_large_bf16_nf4_full():
    """bf16 n = 2^29 (1 GiB) N(0, 0.02) with 0.1% outliers, NF4, blocksize 64:
    every output (the persistent rings wrap hundreds of times per CTA)."""
    x, count = synth.large_outliers()
    assert 0.0009 < count / x.numel() < 0.0011
    _run_full(x, "bf16", 64, "nf4")


def test_config_llama_weight_set_full():
    """All 224 Llama-3-8B-shaped matrices (bf16 N(0, 0.02), NF4 blocksize 64),
    every output of each; the next matrix's input is drawn while the current
    one is checked."""
    from concurrent.futures import ThreadPoolExecutor
    mats = synth.llama_matrices(layers=32)
    draw = lambda m: synth.normal(m[3] * m[4], "bf16", m[5], std=0.02)  # noqa: E731
    with ThreadPoolExecutor(1) as ex:
        nxt = ex.submit(draw, mats[0])
        for k, m in enumerate(mats):
            x = nxt.result()
            if k + 1 < len(mats):
                nxt = ex.submit(draw, mats[k + 1])
            _run_full(x, "bf16", 64, "nf4")


# ---------------------------------------------------------- exhaustive ----

@pytest.fixture(scope="module")
def probes():
    import os
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(__file__), "gpu_probes"))
    import build as pbuild
    L = ctypes.CDLL(pbuild.build())
    u64p, u32p = ctypes.POINTER(ctypes.c_ulonglong), ctypes.POINTER(ctypes.c_uint)
    L.probe_div16.argtypes = [ctypes.c_int, u64p, u32p, u32p]
    L.probe_div32.argtypes = [ctypes.c_ulonglong, ctypes.c_ulonglong, u64p, u32p, u32p]
    L.probe_search.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                               ctypes.POINTER(ctypes.c_int), u64p, u32p, u32p]
    L.probe_wait_timeout.argtypes = [ctypes.POINTER(ctypes.c_int)]
    return L


def _outs():
    return ctypes.c_ulonglong(0), ctypes.c_uint(0), ctypes.c_uint(0)


@pytest.mark.parametrize("dt", [1, 2], ids=["f16", "bf16"])
def test_division_exhaustive_16bit(probes, dt):
    mm, fa, fb = _outs()
    assert probes.probe_div16(dt, ctypes.byref(mm), ctypes.byref(fa), ctypes.byref(fb)) == 0
    assert mm.value == 0, f"{mm.value} quotients differ, first x={fa.value:#x} A={fb.value:#x}"


def test_division_fp32_random(probes):
    mm, fa, fb = _outs()
    assert probes.probe_div32(1 << 34, 12345, ctypes.byref(mm), ctypes.byref(fa),
                              ctypes.byref(fb)) == 0
    assert mm.value == 0, f"{mm.value} quotients differ, first x={fa.value:#x} A={fb.value:#x}"


# search forms: 0 = bucket table, integer select; 3 = bucket table, float
# select (codes step by one at every threshold; FP4's +-0 pair, the one step
# of two, is handled by selecting over ranks and adding 1 from rank 8 on);
# 4 = 256-entry tables: 4-byte entries over finer buckets, select on the
# float bits.  "dup34" repeats entries 3 and 4, a step of two that only the
# integer select handles.
_DUP34 = TABLES["nf4"].copy()
_DUP34[4] = _DUP34[3]
# dyn8 with its codes -5.5e-7, 0, 5.5e-7 replaced by -1e-6, -2.5e-7, 2.9e-7:
# every gap still exceeds 2 ulp(1 + max|c|), but the threshold between the
# last two (about 2e-8) falls in the fine bucket around zero, so the 4-byte
# form is refused and the float select is built
_DYN8TINY = TABLES["dyn8"].copy()
_k0 = int(np.nonzero(_DYN8TINY == 0)[0][0])
_DYN8TINY[_k0 - 1:_k0 + 2] = np.array([-1.0e-6, -2.5e-7, 2.9e-7], np.float32)
_NAMED = {"dup34": _DUP34, "dyn8tiny": _DYN8TINY}


@pytest.mark.parametrize("name,expect_mode", [("nf4", 3), ("fp4", 3), ("dyn8", 4),
                                              ("dup34", 0), ("dyn8tiny", 3)])
@pytest.mark.parametrize("force", [-1, 1], ids=["chosen", "bisection"])
def test_search_exhaustive(probes, name, expect_mode, force):
    table = _NAMED.get(name, TABLES.get(name))
    code = code_dev(table)
    mode = ctypes.c_int(-1)
    mm, fa, fb = _outs()
    assert probes.probe_search(code.data_ptr(), table.size, force, ctypes.byref(mode),
                               ctypes.byref(mm), ctypes.byref(fa), ctypes.byref(fb)) == 0
    assert mode.value == expect_mode
    assert mm.value == 0, f"{mm.value} mismatches, first xn bits {fa.value:#x} got|want {fb.value:#x}"


def test_search_exhaustive_dyn8_float_select(probes):
    """The float-select form of a 256-entry table, which dyn8 no longer gets
    by default, checked over every float in [-1, 1] too."""
    table = TABLES["dyn8"]
    code = code_dev(table)
    mode = ctypes.c_int(-1)
    mm, fa, fb = _outs()
    assert probes.probe_search(code.data_ptr(), table.size, 3, ctypes.byref(mode),
                               ctypes.byref(mm), ctypes.byref(fa), ctypes.byref(fb)) == 0
    assert mode.value == 3
    assert mm.value == 0, f"{mm.value} mismatches, first xn bits {fa.value:#x} got|want {fb.value:#x}"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_256_entry_float_select_in_kernel(dtype):
    """The quantize kernel on a 256-entry table that gets the float select
    (the dyn8 variant above): codes, absmax and dequantized values equal the
    oracle's; tiles, tail blocks and an all-zero block included."""
    n, bs = 3 * 8192 + 333, 64
    x = small_input(n, dtype, bs, seed=31)
    table = _DYN8TINY
    ga, go, _ = gpu_quantize(x, dtype, bs, table)
    oa, oo = oracle.quantize_blockwise(x, dtype, bs, table)
    assert np.array_equal(ga.view(np.uint32), oa.view(np.uint32))
    assert np.array_equal(go, oo)
    gy = gpu_dequantize(oo, oa, n, bs, table, dtype)
    oy = oracle.dequantize_blockwise(oo, oa, n, bs, table, dtype)
    assert np.array_equal(gy.view(np.uint32 if dtype == "f32" else np.uint16),
                          oy.view(np.uint32 if dtype == "f32" else np.uint16))


def test_bounded_wait_gives_up_and_context_survives(probes):
    """An mbarrier wait that nothing completes returns 'timed out' after the
    library's limit (about 2 s) instead of hanging; the GPU stays usable."""
    res = (ctypes.c_int * 2)(-1, -1)
    assert probes.probe_wait_timeout(res) == 0
    assert res[0] == 0, "the wait claims to have completed"
    assert 1500 <= res[1] <= 10000, f"gave up after {res[1]} ms"
    # the context is still healthy: a normal quantize call works
    x = small_input(8192 * 2 + 5, "bf16", 64, seed=1)
    check_quant(x, "bf16", 64, "nf4")


# ------------------------------------------------- compressed statistics ---

def _oracle_nested(xh, dtype, bs, bs2, n, ydtype, table=None):
    """The composition of oracle calls that defines compressed statistics."""
    nf4, dyn = table if table is not None else TABLES["nf4"], TABLES["dyn8"]
    oa, oq = oracle.quantize_blockwise(xh, dtype, bs, nf4)
    oa2, oqa = oracle.quantize_blockwise(oa, "f32", bs2, dyn)
    oa_back = oracle.dequantize_blockwise(oqa, oa2, oa.size, bs2, dyn, "f32")
    oy = oracle.dequantize_blockwise(oq, oa_back, n, bs, nf4, ydtype)
    return oa, oq, oa2, oqa, oy


@pytest.mark.parametrize("dtype,bs,bs2", [("bf16", 64, 256), ("f16", 4096, 256), ("f32", 32, 256),
                                          ("bf16", 256, 32), ("f16", 32, 4096), ("bf16", 32, 64)])
def test_nested_statistics_parity(dtype, bs, bs2):
    """Compressed statistics: the absmax array quantized with the dynamic
    8-bit table in blocks of blocksize2, against the same composition of
    oracle calls; the fused dequantization against the oracle's two-step
    inverse, to every output dtype."""
    n = 300 * bs + 37
    x = synth.with_zero_block(synth.normal(n, dtype, seed=bs + bs2), bs)
    nf4, dyn = TABLES["nf4"], TABLES["dyn8"]
    q, qa, a2, a = bq.quantize_blockwise_nested(x.cuda(), code_dev(nf4), bs, code_dev(dyn), bs2)
    torch.cuda.synchronize()
    xh = np_bits(x)
    oa, oq, oa2, oqa, oy = _oracle_nested(xh, dtype, bs, bs2, n, dtype)
    assert np.array_equal(a.cpu().numpy(), oa)
    assert np.array_equal(q.cpu().numpy(), oq)
    assert np.array_equal(qa.cpu().numpy(), oqa)
    assert np.array_equal(a2.cpu().numpy(), oa2)
    for ydt in ("bf16", "f16", "f32"):
        y = bq.dequantize_blockwise_nested(q, qa, a2, n, bs, code_dev(nf4), code_dev(dyn), bs2,
                                           dtype=synth.TORCH_DTYPES[ydt])
        want = oracle.dequantize_blockwise(
            oq, oracle.dequantize_blockwise(oqa, oa2, oa.size, bs2, dyn, "f32"), n, bs, nf4, ydt)
        assert np.array_equal(np_bits(y.cpu()), want), ydt
    assert bq.bq_device_fault() == 0


def test_nested_dequant_unaligned_and_8bit():
    """The fused nested dequantization on its element-wise path (output not
    16-byte aligned) and with an 8-bit element codebook."""
    bs, bs2 = 64, 256
    n = 517 * bs + 9
    x = synth.normal(n, "bf16", seed=71)
    dyn = TABLES["dyn8"]
    for table in (TABLES["nf4"], dyn):
        q, qa, a2, a = bq.quantize_blockwise_nested(x.cuda(), code_dev(table), bs, code_dev(dyn),
                                                    bs2)
        oa, oq, oa2, oqa, oy = _oracle_nested(np_bits(x), "bf16", bs, bs2, n, "bf16", table)
        assert np.array_equal(q.cpu().numpy(), oq)
        y = Guarded(2 * n, offset=2)
        assert bq.bq_dequantize_blockwise_nested(
            q.data_ptr(), qa.data_ptr(), a2.data_ptr(), n, bs, code_dev(table).data_ptr(),
            table.size, code_dev(dyn).data_ptr(), 256, bs2, y.ptr, bq.BQ_BF16, 0) == bq.BQ_OK
        torch.cuda.synchronize()
        assert y.guards_intact()
        assert np.array_equal(y.host().view(np.uint16), oy)


def test_nested_rejects_bad_arguments():
    E = bq.BQ_ERR_INVALID_ARG
    x = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
    c16 = code_dev(TABLES["nf4"])
    c256 = code_dev(TABLES["dyn8"])
    buf = torch.zeros(8192, dtype=torch.uint8, device="cuda")
    P = buf.data_ptr()
    # code2 must have 256 entries; blocksize2 a power of two in [32, 4096]
    assert bq.bq_quantize_blockwise_nested(x.data_ptr(), bq.BQ_BF16, 4096, 64, c16.data_ptr(), 16,
                                           c16.data_ptr(), 16, 256, P, P, P, P, 0) == E
    assert bq.bq_quantize_blockwise_nested(x.data_ptr(), bq.BQ_BF16, 4096, 64, c16.data_ptr(), 16,
                                           c256.data_ptr(), 256, 100, P, P, P, P, 0) == E
    assert bq.bq_dequantize_blockwise_nested(P, P, P, 4096, 64, c16.data_ptr(), 16, 0, 256, 256,
                                             P, bq.BQ_BF16, 0) == E
    assert bq.bq_device_fault() == 0


# ------------------------------------------------------ host-input pipeline --

def _oracle_host(xh, dtype, bs, bs2, nested):
    oa, oq = oracle.quantize_blockwise(xh, dtype, bs, TABLES["nf4"])
    if not nested:
        return oa, oq
    oa2, oqa = oracle.quantize_blockwise(oa, "f32", bs2, TABLES["dyn8"])
    return oq, oqa, oa2, oa


@pytest.mark.parametrize("nested", [False, True])
@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_host_pipeline_against_oracle(nested, pinned, dtype):
    """The two-stream host pipeline against the oracle (and against one call
    on the whole device-resident input): several chunks and a ragged last
    chunk, both halves of the staging buffer reused more than once, so every
    chunk's offsets into absmax, the codes and the second-level statistics
    are checked."""
    bs, bs2 = 64, 256
    chunk = bs * bs2 * 3                        # 49152 elements
    n = chunk * 5 + 1000 * bs + 17              # 5 whole chunks and a partial one
    x = synth.with_zero_block(synth.normal(n, dtype, seed=5 + nested), bs)
    xh = x.pin_memory() if pinned else x
    nf4, dyn = code_dev(TABLES["nf4"]), code_dev(TABLES["dyn8"])
    if nested:
        got = bq.quantize_blockwise_host(xh, nf4, bs, dyn, bs2, chunk_elements=chunk)
        dev_call = bq.quantize_blockwise_nested(x.cuda(), nf4, bs, dyn, bs2)
    else:
        got = bq.quantize_blockwise_host(xh, nf4, bs, chunk_elements=chunk)
        dev_call = bq.quantize_blockwise(x.cuda(), nf4, bs)
    torch.cuda.synchronize()
    want = _oracle_host(np_bits(x), dtype, bs, bs2, nested)
    assert len(got) == len(want) == len(dev_call)
    for i, (g, w, d) in enumerate(zip(got, want, dev_call)):
        _assert_same(f"output {i}", g.cpu().numpy(), w)
        assert torch.equal(g, d)
    assert bq.bq_device_fault() == 0


def test_host_pipeline_waits_for_work_queued_on_stream0():
    """Work queued on stream0 before the call - here a delayed fill of the
    output buffers - lands before the second stream's chunks write them: the
    C call orders its second stream after stream0 by itself (the second
    stream is never synchronised with stream0 by the caller)."""
    bs = 64
    chunk = 1 << 16
    n = 7 * chunk + 333
    x = synth.normal(n, "bf16", seed=17).pin_memory()
    nf4 = code_dev(TABLES["nf4"])
    want_a, want_q = _oracle_host(np_bits(x), "bf16", bs, 256, False)
    a = torch.empty(want_a.size, device="cuda")
    q = torch.empty(want_q.size, dtype=torch.uint8, device="cuda")
    staging = torch.empty(2 * chunk * 2, dtype=torch.uint8, device="cuda")
    s0, s1 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s0):
        torch.cuda._sleep(50_000_000)        # a bounded spin, tens of ms
        a.fill_(-1.0)
        q.fill_(0xFF)
    assert bq.bq_quantize_blockwise_host(x.data_ptr(), bq.BQ_BF16, n, bs, nf4.data_ptr(), 16,
                                         None, 0, 0, a.data_ptr(), q.data_ptr(), None, None,
                                         staging.data_ptr(), staging.numel(), chunk,
                                         s0.cuda_stream, s1.cuda_stream) == bq.BQ_OK
    torch.cuda.synchronize()
    _assert_same("absmax", a.cpu().numpy(), want_a)
    _assert_same("codes", q.cpu().numpy(), want_q)


def test_host_pipeline_single_stream_and_one_chunk():
    bs = 256
    n = 3 * 65536 + 5
    x = synth.normal(n, "f16", seed=8).pin_memory()
    nf4 = code_dev(TABLES["nf4"])
    want_a, want_q = bq.quantize_blockwise(x.cuda(), nf4, bs)
    a = torch.empty_like(want_a)
    q = torch.empty_like(want_q)
    staging = torch.empty(2 * 65536 * 2, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    # both streams the same: sequential chunks
    assert bq.bq_quantize_blockwise_host(x.data_ptr(), bq.BQ_F16, n, bs, nf4.data_ptr(), 16, None,
                                         0, 0, a.data_ptr(), q.data_ptr(), None, None,
                                         staging.data_ptr(), staging.numel(), 65536, s, s) == bq.BQ_OK
    torch.cuda.synchronize()
    assert torch.equal(a, want_a) and torch.equal(q, want_q)
    # one chunk covering everything needs only one chunk of staging
    big = torch.empty(n * 2 + 64, dtype=torch.uint8, device="cuda")
    a.zero_()
    q.zero_()
    assert bq.bq_quantize_blockwise_host(x.data_ptr(), bq.BQ_F16, n, bs, nf4.data_ptr(), 16, None,
                                         0, 0, a.data_ptr(), q.data_ptr(), None, None,
                                         big.data_ptr(), big.numel(), 1 << 20, s, s) == bq.BQ_OK
    torch.cuda.synchronize()
    assert torch.equal(a, want_a) and torch.equal(q, want_q)
    # staging too small, or a chunk that is not whole blocks
    E = bq.BQ_ERR_INVALID_ARG
    assert bq.bq_quantize_blockwise_host(x.data_ptr(), bq.BQ_F16, n, bs, nf4.data_ptr(), 16, None,
                                         0, 0, a.data_ptr(), q.data_ptr(), None, None,
                                         staging.data_ptr(), staging.numel() - 16, 65536, s,
                                         s) == E
    assert bq.bq_quantize_blockwise_host(x.data_ptr(), bq.BQ_F16, n, bs, nf4.data_ptr(), 16, None,
                                         0, 0, a.data_ptr(), q.data_ptr(), None, None,
                                         staging.data_ptr(), staging.numel(), 65536 + 128, s,
                                         s) == E
    assert bq.bq_device_fault() == 0


def test_torch_helpers_check_option():
    """check=True synchronizes and reads the fault word after the launch; a
    clean run returns the same outputs as without it."""
    x = synth.normal(3 * 8192 + 101, "bf16", seed=23).cuda()
    nf4, dyn = code_dev(TABLES["nf4"]), code_dev(TABLES["dyn8"])
    a, q = bq.quantize_blockwise(x, nf4, 64, check=True)
    a0, q0 = bq.quantize_blockwise(x, nf4, 64)
    assert torch.equal(a, a0) and torch.equal(q, q0)
    y = bq.dequantize_blockwise(q, a, x.numel(), 64, nf4, check=True)
    assert torch.equal(y, bq.dequantize_blockwise(q, a, x.numel(), 64, nf4))
    qn, qa, a2, _ = bq.quantize_blockwise_nested(x, nf4, 64, dyn, 256, check=True)
    bq.dequantize_blockwise_nested(qn, qa, a2, x.numel(), 64, nf4, dyn, 256, check=True)
    blocks = bq.quantize_gguf("q4_0", x[: x.numel() // 32 * 32], check=True)
    bq.dequant_gguf("q4_0", blocks, check=True)
    bq.quantize_blockwise_host(x.cpu(), nf4, 64, chunk_elements=8192, check=True)


@pytest.mark.parametrize("bs,name", [(64, "nf4"), (4096, "nf4"), (4096, "dyn8")])
def test_ring_stage_reuse_stress(bs, name):
    """Thousands of quantize -> dequantize round trips of two alternating
    inputs through the same buffers (a 14336 x 4096 bf16 matrix), every
    output compared with references that are checked against the oracle.
    This catches a stage of a shared-memory ring being refilled by its next
    bulk copy before every consumer has read it: before the consumers'
    async-proxy fence, 16-warp dequantization CTAs gave a few wrong warps per
    thousand round trips.  Blocksize 4096 runs the statistics-warp forms of
    the quantize kernel (their tamax slots are reused every four tiles) and,
    for NF4, the streaming dequantization whose producer copies the scales."""
    table = TABLES[name]
    code = code_dev(table)
    n = 14336 * 4096
    xs, refs = [], []
    for seed in (1, 2):
        x = synth.normal(n, "bf16", seed=900 + seed, std=0.02)
        oa, oq = oracle.quantize_blockwise_threaded(np_bits(x), "bf16", bs, table, THREADS)
        oy = oracle.dequantize_blockwise_threaded(oq, oa, n, bs, table, "bf16", THREADS)
        xs.append(x.cuda())
        refs.append((torch.from_numpy(oa).cuda(), torch.from_numpy(oq).cuda(),
                     torch.from_numpy(oy.view(np.int16)).cuda()))
    a = torch.empty(n // bs, device="cuda")
    q = torch.empty(n // 2 if table.size == 16 else n, dtype=torch.uint8, device="cuda")
    y = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    bad = []
    for i in range(3000):
        k = i % 2
        bq.quantize_blockwise(xs[k], code, bs, absmax=a, out=q)
        bq.dequantize_blockwise(q, a, n, bs, code, out=y)
        ra, rq, ry = refs[k]
        if not (torch.equal(a, ra) and torch.equal(q, rq) and torch.equal(y.view(torch.int16), ry)):
            bad.append(i)
    assert not bad, f"{len(bad)} of 3000 round trips differ from the oracle, first {bad[:5]}"
