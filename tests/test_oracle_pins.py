"""Pins for the CPU oracle against things other than itself.

Each test checks the oracle against a library routine, a closed form, an
invariant, a hand-worked block or an exact brute force, chosen so that a
plausible slip anywhere in the oracle (a swapped nibble, a dropped term, a
wrong sign or index, a wrong tie rule) fails at least one of them.  The
mutation tests in test_oracle_mutants.py plant such slips and check that.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from bq_inputs import codebooks, synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------ conversions --

def test_f16_widen_matches_numpy_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_to_f32(bits)
    ref = bits.view(np.float16).astype(np.float32)
    both_nan = np.isnan(ours) & np.isnan(ref)
    assert np.array_equal(ours.view(np.uint32)[~both_nan], ref.view(np.uint32)[~both_nan])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))


def test_bf16_widen_matches_torch_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_f32(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    both_nan = np.isnan(ours) & np.isnan(ref)
    assert np.array_equal(ours.view(np.uint32)[~both_nan], ref.view(np.uint32)[~both_nan])


def _narrow_cases():
    """float32 values around every rounding boundary of binary16/bfloat16."""
    rng = np.random.default_rng(7)
    f16 = np.arange(0, 0x7C00, 97, dtype=np.uint32).astype(np.uint16).view(np.float16)
    f16 = f16.astype(np.float64)
    mids = (f16[:-1] + f16[1:]) / 2                    # exact ties for f16
    bf = np.arange(0, 0x7F80, 61, dtype=np.uint32).astype(np.uint16)
    bfv = torch.from_numpy(bf.view(np.int16)).view(torch.bfloat16).double().numpy()
    bmids = (bfv[:-1] + bfv[1:]) / 2                   # exact ties for bf16
    base = np.concatenate([f16, mids, bfv, bmids]).astype(np.float32)
    up = np.nextafter(base, np.float32(np.inf))
    dn = np.nextafter(base, np.float32(-np.inf))
    special = np.array([65504, 65519.996, 65520, 65536, 1e-8, 2.9802322e-08, 2.98023259e-08,
                        5.9604645e-08, 6.0975552e-05, 6.1035156e-05, 3.0e38, 1e-40],
                       dtype=np.float32)
    rand = (rng.standard_normal(4000) * np.exp(rng.uniform(-30, 30, 4000))).astype(np.float32)
    vals = np.concatenate([base, up, dn, special, rand])
    vals = vals[np.isfinite(vals)]
    return np.concatenate([vals, -vals])


def test_f32_to_f16_matches_numpy_rne():
    vals = _narrow_cases()
    ours = oracle.f32_to_f16(vals)
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


def test_f32_to_bf16_matches_torch_rne():
    vals = _narrow_cases()
    ours = oracle.f32_to_bf16(vals)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# ------------------------------------------------------------------- GGUF --

def _load_hand_blocks():
    recs = []
    with open(os.path.join(GOLDEN, "gguf_hand_blocks.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            blk = np.frombuffer(bytes.fromhex(parts[1]), np.uint8)
            vals = []
            for tok in parts[2:]:
                v, _, k = tok.partition("*")
                vals += [float(v)] * (int(k) if k else 1)
            recs.append((parts[0], blk, np.array(vals, np.float32)))
    return recs


def test_gguf_hand_worked_blocks():
    recs = _load_hand_blocks()
    assert len(recs) == 16
    assert {r[0] for r in recs} == set(oracle.GGUF_TYPES)
    for kind, blk, expect in recs:
        per, bb = oracle.GGUF_TYPES[kind]
        assert blk.size % bb == 0 and expect.size == per * (blk.size // bb), kind
        fn = lambda b, dt, kind=kind: oracle.dequant_gguf(kind, b, dt)
        y = fn(blk, "f32")
        # bit equality (keeps the sign of zero: d = -0.5 times q = 0 is -0)
        assert np.array_equal(y.view(np.uint32), expect.view(np.uint32)), (kind, y, expect)
        # narrowed outputs are the round-to-nearest-even of the exact value
        yb = fn(blk, "bf16")
        ref_b = torch.from_numpy(expect).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(yb, ref_b)
        yh = fn(blk, "f16")
        with np.errstate(over="ignore"):
            ref_h = expect.astype(np.float16).view(np.uint16)
        assert np.array_equal(yh, ref_h)


def test_gguf_closed_form_exhaustive_bytes():
    """Every quant byte value and a sweep of d: Q8_0 = d*q, Q4_0 = d*(nib-8),
    all exact in binary32 (an fp16 d times |q| <= 128 needs <= 19 bits)."""
    ds = np.array([0x3C00, 0xB800, 0x0001, 0x03FF, 0x0400, 0x7BFF, 0x8001, 0x2E66, 0x1A3B],
                  np.uint16)
    qbytes = np.arange(256, dtype=np.uint8)
    for d in ds:
        dval = Fraction(float(np.uint16(d).view(np.float16)))
        q8 = np.zeros((8, 34), np.uint8)
        q8[:, 0], q8[:, 1] = d & 0xFF, d >> 8
        q8[:, 2:] = qbytes.reshape(8, 32)
        y = oracle.dequant_q8_0(q8, "f32")
        exp = [float(dval * int(np.int8(b))) for b in qbytes.view(np.int8)]
        assert np.array_equal(y, np.array(exp, np.float32))
        q4 = np.zeros((16, 18), np.uint8)
        q4[:, 0], q4[:, 1] = d & 0xFF, d >> 8
        q4[:, 2:] = qbytes.reshape(16, 16)
        y4 = oracle.dequant_q4_0(q4, "f32").reshape(16, 32)
        for k in range(16):
            for j in range(16):
                b = int(qbytes[16 * k + j])
                assert y4[k, j] == np.float32(float(dval * ((b & 15) - 8)))
                assert y4[k, 16 + j] == np.float32(float(dval * ((b >> 4) - 8)))


def test_gguf_matches_gguf_package():
    """Independent cross-check: the installed gguf package's numpy dequantizer,
    every block type, bit for bit (including the sign of zero)."""
    gq = pytest.importorskip("gguf.quants")
    import gguf
    T = gguf.GGMLQuantizationType
    qts = {"q8_0": T.Q8_0, "q4_0": T.Q4_0, "q4_1": T.Q4_1, "q5_0": T.Q5_0, "q5_1": T.Q5_1,
           "q2_k": T.Q2_K, "q3_k": T.Q3_K, "q4_k": T.Q4_K, "q5_k": T.Q5_K, "q6_k": T.Q6_K,
           "bf16": T.BF16}
    assert set(qts) == set(oracle.GGUF_TYPES)
    for kind, qt in qts.items():
        per = oracle.GGUF_TYPES[kind][0]
        blocks = synth.gguf_blocks({32: 512, 256: 64, 1: 4096}[per], kind, seed=11)
        ref = gq.dequantize(blocks.reshape(-1), qt).astype(np.float32).reshape(-1)
        y = oracle.dequant_gguf(kind, blocks, "f32")
        assert np.array_equal(y.view(np.uint32), ref.view(np.uint32)), kind
        if kind == "q8_0":
            assert np.array_equal(oracle.dequant_q8_0(blocks, "f32"), y)
        if kind == "q4_0":
            assert np.array_equal(oracle.dequant_q4_0(blocks, "f32"), y)


def test_gguf_more_types_exact_products():
    """Closed form of the scale arithmetic: every product in these formats is
    exact in binary32 (fp16 d: 11 bits; Q4_K d*sc*q: 11+6+4 bits; Q6_K
    d*sc*(q-32): 11+7+5 bits), so with exact rationals the only rounding is
    the add of a min, and for Q5_0 / Q6_K there is none at all."""
    for kind in ("q5_0", "q6_k"):
        blocks = synth.gguf_blocks(64, kind, seed=21)
        y = oracle.dequant_gguf(kind, blocks, "f32")
        # dequantizing in double gives bit-identical values: no rounding occurred
        per, bb = oracle.GGUF_TYPES[kind]
        d_off = 0 if kind == "q5_0" else 208
        d = blocks[:, d_off:d_off + 2].copy().view(np.float16).astype(np.float64).reshape(-1)
        scale = np.repeat(d, per) if kind == "q5_0" else None
        if kind == "q5_0":
            q = (y.astype(np.float64) / np.where(scale == 0, 1, scale))
            assert np.all(np.abs(q - np.round(q)) == 0) and q.min() >= -16 and q.max() <= 15
        else:
            sc = blocks[:, 192:208].view(np.int8).astype(np.float64)
            a = np.repeat((d[:, None] * sc).reshape(-1), 16)
            q = y.astype(np.float64) / np.where(a == 0, 1, a)
            ok = a != 0
            assert np.all(q[ok] == np.round(q[ok])) and q[ok].min() >= -32 and q[ok].max() <= 31


# ---------------------------------------------------------- GGUF encoders --

def _load_encode_blocks():
    recs = []
    with open(os.path.join(GOLDEN, "gguf_encode_blocks.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            blk = np.frombuffer(bytes.fromhex(parts[1]), np.uint8)
            x = np.array([float(v) for v in parts[2:]], np.float32)
            recs.append((parts[0], blk, x))
    return recs


def test_gguf_encode_hand_worked_blocks():
    recs = _load_encode_blocks()
    assert len(recs) == 7
    for kind, blk, x in recs:
        assert x.size == 32 and blk.size == oracle.GGUF_TYPES[kind][1]
        for dt, xv in (("f32", x), ("f16", x.astype(np.float16)),
                       ("bf16", torch.from_numpy(x).to(torch.bfloat16).view(torch.int16)
                        .numpy().view(np.uint16))):
            got = oracle.quantize_gguf(kind, xv, dt).reshape(-1)
            assert np.array_equal(got, blk), (kind, dt, got.tobytes().hex())


def test_gguf_encode_matches_gguf_package():
    """Independent cross-check: the gguf package's quantizer (bit-exact with
    the format's reference implementation), on normal data, data with many
    ties, zero blocks (one starting with -0), bf16 input widened."""
    gq = pytest.importorskip("gguf.quants")
    import gguf
    T = gguf.GGMLQuantizationType
    g = torch.Generator().manual_seed(31)
    base = torch.randn(32 * 4096, generator=g).mul_(0.02)
    cases = [base.numpy(), (base * 1000).round().numpy()]
    z = base.numpy().copy()
    z[:64] = 0.0
    z[64:96] = -0.0
    z[128] = -0.0
    z[129:160] = 0.0
    cases.append(z)
    for kind, qt in (("q8_0", T.Q8_0), ("q4_0", T.Q4_0)):
        for x in cases:
            x = np.ascontiguousarray(x, np.float32)
            ref = gq.quantize(x.reshape(-1, 32), qt)
            assert np.array_equal(oracle.quantize_gguf(kind, x, "f32"), ref), kind
        xb = base.to(torch.bfloat16)
        ref = gq.quantize(xb.float().numpy().reshape(-1, 32), qt)
        got = oracle.quantize_gguf(kind, xb.view(torch.int16).numpy().view(np.uint16), "bf16")
        assert np.array_equal(got, ref), kind


def test_gguf_encode_round_trip_bound():
    """Decoding an encoded block lands within the format's step of the input:
    |x - d*q| <= |d|/2 (Q8_0) and <= |d| (Q4_0, truncation after +8.5 can lose
    up to one step at the clamp), d being the stored fp16 scale, up to the fp16
    rounding of d times |q|."""
    g = torch.Generator().manual_seed(5)
    x = torch.randn(32 * 2048, generator=g).mul_(0.02).numpy()
    for kind, step in (("q8_0", 0.5), ("q4_0", 1.0)):
        blocks = oracle.quantize_gguf(kind, x, "f32")
        y = oracle.dequant_gguf(kind, blocks, "f32").astype(np.float64)
        d = np.abs(blocks[:, :2].copy().view(np.float16).astype(np.float64)).reshape(-1)
        dd = np.repeat(d, 32)
        # fp16 rounding of d moves every output by at most |q| * ulp16(d) / 2
        slack = 16 * dd * 2.0 ** -10 if kind == "q4_0" else 127 * dd * 2.0 ** -10
        assert np.all(np.abs(x - y) <= step * dd + slack + 1e-12), kind


# ----------------------------------------------------------- nearest code --

def _exact_nearest(xn, table):
    """Exact argmin over |xn - c_j| with rational arithmetic, lowest j on ties."""
    x = Fraction(float(xn))
    dists = [abs(x - Fraction(float(c))) for c in table]
    m = min(dists)
    return dists.index(m), dists


def _f32_round(fr):
    return np.float32(float(fr))  # Fraction -> double (exact here) -> float32 (RNE)


@pytest.mark.parametrize("name", ["nf4", "fp4", "dyn8"])
def test_nearest_code_brute_force(name):
    table = codebooks.get(name)
    rng = np.random.default_rng(3)
    xs = list(rng.uniform(-1, 1, 300).astype(np.float32))
    # every entry, every midpoint of neighbours and the floats next to them
    for a, b in zip(table[:-1], table[1:]):
        m = np.float32((np.float64(a) + np.float64(b)) / 2)
        xs += [a, b, m, np.nextafter(m, np.float32(2)), np.nextafter(m, np.float32(-2))]
    xs += [np.float32(0), np.float32(-0.0), np.float32(1), np.float32(-1), np.float32(1e-30)]
    if name == "dyn8":
        xs = xs[:: 3]
    near_ties = 0
    for xn in xs:
        got = oracle.nearest_code(xn, table)
        best, dists = _exact_nearest(xn, table)
        if got == best:
            continue
        # a difference is only allowed where rounding the distances to binary32
        # makes them equal, and then the lower index must win
        assert _f32_round(dists[got]) == _f32_round(dists[best]), (xn, got, best)
        assert got < best
        near_ties += 1
    assert near_ties <= 3


def test_nearest_code_ties_go_low():
    fp4 = codebooks.fp4()
    # -0 (index 7) and +0 (index 8) are at the same distance from every input
    assert oracle.nearest_code(0.0, fp4) == 7
    assert oracle.nearest_code(-0.0, fp4) == 7
    assert oracle.nearest_code(0.01, fp4) == 7
    # an exact midpoint between two entries goes to the lower one
    table = np.array([-1, -0.5, 0, 0.5, 1] + [2.0] * 11, np.float32)
    assert oracle.nearest_code(0.25, table) == 2
    assert oracle.nearest_code(-0.25, table) == 1
    assert oracle.nearest_code(0.75, table) == 3
    # a duplicated value: the first copy wins
    assert oracle.nearest_code(1.7, table) == 5


# ------------------------------------------------------------- quantize ----

def _unpack4(out, n):
    hi = out >> 4
    lo = out & 15
    codes = np.empty(2 * out.size, np.int64)
    codes[0::2], codes[1::2] = hi, lo
    return codes[:n]


def _widen(xb, dtype):
    if dtype == "f32":
        return xb.astype(np.float32)
    if dtype == "f16":
        return xb.view(np.float16).astype(np.float32)
    return torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).float().numpy()


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("bs", [32, 64, 256])
def test_quantize_absmax_and_codes_reference(dtype, bs):
    """absmax = max|x| per block (numpy reduction); codes = exact nearest code
    of the float32 quotient x/absmax (numpy's IEEE division)."""
    n = 3 * bs + 37
    x = synth.to_numpy_bits(synth.with_zero_block(synth.normal(n, dtype, seed=bs), bs))
    xf = _widen(x, dtype)
    for name in ("nf4", "fp4", "dyn8"):
        table = codebooks.get(name)
        absmax, out = oracle.quantize_blockwise(x, dtype, bs, table)
        nb = (n + bs - 1) // bs
        ref_amax = np.array([np.abs(xf[b * bs:(b + 1) * bs]).max() for b in range(nb)], np.float32)
        assert np.array_equal(absmax, ref_amax)
        codes = _unpack4(out, n) if table.size == 16 else out.astype(np.int64)
        if table.size == 16 and n % 2:
            assert out[-1] & 15 == 0
        A = np.repeat(ref_amax, bs)[:n]
        with np.errstate(invalid="ignore", divide="ignore"):
            xn = np.where(A == 0, np.float32(0), xf / A).astype(np.float32)
        d = np.abs(xn.astype(np.float64)[:, None] - table.astype(np.float64)[None, :])
        exact = d.argmin(axis=1)   # first minimum = lowest index on exact ties
        bad = np.nonzero(codes != exact)[0]
        for i in bad:
            got, want = int(codes[i]), int(exact[i])
            assert np.float32(d[i, got]) == np.float32(d[i, want]) and got < want, (name, i)
        assert bad.size <= 2


def test_quantize_hand_worked_packing():
    nf4 = codebooks.nf4()
    # n = 3: codes [15, 0, 7] -> bytes 0xF0, 0x70 (low nibble of the tail byte is 0)
    x = np.array([2.0, -2.0, 0.0], np.float32)
    absmax, out = oracle.quantize_blockwise(x, "f32", 32, nf4)
    assert absmax.tolist() == [2.0]
    assert out.tolist() == [0xF0, 0x70]
    # 8-bit table: one byte per element, in element order
    dyn = codebooks.dynamic8()
    absmax, out = oracle.quantize_blockwise(np.array([-1, 1, 0, 0.5], np.float32), "f32", 32, dyn)
    zero_idx = int(np.nonzero(dyn == 0)[0][0])
    assert out.tolist() == [0, 255, zero_idx, int(np.abs(dyn - 0.5).argmin())]


@pytest.mark.parametrize("name", ["nf4", "fp4", "dyn8"])
def test_round_trip_every_entry(name):
    """dequant(quant(c * A)) == c * A for every codebook entry c, fp32 input,
    A a power of two (c * A exact) or a random scale."""
    table = codebooks.get(name)
    first = {}
    for j, c in enumerate(table):
        first.setdefault(float(c), j)
    scales = [2.0 ** e for e in range(-20, 21, 5)] + [3.7, 0.011, 123.25]
    bs = 32
    for A in scales:
        A = np.float32(A)
        x = np.zeros(bs * table.size, np.float32)
        for j, c in enumerate(table):
            x[j * bs] = A                       # pins the block's absmax to A
            x[j * bs + 1] = np.float32(c) * A
            x[j * bs + 2] = -A
        absmax, out = oracle.quantize_blockwise(x, "f32", bs, table)
        assert np.all(absmax == A)
        codes = _unpack4(out, x.size) if table.size == 16 else out.astype(np.int64)
        y = oracle.dequantize_blockwise(out, absmax, x.size, bs, table, "f32")
        for j, c in enumerate(table):
            cA = np.float32(c) * A
            assert codes[j * bs + 1] == first[float(c)], (name, A, j)
            assert y[j * bs + 1] == cA
            assert y[j * bs] == A            # x = A normalises to 1, the last entry


@pytest.mark.parametrize("name,zero_code", [("nf4", 7), ("fp4", 7), ("dyn8", 127)])
def test_all_zero_block(name, zero_code):
    table = codebooks.get(name)
    assert table[zero_code] == 0
    for dtype in ("f32", "f16", "bf16"):
        x = np.zeros(64 + 5, np.float32 if dtype == "f32" else np.uint16)
        absmax, out = oracle.quantize_blockwise(x, dtype, 64, table)
        assert np.all(absmax == 0) and not np.signbit(absmax).any()
        codes = _unpack4(out, x.size) if table.size == 16 else out
        assert np.all(codes == zero_code)
        if table.size == 16:
            assert np.all(out[:-1] == (zero_code << 4 | zero_code))
        y = oracle.dequantize_blockwise(out, absmax, x.size, 64, table, "f32")
        assert np.all(y == 0)


# ----------------------------------------------------------- dequantize ----

@pytest.mark.parametrize("ydtype", ["f32", "f16", "bf16"])
def test_dequantize_is_one_product_then_narrow(ydtype):
    rng = np.random.default_rng(5)
    for table in (codebooks.nf4(), codebooks.dynamic8()):
        n, bs = 1000 + 7, 64
        nb = (n + bs - 1) // bs
        absmax = (rng.standard_normal(nb) ** 2 * 3).astype(np.float32)
        nbytes = (n + 1) // 2 if table.size == 16 else n
        q = rng.integers(0, 256, nbytes).astype(np.uint8)
        y = oracle.dequantize_blockwise(q, absmax, n, bs, table, ydtype)
        idx = _unpack4(q, n) if table.size == 16 else q.astype(np.int64)
        prod = table[idx] * np.repeat(absmax, bs)[:n]          # numpy float32 product
        if ydtype == "f32":
            assert np.array_equal(y, prod)
        elif ydtype == "f16":
            assert np.array_equal(y, prod.astype(np.float16).view(np.uint16))
        else:
            ref = torch.from_numpy(prod).to(torch.bfloat16).view(torch.int16).numpy()
            assert np.array_equal(y, ref.view(np.uint16))


def test_threaded_driver_equals_single_call():
    x = synth.to_numpy_bits(synth.normal(10000 + 37, "bf16", seed=9))
    nf4 = codebooks.nf4()
    a1, o1 = oracle.quantize_blockwise(x, "bf16", 64, nf4)
    a2, o2 = oracle.quantize_blockwise_threaded(x, "bf16", 64, nf4, threads=3)
    assert np.array_equal(a1, a2) and np.array_equal(o1, o2)
    y1 = oracle.dequantize_blockwise(o1, a1, x.size, 64, nf4, "bf16")
    y2 = oracle.dequantize_blockwise_threaded(o1, a1, x.size, 64, nf4, "bf16", threads=3)
    assert np.array_equal(y1, y2)


def test_rejects_bad_arguments():
    nf4 = codebooks.nf4()
    x = np.zeros(10, np.float32)
    with pytest.raises(ValueError):
        oracle.quantize_blockwise(x, "f32", 48, nf4)
    with pytest.raises(ValueError):
        oracle.quantize_blockwise(x, "f32", 8192, nf4)
    with pytest.raises(ValueError):
        oracle.quantize_blockwise(x, "f32", 64, np.zeros(8, np.float32))
