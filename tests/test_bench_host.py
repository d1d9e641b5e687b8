"""Host-side checks of bench.py: the algorithmic byte counts behind every GB/s
and roofline figure, the percentile helper, and the JSON line of the
reference arm (the oracle timed on the host cores), run on the CPU."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_quantize_bytes_match_the_per_element_figures():
    # in + out per element: s + 1/2 + 4/bs for 4-bit codes, s + 1 + 4/bs for
    # 8-bit codes; the 1 GiB bf16 NF4 bs 64 case moves 2^30 + 2^28 + 2^25 bytes
    n = 1 << 29
    assert bench.quant_bytes(n, 64) == (1 << 30) + (1 << 28) + (1 << 25) == 1_375_731_712
    assert bench.quant_bytes(n, 64, entries=256) == (1 << 30) + (1 << 29) + (1 << 25)
    assert bench.quant_bytes(n, 64, elem=4) == (1 << 31) + (1 << 28) + (1 << 25)
    # odd n: the last packed byte is shared, the tail block has its own absmax
    assert bench.quant_bytes(8388645, 64) == 2 * 8388645 + 4194323 + 4 * 131073


def test_gguf_bytes_match_the_block_formats():
    nblk = 4096 * 14336 // 32
    assert bench.gguf_bytes(nblk, 34) == 62_390_272 + 117_440_512   # Q8_0 -> bf16
    assert bench.gguf_bytes(nblk, 18) == 33_030_144 + 117_440_512   # Q4_0 -> bf16
    parts = bench.step_bytes(1 << 29, nblk)
    assert set(parts) == {"quantize", "dequantize", "q8_0", "q4_0"}
    assert parts["quantize"] == parts["dequantize"] == 1_375_731_712
    assert bench.step_bytes(1 << 29, nblk, "q4_0") == {"q4_0": 150_470_656}


def test_percentiles():
    ts = sorted([5.0, 1.0, 4.0, 2.0, 3.0, 9.0, 7.0, 8.0, 6.0, 10.0, 11.0])
    assert bench._pct(ts, 0.0) == 1.0
    assert bench._pct(ts, 0.5) == 6.0
    assert bench._pct(ts, 1.0) == 11.0
    assert bench._pct([3.0], 0.9) == 3.0


def test_reference_arm_json_line():
    """`--impl reference` times the oracle on the host and prints one line
    with the same metric and unit as the GPU arm, its e2e object and its
    cpu_baseline object."""
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["higher_is_better"] is True and d["steps"] == 1 and d["warmup"] == 1
    assert d["value"] > 0
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert cb["sample"]


def test_codebook_option_needs_no_e2e(monkeypatch):
    """The end-to-end path is NF4-only; other tables must be asked for with
    --no-e2e (checked before any device work)."""
    monkeypatch.setattr(sys, "argv", ["bench.py", "--codebook", "dyn8"])
    args = bench.parse_args()
    assert args.codebook == "dyn8" and not args.no_e2e
    with pytest.raises(SystemExit):
        bench.run_ours(args, 0, 1, 0)


class _FakeStep:
    """The attributes bench.verify_step reads, on the CPU, holding outputs
    computed by the oracle itself (so that they are right by construction)."""

    def __init__(self, n, nblk):
        import oracle
        from bq_inputs import codebooks, synth
        self.codebook = "nf4"
        self.n = n
        self.x_cpu, _ = synth.large_outliers(n=n, seed=9, chunk=1 << 14)
        table = codebooks.nf4()
        a, q = oracle.quantize_blockwise(synth.to_numpy_bits(self.x_cpu), "bf16", bench.BS, table)
        y = oracle.dequantize_blockwise(q, a, n, bench.BS, table, "bf16")
        self.q8_cpu = torch.from_numpy(synth.gguf_blocks(nblk, "q8_0", seed=4).reshape(-1))
        self.q4_cpu = torch.from_numpy(synth.gguf_blocks(nblk, "q4_0", seed=5).reshape(-1))
        bf = lambda h: torch.from_numpy(h.view(np.int16)).view(torch.bfloat16)  # noqa: E731
        self.absmax, self.q, self.y = torch.from_numpy(a), torch.from_numpy(q), bf(y)
        self.y8 = bf(oracle.dequant_gguf("q8_0", self.q8_cpu.numpy(), "bf16"))
        self.y4 = bf(oracle.dequant_gguf("q4_0", self.q4_cpu.numpy(), "bf16"))


def test_step_verification_accepts_right_and_rejects_any_flipped_bit():
    """bench.verify_step compares every output bit for bit: the oracle's own
    outputs pass, and one flipped bit in any of them fails the run."""
    names = ["quantize", "dequantize", "q8_0", "q4_0"]
    w = _FakeStep(3 * 8192 + 64 * 5 + 6, 1000)
    summary, expected = bench.verify_step(w, names, 1)
    assert summary["ok"] and summary["values_differing"] == 0
    assert summary["values_compared"] == sum(t.numel() for t in (w.absmax, w.q, w.y, w.y8, w.y4))
    assert set(expected) == {"absmax", "codes", "dequantize", "q8_0", "q4_0"}
    for attr in ("absmax", "q", "y", "y8", "y4"):
        t = getattr(w, attr)
        raw = t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.uint8)
        k = raw.numel() // 3
        raw[k] ^= 1                        # one bit of one value
        with pytest.raises(RuntimeError, match="differ from the oracle"):
            bench.verify_step(w, names, 1)
        raw[k] ^= 1
    # one-kernel profiling runs are not checked
    assert bench.verify_step(w, ["quantize"], 1) == (None, None)


@pytest.mark.parametrize("dtype,name,bs", [("bf16", "nf4", 64), ("f32", "dyn8", 32),
                                           ("f16", "fp4", 256)])
def test_sweep_sample_check_accepts_right_and_rejects_flipped_bits(dtype, name, bs):
    """bench.sample_check (the 1 GiB sweep's check) compares the sampled
    blocks and the tail block with the oracle: the oracle's own outputs pass,
    a flipped bit inside a sampled block or in the tail block is counted, and
    one in a block outside the sample is not."""
    import oracle
    from bq_inputs import codebooks, synth
    n = 40 * bs + 17                    # 40 whole blocks and a tail block
    table = codebooks.get(name)
    x = synth.normal(n, dtype, seed=11)
    xb = synth.to_numpy_bits(x)
    a, q = oracle.quantize_blockwise(xb.view(np.float32) if dtype == "f32" else xb, dtype, bs,
                                     table)
    y = oracle.dequantize_blockwise(q, a, n, bs, table, dtype)
    tdt = synth.TORCH_DTYPES[dtype]
    tt = lambda h: torch.from_numpy(h.view(np.int16 if h.itemsize == 2 else h.dtype)).view(tdt)  # noqa: E731
    xa, at, qt, yt = x.clone(), torch.from_numpy(a), torch.from_numpy(q), tt(y)
    # sample every 4th block (40 // 10), so blocks 0, 4, ..., 36 and the tail
    c, d, nsel = bench.sample_check(xa, at, qt, yt, bs, table, dtype, 10, 2)
    assert d == 0 and nsel == 11
    cb = bs // 2 if table.size == 16 else bs
    assert c == nsel + (10 * cb + (qt.numel() - 40 * cb)) + (10 * bs + 17)
    raw_y = yt.view(torch.int16) if yt.element_size() == 2 else yt.view(torch.int32)
    for flip, counted in ((lambda: raw_y.__setitem__(8 * bs + 3, raw_y[8 * bs + 3] ^ 1), True),
                          (lambda: raw_y.__setitem__(n - 1, raw_y[n - 1] ^ 1), True),
                          (lambda: raw_y.__setitem__(5 * bs + 3, raw_y[5 * bs + 3] ^ 1), False)):
        flip()
        _, d, _ = bench.sample_check(xa, at, qt, yt, bs, table, dtype, 10, 2)
        assert d == (1 if counted else 0)
        flip()
    qt[4 * cb] ^= 1                      # a code byte of sampled block 4
    _, d, _ = bench.sample_check(xa, at, qt, yt, bs, table, dtype, 10, 2)
    assert d >= 1
    qt[4 * cb] ^= 1
    at[36] = at[36] * 2                 # absmax of sampled block 36
    _, d, _ = bench.sample_check(xa, at, qt, yt, bs, table, dtype, 10, 2)
    assert d >= 1
