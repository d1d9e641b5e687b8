#!/usr/bin/env python
"""Benchmark: quantize / dequantize HBM GB/s (input + output bytes) on B200.

One step = the whole hot path over one batch of synthetic input:
  1. blockwise quantize   bf16 n = 2^29 (1 GiB), NF4, blocksize 64
     (N(0, 0.02) with 0.1% outliers from N(0, 0.4))
  2. blockwise dequantize of the result back to bf16
  3. GGUF Q8_0 dequant of a 4096 x 14336 matrix (1,835,008 blocks) to bf16
  4. GGUF Q4_0 dequant of a 4096 x 14336 matrix to bf16
value = (input + output bytes of the four kernels) / device time, in GB/s.
Inputs (1 GiB) are larger than L2 (126 MB), so no flush is needed.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch with torch.distributed.run; every rank runs the same workload
on its own GPU (weak scaling, no collective on the data path).
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bq_inputs import codebooks, synth  # noqa: E402
from dequantization_bq_quantize_b200 import shard  # noqa: E402

METRIC = "quantize/dequantize HBM GB/s (in+out bytes) and % of B200 HBM peak"
N_LARGE = synth.LARGE_N
BS = 64
GGUF_BLOCKS = 4096 * 14336 // 32
WORKLOAD = ("bf16 NF4 blocksize-64 quantize + dequantize of n=2^29 (1 GiB, N(0,0.02) + 0.1% "
            "N(0,0.4) outliers), then GGUF Q8_0 and Q4_0 dequant of a 4096x14336 matrix to bf16")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--n", type=int, default=N_LARGE, help="elements of the quantize input")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the sweep / weight-set / other-codebook figures of the default line")
    ap.add_argument("--only", choices=["all", "quantize", "dequantize", "q8_0", "q4_0"],
                    default="all", help="run one kernel per step (profiling aid)")
    ap.add_argument("--codebook", choices=["nf4", "fp4", "dyn8"], default="nf4",
                    help="table of the step's quantize / dequantize (profiling aid; the benchmark "
                         "line is nf4; other tables need --no-e2e)")
    ap.add_argument("--gguf-kinds", default="",
                    help="gguf workload: comma-separated types to run (e.g. q4_k,q8_0_encode)")
    ap.add_argument("--gguf-sizes", default="small,matrix",
                    help="gguf workload: 'small' (4096 blocks), 'matrix' (4096 x 14336) or both")
    ap.add_argument("--workload", choices=["step", "sweep", "sweep1g", "llama", "gguf", "nested", "h2d"], default="step",
                    help="step: the benchmark line; the others: informational tables")
    return ap.parse_args()


# ------------------------------------------------------------------ bytes --

def quant_bytes(n, bs, elem=2, entries=16):
    """Algorithmic bytes of one quantize (or dequantize) launch: n*elem input
    (output), ceil(n/2) packed 4-bit codes (n 8-bit codes for 256-entry
    tables), 4 bytes of absmax per block."""
    codes = (n + 1) // 2 if entries == 16 else n
    return n * elem + codes + 4 * ((n + bs - 1) // bs)


def gguf_bytes(nblk, block_bytes, out_elem=2):
    return nblk * block_bytes + 32 * nblk * out_elem


def step_bytes(n, nblk, only="all", entries=16):
    parts = {"quantize": quant_bytes(n, BS, entries=entries),
             "dequantize": quant_bytes(n, BS, entries=entries),
             "q8_0": gguf_bytes(nblk, 34), "q4_0": gguf_bytes(nblk, 18)}
    if only != "all":
        return {only: parts[only]}
    return parts


# ----------------------------------------------------------------- clocks --

class ClockSampler:
    """SM clock and throttle reasons sampled with NVML every ~2 ms from a
    thread while the timed region runs (the region is milliseconds long, far
    shorter than nvidia-smi's sampling interval)."""

    REASONS = ("hw_slowdown", "sw_thermal_slowdown", "hw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device):
        self.samples = []
        self.max_mhz = None
        self.error = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self._nvml = pynvml
            self._bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                          "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                          "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                          "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception as e:  # pragma: no cover - no NVML
            self.error = str(e)

    def _run(self):
        nv, h = self._nvml, self._h
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((mhz, reasons))
            except Exception as e:  # pragma: no cover
                self.error = str(e)
                return
            time.sleep(0.002)

    def stop(self):
        self._stop.set()
        if self.error and not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [f"nvml: {self.error}"]}
        self._thread.join(timeout=1)
        mhz = [m for m, _ in self.samples]
        reasons = set()
        for _, r in self.samples:
            for name, bit in self._bits.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(mhz)}


# ------------------------------------------------------------------ peaks --

def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def csrc_digest():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "dequantization_bq_quantize_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, key="dram_bytes_per_launch"):
    """Bytes per launch of `kernel` from the committed ncu summary (DRAM read
    + write by default; key "l2_write_bytes_per_launch" for the bytes the SMs
    wrote to L2), or None when the kernel sources changed since those
    counters were taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
    except Exception:
        return None
    if t.get("csrc_sha") != csrc_digest():
        return None
    v = t.get("kernels", {}).get(kernel, {}).get(key)
    return None if v is None else float(v)


# ---------------------------------------------------------- distributed ----

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    if args.gpus != world and not (world == 1 and args.gpus == 1):
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v, world):
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------- reference ---

def run_reference(args, rank, world):
    """The oracle (plain single-threaded C, driven over disjoint block ranges
    on every host core) on a bounded sample of the same workload."""
    if rank != 0:
        return
    import oracle
    threads = oracle.host_threads()
    n_s = 1 << 25
    nblk_s = 1 << 16
    x, _ = synth.large_outliers(n=n_s)
    xb = synth.to_numpy_bits(x)
    nf4 = codebooks.nf4()
    q8 = synth.gguf_blocks(nblk_s, "q8_0", seed=4)
    q4 = synth.gguf_blocks(nblk_s, "q4_0", seed=5)
    byts = sum(step_bytes(n_s, nblk_s).values())

    def one_step():
        a, q = oracle.quantize_blockwise_threaded(xb, "bf16", BS, nf4, threads)
        oracle.dequantize_blockwise_threaded(q, a, n_s, BS, nf4, "bf16", threads)
        oracle.dequant_q8_0(q8, "bf16")
        oracle.dequant_q4_0(q4, "bf16")

    for _ in range(args.warmup):
        one_step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one_step()
    dt = (time.perf_counter() - t0) / args.steps
    value = byts / dt / 1e9
    sample = (f"per step: quantize+dequantize of the first 2^25 elements of the bf16 workload "
              f"and Q8_0/Q4_0 dequant of 2^16 blocks each; {threads} host threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample_elements": n_s, "sample_gguf_blocks": nblk_s},
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(n, nblk, x_cpu):
    """Oracle timed on the host cores on a bounded sample (~10-30 s of CPU work)."""
    import oracle
    threads = oracle.host_threads()
    n_s = min(n, 1 << 28)
    nblk_s = min(nblk, 1 << 18)
    xb = synth.to_numpy_bits(x_cpu[:n_s])
    nf4 = codebooks.nf4()
    q8 = synth.gguf_blocks(nblk_s, "q8_0", seed=4)
    q4 = synth.gguf_blocks(nblk_s, "q4_0", seed=5)
    t0 = time.perf_counter()
    a, q = oracle.quantize_blockwise_threaded(xb, "bf16", BS, nf4, threads)
    oracle.dequantize_blockwise_threaded(q, a, n_s, BS, nf4, "bf16", threads)
    oracle.dequant_q8_0(q8, "bf16")
    oracle.dequant_q4_0(q4, "bf16")
    dt = time.perf_counter() - t0
    byts = sum(step_bytes(n_s, nblk_s).values())
    # one thread, the plain oracle calls: median of 3 on the first 2^23 elements
    n_1 = min(n_s, 1 << 23)
    t1 = []
    for _ in range(3):
        t = time.perf_counter()
        a1, q1 = oracle.quantize_blockwise(xb[:n_1], "bf16", BS, nf4)
        oracle.dequantize_blockwise(q1, a1, n_1, BS, nf4, "bf16")
        t1.append(time.perf_counter() - t)
    one = 2 * quant_bytes(n_1, BS) / statistics.median(t1) / 1e9
    return {"value": round(byts / dt / 1e9, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "cpu_model": _cpu_model(), "single_thread_gbs": round(one, 3),
            "sample": (f"quantize+dequantize of the first 2^28 elements of the step's bf16 input "
                       f"({threads} threads over disjoint block ranges) and single-threaded "
                       f"Q8_0/Q4_0 dequant of 2^18 blocks each; {dt:.2f} s wall.  "
                       f"single_thread_gbs: quantize+dequantize of 2^23 elements on one "
                       f"thread, median of 3")}


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def _pct(sorted_ts, f):
    """Nearest-rank percentile of an already sorted list."""
    return sorted_ts[min(len(sorted_ts) - 1, int(f * (len(sorted_ts) - 1) + 0.5))]


# ------------------------------------------------------------- checking --

def _raw_bits(a):
    """Bit patterns of a numpy array (so -0 / +0 count as different)."""
    a = np.ascontiguousarray(a)
    return a.view({4: np.uint32, 2: np.uint16, 1: np.uint8}[a.itemsize])


def _host_bits(t):
    t = t.cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        t = t.view(torch.int16)
    return _raw_bits(t.numpy())


def verify_step(w, names, world):
    """Every output of the last timed step against the oracle: absmax, codes
    and the dequantized tensor of the 2^29-element input, and both GGUF
    matrices, bit for bit.  The oracle runs over disjoint block ranges on the
    host threads (blocks are independent, so this is the single call's
    result).  Returns (summary, the oracle's outputs) - (None, None) for the
    one-kernel profiling runs - and raises if any output differs."""
    if names != ["quantize", "dequantize", "q8_0", "q4_0"]:
        return None, None
    import oracle
    threads = max(1, oracle.host_threads() // world)
    t0 = time.perf_counter()
    table = codebooks.get(w.codebook)
    oa, oq = oracle.quantize_blockwise_threaded(synth.to_numpy_bits(w.x_cpu), "bf16", BS, table,
                                                threads)
    expected = {
        "absmax": oa, "codes": oq,
        "dequantize": oracle.dequantize_blockwise_threaded(oq, oa, w.n, BS, table, "bf16",
                                                           threads),
        "q8_0": oracle.dequant_gguf("q8_0", w.q8_cpu.numpy(), "bf16"),
        "q4_0": oracle.dequant_gguf("q4_0", w.q4_cpu.numpy(), "bf16"),
    }
    got = {"absmax": w.absmax, "codes": w.q, "dequantize": w.y, "q8_0": w.y8, "q4_0": w.y4}
    differ, values = {}, 0
    for k, t in got.items():
        g, e = _host_bits(t), _raw_bits(expected[k])
        differ[k] = int(np.count_nonzero(g != e)) if g.shape == e.shape else int(g.size)
        values += g.size
    worst = max_over_ranks(float(sum(differ.values())), world)
    if worst != 0:
        raise RuntimeError(f"bench: outputs of the timed step differ from the oracle: {differ}")
    return {"ok": True, "against": "oracle", "outputs": list(got), "values_compared": values,
            "values_differing": 0, "threads": threads,
            "seconds": round(time.perf_counter() - t0, 2),
            "what": "every output of the last timed step, bit for bit"}, expected


# ---------------------------------------------- figures beyond the step --

def _event_ms(fn, reps=5):
    """Median device time (ms) of fn() over `reps` calls, each bracketed by
    its own CUDA events on the current stream.  For calls of hundreds of
    microseconds or more: event timestamps here advance in steps of about
    2 us."""
    fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        ts.append((e0, e1))
    torch.cuda.synchronize()
    ms = sorted(a.elapsed_time(b) for a, b in ts)
    return ms[len(ms) // 2]


def _flush_graph_ms(flush, reps):
    """Replay time (ms) of a CUDA graph of `reps` reads of the flush buffer."""
    g = _capture(lambda: [flush.sum() for _ in range(reps)])
    ms = _replay_ms(g)
    del g
    return ms


def _flushed_ms(fn, flush, reps, base_ms):
    """Device time (ms) of one fn() call that starts with a cold, clean L2:
    `reps` pairs (read the flush buffer, fn()) captured in one CUDA graph,
    minus `base_ms` (the same number of flush reads alone), divided by reps.
    Reading (not writing) the buffer evicts the inputs and leaves L2 clean, so
    the call pays no write-back of the flush; the graph removes host launch
    gaps, and dividing by reps the event resolution."""
    def both():
        for _ in range(reps):
            flush.sum()
            fn()
    g = _capture(both)
    ms = _replay_ms(g)
    del g
    return max((ms - base_ms) / reps, 0.0)


def _codebook_figures(w, peak):
    """FP4 and dyn8 (256-entry) quantize + dequantize of the step's 1 GiB bf16
    input, blocksize 64 (the input is larger than L2: no flush)."""
    bq = w.bq
    dev = w.x.device
    rows = {}
    q8 = torch.empty(w.n, dtype=torch.uint8, device=dev)
    for name in ("fp4", "dyn8"):
        code = torch.from_numpy(codebooks.get(name)).to(dev)
        q = w.q if code.numel() == 16 else q8
        nbytes = quant_bytes(w.n, BS, entries=code.numel())
        tq = _event_ms(lambda: bq.quantize_blockwise(w.x, code, BS, absmax=w.absmax, out=q))
        td = _event_ms(lambda: bq.dequantize_blockwise(q, w.absmax, w.n, BS, code, out=w.y))
        rows[name] = {"quantize_us": round(tq * 1e3, 1),
                      "quantize_frac": round(nbytes / (tq / 1e3) / 1e9 / peak, 4),
                      "dequantize_us": round(td * 1e3, 1),
                      "dequantize_frac": round(nbytes / (td / 1e3) / 1e9 / peak, 4),
                      "bytes": nbytes}
    del q8
    return rows


def sweep_cells(peak, reps=10):
    """The 45-cell sweep: {fp16, bf16, fp32} x {NF4, FP4, dyn8} x blocksize
    {32, 64, 256, 1024, 4096} at n = 8388608 + 37, N(0, 1) with one all-zero
    block (block nb // 2), drawn on the device from a generator seeded with
    1 + cell.  Quantize, and dequantize to the input dtype, each timed on its
    own after an L2 flush (the cell's tensors fit in L2; _flushed_ms)."""
    import dequantization_bq_quantize_b200 as bq
    dev = torch.device("cuda", torch.cuda.current_device())
    flush = torch.zeros(80 << 20, dtype=torch.int32, device=dev)   # 320 MiB
    base = _flush_graph_ms(flush, reps)
    n = synth.SWEEP_N
    cells = []
    ci = 0
    for dtype in ("f16", "bf16", "f32"):
        for name in ("nf4", "fp4", "dyn8"):
            code = torch.from_numpy(codebooks.get(name)).to(dev)
            for bs in (32, 64, 256, 1024, 4096):
                g = torch.Generator(device=dev)
                g.manual_seed(1 + ci)
                x = torch.randn(n, generator=g, device=dev).to(synth.TORCH_DTYPES[dtype])
                nb = (n + bs - 1) // bs
                x[(nb // 2) * bs: min(n, (nb // 2 + 1) * bs)] = 0
                a, q = bq.quantize_blockwise(x, code, bs)
                y = torch.empty_like(x)
                nbytes = quant_bytes(n, bs, x.element_size(), code.numel())
                tq = _flushed_ms(lambda: bq.quantize_blockwise(x, code, bs, absmax=a, out=q),
                                 flush, reps, base)
                td = _flushed_ms(lambda: bq.dequantize_blockwise(q, a, n, bs, code, out=y),
                                 flush, reps, base)
                cells.append({"dtype": dtype, "codebook": name, "blocksize": bs,
                              "quantize_us": round(tq * 1e3, 1),
                              "quantize_gbs": round(nbytes / (tq / 1e3) / 1e9, 1),
                              "dequantize_us": round(td * 1e3, 1),
                              "dequantize_gbs": round(nbytes / (td / 1e3) / 1e9, 1)})
                ci += 1
    del flush
    fr = lambda k: sorted(c[k] / peak for c in cells)  # noqa: E731
    summary = {k: {"min": round(fr(k)[0], 4), "median": round(fr(k)[len(cells) // 2], 4),
                   "max": round(fr(k)[-1], 4)} for k in ("quantize_gbs", "dequantize_gbs")}
    return cells, summary


SWEEP_1GIB_TAIL = 37


def _block_rows(t, nfull, per_block, sel):
    """Rows `sel` of the first nfull * per_block values of t, viewed as
    nfull rows of per_block, brought to the host as raw bits."""
    return _host_bits(t[: nfull * per_block].view(nfull, per_block)[sel].reshape(-1))


def sample_check(x, a, q, y, bs, table, dtype, sample_blocks, threads):
    """Compare a stratified sample of quantization blocks with the oracle,
    bit for bit: every (nfull // sample_blocks)-th whole block, the block at
    element 2^28 (the sweep's zero block, when the input reaches it) and the
    tail block.  x, a, q, y are the input, absmax, codes and dequantized
    tensors (any device).  Returns (values compared, values differing,
    blocks compared)."""
    import oracle
    n = x.numel()
    e = table.size
    nfull = n // bs
    stride = max(1, nfull // sample_blocks)
    sel = set(range(0, nfull, stride))
    if (1 << 28) // bs < nfull:
        sel.add((1 << 28) // bs)
    sel_t = torch.tensor(sorted(sel), dtype=torch.int64, device=x.device)
    cb = bs // 2 if e == 16 else bs     # code bytes of a whole block
    xs = np.concatenate([_block_rows(x, nfull, bs, sel_t), _host_bits(x[nfull * bs:])])
    got = (np.concatenate([_raw_bits(a[sel_t].cpu().numpy()), _raw_bits(a[nfull:].cpu().numpy())]),
           np.concatenate([_block_rows(q, nfull, cb, sel_t), _host_bits(q[nfull * cb:])]),
           np.concatenate([_block_rows(y, nfull, bs, sel_t), _host_bits(y[nfull * bs:])]))
    xin = xs.view(np.float32) if dtype == "f32" else xs
    oa, oq = oracle.quantize_blockwise_threaded(xin, dtype, bs, table, threads)
    oy = oracle.dequantize_blockwise_threaded(oq, oa, xs.size, bs, table, dtype, threads)
    checked = differing = 0
    for g, exp in zip(got, (oa, oq, oy)):
        exp = _raw_bits(exp)
        checked += exp.size
        differing += int(np.count_nonzero(g != exp)) if g.shape == exp.shape else int(exp.size)
    return checked, differing, len(sel) + (1 if n % bs else 0)


def sweep_1gib(peak, reps=5, sample_blocks=1024):
    """The sweep at 1 GiB: {fp16, bf16, fp32} x {NF4, FP4, dyn8} x blocksize
    {32, 64, 256, 1024, 4096}, each cell on n = 2^30 / element size + 37
    elements (1 GiB of input and a 37-element tail block), N(0, 1) drawn on
    the device from a generator seeded per dtype, with one all-zero block (the
    4096 elements from 2^28 on are zero, a whole block at every blocksize).
    Quantize, and dequantize to the input dtype, each timed with CUDA events
    (median of `reps` calls; the tensors exceed L2, so no flush).  A
    stratified sample of each cell's blocks - every (nfull // sample_blocks)-th
    whole block, the zero block and the tail block (sample_check) - is
    compared bit for bit with the oracle: absmax, codes and dequantized
    values."""
    import dequantization_bq_quantize_b200 as bq
    import oracle
    dev = torch.device("cuda", torch.cuda.current_device())
    threads = oracle.host_threads()
    cells, checked, differing = [], 0, 0
    for di, dtype in enumerate(("f16", "bf16", "f32")):
        tdt = synth.TORCH_DTYPES[dtype]
        es = torch.empty(0, dtype=tdt).element_size()
        n = (1 << 30) // es + SWEEP_1GIB_TAIL
        g = torch.Generator(device=dev)
        g.manual_seed(200 + di)
        x = torch.randn(n, generator=g, device=dev, dtype=torch.float32).to(tdt)
        x[1 << 28: (1 << 28) + 4096] = 0
        y = torch.empty_like(x)
        for name in ("nf4", "fp4", "dyn8"):
            table = codebooks.get(name)
            code = torch.from_numpy(table).to(dev)
            e = code.numel()
            for bs in (32, 64, 256, 1024, 4096):
                nb = (n + bs - 1) // bs
                nfull = n // bs
                a = torch.empty(nb, dtype=torch.float32, device=dev)
                q = torch.empty((n + 1) // 2 if e == 16 else n, dtype=torch.uint8, device=dev)
                nbytes = quant_bytes(n, bs, es, e)
                tq = _event_ms(lambda: bq.quantize_blockwise(x, code, bs, absmax=a, out=q), reps)
                td = _event_ms(lambda: bq.dequantize_blockwise(q, a, n, bs, code, out=y), reps)
                c, d, nsel = sample_check(x, a, q, y, bs, table, dtype, sample_blocks, threads)
                checked += c
                differing += d
                cells.append({"dtype": dtype, "codebook": name, "blocksize": bs, "n": n,
                              "quantize_us": round(tq * 1e3, 1),
                              "quantize_frac": round(nbytes / (tq / 1e3) / 1e9 / peak, 4),
                              "dequantize_us": round(td * 1e3, 1),
                              "dequantize_frac": round(nbytes / (td / 1e3) / 1e9 / peak, 4),
                              "bytes": nbytes, "blocks_checked": nsel})
                del a, q
        del x, y
    if differing:
        raise RuntimeError(f"bench: the 1 GiB sweep differs from the oracle in {differing} of "
                           f"{checked} sampled values")
    fr = lambda k: sorted(c[k] for c in cells)  # noqa: E731
    summary = {k: {"min": fr(k)[0], "median": fr(k)[len(cells) // 2], "max": fr(k)[-1]}
               for k in ("quantize_frac", "dequantize_frac")}
    return {"n": "2^30 / element size + 37", "l2": "inputs larger than L2; no flush",
            "frac_summary": summary,
            "below_0.80": [f"{c['dtype']}/{c['codebook']}/bs{c['blocksize']}/{k[:-5]}"
                           for c in cells for k in ("quantize_frac", "dequantize_frac")
                           if c[k] < 0.80],
            "verified": {"values_compared": checked, "values_differing": differing,
                         "what": "absmax, codes and dequantized values of a stratified sample of "
                                 "blocks per cell (about 1024, the zero block and the tail)"},
            "cells": cells}


def llama_weight_set(steps=3, warmup=1):
    """The 224 weight matrices of a Llama-3-8B-shaped model (32 layers), bf16
    N(0, 0.02) drawn on the device from a generator seeded per matrix; NF4
    blocksize 64 quantize then dequantize of every matrix back to back on one
    stream, eager and as one CUDA-graph replay (the 448 launches captured
    once).  Returns the figures and the total bytes."""
    import dequantization_bq_quantize_b200 as bq
    dev = torch.device("cuda", torch.cuda.current_device())
    code = torch.from_numpy(codebooks.nf4()).to(dev)
    mats, outs = [], []
    total = 0
    for layer, i, name, r, c, seed in synth.llama_matrices():
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        x = torch.randn(r * c, generator=g, device=dev, dtype=torch.float32).mul_(0.02).to(
            torch.bfloat16)
        n = x.numel()
        a = torch.empty((n + BS - 1) // BS, dtype=torch.float32, device=dev)
        q = torch.empty(n // 2, dtype=torch.uint8, device=dev)
        y = torch.empty_like(x)
        mats.append(x)
        outs.append((a, q, y))
        total += 2 * quant_bytes(n, BS)

    def everything():
        for x, (a, q, y) in zip(mats, outs):
            bq.quantize_blockwise(x, code, BS, absmax=a, out=q)
            bq.dequantize_blockwise(q, a, x.numel(), BS, code, out=y)

    for _ in range(max(1, warmup)):
        everything()
    torch.cuda.synchronize()
    ms_eager = _event_ms(everything, max(1, steps))
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            everything()
    torch.cuda.current_stream().wait_stream(side)
    graph.replay()
    torch.cuda.synchronize()
    ms = _event_ms(graph.replay, max(1, steps))
    del graph
    return {"matrices": len(mats), "elements": sum(m.numel() for m in mats), "bytes": total,
            "eager_ms": round(ms_eager, 3), "graph_ms": round(ms, 3),
            "graph_gbs": round(total / (ms / 1e3) / 1e9, 1),
            "eager_gbs": round(total / (ms_eager / 1e3) / 1e9, 1)}


def run_extras(w):
    """Figures beyond the step, reported next to `value` (not part of it):
    the 45-cell sweep at n = 8388645 and at 1 GiB of input per cell, the
    Llama-3-8B-shaped weight set and the 1 GiB quantize / dequantize with the
    FP4 and dyn8 tables, each against the measured copy bandwidth.  The fault word is checked after them."""
    peak, kind = measured_peaks()
    t0 = time.perf_counter()
    other = _codebook_figures(w, peak)
    cells, summary = sweep_cells(peak)
    big = sweep_1gib(peak)
    llama = llama_weight_set()
    llama["graph_frac"] = round(llama["graph_gbs"] / peak, 4)
    llama["eager_frac"] = round(llama["eager_gbs"] / peak, 4)
    fault = w.bq.bq_device_fault(reset=True)
    if fault:
        raise SystemExit(f"bench: the fault word was set during the extra figures ({fault:#x})")
    torch.cuda.empty_cache()
    return {"codebooks_1gib": other,
            "sweep": {"n": synth.SWEEP_N, "l2": "flushed (320 MiB read) before every call",
                      "frac_summary": summary, "cells": cells},
            "sweep_1gib": big,
            "llama_weight_set": llama,
            "extras_peak": f"{peak} GB/s {kind}",
            "extras_seconds": round(time.perf_counter() - t0, 1)}


# -------------------------------------------------------------------- ours --

class Workload:
    def __init__(self, n, rank, device, codebook="nf4"):
        import dequantization_bq_quantize_b200 as bq
        self.bq = bq
        bq.lib()
        self.n = n
        self.nb = (n + BS - 1) // BS
        self.nblk = GGUF_BLOCKS
        x_cpu, self.outliers = synth.large_outliers(n=n, seed=3 + 1000 * rank)
        self.x_cpu = x_cpu
        self.x = x_cpu.to(device)
        self.codebook = codebook
        self.code = torch.from_numpy(codebooks.get(codebook)).to(device)
        self.entries = self.code.numel()
        self.absmax = torch.empty(self.nb, dtype=torch.float32, device=device)
        self.q = torch.empty((n + 1) // 2 if self.entries == 16 else n, dtype=torch.uint8,
                             device=device)
        self.y = torch.empty(n, dtype=torch.bfloat16, device=device)
        q8 = synth.gguf_blocks(self.nblk, "q8_0", seed=4 + 1000 * rank)
        q4 = synth.gguf_blocks(self.nblk, "q4_0", seed=5 + 1000 * rank)
        self.q8_cpu = torch.from_numpy(q8.reshape(-1))
        self.q4_cpu = torch.from_numpy(q4.reshape(-1))
        self.q8 = self.q8_cpu.to(device)
        self.q4 = self.q4_cpu.to(device)
        self.y8 = torch.empty(32 * self.nblk, dtype=torch.bfloat16, device=device)
        self.y4 = torch.empty(32 * self.nblk, dtype=torch.bfloat16, device=device)

    def kernels(self, only):
        bq = self.bq
        names = ["quantize", "dequantize", "q8_0", "q4_0"] if only == "all" else [only]
        return names

    def launch(self, name, stream):
        bq = self.bq
        if name == "quantize":
            st = bq.bq_quantize_blockwise(self.x.data_ptr(), bq.BQ_BF16, self.n, BS,
                                          self.code.data_ptr(), self.entries, self.absmax.data_ptr(),
                                          self.q.data_ptr(), stream)
        elif name == "dequantize":
            st = bq.bq_dequantize_blockwise(self.q.data_ptr(), self.absmax.data_ptr(), self.n, BS,
                                            self.code.data_ptr(), self.entries, self.y.data_ptr(),
                                            bq.BQ_BF16, stream)
        elif name == "q8_0":
            st = bq.bq_dequant_q8_0(self.q8.data_ptr(), self.nblk, self.y8.data_ptr(), bq.BQ_BF16,
                                    stream)
        else:
            st = bq.bq_dequant_q4_0(self.q4.data_ptr(), self.nblk, self.y4.data_ptr(), bq.BQ_BF16,
                                    stream)
        if st != bq.BQ_OK:
            raise RuntimeError(f"{name}: {bq.bq_status_string(st)} {bq.bq_last_cuda_error()}")


def run_ours(args, rank, world, local):
    if args.codebook != "nf4" and not args.no_e2e:
        raise SystemExit("--codebook other than nf4 needs --no-e2e")
    dev = torch.device("cuda", torch.cuda.current_device())
    w = Workload(args.n, rank, dev, args.codebook)
    names = w.kernels(args.only)
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    byts = step_bytes(w.n, w.nblk, args.only, w.entries)
    step_total = sum(byts.values())

    for _ in range(args.warmup):
        for k in names:
            w.launch(k, sh)
    torch.cuda.synchronize()

    # ---- device-resident timed region
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
          for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(dev)
    time.sleep(0.01)
    for s in range(args.steps):
        ev[s][0].record(stream)
        for i, k in enumerate(names):
            w.launch(k, sh)
            ev[s][i + 1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    # a kernel that gave up on a bounded wait returns early and would make the
    # step look faster: such a run gives no result
    fault = w.bq.bq_device_fault(reset=True)
    if max_over_ranks(float(fault), world) != 0:
        raise SystemExit(f"bench: the fault word was set during the timed region ({fault:#x}) "
                         "- a kernel gave up waiting; no result is reported")
    verification, expected = verify_step(w, names, world)
    total_ms = ev[0][0].elapsed_time(ev[-1][-1])
    per_kernel = {k: [ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(args.steps)]
                  for i, k in enumerate(names)}
    max_ms = max_over_ranks(total_ms, world)
    ms_per_step = max_ms / args.steps
    value = shard.aggregate_gbs(step_total, world, ms_per_step)

    # ---- end to end: host buffers in, results back to the host, every step
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, names, stream, sh, byts, world, expected)

    extras = None
    if world == 1 and not args.no_extras and args.only == "all" and args.codebook == "nf4":
        extras = run_extras(w)

    peak, peak_kind = measured_peaks()
    kern = {}
    for k in names:
        ms = statistics.mean(per_kernel[k])
        gbs = byts[k] / (ms / 1e3) / 1e9
        ts = sorted(per_kernel[k])
        kern[k] = {"ms": round(ms, 4), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
                   "bytes": byts[k], "median_ms": round(statistics.median(ts), 4),
                   "p10_ms": round(_pct(ts, 0.1), 4), "p90_ms": round(_pct(ts, 0.9), 4)}
    # the dominant kernel: the one that takes the longest in the step
    dom = max(kern, key=lambda k: kern[k]["ms"])
    cb = w.codebook
    kname = {"quantize": f"quantize_kernel<bf16,{cb},bs64>",
             "dequantize": (f"dequant_stream_kernel<{cb},bf16>" if w.entries == 16
                            else f"dequant_kernel<{cb},bf16>"),
             "q8_0": "gguf_kernel<q8_0,bf16>", "q4_0": "gguf_kernel<q4_0,bf16>"}[dom]
    roof = {"bound": "hbm", "achieved": kern[dom]["gbs"], "peak": peak, "unit": "GB/s",
            "frac": kern[dom]["frac"], "traffic": recorded_traffic(kname),
            "traffic_l2_write": recorded_traffic(kname, "l2_write_bytes_per_launch"),
            "kernel": kname, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(w.n, w.nblk, w.x_cpu)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": WORKLOAD.replace("NF4", w.codebook.upper()), "n": w.n,
                       "blocksize": BS, "codebook": w.codebook,
                       "gguf_blocks": w.nblk, "outliers": w.outliers, "kernels": names,
                       "l2": "inputs larger than L2 (126 MB); no flush",
                       "parallelism": f"dp{world} (independent shards, no collective)"},
            "roofline": roof,
            "kernels": kern,
            "pct_of_nominal_8tbs": {k: round(v["gbs"] / 8000.0, 4) for k, v in kern.items()},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "verified": verification is not None and verification["ok"],
            "verification": verification,
            "gpu_launches": len(names) * args.steps,
            "clocks": clocks,
        }
        if extras:
            line.update(extras)
        print(json.dumps(line), flush=True)


def run_e2e(args, w, names, stream, sh, byts, world, expected, chunks=8):
    """Same step through the public API with host buffers, every step: pinned
    host->device copy of the step's inputs and device->host copy of all its
    results inside the timed region.  The work is cut into `chunks` pieces on
    quantization-block boundaries (blocks are independent, so the results are
    identical) and pipelined over three streams: copies in, kernels, copies
    out, so that PCIe traffic in both directions overlaps the kernels."""
    bq = w.bq
    n, nblk = w.n, w.nblk
    xh = w.x_cpu.pin_memory()
    q8h, q4h = w.q8_cpu.pin_memory(), w.q4_cpu.pin_memory()
    pinned = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)  # noqa: E731
    ah, qh, yh, y8h, y4h = pinned(w.absmax), pinned(w.q), pinned(w.y), pinned(w.y8), pinned(w.y4)
    s_in, s_k, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    # chunk boundaries: whole blocks (and an even element count) per chunk
    per = -(-w.nb // chunks) * BS
    ranges = [(lo, min(n, lo + per)) for lo in range(0, n, per)]
    gper = -(-nblk // chunks)
    granges = [(lo, min(nblk, lo + gper)) for lo in range(0, nblk, gper)]
    h2d = d2h = 0

    # per chunk: the previous step's kernel and copy-out events (buffer reuse)
    prev_k = [None] * len(ranges)
    prev_out = [None] * len(ranges)

    def one():
        nonlocal h2d, d2h
        h2d = d2h = 0
        for ci in range(len(ranges)):
            lo, hi = ranges[ci]
            glo, ghi = granges[ci] if ci < len(granges) else (0, 0)
            b0, b1 = lo // BS, -(-hi // BS)
            e_in = torch.cuda.Event()
            with torch.cuda.stream(s_in):
                if prev_k[ci] is not None:
                    s_in.wait_event(prev_k[ci])  # inputs still read by last step's kernels
                if "quantize" in names:
                    w.x[lo:hi].copy_(xh[lo:hi], non_blocking=True)
                    h2d += (hi - lo) * 2
                if "q8_0" in names and ghi > glo:
                    w.q8[glo * 34:ghi * 34].copy_(q8h[glo * 34:ghi * 34], non_blocking=True)
                    h2d += (ghi - glo) * 34
                if "q4_0" in names and ghi > glo:
                    w.q4[glo * 18:ghi * 18].copy_(q4h[glo * 18:ghi * 18], non_blocking=True)
                    h2d += (ghi - glo) * 18
                e_in.record(s_in)
            e_k = torch.cuda.Event()
            with torch.cuda.stream(s_k):
                s_k.wait_event(e_in)
                if prev_out[ci] is not None:
                    s_k.wait_event(prev_out[ci])  # outputs still copied out by last step
                ks = s_k.cuda_stream
                if "quantize" in names:
                    st = bq.bq_quantize_blockwise(w.x.data_ptr() + 2 * lo, bq.BQ_BF16, hi - lo, BS,
                                                  w.code.data_ptr(), 16,
                                                  w.absmax.data_ptr() + 4 * b0,
                                                  w.q.data_ptr() + lo // 2, ks)
                    assert st == bq.BQ_OK, bq.bq_last_cuda_error()
                if "dequantize" in names:
                    st = bq.bq_dequantize_blockwise(w.q.data_ptr() + lo // 2,
                                                    w.absmax.data_ptr() + 4 * b0, hi - lo, BS,
                                                    w.code.data_ptr(), 16,
                                                    w.y.data_ptr() + 2 * lo, bq.BQ_BF16, ks)
                    assert st == bq.BQ_OK, bq.bq_last_cuda_error()
                if "q8_0" in names and ghi > glo:
                    st = bq.bq_dequant_q8_0(w.q8.data_ptr() + 34 * glo, ghi - glo,
                                            w.y8.data_ptr() + 64 * glo, bq.BQ_BF16, ks)
                    assert st == bq.BQ_OK, bq.bq_last_cuda_error()
                if "q4_0" in names and ghi > glo:
                    st = bq.bq_dequant_q4_0(w.q4.data_ptr() + 18 * glo, ghi - glo,
                                            w.y4.data_ptr() + 64 * glo, bq.BQ_BF16, ks)
                    assert st == bq.BQ_OK, bq.bq_last_cuda_error()
                e_k.record(s_k)
            with torch.cuda.stream(s_out):
                s_out.wait_event(e_k)
                if "quantize" in names:
                    ah[b0:b1].copy_(w.absmax[b0:b1], non_blocking=True)
                    qh[lo // 2:(hi + 1) // 2].copy_(w.q[lo // 2:(hi + 1) // 2], non_blocking=True)
                    d2h += (b1 - b0) * 4 + ((hi + 1) // 2 - lo // 2)
                if "dequantize" in names:
                    yh[lo:hi].copy_(w.y[lo:hi], non_blocking=True)
                    d2h += (hi - lo) * 2
                if "q8_0" in names and ghi > glo:
                    y8h[32 * glo:32 * ghi].copy_(w.y8[32 * glo:32 * ghi], non_blocking=True)
                    d2h += (ghi - glo) * 64
                if "q4_0" in names and ghi > glo:
                    y4h[32 * glo:32 * ghi].copy_(w.y4[32 * glo:32 * ghi], non_blocking=True)
                    d2h += (ghi - glo) * 64
                e_out = torch.cuda.Event()
                e_out.record(s_out)
            prev_k[ci], prev_out[ci] = e_k, e_out

    one()
    torch.cuda.synchronize()
    barrier(world)
    steps = max(1, min(args.steps, 5))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for _ in range(steps):
        one()
    for st_ in (s_in, s_k):
        ev = torch.cuda.Event()
        ev.record(st_)
        s_out.wait_event(ev)
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world) / steps
    # every output the pipelined, chunked calls brought back to the host must
    # equal the oracle's (whole arrays)
    checked = 0
    if expected is not None:
        for key, host in (("absmax", ah), ("codes", qh), ("dequantize", yh), ("q8_0", y8h),
                          ("q4_0", y4h)):
            if key not in expected:
                continue
            if not np.array_equal(_host_bits(host), _raw_bits(expected[key])):
                raise RuntimeError(f"end-to-end {key} differs from the oracle")
            checked += host.numel()
    total = sum(byts.values()) * world
    return {"value": round(total / (ms / 1e3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3),
            "steps": steps, "pipeline": f"{len(ranges)} chunks over 3 streams (in / kernels / out)",
            "outputs_checked_against_oracle": checked}


# ------------------------------------------------------ informational ---

def _capture(body):
    """A CUDA graph of body() captured on a side stream (body() is run once
    first, outside the capture)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        body()
        with torch.cuda.graph(g, stream=side):
            body()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    return g


def _replay_ms(g, times=5):
    """Median device time (ms) of one replay of graph g."""
    ts = []
    for _ in range(times):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    return sorted(ts)[len(ts) // 2]


def _timed(fn, reps, flush=None):
    """Device time (ms) of one fn() call.  Without `flush`: `reps` calls back
    to back between two events, divided by reps.  With `flush` (a buffer
    larger than L2): `reps` pairs (write the flush buffer, fn()) are captured
    in one CUDA graph and `reps` flushes alone in another; the difference of
    their replay times, divided by reps, is fn's time with a cold L2 and
    without host launch gaps."""
    fn()  # warm
    torch.cuda.synchronize()
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    def both():
        for _ in range(reps):
            flush.zero_()
            fn()

    def alone():
        for _ in range(reps):
            flush.zero_()

    g1, g0 = _capture(both), _capture(alone)
    ms = (_replay_ms(g1) - _replay_ms(g0)) / reps
    del g1, g0
    return max(ms, 0.0)


def _graph_timed(fn, reps=50):
    """Device time (ms) of one fn() call, fn launched `reps` times inside one
    CUDA graph and the graph replayed: no host launch overhead, only the
    device's own launch gaps.  For launch-bound calls whose data fit in L2."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        fn()  # warm outside the capture
        with torch.cuda.graph(g, stream=side):
            for _ in range(reps):
                fn()
    torch.cuda.current_stream().wait_stream(side)
    g.replay()
    torch.cuda.synchronize()
    ms = _timed(g.replay, 5)
    del g
    return ms / reps


def run_sweep(args):
    """The 45 sweep cells (sweep_cells), one JSON line."""
    cells, summary = sweep_cells(measured_peaks()[0], reps=max(10, args.steps))
    print(json.dumps({"workload": "sweep", "n": synth.SWEEP_N, "frac_summary": summary,
                      "cells": cells}), flush=True)


def run_sweep1g(args):
    """The 45 sweep cells at 1 GiB of input each (sweep_1gib), one JSON line."""
    torch.cuda.set_device(0)
    res = sweep_1gib(measured_peaks()[0], reps=max(5, args.steps))
    import dequantization_bq_quantize_b200 as bq
    fault = bq.bq_device_fault(reset=True)
    if fault:
        raise SystemExit(f"bench: the fault word was set during the 1 GiB sweep ({fault:#x})")
    print(json.dumps({"workload": "sweep1g", **res}), flush=True)


def run_llama(args):
    """The Llama-3-8B-shaped weight set (llama_weight_set), one JSON line."""
    r = llama_weight_set(steps=max(1, args.steps), warmup=max(1, args.warmup))
    r["frac_of_measured_peak"] = round(r["graph_gbs"] / measured_peaks()[0], 4)
    print(json.dumps(dict({"workload": "llama3-8b-shaped weight set"}, **r)), flush=True)


def run_gguf(args):
    """Every GGUF block type on two workloads, bf16 target: the Verification
    table's 4096 blocks (fits in L2 and is launch-bound: 50 calls captured in
    one CUDA graph, replayed) and a 4096 x 14336 weight matrix (a 320 MiB
    flush precedes each call and its time is subtracted)."""
    import dequantization_bq_quantize_b200 as bq
    dev = torch.device("cuda", torch.cuda.current_device())
    flush = torch.empty(320 << 20, dtype=torch.uint8, device=dev)
    peak = measured_peaks()[0]
    rows = []
    kinds = set(k for k in args.gguf_kinds.split(",") if k)
    sizes = set(args.gguf_sizes.split(","))
    want = lambda k: not kinds or k in kinds
    pick = lambda pairs: [p for p, tag in zip(pairs, ("small", "matrix")) if tag in sizes]
    for kind, (per, bb) in bq.GGUF_TYPES.items():
        if not want(kind):
            continue
        for label, nblk in pick((("4096 blocks", 4096), ("4096x14336", 4096 * 14336 // per))):
            blocks = torch.from_numpy(synth.gguf_blocks(nblk, kind, seed=9).reshape(-1)).to(dev)
            y = torch.empty(nblk * per, dtype=torch.bfloat16, device=dev)
            bq.dequant_gguf(kind, blocks, out=y)
            # the page's 4096 blocks fit in L2 and are launch-bound: timed warm,
            # back to back; the matrix with a flush before each call
            call = lambda: bq.dequant_gguf(kind, blocks, out=y)
            ms = _graph_timed(call) if label == "4096 blocks" else _timed(call, 50, flush)
            nbytes = nblk * bb + 2 * per * nblk  # blocks read + bf16 written
            rows.append({"type": kind, "workload": label, "blocks": nblk, "us": round(ms * 1e3, 2),
                         "gbs": round(nbytes / (ms / 1e3) / 1e9, 1),
                         "frac_of_measured_peak": round(nbytes / (ms / 1e3) / 1e9 / peak, 4)})
            del blocks, y
    # the encoders, bf16 input of the same two sizes
    for kind in bq.GGUF_ENCODERS:
        if not want(kind + "_encode"):
            continue
        bb = bq.GGUF_TYPES[kind][1]
        for label, nblk in pick((("4096 blocks", 4096), ("4096x14336", 4096 * 14336 // 32))):
            g = torch.Generator(device=dev)
            g.manual_seed(17)
            x = torch.randn(nblk * 32, generator=g, device=dev).mul_(0.02).to(torch.bfloat16)
            out = bq.quantize_gguf(kind, x)
            call = lambda: bq.quantize_gguf(kind, x, out=out)
            ms = _graph_timed(call) if label == "4096 blocks" else _timed(call, 50, flush)
            nbytes = nblk * (64 + bb)  # bf16 read + blocks written
            rows.append({"type": kind + " encode", "workload": label, "blocks": nblk,
                         "us": round(ms * 1e3, 2), "gbs": round(nbytes / (ms / 1e3) / 1e9, 1),
                         "frac_of_measured_peak": round(nbytes / (ms / 1e3) / 1e9 / peak, 4)})
            del x, out
    print(json.dumps({"workload": "gguf", "target": "bf16", "rows": rows}), flush=True)


def run_nested(args):
    """Compressed statistics on the step's tensor (bf16 NF4 blocksize 64,
    n = 2^29): the absmax array quantized again with the dynamic 8-bit table
    in blocks of 256, then both dequantized; timed against the plain pair."""
    import dequantization_bq_quantize_b200 as bq
    dev = torch.device("cuda", torch.cuda.current_device())
    n = 1 << 29
    x = synth.large_outliers()[0].to(dev)
    nf4 = torch.from_numpy(codebooks.nf4()).to(dev)
    dyn = torch.from_numpy(codebooks.dynamic8()).to(dev)
    nb = n // BS
    a = torch.empty(nb, dtype=torch.float32, device=dev)
    q = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    a2 = torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev)
    qa = torch.empty(nb, dtype=torch.uint8, device=dev)
    y = torch.empty(n, dtype=torch.bfloat16, device=dev)

    def plain():
        bq.quantize_blockwise(x, nf4, BS, absmax=a, out=q)
        bq.dequantize_blockwise(q, a, n, BS, nf4, out=y)

    def nested():
        bq.quantize_blockwise_nested(x, nf4, BS, dyn, 256, absmax=a, out=q, absmax2=a2,
                                     qabsmax=qa)
        bq.dequantize_blockwise_nested(q, qa, a2, n, BS, nf4, dyn, 256, out=y)

    def nested_parts():
        # the same four kernels timed apart: two quantize passes, the fused
        # dequantization
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record()
        bq.quantize_blockwise(x, nf4, BS, absmax=a, out=q)
        e[1].record()
        bq.quantize_blockwise(a, dyn, 256, absmax=a2, out=qa)
        e[2].record()
        bq.dequantize_blockwise_nested(q, qa, a2, n, BS, nf4, dyn, 256, out=y)
        e[3].record()
        torch.cuda.synchronize()
        return [e[i].elapsed_time(e[i + 1]) for i in range(3)]

    for _ in range(3):
        plain()
        nested()
    torch.cuda.synchronize()
    reps = max(3, args.steps)
    ms_plain = _timed(plain, reps)
    ms_nested = _timed(nested, reps)
    parts = [sorted(x) [len(x) // 2] for x in zip(*[nested_parts() for _ in range(reps)])]
    stats_plain = 4 * nb
    stats_nested = nb + 4 * a2.numel()
    print(json.dumps({"workload": "nested statistics, bf16 NF4 bs64 + dyn8 bs256 on absmax",
                      "n": n, "plain_ms": round(ms_plain, 3), "nested_ms": round(ms_nested, 3),
                      "overhead_pct": round(100 * (ms_nested / ms_plain - 1), 2),
                      "nested_parts_ms": {"quantize": round(parts[0], 4),
                                          "quantize_statistics": round(parts[1], 4),
                                          "dequantize_fused": round(parts[2], 4)},
                      "stat_bytes_plain": stats_plain, "stat_bytes_nested": stats_nested,
                      "bits_per_element_plain": round(4 + 8 * stats_plain / n, 4),
                      "bits_per_element_nested": round(4 + 8 * stats_nested / n, 4)}),
          flush=True)


def run_h2d(args):
    """Host input to quantized device output, bf16 NF4 bs64 with compressed
    statistics (dyn8, blocks of 256), n = 2^28 in pinned host memory: the
    serialized form (copy everything, then quantize on one stream - the
    baseline of the bnb page's two-stream pipeline cells) against the
    two-stream chunked pipeline at several chunk sizes.  GB/s of host input."""
    import dequantization_bq_quantize_b200 as bq
    dev = torch.device("cuda", torch.cuda.current_device())
    n = 1 << 28
    g = torch.Generator().manual_seed(11)
    x = torch.empty(n, dtype=torch.bfloat16).pin_memory()
    for lo in range(0, n, 1 << 24):
        x[lo:lo + (1 << 24)] = torch.randn(1 << 24, generator=g).mul_(0.02).to(torch.bfloat16)
    nf4 = torch.from_numpy(codebooks.nf4()).to(dev)
    dyn = torch.from_numpy(codebooks.dynamic8()).to(dev)
    xd = torch.empty(n, dtype=torch.bfloat16, device=dev)
    nb = n // BS
    a = torch.empty(nb, dtype=torch.float32, device=dev)
    q = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    a2 = torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev)
    qa = torch.empty(nb, dtype=torch.uint8, device=dev)

    def serial():
        xd.copy_(x, non_blocking=True)
        bq.quantize_blockwise_nested(xd, nf4, BS, dyn, 256, absmax=a, out=q, absmax2=a2, qabsmax=qa)

    reps = max(3, args.steps)
    rows = []
    for _ in range(2):
        serial()
    torch.cuda.synchronize()
    ms = _timed(serial, reps)
    rows.append({"form": "serial", "ms": round(ms, 3), "gbs": round(2 * n / (ms / 1e3) / 1e9, 2)})
    ref = (q.clone(), qa.clone(), a2.clone())
    for chunk in (1 << 22, 1 << 23, 1 << 24, 1 << 25):
        staging = torch.empty(2 * chunk * 2, dtype=torch.uint8, device=dev)
        side = torch.cuda.Stream(device=dev)
        cur = torch.cuda.current_stream(dev)

        def piped():
            side.wait_stream(cur)
            st = bq.bq_quantize_blockwise_host(
                x.data_ptr(), bq.BQ_BF16, n, BS, nf4.data_ptr(), 16, dyn.data_ptr(), 256, 256,
                a.data_ptr(), q.data_ptr(), a2.data_ptr(), qa.data_ptr(), staging.data_ptr(),
                staging.numel(), chunk, cur.cuda_stream, side.cuda_stream)
            assert st == bq.BQ_OK

        q.zero_()
        piped()
        torch.cuda.synchronize()
        same = bool(torch.equal(q, ref[0]) and torch.equal(qa, ref[1]) and torch.equal(a2, ref[2]))
        ms = _timed(piped, reps)
        rows.append({"form": "two-stream pipeline", "chunk_elements": chunk, "ms": round(ms, 3),
                     "gbs": round(2 * n / (ms / 1e3) / 1e9, 2), "identical_to_serial": same})
    print(json.dumps({"workload": "h2d + nested NF4 quantize, bf16 n=2^28 pinned", "rows": rows}),
          flush=True)


def main():
    args = parse_args()
    rank, world, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        elif args.workload == "sweep":
            run_sweep(args)
        elif args.workload == "sweep1g":
            run_sweep1g(args)
        elif args.workload == "llama":
            run_llama(args)
        elif args.workload == "gguf":
            run_gguf(args)
        elif args.workload == "nested":
            run_nested(args)
        elif args.workload == "h2d":
            run_h2d(args)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
