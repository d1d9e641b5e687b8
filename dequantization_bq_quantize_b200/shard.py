"""Splitting the work across GPUs (one process per GPU).

Quantization blocks and GGUF blocks are independent, so the path shards with
no exchange: each rank takes a contiguous range of whole blocks and calls the
library on its range with pointer offsets; the shards' absmax, codes and
outputs concatenate by offset.  A collective is only needed to gather results
somewhere, never to compute them.
"""


def block_ranges(n, blocksize, world):
    """Element ranges [lo, hi) per rank: contiguous, every boundary on a
    quantization-block boundary (so also on an even element, as the 4-bit
    packing needs), sizes as equal as whole blocks allow."""
    if n < 0 or world < 1 or blocksize < 2 or blocksize % 2:
        raise ValueError("bad shard request")
    nb = (n + blocksize - 1) // blocksize
    out = []
    for r in range(world):
        b0 = nb * r // world
        b1 = nb * (r + 1) // world
        out.append((min(n, b0 * blocksize), min(n, b1 * blocksize)))
    return out


def shard_offsets(lo, hi, blocksize, code_entries):
    """Offsets of a shard [lo, hi) into the whole tensor's outputs: first
    absmax index, absmax count, first code byte, code byte count."""
    if lo % blocksize:
        raise ValueError("a shard must start on a block boundary")
    a0 = lo // blocksize
    na = (hi - lo + blocksize - 1) // blocksize
    if code_entries == 16:
        return a0, na, lo // 2, (hi - lo + 1) // 2
    return a0, na, lo, hi - lo


def gguf_ranges(n_blocks, world):
    """GGUF block ranges [b0, b1) per rank."""
    if n_blocks < 0 or world < 1:
        raise ValueError("bad shard request")
    return [(n_blocks * r // world, n_blocks * (r + 1) // world) for r in range(world)]


def aggregate_gbs(step_bytes_per_rank, world, max_ms_per_step):
    """Whole-job throughput: bytes moved by all ranks over the slowest rank's
    time per step."""
    return step_bytes_per_rank * world / (max_ms_per_step / 1e3) / 1e9
