"""Helpers shared by the GPU tests: device buffers with guard bands, host
copies in the oracle's conventions, sampled-block oracle checks."""
import numpy as np
import torch

import oracle
from bq_inputs import synth

GUARD = 4096          # bytes of sentinel before and after every output buffer
SENTINEL = 0xA5


class Guarded:
    """A device byte buffer with sentinel guard bands on both sides."""

    def __init__(self, nbytes, offset=0):
        self.nbytes = nbytes
        self.offset = offset
        self.raw = torch.full((GUARD + offset + nbytes + GUARD,), SENTINEL, dtype=torch.uint8,
                              device="cuda")

    @property
    def ptr(self):
        return self.raw.data_ptr() + GUARD + self.offset

    def body(self):
        return self.raw[GUARD + self.offset: GUARD + self.offset + self.nbytes]

    def host(self):
        return self.body().cpu().numpy()

    def guards_intact(self):
        r = self.raw.cpu().numpy()
        lo = r[:GUARD + self.offset]
        hi = r[GUARD + self.offset + self.nbytes:]
        return bool((lo == SENTINEL).all() and (hi == SENTINEL).all())


def device_copy(host_bytes, offset=0):
    """Copy a numpy array's bytes to a device buffer starting `offset` bytes
    past a 256-byte aligned base; returns (keepalive tensor, pointer)."""
    b = np.ascontiguousarray(host_bytes).view(np.uint8).reshape(-1)
    t = torch.zeros(b.size + offset + 16, dtype=torch.uint8, device="cuda")
    t[offset: offset + b.size] = torch.from_numpy(b).cuda()
    return t, t.data_ptr() + offset


def np_bits(t):
    return synth.to_numpy_bits(t.cpu())


def oracle_blocks(x_np, dtype, bs, table, blocks):
    """Oracle absmax / codes for selected whole blocks of x (block indices)."""
    n = x_np.size
    res = {}
    for b in blocks:
        lo, hi = b * bs, min(n, (b + 1) * bs)
        res[b] = oracle.quantize_blockwise(x_np[lo:hi], dtype, bs, table)
    return res


def sample_blocks(nb, count, seed, extra=()):
    rng = np.random.default_rng(seed)
    pick = set(int(v) for v in rng.integers(0, nb, size=min(count, nb)))
    pick |= {0, nb - 1, nb // 2}
    pick |= set(b for b in extra if 0 <= b < nb)
    return sorted(pick)
