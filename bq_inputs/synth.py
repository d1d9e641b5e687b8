"""Seeded synthetic inputs for the quantize / dequantize workloads.

This module holds no arithmetic of the method: it only draws random numbers
(``torch.Generator('cpu')``, so the bytes are the same on every machine with
the same torch build) and lays them out in the input formats.  The same host
bytes feed the CUDA path and the oracle.

Workloads (shapes and value distributions of the sizes the method targets):
  * small:   fp32 N(0,1), n = 65536                       (NF4, blocksize 64)
  * sweep:   N(0,1) at n = 8388608 + 37 in fp16/bf16/fp32, one all-zero block
  * large:   bf16 N(0, 0.02), n = 2^29, 0.1% outliers drawn from N(0, 0.4)
  * gguf:    Q8_0 / Q4_0 blocks, qs bytes uniform in 0..255,
             d = fp16(|N(0,1)| * 0.01)
  * llama:   the 7 matrix shapes of one Llama-3-8B layer, 32 layers, bf16 N(0, 0.02)
"""
import numpy as np
import torch

TORCH_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}

SWEEP_N = 8388608 + 37
LARGE_N = 1 << 29
SMALL_N = 65536

# (name, rows, cols) of the weight matrices of one Llama-3-8B layer
LLAMA3_8B_LAYER = [
    ("q", 4096, 4096),
    ("k", 1024, 4096),
    ("v", 1024, 4096),
    ("o", 4096, 4096),
    ("gate", 14336, 4096),
    ("up", 14336, 4096),
    ("down", 4096, 14336),
]
LLAMA3_8B_LAYERS = 32


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal(n, dtype, seed, std=1.0):
    """n samples of N(0, std^2) drawn in fp32, rounded to ``dtype`` (nearest-even)."""
    x = torch.randn(n, generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(TORCH_DTYPES[dtype])


def with_zero_block(x, blocksize):
    """Return x with block number nb//2 (of blocksize elements) set to zero."""
    n = x.numel()
    nb = (n + blocksize - 1) // blocksize
    b = nb // 2
    x = x.clone()
    x[b * blocksize: min(n, (b + 1) * blocksize)] = 0
    return x


def sweep(dtype, blocksize, seed, n=SWEEP_N):
    """Sweep workload: N(0,1) with one all-zero block (block nb//2)."""
    return with_zero_block(normal(n, dtype, seed), blocksize)


def large_outliers(n=LARGE_N, seed=3, std=0.02, outlier_std=0.4, rate=0.001,
                   chunk=1 << 24):
    """bf16 N(0, std^2) with a Bernoulli(rate) share of elements replaced by
    N(0, outlier_std^2) samples.  Drawn chunk by chunk from one generator:
    per chunk the base samples, then the mask draws, then the outliers.
    Returns (bf16 tensor, number of outliers)."""
    g = _gen(seed)
    out = torch.empty(n, dtype=torch.bfloat16)
    count = 0
    for lo in range(0, n, chunk):
        m = min(chunk, n - lo)
        base = torch.randn(m, generator=g, dtype=torch.float32).mul_(std)
        mask = torch.rand(m, generator=g, dtype=torch.float32) < rate
        k = int(mask.sum())
        base[mask] = torch.randn(k, generator=g, dtype=torch.float32).mul_(outlier_std)
        out[lo:lo + m] = base.to(torch.bfloat16)
        count += k
    return out, count


# GGUF block types: bytes per block and the byte offsets of the fp16 fields
# (scale d, min m, super-block dmin) as (offset, signed).  Format facts only.
GGUF_LAYOUT = {
    "q8_0": (34, ((0, False),)),
    "q4_0": (18, ((0, False),)),
    "q4_1": (20, ((0, False), (2, True))),
    "q5_0": (22, ((0, False),)),
    "q5_1": (24, ((0, False), (2, True))),
    "q2_k": (84, ((80, False), (82, False))),
    "q3_k": (110, ((108, False),)),
    "q4_k": (144, ((0, False), (2, False))),
    "q5_k": (176, ((0, False), (2, False))),
    "q6_k": (210, ((208, False),)),
}


def gguf_blocks(n_blocks, kind, seed=4):
    """GGUF blocks of `kind` as a uint8 numpy array [n_blocks, block_bytes]
    ("bf16": n_blocks single values of 2 bytes, N(0, 0.02)).

    Each fp16 field is |N(0,1)| * 0.01 (a signed N(0,1) * 0.01 for a min
    field), stored little-endian at its offset; every other byte (quant bytes,
    high-bit words, packed sub-block scales) is uniform on 0..255."""
    if kind == "bf16":
        # plain bfloat16 weights, N(0, 0.02): [n_blocks, 2] little-endian bytes
        g = _gen(seed)
        v = torch.randn(n_blocks, generator=g).mul_(0.02).to(torch.bfloat16)
        return v.view(torch.int16).numpy().view(np.uint8).reshape(n_blocks, 2).copy()
    bb, fields = GGUF_LAYOUT[kind]
    g = _gen(seed)
    vals = []
    for _, signed in fields:
        d = torch.randn(n_blocks, generator=g, dtype=torch.float32)
        if not signed:
            d.abs_()
        vals.append(d.mul_(0.01).to(torch.float16).numpy().view(np.uint16))
    rest = bb - 2 * len(fields)
    qs = torch.randint(0, 256, (n_blocks, rest), generator=g, dtype=torch.uint8).numpy()
    blocks = np.empty((n_blocks, bb), np.uint8)
    free = np.ones(bb, bool)
    for (off, _), h in zip(fields, vals):
        blocks[:, off] = (h & 0xFF).astype(np.uint8)
        blocks[:, off + 1] = (h >> 8).astype(np.uint8)
        free[off:off + 2] = False
    blocks[:, free] = qs
    return blocks


def llama_matrices(layers=LLAMA3_8B_LAYERS):
    """(layer, index, name, rows, cols, seed) for every matrix of the weight set."""
    out = []
    for layer in range(layers):
        for i, (name, r, c) in enumerate(LLAMA3_8B_LAYER):
            out.append((layer, i, name, r, c, 5000 + 7 * layer + i))
    return out


def to_numpy_bits(t):
    """CPU tensor -> numpy array in the oracle's convention (bf16/f16 as uint16 bits)."""
    t = t.contiguous()
    if t.dtype == torch.float32:
        return t.numpy()
    return t.view(torch.int16).numpy().view(np.uint16)
