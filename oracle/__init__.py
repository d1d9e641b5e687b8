"""CPU oracle for blockwise codebook quantization and GGUF block dequantization.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never calls it, and it shares no code with the CUDA library: this module is a
ctypes wrapper around ``bq_oracle.c``, a plain single-threaded C transcription
of the definitions (see the header comment of ``bq_oracle.h`` for the pages and
sections it follows).

Arrays are numpy arrays.  bfloat16 data is carried as ``uint16`` bit patterns,
float16 as ``float16`` or ``uint16`` bit patterns, float32 as ``float32``.
"""
import ctypes
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from . import build as _build

DTYPES = {"f32": 0, "f16": 1, "bf16": 2}

# GGUF block types: (elements per block, bytes per block)
GGUF_TYPES = {"q8_0": (32, 34), "q4_0": (32, 18), "q4_1": (32, 20), "q5_0": (32, 22),
              "q5_1": (32, 24), "q2_k": (256, 84), "q3_k": (256, 110), "q4_k": (256, 144),
              "q5_k": (256, 176), "q6_k": (256, 210), "bf16": (1, 2)}
_ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2}

_lib = None


def lib():
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = _declare(ctypes.CDLL(path))
    return _lib


def _declare(L):
    c_void_p, c_int, c_int64, c_float = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    L.bqo_f16_to_f32.argtypes = [ctypes.c_uint16]
    L.bqo_f16_to_f32.restype = c_float
    L.bqo_bf16_to_f32.argtypes = [ctypes.c_uint16]
    L.bqo_bf16_to_f32.restype = c_float
    L.bqo_f32_to_f16.argtypes = [c_float]
    L.bqo_f32_to_f16.restype = ctypes.c_uint16
    L.bqo_f32_to_bf16.argtypes = [c_float]
    L.bqo_f32_to_bf16.restype = ctypes.c_uint16
    L.bqo_nearest_code.argtypes = [c_float, c_void_p, c_int]
    L.bqo_nearest_code.restype = c_int
    L.bqo_quantize_blockwise.argtypes = [c_void_p, c_int, c_int64, c_int, c_void_p, c_int, c_void_p, c_void_p]
    L.bqo_quantize_blockwise.restype = c_int
    L.bqo_dequantize_blockwise.argtypes = [c_void_p, c_void_p, c_int64, c_int, c_void_p, c_int, c_void_p, c_int]
    L.bqo_dequantize_blockwise.restype = c_int
    L.bqo_dequant_q8_0.argtypes = [c_void_p, c_int64, c_void_p, c_int]
    L.bqo_dequant_q8_0.restype = c_int
    L.bqo_dequant_q4_0.argtypes = [c_void_p, c_int64, c_void_p, c_int]
    L.bqo_dequant_q4_0.restype = c_int
    for kind in ("q8_0", "q4_0"):
        f = getattr(L, "bqo_quantize_" + kind)
        f.argtypes = [c_void_p, c_int, c_int64, c_void_p]
        f.restype = c_int
    for kind in GGUF_TYPES:
        f = getattr(L, "bqo_dequant_" + kind)
        f.argtypes = [c_void_p, c_int64, c_void_p, c_int]
        f.restype = c_int
    return L


def load_library(path):
    """Load another build of the oracle source (used by the mutation tests)."""
    return _declare(ctypes.CDLL(path))


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def _as_bits(x, dtype):
    x = np.ascontiguousarray(x)
    if dtype == "f32":
        return x.astype(np.float32, copy=False)
    if dtype == "f16" and x.dtype == np.float16:
        return x.view(np.uint16)
    if x.dtype != np.uint16:
        raise TypeError(f"{dtype} input must be uint16 bit patterns (got {x.dtype})")
    return x


def _out_array(n, dtype):
    if dtype == "f32":
        return np.empty(n, np.float32)
    return np.empty(n, np.uint16)


def code_bytes(n, entries):
    """Bytes of packed codes for n elements."""
    return (n + 1) // 2 if entries == 16 else n


def quantize_blockwise(x, dtype, blocksize, code, L=None):
    """Return (absmax float32[nb], codes uint8[...]) for the 1-D input x."""
    L = L or lib()
    xb = _as_bits(x, dtype).reshape(-1)
    code = np.ascontiguousarray(code, dtype=np.float32)
    n = xb.size
    nb = (n + blocksize - 1) // blocksize
    absmax = np.empty(nb, np.float32)
    out = np.empty(code_bytes(n, code.size), np.uint8)
    rc = L.bqo_quantize_blockwise(_ptr(xb), DTYPES[dtype], n, blocksize, _ptr(code), code.size,
                                  _ptr(absmax), _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return absmax, out


def dequantize_blockwise(q, absmax, n, blocksize, code, ydtype, L=None):
    """Return y (float32, or uint16 bit patterns for f16/bf16) of n elements."""
    L = L or lib()
    q = np.ascontiguousarray(q, dtype=np.uint8)
    absmax = np.ascontiguousarray(absmax, dtype=np.float32)
    code = np.ascontiguousarray(code, dtype=np.float32)
    y = _out_array(n, ydtype)
    rc = L.bqo_dequantize_blockwise(_ptr(q), _ptr(absmax), n, blocksize, _ptr(code), code.size,
                                    _ptr(y), DTYPES[ydtype])
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return y


def dequant_q8_0(blocks, ydtype, L=None):
    L = L or lib()
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8).reshape(-1)
    nblk = blocks.size // 34
    y = _out_array(32 * nblk, ydtype)
    if L.bqo_dequant_q8_0(_ptr(blocks), nblk, _ptr(y), DTYPES[ydtype]) != 0:
        raise ValueError("oracle rejected the arguments")
    return y


def dequant_q4_0(blocks, ydtype, L=None):
    L = L or lib()
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8).reshape(-1)
    nblk = blocks.size // 18
    y = _out_array(32 * nblk, ydtype)
    if L.bqo_dequant_q4_0(_ptr(blocks), nblk, _ptr(y), DTYPES[ydtype]) != 0:
        raise ValueError("oracle rejected the arguments")
    return y


def dequant_gguf(kind, blocks, ydtype, L=None):
    """Dequantize GGUF blocks of type `kind` (a key of GGUF_TYPES)."""
    L = L or lib()
    per, bb = GGUF_TYPES[kind]
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8).reshape(-1)
    nblk = blocks.size // bb
    y = _out_array(per * nblk, ydtype)
    if getattr(L, "bqo_dequant_" + kind)(_ptr(blocks), nblk, _ptr(y), DTYPES[ydtype]) != 0:
        raise ValueError("oracle rejected the arguments")
    return y


def quantize_gguf(kind, x, dtype, L=None):
    """Encode x (n a multiple of 32) as GGUF Q8_0 or Q4_0 blocks
    (uint8 array [n / 32, block bytes])."""
    L = L or lib()
    per, bb = GGUF_TYPES[kind]
    xb = _as_bits(x, dtype).reshape(-1)
    out = np.empty((xb.size // 32, bb), np.uint8)
    if getattr(L, "bqo_quantize_" + kind)(_ptr(xb), DTYPES[dtype], xb.size, _ptr(out)) != 0:
        raise ValueError("oracle rejected the arguments")
    return out


def nearest_code(xn, code, L=None):
    L = L or lib()
    code = np.ascontiguousarray(code, dtype=np.float32)
    return L.bqo_nearest_code(float(np.float32(xn)), _ptr(code), code.size)


def f16_to_f32(h):
    return np.array([lib().bqo_f16_to_f32(int(v)) for v in np.asarray(h).reshape(-1)], np.float32)


def bf16_to_f32(h):
    return np.array([lib().bqo_bf16_to_f32(int(v)) for v in np.asarray(h).reshape(-1)], np.float32)


def f32_to_f16(f):
    return np.array([lib().bqo_f32_to_f16(float(v)) for v in np.asarray(f, np.float32).reshape(-1)],
                    np.uint16)


def f32_to_bf16(f):
    return np.array([lib().bqo_f32_to_bf16(float(v)) for v in np.asarray(f, np.float32).reshape(-1)],
                    np.uint16)


# ------------------------------------------------------------------ driving --

def quantize_blockwise_threaded(x, dtype, blocksize, code, threads):
    """Run the single-threaded oracle over disjoint block ranges on ``threads``
    host threads (ctypes releases the GIL during each call).  Blocks are
    independent, so the result equals one single-threaded call; the oracle's
    own arithmetic is untouched.  Used only to time the CPU baseline."""
    L = lib()
    xb = _as_bits(x, dtype).reshape(-1)
    code = np.ascontiguousarray(code, dtype=np.float32)
    n = xb.size
    nb = (n + blocksize - 1) // blocksize
    absmax = np.empty(nb, np.float32)
    out = np.empty(code_bytes(n, code.size), np.uint8)
    eb = _ELEM_BYTES[dtype]
    per = (nb + threads - 1) // threads

    def run(t):
        b0, b1 = t * per, min(nb, (t + 1) * per)
        if b0 >= b1:
            return 0
        e0, e1 = b0 * blocksize, min(n, b1 * blocksize)
        o0 = e0 // 2 if code.size == 16 else e0
        return L.bqo_quantize_blockwise(
            ctypes.c_void_p(xb.ctypes.data + e0 * eb), DTYPES[dtype], e1 - e0, blocksize,
            _ptr(code), code.size, ctypes.c_void_p(absmax.ctypes.data + 4 * b0),
            ctypes.c_void_p(out.ctypes.data + o0))

    with ThreadPoolExecutor(threads) as ex:
        rcs = list(ex.map(run, range(threads)))
    if any(rcs):
        raise ValueError("oracle rejected the arguments")
    return absmax, out


def dequantize_blockwise_threaded(q, absmax, n, blocksize, code, ydtype, threads):
    """Dequantize over disjoint block ranges on ``threads`` host threads."""
    L = lib()
    q = np.ascontiguousarray(q, dtype=np.uint8)
    absmax = np.ascontiguousarray(absmax, dtype=np.float32)
    code = np.ascontiguousarray(code, dtype=np.float32)
    y = _out_array(n, ydtype)
    yb = y.itemsize
    nb = (n + blocksize - 1) // blocksize
    per = (nb + threads - 1) // threads

    def run(t):
        b0, b1 = t * per, min(nb, (t + 1) * per)
        if b0 >= b1:
            return 0
        e0, e1 = b0 * blocksize, min(n, b1 * blocksize)
        o0 = e0 // 2 if code.size == 16 else e0
        return L.bqo_dequantize_blockwise(
            ctypes.c_void_p(q.ctypes.data + o0), ctypes.c_void_p(absmax.ctypes.data + 4 * b0),
            e1 - e0, blocksize, _ptr(code), code.size,
            ctypes.c_void_p(y.ctypes.data + e0 * yb), DTYPES[ydtype])

    with ThreadPoolExecutor(threads) as ex:
        rcs = list(ex.map(run, range(threads)))
    if any(rcs):
        raise ValueError("oracle rejected the arguments")
    return y


def host_threads():
    """Threads the CPU baseline may use: the cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1
