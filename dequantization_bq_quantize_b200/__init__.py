"""Blockwise codebook quantization / dequantization (plain and with compressed
statistics), GGUF block dequantization (Q8_0, Q4_0, Q4_1, Q5_0, Q5_1, Q2_K,
Q3_K, Q4_K, Q5_K, Q6_K, BF16), GGUF Q8_0 / Q4_0 encoding, and a two-stream
host-input quantization pipeline, on NVIDIA B200 (sm_100a).

A thin ctypes binding over ``libbq.so`` (C ABI in ``include/bq.h``).  Every
step of the computation runs in the library's CUDA kernels; this module only
marshals arguments.  torch is used for device memory and streams.  There is no
CPU fallback: if ``libbq.so`` is missing, every call raises.

Raw ABI functions keep the C names (``bq_quantize_blockwise`` ...) and take
integer device addresses.  The torch helpers (``quantize_blockwise`` ...) take
CUDA tensors, allocate missing outputs with torch, and launch on the current
torch stream unless a stream is given.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbq.so")

BQ_OK, BQ_ERR_INVALID_ARG, BQ_ERR_UNSUPPORTED, BQ_ERR_CUDA = 0, 1, 2, 3
BQ_F32, BQ_F16, BQ_BF16 = 0, 1, 2
BQ_NOALLOC_MAX_BLOCKS = 1 << 20  # bq_quantize_blockwise_nested_noalloc's limit

# GGUF block types: (outputs per block, bytes per block)
# ("bf16": plain bfloat16 values, one per 2-byte "block")
GGUF_TYPES = {"q8_0": (32, 34), "q4_0": (32, 18), "q4_1": (32, 20), "q5_0": (32, 22),
              "q5_1": (32, 24), "q2_k": (256, 84), "q3_k": (256, 110), "q4_k": (256, 144),
              "q5_k": (256, 176), "q6_k": (256, 210), "bf16": (1, 2)}

GGUF_ENCODERS = ("q8_0", "q4_0")

EXPORTED = (
    "bq_quantize_blockwise", "bq_dequantize_blockwise", "bq_quantize_blockwise_nested",
    "bq_quantize_blockwise_nested_noalloc", "bq_dequantize_blockwise_nested",
    "bq_quantize_blockwise_host",
) + tuple("bq_dequant_" + k for k in GGUF_TYPES) + tuple(
    "bq_quantize_" + k for k in GGUF_ENCODERS) + (
    "bq_status_string", "bq_last_cuda_error", "bq_device_fault", "bq_abi_version",
)

_lib = None


class BQError(RuntimeError):
    """A bq entry point returned a status other than BQ_OK."""

    def __init__(self, fn, status, detail):
        self.status = status
        super().__init__(f"{fn}: {detail}")


def lib():
    """The loaded libbq.so.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m dequantization_bq_quantize_b200._build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        L.bq_quantize_blockwise.argtypes = [vp, i32, i64, i32, vp, i32, vp, vp, vp]
        L.bq_dequantize_blockwise.argtypes = [vp, vp, i64, i32, vp, i32, vp, i32, vp]
        for k in GGUF_TYPES:
            getattr(L, "bq_dequant_" + k).argtypes = [vp, i64, vp, i32, vp]
            getattr(L, "bq_dequant_" + k).restype = ctypes.c_int
        for k in GGUF_ENCODERS:
            getattr(L, "bq_quantize_" + k).argtypes = [vp, i32, i64, vp, vp]
            getattr(L, "bq_quantize_" + k).restype = ctypes.c_int
        L.bq_quantize_blockwise_nested.argtypes = [vp, i32, i64, i32, vp, i32, vp, i32, i32, vp,
                                                   vp, vp, vp, vp]
        L.bq_quantize_blockwise_nested_noalloc.argtypes = [vp, i32, i64, i32, vp, i32, vp, i32,
                                                           i32, vp, vp, vp, vp]
        L.bq_dequantize_blockwise_nested.argtypes = [vp, vp, vp, i64, i32, vp, i32, vp, i32, i32,
                                                     vp, i32, vp]
        L.bq_quantize_blockwise_host.argtypes = [vp, i32, i64, i32, vp, i32, vp, i32, i32, vp, vp,
                                                 vp, vp, vp, i64, i64, vp, vp]
        for f in ("bq_quantize_blockwise", "bq_dequantize_blockwise", "bq_device_fault",
                  "bq_quantize_blockwise_nested", "bq_dequantize_blockwise_nested",
                  "bq_quantize_blockwise_nested_noalloc", "bq_quantize_blockwise_host"):
            getattr(L, f).restype = ctypes.c_int
        L.bq_status_string.argtypes = [ctypes.c_int]
        L.bq_status_string.restype = ctypes.c_char_p
        L.bq_last_cuda_error.argtypes = []
        L.bq_last_cuda_error.restype = ctypes.c_char_p
        L.bq_device_fault.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int32]
        L.bq_abi_version.argtypes = []
        L.bq_abi_version.restype = ctypes.c_int32
        _lib = L
    return _lib


def build(force=False):
    """Compile libbq.so in-tree (nvcc, sm_100a)."""
    from . import _build
    return _build.build(force=force)


# ------------------------------------------------------------ raw C ABI ----

def bq_quantize_blockwise(x, x_dtype, n, blocksize, code, code_entries, absmax, out, stream):
    return lib().bq_quantize_blockwise(x, x_dtype, n, blocksize, code, code_entries, absmax, out,
                                       stream)


def bq_dequantize_blockwise(q, absmax, n, blocksize, code, code_entries, y, y_dtype, stream):
    return lib().bq_dequantize_blockwise(q, absmax, n, blocksize, code, code_entries, y, y_dtype,
                                         stream)


def bq_quantize_blockwise_nested(x, x_dtype, n, blocksize, code, code_entries, code2,
                                 code2_entries, blocksize2, absmax, out, absmax2, qabsmax, stream):
    return lib().bq_quantize_blockwise_nested(x, x_dtype, n, blocksize, code, code_entries, code2,
                                              code2_entries, blocksize2, absmax, out, absmax2,
                                              qabsmax, stream)


def bq_quantize_blockwise_nested_noalloc(x, x_dtype, n, blocksize, code, code_entries, code2,
                                         code2_entries, blocksize2, out, absmax2, qabsmax,
                                         stream):
    return lib().bq_quantize_blockwise_nested_noalloc(x, x_dtype, n, blocksize, code,
                                                      code_entries, code2, code2_entries,
                                                      blocksize2, out, absmax2, qabsmax, stream)


def bq_dequantize_blockwise_nested(q, qabsmax, absmax2, n, blocksize, code, code_entries, code2,
                                   code2_entries, blocksize2, y, y_dtype, stream):
    return lib().bq_dequantize_blockwise_nested(q, qabsmax, absmax2, n, blocksize, code,
                                                code_entries, code2, code2_entries, blocksize2, y,
                                                y_dtype, stream)


def bq_quantize_blockwise_host(x_host, x_dtype, n, blocksize, code, code_entries, code2,
                               code2_entries, blocksize2, absmax, out, absmax2, qabsmax, staging,
                               staging_bytes, chunk_elements, stream0, stream1):
    return lib().bq_quantize_blockwise_host(x_host, x_dtype, n, blocksize, code, code_entries,
                                            code2, code2_entries, blocksize2, absmax, out,
                                            absmax2, qabsmax, staging, staging_bytes,
                                            chunk_elements, stream0, stream1)


def bq_dequant_q8_0(blocks, n_blocks, y, y_dtype, stream):
    return lib().bq_dequant_q8_0(blocks, n_blocks, y, y_dtype, stream)


def bq_dequant_q4_0(blocks, n_blocks, y, y_dtype, stream):
    return lib().bq_dequant_q4_0(blocks, n_blocks, y, y_dtype, stream)


def bq_dequant_q4_1(blocks, n_blocks, y, y_dtype, stream):
    return lib().bq_dequant_q4_1(blocks, n_blocks, y, y_dtype, stream)


def bq_dequant_q5_0(blocks, n_blocks, y, y_dtype, stream):
    return lib().bq_dequant_q5_0(blocks, n_blocks, y, y_dtype, stream)


def bq_dequant_q5_1(blocks, n_blocks, y, y_dtype, stream):
    return lib().bq_dequant_q5_1(blocks, n_blocks, y, y_dtype, stream)


def bq_dequant_q4_k(blocks, n_blocks, y, y_dtype, stream):
    return lib().bq_dequant_q4_k(blocks, n_blocks, y, y_dtype, stream)


def bq_dequant_q6_k(blocks, n_blocks, y, y_dtype, stream):
    return lib().bq_dequant_q6_k(blocks, n_blocks, y, y_dtype, stream)


def bq_quantize_q8_0(x, x_dtype, n, blocks, stream):
    return lib().bq_quantize_q8_0(x, x_dtype, n, blocks, stream)


def bq_quantize_q4_0(x, x_dtype, n, blocks, stream):
    return lib().bq_quantize_q4_0(x, x_dtype, n, blocks, stream)


def bq_dequant_q2_k(blocks, n_blocks, y, y_dtype, stream):
    return lib().bq_dequant_q2_k(blocks, n_blocks, y, y_dtype, stream)


def bq_dequant_q3_k(blocks, n_blocks, y, y_dtype, stream):
    return lib().bq_dequant_q3_k(blocks, n_blocks, y, y_dtype, stream)


def bq_dequant_q5_k(blocks, n_blocks, y, y_dtype, stream):
    return lib().bq_dequant_q5_k(blocks, n_blocks, y, y_dtype, stream)


def bq_dequant_bf16(x, n, y, y_dtype, stream):
    return lib().bq_dequant_bf16(x, n, y, y_dtype, stream)


def bq_status_string(status):
    return lib().bq_status_string(status).decode()


def bq_last_cuda_error():
    return lib().bq_last_cuda_error().decode()


def bq_device_fault(reset=True):
    """Read (and by default clear) the device fault word; synchronizes."""
    v = ctypes.c_uint32(0)
    _check("bq_device_fault", lib().bq_device_fault(ctypes.byref(v), 1 if reset else 0))
    return v.value


def bq_abi_version():
    return lib().bq_abi_version()


def _check(fn, status):
    if status != BQ_OK:
        detail = bq_status_string(status)
        extra = bq_last_cuda_error()
        raise BQError(fn, status, f"{detail} ({extra})" if extra else detail)


def _check_fault(fn):
    """Read and clear the device fault word (this synchronizes the device);
    raise if a kernel gave up on a bounded wait, which leaves its outputs
    invalid."""
    f = bq_device_fault(reset=True)
    if f:
        raise BQError(fn, BQ_ERR_CUDA,
                      f"a kernel gave up waiting (device fault word {f:#x}); outputs are invalid")


# --------------------------------------------------------- torch helpers ----
#
# Every helper takes check=False.  With check=True it synchronizes after the
# launch and raises BQError if a kernel gave up on one of its bounded waits
# (the launch itself succeeded, so nothing else would report it).

def _torch():
    import torch
    return torch


def _dtype_code(dt):
    torch = _torch()
    return {torch.float32: BQ_F32, torch.float16: BQ_F16, torch.bfloat16: BQ_BF16}[dt]


def _stream_handle(stream):
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _need_cuda(t, name):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def code_bytes(n, entries):
    """Bytes of packed codes for n elements (two per byte for 16 entries)."""
    return (n + 1) // 2 if entries == 16 else n


def quantize_blockwise(x, code, blocksize, absmax=None, out=None, stream=None, check=False):
    """Quantize the CUDA tensor x (fp32/fp16/bf16, any shape, flattened).

    code: CUDA float32 tensor of 16 or 256 sorted entries.
    Returns (absmax float32[ceil(n/blocksize)], packed codes uint8)."""
    torch = _torch()
    _need_cuda(x, "x")
    _need_cuda(code, "code")
    n = x.numel()
    entries = code.numel()
    nb = (n + blocksize - 1) // blocksize
    if absmax is None:
        absmax = torch.empty(nb, dtype=torch.float32, device=x.device)
    if out is None:
        out = torch.empty(code_bytes(n, entries), dtype=torch.uint8, device=x.device)
    _check("bq_quantize_blockwise", bq_quantize_blockwise(
        x.data_ptr(), _dtype_code(x.dtype), n, blocksize, code.data_ptr(), entries,
        absmax.data_ptr(), out.data_ptr(), _stream_handle(stream)))
    if check:
        _check_fault("bq_quantize_blockwise")
    return absmax, out


def dequantize_blockwise(q, absmax, n, blocksize, code, dtype=None, out=None, stream=None,
                         check=False):
    """Inverse of quantize_blockwise: n values of ``dtype`` (default bf16)."""
    torch = _torch()
    _need_cuda(q, "q")
    _need_cuda(absmax, "absmax")
    _need_cuda(code, "code")
    if out is None:
        out = torch.empty(n, dtype=dtype or torch.bfloat16, device=q.device)
    _check("bq_dequantize_blockwise", bq_dequantize_blockwise(
        q.data_ptr(), absmax.data_ptr(), n, blocksize, code.data_ptr(), code.numel(),
        out.data_ptr(), _dtype_code(out.dtype), _stream_handle(stream)))
    if check:
        _check_fault("bq_dequantize_blockwise")
    return out


def dequant_gguf(kind, blocks, dtype=None, out=None, stream=None, check=False):
    """GGUF blocks of type ``kind`` (a key of GGUF_TYPES; uint8 CUDA tensor of
    n_blocks * block bytes) -> outputs-per-block * n_blocks values of ``dtype``
    (default bf16)."""
    torch = _torch()
    _need_cuda(blocks, "blocks")
    per, bbytes = GGUF_TYPES[kind]
    if blocks.numel() % bbytes:
        raise ValueError(f"{kind}: {blocks.numel()} bytes is not a whole number of "
                         f"{bbytes}-byte blocks")
    nblk = blocks.numel() // bbytes
    if out is None:
        out = torch.empty(per * nblk, dtype=dtype or torch.bfloat16, device=blocks.device)
    fn = globals()["bq_dequant_" + kind]
    _check(fn.__name__, fn(blocks.data_ptr(), nblk, out.data_ptr(), _dtype_code(out.dtype),
                           _stream_handle(stream)))
    if check:
        _check_fault(fn.__name__)
    return out


def dequant_q8_0(blocks, dtype=None, out=None, stream=None):
    """GGUF Q8_0 blocks (uint8 CUDA tensor of n_blocks*34 bytes) -> 32*n_blocks values."""
    return dequant_gguf("q8_0", blocks, dtype, out, stream)


def dequant_q4_0(blocks, dtype=None, out=None, stream=None):
    """GGUF Q4_0 blocks (uint8 CUDA tensor of n_blocks*18 bytes) -> 32*n_blocks values."""
    return dequant_gguf("q4_0", blocks, dtype, out, stream)


def dequant_q4_1(blocks, dtype=None, out=None, stream=None):
    """GGUF Q4_1 blocks (n_blocks*20 bytes) -> 32*n_blocks values."""
    return dequant_gguf("q4_1", blocks, dtype, out, stream)


def dequant_q5_0(blocks, dtype=None, out=None, stream=None):
    """GGUF Q5_0 blocks (n_blocks*22 bytes) -> 32*n_blocks values."""
    return dequant_gguf("q5_0", blocks, dtype, out, stream)


def dequant_q5_1(blocks, dtype=None, out=None, stream=None):
    """GGUF Q5_1 blocks (n_blocks*24 bytes) -> 32*n_blocks values."""
    return dequant_gguf("q5_1", blocks, dtype, out, stream)


def dequant_q2_k(blocks, dtype=None, out=None, stream=None):
    """GGUF Q2_K super-blocks (n_blocks*84 bytes) -> 256*n_blocks values."""
    return dequant_gguf("q2_k", blocks, dtype, out, stream)


def dequant_q3_k(blocks, dtype=None, out=None, stream=None):
    """GGUF Q3_K super-blocks (n_blocks*110 bytes) -> 256*n_blocks values."""
    return dequant_gguf("q3_k", blocks, dtype, out, stream)


def dequant_q5_k(blocks, dtype=None, out=None, stream=None):
    """GGUF Q5_K super-blocks (n_blocks*176 bytes) -> 256*n_blocks values."""
    return dequant_gguf("q5_k", blocks, dtype, out, stream)


def dequant_bf16(values, dtype=None, out=None, stream=None):
    """GGUF BF16 tensor data (uint8 CUDA tensor of 2*n bytes) -> n values."""
    return dequant_gguf("bf16", values, dtype, out, stream)


def dequant_q4_k(blocks, dtype=None, out=None, stream=None):
    """GGUF Q4_K super-blocks (n_blocks*144 bytes) -> 256*n_blocks values."""
    return dequant_gguf("q4_k", blocks, dtype, out, stream)


def dequant_q6_k(blocks, dtype=None, out=None, stream=None):
    """GGUF Q6_K super-blocks (n_blocks*210 bytes) -> 256*n_blocks values."""
    return dequant_gguf("q6_k", blocks, dtype, out, stream)


def quantize_gguf(kind, x, out=None, stream=None, check=False):
    """Encode the CUDA tensor x (fp32/fp16/bf16, numel a multiple of 32) as
    GGUF ``kind`` blocks ("q8_0" or "q4_0"): a uint8 tensor of
    numel/32 * block bytes."""
    torch = _torch()
    _need_cuda(x, "x")
    if kind not in GGUF_ENCODERS:
        raise ValueError(f"no encoder for {kind}")
    n = x.numel()
    if n % 32:
        raise ValueError(f"{n} elements is not a whole number of 32-element blocks")
    bbytes = GGUF_TYPES[kind][1]
    if out is None:
        out = torch.empty(n // 32 * bbytes, dtype=torch.uint8, device=x.device)
    fn = globals()["bq_quantize_" + kind]
    _check(fn.__name__, fn(x.data_ptr(), _dtype_code(x.dtype), n, out.data_ptr(),
                           _stream_handle(stream)))
    if check:
        _check_fault(fn.__name__)
    return out


# -------------------------------------------------- compressed statistics ----

def quantize_blockwise_nested(x, code, blocksize, code2, blocksize2=256, absmax=None, out=None,
                              absmax2=None, qabsmax=None, stream=None, check=False):
    """Blockwise quantization with compressed statistics: the fp32 absmax array
    of the first pass is itself quantized blockwise with `code2` (the 256-entry
    dynamic 8-bit table) in blocks of `blocksize2`.  Returns (codes, absmax
    codes, absmax2, absmax), absmax being the first pass's fp32 statistics."""
    torch = _torch()
    _need_cuda(x, "x")
    _need_cuda(code, "code")
    _need_cuda(code2, "code2")
    n = x.numel()
    nb = (n + blocksize - 1) // blocksize
    dev = x.device
    if absmax is None:
        absmax = torch.empty(nb, dtype=torch.float32, device=dev)
    if out is None:
        out = torch.empty(code_bytes(n, code.numel()), dtype=torch.uint8, device=dev)
    if absmax2 is None:
        absmax2 = torch.empty((nb + blocksize2 - 1) // blocksize2, dtype=torch.float32, device=dev)
    if qabsmax is None:
        qabsmax = torch.empty(nb, dtype=torch.uint8, device=dev)
    _check("bq_quantize_blockwise_nested", bq_quantize_blockwise_nested(
        x.data_ptr(), _dtype_code(x.dtype), n, blocksize, code.data_ptr(), code.numel(),
        code2.data_ptr(), code2.numel(), blocksize2, absmax.data_ptr(), out.data_ptr(),
        absmax2.data_ptr(), qabsmax.data_ptr(), _stream_handle(stream)))
    if check:
        _check_fault("bq_quantize_blockwise_nested")
    return out, qabsmax, absmax2, absmax


def dequantize_blockwise_nested(q, qabsmax, absmax2, n, blocksize, code, code2, blocksize2=256,
                                dtype=None, out=None, stream=None, check=False):
    """Inverse of quantize_blockwise_nested in one launch: each block's scale
    is rebuilt from its code and the second-level scale inside the kernel."""
    torch = _torch()
    for t, name in ((q, "q"), (qabsmax, "qabsmax"), (absmax2, "absmax2"), (code, "code"),
                    (code2, "code2")):
        _need_cuda(t, name)
    if out is None:
        out = torch.empty(n, dtype=dtype or torch.bfloat16, device=q.device)
    _check("bq_dequantize_blockwise_nested", bq_dequantize_blockwise_nested(
        q.data_ptr(), qabsmax.data_ptr(), absmax2.data_ptr(), n, blocksize, code.data_ptr(),
        code.numel(), code2.data_ptr(), code2.numel(), blocksize2, out.data_ptr(),
        _dtype_code(out.dtype), _stream_handle(stream)))
    if check:
        _check_fault("bq_dequantize_blockwise_nested")
    return out


# ------------------------------------------------------ host-input pipeline ----

_side_streams = {}


def quantize_blockwise_host(x_host, code, blocksize, code2=None, blocksize2=256,
                            chunk_elements=1 << 24, staging=None, device=None, check=False):
    """Quantize a CPU tensor (pin it for overlap) straight into device outputs,
    copying and quantizing chunk by chunk over two streams: torch's current
    stream and a side stream, joined back into the current stream.  Returns
    (absmax, codes) or, with code2, (codes, absmax codes, absmax2, absmax)
    like quantize_blockwise_nested."""
    torch = _torch()
    if x_host.is_cuda or not x_host.is_contiguous():
        raise ValueError("x_host must be a contiguous CPU tensor")
    dev = torch.device(device) if device is not None else torch.device(
        "cuda", torch.cuda.current_device())
    n = x_host.numel()
    nb = (n + blocksize - 1) // blocksize
    eb = x_host.element_size()
    absmax = torch.empty(nb, dtype=torch.float32, device=dev)
    out = torch.empty(code_bytes(n, code.numel()), dtype=torch.uint8, device=dev)
    absmax2 = qabsmax = None
    if code2 is not None:
        absmax2 = torch.empty((nb + blocksize2 - 1) // blocksize2, dtype=torch.float32, device=dev)
        qabsmax = torch.empty(nb, dtype=torch.uint8, device=dev)
    chunks = max(1, (n + chunk_elements - 1) // chunk_elements)
    need = 2 * chunk_elements * eb if chunks > 1 else max(n, 1) * eb
    if staging is None:
        staging = torch.empty(need, dtype=torch.uint8, device=dev)
    cur = torch.cuda.current_stream(dev)
    side = _side_streams.get(dev.index)
    if side is None:
        side = _side_streams[dev.index] = torch.cuda.Stream(device=dev)
    _check("bq_quantize_blockwise_host", bq_quantize_blockwise_host(
        x_host.data_ptr(), _dtype_code(x_host.dtype), n, blocksize, code.data_ptr(), code.numel(),
        code2.data_ptr() if code2 is not None else None, 256, blocksize2, absmax.data_ptr(),
        out.data_ptr(), absmax2.data_ptr() if absmax2 is not None else None,
        qabsmax.data_ptr() if qabsmax is not None else None, staging.data_ptr(),
        staging.numel(), chunk_elements, cur.cuda_stream, side.cuda_stream))
    if check:
        _check_fault("bq_quantize_blockwise_host")
    if code2 is None:
        return absmax, out
    return out, qabsmax, absmax2, absmax
