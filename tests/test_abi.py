"""The C-ABI library: it loads, exports every symbol include/bq.h declares,
and validates arguments on the host before any CUDA call (so these run
without a GPU)."""
import ctypes
import os
import re

import pytest

import dequantization_bq_quantize_b200 as bq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "bq.h")).read()
    return re.findall(r"BQ_API\s+[\w\s\*]+?\b(bq_\w+)\s*\(", text)


@pytest.fixture(scope="module")
def L():
    bq.build()
    return bq.lib()


def test_header_declares_the_compute_calls():
    syms = declared_symbols()
    for name in ("bq_quantize_blockwise", "bq_dequantize_blockwise", "bq_dequant_q8_0",
                 "bq_dequant_q4_0", "bq_dequant_q4_1", "bq_dequant_q5_0", "bq_dequant_q5_1",
                 "bq_dequant_q4_k", "bq_dequant_q6_k", "bq_quantize_q8_0", "bq_quantize_q4_0",
                 "bq_dequant_q2_k", "bq_dequant_q3_k", "bq_dequant_q5_k", "bq_dequant_bf16",
                 "bq_quantize_blockwise_nested", "bq_dequantize_blockwise_nested",
                 "bq_quantize_blockwise_host"):
        assert name in syms


def test_every_declared_symbol_is_exported(L):
    syms = declared_symbols()
    assert len(syms) >= 22
    assert set(syms) == set(bq.EXPORTED)
    for name in syms:
        assert hasattr(L, name), name
        assert name in bq.EXPORTED


def test_abi_version_and_status_strings(L):
    assert bq.bq_abi_version() == 1
    assert bq.bq_status_string(bq.BQ_OK) == "ok"
    assert bq.bq_status_string(bq.BQ_ERR_INVALID_ARG) == "invalid argument"
    assert bq.bq_status_string(bq.BQ_ERR_CUDA) == "CUDA error"
    assert bq.bq_status_string(99) == "unknown status"


P = 0x10000  # a fake, 64 KiB-aligned device address: never dereferenced here


@pytest.mark.parametrize("bs", [0, 16, 48, 8192, -64, 100])
def test_rejects_bad_blocksize(L, bs):
    assert bq.bq_quantize_blockwise(P, bq.BQ_BF16, 100, bs, P, 16, P, P, 0) == bq.BQ_ERR_INVALID_ARG
    assert bq.bq_dequantize_blockwise(P, P, 100, bs, P, 16, P, bq.BQ_BF16, 0) == bq.BQ_ERR_INVALID_ARG


@pytest.mark.parametrize("entries", [0, 8, 15, 17, 255, 512])
def test_rejects_bad_codebook_length(L, entries):
    assert bq.bq_quantize_blockwise(P, bq.BQ_F32, 100, 64, P, entries, P, P, 0) == bq.BQ_ERR_INVALID_ARG


def test_rejects_bad_sizes_pointers_dtypes(L):
    E = bq.BQ_ERR_INVALID_ARG
    assert bq.bq_quantize_blockwise(P, bq.BQ_F32, -1, 64, P, 16, P, P, 0) == E
    assert bq.bq_quantize_blockwise(P, 7, 100, 64, P, 16, P, P, 0) == E
    assert bq.bq_quantize_blockwise(0, bq.BQ_F32, 100, 64, P, 16, P, P, 0) == E
    assert bq.bq_quantize_blockwise(P, bq.BQ_F32, 100, 64, 0, 16, P, P, 0) == E
    assert bq.bq_quantize_blockwise(P, bq.BQ_F32, 100, 64, P, 16, 0, P, 0) == E
    assert bq.bq_quantize_blockwise(P, bq.BQ_F32, 100, 64, P, 16, P, 0, 0) == E
    # element misaligned for its type
    assert bq.bq_quantize_blockwise(P + 2, bq.BQ_F32, 100, 64, P, 16, P, P, 0) == E
    assert bq.bq_quantize_blockwise(P + 1, bq.BQ_BF16, 100, 64, P, 16, P, P, 0) == E
    assert bq.bq_quantize_blockwise(P, bq.BQ_BF16, 100, 64, P, 16, P + 2, P, 0) == E
    assert bq.bq_dequantize_blockwise(P, P, 100, 64, P, 16, P + 1, bq.BQ_F16, 0) == E
    assert bq.bq_dequantize_blockwise(0, P, 100, 64, P, 16, P, bq.BQ_F16, 0) == E
    assert bq.bq_dequant_q8_0(P, -1, P, bq.BQ_BF16, 0) == E
    assert bq.bq_dequant_q4_0(0, 10, P, bq.BQ_BF16, 0) == E
    assert bq.bq_dequant_q4_0(P, 10, P + 1, bq.BQ_BF16, 0) == E
    assert bq.bq_dequant_q4_0(P, 10, P, 9, 0) == E
    assert bq.bq_dequant_bf16(P + 1, 10, P, bq.BQ_F32, 0) == E       # x not 2-byte aligned
    for kind in bq.GGUF_TYPES:
        fn = getattr(bq, "bq_dequant_" + kind)
        assert fn(P, -1, P, bq.BQ_BF16, 0) == E, kind
        assert fn(0, 10, P, bq.BQ_BF16, 0) == E, kind
        assert fn(P, 10, 0, bq.BQ_BF16, 0) == E, kind
        assert fn(P, 10, P + 1, bq.BQ_F16, 0) == E, kind
        assert fn(P, 10, P + 2, bq.BQ_F32, 0) == E, kind
        assert fn(P, 10, P, 3, 0) == E, kind
        assert fn(P, 1 << 57, P, bq.BQ_BF16, 0) == E, kind
    for kind in bq.GGUF_ENCODERS:
        fn = getattr(bq, "bq_quantize_" + kind)
        assert fn(P, bq.BQ_BF16, -32, P, 0) == E, kind
        assert fn(P, bq.BQ_BF16, 33, P, 0) == E, kind       # not whole blocks
        assert fn(P, bq.BQ_BF16, 48, P, 0) == E, kind
        assert fn(0, bq.BQ_BF16, 64, P, 0) == E, kind
        assert fn(P, bq.BQ_BF16, 64, 0, 0) == E, kind
        assert fn(P + 1, bq.BQ_BF16, 64, P, 0) == E, kind
        assert fn(P + 2, bq.BQ_F32, 64, P, 0) == E, kind
        assert fn(P, 5, 64, P, 0) == E, kind
        assert fn(P, bq.BQ_F32, 1 << 51, P, 0) == E, kind


def test_nested_and_host_pipeline_reject_bad_arguments(L):
    E = bq.BQ_ERR_INVALID_ARG
    B = bq.BQ_BF16
    q_n = bq.bq_quantize_blockwise_nested
    assert q_n(P, B, 4096, 64, P, 16, P, 16, 256, P, P, P, P, 0) == E      # code2 not 256 entries
    assert q_n(P, B, 4096, 64, P, 16, P, 256, 100, P, P, P, P, 0) == E     # blocksize2
    assert q_n(P, B, 4096, 64, P, 16, P, 256, 8192, P, P, P, P, 0) == E
    assert q_n(P, B, 4096, 64, P, 16, 0, 256, 256, P, P, P, P, 0) == E     # null code2
    assert q_n(P, B, 4096, 64, P, 16, P, 256, 256, P, P, 0, P, 0) == E     # null absmax2
    assert q_n(P, B, 4096, 64, P, 16, P, 256, 256, P, P, P, 0, 0) == E     # null qabsmax
    assert q_n(P, B, 4096, 64, P, 16, P + 2, 256, 256, P, P, P, P, 0) == E
    d_n = bq.bq_dequantize_blockwise_nested
    assert d_n(P, P, P, 4096, 64, P, 16, P, 16, 256, P, B, 0) == E
    assert d_n(P, P, P, 4096, 64, P, 16, P, 256, 48, P, B, 0) == E
    assert d_n(P, 0, P, 4096, 64, P, 16, P, 256, 256, P, B, 0) == E
    assert d_n(P, P, 0, 4096, 64, P, 16, P, 256, 256, P, B, 0) == E
    assert d_n(P, P, P, 4096, 64, P, 16, P, 256, 256, P + 1, B, 0) == E
    assert d_n(P, P, P, -1, 64, P, 16, P, 256, 256, P, B, 0) == E
    h = bq.bq_quantize_blockwise_host
    # chunk not whole blocks / not whole second-level blocks / not positive
    assert h(P, B, 4096, 64, P, 16, None, 0, 0, P, P, None, None, P, 1 << 20, 100, 0, 0) == E
    assert h(P, B, 4096, 64, P, 16, P, 256, 256, P, P, P, P, P, 1 << 20, 64 * 100, 0, 0) == E
    assert h(P, B, 4096, 64, P, 16, None, 0, 0, P, P, None, None, P, 1 << 20, 0, 0, 0) == E
    # staging too small for two chunks, or misaligned
    assert h(P, B, 1 << 20, 64, P, 16, None, 0, 0, P, P, None, None, P, 4096, 4096, 0, 0) == E
    assert h(P, B, 4096, 64, P, 16, None, 0, 0, P, P, None, None, P + 8, 1 << 20, 64, 0, 0) == E
    # null host input, misaligned host input, null outputs
    assert h(0, B, 4096, 64, P, 16, None, 0, 0, P, P, None, None, P, 1 << 20, 64, 0, 0) == E
    assert h(P + 1, B, 4096, 64, P, 16, None, 0, 0, P, P, None, None, P, 1 << 20, 64, 0, 0) == E
    assert h(P, B, 4096, 64, P, 16, None, 0, 0, 0, P, None, None, P, 1 << 20, 64, 0, 0) == E
    # nested without its outputs
    assert h(P, B, 4096, 64, P, 16, P, 256, 256, P, P, None, P, P, 1 << 20, 64 * 256, 0, 0) == E
    # n == 0 is fine with no buffers at all
    assert h(0, B, 0, 64, 0, 16, None, 0, 0, 0, 0, None, None, 0, 0, 64, 0, 0) == bq.BQ_OK


def test_zero_length_is_ok_without_touching_the_device(L):
    # n == 0 returns before any CUDA call, even with null buffers
    assert bq.bq_quantize_blockwise(0, bq.BQ_F32, 0, 64, 0, 16, 0, 0, 0) == bq.BQ_OK
    assert bq.bq_dequantize_blockwise(0, 0, 0, 64, 0, 256, 0, bq.BQ_BF16, 0) == bq.BQ_OK
    assert bq.bq_dequant_q8_0(0, 0, 0, bq.BQ_BF16, 0) == bq.BQ_OK
    assert bq.bq_dequant_q4_0(0, 0, 0, bq.BQ_F32, 0) == bq.BQ_OK
    for kind in bq.GGUF_TYPES:
        assert getattr(bq, "bq_dequant_" + kind)(0, 0, 0, bq.BQ_BF16, 0) == bq.BQ_OK, kind
    for kind in bq.GGUF_ENCODERS:
        assert getattr(bq, "bq_quantize_" + kind)(0, bq.BQ_BF16, 0, 0, 0) == bq.BQ_OK, kind


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(bq, "_lib", None)
    monkeypatch.setattr(bq, "LIB_PATH", str(tmp_path / "libbq.so"))
    with pytest.raises(ImportError):
        bq.lib()


def test_library_has_no_oracle_dependency(L):
    # the product library links neither the oracle nor anything under tests/
    out = os.popen(f"ldd {bq.LIB_PATH} 2>/dev/null").read()
    assert "oracle" not in out
    src = open(os.path.join(ROOT, "dequantization_bq_quantize_b200", "__init__.py")).read()
    assert "import oracle" not in src and "from oracle" not in src


def test_noalloc_entry_rejects_sizes_beyond_its_array(L):
    """The allocation-free nested quantize refuses inputs with more blocks
    than its fixed statistics array before touching the device."""
    E = bq.BQ_ERR_INVALID_ARG
    too_many = (bq.BQ_NOALLOC_MAX_BLOCKS + 1) * 64
    assert bq.bq_quantize_blockwise_nested_noalloc(P, bq.BQ_BF16, too_many, 64, P, 16, P, 256,
                                                   256, P, P, P, 0) == E
    assert "BQ_NOALLOC_MAX_BLOCKS" in bq.bq_last_cuda_error()
    assert bq.bq_quantize_blockwise_nested_noalloc(P, bq.BQ_BF16, 0, 64, P, 16, P, 256, 256, P, P,
                                                   P, 0) == bq.BQ_OK
    assert bq.bq_quantize_blockwise_nested_noalloc(P, bq.BQ_BF16, 100, 64, P, 16, P, 16, 256, P, P,
                                                   P, 0) == E
