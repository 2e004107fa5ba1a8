"""The C ABI on the host (CPU only): the library loads, exports every symbol the
header declares, validates its arguments, and its host-side byte arithmetic
agrees with the pages' numbers and with the oracle."""
import ctypes
import os
import re

import pytest

import oracle as O
from decode_attention_kivi_b200 import _native as N
from decode_attention_kivi_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return N.lib()


def _header_functions(header="kivi.h"):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kivi_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = _header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n


def test_debug_library_exports_its_header():
    """libkivi_debug.so exports the regular ABI plus the debug header's hook; the
    regular library does not carry the hook."""
    dbg = ctypes.CDLL(B.build(debug=True))
    for n in _header_functions() + _header_functions("kivi_debug.h"):
        assert hasattr(dbg, n), n
    assert _header_functions("kivi_debug.h") == ["kivi_debug_overstate_copies"]
    assert not hasattr(ctypes.CDLL(B.build()), "kivi_debug_overstate_copies")


def cfg(**kw):
    base = dict(batch=16, num_layers=32, num_kv_heads=8, num_q_heads=32, head_dim=128, bits=2,
                group_size=32, residual=128, max_tokens=8192 + 64)
    base.update(kw)
    return N.KiviConfig(*[base[f] for f, _ in N.KiviConfig._fields_])


def test_required_bytes_layout(lib):
    s = N.KiviSizes()
    c = cfg()
    assert lib.kivi_required_bytes(ctypes.byref(c), ctypes.byref(s)) == 0
    ngcap = O.num_groups(c.max_tokens)
    assert s.records_bytes == 32 * 16 * 8 * ngcap * 3072
    assert s.resid_k_bytes == s.resid_v_bytes == 32 * 16 * 8 * 160 * 128 * 2
    # status header, one ticket per (sequence, kv head) rounded to 256 bytes, and two
    # (m, l, acc) partials of the 4 query heads of a kv head per CTA, for 256 CTAs
    pairs = 16 * 8
    tickets = (4 * pairs + 255) // 256 * 256
    # then the prompt lengths of ragged layers, [32 layers][16 sequences] int32
    lens = (32 * 16 * 4 + 255) // 256 * 256
    assert s.workspace_bytes == 256 + tickets + 256 * 2 * 4 * (128 + 2) * 4 + lens


@pytest.mark.parametrize("field,value,code", [
    ("bits", 3, 2), ("group_size", 64, 2), ("residual", 64, 2), ("head_dim", 96, 2),
    ("num_q_heads", 12, 2), ("num_q_heads", 24, 2), ("batch", 0, 1), ("max_tokens", 0, 1),
])
def test_rejects_bad_configs(lib, field, value, code):
    s = N.KiviSizes()
    c = cfg(**{field: value})
    assert lib.kivi_required_bytes(ctypes.byref(c), ctypes.byref(s)) == code
    assert lib.kivi_required_bytes(None, ctypes.byref(s)) == 1


def test_create_validates_buffers_before_touching_the_device(lib):
    c = cfg(num_layers=1, batch=1, max_tokens=1000)
    s = N.KiviSizes()
    assert lib.kivi_required_bytes(ctypes.byref(c), ctypes.byref(s)) == 0
    fake = 1 << 20  # never dereferenced: the call fails on sizes first
    small = N.KiviSizes(s.records_bytes - 1, s.resid_k_bytes, s.resid_v_bytes, s.workspace_bytes)
    bufs = N.KiviBuffers(fake, fake, fake, fake, small)
    h = ctypes.c_void_p()
    assert lib.kivi_cache_create(ctypes.byref(c), ctypes.byref(bufs), ctypes.byref(h)) == 3
    misaligned = N.KiviBuffers(fake + 4, fake, fake, fake, s)
    assert lib.kivi_cache_create(ctypes.byref(c), ctypes.byref(misaligned), ctypes.byref(h)) == 1
    nulls = N.KiviBuffers(None, None, None, None, s)
    assert lib.kivi_cache_create(ctypes.byref(c), ctypes.byref(nulls), ctypes.byref(h)) == 1
    assert not h.value


def test_null_handle_calls_fail_cleanly(lib):
    S = ctypes.c_int32()
    assert lib.kivi_cache_length(None, 0, ctypes.byref(S), None) == 1
    assert lib.kivi_cache_reset(None, 0) == 1
    assert lib.kivi_quantize_prefill(None, 0, None, None, 0, None) == 1
    assert lib.kivi_append_token(None, 0, None, None, None) == 1
    assert lib.kivi_decode_attention(None, 0, None, None, 0.0, None) == 1
    assert lib.kivi_check_device_status(None, None, None) == 1
    lib.kivi_cache_destroy(None)


def test_status_strings(lib):
    for code in range(9):
        assert lib.kivi_status_string(code)
    assert lib.kivi_status_string(99) == b"unknown status"


@pytest.mark.parametrize("bits,S", [(2, 8192), (4, 8192), (2, 4096), (2, 300), (4, 161)])
def test_cache_bytes_agree_with_oracle(lib, bits, S):
    c = cfg(bits=bits)
    vals = [ctypes.c_double() for _ in range(3)]
    assert lib.kivi_cache_bytes(ctypes.byref(c), S, *[ctypes.byref(v) for v in vals]) == 0
    o = O.cache_bytes(32, 8, 128, bits, S)
    assert vals[0].value == pytest.approx(o["stored"], rel=1e-15)
    assert vals[1].value == pytest.approx(o["codes_only"], rel=1e-15)
    assert vals[2].value == pytest.approx(o["convention"], rel=1e-15)


def test_cache_bytes_pages_numbers(lib):
    """The record's printed figures: 18,432 (convention) and 18,176 (exact) B/token at
    2 bits, 34,816 at 4 bits, Llama-3-8B skeleton at 8,192 tokens."""
    out = [ctypes.c_double() for _ in range(3)]
    c = cfg(bits=2)
    lib.kivi_cache_bytes(ctypes.byref(c), 8192, *[ctypes.byref(v) for v in out])
    assert out[2].value == 18432 and out[1].value == 18176
    c = cfg(bits=4)
    lib.kivi_cache_bytes(ctypes.byref(c), 8192, None, None, ctypes.byref(out[2]))
    assert out[2].value == 34816
    assert lib.kivi_cache_bytes(ctypes.byref(c), 0, None, None, None) == 1


def test_bf16_workspace_bytes_and_validation(lib):
    """The bf16 baseline's host checks (no launch happens on these paths)."""
    n = ctypes.c_size_t()
    assert lib.kivi_bf16_workspace_bytes(16, 8, 32, 128, ctypes.byref(n)) == 0
    # header, 128 tickets rounded to 256 bytes, 256 CTAs x 2 partials of 4 heads
    assert n.value == 256 + 512 + 256 * 2 * 4 * 130 * 4
    assert N.STATUS[lib.kivi_bf16_workspace_bytes(1, 8, 24, 128, ctypes.byref(n))] == \
        "KIVI_ERR_UNSUPPORTED"
    assert N.STATUS[lib.kivi_bf16_workspace_bytes(1, 8, 8, 96, ctypes.byref(n))] == \
        "KIVI_ERR_UNSUPPORTED"
    fake = 1 << 20
    call = lambda S, Smax, ws: lib.kivi_bf16_decode_attention(  # noqa: E731
        fake, fake, 2, 2, 4, 128, Smax, S, fake, fake, 0.0, fake, ws, None)
    assert N.STATUS[call(0, 10, 1 << 30)] == "KIVI_ERR_INVALID_ARG"     # S < 1
    assert N.STATUS[call(11, 10, 1 << 30)] == "KIVI_ERR_INVALID_ARG"    # S > max_tokens
    assert N.STATUS[call(5, 10, 100)] == "KIVI_ERR_INVALID_ARG"         # workspace too small
    assert N.STATUS[lib.kivi_bf16_decode_attention(
        fake + 2, fake, 2, 2, 4, 128, 10, 5, fake, fake, 0.0, fake, 1 << 30, None)] == \
        "KIVI_ERR_INVALID_ARG"                                             # unaligned


def test_fake_quant_keys_validation(lib):
    fake = 1 << 20
    assert N.STATUS[lib.kivi_fake_quant_keys(fake, 33, 128, 2, 0, fake, None)] == \
        "KIVI_ERR_INVALID_ARG"
    assert N.STATUS[lib.kivi_fake_quant_keys(fake, 32, 128, 3, 0, fake, None)] == \
        "KIVI_ERR_UNSUPPORTED"
    assert N.STATUS[lib.kivi_fake_quant_keys(fake, 32, 96, 2, 0, fake, None)] == \
        "KIVI_ERR_UNSUPPORTED"
    assert lib.kivi_fake_quant_keys(fake, 0, 128, 2, 1, fake, None) == 0  # nothing to do


def test_record_layout_query(lib):
    """The binding's record views take the record size and count from the library."""
    import oracle as O2
    for D, bits, mt in [(128, 2, 8192 + 64), (128, 4, 300), (64, 2, 100)]:
        c = cfg(head_dim=D, bits=bits, max_tokens=mt)
        rb, ng = ctypes.c_size_t(), ctypes.c_int32()
        assert lib.kivi_record_layout(ctypes.byref(c), ctypes.byref(rb), ctypes.byref(ng)) == 0
        assert rb.value == O2.record_bytes(D, bits)
        assert ng.value == O2.num_groups(mt)
    assert N.STATUS[lib.kivi_record_layout(None, None, None)] == "KIVI_ERR_INVALID_ARG"


def test_ragged_entry_points_validate_without_a_handle(lib):
    lens = (ctypes.c_int32 * 2)(3, 5)
    assert N.STATUS[lib.kivi_quantize_prefill_ragged(None, 0, None, None, 8, lens, None)] == \
        "KIVI_ERR_INVALID_ARG"
    out = (ctypes.c_int32 * 2)()
    assert N.STATUS[lib.kivi_cache_lengths(None, 0, out)] == "KIVI_ERR_INVALID_ARG"


def test_prefill_attention_validation(lib):
    """Host checks of the prefill-attention entry points (no launch on these paths)."""
    fake = 1 << 20
    call = lambda B, hkv, hq, D, S, q=fake, status=None: lib.kivi_causal_attention(  # noqa: E731
        q, fake, fake, B, hkv, hq, D, S, fake, 0.0, status, None)
    assert N.STATUS[call(1, 8, 32, 128, 0)] == "KIVI_ERR_INVALID_ARG"        # S < 1
    assert N.STATUS[call(0, 8, 32, 128, 10)] == "KIVI_ERR_INVALID_ARG"       # no sequences
    assert N.STATUS[call(1, 8, 20, 128, 10)] == "KIVI_ERR_UNSUPPORTED"       # Hq % Hkv
    assert N.STATUS[call(1, 8, 32, 96, 10)] == "KIVI_ERR_UNSUPPORTED"        # head_dim
    assert N.STATUS[call(1, 8, 32, 128, 10, q=fake + 2)] == "KIVI_ERR_INVALID_ARG"   # unaligned
    assert N.STATUS[call(1, 8, 32, 128, 10, q=None)] == "KIVI_ERR_INVALID_ARG"       # NULL
    assert N.STATUS[call(1, 8, 32, 128, 10, status=fake + 2)] == "KIVI_ERR_INVALID_ARG"
    assert N.STATUS[call(4096, 8, 32, 128, 1 << 14)] == "KIVI_ERR_INVALID_ARG"  # rows >= 2^31
    assert N.STATUS[lib.kivi_prefill_attention(None, 0, fake, fake, fake, 16, fake, 0.0,
                                               None)] == "KIVI_ERR_INVALID_ARG"
