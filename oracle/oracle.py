"""ctypes wrapper of the C oracle, the cache state machine and the byte arithmetic.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources, by page title and section:
  [KIVI page]   "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache".
  [HF page]     "KV cache quantization squeezes 5GB down to fit longer LLM
                generations".
  [Llama-3 rec] record "kv-efficiency/kivi-2bit-llama3-8b-gqa-8k", fields
                "Model", "KV bytes basis", "Methodology", "notes".

All bf16 tensors cross this module as numpy uint16 arrays of their bit patterns.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import tempfile

import numpy as np

G = 32   # group size of keys (tokens) and values (channels), [Llama-3 rec] "Methodology"
R = 128  # residual length in tokens, [Llama-3 rec] "Methodology"

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kivi_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compiles kivi_oracle.c with gcc into oracle/_build/liboracle.so when stale."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    os.makedirs(_LIB_DIR, exist_ok=True)
    fd, tmp = tempfile.mkstemp(suffix=".so", dir=_LIB_DIR)
    os.close(fd)
    subprocess.run(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _c():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i, l, d = ctypes.c_int, ctypes.c_long, ctypes.c_double
        lib.oracle_f32_to_f16_bits.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_f16_bits.restype = ctypes.c_uint16
        lib.oracle_f16_bits_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_bits_to_double.restype = d
        lib.oracle_quantize_group.argtypes = [f32p, i, i, i, f32p, f32p, u8p]
        lib.oracle_quantize_group.restype = None
        lib.oracle_record_bytes.argtypes = [i, i]
        lib.oracle_record_bytes.restype = l
        lib.oracle_num_groups.argtypes = [i]
        lib.oracle_num_groups.restype = i
        lib.oracle_make_record.argtypes = [u16p, u16p, l, i, i, u8p]
        lib.oracle_make_record.restype = None
        lib.oracle_dequant_record.argtypes = [u8p, i, i, f64p, f64p]
        lib.oracle_dequant_record.restype = None
        lib.oracle_prefill.argtypes = [u16p, u16p, i, i, i, i, i, i, u8p, u16p, u16p]
        lib.oracle_prefill.restype = None
        lib.oracle_append.argtypes = [u16p, u16p, i, i, i, i, i, i, u8p, u16p, u16p]
        lib.oracle_append.restype = i
        lib.oracle_attend_one.argtypes = [u8p, u16p, u16p, u16p, i, i, i, d, f64p]
        lib.oracle_attend_one.restype = None
        lib.oracle_attention.argtypes = [u8p, u16p, u16p, u16p, i, i, i, i, i, i, i, d, f64p]
        lib.oracle_attention.restype = None
        lib.oracle_attention_bf16.argtypes = [u16p, u16p, u16p, i, i, i, i, i, i, d, f64p]
        lib.oracle_attention_bf16.restype = None
        lib.oracle_prefill_attention.argtypes = [u16p, u16p, u16p, i, i, i, i, i, d, f64p]
        lib.oracle_prefill_attention.restype = None
        lib.oracle_fake_quant_keys.argtypes = [u16p, i, i, i, i, f64p]
        lib.oracle_fake_quant_keys.restype = None
        _lib = lib
    return _lib


def _p(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.POINTER(ctype))


# --------------------------------------------------------------------------
# Scalar and group functions
# --------------------------------------------------------------------------

def f32_to_f16_bits(x: float) -> int:
    """IEEE binary16 bits of fp32 x, round to nearest even."""
    return int(_c().oracle_f32_to_f16_bits(ctypes.c_float(x)))


def f16_bits_to_double(h: int) -> float:
    return float(_c().oracle_f16_bits_to_double(h))


def quantize_group(x: np.ndarray, bits: int):
    """Asymmetric quantizer of one group (fp32 values): returns (scale32, min32, codes).

    zero point = min, scale = (max - min) / (2^b - 1), codes round half to even.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.zeros(x.size, np.uint8)
    scale = ctypes.c_float()
    mn = ctypes.c_float()
    _c().oracle_quantize_group(_p(x, ctypes.c_float), x.size, 1, bits,
                               ctypes.byref(scale), ctypes.byref(mn), _p(codes, ctypes.c_uint8))
    return np.float32(scale.value), np.float32(mn.value), codes


def num_groups(S: int) -> int:
    """NG(S) = max(0, floor((S - R) / G)) ([Llama-3 rec] "KV bytes basis")."""
    return int(_c().oracle_num_groups(S))


def record_bytes(D: int, bits: int) -> int:
    return int(_c().oracle_record_bytes(D, bits))


def make_record(k_tile: np.ndarray, v_tile: np.ndarray, bits: int) -> np.ndarray:
    """One group record from bf16-bit tiles [G][D] of keys and values."""
    k_tile = np.ascontiguousarray(k_tile, dtype=np.uint16)
    v_tile = np.ascontiguousarray(v_tile, dtype=np.uint16)
    D = k_tile.shape[1]
    rec = np.zeros(record_bytes(D, bits), np.uint8)
    _c().oracle_make_record(_p(k_tile, ctypes.c_uint16), _p(v_tile, ctypes.c_uint16), D, D,
                            bits, _p(rec, ctypes.c_uint8))
    return rec


def dequant_record(rec: np.ndarray, D: int, bits: int):
    """Dequantized (k_hat, v_hat) tiles [G][D] in float64 from a record."""
    rec = np.ascontiguousarray(rec, dtype=np.uint8)
    k = np.zeros((G, D), np.float64)
    v = np.zeros((G, D), np.float64)
    _c().oracle_dequant_record(_p(rec, ctypes.c_uint8), D, bits, _p(k, ctypes.c_double),
                               _p(v, ctypes.c_double))
    return k, v


def attend_one(seq_records, seq_ring_k, seq_ring_v, q_row, S, bits, sm_scale):
    """Attention of one query head (bf16 bits [D]) over one kv head's state."""
    D = q_row.shape[-1]
    out = np.zeros(D, np.float64)
    _c().oracle_attend_one(_p(seq_records, ctypes.c_uint8), _p(seq_ring_k, ctypes.c_uint16),
                           _p(seq_ring_v, ctypes.c_uint16),
                           _p(np.ascontiguousarray(q_row, np.uint16), ctypes.c_uint16),
                           S, D, bits, float(sm_scale), _p(out, ctypes.c_double))
    return out


def attention_bf16(k: np.ndarray, v: np.ndarray, q: np.ndarray, S: int | None = None,
                   sm_scale: float | None = None) -> np.ndarray:
    """Decode attention over an unquantized bf16 cache (the 16-bit baseline).

    k, v: bf16 bits [B][Hkv][Smax][D] (tokens 0..S-1 used); q: bf16 bits [B][Hq][D]
    -> float64 [B][Hq][D]; query head h reads kv head h // (Hq // Hkv).
    """
    k = np.ascontiguousarray(k, np.uint16)
    v = np.ascontiguousarray(v, np.uint16)
    q = np.ascontiguousarray(q, np.uint16)
    B, Hkv, Smax, D = k.shape
    Hq = q.shape[1]
    assert Hq % Hkv == 0 and q.shape == (B, Hq, D)
    S = Smax if S is None else S
    scale = 1.0 / math.sqrt(D) if sm_scale is None or sm_scale <= 0 else float(sm_scale)
    out = np.zeros((B, Hq, D), np.float64)
    _c().oracle_attention_bf16(_p(k, ctypes.c_uint16), _p(v, ctypes.c_uint16),
                               _p(q, ctypes.c_uint16), B, Hkv, Hq, S, Smax, D, scale,
                               _p(out, ctypes.c_double))
    return out


def prefill_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                      sm_scale: float | None = None) -> np.ndarray:
    """Causal attention of a prompt: q bf16 bits [B][Hq][S][D], k, v [B][Hkv][S][D]
    -> float64 [B][Hq][S][D]; position i attends tokens 0..i."""
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    v = np.ascontiguousarray(v, np.uint16)
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    assert k.shape == (B, Hkv, S, D) and v.shape == k.shape and Hq % Hkv == 0
    scale = 1.0 / math.sqrt(D) if sm_scale is None or sm_scale <= 0 else float(sm_scale)
    out = np.zeros((B, Hq, S, D), np.float64)
    _c().oracle_prefill_attention(_p(q, ctypes.c_uint16), _p(k, ctypes.c_uint16),
                                  _p(v, ctypes.c_uint16), B, Hkv, Hq, S, D, scale,
                                  _p(out, ctypes.c_double))
    return out


def fake_quant_keys(k: np.ndarray, bits: int, per_token: bool) -> np.ndarray:
    """Quantize-dequantize keys (bf16 bits [T][D], T a multiple of G) -> float64.

    per_token=False: per channel over G-token groups (KIVI's key rule);
    per_token=True: per token over G-channel blocks (the values' rule applied to
    keys, the granularity the [KIVI page] and the [HF page] argue against).
    """
    k = np.ascontiguousarray(k, np.uint16)
    T, D = k.shape
    assert T % G == 0 and D % G == 0
    out = np.zeros((T, D), np.float64)
    _c().oracle_fake_quant_keys(_p(k, ctypes.c_uint16), T, D, bits, int(per_token),
                                _p(out, ctypes.c_double))
    return out


# --------------------------------------------------------------------------
# Cache state of one layer
# --------------------------------------------------------------------------

class OracleCache:
    """Quantized history plus bf16 residual of one layer ([Llama-3 rec] "KV bytes basis").

    records: uint8 [B][Hkv][NGcap][record bytes]; ring_k, ring_v: bf16 bits
    [B][Hkv][R+G][D], token t at slot t mod (R+G).
    """

    def __init__(self, B: int, Hkv: int, D: int, bits: int, max_tokens: int):
        self.B, self.Hkv, self.D, self.bits = B, Hkv, D, bits
        self.max_tokens = max_tokens
        self.NGcap = num_groups(max_tokens)
        self.rb = record_bytes(D, bits)
        self.records = np.zeros((B, Hkv, max(self.NGcap, 1), self.rb), np.uint8)
        self.ring_k = np.zeros((B, Hkv, R + G, D), np.uint16)
        self.ring_v = np.zeros((B, Hkv, R + G, D), np.uint16)
        self.S = 0

    @property
    def NG(self) -> int:
        return num_groups(self.S)

    def _rec_ptr(self):
        return _p(self.records, ctypes.c_uint8)

    def prefill(self, k: np.ndarray, v: np.ndarray) -> None:
        """k, v: bf16 bits [B][Hkv][S][D]."""
        assert self.S == 0
        k = np.ascontiguousarray(k, np.uint16)
        v = np.ascontiguousarray(v, np.uint16)
        S = k.shape[2]
        assert S <= self.max_tokens
        _c().oracle_prefill(_p(k, ctypes.c_uint16), _p(v, ctypes.c_uint16), self.B, self.Hkv,
                            S, self.D, self.bits, self.records.shape[2], self._rec_ptr(),
                            _p(self.ring_k, ctypes.c_uint16), _p(self.ring_v, ctypes.c_uint16))
        self.S = S

    def append(self, k_new: np.ndarray, v_new: np.ndarray) -> None:
        """k_new, v_new: bf16 bits [B][Hkv][D]; flushes a group when due."""
        assert self.S + 1 <= self.max_tokens
        k_new = np.ascontiguousarray(k_new, np.uint16)
        v_new = np.ascontiguousarray(v_new, np.uint16)
        self.S = int(_c().oracle_append(
            _p(k_new, ctypes.c_uint16), _p(v_new, ctypes.c_uint16), self.B, self.Hkv, self.S,
            self.D, self.bits, self.records.shape[2], self._rec_ptr(),
            _p(self.ring_k, ctypes.c_uint16), _p(self.ring_v, ctypes.c_uint16)))

    def attention(self, q: np.ndarray, sm_scale: float | None = None) -> np.ndarray:
        """q: bf16 bits [B][Hq][D] -> float64 [B][Hq][D]."""
        q = np.ascontiguousarray(q, np.uint16)
        B, Hq, D = q.shape
        assert Hq % self.Hkv == 0
        scale = 1.0 / math.sqrt(D) if sm_scale is None or sm_scale <= 0 else float(sm_scale)
        out = np.zeros((B, Hq, D), np.float64)
        _c().oracle_attention(self._rec_ptr(), _p(self.ring_k, ctypes.c_uint16),
                              _p(self.ring_v, ctypes.c_uint16), _p(q, ctypes.c_uint16), B,
                              self.Hkv, Hq, self.S, D, self.bits, self.records.shape[2], scale,
                              _p(out, ctypes.c_double))
        return out

    def attend(self, b: int, h: int, q_row: np.ndarray, Hq: int,
               sm_scale: float | None = None) -> np.ndarray:
        """One (sequence, query head) row of ``attention`` (for sampled checks)."""
        kvh = h // (Hq // self.Hkv)
        scale = 1.0 / math.sqrt(self.D) if sm_scale is None or sm_scale <= 0 else sm_scale
        return attend_one(np.ascontiguousarray(self.records[b, kvh]),
                          np.ascontiguousarray(self.ring_k[b, kvh]),
                          np.ascontiguousarray(self.ring_v[b, kvh]), q_row, self.S, self.bits,
                          scale)


# --------------------------------------------------------------------------
# Byte arithmetic ([Llama-3 rec] "KV bytes basis" and "notes")
# --------------------------------------------------------------------------

def cache_bytes(num_layers: int, num_kv_heads: int, head_dim: int, bits: int, S: int) -> dict:
    """KV-cache bytes per token of one sequence holding S tokens, all layers.

    convention: grouped codes counted at every token (layers x kv heads x
      head_dim x 2 (K and V) x bits/8) plus the bf16 residual of R tokens
      amortised over S - the record's convention.
    codes_only: grouped codes over the NG(S)*G quantized tokens plus the r bf16
      residual tokens, over S - the record's "exact stored amount".
    stored: NG(S) whole group records (codes and fp16 metadata) plus the r
      residual tokens, over S - what the packed layout occupies.
    """
    per_tok_codes = num_layers * num_kv_heads * head_dim * 2 * bits / 8
    per_tok_bf16 = num_layers * num_kv_heads * head_dim * 2 * 2
    NG = num_groups(S)
    r = S - NG * G
    return {
        "convention": per_tok_codes + R * per_tok_bf16 / S,
        "codes_only": (NG * G * per_tok_codes + r * per_tok_bf16) / S,
        "stored": (NG * num_layers * num_kv_heads * record_bytes(head_dim, bits)
                   + r * per_tok_bf16) / S,
        "bf16": per_tok_bf16,
    }
