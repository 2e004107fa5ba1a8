"""KIVI packed KV cache with fused decode attention for B200 (sm_100a).

A thin binding of the C ABI in ``include/kivi.h`` (``libkivi.so``): the
functions below carry the C names and only marshal arguments; every step of the
path runs in the library's CUDA kernels.  PyTorch supplies device memory and
streams.  There is no CPU fallback: if the library is missing, calls raise.

``KiviCache`` is a convenience owner of the device buffers (allocated with
torch) around one handle.
"""
from __future__ import annotations

import ctypes

import torch

from ._native import KiviBuffers, KiviConfig, KiviError, KiviSizes, check, lib

__all__ = [
    "KiviCache", "KiviConfig", "KiviError", "make_config",
    "kivi_required_bytes", "kivi_record_layout", "kivi_cache_create", "kivi_cache_destroy",
    "kivi_cache_length",
    "kivi_cache_reset", "kivi_quantize_prefill", "kivi_quantize_prefill_ragged",
    "kivi_cache_lengths", "kivi_append_token", "kivi_decode_attention",
    "kivi_check_device_status", "kivi_cache_bytes", "kivi_status_string",
    "kivi_decode_attention_static_scratch", "kivi_static_scratch_status",
    "kivi_bf16_workspace_bytes", "kivi_bf16_decode_attention", "kivi_bf16_status",
    "Bf16Attention", "kivi_fake_quant_keys", "kivi_prefill_attention", "kivi_causal_attention",
]

GROUP_SIZE = 32
RESIDUAL = 128


def make_config(*, batch, num_layers, num_kv_heads, num_q_heads, head_dim, bits, max_tokens,
                group_size=GROUP_SIZE, residual=RESIDUAL) -> KiviConfig:
    return KiviConfig(batch, num_layers, num_kv_heads, num_q_heads, head_dim, bits,
                      group_size, residual, max_tokens)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor | None, dtype=None, name="tensor") -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def kivi_required_bytes(cfg: KiviConfig) -> KiviSizes:
    out = KiviSizes()
    check(lib().kivi_required_bytes(ctypes.byref(cfg), ctypes.byref(out)), "kivi_required_bytes")
    return out


def kivi_record_layout(cfg: KiviConfig) -> tuple[int, int]:
    """(bytes of one group record, records per (layer, sequence, kv head))."""
    rb, ng = ctypes.c_size_t(), ctypes.c_int32()
    check(lib().kivi_record_layout(ctypes.byref(cfg), ctypes.byref(rb), ctypes.byref(ng)),
          "kivi_record_layout")
    return rb.value, ng.value


def kivi_cache_create(cfg: KiviConfig, buffers: KiviBuffers) -> int:
    h = ctypes.c_void_p()
    check(lib().kivi_cache_create(ctypes.byref(cfg), ctypes.byref(buffers), ctypes.byref(h)),
          "kivi_cache_create")
    return h.value


def kivi_cache_destroy(handle: int) -> None:
    lib().kivi_cache_destroy(handle)


def kivi_cache_length(handle: int, layer: int) -> tuple[int, int]:
    S, NG = ctypes.c_int32(), ctypes.c_int32()
    check(lib().kivi_cache_length(handle, layer, ctypes.byref(S), ctypes.byref(NG)),
          "kivi_cache_length")
    return S.value, NG.value


def kivi_cache_reset(handle: int, layer: int) -> None:
    check(lib().kivi_cache_reset(handle, layer), "kivi_cache_reset")


def kivi_quantize_prefill(handle: int, layer: int, k: torch.Tensor, v: torch.Tensor,
                          S: int | None = None, stream=None) -> None:
    """k, v: bf16 [B][Hkv][S][D] on the device."""
    S = k.shape[2] if S is None else S
    check(lib().kivi_quantize_prefill(handle, layer, _ptr(k, torch.bfloat16, "k"),
                                      _ptr(v, torch.bfloat16, "v"), S, _stream(stream)),
          "kivi_quantize_prefill")


def kivi_quantize_prefill_ragged(handle: int, layer: int, k: torch.Tensor, v: torch.Tensor,
                                 lengths, stream=None) -> None:
    """k, v: bf16 [B][Hkv][S_max][D] on the device; lengths: B ints (tokens per sequence)."""
    lens = (ctypes.c_int32 * len(lengths))(*[int(x) for x in lengths])
    check(lib().kivi_quantize_prefill_ragged(handle, layer, _ptr(k, torch.bfloat16, "k"),
                                             _ptr(v, torch.bfloat16, "v"), k.shape[2], lens,
                                             _stream(stream)), "kivi_quantize_prefill_ragged")


def kivi_cache_lengths(handle: int, layer: int, batch: int) -> list:
    out = (ctypes.c_int32 * batch)()
    check(lib().kivi_cache_lengths(handle, layer, out), "kivi_cache_lengths")
    return list(out)


def kivi_append_token(handle: int, layer: int, k_new: torch.Tensor, v_new: torch.Tensor,
                      stream=None) -> None:
    """k_new, v_new: bf16 [B][Hkv][D] on the device."""
    check(lib().kivi_append_token(handle, layer, _ptr(k_new, torch.bfloat16, "k_new"),
                                  _ptr(v_new, torch.bfloat16, "v_new"), _stream(stream)),
          "kivi_append_token")


def kivi_decode_attention(handle: int, layer: int, q: torch.Tensor, out: torch.Tensor,
                          sm_scale: float = 0.0, stream=None) -> torch.Tensor:
    """q: bf16 [B][Hq][D]; out: fp32 [B][Hq][D] (written)."""
    check(lib().kivi_decode_attention(handle, layer, _ptr(q, torch.bfloat16, "q"),
                                      _ptr(out, torch.float32, "out"), float(sm_scale),
                                      _stream(stream)),
          "kivi_decode_attention")
    return out


def kivi_decode_attention_static_scratch(cfg: KiviConfig, records: int, resid_k: int,
                                         resid_v: int, layer: int, S: int, q: torch.Tensor,
                                         out: torch.Tensor, sm_scale: float = 0.0,
                                         stream=None) -> torch.Tensor:
    """Decode attention for callers that cannot allocate device memory.

    Takes the cache buffers (device addresses) and the layer's token count S
    instead of a handle, and keeps its split-K partials in the library's static
    device array (no workspace).  Calls whose kernels overlap on the GPU share
    that array and race; serialise them.  The first call on a device sets the
    array up and should come before any stream capture.
    """
    check(lib().kivi_decode_attention_static_scratch(
        ctypes.byref(cfg), records, resid_k, resid_v, layer, S, _ptr(q, torch.bfloat16, "q"),
        _ptr(out, torch.float32, "out"), float(sm_scale), _stream(stream)),
        "kivi_decode_attention_static_scratch")
    return out


def kivi_static_scratch_status(stream=None) -> int:
    """Reads and clears the status word of the static-scratch decode call on the
    current device (0 = no kernel recorded a failure)."""
    code = ctypes.c_uint32()
    rc = lib().kivi_static_scratch_status(_stream(stream), ctypes.byref(code))
    if rc not in (0, 7):
        check(rc, "kivi_static_scratch_status")
    return code.value


def kivi_check_device_status(handle: int, stream=None) -> int:
    code = ctypes.c_uint32()
    rc = lib().kivi_check_device_status(handle, _stream(stream), ctypes.byref(code))
    if rc not in (0, 7):
        check(rc, "kivi_check_device_status")
    return code.value


def kivi_cache_bytes(cfg: KiviConfig, S: int) -> dict:
    a, b, c = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    check(lib().kivi_cache_bytes(ctypes.byref(cfg), S, ctypes.byref(a), ctypes.byref(b),
                                 ctypes.byref(c)), "kivi_cache_bytes")
    return {"stored": a.value, "codes_only": b.value, "convention": c.value}


def kivi_bf16_workspace_bytes(batch: int, num_kv_heads: int, num_q_heads: int,
                              head_dim: int) -> int:
    n = ctypes.c_size_t()
    check(lib().kivi_bf16_workspace_bytes(batch, num_kv_heads, num_q_heads, head_dim,
                                          ctypes.byref(n)), "kivi_bf16_workspace_bytes")
    return n.value


def kivi_bf16_decode_attention(k_cache: torch.Tensor, v_cache: torch.Tensor, S: int,
                               q: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                               sm_scale: float = 0.0, stream=None) -> torch.Tensor:
    """k_cache, v_cache: bf16 [B][Hkv][Smax][D]; q: bf16 [B][Hq][D]; out: fp32 like q."""
    B, Hkv, Smax, D = k_cache.shape
    Hq = q.shape[1]
    if v_cache.shape != k_cache.shape or q.shape != (B, Hq, D) or out.shape != q.shape:
        raise ValueError("shapes: k/v [B][Hkv][Smax][D], q and out [B][Hq][D]")
    check(lib().kivi_bf16_decode_attention(
        _ptr(k_cache, torch.bfloat16, "k_cache"), _ptr(v_cache, torch.bfloat16, "v_cache"),
        B, Hkv, Hq, D, Smax, S, _ptr(q, torch.bfloat16, "q"), _ptr(out, torch.float32, "out"),
        float(sm_scale), _ptr(workspace, name="workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)),
        "kivi_bf16_decode_attention")
    return out


def kivi_bf16_status(workspace: torch.Tensor, batch: int, num_kv_heads: int, stream=None) -> int:
    code = ctypes.c_uint32()
    rc = lib().kivi_bf16_status(_ptr(workspace, name="workspace"), batch, num_kv_heads,
                                _stream(stream), ctypes.byref(code))
    if rc not in (0, 7):
        check(rc, "kivi_bf16_status")
    return code.value


def kivi_fake_quant_keys(k: torch.Tensor, bits: int, per_token: bool,
                         k_hat: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Quantize-dequantize keys (bf16 [rows][D], rows a multiple of 32) per channel
    (KIVI) or per token; returns fp32 k_hat [rows][D]."""
    rows, D = k.shape
    if k_hat is None:
        k_hat = torch.empty((rows, D), dtype=torch.float32, device=k.device)
    check(lib().kivi_fake_quant_keys(_ptr(k, torch.bfloat16, "k"), rows, D, bits,
                                     int(bool(per_token)), _ptr(k_hat, torch.float32, "k_hat"),
                                     _stream(stream)), "kivi_fake_quant_keys")
    return k_hat


def _prefill_shapes(q, k, v, out):
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, S, D) or v.shape != k.shape or out.shape != q.shape:
        raise ValueError("shapes: q and out [B][Hq][S][D], k and v [B][Hkv][S][D]")
    return B, Hkv, Hq, S, D


def kivi_prefill_attention(handle: int, layer: int, q: torch.Tensor, k: torch.Tensor,
                           v: torch.Tensor, out: torch.Tensor, sm_scale: float = 0.0,
                           stream=None) -> torch.Tensor:
    """Causal attention of the prompt (q bf16 [B][Hq][S][D], k, v bf16 [B][Hkv][S][D])
    into out (fp32 like q), with the prompt quantized into the layer as it goes."""
    S = _prefill_shapes(q, k, v, out)[3]
    check(lib().kivi_prefill_attention(handle, layer, _ptr(q, torch.bfloat16, "q"),
                                       _ptr(k, torch.bfloat16, "k"), _ptr(v, torch.bfloat16, "v"),
                                       S, _ptr(out, torch.float32, "out"), float(sm_scale),
                                       _stream(stream)), "kivi_prefill_attention")
    return out


def kivi_causal_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                          out: torch.Tensor | None = None, sm_scale: float = 0.0,
                          status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Causal attention alone (no cache): q bf16 [B][Hq][S][D], k, v bf16 [B][Hkv][S][D]
    -> out fp32 [B][Hq][S][D]; status: an optional zeroed int32 device word that a
    timed-out wait sets."""
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    B, Hkv, Hq, S, D = _prefill_shapes(q, k, v, out)
    check(lib().kivi_causal_attention(_ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
                                      _ptr(v, torch.bfloat16, "v"), B, Hkv, Hq, D, S,
                                      _ptr(out, torch.float32, "out"), float(sm_scale),
                                      _ptr(status, torch.int32, "status"), _stream(stream)),
          "kivi_causal_attention")
    return out


class Bf16Attention:
    """Owns the zeroed workspace of kivi_bf16_decode_attention for one shape."""

    def __init__(self, *, batch, num_kv_heads, num_q_heads, head_dim, device=None):
        self.B, self.Hkv, self.Hq, self.D = batch, num_kv_heads, num_q_heads, head_dim
        n = kivi_bf16_workspace_bytes(batch, num_kv_heads, num_q_heads, head_dim)
        self.workspace = torch.zeros(n, dtype=torch.uint8, device=device or "cuda")

    def attend(self, k_cache, v_cache, S, q, out=None, sm_scale=0.0, stream=None):
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        return kivi_bf16_decode_attention(k_cache, v_cache, S, q, out, self.workspace, sm_scale,
                                          stream)

    def check_device_status(self, stream=None) -> int:
        return kivi_bf16_status(self.workspace, self.B, self.Hkv, stream)


def kivi_status_string(code: int) -> str:
    return lib().kivi_status_string(code).decode()


class KiviCache:
    """Device buffers (torch allocations) plus one libkivi handle."""

    def __init__(self, *, batch, num_layers, num_kv_heads, num_q_heads, head_dim, bits,
                 max_tokens, device="cuda"):
        self.cfg = make_config(batch=batch, num_layers=num_layers, num_kv_heads=num_kv_heads,
                               num_q_heads=num_q_heads, head_dim=head_dim, bits=bits,
                               max_tokens=max_tokens)
        sizes = kivi_required_bytes(self.cfg)
        dev = torch.device(device)
        self.records = torch.empty(max(sizes.records_bytes, 16), dtype=torch.uint8, device=dev)
        self.resid_k = torch.empty(sizes.resid_k_bytes, dtype=torch.uint8, device=dev)
        self.resid_v = torch.empty(sizes.resid_v_bytes, dtype=torch.uint8, device=dev)
        self.workspace = torch.empty(sizes.workspace_bytes, dtype=torch.uint8, device=dev)
        bufs = KiviBuffers(self.records.data_ptr(), self.resid_k.data_ptr(),
                           self.resid_v.data_ptr(), self.workspace.data_ptr(),
                           KiviSizes(self.records.numel(), self.resid_k.numel(),
                                     self.resid_v.numel(), self.workspace.numel()))
        self.sizes = sizes
        self.handle = kivi_cache_create(self.cfg, bufs)

    # -- views of the packed state (for tests and inspection) --
    def record_bytes(self) -> int:
        return kivi_record_layout(self.cfg)[0]

    def ngcap(self) -> int:
        return kivi_record_layout(self.cfg)[1]

    def records_view(self, layer: int) -> torch.Tensor:
        c = self.cfg
        n = c.batch * c.num_kv_heads * self.ngcap() * self.record_bytes()
        return self.records[layer * n:(layer + 1) * n].view(
            c.batch, c.num_kv_heads, self.ngcap(), self.record_bytes())

    def ring_view(self, which: str, layer: int) -> torch.Tensor:
        c = self.cfg
        buf = self.resid_k if which == "k" else self.resid_v
        per_layer = c.batch * c.num_kv_heads * (RESIDUAL + GROUP_SIZE) * c.head_dim
        return buf.view(torch.bfloat16)[layer * per_layer:(layer + 1) * per_layer].view(
            c.batch, c.num_kv_heads, RESIDUAL + GROUP_SIZE, c.head_dim)

    # -- calls --
    def prefill(self, layer, k, v, stream=None):
        kivi_quantize_prefill(self.handle, layer, k, v, stream=stream)

    def prefill_attention(self, layer, q, k, v, out=None, sm_scale=0.0, stream=None):
        """Causal attention of the prompt with the prompt quantized into `layer`."""
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        return kivi_prefill_attention(self.handle, layer, q, k, v, out, sm_scale, stream)

    def prefill_ragged(self, layer, k, v, lengths, stream=None):
        return kivi_quantize_prefill_ragged(self.handle, layer, k, v, lengths, stream)

    def lengths(self, layer) -> list:
        return kivi_cache_lengths(self.handle, layer, self.cfg.batch)

    def append(self, layer, k_new, v_new, stream=None):
        kivi_append_token(self.handle, layer, k_new, v_new, stream=stream)

    def attend(self, layer, q, out=None, sm_scale=0.0, stream=None):
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        return kivi_decode_attention(self.handle, layer, q, out, sm_scale, stream=stream)

    def length(self, layer):
        return kivi_cache_length(self.handle, layer)

    def reset(self, layer):
        kivi_cache_reset(self.handle, layer)

    def check_device_status(self, stream=None) -> int:
        return kivi_check_device_status(self.handle, stream)

    def close(self):
        if getattr(self, "handle", None):
            kivi_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
