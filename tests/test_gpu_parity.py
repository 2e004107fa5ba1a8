"""GPU path against the CPU oracle on the same seeded inputs (needs a B200).

Packed codes, zero points and scales (the whole group record) and the bf16
residual ring must match the oracle byte for byte: both sides take every
quantization decision with the same IEEE fp32 operations.  Attention outputs
must satisfy |gpu - oracle| <= 2e-3 + 2e-3 |oracle| elementwise (abs 2e-3 /
rel 2e-3).  Small cases compare every output and every record; the full-size
workloads compare every record of the checked layers and all or a seeded
sample of the (sequence, query head) rows, in the launch configuration the
benchmark uses (the library picks it from the shapes alone).
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from gpu_util import assert_attention_close, assert_state_equal, load_kivi

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kivi():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return load_kivi()


def _rand(shape, gen, scale=None):
    x = torch.randn(shape, generator=gen)
    if scale is not None:
        x = x * scale
    return x.to(torch.bfloat16)


def _run_small(K, B, Hkv, Hq, D, bits, S0, steps, seed, check_each=True):
    gen = torch.Generator().manual_seed(seed)
    ch_scale = torch.exp(torch.randn(Hkv, D, generator=gen))[None, :, None, :]
    k = _rand((B, Hkv, S0, D), gen, ch_scale)
    v = _rand((B, Hkv, S0, D), gen)
    max_tokens = S0 + steps
    cache = K.KiviCache(batch=B, num_layers=2, num_kv_heads=Hkv, num_q_heads=Hq, head_dim=D,
                        bits=bits, max_tokens=max_tokens)
    ref = O.OracleCache(B, Hkv, D, bits, max_tokens)
    layer = 1
    cache.prefill(layer, k.cuda(), v.cuda())
    ref.prefill(synth.bf16_bits(k), synth.bf16_bits(v))
    torch.cuda.synchronize()
    assert_state_equal(cache, layer, ref, f"after prefill S={S0}")
    for step in range(steps):
        kn = _rand((B, Hkv, D), gen, ch_scale[:, :, 0, :])
        vn = _rand((B, Hkv, D), gen)
        q = _rand((B, Hq, D), gen)
        cache.append(layer, kn.cuda(), vn.cuda())
        ref.append(synth.bf16_bits(kn), synth.bf16_bits(vn))
        if check_each or step == steps - 1:
            out = cache.attend(layer, q.cuda()).cpu().numpy()
            assert_attention_close(out, ref.attention(synth.bf16_bits(q)),
                                   f"S={ref.S} B={B} Hkv={Hkv} Hq={Hq} D={D} b={bits}")
            assert_state_equal(cache, layer, ref, f"after append S={ref.S}")
    assert cache.check_device_status() == 0
    cache.close()


@pytest.mark.parametrize("S0,steps", [
    (0, 3), (1, 2), (127, 3), (128, 2), (159, 3), (160, 1), (161, 2), (190, 4),
    (255, 40), (512, 1),
])
def test_small_edges_2bit_gqa(kivi, S0, steps):
    _run_small(kivi, B=2, Hkv=2, Hq=4, D=64, bits=2, S0=S0, steps=steps, seed=S0 + 17)


@pytest.mark.parametrize("D,bits,hpk", [(128, 2, 1), (128, 4, 4), (64, 4, 1), (128, 2, 4),
                                        (128, 4, 2), (64, 2, 8)])
def test_small_shapes(kivi, D, bits, hpk):
    _run_small(kivi, B=3, Hkv=2, Hq=2 * hpk, D=D, bits=bits, S0=700, steps=35,
               seed=D + bits + hpk, check_each=False)


def test_many_splits(kivi):
    """One sequence and kv head at 8K tokens: 28 group splits plus 5 residual chunks, so the
    combine merges more than 32 partials (two per lane of its first warp)."""
    _run_small(kivi, B=1, Hkv=1, Hq=4, D=128, bits=2, S0=8192, steps=1, seed=91)


@pytest.mark.parametrize("B,Hkv,Hq,D,bits,S0", [(128, 16, 16, 64, 2, 300), (80, 16, 128, 64, 4, 200),
                                                (128, 16, 64, 128, 2, 161)])
def test_more_pairs_than_warps_per_cta(kivi, B, Hkv, Hq, D, bits, S0):
    """Thousands of short (sequence, kv head) pairs: every CTA holds more pairs than warps,
    so each warp sweeps whole pairs and finishes each from its registers (the output, or
    the CTA's partial and ticket for its first and last pair)."""
    _run_small(kivi, B=B, Hkv=Hkv, Hq=Hq, D=D, bits=bits, S0=S0, steps=2, seed=B + Hq + S0,
               check_each=False)


def test_decode_without_prefill(kivi):
    """Append-only growth from an empty layer through the first flush."""
    _run_small(kivi, B=1, Hkv=1, Hq=1, D=128, bits=2, S0=0, steps=165, seed=5, check_each=False)


def test_sm_scale_argument(kivi):
    gen = torch.Generator().manual_seed(3)
    B, Hkv, Hq, D = 2, 2, 4, 64
    k, v = _rand((B, Hkv, 300, D), gen), _rand((B, Hkv, 300, D), gen)
    q = _rand((B, Hq, D), gen)
    cache = kivi.KiviCache(batch=B, num_layers=1, num_kv_heads=Hkv, num_q_heads=Hq,
                           head_dim=D, bits=2, max_tokens=300)
    ref = O.OracleCache(B, Hkv, D, 2, 300)
    cache.prefill(0, k.cuda(), v.cuda())
    ref.prefill(synth.bf16_bits(k), synth.bf16_bits(v))
    for scale in (0.05, 0.5):
        out = cache.attend(0, q.cuda(), sm_scale=scale).cpu().numpy()
        assert_attention_close(out, ref.attention(synth.bf16_bits(q), sm_scale=scale))


def test_state_errors(kivi):
    cache = kivi.KiviCache(batch=1, num_layers=1, num_kv_heads=1, num_q_heads=1, head_dim=64,
                           bits=2, max_tokens=4)
    q = torch.zeros(1, 1, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kivi.KiviError, match="STATE"):
        cache.attend(0, q)
    kv = torch.zeros(1, 1, 5, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kivi.KiviError, match="CAPACITY"):
        cache.prefill(0, kv, kv)
    cache.prefill(0, kv[:, :, :4].contiguous(), kv[:, :, :4].contiguous())
    with pytest.raises(kivi.KiviError, match="STATE"):
        cache.prefill(0, kv[:, :, :4].contiguous(), kv[:, :, :4].contiguous())
    with pytest.raises(kivi.KiviError, match="CAPACITY"):
        cache.append(0, kv[:, :, 0].contiguous(), kv[:, :, 0].contiguous())
    with pytest.raises(kivi.KiviError, match="INVALID_ARG"):
        cache.attend(5, q)
    cache.close()


# ---------------------------------------------------------------------------
# The five workloads
# ---------------------------------------------------------------------------

def _workload_layer(K, w: synth.Workload, layers, steps, sample_rows=None, seed=0):
    """Prefill + `steps` decode steps on `layers` of workload w; compares state
    after prefill and after the last step, attention at the first and last step."""
    max_tokens = w.context + max(steps, 1)
    cache = K.KiviCache(batch=w.batch, num_layers=w.num_layers, num_kv_heads=w.num_kv_heads,
                        num_q_heads=w.num_q_heads, head_dim=w.head_dim, bits=w.bits,
                        max_tokens=max_tokens)
    rng = np.random.default_rng(seed)
    for layer in layers:
        k, v = synth.prefill_kv(w, layer)
        ref = O.OracleCache(w.batch, w.num_kv_heads, w.head_dim, w.bits, max_tokens)
        cache.prefill(layer, k.cuda(), v.cuda())
        ref.prefill(synth.bf16_bits(k), synth.bf16_bits(v))
        del k, v
        torch.cuda.synchronize()
        assert_state_equal(cache, layer, ref, f"{w.name} layer {layer} prefill")
        for step in range(steps):
            kn, vn = synth.step_kv(w, layer, step)
            cache.append(layer, kn.cuda(), vn.cuda())
            ref.append(synth.bf16_bits(kn), synth.bf16_bits(vn))
            if step in (0, steps - 1):
                q = synth.query(w, layer, step)
                out = cache.attend(layer, q.cuda()).cpu().numpy()
                qb = synth.bf16_bits(q)
                if sample_rows is None:
                    assert_attention_close(out, ref.attention(qb), f"{w.name} S={ref.S}")
                else:
                    rows = [(int(b), int(h)) for b, h in zip(
                        rng.integers(0, w.batch, sample_rows),
                        rng.integers(0, w.num_q_heads, sample_rows))]
                    rows += [(0, 0), (w.batch - 1, w.num_q_heads - 1)]
                    for b, h in rows:
                        assert_attention_close(out[b, h], ref.attend(b, h, qb[b, h],
                                                                     w.num_q_heads),
                                               f"{w.name} S={ref.S} row ({b},{h})")
                    assert np.isfinite(out).all()
        torch.cuda.synchronize()
        assert_state_equal(cache, layer, ref, f"{w.name} layer {layer} after {steps} steps")
    assert cache.check_device_status() == 0
    cache.close()


def test_workload_tiny(kivi):
    w = synth.WORKLOADS["tiny"]
    _workload_layer(kivi, w, layers=[0], steps=w.decode_steps)


def test_workload_llama2_7b_mha_layer(kivi):
    w = synth.WORKLOADS["llama2_7b_mha_layer"]
    _workload_layer(kivi, w, layers=[0], steps=w.decode_steps)


def test_workload_llama3_8b_gqa_8k(kivi):
    w = synth.WORKLOADS["llama3_8b_gqa_8k"]
    _workload_layer(kivi, w, layers=[0, 31], steps=33, sample_rows=48)


def test_workload_llama3_8b_gqa_8k_4bit(kivi):
    w = synth.WORKLOADS["llama3_8b_gqa_8k_4bit"]
    _workload_layer(kivi, w, layers=[0], steps=1, sample_rows=48)


def test_workload_llama2_13b_mha_b16(kivi):
    w = synth.WORKLOADS["llama2_13b_mha_sweep"]
    _workload_layer(kivi, w, layers=[39], steps=1, sample_rows=48)
