"""Causal prefill attention on the tensor cores, with the prompt quantized into the
cache in its epilogue (needs a B200).

Attention is compared with the oracle's causal attention (fp64) element by
element.  The kernel's scores and sums are fp32 on exact bf16 products; the one
coarser rounding is the softmax weight, rounded to bf16 (relative error at most
2^-9) before the second product, so

    |gpu - oracle| <= 2^-9 * sum_j p_ij |v_j| / sum_j p_ij  (+ fp32 rounding),

and the test allows 2^-8 times that weighted mean of |v| (the oracle's own
attention over |v|) plus 1e-5.  The cache a fused prefill leaves is compared
with the oracle's prefill byte for byte (records of the NG(S) groups, the live
ring slots), and a decode step after it with the oracle's decode.
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


def _abs_bits(x: np.ndarray) -> np.ndarray:
    return x & np.uint16(0x7FFF)


def _assert_within_weight_rounding(got, expect, expect_abs, what):
    err = np.abs(got.astype(np.float64) - expect)
    bound = 2.0 ** -8 * expect_abs + 1e-5
    bad = err > bound
    assert not np.isnan(got).any(), f"{what}: NaN"
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside the bound, max err "
                           f"{err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}")


def _inputs(B, Hkv, Hq, S, D, seed, k_growth=0.0):
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, S, D, generator=gen)
    k = torch.randn(B, Hkv, S, D, generator=gen)
    if k_growth:  # scores that grow along the prompt: the row maximum keeps rising
        k = k * (1 + k_growth * torch.arange(S, dtype=torch.float32))[None, None, :, None]
    v = torch.randn(B, Hkv, S, D, generator=gen)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


@pytest.mark.parametrize("B,Hkv,Hq,S,D", [
    (1, 1, 1, 1, 64),        # one token
    (1, 2, 8, 300, 128),     # GQA, three query tiles, ragged tail
    (2, 1, 2, 129, 64),      # one row past a tile
    (1, 2, 4, 256, 128),     # whole tiles
    (2, 2, 2, 383, 128),     # MHA, tail of 127
])
def test_causal_attention_matches_oracle(kivi, B, Hkv, Hq, S, D):
    q, k, v = _inputs(B, Hkv, Hq, S, D, seed=S + D)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = kivi.kivi_causal_attention(q.cuda(), k.cuda(), v.cuda(), status=status).cpu().numpy()
    qb, kb, vb = synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v)
    expect = O.prefill_attention(qb, kb, vb)
    expect_abs = O.prefill_attention(qb, kb, _abs_bits(vb))
    _assert_within_weight_rounding(got, expect, expect_abs, f"B{B} Hkv{Hkv} Hq{Hq} S{S} D{D}")
    assert int(status.item()) == 0


@pytest.mark.parametrize("sm_scale,k_growth", [(1.0, 0.02), (0.3, 0.0), (2.0, 0.05)])
def test_rising_scores_rescale_the_output(kivi, sm_scale, k_growth):
    """Row maxima that grow by far more than 2^8 across key tiles (the output is
    rescaled in TMEM) and strongly peaked rows."""
    B, Hkv, Hq, S, D = 1, 1, 2, 520, 128
    q, k, v = _inputs(B, Hkv, Hq, S, D, seed=7, k_growth=k_growth)
    got = kivi.kivi_causal_attention(q.cuda(), k.cuda(), v.cuda(), sm_scale=sm_scale)
    qb, kb, vb = synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v)
    expect = O.prefill_attention(qb, kb, vb, sm_scale)
    expect_abs = O.prefill_attention(qb, kb, _abs_bits(vb), sm_scale)
    _assert_within_weight_rounding(got.cpu().numpy(), expect, expect_abs,
                                   f"sm_scale {sm_scale} growth {k_growth}")


@pytest.mark.parametrize("S,D,bits", [(1, 64, 2), (127, 128, 2), (160, 128, 4), (161, 64, 2),
                                      (300, 128, 2), (513, 128, 4), (640, 64, 4)])
def test_fused_prefill_fills_the_cache(kivi, S, D, bits):
    """The fused prefill leaves the oracle's cache (records and ring byte for byte),
    and the decode step after it matches the oracle's."""
    B, Hkv, Hq = 2, 2, 4
    q, k, v = _inputs(B, Hkv, Hq, S, D, seed=S * 3 + bits)
    cache = kivi.KiviCache(batch=B, num_layers=2, num_kv_heads=Hkv, num_q_heads=Hq,
                           head_dim=D, bits=bits, max_tokens=S + 1)
    ref = O.OracleCache(B, Hkv, D, bits, S + 1)
    qb, kb, vb = synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v)
    got = cache.prefill_attention(1, q.cuda(), k.cuda(), v.cuda()).cpu().numpy()
    ref.prefill(kb, vb)
    torch.cuda.synchronize()
    assert_state_equal(cache, 1, ref, f"fused prefill S={S} D={D} b={bits}")
    _assert_within_weight_rounding(got, O.prefill_attention(qb, kb, vb),
                                   O.prefill_attention(qb, kb, _abs_bits(vb)), f"S={S}")
    gen = torch.Generator().manual_seed(S)
    kn = torch.randn(B, Hkv, D, generator=gen).to(torch.bfloat16)
    vn = torch.randn(B, Hkv, D, generator=gen).to(torch.bfloat16)
    qn = torch.randn(B, Hq, D, generator=gen).to(torch.bfloat16)
    cache.append(1, kn.cuda(), vn.cuda())
    ref.append(synth.bf16_bits(kn), synth.bf16_bits(vn))
    assert_attention_close(cache.attend(1, qn.cuda()).cpu().numpy(),
                           ref.attention(synth.bf16_bits(qn)), "decode after fused prefill")
    assert cache.check_device_status() == 0
    # a second prefill of a filled layer is refused
    with pytest.raises(kivi.KiviError) as e:
        cache.prefill_attention(1, q.cuda(), k.cuda(), v.cuda())
    assert e.value.status == "KIVI_ERR_STATE"
    cache.close()


def test_llama3_8b_gqa_8k_prompt_sampled_rows(kivi):
    """The Llama-3-8B GQA shape (Hkv 8, Hq 32, D 128) at an 8K prompt, 2 sequences:
    sampled positions of every head against the oracle's attention over the prefix,
    and the fused cache byte for byte equal to the separate quantize path's."""
    B, Hkv, Hq, S, D = 2, 8, 32, 8192, 128
    q, k, v = _inputs(B, Hkv, Hq, S, D, seed=11)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    fused = kivi.KiviCache(batch=B, num_layers=1, num_kv_heads=Hkv, num_q_heads=Hq,
                           head_dim=D, bits=2, max_tokens=S)
    out = fused.prefill_attention(0, qd, kd, vd)
    separate = kivi.KiviCache(batch=B, num_layers=1, num_kv_heads=Hkv, num_q_heads=Hq,
                              head_dim=D, bits=2, max_tokens=S)
    separate.prefill(0, kd, vd)
    torch.cuda.synchronize()
    assert torch.equal(fused.records_view(0), separate.records_view(0))
    NG = fused.length(0)[1]
    for which in ("k", "v"):
        for t in range(NG * O.G, S):
            slot = t % (O.R + O.G)
            assert torch.equal(fused.ring_view(which, 0)[:, :, slot],
                               separate.ring_view(which, 0)[:, :, slot])
    kb, vb = synth.bf16_bits(k), synth.bf16_bits(v)
    for b, i in [(0, 0), (0, 127), (1, 128), (0, 4095), (1, 5000), (0, 8191), (1, 8191)]:
        qi = synth.bf16_bits(q[b:b + 1, :, i])
        expect = O.attention_bf16(kb[b:b + 1], vb[b:b + 1], qi, S=i + 1)
        expect_abs = O.attention_bf16(kb[b:b + 1], _abs_bits(vb[b:b + 1]), qi, S=i + 1)
        _assert_within_weight_rounding(out[b:b + 1, :, i].cpu().numpy(), expect, expect_abs,
                                       f"sequence {b} position {i}")
    assert fused.check_device_status() == 0
    fused.close()
    separate.close()
