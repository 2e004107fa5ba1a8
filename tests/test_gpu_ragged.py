"""Ragged batches: a prompt length per sequence (needs a B200).

Each sequence of the GPU cache is checked against its own single-sequence oracle
cache: its group records byte for byte (groups aligned to its own token 0), its
live ring slots, and its attention rows within abs 2e-3 + rel 2e-3, after the
ragged prefill and after every append (each sequence flushes on its own
schedule).
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from gpu_util import assert_attention_close, load_kivi

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kivi():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return load_kivi()


def _check_states(cache, layer, refs, what):
    recs = cache.records_view(layer).cpu().numpy()
    ring_k = synth.bf16_bits(cache.ring_view("k", layer).cpu())
    ring_v = synth.bf16_bits(cache.ring_view("v", layer).cpu())
    assert cache.lengths(layer) == [r.S for r in refs], what
    for b, ref in enumerate(refs):
        if ref.NG:
            assert np.array_equal(recs[b, :, :ref.NG], ref.records[0, :, :ref.NG]), \
                f"{what}: records of sequence {b}"
        for t in range(ref.NG * O.G, ref.S):
            slot = t % (O.R + O.G)
            assert np.array_equal(ring_k[b, :, slot], ref.ring_k[0, :, slot]), f"{what} k {b} {t}"
            assert np.array_equal(ring_v[b, :, slot], ref.ring_v[0, :, slot]), f"{what} v {b} {t}"


def _run(K, lengths, Hkv, Hq, D, bits, steps, seed, check_every=1):
    gen = torch.Generator().manual_seed(seed)
    B, Smax = len(lengths), max(max(lengths), 1)
    max_tokens = Smax + steps
    scale = torch.exp(torch.randn(Hkv, D, generator=gen))[None, :, None, :]
    k = (torch.randn(B, Hkv, Smax, D, generator=gen) * scale).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Smax, D, generator=gen).to(torch.bfloat16)
    cache = K.KiviCache(batch=B, num_layers=2, num_kv_heads=Hkv, num_q_heads=Hq, head_dim=D,
                        bits=bits, max_tokens=max_tokens)
    layer = 1
    cache.prefill_ragged(layer, k.cuda(), v.cuda(), lengths)
    refs = []
    for b, n in enumerate(lengths):
        ref = O.OracleCache(1, Hkv, D, bits, max_tokens)
        if n:
            ref.prefill(synth.bf16_bits(k[b:b + 1, :, :n]), synth.bf16_bits(v[b:b + 1, :, :n]))
        refs.append(ref)
    torch.cuda.synchronize()
    _check_states(cache, layer, refs, "after the ragged prefill")
    for step in range(steps):
        kn = (torch.randn(B, Hkv, D, generator=gen) * scale[:, :, 0, :]).to(torch.bfloat16)
        vn = torch.randn(B, Hkv, D, generator=gen).to(torch.bfloat16)
        cache.append(layer, kn.cuda(), vn.cuda())
        for b, ref in enumerate(refs):
            ref.append(synth.bf16_bits(kn[b:b + 1]), synth.bf16_bits(vn[b:b + 1]))
        if step % check_every and step != steps - 1:
            continue
        q = torch.randn(B, Hq, D, generator=gen).to(torch.bfloat16)
        got = cache.attend(layer, q.cuda()).cpu().numpy()
        qb = synth.bf16_bits(q)
        expect = np.concatenate([ref.attention(qb[b:b + 1]) for b, ref in enumerate(refs)])
        assert_attention_close(got, expect, f"ragged step {step} lengths {[r.S for r in refs]}")
        _check_states(cache, layer, refs, f"after append {step}")
    assert cache.check_device_status() == 0
    cache.close()


def test_ragged_prefill_appends_and_decode(kivi):
    """Lengths on both sides of R, R + G and a group edge, one empty sequence; 40 steps
    cross every sequence's next flush."""
    _run(kivi, [0, 1, 127, 159, 161, 700], Hkv=2, Hq=8, D=64, bits=2, steps=40, seed=1,
         check_every=5)


def test_ragged_4bit_mha(kivi):
    _run(kivi, [300, 2000, 33], Hkv=2, Hq=2, D=128, bits=4, steps=3, seed=2)


def test_ragged_many_sequences(kivi):
    """64 sequences of random lengths: CTAs whose ranges hold only the empty items of
    short sequences, and pairs split across CTAs."""
    rng = np.random.default_rng(3)
    lengths = [int(x) for x in rng.integers(1, 900, 64)]
    _run(kivi, lengths, Hkv=4, Hq=16, D=128, bits=2, steps=2, seed=3)


def test_ragged_decode_needs_a_token_per_sequence(kivi):
    B, Hkv, D = 2, 1, 64
    cache = kivi.KiviCache(batch=B, num_layers=1, num_kv_heads=Hkv, num_q_heads=1, head_dim=D,
                           bits=2, max_tokens=64)
    k = torch.zeros(B, Hkv, 4, D, dtype=torch.bfloat16, device="cuda")
    cache.prefill_ragged(0, k, k, [0, 4])
    with pytest.raises(kivi.KiviError) as e:
        cache.attend(0, torch.zeros(B, 1, D, dtype=torch.bfloat16, device="cuda"))
    assert e.value.status == "KIVI_ERR_STATE"
    assert cache.lengths(0) == [0, 4]
    cache.close()


def test_ragged_shorter_sequence_has_more_items(kivi):
    """After one append the 862-token sequence (22 groups, 158 residual tokens) has more
    work items than the 878-token one (23 groups, 142 residual tokens): the split must
    give every pair the larger count."""
    _run(kivi, [877, 861, 5], Hkv=2, Hq=8, D=128, bits=2, steps=2, seed=4)
