"""The quantizer's degenerate cases and wide-range inputs on the GPU path (needs a B200).

The random-normal workloads never produce an exact .5 tie or a constant group,
so these cases build them on purpose and push them through prefill, append
(with a residual flush) and decode attention, on the GPU and in the oracle side
by side:

* constant key channels and constant value blocks: scale 0, every code 0, the
  group dequantizes to its min (the reading for max == min);
* inputs on the quantization grid mn + c * 2^e with both ends present: the
  dequantized cache equals the input exactly, so attention must also equal the
  textbook softmax attention over the original tensors;
* exact ties x = mn + (c + 1/2) * scale (exact in bf16): round half to even;
* wide dynamic range: key outlier channels x100, values of 1e-3 and 1e2 in one
  sequence, a strongly peaked softmax, query heads of very different norms.

Records are compared byte for byte; attention within abs 2e-3 + rel 2e-3 of
the oracle ("KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache":
keys per channel, values per token; record "kv-efficiency/kivi-2bit-llama3-8b-
gqa-8k", "Methodology": group size 32, residual 128).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import assert_attention_close, load_kivi, run_sequence

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kivi():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return load_kivi()


def _split_steps(k, v, S0):
    """Full bf16 sequences [B][Hkv][S][D] -> prefill part and per-token append steps."""
    steps = [(k[:, :, t].contiguous(), v[:, :, t].contiguous()) for t in range(S0, k.shape[2])]
    return k[:, :, :S0].contiguous(), v[:, :, :S0].contiguous(), steps


def _queries(gen, n, B, Hq, D, scale=1.0):
    return [(torch.randn(B, Hq, D, generator=gen) * scale).to(torch.bfloat16) for _ in range(n)]


def _textbook(q, k, v, scale):
    """Softmax attention in float64 over bf16 K/V [B][Hkv][S][D], GQA by consecutive heads."""
    B, Hq, D = q.shape
    Hkv = k.shape[1]
    kr = k.double().repeat_interleave(Hq // Hkv, dim=1)
    vr = v.double().repeat_interleave(Hq // Hkv, dim=1)
    s = torch.einsum("bhd,bhsd->bhs", q.double(), kr) * scale
    return torch.einsum("bhs,bhsd->bhd", torch.softmax(s, dim=-1), vr).numpy()


# S0 = 224 leaves NG = 3 groups and 128 ring tokens; the 32nd append (S = 255 -> 256)
# flushes ring tokens 96..127 into group 3.
S0_FLUSH, STEPS_FLUSH = 224, 34


# ---------------------------------------------------------------------------
# Constant groups
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("D,Hq", [(128, 8), (64, 4)])
def test_constant_groups(kivi, bits, D, Hq):
    gen = torch.Generator().manual_seed(100 + bits + D)
    B, Hkv = 2, 2
    S = S0_FLUSH + STEPS_FLUSH
    k = torch.randn(B, Hkv, S, D, generator=gen)
    v = torch.randn(B, Hkv, S, D, generator=gen)
    const_ch = torch.arange(D) % 3 == 0
    k[:, :, :, const_ch] = torch.randn(B, Hkv, 1, int(const_ch.sum()), generator=gen)
    v[:, :, :, 32:64] = torch.randn(B, Hkv, S, 1, generator=gen)  # block 1 constant per token
    k[1], v[1] = 0.75, -1.25  # sequence 1: every group constant, every scale 0
    k, v = k.to(torch.bfloat16), v.to(torch.bfloat16)
    kp, vp, steps = _split_steps(k, v, S0_FLUSH)
    outs = run_sequence(kivi, kp, vp, steps, _queries(gen, len(steps), B, Hq, D), bits, Hq=Hq,
                        what=f"constant groups b={bits} D={D}")
    for out, _ in outs:  # a constant cache attends to its constant value exactly
        assert np.all(np.abs(out[1] + 1.25) <= 2e-3 + 2e-3 * 1.25)


def test_constant_groups_records_have_zero_scale(kivi):
    """The oracle's record of a constant key channel holds scale 0 and min = the value;
    the GPU record is byte-identical (checked in run_sequence), so it does too."""
    tile = np.full((32, 64), 0x3F40, np.uint16)  # bf16 0.75
    rec = O.make_record(tile, tile, 2)
    k_hat, v_hat = O.dequant_record(rec, 64, 2)
    assert np.all(k_hat == 0.75) and np.all(v_hat == 0.75)


# ---------------------------------------------------------------------------
# Inputs on the quantization grid
# ---------------------------------------------------------------------------

def _grid(gen, B, Hkv, S, D, bits, axis):
    """Every quantization group on its grid mn + c * 2^e with c = 0 and c = 2^b - 1
    present: exact in bf16 and fp16, so the quantizer reproduces it exactly."""
    qmax = (1 << bits) - 1
    c = torch.randint(0, qmax + 1, (B, Hkv, S, D), generator=gen).double()
    if axis == "k":  # per channel over 32-token groups aligned to token 0
        c[:, :, 0::32, :], c[:, :, 1::32, :] = 0, qmax
        shape = (B, Hkv, S // 32 + 1, 1, D)
        step = 2.0 ** torch.randint(-3, 2, shape, generator=gen).double()
        mn = step * torch.randint(-8, 8, shape, generator=gen).double()
        step = step.repeat_interleave(32, dim=2).reshape(B, Hkv, -1, D)[:, :, :S]
        mn = mn.repeat_interleave(32, dim=2).reshape(B, Hkv, -1, D)[:, :, :S]
    else:  # per token over 32-channel blocks
        c[..., 0::32], c[..., 1::32] = 0, qmax
        shape = (B, Hkv, S, D // 32, 1)
        step = 2.0 ** torch.randint(-3, 2, shape, generator=gen).double()
        mn = step * torch.randint(-8, 8, shape, generator=gen).double()
        step = step.expand(B, Hkv, S, D // 32, 32).reshape(B, Hkv, S, D)
        mn = mn.expand(B, Hkv, S, D // 32, 32).reshape(B, Hkv, S, D)
    x = mn + step * c
    assert torch.equal(x.to(torch.bfloat16).double(), x)
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("Hkv,Hq", [(2, 8), (4, 4)])
def test_grid_inputs_attend_like_the_textbook(kivi, bits, Hkv, Hq):
    gen = torch.Generator().manual_seed(200 + bits + Hq)
    B, D = 2, 128
    S = S0_FLUSH + STEPS_FLUSH
    k = _grid(gen, B, Hkv, S, D, bits, "k")
    v = _grid(gen, B, Hkv, S, D, bits, "v")
    kp, vp, steps = _split_steps(k, v, S0_FLUSH)
    qs = _queries(gen, len(steps), B, Hq, D)
    outs = run_sequence(kivi, kp, vp, steps, qs, bits, Hq=Hq, what=f"grid b={bits}")
    for i, (out, _) in enumerate(outs):
        n = S0_FLUSH + i + 1
        expect = _textbook(qs[i], k[:, :, :n], v[:, :, :n], 1.0 / math.sqrt(D))
        assert_attention_close(out, expect, f"grid vs textbook S={n}")


# ---------------------------------------------------------------------------
# Exact ties
# ---------------------------------------------------------------------------

def _ties(gen, B, Hkv, S, D, bits, axis):
    """Groups whose values are mn + step * h/2 for h in 0..2 qmax with both ends
    present, so (x - mn) / scale lands exactly on .5 for odd h."""
    qmax = (1 << bits) - 1
    h = torch.randint(0, 2 * qmax + 1, (B, Hkv, S, D), generator=gen).double()
    if axis == "k":
        h[:, :, 0::32, :], h[:, :, 1::32, :] = 0, 2 * qmax
        h[:, :, 2::32, :] = 1  # a .5 tie that rounds down to 0 (even)
        h[:, :, 3::32, :] = 3  # 1.5 -> 2
    else:
        h[..., 0::32], h[..., 1::32] = 0, 2 * qmax
        h[..., 2::32], h[..., 3::32] = 1, 3
    step = 2.0 ** torch.randint(-2, 2, (B, Hkv, 1, 1), generator=gen).double()
    mn = step * torch.randint(-4, 4, (B, Hkv, 1, 1), generator=gen).double()
    x = mn + step * h / 2
    assert torch.equal(x.to(torch.bfloat16).double(), x)
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("bits", [2, 4])
def test_exact_ties_round_half_to_even(kivi, bits):
    gen = torch.Generator().manual_seed(300 + bits)
    B, Hkv, Hq, D = 2, 2, 8, 128
    S = S0_FLUSH + STEPS_FLUSH
    k = _ties(gen, B, Hkv, S, D, bits, "k")
    v = _ties(gen, B, Hkv, S, D, bits, "v")
    kp, vp, steps = _split_steps(k, v, S0_FLUSH)
    run_sequence(kivi, kp, vp, steps, _queries(gen, len(steps), B, Hq, D), bits, Hq=Hq,
                 what=f"ties b={bits}")
    # the oracle (whose records the GPU's equal byte for byte) rounds those ties to even
    qmax = (1 << bits) - 1
    x = np.array([0.0, qmax, 0.5, 1.5] + [0.0] * 28, np.float32)
    _, _, codes = O.quantize_group(x, bits)
    assert list(codes[:4]) == [0, qmax, 0, 2]


# ---------------------------------------------------------------------------
# Wide dynamic range
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 4])
def test_key_outlier_channels_x100(kivi, bits):
    gen = torch.Generator().manual_seed(400 + bits)
    B, Hkv, Hq, D = 2, 2, 8, 128
    S = 1000 + 25  # the 24th append flushes a group
    sk = torch.ones(Hkv, D)
    for h in range(Hkv):
        sk[h, torch.randperm(D, generator=gen)[:4]] = 100.0
    k = (torch.randn(B, Hkv, S, D, generator=gen) * sk[None, :, None, :]).to(torch.bfloat16)
    v = torch.randn(B, Hkv, S, D, generator=gen).to(torch.bfloat16)
    kp, vp, steps = _split_steps(k, v, 1000)
    run_sequence(kivi, kp, vp, steps, _queries(gen, len(steps), B, Hq, D), bits, Hq=Hq,
                 check_state=False, what=f"outliers x100 b={bits}")


def test_values_1e_minus_3_next_to_1e2(kivi):
    gen = torch.Generator().manual_seed(500)
    B, Hkv, Hq, D = 2, 2, 8, 128
    S = 700 + 3
    k = torch.randn(B, Hkv, S, D, generator=gen).to(torch.bfloat16)
    mag = torch.tensor([1e-3, 1.0, 1e2])[torch.randint(0, 3, (B, Hkv, S, D // 32), generator=gen)]
    v = torch.randn(B, Hkv, S, D // 32, 32, generator=gen) * mag[..., None]
    v = v.reshape(B, Hkv, S, D).to(torch.bfloat16)
    kp, vp, steps = _split_steps(k, v, 700)
    run_sequence(kivi, kp, vp, steps, _queries(gen, len(steps), B, Hq, D), 2, Hq=Hq,
                 check_state=False, what="values 1e-3 and 1e2")


@pytest.mark.parametrize("sm_scale", [2.0, 4.0])
def test_peaked_softmax(kivi, sm_scale):
    """One key per sequence aligned with the query (in the quantized history for
    sequence 0, in the residual for sequence 1): the softmax is nearly one-hot."""
    gen = torch.Generator().manual_seed(600 + int(sm_scale))
    B, Hkv, Hq, D = 2, 2, 4, 64
    S0 = 600
    q = (torch.randn(B, Hq, D, generator=gen) * 0.5).to(torch.bfloat16)
    k = torch.randn(B, Hkv, S0 + 1, D, generator=gen) * 0.5
    v = torch.randn(B, Hkv, S0 + 1, D, generator=gen)
    for h in range(Hkv):
        k[0, h, 77] = q[0, 2 * h].float()       # quantized group 2
        k[1, h, S0 - 5] = q[1, 2 * h].float()   # residual ring
    k, v = k.to(torch.bfloat16), v.to(torch.bfloat16)
    kp, vp, steps = _split_steps(k, v, S0)
    run_sequence(kivi, kp, vp, steps, [q], 2, Hq=Hq, sm_scale=sm_scale, check_state=False,
                 what=f"peaked softmax sm_scale={sm_scale}")


def test_query_heads_of_very_different_norms(kivi):
    gen = torch.Generator().manual_seed(700)
    B, Hkv, Hq, D = 2, 2, 8, 128
    S0 = 900
    k = (torch.randn(B, Hkv, S0 + 1, D, generator=gen)
         * torch.exp(torch.randn(Hkv, D, generator=gen))[None, :, None, :]).to(torch.bfloat16)
    v = torch.randn(B, Hkv, S0 + 1, D, generator=gen).to(torch.bfloat16)
    q = torch.randn(B, Hq, D, generator=gen)
    q[:, 0::4] *= 30.0    # large-norm heads
    q[:, 1::4] *= 1e-3    # tiny heads next to them
    kp, vp, steps = _split_steps(k, v, S0)
    run_sequence(kivi, kp, vp, steps, [q.to(torch.bfloat16)], 2, Hq=Hq, check_state=False,
                 what="query norms 30 and 1e-3")
