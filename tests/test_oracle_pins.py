"""Pins of the CPU oracle to things other than itself (CPU only).

Each test checks the oracle against a value the pages print, a hand-worked
value, a closed form, an invariant, an independent library routine, or brute
force, chosen so that a dropped term, a wrong index or sign, or a transposed
operand in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bits(x: torch.Tensor) -> np.ndarray:
    return synth.bf16_bits(x.to(torch.bfloat16))


# ---------------------------------------------------------------------------
# Number formats: the oracle's fp16 rounding against numpy's (independent)
# ---------------------------------------------------------------------------

@pytest.mark.filterwarnings("ignore:overflow encountered")
def test_f32_to_f16_matches_numpy():
    rng = np.random.default_rng(1)
    xs = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * np.float32(10.0) ** rng.integers(-9, 5, 4000),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 7e4, 6.1035156e-05, 5.9604645e-08,
                  2.9802322e-08, 2.98023224e-08 * 1.5, 1.0 + 2.0**-11, 1.0 + 3 * 2.0**-11,
                  -2.5, 1e-8, 3.0e-5], np.float32),
    ])
    for x in xs:
        expect = int(np.float32(x).astype(np.float16).view(np.uint16))
        assert O.f32_to_f16_bits(float(x)) == expect, x


def test_f16_to_double_matches_numpy():
    for h in list(range(0, 0x7C00, 37)) + [0x0001, 0x03FF, 0x0400, 0x3C00, 0x7BFF, 0x8001, 0xBC00]:
        assert O.f16_bits_to_double(h) == float(np.uint16(h).view(np.float16))


# ---------------------------------------------------------------------------
# Quantizer
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 4])
def test_grid_inputs_round_trip_exactly(bits):
    qmax = (1 << bits) - 1
    ks = np.arange(32) % (qmax + 1)
    x = (-1.5 + 0.5 * ks).astype(np.float32)
    scale, mn, codes = O.quantize_group(x, bits)
    assert scale == np.float32(0.5) and mn == np.float32(-1.5)
    assert np.array_equal(codes, ks)


@pytest.mark.parametrize("bits", [2, 4])
def test_ties_round_half_to_even(bits):
    qmax = (1 << bits) - 1
    x = np.zeros(32, np.float32)
    x[1] = qmax  # scale = 1, min = 0
    ties = np.arange(qmax) + 0.5
    x[2:2 + qmax] = ties
    _, _, codes = O.quantize_group(x, bits)
    expect = [int(2 * round(t / 2)) if (t - 0.5) % 2 == 0 else int(t + 0.5) for t in ties]
    # half-even: 0.5->0, 1.5->2, 2.5->2, 3.5->4 ...
    assert list(codes[2:2 + qmax]) == [int(np.round(t)) for t in ties] == expect


def test_constant_group():
    x = np.full(32, 1.25, np.float32)
    scale, mn, codes = O.quantize_group(x, 2)
    assert scale == 0.0 and mn == np.float32(1.25) and not codes.any()


@pytest.mark.parametrize("bits", [2, 4])
def test_codes_equal_nearest_level_brute_force(bits):
    """The code is the nearest of the 2^b levels mn + c*scale (brute force over c),
    except within 1e-4 of a tie; min maps to 0, max to 2^b-1; codes are monotone."""
    rng = np.random.default_rng(bits)
    qmax = (1 << bits) - 1
    for trial in range(300):
        x = (rng.standard_normal(32) * rng.choice([1e-3, 1.0, 30.0])).astype(np.float32)
        x = torch.tensor(x).to(torch.bfloat16).float().numpy()
        scale, mn, codes = O.quantize_group(x, bits)
        levels = float(mn) + float(scale) * np.arange(qmax + 1)
        nearest = np.abs(x[:, None].astype(np.float64) - levels[None, :]).argmin(axis=1)
        t = (x.astype(np.float64) - float(mn)) / float(scale)
        near_tie = np.abs(t - np.floor(t) - 0.5) < 1e-4
        assert np.array_equal(codes[~near_tie], nearest[~near_tie])
        assert codes[np.argmin(x)] == 0 and codes[np.argmax(x)] == qmax
        order = np.argsort(x, kind="stable")
        assert np.all(np.diff(codes[order].astype(int)) >= 0)
        # error bound with the fp32 parameters: |x - (scale*c + mn)| <= scale/2 (+ fp32 slack)
        err = np.abs(x.astype(np.float64) - (float(scale) * codes + float(mn)))
        assert np.all(err <= float(scale) * (0.5 + 2.0**-20) + 1e-30)


@pytest.mark.parametrize("bits", [2, 4])
def test_error_bound_with_fp16_metadata(bits):
    """|x - x_hat| <= scale/2 + |mn - mn_h| + c*|scale - scale_h| with the stored fp16 pair."""
    rng = np.random.default_rng(10 + bits)
    D = 64
    k = torch.tensor(rng.standard_normal((32, D)) * 3).to(torch.bfloat16)
    v = torch.tensor(rng.standard_normal((32, D))).to(torch.bfloat16)
    rec = O.make_record(_bits(k), _bits(v), bits)
    k_hat, v_hat = O.dequant_record(rec, D, bits)
    kf, vf = k.double().numpy(), v.double().numpy()
    for d in range(D):
        scale, mn, codes = O.quantize_group(k.float().numpy()[:, d], bits)
        sh = O.f16_bits_to_double(O.f32_to_f16_bits(float(scale)))
        mh = O.f16_bits_to_double(O.f32_to_f16_bits(float(mn)))
        bound = float(scale) * (0.5 + 2.0**-20) + abs(float(mn) - mh) + codes * abs(float(scale) - sh)
        assert np.all(np.abs(kf[:, d] - k_hat[:, d]) <= bound + 1e-12)
    for t in range(32):
        for j in range(0, D, 32):
            scale, mn, codes = O.quantize_group(v.float().numpy()[t, j:j + 32], bits)
            sh = O.f16_bits_to_double(O.f32_to_f16_bits(float(scale)))
            mh = O.f16_bits_to_double(O.f32_to_f16_bits(float(mn)))
            bound = (float(scale) * (0.5 + 2.0**-20) + abs(float(mn) - mh)
                     + codes * abs(float(scale) - sh))
            assert np.all(np.abs(vf[t, j:j + 32] - v_hat[t, j:j + 32]) <= bound + 1e-12)


# ---------------------------------------------------------------------------
# Packed record layout (hand-worked words)
# ---------------------------------------------------------------------------

def _word(rec, byte_offset):
    return int.from_bytes(bytes(rec[byte_offset:byte_offset + 4]), "little")


def test_record_sizes():
    g = _golden("hand_worked.json")["packing"]["record_bytes"]
    assert O.record_bytes(128, 2) == g["D128_b2"]
    assert O.record_bytes(128, 4) == g["D128_b4"]
    assert O.record_bytes(64, 2) == g["D64_b2"]


@pytest.mark.parametrize("bits", [2, 4])
def test_packed_words_hand_worked(bits):
    g = _golden("hand_worked.json")["packing"]
    D = 128
    t = np.arange(32)[:, None]
    d = np.arange(D)[None, :]
    tile = ((t + d) % (1 << bits)).astype(np.float32)
    kb = _bits(torch.tensor(tile))
    rec = O.make_record(kb, kb, bits)
    row_bytes_k = D * bits // 8
    if bits == 2:
        assert _word(rec, 0) == int(g["2bit_k_row0_word0"], 16)
        assert _word(rec, row_bytes_k) == int(g["2bit_k_row1_word0"], 16)
    else:
        assert _word(rec, 0) == int(g["4bit_k_row0_word0"], 16)
        assert _word(rec, 16) == int(g["4bit_k_row0_word4"], 16)
        assert _word(rec, row_bytes_k) == int(g["4bit_k_row1_word0"], 16)
    kscale = 2 * 32 * row_bytes_k
    kmin, vscale = kscale + 2 * D, kscale + 4 * D
    vmin = vscale + 2 * D
    assert list(rec[kscale:kscale + 2]) == g["fp16_one_bytes"]
    assert list(rec[kmin:kmin + 2]) == g["fp16_zero_bytes"]
    assert list(rec[vscale:vscale + 2]) == g["fp16_one_bytes"]
    assert list(rec[vmin:vmin + 2]) == g["fp16_zero_bytes"]
    assert len(rec) == vmin + 2 * D
    k_hat, v_hat = O.dequant_record(rec, D, bits)
    assert np.array_equal(k_hat, tile) and np.array_equal(v_hat, tile)


@pytest.mark.parametrize("case", range(4))
def test_one_hot_positions_hand_worked(case):
    """A single non-zero code lands at the word, bit and metadata slot the layout
    definition gives (positions worked by hand in tests/golden/hand_worked.json)."""
    c = _golden("hand_worked.json")["one_hot"]["cases"][case]
    bits, i, d, D = c["bits"], c["i"], c["d"], 128
    tile = np.zeros((32, D), np.float32)
    tile[i, d] = (1 << bits) - 1
    tb = _bits(torch.tensor(tile))
    rec = O.make_record(tb, tb, bits)
    words = rec[:len(rec) - 8 * D].view("<u4")
    n_k = 32 * D * bits // 32
    kw, vw = words[:n_k], words[n_k:2 * n_k]
    assert np.count_nonzero(kw) == 1 and kw[c["k_word"]] == int(c["k_value"], 16)
    assert np.count_nonzero(vw) == 1 and vw[c["v_word"]] == int(c["v_value"], 16)
    meta = rec[len(rec) - 8 * D:].view("<u2")
    kscale, kmin, vscale, vmin = meta[:D], meta[D:2 * D], meta[2 * D:3 * D], meta[3 * D:]
    one = 0x3C00
    assert np.count_nonzero(kscale) == 1 and kscale[c["k_scale_f16_index"]] == one
    assert np.count_nonzero(vscale) == 1 and vscale[c["v_scale_f16_index"]] == one
    assert not kmin.any() and not vmin.any()
    k_hat, v_hat = O.dequant_record(rec, D, bits)
    assert np.array_equal(k_hat, tile) and np.array_equal(v_hat, tile)


def _grid_tile(rng, n_tok, D, bits, axis):
    """bf16 tile whose every quantization group lies on its grid mn + c*2^e with
    both ends present (exact in bf16 and fp16): groups per channel over 32 tokens
    (axis='k') or per token over 32 channels (axis='v')."""
    qmax = (1 << bits) - 1
    codes = rng.integers(0, qmax + 1, (n_tok, D))
    x = np.zeros((n_tok, D))
    if axis == "k":
        for g0 in range(0, n_tok, 32):
            for d in range(D):
                c = codes[g0:g0 + 32, d]
                c[0], c[1] = 0, qmax
                step = 2.0 ** int(rng.integers(-3, 2))
                mn = step * int(rng.integers(-8, 8))
                x[g0:g0 + 32, d] = mn + step * c
    else:
        for t in range(n_tok):
            for j in range(0, D, 32):
                c = codes[t, j:j + 32]
                c[0], c[1] = 0, qmax
                step = 2.0 ** int(rng.integers(-3, 2))
                mn = step * int(rng.integers(-8, 8))
                x[t, j:j + 32] = mn + step * c
    return torch.tensor(x, dtype=torch.float64)


@pytest.mark.parametrize("bits", [2, 4])
def test_grid_record_dequantizes_exactly(bits):
    rng = np.random.default_rng(3)
    D = 128
    k = _grid_tile(rng, 32, D, bits, "k")
    v = _grid_tile(rng, 32, D, bits, "v")
    rec = O.make_record(_bits(k), _bits(v), bits)
    k_hat, v_hat = O.dequant_record(rec, D, bits)
    assert np.array_equal(k_hat, k.numpy()) and np.array_equal(v_hat, v.numpy())


# ---------------------------------------------------------------------------
# Cache state rule
# ---------------------------------------------------------------------------

def test_num_groups_table():
    g = _golden("hand_worked.json")["num_groups"]
    assert [O.num_groups(s) for s in g["S"]] == g["NG"]
    for S in range(O.R, 2000):
        r = S - O.num_groups(S) * O.G
        assert O.R <= r < O.R + O.G


@pytest.mark.parametrize("S0,steps", [(0, 200), (100, 70), (159, 3), (190, 40)])
def test_prefill_plus_appends_equals_prefill(S0, steps):
    rng = np.random.default_rng(S0)
    B, H, D, bits = 2, 2, 64, 2
    S1 = S0 + steps
    k = _bits(torch.tensor(rng.standard_normal((B, H, S1, D))))
    v = _bits(torch.tensor(rng.standard_normal((B, H, S1, D))))
    a = O.OracleCache(B, H, D, bits, S1)
    a.prefill(k[:, :, :S0], v[:, :, :S0])
    for t in range(S0, S1):
        a.append(k[:, :, t], v[:, :, t])
    b = O.OracleCache(B, H, D, bits, S1)
    b.prefill(k, v)
    assert a.S == b.S == S1
    NG = O.num_groups(S1)
    assert np.array_equal(a.records[:, :, :NG], b.records[:, :, :NG])
    for t in range(NG * O.G, S1):
        slot = t % (O.R + O.G)
        assert np.array_equal(a.ring_k[:, :, slot], b.ring_k[:, :, slot])
        assert np.array_equal(a.ring_v[:, :, slot], b.ring_v[:, :, slot])


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def _sdpa(q, k, v, scale):
    """Textbook attention in float64 via torch: q [B][Hq][D], k/v [B][Hkv][S][D]."""
    rep = q.shape[1] // k.shape[1]
    k = k.double().repeat_interleave(rep, dim=1)
    v = v.double().repeat_interleave(rep, dim=1)
    out = torch.nn.functional.scaled_dot_product_attention(
        q.double()[:, :, None, :], k, v, scale=scale)
    return out[:, :, 0, :].numpy()


def test_attention_hand_worked():
    g = _golden("hand_worked.json")["attention"]
    D = 32
    k = torch.zeros(1, 1, 2, D)
    v = torch.zeros(1, 1, 2, D)
    q = torch.zeros(1, 1, D)
    q[0, 0, 0] = 1
    k[0, 0, 0, 0] = 1
    v[0, 0, 0, 0] = 1
    v[0, 0, 1, 1] = 1
    c = O.OracleCache(1, 1, D, 2, 2)
    c.prefill(_bits(k), _bits(v))
    out = c.attention(_bits(q), sm_scale=1.0)
    assert out[0, 0, 0] == pytest.approx(g["out0"], abs=1e-15)
    assert out[0, 0, 1] == pytest.approx(g["out1"], abs=1e-15)
    assert np.all(out[0, 0, 2:] == 0)


@pytest.mark.parametrize("S", [1, 37, 128])
def test_residual_only_equals_textbook(S):
    rng = np.random.default_rng(S)
    B, Hkv, Hq, D = 2, 2, 4, 64
    k = torch.tensor(rng.standard_normal((B, Hkv, S, D))).to(torch.bfloat16)
    v = torch.tensor(rng.standard_normal((B, Hkv, S, D))).to(torch.bfloat16)
    q = torch.tensor(rng.standard_normal((B, Hq, D))).to(torch.bfloat16)
    c = O.OracleCache(B, Hkv, D, 2, S)
    c.prefill(_bits(k), _bits(v))
    out = c.attention(_bits(q))
    np.testing.assert_allclose(out, _sdpa(q, k, v, 1 / math.sqrt(D)), rtol=0, atol=1e-12)


@pytest.mark.parametrize("bits,S,Hq", [(2, 300, 4), (4, 261, 2), (2, 545, 2), (2, 200, 8)])
def test_grid_cache_attention_equals_textbook(bits, S, Hq):
    """Keys/values on their quantization grids dequantize exactly, so attention
    over the packed cache (groups plus residual, GQA mapping) must equal plain
    attention over the original tensors."""
    rng = np.random.default_rng(bits * 1000 + S)
    B, Hkv, D = 2, 2, 64
    k = torch.zeros(B, Hkv, S, D, dtype=torch.float64)
    v = torch.zeros(B, Hkv, S, D, dtype=torch.float64)
    n_q = (S // 32) * 32
    for b in range(B):
        for h in range(Hkv):
            k[b, h, :n_q] = _grid_tile(rng, n_q, D, bits, "k")
            v[b, h, :n_q] = _grid_tile(rng, n_q, D, bits, "v")
            k[b, h, n_q:] = torch.tensor(rng.standard_normal((S - n_q, D)))
            v[b, h, n_q:] = torch.tensor(rng.standard_normal((S - n_q, D)))
    k, v = k.to(torch.bfloat16), v.to(torch.bfloat16)
    q = torch.tensor(rng.standard_normal((B, Hq, D)) * 0.3).to(torch.bfloat16)
    c = O.OracleCache(B, Hkv, D, bits, S)
    c.prefill(_bits(k), _bits(v))
    assert c.NG == O.num_groups(S) > 0
    np.testing.assert_allclose(c.attention(_bits(q)), _sdpa(q, k, v, 1 / math.sqrt(D)),
                               rtol=0, atol=1e-12)
    for b, h in [(0, 0), (1, Hq - 1)]:
        np.testing.assert_array_equal(c.attend(b, h, _bits(q)[b, h], Hq),
                                      c.attention(_bits(q))[b, h])


def test_identical_keys_give_mean_of_values():
    rng = np.random.default_rng(7)
    D, S = 64, 200
    k = torch.tensor(rng.standard_normal(D)).to(torch.bfloat16).expand(1, 1, S, D).contiguous()
    v = _grid_tile(rng, S, D, 2, "v")[None, None].to(torch.bfloat16)
    q = torch.tensor(rng.standard_normal((1, 1, D))).to(torch.bfloat16)
    c = O.OracleCache(1, 1, D, 2, S)
    c.prefill(_bits(k), _bits(v))
    # constant key groups: scale 0, dequantized key = fp16(min) = the key itself
    np.testing.assert_allclose(c.attention(_bits(q))[0, 0], v.double().numpy()[0, 0].mean(0),
                               rtol=0, atol=1e-12)


def test_dominant_score_selects_its_value():
    D, S = 64, 300
    rng = np.random.default_rng(8)
    k = torch.tensor(rng.standard_normal((1, 1, S, D)) * 0.01).to(torch.bfloat16)
    k[0, 0, 250, :] = 4.0  # NG(300) = 5 groups cover tokens [0, 160); 250 is residual
    v = torch.tensor(rng.standard_normal((1, 1, S, D))).to(torch.bfloat16)
    q = torch.full((1, 1, D), 4.0).to(torch.bfloat16)
    c = O.OracleCache(1, 1, D, 2, S)
    c.prefill(_bits(k), _bits(v))
    np.testing.assert_allclose(c.attention(_bits(q))[0, 0], v.double().numpy()[0, 0, 250],
                               atol=1e-9)


# ---------------------------------------------------------------------------
# The pages' byte arithmetic
# ---------------------------------------------------------------------------

def test_cache_bytes_match_pages():
    g = _golden("cache_bytes.json")
    sk = g["llama3_8b_skeleton"]
    b2 = O.cache_bytes(sk["num_layers"], sk["num_kv_heads"], sk["head_dim"], 2, sk["context"])
    b4 = O.cache_bytes(sk["num_layers"], sk["num_kv_heads"], sk["head_dim"], 4, sk["context"])
    res = b2["convention"] - g["grouped_2bit_per_token"]
    assert res == g["residual_per_token"]
    assert res * sk["context"] == g["residual_total_bytes_R128"]
    assert b2["convention"] == g["convention_2bit_per_token"]
    assert b2["bf16"] == g["bf16_per_token"]
    assert round(b2["bf16"] / b2["convention"], 2) == g["convention_2bit_ratio"]
    assert b2["codes_only"] == g["codes_only_2bit_per_token"]
    assert round(b2["bf16"] / b2["codes_only"], 2) == g["codes_only_2bit_ratio"]
    assert b4["convention"] - res == g["grouped_4bit_per_token"]
    assert b4["convention"] == g["convention_4bit_per_token"]
    assert round(b4["bf16"] / b4["convention"], 2) == g["convention_4bit_ratio"]
    flat = b2["bf16"] / (b2["convention"] - res)
    assert flat == g["flat_2bit_vs_fp16_ratio"]
    # stored bytes add the fp16 metadata: 8*D bytes per 32-token group record
    assert b2["stored"] == (252 * 32 * 8 * 3072 + 128 * 131072) / 8192
    llama2_7b = 32 * 32 * 128 * 2 * 2 * 10_000
    assert round(llama2_7b / 1e9) == g["llama2_7b_bf16_10k_tokens_gb_roughly"]


def test_per_channel_keys_beat_per_token_on_outlier_channels():
    """Keys with outlier channels quantize with a smaller error per channel than per
    token, the granularity argument of the KIVI and news pages (an assertion on
    synthetic keys, not a reproduction of the papers' accuracy)."""
    w = synth.WORKLOADS["tiny"]
    k, _ = synth.prefill_kv(w, 0, S=256)
    kf = k.float().numpy()[0, 0]  # [S][D]
    err_c, err_t = 0.0, 0.0
    for g0 in range(0, 256, 32):
        for d in range(kf.shape[1]):
            s, m, c = O.quantize_group(kf[g0:g0 + 32, d], 2)
            err_c += np.abs(kf[g0:g0 + 32, d] - (s * c + m)).sum()
    for t in range(256):
        for j in range(0, kf.shape[1], 32):
            s, m, c = O.quantize_group(kf[t, j:j + 32], 2)
            err_t += np.abs(kf[t, j:j + 32] - (s * c + m)).sum()
    assert err_c < err_t


# ---------------------------------------------------------------------------
# The 16-bit baseline: attention over an unquantized bf16 cache
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("B,Hkv,Hq,S,Smax,D", [(2, 2, 8, 77, 80, 64), (1, 3, 3, 1, 4, 128),
                                               (2, 1, 4, 300, 300, 128)])
def test_bf16_attention_equals_library_sdpa(B, Hkv, Hq, S, Smax, D):
    """Unused capacity (tokens S..Smax-1) holds NaN and must not reach the result."""
    rng = np.random.default_rng(S + D)
    k = torch.tensor(rng.standard_normal((B, Hkv, Smax, D))).to(torch.bfloat16)
    v = torch.tensor(rng.standard_normal((B, Hkv, Smax, D))).to(torch.bfloat16)
    k[:, :, S:] = float("nan")
    v[:, :, S:] = float("nan")
    q = torch.tensor(rng.standard_normal((B, Hq, D))).to(torch.bfloat16)
    out = O.attention_bf16(_bits(k), _bits(v), _bits(q), S)
    np.testing.assert_allclose(out, _sdpa(q, k[:, :, :S], v[:, :, :S], 1 / math.sqrt(D)),
                               rtol=0, atol=1e-12)


def test_bf16_attention_hand_worked():
    g = _golden("hand_worked.json")["attention"]
    D = 32
    k = torch.zeros(1, 1, 2, D)
    v = torch.zeros(1, 1, 2, D)
    q = torch.zeros(1, 1, D)
    q[0, 0, 0] = k[0, 0, 0, 0] = v[0, 0, 0, 0] = v[0, 0, 1, 1] = 1
    out = O.attention_bf16(_bits(k), _bits(v), _bits(q), sm_scale=1.0)
    assert out[0, 0, 0] == pytest.approx(g["out0"], abs=1e-15)
    assert out[0, 0, 1] == pytest.approx(g["out1"], abs=1e-15)
    assert np.all(out[0, 0, 2:] == 0)


@pytest.mark.parametrize("bits", [2, 4])
def test_bf16_attention_equals_quantized_cache_on_grid_inputs(bits):
    """On grid inputs the quantized cache dequantizes exactly, so the two oracles,
    which share only the final softmax loop, must agree."""
    rng = np.random.default_rng(40 + bits)
    B, Hkv, Hq, D, S = 1, 2, 4, 64, 290
    n_q = O.num_groups(S) * O.G
    k = torch.tensor(rng.standard_normal((B, Hkv, S, D)), dtype=torch.float64)
    v = torch.tensor(rng.standard_normal((B, Hkv, S, D)), dtype=torch.float64)
    for h in range(Hkv):
        k[0, h, :n_q] = _grid_tile(rng, n_q, D, bits, "k")
        v[0, h, :n_q] = _grid_tile(rng, n_q, D, bits, "v")
    k, v = k.to(torch.bfloat16), v.to(torch.bfloat16)
    q = torch.tensor(rng.standard_normal((B, Hq, D)) * 0.3).to(torch.bfloat16)
    c = O.OracleCache(B, Hkv, D, bits, S)
    c.prefill(_bits(k), _bits(v))
    np.testing.assert_allclose(O.attention_bf16(_bits(k), _bits(v), _bits(q)),
                               c.attention(_bits(q)), rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------
# Key-granularity ablation: per channel (KIVI) against per token
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 4])
def test_fake_quant_keys_matches_the_record_paths(bits):
    """Per channel is the record's key path; per token is the record's value path
    applied to the keys (both packed, stored and read back by the record code)."""
    rng = np.random.default_rng(bits)
    D = 128
    k = torch.tensor(rng.standard_normal((64, D)) * np.exp(rng.standard_normal(D))).to(
        torch.bfloat16)
    kb = _bits(k)
    per_c = O.fake_quant_keys(kb, bits, per_token=False)
    per_t = O.fake_quant_keys(kb, bits, per_token=True)
    for g0 in (0, 32):
        rec = O.make_record(kb[g0:g0 + 32], kb[g0:g0 + 32], bits)
        k_hat, v_hat = O.dequant_record(rec, D, bits)
        np.testing.assert_array_equal(per_c[g0:g0 + 32], k_hat)
        np.testing.assert_array_equal(per_t[g0:g0 + 32], v_hat)


@pytest.mark.parametrize("bits", [2, 4])
def test_fake_quant_keys_exact_on_its_own_grid(bits):
    rng = np.random.default_rng(50 + bits)
    kc = _grid_tile(rng, 64, 64, bits, "k")
    kt = _grid_tile(rng, 64, 64, bits, "v")
    assert np.array_equal(O.fake_quant_keys(_bits(kc), bits, False), kc.numpy())
    assert np.array_equal(O.fake_quant_keys(_bits(kt), bits, True), kt.numpy())
    # and the other granularity is not exact on them
    assert not np.array_equal(O.fake_quant_keys(_bits(kc), bits, True), kc.numpy())


# ---------------------------------------------------------------------------
# Prefill attention (causal), the step before the cache is filled
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("B,Hkv,Hq,S,D", [(1, 1, 1, 1, 64), (2, 2, 8, 70, 64), (1, 2, 2, 33, 128)])
def test_prefill_attention_equals_causal_sdpa(B, Hkv, Hq, S, D):
    rng = np.random.default_rng(S + Hq)
    q = torch.tensor(rng.standard_normal((B, Hq, S, D))).to(torch.bfloat16)
    k = torch.tensor(rng.standard_normal((B, Hkv, S, D))).to(torch.bfloat16)
    v = torch.tensor(rng.standard_normal((B, Hkv, S, D))).to(torch.bfloat16)
    out = O.prefill_attention(_bits(q), _bits(k), _bits(v))
    rep = Hq // Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double().repeat_interleave(rep, 1), v.double().repeat_interleave(rep, 1),
        is_causal=True, scale=1 / math.sqrt(D)).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    # position 0 sees only token 0: its value row, exactly
    np.testing.assert_array_equal(out[:, :, 0], v.double().numpy().repeat(rep, 1)[:, :, 0])


def test_prefill_attention_hand_worked():
    """Two positions, D = 2, sm_scale = ln 3: position 1 scores (0, ln 3) against keys
    (0, 0) and (1, 0), so its weights are 1/4 and 3/4 and its output is
    v0/4 + 3 v1/4 = (1, 6) for v0 = (4, 0), v1 = (0, 8); position 0 sees only key 0 and
    returns v0.  All inputs are exact in bf16."""
    f = lambda a: _bits(torch.tensor(a, dtype=torch.float32).to(torch.bfloat16))  # noqa: E731
    q = f([[[[5.0, -3.0], [1.0, 0.0]]]])
    k = f([[[[0.0, 0.0], [1.0, 0.0]]]])
    v = f([[[[4.0, 0.0], [0.0, 8.0]]]])
    out = O.prefill_attention(q, k, v, sm_scale=math.log(3.0))
    np.testing.assert_allclose(out[0, 0], [[4.0, 0.0], [1.0, 6.0]], rtol=0, atol=1e-12)
