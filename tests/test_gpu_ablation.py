"""Key-granularity ablation on the GPU (needs a B200): kivi_fake_quant_keys
against the oracle, bit for bit.

The oracle computes k_hat = fp16(scale) * code + fp16(min) exactly in double;
the kernel rounds that value once to fp32 (one fma), so the kernel's output
must equal the oracle's value rounded to fp32, element for element.  The codes
are decided in fp32 on both sides.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from gpu_util import load_kivi

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kivi():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return load_kivi()


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("per_token", [False, True])
@pytest.mark.parametrize("D,rows,dist", [(128, 256, "lognormal"), (64, 96, "outlier"),
                                         (128, 32, "constant")])
def test_fake_quant_keys_bit_exact(kivi, bits, per_token, D, rows, dist):
    gen = torch.Generator().manual_seed(rows + D + bits)
    k = torch.randn(rows, D, generator=gen)
    if dist == "lognormal":
        k = k * torch.exp(torch.randn(D, generator=gen))
    elif dist == "outlier":
        k[:, torch.randperm(D, generator=gen)[:4]] *= 10
    else:  # constant groups in both directions: scale 0, codes 0
        k = torch.full((rows, D), 0.75)
    k = k.to(torch.bfloat16)
    got = kivi.kivi_fake_quant_keys(k.cuda(), bits, per_token).cpu().numpy()
    ref = O.fake_quant_keys(synth.bf16_bits(k), bits, per_token).astype(np.float32)
    assert np.array_equal(got, ref), f"{(got != ref).sum()} elements differ"


def test_fake_quant_keys_full_layer_per_channel_beats_per_token(kivi):
    """One Llama-3-8B layer of synthetic keys with log-normal channel scales
    (16 x 8 x 8192 rows): per-channel quantization has the smaller error, at 2
    and at 4 bits; a sampled group is checked against the oracle."""
    w = synth.WORKLOADS["llama3_8b_gqa_8k"]
    k, _ = synth.prefill_kv(w, 0, device="cuda")
    rows = k.reshape(-1, w.head_dim)
    kf = rows.float()
    for bits in (2, 4):
        e = {}
        for pt in (False, True):
            k_hat = kivi.kivi_fake_quant_keys(rows, bits, pt)
            e[pt] = float((k_hat - kf).norm() / kf.norm())
            ref = O.fake_quant_keys(synth.bf16_bits(rows[4096:4160].cpu()), bits, pt)
            assert np.array_equal(k_hat[4096:4160].cpu().numpy(), ref.astype(np.float32))
        assert e[False] < e[True], e
