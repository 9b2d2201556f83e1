"""Pins of the oracle's token-sharded 8-bit pre-pass (CPU only).

Each device of a Ulysses group reduces its token slice to per-channel K sums
and V maxima; combined, they must reproduce the single-device statistics
exactly (bf16 values sum exactly in fp64), so the codes each device writes for
its tokens are the single-device codes, bit for bit, whenever the slices hold
whole 128-token blocks.  The stand-alone routines are checked against the
single-device ones (an independent implementation each: numpy here, C there).
"""
import numpy as np
import pytest

import oracle
from diffusion_transformer_attention_attn_b200 import inputs


def _case(N=1024, H=3, k_off=3.0, seed=4):
    return inputs.attn_inputs(inputs.AttnCase("sh", 1, H, N, 128, k_offset_std=k_off, seed=seed))


def test_sums_and_maxima_match_the_single_device_statistics():
    q, k, v = _case()
    N = k.shape[2]
    assert np.array_equal(oracle.mean_from_sums(oracle.k_channel_sums(k), N), oracle.channel_mean(k))
    codes, scales = oracle.quant_e4m3_channels(v)
    c2, s2 = oracle.quant_e4m3_with_amax(v, oracle.channel_amax(v))
    assert np.array_equal(codes, c2) and np.array_equal(scales, s2)


@pytest.mark.parametrize("world", [2, 4])
def test_shards_combine_to_the_whole_and_quantise_identically(world):
    q, k, v = _case()
    N = k.shape[2]
    Nl = N // world
    sl = [slice(r * Nl, (r + 1) * Nl) for r in range(world)]
    ksum = sum(oracle.k_channel_sums(k[:, :, s]) for s in sl)
    vmax = np.maximum.reduce([oracle.channel_amax(v[:, :, s]) for s in sl])
    assert np.array_equal(ksum, oracle.k_channel_sums(k))
    assert np.array_equal(vmax, oracle.channel_amax(v))
    mean = oracle.mean_from_sums(ksum, N)
    qc, qs = oracle.quant_int8_blocks(q, 128)
    kc, ks = oracle.quant_int8_blocks(k, 64, mean)
    vc, vs = oracle.quant_e4m3_with_amax(v, vmax)
    for r, s in enumerate(sl):
        qcr, qsr = oracle.quant_int8_blocks(q[:, :, s], 128)
        kcr, ksr = oracle.quant_int8_blocks(k[:, :, s], 64, mean)
        vcr, vsr = oracle.quant_e4m3_with_amax(v[:, :, s], vmax)
        assert np.array_equal(qcr, qc[:, :, s]) and np.array_equal(kcr, kc[:, :, s]) and np.array_equal(vcr, vc[:, :, s])
        assert np.array_equal(qsr, qs[:, :, r * Nl // 128:(r + 1) * Nl // 128])
        assert np.array_equal(ksr, ks[:, :, r * Nl // 64:(r + 1) * Nl // 64])
        assert np.array_equal(vsr, vs)
    # a slice that splits a 128-token block gets other Q scales (the reason
    # the sharded path asks for whole blocks)
    qc3, qs3 = oracle.quant_int8_blocks(q[:, :, 64:320], 128)
    assert not np.array_equal(qs3, qs[:, :, 0:2])


def test_zero_channel_guard_with_given_maxima():
    _, _, v = _case(N=256, H=1)
    v = v.copy()
    v[..., 5] = 0
    c, s = oracle.quant_e4m3_with_amax(v, oracle.channel_amax(v))
    assert s[0, 0, 5] == 0 and not c[..., 5].any() and np.isfinite(s).all()


def test_attention_from_codes_is_the_emulated_path():
    q, k, v = _case(N=384, H=2)
    rows = np.array([0, 100, 383])
    ref = oracle.emulated_q8_attention(q, k, v, smooth_k=True, rows=rows)
    qc, qs = oracle.quant_int8_blocks(q, 128)
    kc, ks = oracle.quant_int8_blocks(k, 64, oracle.channel_mean(k))
    vc, vs = oracle.quant_e4m3_channels(v)
    got = oracle.attention_from_codes(qc, qs, kc, ks, vc, vs, rows=rows)
    assert np.array_equal(got, ref)
    # bf16 V: dequantised Q and K against the exact V; as the scales go to the
    # exact inputs (all-zero codes error aside) this stays near the true attention
    exact = oracle.attention(q, k, v, rows=rows)
    near = oracle.attention_from_codes(qc, qs, kc, ks, v, None, rows=rows)
    assert np.abs(near - exact).max() < 0.05
