"""Pins for the fp64 oracle: closed forms, invariants, hand cases, brute force.

Each test checks the oracle against something other than itself, chosen so
that a plausible slip (a dropped term, a wrong sign or index, a transposed
operand, a wrong scale) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest

import oracle
from diffusion_transformer_attention_attn_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(t) for t in line.split()])
    return np.array(rows)


def _rand(shape, seed, scale=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * scale


# ---------------------------------------------------------------- attention

def test_hand_case_d1():
    t = _load_rows("attn_hand_d1.txt")
    q = t[:, 0].reshape(1, 1, 2, 1)
    k = t[:, 1].reshape(1, 1, 2, 1)
    v = t[:, 2].reshape(1, 1, 2, 1)
    o = oracle.attention(q, k, v, scale=1.0)
    np.testing.assert_allclose(o.reshape(-1), t[:, 3], rtol=0, atol=1e-14)


def _brute(q, k, v, scale):
    """Direct softmax: exp of the raw logits, no max shift (small inputs only)."""
    B, H, N, d = q.shape
    out = np.zeros((B, H, N, d))
    for b in range(B):
        for h in range(H):
            for i in range(N):
                w = np.array([math.exp(scale * sum(q[b, h, i, c] * k[b, h, j, c] for c in range(d)))
                              for j in range(N)])
                out[b, h, i] = (w[:, None] * v[b, h]).sum(0) / w.sum()
    return out


@pytest.mark.parametrize("N,d", [(1, 1), (2, 3), (5, 4), (8, 8), (7, 2)])
def test_brute_force_small(N, d):
    q, k, v = (_rand((1, 2, N, d), s) for s in (1, 2, 3))
    scale = 1.0 / math.sqrt(d)
    np.testing.assert_allclose(oracle.attention(q, k, v, scale=scale), _brute(q, k, v, scale),
                               rtol=1e-12, atol=1e-13)


def test_asymmetric_operands():
    # Q K^T vs K Q^T and P V vs V P differ here; a transposed operand fails.
    q = np.array([[[[1.0, 0.0], [0.0, 2.0], [1.0, 1.0]]]])
    k = np.array([[[[0.5, -1.0], [2.0, 0.0], [0.0, 0.3]]]])
    v = np.array([[[[1.0, 10.0], [2.0, 20.0], [4.0, -5.0]]]])
    np.testing.assert_allclose(oracle.attention(q, k, v, scale=0.7), _brute(q, k, v, 0.7),
                               rtol=1e-13, atol=1e-13)


def test_v_ones_gives_ones():
    q, k = _rand((1, 2, 300, 16), 4, 3.0), _rand((1, 2, 300, 16), 5, 3.0)
    o = oracle.attention(q, k, np.ones((1, 2, 300, 16)))
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-13)


def test_q_zero_gives_column_mean():
    k, v = _rand((2, 1, 257, 8), 6), _rand((2, 1, 257, 8), 7)
    o = oracle.attention(np.zeros_like(k), k, v)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape),
                               rtol=0, atol=1e-13)


def test_joint_permutation_of_keys_values():
    q, k, v = (_rand((1, 2, 129, 16), s) for s in (8, 9, 10))
    perm = np.random.Generator(np.random.PCG64(11)).permutation(129)
    np.testing.assert_allclose(oracle.attention(q, k[:, :, perm], v[:, :, perm]),
                               oracle.attention(q, k, v), rtol=0, atol=1e-12)


def test_per_row_logit_constant_k_offset():
    # q.(k_j + mu) = q.k_j + q.mu: a per-row constant -> O unchanged.
    q, k, v = (_rand((1, 3, 100, 16), s) for s in (12, 13, 14))
    mu = _rand((1, 3, 1, 16), 15, 5.0)
    np.testing.assert_allclose(oracle.attention(q, k + mu, v), oracle.attention(q, k, v),
                               rtol=0, atol=1e-11)


def test_single_key_returns_value_row():
    q, k, v = (_rand((1, 2, 1, 64), s) for s in (16, 17, 18))
    np.testing.assert_allclose(oracle.attention(q, k, v), v, rtol=0, atol=1e-15)


def test_scale_limits():
    q, k, v = (_rand((1, 1, 20, 4), s) for s in (19, 20, 21))
    # s -> 0: uniform weights, O = mean of V.
    o0 = oracle.attention(q, k, v, scale=1e-13)
    np.testing.assert_allclose(o0, np.broadcast_to(v.mean(axis=2, keepdims=True), o0.shape), atol=1e-11)
    # s -> inf: hard attention on the argmax key of each row.
    o_inf = oracle.attention(q, k, v, scale=1e8)
    arg = np.argmax(q[0, 0] @ k[0, 0].T, axis=1)
    np.testing.assert_allclose(o_inf[0, 0], v[0, 0, arg], atol=1e-9)


def test_linearity_in_v():
    q, k, v1, v2 = (_rand((1, 2, 64, 8), s) for s in (22, 23, 24, 25))
    a, b = 0.75, -2.5
    np.testing.assert_allclose(oracle.attention(q, k, a * v1 + b * v2),
                               a * oracle.attention(q, k, v1) + b * oracle.attention(q, k, v2),
                               rtol=0, atol=1e-12)


def test_row_subset_matches_full():
    q, k, v = (_rand((2, 2, 90, 8), s) for s in (26, 27, 28))
    rows = np.array([0, 5, 44, 89])
    np.testing.assert_array_equal(oracle.attention(q, k, v, rows=rows),
                                  oracle.attention(q, k, v)[:, :, rows])


def test_bf16_inputs_widen_exactly():
    q, k, v = inputs.attn_inputs(inputs.TINY, N=70)
    wq, wk, wv = (inputs.bf16_to_f32(t).astype(np.float64) for t in (q, k, v))
    np.testing.assert_array_equal(oracle.attention(q, k, v), oracle.attention(wq, wk, wv))


def test_default_scale_is_fp32_inverse_sqrt_d():
    q, k, v = (_rand((1, 1, 10, 64), s) for s in (29, 30, 31))
    s32 = float(np.float32(1.0) / np.sqrt(np.float32(64)))
    assert s32 == 0.125
    np.testing.assert_array_equal(oracle.attention(q, k, v), oracle.attention(q, k, v, scale=0.125))


def test_large_logits_no_overflow():
    # Two-pass max subtraction keeps exp() finite for logits ~ 1e3.
    q = np.full((1, 1, 3, 2), 30.0)
    k = np.array([[[[30.0, 0.0], [29.0, 0.0], [-30.0, 0.0]]]])
    v = np.array([[[[1.0, 0.0], [0.0, 1.0], [5.0, 5.0]]]])
    o = oracle.attention(q, k, v, scale=1.0)
    w = np.array([1.0, math.exp(-30.0), 0.0])
    exp = (w[:, None] * v[0, 0]).sum(0) / w.sum()
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(exp, (3, 2)), rtol=1e-12, atol=1e-300)


# ---------------------------------------------------------------- first-block cache

def test_fbc_hand_case():
    prev = np.array([1, -2, 3, -4], dtype=np.float32)
    cur = np.array([1.5, -2, 2, -4], dtype=np.float32)
    for thr, rel_exp, skip_exp in _load_rows("fbc_hand.txt"):
        rel, skip = oracle.fbc_rel_l1(cur, prev, thr)
        assert abs(rel - rel_exp) < 1e-15
        assert skip == int(skip_exp)


def test_fbc_identical_is_zero_and_skips():
    cur, prev = inputs.fbc_inputs(inputs.FBC_TINY)
    rel, skip = oracle.fbc_rel_l1(prev, prev, 0.08)
    assert rel == 0.0 and skip == 1


@pytest.mark.parametrize("alpha", [0.25, -0.5, 0.03125, 2.0])
def test_fbc_scaled_copy(alpha):
    # cur = (1 + alpha) prev -> rel = |alpha| (exact: power-of-two-ish alphas).
    prev = np.array([1.0, -3.0, 0.5, 8.0, -0.25], dtype=np.float32)
    cur = (prev * np.float32(1 + alpha)).astype(np.float32)
    rel, _ = oracle.fbc_rel_l1(cur, prev, 0.08)
    assert abs(rel - abs(alpha)) < 1e-15


def test_fbc_threshold_is_strict():
    prev = np.array([1.0, -2.0, 3.0, -2.0], dtype=np.float32)   # sum |prev| = 8
    cur = np.array([2.0, -2.0, 3.0, -2.0], dtype=np.float32)    # sum |diff| = 1
    rel, skip = oracle.fbc_rel_l1(cur, prev, 0.125)
    assert rel == 0.125 and skip == 0                            # equality -> compute
    assert oracle.fbc_rel_l1(cur, prev, 0.1251)[1] == 1


def test_fbc_zero_denominator():
    z = np.zeros(8, dtype=np.float32)
    assert oracle.fbc_rel_l1(z, z, 0.08) == (0.0, 1)
    rel, skip = oracle.fbc_rel_l1(np.ones(8, dtype=np.float32), z, 0.08)
    assert math.isinf(rel) and skip == 0


def test_fbc_bf16_matches_f32_widening():
    cur, prev = inputs.fbc_inputs(inputs.FbcCase("x", 33, 65, "bf16", 0.03, 0.08))
    r16 = oracle.fbc_rel_l1(cur, prev, 0.08)
    r32 = oracle.fbc_rel_l1(inputs.bf16_to_f32(cur), inputs.bf16_to_f32(prev), 0.08)
    assert r16 == r32


def test_fbc_workloads_decisions():
    # Drift 0.05 and 0.03 against 0.08: mean|drift|/mean|prev| ~= drift std -> skip.
    for case, expect in ((inputs.FBC_TINY, 0.05), (inputs.FbcCase("s", 512, 384, "bf16", 0.03, 0.08), 0.03)):
        cur, prev = inputs.fbc_inputs(case)
        rel, skip = oracle.fbc_rel_l1(cur, prev, case.threshold)
        assert abs(rel - expect) < 0.1 * expect and skip == 1


# ---------------------------------------------------------------- quantiser

def test_e4m3_decode_matches_torch_table():
    torch = pytest.importorskip("torch")
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    ours = oracle.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert (np.isnan(ours) == nan).all()
    np.testing.assert_array_equal(ours[~nan], ref[~nan])


def test_e4m3_encode_matches_torch_in_range():
    torch = pytest.importorskip("torch")
    rng = np.random.Generator(np.random.PCG64(40))
    # every representable value, every midpoint (ties), and random values
    reps = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    reps = np.sort(reps[np.isfinite(reps) & (reps >= 0)])
    mids = (reps[1:] + reps[:-1]) / 2
    x = np.concatenate([reps, mids, rng.uniform(0, 460, 3000), rng.uniform(0, 0.02, 2000)]).astype(np.float32)
    x = x[np.abs(x) < 464.0]
    x = np.concatenate([x, -x])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode(x), ref)


def test_e4m3_saturates():
    out = oracle.e4m3_encode(np.array([448.0, 464.0, 1e6, -500.0], dtype=np.float32))
    np.testing.assert_array_equal(out, [0x7E, 0x7E, 0x7E, 0xFE])


def _bits(vals):
    return inputs.bf16_bits(np.asarray(vals, dtype=np.float32))


def test_int8_block_exact_integers_and_ties():
    # amax = 127 -> inv = 1, scale = 1: integers map to themselves, .5 ties go to even.
    x = np.zeros((1, 1, 4, 4), dtype=np.float32)
    x[0, 0, 0] = [127, -3, 2.5, 3.5]
    x[0, 0, 1] = [-2.5, 0.5, 1.5, -127]
    codes, scales = oracle.quant_int8_blocks(_bits(x), 4)
    assert scales[0, 0, 0] == 1.0
    np.testing.assert_array_equal(codes[0, 0, 0], [127, -3, 2, 4])
    np.testing.assert_array_equal(codes[0, 0, 1], [-2, 0, 2, -127])


def test_int8_zero_block_guard():
    # An all-zero block and an all-zero channel give scale 0 and code 0, never NaN.
    x = np.zeros((1, 1, 8, 4), dtype=np.float32)
    x[0, 0, 4:, 1:] = 3.0                      # block 1 nonzero except channel 0
    codes, scales = oracle.quant_int8_blocks(_bits(x), 4)
    assert scales[0, 0, 0] == 0.0 and (codes[0, 0, :4] == 0).all()
    assert np.isfinite(scales).all()
    assert (codes[0, 0, 4:, 0] == 0).all() and (codes[0, 0, 4:, 1:] == 127).all()


def test_int8_reconstruction_bound_and_ragged_tail():
    x = inputs.bf16_to_f32(inputs.attn_inputs(inputs.TINY, N=200)[1])
    b = inputs.bf16_bits(x)
    codes, scales = oracle.quant_int8_blocks(b, 64)
    assert scales.shape == (1, 2, 4)            # ceil(200 / 64)
    tok = np.arange(200)
    recon = codes.astype(np.float64) * scales[:, :, tok // 64, None]
    err = np.abs(recon - x)
    bound = scales[:, :, tok // 64, None] * 0.5 * (1 + 1e-5) + 1e-7
    assert (err <= bound).all()
    # the tail block's amax is over its 8 valid tokens only
    tail = np.abs(x[:, :, 192:200]).max(axis=(2, 3))
    np.testing.assert_allclose(scales[:, :, 3], (tail / np.float32(127)).astype(np.float32), rtol=1e-7)


def test_channel_mean_and_smoothing():
    k = inputs.attn_inputs(inputs.IMAGE_Q8, N=300)[1]
    m = oracle.channel_mean(k)
    ref = inputs.bf16_to_f32(k).astype(np.float64).mean(axis=2).astype(np.float32)
    np.testing.assert_array_equal(m, ref)
    codes, scales = oracle.quant_int8_blocks(k, 64, m)
    # with the shared offsets removed, the scales shrink well below the raw ones
    _, raw = oracle.quant_int8_blocks(k, 64)
    assert (scales < raw).mean() > 0.9


def test_e4m3_channel_quant_bound_and_zero_channel():
    v = inputs.bf16_to_f32(inputs.attn_inputs(inputs.TINY, N=100)[2]).copy()
    v[0, 1, :, 5] = 0.0
    codes, scales = oracle.quant_e4m3_channels(inputs.bf16_bits(v))
    assert scales[0, 1, 5] == 0.0 and (codes[0, 1, :, 5] == 0).all()
    recon = oracle.e4m3_decode(codes).astype(np.float64) * scales[:, :, None, :]
    # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 in the normal range,
    # absolute error <= 2^-10 * scale in the subnormal range.
    err = np.abs(recon - v)
    assert (err <= np.maximum(np.abs(v) * 2.0 ** -4, scales[:, :, None, :] * 2.0 ** -10) * 1.0001 + 1e-12).all()
    amax = np.abs(v).max(axis=2)
    np.testing.assert_array_equal(scales, (amax / np.float32(448)).astype(np.float32))


def test_emulated_q8_is_exact_when_inputs_are_representable():
    # Q, K: integer values with |max| = 127 in every block -> codes exact, scale 1.
    # V: e4m3-representable values with channel max 448 -> codes exact, scale 1.
    rng = np.random.Generator(np.random.PCG64(50))
    N, d = 130, 8
    q = rng.integers(-127, 128, (1, 1, N, d)).astype(np.float32)
    k = rng.integers(-127, 128, (1, 1, N, d)).astype(np.float32)
    q[0, 0, ::64, 0] = 127.0
    k[0, 0, ::32, 0] = 127.0
    reps = oracle.e4m3_decode(np.arange(0, 127, dtype=np.uint8))
    v = rng.choice(reps, (1, 1, N, d)).astype(np.float32)
    v[0, 0, 0, :] = 448.0
    qb, kb, vb = (inputs.bf16_bits(t) for t in (q, k, v))
    exact = oracle.attention(qb, kb, vb, scale=0.01)
    emu = oracle.emulated_q8_attention(qb, kb, vb, scale=0.01, smooth_k=False)
    np.testing.assert_allclose(emu, exact, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- input generators

def test_bf16_rounding_is_rne():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5], dtype=np.float32)
    b = inputs.bf16_bits(x)
    # 1+2^-8 is a tie -> even (1.0); 1+3*2^-8 is a tie -> even (1+2^-6... i.e. 1+4*2^-8)
    np.testing.assert_array_equal(inputs.bf16_to_f32(b), [1.0, 1.0, 1.0 + 4 * 2 ** -8, 1.0, -2.5])


def test_generators_are_seeded_and_shaped():
    a = inputs.attn_inputs(inputs.IMAGE_Q8, N=1000)
    b = inputs.attn_inputs(inputs.IMAGE_Q8, N=1000)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    q = a[0]
    assert q.shape == (1, 24, 1000, 128)
    assert (q[..., 7] == 0).all() and (q[:, :, 640:768] == 0).all()


def test_fp8_value_rounding_floor():
    # A property of the 8-bit recipe, computed with the oracle alone: rounding
    # V to per-channel e4m3 (3 mantissa bits) moves attention outputs on
    # i.i.d. N(0,1) data by about 2.7% in relative L1, while per-block INT8
    # Q/K costs about 1.3%.  The FP8-PV parity bound rests on these figures.
    case = inputs.AttnCase("floor", 1, 2, 1024, 128, seed=3)
    q, k, v = inputs.attn_inputs(case)
    f = lambda t: inputs.bf16_to_f32(t).astype(np.float64)
    rows = np.arange(0, 1024, 32)
    ref = oracle.attention(f(q), f(k), f(v), rows=rows)
    vc, vs = oracle.quant_e4m3_channels(v)
    vd = oracle.e4m3_decode(vc).astype(np.float64) * vs[:, :, None, :]
    rel_v = np.abs(oracle.attention(f(q), f(k), vd, rows=rows) - ref).sum() / np.abs(ref).sum()
    assert 0.018 < rel_v < 0.036
    qc, qs = oracle.quant_int8_blocks(q, 128)
    kc, ks = oracle.quant_int8_blocks(k, 64, oracle.channel_mean(k))
    tok = np.arange(case.N)
    qd = qc * qs[:, :, tok // 128, None].astype(np.float64)
    kd = kc * ks[:, :, tok // 64, None].astype(np.float64)
    rel_qk = np.abs(oracle.attention(qd, kd, f(v), rows=rows) - ref).sum() / np.abs(ref).sum()
    assert 0.005 < rel_qk < 0.02


def test_fbc_sums_of_shards_add_up_and_give_rel():
    rng = np.random.default_rng(11)
    prev = rng.standard_normal(10007).astype(np.float32)
    cur = (prev + 0.05 * rng.standard_normal(prev.size)).astype(np.float32)
    num, den = oracle.fbc_sums(cur, prev)
    parts = [oracle.fbc_sums(cur[a:b], prev[a:b]) for a, b in ((0, 3000), (3000, 3001), (3001, 10007))]
    assert abs(sum(x for x, _ in parts) - num) <= 1e-9 * num
    assert abs(sum(y for _, y in parts) - den) <= 1e-9 * den
    rel, skip = oracle.rel_from_sums(num, den, 0.08)
    rel_ref, skip_ref = oracle.fbc_rel_l1(cur, prev, 0.08)
    assert abs(rel - rel_ref) <= 1e-12 * rel_ref and skip == skip_ref
    # the hand case of the First Block Cache reading: 1.5 / 10
    assert oracle.fbc_sums(np.float32([1.5, -2, 2, -4]), np.float32([1, -2, 3, -4])) == (1.5, 10.0)
    assert oracle.rel_from_sums(0.0, 0.0, 0.1) == (0.0, 1)
    assert oracle.rel_from_sums(1.0, 0.0, 0.1) == (float("inf"), 0)


# ---------------------------------------------------------------- 8-bit block-scale indexing

def _scaled_blocks(rng, n_tok, d, blk, halves):
    """Values exactly representable after INT8 quantisation: block b holds
    integers in [-127, 127] with 127 present (amax 127: inv 1, scale 1) when
    halves[b] is False, else multiples of 1/2 in [-63.5, 63.5] with 63.5
    present (amax 63.5: inv 2, scale 1/2).  The second half of each block is
    the negation of its first half, so every channel's mean is exactly 0."""
    x = np.empty((1, 1, n_tok, d), dtype=np.float32)
    for b in range(n_tok // blk):
        half = rng.integers(-127, 128, (blk // 2, d)).astype(np.float32)
        half[0, 0] = 127.0
        if halves[b]:
            half = half / np.float32(2.0)
        x[0, 0, b * blk:b * blk + blk // 2] = half
        x[0, 0, b * blk + blk // 2:(b + 1) * blk] = -half
    return x


@pytest.mark.parametrize("smooth_k", [False, True])
def test_q8_dequantisation_uses_each_tokens_own_block_scale(smooth_k):
    # Q blocks of 128 tokens with scales 1, 1/2; K blocks of 64 tokens with
    # scales 1, 1/2, 1, 1/2; V e4m3-representable with channel maxima 448.
    # Every code is exact, so both quantised-attention replays equal the exact
    # attention; a swapped (64 <-> 128) or shifted block index does not.
    rng = np.random.Generator(np.random.PCG64(77))
    N, d, s = 256, 8, 1e-4
    q = _scaled_blocks(rng, N, d, 128, [False, True])
    k = _scaled_blocks(rng, N, d, 64, [False, True, False, True])
    reps = oracle.e4m3_decode(np.arange(0, 127, dtype=np.uint8))
    v = rng.choice(reps, (1, 1, N, d)).astype(np.float32) * rng.choice([-1.0, 1.0], (1, 1, N, d)).astype(np.float32)
    v[0, 0, 5, :] = 448.0
    qb, kb, vb = (inputs.bf16_bits(t) for t in (q, k, v))
    exact = oracle.attention(qb, kb, vb, scale=s)
    qc, qs = oracle.quant_int8_blocks(qb, 128)
    kc, ks = oracle.quant_int8_blocks(kb, 64, oracle.channel_mean(kb) if smooth_k else None)
    vc, vs = oracle.quant_e4m3_channels(vb)
    np.testing.assert_array_equal(qs[0, 0], [1.0, 0.5])
    np.testing.assert_array_equal(ks[0, 0], [1.0, 0.5, 1.0, 0.5])
    np.testing.assert_array_equal(vs, np.ones((1, 1, d), dtype=np.float32))
    emu = oracle.emulated_q8_attention(qb, kb, vb, scale=s, smooth_k=smooth_k)
    np.testing.assert_allclose(emu, exact, rtol=0, atol=1e-12)
    codes = oracle.attention_from_codes(qc, qs, kc, ks, vc, vs, scale=s)
    np.testing.assert_allclose(codes, exact, rtol=0, atol=1e-12)
    # The same replay with a wrong block index is far off: this input tells
    # the indexings apart.
    tok = np.arange(N)
    vd = oracle.e4m3_decode(vc).astype(np.float64)
    for qi, ki in ((np.minimum(tok // 64, 1), tok // 64),           # Q indexed per 64 tokens
                   (tok // 128, np.minimum(tok // 128, 3)),         # K indexed per 128 tokens
                   (tok // 128, (tok // 64 + 1) % 4)):              # K shifted by one block
        wrong = oracle.attention(qc * qs[:, :, qi, None].astype(np.float64),
                                 kc * ks[:, :, ki, None].astype(np.float64), vd, scale=s)
        assert np.abs(wrong - exact).max() > 1e-2


# ---------------------------------------------------------------- zero-scale guard, tiny maxima

def test_zero_scale_guard_covers_maxima_without_a_finite_inverse():
    # TMAP page, operator details: the quantisation scale of an all-zero
    # channel made the output NaN.  The same happens when amax is so small
    # that 127/amax (or 448/amax) overflows fp32: inv = inf and 0 * inf = NaN.
    # Such a block or channel counts as zero; one whose inverse is finite is
    # quantised normally.
    x = np.zeros((1, 1, 384, 4), dtype=np.float32)
    x[0, 0, 1:128:3, 2] = 1e-37                   # block 0: amax 1e-37, 127/amax overflows
    x[0, 0, 128:256, :] = 1e-36                    # block 1: 127/1e-36 = 1.27e38, finite
    x[0, 0, 130, 1] = 0.0
    x[0, 0, 256:384, :] = 0.0                      # block 2: all zero
    xb = inputs.bf16_bits(x)
    codes, scales = oracle.quant_int8_blocks(xb, 128)
    assert scales[0, 0, 0] == 0.0 and (codes[0, 0, :128] == 0).all()
    a1 = np.float32(inputs.bf16_to_f32(xb)[0, 0, 128, 0])
    assert scales[0, 0, 1] == a1 / np.float32(127) and scales[0, 0, 1] > 0
    assert (codes[0, 0, 128:256][x[0, 0, 128:256] != 0] == 127).all() and codes[0, 0, 130, 1] == 0
    assert scales[0, 0, 2] == 0.0 and (codes[0, 0, 256:] == 0).all()
    # V per channel: channel 0 holds {0, 1e-37}, channel 1 has amax 1e-36
    # (448/1e-36 overflows too), channel 2 amax 1e-35 (finite inverse).
    v = np.zeros((1, 1, 64, 3), dtype=np.float32)
    v[0, 0, ::2, 0] = 1e-37
    v[0, 0, 3, 1] = 1e-36
    v[0, 0, 7, 2] = 1e-35
    vb = inputs.bf16_bits(v)
    vc, vs = oracle.quant_e4m3_channels(vb)
    assert vs[0, 0, 0] == 0.0 and vs[0, 0, 1] == 0.0 and vs[0, 0, 2] > 0
    assert (vc[0, 0, :, :2] == 0).all() and vc[0, 0, 7, 2] == 0x7E    # 448 -> largest e4m3
    amax = np.abs(inputs.bf16_to_f32(vb)).max(axis=2)
    vc2, vs2 = oracle.quant_e4m3_with_amax(vb, amax)
    np.testing.assert_array_equal(vc2, vc)
    np.testing.assert_array_equal(vs2, vs)
    assert np.isfinite(oracle.e4m3_decode(vc)).all()
