"""Pins of the oracle's log-sum-exp attention and chunk merge (CPU only).

attention_lse is checked against a direct numpy evaluation with scipy's
logsumexp and against closed forms; merge_partials against the identity that
makes key-chunked (ring) attention exact: merging the chunks' results gives
the attention over all keys.
"""
import math

import numpy as np
import pytest

import oracle
from diffusion_transformer_attention_attn_b200 import inputs


def _bits(x):
    return inputs.bf16_bits(np.asarray(x, dtype=np.float32))


def _wide(b):
    return inputs.bf16_to_f32(b).astype(np.float64)


def _case(Nq, Nkv, d=16, B=1, H=2, seed=0):
    rng = np.random.default_rng(seed)
    q = _bits(rng.standard_normal((B, H, Nq, d)))
    k = _bits(rng.standard_normal((B, H, Nkv, d)) + 0.5)
    v = _bits(rng.standard_normal((B, H, Nkv, d)))
    return q, k, v


def test_lse_and_output_against_numpy_and_scipy():
    special = pytest.importorskip("scipy.special")
    q, k, v = _case(7, 13, d=16)
    scale = 0.25
    o, lse = oracle.attention_lse(q, k, v, scale)
    s = scale * np.einsum("bhid,bhjd->bhij", _wide(q), _wide(k))
    ref_lse = special.logsumexp(s, axis=-1)
    p = special.softmax(s, axis=-1)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)
    np.testing.assert_allclose(o, p @ _wide(v), rtol=0, atol=1e-12)


def test_single_key_and_identical_keys():
    q, k, v = _case(5, 1, d=8, seed=1)
    o, lse = oracle.attention_lse(q, k, v, 0.5)
    dot = (_wide(q) * _wide(k)).sum(-1)       # one key: the logit itself, weight 1
    np.testing.assert_allclose(lse, 0.5 * dot, atol=1e-12)
    np.testing.assert_allclose(o, np.broadcast_to(_wide(v), o.shape), atol=0)
    # N equal keys: lse gains ln N and the output is the mean of V
    k4 = np.repeat(k, 4, axis=2)
    rng = np.random.default_rng(2)
    v4 = _bits(rng.standard_normal((1, 2, 4, 8)))
    o4, lse4 = oracle.attention_lse(q, k4, v4, 0.5)
    np.testing.assert_allclose(lse4, 0.5 * dot + math.log(4.0), atol=1e-12)
    np.testing.assert_allclose(o4, np.broadcast_to(_wide(v4).mean(axis=2, keepdims=True), o4.shape), atol=1e-12)


@pytest.mark.parametrize("cuts", [[13], [1, 12], [5, 5, 3], [4, 4, 4, 1]])
def test_merge_of_chunks_is_attention_over_all_keys(cuts):
    q, k, v = _case(9, sum(cuts), d=16, seed=len(cuts))
    o_all, l_all = oracle.attention_lse(q, k, v)
    outs, lses, a = [], [], 0
    for c in cuts:
        o_c, l_c = oracle.attention_lse(q, k[:, :, a:a + c], v[:, :, a:a + c])
        outs.append(o_c)
        lses.append(l_c)
        a += c
    o_m, l_m = oracle.merge_partials(outs, lses)
    np.testing.assert_allclose(o_m, o_all, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l_m, l_all, rtol=0, atol=1e-12)
    if len(cuts) > 1:
        # a plausible mistake, averaging the chunk outputs, is far from the truth
        assert np.abs(np.mean(outs, axis=0) - o_all).max() > 1e-3


def test_merge_is_invariant_to_chunk_order_and_large_lse():
    rng = np.random.default_rng(4)
    outs = [rng.standard_normal((3, 8)) for _ in range(3)]
    lses = [rng.uniform(700, 760, size=3) for _ in range(3)]     # exp would overflow without the shift
    o1, l1 = oracle.merge_partials(outs, lses)
    o2, l2 = oracle.merge_partials(outs[::-1], lses[::-1])
    assert np.isfinite(o1).all() and np.isfinite(l1).all()
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)
    # two chunks with equal lse: plain average, lse + ln 2
    o, l = oracle.merge_partials([outs[0], outs[1]], [lses[0], lses[0]])
    np.testing.assert_allclose(o, 0.5 * (outs[0] + outs[1]), atol=1e-12)
    np.testing.assert_allclose(l, lses[0] + math.log(2.0), atol=1e-12)
