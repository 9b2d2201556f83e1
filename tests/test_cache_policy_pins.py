"""Pins of the oracle's step-caching policies and error measures (CPU only).

The expected decision sequences below are written out by hand from the
parameter descriptions (vLLM-Omni cache-dit page, "DBCache" key parameters and
the "DiffusionCacheConfig" table; TMAP image-to-video page, "TeaCache"
inference flow), not produced by the oracle.  The residual sequences are
geometric, x * (9/8)^s, so every relative difference has the closed form
(9/8)^k - 1 and is exact in fp32 and fp64.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import cache_policy as cp

W, N, U, A, MC, MX = cp.WARMUP, cp.NO_PREV, cp.USE_CACHE, cp.ABOVE_THRESHOLD, cp.MAX_CACHED, cp.MAX_CONTINUOUS


def _rel(cur, prev):
    return oracle.fbc_rel_l1(cur, prev, 0.0)[0]


def test_policy_defaults_match_the_config_table():
    p = cp.CachePolicy()
    assert (p.max_warmup_steps, p.max_cached_steps, p.max_continuous_cached_steps) == (4, -1, 3)
    assert p.residual_diff_threshold == 0.24


def test_stable_residual_hits_the_continuous_limit():
    # Difference 0 everywhere: 4 warm-up steps, then runs of 3 cached steps
    # separated by one forced computation.
    got = cp.fbcache_decisions([0.0] * 12, cp.CachePolicy())
    assert got == [W, W, W, W, U, U, U, MX, U, U, U, MX]


def test_total_cached_limit():
    p = cp.CachePolicy(max_warmup_steps=1, max_cached_steps=2, max_continuous_cached_steps=-1)
    assert cp.fbcache_decisions([0.0] * 6, p) == [W, U, U, MC, MC, MC]


def test_unlimited_caching_and_no_warmup():
    p = cp.CachePolicy(max_warmup_steps=0, max_cached_steps=-1, max_continuous_cached_steps=-1)
    # Step 0 has nothing to compare with; afterwards every step is cached.
    assert cp.fbcache_decisions([0.0] * 5, p) == [N, U, U, U, U]


def test_threshold_is_strict_and_taken_in_fp32():
    p = cp.CachePolicy(max_warmup_steps=1, max_continuous_cached_steps=-1)
    t32 = float(np.float32(0.24))           # 0.23999999463558197
    assert t32 < 0.24
    seq = [0.0, t32, 0.5 * (t32 + 0.24), math.nextafter(t32, 0.0), 0.0]
    assert cp.fbcache_decisions(seq, p) == [W, A, A, U, U]


def test_above_threshold_resets_the_run():
    p = cp.CachePolicy(max_warmup_steps=1, max_continuous_cached_steps=2)
    seq = [0.0, 0.1, 0.1, 0.1, 0.3, 0.1, 0.1, 0.1]
    assert cp.fbcache_decisions(seq, p) == [W, U, U, MX, A, U, U, MX]


def _valid_fbcache(rels, decisions, p):
    """The rules as global properties of a whole sequence (an independent check)."""
    thr = float(np.float32(p.residual_diff_threshold))
    run, total, seen_compute = 0, 0, False
    for s, (r, d) in enumerate(zip(rels, decisions)):
        if s < p.max_warmup_steps or not seen_compute:
            if d == U:
                return False
        elif d == U:
            if not r < thr:
                return False
        else:
            # Computing although the difference was small is allowed only
            # when a limit binds.
            limit = ((p.max_cached_steps >= 0 and total == p.max_cached_steps)
                     or (p.max_continuous_cached_steps >= 0 and run == p.max_continuous_cached_steps))
            if r < thr and not limit:
                return False
        if d == U:
            run, total = run + 1, total + 1
        else:
            run, seen_compute = 0, True
        if p.max_continuous_cached_steps >= 0 and run > p.max_continuous_cached_steps:
            return False
        if p.max_cached_steps >= 0 and total > p.max_cached_steps:
            return False
    return True


@pytest.mark.parametrize("seed", range(6))
def test_random_sequences_obey_every_rule(seed):
    rng = np.random.default_rng(seed)
    for _ in range(50):
        p = cp.CachePolicy(max_warmup_steps=int(rng.integers(0, 5)),
                           max_cached_steps=int(rng.integers(-1, 8)),
                           max_continuous_cached_steps=int(rng.integers(-1, 4)),
                           residual_diff_threshold=float(rng.uniform(0.05, 0.5)))
        rels = list(rng.uniform(0.0, 0.6, size=int(rng.integers(1, 40))))
        d = cp.fbcache_decisions(rels, p)
        assert _valid_fbcache(rels, d, p)
        # a planted mistake (a limit ignored) must be caught by the checker
        if p.max_continuous_cached_steps >= 0:
            bad = cp.fbcache_decisions(rels, cp.CachePolicy(p.max_warmup_steps, p.max_cached_steps, -1,
                                                            p.residual_diff_threshold))
            if bad != d:
                assert not _valid_fbcache(rels, bad, p)


def _geometric(steps, n=4096, seed=3, dtype=np.float32):
    rng = np.random.default_rng(seed)
    # values m * 2^e with |m| <= 255: times 9^s / 8^s stays exact for s <= 5
    x = rng.integers(-255, 256, size=n).astype(np.float64) * np.exp2(rng.integers(-6, 6, size=n))
    return [(x * (9.0 / 8.0) ** s).astype(dtype) for s in range(steps)]


def test_stored_residual_is_the_last_computed_one():
    # Against the last computed step the difference grows as (9/8)^k - 1:
    # 0.125, 0.265625, 0.423828125 ...; against the previous step it would
    # stay 0.125 and every step would be cached.
    res = _geometric(6)[:3] + _geometric(6)[:3]
    p = cp.CachePolicy(max_warmup_steps=1, max_continuous_cached_steps=-1, residual_diff_threshold=0.3)
    rels, dec, counters = cp.fbcache_schedule(_geometric(6), p, _rel)
    assert dec == [W, U, U, A, U, U]
    assert math.isnan(rels[0])
    np.testing.assert_allclose(rels[1:], [0.125, 0.265625, 0.423828125, 0.125, 0.265625], rtol=0, atol=1e-15)
    assert counters == (6, 4, 2, True)
    # a residual sequence that returns to its start is cached against step 0
    rels2, dec2, _ = cp.fbcache_schedule(res, p, _rel)
    assert dec2 == [W, U, U, U, U, U]
    assert rels2[3] == 0.0


def test_teacache_accumulates_and_restarts():
    x = _geometric(6) + _geometric(6)[5:]          # adjacent difference 0.125 each step, then 0
    rels, resc, accs, dec = cp.teacache_schedule(x, [0.0, 1.0], 0.3, _rel)
    assert dec == [N, U, U, A, U, U, U]
    np.testing.assert_allclose(rels[1:6], [0.125] * 5, atol=1e-15)
    assert rels[6] == 0.0
    np.testing.assert_allclose(accs, [0.0, 0.125, 0.25, 0.0, 0.125, 0.25, 0.25], atol=1e-15)


def test_teacache_polynomial_order_is_ascending():
    x = _geometric(5)
    # 8 * rel^2 = 8 / 64 = 0.125 per step, the same pattern as the identity
    _, resc, _, dec = cp.teacache_schedule(x, [0.0, 0.0, 8.0], 0.3, _rel)
    assert dec == [N, U, U, A, U]
    np.testing.assert_allclose(resc[1:], [0.125] * 4, atol=1e-15)
    # [1, 0] is the constant 1 (ascending powers), so every step computes
    _, resc, _, dec = cp.teacache_schedule(x, [1.0, 0.0], 0.3, _rel)
    assert dec == [N, A, A, A, A] and resc[1:] == [1.0] * 4
    assert cp.polyval_ascending([1.0, -2.0, 3.0], 2.0) == 1.0 - 4.0 + 12.0


def test_compare_stats_closed_forms():
    a = np.float32([1, -2, 3, -4])
    b = np.float32([1.5, -2, 2, -4])
    rel, cos, mx = oracle.compare_stats(a, b)
    assert rel[0] == pytest.approx(1.5 / 10.0, abs=1e-15)
    assert cos[0] == pytest.approx(27.5 / math.sqrt(30.0 * 26.25), abs=1e-15)
    assert mx[0] == 1.0
    rel, cos, mx = oracle.compare_stats(a, -a)
    assert (rel[0], cos[0], mx[0]) == (2.0, -1.0, 8.0)
    rel, cos, mx = oracle.compare_stats(a, 2 * a)
    assert rel[0] == 1.0 and cos[0] == pytest.approx(1.0, abs=1e-15)
    rel, cos, _ = oracle.compare_stats(np.float32([1, 0]), np.float32([0, 1]))
    assert (rel[0], cos[0]) == (2.0, 0.0)
    rel, cos, mx = oracle.compare_stats(np.zeros(4, np.float32), np.zeros(4, np.float32))
    assert (rel[0], cos[0], mx[0]) == (0.0, 1.0, 0.0)
    rel, cos, _ = oracle.compare_stats(np.zeros(2, np.float32), np.float32([0, 1]))
    assert rel[0] == math.inf and cos[0] == 0.0


def test_compare_stats_segments_and_library_cosine():
    scipy_distance = pytest.importorskip("scipy.spatial.distance")
    rng = np.random.default_rng(7)
    a = rng.standard_normal(3 * 500).astype(np.float32)
    b = (a + 0.05 * rng.standard_normal(a.size)).astype(np.float32)
    bits_a = a.view(np.uint32) >> 16
    rel, cos, mx = oracle.compare_stats(a, b, segments=3)
    for s in range(3):
        x, y = a[s * 500:(s + 1) * 500].astype(np.float64), b[s * 500:(s + 1) * 500].astype(np.float64)
        assert cos[s] == pytest.approx(1.0 - scipy_distance.cosine(x, y), abs=1e-13)
        assert rel[s] == pytest.approx(np.linalg.norm(y - x, 1) / np.linalg.norm(x, 1), rel=1e-13)
        assert mx[s] == np.linalg.norm(y - x, np.inf)
    # bf16 bits widen exactly: truncated values compared with themselves
    r2, c2, m2 = oracle.compare_stats(bits_a.astype(np.uint16), bits_a.astype(np.uint16))
    assert (r2[0], m2[0]) == (0.0, 0.0) and c2[0] == pytest.approx(1.0, abs=1e-15)
