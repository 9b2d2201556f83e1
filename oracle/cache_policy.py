"""Step-caching policies of the oracle: plain Python over the fp64 residual
difference of ``oracle.fbc_rel_l1``.

TEST INFRASTRUCTURE ONLY (imported by ``tests/`` and never by the CUDA
library or its binding).

Two policies decide, once per denoising step, whether the expensive part of
the transformer runs ("compute") or the cached result is reused ("use cache"):

* ``fbcache_schedule`` — the first-block / dual-block cache.  ParaAttention
  page, "First Block Cache": the relative L1 change of the residual of the
  first block(s) against the stored residual decides; when it is small enough
  the cached residual of the remaining blocks is reused.  vLLM-Omni cache-dit
  page, "DBCache" key parameters and the "DiffusionCacheConfig" table: caching
  is disabled for the first ``max_warmup_steps`` steps, at most
  ``max_cached_steps`` steps are served from the cache in all (-1: no limit),
  at most ``max_continuous_cached_steps`` in a row, and a step is cached only
  when the difference is below ``residual_diff_threshold``.
* ``teacache_schedule`` — TMAP image-to-video page, "TeaCache" (difference
  estimation and rescaling; inference flow): the relative L1 distance of the
  timestep-modulated input between adjacent steps is mapped through a
  calibrated polynomial and summed; while the sum stays below the threshold
  the cache is reused, otherwise the step computes and the sum restarts.

Readings where the pages leave a step open (each also listed in the design
notes): a step with no stored residual computes; the stored residual is the
one of the last computed step (a cached step produces none); the comparison
is strict (``rel < threshold``, the threshold rounded to fp32 first, the
type the library takes it in); a negative ``max_continuous_cached_steps``
means no limit, as -1 does for ``max_cached_steps``; during warm-up, and with
no stored residual, the difference is not evaluated (reported as NaN); the
TeaCache sum restarts at zero on every computed step; polynomial coefficients
are given in ascending powers.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

# Decision codes (0 = reuse the cache; every other value = compute, and why).
USE_CACHE = 0
WARMUP = 1
NO_PREV = 2
ABOVE_THRESHOLD = 3
MAX_CACHED = 4
MAX_CONTINUOUS = 5


@dataclass(frozen=True)
class CachePolicy:
    """Defaults of the vLLM-Omni cache-dit page's "DiffusionCacheConfig" table."""
    max_warmup_steps: int = 4
    max_cached_steps: int = -1
    max_continuous_cached_steps: int = 3
    residual_diff_threshold: float = 0.24


def fbcache_decide(step: int, rel: float, has_prev: bool, cached_steps: int, continuous: int,
                   policy: CachePolicy) -> int:
    """One decision of the first-block cache from the counters before the step."""
    if step < policy.max_warmup_steps:
        return WARMUP
    if not has_prev:
        return NO_PREV
    if not rel < float(np.float32(policy.residual_diff_threshold)):
        return ABOVE_THRESHOLD
    if policy.max_cached_steps >= 0 and cached_steps >= policy.max_cached_steps:
        return MAX_CACHED
    if policy.max_continuous_cached_steps >= 0 and continuous >= policy.max_continuous_cached_steps:
        return MAX_CONTINUOUS
    return USE_CACHE


def fbcache_decisions(rels, policy: CachePolicy):
    """Decisions for a given sequence of per-step differences.

    ``rels[s]`` is the difference step ``s`` would see against the stored
    residual; it is ignored where the policy does not evaluate it.  Step 0
    has no stored residual.  Returns the list of decision codes.
    """
    out = []
    has_prev, cached, cont = False, 0, 0
    for s, rel in enumerate(rels):
        d = fbcache_decide(s, rel, has_prev, cached, cont, policy)
        out.append(d)
        if d == USE_CACHE:
            cached += 1
            cont += 1
        else:
            cont = 0
            has_prev = True
    return out


def fbcache_schedule(residuals, policy: CachePolicy, rel_fn):
    """Run the policy over a sequence of first-block residuals.

    ``rel_fn(cur, prev) -> float`` is the relative L1 difference (the oracle's
    ``fbc_rel_l1``).  A computed step stores its residual; a cached step
    leaves the stored one in place.  Returns ``(rels, decisions, counters)``
    with ``rels[s]`` NaN where the difference was not evaluated and
    ``counters = (steps, cached_steps, continuous_cached, has_prev)`` after
    the last step.
    """
    rels, decisions = [], []
    prev = None
    cached, cont = 0, 0
    for s, cur in enumerate(residuals):
        evaluated = s >= policy.max_warmup_steps and prev is not None
        rel = rel_fn(cur, prev) if evaluated else math.nan
        d = fbcache_decide(s, rel, prev is not None, cached, cont, policy)
        rels.append(rel)
        decisions.append(d)
        if d == USE_CACHE:
            cached += 1
            cont += 1
        else:
            cont = 0
            prev = cur
    return rels, decisions, (len(decisions), cached, cont, prev is not None)


def polyval_ascending(coeffs, x: float) -> float:
    """c[0] + c[1] x + c[2] x^2 + ... in fp64 (Horner's scheme)."""
    acc = 0.0
    for c in reversed(list(coeffs)):
        acc = acc * x + float(c)
    return acc


def teacache_schedule(inputs, coeffs, threshold: float, rel_fn):
    """Run the TeaCache accumulator over a sequence of modulated inputs.

    Every step stores its input (the modulated input is computed on every
    step, cached or not).  Returns ``(rels, rescaled, accs, decisions)``:
    ``accs[s]`` is the sum after step ``s`` (zero after a computed step).
    """
    rels, resc, accs, decisions = [], [], [], []
    prev = None
    acc = 0.0
    for cur in inputs:
        if prev is None:
            rel, r, d = math.nan, math.nan, NO_PREV
            acc = 0.0
        else:
            rel = rel_fn(cur, prev)
            r = polyval_ascending(coeffs, rel)
            acc += r
            if acc < float(np.float32(threshold)):
                d = USE_CACHE
            else:
                d = ABOVE_THRESHOLD
                acc = 0.0
        rels.append(rel)
        resc.append(r)
        accs.append(acc)
        decisions.append(d)
        prev = cur
    return rels, resc, accs, decisions
