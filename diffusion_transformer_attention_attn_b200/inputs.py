"""Seeded synthetic inputs for the attention and first-block-cache workloads.

This module only draws random numbers and encodes them as bf16 / fp32 bit
patterns.  It holds none of the method's arithmetic and serves both the CUDA
path (tests, bench) and the fp64 oracle, so both read identical bits.

Recipe (numpy PCG64 streams keyed by ``SeedSequence`` entropy lists, so the
pieces can be drawn in parallel threads and still be identical every run):
  * Q, K, V: one stream per tensor t (0, 1, 2) and head (b, h), keyed
    [seed, t, b, h]; N(0, 1) drawn in fp32 and rounded to bf16 (round to
    nearest even) on the host;
  * per-channel K offsets: one stream keyed [seed, 3], N(0, std^2) per
    (b, h, channel), added to every token of K in fp32 before the bf16
    rounding; zeroed Q channels / token ranges are set afterwards;
  * residual pairs: 2^24-element chunks c, r_prev from [seed, 0, c] and the
    drift from [seed, 1, c].

Workload shapes follow the token counts the pages quote: FLUX.1-dev at 1024x1024
(4096 image + 512 text tokens, ParaAttention page, "First Block Cache"; Z-Image
page: single-stream joint tokens), a 704x1280x49 video (13x44x80 latent tokens,
vLLM-Omni "Diffusion Attention Backends"), and HunyuanVideo 720p x 129 frames
(33x45x80 latent + 256 text tokens, ParaAttention page, benchmark table).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

_THREADS = max(1, min(16, os.cpu_count() or 1))


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def _parallel(fn, items):
    items = list(items)
    if len(items) <= 1 or _THREADS == 1:
        return [fn(i) for i in items]
    with ThreadPoolExecutor(_THREADS) as ex:
        return list(ex.map(fn, items))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 (exact widening)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass(frozen=True)
class AttnCase:
    name: str
    B: int
    H: int
    N: int
    d: int
    k_offset_std: float = 0.0      # per-(b,h,channel) offset added to every K token
    zero_q_channel: int = -1       # channel of Q set to 0 for all tokens (-1: none)
    zero_q_tokens: tuple = ()      # [lo, hi) token range of Q set to 0
    seed: int = 0

    @property
    def flops(self) -> float:
        """4*B*H*N^2*d: two contractions (QK^T and PV) of 2*N^2*d each."""
        return 4.0 * self.B * self.H * self.N * self.N * self.d


@dataclass(frozen=True)
class FbcCase:
    name: str
    rows: int
    cols: int
    dtype: str            # "f32" or "bf16"
    drift_std: float
    threshold: float
    seed: int = 0

    @property
    def n(self) -> int:
        return self.rows * self.cols


# The five workloads (tiny, image, 8-bit image, mid video, long video).
TINY = AttnCase("tiny_b1h2n256d64", 1, 2, 256, 64)
IMAGE = AttnCase("image1024_b1h24n4608d128", 1, 24, 4608, 128)
IMAGE_Q8 = AttnCase("image1024_q8_b1h24n4608d128", 1, 24, 4608, 128,
                    k_offset_std=5.0, zero_q_channel=7, zero_q_tokens=(640, 768))
VIDEO_MID = AttnCase("video704p49_b1h24n45760d128", 1, 24, 45760, 128)
VIDEO_LONG = AttnCase("video720p129_b1h24n119056d128", 1, 24, 119056, 128, k_offset_std=2.0)

FBC_TINY = FbcCase("fbc_256x128_f32", 256, 128, "f32", 0.05, 0.08)
FBC_IMAGE = FbcCase("fbc_4608x3072_bf16", 4608, 3072, "bf16", 0.03, 0.08)
# Residual of the long-video workload: one row per token, H*d = 3072 wide.
FBC_VIDEO_LONG = FbcCase("fbc_119056x3072_bf16", 119056, 3072, "bf16", 0.03, 0.08)

ATTN_CASES = {c.name: c for c in (TINY, IMAGE, IMAGE_Q8, VIDEO_MID, VIDEO_LONG)}
FBC_CASES = {c.name: c for c in (FBC_TINY, FBC_IMAGE, FBC_VIDEO_LONG)}


def attn_inputs(case: AttnCase, N: int | None = None):
    """Q, K, V as bf16 bit arrays of shape [B, H, N, d] (uint16).

    ``N`` overrides the case's sequence length (ragged-size parity cases reuse
    a case's distribution at other lengths).
    """
    N = case.N if N is None else N
    shape = (case.B, case.H, N, case.d)
    mu = None
    if case.k_offset_std > 0.0:
        mu = _rng(case.seed, 3).standard_normal((case.B, case.H, case.d), dtype=np.float32)
        mu *= np.float32(case.k_offset_std)
    out = [np.empty(shape, dtype=np.uint16) for _ in range(3)]

    def fill(item):
        t, b, h = item
        x = _rng(case.seed, t, b, h).standard_normal((N, case.d), dtype=np.float32)
        if t == 1 and mu is not None:
            x += mu[b, h][None, :]
        out[t][b, h] = bf16_bits(x)

    _parallel(fill, [(t, b, h) for t in range(3) for b in range(case.B) for h in range(case.H)])
    q, k, v = out
    if case.zero_q_channel >= 0 and case.zero_q_channel < case.d:
        q[..., case.zero_q_channel] = 0
    if case.zero_q_tokens:
        lo, hi = case.zero_q_tokens
        q[:, :, min(lo, N):min(hi, N), :] = 0
    return q, k, v


_CHUNK = 1 << 24


def fbc_inputs(case: FbcCase):
    """(r_cur, r_prev): r_prev ~ N(0,1), r_cur = r_prev + N(0, drift^2).

    fp32 cases return float32 arrays; bf16 cases return bf16 bit arrays (uint16),
    with r_prev rounded to bf16 first and r_cur formed in fp32 from that bf16
    value plus the drift, rounded once to bf16.
    """
    n = case.n
    if case.dtype not in ("f32", "bf16"):
        raise ValueError(f"unknown dtype {case.dtype}")
    odt = np.float32 if case.dtype == "f32" else np.uint16
    cur = np.empty(n, dtype=odt)
    prev = np.empty(n, dtype=odt)

    def fill(c):
        s, e = c * _CHUNK, min(n, (c + 1) * _CHUNK)
        p = _rng(case.seed, 0, c).standard_normal(e - s, dtype=np.float32)
        drift = _rng(case.seed, 1, c).standard_normal(e - s, dtype=np.float32) * np.float32(case.drift_std)
        if case.dtype == "f32":
            prev[s:e] = p
            cur[s:e] = p + drift
        else:
            pb = bf16_bits(p)
            prev[s:e] = pb
            cur[s:e] = bf16_bits(bf16_to_f32(pb) + drift)

    _parallel(fill, range((n + _CHUNK - 1) // _CHUNK))
    return cur.reshape(case.rows, case.cols), prev.reshape(case.rows, case.cols)


@dataclass(frozen=True)
class TrajectoryCase:
    """A sequence of per-step tensors (first-block residuals or modulated
    inputs) over the denoising steps of one generation: each step adds a
    random drift whose size is drawn per step from [drift_lo, drift_hi]."""
    name: str
    rows: int
    cols: int
    dtype: str            # "f32" or "bf16"
    steps: int
    drift_lo: float
    drift_hi: float
    seed: int = 0

    @property
    def n(self) -> int:
        return self.rows * self.cols


# 28 steps (the FLUX.1-dev step count of the ParaAttention page) over a
# 1024-token, 3072-wide residual; a ragged fp32 case; the long-video residual
# width over 30 steps (the HunyuanVideo step count) at a reduced token count.
TRAJ_IMAGE = TrajectoryCase("traj_flux28_1024x3072_bf16", 1024, 3072, "bf16", 28, 0.02, 0.2)
TRAJ_RAGGED = TrajectoryCase("traj_ragged_999x37_f32", 999, 37, "f32", 24, 0.01, 0.3, seed=5)
TRAJ_VIDEO = TrajectoryCase("traj_video30_4096x3072_bf16", 4096, 3072, "bf16", 30, 0.02, 0.15, seed=11)


def trajectory(case: TrajectoryCase):
    """List of ``steps`` arrays [rows, cols]: x_0 ~ N(0,1),
    x_s = x_{s-1} + a_s * N(0,1) with a_s ~ U(drift_lo, drift_hi).

    fp32 cases return float32 arrays; bf16 cases bf16 bit arrays (uint16),
    each step formed in fp32 from the previous bf16 value and rounded once.
    """
    if case.dtype not in ("f32", "bf16"):
        raise ValueError(f"unknown dtype {case.dtype}")
    n = case.n
    amp = _rng(case.seed, 7).uniform(case.drift_lo, case.drift_hi, size=case.steps).astype(np.float32)
    out = []
    x = _rng(case.seed, 8, 0).standard_normal(n, dtype=np.float32)
    for s in range(case.steps):
        if s > 0:
            x = x + amp[s] * _rng(case.seed, 8, s).standard_normal(n, dtype=np.float32)
        if case.dtype == "bf16":
            b = bf16_bits(x)
            x = bf16_to_f32(b)
            out.append(b.reshape(case.rows, case.cols))
        else:
            out.append(x.reshape(case.rows, case.cols).copy())
    return out


def sample_rows(N: int, count: int, seed: int = 1) -> np.ndarray:
    """Sorted distinct query-row indices for sampled parity checks at full size.

    Always includes the first and the last row (the ragged tail)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    count = min(count, N)
    rows = set(rng.choice(N, size=count, replace=False).tolist())
    rows.discard(0)
    rows.discard(N - 1)
    rows = sorted(rows)[: max(0, count - 2)]
    return np.array(sorted({0, N - 1, *rows}), dtype=np.int64)
