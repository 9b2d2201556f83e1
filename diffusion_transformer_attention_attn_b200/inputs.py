"""Seeded synthetic inputs for the attention and first-block-cache workloads.

This module only draws random numbers and encodes them as bf16 / fp32 bit
patterns.  It holds none of the method's arithmetic and serves both the CUDA
path (tests, bench) and the fp64 oracle, so both read identical bits.

Recipe (one ``numpy.random.Generator(PCG64(seed))`` per case):
  * draw order Q, K, V, then extras (per-channel K offsets, zeroed channels);
  * values drawn in fp32, rounded to bf16 round-to-nearest-even on the host.

Workload shapes follow the token counts the pages quote: FLUX.1-dev at 1024x1024
(4096 image + 512 text tokens, ParaAttention page, "First Block Cache"; Z-Image
page: single-stream joint tokens), a 704x1280x49 video (13x44x80 latent tokens,
vLLM-Omni "Diffusion Attention Backends"), and HunyuanVideo 720p x 129 frames
(33x45x80 latent + 256 text tokens, ParaAttention page, benchmark table).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


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


def _normal_bf16(rng: np.random.Generator, shape, std: float = 1.0,
                 chunk: int = 1 << 24) -> np.ndarray:
    """N(0, std^2) drawn in fp32, returned as bf16 bits, chunked to bound memory."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        x = rng.standard_normal(e - s, dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        out[s:e] = bf16_bits(x)
    return out.reshape(shape)


def attn_inputs(case: AttnCase, N: int | None = None):
    """Q, K, V as bf16 bit arrays of shape [B, H, N, d] (uint16).

    ``N`` overrides the case's sequence length (ragged-size parity cases reuse
    a case's distribution at other lengths).
    """
    N = case.N if N is None else N
    shape = (case.B, case.H, N, case.d)
    rng = np.random.Generator(np.random.PCG64(case.seed))
    q = _normal_bf16(rng, shape)
    k = _normal_bf16(rng, shape)
    v = _normal_bf16(rng, shape)
    if case.k_offset_std > 0.0:
        mu = rng.standard_normal((case.B, case.H, 1, case.d), dtype=np.float32)
        mu *= np.float32(case.k_offset_std)
        # K = N(0,1) + mu, formed in fp32 from the bf16 draw, rounded once to bf16.
        kb = k.reshape(case.B, case.H, N, case.d)
        for b in range(case.B):
            for h in range(case.H):
                kb[b, h] = bf16_bits(bf16_to_f32(kb[b, h]) + mu[b, h])
    if case.zero_q_channel >= 0 and case.zero_q_channel < case.d:
        q[..., case.zero_q_channel] = 0
    if case.zero_q_tokens:
        lo, hi = case.zero_q_tokens
        q[:, :, min(lo, N):min(hi, N), :] = 0
    return q, k, v


def fbc_inputs(case: FbcCase):
    """(r_cur, r_prev): r_prev ~ N(0,1), r_cur = r_prev + N(0, drift^2).

    fp32 cases return float32 arrays; bf16 cases return bf16 bit arrays (uint16),
    with r_cur formed in fp32 from the bf16 r_prev and rounded once to bf16.
    """
    rng = np.random.Generator(np.random.PCG64(case.seed))
    n = case.n
    if case.dtype == "f32":
        prev = rng.standard_normal(n, dtype=np.float32)
        drift = rng.standard_normal(n, dtype=np.float32) * np.float32(case.drift_std)
        cur = (prev + drift).astype(np.float32)
        return cur.reshape(case.rows, case.cols), prev.reshape(case.rows, case.cols)
    if case.dtype == "bf16":
        prev = _normal_bf16(rng, (n,))
        cur = np.empty(n, dtype=np.uint16)
        chunk = 1 << 24
        for s in range(0, n, chunk):
            e = min(n, s + chunk)
            drift = rng.standard_normal(e - s, dtype=np.float32) * np.float32(case.drift_std)
            cur[s:e] = bf16_bits(bf16_to_f32(prev[s:e]) + drift)
        return cur.reshape(case.rows, case.cols), prev.reshape(case.rows, case.cols)
    raise ValueError(f"unknown dtype {case.dtype}")


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
