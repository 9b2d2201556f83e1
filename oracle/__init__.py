"""fp64 CPU oracle (ctypes wrapper around ``dit_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``, never by the CUDA library or its
Python binding.  It shares no code with the CUDA path.

Every function here follows the definitions cited in ``dit_oracle.c``:
softmax attention (Z-Image FlashAttention-2 page, opening section; TMAP
image-to-video page, FLOP table), the first-block-cache residual difference
(ParaAttention page, "First Block Cache") and the 8-bit quantiser with its
zero-scale guard (TMAP page, "optimising operator details").

``emulated_q8_attention`` and ``attention_from_codes`` replay the quantised
arithmetic in fp64 to separate quantisation error from kernel error; they are
never the parity reference (that is the exact fp64 attention on the
unquantised inputs).  They are pinned on inputs whose every code is exact, with
a different scale in each Q and K block, where they must equal the exact
attention.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dit_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_i64 = ctypes.c_int64
_p = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile the oracle with gcc + OpenMP (no fast-math: IEEE fp64/fp32)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.oracle_attn_f64.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64, _i64, ctypes.c_double, _p, _i64]
        lib.oracle_attn_bf16in.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64, _i64, ctypes.c_double, _p, _i64]
        lib.oracle_attn_lse_bf16in.argtypes = [_p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _i64, ctypes.c_double]
        lib.oracle_fbc_rel_l1.argtypes = [_p, _p, _i64, ctypes.c_int, ctypes.c_double, _p, _p]
        lib.oracle_channel_mean.argtypes = [_p, _i64, _i64, _i64, _p]
        lib.oracle_quant_int8_blocks.argtypes = [_p, _i64, _i64, _i64, _i64, _p, _p, _p]
        lib.oracle_quant_e4m3_channels.argtypes = [_p, _i64, _i64, _i64, _p, _p]
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_float
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def attention(q, k, v, scale: float | None = None, rows=None) -> np.ndarray:
    """O = softmax(scale * Q K^T) V in fp64.

    q, k, v: [B, H, N, d] as float64 arrays, or uint16 arrays of bf16 bits
    (widened exactly).  ``scale`` defaults to 1/sqrt(d) computed in fp32 and
    widened, the value the CUDA path receives.  ``rows``: optional query-row
    indices; the result is then [B, H, len(rows), d].
    """
    B, H, N, d = q.shape
    assert k.shape == (B, H, N, d) and v.shape == (B, H, N, d)
    if scale is None:
        scale = float(np.float32(1.0) / np.sqrt(np.float32(d)))
    nrows = N
    rows_arr = None
    if rows is not None:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        assert rows_arr.ndim == 1 and (rows_arr >= 0).all() and (rows_arr < N).all()
        nrows = len(rows_arr)
    out = np.empty((B, H, nrows, d), dtype=np.float64)
    lib = _load()
    rp = _ptr(rows_arr) if rows_arr is not None else None
    if q.dtype == np.uint16:
        q, k, v = (np.ascontiguousarray(t, dtype=np.uint16) for t in (q, k, v))
        rc = lib.oracle_attn_bf16in(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d,
                                    float(scale), rp, nrows)
    else:
        q, k, v = (np.ascontiguousarray(t, dtype=np.float64) for t in (q, k, v))
        rc = lib.oracle_attn_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d,
                                 float(scale), rp, nrows)
    if rc != 0:
        raise RuntimeError(f"oracle attention failed ({rc})")
    return out


def fbc_rel_l1(cur, prev, threshold: float):
    """(rel, skip) for two residuals: fp32 arrays or uint16 bf16 bit arrays."""
    cur = np.ascontiguousarray(cur).reshape(-1)
    prev = np.ascontiguousarray(prev).reshape(-1)
    assert cur.shape == prev.shape and cur.dtype == prev.dtype
    if cur.dtype == np.float32:
        dt = 0
    elif cur.dtype == np.uint16:
        dt = 1
    else:
        raise TypeError(cur.dtype)
    rel = ctypes.c_double()
    skip = ctypes.c_int32()
    thr = float(np.float32(threshold))
    rc = _load().oracle_fbc_rel_l1(_ptr(cur), _ptr(prev), cur.size, dt, thr,
                                   ctypes.byref(rel), ctypes.byref(skip))
    if rc != 0:
        raise RuntimeError("oracle fbc failed")
    return rel.value, int(skip.value)


def channel_mean(x: np.ndarray) -> np.ndarray:
    """[B, H, N, d] bf16 bits -> [B, H, d] fp32 means (fp64 sum, one rounding)."""
    B, H, N, d = x.shape
    x = np.ascontiguousarray(x, dtype=np.uint16)
    out = np.empty((B, H, d), dtype=np.float32)
    _load().oracle_channel_mean(_ptr(x), B * H, N, d, _ptr(out))
    return out


def quant_int8_blocks(x: np.ndarray, blk: int, mean: np.ndarray | None = None):
    """Per-block INT8 codes [B,H,N,d] and scales [B,H,ceil(N/blk)] (fp32 mirror)."""
    B, H, N, d = x.shape
    x = np.ascontiguousarray(x, dtype=np.uint16)
    nblk = (N + blk - 1) // blk
    codes = np.empty((B, H, N, d), dtype=np.int8)
    scales = np.empty((B, H, nblk), dtype=np.float32)
    mp = None
    if mean is not None:
        mean = np.ascontiguousarray(mean, dtype=np.float32)
        assert mean.shape == (B, H, d)
        mp = _ptr(mean)
    rc = _load().oracle_quant_int8_blocks(_ptr(x), B * H, N, d, blk, mp, _ptr(codes), _ptr(scales))
    if rc != 0:
        raise RuntimeError("oracle quant failed")
    return codes, scales


def quant_e4m3_channels(x: np.ndarray):
    """Per-channel e4m3 codes [B,H,N,d] (uint8) and scales [B,H,d] (fp32 mirror)."""
    B, H, N, d = x.shape
    x = np.ascontiguousarray(x, dtype=np.uint16)
    codes = np.empty((B, H, N, d), dtype=np.uint8)
    scales = np.empty((B, H, d), dtype=np.float32)
    _load().oracle_quant_e4m3_channels(_ptr(x), B * H, N, d, _ptr(codes), _ptr(scales))
    return codes, scales


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.asarray(x, dtype=np.float32).reshape(-1)
    return np.array([lib.oracle_e4m3_encode(float(t)) for t in flat], dtype=np.uint8).reshape(np.shape(x))


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.asarray(b, dtype=np.uint8).reshape(-1)
    return np.array([lib.oracle_e4m3_decode(int(t)) for t in flat], dtype=np.float32).reshape(np.shape(b))


def emulated_q8_attention(q, k, v, scale: float | None = None, smooth_k: bool = True,
                          rows=None) -> np.ndarray:
    """fp64 attention over the dequantised 8-bit inputs.

    Replays the quantiser (Q per 128 tokens, K per 64 tokens after the optional
    channel-mean subtraction, V per channel e4m3) and runs the exact fp64
    attention on code * scale.  P's own rounding is not modelled.
    """
    B, H, N, d = q.shape
    qc, qs = quant_int8_blocks(q, 128)
    mean = channel_mean(k) if smooth_k else None
    kc, ks = quant_int8_blocks(k, 64, mean)
    vc, vs = quant_e4m3_channels(v)
    tok = np.arange(N)
    qd = qc.astype(np.float64) * qs[:, :, tok // 128, None].astype(np.float64)
    kd = kc.astype(np.float64) * ks[:, :, tok // 64, None].astype(np.float64)
    vd = e4m3_decode(vc).astype(np.float64) * vs[:, :, None, :].astype(np.float64)
    return attention(qd, kd, vd, scale=scale, rows=rows)


def _widen(x) -> np.ndarray:
    """fp32 array, or uint16 array of bf16 bits, to fp64 (exact)."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if x.dtype in (np.float32, np.float64):
        return x.astype(np.float64)
    raise TypeError(x.dtype)


def compare_stats(ref, test, segments: int = 1):
    """Error of ``test`` against ``ref`` per contiguous segment, in fp64.

    TMAP image-to-video page, "keeping video quality": the attention error of
    each layer over the denoising steps is what singles out the layers whose
    8-bit attention is switched back to 16 bits.  The error measures are the
    relative L1 distance sum|test - ref| / sum|ref|, the cosine similarity
    sum(ref*test) / sqrt(sum(ref^2) sum(test^2)) and max|test - ref|.
    Both inputs are fp32 arrays or uint16 arrays of bf16 bits with the same
    number of elements, which ``segments`` divides.  Conventions for empty
    norms: rel_l1 is 0 if both sums are 0 and +inf if only sum|ref| is;
    cosine is 1 if both vectors are zero and 0 if exactly one is.
    Returns three float64 arrays of length ``segments``.
    """
    a = _widen(ref).reshape(segments, -1)
    b = _widen(test).reshape(segments, -1)
    assert a.shape == b.shape
    rel = np.empty(segments)
    cos = np.empty(segments)
    mx = np.empty(segments)
    for s in range(segments):
        x, y = a[s], b[s]
        num = np.abs(y - x).sum()
        den = np.abs(x).sum()
        rel[s] = num / den if den > 0 else (np.inf if num > 0 else 0.0)
        xx, yy, xy = (x * x).sum(), (y * y).sum(), (x * y).sum()
        if xx > 0 and yy > 0:
            cos[s] = xy / np.sqrt(xx * yy)
        else:
            cos[s] = 1.0 if (xx == 0 and yy == 0) else 0.0
        mx[s] = np.abs(y - x).max() if x.size else 0.0
    return rel, cos, mx


def attention_lse(q, k, v, scale: float | None = None):
    """(O, lse) for bf16-bit inputs q [B,H,Nq,d], k and v [B,H,Nkv,d], in fp64.

    lse[b,h,i] = ln sum_j exp(scale * q_i . k_j), the log-sum-exp of the row's
    logits.  ParaAttention page, "Context Parallelism": the keys of one
    attention may be split into chunks; these two results per chunk are what
    ``merge_partials`` combines.
    """
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    assert k.shape == (B, H, Nkv, d) and v.shape == k.shape
    if scale is None:
        scale = float(np.float32(1.0) / np.sqrt(np.float32(d)))
    q, k, v = (np.ascontiguousarray(t, dtype=np.uint16) for t in (q, k, v))
    out = np.empty((B, H, Nq, d), dtype=np.float64)
    lse = np.empty((B, H, Nq), dtype=np.float64)
    rc = _load().oracle_attn_lse_bf16in(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Nq, Nkv, d,
                                        float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle attention failed ({rc})")
    return out, lse


def merge_partials(outs, lses):
    """Attention over the union of key chunks from the per-chunk results, fp64.

    With L_c the log-sum-exp of chunk c and O_c its normalised output:
    L = ln sum_c exp(L_c) and O = sum_c exp(L_c - L) O_c (each chunk's
    softmax denominator is exp(L_c); the union's is their sum).  The largest
    L_c is subtracted before exponentiating.
    outs: list of [..., d] arrays; lses: list of matching [...] arrays.
    """
    L = np.stack([np.asarray(x, dtype=np.float64) for x in lses])
    O = np.stack([np.asarray(x, dtype=np.float64) for x in outs])
    top = L.max(axis=0)
    w = np.exp(L - top[None])
    den = w.sum(axis=0)
    out = (w[..., None] * O).sum(axis=0) / den[..., None]
    return out, top + np.log(den)


def fbc_sums(cur, prev):
    """(sum|cur - prev|, sum|prev|) in fp64: the two sums behind fbc_rel_l1.

    A residual split across devices reduces to rel with one all-reduce of
    these two numbers (ParaAttention page, "First Block Cache", with the
    residual sharded as the sequence is in "Context Parallelism")."""
    c = _widen(np.ascontiguousarray(cur).reshape(-1))
    p = _widen(np.ascontiguousarray(prev).reshape(-1))
    return float(np.abs(c - p).sum()), float(np.abs(p).sum())


def rel_from_sums(num: float, den: float, threshold: float):
    """(rel, skip) from the two sums, with fbc_rel_l1's conventions."""
    if den > 0:
        rel = num / den
    else:
        rel = float("inf") if num > 0 else 0.0
    return rel, int(rel < float(np.float32(threshold)))


# ---- 8-bit pre-pass over a token-sharded sequence --------------------------
# Under Ulysses context parallelism (ParaAttention page, "Context
# Parallelism"; TMAP image-to-video page, sequence parallelism combined with
# the 8-bit attention) each device holds a slice of the tokens.  The K mean and
# the V channel maxima span all tokens, so each device reduces its slice to
# per-channel sums and maxima, the devices combine them, and each quantises its
# own tokens with the combined statistics; the 1-byte codes then travel in the
# all-to-all instead of the bf16 values.

def k_channel_sums(k: np.ndarray) -> np.ndarray:
    """[B, H, N, d] bf16 bits -> [B, H, d] fp64 sums over the tokens."""
    return _widen(k).sum(axis=2)


def channel_amax(v: np.ndarray) -> np.ndarray:
    """[B, H, N, d] bf16 bits -> [B, H, d] fp32 max |v| over the tokens."""
    return np.abs(_widen(v)).max(axis=2).astype(np.float32)


def mean_from_sums(sums: np.ndarray, n_total: int) -> np.ndarray:
    """fp64 sums / N, rounded once to fp32 (the rounding of channel_mean)."""
    return (np.asarray(sums, dtype=np.float64) / float(n_total)).astype(np.float32)


def quant_e4m3_with_amax(x: np.ndarray, amax: np.ndarray):
    """Per-channel e4m3 codes of x [B,H,N,d] (bf16 bits) with the channel maxima
    given ([B,H,d] fp32): scale = amax/448 and inv = 448/amax as fp32
    divisions, code = e4m3(x·inv) (fp32 product); amax = 0, or an amax whose
    inverse 448/amax is not a finite fp32 number, gives zero codes and scales
    (the zero-scale guard).  Returns (codes, scales)."""
    amax = np.asarray(amax, dtype=np.float32)
    with np.errstate(divide="ignore", over="ignore"):
        inv_raw = (np.float32(448.0) / amax).astype(np.float32)
        ok = (amax > 0) & np.isfinite(inv_raw)
        scale = np.where(ok, amax / np.float32(448.0), np.float32(0.0)).astype(np.float32)
        inv = np.where(ok, inv_raw, np.float32(0.0)).astype(np.float32)
    xf = _widen(x).astype(np.float32)
    prod = (xf * inv[:, :, None, :]).astype(np.float32)
    return e4m3_encode(prod), scale


def attention_from_codes(qc, qs, kc, ks, v, vs=None, scale: float | None = None, rows=None) -> np.ndarray:
    """fp64 attention over dequantised codes: Q = qc·qs (per 128 tokens),
    K = kc·ks (per 64 tokens), V = e4m3(v)·vs per channel when vs is given,
    else v as bf16 bits.  The scale defaults to the fp32 1/sqrt(d)."""
    B, H, N, d = qc.shape
    tok = np.arange(N)
    qd = qc.astype(np.float64) * qs[:, :, tok // 128, None].astype(np.float64)
    kd = kc.astype(np.float64) * ks[:, :, tok // 64, None].astype(np.float64)
    if vs is not None:
        vd = e4m3_decode(v).astype(np.float64) * vs[:, :, None, :].astype(np.float64)
    else:
        vd = _widen(v)
    if scale is None:
        scale = float(np.float32(1.0) / np.sqrt(np.float32(d)))
    return attention(qd, kd, vd, scale=scale, rows=rows)
