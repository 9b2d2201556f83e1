"""Python binding of libditattn.so, the B200 (sm_100a) diffusion-transformer
attention library.

Argument marshalling only: every step of every call runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  There
is no fallback: if the library is missing, importing the binding's entry
points raises.

Entry points (same names as the C ABI in ``include/dit_attn.h``):
  * ``dit_attn_fwd(q, k, v, o=None, scale=None)``  — bf16 softmax attention
  * ``dit_attn_fwd_ex(q, k, v, ..., lse=...)``      — Nq queries x Nkv keys, optional log-sum-exp
  * ``dit_attn_merge(o_parts, lse_parts)``          — attention over the union of key chunks
  * ``dit_attn_fwd_q8(q, k, v, ...)``              — 8-bit attention (INT8 QKᵀ, FP8 or bf16 PV)
  * ``dit_attn_q8_quantize(q, k, v, ...)``         — its pre-pass alone
  * ``fbc_rel_l1(r_cur, r_prev, threshold, ...)``   — first-block-cache decision
  * ``fbc_rel_l1_noalloc(...)``                     — the same, allocating nothing
  * ``dit_compare_stats(ref, test, segments)``       — rel-L1 / cosine / max error per segment
  * ``dit_get_device_status()``                     — device-side error word
  * ``dit_wait_selftest()``                         — makes a bounded wait run out (failure-path test)

and of ``include/dit_cache.h``:
  * ``fbcache_step(...)`` / ``teacache_step(...)``  — step-cache decisions kept on the device
  * ``dit_cache_state_reset``, ``dit_graph_*``     — device state and CUDA-graph conditional plumbing

Modules on top: ``step_cache`` (a captured denoising step that skips its
expensive part on cached steps) and ``context_parallel`` (Ulysses and ring
attention, the sharded cache decision, over ``torch.distributed``).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libditattn.so")

DIT_OK = 0
DIT_ERR_INVALID_ARG = 1
DIT_ERR_UNSUPPORTED = 2
DIT_ERR_WORKSPACE = 3
DIT_ERR_CUDA = 4
DIT_ERR_TIMEOUT = 5
DIT_DTYPE_F32 = 0
DIT_DTYPE_BF16 = 1
DIT_PV_FP8_E4M3 = 0
DIT_PV_BF16 = 1
PV_MODES = {"fp8": DIT_PV_FP8_E4M3, "bf16": DIT_PV_BF16}

# Every symbol include/dit_attn.h declares, with (restype, argtypes).
_p = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_f = ctypes.c_float
_sz = ctypes.c_size_t
SIGNATURES = {
    "dit_attn_fwd": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _p, _f, _p]),
    "dit_attn_fwd_ex": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p, _p, _f, _p]),
    "dit_attn_merge": (_i, [_p, _p, _i, _i, _i, _i, _i, _p, _p, _p, _p]),
    "dit_attn_q8_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "dit_attn_fwd_q8": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _p, _f, _i, _i, _p, _sz, _p]),
    "dit_attn_q8_quantize": (_i, [_p, _p, _p, _i, _i, _i, _i, _p, _i, _i, _p, _sz, _p]),
    "dit_attn_q8_workspace_layout": (_i, [_i, _i, _i, _i, _i, _p]),
    "dit_attn_q8_channel_stats": (_i, [_p, _p, _i, _i, _i, _i, _p, _i, _i, _p, _p, _p, _sz, _p]),
    "dit_attn_q8_quantize_global": (_i, [_p, _p, _p, _i, _i, _i, _i, _p, _i, _i, _p, _p, _i64, _p, _sz, _p]),
    "dit_attn_fwd_q8_prequantized": (_i, [_p, _sz, _p, _p, _i, _i, _i, _i, _p, _f, _i, _p]),
    "dit_attn_q8_quantize_scatter": (_i, [_p, _p, _p, _i, _i, _i, _i, _p, _i, _i, _p, _p, _i, _i, _p, _sz, _p, _sz,
                                          _p]),
    "fbc_rel_l1_workspace_bytes": (_sz, [_i64]),
    "fbc_rel_l1": (_i, [_p, _p, _i64, _i, _f, _p, _p, _p, _sz, _p]),
    "fbc_rel_l1_noalloc": (_i, [_p, _p, _i64, _i, _f, _p, _p, _p]),
    "fbc_rel_l1_sums": (_i, [_p, _p, _i64, _i, _p, _p, _sz, _p]),
    "fbc_rel_l1_finish": (_i, [_p, _f, _p, _p, _p]),
    "dit_compare_workspace_bytes": (_sz, [_i64, _i64, _i]),
    "dit_compare_stats": (_i, [_p, _p, _i64, _i64, _i, _p, _p, _sz, _p]),
    "dit_get_device_status": (_i, [_p]),
    "dit_wait_selftest": (_i, [_p, _p]),
    "dit_status_string": (ctypes.c_char_p, [_i]),
    # include/dit_cache.h
    "dit_cache_state_reset": (_i, [_p, _p]),
    "dit_cache_workspace_bytes": (_sz, [_i64]),
    "fbcache_step": (_i, [_p, _p, _i64, _i, _p, _p, _p, ctypes.c_int32, _i, ctypes.c_ulonglong, _p, _sz, _p]),
    "teacache_step": (_i, [_p, _p, _i64, _i, _p, ctypes.c_int32, _f, _p, _p, ctypes.c_int32, _i,
                           ctypes.c_ulonglong, _p, _sz, _p]),
    "dit_graph_capture_begin": (_i, [_p]),
    "dit_graph_cond_create": (_i, [_p, _p]),
    "dit_graph_cond_body_begin": (_i, [_p, ctypes.c_ulonglong, _p]),
    "dit_graph_cond_body_end": (_i, [_p]),
    "dit_graph_capture_end": (_i, [_p, _p]),
    "dit_graph_launch": (_i, [_p, _p]),
    "dit_graph_destroy": (_i, [_p]),
}

_lib = None


class DitError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def load_library(path: str = LIB_PATH):
    """Load libditattn.so and bind every declared symbol (raises if missing)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is not built; run `python -m diffusion_transformer_attention_attn_b200.build_lib`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().dit_status_string(int(status)).decode()


def _stream_ptr(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str):
    if status != DIT_OK:
        raise DitError(status, what)


def _same_layout(a, b) -> bool:
    """Same shape, and the same strides in every dimension longer than 1 (the
    stride of a length-1 dimension never addresses anything)."""
    return a.shape == b.shape and all(x == y or n == 1 for x, y, n in zip(a.stride(), b.stride(), a.shape))


def _attn_strides(t):
    """(b, h, n) element strides of a [B, H, N, d] tensor with unit d stride."""
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("expected a [B, H, N, d] tensor with contiguous d")
    return (ctypes.c_int64 * 3)(t.stride(0), t.stride(1), t.stride(2))


def dit_attn_fwd(q, k, v, o=None, scale: float | None = None, stream=None):
    """O = softmax(scale · Q Kᵀ) V for bf16 CUDA tensors [B, H, N, d] (d ∈ {64, 128}).

    q, k, v and o must share shape and strides.  Returns o.
    """
    import torch
    lib = load_library()
    if o is None:
        o = torch.empty_like(q)
    for t in (q, k, v, o):
        if t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError("dit_attn_fwd expects bf16 CUDA tensors")
        if not _same_layout(t, q):
            raise ValueError("q, k, v, o must share shape and strides")
    B, H, N, d = q.shape
    st = lib.dit_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), B, H, N, d,
                          _attn_strides(q), float(scale) if scale else 0.0, _stream_ptr(stream))
    _check(st, "dit_attn_fwd")
    return o


def dit_attn_fwd_ex(q, k, v, o=None, lse=None, scale: float | None = None, stream=None):
    """Attention of q [B, H, Nq, d] against k, v [B, H, Nkv, d] (bf16 CUDA
    tensors, unit stride in d; q and o share strides, k and v share theirs).

    ``lse``: None (not computed), True (allocate), or an fp32 CUDA tensor
    [B, H, Nq] to fill with each row's natural-log log-sum-exp.
    Returns (o, lse or None)."""
    import torch
    lib = load_library()
    if o is None:
        o = torch.empty_like(q)
    for t in (q, k, v, o):
        if t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError("dit_attn_fwd_ex expects bf16 CUDA tensors")
    if not _same_layout(o, q):
        raise ValueError("q and o must share shape and strides")
    if not _same_layout(v, k):
        raise ValueError("k and v must share shape and strides")
    B, H, Nq, d = q.shape
    if k.shape[0] != B or k.shape[1] != H or k.shape[3] != d:
        raise ValueError("k must be [B, H, Nkv, d] with q's B, H and d")
    Nkv = k.shape[2]
    if lse is True:
        lse = torch.empty(B, H, Nq, dtype=torch.float32, device=q.device)
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_contiguous() or lse.numel() != B * H * Nq):
        raise ValueError("lse must be a contiguous fp32 tensor of B*H*Nq elements")
    st = lib.dit_attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             lse.data_ptr() if lse is not None else None, B, H, Nq, Nkv, d,
                             _attn_strides(q), _attn_strides(k), float(scale) if scale else 0.0, _stream_ptr(stream))
    _check(st, "dit_attn_fwd_ex")
    return o, lse


def dit_attn_merge(o_parts, lse_parts, o=None, lse=None, stream=None):
    """Merge per-key-chunk outputs (bf16 [B, H, N, d], equal strides) and their
    log-sum-exps (fp32 [B, H, N]) into the attention over all chunks.
    ``lse``: None, True (allocate) or an fp32 tensor.  Returns (o, lse or None)."""
    import torch
    lib = load_library()
    n = len(o_parts)
    if n != len(lse_parts) or n < 1:
        raise ValueError("need as many log-sum-exps as outputs, at least one")
    ref = o_parts[0]
    for t in o_parts:
        if t.dtype != torch.bfloat16 or not _same_layout(t, ref):
            raise ValueError("o_parts must be bf16 tensors of one shape and stride")
    B, H, N, d = ref.shape
    for t in lse_parts:
        if t.dtype != torch.float32 or not t.is_contiguous() or t.numel() != B * H * N:
            raise ValueError("lse_parts must be contiguous fp32 tensors of B*H*N elements")
    if o is None:
        o = torch.empty_like(ref)
    if not _same_layout(o, ref):
        raise ValueError("o must share the parts' shape and strides")
    if lse is True:
        lse = torch.empty(B, H, N, dtype=torch.float32, device=ref.device)
    op = (ctypes.c_void_p * n)(*[t.data_ptr() for t in o_parts])
    lp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in lse_parts])
    st = lib.dit_attn_merge(op, lp, n, B, H, N, d, _attn_strides(ref), o.data_ptr(),
                            lse.data_ptr() if lse is not None else None, _stream_ptr(stream))
    _check(st, "dit_attn_merge")
    return o, lse


def _pv(pv_mode):
    return PV_MODES[pv_mode] if isinstance(pv_mode, str) else int(pv_mode)


def dit_attn_q8_workspace_bytes(B: int, H: int, N: int, d: int, pv_mode="fp8") -> int:
    return int(load_library().dit_attn_q8_workspace_bytes(B, H, N, d, _pv(pv_mode)))


def q8_workspace(B: int, H: int, N: int, d: int, pv_mode="fp8", device=None):
    """An (uninitialised) workspace tensor for the 8-bit path."""
    import torch
    n = dit_attn_q8_workspace_bytes(B, H, N, d, pv_mode)
    if n == 0:
        raise ValueError("unsupported shape for the 8-bit path")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


Q8_SEGMENTS = ("q_codes", "k_codes", "v_codes", "q_scale", "k_scale", "k_mean", "v_scale", "v_inv")


def dit_attn_q8_workspace_layout(B: int, H: int, N: int, d: int, pv_mode="fp8") -> dict:
    off = (ctypes.c_size_t * 8)()
    _check(load_library().dit_attn_q8_workspace_layout(B, H, N, d, _pv(pv_mode), off), "dit_attn_q8_workspace_layout")
    return dict(zip(Q8_SEGMENTS, (int(x) for x in off)))


def q8_views(workspace, B: int, H: int, N: int, d: int, pv_mode="fp8") -> dict:
    """Typed views of the pre-pass products inside a workspace tensor."""
    import torch
    off = dit_attn_q8_workspace_layout(B, H, N, d, pv_mode)
    n_q, n_k, e = (N + 127) // 128, (N + 63) // 64, B * H * N * d

    def seg(name, count, dtype, shape):
        nbytes = count * torch.empty((), dtype=dtype).element_size()
        return workspace[off[name]:off[name] + nbytes].view(dtype).view(shape)

    views = {
        "q_codes": seg("q_codes", e, torch.int8, (B, H, N, d)),
        "k_codes": seg("k_codes", e, torch.int8, (B, H, N, d)),
        "q_scale": seg("q_scale", B * H * n_q, torch.float32, (B, H, n_q)),
        "k_scale": seg("k_scale", B * H * n_k, torch.float32, (B, H, n_k)),
        "k_mean": seg("k_mean", B * H * d, torch.float32, (B, H, d)),
    }
    if _pv(pv_mode) == DIT_PV_FP8_E4M3:
        views["v_codes"] = seg("v_codes", e, torch.uint8, (B, H, N, d))
        views["v_scale"] = seg("v_scale", B * H * d, torch.float32, (B, H, d))
    return views


def _check_attn_tensors(q, k, v, o):
    import torch
    for t in (q, k, v) + ((o,) if o is not None else ()):
        if t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError("expected bf16 CUDA tensors")
        if not _same_layout(t, q):
            raise ValueError("q, k, v, o must share shape and strides")


def dit_attn_fwd_q8(q, k, v, o=None, scale: float | None = None, smooth_k: bool = True, pv_mode="fp8",
                    workspace=None, stream=None):
    """8-bit attention: INT8 Q (per 128 tokens) and K (per 64 tokens, optional
    channel-mean smoothing), S in int32, P·V in FP8 e4m3 or bf16.  bf16 CUDA
    tensors [B, H, N, d], d = 64 or 128.  Returns o."""
    import torch
    lib = load_library()
    if o is None:
        o = torch.empty_like(q)
    _check_attn_tensors(q, k, v, o)
    B, H, N, d = q.shape
    if workspace is None:
        workspace = q8_workspace(B, H, N, d, pv_mode, q.device)
    st = lib.dit_attn_fwd_q8(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), B, H, N, d, _attn_strides(q),
                             float(scale) if scale else 0.0, int(bool(smooth_k)), _pv(pv_mode),
                             workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    _check(st, "dit_attn_fwd_q8")
    return o


def dit_attn_q8_quantize(q, k, v, smooth_k: bool = True, pv_mode="fp8", workspace=None, stream=None):
    """Run only the 8-bit pre-pass; returns the workspace tensor."""
    lib = load_library()
    _check_attn_tensors(q, k, v, None)
    B, H, N, d = q.shape
    if workspace is None:
        workspace = q8_workspace(B, H, N, d, pv_mode, q.device)
    st = lib.dit_attn_q8_quantize(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, N, d, _attn_strides(q),
                                  int(bool(smooth_k)), _pv(pv_mode), workspace.data_ptr(), workspace.numel(),
                                  _stream_ptr(stream))
    _check(st, "dit_attn_q8_quantize")
    return workspace


def dit_attn_q8_channel_stats(k, v, smooth_k: bool = True, pv_mode="fp8", k_sum=None, v_amax=None, workspace=None,
                              stream=None):
    """Per-channel K sums (float64 [B,H,d]) and V maxima (float32 [B,H,d])
    over this slice of the tokens, for the devices of a Ulysses group to
    combine (sum, max).  Returns (k_sum, v_amax)."""
    import torch
    lib = load_library()
    _check_attn_tensors(k, k, v, None)
    B, H, N, d = k.shape
    if k_sum is None:
        k_sum = torch.empty(B, H, d, dtype=torch.float64, device=k.device)
    if v_amax is None:
        v_amax = torch.empty(B, H, d, dtype=torch.float32, device=k.device)
    if workspace is None:
        workspace = q8_workspace(B, H, N, d, pv_mode, k.device)
    st = lib.dit_attn_q8_channel_stats(k.data_ptr(), v.data_ptr(), B, H, N, d, _attn_strides(k), int(bool(smooth_k)),
                                       _pv(pv_mode), k_sum.data_ptr(), v_amax.data_ptr(), workspace.data_ptr(),
                                       workspace.numel(), _stream_ptr(stream))
    _check(st, "dit_attn_q8_channel_stats")
    return k_sum, v_amax


def dit_attn_q8_quantize_global(q, k, v, k_sum, v_amax, n_total: int, smooth_k: bool = True, pv_mode="fp8",
                                workspace=None, stream=None):
    """Quantise this slice of the tokens with statistics combined over all
    n_total tokens; returns the workspace (codes and scales)."""
    lib = load_library()
    _check_attn_tensors(q, k, v, None)
    B, H, N, d = q.shape
    if workspace is None:
        workspace = q8_workspace(B, H, N, d, pv_mode, q.device)
    st = lib.dit_attn_q8_quantize_global(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, N, d, _attn_strides(q),
                                         int(bool(smooth_k)), _pv(pv_mode), k_sum.data_ptr(), v_amax.data_ptr(),
                                         int(n_total), workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    _check(st, "dit_attn_q8_quantize_global")
    return workspace


def dit_attn_q8_quantize_scatter(q, k, v, k_sum, v_amax, rank: int, world: int, dst_workspaces, dst_workspace_bytes,
                                 smooth_k: bool = True, pv_mode="fp8", workspace=None, stream=None):
    """Quantise this rank's token slice with the combined statistics and store
    its codes and block scales straight into the head-sharded workspaces of
    the group's ranks (``dst_workspaces``: ``world`` device addresses, ints;
    peer-mapped on a multi-GPU node).  The caller completes every rank's
    stores before running dit_attn_fwd_q8_prequantized.  Returns the slice
    workspace (K mean, V scales)."""
    lib = load_library()
    _check_attn_tensors(q, k, v, None)
    B, H, N, d = q.shape
    if workspace is None:
        workspace = q8_workspace(B, H, N, d, pv_mode, q.device)
    ptrs = (ctypes.c_void_p * len(dst_workspaces))(*[int(x) for x in dst_workspaces])
    st = lib.dit_attn_q8_quantize_scatter(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, N, d, _attn_strides(q),
                                          int(bool(smooth_k)), _pv(pv_mode), k_sum.data_ptr(), v_amax.data_ptr(),
                                          int(rank), int(world), ptrs, int(dst_workspace_bytes),
                                          workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    _check(st, "dit_attn_q8_quantize_scatter")
    return workspace


def dit_attn_fwd_q8_prequantized(workspace, B: int, H: int, N: int, o=None, v=None, scale: float | None = None,
                                 pv_mode="fp8", d: int = 128, stream=None):
    """The 8-bit attention kernel alone, on a workspace whose codes and scales
    the caller filled (layout of dit_attn_q8_workspace_layout for B, H, N).
    v: the bf16 V in bf16-PV mode.  Returns o (bf16 [B, H, N, d])."""
    import torch
    lib = load_library()
    if o is None:
        o = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=workspace.device)
    if v is not None and not _same_layout(v, o):
        raise ValueError("v and o must share shape and strides")
    st = lib.dit_attn_fwd_q8_prequantized(workspace.data_ptr(), workspace.numel(),
                                          v.data_ptr() if v is not None else None, o.data_ptr(), B, H, N, d,
                                          _attn_strides(o), float(scale) if scale else 0.0, _pv(pv_mode),
                                          _stream_ptr(stream))
    _check(st, "dit_attn_fwd_q8_prequantized")
    return o


def fbc_rel_l1_workspace_bytes(n: int) -> int:
    return int(load_library().fbc_rel_l1_workspace_bytes(int(n)))


def fbc_workspace(n: int, device=None):
    """A zero-filled workspace tensor for fbc_rel_l1 over n elements."""
    import torch
    return torch.zeros(fbc_rel_l1_workspace_bytes(n), dtype=torch.uint8, device=device or "cuda")


def fbc_rel_l1(r_cur, r_prev, threshold: float, out_rel=None, out_skip=None, workspace=None, stream=None):
    """First-block-cache residual difference on the device.

    r_cur, r_prev: CUDA tensors (fp32 or bf16) of equal shape, contiguous.
    Returns (out_rel, out_skip): device tensors float64[1] and int32[1]; no
    host synchronisation happens here.
    """
    import torch
    lib = load_library()
    if r_cur.shape != r_prev.shape or r_cur.dtype != r_prev.dtype:
        raise ValueError("r_cur and r_prev must match in shape and dtype")
    if not (r_cur.is_contiguous() and r_prev.is_contiguous()):
        raise ValueError("r_cur and r_prev must be contiguous")
    dt = {torch.float32: DIT_DTYPE_F32, torch.bfloat16: DIT_DTYPE_BF16}.get(r_cur.dtype)
    if dt is None:
        raise TypeError("fbc_rel_l1 expects fp32 or bf16 tensors")
    n = r_cur.numel()
    dev = r_cur.device
    if out_rel is None:
        out_rel = torch.empty(1, dtype=torch.float64, device=dev)
    if out_skip is None:
        out_skip = torch.empty(1, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = fbc_workspace(n, dev)
    st = lib.fbc_rel_l1(r_cur.data_ptr(), r_prev.data_ptr(), n, dt, float(threshold), out_rel.data_ptr(),
                        out_skip.data_ptr(), workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    _check(st, "fbc_rel_l1")
    return out_rel, out_skip


def fbc_rel_l1_sums(r_cur, r_prev, out_sums=None, workspace=None, stream=None):
    """Σ|r_cur − r_prev| and Σ|r_prev| over these tensors (device float64[2])."""
    import torch
    lib = load_library()
    if r_cur.shape != r_prev.shape or r_cur.dtype != r_prev.dtype:
        raise ValueError("r_cur and r_prev must match in shape and dtype")
    if not (r_cur.is_contiguous() and r_prev.is_contiguous()):
        raise ValueError("r_cur and r_prev must be contiguous")
    dt = _dtype_code(r_cur, "fbc_rel_l1_sums")
    n = r_cur.numel()
    if out_sums is None:
        out_sums = torch.empty(2, dtype=torch.float64, device=r_cur.device)
    if workspace is None:
        workspace = fbc_workspace(n, r_cur.device)
    st = lib.fbc_rel_l1_sums(r_cur.data_ptr(), r_prev.data_ptr(), n, dt, out_sums.data_ptr(), workspace.data_ptr(),
                             workspace.numel(), _stream_ptr(stream))
    _check(st, "fbc_rel_l1_sums")
    return out_sums


def fbc_rel_l1_finish(sums, threshold: float, out_rel=None, out_skip=None, stream=None):
    """(rel, skip) device tensors from a float64[2] sums tensor."""
    import torch
    lib = load_library()
    if out_rel is None:
        out_rel = torch.empty(1, dtype=torch.float64, device=sums.device)
    if out_skip is None:
        out_skip = torch.empty(1, dtype=torch.int32, device=sums.device)
    st = lib.fbc_rel_l1_finish(sums.data_ptr(), float(threshold), out_rel.data_ptr(), out_skip.data_ptr(),
                               _stream_ptr(stream))
    _check(st, "fbc_rel_l1_finish")
    return out_rel, out_skip


def fbc_rel_l1_noalloc(r_cur, r_prev, threshold: float, out_rel, out_skip, stream=None):
    """fbc_rel_l1 without a workspace, for callers that cannot allocate device
    memory.  The caller passes the output tensors (float64[1], int32[1]); the
    scratch is a fixed array inside the library, shared by every call, so calls
    must not overlap on the GPU."""
    import torch
    lib = load_library()
    if r_cur.shape != r_prev.shape or r_cur.dtype != r_prev.dtype:
        raise ValueError("r_cur and r_prev must match in shape and dtype")
    if not (r_cur.is_contiguous() and r_prev.is_contiguous()):
        raise ValueError("r_cur and r_prev must be contiguous")
    dt = {torch.float32: DIT_DTYPE_F32, torch.bfloat16: DIT_DTYPE_BF16}.get(r_cur.dtype)
    if dt is None:
        raise TypeError("fbc_rel_l1_noalloc expects fp32 or bf16 tensors")
    st = lib.fbc_rel_l1_noalloc(r_cur.data_ptr(), r_prev.data_ptr(), r_cur.numel(), dt, float(threshold),
                                out_rel.data_ptr(), out_skip.data_ptr(), _stream_ptr(stream))
    _check(st, "fbc_rel_l1_noalloc")
    return out_rel, out_skip


def dit_get_device_status(stream=None) -> int:
    """Synchronise the stream; return (and clear) the device error word."""
    return int(load_library().dit_get_device_status(_stream_ptr(stream)))


def dit_wait_selftest(stream=None) -> int:
    """Run the bounded-wait self-test (about 1 s on the stream).  Returns the
    kernel's 'completed' flag: 0 when the wait gave up, as it must.  The device
    error word then holds DIT_ERR_TIMEOUT (read it with dit_get_device_status)."""
    import torch
    lib = load_library()
    s = torch.cuda.current_stream() if stream is None else stream
    flag = torch.full((1,), -1, dtype=torch.int32, device=s.device)
    _check(lib.dit_wait_selftest(flag.data_ptr(), _stream_ptr(stream)), "dit_wait_selftest")
    s.synchronize()
    return int(flag.item())


def dit_compare_workspace_bytes(n_segments: int, segment_len: int, dtype) -> int:
    return int(load_library().dit_compare_workspace_bytes(int(n_segments), int(segment_len), int(dtype)))


def _dtype_code(t, what):
    import torch
    dt = {torch.float32: DIT_DTYPE_F32, torch.bfloat16: DIT_DTYPE_BF16}.get(t.dtype)
    if dt is None:
        raise TypeError(f"{what} expects fp32 or bf16 tensors")
    return dt


def dit_compare_stats(ref, test, segments: int = 1, out=None, workspace=None, stream=None):
    """Error of ``test`` against ``ref`` per contiguous segment, on the device.

    Returns a float64 device tensor [segments, 3]: relative L1, cosine
    similarity, max abs difference.  No host synchronisation.
    """
    import torch
    lib = load_library()
    if ref.shape != test.shape or ref.dtype != test.dtype:
        raise ValueError("ref and test must match in shape and dtype")
    if not (ref.is_contiguous() and test.is_contiguous()):
        raise ValueError("ref and test must be contiguous")
    dt = _dtype_code(ref, "dit_compare_stats")
    n = ref.numel()
    if segments < 1 or n % segments:
        raise ValueError("segments must divide the element count")
    seg_len = n // segments
    if out is None:
        out = torch.empty(segments, 3, dtype=torch.float64, device=ref.device)
    if workspace is None:
        workspace = torch.zeros(dit_compare_workspace_bytes(segments, seg_len, dt), dtype=torch.uint8,
                                device=ref.device)
    st = lib.dit_compare_stats(ref.data_ptr(), test.data_ptr(), segments, seg_len, dt, out.data_ptr(),
                               workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    _check(st, "dit_compare_stats")
    return out


# ---- step caches (include/dit_cache.h) ------------------------------------

DIT_CACHE_USE = 0
DIT_CACHE_WARMUP = 1
DIT_CACHE_NO_PREV = 2
DIT_CACHE_ABOVE_THRESHOLD = 3
DIT_CACHE_MAX_CACHED = 4
DIT_CACHE_MAX_CONTINUOUS = 5
CACHE_STATE_BYTES = 40
CACHE_TRACE_BYTES = 24


class dit_cache_policy(ctypes.Structure):
    """Policy of fbcache_step; defaults of the DiffusionCacheConfig table."""
    _fields_ = [("max_warmup_steps", ctypes.c_int32), ("max_cached_steps", ctypes.c_int32),
                ("max_continuous_cached_steps", ctypes.c_int32), ("residual_diff_threshold", ctypes.c_float)]

    def __init__(self, max_warmup_steps=4, max_cached_steps=-1, max_continuous_cached_steps=3,
                 residual_diff_threshold=0.24):
        super().__init__(int(max_warmup_steps), int(max_cached_steps), int(max_continuous_cached_steps),
                         float(residual_diff_threshold))


def cache_state(device=None):
    """A fresh (zeroed) device-resident dit_cache_state."""
    import torch
    return torch.zeros(CACHE_STATE_BYTES, dtype=torch.uint8, device=device or "cuda")


def cache_trace(capacity: int, device=None):
    import torch
    return torch.zeros(int(capacity) * CACHE_TRACE_BYTES, dtype=torch.uint8, device=device or "cuda")


def read_cache_state(state) -> dict:
    """Copy a dit_cache_state to the host (synchronises)."""
    import numpy as np
    b = state.detach().cpu().numpy().tobytes()
    i = np.frombuffer(b[:24], dtype=np.int32)
    f = np.frombuffer(b[24:40], dtype=np.float64)
    return {"step": int(i[0]), "cached_steps": int(i[1]), "continuous_cached": int(i[2]),
            "has_prev": int(i[3]), "last_decision": int(i[4]), "last_rel": float(f[0]), "acc": float(f[1])}


def read_cache_trace(trace, count: int):
    """First ``count`` trace entries as a numpy record array (rel, acc, decision)."""
    import numpy as np
    dt = np.dtype([("rel", "<f8"), ("acc", "<f8"), ("decision", "<i4"), ("reserved", "<i4")])
    return np.frombuffer(trace.detach().cpu().numpy().tobytes(), dtype=dt)[:count]


def dit_cache_workspace_bytes(n: int) -> int:
    return int(load_library().dit_cache_workspace_bytes(int(n)))


def cache_workspace(n: int, device=None):
    import torch
    return torch.zeros(dit_cache_workspace_bytes(n), dtype=torch.uint8, device=device or "cuda")


def dit_cache_state_reset(state, stream=None):
    _check(load_library().dit_cache_state_reset(state.data_ptr(), _stream_ptr(stream)), "dit_cache_state_reset")


def _step_args(cur, prev, what):
    if cur.shape != prev.shape or cur.dtype != prev.dtype:
        raise ValueError(f"{what}: inputs must match in shape and dtype")
    if not (cur.is_contiguous() and prev.is_contiguous()):
        raise ValueError(f"{what}: inputs must be contiguous")
    return _dtype_code(cur, what)


def fbcache_step(r_cur, r_prev, policy: dit_cache_policy, state, trace=None, cond_handle=None, workspace=None,
                 stream=None):
    """One first-block-cache decision; updates ``state`` on the device."""
    lib = load_library()
    dt = _step_args(r_cur, r_prev, "fbcache_step")
    n = r_cur.numel()
    if workspace is None:
        workspace = cache_workspace(n, r_cur.device)
    cap = trace.numel() // CACHE_TRACE_BYTES if trace is not None else 0
    st = lib.fbcache_step(r_cur.data_ptr(), r_prev.data_ptr(), n, dt, ctypes.byref(policy), state.data_ptr(),
                          trace.data_ptr() if trace is not None else None, cap,
                          0 if cond_handle is None else 1, 0 if cond_handle is None else int(cond_handle),
                          workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    _check(st, "fbcache_step")
    return state


def teacache_step(x_cur, x_prev, coeffs, threshold: float, state, trace=None, cond_handle=None, workspace=None,
                  stream=None):
    """One TeaCache decision; updates ``state`` and stores x_cur into x_prev."""
    lib = load_library()
    dt = _step_args(x_cur, x_prev, "teacache_step")
    n = x_cur.numel()
    if workspace is None:
        workspace = cache_workspace(n, x_cur.device)
    c = (ctypes.c_double * len(coeffs))(*[float(v) for v in coeffs])
    cap = trace.numel() // CACHE_TRACE_BYTES if trace is not None else 0
    st = lib.teacache_step(x_cur.data_ptr(), x_prev.data_ptr(), n, dt, c, len(coeffs), float(threshold),
                           state.data_ptr(), trace.data_ptr() if trace is not None else None, cap,
                           0 if cond_handle is None else 1, 0 if cond_handle is None else int(cond_handle),
                           workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    _check(st, "teacache_step")
    return state


def dit_graph_capture_begin(stream):
    _check(load_library().dit_graph_capture_begin(_stream_ptr(stream)), "dit_graph_capture_begin")


def dit_graph_cond_create(stream) -> int:
    h = ctypes.c_ulonglong(0)
    _check(load_library().dit_graph_cond_create(_stream_ptr(stream), ctypes.byref(h)), "dit_graph_cond_create")
    return int(h.value)


def dit_graph_cond_body_begin(stream, cond_handle: int, body_stream):
    _check(load_library().dit_graph_cond_body_begin(_stream_ptr(stream), int(cond_handle), _stream_ptr(body_stream)),
           "dit_graph_cond_body_begin")


def dit_graph_cond_body_end(body_stream):
    _check(load_library().dit_graph_cond_body_end(_stream_ptr(body_stream)), "dit_graph_cond_body_end")


def dit_graph_capture_end(stream) -> int:
    g = ctypes.c_void_p(0)
    _check(load_library().dit_graph_capture_end(_stream_ptr(stream), ctypes.byref(g)), "dit_graph_capture_end")
    return int(g.value)


def dit_graph_launch(graph_exec: int, stream):
    _check(load_library().dit_graph_launch(ctypes.c_void_p(graph_exec), _stream_ptr(stream)), "dit_graph_launch")


def dit_graph_destroy(graph_exec: int):
    _check(load_library().dit_graph_destroy(ctypes.c_void_p(graph_exec)), "dit_graph_destroy")
