"""Python binding of libditattn.so, the B200 (sm_100a) diffusion-transformer
attention library.

Argument marshalling only: every step of every call runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  There
is no fallback: if the library is missing, importing the binding's entry
points raises.

Entry points (same names as the C ABI in ``include/dit_attn.h``):
  * ``dit_attn_fwd(q, k, v, o=None, scale=None)``  — bf16 softmax attention
  * ``dit_attn_fwd_q8(q, k, v, ...)``              — 8-bit attention (INT8 QKᵀ, FP8 or bf16 PV)
  * ``dit_attn_q8_quantize(q, k, v, ...)``         — its pre-pass alone
  * ``fbc_rel_l1(r_cur, r_prev, threshold, ...)``   — first-block-cache decision
  * ``fbc_rel_l1_noalloc(...)``                     — the same, allocating nothing
  * ``dit_get_device_status()``                     — device-side error word
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
    "dit_attn_q8_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "dit_attn_fwd_q8": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _p, _f, _i, _i, _p, _sz, _p]),
    "dit_attn_q8_quantize": (_i, [_p, _p, _p, _i, _i, _i, _i, _p, _i, _i, _p, _sz, _p]),
    "dit_attn_q8_workspace_layout": (_i, [_i, _i, _i, _i, _i, _p]),
    "fbc_rel_l1_workspace_bytes": (_sz, [_i64]),
    "fbc_rel_l1": (_i, [_p, _p, _i64, _i, _f, _p, _p, _p, _sz, _p]),
    "fbc_rel_l1_noalloc": (_i, [_p, _p, _i64, _i, _f, _p, _p, _p]),
    "dit_get_device_status": (_i, [_p]),
    "dit_status_string": (ctypes.c_char_p, [_i]),
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
        if t.shape != q.shape or t.stride() != q.stride():
            raise ValueError("q, k, v, o must share shape and strides")
    B, H, N, d = q.shape
    st = lib.dit_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), B, H, N, d,
                          _attn_strides(q), float(scale) if scale else 0.0, _stream_ptr(stream))
    _check(st, "dit_attn_fwd")
    return o


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
        if t.shape != q.shape or t.stride() != q.stride():
            raise ValueError("q, k, v, o must share shape and strides")


def dit_attn_fwd_q8(q, k, v, o=None, scale: float | None = None, smooth_k: bool = True, pv_mode="fp8",
                    workspace=None, stream=None):
    """8-bit attention: INT8 Q (per 128 tokens) and K (per 64 tokens, optional
    channel-mean smoothing), S in int32, P·V in FP8 e4m3 or bf16.  bf16 CUDA
    tensors [B, H, N, 128].  Returns o."""
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
