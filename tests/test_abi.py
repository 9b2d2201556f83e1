"""CPU-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments with the documented status before
touching the device (no GPU is needed for any of these)."""
import ctypes
import os
import re

import pytest

import diffusion_transformer_attention_attn_b200 as dit
from diffusion_transformer_attention_attn_b200 import build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return dit.load_library()


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(HEADER_DIR)):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(HEADER_DIR, fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M):
            if m.group(1) not in ("if", "defined"):
                names.append(m.group(1))
    return names


def test_header_declares_the_boundary():
    names = _declared_functions()
    for expected in ("dit_attn_fwd", "fbc_rel_l1", "fbc_rel_l1_workspace_bytes", "dit_get_device_status",
                     "dit_status_string"):
        assert expected in names
    assert set(names) == set(dit.SIGNATURES), "binding and header disagree"


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert dit.status_string(0) == "DIT_OK"
    assert dit.status_string(5) == "DIT_ERR_TIMEOUT"
    assert dit.status_string(99) == "DIT_ERR_UNKNOWN"


# Fake, 16-byte-aligned, non-overlapping "device" addresses: every case below
# is rejected during validation, before any pointer is used.
Q, K, V, O = 0x10000000, 0x20000000, 0x30000000, 0x40000000


def _attn(lib, q=Q, k=K, v=V, o=O, B=1, H=2, N=256, d=64, strides=None, scale=0.0):
    st = None
    if strides is not None:
        st = (ctypes.c_int64 * 3)(*strides)
    return lib.dit_attn_fwd(q, k, v, o, B, H, N, d, st, scale, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=0), dit.DIT_ERR_INVALID_ARG),
    (dict(o=0), dit.DIT_ERR_INVALID_ARG),
    (dict(N=0), dit.DIT_ERR_INVALID_ARG),
    (dict(B=0), dit.DIT_ERR_INVALID_ARG),
    (dict(H=-1), dit.DIT_ERR_INVALID_ARG),
    (dict(d=96), dit.DIT_ERR_UNSUPPORTED),
    (dict(d=256), dit.DIT_ERR_UNSUPPORTED),
    (dict(k=K + 8), dit.DIT_ERR_INVALID_ARG),            # misaligned
    (dict(o=Q + 64), dit.DIT_ERR_INVALID_ARG),           # output overlaps q
    (dict(strides=(256 * 64 * 2, 256 * 64, 60)), dit.DIT_ERR_INVALID_ARG),  # row stride < d
    (dict(strides=(256 * 64 * 2, 256 * 64, 68)), dit.DIT_ERR_INVALID_ARG),  # 136 B: not a multiple of 16
    (dict(scale=float("nan")), dit.DIT_ERR_INVALID_ARG),
])
def test_attn_argument_errors(lib, kw, status):
    assert _attn(lib, **kw) == status


def test_fbc_argument_errors(lib):
    n = 1000
    ws = lib.fbc_rel_l1_workspace_bytes(n)
    assert ws >= 16
    assert lib.fbc_rel_l1_workspace_bytes(0) == 0
    call = lambda **kw: lib.fbc_rel_l1(kw.get("cur", Q), kw.get("prev", K), kw.get("n", n), kw.get("dtype", 0),
                                       kw.get("thr", 0.08), kw.get("rel", V), kw.get("skip", V + 64),
                                       kw.get("ws", O), kw.get("wsb", ws), None)
    assert call(cur=0) == dit.DIT_ERR_INVALID_ARG
    assert call(n=0) == dit.DIT_ERR_INVALID_ARG
    assert call(dtype=7) == dit.DIT_ERR_INVALID_ARG
    assert call(prev=K + 4) == dit.DIT_ERR_INVALID_ARG
    assert call(rel=V + 4) == dit.DIT_ERR_INVALID_ARG
    assert call(thr=float("nan")) == dit.DIT_ERR_INVALID_ARG
    assert call(ws=0) == dit.DIT_ERR_WORKSPACE
    assert call(wsb=ws - 1) == dit.DIT_ERR_WORKSPACE
    assert call(ws=O + 8) == dit.DIT_ERR_WORKSPACE


def test_product_path_does_not_reach_the_oracle():
    # The binding and the library sources never name the oracle.
    pkg = os.path.join(ROOT, "diffusion_transformer_attention_attn_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "liboracle" not in text, f


def test_q8_workspace_size_and_layout(lib):
    assert lib.dit_attn_q8_workspace_bytes(1, 2, 256, 96, 0) == 0          # d = 96: not served
    d64 = lib.dit_attn_q8_workspace_bytes(1, 2, 256, 64, 0)                 # d = 64: half the codes
    assert 3 * 2 * 256 * 64 <= d64 < lib.dit_attn_q8_workspace_bytes(1, 2, 256, 128, 0)
    assert lib.dit_attn_q8_workspace_bytes(1, 2, 256, 128, 7) == 0         # bad mode
    fp8 = lib.dit_attn_q8_workspace_bytes(1, 24, 4608, 128, dit.DIT_PV_FP8_E4M3)
    bf = lib.dit_attn_q8_workspace_bytes(1, 24, 4608, 128, dit.DIT_PV_BF16)
    codes = 24 * 4608 * 128
    assert fp8 >= 3 * codes and bf >= 2 * codes and fp8 - bf >= codes
    off = dit.dit_attn_q8_workspace_layout(1, 24, 4608, 128, "fp8")
    vals = [off[k] for k in dit.Q8_SEGMENTS]
    assert all(v % 256 == 0 for v in vals) and vals == sorted(vals) and vals[-1] < fp8
    assert off["k_codes"] - off["q_codes"] >= codes


WS = 0x50000000


def _q8(lib, q=Q, k=K, v=V, o=O, B=1, H=2, N=256, d=128, smooth=1, mode=0, ws=WS, wsb=None):
    if wsb is None:
        wsb = lib.dit_attn_q8_workspace_bytes(B, H, N, 128, 0)
    return lib.dit_attn_fwd_q8(q, k, v, o, B, H, N, d, None, 0.0, smooth, mode, ws, wsb, None)


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), dit.DIT_ERR_UNSUPPORTED),
    (dict(mode=5), dit.DIT_ERR_INVALID_ARG),
    (dict(smooth=2), dit.DIT_ERR_INVALID_ARG),
    (dict(ws=0), dit.DIT_ERR_WORKSPACE),
    (dict(ws=WS + 128), dit.DIT_ERR_WORKSPACE),                 # not 256-byte aligned
    (dict(wsb=1024), dit.DIT_ERR_WORKSPACE),
    (dict(ws=Q), dit.DIT_ERR_WORKSPACE),                        # overlaps q
    (dict(v=0), dit.DIT_ERR_INVALID_ARG),
    (dict(N=0), dit.DIT_ERR_INVALID_ARG),
])
def test_q8_argument_errors(lib, kw, status):
    assert _q8(lib, **kw) == status


def test_q8_quantize_argument_errors(lib):
    wsb = lib.dit_attn_q8_workspace_bytes(1, 2, 256, 128, 0)
    assert lib.dit_attn_q8_quantize(Q, K, V, 1, 2, 256, 96, None, 1, 0, WS, wsb, None) == dit.DIT_ERR_UNSUPPORTED
    assert lib.dit_attn_q8_quantize(Q, K, V, 1, 2, 256, 128, None, 1, 0, WS, 100, None) == dit.DIT_ERR_WORKSPACE
    assert lib.dit_attn_q8_quantize(0, K, V, 1, 2, 256, 128, None, 1, 0, WS, wsb, None) == dit.DIT_ERR_INVALID_ARG


def test_cache_step_argument_errors(lib):
    n = 4096
    ws = lib.dit_cache_workspace_bytes(n)
    assert ws == lib.fbc_rel_l1_workspace_bytes(n) and lib.dit_cache_workspace_bytes(0) == 0
    pol = dit.dit_cache_policy()
    ST, TR = 0x60000000, 0x61000000

    def fb(**kw):
        return lib.fbcache_step(kw.get("cur", Q), kw.get("prev", K), kw.get("n", n), kw.get("dtype", 1),
                                kw.get("policy", ctypes.byref(pol)), kw.get("state", ST), kw.get("trace", TR),
                                kw.get("cap", 8), kw.get("use_cond", 0), kw.get("cond", 0),
                                kw.get("ws", O), kw.get("wsb", ws), None)
    assert fb(cur=0) == dit.DIT_ERR_INVALID_ARG
    assert fb(n=0) == dit.DIT_ERR_INVALID_ARG
    assert fb(dtype=3) == dit.DIT_ERR_INVALID_ARG
    assert fb(prev=K + 8) == dit.DIT_ERR_INVALID_ARG
    assert fb(state=ST + 4) == dit.DIT_ERR_INVALID_ARG
    assert fb(trace=TR + 4) == dit.DIT_ERR_INVALID_ARG
    assert fb(cap=-1) == dit.DIT_ERR_INVALID_ARG
    assert fb(policy=None) == dit.DIT_ERR_INVALID_ARG
    assert fb(policy=ctypes.byref(dit.dit_cache_policy(max_warmup_steps=-1))) == dit.DIT_ERR_INVALID_ARG
    assert fb(policy=ctypes.byref(dit.dit_cache_policy(residual_diff_threshold=float("inf")))) == \
        dit.DIT_ERR_INVALID_ARG
    assert fb(use_cond=2) == dit.DIT_ERR_INVALID_ARG
    # a conditional handle that no capture on this stream created is refused
    assert fb(use_cond=1, cond=12345) == dit.DIT_ERR_INVALID_ARG
    assert fb(ws=0) == dit.DIT_ERR_WORKSPACE
    assert fb(wsb=ws - 1) == dit.DIT_ERR_WORKSPACE

    coeffs = (ctypes.c_double * 3)(0.0, 1.0, 0.0)

    def tea(**kw):
        return lib.teacache_step(kw.get("cur", Q), kw.get("prev", K), kw.get("n", n), kw.get("dtype", 1),
                                 kw.get("coeffs", coeffs), kw.get("nc", 3), kw.get("thr", 0.1),
                                 kw.get("state", ST), None, 0, kw.get("use_cond", 0), 0,
                                 kw.get("ws", O), kw.get("wsb", ws), None)
    assert tea(nc=0) == dit.DIT_ERR_INVALID_ARG
    assert tea(nc=9) == dit.DIT_ERR_INVALID_ARG
    assert tea(coeffs=None) == dit.DIT_ERR_INVALID_ARG
    assert tea(coeffs=(ctypes.c_double * 3)(0.0, float("nan"), 0.0)) == dit.DIT_ERR_INVALID_ARG
    assert tea(thr=float("nan")) == dit.DIT_ERR_INVALID_ARG
    assert tea(prev=Q + 16) == dit.DIT_ERR_INVALID_ARG            # overlaps x_cur
    assert tea(state=0) == dit.DIT_ERR_INVALID_ARG
    assert tea(use_cond=1) == dit.DIT_ERR_INVALID_ARG
    assert tea(wsb=0) == dit.DIT_ERR_WORKSPACE
    assert lib.dit_cache_state_reset(None, None) == dit.DIT_ERR_INVALID_ARG
    assert lib.dit_cache_state_reset(ST + 4, None) == dit.DIT_ERR_INVALID_ARG


def test_graph_plumbing_argument_errors(lib):
    h = ctypes.c_ulonglong(0)
    g = ctypes.c_void_p(0)
    assert lib.dit_graph_capture_begin(None) == dit.DIT_ERR_INVALID_ARG
    assert lib.dit_graph_cond_create(None, ctypes.byref(h)) == dit.DIT_ERR_INVALID_ARG
    assert lib.dit_graph_cond_body_begin(None, 0, None) == dit.DIT_ERR_INVALID_ARG
    assert lib.dit_graph_cond_body_begin(0x1000, 0, 0x1000) == dit.DIT_ERR_INVALID_ARG   # same stream
    assert lib.dit_graph_cond_body_end(None) == dit.DIT_ERR_INVALID_ARG
    assert lib.dit_graph_capture_end(None, ctypes.byref(g)) == dit.DIT_ERR_INVALID_ARG
    assert lib.dit_graph_launch(None, None) == dit.DIT_ERR_INVALID_ARG
    assert lib.dit_graph_destroy(None) == dit.DIT_ERR_INVALID_ARG


def test_compare_argument_errors(lib):
    assert lib.dit_compare_workspace_bytes(0, 10, 1) == 0
    assert lib.dit_compare_workspace_bytes(65536, 10, 1) == 0
    assert lib.dit_compare_workspace_bytes(4, 10, 9) == 0
    ws = lib.dit_compare_workspace_bytes(4, 1000, 1)
    assert ws >= 256 + 4 * 48

    def cmp(**kw):
        return lib.dit_compare_stats(kw.get("ref", Q), kw.get("test", K), kw.get("nseg", 4), kw.get("len", 1000),
                                     kw.get("dtype", 1), kw.get("out", V), kw.get("ws", O), kw.get("wsb", ws), None)
    assert cmp(ref=0) == dit.DIT_ERR_INVALID_ARG
    assert cmp(nseg=0) == dit.DIT_ERR_INVALID_ARG
    assert cmp(len=0) == dit.DIT_ERR_INVALID_ARG
    assert cmp(dtype=2) == dit.DIT_ERR_INVALID_ARG
    assert cmp(test=K + 1) == dit.DIT_ERR_INVALID_ARG                # not element aligned
    assert cmp(out=V + 4) == dit.DIT_ERR_INVALID_ARG
    assert cmp(ws=0) == dit.DIT_ERR_WORKSPACE
    assert cmp(wsb=ws - 1) == dit.DIT_ERR_WORKSPACE


def test_attn_ex_and_merge_argument_errors(lib):
    def ex(**kw):
        qs = kw.get("qs")
        ks = kw.get("ks")
        return lib.dit_attn_fwd_ex(kw.get("q", Q), kw.get("k", K), kw.get("v", V), kw.get("o", O), kw.get("lse", None),
                                   1, 2, kw.get("Nq", 256), kw.get("Nkv", 512), kw.get("d", 64),
                                   (ctypes.c_int64 * 3)(*qs) if qs else None,
                                   (ctypes.c_int64 * 3)(*ks) if ks else None, kw.get("scale", 0.0), None)
    assert ex(Nq=0) == dit.DIT_ERR_INVALID_ARG
    assert ex(Nkv=0) == dit.DIT_ERR_INVALID_ARG
    assert ex(d=96) == dit.DIT_ERR_UNSUPPORTED
    assert ex(o=0) == dit.DIT_ERR_INVALID_ARG
    assert ex(v=V + 8) == dit.DIT_ERR_INVALID_ARG
    assert ex(o=K + 1024) == dit.DIT_ERR_INVALID_ARG               # inside k
    assert ex(lse=O + 2) == dit.DIT_ERR_INVALID_ARG                # misaligned
    assert ex(lse=O + 64) == dit.DIT_ERR_INVALID_ARG               # overlaps o
    assert ex(ks=(512 * 64 * 2, 512 * 64, 60)) == dit.DIT_ERR_INVALID_ARG
    assert ex(scale=float("inf")) == dit.DIT_ERR_INVALID_ARG

    def merge(n=2, parts=None, lparts=None, o=0x70000000, lse=None, N=256, d=64):
        parts = parts or [Q, K][:n] + [V] * max(0, n - 2)
        lparts = lparts or [0x71000000 + 0x100000 * i for i in range(n)]
        op = (ctypes.c_void_p * max(n, 1))(*parts[:max(n, 1)])
        lp = (ctypes.c_void_p * max(n, 1))(*lparts[:max(n, 1)])
        return lib.dit_attn_merge(op, lp, n, 1, 2, N, d, None, o, lse, None)
    assert merge(n=0) == dit.DIT_ERR_INVALID_ARG
    assert merge(n=17) == dit.DIT_ERR_INVALID_ARG
    assert merge(d=12) == dit.DIT_ERR_INVALID_ARG
    assert merge(o=0x70000008) == dit.DIT_ERR_INVALID_ARG           # misaligned output
    assert merge(parts=[Q + 8, K]) == dit.DIT_ERR_INVALID_ARG       # misaligned part
    assert merge(lparts=[0x71000002, 0x71100000]) == dit.DIT_ERR_INVALID_ARG
    assert merge(o=Q) == dit.DIT_ERR_INVALID_ARG                    # output overwrites a part
    assert merge(lse=0x71000000) == dit.DIT_ERR_INVALID_ARG         # lse overwrites a part's lse


def test_fbc_sums_and_finish_argument_errors(lib):
    ws = lib.fbc_rel_l1_workspace_bytes(64)
    assert lib.fbc_rel_l1_sums(Q, K, 0, 0, V, O, ws, None) == dit.DIT_ERR_INVALID_ARG
    assert lib.fbc_rel_l1_sums(Q, K, 64, 0, V + 4, O, ws, None) == dit.DIT_ERR_INVALID_ARG
    assert lib.fbc_rel_l1_sums(Q, K + 8, 64, 0, V, O, ws, None) == dit.DIT_ERR_INVALID_ARG
    assert lib.fbc_rel_l1_sums(Q, K, 64, 0, V, O, ws - 1, None) == dit.DIT_ERR_WORKSPACE
    assert lib.fbc_rel_l1_finish(None, 0.1, V, V + 64, None) == dit.DIT_ERR_INVALID_ARG
    assert lib.fbc_rel_l1_finish(Q + 4, 0.1, V, V + 64, None) == dit.DIT_ERR_INVALID_ARG
    assert lib.fbc_rel_l1_finish(Q, float("nan"), V, V + 64, None) == dit.DIT_ERR_INVALID_ARG


def test_sharded_q8_argument_errors(lib):
    wsb = lib.dit_attn_q8_workspace_bytes(1, 2, 256, 128, 0)
    KS, VA = 0x62000000, 0x63000000
    st = lambda **kw: lib.dit_attn_q8_channel_stats(kw.get("k", K), kw.get("v", V), 1, 2, 256, kw.get("d", 128), None,
                                                    kw.get("smooth", 1), kw.get("mode", 0), kw.get("ks", KS),
                                                    kw.get("va", VA), kw.get("ws", WS), kw.get("wsb", wsb), None)
    assert st(k=0) == dit.DIT_ERR_INVALID_ARG
    assert st(d=96) == dit.DIT_ERR_UNSUPPORTED
    assert st(mode=3) == dit.DIT_ERR_INVALID_ARG
    assert st(ks=0) == dit.DIT_ERR_INVALID_ARG
    assert st(ks=KS + 4) == dit.DIT_ERR_INVALID_ARG
    assert st(va=WS + 256) == dit.DIT_ERR_INVALID_ARG             # inside the workspace
    assert st(wsb=16) == dit.DIT_ERR_WORKSPACE
    qg = lambda **kw: lib.dit_attn_q8_quantize_global(Q, K, V, 1, 2, 256, 128, None, 1, 0, kw.get("ks", KS), VA,
                                                      kw.get("n", 512), WS, wsb, None)
    assert qg(n=100) == dit.DIT_ERR_INVALID_ARG                   # n_total below this slice's tokens
    assert qg(ks=0) == dit.DIT_ERR_INVALID_ARG
    pq = lambda **kw: lib.dit_attn_fwd_q8_prequantized(kw.get("ws", WS), kw.get("wsb", wsb), kw.get("v", None),
                                                       kw.get("o", O), 1, 2, 256, 128, None, kw.get("scale", 0.0),
                                                       kw.get("mode", 0), None)
    assert pq(o=0) == dit.DIT_ERR_INVALID_ARG
    assert pq(mode=1) == dit.DIT_ERR_INVALID_ARG                  # bf16 PV needs V
    assert pq(scale=float("nan")) == dit.DIT_ERR_INVALID_ARG
    assert pq(wsb=1) == dit.DIT_ERR_WORKSPACE
    assert pq(ws=WS + 128) == dit.DIT_ERR_WORKSPACE


def test_quantize_scatter_argument_errors(lib):
    # all rejected on the host before any launch (the pointers are never touched)
    wsb = lib.dit_attn_q8_workspace_bytes(1, 4, 256, 128, 0)
    dwb = lib.dit_attn_q8_workspace_bytes(1, 2, 512, 128, 0)
    KS, VA = 0x62000000, 0x63000000
    D0, D1 = 0x64000000, 0x64000000 + ((dwb + 255) // 256) * 256

    def sc(world=2, rank=0, H=4, N=256, dst=(D0, D1), dwb=dwb, ks=KS):
        arr = (ctypes.c_void_p * len(dst))(*dst) if dst is not None else None
        return lib.dit_attn_q8_quantize_scatter(Q, K, V, 1, H, N, 128, None, 1, 0, ks, VA, rank, world, arr, dwb,
                                                WS, wsb, None)
    assert sc(world=0, dst=()) == dit.DIT_ERR_INVALID_ARG
    assert sc(world=17, dst=(D0,) * 17) == dit.DIT_ERR_INVALID_ARG
    assert sc(rank=2) == dit.DIT_ERR_INVALID_ARG
    assert sc(H=3) == dit.DIT_ERR_INVALID_ARG                      # heads do not split over the ranks
    assert sc(N=200) == dit.DIT_ERR_INVALID_ARG                    # whole 128-token blocks per rank
    assert sc(dst=None) == dit.DIT_ERR_INVALID_ARG
    assert sc(ks=0) == dit.DIT_ERR_INVALID_ARG
    assert sc(dwb=dwb - 256) == dit.DIT_ERR_WORKSPACE
    assert sc(dst=(D0, D0 + 256)) == dit.DIT_ERR_WORKSPACE         # destinations overlap
    assert sc(dst=(D0, D1 + 128)) == dit.DIT_ERR_WORKSPACE         # not 256-byte aligned
    assert sc(dst=(D0, WS)) == dit.DIT_ERR_WORKSPACE               # the slice workspace itself


def test_wait_selftest_argument_error(lib):
    assert lib.dit_wait_selftest(None, None) == dit.DIT_ERR_INVALID_ARG
