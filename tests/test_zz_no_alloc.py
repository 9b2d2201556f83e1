"""fbc_rel_l1_noalloc, the first-block-cache decision for callers that cannot
allocate device memory, called through the C ABI.

Some callers hold only their input and output pointers, for example a plugin
inside an inference engine, or a module whose framework's caching allocator
owns all device memory.  They cannot pass fbc_rel_l1 a workspace.  The
no-alloc variant keeps its scratch in a fixed array inside the library.  Its
result must match the fp64 oracle and the workspace entry point on the same
inputs, and stay correct from one call to the next, since every call shares
that array.

This file is collected last on purpose.  If it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle
from diffusion_transformer_attention_attn_b200 import inputs
from tests.common import FBC_REL_ERR

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from diffusion_transformer_attention_attn_b200 import build_lib
    import diffusion_transformer_attention_attn_b200 as dit
    build_lib.build()
    return dit.load_library()


def _dev(x):
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _with_workspace(lib, cur, prev, n, dtype, thr, stream):
    rel = torch.empty(1, dtype=torch.float64, device="cuda")
    skip = torch.empty(1, dtype=torch.int32, device="cuda")
    wsb = lib.fbc_rel_l1_workspace_bytes(n)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    st = lib.fbc_rel_l1(cur.data_ptr(), prev.data_ptr(), n, dtype, thr, rel.data_ptr(), skip.data_ptr(),
                        ws.data_ptr(), wsb, stream)
    assert st == 0, st
    return rel, skip


def _no_alloc(lib, cur, prev, n, dtype, thr, stream):
    rel = torch.full((1,), -1.0, dtype=torch.float64, device="cuda")
    skip = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    st = lib.fbc_rel_l1_noalloc(cur.data_ptr(), prev.data_ptr(), n, dtype, thr, rel.data_ptr(), skip.data_ptr(),
                                stream)
    assert st == 0, st
    return rel, skip


def test_no_alloc_matches_workspace_entry_point_on_consecutive_calls(lib):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [
        (inputs.FBC_IMAGE, 1, 0.08),                                     # 4608 x 3072 bf16
        (inputs.FBC_TINY, 0, 0.08),                                      # 256 x 128 fp32
        (inputs.FbcCase("odd_bf16", 1, 1_000_003, "bf16", 0.2, 0.1), 1, 0.1),   # ragged tail, compute decision
    ]
    for case, dtype, thr in cases:
        cur, prev = inputs.fbc_inputs(case)
        dc, dp = _dev(cur.reshape(-1)), _dev(prev.reshape(-1))
        n = cur.size
        ref_rel, ref_skip = _with_workspace(lib, dc, dp, n, dtype, thr, stream)
        o_rel, o_skip = oracle.fbc_rel_l1(cur, prev, thr)
        # two calls in a row through the shared scratch array
        for _ in range(2):
            rel, skip = _no_alloc(lib, dc, dp, n, dtype, thr, stream)
            torch.cuda.synchronize()
            r, rr = rel.item(), ref_rel.item()
            assert abs(r - o_rel) <= FBC_REL_ERR * abs(o_rel), (case.name, r, o_rel)
            assert int(skip.item()) == o_skip, case.name
            assert abs(r - rr) <= FBC_REL_ERR * abs(rr), (case.name, r, rr)
            assert int(skip.item()) == int(ref_skip.item()), case.name
    import diffusion_transformer_attention_attn_b200 as dit
    assert dit.dit_get_device_status() == 0


def test_no_alloc_rejects_bad_arguments(lib):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    x = torch.zeros(64, dtype=torch.float32, device="cuda")
    rel = torch.empty(1, dtype=torch.float64, device="cuda")
    skip = torch.empty(1, dtype=torch.int32, device="cuda")
    assert lib.fbc_rel_l1_noalloc(x.data_ptr(), x.data_ptr(), 0, 0, 0.08, rel.data_ptr(), skip.data_ptr(),
                                  stream) == 1
    assert lib.fbc_rel_l1_noalloc(x.data_ptr(), x.data_ptr(), 64, 9, 0.08, rel.data_ptr(), skip.data_ptr(),
                                  stream) == 1
    assert lib.fbc_rel_l1_noalloc(x.data_ptr() + 4, x.data_ptr(), 60, 0, 0.08, rel.data_ptr(), skip.data_ptr(),
                                  stream) == 1
