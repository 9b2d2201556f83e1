"""The token-sharded 8-bit path through the C ABI on one GPU.

dit_attn_q8_channel_stats / dit_attn_q8_quantize_global / the codes' move to
the head-sharded layout / dit_attn_fwd_q8_prequantized must give, bit for
bit, the codes and the output of the single dit_attn_fwd_q8 call when every
token slice holds whole 128-token blocks.  Here the slices are views of one
tensor and their combination (sum, max) and the all-to-all are done with
device copies, as the collectives of a Ulysses group would.
"""
import numpy as np
import pytest

from diffusion_transformer_attention_attn_b200 import inputs
from tests.common import to_device_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import diffusion_transformer_attention_attn_b200 as dit
    dit.load_library()
    yield
    assert dit.dit_get_device_status() == 0


def _dit():
    import diffusion_transformer_attention_attn_b200 as dit
    return dit


def _inputs(N=1024, H=4, seed=2):
    case = inputs.AttnCase("shq8", 1, H, N, 128, k_offset_std=3.0, zero_q_channel=7, seed=seed)
    return [to_device_bf16(x) for x in inputs.attn_inputs(case)]


@pytest.mark.parametrize("pv_mode", ["fp8", "bf16"])
@pytest.mark.parametrize("smooth_k", [True, False])
@pytest.mark.parametrize("world", [2, 4])
def test_slices_reproduce_the_single_call(pv_mode, smooth_k, world):
    dit = _dit()
    q, k, v = _inputs()
    B, H, N, d = q.shape
    Nl, hp = N // world, H // world
    ref = dit.dit_attn_fwd_q8(q, k, v, smooth_k=smooth_k, pv_mode=pv_mode)
    ref_ws = dit.dit_attn_q8_quantize(q, k, v, smooth_k=smooth_k, pv_mode=pv_mode)
    ref_v = dit.q8_views(ref_ws, B, H, N, d, pv_mode)
    sl = [slice(r * Nl, (r + 1) * Nl) for r in range(world)]
    # per-slice statistics, combined as two all-reduces would
    stats = [dit.dit_attn_q8_channel_stats(k[:, :, s], v[:, :, s], smooth_k=smooth_k, pv_mode=pv_mode) for s in sl]
    k_sum = sum(x for x, _ in stats)
    v_amax = torch.stack([y for _, y in stats]).amax(dim=0)
    local = []
    for s in sl:
        ws = dit.dit_attn_q8_quantize_global(q[:, :, s], k[:, :, s], v[:, :, s], k_sum, v_amax, N, smooth_k=smooth_k,
                                             pv_mode=pv_mode)
        local.append(dit.q8_views(ws, B, H, Nl, d, pv_mode))
    torch.cuda.synchronize()
    # the slices' codes are the single call's codes
    for r, s in enumerate(sl):
        assert torch.equal(local[r]["q_codes"], ref_v["q_codes"][:, :, s])
        assert torch.equal(local[r]["k_codes"], ref_v["k_codes"][:, :, s])
        assert torch.equal(local[r]["q_scale"], ref_v["q_scale"][:, :, r * Nl // 128:(r + 1) * Nl // 128])
        assert torch.equal(local[r]["k_scale"], ref_v["k_scale"][:, :, r * Nl // 64:(r + 1) * Nl // 64])
        if pv_mode == "fp8":
            assert torch.equal(local[r]["v_codes"], ref_v["v_codes"][:, :, s])
            assert torch.equal(local[r]["v_scale"], ref_v["v_scale"])
    # head group g gathers its heads' codes from every slice (the all-to-all)
    out = torch.empty_like(q)
    for g in range(world):
        heads = slice(g * hp, (g + 1) * hp)
        ws = dit.q8_workspace(B, hp, N, d, pv_mode)
        dst = dit.q8_views(ws, B, hp, N, d, pv_mode)
        names = ["q_codes", "k_codes", "q_scale", "k_scale"] + (["v_codes"] if pv_mode == "fp8" else [])
        for n in names:
            dst[n].copy_(torch.cat([local[r][n][:, heads] for r in range(world)], dim=2))
        if pv_mode == "fp8":
            dst["v_scale"].copy_(local[0]["v_scale"][:, heads])
        vh = None if pv_mode == "fp8" else v[:, heads].contiguous()
        out[:, heads] = dit.dit_attn_fwd_q8_prequantized(ws, B, hp, N, v=vh, pv_mode=pv_mode)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("pv_mode", ["fp8", "bf16"])
def test_ulysses_q8_on_a_group_of_one(pv_mode):
    import torch.distributed as dist
    from diffusion_transformer_attention_attn_b200 import context_parallel as cp
    dit = _dit()
    if dist.is_initialized():
        pytest.skip("a process group is already initialised")
    dist.init_process_group("gloo", store=dist.HashStore(), rank=0, world_size=1)
    try:
        q, k, v = _inputs(N=512, H=2, seed=5)
        ref = dit.dit_attn_fwd_q8(q, k, v, smooth_k=True, pv_mode=pv_mode)
        out = cp.ulysses_attention_q8(q, k, v, smooth_k=True, pv_mode=pv_mode)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    finally:
        dist.destroy_process_group()


def test_prequantized_argument_errors():
    dit = _dit()
    lib = dit.load_library()
    ws = dit.q8_workspace(1, 2, 256, 128, "fp8")
    o = torch.empty(1, 2, 256, 128, dtype=torch.bfloat16, device="cuda")
    assert lib.dit_attn_fwd_q8_prequantized(ws.data_ptr(), 100, None, o.data_ptr(), 1, 2, 256, 128, None, 0.0, 0,
                                            None) == dit.DIT_ERR_WORKSPACE
    assert lib.dit_attn_fwd_q8_prequantized(ws.data_ptr(), ws.numel(), None, o.data_ptr(), 1, 2, 256, 64, None, 0.0,
                                            0, None) == dit.DIT_ERR_UNSUPPORTED
    # bf16-PV mode needs V
    assert lib.dit_attn_fwd_q8_prequantized(ws.data_ptr(), ws.numel(), None, o.data_ptr(), 1, 2, 256, 128, None, 0.0,
                                            1, None) == dit.DIT_ERR_INVALID_ARG
    # the output may not lie inside the workspace
    assert lib.dit_attn_fwd_q8_prequantized(ws.data_ptr(), ws.numel(), None, ws.data_ptr() + 4096, 1, 2, 256, 128,
                                            None, 0.0, 0, None) == dit.DIT_ERR_WORKSPACE
