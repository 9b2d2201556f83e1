"""The token-sharded 8-bit path through the C ABI on one GPU.

Against the oracle: each split entry point on its own —
dit_attn_q8_channel_stats against oracle.k_channel_sums / channel_amax,
dit_attn_q8_quantize_global against the oracle's quantisers with the
combined statistics (both bit for bit), and dit_attn_fwd_q8_prequantized
against the exact fp64 attention (the 8-bit bar) and against the fp64
attention over the same codes.

Against the single call:

dit_attn_q8_channel_stats / dit_attn_q8_quantize_global / the codes' move to
the head-sharded layout / dit_attn_fwd_q8_prequantized must give, bit for
bit, the codes and the output of the single dit_attn_fwd_q8 call when every
token slice holds whole 128-token blocks.  Here the slices are views of one
tensor and their combination (sum, max) and the all-to-all are done with
device copies, as the collectives of a Ulysses group would.
"""
import numpy as np
import pytest

import oracle
from diffusion_transformer_attention_attn_b200 import inputs
from tests.common import Q8_COSINE, Q8_REL_L1, cosine, from_device_bf16, rel_l1, to_device_bf16

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


FP8_REL_L1 = 5e-2      # FP8 P·V: e4m3 rounding of V alone costs about 2.7% (see tests/test_q8_gpu.py)


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("pv_mode", ["fp8", "bf16"])
@pytest.mark.parametrize("smooth_k", [True, False])
def test_split_entry_points_match_the_oracle(d, pv_mode, smooth_k):
    dit = _dit()
    world, N, H = 2, 1024, 4
    # K's per-channel offsets need the smoothing to meet the 8-bit bar (without
    # it they set the INT8 scale); the unsmoothed runs take plain N(0,1) keys.
    case = inputs.AttnCase(f"shq8o{d}", 1, H, N, d, k_offset_std=3.0 if smooth_k else 0.0, zero_q_channel=7, seed=9)
    q, k, v = inputs.attn_inputs(case)
    qd, kd, vd = (to_device_bf16(t) for t in (q, k, v))
    B = 1
    Nl, hp = N // world, H // world
    sl = [slice(r * Nl, (r + 1) * Nl) for r in range(world)]
    fp8 = pv_mode == "fp8"
    # 1. per-slice statistics against the oracle's sums and maxima
    stats = [dit.dit_attn_q8_channel_stats(kd[:, :, s], vd[:, :, s], smooth_k=smooth_k, pv_mode=pv_mode) for s in sl]
    torch.cuda.synchronize()
    for (ks_dev, va_dev), s in zip(stats, sl):
        want_sum = oracle.k_channel_sums(k[:, :, s]) if smooth_k else np.zeros((B, H, d))
        want_max = oracle.channel_amax(v[:, :, s]) if fp8 else np.zeros((B, H, d), dtype=np.float32)
        np.testing.assert_array_equal(ks_dev.cpu().numpy(), want_sum)
        np.testing.assert_array_equal(va_dev.cpu().numpy(), want_max)
    k_sum = sum(x for x, _ in stats)
    v_amax = torch.stack([y for _, y in stats]).amax(dim=0)
    # 2. each slice's codes and scales with the combined statistics
    mean = oracle.mean_from_sums(oracle.k_channel_sums(k), N) if smooth_k else None
    amax = oracle.channel_amax(v)
    local = []
    for s in sl:
        ws = dit.dit_attn_q8_quantize_global(qd[:, :, s], kd[:, :, s], vd[:, :, s], k_sum, v_amax, N,
                                             smooth_k=smooth_k, pv_mode=pv_mode)
        views = dit.q8_views(ws, B, H, Nl, d, pv_mode)
        local.append(views)
        got = {n: t.cpu().numpy() for n, t in views.items()}
        qc, qs = oracle.quant_int8_blocks(q[:, :, s], 128)
        kc, ks = oracle.quant_int8_blocks(k[:, :, s], 64, mean)
        np.testing.assert_array_equal(got["q_codes"], qc)
        np.testing.assert_array_equal(got["q_scale"], qs)
        np.testing.assert_array_equal(got["k_codes"], kc)
        np.testing.assert_array_equal(got["k_scale"], ks)
        if smooth_k:
            np.testing.assert_array_equal(got["k_mean"], mean)
        if fp8:
            vc, vs = oracle.quant_e4m3_with_amax(v[:, :, s], amax)
            np.testing.assert_array_equal(got["v_codes"], vc)
            np.testing.assert_array_equal(got["v_scale"], vs)
    # 3. the attention kernel alone on the gathered head groups
    out = torch.empty_like(qd)
    for g in range(world):
        heads = slice(g * hp, (g + 1) * hp)
        ws = dit.q8_workspace(B, hp, N, d, pv_mode)
        dst = dit.q8_views(ws, B, hp, N, d, pv_mode)
        names = ["q_codes", "k_codes", "q_scale", "k_scale"] + (["v_codes"] if fp8 else [])
        for n in names:
            dst[n].copy_(torch.cat([local[r][n][:, heads] for r in range(world)], dim=2))
        if fp8:
            dst["v_scale"].copy_(local[0]["v_scale"][:, heads])
        vh = None if fp8 else vd[:, heads].contiguous()
        out[:, heads] = dit.dit_attn_fwd_q8_prequantized(ws, B, hp, N, v=vh, pv_mode=pv_mode, d=d)
    torch.cuda.synchronize()
    o = from_device_bf16(out)
    ref = oracle.attention(q, k, v)
    c, r = cosine(o, ref), rel_l1(o, ref)
    assert c >= Q8_COSINE and r <= (FP8_REL_L1 if fp8 else Q8_REL_L1), (c, r)
    # against fp64 attention over the very codes the kernel read (whole sequence)
    qc, qs = oracle.quant_int8_blocks(q, 128)
    kc, ks = oracle.quant_int8_blocks(k, 64, mean)
    if fp8:
        vc, vs = oracle.quant_e4m3_with_amax(v, amax)
        emu = oracle.attention_from_codes(qc, qs, kc, ks, vc, vs)
    else:
        emu = oracle.attention_from_codes(qc, qs, kc, ks, v)
    c, r = cosine(o, emu), rel_l1(o, emu)
    # bf16 P·V: only P's bf16 rounding and fp32 sums remain; FP8 P·V: P's e4m3 rounding too
    assert c >= 0.9995 and r <= (3.5e-2 if fp8 else 5e-3), (c, r)


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("pv_mode", ["fp8", "bf16"])
@pytest.mark.parametrize("world", [2, 4])
def test_quantize_scatter_matches_the_oracle_and_the_single_call(world, pv_mode, d):
    # Each rank's quantisers store straight into every rank's head-sharded
    # workspace (the fused all-to-all).  The ranks run one after another on the
    # one GPU; each writes disjoint parts of the destinations.
    dit = _dit()
    H, N = 8, 1024
    case = inputs.AttnCase(f"scat{d}", 1, H, N, d, k_offset_std=3.0, zero_q_channel=5, seed=17)
    q, k, v = inputs.attn_inputs(case)
    qd, kd, vd = (to_device_bf16(t) for t in (q, k, v))
    B, fp8 = 1, pv_mode == "fp8"
    Nl, hp = N // world, H // world
    sl = [slice(r * Nl, (r + 1) * Nl) for r in range(world)]
    stats = [dit.dit_attn_q8_channel_stats(kd[:, :, s], vd[:, :, s], smooth_k=True, pv_mode=pv_mode) for s in sl]
    k_sum = sum(x for x, _ in stats)
    v_amax = torch.stack([y for _, y in stats]).amax(dim=0)
    nbytes = dit.dit_attn_q8_workspace_bytes(B, hp, N, d, pv_mode)
    dst = [torch.full((nbytes,), 0x5A, dtype=torch.uint8, device="cuda") for _ in range(world)]
    ptrs = [t.data_ptr() for t in dst]
    for r, s in enumerate(sl):
        dit.dit_attn_q8_quantize_scatter(qd[:, :, s].contiguous(), kd[:, :, s].contiguous(),
                                         vd[:, :, s].contiguous(), k_sum, v_amax, r, world, ptrs, nbytes,
                                         smooth_k=True, pv_mode=pv_mode)
    torch.cuda.synchronize()
    # codes and scales of every destination against the oracle's whole-sequence quantisers
    mean = oracle.mean_from_sums(oracle.k_channel_sums(k), N)
    qc, qs = oracle.quant_int8_blocks(q, 128)
    kc, ks = oracle.quant_int8_blocks(k, 64, mean)
    vc, vs = oracle.quant_e4m3_with_amax(v, oracle.channel_amax(v))
    out = torch.empty_like(qd)
    for g in range(world):
        heads = slice(g * hp, (g + 1) * hp)
        got = {n: t.cpu().numpy() for n, t in dit.q8_views(dst[g], B, hp, N, d, pv_mode).items()}
        np.testing.assert_array_equal(got["q_codes"], qc[:, heads])
        np.testing.assert_array_equal(got["q_scale"], qs[:, heads])
        np.testing.assert_array_equal(got["k_codes"], kc[:, heads])
        np.testing.assert_array_equal(got["k_scale"], ks[:, heads])
        if fp8:
            np.testing.assert_array_equal(got["v_codes"], vc[:, heads])
            np.testing.assert_array_equal(got["v_scale"], vs[:, heads])
        vh = None if fp8 else vd[:, heads].contiguous()
        out[:, heads] = dit.dit_attn_fwd_q8_prequantized(dst[g], B, hp, N, v=vh, pv_mode=pv_mode, d=d)
    torch.cuda.synchronize()
    assert torch.equal(out, dit.dit_attn_fwd_q8(qd, kd, vd, smooth_k=True, pv_mode=pv_mode))
    o = from_device_bf16(out)
    ref = oracle.attention(q, k, v)
    c, r = cosine(o, ref), rel_l1(o, ref)
    assert c >= Q8_COSINE and r <= (FP8_REL_L1 if fp8 else Q8_REL_L1), (c, r)


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
    assert lib.dit_attn_fwd_q8_prequantized(ws.data_ptr(), ws.numel(), None, o.data_ptr(), 1, 2, 256, 96, None, 0.0,
                                            0, None) == dit.DIT_ERR_UNSUPPORTED
    # bf16-PV mode needs V
    assert lib.dit_attn_fwd_q8_prequantized(ws.data_ptr(), ws.numel(), None, o.data_ptr(), 1, 2, 256, 128, None, 0.0,
                                            1, None) == dit.DIT_ERR_INVALID_ARG
    # the output may not lie inside the workspace
    assert lib.dit_attn_fwd_q8_prequantized(ws.data_ptr(), ws.numel(), None, ws.data_ptr() + 4096, 1, 2, 256, 128,
                                            None, 0.0, 0, None) == dit.DIT_ERR_WORKSPACE
