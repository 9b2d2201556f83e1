"""8-bit attention path through the C ABI.

Two layers of checks:
  * the pre-pass (INT8 Q per 128 tokens, INT8 K per 64 tokens after the
    optional channel-mean subtraction, per-channel e4m3 V) must reproduce the
    oracle's fp32 quantiser bit for bit, including the zero-scale guard;
  * the attention output is compared with the exact fp64 attention on the
    unquantised bf16 inputs, so quantisation error counts against it.

Tolerances (see tests/common.py):
  * PV in bf16 (INT8 QKᵀ only): cosine >= 0.999 and relative L1 <= 2e-2, the
    parity bar for the 8-bit path.
  * PV in FP8 e4m3: cosine >= 0.999, and relative L1 <= 5e-2.  Rounding V to
    e4m3's 3-bit mantissa alone gives a relative L1 of about 2.7% on i.i.d.
    N(0,1) data (measured with the oracle, no kernel involved: see
    test_fp8_value_rounding_floor in tests/test_oracle_pins.py).  P's own e4m3
    rounding adds a similar independent term, and INT8 QKᵀ about 1.3%; their
    root-sum-square is about 4%.
"""
import numpy as np
import pytest

import oracle
from diffusion_transformer_attention_attn_b200 import inputs
from tests.common import Q8_COSINE, Q8_REL_L1, cosine, from_device_bf16, rel_l1, to_device_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

FP8_REL_L1 = 5e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import diffusion_transformer_attention_attn_b200 as dit
    dit.load_library()
    yield
    assert dit.dit_get_device_status() == 0


def _dev(q, k, v):
    return tuple(to_device_bf16(t) for t in (q, k, v))


def _run(q, k, v, mode, smooth=True):
    import diffusion_transformer_attention_attn_b200 as dit
    o = dit.dit_attn_fwd_q8(*_dev(q, k, v), smooth_k=smooth, pv_mode=mode)
    torch.cuda.synchronize()
    return from_device_bf16(o)


def _check(out, ref, mode, what):
    assert np.isfinite(out).all(), what
    c, r = cosine(out, ref), rel_l1(out, ref)
    bound = Q8_REL_L1 if mode == "bf16" else FP8_REL_L1
    assert c >= Q8_COSINE and r <= bound, f"{what} [{mode}]: cos={c:.6f} relL1={r:.3e}"
    return c, r


# ---------------------------------------------------------------- pre-pass, bit for bit

def _check_prepass(q, k, v, smooth):
    """The pre-pass products equal the oracle's fp32 quantiser bit for bit."""
    import diffusion_transformer_attention_attn_b200 as dit
    B, H, n, d = q.shape
    ws = dit.dit_attn_q8_quantize(*_dev(q, k, v), smooth_k=smooth, pv_mode="fp8")
    torch.cuda.synchronize()
    views = {name: t.cpu().numpy() for name, t in dit.q8_views(ws, B, H, n, d, "fp8").items()}
    mean = oracle.channel_mean(k) if smooth else None
    if smooth:
        np.testing.assert_array_equal(views["k_mean"], mean)
    qc, qs = oracle.quant_int8_blocks(q, 128)
    kc, ks = oracle.quant_int8_blocks(k, 64, mean)
    vc, vs = oracle.quant_e4m3_channels(v)
    np.testing.assert_array_equal(views["q_scale"], qs)
    np.testing.assert_array_equal(views["q_codes"], qc)
    np.testing.assert_array_equal(views["k_scale"], ks)
    np.testing.assert_array_equal(views["k_codes"], kc)
    np.testing.assert_array_equal(views["v_scale"], vs)
    np.testing.assert_array_equal(views["v_codes"], vc)


@pytest.mark.parametrize("case,N,smooth", [
    (inputs.IMAGE_Q8, 1000, True),
    (inputs.IMAGE_Q8, 1000, False),
    (inputs.AttnCase("q8_small", 2, 3, 333, 128, k_offset_std=2.0, seed=21), None, True),
    (inputs.AttnCase("q8_one", 1, 1, 1, 128, seed=22), None, True),
    (inputs.AttnCase("q8_d64", 2, 3, 333, 64, k_offset_std=3.0, zero_q_channel=5, zero_q_tokens=(128, 256),
                     seed=23), None, True),
    (inputs.AttnCase("q8_d64", 2, 3, 333, 64, k_offset_std=3.0, zero_q_channel=5, zero_q_tokens=(128, 256),
                     seed=23), None, False),
    (inputs.AttnCase("q8_d64_one", 1, 1, 1, 64, seed=25), None, True),
], ids=lambda x: getattr(x, "name", str(x)))
def test_prepass_matches_oracle_quantiser(case, N, smooth):
    _check_prepass(*inputs.attn_inputs(case, N=N), smooth)


def _tiny_maxima_inputs(d):
    """Q block 2 (tokens 256-383) with amax 1e-37, K block 1 (tokens 64-127)
    with amax 1e-37, V channel 9 of {0, 1e-37} and channel 10 with amax 1e-36:
    every one of them has a maximum whose inverse overflows fp32."""
    case = inputs.AttnCase(f"q8tiny{d}", 1, 2, 512, d, seed=24)
    q, k, v = (inputs.bf16_to_f32(t).copy() for t in inputs.attn_inputs(case))
    q[:, :, 256:384, :] = 0.0
    q[:, :, 256:384:2, 3] = 1e-37
    k[:, :, 64:128, :] = 0.0
    k[:, :, 64:128:5, 1] = -1e-37
    v[:, :, :, 9] = 0.0
    v[:, :, ::3, 9] = 1e-37
    v[:, :, :, 10] = 0.0
    v[:, :, 7, 10] = 1e-36
    return tuple(inputs.bf16_bits(t) for t in (q, k, v))


@pytest.mark.parametrize("d", [128, 64])
def test_zero_scale_guard_for_maxima_without_a_finite_inverse(d):
    # An amax so small that 127/amax (or 448/amax) overflows fp32 would give
    # inv = inf and turn the block's zeros into NaN codes.  The guard treats
    # such a block or channel as zero: codes and scales equal the oracle's, and
    # the outputs are finite and meet the 8-bit bar.
    import diffusion_transformer_attention_attn_b200 as dit
    q, k, v = _tiny_maxima_inputs(d)
    _check_prepass(q, k, v, smooth=False)
    ws = dit.dit_attn_q8_quantize(*_dev(q, k, v), smooth_k=False, pv_mode="fp8")
    views = dit.q8_views(ws, 1, 2, 512, d, "fp8")
    assert (views["q_scale"][:, :, 2] == 0).all().item() and (views["k_scale"][:, :, 1] == 0).all().item()
    assert (views["v_scale"][:, :, 9:11] == 0).all().item()
    ref = oracle.attention(q, k, v)
    for mode in ("fp8", "bf16"):
        for smooth in (False, True):
            _check(_run(q, k, v, mode, smooth), ref, mode, f"d={d} smooth={smooth}")


def test_zero_scale_guard():
    # Q channel 7 and Q tokens [640, 768) (one whole 128-token block) are zero.
    import diffusion_transformer_attention_attn_b200 as dit
    case = inputs.IMAGE_Q8
    q, k, v = inputs.attn_inputs(case, N=1000)
    ws = dit.dit_attn_q8_quantize(*_dev(q, k, v), smooth_k=True, pv_mode="fp8")
    views = dit.q8_views(ws, 1, 24, 1000, 128, "fp8")
    assert (views["q_scale"][:, :, 5] == 0).all().item()
    assert (views["q_codes"][:, :, 640:768] == 0).all().item()
    assert (views["q_codes"][..., 7] == 0).all().item()
    for mode in ("fp8", "bf16"):
        out = _run(q, k, v, mode)
        assert np.isfinite(out).all()
        # a zero query row attends uniformly: O = column mean of V
        mean_v = inputs.bf16_to_f32(v).astype(np.float64).mean(axis=2)
        assert np.abs(out[:, :, 640:768] - mean_v[:, :, None, :]).max() <= (2e-3 if mode == "bf16" else 6e-3)


# ---------------------------------------------------------------- attention parity

@pytest.mark.parametrize("mode", ["bf16", "fp8"])
@pytest.mark.parametrize("N", [1, 63, 64, 65, 127, 128, 129, 255, 256, 300, 1000])
def test_ragged_lengths(N, mode):
    case = inputs.AttnCase(f"q8r{N}", 1, 2, N, 128, k_offset_std=2.0, seed=100 + N)
    q, k, v = inputs.attn_inputs(case)
    _check(_run(q, k, v, mode), oracle.attention(q, k, v), mode, f"N={N}")


@pytest.mark.parametrize("mode", ["bf16", "fp8"])
@pytest.mark.parametrize("N", [1, 63, 64, 65, 127, 128, 129, 255, 256, 300, 1000])
def test_ragged_lengths_d64(N, mode):
    case = inputs.AttnCase(f"q8r{N}d64", 1, 2, N, 64, k_offset_std=2.0, seed=300 + N)
    q, k, v = inputs.attn_inputs(case)
    _check(_run(q, k, v, mode), oracle.attention(q, k, v), mode, f"d=64 N={N}")


@pytest.mark.parametrize("mode", ["bf16", "fp8"])
def test_image_shape_d64_sampled_rows(mode):
    # The 8-bit image recipe (K offsets, a zero Q channel and a zero Q block)
    # at head dimension 64: B=1, H=24, N=4608.
    import diffusion_transformer_attention_attn_b200 as dit
    case = inputs.AttnCase("image_q8_d64", 1, 24, 4608, 64, k_offset_std=5.0, zero_q_channel=7,
                           zero_q_tokens=(640, 768), seed=26)
    q, k, v = inputs.attn_inputs(case)
    o = dit.dit_attn_fwd_q8(*_dev(q, k, v), smooth_k=True, pv_mode=mode)
    torch.cuda.synchronize()
    rows = np.union1d(inputs.sample_rows(case.N, 64), [640, 767, 4607])
    out = from_device_bf16(o[:, :, torch.from_numpy(rows).cuda()])
    _check(out, oracle.attention(q, k, v, rows=rows), mode, case.name)
    assert torch.isfinite(o.float()).all().item()


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("mode", ["bf16", "fp8"])
def test_token_major_strided_layout(mode, d):
    # [B, N, H, d] storage viewed as [B, H, N, d]: the pre-pass reads and the
    # output is written through the strides; same result as the contiguous call.
    import diffusion_transformer_attention_attn_b200 as dit
    case = inputs.AttnCase(f"q8str{d}", 2, 3, 300, d, k_offset_std=2.0, seed=71)
    q, k, v = inputs.attn_inputs(case)
    qs, ks, vs = (to_device_bf16(np.ascontiguousarray(t.transpose(0, 2, 1, 3))).permute(0, 2, 1, 3)
                  for t in (q, k, v))
    o = torch.empty_like(qs)
    dit.dit_attn_fwd_q8(qs, ks, vs, o=o, smooth_k=True, pv_mode=mode)
    ref = dit.dit_attn_fwd_q8(*_dev(q, k, v), smooth_k=True, pv_mode=mode)
    torch.cuda.synchronize()
    assert torch.equal(o, ref)
    _check(from_device_bf16(o), oracle.attention(q, k, v), mode, f"strided d={d}")


@pytest.mark.parametrize("mode", ["bf16", "fp8"])
def test_batch_heads_and_explicit_scale(mode):
    import diffusion_transformer_attention_attn_b200 as dit
    case = inputs.AttnCase("q8bh", 2, 3, 200, 128, seed=31)
    q, k, v = inputs.attn_inputs(case)
    o = dit.dit_attn_fwd_q8(*_dev(q, k, v), scale=0.05, pv_mode=mode)
    torch.cuda.synchronize()
    _check(from_device_bf16(o), oracle.attention(q, k, v, scale=float(np.float32(0.05))), mode, "B=2 H=3 s=0.05")


@pytest.mark.parametrize("mode", ["bf16", "fp8"])
def test_image_q8_workload_sampled_rows(mode):
    # The 8-bit image workload at full size (N=4608), smooth_k on (held to the 8-bit tolerances).
    import diffusion_transformer_attention_attn_b200 as dit
    case = inputs.IMAGE_Q8
    q, k, v = inputs.attn_inputs(case)
    o = dit.dit_attn_fwd_q8(*_dev(q, k, v), smooth_k=True, pv_mode=mode)
    torch.cuda.synchronize()
    rows = inputs.sample_rows(case.N, 96)
    rows = np.union1d(rows, [640, 700, 767])   # rows of the zero Q block
    out = from_device_bf16(o[:, :, torch.from_numpy(rows).cuda()])
    _check(out, oracle.attention(q, k, v, rows=rows), mode, case.name)


def test_image_q8_without_smoothing_reported():
    # smooth_k = 0: K's per-channel offsets (std 5) set the INT8 scale, so the
    # N(0,1) part is quantised coarsely.  Reported, not held to the tolerances: finite, and
    # still strongly correlated with the exact result.
    import diffusion_transformer_attention_attn_b200 as dit
    case = inputs.IMAGE_Q8
    q, k, v = inputs.attn_inputs(case, N=2048)
    o = from_device_bf16(dit.dit_attn_fwd_q8(*_dev(q, k, v), smooth_k=False, pv_mode="fp8"))
    ref = oracle.attention(q, k, v, rows=np.arange(0, 2048, 16))
    out = o[:, :, ::16]
    assert np.isfinite(o).all() and cosine(out, ref) >= 0.99


def test_fp8_kernel_tracks_quantised_emulation():
    # Kernel error beyond quantisation: compare with fp64 attention on the
    # dequantised Q, K, V (P's e4m3 rounding is the only unmodelled step).
    case = inputs.AttnCase("q8emu", 1, 2, 777, 128, k_offset_std=2.0, seed=41)
    q, k, v = inputs.attn_inputs(case)
    out = _run(q, k, v, "fp8")
    emu = oracle.emulated_q8_attention(q, k, v, smooth_k=True)
    assert cosine(out, emu) >= 0.9995 and rel_l1(out, emu) <= 3.5e-2


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("mode", ["fp8", "bf16"])
def test_growing_logits_rescaling_path(mode, d):
    # Logits grow along the key axis, so each row's running max moves past the
    # rescale threshold tile after tile (2 in log2 units with FP8 P, 8 with bf16
    # P) and O is rescaled in tensor memory again and again.  Logits this large
    # magnify the INT8 rounding of Q and K beyond the 8-bit bar, so the kernel
    # is held to the fp64 attention over the same dequantised codes (which
    # models everything but P's own rounding), and to the exact attention only
    # loosely.  V is scaled by 1/4 so the nearly one-hot rows keep |O| in the
    # workloads' range.
    case = inputs.AttnCase("q8grow", 1, 2, 1024, d, seed=71)
    q, k, v = inputs.attn_inputs(case)
    qf = inputs.bf16_to_f32(q) * np.float32(3.0)
    ramp = np.linspace(0.0, 4.0, case.N, dtype=np.float32)[None, None, :, None]
    kf = inputs.bf16_to_f32(k) * (1.0 + ramp)
    q, k = inputs.bf16_bits(qf), inputs.bf16_bits(kf)
    v = inputs.bf16_bits(inputs.bf16_to_f32(v) * np.float32(0.25))
    out = _run(q, k, v, mode)
    assert np.isfinite(out).all()
    if mode == "fp8":
        emu = oracle.emulated_q8_attention(q, k, v, smooth_k=True)
    else:
        # bf16 P·V keeps V in bf16: only Q and K are dequantised codes
        qc, qs = oracle.quant_int8_blocks(q, 128)
        kc, ks = oracle.quant_int8_blocks(k, 64, oracle.channel_mean(k))
        tok = np.arange(case.N)
        qd = qc.astype(np.float64) * qs[:, :, tok // 128, None].astype(np.float64)
        kd = kc.astype(np.float64) * ks[:, :, tok // 64, None].astype(np.float64)
        emu = oracle.attention(qd, kd, inputs.bf16_to_f32(v).astype(np.float64))
    c, r = cosine(out, emu), rel_l1(out, emu)
    print(f"growing logits d={d} [{mode}] vs dequantised fp64: cos={c:.6f} relL1={r:.3e}")
    if mode == "fp8":
        assert c >= 0.9995 and r <= 3.5e-2, (c, r)
    else:
        assert c >= 0.99999 and r <= 5e-3, (c, r)
    ref = oracle.attention(q, k, v)
    print(f"  vs exact fp64: cos={cosine(out, ref):.6f} relL1={rel_l1(out, ref):.3e}")
    assert cosine(out, ref) >= 0.995


def test_smoothing_is_softmax_invariant():
    # Adding a per-channel offset to every key leaves the smoothed path's
    # quantised K unchanged up to rounding: outputs agree closely.
    case = inputs.AttnCase("q8inv", 1, 2, 640, 128, seed=51)
    q, k, v = inputs.attn_inputs(case)
    mu = np.random.Generator(np.random.PCG64(52)).standard_normal((1, 2, 1, 128)).astype(np.float32) * 3
    k2 = inputs.bf16_bits(inputs.bf16_to_f32(k) + mu)
    a, b = _run(q, k, v, "bf16"), _run(q, k2, v, "bf16")
    assert cosine(a, b) >= 0.999 and rel_l1(a, b) <= 2e-2


@pytest.mark.parametrize("mode", ["bf16", "fp8"])
def test_deterministic(mode):
    case = inputs.AttnCase("q8det", 1, 4, 1500, 128, seed=61)
    q, k, v = inputs.attn_inputs(case)
    assert np.array_equal(_run(q, k, v, mode), _run(q, k, v, mode))


def test_video_mid_workload_sampled_rows():
    # Mid video (N=45760) with K-mean smoothing and FP8 PV, the bench's launch.
    import diffusion_transformer_attention_attn_b200 as dit
    case = inputs.VIDEO_MID
    q, k, v = inputs.attn_inputs(case)
    for mode in ("fp8", "bf16"):
        o = dit.dit_attn_fwd_q8(*_dev(q, k, v), smooth_k=True, pv_mode=mode)
        torch.cuda.synchronize()
        rows = inputs.sample_rows(case.N, 16)
        out = from_device_bf16(o[:, :, torch.from_numpy(rows).cuda()])
        _check(out, oracle.attention(q, k, v, rows=rows), mode, case.name)
        assert torch.isfinite(o.float()).all().item()


def test_video_long_workload_sampled_rows():
    # The benchmark's workload (N=119056, K offsets) in the benchmark's launch:
    # K-mean smoothing, FP8 PV; 64 sampled rows per head against all keys.
    import diffusion_transformer_attention_attn_b200 as dit
    case = inputs.VIDEO_LONG
    q, k, v = inputs.attn_inputs(case)
    o = dit.dit_attn_fwd_q8(*_dev(q, k, v), smooth_k=True, pv_mode="fp8")
    torch.cuda.synchronize()
    rows = inputs.sample_rows(case.N, 64)
    out = from_device_bf16(o[:, :, torch.from_numpy(rows).cuda()])
    _check(out, oracle.attention(q, k, v, rows=rows), "fp8", case.name)
    assert torch.isfinite(o.float()).all().item()
