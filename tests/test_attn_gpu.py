"""Parity of the bf16 attention kernel (through the C ABI) with the fp64 oracle.

Small sizes are compared element by element over the whole output; the
full-size workloads are compared on sampled query rows against all keys
(the oracle computes each sampled row exactly), in the same launch
configuration the bench times.
"""
import math

import numpy as np
import pytest

import oracle
from diffusion_transformer_attention_attn_b200 import inputs
from tests.common import BF16_MAX_ABS, BF16_REL_L1, assert_bf16_parity, from_device_bf16, max_abs, rel_l1, \
    to_device_bf16

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


def _run(q, k, v, scale=None):
    import diffusion_transformer_attention_attn_b200 as dit
    qd, kd, vd = (to_device_bf16(t) for t in (q, k, v))
    od = dit.dit_attn_fwd(qd, kd, vd, scale=scale)
    torch.cuda.synchronize()
    return from_device_bf16(od)


def test_tiny_workload_full_parity():
    c = inputs.TINY
    q, k, v = inputs.attn_inputs(c)
    ref = oracle.attention(q, k, v)
    out = _run(q, k, v)
    assert_bf16_parity(out, ref, c.name)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 7, 63, 64, 127, 128, 129, 255, 256, 257, 383, 640, 1000])
def test_ragged_lengths(N, d):
    case = inputs.AttnCase(f"ragged_{N}_{d}", 1, 3, N, d, seed=N * 7 + d)
    q, k, v = inputs.attn_inputs(case)
    ref = oracle.attention(q, k, v)
    out = _run(q, k, v)
    assert_bf16_parity(out, ref, case.name)


def test_batch_and_heads_layout():
    case = inputs.AttnCase("bh", 2, 3, 300, 128, seed=5)
    q, k, v = inputs.attn_inputs(case)
    assert_bf16_parity(_run(q, k, v), oracle.attention(q, k, v), "B=2 H=3")


def test_explicit_scale():
    case = inputs.AttnCase("scale", 1, 2, 200, 64, seed=6)
    q, k, v = inputs.attn_inputs(case)
    assert_bf16_parity(_run(q, k, v, scale=0.3), oracle.attention(q, k, v, scale=float(np.float32(0.3))), "s=0.3")


def test_large_logits_rescaling_path():
    # Logits grow along the key axis (std up to ~15), so the running max moves
    # by more than the rescale threshold several times: exercises the O rescale
    # in tensor memory.  V is scaled by 1/4 (exact in bf16) so that the nearly
    # one-hot rows keep |O| in the workloads' range, where bf16 rounding of O
    # stays well inside the absolute bound.
    case = inputs.AttnCase("grow", 1, 2, 1024, 128, seed=9)
    q, k, v = inputs.attn_inputs(case)
    qf = inputs.bf16_to_f32(q) * np.float32(3.0)
    ramp = np.linspace(0.0, 4.0, case.N, dtype=np.float32)[None, None, :, None]
    kf = inputs.bf16_to_f32(k) * (1.0 + ramp)
    q, k = inputs.bf16_bits(qf), inputs.bf16_bits(kf)
    v = inputs.bf16_bits(inputs.bf16_to_f32(v) * np.float32(0.25))
    assert_bf16_parity(_run(q, k, v), oracle.attention(q, k, v), "growing logits")


def test_strided_view():
    # q/k/v/o as [B, N, H, d] memory viewed as [B, H, N, d].
    import diffusion_transformer_attention_attn_b200 as dit
    B, H, N, d = 1, 4, 333, 64
    rng = np.random.Generator(np.random.PCG64(12))
    base = [inputs.bf16_bits(rng.standard_normal((B, N, H, d), dtype=np.float32)) for _ in range(3)]
    dev = [to_device_bf16(t).permute(0, 2, 1, 3) for t in base]
    o = torch.empty((B, N, H, d), dtype=torch.bfloat16, device="cuda").permute(0, 2, 1, 3)
    dit.dit_attn_fwd(*dev, o=o)
    torch.cuda.synchronize()
    q, k, v = (np.ascontiguousarray(t.transpose(0, 2, 1, 3)) for t in base)
    assert_bf16_parity(from_device_bf16(o), oracle.attention(q, k, v), "strided")


# ---------------------------------------------------------------- invariants on the device

def test_v_ones_gives_ones():
    case = inputs.AttnCase("v1", 1, 2, 700, 128, seed=13)
    q, k, _ = inputs.attn_inputs(case)
    v = inputs.bf16_bits(np.ones((1, 2, 700, 128), dtype=np.float32))
    out = _run(q, k, v)
    assert np.abs(out - 1.0).max() <= 2 ** -7


def test_q_zero_gives_column_mean():
    case = inputs.AttnCase("q0", 1, 2, 517, 64, seed=14)
    _, k, v = inputs.attn_inputs(case)
    q = np.zeros_like(k)
    out = _run(q, k, v)
    mean = inputs.bf16_to_f32(v).astype(np.float64).mean(axis=2, keepdims=True)
    assert max_abs(out, np.broadcast_to(mean, out.shape)) <= 2e-3


def test_joint_key_value_permutation():
    case = inputs.AttnCase("perm", 1, 2, 450, 128, seed=15)
    q, k, v = inputs.attn_inputs(case)
    perm = np.random.Generator(np.random.PCG64(16)).permutation(case.N)
    a = _run(q, k, v)
    b = _run(q, k[:, :, perm], v[:, :, perm])
    ref = oracle.attention(q, k, v)
    assert_bf16_parity(b, ref, "permuted")
    assert rel_l1(a, b) <= BF16_REL_L1


def test_key_offset_invariance():
    # K + 1·mu shifts every logit of a row by q·mu: O is unchanged.
    case = inputs.AttnCase("koff", 1, 2, 300, 64, seed=17)
    q, k, v = inputs.attn_inputs(case)
    mu = np.random.Generator(np.random.PCG64(18)).standard_normal((1, 2, 1, 64)).astype(np.float32) * 2
    k2 = inputs.bf16_bits(inputs.bf16_to_f32(k) + mu)
    ref = oracle.attention(q, k2, v)
    assert_bf16_parity(_run(q, k2, v), ref, "offset K")
    assert rel_l1(_run(q, k2, v), oracle.attention(q, k, v)) <= 2 * BF16_REL_L1


def test_deterministic():
    case = inputs.AttnCase("det", 1, 4, 1500, 128, seed=19)
    q, k, v = inputs.attn_inputs(case)
    a, b = _run(q, k, v), _run(q, k, v)
    assert np.array_equal(a, b)


# ---------------------------------------------------------------- full-size workloads, sampled rows

@pytest.mark.parametrize("case,count", [(inputs.IMAGE, 96), (inputs.VIDEO_MID, 24), (inputs.VIDEO_LONG, 64),
                                        (inputs.AttnCase("image_b1h24n4608d64", 1, 24, 4608, 64, seed=27), 96)],
                         ids=lambda x: getattr(x, "name", str(x)))
def test_full_size_sampled_rows(case, count):
    import diffusion_transformer_attention_attn_b200 as dit
    q, k, v = inputs.attn_inputs(case)
    qd, kd, vd = (to_device_bf16(t) for t in (q, k, v))
    od = dit.dit_attn_fwd(qd, kd, vd)
    torch.cuda.synchronize()
    rows = inputs.sample_rows(case.N, count)
    out = from_device_bf16(od[:, :, torch.from_numpy(rows).cuda()])
    ref = oracle.attention(q, k, v, rows=rows)
    assert_bf16_parity(out, ref, case.name)
    # every output finite, and no untouched (garbage) rows
    assert torch.isfinite(od.float()).all().item()
