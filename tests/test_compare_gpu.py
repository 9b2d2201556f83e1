"""Parity of the on-device output comparison (dit_compare_stats, through the C
ABI) with the oracle's fp64 error measures.

Bar: relative L1 within 1e-5 (relative), cosine within 1e-6 (absolute),
max |difference| within 1e-6 (relative); closed forms exactly.
"""
import numpy as np
import pytest

import oracle
from diffusion_transformer_attention_attn_b200 import inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

REL_L1_ERR = 1e-5
COS_ERR = 1e-6
MAX_ERR = 1e-6


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


def _dev(x):
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _bits(t):
    """Device tensor -> host array of the oracle's input types."""
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return t.contiguous().cpu().numpy()


def _check(ref_t, test_t, segments):
    dit = _dit()
    out = dit.dit_compare_stats(ref_t, test_t, segments).cpu().numpy()
    rel, cos, mx = oracle.compare_stats(_bits(ref_t), _bits(test_t), segments)
    for s in range(segments):
        if np.isinf(rel[s]) or rel[s] == 0.0:
            assert out[s, 0] == rel[s]
        else:
            assert abs(out[s, 0] - rel[s]) <= REL_L1_ERR * rel[s], (s, out[s, 0], rel[s])
        assert abs(out[s, 1] - cos[s]) <= COS_ERR, (s, out[s, 1], cos[s])
        assert abs(out[s, 2] - mx[s]) <= MAX_ERR * max(mx[s], 1e-30), (s, out[s, 2], mx[s])
    return out


def test_bf16_against_q8_attention_per_head():
    # the per-layer probe: 16-bit vs 8-bit output of one attention layer
    dit = _dit()
    q, k, v = (_dev(x) for x in inputs.attn_inputs(inputs.IMAGE_Q8, N=1536))
    o16 = dit.dit_attn_fwd(q, k, v)
    o8 = dit.dit_attn_fwd_q8(q, k, v, smooth_k=True, pv_mode="fp8")
    B, H, N, d = q.shape
    out = _check(o16, o8, B * H)
    assert (out[:, 1] > 0.99).all()
    _check(o16, o8, 1)


@pytest.mark.parametrize("segments,seg_len", [(1, 1), (1, 7), (3, 1000), (5, 4099), (48, 4096), (1, 3 << 20),
                                              (4000, 96)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_random_shapes(segments, seg_len, dtype):
    rng = np.random.default_rng(segments * 7919 + seg_len)
    a = rng.standard_normal(segments * seg_len).astype(np.float32)
    b = (a * rng.uniform(0.9, 1.1, a.size) + 0.01 * rng.standard_normal(a.size)).astype(np.float32)
    if dtype == "bf16":
        a, b = inputs.bf16_bits(a), inputs.bf16_bits(b)
    _check(_dev(a), _dev(b), segments)


def test_unaligned_views_take_the_scalar_path():
    rng = np.random.default_rng(3)
    a = _dev(inputs.bf16_bits(rng.standard_normal(10001).astype(np.float32)))
    b = _dev(inputs.bf16_bits(rng.standard_normal(10001).astype(np.float32)))
    _check(a[1:], b[1:], 4)          # base 2 bytes off a 16-byte boundary, 2500 per segment


def test_closed_forms_on_device():
    dit = _dit()
    x = _dev(np.linspace(-3, 5, 4096).astype(np.float32))
    out = dit.dit_compare_stats(x, x.clone(), 2).cpu().numpy()
    assert (out[:, 0] == 0).all() and (out[:, 2] == 0).all()
    np.testing.assert_allclose(out[:, 1], 1.0, atol=1e-12)
    out = dit.dit_compare_stats(x, -x, 1).cpu().numpy()
    assert out[0, 0] == 2.0 and abs(out[0, 1] + 1.0) < 1e-12 and out[0, 2] == 10.0
    z = torch.zeros(256, device="cuda")
    out = dit.dit_compare_stats(z, z, 1).cpu().numpy()
    assert tuple(out[0]) == (0.0, 1.0, 0.0)
    out = dit.dit_compare_stats(z, torch.ones_like(z), 1).cpu().numpy()
    assert out[0, 0] == np.inf and out[0, 1] == 0.0 and out[0, 2] == 1.0


def test_workspace_reuse_is_deterministic():
    dit = _dit()
    rng = np.random.default_rng(9)
    a = _dev(rng.standard_normal(1 << 20).astype(np.float32))
    b = _dev(rng.standard_normal(1 << 20).astype(np.float32))
    ws = torch.zeros(dit.dit_compare_workspace_bytes(8, 1 << 17, dit.DIT_DTYPE_F32), dtype=torch.uint8,
                     device="cuda")
    first = dit.dit_compare_stats(a, b, 8, workspace=ws).cpu().numpy()
    for _ in range(3):
        again = dit.dit_compare_stats(a, b, 8, workspace=ws).cpu().numpy()
        assert np.array_equal(first, again)
