"""Parity of the first-block-cache reduction (through the C ABI) with the fp64
oracle: relative error of rel <= 1e-5 and the identical skip decision."""
import math

import numpy as np
import pytest

import oracle
from diffusion_transformer_attention_attn_b200 import inputs
from tests.common import FBC_REL_ERR

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


def _dev(x):
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _gpu_rel(cur, prev, thr, ws=None):
    import diffusion_transformer_attention_attn_b200 as dit
    rel, skip = dit.fbc_rel_l1(_dev(cur), _dev(prev), thr, workspace=ws)
    return rel.item(), int(skip.item())


def _check(cur, prev, thr):
    rel_ref, skip_ref = oracle.fbc_rel_l1(cur, prev, thr)
    rel, skip = _gpu_rel(cur, prev, thr)
    if math.isinf(rel_ref) or rel_ref == 0.0:
        assert rel == rel_ref
    else:
        assert abs(rel - rel_ref) <= FBC_REL_ERR * abs(rel_ref), (rel, rel_ref)
    assert skip == skip_ref
    return rel


@pytest.mark.parametrize("case", [inputs.FBC_TINY, inputs.FBC_IMAGE, inputs.FBC_VIDEO_LONG], ids=lambda c: c.name)
def test_workloads(case):
    cur, prev = inputs.fbc_inputs(case)
    _check(cur, prev, case.threshold)


@pytest.mark.parametrize("n", [1, 3, 4, 7, 8, 9, 15, 17, 1000, 4097, 65543, 1 << 20, (1 << 21) + 5])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ragged_sizes(n, dtype):
    case = inputs.FbcCase(f"r{n}", 1, n, dtype, 0.05, 0.08, seed=n % 977)
    cur, prev = inputs.fbc_inputs(case)
    _check(cur.reshape(-1), prev.reshape(-1), 0.08)


def test_decision_both_ways_and_strict_threshold():
    prev = np.array([1.0, -2.0, 3.0, -2.0] * 8, dtype=np.float32)
    cur = prev.copy()
    cur[0::4] += 1.0                            # |diff| sum 8, |prev| sum 64 -> 0.125
    assert _gpu_rel(cur, prev, 0.125) == (0.125, 0)   # equality -> compute
    assert _gpu_rel(cur, prev, 0.13)[1] == 1
    assert _gpu_rel(cur, prev, 0.12)[1] == 0


def test_zero_denominator():
    z = np.zeros(40, dtype=np.float32)
    assert _gpu_rel(z, z, 0.08) == (0.0, 1)
    rel, skip = _gpu_rel(np.ones(40, dtype=np.float32), z, 0.08)
    assert math.isinf(rel) and skip == 0


def test_deterministic_and_workspace_reusable():
    import diffusion_transformer_attention_attn_b200 as dit
    cur, prev = inputs.fbc_inputs(inputs.FbcCase("det", 1000, 3072, "bf16", 0.03, 0.08, seed=3))
    ws = dit.fbc_workspace(cur.size)
    first = _gpu_rel(cur, prev, 0.08, ws)
    for _ in range(3):
        assert _gpu_rel(cur, prev, 0.08, ws) == first
    # the ticket counter is back at zero after each call
    assert int(ws[:4].view(torch.int32).item()) == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_sums_then_finish_equals_one_call_and_shards_add_up(dtype):
    import diffusion_transformer_attention_attn_b200 as dit
    case = inputs.FbcCase(f"s_{dtype}", 1000, 3072, dtype, 0.05, 0.08, seed=3)
    cur, prev = inputs.fbc_inputs(case)
    c, p = _dev(cur).reshape(-1), _dev(prev).reshape(-1)
    rel1, skip1 = dit.fbc_rel_l1(c, p, 0.08)
    sums = dit.fbc_rel_l1_sums(c, p)
    rel2, skip2 = dit.fbc_rel_l1_finish(sums, 0.08)
    assert rel1.item() == rel2.item() and skip1.item() == skip2.item()
    num, den = oracle.fbc_sums(cur, prev)
    s = sums.cpu().numpy()
    assert abs(s[0] - num) <= FBC_REL_ERR * num and abs(s[1] - den) <= FBC_REL_ERR * den
    # three shards of the same residual (as three devices would hold it), added on the device
    n = c.numel()
    cuts = [0, n // 3, n // 3 + 8, n]
    total = sum(dit.fbc_rel_l1_sums(c[a:b], p[a:b]) for a, b in zip(cuts[:-1], cuts[1:]))
    rel3, skip3 = dit.fbc_rel_l1_finish(total.contiguous(), 0.08)
    rel_ref, skip_ref = oracle.fbc_rel_l1(cur, prev, 0.08)
    assert abs(rel3.item() - rel_ref) <= FBC_REL_ERR * rel_ref and int(skip3.item()) == skip_ref
