"""Parity of attention over separate query / key lengths with log-sum-exp
output (dit_attn_fwd_ex) and of the key-chunk merge (dit_attn_merge), through
the C ABI, with the fp64 oracle.

Bar: outputs within the bf16 bar (max |dO| <= 2e-2, relative L1 <= 5e-3);
log-sum-exp within 1e-3 absolute (fp32 row max and sum, exp2 approximations
of relative error <= 7.5e-5).
"""
import numpy as np
import pytest

import oracle
from diffusion_transformer_attention_attn_b200 import inputs
from tests.common import assert_bf16_parity, from_device_bf16, to_device_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

LSE_ABS = 1e-3


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


def _qkv(Nq, Nkv, d, H=2, B=1, seed=0):
    """q from one case draw, k and v from another length of the same distribution."""
    case = inputs.AttnCase(f"ex_{Nq}_{Nkv}_{d}", B, H, max(Nq, Nkv), d, seed=seed)
    q, k, v = inputs.attn_inputs(case)
    return (np.ascontiguousarray(q[:, :, :Nq]), np.ascontiguousarray(k[:, :, :Nkv]),
            np.ascontiguousarray(v[:, :, :Nkv]))


def _check_lse(got, ref, what=""):
    err = float(np.abs(got.cpu().numpy().astype(np.float64) - ref).max())
    assert err <= LSE_ABS, f"{what}: max|dlse|={err:.3e}"


@pytest.mark.parametrize("Nq,Nkv", [(300, 1000), (4608, 512), (129, 1), (1, 257), (256, 256), (1000, 4097)])
@pytest.mark.parametrize("d", [64, 128])
def test_ex_against_oracle(Nq, Nkv, d):
    dit = _dit()
    q, k, v = _qkv(Nq, Nkv, d, seed=Nq + Nkv)
    o, lse = dit.dit_attn_fwd_ex(to_device_bf16(q), to_device_bf16(k), to_device_bf16(v), lse=True)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_lse(q, k, v)
    assert_bf16_parity(from_device_bf16(o), o_ref, f"Nq={Nq} Nkv={Nkv} d={d}")
    _check_lse(lse, lse_ref, f"Nq={Nq} Nkv={Nkv} d={d}")


def test_ex_equals_fwd_when_lengths_match():
    dit = _dit()
    q, k, v = (to_device_bf16(x) for x in inputs.attn_inputs(inputs.TINY))
    o1 = dit.dit_attn_fwd(q, k, v)
    o2, _ = dit.dit_attn_fwd_ex(q, k, v)
    o3, _ = dit.dit_attn_fwd_ex(q, k, v, lse=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(o1, o3)


def test_ex_strided_token_major_layout():
    # q/o and k/v as [B, N, H, d] buffers viewed as [B, H, N, d]
    dit = _dit()
    q, k, v = _qkv(700, 900, 128, H=3, seed=5)
    tq = to_device_bf16(np.ascontiguousarray(q.transpose(0, 2, 1, 3))).permute(0, 2, 1, 3)
    tk = to_device_bf16(np.ascontiguousarray(k.transpose(0, 2, 1, 3))).permute(0, 2, 1, 3)
    tv = to_device_bf16(np.ascontiguousarray(v.transpose(0, 2, 1, 3))).permute(0, 2, 1, 3)
    o = torch.empty_like(tq)
    o, lse = dit.dit_attn_fwd_ex(tq, tk, tv, o=o, lse=True)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_lse(q, k, v)
    assert_bf16_parity(from_device_bf16(o), o_ref, "token-major")
    _check_lse(lse, lse_ref, "token-major")


def _chunked(dit, q, k, v, cuts):
    """Ring-style key chunks on one GPU: one dit_attn_fwd_ex per chunk on a
    view of K/V, then dit_attn_merge."""
    outs, lses, a = [], [], 0
    for c in cuts:
        o_c, l_c = dit.dit_attn_fwd_ex(q, k[:, :, a:a + c], v[:, :, a:a + c], lse=True)
        outs.append(o_c)
        lses.append(l_c)
        a += c
    return dit.dit_attn_merge(outs, lses, lse=True)


@pytest.mark.parametrize("N,cuts,d", [(1000, [1000], 64), (1000, [300, 700], 128), (4608, [1152] * 4, 128),
                                      (4099, [1, 2048, 2050], 128), (2000, [125] * 16, 64)])
def test_chunk_merge_equals_full_attention(N, cuts, d):
    dit = _dit()
    assert sum(cuts) == N
    q, k, v = _qkv(N, N, d, H=4, seed=len(cuts))
    tq, tk, tv = (to_device_bf16(x) for x in (q, k, v))
    o, lse = _chunked(dit, tq, tk, tv, cuts)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_lse(q, k, v)
    assert_bf16_parity(from_device_bf16(o), o_ref, f"cuts={cuts}")
    _check_lse(lse, lse_ref, f"cuts={cuts}")


def test_merge_single_part_and_empty_part():
    dit = _dit()
    q, k, v = (to_device_bf16(x) for x in _qkv(512, 512, 128, H=2, seed=9))
    o1, l1 = dit.dit_attn_fwd_ex(q, k, v, lse=True)
    m, ml = dit.dit_attn_merge([o1], [l1], lse=True)
    torch.cuda.synchronize()
    assert torch.equal(m, o1) and torch.equal(ml, l1)
    # a part whose rows all have lse = -inf carries no weight
    junk = torch.randn_like(o1.float()).to(torch.bfloat16)
    none = torch.full_like(l1, float("-inf"))
    m2, ml2 = dit.dit_attn_merge([o1, junk], [l1, none], lse=True)
    torch.cuda.synchronize()
    assert torch.equal(m2, o1) and torch.equal(ml2, l1)
    # every part empty: zeros and -inf
    m3, ml3 = dit.dit_attn_merge([junk], [none], lse=True)
    torch.cuda.synchronize()
    assert not m3.float().abs().any() and torch.isneginf(ml3).all()
