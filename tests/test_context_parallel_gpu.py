"""Context-parallel attention with the library's kernels in the loop, P ranks
simulated in one process on the one GPU.

ParaAttention page, "Context Parallelism" (Ulysses and ring attention), and
the TMAP image-to-video blog, sequence parallelism with 8-bit attention: each
rank holds N/P tokens of every head.  Here each rank is a thread that runs the
real ``context_parallel`` functions with their default kernels
(dit_attn_fwd, dit_attn_fwd_ex + dit_attn_merge, the split 8-bit entry points,
fbc_rel_l1_sums / fbc_rel_l1_finish).  Only the collectives are stood in for:
``LocalComm`` moves the tensors between the ranks with device copies, the
ranks meeting at a host barrier.  No kernel waits on another rank's kernel.

The gathered outputs must match the oracle's full-sequence results, and the
Ulysses outputs must equal the single-device calls bit for bit (every head
sees the same keys in the same order).  A layout slip between the all-to-all
and the kernels' strides fails here.  The 8-bit Ulysses runs both with the
code all-to-all and with the fused quantise-and-scatter, each rank's
quantisers storing into every rank's workspace (here all on the one GPU).
"""
import threading

import numpy as np
import pytest

import oracle
from diffusion_transformer_attention_attn_b200 import inputs
from tests.common import (FBC_REL_ERR, Q8_COSINE, Q8_REL_L1, assert_bf16_parity, cosine, from_device_bf16, rel_l1,
                          to_device_bf16)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

FP8_REL_L1 = 5e-2     # FP8 P·V (see tests/test_q8_gpu.py)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import diffusion_transformer_attention_attn_b200 as dit
    dit.load_library()
    yield
    assert dit.dit_get_device_status() == 0


class _Hub:
    def __init__(self, world):
        self.world = world
        self.barrier = threading.Barrier(world, timeout=300)
        self.slots = [None] * world


class LocalComm:
    """The collectives of ``context_parallel.TorchComm`` among threads of one
    process: every step publishes this rank's tensor, copies what it needs
    from the others' on the device, and waits at the barrier until all copies
    have completed, so no rank frees or rewrites a tensor another still reads."""

    def __init__(self, hub, rank):
        self.hub, self.rank, self.world = hub, rank, hub.world

    def _gather(self, t):
        torch.cuda.synchronize()
        self.hub.slots[self.rank] = t
        self.hub.barrier.wait()
        return list(self.hub.slots)

    def _done(self):
        torch.cuda.synchronize()
        self.hub.barrier.wait()

    def all_to_all(self, recv, send):
        parts = self._gather(send)
        for i in range(self.world):
            recv[i].copy_(parts[i][self.rank])
        self._done()

    def all_reduce(self, t, op="sum"):
        parts = self._gather(t.clone())
        acc = parts[0].clone()
        for p in parts[1:]:
            acc = acc + p if op == "sum" else torch.maximum(acc, p)
        self._done()
        t.copy_(acc)

    def ring_exchange(self, send, recv):
        parts = self._gather(send)
        recv.copy_(parts[(self.rank - 1) % self.world])
        self._done()
        return []

    def shared_workspace(self, nbytes, device):
        buf = torch.empty(int(nbytes), dtype=torch.uint8, device=device)
        parts = self._gather(buf)
        ptrs = [t.data_ptr() for t in parts]
        self._done()
        return buf, ptrs

    def barrier(self):
        torch.cuda.synchronize()
        self.hub.barrier.wait()


def _run_ranks(world, fn):
    """fn(rank, comm) on `world` threads; returns the per-rank results."""
    hub = _Hub(world)
    results, errors = [None] * world, []

    def body(r):
        try:
            results[r] = fn(r, LocalComm(hub, r))
        except BaseException as e:   # noqa: BLE001 - reported below
            errors.append(e)
            hub.barrier.abort()
    threads = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    if errors:
        raise errors[0]
    torch.cuda.synchronize()
    return results


def _case(H, N, d, seed, **kw):
    q, k, v = inputs.attn_inputs(inputs.AttnCase(f"cpg{seed}", 1, H, N, d, seed=seed, **kw))
    return (q, k, v), tuple(to_device_bf16(t) for t in (q, k, v))


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("d", [128, 64])
def test_ulysses_with_the_kernels(world, d):
    import diffusion_transformer_attention_attn_b200 as dit
    from diffusion_transformer_attention_attn_b200 import context_parallel as cp
    (q, k, v), (qd, kd, vd) = _case(8, 1024, d, seed=40 + world)
    Nl = qd.shape[2] // world
    sl = [slice(r * Nl, (r + 1) * Nl) for r in range(world)]
    outs = _run_ranks(world, lambda r, comm: cp.ulysses_attention(
        qd[:, :, sl[r]].contiguous(), kd[:, :, sl[r]].contiguous(), vd[:, :, sl[r]].contiguous(), comm=comm))
    o = torch.cat(outs, dim=2)
    assert torch.equal(o, dit.dit_attn_fwd(qd, kd, vd))
    rows = np.arange(0, 1024, 7)
    assert_bf16_parity(from_device_bf16(o[:, :, rows]), oracle.attention(q, k, v, rows=rows), f"ulysses P={world}")


@pytest.mark.parametrize("fused", [False, True], ids=["all-to-all", "scatter"])
@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("pv_mode", ["fp8", "bf16"])
def test_ulysses_q8_with_the_kernels(world, pv_mode, fused):
    import diffusion_transformer_attention_attn_b200 as dit
    from diffusion_transformer_attention_attn_b200 import context_parallel as cp
    (q, k, v), (qd, kd, vd) = _case(8, 1024, 128, seed=50 + world, k_offset_std=3.0, zero_q_channel=7)
    Nl = qd.shape[2] // world
    sl = [slice(r * Nl, (r + 1) * Nl) for r in range(world)]
    outs = _run_ranks(world, lambda r, comm: cp.ulysses_attention_q8(
        qd[:, :, sl[r]].contiguous(), kd[:, :, sl[r]].contiguous(), vd[:, :, sl[r]].contiguous(), smooth_k=True,
        pv_mode=pv_mode, comm=comm, fused=fused))
    o = torch.cat(outs, dim=2)
    assert torch.equal(o, dit.dit_attn_fwd_q8(qd, kd, vd, smooth_k=True, pv_mode=pv_mode))
    rows = np.arange(0, 1024, 7)
    out, ref = from_device_bf16(o[:, :, rows]), oracle.attention(q, k, v, rows=rows)
    c, r = cosine(out, ref), rel_l1(out, ref)
    assert c >= Q8_COSINE and r <= (FP8_REL_L1 if pv_mode == "fp8" else Q8_REL_L1), (c, r)


@pytest.mark.parametrize("world", [2, 4])
def test_ring_with_the_kernels(world):
    from diffusion_transformer_attention_attn_b200 import context_parallel as cp
    (q, k, v), (qd, kd, vd) = _case(4, 1000, 128, seed=60 + world)
    Nl = qd.shape[2] // world
    sl = [slice(r * Nl, (r + 1) * Nl) for r in range(world)]
    res = _run_ranks(world, lambda r, comm: cp.ring_attention(
        qd[:, :, sl[r]].contiguous(), kd[:, :, sl[r]].contiguous(), vd[:, :, sl[r]].contiguous(), comm=comm))
    o = torch.cat([x[0] for x in res], dim=2)
    lse = torch.cat([x[1] for x in res], dim=2)
    ref_o, ref_lse = oracle.attention_lse(q, k, v)
    assert_bf16_parity(from_device_bf16(o), ref_o, f"ring P={world}")
    assert np.abs(lse.cpu().numpy().astype(np.float64) - ref_lse).max() <= 1e-3


@pytest.mark.parametrize("world", [2, 4])
def test_sharded_fbc_with_the_kernels(world):
    from diffusion_transformer_attention_attn_b200 import context_parallel as cp
    cur, prev = inputs.fbc_inputs(inputs.FBC_IMAGE)
    cur, prev = cur.reshape(-1), prev.reshape(-1)
    dc, dp = (torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16) for x in (cur, prev))
    n = cur.size
    cuts = [n * r // world // 8 * 8 for r in range(world)] + [n]      # 16-byte aligned shard starts
    res = _run_ranks(world, lambda r, comm: cp.sharded_fbc_rel_l1(dc[cuts[r]:cuts[r + 1]], dp[cuts[r]:cuts[r + 1]],
                                                                  0.08, comm=comm))
    rel_ref, skip_ref = oracle.fbc_rel_l1(cur, prev, 0.08)
    for rel, skip in res:
        assert abs(rel.item() - rel_ref) <= FBC_REL_ERR * rel_ref and int(skip.item()) == skip_ref
