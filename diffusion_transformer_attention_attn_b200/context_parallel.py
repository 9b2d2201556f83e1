"""Context parallelism for the attention call: one process per GPU, the token
sequence split evenly across the ranks of a ``torch.distributed`` group.

Two attention schemes, both from "ParaAttention" (diffusers docs), section
"Context Parallelism", and the TMAP image-to-video blog, section on sequence
parallelism (Ulysses, with its all-to-all overlapped with the surrounding
work), and the cache decision over a sharded residual:

* ``ulysses_attention`` — each rank holds all heads of its N/P tokens.  One
  all-to-all regroups Q, K and V so that each rank holds H/P heads of all N
  tokens; attention runs locally per head (the DiT attention has no mask and
  heads are independent); a second all-to-all returns each rank's tokens.
* ``ring_attention`` — each rank keeps its queries and passes its K/V chunk
  around the ring; every step attends the local queries to the chunk in hand
  (``dit_attn_fwd_ex`` with log-sum-exp), while the next chunk is already in
  flight, and the per-chunk results are merged (``dit_attn_merge``).
* ``ulysses_attention_q8`` — Ulysses with the 8-bit attention, the all-to-all
  moving 1-byte codes: each rank reduces its tokens to per-channel K sums and
  V maxima (``dit_attn_q8_channel_stats``), two all-reduces combine them, each
  rank quantises its own tokens (``dit_attn_q8_quantize_global``), the codes
  and block scales travel to the head-sharded layout, and the attention runs
  on them (``dit_attn_fwd_q8_prequantized``).  With ``fused=True`` the
  quantisers store the codes straight into every rank's head-sharded
  workspace (``dit_attn_q8_quantize_scatter``, peer memory between GPUs), so
  the all-to-all of the codes is no separate step.
* ``sharded_fbc_rel_l1`` — the first-block-cache difference of a residual
  sharded like the sequence: each rank reduces its slice to two sums
  (``fbc_rel_l1_sums``), one all-reduce adds them, and ``fbc_rel_l1_finish``
  forms rel and the decision on every rank.

The collectives go through a communicator (``TorchComm``: torch.distributed
calls, NCCL between GPUs); the attention, the merge and the reductions are the
library's kernels.  ``attn_fn``, ``attn_lse_fn``, ``merge_fn``, ``stats_fn``,
``quant_fn``, ``codes_attn_fn``, ``sums_fn`` and ``finish_fn`` may be
replaced, e.g. to run the data movement on CPU ranks, and so may ``comm``,
any object with the methods of ``TorchComm`` (the fused 8-bit path also uses
``shared_workspace`` and ``barrier``).
"""
from __future__ import annotations


class TorchComm:
    """The four collective steps the context-parallel schemes take, over a
    torch.distributed process group (``group`` None: the default group)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self._shared = {}

    def all_to_all(self, recv, send):
        """Equal split along dim 0: recv[i] = rank i's send[this rank]."""
        import torch.distributed as dist
        dist.all_to_all_single(recv, send, group=self.group)

    def all_reduce(self, t, op: str = "sum"):
        """In place: the elementwise sum ("sum") or maximum ("max") over ranks."""
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.SUM if op == "sum" else dist.ReduceOp.MAX, group=self.group)

    def ring_exchange(self, send, recv):
        """Start sending ``send`` to rank+1 and receiving rank-1's into
        ``recv``; returns handles whose ``wait()`` completes the exchange."""
        import torch.distributed as dist
        nxt = (self.rank + 1) % self.world
        prv = (self.rank - 1) % self.world
        if self.group is not None:
            nxt = dist.get_global_rank(self.group, nxt)
            prv = dist.get_global_rank(self.group, prv)
        ops = [dist.P2POp(dist.isend, send, nxt, self.group), dist.P2POp(dist.irecv, recv, prv, self.group)]
        return dist.batch_isend_irecv(ops)

    def shared_workspace(self, nbytes: int, device):
        """A device buffer of ``nbytes`` on every rank, mapped into every
        rank's address space (torch symmetric memory over NVLink): returns
        (this rank's buffer, every rank's device address).  The buffer of a
        given size is made once and reused.  Not run on more than one GPU
        here."""
        import torch
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm
        key = (int(nbytes), str(device))
        if key not in self._shared:
            buf = symm.empty(nbytes, dtype=torch.uint8, device=device)
            handle = symm.rendezvous(buf, self.group if self.group is not None else dist.group.WORLD)
            self._shared[key] = (buf, [int(p) for p in handle.buffer_ptrs])
        return self._shared[key]

    def barrier(self):
        """Every rank's work issued so far on the current stream has completed."""
        import torch
        import torch.distributed as dist
        torch.cuda.current_stream().synchronize()
        dist.barrier(group=self.group)


def _comm(group, comm):
    return comm if comm is not None else TorchComm(group)


def _default_attn(q, k, v):
    from . import dit_attn_fwd
    return dit_attn_fwd(q, k, v)


def _default_attn_lse(q, k, v):
    from . import dit_attn_fwd_ex
    return dit_attn_fwd_ex(q, k, v, lse=True)


def _default_merge(outs, lses):
    from . import dit_attn_merge
    return dit_attn_merge(outs, lses, lse=True)


def seq_to_heads(xs, world: int, group=None, comm=None):
    """All-to-all of sequence-sharded tensors to head-sharded ones.

    xs: list of [B, H, Nl, d] tensors (this rank's Nl = N/P tokens, all heads),
    H divisible by the group size P.  Returns [B, H/P, P*Nl, d] tensors: head
    group r of this rank r, tokens in global order (rank-major).  All tensors
    travel in one all-to-all.
    """
    import torch
    B, H, Nl, d = xs[0].shape
    P = world
    hp = H // P
    # [P (destination head group), T, B, H/P, Nl, d]
    send = torch.stack([x.reshape(B, P, hp, Nl, d) for x in xs], dim=0).permute(2, 0, 1, 3, 4, 5).contiguous()
    recv = torch.empty_like(send)
    _comm(group, comm).all_to_all(recv, send)
    # recv[src] = src's tokens of my heads -> [T, B, H/P, P*Nl, d]
    out = recv.permute(1, 2, 3, 0, 4, 5).reshape(len(xs), B, hp, P * Nl, d)
    return [out[i] for i in range(len(xs))]


def heads_to_seq(y, world: int, group=None, comm=None):
    """Inverse of ``seq_to_heads`` for one tensor: [B, H/P, P*Nl, d] ->
    [B, H, Nl, d] (this rank's tokens, all heads, head groups rank-major)."""
    import torch
    B, hp, N, d = y.shape
    P = world
    Nl = N // P
    send = y.reshape(B, hp, P, Nl, d).permute(2, 0, 1, 3, 4).contiguous()   # [P (token owner), B, H/P, Nl, d]
    recv = torch.empty_like(send)
    _comm(group, comm).all_to_all(recv, send)
    return recv.permute(1, 0, 2, 3, 4).reshape(B, P * hp, Nl, d)


def ulysses_attention(q, k, v, group=None, attn_fn=None, comm=None):
    """Attention over the full sequence from sequence-sharded [B, H, N/P, d]
    q, k, v; returns this rank's [B, H, N/P, d] output."""
    comm = _comm(group, comm)
    world = comm.world
    B, H, Nl, d = q.shape
    if H % world:
        raise ValueError(f"{H} heads do not split over {world} ranks")
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share their shape")
    attn = attn_fn or _default_attn
    if world == 1:
        return attn(q, k, v)
    qh, kh, vh = seq_to_heads([q, k, v], world, comm=comm)
    return heads_to_seq(attn(qh, kh, vh), world, comm=comm)


def ring_attention(q, k, v, group=None, attn_lse_fn=None, merge_fn=None, comm=None):
    """Attention of this rank's queries [B, H, Nl, d] to all ranks' keys, the
    K/V chunks travelling around the ring (rank r sends to r+1 and receives
    from r-1).  Returns (o, lse) for the local queries."""
    import torch
    comm = _comm(group, comm)
    world = comm.world
    attn = attn_lse_fn or _default_attn_lse
    merge = merge_fn or _default_merge
    kv = torch.stack([k, v], dim=0).contiguous()
    outs, lses = [], []
    for step in range(world):
        reqs = []
        if step + 1 < world:
            buf = torch.empty_like(kv)
            reqs = comm.ring_exchange(kv, buf)
        o_c, l_c = attn(q, kv[0], kv[1])
        outs.append(o_c)
        lses.append(l_c)
        for r in reqs:
            r.wait()
        if step + 1 < world:
            kv = buf
        # Merge as the parts arrive once the merge kernel's fan-in is reached.
        if len(outs) == 16:
            o_m, l_m = merge(outs, lses)
            outs, lses = [o_m], [l_m]
    if len(outs) == 1:
        return outs[0], lses[0]
    return merge(outs, lses)


def _default_sums(cur, prev):
    from . import fbc_rel_l1_sums
    return fbc_rel_l1_sums(cur, prev)


def _default_finish(sums, threshold):
    from . import fbc_rel_l1_finish
    return fbc_rel_l1_finish(sums, threshold)


def sharded_fbc_rel_l1(r_cur, r_prev, threshold: float, group=None, sums_fn=None, finish_fn=None, comm=None):
    """(rel, skip) of a residual whose elements are split across the ranks of
    ``group``; every rank gets the same result."""
    sums = (sums_fn or _default_sums)(r_cur, r_prev)
    comm = _comm(group, comm)
    if comm.world > 1:
        comm.all_reduce(sums, "sum")
    return (finish_fn or _default_finish)(sums, threshold)


# ---- Ulysses with 8-bit transport --------------------------------------------

CODE_KEYS = ("q_codes", "k_codes", "v_codes")


def _default_stats(k, v, smooth_k, pv_mode):
    from . import dit_attn_q8_channel_stats
    return dit_attn_q8_channel_stats(k, v, smooth_k=smooth_k, pv_mode=pv_mode)


def _default_quant(q, k, v, k_sum, v_amax, n_total, smooth_k, pv_mode):
    from . import dit_attn_q8_quantize_global, q8_views
    B, H, N, d = q.shape
    ws = dit_attn_q8_quantize_global(q, k, v, k_sum, v_amax, n_total, smooth_k=smooth_k, pv_mode=pv_mode)
    return q8_views(ws, B, H, N, d, pv_mode)


def _default_codes_attn(parts, v, pv_mode):
    """parts: head-sharded codes and scales (q8_views names)."""
    from . import dit_attn_fwd_q8_prequantized, q8_views, q8_workspace
    B, H, N, d = parts["q_codes"].shape
    ws = q8_workspace(B, H, N, d, pv_mode, parts["q_codes"].device)
    dst = q8_views(ws, B, H, N, d, pv_mode)
    for name, t in parts.items():
        dst[name].copy_(t)
    return dit_attn_fwd_q8_prequantized(ws, B, H, N, v=v, pv_mode=pv_mode, d=d)


def ulysses_attention_q8(q, k, v, group=None, smooth_k: bool = True, pv_mode="fp8", stats_fn=None, quant_fn=None,
                         codes_attn_fn=None, comm=None, fused: bool = False):
    """8-bit attention over the full sequence from sequence-sharded
    [B, H, N/P, d] q, k, v, with the all-to-all carrying the 8-bit codes
    (bf16 V instead in bf16-PV mode).  N/P must be a multiple of 128 (whole
    Q blocks per rank).  With ``fused`` the quantisers scatter the codes into
    every rank's workspace directly (the communicator supplies the shared
    workspaces).  Returns this rank's [B, H, N/P, d] output."""
    import torch
    comm = _comm(group, comm)
    world, rank = comm.world, comm.rank
    if fused and world > 1:
        return _ulysses_q8_fused(q, k, v, comm, smooth_k, pv_mode, stats_fn)
    B, H, Nl, d = q.shape
    if H % world:
        raise ValueError(f"{H} heads do not split over {world} ranks")
    if Nl % 128:
        raise ValueError("each rank must hold whole 128-token blocks")
    fp8 = pv_mode in ("fp8", 0)
    k_sum, v_amax = (stats_fn or _default_stats)(k, v, smooth_k, pv_mode)
    if world > 1:
        comm.all_reduce(k_sum, "sum")
        comm.all_reduce(v_amax, "max")
    local = (quant_fn or _default_quant)(q, k, v, k_sum, v_amax, Nl * world, smooth_k, pv_mode)
    hp = H // world
    names = [n for n in CODE_KEYS if n in local]
    parts = {}
    if world > 1:
        # 1-byte codes travel as 32-bit words (d is a multiple of 4).
        moved = seq_to_heads([local[n].contiguous().view(torch.int32) for n in names], world, comm=comm)
        for n, t in zip(names, moved):
            parts[n] = t.contiguous().view(local[n].dtype)
        for n in ("q_scale", "k_scale"):
            parts[n] = seq_to_heads([local[n].unsqueeze(-1)], world, comm=comm)[0].squeeze(-1).contiguous()
        vh = None if fp8 else seq_to_heads([v], world, comm=comm)[0].contiguous()
    else:
        parts = {n: local[n] for n in names + ["q_scale", "k_scale"]}
        vh = None if fp8 else v
    if fp8:
        parts["v_scale"] = local["v_scale"][:, rank * hp:(rank + 1) * hp].contiguous()
    oh = (codes_attn_fn or _default_codes_attn)(parts, vh, pv_mode)
    return oh if world == 1 else heads_to_seq(oh, world, comm=comm)


def _ulysses_q8_fused(q, k, v, comm, smooth_k, pv_mode, stats_fn):
    """``ulysses_attention_q8`` with the code all-to-all fused into the
    quantisers (dit_attn_q8_quantize_scatter)."""
    from . import dit_attn_fwd_q8_prequantized, dit_attn_q8_quantize_scatter, dit_attn_q8_workspace_bytes
    world, rank = comm.world, comm.rank
    B, H, Nl, d = q.shape
    if H % world:
        raise ValueError(f"{H} heads do not split over {world} ranks")
    if Nl % 128:
        raise ValueError("each rank must hold whole 128-token blocks")
    fp8 = pv_mode in ("fp8", 0)
    hp, N = H // world, Nl * world
    k_sum, v_amax = (stats_fn or _default_stats)(k, v, smooth_k, pv_mode)
    comm.all_reduce(k_sum, "sum")
    comm.all_reduce(v_amax, "max")
    nbytes = dit_attn_q8_workspace_bytes(B, hp, N, d, pv_mode)
    ws_dst, ptrs = comm.shared_workspace(nbytes, q.device)
    dit_attn_q8_quantize_scatter(q, k, v, k_sum, v_amax, rank, world, ptrs, nbytes, smooth_k=smooth_k,
                                 pv_mode=pv_mode)
    vh = None if fp8 else seq_to_heads([v], world, comm=comm)[0].contiguous()
    comm.barrier()          # every rank's codes have landed in every workspace
    oh = dit_attn_fwd_q8_prequantized(ws_dst, B, hp, N, v=vh, pv_mode=pv_mode, d=d)
    out = heads_to_seq(oh, world, comm=comm)
    comm.barrier()          # no rank reuses its workspace before the others finished reading theirs
    return out
