"""The data movement of the context-parallel attention on CPU ranks (gloo).

Each rank holds N/P tokens of Q, K and V.  With the oracle's fp64 attention
standing in for the kernel (injected through the attn_fn / attn_lse_fn /
merge_fn arguments), Ulysses must reproduce the full-sequence attention
exactly (every head sees the same keys in the same order) and the ring must
match it to fp64 rounding (chunks merged through their log-sum-exps).
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _global_inputs(B, H, N, d, seed=0):
    from diffusion_transformer_attention_attn_b200 import inputs
    return inputs.attn_inputs(inputs.AttnCase("cp", B, H, N, d, seed=seed))


def _fbc_worker(rank, world, port, results):
    import torch.distributed as dist

    import oracle
    from diffusion_transformer_attention_attn_b200 import context_parallel as cp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(5)
        prev = rng.standard_normal(10000).astype(np.float32)
        cur = (prev + 0.07 * rng.standard_normal(prev.size)).astype(np.float32)
        cuts = np.linspace(0, prev.size, world + 1).astype(int)
        a, b = cuts[rank], cuts[rank + 1]

        def sums(c, p):
            return torch.tensor(oracle.fbc_sums(c.numpy(), p.numpy()), dtype=torch.float64)

        def finish(s, thr):
            return oracle.rel_from_sums(float(s[0]), float(s[1]), thr)
        results[rank] = cp.sharded_fbc_rel_l1(torch.from_numpy(cur[a:b]), torch.from_numpy(prev[a:b]), 0.08,
                                              sums_fn=sums, finish_fn=finish)
    finally:
        dist.destroy_process_group()


def test_sharded_fbc_gives_every_rank_the_whole_residuals_decision():
    import oracle
    import torch.multiprocessing as mp
    world = 3
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_fbc_worker, args=(world, port, results), nprocs=world, join=True, start_method="spawn")
        res = dict(results)
    rng = np.random.default_rng(5)
    prev = rng.standard_normal(10000).astype(np.float32)
    cur = (prev + 0.07 * rng.standard_normal(prev.size)).astype(np.float32)
    rel_ref, skip_ref = oracle.fbc_rel_l1(cur, prev, 0.08)
    for r in range(world):
        rel, skip = res[r]
        assert abs(rel - rel_ref) <= 1e-12 * rel_ref and skip == skip_ref


def _worker(rank, world, port, scheme, shape, results):
    import torch.distributed as dist

    import oracle
    from diffusion_transformer_attention_attn_b200 import context_parallel as cp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, N, d = shape
        q, k, v = _global_inputs(B, H, N, d)
        Nl = N // world
        sl = slice(rank * Nl, (rank + 1) * Nl)
        # bf16 values travel widened to fp32 (exact); gloo has no 16-bit all-to-all
        from diffusion_transformer_attention_attn_b200 import inputs
        tq, tk, tv = (torch.from_numpy(inputs.bf16_to_f32(np.ascontiguousarray(x[:, :, sl]))) for x in (q, k, v))

        def bits(t):
            return inputs.bf16_bits(t.contiguous().numpy())

        if scheme == "ulysses":
            def attn(a, b, c):
                return torch.from_numpy(oracle.attention(bits(a), bits(b), bits(c)))
            out = cp.ulysses_attention(tq, tk, tv, attn_fn=attn)
            results[rank] = out.numpy()
        else:
            def attn_lse(a, b, c):
                o, l = oracle.attention_lse(bits(a), bits(b), bits(c))
                return torch.from_numpy(o), torch.from_numpy(l)

            def merge(outs, lses):
                o, l = oracle.merge_partials([x.numpy() for x in outs], [x.numpy() for x in lses])
                return torch.from_numpy(o), torch.from_numpy(l)
            o, l = cp.ring_attention(tq, tk, tv, attn_lse_fn=attn_lse, merge_fn=merge)
            results[rank] = (o.numpy(), l.numpy())
    finally:
        dist.destroy_process_group()


def _run(scheme, world, shape):
    import torch.multiprocessing as mp
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_worker, args=(world, port, scheme, shape, results), nprocs=world, join=True,
                           start_method="spawn")
        return dict(results)


@pytest.mark.parametrize("world,shape", [(2, (1, 4, 96, 16)), (4, (2, 8, 64, 32))])
def test_ulysses_matches_full_attention_exactly(world, shape):
    import oracle
    B, H, N, d = shape
    q, k, v = _global_inputs(B, H, N, d)
    ref = oracle.attention(q, k, v)
    res = _run("ulysses", world, shape)
    got = np.concatenate([res[r] for r in range(world)], axis=2)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("world,shape", [(2, (1, 2, 96, 16)), (4, (1, 3, 128, 8))])
def test_ring_matches_full_attention(world, shape):
    import oracle
    B, H, N, d = shape
    q, k, v = _global_inputs(B, H, N, d)
    ref, ref_lse = oracle.attention_lse(q, k, v)
    res = _run("ring", world, shape)
    got = np.concatenate([res[r][0] for r in range(world)], axis=2)
    lse = np.concatenate([res[r][1] for r in range(world)], axis=2)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_world_of_one_runs_locally():
    from diffusion_transformer_attention_attn_b200 import context_parallel as cp
    import torch.distributed as dist
    if dist.is_initialized():
        pytest.skip("a process group is already initialised")
    store = dist.HashStore()
    dist.init_process_group("gloo", store=store, rank=0, world_size=1)
    try:
        x = torch.zeros(1, 3, 4, 8)
        # world 1: the attention runs locally, no collective
        out = cp.ulysses_attention(x, x, x, attn_fn=lambda a, b, c: a + 1)
        assert torch.equal(out, x + 1)
    finally:
        dist.destroy_process_group()


def _q8_worker(rank, world, port, shape, pv_mode, smooth_k, results):
    import torch.distributed as dist

    import oracle
    from diffusion_transformer_attention_attn_b200 import context_parallel as cp
    from diffusion_transformer_attention_attn_b200 import inputs

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, N, d = shape
        q, k, v = inputs.attn_inputs(inputs.AttnCase("cpq8", B, H, N, d, k_offset_std=3.0))
        Nl = N // world
        sl = slice(rank * Nl, (rank + 1) * Nl)
        tq, tk, tv = (torch.from_numpy(inputs.bf16_to_f32(np.ascontiguousarray(x[:, :, sl]))) for x in (q, k, v))

        def bits(t):
            return inputs.bf16_bits(t.contiguous().numpy())

        def stats(k_, v_, smooth, mode):
            ks = oracle.k_channel_sums(bits(k_)) if smooth else np.zeros(k_.shape[:2] + (d,))
            va = oracle.channel_amax(bits(v_)) if mode == "fp8" else np.zeros(v_.shape[:2] + (d,), np.float32)
            return torch.from_numpy(ks), torch.from_numpy(va)

        def quant(q_, k_, v_, k_sum, v_amax, n_total, smooth, mode):
            qc, qs = oracle.quant_int8_blocks(bits(q_), 128)
            mean = oracle.mean_from_sums(k_sum.numpy(), n_total) if smooth else None
            kc, ks = oracle.quant_int8_blocks(bits(k_), 64, mean)
            out = {"q_codes": qc, "q_scale": qs, "k_codes": kc, "k_scale": ks}
            if mode == "fp8":
                out["v_codes"], out["v_scale"] = oracle.quant_e4m3_with_amax(bits(v_), v_amax.numpy())
            return {n: torch.from_numpy(np.ascontiguousarray(a)) for n, a in out.items()}

        def codes_attn(parts, vh, mode):
            p = {n: t.numpy() for n, t in parts.items()}
            if mode == "fp8":
                o = oracle.attention_from_codes(p["q_codes"], p["q_scale"], p["k_codes"], p["k_scale"],
                                                p["v_codes"], p["v_scale"])
            else:
                o = oracle.attention_from_codes(p["q_codes"], p["q_scale"], p["k_codes"], p["k_scale"], bits(vh))
            return torch.from_numpy(o)
        out = cp.ulysses_attention_q8(tq, tk, tv, smooth_k=smooth_k, pv_mode=pv_mode, stats_fn=stats, quant_fn=quant,
                                      codes_attn_fn=codes_attn)
        results[rank] = out.numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,pv_mode,smooth_k", [(2, "fp8", True), (4, "fp8", False), (2, "bf16", True)])
def test_ulysses_q8_moves_codes_and_matches_the_single_device_codes(world, pv_mode, smooth_k):
    import oracle
    import torch.multiprocessing as mp
    from diffusion_transformer_attention_attn_b200 import inputs
    shape = (1, 4, 1024, 128)
    B, H, N, d = shape
    q, k, v = inputs.attn_inputs(inputs.AttnCase("cpq8", B, H, N, d, k_offset_std=3.0))
    qc, qs = oracle.quant_int8_blocks(q, 128)
    kc, ks = oracle.quant_int8_blocks(k, 64, oracle.channel_mean(k) if smooth_k else None)
    if pv_mode == "fp8":
        vc, vs = oracle.quant_e4m3_channels(v)
        ref = oracle.attention_from_codes(qc, qs, kc, ks, vc, vs)
    else:
        ref = oracle.attention_from_codes(qc, qs, kc, ks, v)
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_q8_worker, args=(world, port, shape, pv_mode, smooth_k, results), nprocs=world,
                           join=True, start_method="spawn")
        res = dict(results)
    got = np.concatenate([res[r] for r in range(world)], axis=2)
    assert np.array_equal(got, ref)
