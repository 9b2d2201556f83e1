"""Parity of the device-side step caches (through the C ABI) with the oracle's
policies, and of the CUDA-graph conditional that they drive.

Bar: identical decisions at every step, relative error of every evaluated
difference <= 1e-5, identical counters; in a captured graph the skippable
body runs exactly on the steps the oracle computes.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import cache_policy as cp
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


def _dit():
    import diffusion_transformer_attention_attn_b200 as dit
    return dit


def _dev(x):
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _rel(c, p):
    return oracle.fbc_rel_l1(c, p, 0.0)[0]


def _check_rels(got, ref):
    for g, r in zip(got, ref):
        if math.isnan(r):
            assert math.isnan(g)
        elif math.isinf(r) or r == 0.0:
            assert g == r
        else:
            assert abs(g - r) <= FBC_REL_ERR * abs(r), (g, r)


def _margin_ok(rels, thr):
    """No evaluated difference within 1e-4 (relative) of the threshold, so both
    sides must take the same decision."""
    t = float(np.float32(thr))
    return all(math.isnan(r) or abs(r - t) > 1e-4 * t for r in rels)


def _policy_pair(**kw):
    dit = _dit()
    return cp.CachePolicy(**kw), dit.dit_cache_policy(**kw)


def _run_fbcache_eager(traj, pol):
    """Steps through the C ABI; the caller refreshes r_prev on computed steps
    with a device-side select (no host synchronisation per step)."""
    dit = _dit()
    cur = [_dev(x) for x in traj]
    prev = torch.zeros_like(cur[0])
    state, trace = dit.cache_state(), dit.cache_trace(len(traj))
    ws = dit.cache_workspace(cur[0].numel())
    dec = state[16:20].view(torch.int32)
    for c in cur:
        dit.fbcache_step(c, prev, pol, state, trace, workspace=ws)
        prev.copy_(torch.where(dec != 0, c, prev))
    torch.cuda.synchronize()
    return dit.read_cache_trace(trace, len(traj)), dit.read_cache_state(state)


POLICIES = [
    dict(),                                                     # the table's defaults
    dict(max_warmup_steps=2, residual_diff_threshold=0.2),
    dict(max_warmup_steps=0, max_cached_steps=5, max_continuous_cached_steps=-1, residual_diff_threshold=0.3),
    dict(max_warmup_steps=1, max_cached_steps=-1, max_continuous_cached_steps=1, residual_diff_threshold=0.12),
]


@pytest.mark.parametrize("case", [inputs.TRAJ_IMAGE, inputs.TRAJ_RAGGED], ids=lambda c: c.name)
@pytest.mark.parametrize("kw", POLICIES)
def test_fbcache_eager_matches_oracle(case, kw):
    traj = inputs.trajectory(case)
    p_ref, p_dev = _policy_pair(**kw)
    rels, dec, (steps, cached, cont, has_prev) = cp.fbcache_schedule(traj, p_ref, _rel)
    assert _margin_ok(rels, p_ref.residual_diff_threshold)
    tr, st = _run_fbcache_eager(traj, p_dev)
    assert list(tr["decision"]) == dec
    _check_rels(list(tr["rel"]), rels)
    assert (st["step"], st["cached_steps"], st["continuous_cached"], st["has_prev"]) == \
        (steps, cached, cont, int(has_prev))
    assert st["last_decision"] == dec[-1]


def test_fbcache_zero_and_identical_residuals():
    # identical residuals: rel 0 (cached); an all-zero stored residual with a
    # non-zero current one: rel +inf (computed)
    dit = _dit()
    p_ref, p_dev = _policy_pair(max_warmup_steps=1, max_continuous_cached_steps=-1)
    z = np.zeros((16, 8), np.float32)
    o = np.ones((16, 8), np.float32)
    traj = [z, z, o, o, o]
    rels, dec, _ = cp.fbcache_schedule(traj, p_ref, _rel)
    assert dec == [cp.WARMUP, cp.USE_CACHE, cp.ABOVE_THRESHOLD, cp.USE_CACHE, cp.USE_CACHE]
    assert rels[1] == 0.0 and rels[2] == math.inf
    tr, _ = _run_fbcache_eager(traj, p_dev)
    assert list(tr["decision"]) == dec
    _check_rels(list(tr["rel"]), rels)


def test_fbcache_trace_capacity_and_reset():
    dit = _dit()
    traj = inputs.trajectory(inputs.TRAJ_RAGGED)[:10]
    p_ref, p_dev = _policy_pair(max_warmup_steps=1)
    _, dec, _ = cp.fbcache_schedule(traj, p_ref, _rel)
    cur = [_dev(x) for x in traj]
    prev = torch.zeros_like(cur[0])
    state, trace = dit.cache_state(), dit.cache_trace(4)
    sentinel = dit.cache_trace(1)
    ws = dit.cache_workspace(cur[0].numel())
    dec_d = state[16:20].view(torch.int32)
    for run in range(2):
        dit.dit_cache_state_reset(state)
        prev.zero_()
        for c in cur:
            dit.fbcache_step(c, prev, p_dev, state, trace, workspace=ws)
            prev.copy_(torch.where(dec_d != 0, c, prev))
        torch.cuda.synchronize()
        assert list(dit.read_cache_trace(trace, 4)["decision"]) == dec[:4]
        assert dit.read_cache_state(state)["step"] == 10
    assert bytes(sentinel.cpu().numpy()) == bytes(24)


@pytest.mark.parametrize("case", [inputs.TRAJ_IMAGE, inputs.TRAJ_RAGGED], ids=lambda c: c.name)
@pytest.mark.parametrize("coeffs,thr", [([0.0, 1.0], 0.3), ([0.01, 0.5, 4.0], 0.25), ([0.05], 0.12)])
def test_teacache_eager_matches_oracle(case, coeffs, thr):
    dit = _dit()
    traj = inputs.trajectory(case)
    rels, resc, accs, dec = cp.teacache_schedule(traj, coeffs, thr, _rel)
    t32 = float(np.float32(thr))
    assert all(math.isnan(a) or a == 0.0 or abs(a - t32) > 1e-4 * t32 for a in accs)
    cur = [_dev(x) for x in traj]
    prev = torch.zeros_like(cur[0])
    state, trace = dit.cache_state(), dit.cache_trace(len(traj))
    ws = dit.cache_workspace(cur[0].numel())
    for c in cur:
        dit.teacache_step(c, prev, coeffs, thr, state, trace, workspace=ws)
    torch.cuda.synchronize()
    tr = dit.read_cache_trace(trace, len(traj))
    assert list(tr["decision"]) == dec
    _check_rels(list(tr["rel"]), rels)
    for g, r in zip(tr["acc"], accs):
        assert abs(g - r) <= 1e-5 * max(abs(r), 1e-3), (g, r)
    # the stored input is the last step's, bit for bit
    assert torch.equal(prev.view(torch.int16 if prev.dtype == torch.bfloat16 else torch.int32),
                       cur[-1].view(torch.int16 if prev.dtype == torch.bfloat16 else torch.int32))
    st = dit.read_cache_state(state)
    assert st["step"] == len(traj) and st["cached_steps"] == dec.count(cp.USE_CACHE)


def _capture_step_graph(s, body, step_fn, body_fn):
    """Capture [step_fn] -> IF(decision computes) { body_fn } on stream s."""
    dit = _dit()
    dit.dit_graph_capture_begin(s)
    body_open = False
    try:
        h = dit.dit_graph_cond_create(s)
        step_fn(h)
        dit.dit_graph_cond_body_begin(s, h, body)
        body_open = True
        with torch.cuda.stream(body):
            body_fn()
    finally:
        if body_open:
            dit.dit_graph_cond_body_end(body)
        exe = dit.dit_graph_capture_end(s)
    return exe


def test_fbcache_graph_conditional_runs_body_on_computed_steps():
    dit = _dit()
    case = inputs.TRAJ_IMAGE
    traj = inputs.trajectory(case)
    p_ref, p_dev = _policy_pair(max_warmup_steps=2, residual_diff_threshold=0.2)
    rels, dec, _ = cp.fbcache_schedule(traj, p_ref, _rel)
    assert _margin_ok(rels, 0.2)
    steps = [_dev(x) for x in traj]
    cur = torch.empty_like(steps[0])
    prev = torch.zeros_like(steps[0])
    state, trace = dit.cache_state(), dit.cache_trace(len(traj))
    ws = dit.cache_workspace(cur.numel())
    counter = torch.zeros(1, dtype=torch.int32, device="cuda")
    # the skippable work: an attention call on fixed inputs
    q, k, v = (_dev(x) for x in inputs.attn_inputs(inputs.TINY))
    o = torch.zeros_like(q)
    o_ref = dit.dit_attn_fwd(q, k, v)
    torch.cuda.synchronize()
    s, body = torch.cuda.Stream(), torch.cuda.Stream()

    def body_fn():
        prev.copy_(cur)
        counter.add_(1)
        dit.dit_attn_fwd(q, k, v, o, stream=body)

    exe = _capture_step_graph(
        s, body, lambda h: dit.fbcache_step(cur, prev, p_dev, state, trace, cond_handle=h, workspace=ws, stream=s),
        body_fn)
    try:
        with torch.cuda.stream(s):
            for x in steps:
                cur.copy_(x)
                dit.dit_graph_launch(exe, s)
        s.synchronize()
    finally:
        dit.dit_graph_destroy(exe)
    tr = dit.read_cache_trace(trace, len(traj))
    assert list(tr["decision"]) == dec
    _check_rels(list(tr["rel"]), rels)
    n_compute = sum(1 for d in dec if d != cp.USE_CACHE)
    assert int(counter.item()) == n_compute
    assert torch.equal(o, o_ref)
    # the stored residual is the last computed step's
    last = max(i for i, d in enumerate(dec) if d != cp.USE_CACHE)
    assert torch.equal(prev.view(torch.int16), steps[last].view(torch.int16))


def test_teacache_graph_conditional():
    dit = _dit()
    traj = inputs.trajectory(inputs.TRAJ_RAGGED)
    coeffs, thr = [0.0, 1.0], 0.3
    _, _, _, dec = cp.teacache_schedule(traj, coeffs, thr, _rel)
    steps = [_dev(x) for x in traj]
    cur = torch.empty_like(steps[0])
    prev = torch.zeros_like(steps[0])
    state, trace = dit.cache_state(), dit.cache_trace(len(traj))
    ws = dit.cache_workspace(cur.numel())
    counter = torch.zeros(1, dtype=torch.int32, device="cuda")
    s, body = torch.cuda.Stream(), torch.cuda.Stream()
    exe = _capture_step_graph(
        s, body,
        lambda h: dit.teacache_step(cur, prev, coeffs, thr, state, trace, cond_handle=h, workspace=ws, stream=s),
        lambda: counter.add_(1))
    try:
        with torch.cuda.stream(s):
            for x in steps:
                cur.copy_(x)
                dit.dit_graph_launch(exe, s)
        s.synchronize()
    finally:
        dit.dit_graph_destroy(exe)
    assert list(dit.read_cache_trace(trace, len(traj))["decision"]) == dec
    assert int(counter.item()) == sum(1 for d in dec if d != cp.USE_CACHE)


def test_conditional_handle_of_another_capture_is_refused():
    dit = _dit()
    x = torch.zeros(64, dtype=torch.float32, device="cuda")
    y = torch.zeros_like(x)
    state = dit.cache_state()
    ws = dit.cache_workspace(64)
    s1, s2, body = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    handles = {}

    def step_fn(h):
        handles["h1"] = h
        # the same handle, offered to a step on another capturing stream
        dit.dit_graph_capture_begin(s2)
        try:
            with pytest.raises(dit.DitError) as e:
                dit.fbcache_step(x, y, dit.dit_cache_policy(), state, cond_handle=h, workspace=ws, stream=s2)
            assert e.value.status == dit.DIT_ERR_INVALID_ARG
        finally:
            handles["g2"] = dit.dit_graph_capture_end(s2)
        dit.fbcache_step(x, y, dit.dit_cache_policy(), state, cond_handle=h, workspace=ws, stream=s1)

    g1 = _capture_step_graph(s1, body, step_fn, lambda: y.add_(1.0))
    for g in (g1, handles["g2"]):
        dit.dit_graph_destroy(g)
    # after its capture ended, the handle is refused outside any capture too
    with pytest.raises(dit.DitError):
        dit.fbcache_step(x, y, dit.dit_cache_policy(), state, cond_handle=handles["h1"], workspace=ws)
    torch.cuda.synchronize()
