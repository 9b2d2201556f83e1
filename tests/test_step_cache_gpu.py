"""CachedStep: a captured denoising step whose skippable part runs only on the
steps the device-side policy computes.  A two-block toy transformer (random
weights, bf16) stands in for the model; the reference replays the same torch
operations eagerly with the oracle's decisions.
"""
import numpy as np
import pytest

import oracle
from oracle import cache_policy as cp
from diffusion_transformer_attention_attn_b200 import inputs

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


class Toy:
    """first block: h1 = x + relu(x W1); remaining blocks: out = h1 + h1 W2."""

    def __init__(self, T=512, C=256, seed=0):
        g = torch.Generator(device="cpu").manual_seed(seed)
        self.w1 = (torch.randn(C, C, generator=g) / C ** 0.5).to(torch.bfloat16).cuda()
        self.w2 = (torch.randn(C, C, generator=g) / C ** 0.5).to(torch.bfloat16).cuda()
        z = lambda: torch.zeros(T, C, dtype=torch.bfloat16, device="cuda")
        self.x, self.t1, self.h1, self.r, self.t2, self.out, self.res, self.y = (z() for _ in range(8))

    def head(self):
        torch.matmul(self.x, self.w1, out=self.t1)
        self.t1.relu_()
        torch.add(self.x, self.t1, out=self.h1)
        torch.sub(self.h1, self.x, out=self.r)

    def body(self):
        torch.matmul(self.h1, self.w2, out=self.t2)
        torch.add(self.h1, self.t2, out=self.out)
        torch.sub(self.out, self.h1, out=self.res)

    def tail(self):
        torch.add(self.h1, self.res, out=self.y)


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _inputs(steps, T=512, C=256):
    traj = inputs.trajectory(inputs.TrajectoryCase("toy", T, C, "bf16", steps, 0.01, 0.12, seed=3))
    return [torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16) for x in traj]


@pytest.mark.parametrize("mode", ["fbcache", "teacache"])
def test_cached_step_matches_eager_replay(mode):
    import diffusion_transformer_attention_attn_b200 as dit
    from diffusion_transformer_attention_attn_b200.step_cache import CachedStep
    steps = 20
    xs = _inputs(steps)
    toy = Toy()
    if mode == "fbcache":
        policy = dict(max_warmup_steps=2, max_continuous_cached_steps=3, residual_diff_threshold=0.2)
        step = CachedStep(toy.head, toy.body, toy.r, policy=dit.dit_cache_policy(**policy), tail_fn=toy.tail)
    else:
        coeffs, thr = [0.0, 1.5], 0.2
        step = CachedStep(toy.head, toy.body, toy.r, teacache=(coeffs, thr), tail_fn=toy.tail)
    outs, rs = [], []
    try:
        for x in xs:
            with torch.cuda.stream(step.stream):
                toy.x.copy_(x)
                step()
                outs.append(toy.y.clone())
                rs.append(toy.r.clone())
        torch.cuda.synchronize()
        dec = [int(d) for d in step.decisions()["decision"]]
        counters = step.counters()
    finally:
        step.close()
    # the oracle's decisions on the same residuals
    rel = lambda c, p: oracle.fbc_rel_l1(c, p, 0.0)[0]
    r_np = [_bits(r) for r in rs]
    if mode == "fbcache":
        _, dec_ref, _ = cp.fbcache_schedule(r_np, cp.CachePolicy(**policy), rel)
    else:
        _, _, _, dec_ref = cp.teacache_schedule(r_np, coeffs, thr, rel)
    assert dec == dec_ref
    assert counters["step"] == steps and counters["cached_steps"] == dec.count(cp.USE_CACHE)
    assert 0 < dec.count(cp.USE_CACHE) < steps
    # eager replay with those decisions: the cached residual refreshes on computed steps only
    ref = Toy()
    for x, d, y in zip(xs, dec_ref, outs):
        ref.x.copy_(x)
        ref.head()
        if d != cp.USE_CACHE:
            ref.body()
        ref.tail()
        torch.cuda.synchronize()
        assert torch.equal(ref.y, y)


def test_reset_starts_a_new_generation():
    import diffusion_transformer_attention_attn_b200 as dit
    from diffusion_transformer_attention_attn_b200.step_cache import CachedStep
    xs = _inputs(6)
    toy = Toy()
    step = CachedStep(toy.head, toy.body, toy.r, policy=dit.dit_cache_policy(max_warmup_steps=1), tail_fn=toy.tail)
    try:
        runs = []
        for _ in range(2):
            step.reset()
            for x in xs:
                with torch.cuda.stream(step.stream):
                    toy.x.copy_(x)
                    step()
            runs.append([int(d) for d in step.decisions()["decision"]])
        assert runs[0] == runs[1] and runs[0][0] == cp.WARMUP
    finally:
        step.close()


def test_needs_exactly_one_policy():
    import diffusion_transformer_attention_attn_b200 as dit
    from diffusion_transformer_attention_attn_b200.step_cache import CachedStep
    toy = Toy(T=16, C=32)
    with pytest.raises(ValueError):
        CachedStep(toy.head, toy.body, toy.r)
    with pytest.raises(ValueError):
        CachedStep(toy.head, toy.body, toy.r, policy=dit.dit_cache_policy(), teacache=([0.0, 1.0], 0.1))
