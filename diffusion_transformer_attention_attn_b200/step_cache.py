"""A denoising step captured once as a CUDA graph whose expensive part runs
only on the steps the device-side cache policy decides to compute.

This is the library-level counterpart of applying a step cache to a
diffusion pipeline ("ParaAttention" (diffusers docs), "First Block Cache";
vLLM-Omni cache-dit guide, "DBCache"; TMAP image-to-video blog, "TeaCache"):
the caller splits one step of its transformer into

* ``head_fn()`` — the part that always runs (the first Fn blocks, or the
  timestep-modulated input for TeaCache); it leaves the signal the policy
  compares in ``signal``;
* ``body_fn()`` — the part that is skipped when the cache is reused (the
  remaining blocks, and the refresh of whatever the cache holds);
* ``tail_fn()`` (optional) — the part after the decision that always runs
  (e.g. the trailing Bn blocks, or adding the cached residual).

Each function only enqueues work on the current CUDA stream, on tensors that
live as long as the step (graph capture records their addresses), and must
not allocate: use preallocated tensors and ``out=`` forms.  Each runs once
eagerly before the capture.  The decision is taken on the device
(``fbcache_step`` / ``teacache_step``) and sets the graph's conditional node,
so replaying the step never synchronises with the host.  With ``policy=`` the first-block cache stores the signal of the
last computed step (the copy runs inside the skippable part); with
``teacache=`` the stored input is refreshed on every step by the decision
kernel itself.
"""
from __future__ import annotations

from . import (cache_state, cache_trace, cache_workspace, dit_cache_policy, dit_cache_state_reset,
               dit_graph_capture_begin, dit_graph_capture_end, dit_graph_cond_body_begin, dit_graph_cond_body_end,
               dit_graph_cond_create, dit_graph_destroy, dit_graph_launch, fbcache_step, read_cache_state,
               read_cache_trace, teacache_step)


class CachedStep:
    """One captured denoising step with a device-side cache decision.

    signal: CUDA tensor (fp32 or bf16, contiguous) that ``head_fn`` writes.
    policy: a ``dit_cache_policy`` (first-block cache), or
    teacache: ``(coeffs, threshold)`` for the TeaCache accumulator.
    trace_capacity: steps whose (difference, sum, decision) are recorded.
    """

    def __init__(self, head_fn, body_fn, signal, policy: dit_cache_policy | None = None, teacache=None,
                 tail_fn=None, trace_capacity: int = 256):
        import torch
        if (policy is None) == (teacache is None):
            raise ValueError("give exactly one of policy= (first-block cache) or teacache=(coeffs, threshold)")
        if not signal.is_cuda or not signal.is_contiguous():
            raise ValueError("signal must be a contiguous CUDA tensor")
        self.signal = signal
        self.stored = torch.zeros_like(signal)
        self.state = cache_state(signal.device)
        self.trace = cache_trace(trace_capacity, signal.device)
        self.trace_capacity = trace_capacity
        self._ws = cache_workspace(signal.numel(), signal.device)
        self.stream = torch.cuda.Stream(signal.device)
        self._body_stream = torch.cuda.Stream(signal.device)
        self._exe = None
        # One eager run of each part on the streams it will be captured on, so
        # that lazy set-up (library handles, their workspaces) happens outside
        # the capture.
        torch.cuda.synchronize(signal.device)
        with torch.cuda.stream(self.stream):
            head_fn()
        with torch.cuda.stream(self._body_stream):
            body_fn()
        if tail_fn is not None:
            with torch.cuda.stream(self.stream):
                tail_fn()
        torch.cuda.synchronize(signal.device)
        dit_graph_capture_begin(self.stream)
        body_open = False
        try:
            with torch.cuda.stream(self.stream):
                head_fn()
                h = dit_graph_cond_create(self.stream)
                if policy is not None:
                    fbcache_step(self.signal, self.stored, policy, self.state, self.trace, cond_handle=h,
                                 workspace=self._ws, stream=self.stream)
                else:
                    coeffs, threshold = teacache
                    teacache_step(self.signal, self.stored, coeffs, threshold, self.state, self.trace,
                                  cond_handle=h, workspace=self._ws, stream=self.stream)
                dit_graph_cond_body_begin(self.stream, h, self._body_stream)
                body_open = True
                with torch.cuda.stream(self._body_stream):
                    body_fn()
                    if policy is not None:
                        # the first-block cache compares with the last computed step
                        self.stored.copy_(self.signal)
                dit_graph_cond_body_end(self._body_stream)
                body_open = False
                if tail_fn is not None:
                    tail_fn()
        finally:
            if body_open:
                dit_graph_cond_body_end(self._body_stream)
            self._exe = dit_graph_capture_end(self.stream)

    def __call__(self):
        """Enqueue one step (on this object's stream)."""
        dit_graph_launch(self._exe, self.stream)

    def reset(self):
        """Start a new generation: clear the counters (on this object's stream)."""
        dit_cache_state_reset(self.state, self.stream)

    def counters(self) -> dict:
        """The device-resident counters (synchronises the stream)."""
        self.stream.synchronize()
        return read_cache_state(self.state)

    def decisions(self, steps: int | None = None):
        """Per-step records (rel, acc, decision) of the current generation."""
        self.stream.synchronize()
        n = read_cache_state(self.state)["step"] if steps is None else steps
        return read_cache_trace(self.trace, min(n, self.trace_capacity))

    def close(self):
        if self._exe:
            dit_graph_destroy(self._exe)
            self._exe = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
