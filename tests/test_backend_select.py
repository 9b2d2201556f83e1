"""Backend selection by name (vLLM-Omni "Diffusion Attention Backends":
argument, then DIFFUSION_ATTENTION_BACKEND, then the platform default).  CPU
only: the two entry points are replaced by recorders."""
import pytest

import diffusion_transformer_attention_attn_b200 as dit


@pytest.fixture
def calls(monkeypatch):
    seen = []
    monkeypatch.setattr(dit, "dit_attn_fwd", lambda q, k, v, scale=None, stream=None: seen.append("bf16") or "o16")
    monkeypatch.setattr(dit, "dit_attn_fwd_q8",
                        lambda q, k, v, scale=None, smooth_k=True, pv_mode="fp8", stream=None:
                        seen.append(("q8", smooth_k, pv_mode)) or "o8")
    monkeypatch.delenv("DIFFUSION_ATTENTION_BACKEND", raising=False)
    return seen


def test_default_is_the_bf16_kernel(calls):
    assert dit.attention_backend() == "FLASH_ATTN"
    assert dit.attention(1, 2, 3) == "o16" and calls == ["bf16"]


def test_environment_then_argument(calls, monkeypatch):
    monkeypatch.setenv("DIFFUSION_ATTENTION_BACKEND", "SAGE_ATTN")
    assert dit.attention(1, 2, 3) == "o8"
    assert dit.attention(1, 2, 3, backend="flash_attn") == "o16"
    assert calls == [("q8", True, "fp8"), "bf16"]


def test_unknown_backend_is_refused(calls, monkeypatch):
    with pytest.raises(ValueError, match="no PyTorch SDPA fallback"):
        dit.attention(1, 2, 3, backend="TORCH_SDPA")
    monkeypatch.setenv("DIFFUSION_ATTENTION_BACKEND", "XFORMERS")
    with pytest.raises(ValueError):
        dit.attention_backend()
    assert calls == []
