"""Failure detection on the GPU without a fault: the bounded-wait self-test
makes a wait run out (an mbarrier nothing arrives on).  The library must
report DIT_ERR_TIMEOUT through the device error word, and the context must
stay usable: an attention call right after it matches the oracle.
"""
import time

import pytest

import oracle
from diffusion_transformer_attention_attn_b200 import inputs

from common import assert_bf16_parity, from_device_bf16, to_device_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import diffusion_transformer_attention_attn_b200 as dit
    dit.load_library()
    assert dit.dit_get_device_status() == 0
    yield


def test_bounded_wait_runs_out_and_is_reported():
    import diffusion_transformer_attention_attn_b200 as dit
    t0 = time.monotonic()
    completed = dit.dit_wait_selftest()
    status = dit.dit_get_device_status()
    elapsed = time.monotonic() - t0
    assert completed == 0, "the wait must give up, not complete"
    assert status == dit.DIT_ERR_TIMEOUT
    assert 0.5 < elapsed < 60.0, elapsed
    # reading the status cleared the word
    assert dit.dit_get_device_status() == dit.DIT_OK


def test_context_usable_after_a_timeout():
    import diffusion_transformer_attention_attn_b200 as dit
    assert dit.dit_wait_selftest() == 0
    assert dit.dit_get_device_status() == dit.DIT_ERR_TIMEOUT
    case = inputs.AttnCase("after_timeout", 1, 2, 200, 128, seed=11)
    qn, kn, vn = inputs.attn_inputs(case)
    o = dit.dit_attn_fwd(to_device_bf16(qn), to_device_bf16(kn), to_device_bf16(vn))
    assert dit.dit_get_device_status() == dit.DIT_OK
    assert_bf16_parity(from_device_bf16(o), oracle.attention(qn, kn, vn), "attention after a timeout")
