"""Failure detection without a GPU fault: a wait that can never complete gives up after
its bounded spin limit, the host reads FLUX_ERR_TIMEOUT, and the context keeps working."""

import pytest
import torch

import oracle
from sparse_attention_flux_b200 import synth
from sparse_attention_flux_b200.flux import Context, FluxError, FLUX_ERR_TIMEOUT
from helpers import assert_close_attn, bits_of

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_stays_usable():
    with Context(0) as ctx:
        waited = torch.zeros(1, dtype=torch.int32, device=ctx.device)
        ctx.selftest_bounded_wait(200, waited)
        with pytest.raises(FluxError) as e:
            ctx.check()
        assert e.value.code == FLUX_ERR_TIMEOUT
        us = int(waited.item())
        assert 200_000 <= us < 5_000_000, us          # gave up after the limit, not before
        ctx.check()                                     # the word was cleared
        # the same context still computes correct attention
        q, k, v = synth.attention_inputs(1, 256, 2, 1, 64, seed=5)
        qt, kt, vt = (synth.torch_from_bits(x).to(ctx.device) for x in (q, k, v))
        o = torch.empty_like(qt)
        ctx.attn_prefill(qt, kt, vt, o, 0.125)
        ctx.check()
        ref, _ = oracle.attn_prefill(q, k, v, 0.125)
        assert_close_attn(bits_of(o), ref, "after a timeout")


def test_selftest_rejects_bad_limits():
    with Context(0) as ctx:
        with pytest.raises(FluxError):
            ctx.selftest_bounded_wait(0)
        with pytest.raises(FluxError):
            ctx.selftest_bounded_wait(20000)
