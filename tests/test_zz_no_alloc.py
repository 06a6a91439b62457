"""flux_attn_decode_noalloc, the decode entry point that allocates nothing.

Some callers cannot call cudaMalloc -- an engine that reserves all device
memory at start-up and hands it out through its own pool, or a plugin host
that forbids libraries from allocating -- so they cannot create the flux_ctx
that holds flux_attn_decode's split-KV scratch.  This entry point keeps that
scratch in a static device array inside libflux.so instead.  The tests call it
through the C ABI and check it against flux_attn_decode and against the oracle,
within the parity tolerance of the other tests, on two calls in a row; they
cover both head dimensions, an absent routing vector (FA), a short cache that
takes a single split, and an out-of-range length reported through `status`
and cleared by the next call.  This file is named so that pytest collects it
last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_flux_b200 import flux, synth
from sparse_attention_flux_b200.flux import Context
from helpers import assert_close_attn, assert_close_lse, bits_of

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(None if t is None else t.data_ptr())


def _call_noalloc(q, kc, vc, sl, o, lse, scale, lm, sink, W, block, status):
    B, Hq, d = q.shape
    _, S_max, Hkv, _ = kc.shape
    return flux.lib().flux_attn_decode_noalloc(
        _p(q), _p(kc), _p(vc), S_max, _p(sl), _p(o), _p(lse), B, Hq, Hkv, d, _p(lm), 0, sink, W,
        block, scale, _p(status), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


CASES = [  # B, S_max, seqlens, Hq, Hkv, d, block, sink, W, routing
    (4, 9000, [9000, 8191, 4097, 130], 32, 8, 128, 128, 1, 16, "layer_mode"),
    (3, 5000, [5000, 64, 2500], 8, 2, 64, 64, 1, 4, "layer_mode"),
    (2, 3000, [3000, 1777], 4, 1, 128, 128, 0, 2, None),       # no routing vector: FA
    # 160 kv groups over a 64-token cache: the plan takes a single split
    (40, 64, [1 + (7 * b) % 64 for b in range(40)], 8, 4, 64, 64, 1, 1, "layer_mode"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}-S{c[1]}-d{c[5]}-{c[9]}")
def test_noalloc_decode_matches_ctx_decode_and_oracle_twice_in_a_row(case):
    B, S_max, seqlens, Hq, Hkv, d, block, sink, W, routing = case
    dev = torch.device("cuda", 0)
    q_b = synth.to_bf16_bits(synth.rng(11 + d).standard_normal((B, Hq, d), np.float32))
    k_b = synth.to_bf16_bits(synth.rng(12 + d).standard_normal((B, S_max, Hkv, d), np.float32))
    v_b = synth.to_bf16_bits(synth.rng(13 + d).standard_normal((B, S_max, Hkv, d), np.float32))
    q, kc, vc = (synth.torch_from_bits(x).to(dev) for x in (q_b, k_b, v_b))
    sl = torch.tensor(seqlens, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(d)
    modes = (1, 0) if routing else (1, 1)
    with Context(0) as ctx:
        for call, mode in enumerate(modes):      # two calls in a row (FA then SA when routed)
            lm = torch.tensor([mode], dtype=torch.uint8, device=dev) if routing else None
            o_ref = torch.empty_like(q)
            lse_ref = torch.empty((B, Hq), dtype=torch.float32, device=dev)
            ctx.attn_decode(q, kc, vc, sl, o_ref, scale, layer_mode=lm, sink_blocks=sink,
                            window_blocks=W, block=block, lse=lse_ref)
            ctx.check()
            o = torch.full_like(q, float("nan"))
            lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=dev)
            status = torch.full((1,), -1, dtype=torch.int32, device=dev)
            rc = _call_noalloc(q, kc, vc, sl, o, lse, scale, lm, sink, W, block, status)
            assert rc == flux.FLUX_OK, flux.lib().flux_last_error()
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            # the same kernel with the same split plan (same SM count): bit-identical
            assert torch.equal(o, o_ref), (call, mode, (o.float() - o_ref.float()).abs().max().item())
            assert torch.equal(lse, lse_ref), (call, mode)
            ro, rl = oracle.attn_decode(q_b, k_b, v_b, np.asarray(seqlens, np.int32), scale, mode,
                                        sink, W, block)
            assert_close_attn(bits_of(o), ro, f"no-alloc decode vs oracle, call {call}")
            assert_close_lse(lse.cpu().numpy(), rl, f"no-alloc decode lse vs oracle, call {call}")


def test_noalloc_reports_a_bad_length_and_the_next_call_clears_it():
    """A seqlens entry above S_max: status 2 and that sequence's output zeroed; the
    next call on the same stream starts from a clear error word and clear tickets."""
    dev = torch.device("cuda", 0)
    B, S_max, Hq, Hkv, d, block = 3, 4096, 8, 2, 128, 128
    q_b = synth.to_bf16_bits(synth.rng(21).standard_normal((B, Hq, d), np.float32))
    k_b = synth.to_bf16_bits(synth.rng(22).standard_normal((B, S_max, Hkv, d), np.float32))
    v_b = synth.to_bf16_bits(synth.rng(23).standard_normal((B, S_max, Hkv, d), np.float32))
    q, kc, vc = (synth.torch_from_bits(x).to(dev) for x in (q_b, k_b, v_b))
    scale = 1.0 / math.sqrt(d)
    lm = torch.tensor([1], dtype=torch.uint8, device=dev)
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)
    o = torch.full_like(q, float("nan"))
    bad = torch.tensor([4096, S_max + 1, 1000], dtype=torch.int32, device=dev)
    assert _call_noalloc(q, kc, vc, bad, o, None, scale, lm, 1, 16, block, status) == flux.FLUX_OK
    torch.cuda.synchronize()
    assert int(status.item()) == 2
    assert torch.all(o[1] == 0)
    good = [4096, 4095, 1000]
    o2 = torch.full_like(q, float("nan"))
    sl = torch.tensor(good, dtype=torch.int32, device=dev)
    assert _call_noalloc(q, kc, vc, sl, o2, None, scale, lm, 1, 16, block, status) == flux.FLUX_OK
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ro, _ = oracle.attn_decode(q_b, k_b, v_b, np.asarray(good, np.int32), scale, 1, 1, 16, block)
    assert_close_attn(bits_of(o2), ro, "no-alloc decode after an error")
    with Context(0) as ctx:
        o_ref = torch.empty_like(q)
        ctx.attn_decode(q, kc, vc, sl, o_ref, scale, layer_mode=lm, sink_blocks=1,
                        window_blocks=16, block=block)
        ctx.check()
    assert torch.equal(o2, o_ref)   # the same kernel and split plan as the ctx call


def test_noalloc_decode_rejects_shapes_beyond_its_scratch():
    dev = torch.device("cuda", 0)
    q = torch.zeros((8192, 2, 64), dtype=torch.bfloat16, device=dev)
    kc = torch.zeros((8192, 1, 1, 64), dtype=torch.bfloat16, device=dev)
    sl = torch.ones(8192, dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    rc = flux.lib().flux_attn_decode_noalloc(
        _p(q), _p(kc), _p(kc), 1, _p(sl), _p(o), None, 8192, 2, 1, 64, None, 0, 1, 1, 64, 0.1,
        None, None)
    assert rc == flux.FLUX_ERR_SHAPE
    assert b"4096" in flux.lib().flux_last_error()
