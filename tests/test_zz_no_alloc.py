"""flux_attn_decode_noalloc, the decode entry point that allocates nothing.

Some callers cannot call cudaMalloc -- an engine that reserves all device
memory at start-up and hands it out through its own pool, or a plugin host
that forbids libraries from allocating -- so they cannot create the flux_ctx
that holds flux_attn_decode's split-KV scratch.  This entry point keeps that
scratch in a static device array inside libflux.so instead.  The test calls it
through the C ABI and checks it against flux_attn_decode, within the parity
tolerance of the other tests, on two calls in a row.  This file is named so
that pytest collects it last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from sparse_attention_flux_b200 import flux, synth
from sparse_attention_flux_b200.flux import Context
from helpers import MAX_ABS, MEAN_ABS

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_noalloc(q, kc, vc, sl, o, lse, scale, lm, sink, W, block, status):
    B, Hq, d = q.shape
    _, S_max, Hkv, _ = kc.shape
    return flux.lib().flux_attn_decode_noalloc(
        _p(q), _p(kc), _p(vc), S_max, _p(sl), _p(o), _p(lse), B, Hq, Hkv, d, _p(lm), 0, sink, W,
        block, scale, _p(status), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_decode_matches_ctx_decode_twice_in_a_row():
    dev = torch.device("cuda", 0)
    B, S_max, Hq, Hkv, d, block, sink, W = 4, 9000, 32, 8, 128, 128, 1, 16
    q = synth.torch_normal_bf16((B, Hq, d), 11, dev)
    kc = synth.torch_normal_bf16((B, S_max, Hkv, d), 12, dev)
    vc = synth.torch_normal_bf16((B, S_max, Hkv, d), 13, dev)
    sl = torch.tensor([9000, 8191, 4097, 130], dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(d)
    with Context(0) as ctx:
        for call, mode in enumerate((1, 0)):      # FA then SA: two calls in a row
            lm = torch.tensor([mode], dtype=torch.uint8, device=dev)
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
            err = (o.double() - o_ref.double()).abs()
            assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, (call, mode)
            assert torch.allclose(lse, lse_ref, atol=2e-3, rtol=0)


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
