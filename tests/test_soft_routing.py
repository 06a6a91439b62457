"""Soft-routing forward blend r * FA + (1 - r) * SA against the oracle; r read on the device
(from flux_route's score output in the end-to-end case)."""
import math

import pytest
import torch

import oracle
from sparse_attention_flux_b200 import synth
from sparse_attention_flux_b200.flux import Context
from helpers import assert_close_attn, bits_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    with Context(0) as c:
        yield c


def _index(ctx, T, block, sink, W):
    nb = (T + block - 1) // block
    m = torch.empty((nb, nb), dtype=torch.uint8, device=ctx.device)
    ctx.build_streaming_mask(nb, nb, sink, W, m)
    rp = torch.empty(nb + 1, dtype=torch.int32, device=ctx.device)
    col = torch.empty(nb * nb, dtype=torch.int32, device=ctx.device)
    ctx.build_block_index(m, rp, col)
    return rp, col


@pytest.mark.parametrize("case", [(1, 256, 2, 1, 64, 64, 1, 2), (1, 1500, 8, 2, 128, 128, 1, 3),
                                  (2, 700, 4, 4, 128, 256, 1, 1)])
@pytest.mark.parametrize("r", [0.0, 0.3, 0.8, 1.0])
def test_soft_blend_matches_oracle(ctx, case, r):
    B, T, Hq, Hkv, d, block, sink, W = case
    dev = ctx.device
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=3000 + T)
    qt, kt, vt = (synth.torch_from_bits(x).to(dev) for x in (q, k, v))
    rp, col = _index(ctx, T, block, sink, W)
    scale = 1.0 / math.sqrt(d)
    score = torch.tensor([0.5, r], dtype=torch.float32, device=dev)
    o = torch.full_like(qt, float("nan"))
    ctx.attn_prefill_soft(qt, kt, vt, o, scale, score, 1, rp, col, block)
    ctx.check()
    nb = (T + block - 1) // block
    ref = oracle.attn_prefill_soft(q, k, v, scale, r, oracle.streaming_mask(nb, nb, sink, W), block)
    assert_close_attn(bits_of(o), ref, f"soft r={r}")
    if r in (0.0, 1.0):   # exactly the SA / FA output of the plain call
        o2 = torch.empty_like(qt)
        lm = torch.tensor([int(r)], dtype=torch.uint8, device=dev)
        ctx.attn_prefill(qt, kt, vt, o2, scale, layer_mode=lm, row_ptr=rp, col=col, block=block)
        ctx.check()
        assert torch.equal(o, o2)


def test_soft_blend_with_router_score(ctx):
    """Router score (r_soft = sigmoid(z)) feeds the blend without leaving the device."""
    dev = ctx.device
    hidden, W1, b1, W2, b2 = synth.router_inputs(512, 64, 32, 3, 71)
    _, _, r_o = oracle.route(hidden, W1, b1, W2, b2, 0.5)
    lm = torch.empty(3, dtype=torch.uint8, device=dev)
    score = torch.empty(3, dtype=torch.float32, device=dev)
    ctx.route(synth.torch_from_bits(hidden).to(dev),
              *(torch.from_numpy(x).to(dev) for x in (W1, b1, W2, b2)), 0.5, lm, score)
    B, T, Hq, Hkv, d, block = 1, 512, 4, 2, 64, 64
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=72)
    qt, kt, vt = (synth.torch_from_bits(x).to(dev) for x in (q, k, v))
    rp, col = _index(ctx, T, block, 1, 2)
    o = torch.empty_like(qt)
    ctx.attn_prefill_soft(qt, kt, vt, o, 0.125, score, 2, rp, col, block)
    ctx.check()
    ref = oracle.attn_prefill_soft(q, k, v, 0.125, float(r_o[2]), oracle.streaming_mask(8, 8, 1, 2),
                                   block)
    assert_close_attn(bits_of(o), ref, "soft with router score")
