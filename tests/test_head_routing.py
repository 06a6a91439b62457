"""Per-head routing (the contrast case): every query head equals its own FA or SA
oracle result; uniform head modes equal the layer-level call exactly, in prefill and decode."""
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_flux_b200 import synth
from sparse_attention_flux_b200.flux import Context
from helpers import assert_close_attn, bits_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    with Context(0, 128 << 20) as c:
        yield c


def _index(ctx, T, block, sink, W):
    nb = (T + block - 1) // block
    m = torch.empty((nb, nb), dtype=torch.uint8, device=ctx.device)
    ctx.build_streaming_mask(nb, nb, sink, W, m)
    rp = torch.empty(nb + 1, dtype=torch.int32, device=ctx.device)
    col = torch.empty(nb * nb, dtype=torch.int32, device=ctx.device)
    ctx.build_block_index(m, rp, col)
    return rp, col


@pytest.mark.parametrize("case", [(1, 1000, 8, 2, 128, 128, 1, 3), (2, 300, 4, 2, 64, 64, 1, 2)])
def test_prefill_per_head_matches_oracle(ctx, case):
    B, T, Hq, Hkv, d, block, sink, W = case
    dev = ctx.device
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=4000 + T)
    qt, kt, vt = (synth.torch_from_bits(x).to(dev) for x in (q, k, v))
    rp, col = _index(ctx, T, block, sink, W)
    hm = (synth.rng(T).random(Hq) < 0.5).astype(np.uint8)
    hm[0], hm[-1] = 1, 0
    o = torch.full_like(qt, float("nan"))
    ctx.attn_prefill_heads(qt, kt, vt, o, 1 / math.sqrt(d), torch.from_numpy(hm).to(dev), rp, col,
                           block)
    ctx.check()
    nb = (T + block - 1) // block
    fa, _ = oracle.attn_prefill(q, k, v, 1 / math.sqrt(d))
    sa, _ = oracle.attn_prefill(q, k, v, 1 / math.sqrt(d),
                                block_mask=oracle.streaming_mask(nb, nb, sink, W), block=block)
    ref = np.where(hm[None, None, :, None] == 1, fa, sa)
    assert_close_attn(bits_of(o), ref, "per-head prefill")


@pytest.mark.parametrize("case", [(1, 1000, 8, 2, 128, 128, 1, 3),   # G 4: layer-level uses head pairs
                                  (2, 300, 6, 2, 64, 64, 0, 2),     # G 3: row pairs in both
                                  (1, 777, 4, 1, 128, 64, 2, 5)])   # block 64: the CSR map path
@pytest.mark.parametrize("mode", [1, 0])
def test_prefill_uniform_head_modes_equal_the_layer_call(ctx, case, mode):
    """Every head FA (or every head SA) gives exactly the layer-level call's output: each
    query row meets the same key tiles in the same order; the extra tiles a row-pair unit
    walks are fully masked for that row, so they add exact zeros."""
    B, T, Hq, Hkv, d, block, sink, W = case
    dev = ctx.device
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=4100 + T + mode)
    qt, kt, vt = (synth.torch_from_bits(x).to(dev) for x in (q, k, v))
    rp, col = _index(ctx, T, block, sink, W)
    scale = 1 / math.sqrt(d)
    o_heads = torch.full_like(qt, float("nan"))
    ctx.attn_prefill_heads(qt, kt, vt, o_heads, scale,
                           torch.full((Hq,), mode, dtype=torch.uint8, device=dev), rp, col, block)
    o_layer = torch.full_like(qt, float("nan"))
    ctx.attn_prefill(qt, kt, vt, o_layer, scale,
                     layer_mode=torch.tensor([mode], dtype=torch.uint8, device=dev),
                     row_ptr=rp, col=col, block=block)
    ctx.check()
    assert torch.equal(o_heads, o_layer), (o_heads.float() - o_layer.float()).abs().max().item()


@pytest.mark.parametrize("pattern", ["mixed", "all_fa", "all_sa", "one_fa_per_group"])
def test_decode_per_head_matches_oracle(ctx, pattern):
    B, S_max, Hq, Hkv, d, block, sink, W = 3, 6000, 8, 2, 128, 128, 1, 4
    dev = ctx.device
    q, kc, vc = synth.decode_inputs(B, S_max, Hq, Hkv, d, seed=77)
    seqlens = np.array([6000, 1234, 300], np.int32)
    hm = {"mixed": np.array([1, 0, 0, 1, 0, 0, 0, 0]), "all_fa": np.ones(Hq),
          "all_sa": np.zeros(Hq), "one_fa_per_group": np.array([0, 0, 1, 0, 0, 0, 0, 1])}[pattern]
    hm = hm.astype(np.uint8)
    qt, kt, vt = (synth.torch_from_bits(x).to(dev) for x in (q, kc, vc))
    sl = torch.from_numpy(seqlens).to(dev)
    o = torch.full_like(qt, float("nan"))
    scale = 1 / math.sqrt(d)
    ctx.attn_decode_heads(qt, kt, vt, sl, o, scale, torch.from_numpy(hm).to(dev), sink, W, block)
    ctx.check()
    fa, _ = oracle.attn_decode(q, kc, vc, seqlens, scale, 1, sink, W, block)
    sa, _ = oracle.attn_decode(q, kc, vc, seqlens, scale, 0, sink, W, block)
    ref = np.where(hm[None, :, None] == 1, fa, sa)
    assert_close_attn(bits_of(o), ref, f"per-head decode {pattern}")
    if pattern in ("all_fa", "all_sa"):   # uniform heads = the layer-level call, bit for bit
        o2 = torch.empty_like(qt)
        lm = torch.tensor([1 if pattern == "all_fa" else 0], dtype=torch.uint8, device=dev)
        ctx.attn_decode(qt, kt, vt, sl, o2, scale, layer_mode=lm, sink_blocks=sink,
                        window_blocks=W, block=block)
        ctx.check()
        assert torch.equal(o, o2)


def test_decode_per_head_group_of_8(ctx):
    # Eight query heads per kv head (the largest group decode takes), heads of one group
    # routed differently: the group reads the FA range and its SA heads mask the rest.
    B, S_max, Hq, Hkv, d, block, sink, W = 2, 3000, 16, 2, 128, 64, 1, 6
    dev = ctx.device
    q, kc, vc = synth.decode_inputs(B, S_max, Hq, Hkv, d, seed=78)
    seqlens = np.array([3000, 1777], np.int32)
    hm = (synth.rng(79).random(Hq) < 0.5).astype(np.uint8)
    hm[:8] = [0, 1, 0, 0, 0, 0, 0, 0]          # group 0: one FA head among seven SA heads
    qt, kt, vt = (synth.torch_from_bits(x).to(dev) for x in (q, kc, vc))
    sl = torch.from_numpy(seqlens).to(dev)
    o = torch.full_like(qt, float("nan"))
    scale = 1 / math.sqrt(d)
    ctx.attn_decode_heads(qt, kt, vt, sl, o, scale, torch.from_numpy(hm).to(dev), sink, W, block)
    ctx.check()
    fa, _ = oracle.attn_decode(q, kc, vc, seqlens, scale, 1, sink, W, block)
    sa, _ = oracle.attn_decode(q, kc, vc, seqlens, scale, 0, sink, W, block)
    ref = np.where(hm[None, :, None] == 1, fa, sa)
    assert_close_attn(bits_of(o), ref, "per-head decode, group of 8")
