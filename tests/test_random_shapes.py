"""Seeded random shapes against the oracle: prefill (FA and SA, random block, sink,
window, GQA group and ragged T) and decode (full cache FA/SA, compact ring with the
fused append), element by element.  Sizes stay small so that the oracle runs each
case in well under a second."""
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_flux_b200 import synth
from sparse_attention_flux_b200.flux import Context
from helpers import assert_close_attn, assert_close_lse, bits_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    with Context(0, 64 << 20) as c:
        yield c


def _prefill_case(seed):
    r = np.random.default_rng(seed)
    G = int(r.choice([1, 2, 3, 4, 6]))
    Hkv = int(r.choice([1, 2]))
    d = int(r.choice([64, 128]))
    block = int(r.choice([64, 128, 256]))
    T = int(r.integers(1, 1400))
    B = int(r.choice([1, 2]))
    sink = int(r.integers(0, 3))
    W = int(r.integers(1, 6))
    mode = int(r.integers(0, 2))
    return B, T, Hkv * G, Hkv, d, block, sink, W, mode


@pytest.mark.parametrize("seed", range(12))
def test_prefill_random_shape(ctx, seed):
    B, T, Hq, Hkv, d, block, sink, W, mode = _prefill_case(7000 + seed)
    dev = ctx.device
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=8000 + seed)
    qt, kt, vt = (synth.torch_from_bits(x).to(dev) for x in (q, k, v))
    nb = (T + block - 1) // block
    m = torch.empty((nb, nb), dtype=torch.uint8, device=dev)
    ctx.build_streaming_mask(nb, nb, sink, W, m)
    rp = torch.empty(nb + 1, dtype=torch.int32, device=dev)
    col = torch.empty(nb * nb, dtype=torch.int32, device=dev)
    ctx.build_block_index(m, rp, col)
    o = torch.full_like(qt, float("nan"))
    lse = torch.full((B, Hq, T), float("nan"), dtype=torch.float32, device=dev)
    lm = torch.tensor([mode], dtype=torch.uint8, device=dev)
    scale = 1 / math.sqrt(d)
    ctx.attn_prefill(qt, kt, vt, o, scale, layer_mode=lm, row_ptr=rp, col=col, block=block, lse=lse)
    ctx.check()
    mask = None if mode == 1 else oracle.streaming_mask(nb, nb, sink, W)
    ro, rl = oracle.attn_prefill(q, k, v, scale, block_mask=mask, block=block)
    tag = f"prefill seed {seed}: B {B} T {T} Hq {Hq} Hkv {Hkv} d {d} block {block} sink {sink} W {W} mode {mode}"
    assert_close_attn(bits_of(o), ro, tag)
    assert_close_lse(lse.cpu().numpy(), np.transpose(rl, (0, 2, 1)), tag)


def _decode_case(seed):
    r = np.random.default_rng(seed)
    G = int(r.choice([1, 2, 3, 4, 5, 6, 7, 8]))
    Hkv = int(r.choice([1, 2, 3]))
    d = int(r.choice([64, 128]))
    block = int(r.choice([64, 128]))
    sink = int(r.integers(0, 3))
    W = int(r.integers(1, 5))
    B = int(r.integers(1, 5))
    S_max = int(r.integers(1, 3000))
    s = r.integers(1, S_max + 1, size=B).astype(np.int32)
    return B, Hkv * G, Hkv, d, block, sink, W, S_max, s


@pytest.mark.parametrize("seed", range(12))
def test_decode_random_shape(ctx, seed):
    B, Hq, Hkv, d, block, sink, W, S_max, s = _decode_case(9000 + seed)
    dev = ctx.device
    q = synth.normal_bf16_bits((B, Hq, d), 9100 + seed)
    kc = synth.normal_bf16_bits((B, S_max, Hkv, d), 9200 + seed)
    vc = synth.normal_bf16_bits((B, S_max, Hkv, d), 9300 + seed)
    qt, kt, vt = (synth.torch_from_bits(x).to(dev) for x in (q, kc, vc))
    sl = torch.from_numpy(s).to(dev)
    scale = 1 / math.sqrt(d)
    tag = f"decode seed {seed}: B {B} Hq {Hq} Hkv {Hkv} d {d} block {block} sink {sink} W {W} S_max {S_max} s {s.tolist()}"
    for mode in (1, 0):
        o = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device=dev)
        lm = torch.tensor([mode], dtype=torch.uint8, device=dev)
        ctx.attn_decode(qt, kt, vt, sl, o, scale, layer_mode=lm, sink_blocks=sink, window_blocks=W,
                        block=block)
        ctx.check()
        ro, _ = oracle.attn_decode(q, kc, vc, s, scale, mode, sink, W, block)
        assert_close_attn(bits_of(o), ro, f"{tag} mode {mode}")
    # the same SA decode through a compact ring: each sequence's first s - 1 tokens
    # written by flux_kv_write (prompt fill), token s - 1 appended by the decode launch
    rows = (sink + W) * block
    kr = torch.zeros((B, rows, Hkv, d), dtype=torch.bfloat16, device=dev)
    vr = torch.zeros_like(kr)
    for b in range(B):
        n = int(s[b]) - 1
        if n > 0:
            ctx.kv_write(kt[b:b + 1, :n].contiguous(), vt[b:b + 1, :n].contiguous(),
                         torch.tensor([n], dtype=torch.int32, device=dev), kr[b:b + 1],
                         vr[b:b + 1], sink, W, block)
    nk = torch.stack([kt[b, int(s[b]) - 1] for b in range(B)]).contiguous()
    nv = torch.stack([vt[b, int(s[b]) - 1] for b in range(B)]).contiguous()
    o = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device=dev)
    ctx.attn_decode_append(qt, nk, nv, kr, vr, sl, o, scale, sink_blocks=sink, window_blocks=W,
                           block=block, compact=True)
    ctx.check()
    ro, _ = oracle.attn_decode(q, kc, vc, s, scale, 0, sink, W, block)
    assert_close_attn(bits_of(o), ro, f"{tag} ring + fused append")
