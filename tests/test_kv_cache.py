"""The compact SA KV cache: ring layout (bit-exact), prompt fill and per-step
append, and SA decode over the ring equal to SA decode over the full cache
(oracle).  The full-cache append of FA layers is checked bit for bit too."""
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_flux_b200 import synth
from sparse_attention_flux_b200.flux import Context, FluxError, FLUX_ERR_DEVICE_CHECK
from helpers import assert_close_attn, assert_close_lse, bits_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    with Context(0, 64 << 20) as c:
        yield c


def ring_row(u, s, sink, W, blk):
    """Where token u lives in the ring at sequence length s (None: not kept)."""
    j, nbs = u // blk, -(-s // blk)
    if j < sink:
        return u
    if j >= nbs - W:
        return (sink + j % W) * blk + u % blk
    return None


@pytest.mark.parametrize("T,sink,W,blk", [(1000, 1, 3, 64), (4096, 1, 16, 128), (300, 2, 2, 64),
                                          (100, 2, 4, 64), (129, 1, 1, 128)])
def test_ring_fill_layout_is_bit_exact(ctx, T, sink, W, blk):
    B, Hkv, d = 2, 2, 64
    dev = ctx.device
    k = synth.normal_bf16_bits((B, T, Hkv, d), 1)
    v = synth.normal_bf16_bits((B, T, Hkv, d), 2)
    rows = (sink + W) * blk
    kr = torch.full((B, rows, Hkv, d), 7.0, dtype=torch.bfloat16, device=dev)
    vr = torch.full_like(kr, -7.0)
    sl = torch.full((B,), T, dtype=torch.int32, device=dev)
    ctx.kv_write(synth.torch_from_bits(k).to(dev), synth.torch_from_bits(v).to(dev), sl, kr, vr,
                 sink, W, blk)
    ctx.check()
    kb, vb = bits_of(kr), bits_of(vr)
    seven = synth.to_bf16_bits(np.array([7.0], np.float32))[0]
    written = np.zeros(rows, bool)
    for u in range(T):
        r = ring_row(u, T, sink, W, blk)
        if r is not None:
            assert np.array_equal(kb[:, r], k[:, u]) and np.array_equal(vb[:, r], v[:, u]), u
            written[r] = True
    assert np.all(kb[:, ~written] == seven)


def test_full_cache_append_is_bit_exact(ctx):
    B, S_max, Hkv, d = 3, 50, 2, 64
    dev = ctx.device
    kc = torch.zeros((B, S_max, Hkv, d), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    new_k = synth.torch_normal_bf16((B, 1, Hkv, d), 3, dev)
    new_v = synth.torch_normal_bf16((B, 1, Hkv, d), 4, dev)
    sl = torch.tensor([1, 17, 50], dtype=torch.int32, device=dev)
    ctx.kv_write(new_k, new_v, sl, kc, vc)
    ctx.check()
    for b, s in enumerate([1, 17, 50]):
        assert torch.equal(kc[b, s - 1], new_k[b, 0]) and torch.equal(vc[b, s - 1], new_v[b, 0])
        assert (kc[b, :s - 1] == 0).all() and (kc[b, s:] == 0).all()


@pytest.mark.parametrize("blk,sink,W,d,G", [(128, 1, 16, 128, 4), (64, 1, 3, 64, 2),
                                            (128, 2, 4, 128, 1)])
def test_decode_over_ring_matches_oracle_through_appends(ctx, blk, sink, W, d, G):
    """Prompt fill, then 300 appends across block boundaries; at several steps SA decode
    over the ring equals SA decode over the full cache (oracle and GPU)."""
    B, Hkv = 3, 2
    Hq = Hkv * G
    T0, steps = [1500, 40, 700], 300
    S_max = max(T0) + steps
    dev = ctx.device
    seed = 900 + blk + W
    kfull = synth.normal_bf16_bits((B, S_max, Hkv, d), seed)
    vfull = synth.normal_bf16_bits((B, S_max, Hkv, d), seed + 1)
    kf_t = synth.torch_from_bits(kfull).to(dev)
    vf_t = synth.torch_from_bits(vfull).to(dev)
    rows = (sink + W) * blk
    kr = torch.zeros((B, rows, Hkv, d), dtype=torch.bfloat16, device=dev)
    vr = torch.zeros_like(kr)
    # prompt fill: each sequence writes its first T0[b] tokens (one call per sequence length)
    for b in range(B):
        sl = torch.zeros(B, dtype=torch.int32, device=dev)
        sl[b] = T0[b]
        ctx.kv_write(kf_t[b:b + 1, :T0[b]].contiguous(), vf_t[b:b + 1, :T0[b]].contiguous(),
                     sl[b:b + 1], kr[b:b + 1], vr[b:b + 1], sink, W, blk)
    scale = 1.0 / math.sqrt(d)
    for step in range(steps + 1):
        s = np.array([t + step for t in T0], np.int32)
        sl = torch.from_numpy(s).to(dev)
        if step > 0:   # append token s-1 of every sequence
            idx = torch.from_numpy(s - 1).long().to(dev)
            nk = kf_t[torch.arange(B, device=dev), idx].unsqueeze(1).contiguous()
            nv = vf_t[torch.arange(B, device=dev), idx].unsqueeze(1).contiguous()
            ctx.kv_write(nk, nv, sl, kr, vr, sink, W, blk)
        if step not in (0, 1, 23, 64, 127, 128, 200, steps):
            continue
        q = synth.torch_normal_bf16((B, Hq, d), seed + step, dev)
        o = torch.full_like(q, float("nan"))
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
        ctx.attn_decode_sa_compact(q, kr, vr, sl, o, scale, sink, W, blk, lse=lse)
        o_full = torch.empty_like(q)
        lse_full = torch.empty_like(lse)
        ctx.attn_decode(q, kf_t, vf_t, sl, o_full, scale,
                        layer_mode=torch.zeros(1, dtype=torch.uint8, device=dev),
                        sink_blocks=sink, window_blocks=W, block=blk, lse=lse_full)
        ctx.check()
        ro, rl = oracle.attn_decode(bits_of(q), kfull, vfull, s, scale, 0, sink, W, blk)
        assert_close_attn(bits_of(o), ro, f"ring decode step {step}")
        assert_close_lse(lse.cpu().numpy(), rl, f"ring lse step {step}")
        # Same tokens in the same 64-token tiles, the same SA splits and merge: the ring and
        # the full cache give bit-identical outputs and LSE.
        assert torch.equal(o, o_full), (step, (o.float() - o_full.float()).abs().max().item())
        assert torch.equal(lse, lse_full), step


def test_ring_write_rejects_short_seqlen(ctx):
    dev = ctx.device
    k = torch.zeros((1, 10, 1, 64), dtype=torch.bfloat16, device=dev)
    kr = torch.zeros((1, 3 * 64, 1, 64), dtype=torch.bfloat16, device=dev)
    ctx.kv_write(k, k, torch.tensor([5], dtype=torch.int32, device=dev), kr, kr.clone(), 1, 2, 64)
    with pytest.raises(FluxError) as e:
        ctx.check()
    assert e.value.code == FLUX_ERR_DEVICE_CHECK
    with pytest.raises(FluxError):   # ring size must be (sink + window) * block
        ctx.kv_write(k, k, torch.tensor([10], dtype=torch.int32, device=dev), kr, kr, 1, 3, 64)
