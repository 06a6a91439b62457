"""Fused append + decode (flux_attn_decode_append): one launch that writes the step's
token into the cache and decodes.  It must equal flux_kv_write followed by the decode
bit for bit -- outputs, LSE and the whole cache -- for full caches (FA and SA via the
device bit) and SA rings, at lengths that put the new token on a block boundary (a ring
slot being reused), in the sink, and at capacity; a multi-step run is checked against
the oracle; a length of 0 is a device-checked error that writes nothing."""
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_flux_b200 import synth
from sparse_attention_flux_b200.flux import Context, FluxError, FLUX_ERR_DEVICE_CHECK
from helpers import assert_close_attn, bits_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    with Context(0, 64 << 20) as c:
        yield c


def _run_pair(ctx, q, new_k, new_v, kc, vc, sl, mode, sink, W, blk, compact):
    """(fused outputs and caches, separate-launch outputs and caches)."""
    dev = ctx.device
    scale = 1 / math.sqrt(q.shape[-1])
    lm = None if mode is None else torch.tensor([mode], dtype=torch.uint8, device=dev)
    B, Hq, _ = q.shape
    res = []
    for fused in (True, False):
        k, v = kc.clone(), vc.clone()
        o = torch.full_like(q, float("nan"))
        lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=dev)
        if fused:
            ctx.attn_decode_append(q, new_k, new_v, k, v, sl, o, scale, layer_mode=lm,
                                   sink_blocks=sink, window_blocks=W, block=blk, compact=compact,
                                   lse=lse)
        elif compact:
            ctx.kv_write(new_k.unsqueeze(1), new_v.unsqueeze(1), sl, k, v, sink, W, blk)
            ctx.attn_decode_sa_compact(q, k, v, sl, o, scale, sink, W, blk, lse=lse)
        else:
            ctx.kv_write(new_k.unsqueeze(1), new_v.unsqueeze(1), sl, k, v)
            ctx.attn_decode(q, k, v, sl, o, scale, layer_mode=lm, sink_blocks=sink,
                            window_blocks=W, block=blk, lse=lse)
        ctx.check()
        res.append((o, lse, k, v))
    return res


@pytest.mark.parametrize("mode", [None, 1, 0])
@pytest.mark.parametrize("d,G", [(128, 4), (64, 1)])
def test_full_cache_fused_equals_write_then_decode(ctx, mode, d, G):
    B, Hkv, S_max, blk, sink, W = 5, 2, 1000, 64, 1, 3
    Hq = Hkv * G
    dev = ctx.device
    q = synth.torch_normal_bf16((B, Hq, d), 11, dev)
    kc = synth.torch_normal_bf16((B, S_max, Hkv, d), 12, dev)
    vc = synth.torch_normal_bf16((B, S_max, Hkv, d), 13, dev)
    new_k = synth.torch_normal_bf16((B, Hkv, d), 14, dev)
    new_v = synth.torch_normal_bf16((B, Hkv, d), 15, dev)
    # only the new token, a block's first token, mid-block, one before capacity, capacity
    sl = torch.tensor([1, 129, 777, 999, 1000], dtype=torch.int32, device=dev)
    (o1, l1, k1, v1), (o2, l2, k2, v2) = _run_pair(ctx, q, new_k, new_v, kc, vc, sl, mode,
                                                   sink, W, blk, False)
    assert torch.equal(k1, k2) and torch.equal(v1, v2)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for b, s in enumerate(sl.tolist()):
        assert torch.equal(k1[b, s - 1], new_k[b]) and torch.equal(v1[b, s - 1], new_v[b])


@pytest.mark.parametrize("blk,sink,W", [(64, 1, 3), (128, 1, 16), (64, 2, 1)])
def test_ring_fused_equals_write_then_decode(ctx, blk, sink, W):
    B, Hkv, G, d = 6, 2, 2, 128
    Hq = Hkv * G
    rows = (sink + W) * blk
    dev = ctx.device
    q = synth.torch_normal_bf16((B, Hq, d), 21, dev)
    kr = synth.torch_normal_bf16((B, rows, Hkv, d), 22, dev)
    vr = synth.torch_normal_bf16((B, rows, Hkv, d), 23, dev)
    new_k = synth.torch_normal_bf16((B, Hkv, d), 24, dev)
    new_v = synth.torch_normal_bf16((B, Hkv, d), 25, dev)
    # in the sink, the first window token, a block boundary far along (slot reuse),
    # mid-block, a long sequence ending a block, a long sequence starting one
    sl = torch.tensor([1, sink * blk + 1, 7 * blk + 1, 5 * blk + 17, 4096 * blk, 4096 * blk + 1],
                      dtype=torch.int32, device=dev)
    (o1, l1, k1, v1), (o2, l2, k2, v2) = _run_pair(ctx, q, new_k, new_v, kr, vr, sl, None,
                                                   sink, W, blk, True)
    assert torch.equal(k1, k2) and torch.equal(v1, v2)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fused_steps_match_oracle(ctx):
    """Prompt fill, then 40 fused steps across block boundaries on a ring and on a full
    cache; at several steps both decodes are compared with the oracle over the history."""
    B, Hkv, G, d, T0, steps = 2, 2, 2, 64, 200, 40
    sink, W, blk = 1, 2, 64
    Hq = Hkv * G
    dev = ctx.device
    S_max = T0 + steps
    k_all = synth.normal_bf16_bits((B, S_max, Hkv, d), 31)
    v_all = synth.normal_bf16_bits((B, S_max, Hkv, d), 32)
    q_all = synth.normal_bf16_bits((steps, B, Hq, d), 33)
    kt, vt = synth.torch_from_bits(k_all).to(dev), synth.torch_from_bits(v_all).to(dev)
    rows = (sink + W) * blk
    kr = torch.zeros((B, rows, Hkv, d), dtype=torch.bfloat16, device=dev)
    vr = torch.zeros_like(kr)
    kf = torch.zeros((B, S_max, Hkv, d), dtype=torch.bfloat16, device=dev)
    vf = torch.zeros_like(kf)
    sl0 = torch.full((B,), T0, dtype=torch.int32, device=dev)
    ctx.kv_write(kt[:, :T0].contiguous(), vt[:, :T0].contiguous(), sl0, kr, vr, sink, W, blk)
    ctx.kv_write(kt[:, :T0].contiguous(), vt[:, :T0].contiguous(), sl0, kf, vf)
    scale = 1 / math.sqrt(d)
    sa = torch.zeros(1, dtype=torch.uint8, device=dev)
    for i in range(steps):
        s = T0 + i + 1
        sl = torch.full((B,), s, dtype=torch.int32, device=dev)
        q = synth.torch_from_bits(q_all[i]).to(dev)
        nk, nv = kt[:, s - 1].contiguous(), vt[:, s - 1].contiguous()
        o_r, o_f = torch.empty_like(q), torch.empty_like(q)
        ctx.attn_decode_append(q, nk, nv, kr, vr, sl, o_r, scale, sink_blocks=sink,
                               window_blocks=W, block=blk, compact=True)
        ctx.attn_decode_append(q, nk, nv, kf, vf, sl, o_f, scale, layer_mode=sa, sink_blocks=sink,
                               window_blocks=W, block=blk)
        ctx.check()
        if i in (0, 23, 24, 39):   # 24: the new token starts block 3 (ring slot reused)
            ro, _ = oracle.attn_decode(q_all[i], k_all[:, :s], v_all[:, :s],
                                       np.full(B, s, np.int32), scale, 0, sink, W, blk)
            assert_close_attn(bits_of(o_r), ro, f"ring step {i}")
            assert_close_attn(bits_of(o_f), ro, f"full step {i}")
    # the full cache now holds every token
    assert torch.equal(kf, kt) and torch.equal(vf, vt)


def test_zero_length_is_a_device_error_and_writes_nothing(ctx):
    B, Hkv, d, S_max = 2, 1, 64, 128
    dev = ctx.device
    q = synth.torch_normal_bf16((B, 2, d), 41, dev)
    kc = torch.zeros((B, S_max, Hkv, d), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    nk = synth.torch_normal_bf16((B, Hkv, d), 42, dev)
    o = torch.empty_like(q)
    sl = torch.tensor([0, 5], dtype=torch.int32, device=dev)
    ctx.attn_decode_append(q, nk, nk, kc, vc, sl, o, 0.1, sink_blocks=1, window_blocks=1, block=64)
    with pytest.raises(FluxError) as e:
        ctx.check()
    assert e.value.code == FLUX_ERR_DEVICE_CHECK
    assert (kc[0] == 0).all()
    assert torch.equal(kc[1, 4], nk[1])
    assert (o[0] == 0).all()


def test_rejects_a_ring_of_the_wrong_size(ctx):
    dev = ctx.device
    q = torch.zeros((1, 2, 64), dtype=torch.bfloat16, device=dev)
    kr = torch.zeros((1, 100, 1, 64), dtype=torch.bfloat16, device=dev)
    nk = torch.zeros((1, 1, 64), dtype=torch.bfloat16, device=dev)
    sl = torch.ones(1, dtype=torch.int32, device=dev)
    with pytest.raises(FluxError):
        ctx.attn_decode_append(q, nk, nk, kr, kr.clone(), sl, torch.empty_like(q), 0.1,
                               sink_blocks=1, window_blocks=1, block=64, compact=True)
