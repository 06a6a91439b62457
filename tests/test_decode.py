"""Split-KV decode attention against the fp64 oracle (FA and SA per layer; GQA group sizes 1 to 8)."""
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
    with Context(0, 256 << 20) as c:
        yield c


def _run(ctx, q, kc, vc, seqlens, scale, mode, sink, W, block):
    dev = ctx.device
    qt = synth.torch_from_bits(q).to(dev)
    kt = synth.torch_from_bits(kc).to(dev)
    vt = synth.torch_from_bits(vc).to(dev)
    sl = torch.from_numpy(np.asarray(seqlens, np.int32)).to(dev)
    o = torch.full_like(qt, float("nan"))
    lse = torch.full(q.shape[:2], float("nan"), dtype=torch.float32, device=dev)
    lm = None if mode is None else torch.tensor([mode, 1 - mode], dtype=torch.uint8, device=dev)
    ctx.attn_decode(qt, kt, vt, sl, o, scale, layer_mode=lm, layer=0, sink_blocks=sink,
                    window_blocks=W, block=block, lse=lse)
    ctx.check()
    return bits_of(o), lse.cpu().numpy()


CASES = [  # B, S_max, seqlens, Hq, Hkv, d, block, sink, W
    (2, 300, [300, 77], 2, 1, 64, 64, 1, 2),          # tiny oracle shapes
    (3, 5000, [5000, 1, 2049], 8, 2, 128, 128, 1, 16),
    (2, 4100, [4100, 4033], 8, 2, 128, 128, 1, 3),
    (1, 9000, [8999], 4, 4, 128, 128, 2, 4),
    (2, 777, [0, 776], 4, 2, 64, 64, 0, 1),
    (4, 2600, [2600, 2500, 130, 64], 32, 8, 128, 128, 1, 16),
    # group sizes other than 1, 2, 4 (up to 8 query heads per kv head)
    (2, 1500, [1500, 700], 6, 2, 128, 128, 1, 4),      # G 3
    (1, 2100, [2033], 5, 1, 64, 64, 1, 5),            # G 5
    (2, 1300, [1300, 1], 12, 2, 128, 64, 2, 3),       # G 6
    (3, 900, [900, 450, 129], 7, 1, 64, 128, 0, 2),   # G 7
    (2, 3000, [3000, 2999], 64, 8, 128, 128, 1, 16),  # G 8 (a 64 / 8 head layout)
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("mode", [None, 1, 0])
def test_decode_matches_oracle(ctx, case, mode):
    B, S_max, seqlens, Hq, Hkv, d, block, sink, W = case
    q, kc, vc = synth.decode_inputs(B, S_max, Hq, Hkv, d, seed=2000 + S_max)
    scale = 1.0 / math.sqrt(d)
    o, lse = _run(ctx, q, kc, vc, seqlens, scale, mode, sink, W, block)
    ro, rl = oracle.attn_decode(q, kc, vc, seqlens, scale, 1 if mode is None else mode, sink, W,
                                block)
    assert_close_attn(o, ro, f"decode {case} mode {mode}")
    assert_close_lse(lse, rl, "decode lse")


def test_no_routing_bits_is_the_fa_path_exactly(ctx):
    """layer_mode NULL and a routing bit of 1 take the same FA path: identical output and LSE."""
    B, S_max, seqlens, Hq, Hkv, d, block, sink, W = CASES[1]
    q, kc, vc = synth.decode_inputs(B, S_max, Hq, Hkv, d, seed=2100)
    o_none, l_none = _run(ctx, q, kc, vc, seqlens, 0.088, None, sink, W, block)
    o_fa, l_fa = _run(ctx, q, kc, vc, seqlens, 0.088, 1, sink, W, block)
    assert np.array_equal(o_none, o_fa)
    assert np.array_equal(l_none, l_fa)


def test_decode_twice_in_a_row_and_mode_switch(ctx):
    # Tickets reset themselves: repeated calls and FA/SA alternation agree.
    B, S_max, Hq, Hkv, d = 2, 3000, 8, 2, 128
    q, kc, vc = synth.decode_inputs(B, S_max, Hq, Hkv, d, seed=7)
    sl = [3000, 2222]
    a = _run(ctx, q, kc, vc, sl, 0.08, 1, 1, 4, 128)
    b = _run(ctx, q, kc, vc, sl, 0.08, 0, 1, 4, 128)
    c = _run(ctx, q, kc, vc, sl, 0.08, 1, 1, 4, 128)
    assert np.array_equal(a[0], c[0])
    ro, _ = oracle.attn_decode(q, kc, vc, sl, 0.08, 0, 1, 4, 128)
    assert_close_attn(b[0], ro, "SA after FA")


def test_bad_seqlen_is_reported_and_output_zeroed(ctx):
    B, S_max, Hq, Hkv, d = 2, 256, 4, 1, 64
    q, kc, vc = synth.decode_inputs(B, S_max, Hq, Hkv, d, seed=9)
    dev = ctx.device
    qt, kt, vt = (synth.torch_from_bits(x).to(dev) for x in (q, kc, vc))
    sl = torch.tensor([S_max + 5, 100], dtype=torch.int32, device=dev)
    o = torch.full_like(qt, 3.0)
    ctx.attn_decode(qt, kt, vt, sl, o, 0.125, sink_blocks=1, window_blocks=2, block=64)
    with pytest.raises(FluxError) as e:
        ctx.check()
    assert e.value.code == FLUX_ERR_DEVICE_CHECK
    assert (o[0].float() == 0).all()
    ro, _ = oracle.attn_decode(q, kc, vc, [0, 100], 0.125, 1, 1, 2, 64)
    assert_close_attn(bits_of(o[1:]), ro[1:], "valid sequence next to a bad one")
    ctx.check()


def test_decode_equals_prefill_last_row_on_gpu(ctx):
    # Cross-path invariant: decode at s equals the last row of prefill at T = s.
    B, T, Hq, Hkv, d = 1, 1200, 8, 2, 128
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=31)
    dev = ctx.device
    for mode in (1, 0):
        lm = torch.tensor([mode], dtype=torch.uint8, device=dev)
        nb = (T + 127) // 128
        m = torch.empty((nb, nb), dtype=torch.uint8, device=dev)
        ctx.build_streaming_mask(nb, nb, 1, 3, m)
        rp = torch.empty(nb + 1, dtype=torch.int32, device=dev)
        col = torch.empty(nb * nb, dtype=torch.int32, device=dev)
        ctx.build_block_index(m, rp, col)
        qt, kt, vt = (synth.torch_from_bits(x).to(dev) for x in (q, k, v))
        op = torch.empty_like(qt)
        ctx.attn_prefill(qt, kt, vt, op, 0.088, layer_mode=lm, layer=0, row_ptr=rp, col=col,
                         block=128)
        od = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev)
        sl = torch.tensor([T], dtype=torch.int32, device=dev)
        ctx.attn_decode(qt[:, T - 1].contiguous(), kt, vt, sl, od, 0.088, layer_mode=lm,
                        sink_blocks=1, window_blocks=3, block=128)
        ctx.check()
        diff = (op[:, T - 1].float() - od.float()).abs().max().item()
        assert diff < 2e-2, (mode, diff)


@pytest.mark.parametrize("mode", [1, 0])
def test_qwen3_4b_decode_workload_sampled_sequences(ctx, mode):
    """Qwen3-4B-shaped decode: batch 16, KV 131072 (+ step), Hkv 8, d 128, Hq 32;
    SA reads sink 1 block + last 16 blocks of 128.  Every sequence's output is
    computed on the GPU; two sequences are checked against the oracle."""
    B, S_max, Hq, Hkv, d = 16, 131072 + 64, 32, 8, 128
    dev = ctx.device
    seed = synth.seed_for(3)
    kc = synth.torch_normal_bf16((B, S_max, Hkv, d), seed + 1, dev)
    vc = synth.torch_normal_bf16((B, S_max, Hkv, d), seed + 2, dev)
    q = synth.torch_normal_bf16((B, Hq, d), seed, dev)
    seqlens = np.array([131072 + (7 * b) % 64 for b in range(B)], np.int32)
    sl = torch.from_numpy(seqlens).to(dev)
    o = torch.full_like(q, float("nan"))
    lm = torch.tensor([mode], dtype=torch.uint8, device=dev)
    scale = 1.0 / math.sqrt(d)
    ctx.attn_decode(q, kc, vc, sl, o, scale, layer_mode=lm, sink_blocks=1, window_blocks=16,
                    block=128)
    ctx.check()
    ob = bits_of(o)
    assert np.all(np.isfinite(synth.bf16_bits_to_f32(ob)))
    qb = bits_of(q)
    for b in (0, 11):
        kb, vb = bits_of(kc[b:b + 1]), bits_of(vc[b:b + 1])
        ro, _ = oracle.attn_decode(qb[b:b + 1], kb, vb, seqlens[b:b + 1], scale, mode, 1, 16, 128)
        assert_close_attn(ob[b:b + 1], ro, f"decode seq {b} mode {mode}")
