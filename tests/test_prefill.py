"""Prefill attention (tcgen05/TMEM/TMA kernel) against the fp64 oracle.

Small cases are compared element by element over every row; the
Qwen3-4B-shaped layer (T = 32768, Hq 32, Hkv 8, d 128, with needles) is
compared on rows sampled per head, in the launch configuration the benchmark
times.  Tolerance: max-abs 2e-2, mean-abs 2e-3 on the bf16 output.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_flux_b200 import synth
from sparse_attention_flux_b200.flux import Context, FluxError
from helpers import assert_close_attn, assert_close_lse, bits_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    with Context(0) as c:
        yield c


def _sa_index(ctx, T, block, sink, W):
    nb = (T + block - 1) // block
    m = torch.empty((nb, nb), dtype=torch.uint8, device=ctx.device)
    ctx.build_streaming_mask(nb, nb, sink, W, m)
    rp = torch.empty(nb + 1, dtype=torch.int32, device=ctx.device)
    col = torch.empty(nb * nb, dtype=torch.int32, device=ctx.device)
    ctx.build_block_index(m, rp, col)
    return m, rp, col


def _run(ctx, q, k, v, scale, mode, block=128, sink=1, W=2, want_lse=True):
    """mode None -> FA without routing; 1 -> FA via layer_mode; 0 -> SA via layer_mode."""
    dev = ctx.device
    qt, kt, vt = (synth.torch_from_bits(x).to(dev) for x in (q, k, v))
    o = torch.full_like(qt, float("nan"))
    B, T, Hq, d = q.shape
    lse = torch.full((B, Hq, T), float("nan"), dtype=torch.float32, device=dev) if want_lse else None
    if mode is None:
        ctx.attn_prefill(qt, kt, vt, o, scale, lse=lse, block=block)
    else:
        _, rp, col = _sa_index(ctx, T, block, sink, W)
        lm = torch.tensor([1 - mode, mode, 0], dtype=torch.uint8, device=dev)
        ctx.attn_prefill(qt, kt, vt, o, scale, layer_mode=lm, layer=1, row_ptr=rp, col=col,
                         block=block, lse=lse)
    ctx.check()
    return bits_of(o), (lse.cpu().numpy() if want_lse else None)


def _oracle(q, k, v, scale, sparse, block, sink, W):
    T = q.shape[1]
    nb = (T + block - 1) // block
    m = oracle.streaming_mask(nb, nb, sink, W) if sparse else None
    return oracle.attn_prefill(q, k, v, scale, block_mask=m, block=block)


CASES = [  # B, T, Hq, Hkv, d, block, sink, W
    (1, 256, 2, 1, 64, 64, 1, 2),       # the tiny oracle case
    (1, 1, 2, 1, 64, 64, 1, 2),
    (1, 100, 4, 2, 128, 128, 1, 2),
    (1, 129, 4, 2, 128, 128, 1, 2),
    (2, 300, 8, 2, 128, 128, 1, 2),
    (1, 513, 4, 1, 128, 128, 1, 3),
    (1, 700, 2, 2, 64, 64, 1, 3),
    (1, 1000, 4, 4, 128, 256, 1, 2),
    (1, 1500, 8, 2, 128, 128, 0, 4),
    (1, 777, 6, 2, 128, 128, 1, 3),     # odd group size (3): row-pair CTAs
    (2, 384, 12, 2, 64, 64, 2, 2),      # group size 6: head-pair CTAs across three pairs
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("mode", [None, 1, 0])
def test_prefill_matches_oracle(ctx, case, mode):
    B, T, Hq, Hkv, d, block, sink, W = case
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=1000 + T + d)
    scale = 1.0 / math.sqrt(d)
    o, lse = _run(ctx, q, k, v, scale, mode, block, sink, W)
    ro, rl = _oracle(q, k, v, scale, mode == 0, block, sink, W)
    assert_close_attn(o, ro, f"prefill {case} mode {mode}")
    assert_close_lse(lse, np.transpose(rl, (0, 2, 1)), f"lse {case} mode {mode}")


def test_sa_with_window_covering_everything_equals_fa(ctx):
    B, T, Hq, Hkv, d = 1, 640, 4, 2, 128
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=55)
    o_fa, _ = _run(ctx, q, k, v, 0.1, 1, 128, 1, 2)
    o_sa, _ = _run(ctx, q, k, v, 0.1, 0, 128, 0, 5)
    assert np.array_equal(o_fa, o_sa)


def test_routing_bit_is_read_on_device(ctx):
    # Same call, only the device-side bit differs: SA must differ from FA on a
    # long enough prompt and match its own oracle.
    B, T, Hq, Hkv, d = 1, 1024, 2, 1, 128
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=56)
    o_fa, _ = _run(ctx, q, k, v, 0.09, 1, 128, 1, 2)
    o_sa, _ = _run(ctx, q, k, v, 0.09, 0, 128, 1, 2)
    assert not np.array_equal(o_fa, o_sa)
    ro, _ = _oracle(q, k, v, 0.09, True, 128, 1, 2)
    assert_close_attn(o_sa, ro, "SA")


def test_bad_arguments_are_rejected(ctx):
    q, k, v = synth.attention_inputs(1, 64, 2, 1, 128, seed=1)
    dev = ctx.device
    qt, kt, vt = (synth.torch_from_bits(x).to(dev) for x in (q, k, v))
    o = torch.empty_like(qt)
    with pytest.raises(FluxError):
        ctx.attn_prefill(qt, kt, vt, o, 0.1, block=96)
    lm = torch.ones(1, dtype=torch.uint8, device=dev)
    with pytest.raises(FluxError):   # routing needs a block index
        ctx.attn_prefill(qt, kt, vt, o, 0.1, layer_mode=lm)
    q3, k3, v3 = synth.attention_inputs(1, 64, 3, 2, 128, seed=1)
    with pytest.raises(FluxError):   # Hq % Hkv != 0
        ctx.attn_prefill(*(synth.torch_from_bits(x).to(dev) for x in (q3, k3, v3)),
                         torch.empty((1, 64, 3, 128), dtype=torch.bfloat16, device=dev), 0.1)


def _sample_rows(T, Hq, needles, seed, per_head=48):
    r = synth.rng(seed)
    rows = []
    fixed = [0, 1, 127, 128, 129, 255, 256, T // 2, T - 129, T - 128, T - 1]
    for h in range(Hq):
        ts = set(int(x) for x in r.integers(0, T, per_head)) | set(fixed)
        for (hh, rr, _) in needles:
            if hh == h:
                ts.add(rr)
        rows += [(0, h, t) for t in sorted(ts)]
    return np.array(rows, np.int32)


@pytest.mark.parametrize("mode", [1, 0])
def test_qwen3_4b_layer_prefill_sampled_rows(ctx, mode):
    """Qwen3-4B-shaped layer: B 1, T 32768, Hq 32, Hkv 8, d 128, needles; FA and SA
    (block 128, sink 1, window 16) -- sampled rows against the oracle."""
    B, T, Hq, Hkv, d = 1, 32768, 32, 8, 128
    seed = synth.seed_for(1)
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed)
    needles = synth.plant_needles_np(q, k, seed)
    scale = 1.0 / math.sqrt(d)
    o, lse = _run(ctx, q, k, v, scale, mode, 128, 1, 16)
    rows = _sample_rows(T, Hq, needles, seed + 5)
    m = oracle.streaming_mask(T // 128, T // 128, 1, 16) if mode == 0 else None
    ro, rl = oracle.attn_prefill(q, k, v, scale, block_mask=m, block=128, rows=rows)
    got = o[rows[:, 0], rows[:, 2], rows[:, 1]]
    assert_close_attn(got, ro, f"Qwen3-4B layer mode {mode}")
    assert_close_lse(lse[rows[:, 0], rows[:, 1], rows[:, 2]], rl, "lse")
    if mode == 1:
        # Each needle query finds its 16 planted keys: o is close to their mean value row.
        V = synth.bf16_bits_to_f32(v).astype(np.float64)
        for (h, r, pos) in needles:
            target = V[0, pos, h // (Hq // Hkv)].mean(0)
            assert np.abs(synth.bf16_bits_to_f32(o[0, r, h]) - target).max() < 0.1
