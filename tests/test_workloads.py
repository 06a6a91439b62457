"""The large routed workloads against the oracle, in the launch configuration
the library uses: the 36-layer Qwen3-4B-shaped routed prefill (T 65536; the
router's device bits choose FA or SA per layer) and the Llama-3.1-8B-shaped
sweep (prefill T 131072 with the SA window at 8/16/32 blocks; 32-layer decode
at batch 4 with the SA fraction at 0/25/50/75/100 %).  Rows and sequences are
sampled: rows are independent, so the oracle's values for them are exact."""
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_flux_b200 import synth
from sparse_attention_flux_b200.flux import Context
from helpers import assert_close_attn, assert_close_lse, bits_of

pytestmark = pytest.mark.gpu

HQ, HKV, D = 32, 8, 128
SCALE = 1.0 / math.sqrt(D)


@pytest.fixture(scope="module")
def ctx():
    with Context(0, 256 << 20) as c:
        yield c


def _index(ctx, T, block, sink, W):
    nb = (T + block - 1) // block
    m = torch.empty((nb, nb), dtype=torch.uint8, device=ctx.device)
    ctx.build_streaming_mask(nb, nb, sink, W, m)
    rp = torch.empty(nb + 1, dtype=torch.int32, device=ctx.device)
    col = torch.empty(nb * (sink + W + 1), dtype=torch.int32, device=ctx.device)
    ctx.build_block_index(m, rp, col)
    return rp, col


def _rows(T, seed, per_head, extra=()):
    r = synth.rng(seed)
    out = []
    for h in range(HQ):
        ts = set(int(x) for x in r.integers(0, T, per_head)) | {0, 127, 128, T - 1, *extra}
        out += [(0, h, t) for t in sorted(ts)]
    return np.array(out, np.int32)


def _check_rows(o, lse, q, k, v, rows, block_mask, block, what):
    ro, rl = oracle.attn_prefill(q, k, v, SCALE, block_mask=block_mask, block=block, rows=rows)
    got = o[rows[:, 0], rows[:, 2], rows[:, 1]]
    assert_close_attn(got, ro, what)
    assert_close_lse(lse[rows[:, 0], rows[:, 1], rows[:, 2]], rl, what)


def test_qwen3_4b_36_layer_routed_prefill(ctx):
    """The bench's routed step at T 65536 with the bench's own inputs: the router on hidden
    65536 x 2560 (MLP 5120 -> 512 -> 36, b2 = +4 on 18 seeded layers and -4 on the rest),
    bit-exact against the oracle's routing (18 FA / 18 SA); then the first FA-routed and the
    first SA-routed layer, each with its own Q/K/V and planted needles as the bench draws
    them (block 128, sink 1, window 16), each reading its bit on the device; sampled rows
    and every needle row against the oracle."""
    T, dev = 65536, ctx.device
    hidden, W1, b1, W2, b2 = synth.router_inputs(T, 2560, 512, 36, synth.seed_for(2),
                                                 coin_bias=4.0, n_positive=18)
    mode_o, z, _ = oracle.route(hidden, W1, b1, W2, b2, 0.5)
    lm = torch.empty(36, dtype=torch.uint8, device=dev)
    ctx.route(synth.torch_from_bits(hidden).to(dev),
              *(torch.from_numpy(x).to(dev) for x in (W1, b1, W2, b2)), 0.5, lm)
    assert np.array_equal(lm.cpu().numpy(), mode_o)
    assert int(mode_o.sum()) == 18 and np.abs(z).min() > 1.0
    del hidden
    rp, col = _index(ctx, T, 128, 1, 16)
    nb = T // 128
    mask = oracle.streaming_mask(nb, nb, 1, 16)
    for layer in (int(np.argmax(mode_o == 1)), int(np.argmax(mode_o == 0))):
        q = synth.torch_normal_bf16((1, T, HQ, D), synth.seed_for(2, layer, 1), dev)
        k = synth.torch_normal_bf16((1, T, HKV, D), synth.seed_for(2, layer, 2), dev)
        v = synth.torch_normal_bf16((1, T, HKV, D), synth.seed_for(2, layer, 3), dev)
        needles = synth.plant_needles_torch(q, k, synth.seed_for(2, layer, 0))
        o = torch.empty_like(q)
        lse = torch.empty((1, HQ, T), dtype=torch.float32, device=dev)
        ctx.attn_prefill(q, k, v, o, SCALE, layer_mode=lm, layer=layer, row_ptr=rp, col=col,
                         block=128, lse=lse)
        ctx.check()
        rows = _rows(T, synth.seed_for(2, layer, 7), 10)
        rows = np.concatenate([rows, np.array([(0, h, r) for (h, r, _) in needles], np.int32)])
        _check_rows(bits_of(o), lse.cpu().numpy(), bits_of(q), bits_of(k), bits_of(v), rows,
                    None if mode_o[layer] else mask, 128, f"layer {layer} mode {mode_o[layer]}")


def test_llama_8b_prefill_131072_window_sweep(ctx):
    """Llama-3.1-8B-shaped layer at T 131072: FA, and SA with window 8 / 16 / 32 blocks."""
    T, dev = 131072, ctx.device
    seed = synth.seed_for(4)
    q = synth.torch_normal_bf16((1, T, HQ, D), seed, dev)
    k = synth.torch_normal_bf16((1, T, HKV, D), seed + 1, dev)
    v = synth.torch_normal_bf16((1, T, HKV, D), seed + 2, dev)
    qb, kb, vb = bits_of(q), bits_of(k), bits_of(v)
    o = torch.empty_like(q)
    lse = torch.empty((1, HQ, T), dtype=torch.float32, device=dev)
    rows = _rows(T, seed + 7, 3, extra=(T - 129, T // 2))
    nb = T // 128
    for W in (None, 8, 16, 32):
        mode = 1 if W is None else 0
        rp, col = _index(ctx, T, 128, 1, W or 1)
        lm = torch.tensor([mode], dtype=torch.uint8, device=dev)
        ctx.attn_prefill(q, k, v, o, SCALE, layer_mode=lm, row_ptr=rp, col=col, block=128,
                         lse=lse)
        ctx.check()
        mask = None if W is None else oracle.streaming_mask(nb, nb, 1, W)
        _check_rows(bits_of(o), lse.cpu().numpy(), qb, kb, vb, rows, mask, 128, f"W {W}")


@pytest.mark.parametrize("sa_fraction", [0.0, 0.25, 0.5, 0.75, 1.0])
def test_llama_8b_decode_sa_fraction_sweep(ctx, sa_fraction):
    """32 layers at batch 4, KV 131072 (+ a step), routing mask with the given SA fraction;
    every layer decodes on the GPU, one FA and one SA layer (where present) are checked on
    two sequences against the oracle, with the window at 16 blocks."""
    B, S, L, dev = 4, 131072, 32, ctx.device
    S_max = S + 8
    seed = synth.seed_for(4, salt=1)
    kc = synth.torch_normal_bf16((B, S_max, HKV, D), seed + 1, dev)
    vc = synth.torch_normal_bf16((B, S_max, HKV, D), seed + 2, dev)
    q = synth.torch_normal_bf16((B, HQ, D), seed, dev)
    seqlens = np.array([S + 7, S + 1, S, S - 77], np.int32)
    sl = torch.from_numpy(seqlens).to(dev)
    n_fa = int(round(L * (1 - sa_fraction)))
    mode = synth.layer_mode_choice(L, n_fa, seed)
    lm = torch.from_numpy(mode).to(dev)
    outs = {}
    for layer in range(L):
        o = torch.empty_like(q)
        ctx.attn_decode(q, kc, vc, sl, o, SCALE, layer_mode=lm, layer=layer, sink_blocks=1,
                        window_blocks=16, block=128)
        outs[layer] = o
    ctx.check()
    qb = bits_of(q)
    checked = [int(np.argmax(mode == m)) for m in (1, 0) if (mode == m).any()]
    for layer in checked:
        ob = bits_of(outs[layer])
        for b in (0, 3):
            ro, _ = oracle.attn_decode(qb[b:b + 1], bits_of(kc[b:b + 1]), bits_of(vc[b:b + 1]),
                                       seqlens[b:b + 1], SCALE, int(mode[layer]), 1, 16, 128)
            assert_close_attn(ob[b:b + 1], ro, f"layer {layer} mode {mode[layer]} seq {b}")
