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


def test_no_routing_bits_is_the_fa_path_exactly(ctx):
    """layer_mode NULL and a routing bit of 1 take the same FA path: identical output and LSE."""
    B, T, Hq, Hkv, d = 2, 777, 8, 2, 128
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=57)
    o_none, l_none = _run(ctx, q, k, v, 0.09, None)
    o_fa, l_fa = _run(ctx, q, k, v, 0.09, 1)
    assert np.array_equal(o_none, o_fa)
    assert np.array_equal(l_none, l_fa)


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


@pytest.mark.parametrize("mode", [1, 0])
def test_batch_of_two_chunked_unit_order(ctx, mode):
    """B 2, ragged T 20000, Hkv 8: the K/V of one kv group take 10 MB, so units run per
    sequence in chunks of 4 kv groups (of 8); sampled rows of both sequences and every
    head against the oracle, FA and SA (block 128, sink 1, window 16)."""
    B, T, Hq, Hkv, d = 2, 20000, 16, 8, 128
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=4242)
    scale = 1.0 / math.sqrt(d)
    o, lse = _run(ctx, q, k, v, scale, mode, 128, 1, 16)
    r = synth.rng(4243)
    rows = []
    for b in range(B):
        for h in range(Hq):
            ts = set(int(x) for x in r.integers(0, T, 12)) | {0, 127, 128, T - 129, T - 1}
            rows += [(b, h, t) for t in sorted(ts)]
    rows = np.array(rows, np.int32)
    nb = (T + 127) // 128
    m = oracle.streaming_mask(nb, nb, 1, 16) if mode == 0 else None
    ro, rl = oracle.attn_prefill(q, k, v, scale, block_mask=m, block=128, rows=rows)
    got = o[rows[:, 0], rows[:, 2], rows[:, 1]]
    assert_close_attn(got, ro, f"B 2 T 20000 mode {mode}")
    assert_close_lse(lse[rows[:, 0], rows[:, 1], rows[:, 2]], rl, "lse")


def _random_causal_block_mask(nb, keep, seed):
    r = np.random.default_rng(seed)
    m = (r.random((nb, nb)) < keep).astype(np.uint8)
    m[np.arange(nb), np.arange(nb)] = 1          # every row keeps its diagonal block
    return np.tril(m)


@pytest.mark.parametrize("case", [  # B, T, Hq, Hkv, d, block
    (1, 1000, 8, 2, 128, 128),      # head pairs, direct list (one CSR row per unit)
    (1, 1000, 4, 4, 128, 128),      # row pairs (G = 1): union of two CSR rows
    (1, 1100, 8, 2, 128, 256),      # head pairs, two key tiles per block
    (2, 900, 6, 6, 64, 256),        # row pairs inside one 256-row block: direct list
    (1, 700, 4, 1, 128, 64),        # block 64: per-64 sub-block masks
])
def test_random_block_mask_matches_oracle(ctx, case):
    """Arbitrary kept-block sets (not only sink + window), through the CSR list."""
    B, T, Hq, Hkv, d, block = case
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=77 + T + block)
    nb = (T + block - 1) // block
    mask = _random_causal_block_mask(nb, 0.35, seed=T + block)
    dev = ctx.device
    m_t = torch.from_numpy(mask).to(dev)
    rp = torch.empty(nb + 1, dtype=torch.int32, device=dev)
    col = torch.empty(nb * nb, dtype=torch.int32, device=dev)
    ctx.build_block_index(m_t, rp, col)
    qt, kt, vt = (synth.torch_from_bits(x).to(dev) for x in (q, k, v))
    o = torch.full_like(qt, float("nan"))
    lm = torch.zeros(1, dtype=torch.uint8, device=dev)
    ctx.attn_prefill(qt, kt, vt, o, 1 / np.sqrt(d), layer_mode=lm, row_ptr=rp, col=col,
                     block=block)
    ctx.check()
    ro, _ = oracle.attn_prefill(q, k, v, 1 / np.sqrt(d), block_mask=mask, block=block)
    assert_close_attn(bits_of(o), ro, f"random mask {case}")


@pytest.mark.parametrize("block", [128, 64])
@pytest.mark.parametrize("bad", ["out_of_range", "descending", "repeat"])
def test_malformed_csr_is_a_device_error(ctx, block, bad):
    """A CSR row out of range, out of order or with a repeated column is reported
    (FLUX_ERR_DEVICE_CHECK) and the context keeps working."""
    from sparse_attention_flux_b200.flux import FLUX_ERR_DEVICE_CHECK
    B, T, Hq, Hkv, d = 1, 512, 4, 2, 128
    nb = T // block
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=3)
    dev = ctx.device
    qt, kt, vt = (synth.torch_from_bits(x).to(dev) for x in (q, k, v))
    o = torch.empty_like(qt)
    rows = [list(range(i + 1)) for i in range(nb)]       # causal, all blocks kept
    last = rows[-1]
    if bad == "out_of_range":
        last[1] = nb + 3
    elif bad == "descending":
        last[0], last[1] = last[1], last[0]
    else:
        last[1] = last[0]
    rp = torch.tensor(np.cumsum([0] + [len(r) for r in rows]), dtype=torch.int32, device=dev)
    col = torch.tensor([c for r in rows for c in r], dtype=torch.int32, device=dev)
    lm = torch.zeros(1, dtype=torch.uint8, device=dev)
    ctx.attn_prefill(qt, kt, vt, o, 0.1, layer_mode=lm, row_ptr=rp, col=col, block=block)
    with pytest.raises(FluxError) as e:
        ctx.check()
    assert e.value.code == FLUX_ERR_DEVICE_CHECK
    # the rows that read the malformed CSR row are zeroed, the others computed
    o_b = bits_of(o)
    assert np.all(o_b[:, (nb - 1) * block:] == 0)
    assert np.any(o_b[:, :block] != 0)
    # the context is still usable: a well-formed call gives the oracle's answer
    o_ok, _ = _run(ctx, q, k, v, 0.1, 0, block, 1, 2)
    ro, _ = _oracle(q, k, v, 0.1, True, block, 1, 2)
    assert_close_attn(o_ok, ro, "after malformed CSR")
