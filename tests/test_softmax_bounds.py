"""The prefill softmax takes exponentials against the running max and redoes a tile
only when its row sum passes 2^20.  These cases drive that path hard and compare
with the oracle: scores that climb steadily along the keys (the running max goes
stale by tens of log2 units per tile), one key far above the rest at several
positions within a tile (P overflows to infinity in the first pass and must be
caught), and SA without sink blocks, where a row's first tiles can be fully
masked."""
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
    with Context(0) as c:
        yield c


def _run(ctx, q, k, v, scale, mode, block=128, sink=1, W=2):
    dev = ctx.device
    B, T, Hq, d = q.shape
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
    ctx.attn_prefill(qt, kt, vt, o, scale, layer_mode=lm, row_ptr=rp, col=col, block=block, lse=lse)
    ctx.check()
    mask = None if mode == 1 else oracle.streaming_mask(nb, nb, sink, W)
    ro, rl = oracle.attn_prefill(q, k, v, scale, block_mask=mask, block=block)
    return bits_of(o), lse.cpu().numpy(), ro, np.transpose(rl, (0, 2, 1))


def _climbing(T, Hq, Hkv, d, rate, seed):
    """q rows all equal; key u = (rate * u) * q_dir + noise: scores rise along the keys."""
    r = np.random.default_rng(seed)
    qdir = r.standard_normal(d).astype(np.float32)
    qdir /= np.linalg.norm(qdir)
    q = np.broadcast_to(qdir * 2.0, (1, T, Hq, d)).astype(np.float32)
    u = np.arange(T, dtype=np.float32)[:, None, None]
    k = (rate * u) * qdir + 0.1 * r.standard_normal((T, Hkv, d)).astype(np.float32)
    v = r.standard_normal((1, T, Hkv, d)).astype(np.float32)
    return synth.to_bf16_bits(q.copy()), synth.to_bf16_bits(k[None]), synth.to_bf16_bits(v)


@pytest.mark.parametrize("rate", [0.05, 0.3])
@pytest.mark.parametrize("mode", [1, 0])
def test_scores_climbing_along_the_keys(ctx, rate, mode):
    # scale 1/8, |q| = 2: the score of key u is about 0.25 * rate * u natural units,
    # so across one 128-key tile the max climbs by 0.25 * rate * 128 * 1.44 log2 units
    # (2.3 at rate 0.05, 14 at rate 0.3) and by hundreds over the whole row.
    T, Hq, Hkv, d = 1536, 4, 2, 64
    q, k, v = _climbing(T, Hq, Hkv, d, rate, seed=int(rate * 100) + mode)
    o, lse, ro, rl = _run(ctx, q, k, v, 0.125, mode)
    assert_close_attn(o, ro, f"climbing rate {rate} mode {mode}")
    assert_close_lse(lse, rl, f"climbing lse rate {rate} mode {mode}")


@pytest.mark.parametrize("row,key", [
    (1023, 984),    # key 88 of the row's last tile
    (1023, 901),    # key 5: the tile's first 32-key chunk
    (1023, 996),    # key 100: its last chunk
    (1023, 1023),   # the diagonal key, the tile's last
    (520, 500),     # key 116 of a middle tile, with more tiles after it
])
@pytest.mark.parametrize("mode", [1, 0])
def test_one_key_far_above_the_rest(ctx, mode, row, key):
    # One key scores ~250 log2 units above everything before it in one query row: the
    # exponentials against the running max overflow to infinity and the tile must be
    # redone with O and l rescaled.
    T, Hq, Hkv, d = 1024, 2, 1, 128
    q, k, v = synth.attention_inputs(1, T, Hq, Hkv, d, seed=77)
    qf = synth.bf16_bits_to_f32(q)
    kf = synth.bf16_bits_to_f32(k)
    # align the key with query row `row` of head 0, scaled so its score is ~ +180 natural units
    qrow = qf[0, row, 0]
    kf[0, key, 0] = qrow / np.dot(qrow, qrow) * 180.0 / (1 / math.sqrt(d))
    k = synth.to_bf16_bits(kf)
    o, lse, ro, rl = _run(ctx, q, k, v, 1 / math.sqrt(d), mode)
    assert np.isfinite(lse).all()
    assert_close_attn(o, ro, f"far key {key} row {row} mode {mode}")
    assert_close_lse(lse, rl, f"far key {key} row {row} lse mode {mode}")
    # the row is (nearly) the far key's value row
    assert rl[0, 0, row] > 170.0


def test_sa_without_sink_blocks(ctx):
    # sink 0: a row's first listed tile can be fully masked for some of its rows.
    T, Hq, Hkv, d = 1000, 4, 2, 128
    q, k, v = synth.attention_inputs(1, T, Hq, Hkv, d, seed=78)
    for block, W in ((64, 1), (128, 2), (256, 1)):
        o, lse, ro, rl = _run(ctx, q, k, v, 1 / math.sqrt(d), 0, block=block, sink=0, W=W)
        assert_close_attn(o, ro, f"sink 0 block {block} W {W}")
        assert_close_lse(lse, rl, f"sink 0 lse block {block} W {W}")
