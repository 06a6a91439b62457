"""Dynamic SA block selection on the GPU against the oracle.

Scores: the GPU's fp32 scores are compared with the oracle's fp64 scores element
by element, within a bound relative to each element (SCORE_RTOL * P + SCORE_ATOL;
see helpers.score_bound).  Mask: (1) the GPU mask equals the oracle's selection run on the
GPU's own fp32 scores, bit for bit (the selection kernel against its definition);
(2) end to end, the GPU mask equals the oracle's own pipeline (oracle scores, then
the oracle's fp32 selection), except at candidates whose decision the score bound
leaves open -- where the oracle's running sum before the candidate lies within the
row's summed score bound of tau, or where two differing candidates' scores are
within their bounds of each other -- and the tests count such bits (zero in every
case measured).  The selected mask then drives the CSR builder and SA prefill,
compared with the oracle's attention under the same mask."""
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_flux_b200 import synth
from sparse_attention_flux_b200.flux import Context
from helpers import assert_close_attn, bits_of

pytestmark = pytest.mark.gpu

from helpers import (SCORE_ATOL, SCORE_RTOL, assert_scores_within_bound as _assert_scores_within_bound,
                     mask_vs_oracle_pipeline as _mask_vs_oracle_pipeline)


@pytest.fixture(scope="module")
def ctx():
    with Context(0, 128 << 20) as c:
        yield c


def _select(ctx, q, k, stride, tau, sink):
    dev = ctx.device
    qt, kt = synth.torch_from_bits(q).to(dev), synth.torch_from_bits(k).to(dev)
    T, d = q.shape[1], q.shape[3]
    nb = (T + 127) // 128
    mask = torch.full((nb, nb), 7, dtype=torch.uint8, device=dev)
    score = torch.full((nb, nb), float("nan"), dtype=torch.float32, device=dev)
    ctx.select_blocks(qt, kt, mask, 1 / math.sqrt(d), tau, sink, stride=stride, block_score=score)
    ctx.check()
    return mask.cpu().numpy(), score.cpu().numpy()


CASES = [  # B, T, Hq, Hkv, d, stride, tau, sink
    (1, 1024, 4, 2, 128, 8, 0.9, 1),
    (2, 700, 6, 2, 64, 8, 0.8, 0),       # ragged T; 3 query heads per kv head
    (1, 1500, 8, 1, 128, 8, 0.95, 2),    # 8 heads per kv head: two CTAs of four
    (1, 128, 2, 2, 64, 8, 0.5, 0),       # a single block
    (1, 3000, 5, 1, 64, 8, 0.9, 1),      # 5 heads per kv head: one per CTA
    (1, 2049, 4, 1, 128, 8, 0.7, 1),     # one token past a block boundary
    (1, 1, 4, 1, 128, 8, 0.9, 1),        # a single token
    (3, 130, 2, 1, 64, 8, 0.9, 0),       # two blocks, the second two tokens long; 2 heads per CTA
    (1, 1100, 1, 1, 64, 8, 0.6, 20),     # sink beyond the block count: every block forced
    (1, 4500, 8, 2, 128, 8, 0.99, 1),    # 9 key-block groups of 8 at the last query block
]


@pytest.mark.parametrize("case", CASES)
def test_scores_and_mask_match_oracle(ctx, case):
    B, T, Hq, Hkv, d, stride, tau, sink = case
    q, k, _ = synth.attention_inputs(B, T, Hq, Hkv, d, seed=600 + T)
    mask, score = _select(ctx, q, k, stride, tau, sink)
    P = oracle.block_scores(q, k, 128, stride, 1 / math.sqrt(d))
    nb = P.shape[0]
    lower = np.tril(np.ones((nb, nb), bool))
    for i in range(nb):
        _assert_scores_within_bound(score[i, :i + 1], P[i, :i + 1], f"{case} row {i}")
    assert np.all(score[~lower] == 0)
    # the row sums follow from the per-element bound
    np.testing.assert_allclose(score.astype(np.float64).sum(axis=1), 1.0,
                               atol=SCORE_RTOL + nb * SCORE_ATOL)
    # the selection kernel against its definition, on the GPU's own fp32 scores
    np.testing.assert_array_equal(mask, oracle.select_blocks(score, tau, sink), err_msg=str(case))
    # end to end against the oracle's own scores and selection
    open_bits = _mask_vs_oracle_pipeline(mask, P, list(range(nb)), tau, sink, str(case))
    print(f"{case}: {open_bits} mask bits differ from the oracle pipeline (all open decisions)")


@pytest.mark.parametrize("tau", [0.0, 1.0, 2.0])
def test_tau_edges(ctx, tau):
    """tau 0 keeps the forced blocks alone (sinks and the diagonal); tau above 1 is
    never reached, so every causal block is kept; tau 1 is the rounding edge, held to
    the oracle pipeline with its open decisions."""
    B, T, Hq, Hkv, d, sink = 1, 1700, 4, 2, 128, 1
    q, k, _ = synth.attention_inputs(B, T, Hq, Hkv, d, seed=640)
    mask, score = _select(ctx, q, k, 8, tau, sink)
    nb = mask.shape[0]
    lower = np.tril(np.ones((nb, nb), bool))
    if tau == 0.0:
        want = np.zeros((nb, nb), np.uint8)
        want[:, :sink] = 1
        np.fill_diagonal(want, 1)
        np.testing.assert_array_equal(mask, want * lower)
    elif tau == 2.0:
        np.testing.assert_array_equal(mask, lower.astype(np.uint8))
    np.testing.assert_array_equal(mask, oracle.select_blocks(score, tau, sink))
    P = oracle.block_scores(q, k, 128, 8, 1 / math.sqrt(d))
    _mask_vs_oracle_pipeline(mask, P, list(range(nb)), tau, sink, f"tau {tau}")


def test_planted_block_is_selected(ctx):
    # Keys of block 3 are the antidiagonal partners of query block 9's rows times 4:
    # block 3 takes almost all of query block 9's mass, far outside any local window.
    T, Hq, Hkv, d, S = 1536, 2, 1, 64, 8
    q, k, _ = synth.attention_inputs(1, T, Hq, Hkv, d, seed=21)
    qf, kf = synth.bf16_bits_to_f32(q), synth.bf16_bits_to_f32(k)
    R = 128 // S
    for c in range(3 * R, 4 * R):
        for kk in range(S):
            kf[0, c * S + S - 1 - kk, 0] = 4.0 * (qf[0, 9 * 128 + kk, 0] + qf[0, 9 * 128 + kk, 1])
    k = synth.to_bf16_bits(kf)
    mask, score = _select(ctx, q, k, S, 0.5, 1)
    assert np.argmax(score[9, :10]) == 3
    assert list(np.nonzero(mask[9])[0]) == [0, 3, 9]


def test_selected_mask_drives_sa_prefill(ctx):
    B, T, Hq, Hkv, d = 1, 1900, 4, 2, 128
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=33)
    dev = ctx.device
    qt, kt, vt = (synth.torch_from_bits(x).to(dev) for x in (q, k, v))
    nb = (T + 127) // 128
    mask = torch.empty((nb, nb), dtype=torch.uint8, device=dev)
    ctx.select_blocks(qt, kt, mask, 1 / math.sqrt(d), 0.8, 1)
    rp = torch.empty(nb + 1, dtype=torch.int32, device=dev)
    col = torch.empty(nb * nb, dtype=torch.int32, device=dev)
    ctx.build_block_index(mask, rp, col)
    o = torch.full_like(qt, float("nan"))
    lm = torch.tensor([0], dtype=torch.uint8, device=dev)
    ctx.attn_prefill(qt, kt, vt, o, 1 / math.sqrt(d), layer_mode=lm, row_ptr=rp, col=col, block=128)
    ctx.check()
    m = mask.cpu().numpy()
    assert m.sum() < np.tril(np.ones((nb, nb))).sum()   # something was skipped
    ro, _ = oracle.attn_prefill(q, k, v, 1 / math.sqrt(d), block_mask=m, block=128)
    assert_close_attn(bits_of(o), ro, "SA prefill over the selected mask")


def test_deterministic(ctx):
    q, k, _ = synth.attention_inputs(2, 2500, 8, 2, 128, seed=44)
    m1, s1 = _select(ctx, q, k, 8, 0.9, 1)
    m2, s2 = _select(ctx, q, k, 8, 0.9, 1)
    assert np.array_equal(m1, m2) and np.array_equal(s1, s2)


def _sampled_rows_check(score, mask, q, k, d, rows, tau, sink, what):
    """Sampled score rows against the oracle within the per-element bound; properties
    of the whole GPU matrix (rows sum to 1, nothing above the diagonal, the mask is the
    oracle's selection on the GPU's fp32 scores, bit for bit); and the sampled rows of
    the mask against the oracle's own pipeline."""
    nb = score.shape[0]
    P = oracle.block_scores_rows(q, k, 128, 8, 1 / math.sqrt(d), rows)
    for n, i in enumerate(rows):
        _assert_scores_within_bound(score[i, :i + 1], P[n, :i + 1], f"{what} row {i}")
    upper = np.triu(np.ones((nb, nb), bool), 1)
    assert np.all(score[upper] == 0) and np.all(mask[upper] == 0)
    # the row sums follow from the per-element bound
    np.testing.assert_allclose(score.astype(np.float64).sum(axis=1), 1.0,
                               atol=SCORE_RTOL + nb * SCORE_ATOL)
    np.testing.assert_array_equal(mask, oracle.select_blocks(score, tau, sink), err_msg=what)
    open_bits = _mask_vs_oracle_pipeline(mask, P, rows, tau, sink, what)
    print(f"{what}: {open_bits} mask bits of the sampled rows differ from the oracle pipeline "
          f"(all open decisions)")


def test_qwen3_4b_layer_sampled_rows(ctx):
    """The bench's layer: B 1, T 32768, Hq 32, Hkv 8, d 128 with planted needles;
    stride 8, tau 0.9, sink 1.  Sampled query blocks (first, second, last, every needle
    row's block, and seeded others) against the oracle; the whole mask bit-exact on the
    GPU's scores; and the selected mask keeps more of the needles' key blocks than the
    sink + window mask."""
    B, T, Hq, Hkv, d, tau, sink = 1, 32768, 32, 8, 128, 0.9, 1
    seed = synth.seed_for(1)
    q, k, _ = synth.attention_inputs(B, T, Hq, Hkv, d, seed)
    needles = synth.plant_needles_np(q, k, seed)
    mask, score = _select(ctx, q, k, 8, tau, sink)
    nb = T // 128
    r = synth.rng(seed + 9)
    rows = sorted({0, 1, nb - 1} | {rr // 128 for (_, rr, _) in needles}
                  | set(int(x) for x in r.integers(0, nb, 6)))
    _sampled_rows_check(score, mask, q, k, d, rows, tau, sink, "T 32768")
    stream = oracle.streaming_mask(nb, nb, sink, 16)
    hit_sel = hit_stream = 0
    for (_h, rr, pos) in needles:
        for j in set(int(p) // 128 for p in pos):
            hit_sel += int(mask[rr // 128, j])
            hit_stream += int(stream[rr // 128, j])
    assert hit_sel > hit_stream


def test_largest_supported_layer(ctx):
    """T 131072 = 1024 key blocks, the largest the selector takes (the shared-memory
    log-sum-exp row and the sort are sized for it): sampled rows against the oracle and
    the whole mask bit-exact (one token more is refused on the host: test_abi)."""
    B, T, Hq, Hkv, d, tau, sink = 1, 131072, 4, 1, 128, 0.9, 1
    q, k, _ = synth.attention_inputs(B, T, Hq, Hkv, d, seed=777)
    mask, score = _select(ctx, q, k, 8, tau, sink)
    assert score.shape == (1024, 1024)
    _sampled_rows_check(score, mask, q, k, d, [0, 7, 8, 513, 1016, 1023], tau, sink, "T 131072")
