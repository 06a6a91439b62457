"""Pins for the oracle's dynamic SA block selector.

The pages name a block-sparse selector for the SA side but print no algorithm, so
the oracle implements a stated reading (strided antidiagonal block scores, then
the fewest blocks whose score mass reaches tau; see oracle/flux_oracle.c).  Its
parity against the pages is unpinned; these tests pin the oracle to the
definition itself by routes that share none of its code: the full T x T score
matrix from a library matmul with the antidiagonals indexed explicitly, closed
forms, invariants and hand-enumerated selections."""
import math

import numpy as np
import pytest

import oracle
from sparse_attention_flux_b200 import synth


def _widen(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def _brute_scores(q, k, block, S, scale):
    """P[i][j] from the full score matrix: z[r][c] = scale * sum_k A[rS+k, cS+S-1-k]."""
    qf, kf = _widen(q), _widen(k)
    B, T, Hq, d = qf.shape
    Hkv = kf.shape[2]
    G = Hq // Hkv
    nr = -(-T // S)
    R = block // S
    nb = -(-nr // R)
    pad = nr * S
    P = np.zeros((nb, nb))
    for b in range(B):
        for h in range(Hq):
            A = np.zeros((pad, pad))
            A[:T, :T] = qf[b, :, h] @ kf[b, :, h // G].T
            z = np.full((nr, nr), -np.inf)
            for r in range(nr):
                for c in range(r + 1):
                    z[r, c] = scale * sum(A[r * S + kk, c * S + S - 1 - kk] for kk in range(S))
            for i in range(nb):
                rows = range(i * R, min((i + 1) * R, nr))
                E = np.zeros(nb)
                zmax = max(z[r, c] for r in rows for c in range(r + 1))
                for j in range(i + 1):
                    E[j] = sum(np.exp(z[r, c] - zmax) for r in rows
                               for c in range(j * R, min((j + 1) * R, r + 1)))
                P[i] += E / E.sum()
    return P / (B * Hq)


@pytest.mark.parametrize("T,Hq,Hkv,d,block,S", [
    (64, 2, 1, 16, 16, 4),
    (77, 4, 2, 16, 16, 8),     # ragged: the last strided row is part padding
    (96, 3, 3, 32, 32, 8),
    (50, 2, 2, 16, 8, 2),
])
def test_scores_match_brute_force(T, Hq, Hkv, d, block, S):
    q, k, _ = synth.attention_inputs(2, T, Hq, Hkv, d, seed=T * 7 + S)
    scale = 1 / np.sqrt(d)
    P = oracle.block_scores(q, k, block, S, scale)
    ref = _brute_scores(q, k, block, S, scale)
    assert P.shape == ref.shape
    np.testing.assert_allclose(P, ref, rtol=0, atol=1e-12)


def test_rows_sum_to_one_and_upper_triangle_is_zero():
    q, k, _ = synth.attention_inputs(1, 1000, 4, 2, 64, seed=5)
    P = oracle.block_scores(q, k, 128, 8, 0.125)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(P[np.triu_indices_from(P, 1)] == 0)
    assert np.all(P[np.tril_indices_from(P)] > 0)


def test_zero_keys_closed_form():
    # All logits 0: block mass = number of strided pairs, R^2 off the diagonal and
    # R(R+1)/2 on it, so P[i][j] = R^2 / (i R^2 + R(R+1)/2) for j < i.
    T, block, S = 512, 64, 8
    R = block // S
    q, _, _ = synth.attention_inputs(1, T, 2, 1, 32, seed=9)
    k = np.zeros((1, T, 1, 32), np.uint16)       # bf16 +0.0
    P = oracle.block_scores(q, k, block, S, 0.2)
    nb = T // block
    for i in range(nb):
        den = i * R * R + R * (R + 1) / 2
        np.testing.assert_allclose(P[i, :i], R * R / den, rtol=0, atol=1e-14)
        np.testing.assert_allclose(P[i, i], R * (R + 1) / 2 / den, rtol=0, atol=1e-14)


def test_planted_block_dominates():
    # Keys of block 2 set to a large multiple of the antidiagonal partner rows of
    # query block 5: key block 2 takes nearly all of query block 5's mass.
    T, Hq, d, block, S = 768, 1, 32, 128, 8
    R = block // S
    q, k, _ = synth.attention_inputs(1, T, Hq, 1, d, seed=11)
    qf, kf = _widen(q), _widen(k)
    for c in range(2 * R, 3 * R):
        for kk in range(S):
            kf[0, c * S + S - 1 - kk, 0] = 4.0 * qf[0, 5 * block + kk, 0]
    k2 = synth.to_bf16_bits(kf.astype(np.float32))
    P = oracle.block_scores(q, k2, block, S, 1 / np.sqrt(d))
    assert np.argmax(P[5, :6]) == 2 and P[5, 2] > 0.9
    m = oracle.select_blocks(P, 0.5, 0)
    assert list(np.nonzero(m[5])[0]) == [2, 5]


def test_selection_hand_enumerated():
    P = np.array([[1.0, 0, 0, 0],
                  [0.3, 0.7, 0, 0],
                  [0.5, 0.1, 0.4, 0],
                  [0.05, 0.6, 0.15, 0.2]], np.float32)
    # sink 0, tau 0.85: row 1 keeps 1 (forced, 0.7) then 0 (0.3); row 2 keeps 2
    # (forced, 0.4) then 0 (0.5) -> 0.9; row 3 keeps 3 (0.2), then 1 (0.6) -> 0.8,
    # then 2 (0.15) -> 0.95.
    m = oracle.select_blocks(P, 0.85, 0)
    np.testing.assert_array_equal(m, [[1, 0, 0, 0], [1, 1, 0, 0], [1, 0, 1, 0], [0, 1, 1, 1]])
    # tau 0.75: row 3 stops after block 1 (0.8).
    m = oracle.select_blocks(P, 0.75, 0)
    np.testing.assert_array_equal(m[3], [0, 1, 0, 1])
    # sink 1: block 0 is always kept.
    m = oracle.select_blocks(P, 0.5, 1)
    np.testing.assert_array_equal(m, [[1, 0, 0, 0], [1, 1, 0, 0], [1, 0, 1, 0], [1, 1, 0, 1]])


def test_selection_tau_extremes_and_ties():
    rng = np.random.default_rng(3)
    nb = 12
    P = np.tril(rng.random((nb, nb))).astype(np.float32)
    P /= P.sum(axis=1, keepdims=True)
    assert np.array_equal(oracle.select_blocks(P, 1.5, 0), np.tril(np.ones((nb, nb), np.uint8)))
    only_forced = oracle.select_blocks(P, 0.0, 2)
    expect = np.zeros((nb, nb), np.uint8)
    for i in range(nb):
        expect[i, i] = 1
        expect[i, :min(2, i + 1)] = 1
    np.testing.assert_array_equal(only_forced, expect)
    # equal scores: the smaller block index goes first
    T = np.zeros((4, 4), np.float32)
    T[3, :4] = [0.25, 0.25, 0.25, 0.25]
    m = oracle.select_blocks(T, 0.5, 0)
    np.testing.assert_array_equal(m[3], [1, 0, 0, 1])


def _select_reference(P, tau, sink):
    """The selection rule restated with Python's sort and numpy float32 sums."""
    nb = P.shape[0]
    m = np.zeros((nb, nb), np.uint8)
    for i in range(nb):
        forced = [j for j in range(i + 1) if j < sink or j == i]
        cum = np.float32(0)
        for j in forced:
            m[i, j] = 1
            cum = np.float32(cum + P[i, j])
        cand = sorted((j for j in range(i + 1) if j not in forced), key=lambda j: (-P[i, j], j))
        for j in cand:
            if not cum < np.float32(tau):
                break
            m[i, j] = 1
            cum = np.float32(cum + P[i, j])
    return m


@pytest.mark.parametrize("seed", range(5))
def test_selection_matches_restated_rule(seed):
    rng = np.random.default_rng(seed)
    nb = int(rng.integers(1, 40))
    P = np.tril(rng.random((nb, nb)) ** 3).astype(np.float32)
    P /= np.maximum(P.sum(axis=1, keepdims=True), 1e-30)
    P = P.astype(np.float32)
    tau = float(rng.choice([0.5, 0.8, 0.9, 0.95]))
    sink = int(rng.integers(0, 3))
    np.testing.assert_array_equal(oracle.select_blocks(P, tau, sink), _select_reference(P, tau, sink))


@pytest.mark.parametrize("T,Hq,Hkv,d,rows", [
    (1000, 4, 2, 64, [7, 0, 3]),        # unsorted, first and last blocks
    (777, 3, 1, 32, [6, 6, 2]),         # ragged T, a repeated block
    (300, 2, 2, 16, [1]),
])
def test_sampled_rows_equal_full_matrix(T, Hq, Hkv, d, rows):
    # Each query block's row depends on its own queries only: the sampled rows are the
    # full matrix's rows, bit for bit.
    q, k, _ = synth.attention_inputs(2, T, Hq, Hkv, d, seed=T + d)
    P = oracle.block_scores(q, k, 128, 8, 1 / np.sqrt(d))
    Pr = oracle.block_scores_rows(q, k, 128, 8, 1 / np.sqrt(d), rows)
    assert Pr.shape == (len(rows), P.shape[0])
    np.testing.assert_array_equal(Pr, P[rows])


def test_sampled_rows_reject_out_of_range():
    q, k, _ = synth.attention_inputs(1, 256, 2, 1, 16, seed=1)
    with pytest.raises(ValueError):
        oracle.block_scores_rows(q, k, 128, 8, 0.25, [2])
    with pytest.raises(ValueError):
        oracle.block_scores_rows(q, k, 128, 8, 0.25, [-1])


def _selection_boundary_case():
    """Oracle scores of a small layer and a tau that lies just above the running sum
    before one candidate of the last query block, so that any score error larger than
    the bound moves that decision."""
    q, k, _ = synth.attention_inputs(1, 2048, 2, 1, 64, seed=71)
    P = oracle.block_scores(q, k, 128, 8, 1 / math.sqrt(64))
    nb = P.shape[0]
    i = nb - 1
    p32 = P[i, :i + 1].astype(np.float32)
    forced = [0, i]
    cand = sorted((j for j in range(1, i)), key=lambda j: (-p32[j], j))
    cum = np.float32(0)
    for j in forced:
        cum = np.float32(cum + p32[j])
    for j in cand[:4]:
        cum = np.float32(cum + p32[j])
    # the fifth candidate is taken iff the running sum (cum) is below tau
    tau = float(np.float32(cum) + np.float32(2e-4))
    return P, tau


def test_mask_check_rejects_a_biased_selection():
    """The parity check of the GPU selector, pinned by planting a mistake in the oracle:
    scores with a systematic relative bias 20x the stated bound flip a selection near
    tau; the score check and the mask check against the oracle's own pipeline both
    reject them, while scores within the bound pass both."""
    from helpers import (SCORE_RTOL, assert_scores_within_bound, mask_vs_oracle_pipeline)
    P, tau = _selection_boundary_case()
    nb = P.shape[0]
    i = nb - 1
    rows = [i]
    # a bias that raises the forced and first candidates' shares: the fifth candidate drops
    biased = P.copy()
    biased[i, :i + 1] *= 1.0 + 20 * SCORE_RTOL
    m_biased = oracle.select_blocks(biased, tau, 1)
    m_exact = oracle.select_blocks(P, tau, 1)
    assert (m_biased[i] != m_exact[i]).any(), "the planted bias must change the selection"
    with pytest.raises(AssertionError):
        assert_scores_within_bound(biased[i, :i + 1].astype(np.float32), P[i, :i + 1], "biased")
    with pytest.raises(AssertionError):
        mask_vs_oracle_pipeline(m_biased, P[rows], rows, tau, 1, "biased")
    # within the bound: both checks pass and no mask bit differs
    small = P.copy()
    small[i, :i + 1] *= 1.0 + 0.1 * SCORE_RTOL
    assert_scores_within_bound(small[i, :i + 1].astype(np.float32), P[i, :i + 1], "small")
    m_small = oracle.select_blocks(small, tau, 1)
    assert mask_vs_oracle_pipeline(m_small, P[rows], rows, tau, 1, "small") == 0
