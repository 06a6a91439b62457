"""Shared test utilities: tolerances, conversions and parity reports."""
from __future__ import annotations

import numpy as np

import oracle
from sparse_attention_flux_b200 import synth

# Attention outputs (bf16 inputs, fp32 accumulation, bf16 output) against the
# fp64 oracle: the bound the routed-attention spec states.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def bits_of(t) -> np.ndarray:
    """bf16 torch tensor (any device) -> numpy uint16 bit patterns."""
    return synth.torch_to_bits(t)


def f32_of_bits(b) -> np.ndarray:
    return synth.bf16_bits_to_f32(b).astype(np.float64)


def assert_close_attn(gpu_bf16_bits: np.ndarray, ref: np.ndarray, what: str = "",
                      max_abs: float = MAX_ABS, mean_abs: float = MEAN_ABS):
    got = f32_of_bits(gpu_bf16_bits)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    mx, mn = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert mx <= max_abs and mn <= mean_abs, f"{what}: max-abs {mx:.3e} mean-abs {mn:.3e}"
    return mx, mn


def assert_close_lse(gpu_lse: np.ndarray, ref: np.ndarray, what: str = "", tol: float = 2e-3):
    g = np.asarray(gpu_lse, np.float64)
    r = np.asarray(ref, np.float64)
    inf_g, inf_r = np.isneginf(g), np.isneginf(r)
    assert np.array_equal(inf_g, inf_r), f"{what}: -inf pattern differs"
    d = np.abs(g[~inf_g] - r[~inf_r])
    assert d.size == 0 or d.max() <= tol, f"{what}: lse max diff {d.max():.3e}"


# ---- dynamic SA block selection: the scores' bound and the mask check against the oracle
# Per-element score bound.  The GPU's logits are fp32 tensor-core sums of 8 d exact
# bf16 products, turned into per-key-block log-sum-exps with ex2/lg2 (about 2^-22
# relative each); a share P = 2^(lse_j - lse_total) then carries a relative error
# of a few logit roundings.  Measured on B200 over every case below and the full
# sizes: at most 8.2e-6 relative (6.1e-7 absolute).  The bound leaves a factor of
# about 6 above that, and an absolute floor for shares near fp32's underflow.
SCORE_RTOL = 5e-5
SCORE_ATOL = 1e-7


def score_bound(P):
    return SCORE_ATOL + SCORE_RTOL * np.abs(P)


def assert_scores_within_bound(score_row, P_row, what):
    err = np.abs(score_row.astype(np.float64) - P_row)
    bound = score_bound(P_row)
    worst = int(np.argmax(err - bound))
    assert np.all(err <= bound), (f"{what}: score error {err[worst]:.3e} at key block {worst} "
                                  f"(oracle {P_row[worst]:.6e}, bound {bound[worst]:.3e})")


def open_decisions(p, tau, sink, i):
    """For query block i with oracle scores p[0..i] (fp64): the oracle's order of the
    candidates (score descending, block ascending, as fp32 -- the selection's own
    precision) and, per candidate, the fp32 running sum before it."""
    p32 = p[:i + 1].astype(np.float32)
    forced = [j for j in range(i + 1) if j < sink or j == i]
    cand = sorted((j for j in range(i + 1) if not (j < sink or j == i)),
                  key=lambda j: (-p32[j], j))
    cum = np.float32(0)
    for j in forced:
        cum = np.float32(cum + p32[j])
    before = {}
    for j in cand:
        before[j] = float(cum)
        cum = np.float32(cum + p32[j])
    return before


def mask_vs_oracle_pipeline(mask, P_rows, rows, tau, sink, what):
    """The GPU mask against the oracle's own pipeline (oracle scores -> oracle
    selection) on the listed query blocks.  A differing bit is allowed only where
    the decision is open under the score bound: the oracle's running sum before
    that candidate within the row's summed bound of tau, or another differing
    candidate whose score is within both bounds of this one.  Returns how many
    such bits there were."""
    nb = mask.shape[1]
    full = np.zeros((nb, nb), np.float64)
    for n, i in enumerate(rows):
        full[i] = P_rows[n]
    m_or = oracle.select_blocks(full, tau, sink)
    open_bits = 0
    for n, i in enumerate(rows):
        diff = np.nonzero(m_or[i] != mask[i])[0]
        if diff.size == 0:
            continue
        p = P_rows[n]
        e = score_bound(p)
        row_bound = float(e[:i + 1].sum())
        before = open_decisions(p, tau, sink, i)
        for j in diff:
            near_tau = j in before and abs(before[j] - tau) <= row_bound
            near_tie = any(j2 != j and abs(p[j] - p[j2]) <= e[j] + e[j2] for j2 in diff)
            assert near_tau or near_tie, (f"{what}: query block {i}, key block {j}: GPU mask "
                                          f"{mask[i, j]} vs oracle {m_or[i, j]} with the decision "
                                          f"not open under the score bound")
            open_bits += 1
    return open_bits
