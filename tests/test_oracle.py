"""Pins for the oracle: each check ties it to something other than itself.

* closed forms and hand-enumerated fixtures (tests/golden/, each citing the
  passage it is derived from);
* a library routine: torch's scaled_dot_product_attention in fp64 with an
  explicit boolean mask built from the mask definition;
* invariants the mathematics fixes (rows of P sum to one, masked entries are
  exactly zero, SA with a window covering everything is FA, q = 0 gives the
  mean of the allowed values, decode equals the last prefill row, ...).
A dropped term, a wrong sign or index, or a transposed operand anywhere in
the oracle breaks at least one of these.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_flux_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        lines = [ln.split("#")[0].strip() for ln in f]
    lines = [ln for ln in lines if ln]
    i = 0
    out = []
    while i < len(lines):
        out.append(lines[i].split())
        i += 1
    for parts in out:
        rows.setdefault(parts[0], []).append(parts[1:])
    return rows, out


# --------------------------------------------------------------------------- router

def test_pool_closed_form():
    g, _ = _golden("router_closed_form.txt")
    scale = np.array([1.0, 0.5, -1.0, 0.25], np.float32)
    for T, n, head_f, tail_f in g["pool"]:
        T, n, head_f, tail_f = int(T), int(n), float(head_f), float(tail_f)
        h = (np.arange(1, T + 1, dtype=np.float32)[:, None] * scale[None, :])
        bits = synth.to_bf16_bits(h)
        assert np.array_equal(synth.bf16_bits_to_f32(bits), h), "fixture must be exact in bf16"
        p = oracle.pool(bits, 100)
        np.testing.assert_allclose(p[:4], head_f * scale, rtol=0, atol=1e-12)
        np.testing.assert_allclose(p[4:], tail_f * scale, rtol=0, atol=1e-12)


def test_mlp_hand_values():
    g, _ = _golden("router_closed_form.txt")
    f = lambda k: np.array([float(x) for x in g[k][0]])
    p = f("mlp_p")
    W1 = f("mlp_W1").reshape(3, 4).astype(np.float32)
    W2 = f("mlp_W2").reshape(2, 3).astype(np.float32)
    z = oracle.mlp(p, W1, f("mlp_b1"), W2, f("mlp_b2"))
    np.testing.assert_allclose(z, f("mlp_z"), rtol=0, atol=1e-12)


def test_threshold_hand_values():
    g, _ = _golden("router_closed_form.txt")
    for z, thr, want in g["thr"]:
        mode, r = oracle.threshold(np.array([float(z)]), float(thr))
        assert int(mode[0]) == int(want), (z, thr)
        assert abs(r[0] - 1.0 / (1.0 + math.exp(-float(z)))) < 1e-15


def test_route_composes_pool_mlp_threshold():
    hidden, W1, b1, W2, b2 = synth.router_inputs(256, 64, 32, 4, synth.seed_for(0))
    mode, z, r = oracle.route(hidden, W1, b1, W2, b2, 0.5)
    p = oracle.pool(hidden, 100)
    z2 = oracle.mlp(p, W1, b1, W2, b2)
    assert np.array_equal(z, z2)
    m2, _ = oracle.threshold(z2, 0.5)
    assert np.array_equal(mode, m2)
    # the pooled vector equals the plain means of the two windows
    hf = synth.bf16_bits_to_f32(hidden).astype(np.float64)
    np.testing.assert_allclose(p, np.concatenate([hf[:100].mean(0), hf[-100:].mean(0)]),
                               rtol=0, atol=1e-12)


def test_relu_zeroes_negative_hidden_units():
    # W1 p + b1 < 0 for every unit -> u = 0 -> z = b2 exactly.
    p = np.ones(4)
    W1 = -np.ones((5, 4), np.float32)
    b1 = np.zeros(5, np.float32)
    W2 = np.arange(10, dtype=np.float32).reshape(2, 5)
    b2 = np.array([0.125, -3.5], np.float32)
    assert np.array_equal(oracle.mlp(p, W1, b1, W2, b2), b2.astype(np.float64))


# --------------------------------------------------------------------------- mask / CSR

def test_tiny_mask_and_block_index_golden():
    g, _ = _golden("tiny_block_index.txt")
    nqb, nkb = int(g["nqb"][0][0]), int(g["nkb"][0][0])
    sink, W = int(g["sink"][0][0]), int(g["window"][0][0])
    mask_rows = [r for r in _golden("tiny_block_index.txt")[1] if r[0] in ("0", "1")]
    want_mask = np.array([[int(x) for x in r] for r in mask_rows], np.uint8)
    m = oracle.streaming_mask(nqb, nkb, sink, W)
    assert np.array_equal(m, want_mask)
    rp, col = oracle.block_index(m)
    assert rp.tolist() == [int(x) for x in g["row_ptr"][0]]
    assert col.tolist() == [int(x) for x in g["col"][0]]


@pytest.mark.parametrize("nb,sink,W", [(1, 1, 1), (7, 0, 1), (16, 1, 16), (256, 1, 16), (33, 2, 5),
                                       (10, 3, 20)])
def test_block_index_count_formula(nb, sink, W):
    m = oracle.streaming_mask(nb, nb, sink, W)
    rp, col = oracle.block_index(m)
    # row i keeps |{j <= i : j < sink or j >= i-W+1}| = min(i+1, sink) + |[max(sink, i-W+1), i]|
    want = [min(i + 1, sink) + max(0, i - max(sink, i - W + 1) + 1) for i in range(nb)]
    assert np.diff(rp).tolist() == want
    for i in range(nb):
        row = col[rp[i]:rp[i + 1]]
        assert np.all(np.diff(row) > 0)
        assert set(row.tolist()) == {j for j in range(i + 1) if j < sink or j >= i - W + 1}


# --------------------------------------------------------------------------- attention

def _token_mask(T, block_mask, block):
    t = np.arange(T)[:, None]
    u = np.arange(T)[None, :]
    allowed = u <= t
    if block_mask is not None:
        allowed &= block_mask[t // block, u // block].astype(bool)
    return allowed


def _sdpa_reference(q, k, v, scale, allowed):
    """torch's SDPA (library routine) in fp64 over an explicit boolean mask."""
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    f = lambda x: torch.from_numpy(synth.bf16_bits_to_f32(x).astype(np.float64))
    Q = f(q).permute(0, 2, 1, 3)
    K = f(k).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, dim=1)
    V = f(v).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, dim=1)
    M = torch.from_numpy(allowed)
    O = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=M, scale=scale)
    return O.permute(0, 2, 1, 3).numpy()


CASES = [  # (B, T, Hq, Hkv, d, block, sink, W)
    (1, 1, 1, 1, 16, 16, 1, 1),
    (1, 63, 2, 1, 16, 16, 1, 2),
    (1, 64, 4, 2, 32, 16, 1, 2),
    (2, 65, 2, 1, 16, 16, 0, 2),
    (1, 256, 2, 1, 64, 64, 1, 2),
    (1, 200, 4, 4, 32, 32, 2, 3),
]


@pytest.mark.parametrize("case", CASES)
def test_prefill_matches_library_sdpa(case):
    B, T, Hq, Hkv, d, block, sink, W = case
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=99 + T)
    scale = 1.0 / math.sqrt(d)
    nb = (T + block - 1) // block
    fa, _ = oracle.attn_prefill(q, k, v, scale)
    np.testing.assert_allclose(fa, _sdpa_reference(q, k, v, scale, _token_mask(T, None, block)),
                               rtol=0, atol=1e-12)
    m = oracle.streaming_mask(nb, nb, sink, W)
    sa, _ = oracle.attn_prefill(q, k, v, scale, block_mask=m, block=block)
    np.testing.assert_allclose(sa, _sdpa_reference(q, k, v, scale, _token_mask(T, m, block)),
                               rtol=0, atol=1e-12)


def test_lse_matches_logsumexp():
    B, T, Hq, Hkv, d = 1, 70, 2, 1, 16
    q, k, _ = synth.attention_inputs(B, T, Hq, Hkv, d, seed=5)
    v = k.copy()
    scale = 0.3
    _, lse = oracle.attn_prefill(q, k, v, scale)
    Q = synth.bf16_bits_to_f32(q).astype(np.float64)
    K = synth.bf16_bits_to_f32(k).astype(np.float64)
    for h in range(Hq):
        S = scale * Q[0, :, h] @ K[0, :, 0].T
        S[np.triu_indices(T, 1)] = -np.inf
        want = torch.logsumexp(torch.from_numpy(S), dim=1).numpy()
        np.testing.assert_allclose(lse[0, :, h], want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("sparse", [False, True])
def test_probability_rows_sum_to_one_and_masked_are_zero(sparse):
    B, T, Hq, Hkv, d, block = 1, 96, 2, 1, 16, 16
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=21)
    nb = T // block
    m = oracle.streaming_mask(nb, nb, 1, 2) if sparse else None
    allowed = _token_mask(T, m, block)
    for h in range(Hq):
        P = oracle.attn_probs(q, k, 0.25, 0, h, block_mask=m, block=block)
        np.testing.assert_allclose(P.sum(1), np.ones(T), rtol=0, atol=1e-12)
        assert np.all(P[~allowed] == 0.0)
        assert np.all(P[allowed] > 0.0)
        o, _ = oracle.attn_prefill(q, k, v, 0.25, block_mask=m, block=block)
        V = synth.bf16_bits_to_f32(v[0, :, h * Hkv // Hq]).astype(np.float64)
        np.testing.assert_allclose(o[0, :, h], P @ V, rtol=0, atol=1e-12)


def test_sa_with_window_covering_all_blocks_is_fa_exactly():
    B, T, Hq, Hkv, d, block = 1, 130, 4, 2, 16, 32
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=3)
    nb = (T + block - 1) // block
    fa, lfa = oracle.attn_prefill(q, k, v, 0.2)
    for sink, W in [(0, nb), (1, nb + 3), (nb, 1)]:
        m = oracle.streaming_mask(nb, nb, sink, W)
        sa, lsa = oracle.attn_prefill(q, k, v, 0.2, block_mask=m, block=block)
        assert np.array_equal(fa, sa) and np.array_equal(lfa, lsa)


def test_zero_query_gives_mean_of_allowed_values():
    B, T, Hq, Hkv, d, block = 1, 100, 2, 1, 8, 16
    q, k, _ = synth.attention_inputs(B, T, Hq, Hkv, d, seed=8)
    q[:] = 0
    # v[u] = u in every channel (exact in bf16 for u <= 256): o = mean of allowed positions
    v = synth.to_bf16_bits(np.broadcast_to(np.arange(T, dtype=np.float32)[None, :, None, None],
                                           (B, T, Hkv, d)).copy())
    nb = (T + block - 1) // block
    m = oracle.streaming_mask(nb, nb, 1, 2)
    allowed = _token_mask(T, m, block)
    o, lse = oracle.attn_prefill(q, k, v, 1.0, block_mask=m, block=block)
    for t in range(T):
        keys = np.nonzero(allowed[t])[0]
        np.testing.assert_allclose(o[0, t, :, :], keys.mean(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[0, t, :], math.log(len(keys)), rtol=0, atol=1e-12)


def test_constant_values_give_constant_output():
    B, T, Hq, Hkv, d = 1, 50, 2, 2, 8
    q, k, _ = synth.attention_inputs(B, T, Hq, Hkv, d, seed=9)
    v = np.full((B, T, Hkv, d), synth.to_bf16_bits(np.array([-1.75], np.float32))[0], np.uint16)
    o, _ = oracle.attn_prefill(q, k, v, 0.5)
    np.testing.assert_allclose(o, -1.75, rtol=0, atol=1e-12)


def test_gqa_equals_mha_with_repeated_kv_heads():
    B, T, Hq, Hkv, d = 1, 40, 4, 2, 16
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=10)
    o_gqa, _ = oracle.attn_prefill(q, k, v, 0.25)
    k_rep = np.repeat(k, Hq // Hkv, axis=2)
    v_rep = np.repeat(v, Hq // Hkv, axis=2)
    o_mha, _ = oracle.attn_prefill(q, k_rep, v_rep, 0.25)
    assert np.array_equal(o_gqa, o_mha)
    # a transposed head mapping (h % Hkv instead of h // G) would differ
    k_bad = np.tile(k, (1, 1, Hq // Hkv, 1))
    v_bad = np.tile(v, (1, 1, Hq // Hkv, 1))
    o_bad, _ = oracle.attn_prefill(q, k_bad, v_bad, 0.25)
    assert not np.allclose(o_gqa, o_bad)


def test_selected_rows_equal_full_run():
    B, T, Hq, Hkv, d, block = 2, 80, 2, 1, 16, 16
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=12)
    m = oracle.streaming_mask(5, 5, 1, 2)
    o, lse = oracle.attn_prefill(q, k, v, 0.3, block_mask=m, block=block)
    rows = np.array([[1, 1, 79], [0, 0, 0], [1, 0, 33], [0, 1, 64]], np.int32)
    o_r, l_r = oracle.attn_prefill(q, k, v, 0.3, block_mask=m, block=block, rows=rows)
    for i, (b, h, t) in enumerate(rows):
        assert np.array_equal(o_r[i], o[b, t, h]) and l_r[i] == lse[b, t, h]


# --------------------------------------------------------------------------- decode

@pytest.mark.parametrize("s,block,sink,W", [(1, 16, 1, 2), (37, 16, 1, 2), (64, 16, 1, 2),
                                            (97, 16, 2, 3), (160, 32, 1, 16), (130, 64, 0, 1)])
def test_decode_equals_last_prefill_row(s, block, sink, W):
    B, Hq, Hkv, d = 2, 4, 2, 16
    S_max = s + 5
    q, k, v = synth.attention_inputs(B, S_max, Hq, Hkv, d, seed=40 + s)
    nb = (s + block - 1) // block
    m = oracle.streaming_mask(nb, nb, sink, W)
    fa_p, fa_l = oracle.attn_prefill(q[:, :s], k[:, :s], v[:, :s], 0.25)
    sa_p, sa_l = oracle.attn_prefill(q[:, :s], k[:, :s], v[:, :s], 0.25, block_mask=m, block=block)
    seqlens = np.full(B, s, np.int32)
    qd = np.ascontiguousarray(q[:, s - 1])
    fa_d, fa_dl = oracle.attn_decode(qd, k, v, seqlens, 0.25, 1, sink, W, block)
    sa_d, sa_dl = oracle.attn_decode(qd, k, v, seqlens, 0.25, 0, sink, W, block)
    np.testing.assert_allclose(fa_d, fa_p[:, s - 1], rtol=0, atol=1e-12)
    np.testing.assert_allclose(sa_d, sa_p[:, s - 1], rtol=0, atol=1e-12)
    np.testing.assert_allclose(fa_dl, fa_l[:, s - 1], rtol=0, atol=1e-12)
    np.testing.assert_allclose(sa_dl, sa_l[:, s - 1], rtol=0, atol=1e-12)


def test_decode_sa_reads_only_sink_and_window_tokens():
    B, Hq, Hkv, d, block, sink, W = 3, 2, 1, 8, 16, 1, 2
    S_max = 200
    seqlens = np.array([200, 33, 5], np.int32)
    q = np.zeros((B, Hq, d), np.uint16)  # q = 0: o = mean of the allowed positions
    pos = np.broadcast_to(np.arange(S_max, dtype=np.float32)[None, :, None, None],
                          (B, S_max, Hkv, d)).copy()
    v = synth.to_bf16_bits(pos)
    k = synth.normal_bf16_bits((B, S_max, Hkv, d), 1)
    o, lse = oracle.attn_decode(q, k, v, seqlens, 1.0, 0, sink, W, block)
    for b, s in enumerate(seqlens):
        nbs = -(-s // block)
        keys = [u for u in range(s) if u // block < sink or u // block >= nbs - W]
        np.testing.assert_allclose(o[b], np.mean(keys), rtol=0, atol=1e-9)
        np.testing.assert_allclose(lse[b], math.log(len(keys)), rtol=0, atol=1e-12)
    # history beyond the window never matters: poison it and nothing changes
    k2, v2 = k.copy(), v.copy()
    for b, s in enumerate(seqlens):
        nbs = -(-s // block)
        for u in range(s):
            if not (u // block < sink or u // block >= nbs - W):
                k2[b, u] = synth.to_bf16_bits(np.full(d, 1e4, np.float32))
                v2[b, u] = synth.to_bf16_bits(np.full(d, -1e4, np.float32))
        k2[b, s:] = synth.to_bf16_bits(np.full((S_max - s, Hkv, d), 7.0, np.float32))
    q3 = synth.normal_bf16_bits((B, Hq, d), 2)
    a, _ = oracle.attn_decode(q3, k, v, seqlens, 0.5, 0, sink, W, block)
    b_, _ = oracle.attn_decode(q3, k2, v2, seqlens, 0.5, 0, sink, W, block)
    assert np.array_equal(a, b_)


def test_needle_query_concentrates_on_needles():
    # A query whose scaled copy appears 16 times among the keys puts nearly all
    # probability there; o is then close to the mean of those value rows.
    B, T, Hq, Hkv, d = 1, 512, 4, 2, 64
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=77)
    needles = synth.plant_needles_np(q, k, seed=77)
    scale = 1.0 / math.sqrt(d)
    rows = np.array([[0, h, r] for (h, r, _) in needles], np.int32)
    o, _ = oracle.attn_prefill(q, k, v, scale, rows=rows)
    V = synth.bf16_bits_to_f32(v).astype(np.float64)
    for i, (h, r, pos) in enumerate(needles):
        target = V[0, pos, h // (Hq // Hkv)].mean(0)
        assert np.abs(o[i] - target).max() < 0.05


def test_soft_blend_reduces_to_fa_and_sa_and_is_convex():
    # r = 1 and r = 0 give FA and SA exactly; any r lies on the segment between them.
    B, T, Hq, Hkv, d, block = 1, 160, 2, 1, 16, 32
    q, k, v = synth.attention_inputs(B, T, Hq, Hkv, d, seed=61)
    m = oracle.streaming_mask(5, 5, 1, 2)
    fa, _ = oracle.attn_prefill(q, k, v, 0.25)
    sa, _ = oracle.attn_prefill(q, k, v, 0.25, block_mask=m, block=block)
    assert np.array_equal(oracle.attn_prefill_soft(q, k, v, 0.25, 1.0, m, block), fa)
    assert np.array_equal(oracle.attn_prefill_soft(q, k, v, 0.25, 0.0, m, block), sa)
    mid = oracle.attn_prefill_soft(q, k, v, 0.25, 0.3, m, block)
    np.testing.assert_allclose(mid, 0.3 * fa + 0.7 * sa, rtol=0, atol=1e-15)
    # rows where the SA mask keeps every key (the first W blocks) are unchanged by r
    np.testing.assert_allclose(mid[0, :64], fa[0, :64], rtol=0, atol=1e-15)
