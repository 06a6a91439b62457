"""Seeded synthetic inputs for the routed-attention hot path.

This module is shared by the tests, the benchmark and the oracle checks, and
holds none of the method's arithmetic: it only draws random numbers, rounds
them to bf16 storage and plants the needle pattern of the Qwen3-4B-shaped
prefill workload.  The pages' own workloads (LongBench-E, RULER, LongBench-V2,
math reasoning; gist.science summary section 4 "Results") are datasets that
are not available here; these seeded tensors with the models' shapes stand
in for them.

Recipes
-------
* Q/K/V, hidden states, KV caches: i.i.d. N(0, 1), drawn in fp32 and rounded
  to bf16 (round-to-nearest-even).  Small tensors come from numpy's PCG64;
  tensors too large for host generation come from torch's CUDA generator and
  are copied back to the host only where the oracle needs them.
* Needles: for each kv head g, one query row r_g ~ U[T/2, T) of query head
  g*G is chosen, and 16 distinct key positions ~ U[0, r_g] get key := 3 * q.
* Router weights: W ~ N(0, 0.1), b1 ~ N(0, 0.1); b2 either N(0, 0.1) (the
  tiny case) or +-2 from a seeded coin so that about half of the layers go
  to each mode with a wide margin.
* Seeds: 1234 + 100 * config_index + layer.
"""
from __future__ import annotations

import numpy as np

BASE_SEED = 1234


def seed_for(config_index: int, layer: int = 0, salt: int = 0) -> int:
    return BASE_SEED + 100 * config_index + layer + 7919 * salt


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16 (nearest even) and return the 16-bit patterns.

    uint32 arithmetic is exact here: a finite value's pattern plus 0x8000 stays
    below 2^32."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16_bits(shape, seed: int, std: float = 1.0) -> np.ndarray:
    x = rng(seed).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return to_bf16_bits(x)


def attention_inputs(B: int, T: int, Hq: int, Hkv: int, d: int, seed: int):
    """(q, k, v) as bf16 bit patterns: q [B,T,Hq,d], k and v [B,T,Hkv,d]."""
    q = normal_bf16_bits((B, T, Hq, d), seed)
    k = normal_bf16_bits((B, T, Hkv, d), seed + 1)
    v = normal_bf16_bits((B, T, Hkv, d), seed + 2)
    return q, k, v


def needle_positions(T: int, Hkv: int, G: int, seed: int, n_needles: int = 16):
    """Per kv head g: (query head, query row r_g, sorted distinct key positions)."""
    g_rng = rng(seed + 3)
    out = []
    for g in range(Hkv):
        r = int(g_rng.integers(T // 2, T))
        n = min(n_needles, r + 1)
        pos = np.sort(g_rng.choice(r + 1, size=n, replace=False)).astype(np.int64)
        out.append((g * G, r, pos))
    return out


def plant_needles_np(q: np.ndarray, k: np.ndarray, seed: int, n_needles: int = 16,
                     factor: float = 3.0):
    """Set the chosen keys of every kv head to factor * (the chosen query row); in place."""
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    needles = needle_positions(T, Hkv, Hq // Hkv, seed, n_needles)
    for b in range(B):
        for g, (h, r, pos) in enumerate(needles):
            row = bf16_bits_to_f32(q[b, r, h]) * np.float32(factor)
            k[b, pos, g] = to_bf16_bits(row)
    return needles


def plant_needles_torch(q, k, seed: int, n_needles: int = 16, factor: float = 3.0):
    """plant_needles_np for device tensors (bf16 [B,T,Hq,d] / [B,T,Hkv,d]): the same
    positions; key := factor * q row, multiplied in fp32 and rounded to bf16 (nearest
    even), as the host version does.  In place."""
    import torch
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    needles = needle_positions(T, Hkv, Hq // Hkv, seed, n_needles)
    for b in range(B):
        for g, (h, r, pos) in enumerate(needles):
            row = (q[b, r, h].float() * factor).to(torch.bfloat16)
            k[b, torch.from_numpy(pos).to(k.device), g] = row
    return needles


def router_inputs(T: int, Hd: int, H1: int, L: int, seed: int, coin_bias: float | None = None,
                  n_positive: int | None = None):
    """(hidden bits [T,Hd], W1 [H1,2Hd], b1 [H1], W2 [L,H1], b2 [L]) with fp32 weights.

    coin_bias=None draws b2 ~ N(0, 0.1); otherwise b2 = +-coin_bias from a
    seeded fair coin per layer, or, with n_positive given, +coin_bias on exactly
    n_positive layers chosen by a seeded permutation and -coin_bias on the rest.
    """
    hidden = normal_bf16_bits((T, Hd), seed)
    r = rng(seed + 11)
    W1 = (r.standard_normal((H1, 2 * Hd), dtype=np.float32) * np.float32(0.1))
    b1 = (r.standard_normal(H1, dtype=np.float32) * np.float32(0.1))
    W2 = (r.standard_normal((L, H1), dtype=np.float32) * np.float32(0.1))
    if coin_bias is None:
        b2 = r.standard_normal(L, dtype=np.float32) * np.float32(0.1)
    else:
        coins = r.integers(0, 2, size=L)
        if n_positive is not None:
            coins = (rng(seed + 12).permutation(L) < n_positive).astype(np.int64)
        b2 = np.where(coins == 1, np.float32(coin_bias), np.float32(-coin_bias)).astype(np.float32)
    return hidden, W1, b1, W2, b2


def layer_mode_choice(L: int, n_fa: int, seed: int) -> np.ndarray:
    """A fixed routing mask with exactly n_fa FA layers (1) chosen by a seeded permutation."""
    mode = np.zeros(L, np.uint8)
    mode[rng(seed + 13).permutation(L)[:n_fa]] = 1
    return mode


def decode_inputs(B: int, S_max: int, Hq: int, Hkv: int, d: int, seed: int):
    """(q [B,Hq,d], k_cache, v_cache [B,S_max,Hkv,d]) as bf16 bit patterns (host)."""
    q = normal_bf16_bits((B, Hq, d), seed)
    kc = normal_bf16_bits((B, S_max, Hkv, d), seed + 1)
    vc = normal_bf16_bits((B, S_max, Hkv, d), seed + 2)
    return q, kc, vc


# --- torch helpers (device-resident inputs for the large workloads) --------

def torch_from_bits(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def torch_to_bits(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def torch_normal_bf16(shape, seed: int, device, out=None):
    """N(0,1) drawn in fp32 by torch's generator on `device`, rounded to bf16.

    Fills `out` (a bf16 tensor) in chunks when given, so that tensors of tens
    of GB need no fp32 staging copy of their full size.
    """
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    chunk = 1 << 26
    for s in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - s)
        flat[s:s + n].copy_(torch.randn(n, generator=g, device=device, dtype=torch.float32))
    return out
