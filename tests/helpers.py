"""Shared test utilities: tolerances, conversions and parity reports."""
from __future__ import annotations

import numpy as np

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
