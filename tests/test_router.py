"""Layer Router on the GPU against the oracle: routing bits bit-exact, scores
within fp32 rounding of the fp64 sigmoid."""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_flux_b200 import synth
from sparse_attention_flux_b200.flux import Context, FluxError

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    with Context(0, 256 << 20) as c:
        yield c


def _run(ctx, hidden, W1, b1, W2, b2, thresh, n_pool=100):
    dev = ctx.device
    L = W2.shape[0]
    mode = torch.full((L,), 7, dtype=torch.uint8, device=dev)
    score = torch.empty(L, dtype=torch.float32, device=dev)
    ctx.route(synth.torch_from_bits(hidden).to(dev), torch.from_numpy(W1).to(dev),
              torch.from_numpy(b1).to(dev), torch.from_numpy(W2).to(dev),
              torch.from_numpy(b2).to(dev), thresh, mode, score, n_pool=n_pool)
    ctx.check()
    return mode.cpu().numpy(), score.cpu().numpy()


@pytest.mark.parametrize("T,Hd,H1,L,bias", [
    (256, 64, 32, 4, None),        # the tiny oracle case
    (150, 64, 32, 4, None),        # the two 100-token windows overlap
    (50, 64, 32, 4, None),         # fewer than 100 tokens
    (1, 16, 8, 3, None),
    (300, 36, 20, 5, 2.0),         # Hd not a multiple of 8
    (4096, 2560, 512, 36, 2.0),
])
def test_route_matches_oracle(ctx, T, Hd, H1, L, bias):
    hidden, W1, b1, W2, b2 = synth.router_inputs(T, Hd, H1, L, synth.seed_for(0, salt=T),
                                                 coin_bias=bias)
    mode_o, z, r = oracle.route(hidden, W1, b1, W2, b2, 0.5)
    mode_g, score_g = _run(ctx, hidden, W1, b1, W2, b2, 0.5)
    assert np.array_equal(mode_g, mode_o), (mode_g, mode_o, z)
    np.testing.assert_allclose(score_g, r, rtol=0, atol=2e-6)
    assert np.abs(z).min() > 1e-5  # decisions had a margin above fp32 rounding


def test_route_qwen3_4b_router_workload(ctx):
    """36-layer Qwen3-4B-shaped router: hidden 65536 x 2560, MLP 5120 -> 512 -> 36."""
    hidden, W1, b1, W2, b2 = synth.router_inputs(65536, 2560, 512, 36, synth.seed_for(2),
                                                 coin_bias=2.0)
    mode_o, z, r = oracle.route(hidden, W1, b1, W2, b2, 0.5)
    mode_g, score_g = _run(ctx, hidden, W1, b1, W2, b2, 0.5)
    assert np.array_equal(mode_g, mode_o)
    np.testing.assert_allclose(score_g, r, rtol=0, atol=2e-6)
    assert 8 <= int(mode_o.sum()) <= 28       # about half the layers go to each mode
    # The +-2 coin biases keep every logit far from the threshold's fp32 rounding gap
    # (|z| ~ 1e-6 would be needed for fp32 and fp64 to disagree).
    assert np.abs(z).min() > 0.05, np.abs(z).min()


def test_route_threshold_and_tie(ctx):
    # W2 = 0 -> z = b2 exactly; sigmoid(0) = 0.5 is a tie and goes to SA.
    hidden = synth.normal_bf16_bits((64, 16), 3)
    W1 = np.ones((4, 32), np.float32)
    b1 = np.zeros(4, np.float32)
    W2 = np.zeros((5, 4), np.float32)
    b2 = np.array([0.0, 1e-3, -1e-3, 3.0, -3.0], np.float32)
    mode_g, score_g = _run(ctx, hidden, W1, b1, W2, b2, 0.5)
    assert mode_g.tolist() == [0, 1, 0, 1, 0]
    mode_o, _, _ = oracle.route(hidden, W1, b1, W2, b2, 0.5)
    assert np.array_equal(mode_g, mode_o)


def test_route_rejects_bad_threshold(ctx):
    hidden, W1, b1, W2, b2 = synth.router_inputs(64, 16, 8, 2, 5)
    with pytest.raises(FluxError):
        _run(ctx, hidden, W1, b1, W2, b2, float("nan"))


def test_route_twice_in_a_row_is_stable(ctx):
    hidden, W1, b1, W2, b2 = synth.router_inputs(512, 64, 32, 6, 17)
    a = _run(ctx, hidden, W1, b1, W2, b2, 0.5)
    b = _run(ctx, hidden, W1, b1, W2, b2, 0.5)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("T,Hd,H1,L,n_pool", [
    (4096, 64, 32, 4, 104),        # the most rows whose loads the pool issues at once
    (4096, 64, 32, 4, 105),        # one more: the pool's row loop
    (4096, 256, 64, 6, 400),       # a wider pooling window than the pages' 100
    (333, 17, 7, 3, 100),          # odd Hd: scalar pool and W1 dot; H1 % 4 != 0: scalar W2
    (333, 17, 8, 3, 100),          # odd Hd with float4 W2: hidden1 after 34 pooled floats
    (512, 3072, 36, 5, 100),       # in_dim 6144: W1 streamed rather than held ahead
    (512, 2562, 130, 9, 100),      # in_dim 5124: just past the held W1 slice
])
def test_route_every_kernel_path(ctx, T, Hd, H1, L, n_pool):
    hidden, W1, b1, W2, b2 = synth.router_inputs(T, Hd, H1, L, synth.seed_for(0, salt=Hd + n_pool),
                                                 coin_bias=2.0)
    mode_o, z, r = oracle.route(hidden, W1, b1, W2, b2, 0.5, n_pool=n_pool)
    mode_g, score_g = _run(ctx, hidden, W1, b1, W2, b2, 0.5, n_pool=n_pool)
    assert np.array_equal(mode_g, mode_o), (mode_g, mode_o, z)
    np.testing.assert_allclose(score_g, r, rtol=0, atol=2e-6)
    assert np.abs(z).min() > 1e-5


def test_route_rejects_misaligned_weights(ctx):
    """W1 and W2 are read in 16-byte vectors; a view 4 bytes off is refused on the host."""
    hidden, W1, b1, W2, b2 = synth.router_inputs(64, 16, 8, 2, 5)
    dev = ctx.device
    mode = torch.zeros(2, dtype=torch.uint8, device=dev)
    args = dict(hidden=synth.torch_from_bits(hidden).to(dev), W1=torch.from_numpy(W1).to(dev),
                b1=torch.from_numpy(b1).to(dev), W2=torch.from_numpy(W2).to(dev),
                b2=torch.from_numpy(b2).to(dev))
    for name in ("W1", "W2"):
        t = args[name]
        off = torch.empty(t.numel() + 1, dtype=torch.float32, device=dev)[1:].view(t.shape)
        off.copy_(t)
        bad = dict(args, **{name: off})
        with pytest.raises(FluxError):
            ctx.route(bad["hidden"], bad["W1"], bad["b1"], bad["W2"], bad["b2"], 0.5, mode)
    ctx.check()
