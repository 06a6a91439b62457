"""The Python binding refuses tensors whose shapes disagree before anything reaches
the library (the C ABI takes the sizes on trust: a short k would be read past its end)."""
import pytest
import torch

from sparse_attention_flux_b200.flux import Context

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    with Context(0, 16 << 20) as c:
        yield c


def _bf16(dev, *shape):
    return torch.zeros(shape, dtype=torch.bfloat16, device=dev)


def test_select_blocks_k_shorter_than_q(ctx):
    dev = ctx.device
    q, k = _bf16(dev, 1, 512, 4, 64), _bf16(dev, 1, 256, 1, 64)
    m = torch.empty((4, 4), dtype=torch.uint8, device=dev)
    with pytest.raises(ValueError, match="inconsistent"):
        ctx.select_blocks(q, k, m, 0.125, 0.9, 1)


def test_prefill_heads_checks(ctx):
    dev = ctx.device
    q, k = _bf16(dev, 1, 256, 4, 64), _bf16(dev, 1, 256, 2, 64)
    hm = torch.ones(4, dtype=torch.uint8, device=dev)
    rp = torch.tensor([0, 1, 3], dtype=torch.int32, device=dev)
    col = torch.tensor([0, 0, 1], dtype=torch.int32, device=dev)
    with pytest.raises(ValueError, match="inconsistent"):
        ctx.attn_prefill_heads(q, k, k, _bf16(dev, 1, 128, 4, 64), 0.125, hm, rp, col)
    with pytest.raises(ValueError, match="lse"):
        ctx.attn_prefill_heads(q, k, k, torch.empty_like(q), 0.125, hm, rp, col,
                               lse=torch.empty(10, dtype=torch.float32, device=dev))
    with pytest.raises(ValueError, match="required"):
        ctx.attn_prefill_heads(q, k, k, torch.empty_like(q), 0.125, hm, None, None)


def test_decode_heads_checks(ctx):
    dev = ctx.device
    q = _bf16(dev, 2, 4, 64)
    kc = _bf16(dev, 1, 256, 2, 64)             # one sequence of cache for a batch of two
    sl = torch.tensor([10, 10], dtype=torch.int32, device=dev)
    hm = torch.ones(4, dtype=torch.uint8, device=dev)
    with pytest.raises(ValueError, match="inconsistent"):
        ctx.attn_decode_heads(q, kc, kc, sl, torch.empty_like(q), 0.125, hm)
    kc2 = _bf16(dev, 2, 256, 2, 64)
    with pytest.raises(ValueError, match="inconsistent"):
        ctx.attn_decode_heads(q, kc2, kc2, sl[:1], torch.empty_like(q), 0.125, hm)
    with pytest.raises(ValueError, match="lse"):
        ctx.attn_decode_heads(q, kc2, kc2, sl, torch.empty_like(q), 0.125, hm,
                              lse=torch.empty(3, dtype=torch.float32, device=dev))
