"""Block mask and compressed block-index list on the GPU: bit-exact against
the oracle and the hand-enumerated fixture."""

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_flux_b200 import synth
from sparse_attention_flux_b200.flux import Context

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    with Context(0) as c:
        yield c


def _gpu_mask(ctx, nqb, nkb, sink, W):
    m = torch.full((nqb, nkb), 9, dtype=torch.uint8, device=ctx.device)
    ctx.build_streaming_mask(nqb, nkb, sink, W, m)
    return m


def _gpu_csr(ctx, mask_t, cap=None):
    nqb, nkb = mask_t.shape
    cap = nqb * nkb if cap is None else cap
    rp = torch.full((nqb + 1,), -5, dtype=torch.int32, device=ctx.device)
    col = torch.full((max(cap, 1),), -7, dtype=torch.int32, device=ctx.device)
    ctx.build_block_index(mask_t, rp, col)
    return rp, col


def test_tiny_fixture(ctx):
    m = _gpu_mask(ctx, 4, 4, 1, 2)
    rp, col = _gpu_csr(ctx, m)
    ctx.check()
    assert m.cpu().numpy().tolist() == [[1, 0, 0, 0], [1, 1, 0, 0], [1, 1, 1, 0], [1, 0, 1, 1]]
    assert rp.cpu().tolist() == [0, 1, 3, 6, 9]
    assert col.cpu().tolist()[:9] == [0, 0, 1, 0, 1, 2, 0, 2, 3]


@pytest.mark.parametrize("nb,sink,W", [(256, 1, 16), (512, 1, 16), (1024, 1, 8), (1024, 1, 32),
                                       (300, 0, 1), (5, 3, 9), (1, 1, 1)])
def test_streaming_mask_and_index_match_oracle(ctx, nb, sink, W):
    m = _gpu_mask(ctx, nb, nb, sink, W)
    rp, col = _gpu_csr(ctx, m)
    ctx.check()
    mo = oracle.streaming_mask(nb, nb, sink, W)
    rpo, colo = oracle.block_index(mo)
    assert np.array_equal(m.cpu().numpy(), mo)
    assert np.array_equal(rp.cpu().numpy(), rpo)
    assert np.array_equal(col.cpu().numpy()[:colo.size], colo)


@pytest.mark.parametrize("nqb,nkb,density", [(37, 41, 0.3), (600, 333, 0.05), (3, 1000, 0.5)])
def test_random_mask_index_matches_oracle(ctx, nqb, nkb, density):
    rng = synth.rng(nqb * 1000 + nkb)
    mo = (rng.random((nqb, nkb)) < density).astype(np.uint8) * rng.integers(1, 255, (nqb, nkb),
                                                                             dtype=np.uint8)
    m = torch.from_numpy(mo).to(ctx.device)
    rp, col = _gpu_csr(ctx, m)
    ctx.check()
    rpo, colo = oracle.block_index(mo)
    assert np.array_equal(rp.cpu().numpy(), rpo)
    assert np.array_equal(col.cpu().numpy()[:colo.size], colo)


def test_capacity_overflow_is_reported_and_nothing_written_past_cap(ctx):
    from sparse_attention_flux_b200.flux import FluxError, FLUX_ERR_DEVICE_CHECK
    m = _gpu_mask(ctx, 16, 16, 1, 4)
    nnz = int(oracle.block_index(oracle.streaming_mask(16, 16, 1, 4))[0][-1])
    cap = nnz - 5
    rp = torch.zeros(17, dtype=torch.int32, device=ctx.device)
    col = torch.full((nnz,), -7, dtype=torch.int32, device=ctx.device)
    ctx.build_block_index(m, rp, col[:cap])
    with pytest.raises(FluxError) as e:
        ctx.check()
    assert e.value.code == FLUX_ERR_DEVICE_CHECK
    assert int(rp[-1]) == nnz
    assert (col[cap:] == -7).all()
    ctx.check()  # the error word was cleared
