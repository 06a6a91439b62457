"""The routed path can be captured in a CUDA graph and replayed: router, block index,
FA/SA prefill, KV appends and decode (full cache and ring) give the same bits replayed
as run eagerly, and per-step inputs (seqlens) are read at replay time."""
import math

import pytest
import torch

from sparse_attention_flux_b200 import synth
from sparse_attention_flux_b200.flux import Context

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fused", [False, True])
def test_routed_step_graph_replay_matches_eager(fused):
    """fused: the decodes append the step's token themselves (flux_attn_decode_append)."""
    dev = torch.device("cuda", 0)
    T, Hq, Hkv, d, blk = 1024, 8, 2, 128, 128
    B, S_max = 2, 3000
    with Context(0, 64 << 20) as ctx:
        hidden, W1, b1, W2, b2 = synth.router_inputs(T, 64, 32, 2, 8, coin_bias=4.0)
        b2[:] = [4.0, -4.0]
        hid = synth.torch_from_bits(hidden).to(dev)
        w = [torch.from_numpy(x).to(dev) for x in (W1, b1, W2, b2)]
        q = synth.torch_normal_bf16((1, T, Hq, d), 1, dev)
        k = synth.torch_normal_bf16((1, T, Hkv, d), 2, dev)
        v = synth.torch_normal_bf16((1, T, Hkv, d), 3, dev)
        kc = synth.torch_normal_bf16((B, S_max, Hkv, d), 4, dev)
        vc = synth.torch_normal_bf16((B, S_max, Hkv, d), 5, dev)
        kr = synth.torch_normal_bf16((B, 17 * blk, Hkv, d), 6, dev)
        vr = synth.torch_normal_bf16((B, 17 * blk, Hkv, d), 7, dev)
        qd = synth.torch_normal_bf16((B, Hq, d), 8, dev)
        nk = synth.torch_normal_bf16((B, 1, Hkv, d), 9, dev)
        nv = synth.torch_normal_bf16((B, 1, Hkv, d), 10, dev)
        nb = T // blk
        mode = torch.empty(2, dtype=torch.uint8, device=dev)
        mask = torch.empty((nb, nb), dtype=torch.uint8, device=dev)
        rp = torch.empty(nb + 1, dtype=torch.int32, device=dev)
        col = torch.empty(nb * nb, dtype=torch.int32, device=dev)
        sl = torch.empty(B, dtype=torch.int32, device=dev)
        outs = [torch.empty_like(q), torch.empty_like(q), torch.empty_like(qd), torch.empty_like(qd)]

        def step():
            ctx.route(hid, *w, 0.5, mode)
            ctx.build_streaming_mask(nb, nb, 1, 16, mask)
            ctx.build_block_index(mask, rp, col)
            for layer in (0, 1):
                ctx.attn_prefill(q, k, v, outs[layer], 1 / math.sqrt(d), layer_mode=mode,
                                 layer=layer, row_ptr=rp, col=col, block=blk)
            if fused:
                ctx.attn_decode_append(qd, nk, nv, kc, vc, sl, outs[2], 1 / math.sqrt(d),
                                       layer_mode=mode, layer=0, sink_blocks=1, window_blocks=16,
                                       block=blk)
                ctx.attn_decode_append(qd, nk, nv, kr, vr, sl, outs[3], 1 / math.sqrt(d),
                                       sink_blocks=1, window_blocks=16, block=blk, compact=True)
            else:
                ctx.kv_write(nk, nv, sl, kc, vc)
                ctx.attn_decode(qd, kc, vc, sl, outs[2], 1 / math.sqrt(d), layer_mode=mode,
                                layer=0, sink_blocks=1, window_blocks=16, block=blk)
                ctx.kv_write(nk, nv, sl, kr, vr, 1, 16, blk)
                ctx.attn_decode_sa_compact(qd, kr, vr, sl, outs[3], 1 / math.sqrt(d), 1, 16, blk)

        # The caches are state (appends; the ring reuses slots), so every run starts from
        # the same contents.
        initial = [x.clone() for x in (kc, vc, kr, vr)]

        def reset():
            for x, x0 in zip((kc, vc, kr, vr), initial):
                x.copy_(x0)

        results = {}
        for s_val in (2500, 2999):
            reset()
            sl.fill_(s_val)
            step()
            ctx.check()
            results[s_val] = [o.clone() for o in outs] + [x.clone() for x in (kc, vc, kr, vr)]

        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(dev)
        cs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(g, stream=cs):
            step()
        torch.cuda.current_stream().wait_stream(cs)
        for s_val in (2500, 2999):          # seqlens are read at replay time
            reset()
            sl.fill_(s_val)
            for o in outs:
                o.fill_(float("nan"))
            g.replay()
            torch.cuda.synchronize()
            ctx.check()
            for got, want in zip(outs + [kc, vc, kr, vr], results[s_val]):
                assert torch.equal(got, want), s_val
        del g
