"""Two contexts used at the same time on two streams: each owns its workspace,
merge tickets and error word, so decodes and prefills issued concurrently give
the same bits as the same calls run one after another, and an error raised in one
context is not seen by the other."""
import math

import pytest
import torch

from sparse_attention_flux_b200 import synth
from sparse_attention_flux_b200.flux import Context, FluxError, FLUX_ERR_DEVICE_CHECK

pytestmark = pytest.mark.gpu


def _inputs(dev, seed):
    B, S, Hq, Hkv, d, T = 4, 8192, 8, 2, 128, 1536
    return {
        "q": synth.torch_normal_bf16((B, Hq, d), seed + 1, dev),
        "kc": synth.torch_normal_bf16((B, S, Hkv, d), seed + 2, dev),
        "vc": synth.torch_normal_bf16((B, S, Hkv, d), seed + 3, dev),
        "sl": torch.tensor([S, 5000, 64, 8191], dtype=torch.int32, device=dev),
        "pq": synth.torch_normal_bf16((1, T, Hq, d), seed + 4, dev),
        "pk": synth.torch_normal_bf16((1, T, Hkv, d), seed + 5, dev),
        "pv": synth.torch_normal_bf16((1, T, Hkv, d), seed + 6, dev),
    }


def _calls(ctx, x, outs, stream):
    dev = x["q"].device
    nb = x["pq"].shape[1] // 128
    fa = torch.ones(1, dtype=torch.uint8, device=dev)
    sa = torch.zeros(1, dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        mask = torch.empty((nb, nb), dtype=torch.uint8, device=dev)
        rp = torch.empty(nb + 1, dtype=torch.int32, device=dev)
        col = torch.empty(nb * nb, dtype=torch.int32, device=dev)
        ctx.build_streaming_mask(nb, nb, 1, 4, mask, stream=stream)
        ctx.build_block_index(mask, rp, col, stream=stream)
        scale = 1 / math.sqrt(128)
        for i, lm in enumerate((fa, sa, fa, sa)):
            ctx.attn_decode(x["q"], x["kc"], x["vc"], x["sl"], outs[i], scale, layer_mode=lm,
                            sink_blocks=1, window_blocks=4, block=128, stream=stream)
        for i, lm in enumerate((fa, sa)):
            ctx.attn_prefill(x["pq"], x["pk"], x["pv"], outs[4 + i], scale, layer_mode=lm,
                             row_ptr=rp, col=col, block=128, stream=stream)


def _outs(x):
    return [torch.empty_like(x["q"]) for _ in range(4)] + [torch.empty_like(x["pq"]) for _ in range(2)]


def test_two_contexts_on_two_streams_match_sequential_runs():
    dev = torch.device("cuda", 0)
    xs = [_inputs(dev, 100), _inputs(dev, 200)]
    with Context(0, 64 << 20) as c0, Context(0, 64 << 20) as c1:
        ctxs = (c0, c1)
        ref = [_outs(x) for x in xs]
        s_main = torch.cuda.current_stream()
        for c, x, o in zip(ctxs, xs, ref):
            _calls(c, x, o, s_main)
            c.check()
        streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
        for s in streams:
            s.wait_stream(s_main)
        for rep in range(3):
            got = [_outs(x) for x in xs]
            for c, x, o, s in zip(ctxs, xs, got, streams):
                _calls(c, x, o, s)          # both streams in flight at once
            torch.cuda.synchronize()
            for c in ctxs:
                c.check()
            for g, r in zip(got, ref):
                for a, b in zip(g, r):
                    assert torch.equal(a, b), rep


def test_an_error_in_one_context_is_not_seen_by_another():
    dev = torch.device("cuda", 0)
    x = _inputs(dev, 300)
    bad = x["sl"].clone()
    bad[1] = 1 << 20                        # beyond S_max: a device-checked error
    with Context(0, 64 << 20) as c0, Context(0, 64 << 20) as c1:
        o0, o1 = torch.empty_like(x["q"]), torch.empty_like(x["q"])
        c0.attn_decode(x["q"], x["kc"], x["vc"], bad, o0, 0.1, sink_blocks=1, window_blocks=4,
                       block=128)
        c1.attn_decode(x["q"], x["kc"], x["vc"], x["sl"], o1, 0.1, sink_blocks=1, window_blocks=4,
                       block=128)
        c1.check()                          # clean
        with pytest.raises(FluxError) as e:
            c0.check()
        assert e.value.code == FLUX_ERR_DEVICE_CHECK
