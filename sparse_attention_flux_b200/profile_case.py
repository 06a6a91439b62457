"""Run one hot-path kernel on one case, for profilers (ncu) and quick timing.

    python -m sparse_attention_flux_b200.profile_case prefill --mode fa --T 16384 --iters 3
    python -m sparse_attention_flux_b200.profile_case decode --mode sa --B 4 --S 32768
    python -m sparse_attention_flux_b200.profile_case decode --mode ring --B 16 --S 131072
    python -m sparse_attention_flux_b200.profile_case append --mode ring --B 16 --S 131072
    python -m sparse_attention_flux_b200.profile_case select --T 32768

Inputs are seeded N(0, 1) bf16 drawn on the device; nothing is checked here
(the test suite does that).  Prints the CUDA-event time per launch.
"""
from __future__ import annotations

import argparse
import math

import torch

from sparse_attention_flux_b200 import synth
from sparse_attention_flux_b200.flux import Context


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("kernel", choices=["prefill", "decode", "route", "append", "select"])
    ap.add_argument("--mode", choices=["fa", "sa", "ring"], default="fa",
                    help="ring: SA decode / append over the compact sink + window cache")
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--T", type=int, default=16384)
    ap.add_argument("--S", type=int, default=32768)
    ap.add_argument("--Hq", type=int, default=32)
    ap.add_argument("--Hkv", type=int, default=8)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--block", type=int, default=128)
    ap.add_argument("--sink", type=int, default=1)
    ap.add_argument("--window", type=int, default=16)
    ap.add_argument("--iters", type=int, default=3)
    args = ap.parse_args()

    dev = torch.device("cuda", 0)
    ctx = Context(0, 512 << 20)
    mode = torch.tensor([1 if args.mode == "fa" else 0], dtype=torch.uint8, device=dev)
    if args.kernel == "prefill" and args.mode == "ring":
        ap.error("--mode ring applies to decode and append")
    scale = 1.0 / math.sqrt(args.d)
    if args.kernel == "prefill":
        B, T = args.B, args.T
        q = synth.torch_normal_bf16((B, T, args.Hq, args.d), 1, dev)
        k = synth.torch_normal_bf16((B, T, args.Hkv, args.d), 2, dev)
        v = synth.torch_normal_bf16((B, T, args.Hkv, args.d), 3, dev)
        o = torch.empty_like(q)
        nb = (T + args.block - 1) // args.block
        m = torch.empty((nb, nb), dtype=torch.uint8, device=dev)
        ctx.build_streaming_mask(nb, nb, args.sink, args.window, m)
        rp = torch.empty(nb + 1, dtype=torch.int32, device=dev)
        col = torch.empty(nb * nb, dtype=torch.int32, device=dev)
        ctx.build_block_index(m, rp, col)
        run = lambda: ctx.attn_prefill(q, k, v, o, scale, layer_mode=mode, row_ptr=rp, col=col,
                                       block=args.block)
    elif args.kernel in ("decode", "append"):
        B, S = args.B, args.S
        rows = (args.sink + args.window) * args.block if args.mode == "ring" else S
        q = synth.torch_normal_bf16((B, args.Hq, args.d), 1, dev)
        kc = synth.torch_normal_bf16((B, rows, args.Hkv, args.d), 2, dev)
        vc = synth.torch_normal_bf16((B, rows, args.Hkv, args.d), 3, dev)
        sl = torch.full((B,), S, dtype=torch.int32, device=dev)
        o = torch.empty_like(q)
        if args.kernel == "append":
            nk = synth.torch_normal_bf16((B, 1, args.Hkv, args.d), 4, dev)
            nv = synth.torch_normal_bf16((B, 1, args.Hkv, args.d), 5, dev)
            ring = args.mode == "ring"
            run = lambda: ctx.kv_write(nk, nv, sl, kc, vc, args.sink if ring else 0,
                                       args.window if ring else 0, args.block)
        elif args.mode == "ring":
            run = lambda: ctx.attn_decode_sa_compact(q, kc, vc, sl, o, scale, args.sink,
                                                     args.window, args.block)
        else:
            run = lambda: ctx.attn_decode(q, kc, vc, sl, o, scale, layer_mode=mode,
                                          sink_blocks=args.sink, window_blocks=args.window,
                                          block=args.block)
    elif args.kernel == "select":
        B, T = args.B, args.T
        q = synth.torch_normal_bf16((B, T, args.Hq, args.d), 1, dev)
        k = synth.torch_normal_bf16((B, T, args.Hkv, args.d), 2, dev)
        nb = (T + 127) // 128
        m = torch.empty((nb, nb), dtype=torch.uint8, device=dev)
        run = lambda: ctx.select_blocks(q, k, m, scale, 0.9, args.sink, stride=8)
    else:
        T, Hd, H1, L = args.T, 2560, 512, 36
        hidden = synth.torch_normal_bf16((T, Hd), 1, dev)
        W1 = torch.randn(H1, 2 * Hd, device=dev) * 0.1
        b1 = torch.randn(H1, device=dev) * 0.1
        W2 = torch.randn(L, H1, device=dev) * 0.1
        b2 = torch.randn(L, device=dev) * 0.1
        lm = torch.empty(L, dtype=torch.uint8, device=dev)
        run = lambda: ctx.route(hidden, W1, b1, W2, b2, 0.5, lm)
    run()
    ctx.check()
    for _ in range(args.iters):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        run()
        b.record()
        b.synchronize()
        print(f"{args.kernel} {args.mode}: {a.elapsed_time(b):.4f} ms")
    ctx.check()
    ctx.close()


if __name__ == "__main__":
    main()
