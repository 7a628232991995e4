"""One decode layer of a chosen shape, for timing sweeps and ncu captures.

  python -m compressed_decode_attention_kvk_b200.profile_case --d 512 --b 16 --heads 40 \\
      --batch 32 --tokens 8192 --iters 20 [--path tensor|cuda_core] [--ctas N] [--op write]

Fills one anchor layer's cache through kvk_quant_write with seeded N(0,1) bf16 data, then
runs kvk_mla_decode `iters` times and prints the mean device time per call (CUDA events on
the launching stream, after warm-up) and the algorithmic bytes per second
(batch * tokens * (row_bytes + 2) per call; b = 0, the uncompressed bf16 anchor, reads no
scales).  At the default shape the cache is ~300 MB,
larger than the 126 MB L2.

--op write times the quantise-on-write of the whole cache instead (a prefill of batch x
tokens tokens): algorithmic bytes per call = batch * tokens * ((d + d_rope) * 2 read from
the bf16 inputs + row_bytes + 2 written).

--op absorb times the two absorbed projections of a decode step on the tensor cores
(kvk_absorb): the query side q_lat[b, h] = q_nope[b, h] . W_UK[h] (K = --nope, n = r) and the
output side o[b, h] = out_lat[b, h] . W_UV[h] (K = r, n = --nope), bf16 weights, fp32
activations; algorithmic bytes = weights + activations read + outputs written.
"""
from __future__ import annotations

import argparse
import json
import math

import torch


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--d", type=int, default=512)
    ap.add_argument("--b", type=int, default=16)
    ap.add_argument("--r", type=int, default=512)
    ap.add_argument("--d-rope", type=int, default=64)
    ap.add_argument("--heads", type=int, default=40)
    ap.add_argument("--batch", type=int, default=32)
    ap.add_argument("--tokens", type=int, default=8192)
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--path", default="auto", choices=["auto", "tensor", "cuda_core"])
    ap.add_argument("--ctas", type=int, default=0)
    ap.add_argument("--op", default="decode", choices=["decode", "write", "absorb"])
    ap.add_argument("--nope", type=int, default=128, help="per-head no-RoPE width (absorb)")
    args = ap.parse_args()

    from . import build as kb
    kb.build()
    from . import kvk

    dev = torch.device("cuda")
    B, T, H = args.batch, args.tokens, args.heads
    if args.op == "absorb":
        g = torch.Generator(device=dev)
        g.manual_seed(2)
        res = []
        for name, K, n in (("q_side", args.nope, args.r), ("o_side", args.r, args.nope)):
            x = torch.randn(B, H, K, generator=g, device=dev)
            w = (torch.randn(H, K, n, generator=g, device=dev) / math.sqrt(K)).to(torch.bfloat16)
            y = torch.empty(B, H, n, device=dev)
            for _ in range(args.warmup):
                kvk.kvk_absorb(x, w, y)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(args.iters):
                kvk.kvk_absorb(x, w, y)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / args.iters
            nbytes = H * K * n * 2 + B * H * (K + n) * 4
            flops = 2 * B * H * K * n
            res.append({"side": name, "K": K, "n": n, "ms_per_call": round(ms, 5),
                        "bytes_per_call": nbytes, "GBps": round(nbytes / ms / 1e6, 1),
                        "TFLOPs": round(flops / ms / 1e9, 3)})
        print(json.dumps({"op": "absorb", "batch": B, "heads": H, "results": res}))
        return
    lay = kvk.Layout([0], [args.d], [args.b], args.r, args.d_rope, B, T, device=dev)
    lay.set_decode_path({"auto": 0, "tensor": 1, "cuda_core": 2}[args.path])
    lay.set_decode_ctas(args.ctas)
    g = torch.Generator(device=dev)
    g.manual_seed(1)
    zero = torch.zeros(B, dtype=torch.int32, device=dev)
    c = torch.randn(B, T, args.r, generator=g, device=dev).to(torch.bfloat16)
    kr = torch.randn(B, T, args.d_rope, generator=g, device=dev).to(torch.bfloat16)
    lay.quant_write(0, c, kr, zero)
    if args.op == "write":
        for _ in range(args.warmup):
            lay.quant_write(0, c, kr, zero)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.iters):
            lay.quant_write(0, c, kr, zero)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / args.iters
        row = lay.layer_info(0)["row_bytes"]
        nbytes = B * T * ((args.d + args.d_rope) * 2 + row + 2)
        print(json.dumps({"op": "write", "d": args.d, "b": args.b, "batch": B, "tokens": T,
                          "ms_per_call": round(ms, 5), "bytes_per_call": nbytes,
                          "GBps": round(nbytes / ms / 1e6, 1), "status": lay.read_status()}))
        lay.close()
        return
    del c, kr
    ql = torch.randn(B, H, args.r, generator=g, device=dev).to(torch.bfloat16)
    qr = torch.randn(B, H, args.d_rope, generator=g, device=dev).to(torch.bfloat16)
    lens = torch.full((B,), T, dtype=torch.int32, device=dev)
    out = torch.empty(B, H, args.d, dtype=torch.float32, device=dev)
    ws = lay.new_workspace(0, B, H)
    sigma = 1.0 / math.sqrt(args.d + args.d_rope)
    for _ in range(args.warmup):
        kvk.kvk_mla_decode(lay.handle, 0, ql, qr, lens, sigma, out, ws)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.iters):
        kvk.kvk_mla_decode(lay.handle, 0, ql, qr, lens, sigma, out, ws)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.iters
    row = lay.layer_info(0)["row_bytes"]
    # rows and their scales (an uncompressed bf16 anchor, b = 0, reads no scale)
    nbytes = B * T * (row + (0 if args.b == 0 else 2))
    path = lay.decode_path_for(0, torch.bfloat16, H)
    print(json.dumps({"d": args.d, "b": args.b, "heads": H, "batch": B, "tokens": T,
                      "path": {1: "tensor", 2: "cuda_core"}[path], "ms_per_call": round(ms, 5),
                      "bytes_per_call": nbytes, "GBps": round(nbytes / ms / 1e6, 1),
                      "status": lay.read_status()}))
    lay.close()


if __name__ == "__main__":
    main()
