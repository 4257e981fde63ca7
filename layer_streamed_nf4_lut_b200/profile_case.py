"""Small, fixed workloads for profiler captures of single libsoup kernels.

A full-size step holds ~8 GB on the device and launches ~10k kernels; a profiler that replays
each captured kernel ~40 times wants far less.  These cases keep the per-kernel shapes of the
8B-shaped step but hold only a few GB:

  python -m layer_streamed_nf4_lut_b200.profile_case nf4-gemm --n 6144 --k 4096 --m 512 [--transposed]
      6 launches of one NF4 GEMM through soup_nf4_matmul (forward x W^T, or x W with
      --transposed); weights N(0, 0.02), activations N(0, 1) in bf16.
  python -m layer_streamed_nf4_lut_b200.profile_case nf4-sweep [--m 512 2048]
      CUDA-event timing (warm L2, 20 launches after 3 warm-up) of the four 8B projection
      GEMMs, forward and dX, one JSON line per shape.
  python -m layer_streamed_nf4_lut_b200.profile_case step --layers 2 [--batch 1] [--seq 512]
      the 8B-shaped SFT step (hidden 4096, 32/8 heads, intermediate 14336, vocab 128256,
      LoRA r=64) with fewer decoder layers, streamed through 2 layer buffers, 3 steps.

Run from the repository root (the seeded input generators live in the top-level synth module).
"""
from __future__ import annotations

import argparse
import math
import sys

import torch


def _nf4_gemm(args):
    import synth
    from . import model as M
    N, K, Mr = args.n, args.k, args.m
    w = synth.normal_device((N, K), 3, 0.02)
    q = M.nf4_quantize(w)
    del w
    x = synth.normal_device((Mr, N if args.transposed else K), 4, 1.0).to(torch.bfloat16)
    for _ in range(args.launches):
        y = M.nf4_matmul(x, q, transpose_w=args.transposed)
    torch.cuda.synchronize()
    print("nf4-gemm ok", N, K, Mr, args.transposed, float(y.float().abs().mean()))


SHAPES = [(6144, 4096, "qkv"), (4096, 4096, "o"), (28672, 4096, "gate_up"), (4096, 14336, "down")]


def _nf4_sweep(args):
    import json
    import synth
    from . import model as M
    for m_rows in args.m:
        for N, K, name in SHAPES:
            w = synth.normal_device((N, K), 3, 0.02)
            q = M.nf4_quantize(w)
            del w
            for tr in (False, True):
                x = synth.normal_device((m_rows, N if tr else K), 4, 1.0).to(torch.bfloat16)
                for _ in range(3):
                    M.nf4_matmul(x, q, transpose_w=tr)
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(args.iters):
                    M.nf4_matmul(x, q, transpose_w=tr)
                e1.record()
                e1.synchronize()
                ms = e0.elapsed_time(e1) / args.iters
                print(json.dumps(dict(M=m_rows, N=N, K=K, name=name, transposed=tr, us=round(ms * 1e3, 1),
                                      tflops=round(2.0 * m_rows * N * K / (ms * 1e-3) / 1e12, 1))), flush=True)


def _step(args):
    import synth
    from .model import SoupModel, lora_offset
    cfg = dict(synth.L8B, n_layers=args.layers)
    B, S = args.batch, args.seq
    gm = SoupModel(cfg, mode="streamed", n_layer_buffers=2, max_tokens=B * S)
    ones = torch.ones(cfg["hidden"], dtype=torch.bfloat16, device="cuda")
    for i in range(cfg["n_layers"]):
        w = {p: synth.normal_device(synth.proj_shape(cfg, p), 100003 + 16 * i + j, 0.02)
             for j, p in enumerate(synth.PROJ_NAMES)}
        gm.quantize_layer(i, w, ones, ones)
        del w
    V, h = cfg["vocab"], cfg["hidden"]
    gm.set_head(synth.normal_device((V, h), 8, 0.02).to(torch.bfloat16), ones.clone(),
                synth.normal_device((V, h), 9, 0.02).to(torch.bfloat16))
    params = torch.empty(gm.lora_n, dtype=torch.float32, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    for layer in range(cfg["n_layers"]):
        for j in range(len(synth.PROJ_NAMES)):
            oa, ra, ca = lora_offset(cfg, layer, j, 0)
            ob, rb, cb = lora_offset(cfg, layer, j, 1)
            params[oa:oa + ra * ca].uniform_(-1.0 / math.sqrt(ca), 1.0 / math.sqrt(ca), generator=g)
            params[ob:ob + rb * cb].normal_(0.0, 0.01, generator=g)
    gm.set_lora(params)
    ids = torch.from_numpy(synth.token_batch(dict(cfg, batch=B, seq=S), 77)).cuda()
    for _ in range(args.steps):
        loss = gm.step(ids, apply_optimizer=True, lr=2e-5)
    torch.cuda.synchronize()
    print("step ok", args.layers, B, S, loss, gm.stats())
    gm.close()


def main(argv=None):
    ap = argparse.ArgumentParser()
    sub = ap.add_subparsers(dest="case", required=True)
    a = sub.add_parser("nf4-gemm")
    a.add_argument("--n", type=int, default=6144)
    a.add_argument("--k", type=int, default=4096)
    a.add_argument("--m", type=int, default=512)
    a.add_argument("--transposed", action="store_true")
    a.add_argument("--launches", type=int, default=6)
    c = sub.add_parser("nf4-sweep")
    c.add_argument("--m", type=int, nargs="+", default=[512, 2048])
    c.add_argument("--iters", type=int, default=20)
    b = sub.add_parser("step")
    b.add_argument("--layers", type=int, default=2)
    b.add_argument("--batch", type=int, default=1)
    b.add_argument("--seq", type=int, default=512)
    b.add_argument("--steps", type=int, default=3)
    args = ap.parse_args(argv)
    if not torch.cuda.is_available():
        raise SystemExit("profile_case needs a CUDA device")
    {"nf4-gemm": _nf4_gemm, "nf4-sweep": _nf4_sweep, "step": _step}[args.case](args)
    return 0


if __name__ == "__main__":
    sys.exit(main())
