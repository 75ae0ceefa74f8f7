#!/usr/bin/env python
"""Timing table of the attention kernels over the shapes beside the headline
workload: dense forward/backward (atomic and deterministic dQ), dropout,
packed variable-length batches and decode.  One JSON line per row.

    python bench_table.py [--only dense,dropout,varlen,decode] [--iters N]

Device time with CUDA events on the launching stream, at least 3 warm-up
calls, the mean of ``--iters`` calls, queued behind a ~10 ms spin so that the
host's launch overhead never shows in a short call's events.  The forward/backward rows write a
256 MiB buffer (above the 126 MB L2) between calls, outside the event pairs;
the decode rows alternate two input sets instead (each set's caches exceed
L2).  FLOPs follow bench.py's convention (forward 4*S^2*D per head, halved
under a causal mask; backward 2.5x that); decode counts the K and V cache
bytes read once.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DENSE = [  # (B, H, S, D, dtype, causal)
    (1, 2, 256, 64, "bf16", False),
    (2, 8, 512, 64, "bf16", True),
    (2, 8, 512, 64, "fp16", True),
    (1, 32, 512, 128, "bf16", True),
    (1, 32, 1024, 128, "bf16", True),
    (1, 32, 2048, 128, "bf16", True),
    (1, 32, 4096, 128, "bf16", True),
    (1, 32, 4096, 128, "fp16", True),
    (1, 32, 4096, 128, "bf16", False),
    (4, 16, 8192, 128, "bf16", True),
    (1, 32, 32768, 128, "bf16", True),
]
DECODE = [  # (B, Hq, Hkv, L, D)
    (8, 32, 8, 8192, 128),
    (8, 32, 32, 4096, 128),
    (32, 32, 8, 2048, 128),
    (64, 32, 8, 1024, 128),
    (1, 32, 8, 32768, 128),
    (16, 16, 1, 8192, 64),
]


def flop_count(lengths, heads: int, d: int, causal: bool):
    f = sum(4.0 * L * L * d for L in lengths) * heads * (0.5 if causal else 1.0)
    return f, 2.5 * f


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--only", default="dense,dropout,varlen,decode")
    ap.add_argument("--iters", type=int, default=20)
    args = ap.parse_args()
    parts = set(args.only.split(","))

    import torch

    import exact_tiled_attention_31_b200 as fa
    from exact_tiled_attention_31_b200 import inputs

    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def timed(fn, iters, do_flush=True):
        for _ in range(3):
            if do_flush:
                flush.zero_()
            fn(0)
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
        # keep the GPU busy while the host queues the timed calls, so a short
        # call's events measure the device, not the host's launch overhead
        torch.cuda._sleep(20_000_000)
        for i, (e0, e1) in enumerate(evs):
            if do_flush:
                flush.zero_()
            e0.record(stream)
            fn(i)
            e1.record(stream)
        torch.cuda.synchronize()
        fa.check_device_error()
        return statistics.mean(a.elapsed_time(b) for a, b in evs)

    def emit(row):
        print(json.dumps(row), flush=True)

    def dense_row(B, H, S, D, dtype, causal, dropout_p=0.0):
        t = inputs.make_dense(B, H, S, D, dtype, seed=42, with_do=True)
        q, k, v, do = (t[x].to(dev) for x in ("q", "k", "v", "do"))
        scale = 1.0 / math.sqrt(D)
        o = torch.empty_like(q)
        lse = torch.empty((B, H, S), device=dev, dtype=torch.float32)
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
        ws = torch.empty(fa.fa_bwd_workspace_size(B, H, S, D), device=dev, dtype=torch.uint8)
        kw = dict(dropout_p=dropout_p, seed=7, offset=1) if dropout_p else {}
        it = args.iters if B * H * S * S * D < 2 ** 38 else max(5, args.iters // 4)

        def fwd(_):
            fa.forward(q, k, v, causal, scale, out=o, lse=lse, **kw)

        def bwd(det):
            return lambda _: fa.backward(q, k, v, o, do, lse, causal, scale, deterministic=det, workspace=ws,
                                         out=grads, **kw)

        t_f = timed(fwd, it)
        t_b = timed(bwd(False), it)
        t_d = timed(bwd(True), it)
        f_f, f_b = flop_count([S] * B, H, D, causal)
        emit({"kind": "dropout" if dropout_p else "dense", "shape": f"B{B} H{H} S{S} D{D}", "dtype": dtype,
              "causal": causal, "dropout_p": dropout_p, "fwd_us": t_f * 1e3, "bwd_us": t_b * 1e3,
              "bwd_det_us": t_d * 1e3, "det_over_atomic": t_d / t_b,
              "fwd_tflops": f_f / t_f / 1e9, "bwd_tflops": f_b / t_b / 1e9,
              "fwd_bwd_tflops": (f_f + f_b) / (t_f + t_b) / 1e9,
              "pct_2250_fwd_bwd": [100 * f_f / t_f / 1e9 / 2250, 100 * f_b / t_b / 1e9 / 2250]})

    if "dense" in parts:
        for c in DENSE:
            dense_row(*c)
    if "dropout" in parts:
        dense_row(1, 32, 4096, 128, "bf16", True, dropout_p=0.1)
        dense_row(1, 32, 4096, 128, "bf16", False, dropout_p=0.1)
    if "varlen" in parts:
        # the 32-sequence pack draws Q, K as N(0,1) * 8 (scores up to about +-64)
        for name, (n, lo, hi, H, D, mult) in {"packed 32 seqs, Q/K x 8": (32, 128, 4096, 16, 64, 8.0),
                                              "packed 16 seqs D128": (16, 512, 8192, 16, 128, 1.0)}.items():
            t = inputs.make_varlen(n, lo, hi, H, D, "bf16", seed=42, qk_mult=mult, with_do=True)
            q, k, v, do = (t[x].to(dev) for x in ("q", "k", "v", "do"))
            cu = t["cu_seqlens"].to(dev)
            L = max(t["lengths"])
            scale = 1.0 / math.sqrt(D)
            ws = torch.empty(fa.fa_bwd_varlen_workspace_size(n, L, t["total"], H, D), device=dev, dtype=torch.uint8)
            res = {}

            def vf(_):
                res["o"], res["lse"] = fa.forward_varlen(q, k, v, cu, L, True, scale)

            t_f = timed(vf, args.iters)

            def vb(_):
                fa.backward_varlen(q, k, v, res["o"], do, res["lse"], cu, L, True, scale, workspace=ws)

            t_b = timed(vb, args.iters)
            f_f, f_b = flop_count(t["lengths"], H, D, True)
            emit({"kind": "varlen", "shape": f"{name}: T={t['total']} H{H} D{D} lengths {lo}..{hi}", "dtype": "bf16",
                  "causal": True, "fwd_us": t_f * 1e3, "bwd_us": t_b * 1e3, "fwd_tflops": f_f / t_f / 1e9,
                  "bwd_tflops": f_b / t_b / 1e9, "fwd_bwd_tflops": (f_f + f_b) / (t_f + t_b) / 1e9})
    if "decode" in parts:
        del flush
        for B, Hq, Hkv, L, D in DECODE:
            sets = []
            for seed in (42, 43):
                h = inputs.make_decode(B, Hq, Hkv, L, D, "bf16", seed=seed)
                sets.append(tuple(h[x].to(dev) for x in ("q", "k", "v")))
            lens = torch.full((B,), L, dtype=torch.int32, device=dev)
            nbytes = 2 * B * Hkv * L * D * 2
            for n in (fa.fa_decode_num_splits(B, Hkv, L), 0):
                ws = torch.empty(max(1, fa.fa_decode_workspace_size(B, Hq, n, D)), device=dev, dtype=torch.uint8)
                o = torch.empty_like(sets[0][0])
                lse = torch.empty((B, Hq), device=dev, dtype=torch.float32)

                def dec(i):
                    q, k, v = sets[i % 2]
                    fa.decode(q, k, v, lens, n_splits=n, out=o, lse=lse, workspace=ws)

                t_d = timed(dec, max(args.iters, 30), do_flush=False)
                emit({"kind": "decode", "shape": f"B{B} Hq{Hq} Hkv{Hkv} L{L} D{D}", "dtype": "bf16",
                      "n_splits": n if n else "balanced (0)", "us": t_d * 1e3, "gbs": nbytes / t_d / 1e6})


if __name__ == "__main__":
    main()
