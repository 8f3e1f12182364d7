"""Run a few passes of the hot path of one workload, for a profiler to capture.

  python -m long_context_rope_b200.profile_step --workload prefill_64k --steps 2
  python -m long_context_rope_b200.profile_step --workload decode_16x32k --steps 2
  python -m long_context_rope_b200.profile_step --workload prefill_64k --seq-len 32768

--seq-len / --batch shrink a workload (same heads and routing) for captures
that replay each launch many times.

Setup (input draw, query rotation, and for decode the summaries/cache build)
happens before the steps; each prefill step is summaries -> q-bar ->
route_chunks -> route_groups -> attend; a decode step over the resident
cache is one decode_step_kernel launch (--separate: route_chunks ->
route_groups -> attend), a tiered decode step one decode_step_kernel launch
reading the routed groups from host memory (--separate: decode_step_kernel
routing only -> gather -> attend). Variants of the resident decode:
--fp8-kv (E4M3 cache), --per-q-head (per-query-head routing),
--bf16-summaries (bf16 tables). Kernel names: summaries_kernel, qbar_kernel,
route_chunks_tiled_kernel / route_chunks_kernel, route_groups_kernel,
attend_tc_kernel / attend_decode_kernel / attend_simt_kernel,
decode_step_kernel, gather_*_kernel.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from long_context_rope_b200 import hga, pipeline, synth  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="prefill_64k")
    ap.add_argument("--steps", type=int, default=2)
    ap.add_argument("--gathered", action="store_true", help="decode: gather, then attend")
    ap.add_argument("--separate", action="store_true",
                    help="decode: routing levels and attention as separate launches")
    ap.add_argument("--seq-len", type=int, default=None, help="override the context length")
    ap.add_argument("--batch", type=int, default=None, help="override the batch")
    ap.add_argument("--fp8-kv", action="store_true", help="decode: E4M3 key/value cache")
    ap.add_argument("--per-q-head", action="store_true", help="decode: per-query-head routing")
    ap.add_argument("--bf16-summaries", action="store_true", help="bf16 summary tables")
    args = ap.parse_args()
    w = synth.WORKLOADS[args.workload]
    if args.seq_len is not None:
        w = w.replace(seq_len=args.seq_len)
    if args.batch is not None:
        w = w.replace(batch=args.batch)
    cfg = hga.config_from(
        w, summary_type=hga.HGA_SUMMARY_BF16 if args.bf16_summaries else hga.HGA_SUMMARY_F32,
        routing=hga.HGA_ROUTE_PER_Q_HEAD if args.per_q_head else hga.HGA_ROUTE_PER_KV_HEAD)
    x = synth.draw(w, seed=0)
    k_raw = x["k_raw"].cuda()
    q_rot = pipeline.rotate_queries(cfg, x["q_raw"].cuda())
    cs, gs = pipeline.alloc_summaries(cfg)
    k_rot = torch.empty_like(k_raw)
    rb = pipeline.alloc_route(cfg)
    out = torch.empty_like(q_rot)
    if w.mode == "prefill":
        v = x["v"].cuda()
        for _ in range(args.steps):
            pipeline.prefill(cfg, k_raw, v, q_rot, cs, gs, k_rot, rb, out)
    else:
        pipeline.summaries(cfg, k_raw, cs, gs, k_rot)
        del k_raw
        if w.tiered:
            k_host = torch.empty(k_rot.shape, dtype=k_rot.dtype, pin_memory=True)
            k_host.copy_(k_rot)
            v_host = x["v"].pin_memory()
            del k_rot
            W = hga.window_slots(cfg)
            shape = (w.batch, w.n_kv_heads, W * w.chunk_size, w.head_dim)
            k_win = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
            v_win = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
            pipeline.fill_windows(cfg, k_host, v_host, k_win, v_win)
            cfg_w = cfg.copy(kv_layout=hga.HGA_KV_WINDOWS)
            gat = pipeline.alloc_gathered(cfg)
            for _ in range(args.steps):
                if args.separate:
                    pipeline.decode(cfg_w, q_rot, cs, gs, k_win, v_win, rb, out, gathered=gat,
                                    k_src=k_host, v_src=v_host, src_is_host=True)
                else:
                    pipeline.decode_tiered(cfg_w, q_rot, cs, gs, k_win, v_win, k_host, v_host,
                                           rb, out)
        else:
            v = x["v"].cuda()
            if args.fp8_kv:  # the cache as E4M3 codes with a per-tensor scale each
                k_rot, ks = synth.to_e4m3(k_rot)
                v, vs = synth.to_e4m3(v)
                cfg = cfg.copy(kv_type=hga.HGA_KV_E4M3, k_scale=ks, v_scale=vs)
            gat = pipeline.alloc_gathered(cfg) if args.gathered else None
            for _ in range(args.steps):
                pipeline.decode(cfg, q_rot, cs, gs, k_rot, v, rb, out, gathered=gat,
                                k_src=k_rot, v_src=v, separate=args.separate)
    torch.cuda.synchronize()
    err = hga.get_device_error()
    print(f"{args.workload}: {args.steps} steps done, device error word {err}")
    sys.exit(1 if err else 0)


if __name__ == "__main__":
    main()
