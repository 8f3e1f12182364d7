"""Benchmark of the HGA hot path on B200: routed prefill tok/s at 64K context
(the headline value) and decode µs/step, with roofline, CPU-oracle baseline,
end-to-end (host-buffer) throughput and SM clocks, printed as one JSON line.

  python bench.py [--gpus N --steps K --warmup W] [--impl hga|reference]

For N > 1 launch with torch.distributed.run: every rank runs its own
independent sequence (weak scaling, no collective on the data path); times
are the max over ranks and `value` counts the tokens of all ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_rope_b200 import dist_util, synth  # noqa: E402

METRIC = "routed attn prefill tok/s & decode µs/step at 64K; % of HBM/TC roofline"

# DRAM bytes (read + write) of one prefill attention launch at 64K context,
# from an ncu capture of attend_tc_kernel at 32K context (579.4 MB: Q and O
# once, K/V from L2) scaled x2 (one unit per query chunk). Valid for the
# kernel as captured; set to None when attend_tc_kernel changes until it is
# captured again.
TC_TRAFFIC_BYTES = 2 * 579.4e6
TC_TRAFFIC_NOTE = ("ncu dram__bytes_read+write of attend_tc_kernel at 32K context x2 "
                   "(profiles/attend_tc_prefill_32k_ncu.md)")
PREFILL = "prefill_64k"
# ":bf16sum" = the same workload with bf16 summary tables; ":fp8kv" = with an
# FP8 (E4M3) key/value cache; ":perhead" = with per-query-head routing
DECODES = ("decode_16x32k", "decode_16x32k:bf16sum", "decode_16x32k:fp8kv",
           "decode_16x32k:perhead", "tiered_decode_4x64k")


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return dict(hbm=float(pk["hbm_gbs"]), tc=float(pk["bf16_tflops"]),
                    tc_sustained=float(pk["bf16_tflops_sustained"]), src="measured")
    except Exception:
        return dict(hbm=6650.0, tc=1590.0, tc_sustained=1400.0, src="fallback")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock and clock-event reasons of this GPU, sampled every 5 ms through
    NVML (read-only queries) from a background thread during the timed region."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device: torch.device):
        self.device = device
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.handle = None
        self._stop = threading.Event()

    def __enter__(self):
        try:
            import pynvml
            self.nv = pynvml
            pynvml.nvmlInit()
            self.handle = None
            uuid = getattr(torch.cuda.get_device_properties(self.device), "uuid", None)
            if uuid is not None:
                text = str(uuid)
                if not text.startswith("GPU-"):
                    text = "GPU-" + text
                try:
                    self.handle = pynvml.nvmlDeviceGetHandleByUUID(text)
                except Exception:
                    self.handle = None
            if self.handle is None and pynvml.nvmlDeviceGetCount() == 1:
                self.handle = pynvml.nvmlDeviceGetHandleByIndex(0)
            if self.handle is None:
                return self
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        except Exception:
            self.handle = None
        return self

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(float(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                for name, const in self.REASONS:
                    if bits & getattr(nv, const):
                        self.reasons.add(name)
            except Exception:
                break
            time.sleep(0.005)

    def __exit__(self, *a):
        self._stop.set()
        if self.handle is not None:
            self.t.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples),
                "source": "NVML, 5 ms"}


# ----------------------------------------------------------------- timing
class Events:
    def __init__(self, n):
        self.ev = [torch.cuda.Event(enable_timing=True) for _ in range(n)]

    def rec(self, i, stream):
        self.ev[i].record(stream)

    def ms(self, a, b):
        return self.ev[a].elapsed_time(self.ev[b])


def prefill_flops(cfg, n_sel_groups: np.ndarray) -> float:
    """Algorithmic FLOPs of one prefill attention launch: 4*d per (query row,
    visible key) pair (QK^T and PV, 2 FLOPs per multiply-add). Visible keys of
    query token t of chunk j: routed groups*16 + full forced chunks before j
    + (t - jC + 1) keys of the current chunk (causal)."""
    C, d, gq = cfg.chunk_size, cfg.head_dim, cfg.n_q_heads // cfg.n_kv_heads
    total = 0
    nC = cfg.n_chunks
    for j in range(nC):
        s_end = min(cfg.n_sink, j + 1)
        n_forced = s_end + (j + 1 - max(s_end, j - cfg.n_local))
        n_tok = min((j + 1) * C, cfg.seq_len) - j * C
        base = (n_forced - 1) * C
        per_tok = n_tok * base + n_tok * (n_tok + 1) // 2
        routed = int(n_sel_groups[..., j].sum()) * 16 * n_tok
        total += gq * (per_tok * cfg.batch * cfg.n_kv_heads + routed)
    return 4.0 * d * total


def run_prefill(args, dist, peaks):
    from long_context_rope_b200 import hga, pipeline
    w = synth.WORKLOADS[args.workload]
    cfg = hga.config_from(w)
    seed = dist.seed(args.seed)
    x = synth.draw(w, seed=seed)
    dev = torch.device("cuda", torch.cuda.current_device())
    st = torch.cuda.current_stream()
    k_raw = x["k_raw"].to(dev)
    v = x["v"].to(dev)
    q_rot = pipeline.rotate_queries(cfg, x["q_raw"].to(dev))
    cs, gs = pipeline.alloc_summaries(cfg, dev)
    k_rot = torch.empty_like(k_raw)
    rb = pipeline.alloc_route(cfg, dev)
    out = torch.empty_like(q_rot)

    def step(ev=None, base=0):
        if ev:
            ev.rec(base, st)
        pipeline.summaries(cfg, k_raw, cs, gs, k_rot)
        if ev:
            ev.rec(base + 1, st)
        # q-bar, then both routing levels in one launch (hga_route, prefill form)
        hga.route(cfg, q_rot, cs, gs, rb.qbar, rb.sel_chunks, rb.n_sel_chunks, rb.sel_groups,
                  rb.n_sel_groups)
        if ev:
            ev.rec(base + 2, st)
        hga.attend(cfg, q_rot, k_rot, v, rb.sel_groups, rb.n_sel_groups, out)
        if ev:
            ev.rec(base + 3, st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if hga.get_device_error() != 0:
        raise RuntimeError("device error word set during warm-up")
    flops = prefill_flops(cfg, rb.n_sel_groups.cpu().numpy())
    recall = planted_recall(w, x["planted"], rb.sel_chunks.cpu().numpy(),
                            rb.n_sel_chunks.cpu().numpy())

    K = args.steps
    ev = Events(4 * K)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        start.record(st)
        for i in range(K):
            step(ev, 4 * i)
        stop.record(st)
        torch.cuda.synchronize()
    dist.barrier()
    total_ms = start.elapsed_time(stop)
    stage = {n: [] for n in ("summaries", "route", "attend")}
    for i in range(K):
        for s_i, n in enumerate(stage):
            stage[n].append(ev.ms(4 * i + s_i, 4 * i + s_i + 1))
    attend_ms = float(np.mean(stage["attend"]))
    res = dict(total_ms=dist.max(total_ms), attend_ms=dist.max(attend_ms),
               stage_ms={n: float(np.mean(vs)) for n, vs in stage.items()},
               flops=flops, tokens=w.batch * w.q_len, clocks=clk.summary(), recall=recall,
               launches_per_step=4)

    # end to end through the public API with host buffers (pinned), H2D + D2H inside
    if not args.no_e2e:
        hk, hv, hq = (t.cpu().pin_memory() for t in (k_raw, v, q_rot))
        ho = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        # the public API with host buffers: K, V and Q in, O out over the host
        # link, overlapped with slice-by-slice routing and attention
        hp = pipeline.HostPrefill(cfg, chunks_per_slice=64, device=dev)

        def e2e_step():
            hp.run(hk, hv, hq, ho)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        n_e2e = max(1, min(K, 5))
        dist.barrier()
        torch.cuda.synchronize()
        start.record(st)
        for _ in range(n_e2e):
            e2e_step()
        stop.record(st)
        torch.cuda.synchronize()
        dist.barrier()
        e2e_ms = dist.max(start.elapsed_time(stop)) / n_e2e
        res["e2e"] = dict(ms=e2e_ms, h2d=hk.numel() * 2 + hv.numel() * 2 + hq.numel() * 2,
                          d2h=ho.numel() * 2)
    res["cfg"] = cfg
    return res


def run_decode(name, args, dist):
    from long_context_rope_b200 import hga, pipeline
    base, _, variant = name.partition(":")
    w = synth.WORKLOADS[base]
    bf16_sum = variant == "bf16sum"
    fp8_kv = variant == "fp8kv"
    per_head = variant == "perhead"
    kv_es = 1 if fp8_kv else 2  # bytes per K/V element
    cfg = hga.config_from(w, summary_type=hga.HGA_SUMMARY_BF16 if bf16_sum else hga.HGA_SUMMARY_F32,
                          routing=hga.HGA_ROUTE_PER_Q_HEAD if per_head else hga.HGA_ROUTE_PER_KV_HEAD)
    x = synth.draw(w, seed=dist.seed(args.seed))
    dev = torch.device("cuda", torch.cuda.current_device())
    st = torch.cuda.current_stream()
    k_raw = x["k_raw"].to(dev)
    cs, gs = pipeline.alloc_summaries(cfg, dev)
    k_rot = torch.empty_like(k_raw)
    pipeline.summaries(cfg, k_raw, cs, gs, k_rot)
    del k_raw
    q_rot = pipeline.rotate_queries(cfg, x["q_raw"].to(dev))
    rb = pipeline.alloc_route(cfg, dev)
    out = torch.empty_like(q_rot)
    gat = pipeline.alloc_gathered(cfg, dev)
    if w.tiered:
        k_host = torch.empty(k_rot.shape, dtype=k_rot.dtype, pin_memory=True)
        k_host.copy_(k_rot)
        v_host = x["v"].pin_memory()
        del k_rot
        W = hga.window_slots(cfg)
        shape = (w.batch, w.n_kv_heads, W * w.chunk_size, w.head_dim)
        k_win = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
        v_win = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
        pipeline.fill_windows(cfg, k_host, v_host, k_win, v_win)
        cfg_w = cfg.copy(kv_layout=hga.HGA_KV_WINDOWS)

        # warm tier: a VRAM pool of 4 x top_k_groups groups per (sequence, KV head)
        pool = pipeline.alloc_warm_pool(cfg, 4 * cfg.top_k_groups, dev)

        def step_fn(separate=False, warm=False):
            if separate or warm:  # route (one launch), [warm] gather, attend
                pipeline.decode(cfg_w, q_rot, cs, gs, k_win, v_win, rb, out, gathered=gat,
                                k_src=k_host, v_src=v_host, src_is_host=True,
                                warm=pool if warm else None)
            else:  # one launch: routed groups read from the host inside the kernel
                pipeline.decode_tiered(cfg_w, q_rot, cs, gs, k_win, v_win, k_host, v_host, rb,
                                       out)
        launches, launches_sep = 1, 3
    else:
        v = x["v"].to(dev)
        if fp8_kv:  # the cache stored as E4M3 codes with a per-tensor scale each
            k_rot, ks = synth.to_e4m3(k_rot)
            v, vs = synth.to_e4m3(v)
            cfg = cfg.copy(kv_type=hga.HGA_KV_E4M3, k_scale=ks, v_scale=vs)
            gat = pipeline.alloc_gathered(cfg, dev)

        def step_fn(separate=False, warm=False):
            pipeline.decode(cfg, q_rot, cs, gs, k_rot, v, rb, out, separate=separate)
        launches, launches_sep = 1, 3  # one-launch decode step
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    K = max(args.steps, 20)

    def timed(separate, warm=False, fn=None):
        """Device time of one step, L2 flushed before every step. Primary: one
        CUDA graph of KP x (flush, step) minus one graph of the same KP
        flushes, each replayed 5 times between events (medians), over KP: the
        time a step adds to a stream of device work, its launch following the
        previous kernel as in a decode loop. Also the median of single graph
        replays between events after a flush (each then starts on an idle
        device, launch latency included) and of eager launches."""
        if fn is not None:
            step = lambda separate, warm: fn()  # noqa: E731
        else:
            step = step_fn
        for _ in range(max(3, args.warmup)):
            step(separate, warm)
        torch.cuda.synchronize()
        if hga.get_device_error() != 0:
            raise RuntimeError(f"device error word set in {name}")
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="relaxed"):
            step(separate, warm)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        if hga.get_device_error() != 0:
            raise RuntimeError(f"device error word set in {name} (graph)")
        ev = Events(2 * K)
        for i in range(K):
            flush.fill_(i & 0xff)  # write a buffer larger than L2 between steps
            ev.rec(2 * i, st)
            graph.replay()
            ev.rec(2 * i + 1, st)
        torch.cuda.synchronize()
        times = [ev.ms(2 * i, 2 * i + 1) * 1000.0 for i in range(K)]
        ev2 = Events(2 * 5)
        for i in range(5):
            flush.fill_(i & 0xff)
            ev2.rec(2 * i, st)
            step(separate, warm)
            ev2.rec(2 * i + 1, st)
        torch.cuda.synchronize()
        eager = float(np.median([ev2.ms(2 * i, 2 * i + 1) * 1000.0 for i in range(5)]))
        del graph
        KP = 16
        g_pipe, g_flush = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_pipe, capture_error_mode="relaxed"):
            for i in range(KP):
                flush.fill_(i & 0xff)
                step(separate, warm)
        with torch.cuda.graph(g_flush, capture_error_mode="relaxed"):
            for i in range(KP):
                flush.fill_(i & 0xff)

        def graph_ms(g):
            g.replay()
            e = Events(2 * 5)
            for i in range(5):
                e.rec(2 * i, st)
                g.replay()
                e.rec(2 * i + 1, st)
            torch.cuda.synchronize()
            return float(np.median([e.ms(2 * i, 2 * i + 1) for i in range(5)]))

        pipelined = (graph_ms(g_pipe) - graph_ms(g_flush)) * 1000.0 / KP
        if hga.get_device_error() != 0:
            raise RuntimeError(f"device error word set in {name} (pipelined graph)")
        del g_pipe, g_flush
        return dict(pipelined=pipelined, single=times, eager=eager)

    # the separate routing calls read fp32 tables of per-KV-head routing only
    t_sep = None if bf16_sum or per_head else timed(True)
    t_one = timed(False)
    times, eager_us = t_one["single"], t_one["eager"]
    us = dist.max(t_one["pipelined"])
    us_single = dist.max(float(np.median(times)))
    us_sep = dist.max(t_sep["pipelined"]) if t_sep else None
    eager_sep = t_sep["eager"] if t_sep else None
    warm_info = None
    if w.tiered:
        # steady state of the warm tier for this (fixed) query: its routed groups
        # stay in the pool, so no group crosses the host link after the first step
        t_warm = timed(False, warm=True)
        hits_misses = pool.stats.cpu().numpy().reshape(-1, 2).sum(0)
        warm_info = dict(us_per_step=dist.max(t_warm["pipelined"]),
                         us_per_step_single_replay=dist.max(float(np.median(t_warm["single"]))),
                         pool_slots=int(pool.tag.shape[-1]),
                         hit_rate=float(hits_misses[0] / max(1, hits_misses.sum())),
                         host_bytes_per_step=int(hits_misses[1]) * 16 * w.head_dim * 2 * 2,
                         note="fixed query: the all-hits steady state of the warm tier")
        warm_info["drifting"] = run_warm_drift(w, args, dist, cfg, cfg_w, cs, gs, k_win, v_win,
                                               k_host, v_host, st)
    n_sel = rb.n_sel_groups.cpu().numpy()
    moved = int(n_sel.sum()) * 16 * w.head_dim * kv_es * 2  # routed K+V bytes read
    if per_head:  # distinct routed groups per (sequence, KV head): the bytes HBM must supply
        gq = w.n_q_heads // w.n_kv_heads
        sg = rb.sel_groups.cpu().numpy().reshape(w.batch, w.n_kv_heads, gq, -1)
        ng = n_sel.reshape(w.batch, w.n_kv_heads, gq)
        uniq = sum(len(set(int(v) for i in range(gq) for v in sg[b, k, i, :ng[b, k, i]]))
                   for b in range(w.batch) for k in range(w.n_kv_heads))
        moved_unique = uniq * 16 * w.head_dim * kv_es * 2
    else:
        moved_unique = moved
    recall = planted_recall(w, x["planted"], rb.sel_chunks.cpu().numpy(),
                            rb.n_sel_chunks.cpu().numpy())
    gather_info = None
    if not w.tiered and not variant:
        # the exact-token gather from HBM alone (hga_gather_kv): (1) one launch
        # replayed from a CUDA graph after an L2 flush (includes the graph's
        # launch latency); (2) launches back to back, cycling through the
        # selections of 8 different queries, so each launch reads groups the
        # previous seven launches' 700 MB of traffic has evicted from L2 and
        # the launch latency overlaps the previous launch (the kernel's
        # throughput). Each launch reads and writes every routed group's K
        # and V once.
        t_g = timed(False, fn=lambda: hga.gather_kv(
            cfg, k_rot, v, False, rb.sel_groups, rb.n_sel_groups, gat[0], gat[1]))
        sels = []
        for i in range(8):
            xi = synth.draw(w, seed=dist.seed(args.seed) + 104729 * (i + 1), with_kv=False)
            rbi = pipeline.alloc_route(cfg, dev)
            pipeline.route(cfg, pipeline.rotate_queries(cfg, xi["q_raw"].to(dev)), cs, gs, rbi)
            sels.append(rbi)
        torch.cuda.synchronize()
        moved_seq = sum(int(r.n_sel_groups.sum()) for r in sels) * 16 * w.head_dim * 2 * 2 / 8
        n_seq = 32
        flush.fill_(1)
        ev = Events(2)
        ev.rec(0, st)
        for i in range(n_seq):
            r_i = sels[i % 8]
            hga.gather_kv(cfg, k_rot, v, False, r_i.sel_groups, r_i.n_sel_groups, gat[0], gat[1])
        ev.rec(1, st)
        torch.cuda.synchronize()
        if hga.get_device_error() != 0:
            raise RuntimeError("device error word set in the gather run")
        seq_us = dist.max(ev.ms(0, 1) * 1000.0 / n_seq)
        g_us = dist.max(float(np.median(t_g["single"])))
        g_bytes = 2 * moved
        peak = load_peaks()["hbm"]
        gather_info = dict(kernel="gather_hbm_kernel (hga_gather_kv, HBM source)",
                           us=seq_us, bytes=2 * moved_seq,
                           hbm_gbs=2 * moved_seq / (seq_us * 1e-6) / 1e9,
                           hbm_frac=2 * moved_seq / (seq_us * 1e-6) / 1e9 / peak,
                           timing=f"{n_seq} launches back to back over 8 queries' selections",
                           us_single_graph=g_us, bytes_single=g_bytes,
                           hbm_frac_single_graph=g_bytes / (g_us * 1e-6) / 1e9 / peak,
                           launches=1)
    # algorithmic HBM bytes of one step (each byte the step must touch, once)
    n_forced_tok = (min(w.n_sink, w.n_chunks) + w.n_local + 1) * w.chunk_size
    forced_kv = w.batch * w.n_kv_heads * n_forced_tok * w.head_dim * kv_es * 2
    se = 2 if bf16_sum else 4  # summary element bytes
    chunk_sums = w.batch * w.n_kv_heads * w.n_chunks * w.head_dim * se
    group_sums = int(rb.n_sel_chunks.cpu().numpy().sum()) * w.groups_per_chunk * w.head_dim * se
    if per_head:  # distinct selected chunks' group rows per (sequence, KV head)
        gq = w.n_q_heads // w.n_kv_heads
        sc = rb.sel_chunks.cpu().numpy().reshape(w.batch, w.n_kv_heads, gq, -1)
        nc = rb.n_sel_chunks.cpu().numpy().reshape(w.batch, w.n_kv_heads, gq)
        uc = sum(len(set(int(v) for i in range(gq) for v in sc[b, k, i, :nc[b, k, i]]))
                 for b in range(w.batch) for k in range(w.n_kv_heads))
        group_sums = uc * w.groups_per_chunk * w.head_dim * se
    q_o = 2 * w.batch * w.n_q_heads * w.head_dim * 2
    # tiered: the one-launch step reads the routed groups from the host, not
    # from HBM (the three-launch path also writes and reads them in a buffer)
    hbm_bytes = forced_kv + chunk_sums + group_sums + q_o + (0 if w.tiered else moved_unique)
    return dict(workload=name, summary_tables="bf16" if bf16_sum else "fp32",
                kv_cache="e4m3" if fp8_kv else "bf16",
                routing="per query head" if per_head else "per KV head", us_per_step=us,
                timing="device time a step adds to a CUDA graph of 16 x (L2 flush, step), "
                       "less the graph of the 16 flushes alone",
                us_per_step_single_replay=us_single, us_min_single_replay=float(np.min(times)),
                steps=K,
                hbm_bytes_per_step=hbm_bytes, hbm_gbs=hbm_bytes / (us * 1e-6) / 1e9,
                hbm_frac=hbm_bytes / (us * 1e-6) / 1e9 / load_peaks()["hbm"],
                us_per_step_eager=eager_us, cuda_graph=True,
                launches_per_step=launches, routed_kv_bytes=moved,
                routed_kv_bytes_distinct=moved_unique,
                us_per_step_separate_kernels=us_sep, us_per_step_separate_eager=eager_sep,
                launches_per_step_separate=launches_sep, warm_tier=warm_info,
                gather=gather_info, planted_recall=recall,
                host_link_gbs=(moved / (us * 1e-6) / 1e9) if w.tiered else None,
                host_link_gbs_separate=(moved / (us_sep * 1e-6) / 1e9) if w.tiered else None)


def run_warm_drift(w, args, dist, cfg, cfg_w, cs, gs, k_win, v_win, k_host, v_host, st,
                   n_queries=8, steps_per_query=4, n_steps=48):
    """The warm tier on a decode sequence whose planted topic drifts: step s
    uses query q[(s // steps_per_query) % n_queries], each drawn with its own
    seed (its own planted source chunk and noise), so routed groups enter and
    age out of the pool. After one pass over the queries (pool warm-up), the
    timed steps report the hit rate, the host-link bytes per step and the
    device time per step (route + warm gather + attention, eager launches)."""
    from long_context_rope_b200 import hga, pipeline
    dev = torch.device("cuda", torch.cuda.current_device())
    qs = []
    for i in range(n_queries):
        xi = synth.draw(w, seed=dist.seed(args.seed) + 7919 * (i + 1), with_kv=False)
        qs.append(pipeline.rotate_queries(cfg, xi["q_raw"].to(dev)))
    pool = pipeline.alloc_warm_pool(cfg, 4 * cfg.top_k_groups, dev)
    rb = pipeline.alloc_route(cfg, dev)
    gat = pipeline.alloc_gathered(cfg, dev)
    out = torch.empty_like(qs[0])

    def step(s):
        pipeline.decode(cfg_w, qs[(s // steps_per_query) % n_queries], cs, gs, k_win, v_win, rb,
                        out, gathered=gat, k_src=k_host, v_src=v_host, src_is_host=True,
                        warm=pool)

    warm_steps = n_queries * steps_per_query
    for s in range(warm_steps):
        step(s)
    torch.cuda.synchronize()
    ev = Events(2 * n_steps)
    hits = misses = 0
    for i in range(n_steps):
        ev.rec(2 * i, st)
        step(warm_steps + i)
        ev.rec(2 * i + 1, st)
        hm = pool.stats.sum(dim=(0, 1))
        hits += int(hm[0])
        misses += int(hm[1])
    torch.cuda.synchronize()
    if hga.get_device_error() != 0:
        raise RuntimeError("device error word set in the drifting warm-tier run")
    times = [ev.ms(2 * i, 2 * i + 1) * 1000.0 for i in range(n_steps)]
    group_bytes = 16 * w.head_dim * 2 * 2
    return dict(us_per_step=dist.max(float(np.median(times))), steps=n_steps,
                hit_rate=hits / max(1, hits + misses),
                host_bytes_per_step=misses * group_bytes / n_steps,
                schedule=f"{n_queries} planted queries, each for {steps_per_query} consecutive "
                         f"steps, cycled; pool {pool.tag.shape[-1]} groups per (sequence, KV head)")


def planted_recall(w, planted, sel_chunks: np.ndarray, n_sel_chunks: np.ndarray) -> dict:
    """How often the chunk whose topic was planted into a query chunk is in
    that query chunk's visible set: selected by level-1 routing, or always
    visible (sinks, locals, current). Reported as a statistic of the
    synthetic data, not a parity bar."""
    C = w.chunk_size
    j0 = w.q_begin // C
    seen = routed = total = cand = 0
    for b, per_b in enumerate(planted):
        for jj, srcs in enumerate(per_b):
            j = j0 + jj
            if jj >= sel_chunks.shape[2]:
                continue
            for h in range(sel_chunks.shape[1]):  # KV heads, or query heads (per-head routing)
                sel = set(sel_chunks[b, h, jj, :n_sel_chunks[b, h, jj]].tolist())
                for c in srcs:
                    forced = c < w.n_sink or j - w.n_local <= c <= j
                    total += 1
                    seen += int(forced or c in sel)
                    if not forced:
                        cand += 1
                        routed += int(c in sel)
    return dict(visible=seen / max(1, total), routed_among_candidates=routed / max(1, cand),
                planted=total, planted_candidates=cand)


def host_link_peak_gbs(dev) -> float:
    """Measured pinned host -> device copy bandwidth (256 MiB, best of 5): the
    denominator of the host-link (cold tier) gather."""
    src = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(src.shape, dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()
    best = 0.0
    for _ in range(6):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        dst.copy_(src, non_blocking=True)
        b.record(st)
        torch.cuda.synchronize()
        best = max(best, src.numel() / (a.elapsed_time(b) * 1e-3) / 1e9)
    return best


def cpu_baseline(args, n_chunks_sample=4, threads=None):
    """The oracle, as it stands, on a bounded sample of the 64K workload:
    whole-sequence work (key rotation, summaries) timed once and charged per
    token; per-query-chunk work (query rotation, q-bar, routing, attention)
    timed on `n_chunks_sample` query chunks. `threads`: the oracle's thread
    count for this measurement (None: all host cores); restored afterwards."""
    from oracle import hga_oracle as O
    if threads is not None:
        all_threads = O.num_threads()
        O.set_threads(threads)
        try:
            return cpu_baseline(args, n_chunks_sample)
        finally:
            O.set_threads(all_threads)
    w = synth.WORKLOADS[args.workload]
    x = synth.draw(w, seed=args.seed)
    cfg = O.cfg_of(w)
    k_raw = x["k_raw"].float().numpy()
    q_raw = x["q_raw"].float().numpy()
    v = x["v"].float().numpy()
    t0 = time.perf_counter()
    k_rot = np.empty_like(k_raw)
    for h in range(w.n_kv_heads):
        k_rot[0, h] = O.rope_f32(cfg, k_raw[0, h][:, None, :], 0, True)[:, 0, :]
    cs, gs = O.build_summaries(cfg, k_raw)
    t_seq = time.perf_counter() - t0
    rng = np.random.default_rng(0)
    js = sorted(rng.choice(np.arange(1, w.n_chunks), size=n_chunks_sample, replace=False).tolist())
    t1 = time.perf_counter()
    for j in js:
        C = w.chunk_size
        cj = O.cfg_of(w, q_begin=j * C, q_len=C)
        q_rot = O.rope_f32(cfg, q_raw[0, j * C:(j + 1) * C], j * C, True)[None]
        qb = O.qbar(cj, q_rot)
        sel, nsel, _ = O.route_chunks(cj, qb, cs, False)
        gsel, gnsel, _ = O.route_groups(cj, qb, gs, sel, nsel, False)
        O.attend(cj, q_rot, k_rot, v, gsel, gnsel)
    t_chunks = time.perf_counter() - t1
    tok = n_chunks_sample * w.chunk_size
    sec_per_tok = t_seq / w.seq_len + t_chunks / tok
    return dict(value=1.0 / sec_per_tok, unit="tok/s", cores=O.num_threads(), kind="oracle",
                sample=(f"{args.workload}: key rotation + summaries of all {w.n_chunks} chunks "
                        f"({t_seq:.2f} s, charged per token) + rotation, q-bar, routing and "
                        f"attention of {n_chunks_sample} query chunks {js} ({t_chunks:.2f} s)"),
                seconds=t_seq + t_chunks)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="hga", choices=["hga", "reference"])
    ap.add_argument("--workload", default=PREFILL)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    peaks = load_peaks()
    w = synth.WORKLOADS[args.workload]

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        vals = []
        cb = None
        for i in range(args.warmup + args.steps):
            cb = cpu_baseline(args, n_chunks_sample=1)
            if i >= args.warmup:
                vals.append(cb["value"])
        v = float(np.median(vals))
        line = {"metric": METRIC, "value": v, "unit": "tok/s", "impl": "reference",
                "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": cb["seconds"] * 1000.0,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic",
                "config": {"workload": args.workload, "seq_len": w.seq_len, "batch": w.batch},
                "cpu_baseline": {"value": v, "unit": "tok/s", "cores": cb["cores"],
                                 "kind": "oracle", "sample": cb["sample"]},
                "e2e": {"value": v, "unit": "tok/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    dist = dist_util.Dist("nccl")
    try:
        pre = run_prefill(args, dist, peaks)
        decodes = []
        if not args.no_decode:
            link = host_link_peak_gbs(torch.device("cuda", torch.cuda.current_device()))
            for name in DECODES:
                d = run_decode(name, args, dist)
                if d.get("host_link_gbs") is not None:
                    d["host_link_peak_gbs"] = link
                    d["host_link_frac"] = d["host_link_gbs"] / link
                decodes.append(d)
        n = dist.world
        value = n * pre["tokens"] / (pre["total_ms"] / args.steps / 1000.0)
        ach = pre["flops"] / (pre["attend_ms"] * 1e-3) / 1e12
        # the burst GEMM peak while the SM clock stayed at its maximum during
        # the timed region (no power cap reached), else the sustained one
        ck = pre["clocks"] or {}
        at_max = bool(ck.get("sm_mhz")) and ck["sm_mhz"] >= 0.95 * ck.get("sm_max_mhz", 1e9)
        tc_peak = peaks["tc"] if at_max else peaks["tc_sustained"]
        tc_note = (f"bf16 {'burst' if at_max else 'sustained'} cuBLAS GEMM, {peaks['src']} "
                   f"(SM clock {'at' if at_max else 'below'} max during the timed region)")
        line = {
            "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": n,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": pre["total_ms"] / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded planted-topic generator)",
            "config": {"workload": args.workload, "batch": w.batch, "seq_len": w.seq_len,
                       "heads": f"{w.n_q_heads}q/{w.n_kv_heads}kv", "head_dim": w.head_dim,
                       "routing": f"C{w.chunk_size} G{w.groups_per_chunk} sink{w.n_sink} "
                                  f"local{w.n_local} kc{w.top_k_chunks} kg{w.top_k_groups}",
                       "l2": "inputs larger than L2 (Q 512 MiB, K/V 128 MiB per step)",
                       "parallelism": f"independent sequence per rank x{n}"},
            "stage_ms": pre["stage_ms"],
            "roofline": {"kernel": "hga_attend (prefill)", "bound": "tensor",
                         "achieved": ach, "peak": tc_peak, "unit": "TFLOP/s",
                         "frac": ach / tc_peak,
                         "frac_of_sustained": ach / peaks["tc_sustained"],
                         "traffic": TC_TRAFFIC_BYTES if args.workload == "prefill_64k" else None,
                         "traffic_note": TC_TRAFFIC_NOTE if args.workload == "prefill_64k"
                         else None,
                         "flops_per_launch": pre["flops"],
                         "peak_note": tc_note},
            "planted_recall": pre["recall"],
            "gpu_launches": pre["launches_per_step"] * args.steps,
            "clocks": pre["clocks"],
        }
        if "e2e" in pre:
            e = pre["e2e"]
            line["e2e"] = {"value": n * pre["tokens"] / (e["ms"] / 1000.0), "unit": "tok/s",
                           "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"]}
        if decodes:
            line["decode"] = decodes
        if n == 1 and dist.rank == 0 and not args.no_cpu_baseline:
            cb = cpu_baseline(args)
            cb.pop("seconds")
            one = cpu_baseline(args, threads=1)
            cb["value_1_thread"] = one["value"]
            line["cpu_baseline"] = cb
        if dist.rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
