"""The HGA hot path end to end on one GPU, through the C ABI.

Allocates the device buffers of a configuration (torch supplies the memory)
and calls the library's entry points in order:

  prefill: hga_build_summaries -> hga_route (q-bar, then both levels in one
           launch) -> hga_attend (index mode: the kernel fetches routed groups
           itself); HostPrefill does the same slice by slice from host buffers
  decode:  hga_decode_step (one launch), or hga_route -> [hga_gather_kv]
           -> hga_attend (summaries are built once beforehand, as for a KV
           cache; decode_append keeps them current in a decode loop)

Nothing here computes: every step is a kernel of libhga.so.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

from . import hga


@dataclasses.dataclass
class RouteBuffers:
    qbar: torch.Tensor
    sel_chunks: torch.Tensor
    n_sel_chunks: torch.Tensor
    sel_groups: torch.Tensor
    n_sel_groups: torch.Tensor
    chunk_scores: Optional[torch.Tensor] = None
    group_scores: Optional[torch.Tensor] = None


@dataclasses.dataclass
class WarmPool:
    """Warm tier: a VRAM pool of n_slots routed groups per (sequence, KV
    head), their tags and last-use steps, and per-call outputs."""
    k: torch.Tensor
    v: torch.Tensor
    tag: torch.Tensor
    last: torch.Tensor
    src: torch.Tensor
    stats: torch.Tensor
    step: int = 0


def alloc_warm_pool(cfg: hga.HgaConfig, n_slots: int, device="cuda") -> WarmPool:
    B, H, d, g = cfg.batch, cfg.n_kv_heads, cfg.head_dim, cfg.group_size
    i32 = dict(dtype=torch.int32, device=device)
    return WarmPool(
        k=torch.zeros(B, H, n_slots, g, d, dtype=cfg.kv_torch_dtype(), device=device),
        v=torch.zeros(B, H, n_slots, g, d, dtype=cfg.kv_torch_dtype(), device=device),
        tag=torch.full((B, H, n_slots), -1, **i32), last=torch.full((B, H, n_slots), -1, **i32),
        src=torch.empty(B, H, cfg.top_k_groups, **i32), stats=torch.zeros(B, H, 2, **i32))


def alloc_summaries(cfg: hga.HgaConfig, device="cuda"):
    B, H, d, nC, G = cfg.batch, cfg.n_kv_heads, cfg.head_dim, cfg.n_chunks, cfg.groups_per_chunk
    dt = cfg.summary_torch_dtype()
    cs = torch.empty(B, H, nC, d, dtype=dt, device=device)
    gs = torch.empty(B, H, nC * G, d, dtype=dt, device=device)
    return cs, gs


def alloc_route(cfg: hga.HgaConfig, device="cuda", with_scores: bool = False) -> RouteBuffers:
    B, H, d, nQC = cfg.batch, cfg.route_heads, cfg.head_dim, cfg.n_qchunks
    i32 = dict(dtype=torch.int32, device=device)
    rb = RouteBuffers(
        qbar=torch.empty(B, H, nQC, d, dtype=torch.float32, device=device),
        sel_chunks=torch.empty(B, H, nQC, cfg.top_k_chunks, **i32),
        n_sel_chunks=torch.empty(B, H, nQC, **i32),
        sel_groups=torch.empty(B, H, nQC, cfg.top_k_groups, **i32),
        n_sel_groups=torch.empty(B, H, nQC, **i32))
    if with_scores:
        rb.chunk_scores = torch.empty(B, H, nQC, cfg.n_chunks, dtype=torch.float32, device=device)
        rb.group_scores = torch.empty(B, H, nQC, cfg.top_k_chunks * cfg.groups_per_chunk,
                                      dtype=torch.float32, device=device)
    return rb


def alloc_gathered(cfg: hga.HgaConfig, device="cuda"):
    shape = (cfg.batch, cfg.n_kv_heads, cfg.n_qchunks, cfg.top_k_groups * cfg.group_size,
             cfg.head_dim)
    return (torch.zeros(shape, dtype=cfg.kv_torch_dtype(), device=device),
            torch.zeros(shape, dtype=cfg.kv_torch_dtype(), device=device))


def rotate_queries(cfg: hga.HgaConfig, q_raw: torch.Tensor, stream=None) -> torch.Tensor:
    q_rot = torch.empty_like(q_raw)
    hga.apply_rope(cfg, q_raw, q_rot, cfg.batch, cfg.q_len, cfg.n_q_heads, cfg.q_begin, stream)
    return q_rot


def summaries(cfg: hga.HgaConfig, k_raw, cs, gs, k_rot=None, stream=None):
    hga.build_summaries(cfg, k_raw, cs, gs, k_rot, 0, cfg.n_chunks, stream)


def route(cfg: hga.HgaConfig, q_rot, cs, gs, rb: RouteBuffers, stream=None,
          separate: bool = False):
    """Both routing levels. With score buffers (or separate=True) the two
    levels run as their own calls, which also write the scores; otherwise
    one hga_route call (decode: one launch; prefill: q-bar, then one launch
    for both levels)."""
    if separate or rb.chunk_scores is not None or rb.group_scores is not None:
        hga.route_chunks(cfg, q_rot, cs, rb.qbar, rb.sel_chunks, rb.n_sel_chunks,
                         rb.chunk_scores, stream)
        hga.route_groups(cfg, rb.qbar, gs, rb.sel_chunks, rb.n_sel_chunks, rb.sel_groups,
                         rb.n_sel_groups, rb.group_scores, stream)
    else:
        hga.route(cfg, q_rot, cs, gs, rb.qbar, rb.sel_chunks, rb.n_sel_chunks, rb.sel_groups,
                  rb.n_sel_groups, stream)


def prefill(cfg: hga.HgaConfig, k_raw, v, q_rot, cs, gs, k_rot, rb: RouteBuffers, out,
            stream=None):
    """One pass of the prefill hot path (summaries, routing, attention)."""
    summaries(cfg, k_raw, cs, gs, k_rot, stream)
    route(cfg, q_rot, cs, gs, rb, stream)
    hga.attend(cfg, q_rot, k_rot, v, rb.sel_groups, rb.n_sel_groups, out, stream=stream)


def decode(cfg: hga.HgaConfig, q_rot, cs, gs, k_res, v_res, rb: RouteBuffers, out,
           gathered=None, k_src=None, v_src=None, src_is_host=False, stream=None,
           separate: bool = False, warm: Optional[WarmPool] = None):
    """One decode step: routing, optional gather into `gathered` (k, v) from
    k_src/v_src, attention (forced chunks from k_res/v_res). Without a
    gather (full resident cache) this is one hga_decode_step call unless
    separate=True (routing and attention as their own calls)."""
    if gathered is None and not separate and rb.chunk_scores is None and rb.group_scores is None:
        hga.decode_step(cfg, q_rot, cs, gs, k_res, v_res, rb.qbar, rb.sel_chunks,
                        rb.n_sel_chunks, rb.sel_groups, rb.n_sel_groups, out, stream)
        return
    route(cfg, q_rot, cs, gs, rb, stream, separate=separate)
    if gathered is not None and warm is not None:
        # host store behind the VRAM warm tier: only pool misses cross the link
        hga.gather_kv_warm(cfg, k_src, v_src, rb.sel_groups, rb.n_sel_groups, warm.k, warm.v,
                           warm.tag, warm.last, warm.step, warm.src, gathered[0], gathered[1],
                           warm.stats, stream)
        warm.step += 1
        hga.attend(cfg, q_rot, k_res, v_res, rb.sel_groups, rb.n_sel_groups, out,
                   k_gat=gathered[0], v_gat=gathered[1], stream=stream)
    elif gathered is not None:
        hga.gather_kv(cfg, k_src, v_src, src_is_host, rb.sel_groups, rb.n_sel_groups,
                      gathered[0], gathered[1], stream)
        hga.attend(cfg, q_rot, k_res, v_res, rb.sel_groups, rb.n_sel_groups, out,
                   k_gat=gathered[0], v_gat=gathered[1], stream=stream)
    else:
        hga.attend(cfg, q_rot, k_res, v_res, rb.sel_groups, rb.n_sel_groups, out, stream=stream)


def decode_tiered(cfg_w: hga.HgaConfig, q_rot, cs, gs, k_win, v_win, k_host, v_host,
                  rb: RouteBuffers, out, stream=None):
    """One decode step over the tiered store in one launch
    (hga_decode_step_tiered): the forced chunks from the resident windows,
    the routed groups read from the host store inside the kernel."""
    hga.decode_step_tiered(cfg_w, q_rot, cs, gs, k_win, v_win, k_host, v_host, rb.qbar,
                           rb.sel_chunks, rb.n_sel_chunks, rb.sel_groups, rb.n_sel_groups, out,
                           stream)


def forced_window_chunks(cfg: hga.HgaConfig):
    """Forced chunks of the decode query chunk, ascending (the slot order of
    the HGA_KV_WINDOWS buffer)."""
    j = (cfg.seq_len - 1) // cfg.chunk_size
    s_end = min(cfg.n_sink, j + 1)
    return list(range(s_end)) + list(range(max(s_end, j - cfg.n_local), j + 1))


def fill_windows(cfg: hga.HgaConfig, k_full, v_full, k_win, v_win):
    """Copy the forced chunks of the decode query chunk from the full store
    (host or device) into the resident window buffers (device). Copies only."""
    C = cfg.chunk_size
    for w, c in enumerate(forced_window_chunks(cfg)):
        hi = min((c + 1) * C, cfg.seq_len)
        k_win[:, :, w * C: w * C + hi - c * C].copy_(k_full[:, :, c * C: hi], non_blocking=True)
        v_win[:, :, w * C: w * C + hi - c * C].copy_(v_full[:, :, c * C: hi], non_blocking=True)


def decode_append(cfg_cap: hga.HgaConfig, pos: int, k_new_raw, v_new, q_rot_new, k_raw_cache,
                  k_rot_cache, v_cache, cs, gs, rb: RouteBuffers, out, stream=None):
    """One step of a decode loop over caches of fixed capacity cfg_cap.seq_len
    ([B, Hkv, capacity, d]) at token position `pos`.

    Appends the new token (k_new_raw, v_new: [B, Hkv, d]) to the caches,
    rotates its key into the rotated cache (hga_apply_rope at position pos),
    and when the token completes its chunk, finalises that chunk's summaries
    and rotated keys (hga_build_summaries on that one chunk). Then routes and
    attends for the query q_rot_new [B, 1, Hq, d] at position pos
    (hga_decode_step with q_begin = pos, q_len = 1): routing reads only the
    summaries of chunks before the query's chunk, and attention masks keys
    after pos, so cache rows past pos are never used."""
    B, H, d = cfg_cap.batch, cfg_cap.n_kv_heads, cfg_cap.head_dim
    k_new_raw = k_new_raw.contiguous()
    k_raw_cache[:, :, pos].copy_(k_new_raw, non_blocking=True)
    v_cache[:, :, pos].copy_(v_new, non_blocking=True)
    rot = torch.empty_like(k_new_raw)
    hga.apply_rope(cfg_cap, k_new_raw, rot, B * H, 1, 1, pos, stream)
    k_rot_cache[:, :, pos].copy_(rot, non_blocking=True)
    if (pos + 1) % cfg_cap.chunk_size == 0:
        c = pos // cfg_cap.chunk_size
        hga.build_summaries(cfg_cap, k_raw_cache, cs, gs, k_rot_cache, c, c + 1, stream)
    cfg_q = cfg_cap.copy(q_begin=pos, q_len=1)
    hga.decode_step(cfg_q, q_rot_new, cs, gs, k_rot_cache, v_cache, rb.qbar, rb.sel_chunks,
                    rb.n_sel_chunks, rb.sel_groups, rb.n_sel_groups, out, stream)


def slice_bounds(n_qchunks: int, chunk_size: int, q_len: int, chunks_per_slice: int):
    """Row boundaries [0, ..., q_len] of HostPrefill's slices of a query span
    that starts on a chunk boundary: on chunk boundaries, about
    chunks_per_slice query chunks each and never fewer (all of them if there
    are fewer), so every slice is routed by the same kernel as the whole span
    would be."""
    n_sl = max(1, n_qchunks // max(1, chunks_per_slice))
    return [min(q_len, (i * n_qchunks // n_sl) * chunk_size) for i in range(n_sl)] + [q_len]


class HostPrefill:
    """Prefill whose inputs and output live in (pinned) host memory, with the
    host-link copies overlapped with the computation.

    The query span is cut into slices of at least `chunks_per_slice` query
    chunks (all of them if there are fewer), per sequence. One copy stream brings K, then the first slice's queries,
    then V, then the other slices' queries to the device; the compute stream
    builds the summaries once K has landed and routes and attends each slice
    (hga_route and hga_attend on the slice's span, q_begin / q_len) once its
    queries have landed; a second copy stream returns each slice's output as
    soon as it is computed. Host-to-device and device-to-host copies use
    separate copy engines, so after the first slice the link carries both
    directions at once and the kernels run under the copies. A slice's
    routing and attention are exactly those of the whole span restricted to
    its query chunks (every unit is independent), so the output equals the
    one-call prefill bitwise.

    Device buffers (allocated once, by torch): k_raw, v, q_rot, out of the
    whole problem, the summaries, the rotated keys and one RouteBuffers per
    slice. run() enqueues on the caller's current stream and makes it wait
    for the last output copy."""

    def __init__(self, cfg: hga.HgaConfig, chunks_per_slice: int = 64, device="cuda"):
        if cfg.q_begin % cfg.chunk_size != 0:
            raise ValueError("HostPrefill: the span must start on a chunk boundary")
        self.cfg = cfg
        B, L, Hq, d = cfg.batch, cfg.q_len, cfg.n_q_heads, cfg.head_dim
        dt = cfg.kv_torch_dtype()
        self.k_raw = torch.empty(B, cfg.n_kv_heads, cfg.seq_len, d, dtype=dt, device=device)
        self.v = torch.empty_like(self.k_raw)
        self.k_rot = torch.empty_like(self.k_raw)
        self.q_rot = torch.empty(B, L, Hq, d, dtype=dt, device=device)
        self.out = torch.empty_like(self.q_rot)
        self.cs, self.gs = alloc_summaries(cfg, device)
        self.cfg1 = cfg.copy(batch=1)
        bounds = slice_bounds(cfg.n_qchunks, cfg.chunk_size, L, chunks_per_slice)
        self.slices = []  # (b, row0, row1, cfg of the span, RouteBuffers)
        for b in range(B):
            for r0, r1 in zip(bounds[:-1], bounds[1:]):
                c = self.cfg1.copy(q_begin=cfg.q_begin + r0, q_len=r1 - r0)
                self.slices.append((b, r0, r1, c, alloc_route(c, device)))
        self.s_in = torch.cuda.Stream(device=device)
        self.s_out = torch.cuda.Stream(device=device)

    def sel_groups_of(self, b: int) -> torch.Tensor:
        """Group selections of sequence b, all slices' query chunks in order
        ([Hkv, nQC, k_g], host copy)."""
        return torch.cat([rb.sel_groups[0].cpu() for (bb, _, _, _, rb) in self.slices if bb == b],
                         dim=1)

    def run(self, hk, hv, hq, ho):
        """hk, hv [B, Hkv, L, d], hq (rotated queries) [B, q_len, Hq, d] in,
        ho [B, q_len, Hq, d] out; pinned host tensors."""
        comp = torch.cuda.current_stream()
        s_in, s_out = self.s_in, self.s_out
        s_in.wait_stream(comp)   # the device buffers are free
        s_out.wait_stream(comp)
        B = self.cfg.batch
        ev_k = [torch.cuda.Event() for _ in range(B)]
        ev_v = [torch.cuda.Event() for _ in range(B)]
        ev_q = [torch.cuda.Event() for _ in self.slices]
        ev_c = [torch.cuda.Event() for _ in self.slices]
        with torch.cuda.stream(s_in):
            for i, (b, r0, r1, _, _) in enumerate(self.slices):
                if r0 == 0:
                    self.k_raw[b].copy_(hk[b], non_blocking=True)
                    ev_k[b].record(s_in)
                self.q_rot[b, r0:r1].copy_(hq[b, r0:r1], non_blocking=True)
                ev_q[i].record(s_in)
                if r0 == 0:
                    self.v[b].copy_(hv[b], non_blocking=True)
                    ev_v[b].record(s_in)
        for i, (b, r0, r1, c, rb) in enumerate(self.slices):
            k_b, v_b, kr_b = self.k_raw[b:b + 1], self.v[b:b + 1], self.k_rot[b:b + 1]
            cs_b, gs_b = self.cs[b:b + 1], self.gs[b:b + 1]
            if r0 == 0:
                comp.wait_event(ev_k[b])
                hga.build_summaries(self.cfg1, k_b, cs_b, gs_b, kr_b, 0, self.cfg1.n_chunks)
            comp.wait_event(ev_q[i])
            q_s, o_s = self.q_rot[b:b + 1, r0:r1], self.out[b:b + 1, r0:r1]
            route(c, q_s, cs_b, gs_b, rb)
            if r0 == 0:
                comp.wait_event(ev_v[b])
            hga.attend(c, q_s, kr_b, v_b, rb.sel_groups, rb.n_sel_groups, o_s)
            ev_c[i].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c[i])
                ho[b, r0:r1].copy_(self.out[b, r0:r1], non_blocking=True)
        comp.wait_stream(s_out)
