"""GPU tests of the warm tier (hga_gather_kv_warm): a VRAM pool of recently
routed groups between the host store and attention.

Over a sequence of decode queries (repeats, new routes, evictions from a
pool smaller than two routes) every call must give bitwise the same gathered
K/V as the cold gather from host memory, the same attention output (and that
output within the bf16 tolerance of the CPU oracle's attention over the same
selection, from the oracle's own rotations), and pool
tags, last-use steps and hit / miss counts equal to a plain-Python model of
the rule: hits keep their slots; the i-th miss in list order takes the i-th
victim, victims being the slots not hit this call with the oldest last use
(never used first, ties to the lower slot), in ascending slot order."""
import numpy as np
import pytest
import torch

from long_context_rope_b200 import synth
from oracle import hga_oracle as O
from parity_util import OUT_TOL

pytestmark = pytest.mark.gpu


def _lru_model(S, sels):
    tags, last = [-1] * S, [-1] * S
    out = []
    for step, sel in enumerate(sels):
        where = {tags[t]: t for t in range(S) if tags[t] >= 0}
        hit_slots = {where[g] for g in sel if g in where}
        misses = [g for g in sel if g not in where]
        cand = sorted((t for t in range(S) if t not in hit_slots), key=lambda t: (last[t], t))
        victims = sorted(cand[:len(misses)])
        for g in sel:
            if g in where:
                last[where[g]] = step
        for g, v in zip(misses, victims):
            tags[v], last[v] = g, step
        out.append((len(sel) - len(misses), len(misses), list(tags), list(last)))
    return out


def test_warm_tier_matches_cold_gather_and_lru_model():
    from long_context_rope_b200 import hga, pipeline
    w = synth.WORKLOADS["tiered_decode_4x64k"].replace(name="warm", batch=2, seq_len=16384)
    x = synth.draw(w, seed=11)
    queries = [x["q_raw"]] + [synth.draw(w, seed=s, with_kv=False)["q_raw"] for s in (12, 13)]
    order = [0, 0, 1, 2, 0, 1, 1, 2]
    cfg = hga.config_from(w)
    k_raw = x["k_raw"].cuda()
    cs, gs = pipeline.alloc_summaries(cfg)
    k_rot = torch.empty_like(k_raw)
    pipeline.summaries(cfg, k_raw, cs, gs, k_rot)
    del k_raw
    k_host = torch.empty(k_rot.shape, dtype=k_rot.dtype, pin_memory=True)
    k_host.copy_(k_rot)
    v_host = x["v"].pin_memory()
    W = hga.window_slots(cfg)
    shape = (w.batch, w.n_kv_heads, W * w.chunk_size, w.head_dim)
    k_win = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    v_win = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    pipeline.fill_windows(cfg, k_host, v_host, k_win, v_win)
    cfg_w = cfg.copy(kv_layout=hga.HGA_KV_WINDOWS)
    S = 128  # smaller than two routes of 96 groups: evictions happen
    pool = pipeline.alloc_warm_pool(cfg, S)
    sels = {}
    # the oracle's own bf16 rotations of the keys and of each query
    ocfg = O.cfg_of(w)
    ref = O.pipeline(w, x, want_scores=False, attend_out=False)
    q_ref = [np.stack([O.rope_f32(ocfg, q[b].float().numpy(), ocfg.q_begin, True)
                       for b in range(w.batch)]) for q in queries]
    v_np = x["v"].float().numpy()
    worst = 0.0
    for step, qi in enumerate(order):
        q_rot = pipeline.rotate_queries(cfg, queries[qi].cuda())
        rb = pipeline.alloc_route(cfg)
        gat_w, gat_c = pipeline.alloc_gathered(cfg), pipeline.alloc_gathered(cfg)
        out_w, out_c = torch.empty_like(q_rot), torch.empty_like(q_rot)
        pipeline.decode(cfg_w, q_rot, cs, gs, k_win, v_win, rb, out_w, gathered=gat_w,
                        k_src=k_host, v_src=v_host, src_is_host=True, warm=pool)
        hga.gather_kv(cfg_w, k_host, v_host, True, rb.sel_groups, rb.n_sel_groups, gat_c[0],
                      gat_c[1])
        hga.attend(cfg_w, q_rot, k_win, v_win, rb.sel_groups, rb.n_sel_groups, out_c,
                   k_gat=gat_c[0], v_gat=gat_c[1])
        torch.cuda.synchronize()
        assert hga.get_device_error() == 0
        n = rb.n_sel_groups.cpu().numpy().reshape(-1)
        for u in range(w.batch * w.n_kv_heads):
            b, h = divmod(u, w.n_kv_heads)
            rows = int(n[u]) * 16
            for a, c in ((gat_w[0], gat_c[0]), (gat_w[1], gat_c[1])):
                assert torch.equal(a[b, h, 0, :rows], c[b, h, 0, :rows]), (step, u)
            sel = rb.sel_groups[b, h, 0, :n[u]].tolist()
            sels.setdefault(u, []).append(sel)
        assert torch.equal(out_w, out_c), step
        # the oracle's attention over the GPU's own selection of this step
        r_out = O.attend(ocfg, q_ref[qi], ref["k_rot"], v_np, rb.sel_groups.cpu().numpy(),
                         rb.n_sel_groups.cpu().numpy())
        err = float(np.abs(out_w.float().cpu().numpy() - r_out).max())
        assert err <= OUT_TOL["bf16"], (step, err)
        worst = max(worst, err)
        model_stats = pool.stats.cpu().numpy().reshape(-1, 2)
        tags, last = pool.tag.cpu().numpy(), pool.last.cpu().numpy()
        for u in range(w.batch * w.n_kv_heads):
            b, h = divmod(u, w.n_kv_heads)
            hits, misses, mtags, mlast = _lru_model(S, sels[u])[-1]
            assert tuple(model_stats[u]) == (hits, misses), (step, u, model_stats[u], hits, misses)
            assert np.array_equal(tags[b, h], mtags), (step, u)
            assert np.array_equal(last[b, h], mlast), (step, u)
        print(f"step {step} query {qi}: hits {model_stats[:, 0].sum()} misses "
              f"{model_stats[:, 1].sum()}")
    st = _lru_model(S, sels[0])
    assert st[1][1] == 0, "a repeated query must hit every group"
    print(f"warm tier vs oracle on the GPU's selections: max abs error {worst:.3e}")
