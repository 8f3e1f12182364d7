"""GPU parity of the one-launch decode step (hga_decode_step) and of the
two-level hga_route.

Two bars:
  * against the separate calls (hga_route_chunks, hga_route_groups,
    hga_attend) on the same device inputs: q-bar and both selections
    bitwise identical (same fp32 dot products, exact top-k on both sides);
    outputs within 1e-2 (the two paths split the fp32 softmax sums
    differently, then round to bf16);
  * against the CPU oracle (where the oracle runs in seconds): selections
    identical up to the near-tie exemption (groups compared on the GPU's own
    chunk selection), every unit's output within the bf16 tolerance (on the
    GPU's own selection where routing differs).
The configurations cover the benchmark shape, contexts with no routing
candidates or fewer candidates than top_k_chunks, a ragged current chunk,
cluster sizes from 1 to 16, gq < 8, G = 8, and the largest top_k_chunks the
one-launch path takes (64).
"""
import numpy as np
import pytest
import torch

from long_context_rope_b200 import synth
from oracle import hga_oracle as O
from parity_util import assert_close, compare_outputs, compare_routing

pytestmark = pytest.mark.gpu

BASE = synth.WORKLOADS["decode_16x32k"]

VARIANTS = {
    "few_candidates_2k": dict(batch=2, seq_len=2048),
    "one_candidate": dict(batch=3, seq_len=64 * 5),
    "no_candidate": dict(batch=2, seq_len=64),
    "ragged_current_chunk": dict(batch=2, seq_len=64 * 200 + 48),
    "cluster16_b1": dict(batch=1, seq_len=16384),
    "cluster1_b40": dict(batch=40, seq_len=4096),
    "gq2_kc64": dict(batch=2, seq_len=8192, n_q_heads=8, n_kv_heads=4, top_k_chunks=64,
                     top_k_groups=200, n_sink=3, n_local=4),
    "g8_c128": dict(batch=2, seq_len=16384, chunk_size=128, groups_per_chunk=8,
                    top_k_chunks=16, top_k_groups=100),
}
ORACLE_VARIANTS = ["few_candidates_2k", "ragged_current_chunk", "gq2_kc64", "one_candidate"]


def _np(t):
    return t.detach().float().cpu().numpy() if t.dtype != torch.int32 else t.cpu().numpy()


def _setup(w, x, r=None):
    """GPU summaries from the raw keys; the query and the cache are the GPU's
    own rotations, or the oracle's bf16 ones when `r` is given."""
    from long_context_rope_b200 import hga, pipeline
    cfg = hga.config_from(w)
    k_raw = x["k_raw"].cuda()
    cs, gs = pipeline.alloc_summaries(cfg)
    k_rot = torch.empty_like(k_raw)
    pipeline.summaries(cfg, k_raw, cs, gs, k_rot)
    del k_raw
    q_rot = pipeline.rotate_queries(cfg, x["q_raw"].cuda())
    if r is not None:
        k_rot = torch.from_numpy(np.ascontiguousarray(r["k_rot"])).to(torch.bfloat16).cuda()
        q_rot = torch.from_numpy(np.ascontiguousarray(r["q_rot"])).to(torch.bfloat16).cuda()
    return cfg, cs, gs, k_rot, q_rot


def _run_both(w, x, r=None):
    from long_context_rope_b200 import hga, pipeline
    cfg, cs, gs, k_rot, q_rot = _setup(w, x, r)
    v = x["v"].cuda()
    rb_s = pipeline.alloc_route(cfg, with_scores=True)
    out_s = torch.full_like(q_rot, float("nan"))
    pipeline.decode(cfg, q_rot, cs, gs, k_rot, v, rb_s, out_s, separate=True)
    rb_f = pipeline.alloc_route(cfg)
    for t in (rb_f.sel_chunks, rb_f.sel_groups, rb_f.n_sel_chunks, rb_f.n_sel_groups):
        t.fill_(-7)
    out_f = torch.full_like(q_rot, float("nan"))
    pipeline.decode(cfg, q_rot, cs, gs, k_rot, v, rb_f, out_f)
    rb_r = pipeline.alloc_route(cfg)
    pipeline.route(cfg, q_rot, cs, gs, rb_r)
    torch.cuda.synchronize()
    assert hga.get_device_error() == 0
    for name in ("qbar", "sel_chunks", "n_sel_chunks", "sel_groups", "n_sel_groups"):
        a, b, c = getattr(rb_s, name), getattr(rb_f, name), getattr(rb_r, name)
        assert torch.equal(a, b), f"decode step {name} differs from the separate calls"
        assert torch.equal(a, c), f"hga_route {name} differs from the separate calls"
    assert torch.isfinite(out_f.float()).all()
    diff = (out_f.float() - out_s.float()).abs().max().item()
    assert diff <= 1e-2, f"decode step vs separate calls: max abs diff {diff}"
    # the separate calls' scores belong to the step's selections (bitwise equal)
    rb_f.chunk_scores, rb_f.group_scores = rb_s.chunk_scores, rb_s.group_scores
    return rb_f, out_f, diff, cs, gs


def _oracle_compare(w, x, r, rb, out, cs, gs):
    """Routing against the oracle (groups on the GPU's chunk selection), and
    the output of every (sequence, KV head) unit: against the oracle's own
    output where routing agrees, else the oracle run on the GPU's selection."""
    # caches of a larger capacity (decode loop): the chunks past the oracle's
    # context are not candidates (NaN scores) and their summaries unused
    nC = r["chunk_scores"].shape[-1]
    g = dict(qbar=_np(rb.qbar), chunk_sum=_np(cs)[:, :, :nC],
             group_sum=_np(gs)[:, :, :nC * w.groups_per_chunk],
             sel_chunks=_np(rb.sel_chunks), n_sel_chunks=_np(rb.n_sel_chunks),
             chunk_scores=_np(rb.chunk_scores)[..., :nC], sel_groups=_np(rb.sel_groups),
             n_sel_groups=_np(rb.n_sel_groups), group_scores=_np(rb.group_scores))
    assert np.isnan(_np(rb.chunk_scores)[..., nC:]).all()
    assert_close("qbar", g["qbar"], r["qbar"], atol=2e-5, rtol=2e-5)
    same = compare_routing(w, g, r, O)
    assert same.mean() >= 0.99, same.mean()
    v = x["v"].float().numpy()

    def oracle_alt(units):
        return O.attend(O.cfg_of(w), r["q_rot"], r["k_rot"], v, g["sel_groups"],
                        g["n_sel_groups"], units=np.array(units, dtype=np.int32))

    worst, _ = compare_outputs(w, _np(out), r["out"], same, oracle_alt)
    return worst


def test_decode_step_benchmark_shape_vs_oracle():
    w = BASE
    x = synth.draw(w, seed=4)
    r = O.pipeline(w, x)
    rb, out, diff, cs, gs = _run_both(w, x, r)
    worst = _oracle_compare(w, x, r, rb, out, cs, gs)
    print(f"decode_16x32k one-launch step: vs oracle {worst:.3e}, vs separate calls {diff:.3e}")


@pytest.mark.parametrize("name", sorted(VARIANTS))
def test_decode_step_variants(name):
    w = BASE.replace(name=name, **VARIANTS[name])
    x = synth.draw(w, seed=5)
    r = O.pipeline(w, x) if name in ORACLE_VARIANTS else None
    rb, out, diff, cs, gs = _run_both(w, x, r)
    msg = f"{name}: vs separate calls {diff:.3e}"
    if r is not None:
        msg += f", vs oracle {_oracle_compare(w, x, r, rb, out, cs, gs):.3e}"
    print(msg)


def test_decode_step_repeat_and_prefill_route():
    """Two steps in a row give identical results; hga_route on a prefill span
    (separate kernels inside) equals the two routing calls."""
    from long_context_rope_b200 import hga, pipeline
    w = BASE.replace(name="repeat", batch=4, seq_len=8192)
    x = synth.draw(w, seed=6)
    cfg, cs, gs, k_rot, q_rot = _setup(w, x)
    v = x["v"].cuda()
    res = []
    for _ in range(2):
        rb = pipeline.alloc_route(cfg)
        out = torch.empty_like(q_rot)
        pipeline.decode(cfg, q_rot, cs, gs, k_rot, v, rb, out)
        res.append((rb, out))
    torch.cuda.synchronize()
    assert torch.equal(res[0][1], res[1][1])
    assert torch.equal(res[0][0].sel_groups, res[1][0].sel_groups)

    # prefill: hga_route runs both levels in one launch after q-bar (the tiled
    # chunk router with level 2 fused); the separate calls must agree bitwise
    base = synth.WORKLOADS["prefill_4k"]
    for wp in (base,
               base.replace(batch=2, seq_len=1500, n_q_heads=8, n_kv_heads=2, top_k_chunks=5,
                            top_k_groups=13, n_local=1, n_sink=1),
               base.replace(seq_len=4000, chunk_size=128, groups_per_chunk=8, top_k_chunks=16,
                            top_k_groups=60)):
        xp = synth.draw(wp, seed=1)
        cfgp = hga.config_from(wp)
        k_raw = xp["k_raw"].cuda()
        csp, gsp = pipeline.alloc_summaries(cfgp)
        pipeline.summaries(cfgp, k_raw, csp, gsp, None)
        qp = pipeline.rotate_queries(cfgp, xp["q_raw"].cuda())
        rb1 = pipeline.alloc_route(cfgp)
        pipeline.route(cfgp, qp, csp, gsp, rb1, separate=True)
        rb2 = pipeline.alloc_route(cfgp)
        pipeline.route(cfgp, qp, csp, gsp, rb2)
        torch.cuda.synchronize()
        assert hga.get_device_error() == 0
        for name in ("qbar", "sel_chunks", "n_sel_chunks", "sel_groups", "n_sel_groups"):
            assert torch.equal(getattr(rb1, name), getattr(rb2, name)), (wp.seq_len, name)


def test_decode_loop_appends_and_finalises_chunks():
    """A decode loop over caches of fixed capacity (pipeline.decode_append):
    each step appends a token, rotates its key into the cache, finalises the
    summaries of the chunk it completes, and routes + attends at its position
    with the one-launch step. Checked against the oracle run from scratch on
    the prefix up to that position, at steps around two chunk ends; with no
    local window, the chunk finished at position 1343 is a routing candidate
    at position 1344, so its freshly built summary is used."""
    from long_context_rope_b200 import hga, pipeline
    cap = 64 * 24
    wp = BASE.replace(name="loop", batch=2, seq_len=cap, mode="prefill", n_local=0,
                      plant_every=1, plant_count=2)
    x = synth.draw(wp, seed=7)  # keys, values and queries at every position
    cfg_cap = hga.config_from(wp)
    L0 = 64 * 20 - 3
    B, H, d = wp.batch, wp.n_kv_heads, wp.head_dim
    k_raw_cache = torch.zeros(B, H, cap, d, dtype=torch.bfloat16, device="cuda")
    v_cache = torch.zeros_like(k_raw_cache)
    k_raw_cache[:, :, :L0] = x["k_raw"][:, :, :L0].cuda()
    v_cache[:, :, :L0] = x["v"][:, :, :L0].cuda()
    k_rot_cache = torch.zeros_like(k_raw_cache)
    cs, gs = pipeline.alloc_summaries(cfg_cap)
    hga.build_summaries(cfg_cap, k_raw_cache, cs, gs, k_rot_cache, 0, L0 // 64 + 1)
    check = {L0, 64 * 20 - 1, 64 * 20, 64 * 20 + 1, 64 * 21 - 1, 64 * 21, 64 * 21 + 1}
    n_checked = 0
    for pos in range(L0, 64 * 21 + 2):
        cfg_q = cfg_cap.copy(q_begin=pos, q_len=1)
        r = None
        if pos in check:
            w_pos = wp.replace(seq_len=pos + 1, mode="decode")
            r = O.pipeline(w_pos, {"k_raw": x["k_raw"][:, :, :pos + 1], "v": x["v"][:, :, :pos + 1],
                                   "q_raw": x["q_raw"][:, pos:pos + 1]})
            q_rot = torch.from_numpy(np.ascontiguousarray(r["q_rot"])).to(torch.bfloat16).cuda()
        else:
            q_rot = pipeline.rotate_queries(cfg_q, x["q_raw"][:, pos:pos + 1].cuda())
        rb = pipeline.alloc_route(cfg_q)
        out = torch.full_like(q_rot, float("nan"))
        pipeline.decode_append(cfg_cap, pos, x["k_raw"][:, :, pos].cuda(), x["v"][:, :, pos].cuda(),
                               q_rot, k_raw_cache, k_rot_cache, v_cache, cs, gs, rb, out)
        if r is not None:
            # the separate routing calls with scores on the same inputs: the
            # same selections (bitwise), and the scores the comparison needs
            rb_sc = pipeline.alloc_route(cfg_q, with_scores=True)
            pipeline.route(cfg_q, q_rot, cs, gs, rb_sc, separate=True)
            torch.cuda.synchronize()
            assert hga.get_device_error() == 0
            for name in ("qbar", "sel_chunks", "n_sel_chunks", "sel_groups", "n_sel_groups"):
                assert torch.equal(getattr(rb, name), getattr(rb_sc, name)), name
            rb.chunk_scores, rb.group_scores = rb_sc.chunk_scores, rb_sc.group_scores
            w_pos = wp.replace(seq_len=pos + 1, mode="decode")
            worst = _oracle_compare(w_pos, {"v": x["v"][:, :, :pos + 1]}, r, rb, out, cs, gs)
            n_checked += 1
            print(f"pos {pos}: chunks {int(rb.n_sel_chunks[0, 0, 0])} groups "
                  f"{int(rb.n_sel_groups[0, 0, 0])} max abs error {worst:.3e}")
    assert n_checked == len(check)


def test_decode_step_bf16_summaries_vs_oracle():
    """bf16 summary tables (the variant that halves the routing bytes of a
    decode step): hga_build_summaries writes the fp32 summaries rounded to
    bf16, and the one-launch step routes on them. The oracle's reading is its
    double summaries rounded to bf16 (nearest even, through fp32); the GPU's
    tables are equal up to one bf16 ulp where the fp32 and double sums fall on
    either side of a rounding boundary, so routing is compared with the
    slack bound of those measured differences (tests/parity_util.py), and
    every output against the oracle on the GPU's selection where it
    differs. The separate routing calls refuse bf16 tables."""
    from long_context_rope_b200 import hga, pipeline
    w = BASE.replace(name="bf16sum", batch=4, seq_len=16384)
    x = synth.draw(w, seed=8)
    r = O.pipeline(w, x, bf16_summaries=True)
    cfg = hga.config_from(w, summary_type=hga.HGA_SUMMARY_BF16)
    k_raw = x["k_raw"].cuda()
    cs, gs = pipeline.alloc_summaries(cfg)
    assert cs.dtype == torch.bfloat16
    pipeline.summaries(cfg, k_raw, cs, gs, None)
    k_rot = torch.from_numpy(np.ascontiguousarray(r["k_rot"])).to(torch.bfloat16).cuda()
    q_rot = torch.from_numpy(np.ascontiguousarray(r["q_rot"])).to(torch.bfloat16).cuda()
    v = x["v"].cuda()
    rb = pipeline.alloc_route(cfg)
    out = torch.full_like(q_rot, float("nan"))
    pipeline.decode(cfg, q_rot, cs, gs, k_rot, v, rb, out)
    torch.cuda.synchronize()
    assert hga.get_device_error() == 0
    # a GPU table value is the bf16 rounding of an fp32 summary within the
    # fp32 tolerance (2e-5 abs + rel) of the oracle's double one, so it lies
    # within that tolerance plus one bf16 ulp of the oracle's rounded value
    for name, got, want in (("chunk_sum", cs, r["chunk_sum"]), ("group_sum", gs, r["group_sum"])):
        got = _np(got).astype(np.float64)
        diff = got != want
        bound = 2e-5 * (1.0 + np.abs(want)) + np.abs(want) * 2.0 ** -7
        assert np.all(np.abs(got - want) <= bound), name
        assert diff.mean() <= 1e-3, (name, diff.mean())
    g = dict(qbar=_np(rb.qbar), chunk_sum=_np(cs), group_sum=_np(gs),
             sel_chunks=_np(rb.sel_chunks), n_sel_chunks=_np(rb.n_sel_chunks), chunk_scores=None,
             sel_groups=_np(rb.sel_groups), n_sel_groups=_np(rb.n_sel_groups), group_scores=None)
    assert_close("qbar", g["qbar"], r["qbar"], atol=2e-5, rtol=2e-5)
    same = compare_routing(w, g, r, O, slack=True)
    assert same.mean() >= 0.9, same.mean()
    vv = x["v"].float().numpy()

    def oracle_alt(units):
        return O.attend(O.cfg_of(w), r["q_rot"], r["k_rot"], vv, g["sel_groups"],
                        g["n_sel_groups"], units=np.array(units, dtype=np.int32))

    worst, n_alt = compare_outputs(w, _np(out), r["out"], same, oracle_alt)
    rb2 = pipeline.alloc_route(cfg, with_scores=True)
    with pytest.raises(hga.HgaError) as e:
        pipeline.route(cfg, q_rot, cs, gs, rb2, separate=True)
    assert e.value.status == -8
    print(f"bf16 summaries: {same.mean():.3f} identical routing ({n_alt} units on the GPU's "
          f"selection), max abs error {worst:.3e}")
