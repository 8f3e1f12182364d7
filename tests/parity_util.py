"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (stated once, used by every test):
  * outputs: max |gpu - oracle| <= 2e-2 for bf16 I/O and <= 1e-4 for fp32 I/O;
  * routing: selections identical, except that a candidate may be swapped for
    another whose oracle fp32 scores differ by <= 1e-5 relative;
  * intermediates in fp32 (summaries, q-bar, scores): |gpu - oracle| <=
    atol + rtol * |oracle| with values derived from fp32 rounding of sums of
    at most a few hundred terms (see each call).
"""
from __future__ import annotations

import numpy as np

OUT_TOL = {"bf16": 2e-2, "f32": 1e-4}
TIE_REL = 1e-5


def assert_close(name, got, ref, atol, rtol=0.0):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{name}: {bad.sum()} of {err.size} beyond tolerance; worst at {i}: "
                             f"got {got[i]!r} ref {ref[i]!r} (atol {atol}, rtol {rtol})")


def selection_sets(sel, n):
    sel = np.asarray(sel)
    n = np.asarray(n)
    flat = sel.reshape(-1, sel.shape[-1])
    nf = n.reshape(-1)
    return [tuple(flat[i, : nf[i]].tolist()) for i in range(flat.shape[0])], flat, nf


def score_slack(qbar_g, qbar_r, rows_g, rows_r):
    """Upper bound, per row, on |GPU fp32 score - oracle fp32 score| of the
    summary rows [n, d] against a routing query, when the two sides' inputs
    differ: the GPU scores fl32(qbar_g . row_g) in fp32 (any summation order
    of d terms: error <= d u sum|terms|, u = 2^-24), the oracle
    fl32(qbar_r . row_r) from a double sum (error <= u |score|), and
    qbar_g . row_g - qbar_r . row_r = (qbar_g - qbar_r) . row_r
    + qbar_g . (row_g - row_r) exactly. The differences of the inputs are the
    measured ones: the GPU's q-bar comes from its own bf16 rotation (at most
    one bf16 ulp from the oracle's in each element, checked separately) and
    its summaries are fp32 (checked to 2e-5 separately)."""
    qg = np.asarray(qbar_g, np.float64)
    qr = np.asarray(qbar_r, np.float64)
    rg = np.asarray(rows_g, np.float64)
    rr = np.asarray(rows_r, np.float64)
    u = 2.0 ** -24
    d = qg.shape[-1]
    return (np.abs(rr) @ np.abs(qg - qr) + np.abs(rg - rr) @ np.abs(qg)
            + d * u * (np.abs(rg) @ np.abs(qg)) + u * np.abs(rr @ qr))


def compare_selections(name, gsel, gn, rsel, rn, ref_score_of, slack_of=None):
    """GPU vs oracle selections with the near-tie exemption. ref_score_of(p, x)
    returns the oracle fp32 score of candidate x in problem p. A swap of x
    (GPU only) for y (oracle only) is allowed when the two oracle scores are
    within the near-tie band, plus, if slack_of is given, slack_of(p, x) +
    slack_of(p, y): the most the GPU's score of each can differ from the
    oracle's because the two sides' inputs differ (score_slack). Returns a
    boolean array: True where the two selections are identical."""
    g_sets, g_flat, g_n = selection_sets(gsel, gn)
    r_sets, r_flat, r_n = selection_sets(rsel, rn)
    same = np.zeros(len(g_sets), dtype=bool)
    for p, (a, b) in enumerate(zip(g_sets, r_sets)):
        # layout: ascending, distinct, padded with -1
        assert list(a) == sorted(set(a)), (name, p, a)
        assert np.all(g_flat[p, g_n[p]:] == -1), (name, p)
        if a == b:
            same[p] = True
            continue
        assert len(a) == len(b), (name, p, a, b)
        only_g = set(a) - set(b)
        only_r = set(b) - set(a)
        for x in only_g:
            for y in only_r:
                sx, sy = float(ref_score_of(p, x)), float(ref_score_of(p, y))
                allowed = TIE_REL * max(abs(sx), abs(sy))
                if slack_of is not None:
                    allowed += float(slack_of(p, x)) + float(slack_of(p, y))
                assert abs(sx - sy) <= allowed, (
                    f"{name}: problem {p}: gpu picked {x} (score {sx}) over {y} (score {sy}); "
                    f"allowed difference {allowed}")
    return same


def topk_by_scores(scores, candidates, k):
    """Top-k of `candidates` by (score desc, index asc; NaN last), ascending."""
    def key(c):
        s = float(scores[c])
        return (1, 0.0, c) if np.isnan(s) else (0, -s + 0.0, c)
    return tuple(sorted(sorted(candidates, key=key)[:k]))


def check_chunk_selection_matches_own_scores(gsel, gn, gscores, k):
    """Exact check of the select step: the GPU's chosen chunks are the top-k of
    the GPU's own fp32 scores (candidates = entries with a non-NaN score)."""
    g_sets, _, _ = selection_sets(gsel, gn)
    sc = np.asarray(gscores).reshape(len(g_sets), -1)
    for p, a in enumerate(g_sets):
        cand = np.flatnonzero(~np.isnan(sc[p])).tolist()
        assert a == topk_by_scores(sc[p], cand, k), (p, a)


def check_group_selection_matches_own_scores(gsel, gn, gscores, gsel_chunks, gn_chunks, G, k):
    g_sets, _, _ = selection_sets(gsel, gn)
    c_sets, _, _ = selection_sets(gsel_chunks, gn_chunks)
    sc = np.asarray(gscores).reshape(len(g_sets), -1)
    for p, a in enumerate(g_sets):
        chunks = c_sets[p]
        cand_pos = list(range(len(chunks) * G))
        by_gi = {chunks[x // G] * G + x % G: float(sc[p, x]) for x in cand_pos}
        want = topk_by_scores(by_gi, list(by_gi.keys()), k)
        assert a == want, (p, a, want)


def _flat_rows(a, n_lead):
    a = np.asarray(a)
    return a.reshape((-1,) + a.shape[n_lead:])


def compare_routing(w, g, r, oracle, slack=False):
    """Stage-by-stage routing parity of the GPU (dict g) against the oracle
    (dict r; both hold qbar, chunk_sum, group_sum, sel_chunks, n_sel_chunks,
    chunk_scores, sel_groups, n_sel_groups, group_scores).

    Chunks: every GPU selection equals the oracle's up to swaps that the
    near-tie band explains (shared inputs), or, with slack=True (each side
    rotated its own queries), that the near-tie band plus score_slack
    explains; the GPU's scores must also lie within that slack of the
    oracle's. Groups: compared conditional on the GPU's own chunk selection,
    with the oracle re-run on it ("several results correct" reading). The
    select step is also checked exactly: the GPU's picks are the top-k of its
    own scores. Returns the boolean mask (per problem) of group selections
    identical to the oracle's own."""
    kc, kg, G = w.top_k_chunks, w.top_k_groups, w.groups_per_chunk
    cfg = oracle.cfg_of(w)
    B, H, nQC, d = np.asarray(r["qbar"]).shape
    qg = np.asarray(g["qbar"], np.float64).reshape(-1, d)
    qr = np.asarray(r["qbar"], np.float64).reshape(-1, d)
    csg = _flat_rows(g["chunk_sum"], 2)   # [B*H, nC, d]
    csr = _flat_rows(r["chunk_sum"], 2)
    gsg = _flat_rows(g["group_sum"], 2)   # [B*H, nC*G, d]
    gsr = _flat_rows(r["group_sum"], 2)
    # scores of every candidate; NaN marks non-candidates identically. A path
    # that writes no scores (g["chunk_scores"] None: the one-launch decode
    # step on bf16 summary tables) is checked on its selections alone.
    has_scores = g.get("chunk_scores") is not None
    rcs = np.asarray(r["chunk_scores"], np.float64).reshape(B * H * nQC, -1)
    gcs = np.asarray(g["chunk_scores"], np.float64).reshape(B * H * nQC, -1) if has_scores else None
    if not has_scores:
        pass
    elif slack:
        assert np.array_equal(np.isnan(gcs), np.isnan(rcs))
        for p in range(B * H * nQC):
            cand = np.flatnonzero(~np.isnan(rcs[p]))
            if cand.size == 0:
                continue
            sl = score_slack(qg[p], qr[p], csg[p // nQC][cand], csr[p // nQC][cand])
            err = np.abs(gcs[p, cand] - rcs[p, cand])
            assert np.all(err <= sl * 1.0001 + 1e-30), (
                f"chunk scores of problem {p} beyond the input-perturbation bound")
    else:
        assert np.array_equal(np.isnan(gcs), np.isnan(rcs))
        rs = np.nan_to_num(rcs)
        scale = np.abs(rs).max(axis=-1, keepdims=True) + 1e-6
        assert_close("chunk scores / scale", np.nan_to_num(gcs) / scale, rs / scale, atol=2e-5)

    def slack_c(p, x):
        return score_slack(qg[p], qr[p], csg[p // nQC][x][None], csr[p // nQC][x][None])[0]

    same_c = compare_selections("chunks", g["sel_chunks"], g["n_sel_chunks"], r["sel_chunks"],
                                r["n_sel_chunks"], lambda p, x: rcs[p, x],
                                slack_c if slack else None)
    if has_scores:
        check_chunk_selection_matches_own_scores(g["sel_chunks"], g["n_sel_chunks"],
                                                 g["chunk_scores"], kc)
        check_group_selection_matches_own_scores(g["sel_groups"], g["n_sel_groups"],
                                                 g["group_scores"], g["sel_chunks"],
                                                 g["n_sel_chunks"], G, kg)
    # groups: the oracle re-run on the GPU's own chunk selection
    rsel2, rn2, rgs2 = oracle.route_groups(cfg, r["qbar"], r["group_sum"], g["sel_chunks"],
                                           g["n_sel_chunks"])
    rgs2 = np.asarray(rgs2, np.float64).reshape(B * H * nQC, -1)
    gsel_c = np.asarray(g["sel_chunks"]).reshape(-1, kc)
    if has_scores:
        ggs = np.asarray(g["group_scores"], np.float64).reshape(B * H * nQC, -1)
        assert np.array_equal(np.isnan(ggs), np.isnan(rgs2))
    if not has_scores:
        pass
    elif slack:
        for p in range(B * H * nQC):
            pos = np.flatnonzero(~np.isnan(rgs2[p]))
            if pos.size == 0:
                continue
            gi = gsel_c[p][pos // G] * G + pos % G
            sl = score_slack(qg[p], qr[p], gsg[p // nQC][gi], gsr[p // nQC][gi])
            assert np.all(np.abs(ggs[p, pos] - rgs2[p, pos]) <= sl * 1.0001 + 1e-30), (
                f"group scores of problem {p} beyond the input-perturbation bound")
    else:
        rg = np.nan_to_num(rgs2)
        gscale = np.abs(rg).max(axis=-1, keepdims=True) + 1e-6
        assert_close("group scores / scale", np.nan_to_num(ggs) / gscale, rg / gscale, atol=2e-5)

    def ref_group_score(p, gi):
        pos = list(gsel_c[p]).index(gi // G) * G + gi % G
        return rgs2[p, pos]

    def slack_g(p, gi):
        return score_slack(qg[p], qr[p], gsg[p // nQC][gi][None], gsr[p // nQC][gi][None])[0]

    compare_selections("groups", g["sel_groups"], g["n_sel_groups"], rsel2, rn2,
                       ref_group_score, slack_g if slack else None)
    same = (np.asarray(g["sel_groups"]).reshape(-1, kg) ==
            np.asarray(r["sel_groups"]).reshape(-1, kg)).all(-1)
    same &= np.asarray(g["n_sel_groups"]).reshape(-1) == np.asarray(r["n_sel_groups"]).reshape(-1)
    return same & same_c


def compare_outputs(w, g_out, r_out, same, oracle_on_gpu_selection, units=None):
    """Max-abs parity of the outputs of every unit (b, KV head, query chunk):
    against the oracle's own output where the routing agrees, and against the
    oracle run on the GPU's own selection (oracle_on_gpu_selection(units) ->
    output array) where it does not."""
    B, H, C, gq = w.batch, w.n_kv_heads, w.chunk_size, w.n_q_heads // w.n_kv_heads
    j0 = w.q_begin // C
    nQC = (w.q_begin + w.q_len - 1) // C - j0 + 1
    if units is None:
        units = [(b, h, jj) for b in range(B) for h in range(H) for jj in range(nQC)]
    units = [tuple(int(v) for v in u) for u in units]
    differ = [u for u in units if not same[(u[0] * H + u[1]) * nQC + u[2]]]
    r_alt = oracle_on_gpu_selection(differ) if differ else None
    tol = OUT_TOL[w.dtype]
    worst = 0.0
    for u in units:
        b, h, jj = u
        ref = r_out if same[(b * H + h) * nQC + jj] else r_alt
        j = j0 + jj
        t0 = max(j * C, w.q_begin) - w.q_begin
        t1 = min((j + 1) * C, w.q_begin + w.q_len) - w.q_begin
        gg = np.asarray(g_out[b, t0:t1, h * gq:(h + 1) * gq], np.float64)
        rr = np.asarray(ref[b, t0:t1, h * gq:(h + 1) * gq], np.float64)
        assert np.isfinite(gg).all() and np.isfinite(rr).all(), u
        worst = max(worst, float(np.abs(gg - rr).max()))
    assert worst <= tol, f"max abs error {worst} > {tol}"
    return worst, len(differ)
