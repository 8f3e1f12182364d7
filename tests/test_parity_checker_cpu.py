"""CPU tests of the parity checker itself (tests/parity_util.py), with the
oracle standing in for the GPU side. A checker that accepts a wrong routing
decision would make every GPU parity test meaningless, so mistakes are
planted in the oracle-made "GPU" results and must be caught; the legitimate
input perturbation of an end-to-end run (a q-bar moved by bf16 rounding
flips of the rotation) must be accepted."""
import numpy as np
import pytest

from long_context_rope_b200 import synth
from oracle import hga_oracle as O
from parity_util import compare_outputs, compare_routing, score_slack, topk_by_scores

KEYS = ("qbar", "chunk_sum", "group_sum", "sel_chunks", "n_sel_chunks", "chunk_scores",
        "sel_groups", "n_sel_groups", "group_scores", "out", "q_rot", "k_rot")


@pytest.fixture(scope="module")
def case():
    w = synth.WORKLOADS["prefill_4k"].replace(
        name="checker", seq_len=1024, n_q_heads=8, n_kv_heads=2, top_k_chunks=4,
        top_k_groups=12)
    x = synth.draw(w, seed=3)
    r = O.pipeline(w, x)
    return w, x, r


def _copy(r):
    return {k: np.array(r[k], copy=True) for k in KEYS}


def _rerun_from_qbar(w, r, qbar):
    """GPU-like routing from a perturbed q-bar: fp32 scores of every
    candidate, exact top-k of them, groups by the oracle on that selection."""
    cfg = O.cfg_of(w)
    g = _copy(r)
    g["qbar"] = qbar
    B, H, nQC, d = qbar.shape
    cs = r["chunk_sum"].reshape(B * H, -1, d)
    sc = g["chunk_scores"].reshape(B * H * nQC, -1)
    sel = g["sel_chunks"].reshape(B * H * nQC, -1)
    n = g["n_sel_chunks"].reshape(-1)
    for p in range(B * H * nQC):
        cand = np.flatnonzero(~np.isnan(sc[p]))
        if cand.size:
            sc[p, cand] = (cs[p // nQC][cand] @ qbar.reshape(-1, d)[p]).astype(np.float32)
        picked = topk_by_scores(sc[p], cand.tolist(), w.top_k_chunks)
        sel[p] = -1
        sel[p, :len(picked)] = picked
        n[p] = len(picked)
    sg, ng, gsc = O.route_groups(cfg, qbar, r["group_sum"], g["sel_chunks"], g["n_sel_chunks"])
    g["sel_groups"], g["n_sel_groups"], g["group_scores"] = sg, ng, gsc
    return g


def _alt(w, x, r, g):
    v = x["v"].float().numpy()
    return lambda units: O.attend(O.cfg_of(w), r["q_rot"], r["k_rot"], v, g["sel_groups"],
                                  g["n_sel_groups"], units=np.array(units, dtype=np.int32))


def test_identical_results_pass(case):
    w, x, r = case
    g = _copy(r)
    same = compare_routing(w, g, r, O)
    assert same.all()
    worst, n_alt = compare_outputs(w, g["out"], r["out"], same, _alt(w, x, r, g))
    assert worst == 0.0 and n_alt == 0


def test_planted_wrong_chunk_is_caught(case):
    """One problem picks its worst candidate instead of its best: caught."""
    w, x, r = case
    g = _copy(r)
    B, H, nQC, _ = g["qbar"].shape
    sc = g["chunk_scores"].reshape(B * H * nQC, -1)
    sel = g["sel_chunks"].reshape(B * H * nQC, -1)
    n = g["n_sel_chunks"].reshape(-1)
    p = next(p for p in range(B * H * nQC)
             if n[p] >= 1 and np.count_nonzero(~np.isnan(sc[p])) > n[p])
    cand = np.flatnonzero(~np.isnan(sc[p]))
    worst = cand[np.argmin(sc[p, cand])]
    best = sel[p, np.argmax(sc[p, sel[p, :n[p]]])]
    picked = sorted([c for c in sel[p, :n[p]] if c != best] + [worst])
    sel[p, :n[p]] = picked
    with pytest.raises(AssertionError):
        compare_routing(w, g, r, O)


def test_planted_output_error_is_caught(case):
    w, x, r = case
    g = _copy(r)
    g["out"][0, 100, 3, 7] += 0.05  # one element of one unit, above the 2e-2 bound
    same = compare_routing(w, g, r, O)
    with pytest.raises(AssertionError):
        compare_outputs(w, g["out"], r["out"], same, _alt(w, x, r, g))


def _swap_perturbation(w, r):
    """A q-bar perturbation that flips the closest level-1 decision: in the
    problem whose k-th and (k+1)-th candidates are nearest, q-bar moves along
    (row_y - row_x) by 1.5x the amount that ties them."""
    B, H, nQC, d = r["qbar"].shape
    sc = r["chunk_scores"].reshape(B * H * nQC, -1).astype(np.float64)
    cs = r["chunk_sum"].reshape(B * H, -1, d)
    k = w.top_k_chunks
    best = None
    for p in range(B * H * nQC):
        cand = np.flatnonzero(~np.isnan(sc[p]))
        if cand.size <= k:
            continue
        order = cand[np.lexsort((cand, -sc[p, cand]))]
        x, y = order[k - 1], order[k]
        gap = sc[p, x] - sc[p, y]
        if best is None or gap < best[0]:
            best = (gap, p, x, y)
    gap, p, x, y = best
    dirn = cs[p // nQC][y] - cs[p // nQC][x]
    qb = np.array(r["qbar"], copy=True).reshape(-1, d)
    qb[p] += 1.5 * (gap + 1e-6) * dirn / (dirn @ dirn)
    return qb.reshape(r["qbar"].shape), p


def test_perturbed_qbar_divergence_is_explained(case):
    """A q-bar moved just enough to flip the closest level-1 decision (and
    whatever level-2 decisions follow): the slack bound, computed from the
    measured q-bar difference, explains the swap."""
    w, x, r = case
    qb, p = _swap_perturbation(w, r)
    g = _rerun_from_qbar(w, r, qb)
    assert not np.array_equal(g["sel_chunks"].reshape(-1, w.top_k_chunks)[p],
                              r["sel_chunks"].reshape(-1, w.top_k_chunks)[p])
    same = compare_routing(w, g, r, O, slack=True)
    assert not same.reshape(-1)[p] and same.mean() > 0.9


def test_perturbed_qbar_cannot_hide_a_wrong_pick(case):
    """The same perturbation plus one planted far-off pick in another problem:
    the slack bound does not cover it."""
    w, x, r = case
    qb, p0 = _swap_perturbation(w, r)
    g = _rerun_from_qbar(w, r, qb)
    B, H, nQC, d = g["qbar"].shape
    sc = r["chunk_scores"].reshape(B * H * nQC, -1)
    sel = g["sel_chunks"].reshape(B * H * nQC, -1)
    n = g["n_sel_chunks"].reshape(-1)
    cs = r["chunk_sum"].reshape(B * H, -1, d)
    for p in range(B * H * nQC):
        cand = np.flatnonzero(~np.isnan(sc[p]))
        if p == p0 or n[p] < 1 or cand.size <= n[p]:
            continue
        worst = cand[np.argmin(sc[p, cand])]
        best = sel[p, np.argmax(sc[p, sel[p, :n[p]]])]
        slack = score_slack(qb.reshape(-1, d)[p], r["qbar"].reshape(-1, d)[p],
                            cs[p // nQC][[worst, best]], cs[p // nQC][[worst, best]])
        if sc[p, best] - sc[p, worst] > 10 * slack.sum():
            sel[p, :n[p]] = sorted([c for c in sel[p, :n[p]] if c != best] + [worst])
            break
    else:
        pytest.fail("no problem with a far-off candidate")
    with pytest.raises(AssertionError):
        compare_routing(w, g, r, O, slack=True)
