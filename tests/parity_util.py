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


def compare_selections(name, gsel, gn, rsel, rn, ref_score_of):
    """GPU vs oracle selections with the near-tie exemption. ref_score_of(p, x)
    returns the oracle fp32 score of candidate x in problem p. Returns a boolean
    array: True where the two selections are identical."""
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
                assert abs(sx - sy) <= TIE_REL * max(abs(sx), abs(sy)), (
                    f"{name}: problem {p}: gpu picked {x} (score {sx}) over {y} (score {sy})")
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
