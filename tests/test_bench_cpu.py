"""CPU tests of the benchmark's host-side arithmetic: the algorithmic FLOP
count of a prefill attention launch (the roofline numerator) and the
planted-topic recall statistic."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from long_context_rope_b200 import hga, synth  # noqa: E402


def test_prefill_flops_equals_dense_causal_when_everything_is_routed():
    # with every earlier non-forced group selected, each query token t sees
    # keys 0..t: 4*d FLOPs per (query row, visible key), rows = tokens x Hq
    w = synth.WORKLOADS["prefill_4k"].replace(seq_len=1024, top_k_chunks=1024,
                                              top_k_groups=4096)
    cfg = hga.config_from(w)
    nC, G = w.n_chunks, w.groups_per_chunk
    n_sel = np.zeros((1, w.n_kv_heads, nC), dtype=np.int64)
    for j in range(nC):
        forced = {c for c in range(j + 1) if c < w.n_sink or j - w.n_local <= c <= j}
        n_sel[..., j] = G * (j + 1 - len(forced))
    L, d, Hq = w.seq_len, w.head_dim, w.n_q_heads
    dense = 4.0 * d * Hq * (L * (L + 1) // 2)
    assert bench.prefill_flops(cfg, n_sel) == dense


def test_planted_recall_counts_forced_and_routed_sources():
    w = synth.WORKLOADS["prefill_4k"].replace(seq_len=64 * 8, n_kv_heads=1, n_q_heads=8,
                                              n_sink=1, n_local=2)
    # query chunk 6 planted from chunks 0 (sink), 5 (local), 2 and 3 (candidates)
    planted = [[[] for _ in range(8)]]
    planted[0][6] = [0, 5, 2, 3]
    sel = np.full((1, 1, 8, w.top_k_chunks), -1, dtype=np.int32)
    nsel = np.zeros((1, 1, 8), dtype=np.int32)
    sel[0, 0, 6, :2] = [1, 2]  # chunk 2 routed, chunk 3 missed
    nsel[0, 0, 6] = 2
    r = bench.planted_recall(w, planted, sel, nsel)
    assert r["planted"] == 4 and r["planted_candidates"] == 2
    assert r["visible"] == 3 / 4
    assert r["routed_among_candidates"] == 1 / 2
