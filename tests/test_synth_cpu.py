"""The seeded input generator (no GPU): query spans of the workloads and the
draw's independence from how a whole-context span is spelled."""
import torch

from long_context_rope_b200 import synth


def test_default_spans():
    p = synth.WORKLOADS["prefill_4k"]
    assert (p.q_begin, p.q_len) == (0, p.seq_len)
    d = synth.WORKLOADS["decode_16x32k"]
    assert (d.q_begin, d.q_len) == (d.seq_len - 1, 1)
    s = p.replace(span_begin=170, span_len=690)
    assert (s.q_begin, s.q_len) == (170, 690)


def test_explicit_whole_context_span_draws_the_same_inputs():
    w = synth.WORKLOADS["prefill_4k"].replace(seq_len=1000, n_q_heads=8, n_kv_heads=2)
    a = synth.draw(w, seed=7)
    b = synth.draw(w.replace(span_begin=0, span_len=w.seq_len), seed=7)
    for k in ("q_raw", "k_raw", "v"):
        assert torch.equal(a[k], b[k]), k
    assert a["planted"] == b["planted"]


def test_span_draw_shapes():
    w = synth.WORKLOADS["prefill_4k"].replace(seq_len=1000, n_q_heads=8, n_kv_heads=2,
                                               span_begin=170, span_len=690)
    x = synth.draw(w, seed=4)
    assert tuple(x["q_raw"].shape) == (1, 690, 8, w.head_dim)
    assert tuple(x["k_raw"].shape) == (1, 2, 1000, w.head_dim)
