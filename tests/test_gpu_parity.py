"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Every input comes from the seeded generator; each side computes every
intermediate itself (the oracle never receives a value the GPU produced).
Stages compared: rotated queries and keys, chunk and group summaries, q-bar,
routing scores, selections (with the near-tie exemption; groups on the GPU's
own chunk selection), and the outputs of every unit (on the GPU's own
selection where routing differs). Tolerances: tests/parity_util.py.
"""
import numpy as np
import pytest
import torch

from long_context_rope_b200 import synth
from oracle import hga_oracle as O
from parity_util import assert_close, compare_outputs, compare_routing

pytestmark = pytest.mark.gpu


def _mods():
    from long_context_rope_b200 import hga, pipeline
    return hga, pipeline


def _np(t):
    return t.detach().float().cpu().numpy() if t.dtype != torch.int32 else t.cpu().numpy()


def bf16_ulp_check(name, got, ref, max_frac=1e-3):
    """Rounded-to-bf16 values from two computations of the same real number
    (an fp32 rotation on the GPU, a double one in the oracle): equal, or one
    bf16 ulp apart, in a small fraction of elements. Near cancellation the
    fp32 rotation carries an absolute error of a few 1e-7 times the input
    magnitude (inputs here are O(10) at most), hence the 1e-5 floor."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = got != ref
    ulp = np.abs(ref) * 2.0 ** -7 + 1e-5
    assert np.all(np.abs(got - ref)[diff] <= ulp[diff] * 1.0001), f"{name}: beyond one bf16 ulp"
    assert diff.mean() <= max_frac, f"{name}: {diff.mean():.2e} of elements differ"


def _bf16_or_f32(w, a):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(w.torch_dtype())


def run_gpu_prefill(w, x, r=None):
    """The GPU prefill path. Rotation and summaries start from the raw drawn
    inputs. When the oracle's results `r` are given, routing and attention
    take the oracle's bf16 rotated queries and keys as their inputs (the
    queries arrive rotated at the routing boundary; sharing them keeps bf16
    rounding-boundary flips of the two rotations out of the routing decisions);
    the GPU's own rotations are compared separately."""
    hga, pipeline = _mods()
    cfg = hga.config_from(w)
    k_raw, v, q_raw = (x[n].cuda() for n in ("k_raw", "v", "q_raw"))
    q_rot = pipeline.rotate_queries(cfg, q_raw)
    cs, gs = pipeline.alloc_summaries(cfg)
    k_rot = torch.empty_like(k_raw)
    rb = pipeline.alloc_route(cfg, with_scores=True)
    out = torch.full_like(q_rot, float("nan"))
    pipeline.summaries(cfg, k_raw, cs, gs, k_rot)
    q_use = _bf16_or_f32(w, r["q_rot"]).cuda() if r is not None else q_rot
    k_use = _bf16_or_f32(w, r["k_rot"]).cuda() if r is not None else k_rot
    pipeline.route(cfg, q_use, cs, gs, rb)
    hga.attend(cfg, q_use, k_use, v, rb.sel_groups, rb.n_sel_groups, out)
    assert hga.get_device_error() == 0
    return dict(q_rot=_np(q_rot), k_rot=_np(k_rot), chunk_sum=_np(cs), group_sum=_np(gs),
                qbar=_np(rb.qbar), sel_chunks=_np(rb.sel_chunks), n_sel_chunks=_np(rb.n_sel_chunks),
                chunk_scores=_np(rb.chunk_scores), sel_groups=_np(rb.sel_groups),
                n_sel_groups=_np(rb.n_sel_groups), group_scores=_np(rb.group_scores),
                out=_np(out))


def _oracle_on_gpu_selection(w, r, v, g):
    """The oracle's attention (its own bf16 rotations) over the GPU's own
    group selection, for the given units."""
    def run(units):
        return O.attend(O.cfg_of(w), r["q_rot"], r["k_rot"], v, g["sel_groups"],
                        g["n_sel_groups"], units=np.array(units, dtype=np.int32))
    return run


def compare_prefill(w, x, units=None):
    r = O.pipeline(w, x, units=units)
    g = run_gpu_prefill(w, x, r)
    rot_check = (lambda n, a, b: bf16_ulp_check(n, a, b)) if w.dtype == "bf16" else (
        lambda n, a, b: assert_close(n, a, b, atol=1e-5, rtol=1e-6))
    rot_check("q_rot", g["q_rot"], r["q_rot"])
    rot_check("k_rot", g["k_rot"], r["k_rot"])
    assert_close("chunk_sum", g["chunk_sum"], r["chunk_sum"], atol=2e-5, rtol=2e-5)
    assert_close("group_sum", g["group_sum"], r["group_sum"], atol=2e-5, rtol=2e-5)
    assert_close("qbar", g["qbar"], r["qbar"], atol=2e-5, rtol=2e-5)
    same = compare_routing(w, g, r, O)
    assert same.mean() >= 0.99, f"only {same.mean():.3f} of problems route identically"
    worst, n_alt = compare_outputs(w, g["out"], r["out"], same,
                                   _oracle_on_gpu_selection(w, r, _np_v(x), g), units)
    return worst


def _np_v(x):
    return x["v"].float().numpy()


@pytest.mark.parametrize("name", ["tiny_f32", "prefill_4k"])
def test_prefill_parity_full(name):
    w = synth.WORKLOADS[name]
    x = synth.draw(w, seed=0)
    worst = compare_prefill(w, x)
    print(f"{name}: max abs error {worst:.3e}")


def test_prefill_end_to_end_from_raw_inputs():
    """Everything from the raw drawn inputs on both sides: each side rotates
    its own queries and keys, so the GPU's q-bar differs from the oracle's by
    the bf16 rounding flips of its fp32 rotation (each at most one bf16 ulp,
    checked here). Every routing decision that differs from the oracle's must
    be explained by that input difference: the two oracle scores of each
    swapped pair lie within the near-tie band plus the score perturbation the
    measured q-bar and summary differences can cause (score_slack, which
    also bounds the GPU's score of every candidate). Groups are compared on
    the GPU's chunk selection (the oracle re-run on it); every unit's output
    is compared, on the GPU's selection where it differs."""
    w = synth.WORKLOADS["prefill_4k"]
    x = synth.draw(w, seed=2)
    r = O.pipeline(w, x)
    g = run_gpu_prefill(w, x)
    bf16_ulp_check("q_rot", g["q_rot"], r["q_rot"])
    bf16_ulp_check("k_rot", g["k_rot"], r["k_rot"])
    assert_close("chunk_sum", g["chunk_sum"], r["chunk_sum"], atol=2e-5, rtol=2e-5)
    assert_close("group_sum", g["group_sum"], r["group_sum"], atol=2e-5, rtol=2e-5)
    same = compare_routing(w, g, r, O, slack=True)
    assert same.mean() >= 0.95, same.mean()

    def oracle_alt(units):  # the oracle's rotations, the GPU's selection
        return O.attend(O.cfg_of(w), r["q_rot"], r["k_rot"], _np_v(x), g["sel_groups"],
                        g["n_sel_groups"], units=np.array(units, dtype=np.int32))

    worst, n_alt = compare_outputs(w, g["out"], r["out"], same, oracle_alt)
    print(f"end-to-end: {same.mean():.4f} identical routing ({n_alt} units on the GPU's "
          f"selection), max abs error {worst:.3e}")


@pytest.mark.parametrize("L,F,dtype", [(1000, 32, "bf16"), (16 * 64 + 16 * 5 + 3, 7, "bf16"),
                                       (777, 9, "f32")])
def test_prefill_parity_ragged_small(L, F, dtype):
    """Ragged context (L % C != 0), several tiles, fewer heads, odd F."""
    w = synth.WORKLOADS["prefill_4k"].replace(
        name="ragged", seq_len=L, n_q_heads=8, n_kv_heads=2, n_high_freq_pairs=F, dtype=dtype,
        top_k_chunks=5, top_k_groups=13, n_local=1, n_sink=2)
    if dtype == "f32":
        w = w.replace(head_dim=64)
    x = synth.draw(w, seed=3)
    compare_prefill(w, x)


def test_prefill_parity_batch2():
    """Two sequences in one call (ragged length, reduced heads): the second
    sequence's units, query rows and key rows in every prefill kernel."""
    w = synth.WORKLOADS["prefill_4k"].replace(
        name="batch2", batch=2, seq_len=968, n_q_heads=16, n_kv_heads=2, top_k_chunks=4,
        top_k_groups=11, n_local=1, n_sink=1)
    x = synth.draw(w, seed=5)
    compare_prefill(w, x)


def test_prefill_parity_chunked_span():
    """A prefill span that starts and ends inside chunks (a chunked prefill,
    tokens [170, 860) of 1000): the attention kernel skips the 32-token query
    pairs that lie wholly before or after the span and masks the rows of the
    partial M tiles at both ends; routing starts at query chunk 2."""
    w = synth.WORKLOADS["prefill_4k"].replace(
        name="span", seq_len=1000, n_q_heads=8, n_kv_heads=2, top_k_chunks=5, top_k_groups=13,
        n_local=1, n_sink=2, span_begin=170, span_len=690)
    assert (w.q_begin, w.q_len) == (170, 690)
    x = synth.draw(w, seed=4)
    compare_prefill(w, x)


@pytest.mark.parametrize("span", [None, (256, 1244)])
def test_host_prefill_overlapped_equals_one_call(span):
    """pipeline.HostPrefill (inputs and output in pinned host memory, the copies
    overlapped with slice-by-slice routing and attention on other streams):
    two sequences, ragged length (24 query chunks each, the last one partial),
    two slices of 12 query chunks per sequence; or a chunked-prefill span from
    token 256 (20 query chunks: slices of 10). Its output must equal the
    one-call prefill on device buffers bitwise, and that one the oracle
    (compare_prefill on the same inputs)."""
    hga, pipeline = _mods()
    w = synth.WORKLOADS["prefill_4k"].replace(
        name="host_prefill", batch=2, seq_len=1500, n_q_heads=8, n_kv_heads=2, top_k_chunks=5,
        top_k_groups=13, n_local=1, n_sink=1)
    if span is not None:
        w = w.replace(span_begin=span[0], span_len=span[1])
    x = synth.draw(w, seed=6)
    cfg = hga.config_from(w)
    k_raw, v = x["k_raw"].cuda(), x["v"].cuda()
    q_rot = pipeline.rotate_queries(cfg, x["q_raw"].cuda())
    cs, gs = pipeline.alloc_summaries(cfg)
    k_rot = torch.empty_like(k_raw)
    rb = pipeline.alloc_route(cfg)
    out = torch.full_like(q_rot, float("nan"))
    pipeline.prefill(cfg, k_raw, v, q_rot, cs, gs, k_rot, rb, out)
    hp = pipeline.HostPrefill(cfg, chunks_per_slice=10)
    want = [(0, 768), (768, 1500)] if span is None else [(0, 640), (640, 1244)]
    assert [(r0, r1) for (_, r0, r1, _, _) in hp.slices] == want * 2
    hk, hv, hq = (t.cpu().pin_memory() for t in (k_raw, v, q_rot))
    ho = torch.full(out.shape, float("nan"), dtype=out.dtype).pin_memory()
    for _ in range(2):  # the second run reuses every buffer
        hp.run(hk, hv, hq, ho)
        torch.cuda.synchronize()
        assert hga.get_device_error() == 0
        assert torch.equal(ho, out.cpu()), "overlapped host prefill differs from the one-call prefill"
    assert torch.equal(hp.sel_groups_of(0), rb.sel_groups[0].cpu())
    compare_prefill(w, x)


def test_prefill_64k_sampled():
    """The 64K-context workload at full size: every rotation, summary, score
    and selection, and the outputs of 64 sampled (KV head, query chunk) units."""
    w = synth.WORKLOADS["prefill_64k"]
    x = synth.draw(w, seed=0)
    rng = np.random.default_rng(0)
    nQC = w.n_chunks
    units = np.array([[0, int(rng.integers(0, w.n_kv_heads)), int(j)]
                      for j in sorted(rng.choice(nQC, size=64, replace=False))])
    units[:4, 2] = [0, 1, nQC - 2, nQC - 1]
    worst = compare_prefill(w, x, units=units)
    print(f"prefill_64k sampled: max abs error {worst:.3e}")


def _decode_setup(w, x, r):
    """GPU summaries from the raw keys; the decode query and the attention
    cache are the oracle's bf16 rotated values (see run_gpu_prefill); the
    GPU's own rotations are compared against them here."""
    hga, pipeline = _mods()
    cfg = hga.config_from(w)
    k_raw = x["k_raw"].cuda()
    cs, gs = pipeline.alloc_summaries(cfg)
    k_rot = torch.empty_like(k_raw)
    pipeline.summaries(cfg, k_raw, cs, gs, k_rot)
    del k_raw
    q_gpu = pipeline.rotate_queries(cfg, x["q_raw"].cuda())
    bf16_ulp_check("k_rot", _np(k_rot), r["k_rot"])
    bf16_ulp_check("q_rot", _np(q_gpu), r["q_rot"])
    k_rot = _bf16_or_f32(w, r["k_rot"]).cuda()
    q_rot = _bf16_or_f32(w, r["q_rot"]).cuda()
    return cfg, cs, gs, k_rot, q_rot


def _decode_compare(w, x, r, g_out, rb, cs, gs):
    g = dict(qbar=_np(rb.qbar), chunk_sum=_np(cs), group_sum=_np(gs),
             sel_chunks=_np(rb.sel_chunks), n_sel_chunks=_np(rb.n_sel_chunks),
             chunk_scores=_np(rb.chunk_scores), sel_groups=_np(rb.sel_groups),
             n_sel_groups=_np(rb.n_sel_groups), group_scores=_np(rb.group_scores))
    assert_close("qbar", g["qbar"], r["qbar"], atol=2e-5, rtol=2e-5)
    same = compare_routing(w, g, r, O)
    assert same.mean() >= 0.99, same.mean()
    worst, _ = compare_outputs(w, _np(g_out), r["out"], same,
                               _oracle_on_gpu_selection(w, r, _np_v(x), g))
    return worst


@pytest.mark.parametrize("mode", ["index", "gathered"])
def test_decode_16x32k(mode):
    hga, pipeline = _mods()
    w = synth.WORKLOADS["decode_16x32k"]
    x = synth.draw(w, seed=0)
    r = O.pipeline(w, x)
    cfg, cs, gs, k_rot, q_rot = _decode_setup(w, x, r)
    v = x["v"].cuda()
    rb = pipeline.alloc_route(cfg, with_scores=True)
    out = torch.full_like(q_rot, float("nan"))
    if mode == "index":
        pipeline.decode(cfg, q_rot, cs, gs, k_rot, v, rb, out)
    else:
        gat = pipeline.alloc_gathered(cfg)
        pipeline.decode(cfg, q_rot, cs, gs, k_rot, v, rb, out, gathered=gat, k_src=k_rot,
                        v_src=v)
    assert hga.get_device_error() == 0
    worst = _decode_compare(w, x, r, out, rb, cs, gs)
    print(f"decode {mode}: max abs error {worst:.3e}")


def test_tiered_decode_4x64k():
    """Cold tier in pinned host memory; only the summaries and the forced
    windows resident in HBM; routed groups gathered over the host link."""
    hga, pipeline = _mods()
    w = synth.WORKLOADS["tiered_decode_4x64k"]
    x = synth.draw(w, seed=0)
    r = O.pipeline(w, x)
    cfg, cs, gs, k_rot, q_rot = _decode_setup(w, x, r)
    k_host = torch.empty(k_rot.shape, dtype=k_rot.dtype, pin_memory=True)
    k_host.copy_(k_rot)
    v_host = x["v"].pin_memory()
    del k_rot
    cfg_w = cfg.copy(kv_layout=hga.HGA_KV_WINDOWS)
    W = hga.window_slots(cfg)
    shape = (w.batch, w.n_kv_heads, W * w.chunk_size, w.head_dim)
    k_win = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    v_win = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    pipeline.fill_windows(cfg, k_host, v_host, k_win, v_win)
    rb = pipeline.alloc_route(cfg, with_scores=True)
    gat = pipeline.alloc_gathered(cfg)
    out = torch.full_like(q_rot, float("nan"))
    pipeline.decode(cfg_w, q_rot, cs, gs, k_win, v_win, rb, out, gathered=gat, k_src=k_host,
                    v_src=v_host, src_is_host=True)
    assert hga.get_device_error() == 0
    worst = _decode_compare(w, x, r, out, rb, cs, gs)
    # the same step in one launch (hga_decode_step_tiered): routed groups read
    # from the host store inside the attention kernel, nothing gathered
    rb_f = pipeline.alloc_route(cfg)
    out_f = torch.full_like(q_rot, float("nan"))
    pipeline.decode_tiered(cfg_w, q_rot, cs, gs, k_win, v_win, k_host, v_host, rb_f, out_f)
    torch.cuda.synchronize()
    assert hga.get_device_error() == 0
    for name in ("qbar", "sel_chunks", "n_sel_chunks", "sel_groups", "n_sel_groups"):
        assert torch.equal(getattr(rb_f, name), getattr(rb, name)), name
    rb_f.chunk_scores, rb_f.group_scores = rb.chunk_scores, rb.group_scores
    worst_f = _decode_compare(w, x, r, out_f, rb_f, cs, gs)
    diff = (out_f.float() - out.float()).abs().max().item()
    assert diff <= 1e-2, diff
    print(f"tiered decode: max abs error {worst:.3e}; one launch {worst_f:.3e} "
          f"(vs three launches {diff:.3e})")


def test_incremental_summaries_bitwise():
    """Building the summaries chunk range by chunk range equals one build."""
    hga, pipeline = _mods()
    w = synth.WORKLOADS["prefill_4k"]
    x = synth.draw(w, seed=1)
    cfg = hga.config_from(w)
    k_raw = x["k_raw"].cuda()
    cs1, gs1 = pipeline.alloc_summaries(cfg)
    kr1 = torch.empty_like(k_raw)
    hga.build_summaries(cfg, k_raw, cs1, gs1, kr1)
    cs2, gs2 = pipeline.alloc_summaries(cfg)
    kr2 = torch.empty_like(k_raw)
    for c0, c1 in [(0, 1), (1, 7), (7, 40), (40, cfg.n_chunks)]:
        hga.build_summaries(cfg, k_raw, cs2, gs2, kr2, c0, c1)
    torch.cuda.synchronize()
    assert torch.equal(cs1, cs2) and torch.equal(gs1, gs2) and torch.equal(kr1, kr2)
