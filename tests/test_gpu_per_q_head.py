"""GPU parity of per-query-head routing (hga_config.routing =
HGA_ROUTE_PER_Q_HEAD), through the C ABI.

Each query head routes on its own rotated query against its KV head's
summaries and attends over its own selection. The oracle states this as the
plain routing of an expanded problem (oracle.hga_oracle.per_q_head: every
query head gets its own copy of its KV head's keys and values). Bars: q-bar
within 2e-5; selections identical to the oracle's up to the near-tie band
(groups on the GPU's own chunk selection); every unit's output within the
bf16 tolerance of the oracle (on the GPU's selection where it differs);
hga_route and hga_attend (index mode) agree with the one-launch step
(selections bitwise, outputs within 1e-2); the calls this variant does not
cover refuse it.
"""
import numpy as np
import pytest
import torch

from long_context_rope_b200 import synth
from oracle import hga_oracle as O
from parity_util import assert_close, compare_outputs, compare_routing

pytestmark = pytest.mark.gpu

BASE = synth.WORKLOADS["decode_16x32k"]


def _np(t):
    if t.dtype == torch.int32:
        return t.cpu().numpy()
    return t.detach().float().cpu().numpy()


@pytest.mark.parametrize("shape", [dict(batch=2, seq_len=8192), dict(batch=3, seq_len=64 * 70 + 32)])
def test_per_q_head_decode_vs_oracle(shape):
    from long_context_rope_b200 import hga, pipeline
    w = BASE.replace(name="perhead", **shape)
    gq = w.n_q_heads // w.n_kv_heads
    x = synth.draw(w, seed=12)
    wh, xh = O.per_q_head(w, x)
    r = O.pipeline(wh, xh)
    cfg = hga.config_from(w, routing=hga.HGA_ROUTE_PER_Q_HEAD)
    assert cfg.route_heads == w.n_q_heads
    k_raw = x["k_raw"].cuda()
    cs, gs = pipeline.alloc_summaries(cfg)
    pipeline.summaries(cfg, k_raw, cs, gs, None)
    del k_raw
    # the oracle's bf16 rotations; its expanded cache holds gq equal copies per KV head
    k_rot = torch.from_numpy(np.ascontiguousarray(r["k_rot"][:, ::gq])).to(torch.bfloat16).cuda()
    q_rot = torch.from_numpy(np.ascontiguousarray(r["q_rot"])).to(torch.bfloat16).cuda()
    v = x["v"].cuda()
    rb = pipeline.alloc_route(cfg)
    assert rb.sel_groups.shape[1] == w.n_q_heads
    out = torch.full_like(q_rot, float("nan"))
    pipeline.decode(cfg, q_rot, cs, gs, k_rot, v, rb, out)
    rb2 = pipeline.alloc_route(cfg)
    pipeline.route(cfg, q_rot, cs, gs, rb2)
    out2 = torch.full_like(q_rot, float("nan"))
    hga.attend(cfg, q_rot, k_rot, v, rb.sel_groups, rb.n_sel_groups, out2)
    torch.cuda.synchronize()
    assert hga.get_device_error() == 0
    for name in ("qbar", "sel_chunks", "n_sel_chunks", "sel_groups", "n_sel_groups"):
        assert torch.equal(getattr(rb, name), getattr(rb2, name)), name
    diff = (out.float() - out2.float()).abs().max().item()
    assert diff <= 1e-2, diff

    g = dict(qbar=_np(rb.qbar), chunk_sum=np.repeat(_np(cs), gq, axis=1),
             group_sum=np.repeat(_np(gs), gq, axis=1), sel_chunks=_np(rb.sel_chunks),
             n_sel_chunks=_np(rb.n_sel_chunks), chunk_scores=None,
             sel_groups=_np(rb.sel_groups), n_sel_groups=_np(rb.n_sel_groups),
             group_scores=None)
    assert_close("qbar", g["qbar"], r["qbar"], atol=2e-5, rtol=2e-5)
    same = compare_routing(wh, g, r, O)
    assert same.mean() >= 0.99, same.mean()
    vv = xh["v"]

    def oracle_alt(units):
        return O.attend(O.cfg_of(wh), r["q_rot"], r["k_rot"], vv, g["sel_groups"],
                        g["n_sel_groups"], units=np.array(units, dtype=np.int32))

    worst, n_alt = compare_outputs(wh, _np(out), r["out"], same, oracle_alt)
    # the query heads of a KV head do route differently
    sel = g["sel_groups"].reshape(w.batch, w.n_kv_heads, gq, -1)
    assert any(not np.array_equal(sel[b, k, 0], sel[b, k, i]) for b in range(w.batch)
               for k in range(w.n_kv_heads) for i in range(1, gq))
    # calls the variant does not cover refuse it
    rb3 = pipeline.alloc_route(cfg, with_scores=True)
    with pytest.raises(hga.HgaError) as e:
        pipeline.route(cfg, q_rot, cs, gs, rb3, separate=True)
    assert e.value.status == -8
    print(f"per-query-head routing {shape}: {same.mean():.3f} identical ({n_alt} units on the "
          f"GPU's selection), max abs error {worst:.3e}, attend vs step {diff:.3e}")
