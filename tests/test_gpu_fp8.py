"""GPU parity of the FP8 (E4M3) K/V variant, through the C ABI.

The key and value caches hold E4M3 codes with a per-tensor scale each
(hga_config.kv_type = HGA_KV_E4M3); the decode paths read them, the gathers
move them. Bars:
  * routing does not depend on the K/V storage: every path's selections are
    bitwise those of the bf16 cache's one-launch step on the same inputs,
    which are checked against the oracle's routing;
  * gathered buffers are bitwise the codes of the routed groups (a torch
    index copy), from HBM, from mapped host memory and through the warm tier;
  * every unit's output is within the bf16 tolerance of the oracle's
    attention over the decoded cache (code value x scale, the oracle's own
    E4M3 decoder) on the GPU's selection, for the one-launch step, the
    separate calls (index and gathered), the host-tier gathers and the
    one-launch tiered step.
"""
import numpy as np
import pytest
import torch

from long_context_rope_b200 import synth
from oracle import hga_oracle as O
from parity_util import assert_close, compare_routing

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS["decode_16x32k"].replace(name="fp8kv", batch=4, seq_len=16384)
TOL = 2e-2  # bf16 outputs, as for the bf16 cache


def _np(t):
    if t.dtype == torch.int32:
        return t.cpu().numpy()
    return t.detach().float().cpu().numpy()


@pytest.fixture(scope="module")
def case():
    from long_context_rope_b200 import hga, pipeline
    x = synth.draw(W, seed=11)
    r = O.pipeline(W, x)
    k_rot_bf = torch.from_numpy(np.ascontiguousarray(r["k_rot"])).to(torch.bfloat16)
    k8, ks = synth.to_e4m3(k_rot_bf)
    v8, vs = synth.to_e4m3(x["v"])
    cfg = hga.config_from(W)
    cfg8 = hga.config_from(W, kv_type=hga.HGA_KV_E4M3, k_scale=ks, v_scale=vs)
    k_raw = x["k_raw"].cuda()
    cs, gs = pipeline.alloc_summaries(cfg)
    pipeline.summaries(cfg, k_raw, cs, gs, None)
    del k_raw
    q_rot = torch.from_numpy(np.ascontiguousarray(r["q_rot"])).to(torch.bfloat16).cuda()
    # reference routing: the bf16 cache's one-launch step
    rb0 = pipeline.alloc_route(cfg)
    out0 = torch.empty_like(q_rot)
    pipeline.decode(cfg, q_rot, cs, gs, k_rot_bf.cuda(), x["v"].cuda(), rb0, out0)
    rbs = pipeline.alloc_route(cfg, with_scores=True)
    pipeline.route(cfg, q_rot, cs, gs, rbs, separate=True)
    torch.cuda.synchronize()
    assert hga.get_device_error() == 0
    for name in ("qbar", "sel_chunks", "n_sel_chunks", "sel_groups", "n_sel_groups"):
        assert torch.equal(getattr(rb0, name), getattr(rbs, name)), name
    g = dict(qbar=_np(rbs.qbar), chunk_sum=_np(cs), group_sum=_np(gs),
             sel_chunks=_np(rbs.sel_chunks), n_sel_chunks=_np(rbs.n_sel_chunks),
             chunk_scores=_np(rbs.chunk_scores), sel_groups=_np(rbs.sel_groups),
             n_sel_groups=_np(rbs.n_sel_groups), group_scores=_np(rbs.group_scores))
    assert_close("qbar", g["qbar"], r["qbar"], atol=2e-5, rtol=2e-5)
    same = compare_routing(W, g, r, O)
    assert same.mean() >= 0.99, same.mean()
    # the oracle's attention over the decoded FP8 cache, on the GPU's selection
    k_dec = O.e4m3_decode(k8.view(torch.uint8).numpy(), ks)
    v_dec = O.e4m3_decode(v8.view(torch.uint8).numpy(), vs)
    want = O.attend(O.cfg_of(W), r["q_rot"], k_dec, v_dec, g["sel_groups"], g["n_sel_groups"])
    return dict(x=x, r=r, cfg=cfg, cfg8=cfg8, cs=cs, gs=gs, q_rot=q_rot, k8=k8, v8=v8,
                rb0=rb0, want=want)


def _check_out(name, out, want):
    got = _np(out)
    assert np.isfinite(got).all(), name
    err = float(np.abs(got - want).max())
    assert err <= TOL, f"{name}: max abs error {err:.3e}"
    return err


def _same_routing(rb, rb0):
    for name in ("qbar", "sel_chunks", "n_sel_chunks", "sel_groups", "n_sel_groups"):
        assert torch.equal(getattr(rb, name), getattr(rb0, name)), name


def _gathered_codes(c, k8):
    """The routed groups' codes by a torch index copy: [B, Hkv, 1, kg*g, d]."""
    cfg, rb0 = c["cfg"], c["rb0"]
    B, H, kg, g, d = cfg.batch, cfg.n_kv_heads, cfg.top_k_groups, cfg.group_size, cfg.head_dim
    sel = rb0.sel_groups.cpu().reshape(B, H, kg)
    n = rb0.n_sel_groups.cpu().reshape(B, H)
    raw = k8.view(torch.uint8)
    out = torch.zeros(B, H, 1, kg * g, d, dtype=torch.uint8)
    for b in range(B):
        for h in range(H):
            for s in range(int(n[b, h])):
                gi = int(sel[b, h, s])
                out[b, h, 0, s * g:(s + 1) * g] = raw[b, h, gi * g:(gi + 1) * g]
    return out


def test_fp8_decode_step_and_separate_calls(case):
    from long_context_rope_b200 import hga, pipeline
    c = case
    cfg8, q_rot = c["cfg8"], c["q_rot"]
    k8, v8 = c["k8"].cuda(), c["v8"].cuda()
    rb = pipeline.alloc_route(cfg8)
    out = torch.full_like(q_rot, float("nan"))
    pipeline.decode(cfg8, q_rot, c["cs"], c["gs"], k8, v8, rb, out)
    torch.cuda.synchronize()
    assert hga.get_device_error() == 0
    _same_routing(rb, c["rb0"])
    e1 = _check_out("one-launch step", out, c["want"])
    # separate calls: routing, then decode attention in index mode
    rb2 = pipeline.alloc_route(cfg8)
    out2 = torch.full_like(q_rot, float("nan"))
    pipeline.decode(cfg8, q_rot, c["cs"], c["gs"], k8, v8, rb2, out2, separate=True)
    torch.cuda.synchronize()
    assert hga.get_device_error() == 0
    _same_routing(rb2, c["rb0"])
    e2 = _check_out("separate calls", out2, c["want"])
    # HBM gather (bitwise the codes), then attention over the compact buffers
    gat = pipeline.alloc_gathered(cfg8)
    assert gat[0].dtype == torch.float8_e4m3fn
    rb3 = pipeline.alloc_route(cfg8)
    out3 = torch.full_like(q_rot, float("nan"))
    pipeline.decode(cfg8, q_rot, c["cs"], c["gs"], k8, v8, rb3, out3, gathered=gat, k_src=k8,
                    v_src=v8)
    torch.cuda.synchronize()
    assert hga.get_device_error() == 0
    assert torch.equal(gat[0].view(torch.uint8).cpu(), _gathered_codes(c, c["k8"]))
    assert torch.equal(gat[1].view(torch.uint8).cpu(), _gathered_codes(c, c["v8"]))
    e3 = _check_out("gathered", out3, c["want"])
    print(f"fp8 K/V: one launch {e1:.3e}, separate {e2:.3e}, gathered {e3:.3e}")


def test_fp8_host_tier(case):
    """The cold tier in pinned host memory as E4M3 codes: the host-link gather,
    the warm tier (bitwise the cold gather) and the one-launch tiered step."""
    from long_context_rope_b200 import hga, pipeline
    c = case
    cfg8, q_rot = c["cfg8"], c["q_rot"]
    k_host = c["k8"].pin_memory()
    v_host = c["v8"].pin_memory()
    cfg_w = cfg8.copy(kv_layout=hga.HGA_KV_WINDOWS)
    Wn = hga.window_slots(cfg8)
    shape = (W.batch, W.n_kv_heads, Wn * W.chunk_size, W.head_dim)
    k_win = torch.zeros(shape, dtype=torch.float8_e4m3fn, device="cuda")
    v_win = torch.zeros(shape, dtype=torch.float8_e4m3fn, device="cuda")
    pipeline.fill_windows(cfg8, k_host, v_host, k_win, v_win)
    # three launches: route, host gather, attend
    rb = pipeline.alloc_route(cfg8)
    gat = pipeline.alloc_gathered(cfg8)
    out = torch.full_like(q_rot, float("nan"))
    pipeline.decode(cfg_w, q_rot, c["cs"], c["gs"], k_win, v_win, rb, out, gathered=gat,
                    k_src=k_host, v_src=v_host, src_is_host=True)
    torch.cuda.synchronize()
    assert hga.get_device_error() == 0
    _same_routing(rb, c["rb0"])
    assert torch.equal(gat[0].view(torch.uint8).cpu(), _gathered_codes(c, c["k8"]))
    e1 = _check_out("host gather", out, c["want"])
    # warm tier, twice (misses, then hits): bitwise the cold gather
    pool = pipeline.alloc_warm_pool(cfg8, n_slots=2 * W.top_k_groups)
    for it in range(2):
        gw = pipeline.alloc_gathered(cfg8)
        outw = torch.full_like(q_rot, float("nan"))
        pipeline.decode(cfg_w, q_rot, c["cs"], c["gs"], k_win, v_win, rb, outw, gathered=gw,
                        k_src=k_host, v_src=v_host, src_is_host=True, warm=pool)
        torch.cuda.synchronize()
        assert hga.get_device_error() == 0
        assert torch.equal(gw[0].view(torch.uint8), gat[0].view(torch.uint8)), it
        assert torch.equal(gw[1].view(torch.uint8), gat[1].view(torch.uint8)), it
        assert torch.equal(outw, out), it
    hits = pool.stats[..., 0].sum().item()
    assert hits == int(rb.n_sel_groups.sum().item())  # the second call hit every group
    # one launch: routed groups read from the host store inside the kernel
    rb_f = pipeline.alloc_route(cfg8)
    out_f = torch.full_like(q_rot, float("nan"))
    pipeline.decode_tiered(cfg_w, q_rot, c["cs"], c["gs"], k_win, v_win, k_host, v_host, rb_f,
                           out_f)
    torch.cuda.synchronize()
    assert hga.get_device_error() == 0
    _same_routing(rb_f, c["rb0"])
    e2 = _check_out("tiered one launch", out_f, c["want"])
    print(f"fp8 K/V host tier: gather {e1:.3e}, one launch {e2:.3e}")
