"""GPU error paths: invalid caller-supplied selections are reported through
the device error word and skipped (no fault, no trap); invalid memory spaces
are refused on the host before anything is launched."""
import numpy as np
import pytest
import torch

from long_context_rope_b200 import synth

pytestmark = pytest.mark.gpu


def _setup():
    from long_context_rope_b200 import hga, pipeline
    w = synth.WORKLOADS["prefill_4k"].replace(seq_len=1024)
    x = synth.draw(w, seed=5)
    cfg = hga.config_from(w)
    k_raw, v, q_raw = (x[n].cuda() for n in ("k_raw", "v", "q_raw"))
    q_rot = pipeline.rotate_queries(cfg, q_raw)
    cs, gs = pipeline.alloc_summaries(cfg)
    k_rot = torch.empty_like(k_raw)
    rb = pipeline.alloc_route(cfg)
    out = torch.empty_like(q_rot)
    pipeline.prefill(cfg, k_raw, v, q_rot, cs, gs, k_rot, rb, out)
    assert hga.get_device_error() == 0
    return hga, pipeline, cfg, q_rot, k_rot, v, rb, out


def test_invalid_group_entries_flagged_and_skipped():
    hga, pipeline, cfg, q_rot, k_rot, v, rb, out = _setup()
    bad = rb.sel_groups.clone()
    bad[0, 0, 10, 0] = 10 ** 6          # out of range
    bad[0, 1, 12, 1] = bad[0, 1, 12, 0]  # not strictly ascending
    out2 = torch.empty_like(out)
    hga.attend(cfg, q_rot, k_rot, v, bad, rb.n_sel_groups, out2)
    assert hga.get_device_error() == 2
    assert torch.isfinite(out2.float()).all()
    # untouched problems give the same result as before
    assert torch.equal(out2[0, 20 * 64: 21 * 64], out[0, 20 * 64: 21 * 64])
    # the error word was cleared by the read
    hga.attend(cfg, q_rot, k_rot, v, rb.sel_groups, rb.n_sel_groups, out2)
    assert hga.get_device_error() == 0
    assert torch.equal(out2, out)


def test_invalid_counts_and_chunk_entries_flagged():
    hga, pipeline, cfg, q_rot, k_rot, v, rb, out = _setup()
    n_bad = rb.n_sel_groups.clone()
    n_bad[0, 2, 5] = cfg.top_k_groups + 7
    hga.attend(cfg, q_rot, k_rot, v, rb.sel_groups, n_bad, out)
    assert hga.get_device_error() == 3
    sc = rb.sel_chunks.clone()
    sc[0, 0, 9, 0] = 9  # the current chunk is forced, never routed
    sg = torch.empty_like(rb.sel_groups)
    ng = torch.empty_like(rb.n_sel_groups)
    hga.route_groups(cfg, rb.qbar, *pipeline.alloc_summaries(cfg)[1:], sc, rb.n_sel_chunks, sg, ng)
    assert hga.get_device_error() == 1


def test_gather_memory_space_checks():
    hga, pipeline, cfg, q_rot, k_rot, v, rb, out = _setup()
    gat = pipeline.alloc_gathered(cfg)
    pageable = torch.empty(k_rot.shape, dtype=k_rot.dtype)  # not page-locked
    with pytest.raises(hga.HgaError) as e:
        hga.gather_kv(cfg, pageable, pageable, True, rb.sel_groups, rb.n_sel_groups, *gat)
    assert e.value.status == -9
    with pytest.raises(hga.HgaError) as e:  # device memory passed as host
        hga._check(hga._lib.hga_gather_kv(
            hga.ctypes.byref(cfg), k_rot.data_ptr(), v.data_ptr(), 1, rb.sel_groups.data_ptr(),
            rb.n_sel_groups.data_ptr(), gat[0].data_ptr(), gat[1].data_ptr(), None), "gather")
    assert e.value.status == -9
    assert hga.get_device_error() == 0


def test_gather_hbm_matches_indexing():
    hga, pipeline, cfg, q_rot, k_rot, v, rb, out = _setup()
    kg, vg = pipeline.alloc_gathered(cfg)
    hga.gather_kv(cfg, k_rot, v, False, rb.sel_groups, rb.n_sel_groups, kg, vg)
    assert hga.get_device_error() == 0
    sel = rb.sel_groups.cpu().numpy()
    n = rb.n_sel_groups.cpu().numpy()
    kr, vv, kgh, vgh = (t.cpu() for t in (k_rot, v, kg, vg))
    for h in range(cfg.n_kv_heads):
        for jj in (3, 9, cfg.n_qchunks - 1):
            for s in range(n[0, h, jj]):
                gi = sel[0, h, jj, s]
                assert torch.equal(kgh[0, h, jj, 16 * s:16 * s + 16], kr[0, h, 16 * gi:16 * gi + 16])
                assert torch.equal(vgh[0, h, jj, 16 * s:16 * s + 16], vv[0, h, 16 * gi:16 * gi + 16])


def test_zero_length_queries_are_noops():
    hga, pipeline, cfg, q_rot, k_rot, v, rb, out = _setup()
    c0 = cfg.copy(q_begin=cfg.seq_len, q_len=0)
    empty = torch.empty(1, 0, cfg.n_q_heads, cfg.head_dim, dtype=torch.bfloat16, device="cuda")
    e32 = torch.empty(1, cfg.n_kv_heads, 0, cfg.head_dim, device="cuda")
    ei = torch.empty(1, cfg.n_kv_heads, 0, dtype=torch.int32, device="cuda")
    hga._check(hga._lib.hga_attend(hga.ctypes.byref(c0), empty.data_ptr(), k_rot.data_ptr(),
                                   v.data_ptr(), None, None, ei.data_ptr(), ei.data_ptr(),
                                   empty.data_ptr(), None), "attend")
    assert hga.get_device_error() == 0
