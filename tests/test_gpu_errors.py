"""GPU error paths, through the C ABI.

* An invalid entry in a caller-supplied selection list is recorded in the
  device error word and skipped: its own unit computes over the rest of its
  keys, every other unit of the launch is bitwise what a clean launch gives,
  and a later launch with the word still set is bitwise clean too (the word
  is written by kernels, never read by them). Outputs start as NaN, so a row
  a kernel did not write shows up.
* A bounded device wait that runs out (here: a wait limit of 1 ns, which the
  pipeline waits of every kernel exceed) reports HGA_ERR_TIMEOUT; the kernel
  retires the copies it had issued before it exits, and the next launch with
  the default limit is bitwise clean.
* Invalid memory spaces are refused on the host before anything is launched.
"""
import numpy as np
import pytest
import torch

from long_context_rope_b200 import synth

pytestmark = pytest.mark.gpu

NAN = float("nan")


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
    out = torch.full_like(q_rot, NAN)
    pipeline.prefill(cfg, k_raw, v, q_rot, cs, gs, k_rot, rb, out)
    assert hga.get_device_error() == 0
    assert torch.isfinite(out.float()).all()
    return hga, pipeline, cfg, q_rot, k_rot, v, rb, out


def _setup_decode():
    """Decode (one query token) over a full resident cache: 2 sequences x 4K."""
    from long_context_rope_b200 import hga, pipeline
    w = synth.WORKLOADS["decode_16x32k"].replace(batch=2, seq_len=4096)
    x = synth.draw(w, seed=6)
    cfg = hga.config_from(w)
    k_raw, v = x["k_raw"].cuda(), x["v"].cuda()
    cs, gs = pipeline.alloc_summaries(cfg)
    k_rot = torch.empty_like(k_raw)
    pipeline.summaries(cfg, k_raw, cs, gs, k_rot)
    q_rot = pipeline.rotate_queries(cfg, x["q_raw"].cuda())
    rb = pipeline.alloc_route(cfg)
    pipeline.route(cfg, q_rot, cs, gs, rb)
    out = torch.full_like(q_rot, NAN)
    hga.attend(cfg, q_rot, k_rot, v, rb.sel_groups, rb.n_sel_groups, out)
    assert hga.get_device_error() == 0
    assert torch.isfinite(out.float()).all()
    return hga, pipeline, cfg, q_rot, cs, gs, k_rot, v, rb, out


def _unit_rows(cfg, b, h, jj):
    """(batch, token slice, head slice) of unit (b, h, query chunk jj) in an
    output [B, q_len, Hq, d]."""
    C, gq = cfg.chunk_size, cfg.n_q_heads // cfg.n_kv_heads
    j = cfg.q_begin // C + jj
    t0 = max(j * C, cfg.q_begin) - cfg.q_begin
    t1 = min((j + 1) * C, cfg.q_begin + cfg.q_len) - cfg.q_begin
    return b, slice(t0, t1), slice(h * gq, (h + 1) * gq)


def _drop_last_entry(sel, nsel, unit):
    """Selection lists with the last valid entry of `unit` removed."""
    s2, n2 = sel.clone(), nsel.clone()
    n = int(n2[unit])
    s2[unit + (n - 1,)] = -1
    n2[unit] = n - 1
    return s2, n2


def _check_only_unit_differs(cfg, got, clean, want_unit, unit):
    b0, h0, jj0 = unit
    for b in range(cfg.batch):
        for h in range(cfg.n_kv_heads):
            for jj in range(cfg.n_qchunks):
                r = _unit_rows(cfg, b, h, jj)
                ref = want_unit if (b, h, jj) == (b0, h0, jj0) else clean
                assert torch.equal(got[r], ref[r]), (b, h, jj)


@pytest.mark.parametrize("mode", ["prefill", "decode"])
def test_invalid_entry_touches_only_its_unit(mode):
    """One out-of-range entry (the last of its list, so the list stays
    ascending) in one unit: that unit equals the launch whose list omits the
    entry, every other unit equals the clean launch, bitwise. A second clean
    launch with the error word still set is bitwise clean."""
    if mode == "prefill":
        hga, pipeline, cfg, q_rot, k_rot, v, rb, clean = _setup()
        unit = (0, 1, 12)
    else:
        hga, pipeline, cfg, q_rot, cs, gs, k_rot, v, rb, clean = _setup_decode()
        unit = (1, 2, 0)
    n = int(rb.n_sel_groups[unit])
    assert n >= 2
    bad = rb.sel_groups.clone()
    bad[unit + (n - 1,)] = 10 ** 6
    got = torch.full_like(clean, NAN)
    hga.attend(cfg, q_rot, k_rot, v, bad, rb.n_sel_groups, got)
    # the word is left set (no read in between) for the next clean launch
    again = torch.full_like(clean, NAN)
    hga.attend(cfg, q_rot, k_rot, v, rb.sel_groups, rb.n_sel_groups, again)
    assert hga.get_device_error() == 2
    assert torch.equal(again, clean)
    s2, n2 = _drop_last_entry(rb.sel_groups, rb.n_sel_groups, unit)
    want = torch.full_like(clean, NAN)
    hga.attend(cfg, q_rot, k_rot, v, s2, n2, want)
    assert hga.get_device_error() == 0
    assert torch.isfinite(got.float()).all()
    _check_only_unit_differs(cfg, got, clean, want, unit)


def test_non_ascending_entry_flagged_and_skipped():
    hga, pipeline, cfg, q_rot, k_rot, v, rb, out = _setup()
    bad = rb.sel_groups.clone()
    unit = (0, 1, 12)
    bad[unit + (1,)] = bad[unit + (0,)]  # not strictly ascending
    out2 = torch.full_like(out, NAN)
    hga.attend(cfg, q_rot, k_rot, v, bad, rb.n_sel_groups, out2)
    assert hga.get_device_error() == 2
    assert torch.isfinite(out2.float()).all()
    for jj in range(cfg.n_qchunks):
        if jj != 12:
            r = _unit_rows(cfg, 0, 1, jj)
            assert torch.equal(out2[r], out[r])
    # the error word was cleared by the read
    hga.attend(cfg, q_rot, k_rot, v, rb.sel_groups, rb.n_sel_groups, out2)
    assert hga.get_device_error() == 0
    assert torch.equal(out2, out)


def test_invalid_counts_and_chunk_entries_flagged():
    hga, pipeline, cfg, q_rot, k_rot, v, rb, out = _setup()
    n_bad = rb.n_sel_groups.clone()
    n_bad[0, 2, 5] = cfg.top_k_groups + 7
    out2 = torch.full_like(out, NAN)
    hga.attend(cfg, q_rot, k_rot, v, rb.sel_groups, n_bad, out2)
    assert hga.get_device_error() == 3
    assert torch.isfinite(out2.float()).all()
    sc = rb.sel_chunks.clone()
    sc[0, 0, 9, 0] = 9  # the current chunk is forced, never routed
    sg = torch.empty_like(rb.sel_groups)
    ng = torch.empty_like(rb.n_sel_groups)
    hga.route_groups(cfg, rb.qbar, *pipeline.alloc_summaries(cfg)[1:], sc, rb.n_sel_chunks, sg, ng)
    assert hga.get_device_error() == 1


def _with_wait_limit(hga, ns, fn):
    hga.set_wait_limit_ns(ns)
    try:
        fn()
        return hga.get_device_error()
    finally:
        hga.set_wait_limit_ns(0)


def _run_or_time_out(hga, fn):
    """Run fn under a 1 ns wait limit; the status is HGA_ERR_TIMEOUT (code 4)
    if one of its waits ran out, else 0 (every wait completed within its
    first poll: the data it waited for had already landed)."""
    code = _with_wait_limit(hga, 1, fn)
    assert code in (0, 4), code
    return code


def test_wait_timeout_reported_and_next_launch_clean():
    """Every wait bounded by 1 ns. The prefill attention's pipeline waits (a
    unit waits for its first tiles, its softmax for each S) run out: the
    launch reports HGA_ERR_TIMEOUT (code 4), retires the copies and MMAs it
    had issued, and the same launch with the default limit afterwards is
    bitwise equal to the clean result. The decode attention, the one-launch
    decode step and the HBM gather take the same steps when a wait runs out;
    their rings run ahead of their consumers, so their waits usually find the
    data landed and complete: then the result must be complete and exact."""
    hga, pipeline, cfg, q_rot, k_rot, v, rb, clean = _setup()
    junk = torch.full_like(clean, NAN)
    assert _with_wait_limit(hga, 1, lambda: hga.attend(
        cfg, q_rot, k_rot, v, rb.sel_groups, rb.n_sel_groups, junk)) == 4
    again = torch.full_like(clean, NAN)
    hga.attend(cfg, q_rot, k_rot, v, rb.sel_groups, rb.n_sel_groups, again)
    assert hga.get_device_error() == 0
    assert torch.equal(again, clean)

    kg, vg = pipeline.alloc_gathered(cfg)
    hga.gather_kv(cfg, k_rot, v, False, rb.sel_groups, rb.n_sel_groups, kg, vg)
    assert hga.get_device_error() == 0
    kg2, vg2 = (torch.zeros_like(t) for t in (kg, vg))
    codes = {}
    codes["gather"] = _run_or_time_out(hga, lambda: hga.gather_kv(
        cfg, k_rot, v, False, rb.sel_groups, rb.n_sel_groups, kg2, vg2))
    if codes["gather"] == 0:
        assert torch.equal(kg2, kg) and torch.equal(vg2, vg)
    hga.gather_kv(cfg, k_rot, v, False, rb.sel_groups, rb.n_sel_groups, kg2, vg2)
    assert hga.get_device_error() == 0
    assert torch.equal(kg2, kg) and torch.equal(vg2, vg)

    hga, pipeline, cfg, q_rot, cs, gs, k_rot, v, rb, clean = _setup_decode()
    junk = torch.full_like(clean, NAN)
    codes["decode attention"] = _run_or_time_out(hga, lambda: hga.attend(
        cfg, q_rot, k_rot, v, rb.sel_groups, rb.n_sel_groups, junk))
    if codes["decode attention"] == 0:
        assert torch.equal(junk, clean)
    again = torch.full_like(clean, NAN)
    hga.attend(cfg, q_rot, k_rot, v, rb.sel_groups, rb.n_sel_groups, again)
    assert hga.get_device_error() == 0
    assert torch.equal(again, clean)

    rb2 = pipeline.alloc_route(cfg)
    step_out = torch.full_like(clean, NAN)
    pipeline.decode(cfg, q_rot, cs, gs, k_rot, v, rb2, step_out)
    assert hga.get_device_error() == 0
    junk = torch.full_like(clean, NAN)
    codes["decode step"] = _run_or_time_out(hga, lambda: pipeline.decode(
        cfg, q_rot, cs, gs, k_rot, v, pipeline.alloc_route(cfg), junk))
    if codes["decode step"] == 0:
        assert torch.equal(junk, step_out)
    again = torch.full_like(clean, NAN)
    pipeline.decode(cfg, q_rot, cs, gs, k_rot, v, rb2, again)
    assert hga.get_device_error() == 0
    assert torch.equal(again, step_out)
    print("status under a 1 ns wait limit:", codes)


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
        for jj in range(cfg.n_qchunks):
            for s in range(n[0, h, jj]):
                gi = sel[0, h, jj, s]
                assert torch.equal(kgh[0, h, jj, 16 * s:16 * s + 16], kr[0, h, 16 * gi:16 * gi + 16])
                assert torch.equal(vgh[0, h, jj, 16 * s:16 * s + 16], vv[0, h, 16 * gi:16 * gi + 16])
            # slots past the count are not written (the buffers start at zero)
            assert not kgh[0, h, jj, 16 * n[0, h, jj]:].any()


def test_zero_length_queries_are_noops():
    hga, pipeline, cfg, q_rot, k_rot, v, rb, out = _setup()
    c0 = cfg.copy(q_begin=cfg.seq_len, q_len=0)
    empty = torch.empty(1, 0, cfg.n_q_heads, cfg.head_dim, dtype=torch.bfloat16, device="cuda")
    ei = torch.empty(1, cfg.n_kv_heads, 0, dtype=torch.int32, device="cuda")
    hga._check(hga._lib.hga_attend(hga.ctypes.byref(c0), empty.data_ptr(), k_rot.data_ptr(),
                                   v.data_ptr(), None, None, ei.data_ptr(), ei.data_ptr(),
                                   empty.data_ptr(), None), "attend")
    assert hga.get_device_error() == 0
