"""hga_gather_kv_warm_noalloc: the warm-tier gather for callers that may not
allocate device memory (a serving engine that has reserved its HBM up front
and hands out only fixed buffers, or a decode loop that cannot afford the
device-wide synchronisation of cudaFree). Its plan-to-copy scratch is a fixed
65536-entry array inside the library instead of a caller buffer.

The GPU test runs two calls in a row on one pool through the new entry point
and on a second, identical pool through hga_gather_kv_warm, and requires the
same gathered K/V (bitwise, as for every gather test: the call copies), pool
contents, tags, last-use steps and hit / miss counts after each call. All
calls go on one explicit stream, so the second call is ordered after the
first and finds the first call's contents in the scratch array.

This file is named so that pytest collects it last."""
import ctypes

import pytest
import torch

from long_context_rope_b200 import synth


@pytest.fixture(scope="module")
def hga():
    from long_context_rope_b200 import build
    build.build()
    from long_context_rope_b200 import hga as mod
    return mod


def test_noalloc_rejects_more_than_its_scratch_holds(hga):
    # 4 KV heads x 96 selected groups = 384 entries per sequence: 170
    # sequences fit in 65536 entries, 171 do not. Refused on the host before
    # any CUDA call (the fake pointers are never dereferenced).
    w = synth.WORKLOADS["tiered_decode_4x64k"]
    cfg = hga.config_from(w, batch=171)
    assert cfg.batch * cfg.n_kv_heads * cfg.top_k_groups > 65536
    P = ctypes.c_void_p(4096)
    st = hga.library().hga_gather_kv_warm_noalloc(ctypes.byref(cfg), P, P, P, P, P, P, P, P,
                                                   128, 0, None, P, P, None)
    assert st == -10
    assert hga.STATUS[st] == "HGA_ERR_SCRATCH_LIMIT"
    assert hga.library().hga_status_string(st).decode().startswith("HGA_ERR_SCRATCH_LIMIT")


def test_noalloc_validates_like_the_warm_gather(hga):
    # decode only, pool at least top_k_groups slots, 16-byte pointers; all
    # checked on the host before any CUDA call (fake pointers, never read)
    L = hga.library()
    P = ctypes.c_void_p(16 * 1024)
    by = ctypes.byref
    dec = hga.config_from(synth.WORKLOADS["prefill_4k"], q_begin=4095, q_len=1)
    pre = hga.config_from(synth.WORKLOADS["prefill_4k"])
    assert L.hga_gather_kv_warm_noalloc(by(dec), P, P, P, P, P, P, P, None, 128, 0, None, P, P,
                                        None) == -1
    assert L.hga_gather_kv_warm_noalloc(by(pre), P, P, P, P, P, P, P, P, 128, 0, None, P, P,
                                        None) == -8
    assert L.hga_gather_kv_warm_noalloc(by(dec), P, P, P, P, P, P, P, P, 64, 0, None, P, P,
                                        None) == -2
    assert L.hga_gather_kv_warm_noalloc(by(dec), P, P, P, P, P, P, P, P, 128, -1, None, P, P,
                                        None) == -2
    assert L.hga_gather_kv_warm_noalloc(by(dec), P, P, P, P, P, P, P, P, 128, 0,
                                        ctypes.c_void_p(16 * 1024 + 4), P, P, None) == -3


@pytest.mark.gpu
def test_noalloc_matches_warm_gather_on_two_calls_in_a_row(hga):
    from long_context_rope_b200 import pipeline
    w = synth.WORKLOADS["tiered_decode_4x64k"].replace(name="noalloc", batch=2, seq_len=16384)
    x = synth.draw(w, seed=21)
    q_other = synth.draw(w, seed=22, with_kv=False)["q_raw"]
    # call 2: sequence 0 repeats its query (all hits), sequence 1 takes a new
    # one (mostly misses, with evictions from a pool smaller than two routes)
    q_second = x["q_raw"].clone()
    q_second[1] = q_other[1]
    cfg = hga.config_from(w)
    k_raw = x["k_raw"].cuda()
    cs, gs = pipeline.alloc_summaries(cfg)
    k_rot = torch.empty_like(k_raw)
    pipeline.summaries(cfg, k_raw, cs, gs, k_rot)
    del k_raw
    k_host = torch.empty(k_rot.shape, dtype=k_rot.dtype, pin_memory=True)
    k_host.copy_(k_rot)
    v_host = x["v"].pin_memory()
    S = 128
    ref, new = pipeline.alloc_warm_pool(cfg, S), pipeline.alloc_warm_pool(cfg, S)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):  # every call below: this one stream
        _two_calls(hga, pipeline, w, cfg, x, q_second, cs, gs, k_host, v_host, ref, new)


def _two_calls(hga, pipeline, w, cfg, x, q_second, cs, gs, k_host, v_host, ref, new):
    for step, q_raw in enumerate((x["q_raw"], q_second)):
        q_rot = pipeline.rotate_queries(cfg, q_raw.cuda())
        rb = pipeline.alloc_route(cfg)
        pipeline.route(cfg, q_rot, cs, gs, rb)
        g_ref, g_new = pipeline.alloc_gathered(cfg), pipeline.alloc_gathered(cfg)
        hga.gather_kv_warm(cfg, k_host, v_host, rb.sel_groups, rb.n_sel_groups, ref.k, ref.v,
                           ref.tag, ref.last, step, ref.src, g_ref[0], g_ref[1],
                           stats=ref.stats)
        hga.gather_kv_warm_noalloc(cfg, k_host, v_host, rb.sel_groups, rb.n_sel_groups, new.k,
                                   new.v, new.tag, new.last, step, g_new[0], g_new[1],
                                   stats=new.stats)
        assert hga.get_device_error() == 0  # synchronises the current (explicit) stream
        n = rb.n_sel_groups.cpu().reshape(-1)
        assert int(n.min()) > 0
        for u in range(w.batch * w.n_kv_heads):
            b, h = divmod(u, w.n_kv_heads)
            rows = int(n[u]) * 16
            for a, c in ((g_new[0], g_ref[0]), (g_new[1], g_ref[1])):
                assert torch.equal(a[b, h, 0, :rows], c[b, h, 0, :rows]), (step, u)
        assert torch.equal(new.tag, ref.tag), step
        assert torch.equal(new.last, ref.last), step
        assert torch.equal(new.stats, ref.stats), step
        assert torch.equal(new.k, ref.k) and torch.equal(new.v, ref.v), step
        stats = new.stats.cpu()
        if step == 0:
            assert int(stats[..., 0].sum()) == 0  # empty pools: every group a miss
        else:
            assert torch.equal(stats[0, :, 1], torch.zeros_like(stats[0, :, 1]))  # repeat
            assert int(stats[1, :, 1].sum()) > 0  # new route: misses
