"""The C-ABI library loads, exports every symbol include/hga.h declares, and
rejects invalid arguments on the host (no GPU needed, no compute launched)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "hga.h")).read()
    return sorted(set(re.findall(r"^\s*(?:hga_status|const char\*|int32_t|void)\s+(hga_\w+)\s*\(",
                                 text, flags=re.M)))


@pytest.fixture(scope="module")
def hga():
    from long_context_rope_b200 import build
    build.build()
    from long_context_rope_b200 import hga as mod
    return mod


def test_exports_every_declared_symbol(hga):
    names = _declared()
    assert len(names) >= 9, names
    for n in names:
        assert hasattr(hga.library(), n), n


def test_struct_layout_matches_header(hga):
    # 12 int32 (48 bytes), a double at offset 48, 6 int32 (80), two floats, one
    # int32 (92), 8-byte aligned: 96
    assert ctypes.sizeof(hga.HgaConfig) == 96
    assert hga.HgaConfig.routing.offset == 88
    assert hga.HgaConfig.rope_theta.offset == 48
    assert hga.HgaConfig.summary_type.offset == 72
    assert hga.HgaConfig.kv_type.offset == 76
    assert hga.HgaConfig.k_scale.offset == 80
    assert hga.HgaConfig.v_scale.offset == 84


def _cfg(hga, **kw):
    from long_context_rope_b200 import synth
    return hga.config_from(synth.WORKLOADS["prefill_4k"], **kw)


def test_summary_type_validation_without_gpu(hga):
    L = hga.library()
    P = 16 * 1024  # never dereferenced: refused on the host
    by = ctypes.byref
    bad = _cfg(hga, summary_type=7)
    assert L.hga_route_chunks(by(bad), P, P, P, P, P, None, None) == -4
    bf = _cfg(hga, summary_type=hga.HGA_SUMMARY_BF16)
    # the separate routing calls do not read bf16 tables
    assert L.hga_route_chunks(by(bf), P, P, P, P, P, None, None) == -8
    assert L.hga_route_groups(by(bf), P, P, P, P, P, P, None, None) == -8


def test_fp8_kv_validation_without_gpu(hga):
    """E4M3 K/V: scales must be finite and positive, the queries bf16 and
    d = 128; prefill attention and a rotated-key output are refused."""
    L = hga.library()
    P = 16 * 1024  # never dereferenced: refused on the host
    by = ctypes.byref
    attend = [P] * 3 + [None, None] + [P] * 3 + [None]
    assert L.hga_attend(by(_cfg(hga, kv_type=5)), *attend) == -4
    for ks, vs in ((0.0, 1.0), (1.0, -1.0), (float("nan"), 1.0), (1.0, float("inf"))):
        bad = _cfg(hga, kv_type=hga.HGA_KV_E4M3, k_scale=ks, v_scale=vs)
        assert L.hga_attend(by(bad), *attend) == -4, (ks, vs)
    ok = dict(kv_type=hga.HGA_KV_E4M3, k_scale=0.01, v_scale=0.02)
    assert L.hga_attend(by(_cfg(hga, dtype=hga.HGA_F32, **ok)), *attend) == -8
    assert L.hga_attend(by(_cfg(hga, **ok)), *attend) == -8  # prefill span (q_len > 1)
    assert L.hga_build_summaries(by(_cfg(hga, **ok)), P, P, P, P, 0, 4, None) == -8
    # decode span: the host checks pass, so a NULL output is what is reported
    dec = _cfg(hga, q_begin=4095, q_len=1, **ok)
    assert L.hga_attend(by(dec), *attend[:-2], None, None) == -1


def test_per_q_head_routing_validation_without_gpu(hga):
    """Per-query-head routing: the separate routing calls, the gathers and
    prefill attention refuse it; an unknown routing value is a config error."""
    L = hga.library()
    P = 16 * 1024  # never dereferenced: refused on the host
    by = ctypes.byref
    assert L.hga_route_chunks(by(_cfg(hga, routing=3)), P, P, P, P, P, None, None) == -4
    ph = _cfg(hga, q_begin=4095, q_len=1, routing=hga.HGA_ROUTE_PER_Q_HEAD)
    assert L.hga_route_chunks(by(ph), P, P, P, P, P, None, None) == -8
    assert L.hga_route_groups(by(ph), P, P, P, P, P, P, None, None) == -8
    assert L.hga_gather_kv(by(ph), P, P, 0, P, P, P, P, None) == -8
    attend = [P] * 3 + [None, None] + [P] * 3 + [None]
    assert L.hga_attend(by(_cfg(hga, routing=hga.HGA_ROUTE_PER_Q_HEAD)), *attend) == -8
    assert L.hga_attend(by(ph), P, P, P, P, P, P, P, P, None) == -8  # gathered mode


def test_tiered_step_validation_without_gpu(hga):
    L = hga.library()
    P = 16 * 1024  # never dereferenced: refused on the host
    by = ctypes.byref
    dec = _cfg(hga, q_begin=4095, q_len=1, kv_layout=hga.HGA_KV_WINDOWS)
    args = [P] * 13 + [None]
    nul = list(args)
    nul[5] = None  # k_host
    assert L.hga_decode_step_tiered(by(dec), *nul) == -1
    full = _cfg(hga, q_begin=4095, q_len=1)  # resident windows are required
    assert L.hga_decode_step_tiered(by(full), *args) == -8
    mid = _cfg(hga, q_begin=2000, q_len=1, kv_layout=hga.HGA_KV_WINDOWS)  # not the last token
    assert L.hga_decode_step_tiered(by(mid), *args) == -8


def test_status_strings(hga):
    for code, name in hga.STATUS.items():
        assert hga.library().hga_status_string(code).decode().startswith(name)


def test_host_validation_without_gpu(hga):
    L = hga.library()
    P = 16 * 1024  # any aligned non-null value: nothing is dereferenced on these paths
    by = ctypes.byref
    assert L.hga_attend(None, P, P, P, None, None, P, P, P, None) == -1
    assert L.hga_attend(by(_cfg(hga)), P, P, P, None, None, None, P, P, None) == -1
    assert L.hga_attend(by(_cfg(hga)), P + 4, P, P, None, None, P, P, P, None) == -3
    assert L.hga_attend(by(_cfg(hga)), P, P, P, P, None, P, P, P, None) == -1
    assert L.hga_attend(by(_cfg(hga, head_dim=96)), P, P, P, None, None, P, P, P, None) == -8
    assert L.hga_attend(by(_cfg(hga, top_k_chunks=0)), P, P, P, None, None, P, P, P, None) == -4
    assert L.hga_attend(by(_cfg(hga, n_q_heads=30)), P, P, P, None, None, P, P, P, None) == -2
    assert L.hga_attend(by(_cfg(hga, q_begin=4000, q_len=100)), P, P, P, None, None, P, P, P,
                        None) == -2
    assert L.hga_attend(by(_cfg(hga, rope_theta=0.5)), P, P, P, None, None, P, P, P, None) == -4
    assert L.hga_attend(by(_cfg(hga, chunk_size=48)), P, P, P, None, None, P, P, P, None) == -8
    assert L.hga_attend(by(_cfg(hga, n_high_freq_pairs=65)), P, P, P, None, None, P, P, P,
                        None) == -4
    assert L.hga_attend(by(_cfg(hga, kv_layout=1)), P, P, P, None, None, P, P, P, None) == -8
    assert L.hga_build_summaries(by(_cfg(hga)), P, P, P, None, 5, 3, None) == -2
    assert L.hga_build_summaries(by(_cfg(hga)), P, P, P, None, 0, 65, None) == -2
    assert L.hga_build_summaries(by(_cfg(hga)), P, P, P, None, 3, 3, None) == 0  # empty range
    assert L.hga_route_chunks(by(_cfg(hga)), P, P, None, P, P, None, None) == -1
    assert L.hga_route_groups(by(_cfg(hga)), P, P, P, P, P + 8, P, None, None) == -3
    assert L.hga_gather_kv(by(_cfg(hga)), P, P, 0, P, P, None, P, None) == -1
    assert L.hga_apply_rope(by(_cfg(hga)), P, P, 1, 4, 0, 0, None) == -2
    assert L.hga_apply_rope(by(_cfg(hga)), P, P, 0, 4, 1, 0, None) == 0  # nothing to do
    # hga_route / hga_decode_step: required outputs, alignment, layout
    assert L.hga_route(by(_cfg(hga)), P, P, P, None, P, P, P, P, None) == -1
    assert L.hga_route(by(_cfg(hga)), P, P, P, P, P, P, P + 4, P, None) == -3
    assert L.hga_decode_step(by(_cfg(hga)), P, P, P, P, P, P, P, P, P, P, None, None) == -1
    assert L.hga_decode_step(by(_cfg(hga)), P, P, P, P, P + 2, P, P, P, P, P, P, None) == -3
    assert L.hga_decode_step(by(_cfg(hga, kv_layout=1)), P, P, P, P, P, P, P, P, P, P, P,
                             None) == -8
    assert L.hga_decode_step(by(_cfg(hga, q_len=0)), P, P, P, P, P, P, P, P, P, P, P,
                             None) == 0  # empty span
    # hga_gather_kv_warm: decode only, pool at least top_k_groups slots
    dec = _cfg(hga, q_begin=4095, q_len=1)
    assert L.hga_gather_kv_warm(by(dec), P, P, P, P, P, P, P, None, 128, 0, P, None, P, P,
                                None) == -1
    assert L.hga_gather_kv_warm(by(_cfg(hga)), P, P, P, P, P, P, P, P, 128, 0, P, None, P, P,
                                None) == -8
    assert L.hga_gather_kv_warm(by(dec), P, P, P, P, P, P, P, P, 64, 0, P, None, P, P,
                                None) == -2
    assert L.hga_gather_kv_warm(by(dec), P, P, P, P, P, P, P, P, 128, 0, P, P + 4, P, P,
                                None) == -3
