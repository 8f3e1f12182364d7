"""TEST INFRASTRUCTURE ONLY: Python front end of the double-precision CPU oracle.

Loads (building it first if needed) ``oracle/libhga_oracle.so`` compiled
from ``hga_oracle.c`` and exposes its functions on numpy arrays. Only the
test suite, the smoke check and the benchmark's CPU-baseline leg use this
module; the product path never imports it. It shares no code with the CUDA
library and imports nothing from the product package (``pipeline`` reads the
workload description it is given by attribute only).

Method source: "Technische Samenvatting: Hierarchical Global Attention (HGA)"
(gist.science), section "Kernmechanisme" items 1-4; see hga_oracle.c for the
readings taken where the page is silent. Parity unpinned (the pages cannot
decide them): the RoPE pairing, the representative position and the routing
query's aggregation; everything else is pinned in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hga_oracle.c")
_LIB = os.path.join(_HERE, "libhga_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain C, OpenMP over independent units)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-ffp-contract=off", "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


class OracleCfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "seq_len", "n_q_heads", "n_kv_heads", "head_dim", "chunk_size",
        "groups_per_chunk", "n_sink", "n_local", "top_k_chunks", "top_k_groups",
        "n_high_freq_pairs")] + [("rope_theta", ctypes.c_double),
                                 ("q_begin", ctypes.c_int32), ("q_len", ctypes.c_int32)]


_P = ctypes.c_void_p


def lib():
    global _lib
    with _lock:
        if _lib is None:
            handle = ctypes.CDLL(build())
            sig = {
                "hgaref_round_bf16": (ctypes.c_double, [ctypes.c_double]),
                "hgaref_round_bf16_n": (None, [_P, _P, ctypes.c_int64]),
                "hgaref_e4m3_value": (ctypes.c_double, [ctypes.c_uint8]),
                "hgaref_e4m3_decode_n": (None, [_P, ctypes.c_int64, ctypes.c_double, _P]),
                "hgaref_rope": (None, [_P, _P, ctypes.c_int64, ctypes.c_int, ctypes.c_int64,
                                       ctypes.c_int, _P]),
                "hgaref_build_summaries": (None, [_P, _P, _P, _P]),
                "hgaref_qbar": (None, [_P, _P, _P]),
                "hgaref_is_forced": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.c_int64]),
                "hgaref_route_chunks": (None, [_P, _P, _P, _P, _P, _P]),
                "hgaref_route_groups": (None, [_P, _P, _P, _P, _P, _P, _P, _P]),
                "hgaref_attend": (None, [_P, _P, _P, _P, _P, _P, _P, ctypes.c_int64, _P]),
                "hgaref_num_threads": (ctypes.c_int, []),
                "hgaref_set_num_threads": (None, [ctypes.c_int]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(handle, name)
                fn.restype = res
                fn.argtypes = args
            _lib = handle
    return _lib


def make_cfg(batch, seq_len, n_q_heads, n_kv_heads, head_dim, chunk_size, groups_per_chunk,
             n_sink, n_local, top_k_chunks, top_k_groups, n_high_freq_pairs, rope_theta,
             q_begin=0, q_len=None) -> OracleCfg:
    if head_dim > 512 or head_dim % 2:
        raise ValueError("oracle supports even head_dim <= 512")
    if chunk_size % groups_per_chunk:
        raise ValueError("groups_per_chunk must divide chunk_size")
    return OracleCfg(batch, seq_len, n_q_heads, n_kv_heads, head_dim, chunk_size,
                     groups_per_chunk, n_sink, n_local, top_k_chunks, top_k_groups,
                     n_high_freq_pairs, float(rope_theta), q_begin,
                     seq_len - q_begin if q_len is None else q_len)


def cfg_of(w, q_begin: Optional[int] = None, q_len: Optional[int] = None) -> OracleCfg:
    """OracleCfg from a synth.Workload-like object (attribute access only)."""
    qb = w.q_begin if q_begin is None else q_begin
    ql = w.q_len if q_len is None else q_len
    return make_cfg(w.batch, w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk_size,
                    w.groups_per_chunk, w.n_sink, w.n_local, w.top_k_chunks, w.top_k_groups,
                    w.n_high_freq_pairs, w.rope_theta, qb, ql)


def _f32(a) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def n_chunks(cfg: OracleCfg) -> int:
    return -(-cfg.seq_len // cfg.chunk_size)


def n_qchunks(cfg: OracleCfg) -> int:
    if cfg.q_len <= 0:
        return 0
    return (cfg.q_begin + cfg.q_len - 1) // cfg.chunk_size - cfg.q_begin // cfg.chunk_size + 1


def round_bf16(x: float) -> float:
    return lib().hgaref_round_bf16(float(x))


def round_bf16_array(a) -> np.ndarray:
    """Every element rounded to bf16 (as round_bf16), float64 out."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    out = np.empty_like(a)
    lib().hgaref_round_bf16_n(_ptr(a), _ptr(out), a.size)
    return out


def e4m3_value(code: int) -> float:
    """Value of one E4M3 (FP8) code."""
    return lib().hgaref_e4m3_value(int(code) & 0xFF)


def e4m3_decode(codes, scale: float = 1.0) -> np.ndarray:
    """Every E4M3 code (uint8 array, any shape) decoded and times scale,
    float64 out: an FP8 K or V cache as the attention reads it."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    lib().hgaref_e4m3_decode_n(_ptr(c), c.size, float(scale), _ptr(out))
    return out


def rope(cfg: OracleCfg, x, pos0: int, round_bf16: bool) -> np.ndarray:
    """x [n_tok, n_heads, d] -> R(pos) x in float64 (bf16-rounded if asked)."""
    x = _f32(x)
    n_tok, n_heads, d = x.shape
    assert d == cfg.head_dim
    out = np.empty(x.shape, dtype=np.float64)
    lib().hgaref_rope(ctypes.byref(cfg), _ptr(x), n_tok, n_heads, pos0, int(round_bf16),
                      _ptr(out))
    return out


def rope_f32(cfg: OracleCfg, x, pos0: int, round_bf16: bool, slab: int = 4096) -> np.ndarray:
    """As rope() but returns float32, processing slabs of tokens to bound memory.
    With round_bf16 the float32 result holds exact bf16 values."""
    x = np.asarray(x)
    out = np.empty(x.shape, dtype=np.float32)
    for t0 in range(0, x.shape[0], slab):
        out[t0:t0 + slab] = rope(cfg, x[t0:t0 + slab], pos0 + t0, round_bf16)
    return out


def build_summaries(cfg: OracleCfg, k_raw):
    k_raw = _f32(k_raw)
    B, H, L, d = k_raw.shape
    nC = n_chunks(cfg)
    cs = np.empty((B, H, nC, d), dtype=np.float64)
    gs = np.empty((B, H, nC * cfg.groups_per_chunk, d), dtype=np.float64)
    lib().hgaref_build_summaries(ctypes.byref(cfg), _ptr(k_raw), _ptr(cs), _ptr(gs))
    return cs, gs


def qbar(cfg: OracleCfg, q_rot) -> np.ndarray:
    q_rot = _f32(q_rot)
    out = np.empty((cfg.batch, cfg.n_kv_heads, n_qchunks(cfg), cfg.head_dim), dtype=np.float64)
    lib().hgaref_qbar(ctypes.byref(cfg), _ptr(q_rot), _ptr(out))
    return out


def is_forced(cfg: OracleCfg, j: int, ch: int) -> bool:
    return bool(lib().hgaref_is_forced(ctypes.byref(cfg), j, ch))


def route_chunks(cfg: OracleCfg, qb, chunk_sum, want_scores: bool = True):
    qb = np.ascontiguousarray(qb, dtype=np.float64)
    chunk_sum = np.ascontiguousarray(chunk_sum, dtype=np.float64)
    B, H, nQC, _ = qb.shape
    kc = cfg.top_k_chunks
    sel = np.empty((B, H, nQC, kc), dtype=np.int32)
    nsel = np.empty((B, H, nQC), dtype=np.int32)
    sc = np.empty((B, H, nQC, n_chunks(cfg)), dtype=np.float32) if want_scores else None
    lib().hgaref_route_chunks(ctypes.byref(cfg), _ptr(qb), _ptr(chunk_sum), _ptr(sel),
                              _ptr(nsel), _ptr(sc) if sc is not None else None)
    return sel, nsel, sc


def route_groups(cfg: OracleCfg, qb, group_sum, sel_chunks, n_sel_chunks, want_scores=True):
    qb = np.ascontiguousarray(qb, dtype=np.float64)
    group_sum = np.ascontiguousarray(group_sum, dtype=np.float64)
    sel_chunks = np.ascontiguousarray(sel_chunks, dtype=np.int32)
    n_sel_chunks = np.ascontiguousarray(n_sel_chunks, dtype=np.int32)
    B, H, nQC, _ = qb.shape
    kg, kc, G = cfg.top_k_groups, cfg.top_k_chunks, cfg.groups_per_chunk
    sel = np.empty((B, H, nQC, kg), dtype=np.int32)
    nsel = np.empty((B, H, nQC), dtype=np.int32)
    sc = np.empty((B, H, nQC, kc * G), dtype=np.float32) if want_scores else None
    lib().hgaref_route_groups(ctypes.byref(cfg), _ptr(qb), _ptr(group_sum), _ptr(sel_chunks),
                              _ptr(n_sel_chunks), _ptr(sel), _ptr(nsel),
                              _ptr(sc) if sc is not None else None)
    return sel, nsel, sc


def attend(cfg: OracleCfg, q_rot, k_rot, v, sel_groups, n_sel_groups, units=None,
           out: Optional[np.ndarray] = None) -> np.ndarray:
    """Exact softmax attention over the routed set. units: int array [n,3] of
    (b, kv head, query-chunk index) to compute, or None for all."""
    q_rot, k_rot, v = _f32(q_rot), _f32(k_rot), _f32(v)
    sel_groups = np.ascontiguousarray(sel_groups, dtype=np.int32)
    n_sel_groups = np.ascontiguousarray(n_sel_groups, dtype=np.int32)
    if out is None:
        out = np.full(q_rot.shape, np.nan, dtype=np.float64)
    u = None
    n_units = 0
    if units is not None:
        u = np.ascontiguousarray(units, dtype=np.int32).reshape(-1, 3)
        n_units = u.shape[0]
    lib().hgaref_attend(ctypes.byref(cfg), _ptr(q_rot), _ptr(k_rot), _ptr(v), _ptr(sel_groups),
                        _ptr(n_sel_groups), _ptr(u) if u is not None else None, n_units,
                        _ptr(out))
    return out


def set_threads(n: int) -> None:
    lib().hgaref_set_num_threads(int(n))


def num_threads() -> int:
    return int(lib().hgaref_num_threads())


def pipeline(w, inputs, units=None, want_scores: bool = True, attend_out: bool = True,
             bf16_summaries: bool = False):
    """The whole oracle hot path on drawn inputs (torch CPU tensors or numpy).

    Steps, each the oracle's own: rotate queries and keys (rounded to bf16 for
    bf16 workloads: the storage type of the query and of the attention cache),
    build summaries from the raw keys (rounded to bf16 when bf16_summaries:
    the bf16 summary-table variant routes on the rounded values), q-bar,
    chunk routing, group routing, and exact attention (on `units` only, if
    given).
    """
    cfg = cfg_of(w)
    rb = w.dtype == "bf16"
    k_raw = _as_np(inputs["k_raw"])
    v = _as_np(inputs["v"])
    q_raw = _as_np(inputs["q_raw"])
    B, H, L, d = k_raw.shape
    k_rot = np.empty_like(k_raw)
    for b in range(B):
        for h in range(H):
            k_rot[b, h] = rope_f32(cfg, k_raw[b, h][:, None, :], 0, rb)[:, 0, :]
    q_rot = np.empty_like(q_raw)
    for b in range(B):
        q_rot[b] = rope_f32(cfg, q_raw[b], cfg.q_begin, rb)
    cs, gs = build_summaries(cfg, k_raw)
    if bf16_summaries:
        cs, gs = round_bf16_array(cs), round_bf16_array(gs)
    qb = qbar(cfg, q_rot)
    sel_c, nsel_c, sc_c = route_chunks(cfg, qb, cs, want_scores)
    sel_g, nsel_g, sc_g = route_groups(cfg, qb, gs, sel_c, nsel_c, want_scores)
    res = dict(cfg=cfg, k_rot=k_rot, q_rot=q_rot, chunk_sum=cs, group_sum=gs, qbar=qb,
               sel_chunks=sel_c, n_sel_chunks=nsel_c, chunk_scores=sc_c,
               sel_groups=sel_g, n_sel_groups=nsel_g, group_scores=sc_g)
    if attend_out:
        res["out"] = attend(cfg, q_rot, k_rot, v, sel_g, nsel_g, units)
    return res


def per_q_head(w, inputs):
    """Per-query-head routing (the variant in which every query head routes
    on its own rotated queries instead of the KV head's shared q-bar), stated
    as the plain routing of an expanded problem: query head h gets its own
    copy of the raw keys and values of its KV head h // gq, so its routing
    query is the mean of its own queries over the chunk's tokens, it scores
    and selects over that KV head's summaries, and it attends over its own
    selection. Returns (w_h, inputs_h) to give to pipeline(); w_h has as many
    KV heads as query heads (w.replace is the workload's own copy-with)."""
    gq = w.n_q_heads // w.n_kv_heads
    w_h = w.replace(n_kv_heads=w.n_q_heads)
    inputs_h = dict(inputs)
    inputs_h["k_raw"] = np.repeat(_as_np(inputs["k_raw"]), gq, axis=1)
    inputs_h["v"] = np.repeat(_as_np(inputs["v"]), gq, axis=1)
    return w_h, inputs_h


def _as_np(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, dtype=np.float32)
    return t.float().contiguous().numpy()
