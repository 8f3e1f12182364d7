"""Thin ctypes binding of libhga.so (the C ABI declared in include/hga.h).

Argument marshalling only: each function checks that the torch tensors it is
given live on the current CUDA device with the dtype, shape and contiguity
the call expects, passes their data pointers and the current CUDA stream to
the C entry point of the same name, and raises HgaError on a non-OK status.
Every step of the hot path runs in the library's kernels; there is no other
implementation behind these functions. Importing this module fails loudly if
libhga.so has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhga.so")

HGA_OK = 0
HGA_BF16, HGA_F32 = 0, 1
HGA_KV_FULL, HGA_KV_WINDOWS = 0, 1
HGA_SUMMARY_F32, HGA_SUMMARY_BF16 = 0, 1
HGA_KV_AS_DTYPE, HGA_KV_E4M3 = 0, 1
HGA_ROUTE_PER_KV_HEAD, HGA_ROUTE_PER_Q_HEAD = 0, 1
STATUS = {0: "HGA_OK", -1: "HGA_ERR_NULL", -2: "HGA_ERR_SHAPE", -3: "HGA_ERR_ALIGN",
          -4: "HGA_ERR_CONFIG", -5: "HGA_ERR_CUDA", -6: "HGA_ERR_DEVICE_INDEX",
          -7: "HGA_ERR_TIMEOUT", -8: "HGA_ERR_UNSUPPORTED", -9: "HGA_ERR_MEMORY",
          -10: "HGA_ERR_SCRATCH_LIMIT"}


class HgaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {_lib.hga_status_string(status).decode()}"
        if status == -5:  # HGA_ERR_CUDA: name the failed CUDA call's error
            code = int(_lib.hga_last_cuda_error())
            msg += f" (cudaError {code}: {_lib.hga_cuda_error_string(code).decode()})"
        super().__init__(msg)


class HgaConfig(ctypes.Structure):
    """Mirror of hga_config."""
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "seq_len", "n_q_heads", "n_kv_heads", "head_dim", "chunk_size",
        "groups_per_chunk", "n_sink", "n_local", "top_k_chunks", "top_k_groups",
        "n_high_freq_pairs")] + [("rope_theta", ctypes.c_double)] + [
        (n, ctypes.c_int32) for n in ("dtype", "q_begin", "q_len", "kv_layout", "summary_type",
                                      "kv_type")] + [
        ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float), ("routing", ctypes.c_int32)]

    @property
    def n_chunks(self) -> int:
        return -(-self.seq_len // self.chunk_size)

    @property
    def n_qchunks(self) -> int:
        if self.q_len <= 0:
            return 0
        return (self.q_begin + self.q_len - 1) // self.chunk_size - self.q_begin // self.chunk_size + 1

    @property
    def route_heads(self) -> int:
        """Rows of q-bar and of the selection lists per sequence."""
        return self.n_q_heads if self.routing == HGA_ROUTE_PER_Q_HEAD else self.n_kv_heads

    @property
    def group_size(self) -> int:
        return self.chunk_size // self.groups_per_chunk

    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == HGA_BF16 else torch.float32

    def summary_torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.summary_type == HGA_SUMMARY_BF16 else torch.float32

    def kv_torch_dtype(self) -> torch.dtype:
        """Element type of the key/value stores and buffers."""
        return torch.float8_e4m3fn if self.kv_type == HGA_KV_E4M3 else self.torch_dtype()

    def copy(self, **kw) -> "HgaConfig":
        c = HgaConfig()
        ctypes.pointer(c)[0] = self
        for k, v in kw.items():
            setattr(c, k, v)
        return c


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build the CUDA library first "
            "(python -m long_context_rope_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    C = ctypes.POINTER(HgaConfig)
    sig = {
        "hga_apply_rope": [C, P, P, I64, I64, I32, I64, P],
        "hga_build_summaries": [C, P, P, P, P, I32, I32, P],
        "hga_route_chunks": [C, P, P, P, P, P, P, P],
        "hga_route_groups": [C, P, P, P, P, P, P, P, P],
        "hga_gather_kv": [C, P, P, I32, P, P, P, P, P],
        "hga_attend": [C, P, P, P, P, P, P, P, P, P],
        "hga_route": [C, P, P, P, P, P, P, P, P, P],
        "hga_decode_step": [C, P, P, P, P, P, P, P, P, P, P, P, P],
        "hga_decode_step_tiered": [C, P, P, P, P, P, P, P, P, P, P, P, P, P, P],
        "hga_gather_kv_warm": [C, P, P, P, P, P, P, P, P, I32, I32, P, P, P, P, P],
        "hga_gather_kv_warm_noalloc": [C, P, P, P, P, P, P, P, P, I32, I32, P, P, P, P],
        "hga_get_device_error": [P, ctypes.POINTER(I32)],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.hga_status_string.argtypes = [ctypes.c_int]
    lib.hga_status_string.restype = ctypes.c_char_p
    lib.hga_version.restype = ctypes.c_int32
    lib.hga_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.hga_set_wait_limit_ns.restype = None
    lib.hga_last_cuda_error.argtypes = []
    lib.hga_last_cuda_error.restype = ctypes.c_int32
    lib.hga_cuda_error_string.argtypes = [ctypes.c_int32]
    lib.hga_cuda_error_string.restype = ctypes.c_char_p
    return lib


_lib = _load()


def library() -> ctypes.CDLL:
    return _lib


def config_from(w, **overrides) -> HgaConfig:
    """HgaConfig from a synth.Workload (or any object with the same fields)."""
    c = HgaConfig()
    for f in ("batch", "seq_len", "n_q_heads", "n_kv_heads", "head_dim", "chunk_size",
              "groups_per_chunk", "n_sink", "n_local", "top_k_chunks", "top_k_groups",
              "n_high_freq_pairs"):
        setattr(c, f, int(getattr(w, f)))
    c.rope_theta = float(w.rope_theta)
    c.dtype = HGA_BF16 if w.dtype == "bf16" else HGA_F32
    c.q_begin = int(w.q_begin)
    c.q_len = int(w.q_len)
    c.kv_layout = HGA_KV_FULL
    c.summary_type = HGA_SUMMARY_F32
    c.kv_type = HGA_KV_AS_DTYPE
    c.k_scale = c.v_scale = 1.0
    c.routing = HGA_ROUTE_PER_KV_HEAD
    for k, v in overrides.items():
        setattr(c, k, v)
    return c


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None, shape=None, device=True,
         nullable=False) -> Optional[int]:
    if t is None:
        if nullable:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _check(status: int, where: str) -> None:
    if status != HGA_OK:
        raise HgaError(status, where)


def apply_rope(cfg: HgaConfig, x: torch.Tensor, x_rot: torch.Tensor, n_outer: int,
               n_tokens: int, n_heads: int, pos0: int, stream=None) -> None:
    shape = (n_outer, n_tokens, n_heads, cfg.head_dim)
    if x.numel() != n_outer * n_tokens * n_heads * cfg.head_dim:
        raise ValueError(f"x must hold {shape} elements")
    _check(_lib.hga_apply_rope(ctypes.byref(cfg), _ptr(x, "x", cfg.torch_dtype()),
                               _ptr(x_rot, "x_rot", cfg.torch_dtype(), x.shape), n_outer,
                               n_tokens, n_heads, pos0, _stream(stream)), "hga_apply_rope")


def build_summaries(cfg: HgaConfig, k_raw, chunk_sum, group_sum, k_rot=None, chunk_begin=0,
                    chunk_end=None, stream=None) -> None:
    B, H, L, d, nC, G = (cfg.batch, cfg.n_kv_heads, cfg.seq_len, cfg.head_dim, cfg.n_chunks,
                         cfg.groups_per_chunk)
    dt = cfg.torch_dtype()
    _check(_lib.hga_build_summaries(
        ctypes.byref(cfg), _ptr(k_raw, "k_raw", dt, (B, H, L, d)),
        _ptr(chunk_sum, "chunk_sum", cfg.summary_torch_dtype(), (B, H, nC, d)),
        _ptr(group_sum, "group_sum", cfg.summary_torch_dtype(), (B, H, nC * G, d)),
        _ptr(k_rot, "k_rot", dt, (B, H, L, d), nullable=True), int(chunk_begin),
        int(nC if chunk_end is None else chunk_end), _stream(stream)), "hga_build_summaries")


def route_chunks(cfg: HgaConfig, q_rot, chunk_sum, qbar, sel_chunks, n_sel_chunks, scores=None,
                 stream=None) -> None:
    B, H, d, nQC = cfg.batch, cfg.n_kv_heads, cfg.head_dim, cfg.n_qchunks
    R = cfg.route_heads
    _check(_lib.hga_route_chunks(
        ctypes.byref(cfg), _ptr(q_rot, "q_rot", cfg.torch_dtype(),
                                (B, cfg.q_len, cfg.n_q_heads, d)),
        _ptr(chunk_sum, "chunk_sum", cfg.summary_torch_dtype(), (B, H, cfg.n_chunks, d)),
        _ptr(qbar, "qbar", torch.float32, (B, R, nQC, d)),
        _ptr(sel_chunks, "sel_chunks", torch.int32, (B, R, nQC, cfg.top_k_chunks)),
        _ptr(n_sel_chunks, "n_sel_chunks", torch.int32, (B, R, nQC)),
        _ptr(scores, "scores", torch.float32, (B, R, nQC, cfg.n_chunks), nullable=True),
        _stream(stream)), "hga_route_chunks")


def route_groups(cfg: HgaConfig, qbar, group_sum, sel_chunks, n_sel_chunks, sel_groups,
                 n_sel_groups, scores=None, stream=None) -> None:
    B, H, d, nQC, G = cfg.batch, cfg.n_kv_heads, cfg.head_dim, cfg.n_qchunks, cfg.groups_per_chunk
    R = cfg.route_heads
    _check(_lib.hga_route_groups(
        ctypes.byref(cfg), _ptr(qbar, "qbar", torch.float32, (B, R, nQC, d)),
        _ptr(group_sum, "group_sum", cfg.summary_torch_dtype(), (B, H, cfg.n_chunks * G, d)),
        _ptr(sel_chunks, "sel_chunks", torch.int32, (B, R, nQC, cfg.top_k_chunks)),
        _ptr(n_sel_chunks, "n_sel_chunks", torch.int32, (B, R, nQC)),
        _ptr(sel_groups, "sel_groups", torch.int32, (B, R, nQC, cfg.top_k_groups)),
        _ptr(n_sel_groups, "n_sel_groups", torch.int32, (B, R, nQC)),
        _ptr(scores, "scores", torch.float32, (B, R, nQC, cfg.top_k_chunks * G), nullable=True),
        _stream(stream)), "hga_route_groups")


def _route_ptrs(cfg: HgaConfig, q_rot, chunk_sum, group_sum, qbar, sel_chunks, n_sel_chunks,
                sel_groups, n_sel_groups):
    B, H, d, nQC, G = cfg.batch, cfg.n_kv_heads, cfg.head_dim, cfg.n_qchunks, cfg.groups_per_chunk
    R = cfg.route_heads
    return [
        _ptr(q_rot, "q_rot", cfg.torch_dtype(), (B, cfg.q_len, cfg.n_q_heads, d)),
        _ptr(chunk_sum, "chunk_sum", cfg.summary_torch_dtype(), (B, H, cfg.n_chunks, d)),
        _ptr(group_sum, "group_sum", cfg.summary_torch_dtype(), (B, H, cfg.n_chunks * G, d)),
        _ptr(qbar, "qbar", torch.float32, (B, R, nQC, d)),
        _ptr(sel_chunks, "sel_chunks", torch.int32, (B, R, nQC, cfg.top_k_chunks)),
        _ptr(n_sel_chunks, "n_sel_chunks", torch.int32, (B, R, nQC)),
        _ptr(sel_groups, "sel_groups", torch.int32, (B, R, nQC, cfg.top_k_groups)),
        _ptr(n_sel_groups, "n_sel_groups", torch.int32, (B, R, nQC)),
    ]


def route(cfg: HgaConfig, q_rot, chunk_sum, group_sum, qbar, sel_chunks, n_sel_chunks, sel_groups,
          n_sel_groups, stream=None) -> None:
    """Both routing levels (one launch for a one-token span)."""
    args = _route_ptrs(cfg, q_rot, chunk_sum, group_sum, qbar, sel_chunks, n_sel_chunks,
                       sel_groups, n_sel_groups)
    _check(_lib.hga_route(ctypes.byref(cfg), *args, _stream(stream)), "hga_route")


def decode_step(cfg: HgaConfig, q_rot, chunk_sum, group_sum, k_cache, v_cache, qbar, sel_chunks,
                n_sel_chunks, sel_groups, n_sel_groups, out, stream=None) -> None:
    """Routing plus attention over the full resident cache (one launch for decode)."""
    B, H, L, d = cfg.batch, cfg.n_kv_heads, cfg.seq_len, cfg.head_dim
    dt, kvt = cfg.torch_dtype(), cfg.kv_torch_dtype()
    r = _route_ptrs(cfg, q_rot, chunk_sum, group_sum, qbar, sel_chunks, n_sel_chunks, sel_groups,
                    n_sel_groups)
    _check(_lib.hga_decode_step(
        ctypes.byref(cfg), r[0], r[1], r[2],
        _ptr(k_cache, "k_cache", kvt, (B, H, L, d)), _ptr(v_cache, "v_cache", kvt, (B, H, L, d)),
        *r[3:], _ptr(out, "out", dt, (B, cfg.q_len, cfg.n_q_heads, d)), _stream(stream)),
        "hga_decode_step")


def decode_step_tiered(cfg: HgaConfig, q_rot, chunk_sum, group_sum, k_win, v_win, k_host, v_host,
                       qbar, sel_chunks, n_sel_chunks, sel_groups, n_sel_groups, out,
                       stream=None) -> None:
    """One tiered decode step in one launch: routing, attention over the
    resident forced windows and the routed groups read from host memory."""
    B, H, L, d = cfg.batch, cfg.n_kv_heads, cfg.seq_len, cfg.head_dim
    dt, kvt = cfg.torch_dtype(), cfg.kv_torch_dtype()
    win = (B, H, window_slots(cfg) * cfg.chunk_size, d)
    r = _route_ptrs(cfg, q_rot, chunk_sum, group_sum, qbar, sel_chunks, n_sel_chunks, sel_groups,
                    n_sel_groups)
    _check(_lib.hga_decode_step_tiered(
        ctypes.byref(cfg), r[0], r[1], r[2], _ptr(k_win, "k_win", kvt, win),
        _ptr(v_win, "v_win", kvt, win), _ptr(k_host, "k_host", kvt, (B, H, L, d), device=False),
        _ptr(v_host, "v_host", kvt, (B, H, L, d), device=False), *r[3:],
        _ptr(out, "out", dt, (B, cfg.q_len, cfg.n_q_heads, d)), _stream(stream)),
        "hga_decode_step_tiered")


def gather_kv(cfg: HgaConfig, k_src, v_src, src_is_host: bool, sel_groups, n_sel_groups, k_dst,
              v_dst, stream=None) -> None:
    B, H, L, d, nQC = cfg.batch, cfg.n_kv_heads, cfg.seq_len, cfg.head_dim, cfg.n_qchunks
    dt = cfg.kv_torch_dtype()
    dst_shape = (B, H, nQC, cfg.top_k_groups * cfg.group_size, d)
    _check(_lib.hga_gather_kv(
        ctypes.byref(cfg), _ptr(k_src, "k_src", dt, (B, H, L, d), device=not src_is_host),
        _ptr(v_src, "v_src", dt, (B, H, L, d), device=not src_is_host), int(bool(src_is_host)),
        _ptr(sel_groups, "sel_groups", torch.int32, (B, H, nQC, cfg.top_k_groups)),
        _ptr(n_sel_groups, "n_sel_groups", torch.int32, (B, H, nQC)),
        _ptr(k_dst, "k_dst", dt, dst_shape), _ptr(v_dst, "v_dst", dt, dst_shape),
        _stream(stream)), "hga_gather_kv")


def gather_kv_warm(cfg: HgaConfig, k_host, v_host, sel_groups, n_sel_groups, pool_k, pool_v,
                   pool_tag, pool_last, step: int, src_out, k_dst, v_dst, stats=None,
                   stream=None) -> None:
    """Warm-tier gather for a one-token query span (see hga_gather_kv_warm)."""
    B, H, d, kg, g = cfg.batch, cfg.n_kv_heads, cfg.head_dim, cfg.top_k_groups, cfg.group_size
    dt = cfg.kv_torch_dtype()
    n_slots = pool_tag.shape[-1]
    store = (B, H, cfg.seq_len, d)
    gat_shape = (B, H, cfg.n_qchunks, kg * g, d)
    _check(_lib.hga_gather_kv_warm(
        ctypes.byref(cfg), _ptr(k_host, "k_host", dt, store, device=False),
        _ptr(v_host, "v_host", dt, store, device=False),
        _ptr(sel_groups, "sel_groups", torch.int32, (B, H, cfg.n_qchunks, kg)),
        _ptr(n_sel_groups, "n_sel_groups", torch.int32, (B, H, cfg.n_qchunks)),
        _ptr(pool_k, "pool_k", dt, (B, H, n_slots, g, d)),
        _ptr(pool_v, "pool_v", dt, (B, H, n_slots, g, d)),
        _ptr(pool_tag, "pool_tag", torch.int32, (B, H, n_slots)),
        _ptr(pool_last, "pool_last", torch.int32, (B, H, n_slots)), n_slots, step,
        _ptr(src_out, "src_out", torch.int32, (B, H, kg)),
        _ptr(stats, "stats", torch.int32, (B, H, 2), nullable=True),
        _ptr(k_dst, "k_dst", dt, gat_shape), _ptr(v_dst, "v_dst", dt, gat_shape),
        _stream(stream)), "hga_gather_kv_warm")


def gather_kv_warm_noalloc(cfg: HgaConfig, k_host, v_host, sel_groups, n_sel_groups, pool_k,
                           pool_v, pool_tag, pool_last, step: int, k_dst, v_dst, stats=None,
                           stream=None) -> None:
    """gather_kv_warm for callers that may not allocate device memory: the
    plan-to-copy source list lives in the library's fixed scratch array
    (see hga_gather_kv_warm_noalloc). Allocates nothing itself either."""
    B, H, d, kg, g = cfg.batch, cfg.n_kv_heads, cfg.head_dim, cfg.top_k_groups, cfg.group_size
    dt = cfg.kv_torch_dtype()
    n_slots = pool_tag.shape[-1]
    store = (B, H, cfg.seq_len, d)
    gat_shape = (B, H, cfg.n_qchunks, kg * g, d)
    _check(_lib.hga_gather_kv_warm_noalloc(
        ctypes.byref(cfg), _ptr(k_host, "k_host", dt, store, device=False),
        _ptr(v_host, "v_host", dt, store, device=False),
        _ptr(sel_groups, "sel_groups", torch.int32, (B, H, cfg.n_qchunks, kg)),
        _ptr(n_sel_groups, "n_sel_groups", torch.int32, (B, H, cfg.n_qchunks)),
        _ptr(pool_k, "pool_k", dt, (B, H, n_slots, g, d)),
        _ptr(pool_v, "pool_v", dt, (B, H, n_slots, g, d)),
        _ptr(pool_tag, "pool_tag", torch.int32, (B, H, n_slots)),
        _ptr(pool_last, "pool_last", torch.int32, (B, H, n_slots)), n_slots, step,
        _ptr(stats, "stats", torch.int32, (B, H, 2), nullable=True),
        _ptr(k_dst, "k_dst", dt, gat_shape), _ptr(v_dst, "v_dst", dt, gat_shape),
        _stream(stream)), "hga_gather_kv_warm_noalloc")


def window_slots(cfg: HgaConfig) -> int:
    """Chunk slots of the resident forced-window buffer (HGA_KV_WINDOWS)."""
    return cfg.n_sink + cfg.n_local + 1


def attend(cfg: HgaConfig, q_rot, k_res, v_res, sel_groups, n_sel_groups, out, k_gat=None,
           v_gat=None, stream=None) -> None:
    B, H, L, d, nQC = cfg.batch, cfg.n_kv_heads, cfg.seq_len, cfg.head_dim, cfg.n_qchunks
    dt, kvt = cfg.torch_dtype(), cfg.kv_torch_dtype()
    res_len = L if cfg.kv_layout == HGA_KV_FULL else window_slots(cfg) * cfg.chunk_size
    gat_shape = (B, H, nQC, cfg.top_k_groups * cfg.group_size, d)
    q_shape = (B, cfg.q_len, cfg.n_q_heads, d)
    _check(_lib.hga_attend(
        ctypes.byref(cfg), _ptr(q_rot, "q_rot", dt, q_shape),
        _ptr(k_res, "k_res", kvt, (B, H, res_len, d)),
        _ptr(v_res, "v_res", kvt, (B, H, res_len, d)),
        _ptr(k_gat, "k_gat", kvt, gat_shape, nullable=True),
        _ptr(v_gat, "v_gat", kvt, gat_shape, nullable=True),
        _ptr(sel_groups, "sel_groups", torch.int32, (B, cfg.route_heads, nQC, cfg.top_k_groups)),
        _ptr(n_sel_groups, "n_sel_groups", torch.int32, (B, cfg.route_heads, nQC)),
        _ptr(out, "out", dt, q_shape), _stream(stream)), "hga_attend")


def get_device_error(stream=None) -> int:
    """Synchronise the stream and read (and clear) the device error word.
    Returns 0 when clean; raises HgaError on HGA_ERR_CUDA."""
    detail = ctypes.c_int32(0)
    st = _lib.hga_get_device_error(_stream(stream), ctypes.byref(detail))
    if st == -5:
        raise HgaError(st, "hga_get_device_error")
    return int(detail.value) if st != HGA_OK else 0


def set_wait_limit_ns(limit_ns: int) -> None:
    """Limit of every bounded device wait of later launches (0 = default 1 s)."""
    _lib.hga_set_wait_limit_ns(int(limit_ns))


def version() -> int:
    return int(_lib.hga_version())
