"""Seeded synthetic inputs for the HGA hot path: planted-topic workloads.

This module draws random tensors and nothing else. It holds no step of the
method (no rotation, no summary, no score, no selection, no softmax), so both
the CUDA path and the CPU oracle can take their inputs from it. It imports
nothing from the rest of the package.

Workload shapes follow the HGA technical summary (gist.science, "Technische
Samenvatting: Hierarchical Global Attention (HGA)"), section "Kernmechanisme"
item 1 (fixed chunks, e.g. C=64, split into groups) and section
"Experimentele Resultaten" (4K-64K context, about 3% of tokens attended).

Recipe (one torch CPU generator per call, seeded; draw order fixed):
  1. topics  ~ N(0, 4) per (sequence, KV head, chunk), shape [B, Hkv, nC, d]
  2. k_raw   ~ N(0, 1) [B, Hkv, L, d], plus the topic of the token's own chunk
  3. v       ~ N(0, 1) [B, Hkv, L, d]
  4. q_raw   ~ N(0, 1) [B, Lq, Hq, d]
  5. plant choices: a query chunk j gets the sum of the topic vectors of
     `plant_count` distinct chunks drawn uniformly from [0, j), added to every
     query token of chunk j for all query heads of the topic's KV head.
All values are drawn in float32 and then cast to the workload's dtype.

FP8 K/V caches (the E4M3 storage variant) are made from drawn or rotated
tensors by `to_e4m3`: a per-tensor scale amax / 448 and torch's
float8_e4m3fn cast, the same kind of storage conversion as the bf16 cast.
"""
from __future__ import annotations

import dataclasses
from typing import Dict

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and routing parameters of one synthetic HGA workload."""

    name: str
    batch: int
    seq_len: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    chunk_size: int
    groups_per_chunk: int
    n_sink: int
    n_local: int
    top_k_chunks: int
    top_k_groups: int
    rope_theta: float
    n_high_freq_pairs: int
    dtype: str  # "bf16" or "f32"
    mode: str  # "prefill" or "decode"
    plant_every: int  # prefill: plant into query chunks j>0 with j % plant_every == 0
    plant_count: int  # prefill: earlier chunks planted per query chunk (clamped to j)
    tiered: bool = False  # decode only: token K/V lives in pinned host memory
    # prefill only: an explicit query span [span_begin, span_begin + span_len)
    # (a chunked prefill); -1 = the whole context
    span_begin: int = -1
    span_len: int = -1

    @property
    def n_chunks(self) -> int:
        return (self.seq_len + self.chunk_size - 1) // self.chunk_size

    @property
    def group_size(self) -> int:
        return self.chunk_size // self.groups_per_chunk

    @property
    def q_begin(self) -> int:
        if self.mode != "prefill":
            return self.seq_len - 1
        return 0 if self.span_begin < 0 else self.span_begin

    @property
    def q_len(self) -> int:
        if self.mode != "prefill":
            return 1
        return self.seq_len if self.span_begin < 0 else self.span_len

    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _gqa_heads(n_q_heads: int, n_kv_heads: int) -> int:
    if n_q_heads % n_kv_heads:
        raise ValueError("n_q_heads must be a multiple of n_kv_heads")
    return n_q_heads // n_kv_heads


# The five workloads. Sizes and routing parameters as stated for each; the
# routing parameters of the bf16 workloads are shared.
_BF16_ROUTING = dict(n_q_heads=32, n_kv_heads=4, head_dim=128, chunk_size=64,
                     groups_per_chunk=4, n_sink=1, n_local=2, top_k_chunks=32,
                     top_k_groups=96, rope_theta=1e6, n_high_freq_pairs=32,
                     dtype="bf16")

WORKLOADS: Dict[str, Workload] = {
    "tiny_f32": Workload(
        name="tiny_f32", batch=1, seq_len=1024, n_q_heads=1, n_kv_heads=1,
        head_dim=64, chunk_size=64, groups_per_chunk=4, n_sink=1, n_local=1,
        top_k_chunks=2, top_k_groups=4, rope_theta=1e4, n_high_freq_pairs=16,
        dtype="f32", mode="prefill", plant_every=8, plant_count=1),
    "prefill_4k": Workload(name="prefill_4k", batch=1, seq_len=4096,
                           mode="prefill", plant_every=1, plant_count=3,
                           **_BF16_ROUTING),
    "decode_16x32k": Workload(name="decode_16x32k", batch=16, seq_len=32768,
                              mode="decode", plant_every=0, plant_count=1,
                              **_BF16_ROUTING),
    "prefill_64k": Workload(name="prefill_64k", batch=1, seq_len=65536,
                            mode="prefill", plant_every=1, plant_count=3,
                            **_BF16_ROUTING),
    "tiered_decode_4x64k": Workload(name="tiered_decode_4x64k", batch=4,
                                    seq_len=65536, mode="decode", plant_every=0,
                                    plant_count=1, tiered=True, **_BF16_ROUTING),
}


def draw(w: Workload, seed: int = 0, with_kv: bool = True) -> Dict[str, object]:
    """Draw the inputs of workload `w` on the CPU.

    Returns k_raw [B,Hkv,L,d] (pre-RoPE keys), v [B,Hkv,L,d],
    q_raw [B,Lq,Hq,d] (pre-RoPE queries at positions q_begin..q_begin+Lq-1)
    in the workload dtype, plus `planted` (list per (b, query chunk) of the
    source chunks whose topics were added; used only for recall statistics).
    With with_kv=False the key/value tensors are drawn and discarded, so the
    queries are identical to a full draw.
    """
    B, L, Hq, Hkv, d = w.batch, w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim
    C, nC = w.chunk_size, w.n_chunks
    gq = _gqa_heads(Hq, Hkv)
    g = torch.Generator().manual_seed(int(seed))
    out_dtype = w.torch_dtype()

    topics = torch.randn(B, Hkv, nC, d, generator=g) * 2.0  # variance 4
    k_raw = torch.randn(B, Hkv, L, d, generator=g)
    if with_kv:
        full = (L // C) * C
        if full:
            k_raw[:, :, :full].view(B, Hkv, full // C, C, d).add_(
                topics[:, :, : full // C].unsqueeze(3))
        if full < L:
            k_raw[:, :, full:].add_(topics[:, :, nC - 1: nC])
    v = torch.randn(B, Hkv, L, d, generator=g)

    Lq = w.q_len
    q_raw = torch.randn(B, Lq, Hq, d, generator=g)
    planted = []
    if w.mode == "prefill":
        for b in range(B):
            per_b = []
            for j in range(nC):
                src: list = []
                due = j > 0 and (w.plant_every <= 1 or j % w.plant_every == 0)
                if due:
                    n_src = min(w.plant_count, j)
                    src = torch.randperm(j, generator=g)[:n_src].tolist()
                    add = topics[b, :, src].sum(dim=1)  # [Hkv, d]
                    add = add.repeat_interleave(gq, dim=0)  # [Hq, d]
                    lo = max(j * C, w.q_begin)
                    hi = min((j + 1) * C, L, w.q_begin + w.q_len)
                    if hi > lo:
                        q_raw[b, lo - w.q_begin: hi - w.q_begin] += add
                per_b.append(src)
            planted.append(per_b)
    else:
        j_q = (L - 1) // C
        for b in range(B):
            src = []
            if j_q > 0:
                src = [int(torch.randint(0, j_q, (1,), generator=g).item())]
                add = topics[b, :, src].sum(dim=1).repeat_interleave(gq, dim=0)
                q_raw[b, 0] += add
            planted.append([src])

    res = {"q_raw": q_raw.to(out_dtype), "planted": planted}
    if with_kv:
        res["k_raw"] = k_raw.to(out_dtype)
        res["v"] = v.to(out_dtype)
    return res


def bytes_per_step(w: Workload) -> Dict[str, int]:
    """Element counts turned into bytes for the host<->device copies of a step."""
    es = 2 if w.dtype == "bf16" else 4
    n_kv = w.batch * w.n_kv_heads * w.seq_len * w.head_dim
    n_q = w.batch * w.q_len * w.n_q_heads * w.head_dim
    return {"k": n_kv * es, "v": n_kv * es, "q": n_q * es, "o": n_q * es}


E4M3_MAX = 448.0


def to_e4m3(x: torch.Tensor):
    """An FP8 cache of x: (codes as torch.float8_e4m3fn, scale), with the
    per-tensor scale amax(|x|) / 448 so the largest element maps to the
    format's largest finite value; each code is x / scale cast to E4M3
    (values clamped to +-448 first, so none overflows to NaN)."""
    xf = x.float()
    amax = float(xf.abs().max()) if xf.numel() else 0.0
    scale = amax / E4M3_MAX if amax > 0 else 1.0
    scale = float(torch.tensor(scale, dtype=torch.float32))  # an fp32 scale, as the ABI takes
    codes = (xf / scale).clamp_(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return codes, scale


def seed_for_rank(base_seed: int, rank: int) -> int:
    """Each rank of a weak-scaling run draws its own independent sequence."""
    return int(base_seed) + 1000003 * int(rank)


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def describe(w: Workload) -> str:
    attended = (w.n_sink + w.n_local + 1) * w.chunk_size + w.top_k_groups * w.group_size
    return (f"{w.name}: B={w.batch} L={w.seq_len} Hq={w.n_q_heads} Hkv={w.n_kv_heads} "
            f"d={w.head_dim} C={w.chunk_size} G={w.groups_per_chunk} sink={w.n_sink} "
            f"local={w.n_local} kc={w.top_k_chunks} kg={w.top_k_groups} "
            f"theta={w.rope_theta:g} F={w.n_high_freq_pairs} {w.dtype} {w.mode}"
            f" attended<= {attended} ({100.0 * attended / w.seq_len:.2f}%)")


__all__ = ["Workload", "WORKLOADS", "draw", "bytes_per_step", "seed_for_rank",
           "ceil_div", "describe", "to_e4m3", "E4M3_MAX"]
