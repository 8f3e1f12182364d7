"""GPU: routing that keeps everything is dense causal attention.

"Technische Samenvatting: Hierarchical Global Attention (HGA)", "Kernmechanisme"
items 2 and 4: when top_k_chunks and top_k_groups cover every candidate,
the routed set of a query chunk is every earlier chunk plus the forced ones,
and exact attention over it is plain causal softmax attention. This checks
the CUDA path against torch's dense causal attention (fp32, on the GPU's own
rotated bf16 inputs), independently of the oracle:
  * every selection list is exactly the ascending list of all non-forced
    earlier chunks, and of all their groups;
  * every output is within the bf16 output tolerance (2e-2) of dense
    attention.
Prefill runs at the largest key set a unit may hold (512 blocks of 16 keys:
the forced 16 plus 496 routed groups), through the tiled chunk routing, the
large-candidate group routing and the tcgen05 attention; decode at the
largest top_k_chunks of the one-launch step (64), both as one launch and as
separate calls.
"""
import pytest
import torch

from long_context_rope_b200 import synth

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-2


def _forced(w, j):
    s_end = min(w.n_sink, j + 1)
    return set(range(s_end)) | set(range(max(s_end, j - w.n_local), j + 1))


def _expected_selection(w, j):
    chunks = [c for c in range(j) if c not in _forced(w, j)]
    groups = [c * w.groups_per_chunk + g for c in chunks for g in range(w.groups_per_chunk)]
    return chunks, groups


def _dense(q_rot, k_rot, v, q_begin):
    """Causal softmax attention in fp32: q [B, Lq, Hq, d] at positions
    q_begin.., k/v [B, Hkv, L, d]; every query head attends its KV head."""
    B, Lq, Hq, d = q_rot.shape
    Hkv, L = k_rot.shape[1], k_rot.shape[2]
    gq = Hq // Hkv
    q = q_rot.float().permute(0, 2, 1, 3)                      # [B, Hq, Lq, d]
    k = k_rot.float().repeat_interleave(gq, dim=1)             # [B, Hq, L, d]
    vv = v.float().repeat_interleave(gq, dim=1)
    pos_q = torch.arange(q_begin, q_begin + Lq, device=q.device)
    mask = torch.arange(L, device=q.device)[None, :] <= pos_q[:, None]  # [Lq, L]
    o = torch.nn.functional.scaled_dot_product_attention(q, k, vv, attn_mask=mask)
    return o.permute(0, 2, 1, 3)                               # [B, Lq, Hq, d]


def _check_lists(w, rb, j_of):
    sc, nc = rb.sel_chunks.cpu().numpy(), rb.n_sel_chunks.cpu().numpy()
    sg, ng = rb.sel_groups.cpu().numpy(), rb.n_sel_groups.cpu().numpy()
    for b in range(sc.shape[0]):
        for h in range(sc.shape[1]):
            for jj in range(sc.shape[2]):
                chunks, groups = _expected_selection(w, j_of(jj))
                assert nc[b, h, jj] == len(chunks) and list(sc[b, h, jj, :nc[b, h, jj]]) == chunks
                assert (sc[b, h, jj, nc[b, h, jj]:] == -1).all()
                assert ng[b, h, jj] == len(groups) and list(sg[b, h, jj, :ng[b, h, jj]]) == groups
                assert (sg[b, h, jj, ng[b, h, jj]:] == -1).all()


def test_prefill_route_everything_is_dense_causal():
    from long_context_rope_b200 import hga, pipeline
    # 128 chunks: the last query chunk has 124 routable chunks (496 groups)
    # beside its 4 forced ones, so it holds 512 key blocks
    w = synth.WORKLOADS["prefill_4k"].replace(name="dense_prefill", seq_len=8192,
                                              top_k_chunks=128, top_k_groups=496)
    cfg = hga.config_from(w)
    x = synth.draw(w, seed=11)
    k_raw, v = x["k_raw"].cuda(), x["v"].cuda()
    q_rot = pipeline.rotate_queries(cfg, x["q_raw"].cuda())
    cs, gs = pipeline.alloc_summaries(cfg)
    k_rot = torch.empty_like(k_raw)
    rb = pipeline.alloc_route(cfg)
    out = torch.full_like(q_rot, float("nan"))
    pipeline.prefill(cfg, k_raw, v, q_rot, cs, gs, k_rot, rb, out)
    torch.cuda.synchronize()
    assert hga.get_device_error() == 0
    _check_lists(w, rb, lambda jj: jj)
    ref = _dense(q_rot, k_rot, v, 0)
    err = (out.float() - ref).abs().max().item()
    print(f"prefill, every chunk and group routed: max abs error vs dense {err:.3e}")
    assert err <= OUT_TOL


@pytest.mark.parametrize("separate", [False, True])
def test_decode_route_everything_is_dense(separate):
    from long_context_rope_b200 import hga, pipeline
    # 64 chunks: the query chunk (63) has 60 routable chunks beside its 4 forced
    # ones (sink 0, locals 61 and 62, itself)
    w = synth.WORKLOADS["decode_16x32k"].replace(name="dense_decode", batch=3, seq_len=4096,
                                                 top_k_chunks=64, top_k_groups=60 * 4)
    cfg = hga.config_from(w)
    x = synth.draw(w, seed=12)
    k_raw, v = x["k_raw"].cuda(), x["v"].cuda()
    cs, gs = pipeline.alloc_summaries(cfg)
    k_rot = torch.empty_like(k_raw)
    pipeline.summaries(cfg, k_raw, cs, gs, k_rot)
    q_rot = pipeline.rotate_queries(cfg, x["q_raw"].cuda())
    rb = pipeline.alloc_route(cfg)
    out = torch.full_like(q_rot, float("nan"))
    pipeline.decode(cfg, q_rot, cs, gs, k_rot, v, rb, out, separate=separate)
    torch.cuda.synchronize()
    assert hga.get_device_error() == 0
    j = (w.seq_len - 1) // w.chunk_size
    _check_lists(w, rb, lambda jj: j)
    ref = _dense(q_rot, k_rot, v, w.seq_len - 1)
    err = (out.float() - ref).abs().max().item()
    print(f"decode ({'separate calls' if separate else 'one launch'}), everything routed: "
          f"max abs error vs dense {err:.3e}")
    assert err <= OUT_TOL
