"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks the oracle against something the HGA pages or mathematics
fix: a library routine for a special case (complex multiplication for RoPE,
torch SDPA for dense causal attention, torch's bf16 cast), a closed form
(the Dirichlet-kernel mean of rotations, single-token chunks), an invariant
(relative position, linearity, forced visibility, incremental build) or
brute force on tiny inputs. Method source: "Technische Samenvatting:
Hierarchical Global Attention (HGA)" (gist.science), "Kernmechanisme" items
1-4. No GPU is used.
"""
import itertools

import numpy as np
import pytest
import torch

from oracle import hga_oracle as O


def tiny_cfg(**kw):
    base = dict(batch=1, seq_len=256, n_q_heads=4, n_kv_heads=2, head_dim=32, chunk_size=16,
                groups_per_chunk=4, n_sink=1, n_local=1, top_k_chunks=3, top_k_groups=5,
                n_high_freq_pairs=8, rope_theta=1e4)
    base.update(kw)
    return O.make_cfg(**base)


def freqs(cfg):
    h = cfg.head_dim // 2
    return cfg.rope_theta ** (-2.0 * np.arange(h) / cfg.head_dim)


def as_complex(x):
    h = x.shape[-1] // 2
    return x[..., :h] + 1j * x[..., h:]


# ---------------------------------------------------------------- RoPE ---

@pytest.mark.parametrize("d,theta", [(32, 1e4), (64, 1e4), (128, 1e6)])
def test_rope_is_complex_multiplication(d, theta):
    """Half-split RoPE equals multiplying (x_i + i x_{i+d/2}) by exp(i p theta_i)."""
    cfg = tiny_cfg(head_dim=d, rope_theta=theta)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, 3, d)).astype(np.float32)
    pos0 = 65530
    got = O.rope(cfg, x, pos0, False)
    pos = pos0 + np.arange(7)[:, None, None]
    want = as_complex(x.astype(np.float64)) * np.exp(1j * pos * freqs(cfg))
    # angles near 6.5e4 rad carry ~1e-11 of double rounding in either computation
    np.testing.assert_allclose(as_complex(got), want, rtol=0, atol=1e-9)


def test_rope_basis_vector_closed_form():
    """Pair 0 has frequency 1: R(p) e_0 = cos(p) e_0 + sin(p) e_{d/2}."""
    cfg = tiny_cfg()
    e0 = np.zeros((1, 1, 32), np.float32)
    e0[0, 0, 0] = 1
    got = O.rope(cfg, e0, 5, False)[0, 0]
    want = np.zeros(32)
    want[0], want[16] = np.cos(5.0), np.sin(5.0)
    np.testing.assert_allclose(got, want, atol=1e-15)


def test_rope_relative_position_and_norm():
    cfg = tiny_cfg(head_dim=64)
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 1, 64)).astype(np.float32)
    k = rng.standard_normal((1, 1, 64)).astype(np.float32)
    dots = []
    for shift in (0, 17, 40000):
        qr = O.rope(cfg, q, 100 + shift, False)
        kr = O.rope(cfg, k, 37 + shift, False)
        dots.append(float((qr * kr).sum()))
        np.testing.assert_allclose(np.linalg.norm(qr), np.linalg.norm(q.astype(np.float64)),
                                   rtol=1e-13)
    np.testing.assert_allclose(dots, dots[0], rtol=1e-10)


def test_round_bf16_matches_torch_cast():
    rng = np.random.default_rng(3)
    xs = np.concatenate([rng.standard_normal(4000) * 10.0 ** rng.integers(-5, 5, 4000),
                         # exact halfway cases between two bf16 values
                         np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0, -0.0])])
    xs = xs.astype(np.float32)
    want = torch.from_numpy(xs).to(torch.bfloat16).float().numpy()
    got = np.array([O.round_bf16(float(x)) for x in xs])
    np.testing.assert_array_equal(got, want.astype(np.float64))


def test_round_bf16_array_matches_scalar_and_torch_cast():
    """The array form used for bf16 summary tables: element by element the
    scalar rounding, and torch's bf16 cast for float32-exact inputs."""
    rng = np.random.default_rng(4)
    xs = (rng.standard_normal(3000) * 10.0 ** rng.integers(-4, 4, 3000)).reshape(30, 100)
    got = O.round_bf16_array(xs)
    np.testing.assert_array_equal(got.ravel(), [O.round_bf16(float(x)) for x in xs.ravel()])
    x32 = xs.astype(np.float32)
    want = torch.from_numpy(x32).to(torch.bfloat16).float().numpy().astype(np.float64)
    np.testing.assert_array_equal(O.round_bf16_array(x32), want)


def test_e4m3_every_code_matches_torch_float8_cast():
    """All 256 E4M3 codes decode to the values of torch's float8_e4m3fn type
    (NaN where torch has NaN)."""
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    got = O.e4m3_decode(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    np.testing.assert_array_equal(got[ok], want[ok])
    np.testing.assert_array_equal(np.signbit(got[ok]), np.signbit(want[ok]))


def test_e4m3_closed_forms():
    """Values fixed by the format's definition: one, the largest finite value,
    the smallest normal and subnormal, signed zero, NaN; positive codes are
    strictly increasing; the scale multiplies every value."""
    assert O.e4m3_value(0x38) == 1.0
    assert O.e4m3_value(0xB8) == -1.0
    assert O.e4m3_value(0x7E) == 448.0
    assert O.e4m3_value(0x08) == 2.0 ** -6
    assert O.e4m3_value(0x01) == 2.0 ** -9
    assert O.e4m3_value(0x07) == 7 * 2.0 ** -9
    assert O.e4m3_value(0x3C) == 1.5
    z = O.e4m3_value(0x80)
    assert z == 0.0 and np.signbit(z)
    assert np.isnan(O.e4m3_value(0x7F)) and np.isnan(O.e4m3_value(0xFF))
    pos = O.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)
    np.testing.assert_array_equal(O.e4m3_decode(np.arange(0x7F, dtype=np.uint8), 0.375),
                                  pos * 0.375)


# ----------------------------------------------------------- summaries ---

def _k(cfg, seed=4):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((cfg.batch, cfg.n_kv_heads, cfg.seq_len, cfg.head_dim)).astype(
        np.float32)


def test_single_token_chunk_summary_is_rotated_key():
    """C = 1 (one group of one token): the summary is that token's rotated key,
    whatever the frequency split."""
    for F in (0, 5, 16):
        cfg = tiny_cfg(seq_len=40, chunk_size=1, groups_per_chunk=1, n_high_freq_pairs=F)
        k = _k(cfg)
        cs, gs = O.build_summaries(cfg, k)
        for b, h in itertools.product(range(cfg.batch), range(cfg.n_kv_heads)):
            rot = O.rope(cfg, k[b, h][:, None, :], 0, False)[:, 0, :]
            np.testing.assert_allclose(cs[b, h], rot, atol=1e-12)
            np.testing.assert_allclose(gs[b, h], rot, atol=1e-12)


def _complex_summaries(cfg, k, lo, hi):
    """Reference values for one token range [lo, hi) of k[b, h]: the mean of
    rotated keys (all pairs high-frequency) and the rotation of the mean raw
    key to the mean position (all pairs low-frequency), via numpy complex."""
    w = freqs(cfg)
    pos = np.arange(lo, hi, dtype=np.float64)
    z = as_complex(k[lo:hi].astype(np.float64))
    high = (z * np.exp(1j * pos[:, None] * w)).mean(axis=0)
    low = z.mean(axis=0) * np.exp(1j * pos.mean() * w)
    return high, low


@pytest.mark.parametrize("F", [0, 16, 5])
def test_summary_frequency_split_closed_forms(F):
    """F = d/2: mean of rotated keys. F = 0: mean raw key rotated to the mean
    position. Mixed F: pairs < F as the first, pairs >= F as the second."""
    cfg = tiny_cfg(n_high_freq_pairs=F)
    k = _k(cfg)
    cs, gs = O.build_summaries(cfg, k)
    C, G = cfg.chunk_size, cfg.groups_per_chunk
    g = C // G
    for b, h in itertools.product(range(cfg.batch), range(cfg.n_kv_heads)):
        for ch in range(cfg.seq_len // C):
            for lo, hi, got in [(ch * C, ch * C + C, cs[b, h, ch])] + [
                    (ch * C + r * g, ch * C + r * g + g, gs[b, h, ch * G + r]) for r in range(G)]:
                high, low = _complex_summaries(cfg, k[b, h], lo, hi)
                want = np.where(np.arange(cfg.head_dim // 2) < F, high, low)
                np.testing.assert_allclose(as_complex(got), want, atol=1e-12)


def test_constant_key_dirichlet_closed_form():
    """n equal keys k at positions s..s+n-1: the high-frequency part equals
    D_n(theta_i) R(pbar theta_i) k with D_n(w) = sin(n w / 2) / (n sin(w / 2))
    (a geometric series), the low-frequency part R(pbar theta_i) k, with pbar
    = s + (n-1)/2."""
    cfg = tiny_cfg(seq_len=64, chunk_size=16, groups_per_chunk=4, n_high_freq_pairs=9,
                   batch=1, n_kv_heads=1)
    rng = np.random.default_rng(5)
    kv = rng.standard_normal(cfg.head_dim).astype(np.float32)
    k = np.broadcast_to(kv, (1, 1, 64, cfg.head_dim)).copy()
    cs, gs = O.build_summaries(cfg, k)
    w = freqs(cfg)
    z = as_complex(kv.astype(np.float64))
    for (n, s, got) in [(16, 32, cs[0, 0, 2]), (4, 52, gs[0, 0, 13])]:
        pbar = s + (n - 1) / 2.0
        dn = np.sin(n * w / 2) / (n * np.sin(w / 2))
        want = np.where(np.arange(len(w)) < 9, dn, 1.0) * z * np.exp(1j * pbar * w)
        np.testing.assert_allclose(as_complex(got), want, atol=1e-12)


def test_ragged_tail_summary_uses_present_tokens():
    """L not a multiple of C: the last chunk and its groups cover only the
    tokens that exist; groups with no token are zero."""
    cfg = tiny_cfg(seq_len=16 * 3 + 6, n_high_freq_pairs=6)
    k = _k(cfg)
    cs, gs = O.build_summaries(cfg, k)
    for b, h in itertools.product(range(cfg.batch), range(cfg.n_kv_heads)):
        high, low = _complex_summaries(cfg, k[b, h], 48, 54)
        want = np.where(np.arange(16) < 6, high, low)
        np.testing.assert_allclose(as_complex(cs[b, h, 3]), want, atol=1e-12)
        high, low = _complex_summaries(cfg, k[b, h], 52, 54)  # group 1 holds 2 tokens
        np.testing.assert_allclose(as_complex(gs[b, h, 13]), np.where(np.arange(16) < 6, high, low),
                                   atol=1e-12)
        assert np.all(gs[b, h, 14] == 0) and np.all(gs[b, h, 15] == 0)


def test_incremental_build_equals_one_shot():
    """Building over a growing prefix (chunk by chunk) gives bitwise the same
    summaries for every complete chunk as building once over the whole sequence."""
    cfg_full = tiny_cfg()
    k = _k(cfg_full)
    cs_full, gs_full = O.build_summaries(cfg_full, k)
    C, G = cfg_full.chunk_size, cfg_full.groups_per_chunk
    for n_ch in (1, 5, 16):
        cfg = tiny_cfg(seq_len=n_ch * C)
        cs, gs = O.build_summaries(cfg, np.ascontiguousarray(k[:, :, : n_ch * C]))
        assert np.array_equal(cs, cs_full[:, :, :n_ch])
        assert np.array_equal(gs, gs_full[:, :, : n_ch * G])


def test_summaries_are_linear_in_keys():
    cfg = tiny_cfg()
    k1, k2 = _k(cfg, 6), _k(cfg, 7)
    a, b = 0.75, -2.5
    cs1, gs1 = O.build_summaries(cfg, k1)
    cs2, gs2 = O.build_summaries(cfg, k2)
    mix = (a * k1.astype(np.float64) + b * k2).astype(np.float32)
    # the float32 rounding of the mix is carried through the linear map
    cs3, gs3 = O.build_summaries(cfg, mix)
    np.testing.assert_allclose(cs3, a * cs1 + b * cs2, atol=1e-5)
    np.testing.assert_allclose(gs3, a * gs1 + b * gs2, atol=1e-5)


# ------------------------------------------------------------- routing ---

def test_qbar_score_is_mean_of_per_query_scores():
    cfg = tiny_cfg(seq_len=64, n_q_heads=6, n_kv_heads=2)
    rng = np.random.default_rng(8)
    q = rng.standard_normal((1, 64, 6, 32)).astype(np.float32)
    s = rng.standard_normal(32)
    qb = O.qbar(cfg, q)
    for h in range(2):
        for j in range(4):
            per_q = q[0, j * 16:(j + 1) * 16, 3 * h:3 * h + 3].astype(np.float64) @ s
            np.testing.assert_allclose(qb[0, h, j] @ s, per_q.mean(), rtol=1e-12)


def test_qbar_decode_and_ragged_span():
    """A single query token: the mean over its KV head's query heads. A span
    starting inside a chunk covers only its own tokens."""
    rng = np.random.default_rng(9)
    cfg = tiny_cfg(seq_len=200, n_q_heads=8, n_kv_heads=2, q_begin=199, q_len=1)
    q = rng.standard_normal((1, 1, 8, 32)).astype(np.float32)
    qb = O.qbar(cfg, q)
    assert qb.shape == (1, 2, 1, 32)
    np.testing.assert_allclose(qb[0, 1, 0], q[0, 0, 4:8].astype(np.float64).mean(0), atol=1e-15)
    cfg = tiny_cfg(seq_len=200, n_q_heads=8, n_kv_heads=2, q_begin=150, q_len=50)
    q = rng.standard_normal((1, 50, 8, 32)).astype(np.float32)
    qb = O.qbar(cfg, q)
    assert qb.shape == (1, 2, 4, 32)  # chunks 9..12
    np.testing.assert_allclose(qb[0, 0, 0], q[0, :10, 0:4].astype(np.float64).mean((0, 1)),
                               atol=1e-14)
    np.testing.assert_allclose(qb[0, 1, 3], q[0, 42:, 4:8].astype(np.float64).mean((0, 1)),
                               atol=1e-14)


def forced_set(j, n_sink, n_local):
    """Always-visible chunks of query chunk j, from the page's wording: the
    current chunk, the first n_sink chunks and the n_local previous chunks."""
    return {j} | {c for c in range(n_sink) if c <= j} | {c for c in range(j - n_local, j) if c >= 0}


def brute_route(qb, chunk_sum, group_sum, j, n_sink, n_local, kc, kg, G):
    cands = [c for c in range(j) if c not in forced_set(j, n_sink, n_local)]
    sc = {c: np.float32(np.dot(qb, chunk_sum[c])) for c in cands}
    order = sorted(cands, key=lambda c: (-float(sc[c]), c))
    chunks = sorted(order[:kc])
    gc = [c * G + r for c in chunks for r in range(G)]
    gsc = {gi: np.float32(np.dot(qb, group_sum[gi])) for gi in gc}
    gorder = sorted(gc, key=lambda gi: (-float(gsc[gi]), gi))
    return chunks, sorted(gorder[:kg])


@pytest.mark.parametrize("n_sink,n_local,kc,kg", [(1, 1, 3, 5), (2, 3, 1, 4), (0, 0, 20, 80),
                                                    (1, 2, 4, 1)])
def test_routing_brute_force(n_sink, n_local, kc, kg):
    cfg = tiny_cfg(n_sink=n_sink, n_local=n_local, top_k_chunks=kc, top_k_groups=kg,
                   batch=2, seq_len=16 * 13 + 5)
    rng = np.random.default_rng(10)
    k = _k(cfg, 11)
    q = rng.standard_normal((2, cfg.seq_len, 4, 32)).astype(np.float32)
    cs, gs = O.build_summaries(cfg, k)
    qb = O.qbar(cfg, q)
    sel, nsel, scs = O.route_chunks(cfg, qb, cs)
    gsel, gnsel, gscs = O.route_groups(cfg, qb, gs, sel, nsel)
    for b, h, j in itertools.product(range(2), range(2), range(qb.shape[2])):
        ch, gr = brute_route(qb[b, h, j], cs[b, h], gs[b, h], j, n_sink, n_local, kc, kg, 4)
        assert list(sel[b, h, j, :nsel[b, h, j]]) == ch
        assert np.all(sel[b, h, j, nsel[b, h, j]:] == -1)
        assert list(gsel[b, h, j, :gnsel[b, h, j]]) == gr
        assert np.all(gsel[b, h, j, gnsel[b, h, j]:] == -1)
        # the score table marks exactly the candidates
        cand = [c for c in range(j) if c not in forced_set(j, n_sink, n_local)]
        assert set(np.flatnonzero(~np.isnan(scs[b, h, j]))) == set(cand)


def test_forced_visibility_and_clamping():
    """Forced chunks are never routed (they are always visible), only earlier
    chunks are routed, and k is clamped to the candidates available."""
    cfg = tiny_cfg(n_sink=2, n_local=3, top_k_chunks=6, top_k_groups=30, seq_len=16 * 16)
    k = _k(cfg)
    rng = np.random.default_rng(12)
    q = rng.standard_normal((1, 256, 4, 32)).astype(np.float32)
    cs, gs = O.build_summaries(cfg, k)
    qb = O.qbar(cfg, q)
    sel, nsel, _ = O.route_chunks(cfg, qb, cs)
    for h, j in itertools.product(range(2), range(16)):
        n_cand = j - len(forced_set(j, 2, 3) - {j})
        assert nsel[0, h, j] == min(6, max(n_cand, 0))
        chosen = sel[0, h, j, :nsel[0, h, j]]
        assert all(c < j and c not in forced_set(j, 2, 3) for c in chosen)
        assert list(chosen) == sorted(set(chosen))
        for c in range(j + 1):
            assert O.is_forced(cfg, j, c) == (c in forced_set(j, 2, 3))


def test_ties_prefer_lower_index_and_nan_ranks_last():
    cfg = tiny_cfg(batch=1, n_kv_heads=1, n_q_heads=1, seq_len=16 * 8, n_sink=0, n_local=0,
                   top_k_chunks=3)
    qb = np.zeros((1, 1, 8, 32))
    qb[..., 0] = 1.0
    cs = np.zeros((1, 1, 8, 32))
    cs[0, 0, :, 0] = [5.0, 7.0, 7.0, np.nan, 7.0, -0.0, 7.0, 1.0]
    sel, nsel, _ = O.route_chunks(cfg, qb, cs)
    assert list(sel[0, 0, 7]) == [1, 2, 4]   # four 7.0 ties: lowest indices
    assert list(sel[0, 0, 4]) == [0, 1, 2]
    cs[0, 0, :, 0] = [np.nan, np.nan, 0.0, -0.0, -1.0, 0, 0, 0]
    sel, nsel, _ = O.route_chunks(cfg, qb, cs)
    assert list(sel[0, 0, 5]) == [2, 3, 4]   # +0 and -0 tie; NaNs last


# ----------------------------------------------------------- attention ---

def _dense_sdpa(q, k, v):
    """Dense causal GQA attention by torch SDPA in float64 (library routine)."""
    B, L, Hq, d = q.shape
    Hkv = k.shape[1]
    qt = torch.from_numpy(q.astype(np.float64)).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k.astype(np.float64)).repeat_interleave(Hq // Hkv, dim=1)
    vt = torch.from_numpy(v.astype(np.float64)).repeat_interleave(Hq // Hkv, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("seq_len", [16 * 12, 16 * 12 + 7])
def test_routing_everything_equals_dense_causal(seq_len):
    """When top-k takes every chunk and every group, routed attention is dense
    causal attention ("Exact-Token Attention" with nothing left out)."""
    cfg = tiny_cfg(batch=2, seq_len=seq_len, top_k_chunks=64, top_k_groups=256)
    rng = np.random.default_rng(13)
    q = rng.standard_normal((2, seq_len, 4, 32)).astype(np.float32)
    k = _k(cfg, 14)
    v = rng.standard_normal(k.shape).astype(np.float32)
    cs, gs = O.build_summaries(cfg, k)
    qb = O.qbar(cfg, q)
    sel, nsel, _ = O.route_chunks(cfg, qb, cs)
    gsel, gnsel, _ = O.route_groups(cfg, qb, gs, sel, nsel)
    out = O.attend(cfg, q, k, v, gsel, gnsel)
    np.testing.assert_allclose(out, _dense_sdpa(q, k, v), atol=1e-12)


def test_all_chunks_forced_equals_dense_causal():
    cfg = tiny_cfg(seq_len=160, n_local=100, top_k_chunks=1, top_k_groups=1)
    rng = np.random.default_rng(15)
    q = rng.standard_normal((1, 160, 4, 32)).astype(np.float32)
    k = _k(cfg)
    v = rng.standard_normal(k.shape).astype(np.float32)
    qb = O.qbar(cfg, q)
    cs, gs = O.build_summaries(cfg, k)
    sel, nsel, _ = O.route_chunks(cfg, qb, cs)
    assert np.all(nsel == 0)
    gsel, gnsel, _ = O.route_groups(cfg, qb, gs, sel, nsel)
    out = O.attend(cfg, q, k, v, gsel, gnsel)
    np.testing.assert_allclose(out, _dense_sdpa(q, k, v), atol=1e-12)


def brute_attend_row(q, k, v, keys):
    s = np.array([np.dot(q, k[p]) for p in keys]) / np.sqrt(len(q))
    p = np.exp(s - s.max())
    return (p[:, None] * v[keys]).sum(0) / p.sum()


def test_attention_brute_force_on_routed_set():
    """Random valid selections: each output row equals softmax over exactly
    the forced-chunk keys (causal) and the selected groups' keys."""
    cfg = tiny_cfg(batch=1, seq_len=16 * 10 + 3, n_sink=1, n_local=1, top_k_chunks=2,
                   top_k_groups=3)
    rng = np.random.default_rng(16)
    L = cfg.seq_len
    q = rng.standard_normal((1, L, 4, 32)).astype(np.float32)
    k = _k(cfg)
    v = rng.standard_normal(k.shape).astype(np.float32)
    nQC = O.n_qchunks(cfg)
    gsel = np.full((1, 2, nQC, 3), -1, np.int32)
    gnsel = np.zeros((1, 2, nQC), np.int32)
    for h, j in itertools.product(range(2), range(nQC)):
        cand = [c * 4 + r for c in range(j) if c not in forced_set(j, 1, 1) for r in range(4)]
        pick = sorted(rng.choice(cand, size=min(3, len(cand)), replace=False)) if cand else []
        gsel[0, h, j, :len(pick)] = pick
        gnsel[0, h, j] = len(pick)
    out = O.attend(cfg, q, k, v, gsel, gnsel)
    for h, j in itertools.product(range(2), range(nQC)):
        visible = set()
        for c in forced_set(j, 1, 1):
            visible |= set(range(c * 16, min(c * 16 + 16, L)))
        for gi in gsel[0, h, j, :gnsel[0, h, j]]:
            visible |= set(range(gi * 4, gi * 4 + 4))
        for t in range(j * 16, min(j * 16 + 16, L)):
            keys = sorted(p for p in visible if p <= t)
            for hq in (2 * h, 2 * h + 1):
                want = brute_attend_row(q[0, t, hq].astype(np.float64), k[0, h].astype(np.float64),
                                        v[0, h].astype(np.float64), keys)
                np.testing.assert_allclose(out[0, t, hq], want, atol=1e-12)


def test_first_token_sees_only_itself_and_units_subset():
    cfg = tiny_cfg(batch=2, seq_len=96)
    rng = np.random.default_rng(17)
    q = rng.standard_normal((2, 96, 4, 32)).astype(np.float32)
    k = _k(cfg)
    v = rng.standard_normal(k.shape).astype(np.float32)
    cs, gs = O.build_summaries(cfg, k)
    qb = O.qbar(cfg, q)
    sel, nsel, _ = O.route_chunks(cfg, qb, cs)
    gsel, gnsel, _ = O.route_groups(cfg, qb, gs, sel, nsel)
    full = O.attend(cfg, q, k, v, gsel, gnsel)
    for b in range(2):
        for hq in range(4):
            np.testing.assert_array_equal(full[b, 0, hq], v[b, hq // 2, 0].astype(np.float64))
    units = np.array([[1, 0, 3], [0, 1, 5]])
    part = O.attend(cfg, q, k, v, gsel, gnsel, units=units)
    np.testing.assert_array_equal(part[1, 48:64, 0:2], full[1, 48:64, 0:2])
    np.testing.assert_array_equal(part[0, 80:96, 2:4], full[0, 80:96, 2:4])
    assert np.isnan(part[0, 0]).all()


def test_decode_query_at_last_position():
    """q_begin = L-1, q_len = 1: the current chunk is fully visible and the
    result equals the last row of the full prefill with the same routing."""
    cfg_p = tiny_cfg(seq_len=128, top_k_chunks=64, top_k_groups=256)
    cfg_d = tiny_cfg(seq_len=128, top_k_chunks=64, top_k_groups=256, q_begin=127, q_len=1)
    rng = np.random.default_rng(18)
    q = rng.standard_normal((1, 128, 4, 32)).astype(np.float32)
    k = _k(cfg_p)
    v = rng.standard_normal(k.shape).astype(np.float32)
    cs, gs = O.build_summaries(cfg_d, k)
    qd = np.ascontiguousarray(q[:, 127:])
    qb = O.qbar(cfg_d, qd)
    sel, nsel, _ = O.route_chunks(cfg_d, qb, cs)
    gsel, gnsel, _ = O.route_groups(cfg_d, qb, gs, sel, nsel)
    out = O.attend(cfg_d, qd, k, v, gsel, gnsel)
    np.testing.assert_allclose(out[0, 0], _dense_sdpa(q, k, v)[0, 127], atol=1e-12)


# ------------------------------------------------- per-query-head routing ---

def _per_head_case(equal_heads: bool):
    from long_context_rope_b200 import synth
    w = synth.WORKLOADS["prefill_4k"].replace(name="perhead", seq_len=2048, n_q_heads=8,
                                              n_kv_heads=2, top_k_chunks=2, top_k_groups=5)
    x = synth.draw(w, seed=21)
    if equal_heads:  # every query head of a KV head carries the same query
        q = x["q_raw"].clone()
        gq = w.n_q_heads // w.n_kv_heads
        for h in range(w.n_q_heads):
            q[:, :, h] = x["q_raw"][:, :, (h // gq) * gq]
        x = dict(x, q_raw=q)
    return w, x


def test_per_q_head_routing_reduces_to_shared_routing():
    """With the query heads of each KV head all equal, each head's own routing
    query is the shared q-bar, so per-query-head routing selects exactly the
    shared selections (per query head) and attends to the same keys."""
    w, x = _per_head_case(equal_heads=True)
    gq = w.n_q_heads // w.n_kv_heads
    r = O.pipeline(w, x)
    rh = O.pipeline(*O.per_q_head(w, x))
    for h in range(w.n_q_heads):
        for key in ("sel_chunks", "n_sel_chunks", "sel_groups", "n_sel_groups"):
            np.testing.assert_array_equal(rh[key][:, h], r[key][:, h // gq], err_msg=key)
        np.testing.assert_allclose(rh["qbar"][:, h], r["qbar"][:, h // gq], rtol=1e-12,
                                   atol=1e-12)
    np.testing.assert_allclose(rh["out"], r["out"], rtol=0, atol=1e-12)


def test_per_q_head_qbar_is_the_heads_own_mean():
    """Distinct query heads: head h's routing query is the mean of its own
    rotated queries over the chunk's tokens, and its summaries are its KV
    head's."""
    w, x = _per_head_case(equal_heads=False)
    gq = w.n_q_heads // w.n_kv_heads
    r = O.pipeline(w, x)
    rh = O.pipeline(*O.per_q_head(w, x))
    C = w.chunk_size
    q_rot = rh["q_rot"].astype(np.float64)
    for j in range(w.seq_len // C):
        want = q_rot[:, j * C:(j + 1) * C].mean(axis=1)  # [B, Hq, d]
        np.testing.assert_allclose(rh["qbar"][:, :, j], want, rtol=1e-12, atol=1e-12)
    for h in range(w.n_q_heads):
        np.testing.assert_array_equal(rh["chunk_sum"][:, h], r["chunk_sum"][:, h // gq])
    # distinct queries do route differently somewhere
    assert any(not np.array_equal(rh["sel_groups"][:, h], r["sel_groups"][:, h // gq])
               for h in range(w.n_q_heads))
