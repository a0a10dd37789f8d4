"""Pins of the fp64 oracle to facts other than itself: closed forms, limits, invariants, the
OCP format tables, library routines (torch) on special cases and brute force on tiny inputs.

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a wrong sign or
index, swapped halves, a transposed operand, a wrong tie rule) fails at least one of them.
CPU only.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def randn(*s):
    return RNG.standard_normal(s)


# ---------------------------------------------------------------------------------------------
# CSA compression (V4 paper notes Sec. 2.3, Eq. 11-12 and the Compressor listing)
# ---------------------------------------------------------------------------------------------

def _csa_inputs(T=24, c=5, m=4):
    return randn(T, c), randn(T, c), randn(T, c), randn(T, c), 0.3 * randn(2 * m, c)


def test_csa_weights_sum_to_one():
    Ca, Cb, Za, Zb, B = _csa_inputs()
    out = O.csa_compress(np.ones_like(Ca), np.ones_like(Cb), Za, Zb, B, 4)
    assert out.shape == (6, 5)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-14)


def test_csa_uniform_logits_give_block_means():
    T, c, m = 24, 5, 4
    Ca, Cb, _, _, _ = _csa_inputs(T, c, m)
    Z = np.full((T, c), 0.7)
    out = O.csa_compress(Ca, Cb, Z, Z, np.zeros((2 * m, c)), m)
    # entry 0: its own 4 tokens of C^a; entry i: C^a of block i and C^b of block i-1
    np.testing.assert_allclose(out[0], Ca[0:4].mean(0), rtol=1e-13)
    for i in range(1, T // m):
        ref = np.concatenate([Ca[i * m:(i + 1) * m], Cb[(i - 1) * m:i * m]]).mean(0)
        np.testing.assert_allclose(out[i], ref, rtol=1e-13)


@pytest.mark.parametrize("j", [0, 3])
def test_csa_dominant_logit_selects_token(j):
    T, c, m, i = 24, 5, 4, 3
    Ca, Cb, Za, Zb, B = _csa_inputs(T, c, m)
    Za2 = Za.copy()
    Za2[i * m + j] += 80.0
    np.testing.assert_allclose(O.csa_compress(Ca, Cb, Za2, Zb, B, m)[i], Ca[i * m + j], rtol=1e-12)
    Zb2 = Zb.copy()
    Zb2[(i - 1) * m + j] += 80.0
    np.testing.assert_allclose(O.csa_compress(Ca, Cb, Za, Zb2, B, m)[i], Cb[(i - 1) * m + j], rtol=1e-12)


@pytest.mark.parametrize("j", [1, 2])
def test_csa_bias_rows_layout(j):
    """Rows 0..m-1 of B bias the current block (B^a), rows m..2m-1 the previous block (B^b)."""
    T, c, m, i = 24, 5, 4, 2
    Ca, Cb, Za, Zb, _ = _csa_inputs(T, c, m)
    B = np.zeros((2 * m, c))
    B[j] = 80.0
    np.testing.assert_allclose(O.csa_compress(Ca, Cb, Za, Zb, B, m)[i], Ca[i * m + j], rtol=1e-12)
    B = np.zeros((2 * m, c))
    B[m + j] = 80.0
    np.testing.assert_allclose(O.csa_compress(Ca, Cb, Za, Zb, B, m)[i], Cb[(i - 1) * m + j], rtol=1e-12)
    # entry 0 has no previous block: B^b cannot select anything there
    np.testing.assert_allclose(O.csa_compress(Ca, Cb, Za, Zb, B, m)[0],
                               O.csa_compress(Ca, Cb, Za, Zb, np.zeros((2 * m, c)), m)[0], rtol=1e-14)


def test_csa_entry0_and_causality():
    T, c, m = 24, 5, 4
    Ca, Cb, Za, Zb, B = _csa_inputs(T, c, m)
    base = O.csa_compress(Ca, Cb, Za, Zb, B, m)
    # the C^b/Z^b rows of block 0 feed entry 1 only; entry 0 never reads C^b / Z^b
    Cb2, Zb2 = Cb.copy(), Zb.copy()
    Cb2[0:4] += 5.0
    Zb2[0:4] -= 3.0
    out = O.csa_compress(Ca, Cb2, Za, Zb2, B, m)
    assert np.array_equal(out[0], base[0])
    assert not np.allclose(out[1], base[1])
    assert np.array_equal(out[2:], base[2:])
    # tokens of blocks > i never influence entries <= i
    for i in range(T // m):
        Ca3, Za3 = Ca.copy(), Za.copy()
        Ca3[(i + 1) * m:] = 99.0
        Za3[(i + 1) * m:] = -7.0
        assert np.array_equal(O.csa_compress(Ca3, Cb, Za3, Zb, B, m)[:i + 1], base[:i + 1])


def test_csa_partial_tail_not_emitted():
    Ca, Cb, Za, Zb, B = _csa_inputs(T=10, c=3, m=4)
    out = O.csa_compress(Ca, Cb, Za, Zb, B, 4)
    assert out.shape == (2, 3)
    Ca[8:] = 1e3
    assert np.array_equal(O.csa_compress(Ca, Cb, Za, Zb, B, 4), out)


def test_csa_logit_shift_invariance():
    Ca, Cb, Za, Zb, B = _csa_inputs()
    shift = randn(1, 5) * 10
    a = O.csa_compress(Ca, Cb, Za, Zb, B, 4)
    b = O.csa_compress(Ca, Cb, Za + shift, Zb + shift, B, 4)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


def test_csa_brute_force_tiny():
    T, c, m = 12, 3, 4
    Ca, Cb, Za, Zb, B = _csa_inputs(T, c, m)
    out = O.csa_compress(Ca, Cb, Za, Zb, B, m)
    for i in range(T // m):
        for d in range(c):
            cands = [(Ca[i * m + j, d], Za[i * m + j, d] + B[j, d]) for j in range(m)]
            if i > 0:
                cands += [(Cb[(i - 1) * m + j, d], Zb[(i - 1) * m + j, d] + B[m + j, d]) for j in range(m)]
            ws = [math.exp(z) for _, z in cands]
            ref = sum(wt * v for wt, (v, _) in zip(ws, cands)) / sum(ws)
            assert abs(out[i, d] - ref) <= 1e-13 * max(1.0, abs(ref))


# ---------------------------------------------------------------------------------------------
# HCA compression (V4 paper notes Sec. 2.4, Eq. 22-23)
# ---------------------------------------------------------------------------------------------

def test_hca_ratio_one_is_identity():
    C, Z = randn(17, 6), randn(17, 6)
    out = O.hca_compress(C, Z, randn(1, 6), 1)
    assert np.array_equal(out, C)


def test_hca_sum_mean_and_select():
    T, c, m = 40, 4, 8
    C, Z, B = randn(T, c), randn(T, c), 0.2 * randn(m, c)
    np.testing.assert_allclose(O.hca_compress(np.ones_like(C), Z, B, m), 1.0, atol=1e-14)
    Zc = np.full((T, c), -2.0)
    out = O.hca_compress(C, Zc, np.zeros((m, c)), m)
    assert out.shape == (5, c)
    for i in range(5):
        np.testing.assert_allclose(out[i], C[i * m:(i + 1) * m].mean(0), rtol=1e-13)
    B2 = np.zeros((m, c))
    B2[5] = 90.0
    np.testing.assert_allclose(O.hca_compress(C, Z, B2, m), C[5::m][:5], rtol=1e-12)


def test_hca_brute_force_tiny():
    T, c, m = 11, 2, 3
    C, Z, B = randn(T, c), randn(T, c), randn(m, c)
    out = O.hca_compress(C, Z, B, m)
    assert out.shape == (3, 2)
    for i in range(3):
        for d in range(c):
            ws = [math.exp(Z[i * m + j, d] + B[j, d]) for j in range(m)]
            ref = sum(wt * C[i * m + j, d] for j, wt in enumerate(ws)) / sum(ws)
            assert abs(out[i, d] - ref) <= 1e-13 * max(1, abs(ref))


@pytest.mark.parametrize("line", [l for l in open(os.path.join(GOLD, "entry_counts.txt"))
                                  if l.strip() and not l.startswith("#")])
def test_entry_counts_golden(line):
    T, m, n = map(int, line.split())
    assert T // m == n
    if T <= 4096:
        C = np.zeros((T, 1))
        assert O.hca_compress(C, C, np.zeros((m, 1)), m).shape[0] == n
        if m == 4:
            assert O.csa_compress(C, C, C, C, np.zeros((8, 1)), 4).shape[0] == n
    # the last query (t = T-1) sees exactly floor(T/m) entries
    assert int(O.n_vis(T - 1, m)) == n


# ---------------------------------------------------------------------------------------------
# Lightning indexer (Eq. 16) and top-k
# ---------------------------------------------------------------------------------------------

def test_indexer_single_head_is_relu_dot():
    q, K = randn(6, 1, 8), randn(10, 8)
    S = O.indexer_scores(q, np.ones((6, 1)), K, np.full(6, 10))
    np.testing.assert_allclose(S, np.maximum(0.0, q[:, 0, :] @ K.T), rtol=1e-13, atol=1e-14)


def test_indexer_weight_outside_relu_and_linear():
    q, K = randn(5, 3, 8), randn(9, 8)
    w1, w2 = RNG.random((5, 3)), RNG.random((5, 3))
    nv = np.full(5, 9)
    S1, S2 = O.indexer_scores(q, w1, K, nv), O.indexer_scores(q, w2, K, nv)
    np.testing.assert_allclose(O.indexer_scores(q, w1 + w2, K, nv), S1 + S2, rtol=1e-12, atol=1e-13)
    # w * ReLU(dot), not ReLU(w * dot): a negative weight gives a negative score
    Sneg = O.indexer_scores(q[:, :1], -np.ones((5, 1)), K, nv)
    np.testing.assert_allclose(Sneg, -np.maximum(0.0, q[:, 0] @ K.T), rtol=1e-13, atol=1e-14)
    # ReLU(x) - ReLU(-x) = x: scores of q and -q differ by the plain dot product
    Sp = O.indexer_scores(q[:, :1], np.ones((5, 1)), K, nv)
    Sm = O.indexer_scores(-q[:, :1], np.ones((5, 1)), K, nv)
    np.testing.assert_allclose(Sp - Sm, q[:, 0] @ K.T, rtol=1e-12, atol=1e-13)


def test_indexer_heads_add_up_and_key_base_shifts():
    """Eq. 16 sums over index heads: the H-head score is the sum of the H single-head scores
    (each pinned to ReLU(q k) above), and reading keys from row kbase[r] on is the same as
    passing the keys from that row on."""
    Nq, H, d = 6, 4, 8
    q, K, w = randn(Nq, H, d), randn(30, d), randn(Nq, H)
    nv = np.array([0, 1, 5, 9, 12, 17])
    kb = np.array([3, 0, 7, 2, 11, 13])
    S = O.indexer_scores(q, w, K, nv, kb)
    for r in range(Nq):
        parts = [O.indexer_scores(q[r:r + 1, h:h + 1], w[r:r + 1, h:h + 1], K[kb[r]:], nv[r:r + 1])
                 for h in range(H)]
        ref = sum(p[0, :nv[r]] for p in parts) if nv[r] else np.zeros(0)
        np.testing.assert_allclose(S[r, :nv[r]], ref, rtol=1e-12, atol=1e-13)
        assert np.all(np.isneginf(S[r, nv[r]:]))


def test_indexer_visibility_rule():
    m = 4
    t = np.arange(20)
    nv = O.n_vis(t, m)
    assert list(nv[:9]) == [0, 0, 0, 1, 1, 1, 1, 2, 2]
    q, K = randn(20, 2, 4), randn(5, 4)
    idx, S = O.indexer_topk(q, RNG.random((20, 2)), K, t, m, 3)
    for r in range(20):
        assert np.all(np.isfinite(S[r, :nv[r]]))
        assert np.all(np.isneginf(S[r, nv[r]:]))
        assert np.all(idx[r] < max(nv[r], 1)) and (idx[r] >= 0).sum() == min(3, nv[r])


def test_topk_matches_full_sort_with_ties():
    S = np.round(randn(30, 50), 1)  # many exact ties
    nv = RNG.integers(0, 51, size=30)
    S[np.arange(50)[None, :] >= nv[:, None]] = -np.inf
    k = 12
    idx = O.topk(S, nv, k)
    for r in range(30):
        order = sorted(range(nv[r]), key=lambda s: (-S[r, s], s))[:k]
        ref = order + [-1] * (k - len(order))
        assert list(idx[r]) == ref


def test_topk_values_match_torch_topk():
    S = randn(8, 300)
    idx = O.topk(S, np.full(8, 300), 40)
    tv = torch.topk(torch.from_numpy(S), 40, dim=1).values.numpy()
    np.testing.assert_array_equal(np.take_along_axis(S, idx.astype(np.int64), 1), tv)


def test_topk_all_equal_scores_gives_first_indices():
    q = np.zeros((3, 2, 4))
    idx, _ = O.indexer_topk(q, np.ones((3, 2)), randn(40, 4), np.array([39, 11, 2]), 1, 16)
    assert list(idx[0]) == list(range(16))
    assert list(idx[1]) == list(range(12)) + [-1] * 4
    assert list(idx[2]) == [0, 1, 2] + [-1] * 13


# ---------------------------------------------------------------------------------------------
# Hybrid attention (V4 paper notes Sec. 2.3-2.4; Q&A essay Question 1 mechanisms 1 and 3)
# ---------------------------------------------------------------------------------------------

def _dense_causal(q, K, scale, extra_logit=None):
    """Library reference: torch fp64 attention with K = V (optionally one extra value-less logit)."""
    qt = torch.from_numpy(q).permute(1, 0, 2)  # [H,T,c]
    Kt = torch.from_numpy(K)
    if extra_logit is None:
        o = torch.nn.functional.scaled_dot_product_attention(
            qt[None], Kt[None, None].expand(1, qt.shape[0], -1, -1),
            Kt[None, None].expand(1, qt.shape[0], -1, -1), is_causal=True, scale=scale)[0]
        return o.permute(1, 0, 2).numpy()
    T = K.shape[0]
    z = scale * torch.einsum("htc,sc->hts", qt, Kt)
    z = z.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), -torch.inf)
    ex = torch.from_numpy(np.asarray(extra_logit))[:, None, None].expand(-1, T, 1)
    p = torch.softmax(torch.cat([z, ex], dim=-1), dim=-1)[..., :T]
    return torch.einsum("hts,sc->htc", p, Kt).permute(1, 0, 2).numpy()


def test_attention_dense_limit_no_sink():
    """m=1 (identity compression), all entries visible, W=T, sink=-inf: every key appears twice
    (window and compressed), which cancels, leaving dense causal attention with K=V."""
    T, H, c = 19, 3, 8
    X, q = randn(T, c), randn(T, H, c)
    KVc = O.hca_compress(X, randn(T, c), randn(1, c), 1)
    o, _ = O.hybrid_attn_prefill(q, X, KVc, np.full(H, -np.inf), 0.37, m=1, W=T)
    np.testing.assert_allclose(o, _dense_causal(q, X, 0.37), rtol=1e-12, atol=1e-13)


def test_attention_dense_limit_with_sink():
    """Same limit with finite sinks: duplicated keys turn the sink into an extra logit sink-ln2."""
    T, H, c = 13, 2, 6
    X, q, sink = randn(T, c), randn(T, H, c), randn(H)
    o, _ = O.hybrid_attn_prefill(q, X, X.copy(), sink, 0.5, m=1, W=T)
    np.testing.assert_allclose(o, _dense_causal(q, X, 0.5, sink - math.log(2.0)), rtol=1e-12, atol=1e-13)


def test_attention_window_only_is_dense_causal():
    """W=T with an empty top-k list (all -1) is plain dense causal attention."""
    T, H, c = 16, 2, 8
    X, q = randn(T, c), randn(T, H, c)
    idx = -np.ones((T, 4), np.int32)
    o, _ = O.hybrid_attn_prefill(q, X, randn(4, c), np.full(H, -np.inf), 0.3, m=4, W=T, idx=idx)
    np.testing.assert_allclose(o, _dense_causal(q, X, 0.3), rtol=1e-12, atol=1e-13)


def test_attention_banded_window():
    """W < T, no visible compressed entries: a banded causal mask of width W (library SDPA)."""
    T, H, c, W = 20, 2, 8, 5
    X, q = randn(T, c), randn(T, H, c)
    o, _ = O.hybrid_attn_prefill(q, X, randn(0, c), np.full(H, -np.inf), 0.4, m=64, W=W)
    t = torch.arange(T)
    mask = (t[None, :] <= t[:, None]) & (t[None, :] > t[:, None] - W)
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    Kt = torch.from_numpy(X)[None, None].expand(1, H, -1, -1)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Kt, attn_mask=mask, scale=0.4)[0]
    np.testing.assert_allclose(o, ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)


def test_attention_single_key_closed_form():
    c = 4
    v = randn(1, c)
    q = randn(1, 2, c)
    sink = np.array([0.3, -np.inf])
    o, lse = O.hybrid_attn_prefill(q, v, randn(1, c), sink, 1.0, m=8, W=1)
    for h in range(2):
        z = float(q[0, h] @ v[0])
        w = math.exp(z) / (math.exp(z) + math.exp(sink[h]))
        np.testing.assert_allclose(o[0, h], w * v[0], rtol=1e-13)
        np.testing.assert_allclose(lse[0, h], math.log(math.exp(z) + math.exp(sink[h])), rtol=1e-13)


def test_attention_causality_and_no_dedup():
    T, H, c, m, W = 24, 2, 6, 4, 6
    X, q, sink = randn(T, c), randn(T, H, c), randn(H)
    KVc = randn(T // m, c)
    idx = np.tile(np.array([0, 2, -1, 1], np.int32), (T, 1))
    o, _ = O.hybrid_attn_prefill(q, X, KVc, sink, 0.5, m, W, idx=idx)
    for t in [3, 10, 23]:
        X2 = X.copy()
        X2[t + 1:] = 50.0
        o2, _ = O.hybrid_attn_prefill(q, X2, KVc, sink, 0.5, m, W, idx=idx, rows=[t])
        assert np.array_equal(o2[0], o[t])
    # a repeated index counts twice (concatenation, no de-duplication)
    idx2 = np.tile(np.array([0, 0, -1, -1], np.int32), (T, 1))
    idx1 = np.tile(np.array([0, -1, -1, -1], np.int32), (T, 1))
    a, _ = O.hybrid_attn_prefill(q, X, KVc, sink, 0.5, m, W, idx=idx2, rows=[9])
    b, _ = O.hybrid_attn_prefill(q, X, KVc, sink, 0.5, m, W, idx=idx1, rows=[9])
    assert not np.allclose(a, b)


def test_decode_equals_prefill_row():
    T, H, c, m, W = 40, 3, 8, 4, 7
    X, q, sink = randn(T, c), randn(T, H, c), randn(H)
    KVc = randn(T // m, c)
    o, lse = O.hybrid_attn_prefill(q, X, KVc, sink, 0.6, m, W)  # HCA-style: all visible
    for t in [0, 5, 39]:
        lo = max(0, t - W + 1)
        win = np.zeros((W, c))
        win[:t + 1 - lo] = X[lo:t + 1][::-1]  # any order: attention is permutation-invariant
        od, ld = O.hybrid_attn_decode(q[t:t + 1], KVc, [0], [t], win, [t + 1 - lo], sink, 0.6, m, W)
        np.testing.assert_allclose(od[0], o[t], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(ld[0], lse[t], rtol=1e-12)


def test_decode_several_sequences_csa_equals_prefill_rows():
    """Decode of two sequences whose compressed rows share one cache (the second starting at
    comp_off[1]) gives, per sequence, that sequence's own prefill row at the same position,
    with the same top-k list (padding -1 skipped in both)."""
    H, c, m, W, k = 2, 8, 4, 7, 5
    lens = [30, 45]
    Xs = [randn(T, c) for T in lens]
    Cs = [randn(T // m, c) for T in lens]
    q, sink = randn(2, H, c), randn(H)
    comp_off = [0, len(Cs[0])]
    pos = [lens[0] - 1, lens[1] - 1]
    idx = -np.ones((2, k), np.int32)
    win = np.zeros((2 * W, c))
    for b in range(2):
        nv = int(O.n_vis(pos[b], m))
        pick = RNG.permutation(nv)[:k - 1 - b]
        idx[b, :len(pick)] = pick
        win[b * W:(b + 1) * W] = Xs[b][pos[b] - W + 1:pos[b] + 1]
    od, ld = O.hybrid_attn_decode(q, np.concatenate(Cs), comp_off, pos, win, [W, W], sink, 0.45, m,
                                  W, idx=idx)
    for b in range(2):
        full_idx = -np.ones((lens[b], k), np.int32)
        full_idx[pos[b]] = idx[b]
        qf = np.zeros((lens[b], H, c))
        qf[pos[b]] = q[b]
        op, lp = O.hybrid_attn_prefill(qf, Xs[b], Cs[b], sink, 0.45, m, W, idx=full_idx, rows=[pos[b]])
        np.testing.assert_allclose(od[b], op[0], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(ld[b], lp[0], rtol=1e-12)


# ---------------------------------------------------------------------------------------------
# Storage formats (OCP OFP8 E4M3, OCP MX FP4 E2M1 + E8M0, bf16)
# ---------------------------------------------------------------------------------------------

def _table(name):
    rows = []
    for line in open(os.path.join(GOLD, name)):
        if line.strip() and not line.startswith("#"):
            a, b = line.split()
            rows.append((a, b))
    return rows


def test_e2m1_decode_golden():
    for code, val in _table("fp4_e2m1_values.txt"):
        assert O.e2m1_decode(int(code)) == float(val)


def test_e2m1_encode_golden_rounding_and_roundtrip():
    for x, code in _table("fp4_e2m1_rounding.txt"):
        assert O.e2m1_encode(float(x)) == int(code), x
    for code in range(16):
        v = O.e2m1_decode(code)
        assert O.e2m1_encode(v) == (0 if code == 8 else code)


def test_e4m3_decode_golden_and_torch():
    for code, val in _table("fp8_e4m3_values.txt"):
        got = O.e4m3_decode(int(code, 16))
        assert (math.isnan(got) and val == "nan") or got == float(val)
    allc = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([O.e4m3_decode(b) for b in range(256)])
    np.testing.assert_array_equal(np.isnan(mine), np.isnan(allc))
    ok = ~np.isnan(allc)
    np.testing.assert_array_equal(mine[ok], allc[ok])


def test_e4m3_encode_matches_torch_rne():
    x = np.concatenate([RNG.standard_normal(20000) * 60, RNG.standard_normal(5000) * 0.01,
                        np.array([447.9, 448.0, -448.0, 2 ** -10, 3 * 2 ** -10, 0.0])]).astype(np.float32)
    x = np.clip(x, -448, 448)
    tor = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()
    tor[tor == 0x80] = 0  # every zero is +0 in our encoding
    mine = np.array([O.e4m3_encode(float(v)) for v in x], np.uint8)
    np.testing.assert_array_equal(mine, tor)


def test_bf16_rounding_matches_torch():
    x = np.concatenate([RNG.standard_normal(10000).astype(np.float32),
                        (np.arange(1, 2000, dtype=np.uint32) << 15 | 0x3F800000).view(np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(O.bf16_bits(x), ref)
    pick = np.r_[0:500, 10000:10500]  # random values, then exact halfway cases
    scalar = np.array([O.lib().orc_bf16_bits(float(v)) for v in x[pick]], np.uint16)
    np.testing.assert_array_equal(scalar, ref[pick])


def test_fp4_scale_exponent_rule():
    for e in range(-20, 20):
        assert O.fp4_scale_exp(6.0 * 2.0 ** e) == e
        assert O.fp4_scale_exp(float(np.nextafter(np.float32(6.0 * 2.0 ** e), np.float32(np.inf)))) == e + 1
    for a in RNG.random(2000) * 100 + 1e-3:
        a = float(np.float32(a))
        assert O.fp4_scale_exp(a) == math.ceil(math.log2(a / 6.0)), a
    assert O.fp4_scale_exp(0.0) == -127


def test_fp4_rows_on_grid_roundtrip_and_bounds():
    codes = RNG.integers(0, 16, size=(7, 64)).astype(np.uint8)
    codes[:, 0] = 7  # each block holds +6 so the scale exponent equals the drawn one
    codes[:, 32] = 15
    ex = RNG.integers(-5, 6, size=(7, 2))
    vals = np.array([[O.e2m1_decode(c) for c in row] for row in codes]) * np.repeat(2.0 ** ex, 32, axis=1)
    cq, sq = O.quant_fp4(vals.astype(np.float32))
    np.testing.assert_array_equal(O.dequant_fp4(cq, sq), vals)
    assert np.array_equal(sq.astype(int) - 127, ex)
    # random data: error at most half the largest grid step (1.0 at the top of the grid) * scale
    x = RNG.standard_normal((50, 128)).astype(np.float32)
    cq, sq = O.quant_fp4(x)
    err = np.abs(O.dequant_fp4(cq, sq) - x).reshape(50, 4, 32)
    scale = 2.0 ** (sq.astype(np.float64) - 127)
    assert np.all(err <= scale[:, :, None] * 1.0 + 1e-12)
    assert np.all(np.abs(x).reshape(50, 4, 32).max(-1) <= 6 * scale)


def test_kv_rows_amax_maps_to_448_and_rope_is_bf16():
    x = RNG.standard_normal((30, 512)).astype(np.float32)
    fp8, rb, sc = O.quant_kv(x, rope=64)
    am = np.abs(x[:, :448]).argmax(1)
    for r in range(30):
        assert fp8[r, am[r]] in (0x7E, 0xFE)
        assert sc[r] == np.float32(np.abs(x[r, :448]).max() / np.float32(448.0))
    np.testing.assert_array_equal(rb, torch.from_numpy(x[:, 448:].copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    deq = O.dequant_kv(fp8, rb, sc)
    # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 in the normal range
    err = np.abs(deq[:, :448] - x[:, :448])
    assert np.all(err <= np.abs(x[:, :448]) * 2.0 ** -4 + sc[:, None] * 2.0 ** -10)
    z = np.zeros((2, 512), np.float32)
    f0, _, s0 = O.quant_kv(z)
    assert np.all(f0 == 0) and np.all(s0 == 1.0)


# ---------------------------------------------------------------------------------------------
# inter-layer glue of the stacked decode workload (not on the pages)
# ---------------------------------------------------------------------------------------------

def test_glue_normalisation_identity_and_symmetry():
    R, c, d = 9, 16, 8
    o = randn(R, c)
    P, Rm = randn(c, c), randn(d, c)
    qn, zi = O.decode_glue(o, P, Rm)
    np.testing.assert_allclose(np.sqrt((qn ** 2).mean(1)), 1 / np.sqrt(c), rtol=1e-13)
    np.testing.assert_allclose(np.sqrt((zi ** 2).mean(1)), 1.0, rtol=1e-13)
    # scale invariance and odd symmetry in o
    qn2, zi2 = O.decode_glue(3.5 * o, P, Rm)
    np.testing.assert_allclose(qn2, qn, rtol=1e-12, atol=1e-14)
    qn3, zi3 = O.decode_glue(-o, P, Rm)
    np.testing.assert_allclose(qn3, -qn, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(zi3, -zi, rtol=1e-12, atol=1e-14)
    # identity projection: the normalised input itself (the projection is P o, not P^T o)
    qi, _ = O.decode_glue(o, np.eye(c), Rm)
    np.testing.assert_allclose(qi, o / np.sqrt((o ** 2).mean(1, keepdims=True)) / np.sqrt(c), rtol=1e-13)
    A = np.zeros((c, c)); A[0, 1] = 1.0; A[1, 0] = 1.0; A[2, 5] = 2.0  # non-symmetric part pins P o
    qa, _ = O.decode_glue(o, A, Rm)
    y = o @ A.T
    np.testing.assert_allclose(qa, y / np.sqrt((y ** 2).mean(1, keepdims=True)) / np.sqrt(c), rtol=1e-12)
    z0, _ = O.decode_glue(np.zeros((2, c)), P, Rm)
    assert np.all(z0 == 0)


# ---------------------------------------------------------------------------------------------
# layer fidelity: RMSNorm of entries, rotary embedding, Hadamard rotation
# ([notes] Sec. 2.3 Compressor and Indexer listings)
# ---------------------------------------------------------------------------------------------

def test_rmsnorm_unit_rms_scale_invariance_and_gain():
    g = np.random.default_rng(30)
    x = g.standard_normal((6, 512))
    y = O.rmsnorm(x, np.ones(512), 0.0)
    np.testing.assert_allclose(np.sqrt((y ** 2).mean(1)), 1.0, rtol=1e-12)       # unit RMS per row
    np.testing.assert_allclose(O.rmsnorm(7.5 * x, np.ones(512), 0.0), y, rtol=1e-12)  # scale invariance
    gain = g.standard_normal(512)
    np.testing.assert_allclose(O.rmsnorm(x, gain, 0.0), y * gain, rtol=1e-12)   # gain per channel
    # hand example: [3, 4] has mean square 12.5; with eps = 0.5 the divisor is sqrt(13)
    np.testing.assert_allclose(O.rmsnorm(np.array([[3.0, 4.0]]), np.ones(2), 0.5), [[3 / np.sqrt(13), 4 / np.sqrt(13)]])
    assert np.all(O.rmsnorm(np.zeros((1, 8)), np.ones(8), 1e-6) == 0.0)


def test_rope_identity_norms_and_untouched_leading_channels():
    g = np.random.default_rng(31)
    x = g.standard_normal((4, 512))
    y = O.rope(x, np.zeros(4, np.int64), 64)
    np.testing.assert_array_equal(y, x)                                    # position 0: identity
    y = O.rope(x, np.array([1, 77, 4096, 1048576]), 64)
    np.testing.assert_array_equal(y[:, :448], x[:, :448])                  # only the last 64 rotate
    pairs_x = x[:, 448:].reshape(4, 32, 2)
    pairs_y = y[:, 448:].reshape(4, 32, 2)
    np.testing.assert_allclose(np.linalg.norm(pairs_y, axis=-1), np.linalg.norm(pairs_x, axis=-1), rtol=1e-12)


def test_rope_frequencies_and_rotation_direction():
    """Unit vectors (1, 0) in every pair at position 1 come out at the angle of the pair's
    frequency base^(-2i/rd), counter-clockwise: (cos f, sin f)."""
    rd, base = 64, 10000.0
    x = np.tile([1.0, 0.0], rd // 2)[None, :]
    y = O.rope(x, np.array([1]), rd, base).reshape(rd // 2, 2)
    f = base ** (-np.arange(rd // 2) * 2.0 / rd)
    np.testing.assert_allclose(np.arctan2(y[:, 1], y[:, 0]), f, rtol=1e-12)
    np.testing.assert_allclose(y[0], [np.cos(1.0), np.sin(1.0)], rtol=1e-14)


def test_rope_composes_and_keeps_relative_positions():
    g = np.random.default_rng(32)
    q, k = g.standard_normal((2, 128))
    a, b, s = 300, 41, 9000
    two = O.rope(O.rope(q[None], np.array([a]), 64), np.array([b]), 64)
    np.testing.assert_allclose(two, O.rope(q[None], np.array([a + b]), 64), atol=1e-9)
    d1 = O.rope(q[None], np.array([a]), 64) @ O.rope(k[None], np.array([b]), 64).T
    d2 = O.rope(q[None], np.array([a + s]), 64) @ O.rope(k[None], np.array([b + s]), 64).T
    np.testing.assert_allclose(d1, d2, rtol=1e-9)


def test_hadamard_matches_the_library_matrix_and_is_an_involution():
    import scipy.linalg
    g = np.random.default_rng(33)
    for d in (32, 128, 512):
        x = g.standard_normal((3, d))
        y = O.hadamard(x)
        np.testing.assert_allclose(y, x @ scipy.linalg.hadamard(d) / np.sqrt(d), atol=1e-12)
        np.testing.assert_allclose(O.hadamard(y), x, atol=1e-12)          # normalised Sylvester: H H = I
        np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    e0 = np.zeros((1, 128))
    e0[0, 0] = 1.0
    np.testing.assert_allclose(O.hadamard(e0), np.full((1, 128), 1 / np.sqrt(128)), rtol=1e-14)


def test_hadamard_recursive_definition():
    """H_2n = [[H_n, H_n], [H_n, -H_n]] built recursively, column by column."""
    H = np.array([[1.0]])
    while H.shape[0] < 64:
        H = np.block([[H, H], [H, -H]])
    np.testing.assert_allclose(O.hadamard(np.eye(64)), H / 8.0, atol=1e-14)


# ---------------------------------------------------------------------------------------------
# decode append path ([qa] Question 5 state cache; [notes] Sec. 2.3 Compressor decode branch)
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("overlap,m,T", [(True, 4, 61), (False, 16, 70), (True, 1, 9), (False, 1, 5)])
def test_append_one_token_at_a_time_equals_the_prefill_compression(overlap, m, T):
    """Entries emitted by the state cache as tokens arrive one by one are bit for bit the prefill
    compression's entries, in order, one per completed block (a trailing partial block emits
    nothing)."""
    g = np.random.default_rng(40 + m)
    c = 16
    n_arr = 4 if overlap else 2
    X = [g.standard_normal((T, c)) for _ in range(n_arr)]
    B = 0.1 * g.standard_normal((2 * m if overlap else m, c))
    st = O.AppendState(overlap, m, B)
    got = []
    for t in range(T):
        e = st.append(t, [x[t] for x in X])
        assert (e is not None) == ((t + 1) % m == 0)
        if e is not None:
            got.append(e)
    ref = O.csa_compress(*X, B, m) if overlap else O.hca_compress(*X, B, m)
    assert len(got) == T // m
    np.testing.assert_array_equal(np.stack(got), ref)
