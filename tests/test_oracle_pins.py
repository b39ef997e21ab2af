"""Pins of the fp64 oracle to things other than itself: closed forms, the pages' stated
structure, textbook special cases checked against library routines (scipy, torch), and brute
force on tiny inputs. Every test here runs on the CPU."""
import os

import numpy as np
import pytest
import torch
from scipy.spatial.distance import cdist

import oracle as O
from msa_inputs import rng, workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ------------------------------------------------------------------------------- generator
def test_splitmix64_published_outputs():
    want = [int(x[0], 16) for x in _golden("splitmix64_state0.txt")]
    assert [int(v) for v in rng.splitmix64_stream(0, 3)] == want


def test_generator_moments_and_support():
    x = rng.normal(123, 7, 0, 1 << 20).astype(np.float64)
    assert abs(x.mean()) < 5e-3 and abs(x.var() - 1.0) < 5e-3
    assert np.abs(x).max() <= 2 * np.sqrt(3) + 1e-6
    # counter-based: any sub-range equals the same elements of a longer draw
    np.testing.assert_array_equal(rng.normal(123, 7, 1000, 50), x[1000:1050].astype(np.float32))


def test_distinct_ints_are_distinct_and_refuse_impossible_requests():
    got = rng.distinct_ints(5, 9, 40, 50, exclude=(3, 7, 60))
    assert len(set(got.tolist())) == 40 and not ({3, 7} & set(got.tolist())) and got.min() >= 0 and got.max() < 50
    assert sorted(rng.distinct_ints(5, 9, 48, 50, exclude=(3, 7)).tolist()) == [i for i in range(50) if i not in (3, 7)]
    with pytest.raises(ValueError):
        rng.distinct_ints(5, 9, 49, 50, exclude=(3, 7))   # 48 values exist: no endless draw


def test_bf16_round_to_nearest_even():
    one = np.float32(1.0)
    cases = np.array([one + 2.0 ** -8, one + 3 * 2.0 ** -8, one + 2.0 ** -9, -(one + 2.0 ** -8)], dtype=np.float32)
    got = rng.round_to(cases, "bf16")
    np.testing.assert_array_equal(got, np.array([1.0, 1.0 + 2.0 ** -6, 1.0, -1.0], dtype=np.float32))


# ------------------------------------------------------------------------------- RoPE
def test_rope_identity_at_position_zero():
    x = np.random.default_rng(0).standard_normal((5, 3, 16))
    np.testing.assert_array_equal(O.apply_rope(x, np.zeros(5, dtype=np.int64), 1e6), x)


def test_rope_d2_closed_form():
    p = np.array([0.3, 1.0, 2.5])
    got = O.apply_rope(np.tile([[1.0, 0.0]], (3, 1)), p, 1e6)
    np.testing.assert_allclose(got, np.stack([np.cos(p), np.sin(p)], 1), atol=1e-15)
    got = O.apply_rope(np.tile([[0.0, 1.0]], (3, 1)), p, 1e6)
    np.testing.assert_allclose(got, np.stack([-np.sin(p), np.cos(p)], 1), atol=1e-15)


def test_rope_rotate_half_pairing_and_frequency():
    # d = 4: element 1 pairs with element 3 and turns at w_1 = base^(-2/4)
    base, p = 100.0, 3.0
    x = np.array([[0.0, 1.0, 0.0, 0.0]])
    got = O.apply_rope(x, np.array([p]), base)[0]
    w1 = base ** -0.5
    np.testing.assert_allclose(got, [0.0, np.cos(p * w1), 0.0, np.sin(p * w1)], atol=1e-15)


def test_rope_norm_relative_position_and_composition():
    r = np.random.default_rng(1)
    x = r.standard_normal((64, 2, 128))
    y = r.standard_normal((64, 2, 128))
    m = r.integers(0, 2048, 64)
    n = r.integers(0, 2048, 64)
    s = r.integers(0, 2048, 64)
    np.testing.assert_allclose(np.linalg.norm(O.apply_rope(x, m, 1e6), axis=-1), np.linalg.norm(x, axis=-1),
                               rtol=1e-13)
    a = (O.apply_rope(x, m, 1e6) * O.apply_rope(y, n, 1e6)).sum(-1)
    b = (O.apply_rope(x, m + s, 1e6) * O.apply_rope(y, n + s, 1e6)).sum(-1)
    np.testing.assert_allclose(a, b, atol=1e-9)
    np.testing.assert_allclose(O.apply_rope(O.apply_rope(x, m, 1e6), n, 1e6), O.apply_rope(x, m + n, 1e6),
                               atol=1e-9)


def test_doc_positions_restart_at_zero():
    off, want = _golden("doc_positions.txt")
    got = O.doc_positions(np.array([int(v) for v in off]))
    np.testing.assert_array_equal(got, [int(v) for v in want])


def test_global_positions_start_at_k():
    np.testing.assert_array_equal(O.global_positions(4, 0, 3), [4, 5, 6])
    np.testing.assert_array_equal(O.global_positions(12, 96, 2), [108, 109])


# ------------------------------------------------------------------------------- pooling
def _ragged(seed=0, lens=(300, 128, 1, 129, 0, 257), H=2, d=8):
    r = np.random.default_rng(seed)
    off = np.zeros(len(lens) + 1, dtype=np.int64)
    off[1:] = np.cumsum(lens)
    return off, r.standard_normal((off[-1], H, d))


def test_pool_chunk_one_is_identity():
    off, x = _ragged()
    np.testing.assert_array_equal(O.pool_chunks(x, off, 1), x)


def test_pool_big_chunk_is_document_mean():
    off, x = _ragged()
    got = O.pool_chunks(x, off, 10_000)
    want = [x[a:b].mean(0) for a, b in zip(off[:-1], off[1:]) if b > a]
    np.testing.assert_allclose(got, np.stack(want), rtol=1e-14)


def test_pool_ragged_last_chunk_and_counts():
    off, x = _ragged()
    doc_chunk_off, bounds = O.chunk_layout(off, 128)
    np.testing.assert_array_equal(np.diff(doc_chunk_off), [3, 1, 1, 2, 0, 3])
    got = O.pool_chunks(x, off, 128)
    # doc 0 (300 tokens): last chunk is the mean of its 44 real tokens
    np.testing.assert_allclose(got[2], x[256:300].mean(0), rtol=1e-14)
    # doc 3 (129 tokens, starting at 429): second chunk is the single token 557
    np.testing.assert_allclose(got[6], x[557], rtol=0)
    assert all(b - a <= 128 for a, b in bounds)


def test_pool_constant_chunk_and_linearity():
    off, x = _ragged()
    x2 = np.random.default_rng(5).standard_normal(x.shape)
    x[0:128] = x[7]
    p = O.pool_chunks(x, off, 128)
    np.testing.assert_allclose(p[0], x[7], rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(O.pool_chunks(2.5 * x - 0.5 * x2, off, 128),
                               2.5 * p - 0.5 * O.pool_chunks(x2, off, 128), atol=1e-13)


def test_encode_translation_invariance_of_a_document():
    """A document's pooled, document-wise-rotated K-bar does not depend on where it sits in the bank."""
    r = np.random.default_rng(2)
    lens = [200, 300, 130]
    docs = [r.standard_normal((n, 2, 16)) for n in lens]
    for order in ([0, 1, 2], [2, 0, 1], [1, 2, 0]):
        ls = [lens[i] for i in order]
        off = np.zeros(4, dtype=np.int64)
        off[1:] = np.cumsum(ls)
        kbar, _, _ = O.encode_memory(np.concatenate([docs[i] for i in order]), None, None, off, 64, 1e4)
        dco, _ = O.chunk_layout(off, 64)
        where = order.index(1)
        got = kbar[dco[where]:dco[where + 1]]
        if order == [0, 1, 2]:
            ref = got
        else:
            np.testing.assert_allclose(got, ref, atol=1e-15)


# ------------------------------------------------------------------------------- router scoring
def test_route_reduction_order_golden():
    want = float(_golden("route_reduction_order.txt")[0][0])
    krbar = np.array([[[1.0, 0.0], [1.0, 0.0]]])                    # [C=1, H=2, d=2]
    qr = np.array([[[1.0, 0.0], [-1.0, 0.0]], [[1.0, np.sqrt(3)], [1.0, np.sqrt(3)]]])  # [T=2, H=2, d=2]
    assert abs(O.chunk_scores_one_query(krbar, qr)[0] - want) < 1e-15


def test_route_brute_force_against_scipy_cosine():
    r = np.random.default_rng(3)
    C, T, H, d = 37, 5, 4, 16
    krbar, qr = r.standard_normal((C, H, d)), r.standard_normal((T, H, d))
    cos = np.stack([1.0 - cdist(qr[:, h], krbar[:, h], metric="cosine") for h in range(H)], -1)  # [T, C, H]
    want = cos.mean(-1).max(0)
    np.testing.assert_allclose(O.chunk_scores_one_query(krbar, qr), want, atol=1e-13)


def test_route_range_folded_identity_scale_invariance():
    r = np.random.default_rng(4)
    C, T, H, d = 200, 7, 8, 32
    krbar, qr = r.standard_normal((C, H, d)), r.standard_normal((T, H, d))
    s = O.chunk_scores_one_query(krbar, qr)
    assert np.all(s <= 1.0) and np.all(s >= -1.0)
    np.testing.assert_allclose(O.chunk_scores_folded(krbar, qr), s, atol=1e-12)
    scale_k = r.uniform(0.1, 10.0, (C, H, 1))
    scale_q = r.uniform(0.1, 10.0, (T, H, 1))
    np.testing.assert_allclose(O.chunk_scores_one_query(krbar * scale_k, qr * scale_q), s, atol=1e-12)


def test_route_planted_chunk_scores_one_and_is_selected():
    r = np.random.default_rng(5)
    C, T, H, d = 64, 9, 8, 128
    krbar, qr = r.standard_normal((C, H, d)), r.standard_normal((T, H, d))
    krbar[41] = 3.0 * qr[4]
    off = np.arange(0, C + 1, 8)
    ds, cs = O.route(krbar, off, qr[None])
    assert abs(cs[0, 41] - 1.0) < 1e-12
    assert abs(ds[0, 5] - 1.0) < 1e-12
    idx, _ = O.topk_docs(ds, 1)
    assert idx[0, 0] == 5


def test_route_zero_norm_vector_has_cosine_zero():
    krbar = np.zeros((2, 2, 4))
    krbar[1, 0] = [1, 0, 0, 0]
    qr = np.array([[[1.0, 0, 0, 0], [0, 0, 0, 0]]])
    np.testing.assert_allclose(O.chunk_scores_one_query(krbar, qr), [0.0, 0.5], atol=0)


def test_doc_score_is_max_over_its_chunks():
    cs = np.array([0.1, 0.9, 0.3, 0.2, -0.4, -0.1])
    np.testing.assert_array_equal(O.doc_scores_from_chunks(cs, np.array([0, 3, 4, 6])), [0.9, 0.2, -0.1])


# ------------------------------------------------------------------------------- top-k
def test_topk_matches_full_sort_with_ties():
    r = np.random.default_rng(6)
    for trial in range(20):
        D = int(r.integers(1, 60))
        s = np.round(r.uniform(-1, 1, D), 1)              # many exact ties
        k = int(r.integers(1, D + 1))
        want = sorted(range(D), key=lambda i: (-s[i], i))[:k]
        idx, val = O.topk_docs(s[None], k)
        assert list(idx[0]) == want
        np.testing.assert_array_equal(val[0], s[want])


def test_topk_permutation_equivariance():
    r = np.random.default_rng(7)
    s = r.standard_normal(100)
    perm = r.permutation(100)
    idx, _ = O.topk_docs(s[None], 10)
    idx_p, _ = O.topk_docs(s[perm][None], 10)
    np.testing.assert_array_equal(perm[idx_p[0]], idx[0])


# ------------------------------------------------------------------------------- gather + attention
def test_gather_is_rank_ordered_row_copy():
    r = np.random.default_rng(8)
    kv = r.standard_normal((10, 2, 2, 4))
    off = np.array([0, 3, 4, 8, 10])
    got = O.gather_memory(kv, off, [2, 0, 3])
    np.testing.assert_array_equal(got, np.concatenate([kv[4:8], kv[0:3], kv[8:10]]))


def _sdpa(q, k, v, causal=False):
    """torch's scaled_dot_product_attention in fp64 on [T, h, d] tensors with GQA expansion."""
    hq, hkv = q.shape[1], k.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(hq // hkv, 0)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(hq // hkv, 0)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal)
    return o[0].permute(1, 0, 2).numpy()


def test_attention_reduces_to_dense_attention():
    """chunk = 1 and k = all docs, no local KV: sparse attention is dense softmax attention."""
    r = np.random.default_rng(9)
    n_tok, hq, hkv, d = 40, 8, 2, 16
    k, v, q = r.standard_normal((n_tok, hkv, d)), r.standard_normal((n_tok, hkv, d)), r.standard_normal((6, hq, d))
    off = np.array([0, 10, 25, 40])
    kbar, vbar, _ = O.encode_memory(k, v, None, off, 1, 1e6)
    kv = np.stack([kbar, vbar], 1)
    dco, _ = O.chunk_layout(off, 1)
    mem = O.gather_memory(kv, dco, [0, 1, 2])
    empty = np.zeros((0, hkv, d))
    got = O.sparse_attention(q, mem[:, 0], mem[:, 1], empty, empty, 0, 1 / np.sqrt(d))
    np.testing.assert_allclose(got, _sdpa(q, mem[:, 0], mem[:, 1]), atol=1e-12)


def test_attention_local_causal_matches_sdpa():
    r = np.random.default_rng(10)
    T, hq, hkv, d = 12, 4, 2, 8
    q, k, v = r.standard_normal((T, hq, d)), r.standard_normal((T, hkv, d)), r.standard_normal((T, hkv, d))
    empty = np.zeros((0, hkv, d))
    got = O.sparse_attention(q, empty, empty, k, v, 0, 1 / np.sqrt(d))
    np.testing.assert_allclose(got, _sdpa(q, k, v, causal=True), atol=1e-12)


def test_attention_special_cases():
    r = np.random.default_rng(11)
    hq, hkv, d = 4, 1, 8
    q = r.standard_normal((3, hq, d))
    k1, v1 = r.standard_normal((1, hkv, d)), r.standard_normal((1, hkv, d))
    empty = np.zeros((0, hkv, d))
    got = O.sparse_attention(q, k1, v1, empty, empty, 0, 0.3)
    np.testing.assert_allclose(got, np.broadcast_to(v1[0, 0], got.shape), atol=1e-15)
    ks = np.repeat(k1, 5, 0)
    vs = r.standard_normal((5, hkv, d))
    got = O.sparse_attention(q, ks, vs, empty, empty, 0, 0.3)
    np.testing.assert_allclose(got, np.broadcast_to(vs.mean(0)[0], got.shape), atol=1e-14)


def test_attention_memory_order_invariance_and_causality():
    r = np.random.default_rng(12)
    T, hq, hkv, d, M, L = 4, 8, 2, 16, 9, 10
    q = r.standard_normal((T, hq, d))
    mk, mv = r.standard_normal((M, hkv, d)), r.standard_normal((M, hkv, d))
    lk, lv = r.standard_normal((L, hkv, d)), r.standard_normal((L, hkv, d))
    q_start = 5
    base = O.sparse_attention(q, mk, mv, lk, lv, q_start, 0.25)
    perm = r.permutation(M)
    np.testing.assert_allclose(O.sparse_attention(q, mk[perm], mv[perm], lk, lv, q_start, 0.25), base, atol=1e-13)
    # token 0 sees local keys 0..5 only: changing key 6.. leaves it unchanged, changing key 5 does not
    lk2 = lk.copy()
    lk2[6:] += 3.0
    np.testing.assert_array_equal(O.sparse_attention(q, mk, mv, lk2, lv, q_start, 0.25)[0], base[0])
    lk3 = lk.copy()
    lk3[5] += 3.0
    assert np.abs(O.sparse_attention(q, mk, mv, lk3, lv, q_start, 0.25)[0] - base[0]).max() > 1e-6


# ------------------------------------------------------------------------------- interleave
def _small_chain(rounds=3):
    return workloads.Workload("chain-small", 77, np.full(48, 256), 64, "f32", n_q=2, T0=8, k=3, prepooled=True,
                              layers=2, rounds=rounds, T_new=4, H=2, d=16, hq=4, hkv=2, plant_kind="chain")


def test_interleave_chain_docs_selected_each_round():
    w = _small_chain()
    for layer in range(w.layers):
        krbar = w.host_tensor(layer, "krbar")
        kv = w.host_tensor(layer, "bank")
        qr, q, kn, vn = w.qr(layer), w.q(layer), w.k_new(layer), w.v_new(layer)
        for qi in range(w.n_q):
            rounds = O.interleave(krbar, w.doc_chunk_off, kv, qr[qi], q[qi], kn[qi], vn[qi], w.T0, w.T_new, w.rounds,
                                  w.k, w.rope_base)
            for rnd, (idx, val, ds, o) in enumerate(rounds):
                for doc in w.expected(layer, rnd, qi):
                    assert doc in idx, (layer, rnd, qi, doc, idx)
                assert o.shape == (w.round_tokens(rnd)[1], w.hq, w.d)
                np.testing.assert_array_equal(val, ds[idx])


def test_interleave_single_round_is_one_route_and_attend():
    w = _small_chain(rounds=1)
    krbar, kv = w.host_tensor(0, "krbar"), w.host_tensor(0, "bank")
    qr, q, kn, vn = w.qr(0), w.q(0), w.k_new(0), w.v_new(0)
    idx, val, o = O.route_and_attend(krbar, w.doc_chunk_off, kv, qr[0, :8], q[0, :8], kn[0], vn[0], 0, 3, 1e6)
    ds, _ = O.route(krbar, w.doc_chunk_off, qr[0:1, :8])
    i2, v2 = O.topk_docs(ds, 3)
    np.testing.assert_array_equal(idx, i2[0])
    mem = O.gather_memory(kv, w.doc_chunk_off, i2[0])
    kr = O.apply_rope(kn[0, :8], np.arange(3, 11), 1e6)
    qq = O.apply_rope(q[0, :8], np.arange(3, 11), 1e6)
    np.testing.assert_allclose(o, O.sparse_attention(qq, mem[:, 0], mem[:, 1], kr, vn[0, :8], 0, 0.25), atol=1e-15)
    # the interleave loop with one round is exactly this route-and-attend
    (i3, v3, _, o3), = O.interleave(krbar, w.doc_chunk_off, kv, qr[0, :8], q[0, :8], kn[0, :8], vn[0, :8], 8, 4, 1,
                                    3, 1e6)
    np.testing.assert_array_equal(i3, idx)
    np.testing.assert_array_equal(v3, val)
    np.testing.assert_array_equal(o3, o)


def _interleave_case(seed, T0=6, T_new=3, rounds=3, n_docs=30, H=2, d=16, hq=4, hkv=2):
    r = np.random.default_rng(seed)
    counts = r.integers(1, 5, n_docs)
    off = np.concatenate([[0], np.cumsum(counts)])
    C = int(off[-1])
    T_total = T0 + T_new * (rounds - 1)
    return (off, r.standard_normal((C, H, d)), r.standard_normal((C, 2, hkv, d)),
            r.standard_normal((T_total, H, d)), r.standard_normal((T_total, hq, d)),
            r.standard_normal((T_total, hkv, d)), r.standard_normal((T_total, hkv, d)))


def test_interleave_rounds_are_prefixes_of_one_causal_pass():
    """With every router token equal, every round selects the same documents; the appended tokens
    then attend exactly as they would in one causal pass over the whole context: the rounds'
    outputs, concatenated, equal a single round over all tokens. A wrong global offset, a local
    context that does not accumulate, or a wrong causal start in a later round breaks this."""
    off, krbar, kv, qr, q, kn, vn = _interleave_case(31)
    qr[:] = qr[0]
    T0, T_new, R, k = 6, 3, 3, 4
    rounds = O.interleave(krbar, off, kv, qr, q, kn, vn, T0, T_new, R, k, 1e6)
    (i1, _, _, whole), = O.interleave(krbar, off, kv, qr, q, kn, vn, T0 + T_new * (R - 1), 0, 1, k, 1e6)
    for idx, _, _, _ in rounds:
        np.testing.assert_array_equal(idx, i1)
    np.testing.assert_allclose(np.concatenate([o for *_, o in rounds]), whole, atol=1e-13)
    assert [o.shape[0] for *_, o in rounds] == [6, 3, 3]


def test_interleave_routes_with_every_active_token():
    """Round r routes with all tokens active so far (the max over tokens runs over a growing set):
    every document's score, hence the score at each rank of the top-k, never falls from one round
    to the next; routing with only the appended tokens would break that on random inputs, and a
    later round's scores are the max of the earlier round's and the appended tokens' own."""
    off, krbar, kv, qr, q, kn, vn = _interleave_case(32, rounds=4)
    rounds = O.interleave(krbar, off, kv, qr, q, kn, vn, 6, 3, 4, 5, 1e6)
    for (ia, va, da, _), (ib, vb, db, _) in zip(rounds[:-1], rounds[1:]):
        assert np.all(db >= da)
        assert np.all(vb >= va)
    for r in range(1, 4):
        L_prev, n = O.interleave_round_tokens(r, 6, 3)
        new_only, _ = O.route(krbar, off, qr[None, L_prev:L_prev + n])
        np.testing.assert_allclose(rounds[r][2], np.maximum(rounds[r - 1][2], new_only[0]), atol=1e-15)
    assert any(np.any(rounds[r][2] > rounds[r - 1][2]) for r in range(1, 4))


def test_interleave_select_override_keeps_routing():
    """`select` replaces only the documents the attention reads: routing, top-k and scores stay the
    oracle's, and attending over the oracle's own choice reproduces the default output."""
    off, krbar, kv, qr, q, kn, vn = _interleave_case(33)
    base = O.interleave(krbar, off, kv, qr, q, kn, vn, 6, 3, 3, 4, 1e6)
    same = O.interleave(krbar, off, kv, qr, q, kn, vn, 6, 3, 3, 4, 1e6, select=[b[0] for b in base])
    other = O.interleave(krbar, off, kv, qr, q, kn, vn, 6, 3, 3, 4, 1e6, select=[[0, 1, 2, 3]] * 3)
    for b, s_, o_ in zip(base, same, other):
        np.testing.assert_array_equal(b[3], s_[3])
        np.testing.assert_array_equal(b[0], o_[0])
        np.testing.assert_array_equal(b[2], o_[2])


@pytest.mark.parametrize("name", ["tiny"])
def test_tiny_workload_planted_docs_route_first(name):
    """On the tiny configuration the two planted documents are the oracle's top-2."""
    w = workloads.CONFIGS[name]()
    kr = w.host_tensor(0, "kr")
    _, _, krbar = O.encode_memory(None, None, kr, w.doc_tok_off, w.chunk, w.rope_base)
    ds, _ = O.route(krbar, w.doc_chunk_off, w.qr(0)[:, :w.T0])
    idx, val = O.topk_docs(ds, w.k)
    assert set(idx[0, :2]) == {17, 42}
    assert val[0, 1] > 0.9 and val[0, 2] < 0.5


# ------------------------------------------------------------------------------- fine stage
def test_token_bank_rows_rotate_keys_by_document_position():
    """K of the first token of every document is unrotated (position 0), every V row is the raw
    value, every key keeps its norm, and a key at position p equals the closed-form rotation."""
    r = np.random.default_rng(21)
    off = np.array([0, 5, 5, 12, 20])               # includes an empty document
    k, v = r.standard_normal((20, 2, 8)), r.standard_normal((20, 2, 8))
    tb = O.token_bank(k, v, off, 1e4)
    assert tb.shape == (20, 2, 2, 8)
    np.testing.assert_array_equal(tb[:, 1], v)
    for s in (0, 5, 12):
        np.testing.assert_array_equal(tb[s, 0], k[s])
    np.testing.assert_allclose(np.linalg.norm(tb[:, 0], axis=-1), np.linalg.norm(k, axis=-1), rtol=1e-13)
    # token 15 is position 3 of the document starting at 12: pair i rotates by 3 * 1e4^(-2i/8)
    w = 1e4 ** (-2.0 * np.arange(4) / 8)
    c, sn = np.cos(3 * w), np.sin(3 * w)
    x = k[15]
    want = np.concatenate([x[:, :4] * c - x[:, 4:] * sn, x[:, 4:] * c + x[:, :4] * sn], axis=-1)
    np.testing.assert_allclose(tb[15, 0], want, atol=1e-14)


def test_token_bank_translation_invariance():
    """A document's token rows do not depend on where it sits in the bank (positions restart at 0)."""
    r = np.random.default_rng(22)
    doc = r.standard_normal((9, 1, 8)), r.standard_normal((9, 1, 8))
    pre = r.standard_normal((7, 1, 8)), r.standard_normal((7, 1, 8))
    a = O.token_bank(doc[0], doc[1], np.array([0, 9]), 1e6)
    b = O.token_bank(np.concatenate([pre[0], doc[0]]), np.concatenate([pre[1], doc[1]]), np.array([0, 7, 16]), 1e6)
    np.testing.assert_allclose(b[7:], a, atol=1e-15)


def test_fine_stage_with_chunk_one_equals_coarse():
    """With chunks of one token the chunk means are the tokens themselves, so the fine stage and the
    coarse path attend over identical memories and give the same result."""
    w = _small_chain(rounds=1)
    r = np.random.default_rng(23)
    n_docs = 12
    off = np.arange(0, 4 * n_docs + 1, 4)
    k, v = r.standard_normal((4 * n_docs, w.hkv, w.d)), r.standard_normal((4 * n_docs, w.hkv, w.d))
    kr = r.standard_normal((4 * n_docs, w.H, w.d))
    kbar, vbar, krbar = O.encode_memory(k, v, kr, off, 1, 1e6)
    dco, _ = O.chunk_layout(off, 1)
    qr, q, kn, vn = r.standard_normal((6, w.H, w.d)), r.standard_normal((6, w.hq, w.d)), \
        r.standard_normal((6, w.hkv, w.d)), r.standard_normal((6, w.hkv, w.d))
    coarse = O.route_and_attend(krbar, dco, np.stack([kbar, vbar], 1), qr, q, kn, vn, 0, 3, 1e6)
    fine = O.route_and_attend_fine(krbar, dco, O.token_bank(k, v, off, 1e6), off, qr, q, kn, vn, 0, 3, 1e6)
    np.testing.assert_array_equal(coarse[0], fine[0])
    np.testing.assert_allclose(fine[2], coarse[2], atol=1e-13)


def test_fine_stage_over_every_document_is_dense_attention():
    """Selecting every document, the fine stage is dense softmax attention over all memory tokens
    (doc-wise rotated keys, fully visible) followed by the causal local keys: compared with torch's
    scaled_dot_product_attention on the concatenated keys with an explicit mask."""
    r = np.random.default_rng(24)
    off = np.array([0, 7, 19, 24])
    hq, hkv, d, T = 4, 2, 16, 5
    k, v = r.standard_normal((24, hkv, d)), r.standard_normal((24, hkv, d))
    kr = r.standard_normal((24, 2, d))
    _, _, krbar = O.encode_memory(None, None, kr, off, 8, 1e6)
    dco, _ = O.chunk_layout(off, 8)
    qr, q = r.standard_normal((T, 2, d)), r.standard_normal((T, hq, d))
    kn, vn = r.standard_normal((T, hkv, d)), r.standard_normal((T, hkv, d))
    idx, _, got = O.route_and_attend_fine(krbar, dco, O.token_bank(k, v, off, 1e6), off, qr, q, kn, vn, 0, 3, 1e6)
    pos = np.concatenate([np.arange(7), np.arange(12), np.arange(5)])
    mem_k = O.apply_rope(k, pos, 1e6)
    order = np.concatenate([np.arange(off[i], off[i + 1]) for i in idx])
    keys = np.concatenate([mem_k[order], O.apply_rope(kn, np.arange(3, 3 + T), 1e6)])
    vals = np.concatenate([v[order], vn])
    qt = torch.from_numpy(O.apply_rope(q, np.arange(3, 3 + T), 1e6)).permute(1, 0, 2)[None]
    kt = torch.from_numpy(keys).permute(1, 0, 2).repeat_interleave(hq // hkv, 0)[None]
    vt = torch.from_numpy(vals).permute(1, 0, 2).repeat_interleave(hq // hkv, 0)[None]
    mask = torch.ones(T, 24 + T, dtype=torch.bool)
    mask[:, 24:] = torch.tril(torch.ones(T, T, dtype=torch.bool))
    want = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)[0].permute(1, 0, 2).numpy()
    np.testing.assert_allclose(got, want, atol=1e-12)
