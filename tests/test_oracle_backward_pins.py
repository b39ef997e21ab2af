"""Pins of the fp64 backward oracle against things other than itself: torch autograd of scaled dot
product attention, central finite differences of the forward oracle, adjoint (dot-product)
identities of the linear steps, and closed forms of the auxiliary loss."""
import numpy as np
import pytest
import torch

import oracle as O


def _rng(s):
    return np.random.default_rng(s)


def _fd(f, x, idx, h=1e-6):
    """Central differences of scalar f at the flat positions idx of x."""
    out = []
    for i in idx:
        xp, xm = x.copy(), x.copy()
        xp.flat[i] += h
        xm.flat[i] -= h
        out.append((f(xp) - f(xm)) / (2 * h))
    return np.array(out)


# ------------------------------------------------------------------------------------------ attention
def test_attention_backward_matches_torch_autograd_of_sdpa():
    r = _rng(1)
    T, hq, hkv, d, M = 6, 8, 2, 16, 11
    q, k, v = r.standard_normal((T, hq, d)), r.standard_normal((M, hkv, d)), r.standard_normal((M, hkv, d))
    do = r.standard_normal((T, hq, d))
    empty = np.zeros((0, hkv, d))
    dq, dk, dv, _, _ = O.sparse_attention_backward(q, k, v, empty, empty, 0, 1 / np.sqrt(d), do)
    qt = torch.tensor(q, requires_grad=True)
    kt = torch.tensor(k, requires_grad=True)
    vt = torch.tensor(v, requires_grad=True)
    o = torch.nn.functional.scaled_dot_product_attention(
        qt.permute(1, 0, 2)[None], kt.permute(1, 0, 2).repeat_interleave(hq // hkv, 0)[None],
        vt.permute(1, 0, 2).repeat_interleave(hq // hkv, 0)[None])
    o.backward(torch.tensor(do).permute(1, 0, 2)[None])
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-12)


def test_attention_backward_with_causal_local_keys_matches_finite_differences():
    r = _rng(2)
    T, hq, hkv, d, M, L, q_start = 3, 4, 2, 4, 5, 5, 2
    args = [r.standard_normal((T, hq, d)), r.standard_normal((M, hkv, d)), r.standard_normal((M, hkv, d)),
            r.standard_normal((L, hkv, d)), r.standard_normal((L, hkv, d))]
    w = r.standard_normal((T, hq, d))
    grads = O.sparse_attention_backward(*args, q_start, 0.5, w)
    for a in range(5):
        def f(x, a=a):
            xs = list(args)
            xs[a] = x
            return float((O.sparse_attention(*xs, q_start, 0.5) * w).sum())
        idx = r.choice(args[a].size, 12, replace=False)
        np.testing.assert_allclose(grads[a].flat[idx], _fd(f, args[a], idx), atol=1e-8)
    # a local key past every query's window gets no gradient
    assert np.all(grads[3][q_start + T:] == 0) and np.all(grads[4][q_start + T:] == 0)


# ------------------------------------------------------------------------------------------ linear steps
def test_gather_pool_rope_adjoint_identities():
    r = _rng(3)
    off_tok = np.array([0, 5, 5, 12, 30])
    chunk = 4
    dco, _ = O.chunk_layout(off_tok, chunk)
    C = int(dco[-1])
    idx = [2, 0, 2]                                                  # a document fetched twice
    x = r.standard_normal((C, 2, 3))
    y = r.standard_normal((int(dco[3] - dco[2]) * 2 + int(dco[1] - dco[0]), 2, 3))
    assert np.isclose((O.gather_memory(x, dco, idx) * y).sum(), (x * O.gather_memory_backward(y, dco, idx, C)).sum())
    t = r.standard_normal((30, 2, 3))
    cb = r.standard_normal((C, 2, 3))
    assert np.isclose((O.pool_chunks(t, off_tok, chunk) * cb).sum(), (t * O.pool_chunks_backward(cb, off_tok, chunk)).sum())
    pos = r.integers(0, 3000, 30)
    a, b = r.standard_normal((30, 2, 8)), r.standard_normal((30, 2, 8))
    assert np.isclose((O.apply_rope(a, pos, 1e6) * b).sum(), (a * O.apply_rope_backward(b, pos, 1e6)).sum())
    k, dk = r.standard_normal((30, 2, 8)), r.standard_normal((C, 2, 8))
    kb, _, _ = O.encode_memory(k, None, None, off_tok, chunk, 1e6)
    gk, _, _ = O.encode_memory_backward(dk, None, None, off_tok, chunk, 1e6)
    assert np.isclose((kb * dk).sum(), (k * gk).sum())


def test_unit_backward_finite_differences_and_zero_vector():
    r = _rng(4)
    x, w = r.standard_normal((3, 2, 6)), r.standard_normal((3, 2, 6))
    g = O.unit_backward(x, w)
    idx = r.choice(x.size, 10, replace=False)
    np.testing.assert_allclose(g.flat[idx], _fd(lambda z: float((O.unit(z) * w).sum()), x, idx), atol=1e-8)
    assert np.all(O.unit_backward(np.zeros((1, 4)), np.ones((1, 4))) == 0)


# ------------------------------------------------------------------------------------------ auxiliary loss
def test_aux_loss_two_documents_is_logistic_and_gradients_sum_to_zero():
    s = np.array([[0.3, -0.1]])
    tau = 0.05
    loss, g = O.router_aux_loss(s, [[0]], tau)
    z = (s[0, 0] - s[0, 1]) / tau
    assert np.isclose(loss, np.log1p(np.exp(-z)))
    sig = 1 / (1 + np.exp(-z))
    np.testing.assert_allclose(g[0], [-(1 - sig) / tau, (1 - sig) / tau], rtol=1e-12)
    r = _rng(5)
    s = r.uniform(-1, 1, (3, 40))
    ev = [[3, 7], [0], [39, 1, 2]]
    loss, g = O.router_aux_loss(s, ev, 0.1)
    np.testing.assert_allclose(g.sum(axis=1), 0, atol=1e-12)
    idx = r.choice(s.size, 8, replace=False)
    np.testing.assert_allclose(g.flat[idx], _fd(lambda z: O.router_aux_loss(z, ev, 0.1)[0], s, idx), atol=1e-7)


def test_route_backward_matches_finite_differences():
    r = _rng(6)
    off = np.array([0, 3, 4, 8, 8, 11])                              # includes a document without chunks
    H, d, T, n_q = 2, 5, 4, 2
    kr = r.standard_normal((11, H, d))
    qr = r.standard_normal((n_q, T, H, d))
    w = r.standard_normal((n_q, 5))
    w[:, 3] = 0.0                                                     # the empty document's score is -inf

    def f_q(x):
        return float((O.route(kr, off, x)[0][:, [0, 1, 2, 4]] * w[:, [0, 1, 2, 4]]).sum())

    def f_k(x):
        return float((O.route(x, off, qr)[0][:, [0, 1, 2, 4]] * w[:, [0, 1, 2, 4]]).sum())

    dqr, dkh = O.route_backward(kr, off, qr, w)
    dkr = O.unit_backward(kr, dkh)
    iq = r.choice(qr.size, 15, replace=False)
    ik = r.choice(kr.size, 15, replace=False)
    np.testing.assert_allclose(dqr.flat[iq], _fd(f_q, qr, iq), atol=1e-7)
    np.testing.assert_allclose(dkr.flat[ik], _fd(f_k, kr, ik), atol=1e-7)


def test_route_backward_on_exact_unit_index_equals_normalising_form():
    """For exactly unit key vectors, scoring them as stored (index form) is the cosine itself."""
    r = _rng(8)
    off = np.array([0, 2, 5, 9])
    kr = O.unit(r.standard_normal((9, 2, 6)))
    qr = r.standard_normal((2, 3, 2, 6))
    w = r.standard_normal((2, 3))
    a = O.route_backward(kr, off, qr, w)
    b = O.route_backward(kr, off, qr, w, index_is_unit=True)
    np.testing.assert_allclose(a[0], b[0], atol=1e-14)
    np.testing.assert_allclose(a[1], b[1], atol=1e-14)


# ------------------------------------------------------------------------------------------ chained training loss
def test_training_loss_gradient_through_encode_route_and_attention():
    """L = <W, attention output> + lam * aux(router scores) with the selection held fixed: the
    composed backward oracle against finite differences of the forward oracle in token K, V, K^R."""
    r = _rng(7)
    off_tok = np.array([0, 9, 20, 26, 40])
    chunk, base, hq, hkv, H, d, T, k_sel, lam, tau = 4, 1e4, 4, 2, 2, 8, 3, 2, 0.7, 0.2
    dco, _ = O.chunk_layout(off_tok, chunk)
    C = int(dco[-1])
    k, v = r.standard_normal((40, hkv, d)), r.standard_normal((40, hkv, d))
    kr = r.standard_normal((40, H, d))
    qr, q = r.standard_normal((1, T, H, d)), r.standard_normal((T, hq, d))
    lk, lv = r.standard_normal((T, hkv, d)), r.standard_normal((T, hkv, d))
    W = r.standard_normal((T, hq, d))
    ev = [[1, 3]]
    kb0, vb0, krb0 = O.encode_memory(k, v, kr, off_tok, chunk, base)
    idx = O.topk_docs(O.route(krb0, dco, qr)[0], k_sel)[0][0]        # selection held fixed

    def loss(k_, v_, kr_):
        kb, vb, krb = O.encode_memory(k_, v_, kr_, off_tok, chunk, base)
        mem = O.gather_memory(np.stack([kb, vb], 1), dco, idx)
        o = O.sparse_attention(q, mem[:, 0], mem[:, 1], lk, lv, 0, 1 / np.sqrt(d))
        return float((W * o).sum() + lam * O.router_aux_loss(O.route(krb, dco, qr)[0], ev, tau)[0])

    mem = O.gather_memory(np.stack([kb0, vb0], 1), dco, idx)
    _, dmk, dmv, _, _ = O.sparse_attention_backward(q, mem[:, 0], mem[:, 1], lk, lv, 0, 1 / np.sqrt(d), W)
    dbar = O.gather_memory_backward(np.stack([dmk, dmv], 1), dco, idx, C)
    _, g_aux = O.router_aux_loss(O.route(krb0, dco, qr)[0], ev, tau)
    _, dkh = O.route_backward(krb0, dco, qr, lam * g_aux)
    dk, dv, dkr = O.encode_memory_backward(dbar[:, 0], dbar[:, 1], O.unit_backward(krb0, dkh), off_tok, chunk, base)
    for x, g, which in ((k, dk, 0), (v, dv, 1), (kr, dkr, 2)):
        def f(z, which=which):
            a = [k, v, kr]
            a[which] = z
            return loss(*a)
        i = r.choice(x.size, 12, replace=False)
        np.testing.assert_allclose(g.flat[i], _fd(f, x, i), atol=1e-7)


def test_three_term_bf16_split_of_fp32_is_exact():
    """The tensor-core best-token search of the router backward feeds the fp32 normalised queries as
    three bf16 terms (hi = bf16(x), mid = bf16(x - hi), lo = bf16(x - hi - mid), each difference exact
    in fp32): their sum gives x back exactly, so the bf16 tensor cores see the fp32 operand itself.
    Checked on normal values over several magnitudes, including the scale the folded queries have
    (unit heads divided by H)."""
    from msa_inputs import rng as R

    r = np.random.default_rng(21)
    for scale in (1.0, 1.0 / 8 / np.sqrt(128), 1e-3, 1e3):
        x = (r.standard_normal(1 << 18) * scale).astype(np.float32)
        hi = R.round_to(x, "bf16")
        r1 = (x - hi).astype(np.float32)
        mid = R.round_to(r1, "bf16")
        lo = R.round_to((r1 - mid).astype(np.float32), "bf16")
        np.testing.assert_array_equal(hi.astype(np.float64) + mid + lo, x.astype(np.float64))
