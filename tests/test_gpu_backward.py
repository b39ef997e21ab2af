"""Backward pass of the CUDA path (through the C ABI) against the fp64 backward oracle: attention,
fetch, pooling with document-wise RoPE and index normalisation, the auxiliary router loss, the
router's gradient, and the chained training loss on a 64K-token training context."""
import numpy as np
import pytest
import torch

import oracle as O
from msa_inputs import rng, workloads
from msa_inputs.device import memory_tensor, small_tensors, upload

pytestmark = pytest.mark.gpu

SEED = 0xBAC4


@pytest.fixture(scope="module")
def m():
    import routed_long_context_b200 as m

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _gen(tid, shape, dtype="f32", sigma=1.0):
    return rng.normal(SEED, tid, 0, int(np.prod(shape)), sigma, dtype).reshape(shape)


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def _rel(got, ref):
    """Relative Frobenius error of a whole gradient tensor."""
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))


# The bf16 attention backward rounds P and dS to bf16 as tensor-core operands and takes
# D = rowsum(dO * O) from the bf16 forward output; everything else is fp32. Per gradient tensor
# that stays within 1e-2 of the exact result in relative Frobenius norm (the second check).
ATTN_BWD_TOL = 1e-2
# Per gradient row (a key's dK or dV, a (token, head)'s dq), the first check. Each bf16-rounded
# operand (P, dS) carries a relative error of at most u = 2^-8 (bf16 keeps 8 significant bits), and
# D_t = dO_t . O_t inherits the forward output's error: |dD_t| <= |dO_t| |O_t(GPU) - O_t| by
# Cauchy-Schwarz (the forward's deviation from the oracle, measured in the test; plus fp32 rounding).
# By the triangle inequality a row's error is then at most
#   dV_j : u sum_t P_tj |dO_t|
#   dK_j : scale sum_t (u |dS_tj| + P_tj |dD_t|) |q_t|,   dq_t : scale sum_j (u |dS_tj| + P_tj |dD_t|) |k_j|
# (summed over the heads that share a kv head), to first order; the rows are held to twice that
# (second-order terms, fp32 accumulation over up to ~10^4 terms).
BF16_U = 2.0 ** -8


def attn_bwd_row_bounds(q, mem_k, mem_v, local_k, local_v, q_start, scale, dout, d_err):
    """First-order error bound of every gradient row of the sparse-attention backward (fp64):
    (dq [T, hq], dmem_k [M, hkv], dmem_v, dlocal_k [L, hkv], dlocal_v); d_err [T, hq] bounds |dD|."""
    q, dout = np.asarray(q, np.float64), np.asarray(dout, np.float64)
    T, hq, d = q.shape
    hkv = local_k.shape[1] if local_k.shape[0] else mem_k.shape[1]
    G = hq // hkv
    M, L = mem_k.shape[0], local_k.shape[0]
    bq, bk, bv = np.zeros((T, hq)), np.zeros((M + L, hkv)), np.zeros((M + L, hkv))
    vis = np.ones((T, M + L), dtype=bool)
    for t in range(T):
        vis[t, M:] = np.arange(L) <= q_start + t
    for h in range(hq):
        g = h // G
        keys = np.concatenate([mem_k[:, g], local_k[:, g]]).astype(np.float64)
        vals = np.concatenate([mem_v[:, g], local_v[:, g]]).astype(np.float64)
        lg = np.where(vis, (q[:, h] @ keys.T) * scale, -np.inf)
        p = np.exp(lg - lg.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        o, do = p @ vals, dout[:, h]
        ds = p * (do @ vals.T - (do * o).sum(axis=1, keepdims=True))
        wgt = BF16_U * np.abs(ds) + p * d_err[:, h][:, None]
        bq[:, h] = scale * (wgt @ np.linalg.norm(keys, axis=1))
        bk[:, g] += scale * (wgt.T @ np.linalg.norm(q[:, h], axis=1))
        bv[:, g] += BF16_U * (p.T @ np.linalg.norm(do, axis=1))
    return bq, bk[:M], bv[:M], bk[M:], bv[M:]


def forward_d_error(out_gpu, out_ref, dout):
    """Bound on |D_t(GPU) - D_t| per (token, head): |dO_t| |O_t(GPU) - O_t| + fp32 rounding."""
    dn = np.linalg.norm(np.asarray(dout, np.float64), axis=-1)
    return dn * np.linalg.norm(out_gpu - out_ref, axis=-1) + 2.0 ** -20 * dn * np.linalg.norm(out_ref, axis=-1)


def assert_rows_within(got, ref, bound, factor, what):
    """Every row (last axis) of got within factor * bound[row] of ref."""
    err = np.linalg.norm(got - ref, axis=-1)
    worst = float((err / np.maximum(bound, 1e-300)).max()) if err.size else 0.0
    assert np.all(err <= factor * bound), (what, worst, factor)


@pytest.mark.parametrize("impl", [0, 2, 3])
@pytest.mark.parametrize("hq,hkv", [(32, 8), (8, 8), (32, 4)])
@pytest.mark.parametrize("T,max_mem,mem_lens,q_start", [(13, 40, (0, 5, 37), 7), (64, 140, (130, 64, 1), 0),
                                                        (100, 300, (256, 300, 77), 20)])
def test_attention_backward_matches_oracle(m, impl, hq, hkv, T, max_mem, mem_lens, q_start):
    """impl 0: tcgen05 (forward split and dQ), impl 2: mma.sync throughout, impl 3: dK/dV on tcgen05 too."""
    n_q, d, dt = 3, 128, "bf16"
    L = q_start + T
    q = _gen(1, (n_q, T, hq, d), dt)
    mem = _gen(2, (n_q, max_mem, 2, hkv, d), dt)
    lk, lv = _gen(3, (n_q, L + 3, hkv, d), dt), _gen(4, (n_q, L + 3, hkv, d), dt)
    dout = _gen(5, (n_q, T, hq, d), dt)
    mem_len = torch.from_numpy(np.array(mem_lens, dtype=np.int32)).cuda()
    qd, memd, lkd, lvd, dod = (upload(x, dt) for x in (q, mem, lk, lv, dout))
    lse = torch.empty((n_q, T, hq), dtype=torch.float32, device="cuda")
    m.attn_set_impl(impl)
    try:
        out = m.msa_sparse_attn_split(qd, memd, mem_len, lkd, lvd, L, q_start, lse=lse)
        dq, dmem, dlk, dlv = m.msa_sparse_attn_backward(qd, memd, mem_len, lkd, lvd, L, q_start, out, dod, lse)
    finally:
        m.attn_set_impl(0)
    assert m.device_status() == 0
    scale = 1 / np.sqrt(d)
    for qi in range(n_q):
        ml = mem_lens[qi]
        ref = O.sparse_attention_backward(q[qi], mem[qi, :ml, 0], mem[qi, :ml, 1], lk[qi, :L], lv[qi, :L], q_start,
                                          scale, dout[qi])
        got = (_np(dq[qi]), _np(dmem[qi, :ml, 0]), _np(dmem[qi, :ml, 1]), _np(dlk[qi, :L]), _np(dlv[qi, :L]))
        o_ref = O.sparse_attention(q[qi], mem[qi, :ml, 0], mem[qi, :ml, 1], lk[qi, :L], lv[qi, :L], q_start, scale)
        d_err = forward_d_error(_np(out[qi]), o_ref, dout[qi])
        bounds = attn_bwd_row_bounds(q[qi], mem[qi, :ml, 0], mem[qi, :ml, 1], lk[qi, :L], lv[qi, :L], q_start, scale,
                                     dout[qi], d_err)
        for name, g, r, b in zip(("dq", "dmem_k", "dmem_v", "dlocal_k", "dlocal_v"), got, ref, bounds):
            if r.size:
                assert_rows_within(g, r, b, 2.0, (qi, name))
                assert _rel(g, r) <= ATTN_BWD_TOL, (qi, name, _rel(g, r))
        # log-sum-exp of the forward rows
        o_lse = []
        for h in range(hq):
            g_ = h // (hq // hkv)
            keys = np.concatenate([mem[qi, :ml, 0, g_], lk[qi, :L, g_]])
            lg = (q[qi, :, h] @ keys.T) * scale
            vis = np.ones_like(lg, dtype=bool)
            vis[:, ml:] = np.arange(L)[None, :] <= q_start + np.arange(T)[:, None]
            lg = np.where(vis, lg, -np.inf)
            mx = lg.max(axis=1)
            o_lse.append(mx + np.log(np.exp(lg - mx[:, None]).sum(axis=1)))
        np.testing.assert_allclose(_np(lse[qi]), np.stack(o_lse, axis=1), atol=2e-3)


def test_gather_backward_sums_rows_of_documents_fetched_twice(m):
    counts = np.array([3, 1, 4, 0, 2, 5], dtype=np.int64)
    off = np.concatenate([[0], np.cumsum(counts)])
    C = int(off[-1])
    idx = np.array([[2, 0, 5], [5, 1, 2]], dtype=np.int32)           # documents 2 and 5 twice
    dmem = _gen(6, (2, 14, 2, 8, 128))
    got = m.msa_gather_kv_backward(torch.from_numpy(dmem).float().cuda(), torch.from_numpy(off).cuda(),
                                   torch.from_numpy(idx).cuda(), C)
    assert m.device_status() == 0
    ref = sum(O.gather_memory_backward(dmem[q], off, idx[q].tolist(), C) for q in range(2))
    np.testing.assert_allclose(_np(got), ref, rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("kr_dt,chunk,parts", [("f32", 128, "both"), ("bf16", 128, "both"), ("bf16", 96, "kv"),
                                               ("bf16", 96, "kr"), ("f32", 1, "both"), ("bf16", 200, "both")])
def test_pool_backward_matches_oracle(m, kr_dt, chunk, parts):
    """Token gradients of pooling: keys through the transposed document-wise rotation, values, and
    router keys through the index normalisation; ragged documents (one empty), chunks that end
    inside a token slice, and either group of gradients alone."""
    from routed_long_context_b200.bank import BankLayout

    lens = np.array([300, 0, 255, 129, 1000, 1], dtype=np.int64)
    hkv, hr, d, base = 8, 8, 128, 1e6
    lay = BankLayout.from_doc_lengths(lens, chunk)
    n = int(lay.doc_tok_off_host[-1])
    C = lay.n_chunks
    kr = _gen(7, (n, hr, d), kr_dt)
    dkv = _gen(8, (C, 2, hkv, d))
    dki = _gen(9, (C, hr, d))
    cs = m.rope_table(2048, d, base)
    g_kv = torch.from_numpy(dkv).float().cuda() if parts in ("both", "kv") else None
    g_kr = torch.from_numpy(dki).float().cuda() if parts in ("both", "kr") else None
    dk, dv, dkr = m.msa_pool_chunks_backward(g_kv, g_kr, lay.doc_tok_off, lay.doc_chunk_off, lay.chunk_doc, chunk, n,
                                             kr=upload(kr, kr_dt), cos_sin=cs)
    assert m.device_status() == 0
    _, _, krb = O.encode_memory(None, None, kr, lay.doc_tok_off_host, chunk, base)
    rk, rv, rkr = O.encode_memory_backward(dkv[:, 0], dkv[:, 1], O.unit_backward(krb, dki), lay.doc_tok_off_host,
                                           chunk, base)
    if g_kv is not None:
        np.testing.assert_allclose(_np(dk), rk, rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(_np(dv), rv, rtol=1e-6, atol=1e-7)
    else:
        assert dk is None and dv is None
    if g_kr is not None:
        np.testing.assert_allclose(_np(dkr), rkr, rtol=1e-4, atol=1e-6)
    else:
        assert dkr is None


@pytest.mark.parametrize("n_q,D,tau", [(3, 1000, 0.1), (2, 97657, 0.05)])
def test_aux_loss_matches_oracle(m, n_q, D, tau):
    s = np.clip(_gen(10, (n_q, D)) * 0.3, -1, 1).astype(np.float32)
    ev = np.full((n_q, 3), -1, dtype=np.int32)
    ev[0, :2] = [5, D - 1]
    ev[1, :1] = [17]
    if n_q > 2:
        ev[2] = [0, 1, 2]
    loss, grad = m.msa_router_aux_loss(torch.from_numpy(s).cuda(), torch.from_numpy(ev), tau)
    assert m.device_status() == 0
    rl, rg = O.router_aux_loss(s, [[e for e in row if e >= 0] for row in ev], tau)
    assert abs(float(loss.mean()) - rl) <= 1e-4 * max(1.0, abs(rl))
    np.testing.assert_allclose(_np(grad), rg, rtol=1e-3, atol=1e-7 / n_q)


@pytest.mark.parametrize("dt,impl,n_docs,T", [("f32", 0, 40, 17), ("bf16", 0, 40, 17), ("bf16", 1, 40, 17),
                                              ("bf16", 0, 300, 70), ("bf16", 1, 300, 70), ("bf16", 0, 3, 64)])
def test_route_backward_matches_oracle(m, dt, impl, n_docs, T):
    """The index is built on the host (unit vectors rounded to dt) and both sides score those stored
    values as they are, so they find the same attaining (chunk, token) pairs. bf16 runs the best-token
    search on the tensor cores (impl 0: chunk tiles of 128, token tiles of 32, padded token rows) or on
    CUDA cores (impl 1). Query 0 repeats token 3 at token 9 and at token T-2, so its scores tie exactly
    within a token tile and across tiles: the first token must take the gradient."""
    r = np.random.default_rng(12)
    counts = r.integers(0, 13, n_docs)
    counts[0] = max(counts[0], 1)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    C, H, d, n_q = int(off[-1]), 8, 128, 2
    index = rng.round_to(O.unit(_gen(11, (C, H, d))).astype(np.float32), dt).astype(np.float64)
    qr = _gen(13, (n_q, T, H, d), dt)
    qr[0, 9] = qr[0, 3]
    qr[0, T - 2] = qr[0, 3]
    # chunk 0 is attained by the repeated token
    index[0] = rng.round_to(O.unit(qr[0, 3]).astype(np.float32), dt)
    ds = _gen(14, (n_q, n_docs))
    m.route_set_impl(impl)
    try:
        dqr, dkh = m.msa_route_backward(upload(index, dt), torch.from_numpy(off).cuda(), upload(qr, dt),
                                        torch.from_numpy(ds).float().cuda())
        assert m.device_status() == 0
    finally:
        m.route_set_impl(0)
    rq, rk = O.route_backward(index, off, qr, ds, index_is_unit=True)
    # fp32 on both sides from the same stored index. Per row (a query token's head, a chunk's head):
    # the error is a few fp32 roundings of the row's terms before the normalisation's transpose, which
    # divides by |Q^R_{t,h}| and can cancel almost all of a row (the planted chunk is token 3's own
    # query): bound = 1e-5 x (sum of the row's |terms|) [/ |Q^R_{t,h}|] + 1e-4 x |row|; a row that
    # no (query, document) attains stays exactly zero
    arg_c, arg_t = O.route_argmax(index, off, qr, index_is_unit=True)
    qh = O.unit(qr.astype(np.float64))
    mq, mk = np.zeros(qr.shape[:3]), np.zeros(index.shape[:2])
    for qi in range(n_q):
        for i in range(n_docs):
            c_, t_ = arg_c[qi, i], arg_t[qi, i]
            if c_ >= 0:
                mq[qi, t_] += abs(ds[qi, i]) * np.linalg.norm(index[c_], axis=-1) / H
                mk[c_] += abs(ds[qi, i]) * np.linalg.norm(qh[qi, t_], axis=-1) / H
    bq = 1e-5 * mq / np.linalg.norm(qr.astype(np.float64), axis=-1) + 1e-4 * np.linalg.norm(rq, axis=-1)
    assert_rows_within(_np(dqr), rq, bq, 1.0, "dqr")
    assert_rows_within(_np(dkh), rk, 1e-5 * mk + 1e-4 * np.linalg.norm(rk, axis=-1), 1.0, "dk_hat")
    assert _rel(_np(dqr), rq) <= 1e-4 and _rel(_np(dkh), rk) <= 1e-4
    g = _np(dqr)
    assert np.abs(g[0, 3]).max() > 0 and np.abs(g[0, 9]).max() == 0 and np.abs(g[0, T - 2]).max() == 0


def test_training_loss_gradients_on_a_64k_context(m):
    """L = <W, attention output> + lam * aux(router scores) on the train64k context, selection held at
    the GPU's top-k: the chained library calls (encode, route, top-k, fetch, split attention with
    log-sum-exp; attention backward, fetch backward, aux loss, router backward, pooling backward) give
    the token gradients of K, V and K^R of the chained backward oracle."""
    from routed_long_context_b200.bank import BankLayout, encode_tokens

    w = workloads.train64k()
    lay = BankLayout.from_doc_lengths(w.doc_len, w.chunk)
    cs = m.rope_table(8192, w.d, w.rope_base)
    k, v, kr = (memory_tensor(w, 0, n) for n in ("k", "v", "kr"))
    kvbar, index = encode_tokens(lay, k, v, kr, w.chunk, cs)
    sm = small_tensors(w, 0)
    T, lam, tau = w.T0, 0.5, 1.0
    ds = m.msa_route_scores(index, lay.chunk_doc, lay.n_docs, sm["qr"])
    idx, _ = m.msa_topk_docs(ds, w.k)
    max_mem = w.k * int(w.doc_chunks.max())
    mem, mem_len = m.msa_gather_kv_device(kvbar, lay.doc_chunk_off, idx, max_mem)
    seg = torch.tensor([0, T], dtype=torch.int64, device="cuda")
    lk = m.msa_rope_doc(sm["k_new"][0], seg, w.k, cs, out=torch.empty_like(sm["k_new"][0]))
    qq = m.msa_rope_doc(sm["q"][0], seg, w.k, cs, out=torch.empty_like(sm["q"][0]))
    lse = torch.empty((1, T, w.hq), dtype=torch.float32, device="cuda")
    out = m.msa_sparse_attn_split(qq[None], mem, mem_len, lk[None], sm["v_new"], T, 0, lse=lse)
    W = _gen(15, (1, T, w.hq, w.d), "bf16")
    _, dmem, _, _ = m.msa_sparse_attn_backward(qq[None], mem, mem_len, lk[None], sm["v_new"], T, 0, out,
                                               upload(W, "bf16"), lse)
    dkvbar = m.msa_gather_kv_backward(dmem, lay.doc_chunk_off, idx, lay.n_chunks)
    evidence = np.array([w.expected(0, 0, 0)], dtype=np.int32)
    _, g_aux = m.msa_router_aux_loss(ds, torch.from_numpy(evidence), tau)
    _, dkhat = m.msa_route_backward(index, lay.doc_chunk_off, sm["qr"], g_aux * lam)
    dk, dv, dkr = m.msa_pool_chunks_backward(dkvbar, dkhat, lay.doc_tok_off, lay.doc_chunk_off, lay.chunk_doc, w.chunk,
                                             w.n_tok, kr=kr, cos_sin=cs)
    assert m.device_status() == 0
    gi = idx.cpu().numpy()[0]
    assert set(evidence[0].tolist()) <= set(gi.tolist())

    # the chained oracle; the pooled memory rows, the rotated local queries and keys and the router
    # index enter it as stored (rounded to bf16, the storage precision of the path), so both sides
    # attend and route over the same values
    bf = lambda x: rng.round_to(np.asarray(x, np.float32), "bf16").astype(np.float64)
    kh, vh, krh = (w.host_tensor(0, n) for n in ("k", "v", "kr"))
    kb, vb, krb = O.encode_memory(kh, vh, krh, w.doc_tok_off, w.chunk, w.rope_base)
    qr = w.qr(0)
    memo = O.gather_memory(np.stack([bf(kb), bf(vb)], 1), w.doc_chunk_off, gi)
    pos = O.global_positions(w.k, 0, T)
    scale = 1 / np.sqrt(w.d)
    attn_in = (bf(O.apply_rope(w.q(0)[0], pos, w.rope_base)), memo[:, 0], memo[:, 1],
               bf(O.apply_rope(w.k_new(0)[0], pos, w.rope_base)), w.v_new(0)[0], 0, scale)
    _, dmk, dmv, _, _ = O.sparse_attention_backward(*attn_in, W[0])
    dbar = O.gather_memory_backward(np.stack([dmk, dmv], 1), w.doc_chunk_off, gi, w.n_chunks)
    stored = bf(O.unit(krb))                                                  # the index's stored form
    ref_ds, _ = O.route(stored, w.doc_chunk_off, qr)
    _, g = O.router_aux_loss(ref_ds, [evidence[0].tolist()], tau)
    _, dkh = O.route_backward(stored, w.doc_chunk_off, qr, lam * g, index_is_unit=True)
    rk, rv, rkr = O.encode_memory_backward(dbar[:, 0], dbar[:, 1], O.unit_backward(krb, dkh), w.doc_tok_off, w.chunk,
                                           w.rope_base)
    assert _rel(_np(dk), rk) <= ATTN_BWD_TOL
    assert _rel(_np(dv), rv) <= ATTN_BWD_TOL
    assert _rel(_np(dkr), rkr) <= ATTN_BWD_TOL

    # per token row. dK and dV: the chunk's bound from the attention rows of its fetched copies,
    # divided by the chunk's token count (the pooling's transpose; the rotation keeps norms)
    d_err = forward_d_error(_np(out[0]), O.sparse_attention(*attn_in), W[0])
    _, bmk, bmv, _, _ = attn_bwd_row_bounds(*attn_in, W[0], d_err)
    bbar = O.gather_memory_backward(np.stack([bmk, bmv], 1)[..., None], w.doc_chunk_off, gi, w.n_chunks)[..., 0]
    _, cb = O.chunk_layout(w.doc_tok_off, w.chunk)
    tok_chunk = np.repeat(np.arange(len(cb)), cb[:, 1] - cb[:, 0])
    n_c = (cb[:, 1] - cb[:, 0])[tok_chunk][:, None]
    for name, got_, ref_, b in (("dk", dk, rk, bbar[:, 0]), ("dv", dv, rv, bbar[:, 1])):
        assert_rows_within(_np(got_), ref_, 2 * b[tok_chunk] / n_c + 1e-5 * np.linalg.norm(ref_, axis=-1), 1.0, name)
    # dK^R: the only difference between the sides is the forward scores (bf16 queries in the
    # router's contraction), |ds(GPU) - ds| <= eps; through the softmax |dg_d| <= 2 p_d eps / (tau^2 n_q),
    # a chunk's dk_hat per head moves by lam sum_q |dg| / H, the normalisation's transpose divides by
    # |K-bar^R_{c,h}| and the pooling's by the chunk's token count (fp32 elsewhere: 1e-5 relative)
    eps = float(np.abs(_np(ds) - ref_ds).max())
    assert eps <= 2e-3
    sq = ref_ds / tau
    p_soft = np.exp(sq - sq.max(axis=1, keepdims=True))
    p_soft /= p_soft.sum(axis=1, keepdims=True)
    dg = 2 * p_soft * eps / (tau * tau * ref_ds.shape[0])                    # [n_q, D]
    arg_c, _ = O.route_argmax(stored, w.doc_chunk_off, qr, index_is_unit=True)
    bh = np.zeros(w.n_chunks)
    for qi in range(arg_c.shape[0]):
        np.add.at(bh, arg_c[qi][arg_c[qi] >= 0], lam * dg[qi][arg_c[qi] >= 0] / w.H)
    bkr = bh[:, None] / np.linalg.norm(krb, axis=-1)                          # [C, H]
    assert_rows_within(_np(dkr), rkr, 2 * bkr[tok_chunk] / n_c + 1e-5 * np.linalg.norm(rkr, axis=-1), 1.0, "dkr")
