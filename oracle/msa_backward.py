"""fp64 CPU oracle of the MSA backward pass (gradients for end-to-end training).

TEST INFRASTRUCTURE, under the same rules as msa_oracle: only the tests, ``__graft_entry__.smoke()``
and the benchmark's CPU-baseline / reference arm may import or call it; the product path never does.

The pages state that routing, compression and attention are trained jointly in one gradient flow
([P1] 核心创新 端到端可训练性), with a weighted auxiliary loss that supervises every layer's router
toward the evidence documents ([P1] §训练策略 辅助损失; [P2] §训练层面). They give no formula for
that loss; the reading taken here is a softmax cross-entropy over the documents' router scores at
temperature tau, averaged over the query's evidence documents and over queries. The top-k itself
is a selection and carries no gradient: gradients reach the memory through the attention over the
selected documents and through the router scores of every document.

Each function is the chain rule of one forward step of msa_oracle, written out in fp64.
"""
from __future__ import annotations

import numpy as np

from .msa_oracle import F64, apply_rope, chunk_layout, doc_positions, unit


# ---------------------------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------------------------
def sparse_attention_backward(q, mem_k, mem_v, local_k, local_v, q_start: int, scale: float, dout):
    """Gradients of sparse_attention with respect to all its inputs, given dL/dout.

    For each query head h (kv head g = h // (hq / hkv)) with P = softmax(scale * q K^T) over the
    visible keys [mem ; local_j, j <= q_start + t]:
        dV = P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(dO * O)),  dq = scale dS K,  dK = scale dS^T q,
    the kv-head gradients summed over the heads that share it.
    Returns (dq [T, hq, d], dmem_k [M, hkv, d], dmem_v, dlocal_k [L, hkv, d], dlocal_v).
    """
    q = np.asarray(q, dtype=F64)
    dout = np.asarray(dout, dtype=F64)
    mem_k, mem_v = np.asarray(mem_k, dtype=F64), np.asarray(mem_v, dtype=F64)
    local_k, local_v = np.asarray(local_k, dtype=F64), np.asarray(local_v, dtype=F64)
    T, hq, d = q.shape
    hkv = local_k.shape[1] if local_k.shape[0] else mem_k.shape[1]
    group = hq // hkv
    M, L = mem_k.shape[0], local_k.shape[0]
    dq = np.zeros_like(q)
    dk = np.zeros((M + L, hkv, d), dtype=F64)
    dv = np.zeros((M + L, hkv, d), dtype=F64)
    visible = np.ones((T, M + L), dtype=bool)
    j = np.arange(L)
    for t in range(T):
        visible[t, M:] = j <= q_start + t
    for h in range(hq):
        g = h // group
        keys = np.concatenate([mem_k[:, g], local_k[:, g]], axis=0)
        vals = np.concatenate([mem_v[:, g], local_v[:, g]], axis=0)
        logits = np.where(visible, (q[:, h] @ keys.T) * scale, -np.inf)
        m = logits.max(axis=1, keepdims=True)
        m = np.where(np.isfinite(m), m, 0.0)
        p = np.exp(logits - m)
        den = p.sum(axis=1, keepdims=True)
        p = np.where(den > 0, p / np.where(den > 0, den, 1.0), 0.0)
        o = p @ vals
        do = dout[:, h]
        dv[:, g] += p.T @ do
        dp = do @ vals.T
        ds = p * (dp - (do * o).sum(axis=1, keepdims=True))
        dq[:, h] = scale * (ds @ keys)
        dk[:, g] += scale * (ds.T @ q[:, h])
    return dq, dk[:M], dv[:M], dk[M:], dv[M:]


# ---------------------------------------------------------------------------------------------
# fetch, pooling, RoPE, normalisation
# ---------------------------------------------------------------------------------------------
def gather_memory_backward(dmem: np.ndarray, doc_chunk_off: np.ndarray, idx, n_chunks: int) -> np.ndarray:
    """Adjoint of gather_memory: the gradient rows of the concatenated memory go back to the chunk
    rows they were copied from, summed where a chunk was fetched more than once."""
    dmem = np.asarray(dmem, dtype=F64)
    out = np.zeros((n_chunks,) + dmem.shape[1:], dtype=F64)
    at = 0
    for i in idx:
        a, b = int(doc_chunk_off[i]), int(doc_chunk_off[i + 1])
        out[a:b] += dmem[at:at + b - a]
        at += b - a
    return out


def pool_chunks_backward(dbar: np.ndarray, doc_tok_off: np.ndarray, chunk: int) -> np.ndarray:
    """Adjoint of pool_chunks: every token of chunk c receives dbar[c] / (tokens in c)."""
    dbar = np.asarray(dbar, dtype=F64)
    _, bounds = chunk_layout(doc_tok_off, chunk)
    out = np.zeros((int(doc_tok_off[-1]),) + dbar.shape[1:], dtype=F64)
    for c, (a, b) in enumerate(bounds):
        out[a:b] = dbar[c] / (b - a)
    return out


def apply_rope_backward(dy: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Adjoint of apply_rope: a rotation's transpose is the rotation by the opposite angle."""
    return apply_rope(dy, -np.asarray(pos, dtype=np.int64), base)


def encode_memory_backward(dkbar, dvbar, dkrbar, doc_tok_off, chunk: int, base: float):
    """Token gradients of encode_memory: dK = RoPE^T(pool^T(dK-bar)) at document positions,
    dV = pool^T(dV-bar), dK^R = pool^T(dK-bar^R). Any input may be None."""
    dk = None if dkbar is None else apply_rope_backward(pool_chunks_backward(dkbar, doc_tok_off, chunk),
                                                        doc_positions(doc_tok_off), base)
    dv = None if dvbar is None else pool_chunks_backward(dvbar, doc_tok_off, chunk)
    dkr = None if dkrbar is None else pool_chunks_backward(dkrbar, doc_tok_off, chunk)
    return dk, dv, dkr


def unit_backward(x: np.ndarray, dy: np.ndarray) -> np.ndarray:
    """Gradient of unit(x) = x / |x| over the last axis: (dy - y (y . dy)) / |x|; 0 for a zero x."""
    x = np.asarray(x, dtype=F64)
    dy = np.asarray(dy, dtype=F64)
    n = np.linalg.norm(x, axis=-1, keepdims=True)
    y = unit(x)
    g = dy - y * (y * dy).sum(axis=-1, keepdims=True)
    return np.where(n > 0, g / np.where(n > 0, n, 1.0), 0.0)


# ---------------------------------------------------------------------------------------------
# router auxiliary loss and the router's gradient
# ---------------------------------------------------------------------------------------------
def router_aux_loss(doc_scores: np.ndarray, evidence, tau: float):
    """Auxiliary router loss (reading of [P1] §训练策略 辅助损失): for query q with evidence documents
    E_q, loss_q = -(1/|E_q|) sum_{e in E_q} log softmax(s_q / tau)_e; the loss is the mean over
    queries. Returns (loss, dL/ds [n_q, D])."""
    s = np.atleast_2d(np.asarray(doc_scores, dtype=F64)) / tau
    n_q = s.shape[0]
    m = s.max(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.exp(s - m).sum(axis=1))
    p = np.exp(s - lse[:, None])
    loss, grad = 0.0, np.empty_like(s)
    for q in range(n_q):
        e = np.asarray(evidence[q], dtype=np.int64)
        loss += -(s[q, e] - lse[q]).mean()
        y = np.zeros(s.shape[1])
        np.add.at(y, e, 1.0 / len(e))
        grad[q] = (p[q] - y) / tau / n_q
    return loss / n_q, grad


def route_argmax(kr_index: np.ndarray, doc_chunk_off: np.ndarray, qr: np.ndarray, index_is_unit: bool = False):
    """For every (query, document): the chunk c and query token t where the document's score
    max_c max_t mean_h cos is attained (the lowest chunk, then the lowest token, on exact ties;
    -1 for a document without chunks). With index_is_unit the key vectors are taken as stored
    (the index form, already normalised once) instead of being normalised again."""
    qh = unit(np.asarray(qr, dtype=F64))                  # [n_q, T, H, d]
    kh = np.asarray(kr_index, dtype=F64) if index_is_unit else unit(np.asarray(kr_index, dtype=F64))
    H = kh.shape[1]
    D = len(doc_chunk_off) - 1
    n_q = qh.shape[0]
    arg_c = np.full((n_q, D), -1, dtype=np.int64)
    arg_t = np.full((n_q, D), -1, dtype=np.int64)
    for q in range(n_q):
        m = np.einsum("thd,chd->tc", qh[q], kh) / H        # [T, C] mean over heads of the cosines
        for i in range(D):
            a, b = int(doc_chunk_off[i]), int(doc_chunk_off[i + 1])
            if b > a:
                c = a + int(np.argmax(m[:, a:b].max(axis=0)))
                arg_c[q, i], arg_t[q, i] = c, int(np.argmax(m[:, c]))
    return arg_c, arg_t


def route_backward(kr_index: np.ndarray, doc_chunk_off: np.ndarray, qr: np.ndarray, d_doc_scores: np.ndarray,
                   index_is_unit: bool = False):
    """Gradients of the router's document scores (msa_oracle.route) given dL/d doc score.

    The max over chunks and tokens passes the gradient to the attaining pair only; there
    score = (1/H) sum_h <q_hat_h, k_hat_h>, so dq_hat_h = ds k_hat_h / H and dk_hat_h = ds q_hat_h / H.
    Returns (dqr [n_q, T, H, d], the gradient with respect to the raw router queries, through their
    normalisation; dk_hat [C, H, d], the gradient with respect to the unit key vectors k_hat =
    unit(kr_index); unit_backward(kr_index, dk_hat) carries it to kr_index itself). With index_is_unit
    the stored index vectors are the k_hat themselves (how the index form is scored: a dot product
    with vectors normalised once and stored), which also decides the attaining chunks."""
    qr = np.asarray(qr, dtype=F64)
    ds = np.atleast_2d(np.asarray(d_doc_scores, dtype=F64))
    qh = unit(qr)
    kh = np.asarray(kr_index, dtype=F64) if index_is_unit else unit(np.asarray(kr_index, dtype=F64))
    H = kh.shape[1]
    arg_c, arg_t = route_argmax(kr_index, doc_chunk_off, qr, index_is_unit)
    dqh = np.zeros_like(qh)
    dkh = np.zeros_like(kh)
    for q in range(ds.shape[0]):
        for i in range(ds.shape[1]):
            c, t = arg_c[q, i], arg_t[q, i]
            if c < 0:
                continue
            dqh[q, t] += ds[q, i] * kh[c] / H
            dkh[c] += ds[q, i] * qh[q, t] / H
    return unit_backward(qr, dqh), dkh
