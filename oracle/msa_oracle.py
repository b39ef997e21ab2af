"""fp64 CPU oracle of the Memory Sparse Attention (MSA) hot path.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference arm may import or call this module. The
product path (``routed_long_context_b200``) never imports it and shares no code,
header, table or helper with it; the two meet only through the seeded inputs of
``msa_inputs``.

Everything is plain numpy in float64: inputs (fp32 or bf16 values) are
converted to fp64 exactly and every step follows the definition on the pages,
in their order, with no blocking, fusion or reordering beyond slicing memory
chunks into independent groups (each chunk's score depends on that chunk
alone).

Sources, cited by tag below (web pages about the MSA paper, Chen et al.,
"MSA: Memory Sparse Attention for Efficient End-to-End Memory Model Scaling to
100M Tokens", EverMind / Shanda / Peking University):
  [P1] Lighthouse AI-research news digest, "MSA: Memory Sparse Attention for
       Efficient End-to-End Memory Model Scaling to 100M Tokens" (2026-03-27)
  [P2] hotdry blog, "EverMind MSA router sparse attention architecture"
       (2026-03-24)
  [P3] gitcode/CSDN article on MSA (section "四大技术突破")
  [P5] wiselychen blog, "MSA: 4B 模型打贏 235B RAG 系統"

Readings of points the pages leave open (each also listed with its reason in
the design notes): rotate-half RoPE pairing with base 1e6; RoPE on keys and
queries only (not V, not the router vectors); RoPE before pooling; a ragged
last chunk is the mean of its real tokens; a document's score is the max over
its chunks; a zero-norm vector has cosine 0; top-k ties go to the lower
document index; the active context starts at global position k (the top-k
count); attention scale 1/sqrt(d), memory fully visible, local keys causal,
kv head = h // (hq / hkv); memory concatenated in rank order before local.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


# ---------------------------------------------------------------------------------------------
# RoPE: document-wise and global positions
# ---------------------------------------------------------------------------------------------
def rope_angles(pos: np.ndarray, d: int, base: float) -> np.ndarray:
    """theta[p, i] = p * base^(-2i/d) for i in [0, d/2)  ([P1] §组件 2 Document-wise RoPE)."""
    i = np.arange(d // 2, dtype=F64)
    omega = np.power(F64(base), -2.0 * i / d)
    return np.asarray(pos, dtype=F64)[:, None] * omega[None, :]


def apply_rope(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Rotate each vector x[n, ..., d] by its position pos[n] (rotate-half pairing i <-> i + d/2).

    x'_i       = x_i cos(p w_i) - x_{i+d/2} sin(p w_i)
    x'_{i+d/2} = x_{i+d/2} cos(p w_i) + x_i sin(p w_i)
    """
    x = np.asarray(x, dtype=F64)
    d = x.shape[-1]
    ang = rope_angles(pos, d, base)
    shape = (x.shape[0],) + (1,) * (x.ndim - 2) + (d // 2,)
    c = np.cos(ang).reshape(shape)
    s = np.sin(ang).reshape(shape)
    x1, x2 = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def doc_positions(doc_tok_off: np.ndarray) -> np.ndarray:
    """Position of every memory token inside its own document: restarts at 0 per document
    ([P1] §组件 2: each memory document gets position ids from 0; [P2] §工程实现的关键细节)."""
    doc_tok_off = np.asarray(doc_tok_off, dtype=np.int64)
    lens = np.diff(doc_tok_off)
    starts = np.repeat(doc_tok_off[:-1], lens)
    return np.arange(doc_tok_off[-1], dtype=np.int64) - starts


def global_positions(k: int, first: int, n: int) -> np.ndarray:
    """Active-context positions: query / generated token j of the local context sits at k + j,
    k being the top-k count ([P1] §组件 2 活跃上下文; [P2] offset by k retrieved blocks)."""
    return k + first + np.arange(n, dtype=np.int64)


# ---------------------------------------------------------------------------------------------
# chunk-mean pooling (KV-cache compression)
# ---------------------------------------------------------------------------------------------
def chunk_layout(doc_tok_off: np.ndarray, chunk: int):
    """Fixed-size chunks that never cross a document: (doc_chunk_off [D+1], bounds [C, 2]).

    Document i of length n_i holds ceil(n_i / chunk) chunks; chunk j covers tokens
    [s_i + j*chunk, min(s_i + (j+1)*chunk, e_i))  ([P2] §可学习记忆路由层的核心架构).
    """
    doc_tok_off = np.asarray(doc_tok_off, dtype=np.int64)
    bounds, counts = [], []
    for i in range(len(doc_tok_off) - 1):
        s, e = int(doc_tok_off[i]), int(doc_tok_off[i + 1])
        n = 0
        for a in range(s, e, chunk):
            bounds.append((a, min(a + chunk, e)))
            n += 1
        counts.append(n)
    doc_chunk_off = np.zeros(len(counts) + 1, dtype=np.int64)
    np.cumsum(counts, out=doc_chunk_off[1:])
    return doc_chunk_off, np.array(bounds, dtype=np.int64).reshape(-1, 2)


def pool_chunks(x: np.ndarray, doc_tok_off: np.ndarray, chunk: int) -> np.ndarray:
    """Mean of the tokens of every chunk: x[n_tok, ...] -> [C, ...]  ([P2] chunk-mean pooling)."""
    x = np.asarray(x, dtype=F64)
    _, bounds = chunk_layout(doc_tok_off, chunk)
    out = np.empty((len(bounds),) + x.shape[1:], dtype=F64)
    for c, (a, b) in enumerate(bounds):
        out[c] = x[a:b].mean(axis=0)
    return out


def encode_memory(k, v, kr, doc_tok_off, chunk: int, base: float):
    """Offline memory encoding: K-bar = pool(doc-wise RoPE(K)), V-bar = pool(V), K-bar^R = pool(K^R).

    ([P5] §3 inference stage 1 offline encoding; [P2] chunk-mean pooling of K, V and K^R;
    [P1] §组件 2 memory documents use document-wise positions.) Any of k, v, kr may be None.
    """
    out = []
    if k is not None:
        pos = doc_positions(doc_tok_off)
        out.append(pool_chunks(apply_rope(k, pos, base), doc_tok_off, chunk))
    else:
        out.append(None)
    out.append(pool_chunks(v, doc_tok_off, chunk) if v is not None else None)
    out.append(pool_chunks(kr, doc_tok_off, chunk) if kr is not None else None)
    return tuple(out)


def token_bank(k, v, doc_tok_off, base: float) -> np.ndarray:
    """Token-level memory of the fine stage: [n_tok, 2, hkv, d], row r = (K_r rotated to its position
    inside its own document, V_r). Coarse-to-fine reading of [P5] 四個核心機制 §1 (routing on the
    compressed chunks, then the selected documents' own tokens); the keys keep document-wise
    positions as in [P1] §组件 2."""
    pos = doc_positions(doc_tok_off)
    return np.stack([apply_rope(k, pos, base), np.asarray(v, dtype=F64)], axis=1)


# ---------------------------------------------------------------------------------------------
# router scoring
# ---------------------------------------------------------------------------------------------
def unit(x: np.ndarray) -> np.ndarray:
    """x / ||x|| over the last axis; a zero vector stays zero (so its cosine with anything is 0)."""
    x = np.asarray(x, dtype=F64)
    n = np.sqrt((x * x).sum(axis=-1, keepdims=True))
    return np.divide(x, n, out=np.zeros_like(x), where=n > 0)


def chunk_scores_one_query(krbar: np.ndarray, qr: np.ndarray) -> np.ndarray:
    """S_c = max over tokens t of mean over heads h of cos(Q^R_{t,h}, K-bar^R_{c,h}).

    krbar [C, H, d], qr [T, H, d] -> [C]. The mean over heads is taken first, then the max over
    query tokens ([P1] §组件 1 关键公式 and the sentence after it; [P2] mean-pooled over heads,
    then max over tokens).
    """
    kn = unit(krbar)                                   # [C, H, d]
    qn = unit(qr)                                      # [T, H, d]
    H = krbar.shape[1]
    cos = np.empty((qr.shape[0], krbar.shape[0], H), dtype=F64)    # [T, C, H]
    for h in range(H):                                 # cos of unit vectors = their dot product
        cos[:, :, h] = qn[:, h, :] @ kn[:, h, :].T
    mean_h = cos.mean(axis=2)                          # [T, C]
    return mean_h.max(axis=0)                          # [C]


def chunk_scores_folded(krbar: np.ndarray, qr: np.ndarray) -> np.ndarray:
    """The same scores in folded form: <concat_h(q_hat_h / H), concat_h(k_hat_h)>, max over t.

    Used only to check the identity mean_h cos = folded dot / H that the GPU path relies on.
    """
    H = krbar.shape[1]
    kf = unit(krbar).reshape(krbar.shape[0], -1)
    qf = (unit(qr) / H).reshape(qr.shape[0], -1)
    return (qf @ kf.T).max(axis=0)


def doc_scores_from_chunks(chunk_scores: np.ndarray, doc_chunk_off: np.ndarray) -> np.ndarray:
    """Score of document i = max of its chunks' scores (reading of [P1] 关键公式, which scores
    chunk j of document i, together with document-level top-k selection)."""
    doc_chunk_off = np.asarray(doc_chunk_off, dtype=np.int64)
    return np.array([chunk_scores[..., a:b].max(axis=-1) if b > a else -np.inf
                     for a, b in zip(doc_chunk_off[:-1], doc_chunk_off[1:])], dtype=F64).T


def route(krbar: np.ndarray, doc_chunk_off: np.ndarray, qr: np.ndarray, slice_chunks: int = 65536):
    """Router scores for every query: krbar [C, H, d], qr [n_q, T, H, d] ->
    (doc_scores [n_q, D], chunk_scores [n_q, C]).  Chunks are processed in independent slices."""
    qr = np.asarray(qr)
    C = krbar.shape[0]
    cs = np.empty((qr.shape[0], C), dtype=F64)
    for q in range(qr.shape[0]):
        for a in range(0, C, slice_chunks):
            b = min(C, a + slice_chunks)
            cs[q, a:b] = chunk_scores_one_query(krbar[a:b], qr[q])
    ds = np.stack([doc_scores_from_chunks(cs[q], doc_chunk_off) for q in range(cs.shape[0])])
    return ds, cs


# ---------------------------------------------------------------------------------------------
# top-k document selection
# ---------------------------------------------------------------------------------------------
def topk_docs(doc_scores: np.ndarray, k: int):
    """The k best documents per query, by descending score, ties to the lower index
    ([P1] §组件 1 选择 Top-k 文档; [P2] Top-k 选择机制)."""
    doc_scores = np.atleast_2d(np.asarray(doc_scores, dtype=F64))
    D = doc_scores.shape[1]
    idx = np.empty((doc_scores.shape[0], k), dtype=np.int64)
    val = np.empty((doc_scores.shape[0], k), dtype=F64)
    ids = np.arange(D)
    for q in range(doc_scores.shape[0]):
        order = np.lexsort((ids, -doc_scores[q]))     # primary: -score, secondary: index
        idx[q] = order[:k]
        val[q] = doc_scores[q, order[:k]]
    return idx, val


# ---------------------------------------------------------------------------------------------
# KV gather and sparse attention
# ---------------------------------------------------------------------------------------------
def gather_memory(kvbar: np.ndarray, doc_chunk_off: np.ndarray, idx) -> np.ndarray:
    """Compressed K-bar/V-bar rows [C, 2, hkv, d] of the selected docs, concatenated in rank order
    ([P1] §组件 1 将其压缩 KV 与查询的本地 KV 拼接; [P5] §3 content KV loaded after routing)."""
    parts = [kvbar[int(doc_chunk_off[i]):int(doc_chunk_off[i + 1])] for i in idx]
    return np.concatenate(parts, axis=0) if parts else kvbar[:0]


def sparse_attention(q, mem_k, mem_v, local_k, local_v, q_start: int, scale: float) -> np.ndarray:
    """Softmax attention of query tokens over [memory K-bar/V-bar ; local K/V].

    q [T, hq, d] (already rotated), mem_k/mem_v [M, hkv, d] (all visible), local_k/local_v
    [L, hkv, d]; query token t is local position q_start + t and sees local keys j <= q_start + t.
    kv head of query head h is h // (hq / hkv). ([P1] §组件 1 稀疏注意力; [P2] concatenation of the
    selected compressed K/V with the local K/V.)
    """
    q = np.asarray(q, dtype=F64)
    mem_k, mem_v = np.asarray(mem_k, dtype=F64), np.asarray(mem_v, dtype=F64)
    local_k, local_v = np.asarray(local_k, dtype=F64), np.asarray(local_v, dtype=F64)
    T, hq, d = q.shape
    hkv = local_k.shape[1] if local_k.shape[0] else mem_k.shape[1]
    group = hq // hkv
    L = local_k.shape[0]
    out = np.empty((T, hq, d), dtype=F64)
    for h in range(hq):
        g = h // group
        keys = np.concatenate([mem_k[:, g], local_k[:, g]], axis=0)       # [M + L, d]
        vals = np.concatenate([mem_v[:, g], local_v[:, g]], axis=0)
        M = mem_k.shape[0]
        logits = (q[:, h] @ keys.T) * scale                                # [T, M + L]
        visible = np.ones_like(logits, dtype=bool)
        j = np.arange(L)
        for t in range(T):
            visible[t, M:] = j <= q_start + t
        logits = np.where(visible, logits, -np.inf)
        m = logits.max(axis=1, keepdims=True)
        p = np.exp(logits - m)
        p /= p.sum(axis=1, keepdims=True)
        out[:, h] = p @ vals
    return out


# ---------------------------------------------------------------------------------------------
# one interleave round for one layer
# ---------------------------------------------------------------------------------------------
def route_and_attend(krbar, doc_chunk_off, kvbar, qr_active, q_new, k_local_raw, v_local, L_prev: int,
                     k: int, base: float, scale: float | None = None):
    """One routed layer for one query, in one Memory Interleave round.

    krbar [C, H, d] pooled router keys; kvbar [C, 2, hkv, d] pooled content (K-bar already
    document-wise rotated); qr_active [T_act, H, d] router queries of every active token;
    q_new [T_new, hq, d] raw queries of the tokens appended this round; k_local_raw/v_local
    [L_prev + T_new, hkv, d] raw keys / values of the whole active context.
    Route -> top-k -> gather -> attention with global positions starting at k
    ([P1] §组件 3 Memory Interleaving; [P2] re-route with the updated context each round;
    [P5] §4 生成式檢索 -> 上下文擴展 -> 生成 -> 再檢索).
    Returns (idx [k], doc scores of idx [k], output [T_new, hq, d]).
    """
    T_new = q_new.shape[0]
    d = q_new.shape[-1]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    ds, _ = route(krbar, doc_chunk_off, qr_active[None])
    idx, val = topk_docs(ds, k)
    mem = gather_memory(kvbar, doc_chunk_off, idx[0])
    L = L_prev + T_new
    k_local = apply_rope(k_local_raw[:L], global_positions(k, 0, L), base)
    q_rot = apply_rope(q_new, global_positions(k, L_prev, T_new), base)
    o = sparse_attention(q_rot, mem[:, 0], mem[:, 1], k_local, v_local[:L], L_prev, scale)
    return idx[0], val[0], o


def route_and_attend_fine(krbar, doc_chunk_off, tokbank, doc_tok_off, qr_active, q_new, k_local_raw, v_local,
                          L_prev: int, k: int, base: float, scale: float | None = None):
    """route_and_attend with the fine stage: routing and selection on the compressed chunks as
    before, then attention over the selected documents' token-level K/V (token_bank rows, in rank
    order) instead of their chunk means (coarse-to-fine reading of [P5] 四個核心機制 §1).
    Returns (idx [k], doc scores of idx [k], output [T_new, hq, d])."""
    T_new = q_new.shape[0]
    d = q_new.shape[-1]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    ds, _ = route(krbar, doc_chunk_off, qr_active[None])
    idx, val = topk_docs(ds, k)
    mem = gather_memory(tokbank, doc_tok_off, idx[0])
    L = L_prev + T_new
    k_local = apply_rope(k_local_raw[:L], global_positions(k, 0, L), base)
    q_rot = apply_rope(q_new, global_positions(k, L_prev, T_new), base)
    o = sparse_attention(q_rot, mem[:, 0], mem[:, 1], k_local, v_local[:L], L_prev, scale)
    return idx[0], val[0], o


# ---------------------------------------------------------------------------------------------
# the Memory Interleave loop for one routed layer
# ---------------------------------------------------------------------------------------------
def interleave_round_tokens(r: int, T0: int, T_new: int):
    """(L_prev, n_new) of round r (0-based): round 0 brings the T0 prompt tokens into the active
    context, every later round the T_new tokens generated in the round before."""
    return (0, T0) if r == 0 else (T0 + T_new * (r - 1), T_new)


def interleave(krbar, doc_chunk_off, kvbar, qr, q, k_raw, v, T0: int, T_new: int, rounds: int, k: int,
               base: float, scale: float | None = None, select=None):
    """Memory Interleave for one routed layer and one query: `rounds` rounds of route -> attend ->
    append -> re-route ([P1] §组件 3 Memory Interleaving; [P5] §4 生成式檢索 -> 上下文擴展 -> 生成 ->
    再檢索; [P2] re-route with the updated context).

    qr [T_total, H, d], q [T_total, hq, d], k_raw / v [T_total, hkv, d] hold every token the query
    ever has (T_total = T0 + T_new * (rounds - 1)); token j of the active context sits at global
    position k + j. Round r appends its tokens (interleave_round_tokens) to the local context,
    routes with ALL active tokens, replaces the memory set with that round's top-k, and the appended
    tokens attend causally over [selected memory ; local context].

    select: optional list of per-round document indices used for the attention in place of the
    oracle's own top-k (for comparing against an implementation whose scores may order near-tied
    documents differently); routing and its scores are computed either way.
    Returns a list over rounds of (idx [k], scores of idx [k], doc_scores [D], output [n_new, hq, d]).
    """
    d = q.shape[-1]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    out = []
    for r in range(rounds):
        L_prev, n_new = interleave_round_tokens(r, T0, T_new)
        L = L_prev + n_new
        ds, _ = route(krbar, doc_chunk_off, np.asarray(qr)[None, :L])
        idx, val = topk_docs(ds, k)
        use = idx[0] if select is None else np.asarray(select[r])
        mem = gather_memory(kvbar, doc_chunk_off, use)
        k_local = apply_rope(k_raw[:L], global_positions(k, 0, L), base)
        q_rot = apply_rope(q[L_prev:L], global_positions(k, L_prev, n_new), base)
        o = sparse_attention(q_rot, mem[:, 0], mem[:, 1], k_local, v[:L], L_prev, scale)
        out.append((idx[0], val[0], ds[0], o))
    return out
