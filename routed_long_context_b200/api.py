"""Python binding of the MSA C ABI. Same names as the C entry points; argument marshalling only.

PyTorch supplies device memory, pinned host memory and streams; every step of the hot path runs
in the CUDA kernels of libmsa.so. Outputs that the caller does not pass are allocated with torch.
"""
from __future__ import annotations

import ctypes
import math

import numpy as np
import torch

from . import _lib
from ._lib import MSA_BF16, MSA_F32, MSAError, check, lib  # noqa: F401

_DT = {torch.float32: MSA_F32, torch.bfloat16: MSA_BF16}


def _dt(t: torch.Tensor) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)") from None


def _ptr(t, strided: bool = False) -> int | None:
    """Device or host address of a tensor for the C ABI, which reads every array as dense row-major;
    a non-contiguous view is refused unless the entry point takes its stride (strided=True)."""
    if t is None:
        return None
    if not strided and not t.is_contiguous():
        raise ValueError(f"tensor of shape {tuple(t.shape)} and strides {t.stride()} must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ws(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def version() -> str:
    return lib.msa_version().decode()


def device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device-side error word (0 = none)."""
    code = ctypes.c_int32(0)
    check(lib.msa_device_status(ctypes.byref(code), _stream(stream)), "msa_device_status")
    return code.value


def rope_table(max_pos: int, d: int, base: float = 1.0e6, device="cuda") -> torch.Tensor:
    """[max_pos, d/2, 2] float32 (cos, sin) table, computed by the library on the host, then copied."""
    host = np.empty((max_pos, d // 2, 2), dtype=np.float32)
    check(lib.msa_rope_table(max_pos, d, base, host.ctypes.data), "msa_rope_table")
    return torch.from_numpy(host).to(device)


def chunk_doc_map(doc_chunk_off: torch.Tensor, n_chunks: int, stream=None) -> torch.Tensor:
    out = torch.empty(n_chunks, dtype=torch.int32, device=doc_chunk_off.device)
    check(lib.msa_chunk_doc_map(_ptr(doc_chunk_off), doc_chunk_off.numel() - 1, n_chunks, _ptr(out), _stream(stream)),
          "msa_chunk_doc_map")
    return out


def msa_rope_doc(x: torch.Tensor, seg_tok_off: torch.Tensor, pos_offset: int, cos_sin: torch.Tensor,
                 out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Rotate x [n_tok, heads, d]; token t of segment s gets position pos_offset + t - seg_tok_off[s]."""
    out = x if out is None else out
    n_tok, heads, d = x.shape
    check(lib.msa_rope_doc(_ptr(x), _ptr(out), _dt(x), n_tok, heads, d, _ptr(seg_tok_off), seg_tok_off.numel() - 1,
                           pos_offset, _ptr(cos_sin), cos_sin.shape[0], _stream(stream)), "msa_rope_doc")
    return out


def msa_pool_chunks(k, v, kr, doc_tok_off, doc_chunk_off, chunk_doc, chunk: int, cos_sin=None,
                    fuse_doc_rope: bool = True, out_dtype=None, normalize_router: bool = True, kvbar=None,
                    kr_index=None, stream=None):
    """Chunk-mean pooling -> (kvbar [C, 2, hkv, d] or None, kr_index [C, hr, d] or None)."""
    ref = k if k is not None else kr
    n_tok, _, d = ref.shape
    hkv = k.shape[1] if k is not None else 0
    hr = kr.shape[1] if kr is not None else 0
    C = chunk_doc.numel()
    out_dtype = out_dtype or ref.dtype
    if k is not None and kvbar is None:
        kvbar = torch.empty((C, 2, hkv, d), dtype=out_dtype, device=ref.device)
    if kr is not None and kr_index is None:
        kr_index = torch.empty((C, hr, d), dtype=out_dtype, device=ref.device)
    fuse = bool(fuse_doc_rope and k is not None)
    check(lib.msa_pool_chunks(_ptr(k), _ptr(v), _ptr(kr), _dt(ref), n_tok, hkv, hr, d, _ptr(doc_tok_off),
                              _ptr(doc_chunk_off), _ptr(chunk_doc), doc_tok_off.numel() - 1, C, chunk, int(fuse),
                              _ptr(cos_sin) if fuse else None, cos_sin.shape[0] if fuse else 0,
                              _ptr(kvbar) if k is not None else None, _ptr(kr_index) if kr is not None else None,
                              _DT[out_dtype], int(normalize_router), _stream(stream)), "msa_pool_chunks")
    return (kvbar if k is not None else None), (kr_index if kr is not None else None)


def msa_pack_tokens(k, v, doc_tok_off, cos_sin, bank=None, stream=None):
    """Token-level memory bank of the fine stage: k, v [n_tok, hkv, d] -> bank [n_tok, 2, hkv, d] with each
    key rotated to its position inside its document (doc_tok_off [n_docs+1], device int64)."""
    n_tok, hkv, d = k.shape
    if bank is None:
        bank = torch.empty((n_tok, 2, hkv, d), dtype=k.dtype, device=k.device)
    check(lib.msa_pack_tokens(_ptr(k), _ptr(v), _dt(k), n_tok, hkv, d, _ptr(doc_tok_off), doc_tok_off.numel() - 1,
                              _ptr(cos_sin), cos_sin.shape[0], _ptr(bank), _stream(stream)), "msa_pack_tokens")
    return bank


def route_workspace_size(n_q: int, T: int, H: int, d: int, dtype) -> int:
    n = ctypes.c_size_t(0)
    check(lib.msa_route_workspace_size(n_q, T, H, d, _DT[dtype], ctypes.byref(n)), "msa_route_workspace_size")
    return n.value


def attn_set_impl(impl: int) -> None:
    """bf16 attention: 0 = default (split variant on tcgen05, plain on mma.sync), 1 = CUDA cores for the
    plain variant, 2 = mma.sync for both, 3 = as 0 plus the backward's dK/dV on tcgen05 (opt-in; not yet
    validated on a GPU)."""
    check(lib.msa_attn_set_impl(impl), "msa_attn_set_impl")


def pool_set_impl(impl: int) -> None:
    """Chunk-mean pooling: 0 = by size (default), 1 = register streaming, 2 = bulk copy where the layout allows."""
    check(lib.msa_pool_set_impl(impl), "msa_pool_set_impl")


def pool_set_pipeline(n_stages: int = 0, stage_bytes: int = 0, copy_bytes: int = 0) -> None:
    """Tuning knob of the bulk-copy pooling kernel (zeros = default: 3 stages of 32 KiB, one copy per stage)."""
    check(lib.msa_pool_set_pipeline(n_stages, stage_bytes, copy_bytes), "msa_pool_set_pipeline")


def route_set_max_stages(n: int) -> None:
    """Tuning knob: cap on the router's pipeline stages (0 = default budget)."""
    check(lib.msa_route_set_max_stages(n), "msa_route_set_max_stages")


def route_set_impl(impl: int) -> None:
    """0 = automatic, 1 = CUDA-core kernel, 2 = tensor-core kernel, 3 = tensor cores with qhat held in shared memory."""
    check(lib.msa_route_set_impl(impl), "msa_route_set_impl")


def msa_route_scores(kr_index, chunk_doc, n_docs: int, qr, doc_scores=None, chunk_scores=None,
                     want_chunk_scores: bool = False, ws=None, stream=None):
    """Router scores: kr_index [C, H, d] (index form), qr [n_q, T, H, d] -> doc_scores [n_q, n_docs]
    (and chunk_scores [n_q, C] when requested)."""
    C = kr_index.shape[0]
    n_q, T, H, d = qr.shape
    dev = qr.device
    if doc_scores is None:
        doc_scores = torch.empty((n_q, n_docs), dtype=torch.float32, device=dev)
    if want_chunk_scores and chunk_scores is None:
        chunk_scores = torch.empty((n_q, C), dtype=torch.float32, device=dev)
    if ws is None:
        ws = _ws(route_workspace_size(n_q, T, H, d, qr.dtype), dev)
    check(lib.msa_route_scores(_ptr(kr_index), _dt(kr_index), C, _ptr(chunk_doc), n_docs, _ptr(qr), n_q, T, H, d,
                               _ptr(doc_scores), _ptr(chunk_scores), _ptr(ws), ws.numel(), _stream(stream)),
          "msa_route_scores")
    return (doc_scores, chunk_scores) if chunk_scores is not None else doc_scores


def msa_workspace_size(op: int, cfg) -> int:
    """Workspace bytes of the call named by op (_lib.MSA_OP_*), cfg its ctypes configuration struct
    (_lib.RouteWsCfg, TopkWsCfg, AttnWsCfg, RouteBwdWsCfg, or the InterleaveArgs of a round)."""
    n = ctypes.c_size_t(0)
    check(lib.msa_workspace_size(op, ctypes.cast(ctypes.byref(cfg), ctypes.c_void_p), ctypes.byref(n)),
          "msa_workspace_size")
    return n.value


def topk_workspace_size(n_q: int, n_docs: int, k: int) -> int:
    n = ctypes.c_size_t(0)
    check(lib.msa_topk_workspace_size(n_q, n_docs, k, ctypes.byref(n)), "msa_topk_workspace_size")
    return n.value


def msa_topk_docs(doc_scores, k: int, idx=None, score=None, ws=None, stream=None):
    """-> (idx int32 [n_q, k], score float32 [n_q, k]) by descending score, ties to the lower index."""
    n_q, n_docs = doc_scores.shape
    dev = doc_scores.device
    idx = torch.empty((n_q, k), dtype=torch.int32, device=dev) if idx is None else idx
    score = torch.empty((n_q, k), dtype=torch.float32, device=dev) if score is None else score
    if ws is None:
        ws = _ws(topk_workspace_size(n_q, n_docs, k), dev)
    check(lib.msa_topk_docs(_ptr(doc_scores), n_q, n_docs, k, _ptr(idx), _ptr(score), _ptr(ws), ws.numel(),
                            _stream(stream)), "msa_topk_docs")
    return idx, score


def msa_topk_docs_noalloc(doc_scores, k: int, idx=None, score=None, stream=None):
    """msa_topk_docs without a workspace: for callers that cannot allocate device memory at selection
    time. Scratch is the library's fixed device array; calls that overlap on the GPU race."""
    n_q, n_docs = doc_scores.shape
    dev = doc_scores.device
    idx = torch.empty((n_q, k), dtype=torch.int32, device=dev) if idx is None else idx
    score = torch.empty((n_q, k), dtype=torch.float32, device=dev) if score is None else score
    check(lib.msa_topk_docs_noalloc(_ptr(doc_scores), n_q, n_docs, k, _ptr(idx), _ptr(score), _stream(stream)),
          "msa_topk_docs_noalloc")
    return idx, score


def msa_topk_merge(cand_score, cand_idx, shard_doc_off, k: int, idx=None, score=None, shard_stride=None,
                   stream=None):
    """Memory Parallel merge: cand_score float32 / cand_idx int32 lists [n_q, k_cand] of every shard (device,
    shard g's lists shard_stride elements after shard g-1's; default: plain [n_shards, n_q, k_cand] arrays),
    shard_doc_off host int64 [n_shards + 1] -> (idx int32 [n_q, k] global, score float32 [n_q, k])."""
    off = np.ascontiguousarray(shard_doc_off, dtype=np.int64)
    n_shards = len(off) - 1
    n_q, k_cand = cand_score.shape[-2:]
    dev = cand_score.device
    stride = n_q * k_cand if shard_stride is None else int(shard_stride)
    for t in (cand_score, cand_idx):
        # each shard's [n_q, k_cand] lists dense, shards `stride` elements apart
        if t.stride(-1) != 1 or (n_q > 1 and t.stride(-2) != k_cand) or \
                (t.dim() >= 3 and t.shape[0] > 1 and t.stride(0) != stride):
            raise ValueError(f"msa_topk_merge: candidate lists of strides {t.stride()} do not match "
                             f"[n_shards, {n_q}, {k_cand}] with shards {stride} elements apart")
    idx = torch.empty((n_q, k), dtype=torch.int32, device=dev) if idx is None else idx
    score = torch.empty((n_q, k), dtype=torch.float32, device=dev) if score is None else score
    check(lib.msa_topk_merge(_ptr(cand_score, strided=True), _ptr(cand_idx, strided=True), stride, n_shards, n_q,
                             k_cand, off.ctypes.data, k, _ptr(idx), _ptr(score), _stream(stream)), "msa_topk_merge")
    return idx, score


def msa_gather_kv(host_bank, doc_chunk_off_host, idx_host, max_mem: int, dev_mem_kv=None, device="cuda",
                  copy_stream=None):
    """Copy the selected docs' rows [*, 2, hkv, d] from the pinned host bank into
    dev_mem_kv [n_q, max_mem, 2, hkv, d]; returns (dev_mem_kv, mem_len int32 host tensor [n_q])."""
    C, _, hkv, d = host_bank.shape
    n_q, k = idx_host.shape
    if dev_mem_kv is None:
        dev_mem_kv = torch.zeros((n_q, max_mem, 2, hkv, d), dtype=host_bank.dtype, device=device)
    off = torch.as_tensor(np.ascontiguousarray(doc_chunk_off_host, dtype=np.int64))
    idx_c = idx_host.to(torch.int32).contiguous()
    mem_len = torch.empty(n_q, dtype=torch.int32)
    check(lib.msa_gather_kv(_ptr(host_bank), _dt(host_bank), C, _ptr(off), off.numel() - 1, _ptr(idx_c), n_q, k,
                            hkv, d, max_mem, _ptr(dev_mem_kv), _ptr(mem_len), _stream(copy_stream)), "msa_gather_kv")
    return dev_mem_kv, mem_len


def msa_gather_kv_device(host_bank, doc_chunk_off, idx, max_mem: int, dev_mem_kv=None, mem_len=None, stream=None):
    """Device-side fetch: idx [n_q, k] int32 and doc_chunk_off on the device; the pinned host bank is
    read by a kernel. Returns (dev_mem_kv [n_q, max_mem, 2, hkv, d], mem_len int32 [n_q] on the device)."""
    C, _, hkv, d = host_bank.shape
    n_q, k = idx.shape
    dev = idx.device
    if dev_mem_kv is None:
        dev_mem_kv = torch.zeros((n_q, max_mem, 2, hkv, d), dtype=host_bank.dtype, device=dev)
    if mem_len is None:
        mem_len = torch.zeros(n_q, dtype=torch.int32, device=dev)
    check(lib.msa_gather_kv_device(_ptr(host_bank), _dt(host_bank), C, _ptr(doc_chunk_off), doc_chunk_off.numel() - 1,
                                   _ptr(idx), n_q, k, hkv, d, max_mem, _ptr(dev_mem_kv), _ptr(mem_len),
                                   _stream(stream)), "msa_gather_kv_device")
    return dev_mem_kv, mem_len


def msa_sparse_attn(q, mem_kv, mem_len, local_k, local_v, L: int, q_start: int, scale: float | None = None,
                    out=None, stream=None):
    """q [n_q, T, hq, d] (rotated), mem_kv [n_q, max_mem, 2, hkv, d], mem_len int32 [n_q] (device),
    local_k/local_v [n_q, L_max, hkv, d] -> out [n_q, T, hq, d]."""
    n_q, T, hq, d = q.shape
    max_mem = mem_kv.shape[1]
    hkv = mem_kv.shape[3]
    L_max = local_k.shape[1]
    out = torch.empty_like(q) if out is None else out
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    check(lib.msa_sparse_attn(_ptr(q), _ptr(mem_kv), _ptr(mem_len), max_mem, _ptr(local_k), _ptr(local_v), L_max, L,
                              q_start, n_q, T, hq, hkv, d, scale, _ptr(out), _dt(q), _stream(stream)),
          "msa_sparse_attn")
    return out


def sparse_attn_split_workspace_size(n_q: int, T: int, hq: int, hkv: int, max_mem: int, L: int) -> int:
    n = ctypes.c_size_t(0)
    check(lib.msa_sparse_attn_split_workspace_size(n_q, T, hq, hkv, max_mem, L, ctypes.byref(n)),
          "msa_sparse_attn_split_workspace_size")
    return n.value


def sparse_attn_split_plan(n_q: int, T: int, hq: int, hkv: int, max_mem: int, L: int) -> dict:
    """The launch plan of msa_sparse_attn_split on the current device: row blocks per CTA, key ranges,
    and the cluster size when the ranges are merged in distributed shared memory (0: combine pass)."""
    rb, kr, cl = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    check(lib.msa_sparse_attn_split_plan(n_q, T, hq, hkv, max_mem, L, ctypes.byref(rb), ctypes.byref(kr),
                                         ctypes.byref(cl)), "msa_sparse_attn_split_plan")
    return {"row_blocks": rb.value, "key_ranges": kr.value, "cluster": cl.value}


def msa_sparse_attn_split(q, mem_kv, mem_len, local_k, local_v, L: int, q_start: int, scale: float | None = None,
                          out=None, ws=None, lse=None, stream=None):
    """msa_sparse_attn for long memories (token-level fine stage): keys split into ranges that run as
    separate blocks, then merged. Same arguments and result; bf16 only. lse: optional float32
    [n_q, T, hq] output, the log-sum-exp of each row's logits (for the backward pass)."""
    n_q, T, hq, d = q.shape
    max_mem = mem_kv.shape[1]
    hkv = mem_kv.shape[3]
    L_max = local_k.shape[1]
    out = torch.empty_like(q) if out is None else out
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if ws is None:
        ws = _ws(sparse_attn_split_workspace_size(n_q, T, hq, hkv, max_mem, L), q.device)
    check(lib.msa_sparse_attn_split(_ptr(q), _ptr(mem_kv), _ptr(mem_len), max_mem, _ptr(local_k), _ptr(local_v),
                                    L_max, L, q_start, n_q, T, hq, hkv, d, scale, _ptr(out), _ptr(lse), _dt(q),
                                    _ptr(ws), ws.numel(), _stream(stream)), "msa_sparse_attn_split")
    return out


# ------------------------------------------------------------------------------------------------ backward
def msa_sparse_attn_backward(q, mem_kv, mem_len, local_k, local_v, L: int, q_start: int, out, dout, lse,
                             scale: float | None = None, grads=None, ws=None, stream=None):
    """Gradients of the sparse attention (bf16 inputs): returns (dq [n_q, T, hq, d], dmem_kv [n_q, max_mem, 2,
    hkv, d], dlocal_k, dlocal_v [n_q, L_max, hkv, d]), fp32; `grads` may supply those four buffers."""
    n_q, T, hq, d = q.shape
    max_mem, hkv = mem_kv.shape[1], mem_kv.shape[3]
    L_max = local_k.shape[1]
    dev = q.device
    if grads is None:
        grads = (torch.zeros((n_q, T, hq, d), dtype=torch.float32, device=dev),
                 torch.zeros((n_q, max_mem, 2, hkv, d), dtype=torch.float32, device=dev),
                 torch.zeros((n_q, L_max, hkv, d), dtype=torch.float32, device=dev),
                 torch.zeros((n_q, L_max, hkv, d), dtype=torch.float32, device=dev))
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if ws is None:
        n = ctypes.c_size_t(0)
        check(lib.msa_sparse_attn_backward_workspace_size(n_q, T, hq, hkv, max_mem, L, ctypes.byref(n)),
              "msa_sparse_attn_backward_workspace_size")
        ws = _ws(n.value, dev)
    dq, dmem, dlk, dlv = grads
    check(lib.msa_sparse_attn_backward(_ptr(q), _ptr(mem_kv), _ptr(mem_len), max_mem, _ptr(local_k), _ptr(local_v),
                                       L_max, L, q_start, n_q, T, hq, hkv, d, scale, _ptr(out), _ptr(dout), _ptr(lse),
                                       _dt(q), _ptr(dq), _ptr(dmem), _ptr(dlk), _ptr(dlv), _ptr(ws), ws.numel(),
                                       _stream(stream)), "msa_sparse_attn_backward")
    return grads


def msa_gather_kv_backward(dmem_kv, doc_chunk_off, idx, n_chunks: int, dkvbar=None, accumulate: bool = False,
                           stream=None):
    """Memory-row gradients [n_q, max_mem, 2, hkv, d] (fp32) into chunk-row gradients dkvbar [n_chunks, 2, hkv, d]
    (zeroed first unless accumulate)."""
    n_q, max_mem, _, hkv, d = dmem_kv.shape
    k = idx.shape[1]
    if dkvbar is None:
        dkvbar = torch.empty((n_chunks, 2, hkv, d), dtype=torch.float32, device=dmem_kv.device)
        accumulate = False
    check(lib.msa_gather_kv_backward(_ptr(dmem_kv), n_chunks, _ptr(doc_chunk_off), doc_chunk_off.numel() - 1,
                                     _ptr(idx), n_q, k, hkv, d, max_mem, _ptr(dkvbar), int(accumulate),
                                     _stream(stream)), "msa_gather_kv_backward")
    return dkvbar


def msa_pool_chunks_backward(dkvbar, dkr_index, doc_tok_off, doc_chunk_off, chunk_doc, chunk: int, n_tok: int,
                             kr=None, cos_sin=None, fuse_doc_rope: bool = True, normalize_router: bool = True,
                             stream=None):
    """Token gradients (dk, dv [n_tok, hkv, d], dkr [n_tok, hr, d], fp32; None where not asked) from the chunk
    gradients dkvbar [C, 2, hkv, d] and dkr_index [C, hr, d] (either may be None)."""
    ref = dkvbar if dkvbar is not None else dkr_index
    dev = ref.device
    C, d = chunk_doc.numel(), ref.shape[-1]
    hkv = dkvbar.shape[2] if dkvbar is not None else 0
    hr = dkr_index.shape[1] if dkr_index is not None else 0
    dk = dv = dkr = None
    if dkvbar is not None:
        dk = torch.empty((n_tok, hkv, d), dtype=torch.float32, device=dev)
        dv = torch.empty((n_tok, hkv, d), dtype=torch.float32, device=dev)
    if dkr_index is not None:
        dkr = torch.empty((n_tok, hr, d), dtype=torch.float32, device=dev)
    fuse = bool(fuse_doc_rope and dkvbar is not None)
    check(lib.msa_pool_chunks_backward(_ptr(dkvbar), _ptr(dkr_index), _ptr(kr), _dt(kr) if kr is not None else MSA_F32,
                                       n_tok, hkv, hr, d, _ptr(doc_tok_off), _ptr(doc_chunk_off), _ptr(chunk_doc),
                                       doc_tok_off.numel() - 1, C, chunk, int(fuse), _ptr(cos_sin) if fuse else None,
                                       cos_sin.shape[0] if fuse else 0, int(normalize_router), _ptr(dk), _ptr(dv),
                                       _ptr(dkr), _stream(stream)), "msa_pool_chunks_backward")
    return dk, dv, dkr


def msa_router_aux_loss(doc_scores, evidence, tau: float, stream=None):
    """(loss per query [n_q], dL/d doc_scores [n_q, D]) of the auxiliary router loss; evidence int32 [n_q, n_ev]
    (-1 padding). The gradient is that of the mean of the per-query losses."""
    n_q, D = doc_scores.shape
    loss = torch.empty(n_q, dtype=torch.float32, device=doc_scores.device)
    grad = torch.empty_like(doc_scores)
    ev = evidence.to(device=doc_scores.device, dtype=torch.int32).contiguous()
    check(lib.msa_router_aux_loss(_ptr(doc_scores), n_q, D, _ptr(ev), ev.shape[1], tau, _ptr(loss), _ptr(grad),
                                  _stream(stream)), "msa_router_aux_loss")
    return loss, grad


def msa_route_backward(kr_index, doc_chunk_off, qr, d_doc_scores, stream=None):
    """(dqr [n_q, T, H, d], dkhat [C, H, d]) fp32: gradients of the router's document scores."""
    C, H, d = kr_index.shape
    n_q, T = qr.shape[:2]
    dev = qr.device
    n = ctypes.c_size_t(0)
    check(lib.msa_route_backward_workspace_size(C, n_q, T, H, d, ctypes.byref(n)), "msa_route_backward_workspace_size")
    ws = _ws(n.value, dev)
    dqr = torch.empty((n_q, T, H, d), dtype=torch.float32, device=dev)
    dkhat = torch.empty((C, H, d), dtype=torch.float32, device=dev)
    check(lib.msa_route_backward(_ptr(kr_index), _dt(kr_index), C, _ptr(doc_chunk_off), doc_chunk_off.numel() - 1,
                                 _ptr(qr), n_q, T, H, d, _ptr(d_doc_scores), _ptr(dqr), _ptr(dkhat), _ptr(ws),
                                 ws.numel(), _stream(stream)), "msa_route_backward")
    return dqr, dkhat


class InterleaveRound:
    """Marshals msa_interleave_args for one round; holds the ctypes structures alive."""

    def __init__(self, layers, *, n_chunks, n_docs, doc_chunk_off, doc_chunk_off_host, chunk_doc, n_q, H, d, hq, hkv,
                 k, L_prev, T_new, new_q_stride, L_max, max_mem, cos_sin, scale=None, dtype=torch.bfloat16, ws=None,
                 reserved_sms: int = 0, fetch_mode: int = 1):
        self.layer_structs = (_lib.LayerArgs * len(layers))()
        for i, y in enumerate(layers):
            s = self.layer_structs[i]
            for f in ("kr_index", "host_bank", "qr", "q_new", "k_new", "v_new", "local_k", "local_v", "out",
                      "topk_idx_host"):
                setattr(s, f, y[f].data_ptr())
        self._off_host = torch.as_tensor(np.ascontiguousarray(doc_chunk_off_host, dtype=np.int64))
        a = _lib.InterleaveArgs()
        a.n_layers = len(layers)
        a.layers = self.layer_structs
        a.dt = _DT[dtype]
        a.n_chunks, a.n_docs = n_chunks, n_docs
        a.doc_chunk_off = doc_chunk_off.data_ptr()
        a.doc_chunk_off_host = self._off_host.data_ptr()
        a.chunk_doc = chunk_doc.data_ptr()
        a.n_q, a.H, a.d, a.hq, a.hkv, a.k = n_q, H, d, hq, hkv, k
        a.L_prev, a.T_new, a.new_q_stride, a.L_max, a.max_mem = L_prev, T_new, new_q_stride, L_max, max_mem
        a.rope_cos_sin = cos_sin.data_ptr()
        a.rope_max_pos = cos_sin.shape[0]
        a.scale = 1.0 / math.sqrt(d) if scale is None else scale
        a.reserved_sms = reserved_sms
        a.fetch_mode = fetch_mode
        self.args = a
        need = ctypes.c_size_t(0)
        a.ws, a.ws_bytes = None, 0
        check(lib.msa_interleave_workspace_size(ctypes.byref(a), ctypes.byref(need)), "msa_interleave_workspace_size")
        self.ws = _ws(need.value, doc_chunk_off.device) if ws is None else ws
        a.ws, a.ws_bytes = self.ws.data_ptr(), self.ws.numel()

    def run(self, compute=None, copy=None, timeout_us: int = 30_000_000, route_events=None) -> None:
        """route_events: optional list of 2 * n_layers torch.cuda.Event(enable_timing=True), recorded around
        each layer's router kernel on the compute stream."""
        if route_events is not None:
            arr = (ctypes.c_void_p * len(route_events))(*[e.cuda_event for e in route_events])
            self.args.route_events = ctypes.cast(arr, ctypes.c_void_p)
        else:
            arr = None
            self.args.route_events = None
        check(lib.msa_interleave_step(ctypes.byref(self.args), _stream(compute), _stream(copy), timeout_us),
              "msa_interleave_step")
        del arr


    def capture(self, stream) -> "InterleaveGraph":
        """The round captured into a CUDA graph on `stream` (a created stream; fetch_mode 1): see
        msa_interleave_graph_create. Refill the round's inputs in place between replays."""
        return InterleaveGraph(self, stream)


class InterleaveGraph:
    """A captured interleave round (msa_interleave_graph_*): launch(stream) replays it."""

    def __init__(self, rnd: InterleaveRound, stream):
        self._round = rnd                  # keeps the marshalled arguments and buffers alive
        self._g = ctypes.c_void_p(None)
        rnd.args.route_events = None
        check(lib.msa_interleave_graph_create(ctypes.byref(rnd.args), _stream(stream), ctypes.byref(self._g)),
              "msa_interleave_graph_create")

    def launch(self, stream=None) -> None:
        check(lib.msa_interleave_graph_launch(self._g, _stream(stream)), "msa_interleave_graph_launch")

    def close(self) -> None:
        if self._g:
            check(lib.msa_interleave_graph_destroy(self._g), "msa_interleave_graph_destroy")
            self._g = ctypes.c_void_p(None)

    def __del__(self):
        try:
            if self._g:
                lib.msa_interleave_graph_destroy(self._g)
        except Exception:
            pass


def msa_interleave_step(layers, compute=None, copy=None, timeout_us: int = 30_000_000, **kw) -> InterleaveRound:
    """One Memory Interleave round over every routed layer (see include/msa.h). Returns the marshalled
    round so it can be re-run."""
    r = InterleaveRound(layers, **kw)
    r.run(compute, copy, timeout_us)
    return r
