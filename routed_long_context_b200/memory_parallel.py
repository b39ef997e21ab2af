"""Memory Parallel: a layer's router index sharded by documents over the ranks of a process group.

Each rank holds a contiguous run of documents (its chunk rows of the index), scores them against
the broadcast router queries, keeps its local top-k, and one all_gather hands every rank all local
lists; every rank then merges them into the same global top-k ([P2] EverMind MSA router sparse
attention architecture, §工程实现的关键细节: router keys sharded over GPUs, local scoring, a global
reduction of the local best into the global ranking; [P3] §四大技术突破 3). The merge is exact:
with disjoint shards and local lists of length k, the result equals one top-k over all documents.

Host-side pieces (shard_bounds, exchange_candidates) are plain numpy / torch.distributed and run on
any backend; scoring, selection and the merge run in the library's kernels.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist


def shard_bounds(doc_chunk_off_host, world: int, k: int) -> np.ndarray:
    """Document boundaries [world + 1] of `world` contiguous shards with about equal chunk counts (the
    router's work), each holding at least k documents (its local top-k needs k candidates)."""
    off = np.asarray(doc_chunk_off_host, dtype=np.int64)
    n_docs = len(off) - 1
    if world < 1 or k < 1 or n_docs < world * k:
        raise ValueError(f"cannot split {n_docs} documents into {world} shards of at least {k}")
    b = np.zeros(world + 1, dtype=np.int64)
    b[world] = n_docs
    for r in range(1, world):
        target = off[-1] * r // world
        d = int(np.searchsorted(off, target, side="left"))      # first document starting at or after target
        b[r] = min(max(d, b[r - 1] + k), n_docs - (world - r) * k)
    return b


def exchange_candidates(send: torch.Tensor, group=None, out: torch.Tensor | None = None) -> torch.Tensor:
    """All ranks' packed candidate lists: send [2, n_q, k] int32 (row 0 the float32 scores' bits, row 1
    the local indices) -> [world, 2, n_q, k], rank order. One all_gather (none for a single rank)."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if world == 1:
        return send.unsqueeze(0)
    if out is None:
        out = torch.empty((world * send.shape[0],) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
    dist.all_gather_into_tensor(out.view(world * send.shape[0], *send.shape[1:]), send, group=group)
    return out.view(world, *send.shape)


class ShardRouter:
    """One rank's shard of a layer: scores its documents and writes its local top-k into a packed
    candidate buffer (row 0: scores as float32, row 1: indices local to the shard)."""

    def __init__(self, doc_chunk_off_host, index: torch.Tensor, world: int, rank: int, n_q: int, T: int, k: int,
                 device="cuda"):
        from . import api
        from .bank import BankLayout

        off = np.asarray(doc_chunk_off_host, dtype=np.int64)
        self.bounds = shard_bounds(off, world, k)
        self.d0, self.d1 = int(self.bounds[rank]), int(self.bounds[rank + 1])
        self.c0, self.c1 = int(off[self.d0]), int(off[self.d1])
        self.layout = BankLayout(np.diff(off[self.d0:self.d1 + 1]), device)
        # this shard's rows of the index: a view when the caller passes the whole index, else the shard itself
        self.index = index[self.c0:self.c1] if index.shape[0] == off[-1] else index
        assert self.index.shape[0] == self.c1 - self.c0, "index rows do not match the shard"
        H, d = self.index.shape[1], self.index.shape[2]
        self.k, self.n_q = k, n_q
        self.doc_scores = torch.empty((n_q, self.layout.n_docs), dtype=torch.float32, device=device)
        self.route_ws = api._ws(api.route_workspace_size(n_q, T, H, d, self.index.dtype), device)
        self.topk_ws = api._ws(api.topk_workspace_size(n_q, self.layout.n_docs, k), device)
        self.send = torch.empty((2, n_q, k), dtype=torch.int32, device=device)

    def select_local(self, qr: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """Local top-k of qr [n_q, T, H, d] over this shard into out (default: self.send) [2, n_q, k]."""
        from . import api

        out = self.send if out is None else out
        api.msa_route_scores(self.index, self.layout.chunk_doc, self.layout.n_docs, qr, doc_scores=self.doc_scores,
                             ws=self.route_ws, stream=stream)
        api.msa_topk_docs(self.doc_scores, self.k, idx=out[1], score=out[0].view(torch.float32), ws=self.topk_ws,
                          stream=stream)
        return out


def merge_candidates(gathered: torch.Tensor, bounds, k: int, idx=None, score=None, stream=None):
    """Global top-k from the packed lists [n_shards, 2, n_q, k_cand] of every shard (exchange_candidates)."""
    from . import api

    n_q, k_cand = gathered.shape[-2:]
    return api.msa_topk_merge(gathered[:, 0].view(torch.float32), gathered[:, 1], bounds, k, idx=idx, score=score,
                              shard_stride=2 * n_q * k_cand, stream=stream)


class MemoryParallelRouter:
    """Routing and selection of one layer with its index sharded over the process group: local score
    + local top-k, one all_gather of k (score, index) pairs per query, the same merge on every rank.
    select() returns the global (idx, score) on this rank's device."""

    def __init__(self, doc_chunk_off_host, index: torch.Tensor, n_q: int, T: int, k: int, group=None, device="cuda"):
        self.group = group
        world = dist.get_world_size(group) if dist.is_initialized() else 1
        rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.shard = ShardRouter(doc_chunk_off_host, index, world, rank, n_q, T, k, device)
        self.k = k
        self.gathered = torch.empty((world, 2, n_q, k), dtype=torch.int32, device=device)
        self.idx = torch.empty((n_q, k), dtype=torch.int32, device=device)
        self.score = torch.empty((n_q, k), dtype=torch.float32, device=device)

    def select(self, qr: torch.Tensor):
        """Global (idx, score) [n_q, k] for router queries qr [n_q, T, H, d]; every launch and the
        collective go to the current stream, so the whole selection can be captured in a CUDA graph."""
        send = self.shard.select_local(qr)
        gathered = exchange_candidates(send, self.group, out=self.gathered)
        return merge_candidates(gathered, self.shard.bounds, self.k, idx=self.idx, score=self.score)
