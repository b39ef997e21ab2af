"""Memory bank of one routed layer: the HBM-resident router index (per-head unit vectors of the
pooled router keys) and the pinned host content bank of pooled K-bar/V-bar, with the CSR metadata
that maps documents to chunks. Built once (offline encoding) by the library's kernels.
"""
from __future__ import annotations

import numpy as np
import torch

from . import api


class BankLayout:
    """Document -> chunk metadata shared by every layer: host and device CSR offsets, chunk -> doc map."""

    def __init__(self, doc_chunk_counts, device="cuda", doc_tok_off=None):
        counts = np.asarray(doc_chunk_counts, dtype=np.int64)
        self.n_docs = int(len(counts))
        self.doc_chunk_off_host = np.zeros(self.n_docs + 1, dtype=np.int64)
        np.cumsum(counts, out=self.doc_chunk_off_host[1:])
        self.n_chunks = int(self.doc_chunk_off_host[-1])
        self.max_doc_chunks = int(counts.max()) if self.n_docs else 0
        self.device = device
        self.doc_chunk_off = torch.from_numpy(self.doc_chunk_off_host).to(device)
        self.chunk_doc = api.chunk_doc_map(self.doc_chunk_off, self.n_chunks)
        self.doc_tok_off_host = None if doc_tok_off is None else np.asarray(doc_tok_off, dtype=np.int64)
        self.doc_tok_off = None if doc_tok_off is None else torch.from_numpy(self.doc_tok_off_host).to(device)

    @classmethod
    def from_doc_lengths(cls, doc_len, chunk: int, device="cuda"):
        doc_len = np.asarray(doc_len, dtype=np.int64)
        off = np.zeros(len(doc_len) + 1, dtype=np.int64)
        np.cumsum(doc_len, out=off[1:])
        return cls((doc_len + chunk - 1) // chunk, device, doc_tok_off=off)


def encode_tokens(layout: BankLayout, k, v, kr, chunk: int, cos_sin, out_dtype=None, stream=None):
    """Offline encoding of token-level K, V, K^R [n_tok, heads, d]: document-wise RoPE on K fused into
    chunk-mean pooling; returns (kvbar [C, 2, hkv, d] on the device, router index [C, hr, d])."""
    return api.msa_pool_chunks(k, v, kr, layout.doc_tok_off, layout.doc_chunk_off, layout.chunk_doc, chunk,
                               cos_sin=cos_sin, fuse_doc_rope=True, out_dtype=out_dtype, normalize_router=True,
                               stream=stream)


def index_from_prepooled(layout: BankLayout, krbar_raw, out=None, stream=None):
    """Router index from already pooled router keys [C, hr, d]: per-head L2 normalisation
    (pooling with chunk = 1 over the chunk rows)."""
    _, idx = api.msa_pool_chunks(None, None, krbar_raw, layout.doc_chunk_off, layout.doc_chunk_off, layout.chunk_doc,
                                 1, fuse_doc_rope=False, normalize_router=True, kr_index=out, stream=stream)
    return idx


def to_host_bank(kvbar: torch.Tensor) -> torch.Tensor:
    """Pinned host copy of the pooled K-bar/V-bar (the CPU-resident content bank)."""
    host = torch.empty(kvbar.shape, dtype=kvbar.dtype, pin_memory=True)
    host.copy_(kvbar)
    return host


class GrowableBank:
    """A layer's memory that grows by whole documents without re-encoding the earlier ones.

    Holds the router index [capacity, hr, d] and the pooled K-bar/V-bar [capacity, 2, hkv, d] on the
    device with spare capacity, plus the document metadata. append() encodes only the new documents
    (document-wise RoPE + chunk-mean pooling, the same kernels as a full encode) straight into the
    next free rows and extends the offsets; every earlier row is left untouched, so the result is
    bit-identical to encoding all documents at once.
    """

    def __init__(self, capacity_chunks: int, hr: int, hkv: int, d: int, dtype=torch.bfloat16, device="cuda"):
        self.capacity = int(capacity_chunks)
        self.index = torch.empty((self.capacity, hr, d), dtype=dtype, device=device)
        self.kvbar = torch.empty((self.capacity, 2, hkv, d), dtype=dtype, device=device)
        self.device = device
        self.doc_len = np.zeros(0, dtype=np.int64)
        self.doc_chunk_off_host = np.zeros(1, dtype=np.int64)
        self.layout = None

    @property
    def n_chunks(self) -> int:
        return int(self.doc_chunk_off_host[-1])

    def append(self, k, v, kr, doc_len, chunk: int, cos_sin, stream=None):
        """Encode new documents (token-level k, v [n_tok, hkv, d], kr [n_tok, hr, d] of the new documents
        only, doc_len their token counts) into the next free rows. Returns the slice of new chunk rows."""
        doc_len = np.asarray(doc_len, dtype=np.int64)
        new = BankLayout.from_doc_lengths(doc_len, chunk, self.device)
        c0, c1 = self.n_chunks, self.n_chunks + new.n_chunks
        if c1 > self.capacity:
            raise ValueError(f"bank capacity {self.capacity} chunks exceeded ({c1} needed)")
        if new.n_chunks:
            api.msa_pool_chunks(k, v, kr, new.doc_tok_off, new.doc_chunk_off, new.chunk_doc, chunk, cos_sin=cos_sin,
                                fuse_doc_rope=True, normalize_router=True, kvbar=self.kvbar[c0:c1],
                                kr_index=self.index[c0:c1], stream=stream)
        self.doc_len = np.concatenate([self.doc_len, doc_len])
        self.doc_chunk_off_host = np.concatenate([self.doc_chunk_off_host, c0 + new.doc_chunk_off_host[1:]])
        self.layout = BankLayout(np.diff(self.doc_chunk_off_host), self.device)
        return slice(c0, c1)
