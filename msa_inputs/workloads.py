"""Synthetic workloads: the memory banks, router queries and attention inputs
of the five measured configurations, plus small ragged variants for tests.

Everything is built from the counter-based generator in ``rng.py``; nothing
here computes any step of the attention method. Planting only copies a query
vector (plus generated noise) into chosen rows of a memory tensor, so that the
expected routing result is known in advance.

Shapes (row-major, bf16 values carried as float32 on the host):
  token-level memory  K^R [n_tok, H, d], K and V [n_tok, hkv, d]
  pre-pooled memory   raw router keys [C, H, d]; content bank [C, 2, hkv, d]
  per layer           Q^R [n_q, T_total, H, d]; Q [n_q, T_total, hq, d];
                      new-token K and V [n_q, T_total, hkv, d]
where T_total is every token a query holds after the last interleave round.
Round r (0-based) appends T0 (r = 0) or T_new tokens and routes with all of
them; its attention queries are the appended tokens.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import rng

SEED_BASE = 0x4D534100  # "MSA" followed by the configuration number

# tensor kinds, packed into the generator's tensor id
KR_TOK, K_TOK, V_TOK, KRBAR, BANK, QR, Q, KNEW, VNEW, NOISE, PICK = range(1, 12)


def tid(kind: int, layer: int = 0, extra: int = 0) -> int:
    return (kind << 40) | (layer << 20) | extra


@dataclass
class Plant:
    """One planted memory row group: every row of `rows` gets `vec` ([H*d] float32, storage-rounded)."""
    layer: int
    doc: int
    chunk_in_doc: int
    rows: np.ndarray          # token rows (token-level) or one chunk row (pre-pooled)
    vec: np.ndarray


@dataclass
class Workload:
    name: str
    seed: int
    doc_len: np.ndarray       # tokens per memory document
    chunk: int
    dtype: str                # "f32" or "bf16"
    n_q: int
    T0: int
    k: int
    prepooled: bool = False
    H: int = 8
    d: int = 128
    hq: int = 32
    hkv: int = 8
    layers: int = 1
    rounds: int = 1
    T_new: int = 32
    rope_base: float = 1.0e6
    n_host_banks: int = 1
    plant_kind: str = "none"  # tiny | mix | per_query | single | chain | none
    plant_args: dict = field(default_factory=dict)

    # ------------------------------------------------------------------ layout
    def __post_init__(self):
        self.doc_len = np.asarray(self.doc_len, dtype=np.int64)
        self.n_docs = int(len(self.doc_len))
        self.doc_tok_off = np.zeros(self.n_docs + 1, dtype=np.int64)
        np.cumsum(self.doc_len, out=self.doc_tok_off[1:])
        self.doc_chunks = (self.doc_len + self.chunk - 1) // self.chunk
        self.doc_chunk_off = np.zeros(self.n_docs + 1, dtype=np.int64)
        np.cumsum(self.doc_chunks, out=self.doc_chunk_off[1:])
        self.n_tok = int(self.doc_tok_off[-1])
        self.n_chunks = int(self.doc_chunk_off[-1])
        self.chunk_doc = np.repeat(np.arange(self.n_docs, dtype=np.int32), self.doc_chunks)
        self.T_total = self.T0 + self.T_new * (self.rounds - 1)
        self.max_mem = int(self.k * self.doc_chunks.max())
        self._plants = {}
        self._small = {}

    def round_tokens(self, r: int):
        """(L_prev, T_new_r): tokens held before round r and tokens appended in round r."""
        if r == 0:
            return 0, self.T0
        return self.T0 + self.T_new * (r - 1), self.T_new

    def host_bank_slot(self, layer: int) -> int:
        return layer % self.n_host_banks

    # ------------------------------------------------------------------ small per-layer tensors
    def _gen(self, kind, layer, shape, sigma=1.0):
        n = int(np.prod(shape))
        return rng.normal(self.seed, tid(kind, layer), 0, n, sigma, self.dtype).reshape(shape)

    def qr(self, layer: int) -> np.ndarray:
        key = ("qr", layer)
        if key not in self._small:
            qr = self._gen(QR, layer, (self.n_q, self.T_total, self.H, self.d))
            if self.plant_kind == "chain":
                qr = self._chain_queries(layer, qr)
            self._small[key] = qr
        return self._small[key]

    def q(self, layer: int) -> np.ndarray:
        return self._gen(Q, layer, (self.n_q, self.T_total, self.hq, self.d))

    def k_new(self, layer: int) -> np.ndarray:
        return self._gen(KNEW, layer, (self.n_q, self.T_total, self.hkv, self.d))

    def v_new(self, layer: int) -> np.ndarray:
        return self._gen(VNEW, layer, (self.n_q, self.T_total, self.hkv, self.d))

    # ------------------------------------------------------------------ planting
    def _noise(self, layer, slot, sigma):
        hd = self.H * self.d
        return rng.normal(self.seed, tid(NOISE, layer), slot * hd, hd, sigma, "f32")

    def _pick(self, layer, n, hi, extra=0, exclude=()):
        return rng.distinct_ints(self.seed, tid(PICK, layer, extra), n, hi, exclude)

    def _chunk_rows(self, doc, j):
        """Rows of the memory tensor that make up chunk j of doc."""
        if self.prepooled:
            return np.array([self.doc_chunk_off[doc] + j], dtype=np.int64)
        s = self.doc_tok_off[doc] + j * self.chunk
        e = min(s + self.chunk, self.doc_tok_off[doc + 1])
        return np.arange(s, e, dtype=np.int64)

    def plants(self, layer: int):
        """Planted row groups of the router-key memory tensor of `layer` (with expected selections)."""
        if layer in self._plants:
            return self._plants[layer]
        hd = self.H * self.d
        qr = self.qr(layer).reshape(self.n_q, self.T_total, hd)
        out, expect = [], {}
        pk = self.plant_kind
        if pk == "tiny":
            for slot, (doc, j, t) in enumerate(self.plant_args["docs"]):
                vec = rng.round_to(qr[0, t] + self._noise(layer, slot, 0.1), self.dtype)
                out.append(Plant(layer, doc, j, self._chunk_rows(doc, j), vec))
                expect.setdefault((0, 0), []).append(doc)
        elif pk in ("mix", "single"):
            n = self.plant_args["n"]
            docs = self._pick(layer, n, self.n_docs)
            for slot, doc in enumerate(docs):
                j = int(rng.uniform_int(self.seed, tid(PICK, layer, 1000 + slot), 1, int(self.doc_chunks[doc]))[0])
                if pk == "mix":
                    t1, t2 = self._pick(layer, 2, self.T0, extra=2000 + slot)
                    base = (qr[0, t1] + qr[0, t2]) * np.float32(0.5)
                    sig = 0.2
                else:
                    t = int(rng.uniform_int(self.seed, tid(PICK, layer, 3000 + slot), 1, self.T0)[0])
                    base = qr[0, t]
                    sig = 0.1
                vec = rng.round_to(base + self._noise(layer, slot, sig), self.dtype)
                out.append(Plant(layer, int(doc), j, self._chunk_rows(int(doc), j), vec))
                expect.setdefault((0, 0), []).append(int(doc))
        elif pk == "per_query":
            per = self.plant_args["per_query"]
            docs = self._pick(layer, per * self.n_q, self.n_docs).reshape(self.n_q, per)
            for q in range(self.n_q):
                for i, doc in enumerate(docs[q]):
                    slot = q * per + i
                    j = int(rng.uniform_int(self.seed, tid(PICK, layer, 1000 + slot), 1, int(self.doc_chunks[doc]))[0])
                    vec = rng.round_to(qr[q, 0] + self._noise(layer, slot, 0.1), self.dtype)
                    out.append(Plant(layer, int(doc), j, self._chunk_rows(int(doc), j), vec))
                    expect.setdefault((0, q), []).append(int(doc))
        elif pk == "chain":
            out, expect = self._chain_plants(layer)
        self._plants[layer] = (out, expect)
        return self._plants[layer]

    def expected(self, layer: int, rnd: int, q: int):
        """Docs that planting puts in query q's top-k at round rnd of layer."""
        return self.plants(layer)[1].get((rnd, q), [])

    def _chain_docs(self, layer):
        return self._pick(layer, 3 * self.n_q, self.n_docs).reshape(self.n_q, 3)

    def _raw_krbar_row(self, layer, row):
        return rng.normal_rows(self.seed, tid(KRBAR, layer), self.H * self.d, [row], 1.0, self.dtype)[0]

    def _chain_links(self, layer):
        """Link vectors u1, u2 per query: the generated chunk 1 of D1 and of D2."""
        docs = self._chain_docs(layer)
        links = np.zeros((self.n_q, 2, self.H * self.d), dtype=np.float32)
        for q in range(self.n_q):
            for h in range(2):
                links[q, h] = self._raw_krbar_row(layer, int(self.doc_chunk_off[docs[q, h]] + 1))
        return docs, links

    def _chain_queries(self, layer, qr):
        """Tokens appended in round r >= 1 carry the previous round's link vector plus N(0, 0.1)."""
        _, links = self._chain_links(layer)
        hd = self.H * self.d
        qr = qr.reshape(self.n_q, self.T_total, hd).copy()
        for q in range(self.n_q):
            for r in (1, 2):
                if r >= self.rounds:
                    continue
                L_prev, tn = self.round_tokens(r)
                for t in range(L_prev, L_prev + tn):
                    noise = rng.normal(self.seed, tid(NOISE, layer, 1 + q), t * hd, hd, 0.1, "f32")
                    qr[q, t] = rng.round_to(links[q, r - 1] + noise, self.dtype)
        return qr.reshape(self.n_q, self.T_total, self.H, self.d)

    def _chain_plants(self, layer):
        docs, links = self._chain_links(layer)
        hd = self.H * self.d
        qr = self.qr(layer).reshape(self.n_q, self.T_total, hd)
        out, expect = [], {}
        for q in range(self.n_q):
            t_star = int(rng.uniform_int(self.seed, tid(PICK, layer, 5000 + q), 1, self.T0)[0])
            heads = [qr[q, t_star], links[q, 0], links[q, 1]]
            for r in range(3):
                vec = rng.round_to(heads[r] + self._noise(layer, 3 * q + r, 0.1), self.dtype)
                doc = int(docs[q, r])
                out.append(Plant(layer, doc, 0, self._chunk_rows(doc, 0), vec))
                if r < self.rounds:
                    expect.setdefault((r, q), []).append(doc)
        return out, expect

    # ------------------------------------------------------------------ large memory tensors
    def memory_tensors(self, layer: int):
        """name -> (tensor id, shape, row length) of the generated memory tensors of `layer`."""
        if self.prepooled:
            slot = self.host_bank_slot(layer)
            return {
                "krbar": (tid(KRBAR, layer), (self.n_chunks, self.H, self.d), self.H * self.d),
                "bank": (tid(BANK, slot), (self.n_chunks, 2, self.hkv, self.d), 2 * self.hkv * self.d),
            }
        return {
            "kr": (tid(KR_TOK, layer), (self.n_tok, self.H, self.d), self.H * self.d),
            "k": (tid(K_TOK, layer), (self.n_tok, self.hkv, self.d), self.hkv * self.d),
            "v": (tid(V_TOK, layer), (self.n_tok, self.hkv, self.d), self.hkv * self.d),
        }

    def router_tensor_name(self) -> str:
        return "krbar" if self.prepooled else "kr"

    def host_rows(self, layer: int, name: str, rows) -> np.ndarray:
        """Rows of a memory tensor as the host sees them (generated, then planted)."""
        t, shape, row_len = self.memory_tensors(layer)[name]
        rows = np.asarray(rows, dtype=np.int64)
        out = rng.normal_rows(self.seed, t, row_len, rows, 1.0, self.dtype)
        if name == self.router_tensor_name():
            pos = {int(r): i for i, r in enumerate(rows)}
            for p in self.plants(layer)[0]:
                for r in p.rows:
                    i = pos.get(int(r))
                    if i is not None:
                        out[i] = p.vec
        return out

    def host_tensor(self, layer: int, name: str) -> np.ndarray:
        """A whole memory tensor on the host (small workloads only)."""
        t, shape, row_len = self.memory_tensors(layer)[name]
        return self.host_rows(layer, name, np.arange(shape[0])).reshape(shape)

    def chunk_token_rows(self, chunks) -> np.ndarray:
        """Token rows of the given chunks (token-level workloads), concatenated."""
        return np.concatenate([self._chunk_rows(int(self.chunk_doc[c]), int(c - self.doc_chunk_off[self.chunk_doc[c]]))
                               for c in chunks])


# ------------------------------------------------------------------------------------------------
# the five measured configurations
# ------------------------------------------------------------------------------------------------
def tiny() -> Workload:
    """64 docs x 1024 tokens, chunk 128, fp32; 16 query tokens; docs 17 and 42 planted at chunk 5."""
    return Workload("tiny", SEED_BASE + 0, np.full(64, 1024), 128, "f32", n_q=1, T0=16, k=4,
                    plant_kind="tiny", plant_args={"docs": [(17, 5, 3), (42, 5, 3)]})


def mem_1m() -> Workload:
    """1,000 docs, lengths uniform over the 13 multiples of 128 in [256, 1792]; bf16; 64 query tokens."""
    seed = SEED_BASE + 1
    lens = 256 + 128 * rng.uniform_int(seed, tid(PICK, 0, 999_999), 1000, 13).astype(np.int64)
    return Workload("1m", seed, lens, 128, "bf16", n_q=1, T0=64, k=8, plant_kind="mix", plant_args={"n": 8})


def mem_10m(n_docs: int = 9766) -> Workload:
    """9,766 docs x 1024 tokens, chunk 256, bf16; 32 queries of one decode token, 4 planted docs each.
    A smaller n_docs keeps the shapes with a shorter bank (profiling of a small case)."""
    return Workload("10m", SEED_BASE + 2, np.full(n_docs, 1024), 256, "bf16", n_q=32, T0=1, k=16,
                    plant_kind="per_query", plant_args={"per_query": 4})


def mem_100m(layers: int = 18, n_host_banks: int = 2, n_docs: int = 97657) -> Workload:
    """781,250 pre-pooled chunks (chunk 128; 97,656 docs of 1024 tokens + one of 256); 18 routed layers.
    A smaller n_docs keeps the same shapes with a shorter bank (profiling of a small case)."""
    lens = np.full(n_docs, 1024)
    lens[-1] = 256
    return Workload("100m", SEED_BASE + 3, lens, 128, "bf16", n_q=1, T0=64, k=16, prepooled=True,
                    layers=layers, n_host_banks=n_host_banks, plant_kind="single", plant_args={"n": 16})


def interleave(layers: int = 18, n_host_banks: int = 2) -> Workload:
    """10M-token pre-pooled bank (9,766 docs x 8 chunks of 128); 8 queries; 3 rounds of +32 tokens."""
    return Workload("interleave", SEED_BASE + 4, np.full(9766, 1024), 128, "bf16", n_q=8, T0=64, k=12,
                    prepooled=True, layers=layers, rounds=3, T_new=32, n_host_banks=n_host_banks,
                    plant_kind="chain")


def train64k() -> Workload:
    """Training context: 16 docs x 4096 tokens (65,536), chunk 128, bf16; one query of 512 tokens that
    routes and attends (causal over itself); top-4; 2 planted documents (the router's evidence)."""
    return Workload("train64k", SEED_BASE + 5, np.full(16, 4096), 128, "bf16", n_q=1, T0=512, k=4,
                    plant_kind="single", plant_args={"n": 2})


CONFIGS = {"tiny": tiny, "1m": mem_1m, "10m": mem_10m, "100m": mem_100m, "interleave": interleave,
           "train64k": train64k}
