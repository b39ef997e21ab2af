"""Kernel-level parity of the CUDA path (through the C ABI) against the fp64 oracle, on seeded
inputs sized to span several tiles with ragged tails, plus the edge cases of each step."""
import numpy as np
import pytest
import torch

import oracle as O
from msa_inputs import rng
from msa_inputs.device import upload

pytestmark = pytest.mark.gpu

SEED = 0x5EED


@pytest.fixture(scope="module")
def m():
    import routed_long_context_b200 as m

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _gen(tid, shape, dtype="f32", sigma=1.0):
    return rng.normal(SEED, tid, 0, int(np.prod(shape)), sigma, dtype).reshape(shape)


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def _close(got, ref, dtype, what):
    """fp32: |err| <= 1e-5 (values are O(1)); bf16 outputs: one rounding of 2^-9 relative plus fp32 error."""
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    if dtype == "f32":
        tol = 1e-5 + 1e-6 * np.abs(ref)
    else:
        tol = 2.0 ** -8 * np.abs(ref) + 1e-5
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance, max err {np.abs(got - ref).max():.3g}"


def _status(m):
    assert m.device_status() == 0


# -------------------------------------------------------------------------------------- generator
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_device_generator_matches_host_bitwise(m, dtype):
    n, start = 1_000_003, 12345
    t = torch.empty(n, dtype=torch.float32 if dtype == "f32" else torch.bfloat16, device="cuda")
    rng.fill_device(t, 99, 7, start=start, sigma=0.5)
    host = rng.normal(99, 7, start, n, 0.5, dtype)
    np.testing.assert_array_equal(t.float().cpu().numpy(), host)


# -------------------------------------------------------------------------------------- RoPE
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_rope_doc_segments_and_offset(m, dtype):
    off = np.array([0, 300, 300, 555, 1000], dtype=np.int64)        # includes an empty segment
    x = _gen(1, (1000, 8, 128), dtype)
    cs = m.rope_table(2048, 128, 1e6)
    for pos_offset in (0, 12):
        xd = upload(x, dtype)
        out = torch.empty_like(xd)
        m.msa_rope_doc(xd, torch.from_numpy(off).cuda(), pos_offset, cs, out=out)
        ref = O.apply_rope(x, O.doc_positions(off) + pos_offset, 1e6)
        _close(_np(out), ref, dtype, f"rope offset {pos_offset}")
    # in place gives the same bits
    xd = upload(x, dtype)
    m.msa_rope_doc(xd, torch.from_numpy(off).cuda(), 12, cs)
    assert torch.equal(xd, out)
    _status(m)


def test_rope_position_past_table_is_flagged_not_faulted(m):
    x = upload(_gen(2, (10, 1, 128)), "f32")
    cs = m.rope_table(8, 128, 1e6)
    m.msa_rope_doc(x, torch.tensor([0, 10], device="cuda"), 0, cs)
    assert m.device_status() == 1          # MSA_DEV_ROPE_POSITION, rows 8 and 9 left unrotated
    assert m.device_status() == 0          # the word is cleared by the read


# -------------------------------------------------------------------------------------- pooling
RAGGED = [300, 128, 1, 129, 0, 257, 1024, 77]


@pytest.mark.parametrize("in_dt,out_dt", [("f32", "f32"), ("bf16", "bf16"), ("f32", "bf16"), ("bf16", "f32")])
def test_pool_chunks_ragged_documents(m, in_dt, out_dt):
    from routed_long_context_b200.bank import BankLayout

    chunk = 128
    lay = BankLayout.from_doc_lengths(RAGGED, chunk)
    n_tok = sum(RAGGED)
    k, v, kr = (_gen(10 + i, (n_tok, 8, 128), in_dt) for i in range(3))
    cs = m.rope_table(2048, 128, 1e6)
    odt = torch.float32 if out_dt == "f32" else torch.bfloat16
    kvbar, idx = m.msa_pool_chunks(upload(k, in_dt), upload(v, in_dt), upload(kr, in_dt), lay.doc_tok_off,
                                   lay.doc_chunk_off, lay.chunk_doc, chunk, cos_sin=cs, out_dtype=odt)
    kb, vb, krb = O.encode_memory(k, v, kr, lay.doc_tok_off_host, chunk, 1e6)
    dco, _ = O.chunk_layout(lay.doc_tok_off_host, chunk)
    np.testing.assert_array_equal(dco, lay.doc_chunk_off_host)
    np.testing.assert_array_equal(lay.chunk_doc.cpu().numpy(), np.repeat(np.arange(len(RAGGED)), np.diff(dco)))
    _close(_np(kvbar[:, 0]), kb, out_dt, "K-bar")
    _close(_np(kvbar[:, 1]), vb, out_dt, "V-bar")
    _close(_np(idx), O.unit(krb), out_dt, "router index")
    _status(m)


@pytest.mark.parametrize("in_dt,out_dt", [("bf16", "bf16"), ("f32", "f32"), ("bf16", "f32"), ("f32", "bf16")])
@pytest.mark.parametrize("pipeline", [(0, 0, 0), (2, 4096, 0), (3, 5120, 0), (16, 12288, 0), (6, 16384, 2048),
                                      (4, 16384, 1040)])
def test_pool_bulk_copy_kernel_matches_register_kernel_bitwise(m, in_dt, out_dt, pipeline):
    """The bulk-copy pipeline and the register-streaming kernel sum every element in token order with
    the same rotation: identical bits, for ragged documents, router heads != K/V heads and pipeline
    shapes whose stages hold one row, a row and a half (the rest unused) or several rows, filled by
    one copy or by several (of whole rows; a copy size below one row still copies a row)."""
    from routed_long_context_b200.bank import BankLayout

    chunk = 96
    lay = BankLayout.from_doc_lengths(RAGGED, chunk)
    n_tok = sum(RAGGED)
    k, v = (upload(_gen(60 + i, (n_tok, 8, 128), in_dt), in_dt) for i in range(2))
    kr = upload(_gen(62, (n_tok, 4, 128), in_dt), in_dt)
    cs = m.rope_table(2048, 128, 1e6)
    odt = torch.float32 if out_dt == "f32" else torch.bfloat16
    got = []
    try:
        for impl in (1, 2):             # register streaming, bulk copies
            m.pool_set_impl(impl)
            m.pool_set_pipeline(*pipeline)
            got.append(m.msa_pool_chunks(k, v, kr, lay.doc_tok_off, lay.doc_chunk_off, lay.chunk_doc, chunk,
                                         cos_sin=cs, out_dtype=odt))
    finally:
        m.pool_set_impl(0)
        m.pool_set_pipeline(0, 0, 0)
    torch.cuda.synchronize()
    _status(m)
    for other in got[1:]:
        assert torch.equal(got[0][0], other[0]) and torch.equal(got[0][1], other[1])
    kb, vb, krb = O.encode_memory(_np(k), _np(v), _np(kr), lay.doc_tok_off_host, chunk, 1e6)
    _close(_np(got[1][0][:, 0]), kb, out_dt, "K-bar")
    _close(_np(got[1][1]), O.unit(krb), out_dt, "router index")


def test_pool_document_translation_invariance_bitwise(m):
    """Document-wise positions: a document's pooled, rotated K-bar is bit-identical wherever it sits."""
    from routed_long_context_b200.bank import BankLayout

    lens = [200, 300, 130]
    docs = [_gen(20 + i, (n, 8, 128), "bf16") for i, n in enumerate(lens)]
    cs = m.rope_table(2048, 128, 1e6)
    got = []
    for order in ([0, 1, 2], [2, 0, 1]):
        lay = BankLayout.from_doc_lengths([lens[i] for i in order], 64)
        k = upload(np.concatenate([docs[i] for i in order]), "bf16")
        kvbar, _ = m.msa_pool_chunks(k, k, None, lay.doc_tok_off, lay.doc_chunk_off, lay.chunk_doc, 64, cos_sin=cs)
        w = order.index(1)
        got.append(kvbar[lay.doc_chunk_off_host[w]:lay.doc_chunk_off_host[w + 1], 0].clone())
    assert torch.equal(got[0], got[1])


@pytest.mark.parametrize("in_dt,out_dt", [("bf16", "bf16"), ("f32", "f32"), ("bf16", "f32")])
def test_pool_and_route_with_large_magnitude_values(m, in_dt, out_dt):
    """The seeded generator stops at +-3.46 sigma; here 1% of the token elements (and of the router
    queries) are replaced by spikes of +-6 to +-1024 (exact in bf16), so pooling, the rotation, the
    index normalisation and the router's contraction are checked against the oracle over a wide
    range of magnitudes, on ragged documents."""
    from routed_long_context_b200.bank import BankLayout

    chunk = 128
    lay = BankLayout.from_doc_lengths(RAGGED, chunk)
    n_tok = sum(RAGGED)

    def spiked(tid, shape, dt):
        x = _gen(tid, shape, dt).reshape(-1)
        n = x.size // 100
        pos = rng.uniform_int(SEED, 5000 + tid, n, x.size).astype(np.int64)
        mag = np.array([6.0, 12.0, 100.0, 1024.0], dtype=np.float32)[rng.uniform_int(SEED, 6000 + tid, n, 4)]
        sign = np.where(rng.uniform_int(SEED, 7000 + tid, n, 2) == 0, -1.0, 1.0).astype(np.float32)
        x[pos] = mag * sign
        return x.reshape(shape)

    k, v, kr = (spiked(70 + i, (n_tok, 8, 128), in_dt) for i in range(3))
    cs = m.rope_table(2048, 128, 1e6)
    odt = torch.float32 if out_dt == "f32" else torch.bfloat16
    kvbar, idx = m.msa_pool_chunks(upload(k, in_dt), upload(v, in_dt), upload(kr, in_dt), lay.doc_tok_off,
                                   lay.doc_chunk_off, lay.chunk_doc, chunk, cos_sin=cs, out_dtype=odt)
    kb, vb, krb = O.encode_memory(k, v, kr, lay.doc_tok_off_host, chunk, 1e6)
    _close(_np(kvbar[:, 0]), kb, out_dt, "K-bar")
    _close(_np(kvbar[:, 1]), vb, out_dt, "V-bar")
    _close(_np(idx), O.unit(krb), out_dt, "router index")
    qr = spiked(80, (2, 7, 8, 128), out_dt)
    ds = m.msa_route_scores(idx, lay.chunk_doc, lay.n_docs, upload(qr, out_dt))
    # the oracle scores the index as stored (each head a unit vector up to its rounding)
    ref, _ = O.route(_np(idx), lay.doc_chunk_off_host, qr)
    tol = 1e-5 if out_dt == "f32" else 2e-3
    assert np.nanmax(np.abs(np.where(np.isfinite(ref), _np(ds) - ref, 0.0))) <= tol
    assert np.array_equal(np.isfinite(ref), np.isfinite(_np(ds)))
    _status(m)


# -------------------------------------------------------------------------------------- routing
def _route_case(C_docs_seed, n_q, T, dtype, n_docs=140):
    counts = 1 + rng.uniform_int(SEED, 900 + C_docs_seed, n_docs, 12).astype(np.int64)   # 1..12 chunks per doc
    C = int(counts.sum())
    raw = _gen(30 + C_docs_seed, (C, 8, 128))
    index = rng.round_to(O.unit(raw).astype(np.float32), dtype).reshape(C, 8, 128)
    qr = _gen(40 + C_docs_seed, (n_q, T, 8, 128), dtype)
    # plant: the first chunk of doc 3 equals query 0 token T-1 (so a score of ~1 exists)
    off = np.zeros(n_docs + 1, dtype=np.int64)
    np.cumsum(counts, out=off[1:])
    index[off[3]] = rng.round_to(O.unit(qr[0, T - 1]).astype(np.float32), dtype)
    return counts, off, index, qr


@pytest.mark.parametrize("n_q,T", [(1, 5), (3, 5), (2, 16), (1, 33)])
def test_route_fp32_cuda_cores(m, n_q, T):
    from routed_long_context_b200.bank import BankLayout

    counts, off, index, qr = _route_case(n_q * 100 + T, n_q, T, "f32")
    lay = BankLayout(counts)
    ds, cs_ = m.msa_route_scores(upload(index, "f32"), lay.chunk_doc, lay.n_docs, upload(qr, "f32"),
                                 want_chunk_scores=True)
    ref_ds, ref_cs = O.route(index, off, qr)
    assert np.abs(_np(ds) - ref_ds).max() <= 1e-5
    assert np.abs(_np(cs_) - ref_cs).max() <= 1e-5
    assert np.all(_np(ds) <= 1 + 1e-5) and np.all(_np(ds) >= -1 - 1e-5)
    assert abs(_np(ds)[0, 3] - 1.0) < 1e-5
    _status(m)


# (n_q, T) with T dividing 32 take the epilogue that reduces whole queries per 32-column piece:
# padded column blocks (N = 3, 20), two query-column tiles (N = 288, 300, 320) and T = 1..32
@pytest.mark.parametrize("n_q,T", [(1, 16), (1, 64), (2, 48), (3, 100), (32, 1), (8, 128), (1, 3), (3, 1), (5, 4),
                                   (7, 2), (9, 32), (20, 16), (300, 1), (4, 8)])
@pytest.mark.parametrize("impl", [2, 1, 3])
def test_route_bf16_tensor_cores_and_cuda_cores(m, n_q, T, impl):
    from routed_long_context_b200.bank import BankLayout

    counts, off, index, qr = _route_case(n_q * 1000 + T, n_q, T, "bf16")
    lay = BankLayout(counts)
    m.route_set_impl(impl)          # 2 tensor cores, 1 CUDA cores, 3 tensor cores with resident qhat
    try:
        ds, cs_ = m.msa_route_scores(upload(index, "bf16"), lay.chunk_doc, lay.n_docs, upload(qr, "bf16"),
                                     want_chunk_scores=True)
    finally:
        m.route_set_impl(0)
    ref_ds, ref_cs = O.route(index, off, qr)
    err_d, err_c = np.abs(_np(ds) - ref_ds).max(), np.abs(_np(cs_) - ref_cs).max()
    assert err_d <= 2e-3 and err_c <= 2e-3, (err_d, err_c)
    assert abs(_np(ds)[0, 3] - 1.0) < 2e-3
    _status(m)


def test_route_many_tiles_with_ragged_tail(m):
    """13,001 chunks (101 full 128-row tiles plus a 73-row tail) through the tensor-core path."""
    from routed_long_context_b200.bank import BankLayout

    counts = np.full(1626, 8, dtype=np.int64)
    counts[-1] = 1
    C = int(counts.sum())
    assert C % 128 == 73
    lay = BankLayout(counts)
    index = rng.round_to(O.unit(_gen(50, (C, 8, 128))).astype(np.float32), "bf16").reshape(C, 8, 128)
    qr = _gen(51, (1, 64, 8, 128), "bf16")
    index[C - 1] = rng.round_to(O.unit(qr[0, 7]).astype(np.float32), "bf16")     # plant in the tail row
    ds = m.msa_route_scores(upload(index, "bf16"), lay.chunk_doc, lay.n_docs, upload(qr, "bf16"))
    ref, _ = O.route(index, lay.doc_chunk_off_host, qr)
    assert np.abs(_np(ds) - ref).max() <= 2e-3
    assert _np(ds)[0, -1] > 0.99
    _status(m)


# -------------------------------------------------------------------------------------- top-k
@pytest.mark.parametrize("n_q,D,k", [(1, 1, 1), (1, 7, 7), (3, 1000, 4), (32, 9766, 16), (1, 97657, 16),
                                     (2, 5000, 33), (2, 5000, 64), (8, 2000, 12)])
def test_topk_exact_with_ties(m, n_q, D, k):
    s = np.round(_gen(60 + D + k, (n_q, D)) * 4) / 4                 # coarse grid: many exact ties
    s[:, ::17] = -np.inf
    idx, val = m.msa_topk_docs(torch.from_numpy(s.astype(np.float32)).cuda(), k)
    ref_i, ref_v = O.topk_docs(s.astype(np.float32), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_i)
    np.testing.assert_array_equal(val.cpu().numpy(), ref_v.astype(np.float32))


@pytest.mark.parametrize("pattern", ["ascending", "descending", "all_equal", "few_finite", "sawtooth"])
@pytest.mark.parametrize("n_q,D,k", [(1, 97657, 16), (2, 8192, 32), (3, 8193, 1), (1, 16385, 7), (4, 600, 5),
                                     (1, 131072, 32), (2, 131073, 16)])
def test_topk_exact_on_adversarial_orders(m, pattern, n_q, D, k):
    """Orders that defeat a pruning threshold: the best entries last (every round brings better
    candidates), all scores equal (ties decided by index alone), nearly all -inf, and a sawtooth
    whose teeth all reach the same maximum. One block per query up to 8,192 docs, a cluster of up to
    16 blocks up to 131,072, the ticket fold above."""
    base = np.arange(D, dtype=np.float64)
    if pattern == "ascending":
        row = base / D
    elif pattern == "descending":
        row = 1.0 - base / D
    elif pattern == "all_equal":
        row = np.zeros(D)
    elif pattern == "few_finite":
        row = np.full(D, -np.inf)
        row[(np.arange(k + 3) * 7919) % D] = np.linspace(0.0, 1.0, k + 3)
    else:
        row = (base % 97) / 96.0
    s = np.stack([np.roll(row, 13 * q) for q in range(n_q)]).astype(np.float32)
    idx, val = m.msa_topk_docs(torch.from_numpy(s).cuda(), k)
    ref_i, ref_v = O.topk_docs(s, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_i)
    np.testing.assert_array_equal(val.cpu().numpy(), ref_v.astype(np.float32))
    _status(m)


def test_topk_repeatable(m):
    s = torch.from_numpy((np.round(_gen(70, (4, 50000)) * 8) / 8).astype(np.float32)).cuda()
    a, _ = m.msa_topk_docs(s, 16)
    b, _ = m.msa_topk_docs(s, 16)
    assert torch.equal(a, b)


# -------------------------------------------------------------------------------------- gather
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gather_is_exact(m, dtype):
    counts = np.array([3, 1, 4, 0, 2, 5], dtype=np.int64)
    off = np.concatenate([[0], np.cumsum(counts)])
    bank = torch.from_numpy(_gen(80, (int(off[-1]), 2, 8, 128), dtype)).to(
        torch.float32 if dtype == "f32" else torch.bfloat16).pin_memory()
    idx = torch.tensor([[2, 0, 5], [3, 1, 4]], dtype=torch.int32)
    dev, mem_len = m.msa_gather_kv(bank, off, idx, max_mem=12)
    torch.cuda.synchronize()
    assert mem_len.tolist() == [12, 3]
    ref = O.gather_memory(bank.float().numpy(), off, [2, 0, 5])
    np.testing.assert_array_equal(dev[0, :12].float().cpu().numpy(), ref)
    np.testing.assert_array_equal(dev[1, :3].float().cpu().numpy(), O.gather_memory(bank.float().numpy(), off, [3, 1, 4]))


# -------------------------------------------------------------------------------------- attention
def _row_rel_err(got, ref):
    num = np.linalg.norm(got - ref, axis=-1)
    den = np.maximum(np.linalg.norm(ref, axis=-1), 1e-30)
    return (num / den).max()


@pytest.mark.parametrize("dtype,impl", [("f32", 0), ("bf16", 0), ("bf16", 1)])
@pytest.mark.parametrize("hq,hkv", [(32, 8), (8, 8), (16, 8), (32, 4)])
@pytest.mark.parametrize("T,max_mem,mem_lens,q_start", [(13, 40, (0, 5, 37), 7), (37, 140, (130, 64, 1), 50)])
def test_sparse_attention(m, dtype, impl, hq, hkv, T, max_mem, mem_lens, q_start):
    """Both bf16 kernels (tensor cores, CUDA cores) and fp32; one key tile and several key tiles
    with ragged tails, rows past the end of a 64-row block, empty memory."""
    n_q, d = 3, 128
    L = q_start + T
    q = _gen(90, (n_q, T, hq, d), dtype)
    mem = _gen(91, (n_q, max_mem, 2, hkv, d), dtype)
    lk, lv = _gen(92, (n_q, L + 3, hkv, d), dtype), _gen(93, (n_q, L + 3, hkv, d), dtype)
    mem_len = np.array(mem_lens, dtype=np.int32)
    m.attn_set_impl(impl)
    try:
        out = m.msa_sparse_attn(upload(q, dtype), upload(mem, dtype), torch.from_numpy(mem_len).cuda(),
                                upload(lk, dtype), upload(lv, dtype), L, q_start)
    finally:
        m.attn_set_impl(0)
    got = _np(out)
    tol = 1e-5 if dtype == "f32" else 2e-2
    for qi in range(n_q):
        ml = mem_len[qi]
        ref = O.sparse_attention(q[qi], mem[qi, :ml, 0], mem[qi, :ml, 1], lk[qi, :L], lv[qi, :L], q_start,
                                 1 / np.sqrt(d))
        assert _row_rel_err(got[qi], ref) <= tol


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_device_gather_matches_host_gather(m, dtype):
    counts = np.array([3, 1, 4, 0, 2, 5, 8, 8], dtype=np.int64)
    off = np.concatenate([[0], np.cumsum(counts)])
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    bank = torch.from_numpy(_gen(81, (int(off[-1]), 2, 8, 128), dtype)).to(tdt).pin_memory()
    idx = torch.tensor([[2, 0, 5], [3, 1, 4], [7, 6, 0]], dtype=torch.int32)
    ref, ref_len = m.msa_gather_kv(bank, off, idx, max_mem=20)
    dev, dev_len = m.msa_gather_kv_device(bank, torch.from_numpy(off).cuda(), idx.cuda(), max_mem=20)
    torch.cuda.synchronize()
    assert dev_len.cpu().tolist() == ref_len.tolist() == [12, 3, 19]
    for q, n in enumerate(ref_len.tolist()):
        assert torch.equal(dev[q, :n].cpu(), ref[q, :n].cpu())
    _status(m)


def test_device_gather_flags_bad_index_without_faulting(m):
    bank = torch.zeros((10, 2, 8, 128), dtype=torch.bfloat16).pin_memory()
    off = torch.tensor([0, 4, 10], dtype=torch.int64, device="cuda")
    idx = torch.tensor([[1, 5]], dtype=torch.int32, device="cuda")     # doc 5 does not exist
    m.msa_gather_kv_device(bank, off, idx, max_mem=16)
    assert m.device_status() == 3                                      # MSA_DEV_BAD_INDEX


def test_sparse_attention_no_keys_gives_zero(m):
    q = upload(_gen(94, (1, 4, 32, 128)), "f32")
    mem = torch.zeros((1, 4, 2, 8, 128), device="cuda")
    lk = torch.zeros((1, 4, 8, 128), device="cuda")
    out = m.msa_sparse_attn(q, mem, torch.zeros(1, dtype=torch.int32, device="cuda"), lk, lk, 0, 0)
    assert torch.count_nonzero(out) == 0


# -------------------------------------------------------------------------------------- fine stage
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_pack_tokens_matches_oracle(m, dtype):
    """Token bank of the fine stage: keys rotated to their position inside their document, values
    copied bit for bit; empty and one-token documents included."""
    off = np.array([0, 300, 300, 555, 1000, 1001], dtype=np.int64)
    n, hkv, d = int(off[-1]), 8, 128
    k, v = _gen(100, (n, hkv, d), dtype), _gen(101, (n, hkv, d), dtype)
    cs = m.rope_table(1024, d, 1e6)
    bank = m.msa_pack_tokens(upload(k, dtype), upload(v, dtype), torch.from_numpy(off).cuda(), cs)
    _status(m)
    ref = O.token_bank(k, v, off, 1e6)
    _close(_np(bank[:, 0]), ref[:, 0], dtype, "token bank K")
    np.testing.assert_array_equal(_np(bank[:, 1]), v)


def test_pack_tokens_position_past_table_is_flagged_not_faulted(m):
    off = np.array([0, 40], dtype=np.int64)
    k = upload(_gen(106, (40, 8, 128)), "f32")
    m.msa_pack_tokens(k, k, torch.from_numpy(off).cuda(), m.rope_table(32, 128, 1e6))
    assert m.device_status() == 1                                      # MSA_DEV_ROPE_POSITION


def test_device_gather_token_rows_over_many_blocks(m):
    """Token-level documents (hundreds of rows each) are fetched by several blocks per document;
    the result equals the host-issued copies and the rank-ordered row copy."""
    lens = np.array([1000, 1792, 0, 256, 1500, 77], dtype=np.int64)
    off = np.concatenate([[0], np.cumsum(lens)])
    bank = torch.from_numpy(_gen(107, (int(off[-1]), 2, 8, 128), "bf16")).to(torch.bfloat16).pin_memory()
    idx = torch.tensor([[1, 0, 4], [3, 5, 2]], dtype=torch.int32)
    max_mem = 3 * 1792
    ref, ref_len = m.msa_gather_kv(bank, off, idx, max_mem=max_mem)
    dev, dev_len = m.msa_gather_kv_device(bank, torch.from_numpy(off).cuda(), idx.cuda(), max_mem=max_mem)
    torch.cuda.synchronize()
    assert dev_len.cpu().tolist() == ref_len.tolist() == [4292, 333]
    host = bank.float().numpy()
    for q, n in enumerate(ref_len.tolist()):
        assert torch.equal(dev[q, :n].cpu(), ref[q, :n].cpu())
        np.testing.assert_array_equal(dev[q, :n].float().cpu().numpy(), O.gather_memory(host, off, idx[q].tolist()))
    _status(m)


@pytest.mark.parametrize("impl", [0, 2, 3])
@pytest.mark.parametrize("hq,hkv", [(32, 8), (8, 8), (32, 4)])
@pytest.mark.parametrize("T,mem_lens,q_start", [(64, (0, 700, 1537), 0), (24, (4099, 1, 64), 40),
                                                (300, (130, 2200, 64), 5)])
def test_sparse_attention_split_long_memory(m, impl, hq, hkv, T, mem_lens, q_start):
    """Split-key attention over long memories, on tcgen05 with the key ranges merged in a thread-block
    cluster where the grid allows it (impl 0), on tcgen05 with partial results and a combine pass
    (impl 3), and on mma.sync (impl 2): several key ranges per block (some empty), ragged tails,
    empty memory, causal local keys, one and two 128-row blocks per CTA; against the oracle within
    the bf16 bound."""
    n_q, d, dtype = 3, 128, "bf16"
    max_mem = max(mem_lens) + 5
    L = q_start + T
    q = _gen(102, (n_q, T, hq, d), dtype)
    mem = _gen(103, (n_q, max_mem, 2, hkv, d), dtype)
    lk, lv = _gen(104, (n_q, L + 3, hkv, d), dtype), _gen(105, (n_q, L + 3, hkv, d), dtype)
    mem_len = np.array(mem_lens, dtype=np.int32)
    rows = n_q * T * hq
    if T < 300:   # short query blocks: the memory is split into several key ranges
        assert m.sparse_attn_split_workspace_size(n_q, T, hq, hkv, max_mem, L) >= 2 * rows * (d * 4 + 8)
    m.attn_set_impl(impl)
    try:
        plan = m.api.sparse_attn_split_plan(n_q, T, hq, hkv, max_mem, L)
        natural = 2 if T * (hq // hkv) > 128 else 1
        if impl == 2:
            assert plan["row_blocks"] == 0 and plan["cluster"] == 0
        elif impl == 3 or plan["cluster"] == 0:
            assert plan["row_blocks"] == natural and plan["cluster"] == 0 if impl == 3 else plan["row_blocks"] == natural
        else:
            assert plan["row_blocks"] in (1, natural) and plan["key_ranges"] == plan["cluster"]
        lse = torch.empty((n_q, T, hq), dtype=torch.float32, device="cuda")
        out = m.msa_sparse_attn_split(upload(q, dtype), upload(mem, dtype), torch.from_numpy(mem_len).cuda(),
                                      upload(lk, dtype), upload(lv, dtype), L, q_start, lse=lse)
    finally:
        m.attn_set_impl(0)
    _status(m)
    got = _np(out)
    scale = 1 / np.sqrt(d)
    for qi in range(n_q):
        ml = mem_len[qi]
        ref = O.sparse_attention(q[qi], mem[qi, :ml, 0], mem[qi, :ml, 1], lk[qi, :L], lv[qi, :L], q_start, scale)
        assert _row_rel_err(got[qi], ref) <= 2e-2
        # the log-sum-exp of each row's logits (merged in the cluster or by the combine pass)
        ref_lse = np.empty((T, hq))
        for h in range(hq):
            g_ = h // (hq // hkv)
            keys = np.concatenate([mem[qi, :ml, 0, g_], lk[qi, :L, g_]])
            lg = (q[qi, :, h].astype(np.float64) @ keys.T.astype(np.float64)) * scale
            vis = np.ones_like(lg, dtype=bool)
            vis[:, ml:] = np.arange(L)[None, :] <= q_start + np.arange(T)[:, None]
            lg = np.where(vis, lg, -np.inf)
            mx = lg.max(axis=1)
            ref_lse[:, h] = mx + np.log(np.exp(lg - mx[:, None]).sum(axis=1))
        np.testing.assert_allclose(_np(lse[qi]), ref_lse, atol=2e-3)


@pytest.mark.parametrize("T,hq,hkv", [(64, 32, 8), (24, 32, 8), (100, 16, 8)])
def test_sparse_attention_split_one_query_long_memory(m, T, hq, hkv):
    """One query over a long memory (the fine stage's layout: 8 kv heads, 18 key ranges per head,
    more than one co-resident cluster holds): the default plan against the oracle within the bf16
    bound, and its log-sum-exp against the partials + combine path (impl 3)."""
    n_q, d, dtype, q_start = 1, 128, "bf16", 3
    mem_len = np.array([5000], dtype=np.int32)
    max_mem = 5003
    L = q_start + T
    q = _gen(130, (n_q, T, hq, d), dtype)
    mem = _gen(131, (n_q, max_mem, 2, hkv, d), dtype)
    lk, lv = _gen(132, (n_q, L, hkv, d), dtype), _gen(133, (n_q, L, hkv, d), dtype)
    args = (upload(q, dtype), upload(mem, dtype), torch.from_numpy(mem_len).cuda(), upload(lk, dtype),
            upload(lv, dtype), L, q_start)
    plan = m.api.sparse_attn_split_plan(n_q, T, hq, hkv, max_mem, L)
    lse0 = torch.empty((n_q, T, hq), dtype=torch.float32, device="cuda")
    out0 = m.msa_sparse_attn_split(*args, lse=lse0)
    m.attn_set_impl(3)
    try:
        lse3 = torch.empty((n_q, T, hq), dtype=torch.float32, device="cuda")
        out3 = m.msa_sparse_attn_split(*args, lse=lse3)
    finally:
        m.attn_set_impl(0)
    _status(m)
    assert plan["cluster"] == 0 or plan["key_ranges"] == plan["cluster"]
    ref = O.sparse_attention(q[0], mem[0, :5000, 0], mem[0, :5000, 1], lk[0], lv[0], q_start, 1 / np.sqrt(d))
    assert _row_rel_err(_np(out0)[0], ref) <= 2e-2
    assert _row_rel_err(_np(out3)[0], ref) <= 2e-2
    np.testing.assert_allclose(_np(lse0), _np(lse3), atol=1e-4)


def test_sparse_attention_split_no_keys_gives_zero_and_rejects_fp32(m):
    q = upload(_gen(108, (2, 4, 32, 128), "bf16"), "bf16")
    mem = torch.zeros((2, 300, 2, 8, 128), dtype=torch.bfloat16, device="cuda")
    lk = torch.zeros((2, 4, 8, 128), dtype=torch.bfloat16, device="cuda")
    out = m.msa_sparse_attn_split(q, mem, torch.zeros(2, dtype=torch.int32, device="cuda"), lk, lk, 0, 0)
    assert torch.count_nonzero(out) == 0
    with pytest.raises(m.MSAError):
        m.msa_sparse_attn_split(q.float(), mem.float(), torch.zeros(2, dtype=torch.int32, device="cuda"), lk.float(),
                                lk.float(), 0, 0)


# -------------------------------------------------------------------------------------- incremental append
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_growable_bank_append_equals_full_encode_bitwise(m, dtype):
    """Appending documents encodes only them and reproduces a from-scratch encode bit for bit; routing
    over the grown bank finds a planted document of the appended part."""
    from routed_long_context_b200.bank import BankLayout, GrowableBank, encode_tokens

    lens = np.array([300, 128, 1, 129, 257, 1024, 77, 640, 384, 200, 513, 90], dtype=np.int64)
    n_old = 7
    n_tok = int(lens.sum())
    cut = int(lens[:n_old].sum())
    k, v, kr = (_gen(300 + i, (n_tok, 8, 128), dtype) for i in range(3))
    qr = _gen(310, (2, 9, 8, 128), dtype)
    off = np.concatenate([[0], np.cumsum(lens)])
    d_plant = n_old + 1                                              # the second appended document
    kr[off[d_plant] + 128:off[d_plant] + 256] = rng.round_to(qr[1, 4], dtype)   # its whole chunk 1
    cs = m.rope_table(2048, 128, 1e6)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    full = BankLayout.from_doc_lengths(lens, 128)
    kv_ref, idx_ref = encode_tokens(full, upload(k, dtype), upload(v, dtype), upload(kr, dtype), 128, cs)

    bank = GrowableBank(full.n_chunks + 5, 8, 8, 128, dtype=tdt)
    s_old = bank.append(upload(k[:cut], dtype), upload(v[:cut], dtype), upload(kr[:cut], dtype), lens[:n_old], 128, cs)
    s_new = bank.append(upload(k[cut:], dtype), upload(v[cut:], dtype), upload(kr[cut:], dtype), lens[n_old:], 128, cs)
    torch.cuda.synchronize()
    assert s_old.start == 0 and s_new.stop == full.n_chunks
    np.testing.assert_array_equal(bank.doc_chunk_off_host, full.doc_chunk_off_host)
    assert torch.equal(bank.index[:full.n_chunks], idx_ref)
    assert torch.equal(bank.kvbar[:full.n_chunks], kv_ref)
    assert torch.equal(bank.layout.chunk_doc, full.chunk_doc)
    ds = m.msa_route_scores(bank.index[:bank.n_chunks], bank.layout.chunk_doc, bank.layout.n_docs, upload(qr, dtype))
    assert int(torch.argmax(ds[1])) == d_plant
    _status(m)


# -------------------------------------------------------------------------------------- output bounds
def _canaried(shape, dtype, pattern):
    """A tensor of `shape` that is the head of a larger buffer whose 4 KB tail holds `pattern` bits."""
    n = int(np.prod(shape))
    el = torch.empty((), dtype=dtype).element_size()
    extra = 4096 // el
    int_dt = {2: torch.int16, 4: torch.int32}[el]
    buf = torch.full((n + extra,), pattern, dtype=int_dt, device="cuda").view(dtype)
    return buf[:n].view(shape), buf, n


def _tail_intact(buf, n, pattern):
    int_dt = {2: torch.int16, 4: torch.int32}[buf.element_size()]
    return bool((buf[n:].view(int_dt) == pattern).all())


def test_new_kernels_write_nothing_past_their_outputs(m):
    """Canary words after the outputs of the token bank, the split attention (and its log-sum-exp),
    the attention backward, the Memory Parallel merge and the bulk-copy pooling stay untouched."""
    bf, f32 = torch.bfloat16, torch.float32
    n_q, T, hq, hkv, d, L = 2, 24, 32, 8, 128, 30
    mem_lens = np.array([700, 0], dtype=np.int32)
    max_mem = 704
    q = upload(_gen(120, (n_q, T, hq, d), "bf16"), "bf16")
    mem = upload(_gen(121, (n_q, max_mem, 2, hkv, d), "bf16"), "bf16")
    lk, lv = upload(_gen(122, (n_q, L, hkv, d), "bf16"), "bf16"), upload(_gen(123, (n_q, L, hkv, d), "bf16"), "bf16")
    ml = torch.from_numpy(mem_lens).cuda()
    out, ob, on = _canaried((n_q, T, hq, d), bf, 0x3C5A)
    lse, lb, ln_ = _canaried((n_q, T, hq), f32, 0x7FC0DEAD)
    m.msa_sparse_attn_split(q, mem, ml, lk, lv, L, 6, out=out, lse=lse)
    grads = [_canaried(s_, f32, 0x7FC0BEEF) for s_ in ((n_q, T, hq, d), (n_q, max_mem, 2, hkv, d), (n_q, L, hkv, d),
                                                        (n_q, L, hkv, d))]
    m.msa_sparse_attn_backward(q, mem, ml, lk, lv, L, 6, out, q, lse, grads=tuple(g_[0] for g_ in grads))
    off = np.array([0, 300, 300, 555, 1000], dtype=np.int64)
    kt = upload(_gen(124, (1000, hkv, d), "bf16"), "bf16")
    bank, bb, bn = _canaried((1000, 2, hkv, d), bf, 0x3C5A)
    m.msa_pack_tokens(kt, kt, torch.from_numpy(off).cuda(), m.rope_table(1024, d, 1e6), bank=bank)
    cand = torch.rand((3, 2, 16), device="cuda")
    cidx = torch.randint(0, 50, (3, 2, 16), dtype=torch.int32, device="cuda")
    midx, mb, mn = _canaried((2, 16), torch.int32, 0x5A5A5A5A)
    msc, sb, sn = _canaried((2, 16), f32, 0x7FC0DEAD)
    m.msa_topk_merge(cand, cidx, np.array([0, 50, 100, 150]), 16, idx=midx, score=msc)
    from routed_long_context_b200.bank import BankLayout
    play = BankLayout.from_doc_lengths([300, 0, 255, 445], 96)
    pkv, pkb, pkn = _canaried((play.n_chunks, 2, hkv, d), bf, 0x3C5A)
    pki, pib, pin_ = _canaried((play.n_chunks, hkv, d), bf, 0x3C5A)
    m.msa_pool_chunks(kt, kt, kt, play.doc_tok_off, play.doc_chunk_off, play.chunk_doc, 96,
                      cos_sin=m.rope_table(1024, d, 1e6), kvbar=pkv, kr_index=pki)
    torch.cuda.synchronize()
    _status(m)
    assert _tail_intact(pkb, pkn, 0x3C5A) and _tail_intact(pib, pin_, 0x3C5A)
    assert _tail_intact(ob, on, 0x3C5A) and _tail_intact(lb, ln_, 0x7FC0DEAD)
    for g_, b_, n_ in grads:
        assert _tail_intact(b_, n_, 0x7FC0BEEF)
    assert _tail_intact(bb, bn, 0x3C5A)
    assert _tail_intact(mb, mn, 0x5A5A5A5A) and _tail_intact(sb, sn, 0x7FC0DEAD)


@pytest.mark.parametrize("D", [600, 20000, 140000])
def test_topk_and_router_write_nothing_past_their_outputs(m, D):
    """Canary words after the top-k outputs (one block per query, one cluster per query, the ticket
    fold) and after the router's document and chunk scores at T = 1 (the transposed epilogue) with a
    ragged last tile stay untouched."""
    from routed_long_context_b200.bank import BankLayout

    f32 = torch.float32
    s = torch.rand((3, D), device="cuda")
    idx, ib, in_ = _canaried((3, 16), torch.int32, 0x5A5A5A5A)
    sc, sb, sn = _canaried((3, 16), f32, 0x7FC0DEAD)
    m.msa_topk_docs(s, 16, idx=idx, score=sc)
    counts = 1 + rng.uniform_int(SEED, 990, 100, 7).astype(np.int64)     # 1..7 chunks per doc
    lay = BankLayout(counts)
    C = int(counts.sum())
    index = upload(rng.round_to(O.unit(_gen(991, (C, 8, 128))).astype(np.float32), "bf16").reshape(C, 8, 128),
                   "bf16")
    qr = upload(_gen(992, (33, 1, 8, 128), "bf16"), "bf16")
    ds, db, dn = _canaried((33, lay.n_docs), f32, 0x7FC0DEAD)
    cs_, cb, cn = _canaried((33, C), f32, 0x7FC0DEAD)
    m.msa_route_scores(index, lay.chunk_doc, lay.n_docs, qr, doc_scores=ds, chunk_scores=cs_)
    torch.cuda.synchronize()
    _status(m)
    assert _tail_intact(ib, in_, 0x5A5A5A5A) and _tail_intact(sb, sn, 0x7FC0DEAD)
    assert _tail_intact(db, dn, 0x7FC0DEAD) and _tail_intact(cb, cn, 0x7FC0DEAD)
    ref_i, _ = O.topk_docs(s.cpu().numpy(), 16)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_i)
