"""Memory Parallel on one GPU: the shards of a layer are routed and selected one after the other in
this process (no rank waits on another), their packed lists merged by the library's merge kernel,
and the result compared bit for bit with one selection over the whole bank and with the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from msa_inputs import workloads
from msa_inputs.device import memory_tensor, small_tensors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    import routed_long_context_b200 as m

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _scores(n_q, D, seed=11):
    r = np.random.default_rng(seed)
    s = np.round(r.standard_normal((n_q, D)), 2).astype(np.float32)     # many exact ties
    s[:, 5000:5300] = 4.0                                                # a tie block spanning shards
    s[0, 17] = -np.inf
    counts = r.integers(1, 12, D)
    return s, np.concatenate([[0], np.cumsum(counts)])


@pytest.mark.parametrize("world", [1, 2, 3, 8])
@pytest.mark.parametrize("k,k_cand", [(16, 16), (8, 24), (1, 1)])
def test_merge_of_shard_lists_equals_one_topk(m, world, k, k_cand):
    from routed_long_context_b200.memory_parallel import merge_candidates, shard_bounds

    n_q, D = 4, 97657
    s, off = _scores(n_q, D)
    dev = torch.from_numpy(s).cuda()
    b = shard_bounds(off, world, k_cand)
    g = torch.empty((world, 2, n_q, k_cand), dtype=torch.int32, device="cuda")
    for r in range(world):
        part = dev[:, b[r]:b[r + 1]].contiguous()
        m.msa_topk_docs(part, k_cand, idx=g[r, 1], score=g[r, 0].view(torch.float32))
    idx, sc = merge_candidates(g, b, k)
    full_idx, full_sc = m.msa_topk_docs(dev, k)
    assert m.device_status() == 0
    assert torch.equal(idx, full_idx) and torch.equal(sc, full_sc)
    np.testing.assert_array_equal(idx.cpu().numpy(), O.topk_docs(s, k)[0])


def test_merge_empty_slots_short_lists_and_bad_index(m):
    """-1 slots count as no candidate; fewer candidates than k leave -1 / -inf; a local index outside
    its shard is flagged and skipped; -0 ties +0 and goes to the lower index; NaN ranks last."""
    bounds = np.array([0, 5, 9], dtype=np.int64)
    cs = torch.tensor([[[0.5, -0.0, float("nan")]], [[0.0, 0.25, 9.0]]], dtype=torch.float32, device="cuda")
    ci = torch.tensor([[[1, 0, 2]], [[3, -1, 2]]], dtype=torch.int32, device="cuda")
    idx, sc = m.msa_topk_merge(cs, ci, bounds, 7)
    assert idx.cpu().tolist() == [[7, 1, 0, 8, 2, -1, -1]]
    got = sc.cpu().numpy()[0]
    assert got[0] == 9.0 and got[1] == 0.5 and got[2] == 0.0 and got[3] == 0.0 and np.isnan(got[4])
    assert np.all(np.isneginf(got[5:]))
    assert m.device_status() == 0
    ci_bad = torch.tensor([[[1, 0, 7]], [[3, -1, 2]]], dtype=torch.int32, device="cuda")   # 7 is outside shard 0
    idx, _ = m.msa_topk_merge(cs, ci_bad, bounds, 4)
    assert idx.cpu().tolist() == [[7, 1, 0, 8]]
    assert m.device_status() == 3                                                       # MSA_DEV_BAD_INDEX


@pytest.mark.parametrize("world", [2, 8])
def test_sharded_routing_of_a_100m_layer_equals_the_whole_bank(m, world):
    """Every shard routes its rows of the 100M index; the merged selection is the unsharded one, scores
    included, bit for bit (a chunk's score does not depend on the tile it sits in)."""
    from routed_long_context_b200.bank import BankLayout, index_from_prepooled
    from routed_long_context_b200.memory_parallel import ShardRouter, merge_candidates

    w = workloads.mem_100m(layers=1, n_host_banks=1)
    lay = BankLayout(w.doc_chunks)
    index = index_from_prepooled(lay, memory_tensor(w, 0, "krbar"))
    qr = small_tensors(w, 0)["qr"]
    full_idx, full_sc = m.msa_topk_docs(m.msa_route_scores(index, lay.chunk_doc, lay.n_docs, qr), w.k)
    g = torch.empty((world, 2, w.n_q, w.k), dtype=torch.int32, device="cuda")
    for r in range(world):
        sh = ShardRouter(w.doc_chunk_off, index, world, r, w.n_q, w.T0, w.k)
        sh.select_local(qr, out=g[r])
    idx, sc = merge_candidates(g, sh.bounds, w.k)
    assert m.device_status() == 0
    assert torch.equal(idx, full_idx) and torch.equal(sc, full_sc)
    assert set(w.expected(0, 0, 0)) <= set(idx.cpu().numpy()[0].tolist())
    del index
    torch.cuda.empty_cache()


def test_memory_parallel_router_replays_in_a_cuda_graph(m):
    """A single-rank MemoryParallelRouter's selection (route, top-k, merge) captured once in a CUDA
    graph and replayed for new router queries gives the same selection as direct calls."""
    from routed_long_context_b200.bank import BankLayout, index_from_prepooled
    from routed_long_context_b200.memory_parallel import MemoryParallelRouter

    w = workloads.mem_100m(layers=1, n_host_banks=1, n_docs=12500)
    lay = BankLayout(w.doc_chunks)
    index = index_from_prepooled(lay, memory_tensor(w, 0, "krbar"))
    qr = small_tensors(w, 0)["qr"]
    router = MemoryParallelRouter(w.doc_chunk_off, index, w.n_q, w.T0, w.k)
    router.select(qr)                                                   # warm-up outside the capture
    torch.cuda.synchronize()
    qr_in = qr.clone()
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            idx_g, sc_g = router.select(qr_in)
    torch.cuda.current_stream().wait_stream(s)
    for seed in range(3):
        qr_in.copy_(torch.roll(qr, shifts=seed, dims=1))
        graph.replay()
        torch.cuda.synchronize()
        want_idx, want_sc = m.msa_topk_docs(m.msa_route_scores(index, lay.chunk_doc, lay.n_docs, qr_in), w.k)
        assert torch.equal(idx_g, want_idx) and torch.equal(sc_g, want_sc)
    assert m.device_status() == 0
