"""Memory Parallel host logic on CPU: shard boundaries, and two gloo ranks that each select their
shard's local top-k, exchange the packed lists with one all_gather and merge them into the global
top-k of the oracle. The merge kernel itself is covered by the GPU tests."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from routed_long_context_b200.memory_parallel import exchange_candidates, shard_bounds  # noqa: E402


def test_shard_bounds_cover_balance_and_hold_k_docs():
    r = np.random.default_rng(5)
    counts = r.integers(0, 12, 1000)                    # includes documents with no chunk
    off = np.concatenate([[0], np.cumsum(counts)])
    for world in (1, 2, 3, 8):
        for k in (1, 16):
            b = shard_bounds(off, world, k)
            assert b[0] == 0 and b[-1] == 1000 and np.all(np.diff(b) >= k)
            chunks = np.diff(off[b])
            assert chunks.sum() == off[-1]
            assert np.abs(chunks - off[-1] / world).max() <= counts.max() + 1
    with pytest.raises(ValueError):
        shard_bounds(off[:6], 2, 3)                      # 5 documents cannot give 2 shards of 3


def test_shard_bounds_respect_k_when_chunks_are_skewed():
    counts = np.array([1000] + [1] * 40)                 # one huge document first
    off = np.concatenate([[0], np.cumsum(counts)])
    b = shard_bounds(off, 4, 8)
    assert np.all(np.diff(b) >= 8) and b[-1] == 41


def test_single_process_exchange_is_the_local_list():
    send = torch.arange(24, dtype=torch.int32).reshape(2, 3, 4)
    g = exchange_candidates(send)
    assert g.shape == (1, 2, 3, 4) and torch.equal(g[0], send)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _scores(n_q, D):
    r = np.random.default_rng(7)
    s = np.round(r.standard_normal((n_q, D)), 2).astype(np.float32)     # rounding plants many exact ties
    s[:, 120:180] = 3.0                                                  # a tie block across shard boundaries
    counts = r.integers(1, 9, D)
    return s, np.concatenate([[0], np.cumsum(counts)])


def _worker(rank, world, port, k, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import oracle as O

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        n_q, D = 3, 500
        s, off = _scores(n_q, D)
        b = shard_bounds(off, world, k)
        d0, d1 = int(b[rank]), int(b[rank + 1])
        li, lv = O.topk_docs(s[:, d0:d1], k)                             # this shard's local top-k
        send = torch.empty((2, n_q, k), dtype=torch.int32)
        send[0] = torch.from_numpy(lv.astype(np.float32)).view(torch.int32)
        send[1] = torch.from_numpy(li.astype(np.int32))
        g = exchange_candidates(send)
        assert g.shape == (world, 2, n_q, k)
        cs = g[:, 0].contiguous().view(torch.float32).numpy().astype(np.float64)
        ci = g[:, 1].numpy().astype(np.int64) + b[:-1, None, None]          # global document indices
        merged = []
        for q in range(n_q):
            sc, gi = cs[:, q].ravel(), ci[:, q].ravel()
            order = np.lexsort((gi, -sc))                                # score desc, then global index
            merged.append(gi[order[:k]].tolist())
        out[rank] = (merged, O.topk_docs(s, k)[0].tolist())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,k", [(2, 16), (3, 8)])
def test_ranks_merge_to_the_global_topk(world, k):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), k, out), nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        merged, want = out[r]
        assert merged == want
    assert all(out[r][0] == out[0][0] for r in range(world))
