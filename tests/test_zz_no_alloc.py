"""The allocation-free top-k entry point.

Some callers of this library cannot allocate device memory at the moment they select documents
(a host application that loads the library as a plugin and passes only its own buffers, a serving
loop whose memory is reserved up front, a latency-bound loop that cannot take cudaMalloc's
implicit synchronisation). msa_topk_docs_noalloc serves them from a fixed device array inside the
library. This file checks, through the C ABI, that it returns what the workspace-based
msa_topk_docs and the oracle return, on consecutive calls that reuse the array, that calls after the
first take no device memory, and that it refuses sizes that do not fit. It sits last in collection
order so a failure here never hides another test's result.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from msa_inputs import rng

pytestmark = pytest.mark.gpu


def _scores(seed, n_q, n_docs):
    s = rng.normal(0xA110C, seed, 0, n_q * n_docs).reshape(n_q, n_docs)
    s = np.round(s * 8) / 8                      # coarse grid: exact ties exercise the tie rule
    s[:, ::29] = -np.inf
    return torch.from_numpy(s.astype(np.float32)).cuda()


def _noalloc(lib, scores, k):
    n_q, n_docs = scores.shape
    idx = torch.full((n_q, k), -1, dtype=torch.int32, device="cuda")
    val = torch.full((n_q, k), float("nan"), dtype=torch.float32, device="cuda")
    st = lib.msa_topk_docs_noalloc(ctypes.c_void_p(scores.data_ptr()), n_q, n_docs, k,
                                   ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(val.data_ptr()),
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, lib.msa_last_error()
    return idx, val


def test_noalloc_topk_matches_workspace_topk_on_consecutive_calls():
    import routed_long_context_b200 as m
    from routed_long_context_b200 import _lib

    lib = _lib.lib
    assert lib.msa_topk_noalloc_max_scratch() == 1 << 20
    cases = [(3, 97657, 16), (3, 97657, 16), (8, 20000, 12)]   # same call twice, then a different shape
    for n_q, n_docs, k in cases:
        scores = _scores(n_q * 7 + k, n_q, n_docs)
        got_i, got_v = _noalloc(lib, scores, k)
        ref_i, ref_v = m.msa_topk_docs(scores, k)                 # the workspace-based entry point
        torch.cuda.synchronize()
        assert torch.equal(got_i, ref_i)                          # indices: exact
        assert torch.equal(got_v, ref_v)                          # scores are copied values: exact
        # and the oracle's selection over the same fp32 scores: descending, ties to the lower index
        o_i, o_v = O.topk_docs(scores.cpu().numpy().astype(np.float64), k)
        np.testing.assert_array_equal(got_i.cpu().numpy(), o_i)
        np.testing.assert_array_equal(got_v.cpu().numpy().astype(np.float64), o_v)
    assert m.device_status() == 0


def test_noalloc_topk_leaves_device_memory_unchanged():
    """After a first call (which may load the library's kernels), further calls take no device
    memory: the free memory the driver reports is the same before and after them."""
    from routed_long_context_b200 import _lib

    lib = _lib.lib
    n_q, n_docs, k = 4, 97657, 16
    scores = _scores(99, n_q, n_docs)
    idx = torch.empty((n_q, k), dtype=torch.int32, device="cuda")
    val = torch.empty((n_q, k), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call():
        st = lib.msa_topk_docs_noalloc(ctypes.c_void_p(scores.data_ptr()), n_q, n_docs, k,
                                       ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(val.data_ptr()), stream)
        assert st == 0, lib.msa_last_error()

    call()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        call()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)
    o_i, _ = O.topk_docs(scores.cpu().numpy().astype(np.float64), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), o_i)


def test_noalloc_topk_rejects_sizes_beyond_its_array():
    from routed_long_context_b200 import _lib

    lib = _lib.lib
    need = ctypes.c_size_t(0)
    assert lib.msa_topk_workspace_size(4000, 97657, 64, ctypes.byref(need)) == 0
    assert need.value > lib.msa_topk_noalloc_max_scratch()
    st = lib.msa_topk_docs_noalloc(ctypes.c_void_p(256), 4000, 97657, 64, ctypes.c_void_p(256), None, None)
    assert st == 1 and b"scratch" in lib.msa_last_error()
