"""The C-ABI library loads, exports every entry point include/msa.h declares, and rejects bad
arguments on the host before touching the GPU. No test here launches a kernel."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    import importlib.util

    spec = importlib.util.spec_from_file_location("msa_build", os.path.join(ROOT, "routed_long_context_b200", "build.py"))
    builder = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(builder)
    builder.build()                      # rebuilds only when a source is newer than the library
    from routed_long_context_b200 import _lib

    return _lib.lib


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"\b(msa_\w+)\s*\(", txt))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = _declared_symbols()
    assert "msa_route_scores" in names and "msa_interleave_step" in names
    for n in names:
        assert hasattr(lib, n), n
    from routed_long_context_b200 import _lib

    assert set(_lib.SIGNATURES) <= set(names) | {"msa_last_error", "msa_version"}


def test_the_seven_hot_path_calls_are_declared():
    names = _declared_symbols()
    for n in ("msa_rope_doc", "msa_pool_chunks", "msa_route_scores", "msa_topk_docs", "msa_gather_kv",
              "msa_sparse_attn", "msa_interleave_step"):
        assert n in names


def test_rope_table_is_the_rotation_angle_table(lib):
    max_pos, d, base = 40, 8, 1.0e4
    out = np.empty((max_pos, d // 2, 2), dtype=np.float32)
    assert lib.msa_rope_table(max_pos, d, base, out.ctypes.data) == 0
    p = np.arange(max_pos)[:, None]
    w = base ** (-2.0 * np.arange(d // 2) / d)
    np.testing.assert_array_equal(out[..., 0], np.cos(p * w).astype(np.float32))
    np.testing.assert_array_equal(out[..., 1], np.sin(p * w).astype(np.float32))
    assert lib.msa_rope_table(4, 7, base, out.ctypes.data) == 1          # odd d
    assert lib.msa_rope_table(4, 8, base, None) == 1


def test_topk_rejects_k_larger_than_docs_without_launching(lib):
    ws = ctypes.c_size_t(0)
    assert lib.msa_topk_workspace_size(1, 10, 4, ctypes.byref(ws)) == 0 and ws.value > 0
    st = lib.msa_topk_docs(ctypes.c_void_p(16), 1, 10, 11, ctypes.c_void_p(16), None, ctypes.c_void_p(16), 1 << 20,
                           None)
    assert st == 1
    assert b"k" in lib.msa_last_error()
    assert lib.msa_topk_workspace_size(1, 10, 65, ctypes.byref(ws)) == 1


def test_gather_validates_indices_and_capacity_on_host(lib):
    C, hkv, d = 10, 1, 8
    bank = np.zeros((C, 2, hkv, d), dtype=np.float32)
    off = np.array([0, 3, 5, 10], dtype=np.int64)
    mem_len = np.zeros(1, dtype=np.int32)
    bad_idx = np.array([[0, 7]], dtype=np.int32)        # doc 7 does not exist
    st = lib.msa_gather_kv(bank.ctypes.data, 0, C, off.ctypes.data, 3, bad_idx.ctypes.data, 1, 2, hkv, d, 16,
                           ctypes.c_void_p(256), mem_len.ctypes.data, None)
    assert st == 1 and b"out of range" in lib.msa_last_error()
    idx = np.array([[2, 0]], dtype=np.int32)            # 5 + 3 rows > max_mem 6
    st = lib.msa_gather_kv(bank.ctypes.data, 0, C, off.ctypes.data, 3, idx.ctypes.data, 1, 2, hkv, d, 6,
                           ctypes.c_void_p(256), mem_len.ctypes.data, None)
    assert st == 1 and b"max_mem" in lib.msa_last_error()


def test_route_and_attention_reject_bad_shapes(lib):
    ws = ctypes.c_size_t(0)
    assert lib.msa_route_workspace_size(2, 16, 8, 128, 1, ctypes.byref(ws)) == 0
    assert lib.msa_route_workspace_size(0, 16, 8, 128, 1, ctypes.byref(ws)) == 1
    # head_dim 64 is not supported by the attention kernel
    st = lib.msa_sparse_attn(ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.c_void_p(256), 4,
                             ctypes.c_void_p(256), ctypes.c_void_p(256), 8, 8, 0, 1, 4, 8, 2, 64, 0.125,
                             ctypes.c_void_p(256), 0, None)
    assert st == 2
    # misaligned query pointer
    st = lib.msa_sparse_attn(ctypes.c_void_p(258), ctypes.c_void_p(256), ctypes.c_void_p(256), 4,
                             ctypes.c_void_p(256), ctypes.c_void_p(256), 8, 8, 0, 1, 4, 8, 2, 128, 0.125,
                             ctypes.c_void_p(256), 0, None)
    assert st == 1
    # causal window larger than the cache
    st = lib.msa_sparse_attn(ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.c_void_p(256), 4,
                             ctypes.c_void_p(256), ctypes.c_void_p(256), 8, 9, 0, 1, 4, 8, 2, 128, 0.125,
                             ctypes.c_void_p(256), 0, None)
    assert st == 1
    assert lib.msa_route_set_impl(4) == 1 and lib.msa_route_set_impl(0) == 0
    assert lib.msa_pool_set_impl(4) == 1 and lib.msa_pool_set_impl(-1) == 1 and lib.msa_pool_set_impl(0) == 0
    assert lib.msa_attn_set_impl(4) == 1 and lib.msa_attn_set_impl(3) == 0 and lib.msa_attn_set_impl(0) == 0
    assert lib.msa_pool_set_pipeline(1, 0, 0) == 1         # fewer than 2 stages
    assert lib.msa_pool_set_pipeline(0, 1000, 0) == 1      # not a multiple of 1024
    assert lib.msa_pool_set_pipeline(16, 65536, 0) == 1    # ring above 200 KiB
    assert lib.msa_pool_set_pipeline(0, 0, 24) == 1        # copy size not a multiple of 16
    assert lib.msa_pool_set_pipeline(0, 0, 0) == 0


def test_interleave_rejects_local_cache_overflow(lib):
    from routed_long_context_b200 import _lib

    layers = (_lib.LayerArgs * 1)()
    for f, _ in _lib.LayerArgs._fields_:
        setattr(layers[0], f, 256)
    a = _lib.InterleaveArgs()
    a.n_layers, a.layers, a.dt = 1, layers, 1
    a.n_chunks, a.n_docs = 10, 2
    a.doc_chunk_off = a.doc_chunk_off_host = a.chunk_doc = a.rope_cos_sin = 256
    a.n_q, a.H, a.d, a.hq, a.hkv, a.k = 1, 8, 128, 32, 8, 1
    a.L_prev, a.T_new, a.new_q_stride, a.L_max, a.max_mem = 60, 8, 8, 64, 16
    a.rope_max_pos, a.scale, a.ws, a.ws_bytes = 4096, 0.1, 256, 1 << 30
    n = ctypes.c_size_t(0)
    assert lib.msa_interleave_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 1
    assert b"overflow" in lib.msa_last_error()
    a.L_prev = 56
    assert lib.msa_interleave_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0 and n.value > 0


def test_new_entry_points_validate_on_the_host(lib):
    """Fine stage, Memory Parallel merge and backward calls reject bad arguments before any launch."""
    P = ctypes.c_void_p(256)
    # token bank: odd head_dim
    assert lib.msa_pack_tokens(P, P, 1, 10, 8, 127, P, 2, P, 64, P, None) != 0
    # merge: too many shards, k out of range, shard offsets decreasing
    off = np.array([0, 5, 3], dtype=np.int64)
    assert lib.msa_topk_merge(P, P, 16, 65, 1, 4, off.ctypes.data, 4, P, P, None) == 1
    good = np.array([0, 5, 9], dtype=np.int64)
    assert lib.msa_topk_merge(P, P, 16, 2, 1, 4, good.ctypes.data, 65, P, P, None) == 1
    assert lib.msa_topk_merge(P, P, 16, 2, 1, 4, off.ctypes.data, 4, P, P, None) == 1
    assert b"decrease" in lib.msa_last_error()
    # split attention and the backward are bf16 only
    assert lib.msa_sparse_attn_split(P, P, P, 8, P, P, 8, 8, 0, 1, 4, 32, 8, 128, 0.1, P, None, 0, P, 1 << 20,
                                     None) == 2
    assert lib.msa_sparse_attn_backward(P, P, P, 8, P, P, 8, 8, 0, 1, 4, 32, 8, 128, 0.1, P, P, P, 0, P, P, P, P,
                                        P, 1 << 20, None) == 2
    # aux loss: tau must be positive; pooling backward: nothing to do
    assert lib.msa_router_aux_loss(P, 1, 10, P, 2, 0.0, None, P, None) == 1
    assert lib.msa_pool_chunks_backward(None, None, None, 0, 10, 8, 8, 128, P, P, P, 2, 4, 4, 1, P, 64, 1, P, P, P,
                                        None) == 1
    # workspace sizes are queries only
    n = ctypes.c_size_t(0)
    assert lib.msa_sparse_attn_split_workspace_size(1, 64, 32, 8, 8064, 64, ctypes.byref(n)) == 0 and n.value > 0
    assert lib.msa_sparse_attn_backward_workspace_size(1, 512, 32, 8, 128, 512, ctypes.byref(n)) == 0
    assert lib.msa_route_backward_workspace_size(512, 1, 512, 8, 128, ctypes.byref(n)) == 0 and n.value > 0


def test_binding_refuses_views_the_c_abi_would_misread(lib):
    """The C ABI reads dense row-major arrays: a transposed or sliced view is refused before any
    call, and the Memory Parallel merge accepts strided candidate lists only when their layout
    matches the shard stride it is given."""
    import torch

    from routed_long_context_b200 import api

    with pytest.raises(ValueError):
        api._ptr(torch.zeros(4, 6).t())
    with pytest.raises(ValueError):
        api._ptr(torch.zeros(4, 6)[:, 1:3])
    assert api._ptr(torch.zeros(4, 6)[1:3]) is not None           # a leading-dimension slice is dense
    packed = torch.zeros(3, 2, 2, 5, dtype=torch.int32)          # [shards][score, index][n_q][k_cand]
    bounds = np.array([0, 10, 20, 30])
    with pytest.raises(ValueError):                               # the pair is interleaved: stride needed
        api.msa_topk_merge(packed[:, 0].view(torch.float32), packed[:, 1], bounds, 4)
    with pytest.raises(ValueError):                               # inner lists not dense
        api.msa_topk_merge(torch.zeros(3, 5, 2)[:, :, 0], torch.zeros(3, 5, 2, dtype=torch.int32)[:, :, 0],
                           bounds, 4, shard_stride=10)


def test_too_small_workspace_is_refused_before_any_launch(lib):
    """A caller workspace below the size the library asks for (the stand-in for an allocation that
    failed) is refused with MSA_ERR_WORKSPACE and a message naming both sizes; nothing is launched
    (the calls get placeholder pointers that no kernel could read)."""
    from routed_long_context_b200 import _lib

    P = ctypes.c_void_p(256)
    f = ctypes.c_float(0.1)
    calls = {
        "msa_route_scores": lambda: lib.msa_route_scores(P, 1, 1000, P, 100, P, 1, 64, 8, 128, P, None, P, 16, None),
        "msa_topk_docs": lambda: lib.msa_topk_docs(P, 1, 1000, 4, P, P, P, 0, None),
        "msa_route_backward": lambda: lib.msa_route_backward(P, 1, 1000, P, 100, P, 1, 17, 8, 128, P, P, P, P, 16,
                                                             None),
        "msa_sparse_attn_split": lambda: lib.msa_sparse_attn_split(P, P, P, 64, P, P, 16, 16, 0, 1, 16, 32, 8, 128, f,
                                                                   P, None, 1, P, 16, None),
        "msa_sparse_attn_backward": lambda: lib.msa_sparse_attn_backward(P, P, P, 64, P, P, 16, 16, 0, 1, 16, 32, 8,
                                                                         128, f, P, P, P, 1, P, P, P, P, P, 16, None),
    }
    for name, call in calls.items():
        assert call() == _lib.MSA_ERR_WORKSPACE, name
        msg = lib.msa_last_error().decode()
        assert msg.startswith(name) and "workspace" in msg and re.search(r"\d+ < \d+", msg), msg

    layers = (_lib.LayerArgs * 1)()
    for fld, _ in _lib.LayerArgs._fields_:
        setattr(layers[0], fld, 256)
    a = _lib.InterleaveArgs()
    a.n_layers, a.layers, a.dt = 1, layers, 1
    a.n_chunks, a.n_docs = 10, 2
    a.doc_chunk_off = a.doc_chunk_off_host = a.chunk_doc = a.rope_cos_sin = 256
    a.n_q, a.H, a.d, a.hq, a.hkv, a.k = 1, 8, 128, 32, 8, 1
    a.L_prev, a.T_new, a.new_q_stride, a.L_max, a.max_mem = 56, 8, 8, 64, 16
    a.rope_max_pos, a.scale, a.ws, a.ws_bytes = 4096, 0.1, 256, 16
    assert lib.msa_interleave_step(ctypes.byref(a), None, None, 1000) == _lib.MSA_ERR_WORKSPACE
    msg = lib.msa_last_error().decode()
    n = ctypes.c_size_t(0)
    assert lib.msa_interleave_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert f"16 < {n.value}" in msg, msg


def test_generic_workspace_query_matches_every_per_call_query(lib):
    """msa_workspace_size(op, cfg) answers what each call's own *_workspace_size answers, and refuses
    unknown ops and NULL arguments."""
    from routed_long_context_b200 import _lib as L

    def ws(op, cfg):
        n = ctypes.c_size_t(0)
        st = lib.msa_workspace_size(op, ctypes.cast(ctypes.byref(cfg), ctypes.c_void_p), ctypes.byref(n))
        return st, n.value

    def own(fn, *args):
        n = ctypes.c_size_t(0)
        st = fn(*args, ctypes.byref(n))
        return st, n.value

    assert ws(L.MSA_OP_ROUTE, L.RouteWsCfg(3, 64, 8, 128, 1)) == own(lib.msa_route_workspace_size, 3, 64, 8, 128, 1)
    assert ws(L.MSA_OP_TOPK, L.TopkWsCfg(32, 97657, 16)) == own(lib.msa_topk_workspace_size, 32, 97657, 16)
    assert ws(L.MSA_OP_SPARSE_ATTN_SPLIT, L.AttnWsCfg(1, 64, 32, 8, 8064, 64)) == \
        own(lib.msa_sparse_attn_split_workspace_size, 1, 64, 32, 8, 8064, 64)
    assert ws(L.MSA_OP_SPARSE_ATTN_BACKWARD, L.AttnWsCfg(1, 512, 32, 8, 128, 512)) == \
        own(lib.msa_sparse_attn_backward_workspace_size, 1, 512, 32, 8, 128, 512)
    assert ws(L.MSA_OP_ROUTE_BACKWARD, L.RouteBwdWsCfg(512, 1, 512, 8, 128)) == \
        own(lib.msa_route_backward_workspace_size, 512, 1, 512, 8, 128)
    for op, cfg in ((L.MSA_OP_ROUTE, L.RouteWsCfg(3, 64, 8, 128, 1)), (L.MSA_OP_TOPK, L.TopkWsCfg(32, 97657, 16))):
        assert ws(op, cfg)[0] == 0 and ws(op, cfg)[1] > 0
    # a size the call itself refuses is refused the same way
    assert ws(L.MSA_OP_TOPK, L.TopkWsCfg(1, 10, 65))[0] == own(lib.msa_topk_workspace_size, 1, 10, 65)[0] == 1
    assert ws(L.MSA_OP_ROUTE, L.RouteWsCfg(0, 16, 8, 128, 1))[0] == 1
    # unknown op, NULL cfg, NULL bytes
    assert ws(99, L.TopkWsCfg(1, 10, 4))[0] == 1 and b"unknown op" in lib.msa_last_error()
    n = ctypes.c_size_t(0)
    assert lib.msa_workspace_size(L.MSA_OP_TOPK, None, ctypes.byref(n)) == 1
    cfg = L.TopkWsCfg(1, 10, 4)
    assert lib.msa_workspace_size(L.MSA_OP_TOPK, ctypes.cast(ctypes.byref(cfg), ctypes.c_void_p), None) == 1


def test_interleave_graph_validates_before_any_capture(lib):
    """The captured round takes fetch_mode 1 only, no timing events and a created stream; each
    refusal happens before any CUDA call. Destroying NULL is a no-op; launching NULL is refused."""
    from routed_long_context_b200 import _lib

    layers = (_lib.LayerArgs * 1)()
    a = _lib.InterleaveArgs()
    a.n_layers, a.layers = 1, layers
    g = ctypes.c_void_p(None)
    a.fetch_mode = 0
    assert lib.msa_interleave_graph_create(ctypes.byref(a), ctypes.c_void_p(256), ctypes.byref(g)) == 1
    assert b"fetch_mode" in lib.msa_last_error() and not g.value
    a.fetch_mode = 1
    ev = (ctypes.c_void_p * 2)(256, 256)
    a.route_events = ctypes.cast(ev, ctypes.c_void_p)
    assert lib.msa_interleave_graph_create(ctypes.byref(a), ctypes.c_void_p(256), ctypes.byref(g)) == 1
    assert b"route_events" in lib.msa_last_error()
    a.route_events = None
    assert lib.msa_interleave_graph_create(ctypes.byref(a), None, ctypes.byref(g)) == 1
    assert b"stream" in lib.msa_last_error()
    assert lib.msa_interleave_graph_create(None, ctypes.c_void_p(256), ctypes.byref(g)) == 1
    assert lib.msa_interleave_graph_destroy(None) == 0
    assert lib.msa_interleave_graph_launch(None, None) == 1
