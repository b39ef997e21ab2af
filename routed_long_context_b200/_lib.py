"""ctypes loader of libmsa.so with the C signatures of include/msa.h.

There is no fallback: if the library is missing or fails to load, importing the binding raises.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmsa.so")

vp, i32, i64, f32, f64, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_double,
                              ctypes.c_size_t)

MSA_OK, MSA_ERR_INVALID_ARG, MSA_ERR_UNSUPPORTED, MSA_ERR_CUDA, MSA_ERR_TIMEOUT, MSA_ERR_WORKSPACE, MSA_ERR_DEVICE = \
    range(7)
MSA_F32, MSA_BF16 = 0, 1


class LayerArgs(ctypes.Structure):
    _fields_ = [("kr_index", vp), ("host_bank", vp), ("qr", vp), ("q_new", vp), ("k_new", vp), ("v_new", vp),
                ("local_k", vp), ("local_v", vp), ("out", vp), ("topk_idx_host", vp)]


class InterleaveArgs(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("layers", ctypes.POINTER(LayerArgs)), ("dt", i32),
                ("n_chunks", i64), ("n_docs", i64), ("doc_chunk_off", vp), ("doc_chunk_off_host", vp),
                ("chunk_doc", vp), ("n_q", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
                ("hq", ctypes.c_int), ("hkv", ctypes.c_int), ("k", ctypes.c_int), ("L_prev", ctypes.c_int),
                ("T_new", ctypes.c_int), ("new_q_stride", ctypes.c_int), ("L_max", ctypes.c_int),
                ("max_mem", ctypes.c_int), ("rope_cos_sin", vp), ("rope_max_pos", i64), ("scale", f32),
                ("reserved_sms", ctypes.c_int), ("route_events", vp), ("fetch_mode", ctypes.c_int),
                ("ws", vp), ("ws_bytes", sz)]


MSA_OP_ROUTE, MSA_OP_TOPK, MSA_OP_SPARSE_ATTN_SPLIT, MSA_OP_SPARSE_ATTN_BACKWARD, MSA_OP_ROUTE_BACKWARD, \
    MSA_OP_INTERLEAVE = range(1, 7)


class RouteWsCfg(ctypes.Structure):
    _fields_ = [("n_q", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int), ("dt", i32)]


class TopkWsCfg(ctypes.Structure):
    _fields_ = [("n_q", ctypes.c_int), ("n_docs", i64), ("k", ctypes.c_int)]


class AttnWsCfg(ctypes.Structure):
    _fields_ = [("n_q", ctypes.c_int), ("T", ctypes.c_int), ("hq", ctypes.c_int), ("hkv", ctypes.c_int),
                ("max_mem", ctypes.c_int), ("L", ctypes.c_int)]


class RouteBwdWsCfg(ctypes.Structure):
    _fields_ = [("n_chunks", i64), ("n_q", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
                ("d", ctypes.c_int)]


# name -> (restype, argtypes)
SIGNATURES = {
    "msa_last_error": (ctypes.c_char_p, []),
    "msa_version": (ctypes.c_char_p, []),
    "msa_device_status": (i32, [ctypes.POINTER(i32), vp]),
    "msa_rope_table": (i32, [i64, ctypes.c_int, f64, vp]),
    "msa_chunk_doc_map": (i32, [vp, i64, i64, vp, vp]),
    "msa_rope_doc": (i32, [vp, vp, i32, i64, ctypes.c_int, ctypes.c_int, vp, i64, i64, vp, i64, vp]),
    "msa_pool_chunks": (i32, [vp, vp, vp, i32, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp, i64, i64,
                              ctypes.c_int, ctypes.c_int, vp, i64, vp, vp, i32, ctypes.c_int, vp]),
    "msa_pool_set_impl": (i32, [ctypes.c_int]),
    "msa_pool_set_pipeline": (i32, [ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "msa_route_scores": (i32, [vp, i32, i64, vp, i64, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp,
                               vp, vp, sz, vp]),
    "msa_route_workspace_size": (i32, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, i32,
                                       ctypes.POINTER(sz)]),
    "msa_route_set_impl": (i32, [ctypes.c_int]),
    "msa_route_set_max_stages": (i32, [ctypes.c_int]),
    "msa_route_inject_stall": (i32, [ctypes.c_int]),
    "msa_topk_docs": (i32, [vp, ctypes.c_int, i64, ctypes.c_int, vp, vp, vp, sz, vp]),
    "msa_topk_workspace_size": (i32, [ctypes.c_int, i64, ctypes.c_int, ctypes.POINTER(sz)]),
    "msa_topk_docs_noalloc": (i32, [vp, ctypes.c_int, i64, ctypes.c_int, vp, vp, vp]),
    "msa_topk_noalloc_max_scratch": (sz, []),
    "msa_topk_merge": (i32, [vp, vp, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, ctypes.c_int, vp, vp, vp]),
    "msa_gather_kv": (i32, [vp, i32, i64, vp, i64, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                            ctypes.c_int, vp, vp, vp]),
    "msa_gather_kv_device": (i32, [vp, i32, i64, vp, i64, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int, vp, vp, vp]),
    "msa_sparse_attn": (i32, [vp, vp, vp, ctypes.c_int, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                              ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, f32, vp, i32, vp]),
    "msa_attn_set_impl": (i32, [ctypes.c_int]),
    "msa_sparse_attn_split": (i32, [vp, vp, vp, ctypes.c_int, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, f32, vp, vp,
                                    i32, vp, sz, vp]),
    "msa_sparse_attn_split_workspace_size": (i32, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, ctypes.c_int, ctypes.POINTER(sz)]),
    "msa_pack_tokens": (i32, [vp, vp, i32, i64, ctypes.c_int, ctypes.c_int, vp, i64, vp, i64, vp, vp]),
    "msa_sparse_attn_backward": (i32, [vp, vp, vp, ctypes.c_int, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, f32, vp,
                                       vp, vp, i32, vp, vp, vp, vp, vp, sz, vp]),
    "msa_sparse_attn_backward_workspace_size": (i32, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                      ctypes.c_int, ctypes.c_int, ctypes.POINTER(sz)]),
    "msa_gather_kv_backward": (i32, [vp, i64, vp, i64, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, vp, ctypes.c_int, vp]),
    "msa_pool_chunks_backward": (i32, [vp, vp, vp, i32, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp,
                                       i64, i64, ctypes.c_int, ctypes.c_int, vp, i64, ctypes.c_int, vp, vp, vp, vp]),
    "msa_router_aux_loss": (i32, [vp, ctypes.c_int, i64, vp, ctypes.c_int, f32, vp, vp, vp]),
    "msa_route_backward": (i32, [vp, i32, i64, vp, i64, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                 vp, vp, vp, vp, sz, vp]),
    "msa_route_backward_workspace_size": (i32, [i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.POINTER(sz)]),
    "msa_interleave_step": (i32, [ctypes.POINTER(InterleaveArgs), vp, vp, i64]),
    "msa_interleave_workspace_size": (i32, [ctypes.POINTER(InterleaveArgs), ctypes.POINTER(sz)]),
    "msa_interleave_graph_create": (i32, [ctypes.POINTER(InterleaveArgs), vp, ctypes.POINTER(vp)]),
    "msa_interleave_graph_launch": (i32, [vp, vp]),
    "msa_interleave_graph_destroy": (i32, [vp]),
    "msa_workspace_size": (i32, [ctypes.c_int, vp, ctypes.POINTER(sz)]),
    "msa_sparse_attn_split_plan": (i32, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
                                         ctypes.POINTER(ctypes.c_int)]),
}


def load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmsa.so not found at {LIB_PATH}; build it with `python routed_long_context_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = load()


class MSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib.msa_last_error().decode(errors="replace")
        super().__init__(f"{where}: status {status}: {msg}")
        self.status = status


def check(status: int, where: str) -> None:
    if status != MSA_OK:
        raise MSAError(status, where)
