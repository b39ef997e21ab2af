#!/usr/bin/env python
"""Benchmark of the MSA hot path on B200: one step = one Memory Interleave round over the 18 routed
layers of the 100M-token configuration (781,250 pre-pooled chunks of 128 tokens per layer, bf16
router index resident in HBM, pooled K/V in pinned host memory; 64 query tokens, top-16):
per layer append + global RoPE, router scoring, top-k, host-bank fetch and sparse attention.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--layers 18]

Prints one JSON line on rank 0. With N > 1 (torchrun) every rank runs an independent replica
(the path has no exchange step on one GPU's workload): value = all ranks' tokens / max time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "memory tokens routed/s per layer at 100M (frac of HBM peak); route+attn ms/step"
UNIT = "memory tokens/s"
TOKENS_PER_CHUNK = 128
# DRAM bytes (read + write) of one full-size router launch: ncu --set full on a 99,994-chunk case of
# the current kernel (205.53 MB read + 3.54 MB written), scaled by the chunk count to 781,250 chunks.
ROUTER_TRAFFIC_BYTES = (205.53e6 + 3.54e6) * 781250 / 99994


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=18)
    ap.add_argument("--host-banks", type=int, default=2)
    ap.add_argument("--n-docs", type=int, default=97657, help="shorter bank for small profiling cases only")
    ap.add_argument("--fetch-mode", type=int, default=1, choices=[0, 1],
                    help="0: host-issued cudaMemcpyAsync per selected document; 1: device-side fetch kernel")
    ap.add_argument("--router-stages", type=int, default=0,
                    help="cap on the router's pipeline stages (0 = default shared-memory budget)")
    ap.add_argument("--reserved-sms", type=int, default=0,
                    help="SMs the routers leave free for the overlapped selection and attention")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU time of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="headline line only (no per-configuration entries)")
    ap.add_argument("--workload", default="100m",
                    choices=["100m", "tiny", "1m", "encode10m", "decode10m", "interleave", "fine1m", "train64k"],
                    help="100m: the routing step (the reported metric), with every other configuration under "
                         "'configs' in the same line; the others print one configuration as a line of its own: "
                         "tiny and 1m (one-layer step latency), encode10m (offline encoding of the 10M-token bank: "
                         "document-wise RoPE + chunk-mean pooling), decode10m (32 decode queries over it), "
                         "interleave (three Memory Interleave rounds over a 10M-token bank, tensor-bound routing), "
                         "fine1m (the token-level fine stage on the 1M-token bank), train64k (a training step, "
                         "forward + backward, on a 64K-token context)")
    return ap.parse_args()


def max_over_ranks(vals, device):
    """Elementwise max of per-rank timings over all ranks (every rank takes the same collective)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(vals, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Units all ranks processed (independent replicas) per second of the slowest rank."""
    return units_per_rank * world / (ms / 1e3)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ---------------------------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons of this GPU through NVML (read-only) while running."""

    HW_SLOW, HW_THERM, SW_THERM, SW_POWER = 0x8, 0x40, 0x20, 0x4

    def __init__(self, device_index: int):
        self.samples, self.max_mhz, self.ok = [], None, False
        self._stop = threading.Event()
        try:
            import pynvml as nv
            import torch

            nv.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.h = nv.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            self.nv = nv
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((sm, rs))
            except Exception:
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = {self.HW_SLOW: "hw_slowdown", self.HW_THERM: "hw_thermal_slowdown",
                 self.SW_THERM: "sw_thermal_slowdown", self.SW_POWER: "sw_power_cap"}
        seen = sorted({n for _, r in self.samples for bit, n in names.items() if r & bit})
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": seen, "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------------- oracle
def oracle_sample(seconds: float, layer: int = 0):
    """The fp64 oracle's routing + top-k on leading slices of one 100M layer until `seconds` of CPU
    time have passed (bounded sample); returns (memory tokens / s, chunks, threads)."""
    import numpy as np
    from threadpoolctl import threadpool_info

    import oracle as O
    from msa_inputs import workloads

    w = workloads.mem_100m(layers=1)
    qr = w.qr(layer)[:, :w.T0]
    docs_per_slice = 4096
    t0 = time.perf_counter()
    done_docs = 0
    while done_docs < w.n_docs and time.perf_counter() - t0 < seconds:
        d1 = min(w.n_docs, done_docs + docs_per_slice)
        a, b = int(w.doc_chunk_off[done_docs]), int(w.doc_chunk_off[d1])
        rows = w.host_rows(layer, "krbar", np.arange(a, b)).reshape(b - a, w.H, w.d)
        ds, _ = O.route(rows, w.doc_chunk_off[done_docs:d1 + 1] - a, qr)
        O.topk_docs(ds, w.k)
        done_docs = d1
    dt = time.perf_counter() - t0
    chunks = int(w.doc_chunk_off[done_docs])
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return chunks * TOKENS_PER_CHUNK / dt, chunks, threads


def reference_arm(args, rank):
    """The oracle as the reference arm: every step is a bounded sample of the 100M routing workload
    (routing + top-k over leading slices of one layer), timed on the host; ms_per_step is that
    sample's measured time, and the projection to a whole 18-layer step is reported beside it."""
    if rank != 0:
        return
    secs = max(1.0, args.cpu_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(secs)
    vals, step_ms, chunks, thr = [], [], 0, 1
    for _ in range(args.steps):
        t0 = time.perf_counter()
        v, c, thr = oracle_sample(secs)
        step_ms.append((time.perf_counter() - t0) * 1e3)
        vals.append(v)
        chunks = c
    value = statistics.median(vals)
    projected = 781250 * TOKENS_PER_CHUNK / value * 1e3 * args.layers
    sample = f"oracle routing + top-k of the first {chunks} chunks of one 100M layer per step (fp64, numpy)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.median(step_ms),
        "ms_per_step_what": "the timed sample of each step (a bounded slice of one layer), wall clock on the host",
        "projected_full_step_ms": projected,
        "projected_full_step_what": f"{args.layers} layers x 781,250 chunks at the sample's rate (projection)",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "100m-routing (781,250 chunks x 18 layers, 64 query tokens, top-16)",
                   "sample": sample},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


# ---------------------------------------------------------------------------------------------- configurations
# Every configuration of the measured workload set, each reported with its own roofline, the fp64
# oracle timed on the host cores on a bounded sample, and an end-to-end figure through the public API
# with host buffers. The default run puts them under "configs" in the one JSON line; `--workload X`
# prints one of them as a line of its own.
def all_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm": float(p["hbm_gbs"]), "bf16": float(p["bf16_tflops"]),
                "bf16_sustained": float(p["bf16_tflops_sustained"]), "kind": "measured"}
    except Exception:
        return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "kind": "fallback"}


def _ev():
    import torch

    return torch.cuda.Event(enable_timing=True)


def device_ms(fn, steps: int, warmup: int, stream) -> float:
    """Mean ms per call of fn (which launches on `stream`), CUDA events around `steps` calls."""
    import torch

    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = _ev(), _ev()
    a.record(stream)
    for _ in range(steps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def cpu_seconds(fn, min_s: float, max_reps: int) -> float:
    """Seconds per call of fn on the host: repeated until min_s have passed or max_reps calls."""
    t0 = time.perf_counter()
    n = 0
    while True:
        fn()
        n += 1
        dt = time.perf_counter() - t0
        if dt >= min_s or n >= max_reps:
            return dt / n


def oracle_threads() -> int:
    from threadpoolctl import threadpool_info

    return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])


def _free():
    import torch

    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _pinned_like(t):
    import torch

    h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
    h.copy_(t)
    return h


class OneLayerRound:
    """One routed layer of a token-level configuration as one interleave round through the public
    API (append + global RoPE, routing, top-k, fetch from the pinned host bank, attention), plus the
    pinned host copies of its query-side inputs and output for the end-to-end figure."""

    def __init__(self, m, w, lay, index, bank, cs, fetch_mode=1):
        import torch

        from msa_inputs.device import TORCH_DT, small_tensors

        dt = TORCH_DT[w.dtype]
        self.w, self.m = w, m
        self.dv = small_tensors(w, 0)
        self.local = (torch.zeros((w.n_q, w.T_total, w.hkv, w.d), dtype=dt, device="cuda"),
                      torch.zeros((w.n_q, w.T_total, w.hkv, w.d), dtype=dt, device="cuda"))
        self.out = torch.empty((w.n_q, w.T0, w.hq, w.d), dtype=dt, device="cuda")
        self.idx_host = torch.empty((w.n_q, w.k), dtype=torch.int32, pin_memory=True)
        la = [dict(kr_index=index, host_bank=bank, qr=self.dv["qr"], q_new=self.dv["q"], k_new=self.dv["k_new"],
                   v_new=self.dv["v_new"], local_k=self.local[0], local_v=self.local[1], out=self.out,
                   topk_idx_host=self.idx_host)]
        self.rd = m.InterleaveRound(la, n_chunks=lay.n_chunks, n_docs=lay.n_docs, doc_chunk_off=lay.doc_chunk_off,
                                    doc_chunk_off_host=lay.doc_chunk_off_host, chunk_doc=lay.chunk_doc, n_q=w.n_q,
                                    H=w.H, d=w.d, hq=w.hq, hkv=w.hkv, k=w.k, L_prev=0, T_new=w.T0,
                                    new_q_stride=w.T_total, L_max=w.T_total, max_mem=w.max_mem, cos_sin=cs,
                                    dtype=dt, fetch_mode=fetch_mode)
        self.names = ("qr", "q", "k_new", "v_new")
        self.h_in = [_pinned_like(self.dv[n]) for n in self.names]
        self.h_out = torch.empty(self.out.shape, dtype=dt, pin_memory=True)
        self.compute, self.copy = torch.cuda.Stream(), torch.cuda.Stream()

    def step(self, route_events=None):
        self.rd.run(self.compute, self.copy, route_events=route_events)

    def device(self, steps, warmup):
        """(ms per step, router ms per launch) on the compute stream."""
        import torch

        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize()
        evs = [[_ev(), _ev()] for _ in range(steps)]
        for e in evs:
            e[0].record(self.compute)
            e[1].record(self.compute)
        torch.cuda.synchronize()
        a, b = _ev(), _ev()
        a.record(self.compute)
        for i in range(steps):
            self.step(route_events=evs[i])
        b.record(self.compute)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps, sum(e[0].elapsed_time(e[1]) for e in evs) / steps

    def graph_device(self, steps, warmup):
        """ms per step of the round captured once into a CUDA graph (msa_interleave_graph_*) and
        replayed on the compute stream; None with host-issued copies (fetch_mode 0), which wait on
        the host and cannot be captured."""
        if self.rd.args.fetch_mode != 1:
            return None
        self.graph = self.rd.capture(self.compute)
        return device_ms(lambda: self.graph.launch(self.compute), steps, warmup, self.compute)

    def e2e(self, steps, warmup):
        """ms per step with the step's query-side inputs copied host -> device before it and its output
        read back after it, serialised on the compute stream (latency, no overlap between steps); the
        round itself is the graph replay when one was captured."""
        import torch

        graph = getattr(self, "graph", None)

        def one():
            with torch.cuda.stream(self.compute):
                for h, n in zip(self.h_in, self.names):
                    self.dv[n].copy_(h, non_blocking=True)
            if graph is not None:
                graph.launch(self.compute)
            else:
                self.step()
            with torch.cuda.stream(self.compute):
                self.h_out.copy_(self.out, non_blocking=True)

        ms = device_ms(one, steps, warmup, self.compute)
        h2d = sum(h.numel() * h.element_size() for h in self.h_in)
        d2h = self.h_out.numel() * self.h_out.element_size() + self.idx_host.numel() * 4
        return ms, h2d, d2h


def _oracle_pool_router(w, docs, group=64):
    """fp64 oracle K-bar^R of the given documents' chunks (host-regenerated tokens), in doc order."""
    import concurrent.futures as cf

    import numpy as np

    import oracle as O

    def one(g):
        d0, d1 = g
        a, b = int(w.doc_tok_off[d0]), int(w.doc_tok_off[d1])
        x = w.host_rows(0, "kr", np.arange(a, b)).reshape(b - a, w.H, w.d)
        return O.encode_memory(None, None, x, w.doc_tok_off[d0:d1 + 1] - a, w.chunk, w.rope_base)[2]

    groups = [(d0, min(docs, d0 + group)) for d0 in range(0, docs, group)]
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        return np.concatenate(list(ex.map(one, groups)))


def _oracle_kv_of_docs(w, docs):
    """{doc: (K-bar, V-bar)} by the fp64 oracle (document-wise RoPE + pooling) from host tokens."""
    import numpy as np

    import oracle as O

    out = {}
    for doc in docs:
        a, b = int(w.doc_tok_off[doc]), int(w.doc_tok_off[doc + 1])
        t = {n: w.host_rows(0, n, np.arange(a, b)).reshape(b - a, w.hkv, w.d) for n in ("k", "v")}
        kb, vb, _ = O.encode_memory(t["k"], t["v"], None, np.array([0, b - a]), w.chunk, w.rope_base)
        out[int(doc)] = (kb, vb)
    return out


def _oracle_step_fn(w, krb, kv_of, n_chunks_scale=1.0):
    """The oracle's one-layer step (route -> top-k -> gather -> global RoPE -> attention) for every
    query of w over pooled router keys krb (a leading slice of the bank when n_chunks_scale > 1)."""
    import numpy as np

    import oracle as O

    qr, qa, kn, vn = w.qr(0)[:, :w.T0], w.q(0), w.k_new(0), w.v_new(0)
    off = w.doc_chunk_off[:np.searchsorted(w.doc_chunk_off, krb.shape[0]) + 1]
    pos = O.global_positions(w.k, 0, w.T0)

    def step():
        ds, _ = O.route(krb, off, qr)
        idx, _ = O.topk_docs(ds, w.k)
        for q in range(w.n_q):
            docs = [d for d in idx[q] if int(d) in kv_of] or list(kv_of)[:w.k]
            kb = np.concatenate([kv_of[int(d)][0] for d in docs])
            vb = np.concatenate([kv_of[int(d)][1] for d in docs])
            O.sparse_attention(O.apply_rope(qa[q, :w.T0], pos, w.rope_base), kb, vb,
                               O.apply_rope(kn[q, :w.T0], pos, w.rope_base), vn[q, :w.T0], 0, 1 / np.sqrt(w.d))
    return step


def _round_entry(name, metric, w, lay, rb, steps, warmup, pk, route_kind, notes, cpu):
    """Entry of a one-layer round configuration: device step latency, router roofline, e2e, oracle."""
    eager_ms, route_ms = rb.device(steps, warmup)
    graph_ms = rb.graph_device(steps, warmup)
    ms = graph_ms if graph_ms is not None else eager_ms
    e_ms, h2d, d2h = rb.e2e(steps, warmup)
    elem = 4 if w.dtype == "f32" else 2
    route_bytes = lay.n_chunks * w.H * w.d * elem
    route_flops = 2.0 * w.H * w.d * lay.n_chunks * w.n_q * w.T0
    if route_kind == "tensor":
        ach = route_flops / (route_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": pk["bf16"], "unit": "TFLOP/s", "frac": ach / pk["bf16"],
                "traffic": None, "kernel": "route_tc_kernel", "peak_kind": f"{pk['kind']} bf16 burst (cuBLAS)"}
    else:
        ach = route_bytes / (route_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": pk["hbm"], "unit": "GB/s", "frac": ach / pk["hbm"],
                "traffic": None, "kernel": "route_simt_kernel" if w.dtype == "f32" else "route_tc_kernel",
                "peak_kind": f"{pk['kind']} copy bandwidth"}
    roof["note"] = notes
    sel = rb.idx_host.numpy()
    planted_ok = all(set(w.expected(0, 0, q)) <= set(sel[q].tolist()) for q in range(w.n_q))
    launch = ("one CUDA graph replay of the captured round (msa_interleave_graph_launch)" if graph_ms is not None
              else "msa_interleave_step (host-issued copies: not capturable)")
    return {"workload": name, "metric": metric, "value": ms * 1e3, "unit": "us per step", "higher_is_better": False,
            "ms_per_step": ms, "steps": steps, "launch": launch, "eager_us_per_step": eager_ms * 1e3,
            "route_us_per_launch": route_ms * 1e3, "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": e_ms * 1e3, "unit": "us per step", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "how": "public API (msa_interleave_graph_launch, or msa_interleave_step without a graph) with "
                           "pinned host buffers: the step's query-side inputs copied in and its output read back "
                           "inside the timed region, serialised (latency)"},
            "checks": {"planted_docs_selected": planted_ok, "device_status": rb.m.device_status()}}


def cfg_tiny(args, pk):
    import numpy as np

    import oracle as O
    import routed_long_context_b200 as m
    from msa_inputs import workloads
    from msa_inputs.device import memory_tensor
    from routed_long_context_b200.bank import BankLayout, encode_tokens, to_host_bank

    w = workloads.tiny()
    lay = BankLayout.from_doc_lengths(w.doc_len, w.chunk)
    cs = m.rope_table(4096, w.d, w.rope_base)
    k, v, kr = (memory_tensor(w, 0, n) for n in ("k", "v", "kr"))
    kvbar, index = encode_tokens(lay, k, v, kr, w.chunk, cs)
    del k, v, kr
    rb = OneLayerRound(m, w, lay, index, to_host_bank(kvbar), cs, args.fetch_mode)
    # the oracle's step on the full bank (pooling is the offline stage, outside the step)
    kh, vh, krh = (w.host_tensor(0, n) for n in ("k", "v", "kr"))
    kb, vb, krb = O.encode_memory(kh, vh, krh, w.doc_tok_off, w.chunk, w.rope_base)
    kv_of = {d: (kb[w.doc_chunk_off[d]:w.doc_chunk_off[d + 1]], vb[w.doc_chunk_off[d]:w.doc_chunk_off[d + 1]])
             for d in range(w.n_docs)}
    cpu_s = cpu_seconds(_oracle_step_fn(w, krb, kv_of), 2.0, 200)
    cpu = {"value": cpu_s * 1e6, "unit": "us per step", "cores": oracle_threads(), "kind": "oracle",
           "sample": "the whole step (route over all 512 chunks, top-4, gather, attention), fp64"}
    e = _round_entry("tiny: 64 docs x 1024 tokens (65,536), chunk 128, fp32; 1 query x 16 tokens, top-4, GQA 32/8, "
                     "16 causal local tokens", "tiny: route + top-4 + fetch + attention, one layer", w, lay, rb,
                     min(args.steps, 200), args.warmup, pk, "hbm",
                     "latency-bound: a 2 MB fp32 index (L2-resident) and tens of microseconds of launches", cpu)
    del rb, kvbar, index
    _free()
    return e


def cfg_1m(args, pk):
    import numpy as np

    import oracle as O
    import routed_long_context_b200 as m
    from msa_inputs import workloads
    from msa_inputs.device import memory_tensor
    from routed_long_context_b200.bank import BankLayout, encode_tokens, to_host_bank

    w = workloads.mem_1m()
    lay = BankLayout.from_doc_lengths(w.doc_len, w.chunk)
    cs = m.rope_table(4096, w.d, w.rope_base)
    k, v, kr = (memory_tensor(w, 0, n) for n in ("k", "v", "kr"))
    kvbar, index = encode_tokens(lay, k, v, kr, w.chunk, cs)
    del k, v, kr
    _free()
    rb = OneLayerRound(m, w, lay, index, to_host_bank(kvbar), cs, args.fetch_mode)
    # oracle: the pooled router index of the whole bank (untimed offline stage), K-bar/V-bar of the
    # documents its own routing selects; the timed step routes over every chunk
    krb = _oracle_pool_router(w, w.n_docs)
    ds, _ = O.route(krb, w.doc_chunk_off, w.qr(0)[:, :w.T0])
    sel, _ = O.topk_docs(ds, w.k)
    cpu_s = cpu_seconds(_oracle_step_fn(w, krb, _oracle_kv_of_docs(w, sel[0])), 2.0, 20)
    cpu = {"value": cpu_s * 1e6, "unit": "us per step", "cores": oracle_threads(), "kind": "oracle",
           "sample": f"the whole step (route over all {lay.n_chunks:,} chunks, top-8, gather, attention), fp64"}
    e = _round_entry(f"1m: {w.n_docs} docs ({w.n_tok:,} tokens, 128..1792), chunk 128, bf16; 1 query x 64 tokens, "
                     "top-8, GQA 32/8", "1M: route + top-8 + fetch + attention, one layer", w, lay, rb,
                     min(args.steps, 200), args.warmup, pk, "tensor",
                     "16 MB index, L2-resident: the router runs at tensor and launch speed, not HBM", cpu)
    del rb, kvbar, index
    _free()
    return e


# DRAM bytes (read + write) of pool_kernel per launch on the 10M encode: ncu --set full on a
# 400-document case of the current kernel (2,517.15 MB read + 7.77 MB written), scaled by documents
# to the 9,766-document bank (traffic grows with the tokens pooled).
POOL_TRAFFIC_10M = (2517.153e6 + 7.774e6) * 9766 / 400


def cfg_10m(args, pk):
    """Two entries: the offline encode (61.4 GB through document-wise RoPE + pooling) and the decode
    step (32 queries x 1 token routed over 39,064 chunks, top-16, per-query fetch of 8.4 MB from the
    pinned host bank, attention)."""
    import numpy as np

    import oracle as O
    import routed_long_context_b200 as m
    from msa_inputs import workloads
    from msa_inputs.device import memory_tensor
    from routed_long_context_b200.bank import BankLayout, to_host_bank

    import torch

    w = workloads.mem_10m(n_docs=9766 if args.n_docs == 97657 else args.n_docs)    # fewer: a small capture case
    lay = BankLayout.from_doc_lengths(w.doc_len, w.chunk)
    cs = m.rope_table(4096, w.d, w.rope_base)
    k, v, kr = (memory_tensor(w, 0, n) for n in ("k", "v", "kr"))
    kvbar = torch.empty((lay.n_chunks, 2, w.hkv, w.d), dtype=torch.bfloat16, device="cuda")
    index = torch.empty((lay.n_chunks, w.H, w.d), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.current_stream()

    def encode():
        m.msa_pool_chunks(k, v, kr, lay.doc_tok_off, lay.doc_chunk_off, lay.chunk_doc, w.chunk, cos_sin=cs,
                          kvbar=kvbar, kr_index=index)

    steps = max(3, min(args.steps, 10))
    with ClockSampler(torch.cuda.current_device()) as clk:
        enc_ms = device_ms(encode, steps, args.warmup, s)
    read = 3 * w.n_tok * w.H * w.d * 2
    write = lay.n_chunks * 3 * w.H * w.d * 2
    gbs = (read + write) / (enc_ms / 1e3) / 1e9
    del k, v, kr
    _free()
    # oracle: document-wise RoPE + pooling of K, V, K^R of the first 16 documents (16,384 tokens)
    n_s = 16

    def oracle_encode():
        a, b = 0, int(w.doc_tok_off[n_s])
        t = {n: w.host_rows(0, n, np.arange(a, b)).reshape(b - a, -1, w.d) for n in ("k", "v", "kr")}
        O.encode_memory(t["k"], t["v"], t["kr"], w.doc_tok_off[:n_s + 1], w.chunk, w.rope_base)

    enc_cpu = cpu_seconds(oracle_encode, 3.0, 5)
    encode_entry = {
        "workload": f"10m encode: {w.n_docs:,} docs x 1024 tokens, chunk 256, K/V/K^R bf16 [{w.n_tok:,} x 8 x 128]",
        "metric": "10M offline encode (document-wise RoPE + chunk-mean pooling) throughput",
        "value": w.n_tok / (enc_ms / 1e3), "unit": "memory tokens/s", "higher_is_better": True, "ms_per_step": enc_ms,
        "steps": steps,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s", "frac": gbs / pk["hbm"],
                     "traffic": POOL_TRAFFIC_10M if w.n_docs == 9766 else None, "kernel": "pool_kernel",
                     "peak_kind": f"{pk['kind']} copy bandwidth", "bytes": read + write},
        "cpu_baseline": {"value": n_s * 1024 / enc_cpu, "unit": "memory tokens/s", "cores": oracle_threads(),
                         "kind": "oracle", "sample": f"fp64 oracle encode of the first {n_s} documents "
                                                     f"({n_s * 1024:,} tokens, generation included)"},
        "e2e": None,
        "e2e_note": "the encode's inputs are the model's token-level K/V/K^R, produced on the device; with them "
                    "on the host the step is the 61.4 GB host->device copy",
        "clocks": clk.summary(), "checks": {"device_status": m.device_status()}}

    # decode: one round of 32 independent queries x 1 token over the pooled bank
    host_bank = to_host_bank(kvbar)
    rb = OneLayerRound(m, w, lay, index, host_bank, cs, args.fetch_mode)
    entry = _round_entry("10m decode: 39,064 chunks (chunk 256), 32 queries x 1 decode token, top-16, per-query "
                         "fetch from the pinned host bank", "10M decode: route + top-16 + fetch + attention, "
                         "32 queries", w, lay, rb, min(args.steps, 200), args.warmup, pk, "hbm",
                         "80 MB index per step (32 columns: HBM-bound); the fetch reads 8.4 MB over the host link",
                         None)
    # the fetch alone, over the host link, against a pinned copy measured in this process
    idx_dev = torch.from_numpy(rb.idx_host.numpy().copy()).cuda()
    mem = torch.empty((w.n_q, w.max_mem, 2, w.hkv, w.d), dtype=torch.bfloat16, device="cuda")
    mem_len = torch.empty(w.n_q, dtype=torch.int32, device="cuda")
    f_ms = device_ms(lambda: m.msa_gather_kv_device(host_bank, lay.doc_chunk_off, idx_dev, w.max_mem, dev_mem_kv=mem,
                                                    mem_len=mem_len), min(args.steps, 100), args.warmup, s)
    f_bytes = int(mem_len.sum().item()) * 2 * w.hkv * w.d * 2
    link = host_link_gbs()
    entry["fetch"] = {"bound": "host-link", "achieved": f_bytes / (f_ms / 1e3) / 1e9, "peak": link, "unit": "GB/s",
                      "frac": f_bytes / (f_ms / 1e3) / 1e9 / link, "bytes": f_bytes, "us": f_ms * 1e3,
                      "kernel": "gather_device_kernel",
                      "peak_kind": "pinned host->device copy of 1 GiB measured in this process"}
    # oracle: route the 32 decode tokens over the chunks of the first 1,024 documents (4,096 chunks),
    # projected to the whole bank by chunks, plus top-16, gather and attention for every query
    n_d = min(1024, w.n_docs)
    krb = _oracle_pool_router(w, n_d)
    kv_of = _oracle_kv_of_docs(w, range(w.k))
    step = _oracle_step_fn(w, krb, kv_of)
    t_all = cpu_seconds(step, 2.0, 5)
    qr = w.qr(0)[:, :1]
    off = w.doc_chunk_off[:n_d + 1]
    t_route = cpu_seconds(lambda: O.route(krb, off, qr), 1.0, 5)
    proj = t_all + t_route * (lay.n_chunks / krb.shape[0] - 1)
    entry["cpu_baseline"] = {"value": proj * 1e6, "unit": "us per step", "cores": oracle_threads(), "kind": "oracle",
                             "sample": f"fp64 oracle step over the chunks of the first {n_d:,} documents "
                                       f"({krb.shape[0]:,} chunks; {t_all * 1e6:.0f} us), its routing part scaled "
                                       f"by chunks to all {lay.n_chunks:,} (projection)"}
    del rb, mem, host_bank, kvbar, index
    _free()
    return encode_entry, entry


def cfg_interleave(args, pk):
    """Three Memory Interleave rounds (64 + 32 + 32 tokens per query, 8 queries) over a 10M-token
    pre-pooled bank (78,128 chunks of 128) and 18 routed layers; one step = the three rounds."""
    import numpy as np
    import torch

    import oracle as O
    import routed_long_context_b200 as m
    from msa_inputs import workloads
    from msa_inputs.device import memory_tensor, small_tensors
    from routed_long_context_b200.bank import BankLayout, index_from_prepooled

    w = workloads.interleave(layers=args.layers, n_host_banks=args.host_banks)
    lay = BankLayout(w.doc_chunks)
    cs = m.rope_table(4096, w.d, w.rope_base)
    dt = torch.bfloat16
    index = [index_from_prepooled(lay, memory_tensor(w, l, "krbar")) for l in range(w.layers)]
    banks = []
    for s_ in range(w.n_host_banks):
        dev = memory_tensor(w, s_, "bank")
        banks.append(_pinned_like(dev))
        del dev
    small = [small_tensors(w, l) for l in range(w.layers)]
    local = [(torch.zeros((w.n_q, w.T_total, w.hkv, w.d), dtype=dt, device="cuda"),
              torch.zeros((w.n_q, w.T_total, w.hkv, w.d), dtype=dt, device="cuda")) for _ in range(w.layers)]
    outs = [[torch.empty((w.n_q, w.round_tokens(r)[1], w.hq, w.d), dtype=dt, device="cuda") for r in range(w.rounds)]
            for _ in range(w.layers)]
    idx_host = [[torch.empty((w.n_q, w.k), dtype=torch.int32, pin_memory=True) for _ in range(w.rounds)]
                for _ in range(w.layers)]
    compute, copy = torch.cuda.Stream(), torch.cuda.Stream()
    # the routing queries of round r are the first L_prev + n_new tokens: a contiguous copy per round
    qr_round = [[torch.empty((w.n_q, sum(w.round_tokens(r)), w.H, w.d), dtype=dt, device="cuda")
                 for r in range(w.rounds)] for _ in range(w.layers)]

    def refresh_qr():
        for l in range(w.layers):
            for r in range(w.rounds):
                qr_round[l][r].copy_(small[l]["qr"][:, :qr_round[l][r].shape[1]])

    with torch.cuda.stream(compute):
        refresh_qr()
    rounds = []
    for r in range(w.rounds):
        L_prev, tn = w.round_tokens(r)
        la = [dict(kr_index=index[l], host_bank=banks[w.host_bank_slot(l)], qr=qr_round[l][r],
                   q_new=small[l]["q"][:, L_prev:], k_new=small[l]["k_new"][:, L_prev:],
                   v_new=small[l]["v_new"][:, L_prev:], local_k=local[l][0], local_v=local[l][1], out=outs[l][r],
                   topk_idx_host=idx_host[l][r]) for l in range(w.layers)]
        rounds.append(m.InterleaveRound(la, n_chunks=lay.n_chunks, n_docs=lay.n_docs, doc_chunk_off=lay.doc_chunk_off,
                                        doc_chunk_off_host=lay.doc_chunk_off_host, chunk_doc=lay.chunk_doc, n_q=w.n_q,
                                        H=w.H, d=w.d, hq=w.hq, hkv=w.hkv, k=w.k, L_prev=L_prev, T_new=tn,
                                        new_q_stride=w.T_total, L_max=w.T_total, max_mem=w.max_mem, cos_sin=cs,
                                        dtype=dt, fetch_mode=args.fetch_mode))
    steps = max(3, min(args.steps, 20))
    for _ in range(args.warmup):
        for rd in rounds:
            rd.run(compute, copy)
    torch.cuda.synchronize()
    chain_ok = all(set(w.expected(l, r, q)) <= set(idx_host[l][r][q].tolist())
                   for l in range(w.layers) for r in range(w.rounds) for q in range(w.n_q))
    route_ev = [[[_ev() for _ in range(2 * w.layers)] for _ in range(w.rounds)] for _ in range(steps)]
    for a in route_ev:
        for b in a:
            for e in b:
                e.record(compute)
    e0, e1 = _ev(), _ev()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record(compute)
        for i in range(steps):
            for r, rd in enumerate(rounds):
                rd.run(compute, copy, route_events=route_ev[i][r])
        e1.record(compute)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    flops = [2.0 * w.H * w.d * lay.n_chunks * w.n_q * sum(w.round_tokens(r)) for r in range(w.rounds)]
    rms = [sum(route_ev[i][r][2 * l].elapsed_time(route_ev[i][r][2 * l + 1]) for i in range(steps)
               for l in range(w.layers)) / (steps * w.layers) for r in range(w.rounds)]
    tflops = [f / (t / 1e3) / 1e12 for f, t in zip(flops, rms)]
    peak = pk["bf16_sustained"]

    # end to end: every step copies all layers' query-side inputs (pinned host) in, runs the three
    # rounds and reads every round's attention output back, serialised on the compute stream
    names = ("qr", "q", "k_new", "v_new")
    h_in = [[_pinned_like(small[l][n]) for n in names] for l in range(w.layers)]
    h_out = [[_pinned_like(outs[l][r]) for r in range(w.rounds)] for l in range(w.layers)]

    def e2e_step():
        with torch.cuda.stream(compute):
            for l in range(w.layers):
                for h, n in zip(h_in[l], names):
                    small[l][n].copy_(h, non_blocking=True)
            refresh_qr()
        for rd in rounds:
            rd.run(compute, copy)
        with torch.cuda.stream(compute):
            for l in range(w.layers):
                for r in range(w.rounds):
                    h_out[l][r].copy_(outs[l][r], non_blocking=True)

    e_ms = device_ms(e2e_step, steps, 1, compute)
    h2d = sum(h.numel() * h.element_size() for hl in h_in for h in hl)
    d2h = sum(h.numel() * h.element_size() for hl in h_out for h in hl) + \
        sum(t.numel() * 4 for tl in idx_host for t in tl)
    tokens = lay.n_chunks * TOKENS_PER_CHUNK * w.layers * w.rounds

    # oracle: routing of one query's round-3 tokens (128) over leading slices of layer 0's bank for
    # ~3 s (the dominant cost of a round), memory tokens routed per second
    qr3 = w.qr(0)[:1, :sum(w.round_tokens(w.rounds - 1))]
    done, t0 = 0, time.perf_counter()
    while done < w.n_docs and time.perf_counter() - t0 < 3.0:
        d1 = min(w.n_docs, done + 512)
        a, b = int(w.doc_chunk_off[done]), int(w.doc_chunk_off[d1])
        rows = w.host_rows(0, "krbar", np.arange(a, b)).reshape(b - a, w.H, w.d)
        O.topk_docs(O.route(rows, w.doc_chunk_off[done:d1 + 1] - a, qr3)[0], w.k)
        done = d1
    cpu_rate = int(w.doc_chunk_off[done]) * TOKENS_PER_CHUNK / (time.perf_counter() - t0)
    entry = {
        "workload": "interleave: 78,128 chunks x 18 layers, 8 queries, 3 rounds (64/96/128 routing tokens), top-12",
        "metric": "Memory Interleave: memory tokens routed/s (3 rounds x 18 layers over a 10M-token bank)",
        "value": tokens / (ms / 1e3), "unit": "memory tokens/s", "higher_is_better": True, "ms_per_step": ms,
        "steps": steps, "route_ms_per_layer_by_round": rms, "route_tflops_by_round": tflops,
        "roofline": {"bound": "tensor", "achieved": tflops[-1], "peak": peak, "unit": "TFLOP/s",
                     "frac": tflops[-1] / peak, "frac_by_round": [t / peak for t in tflops], "traffic": None,
                     "kernel": "route_tc_kernel, round 3 (1,024 columns)",
                     "peak_kind": f"{pk['kind']} sustained bf16 (cuBLAS)"},
        "cpu_baseline": {"value": cpu_rate, "unit": "memory tokens/s", "cores": oracle_threads(), "kind": "oracle",
                         "sample": f"fp64 oracle routing + top-12 of one query's 128 round-3 tokens over the first "
                                   f"{int(w.doc_chunk_off[done]):,} chunks of one layer"},
        "e2e": {"value": tokens / (e_ms / 1e3), "unit": "memory tokens/s", "ms_per_step": e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "how": "public API (msa_interleave_step per round) with pinned host buffers: all layers' query-side "
                       "inputs in and every round's output back inside the timed region, serialised"},
        "clocks": clk.summary(),
        "checks": {"chain_docs_selected": chain_ok, "device_status": m.device_status()}}
    del rounds, index, banks, small, local, outs
    _free()
    return entry


def host_link_gbs(nbytes: int = 1 << 30, reps: int = 5) -> float:
    """Pinned host -> device copy bandwidth measured in this process (best of reps, CUDA events)."""
    import torch

    h = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    d = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    best = float("inf")
    for _ in range(reps):
        a, b = _ev(), _ev()
        a.record()
        d.copy_(h, non_blocking=True)
        b.record()
        torch.cuda.synchronize()
        best = min(best, a.elapsed_time(b))
    del h, d
    return nbytes / (best / 1e3) / 1e9


def cfg_fine1m(args, pk):
    """Token-level fine stage on the 1M-token bank: one step = route (pooled index) + top-8 + fetch of
    the selected documents' token K/V from the pinned token bank + global RoPE of the local context +
    split-key attention of 64 query tokens over those rows."""
    import numpy as np
    import torch

    import oracle as O
    import routed_long_context_b200 as m
    from msa_inputs import workloads
    from msa_inputs.device import memory_tensor, small_tensors
    from routed_long_context_b200.bank import BankLayout, to_host_bank

    w = workloads.mem_1m()
    lay = BankLayout.from_doc_lengths(w.doc_len, w.chunk)
    cs = m.rope_table(4096, w.d, w.rope_base)
    k, v, kr = (memory_tensor(w, 0, n) for n in ("k", "v", "kr"))
    _, index = m.msa_pool_chunks(None, None, kr, lay.doc_tok_off, lay.doc_chunk_off, lay.chunk_doc, w.chunk)
    tok = m.msa_pack_tokens(k, v, lay.doc_tok_off, cs)
    del k, v, kr
    host_tok = to_host_bank(tok)
    del tok
    _free()
    dv = small_tensors(w, 0)
    T, max_mem = w.T0, w.k * int(w.doc_len.max())
    seg = torch.tensor([0, T], dtype=torch.int64, device="cuda")
    ds = torch.empty((w.n_q, lay.n_docs), dtype=torch.float32, device="cuda")
    idx = torch.empty((w.n_q, w.k), dtype=torch.int32, device="cuda")
    sc = torch.empty((w.n_q, w.k), dtype=torch.float32, device="cuda")
    idx_h = torch.empty((w.n_q, w.k), dtype=torch.int32, pin_memory=True)
    mem = torch.zeros((w.n_q, max_mem, 2, w.hkv, w.d), dtype=torch.bfloat16, device="cuda")
    mem_len = torch.zeros(w.n_q, dtype=torch.int32, device="cuda")
    lk, qq = torch.empty_like(dv["k_new"][0]), torch.empty_like(dv["q"][0])
    out = torch.empty((w.n_q, T, w.hq, w.d), dtype=torch.bfloat16, device="cuda")
    rws = m.api._ws(m.route_workspace_size(w.n_q, T, w.H, w.d, torch.bfloat16), "cuda")
    tws = m.api._ws(m.topk_workspace_size(w.n_q, lay.n_docs, w.k), "cuda")
    aws = m.api._ws(m.sparse_attn_split_workspace_size(w.n_q, T, w.hq, w.hkv, max_mem, T), "cuda")
    s = torch.cuda.current_stream()

    def step(ev=None):
        if ev: ev[0].record(s)
        m.msa_route_scores(index, lay.chunk_doc, lay.n_docs, dv["qr"], doc_scores=ds, ws=rws)
        m.msa_topk_docs(ds, w.k, idx=idx, score=sc, ws=tws)
        if ev: ev[1].record(s)
        if args.fetch_mode == 1:
            m.msa_gather_kv_device(host_tok, lay.doc_tok_off, idx, max_mem, dev_mem_kv=mem, mem_len=mem_len)
        else:
            idx_h.copy_(idx, non_blocking=True)
            s.synchronize()
            _, ml = m.msa_gather_kv(host_tok, w.doc_tok_off, idx_h, max_mem, dev_mem_kv=mem, copy_stream=s)
            mem_len.copy_(ml, non_blocking=True)
        if ev: ev[2].record(s)
        m.msa_rope_doc(dv["k_new"][0], seg, w.k, cs, out=lk)
        m.msa_rope_doc(dv["q"][0], seg, w.k, cs, out=qq)
        if ev: ev[3].record(s)
        m.msa_sparse_attn_split(qq[None], mem, mem_len, lk[None], dv["v_new"], T, 0, out=out, ws=aws)
        if ev: ev[4].record(s)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    rows = int(mem_len.cpu().sum())
    gi = idx.cpu().numpy()[0]
    planted_ok = set(w.expected(0, 0, 0)) <= set(gi.tolist())
    steps = max(3, min(args.steps, 100))
    evs = [[_ev() for _ in range(5)] for _ in range(steps)]
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i in range(steps):
            step(evs[i])
        torch.cuda.synchronize()
    route_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / steps
    fetch_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / steps
    rope_ms = sum(e[2].elapsed_time(e[3]) for e in evs) / steps
    attn_ms = sum(e[3].elapsed_time(e[4]) for e in evs) / steps
    ms = sum(e[0].elapsed_time(e[4]) for e in evs) / steps
    fetch_bytes = rows * 2 * w.hkv * w.d * 2
    link = host_link_gbs()
    fetch_gbs = fetch_bytes / (fetch_ms / 1e3) / 1e9
    attn_flops = 4.0 * w.n_q * T * w.hq * w.d * (rows + T / 2)
    attn_tflops = attn_flops / attn_ms / 1e9

    # end to end: query-side inputs in, the step, the attention output back, serialised
    names = ("qr", "q", "k_new", "v_new")
    h_in = [_pinned_like(dv[n]) for n in names]
    h_out = _pinned_like(out)

    def e2e_step():
        for h, n in zip(h_in, names):
            dv[n].copy_(h, non_blocking=True)
        step()
        h_out.copy_(out, non_blocking=True)

    e_ms = device_ms(e2e_step, steps, 1, s)
    # oracle: routing over the first 125 documents' chunks (projected by chunks to the whole bank)
    # and the token-level attention of the 64 query tokens over the rows of the 8 planted documents
    krb = _oracle_pool_router(w, 125)
    t_route = cpu_seconds(lambda: O.topk_docs(O.route(krb, w.doc_chunk_off[:126], w.qr(0)[:, :T])[0], w.k), 1.0, 5)
    pdocs = w.expected(0, 0, 0)
    trows = np.concatenate([np.arange(w.doc_tok_off[d], w.doc_tok_off[d + 1]) for d in pdocs])
    kt = w.host_rows(0, "k", trows).reshape(len(trows), w.hkv, w.d)
    vt = w.host_rows(0, "v", trows).reshape(len(trows), w.hkv, w.d)
    tb = O.token_bank(kt, vt, np.concatenate([[0], np.cumsum(w.doc_len[pdocs])]), w.rope_base)
    pos = O.global_positions(w.k, 0, T)
    qo = O.apply_rope(w.q(0)[0], pos, w.rope_base)
    kl = O.apply_rope(w.k_new(0)[0], pos, w.rope_base)
    t_attn = cpu_seconds(lambda: O.sparse_attention(qo, tb[:, 0], tb[:, 1], kl, w.v_new(0)[0], 0, 1 / np.sqrt(w.d)),
                         1.0, 5)
    cpu_step = t_route * lay.n_chunks / krb.shape[0] + t_attn * rows / len(trows)
    entry = {
        "workload": f"fine1m: {w.n_docs} docs ({w.n_tok:,} tokens), token bank {w.n_tok * 4096 / 1e9:.1f} GB pinned "
                    f"host, 64 query tokens, top-8 -> {rows} token rows",
        "metric": "1M fine stage: token rows fetched and attended per second (route + top-8 + token fetch + split "
                  "attention)",
        "value": rows / (ms / 1e3), "unit": "memory token rows/s", "higher_is_better": True, "ms_per_step": ms,
        "steps": steps, "fetch_mode": args.fetch_mode,
        "attn_plan": m.api.sparse_attn_split_plan(w.n_q, T, w.hq, w.hkv, max_mem, T),
        "route_topk_ms": route_ms, "fetch_ms": fetch_ms, "rope_ms": rope_ms, "attn_ms": attn_ms,
        "attn_tflops": attn_tflops, "attn_what": "split-key attention + combine (the two RoPE launches of the "
                                                "local context are rope_ms)",
        "attn_roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": pk["bf16"], "unit": "TFLOP/s",
                          "frac": attn_tflops / pk["bf16"], "kernel": "attn_tc_kernel + attn_combine_kernel",
                          "peak_kind": f"{pk['kind']} bf16 burst (cuBLAS)"},
        "roofline": {"bound": "host-link", "achieved": fetch_gbs, "peak": link, "unit": "GB/s",
                     "frac": fetch_gbs / link, "traffic": None,
                     "kernel": "gather_device_kernel" if args.fetch_mode == 1 else "cudaMemcpyAsync per document",
                     "peak_kind": "pinned host->device copy of 1 GiB measured in this process",
                     "bytes": fetch_bytes},
        "cpu_baseline": {"value": rows / cpu_step, "unit": "memory token rows/s", "cores": oracle_threads(),
                         "kind": "oracle",
                         "sample": "fp64 oracle routing over the first 125 documents' chunks scaled by chunks to the "
                                   "bank, plus token-level attention over the 8 planted documents' rows scaled by "
                                   "rows to the step's (projection)"},
        "e2e": {"value": rows / (e_ms / 1e3), "unit": "memory token rows/s", "ms_per_step": e_ms,
                "h2d_bytes_per_step": sum(h.numel() * h.element_size() for h in h_in),
                "d2h_bytes_per_step": h_out.numel() * h_out.element_size(),
                "how": "public API calls with pinned host buffers: query-side inputs in and the output back inside "
                       "the timed region, serialised"},
        "clocks": clk.summary(),
        "checks": {"planted_docs_selected": planted_ok, "device_status": m.device_status()}}
    del host_tok, mem, index
    _free()
    return entry


def run_configs(args, pk):
    """Every configuration, one after the other (each frees its device memory before the next)."""
    out = {}
    for name, fn in (("tiny", cfg_tiny), ("1m", cfg_1m), ("10m", cfg_10m), ("interleave", cfg_interleave),
                     ("fine1m", cfg_fine1m)):
        t0 = time.perf_counter()
        try:
            r = fn(args, pk)
        except Exception as e:  # one configuration failing must not hide the others: report it
            out[name] = {"error": repr(e)[:500]}
            continue
        if name == "10m":
            out["10m_encode"], out["10m_decode"] = r
        else:
            out[name] = r
        out.setdefault("_wall_s", {})[name] = time.perf_counter() - t0
    return out


def workload_line(args, entry, world):
    """A configuration entry printed as a line of its own (`--workload X`)."""
    line = {"metric": entry["metric"], "value": entry["value"], "unit": entry["unit"], "n_gpus": world,
            "steps": entry.get("steps", args.steps), "warmup": args.warmup, "ms_per_step": entry["ms_per_step"],
            "higher_is_better": entry.get("higher_is_better", True), "scaling": "weak", "vs_baseline": None,
            "dtype": "f32" if entry["workload"].startswith("tiny") else "bf16", "data": "synthetic",
            "config": {"workload": entry["workload"]}}
    line.update({k: v for k, v in entry.items() if k not in line and k not in ("workload",)})
    print(json.dumps(line))

# ---------------------------------------------------------------------------------------------- training step
def train_bench(args, rank, world, local_rank):
    """One training step of a routed layer on the 64K-token training context (16 docs x 4096 tokens,
    chunk 128; one query of 512 tokens; top-4): forward (encode, route, top-k, fetch, split attention
    with log-sum-exp) and backward (attention, fetch, auxiliary router loss, router, pooling), each
    call timed with CUDA events."""
    import numpy as np
    import torch

    import routed_long_context_b200 as m
    from msa_inputs import rng, workloads
    from msa_inputs.device import memory_tensor, small_tensors, upload
    from routed_long_context_b200.bank import BankLayout

    torch.cuda.set_device(local_rank)
    w = workloads.train64k()
    lay = BankLayout.from_doc_lengths(w.doc_len, w.chunk)
    cs = m.rope_table(8192, w.d, w.rope_base)
    k, v, kr = (memory_tensor(w, 0, n) for n in ("k", "v", "kr"))
    sm = small_tensors(w, 0)
    T, C, dt = w.T0, lay.n_chunks, torch.bfloat16
    max_mem = w.k * int(w.doc_chunks.max())
    kvbar = torch.empty((C, 2, w.hkv, w.d), dtype=dt, device="cuda")
    index = torch.empty((C, w.H, w.d), dtype=dt, device="cuda")
    ds = torch.empty((1, lay.n_docs), dtype=torch.float32, device="cuda")
    idx = torch.empty((1, w.k), dtype=torch.int32, device="cuda")
    sc = torch.empty((1, w.k), dtype=torch.float32, device="cuda")
    mem = torch.zeros((1, max_mem, 2, w.hkv, w.d), dtype=dt, device="cuda")
    mem_len = torch.zeros(1, dtype=torch.int32, device="cuda")
    seg = torch.tensor([0, T], dtype=torch.int64, device="cuda")
    lk, qq = torch.empty_like(sm["k_new"][0]), torch.empty_like(sm["q"][0])
    out = torch.empty((1, T, w.hq, w.d), dtype=dt, device="cuda")
    lse = torch.empty((1, T, w.hq), dtype=torch.float32, device="cuda")
    dout = upload(rng.normal(w.seed, 1 << 50, 0, T * w.hq * w.d, 1.0, "bf16").reshape(1, T, w.hq, w.d), "bf16")
    grads = (torch.zeros((1, T, w.hq, w.d), dtype=torch.float32, device="cuda"),
             torch.zeros((1, max_mem, 2, w.hkv, w.d), dtype=torch.float32, device="cuda"),
             torch.zeros((1, T, w.hkv, w.d), dtype=torch.float32, device="cuda"),
             torch.zeros((1, T, w.hkv, w.d), dtype=torch.float32, device="cuda"))
    dkvbar = torch.zeros((C, 2, w.hkv, w.d), dtype=torch.float32, device="cuda")
    evidence = torch.tensor([w.expected(0, 0, 0)], dtype=torch.int32, device="cuda")
    rws = m.api._ws(m.route_workspace_size(1, T, w.H, w.d, dt), "cuda")
    tws = m.api._ws(m.topk_workspace_size(1, lay.n_docs, w.k), "cuda")
    aws = m.api._ws(m.sparse_attn_split_workspace_size(1, T, w.hq, w.hkv, max_mem, T), "cuda")
    s = torch.cuda.current_stream()
    names = ["encode", "route+topk", "fetch", "attn_fwd", "attn_bwd", "fetch_bwd", "aux_loss", "route_bwd", "pool_bwd"]

    def step(ev=None):
        def mark(i):
            if ev:
                ev[i].record(s)
        mark(0)
        m.msa_pool_chunks(k, v, kr, lay.doc_tok_off, lay.doc_chunk_off, lay.chunk_doc, w.chunk, cos_sin=cs,
                          kvbar=kvbar, kr_index=index)
        mark(1)
        m.msa_route_scores(index, lay.chunk_doc, lay.n_docs, sm["qr"], doc_scores=ds, ws=rws)
        m.msa_topk_docs(ds, w.k, idx=idx, score=sc, ws=tws)
        mark(2)
        m.msa_gather_kv_device(kvbar, lay.doc_chunk_off, idx, max_mem, dev_mem_kv=mem, mem_len=mem_len)
        mark(3)
        m.msa_rope_doc(sm["k_new"][0], seg, w.k, cs, out=lk)
        m.msa_rope_doc(sm["q"][0], seg, w.k, cs, out=qq)
        m.msa_sparse_attn_split(qq[None], mem, mem_len, lk[None], sm["v_new"], T, 0, out=out, ws=aws, lse=lse)
        mark(4)
        m.msa_sparse_attn_backward(qq[None], mem, mem_len, lk[None], sm["v_new"], T, 0, out, dout, lse, grads=grads)
        mark(5)
        m.msa_gather_kv_backward(grads[1], lay.doc_chunk_off, idx, C, dkvbar=dkvbar)
        mark(6)
        _, g_aux = m.msa_router_aux_loss(ds, evidence, 1.0)
        mark(7)
        _, dkhat = m.msa_route_backward(index, lay.doc_chunk_off, sm["qr"], g_aux)
        mark(8)
        m.msa_pool_chunks_backward(dkvbar, dkhat, lay.doc_tok_off, lay.doc_chunk_off, lay.chunk_doc, w.chunk, w.n_tok,
                                   kr=kr, cos_sin=cs)
        mark(9)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    planted_ok = set(w.expected(0, 0, 0)) <= set(idx.cpu().numpy()[0].tolist())
    steps = min(args.steps, 100)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(10)] for _ in range(steps)]
    with ClockSampler(local_rank) as clk:
        for i in range(steps):
            step(evs[i])
        torch.cuda.synchronize()
    part = {n: sum(e[j].elapsed_time(e[j + 1]) for e in evs) / steps for j, n in enumerate(names)}
    ms = sum(e[0].elapsed_time(e[9]) for e in evs) / steps
    # attention backward FLOPs: rows x visible keys x d x 2, for S, dP, dV, dK (key tiles) and S, dP, dQ (row blocks)
    rows = T * w.hq
    keys = float(mem_len.item()) + (T + 1) / 2.0
    bwd_flops = 7 * 2.0 * rows * keys * w.d
    pool_bwd_bytes = 3 * w.n_tok * w.hkv * w.d * 4 + w.n_tok * w.H * w.d * 2 + C * 3 * w.H * w.d * 4
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        bf16_peak, hbm_peak, kind = float(pk["bf16_tflops"]), float(pk["hbm_gbs"]), "measured"
    except Exception:
        bf16_peak, hbm_peak, kind = 1590.0, 6650.0, "fallback"
    if rank == 0:
        pool_gbs = pool_bwd_bytes / (part["pool_bwd"] / 1e3) / 1e9
        print(json.dumps({
            "metric": "train64k: training step of one routed layer (forward + backward), memory tokens/s",
            "value": w.n_tok / (ms / 1e3), "unit": "memory tokens/s", "n_gpus": 1, "steps": steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "train64k: 16 docs x 4096 tokens, chunk 128, 1 query x 512 tokens, top-4, "
                                   "GQA 32/8, d 128, aux loss tau 1"},
            "ms_by_call": part,
            "attn_bwd_tflops": bwd_flops / (part["attn_bwd"] / 1e3) / 1e12,
            "roofline": {"bound": "hbm", "achieved": pool_gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": pool_gbs / hbm_peak, "traffic": None, "kernel": "pool_bwd_kernel",
                         "bytes": pool_bwd_bytes, "peak_kind": kind},
            "attn_bwd_roofline": {"bound": "tensor", "achieved": bwd_flops / (part["attn_bwd"] / 1e3) / 1e12,
                                  "peak": bf16_peak, "unit": "TFLOP/s",
                                  "frac": bwd_flops / (part["attn_bwd"] / 1e3) / 1e12 / bf16_peak},
            "checks": {"planted_docs_selected": planted_ok, "device_status": m.device_status()},
            "clocks": clk.summary()}))


# ---------------------------------------------------------------------------------------------- ours
def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        return reference_arm(args, rank)
    if args.workload in ("tiny", "1m", "encode10m", "decode10m", "interleave", "fine1m"):
        import torch

        torch.cuda.set_device(local_rank)
        pk = all_peaks()
        fn = {"tiny": cfg_tiny, "1m": cfg_1m, "encode10m": cfg_10m, "decode10m": cfg_10m,
              "interleave": cfg_interleave, "fine1m": cfg_fine1m}[args.workload]
        entry = fn(args, pk)
        if args.workload in ("encode10m", "decode10m"):
            entry = entry[0] if args.workload == "encode10m" else entry[1]
        if rank == 0:
            workload_line(args, entry, world)
        return
    if args.workload == "train64k":
        return train_bench(args, rank, world, local_rank)

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local_rank)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local_rank))
    line = headline(args, rank, world, local_rank)
    _free()                                            # the headline's 30 GB are released here
    if world == 1 and not args.no_configs:
        line["configs"] = run_configs(args, all_peaks())
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


def headline(args, rank, world, local_rank):
    """The 100M routing step: 18 routed layers per step (the reported metric); returns the JSON line."""
    import numpy as np
    import torch
    import torch.distributed as dist

    import routed_long_context_b200 as m
    from msa_inputs import workloads
    from msa_inputs.device import memory_tensor, small_tensors
    from routed_long_context_b200.bank import BankLayout, index_from_prepooled

    m.api.route_set_max_stages(args.router_stages)

    def barrier():
        if world > 1:
            dist.barrier()

    w = workloads.mem_100m(layers=args.layers, n_host_banks=args.host_banks, n_docs=args.n_docs)
    lay = BankLayout(w.doc_chunks)
    cs = m.rope_table(4096, w.d, w.rope_base)
    dt = torch.bfloat16

    # ---- offline encoding: generated raw pooled router keys -> per-head unit vectors (in place)
    index = []
    for l in range(w.layers):
        raw = memory_tensor(w, l, "krbar")
        index.append(index_from_prepooled(lay, raw, out=raw))
    banks = []
    for s in range(w.n_host_banks):
        dev = memory_tensor(w, s, "bank")
        host = torch.empty(dev.shape, dtype=dt, pin_memory=True)
        host.copy_(dev)
        banks.append(host)
        del dev
    torch.cuda.synchronize()
    assert m.device_status() == 0

    small = [small_tensors(w, l) for l in range(w.layers)]
    local = [(torch.zeros((1, w.T0, w.hkv, w.d), dtype=dt, device="cuda"),
              torch.zeros((1, w.T0, w.hkv, w.d), dtype=dt, device="cuda")) for _ in range(w.layers)]
    outs = [torch.empty((1, w.T0, w.hq, w.d), dtype=dt, device="cuda") for _ in range(w.layers)]
    idx_host = [torch.empty((1, w.k), dtype=torch.int32, pin_memory=True) for _ in range(w.layers)]
    layer_args = [dict(kr_index=index[l], host_bank=banks[w.host_bank_slot(l)], qr=small[l]["qr"],
                       q_new=small[l]["q"], k_new=small[l]["k_new"], v_new=small[l]["v_new"], local_k=local[l][0],
                       local_v=local[l][1], out=outs[l], topk_idx_host=idx_host[l]) for l in range(w.layers)]
    compute = torch.cuda.Stream()
    copy = torch.cuda.Stream()
    rnd = m.InterleaveRound(layer_args, n_chunks=lay.n_chunks, n_docs=lay.n_docs, doc_chunk_off=lay.doc_chunk_off,
                            doc_chunk_off_host=lay.doc_chunk_off_host, chunk_doc=lay.chunk_doc, n_q=1, H=w.H, d=w.d,
                            hq=w.hq, hkv=w.hkv, k=w.k, L_prev=0, T_new=w.T0, new_q_stride=w.T0, L_max=w.T0,
                            max_mem=w.max_mem, cos_sin=cs, dtype=dt, reserved_sms=args.reserved_sms,
                            fetch_mode=args.fetch_mode)

    # ---- warm-up, then K timed steps (inputs are 1.6 GB per layer: larger than L2, no flush needed)
    for _ in range(args.warmup):
        rnd.run(compute, copy)
    torch.cuda.synchronize()
    planted_ok = all(set(w.expected(l, 0, 0)) <= set(idx_host[l][0].tolist()) for l in range(w.layers))
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # events around every router launch of every timed step (recorded by the library on `compute`)
    route_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * w.layers)] for _ in range(args.steps)]
    for evs in route_ev:
        for e in evs:
            e.record(compute)                  # materialise the underlying cudaEvent_t
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        ev0.record(compute)
        for i in range(args.steps):
            rnd.run(compute, copy, route_events=route_ev[i])
        ev1.record(compute)
        torch.cuda.synchronize()
    barrier()
    ms_step = ev0.elapsed_time(ev1) / args.steps
    route_ms_live = sum(evs[2 * l].elapsed_time(evs[2 * l + 1]) for evs in route_ev for l in range(w.layers)) / (
        args.steps * w.layers)

    # ---- router scoring alone (isolated loop, for reference), per layer, on the compute stream
    route_ws = torch.empty(m.api.route_workspace_size(1, w.T0, w.H, w.d, dt), dtype=torch.uint8, device="cuda")
    scores = torch.empty((1, lay.n_docs), dtype=torch.float32, device="cuda")
    reps = max(3, min(20, args.steps // 10))
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(compute):
        for l in range(w.layers):
            m.msa_route_scores(index[l], lay.chunk_doc, lay.n_docs, small[l]["qr"], doc_scores=scores, ws=route_ws,
                               stream=compute)
        r0.record(compute)
        for _ in range(reps):
            for l in range(w.layers):
                m.msa_route_scores(index[l], lay.chunk_doc, lay.n_docs, small[l]["qr"], doc_scores=scores,
                                   ws=route_ws, stream=compute)
        r1.record(compute)
    torch.cuda.synchronize()
    route_ms = r0.elapsed_time(r1) / (reps * w.layers)

    # ---- end to end through the public API with host buffers, pipelined as a serving loop runs it:
    # two sets of device input and output buffers; every step copies its query-side inputs (all
    # layers, one contiguous pinned buffer) host -> device on an input stream while the previous
    # step computes, and reads its attention outputs (and, inside the round, the selected indices)
    # back device -> host on an output stream while the next step computes. The timed region ends
    # after the last read-back, so every step's copies are inside it.
    names = ("qr", "q", "k_new", "v_new")
    in_bytes = [[small[l][k_].numel() * small[l][k_].element_size() for k_ in names] for l in range(w.layers)]
    total_in = sum(sum(b_) for b_ in in_bytes)
    host_in = torch.empty(total_in, dtype=torch.uint8, pin_memory=True)
    at = 0
    for l in range(w.layers):
        for k_, nb in zip(names, in_bytes[l]):
            host_in[at:at + nb].copy_(small[l][k_].contiguous().view(-1).view(torch.uint8).cpu())
            at += nb
    out_shape = (w.layers,) + tuple(outs[0].shape)
    sets = []
    for b_ in range(2):
        dev_in = torch.empty(total_in, dtype=torch.uint8, device="cuda")
        dev_in.copy_(host_in)
        dev_out = torch.empty(out_shape, dtype=dt, device="cuda")
        views, at = [], 0
        for l in range(w.layers):
            v_ = {}
            for k_, nb in zip(names, in_bytes[l]):
                v_[k_] = dev_in[at:at + nb].view(dt).view(small[l][k_].shape)
                at += nb
            views.append(v_)
        la = [dict(layer_args[l], qr=views[l]["qr"], q_new=views[l]["q"], k_new=views[l]["k_new"],
                   v_new=views[l]["v_new"], out=dev_out[l]) for l in range(w.layers)]
        rd = m.InterleaveRound(la, n_chunks=lay.n_chunks, n_docs=lay.n_docs, doc_chunk_off=lay.doc_chunk_off,
                               doc_chunk_off_host=lay.doc_chunk_off_host, chunk_doc=lay.chunk_doc, n_q=1, H=w.H,
                               d=w.d, hq=w.hq, hkv=w.hkv, k=w.k, L_prev=0, T_new=w.T0, new_q_stride=w.T0,
                               L_max=w.T0, max_mem=w.max_mem, cos_sin=cs, dtype=dt, reserved_sms=args.reserved_sms,
                               fetch_mode=args.fetch_mode)
        host_out = torch.empty(out_shape, dtype=dt, pin_memory=True)
        sets.append((dev_in, dev_out, rd, host_out))
    h2d = total_in
    d2h = sets[0][1].numel() * sets[0][1].element_size() + sum(t.numel() * 4 for t in idx_host)
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    done = [torch.cuda.Event() for _ in range(2)]
    ready = [torch.cuda.Event() for _ in range(2)]
    read = [torch.cuda.Event() for _ in range(2)]
    for b_ in range(2):
        done[b_].record(compute)
        read[b_].record(s_out)
    for b_ in range(2):                                        # warm the second set's round
        sets[b_][2].run(compute, copy)
    e_steps = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(compute)
    s_in.wait_stream(compute)
    for i in range(e_steps):
        b_ = i % 2
        dev_in, dev_out, rd, host_out = sets[b_]
        s_in.wait_event(done[b_])                               # this set's inputs are free again
        with torch.cuda.stream(s_in):
            dev_in.copy_(host_in, non_blocking=True)
        ready[b_].record(s_in)
        compute.wait_event(ready[b_])
        compute.wait_event(read[b_])                            # its previous outputs were read back
        rd.run(compute, copy)
        done[b_].record(compute)
        s_out.wait_event(done[b_])
        with torch.cuda.stream(s_out):
            host_out.copy_(dev_out, non_blocking=True)
        read[b_].record(s_out)
    compute.wait_stream(s_out)
    e1.record(compute)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e_steps
    assert torch.equal(sets[(e_steps - 1) % 2][3][0].cuda(), sets[(e_steps - 1) % 2][1][0])

    # the same end to end, one step at a time: inputs in, the round, outputs back, all on the compute
    # stream, so each step's copies and compute are serialised (per-step latency, no overlap)
    dev_in, dev_out, rd, host_out = sets[0]

    def serial_step():
        with torch.cuda.stream(compute):
            dev_in.copy_(host_in, non_blocking=True)
        rd.run(compute, copy)
        with torch.cuda.stream(compute):
            host_out.copy_(dev_out, non_blocking=True)

    barrier()
    e2e_serial_ms = device_ms(serial_step, args.steps, 1, compute)
    barrier()

    # ---- max over ranks
    ms_step, e2e_ms, e2e_serial_ms, route_ms, route_ms_live = max_over_ranks(
        [ms_step, e2e_ms, e2e_serial_ms, route_ms, route_ms_live], "cuda")
    tokens_per_step = lay.n_chunks * TOKENS_PER_CHUNK * w.layers
    value = whole_job_rate(tokens_per_step, world, ms_step)
    e2e_value = whole_job_rate(tokens_per_step, world, e2e_ms)
    peak, peak_kind = peaks()
    route_bytes = lay.n_chunks * w.H * w.d * 2            # bf16 index read per layer
    achieved = route_bytes / (route_ms_live / 1e3) / 1e9
    status = m.device_status()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, chunks, thr = oracle_sample(args.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": thr, "kind": "oracle",
               "sample": f"fp64 oracle routing + top-k over the first {chunks} chunks of one 100M layer "
                         f"({chunks * TOKENS_PER_CHUNK} memory tokens), 64 query tokens"}

    return {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded counter-based generator)",
            "config": {"workload": "100m: 781,250 pre-pooled chunks (chunk 128) x 18 routed layers, bf16 index "
                                   "in HBM, K/V bank in pinned host memory, 1 query x 64 tokens, top-16, GQA 32/8, d 128",
                       "layers": w.layers, "n_chunks": lay.n_chunks, "n_docs": lay.n_docs, "k": w.k,
                       "l2": "inputs larger than L2 (1.6 GB index per layer); no flush",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "route_ms_per_layer": route_ms_live,
            "route_ms_per_layer_isolated_loop": route_ms,
            "reserved_sms": args.reserved_sms,
            "router_stages": args.router_stages or "default",
            "fetch_mode": ["host cudaMemcpyAsync per document", "device fetch kernel"][args.fetch_mode],
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": ROUTER_TRAFFIC_BYTES if args.n_docs == 97657 else None,
                         "kernel": "route_tc_kernel, timed by events around each launch inside the timed steps",
                         "peak_kind": f"{peak_kind} (copy bandwidth)"},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "steps": e_steps,
                    "how": "pipelined throughput through the public API with pinned host buffers: double-buffered, "
                           "each step's H2D and D2H on their own streams overlap the neighbouring steps' compute, "
                           "all inside the timed region",
                    "serial_ms_per_step": e2e_serial_ms,
                    "serial_value": whole_job_rate(tokens_per_step, world, e2e_serial_ms),
                    "serial_how": "per-step latency: the step's H2D, its round and its D2H serialised on one "
                                  "stream, no overlap between steps"},
            # per layer: prepass, router, top-k, fetch kernel (mode 1) or memory lengths (mode 0),
            # attention; per step: one fused append for every layer
            "gpu_launches": (5 * w.layers + (w.layers + 23) // 24) * args.steps,
            "clocks": clk.summary(),
            "checks": {"planted_docs_selected": planted_ok, "device_status": status},
    }


if __name__ == "__main__":
    main()
