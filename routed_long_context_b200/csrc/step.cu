// One Memory Interleave round over all routed layers: append -> route -> top-k -> fetch -> attend.
//
// Streams: R = the caller's compute stream (routers only), C = the caller's copy stream (host-issued fetches),
// S = select (library-owned: top-k, index copy to the host, memory lengths),
// A = attend (library-owned: query prepasses, appends, attention).
//   A: every layer's router prepass (record P_l), then one fused append + query rotation launch.
//   R: for every layer: wait P_l, router kernel (optionally on fewer SMs than the GPU has), record R_l.
//   S: for every layer: wait R_l, top-k, indices -> pinned host, memory lengths, record E_l.
//   fetch_mode 0 (host-issued copies): for every layer the host waits E_l (bounded poll), enqueues one
//         cudaMemcpyAsync per document on C, records G_l; A waits G_l and runs the layer's attention.
//   fetch_mode 1 (device fetch): S runs the fetch kernel right after top-k (reading the mapped pinned
//         bank), A waits E_l and attends; the host never waits.
//   join: R waits for the last work of S and A.
// The routers run back to back; selection, fetch and attention of layer l overlap the routing of
// layers l+1.. (on SMs the routers leave free and in the copy engines).
#include <algorithm>
#include <chrono>
#include <new>
#include <mutex>
#include <thread>
#include <vector>

#include "common.cuh"
#include "kernels.cuh"

namespace msa {
namespace {

__global__ void mem_len_kernel(const int32_t* __restrict__ idx, int n_q, int k, const int64_t* __restrict__ doc_chunk_off,
                               int64_t n_docs, int max_mem, int32_t* __restrict__ mem_len, int* err) {
    for (int q = blockIdx.x * blockDim.x + threadIdx.x; q < n_q; q += gridDim.x * blockDim.x) {
        int64_t rows = 0;
        for (int r = 0; r < k; ++r) {
            const int32_t doc = idx[q * k + r];
            if (doc < 0 || doc >= n_docs) {
                record_device_error(err, MSA_DEV_BAD_INDEX);
                continue;
            }
            rows += doc_chunk_off[doc + 1] - doc_chunk_off[doc];
        }
        if (rows > max_mem) {
            record_device_error(err, MSA_DEV_BAD_INDEX);
            rows = max_mem;
        }
        mem_len[q] = (int32_t)rows;
    }
}

struct StepLayout {
    size_t route_ws, scores, topk_ws, idx, mem_len, q_rot, mem_kv;   // all per layer except topk_ws
    size_t off_topk, off_layers, per_layer, total;
    size_t o_route, o_scores, o_idx, o_len, o_qrot, o_mem;           // offsets inside a layer's slot
};

msa_status layout(const msa_interleave_args* a, StepLayout* L) {
    const int T_act = a->L_prev + a->T_new;
    MSA_RETURN_IF(msa_route_workspace_size(a->n_q, T_act, a->H, a->d, a->dt, &L->route_ws));
    MSA_RETURN_IF(msa_topk_workspace_size(a->n_q, a->n_docs, a->k, &L->topk_ws));
    const size_t es = dtype_size(a->dt);
    L->scores = align_up((size_t)a->n_q * a->n_docs * sizeof(float), 256);
    L->idx = align_up((size_t)a->n_q * a->k * sizeof(int32_t), 256);
    L->mem_len = align_up((size_t)a->n_q * sizeof(int32_t), 256);
    L->q_rot = align_up((size_t)a->n_q * a->T_new * a->hq * a->d * es, 256);
    L->mem_kv = align_up((size_t)a->n_q * a->max_mem * 2 * a->hkv * a->d * es, 256);
    L->route_ws = align_up(L->route_ws, 256);
    L->off_topk = 0;
    L->off_layers = align_up(L->topk_ws, 256);
    L->o_route = 0;
    L->o_scores = L->o_route + L->route_ws;
    L->o_idx = L->o_scores + L->scores;
    L->o_len = L->o_idx + L->idx;
    L->o_qrot = L->o_len + L->mem_len;
    L->o_mem = L->o_qrot + L->q_rot;
    L->per_layer = L->o_mem + L->mem_kv;
    L->total = L->off_layers + L->per_layer * (size_t)a->n_layers;
    return MSA_OK;
}

msa_status validate(const msa_interleave_args* a, bool need_ws) {
    MSA_REQUIRE(a != nullptr, "msa_interleave_step: args is NULL");
    MSA_REQUIRE(dtype_ok(a->dt), "msa_interleave_step: bad dtype");
    MSA_REQUIRE(a->n_layers > 0 && a->layers, "msa_interleave_step: no layers");
    MSA_REQUIRE(a->n_q > 0 && a->H > 0 && a->d > 0 && a->hq > 0 && a->hkv > 0 && a->k > 0 && a->T_new > 0 &&
                    a->L_prev >= 0 && a->n_docs > 0 && a->n_chunks > 0 && a->max_mem > 0 && a->reserved_sms >= 0 &&
                    (a->fetch_mode == 0 || a->fetch_mode == 1),
                "msa_interleave_step: bad sizes");
    MSA_REQUIRE(a->L_prev + a->T_new <= a->L_max, "msa_interleave_step: local cache overflow (%d + %d > %d)", a->L_prev,
                a->T_new, a->L_max);
    MSA_REQUIRE(a->new_q_stride >= a->T_new, "msa_interleave_step: new_q_stride < T_new");
    MSA_REQUIRE(a->doc_chunk_off && a->doc_chunk_off_host && a->chunk_doc && a->rope_cos_sin && (a->ws || !need_ws),
                "msa_interleave_step: NULL pointer");
    MSA_REQUIRE(a->rope_max_pos >= (int64_t)a->k + a->L_prev + a->T_new,
                "msa_interleave_step: RoPE table too short for positions up to %d", a->k + a->L_prev + a->T_new);
    for (int l = 0; l < a->n_layers; ++l) {
        const msa_layer_args& y = a->layers[l];
        MSA_REQUIRE(y.kr_index && y.host_bank && y.qr && y.q_new && y.k_new && y.v_new && y.local_k && y.local_v &&
                        y.out && y.topk_idx_host,
                    "msa_interleave_step: layer %d has a NULL pointer", l);
        MSA_REQUIRE(aligned16(y.kr_index) && aligned16(y.qr) && aligned16(y.q_new) && aligned16(y.k_new) &&
                        aligned16(y.v_new) && aligned16(y.local_k) && aligned16(y.local_v) && aligned16(y.out),
                    "msa_interleave_step: layer %d has a misaligned pointer", l);
    }
    return MSA_OK;
}

msa_status wait_event(cudaEvent_t ev, std::chrono::steady_clock::time_point deadline) {
    for (;;) {
        const cudaError_t e = cudaEventQuery(ev);
        if (e == cudaSuccess) return MSA_OK;
        if (e != cudaErrorNotReady)
            return set_error(MSA_ERR_CUDA, "msa_interleave_step: event query failed: %s", cudaGetErrorString(e));
        if (std::chrono::steady_clock::now() > deadline)
            return set_error(MSA_ERR_TIMEOUT, "msa_interleave_step: host wait for a layer's selection timed out");
        std::this_thread::yield();
    }
}

// Events reused across calls: a per-thread, per-device pool (an event belongs to one device;
// re-recording an event does not disturb waits already enqueued on its earlier record).
constexpr int kMaxEvDev = 64;
thread_local std::vector<cudaEvent_t> t_events[kMaxEvDev];

msa_status event_pool(size_t n, cudaEvent_t** out) {
    int dev = 0;
    MSA_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxEvDev) return set_error(MSA_ERR_UNSUPPORTED, "msa_interleave_step: device %d", dev);
    std::vector<cudaEvent_t>& v = t_events[dev];
    while (v.size() < n) {
        cudaEvent_t e = nullptr;
        MSA_CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
        v.push_back(e);
    }
    *out = v.data();
    return MSA_OK;
}

// Library-owned auxiliary streams (select, attend), created once per device.
constexpr int kMaxDev = 64;
cudaStream_t g_aux[kMaxDev][2] = {{nullptr}};
std::mutex g_aux_mu;

msa_status aux_streams(cudaStream_t* sel, cudaStream_t* att) {
    int dev = 0;
    MSA_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDev) return set_error(MSA_ERR_UNSUPPORTED, "msa_interleave_step: device %d", dev);
    std::lock_guard<std::mutex> lk(g_aux_mu);
    for (int i = 0; i < 2; ++i)
        if (!g_aux[dev][i]) MSA_CUDA_TRY(cudaStreamCreateWithFlags(&g_aux[dev][i], cudaStreamNonBlocking));
    *sel = g_aux[dev][0];
    *att = g_aux[dev][1];
    return MSA_OK;
}

}  // namespace
}  // namespace msa

using namespace msa;

extern "C" {

msa_status msa_interleave_workspace_size(const msa_interleave_args* a, size_t* bytes) {
    MSA_REQUIRE(bytes, "msa_interleave_workspace_size: bytes is NULL");
    MSA_RETURN_IF(validate(a, false));
    StepLayout L;
    MSA_RETURN_IF(layout(a, &L));
    *bytes = L.total;
    return MSA_OK;
}

msa_status msa_interleave_step(const msa_interleave_args* a, void* compute, void* copy, int64_t host_wait_timeout_us) {
    MSA_RETURN_IF(validate(a, true));
    StepLayout Lo;
    MSA_RETURN_IF(layout(a, &Lo));
    if (a->ws_bytes < Lo.total)
        return set_error(MSA_ERR_WORKSPACE, "msa_interleave_step: workspace %zu < %zu", a->ws_bytes, Lo.total);
    MSA_REQUIRE(aligned16(a->ws), "msa_interleave_step: workspace must be 16-byte aligned");
    if (!rope_layout_ok(a->dt, a->d))
        return set_error(MSA_ERR_UNSUPPORTED, "msa_interleave_step: head_dim %d unsupported", a->d);

    cudaStream_t sR = static_cast<cudaStream_t>(compute);
    cudaStream_t sC = static_cast<cudaStream_t>(copy);
    cudaStream_t sS = nullptr, sA = nullptr;
    MSA_RETURN_IF(aux_streams(&sS, &sA));
    char* ws = static_cast<char*>(a->ws);
    const size_t es = dtype_size(a->dt);
    const int T_act = a->L_prev + a->T_new;
    const int L = a->n_layers;
    int* err = device_error_word();
    const float2* cs = reinterpret_cast<const float2*>(a->rope_cos_sin);
    RoutePlan plan;
    MSA_RETURN_IF(route_plan(a->dt, a->n_chunks, a->n_q, T_act, a->H, a->d, &plan));
    const int grid_cap = a->reserved_sms > 0 ? std::max(1, sm_count() - a->reserved_sms) : 0;

    // events: P_l, R_l, E_l, G_l, fork, join x2
    cudaEvent_t* ev = nullptr;
    MSA_RETURN_IF(event_pool(4 * (size_t)L + 3, &ev));
    cudaEvent_t ev_fork = ev[4 * L], ev_join_s = ev[4 * L + 1], ev_join_a = ev[4 * L + 2];
    auto P = [&](int l) { return ev[l]; };
    auto R = [&](int l) { return ev[L + l]; };
    auto E = [&](int l) { return ev[2 * L + l]; };
    auto G = [&](int l) { return ev[3 * L + l]; };
    auto slot = [&](int l, size_t off) { return ws + Lo.off_layers + Lo.per_layer * (size_t)l + off; };

    MSA_CUDA_TRY(cudaEventRecord(ev_fork, sR));
    MSA_CUDA_TRY(cudaStreamWaitEvent(sS, ev_fork, 0));
    MSA_CUDA_TRY(cudaStreamWaitEvent(sA, ev_fork, 0));

    // ---- per layer, in enqueue order: prepass on A, router on R, selection on S (the first router
    // is on the GPU after two launches of host time; the rest enqueue while it runs)
    for (int l = 0; l < L; ++l) {
        const msa_layer_args& y = a->layers[l];
        float* scores = reinterpret_cast<float*>(slot(l, Lo.o_scores));
        MSA_RETURN_IF(route_prepare(plan, y.qr, slot(l, Lo.o_route), scores, a->n_docs, nullptr, a->n_chunks, sA));
        MSA_CUDA_TRY(cudaEventRecord(P(l), sA));
        MSA_CUDA_TRY(cudaStreamWaitEvent(sR, P(l), 0));
        if (a->route_events) MSA_CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(a->route_events[2 * l]), sR));
        MSA_RETURN_IF(route_launch(plan, y.kr_index, a->n_chunks, a->chunk_doc, a->n_docs, slot(l, Lo.o_route), scores,
                                   nullptr, grid_cap, sR));
        if (a->route_events) MSA_CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(a->route_events[2 * l + 1]), sR));
        MSA_CUDA_TRY(cudaEventRecord(R(l), sR));

        MSA_CUDA_TRY(cudaStreamWaitEvent(sS, R(l), 0));
        int32_t* idx = reinterpret_cast<int32_t*>(slot(l, Lo.o_idx));
        MSA_RETURN_IF(msa_topk_docs(scores, a->n_q, a->n_docs, a->k, idx, nullptr, ws + Lo.off_topk, Lo.topk_ws, sS));
        if (a->fetch_mode == 1) {
            // fetch right behind the selection on the device; the index copy to the host is output only
            MSA_RETURN_IF(gather_device(y.host_bank, a->dt, a->n_chunks, a->doc_chunk_off, a->n_docs, idx, a->n_q, a->k,
                                        a->hkv, a->d, a->max_mem, slot(l, Lo.o_mem),
                                        reinterpret_cast<int32_t*>(slot(l, Lo.o_len)), sS));
            MSA_CUDA_TRY(cudaEventRecord(E(l), sS));
            MSA_CUDA_TRY(cudaMemcpyAsync(y.topk_idx_host, idx, (size_t)a->n_q * a->k * sizeof(int32_t),
                                         cudaMemcpyDeviceToHost, sS));
        } else {
            MSA_CUDA_TRY(cudaMemcpyAsync(y.topk_idx_host, idx, (size_t)a->n_q * a->k * sizeof(int32_t),
                                         cudaMemcpyDeviceToHost, sS));
            mem_len_kernel<<<(a->n_q + 127) / 128, 128, 0, sS>>>(idx, a->n_q, a->k, a->doc_chunk_off, a->n_docs,
                                                                a->max_mem, reinterpret_cast<int32_t*>(slot(l, Lo.o_len)),
                                                                err);
            MSA_LAUNCH_CHECK();
            MSA_CUDA_TRY(cudaEventRecord(E(l), sS));
        }
    }

    // ---- A: appends and query rotations of every layer, one launch per kMaxAppendLayers layers
    for (int l0 = 0; l0 < L; l0 += kMaxAppendLayers) {
        AppendArgs ap{};
        ap.n_layers = std::min(kMaxAppendLayers, L - l0);
        for (int i = 0; i < ap.n_layers; ++i) {
            const msa_layer_args& y = a->layers[l0 + i];
            ap.layer[i] = AppendLayer{y.k_new, y.v_new, y.q_new, y.local_k, y.local_v, slot(l0 + i, Lo.o_qrot)};
        }
        ap.n_q = a->n_q; ap.T_new = a->T_new; ap.new_q_stride = a->new_q_stride; ap.L_max = a->L_max;
        ap.L_prev = a->L_prev; ap.hkv = a->hkv; ap.hq = a->hq; ap.d = a->d;
        ap.pos_offset = (int64_t)a->k + a->L_prev; ap.cs = cs; ap.max_pos = a->rope_max_pos; ap.err = err;
        MSA_RETURN_IF(launch_append(ap, a->dt, sA));
    }

    // ---- host: per layer, wait for its selection, fetch on C, attend on A
    const auto deadline = std::chrono::steady_clock::now() + std::chrono::microseconds(host_wait_timeout_us);
    std::vector<int32_t> mem_len_host((size_t)a->n_q);
    for (int l = 0; l < L; ++l) {
        const msa_layer_args& y = a->layers[l];
        if (a->fetch_mode == 1) {
            MSA_CUDA_TRY(cudaStreamWaitEvent(sA, E(l), 0));
        } else {
            MSA_RETURN_IF(wait_event(E(l), deadline));
            MSA_RETURN_IF(msa_gather_kv(y.host_bank, a->dt, a->n_chunks, a->doc_chunk_off_host, a->n_docs,
                                        y.topk_idx_host, a->n_q, a->k, a->hkv, a->d, a->max_mem, slot(l, Lo.o_mem),
                                        mem_len_host.data(), sC));
            MSA_CUDA_TRY(cudaEventRecord(G(l), sC));
            MSA_CUDA_TRY(cudaStreamWaitEvent(sA, G(l), 0));
        }
        MSA_RETURN_IF(msa_sparse_attn(slot(l, Lo.o_qrot), slot(l, Lo.o_mem),
                                      reinterpret_cast<const int32_t*>(slot(l, Lo.o_len)), a->max_mem, y.local_k,
                                      y.local_v, a->L_max, T_act, a->L_prev, a->n_q, a->T_new, a->hq, a->hkv, a->d,
                                      a->scale, y.out, a->dt, sA));
    }
    MSA_CUDA_TRY(cudaEventRecord(ev_join_s, sS));
    MSA_CUDA_TRY(cudaEventRecord(ev_join_a, sA));
    MSA_CUDA_TRY(cudaStreamWaitEvent(sR, ev_join_s, 0));
    MSA_CUDA_TRY(cudaStreamWaitEvent(sR, ev_join_a, 0));
    return MSA_OK;
}

struct msa_interleave_graph {
    cudaGraph_t graph;
    cudaGraphExec_t exec;
    int device;
};

msa_status msa_interleave_graph_create(const msa_interleave_args* a, void* stream, msa_interleave_graph** out) {
    MSA_REQUIRE(a && out, "msa_interleave_graph_create: NULL argument");
    *out = nullptr;
    MSA_REQUIRE(a->fetch_mode == 1, "msa_interleave_graph_create: fetch_mode must be 1 (fetch_mode 0 waits on the host)");
    MSA_REQUIRE(a->route_events == nullptr, "msa_interleave_graph_create: route_events must be NULL");
    MSA_REQUIRE(stream != nullptr && stream != static_cast<void*>(cudaStreamLegacy) &&
                    stream != static_cast<void*>(cudaStreamPerThread),
                "msa_interleave_graph_create: needs a created stream, not a default stream");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int dev = 0;
    MSA_CUDA_TRY(cudaGetDevice(&dev));
    // one eager pass: every one-time set-up (library streams, events, kernel attributes, cached
    // plans) happens outside the capture
    MSA_RETURN_IF(msa_interleave_step(a, stream, stream, 0));
    MSA_CUDA_TRY(cudaStreamSynchronize(s));
    MSA_CUDA_TRY(cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal));
    const msa_status st = msa_interleave_step(a, stream, stream, 0);
    cudaGraph_t graph = nullptr;
    const cudaError_t e = cudaStreamEndCapture(s, &graph);
    if (st != MSA_OK || e != cudaSuccess) {
        if (graph) cudaGraphDestroy(graph);
        if (st != MSA_OK) return st;
        return set_error(MSA_ERR_CUDA, "msa_interleave_graph_create: capture failed: %s", cudaGetErrorString(e));
    }
    cudaGraphExec_t exec = nullptr;
    const cudaError_t ie = cudaGraphInstantiate(&exec, graph, 0);
    if (ie != cudaSuccess) {
        cudaGraphDestroy(graph);
        return set_error(MSA_ERR_CUDA, "msa_interleave_graph_create: instantiate failed: %s", cudaGetErrorString(ie));
    }
    msa_interleave_graph* g = new (std::nothrow) msa_interleave_graph{graph, exec, dev};
    if (!g) {
        cudaGraphExecDestroy(exec);
        cudaGraphDestroy(graph);
        return set_error(MSA_ERR_CUDA, "msa_interleave_graph_create: out of host memory");
    }
    *out = g;
    return MSA_OK;
}

msa_status msa_interleave_graph_launch(msa_interleave_graph* g, void* stream) {
    MSA_REQUIRE(g != nullptr, "msa_interleave_graph_launch: graph is NULL");
    int dev = 0;
    MSA_CUDA_TRY(cudaGetDevice(&dev));
    MSA_REQUIRE(dev == g->device, "msa_interleave_graph_launch: graph of device %d launched on device %d", g->device,
                dev);
    MSA_CUDA_TRY(cudaGraphLaunch(g->exec, static_cast<cudaStream_t>(stream)));
    return MSA_OK;
}

msa_status msa_interleave_graph_destroy(msa_interleave_graph* g) {
    if (!g) return MSA_OK;
    const cudaError_t a = cudaGraphExecDestroy(g->exec);
    const cudaError_t b = cudaGraphDestroy(g->graph);
    delete g;
    if (a != cudaSuccess || b != cudaSuccess)
        return set_error(MSA_ERR_CUDA, "msa_interleave_graph_destroy: %s",
                         cudaGetErrorString(a != cudaSuccess ? a : b));
    return MSA_OK;
}

}  // extern "C"
