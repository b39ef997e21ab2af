// One Memory Interleave round over all routed layers: append -> route -> top-k -> fetch -> attend.
//
// Stream schedule (compute = S0, copy = S1):
//   S0: for every layer: rotate+append the new tokens' K/V, rotate their queries, route, top-k,
//       copy the selected indices to pinned host memory, derive per-query memory lengths, record E_l.
//   host: for every layer: wait for E_l (bounded poll), enqueue the layer's document fetches on S1,
//       record G_l; S0 waits for G_l and runs the layer's attention.
// Every layer's routing is enqueued before the host blocks on the first selection, so the host-link
// fetches of layer l overlap the routing of layers l+1.. on the GPU.
#include <chrono>
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
    size_t route_ws, scores, topk_ws, idx, mem_len, q_rot, mem_kv;   // per-layer sizes for the last four
    size_t off_route, off_scores, off_topk, off_layers, per_layer, total;
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
    L->off_route = 0;
    L->off_scores = align_up(L->route_ws, 256);
    L->off_topk = L->off_scores + L->scores;
    L->off_layers = L->off_topk + align_up(L->topk_ws, 256);
    L->per_layer = L->idx + L->mem_len + L->q_rot + L->mem_kv;
    L->total = L->off_layers + L->per_layer * (size_t)a->n_layers;
    return MSA_OK;
}

msa_status validate(const msa_interleave_args* a, bool need_ws) {
    MSA_REQUIRE(a != nullptr, "msa_interleave_step: args is NULL");
    MSA_REQUIRE(dtype_ok(a->dt), "msa_interleave_step: bad dtype");
    MSA_REQUIRE(a->n_layers > 0 && a->layers, "msa_interleave_step: no layers");
    MSA_REQUIRE(a->n_q > 0 && a->H > 0 && a->d > 0 && a->hq > 0 && a->hkv > 0 && a->k > 0 && a->T_new > 0 &&
                    a->L_prev >= 0 && a->n_docs > 0 && a->n_chunks > 0 && a->max_mem > 0,
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

struct Events {
    std::vector<cudaEvent_t> ev;
    ~Events() {
        for (cudaEvent_t e : ev) cudaEventDestroy(e);
    }
};

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

    cudaStream_t s0 = static_cast<cudaStream_t>(compute);
    cudaStream_t s1 = static_cast<cudaStream_t>(copy);
    char* ws = static_cast<char*>(a->ws);
    const size_t es = dtype_size(a->dt);
    const int T_act = a->L_prev + a->T_new;
    int* err = device_error_word();
    const float2* cs = reinterpret_cast<const float2*>(a->rope_cos_sin);

    Events evs;
    evs.ev.resize(2 * (size_t)a->n_layers, nullptr);
    for (auto& e : evs.ev) MSA_CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));

    auto layer_ws = [&](int l, size_t part) { return ws + Lo.off_layers + Lo.per_layer * (size_t)l + part; };
    const size_t o_idx = 0, o_len = Lo.idx, o_qrot = Lo.idx + Lo.mem_len, o_mem = o_qrot + Lo.q_rot;

    // ---- phase 1: append, rotate, route and select for every layer (all on S0)
    for (int l = 0; l < a->n_layers; ++l) {
        const msa_layer_args& y = a->layers[l];
        RopeRowsArgs r{};
        r.heads = a->hkv; r.d = a->d; r.n_rows = (int64_t)a->n_q * a->T_new; r.uniform_len = a->T_new;
        r.in = y.k_new; r.out = y.local_k; r.in_stride = a->new_q_stride; r.out_stride = a->L_max; r.out_off = a->L_prev;
        r.pos_offset = (int64_t)a->k + a->L_prev; r.cs = cs; r.max_pos = a->rope_max_pos; r.err = err;
        MSA_RETURN_IF(launch_rope_rows(r, a->dt, s0));
        const size_t vrow = (size_t)a->hkv * a->d * es;
        MSA_CUDA_TRY(cudaMemcpy2DAsync(static_cast<char*>(y.local_v) + (size_t)a->L_prev * vrow, (size_t)a->L_max * vrow,
                                       y.v_new, (size_t)a->new_q_stride * vrow, (size_t)a->T_new * vrow, a->n_q,
                                       cudaMemcpyDeviceToDevice, s0));
        RopeRowsArgs rq = r;
        rq.heads = a->hq; rq.in = y.q_new; rq.out = layer_ws(l, o_qrot); rq.out_stride = a->T_new; rq.out_off = 0;
        MSA_RETURN_IF(launch_rope_rows(rq, a->dt, s0));

        float* scores = reinterpret_cast<float*>(ws + Lo.off_scores);
        MSA_RETURN_IF(msa_route_scores(y.kr_index, a->dt, a->n_chunks, a->chunk_doc, a->n_docs, y.qr, a->n_q, T_act, a->H,
                                       a->d, scores, nullptr, ws + Lo.off_route, Lo.route_ws, s0));
        int32_t* idx = reinterpret_cast<int32_t*>(layer_ws(l, o_idx));
        MSA_RETURN_IF(msa_topk_docs(scores, a->n_q, a->n_docs, a->k, idx, nullptr, ws + Lo.off_topk, Lo.topk_ws, s0));
        MSA_CUDA_TRY(cudaMemcpyAsync(y.topk_idx_host, idx, (size_t)a->n_q * a->k * sizeof(int32_t),
                                     cudaMemcpyDeviceToHost, s0));
        mem_len_kernel<<<(a->n_q + 127) / 128, 128, 0, s0>>>(idx, a->n_q, a->k, a->doc_chunk_off, a->n_docs, a->max_mem,
                                                            reinterpret_cast<int32_t*>(layer_ws(l, o_len)), err);
        MSA_LAUNCH_CHECK();
        MSA_CUDA_TRY(cudaEventRecord(evs.ev[2 * l], s0));
    }

    // ---- phase 2: per layer, wait for its selection, fetch on S1, attend on S0
    const auto deadline = std::chrono::steady_clock::now() + std::chrono::microseconds(host_wait_timeout_us);
    std::vector<int32_t> mem_len_host((size_t)a->n_q);
    for (int l = 0; l < a->n_layers; ++l) {
        const msa_layer_args& y = a->layers[l];
        MSA_RETURN_IF(wait_event(evs.ev[2 * l], deadline));
        MSA_RETURN_IF(msa_gather_kv(y.host_bank, a->dt, a->n_chunks, a->doc_chunk_off_host, a->n_docs, y.topk_idx_host,
                                    a->n_q, a->k, a->hkv, a->d, a->max_mem, layer_ws(l, o_mem), mem_len_host.data(), s1));
        MSA_CUDA_TRY(cudaEventRecord(evs.ev[2 * l + 1], s1));
        MSA_CUDA_TRY(cudaStreamWaitEvent(s0, evs.ev[2 * l + 1], 0));
        MSA_RETURN_IF(msa_sparse_attn(layer_ws(l, o_qrot), layer_ws(l, o_mem),
                                      reinterpret_cast<const int32_t*>(layer_ws(l, o_len)), a->max_mem, y.local_k,
                                      y.local_v, a->L_max, T_act, a->L_prev, a->n_q, a->T_new, a->hq, a->hkv, a->d,
                                      a->scale, y.out, a->dt, s0));
    }
    return MSA_OK;
}

}  // extern "C"
