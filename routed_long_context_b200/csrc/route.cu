// Router scoring: per-head query normalisation, the fp32 CUDA-core scorer and the dispatcher.
//
// The mean over heads of the cosines, mean_h <q_h/|q_h|, k_h/|k_h|>, equals one dot product of
// concat_h(q_h / (|q_h| H)) with concat_h(k_h / |k_h|). The index already stores the unit
// vectors k_h/|k_h| (msa_pool_chunks with normalize_router), so the prepass below turns every
// query token into q_hat = concat_h(q_h / (|q_h| H)) and the scorer is a plain contraction whose
// epilogue takes the max over each query's tokens and over each document's chunks.
#include <atomic>

#include "common.cuh"
#include "kernels.cuh"

namespace msa {
namespace {

std::atomic<int> g_route_impl{0};   // 0 auto, 1 CUDA cores, 2 tensor cores, 3 tensor cores + resident qhat

// q_hat rows [n_pad][K] of TQ; rows >= N are zero. Also fills doc_scores/chunk_scores with -inf.
template <typename T, typename TQ>
__global__ void __launch_bounds__(128) route_prep_kernel(const T* __restrict__ qr, int N, int n_pad, int H, int d,
                                                         TQ* __restrict__ qhat, float* doc_scores, int64_t n_doc_fill,
                                                         float* chunk_scores, int64_t n_chunk_fill, int* tile_counter) {
    if (blockIdx.x == 0 && threadIdx.x == 0) *tile_counter = 0;
    constexpr int VEC = 16 / sizeof(T);
    const int K = H * d;
    const int lanes_per_head = d / VEC;
    const float inv_h = 1.0f / (float)H;
    for (int r = blockIdx.x; r < n_pad; r += gridDim.x) {
        for (int e0 = threadIdx.x * VEC; e0 - (int)threadIdx.x * VEC < K; e0 += blockDim.x * VEC) {
            const bool active = e0 < K;
            float x[VEC];
            if (active && r < N) {
                load16_f32<T>(qr + (int64_t)r * K + e0, x);
            } else {
#pragma unroll
                for (int j = 0; j < VEC; ++j) x[j] = 0.f;
            }
            float ss = 0.f;
#pragma unroll
            for (int j = 0; j < VEC; ++j) ss = fmaf(x[j], x[j], ss);
            for (int m = lanes_per_head / 2; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
            const float inv = ss > 0.f ? (1.0f / sqrtf(ss)) * inv_h : 0.f;
#pragma unroll
            for (int j = 0; j < VEC; ++j) x[j] *= inv;
            if (active) store_f32<TQ, VEC>(qhat + (int64_t)r * K + e0, x);
        }
    }
    const float ninf = -__int_as_float(0x7f800000);
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_doc_fill; i += stride) doc_scores[i] = ninf;
    if (chunk_scores)
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_chunk_fill; i += stride)
            chunk_scores[i] = ninf;
}

// CUDA-core scorer: one warp per chunk; each lane holds KPL = K/32 index elements in registers.
// q_hat (fp32) is staged in shared memory NT tokens at a time.
constexpr int kSimtWarps = 8;
constexpr int kSimtNT = 16;

template <typename T, int KPL>
__global__ void __launch_bounds__(kSimtWarps * 32) route_simt_kernel(const T* __restrict__ index, int64_t n_chunks,
                                                                     const float* __restrict__ qhat, int N, int T_tok,
                                                                     const int32_t* __restrict__ chunk_doc,
                                                                     int64_t n_docs, float* doc_scores,
                                                                     float* chunk_scores, int* err) {
    constexpr int VEC = 16 / sizeof(T);
    constexpr int K = KPL * 32;
    constexpr int GROUPS = KPL / VEC;          // 16-byte groups per lane
    extern __shared__ float q_s[];             // [kSimtNT][K]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    for (int n0 = 0; n0 < N; n0 += kSimtNT) {
        const int nt = min(kSimtNT, N - n0);
        __syncthreads();
        for (int i = threadIdx.x * 4; i < nt * K; i += blockDim.x * 4)
            *reinterpret_cast<float4*>(q_s + i) = *reinterpret_cast<const float4*>(qhat + (int64_t)n0 * K + i);
        __syncthreads();
        for (int64_t c = (int64_t)blockIdx.x * kSimtWarps + warp; c < n_chunks; c += (int64_t)gridDim.x * kSimtWarps) {
            float kv[KPL];
#pragma unroll
            for (int g = 0; g < GROUPS; ++g)
                load16_f32<T>(index + c * K + lane * VEC + g * 32 * VEC, kv + g * VEC);
            const int doc = chunk_doc[c];
            if (doc < 0 || doc >= n_docs) {
                if (lane == 0) record_device_error(err, MSA_DEV_BAD_INDEX);
                continue;
            }
            int cur_q = n0 / T_tok;
            float cur_max = -__int_as_float(0x7f800000);
            for (int n = 0; n < nt; ++n) {
                const float* qs = q_s + n * K;
                float acc = 0.f;
#pragma unroll
                for (int g = 0; g < GROUPS; ++g) {
#pragma unroll
                    for (int v = 0; v < VEC; v += 4) {
                        const float4 q4 = *reinterpret_cast<const float4*>(qs + lane * VEC + g * 32 * VEC + v);
                        acc = fmaf(kv[g * VEC + v + 0], q4.x, acc);
                        acc = fmaf(kv[g * VEC + v + 1], q4.y, acc);
                        acc = fmaf(kv[g * VEC + v + 2], q4.z, acc);
                        acc = fmaf(kv[g * VEC + v + 3], q4.w, acc);
                    }
                }
#pragma unroll
                for (int m = 16; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
                const int q = (n0 + n) / T_tok;
                if (q != cur_q) {
                    if (lane == 0) {
                        atomic_max_f32(doc_scores + (int64_t)cur_q * n_docs + doc, cur_max);
                        if (chunk_scores) atomic_max_f32(chunk_scores + (int64_t)cur_q * n_chunks + c, cur_max);
                    }
                    cur_q = q;
                    cur_max = -__int_as_float(0x7f800000);
                }
                cur_max = fmaxf(cur_max, acc);
            }
            if (lane == 0) {
                atomic_max_f32(doc_scores + (int64_t)cur_q * n_docs + doc, cur_max);
                if (chunk_scores) atomic_max_f32(chunk_scores + (int64_t)cur_q * n_chunks + c, cur_max);
            }
        }
    }
}

template <typename T>
msa_status launch_simt(const void* index, int64_t n_chunks, int K, const float* qhat, int N, int T_tok,
                       const int32_t* chunk_doc, int64_t n_docs, float* doc_scores, float* chunk_scores, int* err,
                       cudaStream_t s) {
    const size_t smem = (size_t)kSimtNT * K * sizeof(float);
    int64_t blocks = (n_chunks + kSimtWarps - 1) / kSimtWarps;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (blocks > cap) blocks = cap;
    const T* idx = static_cast<const T*>(index);
#define MSA_SIMT_CASE(KPL)                                                                                    \
    case KPL: {                                                                                               \
        auto kern = route_simt_kernel<T, KPL>;                                                                \
        MSA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));     \
        kern<<<(unsigned)blocks, kSimtWarps * 32, smem, s>>>(idx, n_chunks, qhat, N, T_tok, chunk_doc, n_docs, \
                                                             doc_scores, chunk_scores, err);                  \
        break;                                                                                                \
    }
    switch (K / 32) {
        MSA_SIMT_CASE(8)
        MSA_SIMT_CASE(16)
        MSA_SIMT_CASE(32)
        MSA_SIMT_CASE(64)
        default:
            return set_error(MSA_ERR_UNSUPPORTED, "route (CUDA cores): H*d = %d unsupported", K);
    }
#undef MSA_SIMT_CASE
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

bool simt_supported(msa_dtype dt, int K) {
    const int VEC = dt == MSA_BF16 ? 8 : 4;
    const int kpl = K / 32;
    return K % (32 * VEC) == 0 && (kpl == 8 || kpl == 16 || kpl == 32 || kpl == 64);
}

constexpr size_t kCounterBytes = 256;   // the tile counter sits in the first 256 bytes of the workspace

size_t qhat_bytes(int N, int K) {
    const int rows = (N + 255) / 256 * 256;
    return kCounterBytes + align_up((size_t)rows * K * sizeof(float), 256);
}

}  // namespace

int route_impl_setting() { return g_route_impl.load(); }

msa_status route_plan(msa_dtype dt, int64_t n_chunks, int n_q, int T, int H, int d, RoutePlan* plan) {
    MSA_REQUIRE(dtype_ok(dt), "msa_route_scores: bad dtype %d", dt);
    MSA_REQUIRE(n_q > 0 && T > 0 && H > 0 && d > 0, "msa_route_scores: bad sizes");
    MSA_REQUIRE((int64_t)n_q * T <= (1 << 20), "msa_route_scores: too many query tokens");
    if (!rope_layout_ok(dt, d))
        return set_error(MSA_ERR_UNSUPPORTED, "msa_route_scores: head_dim %d unsupported for this dtype", d);
    RoutePlan p{};
    p.dt = dt; p.n_q = n_q; p.T = T; p.H = H; p.d = d; p.K = H * d; p.N = n_q * T;
    const int impl = g_route_impl.load();
    p.resident = impl == 3;
    const int tc_rows = dt == MSA_BF16 ? route_tc_pad_rows(p.N, p.K, p.resident) : 0;
    p.use_tc = dt == MSA_BF16 && impl != 1 && tc_rows > 0 && n_chunks > 0;
    if (impl >= 2 && !p.use_tc)
        return set_error(MSA_ERR_UNSUPPORTED, "msa_route_scores: tensor-core path unavailable for this shape");
    if (!p.use_tc && !simt_supported(dt, p.K))
        return set_error(MSA_ERR_UNSUPPORTED, "msa_route_scores: H*d = %d unsupported", p.K);
    p.n_pad = p.use_tc ? tc_rows : p.N;
    *plan = p;
    return MSA_OK;
}

msa_status route_prepare(const RoutePlan& p, const void* qr, void* ws, float* doc_scores, int64_t n_docs,
                         float* chunk_scores, int64_t n_chunks, cudaStream_t s) {
    int* counter = static_cast<int*>(ws);
    void* qhat = static_cast<char*>(ws) + kCounterBytes;
    const int64_t fill = (int64_t)p.n_q * n_docs;
    const int64_t cfill = chunk_scores ? (int64_t)p.n_q * n_chunks : 0;
    int64_t pblocks = p.n_pad;
    const int64_t want_fill = (fill + cfill + 127) / 128;
    if (pblocks < want_fill) pblocks = want_fill;
    const int64_t cap = (int64_t)sm_count() * 16;
    if (pblocks > cap) pblocks = cap;
    if (pblocks < 1) pblocks = 1;
    if (p.use_tc) {
        route_prep_kernel<__nv_bfloat16, __nv_bfloat16><<<(unsigned)pblocks, 128, 0, s>>>(
            static_cast<const __nv_bfloat16*>(qr), p.N, p.n_pad, p.H, p.d, static_cast<__nv_bfloat16*>(qhat),
            doc_scores, fill, chunk_scores, cfill, counter);
    } else if (p.dt == MSA_BF16) {
        route_prep_kernel<__nv_bfloat16, float><<<(unsigned)pblocks, 128, 0, s>>>(
            static_cast<const __nv_bfloat16*>(qr), p.N, p.n_pad, p.H, p.d, static_cast<float*>(qhat), doc_scores,
            fill, chunk_scores, cfill, counter);
    } else {
        route_prep_kernel<float, float><<<(unsigned)pblocks, 128, 0, s>>>(
            static_cast<const float*>(qr), p.N, p.n_pad, p.H, p.d, static_cast<float*>(qhat), doc_scores, fill,
            chunk_scores, cfill, counter);
    }
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

msa_status route_launch(const RoutePlan& p, const void* kr_index, int64_t n_chunks, const int32_t* chunk_doc,
                        int64_t n_docs, void* ws, float* doc_scores, float* chunk_scores, int grid_cap,
                        cudaStream_t s) {
    if (n_chunks == 0) return MSA_OK;
    int* err = device_error_word();
    const void* qhat = static_cast<char*>(ws) + kCounterBytes;
    if (p.use_tc) {
        RouteTcArgs a{};
        a.index = kr_index; a.qhat = qhat; a.n_chunks = n_chunks; a.K = p.K; a.N = p.N; a.n_pad = p.n_pad;
        a.T = p.T; a.chunk_doc = chunk_doc; a.n_docs = n_docs; a.doc_scores = doc_scores;
        a.chunk_scores = chunk_scores; a.err = err; a.grid_cap = grid_cap; a.tile_counter = static_cast<int*>(ws);
        a.resident = p.resident;
        return launch_route_tc(a, s);
    }
    if (p.dt == MSA_BF16)
        return launch_simt<__nv_bfloat16>(kr_index, n_chunks, p.K, static_cast<const float*>(qhat), p.N, p.T,
                                          chunk_doc, n_docs, doc_scores, chunk_scores, err, s);
    return launch_simt<float>(kr_index, n_chunks, p.K, static_cast<const float*>(qhat), p.N, p.T, chunk_doc, n_docs,
                              doc_scores, chunk_scores, err, s);
}

}  // namespace msa

using namespace msa;

extern "C" {

msa_status msa_route_set_impl(int impl) {
    MSA_REQUIRE(impl >= 0 && impl <= 3, "msa_route_set_impl: impl must be 0, 1, 2 or 3");
    g_route_impl.store(impl);
    return MSA_OK;
}

msa_status msa_route_inject_stall(int on) {
    MSA_REQUIRE(on == 0 || on == 1, "msa_route_inject_stall: on must be 0 or 1");
    route_tc_inject_stall(on);
    return MSA_OK;
}

msa_status msa_route_set_max_stages(int n) {
    MSA_REQUIRE(n >= 0 && n <= 12, "msa_route_set_max_stages: n must be in [0, 12]");
    route_tc_set_max_stages(n);
    return MSA_OK;
}

msa_status msa_route_workspace_size(int n_q, int T, int H, int d, msa_dtype dt, size_t* bytes) {
    MSA_REQUIRE(bytes != nullptr, "msa_route_workspace_size: bytes is NULL");
    MSA_REQUIRE(n_q > 0 && T > 0 && H > 0 && d > 0 && dtype_ok(dt), "msa_route_workspace_size: bad sizes");
    *bytes = qhat_bytes(n_q * T, H * d);
    return MSA_OK;
}

msa_status msa_route_scores(const void* kr_index, msa_dtype dt, int64_t n_chunks, const int32_t* chunk_doc,
                            int64_t n_docs, const void* qr, int n_q, int T, int H, int d, float* doc_scores,
                            float* chunk_scores, void* ws, size_t ws_bytes, void* stream) {
    MSA_REQUIRE(n_chunks >= 0 && n_docs > 0, "msa_route_scores: bad sizes");
    MSA_REQUIRE(qr && doc_scores && ws, "msa_route_scores: NULL pointer");
    MSA_REQUIRE(n_chunks == 0 || (kr_index && chunk_doc), "msa_route_scores: NULL index");
    MSA_REQUIRE(aligned16(qr) && aligned16(ws) && (n_chunks == 0 || aligned16(kr_index)),
                "msa_route_scores: pointers must be 16-byte aligned");
    RoutePlan plan;
    MSA_RETURN_IF(route_plan(dt, n_chunks, n_q, T, H, d, &plan));
    size_t need = 0;
    MSA_RETURN_IF(msa_route_workspace_size(n_q, T, H, d, dt, &need));
    if (ws_bytes < need) return set_error(MSA_ERR_WORKSPACE, "msa_route_scores: workspace %zu < %zu", ws_bytes, need);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    MSA_RETURN_IF(route_prepare(plan, qr, ws, doc_scores, n_docs, chunk_scores, n_chunks, s));
    if (n_chunks == 0) return MSA_OK;
    return route_launch(plan, kr_index, n_chunks, chunk_doc, n_docs, ws, doc_scores, chunk_scores, 0, s);
}

}  // extern "C"
