// Top-k document selection over doc_scores [n_q][n_docs]. k <= 32 uses warp-distributed lists
// (topk_warp_kernel below); larger k uses per-thread lists merged by tournaments.
//
// Order: descending score, ties to the lower document index (a strict total order, so the
// result is unique). One launch: P blocks per query each keep a per-thread sorted list of the
// KT >= k best candidates of a strided slice, merge them per warp and per block by a tournament
// (warp arg-max over list heads, the winner's lane pops its head), and write their KT best to
// the workspace. The last block of a query to finish (an atomic ticket, no spinning) merges the
// P lists and writes the first k. Reading the partial lists goes through L2 (__ldcg).
#include <algorithm>
#include <climits>
#include <mutex>

#include "common.cuh"
#include "tc.cuh"

namespace msa {
namespace {

constexpr int kTopkThreads = 256;
constexpr int kTopkWarps = kTopkThreads / 32;

__device__ __forceinline__ bool better(float a, int ia, float b, int ib) { return a > b || (a == b && ia < ib); }

template <int KT>
struct List {
    float s[KT];
    int i[KT];
    __device__ __forceinline__ void clear() {
#pragma unroll
        for (int j = 0; j < KT; ++j) s[j] = -__int_as_float(0x7f800000), i[j] = INT_MAX;
    }
    // Inserts (v, id) if it beats the current last entry; keeps the list sorted best-first.
    __device__ __forceinline__ bool insert(float v, int id) {
        if (!better(v, id, s[KT - 1], i[KT - 1])) return false;
        s[KT - 1] = v;
        i[KT - 1] = id;
#pragma unroll
        for (int j = KT - 1; j > 0; --j) {
            if (better(s[j], i[j], s[j - 1], i[j - 1])) {
                const float ts = s[j]; s[j] = s[j - 1]; s[j - 1] = ts;
                const int ti = i[j]; i[j] = i[j - 1]; i[j - 1] = ti;
            }
        }
        return true;
    }
    __device__ __forceinline__ void pop() {
#pragma unroll
        for (int j = 0; j < KT - 1; ++j) s[j] = s[j + 1], i[j] = i[j + 1];
        s[KT - 1] = -__int_as_float(0x7f800000);
        i[KT - 1] = INT_MAX;
    }
};

// The warp's KT best entries (over all lanes' sorted lists), written best-first by lane 0.
template <int KT>
__device__ __forceinline__ void warp_tournament(List<KT>& L, float* out_s, int* out_i) {
    const int lane = threadIdx.x & 31;
    for (int r = 0; r < KT; ++r) {
        float bs = L.s[0];
        int bi = L.i[0];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            const float os = __shfl_xor_sync(0xffffffffu, bs, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (better(os, oi, bs, bi)) bs = os, bi = oi;
        }
        if (lane == 0) out_s[r] = bs, out_i[r] = bi;
        if (L.i[0] == bi && L.s[0] == bs) L.pop();
    }
}

// Block-wide merge of every thread's list; the result lands in res_s/res_i [KT] (shared).
template <int KT>
__device__ void block_merge(List<KT>& L, float (*ws)[KT], int (*wi)[KT], float* res_s, int* res_i) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    warp_tournament<KT>(L, ws[warp], wi[warp]);
    __syncthreads();
    if (warp == 0) {
        L.clear();
        if (lane < kTopkWarps) {
#pragma unroll
            for (int j = 0; j < KT; ++j) L.s[j] = ws[lane][j], L.i[j] = wi[lane][j];
        }
        warp_tournament<KT>(L, res_s, res_i);
    }
    __syncthreads();
}

template <int KT>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float* __restrict__ scores, int64_t n_docs, int k,
                                                            int P, float* part_s, int* part_i, int* counters,
                                                            int32_t* out_idx, float* out_score) {
    __shared__ float ws[kTopkWarps][KT];
    __shared__ int wi[kTopkWarps][KT];
    __shared__ float res_s[KT];
    __shared__ int res_i[KT];
    __shared__ int is_last;
    const int q = blockIdx.y;
    const float* row = scores + (int64_t)q * n_docs;

    List<KT> L;
    L.clear();
    // batches of independent loads first, then the inserts (no load waits behind an insert)
    const int64_t stride = (int64_t)P * kTopkThreads;
    for (int64_t i0 = (int64_t)blockIdx.x * kTopkThreads + threadIdx.x; i0 < n_docs; i0 += 8 * stride) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int64_t i = i0 + u * stride;
            v[u] = i < n_docs ? __ldg(row + i) : -__int_as_float(0x7f800000);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int64_t i = i0 + u * stride;
            if (i < n_docs) L.insert(v[u], (int)i);
        }
    }
    block_merge<KT>(L, ws, wi, res_s, res_i);

    float* my_s = part_s + ((int64_t)q * P + blockIdx.x) * KT;
    int* my_i = part_i + ((int64_t)q * P + blockIdx.x) * KT;
    if (threadIdx.x < KT) my_s[threadIdx.x] = res_s[threadIdx.x], my_i[threadIdx.x] = res_i[threadIdx.x];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = (atomicAdd(counters + q, 1) == P - 1);
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    L.clear();
    for (int l = threadIdx.x; l < P; l += kTopkThreads) {
        // the whole list in 16-byte loads first, then inserts (lists are sorted best-first)
        const float4* ps = reinterpret_cast<const float4*>(part_s + ((int64_t)q * P + l) * KT);
        const int4* pi = reinterpret_cast<const int4*>(part_i + ((int64_t)q * P + l) * KT);
        float cs[KT];
        int ci[KT];
#pragma unroll
        for (int j = 0; j < KT / 4; ++j) {
            const float4 a = __ldcg(ps + j);
            const int4 b = __ldcg(pi + j);
            cs[4 * j] = a.x; cs[4 * j + 1] = a.y; cs[4 * j + 2] = a.z; cs[4 * j + 3] = a.w;
            ci[4 * j] = b.x; ci[4 * j + 1] = b.y; ci[4 * j + 2] = b.z; ci[4 * j + 3] = b.w;
        }
        bool more = true;
#pragma unroll
        for (int j = 0; j < KT; ++j)
            if (more) more = L.insert(cs[j], ci[j]);
    }
    block_merge<KT>(L, ws, wi, res_s, res_i);
    if (threadIdx.x < k) {
        out_idx[(int64_t)q * k + threadIdx.x] = res_i[threadIdx.x];
        if (out_score) out_score[(int64_t)q * k + threadIdx.x] = res_s[threadIdx.x];
    }
}

int pick_kt(int k) { return k <= 8 ? 8 : k <= 16 ? 16 : k <= 32 ? 32 : 64; }

int pick_blocks(int64_t n_docs) {
    int64_t p = (n_docs + kTopkThreads * 4 - 1) / (kTopkThreads * 4);
    const int64_t cap = (int64_t)sm_count() * 2;
    if (p > cap) p = cap;
    if (p < 1) p = 1;
    return (int)p;
}


// ------------------------------------------------------------------------------------------------
// k <= 32: warp-distributed lists. Lane i of a warp holds rank i of the warp's sorted list
// (lanes >= k hold sentinels). A warp loads 16 batches of 32 docs (one per lane each) at a time
// and keeps only the entries not worse than a threshold that already has k entries at least as
// good as it; those survivors (few, once the list has filled) go in 32 at a time: filtered against
// the list's k-th entry with one ballot, each one inserted by a rank count (popc of a ballot) and a
// one-lane shift, or, when more than two survive, sorted and merged in one go. Per block warp 0
// folds the other warps' lists in; with one block per query that is the result, otherwise the
// last block of a query (atomic ticket) folds the per-block lists.
// ------------------------------------------------------------------------------------------------
struct WList {
    float s;
    int i;
};

__device__ __forceinline__ void wl_clear(WList& w) {
    w.s = -__int_as_float(0x7f800000);
    w.i = INT_MAX;
}

// One compare-exchange step of a warp-wide bitonic network on (score, id) pairs: this lane keeps
// the better of itself and lane ^ j when keep_better, else the worse.
__device__ __forceinline__ void cmpx(float& s, int& i, int j, bool keep_better) {
    const float ps = __shfl_xor_sync(0xffffffffu, s, j);
    const int pi = __shfl_xor_sync(0xffffffffu, i, j);
    const bool partner_better = better(ps, pi, s, i);
    if (partner_better == keep_better) {
        s = ps;
        i = pi;
    }
}

// Sorts the 32 lanes' pairs best-first (bitonic sort, 15 stages).
__device__ __forceinline__ void warp_sort32(float& s, int& i) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) cmpx(s, i, j, ((lane & j) == 0) == ((lane & k) == 0));
}

// w (sorted best-first) <- the 32 best of w and b (b sorted best-first): the half-cleaner on w and
// reversed b leaves the 32 best as a bitonic sequence, which a 5-stage bitonic merge sorts.
__device__ __forceinline__ void warp_merge32(WList& w, float bs, int bi) {
    const int lane = threadIdx.x & 31;
    const float rs = __shfl_sync(0xffffffffu, bs, 31 - lane);
    const int ri = __shfl_sync(0xffffffffu, bi, 31 - lane);
    if (better(rs, ri, w.s, w.i)) {
        w.s = rs;
        w.i = ri;
    }
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) cmpx(w.s, w.i, j, (lane & j) == 0);
}

// Inserts every lane's candidate (cv, ci) that beats the list's k-th entry; valid marks real ones.
// One or two survivors go in by rank count and shift; more are sorted and merged in one go.
__device__ __forceinline__ void wl_insert_batch(WList& w, int k, float cv, int ci, bool valid) {
    const int lane = threadIdx.x & 31;
    float ts = __shfl_sync(0xffffffffu, w.s, k - 1);
    int ti = __shfl_sync(0xffffffffu, w.i, k - 1);
    unsigned mask = __ballot_sync(0xffffffffu, valid && better(cv, ci, ts, ti));
    if (__popc(mask) > 2) {
        float s = (mask >> lane) & 1u ? cv : -__int_as_float(0x7f800000);
        int i = (mask >> lane) & 1u ? ci : INT_MAX;
        warp_sort32(s, i);
        warp_merge32(w, s, i);
        return;
    }
    while (mask) {
        const int j = __ffs(mask) - 1;
        const float s = __shfl_sync(0xffffffffu, cv, j);
        const int id = __shfl_sync(0xffffffffu, ci, j);
        const bool ahead = lane < k && better(w.s, w.i, s, id);
        const int pos = __popc(__ballot_sync(0xffffffffu, ahead));
        const float ps = __shfl_up_sync(0xffffffffu, w.s, 1);
        const int pi = __shfl_up_sync(0xffffffffu, w.i, 1);
        if (lane == pos) {
            w.s = s;
            w.i = id;
        } else if (lane > pos && lane < k) {
            w.s = ps;
            w.i = pi;
        }
        ts = __shfl_sync(0xffffffffu, w.s, k - 1);
        ti = __shfl_sync(0xffffffffu, w.i, k - 1);
        mask &= ~(1u << j);
        mask &= __ballot_sync(0xffffffffu, valid && better(cv, ci, ts, ti));
    }
}

// One out-of-line copy of the batch insert for the scan's many call sites (the inlined copies
// would not fit the instruction cache).
__device__ __noinline__ WList wl_insert_batch_call(WList w, int k, float cv, int ci, bool valid) {
    wl_insert_batch(w, k, cv, ci, valid);
    return w;
}

constexpr int kWarpTopkThreads = 256;
constexpr int kRoundBatches = 16;   // batches of 32 docs a warp loads before filtering them

// CL: the P blocks of a query form one thread-block cluster and fold their lists over distributed
// shared memory (no partial lists in global memory, no ticket); otherwise the last block to finish
// folds the partial lists.
template <bool CL>
__global__ void __launch_bounds__(kWarpTopkThreads) topk_warp_kernel(const float* __restrict__ scores, int64_t n_docs,
                                                                      int k, int P, float* part_s, int* part_i,
                                                                      int* counters, int32_t* out_idx, float* out_score) {
    constexpr int W = kWarpTopkThreads / 32;
    // per warp: staged candidates during the scan, then its list for the block's fold
    __shared__ float stage_s[W][64];
    __shared__ int stage_i[W][64];
    __shared__ float2 cl_list[32];     // the block's list, read by the cluster's first block
    __shared__ int is_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = blockIdx.y;
    const float* row = scores + (int64_t)q * n_docs;
    WList w;
    wl_clear(w);
    // this warp's slice: batches of 32 consecutive docs, strided over all warps of all blocks,
    // taken kRoundBatches at a time. Per round only the candidates that can still be among the k
    // best reach the list: those not worse than a threshold that has at least k seen entries at
    // least as good as it (the list's k-th entry, tightened, when that leaves more than one batch,
    // by the k-th best of the lanes' own best entries). Survivors are staged in shared memory
    // (at most 63 at a time) and go in 32 at a time.
    const int64_t gw = (int64_t)blockIdx.x * W + warp, nw = (int64_t)P * W;
    float* st_s = stage_s[warp];
    int* st_i = stage_i[warp];
    for (int64_t base = gw * 32; base < n_docs; base += nw * 32 * kRoundBatches) {
        float v[kRoundBatches];
#pragma unroll
        for (int u = 0; u < kRoundBatches; ++u) {
            const int64_t i = base + u * nw * 32 + lane;
            v[u] = i < n_docs ? __ldg(row + i) : -__int_as_float(0x7f800000);
        }
        float ts = __shfl_sync(0xffffffffu, w.s, k - 1);
        int ti = __shfl_sync(0xffffffffu, w.i, k - 1);
        int count = 0;
#pragma unroll
        for (int u = 0; u < kRoundBatches; ++u) {
            const int64_t i = base + u * nw * 32 + lane;
            count += __popc(__ballot_sync(0xffffffffu, i < n_docs && !better(ts, ti, v[u], (int)i)));
        }
        if (count > 32) {
            float bs = -__int_as_float(0x7f800000);
            int bi = INT_MAX;
#pragma unroll
            for (int u = 0; u < kRoundBatches; ++u) {
                const int64_t i = base + u * nw * 32 + lane;
                if (i < n_docs && better(v[u], (int)i, bs, bi)) bs = v[u], bi = (int)i;
            }
            warp_sort32(bs, bi);
            const float ks = __shfl_sync(0xffffffffu, bs, k - 1);
            const int ki = __shfl_sync(0xffffffffu, bi, k - 1);
            if (better(ks, ki, ts, ti)) ts = ks, ti = ki;
        }
        int n_st = 0;
#pragma unroll
        for (int u = 0; u < kRoundBatches; ++u) {
            const int64_t i = base + u * nw * 32 + lane;
            const bool keep = i < n_docs && !better(ts, ti, v[u], (int)i);
            const unsigned mk = __ballot_sync(0xffffffffu, keep);
            if (keep) {
                const int pos = n_st + __popc(mk & ((1u << lane) - 1u));
                st_s[pos] = v[u];
                st_i[pos] = (int)i;
            }
            n_st += __popc(mk);
            if (n_st >= 32) {
                // a full batch goes in; the rest (at most 31) moves to the front
                __syncwarp();
                const float cs = st_s[lane];
                const int ci = st_i[lane];
                const bool more = lane + 32 < n_st;
                const float ms = more ? st_s[lane + 32] : 0.0f;
                const int mi = more ? st_i[lane + 32] : 0;
                __syncwarp();
                if (more) st_s[lane] = ms, st_i[lane] = mi;
                n_st -= 32;
                w = wl_insert_batch_call(w, k, cs, ci, true);
                __syncwarp();
            }
        }
        if (n_st > 0) {
            __syncwarp();
            const bool ok = lane < n_st;
            const float cs = ok ? st_s[lane] : -__int_as_float(0x7f800000);
            const int ci = ok ? st_i[lane] : INT_MAX;
            __syncwarp();
            w = wl_insert_batch_call(w, k, cs, ci, ok);
        }
    }
    // fold the block's warp lists (sorted) into warp 0's
    stage_s[warp][lane] = w.s;
    stage_i[warp][lane] = w.i;
    __syncthreads();
    if (warp == 0) {
        for (int o = 1; o < W; ++o) warp_merge32(w, stage_s[o][lane], stage_i[o][lane]);
        if (P == 1) {
            // one block per query: its list is the result (no partial lists, no ticket)
            if (lane < k) {
                out_idx[(int64_t)q * k + lane] = w.i;
                if (out_score) out_score[(int64_t)q * k + lane] = w.s;
            }
        } else if (CL) {
            cl_list[lane] = make_float2(w.s, __int_as_float(w.i));
        } else {
            part_s[((int64_t)q * P + blockIdx.x) * 32 + lane] = w.s;
            part_i[((int64_t)q * P + blockIdx.x) * 32 + lane] = w.i;
            __threadfence();
            __syncwarp();
            if (lane == 0) is_last = (atomicAdd(counters + q, 1) == P - 1);
        }
    }
    if (CL) {
        // every block's list is in its shared memory after the first barrier; the cluster's first
        // block folds them in, and the second barrier keeps them in place until it has
        cluster_sync_all();
        if (cluster_ctarank() == 0 && warp == 0 && P > 1) {
            for (int r = 1; r < P; ++r) {
                const float2 e = ld_cluster_f2(cluster_map(smem_u32(&cl_list[lane]), (uint32_t)r));
                warp_merge32(w, e.x, __float_as_int(e.y));
            }
            if (lane < k) {
                out_idx[(int64_t)q * k + lane] = w.i;
                if (out_score) out_score[(int64_t)q * k + lane] = w.s;
            }
        }
        cluster_sync_all();
        return;
    }
    __syncthreads();
    if (P == 1 || !is_last) return;
    // last block: warp w folds partial lists w, w + W, ... (loads first), then warp 0 folds the warps
    __threadfence();
    wl_clear(w);
    for (int b0 = warp; b0 < P; b0 += 4 * W) {
        float cv[4];
        int ci[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int b = b0 + u * W;
            const int64_t off = ((int64_t)q * P + b) * 32 + lane;
            cv[u] = b < P ? __ldcg(part_s + off) : -__int_as_float(0x7f800000);
            ci[u] = b < P ? __ldcg(part_i + off) : INT_MAX;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (b0 + u * W < P) warp_merge32(w, cv[u], ci[u]);
    }
    __syncthreads();
    stage_s[warp][lane] = w.s;
    stage_i[warp][lane] = w.i;
    __syncthreads();
    if (warp == 0) {
        for (int o = 1; o < W; ++o) warp_merge32(w, stage_s[o][lane], stage_i[o][lane]);
        if (lane < k) {
            out_idx[(int64_t)q * k + lane] = w.i;
            if (out_score) out_score[(int64_t)q * k + lane] = w.s;
        }
    }
}

int pick_blocks_warp(int64_t n_docs) {
    // two rounds of kRoundBatches batches of 32 docs per warp: up to 8,192 docs take one block
    // per query (no ticket), and few partial lists are left for the last block to fold
    const int64_t per_block = (int64_t)kWarpTopkThreads * kRoundBatches * 2;
    int64_t p = (n_docs + per_block - 1) / per_block;
    const int64_t cap = (int64_t)sm_count() * 2;
    if (p > cap) p = cap;
    if (p < 1) p = 1;
    return (int)p;
}
constexpr int kMaxTopkCluster = 16;   // above 8 a non-portable cluster size

// k <= 32: up to 8,192 docs take one block per query; up to 131,072 the query's blocks (at most
// 16, each on at most 8,192 docs: two rounds per warp) form one cluster; beyond that the ticket
// fold (measured faster there than clusters whose warps take more rounds).
void warp_plan(int64_t n_docs, int* P, bool* cluster) {
    const int64_t per_block = (int64_t)kWarpTopkThreads * kRoundBatches * 2;
    const int64_t pc = (n_docs + per_block - 1) / per_block;
    if (pc <= 1) {
        *P = 1;
        *cluster = false;
    } else if (pc <= kMaxTopkCluster) {
        *P = (int)pc;
        *cluster = true;
    } else {
        *P = pick_blocks_warp(n_docs);
        *cluster = false;
    }
}

// Clusters of more than 8 blocks need the kernel's opt-in, set once per device.
msa_status allow_large_topk_cluster() {
    static std::mutex mu;
    static bool done[64] = {false};
    int dev = 0;
    MSA_CUDA_TRY(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 0 && dev < 64 && done[dev]) return MSA_OK;
    MSA_CUDA_TRY(cudaFuncSetAttribute(topk_warp_kernel<true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
    if (dev >= 0 && dev < 64) done[dev] = true;
    return MSA_OK;
}

// Launches the selection with the workspace (or scratch) w laid out as msa_topk_workspace_size
// sizes it: partial scores, partial indices, one ticket per query.
msa_status launch_topk(const float* doc_scores, int n_q, int64_t n_docs, int k, int32_t* idx, float* score, char* w,
                       cudaStream_t s) {
    const bool warp_lists = k <= 32;
    const int P_ws = warp_lists ? pick_blocks_warp(n_docs) : pick_blocks(n_docs);
    const int KT = warp_lists ? 32 : pick_kt(k);
    const size_t lists = (size_t)n_q * P_ws * KT;
    float* part_s = reinterpret_cast<float*>(w);
    int* part_i = reinterpret_cast<int*>(w + align_up(lists * 4, 256));
    int* counters = reinterpret_cast<int*>(w + 2 * align_up(lists * 4, 256));
    if (warp_lists) {
        int P = 1;
        bool cluster = false;
        warp_plan(n_docs, &P, &cluster);
        if (cluster) {
            cudaLaunchConfig_t cfg{};
            cfg.gridDim = dim3((unsigned)P, (unsigned)n_q);
            cfg.blockDim = dim3(kWarpTopkThreads);
            cfg.dynamicSmemBytes = 0;
            cfg.stream = s;
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = (unsigned)P;
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            cfg.attrs = at;
            cfg.numAttrs = 1;
            if (P > 8) MSA_RETURN_IF(allow_large_topk_cluster());
            MSA_CUDA_TRY(cudaLaunchKernelEx(&cfg, topk_warp_kernel<true>, doc_scores, n_docs, k, P, part_s, part_i,
                                            counters, idx, score));
            MSA_LAUNCH_CHECK();
            return MSA_OK;
        }
        // tickets start at zero (one block per query takes none)
        if (P > 1) MSA_CUDA_TRY(cudaMemsetAsync(counters, 0, (size_t)n_q * sizeof(int), s));
        topk_warp_kernel<false><<<dim3(P, n_q), kWarpTopkThreads, 0, s>>>(doc_scores, n_docs, k, P, part_s, part_i,
                                                                          counters, idx, score);
        MSA_LAUNCH_CHECK();
        return MSA_OK;
    }
    const int P = P_ws;
    MSA_CUDA_TRY(cudaMemsetAsync(counters, 0, (size_t)n_q * sizeof(int), s));
    dim3 grid(P, n_q);
    switch (KT) {
        case 8: topk_kernel<8><<<grid, kTopkThreads, 0, s>>>(doc_scores, n_docs, k, P, part_s, part_i, counters, idx, score); break;
        case 16: topk_kernel<16><<<grid, kTopkThreads, 0, s>>>(doc_scores, n_docs, k, P, part_s, part_i, counters, idx, score); break;
        case 32: topk_kernel<32><<<grid, kTopkThreads, 0, s>>>(doc_scores, n_docs, k, P, part_s, part_i, counters, idx, score); break;
        default: topk_kernel<64><<<grid, kTopkThreads, 0, s>>>(doc_scores, n_docs, k, P, part_s, part_i, counters, idx, score); break;
    }
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

}  // namespace
}  // namespace msa

using namespace msa;

extern "C" {

msa_status msa_topk_workspace_size(int n_q, int64_t n_docs, int k, size_t* bytes) {
    MSA_REQUIRE(bytes, "msa_topk_workspace_size: bytes is NULL");
    MSA_REQUIRE(n_q > 0 && n_docs > 0 && k > 0 && k <= 64, "msa_topk_workspace_size: bad sizes");
    const bool warp_lists = k <= 32;
    const int P = warp_lists ? pick_blocks_warp(n_docs) : pick_blocks(n_docs);
    const int KT = warp_lists ? 32 : pick_kt(k);
    const size_t lists = (size_t)n_q * P * KT;
    *bytes = align_up(lists * 4, 256) * 2 + align_up((size_t)n_q * 4, 256);
    return MSA_OK;
}

msa_status msa_topk_docs(const float* doc_scores, int n_q, int64_t n_docs, int k, int32_t* idx, float* score,
                         void* ws, size_t ws_bytes, void* stream) {
    MSA_REQUIRE(doc_scores && idx && ws, "msa_topk_docs: NULL pointer");
    MSA_REQUIRE(n_q > 0 && n_docs > 0 && n_docs < (int64_t)INT_MAX, "msa_topk_docs: bad sizes");
    MSA_REQUIRE(k >= 1 && k <= 64 && k <= n_docs, "msa_topk_docs: need 1 <= k <= min(64, n_docs), got k=%d", k);
    MSA_REQUIRE(n_q <= 65535, "msa_topk_docs: at most 65535 queries");
    size_t need = 0;
    MSA_RETURN_IF(msa_topk_workspace_size(n_q, n_docs, k, &need));
    if (ws_bytes < need) return set_error(MSA_ERR_WORKSPACE, "msa_topk_docs: workspace %zu < %zu", ws_bytes, need);
    return launch_topk(doc_scores, n_q, n_docs, k, idx, score, static_cast<char*>(ws), static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------
// Allocation-free variant of msa_topk_docs.
//
// Some callers cannot allocate device memory at the point where they select documents: a C host
// application that loads this library as a plugin and hands it only its input and output buffers,
// a serving loop whose device memory is fully reserved up front by its own pool, or a latency-bound
// loop where cudaMalloc's implicit device synchronisation is not acceptable. For them the partial
// lists and ticket counters live in this fixed, file-scope device array instead of a caller
// workspace. Every GPU that loads the library holds the array until the process exits.
// ------------------------------------------------------------------------------------------------
namespace msa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;   // 1 MiB per device
static __device__ __align__(256) unsigned char g_topk_scratch[kNoAllocScratchBytes];

constexpr int kMaxNoAllocDevices = 64;
void* g_scratch_ptr[kMaxNoAllocDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of g_topk_scratch on the current device, looked up once per device. In host code
// the array's name is only a host-side stand-in, so its address must come from the runtime.
msa_status scratch_address(void** out) {
    int dev = 0;
    MSA_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxNoAllocDevices)
        return set_error(MSA_ERR_UNSUPPORTED, "msa_topk_docs_noalloc: device %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_topk_scratch);
        if (e != cudaSuccess || p == nullptr)
            return set_error(MSA_ERR_CUDA, "msa_topk_docs_noalloc: cudaGetSymbolAddress failed: %s",
                             cudaGetErrorString(e));
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return MSA_OK;
}

}  // namespace
}  // namespace msa

extern "C" {

size_t msa_topk_noalloc_max_scratch(void) { return kNoAllocScratchBytes; }

msa_status msa_topk_docs_noalloc(const float* doc_scores, int n_q, int64_t n_docs, int k, int32_t* idx, float* score,
                                 void* stream) {
    MSA_REQUIRE(doc_scores && idx, "msa_topk_docs_noalloc: NULL pointer");
    MSA_REQUIRE(n_q > 0 && n_docs > 0 && n_docs < (int64_t)INT_MAX, "msa_topk_docs_noalloc: bad sizes");
    MSA_REQUIRE(k >= 1 && k <= 64 && k <= n_docs, "msa_topk_docs_noalloc: need 1 <= k <= min(64, n_docs), got k=%d", k);
    MSA_REQUIRE(n_q <= 65535, "msa_topk_docs_noalloc: at most 65535 queries");
    size_t need = 0;
    MSA_RETURN_IF(msa_topk_workspace_size(n_q, n_docs, k, &need));
    if (need > kNoAllocScratchBytes)
        return set_error(MSA_ERR_INVALID_ARG,
                         "msa_topk_docs_noalloc: n_q=%d, n_docs=%lld, k=%d need %zu bytes of scratch, above the fixed "
                         "%zu-byte array; use msa_topk_docs with a workspace",
                         n_q, (long long)n_docs, k, need, kNoAllocScratchBytes);
    void* ws = nullptr;
    MSA_RETURN_IF(scratch_address(&ws));
    // the array keeps the previous call's contents: launch_topk zeroes the tickets it uses
    return launch_topk(doc_scores, n_q, n_docs, k, idx, score, static_cast<char*>(ws), static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------
// Memory Parallel merge: the k best of every shard's local top-k candidates. Each candidate becomes
// one 64-bit key, order-preserving float bits of its score above the complement of its global
// document index, so that a larger key is a better candidate (higher score, then lower index);
// no candidate (-1) gets key 0, a NaN score ranks below -inf. One block per query counts, for each
// candidate, the candidates that beat it (ties of equal keys by position): that count is its rank.
// ------------------------------------------------------------------------------------------------
namespace msa {
namespace {

constexpr int kMergeMaxShards = 64;
constexpr int kMergeMaxCand = 4096;
constexpr int kMergeThreads = 256;

struct MergeArgs {
    const float* cand_score;
    const int32_t* cand_idx;
    int64_t shard_stride;
    int n_shards, n_q, k_cand, k;
    int64_t shard_off[kMergeMaxShards + 1];
    int32_t* idx;
    float* score;
    int* err;
};

__device__ __forceinline__ uint32_t ordered_bits(float f) {
    const uint32_t b = f == 0.f ? 0u : __float_as_uint(f);   // -0 and +0 compare equal
    if (f != f) return 1u;                                  // NaN: just above "no candidate"
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float from_ordered_bits(uint32_t o) {
    if (o == 1u) return __int_as_float(0x7fc00000);
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

__global__ void __launch_bounds__(kMergeThreads) topk_merge_kernel(const MergeArgs a) {
    __shared__ unsigned long long keys[kMergeMaxCand];
    const int q = blockIdx.x;
    const int n = a.n_shards * a.k_cand;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int g = i / a.k_cand, r = i % a.k_cand;
        const int64_t at = (int64_t)g * a.shard_stride + (int64_t)q * a.k_cand + r;
        const int32_t local = a.cand_idx[at];
        const int64_t size = a.shard_off[g + 1] - a.shard_off[g];
        unsigned long long key = 0ull;
        if (local >= 0 && local < size) {
            const uint32_t gi = (uint32_t)(a.shard_off[g] + local);
            key = ((unsigned long long)ordered_bits(a.cand_score[at]) << 32) | (unsigned long long)(0xffffffffu - gi);
        } else if (local != -1) {
            record_device_error(a.err, MSA_DEV_BAD_INDEX);
        }
        keys[i] = key;
    }
    for (int r = n + threadIdx.x; r < a.k; r += blockDim.x) {   // fewer candidates than k
        a.idx[(int64_t)q * a.k + r] = -1;
        if (a.score) a.score[(int64_t)q * a.k + r] = -__int_as_float(0x7f800000);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const unsigned long long ki = keys[i];
        int rank = 0;
        for (int j = 0; j < n && rank < a.k; ++j) {
            const unsigned long long kj = keys[j];
            rank += (kj > ki) || (kj == ki && j < i);
        }
        if (rank < a.k) {
            const bool valid = ki != 0ull;
            a.idx[(int64_t)q * a.k + rank] = valid ? (int32_t)(0xffffffffu - (uint32_t)(ki & 0xffffffffull)) : -1;
            if (a.score)
                a.score[(int64_t)q * a.k + rank] =
                    valid ? from_ordered_bits((uint32_t)(ki >> 32)) : -__int_as_float(0x7f800000);
        }
    }
}

}  // namespace
}  // namespace msa

extern "C" {

msa_status msa_topk_merge(const float* cand_score, const int32_t* cand_idx, int64_t shard_stride, int n_shards,
                          int n_q, int k_cand, const int64_t* shard_doc_off, int k, int32_t* idx, float* score,
                          void* stream) {
    MSA_REQUIRE(cand_score && cand_idx && shard_doc_off && idx, "msa_topk_merge: NULL pointer");
    MSA_REQUIRE(n_shards >= 1 && n_shards <= kMergeMaxShards, "msa_topk_merge: 1 <= n_shards <= %d", kMergeMaxShards);
    MSA_REQUIRE(n_q >= 1 && n_q <= INT_MAX / 2 && k_cand >= 1 && (int64_t)n_shards * k_cand <= kMergeMaxCand,
                "msa_topk_merge: need n_q >= 1, k_cand >= 1, n_shards * k_cand <= %d", kMergeMaxCand);
    MSA_REQUIRE(k >= 1 && k <= 64, "msa_topk_merge: need 1 <= k <= 64, got %d", k);
    MSA_REQUIRE(shard_stride >= (int64_t)n_q * k_cand, "msa_topk_merge: shard_stride < n_q * k_cand");
    MergeArgs a{};
    a.shard_off[0] = shard_doc_off[0];
    MSA_REQUIRE(shard_doc_off[0] >= 0, "msa_topk_merge: negative shard offset");
    for (int g = 0; g < n_shards; ++g) {
        MSA_REQUIRE(shard_doc_off[g + 1] >= shard_doc_off[g], "msa_topk_merge: shard offsets must not decrease");
        a.shard_off[g + 1] = shard_doc_off[g + 1];
    }
    MSA_REQUIRE(shard_doc_off[n_shards] < (int64_t)INT_MAX, "msa_topk_merge: global document index exceeds int32");
    a.cand_score = cand_score; a.cand_idx = cand_idx; a.shard_stride = shard_stride;
    a.n_shards = n_shards; a.n_q = n_q; a.k_cand = k_cand; a.k = k;
    a.idx = idx; a.score = score; a.err = device_error_word();
    topk_merge_kernel<<<n_q, kMergeThreads, 0, static_cast<cudaStream_t>(stream)>>>(a);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

}  // extern "C"
