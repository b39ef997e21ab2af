// Router backward, best-token search on tcgen05 tensor cores (sm_100a).
//
// The document score's subgradient flows to the (chunk, token) pair that attains it. For every
// query q and chunk c this kernel finds the best folded score over the query's tokens and the
// first token attaining it:
//   score[c][t] = <index[c], qhat[q][t]>    (index rows are unit-vector heads, qhat carries 1/H)
// GEMM view (chunks on M, as in the forward router): D[m][n] = sum_k index[m][k] * qhat[n][k].
// The fp32 qhat is split exactly into three bf16 terms (hi + mid + lo, each the bf16 rounding of
// what the previous terms leave), so the bf16 tensor cores see the same fp32 operand the CUDA-core
// kernel reads; products of two bf16 values are exact in the fp32 accumulator. Only the operand is
// exact: the 3 x 4 MMAs per slab add the products in another order than the CUDA-core kernel's fp32
// dot product, so on tokens whose scores differ by a rounding error the two kernels can pick
// different best tokens (exact ties still go to the first token in both).
//
// One CTA per (128 chunks, 32 tokens, query): warp 0 loads 64-element K slabs of the index tile
// and of the three qhat terms by TMA (128-byte swizzle) into 4 stages; warp 1 owns 32 TMEM columns
// and issues 4 x 3 MMAs (M 128, N 32, K 16) per slab into one accumulator; warps 2..5 read their
// 32 TMEM lanes (one chunk per thread), scan the 32 token columns in order (strictly greater
// replaces, so the first maximum stays) and merge (score, first token) into the launch-wide
// 64-bit key with one atomic max per chunk. Every mbarrier wait is bounded; on expiry the CTA
// records MSA_DEV_WAIT_TIMEOUT, writes nothing, waits (bounded) for its copies and MMAs and frees
// TMEM.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace msa {
namespace {

constexpr int BM = 128;                            // chunks per tile = MMA M = TMEM lanes
constexpr int BK = 64;                             // bf16 elements per 128-byte swizzled row
constexpr int BN = 32;                             // query tokens per tile = MMA N
constexpr int kThreads = 192;
constexpr int kStages = 4;
constexpr int kSplits = 3;
constexpr int kStageA = BM * BK * 2;               // 16 KB
constexpr int kSplitB = BN * BK * 2;               // 4 KB per qhat term
constexpr int kStageBytes = kStageA + kSplits * kSplitB;
constexpr int kTmemCols = 32;
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 256;

struct BestTcArgs {
    int64_t n_chunks;
    int K, T, T_pad, n_q;
    uint32_t idesc;
    unsigned long long* best;
    int* err;
};

__device__ __forceinline__ unsigned long long best_key_tc(float score, int t) {
    const uint32_t b = __float_as_uint(score);
    const uint32_t o = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((unsigned long long)o << 32) | (unsigned long long)(0xffffffffu - (uint32_t)t);
}

__global__ void __launch_bounds__(kThreads, 1)
    route_bwd_best_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const BestTcArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(base + kStages * kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* done = empty + kStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t m0 = (int64_t)blockIdx.x * BM;
    const int n0 = blockIdx.y * BN;
    const int q = blockIdx.z;
    const int kblocks = p.K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        mbar_init(smem_u32(done), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------- TMA producer
        if (lane == 0) {
            bool issued[kStages];
            uint32_t issued_phase[kStages];
            for (int s = 0; s < kStages; ++s) issued[s] = false, issued_phase[s] = 0;
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int kb = 0; kb < kblocks; ++kb) {
                if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = smem_u32(&full[stage]);
                uint8_t* sa = base + stage * kStageBytes;
                mbar_expect_tx(fb, (uint32_t)kStageBytes);
                tma_load_2d(smem_u32(sa), &tmA, kb * BK, (int)m0, fb);
                for (int s = 0; s < kSplits; ++s)
                    tma_load_2d(smem_u32(sa + kStageA + s * kSplitB), &tmB, kb * BK, (s * p.n_q + q) * p.T_pad + n0,
                                fb);
                issued[stage] = true;
                issued_phase[stage] = phase;
                if (++stage == kStages) stage = 0, phase ^= 1u;
            }
            if (!ok) {
                // let the copies this thread issued land before the CTA exits
                for (int s = 0; s < kStages; ++s)
                    if (issued[s]) mbar_wait_drain(smem_u32(&full[s]), issued_phase[s]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int kb = 0; kb < kblocks; ++kb) {
                if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(base + stage * kStageBytes);
                const uint64_t adesc = sw128_desc(a_addr);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
#pragma unroll
                    for (int s = 0; s < kSplits; ++s) {
                        // +32 bytes per 16-element step inside the swizzle atom (encoded >> 4)
                        const uint64_t bdesc = sw128_desc(a_addr + (uint32_t)(kStageA + s * kSplitB));
                        umma_bf16(tmem_base, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), p.idesc,
                                  (kb | kk | s) != 0 ? 1u : 0u);
                    }
                }
                umma_commit(smem_u32(&empty[stage]));
                if (++stage == kStages) stage = 0, phase ^= 1u;
            }
            // arrives once every MMA issued above has completed (at once when none was issued)
            umma_commit(smem_u32(done));
            if (!ok) mbar_wait_drain(smem_u32(done), 0);
        }
    } else {
        // ------------------------------------------------------------- epilogue
        const int quarter = warp & 3;
        bool ok = true;
        if (lane == 0) ok = mbar_wait(smem_u32(done), 0, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (ok) {
            tc_fence_after();
            float v[32];
            tmem_ld32(tmem_base + ((uint32_t)(quarter * 32) << 16), v);
            if (*abort_flag == 0) {
                const int64_t c = m0 + quarter * 32 + lane;
                const int nv = min(BN, p.T - n0);   // real tokens in this tile
                float bm = 0.f;
                int bt = -1;
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (j < nv && (bt < 0 || v[j] > bm)) {
                        bm = v[j];
                        bt = j;
                    }
                if (c < p.n_chunks && bt >= 0)
                    atomicMax(p.best + (int64_t)q * p.n_chunks + c, best_key_tc(bm, n0 + bt));
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) record_device_error(p.err, MSA_DEV_WAIT_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace

int route_bwd_tc_token_tile() { return BN; }

msa_status launch_route_bwd_best_tc(const void* index, int64_t n_chunks, const void* qsplit, int n_q, int T,
                                    int T_pad, int K, unsigned long long* best, cudaStream_t s) {
    if (K % BK != 0 || T_pad % BN != 0 || n_chunks <= 0)
        return set_error(MSA_ERR_UNSUPPORTED, "route backward (tensor cores): K %d or padded T %d unsupported", K, T_pad);
    if ((n_chunks + BM - 1) / BM > 0x7fffffff || (int64_t)kSplits * n_q * T_pad > 0x7fffffff)
        return set_error(MSA_ERR_UNSUPPORTED, "route backward (tensor cores): too many rows");
    CUtensorMap tmA, tmB;
    const uint64_t dims_a[2] = {(uint64_t)K, (uint64_t)n_chunks};
    const uint64_t dims_b[2] = {(uint64_t)K, (uint64_t)kSplits * n_q * T_pad};
    const uint64_t strides[1] = {(uint64_t)K * 2};
    const uint32_t box_a[2] = {(uint32_t)BK, (uint32_t)BM};
    const uint32_t box_b[2] = {(uint32_t)BK, (uint32_t)BN};
    MSA_RETURN_IF(make_tensor_map_bf16(&tmA, index, 2, dims_a, strides, box_a));
    MSA_RETURN_IF(make_tensor_map_bf16(&tmB, qsplit, 2, dims_b, strides, box_b));
    BestTcArgs p{};
    p.n_chunks = n_chunks;
    p.K = K; p.T = T; p.T_pad = T_pad; p.n_q = n_q;
    p.idesc = (1u << 4)                            // D format: f32
              | (1u << 7)                          // A format: bf16
              | (1u << 10)                         // B format: bf16
              | ((uint32_t)(BN >> 3) << 17)        // N / 8
              | ((uint32_t)(BM >> 4) << 24);       // M / 16 ; A and B K-major
    p.best = best;
    p.err = device_error_word();
    {
        // once per device: opt the kernel into its dynamic shared memory
        static std::mutex mu;
        static bool opted[64] = {false};
        int dev = 0;
        MSA_CUDA_TRY(cudaGetDevice(&dev));
        std::lock_guard<std::mutex> lk(mu);
        if (dev < 0 || dev >= 64 || !opted[dev]) {
            MSA_CUDA_TRY(cudaFuncSetAttribute(route_bwd_best_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              kSmemBytes));
            if (dev >= 0 && dev < 64) opted[dev] = true;
        }
    }
    const dim3 grid((unsigned)((n_chunks + BM - 1) / BM), (unsigned)(T_pad / BN), (unsigned)n_q);
    route_bwd_best_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(tmA, tmB, p);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

}  // namespace msa
