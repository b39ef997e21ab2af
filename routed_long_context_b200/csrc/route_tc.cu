// Tensor-core router for sm_100a: tcgen05.mma (kind::f16, bf16 in, fp32 accumulate in TMEM),
// operands staged in shared memory by TMA with the 128-byte swizzle, persistent CTAs.
//
// GEMM view (swap-AB: chunks on M because the query side is narrow):
//   D[m][n] = sum_k index[m][k] * qhat[n][k],  m = chunk, n = query token column, k = head*d + i.
// Epilogue: per chunk (TMEM lane), max over each query's token columns, then a segmented max
// over the document runs of the warp's 32 consecutive chunks, then one float atomic max per
// (document, query) run into doc_scores (and per chunk into chunk_scores when requested).
//
// Roles (192 threads): warp 0 = TMA producer, warp 1 = TMEM owner and MMA issuer,
// warps 2..5 = epilogue (warp w reads TMEM lanes 32*(w%4) .. 32*(w%4)+31).
// Two TMEM accumulators let the epilogue of tile i overlap the main loop of tile i+1.
// Tiles are handed out dynamically: the producer takes the next tile index from a launch-wide
// atomic counter and publishes it to the MMA and epilogue warps through a 2-entry shared-memory
// queue, so CTAs that start late (SMs still busy with concurrent kernels) simply take fewer tiles.
// Modes: RESIDENT keeps all of qhat (<= 64 columns) in shared memory, loaded once per CTA,
// so only the index streams; by default qhat tiles of BN <= 256 columns stream (from L2) with A.
// Every mbarrier wait is bounded (about 2 s of %globaltimer); on expiry the CTA records
// MSA_DEV_WAIT_TIMEOUT, all roles leave their loops, in-flight copies and MMAs are waited for
// (again bounded) and TMEM is freed before the kernel returns.
#include <cuda.h>

#include <algorithm>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace msa {
namespace {

constexpr int BM = 128;               // chunks per tile = MMA M = TMEM lanes
constexpr int BK = 64;                // bf16 elements per 128-byte swizzled row
constexpr int kThreads = 192;
constexpr int kMaxStages = 12;
constexpr int kSmemLimit = 232448;    // max dynamic shared memory per block on sm_100
// Default budget: leaves room on each SM (228 KB of shared memory) for one attention block
// (35 KB) and one top-k block (5 KB) of the overlapped selection/attention of earlier layers.
constexpr int kSmemBudget = 188 * 1024;
std::atomic<int> g_max_stages{0};     // testing knob: 0 = as many stages as the budget allows
std::atomic<int> g_inject_stall{0};   // testing knob: make the next launches' waits time out
constexpr int kStageA = BM * BK * 2;  // 16 KB
constexpr int kBarBytes = 512;       // mbarriers, TMEM slot, abort flag, tile queue
// T = 1 epilogue: each epilogue warp's 32 x 32 score block, transposed through shared memory
// (row stride 33 floats: conflict-free both ways), and its 32 chunks' documents
constexpr int kEpiStride = 33;
constexpr int kEpiBytes = 4 * 32 * kEpiStride * 4 + 4 * 32 * 4;

struct TcParams {
    int64_t n_chunks;
    int K, N, T, n_pad, BN, n_tiles_n;
    int acc_stride;        // TMEM columns between the two accumulators: BN rounded up to 32
    int64_t n_tiles;
    int stages;
    uint32_t tmem_cols;
    uint32_t idesc;
    const int32_t* chunk_doc;
    int64_t n_docs;
    float* doc_scores;
    float* chunk_scores;
    int* err;
    int* tile_counter;     // zero at launch; tiles are handed out in order by atomicAdd
    int inject_stall;      // testing: the producer never publishes a tile, so every other wait times out
    int transpose;         // T = 1: the epilogue walks each query's column (kEpiBytes after the barriers)
};

// ------------------------------------------------------------------------------------- kernel
// Max over each of the 32 / T whole queries of one 32-column piece (T static), then the query's
// flush; every step is unrolled, so the queries' shuffle chains interleave.
template <int T, typename Flush>
__device__ __forceinline__ void flush_queries(const float (&v)[32], int q0, int q_end, Flush& flush) {
#pragma unroll
    for (int qi = 0; qi < 32 / T; ++qi) {
        float m = v[qi * T];
#pragma unroll
        for (int j = 1; j < T; ++j) m = fmaxf(m, v[qi * T + j]);
        flush(q0 + qi, m, q0 + qi < q_end);
    }
}

template <bool RESIDENT>
__global__ void __launch_bounds__(kThreads, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int kblocks = p.K / BK;
    const int stage_b = p.BN * BK * 2;                               // bytes of one qhat k-block
    const int b_bytes = RESIDENT ? kblocks * stage_b : p.stages * stage_b;
    uint8_t* smem_b = base;
    uint8_t* smem_a = base + b_bytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem_a + p.stages * kStageA);
    uint64_t* full = bars;                    // [kMaxStages]
    uint64_t* empty = bars + kMaxStages;      // [kMaxStages]
    uint64_t* tfull = bars + 2 * kMaxStages;  // [2]
    uint64_t* tempty = tfull + 2;             // [2]
    uint64_t* bfull = tempty + 2;             // [1]
    uint64_t* tqf = bfull + 1;                // [2] tile queue: entry written
    uint64_t* tqe = tqf + 2;                  // [2] tile queue: entry read by the MMA and 4 epilogue warps
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tqe + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* tile_q = abort_flag + 1;    // [2] tile index per queue entry, -1 = no more tiles
    float* epi_buf = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + kBarBytes);   // [4][32][33]
    int* epi_doc = reinterpret_cast<int*>(epi_buf + 4 * 32 * kEpiStride);                      // [4][32]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 4);
        }
        mbar_init(smem_u32(bfull), 1);
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tqf[a]), 1);
            mbar_init(smem_u32(&tqe[a]), 5);
        }
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
                     "r"(p.tmem_cols)
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
            const uint64_t pol = policy_evict_first();
            uint32_t issued_phase[kMaxStages];
            bool issued[kMaxStages];
            for (int s = 0; s < kMaxStages; ++s) issued[s] = false, issued_phase[s] = 0;
            bool ok = true;
            bool b_issued = false;
            if (RESIDENT) {
                mbar_expect_tx(smem_u32(bfull), (uint32_t)(kblocks * stage_b));
                for (int kb = 0; kb < kblocks; ++kb)
                    tma_load_2d(smem_u32(smem_b + kb * stage_b), &tmB, kb * BK, 0, smem_u32(bfull));
                b_issued = true;
            }
            int stage = 0;
            uint32_t phase = 0;
            for (int seq = 0; ok; ++seq) {
                // next tile from the launch-wide counter, published through the 2-entry tile queue
                const int tslot = seq & 1;
                if (!mbar_wait(smem_u32(&tqe[tslot]), (((uint32_t)seq >> 1) & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                if (p.inject_stall) break;     // nothing issued: the consumers' bounded waits run out
                const int t = atomicAdd(p.tile_counter, 1);
                const int tile = (int64_t)t < p.n_tiles ? t : -1;
                tile_q[tslot] = tile;
                mbar_arrive(smem_u32(&tqf[tslot]));
                if (tile < 0) break;
                const int m0 = (tile / p.n_tiles_n) * BM;
                const int n0 = (tile % p.n_tiles_n) * p.BN;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full[stage]);
                    mbar_expect_tx(fb, (uint32_t)(RESIDENT ? kStageA : kStageA + stage_b));
                    tma_load_2d_evict_first(smem_u32(smem_a + stage * kStageA), &tmA, kb * BK, m0, fb, pol);
                    if (!RESIDENT) tma_load_2d(smem_u32(smem_b + stage * stage_b), &tmB, kb * BK, n0, fb);
                    issued[stage] = true;
                    issued_phase[stage] = phase;
                    if (++stage == p.stages) stage = 0, phase ^= 1;
                }
            }
            if (!ok) {
                // drain: wait (bounded, ignoring the abort flag) for copies this thread issued
                const uint64_t t0 = globaltimer();
                for (int s = 0; s < p.stages; ++s)
                    while (issued[s] && !mbar_try_wait(smem_u32(&full[s]), issued_phase[s]) &&
                           globaltimer() - t0 < kWaitNs) {
                    }
                if (b_issued)
                    while (!mbar_try_wait(smem_u32(bfull), 0) && globaltimer() - t0 < kWaitNs) {
                    }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            bool ok = true;
            if (RESIDENT) ok = mbar_wait(smem_u32(bfull), 0, abort_flag);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool mma_pending = false;
            for (int seq = 0; ok; ++seq) {
                const int tslot = seq & 1;
                if (!mbar_wait(smem_u32(&tqf[tslot]), ((uint32_t)seq >> 1) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                const int tile = tile_q[tslot];
                mbar_arrive(smem_u32(&tqe[tslot]));
                if (tile < 0) break;
                acc = seq & 1;
                acc_phase = ((uint32_t)seq >> 1) & 1u;
                if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * p.acc_stride);
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem_a + stage * kStageA);
                    const uint32_t b_addr = RESIDENT ? smem_u32(smem_b + kb * stage_b) : smem_u32(smem_b + stage * stage_b);
                    const uint64_t adesc = sw128_desc(a_addr);
                    const uint64_t bdesc = sw128_desc(b_addr);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        // +32 bytes per 16-element step inside the swizzle atom (encoded >> 4)
                        umma_bf16(d_tmem, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), p.idesc,
                                  (kb | kk) != 0 ? 1u : 0u);
                    }
                    mma_pending = true;
                    umma_commit(smem_u32(&empty[stage]));
                    if (++stage == p.stages) stage = 0, phase ^= 1;
                }
                if (!ok) break;
                umma_commit(smem_u32(&tfull[acc]));
                mma_pending = false;
            }
            if (!ok && mma_pending) {
                // drain: commit to a free barrier and wait (bounded) for the issued MMAs
                umma_commit(smem_u32(&tfull[acc]));
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(smem_u32(&tfull[acc]), acc_phase) && globaltimer() - t0 < kWaitNs) {
                }
            }
        }
    } else {
        // ------------------------------------------------------------- epilogue
        const int quarter = warp & 3;
        const float ninf = -__int_as_float(0x7f800000);
        for (int seq = 0;; ++seq) {
            const int tslot = seq & 1;
            bool ok = true;
            int tile = -1;
            if (lane == 0) {
                ok = mbar_wait(smem_u32(&tqf[tslot]), ((uint32_t)seq >> 1) & 1u, abort_flag);
                if (ok) {
                    tile = tile_q[tslot];
                    mbar_arrive(smem_u32(&tqe[tslot]));
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            tile = __shfl_sync(0xffffffffu, tile, 0);
            if (!ok || tile < 0) break;
            const int acc = seq & 1;
            const uint32_t acc_phase = ((uint32_t)seq >> 1) & 1u;
            if (lane == 0) ok = mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            tc_fence_after();
            const int64_t m0 = (tile / p.n_tiles_n) * BM;
            const int n0 = (int)(tile % p.n_tiles_n) * p.BN;
            const int64_t c = m0 + quarter * 32 + lane;
            const bool valid = c < p.n_chunks;
            int doc = valid ? p.chunk_doc[c] : -1;
            if (valid && (doc < 0 || doc >= p.n_docs)) {
                record_device_error(p.err, MSA_DEV_BAD_INDEX);
                doc = -1;
            }
            const int col_end = min(n0 + p.BN, p.N);   // columns of this tile that are real tokens
            // 32-column reads stay inside this accumulator's acc_stride columns
            const uint32_t trow = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * p.acc_stride);

            if (p.transpose) {
                // T = 1: lane = chunk on the way in, lane = query on the way out. The warp's 32 x 32
                // block goes through shared memory transposed; each lane then walks its query's
                // column down the 32 chunks, whose document runs are the same for every lane
                // (uniform branches), and one atomic per run covers 32 queries.
                float* tb = epi_buf + quarter * (32 * kEpiStride);
                int* td = epi_doc + quarter * 32;
                td[lane] = doc;
                const int pieces = (max(col_end - n0, 0) + 31) / 32;
                for (int pc = 0; pc < pieces; ++pc) {
                    float v[32];
                    tmem_ld32(trow + (uint32_t)(pc * 32), v);
                    if (pc == pieces - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) tb[j * kEpiStride + lane] = v[j];
                    __syncwarp();
                    const int q = n0 + pc * 32 + lane;
                    const bool real = q < col_end;
                    float* qrow = p.doc_scores + (int64_t)q * p.n_docs;
                    float m = ninf;
                    int run_doc = -1;
#pragma unroll
                    for (int cc = 0; cc < 32; ++cc) {
                        const int dc = td[cc];
                        const float x = tb[lane * kEpiStride + cc];
                        if (dc != run_doc) {
                            if (run_doc >= 0 && real) atomic_max_f32(qrow + run_doc, m);
                            run_doc = dc;
                            m = x;
                        } else {
                            m = fmaxf(m, x);
                        }
                        if (p.chunk_scores && dc >= 0 && real)
                            atomic_max_f32(p.chunk_scores + (int64_t)q * p.n_chunks + (m0 + quarter * 32 + cc), x);
                    }
                    if (run_doc >= 0 && real) atomic_max_f32(qrow + run_doc, m);
                    __syncwarp();
                }
                if (pieces == 0) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));
                }
                continue;
            }

            // The warp's 32 consecutive chunks form runs of equal document. Which lanes a
            // segmented max may combine is the same for every query column: bit i of `same` says
            // lane + 2^i holds this lane's document; `head` marks the first lane of each run.
            unsigned same = 0;
#pragma unroll
            for (int i = 0; i < 5; ++i) {
                const int od = __shfl_down_sync(0xffffffffu, doc, 1 << i);
                if (lane + (1 << i) < 32 && od == doc) same |= 1u << i;
            }
            const int prev = __shfl_up_sync(0xffffffffu, doc, 1);
            const bool head = doc >= 0 && (lane == 0 || prev != doc);

            // segmented max of m over the lane's document run, one float atomic max per run
            auto flush = [&](int q, float m, bool real) {
                float v = doc >= 0 ? m : ninf;
#pragma unroll
                for (int i = 0; i < 5; ++i) {
                    const float ov = __shfl_down_sync(0xffffffffu, v, 1 << i);
                    if ((same >> i) & 1u) v = fmaxf(v, ov);
                }
                if (real && head) atomic_max_f32(p.doc_scores + (int64_t)q * p.n_docs + doc, v);
                if (real && p.chunk_scores && doc >= 0) atomic_max_f32(p.chunk_scores + (int64_t)q * p.n_chunks + c, m);
            };

            const int pieces = (max(col_end - n0, 0) + 31) / 32;
            auto release = [&]() {
                // every TMEM read of this accumulator is done: hand it back to the MMA warp
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));
            };
            if (32 % p.T == 0) {
                // a query's T columns never straddle a 32-column piece (pieces start at multiples of
                // 32 and N is a multiple of T): each piece holds 32 / T whole queries, reduced and
                // flushed without branches; queries past col_end are padding and issue no atomics
                const int q_end = col_end / p.T;
                for (int pc = 0; pc < pieces; ++pc) {
                    float v[32];
                    tmem_ld32(trow + (uint32_t)(pc * 32), v);
                    if (pc == pieces - 1) release();
                    const int q0 = (n0 + pc * 32) / p.T;
                    switch (p.T) {
                        case 1: flush_queries<1>(v, q0, q_end, flush); break;
                        case 2: flush_queries<2>(v, q0, q_end, flush); break;
                        case 4: flush_queries<4>(v, q0, q_end, flush); break;
                        case 8: flush_queries<8>(v, q0, q_end, flush); break;
                        case 16: flush_queries<16>(v, q0, q_end, flush); break;
                        default: flush_queries<32>(v, q0, q_end, flush); break;
                    }
                }
                if (pieces == 0) release();
                continue;
            }

            int run_q = -1;
            float run_max = ninf;
            for (int pc = 0; pc < pieces; ++pc) {
                float v[32];
                tmem_ld32(trow + (uint32_t)(pc * 32), v);
                if (pc == pieces - 1) release();
                const int base_col = n0 + pc * 32;
                const int hi_col = min(base_col + 32, col_end);
                for (int q = base_col / p.T; q * p.T < hi_col; ++q) {
                    const int lo_j = max(q * p.T - base_col, 0);
                    const int hi_j = min((q + 1) * p.T, hi_col) - base_col;
                    float m = (q == run_q) ? run_max : ninf;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (j >= lo_j && j < hi_j) m = fmaxf(m, v[j]);
                    // the query's columns in this tile are complete once they end inside this
                    // piece or the tile's real columns end here; otherwise carry the running max
                    if ((q + 1) * p.T <= hi_col || hi_col == col_end) {
                        flush(q, m, true);
                        run_q = -1;
                    } else {
                        run_q = q;
                        run_max = m;
                    }
                }
            }
            if (pieces == 0) release();
            if (run_q >= 0) flush(run_q, run_max, true);
        }
    }

    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) record_device_error(p.err, MSA_DEV_WAIT_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(p.tmem_cols)
                     : "memory");
    }
}

// ------------------------------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

msa_status make_map(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t rows, uint32_t box_rows, bool l2_256) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return set_error(MSA_ERR_CUDA, "route (tensor cores): cuTensorMapEncodeTiled unavailable");
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {inner * 2};
    const cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    l2_256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(MSA_ERR_CUDA, "route (tensor cores): tensor map encode failed (%d)", (int)r);
    return MSA_OK;
}

}  // namespace

// Tensor map of a bf16 array for TMA loads with the 128-byte swizzle (shared with the attention
// kernels): dims[0] innermost (elements), strides in bytes for dims 1..rank-1.
msa_status make_tensor_map(CUtensorMap* map, const void* ptr, bool fp32, int rank, const uint64_t* dims,
                           const uint64_t* strides, const uint32_t* box, bool swizzle128) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return set_error(MSA_ERR_CUDA, "tensor map: cuTensorMapEncodeTiled unavailable");
    if (rank < 1 || rank > 5) return set_error(MSA_ERR_INVALID_ARG, "tensor map: rank %d", rank);
    cuuint64_t d[5], st[4];
    cuuint32_t b[5], e[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        e[i] = 1;
        if (i + 1 < rank) st[i] = strides[i];
    }
    CUresult r = fn(map, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank,
                    const_cast<void*>(ptr), d, st, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(MSA_ERR_CUDA, "tensor map encode failed (%d)", (int)r);
    return MSA_OK;
}

msa_status make_tensor_map_bf16(CUtensorMap* map, const void* ptr, int rank, const uint64_t* dims,
                                const uint64_t* strides, const uint32_t* box) {
    return make_tensor_map(map, ptr, false, rank, dims, strides, box, true);
}

namespace {

struct Plan {
    bool resident;
    int BN, n_pad, n_tiles_n, stages;
    size_t smem;
};

// Streamed qhat is the default: the query block is re-read from L2 with every index tile, which
// leaves shared memory for more index stages in flight (measured faster than keeping qhat
// resident at 64 columns). `resident` asks for qhat held in shared memory when it fits.
bool make_plan(int N, int K, Plan* pl, bool resident = false, bool transpose = false) {
    if (N <= 0 || K <= 0 || K % BK != 0 || K > 8192) return false;
    const int kblocks = K / BK;
    const int n16 = (N + 15) / 16 * 16;
    const size_t fixed = 1024 + kBarBytes + (transpose ? kEpiBytes : 0);
    if (resident && n16 <= 64) {
        const size_t b = (size_t)kblocks * n16 * BK * 2;
        if (fixed + b + 4 * kStageA <= (size_t)kSmemLimit) {
            int st = (int)((kSmemLimit - fixed - b) / kStageA);
            if (st > kMaxStages) st = kMaxStages;
            *pl = Plan{true, n16, n16, 1, st, fixed + b + (size_t)st * kStageA};
            return true;
        }
    }
    const int BN = n16 <= 256 ? n16 : 256;
    const int n_tiles_n = (N + BN - 1) / BN;
    const size_t stage = (size_t)kStageA + (size_t)BN * BK * 2;
    const int forced = g_max_stages.load();
    int st = (int)((kSmemBudget - fixed) / stage);
    if (st < 4) st = (int)((kSmemLimit - fixed) / stage);      // wide query blocks: use it all
    if (forced > 0) st = std::min(forced, (int)((kSmemLimit - fixed) / stage));
    if (st > kMaxStages) st = kMaxStages;
    if (st < 2) return false;
    *pl = Plan{false, BN, n_tiles_n * BN, n_tiles_n, st, fixed + (size_t)st * stage};
    return true;
}

// Opts both kernel variants into the largest dynamic shared memory once per device.
msa_status allow_max_smem() {
    static std::mutex mu;
    static bool done[64] = {false};
    int dev = 0;
    MSA_CUDA_TRY(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 0 && dev < 64 && done[dev]) return MSA_OK;
    MSA_CUDA_TRY(cudaFuncSetAttribute(route_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit));
    MSA_CUDA_TRY(cudaFuncSetAttribute(route_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit));
    if (dev >= 0 && dev < 64) done[dev] = true;
    return MSA_OK;
}

}  // namespace

void route_tc_set_max_stages(int n) { g_max_stages.store(n); }
void route_tc_inject_stall(int on) { g_inject_stall.store(on); }

int route_tc_pad_rows(int N, int K, bool resident) {
    Plan pl;
    return make_plan(N, K, &pl, resident) ? pl.n_pad : 0;
}

msa_status launch_route_tc(const RouteTcArgs& a, cudaStream_t s) {
    Plan pl;
    const bool transpose = a.T == 1;
    if (!make_plan(a.N, a.K, &pl, a.resident, transpose) || pl.n_pad != a.n_pad)
        return set_error(MSA_ERR_UNSUPPORTED, "route (tensor cores): unsupported shape N=%d K=%d", a.N, a.K);
    CUtensorMap tmA, tmB;
    MSA_RETURN_IF(make_map(&tmA, a.index, (uint64_t)a.K, (uint64_t)a.n_chunks, BM, true));
    MSA_RETURN_IF(make_map(&tmB, a.qhat, (uint64_t)a.K, (uint64_t)pl.n_pad, (uint32_t)pl.BN, false));
    TcParams p{};
    p.n_chunks = a.n_chunks;
    p.K = a.K; p.N = a.N; p.T = a.T; p.n_pad = pl.n_pad; p.BN = pl.BN; p.n_tiles_n = pl.n_tiles_n;
    const int64_t m_tiles = (a.n_chunks + BM - 1) / BM;
    p.n_tiles = m_tiles * pl.n_tiles_n;
    p.stages = pl.stages;
    p.acc_stride = (pl.BN + 31) / 32 * 32;
    uint32_t cols = 32;
    while (cols < (uint32_t)(2 * p.acc_stride)) cols <<= 1;
    if (cols > 512) return set_error(MSA_ERR_UNSUPPORTED, "route (tensor cores): %u TMEM columns needed", cols);
    p.tmem_cols = cols;
    p.idesc = (1u << 4)                      // D format: f32
              | (1u << 7)                    // A format: bf16
              | (1u << 10)                   // B format: bf16
              | ((uint32_t)(pl.BN >> 3) << 17)   // N / 8
              | ((uint32_t)(BM >> 4) << 24);     // M / 16 ; A and B K-major (bits 15, 16 = 0)
    p.chunk_doc = a.chunk_doc; p.n_docs = a.n_docs; p.doc_scores = a.doc_scores; p.chunk_scores = a.chunk_scores;
    p.err = a.err;
    p.tile_counter = a.tile_counter;
    p.inject_stall = g_inject_stall.load();
    p.transpose = transpose ? 1 : 0;
    if (!p.tile_counter) return set_error(MSA_ERR_INVALID_ARG, "route (tensor cores): no tile counter");
    int64_t grid = p.n_tiles < (int64_t)sm_count() ? p.n_tiles : (int64_t)sm_count();
    if (a.grid_cap > 0 && grid > a.grid_cap) grid = a.grid_cap;
    MSA_RETURN_IF(allow_max_smem());
    if (pl.resident)
        route_tc_kernel<true><<<(unsigned)grid, kThreads, pl.smem, s>>>(tmA, tmB, p);
    else
        route_tc_kernel<false><<<(unsigned)grid, kThreads, pl.smem, s>>>(tmA, tmB, p);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

}  // namespace msa
