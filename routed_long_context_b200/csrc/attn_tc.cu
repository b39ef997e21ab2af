// Sparse attention on tcgen05 tensor cores (sm_100a) for long memories: the split-key variant of
// msa_sparse_attn_split (bf16, d = 128), one CTA per (128-row block, kv head, query, key range).
//
// Rows r = t * G + h' are the (token, head) pairs of kv head g: 128 rows = the MMA's M = TMEM lanes.
// Per 64-key tile j of the CTA's range:
//   S_j = Q K_j^T          tcgen05.mma, M = 128, N = 64, K = 128 (two 64-element K blocks), into one
//                          of two TMEM S buffers (the MMA of tile j+1 overlaps the softmax of tile j)
//   softmax                two threads per row (TMEM lane), each on 32 of the tile's keys: online
//                          max (shared by the pair) and sums in fp32 (log2 domain), P_j rounded to
//                          bf16 into the shared-memory P buffer (128-byte swizzle, the K-major A
//                          operand, free again once P_{j-1} V has completed); only when a row's max
//                          grows by more than 2^8 is its O
//                          row in TMEM rescaled (tcgen05.ld / st, after the previous P V has
//                          completed), so most tiles never wait for a P V
//   O += P_j V_j           tcgen05.mma, M = 128, N = 128, K = 64; V_j is read MN-major (d contiguous)
//                          from the same swizzled layout the K tile uses
// The range's unnormalised O and (max, sum) go to the workspace and attn_combine_kernel merges
// the ranges, as for the mma.sync variant.
//
// Roles (320 threads): warp 0 loads Q once (one TMA box per d half) and K/V tiles (TMA where a
// tile is whole memory or whole local rows, cp.async otherwise) into the swizzled layout: 5
// stages, because a stage is released only when its tile's P V completes and a tile's load takes
// about 1.9 us to land, so the ring depth sets the tile period (4 stages: ~1.05 us per tile, above
// the ~0.75 us of softmax per tile); warp 1 owns TMEM (256 columns: S buffers at 0 and 64, O at 128) and issues the MMAs (one
// lane); warps 2..9 run the softmax, warps w and w + 4 on TMEM lanes 32*(w%4) .. +31, one on the
// first and one on the second 32 keys of each tile. Every mbarrier wait is bounded; on expiry the
// CTA records MSA_DEV_WAIT_TIMEOUT, leaves its loops, waits (bounded) for its own copies and MMAs
// and frees TMEM.
#include <algorithm>
#include <map>
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "mma.cuh"
#include "tc.cuh"

namespace msa {

msa_status launch_attn_tc(const void* q, const void* mem_kv, const int32_t* mem_len, int max_mem, const void* local_k,
                          const void* local_v, int L_max, int L, int q_start, int n_q, int T, int hq, int hkv,
                          float scale_log2e, int n_split, float* part_o, float2* part_ml, void* out, float* lse,
                          bool try_cluster, bool* merged, cudaStream_t s);
int attn_tc_splits(int n_q, int T, int hq, int hkv, int max_mem, int L);
msa_status attn_tc_plan(int n_q, int T, int hq, int hkv, int n_split, int* blocks, int* cluster);

namespace {

constexpr int kRows = 128;                     // MMA M, TMEM lanes: the rows of one row block
constexpr int kKeys = 64;                      // keys per tile, MMA N of S
constexpr int kD = 128;
constexpr int kThreads = 64 + 256;             // loader, MMA issuer, 8 softmax warps
constexpr int kHalfQ = kRows * 128;            // one 64-element K block of Q: 128 rows x 128 B
constexpr int kHalfKV = kKeys * 128;           // 64 rows x 128 B
constexpr int kStageBytes = 4 * kHalfKV;       // K (2 halves) + V (2 halves)
constexpr int kPBytes = kRows * 128;           // one P buffer: 128 rows x 64 keys bf16
// NH row blocks of 128 rows per CTA. NH = 1: two softmax warps per row (each on 32 keys of a tile,
// exchanging the row max); NH = 2: one softmax warp per row and both row blocks of a kv head in one
// CTA, so each K/V tile is loaded once for 256 rows.
template <int NH> struct TcShape {
    static constexpr int kSplitKeys = 3 - NH;                  // softmax warps per row
    static constexpr int kKW = kKeys / kSplitKeys;             // keys of a tile per softmax warp
    static constexpr int kOW = kD / kSplitKeys;                // O columns per softmax warp
    static constexpr int kStages = NH == 1 ? 5 : 4;
    static constexpr int kTmemCols = 256 * NH;                 // S (row block r, buffer b) at (2r + b) * 64
    static constexpr int kColO = 128 * NH;                     // O of row block r at kColO + 128 r
    static constexpr int kRedBytes = NH == 1 ? 2 * 2 * kRows * 4 : 0;   // [parity][key half][row]
    static constexpr int kSmemBytes = 1024 + NH * 2 * kHalfQ + kStages * kStageBytes + NH * kPBytes + kRedBytes + 256;
};
// A row's O is rescaled only when its running max grows by more than this (log2 units); otherwise
// the probabilities are taken against the older, smaller max (at most 2^8, exact in fp32 and as
// bf16 operands) and the final normalisation uses the same reference.
constexpr float kRescaleSlack = 8.0f;

struct AttnTcArgs {
    const __nv_bfloat16* q;
    const __nv_bfloat16* mem_kv;
    const int32_t* mem_len;
    int max_mem;
    const __nv_bfloat16* local_k;
    const __nv_bfloat16* local_v;
    int L_max, L, q_start, T, hq, hkv, G;
    float scale_log2e;
    int n_split;
    float* part_o;
    float2* part_ml;
    __nv_bfloat16* out;    // merged in the cluster: the normalised output [n_q][T][hq][d]
    float* lse;            // merged in the cluster, optional: natural-log log-sum-exp [n_q][T][hq]
    int* err;
    int use_tma;           // memory tiles by TMA from tm_mem (otherwise every tile by cp.async)
    int use_tma_loc;       // local-key tiles by TMA from tm_lk / tm_lv
};

// CL: the n_split CTAs of a (row blocks, kv head, query) form one thread-block cluster and merge
// their key ranges through distributed shared memory into the final output (no partial results in
// global memory, no combine kernel); otherwise each CTA writes its range's partial result.
template <int NH, bool CL>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                              const __grid_constant__ CUtensorMap tm_mem,
                                                              const __grid_constant__ CUtensorMap tm_lk,
                                                              const __grid_constant__ CUtensorMap tm_lv,
                                                              const AttnTcArgs a) {
    using Sh = TcShape<NH>;
    constexpr int kStages = Sh::kStages;
    constexpr int kKW = Sh::kKW;
    constexpr int kOW = Sh::kOW;
    constexpr int kColO = Sh::kColO;
    constexpr int kTmemCols = Sh::kTmemCols;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.G;
    const int split = blockIdx.x % a.n_split;
    const int r0 = (blockIdx.x / a.n_split) * (kRows * NH);
    const int qi = blockIdx.z, g = blockIdx.y;
    const int n_rows = a.T * G;
    const int mem_len = max(min(a.mem_len[qi], a.max_mem), 0);
    const int r_last = min(r0 + kRows * NH, n_rows) - 1;
    const int n_local = max(min(a.L, a.q_start + r_last / G + 1), 0);
    const int n_keys = mem_len + n_local;
    const int tiles = (n_keys + kKeys - 1) / kKeys;
    const int per = (tiles + a.n_split - 1) / a.n_split;
    const int k_begin = min(split * per, tiles) * kKeys;
    const int k_end = min(min(split * per + per, tiles) * kKeys, n_keys);
    const int n_t = k_end > k_begin ? (k_end - k_begin + kKeys - 1) / kKeys : 0;
    const int64_t rows_total = (int64_t)gridDim.z * a.T * a.hq;
    const float ninf = -__int_as_float(0x7f800000);

    if (!CL && n_t == 0) {   // an empty key range: the partial result of nothing
        if (warp >= 2) {
            const int sw = (warp - 2) >> 2;
            const int rh = NH == 2 ? sw : 0, ch = NH == 1 ? sw : 0;
            const int row = r0 + rh * kRows + (warp & 3) * 32 + lane;
            if (row < n_rows) {
                const int64_t gr = ((int64_t)qi * a.T + row / G) * a.hq + g * G + row % G;
                float4* po = reinterpret_cast<float4*>(a.part_o + ((int64_t)split * rows_total + gr) * kD);
                for (int i = 0; i < kOW / 4; ++i) po[ch * (kOW / 4) + i] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (ch == 0) a.part_ml[(int64_t)split * rows_total + gr] = make_float2(ninf, 0.f);
            }
        }
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        return;
    }

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = base;                                   // NH row blocks x 2 d-halves x 16 KB
    uint8_t* sKV = sQ + NH * 2 * kHalfQ;                  // kStages x (K 2 halves, V 2 halves)
    uint8_t* sP = sKV + kStages * kStageBytes;            // one 16 KB P buffer per row block
    float* sRed = reinterpret_cast<float*>(sP + NH * kPBytes);  // NH = 1: [2][2][128]
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sRed) + Sh::kRedBytes);
    uint64_t* kv_full = bars;                             // [kStages] loader arrival (+ TMA bytes)
    uint64_t* kv_empty = bars + kStages;                  // [kStages] MMA commit
    uint64_t* q_full = bars + 2 * kStages;                // TMA bytes of Q
    uint64_t* s_full = q_full + 1;                        // [2] MMA commit
    uint64_t* p_full = s_full + 2;                        // [2] 256 softmax arrivals (P of tile j, j & 1)
    uint64_t* o_done = p_full + 2;                        // [2] MMA commit after P V of tile j (j & 1)
    uint64_t* drain = o_done + 2;                         // MMA commit when aborting
    uint64_t* pair = drain + 1;                           // [4 quarters][2 parities] 64 arrivals
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pair + 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&kv_full[s]), 1);
            mbar_init(smem_u32(&kv_empty[s]), 1);
        }
        mbar_init(smem_u32(q_full), 1);
        mbar_init(smem_u32(&s_full[0]), 1);
        mbar_init(smem_u32(&s_full[1]), 1);
        mbar_init(smem_u32(&p_full[0]), 256);
        mbar_init(smem_u32(&p_full[1]), 256);
        mbar_init(smem_u32(&o_done[0]), 1);
        mbar_init(smem_u32(&o_done[1]), 1);
        mbar_init(smem_u32(drain), 1);
        for (int i = 0; i < 8; ++i) mbar_init(smem_u32(&pair[i]), 64);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
    // a CTA of a cluster whose key range is empty takes part in the merge with an empty partial
    const bool work = n_t > 0;

    if (warp == 0) {
        // ------------------------------------------------------------------ loader
        // A tile of 64 memory rows (or of 64 local keys) comes by TMA: four boxes of [64 keys][64 d]
        // in the 128-byte swizzle (K and V halves) on the stage's barrier with its byte count. Other
        // tiles (a tail of memory rows, a tile straddling memory and local keys or the range's end)
        // come by cp.async with zero-filled invalid rows: lane l copies 16-byte chunk c = l % 16 of
        // rows r = l / 16, l / 16 + 2, ..., then the warp waits for its copies, fences them for the
        // tensor core and lane 0 arrives.
        const int c = lane & 15, rsub = lane >> 4;
        const int cc = c & 7;
        const int hq_off = (c >> 3);
        if (lane == 0 && work) {
            // Q: per d half one box [128 / G tokens][G heads][64 d] of the 4D map over q [n_q][T][hq][d]
            // (rows r = t * G + h' land in the swizzled K-major layout; tokens past T are zero-filled);
            // issued first, so its latency overlaps the first K/V tiles'
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_q)) : "memory");
            if (a.use_tma) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_mem)) : "memory");
            mbar_expect_tx(smem_u32(q_full), (uint32_t)(NH * 2 * kHalfQ));
#pragma unroll
            for (int rh = 0; rh < NH; ++rh)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    tma_load_4d(smem_u32(sQ) + (uint32_t)((rh * 2 + h) * kHalfQ), &tm_q, h * 64, g * G,
                                (r0 + rh * kRows) / G, qi, smem_u32(q_full));
        }
        const int64_t mstride = 2LL * a.hkv * kD;                         // elements between memory rows
        const int64_t lstride = (int64_t)a.hkv * kD;                      // elements between local rows
        const __nv_bfloat16* mk0 = a.mem_kv + (int64_t)qi * a.max_mem * mstride + g * kD + c * 8;
        const __nv_bfloat16* lk0 = a.local_k + (int64_t)qi * a.L_max * lstride + g * kD + c * 8;
        const __nv_bfloat16* lv0 = a.local_v + (int64_t)qi * a.L_max * lstride + g * kD + c * 8;
        const int64_t v_in_row = (int64_t)a.hkv * kD;                     // V after K in a memory row
        int tma_phase[kStages];                                           // last TMA phase per stage, -1 none
#pragma unroll
        for (int i = 0; i < kStages; ++i) tma_phase[i] = -1;
        for (int j = 0; j < n_t; ++j) {
            const int st = j % kStages;
            if (!mbar_wait(smem_u32(&kv_empty[st]), ((uint32_t)(j / kStages) & 1u) ^ 1u, abort_flag)) break;
            const uint32_t stage = smem_u32(sKV + st * kStageBytes);
            const uint32_t full = smem_u32(&kv_full[st]);
            const int kb = k_begin + j * kKeys;
            const bool loc_tile = a.use_tma_loc && kb >= mem_len && kb + kKeys <= k_end;
            if (loc_tile) {                       // 64 local keys: K and V halves from the local caches
                if (lane == 0) {
                    mbar_expect_tx(full, (uint32_t)kStageBytes);
                    const int z = qi * a.L_max + (kb - mem_len);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        tma_load_3d(stage + h * kHalfKV, &tm_lk, h * 64, g, z, full);
                        tma_load_3d(stage + 2 * kHalfKV + h * kHalfKV, &tm_lv, h * 64, g, z, full);
                    }
                }
                tma_phase[st] = (j / kStages) & 1;
                continue;
            }
            if (a.use_tma && kb + kKeys <= mem_len) {
                if (lane == 0) {
                    mbar_expect_tx(full, (uint32_t)kStageBytes);
                    const int z = qi * a.max_mem + kb;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        tma_load_3d(stage + h * kHalfKV, &tm_mem, h * 64, g, z, full);                  // K
                        tma_load_3d(stage + 2 * kHalfKV + h * kHalfKV, &tm_mem, h * 64, a.hkv + g, z, full);  // V
                    }
                }
                tma_phase[st] = (j / kStages) & 1;
                continue;
            }
            const uint32_t sb = stage + (uint32_t)(hq_off * kHalfKV);
#pragma unroll 4
            for (int i = 0; i < kKeys / 2; ++i) {
                const int r = rsub + 2 * i;
                const int kk = kb + r;
                const bool v = kk < k_end;
                const __nv_bfloat16* ks;
                const __nv_bfloat16* vs;
                if (kk < mem_len) {
                    ks = mk0 + kk * mstride;
                    vs = ks + v_in_row;
                } else {
                    const int64_t jl = kk - mem_len;
                    ks = lk0 + jl * lstride;
                    vs = lv0 + jl * lstride;
                }
                const uint32_t d = sb + (uint32_t)(r * 128 + ((cc ^ (r & 7)) << 4));
                cp_async16_zfill(d, v ? ks : a.q, v);
                cp_async16_zfill(d + 2 * kHalfKV, v ? vs : a.q, v);
            }
            asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(full);
            tma_phase[st] = -1;
        }
        if (lane == 0 && work && *abort_flag) {
            // leave no TMA copy in flight: wait (bounded, ignoring the abort flag) for Q and the last tiles
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(smem_u32(q_full), 0) && globaltimer() - t0 < kWaitNs) {
            }
            for (int i = 0; i < kStages; ++i)
                while (tma_phase[i] >= 0 && !mbar_try_wait(smem_u32(&kv_full[i]), (uint32_t)tma_phase[i]) &&
                       globaltimer() - t0 < kWaitNs) {
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0 && work) {
            // M = 128, bf16 x bf16 -> fp32; S: N = 64, both K-major; P V: N = 128, B (V) MN-major
            const uint32_t idesc_s = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kKeys >> 3) << 17) |
                                     ((uint32_t)(kRows >> 4) << 24);
            const uint32_t idesc_o = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(kD >> 3) << 17) |
                                     ((uint32_t)(kRows >> 4) << 24);
            bool ok = mbar_wait(smem_u32(q_full), 0, abort_flag);
            bool pending = false;
            auto issue_s = [&](int j) -> bool {
                const int st = j % kStages;
                if (!mbar_wait(smem_u32(&kv_full[st]), (uint32_t)(j / kStages) & 1u, abort_flag)) return false;
                tc_fence_after();
                const uint32_t sb = smem_u32(sKV + st * kStageBytes);
#pragma unroll
                for (int rh = 0; rh < NH; ++rh) {
                    const uint32_t d_tmem = tmem_base + (uint32_t)((2 * rh + (j & 1)) * kKeys);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint64_t ad = sw128_desc(smem_u32(sQ) + (rh * 2 + h) * kHalfQ);
                        const uint64_t bd = sw128_desc(sb + h * kHalfKV);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16(d_tmem, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc_s,
                                      (h | kk) ? 1u : 0u);
                    }
                }
                pending = true;
                umma_commit(smem_u32(&s_full[j & 1]));
                return true;
            };
            if (ok) ok = issue_s(0);
            if (ok && n_t > 1) ok = issue_s(1);
            for (int j = 0; j < n_t && ok; ++j) {
                if (!mbar_wait(smem_u32(&p_full[j & 1]), ((uint32_t)j >> 1) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int st = j % kStages;
                const uint32_t vb = smem_u32(sKV + st * kStageBytes + 2 * kHalfKV);
                const uint64_t vd = sw128_mn_desc(vb, kHalfKV);
#pragma unroll
                for (int rh = 0; rh < NH; ++rh) {
                    const uint64_t pd = sw128_desc(smem_u32(sP + rh * kPBytes));
                    const uint32_t o_tmem = tmem_base + kColO + rh * 128;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)   // 16 keys per step: +32 B along P's rows, +2 KB (16 V rows)
                        umma_bf16(o_tmem, pd + (uint64_t)(kk * 2), vd + (uint64_t)(kk * (2048 >> 4)), idesc_o,
                                  (j > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(smem_u32(&kv_empty[st]));
                umma_commit(smem_u32(&o_done[j & 1]));
                pending = false;
                if (j + 2 < n_t && !issue_s(j + 2)) ok = false;
            }
            if (!ok && pending) {
                umma_commit(smem_u32(drain));
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(smem_u32(drain), 0) && globaltimer() - t0 < kWaitNs) {
                }
            }
        }
    } else {
        // ------------------------------------------------------------------ softmax
        // Two warps per TMEM lane quarter (warp w and w + 4 share lanes 32*(w%4) .. +31): warp half
        // ch takes keys ch*32 .. ch*32+31 of every tile, so each keeps half of a row's chain. Per
        // tile the pair exchanges its partial maxima through shared memory on a bounded mbarrier
        // (64 arrivals, one per tile parity) and both take the same reference max and rescale
        // decision; each keeps the sum of its own keys (added at the end) and rescales its half of
        // the O row.
        const int quarter = warp & 3;
        const int sw = (warp - 2) >> 2;
        const int rh = NH == 2 ? sw : 0;                 // row block of this warp
        const int ch = NH == 1 ? sw : 0;                 // key half of this warp (NH = 1)
        const int rl = quarter * 32 + lane;
        const int row = r0 + rh * kRows + rl;
        const bool rvalid = row < n_rows;
        const int t = rvalid ? row / G : 0;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t o_tmem = tmem_base + lane_off + kColO + rh * 128 + ch * kOW;
        float m = ninf, l = 0.f;      // reference max of the accumulated O row (log2 units), own keys' sum
        bool ok = true;
        // waits (lane 0, broadcast) on an mbarrier phase
        auto wait_bar = [&](uint64_t* bar, uint32_t parity) -> bool {
            bool w = true;
            if (lane == 0) w = mbar_wait(smem_u32(bar), parity, abort_flag);
            return __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
        };
        auto wait_pv = [&](int i) -> bool {
            const bool w = wait_bar(&o_done[i & 1], ((uint32_t)i >> 1) & 1u);
            if (w) tc_fence_after();
            return w;
        };
        // exchange e with the partner warp: writes this row's value at [e & 1][ch][rl], arrives, waits
        // (bounded) for the partner's arrival and reads its value; false when the wait gave up. The
        // warp syncs after lane 0's acquiring wait so every lane sees the partner's write.
        auto exchange = [&](float mine, int e, float* theirs) -> bool {
            sRed[((e & 1) * 2 + ch) * kRows + rl] = mine;
            mbar_arrive(smem_u32(&pair[quarter * 2 + (e & 1)]));
            if (!wait_bar(&pair[quarter * 2 + (e & 1)], ((uint32_t)e >> 1) & 1u)) return false;
            __syncwarp();
            *theirs = sRed[((e & 1) * 2 + (ch ^ 1)) * kRows + rl];
            return true;
        };
        for (int j = 0; j < n_t; ++j) {   // no tile (and no wait) when the range is empty
            if (!wait_bar(&s_full[j & 1], ((uint32_t)j >> 1) & 1u)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float s[kKW];
            if constexpr (kKW == 64)
                tmem_ld64(tmem_base + lane_off + (uint32_t)((2 * rh + (j & 1)) * kKeys), s);
            else
                tmem_ld32(tmem_base + lane_off + (uint32_t)((2 * rh + (j & 1)) * kKeys + ch * kKW), s);
            const int kb = k_begin + j * kKeys + ch * kKW;
            // masked keys to -inf where the tile needs it: inside the range and (a memory row or a
            // causal local key)
            if (!(__all_sync(0xffffffffu, rvalid) && kb + kKW <= k_end && kb + kKW <= mem_len)) {
                const int lim = mem_len + a.q_start + t;
#pragma unroll
                for (int c = 0; c < kKW; ++c) {
                    const int kk = kb + c;
                    const bool vis = rvalid & (kk < k_end) & ((kk < mem_len) | (kk <= lim));
                    s[c] = vis ? s[c] : ninf;
                }
            }
            // the max over this warp's raw scores in four chains (scale > 0 commutes with max and with
            // its rounding), then (NH = 1) the pair's
            float mx[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) mx[i] = s[i];
#pragma unroll
            for (int c = 4; c < kKW; ++c) mx[c & 3] = fmaxf(mx[c & 3], s[c]);
            mx[0] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            float other = ninf;
            if (NH == 1 && !exchange(mx[0], j, &other)) {
                ok = false;
                break;
            }
            const float mt = fmaxf(mx[0], other) * a.scale_log2e;
            // a new reference max only when the row's max grows past the slack (or on its first keys)
            float alpha = 1.f;
            bool rescale = false;
            if (mt != ninf && (m == ninf || mt > m + kRescaleSlack)) {
                rescale = m != ninf;          // an O row without any earlier key is still zero
                alpha = m == ninf ? 1.f : ex2(m - mt);
                m = mt;
            }
            // probabilities (a row without visible keys has m = -inf and gets zeros)
            const float nref = m == ninf ? 0.f : -m;
            float psum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < kKW; ++c) {
                s[c] = ex2(fmaf(s[c], a.scale_log2e, nref));
                psum[c & 3] += s[c];
            }
            l = l * alpha + ((psum[0] + psum[1]) + (psum[2] + psum[3]));
            if (__any_sync(0xffffffffu, rescale)) {
                // O holds tiles < j once the previous P V has completed; this warp's half of the row
                if (j > 0 && !wait_pv(j - 1)) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int part = 0; part < kOW / 32; ++part) {
                    float o[32];
                    tmem_ld32(o_tmem + (uint32_t)(part * 32), o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= alpha;
                    tmem_st32(o_tmem + (uint32_t)(part * 32), o);
                }
            }
            // the P buffer is free once the P V of tile j - 1 has completed
            if (j >= 1 && !wait_pv(j - 1)) {
                ok = false;
                break;
            }
            uint8_t* prow = sP + rh * kPBytes + rl * 128;
#pragma unroll
            for (int c4 = 0; c4 < kKW / 8; ++c4) {
                uint4 u;
                u.x = pack_bf16(s[c4 * 8 + 0], s[c4 * 8 + 1]);
                u.y = pack_bf16(s[c4 * 8 + 2], s[c4 * 8 + 3]);
                u.z = pack_bf16(s[c4 * 8 + 4], s[c4 * 8 + 5]);
                u.w = pack_bf16(s[c4 * 8 + 6], s[c4 * 8 + 7]);
                const int cc = ch * (kKW / 8) + c4;
                *reinterpret_cast<uint4*>(prow + ((cc ^ (rl & 7)) << 4)) = u;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            mbar_arrive(smem_u32(&p_full[j & 1]));
        }
        if (ok && work) ok = wait_pv(n_t - 1);
        float l_other = 0.f;
        if (NH == 1 && ok) ok = exchange(l, n_t, &l_other);
        if (CL) {
            // stage this range's partial in shared memory for the cluster's merge: O rows (fp32,
            // 512 B, 16-byte chunk c stored at chunk c ^ (row % 32), so the 32 lanes' rows of a warp
            // store hit distinct banks) in the idle K/V ring, (max, sum) per row in the idle P
            // buffer; an empty or abandoned range stages (-inf, 0) and no O
            const int rr = rh * kRows + rl;
            float* st_row = reinterpret_cast<float*>(sKV) + rr * kD;
            if (ok && work) {
                float o[kOW];
                if constexpr (kOW == 128) tmem_ld128(o_tmem, o); else tmem_ld64(o_tmem, o);
#pragma unroll
                for (int i = 0; i < kOW / 4; ++i) {
                    const int chunk = ch * (kOW / 4) + i;
                    *reinterpret_cast<float4*>(st_row + ((chunk ^ (rr & 31)) << 2)) =
                        make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
                }
            }
            if (ch == 0)
                reinterpret_cast<float2*>(sP)[rr] = (ok && work) ? make_float2(m, l + l_other) : make_float2(ninf, 0.f);
        } else if (ok) {
            // The range's unnormalised O rows, 32 columns at a time: TMEM -> registers (a row per
            // lane) -> this warp's slot of the (now idle) K/V ring, [32 rows][36 floats] -> global,
            // eight lanes per 128-byte row piece, so each store instruction writes four whole
            // 128-byte pieces instead of 32 scattered 16-byte ones.
            float* slot = reinterpret_cast<float*>(sKV) + (warp - 2) * (32 * 36);
            const int rsub = lane >> 3, c4 = lane & 7;
            float oall[kOW];
            if constexpr (kOW == 128) tmem_ld128(o_tmem, oall); else tmem_ld64(o_tmem, oall);
#pragma unroll
            for (int part = 0; part < kOW / 32; ++part) {
                const float* o = oall + part * 32;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    *reinterpret_cast<float4*>(slot + lane * 36 + 4 * i) =
                        make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
                __syncwarp();
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const int r = it * 4 + rsub;                          // row of this warp's 32
                    const int row_r = r0 + rh * kRows + quarter * 32 + r;
                    if (row_r < n_rows) {
                        const int64_t gr_r = ((int64_t)qi * a.T + row_r / G) * a.hq + g * G + row_r % G;
                        float* dst = a.part_o + ((int64_t)split * rows_total + gr_r) * kD + ch * kOW + part * 32;
                        *reinterpret_cast<float4*>(dst + 4 * c4) = *reinterpret_cast<const float4*>(slot + r * 36 + 4 * c4);
                    }
                }
                __syncwarp();
            }
            // both warps hold the same m; the row's sum is the two halves' (added in key-half order)
            const int64_t gr = ((int64_t)qi * a.T + t) * a.hq + g * G + (rvalid ? row % G : 0);
            if (rvalid && ch == 0) a.part_ml[(int64_t)split * rows_total + gr] = make_float2(m, l + l_other);
        }
    }

    __syncthreads();
    // the combine pass (a programmatic dependent of this grid) may be scheduled now; it reads the
    // partial results only after this grid has completed
    if constexpr (!CL) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0 && *abort_flag) record_device_error(a.err, MSA_DEV_WAIT_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
    if constexpr (CL) {
        // ---------------------------------------------------------------- merge of the cluster's ranges
        // Every thread of every CTA passes both cluster barriers (no early exit above in this
        // variant). CTA rank k merges rows [k R, (k + 1) R) of the block: a warp per row, lane l on
        // O dims 4l .. 4l + 3, reading each range's (max, sum) and O row from that CTA's shared
        // memory: out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, M = max_s m_s (ranges with
        // m_s = -inf skipped, a row no range saw is 0), in range order.
        __syncwarp();
        cluster_sync_all();
        const int n_cl = a.n_split;
        const int rank = (int)cluster_ctarank();
        const int R = (NH * kRows + n_cl - 1) / n_cl;
        const int rr_end = min(NH * kRows, (rank + 1) * R);
        const uint32_t st_base = smem_u32(sKV), ml_base = smem_u32(sP);
        for (int rr = rank * R + warp; rr < rr_end; rr += kThreads / 32) {
            const int row_g = r0 + rr;
            if (row_g >= n_rows) break;                   // rows only grow with rr
            // every range's (max, sum) in one load per lane (lane s0 reads range s0) and every
            // range's O piece in flight at once: the remote loads do not wait on one another
            const float2 ml = lane < n_cl ? ld_cluster_f2(cluster_map(ml_base + rr * 8, (uint32_t)lane))
                                          : make_float2(ninf, 0.f);
            const uint32_t off = st_base + (uint32_t)(rr * kD * 4 + ((lane ^ (rr & 31)) << 4));
            float4 o[16];
#pragma unroll
            for (int s0 = 0; s0 < 16; ++s0)
                if (s0 < n_cl) o[s0] = ld_cluster_f4(cluster_map(off, (uint32_t)s0));
            float M = ml.x;
#pragma unroll
            for (int sh = 16; sh >= 1; sh >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, sh));
            // weights in range order; a range without keys (max -inf) staged no O and is skipped
            const float wl = (ml.x == ninf) ? 0.f : exp2f(ml.x - M);
            float acc[4] = {0.f, 0.f, 0.f, 0.f}, L = 0.f;
#pragma unroll
            for (int s0 = 0; s0 < 16; ++s0) {
                if (s0 >= n_cl) break;
                const float w = __shfl_sync(0xffffffffu, wl, s0);
                const float l_s = __shfl_sync(0xffffffffu, ml.y, s0);
                const float m_s = __shfl_sync(0xffffffffu, ml.x, s0);
                if (m_s == ninf) continue;
                L = fmaf(w, l_s, L);
                acc[0] = fmaf(w, o[s0].x, acc[0]);
                acc[1] = fmaf(w, o[s0].y, acc[1]);
                acc[2] = fmaf(w, o[s0].z, acc[2]);
                acc[3] = fmaf(w, o[s0].w, acc[3]);
            }
            const float inv = L > 0.f ? 1.f / L : 0.f;
            const int64_t gr = ((int64_t)qi * a.T + row_g / G) * a.hq + g * G + row_g % G;
            uint2 u;
            u.x = pack_bf16(acc[0] * inv, acc[1] * inv);
            u.y = pack_bf16(acc[2] * inv, acc[3] * inv);
            *reinterpret_cast<uint2*>(a.out + gr * kD + lane * 4) = u;
            if (a.lse && lane == 0) a.lse[gr] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : ninf;
        }
        __syncwarp();
        cluster_sync_all();   // no CTA leaves while another still reads its shared memory
    }
}

}  // namespace

// Row blocks per CTA: both of a kv head when it has more than 128 rows.
int attn_tc_blocks(int T, int hq, int hkv) { return T * (hq / hkv) > kRows ? 2 : 1; }

// Key ranges per (row blocks, kv head, query): one wave of one CTA per SM (148), at least four
// 64-key tiles per range.
int attn_tc_splits(int n_q, int T, int hq, int hkv, int max_mem, int L) {
    const int G = hq / hkv;
    const int rows = kRows * attn_tc_blocks(T, hq, hkv);
    const int64_t base = (int64_t)((T * G + rows - 1) / rows) * hkv * n_q;
    const int tiles = (max_mem + L + kKeys - 1) / kKeys;
    const int64_t want = 148 / std::max<int64_t>(base, 1);
    return (int)std::max<int64_t>(1, std::min<int64_t>(want, std::max(1, tiles / 4)));
}

namespace {

// Largest cluster (1 to 16 CTAs, one per key range) such that the whole grid of clusters is
// resident at once (one wave), or 0 when no cluster launch of this kernel fits.
// Opts both variants of row-block count NH into their dynamic shared memory and the cluster variant
// into clusters of up to 16 CTAs, once per device.
template <int NH>
msa_status opt_in_tc() {
    constexpr int smem = TcShape<NH>::kSmemBytes;
    static std::mutex mu;
    static int opted[64] = {0};
    int dev = 0;
    MSA_CUDA_TRY(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 0 && dev < 64 && opted[dev]) return MSA_OK;
    MSA_CUDA_TRY(cudaFuncSetAttribute(attn_tc_kernel<NH, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    MSA_CUDA_TRY(cudaFuncSetAttribute(attn_tc_kernel<NH, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    MSA_CUDA_TRY(cudaFuncSetAttribute(attn_tc_kernel<NH, true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
    if (dev >= 0 && dev < 64) opted[dev] = 1;
    return MSA_OK;
}

template <int NH>
int pick_cluster_uncached(int64_t base);

// pick_cluster_uncached asks the driver for cluster occupancy: remembered per (device, NH, base)
template <int NH>
int pick_cluster(int64_t base) {
    static std::mutex mu;
    static std::map<std::pair<int, int64_t>, int> memo;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    {
        std::lock_guard<std::mutex> lk(mu);
        auto it = memo.find({dev, base});
        if (it != memo.end()) return it->second;
    }
    const int cs = pick_cluster_uncached<NH>(base);
    std::lock_guard<std::mutex> lk(mu);
    memo[{dev, base}] = cs;
    return cs;
}

template <int NH>
int pick_cluster_uncached(int64_t base) {
    constexpr int smem = TcShape<NH>::kSmemBytes;
    if (opt_in_tc<NH>() != MSA_OK) return 0;
    for (int cs = 16; cs >= 1; --cs) {   // any size: the GPCs hold e.g. 7 clusters of 16 but 8 of 14
        if ((int64_t)cs * base > 148) continue;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)cs;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3((unsigned)(cs * base), 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, attn_tc_kernel<NH, true>, &cfg) != cudaSuccess) {
            (void)cudaGetLastError();
            continue;
        }
        if ((int64_t)n >= base) return cs;
    }
    return 0;
}

template <int NH>
msa_status launch_tc(const CUtensorMap& tq, const CUtensorMap& tm, const CUtensorMap& tlk, const CUtensorMap& tlv,
                     AttnTcArgs a, int n_q, int n_split, int cs, bool* merged, cudaStream_t s) {
    constexpr int smem = TcShape<NH>::kSmemBytes;
    const int row_blocks = (a.T * a.G + NH * kRows - 1) / (NH * kRows);
    MSA_RETURN_IF(opt_in_tc<NH>());
    *merged = false;
    if (cs >= 1) {
        a.n_split = cs;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)cs;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3((unsigned)(row_blocks * cs), (unsigned)a.hkv, (unsigned)n_q);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        MSA_CUDA_TRY(cudaLaunchKernelEx(&cfg, attn_tc_kernel<NH, true>, tq, tm, tlk, tlv, a));
        *merged = true;
        return MSA_OK;
    }
    attn_tc_kernel<NH, false><<<dim3(row_blocks * n_split, a.hkv, n_q), kThreads, smem, s>>>(tq, tm, tlk, tlv, a);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

}  // namespace

// The launch plan: row blocks per CTA (NH: 2 when the kv head has more than 128 rows) and cluster
// size (0: partial results + combine). The ranges are merged in a cluster when the whole grid of
// clusters is resident in one wave with at least 60 % of the combine layout's ranges per row block
// (measured: clusters of 2 to 5 ranges beat partials + combine by 7-13 %; on the fine stage's 8 kv
// heads the largest co-resident clusters hold 6 of its 18 ranges and lose to the combine, 37 vs 31 us).
void choose_tc_plan(int n_q, int T, int hq, int hkv, int n_split, int* nh, int* cs_out) {
    const int G = hq / hkv;
    const int NH = attn_tc_blocks(T, hq, hkv);
    const int64_t base = (int64_t)((T * G + NH * kRows - 1) / (NH * kRows)) * hkv * n_q;
    const int cs = NH == 2 ? pick_cluster<2>(base) : pick_cluster<1>(base);
    *nh = NH;
    *cs_out = (cs >= 1 && 10 * cs >= 6 * n_split) ? cs : 0;
}

msa_status attn_tc_plan(int n_q, int T, int hq, int hkv, int n_split, int* blocks, int* cluster) {
    choose_tc_plan(n_q, T, hq, hkv, n_split, blocks, cluster);
    return MSA_OK;
}

msa_status launch_attn_tc(const void* q, const void* mem_kv, const int32_t* mem_len, int max_mem, const void* local_k,
                          const void* local_v, int L_max, int L, int q_start, int n_q, int T, int hq, int hkv,
                          float scale_log2e, int n_split, float* part_o, float2* part_ml, void* out, float* lse,
                          bool try_cluster, bool* merged, cudaStream_t s) {
    static_assert(TcShape<1>::kSmemBytes <= 232448 && TcShape<2>::kSmemBytes <= 232448, "shared memory");
    AttnTcArgs a{};
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.mem_kv = static_cast<const __nv_bfloat16*>(mem_kv);
    a.mem_len = mem_len; a.max_mem = max_mem;
    a.local_k = static_cast<const __nv_bfloat16*>(local_k);
    a.local_v = static_cast<const __nv_bfloat16*>(local_v);
    a.L_max = L_max; a.L = L; a.q_start = q_start; a.T = T; a.hq = hq; a.hkv = hkv; a.G = hq / hkv;
    a.scale_log2e = scale_log2e; a.n_split = n_split; a.part_o = part_o; a.part_ml = part_ml;
    a.out = static_cast<__nv_bfloat16*>(out); a.lse = lse;
    a.err = device_error_word();
    // queries [n_q][T][hq][d]: dims (d, head, token, query), box (64, G, 128 / G, 1): one box is 128 rows
    // r = t * G + h' of kv head g in the swizzled K-major layout
    CUtensorMap tq{};
    {
        const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)hq, (uint64_t)T, (uint64_t)n_q};
        const uint64_t strides[3] = {(uint64_t)kD * 2, (uint64_t)hq * kD * 2, (uint64_t)T * hq * kD * 2};
        const uint32_t box[4] = {64, (uint32_t)a.G, (uint32_t)(kRows / a.G), 1};
        MSA_RETURN_IF(make_tensor_map_bf16(&tq, q, 4, dims, strides, box));
    }
    // memory rows [n_q * max_mem][2 (K, V)][hkv][d]: dims (d, K/V x head, row), box (64, 1, 64)
    CUtensorMap tm{};
    a.use_tma = 0;
    if (max_mem >= kKeys && mem_kv) {
        const uint64_t dims[3] = {(uint64_t)kD, 2ull * hkv, (uint64_t)n_q * max_mem};
        const uint64_t strides[2] = {(uint64_t)kD * 2, 2ull * hkv * kD * 2};
        const uint32_t box[3] = {64, 1, (uint32_t)kKeys};
        MSA_RETURN_IF(make_tensor_map_bf16(&tm, mem_kv, 3, dims, strides, box));
        a.use_tma = 1;
    }
    // local caches [n_q * L_max][hkv][d]: dims (d, head, row), box (64, 1, 64)
    CUtensorMap tlk{}, tlv{};
    a.use_tma_loc = 0;
    if (L_max >= kKeys && L > 0 && local_k && local_v) {
        const uint64_t dims[3] = {(uint64_t)kD, (uint64_t)hkv, (uint64_t)n_q * L_max};
        const uint64_t strides[2] = {(uint64_t)kD * 2, (uint64_t)hkv * kD * 2};
        const uint32_t box[3] = {64, 1, (uint32_t)kKeys};
        MSA_RETURN_IF(make_tensor_map_bf16(&tlk, local_k, 3, dims, strides, box));
        MSA_RETURN_IF(make_tensor_map_bf16(&tlv, local_v, 3, dims, strides, box));
        a.use_tma_loc = 1;
    }
    int NH = attn_tc_blocks(T, hq, hkv), cs = 0;
    if (try_cluster && out) choose_tc_plan(n_q, T, hq, hkv, n_split, &NH, &cs);
    if (NH == 2) return launch_tc<2>(tq, tm, tlk, tlv, a, n_q, n_split, cs, merged, s);
    return launch_tc<1>(tq, tm, tlk, tlv, a, n_q, n_split, cs, merged, s);
}

}  // namespace msa
