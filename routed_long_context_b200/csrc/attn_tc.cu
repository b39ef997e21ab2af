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

#include "common.cuh"
#include "kernels.cuh"
#include "mma.cuh"
#include "tc.cuh"

namespace msa {

msa_status launch_attn_tc(const void* q, const void* mem_kv, const int32_t* mem_len, int max_mem, const void* local_k,
                          const void* local_v, int L_max, int L, int q_start, int n_q, int T, int hq, int hkv,
                          float scale_log2e, int n_split, float* part_o, float2* part_ml, cudaStream_t s);
int attn_tc_splits(int n_q, int T, int hq, int hkv, int max_mem, int L);

namespace {

constexpr int kRows = 128;                     // MMA M, TMEM lanes
constexpr int kKeys = 64;                      // keys per tile, MMA N of S
constexpr int kHalfKeys = kKeys / 2;           // keys of a tile per softmax warp
constexpr int kD = 128;
constexpr int kStages = 5;
constexpr int kThreads = 64 + 256;             // loader, MMA issuer, 8 softmax warps
constexpr int kHalfQ = kRows * 128;            // one 64-element K block of Q: 128 rows x 128 B
constexpr int kHalfKV = kKeys * 128;           // 64 rows x 128 B
constexpr int kStageBytes = 4 * kHalfKV;       // K (2 halves) + V (2 halves)
constexpr int kPBytes = kRows * 128;           // one P buffer: 128 rows x 64 keys bf16
constexpr int kTmemCols = 256;                 // S buffers at 0 and 64, O at 128
constexpr int kColO = 2 * kKeys;
constexpr int kRedBytes = 2 * 2 * kRows * 4;   // [tile parity][key half][row] partial maxima / sums
constexpr int kSmemBytes = 1024 + 2 * kHalfQ + kStages * kStageBytes + kPBytes + kRedBytes + 256;
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
    int* err;
    int use_tma;           // memory tiles by TMA from tm_mem (otherwise every tile by cp.async)
    int use_tma_loc;       // local-key tiles by TMA from tm_lk / tm_lv
};

__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                              const __grid_constant__ CUtensorMap tm_mem,
                                                              const __grid_constant__ CUtensorMap tm_lk,
                                                              const __grid_constant__ CUtensorMap tm_lv,
                                                              const AttnTcArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.G;
    const int split = blockIdx.x % a.n_split;
    const int r0 = (blockIdx.x / a.n_split) * kRows;
    const int qi = blockIdx.z, g = blockIdx.y;
    const int n_rows = a.T * G;
    const int mem_len = max(min(a.mem_len[qi], a.max_mem), 0);
    const int r_last = min(r0 + kRows, n_rows) - 1;
    const int n_local = max(min(a.L, a.q_start + r_last / G + 1), 0);
    const int n_keys = mem_len + n_local;
    const int tiles = (n_keys + kKeys - 1) / kKeys;
    const int per = (tiles + a.n_split - 1) / a.n_split;
    const int k_begin = min(split * per, tiles) * kKeys;
    const int k_end = min(min(split * per + per, tiles) * kKeys, n_keys);
    const int n_t = k_end > k_begin ? (k_end - k_begin + kKeys - 1) / kKeys : 0;
    const int64_t rows_total = (int64_t)gridDim.z * a.T * a.hq;
    const float ninf = -__int_as_float(0x7f800000);

    if (n_t == 0) {   // an empty key range: the partial result of nothing
        if (warp >= 2) {
            const int ch = (warp - 2) >> 2;   // half of the O row this warp writes
            const int row = r0 + (warp & 3) * 32 + lane;
            if (row < n_rows) {
                const int64_t gr = ((int64_t)qi * a.T + row / G) * a.hq + g * G + row % G;
                float4* po = reinterpret_cast<float4*>(a.part_o + ((int64_t)split * rows_total + gr) * kD);
                for (int i = 0; i < kD / 8; ++i) po[ch * (kD / 8) + i] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (ch == 0) a.part_ml[(int64_t)split * rows_total + gr] = make_float2(ninf, 0.f);
            }
        }
        return;
    }

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = base;                                   // 2 d-halves x 16 KB
    uint8_t* sKV = sQ + 2 * kHalfQ;                       // kStages x (K 2 halves, V 2 halves)
    uint8_t* sP = sKV + kStages * kStageBytes;            // one 16 KB P buffer
    float* sRed = reinterpret_cast<float*>(sP + kPBytes);  // [2][2][128]
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sRed) + kRedBytes);
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
        if (lane == 0) {
            // Q: per d half one box [128 / G tokens][G heads][64 d] of the 4D map over q [n_q][T][hq][d]
            // (rows r = t * G + h' land in the swizzled K-major layout; tokens past T are zero-filled);
            // issued first, so its latency overlaps the first K/V tiles'
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_q)) : "memory");
            if (a.use_tma) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_mem)) : "memory");
            mbar_expect_tx(smem_u32(q_full), (uint32_t)(2 * kHalfQ));
#pragma unroll
            for (int h = 0; h < 2; ++h)
                tma_load_4d(smem_u32(sQ) + (uint32_t)(h * kHalfQ), &tm_q, h * 64, g * G, r0 / G, qi, smem_u32(q_full));
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
        if (lane == 0 && *abort_flag) {
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
        if (lane == 0) {
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
                const uint32_t d_tmem = tmem_base + (uint32_t)((j & 1) * kKeys);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint64_t ad = sw128_desc(smem_u32(sQ) + h * kHalfQ);
                    const uint64_t bd = sw128_desc(sb + h * kHalfKV);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(d_tmem, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc_s, (h | kk) ? 1u : 0u);
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
                const uint64_t pd = sw128_desc(smem_u32(sP));
                const uint64_t vd = sw128_mn_desc(vb, kHalfKV);
                const uint32_t o_tmem = tmem_base + kColO;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)   // 16 keys per step: +32 B along P's rows, +2 KB (16 V rows)
                    umma_bf16(o_tmem, pd + (uint64_t)(kk * 2), vd + (uint64_t)(kk * (2048 >> 4)), idesc_o,
                              (j > 0 || kk > 0) ? 1u : 0u);
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
        const int ch = (warp - 2) >> 2;
        const int rl = quarter * 32 + lane;
        const int row = r0 + rl;
        const bool rvalid = row < n_rows;
        const int t = rvalid ? row / G : 0;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t o_tmem = tmem_base + lane_off + kColO + ch * (kD / 2);
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
        for (int j = 0; j < n_t; ++j) {
            if (!wait_bar(&s_full[j & 1], ((uint32_t)j >> 1) & 1u)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float s[kHalfKeys];
            tmem_ld32(tmem_base + lane_off + (uint32_t)((j & 1) * kKeys + ch * kHalfKeys), s);
            const int kb = k_begin + j * kKeys + ch * kHalfKeys;
            // masked keys to -inf where the tile needs it: inside the range and (a memory row or a
            // causal local key)
            if (!(__all_sync(0xffffffffu, rvalid) && kb + kHalfKeys <= k_end && kb + kHalfKeys <= mem_len)) {
                const int lim = mem_len + a.q_start + t;
#pragma unroll
                for (int c = 0; c < kHalfKeys; ++c) {
                    const int kk = kb + c;
                    const bool vis = rvalid & (kk < k_end) & ((kk < mem_len) | (kk <= lim));
                    s[c] = vis ? s[c] : ninf;
                }
            }
            // the half tile's max over the raw scores in four chains (scale > 0 commutes with max and
            // with its rounding), then the pair's
            float mx[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) mx[i] = s[i];
#pragma unroll
            for (int c = 4; c < kHalfKeys; ++c) mx[c & 3] = fmaxf(mx[c & 3], s[c]);
            mx[0] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            float other = ninf;
            if (!exchange(mx[0], j, &other)) {
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
            for (int c = 0; c < kHalfKeys; ++c) {
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
                for (int part = 0; part < kD / 64; ++part) {
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
            uint8_t* prow = sP + rl * 128;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                uint4 u;
                u.x = pack_bf16(s[c4 * 8 + 0], s[c4 * 8 + 1]);
                u.y = pack_bf16(s[c4 * 8 + 2], s[c4 * 8 + 3]);
                u.z = pack_bf16(s[c4 * 8 + 4], s[c4 * 8 + 5]);
                u.w = pack_bf16(s[c4 * 8 + 6], s[c4 * 8 + 7]);
                const int cc = ch * 4 + c4;
                *reinterpret_cast<uint4*>(prow + ((cc ^ (rl & 7)) << 4)) = u;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            mbar_arrive(smem_u32(&p_full[j & 1]));
        }
        if (ok) ok = wait_pv(n_t - 1);
        float l_other = 0.f;
        if (ok) ok = exchange(l, n_t, &l_other);
        if (ok) {
            const int64_t gr = ((int64_t)qi * a.T + t) * a.hq + g * G + (rvalid ? row % G : 0);
            float4* po = reinterpret_cast<float4*>(a.part_o + ((int64_t)split * rows_total + gr) * kD);
#pragma unroll
            for (int part = 0; part < kD / 64; ++part) {
                float o[32];
                tmem_ld32(o_tmem + (uint32_t)(part * 32), o);
                if (rvalid)
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        po[(ch * 2 + part) * 8 + i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
            }
            // both warps hold the same m; the row's sum is the two halves' (added in key-half order)
            if (rvalid && ch == 0) a.part_ml[(int64_t)split * rows_total + gr] = make_float2(m, l + l_other);
        }
    }

    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) record_device_error(a.err, MSA_DEV_WAIT_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace

// Key ranges per (128-row block, kv head, query): one wave of one CTA per SM (148), at least four
// 64-key tiles per range.
int attn_tc_splits(int n_q, int T, int hq, int hkv, int max_mem, int L) {
    const int G = hq / hkv;
    const int64_t base = (int64_t)((T * G + kRows - 1) / kRows) * hkv * n_q;
    const int tiles = (max_mem + L + kKeys - 1) / kKeys;
    const int64_t want = 148 / std::max<int64_t>(base, 1);
    return (int)std::max<int64_t>(1, std::min<int64_t>(want, std::max(1, tiles / 4)));
}

msa_status launch_attn_tc(const void* q, const void* mem_kv, const int32_t* mem_len, int max_mem, const void* local_k,
                          const void* local_v, int L_max, int L, int q_start, int n_q, int T, int hq, int hkv,
                          float scale_log2e, int n_split, float* part_o, float2* part_ml, cudaStream_t s) {
    static_assert(kSmemBytes <= 232448, "shared memory");
    AttnTcArgs a{};
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.mem_kv = static_cast<const __nv_bfloat16*>(mem_kv);
    a.mem_len = mem_len; a.max_mem = max_mem;
    a.local_k = static_cast<const __nv_bfloat16*>(local_k);
    a.local_v = static_cast<const __nv_bfloat16*>(local_v);
    a.L_max = L_max; a.L = L; a.q_start = q_start; a.T = T; a.hq = hq; a.hkv = hkv; a.G = hq / hkv;
    a.scale_log2e = scale_log2e; a.n_split = n_split; a.part_o = part_o; a.part_ml = part_ml;
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
    MSA_CUDA_TRY(cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes));
    const int row_blocks = (T * a.G + kRows - 1) / kRows;
    attn_tc_kernel<<<dim3(row_blocks * n_split, hkv, n_q), kThreads, kSmemBytes, s>>>(tq, tm, tlk, tlv, a);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

}  // namespace msa
