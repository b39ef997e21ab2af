// Attention backward on tcgen05 tensor cores (sm_100a, bf16 operands, fp32 accumulation in TMEM).
//
// dQ: one CTA per (128 (token, head) rows of kv head g, query). Per 64-key tile j:
//   S_j = Q K_j^T, dP_j = dO V_j^T      two MMAs (M 128, N 64, K 128) into double-buffered TMEM
//   softmax warps                       P = 2^(S scale log2e - lse) from the forward's log-sum-exp
//                                       (no running max), dS = P (dP - D) with D = rowsum(dO * O),
//                                       dS rounded to bf16 into double-buffered shared memory
//   dQ += dS_j K_j                      M 128, N 128, K 64; K_j read MN-major from its K-major tile
// dQ is scaled by the softmax scale and written once at the end (fp32).
//
// Roles (192 threads) as in the forward kernel: warp 0 loads Q and dO (cp.async, once) and K/V
// tiles (TMA for tiles of memory rows, cp.async with zero fill otherwise) into 3 stages; warp 1
// owns TMEM (512 columns: S at 0/64, dP at 128/192, dQ at 256) and issues the MMAs; warps 2..5
// each own 32 rows. Every mbarrier wait is bounded; on expiry the CTA records
// MSA_DEV_WAIT_TIMEOUT, drains its copies and MMAs and frees TMEM.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "mma.cuh"
#include "tc.cuh"

namespace msa {

namespace {

constexpr int kRows = 128;
constexpr int kKeys = 64;
constexpr int kD = 128;
constexpr int kStages = 3;
constexpr int kThreads = 192;
constexpr int kHalfR = kRows * 128;             // one 64-element half of 128 rows: 16 KB
constexpr int kHalfKV = kKeys * 128;            // 8 KB
constexpr int kStageBytes = 4 * kHalfKV;        // K halves + V halves
constexpr int kDsBytes = kRows * 128;           // dS: 128 rows x 64 keys bf16
constexpr int kTmemCols = 512;
constexpr int kColS = 0, kColDP = 128, kColDQ = 256;
constexpr int kSmemBytes = 1024 + 4 * kHalfR + kStages * kStageBytes + 2 * kDsBytes + 256;
constexpr float kLog2e = 1.4426950408889634f;

__global__ void __launch_bounds__(kThreads, 1) attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_mem,
                                                              const __grid_constant__ CUtensorMap tm_lk,
                                                              const __grid_constant__ CUtensorMap tm_lv,
                                                                     const DqTcArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.G;
    const int r0 = blockIdx.x * kRows;
    const int qi = blockIdx.z, g = blockIdx.y;
    const int n_rows = a.T * G;
    const int mem_len = max(min(a.mem_len[qi], a.max_mem), 0);
    const int r_last = min(r0 + kRows, n_rows) - 1;
    const int n_keys = mem_len + max(min(a.L, a.q_start + r_last / G + 1), 0);
    const int n_t = (n_keys + kKeys - 1) / kKeys;
    const float ninf = -__int_as_float(0x7f800000);

    if (n_t == 0) {   // no key: dq = 0
        if (warp >= 2) {
            const int row = r0 + (warp & 3) * 32 + lane;
            if (row < n_rows) {
                float4* dst = reinterpret_cast<float4*>(
                    a.dq + (((int64_t)qi * a.T + row / G) * a.hq + g * G + row % G) * kD);
                for (int i = 0; i < kD / 4; ++i) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        return;
    }

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = base;                                   // 2 halves x 16 KB
    uint8_t* sO = sQ + 2 * kHalfR;                        // dO, 2 halves x 16 KB
    uint8_t* sKV = sO + 2 * kHalfR;                       // kStages x (K halves, V halves)
    uint8_t* sDS = sKV + kStages * kStageBytes;           // 2 buffers x 16 KB
    uint64_t* bars = reinterpret_cast<uint64_t*>(sDS + 2 * kDsBytes);
    uint64_t* kv_full = bars;                             // [kStages]
    uint64_t* kv_empty = bars + kStages;                  // [kStages]
    uint64_t* q_full = bars + 2 * kStages;
    uint64_t* s_full = q_full + 1;                        // [2] S and dP of tile j in buffer j & 1
    uint64_t* ds_full = s_full + 2;                       // [2] 128 softmax arrivals
    uint64_t* dq_done = ds_full + 2;                      // [2] dQ MMA of tile j finished
    uint64_t* drain = dq_done + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&kv_full[s]), 1);
            mbar_init(smem_u32(&kv_empty[s]), 1);
        }
        mbar_init(smem_u32(q_full), 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&s_full[b]), 1);
            mbar_init(smem_u32(&ds_full[b]), 128);
            mbar_init(smem_u32(&dq_done[b]), 1);
        }
        mbar_init(smem_u32(drain), 1);
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
        const int c = lane & 15, rsub = lane >> 4;
        const int cc = c & 7;
        const int half = c >> 3;
        if (a.use_tma && lane == 0)
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_mem)) : "memory");
        for (int i = 0; i < kRows / 2; ++i) {
            const int rl = rsub + 2 * i;
            const int row = r0 + rl;
            const bool v = row < n_rows;
            const int64_t off = v ? (((int64_t)qi * a.T + row / G) * a.hq + g * G + row % G) * kD + c * 8 : 0;
            const uint32_t d = (uint32_t)(half * kHalfR + rl * 128 + ((cc ^ (rl & 7)) << 4));
            cp_async16_zfill(smem_u32(sQ) + d, v ? a.q + off : a.q, v);
            cp_async16_zfill(smem_u32(sO) + d, v ? a.dout + off : a.q, v);
        }
        asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(q_full));
        const int64_t mstride = 2LL * a.hkv * kD;
        const int64_t lstride = (int64_t)a.hkv * kD;
        const __nv_bfloat16* mk0 = a.mem_kv + (int64_t)qi * a.max_mem * mstride + g * kD + c * 8;
        const __nv_bfloat16* lk0 = a.local_k + (int64_t)qi * a.L_max * lstride + g * kD + c * 8;
        const __nv_bfloat16* lv0 = a.local_v + (int64_t)qi * a.L_max * lstride + g * kD + c * 8;
        const int64_t v_in_row = (int64_t)a.hkv * kD;
        int tma_phase[kStages];
#pragma unroll
        for (int i = 0; i < kStages; ++i) tma_phase[i] = -1;
        for (int j = 0; j < n_t; ++j) {
            const int st = j % kStages;
            if (!mbar_wait(smem_u32(&kv_empty[st]), ((uint32_t)(j / kStages) & 1u) ^ 1u, abort_flag)) break;
            const uint32_t stage = smem_u32(sKV + st * kStageBytes);
            const uint32_t full = smem_u32(&kv_full[st]);
            const int kb = j * kKeys;
            const bool loc_tile = a.use_tma_loc && kb >= mem_len && kb + kKeys <= n_keys;
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
                        tma_load_3d(stage + h * kHalfKV, &tm_mem, h * 64, g, z, full);
                        tma_load_3d(stage + 2 * kHalfKV + h * kHalfKV, &tm_mem, h * 64, a.hkv + g, z, full);
                    }
                }
                tma_phase[st] = (j / kStages) & 1;
                continue;
            }
            const uint32_t sb = stage + (uint32_t)(half * kHalfKV);
#pragma unroll 4
            for (int i = 0; i < kKeys / 2; ++i) {
                const int r = rsub + 2 * i;
                const int kk = kb + r;
                const bool v = kk < n_keys;
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
            const uint64_t t0 = globaltimer();
            for (int i = 0; i < kStages; ++i)
                while (tma_phase[i] >= 0 && !mbar_try_wait(smem_u32(&kv_full[i]), (uint32_t)tma_phase[i]) &&
                       globaltimer() - t0 < kWaitNs) {
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kKeys >> 3) << 17) |
                                     ((uint32_t)(kRows >> 4) << 24);
            const uint32_t idesc_q = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(kD >> 3) << 17) |
                                     ((uint32_t)(kRows >> 4) << 24);
            bool ok = mbar_wait(smem_u32(q_full), 0, abort_flag);
            bool pending = false;
            auto issue_sdp = [&](int j) -> bool {
                const int st = j % kStages;
                if (!mbar_wait(smem_u32(&kv_full[st]), (uint32_t)(j / kStages) & 1u, abort_flag)) return false;
                tc_fence_after();
                const uint32_t sb = smem_u32(sKV + st * kStageBytes);
                const uint32_t ts = tmem_base + kColS + (uint32_t)((j & 1) * kKeys);
                const uint32_t tp = tmem_base + kColDP + (uint32_t)((j & 1) * kKeys);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint64_t qd = sw128_desc(smem_u32(sQ) + h * kHalfR);
                    const uint64_t od = sw128_desc(smem_u32(sO) + h * kHalfR);
                    const uint64_t kd = sw128_desc(sb + h * kHalfKV);
                    const uint64_t vd = sw128_desc(sb + 2 * kHalfKV + h * kHalfKV);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        umma_bf16(ts, qd + (uint64_t)(kk * 2), kd + (uint64_t)(kk * 2), idesc_s, (h | kk) ? 1u : 0u);
                        umma_bf16(tp, od + (uint64_t)(kk * 2), vd + (uint64_t)(kk * 2), idesc_s, (h | kk) ? 1u : 0u);
                    }
                }
                pending = true;
                umma_commit(smem_u32(&s_full[j & 1]));
                return true;
            };
            if (ok) ok = issue_sdp(0);
            if (ok && n_t > 1) ok = issue_sdp(1);
            for (int j = 0; j < n_t && ok; ++j) {
                if (!mbar_wait(smem_u32(&ds_full[j & 1]), ((uint32_t)j >> 1) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int st = j % kStages;
                const uint64_t dd = sw128_desc(smem_u32(sDS + (j & 1) * kDsBytes));
                const uint64_t kmn = sw128_mn_desc(smem_u32(sKV + st * kStageBytes), kHalfKV);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)   // 16 keys per step: +32 B along dS rows, +2 KB (16 K rows)
                    umma_bf16(tmem_base + kColDQ, dd + (uint64_t)(kk * 2), kmn + (uint64_t)(kk * (2048 >> 4)), idesc_q,
                              (j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(smem_u32(&kv_empty[st]));
                umma_commit(smem_u32(&dq_done[j & 1]));
                pending = false;
                if (j + 2 < n_t && !issue_sdp(j + 2)) ok = false;
            }
            if (!ok && pending) {
                umma_commit(smem_u32(drain));
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(smem_u32(drain), 0) && globaltimer() - t0 < kWaitNs) {
                }
            }
        }
    } else {
        // ------------------------------------------------------------------ dS
        const int quarter = warp & 3;
        const int rl = quarter * 32 + lane;
        const int row = r0 + rl;
        const bool rvalid = row < n_rows;
        const int t = rvalid ? row / G : 0;
        const int64_t ri = ((int64_t)qi * a.T + t) * a.hq + g * G + (rvalid ? row % G : 0);
        const float l2 = rvalid ? a.lse[ri] * kLog2e : ninf;
        const float Dr = rvalid ? a.Dvec[ri] : 0.f;
        const bool live = rvalid & (l2 != ninf);
        const int lim = mem_len + a.q_start + t;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        bool ok = true;
        auto wait_dq = [&](int i) -> bool {
            bool w = true;
            if (lane == 0) w = mbar_wait(smem_u32(&dq_done[i & 1]), ((uint32_t)i >> 1) & 1u, abort_flag);
            w = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
            if (w) tc_fence_after();
            return w;
        };
        for (int j = 0; j < n_t; ++j) {
            if (lane == 0) ok = mbar_wait(smem_u32(&s_full[j & 1]), ((uint32_t)j >> 1) & 1u, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            tc_fence_after();
            float sv[kKeys], dp[kKeys];
            tmem_ld32(tmem_base + lane_off + kColS + (uint32_t)((j & 1) * kKeys), sv);
            tmem_ld32(tmem_base + lane_off + kColS + (uint32_t)((j & 1) * kKeys + 32), sv + 32);
            tmem_ld32(tmem_base + lane_off + kColDP + (uint32_t)((j & 1) * kKeys), dp);
            tmem_ld32(tmem_base + lane_off + kColDP + (uint32_t)((j & 1) * kKeys + 32), dp + 32);
            const int kb = j * kKeys;
#pragma unroll
            for (int c2 = 0; c2 < kKeys; ++c2) {
                const int kk = kb + c2;
                const bool vis = live & (kk < n_keys) & ((kk < mem_len) | (kk <= lim));
                const float p = ex2(vis ? sv[c2] * a.scale_log2e - l2 : ninf);
                sv[c2] = p * (dp[c2] - Dr);
            }
            // dS buffer j & 1 is free once the dQ MMA of tile j - 2 has finished
            if (j >= 2 && !wait_dq(j - 2)) {
                ok = false;
                break;
            }
            uint8_t* prow = sDS + (j & 1) * kDsBytes + rl * 128;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                uint4 u;
                u.x = pack_bf16(sv[cc * 8 + 0], sv[cc * 8 + 1]);
                u.y = pack_bf16(sv[cc * 8 + 2], sv[cc * 8 + 3]);
                u.z = pack_bf16(sv[cc * 8 + 4], sv[cc * 8 + 5]);
                u.w = pack_bf16(sv[cc * 8 + 6], sv[cc * 8 + 7]);
                *reinterpret_cast<uint4*>(prow + ((cc ^ (rl & 7)) << 4)) = u;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            mbar_arrive(smem_u32(&ds_full[j & 1]));
        }
        if (ok) ok = wait_dq(n_t - 1);
        if (ok) {
            float4* dst = reinterpret_cast<float4*>(a.dq + ri * kD);
#pragma unroll
            for (int part = 0; part < kD / 32; ++part) {
                float o[32];
                tmem_ld32(tmem_base + lane_off + kColDQ + (uint32_t)(part * 32), o);
                if (rvalid)
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[part * 8 + i] = make_float4(o[4 * i] * a.scale, o[4 * i + 1] * a.scale,
                                                        o[4 * i + 2] * a.scale, o[4 * i + 3] * a.scale);
            }
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

msa_status launch_attn_bwd_dq_tc(DqTcArgs a, int n_q, cudaStream_t s) {
    static_assert(kSmemBytes <= 232448, "shared memory");
    MSA_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes));
    CUtensorMap tm{};
    a.use_tma = 0;
    if (a.max_mem >= kKeys && a.mem_kv) {
        const uint64_t dims[3] = {(uint64_t)kD, 2ull * a.hkv, (uint64_t)n_q * a.max_mem};
        const uint64_t strides[2] = {(uint64_t)kD * 2, 2ull * a.hkv * kD * 2};
        const uint32_t box[3] = {64, 1, (uint32_t)kKeys};
        MSA_RETURN_IF(make_tensor_map_bf16(&tm, a.mem_kv, 3, dims, strides, box));
        a.use_tma = 1;
    }
    CUtensorMap tlk{}, tlv{};
    a.use_tma_loc = 0;
    if (a.L_max >= kKeys && a.L > 0 && a.local_k && a.local_v) {
        const uint64_t dims[3] = {(uint64_t)kD, (uint64_t)a.hkv, (uint64_t)n_q * a.L_max};
        const uint64_t strides[2] = {(uint64_t)kD * 2, (uint64_t)a.hkv * kD * 2};
        const uint32_t box[3] = {64, 1, (uint32_t)kKeys};
        MSA_RETURN_IF(make_tensor_map_bf16(&tlk, a.local_k, 3, dims, strides, box));
        MSA_RETURN_IF(make_tensor_map_bf16(&tlv, a.local_v, 3, dims, strides, box));
        a.use_tma_loc = 1;
    }
    const int row_blocks = (a.T * a.G + kRows - 1) / kRows;
    attn_bwd_dq_tc_kernel<<<dim3(row_blocks, a.hkv, n_q), kThreads, kSmemBytes, s>>>(tm, tlk, tlv, a);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

// ---------------------------------------------------------------------------------------------
// dK, dV: one CTA per (128 keys, kv head g, query, range of 64-row blocks). TMEM lanes are keys.
// Per block j of 64 (token, head) rows:
//   S^T_j = K Q_j^T, dP^T_j = V dO_j^T     two MMAs (M 128 keys, N 64 rows, K 128) into
//                                          double-buffered TMEM
//   softmax warps (a thread per key)       P = 2^(S scale log2e - lse) from the forward's
//                                          log-sum-exp, dS = P (dP - D); P^T and dS^T rounded to
//                                          bf16 into double-buffered shared memory (128 B per key)
//   dV += P^T dO_j, dK += dS^T Q_j          M 128, N 128 (d), K 64 (rows); dO_j and Q_j read
//                                          MN-major from their K-major tiles
// Row blocks that no key of the tile can see (causal local keys) are skipped. At the end the
// four warps read dV and dK (x scale) from TMEM, a key per thread, and write them (or the row
// range's partial). Roles (192 threads): warp 0 loads K/V once and Q/dO blocks with their per-row
// lse, D and causal limit (cp.async, 2 stages); warp 1 owns 512 TMEM columns (S 0/64, dP 128/192,
// dV 256, dK 384) and issues the MMAs; warps 2..5 own 32 keys each. Every wait is bounded.
namespace {

constexpr int kDkKeys = 128;                       // keys per CTA = MMA M
constexpr int kDkRows = 64;                        // rows per block = N of the S / dP MMAs
constexpr int kDkStages = 2;
constexpr int kDkHalfK = kDkKeys * 128;            // one 64-element half of 128 key rows: 16 KB
constexpr int kDkHalfR = kDkRows * 128;            // one half of 64 rows: 8 KB
constexpr int kDkStageBytes = 4 * kDkHalfR;        // Q halves + dO halves
constexpr int kDkOpBytes = kDkKeys * 128;          // P^T or dS^T: 128 keys x 64 rows bf16
constexpr int kDkColS = 0, kDkColDP = 128, kDkColDV = 256, kDkColDK = 384;
constexpr int kDkScalars = 3 * kDkRows * 4;        // per stage: lse * log2e, D, causal limit
constexpr int kDkSmemBytes =
    1024 + 4 * kDkHalfK + kDkStages * kDkStageBytes + 4 * kDkOpBytes + kDkStages * kDkScalars + 256;
constexpr int kDead = -0x7fffffff - 1;             // causal limit of a row that sees no key

__global__ void __launch_bounds__(kThreads, 1) attn_bwd_dkdv_tc_kernel(const DkdvTcArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.G;
    const int qi = blockIdx.z, g = blockIdx.y;
    const int tile = blockIdx.x / a.n_rsplit, split = blockIdx.x % a.n_rsplit;
    const int kb = tile * kDkKeys;
    const int mem_len = max(min(a.mem_len[qi], a.max_mem), 0);
    const int n_keys = mem_len + a.L;
    if (kb >= n_keys) return;                       // no key of this tile exists for this query
    const int n_rows = a.T * G;
    const int nb_all = (n_rows + kDkRows - 1) / kDkRows;
    // the first row that can see a key of the tile: memory keys are seen by every row, a local key
    // j by the tokens t >= j - q_start
    const int t_min = kb < mem_len ? 0 : max(kb - mem_len - a.q_start, 0);
    const int rb_first = min((t_min * G) / kDkRows, nb_all);
    const int span = nb_all - rb_first;
    const int rb0 = rb_first + (int)((int64_t)span * split / a.n_rsplit);
    const int rb1 = rb_first + (int)((int64_t)span * (split + 1) / a.n_rsplit);
    const int nb = rb1 - rb0;
    const float ninf = -__int_as_float(0x7f800000);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sK = base;                                   // 2 halves x 16 KB
    uint8_t* sV = sK + 2 * kDkHalfK;                      // 2 halves x 16 KB
    uint8_t* sQO = sV + 2 * kDkHalfK;                     // kDkStages x (Q halves, dO halves)
    uint8_t* sP = sQO + kDkStages * kDkStageBytes;        // 2 buffers x 16 KB
    uint8_t* sDS = sP + 2 * kDkOpBytes;                   // 2 buffers x 16 KB
    float* sScal = reinterpret_cast<float*>(sDS + 2 * kDkOpBytes);   // [kDkStages][3][64]
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sScal) + kDkStages * kDkScalars);
    uint64_t* kv_full = bars;                             // K and V tiles loaded
    uint64_t* q_full = bars + 1;                          // [kDkStages]
    uint64_t* q_empty = q_full + kDkStages;               // [kDkStages]
    uint64_t* s_full = q_empty + kDkStages;               // [2]
    uint64_t* p_full = s_full + 2;                        // [2] 128 softmax arrivals
    uint64_t* mm_done = p_full + 2;                       // [2] dV / dK MMAs of block j finished
    uint64_t* acc_done = mm_done + 2;
    uint64_t* drain = acc_done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(kv_full), 1);
        for (int s = 0; s < kDkStages; ++s) {
            mbar_init(smem_u32(&q_full[s]), 1);
            mbar_init(smem_u32(&q_empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&s_full[b]), 1);
            mbar_init(smem_u32(&p_full[b]), 128);
            mbar_init(smem_u32(&mm_done[b]), 1);
        }
        mbar_init(smem_u32(acc_done), 1);
        mbar_init(smem_u32(drain), 1);
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
        const int c = lane & 15, rsub = lane >> 4;
        const int cc = c & 7;
        const int half = c >> 3;
        if (nb > 0) {
            const int64_t mstride = 2LL * a.hkv * kD;
            const int64_t lstride = (int64_t)a.hkv * kD;
            for (int i = 0; i < kDkKeys / 2; ++i) {
                const int r = rsub + 2 * i;
                const int kk = kb + r;
                const bool v = kk < n_keys;
                const __nv_bfloat16* ks = a.q;
                const __nv_bfloat16* vs = a.q;
                if (v) {
                    if (kk < mem_len) {
                        ks = a.mem_kv + (int64_t)qi * a.max_mem * mstride + kk * mstride + g * kD + c * 8;
                        vs = ks + (int64_t)a.hkv * kD;
                    } else {
                        const int64_t jl = (int64_t)qi * a.L_max + (kk - mem_len);
                        ks = a.local_k + jl * lstride + g * kD + c * 8;
                        vs = a.local_v + jl * lstride + g * kD + c * 8;
                    }
                }
                const uint32_t d = (uint32_t)(half * kDkHalfK + r * 128 + ((cc ^ (r & 7)) << 4));
                cp_async16_zfill(smem_u32(sK) + d, ks, v);
                cp_async16_zfill(smem_u32(sV) + d, vs, v);
            }
            asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(kv_full));
        }
        for (int j = 0; j < nb; ++j) {
            const int st = j % kDkStages;
            bool ok = true;
            if (lane == 0)
                ok = mbar_wait(smem_u32(&q_empty[st]), ((uint32_t)(j / kDkStages) & 1u) ^ 1u, abort_flag);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
            const int row0 = (rb0 + j) * kDkRows;
            uint8_t* sq = sQO + st * kDkStageBytes;
            for (int i = 0; i < kDkRows / 2; ++i) {
                const int rl = rsub + 2 * i;
                const int row = row0 + rl;
                const bool v = row < n_rows;
                const int64_t off = v ? (((int64_t)qi * a.T + row / G) * a.hq + g * G + row % G) * kD + c * 8 : 0;
                const uint32_t d = (uint32_t)(half * kDkHalfR + rl * 128 + ((cc ^ (rl & 7)) << 4));
                cp_async16_zfill(smem_u32(sq) + d, v ? a.q + off : a.q, v);
                cp_async16_zfill(smem_u32(sq + 2 * kDkHalfR) + d, v ? a.dout + off : a.q, v);
            }
            // per-row scalars: lse * log2e, D, and the last local key the row sees (kDead: none)
            float* sc = sScal + st * (kDkScalars / 4);
            for (int rl = lane; rl < kDkRows; rl += 32) {
                const int row = row0 + rl;
                float l2 = ninf, Dr = 0.f;
                int lim = kDead;
                if (row < n_rows) {
                    const int t = row / G;
                    const int64_t ri = ((int64_t)qi * a.T + t) * a.hq + g * G + row % G;
                    l2 = a.lse[ri] * kLog2e;
                    Dr = a.Dvec[ri];
                    if (l2 != ninf) lim = mem_len + a.q_start + t;
                }
                sc[rl] = l2;
                sc[kDkRows + rl] = Dr;
                reinterpret_cast<int*>(sc)[2 * kDkRows + rl] = lim;
            }
            asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&q_full[st]));
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0 && nb > 0) {
            const uint32_t idesc_s = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kDkRows >> 3) << 17) |
                                     ((uint32_t)(kDkKeys >> 4) << 24);
            const uint32_t idesc_g = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(kD >> 3) << 17) |
                                     ((uint32_t)(kDkKeys >> 4) << 24);
            bool ok = mbar_wait(smem_u32(kv_full), 0, abort_flag);
            bool pending = false;
            auto issue_sdp = [&](int j) -> bool {
                const int st = j % kDkStages;
                if (!mbar_wait(smem_u32(&q_full[st]), (uint32_t)(j / kDkStages) & 1u, abort_flag)) return false;
                tc_fence_after();
                const uint32_t sq = smem_u32(sQO + st * kDkStageBytes);
                const uint32_t ts = tmem_base + kDkColS + (uint32_t)((j & 1) * kDkRows);
                const uint32_t tp = tmem_base + kDkColDP + (uint32_t)((j & 1) * kDkRows);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint64_t kd = sw128_desc(smem_u32(sK) + h * kDkHalfK);
                    const uint64_t vd = sw128_desc(smem_u32(sV) + h * kDkHalfK);
                    const uint64_t qd = sw128_desc(sq + h * kDkHalfR);
                    const uint64_t od = sw128_desc(sq + 2 * kDkHalfR + h * kDkHalfR);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        umma_bf16(ts, kd + (uint64_t)(kk * 2), qd + (uint64_t)(kk * 2), idesc_s, (h | kk) ? 1u : 0u);
                        umma_bf16(tp, vd + (uint64_t)(kk * 2), od + (uint64_t)(kk * 2), idesc_s, (h | kk) ? 1u : 0u);
                    }
                }
                pending = true;
                umma_commit(smem_u32(&s_full[j & 1]));
                return true;
            };
            if (ok) ok = issue_sdp(0);
            if (ok && nb > 1) ok = issue_sdp(1);
            for (int j = 0; j < nb && ok; ++j) {
                if (!mbar_wait(smem_u32(&p_full[j & 1]), ((uint32_t)j >> 1) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int st = j % kDkStages;
                const uint32_t sq = smem_u32(sQO + st * kDkStageBytes);
                const uint64_t pd = sw128_desc(smem_u32(sP + (j & 1) * kDkOpBytes));
                const uint64_t dsd = sw128_desc(smem_u32(sDS + (j & 1) * kDkOpBytes));
                const uint64_t qmn = sw128_mn_desc(sq, kDkHalfR);
                const uint64_t omn = sw128_mn_desc(sq + 2 * kDkHalfR, kDkHalfR);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {   // 16 rows per step: +32 B along P^T rows, +2 KB (16 rows)
                    const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
                    umma_bf16(tmem_base + kDkColDV, pd + (uint64_t)(kk * 2), omn + (uint64_t)(kk * (2048 >> 4)),
                              idesc_g, acc);
                    umma_bf16(tmem_base + kDkColDK, dsd + (uint64_t)(kk * 2), qmn + (uint64_t)(kk * (2048 >> 4)),
                              idesc_g, acc);
                }
                umma_commit(smem_u32(&q_empty[st]));
                umma_commit(smem_u32(&mm_done[j & 1]));
                pending = false;
                if (j + 2 < nb && !issue_sdp(j + 2)) ok = false;
            }
            if (ok) {
                umma_commit(smem_u32(acc_done));
            } else if (pending) {
                umma_commit(smem_u32(drain));
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(smem_u32(drain), 0) && globaltimer() - t0 < kWaitNs) {
                }
            }
        }
    } else {
        // ------------------------------------------------------------------ P, dS and the epilogue
        const int quarter = warp & 3;
        const int kl = quarter * 32 + lane;             // key within the tile = TMEM lane
        const int kk = kb + kl;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        bool ok = true;
        auto wait_mm = [&](int i) -> bool {
            bool w = true;
            if (lane == 0) w = mbar_wait(smem_u32(&mm_done[i & 1]), ((uint32_t)i >> 1) & 1u, abort_flag);
            w = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
            if (w) tc_fence_after();
            return w;
        };
        for (int j = 0; j < nb; ++j) {
            if (lane == 0) ok = mbar_wait(smem_u32(&s_full[j & 1]), ((uint32_t)j >> 1) & 1u, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            tc_fence_after();
            float sv[kDkRows], dp[kDkRows];
            tmem_ld32(tmem_base + lane_off + kDkColS + (uint32_t)((j & 1) * kDkRows), sv);
            tmem_ld32(tmem_base + lane_off + kDkColS + (uint32_t)((j & 1) * kDkRows + 32), sv + 32);
            tmem_ld32(tmem_base + lane_off + kDkColDP + (uint32_t)((j & 1) * kDkRows), dp);
            tmem_ld32(tmem_base + lane_off + kDkColDP + (uint32_t)((j & 1) * kDkRows + 32), dp + 32);
            const float* sc = sScal + (j % kDkStages) * (kDkScalars / 4);
            const int* slim = reinterpret_cast<const int*>(sc) + 2 * kDkRows;
            const bool is_mem = kk < mem_len, is_key = kk < n_keys;
#pragma unroll
            for (int c2 = 0; c2 < kDkRows; ++c2) {
                const int lim = slim[c2];
                const bool vis = (lim != kDead) & (is_mem | (is_key & (kk <= lim)));
                const float p = ex2(vis ? sv[c2] * a.scale_log2e - sc[c2] : ninf);
                sv[c2] = p;
                dp[c2] = p * (dp[c2] - sc[kDkRows + c2]);
            }
            // P / dS buffer j & 1 is free once the dV / dK MMAs of block j - 2 have finished
            if (j >= 2 && !wait_mm(j - 2)) {
                ok = false;
                break;
            }
            uint8_t* prow = sP + (j & 1) * kDkOpBytes + kl * 128;
            uint8_t* drow = sDS + (j & 1) * kDkOpBytes + kl * 128;
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
                uint4 u, w;
                u.x = pack_bf16(sv[c8 * 8 + 0], sv[c8 * 8 + 1]);
                u.y = pack_bf16(sv[c8 * 8 + 2], sv[c8 * 8 + 3]);
                u.z = pack_bf16(sv[c8 * 8 + 4], sv[c8 * 8 + 5]);
                u.w = pack_bf16(sv[c8 * 8 + 6], sv[c8 * 8 + 7]);
                w.x = pack_bf16(dp[c8 * 8 + 0], dp[c8 * 8 + 1]);
                w.y = pack_bf16(dp[c8 * 8 + 2], dp[c8 * 8 + 3]);
                w.z = pack_bf16(dp[c8 * 8 + 4], dp[c8 * 8 + 5]);
                w.w = pack_bf16(dp[c8 * 8 + 6], dp[c8 * 8 + 7]);
                const uint32_t o = (uint32_t)((c8 ^ (kl & 7)) << 4);
                *reinterpret_cast<uint4*>(prow + o) = u;
                *reinterpret_cast<uint4*>(drow + o) = w;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            mbar_arrive(smem_u32(&p_full[j & 1]));
        }
        bool have = false;
        if (ok && nb > 0) {
            bool w = true;
            if (lane == 0) w = mbar_wait(smem_u32(acc_done), 0, abort_flag);
            have = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
            if (have) tc_fence_after();
            ok = have;
        }
        // warp-uniform: the TMEM loads below are warp-collective, only the stores depend on the key
        const bool go = __shfl_sync(0xffffffffu, (ok && *abort_flag == 0) ? 1 : 0, 0) != 0;
        if (go) {
            // gradients of this key (zero when no row block was left to this range)
            const bool key_ok = kk < n_keys;
            float* outk = nullptr;
            float* outv = nullptr;
            if (!key_ok) {
            } else if (a.n_rsplit > 1) {
                outk = a.part_dkv + ((((int64_t)split * gridDim.z + qi) * a.key_pad + kk) * 2) * a.hkv * kD + g * kD;
                outv = outk + (int64_t)a.hkv * kD;
            } else if (kk < mem_len) {
                outk = a.dmem + (((int64_t)qi * a.max_mem + kk) * 2) * a.hkv * kD + g * kD;
                outv = outk + (int64_t)a.hkv * kD;
            } else {
                const int64_t jl = (int64_t)qi * a.L_max + (kk - mem_len);
                outk = a.dlk + (jl * a.hkv + g) * kD;
                outv = a.dlv + (jl * a.hkv + g) * kD;
            }
#pragma unroll
            for (int part = 0; part < kD / 32; ++part) {
                float vv[32], kv[32];
                if (have) {
                    tmem_ld32(tmem_base + lane_off + kDkColDV + (uint32_t)(part * 32), vv);
                    tmem_ld32(tmem_base + lane_off + kDkColDK + (uint32_t)(part * 32), kv);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) vv[i] = kv[i] = 0.f;
                }
                if (key_ok) {
                    float4* dv4 = reinterpret_cast<float4*>(outv + part * 32);
                    float4* dk4 = reinterpret_cast<float4*>(outk + part * 32);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        dv4[i] = make_float4(vv[4 * i], vv[4 * i + 1], vv[4 * i + 2], vv[4 * i + 3]);
                        dk4[i] = make_float4(kv[4 * i] * a.scale, kv[4 * i + 1] * a.scale, kv[4 * i + 2] * a.scale,
                                             kv[4 * i + 3] * a.scale);
                    }
                }
            }
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

msa_status launch_attn_bwd_dkdv_tc(const DkdvTcArgs& a, int n_q, cudaStream_t s) {
    static_assert(kDkSmemBytes <= 232448, "shared memory");
    const int key_tiles = (a.max_mem + a.L + kDkKeys - 1) / kDkKeys;
    if (key_tiles == 0) return MSA_OK;
    if ((int64_t)key_tiles * a.n_rsplit > 0x7fffffff)
        return set_error(MSA_ERR_UNSUPPORTED, "attention backward (tensor cores): too many key tiles");
    MSA_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kDkSmemBytes));
    attn_bwd_dkdv_tc_kernel<<<dim3(key_tiles * a.n_rsplit, a.hkv, n_q), kThreads, kDkSmemBytes, s>>>(a);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

}  // namespace msa
