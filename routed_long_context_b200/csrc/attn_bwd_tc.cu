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

}  // namespace msa
