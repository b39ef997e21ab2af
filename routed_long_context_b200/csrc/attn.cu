// Sparse attention of query tokens over [selected memory K-bar/V-bar ; causal local K/V].
//
// One block per (8 query tokens, kv head g, query q); warp w owns token t0 + w and the G query
// heads that share kv head g (GQA), so each key/value tile staged in shared memory serves 8 x G
// query rows. Keys go through in tiles of 32: lane r scores key r of the tile against the G
// heads (q and K from shared memory, K rows padded to 129 floats so the 32 lanes hit 32 banks),
// then an online softmax (running max and sum per head, exp2 with log2(e) folded into q) and
// the P.V update, where lane r owns output dims 4r..4r+3. Arithmetic and softmax in fp32.
#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "mma.cuh"

namespace msa {

msa_status launch_attn_tc(const void* q, const void* mem_kv, const int32_t* mem_len, int max_mem, const void* local_k,
                          const void* local_v, int L_max, int L, int q_start, int n_q, int T, int hq, int hkv,
                          float scale_log2e, int n_split, float* part_o, float2* part_ml, void* out, float* lse,
                          bool try_cluster, bool* merged, cudaStream_t s);
int attn_tc_splits(int n_q, int T, int hq, int hkv, int max_mem, int L);
msa_status attn_tc_plan(int n_q, int T, int hq, int hkv, int n_split, int* blocks, int* cluster);

namespace {

constexpr int kD = 128;
// bf16: 0 = default (split variant on tcgen05, plain on mma.sync), 1 = CUDA cores for the plain
// variant, 2 = mma.sync for both
std::atomic<int> g_attn_impl{0};
constexpr int kTokPerBlock = 8;
constexpr int kKeyTile = 32;

struct AttnArgs {
    const void* q;
    const void* mem_kv;
    const int32_t* mem_len;
    int max_mem;
    const void* local_k;
    const void* local_v;
    int L_max, L, q_start;
    int T, hq, hkv;
    float scale_log2e;
    void* out;
    int n_split;       // split-KV variant: key ranges per (row block, kv head, query)
    float* part_o;     // [n_split][n_q * T * hq][d] unnormalised outputs
    float2* part_ml;   // [n_split][n_q * T * hq] (running max in log2 units, sum of weights)
    float* lse;        // split variant, optional: [n_q * T * hq] natural-log log-sum-exp of the logits
};

template <typename T>
__device__ __forceinline__ void store4(T* p, const float* v) {
    if constexpr (sizeof(T) == 4) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else {
        __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
        __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t*>(&a);
        u.y = *reinterpret_cast<uint32_t*>(&b);
        *reinterpret_cast<uint2*>(p) = u;
    }
}

template <typename T, int G>
__global__ void __launch_bounds__(kTokPerBlock * 32) attn_kernel(const AttnArgs a) {
    constexpr int VEC = 16 / sizeof(T);
    // dynamic shared memory: Ks [32][129] | Vs [32][128] | Qs [8][G][128] (fp32)
    extern __shared__ __align__(16) float smem_f[];
    float(*Ks)[kD + 1] = reinterpret_cast<float(*)[kD + 1]>(smem_f);
    float(*Vs)[kD] = reinterpret_cast<float(*)[kD]>(smem_f + kKeyTile * (kD + 1));
    float(*Qs)[G][kD] = reinterpret_cast<float(*)[G][kD]>(smem_f + kKeyTile * (kD + 1) + kKeyTile * kD);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qi = blockIdx.z, g = blockIdx.y;
    const int t0 = blockIdx.x * kTokPerBlock;
    const int t = t0 + warp;
    const bool tok_ok = t < a.T;
    const int t_last = min(t0 + kTokPerBlock, a.T) - 1;
    const int mem_len = max(min(a.mem_len[qi], a.max_mem), 0);
    const int n_local = min(a.L, a.q_start + t_last + 1);
    const int n_keys = mem_len + max(n_local, 0);

    const T* Q = static_cast<const T*>(a.q);
    const T* MKV = static_cast<const T*>(a.mem_kv);
    const T* LK = static_cast<const T*>(a.local_k);
    const T* LV = static_cast<const T*>(a.local_v);

    // queries of this warp's token, pre-scaled by scale * log2(e)
    if (tok_ok) {
        for (int e = lane * VEC; e < G * kD; e += 32 * VEC) {
            const int h = e / kD, i = e % kD;
            float x[VEC];
            load16_f32<T>(Q + (((int64_t)qi * a.T + t) * a.hq + g * G + h) * kD + i, x);
#pragma unroll
            for (int j = 0; j < VEC; ++j) Qs[warp][h][i + j] = x[j] * a.scale_log2e;
        }
    }

    const float ninf = -__int_as_float(0x7f800000);
    float m[G], l[G], acc[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m[h] = ninf;
        l[h] = 0.f;
        acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
    }

    for (int tb = 0; tb < n_keys; tb += kKeyTile) {
        __syncthreads();
        // stage 32 keys and values (fp32) for this kv head
        for (int v = threadIdx.x; v < kKeyTile * (kD / VEC) * 2; v += blockDim.x) {
            const int which = v / (kKeyTile * (kD / VEC));          // 0 = K, 1 = V
            const int rem = v % (kKeyTile * (kD / VEC));
            const int r = rem / (kD / VEC), i = (rem % (kD / VEC)) * VEC;
            const int kk = tb + r;
            float x[VEC];
            if (kk < mem_len) {
                load16_f32<T>(MKV + (((int64_t)qi * a.max_mem + kk) * 2 + which) * a.hkv * kD + g * kD + i, x);
            } else if (kk < n_keys) {
                const int j = kk - mem_len;
                load16_f32<T>((which ? LV : LK) + (((int64_t)qi * a.L_max + j) * a.hkv + g) * kD + i, x);
            } else {
#pragma unroll
                for (int jj = 0; jj < VEC; ++jj) x[jj] = 0.f;
            }
            if (which == 0) {
#pragma unroll
                for (int jj = 0; jj < VEC; ++jj) Ks[r][i + jj] = x[jj];
            } else {
#pragma unroll
                for (int jj = 0; jj < VEC; ++jj) Vs[r][i + jj] = x[jj];
            }
        }
        __syncthreads();
        if (!tok_ok) continue;

        const int kk = tb + lane;
        const bool visible = (kk < mem_len) | ((kk < n_keys) & (kk - mem_len <= a.q_start + t));
        float s[G];
#pragma unroll
        for (int h = 0; h < G; ++h) s[h] = 0.f;
#pragma unroll 8
        for (int i = 0; i < kD; ++i) {
            const float kv = Ks[lane][i];
#pragma unroll
            for (int h = 0; h < G; ++h) s[h] = fmaf(Qs[warp][h][i], kv, s[h]);
        }
        float p[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float sv = visible ? s[h] : ninf;
            float mt = sv;
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
            const float m_new = fmaxf(m[h], mt);
            float factor = 1.f;
            if (m_new == ninf) {
                p[h] = 0.f;
            } else {
                factor = exp2f(m[h] - m_new);     // 0 when m[h] = -inf
                p[h] = visible ? exp2f(sv - m_new) : 0.f;
            }
            float ps = p[h];
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
            l[h] = l[h] * factor + ps;
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[h][c] *= factor;
            m[h] = m_new;
        }
#pragma unroll 4
        for (int r = 0; r < kKeyTile; ++r) {
            const float4 v4 = *reinterpret_cast<const float4*>(&Vs[r][lane * 4]);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float pr = __shfl_sync(0xffffffffu, p[h], r);
                acc[h][0] = fmaf(pr, v4.x, acc[h][0]);
                acc[h][1] = fmaf(pr, v4.y, acc[h][1]);
                acc[h][2] = fmaf(pr, v4.z, acc[h][2]);
                acc[h][3] = fmaf(pr, v4.w, acc[h][3]);
            }
        }
    }

    if (tok_ok) {
        T* O = static_cast<T*>(a.out);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float inv = l[h] > 0.f ? 1.0f / l[h] : 0.f;
            float o[4] = {acc[h][0] * inv, acc[h][1] * inv, acc[h][2] * inv, acc[h][3] * inv};
            store4<T>(O + (((int64_t)qi * a.T + t) * a.hq + g * G + h) * kD + lane * 4, o);
        }
    }
}

constexpr size_t attn_smem(int G) { return (size_t)(kKeyTile * (kD + 1) + kKeyTile * kD + kTokPerBlock * G * kD) * 4; }

template <typename T, int G>
msa_status launch_g(const AttnArgs& a, dim3 grid, cudaStream_t s) {
    auto kern = attn_kernel<T, G>;
    const size_t smem = attn_smem(G);
    MSA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    kern<<<grid, kTokPerBlock * 32, smem, s>>>(a);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

template <typename T>
msa_status launch(const AttnArgs& a, int n_q, cudaStream_t s) {
    const int G = a.hq / a.hkv;
    dim3 grid((a.T + kTokPerBlock - 1) / kTokPerBlock, a.hkv, n_q);
    switch (G) {
        case 1: return launch_g<T, 1>(a, grid, s);
        case 2: return launch_g<T, 2>(a, grid, s);
        case 4: return launch_g<T, 4>(a, grid, s);
        case 8: return launch_g<T, 8>(a, grid, s);
        default: return set_error(MSA_ERR_UNSUPPORTED, "msa_sparse_attn: hq/hkv = %d unsupported", G);
    }
}


// ------------------------------------------------------------------------------------------------
// bf16 tensor-core variant (mma.sync m16n8k16, fp32 accumulation): one block of 4 warps per
// (64 query rows, kv head g, query q); rows are (token, head) pairs r = t * G + h of the G heads
// sharing kv head g; warp w owns rows 16w..16w+15. Per tile of 64 keys: S = Q K^T from K rows in
// shared memory (row stride 136 elements: the 32-bit fragment loads of 8 keys x 4 lanes hit 32
// distinct banks), online softmax on the accumulator fragments (row max/sum across the 4 lanes of
// a row), then O += P V with V fragments from ldmatrix.trans. Q stays in registers.
// ------------------------------------------------------------------------------------------------
constexpr int kMmaRows = 64;
constexpr int kMmaKeys = 64;
constexpr int kKvStride = kD + 8;   // bf16 elements per shared-memory row

// Shared memory of one key/value stage: K and V tiles of 64 keys. The split variant double-buffers
// (the next tile's copies are in flight while the current tile is computed); the plain variant keeps
// one stage so that it fits beside the router's blocks on an SM.
constexpr size_t kMmaStageBytes = (size_t)2 * kMmaKeys * kKvStride * sizeof(__nv_bfloat16);

template <int G, bool SPLIT>
__global__ void __launch_bounds__(128, SPLIT ? 3 : 1) attn_mma_kernel(const AttnArgs a) {
    constexpr int STAGES = SPLIT ? 2 : 1;
    extern __shared__ __align__(16) unsigned char attn_mma_smem[];
    typedef __nv_bfloat16 Tile[kMmaKeys][kKvStride];
    Tile* Kst = reinterpret_cast<Tile*>(attn_mma_smem);                                  // [STAGES]
    Tile* Vst = reinterpret_cast<Tile*>(attn_mma_smem + STAGES * (kMmaStageBytes / 2));  // [STAGES]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tig = lane & 3;
    const int qi = blockIdx.z, g = blockIdx.y;
    const int n_rows = a.T * G;
    const int split = SPLIT ? blockIdx.x % a.n_split : 0;
    const int r0 = (SPLIT ? blockIdx.x / a.n_split : blockIdx.x) * kMmaRows;
    const int r_last = min(r0 + kMmaRows, n_rows) - 1;
    const int t_last = r_last / G;
    const int mem_len = max(min(a.mem_len[qi], a.max_mem), 0);
    const int n_local = max(min(a.L, a.q_start + t_last + 1), 0);
    const int n_keys = mem_len + n_local;
    // keys of this block: all of them, or this split's contiguous range of 64-key tiles (ranges
    // start on tile boundaries, so no tile straddles two splits)
    int k_begin = 0, k_end = n_keys;
    if constexpr (SPLIT) {
        const int tiles = (n_keys + kMmaKeys - 1) / kMmaKeys;
        const int per = (tiles + a.n_split - 1) / a.n_split;
        k_begin = min(split * per, tiles) * kMmaKeys;
        k_end = min(min(split * per + per, tiles) * kMmaKeys, n_keys);
    }

    const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(a.q);
    const __nv_bfloat16* MKV = static_cast<const __nv_bfloat16*>(a.mem_kv);
    const __nv_bfloat16* LK = static_cast<const __nv_bfloat16*>(a.local_k);
    const __nv_bfloat16* LV = static_cast<const __nv_bfloat16*>(a.local_v);

    // this thread's two rows (gid, gid + 8 of the warp's 16) and their tokens
    const int ra = r0 + warp * 16 + gid, rb = ra + 8;
    const bool va = ra < n_rows, vb = rb < n_rows;
    const int ta = ra / G, tb = rb / G;
    // Q fragments for the 8 k-steps of d = 128 (zeros for rows past the end)
    uint32_t qf[kD / 16][4];
    {
        const uint32_t* qa = reinterpret_cast<const uint32_t*>(Q + (((int64_t)qi * a.T + ta) * a.hq + g * G + ra % G) * kD);
        const uint32_t* qb = reinterpret_cast<const uint32_t*>(Q + (((int64_t)qi * a.T + tb) * a.hq + g * G + rb % G) * kD);
#pragma unroll
        for (int s = 0; s < kD / 16; ++s) {
            qf[s][0] = va ? qa[s * 8 + tig] : 0u;
            qf[s][1] = vb ? qb[s * 8 + tig] : 0u;
            qf[s][2] = va ? qa[s * 8 + 4 + tig] : 0u;
            qf[s][3] = vb ? qb[s * 8 + 4 + tig] : 0u;
        }
    }
    const float ninf = -__int_as_float(0x7f800000);
    float o[kD / 8][4];
#pragma unroll
    for (int nd = 0; nd < kD / 8; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
    float m_a = ninf, m_b = ninf, l_a = 0.f, l_b = 0.f;

    // stage 64 keys and values of tile kb into buffer b with asynchronous 16-byte copies (all in
    // flight at once); rows past the visible range are zero-filled without reading
    auto stage = [&](int kb, int b) {
        for (int v = threadIdx.x; v < kMmaKeys * (kD / 8) * 2; v += blockDim.x) {
            const int which = v / (kMmaKeys * (kD / 8));
            const int rem = v % (kMmaKeys * (kD / 8));
            const int r = rem / (kD / 8), c = (rem % (kD / 8)) * 8;
            const int kk = kb + r;
            const __nv_bfloat16* src = Q;     // any valid address: zero-filled copies read nothing
            uint32_t bytes = 0;
            if (kk < mem_len) {
                src = MKV + (((int64_t)qi * a.max_mem + kk) * 2 + which) * a.hkv * kD + g * kD + c;
                bytes = 16;
            } else if (kk < n_keys) {
                src = (which ? LV : LK) + (((int64_t)qi * a.L_max + (kk - mem_len)) * a.hkv + g) * kD + c;
                bytes = 16;
            }
            const uint32_t dst =
                static_cast<uint32_t>(__cvta_generic_to_shared(which ? &Vst[b][r][c] : &Kst[b][r][c]));
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    if (k_begin < k_end) stage(k_begin, 0);
    int buf = 0;
    for (int kb = k_begin; kb < k_end; kb += kMmaKeys) {
        if constexpr (STAGES == 2) {
            if (kb + kMmaKeys < k_end) {
                stage(kb + kMmaKeys, buf ^ 1);   // that buffer's readers finished at the last barrier
                asm volatile("cp.async.wait_group 1;" ::: "memory");
            } else {
                asm volatile("cp.async.wait_group 0;" ::: "memory");
            }
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        const Tile& Ks = Kst[buf];
        const Tile& Vs = Vst[buf];

        // S = Q K^T for 8 blocks of 8 keys
        float sc[kMmaKeys / 8][4];
#pragma unroll
        for (int nb = 0; nb < kMmaKeys / 8; ++nb) {
            sc[nb][0] = sc[nb][1] = sc[nb][2] = sc[nb][3] = 0.f;
            const uint32_t* krow = reinterpret_cast<const uint32_t*>(&Ks[nb * 8 + gid][0]);
#pragma unroll
            for (int s = 0; s < kD / 16; ++s) mma_bf16_16816(sc[nb], qf[s], krow[s * 8 + tig], krow[s * 8 + 4 + tig]);
        }
        // mask, scale (log2 domain) and tile row maxima
        float tm_a = ninf, tm_b = ninf;
#pragma unroll
        for (int nb = 0; nb < kMmaKeys / 8; ++nb) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int kk = kb + nb * 8 + tig * 2 + e;
                // branch-free (bitwise) masks: a memory row, or a causal local key inside the range
                const bool vis_a = va & ((kk < mem_len) | ((kk < n_keys) & (kk - mem_len <= a.q_start + ta)));
                const bool vis_b = vb & ((kk < mem_len) | ((kk < n_keys) & (kk - mem_len <= a.q_start + tb)));
                sc[nb][e] = vis_a ? sc[nb][e] * a.scale_log2e : ninf;
                sc[nb][2 + e] = vis_b ? sc[nb][2 + e] * a.scale_log2e : ninf;
                tm_a = fmaxf(tm_a, sc[nb][e]);
                tm_b = fmaxf(tm_b, sc[nb][2 + e]);
            }
        }
        tm_a = fmaxf(tm_a, __shfl_xor_sync(0xffffffffu, tm_a, 1));
        tm_a = fmaxf(tm_a, __shfl_xor_sync(0xffffffffu, tm_a, 2));
        tm_b = fmaxf(tm_b, __shfl_xor_sync(0xffffffffu, tm_b, 1));
        tm_b = fmaxf(tm_b, __shfl_xor_sync(0xffffffffu, tm_b, 2));
        const float mn_a = fmaxf(m_a, tm_a), mn_b = fmaxf(m_b, tm_b);
        const float f_a = mn_a == ninf ? 1.f : ex2(m_a - mn_a);
        const float f_b = mn_b == ninf ? 1.f : ex2(m_b - mn_b);
        const float ref_a = mn_a == ninf ? 0.f : mn_a, ref_b = mn_b == ninf ? 0.f : mn_b;   // masked: 2^-inf = 0
        m_a = mn_a;
        m_b = mn_b;
        float ps_a = 0.f, ps_b = 0.f;
#pragma unroll
        for (int nb = 0; nb < kMmaKeys / 8; ++nb) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                sc[nb][e] = ex2(sc[nb][e] - ref_a);
                sc[nb][2 + e] = ex2(sc[nb][2 + e] - ref_b);
                ps_a += sc[nb][e];
                ps_b += sc[nb][2 + e];
            }
        }
        l_a = l_a * f_a + ps_a;
        l_b = l_b * f_b + ps_b;
#pragma unroll
        for (int nd = 0; nd < kD / 8; ++nd) {
            o[nd][0] *= f_a; o[nd][1] *= f_a;
            o[nd][2] *= f_b; o[nd][3] *= f_b;
        }
        // O += P V: P from the score fragments (bf16), V fragments by ldmatrix.trans
#pragma unroll
        for (int s2 = 0; s2 < kMmaKeys / 16; ++s2) {
            uint32_t pa[4];
            pa[0] = pack_bf16(sc[2 * s2][0], sc[2 * s2][1]);
            pa[1] = pack_bf16(sc[2 * s2][2], sc[2 * s2][3]);
            pa[2] = pack_bf16(sc[2 * s2 + 1][0], sc[2 * s2 + 1][1]);
            pa[3] = pack_bf16(sc[2 * s2 + 1][2], sc[2 * s2 + 1][3]);
#pragma unroll
            for (int nd = 0; nd < kD / 8; nd += 2) {
                // matrices: keys 16s2+0..7 / +8..15, dims 8nd..+7 / 8(nd+1)..+7
                const int key = s2 * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int dim = nd * 8 + (lane >> 4) * 8;
                const uint32_t addr = static_cast<uint32_t>(__cvta_generic_to_shared(&Vs[key][dim]));
                uint32_t b0, b1, b2, b3;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                             : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
                             : "r"(addr));
                mma_bf16_16816(o[nd], pa, b0, b1);
                mma_bf16_16816(o[nd + 1], pa, b2, b3);
            }
        }
        __syncthreads();   // every warp is done with this buffer before it is refilled
        if constexpr (STAGES == 2) {
            buf ^= 1;
        } else if (kb + kMmaKeys < k_end) {
            stage(kb + kMmaKeys, 0);
        }
    }

    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    if constexpr (SPLIT) {
        // partial result of this key range: unnormalised output and (max, sum) per row
        const int64_t rows_total = (int64_t)gridDim.z * a.T * a.hq;
        const int64_t row_a = ((int64_t)qi * a.T + ta) * a.hq + g * G + ra % G;
        const int64_t row_b = ((int64_t)qi * a.T + tb) * a.hq + g * G + rb % G;
        float* po = a.part_o + (int64_t)split * rows_total * kD;
#pragma unroll
        for (int nd = 0; nd < kD / 8; ++nd) {
            if (va) *reinterpret_cast<float2*>(po + row_a * kD + nd * 8 + tig * 2) = make_float2(o[nd][0], o[nd][1]);
            if (vb) *reinterpret_cast<float2*>(po + row_b * kD + nd * 8 + tig * 2) = make_float2(o[nd][2], o[nd][3]);
        }
        if (tig == 0) {
            if (va) a.part_ml[(int64_t)split * rows_total + row_a] = make_float2(m_a, l_a);
            if (vb) a.part_ml[(int64_t)split * rows_total + row_b] = make_float2(m_b, l_b);
        }
        return;
    }
    const float ia = l_a > 0.f ? 1.f / l_a : 0.f, ib = l_b > 0.f ? 1.f / l_b : 0.f;
    __nv_bfloat16* O = static_cast<__nv_bfloat16*>(a.out);
    uint32_t* oa = reinterpret_cast<uint32_t*>(O + (((int64_t)qi * a.T + ta) * a.hq + g * G + ra % G) * kD);
    uint32_t* ob = reinterpret_cast<uint32_t*>(O + (((int64_t)qi * a.T + tb) * a.hq + g * G + rb % G) * kD);
#pragma unroll
    for (int nd = 0; nd < kD / 8; ++nd) {
        if (va) oa[nd * 4 + tig] = pack_bf16(o[nd][0] * ia, o[nd][1] * ia);
        if (vb) ob[nd * 4 + tig] = pack_bf16(o[nd][2] * ib, o[nd][3] * ib);
    }
}

// Merge of the split-KV partial results: one warp per (query, token, head) row, lane l owning dims
// 4l..4l+3. out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s with M = max_s m_s; a row whose
// ranges saw no visible key (all m_s = -inf) is 0. Lane s reads range s's (m, l) (ranges in groups
// of 32) and the max and the weights go round the warp by shuffles, so every range's loads are in
// flight together instead of one dependent round trip per range; the sums run in range order.
__global__ void __launch_bounds__(256) attn_combine_kernel(const float* __restrict__ part_o,
                                                           const float2* __restrict__ part_ml, int n_split,
                                                           int64_t rows, __nv_bfloat16* __restrict__ out,
                                                           float* __restrict__ lse) {
    // launched as a programmatic dependent of the split kernel: its blocks may start while the split
    // kernel finishes; the partial results are read only after it has completed and they are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float ninf = -__int_as_float(0x7f800000);
    float M = ninf;
    for (int s0 = 0; s0 < n_split; s0 += 32) {
        const float m = s0 + lane < n_split ? part_ml[(int64_t)(s0 + lane) * rows + row].x : ninf;
        M = fmaxf(M, m);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, L = 0.f;
    if (M != ninf) {
        for (int s0 = 0; s0 < n_split; s0 += 32) {
            const int n = min(32, n_split - s0);
            const float2 ml = lane < n ? part_ml[(int64_t)(s0 + lane) * rows + row] : make_float2(ninf, 0.f);
            const float w_l = ml.x == ninf ? 0.f : exp2f(ml.x - M);
            float4 o[8];
            for (int b = 0; b < n; b += 8) {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    o[i] = b + i < n ? *reinterpret_cast<const float4*>(part_o + ((int64_t)(s0 + b + i) * rows + row) *
                                                                                     kD + lane * 4)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float w = __shfl_sync(0xffffffffu, w_l, (b + i) & 31);
                    const float ls = __shfl_sync(0xffffffffu, ml.y, (b + i) & 31);
                    if (b + i < n && w != 0.f) {
                        L = fmaf(w, ls, L);
                        acc[0] = fmaf(w, o[i].x, acc[0]);
                        acc[1] = fmaf(w, o[i].y, acc[1]);
                        acc[2] = fmaf(w, o[i].z, acc[2]);
                        acc[3] = fmaf(w, o[i].w, acc[3]);
                    }
                }
            }
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    // natural-log log-sum-exp of the scaled logits (M and the sums are in log2 units)
    if (lse && lane == 0) lse[row] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : ninf;
    uint2 u;
    u.x = pack_bf16(acc[0] * inv, acc[1] * inv);
    u.y = pack_bf16(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(out + row * kD + lane * 4) = u;
}

msa_status launch_combine(const AttnArgs& a, int n_q, cudaStream_t s) {
    const int64_t rows = (int64_t)n_q * a.T * a.hq;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)((rows + 7) / 8), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    MSA_CUDA_TRY(cudaLaunchKernelEx(&cfg, attn_combine_kernel, static_cast<const float*>(a.part_o),
                                    static_cast<const float2*>(a.part_ml), a.n_split, rows,
                                    static_cast<__nv_bfloat16*>(a.out), a.lse));
    return MSA_OK;
}

template <int G, bool SPLIT>
msa_status launch_mma_g(const AttnArgs& a, int n_q, cudaStream_t s) {
    const int row_blocks = (a.T * G + kMmaRows - 1) / kMmaRows;
    dim3 grid(row_blocks * (SPLIT ? a.n_split : 1), a.hkv, n_q);
    const size_t smem = (SPLIT ? 2 : 1) * kMmaStageBytes;
    if constexpr (SPLIT)
        MSA_CUDA_TRY(cudaFuncSetAttribute(attn_mma_kernel<G, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem));
    attn_mma_kernel<G, SPLIT><<<grid, 128, smem, s>>>(a);
    MSA_LAUNCH_CHECK();
    if constexpr (SPLIT) return launch_combine(a, n_q, s);
    return MSA_OK;
}

template <bool SPLIT>
msa_status launch_mma(const AttnArgs& a, int n_q, cudaStream_t s) {
    switch (a.hq / a.hkv) {
        case 1: return launch_mma_g<1, SPLIT>(a, n_q, s);
        case 2: return launch_mma_g<2, SPLIT>(a, n_q, s);
        case 4: return launch_mma_g<4, SPLIT>(a, n_q, s);
        case 8: return launch_mma_g<8, SPLIT>(a, n_q, s);
        default: return set_error(MSA_ERR_UNSUPPORTED, "msa_sparse_attn: hq/hkv unsupported");
    }
}

// Key ranges per (64-row block, kv head, query): as many as keep the grid within one wave of three
// resident blocks per SM (148 SMs; the split kernel is register-bounded to 168 per thread for
// that), at least four 64-key tiles per range.
constexpr int kSplitTargetBlocks = 3 * 148;
constexpr int kMinTilesPerSplit = 4;

int pick_splits(int n_q, int T, int hq, int hkv, int max_mem, int L) {
    const int G = hq / hkv;
    const int64_t base = (int64_t)((T * G + kMmaRows - 1) / kMmaRows) * hkv * n_q;
    const int tiles = (max_mem + L + kMmaKeys - 1) / kMmaKeys;
    const int64_t want = kSplitTargetBlocks / base;
    const int64_t cap = std::max(1, tiles / kMinTilesPerSplit);
    return (int)std::max<int64_t>(1, std::min(want, cap));
}

int split_ws_splits(int n_q, int T, int hq, int hkv, int max_mem, int L) {
    return std::max(pick_splits(n_q, T, hq, hkv, max_mem, L), attn_tc_splits(n_q, T, hq, hkv, max_mem, L));
}

size_t split_ws_bytes(int n_split, int n_q, int T, int hq) {
    const size_t rows = (size_t)n_q * T * hq;
    return align_up((size_t)n_split * rows * kD * 4, 256) + align_up((size_t)n_split * rows * 8, 256);
}

}  // namespace
}  // namespace msa

namespace msa {
int attn_impl_setting() { return g_attn_impl.load(); }
}  // namespace msa

using namespace msa;

extern "C" {

msa_status msa_attn_set_impl(int impl) {
    MSA_REQUIRE(impl >= 0 && impl <= 3, "msa_attn_set_impl: impl must be 0, 1, 2 or 3");
    g_attn_impl.store(impl);
    return MSA_OK;
}

msa_status msa_sparse_attn(const void* q, const void* mem_kv, const int32_t* mem_len, int max_mem,
                           const void* local_k, const void* local_v, int L_max, int L, int q_start, int n_q, int T,
                           int hq, int hkv, int d, float scale, void* out, msa_dtype dt, void* stream) {
    MSA_REQUIRE(dtype_ok(dt), "msa_sparse_attn: bad dtype");
    MSA_REQUIRE(n_q > 0 && T >= 0 && hq > 0 && hkv > 0 && hq % hkv == 0 && max_mem >= 0 && L >= 0 && L <= L_max &&
                    q_start >= 0 && n_q <= 65535 && hkv <= 65535,
                "msa_sparse_attn: bad sizes");
    if (d != kD) return set_error(MSA_ERR_UNSUPPORTED, "msa_sparse_attn: head_dim must be 128, got %d", d);
    const int G = hq / hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8)
        return set_error(MSA_ERR_UNSUPPORTED, "msa_sparse_attn: hq/hkv = %d unsupported", G);
    if (T == 0) return MSA_OK;
    MSA_REQUIRE(q && out && mem_len, "msa_sparse_attn: NULL pointer");
    MSA_REQUIRE(max_mem == 0 || mem_kv, "msa_sparse_attn: NULL mem_kv");
    MSA_REQUIRE(L == 0 || (local_k && local_v), "msa_sparse_attn: NULL local K/V");
    MSA_REQUIRE(aligned16(q) && aligned16(out) && (max_mem == 0 || aligned16(mem_kv)) &&
                    (L == 0 || (aligned16(local_k) && aligned16(local_v))),
                "msa_sparse_attn: pointers must be 16-byte aligned");
    AttnArgs a{};
    a.q = q; a.mem_kv = mem_kv; a.mem_len = mem_len; a.max_mem = max_mem;
    a.local_k = local_k; a.local_v = local_v; a.L_max = L_max; a.L = L; a.q_start = q_start;
    a.T = T; a.hq = hq; a.hkv = hkv; a.scale_log2e = scale * 1.4426950408889634f; a.out = out;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dt == MSA_BF16 && (g_attn_impl.load() == 0 || g_attn_impl.load() == 3)) return launch_mma<false>(a, n_q, s);
    return dt == MSA_BF16 ? launch<__nv_bfloat16>(a, n_q, s) : launch<float>(a, n_q, s);
}

msa_status msa_sparse_attn_split_workspace_size(int n_q, int T, int hq, int hkv, int max_mem, int L, size_t* bytes) {
    MSA_REQUIRE(bytes, "msa_sparse_attn_split_workspace_size: bytes is NULL");
    MSA_REQUIRE(n_q > 0 && T >= 0 && hq > 0 && hkv > 0 && hq % hkv == 0 && max_mem >= 0 && L >= 0,
                "msa_sparse_attn_split_workspace_size: bad sizes");
    *bytes = split_ws_bytes(split_ws_splits(n_q, T, hq, hkv, max_mem, L), n_q, T, hq);
    return MSA_OK;
}

msa_status msa_sparse_attn_split_plan(int n_q, int T, int hq, int hkv, int max_mem, int L, int* row_blocks,
                                      int* key_ranges, int* cluster) {
    MSA_REQUIRE(row_blocks && key_ranges && cluster, "msa_sparse_attn_split_plan: NULL output");
    MSA_REQUIRE(n_q > 0 && T > 0 && hq > 0 && hkv > 0 && hq % hkv == 0 && max_mem >= 0 && L >= 0,
                "msa_sparse_attn_split_plan: bad sizes");
    const bool tc = g_attn_impl.load() == 0 || g_attn_impl.load() == 3;
    *row_blocks = 0;
    *cluster = 0;
    *key_ranges = tc ? attn_tc_splits(n_q, T, hq, hkv, max_mem, L) : pick_splits(n_q, T, hq, hkv, max_mem, L);
    if (!tc) return MSA_OK;
    int blocks = 1, cs = 0;
    MSA_RETURN_IF(attn_tc_plan(n_q, T, hq, hkv, *key_ranges, &blocks, &cs));
    *row_blocks = blocks;
    if (g_attn_impl.load() == 0 && cs >= 1) {
        *key_ranges = cs;
        *cluster = cs;
    }
    return MSA_OK;
}

msa_status msa_sparse_attn_split(const void* q, const void* mem_kv, const int32_t* mem_len, int max_mem,
                                 const void* local_k, const void* local_v, int L_max, int L, int q_start, int n_q,
                                 int T, int hq, int hkv, int d, float scale, void* out, float* lse, msa_dtype dt,
                                 void* ws, size_t ws_bytes, void* stream) {
    MSA_REQUIRE(dtype_ok(dt), "msa_sparse_attn_split: bad dtype");
    if (dt != MSA_BF16) return set_error(MSA_ERR_UNSUPPORTED, "msa_sparse_attn_split: bf16 only");
    MSA_REQUIRE(n_q > 0 && T >= 0 && hq > 0 && hkv > 0 && hq % hkv == 0 && max_mem >= 0 && L >= 0 && L <= L_max &&
                    q_start >= 0 && n_q <= 65535 && hkv <= 65535,
                "msa_sparse_attn_split: bad sizes");
    if (d != kD) return set_error(MSA_ERR_UNSUPPORTED, "msa_sparse_attn_split: head_dim must be 128, got %d", d);
    const int G = hq / hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8)
        return set_error(MSA_ERR_UNSUPPORTED, "msa_sparse_attn_split: hq/hkv = %d unsupported", G);
    if (T == 0) return MSA_OK;
    MSA_REQUIRE(q && out && mem_len && ws, "msa_sparse_attn_split: NULL pointer");
    MSA_REQUIRE(max_mem == 0 || mem_kv, "msa_sparse_attn_split: NULL mem_kv");
    MSA_REQUIRE(L == 0 || (local_k && local_v), "msa_sparse_attn_split: NULL local K/V");
    MSA_REQUIRE(aligned16(q) && aligned16(out) && aligned16(ws) && (max_mem == 0 || aligned16(mem_kv)) &&
                    (L == 0 || (aligned16(local_k) && aligned16(local_v))),
                "msa_sparse_attn_split: pointers must be 16-byte aligned");
    const bool tc = g_attn_impl.load() == 0 || g_attn_impl.load() == 3;
    const int n_split = tc ? attn_tc_splits(n_q, T, hq, hkv, max_mem, L) : pick_splits(n_q, T, hq, hkv, max_mem, L);
    const size_t need = split_ws_bytes(split_ws_splits(n_q, T, hq, hkv, max_mem, L), n_q, T, hq);
    if (ws_bytes < need)
        return set_error(MSA_ERR_WORKSPACE, "msa_sparse_attn_split: workspace %zu < %zu", ws_bytes, need);
    AttnArgs a{};
    a.q = q; a.mem_kv = mem_kv; a.mem_len = mem_len; a.max_mem = max_mem;
    a.local_k = local_k; a.local_v = local_v; a.L_max = L_max; a.L = L; a.q_start = q_start;
    a.T = T; a.hq = hq; a.hkv = hkv; a.scale_log2e = scale * 1.4426950408889634f; a.out = out;
    a.n_split = n_split;
    a.lse = lse;
    a.part_o = static_cast<float*>(ws);
    a.part_ml = reinterpret_cast<float2*>(static_cast<char*>(ws) +
                                          align_up((size_t)n_split * n_q * T * hq * kD * 4, 256));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (tc) {
        // impl 0: key ranges merged inside a thread-block cluster when the grid fits one wave of
        // clusters; impl 3 (and any shape that does not fit) writes partial results and combines them
        bool merged = false;
        MSA_RETURN_IF(launch_attn_tc(q, mem_kv, mem_len, max_mem, local_k, local_v, L_max, L, q_start, n_q, T, hq, hkv,
                                     a.scale_log2e, n_split, a.part_o, a.part_ml, out, lse, g_attn_impl.load() == 0,
                                     &merged, st));
        if (merged) return MSA_OK;
        return launch_combine(a, n_q, st);
    }
    return launch_mma<true>(a, n_q, st);
}

}  // extern "C"
