// Sparse attention of query tokens over [selected memory K-bar/V-bar ; causal local K/V].
//
// One block per (8 query tokens, kv head g, query q); warp w owns token t0 + w and the G query
// heads that share kv head g (GQA), so each key/value tile staged in shared memory serves 8 x G
// query rows. Keys go through in tiles of 32: lane r scores key r of the tile against the G
// heads (q and K from shared memory, K rows padded to 129 floats so the 32 lanes hit 32 banks),
// then an online softmax (running max and sum per head, exp2 with log2(e) folded into q) and
// the P.V update, where lane r owns output dims 4r..4r+3. Arithmetic and softmax in fp32.
#include "common.cuh"

namespace msa {
namespace {

constexpr int kD = 128;
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
        const bool visible = kk < mem_len || (kk < n_keys && kk - mem_len <= a.q_start + t);
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

}  // namespace
}  // namespace msa

using namespace msa;

extern "C" {

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
    return dt == MSA_BF16 ? launch<__nv_bfloat16>(a, n_q, s) : launch<float>(a, n_q, s);
}

}  // extern "C"
