// Document-wise / global RoPE and chunk-mean pooling: HBM-streaming kernels.
//
// Both kernels move 16-byte vectors (4 fp32 or 8 bf16 per lane). A head of d elements is held
// by d/VEC consecutive lanes of one warp, so the rotate-half partner of element i (i + d/2) sits
// in lane ^ (d/2)/VEC and is fetched with one shuffle per 32-bit word. RoPE angles come from a
// host-built fp64 -> fp32 table [max_pos][d/2] of (cos, sin).
#include "common.cuh"
#include "kernels.cuh"

namespace msa {
namespace {

constexpr int kPoolThreads = 128;
constexpr int kPoolUnroll = 8;   // 16-byte loads in flight per thread

template <typename T>
__device__ __forceinline__ uint4 load_stream(const T* p) {
    return __ldcs(reinterpret_cast<const uint4*>(p));
}

// Widen the 16-byte word group to fp32.
template <typename T>
__device__ __forceinline__ void widen(const uint4& u, float* out) {
    if constexpr (sizeof(T) == 4) {
        out[0] = __uint_as_float(u.x); out[1] = __uint_as_float(u.y);
        out[2] = __uint_as_float(u.z); out[3] = __uint_as_float(u.w);
    } else {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = __uint_as_float(w[i] << 16);
            out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
}

__device__ __forceinline__ uint4 shfl_xor_u4(const uint4& u, int m) {
    uint4 r;
    r.x = __shfl_xor_sync(0xffffffffu, u.x, m);
    r.y = __shfl_xor_sync(0xffffffffu, u.y, m);
    r.z = __shfl_xor_sync(0xffffffffu, u.z, m);
    r.w = __shfl_xor_sync(0xffffffffu, u.w, m);
    return r;
}

// Rotates the lane's VEC elements (own) given the partner lane's elements; ci is the index of the
// first element inside the half-head, first_half tells which side of the pair this lane holds.
template <int VEC>
__device__ __forceinline__ void rotate(float* own, const float* partner, const float2* __restrict__ cs_row, int ci,
                                       bool first_half) {
    float cs[2 * VEC];
#pragma unroll
    for (int j = 0; j < VEC / 2; ++j) {
        float4 w = *reinterpret_cast<const float4*>(cs_row + ci + 2 * j);
        cs[4 * j + 0] = w.x; cs[4 * j + 1] = w.y; cs[4 * j + 2] = w.z; cs[4 * j + 3] = w.w;
    }
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
        const float c = cs[2 * j], s = cs[2 * j + 1];
        // first half: x_i cos - x_{i+d/2} sin ; second half: x_{i+d/2} cos + x_i sin
        own[j] = first_half ? fmaf(own[j], c, -partner[j] * s) : fmaf(own[j], c, partner[j] * s);
    }
}

struct PoolArgs {
    const void* src[3];      // K, V, K^R token tensors
    int heads[3];
    int n_parts;
    int parts[3];
    int d;
    const int64_t* doc_tok_off;
    const int64_t* doc_chunk_off;
    const int32_t* chunk_doc;
    int64_t n_docs, n_chunks, n_tok;
    int chunk;
    int fuse_rope;
    const float2* cs;
    int64_t max_pos;
    void* kvbar;
    void* kr_index;
    int hkv;
    int normalize;
    int* err;
};

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const PoolArgs a) {
    constexpr int VEC = 16 / sizeof(TIn);
    // block b handles tensor part b % n_parts of chunks b / n_parts, b / n_parts + stride, ...: the
    // rotated-K blocks (heavier on the load units) interleave with the plain streaming ones
    const int part = a.parts[blockIdx.x % a.n_parts];
    const int64_t c_first = blockIdx.x / a.n_parts;
    const int64_t c_stride = gridDim.x / a.n_parts;
    const TIn* __restrict__ src = static_cast<const TIn*>(a.src[part]);
    const int H = a.heads[part];
    const int d = a.d;
    const int E = H * d;
    const int half_lanes = (d / 2) / VEC;
    const int lane = threadIdx.x & 31;
    const bool rope = (part == 0) && a.fuse_rope;
    const int passes = (E + kPoolThreads * VEC - 1) / (kPoolThreads * VEC);

    for (int64_t c = c_first; c < a.n_chunks; c += c_stride) {
        const int64_t doc = a.chunk_doc[c];
        if (doc < 0 || doc >= a.n_docs) {
            if (threadIdx.x == 0) record_device_error(a.err, MSA_DEV_BAD_INDEX);
            continue;
        }
        const int64_t doc_start = a.doc_tok_off[doc];
        const int64_t t0 = doc_start + (c - a.doc_chunk_off[doc]) * (int64_t)a.chunk;
        const int64_t doc_end = a.doc_tok_off[doc + 1];
        const int64_t t1 = min(t0 + (int64_t)a.chunk, doc_end);
        if (t0 < doc_start || t0 >= t1 || t1 > a.n_tok) {   // inconsistent metadata: skip, never read out of range
            if (threadIdx.x == 0) record_device_error(a.err, MSA_DEV_BAD_INDEX);
            continue;
        }
        const float inv_n = 1.0f / (float)(t1 - t0);

        for (int pass = 0; pass < passes; ++pass) {
            const int e0 = (pass * kPoolThreads + threadIdx.x) * VEC;
            const bool active = e0 < E;
            const int ih = e0 % d;
            const bool first_half = ih < d / 2;
            const int ci = first_half ? ih : ih - d / 2;
            float acc[VEC];
#pragma unroll
            for (int j = 0; j < VEC; ++j) acc[j] = 0.f;

            auto consume = [&](const uint4& raw, int64_t t) {
                float x[VEC];
                widen<TIn>(raw, x);
                if (rope) {
                    uint4 praw = shfl_xor_u4(raw, half_lanes);
                    float px[VEC];
                    widen<TIn>(praw, px);
                    const int64_t p = t - doc_start;
                    if (p < a.max_pos) {
                        rotate<VEC>(x, px, a.cs + p * (d / 2), ci, first_half);
                    } else if (active) {
                        record_device_error(a.err, MSA_DEV_ROPE_POSITION);
                    }
                }
#pragma unroll
                for (int j = 0; j < VEC; ++j) acc[j] += x[j];
            };

            const uint4 zero = make_uint4(0, 0, 0, 0);
            int64_t t = t0;
            if (rope) {
                // rotated keys: 4 tokens in flight (the rotation's table reads and registers dominate)
                for (; t + 4 <= t1; t += 4) {
                    uint4 r[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) r[u] = active ? load_stream(src + (t + u) * E + e0) : zero;
#pragma unroll
                    for (int u = 0; u < 4; ++u) consume(r[u], t + u);
                }
            } else {
                // plain streaming: kPoolUnroll tokens in flight
                for (; t + kPoolUnroll <= t1; t += kPoolUnroll) {
                    uint4 r[kPoolUnroll];
#pragma unroll
                    for (int u = 0; u < kPoolUnroll; ++u) r[u] = active ? load_stream(src + (t + u) * E + e0) : zero;
#pragma unroll
                    for (int u = 0; u < kPoolUnroll; ++u) {
                        float x[VEC];
                        widen<TIn>(r[u], x);
#pragma unroll
                        for (int j = 0; j < VEC; ++j) acc[j] += x[j];
                    }
                }
            }
            for (; t < t1; ++t) {
                uint4 r = active ? load_stream(src + t * E + e0) : zero;
                consume(r, t);
            }

            float mean[VEC];
#pragma unroll
            for (int j = 0; j < VEC; ++j) mean[j] = acc[j] * inv_n;

            if (part == 2) {
                if (a.normalize) {
                    float ss = 0.f;
#pragma unroll
                    for (int j = 0; j < VEC; ++j) ss = fmaf(mean[j], mean[j], ss);
                    // reduce over the d/VEC lanes holding this head (aligned lane groups)
                    for (int m = half_lanes; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
                    const float inv = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
#pragma unroll
                    for (int j = 0; j < VEC; ++j) mean[j] *= inv;
                }
                if (active) store_f32<TOut, VEC>(static_cast<TOut*>(a.kr_index) + c * (int64_t)E + e0, mean);
            } else if (active) {
                TOut* dst = static_cast<TOut*>(a.kvbar) + (c * 2 + part) * (int64_t)a.hkv * d + e0;
                store_f32<TOut, VEC>(dst, mean);
            }
        }
        (void)lane;
    }
}

// ---------------------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) rope_rows_kernel(const RopeRowsArgs a) {
    constexpr int VEC = 16 / sizeof(T);
    const int d = a.d;
    const int E = a.heads * d;
    const int half_lanes = (d / 2) / VEC;
    const int passes = (E + 128 * VEC - 1) / (128 * VEC);
    for (int64_t r = blockIdx.x; r < a.n_rows; r += gridDim.x) {
        int64_t in_row, out_row, u;
        if (a.uniform_len > 0) {
            const int64_t s = r / a.uniform_len;
            u = r - s * a.uniform_len;
            in_row = s * a.in_stride + u;
            out_row = s * a.out_stride + a.out_off + u;
        } else {
            int64_t lo = 0, hi = a.n_seg - 1;   // largest s with seg_off[s] <= r
            while (lo < hi) {
                const int64_t mid = (lo + hi + 1) >> 1;
                if (a.seg_off[mid] <= r) lo = mid; else hi = mid - 1;
            }
            u = r - a.seg_off[lo];
            in_row = out_row = r;
        }
        const int64_t p = a.pos_offset + u;
        const bool pos_ok = p >= 0 && p < a.max_pos;
        if (!pos_ok && threadIdx.x == 0) record_device_error(a.err, MSA_DEV_ROPE_POSITION);
        const T* src = static_cast<const T*>(a.in) + in_row * E;
        T* dst = static_cast<T*>(a.out) + out_row * E;
        for (int pass = 0; pass < passes; ++pass) {
            const int e0 = (pass * 128 + threadIdx.x) * VEC;
            const bool active = e0 < E;
            const uint4 raw = active ? *reinterpret_cast<const uint4*>(src + e0) : make_uint4(0, 0, 0, 0);
            const uint4 praw = shfl_xor_u4(raw, half_lanes);
            float x[VEC], px[VEC];
            widen<T>(raw, x);
            widen<T>(praw, px);
            const int ih = e0 % d;
            const bool first_half = ih < d / 2;
            if (pos_ok) rotate<VEC>(x, px, a.cs + p * (d / 2), first_half ? ih : ih - d / 2, first_half);
            if (active) store_f32<T, VEC>(dst + e0, x);
        }
    }
}


// ---------------------------------------------------------------------------------------------
// Fused append of one interleave round, every layer in one launch: block (layer, query, token)
// rotates the new token's key to its global position into the local cache, copies its value, and
// rotates its query into the attention workspace.
template <typename T>
__device__ __forceinline__ void rotate_copy_row(const T* __restrict__ src, T* __restrict__ dst, int E, int d,
                                                const float2* __restrict__ cs_row, bool do_rotate) {
    constexpr int VEC = 16 / sizeof(T);
    const int half_lanes = (d / 2) / VEC;
    const int passes = (E + 128 * VEC - 1) / (128 * VEC);
    for (int pass = 0; pass < passes; ++pass) {
        const int e0 = (pass * 128 + threadIdx.x) * VEC;
        const bool active = e0 < E;
        const uint4 raw = active ? *reinterpret_cast<const uint4*>(src + e0) : make_uint4(0, 0, 0, 0);
        if (!do_rotate) {
            if (active) *reinterpret_cast<uint4*>(dst + e0) = raw;
            continue;
        }
        const uint4 praw = shfl_xor_u4(raw, half_lanes);
        float x[VEC], px[VEC];
        widen<T>(raw, x);
        widen<T>(praw, px);
        const int ih = e0 % d;
        const bool first_half = ih < d / 2;
        if (cs_row) msa::rotate<VEC>(x, px, cs_row, first_half ? ih : ih - d / 2, first_half);
        if (active) store_f32<T, VEC>(dst + e0, x);
    }
}

template <typename T>
__global__ void __launch_bounds__(128) append_kernel(const AppendArgs a) {
    const int per_layer = a.n_q * a.T_new;
    const int layer = blockIdx.x / per_layer;
    const int rem = blockIdx.x % per_layer;
    const int q = rem / a.T_new, t = rem % a.T_new;
    const AppendLayer& y = a.layer[layer];
    const int64_t p = a.pos_offset + t;
    const bool pos_ok = p >= 0 && p < a.max_pos;
    if (!pos_ok && threadIdx.x == 0) record_device_error(a.err, MSA_DEV_ROPE_POSITION);
    const float2* cs_row = pos_ok ? a.cs + p * (a.d / 2) : nullptr;
    const int Ek = a.hkv * a.d, Eq = a.hq * a.d;
    const int64_t in_row = (int64_t)q * a.new_q_stride + t;
    const int64_t cache_row = (int64_t)q * a.L_max + a.L_prev + t;
    rotate_copy_row<T>(static_cast<const T*>(y.k_new) + in_row * Ek, static_cast<T*>(y.local_k) + cache_row * Ek, Ek,
                       a.d, cs_row, true);
    rotate_copy_row<T>(static_cast<const T*>(y.v_new) + in_row * Ek, static_cast<T*>(y.local_v) + cache_row * Ek, Ek,
                       a.d, nullptr, false);
    rotate_copy_row<T>(static_cast<const T*>(y.q_new) + in_row * Eq,
                       static_cast<T*>(y.q_rot) + ((int64_t)q * a.T_new + t) * Eq, Eq, a.d, cs_row, true);
}

// ---------------------------------------------------------------------------------------------
// Token-level memory bank of the fine stage: block-stride over token rows; row r of document i
// (found by binary search of the token offsets) gets its key rotated to its position inside the
// document, r - doc_tok_off[i], into bank[r][0], and its value copied into bank[r][1].
struct PackArgs {
    const void* k;
    const void* v;
    int64_t n_tok;
    int hkv, d;
    const int64_t* doc_tok_off;
    int64_t n_docs;
    const float2* cs;
    int64_t max_pos;
    void* bank;
    int* err;
};

template <typename T>
__global__ void __launch_bounds__(128) pack_tokens_kernel(const PackArgs a) {
    const int E = a.hkv * a.d;
    for (int64_t r = blockIdx.x; r < a.n_tok; r += gridDim.x) {
        int64_t lo = 0, hi = a.n_docs - 1;   // largest i with doc_tok_off[i] <= r
        while (lo < hi) {
            const int64_t mid = (lo + hi + 1) >> 1;
            if (a.doc_tok_off[mid] <= r) lo = mid; else hi = mid - 1;
        }
        const int64_t p = r - a.doc_tok_off[lo];
        const bool pos_ok = p >= 0 && p < a.max_pos;
        if (!pos_ok && threadIdx.x == 0) record_device_error(a.err, MSA_DEV_ROPE_POSITION);
        T* dst = static_cast<T*>(a.bank) + r * 2 * (int64_t)E;
        rotate_copy_row<T>(static_cast<const T*>(a.k) + r * E, dst, E, a.d, pos_ok ? a.cs + p * (a.d / 2) : nullptr,
                           true);
        rotate_copy_row<T>(static_cast<const T*>(a.v) + r * E, dst + E, E, a.d, nullptr, false);
    }
}

template <typename T>
bool vec_layout_ok(int d) {
    constexpr int VEC = 16 / sizeof(T);
    if (d % (2 * VEC) != 0) return false;
    const int lanes = d / VEC;
    return lanes <= 32 && (lanes & (lanes - 1)) == 0;
}

}  // namespace

msa_status launch_rope_rows(const RopeRowsArgs& a, msa_dtype dt, cudaStream_t s) {
    if (a.n_rows == 0) return MSA_OK;
    const int64_t cap = (int64_t)sm_count() * 32;
    const unsigned blocks = (unsigned)(a.n_rows < cap ? a.n_rows : cap);
    if (dt == MSA_BF16)
        rope_rows_kernel<__nv_bfloat16><<<blocks, 128, 0, s>>>(a);
    else
        rope_rows_kernel<float><<<blocks, 128, 0, s>>>(a);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

msa_status launch_append(const AppendArgs& a, msa_dtype dt, cudaStream_t s) {
    const int64_t blocks = (int64_t)a.n_layers * a.n_q * a.T_new;
    if (blocks == 0) return MSA_OK;
    if (dt == MSA_BF16)
        append_kernel<__nv_bfloat16><<<(unsigned)blocks, 128, 0, s>>>(a);
    else
        append_kernel<float><<<(unsigned)blocks, 128, 0, s>>>(a);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

msa_status launch_pack_tokens(const PackArgs& a, msa_dtype dt, cudaStream_t s) {
    if (a.n_tok == 0) return MSA_OK;
    const int64_t cap = (int64_t)sm_count() * 16;
    const unsigned blocks = (unsigned)(a.n_tok < cap ? a.n_tok : cap);
    if (dt == MSA_BF16)
        pack_tokens_kernel<__nv_bfloat16><<<blocks, 128, 0, s>>>(a);
    else
        pack_tokens_kernel<float><<<blocks, 128, 0, s>>>(a);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

bool rope_layout_ok(msa_dtype dt, int d) {
    return dt == MSA_BF16 ? vec_layout_ok<__nv_bfloat16>(d) : vec_layout_ok<float>(d);
}

}  // namespace msa

using namespace msa;

extern "C" {

msa_status msa_rope_doc(const void* x, void* out, msa_dtype dt, int64_t n_tok, int n_heads, int head_dim,
                        const int64_t* seg_tok_off, int64_t n_seg, int64_t pos_offset, const float* cos_sin,
                        int64_t max_pos, void* stream) {
    MSA_REQUIRE(dtype_ok(dt), "msa_rope_doc: bad dtype %d", dt);
    MSA_REQUIRE(n_tok >= 0 && n_heads > 0 && head_dim > 0 && n_seg > 0 && max_pos > 0 && pos_offset >= 0,
                "msa_rope_doc: bad sizes");
    if (n_tok == 0) return MSA_OK;
    MSA_REQUIRE(x && out && seg_tok_off && cos_sin, "msa_rope_doc: NULL pointer");
    MSA_REQUIRE(aligned16(x) && aligned16(out) && aligned16(cos_sin), "msa_rope_doc: pointers must be 16-byte aligned");
    if (!rope_layout_ok(dt, head_dim))
        return set_error(MSA_ERR_UNSUPPORTED, "msa_rope_doc: head_dim %d unsupported for this dtype", head_dim);
    RopeRowsArgs a{};
    a.in = x; a.out = out; a.n_rows = n_tok; a.heads = n_heads; a.d = head_dim;
    a.seg_off = seg_tok_off; a.n_seg = n_seg; a.uniform_len = 0;
    a.pos_offset = pos_offset; a.cs = reinterpret_cast<const float2*>(cos_sin); a.max_pos = max_pos;
    a.err = device_error_word();
    return launch_rope_rows(a, dt, static_cast<cudaStream_t>(stream));
}

msa_status msa_pack_tokens(const void* k, const void* v, msa_dtype dt, int64_t n_tok, int hkv, int d,
                           const int64_t* doc_tok_off, int64_t n_docs, const float* cos_sin, int64_t max_pos,
                           void* bank, void* stream) {
    MSA_REQUIRE(dtype_ok(dt), "msa_pack_tokens: bad dtype %d", dt);
    MSA_REQUIRE(n_tok >= 0 && hkv > 0 && d > 0 && n_docs > 0 && max_pos > 0, "msa_pack_tokens: bad sizes");
    if (n_tok == 0) return MSA_OK;
    MSA_REQUIRE(k && v && doc_tok_off && cos_sin && bank, "msa_pack_tokens: NULL pointer");
    MSA_REQUIRE(aligned16(k) && aligned16(v) && aligned16(bank) && aligned16(cos_sin),
                "msa_pack_tokens: pointers must be 16-byte aligned");
    if (!rope_layout_ok(dt, d))
        return set_error(MSA_ERR_UNSUPPORTED, "msa_pack_tokens: head layout hkv=%d d=%d unsupported", hkv, d);
    PackArgs a{};
    a.k = k; a.v = v; a.n_tok = n_tok; a.hkv = hkv; a.d = d;
    a.doc_tok_off = doc_tok_off; a.n_docs = n_docs;
    a.cs = reinterpret_cast<const float2*>(cos_sin); a.max_pos = max_pos;
    a.bank = bank; a.err = device_error_word();
    return launch_pack_tokens(a, dt, static_cast<cudaStream_t>(stream));
}

msa_status msa_pool_chunks(const void* k, const void* v, const void* kr, msa_dtype in_dt, int64_t n_tok, int hkv,
                           int hr, int d, const int64_t* doc_tok_off, const int64_t* doc_chunk_off,
                           const int32_t* chunk_doc, int64_t n_docs, int64_t n_chunks, int chunk, int fuse_doc_rope,
                           const float* cos_sin, int64_t max_pos, void* kvbar, void* kr_index, msa_dtype out_dt,
                           int normalize_router, void* stream) {
    MSA_REQUIRE(dtype_ok(in_dt) && dtype_ok(out_dt), "msa_pool_chunks: bad dtype");
    MSA_REQUIRE(n_tok >= 0 && n_docs >= 0 && n_chunks >= 0 && chunk > 0 && d > 0, "msa_pool_chunks: bad sizes");
    MSA_REQUIRE((k == nullptr) == (v == nullptr), "msa_pool_chunks: k and v must both be given or both be NULL");
    MSA_REQUIRE(k != nullptr || kr != nullptr, "msa_pool_chunks: nothing to pool");
    if (n_chunks == 0) return MSA_OK;
    MSA_REQUIRE(doc_tok_off && doc_chunk_off && chunk_doc, "msa_pool_chunks: NULL offsets");
    if (!rope_layout_ok(in_dt, d))
        return set_error(MSA_ERR_UNSUPPORTED, "msa_pool_chunks: head_dim %d unsupported for this dtype", d);
    PoolArgs a{};
    a.n_parts = 0;
    if (k) {
        MSA_REQUIRE(hkv > 0 && kvbar && aligned16(k) && aligned16(v) && aligned16(kvbar),
                    "msa_pool_chunks: K/V need hkv > 0 and 16-byte aligned k, v, kvbar");
        a.src[0] = k; a.src[1] = v; a.heads[0] = a.heads[1] = hkv;
        a.parts[a.n_parts++] = 0;
        a.parts[a.n_parts++] = 1;
        if (fuse_doc_rope) {
            MSA_REQUIRE(cos_sin && max_pos > 0 && aligned16(cos_sin), "msa_pool_chunks: fused RoPE needs a table");
        }
    }
    if (kr) {
        MSA_REQUIRE(hr > 0 && kr_index && aligned16(kr) && aligned16(kr_index),
                    "msa_pool_chunks: K^R needs hr > 0 and 16-byte aligned kr, kr_index");
        a.src[2] = kr; a.heads[2] = hr;
        a.parts[a.n_parts++] = 2;
    }
    // outputs of bf16 with d*... : each lane stores VEC(in) elements of out_dt -> needs alignment of that size
    MSA_REQUIRE(!(in_dt == MSA_F32 && out_dt == MSA_BF16) || (d % 8 == 0), "msa_pool_chunks: bad d for fp32->bf16");
    MSA_REQUIRE(!(in_dt == MSA_BF16 && out_dt == MSA_F32) || (d % 8 == 0), "msa_pool_chunks: bad d for bf16->fp32");
    a.d = d; a.hkv = hkv;
    a.doc_tok_off = doc_tok_off; a.doc_chunk_off = doc_chunk_off; a.chunk_doc = chunk_doc;
    a.n_docs = n_docs; a.n_chunks = n_chunks; a.n_tok = n_tok; a.chunk = chunk; a.fuse_rope = fuse_doc_rope;
    a.cs = reinterpret_cast<const float2*>(cos_sin); a.max_pos = max_pos;
    a.kvbar = kvbar; a.kr_index = kr_index; a.normalize = normalize_router;
    a.err = device_error_word();
    const int64_t cap = 1 << 20;
    const int64_t per_part = n_chunks < cap ? n_chunks : cap;
    dim3 grid((unsigned)(per_part * a.n_parts));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (in_dt == MSA_BF16 && out_dt == MSA_BF16)
        pool_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, kPoolThreads, 0, s>>>(a);
    else if (in_dt == MSA_BF16)
        pool_kernel<__nv_bfloat16, float><<<grid, kPoolThreads, 0, s>>>(a);
    else if (out_dt == MSA_BF16)
        pool_kernel<float, __nv_bfloat16><<<grid, kPoolThreads, 0, s>>>(a);
    else
        pool_kernel<float, float><<<grid, kPoolThreads, 0, s>>>(a);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

}  // extern "C"
