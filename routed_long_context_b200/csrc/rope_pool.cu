// Document-wise / global RoPE and chunk-mean pooling: HBM-streaming kernels.
//
// Both kernels move 16-byte vectors (4 fp32 or 8 bf16 per lane). A head of d elements is held
// by d/VEC consecutive lanes of one warp, so the rotate-half partner of element i (i + d/2) sits
// in lane ^ (d/2)/VEC and is fetched with one shuffle per 32-bit word. RoPE angles come from a
// host-built fp64 -> fp32 table [max_pos][d/2] of (cos, sin).
#include <atomic>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"

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

// Widen an 8-byte word group (4 bf16 or 2 fp32) to fp32.
template <typename T>
__device__ __forceinline__ void widen8(const uint2& u, float* out) {
    if constexpr (sizeof(T) == 4) {
        out[0] = __uint_as_float(u.x); out[1] = __uint_as_float(u.y);
    } else {
        out[0] = __uint_as_float(u.x << 16); out[1] = __uint_as_float(u.x & 0xFFFF0000u);
        out[2] = __uint_as_float(u.y << 16); out[3] = __uint_as_float(u.y & 0xFFFF0000u);
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
    // bulk-copy variant only
    int rows_per_stage[3];   // token rows of each tensor part per pipeline stage
    int rows_per_copy[3];    // token rows of each tensor part per bulk copy (a stage takes one or more)
    int tab_bytes;           // bytes of one RoPE table row (d/2 cos/sin pairs), staged after rotated rows
    int n_stages;
    int stage_bytes;
};

// Rotated keys of one chunk, pair layout: a thread owns F = VEC/2 frequencies of one head, i.e.
// the F elements of the head's first half and their rotate-half partners F elements later by
// d/2, read as two 8-byte streams per token, so no lane needs another lane's data. The RoPE table
// entries (cos, sin) of a batch's positions are loaded together with the batch's key rows, so their
// latency overlaps the HBM loads. Per element the arithmetic is the one of every other pooling
// path: x' = x c -+ partner s (fmaf of the product), then acc += x', tokens in order.
template <typename TIn, typename TOut>
__device__ __forceinline__ void pool_rotated_pairs(const PoolArgs& a, const TIn* __restrict__ src, int64_t c,
                                                   int64_t doc_start, int64_t t0, int64_t t1, float inv_n, int E,
                                                   int passes) {
    constexpr int VEC = 16 / sizeof(TIn);
    constexpr int F = VEC / 2;                 // frequencies per thread (8 bytes of keys per half)
    constexpr int U = 4;                       // tokens per batch
    const int d = a.d;
    const int per_head = d / VEC;              // threads per head
    for (int pass = 0; pass < passes; ++pass) {
        const int pi = pass * kPoolThreads + threadIdx.x;
        const bool active = pi * VEC < E;
        const int h = pi / per_head;
        const int f0 = (pi % per_head) * F;
        const int64_t lo = (int64_t)h * d + f0, hi = lo + d / 2;
        float acc_lo[F], acc_hi[F];
#pragma unroll
        for (int j = 0; j < F; ++j) acc_lo[j] = acc_hi[j] = 0.f;

        auto rotate_add = [&](const uint2& rlo, const uint2& rhi, const float4* tab, bool in_table) {
            float xl[F], xh[F];
            widen8<TIn>(rlo, xl);
            widen8<TIn>(rhi, xh);
            if (in_table) {
#pragma unroll
                for (int j = 0; j < F; ++j) {
                    const float4 w = tab[j / 2];
                    const float cj = (j & 1) ? w.z : w.x, sj = (j & 1) ? w.w : w.y;
                    const float l = fmaf(xl[j], cj, -xh[j] * sj);
                    const float r = fmaf(xh[j], cj, xl[j] * sj);
                    xl[j] = l;
                    xh[j] = r;
                }
            }
#pragma unroll
            for (int j = 0; j < F; ++j) {
                acc_lo[j] += xl[j];
                acc_hi[j] += xh[j];
            }
        };

        const uint2 z2 = make_uint2(0, 0);
        const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        int64_t t = t0;
        for (; t + U <= t1; t += U) {
            uint2 rl[U], rh[U];
            float4 tb[U][F / 2];
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const TIn* row = src + (t + u) * E;
                rl[u] = active ? __ldcs(reinterpret_cast<const uint2*>(row + lo)) : z2;
                rh[u] = active ? __ldcs(reinterpret_cast<const uint2*>(row + hi)) : z2;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t p = t + u - doc_start;
                ok[u] = p < a.max_pos;
                const float4* trow = reinterpret_cast<const float4*>(a.cs + p * (d / 2) + f0);
#pragma unroll
                for (int j = 0; j < F / 2; ++j) tb[u][j] = (active && ok[u]) ? __ldg(trow + j) : z4;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (!ok[u] && active) record_device_error(a.err, MSA_DEV_ROPE_POSITION);
                rotate_add(rl[u], rh[u], tb[u], ok[u]);
            }
        }
        for (; t < t1; ++t) {
            const TIn* row = src + t * E;
            const uint2 rl = active ? __ldcs(reinterpret_cast<const uint2*>(row + lo)) : z2;
            const uint2 rh = active ? __ldcs(reinterpret_cast<const uint2*>(row + hi)) : z2;
            const int64_t p = t - doc_start;
            const bool ok = p < a.max_pos;
            float4 tb[F / 2];
            const float4* trow = reinterpret_cast<const float4*>(a.cs + p * (d / 2) + f0);
#pragma unroll
            for (int j = 0; j < F / 2; ++j) tb[j] = (active && ok) ? __ldg(trow + j) : z4;
            if (!ok && active) record_device_error(a.err, MSA_DEV_ROPE_POSITION);
            rotate_add(rl, rh, tb, ok);
        }
        if (active) {
            float ml[F], mh[F];
#pragma unroll
            for (int j = 0; j < F; ++j) {
                ml[j] = acc_lo[j] * inv_n;
                mh[j] = acc_hi[j] * inv_n;
            }
            TOut* dst = static_cast<TOut*>(a.kvbar) + (c * 2) * (int64_t)a.hkv * d;
            store_f32<TOut, F>(dst + lo, ml);
            store_f32<TOut, F>(dst + hi, mh);
        }
    }
}

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
        if (doc_start < 0 || t0 < doc_start || t0 >= t1 || t1 > a.n_tok) {   // inconsistent metadata: skip
            if (threadIdx.x == 0) record_device_error(a.err, MSA_DEV_BAD_INDEX);
            continue;
        }
        const float inv_n = 1.0f / (float)(t1 - t0);

        if (rope) {
            pool_rotated_pairs<TIn, TOut>(a, src, c, doc_start, t0, t1, inv_n, E, passes);
            continue;
        }
        for (int pass = 0; pass < passes; ++pass) {
            const int e0 = (pass * kPoolThreads + threadIdx.x) * VEC;
            const bool active = e0 < E;
            float acc[VEC];
#pragma unroll
            for (int j = 0; j < VEC; ++j) acc[j] = 0.f;

            const uint4 zero = make_uint4(0, 0, 0, 0);
            int64_t t = t0;
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
            for (; t < t1; ++t) {
                uint4 r = active ? load_stream(src + t * E + e0) : zero;
                float x[VEC];
                widen<TIn>(r, x);
#pragma unroll
                for (int j = 0; j < VEC; ++j) acc[j] += x[j];
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
// Chunk-mean pooling with the token rows staged in shared memory by bulk copies.
//
// A chunk's rows of one tensor part are one contiguous run of HBM ([t0, t1) x H*d). The CTA walks
// its (chunk, part) work items; one producer lane streams each item's run into a ring of
// n_stages stages (stage_bytes each, whole rows) with cp.async.bulk, completing on the stage's
// mbarrier; for rotated keys the RoPE table rows of the stage's positions (contiguous, since the
// positions are) are copied into the stage behind the data rows. The consumer warps (one thread
// per VEC elements of a row) read every row of the stage from shared memory, rotate K (partner
// element and cos/sin from the same stage), accumulate in fp32 and release the stage. The copy queue never drains between a thread's load batches, so the
// SM keeps its share of the HBM bandwidth in flight. Every wait is bounded: on expiry the CTA
// records MSA_DEV_WAIT_TIMEOUT, leaves its loops and lets the copies it issued land before exiting.
struct PoolItem {
    int64_t c, doc_start, t0, t1;
    int part;
};

__device__ __forceinline__ bool pool_item(const PoolArgs& a, int64_t item, PoolItem& it) {
    it.c = item / a.n_parts;
    it.part = a.parts[item % a.n_parts];
    const int64_t doc = a.chunk_doc[it.c];
    if (doc < 0 || doc >= a.n_docs) return false;
    it.doc_start = a.doc_tok_off[doc];
    it.t0 = it.doc_start + (it.c - a.doc_chunk_off[doc]) * (int64_t)a.chunk;
    const int64_t doc_end = a.doc_tok_off[doc + 1];
    it.t1 = min(it.t0 + (int64_t)a.chunk, doc_end);
    return !(it.doc_start < 0 || it.t0 < it.doc_start || it.t0 >= it.t1 || it.t1 > a.n_tok);
}

constexpr int kBulkMaxConsumers = 256;

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kBulkMaxConsumers + 32)
    pool_bulk_kernel(const PoolArgs a) {
    constexpr int VEC = 16 / sizeof(TIn);
    extern __shared__ __align__(128) unsigned char pool_smem[];
    const int S = a.n_stages;
    unsigned char* ring = pool_smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(ring + (size_t)S * a.stage_bytes);
    uint64_t* empty = full + S;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + S);
    const int nc = (int)blockDim.x - 32;   // consumer threads; the last warp produces
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(smem_u32(full + i), 1);
            mbar_init(smem_u32(empty + i), nc / 32);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();
    const int64_t n_items = a.n_chunks * a.n_parts;
    const int d = a.d;

    // producer state, read again by the drain after the final barrier
    int p_st = 0;
    uint32_t p_ph = 0;
    int64_t p_issued = 0;

    if (tid >= nc) {
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            bool stop = false;
            for (int64_t item = blockIdx.x; item < n_items && !stop; item += gridDim.x) {
                PoolItem it;
                if (!pool_item(a, item, it)) continue;
                const int64_t E = (int64_t)a.heads[it.part] * d;
                const TIn* src = static_cast<const TIn*>(a.src[it.part]);
                const int R = a.rows_per_stage[it.part];
                for (int64_t r0 = it.t0; r0 < it.t1; r0 += R) {
                    const int64_t n = min((int64_t)R, it.t1 - r0);
                    if (!mbar_wait(smem_u32(empty + p_st), p_ph ^ 1u, abort_flag)) {
                        stop = true;
                        break;
                    }
                    const int64_t row_bytes = E * (int64_t)sizeof(TIn);
                    // rotated keys: the table rows of the stage's positions follow its R data rows
                    int64_t n_tab = 0;
                    if (it.part == 0 && a.fuse_rope) {
                        n_tab = min(n, a.max_pos - (r0 - it.doc_start));
                        if (n_tab < 0) n_tab = 0;
                    }
                    const uint32_t stage_addr = smem_u32(ring + (size_t)p_st * a.stage_bytes);
                    mbar_expect_tx(smem_u32(full + p_st), (uint32_t)(n * row_bytes + n_tab * a.tab_bytes));
                    const int64_t CR = a.rows_per_copy[it.part];
                    for (int64_t cr = 0; cr < n; cr += CR) {
                        const int64_t m = min(CR, n - cr);
                        bulk_load_evict_first(stage_addr + (uint32_t)(cr * row_bytes), src + (r0 + cr) * E,
                                              (uint32_t)(m * row_bytes), smem_u32(full + p_st), pol);
                    }
                    if (n_tab > 0)
                        bulk_load_evict_first(stage_addr + (uint32_t)(R * row_bytes),
                                              a.cs + (r0 - it.doc_start) * (int64_t)(d / 2),
                                              (uint32_t)(n_tab * a.tab_bytes), smem_u32(full + p_st), pol);
                    ++p_issued;
                    if (++p_st == S) {
                        p_st = 0;
                        p_ph ^= 1u;
                    }
                }
            }
        }
    } else {
        int st = 0;
        uint32_t ph = 0;
        bool stop = false;
        const int half_lanes = (d / 2) / VEC;
        for (int64_t item = blockIdx.x; item < n_items && !stop; item += gridDim.x) {
            PoolItem it;
            if (!pool_item(a, item, it)) {
                if (tid == 0) record_device_error(a.err, MSA_DEV_BAD_INDEX);
                continue;
            }
            const int part = it.part;
            const int E = a.heads[part] * d;
            const int e0 = tid * VEC;
            const bool active = e0 < E;
            const int ih = e0 % d;
            const bool first_half = ih < d / 2;
            const int ci = first_half ? ih : ih - d / 2;
            const int pe0 = first_half ? e0 + d / 2 : e0 - d / 2;   // rotate-half partner
            const bool rope = (part == 0) && a.fuse_rope;
            const int R = a.rows_per_stage[part];
            const int row_bytes = E * (int)sizeof(TIn);
            float acc[VEC];
#pragma unroll
            for (int j = 0; j < VEC; ++j) acc[j] = 0.f;

            for (int64_t r0 = it.t0; r0 < it.t1; r0 += R) {
                const int n = (int)min((int64_t)R, it.t1 - r0);
                // every lane of the warp takes the same way out, so the shuffles below stay converged
                if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(full + st), ph, abort_flag))) {
                    stop = true;
                    break;
                }
                const unsigned char* stage = ring + (size_t)st * a.stage_bytes;
                if (active) {
                    if (rope) {
                        const unsigned char* tab = stage + R * row_bytes;
#pragma unroll 2
                        for (int r = 0; r < n; ++r) {
                            const unsigned char* row = stage + r * row_bytes;
                            float x[VEC], px[VEC];
                            widen<TIn>(*reinterpret_cast<const uint4*>(row + e0 * (int)sizeof(TIn)), x);
                            widen<TIn>(*reinterpret_cast<const uint4*>(row + pe0 * (int)sizeof(TIn)), px);
                            const int64_t p = r0 + r - it.doc_start;
                            if (p < a.max_pos)
                                rotate<VEC>(x, px, reinterpret_cast<const float2*>(tab + r * a.tab_bytes), ci,
                                            first_half);
                            else
                                record_device_error(a.err, MSA_DEV_ROPE_POSITION);
#pragma unroll
                            for (int j = 0; j < VEC; ++j) acc[j] += x[j];
                        }
                    } else {
#pragma unroll 4
                        for (int r = 0; r < n; ++r) {
                            float x[VEC];
                            widen<TIn>(*reinterpret_cast<const uint4*>(stage + r * row_bytes + e0 * (int)sizeof(TIn)),
                                       x);
#pragma unroll
                            for (int j = 0; j < VEC; ++j) acc[j] += x[j];
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(empty + st));
                if (++st == S) {
                    st = 0;
                    ph ^= 1u;
                }
            }
            if (stop) break;

            const float inv_n = 1.0f / (float)(it.t1 - it.t0);
            float mean[VEC];
#pragma unroll
            for (int j = 0; j < VEC; ++j) mean[j] = acc[j] * inv_n;
            if (part == 2) {
                if (a.normalize) {
                    float ss = 0.f;
#pragma unroll
                    for (int j = 0; j < VEC; ++j) ss = fmaf(mean[j], mean[j], ss);
                    for (int m = half_lanes; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
                    const float inv = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
#pragma unroll
                    for (int j = 0; j < VEC; ++j) mean[j] *= inv;
                }
                if (active) store_f32<TOut, VEC>(static_cast<TOut*>(a.kr_index) + it.c * (int64_t)E + e0, mean);
            } else if (active) {
                TOut* dst = static_cast<TOut*>(a.kvbar) + (it.c * 2 + part) * (int64_t)a.hkv * d + e0;
                store_f32<TOut, VEC>(dst, mean);
            }
        }
    }
    __syncwarp();
    __syncthreads();
    if (*abort_flag) {
        if (tid == 0) record_device_error(a.err, MSA_DEV_WAIT_TIMEOUT);
        if (tid == nc) {
            // the last min(issued, S) stages hold the only copies that can still be in flight
            const int64_t back = p_issued < S ? p_issued : S;
            for (int64_t j = 1; j <= back; ++j) {
                int s2 = p_st - (int)j;
                uint32_t ph2 = p_ph;
                if (s2 < 0) {
                    s2 += S;
                    ph2 ^= 1u;
                }
                mbar_wait_drain(smem_u32(full + s2), ph2);
            }
        }
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

namespace {

std::atomic<int> g_pool_impl{0};          // 0: by size, 1: register streaming, 2: bulk copy where the layout allows
std::atomic<int> g_pool_stages{0};        // 0: default
std::atomic<int> g_pool_stage_bytes{0};   // 0: default
std::atomic<int> g_pool_copy_bytes{0};    // 0: one bulk copy per stage
constexpr int kBulkStagesDefault = 3;
constexpr int kBulkStageBytesDefault = 32768;

// Launches the bulk-copy pooling kernel when every part's row fits a stage and a row needs at most
// kBulkMaxConsumers threads; *launched tells whether it did.
template <typename TIn, typename TOut>
msa_status launch_pool_bulk(PoolArgs a, cudaStream_t s, bool* launched) {
    constexpr int VEC = 16 / sizeof(TIn);
    *launched = false;
    a.tab_bytes = (a.d / 2) * (int)sizeof(float2);
    const int S = g_pool_stages.load() > 0 ? g_pool_stages.load() : kBulkStagesDefault;
    const int SB = g_pool_stage_bytes.load() > 0 ? g_pool_stage_bytes.load() : kBulkStageBytesDefault;
    int max_e = 0;
    for (int i = 0; i < a.n_parts; ++i) {
        const int part = a.parts[i];
        const int E = a.heads[part] * a.d;
        const int row_bytes = E * (int)sizeof(TIn);
        // rotated keys carry their table rows in the stage
        const int per_row = row_bytes + ((part == 0 && a.fuse_rope) ? a.tab_bytes : 0);
        if (per_row > SB || row_bytes % 16 != 0 || a.tab_bytes % 16 != 0) return MSA_OK;
        a.rows_per_stage[part] = SB / per_row;
        const int CB = g_pool_copy_bytes.load();
        a.rows_per_copy[part] = CB > 0 ? (CB / row_bytes > 0 ? CB / row_bytes : 1) : a.rows_per_stage[part];
        max_e = E > max_e ? E : max_e;
    }
    const int nc = (max_e / VEC + 31) / 32 * 32;
    if (nc > kBulkMaxConsumers) return MSA_OK;
    a.n_stages = S;
    a.stage_bytes = SB;
    const size_t smem = (size_t)S * SB + 2 * (size_t)S * sizeof(uint64_t) + 16;
    static std::mutex mu;
    static size_t opted[64] = {0};
    int dev = 0;
    MSA_CUDA_TRY(cudaGetDevice(&dev));
    {
        std::lock_guard<std::mutex> lk(mu);
        if (dev < 0 || dev >= 64 || opted[dev] < smem) {
            MSA_CUDA_TRY(cudaFuncSetAttribute(pool_bulk_kernel<TIn, TOut>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              (int)smem));
            // ask for the whole unified L1 as shared memory, so the occupancy computed below is reached
            MSA_CUDA_TRY(cudaFuncSetAttribute(pool_bulk_kernel<TIn, TOut>,
                                              cudaFuncAttributePreferredSharedMemoryCarveout, 100));
            if (dev >= 0 && dev < 64) opted[dev] = smem;
        }
    }
    int occ = 0;
    MSA_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, pool_bulk_kernel<TIn, TOut>, nc + 32, smem));
    if (occ < 1) return MSA_OK;
    const int64_t n_items = a.n_chunks * a.n_parts;
    const int64_t cap = (int64_t)sm_count() * occ;
    const unsigned grid = (unsigned)(n_items < cap ? n_items : cap);
    pool_bulk_kernel<TIn, TOut><<<grid, nc + 32, smem, s>>>(a);
    MSA_LAUNCH_CHECK();
    *launched = true;
    return MSA_OK;
}

}  // namespace

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
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // By size: the register-streaming kernel (one block per chunk and part) keeps more loads in flight
    // per SM once its grid runs for several waves; on grids of under two waves its rotated-key blocks,
    // which wait on their RoPE table reads, make a tail, and the bulk-copy kernel (table rows staged
    // with the keys, items spread over a persistent grid) is faster.
    int impl = g_pool_impl.load();
    if (impl == 0) {
        int occ = 0;
        MSA_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &occ, in_dt == MSA_BF16 ? (out_dt == MSA_BF16 ? (const void*)pool_kernel<__nv_bfloat16, __nv_bfloat16>
                                                         : (const void*)pool_kernel<__nv_bfloat16, float>)
                                   : (out_dt == MSA_BF16 ? (const void*)pool_kernel<float, __nv_bfloat16>
                                                         : (const void*)pool_kernel<float, float>),
            kPoolThreads, 0));
        impl = n_chunks * a.n_parts <= 2 * (int64_t)sm_count() * (occ > 0 ? occ : 1) ? 2 : 1;
    }
    if (impl == 2) {
        bool launched = false;
        if (in_dt == MSA_BF16 && out_dt == MSA_BF16)
            MSA_RETURN_IF((launch_pool_bulk<__nv_bfloat16, __nv_bfloat16>(a, s, &launched)));
        else if (in_dt == MSA_BF16)
            MSA_RETURN_IF((launch_pool_bulk<__nv_bfloat16, float>(a, s, &launched)));
        else if (out_dt == MSA_BF16)
            MSA_RETURN_IF((launch_pool_bulk<float, __nv_bfloat16>(a, s, &launched)));
        else
            MSA_RETURN_IF((launch_pool_bulk<float, float>(a, s, &launched)));
        if (launched) return MSA_OK;
    }
    const int64_t cap = 1 << 20;
    const int64_t per_part = n_chunks < cap ? n_chunks : cap;
    dim3 grid((unsigned)(per_part * a.n_parts));
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

msa_status msa_pool_set_impl(int impl) {
    MSA_REQUIRE(impl >= 0 && impl <= 2, "msa_pool_set_impl: impl must be 0, 1 or 2");
    g_pool_impl.store(impl);
    return MSA_OK;
}

msa_status msa_pool_set_pipeline(int n_stages, int stage_bytes, int copy_bytes) {
    MSA_REQUIRE(n_stages == 0 || (n_stages >= 2 && n_stages <= 16), "msa_pool_set_pipeline: n_stages must be 0 or in [2, 16]");
    MSA_REQUIRE(stage_bytes == 0 || (stage_bytes >= 2048 && stage_bytes <= 65536 && stage_bytes % 1024 == 0),
                "msa_pool_set_pipeline: stage_bytes must be 0 or a multiple of 1024 in [2048, 65536]");
    const int S = n_stages ? n_stages : kBulkStagesDefault;
    const int SB = stage_bytes ? stage_bytes : kBulkStageBytesDefault;
    MSA_REQUIRE((int64_t)S * SB <= 200 * 1024, "msa_pool_set_pipeline: %d stages of %d bytes exceed 200 KiB", S, SB);
    MSA_REQUIRE(copy_bytes >= 0 && copy_bytes % 16 == 0, "msa_pool_set_pipeline: copy_bytes must be a multiple of 16");
    g_pool_stages.store(n_stages);
    g_pool_stage_bytes.store(stage_bytes);
    g_pool_copy_bytes.store(copy_bytes);
    return MSA_OK;
}

}  // extern "C"
