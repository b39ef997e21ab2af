// Backward pass of the MSA hot path for end-to-end training: sparse attention, the fetch of the
// selected documents, chunk-mean pooling with document-wise RoPE and index normalisation, the
// auxiliary router loss and the router scores.
//
// Attention (bf16 inputs, fp32 gradients) follows the two-kernel split of flash-attention training:
//   rows r = (token t, head h) of kv head g, keys = [memory rows ; local keys], P = softmax of the
//   scaled logits from the forward log-sum-exp, D_r = sum_d dO_r . O_r;
//   dK/dV kernel: one block per 64-key tile accumulates, over every row block, dV += P^T dO and
//     dK += dS^T Q with dS = P * (dP - D), dP = dO V^T — no atomics, each key written once;
//   dQ kernel: one block per 64-row block accumulates dQ += dS K over the key tiles.
// Products on tensor cores (mma.sync m16n8k16, bf16 operands, fp32 accumulation); P and dS are
// rounded to bf16 as operands, exactly as P is in the forward P V product.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "mma.cuh"

namespace msa {
namespace {

constexpr int kD = 128;
constexpr int kTile = 64;           // keys per key tile, rows per row block
constexpr int kStride = kD + 8;     // bf16 elements per shared-memory row (conflict-free fragment loads)
constexpr float kLog2e = 1.4426950408889634f;

typedef __nv_bfloat16 Tile[kTile][kStride];

struct BwdArgs {
    const __nv_bfloat16* q;
    const __nv_bfloat16* mem_kv;
    const int32_t* mem_len;
    int max_mem;
    const __nv_bfloat16* local_k;
    const __nv_bfloat16* local_v;
    int L_max, L, q_start;
    int T, hq, hkv;
    float scale, scale_log2e;
    const __nv_bfloat16* out;
    const __nv_bfloat16* dout;
    const float* lse;        // natural log
    float* Dvec;             // [n_q * T * hq]
    float* dq;               // [n_q][T][hq][d]
    float* dmem;             // [n_q][max_mem][2][hkv][d]
    float* dlk;              // [n_q][L_max][hkv][d]
    float* dlv;
};

__device__ __forceinline__ bool key_visible(int kk, int mem_len, int n_keys, int q_start, int t) {
    return kk < mem_len || (kk < n_keys && kk - mem_len <= q_start + t);
}

// D_r = sum_d dO . O: one warp per row, lane l owns dims 4l..4l+3.
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const __nv_bfloat16* __restrict__ out,
                                                            const __nv_bfloat16* __restrict__ dout, int64_t rows,
                                                            float* __restrict__ Dvec) {
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const uint2 o = *reinterpret_cast<const uint2*>(out + row * kD + lane * 4);
    const uint2 g = *reinterpret_cast<const uint2*>(dout + row * kD + lane * 4);
    const uint32_t ow[2] = {o.x, o.y}, gw[2] = {g.x, g.y};
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        s = fmaf(__uint_as_float(ow[i] << 16), __uint_as_float(gw[i] << 16), s);
        s = fmaf(__uint_as_float(ow[i] & 0xffff0000u), __uint_as_float(gw[i] & 0xffff0000u), s);
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
    if (lane == 0) Dvec[row] = s;
}

// Key kk of query qi (memory row or local key), kv head g: address of its K (which = 0) or V row.
__device__ __forceinline__ const __nv_bfloat16* key_row(const BwdArgs& a, int qi, int g, int kk, int mem_len,
                                                        int which) {
    if (kk < mem_len) return a.mem_kv + (((int64_t)qi * a.max_mem + kk) * 2 + which) * a.hkv * kD + g * kD;
    return (which ? a.local_v : a.local_k) + (((int64_t)qi * a.L_max + (kk - mem_len)) * a.hkv + g) * kD;
}

// Stage 64 rows (keys or query rows) of 128 bf16 into a shared tile with asynchronous copies;
// row_ptr(i) gives row i's address or nullptr for a zero row.
template <typename F>
__device__ __forceinline__ void stage_rows(Tile& dst, F row_ptr, const void* any_valid) {
    for (int v = threadIdx.x; v < kTile * (kD / 8); v += blockDim.x) {
        const int r = v / (kD / 8), c = (v % (kD / 8)) * 8;
        const __nv_bfloat16* src = row_ptr(r);
        cp_async16(&dst[r][c], src ? src + c : any_valid, src != nullptr);
    }
}

// ---------------------------------------------------------------------------------------------
// dK, dV: block (key tile, kv head g, query qi); warp w owns keys kb + 16w .. kb + 16w + 15.
template <int G>
__global__ void __launch_bounds__(128) attn_bwd_dkdv_kernel(const BwdArgs a) {
    extern __shared__ __align__(16) unsigned char bwd_smem[];
    Tile& Ks = *reinterpret_cast<Tile*>(bwd_smem);
    Tile& Vs = *reinterpret_cast<Tile*>(bwd_smem + sizeof(Tile));
    Tile& Qs = *reinterpret_cast<Tile*>(bwd_smem + 2 * sizeof(Tile));
    Tile& Os = *reinterpret_cast<Tile*>(bwd_smem + 3 * sizeof(Tile));
    float* lse_s = reinterpret_cast<float*>(bwd_smem + 4 * sizeof(Tile));   // [64], log2 units
    float* D_s = lse_s + kTile;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
    const int qi = blockIdx.z, g = blockIdx.y, kb = blockIdx.x * kTile;
    const int mem_len = max(min(a.mem_len[qi], a.max_mem), 0);
    const int n_keys = mem_len + a.L;
    if (kb >= n_keys) return;
    const int n_rows = a.T * G;
    const float ninf = -__int_as_float(0x7f800000);

    stage_rows(Ks, [&](int r) { return kb + r < n_keys ? key_row(a, qi, g, kb + r, mem_len, 0) : nullptr; }, a.q);
    stage_rows(Vs, [&](int r) { return kb + r < n_keys ? key_row(a, qi, g, kb + r, mem_len, 1) : nullptr; }, a.q);

    // rows that can see a local key j satisfy t >= j - q_start: skip row blocks that see none of this tile
    int t_first = 0;
    if (kb >= mem_len) t_first = max(0, kb - mem_len - a.q_start);

    float dk[kD / 8][4], dv[kD / 8][4];
#pragma unroll
    for (int nd = 0; nd < kD / 8; ++nd)
#pragma unroll
        for (int e = 0; e < 4; ++e) dk[nd][e] = dv[nd][e] = 0.f;
    const int key_a = kb + warp * 16 + gid, key_b = key_a + 8;
    const int kr_a = warp * 16 + gid, kr_b = kr_a + 8;   // rows of Ks / Vs

    for (int r0 = (t_first * G / kTile) * kTile; r0 < n_rows; r0 += kTile) {
        __syncthreads();                                  // previous row block's readers are done
        auto row_src = [&](const __nv_bfloat16* base, int r) -> const __nv_bfloat16* {
            const int row = r0 + r;
            if (row >= n_rows) return nullptr;
            return base + (((int64_t)qi * a.T + row / G) * a.hq + g * G + row % G) * kD;
        };
        stage_rows(Qs, [&](int r) { return row_src(a.q, r); }, a.q);
        stage_rows(Os, [&](int r) { return row_src(a.dout, r); }, a.q);
        if (threadIdx.x < kTile) {
            const int row = r0 + threadIdx.x;
            float l2 = ninf, dd = 0.f;
            if (row < n_rows) {
                const int64_t ri = ((int64_t)qi * a.T + row / G) * a.hq + g * G + row % G;
                l2 = a.lse[ri] * kLog2e;
                dd = a.Dvec[ri];
            }
            lse_s[threadIdx.x] = l2;
            D_s[threadIdx.x] = dd;
        }
        cp_async_wait_all();
        __syncthreads();

        // S^T = K Q^T and dP^T = V dO^T for this warp's 16 keys x 64 rows
        float st[kTile / 8][4], dpt[kTile / 8][4];
#pragma unroll
        for (int nb = 0; nb < kTile / 8; ++nb)
#pragma unroll
            for (int e = 0; e < 4; ++e) st[nb][e] = dpt[nb][e] = 0.f;
#pragma unroll
        for (int s = 0; s < kD / 16; ++s) {
            uint32_t ka[4], va[4];
            ka[0] = *reinterpret_cast<const uint32_t*>(&Ks[kr_a][s * 16 + tig * 2]);
            ka[1] = *reinterpret_cast<const uint32_t*>(&Ks[kr_b][s * 16 + tig * 2]);
            ka[2] = *reinterpret_cast<const uint32_t*>(&Ks[kr_a][s * 16 + 8 + tig * 2]);
            ka[3] = *reinterpret_cast<const uint32_t*>(&Ks[kr_b][s * 16 + 8 + tig * 2]);
            va[0] = *reinterpret_cast<const uint32_t*>(&Vs[kr_a][s * 16 + tig * 2]);
            va[1] = *reinterpret_cast<const uint32_t*>(&Vs[kr_b][s * 16 + tig * 2]);
            va[2] = *reinterpret_cast<const uint32_t*>(&Vs[kr_a][s * 16 + 8 + tig * 2]);
            va[3] = *reinterpret_cast<const uint32_t*>(&Vs[kr_b][s * 16 + 8 + tig * 2]);
#pragma unroll
            for (int nb = 0; nb < kTile / 8; ++nb) {
                const uint32_t* qrow = reinterpret_cast<const uint32_t*>(&Qs[nb * 8 + gid][0]);
                const uint32_t* orow = reinterpret_cast<const uint32_t*>(&Os[nb * 8 + gid][0]);
                mma_bf16_16816(st[nb], ka, qrow[s * 8 + tig], qrow[s * 8 + 4 + tig]);
                mma_bf16_16816(dpt[nb], va, orow[s * 8 + tig], orow[s * 8 + 4 + tig]);
            }
        }
        // P^T and dS^T (elements: key key_a / key_b, row r0 + nb*8 + 2 tig + (e & 1))
#pragma unroll
        for (int nb = 0; nb < kTile / 8; ++nb) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int rl = nb * 8 + tig * 2 + (e & 1);
                const int row = r0 + rl;
                const int key = e < 2 ? key_a : key_b;
                const float l2 = lse_s[rl];
                const bool vis = row < n_rows && l2 != ninf && key_visible(key, mem_len, n_keys, a.q_start, row / G);
                const float p = vis ? exp2f(st[nb][e] * a.scale_log2e - l2) : 0.f;
                st[nb][e] = p;
                dpt[nb][e] = p * (dpt[nb][e] - D_s[rl]);
            }
        }
        // dV += P^T dO, dK += dS^T Q (rows are the reduction dimension, B fragments by ldmatrix.trans)
#pragma unroll
        for (int s2 = 0; s2 < kTile / 16; ++s2) {
            uint32_t pa[4], da[4];
            pa[0] = pack_bf16(st[2 * s2][0], st[2 * s2][1]);
            pa[1] = pack_bf16(st[2 * s2][2], st[2 * s2][3]);
            pa[2] = pack_bf16(st[2 * s2 + 1][0], st[2 * s2 + 1][1]);
            pa[3] = pack_bf16(st[2 * s2 + 1][2], st[2 * s2 + 1][3]);
            da[0] = pack_bf16(dpt[2 * s2][0], dpt[2 * s2][1]);
            da[1] = pack_bf16(dpt[2 * s2][2], dpt[2 * s2][3]);
            da[2] = pack_bf16(dpt[2 * s2 + 1][0], dpt[2 * s2 + 1][1]);
            da[3] = pack_bf16(dpt[2 * s2 + 1][2], dpt[2 * s2 + 1][3]);
            const int rr = s2 * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int nd = 0; nd < kD / 8; nd += 2) {
                const int dim = nd * 8 + (lane >> 4) * 8;
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(&Os[rr][dim], b0, b1, b2, b3);
                mma_bf16_16816(dv[nd], pa, b0, b1);
                mma_bf16_16816(dv[nd + 1], pa, b2, b3);
                ldmatrix_x4_trans(&Qs[rr][dim], b0, b1, b2, b3);
                mma_bf16_16816(dk[nd], da, b0, b1);
                mma_bf16_16816(dk[nd + 1], da, b2, b3);
            }
        }
    }

    // write this thread's two keys' gradients (dims nd*8 + 2 tig, +1)
    auto dst = [&](int key, int which) -> float* {
        if (key < mem_len) return a.dmem + (((int64_t)qi * a.max_mem + key) * 2 + which) * a.hkv * kD + g * kD;
        return (which ? a.dlv : a.dlk) + (((int64_t)qi * a.L_max + (key - mem_len)) * a.hkv + g) * kD;
    };
    if (key_a < n_keys) {
        float* pk = dst(key_a, 0);
        float* pv = dst(key_a, 1);
#pragma unroll
        for (int nd = 0; nd < kD / 8; ++nd) {
            *reinterpret_cast<float2*>(pk + nd * 8 + tig * 2) = make_float2(dk[nd][0] * a.scale, dk[nd][1] * a.scale);
            *reinterpret_cast<float2*>(pv + nd * 8 + tig * 2) = make_float2(dv[nd][0], dv[nd][1]);
        }
    }
    if (key_b < n_keys) {
        float* pk = dst(key_b, 0);
        float* pv = dst(key_b, 1);
#pragma unroll
        for (int nd = 0; nd < kD / 8; ++nd) {
            *reinterpret_cast<float2*>(pk + nd * 8 + tig * 2) = make_float2(dk[nd][2] * a.scale, dk[nd][3] * a.scale);
            *reinterpret_cast<float2*>(pv + nd * 8 + tig * 2) = make_float2(dv[nd][2], dv[nd][3]);
        }
    }
}

// ---------------------------------------------------------------------------------------------
// dQ: block (64-row block, kv head g, query qi); warp w owns rows r0 + 16w .. + 15 (as the forward).
template <int G>
__global__ void __launch_bounds__(128) attn_bwd_dq_kernel(const BwdArgs a) {
    __shared__ __align__(16) Tile Ks;
    __shared__ __align__(16) Tile Vs;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
    const int qi = blockIdx.z, g = blockIdx.y;
    const int n_rows = a.T * G;
    const int r0 = blockIdx.x * kTile;
    const int r_last = min(r0 + kTile, n_rows) - 1;
    const int mem_len = max(min(a.mem_len[qi], a.max_mem), 0);
    const int n_keys_all = mem_len + a.L;
    const int n_keys = mem_len + max(min(a.L, a.q_start + r_last / G + 1), 0);
    const float ninf = -__int_as_float(0x7f800000);

    const int ra = r0 + warp * 16 + gid, rb = ra + 8;
    const bool va = ra < n_rows, vb = rb < n_rows;
    const int ta = ra / G, tb = rb / G;
    const int64_t ia = ((int64_t)qi * a.T + ta) * a.hq + g * G + ra % G;
    const int64_t ib = ((int64_t)qi * a.T + tb) * a.hq + g * G + rb % G;
    uint32_t qf[kD / 16][4], of[kD / 16][4];
    {
        const uint32_t* qa = reinterpret_cast<const uint32_t*>(a.q + ia * kD);
        const uint32_t* qb = reinterpret_cast<const uint32_t*>(a.q + ib * kD);
        const uint32_t* oa = reinterpret_cast<const uint32_t*>(a.dout + ia * kD);
        const uint32_t* ob = reinterpret_cast<const uint32_t*>(a.dout + ib * kD);
#pragma unroll
        for (int s = 0; s < kD / 16; ++s) {
            qf[s][0] = va ? qa[s * 8 + tig] : 0u;
            qf[s][1] = vb ? qb[s * 8 + tig] : 0u;
            qf[s][2] = va ? qa[s * 8 + 4 + tig] : 0u;
            qf[s][3] = vb ? qb[s * 8 + 4 + tig] : 0u;
            of[s][0] = va ? oa[s * 8 + tig] : 0u;
            of[s][1] = vb ? ob[s * 8 + tig] : 0u;
            of[s][2] = va ? oa[s * 8 + 4 + tig] : 0u;
            of[s][3] = vb ? ob[s * 8 + 4 + tig] : 0u;
        }
    }
    const float l2a = va ? a.lse[ia] * kLog2e : ninf, l2b = vb ? a.lse[ib] * kLog2e : ninf;
    const float Da = va ? a.Dvec[ia] : 0.f, Db = vb ? a.Dvec[ib] : 0.f;
    float dq[kD / 8][4];
#pragma unroll
    for (int nd = 0; nd < kD / 8; ++nd) dq[nd][0] = dq[nd][1] = dq[nd][2] = dq[nd][3] = 0.f;

    for (int kb = 0; kb < n_keys; kb += kTile) {
        __syncthreads();
        stage_rows(Ks, [&](int r) { return kb + r < n_keys ? key_row(a, qi, g, kb + r, mem_len, 0) : nullptr; }, a.q);
        stage_rows(Vs, [&](int r) { return kb + r < n_keys ? key_row(a, qi, g, kb + r, mem_len, 1) : nullptr; }, a.q);
        cp_async_wait_all();
        __syncthreads();
        float sc[kTile / 8][4], dp[kTile / 8][4];
#pragma unroll
        for (int nb = 0; nb < kTile / 8; ++nb) {
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[nb][e] = dp[nb][e] = 0.f;
            const uint32_t* krow = reinterpret_cast<const uint32_t*>(&Ks[nb * 8 + gid][0]);
            const uint32_t* vrow = reinterpret_cast<const uint32_t*>(&Vs[nb * 8 + gid][0]);
#pragma unroll
            for (int s = 0; s < kD / 16; ++s) {
                mma_bf16_16816(sc[nb], qf[s], krow[s * 8 + tig], krow[s * 8 + 4 + tig]);
                mma_bf16_16816(dp[nb], of[s], vrow[s * 8 + tig], vrow[s * 8 + 4 + tig]);
            }
        }
#pragma unroll
        for (int nb = 0; nb < kTile / 8; ++nb) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int kk = kb + nb * 8 + tig * 2 + (e & 1);
                const bool first = e < 2;
                const bool vis = (first ? va : vb) && (first ? l2a : l2b) != ninf &&
                                 key_visible(kk, mem_len, n_keys_all, a.q_start, first ? ta : tb);
                const float p = vis ? exp2f(sc[nb][e] * a.scale_log2e - (first ? l2a : l2b)) : 0.f;
                dp[nb][e] = p * (dp[nb][e] - (first ? Da : Db));
            }
        }
        // dQ += dS K: dS fragments as A, K (keys are the reduction dimension) by ldmatrix.trans
#pragma unroll
        for (int s2 = 0; s2 < kTile / 16; ++s2) {
            uint32_t da[4];
            da[0] = pack_bf16(dp[2 * s2][0], dp[2 * s2][1]);
            da[1] = pack_bf16(dp[2 * s2][2], dp[2 * s2][3]);
            da[2] = pack_bf16(dp[2 * s2 + 1][0], dp[2 * s2 + 1][1]);
            da[3] = pack_bf16(dp[2 * s2 + 1][2], dp[2 * s2 + 1][3]);
            const int key = s2 * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int nd = 0; nd < kD / 8; nd += 2) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(&Ks[key][nd * 8 + (lane >> 4) * 8], b0, b1, b2, b3);
                mma_bf16_16816(dq[nd], da, b0, b1);
                mma_bf16_16816(dq[nd + 1], da, b2, b3);
            }
        }
    }
#pragma unroll
    for (int nd = 0; nd < kD / 8; ++nd) {
        if (va) *reinterpret_cast<float2*>(a.dq + ia * kD + nd * 8 + tig * 2) =
                    make_float2(dq[nd][0] * a.scale, dq[nd][1] * a.scale);
        if (vb) *reinterpret_cast<float2*>(a.dq + ib * kD + nd * 8 + tig * 2) =
                    make_float2(dq[nd][2] * a.scale, dq[nd][3] * a.scale);
    }
}

constexpr size_t kDkdvSmem = 4 * sizeof(Tile) + 2 * kTile * sizeof(float);

template <int G>
msa_status launch_attn_bwd_g(const BwdArgs& a, int n_q, cudaStream_t s) {
    const int key_tiles = (a.max_mem + a.L + kTile - 1) / kTile;
    if (key_tiles > 0) {
        MSA_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dkdv_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)kDkdvSmem));
        attn_bwd_dkdv_kernel<G><<<dim3(key_tiles, a.hkv, n_q), 128, kDkdvSmem, s>>>(a);
        MSA_LAUNCH_CHECK();
    }
    attn_bwd_dq_kernel<G><<<dim3((a.T * G + kTile - 1) / kTile, a.hkv, n_q), 128, 0, s>>>(a);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

// ---------------------------------------------------------------------------------------------
// Fetch backward: the memory rows' gradients are added to the chunk rows they were copied from.
// One block per (rank, query), fp32 atomic adds (a document selected by several queries sums).
__global__ void __launch_bounds__(256) gather_bwd_kernel(const float* __restrict__ dmem, int64_t n_chunks,
                                                         const int64_t* __restrict__ doc_chunk_off, int64_t n_docs,
                                                         const int32_t* __restrict__ idx, int k, int row_len,
                                                         int max_mem, float* __restrict__ dkvbar, int* err) {
    const int q = blockIdx.y, r = blockIdx.x;
    const int32_t* sel = idx + (int64_t)q * k;
    int64_t at = 0;
    for (int j = 0; j <= r; ++j) {
        const int32_t doc = sel[j];
        if (doc < 0 || doc >= n_docs || doc_chunk_off[doc] < 0 || doc_chunk_off[doc + 1] < doc_chunk_off[doc] ||
            doc_chunk_off[doc + 1] > n_chunks) {
            if (threadIdx.x == 0) record_device_error(err, MSA_DEV_BAD_INDEX);
            return;
        }
        if (j < r) at += doc_chunk_off[doc + 1] - doc_chunk_off[doc];
    }
    const int64_t c0 = doc_chunk_off[sel[r]], rows = doc_chunk_off[sel[r] + 1] - c0;
    if (at + rows > max_mem) {
        if (threadIdx.x == 0) record_device_error(err, MSA_DEV_BAD_INDEX);
        return;
    }
    const float* src = dmem + ((int64_t)q * max_mem + at) * row_len;
    float* dst = dkvbar + c0 * row_len;
    for (int64_t i = threadIdx.x; i < rows * row_len; i += blockDim.x) atomicAdd(dst + i, src[i]);
}

// ---------------------------------------------------------------------------------------------
// Pooling backward: block per chunk (grid-stride), tensor part from blockIdx (K, V, K^R).
//   K: every token t of chunk c gets R(-p_t) dK-bar_c / n (the rotation's transpose, p_t its
//      position in its document); V: dV-bar_c / n; K^R: through the per-head normalisation of the
//      index when it was normalised (the chunk's raw mean is recomputed from the tokens), then / n.
struct PoolBwdArgs {
    const float* dkvbar;     // [C][2][hkv][d] or null
    const float* dkr_index;  // [C][hr][d] or null
    const void* kr;          // tokens [n_tok][hr][d] of kr_dt (normalised index only)
    int kr_bf16;
    int hkv, hr, d;
    const int64_t* doc_tok_off;
    const int64_t* doc_chunk_off;
    const int32_t* chunk_doc;
    int64_t n_docs, n_chunks, n_tok;
    int chunk;
    int fuse_rope, normalize;
    const float2* cs;
    int64_t max_pos;
    float* dk;
    float* dv;
    float* dkr;
    int n_parts;
    int parts[3];
    int* err;
};

__device__ __forceinline__ float load_elem(const void* p, int64_t i, int bf16) {
    if (bf16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
    return static_cast<const float*>(p)[i];
}

__global__ void __launch_bounds__(128) pool_bwd_kernel(const PoolBwdArgs a) {
    __shared__ float gsh[1024 + 32];
    const int part = a.parts[blockIdx.x % a.n_parts];
    const int64_t c_stride = gridDim.x / a.n_parts;
    const int d = a.d;
    for (int64_t c = blockIdx.x / a.n_parts; c < a.n_chunks; c += c_stride) {
        const int64_t doc = a.chunk_doc[c];
        if (doc < 0 || doc >= a.n_docs) {
            if (threadIdx.x == 0) record_device_error(a.err, MSA_DEV_BAD_INDEX);
            continue;
        }
        const int64_t doc_start = a.doc_tok_off[doc];
        const int64_t t0 = doc_start + (c - a.doc_chunk_off[doc]) * (int64_t)a.chunk;
        const int64_t t1 = min(t0 + (int64_t)a.chunk, a.doc_tok_off[doc + 1]);
        if (t0 < doc_start || t0 >= t1 || t1 > a.n_tok) {
            if (threadIdx.x == 0) record_device_error(a.err, MSA_DEV_BAD_INDEX);
            continue;
        }
        const float inv_n = 1.0f / (float)(t1 - t0);
        if (part == 0 || part == 1) {
            const int E = a.hkv * d;
            const float* g = a.dkvbar + (c * 2 + part) * (int64_t)E;
            float* out = part == 0 ? a.dk : a.dv;
            for (int64_t t = t0; t < t1; ++t) {
                const int64_t p = t - doc_start;
                const bool rot = part == 0 && a.fuse_rope;
                if (rot && p >= a.max_pos && threadIdx.x == 0) record_device_error(a.err, MSA_DEV_ROPE_POSITION);
                for (int e = threadIdx.x; e < E; e += blockDim.x) {
                    float x = g[e] * inv_n;
                    if (rot && p < a.max_pos) {
                        const int i = e % d;
                        const int hi = i < d / 2 ? i : i - d / 2;
                        const float2 cs = a.cs[p * (d / 2) + hi];
                        const int partner = i < d / 2 ? e + d / 2 : e - d / 2;
                        const float y = g[partner] * inv_n;
                        // transpose of the rotation: first half x cos + y sin, second half x cos - y sin
                        x = i < d / 2 ? fmaf(x, cs.x, y * cs.y) : fmaf(x, cs.x, -y * cs.y);
                    }
                    out[t * E + e] = x;
                }
            }
        } else {
            const int E = a.hr * d;
            const float* g = a.dkr_index + c * (int64_t)E;
            // gradient with respect to the raw pooled router key of every head
            for (int e = threadIdx.x; e < E; e += blockDim.x) gsh[e] = g[e];
            __syncthreads();
            if (a.normalize) {
                // raw chunk mean into shared memory (second half of the buffer is not enough for
                // E = 1024, so the mean overwrites nothing: use registers per element)
                for (int h = threadIdx.x >> 5; h < a.hr; h += blockDim.x >> 5) {
                    const int lane = threadIdx.x & 31;
                    float ss = 0.f, dot = 0.f;
                    float mean[8];
                    for (int j = 0; j < d / 32 && j < 8; ++j) {
                        const int e = h * d + lane + 32 * j;
                        float m = 0.f;
                        for (int64_t t = t0; t < t1; ++t) m += load_elem(a.kr, t * E + e, a.kr_bf16);
                        m *= inv_n;
                        mean[j] = m;
                        ss = fmaf(m, m, ss);
                        dot = fmaf(m, gsh[e], dot);
                    }
#pragma unroll
                    for (int o = 16; o >= 1; o >>= 1) {
                        ss += __shfl_xor_sync(0xffffffffu, ss, o);
                        dot += __shfl_xor_sync(0xffffffffu, dot, o);
                    }
                    const float nrm = sqrtf(ss);
                    for (int j = 0; j < d / 32 && j < 8; ++j) {
                        const int e = h * d + lane + 32 * j;
                        // (g - k_hat (k_hat . g)) / |k| with k_hat = mean / |mean|
                        gsh[e] = nrm > 0.f ? (gsh[e] - mean[j] * dot / (nrm * nrm)) / nrm : 0.f;
                    }
                }
                __syncthreads();
            }
            for (int64_t t = t0; t < t1; ++t)
                for (int e = threadIdx.x; e < E; e += blockDim.x) a.dkr[t * E + e] = gsh[e] * inv_n;
            __syncthreads();
        }
    }
}

// ---------------------------------------------------------------------------------------------
// Auxiliary router loss: one block per query. s = doc_scores / tau, lse = log sum exp s,
// loss_q = -(1/|E|) sum_e (s_e - lse), grad = (softmax(s) - y) / tau / n_q with y = 1/|E| on E.
__global__ void __launch_bounds__(1024) aux_loss_kernel(const float* __restrict__ scores, int64_t n_docs,
                                                        const int32_t* __restrict__ evidence, int n_ev, float tau,
                                                        int n_q, float* __restrict__ loss, float* __restrict__ grad,
                                                        int* err) {
    __shared__ float red[32];
    __shared__ float bcast;
    const int q = blockIdx.x;
    const float* s = scores + (int64_t)q * n_docs;
    const float inv_tau = 1.0f / tau;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    auto block_reduce = [&](float v, bool is_max) -> float {
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float w = __shfl_xor_sync(0xffffffffu, v, o);
            v = is_max ? fmaxf(v, w) : v + w;
        }
        if (lane == 0) red[warp] = v;
        __syncthreads();
        if (warp == 0) {
            v = lane < (int)(blockDim.x >> 5) ? red[lane] : (is_max ? -__int_as_float(0x7f800000) : 0.f);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                const float w = __shfl_xor_sync(0xffffffffu, v, o);
                v = is_max ? fmaxf(v, w) : v + w;
            }
            if (lane == 0) bcast = v;
        }
        __syncthreads();
        const float r = bcast;
        __syncthreads();
        return r;
    };
    float m = -__int_as_float(0x7f800000);
    for (int64_t i = threadIdx.x; i < n_docs; i += blockDim.x) m = fmaxf(m, s[i] * inv_tau);
    m = block_reduce(m, true);
    float z = 0.f;
    for (int64_t i = threadIdx.x; i < n_docs; i += blockDim.x) z += expf(s[i] * inv_tau - m);
    z = block_reduce(z, false);
    const float lse = m + logf(z);
    // evidence documents of this query (-1 = padding)
    int n_valid = 0;
    float acc = 0.f;
    for (int j = 0; j < n_ev; ++j) {
        const int32_t e = evidence[(int64_t)q * n_ev + j];
        if (e >= 0 && e < n_docs) {
            ++n_valid;
            acc += s[e] * inv_tau - lse;
        } else if (e != -1 && threadIdx.x == 0) {
            record_device_error(err, MSA_DEV_BAD_INDEX);
        }
    }
    const float yv = n_valid > 0 ? 1.0f / n_valid : 0.f;
    if (threadIdx.x == 0 && loss) loss[q] = n_valid > 0 ? -acc / n_valid : 0.f;
    const float gs = inv_tau / n_q;
    for (int64_t i = threadIdx.x; i < n_docs; i += blockDim.x) {
        float y = 0.f;
        for (int j = 0; j < n_ev; ++j)
            if (evidence[(int64_t)q * n_ev + j] == i) y += yv;
        grad[(int64_t)q * n_docs + i] = (expf(s[i] * inv_tau - lse) - y) * gs;
    }
}

// ---------------------------------------------------------------------------------------------
// Router backward.
// (1) qhat: unit router queries per head, divided by H (the folded form) [n_q][T][H*d] fp32.
__global__ void __launch_bounds__(128) route_bwd_qhat_kernel(const void* __restrict__ qr, int qr_bf16, int64_t rows,
                                                             int H, int d, float* __restrict__ qhat) {
    // one warp per (row, head)
    const int64_t w = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= rows * H) return;
    float ss = 0.f;
    for (int i = lane; i < d; i += 32) {
        const float x = load_elem(qr, w * d + i, qr_bf16);
        ss = fmaf(x, x, ss);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = ss > 0.f ? 1.0f / (sqrtf(ss) * H) : 0.f;
    for (int i = lane; i < d; i += 32) qhat[w * d + i] = load_elem(qr, w * d + i, qr_bf16) * inv;
}

// (2) per (query, chunk): best folded score over the query tokens and the first token attaining it.
//     Block per chunk (grid-stride), the chunk's index row in shared memory, warp per token.
__global__ void __launch_bounds__(256) route_bwd_best_kernel(const void* __restrict__ index, int idx_bf16,
                                                             int64_t n_chunks, const float* __restrict__ qhat, int n_q,
                                                             int T, int K, float* __restrict__ best,
                                                             int* __restrict__ best_t) {
    __shared__ float krow[1024];
    __shared__ float wbest[8];
    __shared__ int wt[8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x) {
        __syncthreads();
        for (int i = threadIdx.x; i < K; i += blockDim.x) krow[i] = load_elem(index, c * K + i, idx_bf16);
        __syncthreads();
        for (int q = 0; q < n_q; ++q) {
            float bs = -__int_as_float(0x7f800000);
            int bt = 0x7fffffff;
            for (int t = warp; t < T; t += 8) {
                const float* qv = qhat + ((int64_t)q * T + t) * K;
                float acc = 0.f;
                for (int i = lane; i < K; i += 32) acc = fmaf(qv[i], krow[i], acc);
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                if (acc > bs) { bs = acc; bt = t; }             // t increases: first maximum kept
            }
            if (lane == 0) { wbest[warp] = bs; wt[warp] = bt; }
            __syncthreads();
            if (threadIdx.x == 0) {
                float b = wbest[0];
                int tt = wt[0];
                for (int w = 1; w < 8; ++w)
                    if (wbest[w] > b || (wbest[w] == b && wt[w] < tt)) { b = wbest[w]; tt = wt[w]; }
                best[(int64_t)q * n_chunks + c] = b;
                best_t[(int64_t)q * n_chunks + c] = tt < T ? tt : -1;
            }
            __syncthreads();
        }
    }
}

// (3) per (query, document): the attaining chunk (first maximum), then scatter
//     dqhat[q][t*] += ds k_hat / H and dkhat[c*] += ds qhat[q][t*] (qhat already carries 1/H).
//     One warp per (query, document).
__global__ void __launch_bounds__(256) route_bwd_scatter_kernel(const void* __restrict__ index, int idx_bf16,
                                                                const int64_t* __restrict__ doc_chunk_off,
                                                                int64_t n_docs, int64_t n_chunks,
                                                                const float* __restrict__ best,
                                                                const int* __restrict__ best_t,
                                                                const float* __restrict__ qhat,
                                                                const float* __restrict__ dscore, int n_q, int T,
                                                                int H, int K, float* __restrict__ dqhat,
                                                                float* __restrict__ dkhat) {
    const int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= (int64_t)n_q * n_docs) return;
    const int q = (int)(w / n_docs);
    const int64_t doc = w % n_docs;
    const float ds = dscore[w];
    const int64_t a = doc_chunk_off[doc], b = doc_chunk_off[doc + 1];
    if (ds == 0.f || b <= a || a < 0 || b > n_chunks) return;
    int64_t cbest = a;
    for (int64_t c = a + 1; c < b; ++c)
        if (best[(int64_t)q * n_chunks + c] > best[(int64_t)q * n_chunks + cbest]) cbest = c;
    const int t = best_t[(int64_t)q * n_chunks + cbest];
    if (t < 0) return;
    const float* qv = qhat + ((int64_t)q * T + t) * K;
    const float invH = 1.0f / H;
    for (int i = lane; i < K; i += 32) {
        atomicAdd(dqhat + ((int64_t)q * T + t) * K + i, ds * load_elem(index, cbest * K + i, idx_bf16) * invH);
        atomicAdd(dkhat + cbest * K + i, ds * qv[i]);
    }
}

// (4) dqr = (g - u (u . g)) / |qr| per head, u = qr / |qr|, g = dqhat (the gradient with respect to the
//     unit query vector).
__global__ void __launch_bounds__(128) route_bwd_qr_kernel(const void* __restrict__ qr, int qr_bf16, int64_t rows,
                                                           int H, int d, const float* __restrict__ dqhat,
                                                           float* __restrict__ dqr) {
    const int64_t w = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= rows * H) return;
    float ss = 0.f, dot = 0.f;
    for (int i = lane; i < d; i += 32) {
        const float x = load_elem(qr, w * d + i, qr_bf16);
        ss = fmaf(x, x, ss);
        dot = fmaf(x, dqhat[w * d + i], dot);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
        dot += __shfl_xor_sync(0xffffffffu, dot, o);
    }
    const float n = sqrtf(ss);
    for (int i = lane; i < d; i += 32) {
        const float x = load_elem(qr, w * d + i, qr_bf16);
        dqr[w * d + i] = n > 0.f ? (dqhat[w * d + i] - x * dot / ss) / n : 0.f;
    }
}

}  // namespace
}  // namespace msa

using namespace msa;

extern "C" {

msa_status msa_sparse_attn_backward_workspace_size(int n_q, int T, int hq, size_t* bytes) {
    MSA_REQUIRE(bytes && n_q > 0 && T >= 0 && hq > 0, "msa_sparse_attn_backward_workspace_size: bad arguments");
    *bytes = align_up((size_t)n_q * T * hq * sizeof(float), 256);
    return MSA_OK;
}

msa_status msa_sparse_attn_backward(const void* q, const void* mem_kv, const int32_t* mem_len, int max_mem,
                                    const void* local_k, const void* local_v, int L_max, int L, int q_start, int n_q,
                                    int T, int hq, int hkv, int d, float scale, const void* out, const void* dout,
                                    const float* lse, msa_dtype dt, float* dq, float* dmem_kv, float* dlocal_k,
                                    float* dlocal_v, void* ws, size_t ws_bytes, void* stream) {
    MSA_REQUIRE(dtype_ok(dt), "msa_sparse_attn_backward: bad dtype");
    if (dt != MSA_BF16) return set_error(MSA_ERR_UNSUPPORTED, "msa_sparse_attn_backward: bf16 only");
    MSA_REQUIRE(n_q > 0 && n_q <= 65535 && T >= 0 && hq > 0 && hkv > 0 && hkv <= 65535 && hq % hkv == 0 &&
                    max_mem >= 0 && L >= 0 && L <= L_max && q_start >= 0,
                "msa_sparse_attn_backward: bad sizes");
    if (d != kD) return set_error(MSA_ERR_UNSUPPORTED, "msa_sparse_attn_backward: head_dim must be 128, got %d", d);
    const int G = hq / hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8)
        return set_error(MSA_ERR_UNSUPPORTED, "msa_sparse_attn_backward: hq/hkv = %d unsupported", G);
    if (T == 0) return MSA_OK;
    MSA_REQUIRE(q && out && dout && lse && mem_len && dq && ws, "msa_sparse_attn_backward: NULL pointer");
    MSA_REQUIRE(max_mem == 0 || (mem_kv && dmem_kv), "msa_sparse_attn_backward: NULL memory or its gradient");
    MSA_REQUIRE(L == 0 || (local_k && local_v && dlocal_k && dlocal_v), "msa_sparse_attn_backward: NULL local K/V");
    MSA_REQUIRE(aligned16(q) && aligned16(out) && aligned16(dout) && aligned16(dq) && aligned16(ws) &&
                    (max_mem == 0 || (aligned16(mem_kv) && aligned16(dmem_kv))) &&
                    (L == 0 || (aligned16(local_k) && aligned16(local_v) && aligned16(dlocal_k) &&
                                aligned16(dlocal_v))),
                "msa_sparse_attn_backward: pointers must be 16-byte aligned");
    size_t need = 0;
    MSA_RETURN_IF(msa_sparse_attn_backward_workspace_size(n_q, T, hq, &need));
    if (ws_bytes < need)
        return set_error(MSA_ERR_WORKSPACE, "msa_sparse_attn_backward: workspace %zu < %zu", ws_bytes, need);
    BwdArgs a{};
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.mem_kv = static_cast<const __nv_bfloat16*>(mem_kv);
    a.mem_len = mem_len; a.max_mem = max_mem;
    a.local_k = static_cast<const __nv_bfloat16*>(local_k);
    a.local_v = static_cast<const __nv_bfloat16*>(local_v);
    a.L_max = L_max; a.L = L; a.q_start = q_start; a.T = T; a.hq = hq; a.hkv = hkv;
    a.scale = scale; a.scale_log2e = scale * kLog2e;
    a.out = static_cast<const __nv_bfloat16*>(out);
    a.dout = static_cast<const __nv_bfloat16*>(dout);
    a.lse = lse; a.Dvec = static_cast<float*>(ws);
    a.dq = dq; a.dmem = dmem_kv; a.dlk = dlocal_k; a.dlv = dlocal_v;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t rows = (int64_t)n_q * T * hq;
    attn_bwd_prep_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(a.out, a.dout, rows, a.Dvec);
    MSA_LAUNCH_CHECK();
    switch (G) {
        case 1: return launch_attn_bwd_g<1>(a, n_q, s);
        case 2: return launch_attn_bwd_g<2>(a, n_q, s);
        case 4: return launch_attn_bwd_g<4>(a, n_q, s);
        default: return launch_attn_bwd_g<8>(a, n_q, s);
    }
}

msa_status msa_gather_kv_backward(const float* dmem_kv, int64_t n_chunks, const int64_t* doc_chunk_off,
                                  int64_t n_docs, const int32_t* idx, int n_q, int k, int hkv, int d, int max_mem,
                                  float* dkvbar, void* stream) {
    MSA_REQUIRE(dmem_kv && doc_chunk_off && idx && dkvbar, "msa_gather_kv_backward: NULL pointer");
    MSA_REQUIRE(n_q > 0 && n_q <= 65535 && k > 0 && hkv > 0 && d > 0 && max_mem >= 0 && n_docs > 0 && n_chunks >= 0,
                "msa_gather_kv_backward: bad sizes");
    gather_bwd_kernel<<<dim3(k, n_q), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        dmem_kv, n_chunks, doc_chunk_off, n_docs, idx, k, 2 * hkv * d, max_mem, dkvbar, device_error_word());
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

msa_status msa_pool_chunks_backward(const float* dkvbar, const float* dkr_index, const void* kr, msa_dtype kr_dt,
                                    int64_t n_tok, int hkv, int hr, int d, const int64_t* doc_tok_off,
                                    const int64_t* doc_chunk_off, const int32_t* chunk_doc, int64_t n_docs,
                                    int64_t n_chunks, int chunk, int fuse_doc_rope, const float* cos_sin,
                                    int64_t max_pos, int normalize_router, float* dk, float* dv, float* dkr,
                                    void* stream) {
    MSA_REQUIRE(n_tok >= 0 && n_docs >= 0 && n_chunks >= 0 && chunk > 0 && d > 0 && d % 2 == 0,
                "msa_pool_chunks_backward: bad sizes");
    MSA_REQUIRE(dkvbar || dkr_index, "msa_pool_chunks_backward: nothing to do");
    if (n_chunks == 0) return MSA_OK;
    MSA_REQUIRE(doc_tok_off && doc_chunk_off && chunk_doc, "msa_pool_chunks_backward: NULL offsets");
    PoolBwdArgs a{};
    a.n_parts = 0;
    if (dkvbar) {
        MSA_REQUIRE(hkv > 0 && dk && dv, "msa_pool_chunks_backward: K/V gradients need hkv > 0, dk and dv");
        MSA_REQUIRE(!fuse_doc_rope || (cos_sin && max_pos > 0), "msa_pool_chunks_backward: RoPE needs a table");
        a.parts[a.n_parts++] = 0;
        a.parts[a.n_parts++] = 1;
    }
    if (dkr_index) {
        MSA_REQUIRE(hr > 0 && dkr && (size_t)hr * d <= 1024, "msa_pool_chunks_backward: K^R needs hr * d <= 1024, dkr");
        MSA_REQUIRE(!normalize_router || (kr && dtype_ok(kr_dt) && d % 32 == 0 && d <= 256),
                    "msa_pool_chunks_backward: the normalised index needs the token K^R and d a multiple of 32 <= 256");
        a.parts[a.n_parts++] = 2;
    }
    a.dkvbar = dkvbar; a.dkr_index = dkr_index; a.kr = kr; a.kr_bf16 = kr_dt == MSA_BF16;
    a.hkv = hkv; a.hr = hr; a.d = d;
    a.doc_tok_off = doc_tok_off; a.doc_chunk_off = doc_chunk_off; a.chunk_doc = chunk_doc;
    a.n_docs = n_docs; a.n_chunks = n_chunks; a.n_tok = n_tok; a.chunk = chunk;
    a.fuse_rope = fuse_doc_rope; a.normalize = normalize_router;
    a.cs = reinterpret_cast<const float2*>(cos_sin); a.max_pos = max_pos;
    a.dk = dk; a.dv = dv; a.dkr = dkr; a.err = device_error_word();
    const int64_t per_part = std::min<int64_t>(n_chunks, (int64_t)sm_count() * 16);
    pool_bwd_kernel<<<(unsigned)(per_part * a.n_parts), 128, 0, static_cast<cudaStream_t>(stream)>>>(a);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

msa_status msa_router_aux_loss(const float* doc_scores, int n_q, int64_t n_docs, const int32_t* evidence, int n_ev,
                               float tau, float* loss, float* d_doc_scores, void* stream) {
    MSA_REQUIRE(doc_scores && evidence && d_doc_scores, "msa_router_aux_loss: NULL pointer");
    MSA_REQUIRE(n_q > 0 && n_docs > 0 && n_ev > 0 && tau > 0.f, "msa_router_aux_loss: bad sizes or tau");
    aux_loss_kernel<<<n_q, 1024, 0, static_cast<cudaStream_t>(stream)>>>(doc_scores, n_docs, evidence, n_ev, tau, n_q,
                                                                         loss, d_doc_scores, device_error_word());
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

msa_status msa_route_backward_workspace_size(int64_t n_chunks, int n_q, int T, int H, int d, size_t* bytes) {
    MSA_REQUIRE(bytes && n_chunks >= 0 && n_q > 0 && T > 0 && H > 0 && d > 0, "msa_route_backward_workspace_size: bad sizes");
    const size_t qk = (size_t)n_q * T * H * d * sizeof(float);
    *bytes = 2 * align_up(qk, 256) + 2 * align_up((size_t)n_q * n_chunks * 4, 256);
    return MSA_OK;
}

msa_status msa_route_backward(const void* kr_index, msa_dtype dt, int64_t n_chunks, const int64_t* doc_chunk_off,
                              int64_t n_docs, const void* qr, int n_q, int T, int H, int d, const float* d_doc_scores,
                              float* dqr, float* dkhat, void* ws, size_t ws_bytes, void* stream) {
    MSA_REQUIRE(dtype_ok(dt), "msa_route_backward: bad dtype");
    MSA_REQUIRE(kr_index && doc_chunk_off && qr && d_doc_scores && dqr && dkhat && ws, "msa_route_backward: NULL pointer");
    MSA_REQUIRE(n_chunks > 0 && n_docs > 0 && n_q > 0 && T > 0 && H > 0 && d > 0 && (size_t)H * d <= 1024,
                "msa_route_backward: bad sizes (H * d <= 1024)");
    size_t need = 0;
    MSA_RETURN_IF(msa_route_backward_workspace_size(n_chunks, n_q, T, H, d, &need));
    if (ws_bytes < need) return set_error(MSA_ERR_WORKSPACE, "msa_route_backward: workspace %zu < %zu", ws_bytes, need);
    const int K = H * d;
    const size_t qk = align_up((size_t)n_q * T * K * sizeof(float), 256);
    char* w = static_cast<char*>(ws);
    float* qhat = reinterpret_cast<float*>(w);
    float* dqhat = reinterpret_cast<float*>(w + qk);
    float* best = reinterpret_cast<float*>(w + 2 * qk);
    int* best_t = reinterpret_cast<int*>(w + 2 * qk + align_up((size_t)n_q * n_chunks * 4, 256));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int bf = dt == MSA_BF16;
    const int64_t rows = (int64_t)n_q * T;
    MSA_CUDA_TRY(cudaMemsetAsync(dqhat, 0, (size_t)n_q * T * K * sizeof(float), s));
    MSA_CUDA_TRY(cudaMemsetAsync(dkhat, 0, (size_t)n_chunks * K * sizeof(float), s));
    route_bwd_qhat_kernel<<<(unsigned)((rows * H + 3) / 4), 128, 0, s>>>(qr, bf, rows, H, d, qhat);
    MSA_LAUNCH_CHECK();
    const unsigned best_blocks = (unsigned)std::min<int64_t>(n_chunks, (int64_t)sm_count() * 8);
    route_bwd_best_kernel<<<best_blocks, 256, 0, s>>>(kr_index, bf, n_chunks, qhat, n_q, T, K, best, best_t);
    MSA_LAUNCH_CHECK();
    route_bwd_scatter_kernel<<<(unsigned)(((int64_t)n_q * n_docs + 7) / 8), 256, 0, s>>>(
        kr_index, bf, doc_chunk_off, n_docs, n_chunks, best, best_t, qhat, d_doc_scores, n_q, T, H, K, dqhat, dkhat);
    MSA_LAUNCH_CHECK();
    route_bwd_qr_kernel<<<(unsigned)((rows * H + 3) / 4), 128, 0, s>>>(qr, bf, rows, H, d, dqhat, dqr);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

}  // extern "C"
