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
    int n_rsplit;            // dK/dV: row ranges per key tile (1 = write the gradients directly)
    int key_pad;             // key tiles x 64
    float* part_dkv;         // [n_rsplit][n_q][key_pad][2][hkv][d] partial dK (x scale) / dV per row range
};

// branch-free (bitwise) visibility: a memory row, or a causal local key inside the key range
__device__ __forceinline__ bool key_visible(int kk, int mem_len, int n_keys, int q_start, int t) {
    return (kk < mem_len) | ((kk < n_keys) & (kk - mem_len <= q_start + t));
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
    const int qi = blockIdx.z, g = blockIdx.y;
    const int rsplit = blockIdx.x % a.n_rsplit, kb = (blockIdx.x / a.n_rsplit) * kTile;
    const int mem_len = max(min(a.mem_len[qi], a.max_mem), 0);
    const int n_keys = mem_len + a.L;
    if (kb >= n_keys) return;
    const int n_rows = a.T * G;
    // this block's contiguous range of 64-row blocks
    const int row_blocks = (n_rows + kTile - 1) / kTile;
    const int rb_per = (row_blocks + a.n_rsplit - 1) / a.n_rsplit;
    const int r_begin = min(rsplit * rb_per, row_blocks) * kTile;
    const int r_end = min(min(rsplit * rb_per + rb_per, row_blocks) * kTile, n_rows);
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

    for (int r0 = max(r_begin, (t_first * G / kTile) * kTile); r0 < r_end; r0 += kTile) {
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
                const bool vis = (row < n_rows) & (l2 != ninf) & key_visible(key, mem_len, n_keys, a.q_start, row / G);
                const float p = ex2(vis ? st[nb][e] * a.scale_log2e - l2 : ninf);
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

    // write this thread's two keys' gradients (dims nd*8 + 2 tig, +1): directly, or as this row
    // range's partial sums for the reduction
    auto dst = [&](int key, int which) -> float* {
        if (a.n_rsplit > 1)
            return a.part_dkv +
                   ((((int64_t)rsplit * gridDim.z + qi) * a.key_pad + key) * 2 + which) * a.hkv * kD + g * kD;
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
                const bool vis = (first ? va : vb) & ((first ? l2a : l2b) != ninf) &
                                 key_visible(kk, mem_len, n_keys_all, a.q_start, first ? ta : tb);
                const float p = ex2(vis ? sc[nb][e] * a.scale_log2e - (first ? l2a : l2b) : ninf);
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

// Sum of the row ranges' partial dK/dV into the outputs: one warp per (query, key, K or V, kv head),
// lane l owning dims 4l..4l+3, the ranges added in order (deterministic).
__global__ void __launch_bounds__(256) attn_bwd_dkdv_reduce_kernel(const BwdArgs a, int n_q) {
    const int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int64_t per_q = (int64_t)a.key_pad * 2 * a.hkv;
    if (w >= n_q * per_q) return;
    const int qi = (int)(w / per_q);
    const int64_t rem = w % per_q;
    const int key = (int)(rem / (2 * a.hkv));
    const int which = (int)((rem / a.hkv) % 2), g = (int)(rem % a.hkv);
    const int mem_len = max(min(a.mem_len[qi], a.max_mem), 0);
    if (key >= mem_len + a.L) return;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = 0; r < a.n_rsplit; ++r) {
        const float4 v = *reinterpret_cast<const float4*>(
            a.part_dkv + ((((int64_t)r * n_q + qi) * a.key_pad + key) * 2 + which) * a.hkv * kD + g * kD + lane * 4);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    float* out = key < mem_len
                     ? a.dmem + (((int64_t)qi * a.max_mem + key) * 2 + which) * a.hkv * kD + g * kD
                     : (which ? a.dlv : a.dlk) + (((int64_t)qi * a.L_max + (key - mem_len)) * a.hkv + g) * kD;
    *reinterpret_cast<float4*>(out + lane * 4) = acc;
}

constexpr size_t kDkdvSmem = 4 * sizeof(Tile) + 2 * kTile * sizeof(float);
// dK/dV blocks resident per SM (255 registers x 128 threads) on 148 SMs: the row ranges per key
// tile are chosen so that the grid fills about one such wave
constexpr int kDkdvWave = 2 * 148;

int pick_rsplit(int n_q, int T, int hq, int hkv, int max_mem, int L) {
    const int key_tiles = (max_mem + L + kTile - 1) / kTile;
    const int64_t base = (int64_t)key_tiles * hkv * n_q;
    const int row_blocks = (T * (hq / hkv) + kTile - 1) / kTile;
    if (base <= 0) return 1;
    return (int)std::max<int64_t>(1, std::min<int64_t>(row_blocks, kDkdvWave / base));
}

size_t bwd_ws_bytes(int n_q, int T, int hq, int hkv, int max_mem, int L) {
    const size_t dvec = align_up((size_t)n_q * T * hq * sizeof(float), 256);
    const int r = pick_rsplit(n_q, T, hq, hkv, max_mem, L);
    if (r <= 1) return dvec;
    const size_t key_pad = (size_t)((max_mem + L + kTile - 1) / kTile) * kTile;
    return dvec + align_up((size_t)r * n_q * key_pad * 2 * hkv * kD * sizeof(float), 256);
}


template <int G>
msa_status launch_attn_bwd_g(const BwdArgs& a, int n_q, cudaStream_t s) {
    const int key_tiles = (a.max_mem + a.L + kTile - 1) / kTile;
    if (key_tiles > 0) {
        if (attn_impl_setting() == 3) {   // dK / dV on tcgen05 (opt-in)
            DkdvTcArgs k{};
            k.q = a.q; k.mem_kv = a.mem_kv; k.mem_len = a.mem_len; k.max_mem = a.max_mem;
            k.local_k = a.local_k; k.local_v = a.local_v; k.L_max = a.L_max; k.L = a.L; k.q_start = a.q_start;
            k.T = a.T; k.hq = a.hq; k.hkv = a.hkv; k.G = G; k.scale = a.scale; k.scale_log2e = a.scale_log2e;
            k.dout = a.dout; k.lse = a.lse; k.Dvec = a.Dvec; k.dmem = a.dmem; k.dlk = a.dlk; k.dlv = a.dlv;
            k.n_rsplit = a.n_rsplit; k.key_pad = a.key_pad; k.part_dkv = a.part_dkv; k.err = device_error_word();
            MSA_RETURN_IF(launch_attn_bwd_dkdv_tc(k, n_q, s));
        } else {
            MSA_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dkdv_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              (int)kDkdvSmem));
            attn_bwd_dkdv_kernel<G><<<dim3(key_tiles * a.n_rsplit, a.hkv, n_q), 128, kDkdvSmem, s>>>(a);
            MSA_LAUNCH_CHECK();
        }
        if (a.n_rsplit > 1) {
            const int64_t warps = (int64_t)n_q * a.key_pad * 2 * a.hkv;
            attn_bwd_dkdv_reduce_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(a, n_q);
            MSA_LAUNCH_CHECK();
        }
    }
    if (attn_impl_setting() == 0 || attn_impl_setting() == 3) {   // dQ on tcgen05
        DqTcArgs d{};
        d.q = a.q; d.mem_kv = a.mem_kv; d.mem_len = a.mem_len; d.max_mem = a.max_mem;
        d.local_k = a.local_k; d.local_v = a.local_v; d.L_max = a.L_max; d.L = a.L; d.q_start = a.q_start;
        d.T = a.T; d.hq = a.hq; d.hkv = a.hkv; d.G = G; d.scale = a.scale; d.scale_log2e = a.scale_log2e;
        d.dout = a.dout; d.lse = a.lse; d.Dvec = a.Dvec; d.dq = a.dq; d.err = device_error_word();
        return launch_attn_bwd_dq_tc(d, n_q, s);
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
    const int64_t step = (int64_t)gridDim.z * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.z * blockDim.x + threadIdx.x; i < rows * row_len; i += step)
        atomicAdd(dst + i, src[i]);
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
    int64_t n_kr_items;      // router-key chunks (0 without dkr_index)
    int64_t n_kv_items;      // (chunk, K or V, token slice) items (0 without dkvbar)
    int kv_slices, slice_tok;
    int* err;
};

__device__ __forceinline__ float load_elem(const void* p, int64_t i, int bf16) {
    if (bf16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
    return static_cast<const float*>(p)[i];
}

// Four consecutive elements at index i (a multiple of 4) of a bf16 or fp32 array, as fp32.
__device__ __forceinline__ float4 load4(const void* p, int64_t i, int bf16) {
    if (bf16) {
        const uint2 u = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(p) + i);
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                           __uint_as_float(u.y & 0xffff0000u));
    }
    return *reinterpret_cast<const float4*>(static_cast<const float*>(p) + i);
}

__device__ __forceinline__ float4 scale4(float4 v, float s) { return make_float4(v.x * s, v.y * s, v.z * s, v.w * s); }

// Work items: first one per chunk of the router-key gradient (it reads the chunk's tokens again
// for the normalisation's backward, so it keeps the whole chunk), then one per (chunk, K or V,
// slice of kPoolBwdSliceTok tokens) — small, even items that the block scheduler spreads over
// the SMs with a short tail. Thread i owns elements 4i..4i+3 of a token row (rows of at most 1024
// elements, one head = d/4 consecutive lanes of a warp); every token gets one 16-byte streaming
// store per thread.
constexpr int kPoolBwdThreads = 256;
constexpr int kPoolBwdSliceTok = 32;

__global__ void __launch_bounds__(kPoolBwdThreads) pool_bwd_kernel(const PoolBwdArgs a) {
    const int d = a.d;
    const int e0 = threadIdx.x * 4;
    const int ih = e0 % d;
    const bool first = ih < d / 2;
    const int hi = first ? ih : ih - d / 2;
    const int head_lanes = d / 4;
    const int64_t total = a.n_kr_items + a.n_kv_items;
    for (int64_t item = blockIdx.x; item < total; item += gridDim.x) {
        int part, slice = 0;
        int64_t c;
        if (item < a.n_kr_items) {
            part = 2;
            c = item;
        } else {
            const int64_t j = item - a.n_kr_items;
            const int64_t per_chunk = 2 * (int64_t)a.kv_slices;
            c = j / per_chunk;
            const int r = (int)(j - c * per_chunk);
            part = r / a.kv_slices;
            slice = r - part * a.kv_slices;
        }
        const int E = (part == 2 ? a.hr : a.hkv) * d;
        const bool active = e0 < E;
        const int64_t doc = a.chunk_doc[c];
        if (doc < 0 || doc >= a.n_docs) {
            if (threadIdx.x == 0) record_device_error(a.err, MSA_DEV_BAD_INDEX);
            continue;
        }
        const int64_t doc_start = a.doc_tok_off[doc];
        const int64_t t0 = doc_start + (c - a.doc_chunk_off[doc]) * (int64_t)a.chunk;
        const int64_t t1 = min(t0 + (int64_t)a.chunk, a.doc_tok_off[doc + 1]);
        if (doc_start < 0 || t0 < doc_start || t0 >= t1 || t1 > a.n_tok) {
            if (threadIdx.x == 0) record_device_error(a.err, MSA_DEV_BAD_INDEX);
            continue;
        }
        const float inv_n = 1.0f / (float)(t1 - t0);
        const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
        if (part == 2) {
            float4 g = active ? *reinterpret_cast<const float4*>(a.dkr_index + c * (int64_t)E + e0) : zero;
            if (a.normalize) {
                // the chunk's raw mean router key (this thread's 4 elements), then per head
                // (g - k_hat (k_hat . g)) / |k| with k_hat = mean / |mean|
                float4 mu = zero;
                if (active) {
                    int64_t t = t0;
                    for (; t + 4 <= t1; t += 4) {                // four loads in flight, added in token order
                        float4 x[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) x[u] = load4(a.kr, (t + u) * E + e0, a.kr_bf16);
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            mu.x += x[u].x; mu.y += x[u].y; mu.z += x[u].z; mu.w += x[u].w;
                        }
                    }
                    for (; t < t1; ++t) {
                        const float4 x = load4(a.kr, t * E + e0, a.kr_bf16);
                        mu.x += x.x; mu.y += x.y; mu.z += x.z; mu.w += x.w;
                    }
                }
                mu = scale4(mu, inv_n);
                float ss = mu.x * mu.x + mu.y * mu.y + mu.z * mu.z + mu.w * mu.w;
                float dg = mu.x * g.x + mu.y * g.y + mu.z * g.z + mu.w * g.w;
                for (int o = head_lanes / 2; o >= 1; o >>= 1) {
                    ss += __shfl_xor_sync(0xffffffffu, ss, o);
                    dg += __shfl_xor_sync(0xffffffffu, dg, o);
                }
                const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
                const float proj = ss > 0.f ? dg / ss : 0.f;
                g = make_float4((g.x - mu.x * proj) * inv, (g.y - mu.y * proj) * inv, (g.z - mu.z * proj) * inv,
                                (g.w - mu.w * proj) * inv);
            }
            g = scale4(g, inv_n);
            if (active)
                for (int64_t t = t0; t < t1; ++t) __stcs(reinterpret_cast<float4*>(a.dkr + t * E + e0), g);
            continue;
        }
        const int64_t ta = t0 + (int64_t)slice * a.slice_tok;
        if (ta >= t1) continue;
        const int64_t tb = min(ta + (int64_t)a.slice_tok, t1);
        const float* grow = a.dkvbar + (c * 2 + part) * (int64_t)E;
        const float4 g = active ? scale4(*reinterpret_cast<const float4*>(grow + e0), inv_n) : zero;
        float* out = part == 0 ? a.dk : a.dv;
        if (part == 1 || !a.fuse_rope) {
            if (active)
                for (int64_t t = ta; t < tb; ++t) __stcs(reinterpret_cast<float4*>(out + t * E + e0), g);
            continue;
        }
        // keys: the transposed rotation of each token's position, R(-p):
        // first half x cos + y sin, second half x cos - y sin (y the rotate-half partner)
        const float4 y = active ? scale4(*reinterpret_cast<const float4*>(grow + (first ? e0 + d / 2 : e0 - d / 2)),
                                         inv_n)
                                : zero;
        const float sg = first ? 1.f : -1.f;
        for (int64_t t = ta; t < tb; ++t) {
            const int64_t p = t - doc_start;
            float4 o = g;
            if (p < a.max_pos) {
                const float4 c01 = *reinterpret_cast<const float4*>(a.cs + p * (d / 2) + hi);
                const float4 c23 = *reinterpret_cast<const float4*>(a.cs + p * (d / 2) + hi + 2);
                o = make_float4(fmaf(g.x, c01.x, sg * y.x * c01.y), fmaf(g.y, c01.z, sg * y.y * c01.w),
                                fmaf(g.z, c23.x, sg * y.z * c23.y), fmaf(g.w, c23.z, sg * y.w * c23.w));
            } else if (threadIdx.x == 0) {
                record_device_error(a.err, MSA_DEV_ROPE_POSITION);
            }
            if (active) __stcs(reinterpret_cast<float4*>(out + t * E + e0), o);
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
// (1) qhat: unit router queries per head, divided by H (the folded form) [n_q][T][H*d] fp32;
//     with qsplit, also its exact three-term bf16 split for the tensor-core search, rows
//     [3][n_q][T_pad][H*d] (term, query, token).
__global__ void __launch_bounds__(128) route_bwd_qhat_kernel(const void* __restrict__ qr, int qr_bf16, int64_t rows,
                                                             int H, int d, float* __restrict__ qhat,
                                                             __nv_bfloat16* __restrict__ qsplit, int T, int T_pad,
                                                             int n_q) {
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
    const int64_t row = w / H;
    const int h = (int)(w - row * H);
    const int64_t qi = row / T, t = row - qi * T;
    const int64_t K = (int64_t)H * d;
    for (int i = lane; i < d; i += 32) {
        const float x = load_elem(qr, w * d + i, qr_bf16) * inv;
        qhat[w * d + i] = x;
        if (qsplit) {
            // x = hi + mid + lo: each term the bf16 rounding of what the previous ones leave (the
            // differences are exact in fp32)
            const __nv_bfloat16 hi = __float2bfloat16_rn(x);
            const float r1 = x - __bfloat162float(hi);
            const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
            const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
            const int64_t o = (qi * T_pad + t) * K + (int64_t)h * d + i;
            const int64_t term = (int64_t)n_q * T_pad * K;
            qsplit[o] = hi;
            qsplit[o + term] = mid;
            qsplit[o + 2 * term] = lo;
        }
    }
}

// (2) per (query, chunk): best folded score over the query tokens and the first token attaining it,
//     as one 64-bit key (order-preserving bits of the score, then the complement of the token) so
//     that an atomic max keeps the best score and, among equal scores, the first token.
//     Block per (group of 8 chunks, slice of 64 tokens), grid-stride: the chunks' index rows in
//     shared memory, each warp scores one token against all 8 chunks per read of its qhat.
constexpr int kBestChunks = 8;
constexpr int kBestTokens = 64;

__device__ __forceinline__ unsigned long long best_key(float score, int t) {
    const uint32_t b = __float_as_uint(score);
    const uint32_t o = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((unsigned long long)o << 32) | (unsigned long long)(0xffffffffu - (uint32_t)t);
}

__device__ __forceinline__ float best_score(unsigned long long key) {
    const uint32_t o = (uint32_t)(key >> 32);
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

__global__ void __launch_bounds__(256) route_bwd_best_kernel(const void* __restrict__ index, int idx_bf16,
                                                             int64_t n_chunks, const float* __restrict__ qhat, int n_q,
                                                             int T, int K, unsigned long long* __restrict__ best) {
    __shared__ float krow[kBestChunks][1024];
    __shared__ unsigned long long wbest[8][kBestChunks];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t groups = (n_chunks + kBestChunks - 1) / kBestChunks;
    const int slices = (T + kBestTokens - 1) / kBestTokens;
    for (int64_t w = blockIdx.x; w < groups * slices; w += gridDim.x) {
        const int64_t c0 = (w / slices) * kBestChunks;
        const int tb = (int)(w % slices) * kBestTokens, te = min(tb + kBestTokens, T);
        const int nc = (int)min((int64_t)kBestChunks, n_chunks - c0);
        __syncthreads();
        for (int i = threadIdx.x; i < kBestChunks * K; i += blockDim.x) {
            const int j = i / K, e = i % K;
            krow[j][e] = j < nc ? load_elem(index, (c0 + j) * K + e, idx_bf16) : 0.f;
        }
        __syncthreads();
        for (int q = 0; q < n_q; ++q) {
            unsigned long long bk[kBestChunks];
#pragma unroll
            for (int j = 0; j < kBestChunks; ++j) bk[j] = 0ull;
            for (int t = tb + warp; t < te; t += 8) {
                const float* qv = qhat + ((int64_t)q * T + t) * K;
                float acc[kBestChunks];
#pragma unroll
                for (int j = 0; j < kBestChunks; ++j) acc[j] = 0.f;
                for (int i = lane; i < K; i += 32) {
                    const float x = qv[i];
#pragma unroll
                    for (int j = 0; j < kBestChunks; ++j) acc[j] = fmaf(x, krow[j][i], acc[j]);
                }
#pragma unroll
                for (int j = 0; j < kBestChunks; ++j) {
#pragma unroll
                    for (int o = 16; o >= 1; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
                    const unsigned long long key = best_key(acc[j], t);
                    bk[j] = key > bk[j] ? key : bk[j];
                }
            }
            if (lane == 0)
#pragma unroll
                for (int j = 0; j < kBestChunks; ++j) wbest[warp][j] = bk[j];
            __syncthreads();
            if (threadIdx.x < nc) {
                const int j = threadIdx.x;
                unsigned long long b = wbest[0][j];
                for (int x = 1; x < 8; ++x) b = wbest[x][j] > b ? wbest[x][j] : b;
                if (b) atomicMax(best + (int64_t)q * n_chunks + c0 + j, b);
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
                                                                const unsigned long long* __restrict__ best,
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
        if (best_score(best[(int64_t)q * n_chunks + c]) > best_score(best[(int64_t)q * n_chunks + cbest])) cbest = c;
    const unsigned long long key = best[(int64_t)q * n_chunks + cbest];
    if (key == 0ull) return;
    const int t = (int)(0xffffffffu - (uint32_t)(key & 0xffffffffull));
    if (t < 0 || t >= T) return;
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

msa_status msa_sparse_attn_backward_workspace_size(int n_q, int T, int hq, int hkv, int max_mem, int L,
                                                   size_t* bytes) {
    MSA_REQUIRE(bytes && n_q > 0 && T >= 0 && hq > 0 && hkv > 0 && hq % hkv == 0 && max_mem >= 0 && L >= 0,
                "msa_sparse_attn_backward_workspace_size: bad arguments");
    *bytes = bwd_ws_bytes(n_q, T, hq, hkv, max_mem, L);
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
    MSA_RETURN_IF(msa_sparse_attn_backward_workspace_size(n_q, T, hq, hkv, max_mem, L, &need));
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
    a.n_rsplit = pick_rsplit(n_q, T, hq, hkv, max_mem, L);
    a.key_pad = ((max_mem + L + kTile - 1) / kTile) * kTile;
    a.part_dkv = reinterpret_cast<float*>(static_cast<char*>(ws) + align_up((size_t)n_q * T * hq * sizeof(float), 256));
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
                                  float* dkvbar, int accumulate, void* stream) {
    MSA_REQUIRE(dmem_kv && doc_chunk_off && idx && dkvbar, "msa_gather_kv_backward: NULL pointer");
    MSA_REQUIRE(n_q > 0 && n_q <= 65535 && k > 0 && hkv > 0 && d > 0 && max_mem >= 0 && n_docs > 0 && n_chunks >= 0,
                "msa_gather_kv_backward: bad sizes");
    if (!accumulate)
        MSA_CUDA_TRY(cudaMemsetAsync(dkvbar, 0, (size_t)n_chunks * 2 * hkv * d * sizeof(float),
                                     static_cast<cudaStream_t>(stream)));
    // a document's rows dealt out to several blocks (about 4K elements each, at most 64)
    const int64_t per_doc = ((int64_t)max_mem * 2 * hkv * d) / k;
    const int parts = (int)std::min<int64_t>(64, std::max<int64_t>(1, (per_doc + 4095) / 4096));
    gather_bwd_kernel<<<dim3(k, n_q, parts), 256, 0, static_cast<cudaStream_t>(stream)>>>(
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
    // one thread per 4 elements of a row, a head on d/4 lanes of one warp
    if (d % 8 != 0 || d / 4 > 32 || ((d / 4) & (d / 4 - 1)) != 0)
        return set_error(MSA_ERR_UNSUPPORTED, "msa_pool_chunks_backward: head_dim %d unsupported (8..128, d/4 a power of two)", d);
    if (dkvbar) {
        MSA_REQUIRE(hkv > 0 && (size_t)hkv * d <= 4 * kPoolBwdThreads && dk && dv,
                    "msa_pool_chunks_backward: K/V gradients need 0 < hkv * d <= 1024, dk and dv");
        MSA_REQUIRE(aligned16(dkvbar) && aligned16(dk) && aligned16(dv), "msa_pool_chunks_backward: unaligned K/V pointer");
        MSA_REQUIRE(!fuse_doc_rope || (cos_sin && max_pos > 0 && aligned16(cos_sin)),
                    "msa_pool_chunks_backward: RoPE needs a table");
    }
    if (dkr_index) {
        MSA_REQUIRE(hr > 0 && dkr && (size_t)hr * d <= 4 * kPoolBwdThreads,
                    "msa_pool_chunks_backward: K^R needs 0 < hr * d <= 1024 and dkr");
        MSA_REQUIRE(aligned16(dkr_index) && aligned16(dkr), "msa_pool_chunks_backward: unaligned K^R pointer");
        MSA_REQUIRE(!normalize_router || (kr && dtype_ok(kr_dt) && aligned16(kr)),
                    "msa_pool_chunks_backward: the normalised index needs the token K^R");
    }
    a.dkvbar = dkvbar; a.dkr_index = dkr_index; a.kr = kr; a.kr_bf16 = kr_dt == MSA_BF16;
    a.hkv = hkv; a.hr = hr; a.d = d;
    a.doc_tok_off = doc_tok_off; a.doc_chunk_off = doc_chunk_off; a.chunk_doc = chunk_doc;
    a.n_docs = n_docs; a.n_chunks = n_chunks; a.n_tok = n_tok; a.chunk = chunk;
    a.fuse_rope = fuse_doc_rope; a.normalize = normalize_router;
    a.cs = reinterpret_cast<const float2*>(cos_sin); a.max_pos = max_pos;
    a.dk = dk; a.dv = dv; a.dkr = dkr; a.err = device_error_word();
    a.slice_tok = kPoolBwdSliceTok;
    a.kv_slices = (chunk + kPoolBwdSliceTok - 1) / kPoolBwdSliceTok;
    a.n_kr_items = dkr_index ? n_chunks : 0;
    a.n_kv_items = dkvbar ? n_chunks * 2 * a.kv_slices : 0;
    const int64_t items = a.n_kr_items + a.n_kv_items;
    const unsigned grid = (unsigned)std::min<int64_t>(items, (int64_t)1 << 24);
    pool_bwd_kernel<<<grid, kPoolBwdThreads, 0, static_cast<cudaStream_t>(stream)>>>(a);
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
    const int tile = route_bwd_tc_token_tile();
    const size_t t_pad = (size_t)(T + tile - 1) / tile * tile;
    const size_t split = 3 * (size_t)n_q * t_pad * H * d * sizeof(__nv_bfloat16);
    *bytes = 2 * align_up(qk, 256) + align_up((size_t)n_q * n_chunks * 8, 256) + align_up(split, 256);
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
    unsigned long long* best = reinterpret_cast<unsigned long long*>(w + 2 * qk);
    const int tile = route_bwd_tc_token_tile();
    const int T_pad = (T + tile - 1) / tile * tile;
    __nv_bfloat16* qsplit =
        reinterpret_cast<__nv_bfloat16*>(w + 2 * qk + align_up((size_t)n_q * n_chunks * 8, 256));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int bf = dt == MSA_BF16;
    const int64_t rows = (int64_t)n_q * T;
    // best-token search: tcgen05 for a bf16 index (K a multiple of 64), CUDA cores otherwise or when
    // the router is set to its CUDA-core kernel
    const bool tc = bf && K % 64 == 0 && route_impl_setting() != 1 && T_pad / tile <= 65535 && n_q <= 65535;
    MSA_CUDA_TRY(cudaMemsetAsync(dqhat, 0, (size_t)n_q * T * K * sizeof(float), s));
    MSA_CUDA_TRY(cudaMemsetAsync(dkhat, 0, (size_t)n_chunks * K * sizeof(float), s));
    MSA_CUDA_TRY(cudaMemsetAsync(best, 0, (size_t)n_q * n_chunks * sizeof(unsigned long long), s));
    if (tc && T_pad != T)   // padding token rows of the split: zero (their columns are never read)
        MSA_CUDA_TRY(cudaMemsetAsync(qsplit, 0, 3 * (size_t)n_q * T_pad * K * sizeof(__nv_bfloat16), s));
    route_bwd_qhat_kernel<<<(unsigned)((rows * H + 3) / 4), 128, 0, s>>>(qr, bf, rows, H, d, qhat, tc ? qsplit : nullptr,
                                                                         T, T_pad, n_q);
    MSA_LAUNCH_CHECK();
    if (tc) {
        MSA_RETURN_IF(launch_route_bwd_best_tc(kr_index, n_chunks, qsplit, n_q, T, T_pad, K, best, s));
    } else {
        const int64_t work = ((n_chunks + kBestChunks - 1) / kBestChunks) * ((T + kBestTokens - 1) / kBestTokens);
        const unsigned best_blocks = (unsigned)std::min<int64_t>(work, (int64_t)sm_count() * 8);
        route_bwd_best_kernel<<<best_blocks, 256, 0, s>>>(kr_index, bf, n_chunks, qhat, n_q, T, K, best);
        MSA_LAUNCH_CHECK();
    }
    route_bwd_scatter_kernel<<<(unsigned)(((int64_t)n_q * n_docs + 7) / 8), 256, 0, s>>>(
        kr_index, bf, doc_chunk_off, n_docs, n_chunks, best, qhat, d_doc_scores, n_q, T, H, K, dqhat, dkhat);
    MSA_LAUNCH_CHECK();
    route_bwd_qr_kernel<<<(unsigned)((rows * H + 3) / 4), 128, 0, s>>>(qr, bf, rows, H, d, dqhat, dqr);
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

}  // extern "C"
