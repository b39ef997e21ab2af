// Internal launchers shared between translation units of the library.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace msa {

// Tensor map of a bf16 array for TMA loads with the 128-byte swizzle (defined with the router):
// dims[0] innermost in elements, strides[i] in bytes for dims i + 1, box in elements.
msa_status make_tensor_map_bf16(CUtensorMap* map, const void* ptr, int rank, const uint64_t* dims,
                                const uint64_t* strides, const uint32_t* box);
// The same for fp32 or bf16 elements, with the 128-byte swizzle or none (a box then lands in shared
// memory in plain row-major order).
msa_status make_tensor_map(CUtensorMap* map, const void* ptr, bool fp32, int rank, const uint64_t* dims,
                           const uint64_t* strides, const uint32_t* box, bool swizzle128);

// The bf16 attention kernel choice of msa_attn_set_impl (0 = default: tcgen05 where it applies).
int attn_impl_setting();
int route_impl_setting();   // msa_route_set_impl's value (1 = CUDA-core kernels)

// Router backward best-token search on tcgen05 (route_bwd_tc.cu): index [n_chunks][K] bf16,
// qsplit [3][n_q][T_pad][K] bf16 (the exact three-term split of qhat), best [n_q][n_chunks]
// 64-bit keys (zeroed by the caller), T_pad a multiple of route_bwd_tc_token_tile().
int route_bwd_tc_token_tile();
msa_status launch_route_bwd_best_tc(const void* index, int64_t n_chunks, const void* qsplit, int n_q, int T,
                                    int T_pad, int K, unsigned long long* best, cudaStream_t s);

// dQ of the attention backward on tcgen05 (bf16, d = 128): the forward's operands, dout, its
// log-sum-exp (natural log) and D = rowsum(dO * O); dq fp32 [n_q][T][hq][d] is overwritten.
struct DqTcArgs {
    const __nv_bfloat16* q;
    const __nv_bfloat16* mem_kv;
    const int32_t* mem_len;
    int max_mem;
    const __nv_bfloat16* local_k;
    const __nv_bfloat16* local_v;
    int L_max, L, q_start, T, hq, hkv, G;
    float scale, scale_log2e;
    const __nv_bfloat16* dout;
    const float* lse;
    const float* Dvec;
    float* dq;
    int* err;
    int use_tma;
    int use_tma_loc;
};
msa_status launch_attn_bwd_dq_tc(DqTcArgs a, int n_q, cudaStream_t s);

// dK / dV of the attention backward on tcgen05 (attn_bwd_tc.cu): the same inputs as DqTcArgs plus
// the gradient outputs. n_rsplit row ranges per key tile; with n_rsplit > 1 each range writes its
// partial (dK already scaled) into part_dkv [n_rsplit][n_q][key_pad][2][hkv][d] for the reduce
// kernel, otherwise the gradients go to dmem [n_q][max_mem][2][hkv][d] and dlk / dlv
// [n_q][L_max][hkv][d] directly.
struct DkdvTcArgs {
    const __nv_bfloat16* q;
    const __nv_bfloat16* mem_kv;
    const int32_t* mem_len;
    int max_mem;
    const __nv_bfloat16* local_k;
    const __nv_bfloat16* local_v;
    int L_max, L, q_start, T, hq, hkv, G;
    float scale, scale_log2e;
    const __nv_bfloat16* dout;
    const float* lse;
    const float* Dvec;
    float* dmem;
    float* dlk;
    float* dlv;
    int n_rsplit, key_pad;
    float* part_dkv;
    int* err;
};
msa_status launch_attn_bwd_dkdv_tc(const DkdvTcArgs& a, int n_q, cudaStream_t s);

// Rotates rows of [*, heads, d] vectors. Row r of the launch belongs to segment s at offset u:
//   uniform_len > 0: s = r / uniform_len, u = r % uniform_len,
//                    input row s*in_stride + u, output row s*out_stride + out_off + u;
//   otherwise      : s from the CSR offsets seg_off[n_seg + 1], input row = output row = r.
// Position = pos_offset + u.
struct RopeRowsArgs {
    const void* in;
    void* out;
    int64_t n_rows;
    int heads;
    int d;
    const int64_t* seg_off;
    int64_t n_seg;
    int64_t uniform_len;
    int64_t in_stride, out_stride, out_off;
    int64_t pos_offset;
    const float2* cs;
    int64_t max_pos;
    int* err;
};
msa_status launch_rope_rows(const RopeRowsArgs& a, msa_dtype dt, cudaStream_t s);

// One interleave round's appends for up to kMaxAppendLayers layers in one launch: new keys rotated
// to positions pos_offset + t into local_k rows L_prev + t, values copied to local_v, queries
// rotated into q_rot [n_q][T_new][hq][d]. New-token buffers: row (q * new_q_stride + t).
struct AppendLayer {
    const void* k_new;
    const void* v_new;
    const void* q_new;
    void* local_k;
    void* local_v;
    void* q_rot;
};
constexpr int kMaxAppendLayers = 24;
struct AppendArgs {
    AppendLayer layer[kMaxAppendLayers];
    int n_layers, n_q, T_new, new_q_stride, L_max, L_prev, hkv, hq, d;
    int64_t pos_offset;
    const float2* cs;
    int64_t max_pos;
    int* err;
};
msa_status launch_append(const AppendArgs& a, msa_dtype dt, cudaStream_t s);
bool rope_layout_ok(msa_dtype dt, int d);

// Tensor-core router (tcgen05 + TMA + TMEM) over a bf16 index in unit-vector form.
//   index [n_chunks][K] bf16; qhat [n_pad][K] bf16 (rows >= N are zero); N = n_q * T columns.
//   doc_scores / chunk_scores pre-filled with -inf; results combined with float atomic max.
struct RouteTcArgs {
    const void* index;
    const void* qhat;
    int64_t n_chunks;
    int K;
    int N, n_pad, T;
    const int32_t* chunk_doc;
    int64_t n_docs;
    float* doc_scores;
    float* chunk_scores;
    int* err;
    int grid_cap;          // > 0: at most this many CTAs (SMs left free for concurrent work)
    int* tile_counter;     // zero at launch (route_prepare zeroes it)
    bool resident;         // keep qhat in shared memory when it fits (default: stream it with the index)
};
// Returns MSA_ERR_UNSUPPORTED (without launching) when the shape does not fit the kernel.
msa_status launch_route_tc(const RouteTcArgs& a, cudaStream_t s);
// Rows the tensor-core path needs in qhat for N columns (0 if unsupported).
int route_tc_pad_rows(int N, int K, bool resident = false);
// Testing knob: cap on the router's pipeline stages (0 = as many as the shared-memory budget allows).
void route_tc_set_max_stages(int n);
// Testing knob: launches withhold every tile so their bounded waits expire (MSA_DEV_WAIT_TIMEOUT).
void route_tc_inject_stall(int on);

// Router scoring split in two launches so a caller can hoist the (tiny) query prepass off the
// router's stream: route_prepare normalises the queries into qhat and fills the score outputs with
// -inf and zeroes the tile counter; route_launch runs the scorer. The workspace holds the tile
// counter in its first 256 bytes and qhat after it. grid_cap > 0 limits the scorer's CTAs.
struct RoutePlan {
    msa_dtype dt;
    int n_q, T, H, d, K, N, n_pad;
    bool use_tc;
    bool resident;
};
msa_status route_plan(msa_dtype dt, int64_t n_chunks, int n_q, int T, int H, int d, RoutePlan* plan);
msa_status route_prepare(const RoutePlan& p, const void* qr, void* ws, float* doc_scores, int64_t n_docs,
                         float* chunk_scores, int64_t n_chunks, cudaStream_t s);
msa_status route_launch(const RoutePlan& p, const void* kr_index, int64_t n_chunks, const int32_t* chunk_doc,
                        int64_t n_docs, void* ws, float* doc_scores, float* chunk_scores, int grid_cap,
                        cudaStream_t s);

// Device-side fetch of the selected documents' rows from a pinned (mapped) host bank.
msa_status gather_device(const void* host_bank, msa_dtype dt, int64_t n_chunks, const int64_t* doc_chunk_off,
                         int64_t n_docs, const int32_t* idx, int n_q, int k, int hkv, int d, int max_mem,
                         void* dev_mem_kv, int32_t* mem_len, cudaStream_t s);

}  // namespace msa
