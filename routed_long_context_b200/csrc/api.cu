// Library-wide entry points: error text, device error word, RoPE table, chunk -> document map.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "common.cuh"

namespace msa {

namespace {
thread_local char g_err[1024] = "";
__device__ int g_device_error = 0;   // first run-time error recorded by any kernel (MSA_DEV_*)

constexpr int kMaxDevices = 64;
int* g_err_ptr[kMaxDevices] = {nullptr};
int g_sms[kMaxDevices] = {0};
std::mutex g_mu;
}  // namespace

msa_status set_error(msa_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return st;
}

int* device_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_err_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        g_err_ptr[dev] = static_cast<int*>(p);
    }
    return g_err_ptr[dev];
}

int sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_sms[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        g_sms[dev] = n;
    }
    return g_sms[dev];
}

namespace {
__global__ void chunk_doc_kernel(const int64_t* __restrict__ doc_chunk_off, int64_t n_docs, int64_t n_chunks,
                                 int32_t* __restrict__ chunk_doc, int* err) {
    for (int64_t doc = blockIdx.x; doc < n_docs; doc += gridDim.x) {
        const int64_t a = doc_chunk_off[doc], b = doc_chunk_off[doc + 1];
        if (a < 0 || b > n_chunks || a > b) {
            if (threadIdx.x == 0) record_device_error(err, MSA_DEV_BAD_INDEX);
            continue;
        }
        for (int64_t c = a + threadIdx.x; c < b; c += blockDim.x) chunk_doc[c] = (int32_t)doc;
    }
}
}  // namespace

}  // namespace msa

using namespace msa;

extern "C" {

const char* msa_last_error(void) { return g_err; }

const char* msa_version(void) { return "msa-b200 0.1 (sm_100a)"; }

msa_status msa_device_status(int32_t* code, void* stream) {
    MSA_REQUIRE(code != nullptr, "msa_device_status: code is NULL");
    int* p = device_error_word();
    if (!p) return set_error(MSA_ERR_CUDA, "msa_device_status: cannot resolve the device error word");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    MSA_CUDA_TRY(cudaStreamSynchronize(s));
    int v = 0;
    MSA_CUDA_TRY(cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost));
    const int zero = 0;
    MSA_CUDA_TRY(cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice));
    *code = v;
    return MSA_OK;
}

msa_status msa_rope_table(int64_t max_pos, int d, double base, float* out_host) {
    MSA_REQUIRE(out_host != nullptr, "msa_rope_table: out_host is NULL");
    MSA_REQUIRE(max_pos > 0 && d > 0 && d % 2 == 0, "msa_rope_table: need max_pos > 0 and even d > 0");
    MSA_REQUIRE(base > 1.0, "msa_rope_table: base must be > 1");
    const int half = d / 2;
    for (int64_t p = 0; p < max_pos; ++p) {
        for (int i = 0; i < half; ++i) {
            const double w = std::pow(base, -2.0 * (double)i / (double)d);
            const double a = (double)p * w;
            out_host[(p * half + i) * 2 + 0] = (float)std::cos(a);
            out_host[(p * half + i) * 2 + 1] = (float)std::sin(a);
        }
    }
    return MSA_OK;
}

msa_status msa_workspace_size(int op, const void* cfg, size_t* bytes) {
    MSA_REQUIRE(cfg != nullptr && bytes != nullptr, "msa_workspace_size: cfg and bytes must not be NULL");
    switch (op) {
        case MSA_OP_ROUTE: {
            const auto* c = static_cast<const msa_route_ws_cfg*>(cfg);
            return msa_route_workspace_size(c->n_q, c->T, c->H, c->d, c->dt, bytes);
        }
        case MSA_OP_TOPK: {
            const auto* c = static_cast<const msa_topk_ws_cfg*>(cfg);
            return msa_topk_workspace_size(c->n_q, c->n_docs, c->k, bytes);
        }
        case MSA_OP_SPARSE_ATTN_SPLIT: {
            const auto* c = static_cast<const msa_attn_ws_cfg*>(cfg);
            return msa_sparse_attn_split_workspace_size(c->n_q, c->T, c->hq, c->hkv, c->max_mem, c->L, bytes);
        }
        case MSA_OP_SPARSE_ATTN_BACKWARD: {
            const auto* c = static_cast<const msa_attn_ws_cfg*>(cfg);
            return msa_sparse_attn_backward_workspace_size(c->n_q, c->T, c->hq, c->hkv, c->max_mem, c->L, bytes);
        }
        case MSA_OP_ROUTE_BACKWARD: {
            const auto* c = static_cast<const msa_route_bwd_ws_cfg*>(cfg);
            return msa_route_backward_workspace_size(c->n_chunks, c->n_q, c->T, c->H, c->d, bytes);
        }
        case MSA_OP_INTERLEAVE:
            return msa_interleave_workspace_size(static_cast<const msa_interleave_args*>(cfg), bytes);
        default:
            return set_error(MSA_ERR_INVALID_ARG, "msa_workspace_size: unknown op %d", op);
    }
}

msa_status msa_chunk_doc_map(const int64_t* doc_chunk_off, int64_t n_docs, int64_t n_chunks, int32_t* chunk_doc,
                             void* stream) {
    MSA_REQUIRE(doc_chunk_off && chunk_doc, "msa_chunk_doc_map: NULL pointer");
    MSA_REQUIRE(n_docs >= 0 && n_chunks >= 0 && n_docs < (int64_t)INT32_MAX, "msa_chunk_doc_map: bad sizes");
    if (n_docs == 0 || n_chunks == 0) return MSA_OK;
    int64_t blocks = n_docs < (int64_t)sm_count() * 64 ? n_docs : (int64_t)sm_count() * 64;
    chunk_doc_kernel<<<(unsigned)blocks, 128, 0, static_cast<cudaStream_t>(stream)>>>(doc_chunk_off, n_docs, n_chunks,
                                                                                      chunk_doc, device_error_word());
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

}  // extern "C"
