// Fetch of the selected documents' compressed K-bar/V-bar rows from the pinned host bank.
//
// The bank is [n_chunks][2][hkv][d]: one document is one contiguous byte run, so each selected
// document is one cudaMemcpyAsync host -> device on the copy stream (the copy engines over the
// host link), written into the query's slot at the running row offset (rank order).
#include "common.cuh"

using namespace msa;

extern "C" {

msa_status msa_gather_kv(const void* host_bank, msa_dtype dt, int64_t n_chunks, const int64_t* doc_chunk_off_host,
                         int64_t n_docs, const int32_t* idx_host, int n_q, int k, int hkv, int d, int max_mem,
                         void* dev_mem_kv, int32_t* mem_len_host, void* copy_stream) {
    MSA_REQUIRE(dtype_ok(dt), "msa_gather_kv: bad dtype");
    MSA_REQUIRE(host_bank && doc_chunk_off_host && idx_host && dev_mem_kv && mem_len_host,
                "msa_gather_kv: NULL pointer");
    MSA_REQUIRE(n_q > 0 && k > 0 && hkv > 0 && d > 0 && max_mem >= 0 && n_docs > 0 && n_chunks >= 0,
                "msa_gather_kv: bad sizes");
    const size_t row = (size_t)2 * hkv * d * dtype_size(dt);
    // validate everything before enqueueing anything
    for (int q = 0; q < n_q; ++q) {
        int64_t rows = 0;
        for (int r = 0; r < k; ++r) {
            const int32_t doc = idx_host[(int64_t)q * k + r];
            MSA_REQUIRE(doc >= 0 && doc < n_docs, "msa_gather_kv: query %d rank %d: doc %d out of range", q, r, doc);
            const int64_t a = doc_chunk_off_host[doc], b = doc_chunk_off_host[doc + 1];
            MSA_REQUIRE(a >= 0 && b >= a && b <= n_chunks, "msa_gather_kv: bad doc_chunk_off for doc %d", doc);
            rows += b - a;
        }
        MSA_REQUIRE(rows <= max_mem, "msa_gather_kv: query %d needs %lld rows > max_mem %d", q, (long long)rows,
                    max_mem);
    }
    cudaStream_t s = static_cast<cudaStream_t>(copy_stream);
    const char* src = static_cast<const char*>(host_bank);
    char* dst = static_cast<char*>(dev_mem_kv);
    for (int q = 0; q < n_q; ++q) {
        int64_t at = 0;
        for (int r = 0; r < k; ++r) {
            const int32_t doc = idx_host[(int64_t)q * k + r];
            const int64_t a = doc_chunk_off_host[doc], b = doc_chunk_off_host[doc + 1];
            if (b > a)
                MSA_CUDA_TRY(cudaMemcpyAsync(dst + ((int64_t)q * max_mem + at) * row, src + a * row, (b - a) * row,
                                             cudaMemcpyHostToDevice, s));
            at += b - a;
        }
        mem_len_host[q] = (int32_t)at;
    }
    return MSA_OK;
}

}  // extern "C"
