// Fetch of the selected documents' compressed K-bar/V-bar rows from the pinned host bank.
//
// The bank is [n_chunks][2][hkv][d]: one document is one contiguous byte run, so each selected
// document is one cudaMemcpyAsync host -> device on the copy stream (the copy engines over the
// host link), written into the query's slot at the running row offset (rank order).
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

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

// ------------------------------------------------------------------------------------------------
// Device-side fetch: a kernel reads the selected documents' rows straight from the pinned host bank
// (mapped into the device's address space) using device-resident indices, so selection and fetch
// need no host round trip. Blocks (rank, query, part): a document's 16-byte words are dealt out to
// gridDim.z blocks (one for compressed chunk rows, up to 32 for the token rows of the fine stage)
// so enough loads are in flight over the host link.
// ------------------------------------------------------------------------------------------------
namespace msa {
namespace {

__global__ void __launch_bounds__(256) gather_device_kernel(const uint4* __restrict__ bank, int64_t n_chunks,
                                                            const int64_t* __restrict__ doc_chunk_off, int64_t n_docs,
                                                            const int32_t* __restrict__ idx, int k, int row_vec,
                                                            int max_mem, uint4* __restrict__ out,
                                                            int32_t* __restrict__ mem_len, int* err) {
    const int q = blockIdx.y, r = blockIdx.x;
    const int32_t* sel = idx + (int64_t)q * k;
    // rows of the ranks before this one, and this document's rows
    int64_t at = 0;
    bool ok = true;
    for (int j = 0; j <= r; ++j) {
        const int32_t doc = sel[j];
        if (doc < 0 || doc >= n_docs) {
            ok = false;
            break;
        }
        const int64_t a = doc_chunk_off[doc], b = doc_chunk_off[doc + 1];
        if (a < 0 || b < a || b > n_chunks) {
            ok = false;
            break;
        }
        if (j < r) at += b - a;
    }
    if (!ok) {
        if (threadIdx.x == 0) record_device_error(err, MSA_DEV_BAD_INDEX);
        return;
    }
    const int32_t doc = sel[r];
    const int64_t a = doc_chunk_off[doc], rows = doc_chunk_off[doc + 1] - a;
    if (at + rows > max_mem) {
        if (threadIdx.x == 0) record_device_error(err, MSA_DEV_BAD_INDEX);
        return;
    }
    if (r == k - 1 && blockIdx.z == 0 && threadIdx.x == 0) mem_len[q] = (int32_t)(at + rows);
    const uint4* src = bank + a * row_vec;
    uint4* dst = out + ((int64_t)q * max_mem + at) * row_vec;
    const int64_t n = rows * row_vec;
    const int64_t step = (int64_t)gridDim.z * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.z * blockDim.x + threadIdx.x; i < n; i += 4 * step) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (i + u * step < n) v[u] = src[i + u * step];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (i + u * step < n) dst[i + u * step] = v[u];
    }
}

}  // namespace

msa_status gather_device(const void* host_bank, msa_dtype dt, int64_t n_chunks, const int64_t* doc_chunk_off,
                         int64_t n_docs, const int32_t* idx, int n_q, int k, int hkv, int d, int max_mem,
                         void* dev_mem_kv, int32_t* mem_len, cudaStream_t s) {
    // a bank in this device's memory (training) is read directly; a host bank through its mapping
    void* dptr = nullptr;
    cudaPointerAttributes attr{};
    int dev = -1;
    if (cudaPointerGetAttributes(&attr, host_bank) == cudaSuccess && attr.type == cudaMemoryTypeDevice &&
        cudaGetDevice(&dev) == cudaSuccess && attr.device == dev) {
        dptr = const_cast<void*>(host_bank);
    } else {
        (void)cudaGetLastError();
        const cudaError_t e = cudaHostGetDevicePointer(&dptr, const_cast<void*>(host_bank), 0);
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            return set_error(MSA_ERR_INVALID_ARG,
                             "device fetch: the bank is neither this device's memory nor pinned, mapped host memory (%s)",
                             cudaGetErrorString(e));
        }
    }
    const size_t row = (size_t)2 * hkv * d * dtype_size(dt);
    if (row % 16 != 0 || !aligned16(dptr) || !aligned16(dev_mem_kv))
        return set_error(MSA_ERR_INVALID_ARG, "device fetch: rows and pointers must be 16-byte aligned");
    // words per document if the rows were spread evenly; one block per 8K words, at most 32
    const int64_t words = ((int64_t)max_mem * (int64_t)(row / 16)) / k;
    const int parts = (int)std::min<int64_t>(32, std::max<int64_t>(1, (words + 8191) / 8192));
    dim3 grid(k, n_q, parts);
    gather_device_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(dptr), n_chunks, doc_chunk_off, n_docs, idx, k,
                                              (int)(row / 16), max_mem, static_cast<uint4*>(dev_mem_kv), mem_len,
                                              device_error_word());
    MSA_LAUNCH_CHECK();
    return MSA_OK;
}

}  // namespace msa

extern "C" {

msa_status msa_gather_kv_device(const void* host_bank, msa_dtype dt, int64_t n_chunks, const int64_t* doc_chunk_off,
                                int64_t n_docs, const int32_t* idx, int n_q, int k, int hkv, int d, int max_mem,
                                void* dev_mem_kv, int32_t* mem_len, void* stream) {
    MSA_REQUIRE(dtype_ok(dt), "msa_gather_kv_device: bad dtype");
    MSA_REQUIRE(host_bank && doc_chunk_off && idx && dev_mem_kv && mem_len, "msa_gather_kv_device: NULL pointer");
    MSA_REQUIRE(n_q > 0 && n_q <= 65535 && k > 0 && hkv > 0 && d > 0 && max_mem >= 0 && n_docs > 0 && n_chunks >= 0,
                "msa_gather_kv_device: bad sizes");
    return gather_device(host_bank, dt, n_chunks, doc_chunk_off, n_docs, idx, n_q, k, hkv, d, max_mem, dev_mem_kv,
                         mem_len, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
