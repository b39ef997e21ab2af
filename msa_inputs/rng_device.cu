// Device side of the seeded input generator (test and benchmark inputs only).
//
// Holds no arithmetic of the attention method. It fills device memory with
// the same values rng_host.c produces for (seed, tensor id, flat index):
// SplitMix64 draws (Steele, Lea and Flood, OOPSLA 2014) turned into an
// Irwin-Hall(4) pseudo-normal, scaled by sigma in fp32 and optionally
// rounded to bf16 with round-to-nearest-even. Every product is written with
// __fmul_rn so the compiler cannot fuse it, which keeps the bits equal to
// the host generator's.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace {

constexpr uint64_t kG = 0x9E3779B97F4A7C15ULL;

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

__device__ __forceinline__ float irwin_hall4(uint64_t h) {
    int s = (int)(h & 0xFFFFULL) + (int)((h >> 16) & 0xFFFFULL) + (int)((h >> 32) & 0xFFFFULL) + (int)(h >> 48);
    float t = __fmul_rn(__int2float_rn(s - 131070), 1.0f / 65536.0f);
    return __fmul_rn(t, 1.7320508075688772f);
}

template <typename T>
__global__ void fill_normal_kernel(T* __restrict__ out, uint64_t base, uint64_t start, int64_t n, float sigma) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n; j += stride) {
        float v = __fmul_rn(irwin_hall4(mix64(base + kG * (start + (uint64_t)j + 1ULL))), sigma);
        if constexpr (sizeof(T) == 4) {
            out[j] = v;
        } else {
            out[j] = __float2bfloat16_rn(v);
        }
    }
}

}  // namespace

extern "C" {

// Fills out[0..n) with the generator's values for flat indices start..start+n-1.
// dtype: 0 = fp32, 1 = bf16. Returns a cudaError_t code (0 = success).
int rng_fill_normal(void* out, int dtype, uint64_t seed, uint64_t tid, uint64_t start, int64_t n, float sigma,
                    void* stream) {
    if (n <= 0) return 0;
    if (out == nullptr || (dtype != 0 && dtype != 1)) return (int)cudaErrorInvalidValue;
    const uint64_t base = mix64(seed + kG * (tid + 1ULL));
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (n + 255) / 256;
    const int64_t cap = (int64_t)sms * 16;
    if (blocks > cap) blocks = cap;
    cudaStream_t s = (cudaStream_t)stream;
    if (dtype == 0)
        fill_normal_kernel<float><<<(unsigned)blocks, 256, 0, s>>>((float*)out, base, start, n, sigma);
    else
        fill_normal_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>((__nv_bfloat16*)out, base, start, n, sigma);
    return (int)cudaGetLastError();
}

}  // extern "C"
