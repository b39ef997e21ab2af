// Shared helpers of the MSA library: error reporting, dtype conversion, vector loads.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "msa.h"

namespace msa {

// Records a formatted message for msa_last_error() and returns `st`.
msa_status set_error(msa_status st, const char* fmt, ...);
// Device address of the device-side error word of the current device (cached per device).
int* device_error_word();
// Number of SMs of the current device (cached per device).
int sm_count();

#define MSA_CUDA_TRY(expr)                                                                                 \
    do {                                                                                                   \
        cudaError_t e_ = (expr);                                                                           \
        if (e_ != cudaSuccess)                                                                             \
            return ::msa::set_error(MSA_ERR_CUDA, "%s failed: %s (%s:%d)", #expr, cudaGetErrorString(e_), \
                                    __FILE__, __LINE__);                                                   \
    } while (0)

#define MSA_LAUNCH_CHECK()                                                                                  \
    do {                                                                                                    \
        cudaError_t e_ = cudaGetLastError();                                                                \
        if (e_ != cudaSuccess)                                                                              \
            return ::msa::set_error(MSA_ERR_CUDA, "kernel launch failed: %s (%s:%d)", cudaGetErrorString(e_), \
                                    __FILE__, __LINE__);                                                    \
    } while (0)

#define MSA_REQUIRE(cond, ...)                                                         \
    do {                                                                               \
        if (!(cond)) return ::msa::set_error(MSA_ERR_INVALID_ARG, __VA_ARGS__);        \
    } while (0)

#define MSA_RETURN_IF(st)               \
    do {                                \
        msa_status s_ = (st);           \
        if (s_ != MSA_OK) return s_;    \
    } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t dtype_size(msa_dtype dt) { return dt == MSA_BF16 ? 2 : 4; }
inline bool dtype_ok(msa_dtype dt) { return dt == MSA_F32 || dt == MSA_BF16; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__device__ __forceinline__ void record_device_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

// ---- element conversion --------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// 16-byte vector of T: 4 floats or 8 bf16.
template <typename T> struct Vec16 { static constexpr int N = 16 / sizeof(T); };

// Loads N = 16/sizeof(T) consecutive elements (16-byte aligned) and widens them to fp32.
template <typename T>
__device__ __forceinline__ void load16_f32(const T* p, float* out) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
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

// Stores n fp32 values as T (n * sizeof(T) bytes, aligned to that size when n*sizeof(T) is 8 or 16).
template <typename T, int N>
__device__ __forceinline__ void store_f32(T* p, const float* v) {
    if constexpr (sizeof(T) == 4) {
        if constexpr (N % 4 == 0) {
#pragma unroll
            for (int i = 0; i < N; i += 4)
                *reinterpret_cast<float4*>(p + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        } else {
#pragma unroll
            for (int i = 0; i < N; ++i) p[i] = v[i];
        }
    } else {
        if constexpr (N % 8 == 0) {
#pragma unroll
            for (int i = 0; i < N; i += 8) {
                uint4 u;
                __nv_bfloat162 a = __floats2bfloat162_rn(v[i], v[i + 1]);
                __nv_bfloat162 b = __floats2bfloat162_rn(v[i + 2], v[i + 3]);
                __nv_bfloat162 c = __floats2bfloat162_rn(v[i + 4], v[i + 5]);
                __nv_bfloat162 d = __floats2bfloat162_rn(v[i + 6], v[i + 7]);
                u.x = *reinterpret_cast<uint32_t*>(&a); u.y = *reinterpret_cast<uint32_t*>(&b);
                u.z = *reinterpret_cast<uint32_t*>(&c); u.w = *reinterpret_cast<uint32_t*>(&d);
                *reinterpret_cast<uint4*>(p + i) = u;
            }
        } else if constexpr (N % 4 == 0) {
#pragma unroll
            for (int i = 0; i < N; i += 4) {
                uint2 u;
                __nv_bfloat162 a = __floats2bfloat162_rn(v[i], v[i + 1]);
                __nv_bfloat162 b = __floats2bfloat162_rn(v[i + 2], v[i + 3]);
                u.x = *reinterpret_cast<uint32_t*>(&a); u.y = *reinterpret_cast<uint32_t*>(&b);
                *reinterpret_cast<uint2*>(p + i) = u;
            }
        } else {
#pragma unroll
            for (int i = 0; i < N; ++i) p[i] = __float2bfloat16_rn(v[i]);
        }
    }
}

// Float atomic max that works for any sign on float storage initialised to -inf (no NaNs):
// values with a clear sign bit order like signed ints, values with the sign bit set order
// inversely as unsigned ints (so -0.0 and negatives go through atomicMin on the bits).
__device__ __forceinline__ void atomic_max_f32(float* addr, float v) {
    if (!(__float_as_uint(v) & 0x80000000u))
        atomicMax(reinterpret_cast<int*>(addr), __float_as_int(v));
    else
        atomicMin(reinterpret_cast<unsigned int*>(addr), __float_as_uint(v));
}

}  // namespace msa
