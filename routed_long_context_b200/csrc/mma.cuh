// Warp-level bf16 tensor-core helpers shared by the attention kernels (mma.sync m16n8k16 with fp32
// accumulation, ldmatrix, cp.async).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace msa {

// c[4] += A[16x16] B[16x8]; a: 4 registers of bf16 pairs (row-major A), b0/b1: col-major B.
__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 2^x by the hardware base-2 exponential (PTX ex2.approx.ftz.f32, relative error about 2^-22;
// 2^-inf = 0). Used where the result is rounded to a bf16 operand right after.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Four transposed 8x8 bf16 matrices from shared memory (lane l supplies the address of row l % 8 of
// matrix l / 8).
__device__ __forceinline__ void ldmatrix_x4_trans(const void* smem_row, uint32_t& b0, uint32_t& b1, uint32_t& b2,
                                                  uint32_t& b3) {
    const uint32_t addr = static_cast<uint32_t>(__cvta_generic_to_shared(smem_row));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
                 : "r"(addr));
}

// 16-byte asynchronous global -> shared copy; with valid == false nothing is read and the
// destination is zero-filled (src must still be a valid address).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* src, bool valid) {
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

}  // namespace msa
