// Small helpers shared by the tensor-core prefill kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace gdn {
namespace tcu {

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ void unpack_bf16x8(uint4 u, float *f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint4 pack_h8(const float *f) {
    return make_uint4(pack_h2(f[0], f[1]), pack_h2(f[2], f[3]), pack_h2(f[4], f[5]), pack_h2(f[6], f[7]));
}

// Float offset of element (r, c) in a row-major fp32 tile with `ld` columns
// whose 16-byte slots are XOR-swizzled by (r % 8).
__device__ __forceinline__ int f32_swz(int r, int c, int ld) {
    return r * ld + ((((c >> 2) ^ (r & 7))) << 2) + (c & 3);
}

// 2^x on the special-function unit (PTX ex2.approx.ftz.f32; relative error near
// the fp32 ulp, flushes subnormal results to zero).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// fp32 -> tf32 (round to nearest, ties away), as a 32-bit operand register.
__device__ __forceinline__ uint32_t f2tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// Warp-level D += A B, A 16x8 (row), B 8x8 (col), tf32 in, fp32 accumulate.
// Fragments (g = lane / 4, q = lane % 4):
//   a = {A[g][q], A[g+8][q], A[g][q+4], A[g+8][q+4]},  b = {B[q][g], B[q+4][g]},
//   d = {D[g][2q], D[g][2q+1], D[g+8][2q], D[g+8][2q+1]}.
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

}  // namespace tcu
}  // namespace gdn
