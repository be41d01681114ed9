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

}  // namespace tcu
}  // namespace gdn
