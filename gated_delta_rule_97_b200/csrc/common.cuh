// Shared device helpers for the gated delta-rule kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

enum Update { kAdditive = 0, kDecay = 1, kDelta = 2 };
enum Gate { kGateNone = 0, kGateScalar = 1, kGateChannel = 2 };

constexpr int kChunk = 64;  // chunk length C of the chunkwise form

// Status codes written to the device status word (mirror gdn.h).
constexpr int kStatusTimeout = -5;
constexpr int kStatusRange = -6;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Multiprocessor count of the current device, cached per device (host side;
// grid sizing).  148 if the query fails.
inline int gdn_sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// Records the first error code seen by any kernel (0 = none yet).
__device__ __forceinline__ void record_status(int *status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// Arguments common to the prefill kernels.  All pointers are device pointers.
struct ChunkArgs {
    const void *q, *k, *v;   // [BH,T,dk] / [BH,T,dv], input dtype
    const float *g;          // [BH,T] or [BH,T,dk] or null
    const float *beta;       // [BH,T] or null
    const float *S0;         // [BH,dv,dk] or null
    void *o;                 // [BH,T,dv], output dtype
    float *ST;               // [BH,dv,dk] or null
    int *status;             // device status word
    int *diag;               // device diagnostic word (first timeout site)
    int BH, T, dk, dv;
    // Substeps per real token (Gated DeltaProduct; 1 otherwise).  T counts the
    // virtual steps (real tokens x nh): k, v, beta are laid out per virtual step,
    // q, g and o per real token; a token's q sits on its last substep, its gate
    // on its first, and only the last substep's output is written.
    int nh;
    int pro;   // GDN_PRO_* input maps
    int mode;  // kMode* bits (internal passes of the segmented prefill), 0 = plain
    float *states;  // kModeSaveStates: the chunk-entry states, else null
};

// Internal pass modes: values taken as zero (v not read), no output written,
// initial state the identity (dv == dk); with all three the pass yields the
// transition of the sequence (S_T = S0 Lambda with S0 = I).
constexpr int kModeZeroV = 1, kModeNoOut = 2, kModeS0Eye = 4;
// Forward for training: the state entering every chunk (before that chunk's
// decay) is also written to ChunkArgs::states [BH][nchunks][dv][dk], for the
// backward pass to start from.
constexpr int kModeSaveStates = 8;
// The tensor-core kernel runs kModeS0Eye from kEyeScale * I and stores S_T /
// kEyeScale (exact, a power of two): a transition that decays far below 1 then
// stays in fp16's normal range in the state's fp16 operand copy, while entries
// bounded by 1 (products of contractions) stay far below fp16's maximum.
constexpr float kEyeScale = 1024.f;

struct DecodeArgs {
    const void *q, *k, *v;   // [BH,T,dk] / [BH,T,dv]
    const float *g;          // [BH,T] or [BH,T,dk] or null
    const float *beta;       // [BH,T] or null
    float *S;                // [BH,dv,dk] in/out
    void *o;                 // [BH,T,dv]
    int BH, T, dk, dv;
    int pro;                 // GDN_PRO_* input maps
    int *status;             // device status word
    unsigned long long wait_ns;  // bound of the bulk-copy waits (0 = 1 s)
};

// Input prologue maps (GDN_PRO_* bits, mirrored here for device code).
constexpr int kProElu1 = 1, kProL2 = 2, kProBetaSigmoid = 4, kProGNegSoftplus = 8;

__device__ __forceinline__ float pro_feature(float x, int pro) {
    return (pro & kProElu1) ? (x > 0.f ? x + 1.f : __expf(x)) : x;
}
__device__ __forceinline__ float pro_beta(float x, int pro) {
    return (pro & kProBetaSigmoid) ? 1.f / (1.f + __expf(-x)) : x;
}
__device__ __forceinline__ float pro_gate(float x, int pro) {
    // -softplus(x) = -(max(x, 0) + log(1 + e^{-|x|}))
    return (pro & kProGNegSoftplus) ? -(fmaxf(x, 0.f) + log1pf(__expf(-fabsf(x)))) : x;
}

}  // namespace gdn

// Launchers (defined in the kernel .cu files).  Return a cudaError_t value.
int gdn_launch_chunk_simt(const gdn::ChunkArgs &a, int update, int gate, int in_bf16, int out_bf16,
                          cudaStream_t stream);
int gdn_launch_decode(const gdn::DecodeArgs &a, int update, int gate, int in_bf16, int out_bf16,
                      cudaStream_t stream);
int gdn_launch_copy_state(const float *S0, float *ST, long n, cudaStream_t stream);
int gdn_launch_compose(const float *S0, const float *H, const float *Lam, float *Sstart, float *ST, int BH, int nseg,
                       int dk, int dv, bool segment_major, cudaStream_t stream);
int gdn_launch_eye(float *L, long BH, int dk, cudaStream_t stream);
