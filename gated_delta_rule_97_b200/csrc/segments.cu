// Composition of per-segment state maps for the segmented (sequence-parallel)
// prefill.  A segment of the recurrence is an affine map of its incoming state,
// S_out = S_in Lambda + H ("Linear Attention, Visualized": "One chunk as an
// affine recurrence" and "Update the state": a run of tokens acts on the state
// through its transition product plus the writes it makes from a zero state).
// Given H_i and Lambda_i of every segment i (from two chunkwise passes), this
// kernel threads the state through the segments in order:
//     S_0 = S0 (or 0),   S_{i+1} = S_i Lambda_i + H_i,
// storing each S_i (the state entering segment i) and S_nseg (the final state).
// One CTA owns one head and 32 value rows; all arithmetic is fp32.
#include "common.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 32;

template <int DK>
__global__ void __launch_bounds__(kThreads) compose_kernel(const float *S0, const float *H, const float *Lam,
                                                           float *Sstart, float *ST, int nseg, int dv) {
    __shared__ float S[kRows][DK];
    const int t = threadIdx.x;
    const long bh = blockIdx.x;
    const int v0 = blockIdx.y * kRows;
    constexpr int CPT = DK / 8;  // columns per thread
    const int r = t >> 3, c0 = (t & 7) * CPT;
    for (int i = t; i < kRows * DK; i += kThreads) {
        const int rr = i / DK, c = i % DK;
        S[rr][c] = S0 ? S0[((size_t)bh * dv + v0 + rr) * DK + c] : 0.f;
    }
    __syncthreads();
    for (int i = 0; i < nseg; ++i) {
        const size_t seg = (size_t)bh * nseg + i;
        float acc[CPT];
#pragma unroll
        for (int e = 0; e < CPT; ++e) {
            Sstart[(seg * dv + v0 + r) * DK + c0 + e] = S[r][c0 + e];
            acc[e] = H[(seg * dv + v0 + r) * DK + c0 + e];
        }
        if (Lam) {
            const float *L = Lam + seg * DK * DK;
            for (int m = 0; m < DK; ++m) {
                const float s = S[r][m];
#pragma unroll
                for (int e = 0; e < CPT; ++e) acc[e] = fmaf(s, L[(size_t)m * DK + c0 + e], acc[e]);
            }
        } else {  // identity transition (no gate, additive write)
#pragma unroll
            for (int e = 0; e < CPT; ++e) acc[e] += S[r][c0 + e];
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < CPT; ++e) S[r][c0 + e] = acc[e];
        __syncthreads();
    }
    if (ST) {
#pragma unroll
        for (int e = 0; e < CPT; ++e) ST[((size_t)bh * dv + v0 + r) * DK + c0 + e] = S[r][c0 + e];
    }
}

}  // namespace
}  // namespace gdn

int gdn_launch_compose(const float *S0, const float *H, const float *Lam, float *Sstart, float *ST, int BH, int nseg,
                       int dk, int dv, cudaStream_t stream) {
    const dim3 grid((unsigned)BH, (unsigned)(dv / gdn::kRows));
    if (BH == 0) return 0;
    if (dk == 64)
        gdn::compose_kernel<64><<<grid, gdn::kThreads, 0, stream>>>(S0, H, Lam, Sstart, ST, nseg, dv);
    else
        gdn::compose_kernel<128><<<grid, gdn::kThreads, 0, stream>>>(S0, H, Lam, Sstart, ST, nseg, dv);
    return (int)cudaGetLastError();
}
