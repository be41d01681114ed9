// Composition of per-segment state maps for the segmented (sequence-parallel)
// prefill.  A segment of the recurrence is an affine map of its incoming state,
// S_out = S_in Lambda + H ("Linear Attention, Visualized": "One chunk as an
// affine recurrence" and "Update the state": a run of tokens acts on the state
// through its transition product plus the writes it makes from a zero state).
// Given H_i and Lambda_i of every segment i (from two chunkwise passes), this
// kernel threads the state through the segments in order:
//     S_0 = S0 (or 0),   S_{i+1} = S_i Lambda_i + H_i,
// storing each S_i (the state entering segment i) and S_nseg (the final state).
// One CTA owns one head and 8 value rows; all arithmetic is fp32.  Matrix
// (head bh, segment i) of H, Lambda and S_i sits at index bh * sb + i * si:
// head-major (sb = nseg, si = 1) inside one call of the segmented prefill,
// segment-major (sb = 1, si = BH) for maps gathered from several devices.
#include "common.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 8;  // value rows per CTA: dv / 8 CTAs per head

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// Shared memory: two stages of {Lambda_i [DK][DK], H_i rows [kRows][DK]} and the
// running state rows S [kRows][DK], all fp32.
template <int DK>
struct ComposeSmem {
    static constexpr int kStage = DK * DK + kRows * DK;  // floats
    static constexpr size_t kBytes = (size_t)(2 * kStage + kRows * DK) * sizeof(float);
};

// Thread t owns column c = t % DK of RPT = kRows * DK / 256 consecutive rows, so
// Lambda reads are conflict-free and the S reads are warp-wide broadcasts.
template <int DK>
__global__ void __launch_bounds__(kThreads) compose_kernel(const float *S0, const float *H, const float *Lam,
                                                           float *Sstart, float *ST, int nseg, int dv, long sb,
                                                           long si) {
    extern __shared__ __align__(16) float sm[];
    constexpr int kStage = ComposeSmem<DK>::kStage;
    constexpr int RPT = kRows * DK / kThreads;  // 4 (DK = 128) or 2 (DK = 64)
    float *S = sm + 2 * kStage;
    const int t = threadIdx.x;
    const long bh = blockIdx.x;
    const int v0 = blockIdx.y * kRows;
    const int c = t % DK, r0 = (t / DK) * RPT;

    // stage i: Lambda_i (unless the transitions are the identity) and H_i's rows
    auto prefetch = [&](int i, int buf) {
        const size_t seg = (size_t)(bh * sb + (long)i * si);
        float *dst = sm + buf * kStage;
        if (Lam) {
            const float *L = Lam + seg * DK * DK;
            for (int e = t * 4; e < DK * DK; e += kThreads * 4) cp_async16(dst + e, L + e);
        }
        const float *Hr = H + (seg * dv + v0) * DK;
        for (int e = t * 4; e < kRows * DK; e += kThreads * 4) cp_async16(dst + DK * DK + e, Hr + e);
        cp_async_commit();
    };

    for (int i = t; i < kRows * DK; i += kThreads) S[i] = S0 ? S0[((size_t)bh * dv + v0) * DK + i] : 0.f;
    prefetch(0, 0);
    for (int i = 0; i < nseg; ++i) {
        const int buf = i & 1;
        if (i + 1 < nseg) {
            prefetch(i + 1, buf ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();  // stage i landed for every thread; S holds S_i
        const float *L = sm + buf * kStage;
        const float *Hs = L + DK * DK;
        const size_t seg = (size_t)(bh * sb + (long)i * si);
        float acc[RPT];
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
            const float sv = S[(r0 + j) * DK + c];
            if (Sstart) Sstart[(seg * dv + v0 + r0 + j) * DK + c] = sv;
            acc[j] = Hs[(r0 + j) * DK + c] + (Lam ? 0.f : sv);
        }
        if (Lam) {
#pragma unroll 4
            for (int m = 0; m < DK; m += 4) {
                const float l0 = L[(m + 0) * DK + c], l1 = L[(m + 1) * DK + c];
                const float l2 = L[(m + 2) * DK + c], l3 = L[(m + 3) * DK + c];
#pragma unroll
                for (int j = 0; j < RPT; ++j) {
                    const float4 sv = *reinterpret_cast<const float4 *>(S + (r0 + j) * DK + m);
                    acc[j] = fmaf(sv.x, l0, acc[j]);
                    acc[j] = fmaf(sv.y, l1, acc[j]);
                    acc[j] = fmaf(sv.z, l2, acc[j]);
                    acc[j] = fmaf(sv.w, l3, acc[j]);
                }
            }
        }
        __syncthreads();  // every read of S and of this stage is done
#pragma unroll
        for (int j = 0; j < RPT; ++j) S[(r0 + j) * DK + c] = acc[j];
    }
    __syncthreads();
    if (ST)
        for (int i = t; i < kRows * DK; i += kThreads) ST[((size_t)bh * dv + v0) * DK + i] = S[i];
}

// BH identity matrices of size dk x dk (the transition of an empty segment).
__global__ void eye_kernel(float *L, long n, int dk) {
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        const long e = i % ((long)dk * dk);
        L[i] = (e / dk == e % dk) ? 1.f : 0.f;
    }
}

}  // namespace
}  // namespace gdn

namespace {
template <int DK>
int launch_compose(const float *S0, const float *H, const float *Lam, float *Sstart, float *ST, int BH, int nseg,
                   int dv, long sb, long si, cudaStream_t stream) {
    constexpr size_t bytes = gdn::ComposeSmem<DK>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(gdn::compose_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e != cudaSuccess) return (int)e;
    const dim3 grid((unsigned)BH, (unsigned)(dv / gdn::kRows));
    gdn::compose_kernel<DK><<<grid, gdn::kThreads, bytes, stream>>>(S0, H, Lam, Sstart, ST, nseg, dv, sb, si);
    return (int)cudaGetLastError();
}
}  // namespace

int gdn_launch_compose(const float *S0, const float *H, const float *Lam, float *Sstart, float *ST, int BH, int nseg,
                       int dk, int dv, bool segment_major, cudaStream_t stream) {
    if (BH == 0) return 0;
    const long sb = segment_major ? 1 : nseg, si = segment_major ? BH : 1;
    if (dk == 64) return launch_compose<64>(S0, H, Lam, Sstart, ST, BH, nseg, dv, sb, si, stream);
    return launch_compose<128>(S0, H, Lam, Sstart, ST, BH, nseg, dv, sb, si, stream);
}

int gdn_launch_eye(float *L, long BH, int dk, cudaStream_t stream) {
    const long n = BH * dk * dk;
    if (n <= 0) return 0;
    long blocks = (n + 255) / 256;
    if (blocks > gdn::gdn_sm_count() * 16L) blocks = gdn::gdn_sm_count() * 16L;
    gdn::eye_kernel<<<(unsigned)blocks, 256, 0, stream>>>(L, n, dk);
    return (int)cudaGetLastError();
}
