// The backward pass through the input prologue maps (gdn_chunk_bwd with
// desc->prologue != 0).  The forward applies, per token row, q, k <- elu(x) + 1
// and/or x / |x|_2, beta <- sigmoid(beta), g <- -softplus(g) ("Linear
// Attention, Visualized": "Linear attention: a running sum" for the feature
// map, the DeltaNet forward's normalised q and k, "Optional: Constructing the
// decay gate").  The backward runs in three steps:
//   1. map: the mapped q, k, beta, g (and v) are written in fp32 to the
//      workspace, as the forward computed them;
//   2. the recurrence's backward (backward.cu) on those mapped inputs;
//   3. chain rule, in place on dq, dk, dbeta, dg, per token row:
//        unit rows y = e / |e|:  de = (dy - y (y . dy)) / |e|  (0 for a zero row)
//        elu(x) + 1:             dx = de (x > 0), de e^x (x <= 0)
//        sigmoid:                db = dbeta s (1 - s)
//        -softplus:              dx = -dg sigmoid(x)
// One warp per token row; lane l holds channels l, l + 32, ...
#include "common.cuh"

namespace gdn {
namespace {

constexpr int kPBThreads = 256;

template <typename TIn>
__device__ __forceinline__ float ld_in(const void *p, size_t i) {
    return to_f32(static_cast<const TIn *>(p)[i]);
}

__device__ __forceinline__ float warp_allsum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// Feature map of one row (NE = dk / 32 channels per lane) from raw values x.
template <int NE>
__device__ __forceinline__ void feature_row(const float (&x)[NE], float (&y)[NE], float &norm, int pro) {
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < NE; ++e) {
        y[e] = pro_feature(x[e], pro);
        ss = fmaf(y[e], y[e], ss);
    }
    norm = sqrtf(warp_allsum(ss));
    if (pro & kProL2) {
        const float inv = norm > 0.f ? 1.f / norm : 0.f;
#pragma unroll
        for (int e = 0; e < NE; ++e) y[e] *= inv;
    }
}

template <int DK, typename TIn>
__global__ void __launch_bounds__(kPBThreads) prologue_map_kernel(const void *q, const void *k, const void *v,
                                                                  const float *g, const float *beta, float *qm,
                                                                  float *km, float *vf, float *gm, float *bm,
                                                                  long rows, int dv, int gate, int pro) {
    constexpr int NE = DK / 32;
    const long row = ((long)blockIdx.x * kPBThreads + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float x[NE], y[NE], n;
#pragma unroll
    for (int e = 0; e < NE; ++e) x[e] = ld_in<TIn>(q, (size_t)row * DK + lane + 32 * e);
    feature_row<NE>(x, y, n, pro);
#pragma unroll
    for (int e = 0; e < NE; ++e) qm[(size_t)row * DK + lane + 32 * e] = y[e];
#pragma unroll
    for (int e = 0; e < NE; ++e) x[e] = ld_in<TIn>(k, (size_t)row * DK + lane + 32 * e);
    feature_row<NE>(x, y, n, pro);
#pragma unroll
    for (int e = 0; e < NE; ++e) km[(size_t)row * DK + lane + 32 * e] = y[e];
    for (int c = lane; c < dv; c += 32) vf[(size_t)row * dv + c] = ld_in<TIn>(v, (size_t)row * dv + c);
    if (bm && lane == 0) bm[row] = pro_beta(beta[row], pro);
    if (gm) {
        if (gate == kGateChannel) {
#pragma unroll
            for (int e = 0; e < NE; ++e)
                gm[(size_t)row * DK + lane + 32 * e] = pro_gate(g[(size_t)row * DK + lane + 32 * e], pro);
        } else if (lane == 0) {
            gm[row] = pro_gate(g[row], pro);
        }
    }
}

template <int NE>
__device__ __forceinline__ void feature_row_back(const float (&x)[NE], float (&d)[NE], int pro) {
    float e_[NE], n;
    feature_row<NE>(x, e_, n, pro & ~kProL2);  // e = elu(x) + 1 (or x), n = |e|
    if (pro & kProL2) {
        const float inv = n > 0.f ? 1.f / n : 0.f;
        float yd = 0.f;
#pragma unroll
        for (int e = 0; e < NE; ++e) yd = fmaf(e_[e] * inv, d[e], yd);
        yd = warp_allsum(yd);
#pragma unroll
        for (int e = 0; e < NE; ++e) d[e] = (d[e] - e_[e] * inv * yd) * inv;
    }
    if (pro & kProElu1) {
#pragma unroll
        for (int e = 0; e < NE; ++e) d[e] = x[e] > 0.f ? d[e] : d[e] * __expf(x[e]);
    }
}

template <int DK, typename TIn>
__global__ void __launch_bounds__(kPBThreads) prologue_grad_kernel(const void *q, const void *k, const float *g,
                                                                   const float *beta, float *dq, float *dk,
                                                                   float *dg, float *dbeta, long rows, int gate,
                                                                   int pro) {
    constexpr int NE = DK / 32;
    const long row = ((long)blockIdx.x * kPBThreads + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    if (pro & (kProElu1 | kProL2)) {
        float x[NE], d[NE];
#pragma unroll
        for (int e = 0; e < NE; ++e) {
            x[e] = ld_in<TIn>(q, (size_t)row * DK + lane + 32 * e);
            d[e] = dq[(size_t)row * DK + lane + 32 * e];
        }
        feature_row_back<NE>(x, d, pro);
#pragma unroll
        for (int e = 0; e < NE; ++e) dq[(size_t)row * DK + lane + 32 * e] = d[e];
#pragma unroll
        for (int e = 0; e < NE; ++e) {
            x[e] = ld_in<TIn>(k, (size_t)row * DK + lane + 32 * e);
            d[e] = dk[(size_t)row * DK + lane + 32 * e];
        }
        feature_row_back<NE>(x, d, pro);
#pragma unroll
        for (int e = 0; e < NE; ++e) dk[(size_t)row * DK + lane + 32 * e] = d[e];
    }
    if (dbeta && (pro & kProBetaSigmoid) && lane == 0) {
        const float s = 1.f / (1.f + __expf(-beta[row]));
        dbeta[row] *= s * (1.f - s);
    }
    if (dg && (pro & kProGNegSoftplus)) {
        if (gate == kGateChannel) {
#pragma unroll
            for (int e = 0; e < NE; ++e) {
                const size_t i = (size_t)row * DK + lane + 32 * e;
                dg[i] *= -1.f / (1.f + __expf(-g[i]));
            }
        } else if (lane == 0) {
            dg[row] *= -1.f / (1.f + __expf(-g[row]));
        }
    }
}

template <int DK, typename TIn>
int launch_map(const void *q, const void *k, const void *v, const float *g, const float *beta, float *qm, float *km,
               float *vf, float *gm, float *bm, long rows, int dv, int gate, int pro, cudaStream_t st) {
    const long blocks = (rows * 32 + kPBThreads - 1) / kPBThreads;
    prologue_map_kernel<DK, TIn><<<(unsigned)blocks, kPBThreads, 0, st>>>(q, k, v, g, beta, qm, km, vf, gm, bm, rows,
                                                                         dv, gate, pro);
    return (int)cudaGetLastError();
}

template <int DK, typename TIn>
int launch_grad(const void *q, const void *k, const float *g, const float *beta, float *dq, float *dk, float *dg,
                float *dbeta, long rows, int gate, int pro, cudaStream_t st) {
    const long blocks = (rows * 32 + kPBThreads - 1) / kPBThreads;
    prologue_grad_kernel<DK, TIn><<<(unsigned)blocks, kPBThreads, 0, st>>>(q, k, g, beta, dq, dk, dg, dbeta, rows,
                                                                          gate, pro);
    return (int)cudaGetLastError();
}

}  // namespace
}  // namespace gdn

// Step 1: the mapped inputs in fp32 (bm / gm null when the mode has no beta /
// gate).  Returns a cudaError_t value.
int gdn_launch_prologue_map(const void *q, const void *k, const void *v, const float *g, const float *beta, float *qm,
                            float *km, float *vf, float *gm, float *bm, long rows, int dk, int dv, int gate,
                            int in_bf16, int pro, cudaStream_t st) {
    using namespace gdn;
    if (rows == 0) return 0;
    if (dk == 128)
        return in_bf16 ? launch_map<128, __nv_bfloat16>(q, k, v, g, beta, qm, km, vf, gm, bm, rows, dv, gate, pro, st)
                       : launch_map<128, float>(q, k, v, g, beta, qm, km, vf, gm, bm, rows, dv, gate, pro, st);
    return in_bf16 ? launch_map<64, __nv_bfloat16>(q, k, v, g, beta, qm, km, vf, gm, bm, rows, dv, gate, pro, st)
                   : launch_map<64, float>(q, k, v, g, beta, qm, km, vf, gm, bm, rows, dv, gate, pro, st);
}

// Step 3: the chain rule back to the raw inputs, in place.
int gdn_launch_prologue_grad(const void *q, const void *k, const float *g, const float *beta, float *dq, float *dk,
                             float *dg, float *dbeta, long rows, int dk_, int gate, int in_bf16, int pro,
                             cudaStream_t st) {
    using namespace gdn;
    if (rows == 0) return 0;
    if (dk_ == 128)
        return in_bf16 ? launch_grad<128, __nv_bfloat16>(q, k, g, beta, dq, dk, dg, dbeta, rows, gate, pro, st)
                       : launch_grad<128, float>(q, k, g, beta, dq, dk, dg, dbeta, rows, gate, pro, st);
    return in_bf16 ? launch_grad<64, __nv_bfloat16>(q, k, g, beta, dq, dk, dg, dbeta, rows, gate, pro, st)
                   : launch_grad<64, float>(q, k, g, beta, dq, dk, dg, dbeta, rows, gate, pro, st);
}
