// Backward pass of the recurrence (gdn_chunk_bwd): gradients of q, k, v, the
// gate, beta and S0 from the upstream gradients of o and S_T.
//
// Reverse mode through the token loop, fp32 throughout ("Linear Attention,
// Visualized", "Update the state": training keeps the state at every chunk
// boundary and recomputes inside the chunk).  One CTA owns one (b,h) head and
// a slice of kSlice = 32 value rows: the rows of the state evolve independently
// in the forward direction and their gradients do too, so the slices of a head
// only meet in the gradients that sum over value rows (dq, dk, the gate, beta),
// which are reduced over the CTA's rows in shared memory and added across
// slices with atomics.  Layout as in the decode kernel: a warp owns kRows = 4
// consecutive rows, lane l holds key channels [l V, l V + V), V = dk / 32.
//
//   phase 1: the forward recurrence from S0, storing the state entering every
//            chunk of kChunkB = 64 tokens into the workspace;
//   phase 2: the chunks in reverse.  A chunk is recomputed forward from its
//            stored state, keeping the state entering each sub-block of kSub =
//            8 tokens in shared memory (each thread keeps only its own
//            entries, so no barrier is needed); each sub-block is recomputed
//            once more with its 8 decayed states S'_t = S_{t-1} Diag(alpha_t) in
//            registers, and the gradient steps back through it:
//              u = beta (v - S' k) (delta) or v;  S_t = S' + u k^T
//              dq_t = S_t^T dO_t;  dS += dO_t q_t^T;  du = dS k_t
//              dk_t = dS^T u;  delta: dbeta_t = du . (v - S' k),
//                   dv_t = beta du, dS' = dS - dv_t k^T, dk_t -= S'^T dv_t;
//              else dv_t = du, dS' = dS
//              dg_t = sum(dS' (.) S') (per key channel for a per-channel gate)
//              dS <- dS' Diag(alpha_t)
// Tokens past T are identity steps (q = k = v = dO = 0, beta = 0, alpha = 1).
#include <string.h>

#include "../../include/gdn.h"
#include "common.cuh"

namespace gdn {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kRows = 4;    // value rows per warp
constexpr int kSlice = 32;  // value rows per CTA
constexpr int kSub = 8;     // tokens per sub-block
constexpr int kChunkB = 64; // tokens per stored state

struct BwdArgs {
    const void *q, *k, *v;
    const float *g, *beta, *S0, *dO, *dST;
    float *dq, *dk, *dv, *dg, *dbeta, *dS0;
    float *ws;  // [BH][nchunks][dv][DK]: the state entering every chunk
    int BH, T, DV, nch;  // DV: value dimension
};

__device__ __forceinline__ float bwd_warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// One token's inputs as this thread sees them (its key channels and its warp's rows).
template <int DK, int UPD, int GATE, typename TIn>
struct BwdTok {
    static constexpr int V = DK / 32;
    float q[V], k[V], al[V], bt, v[kRows], dO[kRows];
    __device__ void load(const BwdArgs &a, long bh, int t, int c0, int i0, bool need_q) {
        if (t >= a.T) {
#pragma unroll
            for (int e = 0; e < V; ++e) {
                q[e] = 0.f;
                k[e] = 0.f;
                al[e] = 1.f;
            }
            bt = 0.f;
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
                v[r] = 0.f;
                dO[r] = 0.f;
            }
            return;
        }
        const long tok = bh * a.T + t;
        const TIn *kp = static_cast<const TIn *>(a.k) + tok * DK + c0;
        const TIn *qp = static_cast<const TIn *>(a.q) + tok * DK + c0;
#pragma unroll
        for (int e = 0; e < V; ++e) {
            k[e] = to_f32(kp[e]);
            q[e] = need_q ? to_f32(qp[e]) : 0.f;
            al[e] = 1.f;
        }
        if (GATE == kGateScalar) {
            const float x = __expf(a.g[tok]);
#pragma unroll
            for (int e = 0; e < V; ++e) al[e] = x;
        } else if (GATE == kGateChannel) {
#pragma unroll
            for (int e = 0; e < V; ++e) al[e] = __expf(a.g[tok * DK + c0 + e]);
        }
        bt = (UPD == kDelta) ? a.beta[tok] : 0.f;
        const TIn *vp = static_cast<const TIn *>(a.v) + tok * a.DV + i0;
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            v[r] = to_f32(vp[r]);
            dO[r] = (need_q && a.dO) ? a.dO[tok * a.DV + i0 + r] : 0.f;
        }
    }
};

// S <- S Diag(alpha); then the write (u = beta (v - S k) or v); returns u and
// r = v - S k (delta) through the arrays.
template <int V, int UPD>
__device__ __forceinline__ void fwd_write(float (&s)[kRows][V], const float *k, const float *v, float bt,
                                          float *u, float *rr) {
    if (UPD == kDelta) {
        float p[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            float x = 0.f;
#pragma unroll
            for (int e = 0; e < V; ++e) x = fmaf(s[r][e], k[e], x);
            p[r] = x;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
            for (int r = 0; r < kRows; ++r) p[r] += __shfl_xor_sync(0xffffffffu, p[r], off);
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            rr[r] = v[r] - p[r];
            u[r] = bt * rr[r];
        }
    } else {
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            rr[r] = 0.f;
            u[r] = v[r];
        }
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
        for (int e = 0; e < V; ++e) s[r][e] = fmaf(u[r], k[e], s[r][e]);
}

template <int DK, int UPD, int GATE, typename TIn>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_kernel(const BwdArgs a) {
    constexpr int V = DK / 32;
    constexpr int NW = kBwdThreads / 32;
    using Tok = BwdTok<DK, UPD, GATE, TIn>;
    extern __shared__ float bsm[];
    float *sub = bsm;                                        // [kSub][kSlice][DK] sub-block entry states
    float *red = sub + kSub * kSlice * DK;                   // [2][NW][3][DK] per-warp partial sums
    float *redb = red + 2 * NW * 3 * DK;                     // [2][NW] beta partials

    const int t_ = threadIdx.x, warp = t_ >> 5, lane = t_ & 31;
    const int nsl = a.DV / kSlice;
    const long bh = blockIdx.x / nsl;
    const int i0 = (blockIdx.x % nsl) * kSlice + warp * kRows;  // first value row of this warp
    const int c0 = lane * V;
    const int T = a.T;
    const int lr = warp * kRows;  // row of this warp inside the slice

    float s[kRows][V];
    // ---------------------------------------------------------------- phase 1
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
        for (int e = 0; e < V; ++e) s[r][e] = a.S0 ? a.S0[((size_t)bh * a.DV + i0 + r) * DK + c0 + e] : 0.f;
    for (int t = 0; t < T; ++t) {
        if (t % kChunkB == 0) {
            float *w = a.ws + (((size_t)bh * a.nch + t / kChunkB) * a.DV + i0) * DK + c0;
#pragma unroll
            for (int r = 0; r < kRows; ++r)
#pragma unroll
                for (int e = 0; e < V; ++e) w[r * DK + e] = s[r][e];
        }
        Tok x;
        x.load(a, bh, t, c0, i0, false);
#pragma unroll
        for (int r = 0; r < kRows; ++r)
#pragma unroll
            for (int e = 0; e < V; ++e) s[r][e] *= x.al[e];
        float u[kRows], rr[kRows];
        fwd_write<V, UPD>(s, x.k, x.v, x.bt, u, rr);
    }

    // ---------------------------------------------------------------- phase 2
    float ds[kRows][V];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
        for (int e = 0; e < V; ++e) ds[r][e] = a.dST ? a.dST[((size_t)bh * a.DV + i0 + r) * DK + c0 + e] : 0.f;
    int par = 0;  // parity of the reduction buffer
    for (int c = a.nch - 1; c >= 0; --c) {
        const int t0 = c * kChunkB;
        const int nsub = (min(T, t0 + kChunkB) - t0 + kSub - 1) / kSub;
        {
            const float *w = a.ws + (((size_t)bh * a.nch + c) * a.DV + i0) * DK + c0;
#pragma unroll
            for (int r = 0; r < kRows; ++r)
#pragma unroll
                for (int e = 0; e < V; ++e) s[r][e] = w[r * DK + e];
        }
        // the state entering each sub-block (own entries only)
        for (int j = 0; j < nsub; ++j) {
            float *sp = sub + ((size_t)j * kSlice + lr) * DK + c0;
#pragma unroll
            for (int r = 0; r < kRows; ++r)
#pragma unroll
                for (int e = 0; e < V; ++e) sp[r * DK + e] = s[r][e];
            for (int tt = 0; tt < kSub; ++tt) {
                Tok x;
                x.load(a, bh, t0 + j * kSub + tt, c0, i0, false);
#pragma unroll
                for (int r = 0; r < kRows; ++r)
#pragma unroll
                    for (int e = 0; e < V; ++e) s[r][e] *= x.al[e];
                float u[kRows], rr[kRows];
                fwd_write<V, UPD>(s, x.k, x.v, x.bt, u, rr);
            }
        }
        for (int j = nsub - 1; j >= 0; --j) {
            // the sub-block's decayed states S'_t in registers
            float Sp[kSub][kRows][V];
            {
                const float *sp = sub + ((size_t)j * kSlice + lr) * DK + c0;
#pragma unroll
                for (int r = 0; r < kRows; ++r)
#pragma unroll
                    for (int e = 0; e < V; ++e) s[r][e] = sp[r * DK + e];
            }
#pragma unroll
            for (int tt = 0; tt < kSub; ++tt) {
                Tok x;
                x.load(a, bh, t0 + j * kSub + tt, c0, i0, false);
#pragma unroll
                for (int r = 0; r < kRows; ++r)
#pragma unroll
                    for (int e = 0; e < V; ++e) {
                        s[r][e] *= x.al[e];
                        Sp[tt][r][e] = s[r][e];
                    }
                float u[kRows], rr[kRows];
                fwd_write<V, UPD>(s, x.k, x.v, x.bt, u, rr);
            }
#pragma unroll
            for (int tt = kSub - 1; tt >= 0; --tt) {
                const int t = t0 + j * kSub + tt;
                Tok x;
                x.load(a, bh, t, c0, i0, true);
                float st[kRows][V], u[kRows], rr[kRows];
#pragma unroll
                for (int r = 0; r < kRows; ++r)
#pragma unroll
                    for (int e = 0; e < V; ++e) st[r][e] = Sp[tt][r][e];
                fwd_write<V, UPD>(st, x.k, x.v, x.bt, u, rr);  // st = S_t
                float dqp[V], dkp[V], dgp[V];
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    float acc = 0.f;
#pragma unroll
                    for (int r = 0; r < kRows; ++r) acc = fmaf(st[r][e], x.dO[r], acc);
                    dqp[e] = acc;
                }
                // dS += dO q^T;  du = dS k
                float du[kRows];
#pragma unroll
                for (int r = 0; r < kRows; ++r) {
                    float acc = 0.f;
#pragma unroll
                    for (int e = 0; e < V; ++e) {
                        ds[r][e] = fmaf(x.dO[r], x.q[e], ds[r][e]);
                        acc = fmaf(ds[r][e], x.k[e], acc);
                    }
                    du[r] = acc;
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                    for (int r = 0; r < kRows; ++r) du[r] += __shfl_xor_sync(0xffffffffu, du[r], off);
                float dvt[kRows], dbp = 0.f;
#pragma unroll
                for (int r = 0; r < kRows; ++r) {
                    dvt[r] = (UPD == kDelta) ? x.bt * du[r] : du[r];
                    if (UPD == kDelta) dbp = fmaf(du[r], rr[r], dbp);
                }
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    float acc = 0.f;
#pragma unroll
                    for (int r = 0; r < kRows; ++r) {
                        acc = fmaf(ds[r][e], u[r], acc);
                        if (UPD == kDelta) acc = fmaf(-Sp[tt][r][e], dvt[r], acc);
                    }
                    dkp[e] = acc;
                }
                // dS' (delta: minus dv k^T), the gate's gradient, then dS <- dS' Diag(alpha)
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    float acc = 0.f;
#pragma unroll
                    for (int r = 0; r < kRows; ++r) {
                        if (UPD == kDelta) ds[r][e] = fmaf(-dvt[r], x.k[e], ds[r][e]);
                        acc = fmaf(ds[r][e], Sp[tt][r][e], acc);
                        ds[r][e] *= x.al[e];
                    }
                    dgp[e] = acc;
                }
                if (t < T) {
                    if (lane == 0) {
                        float *dvp = a.dv + ((size_t)bh * T + t) * a.DV + i0;
#pragma unroll
                        for (int r = 0; r < kRows; ++r) dvp[r] = dvt[r];
                    }
                }
                // per-warp partials, then the CTA's sums over its 32 rows
                float *rp = red + ((size_t)par * NW + warp) * 3 * DK;
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    rp[c0 + e] = dqp[e];
                    rp[DK + c0 + e] = dkp[e];
                    rp[2 * DK + c0 + e] = dgp[e];
                }
                if (lane == 0) redb[par * NW + warp] = dbp;
                __syncthreads();
                if (t < T) {
                    const float *rb = red + (size_t)par * NW * 3 * DK;
                    if (t_ < DK) {
                        float sq = 0.f, sk = 0.f, sg = 0.f;
#pragma unroll
                        for (int w = 0; w < NW; ++w) {
                            sq += rb[w * 3 * DK + t_];
                            sk += rb[w * 3 * DK + DK + t_];
                            sg += rb[w * 3 * DK + 2 * DK + t_];
                        }
                        const size_t o = ((size_t)bh * T + t) * DK + t_;
                        atomicAdd(a.dq + o, sq);
                        atomicAdd(a.dk + o, sk);
                        if (GATE == kGateChannel) {
                            atomicAdd(a.dg + o, sg);
                        } else if (GATE == kGateScalar) {
                            sg = bwd_warp_sum(sg);
                            if ((t_ & 31) == 0) atomicAdd(a.dg + (size_t)bh * T + t, sg);
                        }
                    } else if (UPD == kDelta && t_ == DK) {
                        float sb = 0.f;
#pragma unroll
                        for (int w = 0; w < NW; ++w) sb += redb[par * NW + w];
                        atomicAdd(a.dbeta + (size_t)bh * T + t, sb);
                    }
                }
                par ^= 1;
            }
        }
    }
    if (a.dS0) {
#pragma unroll
        for (int r = 0; r < kRows; ++r)
#pragma unroll
            for (int e = 0; e < V; ++e) a.dS0[((size_t)bh * a.DV + i0 + r) * DK + c0 + e] = ds[r][e];
    }
}

template <int DK, int UPD, int GATE, typename TIn>
int launch_bwd(const BwdArgs &a, cudaStream_t st) {
    constexpr int NW = kBwdThreads / 32;
    const size_t smem = ((size_t)kSub * kSlice * DK + 2 * NW * 3 * DK + 2 * NW) * sizeof(float);
    auto kern = bwd_kernel<DK, UPD, GATE, TIn>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return (int)e;
    const long grid = (long)a.BH * (a.DV / kSlice);
    kern<<<(unsigned)grid, kBwdThreads, smem, st>>>(a);
    return (int)cudaGetLastError();
}

template <int DK, typename TIn>
int launch_bwd_modes(const BwdArgs &a, int update, int gate, cudaStream_t st) {
    if (update == kAdditive) return launch_bwd<DK, kAdditive, kGateNone, TIn>(a, st);
    if (update == kDecay)
        return gate == kGateScalar ? launch_bwd<DK, kDecay, kGateScalar, TIn>(a, st)
                                   : launch_bwd<DK, kDecay, kGateChannel, TIn>(a, st);
    if (gate == kGateNone) return launch_bwd<DK, kDelta, kGateNone, TIn>(a, st);
    return gate == kGateScalar ? launch_bwd<DK, kDelta, kGateScalar, TIn>(a, st)
                               : launch_bwd<DK, kDelta, kGateChannel, TIn>(a, st);
}

}  // namespace
}  // namespace gdn

// Launcher for api.cu: zeroes the gradients that are sums over value slices,
// then runs the kernel.  Returns a cudaError_t value.
int gdn_launch_bwd(const void *q, const void *k, const void *v, const float *g, const float *beta, const float *S0,
                   const float *dO, const float *dST, float *dq, float *dk, float *dv, float *dg, float *dbeta,
                   float *dS0, float *ws, int BH, int T, int dk_, int dv_, int update, int gate, int in_bf16,
                   cudaStream_t st) {
    using namespace gdn;
    const size_t ntok = (size_t)BH * T;
    cudaError_t e = cudaMemsetAsync(dq, 0, ntok * dk_ * sizeof(float), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dk, 0, ntok * dk_ * sizeof(float), st);
    if (e == cudaSuccess && dg) e = cudaMemsetAsync(dg, 0, ntok * (gate == kGateChannel ? dk_ : 1) * sizeof(float), st);
    if (e == cudaSuccess && dbeta) e = cudaMemsetAsync(dbeta, 0, ntok * sizeof(float), st);
    if (e != cudaSuccess) return (int)e;
    BwdArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S0 = S0; a.dO = dO; a.dST = dST;
    a.dq = dq; a.dk = dk; a.dv = dv; a.dg = dg; a.dbeta = dbeta; a.dS0 = dS0; a.ws = ws;
    a.BH = BH; a.T = T; a.DV = dv_;
    a.nch = (T + kChunkB - 1) / kChunkB;
    if (dk_ == 128)
        return in_bf16 ? launch_bwd_modes<128, __nv_bfloat16>(a, update, gate, st)
                       : launch_bwd_modes<128, float>(a, update, gate, st);
    return in_bf16 ? launch_bwd_modes<64, __nv_bfloat16>(a, update, gate, st)
                   : launch_bwd_modes<64, float>(a, update, gate, st);
}
