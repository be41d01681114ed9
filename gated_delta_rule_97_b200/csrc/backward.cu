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
//            chunk of kChunkB = 64 tokens into the workspace (skipped when the
//            tensor-core forward saved those states already);
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
// The inputs of every sub-block are staged in shared memory (coalesced loads of
// the next sub-block issued while the current one is processed), so the token
// steps read shared memory only.
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
    int skip_fwd;        // ws already holds the states (a forward wrote them): no phase 1
};

// Warp sums of four per-lane partials x[0..3] (one per row of the warp), every
// sum returned to every lane: a transposing butterfly (6 shuffles, after which
// lane l holds the sum of row (l >> 3) & 3), then one broadcast per row.
__device__ __forceinline__ void warp_sum_rows(float (&x)[kRows]) {
    static_assert(kRows == 4, "four rows per warp");
    const int lane = threadIdx.x & 31;
    const bool b4 = lane & 16, b3 = lane & 8;
    const float a0 = (b4 ? x[2] : x[0]) + __shfl_xor_sync(0xffffffffu, b4 ? x[0] : x[2], 16);
    const float a1 = (b4 ? x[3] : x[1]) + __shfl_xor_sync(0xffffffffu, b4 ? x[1] : x[3], 16);
    float b = (b3 ? a1 : a0) + __shfl_xor_sync(0xffffffffu, b3 ? a0 : a1, 8);
    b += __shfl_xor_sync(0xffffffffu, b, 4);
    b += __shfl_xor_sync(0xffffffffu, b, 2);
    b += __shfl_xor_sync(0xffffffffu, b, 1);
#pragma unroll
    for (int r = 0; r < kRows; ++r) x[r] = __shfl_sync(0xffffffffu, b, ((r >> 1) << 4) | ((r & 1) << 3));
}

__device__ __forceinline__ float bwd_warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// The inputs of one sub-block of kSub tokens, staged in shared memory as fp32:
// key and query channels, alpha = exp(g) (per channel, or per token), this
// CTA's kSlice value rows of v and dO, and beta.  Tokens past T read as the
// identity step.  With kSub * kSlice == kBwdThreads, thread i stages value row
// i % kSlice of token i / kSlice, and a contiguous run of DK / 32 channels.
template <int DK, int GATE>
struct StageLayout {
    static constexpr int NA = (GATE == kGateChannel) ? kSub * DK : kSub;
    static constexpr int K = 0, Q = kSub * DK, AL = 2 * kSub * DK, VV = AL + NA, DO = VV + kSub * kSlice,
                         BT = DO + kSub * kSlice, FLOATS = BT + kSub;
};

template <int DK, int UPD, int GATE, typename TIn>
struct StageRegs {
    using SL = StageLayout<DK, GATE>;
    static constexpr int EQ = kSub * DK / kBwdThreads;
    float k[EQ], q[EQ], al[EQ], v, dO, bt;
    __device__ void load(const BwdArgs &a, long bh, int tb, int rslice, int t_, bool need_q) {
        const int T = a.T;
        const int e0 = t_ * EQ, t = tb + e0 / DK, ch = e0 % DK;
#pragma unroll
        for (int e = 0; e < EQ; ++e) {
            k[e] = 0.f;
            q[e] = 0.f;
            al[e] = 1.f;
        }
        if (t < T) {
            const size_t off = ((size_t)bh * T + t) * DK + ch;
            const TIn *kp = static_cast<const TIn *>(a.k) + off;
            const TIn *qp = static_cast<const TIn *>(a.q) + off;
#pragma unroll
            for (int e = 0; e < EQ; ++e) {
                k[e] = to_f32(kp[e]);
                if (need_q) q[e] = to_f32(qp[e]);
                if (GATE == kGateChannel) al[e] = __expf(a.g[off + e]);
            }
        }
        const int tv = tb + t_ / kSlice, row = rslice + t_ % kSlice;
        v = 0.f;
        dO = 0.f;
        if (tv < T) {
            const size_t ov = ((size_t)bh * T + tv) * a.DV + row;
            v = to_f32(static_cast<const TIn *>(a.v)[ov]);
            if (need_q && a.dO) dO = a.dO[ov];
        }
        bt = 0.f;
        if (t_ < kSub && tb + t_ < T) {
            const size_t ot = (size_t)bh * T + tb + t_;
            if (UPD == kDelta) bt = a.beta[ot];
            if (GATE == kGateScalar) al[0] = __expf(a.g[ot]);
        }
    }
    __device__ void store(float *st, int t_) const {
        const int e0 = t_ * EQ;
#pragma unroll
        for (int e = 0; e < EQ; ++e) {
            st[SL::K + e0 + e] = k[e];
            st[SL::Q + e0 + e] = q[e];
            if (GATE == kGateChannel) st[SL::AL + e0 + e] = al[e];
        }
        st[SL::VV + t_] = v;
        st[SL::DO + t_] = dO;
        if (t_ < kSub) {
            st[SL::BT + t_] = bt;
            if (GATE != kGateChannel) st[SL::AL + t_] = (GATE == kGateScalar) ? al[0] : 1.f;
        }
    }
};

// One token's inputs as this thread reads them from a staged sub-block.
template <int DK, int UPD, int GATE>
struct BwdTok {
    using SL = StageLayout<DK, GATE>;
    static constexpr int V = DK / 32;
    float q[V], k[V], al[V], bt, v[kRows], dO[kRows];
    __device__ void read(const float *st, int tt, int c0, int lr, bool need_q) {
#pragma unroll
        for (int e = 0; e < V; ++e) {
            k[e] = st[SL::K + tt * DK + c0 + e];
            q[e] = need_q ? st[SL::Q + tt * DK + c0 + e] : 0.f;
            al[e] = (GATE == kGateChannel) ? st[SL::AL + tt * DK + c0 + e] : st[SL::AL + tt];
        }
        bt = st[SL::BT + tt];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            v[r] = st[SL::VV + tt * kSlice + lr + r];
            dO[r] = need_q ? st[SL::DO + tt * kSlice + lr + r] : 0.f;
        }
    }
};

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
        warp_sum_rows(p);
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

// The kernel walks a fixed sequence of sub-block visits: phase 1 visits the
// sub-blocks of the sequence in order; phase 2 visits the chunks from the last,
// each chunk's sub-blocks forward (recompute) and then backward.  Every visit's
// inputs are staged in one of two shared-memory buffers; the next visit's are
// loaded into registers while the current one is processed and stored into the
// other buffer at its end.
struct Visit {
    int tb;     // first token of the sub-block
    int phase;  // 1: forward of phase 1; 2: forward recompute of phase 2; 3: backward
    int j;      // sub-block index inside its chunk
    int c;      // chunk
};

__device__ __forceinline__ Visit visit_at(int n, int T, int nch) {
    const int ns = (T + kSub - 1) / kSub;
    Visit v;
    if (n < ns) {
        v.tb = n * kSub;
        v.phase = 1;
        v.j = n % (kChunkB / kSub);
        v.c = n / (kChunkB / kSub);
        return v;
    }
    n -= ns;
    const int last = nch - 1;
    const int nsub_last = (T - last * kChunkB + kSub - 1) / kSub;
    int c, i, nsub;
    if (n < 2 * nsub_last) {
        c = last;
        i = n;
        nsub = nsub_last;
    } else {
        const int m = n - 2 * nsub_last;
        nsub = kChunkB / kSub;
        c = last - 1 - m / (2 * nsub);
        i = m % (2 * nsub);
    }
    v.c = c;
    v.phase = i < nsub ? 2 : 3;
    v.j = i < nsub ? i : 2 * nsub - 1 - i;
    v.tb = c * kChunkB + v.j * kSub;
    return v;
}

template <int DK, int UPD, int GATE, typename TIn>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_kernel(const BwdArgs a) {
    constexpr int V = DK / 32;
    constexpr int NW = kBwdThreads / 32;
    using SL = StageLayout<DK, GATE>;
    using Tok = BwdTok<DK, UPD, GATE>;
    static_assert(kSub * kSlice == kBwdThreads, "one staged (token, value row) per thread");
    extern __shared__ float bsm[];
    float *sub = bsm;                          // [kSub][kSlice][DK] sub-block entry states
    float *red = sub + kSub * kSlice * DK;     // [2][NW][3][DK] per-warp partial sums
    float *redb = red + 2 * NW * 3 * DK;       // [2][NW] beta partials
    float *stg = redb + 2 * NW;                // [2][SL::FLOATS] staged inputs

    const int t_ = threadIdx.x, warp = t_ >> 5, lane = t_ & 31;
    const int nsl = a.DV / kSlice;
    const long bh = blockIdx.x / nsl;
    const int rslice = (blockIdx.x % nsl) * kSlice;
    const int i0 = rslice + warp * kRows;  // first value row of this warp
    const int c0 = lane * V;
    const int T = a.T;
    const int lr = warp * kRows;  // row of this warp inside the slice
    const int ns = (T + kSub - 1) / kSub;
    const int last = a.nch - 1;
    const int nvis = ns + 2 * ((T - last * kChunkB + kSub - 1) / kSub) + last * 2 * (kChunkB / kSub);
    const int n0 = a.skip_fwd ? ns : 0;  // first visit

    float s[kRows][V], ds[kRows][V];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
        for (int e = 0; e < V; ++e) {
            s[r][e] = a.S0 ? a.S0[((size_t)bh * a.DV + i0 + r) * DK + c0 + e] : 0.f;
            ds[r][e] = a.dST ? a.dST[((size_t)bh * a.DV + i0 + r) * DK + c0 + e] : 0.f;
        }
    StageRegs<DK, UPD, GATE, TIn> R;
    {
        const Visit v0 = visit_at(n0, T, a.nch);
        R.load(a, bh, v0.tb, rslice, t_, v0.phase != 1);
        R.store(stg, t_);
    }
    __syncthreads();
    int par = 0;  // parity of the reduction buffer
    for (int n = n0; n < nvis; ++n) {
        const Visit vi = visit_at(n, T, a.nch);
        const float *st = stg + ((n - n0) & 1) * SL::FLOATS;
        if (n + 1 < nvis) {
            const Visit vn = visit_at(n + 1, T, a.nch);
            R.load(a, bh, vn.tb, rslice, t_, vn.phase != 1);
        }
        if (vi.phase == 1) {
            // forward; the state entering every chunk goes to the workspace
            if (vi.j == 0) {
                float *w = a.ws + (((size_t)bh * a.nch + vi.c) * a.DV + i0) * DK + c0;
#pragma unroll
                for (int r = 0; r < kRows; ++r)
#pragma unroll
                    for (int e = 0; e < V; ++e) w[r * DK + e] = s[r][e];
            }
            for (int tt = 0; tt < kSub; ++tt) {
                Tok x;
                x.read(st, tt, c0, lr, false);
#pragma unroll
                for (int r = 0; r < kRows; ++r)
#pragma unroll
                    for (int e = 0; e < V; ++e) s[r][e] *= x.al[e];
                float u[kRows], rr[kRows];
                fwd_write<V, UPD>(s, x.k, x.v, x.bt, u, rr);
            }
        } else if (vi.phase == 2) {
            // recompute forward from the chunk's stored state, keeping each sub-block's entry state
            if (vi.j == 0) {
                const float *w = a.ws + (((size_t)bh * a.nch + vi.c) * a.DV + i0) * DK + c0;
#pragma unroll
                for (int r = 0; r < kRows; ++r)
#pragma unroll
                    for (int e = 0; e < V; ++e) s[r][e] = w[r * DK + e];
            }
            float *sp = sub + ((size_t)vi.j * kSlice + lr) * DK + c0;
#pragma unroll
            for (int r = 0; r < kRows; ++r)
#pragma unroll
                for (int e = 0; e < V; ++e) sp[r * DK + e] = s[r][e];
            for (int tt = 0; tt < kSub; ++tt) {
                Tok x;
                x.read(st, tt, c0, lr, false);
#pragma unroll
                for (int r = 0; r < kRows; ++r)
#pragma unroll
                    for (int e = 0; e < V; ++e) s[r][e] *= x.al[e];
                float u[kRows], rr[kRows];
                fwd_write<V, UPD>(s, x.k, x.v, x.bt, u, rr);
            }
        } else {
            // the sub-block's decayed states S'_t in registers, then back through it
            float Sp[kSub][kRows][V];
            {
                const float *sp = sub + ((size_t)vi.j * kSlice + lr) * DK + c0;
#pragma unroll
                for (int r = 0; r < kRows; ++r)
#pragma unroll
                    for (int e = 0; e < V; ++e) s[r][e] = sp[r * DK + e];
            }
#pragma unroll
            for (int tt = 0; tt < kSub; ++tt) {
                Tok x;
                x.read(st, tt, c0, lr, false);
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
                const int t = vi.tb + tt;
                Tok x;
                x.read(st, tt, c0, lr, true);
                float stt[kRows][V], u[kRows], rr[kRows];
#pragma unroll
                for (int r = 0; r < kRows; ++r)
#pragma unroll
                    for (int e = 0; e < V; ++e) stt[r][e] = Sp[tt][r][e];
                fwd_write<V, UPD>(stt, x.k, x.v, x.bt, u, rr);  // stt = S_t
                float dqp[V], dkp[V], dgp[V];
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    float acc = 0.f;
#pragma unroll
                    for (int r = 0; r < kRows; ++r) acc = fmaf(stt[r][e], x.dO[r], acc);
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
                warp_sum_rows(du);
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
                if (t < T && lane == 0) {
                    float *dvp = a.dv + ((size_t)bh * T + t) * a.DV + i0;
#pragma unroll
                    for (int r = 0; r < kRows; ++r) dvp[r] = dvt[r];
                }
                // per-warp partials, then the CTA's sums over its kSlice rows
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
        // the next visit's inputs into the other buffer (its last readers passed the
        // barrier that ended the previous visit)
        if (n + 1 < nvis) R.store(stg + ((n + 1 - n0) & 1) * SL::FLOATS, t_);
        __syncthreads();
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
    const size_t smem =
        ((size_t)kSub * kSlice * DK + 2 * NW * 3 * DK + 2 * NW + 2 * StageLayout<DK, GATE>::FLOATS) * sizeof(float);
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
                   int skip_fwd, cudaStream_t st) {
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
    a.skip_fwd = skip_fwd;
    if (dk_ == 128)
        return in_bf16 ? launch_bwd_modes<128, __nv_bfloat16>(a, update, gate, st)
                       : launch_bwd_modes<128, float>(a, update, gate, st);
    return in_bf16 ? launch_bwd_modes<64, __nv_bfloat16>(a, update, gate, st)
                   : launch_bwd_modes<64, float>(a, update, gate, st);
}
