// Chunkwise backward of the recurrence on tensor cores (gdn_chunk_bwd_tc).
//
// The forward's chunk algebra ("Linear Attention, Visualized": "The triangular
// correction system", "Optional: Use UT...", "Correct the incoming state",
// "Update the state"), per chunk r of C = 64 tokens with S = S_r the state
// entering it, G the in-chunk prefix of the log-gate, b = e^G, b_C = e^{G_63},
// Gamma[l,m] = e^{G_l - G_m} (m <= l):
//   Qb = diag(b) q,  Kb = diag(b) k,  Kc = diag(b_C / b) k
//   L  = strict-lower(diag(beta) (k k^T (.) Gamma)),   T = (I + L)^-1
//   W  = T diag(beta) Kb,  U = T diag(beta) v,  Z = U - W S^T      (delta rule)
//   Z  = v                                                         (otherwise)
//   A  = lower-incl(q k^T (.) Gamma),  O = Qb S^T + A Z,  S' = b_C S + Z^T Kc
// is differentiated by reverse mode at chunk granularity.  With dSn the
// gradient of S' and dO that of O:
//   dZ  = A^T dO + Kc dSn^T,        dKc = Z dSn,    dA = dO Z^T,    dQb = dO S
//   dW  = -dZ S,  dT = dZ (diag(beta) v)^T + dW (diag(beta) Kb)^T,
//   dL  = strict-lower(-T^T dT T^T),  dv = diag(beta) T^T dZ (delta) or dZ
//   dS_r = b_C dSn + dO^T Qb - dZ^T W = b_C dSn - (dSn Kc^T) W + dO^T (Qb - A W)
// and the gate's gradient collects every e^{...} factor's share, summed back
// over the prefix (dg_s = sum_{l >= s} dG_l).
//
// Three kernels:
//   prep  (one CTA per chunk and head, all in parallel): T by blocked forward
//         substitution, A, P (.) Gamma, W, Q~ = Qb - A W, Kc, b_C -> workspace
//         (W, Q~, Kc rounded to tf32 there, the chain's operands as stored);
//   chain (one CTA per head, chunks last to first): the only sequential part,
//         dS_r from dS_{r+1} with three products per chunk, storing dS_{r+1}
//         for every chunk; each warp owns 16 value rows of dS in mma
//         accumulators and feeds them back as A operands (the contraction
//         index is permuted inside each 8-wide block so accumulator and
//         operand fragments coincide);
//   local (one CTA per chunk and head, all in parallel): every chunk-local
//         gradient from the saved S_r, the stored dSn and the prep's tiles;
//         value rows go through in slices of 32 (the next slice's S and dSn
//         copied while one is processed), the sums over value rows (dKc, dQb,
//         dW, dA, dT) stay in registers across the slices.
// Every product is a warp-level tf32 tensor-core MMA (m16n8k8, fp32
// accumulation) on fp32 tiles in shared memory; an operand tile is rounded to
// tf32 (nearest) once, where it is written, so the MMA loops of the chain and
// local kernels convert nothing.  dq, dk, dv, dg, dbeta are written once per
// token and the CTA reductions run in a fixed order: no atomics, deterministic.
#include <stddef.h>

#include "../../include/gdn.h"
#include "common.cuh"
#include "sm100.cuh"
#include "tc_util.cuh"

namespace gdn {
namespace {

using tcu::f2tf32;
using tcu::mma_tf32_16x8x8;

constexpr int C = kChunk;   // tokens per chunk
constexpr int DKB = 128;    // key dimension served
constexpr int LK = DKB + 4; // row stride (floats) of [64][128] tiles
constexpr int LKC = DKB + 8; // row stride of the chain's Kc tile (8-byte fragment loads)
constexpr int LC = C + 4;   // row stride of [64][64] tiles
constexpr int kThreads = 256;

struct TcBwdArgs {
    const void *q, *k, *v;
    const float *g, *beta, *states, *dO, *dST;
    float *dq, *dk, *dv, *dg, *dbeta, *dS0;
    // workspace, [BH][nch][...]: T, A, P (.) Gamma [64][64]; W, Kc, Q~ [64][128];
    // dSn [dv][128] (the gradient of the state leaving the chunk); b_C
    float *Tm, *Am, *PGm, *Wm, *Kcm, *Qtm, *dSn, *bC;
    int BH, T, nch;
};

// ---------------------------------------------------------------- warp MMA
// acc[j] (16 x 8 tile j of a 16 x 8NT block) += sum_k A(m,k) B(k, 8j + n) over
// k in [k_begin, k_end) (multiples of 8), with A(m,k) = A[m SAM + k SAK] and
// B(k,n) = B[k SBK + n SBN] (pointers at the block's first row / column), B
// optionally scaled by sck[k].  Fragments (g = lane / 4, t = lane % 4):
// acc[j] = {(g, 8j+2t), (g, 8j+2t+1), (g+8, 8j+2t), (g+8, 8j+2t+1)}.
// PERM: the k slots t and t + 4 of each 8-wide step take k = k0 + 2t and
// k0 + 2t + 1 (a permutation of the summation, the same for A and B): with
// row strides of 4 (mod 32) words, B rows k0 + 2t then fall on distinct banks,
// and so do the rows of a transposed A.
// CVT false: both operands are stored rounded to tf32 already (no conversion).
template <int NT, int SAM, int SAK, int SBK, int SBN, bool SCK = false, bool PERM = false, bool CVT = true>
__device__ __forceinline__ void wmma(float (&acc)[NT][4], const float *A, const float *B, int k_begin, int k_end,
                                     const float *sck = nullptr) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int ka = PERM ? 2 * t : t, kb = PERM ? 2 * t + 1 : t + 4;
    auto op = [](float x) { return CVT ? f2tf32(x) : __float_as_uint(x); };
    for (int k0 = k_begin; k0 < k_end; k0 += 8) {
        uint32_t a[4];
        a[0] = op(A[g * SAM + (k0 + ka) * SAK]);
        a[1] = op(A[(g + 8) * SAM + (k0 + ka) * SAK]);
        a[2] = op(A[g * SAM + (k0 + kb) * SAK]);
        a[3] = op(A[(g + 8) * SAM + (k0 + kb) * SAK]);
        float s0 = 1.f, s1 = 1.f;
        if (SCK) {
            s0 = sck[k0 + ka];
            s1 = sck[k0 + kb];
        }
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            float b0 = B[(k0 + ka) * SBK + (8 * j + g) * SBN], b1 = B[(k0 + kb) * SBK + (8 * j + g) * SBN];
            if (SCK) {
                b0 *= s0;
                b1 *= s1;
            }
            const uint32_t b[2] = {(SCK || CVT) ? f2tf32(b0) : __float_as_uint(b0),
                                   (SCK || CVT) ? f2tf32(b1) : __float_as_uint(b1)};
            mma_tf32_16x8x8(acc[j], a, b);
        }
    }
}

// x rounded to tf32 (nearest, ties away), kept as an fp32 value: an MMA operand
// stored this way needs no conversion when it is read.
__device__ __forceinline__ float tf32r(float x) { return __uint_as_float(f2tf32(x)); }

template <int NT>
__device__ __forceinline__ void zero(float (&a)[NT][4]) {
#pragma unroll
    for (int j = 0; j < NT; ++j) a[j][0] = a[j][1] = a[j][2] = a[j][3] = 0.f;
}

// Accumulator block -> shared tile (row stride LD), times `s`; RND: rounded to
// tf32 (a later MMA operand).
template <int NT, int LD, bool RND = false>
__device__ __forceinline__ void store_frag(float *dst, const float (&a)[NT][4], float s = 1.f) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    auto f = [&](float x) { return RND ? tf32r(s * x) : s * x; };
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        *reinterpret_cast<float2 *>(dst + g * LD + 8 * j + 2 * t) = make_float2(f(a[j][0]), f(a[j][1]));
        *reinterpret_cast<float2 *>(dst + (g + 8) * LD + 8 * j + 2 * t) = make_float2(f(a[j][2]), f(a[j][3]));
    }
}

// Accumulator block -> global rows (row stride ld floats), rows >= nrow skipped;
// RND: rounded to tf32.
template <int NT, bool RND = false>
__device__ __forceinline__ void store_frag_global(float *dst, size_t ld, const float (&a)[NT][4], int row0, int nrow) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    auto f = [](float x) { return RND ? tf32r(x) : x; };
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        if (row0 + g < nrow)
            *reinterpret_cast<float2 *>(dst + (size_t)(row0 + g) * ld + 8 * j + 2 * t) =
                make_float2(f(a[j][0]), f(a[j][1]));
        if (row0 + g + 8 < nrow)
            *reinterpret_cast<float2 *>(dst + (size_t)(row0 + g + 8) * ld + 8 * j + 2 * t) =
                make_float2(f(a[j][2]), f(a[j][3]));
    }
}

// ---------------------------------------------------------------- tile I/O
// Rows [0, 64) x W columns of an fp32 tile (global row stride sw floats) into
// shared memory (row stride LD); rows >= nvalid (or a null source) are zero.
template <int W, int LD, int NTH>
__device__ __forceinline__ void load_f32(float *dst, const float *src, size_t sw, int nvalid, int rows = C) {
    constexpr int V = W / 4;
    for (int i = threadIdx.x; i < rows * V; i += NTH) {
        const int r = i / V, c = (i % V) * 4;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (src && r < nvalid) x = __ldg(reinterpret_cast<const float4 *>(src + (size_t)r * sw + c));
        *reinterpret_cast<float4 *>(dst + r * LD + c) = x;
    }
}

// The same for an input tensor of type TIn (bf16 or fp32), converted to fp32.
template <typename TIn, int W, int LD, int NTH>
__device__ __forceinline__ void load_in(float *dst, const void *src, size_t sw, int nvalid) {
    if constexpr (sizeof(TIn) == 4) {
        // fp32 inputs rounded to tf32 as staged (MMA operands); bf16 values are tf32 already
        const float *s = static_cast<const float *>(src);
        constexpr int V = W / 4;
        for (int i = threadIdx.x; i < C * V; i += NTH) {
            const int r = i / V, c = (i % V) * 4;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < nvalid) x = __ldg(reinterpret_cast<const float4 *>(s + (size_t)r * sw + c));
            *reinterpret_cast<float4 *>(dst + r * LD + c) = make_float4(tf32r(x.x), tf32r(x.y), tf32r(x.z), tf32r(x.w));
        }
    } else {
        constexpr int V = W / 8, N = (C * V + NTH - 1) / NTH;
        const __nv_bfloat16 *s = static_cast<const __nv_bfloat16 *>(src);
        uint4 u[N];
#pragma unroll
        for (int n = 0; n < N; ++n) {  // every load in flight before the first store
            const int i = threadIdx.x + n * NTH, r = i / V, c = (i % V) * 8;
            u[n] = make_uint4(0u, 0u, 0u, 0u);
            if (i < C * V && r < nvalid) u[n] = __ldg(reinterpret_cast<const uint4 *>(s + (size_t)r * sw + c));
        }
#pragma unroll
        for (int n = 0; n < N; ++n) {
            const int i = threadIdx.x + n * NTH, r = i / V, c = (i % V) * 8;
            if (i >= C * V) break;
            float f[8];
            tcu::unpack_bf16x8(u[n], f);
            *reinterpret_cast<float4 *>(dst + r * LD + c) = make_float4(f[0], f[1], f[2], f[3]);
            *reinterpret_cast<float4 *>(dst + r * LD + c + 4) = make_float4(f[4], f[5], f[6], f[7]);
        }
    }
}

// Shared tile (row stride LD) -> dense global [rows][W]; RND: rounded to tf32.
template <int W, int LD, bool RND = false>
__device__ __forceinline__ void store_tile(float *dst, const float *src, int rows = C) {
    constexpr int V = W / 4;
    for (int i = threadIdx.x; i < rows * V; i += kThreads) {
        const int r = i / V, c = (i % V) * 4;
        float4 x = *reinterpret_cast<const float4 *>(src + r * LD + c);
        if (RND) x = make_float4(tf32r(x.x), tf32r(x.y), tf32r(x.z), tf32r(x.w));
        *reinterpret_cast<float4 *>(dst + (size_t)r * W + c) = x;
    }
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sm100::smem_u32(dst)), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Bulk prefetch of `bytes` (a multiple of 16, 16-byte aligned) into L2.
__device__ __forceinline__ void l2_prefetch(const void *p, uint32_t bytes) {
    if (p && bytes) asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// [ROWS][W] fp32 rows of global memory into a shared tile, asynchronously; rows
// >= nvalid (or a null source) are zero-filled.
template <int W, int LD, int NTH, int ROWS = C>
__device__ __forceinline__ void cp_tile(float *dst, const float *src, size_t sw, int nvalid, const void *dummy) {
    constexpr int V = W / 4;
#pragma unroll 4
    for (int i = threadIdx.x; i < ROWS * V; i += NTH) {
        const int r = i / V, c = (i % V) * 4;
        const bool ok = src && r < nvalid;
        cp_async16(dst + r * LD + c, ok ? static_cast<const void *>(src + (size_t)r * sw + c) : dummy, ok);
    }
}

// In-chunk prefix of the log-gate (one warp; lane l holds tokens 2l, 2l+1):
// G, b = e^G, e^{G_63 - G}.  Tokens past the sequence contribute g = 0.
template <bool GATED>
__device__ __forceinline__ void gate_prefix(const float *g, long tok0, int nv, float *Gs, float *bs, float *es) {
    const int lane = threadIdx.x & 31;
    float x0 = 0.f, x1 = 0.f;
    if (GATED) {
        if (2 * lane < nv) x0 = g[tok0 + 2 * lane];
        if (2 * lane + 1 < nv) x1 = g[tok0 + 2 * lane + 1];
    }
    float s = x0 + x1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, s, off);
        if (lane >= off) s += y;
    }
    const float G1 = s, G0 = s - x1, GC = __shfl_sync(0xffffffffu, s, 31);
    Gs[2 * lane] = G0;
    Gs[2 * lane + 1] = G1;
    bs[2 * lane] = GATED ? expf(G0) : 1.f;
    bs[2 * lane + 1] = GATED ? expf(G1) : 1.f;
    es[2 * lane] = GATED ? expf(GC - G0) : 1.f;
    es[2 * lane + 1] = GATED ? expf(GC - G1) : 1.f;
}

// ------------------------------------------------------------------ prep
// Four large tiles, reused: q then W; k; P (.) Gamma then A; T.  L = diag(beta)
// P (.) Gamma is taken from P (.) Gamma when read.  107 KB: two CTAs per SM.
struct PrepSmem {
    static constexpr int qs = 0, ks = qs + C * LK, PGs = ks + C * LK, Ts = PGs + C * LC, Rs = Ts + C * LC,
                         Gs = Rs + 16 * 52, bs = Gs + C, es = bs + C, betas = es + C, bsc = betas + C,
                         floats = bsc + C;
};

template <bool DELTA, bool GATED, typename TIn>
__global__ void __launch_bounds__(kThreads, 2) bwdtc_prep_kernel(TcBwdArgs p) {
    extern __shared__ float4 smem4[];
    float *sm = reinterpret_cast<float *>(smem4);
    using S = PrepSmem;
    float *qs = sm + S::qs, *ks = sm + S::ks, *PGs = sm + S::PGs, *Ts = sm + S::Ts, *Rs = sm + S::Rs,
          *Gs = sm + S::Gs, *bs = sm + S::bs, *es = sm + S::es, *betas = sm + S::betas, *bsc = sm + S::bsc;
    float *Ws = qs, *As = PGs;  // W over q once A is formed; A over P (.) Gamma after the solve
    const int r = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const long tok0 = (long)bh * p.T + (long)r * C;
    const int nv = min(C, p.T - r * C);
    const size_t cidx = (size_t)bh * p.nch + r;
    const TIn *qg = static_cast<const TIn *>(p.q) + tok0 * DKB;

    load_in<TIn, DKB, LK, kThreads>(qs, qg, DKB, nv);
    load_in<TIn, DKB, LK, kThreads>(ks, static_cast<const char *>(p.k) + tok0 * DKB * sizeof(TIn), DKB, nv);
    if (tid < C) betas[tid] = (DELTA && tid < nv) ? p.beta[tok0 + tid] : 0.f;
    if (DELTA)
        for (int i = tid; i < C * LC; i += kThreads) Ts[i] = 0.f;
    if (warp == 0) gate_prefix<GATED>(p.g, tok0, nv, Gs, bs, es);
    __syncthreads();
    if (tid < C) bsc[tid] = betas[tid] * bs[tid];
    const int mt = warp & 3, nb32 = (warp >> 2) * 32, nb64 = (warp >> 2) * 64;
    auto gamma = [&](int l, int m) { return m <= l ? (GATED ? expf(Gs[l] - Gs[m]) : 1.f) : 0.f; };

    if (DELTA) {
        // P (.) Gamma, strict lower
        {
            float ap[4][4];
            zero(ap);
            wmma<4, LK, 1, 1, LK, false, false, false>(ap, ks + 16 * mt * LK, ks + nb32 * LK, 0, DKB);
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int l = 16 * mt + g + 8 * (e >> 1), m = nb32 + 8 * j + 2 * t + (e & 1);
                    PGs[l * LC + m] = m < l ? ap[j][e] * gamma(l, m) : 0.f;
                }
        }
        __syncthreads();
        store_tile<C, LC>(p.PGm + cidx * C * C, PGs);
        // T = (I + L)^-1, L = diag(beta) P (.) Gamma: the four 16 x 16 diagonal blocks
        // by forward substitution (lane c of warp I solves column c of block I), then
        // block rows 1..3: T_IJ = -T_II sum_K L_IK T_KJ
        if (warp < 4 && lane < 16) {
            const int o = 16 * warp, c = lane;
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float s = (i == c) ? 1.f : 0.f;
                const float bi = betas[o + i];
#pragma unroll
                for (int m = 0; m < i; ++m) s -= bi * PGs[(o + i) * LC + o + m] * x[m];
                x[i] = s;
                Ts[(o + i) * LC + o + c] = s;
            }
        }
        __syncthreads();
        for (int I = 1; I < 4; ++I) {
            const int nt = 2 * I;
            if (warp < nt) {
                float acc[1][4];
                zero(acc);
                wmma<1, LC, 1, LC, 1>(acc, PGs + 16 * I * LC, Ts + 8 * warp, 8 * warp, 16 * I);
                const float b0 = betas[16 * I + g], b1 = betas[16 * I + g + 8];
                acc[0][0] *= b0;
                acc[0][1] *= b0;
                acc[0][2] *= b1;
                acc[0][3] *= b1;
                store_frag<1, 52>(Rs + 8 * warp, acc);
            }
            __syncthreads();
            if (warp < nt) {
                float acc[1][4];
                zero(acc);
                wmma<1, LC, 1, 52, 1>(acc, Ts + 16 * I * LC + 16 * I, Rs + 8 * warp, 0, 16);
                store_frag<1, LC>(Ts + 16 * I * LC + 8 * warp, acc, -1.f);
            }
            __syncthreads();
        }
    }
    // A = q k^T (.) Gamma, lower incl. (over P (.) Gamma)
    {
        float aq[4][4];
        zero(aq);
        wmma<4, LK, 1, 1, LK, false, false, false>(aq, qs + 16 * mt * LK, ks + nb32 * LK, 0, DKB);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int l = 16 * mt + g + 8 * (e >> 1), m = nb32 + 8 * j + 2 * t + (e & 1);
                As[l * LC + m] = aq[j][e] * gamma(l, m);
            }
    }
    __syncthreads();
    store_tile<C, LC, true>(p.Am + cidx * C * C, As);
    if (DELTA) {
        // W = T diag(beta b) k, rounded, over q (no warp reads q any more)
        float acc[8][4];
        zero(acc);
        wmma<8, LC, 1, LK, 1, true, true>(acc, Ts + 16 * mt * LC, ks + nb64, 0, 16 * (mt + 1), bsc);
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[j][e] = tf32r(acc[j][e]);
        store_frag<8, LK>(Ws + 16 * mt * LK + nb64, acc);
        __syncthreads();
        store_tile<C, LC, true>(p.Tm + cidx * C * C, Ts);
        store_tile<DKB, LK>(p.Wm + cidx * C * DKB, Ws);
    }
    // Q~ = diag(b) q - A W, rounded (q read back from global memory when W holds its tile)
    {
        float acc[8][4];
        zero(acc);
        if (DELTA) wmma<8, LC, 1, LK, 1, false, true>(acc, As + 16 * mt * LC, Ws + nb64, 0, 16 * (mt + 1));
        float *dst = p.Qtm + cidx * C * DKB;
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int l = 16 * mt + g + 8 * h, i = nb64 + 8 * j + 2 * t;
                float q0 = 0.f, q1 = 0.f;
                if (!DELTA) {
                    q0 = qs[l * LK + i];
                    q1 = qs[l * LK + i + 1];
                } else if (l < nv) {
                    q0 = to_f32(qg[(size_t)l * DKB + i]);
                    q1 = to_f32(qg[(size_t)l * DKB + i + 1]);
                }
                *reinterpret_cast<float2 *>(dst + l * DKB + i) =
                    make_float2(tf32r(bs[l] * q0 - acc[j][2 * h]), tf32r(bs[l] * q1 - acc[j][2 * h + 1]));
            }
    }
    // K> = diag(e^{G_C - G}) k, rounded
    if (DELTA) {
        float *dst = p.Kcm + cidx * C * DKB;
        for (int i = tid; i < C * (DKB / 4); i += kThreads) {
            const int l = i / (DKB / 4), c = (i % (DKB / 4)) * 4;
            const float4 x = *reinterpret_cast<const float4 *>(ks + l * LK + c);
            const float e = es[l];
            *reinterpret_cast<float4 *>(dst + l * DKB + c) =
                make_float4(tf32r(x.x * e), tf32r(x.y * e), tf32r(x.z * e), tf32r(x.w * e));
        }
    }
    if (tid == 0) p.bC[cidx] = GATED ? expf(Gs[C - 1]) : 1.f;
}

// ------------------------------------------------------------------ chain
template <int DV>
struct ChainSmem {
    static constexpr int LO = DV + 4;
    static constexpr int Kc = 0, W = Kc + C * LKC, Qt = W + C * LK, dO = Qt + C * LK, floats = dO + C * LO;
};

template <int DV, bool DELTA>
__global__ void __launch_bounds__(DV * 2, 1) bwdtc_chain_kernel(TcBwdArgs p) {
    constexpr int NTH = DV * 2;  // one warp per 16 value rows
    using S = ChainSmem<DV>;
    constexpr int LO = S::LO;
    extern __shared__ float4 smem4[];
    float *sm = reinterpret_cast<float *>(smem4);
    float *Kcs = sm + S::Kc, *Wss = sm + S::W, *Qts = sm + S::Qt, *dOs = sm + S::dO;
    const int bh = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int v0 = 16 * warp, R = p.nch;
    const void *dummy = p.Qtm;

    float acc[16][4];  // dS rows v0 + g (+8), key channels 8j + 2t (+1)
    if (p.dST) {
        const float *s = p.dST + (size_t)bh * DV * DKB;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float2 a = *reinterpret_cast<const float2 *>(s + (v0 + g) * DKB + 8 * j + 2 * t);
            const float2 b = *reinterpret_cast<const float2 *>(s + (v0 + g + 8) * DKB + 8 * j + 2 * t);
            acc[j][0] = a.x;
            acc[j][1] = a.y;
            acc[j][2] = b.x;
            acc[j][3] = b.y;
        }
    } else {
        zero(acc);
    }
    auto issue_kc = [&](int r) {
        if (DELTA) cp_tile<DKB, LKC, NTH>(Kcs, p.Kcm + ((size_t)bh * R + r) * C * DKB, DKB, C, dummy);
        cp_async_commit();
    };
    auto issue_w = [&](int r) {
        if (DELTA) cp_tile<DKB, LK, NTH>(Wss, p.Wm + ((size_t)bh * R + r) * C * DKB, DKB, C, dummy);
        cp_async_commit();
    };
    auto issue_qd = [&](int r) {
        cp_tile<DKB, LK, NTH>(Qts, p.Qtm + ((size_t)bh * R + r) * C * DKB, DKB, C, dummy);
        const int nv = min(C, p.T - r * C);
        cp_tile<DV, LO, NTH>(dOs, p.dO ? p.dO + ((size_t)bh * p.T + (size_t)r * C) * DV : nullptr, DV, nv, dummy);
        cp_async_commit();
    };
    issue_kc(R - 1);
    issue_w(R - 1);
    issue_qd(R - 1);
    float bc = p.bC[(size_t)bh * R + R - 1];
    for (int r = R - 1; r >= 0; --r) {
        const size_t cidx = (size_t)bh * R + r;
        store_frag_global<16, true>(p.dSn + (cidx * DV + v0) * DKB, DKB, acc, 0, 16);  // a local-kernel operand
        const float bc_next = r > 0 ? p.bC[cidx - 1] : 1.f;
        float X[8][4];  // X = dS Kc^T: rows v0 + g (+8), tokens 8n + 2t (+1)
        cp_async_wait<2>();
        __syncthreads();
        if (DELTA) {
            zero(X);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint32_t a[4] = {f2tf32(acc[j][0]), f2tf32(acc[j][2]), f2tf32(acc[j][1]), f2tf32(acc[j][3])};
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    const float2 kk = *reinterpret_cast<const float2 *>(Kcs + (8 * n + g) * LKC + 8 * j + 2 * t);
                    const uint32_t b[2] = {__float_as_uint(kk.x), __float_as_uint(kk.y)};  // stored as tf32
                    mma_tf32_16x8x8(X[n], a, b);
                }
            }
        }
        __syncthreads();
        if (r > 0) {
            issue_kc(r - 1);
        } else {
            cp_async_commit();
        }
        cp_async_wait<2>();
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 16; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[j][e] *= bc;
        if (DELTA) {
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                const uint32_t a[4] = {f2tf32(-X[n][0]), f2tf32(-X[n][2]), f2tf32(-X[n][1]), f2tf32(-X[n][3])};
                const float *w0 = Wss + (8 * n + 2 * t) * LK + g;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const uint32_t b[2] = {__float_as_uint(w0[8 * j]), __float_as_uint(w0[LK + 8 * j])};
                    mma_tf32_16x8x8(acc[j], a, b);
                }
            }
        }
        __syncthreads();
        if (r > 0) {
            issue_w(r - 1);
        } else {
            cp_async_commit();
        }
        cp_async_wait<2>();
        __syncthreads();
        // dS += dO^T Q~
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            const int l0 = 8 * n + 2 * t;
            const uint32_t a[4] = {f2tf32(dOs[l0 * LO + v0 + g]), f2tf32(dOs[l0 * LO + v0 + g + 8]),
                                   f2tf32(dOs[(l0 + 1) * LO + v0 + g]), f2tf32(dOs[(l0 + 1) * LO + v0 + g + 8])};
            const float *q0 = Qts + l0 * LK + g;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint32_t b[2] = {__float_as_uint(q0[8 * j]), __float_as_uint(q0[LK + 8 * j])};
                mma_tf32_16x8x8(acc[j], a, b);
            }
        }
        __syncthreads();
        if (r > 0) {
            issue_qd(r - 1);
        } else {
            cp_async_commit();
        }
        bc = bc_next;
    }
    cp_async_wait<0>();
    if (p.dS0) store_frag_global<16>(p.dS0 + ((size_t)bh * DV + v0) * DKB, DKB, acc, 0, 16);
}

// ------------------------------------------------------------------ local
template <int DV>
struct LocalSmem {
    static constexpr int VJ = 32, LJ = VJ + 4;
    static constexpr int ks = 0, Ws = ks + C * LK, Ts = Ws + C * LK, As = Ts + C * LC, Rg = As + C * LC;
    // slice region
    static constexpr int Sj = Rg, dSj = Sj + VJ * LK, vj = dSj + VJ * LK, dOj = vj + C * LJ, Zj = dOj + C * LJ,
                         dZj = Zj + C * LJ, Rend = dZj + C * LJ;
    // after the slices: dA (then F), q, P (.) Gamma
    static constexpr int dAs = Rg, qs = dAs + C * LC, PGs = qs + C * LK;
    static_assert(PGs + C * LC <= Rend, "end-phase tiles exceed the slice region");
    // fixed-order partial sums (no float atomics, so the results are deterministic):
    // dbp[2][64] beta gradient by column half, dgp[3][64] gate gradient (element
    // pass, then the two column halves), cpp[2][64] the K> gate term, redw[8]
    // per-warp sums of dSn (.) S
    static_assert(VJ * LK <= C * LC, "an S slice must fit the X0 / X1 tiles");
    static constexpr int X0 = Rend, X1 = X0 + C * LC, Gs = X1 + C * LC, bs = Gs + C, es = bs + C, betas = es + C,
                         dbp = betas + C, dgp = dbp + 2 * C, cpp = dgp + 3 * C, redw = cpp + 2 * C,
                         floats = redw + 8;
};

template <int DV, bool DELTA, bool GATED, typename TIn>
__global__ void __launch_bounds__(kThreads, 1) bwdtc_local_kernel(TcBwdArgs p) {
    using S = LocalSmem<DV>;
    constexpr int VJ = S::VJ, LJ = S::LJ, NSL = DV / VJ;
    extern __shared__ float4 smem4[];
    float *sm = reinterpret_cast<float *>(smem4);
    float *ks = sm + S::ks, *Ws = sm + S::Ws, *Ts = sm + S::Ts, *As = sm + S::As;
    float *Sj0 = sm + S::Sj, *dSj0 = sm + S::dSj, *vj = sm + S::vj, *dOj = sm + S::dOj, *Zj = sm + S::Zj,
          *dZj = sm + S::dZj;
    float *X0 = sm + S::X0, *X1 = sm + S::X1, *Gs = sm + S::Gs, *bs = sm + S::bs, *es = sm + S::es,
          *betas = sm + S::betas, *dbp = sm + S::dbp, *dgp = sm + S::dgp, *cpp = sm + S::cpp, *redw = sm + S::redw;
    const int r = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int mt = warp & 3, nh = warp >> 2;
    const long tok0 = (long)bh * p.T + (long)r * C;
    const int nv = min(C, p.T - r * C);
    const size_t cidx = (size_t)bh * p.nch + r;
    const float *Sr = p.states + cidx * DV * DKB, *dSr = p.dSn + cidx * DV * DKB;

    const void *dummy = p.Am;
    if (tid == 0) {  // everything read after the first tiles, into L2 now
        l2_prefetch(Sr, DV * DKB * 4);
        l2_prefetch(dSr, DV * DKB * 4);
        l2_prefetch(static_cast<const char *>(p.v) + tok0 * DV * sizeof(TIn), nv * DV * sizeof(TIn));
        if (p.dO) l2_prefetch(p.dO + tok0 * DV, nv * DV * 4);
        l2_prefetch(static_cast<const char *>(p.q) + tok0 * DKB * sizeof(TIn), nv * DKB * sizeof(TIn));
        if (DELTA) l2_prefetch(p.PGm + cidx * C * C, C * C * 4);
    }
    cp_tile<C, LC, kThreads>(As, p.Am + cidx * C * C, C, C, dummy);
    if (DELTA) {
        cp_tile<DKB, LK, kThreads>(Ws, p.Wm + cidx * C * DKB, DKB, C, dummy);
        cp_tile<C, LC, kThreads>(Ts, p.Tm + cidx * C * C, C, C, dummy);
    }
    cp_async_commit();
    load_in<TIn, DKB, LK, kThreads>(ks, static_cast<const char *>(p.k) + tok0 * DKB * sizeof(TIn), DKB, nv);
    if (tid < C) betas[tid] = (DELTA && tid < nv) ? p.beta[tok0 + tid] : 0.f;
    for (int i = tid; i < 7 * C; i += kThreads) dbp[i] = 0.f;  // dbp, dgp, cpp
    if (warp == 0) gate_prefix<GATED>(p.g, tok0, nv, Gs, bs, es);

    float dKc[8][4], dQb[8][4], dWa[8][4], dA[4][4], dTv[4][4];
    zero(dKc);
    zero(dQb);
    zero(dWa);
    zero(dA);
    zero(dTv);
    float sds = 0.f;  // sum of dSn (.) S over the thread's loads
    // S and dSn rows go through two buffers: slice s in (Sj0, dSj0) for even s and in
    // (X0, X1), free until the element pass, for odd s; slice s + 1 is copied while
    // slice s is processed
    cp_tile<DKB, LK, kThreads, VJ>(Sj0, Sr, DKB, VJ, dummy);
    cp_tile<DKB, LK, kThreads, VJ>(dSj0, dSr, DKB, VJ, dummy);
    cp_async_commit();
    for (int s = 0; s < NSL; ++s) {
        const int vb = s * VJ;
        float *Sj = (s & 1) ? X0 : Sj0, *dSj = (s & 1) ? X1 : dSj0;
        __syncthreads();
        cp_tile<VJ, LJ, kThreads>(dOj, p.dO ? p.dO + tok0 * DV + vb : nullptr, DV, nv, dummy);
        cp_async_commit();
        if (s + 1 < NSL) {
            cp_tile<DKB, LK, kThreads, VJ>((s & 1) ? Sj0 : X0, Sr + (size_t)(vb + VJ) * DKB, DKB, VJ, dummy);
            cp_tile<DKB, LK, kThreads, VJ>((s & 1) ? dSj0 : X1, dSr + (size_t)(vb + VJ) * DKB, DKB, VJ, dummy);
        }
        cp_async_commit();
        load_in<TIn, VJ, LJ, kThreads>(vj, static_cast<const char *>(p.v) + (tok0 * DV + vb) * sizeof(TIn), DV, nv);
        cp_async_wait<1>();  // all but the next slice's copies
        // the thread's own copies are visible to it: sum of dSn (.) S over them,
        // and S and dO rounded to tf32 in place (MMA operands; dSn is stored so)
        for (int i = tid; i < VJ * (DKB / 4); i += kThreads) {
            const int rr = i / (DKB / 4), c = (i % (DKB / 4)) * 4;
            float4 a = *reinterpret_cast<const float4 *>(Sj + rr * LK + c);
            const float4 b = *reinterpret_cast<const float4 *>(dSj + rr * LK + c);
            sds += a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
            *reinterpret_cast<float4 *>(Sj + rr * LK + c) = make_float4(tf32r(a.x), tf32r(a.y), tf32r(a.z), tf32r(a.w));
        }
        for (int i = tid; i < C * (VJ / 4); i += kThreads) {
            const int rr = i / (VJ / 4), c = (i % (VJ / 4)) * 4;
            const float4 a = *reinterpret_cast<const float4 *>(dOj + rr * LJ + c);
            *reinterpret_cast<float4 *>(dOj + rr * LJ + c) = make_float4(tf32r(a.x), tf32r(a.y), tf32r(a.z), tf32r(a.w));
        }
        __syncthreads();
        // Z and dZ for this slice: warp (mt, nh) owns rows 16 mt, columns 16 nh
        {
            float az[2][4], adz[2][4];
            zero(az);
            zero(adz);
            if (DELTA) {
                float au[2][4];
                zero(au);
                wmma<2, LC, 1, LJ, 1, true, false, false>(au, Ts + 16 * mt * LC, vj + 16 * nh, 0, 16 * (mt + 1),
                                                          betas);
                wmma<2, LK, 1, 1, LK, false, false, false>(az, Ws + 16 * mt * LK, Sj + 16 * nh * LK, 0, DKB);
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e) az[j][e] = au[j][e] - az[j][e];
            }
            wmma<2, LK, 1, 1, LK, false, false, false>(adz, ks + 16 * mt * LK, dSj + 16 * nh * LK, 0, DKB);
            if (GATED) {
                const float e0 = es[16 * mt + g], e1 = es[16 * mt + g + 8];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    adz[j][0] *= e0;
                    adz[j][1] *= e0;
                    adz[j][2] *= e1;
                    adz[j][3] *= e1;
                }
            }
            wmma<2, 1, LC, LJ, 1, false, true, false>(adz, As + 16 * mt, dOj + 16 * nh, 16 * mt, C);
            if (DELTA) store_frag<2, LJ, true>(Zj + 16 * mt * LJ + 16 * nh, az);
            store_frag<2, LJ, true>(dZj + 16 * mt * LJ + 16 * nh, adz);
            if (!DELTA) store_frag_global<2>(p.dv + tok0 * DV + vb + 16 * nh, DV, adz, 16 * mt, nv);
        }
        __syncthreads();
        const float *Zs = DELTA ? Zj : vj;
        wmma<8, LJ, 1, LK, 1, false, true, false>(dKc, Zs + 16 * mt * LJ, dSj + 64 * nh, 0, VJ);
        wmma<8, LJ, 1, LK, 1, false, true, false>(dQb, dOj + 16 * mt * LJ, Sj + 64 * nh, 0, VJ);
        wmma<4, LJ, 1, 1, LJ, false, false, false>(dA, dOj + 16 * mt * LJ, Zs + 32 * nh * LJ, 0, VJ);
        if (DELTA) {
            wmma<8, LJ, 1, LK, 1, false, true, false>(dWa, dZj + 16 * mt * LJ, Sj + 64 * nh, 0, VJ);
            wmma<4, LJ, 1, 1, LJ, false, false, false>(dTv, dZj + 16 * mt * LJ, vj + 32 * nh * LJ, 0, VJ);
            // dv = diag(beta) T^T dZ;  dbeta += rows of (T^T dZ) (.) v
            float ad[2][4];
            zero(ad);
            wmma<2, 1, LC, LJ, 1, false, true, false>(ad, Ts + 16 * mt, dZj + 16 * nh, 16 * mt, C);
            float rb0 = 0.f, rb1 = 0.f;
            const int l0 = 16 * mt + g;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int c = 16 * nh + 8 * j + 2 * t;
                rb0 += ad[j][0] * vj[l0 * LJ + c] + ad[j][1] * vj[l0 * LJ + c + 1];
                rb1 += ad[j][2] * vj[(l0 + 8) * LJ + c] + ad[j][3] * vj[(l0 + 8) * LJ + c + 1];
                ad[j][0] *= betas[l0];
                ad[j][1] *= betas[l0];
                ad[j][2] *= betas[l0 + 8];
                ad[j][3] *= betas[l0 + 8];
            }
            store_frag_global<2>(p.dv + tok0 * DV + vb + 16 * nh, DV, ad, 16 * mt, nv);
            rb0 += __shfl_xor_sync(0xffffffffu, rb0, 1);
            rb0 += __shfl_xor_sync(0xffffffffu, rb0, 2);
            rb1 += __shfl_xor_sync(0xffffffffu, rb1, 1);
            rb1 += __shfl_xor_sync(0xffffffffu, rb1, 2);
            if (t == 0) {
                dbp[nh * C + l0] += rb0;
                dbp[nh * C + l0 + 8] += rb1;
            }
        }
    }
    // sum of dSn (.) S over the chunk's state
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sds += __shfl_xor_sync(0xffffffffu, sds, off);
    if (lane == 0) redw[warp] = sds;
    __syncthreads();

    float *dAs = sm + S::dAs, *qs = sm + S::qs, *PGs = sm + S::PGs;
    if (DELTA) store_frag<8, LK, true>(Ws + 16 * mt * LK + 64 * nh, dWa, -1.f);  // dW
    store_frag<4, LC>(dAs + 16 * mt * LC + 32 * nh, dA);
    if (DELTA) cp_tile<C, LC, kThreads>(PGs, p.PGm + cidx * C * C, C, C, dummy);
    cp_async_commit();
    load_in<TIn, DKB, LK, kThreads>(qs, static_cast<const char *>(p.q) + tok0 * DKB * sizeof(TIn), DKB, nv);
    cp_async_wait<0>();
    __syncthreads();

    if (DELTA) {
        // dT = (dZ v^T + diag(b) ... ) with the column scales: dT[l,m] = beta_m (dTv + b_m (dW k^T))[l,m]
        {
            float a2[4][4];
            zero(a2);
            wmma<4, LK, 1, 1, LK, false, false, false>(a2, Ws + 16 * mt * LK, ks + 32 * nh * LK, 0, DKB);
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int m = 32 * nh + 8 * j + 2 * t + (e & 1);
                    dTv[j][e] = betas[m] * (dTv[j][e] + bs[m] * a2[j][e]);
                }
            store_frag<4, LC, true>(X0 + 16 * mt * LC + 32 * nh, dTv);
        }
        __syncthreads();
        {  // Y = dT T^T
            float y[4][4];
            zero(y);
            wmma<4, LC, 1, 1, LC, false, false, false>(y, X0 + 16 * mt * LC, Ts + 32 * nh * LC, 0, C);
            store_frag<4, LC, true>(X1 + 16 * mt * LC + 32 * nh, y);
        }
        __syncthreads();
        {  // dL = strict-lower(-T^T Y)
            float dl[4][4];
            zero(dl);
            wmma<4, 1, LC, LC, 1, false, true, false>(dl, Ts + 16 * mt, X1 + 32 * nh, 16 * mt, C);
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int l = 16 * mt + g + 8 * (e >> 1), m = 32 * nh + 8 * j + 2 * t + (e & 1);
                    dl[j][e] = m < l ? -dl[j][e] : 0.f;
                }
            store_frag<4, LC>(X0 + 16 * mt * LC + 32 * nh, dl);
        }
        __syncthreads();
    }
    // element pass over (l, m): F = dA (.) Gamma (over dA), E = dL beta_l Gamma
    // (over dL), H = dGamma (.) Gamma (into X1); row sums -> dG, dbeta
    {
        const int l = tid >> 2, m0 = (tid & 3) * 16;
        const float Gl = Gs[l], bl = betas[l];
        float rowH = 0.f, rowB = 0.f;
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
            const int m = m0 + c;
            const float gam = m <= l ? (GATED ? expf(Gl - Gs[m]) : 1.f) : 0.f;
            const float da = dAs[l * LC + m];
            float h = m < l ? da * As[l * LC + m] : 0.f;
            dAs[l * LC + m] = tf32r(da * gam);
            if (DELTA) {
                const float dl = X0[l * LC + m], pg = PGs[l * LC + m];
                h += dl * bl * pg;
                rowB += dl * pg;
                X0[l * LC + m] = tf32r(dl * bl * gam);
            }
            X1[l * LC + m] = h;
            rowH += h;
        }
        rowH += __shfl_xor_sync(0xffffffffu, rowH, 1);
        rowH += __shfl_xor_sync(0xffffffffu, rowH, 2);
        rowB += __shfl_xor_sync(0xffffffffu, rowB, 1);
        rowB += __shfl_xor_sync(0xffffffffu, rowB, 2);
        if ((tid & 3) == 0) {
            dgp[l] = rowH;
            if (DELTA) dbp[l] += rowB;
        }
    }
    __syncthreads();
    if (GATED && tid < C) {
        float s = 0.f;
        for (int l = 0; l < C; ++l) s += X1[l * LC + tid];
        dgp[tid] -= s;
    }
    // dk and dq: warp (mt, nh) owns rows 16 mt, columns 64 nh (the dKc / dQb / dW blocks)
    {
        const int nb = 64 * nh, l0 = 16 * mt + g;
        float dkacc[8][4], dqacc[8][4];
        float rs[2] = {0.f, 0.f}, rc[2] = {0.f, 0.f}, rq[2] = {0.f, 0.f};
        if (DELTA) {
            float kb[8][4];
            zero(kb);
            wmma<8, 1, LC, LK, 1, false, true, false>(kb, Ts + 16 * mt, Ws + nb, 16 * mt, C);  // T^T dW
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int l = l0 + 8 * (e >> 1), i = nb + 8 * j + 2 * t + (e & 1);
                    rs[e >> 1] += kb[j][e] * ks[l * LK + i];
                    dkacc[j][e] = bs[l] * betas[l] * kb[j][e];
                }
        } else {
            zero(dkacc);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int l = l0 + 8 * (e >> 1), i = nb + 8 * j + 2 * t + (e & 1);
                rc[e >> 1] += dKc[j][e] * ks[l * LK + i];
                rq[e >> 1] += dQb[j][e] * qs[l * LK + i];
                dkacc[j][e] += es[l] * dKc[j][e];
                dqacc[j][e] = bs[l] * dQb[j][e];
            }
        if (DELTA) {
            wmma<8, LC, 1, LK, 1, false, true, false>(dkacc, X0 + 16 * mt * LC, ks + nb, 0, 16 * (mt + 1));  // E k
            wmma<8, 1, LC, LK, 1, false, true, false>(dkacc, X0 + 16 * mt, ks + nb, 16 * mt, C);  // E^T k
        }
        wmma<8, 1, LC, LK, 1, false, true, false>(dkacc, dAs + 16 * mt, qs + nb, 16 * mt, C);  // F^T q
        wmma<8, LC, 1, LK, 1, false, true, false>(dqacc, dAs + 16 * mt * LC, ks + nb, 0, 16 * (mt + 1));  // F k
        store_frag_global<8>(p.dk + tok0 * DKB + nb, DKB, dkacc, 16 * mt, nv);
        store_frag_global<8>(p.dq + tok0 * DKB + nb, DKB, dqacc, 16 * mt, nv);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 1);
            rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 2);
            rc[h] += __shfl_xor_sync(0xffffffffu, rc[h], 1);
            rc[h] += __shfl_xor_sync(0xffffffffu, rc[h], 2);
            rq[h] += __shfl_xor_sync(0xffffffffu, rq[h], 1);
            rq[h] += __shfl_xor_sync(0xffffffffu, rq[h], 2);
        }
        if (t == 0) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int l = l0 + 8 * h;
                const float cp = es[l] * rc[h];  // (e^{G_C - G_l} k_l) . dKc_l
                float dgl = bs[l] * rq[h] - cp;
                if (DELTA) {
                    dgl += bs[l] * betas[l] * rs[h];
                    dbp[nh * C + l] += bs[l] * rs[h];
                }
                dgp[(1 + nh) * C + l] = dgl;
                cpp[nh * C + l] = cp;
            }
        }
    }
    __syncthreads();
    if (warp == 0) {
        if (GATED) {
            // dG_63 += b_C sum(dSn (.) S) + sum_l c'_l;  dg_s = sum_{l >= s} dG_l
            auto dG = [&](int l) { return dgp[l] + dgp[C + l] + dgp[2 * C + l]; };
            float x0 = dG(2 * lane), x1 = dG(2 * lane + 1);
            float cs = cpp[2 * lane] + cpp[C + 2 * lane] + cpp[2 * lane + 1] + cpp[C + 2 * lane + 1];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) cs += __shfl_xor_sync(0xffffffffu, cs, off);
            float sds_all = 0.f;
#pragma unroll
            for (int w = 0; w < kThreads / 32; ++w) sds_all += redw[w];
            if (lane == 31) x1 += expf(Gs[C - 1]) * sds_all + cs;
            float s = x0 + x1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, s, off);
                if (lane + off < 32) s += y;
            }
            if (2 * lane < nv) p.dg[tok0 + 2 * lane] = s;
            if (2 * lane + 1 < nv) p.dg[tok0 + 2 * lane + 1] = s - x0;
        }
        if (DELTA) {
            if (2 * lane < nv) p.dbeta[tok0 + 2 * lane] = dbp[2 * lane] + dbp[C + 2 * lane];
            if (2 * lane + 1 < nv) p.dbeta[tok0 + 2 * lane + 1] = dbp[2 * lane + 1] + dbp[C + 2 * lane + 1];
        }
    }
}

// ------------------------------------------------------------------ launch
template <typename K>
int prep_smem(K kern, size_t bytes) {
    return (int)cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int DV, bool DELTA, bool GATED, typename TIn>
int launch_all(const TcBwdArgs &a, cudaStream_t st) {
    const dim3 grid(a.nch, a.BH);
    {
        auto kern = bwdtc_prep_kernel<DELTA, GATED, TIn>;
        const size_t smem = PrepSmem::floats * sizeof(float);
        int e = prep_smem(kern, smem);
        if (e) return e;
        kern<<<grid, kThreads, smem, st>>>(a);
        if ((e = (int)cudaGetLastError())) return e;
    }
    {
        auto kern = bwdtc_chain_kernel<DV, DELTA>;
        const size_t smem = ChainSmem<DV>::floats * sizeof(float);
        int e = prep_smem(kern, smem);
        if (e) return e;
        kern<<<a.BH, DV * 2, smem, st>>>(a);
        if ((e = (int)cudaGetLastError())) return e;
    }
    {
        auto kern = bwdtc_local_kernel<DV, DELTA, GATED, TIn>;
        const size_t smem = LocalSmem<DV>::floats * sizeof(float);
        int e = prep_smem(kern, smem);
        if (e) return e;
        kern<<<grid, kThreads, smem, st>>>(a);
        if ((e = (int)cudaGetLastError())) return e;
    }
    return 0;
}

template <int DV, typename TIn>
int launch_modes(const TcBwdArgs &a, int update, int gate, cudaStream_t st) {
    const bool gated = gate == kGateScalar;
    if (update == kDelta)
        return gated ? launch_all<DV, true, true, TIn>(a, st) : launch_all<DV, true, false, TIn>(a, st);
    return gated ? launch_all<DV, false, true, TIn>(a, st) : launch_all<DV, false, false, TIn>(a, st);
}

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

}  // namespace
}  // namespace gdn

// Workspace of gdn_chunk_bwd_tc: per chunk and head T, A, P (.) Gamma [64][64],
// W, Kc, Q~ [64][dk], dSn [dv][dk], b_C, each region on a 256-byte boundary
// (T, P (.) Gamma, W, Kc only for the delta rule).  off[0..7] receive the byte
// offsets of T, A, PG, W, Kc, Q~, dSn, b_C; returns the total.
size_t gdn_bwd_tc_layout(long BH, int nch, int dk, int dv, int delta, size_t *off) {
    using gdn::align256;
    const size_t n = (size_t)BH * nch, cc = n * gdn::kChunk * gdn::kChunk * 4, cd = n * gdn::kChunk * dk * 4;
    const size_t sizes[8] = {delta ? cc : 0, cc, delta ? cc : 0, delta ? cd : 0, delta ? cd : 0, cd,
                             n * (size_t)dv * dk * 4, n * 4};
    size_t o = 0;
    for (int i = 0; i < 8; ++i) {
        if (off) off[i] = o;
        o = align256(o + sizes[i]);
    }
    return o;
}

// The three passes.  Returns a cudaError_t value.
int gdn_launch_bwd_tc(const void *q, const void *k, const void *v, const float *g, const float *beta,
                      const float *states, const float *dO, const float *dST, float *dq, float *dk, float *dv,
                      float *dg, float *dbeta, float *dS0, void *ws, int BH, int T, int dv_, int update, int gate,
                      int in_bf16, cudaStream_t st) {
    using namespace gdn;
    TcBwdArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.states = states; a.dO = dO; a.dST = dST;
    a.dq = dq; a.dk = dk; a.dv = dv; a.dg = dg; a.dbeta = dbeta; a.dS0 = dS0;
    a.BH = BH; a.T = T; a.nch = (T + kChunk - 1) / kChunk;
    size_t off[8];
    gdn_bwd_tc_layout(BH, a.nch, DKB, dv_, update == kDelta, off);
    char *w = static_cast<char *>(ws);
    a.Tm = reinterpret_cast<float *>(w + off[0]);
    a.Am = reinterpret_cast<float *>(w + off[1]);
    a.PGm = reinterpret_cast<float *>(w + off[2]);
    a.Wm = reinterpret_cast<float *>(w + off[3]);
    a.Kcm = reinterpret_cast<float *>(w + off[4]);
    a.Qtm = reinterpret_cast<float *>(w + off[5]);
    a.dSn = reinterpret_cast<float *>(w + off[6]);
    a.bC = reinterpret_cast<float *>(w + off[7]);
    if (dv_ == 128)
        return in_bf16 ? launch_modes<128, __nv_bfloat16>(a, update, gate, st)
                       : launch_modes<128, float>(a, update, gate, st);
    return in_bf16 ? launch_modes<64, __nv_bfloat16>(a, update, gate, st) : launch_modes<64, float>(a, update, gate, st);
}
