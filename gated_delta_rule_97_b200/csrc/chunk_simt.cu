// Chunkwise prefill in fp32 SIMT arithmetic (all modes, dk in {64,128}).
//
// One CTA owns one (b,h) head and a 32-wide slice of the value dimension (the
// rows of S evolve independently: s_i <- s_i Diag(a)(I - beta k k^T) + beta v_i
// k^T), and walks the chunks of its sequence in order, keeping its state slice
// in shared memory.  Per chunk (C = 64), following "Linear Attention,
// Visualized" -- "Chunkwise algorithm", "Mamba-2 ... Chunkwise form", "Gated
// Linear Attention (GLA)", "The triangular correction system", "Optional: Use
// UT to share the triangular transform", "Correct the incoming state" and the
// GDN / KDA tables:
//   a1  G_l = sum_{s<=l} g_s (inclusive log-gate prefix in the chunk)
//   a2  A[l,m] = sum_i q_li k_mi e^{G_li-G_mi} (m<=l),
//       L[l,m] = beta_l sum_i k_li k_mi e^{G_li-G_mi} (m<l)
//   a3+a4  (I + L) [W | U] = diag(beta) [K< | V]  by forward substitution
//          (the UT transform applied to both right-hand sides at once)
//   a5  Z = U - W S^T             (delta; otherwise Z = V)
//   a6  O = Q< S^T + A Z
//   a7  S <- S Diag(e^{G_C}) + Z^T K>,  K>_m = k_m e^{G_C - G_m}
// The last chunk is padded with identity tokens (q=k=v=0, beta=0, g=0).
// Everything is fp32; this is the kernel for fp32 inputs and the general
// fallback for shapes the tensor-core kernel does not serve.
#include "common.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int kDvs = 32;  // value rows of S per CTA

template <int DK, int UPD, int GATE>
struct SimtSmem {
    static constexpr int C = kChunk;
    static constexpr int LDK = DK + 1;
    static constexpr int LDV = kDvs + 1;
    static constexpr int LDC = C + 1;
    static constexpr int GSZ = (GATE == kGateChannel) ? C * LDK : C;
    static constexpr int LSZ = (UPD == kDelta) ? C * LDC : 0;
    static constexpr int WSZ = (UPD == kDelta) ? C * LDK : 0;
    static constexpr int floats = 2 * C * LDK + C * LDV + GSZ + C * LDC + LSZ + WSZ + kDvs * LDK + C + DK;
    static constexpr size_t bytes = sizeof(float) * floats;
};

template <int DK, int UPD, int GATE, typename TIn, typename TOut>
__global__ void __launch_bounds__(kThreads) chunk_simt_kernel(ChunkArgs a) {
    using L = SimtSmem<DK, UPD, GATE>;
    constexpr int C = kChunk, LDK = L::LDK, LDV = L::LDV, LDC = L::LDC;
    extern __shared__ float sm[];
    float *sQ = sm;               // [C][LDK]  q, later Q< (channel gate)
    float *sK = sQ + C * LDK;     // [C][LDK]  k, later K>
    float *sV = sK + C * LDK;     // [C][LDV]  v slice, later U, then Z
    float *sG = sV + C * LDV;     // [C] or [C][LDK]  log-gate prefix G
    float *sA = sG + L::GSZ;      // [C][LDC]  A
    float *sL = sA + C * LDC;     // [C][LDC]  beta-scaled strict-lower L (delta)
    float *sW = sL + L::LSZ;      // [C][LDK]  W (delta)
    float *sS = sW + L::WSZ;      // [kDvs][LDK]  state slice
    float *sB = sS + kDvs * LDK;  // [C] beta
    float *sBC = sB + C;          // [DK] e^{G_C} per key channel

    const int tid = threadIdx.x;
    const int nslices = a.dv / kDvs;
    const int bh = blockIdx.x / nslices;
    const int v0 = (blockIdx.x % nslices) * kDvs;
    const int T = a.T, dv = a.dv;
    // virtual steps (k, v, beta) vs real tokens (q, g, o); nh = 1 makes them the same
    const int nh = a.nh, Tr = T / nh;
    const TIn *q = static_cast<const TIn *>(a.q) + (size_t)bh * Tr * DK;
    const TIn *k = static_cast<const TIn *>(a.k) + (size_t)bh * T * DK;
    const TIn *v = static_cast<const TIn *>(a.v) + (size_t)bh * T * dv;
    const float *g = nullptr;
    if (GATE == kGateScalar) g = a.g + (size_t)bh * Tr;
    if (GATE == kGateChannel) g = a.g + (size_t)bh * Tr * DK;
    const float *beta = (UPD == kDelta) ? a.beta + (size_t)bh * T : nullptr;
    TOut *o = static_cast<TOut *>(a.o) + (size_t)bh * Tr * dv;

    for (int i = tid; i < kDvs * DK; i += kThreads) {
        const int vv = i / DK, j = i % DK;
        sS[vv * LDK + j] = (a.mode & kModeS0Eye) ? (v0 + vv == j ? 1.f : 0.f)
                           : a.S0 ? a.S0[((size_t)bh * dv + v0 + vv) * DK + j] : 0.f;
    }

    for (int t0 = 0; t0 < T; t0 += C) {
        const int n = min(C, T - t0);
        __syncthreads();
        // ---- load the chunk (identity-token padding past n) ----
        for (int i = tid; i < C * DK; i += kThreads) {
            const int l = i / DK, j = i % DK;
            float qv = 0.f, kv = 0.f, gv = 0.f;
            if (l < n) {
                const int m = t0 + l, tr = m / nh, sub = m - tr * nh;
                if (sub == nh - 1) qv = pro_feature(to_f32(q[(size_t)tr * DK + j]), a.pro);
                kv = pro_feature(to_f32(k[(size_t)m * DK + j]), a.pro);
                if (GATE == kGateChannel && sub == 0) gv = pro_gate(g[(size_t)tr * DK + j], a.pro);
            }
            sQ[l * LDK + j] = qv;
            sK[l * LDK + j] = kv;
            if (GATE == kGateChannel) sG[l * LDK + j] = gv;
        }
        for (int i = tid; i < C * kDvs; i += kThreads) {
            const int l = i / kDvs, c = i % kDvs;
            sV[l * LDV + c] = (l < n && !(a.mode & kModeZeroV)) ? to_f32(v[(size_t)(t0 + l) * dv + v0 + c]) : 0.f;
        }
        if (tid < C) {
            if (GATE == kGateScalar)
                sG[tid] = (tid < n && (t0 + tid) % nh == 0) ? pro_gate(g[(t0 + tid) / nh], a.pro) : 0.f;
            if (UPD == kDelta) sB[tid] = (tid < n) ? pro_beta(beta[t0 + tid], a.pro) : 0.f;
        }
        __syncthreads();
        if (a.pro & kProL2) {
            // unit rows of q and k (the A scratch is free until a2); zero rows stay zero
            float *inv = sA;
            if (tid < 2 * C) {
                const float *row = (tid < C ? sQ : sK) + (tid % C) * LDK;
                float ss = 0.f;
                for (int j = 0; j < DK; ++j) ss = fmaf(row[j], row[j], ss);
                inv[tid] = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
            }
            __syncthreads();
            for (int i = tid; i < C * DK; i += kThreads) {
                const int l = i / DK, j = i % DK;
                sQ[l * LDK + j] *= inv[l];
                sK[l * LDK + j] *= inv[C + l];
            }
            __syncthreads();
        }

        // ---- a1: inclusive prefix of the log-gate ----
        if (GATE == kGateScalar) {
            if (tid < 32) {
                const float x0 = sG[2 * tid], x1 = sG[2 * tid + 1];
                float s = x0 + x1;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, s, off);
                    if (tid >= off) s += y;
                }
                const float excl = s - (x0 + x1);
                sG[2 * tid] = excl + x0;
                sG[2 * tid + 1] = excl + x0 + x1;
            }
        } else if (GATE == kGateChannel) {
            if (tid < DK) {
                float s = 0.f;
                for (int l = 0; l < C; ++l) {
                    s += sG[l * LDK + tid];
                    sG[l * LDK + tid] = s;
                }
            }
        }
        __syncthreads();

        // ---- a2: A (inclusive lower) and L (strict lower, beta-scaled) ----
        for (int p = tid; p < C * C; p += kThreads) {
            const int l = p / C, m = p % C;
            float av = 0.f, lv = 0.f;
            if (m <= l) {
                float dq = 0.f, dkk = 0.f;
                if (GATE == kGateChannel) {
                    for (int j = 0; j < DK; ++j) {
                        const float km = sK[m * LDK + j] * __expf(sG[l * LDK + j] - sG[m * LDK + j]);
                        dq = fmaf(sQ[l * LDK + j], km, dq);
                        if (UPD == kDelta) dkk = fmaf(sK[l * LDK + j], km, dkk);
                    }
                } else {
                    for (int j = 0; j < DK; ++j) {
                        dq = fmaf(sQ[l * LDK + j], sK[m * LDK + j], dq);
                        if (UPD == kDelta) dkk = fmaf(sK[l * LDK + j], sK[m * LDK + j], dkk);
                    }
                    if (GATE == kGateScalar) {
                        const float e = __expf(sG[l] - sG[m]);
                        dq *= e;
                        dkk *= e;
                    }
                }
                av = dq;
                if (UPD == kDelta && m < l) lv = sB[l] * dkk;
            }
            sA[l * LDC + m] = av;
            if (UPD == kDelta) sL[l * LDC + m] = lv;
        }
        __syncthreads();

        if (UPD == kDelta) {
            // ---- a3+a4: forward substitution, one column of [W | U] per thread ----
            constexpr int NC = DK + kDvs;
            if (tid < NC) {
                const int c = tid;
                for (int l = 0; l < C; ++l) {
                    float r;
                    if (c < DK) {
                        float kl = sK[l * LDK + c];
                        if (GATE == kGateScalar) kl *= __expf(sG[l]);
                        if (GATE == kGateChannel) kl *= __expf(sG[l * LDK + c]);
                        r = sB[l] * kl;
                    } else {
                        r = sB[l] * sV[l * LDV + (c - DK)];
                    }
                    for (int m = 0; m < l; ++m) {
                        const float x = (c < DK) ? sW[m * LDK + c] : sV[m * LDV + (c - DK)];
                        r = fmaf(-sL[l * LDC + m], x, r);
                    }
                    if (c < DK)
                        sW[l * LDK + c] = r;
                    else
                        sV[l * LDV + (c - DK)] = r;
                }
            }
            __syncthreads();
            // ---- a5: Z = U - W S^T (in place over U) ----
            for (int p = tid; p < C * kDvs; p += kThreads) {
                const int l = p / kDvs, vv = p % kDvs;
                float acc = sV[l * LDV + vv];
                for (int j = 0; j < DK; ++j) acc = fmaf(-sW[l * LDK + j], sS[vv * LDK + j], acc);
                sV[l * LDV + vv] = acc;
            }
            __syncthreads();
        }

        // ---- a6: O = Q< S^T + A Z ----
        if (GATE == kGateChannel) {
            for (int i = tid; i < C * DK; i += kThreads) {
                const int l = i / DK, j = i % DK;
                sQ[l * LDK + j] *= __expf(sG[l * LDK + j]);
            }
            __syncthreads();
        }
        for (int p = tid; p < C * kDvs; p += kThreads) {
            const int l = p / kDvs, vv = p % kDvs;
            float hist = 0.f;
            for (int j = 0; j < DK; ++j) hist = fmaf(sQ[l * LDK + j], sS[vv * LDK + j], hist);
            if (GATE == kGateScalar) hist *= __expf(sG[l]);
            float loc = 0.f;
            for (int m = 0; m <= l; ++m) loc = fmaf(sA[l * LDC + m], sV[m * LDV + vv], loc);
            if (l < n && (t0 + l) % nh == nh - 1 && !(a.mode & kModeNoOut))
                o[(size_t)((t0 + l) / nh) * dv + v0 + vv] = from_f32<TOut>(hist + loc);
        }
        __syncthreads();

        // ---- a7: S <- S Diag(e^{G_C}) + Z^T K> ----
        for (int i = tid; i < C * DK; i += kThreads) {
            const int l = i / DK, j = i % DK;
            float e = 1.f;
            if (GATE == kGateScalar) e = __expf(sG[C - 1] - sG[l]);
            if (GATE == kGateChannel) e = __expf(sG[(C - 1) * LDK + j] - sG[l * LDK + j]);
            sK[l * LDK + j] *= e;
        }
        if (tid < DK) {
            float e = 1.f;
            if (GATE == kGateScalar) e = __expf(sG[C - 1]);
            if (GATE == kGateChannel) e = __expf(sG[(C - 1) * LDK + tid]);
            sBC[tid] = e;
        }
        __syncthreads();
        for (int p = tid; p < kDvs * DK; p += kThreads) {
            const int vv = p / DK, j = p % DK;
            float acc = sS[vv * LDK + j] * sBC[j];
            for (int l = 0; l < C; ++l) acc = fmaf(sV[l * LDV + vv], sK[l * LDK + j], acc);
            sS[vv * LDK + j] = acc;
        }
    }
    __syncthreads();
    if (a.ST) {
        for (int i = tid; i < kDvs * DK; i += kThreads) {
            const int vv = i / DK, j = i % DK;
            a.ST[((size_t)bh * dv + v0 + vv) * DK + j] = sS[vv * LDK + j];
        }
    }
}

template <int DK, int UPD, int GATE, typename TIn, typename TOut>
int launch_simt(const ChunkArgs &a, cudaStream_t stream) {
    using L = SimtSmem<DK, UPD, GATE>;
    auto kern = chunk_simt_kernel<DK, UPD, GATE, TIn, TOut>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
    if (e != cudaSuccess) return (int)e;
    const long grid = (long)a.BH * (a.dv / kDvs);
    if (grid == 0) return 0;
    kern<<<(unsigned)grid, kThreads, L::bytes, stream>>>(a);
    return (int)cudaGetLastError();
}

template <int DK, int UPD, int GATE>
int launch_types(const ChunkArgs &a, int in_bf16, int out_bf16, cudaStream_t s) {
    if (in_bf16) {
        return out_bf16 ? launch_simt<DK, UPD, GATE, __nv_bfloat16, __nv_bfloat16>(a, s)
                        : launch_simt<DK, UPD, GATE, __nv_bfloat16, float>(a, s);
    }
    return out_bf16 ? launch_simt<DK, UPD, GATE, float, __nv_bfloat16>(a, s)
                    : launch_simt<DK, UPD, GATE, float, float>(a, s);
}

template <int DK>
int launch_modes(const ChunkArgs &a, int update, int gate, int in_bf16, int out_bf16, cudaStream_t s) {
    if (update == kAdditive) return launch_types<DK, kAdditive, kGateNone>(a, in_bf16, out_bf16, s);
    if (update == kDecay) {
        if (gate == kGateScalar) return launch_types<DK, kDecay, kGateScalar>(a, in_bf16, out_bf16, s);
        return launch_types<DK, kDecay, kGateChannel>(a, in_bf16, out_bf16, s);
    }
    if (gate == kGateNone) return launch_types<DK, kDelta, kGateNone>(a, in_bf16, out_bf16, s);
    if (gate == kGateScalar) return launch_types<DK, kDelta, kGateScalar>(a, in_bf16, out_bf16, s);
    return launch_types<DK, kDelta, kGateChannel>(a, in_bf16, out_bf16, s);
}

__global__ void copy_state_kernel(const float *S0, float *ST, long n) {
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
        ST[i] = S0 ? S0[i] : 0.f;
}

}  // namespace
}  // namespace gdn

int gdn_launch_chunk_simt(const gdn::ChunkArgs &a, int update, int gate, int in_bf16, int out_bf16,
                          cudaStream_t stream) {
    if (a.dk == 64) return gdn::launch_modes<64>(a, update, gate, in_bf16, out_bf16, stream);
    return gdn::launch_modes<128>(a, update, gate, in_bf16, out_bf16, stream);
}

int gdn_launch_copy_state(const float *S0, float *ST, long n, cudaStream_t stream) {
    if (n <= 0 || ST == nullptr || ST == S0) return 0;
    long blocks = (n + 255) / 256;
    if (blocks > gdn::gdn_sm_count() * 16L) blocks = gdn::gdn_sm_count() * 16L;
    gdn::copy_state_kernel<<<(unsigned)blocks, 256, 0, stream>>>(S0, ST, n);
    return (int)cudaGetLastError();
}
