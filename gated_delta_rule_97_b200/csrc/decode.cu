// Decode: T (>= 1, small) recurrent steps per (b,h), state updated in place.
//
// Bandwidth-bound rank-1 update ("Linear Attention, Visualized", "Optional:
// Linear attention as an RNN"; per-token recurrences of the Mamba-2, DeltaNet,
// GDN, GLA and KDA sections).  Each warp owns kRowsPerWarp consecutive rows of
// one head's state; lane l holds columns [l*V, l*V+V) of a row (V = dk/32, one
// 16-byte load for dk = 128).  Per row i, with a = exp(g):
//   p_i = sum_j S_ij a_j k_j,  r_i = sum_j S_ij a_j q_j      (two warp sums)
//   u_i = beta (v_i - p_i) (delta) or v_i,
//   S_ij <- S_ij a_j + u_i k_j,  o_i = r_i + u_i (k . q).
// The state is streamed once in and once out with evict-first hints; rows are
// independent, so there is no inter-warp synchronisation.
#include "common.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerWarp = 4;

template <int V>
struct VecF;
template <>
struct VecF<4> {
    using T = float4;
    __device__ static void load(const float *p, float *x) {
        const float4 t = __ldcs(reinterpret_cast<const float4 *>(p));
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    }
    __device__ static void store(float *p, const float *x) {
        __stcs(reinterpret_cast<float4 *>(p), make_float4(x[0], x[1], x[2], x[3]));
    }
};
template <>
struct VecF<2> {
    using T = float2;
    __device__ static void load(const float *p, float *x) {
        const float2 t = __ldcs(reinterpret_cast<const float2 *>(p));
        x[0] = t.x; x[1] = t.y;
    }
    __device__ static void store(float *p, const float *x) {
        __stcs(reinterpret_cast<float2 *>(p), make_float2(x[0], x[1]));
    }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// PRO: the input prologue is compiled in only when a call asks for it, so the
// plain path keeps its registers and straight-line loads.
template <int DK, int UPD, int GATE, typename TIn, bool PRO>
struct StepIn {
    static constexpr int V = DK / 32;
    float qq[V], kk[V], al[V], bt, vv[kRowsPerWarp];
    __device__ void load(const DecodeArgs &a, long bh, int t, int c0, int i0) {
        const int pro = PRO ? a.pro : 0;
        const long tok = bh * a.T + t;
        const TIn *qp = static_cast<const TIn *>(a.q) + tok * DK + c0;
        const TIn *kp = static_cast<const TIn *>(a.k) + tok * DK + c0;
#pragma unroll
        for (int e = 0; e < V; ++e) {
            qq[e] = pro_feature(to_f32(qp[e]), pro);
            kk[e] = pro_feature(to_f32(kp[e]), pro);
            al[e] = 1.f;
        }
        if (pro & kProL2) {
            // unit q and k rows (a zero row stays zero); every lane gets both sums
            float sq = 0.f, sk = 0.f;
#pragma unroll
            for (int e = 0; e < V; ++e) {
                sq = fmaf(qq[e], qq[e], sq);
                sk = fmaf(kk[e], kk[e], sk);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, off);
                sk += __shfl_xor_sync(0xffffffffu, sk, off);
            }
            const float iq = sq > 0.f ? 1.f / sqrtf(sq) : 0.f, ik = sk > 0.f ? 1.f / sqrtf(sk) : 0.f;
#pragma unroll
            for (int e = 0; e < V; ++e) {
                qq[e] *= iq;
                kk[e] *= ik;
            }
        }
        if (GATE == kGateScalar) {
            const float x = __expf(pro_gate(a.g[tok], pro));
#pragma unroll
            for (int e = 0; e < V; ++e) al[e] = x;
        } else if (GATE == kGateChannel) {
#pragma unroll
            for (int e = 0; e < V; ++e) al[e] = __expf(pro_gate(a.g[tok * DK + c0 + e], pro));
        }
        bt = (UPD == kDelta) ? pro_beta(a.beta[tok], pro) : 0.f;
        const TIn *vp = static_cast<const TIn *>(a.v) + tok * a.dv + i0;
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) vv[r] = to_f32(vp[r]);
    }
};

// T >= 1 tokens per call: the state rows stay in registers across the tokens
// (read and written once); the next token's inputs are loaded while the current
// one is applied.
template <int DK, int UPD, int GATE, typename TIn, typename TOut, bool PRO>
__global__ void __launch_bounds__(kThreads) decode_kernel(DecodeArgs a) {
    constexpr int V = DK / 32;
    const long warp = ((long)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long row0 = warp * kRowsPerWarp;
    if (row0 >= (long)a.BH * a.dv) return;
    const long bh = row0 / a.dv;
    const int i0 = (int)(row0 - bh * a.dv);
    const int c0 = lane * V;

    float *Srow = a.S + ((size_t)bh * a.dv + i0) * DK + c0;
    float s[kRowsPerWarp][V];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) VecF<V>::load(Srow + (size_t)r * DK, s[r]);

    StepIn<DK, UPD, GATE, TIn, PRO> cur, nxt;
    cur.load(a, bh, 0, c0, i0);
#pragma unroll 1
    for (int t = 0; t < a.T; ++t) {
        if (t + 1 < a.T) nxt.load(a, bh, t + 1, c0, i0);
        float kq = 0.f;
#pragma unroll
        for (int e = 0; e < V; ++e) kq = fmaf(cur.kk[e], cur.qq[e], kq);
        kq = warp_sum(kq);

        float outv[kRowsPerWarp];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            float p = 0.f, rr = 0.f;
#pragma unroll
            for (int e = 0; e < V; ++e) {
                s[r][e] *= cur.al[e];
                p = fmaf(s[r][e], cur.kk[e], p);
                rr = fmaf(s[r][e], cur.qq[e], rr);
            }
            // two independent butterfly sums, interleaved
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                p += __shfl_xor_sync(0xffffffffu, p, off);
                rr += __shfl_xor_sync(0xffffffffu, rr, off);
            }
            const float u = (UPD == kDelta) ? cur.bt * (cur.vv[r] - p) : cur.vv[r];
#pragma unroll
            for (int e = 0; e < V; ++e) s[r][e] = fmaf(u, cur.kk[e], s[r][e]);
            outv[r] = fmaf(u, kq, rr);
        }
        if (lane < kRowsPerWarp) {
            float x = outv[0];
#pragma unroll
            for (int r = 1; r < kRowsPerWarp; ++r)
                if (lane == r) x = outv[r];
            static_cast<TOut *>(a.o)[(bh * a.T + t) * a.dv + i0 + lane] = from_f32<TOut>(x);
        }
        cur = nxt;
    }
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) VecF<V>::store(Srow + (size_t)r * DK, s[r]);
}

// ---------------------------------------------------------------------------
// T > 1 tokens per call.  The single-token layout above spreads a row over the
// 32 lanes, so each row and token costs two 5-level butterflies: with several
// tokens the shuffles, not the state stream, set the time.  Here lane l owns
// columns [c0, c0 + E) of row l / 8 (E = dk / 8): the row sums take 3-level
// butterflies that reduce the warp's four rows at once (9 shuffles per token
// and warp instead of 45).  The state stays in registers across the tokens.
template <typename TIn, int N>
struct RowLoad;
template <int N>
struct RowLoad<__nv_bfloat16, N> {
    __device__ static void load(const __nv_bfloat16 *p, float *x) {
#pragma unroll
        for (int i = 0; i < N / 8; ++i) {
            const uint4 u = *reinterpret_cast<const uint4 *>(p + 8 * i);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                x[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
                x[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
            }
        }
    }
};
template <int N>
struct RowLoad<float, N> {
    __device__ static void load(const float *p, float *x) {
#pragma unroll
        for (int i = 0; i < N / 4; ++i) {
            const float4 f = *reinterpret_cast<const float4 *>(p + 4 * i);
            x[4 * i] = f.x; x[4 * i + 1] = f.y; x[4 * i + 2] = f.z; x[4 * i + 3] = f.w;
        }
    }
};

__device__ __forceinline__ float row_sum8(float x) {  // over the 8 lanes of a row group
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    return x;
}

template <int DK, int UPD, int GATE, typename TIn, typename TOut, bool PRO>
__global__ void __launch_bounds__(kThreads) decode_multi_kernel(DecodeArgs a) {
    constexpr int E = DK / 8;
    const long warp = ((long)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long row0 = warp * kRowsPerWarp;
    if (row0 >= (long)a.BH * a.dv) return;
    const long bh = row0 / a.dv;
    const int i = (int)(row0 - bh * a.dv) + (lane >> 3);  // this lane's state row
    const int c0 = (lane & 7) * E;
    const int pro = PRO ? a.pro : 0;

    float *Srow = a.S + ((size_t)bh * a.dv + i) * DK + c0;
    float s[E];
#pragma unroll
    for (int e = 0; e < E; e += 4) VecF<4>::load(Srow + e, s + e);

#pragma unroll 1
    for (int t = 0; t < a.T; ++t) {
        const long tok = bh * a.T + t;
        float qq[E], kk[E];
        RowLoad<TIn, E>::load(static_cast<const TIn *>(a.q) + tok * DK + c0, qq);
        RowLoad<TIn, E>::load(static_cast<const TIn *>(a.k) + tok * DK + c0, kk);
        const float vi = to_f32(static_cast<const TIn *>(a.v)[tok * a.dv + i]);
        const float bt = (UPD == kDelta) ? pro_beta(a.beta[tok], pro) : 0.f;
        if (pro) {
            float sq = 0.f, sk = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                qq[e] = pro_feature(qq[e], pro);
                kk[e] = pro_feature(kk[e], pro);
                sq = fmaf(qq[e], qq[e], sq);
                sk = fmaf(kk[e], kk[e], sk);
            }
            if (pro & kProL2) {  // unit q and k rows; a zero row stays zero
                sq = row_sum8(sq);
                sk = row_sum8(sk);
                const float iq = sq > 0.f ? 1.f / sqrtf(sq) : 0.f, ik = sk > 0.f ? 1.f / sqrtf(sk) : 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    qq[e] *= iq;
                    kk[e] *= ik;
                }
            }
        }
        float kq = 0.f, p = 0.f, rr = 0.f;
        if (GATE == kGateChannel) {
            float gg[E];
            RowLoad<float, E>::load(a.g + tok * DK + c0, gg);
#pragma unroll
            for (int e = 0; e < E; ++e) s[e] *= __expf(pro_gate(gg[e], pro));
        } else if (GATE == kGateScalar) {
            const float al = __expf(pro_gate(a.g[tok], pro));
#pragma unroll
            for (int e = 0; e < E; ++e) s[e] *= al;
        }
#pragma unroll
        for (int e = 0; e < E; ++e) {
            kq = fmaf(kk[e], qq[e], kq);
            p = fmaf(s[e], kk[e], p);
            rr = fmaf(s[e], qq[e], rr);
        }
        kq += __shfl_xor_sync(0xffffffffu, kq, 1);
        p += __shfl_xor_sync(0xffffffffu, p, 1);
        rr += __shfl_xor_sync(0xffffffffu, rr, 1);
        kq += __shfl_xor_sync(0xffffffffu, kq, 2);
        p += __shfl_xor_sync(0xffffffffu, p, 2);
        rr += __shfl_xor_sync(0xffffffffu, rr, 2);
        kq += __shfl_xor_sync(0xffffffffu, kq, 4);
        p += __shfl_xor_sync(0xffffffffu, p, 4);
        rr += __shfl_xor_sync(0xffffffffu, rr, 4);
        const float u = (UPD == kDelta) ? bt * (vi - p) : vi;
#pragma unroll
        for (int e = 0; e < E; ++e) s[e] = fmaf(u, kk[e], s[e]);
        if ((lane & 7) == 0) static_cast<TOut *>(a.o)[tok * a.dv + i] = from_f32<TOut>(fmaf(u, kq, rr));
    }
#pragma unroll
    for (int e = 0; e < E; e += 4) VecF<4>::store(Srow + e, s + e);
}

template <int DK, int UPD, int GATE, typename TIn, typename TOut>
int launch(const DecodeArgs &a, cudaStream_t stream) {
    const long rows = (long)a.BH * a.dv;
    const long warps = rows / kRowsPerWarp;
    const long blocks = (warps * 32 + kThreads - 1) / kThreads;
    if (blocks == 0) return 0;
    if (a.T > 1) {
        if (a.pro)
            decode_multi_kernel<DK, UPD, GATE, TIn, TOut, true><<<(unsigned)blocks, kThreads, 0, stream>>>(a);
        else
            decode_multi_kernel<DK, UPD, GATE, TIn, TOut, false><<<(unsigned)blocks, kThreads, 0, stream>>>(a);
    } else if (a.pro) {
        decode_kernel<DK, UPD, GATE, TIn, TOut, true><<<(unsigned)blocks, kThreads, 0, stream>>>(a);
    } else {
        decode_kernel<DK, UPD, GATE, TIn, TOut, false><<<(unsigned)blocks, kThreads, 0, stream>>>(a);
    }
    return (int)cudaGetLastError();
}

template <int DK, int UPD, int GATE>
int launch_types(const DecodeArgs &a, int in_bf16, int out_bf16, cudaStream_t s) {
    if (in_bf16)
        return out_bf16 ? launch<DK, UPD, GATE, __nv_bfloat16, __nv_bfloat16>(a, s)
                        : launch<DK, UPD, GATE, __nv_bfloat16, float>(a, s);
    return out_bf16 ? launch<DK, UPD, GATE, float, __nv_bfloat16>(a, s) : launch<DK, UPD, GATE, float, float>(a, s);
}

template <int DK>
int launch_modes(const DecodeArgs &a, int update, int gate, int in_bf16, int out_bf16, cudaStream_t s) {
    if (update == kAdditive) return launch_types<DK, kAdditive, kGateNone>(a, in_bf16, out_bf16, s);
    if (update == kDecay) {
        if (gate == kGateScalar) return launch_types<DK, kDecay, kGateScalar>(a, in_bf16, out_bf16, s);
        return launch_types<DK, kDecay, kGateChannel>(a, in_bf16, out_bf16, s);
    }
    if (gate == kGateNone) return launch_types<DK, kDelta, kGateNone>(a, in_bf16, out_bf16, s);
    if (gate == kGateScalar) return launch_types<DK, kDelta, kGateScalar>(a, in_bf16, out_bf16, s);
    return launch_types<DK, kDelta, kGateChannel>(a, in_bf16, out_bf16, s);
}

}  // namespace
}  // namespace gdn

int gdn_launch_decode(const gdn::DecodeArgs &a, int update, int gate, int in_bf16, int out_bf16,
                      cudaStream_t stream) {
    if (a.dk == 64) return gdn::launch_modes<64>(a, update, gate, in_bf16, out_bf16, stream);
    return gdn::launch_modes<128>(a, update, gate, in_bf16, out_bf16, stream);
}
