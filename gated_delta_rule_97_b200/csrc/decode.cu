// Decode: T (>= 1, small) recurrent steps per (b,h), state updated in place.
//
// Bandwidth-bound rank-1 update ("Linear Attention, Visualized", "Optional:
// Linear attention as an RNN"; per-token recurrences of the Mamba-2, DeltaNet,
// GDN, GLA and KDA sections).  One token per call: each warp owns kRowsPerWarp
// consecutive rows of one head's state; lane l holds columns [l*V, l*V+V) of a row (V = dk/32, one
// 16-byte load for dk = 128).  Per row i, with a = exp(g):
//   p_i = sum_j S_ij a_j k_j,  r_i = sum_j S_ij a_j q_j      (two warp sums)
//   u_i = beta (v_i - p_i) (delta) or v_i,
//   S_ij <- S_ij a_j + u_i k_j,  o_i = r_i + u_i (k . q).
// The state is streamed once in and once out with evict-first hints; rows are
// independent, so there is no inter-warp synchronisation.
#include "common.cuh"
#include "sm100.cuh"

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
// T > 1 tokens per call.  Persistent warps take tasks of kMRows consecutive
// state rows of one head in a grid-stride loop.  A task's rows reach a
// per-warp shared slot by one bulk copy issued kMSlots tasks ahead, so the
// state stream runs while the warp updates the rows it holds in registers over
// the T tokens; they are then streamed back with evict-first stores.
//
// Lane 8 rg + cg holds rows 4 rg .. 4 rg + 3 of the task and, per 32-column
// block m, columns 32 m + 4 cg .. 32 m + 4 cg + 3.  The q / k values a lane
// loads and converts serve its four rows; the eight per-row sums (S k and S q
// of four rows) are reduced over the eight lanes of a row group by a
// transposing butterfly (7 shuffles, after which lane cg holds sum number cg);
// a scalar gate is carried as one factor c (the true state is c times the held
// one), so it costs no per-element multiply.
constexpr int kMRows = 16;   // rows per task
constexpr int kMWarps = 4;   // warps per block
constexpr int kMSlots = 2;   // state slots per warp (bulk copies in flight)

template <typename TIn, int NC>
struct QKRaw;
template <int NC>
struct QKRaw<__nv_bfloat16, NC> {  // four bf16 per 32-column block
    uint2 w[NC];
    __device__ void load(const __nv_bfloat16 *p) {
#pragma unroll
        for (int m = 0; m < NC; ++m) w[m] = *reinterpret_cast<const uint2 *>(p + 32 * m);
    }
    __device__ void unpack(float *x) const {
#pragma unroll
        for (int m = 0; m < NC; ++m) {
            x[4 * m] = __uint_as_float(w[m].x << 16);
            x[4 * m + 1] = __uint_as_float(w[m].x & 0xffff0000u);
            x[4 * m + 2] = __uint_as_float(w[m].y << 16);
            x[4 * m + 3] = __uint_as_float(w[m].y & 0xffff0000u);
        }
    }
};
template <int NC>
struct QKRaw<float, NC> {
    float4 w[NC];
    __device__ void load(const float *p) {
#pragma unroll
        for (int m = 0; m < NC; ++m) w[m] = *reinterpret_cast<const float4 *>(p + 32 * m);
    }
    __device__ void unpack(float *x) const {
#pragma unroll
        for (int m = 0; m < NC; ++m) {
            x[4 * m] = w[m].x; x[4 * m + 1] = w[m].y; x[4 * m + 2] = w[m].z; x[4 * m + 3] = w[m].w;
        }
    }
};

// One token's inputs as this lane needs them (raw, so the next token's loads
// can be in flight while the current one is applied).
template <int DK, int GATE, typename TIn>
struct TokRaw {
    static constexpr int NC = DK / 32;
    QKRaw<TIn, NC> q, k;
    float4 gc[GATE == kGateChannel ? NC : 1];
    float gs, bt, vi;
    __device__ void load(const DecodeArgs &a, long tok, int col, int row) {
        const TIn *qp = static_cast<const TIn *>(a.q) + tok * DK + col;
        const TIn *kp = static_cast<const TIn *>(a.k) + tok * DK + col;
        q.load(qp);
        k.load(kp);
        if (GATE == kGateChannel) {
#pragma unroll
            for (int m = 0; m < NC; ++m) gc[m] = *reinterpret_cast<const float4 *>(a.g + tok * DK + col + 32 * m);
        }
        gs = (GATE == kGateScalar) ? a.g[tok] : 0.f;
        bt = a.beta ? a.beta[tok] : 0.f;
        vi = to_f32(static_cast<const TIn *>(a.v)[tok * a.dv + row]);
    }
};

// x[0..7] summed over the eight lanes of a row group; lane cg gets sum number cg.
__device__ __forceinline__ float transpose_sum8(const float (&x)[8], int cg) {
    const bool b2 = cg & 4, b1 = cg & 2, b0 = cg & 1;
    float y4[4], y2[2];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float send = b2 ? x[j] : x[j + 4], keep = b2 ? x[j + 4] : x[j];
        y4[j] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const float send = b1 ? y4[j] : y4[j + 2], keep = b1 ? y4[j + 2] : y4[j];
        y2[j] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    const float send = b0 ? y2[0] : y2[1], keep = b0 ? y2[1] : y2[0];
    return keep + __shfl_xor_sync(0xffffffffu, send, 1);
}

template <int DK, int UPD, int GATE, typename TIn, typename TOut, bool PRO>
__global__ void __launch_bounds__(kMWarps * 32, 3) decode_multi_kernel(DecodeArgs a, long ntasks) {
    using namespace sm100;
    constexpr int NC = DK / 32;               // 32-column blocks
    constexpr int NE = 4 * NC;                // columns per lane and row
    constexpr int SLOT = kMRows * DK * 4;     // bytes of one task's rows
    extern __shared__ __align__(128) unsigned char dsm[];
    __shared__ uint64_t bars[kMWarps][kMSlots];
    const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rg = lane >> 3, cg = lane & 7;
    const int col = 4 * cg;
    const int pro = PRO ? a.pro : 0;
    float *slots = reinterpret_cast<float *>(dsm) + (size_t)wib * kMSlots * (SLOT / 4);
    uint64_t *bar = bars[wib];
    const long nwarps = (long)gridDim.x * kMWarps;
    const long w0 = (long)blockIdx.x * kMWarps + wib;
    const int bpr = a.dv / kMRows;  // tasks per head
    const uint64_t wlim = a.wait_ns ? a.wait_ns : 1000000000ull;

    auto issue = [&](long task, int sl) {
        if (lane == 0) {
            const long bh = task / bpr;
            const int i0 = (int)(task - bh * bpr) * kMRows;
            mbar_arrive_expect_tx(&bar[sl], SLOT);
            sm100::bulk_load(slots + sl * (SLOT / 4), a.S + ((size_t)bh * a.dv + i0) * DK, SLOT, &bar[sl]);
            // the task's token inputs, so that its per-token loads hit L2 (the first
            // row block of a head asks for them; the others find them there)
            if (i0 == 0) {
                const size_t tq = (size_t)bh * a.T * DK * sizeof(TIn), nq = (size_t)a.T * DK * sizeof(TIn);
                sm100::bulk_prefetch_l2(static_cast<const char *>(a.q) + tq, (uint32_t)nq);
                sm100::bulk_prefetch_l2(static_cast<const char *>(a.k) + tq, (uint32_t)nq);
                sm100::bulk_prefetch_l2(static_cast<const char *>(a.v) + (size_t)bh * a.T * a.dv * sizeof(TIn),
                                        (uint32_t)((size_t)a.T * a.dv * sizeof(TIn)));
                if (GATE == kGateChannel) sm100::bulk_prefetch_l2(a.g + (size_t)bh * a.T * DK, (uint32_t)nq / sizeof(TIn) * 4);
                if (GATE == kGateScalar) sm100::prefetch_l2(a.g + (size_t)bh * a.T);
                if (a.beta) sm100::prefetch_l2(a.beta + (size_t)bh * a.T);
            }
        }
    };
    if (lane == 0) {
#pragma unroll
        for (int sl = 0; sl < kMSlots; ++sl) mbar_init(&bar[sl], 1);
        fence_mbar_init();
    }
    __syncwarp();
#pragma unroll
    for (int sl = 0; sl < kMSlots; ++sl)
        if (w0 + sl * nwarps < ntasks) issue(w0 + sl * nwarps, sl);

    int it = 0;
    for (long task = w0; task < ntasks; task += nwarps, ++it) {
        const int sl = it % kMSlots;
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar[sl], (it / kMSlots) & 1, wlim));
        if (!ok) {
            // give up: record it, let the copies still in flight land (bounded), leave
            record_status(a.status, kStatusTimeout);
            for (int k = 0; k < kMSlots; ++k) {
                const long t2 = task + k * nwarps;
                if (t2 < ntasks) mbar_wait(&bar[(it + k) % kMSlots], ((it + k) / kMSlots) & 1);
            }
            return;
        }
        const long bh = task / bpr;
        const int i0 = (int)(task - bh * bpr) * kMRows;
        float s[4][NE];
        {
            const float *src = slots + sl * (SLOT / 4);
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int m = 0; m < NC; ++m) {
                    const float4 x = *reinterpret_cast<const float4 *>(src + (4 * rg + j) * DK + 32 * m + col);
                    s[j][4 * m] = x.x; s[j][4 * m + 1] = x.y; s[j][4 * m + 2] = x.z; s[j][4 * m + 3] = x.w;
                }
        }
        __syncwarp();
        if (task + kMSlots * nwarps < ntasks) {
            if (lane == 0) fence_proxy_async_smem();
            issue(task + kMSlots * nwarps, sl);
        }

        const int vrow = i0 + 4 * rg + (cg & 3);  // the row whose S k sum this lane ends with
        TokRaw<DK, GATE, TIn> nxt;
        nxt.load(a, bh * a.T, col, vrow);
        float c = 1.f;  // scalar gate: the true state is c * s
#pragma unroll 1
        for (int t = 0; t < a.T; ++t) {
            const long tok = bh * a.T + t;
            const TokRaw<DK, GATE, TIn> cur = nxt;
            if (t + 1 < a.T) nxt.load(a, tok + 1, col, vrow);
            float qq[NE], kk[NE];
            cur.q.unpack(qq);
            cur.k.unpack(kk);
            if (pro) {
#pragma unroll
                for (int e = 0; e < NE; ++e) {
                    qq[e] = pro_feature(qq[e], pro);
                    kk[e] = pro_feature(kk[e], pro);
                }
                if (pro & kProL2) {  // unit q and k rows; a zero row stays zero
                    float sq = 0.f, sk = 0.f;
#pragma unroll
                    for (int e = 0; e < NE; ++e) {
                        sq = fmaf(qq[e], qq[e], sq);
                        sk = fmaf(kk[e], kk[e], sk);
                    }
#pragma unroll
                    for (int off = 1; off < 8; off <<= 1) {
                        sq += __shfl_xor_sync(0xffffffffu, sq, off);
                        sk += __shfl_xor_sync(0xffffffffu, sk, off);
                    }
                    const float iq = sq > 0.f ? 1.f / sqrtf(sq) : 0.f, ik = sk > 0.f ? 1.f / sqrtf(sk) : 0.f;
#pragma unroll
                    for (int e = 0; e < NE; ++e) {
                        qq[e] *= iq;
                        kk[e] *= ik;
                    }
                }
            }
            if (GATE == kGateChannel) {
#pragma unroll
                for (int m = 0; m < NC; ++m) {
                    const float gm[4] = {cur.gc[m].x, cur.gc[m].y, cur.gc[m].z, cur.gc[m].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float al = __expf(pro_gate(gm[e], pro));
#pragma unroll
                        for (int j = 0; j < 4; ++j) s[j][4 * m + e] *= al;
                    }
                }
            } else if (GATE == kGateScalar) {
                c *= __expf(pro_gate(cur.gs, pro));
                if (c < 0x1p-64f) {  // fold a deep decay into the held rows (same on every lane)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
#pragma unroll
                        for (int e = 0; e < NE; ++e) s[j][e] *= c;
                    c = 1.f;
                }
            }
            float kq = 0.f;
            float x[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float p = 0.f, r = 0.f;
#pragma unroll
                for (int e = 0; e < NE; ++e) {
                    if (UPD == kDelta) p = fmaf(s[j][e], kk[e], p);
                    r = fmaf(s[j][e], qq[e], r);
                }
                x[j] = p;
                x[4 + j] = r;
            }
#pragma unroll
            for (int e = 0; e < NE; ++e) kq = fmaf(kk[e], qq[e], kq);
            kq += __shfl_xor_sync(0xffffffffu, kq, 1);
            kq += __shfl_xor_sync(0xffffffffu, kq, 2);
            kq += __shfl_xor_sync(0xffffffffu, kq, 4);
            // lanes cg < 4: (S k) of row 4 rg + cg; lanes cg >= 4: (S q) of row 4 rg + cg - 4
            const float y = transpose_sum8(x, cg) * c;
            const float u = (UPD == kDelta) ? pro_beta(cur.bt, pro) * (cur.vi - y) : cur.vi;
            const float uo = __shfl_xor_sync(0xffffffffu, u, 4);
            if (cg >= 4) static_cast<TOut *>(a.o)[tok * a.dv + i0 + 4 * rg + cg - 4] = from_f32<TOut>(fmaf(uo, kq, y));
            const float ic = __frcp_rn(c);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float w = __shfl_sync(0xffffffffu, u, (lane & ~7) | j) * ic;
#pragma unroll
                for (int e = 0; e < NE; ++e) s[j][e] = fmaf(w, kk[e], s[j][e]);
            }
        }
        float *dst = a.S + ((size_t)bh * a.dv + i0 + 4 * rg) * DK + col;
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int m = 0; m < NC; ++m)
                __stcs(reinterpret_cast<float4 *>(dst + j * DK + 32 * m),
                       make_float4(s[j][4 * m] * c, s[j][4 * m + 1] * c, s[j][4 * m + 2] * c, s[j][4 * m + 3] * c));
    }
}

// Persistent grid: as many blocks as fit on the device at once (at most one
// warp per task).
template <int DK, int UPD, int GATE, typename TIn, typename TOut, bool PRO>
int launch_multi(const DecodeArgs &a, cudaStream_t stream) {
    constexpr int smem = kMWarps * kMSlots * kMRows * DK * 4;
    static int per_sm[64];  // resident blocks per SM, by device (0 = not yet known)
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return (int)cudaErrorInvalidDevice;
    auto kern = decode_multi_kernel<DK, UPD, GATE, TIn, TOut, PRO>;
    if (per_sm[dev] == 0) {
        int n = 0;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kMWarps * 32, smem) != cudaSuccess || n < 1)
            return (int)cudaErrorInvalidConfiguration;
        per_sm[dev] = n;
    }
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return (int)cudaErrorInvalidDevice;
    const long ntasks = (long)a.BH * (a.dv / kMRows);
    const long need = (ntasks + kMWarps - 1) / kMWarps;
    const long blocks = need < (long)sms * per_sm[dev] ? need : (long)sms * per_sm[dev];
    kern<<<(unsigned)blocks, kMWarps * 32, smem, stream>>>(a, ntasks);
    return (int)cudaGetLastError();
}

template <int DK, int UPD, int GATE, typename TIn, typename TOut>
int launch(const DecodeArgs &a, cudaStream_t stream) {
    const long rows = (long)a.BH * a.dv;
    const long warps = rows / kRowsPerWarp;
    const long blocks = (warps * 32 + kThreads - 1) / kThreads;
    if (blocks == 0) return 0;
    if (a.T > 1)
        return a.pro ? launch_multi<DK, UPD, GATE, TIn, TOut, true>(a, stream)
                     : launch_multi<DK, UPD, GATE, TIn, TOut, false>(a, stream);
    if (a.pro) {
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
