// Tensor-core (tcgen05 / TMEM / TMA) chunkwise prefill for bf16 inputs, dk = 128.
//
// One CTA (8 warps; warp w reads TMEM lane quarter w%4 and column half w/4)
// owns one (b,h) head and a slice of DVS value rows of its state, and walks
// the chunks of the sequence in order.  The state is kept TRANSPOSED in TMEM as an fp32 accumulator
// D_S = S^T [dk=128 lanes][DVS columns], so the per-key-channel decay
// S Diag(e^{G_C}) is a per-lane scale and the state update is one MMA.
//
// Per chunk r (C = 64), "Linear Attention, Visualized" -- "Chunkwise
// algorithm", "Mamba-2 ... Chunkwise form", "Gated Linear Attention (GLA)",
// "The triangular correction system", "Optional: Use UT to share the
// triangular transform", "Correct the incoming state", the GDN / KDA tables:
//   a1  G = inclusive prefix of g; Q< = q e^{G}, K< = k e^{G}, K> = k e^{G_C-G}
//   a2  P = [Q;K] K^T (bf16, scalar/no gate; Gamma applied per element) or
//       [Q<;K<] (k e^{-G})^T (fp16, per-channel gate, range-guarded);
//       A' = P_top masked (m<=l); L = beta_l P_bottom (m<l)
//   a3  T = (I + L)^{-1}: fp32 forward substitution, one column per thread,
//       written as the fp16 operand T2 = T diag(beta)
//   a4  D_W = [T2;0] K<,  D_ZO = [T2;0] V                    (MMA)
//   a5  D_ZO -= [W; -Q<] S^T  -> rows 0..63 = Z = U - W S^T   (MMA, A negated)
//   a6  D_ZO += [0; A'] Z     -> rows 64..127 = O             (MMA)
//   a7  D_S = e^{G_C} D_S + K>^T Z                            (scale + MMA)
// Operands that are intermediates (T2, W, Q<, K<, K>, A', Z, S^T) are fp16
// (11-bit significand); raw bf16 inputs are exact in fp16.  Accumulators and
// the state master are fp32.  Additive / decay modes skip a3-a5 (Z = V).
// An fp16 overflow of an operand is recorded as GDN_ERR_RANGE in the device
// status word.  All waits are bounded; on a timeout the CTA records
// GDN_ERR_TIMEOUT, frees its TMEM and returns.
#include <string.h>

#include "../../include/gdn.h"
#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

#ifdef GDN_TC_PHASE_TIMING
// Per-phase cycle totals of CTA 0 (profiling builds only).
__device__ unsigned long long g_tc_phase[16];
#define TC_MARK(i)                                                              \
    do {                                                                       \
        if (blockIdx.x == 0 && t == 0) {                                       \
            const long long now_ = clock64();                                  \
            atomicAdd(&g_tc_phase[i], (unsigned long long)(now_ - mark_prev)); \
            mark_prev = now_;                                                  \
        }                                                                      \
    } while (0)
#else
#define TC_MARK(i) \
    do {           \
    } while (0)
#endif

namespace gdn {
namespace {

using namespace sm100;

constexpr int kTcThreads = 256;
constexpr int C = kChunk;  // 64
constexpr int DK = 128;
// Largest per-channel decay (nats) inside one chunk for which the factored
// fp16 operands q e^{G}, k e^{-G} stay in range; beyond it the chunk's A' and
// L are computed exactly in fp32 SIMT.
constexpr float kFactorMaxDecay = 10.0f;

struct TcParams {
    CUtensorMap q_map, k_map, v_map, g_map;  // 3-D maps (zero fill past T)
    const float *g;      // scalar gate [BH,T] (channel gate uses g_map)
    const float *beta;   // [BH,T]
    const float *S0;     // [BH,dv,dk] or null
    void *o;             // [BH,T,dv]
    float *ST;           // [BH,dv,dk] or null
    int *status;
    int *diag;           // first timeout: 1 + site * 1e6 + chunk
    int BH, T, dv, nslices;
};

template <int DVS, int GATE>
struct TcSmem {
    static constexpr int RAW_QK = 0;                                   // [Q0 K0 | Q1 K1] bf16, 32 KB
    static constexpr int RAW_V = RAW_QK + 32768;                       // V slice bf16, DVS/64 x 8 KB
    static constexpr int GCH = RAW_V + DVS * 128;                      // channel gate fp32 [64][128]
    static constexpr int AT = GCH + (GATE == kGateChannel ? 32768 : 0);  // [-W | Q< | K<] x 2 halves
    static constexpr int KT = AT + 49152;                              // k e^{-G} (fp16) / L scratch (fp32)
    static constexpr int KR = KT + 16384;                              // K> fp16
    static constexpr int V16 = KR + 16384;                             // V fp16
    static constexpr int TZA = V16 + DVS * 128;                        // [T2 | 0 | A'] fp16, 24 KB
    static constexpr int ZT = TZA + 24576;                             // Z fp16 [64][DVS]
    static constexpr int ST16 = ZT + DVS * 128;                        // S^T fp16 [128][DVS]
    static constexpr int MISC = ST16 + DVS * 256;                      // small arrays + barriers
    static constexpr int MISC_BYTES = 3072;
    static constexpr int TOTAL = MISC + MISC_BYTES;
    static constexpr int DYN = TOTAL + 1024;  // alignment slack
};

// Misc region (floats unless noted): G[64], gamma[64] (e^{G_C-G}), b[64], beta[64],
// GC[128] (e^{G_C} per channel), then flags and barriers.
struct Misc {
    float G[64];
    float gam[64];
    float b[64];
    float beta[64];
    float ib[64];
    float GC[128];
    int abort_flag;
    int range_flag;
    int slow_chunk;
    int abort_site;
    uint32_t tmem_base;
    uint32_t pad1[3];
    uint64_t bar_tma;
    uint64_t bar_p1;
    uint64_t bar_w;
    uint64_t bar_1;
    uint64_t bar_2;
};

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ void unpack_bf16x8(uint4 u, float *f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint4 pack_h8(const float *f) {
    return make_uint4(pack_h2(f[0], f[1]), pack_h2(f[2], f[3]), pack_h2(f[4], f[5]), pack_h2(f[6], f[7]));
}

// Float offset of element (r, c) in a row-major fp32 tile with `ld` columns
// whose 16-byte slots are XOR-swizzled by (r % 8): conflict-free for one row
// per thread writing float4s and for float4 reads of a shared row.
__device__ __forceinline__ int f32_swz(int r, int c, int ld) {
    return r * ld + ((((c >> 2) ^ (r & 7))) << 2) + (c & 3);
}

// Marks the CTA aborted and remembers the first wait that gave up (site, chunk).
template <typename M>
__device__ __forceinline__ void note_timeout(M &ms, int site, int r) {
    if (atomicCAS(&ms.abort_flag, 0, 1) == 0) ms.abort_site = site * 1000000 + r;
}

__device__ __forceinline__ bool out_of_fp16(float x) { return !(fabsf(x) <= 65504.f) && x == x; }

template <int DVS, int UPD, int GATE, bool OUT_BF16>
__global__ void __launch_bounds__(kTcThreads, 1) chunk_tc_kernel(const __grid_constant__ TcParams p) {
    using L = TcSmem<DVS, GATE>;
    constexpr bool DELTA = (UPD == kDelta);
    constexpr int NB = DVS / 64;  // 64-wide value blocks
    constexpr int HV = DVS / 2;   // value columns per column half
    extern __shared__ unsigned char smraw[];
    // Align by an integer offset from the shared array itself, so that every access
    // through `sm` stays in the shared address space (LDS/STS, not generic).
    unsigned char *sm = smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);
    Misc &ms = *reinterpret_cast<Misc *>(sm + L::MISC);

    const int t = threadIdx.x;
    const int warp = t >> 5, lane = t & 31;
    const int sp = warp & 3;          // TMEM lane quarter this warp may access
    const int ch = warp >> 2;         // column half handled by this warp
    const int row = sp * 32 + lane;   // accumulator row (TMEM lane) of this thread
    const int bh = blockIdx.x / p.nslices;
    const int v0 = (blockIdx.x % p.nslices) * DVS;
    const int T = p.T, dv = p.dv;
    const int nchunks = (T + C - 1) / C;

    // ------------------------------------------------------------ setup
    if (t == 0) {
        mbar_init(&ms.bar_tma, 1);
        mbar_init(&ms.bar_p1, 1);
        mbar_init(&ms.bar_w, 1);
        mbar_init(&ms.bar_1, 1);
        mbar_init(&ms.bar_2, 1);
        fence_mbar_init();
        ms.abort_flag = 0;
        ms.range_flag = 0;
        tma_prefetch_desc(&p.q_map);
        tma_prefetch_desc(&p.k_map);
        tma_prefetch_desc(&p.v_map);
        if (GATE == kGateChannel) tma_prefetch_desc(&p.g_map);
    }
    __syncwarp();
    if (warp == 0) {
        tmem_alloc(&ms.tmem_base, 512);
        tmem_relinquish();
    }
    // T2 block (its upper-right 32x32 block stays zero) and the zero block of [0; A']
    for (int i = t; i < 8192 / 16; i += kTcThreads) {
        reinterpret_cast<uint4 *>(sm + L::TZA)[i] = make_uint4(0, 0, 0, 0);
        reinterpret_cast<uint4 *>(sm + L::TZA + 8192)[i] = make_uint4(0, 0, 0, 0);
        if (!DELTA) {  // the W rows of [W; -Q<] are read but must contribute nothing
            reinterpret_cast<uint4 *>(sm + L::AT)[i] = make_uint4(0, 0, 0, 0);
            reinterpret_cast<uint4 *>(sm + L::AT + 24576)[i] = make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms.tmem_base;
    const uint32_t t_lane = tmem + ((uint32_t)(sp * 32) << 16);
    const uint32_t TM_P = 0, TM_W = 64, TM_ZO = 192, TM_S = 192 + DVS;

    auto issue_tma = [&](int r) {
        const int t0 = r * C;
        uint32_t bytes = 32768 + DVS * 128 + (GATE == kGateChannel ? 32768 : 0);
        mbar_arrive_expect_tx(&ms.bar_tma, bytes);
        for (int h = 0; h < 2; ++h) {
            tma_load_3d(sm + L::RAW_QK + h * 16384, &p.q_map, h * 64, t0, bh, &ms.bar_tma);
            tma_load_3d(sm + L::RAW_QK + h * 16384 + 8192, &p.k_map, h * 64, t0, bh, &ms.bar_tma);
        }
        for (int j = 0; j < NB; ++j) tma_load_3d(sm + L::RAW_V + j * 8192, &p.v_map, v0 + j * 64, t0, bh, &ms.bar_tma);
        if (GATE == kGateChannel)
            for (int j = 0; j < 4; ++j) tma_load_3d(sm + L::GCH + j * 8192, &p.g_map, j * 32, t0, bh, &ms.bar_tma);
    };
    if (t == 0 && nchunks > 0) issue_tma(0);
    // gate and beta of a chunk are loaded one chunk ahead into registers
    float gpre0 = 0.f, gpre1 = 0.f, bpre = 0.f;
    auto load_gate_beta = [&](int r) {
        const int t0 = r * C;
        if (GATE == kGateScalar && warp == 0) {
            const int l0 = 2 * lane;
            gpre0 = (t0 + l0 < T) ? p.g[(size_t)bh * T + t0 + l0] : 0.f;
            gpre1 = (t0 + l0 + 1 < T) ? p.g[(size_t)bh * T + t0 + l0 + 1] : 0.f;
        }
        if (DELTA && t < C) bpre = (t0 + t < T) ? p.beta[(size_t)bh * T + t0 + t] : 0.f;
    };
    if (nchunks > 0) load_gate_beta(0);

    // initial state: lane `row` = key channel; this warp's column half of S^T
    for (int j0 = ch * HV; j0 < ch * HV + HV; j0 += 16) {
        float sv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) sv[i] = p.S0 ? p.S0[((size_t)bh * dv + v0 + j0 + i) * DK + row] : 0.f;
        __syncwarp();
        tmem_st16(t_lane + TM_S + j0, sv);
#pragma unroll
        for (int i = 0; i < 16; i += 8) {
            const int j = j0 + i;
            *reinterpret_cast<uint4 *>(sm + L::ST16 + (j >> 6) * 16384 + sw128_off(row, j & 63)) = pack_h8(sv + i);
        }
    }
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

#ifdef GDN_TC_PHASE_TIMING
    long long mark_prev = clock64();
#endif
    bool ok = true;
    float rmax = 0.f;  // largest |value| this thread handed to an fp16 operand (range check)
    for (int r = 0; r < nchunks && ok; ++r) {
        const uint32_t ph = r & 1;
        const int t0 = r * C;
        const int n = min(C, T - t0);
        // ---------------------------------------------------- wait for inputs
        TC_MARK(0);
        if (!mbar_wait(&ms.bar_tma, ph)) note_timeout(ms, 1, r);
        TC_MARK(1);
        // scalar / no gate: P = [Q;K] K^T straight from the bf16 tiles
        if (GATE != kGateChannel && t == 0 && !ms.abort_flag) {
            tc_fence_after();
            const uint32_t qk = smem_u32(sm + L::RAW_QK);
            constexpr uint32_t id = idesc_f16(128, 64, 1, 0, 0);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t ko = (k >> 2) * 16384 + (k & 3) * 32;
                mma_f16(tmem + TM_P, smem_desc_sw128(qk + ko, 16, 1024), smem_desc_sw128(qk + 8192 + ko, 16, 1024), id,
                        k > 0);
            }
            mma_commit(&ms.bar_p1);
        }
        // ---------------------------------------------------- a1: gate prefix
        if (GATE == kGateScalar) {
            if (warp == 0) {
                const int l0 = 2 * lane;
                const float x0 = gpre0, x1 = gpre1;
                float s = x0 + x1;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, s, off);
                    if (lane >= off) s += y;
                }
                const float e = s - (x0 + x1);
                ms.G[l0] = e + x0;
                ms.G[l0 + 1] = e + x0 + x1;
            }
        } else if (GATE == kGateChannel) {
            // channel c = t & 127, token half hf = t >> 7: prefix over 32 tokens, then join
            const int c = t & 127, hf = t >> 7;
            float *gcol = reinterpret_cast<float *>(sm + L::GCH + (c >> 5) * 8192) + (c & 31);
            float s = 0.f;
#pragma unroll 8
            for (int l = 32 * hf; l < 32 * hf + 32; ++l) {
                s += gcol[l * 32];
                gcol[l * 32] = s;
            }
            __syncthreads();
            if (hf == 1) {
                const float base = gcol[31 * 32];
#pragma unroll 8
                for (int l = 32; l < 64; ++l) gcol[l * 32] += base;
                ms.GC[c] = s + base;
            }
        }
        if (DELTA && t < C) ms.beta[t] = bpre;
        if (r + 1 < nchunks) load_gate_beta(r + 1);  // consumed next chunk; latency hidden
        __syncthreads();
        bool fastg = true;  // scalar gate: decay factors as b_l / b_m (chunk decay <= 80 nats)
        if (GATE == kGateScalar) {
            const float gc = ms.G[C - 1];
            fastg = -gc <= 80.f;
            if (t < C) {
                const float G = ms.G[t];
                ms.b[t] = __expf(G);
                ms.gam[t] = __expf(gc - G);
                ms.ib[t] = __expf(-G);
            }
        }
        if (GATE == kGateChannel && warp == 0) {
            float mx = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) mx = fmaxf(mx, -ms.GC[lane + 32 * i]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            if (lane == 0) ms.slow_chunk = !(mx <= kFactorMaxDecay);
        }
        // scale the state by the chunk's total decay: D_S <- e^{G_C} D_S (lane = channel)
        if (GATE != kGateNone) {
            const float dec = (GATE == kGateScalar) ? __expf(ms.G[C - 1]) : __expf(ms.GC[row]);
#pragma unroll
            for (int j0 = 0; j0 < HV; j0 += 32) {
                float sv[32];
                __syncwarp();
                tmem_ld32(t_lane + TM_S + ch * HV + j0, sv);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) sv[i] *= dec;
                tmem_st16(t_lane + TM_S + ch * HV + j0, sv);
                tmem_st16(t_lane + TM_S + ch * HV + j0 + 16, sv + 16);
            }
            tmem_wait_st();
        }
        __syncthreads();

        TC_MARK(2);
        // ---------------------------------------------------- operand conversions
        // Each 16-byte chunk of a 128B-swizzled [64][64] box holds 8 consecutive
        // channels of one token row; the same offset addresses the same element in
        // every tile that shares the layout.  Q< is stored negated: the history
        // MMA negates its A operand [W; -Q<].
        const bool slow = (GATE == kGateChannel) && ms.slow_chunk;
        for (int i = t; i < 2 * 512; i += kTcThreads) {
            const int h = i >> 9, off = (i & 511) * 16;
            const int l = off >> 7;
            const int c0 = h * 64 + ((((off >> 4) & 7) ^ (l & 7)) << 3);
            float qf[8], kf[8], ql[8], kl[8], kr[8];
            unpack_bf16x8(*reinterpret_cast<const uint4 *>(sm + L::RAW_QK + h * 16384 + off), qf);
            unpack_bf16x8(*reinterpret_cast<const uint4 *>(sm + L::RAW_QK + h * 16384 + 8192 + off), kf);
#pragma unroll
            for (int e = 0; e < 8; ++e) rmax = fmaxf(rmax, fmaxf(fabsf(qf[e]), fabsf(kf[e])));
            if (GATE == kGateChannel) {
                const float *gg = reinterpret_cast<const float *>(sm + L::GCH + (c0 >> 5) * 8192) + l * 32 + (c0 & 31);
                float kt[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float G = gg[e];
                    const float eg = __expf(G), emg = __expf(-G);
                    ql[e] = -qf[e] * eg;
                    kl[e] = kf[e] * eg;
                    kt[e] = slow ? 0.f : kf[e] * emg;  // factored fast path only
                    kr[e] = kf[e] * __expf(ms.GC[c0 + e] - G);
                    rmax = fmaxf(rmax, fabsf(kt[e]));
                }
                *reinterpret_cast<uint4 *>(sm + L::KT + h * 8192 + off) = pack_h8(kt);
            } else {
                const float bl = (GATE == kGateScalar) ? ms.b[l] : 1.f;
                const float gl = (GATE == kGateScalar) ? ms.gam[l] : 1.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    ql[e] = -qf[e] * bl;
                    kl[e] = kf[e] * bl;
                    kr[e] = kf[e] * gl;
                }
            }
            *reinterpret_cast<uint4 *>(sm + L::AT + h * 24576 + 8192 + off) = pack_h8(ql);
            if (DELTA) *reinterpret_cast<uint4 *>(sm + L::AT + h * 24576 + 16384 + off) = pack_h8(kl);
            *reinterpret_cast<uint4 *>(sm + L::KR + h * 8192 + off) = pack_h8(kr);
        }
        for (int i = t; i < NB * 512; i += kTcThreads) {
            float vf[8];
            unpack_bf16x8(*reinterpret_cast<const uint4 *>(sm + L::RAW_V + i * 16), vf);
            *reinterpret_cast<uint4 *>(sm + L::V16 + i * 16) = pack_h8(vf);
#pragma unroll
            for (int e = 0; e < 8; ++e) rmax = fmaxf(rmax, fabsf(vf[e]));
        }
        fence_proxy_async_smem();
        __syncthreads();
        // per-channel gate: P = [-Q<; K<] (k e^{-G})^T on fp16 operands
        if (GATE == kGateChannel && t == 0) {
            tc_fence_after();
            const uint32_t at = smem_u32(sm + L::AT), kt = smem_u32(sm + L::KT);
            constexpr uint32_t id = idesc_f16(128, 64, 0, 0, 0);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t ka = (k >> 2) * 24576 + 8192 + (k & 3) * 32;
                const uint32_t kb = (k >> 2) * 8192 + (k & 3) * 32;
                mma_f16(tmem + TM_P, smem_desc_sw128(at + ka, 16, 1024), smem_desc_sw128(kt + kb, 16, 1024), id, k > 0);
            }
            mma_commit(&ms.bar_p1);
        }
        TC_MARK(3);
        if (!mbar_wait(&ms.bar_p1, ph)) note_timeout(ms, 2, r);
        TC_MARK(4);
        tc_fence_after();

        // ---------------------------------------------------- a2: A' and L
        {
            const int l = row & 63;
            const bool top = row < 64;
            const int m0 = ch * 32;  // this warp's 32 columns
            float pr[32];
            __syncwarp();
            tmem_ld32(t_lane + TM_P + m0, pr);
            tmem_wait_ld();
            TC_MARK(15);
            if (GATE == kGateChannel && slow) {
                // exact fp32: sum_c x_lc k_mc e^{G_lc - G_mc}
                const unsigned char *xrow = sm + L::RAW_QK + (top ? 0 : 8192);
                for (int e = 0; e < 32; ++e) {
                    const int m = m0 + e;
                    float acc = 0.f;
                    if (m <= l) {
                        for (int c = 0; c < DK; ++c) {
                            const int h = c >> 6;
                            const uint32_t ox = sw128_off(l, c & 63), om = sw128_off(m, c & 63);
                            const float xv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(xrow + h * 16384 + ox));
                            const float kv = __bfloat162float(
                                *reinterpret_cast<const __nv_bfloat16 *>(sm + L::RAW_QK + h * 16384 + 8192 + om));
                            const float *gc = reinterpret_cast<const float *>(sm + L::GCH + (c >> 5) * 8192);
                            acc = fmaf(xv * kv, __expf(gc[l * 32 + (c & 31)] - gc[m * 32 + (c & 31)]), acc);
                        }
                    }
                    pr[e] = acc;
                }
            } else if (GATE == kGateChannel && top) {
#pragma unroll
                for (int e = 0; e < 32; ++e) pr[e] = -pr[e];  // the factored product used -Q<
            }
            float dec[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int m = m0 + e;
                float d = 1.f;
                if (GATE == kGateScalar) d = fastg ? ms.b[l] * ms.ib[m] : __expf(ms.G[l] - ms.G[m < l ? m : l]);
                dec[e] = d;
            }
            if (top) {
                // A'[l][m] (m <= l) -> fp16, row 64+l of [0; A'] (K-major, K = 64)
#pragma unroll
                for (int e0 = 0; e0 < 32; e0 += 8) {
                    float a[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int m = m0 + e0 + e;
                        a[e] = (m <= l) ? pr[e0 + e] * dec[e0 + e] : 0.f;
                        rmax = fmaxf(rmax, fabsf(a[e]));
                    }
                    *reinterpret_cast<uint4 *>(sm + L::TZA + 16384 + sw128_off(l, m0 + e0)) = pack_h8(a);
                }
            } else if (DELTA) {
                // L[l][m] = beta_l * P[l][m] (m < l), fp32, swizzled rows
                const float bl = ms.beta[l];
                float *Ls = reinterpret_cast<float *>(sm + L::KT);
#pragma unroll
                for (int e0 = 0; e0 < 32; e0 += 4) {
                    float4 v;
                    float *vv = &v.x;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int m = m0 + e0 + e;
                        vv[e] = (m < l) ? bl * pr[e0 + e] * dec[e0 + e] : 0.f;
                    }
                    *reinterpret_cast<float4 *>(Ls + f32_swz(l, m0 + e0, 64)) = v;
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        TC_MARK(5);
        // the raw stage is consumed (P, conversions, exact path): prefetch the next chunk
        if (t == 0 && r + 1 < nchunks && !ms.abort_flag) issue_tma(r + 1);

        if (DELTA) {
            // ------------------------------------------------ a3: T = (I + L)^{-1}
            // Two-level block solve.  Stage 1: the inverses of the two 32x32
            // diagonal blocks by forward substitution, one column per thread
            // (threads 0..63).  Stage 2: T_BA = -T_BB (L_BA T_AA), 4 outputs per
            // thread.  T is written as the fp16 operand T2 = T diag(beta); the fp32
            // blocks T_AA (upper-right block of the L scratch, zero in L), T_BB and
            // X = L_BA T_AA (Z tile region, idle until the history read) feed stage 2.
            float *Ls = reinterpret_cast<float *>(sm + L::KT);
            float *Tbb = reinterpret_cast<float *>(sm + L::ZT);
            float *Xs = Tbb + 32 * 32;
            if (t < 64) {
                const int b = t >> 5, c = t & 31, o = 32 * b;
                float x[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = (i == c) ? 1.f : 0.f;
#pragma unroll
                for (int rr = 1; rr < 32; ++rr) {
                    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
                    for (int mm = 0; mm < rr; mm += 4) {
                        const float4 lv = *reinterpret_cast<const float4 *>(Ls + f32_swz(o + rr, o + mm, 64));
                        s0 = fmaf(lv.x, x[mm], s0);
                        if (mm + 1 < rr) s1 = fmaf(lv.y, x[mm + 1], s1);
                        if (mm + 2 < rr) s2 = fmaf(lv.z, x[mm + 2], s2);
                        if (mm + 3 < rr) s3 = fmaf(lv.w, x[mm + 3], s3);
                    }
                    x[rr] -= (s0 + s1) + (s2 + s3);
                }
                const float bt = ms.beta[o + c];
#pragma unroll
                for (int rr = 0; rr < 32; ++rr) {
                    const float tv = x[rr] * bt;
                    rmax = fmaxf(rmax, fabsf(tv));
                    *reinterpret_cast<__half *>(sm + L::TZA + sw128_off(o + rr, o + c)) = __float2half_rn(tv);
                    if (b == 0)
                        Ls[f32_swz(rr, 32 + c, 64)] = x[rr];
                    else
                        Tbb[f32_swz(rr, c, 32)] = x[rr];
                }
            }
            __syncthreads();
            TC_MARK(14);
            {
                const int rr = t >> 3, c0 = (t & 7) * 4;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int mm = 0; mm < 32; mm += 4) {
                    const float4 lv = *reinterpret_cast<const float4 *>(Ls + f32_swz(32 + rr, mm, 64));
                    const float lm[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float4 a0 = *reinterpret_cast<const float4 *>(Ls + f32_swz(mm + e, 32 + c0, 64));
                        acc[0] = fmaf(lm[e], a0.x, acc[0]);
                        acc[1] = fmaf(lm[e], a0.y, acc[1]);
                        acc[2] = fmaf(lm[e], a0.z, acc[2]);
                        acc[3] = fmaf(lm[e], a0.w, acc[3]);
                    }
                }
                *reinterpret_cast<float4 *>(Xs + f32_swz(rr, c0, 32)) = make_float4(acc[0], acc[1], acc[2], acc[3]);
                __syncthreads();
                acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
#pragma unroll
                for (int mm = 0; mm < 32; mm += 4) {
                    const float4 tv = *reinterpret_cast<const float4 *>(Tbb + f32_swz(rr, mm, 32));
                    const float tm[4] = {tv.x, tv.y, tv.z, tv.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float4 a0 = *reinterpret_cast<const float4 *>(Xs + f32_swz(mm + e, c0, 32));
                        acc[0] = fmaf(tm[e], a0.x, acc[0]);
                        acc[1] = fmaf(tm[e], a0.y, acc[1]);
                        acc[2] = fmaf(tm[e], a0.z, acc[2]);
                        acc[3] = fmaf(tm[e], a0.w, acc[3]);
                    }
                }
                float tb[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    tb[e] = -acc[e] * ms.beta[c0 + e];
                    rmax = fmaxf(rmax, fabsf(tb[e]));
                }
                *reinterpret_cast<uint2 *>(sm + L::TZA + sw128_off(32 + rr, c0)) =
                    make_uint2(pack_h2(tb[0], tb[1]), pack_h2(tb[2], tb[3]));
            }
            fence_proxy_async_smem();
            __syncthreads();
            TC_MARK(6);
            // ------------------------------------------------ a4: W and U
            if (t == 0) {
                tc_fence_after();
                const uint32_t tza = smem_u32(sm + L::TZA), at = smem_u32(sm + L::AT), v16 = smem_u32(sm + L::V16);
                constexpr uint32_t idw = idesc_f16(128, 128, 0, 0, 1);
                constexpr uint32_t idu = idesc_f16(128, DVS, 0, 0, 1);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t a = smem_desc_sw128(tza + k * 32, 16, 1024);
                    mma_f16(tmem + TM_W, a, smem_desc_sw128(at + 16384 + k * 2048, 24576, 1024), idw, k > 0);
                    mma_f16(tmem + TM_ZO, a, smem_desc_sw128(v16 + k * 2048, 8192, 1024), idu, k > 0);
                }
                mma_commit(&ms.bar_w);
            }
            if (!mbar_wait(&ms.bar_w, ph)) note_timeout(ms, 3, r);
            TC_MARK(7);
            tc_fence_after();
            if (sp < 2) {
                // W rows (lanes 0..63): this warp's 64-column half -> W slot of that half
#pragma unroll
                for (int c0 = 0; c0 < 64; c0 += 32) {
                    float w[32];
                    __syncwarp();
                    tmem_ld32(t_lane + TM_W + ch * 64 + c0, w);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) rmax = fmaxf(rmax, fabsf(w[e]));
#pragma unroll
                    for (int e = 0; e < 32; e += 8)
                        *reinterpret_cast<uint4 *>(sm + L::AT + ch * 24576 + sw128_off(row, c0 + e)) = pack_h8(w + e);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
        }
        TC_MARK(8);

        // ---------------------------------------------------- a5: history read (+ correction)
        if (t == 0 && !ms.abort_flag) {
            tc_fence_after();
            const uint32_t at = smem_u32(sm + L::AT), st = smem_u32(sm + L::ST16);
            constexpr uint32_t id = idesc_f16(128, DVS, 0, 0, 1, /*negate A*/ 1);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t ka = (k >> 2) * 24576 + (k & 3) * 32;
                mma_f16(tmem + TM_ZO, smem_desc_sw128(at + ka, 16, 1024), smem_desc_sw128(st + k * 2048, 16384, 1024),
                        id, DELTA ? 1 : (k > 0));
            }
            mma_commit(&ms.bar_1);
        }
        if (!mbar_wait(&ms.bar_1, ph)) note_timeout(ms, 4, r);
        TC_MARK(9);
        tc_fence_after();
        if (DELTA && sp < 2) {
            // Z rows (lanes 0..63), this warp's column half -> fp16 MN-major tile [64 tok][DVS]
#pragma unroll
            for (int j0 = 0; j0 < HV; j0 += 32) {
                float z[32];
                __syncwarp();
                tmem_ld32(t_lane + TM_ZO + ch * HV + j0, z);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) rmax = fmaxf(rmax, fabsf(z[e]));
                const int j = ch * HV + j0;
                unsigned char *zb = sm + L::ZT + (j >> 6) * 8192;
#pragma unroll
                for (int e = 0; e < 32; e += 8)
                    *reinterpret_cast<uint4 *>(zb + sw128_off(row, (j & 63) + e)) = pack_h8(z + e);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        TC_MARK(10);

        // ---------------------------------------------------- a6 + a7: local output and state update
        if (t == 0 && !ms.abort_flag) {
            tc_fence_after();
            const uint32_t tza = smem_u32(sm + L::TZA), kr = smem_u32(sm + L::KR);
            const uint32_t z = smem_u32(sm + (DELTA ? L::ZT : L::V16));
            constexpr uint32_t id2 = idesc_f16(128, DVS, 0, 0, 1);
            constexpr uint32_t id3 = idesc_f16(128, DVS, 0, 1, 1);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t bz = smem_desc_sw128(z + k * 2048, 8192, 1024);
                mma_f16(tmem + TM_ZO, smem_desc_sw128(tza + 8192 + k * 32, 16, 1024), bz, id2, 1);
                mma_f16(tmem + TM_S, smem_desc_sw128(kr + k * 2048, 8192, 1024), bz, id3, 1);
            }
            mma_commit(&ms.bar_2);
        }
        if (!mbar_wait(&ms.bar_2, ph)) note_timeout(ms, 5, r);
        TC_MARK(11);
        tc_fence_after();
        if (sp >= 2) {
            // O rows (lanes 64..127), this warp's column half
            const int l = row - 64;
            const bool valid = l < n;  // tcgen05.ld is warp-collective: every lane loads, valid rows store
            const size_t orow = ((size_t)bh * T + t0 + (valid ? l : 0)) * dv + v0 + ch * HV;
#pragma unroll
            for (int j0 = 0; j0 < HV; j0 += 32) {
                float ov[32];
                __syncwarp();
                tmem_ld32(t_lane + TM_ZO + ch * HV + j0, ov);
                tmem_wait_ld();
                if (valid) {
                    if (OUT_BF16) {
                        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) + orow + j0);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            uint32_t w[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                __nv_bfloat162 b2 = __floats2bfloat162_rn(ov[8 * e + 2 * u], ov[8 * e + 2 * u + 1]);
                                w[u] = *reinterpret_cast<uint32_t *>(&b2);
                            }
                            dst[e] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    } else {
                        float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.o) + orow + j0);
#pragma unroll
                        for (int e = 0; e < 8; ++e) dst[e] = make_float4(ov[4 * e], ov[4 * e + 1], ov[4 * e + 2], ov[4 * e + 3]);
                    }
                }
            }
        }
        TC_MARK(12);
        // new state -> fp16 S^T operand for the next chunk (lane = channel, this warp's half)
#pragma unroll
        for (int j0 = 0; j0 < HV; j0 += 32) {
            float sv[32];
            __syncwarp();
            tmem_ld32(t_lane + TM_S + ch * HV + j0, sv);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) rmax = fmaxf(rmax, fabsf(sv[e]));
            const int j = ch * HV + j0;
            unsigned char *sb = sm + L::ST16 + (j >> 6) * 16384;
#pragma unroll
            for (int e = 0; e < 32; e += 8)
                *reinterpret_cast<uint4 *>(sb + sw128_off(row, (j & 63) + e)) = pack_h8(sv + e);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        ok = !ms.abort_flag;
        TC_MARK(13);
    }

    // ------------------------------------------------------------ final state
    if (ok && p.ST) {
#pragma unroll
        for (int j0 = 0; j0 < HV; j0 += 16) {
            float sv[16];
            __syncwarp();
            tmem_ld16(t_lane + TM_S + ch * HV + j0, sv);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) p.ST[((size_t)bh * dv + v0 + ch * HV + j0 + i) * DK + row] = sv[i];
        }
    }
    if (!(rmax <= 65504.f)) ms.range_flag = 1;
    __syncthreads();
    if (t == 0) {
        if (ms.abort_flag) {
            record_status(p.status, kStatusTimeout);
            if (p.diag) atomicCAS(p.diag, 0, 1 + ms.abort_site);
        } else if (ms.range_flag) {
            record_status(p.status, kStatusRange);
        }
    }
    tc_fence_before();
    __syncthreads();
    __syncwarp();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int DVS, int UPD, int GATE, bool OB>
int launch_one(const TcParams &prm, int grid, cudaStream_t stream) {
    using L = TcSmem<DVS, GATE>;
    auto kern = chunk_tc_kernel<DVS, UPD, GATE, OB>;
    static_assert(L::DYN <= 232448, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::DYN);
    if (e != cudaSuccess) return (int)e;
    kern<<<grid, kTcThreads, L::DYN, stream>>>(prm);
    return (int)cudaGetLastError();
}

template <int DVS, int UPD, int GATE>
int launch_out(const TcParams &prm, int grid, bool ob, cudaStream_t s) {
    return ob ? launch_one<DVS, UPD, GATE, true>(prm, grid, s) : launch_one<DVS, UPD, GATE, false>(prm, grid, s);
}

template <int DVS>
int launch_modes(const TcParams &prm, int grid, int update, int gate, bool ob, cudaStream_t s) {
    if (update == kAdditive) return launch_out<DVS, kAdditive, kGateNone>(prm, grid, ob, s);
    if (update == kDecay) {
        if (gate == kGateScalar) return launch_out<DVS, kDecay, kGateScalar>(prm, grid, ob, s);
        if (DVS == 64) return launch_out<64, kDecay, kGateChannel>(prm, grid, ob, s);
        return (int)cudaErrorInvalidValue;
    }
    if (gate == kGateNone) return launch_out<DVS, kDelta, kGateNone>(prm, grid, ob, s);
    if (gate == kGateScalar) return launch_out<DVS, kDelta, kGateScalar>(prm, grid, ob, s);
    if (DVS == 64) return launch_out<64, kDelta, kGateChannel>(prm, grid, ob, s);
    return (int)cudaErrorInvalidValue;
}

}  // namespace
}  // namespace gdn

#ifdef GDN_TC_PHASE_TIMING
extern "C" int gdn_tc_phase_times(unsigned long long *out, int clear) {
    cudaDeviceSynchronize();
    if (cudaMemcpyFromSymbol(out, g_tc_phase, sizeof(unsigned long long) * 16) != cudaSuccess) return -1;
    if (clear) {
        unsigned long long z[16] = {0};
        cudaMemcpyToSymbol(g_tc_phase, z, sizeof(z));
    }
    return 0;
}
#endif

int gdn_tc_supported(const gdn_desc_t *d) {
    return d->dtype == GDN_BF16 && d->dk == 128 && (d->dv == 64 || d->dv == 128);
}

// Value-slice width: 128 keeps the K-side work unduplicated; 64 doubles the
// CTA count when 128-wide slices would leave most SMs idle.  The per-channel
// gate's extra gate tile needs the 64-wide slice's shared-memory budget.
static int tc_slice(const gdn_desc_t *d) {
    const long bh = (long)d->B * d->H;
    if (d->dv == 64 || d->gate == GDN_GATE_CHANNEL) return 64;
    return (bh * 2 <= 148) ? 64 : 128;
}

int gdn_launch_chunk_tc(const gdn::ChunkArgs &a, const gdn_desc_t *d, cudaStream_t stream) {
    using namespace gdn;
    TcParams prm;
    memset(&prm, 0, sizeof(prm));
    const uint64_t BH = (uint64_t)a.BH, T = (uint64_t)a.T;
    if (!make_map_3d(&prm.q_map, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 128, T, BH, 64, 64, 1, true) ||
        !make_map_3d(&prm.k_map, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 128, T, BH, 64, 64, 1, true) ||
        !make_map_3d(&prm.v_map, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.dv, T, BH, 64, 64, 1, true))
        return (int)cudaErrorInvalidValue;
    if (d->gate == GDN_GATE_CHANNEL &&
        !make_map_3d(&prm.g_map, a.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 128, T, BH, 32, 64, 1, false))
        return (int)cudaErrorInvalidValue;
    prm.g = a.g;
    prm.beta = a.beta;
    prm.S0 = a.S0;
    prm.o = a.o;
    prm.ST = a.ST;
    prm.status = a.status;
    prm.diag = a.diag;
    prm.BH = a.BH;
    prm.T = a.T;
    prm.dv = a.dv;
    const int dvs = tc_slice(d);
    prm.nslices = a.dv / dvs;
    const long grid = (long)a.BH * prm.nslices;
    if (grid == 0) return 0;
    const bool ob = d->out_dtype == GDN_BF16;
    if (dvs == 64) return launch_modes<64>(prm, (int)grid, d->update, d->gate, ob, stream);
    return launch_modes<128>(prm, (int)grid, d->update, d->gate, ob, stream);
}
