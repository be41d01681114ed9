// Warp-specialised tensor-core chunkwise prefill (bf16 inputs, dk = 128).
//
// One CTA owns one (b,h) head and a slice of DVS value rows (64 or 128) and
// walks its chunks (C = 64) with two warp groups that overlap:
//
//   prep group  (warps 0-7) for chunk r+1: TMA of q, k, v (and the channel
//       gate), the gate prefix, fp16 operands Q<, K<, K>, V, A' = P_top
//       masked with decay and L = beta P_bottom from P = [Q;K] K^T, and the UT
//       transform T = (I + L)^{-1} (fp32: 16x16 diagonal blocks by forward
//       substitution, then two block merges on tf32 warp MMAs) as T2 = T diag(beta).
//   state group (warps 8-11) for chunk r, every MMA with M = DVS value rows
//       (the transposed form), so that the state and the correction rows are
//       A operands held in TMEM:
//         [O^T | X^T] = S [Q< ; K<]^T        (one N = 128 chain)
//         Z^T  = V^T T2^T - X^T T2^T         (U^T minus the history correction)
//         O^T += Z^T A'^T
//         S    = S Diag(e^{G_C}) + Z^T K>
//       Its MMA thread also issues the next chunk's P.  O leaves through a
//       staging tile and a TMA store.
//
// Same algebra as "Linear Attention, Visualized": "Chunkwise algorithm",
// "Mamba-2 ... Chunkwise form", "Gated Linear Attention (GLA)", "The triangular
// correction system", "Optional: Use UT to share the triangular transform",
// "Correct the incoming state" and the GDN / KDA tables (W S^T = T2 (K< S^T) is
// evaluated as (S K<^T) T2^T); only the storage is transposed (S is kept
// [dv x dk] with lane = value row).
//
// TMEM (512 columns): P [0,64), Z^T [64,128), O^T|X^T [128,256), S fp32
// [256,384), S fp16 (A operand) [384,448), -X^T / Z^T fp16 (A operand) [448,480).
// Hand-offs: bar_rdy (prep -> state, one phase per chunk), bar_fA (state MMAs
// that read Q<, K<, V, T2 completed), bar_fB0/1 (state MMAs that read A', K>
// of an even / odd chunk completed; A' and K> are double-buffered).  All waits
// are bounded: on a timeout the CTA records GDN_ERR_TIMEOUT and the wait site.
// Intermediates handed to the tensor cores (T2, Q<, K<, K>, V, A', -X, Z and
// the state copy) are fp16 (11-bit significand; raw bf16 inputs are exact in
// it); accumulators and the state master are fp32.  Every value converted to
// fp16 is range-checked and an overflow is recorded as GDN_ERR_RANGE.
#include <string.h>

#include "../../include/gdn.h"
#include "common.cuh"
#include "sm100.cuh"
#include "tc_util.cuh"
#include "tma_host.cuh"

#ifdef GDN_TC_PHASE_TIMING
// Per-phase cycle totals of CTA 0: slots 0..15 prep group, 16..31 state group.
__device__ unsigned long long g_tc2_phase[32];
#define TC2_MARK(who, i)                                                           \
    do {                                                                          \
        if (blockIdx.x == 0 && t == (who)) {                                      \
            const long long now_ = clock64();                                     \
            atomicAdd(&g_tc2_phase[i], (unsigned long long)(now_ - mark_prev));   \
            mark_prev = now_;                                                     \
        }                                                                         \
    } while (0)
#else
#define TC2_MARK(who, i) \
    do {                 \
    } while (0)
#endif

namespace gdn {
namespace {

using namespace sm100;
using namespace tcu;

constexpr int kThreads = 384;  // warps 0-7 prep, 8-11 state
constexpr int C = kChunk;
constexpr int DK = 128;
constexpr float kFactorMaxDecay = 10.0f;
constexpr int kPrepBar = 1, kStateBar = 2, kConvBar = 4, kPairBar = 5, kVBar = 9;  // kPairBar..kPairBar+3

struct Params {
    CUtensorMap q_map, k_map, v_map, g_map, o_map;
    const float *g;
    const float *beta;
    const float *S0;
    void *o;
    float *ST;
    int *status;
    int *diag;
    int BH, T, dv, nslices;
    int nh, cv, tpc;  // Gated DeltaProduct: substeps per token, virtual steps and tokens per chunk
    // and the rows of a chunk that are a token's first / last substep (bit l = row l)
    unsigned long long firstmask, lastmask;
    int pro;   // GDN_PRO_* input maps
    int mode;  // kMode* bits (internal passes of the segmented prefill, saved states)
    float *states;  // kModeSaveStates: the chunk-entry states [BH][nchunks][dv][dk]
    unsigned long long wait_ns;  // bound of the hand-off waits (gdn_set_wait_limit_ns)
};

template <int DVS, int GATE>
struct Smem {
    static constexpr int RAW_QK = 0;                                     // [Q0 K0 | Q1 K1] bf16
    static constexpr int RAW_V = RAW_QK + 32768;                         // V slice bf16
    static constexpr int GCH = RAW_V + DVS * 128;                        // channel gate: 4 x [64][32] fp32, swizzled
    static constexpr int AT = GCH + (GATE == kGateChannel ? 32768 : 0);  // [Q< | K<] x 2 key halves
    static constexpr int KT = AT + 32768;                                // k e^{-G} fp16 / L^T fp32 scratch
    static constexpr int KR = KT + 16384;                                // K> fp16, 2 buffers
    static constexpr int V16 = KR + 32768;                               // V fp16
    static constexpr int TZA = V16 + DVS * 128;                          // [T2 | A'0 | A'1] fp16
    static constexpr int OST = TZA + 24576;                              // O staging [64 tok][DVS] (TMA store)
    static constexpr int DEC = OST + DVS * 256;                          // float dec[2][128]
    static constexpr int MISC = DEC + 1024;
    static constexpr int TOTAL = MISC + 3072;
    static constexpr int DYN = TOTAL + 1024;
};

struct Misc {
    float G[64];
    float b[64];
    float gam[64];
    float ib[64];
    float iq[64], ik[64];  // unit-row factors 1/|q_l|, 1/|k_l| (input map, unit rows only)
    float ibk[64];         // ib * ik
    float beta[2][64];  // by chunk parity: the solve of chunk r overlaps the gate pass of r+1
    float GC[128];
    int abort_flag, range_flag, slow_chunk, abort_site;
    int p_abort, s_abort, n_tma, n_tv;  // n_tma / n_tv: phases armed on bar_tma / bar_tv
    uint32_t tmem_base, pad2[3];
    uint64_t bar_tma, bar_p1, bar_x, bar_rdy, bar_fA, bar_fB0, bar_fB1, bar_tv;
    uint64_t bar_drain;  // after a timeout: every MMA issued has completed
};

static_assert(sizeof(Misc) <= 3072, "the Misc block has 3 KB of shared memory");

template <typename M>
__device__ __forceinline__ void note_timeout(M &ms, int site, int r) {
    if (atomicCAS(&ms.abort_flag, 0, 1) == 0) ms.abort_site = site * 1000000 + r;
}

constexpr uint32_t TP = 0, TZ = 64, TOX = 128, TSM = 256, TS16 = 384, TZ16 = 448;

// Eight raw q / k elements as fp32: bf16 as loaded, fp16 once the input map has run.
__device__ __forceinline__ void unpack_qk8(uint4 u, float *f, bool f16) {
    if (f16) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 x = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
            f[2 * i] = x.x;
            f[2 * i + 1] = x.y;
        }
    } else {
        unpack_bf16x8(u, f);
    }
}

// Float index of gate element (token l, channel c) in the channel-gate tile: four
// [64][32] fp32 sub-tiles loaded by TMA with the 128-byte swizzle (16-byte slot
// XOR token % 8), so reads of one channel group across tokens spread over banks.
__device__ __forceinline__ int gch_idx(int l, int c) {
    return (c >> 5) * 2048 + l * 32 + ((((c & 31) >> 2) ^ (l & 7)) << 2) + (c & 3);
}

// Shared offset of chunk parity `buf`'s fp16 V tile.  Without the delta rule V is
// an operand of the state's last MMAs, so it is double-buffered, the second copy in
// the L^T scratch that those modes leave unused.
template <typename L, int UPD, int GATE>
__device__ __forceinline__ int v16_slot(int buf) {
    return (UPD != kDelta && GATE != kGateChannel && buf) ? L::KT : L::V16;
}

// PROD: Gated DeltaProduct with nh substeps per token ("GDP as GDN over a
// virtual sequence"): T counts virtual steps; k, v, beta are per virtual step,
// while q, g and o are per token.  A chunk covers tpc = 64 / nh whole tokens,
// i.e. cv = tpc * nh virtual steps; when nh does not divide 64 its last 64 - cv
// rows are identity steps (k, beta and g zero, so T2 has zero columns there
// and they neither read nor change the state).  The tokens' q rows arrive
// compact and are moved to each token's last substep (zeros elsewhere), the
// gate sits on each token's first substep, and only each token's last substep
// is written out.
//
// EXT: the input prologue and the segmented prefill's pass modes are compiled
// in only for calls that use them; the plain path (EXT = false) sees both as
// constant zero, so it keeps the registers and code it has without them.
template <int DVS, int UPD, int GATE, bool OUT_BF16, bool PROD, bool EXT>
__global__ void __launch_bounds__(kThreads, 1) chunk_tc2_kernel(const __grid_constant__ Params p) {
    using L = Smem<DVS, GATE>;
    constexpr bool DELTA = (UPD == kDelta);
    const int pro = EXT ? p.pro : 0;
    const int mode = EXT ? p.mode : 0;
    // the hand-off waits, bounded at 1 s; a test's shorter bound is compiled
    // into the EXT instantiation only, so the plain kernel's waits are unchanged
    auto mwait = [&p](uint64_t *bar, uint32_t par) {
        if (EXT && p.wait_ns) return mbar_wait_bounded(bar, par, p.wait_ns);
        return mbar_wait(bar, par);
    };
    // P = [Q;K]K^T of a chunk is issued by the state group's MMA thread right after
    // rdy when the prep group is the longer side (delta rule, scalar / no gate), else
    // by the prep group itself (it then has slack; the channel gate's P also needs
    // the converted operands)
    // With the elu+1 input map (alone or before unit rows) the raw tiles are mapped
    // in place to fp16 after they land, so P follows that pass and is issued by the
    // prep group.  Unit rows alone leave the tiles as they are: the row norms
    // become factors on P (rows and columns) and on the converted operands.
    const bool qkmap = (pro & kProElu1) != 0;
    const bool l2scale = (pro & kProL2) != 0 && !qkmap;
    const bool kStateP1 = DELTA && GATE != kGateChannel && !PROD && !qkmap;
    // In the same modes the V tile has its own TMA barrier (bar_tv): its fp16
    // conversion runs during the 16 -> 32 merge, after the q / k conversion window
    constexpr bool kSplitV = DELTA && GATE != kGateChannel;
    constexpr int NB = DVS / 64;
    extern __shared__ unsigned char smraw[];
    // Align by an integer offset from the shared array itself, so that every access
    // through `sm` stays in the shared address space (LDS/STS, not generic).
    unsigned char *sm = smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);
    Misc &ms = *reinterpret_cast<Misc *>(sm + L::MISC);
    float *dec = reinterpret_cast<float *>(sm + L::DEC);

    const int t = threadIdx.x;
    const int warp = t >> 5, lane = t & 31;
    const int sp = warp & 3;
    const int bh = blockIdx.x / p.nslices;
    const int v0 = (blockIdx.x % p.nslices) * DVS;
    const int T = p.T, dv = p.dv;
    // virtual steps and tokens per chunk, substeps per token (compile-time C, C, 1
    // unless PROD)
    const int CV = PROD ? p.cv : C, TPC = PROD ? p.tpc : C, NH = PROD ? p.nh : 1;
    const int nchunks = (T + CV - 1) / CV;

    if (t == 0) {
        mbar_init(&ms.bar_tma, 1);
        mbar_init(&ms.bar_tv, 1);
        mbar_init(&ms.bar_drain, 2);  // the two MMA-issuing threads
        mbar_init(&ms.bar_p1, 1);
        mbar_init(&ms.bar_x, 1);
        mbar_init(&ms.bar_rdy, 1);
        mbar_init(&ms.bar_fA, 1);
        mbar_init(&ms.bar_fB0, 1);
        mbar_init(&ms.bar_fB1, 1);
        fence_mbar_init();
        ms.abort_flag = 0;
        ms.range_flag = 0;
        ms.p_abort = 0;
        ms.s_abort = 0;
        ms.n_tma = 0;
        ms.n_tv = 0;
        tma_prefetch_desc(&p.q_map);
        tma_prefetch_desc(&p.k_map);
        if (!(mode & kModeZeroV)) tma_prefetch_desc(&p.v_map);
        if (GATE == kGateChannel) tma_prefetch_desc(&p.g_map);
        if (!(mode & kModeNoOut)) tma_prefetch_desc(&p.o_map);
    }
    __syncwarp();
    if (warp == 0) {
        tmem_alloc(&ms.tmem_base, 512);
        tmem_relinquish();
    }
    // T2 tile: its upper-right 32x32 block is never written and stays zero
    for (int i = t; i < 8192 / 16; i += kThreads) reinterpret_cast<uint4 *>(sm + L::TZA)[i] = make_uint4(0, 0, 0, 0);
    const bool zeroV = (mode & kModeZeroV) != 0;
    if (zeroV) {
        // values taken as zero: the fp16 V tiles are cleared once and never loaded
        for (int i = t; i < DVS * 128 / 16; i += kThreads) {
            reinterpret_cast<uint4 *>(sm + L::V16)[i] = make_uint4(0, 0, 0, 0);
            if (!DELTA && GATE != kGateChannel) reinterpret_cast<uint4 *>(sm + L::KT)[i] = make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms.tmem_base;
    const uint32_t lane_addr = tmem + ((uint32_t)(sp * 32) << 16);
    float rmax = 0.f;  // largest |value| this thread handed to an fp16 operand
#ifdef GDN_TC_PHASE_TIMING
    long long mark_prev = clock64();
#endif

    if (warp < 8) {
        // =================================================================== prep group (8 warps)
        const int ch = warp >> 2;          // column half of a TMEM tile handled by this warp
        const int row = sp * 32 + lane;    // TMEM lane (product row) read by this thread
        float gpre0 = 0.f, gpre1 = 0.f, bpre = 0.f;
        // raw gates (warp 4, two tokens a lane) and betas (warps 4-5) of chunk r into registers
        auto load_gate_beta = [&](int r) {
            const int t0 = r * CV;
            if (GATE == kGateScalar && warp == 4) {
                const int l0 = 2 * lane;
                if (PROD) {
                    // the token's gate on its first substep, 1 (g = 0) on the others and
                    // on the identity rows past cv
                    const size_t gb = (size_t)bh * (T / NH) + (size_t)r * TPC;
                    const int l1 = l0 + 1;
                    const unsigned long long fm = p.firstmask;
                    // the token of a first-substep row is the number of first substeps before it
                    gpre0 = (t0 + l0 < T && ((fm >> l0) & 1)) ? pro_gate(p.g[gb + __popcll(fm & ((1ull << l0) - 1))], pro)
                                                             : 0.f;
                    gpre1 = (t0 + l1 < T && ((fm >> l1) & 1)) ? pro_gate(p.g[gb + __popcll(fm & ((1ull << l1) - 1))], pro)
                                                             : 0.f;
                } else {
                    gpre0 = (t0 + l0 < T) ? pro_gate(p.g[(size_t)bh * T + t0 + l0], pro) : 0.f;
                    gpre1 = (t0 + l0 + 1 < T) ? pro_gate(p.g[(size_t)bh * T + t0 + l0 + 1], pro) : 0.f;
                }
            }
            if (DELTA && t >= 128 && t < 128 + C) {
                const int l = t - 128;
                bpre = (t0 + l < T && l < CV) ? pro_beta(p.beta[(size_t)bh * T + t0 + l], pro) : 0.f;
            }
        };
        // scalar gate prefix of chunk r and its factors b = e^G, gamma = e^{G_C-G},
        // 1/b, e^{G_C}; beta of chunk r into its parity slot (warps 4-5)
        auto gate_pass = [&](int r) {
            if (GATE == kGateScalar && warp == 4) {
                const int l0 = 2 * lane;
                const float x0 = gpre0, x1 = gpre1;
                float s = x0 + x1;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, s, off);
                    if (lane >= off) s += y;
                }
                const float G0 = s - x1, G1 = s;
                const float gc = __shfl_sync(0xffffffffu, G1, 31);
                ms.G[l0] = G0;
                ms.G[l0 + 1] = G1;
                ms.b[l0] = __expf(G0);
                ms.b[l0 + 1] = __expf(G1);
                ms.gam[l0] = __expf(gc - G0);
                ms.gam[l0 + 1] = __expf(gc - G1);
                ms.ib[l0] = __expf(-G0);
                ms.ib[l0 + 1] = __expf(-G1);
                if (lane == 0) dec[(r & 1) * 128] = __expf(gc);
            }
            if (DELTA && t >= 128 && t < 128 + C) ms.beta[r & 1][t - 128] = bpre;
        };
        // q, k (+ the channel gate tile) on bar_tma; v on bar_tv when split, else also on bar_tma
        auto issue_tma_v = [&](int r, uint64_t *bar) {
            for (int j = 0; j < NB; ++j)
                tma_load_3d(sm + L::RAW_V + j * 8192, &p.v_map, v0 + j * 64, r * CV, bh, bar);
        };
        auto issue_tma = [&](int r) {
            const int t0 = r * CV;
            const uint32_t qbytes = PROD ? 2u * (uint32_t)TPC * 128u : 16384u;
            const uint32_t gbytes = PROD ? 512u * (uint32_t)TPC : 32768u;  // the channel gate tile
            const uint32_t bytes =
                qbytes + 16384 + ((kSplitV || zeroV) ? 0 : DVS * 128) + (GATE == kGateChannel ? gbytes : 0);
            mbar_arrive_expect_tx(&ms.bar_tma, bytes);
            ++ms.n_tma;
            for (int h = 0; h < 2; ++h) {
                tma_load_3d(sm + L::RAW_QK + h * 16384, &p.q_map, h * 64, PROD ? r * TPC : t0, bh,
                            &ms.bar_tma);
                tma_load_3d(sm + L::RAW_QK + h * 16384 + 8192, &p.k_map, h * 64, t0, bh, &ms.bar_tma);
            }
            if (!kSplitV && !zeroV) issue_tma_v(r, &ms.bar_tma);
            if (GATE == kGateChannel)
                for (int j = 0; j < 4; ++j)
                    tma_load_3d(sm + L::GCH + j * 8192, &p.g_map, j * 32, PROD ? r * TPC : t0, bh, &ms.bar_tma);
        };
        auto issue_tma_split_v = [&](int r) {
            mbar_arrive_expect_tx(&ms.bar_tv, DVS * 128);
            ++ms.n_tv;
            issue_tma_v(r, &ms.bar_tv);
        };
        if (t == 0 && nchunks > 0) {
            issue_tma(0);
            if (kSplitV && !zeroV) issue_tma_split_v(0);
        }
        if (nchunks > 0) {
            load_gate_beta(0);
            if (GATE != kGateChannel) {
                gate_pass(0);
                if (nchunks > 1) load_gate_beta(1);
            }
        }
        named_bar(kPrepBar, 256);

        for (int r = 0; r < nchunks; ++r) {
            if (ms.p_abort) break;
            const uint32_t ph = r & 1;
            const int buf = r & 1;
            const float *bet = ms.beta[buf];
            TC2_MARK(0, 0);
            if (!mwait(&ms.bar_tma, ph)) note_timeout(ms, 1, r);
            if (PROD) {
                // compact q rows j -> row (j + 1) * nh - 1, the rest zero (both key halves);
                // the k rows past cv (the next chunk's first steps, loaded by the 64-row box)
                // become the zero keys of identity steps
                uint4 qv[4];
#pragma unroll
                for (int s4 = 0; s4 < 4; ++s4) {
                    const int i = t + 256 * s4, h = i >> 9, d = (i & 511) >> 3, c = i & 7;
                    qv[s4] = make_uint4(0, 0, 0, 0);
                    if ((p.lastmask >> d) & 1) {
                        const int j = __popcll(p.lastmask & ((1ull << d) - 1));  // the row's token
                        qv[s4] = *reinterpret_cast<const uint4 *>(sm + L::RAW_QK + h * 16384 + j * 128 +
                                                                   ((c ^ (j & 7)) << 4));
                    }
                }
                // the per-channel gate: each token's row (compact, as loaded) moves to the
                // token's first substep, every other row is g = 0 (four 32-channel sub-tiles)
                uint4 gw[GATE == kGateChannel ? 8 : 1];
                if (GATE == kGateChannel) {
#pragma unroll
                    for (int s8 = 0; s8 < 8; ++s8) {
                        const int i = t + 256 * s8, st = i >> 9, d = (i & 511) >> 3, c = i & 7;
                        gw[s8] = make_uint4(0, 0, 0, 0);
                        if ((p.firstmask >> d) & 1) {
                            const int j = __popcll(p.firstmask & ((1ull << d) - 1));  // the row's token
                            gw[s8] = *reinterpret_cast<const uint4 *>(sm + L::GCH + st * 8192 + j * 128 +
                                                                       ((c ^ (j & 7)) << 4));
                        }
                    }
                }
                named_bar(kPrepBar, 256);
                if (GATE == kGateChannel) {
#pragma unroll
                    for (int s8 = 0; s8 < 8; ++s8) {
                        const int i = t + 256 * s8, st = i >> 9, d = (i & 511) >> 3, c = i & 7;
                        *reinterpret_cast<uint4 *>(sm + L::GCH + st * 8192 + d * 128 + ((c ^ (d & 7)) << 4)) = gw[s8];
                    }
                }
#pragma unroll
                for (int s4 = 0; s4 < 4; ++s4) {
                    const int i = t + 256 * s4, h = i >> 9, d = (i & 511) >> 3, c = i & 7;
                    *reinterpret_cast<uint4 *>(sm + L::RAW_QK + h * 16384 + d * 128 + ((c ^ (d & 7)) << 4)) = qv[s4];
                    if (d >= CV)
                        *reinterpret_cast<uint4 *>(sm + L::RAW_QK + h * 16384 + 8192 + d * 128 + ((c ^ (d & 7)) << 4)) =
                            make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
                named_bar(kPrepBar, 256);
            }
            if (qkmap) {
                // q / k input map in place: thread = (tensor, row, key half); the two
                // halves of a row are adjacent lanes.  Rows past T and, for the
                // product, q rows that are not a token's last substep stay zero.
                const int ten = t >> 7, row = (t >> 1) & 63, hk = t & 1;
                const int m = r * CV + row;
                bool valid = m < T && row < CV;
                if (PROD && ten == 0) valid = valid && ((p.lastmask >> row) & 1);
                unsigned char *base = sm + L::RAW_QK + hk * 16384 + ten * 8192 + row * 128;
                float f[64];
                float ss = 0.f;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    unpack_bf16x8(*reinterpret_cast<const uint4 *>(base + ((c ^ (row & 7)) << 4)), f + 8 * c);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        f[8 * c + e] = valid ? pro_feature(f[8 * c + e], pro) : 0.f;
                        ss = fmaf(f[8 * c + e], f[8 * c + e], ss);
                    }
                }
                ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                const float sc = (pro & kProL2) ? (ss > 0.f ? 1.f / sqrtf(ss) : 0.f) : 1.f;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        f[8 * c + e] *= sc;
                        rmax = fmaxf(rmax, fabsf(f[8 * c + e]));
                    }
                    *reinterpret_cast<uint4 *>(base + ((c ^ (row & 7)) << 4)) = pack_h8(f + 8 * c);
                }
                fence_proxy_async_smem();
                named_bar(kPrepBar, 256);
            }
            if (l2scale) {
                // 1 / |row| of every q and k row (thread = tensor, row, key half)
                const int ten = t >> 7, row = (t >> 1) & 63, hk = t & 1;
                const unsigned char *base = sm + L::RAW_QK + hk * 16384 + ten * 8192 + row * 128;
                float ss = 0.f;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    float f[8];
                    unpack_bf16x8(*reinterpret_cast<const uint4 *>(base + ((c ^ (row & 7)) << 4)), f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
                }
                ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                const float inv = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
                if (hk == 0) {
                    if (ten == 0) {
                        ms.iq[row] = inv;
                    } else {
                        ms.ik[row] = inv;
                        ms.ibk[row] = (GATE == kGateScalar ? ms.ib[row] : 1.f) * inv;
                    }
                }
                named_bar(kPrepBar, 256);
            }
            TC2_MARK(0, 1);
            if (!kStateP1 && GATE != kGateChannel && t == 0 && !ms.abort_flag) {
                tc_fence_after();
                const uint32_t qk = smem_u32(sm + L::RAW_QK);
                const uint32_t id = qkmap ? idesc_f16(128, 64, 0, 0, 0) : idesc_f16(128, 64, 1, 0, 0);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t ko = (k >> 2) * 16384 + (k & 3) * 32;
                    mma_f16(tmem + TP, smem_desc_sw128(qk + ko, 16, 1024), smem_desc_sw128(qk + 8192 + ko, 16, 1024),
                            id, k > 0);
                }
                mma_commit(&ms.bar_p1);
            }
            if (GATE == kGateChannel) {
                // ------------------------------------------------ a1: channel gate prefix
                // channel c, token half hf: prefix over 32 tokens, then join the halves
                const int c = t & 127, hf = t >> 7;
                float *gt = reinterpret_cast<float *>(sm + L::GCH);
                float gv[32];
#pragma unroll
                for (int l = 0; l < 32; ++l) {
                    gv[l] = gt[gch_idx(32 * hf + l, c)];
                    // padding (and, for the product, every row but a token's first substep) stays g = 0
                    const bool real = PROD ? ((p.firstmask >> (32 * hf + l)) & 1) != 0 : true;
                    if (r * CV + 32 * hf + l < T && real) gv[l] = pro_gate(gv[l], pro);
                }
#pragma unroll
                for (int l = 1; l < 32; ++l) gv[l] += gv[l - 1];
                if (hf == 0) {
#pragma unroll
                    for (int l = 0; l < 32; ++l) gt[gch_idx(l, c)] = gv[l];
                }
                named_bar(kPrepBar, 256);
                if (hf == 1) {
                    const float base = gt[gch_idx(31, c)];
#pragma unroll
                    for (int l = 0; l < 32; ++l) gt[gch_idx(32 + l, c)] = gv[l] + base;
                    ms.GC[c] = gv[31] + base;
                    dec[buf * 128 + c] = __expf(gv[31] + base);
                }
                named_bar(kPrepBar, 256);
                if (warp == 0) {
                    float mx = 0.f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) mx = fmaxf(mx, -ms.GC[lane + 32 * i]);
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                    if (lane == 0) ms.slow_chunk = !(mx <= kFactorMaxDecay);
                }
                gate_pass(r);
                if (r + 1 < nchunks) load_gate_beta(r + 1);
                named_bar(kPrepBar, 256);
            }
            const bool fastg = (GATE != kGateScalar) || (-ms.G[C - 1] <= 80.f);
            TC2_MARK(0, 2);
            // A'[buf] and K>[buf] were last read by the state's chunk r-2
            if (r >= 2) {
                uint64_t *fb = buf ? &ms.bar_fB1 : &ms.bar_fB0;
                if (!mwait(fb, ((r - 2) >> 1) & 1)) note_timeout(ms, 10, r);
            }
            // the history operands were last read by the state's chunk r-1: Q<, K<, V by
            // its first MMA group (bar_x; fA without the delta rule), T2 also by the
            // correction MMA (fA), the single V tile of the channel modes by its last MMAs
            auto wait_first_mmas = [&]() {
                if (DELTA && r >= 1) {
                    if (!mwait(&ms.bar_x, (r - 1) & 1)) note_timeout(ms, 12, r);
                }
            };
            auto wait_history = [&]() {
                if (r >= 1) {
                    if (DELTA || GATE != kGateChannel) {
                        if (!mwait(&ms.bar_fA, (r - 1) & 1)) note_timeout(ms, 9, r);
                    } else {
                        uint64_t *fb = ((r - 1) & 1) ? &ms.bar_fB1 : &ms.bar_fB0;
                        if (!mwait(fb, ((r - 1) >> 1) & 1)) note_timeout(ms, 10, r);
                    }
                }
            };
            TC2_MARK(0, 3);
            // ---------------------------------------------------- operand conversions
            const bool slow = (GATE == kGateChannel) && ms.slow_chunk;
            if (GATE == kGateChannel) {
                if (DELTA)
                    wait_first_mmas();
                else
                    wait_history();
                {
                    // every raw load of this thread first: a shared store would otherwise
                    // hold each later load behind it (the compiler cannot rule out aliasing)
                    uint4 rq[4], rk[4], rv[2 * NB];
#pragma unroll
                    for (int s4 = 0; s4 < 4; ++s4) {
                        const int i = t + 256 * s4;
                        const int h = i >> 9, off = (i & 511) * 16;
                        rq[s4] = *reinterpret_cast<const uint4 *>(sm + L::RAW_QK + h * 16384 + off);
                        rk[s4] = *reinterpret_cast<const uint4 *>(sm + L::RAW_QK + h * 16384 + 8192 + off);
                    }
#pragma unroll
                    for (int s4 = 0; s4 < 2 * NB; ++s4)
                        rv[s4] = *reinterpret_cast<const uint4 *>(sm + L::RAW_V + (t + 256 * s4) * 16);
#pragma unroll
                    for (int s4 = 0; s4 < 4; ++s4) {
                        const int i = t + 256 * s4;
                        const int h = i >> 9, off = (i & 511) * 16;
                        const int l = off >> 7;
                        const int c0 = h * 64 + ((((off >> 4) & 7) ^ (l & 7)) << 3);
                        float qf[8], kf[8], ql[8], kl[8], kr[8];
                        unpack_qk8(rq[s4], qf, qkmap);
                        unpack_qk8(rk[s4], kf, qkmap);
                        if (l2scale) {
                            const float fq = ms.iq[l], fk = ms.ik[l];
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                qf[e] *= fq;
                                kf[e] *= fk;
                            }
                        }
#pragma unroll
                        for (int e = 0; e < 8; ++e) rmax = fmaxf(rmax, fmaxf(fabsf(qf[e]), fabsf(kf[e])));
                        if (GATE == kGateChannel) {
                            const float *gt = reinterpret_cast<const float *>(sm + L::GCH);
                            const float4 g0 = *reinterpret_cast<const float4 *>(gt + gch_idx(l, c0));
                            const float4 g1 = *reinterpret_cast<const float4 *>(gt + gch_idx(l, c0 + 4));
                            const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                            float kt[8];
                            if (!slow) {
                                // e^{G_C} per channel was stored by the prefix pass; here
                                // e^{G_C - G} = e^{G_C} e^{-G} (e^{-G} <= e^{10})
                                const float4 d0 = *reinterpret_cast<const float4 *>(dec + buf * 128 + c0);
                                const float4 d1 = *reinterpret_cast<const float4 *>(dec + buf * 128 + c0 + 4);
                                const float egc[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
                                for (int e = 0; e < 8; ++e) {
                                    const float x = gg[e] * 1.4426950408889634f;  // log2(e)
                                    const float eg = ex2_approx(x), emg = ex2_approx(-x);
                                    ql[e] = qf[e] * eg;
                                    kl[e] = kf[e] * eg;
                                    kt[e] = kf[e] * emg;
                                    kr[e] = kt[e] * egc[e];
                                    rmax = fmaxf(rmax, fabsf(kt[e]));
                                }
                            } else {
                                // strong decay in this chunk: no k e^{-G} operand (the exact
                                // fp32 path evaluates P), e^{G_C - G} directly
#pragma unroll
                                for (int e = 0; e < 8; ++e) {
                                    const float G = gg[e];
                                    const float eg = __expf(G);
                                    ql[e] = qf[e] * eg;
                                    kl[e] = kf[e] * eg;
                                    kt[e] = 0.f;
                                    kr[e] = kf[e] * __expf(ms.GC[c0 + e] - G);
                                }
                            }
                            *reinterpret_cast<uint4 *>(sm + L::KT + h * 8192 + off) = pack_h8(kt);
                        } else {
                            const float bl = (GATE == kGateScalar) ? ms.b[l] : 1.f;
                            const float gl = (GATE == kGateScalar) ? ms.gam[l] : 1.f;
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                ql[e] = qf[e] * bl;
                                kl[e] = kf[e] * bl;
                                kr[e] = kf[e] * gl;
                            }
                        }
                        *reinterpret_cast<uint4 *>(sm + L::AT + h * 16384 + off) = pack_h8(ql);
                        if (DELTA || GATE == kGateChannel)
                            *reinterpret_cast<uint4 *>(sm + L::AT + h * 16384 + 8192 + off) = pack_h8(kl);
                        *reinterpret_cast<uint4 *>(sm + L::KR + buf * 16384 + h * 8192 + off) = pack_h8(kr);
                    }
#pragma unroll
                    for (int s4 = 0; s4 < 2 * NB; ++s4) {
                        if (zeroV) break;
                        float vf[8];
                        unpack_bf16x8(rv[s4], vf);
                        *reinterpret_cast<uint4 *>(sm + L::V16 + (t + 256 * s4) * 16) = pack_h8(vf);
#pragma unroll
                        for (int e = 0; e < 8; ++e) rmax = fmaxf(rmax, fabsf(vf[e]));
                    }
                }
            } else {
                // K> (the state update) first: no MMA in flight reads its slot, so this
                // overlaps the state's history MMAs of chunk r-1
                uint4 rk[4];
#pragma unroll
                for (int s4 = 0; s4 < 4; ++s4) {
                    const int i = t + 256 * s4;
                    rk[s4] = *reinterpret_cast<const uint4 *>(sm + L::RAW_QK + (i >> 9) * 16384 + 8192 + (i & 511) * 16);
                }
#pragma unroll
                for (int s4 = 0; s4 < 4; ++s4) {
                    const int i = t + 256 * s4;
                    const int h = i >> 9, off = (i & 511) * 16;
                    const int l = off >> 7;
                    float kf[8], kr[8];
                    unpack_qk8(rk[s4], kf, qkmap);
                    const float gl = ((GATE == kGateScalar) ? ms.gam[l] : 1.f) * (l2scale ? ms.ik[l] : 1.f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        rmax = fmaxf(rmax, fabsf(kf[e]));
                        kr[e] = kf[e] * gl;
                    }
                    *reinterpret_cast<uint4 *>(sm + L::KR + buf * 16384 + h * 8192 + off) = pack_h8(kr);
                }
            }
            if (GATE == kGateChannel) {
                // the channel-gate products take the converted operands: P = [Q<;K<] (k e^{-G})^T
                fence_proxy_async_smem();
                named_bar(kPrepBar, 256);
            }
            if (GATE == kGateChannel && t == 0) {
                tc_fence_after();
                const uint32_t at = smem_u32(sm + L::AT), kt = smem_u32(sm + L::KT);
                constexpr uint32_t id = idesc_f16(128, 64, 0, 0, 0);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t ka = (k >> 2) * 16384 + (k & 3) * 32;
                    const uint32_t kb = (k >> 2) * 8192 + (k & 3) * 32;
                    mma_f16(tmem + TP, smem_desc_sw128(at + ka, 16, 1024), smem_desc_sw128(kt + kb, 16, 1024), id,
                            k > 0);
                }
                mma_commit(&ms.bar_p1);
            }
            TC2_MARK(0, 4);
            if (!mwait(&ms.bar_p1, ph)) note_timeout(ms, 2, r);
            TC2_MARK(0, 5);
            tc_fence_after();

            // ---------------------------------------------------- a2: A' and L^T (32 columns per thread)
            {
                const int l = row & 63;
                const bool top = row < 64;
                const int m0 = ch * 32;
                float pr[32];
                __syncwarp();
                tmem_ld32(lane_addr + TP + m0, pr);
                tmem_wait_ld();
                if (GATE == kGateChannel && slow) {
                    const unsigned char *xrow = sm + L::RAW_QK + (top ? 0 : 8192);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int m = m0 + e;
                        float acc = 0.f;
                        if (m <= l) {
#pragma unroll 1
                            for (int c = 0; c < DK; ++c) {
                                const int h = c >> 6;
                                const uint32_t ox = sw128_off(l, c & 63), om = sw128_off(m, c & 63);
                                const void *xp = xrow + h * 16384 + ox, *kp = sm + L::RAW_QK + h * 16384 + 8192 + om;
                                const float xv = qkmap ? __half2float(*reinterpret_cast<const __half *>(xp))
                                                       : __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(xp));
                                const float kv = qkmap ? __half2float(*reinterpret_cast<const __half *>(kp))
                                                       : __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(kp));
                                const float *gt = reinterpret_cast<const float *>(sm + L::GCH);
                                acc = fmaf(xv * kv, __expf(gt[gch_idx(l, c)] - gt[gch_idx(m, c)]), acc);
                            }
                        }
                        pr[e] = l2scale ? acc * (top ? ms.iq[l] : ms.ik[l]) * ms.ik[m] : acc;
                    }
                }
                // decay factors e^{G_l - G_m}: all shared loads first, then the stores
                float dm[32];
                if (GATE == kGateScalar) {
                    if (fastg) {
                        // b_l / b_m (times 1 / |k_m| and the row's 1 / |q_l| or 1 / |k_l|
                        // when rows are made unit)
                        const float bl = ms.b[l] * (l2scale ? (top ? ms.iq[l] : ms.ik[l]) : 1.f);
                        const float *ibm = l2scale ? ms.ibk : ms.ib;
#pragma unroll
                        for (int e = 0; e < 32; e += 4) {
                            const float4 x = *reinterpret_cast<const float4 *>(&ibm[m0 + e]);
                            dm[e] = bl * x.x; dm[e + 1] = bl * x.y; dm[e + 2] = bl * x.z; dm[e + 3] = bl * x.w;
                        }
                    } else {
                        const float Gl = ms.G[l];
#pragma unroll
                        for (int e = 0; e < 32; e += 4) {
                            const float4 x = *reinterpret_cast<const float4 *>(&ms.G[m0 + e]);
                            dm[e] = __expf(Gl - fmaxf(x.x, Gl)); dm[e + 1] = __expf(Gl - fmaxf(x.y, Gl));
                            dm[e + 2] = __expf(Gl - fmaxf(x.z, Gl)); dm[e + 3] = __expf(Gl - fmaxf(x.w, Gl));
                        }
                        if (l2scale) {
                            const float fl = top ? ms.iq[l] : ms.ik[l];
#pragma unroll
                            for (int e = 0; e < 32; ++e) dm[e] *= fl * ms.ik[m0 + e];
                        }
                    }
                } else if (GATE == kGateNone && l2scale) {
                    const float fl = top ? ms.iq[l] : ms.ik[l];
#pragma unroll
                    for (int e = 0; e < 32; ++e) dm[e] = fl * ms.ik[m0 + e];
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) dm[e] = 1.f;
                }
                if (top) {
                    unsigned char *ap = sm + L::TZA + 8192 * (1 + buf);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        pr[e] = (m0 + e <= l) ? pr[e] * dm[e] : 0.f;
                        rmax = fmaxf(rmax, fabsf(pr[e]));
                    }
#pragma unroll
                    for (int e = 0; e < 32; e += 8) *reinterpret_cast<uint4 *>(ap + sw128_off(l, m0 + e)) = pack_h8(pr + e);
                } else if (DELTA) {
                    const float bl = bet[l];
                    float *Lt = reinterpret_cast<float *>(sm + L::KT);
#pragma unroll
                    for (int e = 0; e < 32; ++e) pr[e] = (m0 + e < l) ? bl * pr[e] * dm[e] : 0.f;
#pragma unroll
                    for (int e = 0; e < 32; ++e) Lt[f32_swz(m0 + e, l, 64)] = pr[e];
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(kPrepBar, 256);
            TC2_MARK(0, 6);
            if (GATE == kGateChannel) {
                if (t == 224 && r + 1 < nchunks && !ms.abort_flag) issue_tma(r + 1);
            } else if (!DELTA || warp >= 2) {
                // Q<, K< and V16 (history operands) on warps 2-7 while warps 0-1 run the
                // diagonal solve; then the next chunk's loads (the raw tiles are consumed)
                // and its gate pass (this chunk's factors are no longer read)
                if (DELTA)
                    wait_first_mmas();
                else
                    wait_history();
                TC2_MARK(64, 11);
                {
                    constexpr int NW = DELTA ? 192 : 256;
                    constexpr int NQK = DELTA ? 2048 : 1024;  // q chunks, then (delta) k chunks
                    constexpr int NQV = NQK + (kSplitV ? 0 : 512 * NB);
                    constexpr int IT = (NQV + NW - 1) / NW;
                    const int wt = DELTA ? t - 64 : t;
                    uint4 raw[IT];
#pragma unroll
                    for (int s4 = 0; s4 < IT; ++s4) {
                        const int i = wt + NW * s4;
                        const int j = i & 1023;  // chunk of the q or k tile
                        raw[s4] = make_uint4(0, 0, 0, 0);
                        if (i < NQK)
                            raw[s4] = *reinterpret_cast<const uint4 *>(sm + L::RAW_QK + (j >> 9) * 16384 +
                                                                       (i >> 10) * 8192 + (j & 511) * 16);
                        else if (i < NQV)
                            raw[s4] = *reinterpret_cast<const uint4 *>(sm + L::RAW_V + (i - NQK) * 16);
                    }
#pragma unroll
                    for (int s4 = 0; s4 < IT; ++s4) {
                        const int i = wt + NW * s4;
                        const int j = i & 1023;
                        float f[8];
                        unpack_qk8(raw[s4], f, qkmap && i < NQK);  // v stays bf16
#pragma unroll
                        for (int e = 0; e < 8; ++e) rmax = fmaxf(rmax, fabsf(f[e]));
                        if (i < NQK) {
                            // q -> Q< (i < 1024), k -> K< (delta): row l scaled by b_l = e^{G_l}
                            const int h = j >> 9, off = (j & 511) * 16;
                            float bl = (GATE == kGateScalar) ? ms.b[off >> 7] : 1.f;
                            if (l2scale) bl *= (i < 1024) ? ms.iq[off >> 7] : ms.ik[off >> 7];
#pragma unroll
                            for (int e = 0; e < 8; ++e) f[e] *= bl;
                            *reinterpret_cast<uint4 *>(sm + L::AT + h * 16384 + (i >> 10) * 8192 + off) = pack_h8(f);
                        } else if (i < NQV && !zeroV) {
                            *reinterpret_cast<uint4 *>(sm + v16_slot<L, UPD, GATE>(buf) + (i - NQK) * 16) = pack_h8(f);
                        }
                    }
                }
                TC2_MARK(64, 12);
                fence_proxy_async_smem();
                named_bar(kConvBar, DELTA ? 192 : 256);
                TC2_MARK(64, 13);
                if (t == 224 && r + 1 < nchunks && !ms.abort_flag) issue_tma(r + 1);
                if (!DELTA && r + 1 < nchunks) {
                    gate_pass(r + 1);
                    if (r + 2 < nchunks) load_gate_beta(r + 2);
                }
            }

            if (DELTA) {
                // ------------------------------------------------ a3: T = (I + L)^{-1}
                // The fp32 scratch Ls holds L^T (Ls[m][l] = L[l][m], m < l).  The
                // inverse of a unit lower-triangular matrix is built from its 16x16
                // diagonal blocks (forward substitution, one column per lane), then
                // merged twice, 16 -> 32 -> 64, with T_IJ = -T_II (L_IJ T_JJ) on the
                // warp-level tf32 tensor-core path.  fp32 T blocks go to the diagonal
                // and lower blocks of Ls (its upper blocks keep L^T, which the merges
                // skip); T2 = T diag(beta) goes to the fp16 tile, whose upper blocks
                // stay zero.
                float *Ls = reinterpret_cast<float *>(sm + L::KT);
                unsigned char *t2 = sm + L::TZA;
                if (warp < 2) {
                    // lanes 0-15: block 2w, lanes 16-31: block 2w+1
                    const int o = 16 * (2 * warp + (lane >> 4)), c = lane & 15;
                    float x[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) x[i] = (i == c) ? 1.f : 0.f;
#pragma unroll
                    for (int m = 0; m < 15; ++m) {
                        const float xm = x[m];
#pragma unroll
                        for (int i0 = (m + 1) & ~3; i0 < 16; i0 += 4) {
                            const float4 lv = *reinterpret_cast<const float4 *>(Ls + f32_swz(o + m, o + i0, 64));
                            if (i0 + 0 > m) x[i0 + 0] = fmaf(-lv.x, xm, x[i0 + 0]);
                            if (i0 + 1 > m) x[i0 + 1] = fmaf(-lv.y, xm, x[i0 + 1]);
                            if (i0 + 2 > m) x[i0 + 2] = fmaf(-lv.z, xm, x[i0 + 2]);
                            if (i0 + 3 > m) x[i0 + 3] = fmaf(-lv.w, xm, x[i0 + 3]);
                        }
                    }
                    TC2_MARK(0, 14);
                    wait_history();  // T2 of chunk r-1 has been read
                    __syncwarp();
                    const float bt = bet[o + c];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float tv = x[i] * bt;
                        rmax = fmaxf(rmax, fabsf(tv));
                        Ls[f32_swz(o + i, o + c, 64)] = x[i];
                        *reinterpret_cast<__half *>(t2 + sw128_off(o + i, o + c)) = __float2half_rn(tv);
                    }
                }
                named_bar(kPrepBar, 256);
                TC2_MARK(0, 7);
                const int g = lane >> 2, tq = lane & 3;  // mma fragment coordinates
                if (GATE != kGateChannel && warp >= 4) {
                    // next chunk's gate pass (this chunk's factors were last read by the
                    // conversions before the barrier above)
                    if (r + 1 < nchunks) {
                        gate_pass(r + 1);
                        if (r + 2 < nchunks) load_gate_beta(r + 2);
                    }
                    if (kSplitV && !zeroV) {
                        // V -> fp16 (its slot was released with bar_x(r-1), waited in the
                        // window), then the next chunk's v load
                        if (!mwait(&ms.bar_tv, ph)) note_timeout(ms, 13, r);
                        constexpr int NV = 512 * NB, ITV = NV / 128;
                        const int wt = t - 128;
                        uint4 raw[ITV];
#pragma unroll
                        for (int s4 = 0; s4 < ITV; ++s4)
                            raw[s4] = *reinterpret_cast<const uint4 *>(sm + L::RAW_V + (wt + 128 * s4) * 16);
#pragma unroll
                        for (int s4 = 0; s4 < ITV; ++s4) {
                            float f[8];
                            unpack_bf16x8(raw[s4], f);
#pragma unroll
                            for (int e = 0; e < 8; ++e) rmax = fmaxf(rmax, fabsf(f[e]));
                            *reinterpret_cast<uint4 *>(sm + L::V16 + (wt + 128 * s4) * 16) = pack_h8(f);
                        }
                        fence_proxy_async_smem();
                        named_bar(kVBar, 128);
                        if (t == 224 && r + 1 < nchunks && !ms.abort_flag) issue_tma_split_v(r + 1);
                    }
                }
                if (warp < 4) {
                    // 16 -> 32 for the block pairs (1,0) and (3,2); warp = (pair, 8-column tile)
                    const int pr = warp >> 1, j = warp & 1;
                    const int oJ = 32 * pr, oI = oJ + 16, xr = 32 + 16 * pr;
                    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        const int k0 = oJ + 8 * ks;
                        uint32_t a[4], b[2];
                        a[0] = f2tf32(Ls[f32_swz(k0 + tq, oI + g, 64)]);  // L_IJ[i][k] = Ls[oJ+k][oI+i]
                        a[1] = f2tf32(Ls[f32_swz(k0 + tq, oI + g + 8, 64)]);
                        a[2] = f2tf32(Ls[f32_swz(k0 + tq + 4, oI + g, 64)]);
                        a[3] = f2tf32(Ls[f32_swz(k0 + tq + 4, oI + g + 8, 64)]);
                        b[0] = f2tf32(Ls[f32_swz(k0 + tq, oJ + 8 * j + g, 64)]);  // T_JJ
                        b[1] = f2tf32(Ls[f32_swz(k0 + tq + 4, oJ + 8 * j + g, 64)]);
                        mma_tf32_16x8x8(d, a, b);
                    }
                    // X = L_IJ T_JJ waits in rows 32..63, columns 0..15 (free until the next level)
                    *reinterpret_cast<float2 *>(Ls + f32_swz(xr + g, 8 * j + 2 * tq, 64)) = make_float2(d[0], d[1]);
                    *reinterpret_cast<float2 *>(Ls + f32_swz(xr + g + 8, 8 * j + 2 * tq, 64)) = make_float2(d[2], d[3]);
                    __syncwarp();
                    float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        const int k0 = 8 * ks;
                        uint32_t a[4], b[2];
                        a[0] = f2tf32(Ls[f32_swz(oI + g, oI + k0 + tq, 64)]);  // T_II
                        a[1] = f2tf32(Ls[f32_swz(oI + g + 8, oI + k0 + tq, 64)]);
                        a[2] = f2tf32(Ls[f32_swz(oI + g, oI + k0 + tq + 4, 64)]);
                        a[3] = f2tf32(Ls[f32_swz(oI + g + 8, oI + k0 + tq + 4, 64)]);
                        b[0] = f2tf32(Ls[f32_swz(xr + k0 + tq, 8 * j + g, 64)]);
                        b[1] = f2tf32(Ls[f32_swz(xr + k0 + tq + 4, 8 * j + g, 64)]);
                        mma_tf32_16x8x8(e, a, b);
                    }
                    const int c = oJ + 8 * j + 2 * tq;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float v0 = -e[2 * h], v1 = -e[2 * h + 1];
                        const int row = oI + g + 8 * h;
                        *reinterpret_cast<float2 *>(Ls + f32_swz(row, c, 64)) = make_float2(v0, v1);
                        const float b0 = v0 * bet[c], b1 = v1 * bet[c + 1];
                        rmax = fmaxf(rmax, fmaxf(fabsf(b0), fabsf(b1)));
                        *reinterpret_cast<uint32_t *>(t2 + sw128_off(row, c)) = pack_h2(b0, b1);
                    }
                }
                named_bar(kPrepBar, 256);  // T_10 and T_32 are in Ls
                TC2_MARK(0, 8);
                {
                    // 32 -> 64 on all eight warps: warp = (16-row tile mt, 8-column tile jj) of
                    // T_BA = -T_BB (L_BA T_AA); the two warps of a column tile meet at a
                    // 64-thread barrier to exchange their halves of X = L_BA T_AA
                    const int mt = warp >> 2, jj = warp & 3;
                    const int i0 = 32 + 16 * mt;
                    float dx[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        if (jj >= 2 && ks < 2) continue;  // T_AA[k < 16][c >= 16] = 0
                        const int k0 = 8 * ks;
                        uint32_t a[4], b[2];
                        b[0] = f2tf32(Ls[f32_swz(k0 + tq, 8 * jj + g, 64)]);
                        b[1] = f2tf32(Ls[f32_swz(k0 + tq + 4, 8 * jj + g, 64)]);
                        a[0] = f2tf32(Ls[f32_swz(k0 + tq, i0 + g, 64)]);  // L[i0+i][k] = Ls[k][i0+i]
                        a[1] = f2tf32(Ls[f32_swz(k0 + tq, i0 + g + 8, 64)]);
                        a[2] = f2tf32(Ls[f32_swz(k0 + tq + 4, i0 + g, 64)]);
                        a[3] = f2tf32(Ls[f32_swz(k0 + tq + 4, i0 + g + 8, 64)]);
                        mma_tf32_16x8x8(dx, a, b);
                    }
                    *reinterpret_cast<float2 *>(Ls + f32_swz(i0 + g, 8 * jj + 2 * tq, 64)) = make_float2(dx[0], dx[1]);
                    *reinterpret_cast<float2 *>(Ls + f32_swz(i0 + g + 8, 8 * jj + 2 * tq, 64)) = make_float2(dx[2], dx[3]);
                    named_bar(kPairBar + jj, 64);
                    float ex[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        if (mt == 0 && ks >= 2) continue;  // T_BB[i < 16][k >= 16] = 0
                        const int k0 = 8 * ks;
                        uint32_t a[4], b[2];
                        b[0] = f2tf32(Ls[f32_swz(32 + k0 + tq, 8 * jj + g, 64)]);
                        b[1] = f2tf32(Ls[f32_swz(32 + k0 + tq + 4, 8 * jj + g, 64)]);
                        a[0] = f2tf32(Ls[f32_swz(i0 + g, 32 + k0 + tq, 64)]);
                        a[1] = f2tf32(Ls[f32_swz(i0 + g + 8, 32 + k0 + tq, 64)]);
                        a[2] = f2tf32(Ls[f32_swz(i0 + g, 32 + k0 + tq + 4, 64)]);
                        a[3] = f2tf32(Ls[f32_swz(i0 + g + 8, 32 + k0 + tq + 4, 64)]);
                        mma_tf32_16x8x8(ex, a, b);
                    }
                    const int cc = 8 * jj + 2 * tq;
                    const float bc0 = bet[cc], bc1 = bet[cc + 1];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int row = i0 + g + 8 * h;
                        const float b0 = -ex[2 * h] * bc0, b1 = -ex[2 * h + 1] * bc1;
                        rmax = fmaxf(rmax, fmaxf(fabsf(b0), fabsf(b1)));
                        *reinterpret_cast<uint32_t *>(t2 + sw128_off(row, cc)) = pack_h2(b0, b1);
                    }
                }
                TC2_MARK(0, 9);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            if (t == 0) ms.p_abort = ms.abort_flag;
            named_bar(kPrepBar, 256);
            if (t == 0) mbar_arrive(&ms.bar_rdy);
            TC2_MARK(0, 10);
        }
    } else {
        // =================================================================== state group
        const int ts = t - 256;
        const bool has_row = (DVS == 128) || (lane < 16);
        // P = [Q;K] K^T of chunk r from the raw bf16 tiles, issued by this group's MMA
        // thread (the prep group's threads then never stall on the tensor pipe's queue)
        auto issue_p1 = [&](int r) {
            if (!mwait(&ms.bar_tma, r & 1)) note_timeout(ms, 11, r);
            tc_fence_after();
            const uint32_t qk = smem_u32(sm + L::RAW_QK);
            constexpr uint32_t id = idesc_f16(128, 64, 1, 0, 0);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t ko = (k >> 2) * 16384 + (k & 3) * 32;
                mma_f16(tmem + TP, smem_desc_sw128(qk + ko, 16, 1024), smem_desc_sw128(qk + 8192 + ko, 16, 1024), id,
                        k > 0);
            }
            mma_commit(&ms.bar_p1);
        };
        if (kStateP1 && ts == 0 && nchunks > 0) issue_p1(0);
        const int vrow = (DVS == 128) ? ts : (sp * 16 + lane);
        const size_t srow = ((size_t)bh * dv + v0 + (has_row ? vrow : 0)) * DK;
        // initial state: fp32 master and fp16 operand copy (lane = value row)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float sv[64];
#pragma unroll
            for (int j = 0; j < 64; j += 4) {
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (mode & kModeS0Eye) {
                    // S0 = kEyeScale * I: one entry per row, at column v0 + vrow
                    const int c = h * 64 + j - (v0 + vrow);
                    constexpr float e = kEyeScale;
                    x = make_float4(c == 0 ? e : 0.f, c == -1 ? e : 0.f, c == -2 ? e : 0.f, c == -3 ? e : 0.f);
                    if (!has_row) x = make_float4(0.f, 0.f, 0.f, 0.f);
                } else if (p.S0 && has_row) {
                    x = *reinterpret_cast<const float4 *>(p.S0 + srow + h * 64 + j);
                }
                sv[j] = x.x; sv[j + 1] = x.y; sv[j + 2] = x.z; sv[j + 3] = x.w;
            }
            if ((mode & kModeSaveStates) && has_row && nchunks > 0) {  // the state entering chunk 0
                float *st = p.states + ((size_t)bh * nchunks * dv + v0 + vrow) * DK + h * 64;
#pragma unroll
                for (int j = 0; j < 64; j += 4)
                    __stcs(reinterpret_cast<float4 *>(st + j), make_float4(sv[j], sv[j + 1], sv[j + 2], sv[j + 3]));
            }
            __syncwarp();
            tmem_st32f(lane_addr + TSM + h * 64, sv);
            tmem_st32f(lane_addr + TSM + h * 64 + 32, sv + 32);
            uint32_t w[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) w[c] = pack_h2(sv[2 * c], sv[2 * c + 1]);
            tmem_st32(lane_addr + TS16 + h * 32, w);
        }
        tmem_wait_st();
        tc_fence_before();
        named_bar(kStateBar, 128);

        // the first chunk's decay is applied here; later ones ride on the fp16
        // write-back at the end of the previous chunk
        if (nchunks > 0) {
            if (!mwait(&ms.bar_rdy, 0)) note_timeout(ms, 6, 0);
            tc_fence_after();
            if (GATE != kGateNone) {
#pragma unroll
                for (int j0 = 0; j0 < 128; j0 += 32) {
                    float sv[32];
                    __syncwarp();
                    tmem_ld32(lane_addr + TSM + j0, sv);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) sv[i] *= (GATE == kGateScalar) ? dec[0] : dec[j0 + i];
                    tmem_st32f(lane_addr + TSM + j0, sv);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            named_bar(kStateBar, 128);
        }
        float *ost = reinterpret_cast<float *>(sm + L::OST);
        for (int r = 0; r < nchunks; ++r) {
            if (ms.s_abort) break;
            const uint32_t ph = r & 1;
            const int t0 = r * CV;
            const int buf = r & 1;
            if (GATE != kGateChannel && r > 0) {
                if (!mwait(&ms.bar_rdy, ph)) note_timeout(ms, 6, r);
                tc_fence_after();
            }
            TC2_MARK(256, 17);
            if (ts == 0 && !ms.abort_flag) {
                tc_fence_after();
                // P1 of the next chunk goes to the tensor pipe first: the prep group
                // released TP with rdy(r) and waits on P1 before its A'/L pass
                if (kStateP1 && r + 1 < nchunks) issue_p1(r + 1);
                const uint32_t at = smem_u32(sm + L::AT);
                if (DELTA) {
                    // [O^T | X^T] = S [Q< ; K<]^T in one N = 128 chain (the two B tiles are
                    // adjacent in each key half); Z^T = V^T T2^T (U^T) alongside
                    const uint32_t v16 = smem_u32(sm + L::V16), tza = smem_u32(sm + L::TZA);
                    constexpr uint32_t id1w = idesc_f16(DVS, 128, 0, 0, 0);
                    constexpr uint32_t idu = idesc_f16(DVS, 64, 0, 1, 0);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_f16_ts(tmem + TOX, tmem + TS16 + k * 8,
                                   smem_desc_sw128(at + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024), id1w, k > 0);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_f16(tmem + TZ, smem_desc_sw128(v16 + k * 2048, 8192, 1024),
                                smem_desc_sw128(tza + k * 32, 16, 1024), idu, k > 0);
                    mma_commit(&ms.bar_x);
                } else {
                    constexpr uint32_t id1 = idesc_f16(DVS, 64, 0, 0, 0);
#pragma unroll
                    for (int k = 0; k < 8; ++k)  // O^T = S Q<^T
                        mma_f16_ts(tmem + TOX, tmem + TS16 + k * 8,
                                   smem_desc_sw128(at + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024), id1, k > 0);
                    mma_commit(&ms.bar_fA);
                    // without the delta rule nothing sits between: O^T += V^T A'^T and
                    // S += V^T K> follow at once (S is read from its fp16 copy above)
                    const uint32_t tza = smem_u32(sm + L::TZA), kr = smem_u32(sm + L::KR) + buf * 16384;
                    const uint32_t ap = tza + 8192 * (1 + buf);
                    const uint32_t v16 = smem_u32(sm + v16_slot<L, UPD, GATE>(buf));
                    constexpr uint32_t id2s = idesc_f16(DVS, 64, 0, 1, 0);
                    constexpr uint32_t id3s = idesc_f16(DVS, 128, 0, 1, 1);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t va = smem_desc_sw128(v16 + k * 2048, 8192, 1024);
                        mma_f16(tmem + TOX, va, smem_desc_sw128(ap + k * 32, 16, 1024), id2s, 1);
                        mma_f16(tmem + TSM, va, smem_desc_sw128(kr + k * 2048, 8192, 1024), id3s, 1);
                    }
                    mma_commit(buf ? &ms.bar_fB1 : &ms.bar_fB0);
                }
            }
            TC2_MARK(256, 18);
            if (DELTA) {
                // history correction Z^T = U^T - (S K<^T) T2^T: X^T = S K<^T leaves TMEM as
                // -X^T in fp16 (the A operand of the product with T2)
                if (!mwait(&ms.bar_x, ph)) note_timeout(ms, 3, r);
                tc_fence_after();
                {
                    float x[64];
                    __syncwarp();
                    tmem_ld32(lane_addr + TOX + 64, x);
                    tmem_ld32(lane_addr + TOX + 96, x + 32);
                    tmem_wait_ld();
                    uint32_t w[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        rmax = fmaxf(rmax, fmaxf(fabsf(x[2 * c]), fabsf(x[2 * c + 1])));
                        w[c] = pack_h2(-x[2 * c], -x[2 * c + 1]);
                    }
                    tmem_st32(lane_addr + TZ16, w);
                    tmem_wait_st();
                }
                tc_fence_before();
                named_bar(kStateBar, 128);
                if (ts == 0 && !ms.abort_flag) {
                    tc_fence_after();
                    const uint32_t tza = smem_u32(sm + L::TZA);
                    constexpr uint32_t idz = idesc_f16(DVS, 64, 0, 0, 0);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_f16_ts(tmem + TZ, tmem + TZ16 + k * 8, smem_desc_sw128(tza + k * 32, 16, 1024), idz, 1);
                    mma_commit(&ms.bar_fA);
                }
            }
            if (DELTA) {
                if (!mwait(&ms.bar_fA, ph)) note_timeout(ms, 7, r);
            }
            TC2_MARK(256, 19);
            tc_fence_after();
            if (DELTA) {
                // Z^T -> fp16 A operand (tokens 2c, 2c+1 in column c)
                float z[64];
                __syncwarp();
                tmem_ld32(lane_addr + TZ, z);
                tmem_ld32(lane_addr + TZ + 32, z + 32);
                tmem_wait_ld();
                uint32_t w[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    rmax = fmaxf(rmax, fmaxf(fabsf(z[2 * c]), fabsf(z[2 * c + 1])));
                    w[c] = pack_h2(z[2 * c], z[2 * c + 1]);
                }
                tmem_st32(lane_addr + TZ16, w);
                tmem_wait_st();
                tc_fence_before();
                named_bar(kStateBar, 128);
            }
            TC2_MARK(256, 20);
            uint64_t *fb = buf ? &ms.bar_fB1 : &ms.bar_fB0;
            if (DELTA && ts == 0 && !ms.abort_flag) {
                tc_fence_after();
                const uint32_t tza = smem_u32(sm + L::TZA), kr = smem_u32(sm + L::KR) + buf * 16384;
                const uint32_t ap = tza + 8192 * (1 + buf);
                constexpr uint32_t id2 = idesc_f16(DVS, 64, 0, 0, 0);
                constexpr uint32_t id3 = idesc_f16(DVS, 128, 0, 0, 1);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t za = tmem + TZ16 + k * 8;
                    mma_f16_ts(tmem + TOX, za, smem_desc_sw128(ap + k * 32, 16, 1024), id2, 1);
                    mma_f16_ts(tmem + TSM, za, smem_desc_sw128(kr + k * 2048, 8192, 1024), id3, 1);
                }
                mma_commit(fb);
            }
            TC2_MARK(256, 21);
            if (!mwait(fb, (r >> 1) & 1)) note_timeout(ms, 8, r);
            TC2_MARK(256, 22);
            tc_fence_after();
            if (!(mode & kModeNoOut)) {
                // O^T -> row-major staging [64 tok][DVS] -> one TMA store (rows past T
                // clipped).  Stores issued straight from registers were measured slower:
                // they queue behind the prep group's shared-memory traffic.
                float ov[64];
                __syncwarp();
                tmem_ld32(lane_addr + TOX, ov);
                tmem_ld32(lane_addr + TOX + 32, ov + 32);
                tmem_wait_ld();
                if (ts == 0) bulk_wait_read0();  // the previous chunk's store has read the staging tile
                named_bar(kStateBar, 128);
                if (has_row && PROD) {
                    // each token's last substep, compacted to one row per token
                    const unsigned long long lm = p.lastmask;
                    int row = 0;
#pragma unroll
                    for (int l = 0; l < 64; ++l) {
                        if (!((lm >> l) & 1)) continue;
                        if (OUT_BF16)
                            reinterpret_cast<__nv_bfloat16 *>(ost)[row * DVS + vrow] = __float2bfloat16_rn(ov[l]);
                        else
                            ost[row * DVS + vrow] = ov[l];
                        ++row;
                    }
                } else if (has_row) {
                    if (OUT_BF16) {
                        __nv_bfloat16 *ob = reinterpret_cast<__nv_bfloat16 *>(ost);
#pragma unroll
                        for (int l = 0; l < 64; ++l) ob[l * DVS + vrow] = __float2bfloat16_rn(ov[l]);
                    } else {
#pragma unroll
                        for (int l = 0; l < 64; ++l) ost[l * DVS + vrow] = ov[l];
                    }
                }
                fence_proxy_async_smem();
                named_bar(kStateBar, 128);
                if (ts == 0) {
                    tma_store_3d(&p.o_map, ost, v0, PROD ? r * TPC : t0, bh);
                    bulk_commit();
                }
            }
            TC2_MARK(256, 23);
            // fp16 copy of the new state for the next chunk's history read; the
            // next chunk's decay is applied to the fp32 state in the same pass
            const bool more = r + 1 < nchunks;
            // the channel gate's decay of chunk r+1 comes from that chunk's prep; the
            // scalar gate's was published with rdy(r) (the prep group runs a chunk's
            // gate pass one chunk early), so S16 and the decay need not wait
            if (GATE == kGateChannel && more) {
                if (!mwait(&ms.bar_rdy, (r + 1) & 1)) note_timeout(ms, 6, r + 1);
                tc_fence_after();
            }
            TC2_MARK(256, 25);
            const int nbuf = buf ^ 1;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float sv[64];
                __syncwarp();
                tmem_ld32(lane_addr + TSM + h * 64, sv);
                tmem_ld32(lane_addr + TSM + h * 64 + 32, sv + 32);
                tmem_wait_ld();
                uint32_t w[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    rmax = fmaxf(rmax, fmaxf(fabsf(sv[2 * c]), fabsf(sv[2 * c + 1])));
                    w[c] = pack_h2(sv[2 * c], sv[2 * c + 1]);
                }
                tmem_st32(lane_addr + TS16 + h * 32, w);
                if ((mode & kModeSaveStates) && has_row && more) {  // the state entering chunk r + 1
                    float *st = p.states + (((size_t)bh * nchunks + r + 1) * dv + v0 + vrow) * DK + h * 64;
#pragma unroll
                    for (int j = 0; j < 64; j += 4)
                        __stcs(reinterpret_cast<float4 *>(st + j), make_float4(sv[j], sv[j + 1], sv[j + 2], sv[j + 3]));
                }
                if (GATE != kGateNone && more) {
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        sv[i] *= (GATE == kGateScalar) ? dec[nbuf * 128] : dec[nbuf * 128 + h * 64 + i];
                    tmem_st32f(lane_addr + TSM + h * 64, sv);
                    tmem_st32f(lane_addr + TSM + h * 64 + 32, sv + 32);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            if (ts == 0) ms.s_abort = ms.abort_flag;
            named_bar(kStateBar, 128);
            TC2_MARK(256, 24);
        }
        if (ts == 0) bulk_wait0();  // o is in global memory before the kernel ends
        // final state
        if (!ms.s_abort && p.ST) {
            const float osc = (mode & kModeS0Eye) ? 1.f / kEyeScale : 1.f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float sv[64];
                __syncwarp();
                tmem_ld32(lane_addr + TSM + h * 64, sv);
                tmem_ld32(lane_addr + TSM + h * 64 + 32, sv + 32);
                tmem_wait_ld();
                if (has_row) {
#pragma unroll
                    for (int j = 0; j < 64; j += 4)
                        *reinterpret_cast<float4 *>(p.ST + srow + h * 64 + j) =
                            make_float4(sv[j] * osc, sv[j + 1] * osc, sv[j + 2] * osc, sv[j + 3] * osc);
                }
            }
        }
    }

    if (!(rmax <= 65504.f)) ms.range_flag = 1;
    __syncthreads();
    if (ms.abort_flag) {
        // a wait ran out: let every MMA and TMA load this CTA issued land before
        // its TMEM and shared memory are released (each wait bounded at 1 s)
        if (t == 0 || t == 256) mma_commit(&ms.bar_drain);  // the two MMA-issuing threads
        if (t == 0) {
            mbar_wait(&ms.bar_drain, 0);
            if (ms.n_tma > 0) mbar_wait(&ms.bar_tma, (ms.n_tma - 1) & 1);
            if (ms.n_tv > 0) mbar_wait(&ms.bar_tv, (ms.n_tv - 1) & 1);
        }
        __syncthreads();
    }
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

template <int DVS, int UPD, int GATE, bool OB, bool PROD = false>
int launch_one(const Params &prm, int grid, cudaStream_t stream) {
    using L = Smem<DVS, GATE>;
    auto kern = (prm.pro != 0 || prm.mode != 0 || prm.wait_ns != 0) ? chunk_tc2_kernel<DVS, UPD, GATE, OB, PROD, true>
                                                : chunk_tc2_kernel<DVS, UPD, GATE, OB, PROD, false>;
    static_assert(L::DYN <= 232448, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::DYN);
    if (e != cudaSuccess) return (int)e;
    kern<<<grid, kThreads, L::DYN, stream>>>(prm);
    return (int)cudaGetLastError();
}

template <int DVS, int UPD, int GATE>
int launch_out(const Params &prm, int grid, bool ob, cudaStream_t s) {
    return ob ? launch_one<DVS, UPD, GATE, true>(prm, grid, s) : launch_one<DVS, UPD, GATE, false>(prm, grid, s);
}

template <int DVS, int GATE>
int launch_prod(const Params &prm, int grid, bool ob, cudaStream_t s) {
    return ob ? launch_one<DVS, kDelta, GATE, true, true>(prm, grid, s)
              : launch_one<DVS, kDelta, GATE, false, true>(prm, grid, s);
}

template <int DVS>
int launch_modes(const Params &prm, int grid, int update, int gate, bool ob, cudaStream_t s) {
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
extern "C" int gdn_tc2_phase_times(unsigned long long *out, int clear) {
    cudaDeviceSynchronize();
    if (cudaMemcpyFromSymbol(out, g_tc2_phase, sizeof(unsigned long long) * 32) != cudaSuccess) return -1;
    if (clear) {
        unsigned long long z[32] = {0};
        cudaMemcpyToSymbol(g_tc2_phase, z, sizeof(z));
    }
    return 0;
}
#endif

unsigned long long gdn_wait_limit_ns();  // api.cu

int gdn_tc_supported(const gdn_desc_t *d) {
    return d->dtype == GDN_BF16 && d->dk == 128 && (d->dv == 64 || d->dv == 128);
}

// Value-slice width: 128 keeps the per-chunk K-side work unduplicated; 64
// doubles the CTA count when 128-wide slices would leave most SMs idle.
static int tc2_slice(const gdn_desc_t *d) {
    const long bh = (long)d->B * d->H;
    if (d->dv == 64 || d->gate == GDN_GATE_CHANNEL) return 64;
    return (bh * 2 <= gdn::gdn_sm_count()) ? 64 : 128;
}

int gdn_launch_chunk_tc2(const gdn::ChunkArgs &a, const gdn_desc_t *d, cudaStream_t stream) {
    using namespace gdn;
    Params prm;
    memset(&prm, 0, sizeof(prm));
    const uint64_t BH = (uint64_t)a.BH, T = (uint64_t)a.T;
    // Gated DeltaProduct: T counts virtual steps; q and o have T / nh token rows, a
    // chunk holds rows = 64 / nh whole tokens
    const int nh = a.nh;
    if (nh < 1 || nh > 64) return (int)cudaErrorInvalidValue;
    const uint64_t Tr = T / nh;
    const uint32_t rows = 64u / nh;
    if (!make_map_3d(&prm.q_map, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 128, Tr, BH, 64, rows, 1, true) ||
        !make_map_3d(&prm.k_map, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 128, T, BH, 64, 64, 1, true))
        return (int)cudaErrorInvalidValue;
    if (!(a.mode & kModeZeroV) &&
        !make_map_3d(&prm.v_map, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.dv, T, BH, 64, 64, 1, true))
        return (int)cudaErrorInvalidValue;
    if (d->gate == GDN_GATE_CHANNEL &&
        !make_map_3d(&prm.g_map, a.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 128, Tr, BH, 32, rows, 1, true))
        return (int)cudaErrorInvalidValue;
    const int dvs = tc2_slice(d);
    const bool ob = d->out_dtype == GDN_BF16;
    if (!(a.mode & kModeNoOut) &&
        !make_map_3d(&prm.o_map, a.o, ob ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                     ob ? 2 : 4, (uint64_t)a.dv, Tr, BH, (uint32_t)dvs, rows, 1, false))
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
    prm.nslices = a.dv / dvs;
    prm.nh = nh;
    prm.tpc = (int)rows;
    prm.cv = (int)rows * nh;
    for (int l = 0; l < prm.cv; ++l) {
        if (l % nh == 0) prm.firstmask |= 1ull << l;
        if (l % nh == nh - 1) prm.lastmask |= 1ull << l;
    }
    prm.pro = a.pro;
    prm.mode = a.mode;
    prm.states = a.states;
    prm.wait_ns = gdn_wait_limit_ns();
    const long grid = (long)a.BH * prm.nslices;
    if (grid == 0) return 0;
    if (nh > 1) {
        if (d->gate == GDN_GATE_CHANNEL) return launch_prod<64, kGateChannel>(prm, (int)grid, ob, stream);
        if (dvs == 64)
            return d->gate == GDN_GATE_SCALAR ? launch_prod<64, kGateScalar>(prm, (int)grid, ob, stream)
                                              : launch_prod<64, kGateNone>(prm, (int)grid, ob, stream);
        return d->gate == GDN_GATE_SCALAR ? launch_prod<128, kGateScalar>(prm, (int)grid, ob, stream)
                                          : launch_prod<128, kGateNone>(prm, (int)grid, ob, stream);
    }
    if (dvs == 64) return launch_modes<64>(prm, (int)grid, d->update, d->gate, ob, stream);
    return launch_modes<128>(prm, (int)grid, d->update, d->gate, ob, stream);
}
