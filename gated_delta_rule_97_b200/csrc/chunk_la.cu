// Plain causal linear attention (additive write, no gate) on tcgen05 tensor
// cores: the chunkwise form of "Linear Attention, Visualized", "Linear
// attention: a running sum" and "Chunkwise parallel form".  Per chunk r of
// C = 128 tokens, with S the running state [dv][dk]:
//
//     O_r = Q_r S^T + tril(Q_r K_r^T) V_r,      S <- S + V_r^T K_r
//
// One CTA per (head, 64-row value slice).  S stays fp32 in tensor memory for
// the whole sequence; before each chunk a bf16 copy of it goes to shared
// memory, the B operand of O = Q S^T, whose A operand is the raw bf16 Q tile.
// P = Q K^T is masked in place in tensor memory (bf16, the A operand of P V).
// O has the chunk's tokens on the TMEM lanes; the epilogue writes each token's
// row into a swizzled staging tile that TMA stores drain while the next chunk
// runs.  A tcgen05 MMA here costs
// about the same for N = 64 and N = 128 (its issue, not its arithmetic, sets
// the time), so the chunk is 128 tokens (two 64-row TMA boxes per tile), which
// halves the MMAs per token.  The result does not depend on the chunk length.
// Roles:
//   warp 0      TMA producer (q, k, v tiles; two stages)
//   warp 1      MMA issuer (one thread)
//   warps 4-7   element-wise group: the O epilogue (lane = token), the mask of
//               P to tril bf16 (lane = token), the bf16 copy of S and the
//               initial and final state (lane = value row)
// Per chunk the MMA thread issues O = Q S16^T + P V (two O buffers), then P of
// the next chunk, then S += V^T K.  The element-wise group masks that P while
// S runs, copies S as soon as it lands, and only then stores O, so the copy
// of S is all that lies between one chunk's MMAs and the next.
// Every wait is bounded: one that runs out records GDN_ERR_TIMEOUT; the roles
// then leave their loops (the element-wise group decides by a barrier vote, so
// that its threads leave together), let their copies and MMAs land, and return.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "gdn.h"
#include "sm100.cuh"
#include "tc_util.cuh"
#include "tma_host.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kLAThreads = 256;
constexpr int kLAStages = 2;
constexpr int kLAC = 128;  // chunk length of this kernel
constexpr int kEwBar = 1;  // named barrier of the element-wise group

struct LAParams {
    CUtensorMap q_map, k_map, v_map, o_map;
    const float *S0;
    float *ST;
    int *status;
    int BH, T, dv, nslices;
    unsigned long long wait_ns;  // bound of the hand-off waits (gdn_set_wait_limit_ns)
};

// Stage: Q then K, each [2 key halves][128 rows][64] bf16 (16 KB per half),
// then V [128 rows][64] bf16; every tile 128-byte swizzled.
struct LASmem {
    static constexpr int Q = 0, K = 32768, V = 65536;
    static constexpr int STAGE = 65536 + 16384;
    static constexpr int S16 = kLAStages * STAGE;  // S bf16 [2 key halves][64 value rows][64]
    static constexpr int OST = S16 + 16384;        // O staging: fp32 [2][128 tokens][32] or bf16 [128][64]
    static constexpr int TOTAL = OST + 32768;
    static constexpr int DYN = TOTAL + 1024;      // room to align the base to 1024 bytes
};
constexpr int kDVS = 64;  // value rows per CTA

struct LABars {
    uint64_t full[kLAStages], empty[kLAStages];
    uint64_t s16rdy, pmrdy, pfull, ofull[2], oempty[2], sdone, drain;
    uint32_t tmem_base;
    int abort_flag;
};

// TMEM columns: S fp32 (128; M = 64 layout, value row 16 w + l on lane 32 w + l),
// O x 2 (lanes = tokens, 64 value columns each), P fp32 (lanes = tokens, 128
// columns) and its masked bf16 form (64 columns of pairs).
constexpr uint32_t kTS = 0, kTO = 128, kTP = 256, kTP16 = 384, kTCols = 512;

__device__ __forceinline__ uint32_t pack_bf2(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// TW: a test's short wait bound (gdn_set_wait_limit_ns), compiled in only for it.
template <bool OB, bool TW>
__global__ void __launch_bounds__(kLAThreads, 1) chunk_la_kernel(const __grid_constant__ LAParams p) {
    using L = LASmem;
    constexpr int DVS = kDVS;
    extern __shared__ unsigned char dsm_raw[];
    // 1024-byte aligned by an offset on the shared pointer (a cast through an integer
    // would turn every access into a generic one)
    unsigned char *sm = dsm_raw + ((1024u - (smem_u32(dsm_raw) & 1023u)) & 1023u);
    __shared__ LABars bs;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int bh = blockIdx.x / p.nslices, v0 = (blockIdx.x % p.nslices) * DVS;
    const int n = (p.T + kLAC - 1) / kLAC;

    if (t == 0) {
        for (int i = 0; i < kLAStages; ++i) {
            mbar_init(&bs.full[i], 1);
            mbar_init(&bs.empty[i], 1);
        }
        mbar_init(&bs.s16rdy, 1);
        mbar_init(&bs.pmrdy, 1);
        mbar_init(&bs.pfull, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bs.ofull[i], 1);
            mbar_init(&bs.oempty[i], 1);
        }
        mbar_init(&bs.sdone, 1);
        mbar_init(&bs.drain, 1);
        bs.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&bs.tmem_base, kTCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bs.tmem_base;

    // a wait that runs out stops every role (each then finds its next wait cut
    // short too); the waits on the chunk-to-chunk chain poll without suspending
    auto wait = [&](uint64_t *bar, uint32_t par) -> bool {
        if (mbar_test_wait(bar, par)) return true;
        if (*reinterpret_cast<volatile int *>(&bs.abort_flag)) return false;
        if (TW ? mbar_wait_bounded(bar, par, p.wait_ns) : mbar_wait_spin(bar, par)) return true;
        if (atomicExch(&bs.abort_flag, 1) == 0) record_status(p.status, kStatusTimeout);
        return false;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&p.q_map);
            tma_prefetch_desc(&p.k_map);
            tma_prefetch_desc(&p.v_map);
            int issued = 0;
            for (int r = 0; r < n; ++r) {
                const int s = r & 1;
                if (r >= kLAStages && !wait(&bs.empty[s], ((r >> 1) - 1) & 1)) break;
                unsigned char *st = sm + s * L::STAGE;
                mbar_arrive_expect_tx(&bs.full[s], L::STAGE);
                for (int rb = 0; rb < 2; ++rb) {  // 64-row blocks of the chunk
                    const int y = r * kLAC + rb * 64;
                    for (int h = 0; h < 2; ++h) {
                        tma_load_3d(st + L::Q + h * 16384 + rb * 8192, &p.q_map, h * 64, y, bh, &bs.full[s]);
                        tma_load_3d(st + L::K + h * 16384 + rb * 8192, &p.k_map, h * 64, y, bh, &bs.full[s]);
                    }
                    tma_load_3d(st + L::V + rb * 8192, &p.v_map, v0, y, bh, &bs.full[s]);
                }
                issued = r + 1;
            }
            // no copy may still be landing when the CTA leaves
            for (int r = issued - kLAStages < 0 ? 0 : issued - kLAStages; r < issued; ++r)
                mbar_wait(&bs.full[r & 1], (r >> 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_p = idesc_f16(128, 128, 1, 0, 0);   // Q K^T
            constexpr uint32_t id_o1 = idesc_f16(128, DVS, 1, 0, 0);  // Q S16^T
            constexpr uint32_t id_o2 = idesc_f16(128, DVS, 1, 0, 1);  // P16 V
            constexpr uint32_t id_s = idesc_f16(DVS, 128, 1, 1, 1);   // V^T K
            auto issue_p = [&](int r) {
                const uint32_t st = smem_u32(sm + (r & 1) * L::STAGE);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t ko = (k >> 2) * 16384 + (k & 3) * 32;
                    mma_f16(tmem + kTP, smem_desc_sw128(st + L::Q + ko, 16, 1024),
                            smem_desc_sw128(st + L::K + ko, 16, 1024), id_p, k > 0);
                }
                mma_commit(&bs.pfull);
            };
            bool ok = n > 0 && wait(&bs.full[0], 0);
            tc_fence_after();
            if (ok) issue_p(0);
            for (int r = 0; ok && r < n; ++r) {
                const int s = r & 1;
                if (!wait(&bs.s16rdy, r & 1) || !wait(&bs.pmrdy, r & 1)) break;
                if (r >= 2 && !wait(&bs.oempty[s], ((r >> 1) - 1) & 1)) break;
                tc_fence_after();
                const uint32_t to = tmem + kTO + s * 64;
                const uint32_t st = smem_u32(sm + s * L::STAGE);
                const uint32_t s16 = smem_u32(sm + L::S16);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_f16(to, smem_desc_sw128(st + L::Q + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                            smem_desc_sw128(s16 + (k >> 2) * 8192 + (k & 3) * 32, 16, 1024), id_o1, k > 0);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_f16_ts(to, tmem + kTP16 + 8 * k, smem_desc_sw128(st + L::V + k * 2048, 16384, 1024),
                               id_o2, 1);
                mma_commit(&bs.ofull[s]);
                if (r + 1 < n) {
                    if (!wait(&bs.full[(r + 1) & 1], ((r + 1) >> 1) & 1)) break;
                    tc_fence_after();
                    issue_p(r + 1);
                }
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_f16(tmem + kTS, smem_desc_sw128(st + L::V + k * 2048, 16384, 1024),
                            smem_desc_sw128(st + L::K + k * 2048, 16384, 1024), id_s, 1);
                mma_commit(&bs.empty[s]);
                mma_commit(&bs.sdone);
            }
            // every MMA issued so far has finished before the CTA frees its TMEM
            mma_commit(&bs.drain);
            mbar_wait(&bs.drain, 0);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ element-wise group
        const int e = t - 128, sp = warp & 3;
        const int row = sp * 32 + lane;  // TMEM lane: a token of the chunk (P, O)
        const uint32_t lane_addr = tmem + ((uint32_t)(sp * 32) << 16);
        const bool has_row = lane < 16;  // S has 64 value rows, 16 per warp (M = 64)
        const int vrow = sp * 16 + lane;
        const size_t srow = ((size_t)bh * p.dv + v0 + (has_row ? vrow : 0)) * 128;

        // value row vrow of S (128 fp32) -> row vrow of the bf16 copy in shared memory
        auto store_s16 = [&](const float *sv) {
            if (has_row) {
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const uint32_t w0 = pack_bf2(sv[8 * c], sv[8 * c + 1]), w1 = pack_bf2(sv[8 * c + 2], sv[8 * c + 3]);
                    const uint32_t w2 = pack_bf2(sv[8 * c + 4], sv[8 * c + 5]), w3 = pack_bf2(sv[8 * c + 6], sv[8 * c + 7]);
                    *reinterpret_cast<uint4 *>(sm + L::S16 + (c >> 3) * 8192 + vrow * 128 + (((c & 7) ^ (vrow & 7)) << 4)) =
                        make_uint4(w0, w1, w2, w3);
                }
            }
            fence_proxy_async_smem();
        };
        // initial state: fp32 into S, and its bf16 copy for chunk 0
        {
            float s0[128];
#pragma unroll
            for (int j = 0; j < 128; j += 4) {
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (p.S0 && has_row) x = *reinterpret_cast<const float4 *>(p.S0 + srow + j);
                s0[j] = x.x; s0[j + 1] = x.y; s0[j + 2] = x.z; s0[j + 3] = x.w;
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_st32f(lane_addr + kTS + c * 32, s0 + c * 32);
            tmem_wait_st();
            store_s16(s0);
        }
        tc_fence_before();
        named_bar(kEwBar, 128);
        if (e == 0) mbar_arrive(&bs.s16rdy);

        auto epilogue = [&](int r) -> bool {
            const int b = r & 1;
            if (!named_bar_and(kEwBar, 128, wait(&bs.ofull[b], (r >> 1) & 1))) return false;
            tc_fence_after();
            float ov[DVS];
            tmem_ld32(lane_addr + kTO + b * 64, ov);
            tmem_ld32(lane_addr + kTO + b * 64 + 32, ov + 32);
            tmem_wait_ld();
            if (e == 0) bulk_wait_read0();  // the previous chunk's stores have read the staging tile
            tc_fence_before();
            named_bar(kEwBar, 128);
            if (e == 0) mbar_arrive(&bs.oempty[b]);
            // row = token; 16-byte slot c of a 128-byte staging row sits at c ^ (row % 8)
            if (OB) {
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4 *>(sm + L::OST + row * 128 + ((c ^ (row & 7)) << 4)) =
                        make_uint4(pack_bf2(ov[8 * c], ov[8 * c + 1]), pack_bf2(ov[8 * c + 2], ov[8 * c + 3]),
                                   pack_bf2(ov[8 * c + 4], ov[8 * c + 5]), pack_bf2(ov[8 * c + 6], ov[8 * c + 7]));
            } else {
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    *reinterpret_cast<float4 *>(sm + L::OST + (c >> 3) * 16384 + row * 128 + (((c & 7) ^ (row & 7)) << 4)) =
                        make_float4(ov[4 * c], ov[4 * c + 1], ov[4 * c + 2], ov[4 * c + 3]);
            }
            fence_proxy_async_smem();
            named_bar(kEwBar, 128);
            if (e == 0) {
                // rows past the end of the sequence are clipped by the tensor map
                if (OB) {
                    tma_store_3d(&p.o_map, sm + L::OST, v0, r * kLAC, bh);
                } else {
                    tma_store_3d(&p.o_map, sm + L::OST, v0, r * kLAC, bh);
                    tma_store_3d(&p.o_map, sm + L::OST + 16384, v0 + 32, r * kLAC, bh);
                }
                bulk_commit();
            }
            return true;
        };

        // P(r) = Q K^T -> tril bf16 in place (row t = TMEM lane, columns s)
        auto mask_p = [&](int r) -> bool {
            if (!named_bar_and(kEwBar, 128, wait(&bs.pfull, r & 1))) return false;
            tc_fence_after();
            float pv[kLAC];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(lane_addr + kTP + c * 32, pv + c * 32);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t w[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int s0 = 64 * h + 2 * j;
                    w[j] = pack_bf2(s0 <= row ? pv[s0] : 0.f, s0 + 1 <= row ? pv[s0 + 1] : 0.f);
                }
                tmem_st32(lane_addr + kTP16 + h * 32, w);
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar(kEwBar, 128);
            if (e == 0) mbar_arrive(&bs.pmrdy);
            return true;
        };

        bool ok = n == 0 || mask_p(0);
        for (int r = 0; ok && r < n; ++r) {
            // in the order the MMAs finish: O(r), P(r + 1), S(r)
            if (r + 1 < n) {
                if (!mask_p(r + 1)) { ok = false; break; }
                // the bf16 copy of S for chunk r + 1, once S(r) is in
                if (!named_bar_and(kEwBar, 128, wait(&bs.sdone, r & 1))) { ok = false; break; }
                tc_fence_after();
                float sv[128];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(lane_addr + kTS + c * 32, sv + c * 32);
                tmem_wait_ld();
                store_s16(sv);
                tc_fence_before();
                named_bar(kEwBar, 128);
                if (e == 0) mbar_arrive(&bs.s16rdy);
            }
            if (!epilogue(r)) { ok = false; break; }
        }
        if (e == 0) bulk_wait0();  // every O tile is in global memory
        // final state (the TMEM loads are warp-collective: every lane takes them,
        // and the group decides together whether to)
        if (ok && n > 0) ok = wait(&bs.sdone, (n - 1) & 1);
        ok = named_bar_and(kEwBar, 128, ok);
        tc_fence_after();
        if (ok && p.ST) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float sv[32];
                tmem_ld32(lane_addr + kTS + c * 32, sv);
                tmem_wait_ld();
                if (has_row) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4 *>(p.ST + srow + c * 32 + j) =
                            make_float4(sv[j], sv[j + 1], sv[j + 2], sv[j + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTCols);
    }
}

template <bool OB, bool TW>
int launch_la(const LAParams &prm, int grid, cudaStream_t stream) {
    auto kern = chunk_la_kernel<OB, TW>;
    constexpr int smem = LASmem::DYN;
    static_assert(smem <= 232448, "shared memory of one CTA");
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return (int)e;
    kern<<<grid, kLAThreads, smem, stream>>>(prm);
    return (int)cudaGetLastError();
}

}  // namespace
}  // namespace gdn

unsigned long long gdn_wait_limit_ns();  // api.cu

// The request this kernel serves: additive update without gate, bf16 inputs,
// dk = 128, dv in {64, 128}, no input prologue, a plain forward (no internal
// pass mode).
int gdn_la_supported(const gdn_desc_t *d, int mode) {
    return d->update == GDN_ADDITIVE && d->gate == GDN_GATE_NONE && d->dtype == GDN_BF16 && d->dk == 128 &&
           (d->dv == 64 || d->dv == 128) && d->prologue == 0 && mode == 0;
}

int gdn_launch_chunk_la(const gdn::ChunkArgs &a, const gdn_desc_t *d, cudaStream_t stream) {
    using namespace gdn;
    LAParams prm;
    memset(&prm, 0, sizeof(prm));
    const uint64_t BH = (uint64_t)a.BH, T = (uint64_t)a.T;
    const bool ob = d->out_dtype == GDN_BF16;
    if (!make_map_3d(&prm.q_map, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 128, T, BH, 64, 64, 1, true) ||
        !make_map_3d(&prm.k_map, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 128, T, BH, 64, 64, 1, true) ||
        !make_map_3d(&prm.v_map, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.dv, T, BH, 64, 64, 1, true) ||
        !make_map_3d(&prm.o_map, a.o, ob ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, ob ? 2 : 4,
                     (uint64_t)a.dv, T, BH, ob ? 64 : 32, kLAC, 1, true))
        return (int)cudaErrorInvalidValue;
    prm.S0 = a.S0;
    prm.ST = a.ST;
    prm.status = a.status;
    prm.wait_ns = gdn_wait_limit_ns();
    prm.BH = a.BH;
    prm.T = a.T;
    prm.dv = a.dv;
    prm.nslices = a.dv / kDVS;
    const long grid = (long)a.BH * prm.nslices;
    if (grid == 0) return 0;
    if (prm.wait_ns) return ob ? launch_la<true, true>(prm, (int)grid, stream) : launch_la<false, true>(prm, (int)grid, stream);
    return ob ? launch_la<true, false>(prm, (int)grid, stream) : launch_la<false, false>(prm, (int)grid, stream);
}
