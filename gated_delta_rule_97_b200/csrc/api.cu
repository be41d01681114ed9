// C ABI of libgdn.so: argument validation and kernel dispatch (see gdn.h).
#include <stdint.h>
#include <string.h>

#include "../../include/gdn.h"
#include "common.cuh"

// The library's device status word (first error code any kernel recorded) and
// diagnostic word (where the first timeout happened).
__device__ int g_gdn_status = 0;
__device__ int g_gdn_diag = 0;

// tensor-core launcher (chunk_tc2.cu)
int gdn_tc_supported(const gdn_desc_t *d);
int gdn_launch_chunk_tc2(const gdn::ChunkArgs &a, const gdn_desc_t *d, cudaStream_t stream);
// linear-attention launcher (chunk_la.cu)
int gdn_la_supported(const gdn_desc_t *d, int mode);
int gdn_launch_chunk_la(const gdn::ChunkArgs &a, const gdn_desc_t *d, cudaStream_t stream);

namespace {

int *status_ptr() {
    // The address is per device; looked up on every call (cheap, no allocation).
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_gdn_status) != cudaSuccess) return nullptr;
    return static_cast<int *>(p);
}

int *diag_ptr() {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_gdn_diag) != cudaSuccess) return nullptr;
    return static_cast<int *>(p);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_size(int dtype) { return dtype == GDN_BF16 ? 2 : 4; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

int validate_common(const gdn_desc_t *d) {
    if (!d) return GDN_ERR_ARG;
    if (d->B < 0 || d->H < 0 || d->T < 0) return GDN_ERR_ARG;
    if ((d->dk != 64 && d->dk != 128) || (d->dv != 64 && d->dv != 128)) return GDN_ERR_ARG;
    if (d->update < GDN_ADDITIVE || d->update > GDN_DELTA) return GDN_ERR_ARG;
    if (d->gate < GDN_GATE_NONE || d->gate > GDN_GATE_CHANNEL) return GDN_ERR_ARG;
    if (d->update == GDN_ADDITIVE && d->gate != GDN_GATE_NONE) return GDN_ERR_ARG;
    if (d->update == GDN_DECAY && d->gate == GDN_GATE_NONE) return GDN_ERR_ARG;
    if ((d->dtype != GDN_F32 && d->dtype != GDN_BF16) || (d->out_dtype != GDN_F32 && d->out_dtype != GDN_BF16))
        return GDN_ERR_ARG;
    const long bh = (long)d->B * d->H;
    if (bh > (1L << 30)) return GDN_ERR_ARG;
    if (d->prologue & ~(GDN_PRO_QK_ELU1 | GDN_PRO_QK_L2 | GDN_PRO_BETA_SIGMOID | GDN_PRO_G_NEG_SOFTPLUS))
        return GDN_ERR_ARG;
    return GDN_OK;
}

int from_cuda(int e) { return e == 0 ? GDN_OK : GDN_ERR_CUDA; }

bool tc2_prologue_ok(const gdn_desc_t *d);

// Kernel choice of gdn_chunk_fwd (and of the passes of the segmented prefill):
// the requested kernel, or for AUTO the linear-attention kernel for a plain
// additive request it serves, else the pipelined tensor-core kernel when it
// serves the request and the SIMT kernel otherwise.  The latter two apply the
// input prologue.
int dispatch_chunk(const gdn_desc_t *d, gdn::ChunkArgs &a, cudaStream_t st) {
    if (d->algo == GDN_ALGO_AUTO && gdn_la_supported(d, a.mode)) return from_cuda(gdn_launch_chunk_la(a, d, st));
    const bool tc_ok = gdn_tc_supported(d) != 0 && tc2_prologue_ok(d);
    if (d->algo == GDN_ALGO_TC && !tc_ok) return GDN_ERR_UNSUPPORTED;
    if (d->algo == GDN_ALGO_TC || (d->algo == GDN_ALGO_AUTO && tc_ok)) return from_cuda(gdn_launch_chunk_tc2(a, d, st));
    return from_cuda(gdn_launch_chunk_simt(a, d->update, d->gate, d->dtype == GDN_BF16, d->out_dtype == GDN_BF16, st));
}

// The pipelined tensor-core kernel applies every input prologue map itself.
bool tc2_prologue_ok(const gdn_desc_t *) { return true; }

}  // namespace

// Bound of the kernels' hand-off waits in ns (0 = the default, 1 s); a test
// hook (gdn_set_wait_limit_ns), read by the launchers.
static unsigned long long g_wait_limit_ns = 0;
unsigned long long gdn_wait_limit_ns() { return g_wait_limit_ns; }

extern "C" int gdn_set_wait_limit_ns(unsigned long long ns) {
    g_wait_limit_ns = ns;
    return GDN_OK;
}

extern "C" int gdn_version(void) { return GDN_VERSION; }

extern "C" const char *gdn_strerror(int code) {
    switch (code) {
        case GDN_OK: return "ok";
        case GDN_ERR_ARG: return "invalid argument (null pointer, bad enum, size or overlap)";
        case GDN_ERR_ALIGN: return "pointer not 16-byte aligned";
        case GDN_ERR_UNSUPPORTED: return "request not supported by this build";
        case GDN_ERR_CUDA: return "CUDA runtime error";
        case GDN_ERR_TIMEOUT: return "a bounded wait inside a kernel timed out";
        case GDN_ERR_RANGE: return "an fp16 tensor-core operand overflowed";
        default: return "unknown error";
    }
}

extern "C" int gdn_device_status(int clear) {
    if (cudaDeviceSynchronize() != cudaSuccess) return GDN_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_gdn_status, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
    if (clear) {
        const int z = 0;
        if (cudaMemcpyToSymbol(g_gdn_status, &z, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
        if (cudaMemcpyToSymbol(g_gdn_diag, &z, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
    }
    return v;
}

extern "C" int gdn_device_diag(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return GDN_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_gdn_diag, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
    return v;
}


// Argument rules of gdn_chunk_fwd (sizes, pointers, alignment, overlaps).
// With need_o false (the segment maps) no output rows are read or checked.
static int chunk_fwd_check(const gdn_desc_t *d, const void *q, const void *k, const void *v, const float *g,
                           const float *beta, const float *S0, const void *o, const float *S_T,
                           bool need_o = true) {
    int rc = validate_common(d);
    if (rc != GDN_OK) return rc;
    if (d->chunk != 0 && d->chunk != gdn::kChunk) return GDN_ERR_UNSUPPORTED;
    if (d->algo < GDN_ALGO_AUTO || d->algo > GDN_ALGO_TC) return GDN_ERR_ARG;
    const long BH = (long)d->B * d->H;
    const size_t n_qk = (size_t)BH * d->T * d->dk, n_v = (size_t)BH * d->T * d->dv;
    const size_t n_S = (size_t)BH * d->dv * d->dk;
    const size_t n_g = d->gate == GDN_GATE_CHANNEL ? n_qk : (size_t)BH * d->T;
    const bool has_tokens = BH > 0 && d->T > 0;
    if (has_tokens) {
        if (!q || !k || !v || (need_o && !o)) return GDN_ERR_ARG;
        if (d->update == GDN_DELTA && !beta) return GDN_ERR_ARG;
    }
    if ((d->gate != GDN_GATE_NONE) != (g != nullptr) && has_tokens) return GDN_ERR_ARG;
    if (d->gate == GDN_GATE_NONE && g != nullptr) return GDN_ERR_ARG;
    const void *ptrs[] = {q, k, v, g, beta, S0, o, S_T};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGN;
    const size_t es = elem_size(d->dtype), eo = elem_size(d->out_dtype);
    const size_t no = n_v * eo;
    if (overlaps(o, no, q, n_qk * es) || overlaps(o, no, k, n_qk * es) || overlaps(o, no, v, n_v * es) ||
        overlaps(o, no, g, n_g * 4) || overlaps(o, no, beta, (size_t)BH * d->T * 4) ||
        overlaps(o, no, S0, n_S * 4) || overlaps(o, no, S_T, n_S * 4))
        return GDN_ERR_ARG;
    if (S_T && S0 && S_T != S0 && overlaps(S_T, n_S * 4, S0, n_S * 4)) return GDN_ERR_ARG;

    return GDN_OK;
}

extern "C" int gdn_chunk_fwd(const gdn_desc_t *d, const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *S0, void *o, float *S_T, void *stream) {
    const int rc = chunk_fwd_check(d, q, k, v, g, beta, S0, o, S_T);
    if (rc != GDN_OK) return rc;
    const long BH = (long)d->B * d->H;
    const size_t n_S = (size_t)BH * d->dv * d->dk;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (BH == 0) return GDN_OK;
    if (d->T == 0) return from_cuda(gdn_launch_copy_state(S0, S_T, (long)n_S, st));

    gdn::ChunkArgs a{};
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S0 = S0; a.o = o; a.ST = S_T;
    a.status = status_ptr();
    a.diag = diag_ptr();
    a.BH = (int)BH; a.T = d->T; a.dk = d->dk; a.dv = d->dv;
    a.nh = 1;
    a.pro = d->prologue;
    a.mode = 0;
    return dispatch_chunk(d, a, st);
}

// gdn_chunk_fwd, then the device status word: an fp16 operand overflow of the
// tensor-core kernel (GDN_ERR_RANGE) runs the request again on the fp32 SIMT
// kernel.  Synchronous.
extern "C" int gdn_chunk_fwd_checked(const gdn_desc_t *d, const void *q, const void *k, const void *v,
                                     const float *g, const float *beta, const float *S0, void *o, float *S_T,
                                     void *stream) {
    int rc = chunk_fwd_check(d, q, k, v, g, beta, S0, o, S_T);
    if (rc != GDN_OK) return rc;
    const size_t n_S = (size_t)d->B * d->H * d->dv * d->dk;
    if (overlaps(S0, n_S * 4, S_T, n_S * 4)) return GDN_ERR_ARG;  // the second run reads S0
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int status = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess ||
        cudaMemcpyFromSymbol(&status, g_gdn_status, sizeof(int)) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (status != 0) return status;  // an earlier error the caller has not cleared
    rc = gdn_chunk_fwd(d, q, k, v, g, beta, S0, o, S_T, stream);
    if (rc != GDN_OK) return rc;
    if (cudaStreamSynchronize(st) != cudaSuccess ||
        cudaMemcpyFromSymbol(&status, g_gdn_status, sizeof(int)) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (status == 0) return GDN_OK;
    if (status != GDN_ERR_RANGE) return status;
    const int z = 0;
    if (cudaMemcpyToSymbol(g_gdn_status, &z, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
    gdn_desc_t d2 = *d;
    d2.algo = GDN_ALGO_SIMT;
    rc = gdn_chunk_fwd(&d2, q, k, v, g, beta, S0, o, S_T, stream);
    if (rc != GDN_OK) return rc;
    if (cudaStreamSynchronize(st) != cudaSuccess ||
        cudaMemcpyFromSymbol(&status, g_gdn_status, sizeof(int)) != cudaSuccess)
        return GDN_ERR_CUDA;
    return status != 0 ? status : 1;
}

namespace {

// Byte layout of one slot of the host pipeline's device workspace: the inputs
// and outputs of ``hs`` heads, each tensor on a 256-byte boundary.
struct SlotLayout {
    size_t q, k, v, g, beta, S0, o, ST, bytes;
    size_t nq, nv, ng, nb, nS, no;  // per-head bytes of each tensor
};

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

SlotLayout slot_layout(const gdn_desc_t *d, long hs) {
    SlotLayout L;
    const size_t es = elem_size(d->dtype), T = (size_t)d->T;
    L.nq = T * d->dk * es;
    L.nv = T * d->dv * es;
    L.ng = d->gate == GDN_GATE_NONE ? 0 : (d->gate == GDN_GATE_CHANNEL ? T * d->dk * 4 : T * 4);
    L.nb = d->update == GDN_DELTA ? T * 4 : 0;
    L.nS = (size_t)d->dv * d->dk * 4;
    L.no = T * d->dv * elem_size(d->out_dtype);
    size_t off = 0;
    L.q = off; off += up256(hs * L.nq);
    L.k = off; off += up256(hs * L.nq);
    L.v = off; off += up256(hs * L.nv);
    L.g = off; off += up256(hs * L.ng);
    L.beta = off; off += up256(hs * L.nb);
    L.S0 = off; off += up256(hs * L.nS);
    L.o = off; off += up256(hs * L.no);
    L.ST = off; off += up256(hs * L.nS);
    L.bytes = off;
    return L;
}

long slice_heads(const gdn_desc_t *d, int n_slices) {
    const long BH = (long)d->B * d->H;
    const long n = n_slices < BH ? n_slices : BH;
    return n > 0 ? (BH + n - 1) / n : 0;
}

int h2d(void *dst, const void *src, size_t n, cudaStream_t s) {
    if (n == 0 || !src) return GDN_OK;
    return from_cuda(cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, s));
}

int d2h(void *dst, const void *src, size_t n, cudaStream_t s) {
    if (n == 0 || !dst) return GDN_OK;
    return from_cuda(cudaMemcpyAsync(dst, src, n, cudaMemcpyDeviceToHost, s));
}

}  // namespace

extern "C" size_t gdn_host_workspace_bytes(const gdn_desc_t *d, int n_slices) {
    if (!d || n_slices < 1 || validate_common(d) != GDN_OK) return 0;
    return 2 * slot_layout(d, slice_heads(d, n_slices)).bytes;
}

extern "C" int gdn_chunk_fwd_host(const gdn_desc_t *d, int n_slices, const void *q, const void *k, const void *v,
                                  const float *g, const float *beta, const float *S0, void *o, float *S_T,
                                  void *workspace, size_t workspace_bytes, void *stream) {
    int rc = chunk_fwd_check(d, q, k, v, g, beta, S0, o, S_T);
    if (rc != GDN_OK) return rc;
    if (n_slices < 1) return GDN_ERR_ARG;
    const long BH = (long)d->B * d->H;
    if (BH == 0) return GDN_OK;
    const long hs = slice_heads(d, n_slices);
    const SlotLayout L = slot_layout(d, hs);
    if (!workspace || workspace_bytes < 2 * L.bytes) return GDN_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_ALIGN;

    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev[7] = {};  // start, in[2], comp[2], out[2]
    rc = from_cuda(cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking));
    if (rc == GDN_OK) rc = from_cuda(cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking));
    for (int i = 0; i < 7 && rc == GDN_OK; ++i) rc = from_cuda(cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming));
    cudaEvent_t &start = ev[0], *in = ev + 1, *comp = ev + 3, *out = ev + 5;
    if (rc == GDN_OK) rc = from_cuda(cudaEventRecord(start, cs));
    if (rc == GDN_OK) rc = from_cuda(cudaStreamWaitEvent(s_in, start, 0));
    if (rc == GDN_OK) rc = from_cuda(cudaStreamWaitEvent(s_out, start, 0));

    const char *hq = static_cast<const char *>(q), *hk = static_cast<const char *>(k);
    const char *hv = static_cast<const char *>(v), *hg = reinterpret_cast<const char *>(g);
    const char *hb = reinterpret_cast<const char *>(beta), *hS0 = reinterpret_cast<const char *>(S0);
    char *ho = static_cast<char *>(o), *hST = reinterpret_cast<char *>(S_T);
    const long n = (BH + hs - 1) / hs;
    for (long i = 0; i < n && rc == GDN_OK; ++i) {
        const int slot = (int)(i & 1);
        const long h0 = i * hs, nh = (h0 + hs <= BH) ? hs : BH - h0;
        char *base = static_cast<char *>(workspace) + slot * L.bytes;
        // the slot is free once the copy-out of slice i - 2 (after its kernel) is done
        if (i >= 2) rc = from_cuda(cudaStreamWaitEvent(s_in, out[slot], 0));
        if (rc == GDN_OK) rc = h2d(base + L.q, hq + h0 * L.nq, nh * L.nq, s_in);
        if (rc == GDN_OK) rc = h2d(base + L.k, hk + h0 * L.nq, nh * L.nq, s_in);
        if (rc == GDN_OK) rc = h2d(base + L.v, hv + h0 * L.nv, nh * L.nv, s_in);
        if (rc == GDN_OK && hg) rc = h2d(base + L.g, hg + h0 * L.ng, nh * L.ng, s_in);
        if (rc == GDN_OK && hb) rc = h2d(base + L.beta, hb + h0 * L.nb, nh * L.nb, s_in);
        if (rc == GDN_OK && hS0) rc = h2d(base + L.S0, hS0 + h0 * L.nS, nh * L.nS, s_in);
        if (rc == GDN_OK) rc = from_cuda(cudaEventRecord(in[slot], s_in));
        if (rc == GDN_OK) rc = from_cuda(cudaStreamWaitEvent(cs, in[slot], 0));
        if (rc == GDN_OK) {
            gdn_desc_t sd = *d;
            sd.B = (int)nh;
            sd.H = 1;
            rc = gdn_chunk_fwd(&sd, base + L.q, base + L.k, base + L.v,
                               hg ? reinterpret_cast<const float *>(base + L.g) : nullptr,
                               hb ? reinterpret_cast<const float *>(base + L.beta) : nullptr,
                               hS0 ? reinterpret_cast<const float *>(base + L.S0) : nullptr, base + L.o,
                               hST ? reinterpret_cast<float *>(base + L.ST) : nullptr, cs);
        }
        if (rc == GDN_OK) rc = from_cuda(cudaEventRecord(comp[slot], cs));
        if (rc == GDN_OK) rc = from_cuda(cudaStreamWaitEvent(s_out, comp[slot], 0));
        if (rc == GDN_OK) rc = d2h(ho + h0 * L.no, base + L.o, nh * L.no, s_out);
        if (rc == GDN_OK && hST) rc = d2h(hST + h0 * L.nS, base + L.ST, nh * L.nS, s_out);
        if (rc == GDN_OK) rc = from_cuda(cudaEventRecord(out[slot], s_out));
    }
    // the caller's stream resumes after every copy-out
    for (int j = 0; j < 2 && rc == GDN_OK && j < n; ++j) rc = from_cuda(cudaStreamWaitEvent(cs, out[j], 0));
    // streams and events are released once their pending work completes
    for (int i = 0; i < 7; ++i)
        if (ev[i]) cudaEventDestroy(ev[i]);
    if (s_in) cudaStreamDestroy(s_in);
    if (s_out) cudaStreamDestroy(s_out);
    return rc;
}

extern "C" int gdn_product_fwd(const gdn_desc_t *d, int nh, const void *q, const void *k, const void *v,
                               const float *g, const float *beta, const float *S0, void *o, float *S_T,
                               void *stream) {
    int rc = validate_common(d);
    if (rc != GDN_OK) return rc;
    if (d->update != GDN_DELTA) return GDN_ERR_ARG;  // a product of delta-rule transitions
    if (nh < 1) return GDN_ERR_ARG;
    if (nh > GDN_PRODUCT_MAX_NH) return GDN_ERR_UNSUPPORTED;
    if (nh == 1) return gdn_chunk_fwd(d, q, k, v, g, beta, S0, o, S_T, stream);
    if (d->chunk != 0 && d->chunk != gdn::kChunk) return GDN_ERR_UNSUPPORTED;
    if (d->algo < GDN_ALGO_AUTO || d->algo > GDN_ALGO_TC) return GDN_ERR_ARG;
    // the pipelined tensor-core kernel takes 64 / nh whole tokens per chunk (the
    // remaining rows are identity steps)
    const bool tc_ok = gdn_tc_supported(d) != 0 && tc2_prologue_ok(d);
    if (d->algo == GDN_ALGO_TC && !tc_ok) return GDN_ERR_UNSUPPORTED;
    if ((long)d->T * nh > 0x7fffffffL) return GDN_ERR_UNSUPPORTED;
    const long BH = (long)d->B * d->H;
    const size_t Tr = (size_t)d->T, Tv = Tr * nh;
    const size_t n_q = (size_t)BH * Tr * d->dk, n_k = (size_t)BH * Tv * d->dk, n_v = (size_t)BH * Tv * d->dv;
    const size_t n_o = (size_t)BH * Tr * d->dv, n_S = (size_t)BH * d->dv * d->dk;
    const size_t n_g = d->gate == GDN_GATE_CHANNEL ? n_q : (size_t)BH * Tr;
    const bool has_tokens = BH > 0 && d->T > 0;
    if (has_tokens && (!q || !k || !v || !o || !beta)) return GDN_ERR_ARG;
    if ((d->gate != GDN_GATE_NONE) != (g != nullptr) && has_tokens) return GDN_ERR_ARG;
    if (d->gate == GDN_GATE_NONE && g != nullptr) return GDN_ERR_ARG;
    const void *ptrs[] = {q, k, v, g, beta, S0, o, S_T};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGN;
    const size_t es = elem_size(d->dtype), no = n_o * elem_size(d->out_dtype);
    if (overlaps(o, no, q, n_q * es) || overlaps(o, no, k, n_k * es) || overlaps(o, no, v, n_v * es) ||
        overlaps(o, no, g, n_g * 4) || overlaps(o, no, beta, (size_t)BH * Tv * 4) ||
        overlaps(o, no, S0, n_S * 4) || overlaps(o, no, S_T, n_S * 4))
        return GDN_ERR_ARG;
    if (S_T && S0 && S_T != S0 && overlaps(S_T, n_S * 4, S0, n_S * 4)) return GDN_ERR_ARG;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (BH == 0) return GDN_OK;
    if (d->T == 0) return from_cuda(gdn_launch_copy_state(S0, S_T, (long)n_S, st));
    gdn::ChunkArgs a{};
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S0 = S0; a.o = o; a.ST = S_T;
    a.status = status_ptr();
    a.diag = diag_ptr();
    a.BH = (int)BH; a.T = (int)Tv; a.dk = d->dk; a.dv = d->dv;
    a.nh = nh;
    a.pro = d->prologue;
    a.mode = 0;
    if (d->algo == GDN_ALGO_TC || (d->algo == GDN_ALGO_AUTO && tc_ok)) return from_cuda(gdn_launch_chunk_tc2(a, d, st));
    return from_cuda(gdn_launch_chunk_simt(a, d->update, d->gate, d->dtype == GDN_BF16, d->out_dtype == GDN_BF16, st));
}

extern "C" size_t gdn_segmented_workspace_bytes(const gdn_desc_t *d, int nseg) {
    if (!d || nseg < 1 || d->B < 0 || d->H < 0 || d->dk < 0 || d->dv < 0) return 0;
    // at most 2^30 segment-heads (larger requests are rejected), so the product
    // below cannot wrap
    const long bh = (long)d->B * d->H;
    if (bh > (1L << 30) || bh * nseg > (1L << 30) || d->dk > 128 || d->dv > 128) return 0;
    const size_t segs = (size_t)bh * nseg;
    return segs * ((size_t)2 * d->dv * d->dk + (size_t)d->dk * d->dk) * sizeof(float);
}

// The request rules of the segmented prefill that do not involve pointers (the
// descriptor, the segment count and the total number of segment-heads), shared
// with gdn_chunk_fwd_segmented_noalloc so that both reject a bad request with
// the same code before looking at any scratch size.
int gdn_segmented_request_check(const gdn_desc_t *d, int nseg) {
    int rc = validate_common(d);
    if (rc != GDN_OK) return rc;
    if (nseg < 1) return GDN_ERR_ARG;
    if (nseg == 1) return GDN_OK;
    if (d->T % nseg != 0) return GDN_ERR_ARG;
    if (d->chunk != 0 && d->chunk != gdn::kChunk) return GDN_ERR_UNSUPPORTED;
    if (d->algo < GDN_ALGO_AUTO || d->algo > GDN_ALGO_TC) return GDN_ERR_ARG;
    if ((long)d->B * d->H * nseg > (1L << 30)) return GDN_ERR_ARG;
    return GDN_OK;
}

extern "C" int gdn_chunk_fwd_segmented(const gdn_desc_t *d, int nseg, const void *q, const void *k, const void *v,
                                       const float *g, const float *beta, const float *S0, void *o, float *S_T,
                                       void *workspace, size_t workspace_bytes, void *stream) {
    int rc = gdn_segmented_request_check(d, nseg);
    if (rc != GDN_OK) return rc;
    if (nseg == 1) return gdn_chunk_fwd(d, q, k, v, g, beta, S0, o, S_T, stream);
    const long BH = (long)d->B * d->H;
    const size_t need = gdn_segmented_workspace_bytes(d, nseg);
    if (BH > 0 && d->T > 0) {
        if (!workspace || workspace_bytes < need) return GDN_ERR_ARG;
        if (!aligned16(workspace)) return GDN_ERR_ALIGN;
    }
    // the same argument rules as gdn_chunk_fwd, checked on the whole request
    rc = chunk_fwd_check(d, q, k, v, g, beta, S0, o, S_T);
    if (rc != GDN_OK) return rc;
    // pass 1 writes the workspace and later passes re-read every input, so the
    // workspace may overlap no input and no output
    const size_t es = elem_size(d->dtype), n_tok = (size_t)BH * d->T;
    const size_t n_o = n_tok * d->dv * elem_size(d->out_dtype), n_S = (size_t)BH * d->dv * d->dk * 4;
    const size_t n_g = d->gate == GDN_GATE_CHANNEL ? n_tok * d->dk * 4 : n_tok * 4;
    if (overlaps(workspace, need, o, n_o) || overlaps(workspace, need, S_T, n_S) ||
        overlaps(workspace, need, S0, n_S) || overlaps(workspace, need, q, n_tok * d->dk * es) ||
        overlaps(workspace, need, k, n_tok * d->dk * es) || overlaps(workspace, need, v, n_tok * d->dv * es) ||
        overlaps(workspace, need, g, n_g) || overlaps(workspace, need, beta, n_tok * 4))
        return GDN_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (BH == 0) return GDN_OK;
    if (d->T == 0) return from_cuda(gdn_launch_copy_state(S0, S_T, (long)BH * d->dv * d->dk, st));

    // segments of one sequence are consecutive runs of T / nseg tokens, so the
    // [B,H,T,d] tensors are [B*H*nseg, T/nseg, d] tensors of shorter "heads"
    const int segs = (int)(BH * nseg);
    float *H = static_cast<float *>(workspace);
    float *Sstart = H + (size_t)segs * d->dv * d->dk;
    float *Lam = Sstart + (size_t)segs * d->dv * d->dk;
    gdn_desc_t sd = *d;
    sd.B = (int)BH;
    sd.H = nseg;
    sd.T = d->T / nseg;
    gdn::ChunkArgs a{};
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.o = o;
    a.status = status_ptr();
    a.diag = diag_ptr();
    a.BH = segs; a.T = sd.T; a.dk = d->dk; a.dv = d->dv;
    a.nh = 1;
    a.pro = d->prologue;
    // 1. every segment from a zero state: H_i (no outputs)
    a.S0 = nullptr; a.ST = H; a.mode = gdn::kModeNoOut;
    if ((rc = dispatch_chunk(&sd, a, st)) != GDN_OK) return rc;
    // 2. every segment's transition Lambda_i: zero values from the identity state
    //    (with the additive write and no gate the transition is the identity)
    const bool identity = d->update == GDN_ADDITIVE;
    if (!identity) {
        gdn_desc_t ld = sd;
        ld.dv = d->dk;
        gdn::ChunkArgs b = a;
        b.v = nullptr; b.o = nullptr; b.S0 = nullptr; b.ST = Lam; b.dv = d->dk;
        b.mode = gdn::kModeZeroV | gdn::kModeNoOut | gdn::kModeS0Eye;
        if ((rc = dispatch_chunk(&ld, b, st)) != GDN_OK) return rc;
    }
    // 3. the state entering each segment, and the final state
    if ((rc = from_cuda(gdn_launch_compose(S0, H, identity ? nullptr : Lam, Sstart, S_T, (int)BH, nseg, d->dk,
                                           d->dv, false, st))) != GDN_OK)
        return rc;
    // 4. every segment from its true incoming state: the outputs
    a.S0 = Sstart; a.ST = nullptr; a.mode = 0;
    return dispatch_chunk(&sd, a, st);
}

extern "C" int gdn_segment_maps(const gdn_desc_t *d, const void *q, const void *k, const void *v, const float *g,
                                const float *beta, float *H, float *Lam, void *stream) {
    int rc = chunk_fwd_check(d, q, k, v, g, beta, nullptr, nullptr, nullptr, false);
    if (rc != GDN_OK) return rc;
    const long BH = (long)d->B * d->H;
    const size_t n_S = (size_t)BH * d->dv * d->dk * 4, n_L = (size_t)BH * d->dk * d->dk * 4;
    if (BH > 0 && (!H || !Lam)) return GDN_ERR_ARG;
    if ((H && !aligned16(H)) || (Lam && !aligned16(Lam))) return GDN_ERR_ALIGN;
    const size_t es = elem_size(d->dtype);
    const size_t n_qk = (size_t)BH * d->T * d->dk * es, n_v = (size_t)BH * d->T * d->dv * es;
    const size_t n_g = (d->gate == GDN_GATE_CHANNEL ? (size_t)BH * d->T * d->dk : (size_t)BH * d->T) * 4;
    const size_t n_b = (size_t)BH * d->T * 4;
    if (overlaps(H, n_S, Lam, n_L)) return GDN_ERR_ARG;
    const void *outs[] = {H, Lam};
    const size_t nouts[] = {n_S, n_L};
    for (int i = 0; i < 2; ++i)
        if (overlaps(outs[i], nouts[i], q, n_qk) || overlaps(outs[i], nouts[i], k, n_qk) ||
            overlaps(outs[i], nouts[i], v, n_v) || overlaps(outs[i], nouts[i], g, n_g) ||
            overlaps(outs[i], nouts[i], beta, n_b))
            return GDN_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (BH == 0) return GDN_OK;
    // the additive write without a gate leaves the transition at the identity
    const bool identity = d->update == GDN_ADDITIVE || d->T == 0;
    if (d->T == 0) {
        if ((rc = from_cuda(gdn_launch_copy_state(nullptr, H, (long)BH * d->dv * d->dk, st))) != GDN_OK) return rc;
    } else {
        gdn::ChunkArgs a{};
        a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.o = nullptr;
        a.status = status_ptr();
        a.diag = diag_ptr();
        a.BH = (int)BH; a.T = d->T; a.dk = d->dk; a.dv = d->dv;
        a.nh = 1;
        a.pro = d->prologue;
        a.S0 = nullptr; a.ST = H; a.mode = gdn::kModeNoOut;
        if ((rc = dispatch_chunk(d, a, st)) != GDN_OK) return rc;
        if (!identity) {
            gdn_desc_t ld = *d;
            ld.dv = d->dk;
            gdn::ChunkArgs b = a;
            b.v = nullptr; b.ST = Lam; b.dv = d->dk;
            b.mode = gdn::kModeZeroV | gdn::kModeNoOut | gdn::kModeS0Eye;
            return dispatch_chunk(&ld, b, st);
        }
    }
    return from_cuda(gdn_launch_eye(Lam, BH, d->dk, st));
}

extern "C" int gdn_compose_segments(int BH, int nseg, int dk, int dv, const float *S0, const float *H,
                                    const float *Lam, float *S_in, float *S_T, void *stream) {
    if (BH < 0 || nseg < 1 || BH > (1 << 30) || (long)BH * nseg > (1L << 30)) return GDN_ERR_ARG;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return GDN_ERR_ARG;
    if (BH == 0) return GDN_OK;
    if (!H) return GDN_ERR_ARG;
    const void *ptrs[] = {S0, H, Lam, S_in, S_T};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGN;
    const size_t n_S = (size_t)BH * dv * dk * 4, n_H = n_S * nseg, n_L = (size_t)BH * nseg * dk * dk * 4;
    // outputs overlap no input (S_T may be S0 itself: each row is read before it is written)
    if (overlaps(S_in, n_H, S0, n_S) || overlaps(S_in, n_H, H, n_H) || overlaps(S_in, n_H, Lam, n_L) ||
        overlaps(S_in, n_H, S_T, n_S) || overlaps(S_T, n_S, H, n_H) || overlaps(S_T, n_S, Lam, n_L) ||
        (S_T != S0 && overlaps(S_T, n_S, S0, n_S)))
        return GDN_ERR_ARG;
    return from_cuda(gdn_launch_compose(S0, H, Lam, S_in, S_T, BH, nseg, dk, dv, true,
                                        static_cast<cudaStream_t>(stream)));
}

extern "C" int gdn_decode_step(const gdn_desc_t *d, const void *q, const void *k, const void *v, const float *g,
                               const float *beta, float *S, void *o, void *stream) {
    int rc = validate_common(d);
    if (rc != GDN_OK) return rc;
    if (d->T < 0) return GDN_ERR_ARG;
    if (d->T > GDN_DECODE_MAX_T) return GDN_ERR_UNSUPPORTED;
    const long BH = (long)d->B * d->H;
    if (BH == 0 || d->T == 0) return GDN_OK;
    if (!q || !k || !v || !S || !o) return GDN_ERR_ARG;
    if (d->update == GDN_DELTA && !beta) return GDN_ERR_ARG;
    if ((d->gate != GDN_GATE_NONE) != (g != nullptr)) return GDN_ERR_ARG;
    const void *ptrs[] = {q, k, v, g, beta, S, o};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGN;
    const size_t n_S = (size_t)BH * d->dv * d->dk;
    const size_t BT = (size_t)BH * d->T;
    const size_t no = BT * d->dv * elem_size(d->out_dtype);
    const size_t es = elem_size(d->dtype);
    if (overlaps(o, no, S, n_S * 4) || overlaps(o, no, q, BT * d->dk * es) || overlaps(o, no, k, BT * d->dk * es) ||
        overlaps(o, no, v, BT * d->dv * es))
        return GDN_ERR_ARG;
    gdn::DecodeArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S = S; a.o = o;
    a.BH = (int)BH; a.T = d->T; a.dk = d->dk; a.dv = d->dv;
    a.pro = d->prologue;
    a.status = status_ptr();
    a.wait_ns = g_wait_limit_ns;
    return from_cuda(gdn_launch_decode(a, d->update, d->gate, d->dtype == GDN_BF16, d->out_dtype == GDN_BF16,
                                       static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------------------
// Backward (backward.cu)
int gdn_launch_bwd(const void *q, const void *k, const void *v, const float *g, const float *beta, const float *S0,
                   const float *dO, const float *dST, float *dq, float *dk, float *dv, float *dg, float *dbeta,
                   float *dS0, float *ws, int BH, int T, int dk_, int dv_, int update, int gate, int in_bf16,
                   int skip_fwd, cudaStream_t st);
// input prologue of the backward (prologue_bwd.cu)
int gdn_launch_prologue_map(const void *q, const void *k, const void *v, const float *g, const float *beta, float *qm,
                            float *km, float *vf, float *gm, float *bm, long rows, int dk, int dv, int gate,
                            int in_bf16, int pro, cudaStream_t st);
int gdn_launch_prologue_grad(const void *q, const void *k, const float *g, const float *beta, float *dq, float *dk,
                             float *dg, float *dbeta, long rows, int dk_, int gate, int in_bf16, int pro,
                             cudaStream_t st);

size_t gdn_bwd_tc_layout(long BH, int nch, int dk, int dv, int delta, size_t *off);  // backward_tc.cu
int gdn_launch_bwd_tc(const void *q, const void *k, const void *v, const float *g, const float *beta,
                      const float *states, const float *dO, const float *dST, float *dq, float *dk, float *dv,
                      float *dg, float *dbeta, float *dS0, void *ws, int BH, int T, int dv_, int update, int gate,
                      int in_bf16, cudaStream_t st);

// The per-chunk kernels put the heads on the grid's y dimension (at most 65535).
static bool bwd_tc_supported(const gdn_desc_t *d) {
    return d->prologue == 0 && d->gate != GDN_GATE_CHANNEL && d->dk == 128 && (d->dv == 64 || d->dv == 128) &&
           (d->chunk == 0 || d->chunk == gdn::kChunk) && (long)d->B * d->H <= 65535;
}

// Workspace of gdn_chunk_bwd: the chunk-entry states, then (with an input
// prologue) the mapped inputs in fp32: q, k, v, beta, g, each on a 256-byte
// boundary.  With GDN_ALGO_TC: the states, then the tensor-core backward's
// workspace.
struct BwdLayout {
    size_t states, qm, km, vf, bm, gm, bytes;
};

static size_t round256(size_t n) { return (n + 255) & ~size_t(255); }

static BwdLayout bwd_layout(const gdn_desc_t *d) {
    BwdLayout L{};
    const size_t BH = (size_t)d->B * d->H, ntok = BH * d->T;
    const size_t nch = ((size_t)d->T + gdn::kChunk - 1) / gdn::kChunk;
    L.states = 0;
    size_t off = BH * nch * d->dv * d->dk * sizeof(float);
    if (d->prologue != 0) {
        off = round256(off);
        L.qm = off; off = round256(off + ntok * d->dk * 4);
        L.km = off; off = round256(off + ntok * d->dk * 4);
        L.vf = off; off = round256(off + ntok * d->dv * 4);
        L.bm = off; off = round256(off + (d->update == GDN_DELTA ? ntok * 4 : 0));
        L.gm = off; off += d->gate == GDN_GATE_NONE ? 0 : ntok * (d->gate == GDN_GATE_CHANNEL ? d->dk : 1) * 4;
    }
    L.bytes = off;
    return L;
}

// gdn_chunk_bwd on the tensor-core path: the tensor-core forward writes the
// chunk states (bf16 inputs, dk = 128), then the chunkwise backward.
static bool bwd_algo_tc(const gdn_desc_t *d) { return d->algo == GDN_ALGO_TC; }
static bool bwd_algo_tc_served(const gdn_desc_t *d) { return bwd_tc_supported(d) && gdn_tc_supported(d); }

static size_t bwd_states_bytes(const gdn_desc_t *d) {
    const size_t nch = ((size_t)d->T + gdn::kChunk - 1) / gdn::kChunk;
    return (size_t)d->B * d->H * nch * d->dv * d->dk * sizeof(float);
}

extern "C" size_t gdn_bwd_workspace_bytes(const gdn_desc_t *d) {
    if (!d || validate_common(d) != GDN_OK) return 0;
    if (bwd_algo_tc(d)) {
        if (!bwd_algo_tc_served(d)) return 0;
        const int nch = (d->T + gdn::kChunk - 1) / gdn::kChunk;
        return round256(bwd_states_bytes(d)) +
               gdn_bwd_tc_layout((long)d->B * d->H, nch, d->dk, d->dv, d->update == GDN_DELTA, nullptr);
    }
    return bwd_layout(d).bytes;
}

namespace {

// Argument rules shared by the backward entry points: pointers, alignment, the
// workspace (`need` bytes, required unless `ws_optional`) and overlaps of every
// output (and the workspace) with every input and with each other.
int bwd_check(const gdn_desc_t *d, const void *q, const void *k, const void *v, const float *g, const float *beta,
              const float *S0, const float *saved, size_t saved_bytes, const float *dO, const float *dS_T,
              float *dq, float *dk, float *dv, float *dg, float *dbeta, float *dS0, void *workspace,
              size_t workspace_bytes, size_t need) {
    const long BH = (long)d->B * d->H;
    const size_t ntok = (size_t)BH * d->T;
    const size_t es = elem_size(d->dtype);
    const size_t n_qk = ntok * d->dk, n_v = ntok * d->dv, n_S = (size_t)BH * d->dv * d->dk;
    const size_t n_g = d->gate == GDN_GATE_CHANNEL ? n_qk : ntok;
    const bool has_tokens = ntok > 0;
    if (has_tokens) {
        if (!q || !k || !v || !dq || !dk || !dv) return GDN_ERR_ARG;
        if ((d->update == GDN_DELTA) != (beta != nullptr) || (d->update == GDN_DELTA) != (dbeta != nullptr))
            return GDN_ERR_ARG;
        if ((d->gate != GDN_GATE_NONE) != (g != nullptr) || (d->gate != GDN_GATE_NONE) != (dg != nullptr))
            return GDN_ERR_ARG;
    }
    const void *ptrs[] = {q, k, v, g, beta, S0, saved, dO, dS_T, dq, dk, dv, dg, dbeta, dS0, workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGN;
    if (has_tokens && need && (!workspace || workspace_bytes < need)) return GDN_ERR_ARG;
    if (has_tokens && !need && workspace) return GDN_ERR_ARG;
    struct Span { const void *p; size_t n; };
    const Span ins[] = {{q, n_qk * es}, {k, n_qk * es}, {v, n_v * es}, {g, n_g * 4}, {beta, ntok * 4},
                        {S0, n_S * 4}, {saved, has_tokens ? saved_bytes : 0}, {dO, n_v * 4}, {dS_T, n_S * 4}};
    const Span outs[] = {{dq, n_qk * 4}, {dk, n_qk * 4}, {dv, n_v * 4}, {dg, n_g * 4}, {dbeta, ntok * 4},
                         {dS0, n_S * 4}, {workspace, has_tokens ? need : 0}};
    for (const Span &o : outs) {
        for (const Span &i : ins)
            if (overlaps(o.p, o.n, i.p, i.n)) return GDN_ERR_ARG;
        for (const Span &o2 : outs)
            if (&o2 != &o && overlaps(o.p, o.n, o2.p, o2.n)) return GDN_ERR_ARG;
    }
    return GDN_OK;
}

// gdn_chunk_bwd and gdn_chunk_bwd_states: `saved` holds the chunk-entry states
// written by gdn_chunk_fwd_states (read only, the forward pass is skipped), or
// is null and `workspace` receives them from the backward's own forward pass.
int chunk_bwd_impl(const gdn_desc_t *d, const void *q, const void *k, const void *v, const float *g,
                   const float *beta, const float *S0, const float *saved, const float *dO, const float *dS_T,
                   float *dq, float *dk, float *dv, float *dg, float *dbeta, float *dS0, void *workspace,
                   size_t workspace_bytes, void *stream) {
    int rc = validate_common(d);
    if (rc != GDN_OK) return rc;
    if (d->chunk != 0 && d->chunk != gdn::kChunk) return GDN_ERR_UNSUPPORTED;
    if (d->prologue != 0 && saved) return GDN_ERR_UNSUPPORTED;  // the saved states carry no maps
    const bool tc = !saved && bwd_algo_tc(d);
    if (tc && !bwd_algo_tc_served(d)) return GDN_ERR_UNSUPPORTED;
    const long BH = (long)d->B * d->H;
    const size_t ntok = (size_t)BH * d->T;
    const size_t n_S = (size_t)BH * d->dv * d->dk;
    const size_t need = saved ? 0 : gdn_bwd_workspace_bytes(d);
    rc = bwd_check(d, q, k, v, g, beta, S0, saved, bwd_states_bytes(d), dO, dS_T, dq, dk, dv, dg, dbeta, dS0,
                   workspace, workspace_bytes, need);
    if (rc != GDN_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (BH == 0) return GDN_OK;
    if (d->T == 0) return dS0 ? from_cuda(gdn_launch_copy_state(dS_T, dS0, (long)n_S, st)) : GDN_OK;
    float *ws = saved ? const_cast<float *>(saved) : static_cast<float *>(workspace);
    const int in_bf16 = d->dtype == GDN_BF16;
    if (tc) {
        // the tensor-core forward writes the chunk-entry states (no o, no S_T), then
        // the chunkwise backward runs from them
        gdn::ChunkArgs a{};
        a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S0 = S0; a.o = nullptr; a.ST = nullptr;
        a.status = status_ptr();
        a.diag = diag_ptr();
        a.BH = (int)BH; a.T = d->T; a.dk = d->dk; a.dv = d->dv;
        a.nh = 1;
        a.mode = gdn::kModeSaveStates | gdn::kModeNoOut;
        a.states = ws;
        const int e = gdn_launch_chunk_tc2(a, d, st);
        if (e != 0) return from_cuda(e);
        return from_cuda(gdn_launch_bwd_tc(q, k, v, g, beta, ws, dO, dS_T, dq, dk, dv, dg, dbeta, dS0,
                                           static_cast<char *>(workspace) + round256(bwd_states_bytes(d)), (int)BH,
                                           d->T, d->dv, d->update, d->gate, in_bf16, st));
    }
    if (d->prologue == 0)
        return from_cuda(gdn_launch_bwd(q, k, v, g, beta, S0, dO, dS_T, dq, dk, dv, dg, dbeta, dS0, ws, (int)BH,
                                        d->T, d->dk, d->dv, d->update, d->gate, in_bf16, saved != nullptr, st));
    // input prologue: map the inputs (fp32, into the workspace), run the
    // recurrence's backward on them, then take dq, dk, dbeta, dg back through the maps
    const BwdLayout L = bwd_layout(d);
    char *w = static_cast<char *>(workspace);
    float *qm = reinterpret_cast<float *>(w + L.qm), *km = reinterpret_cast<float *>(w + L.km);
    float *vf = reinterpret_cast<float *>(w + L.vf);
    float *bm = d->update == GDN_DELTA ? reinterpret_cast<float *>(w + L.bm) : nullptr;
    float *gm = d->gate != GDN_GATE_NONE ? reinterpret_cast<float *>(w + L.gm) : nullptr;
    int e = gdn_launch_prologue_map(q, k, v, g, beta, qm, km, vf, gm, bm, (long)ntok, d->dk, d->dv, d->gate, in_bf16,
                                    d->prologue, st);
    if (e == 0)
        e = gdn_launch_bwd(qm, km, vf, gm, bm, S0, dO, dS_T, dq, dk, dv, dg, dbeta, dS0, ws, (int)BH, d->T, d->dk,
                           d->dv, d->update, d->gate, 0, 0, st);
    if (e == 0)
        e = gdn_launch_prologue_grad(q, k, g, beta, dq, dk, dg, dbeta, (long)ntok, d->dk, d->gate, in_bf16,
                                     d->prologue, st);
    return from_cuda(e);
}

}  // namespace

extern "C" int gdn_chunk_bwd(const gdn_desc_t *d, const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *S0, const float *dO, const float *dS_T, float *dq,
                             float *dk, float *dv, float *dg, float *dbeta, float *dS0, void *workspace,
                             size_t workspace_bytes, void *stream) {
    return chunk_bwd_impl(d, q, k, v, g, beta, S0, nullptr, dO, dS_T, dq, dk, dv, dg, dbeta, dS0, workspace,
                          workspace_bytes, stream);
}

extern "C" int gdn_chunk_bwd_states(const gdn_desc_t *d, const void *q, const void *k, const void *v,
                                    const float *g, const float *beta, const float *states, const float *dO,
                                    const float *dS_T, float *dq, float *dk, float *dv, float *dg, float *dbeta,
                                    float *dS0, void *stream) {
    if (d && (long)d->B * d->H * d->T > 0 && !states) return GDN_ERR_ARG;
    return chunk_bwd_impl(d, q, k, v, g, beta, nullptr, states, dO, dS_T, dq, dk, dv, dg, dbeta, dS0, nullptr, 0,
                          stream);
}

extern "C" size_t gdn_bwd_tc_workspace_bytes(const gdn_desc_t *d) {
    if (!d || validate_common(d) != GDN_OK || !bwd_tc_supported(d)) return 0;
    const long BH = (long)d->B * d->H;
    const int nch = (d->T + gdn::kChunk - 1) / gdn::kChunk;
    return gdn_bwd_tc_layout(BH, nch, d->dk, d->dv, d->update == GDN_DELTA, nullptr);
}

extern "C" int gdn_chunk_bwd_tc(const gdn_desc_t *d, const void *q, const void *k, const void *v, const float *g,
                                const float *beta, const float *states, const float *dO, const float *dS_T,
                                float *dq, float *dk, float *dv, float *dg, float *dbeta, float *dS0, void *workspace,
                                size_t workspace_bytes, void *stream) {
    int rc = validate_common(d);
    if (rc != GDN_OK) return rc;
    if (!bwd_tc_supported(d)) return GDN_ERR_UNSUPPORTED;
    const long BH = (long)d->B * d->H;
    const size_t ntok = (size_t)BH * d->T, n_S = (size_t)BH * d->dv * d->dk;
    const int nch = (d->T + gdn::kChunk - 1) / gdn::kChunk;
    if (ntok > 0 && !states) return GDN_ERR_ARG;
    const size_t need = gdn_bwd_tc_workspace_bytes(d);
    rc = bwd_check(d, q, k, v, g, beta, nullptr, states, (size_t)BH * nch * d->dv * d->dk * 4, dO, dS_T, dq, dk,
                   dv, dg, dbeta, dS0, workspace, workspace_bytes, need);
    if (rc != GDN_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (BH == 0) return GDN_OK;
    if (d->T == 0) return dS0 ? from_cuda(gdn_launch_copy_state(dS_T, dS0, (long)n_S, st)) : GDN_OK;
    return from_cuda(gdn_launch_bwd_tc(q, k, v, g, beta, states, dO, dS_T, dq, dk, dv, dg, dbeta, dS0, workspace,
                                       (int)BH, d->T, d->dv, d->update, d->gate, d->dtype == GDN_BF16, st));
}

extern "C" int gdn_chunk_fwd_states(const gdn_desc_t *d, const void *q, const void *k, const void *v,
                                    const float *g, const float *beta, const float *S0, void *o, float *S_T,
                                    float *states, void *stream) {
    const int rc = chunk_fwd_check(d, q, k, v, g, beta, S0, o, S_T);
    if (rc != GDN_OK) return rc;
    if (d->prologue != 0 || d->algo == GDN_ALGO_SIMT || !gdn_tc_supported(d)) return GDN_ERR_UNSUPPORTED;
    const long BH = (long)d->B * d->H;
    const size_t n_S = (size_t)BH * d->dv * d->dk;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (BH == 0) return GDN_OK;
    if (d->T == 0) return from_cuda(gdn_launch_copy_state(S0, S_T, (long)n_S, st));
    if (!states) return GDN_ERR_ARG;
    if (!aligned16(states)) return GDN_ERR_ALIGN;
    const size_t ns = bwd_states_bytes(d);
    const size_t es = elem_size(d->dtype), eo = elem_size(d->out_dtype);
    const size_t ntok = (size_t)BH * d->T;
    const size_t n_qk = ntok * d->dk, n_v = ntok * d->dv;
    const size_t n_g = d->gate == GDN_GATE_CHANNEL ? n_qk : ntok;
    if (overlaps(states, ns, q, n_qk * es) || overlaps(states, ns, k, n_qk * es) || overlaps(states, ns, v, n_v * es) ||
        overlaps(states, ns, g, n_g * 4) || overlaps(states, ns, beta, ntok * 4) || overlaps(states, ns, S0, n_S * 4) ||
        overlaps(states, ns, o, n_v * eo) || overlaps(states, ns, S_T, n_S * 4))
        return GDN_ERR_ARG;
    gdn::ChunkArgs a{};
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S0 = S0; a.o = o; a.ST = S_T;
    a.status = status_ptr();
    a.diag = diag_ptr();
    a.BH = (int)BH; a.T = d->T; a.dk = d->dk; a.dv = d->dv;
    a.nh = 1;
    a.mode = gdn::kModeSaveStates;
    a.states = states;
    return from_cuda(gdn_launch_chunk_tc2(a, d, st));
}
