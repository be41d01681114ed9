// Segmented prefill without a caller workspace.  The scratch of its passes
// (each segment's H and Lambda and its incoming state) lives in a fixed device
// array of this library: a __device__ variable exists once per device context
// that loads the library, and its address is looked up on the calling thread's
// current device at every call.  This file holds no kernel, so with lazy module
// loading (the CUDA default) the array is only mapped when this entry point is
// first used and other callers pay nothing for it.
// Calls that run at the same time on one device share the array: order them
// (one stream, or events), or use gdn_chunk_fwd_segmented with a workspace each.
#include <cuda_runtime.h>

#include "../../include/gdn.h"

__device__ __align__(256) unsigned char g_gdn_scratch[GDN_NOALLOC_SCRATCH_BYTES];

int gdn_segmented_request_check(const gdn_desc_t *d, int nseg);  // api.cu

extern "C" size_t gdn_noalloc_scratch_bytes(void) { return GDN_NOALLOC_SCRATCH_BYTES; }

extern "C" int gdn_chunk_fwd_segmented_noalloc(const gdn_desc_t *d, int nseg, const void *q, const void *k,
                                               const void *v, const float *g, const float *beta, const float *S0,
                                               void *o, float *S_T, void *stream) {
    // a malformed request gets the workspace variant's code, whatever its size
    const int rc = gdn_segmented_request_check(d, nseg);
    if (rc != GDN_OK) return rc;
    // one segment, or nothing to split: no scratch is touched
    if (nseg == 1 || (long)d->B * d->H == 0 || d->T == 0)
        return gdn_chunk_fwd_segmented(d, nseg, q, k, v, g, beta, S0, o, S_T, nullptr, 0, stream);
    if (gdn_segmented_workspace_bytes(d, nseg) > GDN_NOALLOC_SCRATCH_BYTES) return GDN_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if (cudaGetSymbolAddress(&scratch, g_gdn_scratch) != cudaSuccess) return GDN_ERR_CUDA;
    return gdn_chunk_fwd_segmented(d, nseg, q, k, v, g, beta, S0, o, S_T, scratch, GDN_NOALLOC_SCRATCH_BYTES,
                                   stream);
}
