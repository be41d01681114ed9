// Tensor-core (tcgen05) chunkwise prefill -- placeholder until the kernel lands.
#include "../../include/gdn.h"
#include "common.cuh"

int gdn_tc_supported(const gdn_desc_t *d) {
    (void)d;
    return 0;
}

int gdn_launch_chunk_tc(const gdn::ChunkArgs &a, const gdn_desc_t *d, cudaStream_t stream) {
    (void)a; (void)d; (void)stream;
    return (int)cudaErrorNotSupported;
}
