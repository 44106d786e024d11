// ssd_fwd.cu -- Mamba-2 scalar-A chunked (SSD) forward on sm_100a.
#include "mm_common.cuh"
#include "mm_internal.h"

namespace mmscan {

bool ssd_shape_supported(int64_t headdim, int64_t dstate, int64_t chunk) {
    return headdim == 64 && dstate == 128 && chunk == 256;
}

size_t ssd_workspace_bytes(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                           int64_t dstate, int64_t chunk) {
    (void)batch; (void)seqlen; (void)nheads; (void)headdim; (void)dstate; (void)chunk;
    return 256;
}

cudaError_t launch_ssd_fwd(const SSDArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace mmscan
