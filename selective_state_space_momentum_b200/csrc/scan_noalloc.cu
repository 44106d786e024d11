// scan_noalloc.cu -- mm_scan_fwd_noalloc: the forward scan for callers that
// cannot allocate device memory.
//
// The two-launch form of the sequence-split scan (mm_scan_fwd_split_maps,
// then mm_scan_fwd_split_correct on one device) needs a buffer for the
// segment records that pass between its launches.  Some callers cannot get
// that buffer: code running inside a host framework that owns every device
// allocation (a plugin, an inference server's custom-op slot), a process
// whose device memory was sized and reserved once at start-up, or a path
// that must not take cudaMalloc's device-wide synchronisation.  For them the
// records live in one fixed array in the library's own device memory,
// reserved on every GPU that loads the library until the process exits.
//
// The array's host-side name is not a device address; the address each
// device sees comes from cudaGetSymbolAddress, taken once per device (with
// that device current) on the first call there.
#include <cuda_runtime.h>

#include <mutex>

#include "mm_internal.h"
#include "mm_scan.h"

namespace {

// Largest record set one call may use: 8 MiB per GPU.  The long streaming
// workload (batch 1, L 131072, D 2048: eight 16384-step segments of 128
// channel tiles) needs 4.2 MB.
constexpr size_t kScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// The scratch array's device address on the current device (set up on the
// first call there).
cudaError_t scratch_on_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" mm_status mm_scan_fwd_noalloc(const void* x, const void* delta, const float* A, const void* B,
                                         const void* C, const float* h0, const float* v0, float beta,
                                         float alpha, void* y, float* hT, float* vT, const mm_scan_dims* dims,
                                         void* stream) {
    if (!dims) return mmscan::report(MM_ERR_NULL, "dims is NULL");
    int64_t unused = 0;
    if (mm_status st = mm_scan_segment_len(dims, &unused)) return st;     // the size checks
    // segment length: the sequence-split path's own, at least one staged chunk
    const int64_t chunk = mmscan::scan_seg_chunk_steps(dims->io == MM_F32 ? 0 : 1);
    int64_t S = mmscan::scan_seg_default_len(dims->batch, dims->dim);
    if (S < chunk) S = chunk;
    const int64_t nseg = dims->seqlen / S + (dims->seqlen % S != 0);
    size_t bytes = 0;
    if (mm_status st = mm_scan_split_maps_size(dims, nseg, &bytes)) return st;
    if (bytes > kScratchBytes)
        return mmscan::report(MM_ERR_UNSUPPORTED,
                              "mm_scan_fwd_noalloc: these sizes need %zu bytes of segment records "
                              "(%lld segments of %lld steps); the library's fixed scratch holds %zu",
                              bytes, (long long)nseg, (long long)S, kScratchBytes);
    void* scratch = nullptr;
    const cudaError_t e = scratch_on_current_device(&scratch);
    if (e != cudaSuccess)
        return mmscan::report(MM_ERR_CUDA, "mm_scan_fwd_noalloc: scratch address: %s (%s)", cudaGetErrorString(e),
                              cudaGetErrorName(e));
    if (mm_status st = mm_scan_fwd_split_maps(x, delta, A, B, C, beta, alpha, y, scratch, S, dims, stream))
        return st;
    return mm_scan_fwd_split_correct(delta, A, C, h0, v0, beta, alpha, y, hT, vT, scratch, S, 0, dims->seqlen,
                                     dims, stream);
}
