// mm_ipc.cpp -- sharing a device buffer with the other processes of a job.
//
// The scan split across ranks can hand its segment records straight to the
// other ranks' buffers (mm_scan_fwd_split_maps_peers).  Each rank exports
// its buffer of the whole sequence's records as a CUDA IPC handle, the ranks
// exchange the 64-byte handles over their process group, and each opens the
// others' handles into device pointers it can store to (over NVLink between
// GPUs, or within one GPU between processes).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "mm_internal.h"
#include "mm_scan.h"

static_assert(sizeof(cudaIpcMemHandle_t) == MM_IPC_HANDLE_BYTES, "IPC handle size");

namespace {

// The driver's cuMemGetAddressRange, reached through the runtime (the library
// links no driver library).
using AddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

AddressRangeFn address_range_fn() {
    static AddressRangeFn fn = [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            (void)cudaGetLastError();
            return static_cast<AddressRangeFn>(nullptr);
        }
        return reinterpret_cast<AddressRangeFn>(ptr);
    }();
    return fn;
}

}  // namespace

extern "C" mm_status mm_ipc_get_handle(const void* dev_ptr, void* handle, int64_t* offset) {
    if (!dev_ptr || !handle || !offset) return mmscan::report(MM_ERR_NULL, "dev_ptr, handle and offset are required");
    // A handle names the whole allocation that holds dev_ptr (an allocator may
    // hand out pieces of a larger one): the offset of dev_ptr in it goes along.
    AddressRangeFn range = address_range_fn();
    if (!range) return mmscan::report(MM_ERR_CUDA, "mm_ipc_get_handle: cuMemGetAddressRange is not available");
    CUdeviceptr base = 0;
    size_t size = 0;
    if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
        return mmscan::report(MM_ERR_CUDA, "mm_ipc_get_handle: %p is not device memory of this process", dev_ptr);
    cudaIpcMemHandle_t h;
    const cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return mmscan::report(MM_ERR_CUDA, "mm_ipc_get_handle: %s (%s)", cudaGetErrorString(e), cudaGetErrorName(e));
    }
    std::memcpy(handle, &h, sizeof(h));
    *offset = static_cast<int64_t>(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
    return mmscan::report_ok();
}

extern "C" mm_status mm_ipc_open_handle(const void* handle, int64_t offset, void** dev_ptr) {
    if (!handle || !dev_ptr) return mmscan::report(MM_ERR_NULL, "handle and dev_ptr are required");
    if (offset < 0) return mmscan::report(MM_ERR_DIMS, "offset %lld < 0", (long long)offset);
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof(h));
    void* p = nullptr;
    const cudaError_t e = cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return mmscan::report(MM_ERR_CUDA, "mm_ipc_open_handle: %s (%s)", cudaGetErrorString(e), cudaGetErrorName(e));
    }
    *dev_ptr = static_cast<unsigned char*>(p) + offset;
    return mmscan::report_ok();
}

extern "C" mm_status mm_ipc_close_handle(void* dev_ptr, int64_t offset) {
    if (!dev_ptr) return mmscan::report(MM_ERR_NULL, "dev_ptr is required");
    const cudaError_t e = cudaIpcCloseMemHandle(static_cast<unsigned char*>(dev_ptr) - offset);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return mmscan::report(MM_ERR_CUDA, "mm_ipc_close_handle: %s (%s)", cudaGetErrorString(e), cudaGetErrorName(e));
    }
    return mmscan::report_ok();
}
