/* cuda_runtime.h stand-in for compiling the library's host-side code on a
 * machine without CUDA: the harness that includes it defines every function
 * declared here (queues of deferred operations, checked copies, or no-ops). */
#pragma once
#include <cstddef>

typedef int cudaError_t;
typedef struct stub_stream* cudaStream_t;
typedef struct stub_event* cudaEvent_t;
enum { cudaSuccess = 0, cudaErrorInvalidValue = 1 };
enum cudaMemcpyKind { cudaMemcpyHostToDevice = 1, cudaMemcpyDeviceToHost = 2 };
enum { cudaStreamNonBlocking = 1, cudaEventDisableTiming = 2 };

cudaError_t cudaStreamCreateWithFlags(cudaStream_t* s, unsigned flags);
cudaError_t cudaStreamDestroy(cudaStream_t s);
cudaError_t cudaStreamSynchronize(cudaStream_t s);
cudaError_t cudaEventCreateWithFlags(cudaEvent_t* e, unsigned flags);
cudaError_t cudaEventDestroy(cudaEvent_t e);
cudaError_t cudaEventRecord(cudaEvent_t e, cudaStream_t s);
cudaError_t cudaStreamWaitEvent(cudaStream_t s, cudaEvent_t e, unsigned flags);
cudaError_t cudaMemcpyAsync(void* dst, const void* src, size_t n, cudaMemcpyKind k, cudaStream_t s);
cudaError_t cudaMemcpy2DAsync(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width,
                              size_t height, cudaMemcpyKind k, cudaStream_t s);
enum cudaMemoryType { cudaMemoryTypeUnregistered = 0, cudaMemoryTypeHost = 1, cudaMemoryTypeDevice = 2,
                      cudaMemoryTypeManaged = 3 };
struct cudaPointerAttributes {
    enum cudaMemoryType type;
    int device;
    void* devicePointer;
    void* hostPointer;
};
cudaError_t cudaPointerGetAttributes(cudaPointerAttributes* attr, const void* ptr);
cudaError_t cudaGetDevice(int* device);
cudaError_t cudaDeviceSynchronize(void);
const char* cudaGetErrorString(cudaError_t e);
const char* cudaGetErrorName(cudaError_t e);
