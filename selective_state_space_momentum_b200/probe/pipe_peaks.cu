// pipe_peaks.cu -- throughput probes of the B200 execution pipes the scan
// kernels are bound by, built into libmmprobe.so (not part of libmmscan's
// C ABI).  The benchmark divides a kernel's work by these measured rates to
// report its fraction of the roofline.
//
// Each probe runs, per thread, K independent dependency chains of one
// instruction kind for `iters` rounds, so that the pipe, not the latency of
// one chain, bounds the rate.  The caller times the launch with CUDA events
// and converts the count (blocks * threads * iters * K operations) with the
// SM clock it sampled:
//   * ex2:   MUFU base-2 exponential, ex2.approx.ftz.f32 (x <- 2^-x stays in
//            [0.5, 1] for x in [0, 1]);
//   * ffma:  scalar fp32 fused multiply-add (x <- x * c + d);
//   * ffma2: packed f32x2 fused multiply-add (two lanes per instruction);
//   * ex2 at low occupancy (one-warp blocks, a few warps per SM), alone and
//     mixed with dependent packed FMAs, to see how many warps the MUFU pipe
//     needs.
// The chains' final values are summed into `out` (one float per thread) so
// that no work is removed by the compiler.
#include <cuda_runtime.h>
#include <cstdint>

namespace {

constexpr int K = 16;   // independent chains per thread

__device__ __forceinline__ float ex2f_approx(float x) {
    float y;
    asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__global__ void ex2_probe(float* out, int iters) {
    float a[K];
#pragma unroll
    for (int i = 0; i < K; ++i) a[i] = (float)((threadIdx.x * K + i) & 1023) * (1.0f / 1024.0f);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < K; ++i) a[i] = ex2f_approx(-a[i]);
    }
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < K; ++i) s += a[i];
    out[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
}

__global__ void ffma_probe(float* out, int iters, float c, float d) {
    float a[K];
#pragma unroll
    for (int i = 0; i < K; ++i) a[i] = (float)(threadIdx.x + i);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < K; ++i) a[i] = fmaf(a[i], c, d);
    }
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < K; ++i) s += a[i];
    out[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
}

__global__ void ffma2_probe(float* out, int iters, float c, float d) {
    float2 a[K / 2];
#pragma unroll
    for (int i = 0; i < K / 2; ++i) a[i] = make_float2((float)(threadIdx.x + i), (float)(threadIdx.x - i));
    const float2 c2 = make_float2(c, c), d2 = make_float2(d, d);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < K / 2; ++i) a[i] = __ffma2_rn(a[i], c2, d2);
    }
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < K / 2; ++i) s += a[i].x + a[i].y;
    out[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
}

// MUFU rate at low occupancy: 8 independent chains per thread, each ex2
// followed by F dependent packed FMAs (F = 0 or 3), in one-warp blocks.
template <int F>
__global__ void ex2_mix_probe(float* out, int iters) {
    constexpr int KC = 8;
    float a[KC];
    float2 f[KC];
#pragma unroll
    for (int i = 0; i < KC; ++i) {
        a[i] = (float)((threadIdx.x * KC + i) & 1023) * (1.0f / 1024.0f);
        f[i] = make_float2(a[i], -a[i]);
    }
    const float2 c2 = make_float2(0.999f, 0.999f), d2 = make_float2(1e-3f, 1e-3f);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < KC; ++i) {
            a[i] = ex2f_approx(-a[i]);
#pragma unroll
            for (int r = 0; r < F; ++r) f[i] = __ffma2_rn(f[i], c2, d2);
        }
    }
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < KC; ++i) s += a[i] + f[i].x + f[i].y;
    out[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
}

}  // namespace

extern "C" {

// Operations each probe performs per thread and round (fp32 lanes; an f32x2
// instruction counts two).
int mmprobe_ops_per_thread_round(void) { return K; }

// Launch one probe on `stream`: kind 0 = ex2, 1 = ffma, 2 = ffma2 (16 chains
// per thread); 3 = ex2 alone, 4 = ex2 each followed by 3 dependent packed
// FMAs (8 chains per thread, for one-warp blocks at low occupancy).  `out`
// holds blocks * threads floats.  Returns the cudaError_t of the launch.
int mmprobe_launch(int kind, float* out, int blocks, int threads, int iters, void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (kind) {
        case 0: ex2_probe<<<blocks, threads, 0, s>>>(out, iters); break;
        case 1: ffma_probe<<<blocks, threads, 0, s>>>(out, iters, 0.999f, 1e-3f); break;
        case 2: ffma2_probe<<<blocks, threads, 0, s>>>(out, iters, 0.999f, 1e-3f); break;
        case 3: ex2_mix_probe<0><<<blocks, threads, 0, s>>>(out, iters); break;
        case 4: ex2_mix_probe<3><<<blocks, threads, 0, s>>>(out, iters); break;
        default: return (int)cudaErrorInvalidValue;
    }
    return (int)cudaGetLastError();
}

}  // extern "C"
