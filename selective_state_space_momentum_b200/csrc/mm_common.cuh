// mm_common.cuh -- small device helpers shared by the kernels of libmmscan.
// Internal to the library (not installed, not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace mmscan {

// log2(e): exp(z) is evaluated as 2^(z * log2 e) on the MUFU unit.
constexpr float kLog2e = 1.4426950408889634f;

using bf16 = __nv_bfloat16;

// ---------------------------------------------------------------- math ----
// MUFU base-2 exponential (flush-to-zero: results below 2^-126 become 0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// --------------------------------------------------------------- bf16 -----
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two fp32 values to a packed bf16x2 word (round to nearest even); `lo`
// lands in the low half, i.e. at the lower address.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ----------------------------------------------------------- cp.async -----
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte async copy global -> shared; bytes past `src_bytes` (0..16) are
// zero-filled and not read.  Both addresses must be 16-byte aligned.
__device__ __forceinline__ void cp_async_16(void* dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n"
                 :: "r"(smem_u32(dst)), "l"(src), "r"(src_bytes) : "memory");
}

// 4-byte async copy (src_bytes 0 or 4), both addresses 4-byte aligned.
__device__ __forceinline__ void cp_async_4(void* dst, const void* src, int src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n"
                 :: "r"(smem_u32(dst)), "l"(src), "r"(src_bytes) : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" :: "n"(N) : "memory");
}

// -------------------------------------------------------- streamed I/O ----
template <typename IO> struct IOTraits;
template <> struct IOTraits<float> { static constexpr int kBytes = 4; };
template <> struct IOTraits<bf16> { static constexpr int kBytes = 2; };

// Four consecutive elements from shared memory, widened to fp32.
__device__ __forceinline__ float4 load4(const float* p) {
    return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ float4 load4(const bf16* p) {
    const uint2 q = *reinterpret_cast<const uint2*>(p);
    return make_float4(bf16_lo(q.x), bf16_hi(q.x), bf16_lo(q.y), bf16_hi(q.y));
}

// Store four fp32 values to global memory as IO (vector store; address
// aligned to 4 elements).
__device__ __forceinline__ void store4(float* p, float4 v) {
    *reinterpret_cast<float4*>(p) = v;
}
__device__ __forceinline__ void store4(bf16* p, float4 v) {
    uint2 q;
    q.x = pack_bf16x2(v.x, v.y);
    q.y = pack_bf16x2(v.z, v.w);
    *reinterpret_cast<uint2*>(p) = q;
}

__device__ __forceinline__ void store1(float* p, float v) { *p = v; }
__device__ __forceinline__ void store1(bf16* p, float v) { *p = __float2bfloat16_rn(v); }

__device__ __forceinline__ float load1(const float* p) { return *p; }
__device__ __forceinline__ float load1(const bf16* p) { return __bfloat162float(*p); }

}  // namespace mmscan
