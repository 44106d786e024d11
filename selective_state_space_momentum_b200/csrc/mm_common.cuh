// mm_common.cuh -- small device helpers shared by the kernels of libmmscan.
// Internal to the library (not installed, not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace mmscan {

// log2(e): exp(z) is evaluated as 2^(z * log2 e) on the MUFU unit.
constexpr float kLog2e = 1.4426950408889634f;
// Steps between two checkpoints of the scan state (forward writes, backward reads).
constexpr int kCkptSteps = 16;

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

// ----------------------------------------------------- sm_100 async --------
namespace mmscan {

// Upper bound of any device-side wait in this library.  A wait that runs
// past it sets kDevErrTimeout in the calling kernel file's device error
// word and the kernel returns early (the host reads the word in
// mm_device_status()).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s
constexpr unsigned int kDevErrTimeout = 1u;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}

// Arrive on `bar` once every cp.async this thread issued so far has landed.
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" :: "r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}

// Wait for the phase with `parity` to complete, giving up after
// kWaitLimitNs; on give-up `*err` gets kDevErrTimeout and false is returned.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned int* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(err, kDevErrTimeout);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// TMA tile load (no multicast) of a 3-D box into shared memory; completion
// is signalled on `bar` through its transaction count.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* map, uint32_t bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];"
        :: "r"(dst), "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(bar) : "memory");
}

// Byte offset of (row, byte-in-row) inside a tile of 128-byte rows written
// with the 128-byte swizzle (16-byte chunk index XOR row mod 8); the tile
// base must be 1024-byte aligned.
__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t byte_in_row) {
    return row * 128u + ((((byte_in_row >> 4) ^ (row & 7u)) << 4) | (byte_in_row & 15u));
}

}  // namespace mmscan

// ------------------------------------------------------- tcgen05 (UMMA) ----
namespace mmscan {

// Shared-memory matrix descriptor for tcgen05.mma, 128-byte swizzle.
// K-major tiles: rows of 128 bytes (64 bf16 along K), 8-row groups 1024 B
// apart (SBO); LBO unused.  MN-major tiles: rows of 128 bytes hold 64
// consecutive M (or N) elements for one K index; 8-row K groups at SBO and
// 64-element M (or N) groups at LBO.  Tiles are 1024-byte aligned.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;   // descriptor version of sm_100
    d |= 2ull << 61;   // 128-byte swizzle
    return d;
}

// Instruction descriptor, kind::f16 with bf16 operands and fp32 accumulate.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) |
           ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem desc] . B[smem desc]
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
                 :: "r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}

// D[tmem] (+)= A[tmem, K-major, bf16 pairs per column] . B[smem desc]
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n"
                 :: "r"(d_tmem), "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc) : "memory");
}

// Arrive once on `bar` when every tcgen05 operation issued so far by this thread completes.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Whole warp: allocate `ncols` TMEM columns; the base address is written to smem.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" :: "r"(dst_smem), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}

// Whole warp: 32 consecutive 32-bit columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
           "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]) : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// TMA tile load (no multicast) of a 4-D box.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];"
        :: "r"(dst), "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar) : "memory");
}

// TMA tile store (no multicast) of a 4-D box from shared memory, tracked by
// the issuing thread's bulk async-group.
__device__ __forceinline__ void tma_store_4d(const void* map, uint32_t src, int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3, %4}], [%5];"
        :: "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(src) : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk store of this thread has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until every committed bulk store of this thread is complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Named barrier that also returns the AND of `pred` over the participating
// threads, so that a group leaves a loop together when any of them must.
__device__ __forceinline__ bool named_bar_and(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r) : "r"((uint32_t)pred), "r"(id), "r"(nthreads) : "memory");
    return r != 0;
}

// Named barrier for a subset of warps (id 1..15).
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(nthreads) : "memory");
}

}  // namespace mmscan

namespace mmscan {

// ------------------------------------------------- scan helpers -----
// Store `cnt` consecutive steps of one output row.
template <typename IO>
__device__ __forceinline__ void store_steps(IO* dst, const float* v, int cnt, bool vec) {
    if constexpr (sizeof(IO) == 4) {
        if (vec && cnt == 2) {
            *reinterpret_cast<float2*>(dst) = make_float2(v[0], v[1]);
            return;
        }
        if (vec && cnt == 4) {
            *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
            return;
        }
    } else {
        if (vec && cnt == 2) {
            *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(v[0], v[1]);
            return;
        }
        if (vec && cnt == 4) {
            *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
            return;
        }
    }
}

template <typename IO, int PER>
__device__ __forceinline__ void store_steps_n(IO* dst, const float (&v)[PER], int cnt, bool vec) {
    if (vec && cnt == PER && (PER == 2 || PER == 4)) {
        store_steps<IO>(dst, v, PER, true);
        return;
    }
#pragma unroll
    for (int i = 0; i < PER; ++i)
        if (i < cnt) store1(dst + i, v[i]);
}

// Sum, over the G consecutive lanes of a group, of K per-lane partials: a
// butterfly that halves the values each lane carries at every stage (the lane
// whose bit m is set keeps the upper half), so that group lane g ends with
// the sums of entries [g K/G, (g+1) K/G) after log2 G exchanges of K/2, K/4,
// ... values.  The exchanges stay in registers: no shared-memory traffic.
template <int G, int K>
__device__ __forceinline__ void butterfly_sum(const float (&v)[K], float (&out)[K / G], int g) {
    static_assert((G & (G - 1)) == 0 && K % G == 0, "power-of-two group dividing K");
    float cur[K];
#pragma unroll
    for (int i = 0; i < K; ++i) cur[i] = v[i];
#pragma unroll
    for (int m = G / 2, n = K; m >= 1; m >>= 1, n >>= 1) {
        const bool upper = (g & m) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float keep = upper ? cur[n / 2 + i] : cur[i];
            const float send = upper ? cur[i] : cur[n / 2 + i];
            cur[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
#pragma unroll
    for (int e = 0; e < K / G; ++e) out[e] = cur[e];
}

__device__ __forceinline__ float2 shfl_up_f2(float2 v, int delta) {
    return f2(__shfl_up_sync(0xffffffffu, v.x, delta), __shfl_up_sync(0xffffffffu, v.y, delta));
}
__device__ __forceinline__ float2 shfl_down_f2(float2 v, int delta) {
    return f2(__shfl_down_sync(0xffffffffu, v.x, delta), __shfl_down_sync(0xffffffffu, v.y, delta));
}

// softplus(v) = ln(1 + e^v) = max(v, 0) + ln(1 + u) with u = e^-|v| in (0, 1].
// ln(1 + u) = 2 atanh(s) for s = u / (2 + u) in (0, 1/3], summed as the odd
// series s (1 + s^2/3 + s^4/5 + ... + s^14/15): every term is positive (no
// cancellation) and the first one left out is below 2e-9 of the sum, so the
// error is that of fp32 rounding and of the two MUFU operations.
__device__ __forceinline__ float softplus_f32(float v) {
    const float u = ex2_approx(-fabsf(v) * kLog2e);
    const float s = __fdividef(u, 2.0f + u);
    const float q = s * s;
    float p = 1.0f / 15.0f;
    p = fmaf(p, q, 1.0f / 13.0f);
    p = fmaf(p, q, 1.0f / 11.0f);
    p = fmaf(p, q, 1.0f / 9.0f);
    p = fmaf(p, q, 1.0f / 7.0f);
    p = fmaf(p, q, 1.0f / 5.0f);
    p = fmaf(p, q, 1.0f / 3.0f);
    p = fmaf(p, q, 1.0f);
    return fmaxf(v, 0.0f) + 2.0f * s * p;
}

}  // namespace mmscan
