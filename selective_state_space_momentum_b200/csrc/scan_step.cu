// scan_step.cu -- sm_100a kernel for one decode step of the momentum scan.
//
// What it computes (the Mamba module's step() in "Momentum Mamba: Enhanced
// State Space Models with Momentum", section "Mamba Module"; the recurrence
// of "Momentum Mamba Recurrence" with the selective_scan_fn extras): per
// request b, channel d, state n, on the cached (h, v), updated in place:
//     delta' = softplus(delta + bias[d])           (each part optional)
//     v = beta v + alpha delta' B[n] x
//     h = exp(delta' A[d,n]) h + v
//     y = (sum_n C[n] h + D[d] x) * silu(z)        (each part optional)
// It is the one-step case of mm_scan_fwd_gated with (h, v) in and out.
//
// Design (B200-first): one step touches every cached state once, so the
// kernel is a stream over the states (4 D N fp32 bytes read and written per
// request): each lane owns four consecutive states of one channel and moves
// them with one 16-byte load and store each for h and v (streaming cache
// hints: the states are not reused within the step), the NP/4 lanes of a
// channel add their read-out partials by shuffles, and the first of them
// applies the skip and the gate and stores y.  The per-state operations are
// those of the scan kernel in the same order, so L steps leave the states
// bit-identical to one scan over the L steps.
#include <cuda.h>

#include "mm_common.cuh"
#include "mm_internal.h"

namespace mmscan {

template <typename IO, int NP, bool EXT>
__global__ void __launch_bounds__(256) scan_step_kernel(const ScanStepArgs p) {
    constexpr int G = NP / 4;                      // lanes per channel
    const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t ch = gt / G;                     // flat channel b * dim + d
    const int g = (int)(gt % G);
    const int N = p.dstate;
    const bool active = ch < p.batch * p.dim;
    const int64_t chs = active ? ch : 0;
    const int64_t b = chs / p.dim;
    const int64_t d = chs - b * p.dim;
    const int n0 = 4 * g;

    const IO* xs = static_cast<const IO*>(p.x);
    const IO* ds = static_cast<const IO*>(p.delta);
    const float x = load1(xs + chs);
    float dl = load1(ds + chs);
    if constexpr (EXT) {
        if (p.dbias) dl += p.dbias[d];
        if (p.softplus) dl = softplus_f32(dl);
    }
    const float u = dl * x;

    // this lane's four states (zeros past N)
    float A4[4], B4[4], C4[4], h4[4], v4[4];
    const int64_t srow = chs * N;
    const IO* Bs = static_cast<const IO*>(p.B) + b * N;
    const IO* Cs = static_cast<const IO*>(p.C) + b * N;
    if (p.vec && n0 + 4 <= N) {
        const float4 a = *reinterpret_cast<const float4*>(p.A + d * N + n0);
        const float4 bq = load4(Bs + n0);
        const float4 cq = load4(Cs + n0);
        const float4 hq = __ldcs(reinterpret_cast<const float4*>(p.h + srow + n0));
        const float4 vq = __ldcs(reinterpret_cast<const float4*>(p.v + srow + n0));
        A4[0] = a.x; A4[1] = a.y; A4[2] = a.z; A4[3] = a.w;
        B4[0] = bq.x; B4[1] = bq.y; B4[2] = bq.z; B4[3] = bq.w;
        C4[0] = cq.x; C4[1] = cq.y; C4[2] = cq.z; C4[3] = cq.w;
        h4[0] = hq.x; h4[1] = hq.y; h4[2] = hq.z; h4[3] = hq.w;
        v4[0] = vq.x; v4[1] = vq.y; v4[2] = vq.z; v4[3] = vq.w;
    } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool in = n0 + e < N;
            A4[e] = in ? p.A[d * N + n0 + e] : 0.0f;
            B4[e] = in ? load1(Bs + n0 + e) : 0.0f;
            C4[e] = in ? load1(Cs + n0 + e) : 0.0f;
            h4[e] = in ? p.h[srow + n0 + e] : 0.0f;
            v4[e] = in ? p.v[srow + n0 + e] : 0.0f;
        }
    }

    float yp = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float a = ex2_approx(dl * (A4[e] * kLog2e));
        const float w = u * (B4[e] * p.alpha);
        v4[e] = __fmaf_rn(p.beta, v4[e], w);
        h4[e] = __fmaf_rn(a, h4[e], v4[e]);
        yp = __fmaf_rn(C4[e], h4[e], yp);
    }

    if (active) {
        if (p.vec && n0 + 4 <= N) {
            __stcs(reinterpret_cast<float4*>(p.h + srow + n0), make_float4(h4[0], h4[1], h4[2], h4[3]));
            __stcs(reinterpret_cast<float4*>(p.v + srow + n0), make_float4(v4[0], v4[1], v4[2], v4[3]));
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (n0 + e < N) {
                    p.h[srow + n0 + e] = h4[e];
                    p.v[srow + n0 + e] = v4[e];
                }
            }
        }
    }
    // read-out over the G lanes of the channel (groups never straddle a warp)
#pragma unroll
    for (int m = G / 2; m >= 1; m >>= 1) yp += __shfl_xor_sync(0xffffffffu, yp, m);
    if (active && g == 0) {
        float out = yp;
        if constexpr (EXT) {
            if (p.Dskip) out += p.Dskip[d] * x;
            if (p.z) {
                const float z = load1(static_cast<const IO*>(p.z) + chs);
                out *= __fdividef(z, 1.0f + ex2_approx(-z * kLog2e));
            }
        }
        store1(static_cast<IO*>(p.y) + chs, out);
    }
}

namespace {

template <typename IO, int NP>
cudaError_t launch_step_np(const ScanStepArgs& a, cudaStream_t s) {
    constexpr int G = NP / 4;
    const int64_t threads = a.batch * a.dim * G;
    const int64_t blocks = (threads + 255) / 256;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (a.ext) scan_step_kernel<IO, NP, true><<<(unsigned)blocks, 256, 0, s>>>(a);
    else scan_step_kernel<IO, NP, false><<<(unsigned)blocks, 256, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename IO>
cudaError_t launch_step_io(const ScanStepArgs& a, cudaStream_t s) {
    if (a.dstate > 8) return launch_step_np<IO, 16>(a, s);
    if (a.dstate > 4) return launch_step_np<IO, 8>(a, s);
    return launch_step_np<IO, 4>(a, s);
}

}  // namespace

cudaError_t launch_scan_step(const ScanStepArgs& a, int io, cudaStream_t s) {
    if (io == 0) return launch_step_io<float>(a, s);
    return launch_step_io<bf16>(a, s);
}

}  // namespace mmscan
