// scan_fwd.cu -- sm_100a kernel for the Momentum Mamba forward selective scan.
//
// What it computes ("Momentum Mamba: Enhanced State Space Models with
// Momentum", "Momentum Mamba Recurrence" and "Discretization Note"), per
// batch row b, channel d, state n:
//     v_t = beta v_{t-1} + alpha delta_t B_t[n] x_t
//     h_t = exp(delta_t A[d,n]) h_{t-1} + v_t
//     y_t = sum_n C_t[n] h_t[n]
//
// Design (B200-first; the page's CUB two-stage block scan is prior art only):
//  * Work split.  A CTA owns CH channels of one batch row (B_t and C_t are
//    shared by all channels of a row) and walks the whole sequence.  Inside
//    it, G = NP / SPT consecutive lanes share a channel; each lane keeps SPT
//    consecutive states (v, h) in fp32 registers for the whole call, so the
//    recurrence runs exactly in time order with no carry recombination.
//  * Staging.  The sequence is cut into chunks of T steps.  For each chunk
//    the CTA copies its x and delta rows and the B/C rows of its batch row
//    into shared memory with cp.async (16-byte, zero-filled past L), three
//    chunks in flight.  B and C are then transposed to [t][n] in fp32 with
//    alpha folded into B, so a lane reads its SPT states of one step in one
//    vector load.
//  * Arithmetic.  Per step and state: one MUFU ex2 for exp(delta A) (A is
//    pre-scaled by log2 e), and packed f32x2 multiply / FMA for the write,
//    the velocity, the hidden state and the read-out, two states per
//    instruction.  exp of a step is never stored; no (L, D, N) tensor exists.
//  * Read-out.  Each lane forms its partial C_t . h_t over its SPT states;
//    the G partials of a channel meet in shared memory and one pass sums
//    them and writes y with coalesced 16-byte (fp32) or 8-byte (bf16) stores,
//    rounding to nearest-even for bf16.
//  * Final state.  (h, v) after the last step are written to hT, vT.  The
//    per-state operation sequence does not depend on how the sequence is
//    cut into calls, so split calls reproduce hT, vT bit for bit.
#include <atomic>

#include "mm_common.cuh"
#include "mm_internal.h"

namespace mmscan {

template <typename IO, int NP, int SPT, int WARPS>
struct ScanTile {
    static constexpr int G = NP / SPT;          // lanes per channel
    static constexpr int CPW = 32 / G;          // channels per warp
    static constexpr int CH = WARPS * CPW;      // channels per CTA
    static constexpr int NT = WARPS * 32;       // threads per CTA
    static constexpr int T = 32;                // steps per chunk
    static constexpr int STAGES = 3;            // chunks in flight
    static constexpr int EB = IOTraits<IO>::kBytes;
    static constexpr int XP = T + 16 / EB;      // row pitch (elements) of staged rows
    static constexpr int BP = NP + 4;           // row pitch (floats) of transposed B/C
    static constexpr int YP = T + 4;            // row pitch (floats) of read-out partials
    static constexpr int ROWS = 2 * CH + 2 * NP;
    static constexpr int STAGE_ELEMS = ROWS * XP;
    static constexpr int STAGE_BYTES = STAGE_ELEMS * EB;
    static constexpr int BT_FLOATS = T * BP;
    static constexpr int YPART_FLOATS = CH * G * YP;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + (2 * BT_FLOATS + YPART_FLOATS) * 4;
    static constexpr int PPR = T * EB / 16;     // 16-byte pieces per staged row

    static_assert(G >= 1 && (G & (G - 1)) == 0 && 32 % G == 0, "lanes per channel");
    static_assert(SPT % 2 == 0 && SPT <= 8, "states per lane are processed in pairs");
    static_assert(T % 4 == 0 && (T * EB) % 16 == 0, "chunk length");
    static_assert((XP * EB) % 16 == 0 && (STAGE_BYTES % 16) == 0, "16-byte rows");
};

// Copy chunk `k` (steps t0 .. t0+T-1) of the CTA's rows into stage buffer `sbuf`.
template <typename IO, int NP, int SPT, int WARPS>
__device__ __forceinline__ void stage_chunk(const ScanArgs& p, IO* sbuf, int64_t b, int64_t d0,
                                            int64_t t0, int tid) {
    using TL = ScanTile<IO, NP, SPT, WARPS>;
    const int64_t L = p.seqlen;
    const int nval = (int)((L - t0) < TL::T ? (L - t0) : TL::T);
    const IO* xg = static_cast<const IO*>(p.x);
    const IO* dg = static_cast<const IO*>(p.delta);
    const IO* Bg = static_cast<const IO*>(p.B);
    const IO* Cg = static_cast<const IO*>(p.C);

    // row r -> (global row start, number of valid elements)
    auto row_src = [&](int r, int& valid) -> const IO* {
        if (r < 2 * TL::CH) {
            const int c = r < TL::CH ? r : r - TL::CH;
            const int64_t d = d0 + c;
            valid = d < p.dim ? nval : 0;
            const IO* base = r < TL::CH ? xg : dg;
            return valid ? base + ((b * p.dim + d) * L + t0) : base;
        }
        const int rr = r - 2 * TL::CH;
        const int n = rr < NP ? rr : rr - NP;
        valid = n < p.dstate ? nval : 0;
        const IO* base = rr < NP ? Bg : Cg;
        return valid ? base + ((b * p.dstate + n) * L + t0) : base;
    };

    if (p.vec_ok) {
        constexpr int EPP = 16 / TL::EB;  // elements per 16-byte piece
        for (int i = tid; i < TL::ROWS * TL::PPR; i += TL::NT) {
            const int r = i / TL::PPR;
            const int j = i - r * TL::PPR;
            int valid;
            const IO* src = row_src(r, valid);
            int bytes = (valid - j * EPP) * TL::EB;
            bytes = bytes < 0 ? 0 : (bytes > 16 ? 16 : bytes);
            cp_async_16(sbuf + r * TL::XP + j * EPP, bytes ? src + j * EPP : src, bytes);
        }
    } else if constexpr (TL::EB == 4) {
        for (int i = tid; i < TL::ROWS * TL::T; i += TL::NT) {
            const int r = i / TL::T;
            const int e = i - r * TL::T;
            int valid;
            const IO* src = row_src(r, valid);
            const bool ok = e < valid;
            cp_async_4(sbuf + r * TL::XP + e, ok ? src + e : src, ok ? 4 : 0);
        }
    } else {
        // 2-byte elements on rows that are not 4-byte aligned: plain loads.
        for (int i = tid; i < TL::ROWS * TL::T; i += TL::NT) {
            const int r = i / TL::T;
            const int e = i - r * TL::T;
            int valid;
            const IO* src = row_src(r, valid);
            sbuf[r * TL::XP + e] = e < valid ? src[e] : IO(0.0f);
        }
    }
}

template <typename IO, int NP, int SPT, int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
scan_fwd_kernel(const ScanArgs p) {
    using TL = ScanTile<IO, NP, SPT, WARPS>;
    constexpr int G = TL::G, CPW = TL::CPW, CH = TL::CH, NT = TL::NT, T = TL::T;
    constexpr int ST = TL::STAGES, NPAIR = SPT / 2;

    extern __shared__ __align__(128) unsigned char smem_raw[];
    IO* stages = reinterpret_cast<IO*>(smem_raw);
    float* Bt = reinterpret_cast<float*>(smem_raw + ST * TL::STAGE_BYTES);
    float* Ct = Bt + TL::BT_FLOATS;
    float* ypart = Ct + TL::BT_FLOATS;

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int g = lane % G;
    const int c = (tid >> 5) * CPW + lane / G;      // channel within the CTA
    const int64_t b = blockIdx.x / p.tiles_per_batch;
    const int64_t d0 = (int64_t)(blockIdx.x % p.tiles_per_batch) * CH;
    const int64_t d = d0 + c;
    const bool active = d < p.dim;
    const int64_t L = p.seqlen;
    const int N = p.dstate;
    const int64_t nchunks = (L + T - 1) / T;

    // ---- per-lane constants and state ------------------------------------
    float A2[SPT];          // A[d, n] * log2 e
    float2 vv[NPAIR], hh[NPAIR];
#pragma unroll
    for (int s = 0; s < SPT; ++s) {
        const int n = g * SPT + s;
        A2[s] = (active && n < N) ? p.A[d * N + n] * kLog2e : 0.0f;
    }
#pragma unroll
    for (int q = 0; q < NPAIR; ++q) {
        float hv[2] = {0.0f, 0.0f}, vvv[2] = {0.0f, 0.0f};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int n = g * SPT + 2 * q + e;
            if (active && n < N) {
                const int64_t si = ((b * p.dim + d) * N + n);
                if (p.h0) hv[e] = p.h0[si];
                if (p.v0) vvv[e] = p.v0[si];
            }
        }
        hh[q] = f2(hv[0], hv[1]);
        vv[q] = f2(vvv[0], vvv[1]);
    }
    const float2 beta2 = f2(p.beta, p.beta);
    const float alpha = p.alpha;
    float2 A2p[SPT];        // (A2[s], A2[s]) for two steps at once
#pragma unroll
    for (int s = 0; s < SPT; ++s) A2p[s] = f2(A2[s], A2[s]);

    // ---- pipeline prologue -----------------------------------------------
#pragma unroll
    for (int s = 0; s < ST - 1; ++s) {
        if (s < nchunks)
            stage_chunk<IO, NP, SPT, WARPS>(p, stages + s * TL::STAGE_ELEMS, b, d0, (int64_t)s * T, tid);
        cp_async_commit();
    }

    for (int64_t k = 0; k < nchunks; ++k) {
        const int buf = (int)(k % ST);
        const int64_t t0 = k * T;
        const int nval = (int)((L - t0) < T ? (L - t0) : T);
        cp_async_wait<ST - 2>();
        __syncthreads();
        {
            const int64_t kn = k + ST - 1;
            if (kn < nchunks)
                stage_chunk<IO, NP, SPT, WARPS>(p, stages + (int)(kn % ST) * TL::STAGE_ELEMS, b, d0,
                                                kn * T, tid);
            cp_async_commit();
        }
        const IO* sb = stages + buf * TL::STAGE_ELEMS;

        // ---- transpose B, C to [t][n] fp32 (alpha folded into B) ---------
        {
            const IO* Braw = sb + 2 * CH * TL::XP;
            const IO* Craw = Braw + NP * TL::XP;
            constexpr int PER = NP * (T / 4);
            for (int i = tid; i < 2 * PER; i += NT) {
                const int which = i / PER;
                const int rem = i - which * PER;
                const int n = rem % NP;
                const int t4 = (rem / NP) * 4;
                const IO* src = (which ? Craw : Braw) + n * TL::XP + t4;
                float4 v4 = load4(src);
                if (!which) {
                    v4.x *= alpha; v4.y *= alpha; v4.z *= alpha; v4.w *= alpha;
                }
                float* dst = (which ? Ct : Bt) + t4 * TL::BP + n;
                dst[0] = v4.x;
                dst[TL::BP] = v4.y;
                dst[2 * TL::BP] = v4.z;
                dst[3 * TL::BP] = v4.w;
            }
        }
        __syncthreads();

        // ---- the recurrence over this chunk -------------------------------
        {
            const IO* xrow = sb + c * TL::XP;
            const IO* drow = sb + (CH + c) * TL::XP;
            float* yrow = ypart + (c * G + g) * TL::YP;
            const float* Bg = Bt + g * SPT;
            const float* Cg = Ct + g * SPT;

            auto step = [&](int t, float u, const float* a) -> float {
                const float2 uu = f2(u, u);
                float2 yy = f2(0.0f, 0.0f);
#pragma unroll
                for (int q = 0; q < NPAIR; ++q) {
                    const float2 bq = *reinterpret_cast<const float2*>(Bg + t * TL::BP + 2 * q);
                    const float2 cq = *reinterpret_cast<const float2*>(Cg + t * TL::BP + 2 * q);
                    const float2 w = __fmul2_rn(uu, bq);
                    vv[q] = __ffma2_rn(beta2, vv[q], w);
                    hh[q] = __ffma2_rn(f2(a[2 * q], a[2 * q + 1]), hh[q], vv[q]);
                    yy = __ffma2_rn(cq, hh[q], yy);
                }
                return yy.x + yy.y;
            };

            const int nfull = nval & ~3;
#pragma unroll 2
            for (int tau = 0; tau < nfull; tau += 4) {
                const float4 dq = load4(drow + tau);
                const float4 xq = load4(xrow + tau);
                const float2 u01 = __fmul2_rn(f2(dq.x, dq.y), f2(xq.x, xq.y));
                const float2 u23 = __fmul2_rn(f2(dq.z, dq.w), f2(xq.z, xq.w));
                float a0[SPT], a1[SPT], a2[SPT], a3[SPT];
#pragma unroll
                for (int s = 0; s < SPT; ++s) {
                    const float2 r01 = __fmul2_rn(f2(dq.x, dq.y), A2p[s]);
                    const float2 r23 = __fmul2_rn(f2(dq.z, dq.w), A2p[s]);
                    a0[s] = ex2_approx(r01.x);
                    a1[s] = ex2_approx(r01.y);
                    a2[s] = ex2_approx(r23.x);
                    a3[s] = ex2_approx(r23.y);
                }
                float4 yo;
                yo.x = step(tau + 0, u01.x, a0);
                yo.y = step(tau + 1, u01.y, a1);
                yo.z = step(tau + 2, u23.x, a2);
                yo.w = step(tau + 3, u23.y, a3);
                *reinterpret_cast<float4*>(yrow + tau) = yo;
            }
            if (nfull < nval) {   // ragged last steps of the sequence (uniform)
                for (int t = nfull; t < nval; ++t) {
                    const float dt = load1(drow + t);
                    const float u = dt * load1(xrow + t);
                    float a[SPT];
#pragma unroll
                    for (int s = 0; s < SPT; ++s) a[s] = ex2_approx(dt * A2[s]);
                    yrow[t] = step(t, u, a);
                }
            }
        }
        __syncthreads();

        // ---- sum the G partials of each channel and store y -------------
        {
            IO* yg = static_cast<IO*>(p.y);
            constexpr int Q4 = T / 4;
            for (int i = tid; i < CH * Q4; i += NT) {
                const int cc = i / Q4;
                const int t4 = (i - cc * Q4) * 4;
                const int64_t dd = d0 + cc;
                if (dd >= p.dim || t4 >= nval) continue;
                const float* src = ypart + cc * G * TL::YP + t4;
                float4 s4 = *reinterpret_cast<const float4*>(src);
#pragma unroll
                for (int gg = 1; gg < G; ++gg) {
                    const float4 o = *reinterpret_cast<const float4*>(src + gg * TL::YP);
                    s4.x += o.x; s4.y += o.y; s4.z += o.z; s4.w += o.w;
                }
                IO* dst = yg + ((b * p.dim + dd) * L + t0 + t4);
                if (p.vec_ok && t4 + 4 <= nval) {
                    store4(dst, s4);
                } else {
                    const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
                    for (int e = 0; e < 4 && t4 + e < nval; ++e) store1(dst + e, sv[e]);
                }
            }
        }
    }

    // ---- final states -------------------------------------------------------
    if (active) {
#pragma unroll
        for (int q = 0; q < NPAIR; ++q) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int n = g * SPT + 2 * q + e;
                if (n < N) {
                    const int64_t si = ((b * p.dim + d) * N + n);
                    if (p.hT) p.hT[si] = e ? hh[q].y : hh[q].x;
                    if (p.vT) p.vT[si] = e ? vv[q].y : vv[q].x;
                }
            }
        }
    }
}

// ------------------------------------------------------------- launch -----
namespace {

template <typename IO, int NP, int SPT, int WARPS>
cudaError_t launch_variant(const ScanArgs& a0, cudaStream_t stream) {
    using TL = ScanTile<IO, NP, SPT, WARPS>;
    ScanArgs a = a0;
    a.tiles_per_batch = (int)((a.dim + TL::CH - 1) / TL::CH);
    const int64_t grid = a.batch * a.tiles_per_batch;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    auto kern = scan_fwd_kernel<IO, NP, SPT, WARPS>;
    // The dynamic shared-memory limit is raised once per device and variant.
    static std::atomic<uint64_t> attr_done{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_done.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, TL::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_done.fetch_or(bit, std::memory_order_release);
    }
    kern<<<(unsigned)grid, TL::NT, TL::SMEM_BYTES, stream>>>(a);
    return cudaGetLastError();
}

template <typename IO, int NP>
cudaError_t launch_np(const ScanArgs& a, int spt, int warps, cudaStream_t s) {
    if constexpr (NP >= 4) {
        if (spt == 4) {
            if (warps == 1) return launch_variant<IO, NP, 4, 1>(a, s);
            if (warps == 2) return launch_variant<IO, NP, 4, 2>(a, s);
            if (warps == 4) return launch_variant<IO, NP, 4, 4>(a, s);
        }
    }
    if (spt == 2) {
        if (warps == 1) return launch_variant<IO, NP, 2, 1>(a, s);
        if (warps == 2) return launch_variant<IO, NP, 2, 2>(a, s);
        if (warps == 4) return launch_variant<IO, NP, 2, 4>(a, s);
    }
    return cudaErrorInvalidValue;
}

template <typename IO>
cudaError_t launch_io(const ScanArgs& a, int np, int spt, int warps, cudaStream_t s) {
    switch (np) {
        case 2: return launch_np<IO, 2>(a, 2, warps, s);
        case 4: return launch_np<IO, 4>(a, spt, warps, s);
        case 8: return launch_np<IO, 8>(a, spt, warps, s);
        case 16: return launch_np<IO, 16>(a, spt, warps, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool scan_tile_supported(int spt, int warps) {
    return (spt == 2 || spt == 4) && (warps == 1 || warps == 2 || warps == 4);
}

ScanTileChoice choose_scan_tile(int64_t batch, int64_t dim, int64_t dstate, int io,
                                int forced_spt, int forced_warps) {
    ScanTileChoice t;
    t.np = dstate <= 2 ? 2 : dstate <= 4 ? 4 : dstate <= 8 ? 8 : 16;
    if (forced_spt) {
        t.spt = forced_spt;
        t.warps = forced_warps;
    } else {
        (void)batch; (void)dim; (void)io;
        t.spt = 4;
        t.warps = 2;
    }
    if (t.np == 2) t.spt = 2;
    return t;
}

cudaError_t launch_scan_fwd(const ScanArgs& a, const ScanTileChoice& t, int io, cudaStream_t s) {
    if (io == 0) return launch_io<float>(a, t.np, t.spt, t.warps, s);
    return launch_io<bf16>(a, t.np, t.spt, t.warps, s);
}

}  // namespace mmscan
