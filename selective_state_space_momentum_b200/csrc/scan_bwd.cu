// scan_bwd.cu -- sm_100a kernel for the backward of the Momentum Mamba selective scan.
//
// What it computes: the gradients of the forward in scan_fwd.cu ("Momentum
// Mamba: Enhanced State Space Models with Momentum", "Gradient Flow" and
// "Backward Pass: Reconstructed Forward + Reverse Scans").  The printed
// recursions use one symbol for both state gradients and drop a term, so
// they are derived from the recurrence: per (b, d, n), with G_t = dL/dh_t
// and P_t = dL/dv_t (total derivatives),
//     G_t = dy_t C_t[n] + a_{t+1} G_{t+1},    P_t = G_t + beta P_{t+1}
// starting from dhT, dvT after the last step, and
//     dx_t     = alpha delta_t sum_n B_t[n] P_t[n]
//     ddelta_t = alpha x_t sum_n B_t[n] P_t[n] + sum_n A[d,n] a_t h_{t-1}[n] G_t[n]
//     dA[d,n]  = sum_{b,t} delta_t a_t h_{t-1}[n] G_t[n]
//     dB_t[n]  = sum_d alpha delta_t x_t P_t[n],     dC_t[n] = sum_d dy_t h_t[n]
//     dh0 = a_0 G_0,    dv0 = beta P_0                 (a_t = exp(delta_t A[d,n]))
//
// Design (B200-first; the page's reverse block scans are prior art only):
//  * Work split as in the forward: a CTA owns CH channels of one batch row,
//    G = NP / 2 lanes per channel, two states per lane.  The CTA walks the
//    chunks of 64 steps from the last to the first and carries (G, P) in
//    registers, so the reverse recursion runs in time order and needs no
//    carry recombination.
//  * States.  The forward saved (h, v) after every 16 steps.  Each block of
//    16 steps restarts from the checkpoint before it (h0, v0 for the first),
//    rebuilds its 16 states and exponentials in registers and walks them
//    backwards; the next block's checkpoint is loaded while a block runs.  The
//    rebuilt states are those of the forward kernel bit for bit (same
//    operations in the same order).  Nothing of size (L, D, N) is stored.
//  * Reductions.  The sums over a channel's states (for dx, ddelta) use the
//    forward's register butterfly.  dB and dC sum over channels: a butterfly
//    across the channels of a warp (four steps at a time, so the exchanges
//    are independent) into the warp's own slice of one of two buffers, the
//    slices summed when a block is flushed (tiles whose CTAs would then not fit
//    at full occupancy add into one slice with shared-memory atomics), then one
//    vector atomic add per (4 steps, state) into global
//    memory after each block.  dA collects in registers over the whole sequence and is added
//    once per lane.
//  * Staging: x, delta, dy, B and C tiles by TMA (128-byte swizzle, no
//    multicast), two chunks in flight; B and C transposed to [t][n] fp32 with
//    alpha folded into B, as in the forward.
#include <cuda.h>

#include <atomic>
#include <mutex>
#include <type_traits>

#include "mm_common.cuh"
#include "mm_internal.h"
#include "mm_tma_host.h"

namespace mmscan {

// Device error word of this file's kernel (bounded waits that gave up).
static __device__ unsigned int g_bwd_dev_err = 0;

template <typename IO, int NP, int WARPS, bool EXT = false, bool DET = false>
struct BwdTile {
    static constexpr int SPT = 2;                // states per lane
    static constexpr int G = NP / SPT;           // lanes per channel
    static constexpr int CPW = 32 / G;           // channels per warp
    static constexpr int CH = WARPS * CPW;       // channels per CTA
    static constexpr int NT = WARPS * 32;
    static constexpr int EB = IOTraits<IO>::kBytes;
    static constexpr int BOX_T = 128 / EB;       // steps in one 128-byte swizzled row
    static constexpr int T = 64;                 // steps per chunk (the checkpoint interval)
    static constexpr int NBOX = T / BOX_T;
    static constexpr int STAGES = 2;
    static constexpr int NPT = NP < 8 ? 8 : NP;  // B/C rows per box (whole swizzle atoms)
    static constexpr int XBOX = CH * 128;
    static constexpr int BBOX = NPT * 128;
    static constexpr int OFF_X = 0;
    static constexpr int OFF_D = NBOX * XBOX;
    static constexpr int OFF_Y = 2 * NBOX * XBOX;     // dy, the gradient reaching y
    static constexpr int OFF_B = 3 * NBOX * XBOX;
    static constexpr int OFF_C = OFF_B + NBOX * BBOX;
    static constexpr int OFF_Z = OFF_C + NBOX * BBOX;       // the gate z (selective_scan_fn extras)
    static constexpr int STAGE_BYTES = OFF_Z + (EXT ? NBOX * XBOX : 0);
    static constexpr int BP = NP + 4;            // row pitch (floats) of transposed B/C
    static constexpr int BT_BYTES = T * BP * 4;
    static constexpr int KB = kCkptSteps;        // steps per block (the checkpoint interval)
    static constexpr int R = 8;                  // steps per read-out group
    static constexpr int PER = R / G;            // steps of a group whose sums a lane owns
    static constexpr int RP = 2 * NP;            // dB and dC partials per step
    static constexpr int OFF_BT = STAGES * STAGE_BYTES;   // B^T, then C^T
    static constexpr int OFF_RED = OFF_BT + 2 * BT_BYTES;
    // extras: delta' = softplus(delta + bias) and the gated dy = dy silu(z) of
    // the chunk as fp32 in the fp32 box layout (32 steps x CH rows of 128 B)
    static constexpr int XBOX_F32 = CH * 128;
    static constexpr int EXB = EXT ? (T / 32) * XBOX_F32 : 0;
    // 12 resident warps per SM (<= 168 registers a thread, no spills).  Four
    // 4-warp CTAs would fit the shared memory, but at 128 registers the
    // kernel spills and ran 33% slower on the 384-CTA fp32 grid.
    static constexpr int MIN_CTAS = 12 / WARPS > 0 ? 12 / WARPS : 1;
    // Two blocks' dB, dC partials: one slice per warp, summed when a block is
    // flushed, where MIN_CTAS CTAs of that size still fit an SM (always in the
    // deterministic form, whose sums must not depend on the warps' timing);
    // else one slice that the warps add into with shared-memory atomics.
    static constexpr int smem_with(int red_warps) {
        return OFF_RED + 2 * red_warps * KB * RP * 4 + 2 * EXB + STAGES * 8 + 1024;
    }
    static constexpr int RED_WARPS = DET || MIN_CTAS * (smem_with(WARPS) + 1024) <= 228 * 1024 ? WARPS : 1;
    static constexpr int RED_BYTES = 2 * RED_WARPS * KB * RP * 4;
    static constexpr int OFF_DP = OFF_RED + RED_BYTES;
    static constexpr int OFF_GY = OFF_DP + EXB;
    static constexpr int OFF_BAR = OFF_GY + EXB;
    static constexpr int SMEM_BYTES = OFF_BAR + STAGES * 8 + 1024;   // + alignment slack

    static_assert(G >= 1 && G <= 8 && (G & (G - 1)) == 0, "lanes per channel");
    static_assert(R % G == 0 && BOX_T % R == 0 && T % BOX_T == 0 && KB % R == 0 && T % KB == 0,
                  "step grouping");
    static_assert(CH % 8 == 0, "x tiles must be whole 1024-byte swizzle atoms");
    static_assert(STAGE_BYTES % 1024 == 0 && OFF_BT % 16 == 0 && OFF_RED % 16 == 0, "alignment");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <typename IO, int NP, int WARPS, bool EXT, bool DET>
__global__ void __launch_bounds__(WARPS * 32, BwdTile<IO, NP, WARPS, EXT, DET>::MIN_CTAS)
scan_bwd_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_d,
                const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_B,
                const __grid_constant__ CUtensorMap tm_C, const __grid_constant__ CUtensorMap tm_z,
                const ScanBwdArgs p) {
    using TL = BwdTile<IO, NP, WARPS, EXT, DET>;
    constexpr int G = TL::G, CPW = TL::CPW, CH = TL::CH, NT = TL::NT, T = TL::T, R = TL::R;
    constexpr int ST = TL::STAGES, EB = TL::EB, BP = TL::BP, PER = TL::PER, KB = TL::KB;
    constexpr int RP = TL::RP;

    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (base - raw_addr);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int g = lane % G;
    const int c = warp * CPW + lane / G;             // channel within the CTA
    const int n0 = g * 2;                            // first of the lane's two states
    const int64_t b = blockIdx.x / p.tiles_per_batch;
    const int64_t d0 = (int64_t)(blockIdx.x % p.tiles_per_batch) * CH;
    const int64_t d = d0 + c;
    const bool active = d < p.dim;
    const int64_t L = p.seqlen;
    const int N = p.dstate;
    const int64_t nchunks = (L + T - 1) / T;
    const bool use_tma = p.vec_ok != 0;
    const uint32_t bar0 = base + TL::OFF_BAR;
    float* red = reinterpret_cast<float*>(smem + TL::OFF_RED);
    float* Bt = reinterpret_cast<float*>(smem + TL::OFF_BT);
    float* Ct = Bt + T * BP;

    if (tid == 0) {
        for (int s = 0; s < ST; ++s) mbar_init(bar0 + 8 * s, use_tma ? 1u : (uint32_t)NT);
        fence_barrier_init();
    }
    for (int i = tid; i < 2 * TL::RED_WARPS * KB * RP; i += NT) red[i] = 0.0f;
    int nred = 0;                                    // blocks done: picks the partials buffer
    __syncthreads();

    // ---- per-lane constants and carries -------------------------------------
    float A2v[2], Anv[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int n = n0 + e;
        Anv[e] = (active && n < N) ? p.A[d * N + n] : 0.0f;
        A2v[e] = Anv[e] * kLog2e;
    }
    const float2 A2 = f2(A2v[0], A2v[1]);        // exponent scale (log2 e A)
    const float2 An = f2(Anv[0], Anv[1]);        // A itself, for ddelta
    const float2 beta2 = f2(p.beta, p.beta);
    const float alpha = p.alpha;
    const int64_t srow = (b * p.dim + (active ? d : 0)) * N;   // this channel's state row
    auto load_pair = [&](const float* src, int64_t off = 0) {
        float v[2] = {0.0f, 0.0f};
#pragma unroll
        for (int e = 0; e < 2; ++e)
            if (src && active && n0 + e < N) v[e] = src[off + n0 + e];
        return f2(v[0], v[1]);
    };
    // (h, v) where block gblk (of KB steps, counted over the whole sequence)
    // starts: the checkpoint after block gblk - 1, or (h0, v0)
    const int64_t ncks = (L + KB - 1) / KB;
    auto start_state = [&](int64_t gblk, int which) {
        if (gblk == 0) return load_pair(which ? p.v0 : p.h0, srow);
        return load_pair(p.ckpt + ((b * p.dim + (active ? d : 0)) * ncks + gblk - 1) * 2 * N + which * N, 0);
    };
    float2 cg = load_pair(p.dhT ? p.dhT + srow : nullptr);   // a_{t+1} G_{t+1}
    float2 cp = load_pair(p.dvT ? p.dvT + srow : nullptr);   // beta P_{t+1}
    float2 dA2 = f2(0.0f, 0.0f);

    // ---- staging of one chunk into a stage buffer ----------------------------
    auto issue = [&](int64_t k, int s) {
        if (p.stall) return;      // test only: nothing staged, the waits run out
        const int64_t t0 = k * T;
        const uint32_t sb = base + s * TL::STAGE_BYTES;
        const uint32_t bar = bar0 + 8 * s;
        const bool load_z = EXT && p.z != nullptr;
        if (use_tma) {
            if (tid == 0) {
                mbar_expect_tx(bar, TL::STAGE_BYTES - (EXT && !load_z ? TL::NBOX * TL::XBOX : 0));
#pragma unroll
                for (int bx = 0; bx < TL::NBOX; ++bx) {
                    const int tc = (int)(t0 + bx * TL::BOX_T);
                    tma_load_3d(sb + TL::OFF_X + bx * TL::XBOX, &tm_x, bar, tc, (int)d0, (int)b);
                    tma_load_3d(sb + TL::OFF_D + bx * TL::XBOX, &tm_d, bar, tc, (int)d0, (int)b);
                    tma_load_3d(sb + TL::OFF_Y + bx * TL::XBOX, &tm_y, bar, tc, (int)d0, (int)b);
                    tma_load_3d(sb + TL::OFF_B + bx * TL::BBOX, &tm_B, bar, tc, 0, (int)b);
                    tma_load_3d(sb + TL::OFF_C + bx * TL::BBOX, &tm_C, bar, tc, 0, (int)b);
                    if (load_z) tma_load_3d(sb + TL::OFF_Z + bx * TL::XBOX, &tm_z, bar, tc, (int)d0, (int)b);
                }
            }
            return;
        }
        // Element-wise fill of the same swizzled tiles (rows not 16-byte multiples).
        const IO* srcs[4] = {static_cast<const IO*>(p.x), static_cast<const IO*>(p.delta),
                             static_cast<const IO*>(p.dout), static_cast<const IO*>(p.z)};
        const IO* Bg = static_cast<const IO*>(p.B);
        const IO* Cg = static_cast<const IO*>(p.C);
        constexpr int IOROWS = (EXT ? 4 : 3) * CH;
        constexpr int ROWS = IOROWS + 2 * TL::NPT;
        for (int i = tid; i < ROWS * T; i += NT) {
            const int r = i / T;
            const int tau = i - r * T;
            const int bx = tau / TL::BOX_T;
            const int col = tau - bx * TL::BOX_T;
            const int64_t t = t0 + tau;
            const IO* src = nullptr;
            uint32_t off;
            if (r < IOROWS) {
                const int which = r / CH;
                const int cc = r - which * CH;
                off = (which == 3 ? TL::OFF_Z : which * TL::NBOX * TL::XBOX) + bx * TL::XBOX + sw128(cc, col * EB);
                if (srcs[which] && d0 + cc < p.dim && t < L) src = srcs[which] + ((b * p.dim + d0 + cc) * L + t);
            } else {
                const int rr = r - IOROWS;
                const int n = rr < TL::NPT ? rr : rr - TL::NPT;
                off = (rr < TL::NPT ? TL::OFF_B : TL::OFF_C) + bx * TL::BBOX + sw128(n, col * EB);
                if (n < N && t < L) src = (rr < TL::NPT ? Bg : Cg) + ((b * N + n) * L + t);
            }
            if constexpr (EB == 4) {
                cp_async_4(smem + s * TL::STAGE_BYTES + off, src ? src : srcs[0], src ? 4 : 0);
            } else {
                *reinterpret_cast<IO*>(smem + s * TL::STAGE_BYTES + off) = src ? *src : IO(0.0f);
            }
        }
        if constexpr (EB == 4) cp_async_mbar_arrive(bar);
        else mbar_arrive(bar);
    };

    // The i-th chunk processed (chunk nchunks - 1 - i) goes to stage i % ST.
#pragma unroll
    for (int i = 0; i < ST - 1; ++i)
        if (i < nchunks) issue(nchunks - 1 - i, i);

    IO* dxrow = static_cast<IO*>(p.dx) + (b * p.dim + (active ? d : 0)) * L;
    IO* ddrow = static_cast<IO*>(p.ddelta) + (b * p.dim + (active ? d : 0)) * L;
    // selective_scan_fn extras: skip weight, bias, and the per-channel sums dD, d bias
    IO* dzrow = (EXT && p.dz) ? static_cast<IO*>(p.dz) + (b * p.dim + (active ? d : 0)) * L : nullptr;
    const float skip_d = (EXT && p.Dskip && active) ? p.Dskip[d] : 0.0f;
    const float dbias_d = (EXT && p.dbias && active) ? p.dbias[d] : 0.0f;
    float acc_dD = 0.0f, acc_db = 0.0f;
    const bool vec_out = use_tma;
    const bool vec_red = (L % 4) == 0;

    for (int64_t i = 0; i < nchunks; ++i) {
        const int64_t k = nchunks - 1 - i;
        const int s = (int)(i % ST);
        const int64_t t0 = k * T;
        const int nval = (int)((L - t0) < T ? (L - t0) : T);
        const int nblk = (nval + KB - 1) / KB;
        // start state of the chunk's last block: loaded before the wait, and each
        // block's predecessor is fetched while the block runs
        float2 hn = start_state(k * (T / KB) + nblk - 1, 0);
        float2 vn = start_state(k * (T / KB) + nblk - 1, 1);
        // Every thread waits; the outcome is made uniform at the barrier below, so
        // that a wait that gave up makes the whole CTA leave together.
        const bool waited = mbar_wait(bar0 + 8 * s, (uint32_t)((i / ST) & 1), &g_bwd_dev_err);
        const unsigned char* sbuf = smem + s * TL::STAGE_BYTES;

        // ---- transpose B, C to [t][n] fp32 in 4x4 blocks (alpha into B) ----
        if (waited) {
            constexpr int NB4 = NP / 4 > 0 ? NP / 4 : 1;
            constexpr int ITEMS = NB4 * (T / 4);
            for (int it = tid; it < 2 * ITEMS; it += NT) {
                const int which = it / ITEMS;
                const int rem = it - which * ITEMS;
                const int nb = (rem % NB4) * 4;
                const int t4 = (rem / NB4) * 4;
                const int bx = t4 / TL::BOX_T;
                const int col = t4 - bx * TL::BOX_T;
                const unsigned char* tile = sbuf + (which ? TL::OFF_C : TL::OFF_B) + bx * TL::BBOX;
                float m[4][4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    if (nb + r < NP) {
                        const float4 q = load4(reinterpret_cast<const IO*>(tile + sw128(nb + r, col * EB)));
                        m[r][0] = q.x; m[r][1] = q.y; m[r][2] = q.z; m[r][3] = q.w;
                    } else {
                        m[r][0] = m[r][1] = m[r][2] = m[r][3] = 0.0f;
                    }
                }
                const float sc = which ? 1.0f : alpha;
                float* dst = (which ? Ct : Bt) + t4 * BP + nb;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if constexpr (NP >= 4) {
                        *reinterpret_cast<float4*>(dst + j * BP) =
                            make_float4(m[0][j] * sc, m[1][j] * sc, m[2][j] * sc, m[3][j] * sc);
                    } else {
                        dst[j * BP] = m[0][j] * sc;
                        dst[j * BP + 1] = m[1][j] * sc;
                    }
                }
            }
        }
        if constexpr (EXT) {
            // delta' = softplus(delta + bias) and the gated dy = dy silu(z), once per
            // (channel, step), four steps per item, into the fp32 buffers
            for (int it = waited ? tid : CH * (T / 4); it < CH * (T / 4); it += NT) {
                const int cc = it / (T / 4);
                const int t4 = (it - cc * (T / 4)) * 4;
                const int bxs = t4 / TL::BOX_T;
                const uint32_t so = bxs * TL::XBOX + sw128(cc, (t4 - bxs * TL::BOX_T) * EB);
                const float4 dq = load4(reinterpret_cast<const IO*>(sbuf + TL::OFF_D + so));
                const float4 yq = load4(reinterpret_cast<const IO*>(sbuf + TL::OFF_Y + so));
                const float bv = (p.dbias && d0 + cc < p.dim) ? p.dbias[d0 + cc] : 0.0f;
                float dv[4] = {dq.x + bv, dq.y + bv, dq.z + bv, dq.w + bv};
                float gy[4] = {yq.x, yq.y, yq.z, yq.w};
                if (p.softplus) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) dv[e] = softplus_f32(dv[e]);
                }
                if (p.z) {
                    const float4 zq = load4(reinterpret_cast<const IO*>(sbuf + TL::OFF_Z + so));
                    const float zv[4] = {zq.x, zq.y, zq.z, zq.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) gy[e] *= __fdividef(zv[e], 1.0f + ex2_approx(-zv[e] * kLog2e));
                }
                const uint32_t fo = (t4 / 32) * TL::XBOX_F32 + sw128(cc, (t4 % 32) * 4);
                *reinterpret_cast<float4*>(smem + TL::OFF_DP + fo) = make_float4(dv[0], dv[1], dv[2], dv[3]);
                *reinterpret_cast<float4*>(smem + TL::OFF_GY + fo) = make_float4(gy[0], gy[1], gy[2], gy[3]);
            }
        }
        if (!__syncthreads_and(waited)) return;
        // Every thread is past the previous chunk: its stage is free.
        if (i + ST - 1 < nchunks) issue(nchunks - 1 - (i + ST - 1), (int)((i + ST - 1) % ST));

        // delta, x or dy of the 4 steps from tau, this lane's channel
        auto load4s = [&](int off, int tau) {
            const int bx = tau / TL::BOX_T;
            const int col = tau - bx * TL::BOX_T;
            return load4(reinterpret_cast<const IO*>(sbuf + off + bx * TL::XBOX + sw128(c, col * EB)));
        };
        auto load1s = [&](int off, int tau) {
            const int bx = tau / TL::BOX_T;
            const int col = tau - bx * TL::BOX_T;
            return load1(reinterpret_cast<const IO*>(sbuf + off + bx * TL::XBOX + sw128(c, col * EB)));
        };
        // delta' and the dy reaching the read-out (with the extras: the fp32 buffers)
        auto ld_delta4 = [&](int tau) {
            if constexpr (EXT)
                return *reinterpret_cast<const float4*>(smem + TL::OFF_DP + (tau / 32) * TL::XBOX_F32 +
                                                        sw128(c, (tau % 32) * 4));
            else
                return load4s(TL::OFF_D, tau);
        };
        auto ld_dy4 = [&](int tau) {
            if constexpr (EXT)
                return *reinterpret_cast<const float4*>(smem + TL::OFF_GY + (tau / 32) * TL::XBOX_F32 +
                                                        sw128(c, (tau % 32) * 4));
            else
                return load4s(TL::OFF_Y, tau);
        };
        auto ld_f32 = [&](int off, int tau) {      // one value of an fp32 extras buffer
            return *reinterpret_cast<const float*>(smem + off + (tau / 32) * TL::XBOX_F32 +
                                                   sw128(c, (tau % 32) * 4));
        };
        // one forward step of the lane's two states (the forward kernel's operations)
        auto fwd_step = [&](int tau, float dl, float u, float2& h, float2& v, float2& a) {
            const float2 bq = *reinterpret_cast<const float2*>(Bt + tau * BP + n0);
            const float2 r2 = __fmul2_rn(f2(dl, dl), A2);
            a = f2(ex2_approx(r2.x), ex2_approx(r2.y));
            const float2 w = __fmul2_rn(f2(u, u), bq);
            v = __ffma2_rn(beta2, v, w);
            h = __ffma2_rn(a, h, v);
        };
        // dB, dC partials of 4 consecutive steps from tau: summed over the
        // warp's channels by a butterfly (the lane keeps dB or dC, then one of
        // its two states) and stored into the warp's slice (each slot of a step
        // has one writer in the warp; shared-memory atomics across the warps
        // had cost a fifth of the kernel's time)
        auto chan_reduce4 = [&](float* redb, int tau, const float2 (&dBv)[4], const float2 (&dCv)[4]) {
            const bool up1 = (lane & 16) != 0;
            const bool up2 = (lane & 8) != 0;
            float r[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                float k0 = up1 ? dCv[jj].x : dBv[jj].x, k1 = up1 ? dCv[jj].y : dBv[jj].y;
                const float s0 = up1 ? dBv[jj].x : dCv[jj].x, s1 = up1 ? dBv[jj].y : dCv[jj].y;
                k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
                k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
                r[jj] = (up2 ? k1 : k0) + __shfl_xor_sync(0xffffffffu, up2 ? k0 : k1, 8);
            }
#pragma unroll
            for (int m = G; m < 8; m <<= 1) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) r[jj] += __shfl_xor_sync(0xffffffffu, r[jj], m);
            }
            if ((lane & 7) < G) {
                float* dst = redb + tau * RP + (up1 ? NP : 0) + n0 + (up2 ? 1 : 0);
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    if constexpr (TL::RED_WARPS > 1) dst[jj * RP] = r[jj];
                    else atomicAdd(dst + jj * RP, r[jj]);
                }
            }
        };
        // One block of KB steps (the first kmax valid) from its start state:
        // rebuild its states, then walk it backwards (the exponentials are
        // formed again there: two MUFU operations instead of 32 registers).
        // kmax is a compile-time KB for whole blocks.
        auto block = [&](int blk, auto kmax, float2 h, float2 v, float* redb) {
            const int tb = blk * KB;
            float2 ht[KB];
            const float2 hprev0 = h;
#pragma unroll
            for (int j4 = 0; j4 < KB; j4 += 4) {
                if (j4 < kmax) {
                    const float4 dq = ld_delta4(tb + j4);
                    const float4 xq = load4s(TL::OFF_X, tb + j4);
                    const float dl[4] = {dq.x, dq.y, dq.z, dq.w}, xl[4] = {xq.x, xq.y, xq.z, xq.w};
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        float2 a;
                        if (j4 + jj < kmax) fwd_step(tb + j4 + jj, dl[jj], dl[jj] * xl[jj], h, v, a);
                        ht[j4 + jj] = h;
                    }
                }
            }
#pragma unroll
            for (int hf = KB / R - 1; hf >= 0; --hf) {
                if (hf * R >= kmax) continue;
                float sk[R], qk[R], yk[EXT ? R : 1];
#pragma unroll
                for (int j4 = R - 4; j4 >= 0; j4 -= 4) {
                    const int jb = hf * R + j4;              // first of these 4 steps in the block
                    float2 dBv[4], dCv[4];
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        sk[j4 + jj] = qk[j4 + jj] = 0.0f;
                        if constexpr (EXT) yk[j4 + jj] = 0.0f;
                        dBv[jj] = dCv[jj] = f2(0.0f, 0.0f);
                    }
                    if (jb < kmax) {
                        const float4 dq = ld_delta4(tb + jb);
                        const float4 xq = load4s(TL::OFF_X, tb + jb);
                        const float4 yq = ld_dy4(tb + jb);
                        const float dl[4] = {dq.x, dq.y, dq.z, dq.w}, xl[4] = {xq.x, xq.y, xq.z, xq.w};
                        const float yl[4] = {yq.x, yq.y, yq.z, yq.w};
#pragma unroll
                        for (int jj = 3; jj >= 0; --jj) {
                            const int j = jb + jj;
                            if (j < kmax) {
                                const int tau = tb + j;
                                const float2 bq = *reinterpret_cast<const float2*>(Bt + tau * BP + n0);
                                const float2 cq = *reinterpret_cast<const float2*>(Ct + tau * BP + n0);
                                const float2 Gt = __ffma2_rn(cq, f2(yl[jj], yl[jj]), cg);
                                const float2 Pt = __fadd2_rn(Gt, cp);
                                const float2 hp = j > 0 ? ht[j > 0 ? j - 1 : 0] : hprev0;
                                const float2 r2 = __fmul2_rn(f2(dl[jj], dl[jj]), A2);
                                const float2 at = f2(ex2_approx(r2.x), ex2_approx(r2.y));
                                const float2 dt2 = __fmul2_rn(__fmul2_rn(at, hp), Gt);      // a_t h_{t-1} G_t
                                const float2 s2 = __fmul2_rn(Pt, bq);                       // alpha B P
                                const float2 q2 = __fmul2_rn(dt2, An);
                                sk[j4 + jj] = s2.x + s2.y;
                                qk[j4 + jj] = q2.x + q2.y;
                                dA2 = __ffma2_rn(f2(dl[jj], dl[jj]), dt2, dA2);
                                const float ua = dl[jj] * xl[jj] * alpha;
                                dBv[jj] = __fmul2_rn(Pt, f2(ua, ua));
                                dCv[jj] = __fmul2_rn(f2(yl[jj], yl[jj]), ht[j]);
                                if constexpr (EXT) {     // the read-out itself, for dz
                                    const float2 cy = __fmul2_rn(cq, ht[j]);
                                    yk[j4 + jj] = cy.x + cy.y;
                                }
                                cg = __fmul2_rn(at, Gt);
                                cp = __fmul2_rn(beta2, Pt);
                            }
                        }
                        chan_reduce4(redb + (TL::RED_WARPS > 1 ? warp : 0) * (KB * RP), jb, dBv, dCv);
                    }
                }
                // per-channel sums of these R steps; lane g owns PER of them
                float so[PER], qo[PER];
                butterfly_sum<G, R>(sk, so, g);
                butterfly_sum<G, R>(qk, qo, g);
                const int first = tb + hf * R + g * PER;
                const int cnt = nval - first < PER ? nval - first : PER;
                float gx[PER], gd[PER];
                if constexpr (!EXT) {
#pragma unroll
                    for (int e = 0; e < PER; ++e) {
                        gx[e] = load1s(TL::OFF_D, first + e) * so[e];
                        gd[e] = __fmaf_rn(load1s(TL::OFF_X, first + e), so[e], qo[e]);
                    }
                } else {
                    float yo[PER], gz[PER];
                    if (p.z) butterfly_sum<G, R>(yk, yo, g);
#pragma unroll
                    for (int e = 0; e < PER; ++e) {
                        const int st = first + e;
                        const bool valid = e < cnt;
                        const float xe = load1s(TL::OFF_X, st);
                        const float gye = ld_f32(TL::OFF_GY, st);
                        gx[e] = __fmaf_rn(skip_d, gye, ld_f32(TL::OFF_DP, st) * so[e]);
                        gd[e] = __fmaf_rn(xe, so[e], qo[e]);          // d delta'
                        if (p.softplus) {                             // * sigmoid(delta + bias)
                            const float uu = load1s(TL::OFF_D, st) + dbias_d;
                            gd[e] *= __fdividef(1.0f, 1.0f + ex2_approx(-uu * kLog2e));
                        }
                        if (valid) {
                            acc_dD = __fmaf_rn(gye, xe, acc_dD);
                            acc_db += gd[e];
                        }
                        if (p.z) {          // dz = dy (y + D x) s (1 + z (1 - s)), s = sigmoid(z)
                            const float zv = load1s(TL::OFF_Z, st);
                            const float sg = __fdividef(1.0f, 1.0f + ex2_approx(-zv * kLog2e));
                            const float o = __fmaf_rn(skip_d, xe, yo[e]);
                            gz[e] = load1s(TL::OFF_Y, st) * o * sg * __fmaf_rn(zv, 1.0f - sg, 1.0f);
                        }
                    }
                    if (p.z && p.dz && active && cnt > 0)
                        store_steps_n<IO, PER>(dzrow + t0 + first, gz, cnt, vec_out);
                }
                if (active && cnt > 0) {
                    store_steps_n<IO, PER>(dxrow + t0 + first, gx, cnt, vec_out);
                    store_steps_n<IO, PER>(ddrow + t0 + first, gd, cnt, vec_out);
                }
            }
        };

#pragma unroll 1
        for (int blk = nblk - 1; blk >= 0; --blk) {
            const float2 h = hn, v = vn;
            if (blk > 0) {
                hn = start_state(k * (T / KB) + blk - 1, 0);
                vn = start_state(k * (T / KB) + blk - 1, 1);
            }
            const int kmax = nval - blk * KB < KB ? nval - blk * KB : KB;
            float* redb = red + (nred & 1) * (TL::RED_WARPS * KB * RP);
            if (kmax == KB) block(blk, std::integral_constant<int, KB>{}, h, v, redb);
            else block(blk, kmax, h, v, redb);
            ++nred;

            // ---- the block's dB, dC into global memory (the other buffer is
            // the next block's; this one is next written two blocks later) ----
            __syncthreads();
            for (int it = tid; it < (KB / 4) * RP; it += NT) {
                const int slot = it % RP;
                const int t4 = (it / RP) * 4;
                // the warps' slices in a fixed order (entries of steps past kmax
                // are stale and never used); one slice of atomic sums is zeroed
                // for its next block
                float v4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float acc = redb[(t4 + e) * RP + slot];
#pragma unroll
                    for (int w = 1; w < TL::RED_WARPS; ++w) acc += redb[w * (KB * RP) + (t4 + e) * RP + slot];
                    if constexpr (TL::RED_WARPS == 1) redb[(t4 + e) * RP + slot] = 0.0f;
                    v4[e] = acc;
                }
                const int which = slot / NP;
                const int n = slot - which * NP;
                if (DET && n < N && t4 < kmax) {
                    // the deterministic form: this channel tile's partial, stored once
                    // per element, summed over the tiles in order by the reduce kernel
                    const int64_t tile = blockIdx.x % p.tiles_per_batch;
                    float* dst = p.ws_bc + ((tile * 2 + which) * p.batch + b) * N * L + n * L + t0 + blk * KB + t4;
                    if (vec_red && t4 + 4 <= kmax) {
                        *reinterpret_cast<float4*>(dst) = make_float4(v4[0], v4[1], v4[2], v4[3]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (t4 + e < kmax) dst[e] = v4[e];
                    }
                } else if (n < N && t4 < kmax) {
                    float* dst = (which ? p.dC : p.dB) + (b * N + n) * L + t0 + blk * KB + t4;
                    if (vec_red && t4 + 4 <= kmax) {
                        atomicAdd(reinterpret_cast<float4*>(dst), make_float4(v4[0], v4[1], v4[2], v4[3]));
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (t4 + e < kmax) atomicAdd(dst + e, v4[e]);
                    }
                }
            }
        }
    }

    // ---- dD, d bias: this lane's steps, then the G lanes of the channel ----------
    if constexpr (EXT) {
#pragma unroll
        for (int m = G / 2; m >= 1; m >>= 1) {
            acc_dD += __shfl_xor_sync(0xffffffffu, acc_dD, m);
            acc_db += __shfl_xor_sync(0xffffffffu, acc_db, m);
        }
        if (active && g == 0) {
            if constexpr (DET) {
                if (p.dD) p.ws_d[b * p.dim + d] = acc_dD;
                if (p.ddbias) p.ws_d[(p.batch + b) * p.dim + d] = acc_db;
            } else {
                if (p.dD) atomicAdd(p.dD + d, acc_dD);
                if (p.ddbias) atomicAdd(p.ddbias + d, acc_db);
            }
        }
    }

    // ---- gradients of the start state; dA ------------------------------------
    if (active) {
        const float gh[2] = {cg.x, cg.y}, gv[2] = {cp.x, cp.y}, ga[2] = {dA2.x, dA2.y};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int n = n0 + e;
            if (n < N) {
                if (p.dh0) p.dh0[srow + n] = gh[e];
                if (p.dv0) p.dv0[srow + n] = gv[e];
                if constexpr (DET) p.ws_a[(b * p.dim + d) * N + n] = ga[e];
                else atomicAdd(p.dA + d * N + n, ga[e]);
            }
        }
    }
}

// ------------------------------------------------------------- launch -----
namespace {

template <typename IO, int NP, int WARPS, bool EXT, bool DET>
cudaError_t launch_bwd_variant(const ScanBwdArgs& a0, cudaStream_t stream) {
    using TL = BwdTile<IO, NP, WARPS, EXT, DET>;
    ScanBwdArgs a = a0;
    a.tiles_per_batch = (int)((a.dim + TL::CH - 1) / TL::CH);
    const int64_t grid = a.batch * a.tiles_per_batch;
    if (grid > 0x7fffffffLL || a.dim > 0x7fffffffLL || a.batch > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    CUtensorMap mx, md, my, mB, mC, mz;
    memset(&mx, 0, sizeof(mx)); memset(&md, 0, sizeof(md)); memset(&my, 0, sizeof(my));
    memset(&mB, 0, sizeof(mB)); memset(&mC, 0, sizeof(mC)); memset(&mz, 0, sizeof(mz));
    if (a.vec_ok) {
        const bool bf = sizeof(IO) == 2;
        const uint64_t L = (uint64_t)a.seqlen;
        cudaError_t e;
        if ((e = make_map_3d(&mx, a.x, bf, L, a.dim, a.batch, TL::BOX_T, TL::CH)) != cudaSuccess) return e;
        if ((e = make_map_3d(&md, a.delta, bf, L, a.dim, a.batch, TL::BOX_T, TL::CH)) != cudaSuccess) return e;
        if ((e = make_map_3d(&my, a.dout, bf, L, a.dim, a.batch, TL::BOX_T, TL::CH)) != cudaSuccess) return e;
        if ((e = make_map_3d(&mB, a.B, bf, L, a.dstate, a.batch, TL::BOX_T, TL::NPT)) != cudaSuccess) return e;
        if ((e = make_map_3d(&mC, a.C, bf, L, a.dstate, a.batch, TL::BOX_T, TL::NPT)) != cudaSuccess) return e;
        if (EXT && a.z && (e = make_map_3d(&mz, a.z, bf, L, a.dim, a.batch, TL::BOX_T, TL::CH)) != cudaSuccess)
            return e;
    }
    auto kern = scan_bwd_kernel<IO, NP, WARPS, EXT, DET>;
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
    kern<<<(unsigned)grid, TL::NT, TL::SMEM_BYTES, stream>>>(mx, md, my, mB, mC, mz, a);
    return cudaGetLastError();
}

template <typename IO, bool EXT, bool DET>
cudaError_t launch_bwd_io(const ScanBwdArgs& a, cudaStream_t s) {
    const int64_t channels = a.batch * a.dim;
    const int N = a.dstate;
    if (N > 8)
        return channels >= 2048 ? launch_bwd_variant<IO, 16, 4, EXT, DET>(a, s)
                                : launch_bwd_variant<IO, 16, 2, EXT, DET>(a, s);
    if (N > 4) return launch_bwd_variant<IO, 8, 2, EXT, DET>(a, s);
    if (N > 2) return launch_bwd_variant<IO, 4, 2, EXT, DET>(a, s);
    return launch_bwd_variant<IO, 2, 2, EXT, DET>(a, s);
}

// Channels of one CTA of the backward for these sizes (the tile launch_bwd_io picks).
int bwd_tile_channels(int64_t batch, int64_t dim, int N) {
    if (N > 8)
        return batch * dim >= 2048 ? BwdTile<float, 16, 4>::CH : BwdTile<float, 16, 2>::CH;
    if (N > 4) return BwdTile<float, 8, 2>::CH;
    if (N > 2) return BwdTile<float, 4, 2>::CH;
    return BwdTile<float, 2, 2>::CH;
}

// The deterministic form's sums: each output element adds its partials in a
// fixed order -- dB, dC over the channel tiles of the batch row (tile 0
// first), dA, dD and d bias over the batch rows (row 0 first) -- and is
// written, not added to.
__global__ void __launch_bounds__(256) bwd_det_reduce_kernel(const ScanBwdArgs p) {
    const int64_t nbc = p.batch * p.dstate * p.seqlen;     // elements of dB (and of dC)
    const int64_t na = p.dim * p.dstate;
    const int64_t total = 2 * nbc + na + 2 * p.dim;
    const int64_t tiles = p.tiles_per_batch;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        if (i < 2 * nbc) {
            // partials laid out [tile][dB or dC][batch][state][step]
            float acc = 0.0f;
#pragma unroll 8
            for (int64_t k = 0; k < tiles; ++k) acc += p.ws_bc[k * 2 * nbc + i];
            if (i < nbc) p.dB[i] = acc;
            else p.dC[i - nbc] = acc;
        } else if (i < 2 * nbc + na) {
            const int64_t j = i - 2 * nbc;                   // (channel, state)
            float acc = 0.0f;
            for (int64_t r = 0; r < p.batch; ++r) acc += p.ws_a[r * na + j];
            p.dA[j] = acc;
        } else {
            const int64_t j = i - 2 * nbc - na;              // [dD or d bias][channel]
            const int which = j >= p.dim ? 1 : 0;
            const int64_t d = j - which * p.dim;
            float* dst = which ? p.ddbias : p.dD;
            if (!dst) continue;
            float acc = 0.0f;
            for (int64_t r = 0; r < p.batch; ++r) acc += p.ws_d[(which * p.batch + r) * p.dim + d];
            dst[d] = acc;
        }
    }
}

}  // namespace

namespace {

// Stream-ordered memory for the deterministic form's workspace: one pool per
// device, created on first use, keeping up to kDetKeepBytes reserved between
// calls (a workspace given back to the driver at every synchronisation had
// to be mapped again by the next call, which cost more than the backward).
constexpr int kDetPoolDevices = 64;
constexpr uint64_t kDetKeepBytes = uint64_t(2) << 30;
std::mutex g_det_pool_mutex;
cudaMemPool_t g_det_pool[kDetPoolDevices] = {};

cudaMemPool_t det_pool() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDetPoolDevices) {
        (void)cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_det_pool_mutex);
    if (g_det_pool[dev]) return g_det_pool[dev];
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
        (void)cudaGetLastError();
        return nullptr;
    }
    uint64_t keep = kDetKeepBytes;
    (void)cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    g_det_pool[dev] = pool;
    return pool;
}

}  // namespace

bool stream_capturing(cudaStream_t s) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    return cap != cudaStreamCaptureStatusNone;
}

int64_t scan_bwd_det_workspace_bytes(int64_t batch, int64_t dim, int dstate, int64_t seqlen) {
    const int64_t tiles = (dim + bwd_tile_channels(batch, dim, dstate) - 1) / bwd_tile_channels(batch, dim, dstate);
    const double floats = (double)tiles * 2.0 * batch * dstate * seqlen + (double)batch * dim * dstate +
                          2.0 * batch * dim;
    if (floats * 4.0 > 9.0e18) return -1;
    return (int64_t)floats * 4;
}

cudaError_t launch_scan_bwd(const ScanBwdArgs& a0, int io, cudaStream_t s) {
    cudaError_t e;
    if (a0.det) {
        // Per-tile partials into a workspace in stream-ordered memory, then the
        // fixed-order sums; nothing is added atomically.
        const int64_t bytes = scan_bwd_det_workspace_bytes(a0.batch, a0.dim, a0.dstate, a0.seqlen);
        if (bytes < 0) return cudaErrorInvalidValue;
        void* ws = nullptr;
        cudaMemPool_t pool = det_pool();
        if (!pool) return cudaErrorMemoryAllocation;
        if ((e = cudaMallocFromPoolAsync(&ws, (size_t)bytes, pool, s)) != cudaSuccess) return e;
        ScanBwdArgs a = a0;
        a.tiles_per_batch = (int)((a.dim + bwd_tile_channels(a.batch, a.dim, a.dstate) - 1) /
                                  bwd_tile_channels(a.batch, a.dim, a.dstate));
        a.ws_bc = static_cast<float*>(ws);
        a.ws_a = a.ws_bc + (int64_t)a.tiles_per_batch * 2 * a.batch * a.dstate * a.seqlen;
        a.ws_d = a.ws_a + a.batch * a.dim * a.dstate;
        e = a.ext ? (io == 0 ? launch_bwd_io<float, true, true>(a, s) : launch_bwd_io<bf16, true, true>(a, s))
                  : (io == 0 ? launch_bwd_io<float, false, true>(a, s) : launch_bwd_io<bf16, false, true>(a, s));
        if (e == cudaSuccess) {
            const int64_t total = 2 * a.batch * a.dstate * a.seqlen + a.dim * a.dstate + 2 * a.dim;
            int64_t blocks = (total + 255) / 256;
            if (blocks > 148 * 16) blocks = 148 * 16;
            bwd_det_reduce_kernel<<<(unsigned)blocks, 256, 0, s>>>(a);
            e = cudaGetLastError();
        }
        const cudaError_t ef = cudaFreeAsync(ws, s);
        return e != cudaSuccess ? e : ef;
    }
    const ScanBwdArgs& a = a0;
    // dA, dB, dC (and dD, d bias) are sums that the kernel adds into: start them at zero.
    if ((e = cudaMemsetAsync(a.dA, 0, (size_t)a.dim * a.dstate * 4, s)) != cudaSuccess) return e;
    const size_t bc = (size_t)a.batch * a.dstate * a.seqlen * 4;
    if ((e = cudaMemsetAsync(a.dB, 0, bc, s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(a.dC, 0, bc, s)) != cudaSuccess) return e;
    if (a.dD && (e = cudaMemsetAsync(a.dD, 0, (size_t)a.dim * 4, s)) != cudaSuccess) return e;
    if (a.ddbias && (e = cudaMemsetAsync(a.ddbias, 0, (size_t)a.dim * 4, s)) != cudaSuccess) return e;
    if (a.ext) return io == 0 ? launch_bwd_io<float, true, false>(a, s) : launch_bwd_io<bf16, true, false>(a, s);
    return io == 0 ? launch_bwd_io<float, false, false>(a, s) : launch_bwd_io<bf16, false, false>(a, s);
}

unsigned int scan_bwd_read_and_clear_device_error() {
    unsigned int v = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_bwd_dev_err, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_bwd_dev_err, &z, sizeof(z));
    return v;
}

}  // namespace mmscan
