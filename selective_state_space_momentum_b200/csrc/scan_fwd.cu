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
//    shared by all channels of a row) and walks the whole sequence.  G = NP /
//    SPT consecutive lanes share a channel; each lane keeps SPT consecutive
//    states (v, h) in fp32 registers for the whole call, so the recurrence
//    runs in time order and needs no carry recombination.
//  * Staging.  The sequence is cut into chunks of T = 64 steps.  One thread
//    issues TMA tile loads (no multicast) of the chunk's x and delta rows and
//    of the batch row's B and C into shared memory, 128-byte swizzled, with
//    three chunks in flight on mbarriers.  TMA zero-fills past L, D and N.
//    Rows whose byte length is not a multiple of 16 cannot be described to
//    TMA; for them the same tiles are filled element by element.
//  * B and C are transposed to [t][n] fp32 (alpha folded into B) in 4x4
//    blocks, double-buffered, so a lane reads its SPT states of a step with
//    one vector load and the CTA needs one barrier per chunk.
//  * Arithmetic, per group of 8 steps: one MUFU ex2 per (step, state) for
//    exp(delta A) (A pre-scaled by log2 e), and packed f32x2 multiply / FMA
//    for the write, the velocity, the hidden state and the read-out -- two
//    states per instruction.  Nothing of size (L, D, N) is ever stored.
//  * Read-out.  The G lanes of a channel add their partial C_t . h_t by a
//    register butterfly (shuffles, no shared memory) and store y directly:
//    the G lanes write consecutive steps of their channel.
//  * Checkpoints (optional).  (h, v) after every 16 steps go to a
//    (batch, dim, ceil(L / 16), 2, N) buffer that the backward restarts from.
//  * Final state.  (h, v) after the last step go to hT, vT.  With one time
//    lane (TS = 1) the per-state operation sequence does not depend on where
//    the sequence is cut into calls, so split calls reproduce hT, vT bit for
//    bit at any split.  The time split (TS = 2) runs a full 32-step chunk as
//    a zero-start second half plus a carry correction but a ragged chunk in
//    order, so its splits reproduce hT, vT only at multiples of 32 steps.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "mm_common.cuh"
#include "mm_internal.h"
#include "mm_tma_host.h"

namespace mmscan {

// Device error word of this file's kernels (bounded waits that gave up).
static __device__ unsigned int g_scan_dev_err = 0;

template <typename IO, int NP, int SPT, int WARPS, int TS, bool EXT = false>
struct ScanTile {
    static constexpr int G = NP / SPT;           // lanes per (channel, time-lane)
    static constexpr int CPW = 32 / (G * TS);    // channels per warp
    static constexpr int CH = WARPS * CPW;       // channels per CTA
    static constexpr int NT = WARPS * 32;        // threads per CTA
    // The time split doubles the warps; 12 resident warps per SM (<= 168 registers)
    // hold the medium-size grids in one wave.  bf16 tiles need less shared memory,
    // so four 4-warp CTAs fit per SM when registers allow (<= 128 per thread).
    static constexpr int MIN_CTAS = TS == 2 ? (12 / WARPS > 0 ? 12 / WARPS : 1)
                                            : (SPT == 2 && WARPS == 4 && sizeof(IO) == 2 ? 4 : 1);
    static constexpr int NPAIR = SPT / 2;
    static constexpr int EB = IOTraits<IO>::kBytes;
    static constexpr int BOX_T = 128 / EB;       // steps in one 128-byte swizzled row
    static constexpr int T = TS == 1 ? 64 : 32;  // steps per chunk
    static constexpr int NBOX = T / BOX_T;       // boxes per row per chunk
    static constexpr int STAGES = 3;             // chunks in flight
    static constexpr int NPT = NP < 8 ? 8 : NP;  // B/C rows per box (whole swizzle atoms)
    static constexpr int XBOX = CH * 128;        // bytes of one x (or delta) box
    static constexpr int BBOX = NPT * 128;       // bytes of one B (or C) box
    static constexpr int OFF_X = 0;
    static constexpr int OFF_D = NBOX * XBOX;
    static constexpr int OFF_B = 2 * NBOX * XBOX;
    static constexpr int OFF_C = OFF_B + NBOX * BBOX;
    static constexpr int STAGE_BYTES = OFF_C + NBOX * BBOX;
    static constexpr int TX_BYTES = STAGE_BYTES;  // every box is written in full
    static constexpr int BP = NP + 4;            // row pitch (floats) of transposed B/C
    static constexpr int BT_BYTES = T * BP * 4;
    static constexpr int R = 8;                  // steps per inner group
    static constexpr int OFF_BT = STAGES * STAGE_BYTES;    // 2 buffers of B^T, then 2 of C^T
    // selective_scan_fn extras: delta' = softplus(delta + bias) per (channel,
    // step) as fp32 in the fp32 box layout (32 steps x CH rows of 128 bytes):
    // in place in the delta tile for fp32 I/O, else in two buffers of its own.
    static constexpr int XBOX_F32 = CH * 128;    // one 32-step fp32 box of CH rows
    static constexpr int DP_BYTES = (EXT && EB == 2) ? (T / 32) * XBOX_F32 : 0;
    static constexpr int OFF_DP = OFF_BT + 4 * BT_BYTES;
    static constexpr int OFF_BAR = OFF_DP + 2 * DP_BYTES;
    static constexpr int SMEM_BYTES = OFF_BAR + STAGES * 8 + 1024;   // + alignment slack

    static_assert(G >= 1 && G <= 8 && (G & (G - 1)) == 0, "lanes per channel");
    static_assert(SPT % 2 == 0 && SPT <= 8, "states per lane come in pairs");
    static_assert(R % G == 0 && BOX_T % R == 0 && T % BOX_T == 0, "step grouping");
    static_assert(CH % 8 == 0, "x tiles must be whole 1024-byte swizzle atoms");
    static_assert(STAGE_BYTES % 1024 == 0 && (OFF_BT % 16) == 0, "alignment");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    static_assert(TS == 1 || (TS == 2 && EB == 4 && T == 2 * 2 * R && (G == 4 || G == 8)),
                  "time split: fp32 I/O, two groups per lane, 4 or 8 lanes per channel");
    static_assert(!EXT || TS == 1, "the selective_scan_fn extras run without the time split");
    static_assert(kCkptSteps % R == 0 && T % kCkptSteps == 0 || TS == 2, "checkpoints at group ends");
};

template <typename IO, int NP, int SPT, int WARPS, int TS, bool EXT, bool CK>
__global__ void __launch_bounds__(WARPS * 32, ScanTile<IO, NP, SPT, WARPS, TS, EXT>::MIN_CTAS)
scan_fwd_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_d,
                const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_C,
                const ScanArgs p) {
    using TL = ScanTile<IO, NP, SPT, WARPS, TS, EXT>;
    constexpr int G = TL::G, CPW = TL::CPW, CH = TL::CH, NT = TL::NT, T = TL::T, R = TL::R;
    constexpr int ST = TL::STAGES, NPAIR = TL::NPAIR, EB = TL::EB, BP = TL::BP;

    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (base - raw_addr);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int g = lane % G;
    const int yrow_id = lane / G;                    // (time-lane, channel) row of the read-out buffer
    const int j_t = yrow_id % TS;                    // time-lane: which half of each chunk (TS == 2)
    const int cw = yrow_id / TS;
    const int c = warp * CPW + cw;                   // channel within the CTA
    const int64_t b = blockIdx.x / p.tiles_per_batch;
    const int64_t d0 = (int64_t)(blockIdx.x % p.tiles_per_batch) * CH;
    const int64_t d = d0 + c;
    const bool active = d < p.dim;
    // Lanes that own the carried state, store y and write the final state.
    const bool writer = active && (TS == 1 || j_t == 0);
    const int64_t L = p.seqlen;
    const int N = p.dstate;
    const int64_t nchunks = (L + T - 1) / T;
    const int64_t ncks = (L + kCkptSteps - 1) / kCkptSteps;     // checkpoints per channel
    const bool use_tma = p.vec_ok != 0;
    const uint32_t bar0 = base + TL::OFF_BAR;

    if (tid == 0) {
        for (int s = 0; s < ST; ++s) mbar_init(bar0 + 8 * s, use_tma ? 1u : (uint32_t)NT);
        fence_barrier_init();
    }
    __syncthreads();

    // ---- per-lane constants and state ------------------------------------
    float2 A2p[SPT];        // (A[d,n] log2 e) twice, for two steps at once
    float2 vv[NPAIR], hh[NPAIR];
#pragma unroll
    for (int s = 0; s < SPT; ++s) {
        const int n = g * SPT + s;
        const float a2 = (active && n < N) ? p.A[d * N + n] * kLog2e : 0.0f;
        A2p[s] = f2(a2, a2);
    }
#pragma unroll
    for (int q = 0; q < NPAIR; ++q) {
        float hv[2] = {0.0f, 0.0f}, vw[2] = {0.0f, 0.0f};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int n = g * SPT + 2 * q + e;
            if (writer && n < N) {
                const int64_t si = (b * p.dim + d) * N + n;
                if (p.h0) hv[e] = p.h0[si];
                if (p.v0) vw[e] = p.v0[si];
            }
        }
        hh[q] = f2(hv[0], hv[1]);
        vv[q] = f2(vw[0], vw[1]);
    }
    const float2 beta2 = f2(p.beta, p.beta);
    const float alpha = p.alpha;
    // selective_scan_fn extras
    const float skip_d = (EXT && p.Dskip && active) ? p.Dskip[d] : 0.0f;
    const bool has_skip = EXT && p.Dskip != nullptr;
    const IO* zrow = (EXT && p.z) ? static_cast<const IO*>(p.z) + (b * p.dim + (active ? d : 0)) * p.seqlen
                                  : nullptr;
    constexpr int ZN = EXT ? TL::R / G : 1;      // gate values a lane applies per group

    // ---- staging of one chunk into a stage buffer --------------------------
    auto issue = [&](int64_t k, int s) {
        if (p.stall) return;      // test only: nothing staged, the waits run out
        const int64_t t0 = k * T;
        const uint32_t sb = base + s * TL::STAGE_BYTES;
        const uint32_t bar = bar0 + 8 * s;
        if (use_tma) {
            if (tid == 0) {
                mbar_expect_tx(bar, TL::TX_BYTES);
#pragma unroll
                for (int bx = 0; bx < TL::NBOX; ++bx) {
                    const int tc = (int)(t0 + bx * TL::BOX_T);
                    tma_load_3d(sb + TL::OFF_X + bx * TL::XBOX, &tm_x, bar, tc, (int)d0, (int)b);
                    tma_load_3d(sb + TL::OFF_D + bx * TL::XBOX, &tm_d, bar, tc, (int)d0, (int)b);
                    tma_load_3d(sb + TL::OFF_B + bx * TL::BBOX, &tm_B, bar, tc, 0, (int)b);
                    tma_load_3d(sb + TL::OFF_C + bx * TL::BBOX, &tm_C, bar, tc, 0, (int)b);
                }
            }
            return;
        }
        // Element-wise fill of the same swizzled tiles (rows not 16-byte multiples).
        const IO* xg = static_cast<const IO*>(p.x);
        const IO* dg = static_cast<const IO*>(p.delta);
        const IO* Bg = static_cast<const IO*>(p.B);
        const IO* Cg = static_cast<const IO*>(p.C);
        constexpr int ROWS = 2 * CH + 2 * TL::NPT;
        for (int i = tid; i < ROWS * T; i += NT) {
            const int r = i / T;
            const int tau = i - r * T;
            const int bx = tau / TL::BOX_T;
            const int col = tau - bx * TL::BOX_T;
            const int64_t t = t0 + tau;
            const IO* src = nullptr;
            uint32_t off;
            if (r < 2 * CH) {
                const int cc = r < CH ? r : r - CH;
                off = (r < CH ? TL::OFF_X : TL::OFF_D) + bx * TL::XBOX + sw128(cc, col * EB);
                if (d0 + cc < p.dim && t < L) src = (r < CH ? xg : dg) + ((b * p.dim + d0 + cc) * L + t);
            } else {
                const int rr = r - 2 * CH;
                const int n = rr < TL::NPT ? rr : rr - TL::NPT;
                off = (rr < TL::NPT ? TL::OFF_B : TL::OFF_C) + bx * TL::BBOX + sw128(n, col * EB);
                if (n < N && t < L) src = (rr < TL::NPT ? Bg : Cg) + ((b * N + n) * L + t);
            }
            if constexpr (EB == 4) {
                cp_async_4(smem + s * TL::STAGE_BYTES + off, src ? src : xg, src ? 4 : 0);
            } else {
                *reinterpret_cast<IO*>(smem + s * TL::STAGE_BYTES + off) = src ? *src : IO(0.0f);
            }
        }
        if constexpr (EB == 4) cp_async_mbar_arrive(bar);
        else mbar_arrive(bar);
    };

    // ---- pipeline prologue ---------------------------------------------------
#pragma unroll
    for (int s = 0; s < ST - 1; ++s)
        if (s < nchunks) issue(s, s);

    IO* yrow = static_cast<IO*>(p.y) + (b * p.dim + (active ? d : 0)) * L;
    const bool vec_out = use_tma;

    // The gate z of the outputs a lane stores, read from global memory one chunk
    // ahead into registers (ZC values a chunk): the reads of chunk k + 1 are in
    // flight while chunk k runs, so the gate never waits on DRAM.
    // (tiles with few lanes per channel apply many gates each: they read them in
    // the group before, as the ragged chunk does, rather than hold a chunk's worth)
    constexpr bool ZPRE = EXT && (TL::T / TL::R) * ZN <= 16;
    constexpr int ZC = ZPRE ? (TL::T / TL::R) * ZN : 1;
    float znext[ZC];
    auto load_gates = [&](int64_t kz) {
        if constexpr (ZPRE) {
#pragma unroll
            for (int i = 0; i < ZC; ++i) {
                const int64_t tz = kz * T + (i / ZN) * TL::R + g * ZN + (i % ZN);
                znext[i] = (zrow && active && tz < L) ? load1(zrow + tz) : 0.0f;
            }
        }
    };
    if (nchunks > 0) load_gates(0);

    for (int64_t k = 0; k < nchunks; ++k) {
        const int s = (int)(k % ST);
        const int64_t t0 = k * T;
        const int nval = (int)((L - t0) < T ? (L - t0) : T);
        // Every thread waits; the outcome is made uniform at the barrier below, so
        // that a wait that gave up makes the whole CTA leave together.
        const bool waited = mbar_wait(bar0 + 8 * s, (uint32_t)((k / ST) & 1), &g_scan_dev_err);
        const unsigned char* sbuf = smem + s * TL::STAGE_BYTES;
        float* Bt = reinterpret_cast<float*>(smem + TL::OFF_BT + (int)(k & 1) * TL::BT_BYTES);
        float* Ct = reinterpret_cast<float*>(smem + TL::OFF_BT + (2 + (int)(k & 1)) * TL::BT_BYTES);

        // ---- transpose B, C to [t][n] fp32 in 4x4 blocks (alpha into B) ----
        if (waited) {
            constexpr int NB4 = NP / 4 > 0 ? NP / 4 : 1;
            constexpr int ITEMS = NB4 * (T / 4);
            for (int i = tid; i < 2 * ITEMS; i += NT) {
                const int which = i / ITEMS;
                const int rem = i - which * ITEMS;
                const int n0 = (rem % NB4) * 4;
                const int t4 = (rem / NB4) * 4;
                const int bx = t4 / TL::BOX_T;
                const int col = t4 - bx * TL::BOX_T;
                const unsigned char* tile = sbuf + (which ? TL::OFF_C : TL::OFF_B) + bx * TL::BBOX;
                float m[4][4];   // m[row n][step]
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    if (n0 + r < NP) {
                        const float4 q = load4(reinterpret_cast<const IO*>(tile + sw128(n0 + r, col * EB)));
                        m[r][0] = q.x; m[r][1] = q.y; m[r][2] = q.z; m[r][3] = q.w;
                    } else {
                        m[r][0] = m[r][1] = m[r][2] = m[r][3] = 0.0f;
                    }
                }
                const float sc = which ? 1.0f : alpha;
                float* dst = (which ? Ct : Bt) + t4 * BP + n0;
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
            // delta' = softplus(delta + bias) once per (channel, step) of the chunk,
            // four steps per item, as fp32 in the fp32 box layout.
            if (waited && (p.dbias || p.softplus)) {
                unsigned char* dp = (EB == 4) ? smem + s * TL::STAGE_BYTES + TL::OFF_D
                                              : smem + TL::OFF_DP + (int)(k & 1) * TL::DP_BYTES;
                for (int i = tid; i < CH * (T / 4); i += NT) {
                    const int cc = i / (T / 4);
                    const int t4 = (i - cc * (T / 4)) * 4;
                    const int bxs = t4 / TL::BOX_T;
                    const int cols = t4 - bxs * TL::BOX_T;
                    const float4 q = load4(reinterpret_cast<const IO*>(sbuf + TL::OFF_D + bxs * TL::XBOX +
                                                                       sw128(cc, cols * EB)));
                    const float bv = (p.dbias && d0 + cc < p.dim) ? p.dbias[d0 + cc] : 0.0f;
                    float v[4] = {q.x + bv, q.y + bv, q.z + bv, q.w + bv};
                    if (p.softplus) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) v[e] = softplus_f32(v[e]);
                    }
                    *reinterpret_cast<float4*>(dp + (t4 / 32) * TL::XBOX_F32 + sw128(cc, (t4 % 32) * 4)) =
                        make_float4(v[0], v[1], v[2], v[3]);
                }
            }
        }
        if (!__syncthreads_and(waited)) return;
        // Every thread is past compute(k-1): its stage and B^T/C^T buffers are free.
        if (k + ST - 1 < nchunks) issue(k + ST - 1, (int)((k + ST - 1) % ST));
        float zcur[ZC];
#pragma unroll
        for (int i = 0; i < ZC; ++i) zcur[i] = znext[i];
        if (ZPRE && k + 1 < nchunks) load_gates(k + 1);

        // ---- the recurrence over this chunk, R steps at a time -------------
        const float* Bg = Bt + g * SPT;
        const float* Cg = Ct + g * SPT;

        // Loads, delta*x and exponentials of the R steps of group gi.
        const bool dprime_bf16 = EXT && EB == 2 && (p.dbias || p.softplus);
        const unsigned char* dpb = smem + TL::OFF_DP + (int)(k & 1) * TL::DP_BYTES;
        // (`full`: a full chunk, whose groups are unrolled, takes its gates from the
        // registers read a chunk ahead; the ragged last chunk reads them here)
        auto prep = [&](int gi, float (&u)[R], float (&a)[R][SPT], float (&zg)[ZN], bool full) {
            const int tau0 = gi * R;
            const int bx = tau0 / TL::BOX_T;
            const int col = tau0 - bx * TL::BOX_T;
            const unsigned char* xt = sbuf + TL::OFF_X + bx * TL::XBOX;
            const unsigned char* dtl = sbuf + TL::OFF_D + bx * TL::XBOX;
            float dl[R], xl[R];
#pragma unroll
            for (int j = 0; j < R; j += 4) {
                float4 dq;
                if (dprime_bf16)      // delta' kept as fp32 beside the bf16 tiles
                    dq = *reinterpret_cast<const float4*>(dpb + ((tau0 + j) / 32) * TL::XBOX_F32 +
                                                          sw128(c, ((tau0 + j) % 32) * 4));
                else
                    dq = load4(reinterpret_cast<const IO*>(dtl + sw128(c, (col + j) * EB)));
                const float4 xq = load4(reinterpret_cast<const IO*>(xt + sw128(c, (col + j) * EB)));
                dl[j] = dq.x; dl[j + 1] = dq.y; dl[j + 2] = dq.z; dl[j + 3] = dq.w;
                xl[j] = xq.x; xl[j + 1] = xq.y; xl[j + 2] = xq.z; xl[j + 3] = xq.w;
            }
            if constexpr (EXT) {      // the gate of this lane's outputs
                if (ZPRE && full) {
#pragma unroll
                    for (int e = 0; e < ZN; ++e) zg[e] = zcur[(gi * ZN + e) % ZC];
                } else {
#pragma unroll
                    for (int e = 0; e < ZN; ++e) {
                        const int64_t tz = t0 + tau0 + g * ZN + e;
                        zg[e] = (zrow && active && tz < L) ? load1(zrow + tz) : 0.0f;
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < R; j += 2) {
                const float2 uu = __fmul2_rn(f2(dl[j], dl[j + 1]), f2(xl[j], xl[j + 1]));
                u[j] = uu.x;
                u[j + 1] = uu.y;
            }
#pragma unroll
            for (int sI = 0; sI < SPT; ++sI) {
#pragma unroll
                for (int j = 0; j < R; j += 2) {
                    const float2 r2 = __fmul2_rn(f2(dl[j], dl[j + 1]), A2p[sI]);
                    a[j][sI] = ex2_approx(r2.x);
                    a[j + 1][sI] = ex2_approx(r2.y);
                }
            }
        };

        // ---- add the G partials of each channel; store y --------------------
        auto reduce_store = [&](int tau0, const float (&yk)[R], const float (&zg)[ZN]) {
            constexpr int PER = R / G;      // steps each lane finishes
            float out[PER];
            butterfly_sum<G, R>(yk, out, g);
            const int first = tau0 + g * PER;      // step (within the chunk) of out[0]
            const int cnt = nval - first < PER ? nval - first : PER;
            if constexpr (EXT) {
#pragma unroll
                for (int e = 0; e < PER; ++e) {
                    if (has_skip) {               // + D x, x from the staged tile
                        const int st = first + e;
                        const int bxx = st / TL::BOX_T;
                        out[e] += skip_d * load1(reinterpret_cast<const IO*>(
                                      sbuf + TL::OFF_X + bxx * TL::XBOX + sw128(c, (st - bxx * TL::BOX_T) * EB)));
                    }
                    if (zrow) out[e] *= __fdividef(zg[e], 1.0f + ex2_approx(-zg[e] * kLog2e));   // * silu(z)
                }
            }
            if (writer && cnt > 0) store_steps_n<IO, PER>(yrow + t0 + first, out, cnt, vec_out);
        };
        // The same for the 16 steps of one half chunk (time split); both halves store.
        auto reduce16_store = [&](int tau0, const float (&yk)[16]) {
            constexpr int PER = 16 / G;
            float out[PER];
            butterfly_sum<G, 16>(yk, out, g);
            const int first = tau0 + g * PER;
            const int cnt = nval - first < PER ? nval - first : PER;
            if (active && cnt > 0) store_steps_n<IO, PER>(yrow + t0 + first, out, cnt, vec_out);
        };

        // The R full steps of group gi from the lane's state; per-lane partial y into yk.
        auto group_steps = [&](int gi, const float (&u)[R], const float (&a)[R][SPT], float (&yk)[R]) {
            const int tau0 = gi * R;
#pragma unroll
            for (int j = 0; j < R; ++j) {
                const float* brow = Bg + (tau0 + j) * BP;
                const float* crow = Cg + (tau0 + j) * BP;
                float bq[SPT], cq[SPT];
                if constexpr (SPT >= 4) {
#pragma unroll
                    for (int q = 0; q < SPT; q += 4) {
                        const float4 b4 = *reinterpret_cast<const float4*>(brow + q);
                        const float4 c4 = *reinterpret_cast<const float4*>(crow + q);
                        bq[q] = b4.x; bq[q + 1] = b4.y; bq[q + 2] = b4.z; bq[q + 3] = b4.w;
                        cq[q] = c4.x; cq[q + 1] = c4.y; cq[q + 2] = c4.z; cq[q + 3] = c4.w;
                    }
                } else {
                    const float2 b2 = *reinterpret_cast<const float2*>(brow);
                    const float2 c2 = *reinterpret_cast<const float2*>(crow);
                    bq[0] = b2.x; bq[1] = b2.y;
                    cq[0] = c2.x; cq[1] = c2.y;
                }
                const float2 uu = f2(u[j], u[j]);
                float2 yy = f2(0.0f, 0.0f);
#pragma unroll
                for (int q = 0; q < NPAIR; ++q) {
                    const float2 w = __fmul2_rn(uu, f2(bq[2 * q], bq[2 * q + 1]));
                    vv[q] = __ffma2_rn(beta2, vv[q], w);
                    hh[q] = __ffma2_rn(f2(a[j][2 * q], a[j][2 * q + 1]), hh[q], vv[q]);
                    yy = __ffma2_rn(f2(cq[2 * q], cq[2 * q + 1]), hh[q], yy);
                }
                yk[j] = yy.x + yy.y;
            }
        };
        auto full_steps = [&](int gi, const float (&u)[R], const float (&a)[R][SPT], const float (&zg)[ZN]) {
            float yk[R];
            group_steps(gi, u, a, yk);
            reduce_store(gi * R, yk, zg);
        };

        // The remaining nval < T steps of the sequence, one group at a time.
        // (h, v) after steps 16 i + 15 and after the last step: where the
        // backward restarts its 16-step blocks
        // (CK: a compile-time switch, so the kernels without checkpoints carry
        // no trace of them in their unrolled groups)
        auto save_ckpt = [&](int64_t idx) {
            if (!writer) return;
            float* cp = p.ckpt + ((b * p.dim + d) * ncks + idx) * 2 * N;
#pragma unroll
            for (int q = 0; q < NPAIR; ++q) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int n = g * SPT + 2 * q + e;
                    if (n < N) {
                        cp[n] = e ? hh[q].y : hh[q].x;
                        cp[N + n] = e ? vv[q].y : vv[q].x;
                    }
                }
            }
        };

        auto ragged_chunk = [&]() {
            const int ngroups = (nval + R - 1) / R;
            for (int gi = 0; gi < ngroups; ++gi) {
                const int tau0 = gi * R;
                const int kmax = nval - tau0 < R ? nval - tau0 : R;
                float u[R], a[R][SPT], yk[R], zg[ZN];
                prep(gi, u, a, zg, false);
                if (kmax == R) {
                    group_steps(gi, u, a, yk);
                } else {
#pragma unroll
                    for (int j = 0; j < R; ++j) {       // ragged end of the sequence
                        yk[j] = 0.0f;
                        if (j < kmax) {
                            const float* brow = Bg + (tau0 + j) * BP;
                            const float* crow = Cg + (tau0 + j) * BP;
                            const float2 uu = f2(u[j], u[j]);
                            float2 yy = f2(0.0f, 0.0f);
#pragma unroll
                            for (int q = 0; q < NPAIR; ++q) {
                                const float2 w = __fmul2_rn(uu, f2(brow[2 * q], brow[2 * q + 1]));
                                vv[q] = __ffma2_rn(beta2, vv[q], w);
                                hh[q] = __ffma2_rn(f2(a[j][2 * q], a[j][2 * q + 1]), hh[q], vv[q]);
                                yy = __ffma2_rn(f2(crow[2 * q], crow[2 * q + 1]), hh[q], yy);
                            }
                            yk[j] = yy.x + yy.y;
                        }
                    }
                }
                reduce_store(tau0, yk, zg);
                if constexpr (CK) {
                    const int end = tau0 + kmax;
                    if (end % kCkptSteps == 0 || end == nval) save_ckpt((t0 + end - 1) / kCkptSteps);
                }
            }
        };

        if constexpr (TS == 1) {
            if (nval == T) {
                // Full chunk: groups unrolled, each group's exponentials issued one group ahead.
                constexpr int NG = T / R;
                float uA[R], uB[R], aA[R][SPT], aB[R][SPT], zA[ZN], zB[ZN];
                prep(0, uA, aA, zA, true);
#pragma unroll
                for (int gi = 0; gi < NG; ++gi) {
                    if ((gi & 1) == 0) {
                        if (gi + 1 < NG) prep(gi + 1, uB, aB, zB, true);
                        full_steps(gi, uA, aA, zA);
                    } else {
                        if (gi + 1 < NG) prep(gi + 1, uA, aA, zA, true);
                        full_steps(gi, uB, aB, zB);
                    }
                    if constexpr (CK)
                        if (((gi + 1) * R) % kCkptSteps == 0) save_ckpt((t0 + (gi + 1) * R) / kCkptSteps - 1);
                }
            } else {
                ragged_chunk();
            }
        } else {
            // ---- time split: lane half j_t runs steps [16 j_t, 16 j_t + 16) ----
            // The first half starts from the carried state, the second from zero.
            // The recurrence is linear in its start state (v_in, h_in), so the
            // second half's true state is its zero-start state plus the response
            // to (v_in, h_in) alone:  b_t = beta^(t+1) v_in,  c_t = a_t c_{t-1} + b_t
            // with c_{-1} = h_in, which adds C_t . c_t to y_t and (b, c) at the end
            // to (v, h).  The 2x2 carry [[beta, 0], [beta, a_t]] is thus applied
            // across the two halves with one shuffle each way.
            if (nval == T) {
                constexpr int HALF = T / 2;
                const int gi0 = 2 * j_t;
                float uA[R], uB[R], aA[R][SPT], aB[R][SPT], yk[HALF], zd[ZN];
                prep(gi0, uA, aA, zd, true);
                prep(gi0 + 1, uB, aB, zd, true);
                {
                    float y8[R];
                    group_steps(gi0, uA, aA, y8);
#pragma unroll
                    for (int j = 0; j < R; ++j) yk[j] = y8[j];
                    group_steps(gi0 + 1, uB, aB, y8);
#pragma unroll
                    for (int j = 0; j < R; ++j) yk[R + j] = y8[j];
                }
                float2 bv[NPAIR], cc[NPAIR];
                const float2 zero2 = f2(0.0f, 0.0f);
#pragma unroll
                for (int q = 0; q < NPAIR; ++q) {      // first-half lanes take zeros: exact no-op
                    const float2 vi = shfl_up_f2(vv[q], G);
                    const float2 hi = shfl_up_f2(hh[q], G);
                    bv[q] = j_t ? vi : zero2;
                    cc[q] = j_t ? hi : zero2;
                }
                const float* Ch = Cg + (gi0 * R) * BP;
#pragma unroll
                for (int t = 0; t < HALF; ++t) {
                    const float* crow = Ch + t * BP;
                    float cq[SPT];
                    if constexpr (SPT >= 4) {
#pragma unroll
                        for (int q = 0; q < SPT; q += 4) {
                            const float4 c4 = *reinterpret_cast<const float4*>(crow + q);
                            cq[q] = c4.x; cq[q + 1] = c4.y; cq[q + 2] = c4.z; cq[q + 3] = c4.w;
                        }
                    } else {
                        const float2 c2 = *reinterpret_cast<const float2*>(crow);
                        cq[0] = c2.x; cq[1] = c2.y;
                    }
                    float2 yy = zero2;
#pragma unroll
                    for (int q = 0; q < NPAIR; ++q) {
                        const float a0 = t < R ? aA[t][2 * q] : aB[t - R][2 * q];
                        const float a1 = t < R ? aA[t][2 * q + 1] : aB[t - R][2 * q + 1];
                        bv[q] = __fmul2_rn(beta2, bv[q]);
                        cc[q] = __ffma2_rn(f2(a0, a1), cc[q], bv[q]);
                        yy = __ffma2_rn(f2(cq[2 * q], cq[2 * q + 1]), cc[q], yy);
                    }
                    yk[t] += yy.x + yy.y;
                }
#pragma unroll
                for (int q = 0; q < NPAIR; ++q) {
                    vv[q] = __fadd2_rn(vv[q], bv[q]);
                    hh[q] = __fadd2_rn(hh[q], cc[q]);
                }
                reduce16_store(gi0 * R, yk);
                // The second half's end state is the next chunk's start, in the first half's lanes.
#pragma unroll
                for (int q = 0; q < NPAIR; ++q) {
                    const float2 vn = shfl_down_f2(vv[q], G);
                    const float2 hn = shfl_down_f2(hh[q], G);
                    vv[q] = j_t ? zero2 : vn;
                    hh[q] = j_t ? zero2 : hn;
                }
            } else {
                // Ragged end of the sequence: the second half's lanes take the carried
                // state and repeat the first half's work; only the first half stores.
#pragma unroll
                for (int q = 0; q < NPAIR; ++q) {
                    const float2 vi = shfl_up_f2(vv[q], G);
                    const float2 hi = shfl_up_f2(hh[q], G);
                    if (j_t) { vv[q] = vi; hh[q] = hi; }
                }
                ragged_chunk();
            }
        }
    }

    // ---- final states -------------------------------------------------------
    if (writer) {
#pragma unroll
        for (int q = 0; q < NPAIR; ++q) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int n = g * SPT + 2 * q + e;
                if (n < N) {
                    const int64_t si = (b * p.dim + d) * N + n;
                    if (p.hT) p.hT[si] = e ? hh[q].y : hh[q].x;
                    if (p.vT) p.vT[si] = e ? vv[q].y : vv[q].x;
                }
            }
        }
    }
}

// ------------------------------------------------------------- launch -----
namespace {

template <typename IO, int NP, int SPT, int WARPS, int TS = 1, bool EXT = false, bool CK = false>
cudaError_t launch_variant(const ScanArgs& a0, cudaStream_t stream) {
    using TL = ScanTile<IO, NP, SPT, WARPS, TS, EXT>;
    ScanArgs a = a0;
    a.tiles_per_batch = (int)((a.dim + TL::CH - 1) / TL::CH);
    const int64_t grid = a.batch * a.tiles_per_batch;
    if (grid > 0x7fffffffLL || a.dim > 0x7fffffffLL || a.batch > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    CUtensorMap mx, md, mB, mC;
    memset(&mx, 0, sizeof(mx)); memset(&md, 0, sizeof(md));
    memset(&mB, 0, sizeof(mB)); memset(&mC, 0, sizeof(mC));
    if (a.vec_ok) {
        const bool bf = sizeof(IO) == 2;
        const uint64_t L = (uint64_t)a.seqlen;
        cudaError_t e;
        if ((e = make_map_3d(&mx, a.x, bf, L, a.dim, a.batch, TL::BOX_T, TL::CH)) != cudaSuccess) return e;
        if ((e = make_map_3d(&md, a.delta, bf, L, a.dim, a.batch, TL::BOX_T, TL::CH)) != cudaSuccess) return e;
        if ((e = make_map_3d(&mB, a.B, bf, L, a.dstate, a.batch, TL::BOX_T, TL::NPT)) != cudaSuccess) return e;
        if ((e = make_map_3d(&mC, a.C, bf, L, a.dstate, a.batch, TL::BOX_T, TL::NPT)) != cudaSuccess) return e;
    }
    auto kern = scan_fwd_kernel<IO, NP, SPT, WARPS, TS, EXT, CK>;
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
    kern<<<(unsigned)grid, TL::NT, TL::SMEM_BYTES, stream>>>(mx, md, mB, mC, a);
    return cudaGetLastError();
}

// Variants that are built: (states per lane, warps per CTA) for 16 padded states,
// and the natural choices for smaller state counts.
template <typename IO, bool EXT>
cudaError_t launch_ckpt(const ScanArgs& a, int np, int warps, cudaStream_t s) {
    switch (np) {
        case 16:
            if (warps == 2) return launch_variant<IO, 16, 2, 2, 1, EXT, true>(a, s);
            return launch_variant<IO, 16, 2, 4, 1, EXT, true>(a, s);
        case 8: return launch_variant<IO, 8, 2, 2, 1, EXT, true>(a, s);
        case 4: return launch_variant<IO, 4, 2, 2, 1, EXT, true>(a, s);
        case 2: return launch_variant<IO, 2, 2, 1, 1, EXT, true>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

template <typename IO>
cudaError_t launch_io(const ScanArgs& a, int np, int spt, int warps, int ts, cudaStream_t s) {
    if (a.ckpt) {
        // checkpoints: the automatic tiles (two states per lane, one lane along time)
        const int w = (spt == 2 && warps == 2) ? 2 : 4;
        return a.ext ? launch_ckpt<IO, true>(a, np, w, s) : launch_ckpt<IO, false>(a, np, w, s);
    }
    if (a.ext) {
        // selective_scan_fn extras: built for the automatic tiles; a forced
        // tile outside them falls back to the automatic one.
        switch (np) {
            case 16:
                if (spt == 2 && warps == 2) return launch_variant<IO, 16, 2, 2, 1, true>(a, s);
                return launch_variant<IO, 16, 2, 4, 1, true>(a, s);
            case 8: return launch_variant<IO, 8, 2, 2, 1, true>(a, s);
            case 4: return launch_variant<IO, 4, 2, 2, 1, true>(a, s);
            case 2: return launch_variant<IO, 2, 2, 1, 1, true>(a, s);
            default: return cudaErrorInvalidValue;
        }
    }
    if (ts == 2) {
        // Time split: fp32 I/O and 16 padded states only.
        if constexpr (sizeof(IO) == 4) {
            if (np == 16) {
                if (spt == 4 && warps == 2) return launch_variant<IO, 16, 4, 2, 2>(a, s);
                if (spt == 4 && warps == 4) return launch_variant<IO, 16, 4, 4, 2>(a, s);
                if (spt == 2 && warps == 4) return launch_variant<IO, 16, 2, 4, 2>(a, s);
                if (spt == 2 && warps == 8) return launch_variant<IO, 16, 2, 8, 2>(a, s);
            }
        }
        return cudaErrorInvalidValue;
    }
    switch (np) {
        case 16:
            if (spt == 2 && warps == 2) return launch_variant<IO, 16, 2, 2>(a, s);
            if (spt == 2 && warps == 4) return launch_variant<IO, 16, 2, 4>(a, s);
            if (spt == 2 && warps == 8) return launch_variant<IO, 16, 2, 8>(a, s);
            if (spt == 4 && warps == 1) return launch_variant<IO, 16, 4, 1>(a, s);
            if (spt == 4 && warps == 2) return launch_variant<IO, 16, 4, 2>(a, s);
            if (spt == 4 && warps == 4) return launch_variant<IO, 16, 4, 4>(a, s);
            if (spt == 8 && warps == 1) return launch_variant<IO, 16, 8, 1>(a, s);
            if (spt == 8 && warps == 2) return launch_variant<IO, 16, 8, 2>(a, s);
            break;
        case 8:
            if (spt == 2) return launch_variant<IO, 8, 2, 2>(a, s);
            return launch_variant<IO, 8, 4, 2>(a, s);
        case 4:
            return launch_variant<IO, 4, 2, 2>(a, s);
        case 2:
            return launch_variant<IO, 2, 2, 1>(a, s);
        default:
            break;
    }
    return cudaErrorInvalidValue;
}

}  // namespace

bool scan_tile_supported(int spt, int warps, int time_lanes) {
    if (time_lanes == 2)
        return (spt == 4 && (warps == 2 || warps == 4)) || (spt == 2 && (warps == 4 || warps == 8));
    if (time_lanes != 1) return false;
    return (spt == 2 && (warps == 2 || warps == 4 || warps == 8)) ||
           (spt == 4 && (warps == 1 || warps == 2 || warps == 4)) ||
           (spt == 8 && (warps == 1 || warps == 2));
}

ScanTileChoice choose_scan_tile(int64_t batch, int64_t dim, int64_t dstate, int io,
                                int forced_spt, int forced_warps, int forced_ts) {
    // The choice depends on (batch * dim, dstate, io) only, never on L, so calls
    // that split one sequence use the same variant.  Fewer states per lane
    // give more warps (needed when there are few channels); more states per
    // lane need fewer instructions per update.
    ScanTileChoice t;
    t.np = dstate <= 2 ? 2 : dstate <= 4 ? 4 : dstate <= 8 ? 8 : 16;
    t.ts = 1;
    // Two states per lane (8 lanes per channel) keep about 2.5 warps per
    // scheduler on the medium and bf16 workloads; four-warp CTAs share each
    // B/C transpose over 16 channels.
    const int64_t channels = batch * dim;
    t.spt = 2;
    t.warps = channels >= 2048 ? 4 : 2;
    if (t.np == 16 && forced_spt) {
        t.spt = forced_spt;
        t.warps = forced_warps;
        t.ts = (forced_ts == 2 && io == 0) ? 2 : 1;
        if (t.ts == 1 && !scan_tile_supported(t.spt, t.warps, 1)) {
            t.spt = 4;
            t.warps = 2;
        }
    }
    if (t.np == 8 && forced_spt) t.spt = forced_spt == 8 ? 4 : forced_spt;
    if (t.np == 8 && t.spt > 4) t.spt = 4;
    return t;
}

cudaError_t launch_scan_fwd(const ScanArgs& a, const ScanTileChoice& t, int io, cudaStream_t s) {
    if (io == 0) return launch_io<float>(a, t.np, t.spt, t.warps, t.ts, s);
    return launch_io<bf16>(a, t.np, t.spt, t.warps, t.ts, s);
}

unsigned int scan_read_and_clear_device_error() {
    unsigned int v = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_scan_dev_err, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_scan_dev_err, &z, sizeof(z));
    return v;
}

}  // namespace mmscan
