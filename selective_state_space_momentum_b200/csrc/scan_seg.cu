// scan_seg.cu -- sm_100a Momentum Mamba forward scan with the sequence cut
// into segments that run on the CTAs of a thread-block cluster.
//
// What it computes ("Momentum Mamba: Enhanced State Space Models with
// Momentum", "Momentum Mamba Recurrence" and "Discretization Note"), per
// batch row b, channel d, state n:
//     v_t = beta v_{t-1} + alpha delta_t B_t[n] x_t
//     h_t = exp(delta_t A[d,n]) h_{t-1} + v_t
//     y_t = sum_n C_t[n] h_t[n]
//
// Why segments.  A sequence with few channels (one row of 2048 channels, say)
// gives too few independent (channel, state) lanes to keep 148 SMs busy when
// each lane walks the whole sequence.  The recurrence is affine in its start
// state, so the sequence is cut into segments of S steps (S a power of two,
// fixed for a given (batch * dim, dstate, io), never derived from L) that run
// side by side, each from a zero state, and are joined afterwards; this is the
// "Forward Pass: Two-Stage Parallel Scan" of the same page (chunk scans, then
// a running prefix of the chunk carries) with the chunk carry kept as a 2x2
// affine map per lane:
//   * Main pass (one CTA per segment).  From v = h = 0 the CTA runs the
//     segment, stores its read-out y0_t, and keeps, per lane, the zero-start
//     end state (zv, zh), the response of h at the end to a unit velocity at
//     the start, Q = sum_j beta^(j+1) prod_{s>j} a_s (one extra FMA per
//     update: q_t = a_t q_{t-1} + beta^(t+1)), and P = prod_s a_s, formed as
//     2^(A log2e * sum_s delta_s).  The segment maps a start state (v, h) to
//         v' = beta^S v + zv,   h' = P h + Q v + zh.
//   * Carry fold.  The CTAs of a cluster hold consecutive segments of the
//     same channels.  After a cluster barrier each CTA reads the maps of the
//     segments before its own from the other CTAs' shared memory
//     (distributed shared memory, no global scratch) and folds them in
//     segment order onto the concrete carry, starting from (h0, v0).  Every
//     CTA folds the same maps in the same order, so the carries -- and hT, vT,
//     which are the carry after the last segment -- do not depend on how the
//     cluster or the call is cut: two calls split at a multiple of S give hT,
//     vT bit-identical to one call.
//   * Correction.  The true state inside segment k is the zero-start state
//     plus the response to the carry-in (v_in, h_in):  r_v <- beta r_v,
//     r_h <- a_t r_h + r_v, added to y as C_t . r_h.  The response decays; it
//     is run until the bound |r_h| + beta/(1-beta) |r_v| -- which caps every
//     later |r_h| while every a_t <= 1 (A <= 0 and delta >= 0 over the
//     segment, checked) -- falls below 2^-25 of its start value for every lane
//     of the CTA, or to the segment's end.  The y it leaves out is below fp32
//     rounding of the state.
//   * Sequences longer than cluster-size * S: the cluster walks rounds of
//     consecutive segments, each round folding onto the previous one's carry.
//
// Lanes.  One warp owns 16 channels of one batch row: lane = 4 p + g holds
// channels 2p, 2p+1 and states 4g .. 4g+3 (v, h and q in fp32 registers), so
// each B_t / C_t value read from shared memory serves two channels and each
// delta_t / x_t value four states.  The four lanes of a channel pair add
// their read-outs with a register butterfly and store whole 32-byte pieces
// of y.  Staging: one thread issues TMA tile loads (no multicast) of x, delta
// (box 128 bytes of steps x 16 channels) and B, C (x 16 states) into 128-byte
// swizzled tiles; B, C are then transposed to [t][n] fp32 (alpha folded into
// B) so that a lane reads its four states of a step with one vector load.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "mm_common.cuh"
#include "mm_internal.h"
#include "mm_tma_host.h"

namespace mmscan {

// Device error word of this file's kernel (bounded waits that gave up).
static __device__ unsigned int g_seg_dev_err = 0;

// 2^-25: the correction stops once every lane's response bound fell by this factor.
constexpr float kCorrTol = 2.98023223876953125e-8f;

template <typename IO, int W, int ST>
struct SegTile {
    static constexpr int NP = 16;                // states, padded
    static constexpr int G = 4;                  // lanes per channel pair (4 states each)
    static constexpr int CPW = 16;               // channels per warp
    static constexpr int CH = W * CPW;           // channels per CTA
    static constexpr int NT = W * 32;
    static constexpr int EB = IOTraits<IO>::kBytes;
    static constexpr int T = 128 / EB;           // steps per chunk: one 128-byte swizzled row
    static constexpr int XBOX = CH * 128;        // one x (or delta) tile
    static constexpr int BBOX = NP * 128;        // one B (or C) tile
    static constexpr int OFF_X = 0, OFF_D = XBOX, OFF_B = 2 * XBOX, OFF_C = 2 * XBOX + BBOX;
    static constexpr int STAGE_BYTES = 2 * XBOX + 2 * BBOX;
    static constexpr int MAIN_TX = STAGE_BYTES;  // main pass: x, delta, B, C
    static constexpr int CORR_TX = XBOX + BBOX;  // correction: delta, C
    static constexpr int BT_BYTES = T * NP * 4;  // one transposed [t][n] fp32 matrix
    static constexpr int OFF_BT = ST * STAGE_BYTES;  // B^T and C^T interleaved, [t][32] fp32
    // The segment maps (8 float4 per thread) are published in the B^T/C^T area.
    static constexpr int AGG_BYTES = NT * 8 * 16;
    // The concrete carry (v, h) of each lane's 8 states between folds.
    static constexpr int OFF_CARRY = OFF_BT + 2 * BT_BYTES;
    static constexpr int CARRY_BYTES = NT * 16 * 4;
    // Scaled form: alpha beta^-(tau+1) and beta^(tau+1) for the steps tau of a chunk.
    static constexpr int OFF_TAB = OFF_CARRY + CARRY_BYTES;
    static constexpr int TAB_BYTES = 2 * T * 4;
    static constexpr int OFF_BAR = OFF_TAB + TAB_BYTES;
    static constexpr int SMEM_BYTES = OFF_BAR + ST * 8 + 1024;    // + alignment slack
    static_assert(AGG_BYTES <= 2 * BT_BYTES, "segment maps fit the transposed area");
    static_assert(STAGE_BYTES % 1024 == 0, "tiles stay 1024-byte aligned");
    static_assert(T % 8 == 0, "8-step groups");
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t dsmem_map(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ float dsmem_ld1(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ float4 dsmem_ld4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr) : "memory");
    return v;
}

// beta^n by binary powering: the same value wherever a segment's length is n.
__device__ __forceinline__ float pow_steps(float beta, int64_t n) {
    float r = 1.0f, b = beta;
    while (n > 0) {
        if (n & 1) r *= b;
        b *= b;
        n >>= 1;
    }
    return r;
}

// The sequence split over several calls (ranks), in two launches around an
// exchange of segment maps:
//   MODE 1: the main pass of this call's segments only; y gets the zero-start
//     read-out and each segment's map goes to `maps` (record k for the call's
//     segment k) instead of being folded;
//   MODE 2: with the maps of every segment of the whole sequence (all calls'
//     records in segment order), fold segments 0 .. K-1 onto (h0, v0) for this
//     call's segment K (global index seg_first + k), add the response to y,
//     and write hT, vT as the fold of all nseg_total segments.
// A record holds, per (batch row, channel tile) cluster, the 8 float4 maps of
// each of the NT lanes and one float4 whose x is 1 when the segment's delta
// had no negative value; MODE 0 is the fused kernel above.
struct SegSplit {
    float4* maps;             // MODE 1: this call's records; MODE 2: every segment's records (read only)
    int64_t seg_first;        // global index of this call's first segment
    int64_t nseg_total;       // MODE 2: segments of the whole sequence
    int64_t L_total;          // MODE 2: steps of the whole sequence
    // MODE 1 with ndest > 0: each record goes, at its global index, straight into
    // every rank's buffer of the whole sequence's records (device pointers, peer
    // memory over NVLink included) instead of into `maps`
    float4* const* dests;
    int ndest;
};

// Scaled form (SC, used for beta >= 1/2).  Within a chunk of T steps the
// states are carried as v~ = v / beta^(tau+1), h~ = h / beta^(tau+1) (tau the
// step within the chunk), which turns the two recurrences into
//     v~_tau = v~_{tau-1} + u_tau B~_tau,       B~_tau = alpha beta^-(tau+1) B_tau
//     h~_tau = a~_tau h~_{tau-1} + v~_tau,      a~_tau = 2^(delta A log2 e - log2 beta)
//     y_tau  = sum_n C~_tau h~_tau,             C~_tau = beta^(tau+1) C_tau
// with B~ and C~ formed once per chunk by the transpose: one FMA per state
// for the velocity instead of a multiply and an FMA.  At the end of the chunk
// the states are multiplied back by beta^T.  The factors stay within 2^+-32
// (2^+-64 for bf16 chunks of 64 steps) for beta >= 1/2.
template <typename IO, int W, int ST, bool SC, int MODE>
__global__ void __launch_bounds__(W * 32)
scan_seg_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_d,
                const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_C,
                const ScanArgs p, const int64_t seg_len, const int csize, const SegSplit sp) {
    using TL = SegTile<IO, W, ST>;
    constexpr int NT = TL::NT, T = TL::T, CH = TL::CH, EB = TL::EB, G = TL::G;

    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (base - raw_addr);
    float* BCt = reinterpret_cast<float*>(smem + TL::OFF_BT);     // [t][32]: B^T | C^T, swizzled
    float4* agg = reinterpret_cast<float4*>(smem + TL::OFF_BT);
    float* tab_ib = reinterpret_cast<float*>(smem + TL::OFF_TAB);  // alpha beta^-(tau+1)
    float* tab_cb = tab_ib + T;                                      // beta^(tau+1)
    const uint32_t agg_addr = base + TL::OFF_BT;
    const uint32_t bar0 = base + TL::OFF_BAR;

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int g = lane & (G - 1);                 // state group: states 4g .. 4g+3
    const int pr = lane >> 2;                     // channel pair within the warp
    // segment within the round (the split launches run without clusters: the
    // same mapping from the block index)
    const int rank = MODE == 0 ? (int)cluster_ctarank() : (int)(blockIdx.x % (unsigned)csize);
    const int64_t cl = blockIdx.x / csize;        // (batch row, channel tile)
    const int64_t b = cl / p.tiles_per_batch;
    const int64_t d0 = (cl % p.tiles_per_batch) * CH;
    const int cc0 = warp * TL::CPW + 2 * pr;      // first channel of the pair, within the CTA
    const int64_t L = p.seqlen;
    const int N = p.dstate;
    const float beta = p.beta;
    const int64_t nseg = (L + seg_len - 1) / seg_len;
    const int64_t rounds = (nseg + csize - 1) / csize;
    // records of the split launches: (segment, cluster) -> 8 * NT + 1 float4
    const int64_t ncl = (int64_t)gridDim.x / csize;
    constexpr int REC = 8 * NT + 1;

    if (tid == 0) {
        for (int s = 0; s < ST; ++s) mbar_init(bar0 + 8 * s, 1u);
        fence_barrier_init();
    }
    if constexpr (SC) {
        for (int t = tid; t < T; t += NT) {
            const float cb = pow_steps(beta, t + 1);
            tab_cb[t] = cb;
            tab_ib[t] = __fdiv_rn(p.alpha, cb);
        }
    }
    __syncthreads();

    // ---- per-lane constants ---------------------------------------------------
    // The lane's two channels, in an order of its own: lanes 4p+2, 4p+3 take
    // the pair's channels the other way round, so that the first step of the
    // read-out butterfly (lanes g and g^2) exchanges the same register set on
    // every lane and needs no selects.
    bool act[2];
    int64_t dch[2];
    int lch[2];                   // channel within the CTA
    uint32_t dxo[2];              // its row in a swizzled x / delta tile: row * 128 + (row & 7) * 16
    float Al[2][4];               // A[d, 4g + e] log2 e
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        lch[c] = cc0 + (c ^ (g >> 1));
        dxo[c] = (uint32_t)lch[c] * 128u + (((uint32_t)lch[c] & 7u) << 4);
        dch[c] = d0 + lch[c];
        act[c] = dch[c] < p.dim;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int n = 4 * g + e;
            Al[c][e] = (act[c] && n < N) ? p.A[dch[c] * N + n] * kLog2e : 0.0f;
        }
    }
    bool a_nonpos = true;
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int e = 0; e < 4; ++e) a_nonpos = a_nonpos && (Al[c][e] <= 0.0f);
    a_nonpos = __syncthreads_and(a_nonpos) != 0;
    // -log2(beta), added to every exponent of the scaled form
    const float nl2b = SC ? -log2f(beta) : 0.0f;

    // The concrete carry entering the current round, per lane (c, e): starts at
    // (h0, v0); kept in shared memory between folds ([c][e][v/h][thread]).
    float* carry_s = reinterpret_cast<float*>(smem + TL::OFF_CARRY);
    auto carry_at = [&](int c, int e, int which) -> float& { return carry_s[((c * 4 + e) * 2 + which) * NT + tid]; };
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int n = 4 * g + e;
            float v = 0.0f, h = 0.0f;
            if (act[c] && n < N) {
                const int64_t si = (b * p.dim + dch[c]) * N + n;
                if (p.h0) h = p.h0[si];
                if (p.v0) v = p.v0[si];
            }
            carry_at(c, e, 0) = v;
            carry_at(c, e, 1) = h;
        }

    // ---- TMA staging --------------------------------------------------------------
    // Chunks are consumed in the order they are issued; `issued` / `consumed`
    // count them over the whole kernel and give each its stage and phase.
    int64_t issued = 0, consumed = 0;
    bool dead = false;            // a bounded wait gave up: skip the work, keep the barriers
    auto issue = [&](int64_t t0, bool main_pass) {
        const int s = (int)(issued % ST);
        if (tid == 0 && !p.stall) {   // (stall: test only, nothing staged, the waits run out)
            const uint32_t sb = base + s * TL::STAGE_BYTES;
            const uint32_t bar = bar0 + 8 * s;
            mbar_expect_tx(bar, main_pass ? TL::MAIN_TX : TL::CORR_TX);
            const int tc = (int)t0;
            tma_load_3d(sb + TL::OFF_D, &tm_d, bar, tc, (int)d0, (int)b);
            tma_load_3d(sb + TL::OFF_C, &tm_C, bar, tc, 0, (int)b);
            if (main_pass) {
                tma_load_3d(sb + TL::OFF_X, &tm_x, bar, tc, (int)d0, (int)b);
                tma_load_3d(sb + TL::OFF_B, &tm_B, bar, tc, 0, (int)b);
            }
        }
        ++issued;
    };
    // Wait for the oldest issued chunk; the outcome is made uniform over the CTA.
    auto wait_next = [&]() -> const unsigned char* {
        const int s = (int)(consumed % ST);
        const uint32_t par = (uint32_t)((consumed / ST) & 1);
        bool ok = mbar_wait(bar0 + 8 * s, par, &g_seg_dev_err);
        ok = __syncthreads_and(ok) != 0;
        ++consumed;
        if (!ok) dead = true;
        return smem + s * TL::STAGE_BYTES;
    };
    // Drain chunks issued but not consumed (the correction may stop early).
    auto drain = [&]() {
        while (!dead && consumed < issued) (void)wait_next();
    };

    // B, C of a staged chunk into one [t][32] fp32 area: row t holds B_t[0..15]
    // in 16-byte chunks 0-3 and C_t[0..15] in chunks 4-7, chunk c stored at
    // position c ^ ((t >> 2) & 7); B carries alpha (and beta^-(tau+1) in the
    // scaled form), C beta^(tau+1) in the scaled form.  An item moves a 4 x 4
    // block (4 states, 4 steps); the 8 lanes of a quarter warp take 8
    // consecutive 4-step blocks of one (matrix, state block), so that both the
    // swizzled tile reads and the [t] row writes hit 8 distinct bank groups.
    // `withB` false: C only (the correction pass).
    auto transpose = [&](const unsigned char* sbuf, bool withB) {
        const int items = (withB ? 8 : 4) * (T / 4);
        for (int i = tid; i < items; i += NT) {
            const int combo = withB ? ((i >> 3) & 7) : 4 + ((i >> 3) & 3);   // matrix * 4 + state block
            const int tb = (i & 7) | ((withB ? (i >> 6) : (i >> 5)) << 3);    // 4-step block
            const int which = combo >> 2;                                      // 0 = B, 1 = C
            const int n0 = (combo & 3) * 4;
            const int t4 = tb * 4;
            const unsigned char* tile = sbuf + (which ? TL::OFF_C : TL::OFF_B);
            float m[4][4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float4 q = load4(reinterpret_cast<const IO*>(tile + sw128(n0 + r, t4 * EB)));
                m[r][0] = q.x; m[r][1] = q.y; m[r][2] = q.z; m[r][3] = q.w;
            }
            float sc[4];
            if constexpr (SC) {
                const float4 f = *reinterpret_cast<const float4*>((which ? tab_cb : tab_ib) + t4);
                sc[0] = f.x; sc[1] = f.y; sc[2] = f.z; sc[3] = f.w;
            } else {
                sc[0] = sc[1] = sc[2] = sc[3] = which ? 1.0f : p.alpha;
            }
            float* dst = BCt + t4 * 32 + ((combo ^ (tb & 7)) * 4);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                *reinterpret_cast<float4*>(dst + j * 32) =
                    make_float4(m[0][j] * sc[j], m[1][j] * sc[j], m[2][j] * sc[j], m[3][j] * sc[j]);
        }
    };

    // Sum and sign bits of delta per channel: thread pair (2 c, 2 c + 1) of a
    // warp takes channel c of the warp's 16, each half of the chunk's steps.
    float dpart = 0.0f;            // this thread's sum over the current segment
    uint32_t dbits = 0;            // OR of the bit patterns it saw (sign bit: some delta < 0)
    auto delta_sums = [&](const unsigned char* sbuf) {
        const int ch = tid >> 1;
        const int h0s = (tid & 1) * (T / 2);
        float s2 = 0.0f;
#pragma unroll
        for (int k = 0; k < T / 2; k += 4) {
            const float4 q = load4(reinterpret_cast<const IO*>(sbuf + TL::OFF_D + sw128(ch, (h0s + k) * EB)));
            s2 += (q.x + q.y) + (q.z + q.w);
            dbits |= __float_as_uint(q.x) | __float_as_uint(q.y) | __float_as_uint(q.z) | __float_as_uint(q.w);
        }
        dpart += s2;               // steps past the end of the sequence are zero-filled by TMA
    };

    // delta, x of the two channels for 4 steps from a staged tile.
    // (the 128-byte swizzle puts 16-byte chunk k of row r at chunk k ^ (r & 7):
    // with the row's own bits precomputed in dxo, one XOR finds any chunk)
    auto load_dx = [&](const unsigned char* sbuf, int off, int tau, float (&v)[2][4]) {
        const uint32_t kb = (uint32_t)(tau * EB);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const float4 q = load4(reinterpret_cast<const IO*>(sbuf + off + ((dxo[c] ^ (kb & ~15u)) + (kb & 15u))));
            v[c][0] = q.x; v[c][1] = q.y; v[c][2] = q.z; v[c][3] = q.w;
        }
    };

    // The lane's output after the butterfly: its first channel, steps 4 (g & 1) .. + 3 of a group.
    const bool oact = act[0];
    const int64_t odch = dch[0];
    IO* const orow = static_cast<IO*>(p.y) + (b * p.dim + (oact ? odch : 0)) * L;
    const int ostep = (g & 1) * 4;

    const float2 beta2 = f2(beta, beta);
    const float kappa = beta / (1.0f - beta);

    // Four steps of the two channels: the input delta * x (main pass) and the
    // exponentials of the four states (a, or a / beta in the scaled form).
    struct Quad {
        float u[2][4];
        float a[2][4][4];          // [channel][state][step]
    };
    // Main pass state of the segment (zero start).
    float2 vv[2][2], hh[2][2], qq[2][2];
    float2 bp2;                   // forcing of q: beta^(t+1) (plain form) or beta^(chunk start) (scaled form)

    auto prep_load = [&](const unsigned char* sbuf, int tau, float (&dl)[2][4], Quad& Q, bool main_pass) {
        load_dx(sbuf, TL::OFF_D, tau, dl);
        if (main_pass) {
            float xl[2][4];
            load_dx(sbuf, TL::OFF_X, tau, xl);
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int j2 = 0; j2 < 4; j2 += 2) {
                    const float2 uu = __fmul2_rn(f2(dl[c][j2], dl[c][j2 + 1]), f2(xl[c][j2], xl[c][j2 + 1]));
                    Q.u[c][j2] = uu.x;
                    Q.u[c][j2 + 1] = uu.y;
                }
        }
    };
    // Eight of a group's exponentials: channel c, steps 2 jp and 2 jp + 1.
    auto prep_exp = [&](const float (&dl)[2][4], Quad& Q, int c, int jp) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 dd = f2(dl[c][2 * jp], dl[c][2 * jp + 1]);
            const float2 ex = SC ? __ffma2_rn(dd, f2(Al[c][e], Al[c][e]), f2(nl2b, nl2b))
                                 : __fmul2_rn(dd, f2(Al[c][e], Al[c][e]));
            Q.a[c][e][2 * jp] = ex2_approx(ex.x);
            Q.a[c][e][2 * jp + 1] = ex2_approx(ex.y);
        }
    };

    // The four steps of Q from chunk step tau; partial read-outs into yk[c][j0 + j].
    // With `nxt`, step j also forms eight exponentials of the next group, so that
    // the MUFU work is spread between the FMAs instead of issued in bursts.
    // `ragged`: steps at or past nval leave the state alone (the last chunk).
    auto main_steps = [&](const Quad& Q, int tau, int j0, float (&yk)[2][8], bool ragged, int nval,
                          const float (&dln)[2][4], Quad& Qn, bool nxt) {
        const int sw = (tau >> 2) & 7;                 // row swizzle of the 4 steps
        const int bo = (g ^ sw) * 4, co = ((4 + g) ^ sw) * 4;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (nxt) prep_exp(dln, Qn, j & 1, j >> 1);
            const int step = tau + j;
            const bool valid = !ragged || step < nval;
            const float4 b4 = *reinterpret_cast<const float4*>(BCt + step * 32 + bo);
            const float4 c4 = *reinterpret_cast<const float4*>(BCt + step * 32 + co);
            const float2 bq[2] = {f2(b4.x, b4.y), f2(b4.z, b4.w)};
            const float2 cq[2] = {f2(c4.x, c4.y), f2(c4.z, c4.w)};
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const float2 uu = f2(Q.u[c][j], Q.u[c][j]);
                float2 yy;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const float2 aa = f2(Q.a[c][2 * q][j], Q.a[c][2 * q + 1][j]);
                    const float2 vn = SC ? __ffma2_rn(uu, bq[q], vv[c][q])
                                         : __ffma2_rn(beta2, vv[c][q], __fmul2_rn(uu, bq[q]));
                    const float2 hn = __ffma2_rn(aa, hh[c][q], vn);
                    const float2 qn = __ffma2_rn(aa, qq[c][q], bp2);
                    if (valid) { vv[c][q] = vn; hh[c][q] = hn; qq[c][q] = qn; }
                    yy = q == 0 ? __fmul2_rn(cq[0], hh[c][0]) : __ffma2_rn(cq[1], hh[c][1], yy);
                }
                yk[c][j0 + j] = yy.x + yy.y;
            }
            if (!SC && valid) bp2 = __fmul2_rn(bp2, beta2);
        }
    };

    // Add the four lanes' partials of an 8-step group and store y (main pass),
    // or add them to the y stored by the main pass, read ahead into yold.
    auto flush = [&](const float (&yk)[2][8], int64_t t0, int first8, int nval, bool add, const float (&yold)[4]) {
        // lanes g, g^2 hold the pair's channels in opposite order: keep the first,
        // add the partner's second (the same channel); then lanes g, g^1 split the
        // eight steps in halves
        float s1[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) s1[i] = yk[0][i] + __shfl_xor_sync(0xffffffffu, yk[1][i], 2);
        float out[4];
        const bool up = (g & 1) != 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float keep = up ? s1[4 + i] : s1[i];
            const float send = up ? s1[i] : s1[4 + i];
            out[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
        }
        const int first = first8 + ostep;
        const int cnt = nval - first < 4 ? nval - first : 4;
        if (!oact || cnt <= 0) return;
        if (add) {
#pragma unroll
            for (int e = 0; e < 4; ++e) out[e] += yold[e];
        }
        store_steps_n<IO, 4>(orow + t0 + first, out, cnt, true);
    };
    // The main pass's y of the lane's four outputs of the 8-step group at first8.
    auto load_yold = [&](int64_t t0, int first8, int nval, float (&yold)[4]) {
        const int first = first8 + ostep;
        const int cnt = nval - first < 4 ? nval - first : 4;
        yold[0] = yold[1] = yold[2] = yold[3] = 0.0f;
        if (!oact || cnt <= 0) return;
        const IO* yp = orow + t0 + first;
        if (cnt == 4) {
            const float4 q4 = load4(yp);
            yold[0] = q4.x; yold[1] = q4.y; yold[2] = q4.z; yold[3] = q4.w;
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (e < cnt) yold[e] = load1(yp + e);
        }
    };

    // Correction state: the response to the carry-in (in the scaled form the
    // velocity part v~ stays constant within a chunk).
    float2 rvv[2][2], rhh[2][2];
    auto corr_steps = [&](const Quad& Q, int tau, int j0, float (&yk)[2][8], bool ragged, int nval,
                          const float (&dln)[2][4], Quad& Qn, bool nxt) {
        const int sw = (tau >> 2) & 7;
        const int co = ((4 + g) ^ sw) * 4;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (nxt) prep_exp(dln, Qn, j & 1, j >> 1);
            const int step = tau + j;
            const bool valid = !ragged || step < nval;
            const float4 c4 = *reinterpret_cast<const float4*>(BCt + step * 32 + co);
            const float2 cq[2] = {f2(c4.x, c4.y), f2(c4.z, c4.w)};
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float2 yy;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const float2 aa = f2(Q.a[c][2 * q][j], Q.a[c][2 * q + 1][j]);
                    const float2 vn = SC ? rvv[c][q] : __fmul2_rn(beta2, rvv[c][q]);
                    const float2 hn = __ffma2_rn(aa, rhh[c][q], vn);
                    if (valid) { rvv[c][q] = vn; rhh[c][q] = hn; }
                    yy = q == 0 ? __fmul2_rn(cq[0], rhh[c][0]) : __ffma2_rn(cq[1], rhh[c][1], yy);
                }
                yk[c][j0 + j] = yy.x + yy.y;
            }
        }
    };
    auto steps = [&](bool main_pass, const Quad& Q, int tau, int j0, float (&yk)[2][8], bool ragged, int nval,
                     const float (&dln)[2][4], Quad& Qn, bool nxt) {
        if (main_pass) main_steps(Q, tau, j0, yk, ragged, nval, dln, Qn, nxt);
        else corr_steps(Q, tau, j0, yk, ragged, nval, dln, Qn, nxt);
    };

    // One staged chunk.  Full chunks run unpredicated, each group's loads and
    // exponentials formed during the group before; the last chunk of the
    // sequence is ragged.  The correction reads the main pass's y one group ahead.
    auto run_chunk = [&](const unsigned char* sbuf, int64_t t0, int nval, bool main_pass) {
        float yk[2][8] = {};
        float dl[2][4];
        float yold[4] = {0.0f, 0.0f, 0.0f, 0.0f}, ynext[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (nval == T) {
            Quad Q0, Q1;
            prep_load(sbuf, 0, dl, Q0, main_pass);
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int jp = 0; jp < 2; ++jp) prep_exp(dl, Q0, c, jp);
            if (!main_pass) load_yold(t0, 0, T, yold);
#pragma unroll 1
            for (int g8 = 0; g8 < T; g8 += 8) {
                const bool more = g8 + 8 < T;
                if (!main_pass && more) load_yold(t0, g8 + 8, T, ynext);
                prep_load(sbuf, g8 + 4, dl, Q1, main_pass);
                steps(main_pass, Q0, g8, 0, yk, false, T, dl, Q1, true);
                if (more) {
                    prep_load(sbuf, g8 + 8, dl, Q0, main_pass);
                    steps(main_pass, Q1, g8 + 4, 4, yk, false, T, dl, Q0, true);
                } else {
                    steps(main_pass, Q1, g8 + 4, 4, yk, false, T, dl, Q0, false);
                }
                flush(yk, t0, g8, T, !main_pass, yold);
#pragma unroll
                for (int e = 0; e < 4; ++e) yold[e] = ynext[e];
            }
        } else {
#pragma unroll 1
            for (int g8 = 0; g8 < nval; g8 += 8) {
                Quad Q;
                if (!main_pass) load_yold(t0, g8, nval, yold);
                prep_load(sbuf, g8, dl, Q, main_pass);
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int jp = 0; jp < 2; ++jp) prep_exp(dl, Q, c, jp);
                steps(main_pass, Q, g8, 0, yk, true, nval, dl, Q, false);
                if (g8 + 4 < nval) {
                    prep_load(sbuf, g8 + 4, dl, Q, main_pass);
#pragma unroll
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int jp = 0; jp < 2; ++jp) prep_exp(dl, Q, c, jp);
                    steps(main_pass, Q, g8 + 4, 4, yk, true, nval, dl, Q, false);
                }
                flush(yk, t0, g8, nval, !main_pass, yold);
            }
        }
        if constexpr (SC) {
            // back from the scaled variables: multiply by beta^(steps of the chunk)
            const float s = tab_cb[nval - 1];
            const float2 s2 = f2(s, s);
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    if (main_pass) {
                        vv[c][q] = __fmul2_rn(vv[c][q], s2);
                        hh[c][q] = __fmul2_rn(hh[c][q], s2);
                        qq[c][q] = __fmul2_rn(qq[c][q], s2);
                    } else {
                        rvv[c][q] = __fmul2_rn(rvv[c][q], s2);
                        rhh[c][q] = __fmul2_rn(rhh[c][q], s2);
                    }
                }
            if (main_pass) bp2 = __fmul2_rn(bp2, s2);
        }
    };

    // One segment map (zv, zh | Q, P of the lane's two states c, 2q .. 2q+1)
    // applied to a concrete carry (v, h): the same operations in every mode, so
    // that the split launches reproduce the fused kernel bit for bit.
    auto apply_map = [&](float (&cv)[2][4], float (&ch)[2][4], float4 zvh, float4 qp, int c, int q, float bS) {
        const float zv[2] = {zvh.x, zvh.y}, zh[2] = {zvh.z, zvh.w};
        const float Qm[2] = {qp.x, qp.y}, Pm[2] = {qp.z, qp.w};
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
            const int e = 2 * q + e2;
            const float hn = fmaf(Pm[e2], ch[c][e], fmaf(Qm[e2], cv[c][e], zh[e2]));
            cv[c][e] = fmaf(bS, cv[c][e], zv[e2]);
            ch[c][e] = hn;
        }
    };
    // Split launches: the records of segments j0 .. j1-1 of the whole sequence
    // folded in order onto the carry.  Records stream through a ring of
    // kFoldRing slots in the (then idle) staging area, kFoldRing - 1 ahead of
    // the one applied: the fold's time is its FMA chain, not one L2 round trip
    // per segment.  Each lane copies and reads only its own 8 float4 of a
    // record, so no barrier is needed.
    constexpr int kFoldRing = 4;
    static_assert(kFoldRing * 8 * NT * 16 <= ST * TL::STAGE_BYTES, "the fold ring fits the staging area");
    auto fold_records = [&](float (&cv)[2][4], float (&ch)[2][4], int64_t j0, int64_t j1) {
        const int64_t nfold = j1 > j0 ? j1 - j0 : 0;
        const float4* rec0 = sp.maps + (j0 * ncl + (int64_t)(blockIdx.x / csize)) * REC + tid;
        const int64_t seg_stride = ncl * REC;
        float4* ring = reinterpret_cast<float4*>(smem) + tid;        // [slot][8][NT]
        auto fetch = [&](int64_t j) {
            if (j < nfold) {
                const int slot = (int)(j % kFoldRing);
#pragma unroll
                for (int i = 0; i < 8; ++i) cp_async_16(ring + (slot * 8 + i) * NT, rec0 + j * seg_stride + i * NT, 16);
            }
            cp_async_commit();            // one group per record index, empty past the end
        };
        for (int64_t j = 0; j < kFoldRing - 1; ++j) fetch(j);
        for (int64_t j = 0; j < nfold; ++j) {
            fetch(j + kFoldRing - 1);
            cp_async_wait<kFoldRing - 1>();   // record j's group has landed
            const float4* cur = ring + (int)(j % kFoldRing) * 8 * NT;
            const int64_t sj = (j0 + j) * seg_len;
            const int64_t lj = sp.L_total - sj < seg_len ? sp.L_total - sj : seg_len;
            const float bS = pow_steps(beta, lj);
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int i0 = (c * 2 + q) * 2;
                    apply_map(cv, ch, cur[i0 * NT], cur[(i0 + 1) * NT], c, q, bS);
                }
        }
        cp_async_wait<0>();
        // the correction's tiled copies overwrite the ring next (behind a CTA barrier)
        fence_proxy_async_smem();
    };

    // The carry entering the segment rounds: (h0, v0) folded through the
    // earlier pieces' records.  In a piece after the first, one CTA of each
    // cluster (the channel tile's CTAs) folds them and the others copy the
    // result from its shared memory, instead of every CTA reading every
    // earlier record.
    auto load_carry = [&](float (&cv)[2][4], float (&ch)[2][4]) {
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) { cv[c][e] = carry_at(c, e, 0); ch[c][e] = carry_at(c, e, 1); }
    };
    auto store_carry = [&](const float (&cv)[2][4], const float (&ch)[2][4]) {
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) { carry_at(c, e, 0) = cv[c][e]; carry_at(c, e, 1) = ch[c][e]; }
    };
    if constexpr (MODE == 2) {
        if (sp.seg_first > 0) {           // launched in clusters of the tile's csize CTAs
            if (rank == 0) {
                float cv[2][4], ch[2][4];
                load_carry(cv, ch);
                fold_records(cv, ch, 0, sp.seg_first);
                store_carry(cv, ch);
            }
            cluster_sync_all();
            if (rank != 0) {
                const uint32_t src = dsmem_map(base + TL::OFF_CARRY, 0u);
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
#pragma unroll
                        for (int w2 = 0; w2 < 2; ++w2)
                            carry_at(c, e, w2) = dsmem_ld1(src + (uint32_t)(((((c * 4 + e) * 2 + w2) * NT) + tid) * 4));
            }
            cluster_sync_all();           // rank 0's area has been read before any CTA goes on
        }
    }

    for (int64_t r = 0; r < rounds; ++r) {
        const int64_t k = r * csize + rank;                       // this CTA's segment
        const int64_t s0 = k * seg_len;
        const int64_t slen = s0 < L ? (L - s0 < seg_len ? L - s0 : seg_len) : 0;
        const int64_t nch = (slen + T - 1) / T;

        // ================= main pass: the segment from a zero state ==============
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int q = 0; q < 2; ++q) vv[c][q] = hh[c][q] = qq[c][q] = f2(0.0f, 0.0f);
        bp2 = SC ? f2(1.0f, 1.0f) : beta2;
        dpart = 0.0f;
        dbits = 0;
        if (MODE != 2 && !dead && nch > 0) {
            for (int64_t j = 0; j < ST && j < nch; ++j) issue(s0 + j * T, true);
            for (int64_t kc = 0; kc < nch; ++kc) {
                const unsigned char* sbuf = wait_next();
                if (dead) break;
                const int64_t t0 = s0 + kc * T;
                const int nval = (int)(slen - kc * T < T ? slen - kc * T : T);
                transpose(sbuf, true);
                delta_sums(sbuf);
                __syncthreads();
                run_chunk(sbuf, t0, nval, true);
                __syncthreads();          // every lane is done with this stage and B^T, C^T
                const int64_t nx = kc + ST;
                if (nx < nch) issue(s0 + nx * T, true);
            }
            drain();
        }

        // ================= publish this segment's map; fold the carries ===========
        bool seg_nonneg = __syncthreads_and((dbits & 0x80000000u) == 0u) != 0;
        // the channel's delta sum: its two threads' halves, then to the pair's lanes
        const float dch_sum = dpart + __shfl_xor_sync(0xffffffffu, dpart, 1);
        float dsum[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) dsum[c] = __shfl_sync(0xffffffffu, dch_sum, 2 * (lch[c] & 15));
        if constexpr (MODE == 1) {
            // the split's first launch: this segment's map and delta-sign flag to its record
            if (!dead && slen > 0) {
                float4 m[8];
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const float P0 = ex2_approx(Al[c][2 * q] * dsum[c]);
                        const float P1 = ex2_approx(Al[c][2 * q + 1] * dsum[c]);
                        const int i0 = (c * 2 + q) * 2;
                        m[i0] = make_float4(vv[c][q].x, vv[c][q].y, hh[c][q].x, hh[c][q].y);
                        m[i0 + 1] = make_float4(qq[c][q].x, qq[c][q].y, P0, P1);
                    }
                const float4 flag = make_float4(seg_nonneg ? 1.0f : 0.0f, 0.0f, 0.0f, 0.0f);
                const int64_t cli = (int64_t)(blockIdx.x / csize);
                auto put = [&](float4* rec) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) rec[i * NT + tid] = m[i];
                    if (tid == 0) rec[8 * NT] = flag;
                };
                if (sp.ndest > 0) {
                    for (int r = 0; r < sp.ndest; ++r) put(sp.dests[r] + ((sp.seg_first + k) * ncl + cli) * REC);
                } else {
                    put(sp.maps + (k * ncl + cli) * REC);
                }
            }
            continue;                     // no fold and no correction in this launch
        }
        if constexpr (MODE == 0) {
            if (!dead) {
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const float P0 = ex2_approx(Al[c][2 * q] * dsum[c]);
                        const float P1 = ex2_approx(Al[c][2 * q + 1] * dsum[c]);
                        const int i0 = (c * 2 + q) * 2;
                        agg[i0 * NT + tid] = make_float4(vv[c][q].x, vv[c][q].y, hh[c][q].x, hh[c][q].y);
                        agg[(i0 + 1) * NT + tid] = make_float4(qq[c][q].x, qq[c][q].y, P0, P1);
                    }
            }
            cluster_sync_all();           // every segment's map is published
        }
        float cv[2][4], ch[2][4];         // the concrete carry, folded segment by segment
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) { cv[c][e] = carry_at(c, e, 0); ch[c][e] = carry_at(c, e, 1); }
        float rv[2][4], rh[2][4];         // this segment's carry-in
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) { rv[c][e] = 0.0f; rh[c][e] = 0.0f; }
        if constexpr (MODE == 2) {
            // the carry-in of global segment kg: the carry at the round's start (every
            // earlier segment's map, in order, onto (h0, v0)) through the round's
            // segments before it
            const int64_t kg = sp.seg_first + k;
            if (!dead && slen > 0) {
                fold_records(cv, ch, sp.seg_first + r * csize, kg);
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int e = 0; e < 4; ++e) { rv[c][e] = cv[c][e]; rh[c][e] = ch[c][e]; }
                seg_nonneg = sp.maps[(kg * ncl + (int64_t)(blockIdx.x / csize)) * REC + 8 * NT].x != 0.0f;
            }
        }
        for (int jr = 0; MODE == 0 && jr < csize; ++jr) {
            if (jr == rank) {
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int e = 0; e < 4; ++e) { rv[c][e] = cv[c][e]; rh[c][e] = ch[c][e]; }
            }
            const int64_t kj = r * csize + jr;
            const int64_t sj = kj * seg_len;
            const int64_t lj = sj < L ? (L - sj < seg_len ? L - sj : seg_len) : 0;
            if (lj <= 0 || dead) continue;
            const float bS = pow_steps(beta, lj);
            const uint32_t ra = dsmem_map(agg_addr, (uint32_t)jr);
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int i0 = (c * 2 + q) * 2;
                    apply_map(cv, ch, dsmem_ld4(ra + (uint32_t)((i0 * NT + tid) * 16)),
                              dsmem_ld4(ra + (uint32_t)(((i0 + 1) * NT + tid) * 16)), c, q, bS);
                }
        }
        if constexpr (MODE == 0) {
            cluster_sync_all();           // every CTA has read the maps: the area is free again
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int e = 0; e < 4; ++e) { carry_at(c, e, 0) = cv[c][e]; carry_at(c, e, 1) = ch[c][e]; }
        }

        // ================= correction: the response to the carry-in ==============
        bool any = false;
        float bnd0[2][4];
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                bnd0[c][e] = fabsf(rh[c][e]) + kappa * fabsf(rv[c][e]);
                any = any || rv[c][e] != 0.0f || rh[c][e] != 0.0f;
            }
        any = __syncthreads_or(any) != 0;
        const bool can_stop = a_nonpos && seg_nonneg;
        if (!dead && any && nch > 0) {
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    rvv[c][q] = f2(rv[c][2 * q], rv[c][2 * q + 1]);
                    rhh[c][q] = f2(rh[c][2 * q], rh[c][2 * q + 1]);
                }
            for (int64_t j = 0; j < ST && j < nch; ++j) issue(s0 + j * T, false);
            for (int64_t kc = 0; kc < nch; ++kc) {
                const unsigned char* sbuf = wait_next();
                if (dead) break;
                const int64_t t0 = s0 + kc * T;
                const int nval = (int)(slen - kc * T < T ? slen - kc * T : T);
                transpose(sbuf, false);
                __syncthreads();
                run_chunk(sbuf, t0, nval, false);
                // Stop once every lane's response bound has fallen below 2^-25 of its start.
                bool small = can_stop;
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const float b0 = fabsf(rhh[c][q].x) + kappa * fabsf(rvv[c][q].x);
                        const float b1 = fabsf(rhh[c][q].y) + kappa * fabsf(rvv[c][q].y);
                        small = small && b0 <= kCorrTol * bnd0[c][2 * q] && b1 <= kCorrTol * bnd0[c][2 * q + 1];
                    }
                const bool stop = __syncthreads_and(small) != 0;   // also: every lane is done with this stage
                if (stop) break;
                const int64_t nx = kc + ST;
                if (nx < nch) issue(s0 + nx * T, false);
            }
            drain();
        }
        if constexpr (MODE == 2) {
            // the carry at the next round's start: the round's segments of this piece
            const int64_t j0 = sp.seg_first + r * csize;
            const int64_t jend = sp.seg_first + nseg < j0 + csize ? sp.seg_first + nseg : j0 + csize;
            if (!dead && r + 1 < rounds) {
                float cv[2][4], ch[2][4];
                load_carry(cv, ch);
                fold_records(cv, ch, j0, jend);
                store_carry(cv, ch);
            }
        }
    }

    // ---- final states: the carry after the last segment -----------------------
    if constexpr (MODE == 2) {
        // every segment of the whole sequence folded onto (h0, v0): from the carry
        // at the last round's start, through the rest
        if (rank == 0 && !dead) {
            float cv[2][4], ch[2][4];
            load_carry(cv, ch);
            fold_records(cv, ch, sp.seg_first + (rounds - 1) * csize, sp.nseg_total);
            store_carry(cv, ch);
        }
    }
    if constexpr (MODE == 1) {
        // records written into other ranks' memory are visible there before the
        // kernel is seen complete
        if (sp.ndest > 0) __threadfence_system();
    }
    if (MODE != 1 && rank == 0 && !dead) {
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int n = 4 * g + e;
                if (act[c] && n < N) {
                    const int64_t si = (b * p.dim + dch[c]) * N + n;
                    if (p.hT) p.hT[si] = carry_at(c, e, 1);
                    if (p.vT) p.vT[si] = carry_at(c, e, 0);
                }
            }
    }
}

// ------------------------------------------------------------- launch -----
namespace {

constexpr int kSegWarps = 1;
constexpr int kSegStages = 2;

// SMs of the current device (148 on B200; that count when no device answers).
int device_sms() {
    static std::atomic<int> sms_of[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        (void)cudaGetLastError();
        return 148;
    }
    int n = sms_of[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        (void)cudaGetLastError();
        return 148;
    }
    sms_of[dev].store(n, std::memory_order_relaxed);
    return n;
}

template <typename IO, bool SC, int MODE>
cudaError_t launch_seg(const ScanArgs& a0, int64_t seg_len, const SegSplit& sp, cudaStream_t stream) {
    using TL = SegTile<IO, kSegWarps, kSegStages>;
    ScanArgs a = a0;
    a.tiles_per_batch = (int)((a.dim + TL::CH - 1) / TL::CH);
    const int64_t nseg = (a.seqlen + seg_len - 1) / seg_len;
    // A launch in clusters holds at most kSegMaxCluster segments of a channel
    // tile at a time.  A plain grid (the CTAs share nothing) holds as many as
    // fill two one-warp CTAs on every warp scheduler, if that is more: a forced
    // length cutting the long workload into nine segments then runs them in one
    // round (eight per round would leave the ninth to a second round alone).
    const bool clustered = MODE == 0 || (MODE == 2 && sp.seg_first > 0);
    int64_t cap = kSegMaxCluster;
    if (!clustered) {
        const int64_t fill = (int64_t)8 * device_sms() / (a.batch * a.tiles_per_batch);
        if (fill > cap) cap = fill < kSegMaxRound ? fill : kSegMaxRound;
    }
    const int csize = (int)(nseg < cap ? nseg : cap);
    const int64_t grid = (int64_t)csize * a.batch * a.tiles_per_batch;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    CUtensorMap mx, md, mB, mC;
    const bool bf = sizeof(IO) == 2;
    const uint64_t L = (uint64_t)a.seqlen;
    cudaError_t e;
    // (the correction launch of a split reads no x and no B: its maps for them
    // describe delta and C and are never used)
    const void* xs = MODE == 2 ? a.delta : a.x;
    const void* Bs = MODE == 2 ? a.C : a.B;
    if ((e = make_map_3d(&mx, xs, bf, L, a.dim, a.batch, TL::T, TL::CH)) != cudaSuccess) return e;
    if ((e = make_map_3d(&md, a.delta, bf, L, a.dim, a.batch, TL::T, TL::CH)) != cudaSuccess) return e;
    if ((e = make_map_3d(&mB, Bs, bf, L, a.dstate, a.batch, TL::T, TL::NP)) != cudaSuccess) return e;
    if ((e = make_map_3d(&mC, a.C, bf, L, a.dstate, a.batch, TL::T, TL::NP)) != cudaSuccess) return e;
    auto kern = scan_seg_kernel<IO, kSegWarps, kSegStages, SC, MODE>;
    // The shared-memory attribute of all three modes is set on the first launch
    // of any on a device: a later call that switches to the fused launch (under
    // graph capture, say) then makes no such call.
    static std::atomic<uint64_t> attr_done{0};
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_done.load(std::memory_order_acquire) & bit)) {
        const void* kerns[3] = {reinterpret_cast<const void*>(scan_seg_kernel<IO, kSegWarps, kSegStages, SC, 0>),
                                reinterpret_cast<const void*>(scan_seg_kernel<IO, kSegWarps, kSegStages, SC, 1>),
                                reinterpret_cast<const void*>(scan_seg_kernel<IO, kSegWarps, kSegStages, SC, 2>)};
        for (const void* k : kerns)
            if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, TL::SMEM_BYTES)) !=
                cudaSuccess)
                return e;
        attr_done.fetch_or(bit, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(TL::NT, 1, 1);
    cfg.dynamicSmemBytes = TL::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // Load-balancing placement spreads the clusters' one-warp CTAs over all 148
    // SMs (6-8 each for the long workload); the default placement filled 142
    // SMs to 7-8 and left 6 without any.
    attr[1].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
    attr[1].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicyLoadBalancing;
    cfg.attrs = attr;
    // the split launches run as plain grids, placed freely, except the second
    // launch of a piece after the first, whose tiles share one fold of the
    // earlier pieces' records in a cluster
    cfg.numAttrs = clustered ? 2 : 0;
    return cudaLaunchKernelEx(&cfg, kern, mx, md, mB, mC, a, seg_len, csize, sp);
}

template <int MODE>
cudaError_t launch_seg_mode(const ScanArgs& a, int io, int64_t seg_len, const SegSplit& sp, cudaStream_t s) {
    // The scaled form needs beta^-T within range: beta >= 1/2 (see the kernel).
    const bool scaled = a.beta >= 0.5f;
    if (io == 0)
        return scaled ? launch_seg<float, true, MODE>(a, seg_len, sp, s) : launch_seg<float, false, MODE>(a, seg_len, sp, s);
    return scaled ? launch_seg<bf16, true, MODE>(a, seg_len, sp, s) : launch_seg<bf16, false, MODE>(a, seg_len, sp, s);
}

}  // namespace

int64_t scan_seg_default_len(int64_t batch, int64_t dim) {
    // About 2^25 channel-steps per round of segments: 16384 steps for 2048
    // channels (eight segments of a 131072-step sequence), longer for fewer
    // channels, never shorter than 16384 so that the correction -- a few
    // thousand steps at beta = 0.99 -- stays a small part of a segment.
    const int64_t ch = batch * dim;
    int64_t s = kSegMinLen;
    while (s < (int64_t(1) << 30) && s * ch < (int64_t(1) << 25)) s <<= 1;
    return s;
}

namespace {

// Stream-ordered memory for the segment records of the two-launch form: one
// pool per device, created on first use, keeping up to kPoolKeepBytes
// reserved between calls so that a call after a synchronisation does not go
// back to the driver for its records.
constexpr int kPoolDevices = 64;
constexpr uint64_t kPoolKeepBytes = uint64_t(64) << 20;
constexpr int64_t kMaxRecordBytes = int64_t(1) << 30;   // larger record sets run the fused launch
std::mutex g_pool_mutex;
cudaMemPool_t g_pool[kPoolDevices] = {};
bool g_pool_unavailable[kPoolDevices] = {};

cudaMemPool_t records_pool() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kPoolDevices) {
        (void)cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_pool_mutex);
    if (g_pool[dev] || g_pool_unavailable[dev]) return g_pool[dev];
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
        (void)cudaGetLastError();
        g_pool_unavailable[dev] = true;
        return nullptr;
    }
    uint64_t keep = kPoolKeepBytes;
    (void)cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    g_pool[dev] = pool;
    return pool;
}

// Bytes of the records of every segment of the call, or -1 beyond kMaxRecordBytes.
int64_t call_record_bytes(const ScanArgs& a, int64_t seg_len) {
    const int64_t nseg = (a.seqlen + seg_len - 1) / seg_len;
    constexpr int CH = SegTile<float, kSegWarps, kSegStages>::CH;
    const int64_t tiles = (a.dim + CH - 1) / CH;
    const double b = (double)nseg * (double)a.batch * (double)tiles * (double)scan_seg_tile_record_bytes();
    return b > (double)kMaxRecordBytes ? -1 : (int64_t)b;
}

}  // namespace

cudaError_t launch_scan_seg(const ScanArgs& a, int io, int64_t seg_len, bool fused, cudaStream_t s) {
    // A stream being captured into a graph gets the fused launch: no pool is
    // created and nothing is allocated while the capture is open.
    cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &capture) != cudaSuccess) {
        (void)cudaGetLastError();
        capture = cudaStreamCaptureStatusActive;
    }
    if (!fused && capture == cudaStreamCaptureStatusNone) {
        // The two-launch form: main passes with their maps to records in
        // stream-ordered memory, then the fold and correction.  Compiled
        // apart, the main pass runs 6% faster than inside the fused kernel.
        const int64_t bytes = call_record_bytes(a, seg_len);
        cudaMemPool_t pool = bytes > 0 ? records_pool() : nullptr;
        void* rec = nullptr;
        const size_t request = a.deny_records ? (size_t(1) << 62) : (size_t)bytes;
        if (pool && cudaMallocFromPoolAsync(&rec, request, pool, s) == cudaSuccess) {
            SegSplit sp{};
            sp.maps = static_cast<float4*>(rec);
            sp.seg_first = 0;
            sp.L_total = a.seqlen;
            sp.nseg_total = (a.seqlen + seg_len - 1) / seg_len;
            cudaError_t e = launch_seg_mode<1>(a, io, seg_len, sp, s);
            if (e == cudaSuccess) e = launch_seg_mode<2>(a, io, seg_len, sp, s);
            const cudaError_t ef = cudaFreeAsync(rec, s);
            return e != cudaSuccess ? e : ef;
        }
        (void)cudaGetLastError();   // no records: the fused launch needs none
    }
    return launch_seg_mode<0>(a, io, seg_len, SegSplit{}, s);
}

int64_t scan_seg_chunk_steps(int io) {
    return io == 0 ? SegTile<float, kSegWarps, kSegStages>::T : SegTile<bf16, kSegWarps, kSegStages>::T;
}

int64_t scan_seg_tile_channels() { return SegTile<float, kSegWarps, kSegStages>::CH; }

int64_t scan_seg_tile_record_bytes() {
    using TL = SegTile<float, kSegWarps, kSegStages>;
    static_assert(SegTile<bf16, kSegWarps, kSegStages>::CH == TL::CH && SegTile<bf16, kSegWarps, kSegStages>::NT == TL::NT,
                  "one record layout for both element types");
    return (int64_t)(8 * TL::NT + 1) * 16;
}

cudaError_t launch_scan_seg_split(const ScanArgs& a, int io, int64_t seg_len, int mode, void* maps,
                                  int64_t seg_first, int64_t seqlen_total, void* const* dests, int ndest,
                                  cudaStream_t s) {
    SegSplit sp{};
    sp.maps = static_cast<float4*>(maps);
    sp.dests = reinterpret_cast<float4* const*>(dests);
    sp.ndest = ndest;
    sp.seg_first = seg_first;
    sp.L_total = seqlen_total;
    sp.nseg_total = (seqlen_total + seg_len - 1) / seg_len;
    if (mode == 1) return launch_seg_mode<1>(a, io, seg_len, sp, s);
    if (mode == 2) return launch_seg_mode<2>(a, io, seg_len, sp, s);
    return cudaErrorInvalidValue;
}

unsigned int scan_seg_read_and_clear_device_error() {
    unsigned int v = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_seg_dev_err, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_seg_dev_err, &z, sizeof(z));
    return v;
}

}  // namespace mmscan
