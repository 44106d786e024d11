// ssd_fwd.cu -- Mamba-2 scalar-A multi-head scan through the chunked (SSD)
// algorithm on sm_100a tensor cores (tcgen05 / TMEM).
//
// What it computes ("Mamba-2 -- SSM = structured matrix multiply", "4-Step
// Algorithm" and "Multi-Head Expansion"; first-order discretization
// B_bar = delta B as on the Momentum Mamba page), for batch row b, head h
// (group g = h / (H/G)), head channel p, state n:
//     h_t[p, n] = exp(delta_t A_h) h_{t-1}[p, n] + alpha delta_t B_t[n] x_t[p]
//     y_t[p]    = sum_n C_t[n] h_t[p, n]
//
// Design.  One persistent CTA per (b, h) walks the sequence in blocks of
// 128 rows, so the state S (N x P = 128 x 64, fp32) never leaves the SM.
// For a block with in-block cumulative log-decay cs_i = sum_{t<=i} delta_t A_h:
//  1. intra-block:  CB = C . B^T (128 x 128, K = N) on the tensor core into
//     TMEM; the compute warps turn it into the masked, decayed matrix
//     M_ij = CB_ij exp(cs_i - cs_j) alpha delta_j (j <= i), written back into
//     TMEM as bf16 pairs, and Y_diag = M . X runs with A read from TMEM.
//  2. block state:  s = B^T . (w o X), w_j = exp(cs_last - cs_j) alpha delta_j.
//  3. inter-block:  S <- exp(cs_last) S + s, in registers of the compute
//     warps (thread n holds row n of S).
//  4. output:       Y_off = C . S_prev^T on the tensor core with S_prev in
//     shared memory as bf16; y = Y_diag + exp(cs_i) Y_off, stored as bf16.
// A chunk of Q = 256 rows is processed as two such blocks: its two diagonal
// 128 x 128 blocks of the masked matrix are formed densely and its
// off-diagonal block, which is rank <= N (the semiseparable structure the
// page describes), is applied through the block state of step 2-4.  The
// result is the same chunked recurrence up to rounding.
//
// Factored blocks.  With ref = cs_last / 2, exp(cs_i - cs_j) = e_i g_j where
// e_i = 2^(cs_i - ref) and g_j = 2^(ref - cs_j) (log2 units).  When every
// |cs_i - ref| is at most FACTOR_RANGE (the usual case), g_j alpha delta_j is
// folded into X in place (X~), M is CB with the causal mask only, the block
// state is 2^(cs_last - ref) B^T . X~, Y_off uses 2^ref S_prev, and Y_diag
// accumulates onto Y_off, so that y = e_i (M . X~ + C . (2^ref S_prev)^T).
// Blocks with a wider decay range use the per-element form above.
//
// Roles (10 warps): warps 0-3 (mask warpgroup) scale X and form M; warps 4-7
// (state warpgroup) run the decay scan one block ahead, carry S and write y
// through TMA stores; warp 8 issues TMA loads (no multicast) into a 2-deep
// ring whose B/C and X parts are refilled separately; warp 9 issues all
// tcgen05.mma.  Every wait is an mbarrier wait bounded by kWaitLimitNs; on
// give-up the kernel records the fact and every role leaves its loop, TMEM
// is freed and the kernel returns.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "mm_common.cuh"
#include "mm_internal.h"
#include "mm_tma_host.h"

namespace mmscan {

static __device__ unsigned int g_ssd_dev_err = 0;
// First wait that gave up: 0x80000000 | role << 24 | barrier << 16 | block.
static __device__ unsigned int g_ssd_dev_where = 0;

namespace ssd {
constexpr int P = 64;                 // head dimension
constexpr int NS = 128;               // states
constexpr int UB = 128;               // rows per block
constexpr int NCOMP = 128;            // threads of one compute warpgroup
constexpr int NTHREADS = 2 * NCOMP + 64;  // mask warpgroup + state warpgroup + producer + MMA
constexpr int W_PROD = 8, W_MMA = 9;  // warp indices of the producer and the MMA issuer
constexpr int X_TILE = UB * P * 2;          // 16 KB: [128 rows][64] bf16, swizzled
constexpr int BC_SLAB = UB * 64 * 2;        // 16 KB: [128 rows][64 states]
constexpr int BC_TILE = 2 * BC_SLAB;        // 32 KB
constexpr int SLOT = X_TILE + 2 * BC_TILE;  // 80 KB: X, B, C of one block
constexpr int OFF_XHAT = 2 * SLOT;
constexpr int S_TILE = NS * P * 2;         // 16 KB: [128 rows n][64 p] bf16, swizzled
constexpr int OFF_S = OFF_XHAT + X_TILE;    // 2 S buffers
constexpr int Y_STAGE = UB * 32 * 2;       // 8 KB: half a y tile, [128 rows][32] bf16, 64-byte swizzle
constexpr int OFF_YST = OFF_S + 2 * S_TILE;
constexpr int OFF_CS = OFF_YST + Y_STAGE;   // cs[2][128] fp32 (log2 units)
constexpr int OFF_DA = OFF_CS + 2 * UB * 4; // alpha*delta[2][128]
constexpr int OFF_CF = OFF_DA + 2 * UB * 4; // column factors [2][128]
constexpr int OFF_WT = OFF_CF + 2 * UB * 4;  // row factor of X for the block state [2][128]
constexpr int OFF_RED = OFF_WT + 2 * UB * 4;
constexpr int OFF_MODE = OFF_RED + 64;      // per buffer: 1 = factored block (see the kernel comment)
constexpr int OFF_BAR = OFF_MODE + 16;
constexpr int NBAR = 24;
constexpr int OFF_TSLOT = OFF_BAR + NBAR * 8;
constexpr int OFF_ABORT = OFF_TSLOT + 8;
constexpr int SMEM_BYTES = OFF_ABORT + 8 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
// TMEM columns: CB/M + Y_diag for two blocks, Y_off for two blocks, block state.
__device__ __forceinline__ uint32_t tm_cb(int k) { return (uint32_t)k * 128u; }        // 0, 128
__device__ __forceinline__ uint32_t tm_yoff(int k) { return 256u + (uint32_t)k * 64u; }  // 256, 320
constexpr uint32_t TM_STATE = 384;
constexpr uint32_t TM_COLS = 512;
// barriers
// One "ready" barrier per S buffer: the compute warps may publish the state
// of the next block before the MMA warp has consumed this one, so a single
// barrier could run two phases ahead of its waiter.
enum { B_FULL = 0, B_EMPTY = 2, B_CB = 4, B_M = 6, B_Y = 8, B_TFREE = 10,
       B_XHAT = 12, B_STATE = 13, B_SFREE = 14, B_SREADY = 15 /* and 16 */,
       B_SCAL = 17 /* and 18: per-block scalars ready for the state warpgroup */,
       B_FULLX = 19, B_EMPTYX = 21 /* X part of a slot; B_FULL / B_EMPTY cover its B and C */ };
constexpr uint32_t ID_CB = umma_idesc_bf16(128, 128, 0, 0);  // C . B^T
constexpr uint32_t ID_ST = umma_idesc_bf16(128, 64, 1, 1);   // B^T . Xhat (both MN-major)
constexpr uint32_t ID_YD = umma_idesc_bf16(128, 64, 0, 1);   // M(tmem) . X (X MN-major)
constexpr uint32_t ID_YO = umma_idesc_bf16(128, 64, 0, 1);   // C . S^T (S MN-major)
// A block is factored when every |cs_i - cs_last / 2| stays within this many
// powers of two: the factors 2^(cs_i - ref) and 2^(ref - cs_j) then stay far
// from the fp32 / bf16 range limits.
constexpr float FACTOR_RANGE = 60.0f;
}  // namespace ssd

struct SSDKArgs {
    const float* delta;
    const float* A;
    const float* h0;
    bf16* y;
    float* hT;
    int64_t batch, seqlen, nheads, ngroups;
    int nblocks;
    float alpha;
    int stall;
};

__global__ void __launch_bounds__(ssd::NTHREADS, 1)
ssd_fwd_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_B,
               const __grid_constant__ CUtensorMap tm_C, const __grid_constant__ CUtensorMap tm_y,
               const SSDKArgs p) {
    using namespace ssd;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (base - raw_addr);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int64_t b = blockIdx.x / p.nheads;
    const int64_t h = blockIdx.x % p.nheads;
    const int64_t g = h / (p.nheads / p.ngroups);
    const int64_t L = p.seqlen;
    const int nblk = p.nblocks;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
    auto bar = [&](int i) { return base + OFF_BAR + 8u * (uint32_t)i; };

    if (tid == 0) {
        mbar_init(bar(B_FULL + 0), 1); mbar_init(bar(B_FULL + 1), 1);
        mbar_init(bar(B_EMPTY + 0), 1); mbar_init(bar(B_EMPTY + 1), 1);
        mbar_init(bar(B_FULLX + 0), 1); mbar_init(bar(B_FULLX + 1), 1);
        mbar_init(bar(B_EMPTYX + 0), 1); mbar_init(bar(B_EMPTYX + 1), 1);
        mbar_init(bar(B_CB + 0), 1); mbar_init(bar(B_CB + 1), 1);
        mbar_init(bar(B_M + 0), NCOMP); mbar_init(bar(B_M + 1), NCOMP);
        mbar_init(bar(B_Y + 0), 1); mbar_init(bar(B_Y + 1), 1);
        mbar_init(bar(B_TFREE + 0), NCOMP); mbar_init(bar(B_TFREE + 1), NCOMP);
        mbar_init(bar(B_XHAT), NCOMP);
        mbar_init(bar(B_STATE), 1);
        mbar_init(bar(B_SFREE), NCOMP);
        mbar_init(bar(B_SREADY + 0), NCOMP); mbar_init(bar(B_SREADY + 1), NCOMP);
        mbar_init(bar(B_SCAL + 0), NCOMP); mbar_init(bar(B_SCAL + 1), NCOMP);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(base + OFF_TSLOT, TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TSLOT);

    int role = warp == W_PROD ? 1 : warp == W_MMA ? 2 : warp < 4 ? 3 : 4;
    int cur_blk = 0;
    auto wait = [&](int i, uint32_t parity) -> bool {
        if (*abort_flag) return false;
        if (!mbar_wait(bar(i), parity, &g_ssd_dev_err)) {
            atomicCAS(&g_ssd_dev_where, 0u, 0x80000000u | ((uint32_t)role << 24) | ((uint32_t)i << 16) |
                                                ((uint32_t)cur_blk & 0xffffu));
            *abort_flag = 1;
            return false;
        }
        return true;
    };

    if (warp == W_PROD) {
        // ------------------------------------------------------ producer ----
        // (stall: test only, nothing staged, every other role's wait runs out)
        if (lane == 0 && !p.stall) {
            for (int u = 0; u < nblk; ++u) {
                cur_blk = u;
                const int s = u & 1;
                // B and C of a slot are released once the block's state and Y_off
                // products are done, X only after Y_diag, which waits for the mask:
                // the two parts are refilled separately.
                if (!wait(B_EMPTY + s, (uint32_t)(((u >> 1) + 1) & 1))) break;
                const uint32_t slot = base + s * SLOT;
                const uint32_t fb = bar(B_FULL + s);
                mbar_expect_tx(fb, 2 * BC_TILE);
                const int t0 = u * UB;
                tma_load_4d(slot + X_TILE, &tm_B, fb, 0, (int)g, t0, (int)b);
                tma_load_4d(slot + X_TILE + BC_SLAB, &tm_B, fb, 64, (int)g, t0, (int)b);
                tma_load_4d(slot + X_TILE + BC_TILE, &tm_C, fb, 0, (int)g, t0, (int)b);
                tma_load_4d(slot + X_TILE + BC_TILE + BC_SLAB, &tm_C, fb, 64, (int)g, t0, (int)b);
                if (!wait(B_EMPTYX + s, (uint32_t)(((u >> 1) + 1) & 1))) break;
                const uint32_t fx = bar(B_FULLX + s);
                mbar_expect_tx(fx, X_TILE);
                tma_load_4d(slot, &tm_x, fx, 0, (int)h, t0, (int)b);
            }
        }
    } else if (warp == W_MMA) {
        // ----------------------------------------------------------- MMA ----
        // Issue order per block u: block state(u), Y_off(u) (needs only the
        // previous state, and frees the block's B and C), Y_diag(u), then
        // C.B^T(u+1) (one block ahead, so the mask warpgroup can start on it).
        if (lane == 0) {
            const uint32_t xhat = base + OFF_XHAT;
            auto issue_cb = [&](int v) -> bool {
                const int sv = v & 1, kv = v & 1;
                const uint32_t slot = base + sv * SLOT;
                const uint32_t bs = slot + X_TILE, cs = slot + X_TILE + BC_TILE;
                if (!wait(B_FULL + sv, (uint32_t)((v >> 1) & 1))) return false;
                if (!wait(B_TFREE + kv, (uint32_t)(((v >> 1) + 1) & 1))) return false;
                tc_fence_after();
                // C . B^T: M = 128 rows i, N = 128 rows j, K = 128 states
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t koff = (ks >> 2) * BC_SLAB + (ks & 3) * 32;
                    umma_ss(tmem + tm_cb(kv), umma_desc_sw128(cs + koff, 16, 1024),
                            umma_desc_sw128(bs + koff, 16, 1024), ID_CB, ks > 0);
                }
                umma_commit(bar(B_CB + kv));
                return true;
            };
            bool live = nblk > 0 && issue_cb(0);
            for (int u = 0; u < nblk && live; ++u) {
                cur_blk = u;
                const int s = u & 1, k = u & 1;
                const uint32_t slot = base + s * SLOT;
                const uint32_t xs = slot, bs = slot + X_TILE, cs = slot + X_TILE + BC_TILE;
                // block state = B^T . Xhat: M = 128 states, N = 64, K = 128 rows.  A factored
                // block has its scaled X in place in the slot, otherwise in the X_hat buffer.
                if (!(live = wait(B_XHAT, (uint32_t)(u & 1)))) break;
                if (!(live = wait(B_SFREE, (uint32_t)((u + 1) & 1)))) break;
                const bool fac = reinterpret_cast<volatile const int*>(smem + OFF_MODE)[k] != 0;
                const uint32_t xop = fac ? xs : xhat;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_ss(tmem + TM_STATE, umma_desc_sw128(bs + ks * 2048, BC_SLAB, 1024),
                            umma_desc_sw128(xop + ks * 2048, X_TILE, 1024), ID_ST, ks > 0);
                umma_commit(bar(B_STATE));
                // Y_off = C . S_prev^T
                if (!(live = wait(B_SREADY + (u & 1), (uint32_t)((u >> 1) & 1)))) break;
                tc_fence_after();
                const uint32_t sb = base + OFF_S + (u & 1) * S_TILE;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t koff_c = (ks >> 2) * BC_SLAB + (ks & 3) * 32;
                    umma_ss(tmem + tm_yoff(k), umma_desc_sw128(cs + koff_c, 16, 1024),
                            umma_desc_sw128(sb + ks * 2048, S_TILE, 1024), ID_YO, ks > 0);
                }
                umma_commit(bar(B_EMPTY + s));
                // Y_diag = M(tmem) . X
                if (!(live = wait(B_M + k, (uint32_t)((u >> 1) & 1)))) break;
                if (!(live = wait(B_FULLX + s, (uint32_t)((u >> 1) & 1)))) break;
                tc_fence_after();
                // factored: accumulate onto Y_off (y = e_i (Y_diag + Y_off)); else its own columns
                const uint32_t yd = fac ? tmem + tm_yoff(k) : tmem + tm_cb(k) + 64;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_ts(yd, tmem + tm_cb(k) + ks * 8, umma_desc_sw128(xs + ks * 2048, X_TILE, 1024), ID_YD,
                            fac || ks > 0);
                umma_commit(bar(B_Y + k));
                umma_commit(bar(B_EMPTYX + s));
                // C.B^T of the next block last: it waits for that block's B and C and
                // for TMEM buffer k^1, which must not hold up this block's output.
                if (u + 1 < nblk && !(live = issue_cb(u + 1))) break;
            }
            // Drain: the last commit must land before the CTA may exit.
            if (nblk > 0 && !*abort_flag) {
                const int u = nblk - 1;
                wait(B_EMPTYX + (u & 1), (uint32_t)((u >> 1) & 1));
            }
        }
    } else if (warp < 4) {
        // ------------------------------------- mask warpgroup (warps 0-3) ----
        // Per block: w o X and the masked matrix M.
        const int t = tid;                         // TMEM lane = row i of the block
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        // Waits are made uniform over the warpgroup (all leave the loop together),
        // since the named barriers below need every one of its threads.
        auto gwait = [&](int i, uint32_t par) { return named_bar_and(1, NCOMP, wait(i, par)); };
        bool ok = true;
        bool lok = true;    // this thread's own waits since the last uniform check
        for (int u = 0; u < nblk && ok; ++u) {
            cur_blk = u;
            const int k = u & 1;
            const float* cs_sm = reinterpret_cast<const float*>(smem + OFF_CS) + k * UB;
            const float* da_sm = reinterpret_cast<const float*>(smem + OFF_DA) + k * UB;
            const float* cf_sm = reinterpret_cast<const float*>(smem + OFF_CF) + k * UB;
            // (a) the state warpgroup has published block u's decay scalars
            ok = named_bar_and(1, NCOMP, lok && wait(B_SCAL + k, (uint32_t)((u >> 1) & 1)));
            if (!ok) break;
            const float cs = cs_sm[t];
            const bool fac = reinterpret_cast<volatile const int*>(smem + OFF_MODE)[k] != 0;

            // (b) Xhat = diag(f) X with the row factor f of OFF_WT: in place in the slot
            //     for a factored block, else into the X_hat buffer, which is
            //     single-buffered (block u-1's state MMA must be done).  Warp q
            //     scales its own range of rows: the warps with fewer mask batches
            //     in (c) take more rows, so that both steps together take about
            //     as long in every warp.
            if (u >= 1 && !(ok = gwait(B_STATE, (uint32_t)((u - 1) & 1)))) break;
            if (!(ok = gwait(B_FULLX + (u & 1), (uint32_t)((u >> 1) & 1)))) break;
            {
                const float* wt_sm = reinterpret_cast<const float*>(smem + OFF_WT) + k * UB;
                const unsigned char* xs = smem + (u & 1) * SLOT;
                unsigned char* xh = fac ? smem + (u & 1) * SLOT : smem + OFF_XHAT;
                const int r0 = fac ? warp * 32 : (warp == 0 ? 0 : warp == 1 ? 52 : warp == 2 ? 92 : 116);
                const int r1 = fac ? warp * 32 + 32 : (warp == 0 ? 52 : warp == 1 ? 92 : warp == 2 ? 116 : 128);
                const int units = (r1 - r0) * 8;
                for (int i = lane; i < units; i += 32) {
                    const int r = r0 + (i >> 3);
                    const int pc = ((i & 7) ^ (r & 7)) << 4;        // swizzled 16-byte chunk
                    const float w = wt_sm[r];
                    const uint4 q = *reinterpret_cast<const uint4*>(xs + r * 128 + pc);
                    uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) w4[e] = pack_bf16x2(bf16_lo(w4[e]) * w, bf16_hi(w4[e]) * w);
                    *reinterpret_cast<uint4*>(xh + r * 128 + pc) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(bar(B_XHAT));

            // (c) M = CB o exp(cs_i - cs_j) alpha delta_j (j <= i), bf16 pairs into TMEM.
            //     A factored block has both decay factors elsewhere (2^(ref - cs_j)
            //     alpha delta_j in X, 2^(cs_i - ref) in the epilogue): M is CB with the
            //     causal mask.  Otherwise batches below the diagonal use
            //     exp(cs_i - cs_r) exp(cs_r - cs_j), both <= 1.
            // Not a uniform wait: each warp goes on from its share of X_hat to its
            // mask batches without waiting for the others.  A failed wait skips
            // the work; the loop-top check above then ends the loop for all.
            lok = wait(B_CB + k, (uint32_t)((u >> 1) & 1));
            tc_fence_after();
            if (lok) {
                // One batch of 32 columns from its TMEM words r: decayed, masked, packed, stored.
                auto mask_batch = [&](int cb, const uint32_t (&r)[32]) {
                    uint32_t pk[16];
                    if (fac) {
                        if (cb == warp) {          // causal mask inside the diagonal batch
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const int j = cb * 32 + 2 * e;
                                pk[e] = pack_bf16x2(j <= t ? __uint_as_float(r[2 * e]) : 0.0f,
                                                    j + 1 <= t ? __uint_as_float(r[2 * e + 1]) : 0.0f);
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
                        }
                        tmem_st16(tmem + lane_base + tm_cb(k) + cb * 16, pk);
                        return;
                    }
                    // Row factor 2^(cs_i - cs_r) and column factor 2^(cs_r - cs_j) alpha delta_j,
                    // r = last column of the batch.  Below the diagonal both are <= 1; in the
                    // diagonal batch the row factor is >= 1 but bounded by 2^(batch range),
                    // so it is used only when that range stays far from fp32 overflow.
                    const float cs_r = cs_sm[cb * 32 + 31];
                    const bool factored = cb < warp || (cs_sm[cb * 32] - cs_r) <= 100.0f;
                    if (factored) {
                        const float rowf = ex2_approx(cs - cs_r);
                        const float2 rr = f2(rowf, rowf);
#pragma unroll
                        for (int e = 0; e < 16; e += 2) {
                            const float4 cf4 = *reinterpret_cast<const float4*>(cf_sm + cb * 32 + 2 * e);
#pragma unroll
                            for (int h2 = 0; h2 < 2; ++h2) {
                                const int ee = e + h2;
                                const float2 cf = h2 ? f2(cf4.z, cf4.w) : f2(cf4.x, cf4.y);
                                float2 m = __fmul2_rn(__fmul2_rn(f2(__uint_as_float(r[2 * ee]),
                                                                     __uint_as_float(r[2 * ee + 1])), cf), rr);
                                if (cb == warp) {      // causal mask inside the diagonal batch
                                    const int j = cb * 32 + 2 * ee;
                                    m.x = j <= t ? m.x : 0.0f;
                                    m.y = j + 1 <= t ? m.y : 0.0f;
                                }
                                pk[ee] = pack_bf16x2(m.x, m.y);
                            }
                        }
                    } else {
                        float m[32];
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const int j = cb * 32 + jj;
                            m[jj] = j <= t ? __uint_as_float(r[jj]) * (ex2_approx(cs - cs_sm[j]) * da_sm[j]) : 0.0f;
                        }
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(m[2 * e], m[2 * e + 1]);
                    }
                    tmem_st16(tmem + lane_base + tm_cb(k) + cb * 16, pk);
                };
                // The packed batch cb lands on columns 16 cb .. 16 cb + 15 of the same
                // buffer, i.e. on fp32 batch cb / 2, which is always read by then.
                // Batches on or below the diagonal are read two at a time, so that one
                // TMEM round trip covers both; the batches above it are zero and are
                // written last (they overlap fp32 batches this warp still reads).
#pragma unroll 1
                for (int cb = 0; cb <= warp; cb += 2) {
                    uint32_t r0[32], r1[32];
                    const bool two = cb + 1 <= warp;
                    tmem_ld32(tmem + lane_base + tm_cb(k) + cb * 32, r0);
                    if (two) tmem_ld32(tmem + lane_base + tm_cb(k) + (cb + 1) * 32, r1);
                    tmem_wait_ld();
                    mask_batch(cb, r0);
                    if (two) mask_batch(cb + 1, r1);
                }
#pragma unroll 1
                for (int cb = warp + 1; cb < 4; ++cb) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = 0u;
                    tmem_st16(tmem + lane_base + tm_cb(k) + cb * 16, pk);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(B_M + k));
        }
    } else {
        // ------------------------------------ state warpgroup (warps 4-7) ----
        // Per block: S <- exp(cs_last) S + block state, the bf16 S operand for
        // the next block, and the output y = Y_diag + exp(cs_i) Y_off.
        const int t = tid - NCOMP;                 // TMEM lane = state n = row i
        const int wq = warp - 4;
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        float S[P];                                 // row n = t of the state, fp32
        auto gwait = [&](int i, uint32_t par) { return named_bar_and(2, NCOMP, wait(i, par)); };
        {
            const float* h0 = p.h0 ? p.h0 + (((b * p.nheads + h) * P) * NS) : nullptr;
#pragma unroll
            for (int q = 0; q < P; ++q) S[q] = h0 ? h0[q * NS + t] : 0.0f;
        }
        const float a_h = p.A[h] * kLog2e;
        float* red = reinterpret_cast<float*>(smem + OFF_RED);
        auto load_dt = [&](int v) -> float {
            const int64_t tv = (int64_t)v * UB + t;
            return tv < L ? p.delta[((b * L + tv) * p.nheads) + h] : 0.0f;
        };
        // In-block log2-decay scan of block v (row t).  It decides whether the
        // block is factored: with ref = cs_last / 2 and every |cs_i - ref| within
        // FACTOR_RANGE, exp2(cs_i - cs_j) = 2^(cs_i - ref) 2^(ref - cs_j) splits
        // into a row factor applied to y and a column factor folded into X.  It
        // publishes, for the mask warpgroup (buffer v & 1), cs, alpha delta, the
        // per-batch column factors of the unfactored mask, the X row factor
        // (2^(ref - cs_j) alpha delta_j if factored, else 2^(cs_last - cs_j)
        // alpha delta_j) and the mode; it returns this warpgroup's own scalars.
        struct BlockScal {
            float et;     // y row factor: 2^(cs_t - ref) if factored, else 2^cs_t
            float gam;    // 2^cs_last: decay of the carried state over the block
            float gam2;   // factor of the block state B^T Xhat: 2^(cs_last - ref), or 1
            float sref;   // factor of S in the Y_off operand: 2^ref, or 1
            bool fac;
        };
        auto scan_block = [&](int v, float dt) -> BlockScal {
            const int kv = v & 1;
            float cs = dt * a_h;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float o = __shfl_up_sync(0xffffffffu, cs, off);
                if (lane >= off) cs += o;
            }
            if (lane == 31) red[kv * 4 + wq] = cs;
            named_bar_sync(2, NCOMP);
            float prefix = 0.0f, total = 0.0f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float v4 = red[kv * 4 + w];
                if (w < wq) prefix += v4;
                total += v4;
            }
            cs += prefix;
            const float ref = 0.5f * total;
            BlockScal bs;
            bs.fac = named_bar_and(2, NCOMP, fabsf(cs - ref) <= FACTOR_RANGE);
            const float da = p.alpha * dt;
            (reinterpret_cast<float*>(smem + OFF_CS) + kv * UB)[t] = cs;
            (reinterpret_cast<float*>(smem + OFF_DA) + kv * UB)[t] = da;
            const float cs_b = __shfl_sync(0xffffffffu, cs, 31);     // last column of this 32-batch
            (reinterpret_cast<float*>(smem + OFF_CF) + kv * UB)[t] = ex2_approx(cs_b - cs) * da;
            (reinterpret_cast<float*>(smem + OFF_WT) + kv * UB)[t] = ex2_approx((bs.fac ? ref : total) - cs) * da;
            if (t == 0) reinterpret_cast<volatile int*>(smem + OFF_MODE)[kv] = bs.fac ? 1 : 0;
            mbar_arrive(bar(B_SCAL + kv));
            bs.et = ex2_approx(bs.fac ? cs - ref : cs);
            bs.gam = ex2_approx(total);
            bs.gam2 = bs.fac ? ex2_approx(total - ref) : 1.0f;
            bs.sref = bs.fac ? ex2_approx(ref) : 1.0f;
            return bs;
        };
        // S as the bf16 B operand of C . S^T: MN-major, row n holds 64 p.
        auto write_S = [&](int buf, float scale) {
            unsigned char* row = smem + OFF_S + buf * S_TILE + t * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    w4[e] = pack_bf16x2(S[c * 8 + 2 * e] * scale, S[c * 8 + 2 * e + 1] * scale);
                *reinterpret_cast<uint4*>(row + ((c ^ (t & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(bar(B_SREADY + buf));
        };
        BlockScal cur{1.0f, 1.0f, 1.0f, 1.0f, false};   // scalars of the current block
        float dt_next = nblk > 1 ? load_dt(1) : 0.0f;
        if (nblk > 0) cur = scan_block(0, load_dt(0));
        write_S(0, cur.sref);
        bool ok = true;
        for (int u = 0; u < nblk && ok; ++u) {
            cur_blk = u;
            const int k = u & 1;
            const int64_t t0 = (int64_t)u * UB;
            const float dt1 = dt_next;               // delta of block u+1, loaded one block ahead
            if (u + 2 < nblk) dt_next = load_dt(u + 2);
            // The next block's decay scan first: it needs no result of this block,
            // and the mask warpgroup starts on the next block with it.
            BlockScal nxt{1.0f, 1.0f, 1.0f, 1.0f, false};
            if (u + 1 < nblk) nxt = scan_block(u + 1, dt1);

            // (d) S <- exp(cs_last) S + block state; publish S for the next block
            if (!(ok = gwait(B_STATE, (uint32_t)(u & 1)))) break;
            tc_fence_after();
            const float gam = cur.gam, gam2 = cur.gam2, et = cur.et;
            {
                uint32_t r0[32], r1[32];
                tmem_ld32(tmem + lane_base + TM_STATE, r0);
                tmem_ld32(tmem + lane_base + TM_STATE + 32, r1);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    S[q] = fmaf(gam, S[q], gam2 * __uint_as_float(r0[q]));
                    S[32 + q] = fmaf(gam, S[32 + q], gam2 * __uint_as_float(r1[q]));
                }
            }
            tc_fence_before();
            mbar_arrive(bar(B_SFREE));
            write_S((u + 1) & 1, nxt.sref);

            // (e) y = Y_diag + exp(cs_i) Y_off, bf16, row t of block u.  Each half
            //     (32 of the 64 columns) is staged in shared memory in the 64-byte
            //     swizzled layout of the y tensor map and written by one TMA store,
            //     which keeps the row-scattered global writes off the LSU pipe (the
            //     mask warpgroup's loads share it).  Rows past L are clipped by the map.
            if (!(ok = gwait(B_Y + k, (uint32_t)((u >> 1) & 1)))) break;
            tc_fence_after();
            {
                unsigned char* yst = smem + OFF_YST + t * 64;
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) {
                    uint32_t w[16];
                    if (cur.fac) {                           // y = e_i (Y_diag + Y_off), one accumulator
                        uint32_t ro[32];
                        tmem_ld32(tmem + lane_base + tm_yoff(k) + hc * 32, ro);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            w[e] = pack_bf16x2(et * __uint_as_float(ro[2 * e]), et * __uint_as_float(ro[2 * e + 1]));
                    } else {
                        uint32_t rd[32], ro[32];
                        tmem_ld32(tmem + lane_base + tm_cb(k) + 64 + hc * 32, rd);
                        tmem_ld32(tmem + lane_base + tm_yoff(k) + hc * 32, ro);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            w[e] = pack_bf16x2(fmaf(et, __uint_as_float(ro[2 * e]), __uint_as_float(rd[2 * e])),
                                               fmaf(et, __uint_as_float(ro[2 * e + 1]), __uint_as_float(rd[2 * e + 1])));
                    }
                    if (t == 0) bulk_wait_read_all();        // the previous store has read the stage
                    named_bar_sync(2, NCOMP);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        *reinterpret_cast<uint4*>(yst + ((c ^ ((t >> 1) & 3)) << 4)) =
                            make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                    fence_proxy_async_smem();
                    named_bar_sync(2, NCOMP);
                    if (t == 0) {
                        tma_store_4d(&tm_y, base + OFF_YST, hc * 32, (int)h, (int)t0, (int)b);
                        bulk_commit_group();
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(bar(B_TFREE + k));
            cur = nxt;
        }
        if (t == 0) bulk_wait_all();                 // y stores complete before the CTA exits
        if (ok && p.hT) {
            float* hT = p.hT + ((b * p.nheads + h) * P) * NS;
#pragma unroll
            for (int q = 0; q < P; ++q) hT[q * NS + t] = S[q];
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// ------------------------------------------------------------- launch -----
namespace {

// 4-D bf16 map (d0 innermost), box (box0, 1, 128, 1): 64 columns with the
// 128-byte swizzle for the loads, 32 columns with the 64-byte swizzle for the y stores.
cudaError_t make_map_4d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3,
                        uint32_t box0 = 64) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[4] = {d0, d1, d2, d3};
    const cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
    const cuuint32_t box[4] = {box0, 1, 128, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          box0 == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

bool ssd_shape_supported(int64_t headdim, int64_t dstate, int64_t chunk) {
    return headdim == ssd::P && dstate == ssd::NS && (chunk == 128 || chunk == 256);
}


cudaError_t launch_ssd_fwd(const SSDArgs& a, cudaStream_t stream) {
    if (a.batch * a.nheads > 0x7fffffffLL || a.seqlen > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    CUtensorMap mx, mB, mC, my;
    cudaError_t e;
    if ((e = make_map_4d(&mx, a.x, ssd::P, a.nheads, a.seqlen, a.batch)) != cudaSuccess) return e;
    if ((e = make_map_4d(&mB, a.B, ssd::NS, a.ngroups, a.seqlen, a.batch)) != cudaSuccess) return e;
    if ((e = make_map_4d(&mC, a.C, ssd::NS, a.ngroups, a.seqlen, a.batch)) != cudaSuccess) return e;
    if ((e = make_map_4d(&my, a.y, ssd::P, a.nheads, a.seqlen, a.batch, 32)) != cudaSuccess) return e;
    SSDKArgs k{};
    k.delta = a.delta; k.A = a.A; k.h0 = a.h0;
    k.y = static_cast<bf16*>(a.y); k.hT = a.hT;
    k.batch = a.batch; k.seqlen = a.seqlen; k.nheads = a.nheads; k.ngroups = a.ngroups;
    k.nblocks = (int)((a.seqlen + ssd::UB - 1) / ssd::UB);
    k.alpha = a.alpha;
    k.stall = a.stall;
    static std::atomic<uint64_t> attr_done{0};
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_done.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(ssd_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ssd::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_done.fetch_or(bit, std::memory_order_release);
    }
    ssd_fwd_kernel<<<(unsigned)(a.batch * a.nheads), ssd::NTHREADS, ssd::SMEM_BYTES, stream>>>(mx, mB, mC, my, k);
    return cudaGetLastError();
}

unsigned int ssd_read_and_clear_device_error() {
    unsigned int v = 0, w = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_ssd_dev_err, sizeof(v)) != cudaSuccess) return 0;
    if (!v) return 0;
    cudaMemcpyFromSymbol(&w, g_ssd_dev_where, sizeof(w));
    cudaMemcpyToSymbol(g_ssd_dev_err, &z, sizeof(z));
    cudaMemcpyToSymbol(g_ssd_dev_where, &z, sizeof(z));
    return w ? w : v;
}

}  // namespace mmscan
