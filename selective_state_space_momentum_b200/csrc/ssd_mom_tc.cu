// ssd_mom_tc.cu -- the multi-head scalar-A scan with the Momentum Mamba
// velocity, in the chunked (SSD) form, on sm_100a tensor cores (tcgen05 / TMEM).
//
// What it computes ("Momentum Mamba: Enhanced State Space Models with
// Momentum", "Momentum Mamba Recurrence", in the multi-head layout of
// "Mamba-2 -- SSM = structured matrix multiply", "Multi-Head Expansion"), for
// batch row b, head h (group g = h / (H/G)), head channel p, state n:
//     v_t[p, n] = beta v_{t-1}[p, n] + alpha delta_t B_t[n] x_t[p]
//     h_t[p, n] = exp(delta_t A_h) h_{t-1}[p, n] + v_t[p, n]
//     y_t[p]    = sum_n C_t[n] h_t[p, n]
// through the chunked form of the "4-Step Algorithm" of the Mamba-2 page.
// Per block of 128 rows with carried states (H, V) from the block before and
// in-block cumulative log2-decay cs_i:
//     y_i  = sum_{j<=i} M_ij (C_i . B_j) alpha delta_j x_j + 2^cs_i C_i.H + q_i C_i.V
//     M_ij = sum_{k=j}^{i} 2^(cs_i - cs_k) beta^(k-j)     (q_i = beta M_i0)
//     H'   = 2^cs_l H + q_l V + sum_j M_lj alpha delta_j B_j x_j^T
//     V'   = beta^(l+1) V + sum_j beta^(l-j) alpha delta_j B_j x_j^T
// with l the block's last row inside the sequence.  Every factor is a sum of
// positive terms no larger than 1 / (1 - beta) while A <= 0, so nothing
// cancels and nothing overflows.
//
// Tensor-core steps of a block (bf16 operands, fp32 accumulators in TMEM):
//   CB  = C . B^T (128 x 128, K = N = 128)
//   the mask warps form P_ij = M_ij alpha delta_j CB_ij (j <= i) in registers,
//       M by the row recurrence R <- 2^(cs_i - cs_j) + beta R from the
//       diagonal down to column 0, and write P back to TMEM as bf16 pairs
//   Y_diag = P . X (A operand from TMEM)
//   Y_A = C . H^T, Y_V = C . V^T (H, V as bf16 operands in shared memory)
//   s_V = B^T . (w_V o X), s_H = B^T . (w_H o X), w_V = beta^(l-j) alpha delta,
//       w_H = M_lj alpha delta
// and y = Y_diag + 2^cs_i Y_A + q_i Y_V, stored as bf16.  H and V stay in
// TMEM as fp32 accumulators: per block the state warps publish them as the
// bf16 read-out operands, rescale them in place (H <- 2^cs_l H + q_l V,
// V <- beta^(l+1) V) and the block-state products accumulate onto them.
//
// Roles (14 warps): warps 0-3 (mask warpgroup) scale X into w_V o X and,
// once Y_diag has read X, into w_H o X in place, and form P; warps 4-7 and
// 8-11 (state warpgroups, head channels 0-31 and 32-63) publish and rescale
// H and V and write y; warps 4-7 also run the block's scans (cs, the suffix recurrence
// for M_lj) one block ahead; warp 12 issues the TMA loads (no multicast)
// into a 2-deep ring; warp 13 issues every tcgen05.mma.  Every wait is an
// mbarrier wait bounded by kWaitLimitNs; on give-up the kernel records the
// fact, every role leaves its loop (each group together), TMEM is freed and
// the kernel returns.
#include <cuda.h>

#include <atomic>

#include "mm_common.cuh"
#include "mm_internal.h"
#include "mm_tma_host.h"

namespace mmscan {

static __device__ unsigned int g_ssdm_dev_err = 0;

namespace ssdmt {
constexpr int P = 64;                  // head dimension
constexpr int NS = 128;                // states
constexpr int UB = 128;                // rows per block
constexpr int NG = 128;                // threads of one warpgroup
constexpr int NTHREADS = 3 * NG + 64;  // mask warpgroup, two state warpgroups, producer warp, MMA warp
constexpr int W_PROD = 12, W_MMA = 13;
static_assert(NTHREADS == 32 * (W_MMA + 1), "roles cover every warp");
constexpr int X_TILE = UB * P * 2;          // 16 KB: [128 rows][64 p] bf16, 128-byte swizzle
constexpr int BC_SLAB = UB * 64 * 2;        // 16 KB: [128 rows][64 states]
constexpr int BC_TILE = 2 * BC_SLAB;        // 32 KB
constexpr int SLOT = X_TILE + 2 * BC_TILE;  // 80 KB: X, B, C of one block
constexpr int OFF_XV = 2 * SLOT;            // w_V o X
constexpr int S_TILE = NS * P * 2;          // 16 KB: [128 rows n][64 p] bf16, swizzled
constexpr int OFF_SH = OFF_XV + X_TILE;
constexpr int OFF_SV = OFF_SH + S_TILE;
constexpr int OFF_CS = OFF_SV + S_TILE;     // cs[2][128] (log2 units)
constexpr int OFF_DA = OFF_CS + 2 * UB * 4; // alpha delta [2][128]
constexpr int OFF_WV = OFF_DA + 2 * UB * 4; // w_V [2][128]
constexpr int OFF_WH = OFF_WV + 2 * UB * 4; // w_H [2][128]
constexpr int OFF_CF = OFF_WH + 2 * UB * 4; // column factors 2^(ref - cs_j) [2][128]
constexpr int OFF_Q = OFF_CF + 2 * UB * 4;  // q_i [2][128], written by the mask warps
constexpr int OFF_BLK = OFF_Q + 2 * UB * 4; // per buffer: 2^cs_l, q_l, beta^(l+1), ref
constexpr int OFF_MODE = OFF_BLK + 2 * 16;  // per buffer: 1 = factored block
constexpr int OFF_RED = OFF_MODE + 16;      // scan partials
constexpr int OFF_BAR = OFF_RED + 128;
constexpr int NBAR = 24;
constexpr int OFF_TSLOT = OFF_BAR + NBAR * 8;
constexpr int OFF_ABORT = OFF_TSLOT + 8;
constexpr int SMEM_BYTES = OFF_ABORT + 8 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
static_assert(SLOT % 1024 == 0 && OFF_XV % 1024 == 0 && OFF_SH % 1024 == 0 && OFF_SV % 1024 == 0,
              "swizzled tiles are 1024-byte aligned");
// TMEM columns (512): per block buffer k the fp32 C.B^T at 128k, which becomes
// P (bf16 pairs) in its upper 64 columns and Y_diag in its lower 64; the
// carried-state read-outs Y_A, Y_V; the carried states H, V themselves
// (lane n, column p), onto which the block-state products accumulate.
__device__ __forceinline__ uint32_t tm_cb(int k) { return (uint32_t)k * 128u; }
constexpr uint32_t TM_YA = 256, TM_YV = 320, TM_H = 384, TM_V = 448;
constexpr uint32_t TM_COLS = 512;
static_assert(OFF_SV == OFF_SH + S_TILE && TM_YV == TM_YA + 64, "one read-out product spans both state tiles");
enum {
    B_FULL = 0, B_EMPTY = 2, B_CB = 4, B_M = 6, B_Y = 8, B_SCAL = 10, B_TFREE = 12,  // pairs
    B_XV = 14, B_XH = 15, B_STATE = 16, B_SCALED = 17, B_SFREE = 18, B_SREADY = 19, B_YOFREE = 20
};
constexpr uint32_t ID_CB = umma_idesc_bf16(128, 128, 0, 0);  // C . B^T
constexpr uint32_t ID_ST = umma_idesc_bf16(128, 64, 1, 1);   // B^T . (w o X), both MN-major
constexpr uint32_t ID_YD = umma_idesc_bf16(128, 64, 0, 1);   // P(tmem) . X
constexpr uint32_t ID_YO = umma_idesc_bf16(128, 128, 0, 1);  // C . [H | V]^T (both states, N = 128)
// A block is factored when every |cs_i - ref| (ref = cs_l / 2) stays within
// this many powers of two: 2^(cs_i - cs_j) = 2^(cs_i - ref) 2^(ref - cs_j)
// then splits into a row factor applied to Y_diag and column factors the mask
// recurrence sums, far from the fp32 range limits.
constexpr float FACTOR_RANGE = 60.0f;
}  // namespace ssdmt

struct SSDMTArgs {
    const float* delta;
    const float* A;
    const float* h0;
    const float* v0;
    bf16* y;
    float* hT;
    float* vT;
    int64_t batch, seqlen, nheads, ngroups;
    int nblocks;
    float alpha, beta, lb;   // lb = log2(beta), or -1000 for beta = 0
    int stall;
};

// 16 consecutive 32-bit TMEM columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// One batch of 32 columns of row i of P, from column 32 cb + 31 down to 32 cb:
// R <- l_ij + beta R with l_ij = 2^(ref - cs_j) (FAC: the column factor, the
// row factor 2^(cs_i - ref) is applied to Y_diag) or 2^(cs_i - cs_j), zero
// above the diagonal (DIAG: the batch that holds it); P_ij = R alpha delta_j
// CB_ij, packed to bf16 pairs.  v holds cf_j (FAC) or cs_j, da alpha delta_j.
template <bool FAC, bool DIAG>
__device__ __forceinline__ void mom_mask_batch(const uint32_t (&r)[32], uint32_t (&pk)[16], float& R, int cb, int i,
                                               float csi, float beta, const float* v, const float* da) {
#pragma unroll
    for (int e4 = 7; e4 >= 0; --e4) {
        const float4 c4 = *reinterpret_cast<const float4*>(v + cb * 32 + 4 * e4);
        const float4 d4 = *reinterpret_cast<const float4*>(da + cb * 32 + 4 * e4);
        const float vj[4] = {c4.x, c4.y, c4.z, c4.w};
        const float dj[4] = {d4.x, d4.y, d4.z, d4.w};
        float m[4];
#pragma unroll
        for (int jj = 3; jj >= 0; --jj) {
            float l = FAC ? vj[jj] : ex2_approx(csi - vj[jj]);
            if (DIAG) l = cb * 32 + 4 * e4 + jj <= i ? l : 0.0f;
            R = fmaf(beta, R, l);
            m[jj] = R * (dj[jj] * __uint_as_float(r[4 * e4 + jj]));
        }
        pk[2 * e4] = pack_bf16x2(m[0], m[1]);
        pk[2 * e4 + 1] = pack_bf16x2(m[2], m[3]);
    }
}

// 14 warps on the SM's four schedulers: 4 warps x 32 lanes x 128 registers
// fill one scheduler's register file, so 128 is the most a thread may take.
__global__ void __maxnreg__(128)
ssd_mom_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_B,
                  const __grid_constant__ CUtensorMap tm_C, const __grid_constant__ CUtensorMap tm_y,
                  const SSDMTArgs p) {
    using namespace ssdmt;
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
    auto fsm = [&](int off, int k) { return reinterpret_cast<float*>(smem + off) + k * UB; };

    if (tid == 0) {
        for (int k = 0; k < 2; ++k) {
            mbar_init(bar(B_FULL + k), 1);
            mbar_init(bar(B_EMPTY + k), 1);
            mbar_init(bar(B_CB + k), 1);
            mbar_init(bar(B_M + k), NG);
            mbar_init(bar(B_Y + k), 1);
            mbar_init(bar(B_SCAL + k), NG);
            mbar_init(bar(B_TFREE + k), 2 * NG);
        }
        mbar_init(bar(B_XV), NG);
        mbar_init(bar(B_XH), NG);
        mbar_init(bar(B_STATE), 1);
        mbar_init(bar(B_SCALED), 2 * NG);
        mbar_init(bar(B_SFREE), 1);
        mbar_init(bar(B_SREADY), 2 * NG);
        mbar_init(bar(B_YOFREE), 2 * NG);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(base + OFF_TSLOT, TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TSLOT);

    auto wait = [&](int i, uint32_t parity) -> bool {
        if (*abort_flag) return false;
        if (!mbar_wait(bar(i), parity, &g_ssdm_dev_err)) {
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
                const int s = u & 1;
                if (!wait(B_EMPTY + s, (uint32_t)(((u >> 1) + 1) & 1))) break;
                const uint32_t slot = base + s * SLOT;
                const uint32_t fb = bar(B_FULL + s);
                mbar_expect_tx(fb, SLOT);
                const int t0 = u * UB;
                tma_load_4d(slot, &tm_x, fb, 0, (int)h, t0, (int)b);
                tma_load_4d(slot + X_TILE, &tm_B, fb, 0, (int)g, t0, (int)b);
                tma_load_4d(slot + X_TILE + BC_SLAB, &tm_B, fb, 64, (int)g, t0, (int)b);
                tma_load_4d(slot + X_TILE + BC_TILE, &tm_C, fb, 0, (int)g, t0, (int)b);
                tma_load_4d(slot + X_TILE + BC_TILE + BC_SLAB, &tm_C, fb, 64, (int)g, t0, (int)b);
            }
        }
    } else if (warp == W_MMA) {
        // ----------------------------------------------------------- MMA ----
        // Per block u: the carried-state read-outs Y_A, Y_V (they need the
        // states after block u-1), Y_diag (needs P), V's block-state product
        // onto the rescaled V, C.B^T of block u+1, then H's block-state product
        // (its scaled X is formed in place after Y_diag).
        if (lane == 0) {
            auto issue_cb = [&](int v) -> bool {
                const int k = v & 1;
                const uint32_t slot = base + k * SLOT;
                const uint32_t bs = slot + X_TILE, cs = slot + X_TILE + BC_TILE;
                if (!wait(B_FULL + k, (uint32_t)((v >> 1) & 1))) return false;
                if (!wait(B_TFREE + k, (uint32_t)(((v >> 1) + 1) & 1))) return false;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t koff = (ks >> 2) * BC_SLAB + (ks & 3) * 32;
                    umma_ss(tmem + tm_cb(k), umma_desc_sw128(cs + koff, 16, 1024),
                            umma_desc_sw128(bs + koff, 16, 1024), ID_CB, ks > 0);
                }
                umma_commit(bar(B_CB + k));
                return true;
            };
            bool live = nblk > 0 && issue_cb(0);
            for (int u = 0; u < nblk && live; ++u) {
                const int k = u & 1;
                const uint32_t slot = base + k * SLOT;
                const uint32_t xs = slot, bs = slot + X_TILE, cs = slot + X_TILE + BC_TILE;
                // Y_A = C . H^T and Y_V = C . V^T in one product with N = 128 (the H
                // and V operand tiles are adjacent: two 64-column groups), with the
                // states after block u-1
                if (!(live = wait(B_SREADY, (uint32_t)(u & 1)))) break;
                if (!(live = wait(B_YOFREE, (uint32_t)((u + 1) & 1)))) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t koff = (ks >> 2) * BC_SLAB + (ks & 3) * 32;
                    umma_ss(tmem + TM_YA, umma_desc_sw128(cs + koff, 16, 1024),
                            umma_desc_sw128(base + OFF_SH + ks * 2048, S_TILE, 1024), ID_YO, ks > 0);
                }
                umma_commit(bar(B_SFREE));
                // Y_diag = P(tmem) . X
                if (!(live = wait(B_M + k, (uint32_t)((u >> 1) & 1)))) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_ts(tmem + tm_cb(k), tmem + tm_cb(k) + 64 + ks * 8,
                            umma_desc_sw128(xs + ks * 2048, X_TILE, 1024), ID_YD, ks > 0);
                umma_commit(bar(B_Y + k));
                // V += B^T . (w_V o X) once the mask warps have scaled X and the
                // state warps have rescaled V for this block
                if (!(live = wait(B_XV, (uint32_t)(u & 1)))) break;
                if (!(live = wait(B_SCALED, (uint32_t)(u & 1)))) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_ss(tmem + TM_V, umma_desc_sw128(bs + ks * 2048, BC_SLAB, 1024),
                            umma_desc_sw128(base + OFF_XV + ks * 2048, X_TILE, 1024), ID_ST, 1);
                // C.B^T of block u+1, while the mask warps scale X in place for H
                if (u + 1 < nblk && !(live = issue_cb(u + 1))) break;
                // H += B^T . (w_H o X), X scaled in place once Y_diag has read it
                if (!(live = wait(B_XH, (uint32_t)(u & 1)))) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_ss(tmem + TM_H, umma_desc_sw128(bs + ks * 2048, BC_SLAB, 1024),
                            umma_desc_sw128(xs + ks * 2048, X_TILE, 1024), ID_ST, 1);
                umma_commit(bar(B_STATE));
                umma_commit(bar(B_EMPTY + k));
            }
            // Drain: the last commit must land before the CTA may exit.
            if (nblk > 0 && !*abort_flag) {
                const int u = nblk - 1;
                wait(B_EMPTY + (u & 1), (uint32_t)((u >> 1) & 1));
            }
        }
    } else if (warp < 4) {
        // ------------------------------------- mask warpgroup (warps 0-3) ----
        const int i = tid;                          // TMEM lane = row i of the block
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const float beta = p.beta;
        // Waits are warp-uniform (the TMEM accesses are warp-collective) and
        // the warps agree once per block at a named barrier, so that all of
        // them leave the loop together when any wait has given up.
        auto wwait = [&](int bi, uint32_t par) { return __all_sync(0xffffffffu, wait(bi, par)); };
        // Scale rows [r0, r1) of an X tile by the per-row weights w (16-byte chunks,
        // swizzled), four chunks per lane in flight.
        auto scale_rows = [&](const unsigned char* src, unsigned char* dst, const float* w, int r0, int r1) {
            const int units = (r1 - r0) * 8;
            for (int e0 = lane; e0 < units; e0 += 128) {
                uint4 q[4];
                float wr[4];
                int off[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int e = e0 + 32 * c;
                    const int r = r0 + (e >> 3);
                    off[c] = r * 128 + (((e & 7) ^ (r & 7)) << 4);
                    if (e < units) {
                        wr[c] = w[r];
                        q[c] = *reinterpret_cast<const uint4*>(src + off[c]);
                    }
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (e0 + 32 * c >= units) continue;
                    uint32_t w4[4] = {q[c].x, q[c].y, q[c].z, q[c].w};
#pragma unroll
                    for (int h2 = 0; h2 < 4; ++h2)
                        w4[h2] = pack_bf16x2(bf16_lo(w4[h2]) * wr[c], bf16_hi(w4[h2]) * wr[c]);
                    *reinterpret_cast<uint4*>(dst + off[c]) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
        };
        // w_V o X comes right after each warp's share of P: the warps with fewer
        // mask batches are free first and take more of its rows.
        const int v0r = warp == 0 ? 0 : warp == 1 ? 52 : warp == 2 ? 92 : 116;
        const int v1r = warp == 0 ? 52 : warp == 1 ? 92 : warp == 2 ? 116 : 128;
        unsigned char* xv = smem + OFF_XV;
        bool ok = true;
        for (int u = 0; u < nblk; ++u) {
            ok = named_bar_and(1, NG, ok);
            if (!ok) break;
            const int k = u & 1;
            const unsigned char* xs = smem + k * SLOT;
            // (c) P = M o CB o alpha delta_j (j <= i): one batch of 32 columns at a
            //     time from the diagonal batch down to batch 0, the recurrence
            //     running across batches.  Packed batch cb goes to columns
            //     64 + 16 cb, inside fp32 batches 2 and 3, which this warp has read
            //     by then (or never reads).
            bool good = wwait(B_SCAL + k, (uint32_t)((u >> 1) & 1)) && wwait(B_CB + k, (uint32_t)((u >> 1) & 1));
            tc_fence_after();
            if (good) {
                const bool fac = reinterpret_cast<volatile const int*>(smem + OFF_MODE)[k] != 0;
                const float* cs_sm = fsm(OFF_CS, k);
                const float* da_sm = fsm(OFF_DA, k);
                const float* v_sm = fac ? fsm(OFF_CF, k) : cs_sm;
                const float csi = cs_sm[i];
                float R = 0.0f;
#pragma unroll 1
                for (int cb = warp; cb >= 0; --cb) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_base + tm_cb(k) + cb * 32, r);
                    tmem_wait_ld();
                    uint32_t pk[16];
                    if (fac) {
                        if (cb == warp) mom_mask_batch<true, true>(r, pk, R, cb, i, csi, beta, v_sm, da_sm);
                        else mom_mask_batch<true, false>(r, pk, R, cb, i, csi, beta, v_sm, da_sm);
                    } else {
                        if (cb == warp) mom_mask_batch<false, true>(r, pk, R, cb, i, csi, beta, v_sm, da_sm);
                        else mom_mask_batch<false, false>(r, pk, R, cb, i, csi, beta, v_sm, da_sm);
                    }
                    tmem_st16(tmem + lane_base + tm_cb(k) + 64 + cb * 16, pk);
                }
#pragma unroll 1
                for (int cb = warp + 1; cb < 4; ++cb) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = 0u;
                    tmem_st16(tmem + lane_base + tm_cb(k) + 64 + cb * 16, pk);
                }
                // q_i = beta M_i0 (a factored block's R carries M / 2^(cs_i - ref))
                const float ref = (reinterpret_cast<const float*>(smem + OFF_BLK) + k * 4)[3];
                fsm(OFF_Q, k)[i] = beta * (fac ? ex2_approx(csi - ref) * R : R);
                tmem_wait_st();
            }
            tc_fence_before();
            if (good) mbar_arrive(bar(B_M + k));
            // (b) w_V o X into its own tile: raw X has landed and s_V of block u-1
            //     has read the tile's previous contents
            good = good && wwait(B_FULL + k, (uint32_t)((u >> 1) & 1)) &&
                   (u == 0 || wwait(B_STATE, (uint32_t)((u - 1) & 1)));
            if (good) {
                scale_rows(xs, xv, fsm(OFF_WV, k), v0r, v1r);
                fence_proxy_async_smem();
                mbar_arrive(bar(B_XV));
            }
            // (d) w_H o X in place once Y_diag has read X (32 rows per warp)
            good = good && wwait(B_Y + k, (uint32_t)((u >> 1) & 1));
            if (good) {
                scale_rows(xs, const_cast<unsigned char*>(xs), fsm(OFF_WH, k), warp * 32, warp * 32 + 32);
                fence_proxy_async_smem();
                mbar_arrive(bar(B_XH));
            }
            ok = good;
        }
    } else if (warp < 12) {
        // ------------------------- state warpgroups (warps 4-7 and 8-11) ----
        const int sg = (warp - 4) >> 2;             // head channels 32 sg .. 32 sg + 31
        const int t = tid - NG - sg * NG;           // TMEM lane: state n (update) and row i (output)
        const int wq = (warp - 4) & 3;
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        const int pc0 = sg * 32;
        const int64_t sbase = ((b * p.nheads + h) * P + pc0) * NS + t;   // h0[b, h, pc0, t]
        // The initial states into TMEM: lane t = state n, this warpgroup's 32 channels.
#pragma unroll 1
        for (int hc = 0; hc < 2; ++hc) {
            uint32_t wh[16], wv[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int64_t o = sbase + (int64_t)(hc * 16 + q) * NS;
                wh[q] = __float_as_uint(p.h0 ? p.h0[o] : 0.0f);
                wv[q] = __float_as_uint(p.v0 ? p.v0[o] : 0.0f);
            }
            tmem_st16(tmem + lane_base + TM_H + pc0 + hc * 16, wh);
            tmem_st16(tmem + lane_base + TM_V + pc0 + hc * 16, wv);
        }
        tmem_wait_st();
        // 16 channels (pc0 + 16 hc ..) of state row t as bf16 operands (MN-major, swizzled).
        auto write_S16 = [&](int hc, const uint32_t (&rh)[16], const uint32_t (&rv)[16]) {
            unsigned char* sh = smem + OFF_SH + t * 128;
            unsigned char* sv = smem + OFF_SV + t * 128;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int chunk = sg * 4 + hc * 2 + c;
                uint32_t wh[4], wv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    wh[e] = pack_bf16x2(__uint_as_float(rh[c * 8 + 2 * e]), __uint_as_float(rh[c * 8 + 2 * e + 1]));
                    wv[e] = pack_bf16x2(__uint_as_float(rv[c * 8 + 2 * e]), __uint_as_float(rv[c * 8 + 2 * e + 1]));
                }
                const int off = (chunk ^ (t & 7)) << 4;
                *reinterpret_cast<uint4*>(sh + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
                *reinterpret_cast<uint4*>(sv + off) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
        };
        // Block v's scalars (first state warpgroup only; row t of the block):
        // cs (inclusive prefix of delta A log2 e), alpha delta, 2^cs, w_V, w_H
        // (the suffix recurrence r_j = 2^(cs_l - cs_j) + beta r_{j+1} gives
        // M_lj), and per block 2^cs_l, q_l = beta M_l0, beta^(l+1).
        const float a_h = p.A[h] * kLog2e;
        const float beta = p.beta, lb = p.lb;
        float* red = reinterpret_cast<float*>(smem + OFF_RED);
        auto load_dt = [&](int v) -> float {
            const int64_t tv = (int64_t)v * UB + t;
            return tv < L ? p.delta[((b * L + tv) * p.nheads) + h] : 0.0f;
        };
        auto scan_block = [&](int v, float dt) {
            const int kv = v & 1;
            const int64_t left = L - (int64_t)v * UB;
            const int last = left >= UB ? UB - 1 : (int)left - 1;
            float cs = dt * a_h;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float o = __shfl_up_sync(0xffffffffu, cs, off);
                if (lane >= off) cs += o;
            }
            if (lane == 31) red[wq] = cs;
            named_bar_sync(2, NG);
            float prefix = 0.0f;
#pragma unroll
            for (int w = 0; w < 4; ++w)
                if (w < wq) prefix += red[w];
            cs += prefix;
            fsm(OFF_CS, kv)[t] = cs;
            named_bar_sync(2, NG);                  // every cs_t in place (red reusable)
            const float cs_l = fsm(OFF_CS, kv)[last];
            const float da = p.alpha * dt;
            // suffix recurrence over the rows j <= l, in-warp then across warps
            float r = t <= last ? ex2_approx(cs_l - cs) : 0.0f;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float o = __shfl_down_sync(0xffffffffu, r, off);
                if (lane + off < 32) r = fmaf(ex2_approx((float)off * lb), o, r);
            }
            if (lane == 0) red[4 + wq] = r;         // r at row 32 wq, this warp's rows only
            named_bar_sync(2, NG);
            float carry = 0.0f;                     // global r at row 32 (wq + 1)
            for (int w = 3; w > wq; --w) carry = fmaf(ex2_approx(32.0f * lb), carry, red[4 + w]);
            if (wq < 3) r = fmaf(ex2_approx((float)(32 - lane) * lb), carry, r);
            // factored (see FACTOR_RANGE) when every row is within range of ref = cs_l / 2
            const float ref = 0.5f * cs_l;
            const bool fac = named_bar_and(2, NG, fabsf(cs - ref) <= FACTOR_RANGE);
            fsm(OFF_DA, kv)[t] = da;
            fsm(OFF_CF, kv)[t] = fac ? ex2_approx(ref - cs) : 0.0f;
            fsm(OFF_WV, kv)[t] = t <= last ? ex2_approx((float)(last - t) * lb) * da : 0.0f;
            fsm(OFF_WH, kv)[t] = r * da;
            if (t == 0) {
                float* blk = reinterpret_cast<float*>(smem + OFF_BLK) + kv * 4;
                blk[0] = ex2_approx(cs_l);
                blk[1] = beta * r;                  // q_l = beta M_l0
                blk[2] = ex2_approx((float)(last + 1) * lb);
                blk[3] = ref;
                reinterpret_cast<volatile int*>(smem + OFF_MODE)[kv] = fac ? 1 : 0;
            }
            mbar_arrive(bar(B_SCAL + kv));
        };
        auto swait = [&](int bi, uint32_t par) { return __all_sync(0xffffffffu, wait(bi, par)); };
        float dt_next = 0.0f;
        if (sg == 0) {
            dt_next = nblk > 1 ? load_dt(1) : 0.0f;
            if (nblk > 0) scan_block(0, load_dt(0));
        }
        bool ok = true;
        for (int u = 0; u < nblk; ++u) {
            // Both state warpgroups leave together; the second has finished
            // block u-1 (its scalars and the q_i of that buffer) before the first
            // overwrites the buffer with block u+1's; and the y store of block
            // u-1 has read its stage (the H operand tile) before it is rewritten.
            ok = named_bar_and(3, 2 * NG, ok);
            if (!ok) break;
            const int k = u & 1;
            const int64_t t0 = (int64_t)u * UB;
            if (sg == 0 && u + 1 < nblk) {
                const float dt1 = dt_next;
                if (u + 2 < nblk) dt_next = load_dt(u + 2);
                // the mask warps read buffer (u+1)&1 up to their in-place scaling of block u-1
                ok = named_bar_and(2, NG, u == 0 || wait(B_XH, (uint32_t)((u - 1) & 1)));
                if (ok) scan_block(u + 1, dt1);
            }
            // (d) the states after block u-1: publish them as the bf16 operands of
            //     Y_A(u), Y_V(u) (once Y_A(u-1), Y_V(u-1) have read the previous
            //     ones), then rescale them in place for block u:
            //     H <- 2^cs_l H + q_l V, V <- beta^(l+1) V
            bool good = ok && swait(B_SCAL + k, (uint32_t)((u >> 1) & 1));
            if (u >= 1)
                good = good && swait(B_STATE, (uint32_t)((u - 1) & 1)) && swait(B_SFREE, (uint32_t)((u - 1) & 1));
            if (good) {
                tc_fence_after();
                const float* blk = reinterpret_cast<const float*>(smem + OFF_BLK) + k * 4;
                const float gam = blk[0], ql = blk[1], bnv = blk[2];
#pragma unroll 1
                for (int hc = 0; hc < 2; ++hc) {
                    uint32_t rh[16], rv[16];
                    tmem_ld16(tmem + lane_base + TM_H + pc0 + hc * 16, rh);
                    tmem_ld16(tmem + lane_base + TM_V + pc0 + hc * 16, rv);
                    tmem_wait_ld();
                    write_S16(hc, rh, rv);
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const float hv = __uint_as_float(rh[q]), vv = __uint_as_float(rv[q]);
                        rh[q] = __float_as_uint(fmaf(gam, hv, ql * vv));
                        rv[q] = __float_as_uint(bnv * vv);
                    }
                    tmem_st16(tmem + lane_base + TM_H + pc0 + hc * 16, rh);
                    tmem_st16(tmem + lane_base + TM_V + pc0 + hc * 16, rv);
                }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(bar(B_SREADY));
                mbar_arrive(bar(B_SCALED));
            }
            // (e) y = Y_diag + 2^cs_i Y_A + q_i Y_V, bf16, row t of block u, staged
            //     in the H operand tile (Y_A(u), Y_V(u) are done with it: they
            //     completed before Y_diag) in the y map's swizzled layout and
            //     written by one TMA store per block; rows past L are clipped
            good = good && swait(B_M + k, (uint32_t)((u >> 1) & 1)) && swait(B_Y + k, (uint32_t)((u >> 1) & 1));
            if (good) {
                tc_fence_after();
                // y_i = rf_i Y_diag + 2^cs_i Y_A + q_i Y_V; rf_i = 2^(cs_i - ref) on a factored block
                const float csi = fsm(OFF_CS, k)[t], qt = fsm(OFF_Q, k)[t];
                const bool fac = reinterpret_cast<volatile const int*>(smem + OFF_MODE)[k] != 0;
                const float ref = (reinterpret_cast<const float*>(smem + OFF_BLK) + k * 4)[3];
                const float et = ex2_approx(csi), rf = fac ? ex2_approx(csi - ref) : 1.0f;
                unsigned char* yst = smem + OFF_SH + t * 128;
#pragma unroll 1
                for (int hc = 0; hc < 2; ++hc) {
                    uint32_t rd[16], ra[16], rv[16];
                    tmem_ld16(tmem + lane_base + tm_cb(k) + pc0 + hc * 16, rd);
                    tmem_ld16(tmem + lane_base + TM_YA + pc0 + hc * 16, ra);
                    tmem_ld16(tmem + lane_base + TM_YV + pc0 + hc * 16, rv);
                    tmem_wait_ld();
                    uint32_t w[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float y0 = fmaf(qt, __uint_as_float(rv[2 * e]),
                                              fmaf(et, __uint_as_float(ra[2 * e]), rf * __uint_as_float(rd[2 * e])));
                        const float y1 = fmaf(qt, __uint_as_float(rv[2 * e + 1]),
                                              fmaf(et, __uint_as_float(ra[2 * e + 1]),
                                                   rf * __uint_as_float(rd[2 * e + 1])));
                        w[e] = pack_bf16x2(y0, y1);
                    }
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const int chunk = sg * 4 + hc * 2 + c;
                        *reinterpret_cast<uint4*>(yst + ((chunk ^ (t & 7)) << 4)) =
                            make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                    }
                }
                tc_fence_before();
                mbar_arrive(bar(B_TFREE + k));
                mbar_arrive(bar(B_YOFREE));
                fence_proxy_async_smem();
            }
            good = named_bar_and(4, 2 * NG, good);      // every row of the stage written
            if (good && tid == NG) {
                tma_store_4d(&tm_y, base + OFF_SH, 0, (int)h, (int)t0, (int)b);
                bulk_commit_group();
                bulk_wait_read_all();                    // the stage is free again
            }
            ok = good;
        }
        if (tid == NG) bulk_wait_all();                  // y stores complete before the CTA exits
        // the final states once the last block's products have landed
        if (ok && nblk > 0 && (p.hT || p.vT) && swait(B_STATE, (uint32_t)((nblk - 1) & 1))) {
            tc_fence_after();
#pragma unroll 1
            for (int hc = 0; hc < 2; ++hc) {
                uint32_t rh[16], rv[16];
                tmem_ld16(tmem + lane_base + TM_H + pc0 + hc * 16, rh);
                tmem_ld16(tmem + lane_base + TM_V + pc0 + hc * 16, rv);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int64_t o = sbase + (int64_t)(hc * 16 + q) * NS;
                    if (p.hT) p.hT[o] = __uint_as_float(rh[q]);
                    if (p.vT) p.vT[o] = __uint_as_float(rv[q]);
                }
            }
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

// 4-D bf16 map (d0 innermost), box (64, 1, 128, 1) with the 128-byte swizzle
// (the loads of x, B, C and the stores of y).
cudaError_t map_4d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[4] = {d0, d1, d2, d3};
    const cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
    const cuuint32_t box[4] = {64, 1, 128, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

bool ssd_mom_tc_shape_supported(int64_t headdim, int64_t dstate) {
    return headdim == ssdmt::P && dstate == ssdmt::NS;
}

cudaError_t launch_ssd_mom_tc(const SSDMomArgs& a, cudaStream_t stream) {
    if (a.batch * a.nheads > 0x7fffffffLL || a.seqlen > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    CUtensorMap mx, mB, mC, my;
    cudaError_t e;
    if ((e = map_4d(&mx, a.x, ssdmt::P, a.nheads, a.seqlen, a.batch)) != cudaSuccess) return e;
    if ((e = map_4d(&my, a.y, ssdmt::P, a.nheads, a.seqlen, a.batch)) != cudaSuccess) return e;
    if ((e = map_4d(&mB, a.B, ssdmt::NS, a.ngroups, a.seqlen, a.batch)) != cudaSuccess) return e;
    if ((e = map_4d(&mC, a.C, ssdmt::NS, a.ngroups, a.seqlen, a.batch)) != cudaSuccess) return e;
    SSDMTArgs k{};
    k.delta = a.delta; k.A = a.A; k.h0 = a.h0; k.v0 = a.v0;
    k.y = static_cast<bf16*>(a.y); k.hT = a.hT; k.vT = a.vT;
    k.batch = a.batch; k.seqlen = a.seqlen; k.nheads = a.nheads; k.ngroups = a.ngroups;
    k.nblocks = (int)((a.seqlen + ssdmt::UB - 1) / ssdmt::UB);
    k.alpha = a.alpha;
    k.beta = a.beta;
    k.lb = a.beta > 0.0f ? log2f(a.beta) : -1000.0f;
    k.stall = a.stall;
    static std::atomic<uint64_t> attr_done{0};
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_done.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(ssd_mom_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 ssdmt::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_done.fetch_or(bit, std::memory_order_release);
    }
    ssd_mom_tc_kernel<<<(unsigned)(a.batch * a.nheads), ssdmt::NTHREADS, ssdmt::SMEM_BYTES, stream>>>(mx, mB, mC, my, k);
    return cudaGetLastError();
}

unsigned int ssd_mom_tc_read_and_clear_device_error() {
    unsigned int v = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_ssdm_dev_err, sizeof(v)) != cudaSuccess) return 0;
    if (v) cudaMemcpyToSymbol(g_ssdm_dev_err, &z, sizeof(z));
    return v;
}

}  // namespace mmscan
