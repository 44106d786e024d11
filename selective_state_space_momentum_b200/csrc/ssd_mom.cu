// ssd_mom.cu -- sm_100a kernel for the Mamba-2 scalar-A multi-head scan with
// momentum (beta != 0) in the chunked form, on the CUDA cores.
//
// What it computes: the momentum recurrence of "Momentum Mamba: Enhanced
// State Space Models with Momentum" ("Momentum Mamba Recurrence") for the
// multi-head scalar-A layout of "Mamba-2 -- SSM = structured matrix
// multiply" ("Multi-Head Expansion"): for batch row b, head h (group g),
// head channel p, state n,
//     v_t[p, n] = beta v_{t-1}[p, n] + alpha delta_t B_t[n] x_t[p]
//     h_t[p, n] = exp(delta_t A_h) h_{t-1}[p, n] + v_t[p, n]
//     y_t[p]    = sum_n C_t[n] h_t[p, n]
// through the chunked ("4-Step Algorithm") form that momentum leads to: per
// chunk of Q steps starting from (H0, V0), with a_i = exp(delta_i A_h),
// E_i = a_0 ... a_i and w_j = alpha delta_j B_j x_j^T,
//     y_i  = sum_{j<=i} M_ij (C_i . B_j) alpha delta_j x_j + E_i C_i.H0 + m_i C_i.V0
//     M_ij = sum_{k=j}^{i} (a_{k+1} ... a_i) beta^(k-j)   = a_i M_{i-1,j} + beta^(i-j)
//     m_i  = sum_{k=0}^{i} (a_{k+1} ... a_i) beta^(k+1)   = a_i m_{i-1} + beta^(i+1)
//     H_end = E_{q-1} H0 + m_{q-1} V0 + sum_j M_{q-1,j} w_j
//     V_end = beta^q V0 + sum_j beta^(q-1-j) w_j
//
// Design.  A CTA of 256 threads per (b, h, half of the channels) keeps its
// H and V rows (fp32) in shared memory for the whole sequence and walks it
// in chunks of Q = 32 steps (two CTAs per head, each with half of the head
// channels; both form C.B^T): the chunk's B, C (fp32, row pitch N + 1) and
// X^T are staged, Q threads form the columns of M by the recursion above
// (one multiply-add a step, no exponentials of differences, so nothing
// overflows) and one thread the row weights E and m.  C.B^T and the two
// carried-state read-outs (inner dimension N) and the masked product with X
// (inner dimension q) are split over four groups of 64 threads, each a
// quarter of the inner dimension in 4 x 4 register tiles, and the partial
// sums meet in shared memory; the state update is a (p, n) product over the
// q steps with X pre-weighted by the two carry weights, in 2 x 8 tiles.  This form does
// not use the tensor cores: the masked matrix is a product of the decay
// mask and a beta-Toeplitz matrix, which the tcgen05 kernel (ssd_fwd.cu) of
// the plain recurrence does not form.
#include <cuda.h>

#include <atomic>

#include "mm_common.cuh"
#include "mm_internal.h"

namespace mmscan {
namespace ssdm {

constexpr int Q = 32;              // steps per chunk
constexpr int PSPLIT = 2;          // CTAs per head, each with PMAX / PSPLIT head channels
constexpr int PMAX = 64;           // head channels
constexpr int PC = PMAX / PSPLIT;  // head channels of one CTA
constexpr int NMAX = 128;          // states
constexpr int NT = 256;            // threads: a 16 x 16 grid of register tiles
constexpr int KQ = NMAX / 4;       // states per thread group in the split products
constexpr int LDN = NMAX + 1;      // row pitch (floats) of the [*][n] arrays
constexpr int LDQ = Q + 1;         // row pitch of the [*][j] arrays
constexpr int YPP = 40;            // row pitch of a partial-sum tile (conflict-free 8 x 4 writes)
constexpr int YPB = Q * YPP;       // floats of one group's partial-sum tile
constexpr int OFF_H = 0;                        // H[p][n], this CTA's channels
constexpr int OFF_V = OFF_H + PC * LDN;         // V[p][n]
constexpr int OFF_B = OFF_V + PC * LDN;         // B[j][n]
constexpr int OFF_C = OFF_B + Q * LDN;          // C[i][n]
constexpr int OFF_XT = OFF_C + Q * LDN;         // X^T[p][j]
constexpr int OFF_XH = OFF_XT + PC * LDQ;       // M_{q-1,j} alpha delta_j X^T[p][j]
constexpr int OFF_XV = OFF_XH + PC * LDQ;       // beta^(q-1-j) alpha delta_j X^T[p][j]
constexpr int OFF_L = OFF_XV + PC * LDQ;        // M, then the masked matrix L[i][j]
constexpr int OFF_YP = OFF_L + Q * LDQ;         // four groups' partial sums
constexpr int OFF_VEC = OFF_YP + 4 * YPB;       // per-step vectors, Q floats each
constexpr int V_AD = 0, V_A = 1, V_E = 2, V_M = 3, V_WH = 4, V_WV = 5, V_SC = 6;
constexpr int SMEM_BYTES = (OFF_VEC + 7 * Q) * 4;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
static_assert(Q == 32 && PC == 32 && NT == 256 && NMAX % 4 == 0, "the 8 x 8 x 4 and 16 x 16 thread tilings");

}  // namespace ssdm

__global__ void __launch_bounds__(ssdm::NT, 2) ssd_mom_kernel(const SSDMomArgs p) {
    using namespace ssdm;
    extern __shared__ float sm[];
    float* Hs = sm + OFF_H;
    float* Vs = sm + OFF_V;
    float* Bs = sm + OFF_B;
    float* Cs = sm + OFF_C;
    float* XT = sm + OFF_XT;
    float* Ls = sm + OFF_L;
    float* XH = sm + OFF_XH;
    float* XV = sm + OFF_XV;
    float* YP = sm + OFF_YP;
    float* vad = sm + OFF_VEC + V_AD * Q;     // alpha delta_j
    float* va = sm + OFF_VEC + V_A * Q;       // a_i = exp(delta_i A_h)
    float* vE = sm + OFF_VEC + V_E * Q;       // E_i = a_0 ... a_i
    float* vm = sm + OFF_VEC + V_M * Q;       // m_i
    float* vwH = sm + OFF_VEC + V_WH * Q;     // M_{q-1, j} alpha delta_j
    float* vwV = sm + OFF_VEC + V_WV * Q;     // beta^(q-1-j) alpha delta_j
    float* vsc = sm + OFF_VEC + V_SC * Q;     // [0] = beta^q

    const int tid = threadIdx.x;
    const int H = (int)p.nheads, P = (int)p.headdim, N = (int)p.dstate, G = (int)p.ngroups;
    const int64_t b = blockIdx.x / (H * PSPLIT);
    const int hh = (int)((blockIdx.x / PSPLIT) % H);
    const int pbase = (int)(blockIdx.x % PSPLIT) * PC;   // this CTA's first head channel
    const int g = hh / (H / G);
    const int64_t L = p.seqlen;
    const float a2 = p.A[hh] * kLog2e;
    const float beta = p.beta, alpha = p.alpha;
    const bf16* xg = static_cast<const bf16*>(p.x);
    const bf16* Bg = static_cast<const bf16*>(p.B);
    const bf16* Cg = static_cast<const bf16*>(p.C);
    bf16* yg = static_cast<bf16*>(p.y);
    const int64_t srow = (b * H + hh) * P + pbase;     // first state row of this CTA
    const int PL = P - pbase < PC ? P - pbase : PC;     // channels this CTA computes

    for (int e = tid; e < PC * NMAX; e += NT) {
        const int pp = e / NMAX, n = e - (e / NMAX) * NMAX;
        float hv = 0.0f, vv = 0.0f;
        if (pp < PL && n < N) {
            const int64_t si = (srow + pp) * N + n;
            if (p.h0) hv = p.h0[si];
            if (p.v0) vv = p.v0[si];
        }
        Hs[pp * LDN + n] = hv;
        Vs[pp * LDN + n] = vv;
    }
    // split products: group gq (a quarter of the states, or of the steps j) and
    // its 8 x 8 thread grid of 4 x 4 tiles, rows gi + 8 a, columns gj + 8 c
    const int gq = tid / 64, gi = (tid % 64) / 8, gj = tid % 8;

    for (int64_t t0 = 0; t0 < L; t0 += Q) {
        const int q = (int)((L - t0) < Q ? (L - t0) : Q);
        __syncthreads();            // the previous chunk is done with every buffer
        // ---- stage the chunk --------------------------------------------------
        for (int e = tid; e < Q * NMAX; e += NT) {
            const int i = e / NMAX, n = e - (e / NMAX) * NMAX;
            float bv = 0.0f, cv = 0.0f;
            if (i < q && n < N) {
                const int64_t idx = ((b * L + t0 + i) * G + g) * N + n;
                bv = __bfloat162float(Bg[idx]);
                cv = __bfloat162float(Cg[idx]);
            }
            Bs[i * LDN + n] = bv;
            Cs[i * LDN + n] = cv;
        }
        for (int e = tid; e < Q * PC; e += NT) {
            const int i = e / PC, pp = e - (e / PC) * PC;
            float xv = 0.0f;
            if (i < q && pp < PL) xv = __bfloat162float(xg[((b * L + t0 + i) * H + hh) * P + pbase + pp]);
            XT[pp * LDQ + i] = xv;
        }
        if (tid < Q) {
            const float dl = tid < q ? p.delta[(b * L + t0 + tid) * H + hh] : 0.0f;
            vad[tid] = alpha * dl;
            va[tid] = ex2_approx(dl * a2);
        }
        __syncthreads();
        // ---- the mask M (column j on thread j) and the row weights E, m ----------
        if (tid < Q) {
            const int j = tid;
            float M = 0.0f, bp = 1.0f;
            for (int i = 0; i < Q; ++i) {
                if (i == j) {
                    M = 1.0f;
                } else if (i > j) {
                    bp *= beta;                       // beta^(i-j)
                    M = __fmaf_rn(va[i], M, bp);
                }
                Ls[i * LDQ + j] = (i >= j && i < q) ? M : 0.0f;
                if (i == q - 1) {
                    vwH[j] = j < q ? M * vad[j] : 0.0f;
                    vwV[j] = j < q ? bp * vad[j] : 0.0f;
                }
            }
        } else if (tid == Q) {
            float E = 1.0f, m = 0.0f, bpow = 1.0f;
            for (int i = 0; i < Q; ++i) {
                bpow *= beta;                         // beta^(i+1)
                E *= va[i];
                m = __fmaf_rn(va[i], m, bpow);
                vE[i] = E;
                vm[i] = m;
                if (i == q - 1) vsc[0] = bpow;
            }
        }
        __syncthreads();
        // ---- L_ij = M_ij (C_i . B_j) alpha delta_j: four groups of 64 threads each
        // take a quarter of the states (4 x 4 tiles), partial sums meet in YP ----
        {
#pragma unroll
            for (int r = 0; r < (PC * Q) / NT; ++r) {         // weighted X for the state update
                const int e = tid + NT * r;
                const int pp = e / Q, jj = e - (e / Q) * Q;
                XH[pp * LDQ + jj] = vwH[jj] * XT[pp * LDQ + jj];
                XV[pp * LDQ + jj] = vwV[jj] * XT[pp * LDQ + jj];
            }
            float acc[4][4];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[a][c] = 0.0f;
            for (int n = gq * KQ; n < gq * KQ + KQ; ++n) {
                float cv[4], bv[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) cv[a] = Cs[(gi + 8 * a) * LDN + n];
#pragma unroll
                for (int c = 0; c < 4; ++c) bv[c] = Bs[(gj + 8 * c) * LDN + n];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 4; ++c) acc[a][c] = __fmaf_rn(cv[a], bv[c], acc[a][c]);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) YP[gq * YPB + (gi + 8 * a) * YPP + gj + 8 * c] = acc[a][c];
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < (Q * Q) / NT; ++r) {
            const int e = tid + NT * r;
            const int i = e / Q, jj = e - (e / Q) * Q;
            const int o = i * YPP + jj;
            const float cb = YP[o] + YP[YPB + o] + YP[2 * YPB + o] + YP[3 * YPB + o];
            Ls[i * LDQ + jj] *= cb * vad[jj];                   // M is 0 above the diagonal and past q
        }
        __syncthreads();
        // ---- outputs: L X + E_i C_i.H0 + m_i C_i.V0, split the same way ------------
        {
            float yd[4][4], yh[4][4], yv[4][4];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) yd[a][c] = yh[a][c] = yv[a][c] = 0.0f;
            for (int jj = gq * (Q / 4); jj < gq * (Q / 4) + Q / 4; ++jj) {
                float lv[4], xv[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) lv[a] = Ls[(gi + 8 * a) * LDQ + jj];
#pragma unroll
                for (int c = 0; c < 4; ++c) xv[c] = XT[(gj + 8 * c) * LDQ + jj];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 4; ++c) yd[a][c] = __fmaf_rn(lv[a], xv[c], yd[a][c]);
            }
            for (int n = gq * KQ; n < gq * KQ + KQ; ++n) {
                float cv[4], hv[4], vv[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) cv[a] = Cs[(gi + 8 * a) * LDN + n];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    hv[c] = Hs[(gj + 8 * c) * LDN + n];
                    vv[c] = Vs[(gj + 8 * c) * LDN + n];
                }
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        yh[a][c] = __fmaf_rn(cv[a], hv[c], yh[a][c]);
                        yv[a][c] = __fmaf_rn(cv[a], vv[c], yv[a][c]);
                    }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int i = gi + 8 * a;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    YP[gq * YPB + i * YPP + gj + 8 * c] = yd[a][c] + vE[i] * yh[a][c] + vm[i] * yv[a][c];
            }
        }
        __syncthreads();            // every read of the chunk's start state is done
        // ---- y, and the states carried out of the chunk ------------------------------
#pragma unroll
        for (int r = 0; r < (Q * PC) / NT; ++r) {
            const int e = tid + NT * r;
            const int i = e / PC, pp = e - (e / PC) * PC;
            const int o = i * YPP + pp;
            if (i < q && pp < PL) {
                const float out = YP[o] + YP[YPB + o] + YP[2 * YPB + o] + YP[3 * YPB + o];
                yg[((b * L + t0 + i) * H + hh) * P + pbase + pp] = __float2bfloat16_rn(out);
            }
        }
        {
            // H <- E_{q-1} H + m_{q-1} V + (wH o X)^T B,  V <- beta^q V + (wV o X)^T B:
            // 2 x 8 tiles, rows p = sp + 16 r, columns n = sn + 16 c
            const int sp = tid / 16, sn = tid % 16;
            float ah[2][8], av[2][8];
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int c = 0; c < 8; ++c) ah[r][c] = av[r][c] = 0.0f;
            for (int jj = 0; jj < q; ++jj) {
                float xh[2], xv[2], bv[8];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    xh[r] = XH[(sp + 16 * r) * LDQ + jj];
                    xv[r] = XV[(sp + 16 * r) * LDQ + jj];
                }
#pragma unroll
                for (int c = 0; c < 8; ++c) bv[c] = Bs[jj * LDN + sn + 16 * c];
#pragma unroll
                for (int r = 0; r < 2; ++r)
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        ah[r][c] = __fmaf_rn(xh[r], bv[c], ah[r][c]);
                        av[r][c] = __fmaf_rn(xv[r], bv[c], av[r][c]);
                    }
            }
            const float eL = vE[q - 1], mL = vm[q - 1], bq = vsc[0];
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int o = (sp + 16 * r) * LDN + sn + 16 * c;
                    const float h0v = Hs[o], v0v = Vs[o];
                    Hs[o] = __fmaf_rn(eL, h0v, __fmaf_rn(mL, v0v, ah[r][c]));
                    Vs[o] = __fmaf_rn(bq, v0v, av[r][c]);
                }
        }
    }
    __syncthreads();
    for (int e = tid; e < PL * N; e += NT) {
        const int pp = e / N, n = e - (e / N) * N;
        const int64_t si = (srow + pp) * N + n;
        if (p.hT) p.hT[si] = Hs[pp * LDN + n];
        if (p.vT) p.vT[si] = Vs[pp * LDN + n];
    }
}

bool ssd_mom_shape_supported(int64_t headdim, int64_t dstate) {
    return headdim >= 1 && headdim <= ssdm::PMAX && dstate >= 1 && dstate <= ssdm::NMAX;
}

cudaError_t launch_ssd_mom(const SSDMomArgs& a, cudaStream_t s) {
    // The dynamic shared-memory limit is raised once per device.
    static std::atomic<uint64_t> attr_done{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_done.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(ssd_mom_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ssdm::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_done.fetch_or(bit, std::memory_order_release);
    }
    const int64_t grid = a.batch * a.nheads * ssdm::PSPLIT;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    ssd_mom_kernel<<<(unsigned)grid, ssdm::NT, ssdm::SMEM_BYTES, s>>>(a);
    return cudaGetLastError();
}

}  // namespace mmscan
