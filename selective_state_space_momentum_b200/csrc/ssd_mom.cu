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
// overflows) and one thread the row weights E and m; C.B^T, the masked
// product with X and the two carried-state read-outs run as register-tiled
// products over shared memory (a 16 x 16 thread grid), and the state update
// is a rank-q sum per (p, n).  This form does
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
constexpr int TQ = Q / 16;         // tile rows (steps i) and C.B^T columns (steps j) per thread
constexpr int TP = PC / 16;        // tile columns (channels p) per thread
constexpr int LDN = NMAX + 1;      // row pitch (floats) of the [*][n] arrays
constexpr int LDQ = Q + 1;         // row pitch of the [*][j] arrays
constexpr int OFF_H = 0;                        // H[p][n], this CTA's channels
constexpr int OFF_V = OFF_H + PC * LDN;         // V[p][n]
constexpr int OFF_B = OFF_V + PC * LDN;         // B[j][n]
constexpr int OFF_C = OFF_B + Q * LDN;          // C[i][n]
constexpr int OFF_XT = OFF_C + Q * LDN;         // X^T[p][j]
constexpr int OFF_L = OFF_XT + PC * LDQ;        // M, then the masked matrix L[i][j]
constexpr int OFF_VEC = OFF_L + Q * LDQ;        // per-step vectors, Q floats each
constexpr int V_AD = 0, V_A = 1, V_E = 2, V_M = 3, V_WH = 4, V_WV = 5, V_SC = 6;
constexpr int SMEM_BYTES = (OFF_VEC + 7 * Q) * 4;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
static_assert(Q % 16 == 0 && PC % 16 == 0 && Q <= NT, "tiles");

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
    const int ti = tid / 16, tj = tid % 16;    // output rows ti + 16 a, columns tj + 16 c

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
        // ---- L_ij = M_ij (C_i . B_j) alpha delta_j ----------------------------------
        {
            float acc[TQ][TQ];
#pragma unroll
            for (int a = 0; a < TQ; ++a)
#pragma unroll
                for (int c = 0; c < TQ; ++c) acc[a][c] = 0.0f;
            for (int n = 0; n < N; ++n) {
                float cv[TQ], bv[TQ];
#pragma unroll
                for (int a = 0; a < TQ; ++a) cv[a] = Cs[(ti + 16 * a) * LDN + n];
#pragma unroll
                for (int c = 0; c < TQ; ++c) bv[c] = Bs[(tj + 16 * c) * LDN + n];
#pragma unroll
                for (int a = 0; a < TQ; ++a)
#pragma unroll
                    for (int c = 0; c < TQ; ++c) acc[a][c] = __fmaf_rn(cv[a], bv[c], acc[a][c]);
            }
#pragma unroll
            for (int a = 0; a < TQ; ++a)
#pragma unroll
                for (int c = 0; c < TQ; ++c) {
                    const int i = ti + 16 * a, j = tj + 16 * c;
                    Ls[i * LDQ + j] *= acc[a][c] * vad[j];
                }
        }
        __syncthreads();
        // ---- outputs: L X + E_i C_i.H0 + m_i C_i.V0 ----------------------------------
        {
            float yd[TQ][TP], yh[TQ][TP], yv[TQ][TP];
#pragma unroll
            for (int a = 0; a < TQ; ++a)
#pragma unroll
                for (int c = 0; c < TP; ++c) yd[a][c] = yh[a][c] = yv[a][c] = 0.0f;
            for (int j = 0; j < q; ++j) {
                float lv[TQ], xv[TP];
#pragma unroll
                for (int a = 0; a < TQ; ++a) lv[a] = Ls[(ti + 16 * a) * LDQ + j];
#pragma unroll
                for (int c = 0; c < TP; ++c) xv[c] = XT[(tj + 16 * c) * LDQ + j];
#pragma unroll
                for (int a = 0; a < TQ; ++a)
#pragma unroll
                    for (int c = 0; c < TP; ++c) yd[a][c] = __fmaf_rn(lv[a], xv[c], yd[a][c]);
            }
            for (int n = 0; n < N; ++n) {
                float cv[TQ], hv[TP], vv[TP];
#pragma unroll
                for (int a = 0; a < TQ; ++a) cv[a] = Cs[(ti + 16 * a) * LDN + n];
#pragma unroll
                for (int c = 0; c < TP; ++c) {
                    hv[c] = Hs[(tj + 16 * c) * LDN + n];
                    vv[c] = Vs[(tj + 16 * c) * LDN + n];
                }
#pragma unroll
                for (int a = 0; a < TQ; ++a)
#pragma unroll
                    for (int c = 0; c < TP; ++c) {
                        yh[a][c] = __fmaf_rn(cv[a], hv[c], yh[a][c]);
                        yv[a][c] = __fmaf_rn(cv[a], vv[c], yv[a][c]);
                    }
            }
#pragma unroll
            for (int a = 0; a < TQ; ++a) {
                const int i = ti + 16 * a;
                if (i >= q) continue;
#pragma unroll
                for (int c = 0; c < TP; ++c) {
                    const int pp = tj + 16 * c;
                    if (pp >= PL) continue;
                    const float out = yd[a][c] + vE[i] * yh[a][c] + vm[i] * yv[a][c];
                    yg[((b * L + t0 + i) * H + hh) * P + pbase + pp] = __float2bfloat16_rn(out);
                }
            }
        }
        __syncthreads();            // every read of the chunk's start state is done
        // ---- the states carried out of the chunk -----------------------------------
        {
            const float eL = vE[q - 1], mL = vm[q - 1], bq = vsc[0];
            for (int e = tid; e < PL * N; e += NT) {
                const int pp = e / N, n = e - (e / N) * N;
                float sh = 0.0f, sv = 0.0f;
                for (int j = 0; j < q; ++j) {
                    const float u = XT[pp * LDQ + j] * Bs[j * LDN + n];
                    sh = __fmaf_rn(vwH[j], u, sh);
                    sv = __fmaf_rn(vwV[j], u, sv);
                }
                const float h0v = Hs[pp * LDN + n], v0v = Vs[pp * LDN + n];
                Hs[pp * LDN + n] = __fmaf_rn(eL, h0v, __fmaf_rn(mL, v0v, sh));
                Vs[pp * LDN + n] = __fmaf_rn(bq, v0v, sv);
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
