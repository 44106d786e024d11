/*
 * mm_scan.h -- C ABI of libmmscan.so: the forward selective scan of Mamba-1
 * with the Momentum Mamba extension, and its Mamba-2 scalar-A chunked (SSD)
 * form, on NVIDIA B200 (sm_100a).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named as device buffers must be CUDA device (or managed) memory
 *   of the current device; the caller allocates and owns every buffer.  The
 *   library's only device memory of its own is the stream-ordered record
 *   memory of mm_scan_fwd's sequence-split path (a pool per device, see
 *   mm_scan_fwd), the workspace of the deterministic backward (another pool
 *   per device, see mm_scan_set_deterministic; only when switched on) and
 *   the fixed array of mm_scan_fwd_noalloc; it keeps no
 *   other state between calls except a per-thread copy of the last error
 *   message (mm_last_error), the process-wide tuning switches
 *   (mm_scan_set_tile, mm_scan_set_path, mm_scan_set_deterministic) and the
 *   per-thread side streams of
 *   the *_host entry points, which take host buffers and a device workspace.
 * - Every base pointer of a device buffer must be 16-byte aligned
 *   (MM_ERR_ALIGN otherwise).
 *   Tensors are dense and contiguous in the stated layout, last index
 *   fastest.
 * - All argument checks run on the host before anything is launched; a call
 *   that returns an error has launched nothing and touched no buffer.
 * - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is the
 *   legacy default stream) and runs asynchronously: the call returns once
 *   the kernels are queued.  Faults during execution surface at the caller's
 *   next synchronisation with that stream, as for any CUDA kernel.
 * - Calls on different streams that write the same output buffers race.
 */
#ifndef MM_SCAN_H
#define MM_SCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MM_OK = 0,
    MM_ERR_NULL = 1,           /* a required pointer is NULL                      */
    MM_ERR_DIMS = 2,           /* a size is < 1, or sizes are inconsistent         */
    MM_ERR_SCALAR = 3,         /* beta outside [0, 1), alpha < 0, or non-finite    */
    MM_ERR_DTYPE = 4,          /* unknown storage type code                        */
    MM_ERR_ALIGN = 5,          /* a base pointer is not 16-byte aligned            */
    MM_ERR_UNSUPPORTED = 6,    /* valid request outside what this build supports   */
    MM_ERR_CUDA = 7,           /* a CUDA runtime call or a launch failed           */
    MM_ERR_DEVICE_TIMEOUT = 8, /* a bounded device-side wait gave up               */
    MM_ERR_ALIAS = 9           /* an output overlaps an input it may not overlap   */
} mm_status;

/* Storage type of the streamed tensors (x, delta, B, C, y). */
typedef enum { MM_F32 = 0, MM_BF16 = 1 } mm_dtype;

/* Steps between two checkpoints of the forward's state (see mm_scan_bwd). */
#define MM_SCAN_CKPT_STEPS 16

/* Sizes of one Mamba-1 scan call. */
typedef struct {
    int64_t batch;   /* b: independent sequences                          */
    int64_t seqlen;  /* L: time steps                                      */
    int64_t dim;     /* D: channels (d_inner)                              */
    int64_t dstate;  /* N: states per channel, 1..16                       */
    int32_t io;      /* mm_dtype of x, delta, B, C and y                   */
} mm_scan_dims;

/*
 * mm_scan_fwd -- momentum selective scan, forward.
 *
 * Computes, for every batch row b, channel d and state n
 * ("Momentum Mamba: Enhanced State Space Models with Momentum", sections
 * "Momentum Mamba Recurrence" and "Discretization Note"):
 *
 *     v_t = beta * v_{t-1} + alpha * delta_t * B_t[n] * x_t
 *     h_t = exp(delta_t * A[d,n]) * h_{t-1} + v_t
 *     y_t = sum_n C_t[n] * h_t[n]
 *
 * beta = 0, alpha = 1 is the plain Mamba scan (same page, "Hyperparameters").
 * This is the core of the page's `selective_scan_fn` (section
 * "selective_scan_fn") with D = z = delta_bias = None and
 * delta_softplus = False: delta is taken as given, already positive.
 *
 * Arguments (device buffers unless noted):
 *   x      (batch, dim, L)     io     input u
 *   delta  (batch, dim, L)     io     step size
 *   A      (dim, dstate)       fp32   state matrix (any finite values)
 *   B, C   (batch, dstate, L)  io     input / output projections, shared
 *                                      by all channels of a batch row
 *   h0, v0 (batch, dim, dstate) fp32  initial hidden state / velocity, or
 *                                      NULL for zero (the page initialises
 *                                      the velocity to zero)
 *   beta   host scalar in [0, 1)      momentum decay
 *   alpha  host scalar, finite, >= 0  momentum scale
 *   y      (batch, dim, L)     io     output, rounded to nearest-even for bf16
 *   hT, vT (batch, dim, dstate) fp32  final h_{L-1} and v_{L-1}, or NULL to
 *                                      skip ("return_last_state")
 *   dims   host struct of sizes; stream: cudaStream_t or NULL
 *
 * Arithmetic is fp32 with the state held in registers.  exp is evaluated
 * as a base-2 exponential of delta * (A * log2 e).
 *
 * Aliasing: hT may be the same buffer as h0 and vT the same as v0 (in-place
 * streaming: every lane reads its initial state before writing its final
 * one); no other overlap between outputs and inputs is allowed
 * (MM_ERR_ALIAS).
 *
 * Two execution paths, chosen from (batch * dim, dstate, io) and from
 * whether L exceeds one segment of the sequence-split path:
 *   - register-resident: every (channel, state) lane walks the whole
 *     sequence in time order with its state in registers;
 *   - sequence-split (few channels, dstate 9..16, fp32, rows of a whole
 *     number of 16-byte pieces, L > S): the sequence is cut into segments of S
 *     steps (S a power of two, mm_scan_segment_len) at absolute multiples of
 *     S, each run from a zero state on its own CTA, and joined by folding
 *     each segment's 2x2 affine carry map onto the concrete carry in segment
 *     order ("Forward Pass: Two-Stage Parallel Scan" of the same page, with
 *     the chunk carry [[beta^S, 0], [Q, P]] per lane); y gets the response to
 *     each segment's carry-in until that response is below 2^-25 of its start
 *     (when A <= 0 and delta >= 0), else over the whole segment.  It runs as
 *     two launches on `stream` -- the segments' main passes, their maps
 *     written to records, then the folds and corrections -- with the records
 *     (ceil(L / S) * batch * ceil(dim / 16) * 4112 bytes, 4.2 MB for one row
 *     of 2048 channels and 131072 steps) in stream-ordered memory from a
 *     pool the library creates per device on first use and keeps (up to
 *     64 MiB reserved between calls; cudaMallocFromPoolAsync, cudaFreeAsync
 *     on `stream`).  When that memory cannot be had (or records would pass
 *     1 GiB), for in-place streaming (hT = h0 or vT = v0), and while `stream`
 *     is being captured into a CUDA graph (nothing is allocated then), it
 *     runs as one launch whose segments exchange their maps through
 *     distributed shared memory; both forms give bit-identical results.  mm_scan_fwd_noalloc
 *     allocates nothing.
 *
 * Streaming: for a fixed (batch, dim, dstate, io), calling with the first
 * L1 steps and then with the remaining steps, passing (hT, vT) of the first
 * call as (h0, v0) of the second, gives final states bit-identical to one
 * call over all steps, and the same y within rounding, when all three calls
 * take the same path and L1 is a multiple of S (sequence-split path: S is
 * the mm_scan_segment_len() of the calls), of 32 (register-resident time
 * split, mm_scan_set_tile with two time lanes), or any L1 (register-resident
 * path with one time lane, which applies the steps in order).  The path of
 * each call is what mm_scan_segment_len() reports for its sizes (0: the
 * register-resident path); mm_scan_set_path pins it.
 *
 * Errors: MM_ERR_NULL (x, delta, A, B, C, y or dims NULL), MM_ERR_DIMS
 * (a size < 1), MM_ERR_UNSUPPORTED (dstate > 16,
 * seqlen > 2^30, batch or dim >= 2^31), MM_ERR_DTYPE,
 * MM_ERR_SCALAR, MM_ERR_ALIGN, MM_ERR_ALIAS, MM_ERR_CUDA (launch failure;
 * mm_last_error has CUDA's message).
 */
mm_status mm_scan_fwd(const void *x, const void *delta, const float *A,
                      const void *B, const void *C,
                      const float *h0, const float *v0,
                      float beta, float alpha,
                      void *y, float *hT, float *vT,
                      const mm_scan_dims *dims, void *stream);

/*
 * mm_scan_fwd_gated -- the full selective_scan_fn forward: mm_scan_fwd plus
 * the optional arguments the Momentum Mamba README lists for
 * "selective_scan_fn" (D, z, delta_bias, delta_softplus), with the gate
 * after the scan as in "Mamba: Choosing What to Remember Based on the
 * Input", section "Where the state computation sits in a Mamba block":
 *
 *   delta'_t = delta_t + delta_bias[d]            (delta_bias NULL: + 0)
 *   delta'_t = ln(1 + exp(delta'_t))              (delta_softplus != 0)
 *   the recurrence of mm_scan_fwd with delta'
 *   out_t    = y_t + D[d] * x_t                   (D NULL: + 0)
 *   out_t    = out_t * z_t * sigmoid(z_t)         (z NULL: no gate)
 *
 * and y receives out.  D, delta_bias: (dim) fp32; z: (batch, dim, L) in the
 * io dtype; each may be NULL (with delta_softplus = 0 and all three NULL
 * this is mm_scan_fwd).  hT, vT are the recurrence's final states.  Same
 * layouts, alignment (16 bytes for every given pointer), aliasing rules (y
 * may overlap no input, z, D and delta_bias included), streaming property
 * and errors as mm_scan_fwd.  delta' is computed once per (batch, channel,
 * step) in fp32 from the loaded delta; the gate uses a fast exponential.
 *
 *   ckpt   (batch, dim, ceil(L / 16), 2, dstate) fp32, or NULL: for every
 *          block i of MM_SCAN_CKPT_STEPS = 16 steps, (h, v) after its last
 *          step (step min(16 i + 15, L - 1)); [.., 0, :] holds h and
 *          [.., 1, :] holds v.  This is what mm_scan_bwd restarts from.  Size
 *          in bytes: mm_scan_ckpt_size (L * batch * dim * dstate / 2 for L a
 *          multiple of 16).  It may overlap no other argument.
 */
mm_status mm_scan_fwd_gated(const void *x, const void *delta, const float *A,
                            const void *B, const void *C,
                            const float *D, const void *z,
                            const float *delta_bias, int delta_softplus,
                            const float *h0, const float *v0,
                            float beta, float alpha,
                            void *y, float *hT, float *vT, float *ckpt,
                            const mm_scan_dims *dims, void *stream);

/* mm_scan_ckpt_size -- bytes of the checkpoint buffer of mm_scan_fwd_gated
 * and mm_scan_bwd: batch * dim * ceil(seqlen / 16) * 2 * dstate * 4.
 * Errors as the size checks of mm_scan_fwd. */
mm_status mm_scan_ckpt_size(const mm_scan_dims *dims, size_t *bytes);

/*
 * mm_scan_bwd -- gradients of mm_scan_fwd ("Momentum Mamba: Enhanced State
 * Space Models with Momentum", sections "Gradient Flow" and "Backward Pass:
 * Reconstructed Forward + Reverse Scans").  The page's printed recursions
 * use one symbol for both state gradients and omit a term; the ones used
 * here follow from the recurrence.  Per (b, d, n), with G_t = dL/dh_t and
 * P_t = dL/dv_t:
 *
 *   G_t = dy_t C_t[n] + a_{t+1} G_{t+1}      (G after the last step: dhT)
 *   P_t = G_t + beta P_{t+1}                 (P after the last step: dvT)
 *   dx_t     = alpha delta_t sum_n B_t[n] P_t[n]
 *   ddelta_t = alpha x_t sum_n B_t[n] P_t[n] + sum_n A[d,n] a_t h_{t-1}[n] G_t[n]
 *   dA[d,n]  = sum over b, t of delta_t a_t h_{t-1}[n] G_t[n]
 *   dB_t[n]  = sum over d of alpha delta_t x_t P_t[n]   (per batch row)
 *   dC_t[n]  = sum over d of dy_t h_t[n]                (per batch row)
 *   dh0 = a_0 G_0,  dv0 = beta P_0,     a_t = exp(delta_t A[d,n])
 *
 * Inputs: x, delta, A, B, C, h0, v0, beta, alpha and dims exactly as given
 * to the forward; ckpt as mm_scan_fwd_gated wrote it for those inputs (it
 * may be NULL when seqlen <= 16); dy (batch, dim, L) io: the gradient
 * reaching y; dhT, dvT (batch, dim, dstate) fp32: the gradients reaching
 * hT, vT, or NULL for zero.
 * Outputs (overwritten): dx, ddelta (batch, dim, L) io (rounded to nearest
 * even for bf16); dA (dim, dstate), dB, dC (batch, dstate, L) fp32 (sums:
 * by default added atomically across CTAs, in no fixed order, so they can
 * differ in the last bits between runs; after mm_scan_set_deterministic(1)
 * summed in a fixed order and bit-identical between runs); dh0, dv0
 * (batch, dim, dstate) fp32 or NULL.
 * No output may overlap an input or another output (MM_ERR_ALIAS); every
 * pointer must be 16-byte aligned.
 *
 * Work: the kernel restarts every 16-step block from its checkpoint,
 * rebuilds the block's states once and walks them back (forming each
 * exponential a second time there): one forward pass and one reverse pass
 * of arithmetic.
 *
 * Errors: MM_ERR_NULL (a required pointer, or ckpt with seqlen > 16),
 * MM_ERR_DIMS, MM_ERR_UNSUPPORTED (dstate > 16,
 * seqlen > 2^30, batch or dim >= 2^31), MM_ERR_DTYPE,
 * MM_ERR_SCALAR, MM_ERR_ALIGN, MM_ERR_ALIAS, MM_ERR_CUDA.
 */
mm_status mm_scan_bwd(const void *x, const void *delta, const float *A,
                      const void *B, const void *C,
                      const float *h0, const float *v0, float beta, float alpha,
                      const float *ckpt, const void *dy,
                      const float *dhT, const float *dvT,
                      void *dx, void *ddelta, float *dA, float *dB, float *dC,
                      float *dh0, float *dv0,
                      const mm_scan_dims *dims, void *stream);

/*
 * mm_scan_bwd_gated -- gradients of mm_scan_fwd_gated: mm_scan_bwd through
 * the extras, with dy now the gradient reaching the gated output.  With
 * o_t = y_t + D x_t and s_t = sigmoid(z_t), delta'_t = softplus(delta_t +
 * bias):
 *
 *   the scan's read-out receives dy_t z_t s_t (dy_t without the gate);
 *   dx_t     += D dy_t z_t s_t                     (the skip)
 *   dz_t      = dy_t o_t s_t (1 + z_t (1 - s_t))
 *   dD        = sum over b, t of dy_t z_t s_t x_t
 *   ddelta_t  = (ddelta'_t of mm_scan_bwd) * sigmoid(delta_t + bias)  (softplus;
 *               else ddelta'_t),   ddelta_bias = sum over b, t of ddelta_t
 *
 * Inputs as given to mm_scan_fwd_gated (ckpt as it wrote it).  Extra
 * outputs (overwritten; NULL: not formed): dD, ddelta_bias (dim) fp32,
 * summed with atomics like dA; dz (batch, dim, L) io.  Aliasing, alignment
 * and errors as mm_scan_bwd; with D, z, delta_bias NULL and delta_softplus
 * 0 this is mm_scan_bwd.
 */
mm_status mm_scan_bwd_gated(const void *x, const void *delta, const float *A,
                            const void *B, const void *C,
                            const float *D, const void *z,
                            const float *delta_bias, int delta_softplus,
                            const float *h0, const float *v0, float beta, float alpha,
                            const float *ckpt, const void *dy,
                            const float *dhT, const float *dvT,
                            void *dx, void *ddelta, float *dA, float *dB, float *dC,
                            float *dD, void *dz, float *ddelta_bias,
                            float *dh0, float *dv0,
                            const mm_scan_dims *dims, void *stream);

/*
 * mm_scan_step -- one decode step on cached states, updated in place: the
 * Mamba module's step() ("Momentum Mamba: Enhanced State Space Models with
 * Momentum", section "Mamba Module": ssm_state and velocity_state carried
 * from call to call) for the scan part of a layer.  It is mm_scan_fwd_gated
 * with seqlen 1, (h0, v0) = (hT, vT) = (h, v):
 *
 *   delta' = softplus(delta + delta_bias)   (each part optional, as there)
 *   v = beta v + alpha delta' B[n] x,   h = exp(delta' A[d,n]) h + v
 *   y = (sum_n C[n] h + D[d] x) * z * sigmoid(z)
 *
 *   x, delta, z, y (batch, dim) io; B, C (batch, dstate) io; A (dim, dstate),
 *   D, delta_bias (dim) fp32 (D, z, delta_bias may be NULL); h, v (batch,
 *   dim, dstate) fp32, read and overwritten.  dims->seqlen must be 1.
 *
 * The per-state operations are those of mm_scan_fwd in the same order, so L
 * steps leave (h, v) bit-identical to one mm_scan_fwd_gated call over the L
 * steps from the same start (y agrees within rounding of the read-out).
 * No output (h, v, y) may overlap an input or another output.
 *
 * Errors: MM_ERR_NULL, MM_ERR_DIMS (a size < 1 or seqlen != 1),
 * MM_ERR_UNSUPPORTED (dstate > 16,
 * seqlen > 2^30, batch or dim >= 2^31), MM_ERR_DTYPE, MM_ERR_SCALAR,
 * MM_ERR_ALIGN, MM_ERR_ALIAS, MM_ERR_CUDA.
 */
mm_status mm_scan_step(const void *x, const void *delta, const float *A,
                       const void *B, const void *C,
                       const float *D, const void *z,
                       const float *delta_bias, int delta_softplus,
                       float *h, float *v, float beta, float alpha, void *y,
                       const mm_scan_dims *dims, void *stream);

/* Sizes of one Mamba-2 SSD call. */
typedef struct {
    int64_t batch;    /* b                                                  */
    int64_t seqlen;   /* L                                                  */
    int64_t nheads;   /* H                                                  */
    int64_t headdim;  /* P (the page's head dimension, 64 in its example)   */
    int64_t dstate;   /* N                                                  */
    int64_t ngroups;  /* G: B/C groups; head h reads group h / (H / G)      */
    int64_t chunk;    /* Q: chunk length of the 4-step algorithm            */
} mm_ssd_dims;

/*
 * mm_ssd_fwd -- Mamba-2 scalar-A multi-head scan through the chunked (SSD)
 * algorithm ("Mamba-2 -- SSM = structured matrix multiply", sections
 * "4-Step Algorithm" and "Multi-Head Expansion"; first-order
 * discretization B_bar = delta * B as in the Momentum Mamba page).
 *
 * For every batch row b, head h, head channel p and state n:
 *     h_t[p, n] = exp(delta_t[h] * A[h]) * h_{t-1}[p, n]
 *                 + alpha * delta_t[h] * B_t[g(h), n] * x_t[h, p]
 *     y_t[h, p] = sum_n C_t[g(h), n] * h_t[p, n]
 * computed per chunk of Q steps as: intra-chunk products C B^T masked by
 * the decay, the chunk's own final state, a scan of the states across
 * chunks, and the read-out of the carried state (tensor-core GEMMs for the
 * three dense steps).
 *
 * The kernel keeps the state of a (batch row, head) on one SM and walks the
 * sequence in blocks of 128 rows: each block's diagonal 128 x 128 part of
 * the masked decay matrix is formed densely; for chunk = 256 the
 * off-diagonal block of a chunk is applied through its rank-N factors
 * (the block state), the structured-matrix property the page describes.
 * Results equal the chunked recurrence up to rounding.
 *
 * Arguments (device buffers unless noted):
 *   x      (batch, L, H, P)  bf16   input
 *   delta  (batch, L, H)     fp32   step size per head
 *   A      (H)               fp32   one decay rate per head
 *   B, C   (batch, L, G, N)  bf16
 *   h0     (batch, H, P, N)  fp32   initial state or NULL (zero)
 *   beta   in [0, 1); beta != 0 runs mm_ssd_fwd_momentum with v0 = 0
 *          (the final velocity is not returned)
 *   alpha  finite, >= 0
 *   y      (batch, L, H, P)  bf16   output (round to nearest-even)
 *   hT     (batch, H, P, N)  fp32   final state or NULL; may equal h0
 * Supported sizes: headdim 64, dstate 128, chunk 128 or 256, seqlen from
 * 1 to 2^30, batch * H < 2^31, H a multiple of G.  All of x, B, C must be 16-byte aligned.
 * Errors: as mm_scan_fwd; MM_ERR_DIMS for sizes < 1 or H not a multiple
 * of G; MM_ERR_UNSUPPORTED for other headdim, dstate or chunk values.
 */
mm_status mm_ssd_fwd(const void *x, const float *delta, const float *A,
                     const void *B, const void *C, const float *h0,
                     float beta, float alpha,
                     void *y, float *hT,
                     const mm_ssd_dims *dims, void *stream);

/*
 * mm_ssd_fwd_momentum -- the same multi-head scalar-A scan with the
 * Momentum Mamba velocity ("Momentum Mamba Recurrence"):
 *     v_t[p, n] = beta v_{t-1}[p, n] + alpha delta_t[h] B_t[g(h), n] x_t[h, p]
 *     h_t[p, n] = exp(delta_t[h] A[h]) h_{t-1}[p, n] + v_t[p, n]
 *     y_t[h, p] = sum_n C_t[g(h), n] h_t[p, n]
 * in the chunked form momentum leads to (the mask is
 * M_ij = sum_{k=j}^{i} exp(cs_i - cs_k) beta^(k-j), and each chunk carries
 * both h and v).  Layouts as mm_ssd_fwd; v0, vT like h0, hT (NULL: zero /
 * not written; vT may equal v0 and hT h0).  headdim <= 64, dstate <= 128;
 * dims->chunk is not used (any value >= 1).  headdim 64 with dstate 128
 * runs on the tensor cores (tcgen05, blocks of 128 steps); other sizes on
 * the CUDA cores (chunks of 32 steps).  Streaming calls split at a multiple
 * of that block or chunk length reproduce y and the states bit for bit.
 * Errors as mm_ssd_fwd (MM_ERR_UNSUPPORTED for headdim or dstate past those
 * bounds, seqlen > 2^30 or batch * H >= 2^31).
 */
mm_status mm_ssd_fwd_momentum(const void *x, const float *delta, const float *A,
                              const void *B, const void *C,
                              const float *h0, const float *v0, float beta, float alpha,
                              void *y, float *hT, float *vT,
                              const mm_ssd_dims *dims, void *stream);

/*
 * Host-buffer entry points.
 *
 * mm_scan_fwd_host and mm_ssd_fwd_host compute exactly what mm_scan_fwd_gated
 * and mm_ssd_fwd / mm_ssd_fwd_momentum compute, on tensors in HOST memory
 * (same layouts and arguments; every tensor argument is a host pointer).
 * The call streams the sequence through a device workspace in time chunks
 * of `chunk_steps` steps (0: automatic -- about 1/32 of the streamed bytes
 * per chunk, at least 8 MB and 2 KB host rows, a multiple of 32 steps for
 * the scan and of dims->chunk for the SSD).  Chunk i's inputs are copied in
 * on a stream of the call, its device call runs on `stream`, and its
 * outputs are copied out on another stream of the call, through a ring of
 * three workspace slots, so that with page-locked host memory
 * (cudaHostAlloc / cudaHostRegister) both directions of the host link and
 * the kernels overlap.  Pageable host memory works too, without overlap.
 * The carried states stay in the workspace between chunks, so the result
 * is the device call's streaming result for that split (see mm_scan_fwd):
 * with a chunk length that is a multiple of S on the sequence-split path,
 * or on the register-resident path with one time lane, identical to the
 * device entry point on the same sizes.
 *
 * Ordering: the call's copies start after the work queued on `stream`
 * before the call, and work queued on `stream` after the call starts after
 * the last copy-out; synchronise `stream` before reading the outputs.  The
 * call returns once everything is queued (with pageable output buffers the
 * copies themselves may block the host).
 *
 * workspace: device memory of at least the bytes the matching
 * *_workspace_size query returns for the same dims and chunk_steps, 16-byte
 * aligned, owned by the caller, not used by anything else until the call's
 * work on `stream` has completed.  The chunks' scans are mm_scan_fwd calls
 * (with their record memory on the sequence-split path).  A call
 * of more than one chunk runs its copies on two streams of its own, with
 * eleven events; they are created on first use and kept for the calling
 * host thread and device until the thread exits.  A call of one chunk runs
 * everything on `stream`.
 *
 * Errors: those of the device entry point on the same sizes and scalars
 * (checked before anything is queued), and MM_ERR_NULL (workspace NULL),
 * MM_ERR_ALIGN (workspace), MM_ERR_DIMS (workspace too small, chunk_steps
 * < 0), MM_ERR_UNSUPPORTED (a tensor argument in device memory, or the
 * workspace not in device memory), MM_ERR_ALIAS (host output ranges that
 * overlap an input or each other, except hT == h0 and vT == v0).  An error
 * from CUDA after work was queued (MM_ERR_CUDA) leaves the outputs
 * unspecified; the streams are still joined.
 */

/* Device workspace bytes of mm_scan_fwd_host for these sizes, with room for
 * the gate z when with_z != 0. */
mm_status mm_scan_fwd_host_workspace_size(const mm_scan_dims *dims, int with_z,
                                          int64_t chunk_steps, size_t *bytes);

/* mm_scan_fwd_gated over host tensors (D, z, delta_bias, h0, v0, hT, vT
 * optional as there; no checkpoints). */
mm_status mm_scan_fwd_host(const void *x, const void *delta, const float *A,
                           const void *B, const void *C,
                           const float *D, const void *z, const float *delta_bias,
                           int delta_softplus,
                           const float *h0, const float *v0, float beta, float alpha,
                           void *y, float *hT, float *vT,
                           void *workspace, size_t workspace_bytes, int64_t chunk_steps,
                           const mm_scan_dims *dims, void *stream);

/* Device workspace bytes of mm_ssd_fwd_host for these sizes; momentum != 0
 * adds the carried velocity. */
mm_status mm_ssd_fwd_host_workspace_size(const mm_ssd_dims *dims, int momentum,
                                         int64_t chunk_steps, size_t *bytes);

/* The SSD scan over host tensors: mm_ssd_fwd when beta == 0 and v0, vT are
 * NULL, else mm_ssd_fwd_momentum (whose workspace needs momentum != 0). */
mm_status mm_ssd_fwd_host(const void *x, const float *delta, const float *A,
                          const void *B, const void *C,
                          const float *h0, const float *v0, float beta, float alpha,
                          void *y, float *hT, float *vT,
                          void *workspace, size_t workspace_bytes, int64_t chunk_steps,
                          const mm_ssd_dims *dims, void *stream);

/*
 * mm_device_status -- synchronise the current device, then report whether
 * any kernel of this library gave up a bounded device-side wait since the
 * previous call (MM_ERR_DEVICE_TIMEOUT: the outputs of that call are
 * incomplete).  Kernels never wait without a limit (2 s); a wait that runs
 * out records the fact here and the kernel returns.  Clears the record.
 * MM_ERR_CUDA if the synchronisation itself reports an error.
 */
mm_status mm_device_status(void);

/* Static description of a status code (never NULL). */
const char *mm_status_string(mm_status status);

/* Detail of the last error returned on this host thread ("" if none). */
const char *mm_last_error(void);

/*
 * Tuning knob for benchmarks: force the scan's per-thread state count
 * (2, 4 or 8), warps per block (1, 2, 4 or 8) and lanes along time per
 * state group (1, or 2 for the time split: fp32 I/O and 9..16 states
 * only; other calls fall back to one lane).  0, 0, any restores the
 * automatic choice.  Process-wide, not thread-safe with concurrent calls.
 * Returns MM_ERR_UNSUPPORTED for a combination that is not built.
 */
mm_status mm_scan_set_tile(int states_per_thread, int warps_per_block, int time_lanes);

/*
 * Tuning and test knob: force the scan path -- 0 automatic, 1 the
 * register-resident kernel, 2 the sequence-split kernel (used where it
 * applies: no extras, no checkpoints, dstate <= 16, rows of a whole number of
 * 16-byte pieces), 3 the same as one fused launch (no records, see
 * mm_scan_fwd) -- and its segment length (0: automatic, a power of two;
 * else a multiple of 32 in [32, 2^30], rounded up to a multiple of 64 for
 * bf16 calls, one staged chunk of the kernel).  Streaming calls keep
 * bit-identical final states only when split at multiples of S (see
 * mm_scan_fwd), so a forced length that does not divide a caller's split
 * points trades that for the segment count it sets: on one row of 2048
 * channels and 131072 steps (split point 65536), 14592
 * cuts the sequence into nine segments, which fill two one-warp CTAs on each
 * warp scheduler of 148 SMs and ran 9% faster than the automatic eight.
 * Process-wide, not thread-safe with concurrent calls.
 * MM_ERR_UNSUPPORTED for other values.
 */
mm_status mm_scan_set_path(int path, int64_t seg_len);

/*
 * mm_scan_set_deterministic -- 1: mm_scan_bwd and mm_scan_bwd_gated give
 * run-to-run bit-identical dA, dB, dC, dD and ddelta_bias (every other output
 * already is).  Each CTA then writes its channel tile's partial sums to a
 * workspace instead of adding them atomically, and a second kernel adds the
 * partials in a fixed order: dB, dC over the channel tiles of each batch row
 * in tile order, dA, dD, ddelta_bias over the batch rows in row order.  The
 * workspace, (tiles * 2 * batch * dstate * seqlen + batch * dim * (dstate +
 * 2)) * 4 bytes with tiles = ceil(dim / channels per CTA) (dstate 9..16:
 * 16 when batch * dim >= 2048, else 8; dstate 5..8: 16; 3..4: 32; 1..2: 64;
 * 101 MB for batch 4, dim 1536, dstate 16, L 2048), is allocated and freed
 * on the call's stream from a pool the library creates per device on first
 * use (cudaMallocFromPoolAsync / cudaFreeAsync; up to 2 GiB kept reserved
 * between calls); a call on a stream being captured into a graph returns
 * MM_ERR_UNSUPPORTED.  The sums
 * may differ from the default's in the last bits.  0 (the default): atomic
 * sums.  Process-wide, not thread-safe with concurrent calls.
 * MM_ERR_UNSUPPORTED for other values.
 */
mm_status mm_scan_set_deterministic(int on);

/*
 * mm_scan_segment_len -- the segment length S the scan uses for these sizes
 * (*seg_len = 0 when the call runs on the register-resident path, which the
 * automatic choice takes whenever seqlen <= S).  S itself depends on
 * (batch * dim) only.  A streaming caller that splits a sequence at
 * multiples of S, into calls that all take the sequence-split path, gets
 * final states bit-identical to one call (see mm_scan_fwd).  Errors as
 * mm_scan_fwd's size checks; MM_ERR_NULL for a NULL argument.
 */
mm_status mm_scan_segment_len(const mm_scan_dims *dims, int64_t *seg_len);

/*
 * The sequence split across devices.  "Forward Pass: Two-Stage Parallel
 * Scan" of "Momentum Mamba: Enhanced State Space Models with Momentum" joins
 * chunks of the sequence by their 2x2 affine carry maps; here the chunks are
 * segments of S steps (S a power of two) and the sequence of seqlen_total
 * steps is cut into pieces at multiples of S, one per device (rank), every
 * piece but the last a whole number of segments.  A rank holds its piece --
 * steps [seq_first, seq_first + seqlen) of every (batch row, channel) in the
 * usual layouts, with seqlen = dims->seqlen -- and runs:
 *   1. mm_scan_fwd_split_maps: the main pass of the piece's segments, each
 *      from a zero state; y gets that zero-start read-out and `maps` one
 *      record per segment (the lanes' carry maps (beta^S, Q, P, z_v, z_h)
 *      and whether the segment's delta had no negative value);
 *   2. an exchange of the records (an all-gather in piece order, by the
 *      caller: NCCL over NVLink on GPUs), so that one buffer holds the record
 *      of every segment of the sequence in order;
 *   3. mm_scan_fwd_split_correct: each segment's carry-in, the fold of all
 *      earlier segments' maps onto (h0, v0) in order, and its response added
 *      to y (over the whole segment, or until it has fallen below 2^-25 of
 *      its start when A <= 0 and delta >= 0); hT, vT = the fold of every
 *      segment (each rank writes them).
 * y, hT and vT then equal, bit for bit, one mm_scan_fwd over the whole
 * sequence on the sequence-split path with the same S
 * (mm_scan_set_path(2, S)).
 *
 * mm_scan_split_maps_size -- *bytes = the size of `segments` records for
 * dims' (batch, dim).  A piece's buffer holds ceil(seqlen / S) records, the
 * gathered buffer ceil(seqlen_total / S); record j starts at j times the
 * size of one.  Errors as mm_scan_fwd's size checks; MM_ERR_DIMS for
 * segments outside [0, 2^30]; MM_ERR_NULL.
 */
mm_status mm_scan_split_maps_size(const mm_scan_dims *dims, int64_t segments, size_t *bytes);

/*
 * mm_scan_fwd_split_maps -- launch 1 of the split (see above) on `stream`.
 *   x, delta (batch, dim, seqlen) io; A (dim, dstate) fp32;
 *   B, C (batch, dstate, seqlen) io: the piece, device memory, read only;
 *   y    (batch, dim, seqlen) io, written: the zero-start read-out;
 *   maps device memory of mm_scan_split_maps_size(dims, ceil(seqlen / S))
 *        bytes, written; the caller owns every buffer.
 *   seg_len S: a power of two in [32, 2^30] for fp32 I/O, [64, 2^30] for
 *        bf16 (a segment is a whole number of the kernel's staged chunks).
 * Errors: MM_ERR_NULL, MM_ERR_DIMS, MM_ERR_DTYPE, MM_ERR_SCALAR as
 * mm_scan_fwd; MM_ERR_UNSUPPORTED (dstate > 16, S outside its range, rows
 * of seqlen elements not a whole number of 16-byte pieces); MM_ERR_ALIGN
 * (a pointer not 16-byte aligned); MM_ERR_ALIAS (y or maps overlapping an
 * input or each other); MM_ERR_CUDA.  A record is written only by a CTA
 * that finished its segment: after mm_device_status reports
 * MM_ERR_DEVICE_TIMEOUT the records are not to be used.
 */
mm_status mm_scan_fwd_split_maps(const void *x, const void *delta, const float *A,
                                 const void *B, const void *C, float beta, float alpha,
                                 void *y, void *maps, int64_t seg_len,
                                 const mm_scan_dims *dims, void *stream);

/*
 * mm_scan_fwd_split_maps_peers -- launch 1 of the split with the exchange
 * folded into it: instead of into a buffer of the piece's own records, each
 * segment's record is stored, at its global index seq_first / S + k, into
 * every one of `ndest` buffers of the whole sequence's records -- the
 * buffers launch 3 reads on each rank, reached as peer memory (CUDA IPC,
 * mm_ipc_open_handle; over NVLink between GPUs).  After every rank's launch
 * has completed (a stream-ordered barrier across the ranks, e.g. an NCCL
 * all-reduce of one value), launch 3 runs on the local buffer; no gather of
 * records is needed.  The kernel fences its stores at system scope before it
 * completes.
 *   x, delta, A, B, C, y, seg_len, dims: as mm_scan_fwd_split_maps;
 *   dests      device memory: an array of ndest device pointers (8-byte
 *              aligned), each to a 16-byte-aligned buffer of
 *              mm_scan_split_maps_size(dims, ceil(seqlen_total / S)) bytes;
 *   ndest      1 .. MM_SPLIT_MAX_RANKS;
 *   seq_first, seqlen_total: the piece's place, as mm_scan_fwd_split_correct.
 * Errors: as mm_scan_fwd_split_maps and mm_scan_fwd_split_correct's piece
 * checks; MM_ERR_UNSUPPORTED for ndest out of range; MM_ERR_ALIGN for dests.
 * The pointers in dests are not checked (device memory): each must be a
 * buffer as stated.
 */
#define MM_SPLIT_MAX_RANKS 64
mm_status mm_scan_fwd_split_maps_peers(const void *x, const void *delta, const float *A,
                                       const void *B, const void *C, float beta, float alpha,
                                       void *y, void *const *dests, int ndest,
                                       int64_t seq_first, int64_t seg_len, int64_t seqlen_total,
                                       const mm_scan_dims *dims, void *stream);

/*
 * CUDA IPC for the records buffers of the split (wrappers of
 * cudaIpcGetMemHandle, cudaIpcOpenMemHandle with lazy peer access, and
 * cudaIpcCloseMemHandle; the pages have no counterpart).  A handle names the
 * whole allocation (cudaMalloc memory) that holds dev_ptr -- an allocator may
 * hand out pieces of a larger one -- so mm_ipc_get_handle also returns dev_ptr's byte offset in
 * it; the caller exchanges handle (MM_IPC_HANDLE_BYTES opaque bytes) and
 * offset, mm_ipc_open_handle in another process returns the mapped
 * allocation plus the offset, and mm_ipc_close_handle takes that pointer and
 * the same offset.  A handle opens only in another process than the one that
 * made it.  Errors: MM_ERR_NULL, MM_ERR_DIMS (negative offset), MM_ERR_CUDA
 * (with CUDA's message in mm_last_error).
 */
#define MM_IPC_HANDLE_BYTES 64
mm_status mm_ipc_get_handle(const void *dev_ptr, void *handle, int64_t *offset);
mm_status mm_ipc_open_handle(const void *handle, int64_t offset, void **dev_ptr);
mm_status mm_ipc_close_handle(void *dev_ptr, int64_t offset);

/*
 * mm_scan_fwd_split_correct -- launch 3 of the split on `stream`.
 *   delta, A, C   the piece, as for launch 1 (read only);
 *   h0, v0        (batch, dim, dstate) fp32 state at step 0 of the whole
 *                 sequence, or NULL for zero;
 *   y             launch 1's output for this piece, read and updated;
 *   hT, vT        (batch, dim, dstate) fp32, the states after the last step
 *                 of the whole sequence, or NULL;
 *   maps_all      the gathered records of all ceil(seqlen_total / S)
 *                 segments, device memory, read only;
 *   seq_first     the piece's first step: a multiple of S;
 *   seqlen_total  steps of the whole sequence (<= 2^30); a piece that ends
 *                 before it holds whole segments.
 * beta, alpha and S as in launch 1.  Errors as launch 1, and
 * MM_ERR_UNSUPPORTED for a piece outside the sequence or not on segment
 * boundaries; MM_ERR_ALIAS for y, hT or vT overlapping an input (h0, v0
 * and maps_all included) or each other.
 */
mm_status mm_scan_fwd_split_correct(const void *delta, const float *A, const void *C,
                                    const float *h0, const float *v0, float beta, float alpha,
                                    void *y, float *hT, float *vT, const void *maps_all,
                                    int64_t seg_len, int64_t seq_first, int64_t seqlen_total,
                                    const mm_scan_dims *dims, void *stream);

/*
 * mm_scan_fwd_noalloc -- mm_scan_fwd for callers that cannot allocate device
 * memory.  (An addition of this library: the paper has no counterpart.)
 *
 * Who needs it: code that runs where every device allocation belongs to a
 * host framework (a plugin, a serving runtime's custom-op slot), a process
 * whose device memory was reserved once at start-up, or a path that must
 * not pay cudaMalloc's device-wide synchronisation.  The scan's two-launch
 * sequence split (mm_scan_fwd_split_maps, then mm_scan_fwd_split_correct,
 * on this one device) passes segment records between its launches; here
 * they live in a fixed 8 MiB array inside the library, reserved on every GPU
 * that loads the library until the process exits.  Nothing is allocated:
 * no cudaMalloc, no cudaFree, no allocating library routine.
 *
 * Arguments, layouts and results as mm_scan_fwd (the caller owns and passes
 * every input and output); y, hT, vT equal those of one call of the
 * sequence-split path with this entry's segment length S, the path's own
 * length for (batch * dim), at least one staged chunk (32 fp32 / 64 bf16
 * steps).  Limits: the records of ceil(seqlen / S) segments
 * (mm_scan_split_maps_size) must fit in 8 MiB, else MM_ERR_UNSUPPORTED
 * with the bytes needed; rows of seqlen elements must be a whole number of
 * 16-byte pieces and dstate <= 16 (MM_ERR_UNSUPPORTED); hT, vT may not be
 * h0, v0 (MM_ERR_ALIAS).  Other errors as mm_scan_fwd.
 *
 * The first call on a device looks up the array's address on that device
 * (cudaGetSymbolAddress, that device current); make that first call before
 * any stream capture.  Every call shares the one array and leaves its
 * records there: nothing in it has to start at zero (each call writes every
 * record it reads before reading it), but calls whose work overlaps on the
 * GPU -- on two streams, or from two host threads -- race on it and must be
 * ordered by the caller.
 */
mm_status mm_scan_fwd_noalloc(const void *x, const void *delta, const float *A,
                              const void *B, const void *C,
                              const float *h0, const float *v0,
                              float beta, float alpha,
                              void *y, float *hT, float *vT,
                              const mm_scan_dims *dims, void *stream);

/* Library version, major * 10000 + minor * 100 + patch. */
int mm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MM_SCAN_H */
