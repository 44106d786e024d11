// mm_internal.h -- declarations shared by the translation units of
// libmmscan (argument blocks and launchers).  Not part of the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "mm_scan.h"

namespace mmscan {

// Record the calling thread's last error message (mm_last_error) and return
// `st`; report_ok clears the message and returns MM_OK.
mm_status report(mm_status st, const char* fmt, ...);
mm_status report_ok();

// Release the side streams and events the host-buffer entry points keep for
// the calling thread (created again on the next call that needs them).
void host_pipeline_release();

// Arguments of one scan launch (device pointers; sizes as in mm_scan_dims).
struct ScanArgs {
    const void* x;
    const void* delta;
    const float* A;
    const void* B;
    const void* C;
    const float* h0;
    const float* v0;
    void* y;
    float* hT;
    float* vT;
    int64_t batch, seqlen, dim;
    int dstate;
    int tiles_per_batch;   // filled by the launcher
    float beta, alpha;
    int vec_ok;            // rows of L elements are whole 16-byte pieces
    // selective_scan_fn extras (all absent on the plain path)
    const float* Dskip;    // (dim) or null
    const void* z;         // (batch, dim, L) io dtype, or null
    const float* dbias;    // (dim) or null
    int softplus;          // delta' = softplus(delta + dbias)
    int ext;               // any of the four is present
    float* ckpt;           // (batch, dim, ceil(L / 16), 2, dstate): (h, v) after every 16 steps, or null
    int stall;             // test only: stage no input, so that the bounded waits run out
    int deny_records;      // test only: the sequence-split path's record memory request fails
};

// Arguments of one backward launch (device pointers; sizes as in mm_scan_dims).
struct ScanBwdArgs {
    const void* x;
    const void* delta;
    const float* A;
    const void* B;
    const void* C;
    const float* h0;
    const float* v0;
    const float* ckpt;     // the forward's (h, v) after every 16 steps
    const void* dout;      // gradient reaching y (io dtype)
    const float* dhT;      // gradients reaching hT, vT, or null
    const float* dvT;
    void* dx;              // io dtype
    void* ddelta;          // io dtype
    float* dA;             // (dim, dstate), summed over the batch
    float* dB;             // (batch, dstate, L), summed over dim
    float* dC;
    float* dh0;            // (batch, dim, dstate) or null
    float* dv0;
    int64_t batch, seqlen, dim;
    int dstate;
    int tiles_per_batch;   // filled by the launcher
    float beta, alpha;
    int vec_ok;            // rows of L elements are whole 16-byte pieces
    // selective_scan_fn extras (all absent for the plain scan's backward)
    const float* Dskip;    // (dim) or null
    const void* z;         // (batch, dim, L) io, or null
    const float* dbias;    // (dim) or null
    int softplus;
    int ext;               // any of the four is present
    float* dD;             // (dim), summed over batch and steps, or null
    void* dz;              // (batch, dim, L) io, or null
    float* ddbias;         // (dim), or null
    int stall;             // test only: stage no input, so that the bounded waits run out
    // The deterministic form (mm_scan_set_deterministic): per-tile partials of
    // dB, dC and per-row partials of dA, dD, d bias in a workspace (filled by
    // the launcher), summed in a fixed order by a second kernel.
    int det;
    float* ws_bc;          // [tile][dB, dC][batch][dstate][L]
    float* ws_a;           // [batch][dim][dstate]
    float* ws_d;           // [dD, d bias][batch][dim]
};

// Arguments of one decode step (device pointers; states updated in place).
struct ScanStepArgs {
    const void* x;         // (batch, dim) io
    const void* delta;     // (batch, dim) io
    const float* A;        // (dim, dstate)
    const void* B;         // (batch, dstate) io
    const void* C;
    const float* Dskip;    // (dim) or null
    const void* z;         // (batch, dim) io, or null
    const float* dbias;    // (dim) or null
    int softplus;
    int ext;               // any of the four extras is present
    float* h;              // (batch, dim, dstate) fp32, read and written
    float* v;
    void* y;               // (batch, dim) io
    int64_t batch, dim;
    int dstate;
    int vec;               // dstate is a multiple of 4: 16-byte state accesses
    float beta, alpha;
};

struct ScanTileChoice {
    int np;      // states padded to a power of two (2, 4, 8, 16)
    int spt;     // states per lane (2 or 4)
    int warps;   // warps per CTA (1, 2, 4 or 8)
    int ts;      // lanes along time per state group (1, or 2 for the time split)
};

// Sequence-split scan (scan_seg.cu): segments of a power-of-two length at
// absolute multiples of it, one per CTA of a cluster of at most
// kSegMaxCluster CTAs, joined through their 2x2 affine carry maps.
constexpr int kSegMaxCluster = 8;
constexpr int kSegMaxRound = 256;     // segments of a channel tile per round of a plain grid
constexpr int64_t kSegMinLen = 16384;
int64_t scan_seg_default_len(int64_t batch, int64_t dim);
// The sequence-split path of mm_scan_fwd: by default two launches (the main
// passes with their segment maps to records in stream-ordered memory from a
// library pool, then the fold and correction); `fused`, or records that
// cannot be had, run the single fused launch.
cudaError_t launch_scan_seg(const ScanArgs& a, int io, int64_t seg_len, bool fused, cudaStream_t s);
// Steps of one staged chunk of the sequence-split kernel (32 fp32, 64 bf16).
int64_t scan_seg_chunk_steps(int io);
// The sequence split over several calls: the channels of one CTA's tile and
// the bytes of one tile's record of one segment (a segment's records: one
// per (batch row, channel tile), in that order), and the two launches --
// mode 1 the main pass with the maps to `maps`, mode 2 the fold of the whole
// sequence's maps and the correction (seg_first: global index of the call's
// first segment).
int64_t scan_seg_tile_channels();
int64_t scan_seg_tile_record_bytes();
// (mode 1 with ndest > 0: the records go to the ndest buffers whose device
// pointers `dests` (a device array) holds, at their global index)
cudaError_t launch_scan_seg_split(const ScanArgs& a, int io, int64_t seg_len, int mode, void* maps,
                                  int64_t seg_first, int64_t seqlen_total, void* const* dests, int ndest,
                                  cudaStream_t s);
unsigned int scan_seg_read_and_clear_device_error();

bool scan_tile_supported(int spt, int warps, int time_lanes);
ScanTileChoice choose_scan_tile(int64_t batch, int64_t dim, int64_t dstate, int io,
                                int forced_spt, int forced_warps, int forced_ts);
cudaError_t launch_scan_fwd(const ScanArgs& a, const ScanTileChoice& t, int io, cudaStream_t s);
cudaError_t launch_scan_bwd(const ScanBwdArgs& a, int io, cudaStream_t s);
// Bytes of the deterministic backward's workspace (-1 past 2^63).
int64_t scan_bwd_det_workspace_bytes(int64_t batch, int64_t dim, int dstate, int64_t seqlen);
// Whether `s` is being captured into a CUDA graph (false when that cannot be told).
bool stream_capturing(cudaStream_t s);
cudaError_t launch_scan_step(const ScanStepArgs& a, int io, cudaStream_t s);
// Read (and reset) the device error word of the scan / SSD kernels.
unsigned int scan_read_and_clear_device_error();
unsigned int scan_bwd_read_and_clear_device_error();
unsigned int ssd_read_and_clear_device_error();

// Arguments of one SSD call.
struct SSDArgs {
    const void* x;
    const float* delta;
    const float* A;
    const void* B;
    const void* C;
    const float* h0;
    void* y;
    float* hT;
    int64_t batch, seqlen, nheads, headdim, dstate, ngroups, chunk;
    float alpha;
    int stall;             // test only: stage no input, so that the bounded waits run out
};

// Arguments of one momentum SSD call (the CUDA-core chunked kernel).
struct SSDMomArgs {
    const void* x;         // (batch, L, H, P) bf16
    const float* delta;    // (batch, L, H)
    const float* A;        // (H)
    const void* B;         // (batch, L, G, N) bf16
    const void* C;
    const float* h0;       // (batch, H, P, N) fp32 or null
    const float* v0;
    void* y;               // (batch, L, H, P) bf16
    float* hT;             // (batch, H, P, N) fp32 or null
    float* vT;
    int64_t batch, seqlen, nheads, headdim, dstate, ngroups;
    float beta, alpha;
    int stall;             // test only (tensor-core kernel): stage no input, so that the bounded waits run out
};

bool ssd_mom_shape_supported(int64_t headdim, int64_t dstate);
cudaError_t launch_ssd_mom(const SSDMomArgs& a, cudaStream_t s);
// The tensor-core form (ssd_mom_tc.cu) for headdim 64, dstate 128.
bool ssd_mom_tc_shape_supported(int64_t headdim, int64_t dstate);
cudaError_t launch_ssd_mom_tc(const SSDMomArgs& a, cudaStream_t s);
unsigned int ssd_mom_tc_read_and_clear_device_error();

bool ssd_shape_supported(int64_t headdim, int64_t dstate, int64_t chunk);
cudaError_t launch_ssd_fwd(const SSDArgs& a, cudaStream_t s);

}  // namespace mmscan
