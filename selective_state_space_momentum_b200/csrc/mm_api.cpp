// mm_api.cpp -- the C ABI of libmmscan (declared in include/mm_scan.h):
// host-side argument checks, variant choice and launch.  Every check runs
// before anything is enqueued; a rejected call touches no buffer.
#include "mm_scan.h"

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include "mm_internal.h"

namespace {

thread_local std::string g_last_error;

mm_status fail(mm_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

mm_status ok() {
    g_last_error.clear();
    return MM_OK;
}

std::atomic<int> g_forced_spt{0};
std::atomic<int> g_forced_warps{0};
std::atomic<int> g_forced_ts{1};
// Scan path: 0 automatic, 1 the register-resident kernel, 2 the sequence-split
// kernel; and its segment length (0: automatic).
std::atomic<int> g_forced_path{0};
std::atomic<int> g_deterministic{0};
std::atomic<int64_t> g_forced_seg_len{0};

// The automatic path choice depends on (batch * dim, dstate, io) and on
// whether the sequence is longer than one segment.  The sequence-split
// kernel pads the states to 16, so it serves dstate > 8; it pays off when
// there are few channels (the register-resident kernel then cannot fill the
// GPU) and the sequence spans more than one segment (a single segment
// leaves nothing to split).
bool seg_auto(int64_t batch, int64_t dim, int64_t dstate, int io) {
    return dstate > 8 && io == MM_F32 && batch * dim <= 4096;
}

// Segment length of the sequence-split path for these sizes, or 0 when the
// call runs on the register-resident kernel.  The length itself depends on
// (batch * dim) only, never on L.
int64_t seg_len_for(int64_t batch, int64_t L, int64_t dim, int64_t dstate, int io, bool vec_ok) {
    const int path = g_forced_path.load();
    if (!vec_ok || dstate > 16) return 0;
    if (path == 1) return 0;
    if (path == 0 && !seg_auto(batch, dim, dstate, io)) return 0;       // 2, 3: forced
    const int64_t forced = g_forced_seg_len.load();
    int64_t S = forced > 0 ? forced : mmscan::scan_seg_default_len(batch, dim);
    // a segment is a whole number of staged chunks (64 steps for bf16)
    const int64_t chunk = mmscan::scan_seg_chunk_steps(io == MM_F32 ? 0 : 1);
    S = (S + chunk - 1) / chunk * chunk;
    if (path == 0 && L <= S) return 0;
    return S;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// a * b * ... without int64 overflow; false on overflow.
bool mul_ok(int64_t a, int64_t b, int64_t* out) {
    if (a < 0 || b < 0) return false;
    if (a != 0 && b > INT64_MAX / a) return false;
    *out = a * b;
    return true;
}

// The kernels form time coordinates of the tiled copies, grid sizes and
// channel numbers in 32 bits; requests beyond these bounds are refused
// before launch.
constexpr int64_t kMaxSeqlen = int64_t(1) << 30;
constexpr int64_t kMaxIndex = 0x7fffffffLL;

struct Range {
    const char* name;
    uintptr_t lo, hi;   // [lo, hi)
};

Range rng(const char* name, const void* p, int64_t bytes) {
    const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
    return Range{name, lo, p ? lo + static_cast<uintptr_t>(bytes) : lo};
}

bool overlap(const Range& a, const Range& b) {
    if (a.lo == a.hi || b.lo == b.hi) return false;   // NULL / empty
    return a.lo < b.hi && b.lo < a.hi;
}

// Fault-injection hook for the host-side error path: with
// MMSCAN_FAULT_INJECT=launch a call that passed its checks returns
// MM_ERR_CUDA without launching anything.
bool inject_launch_failure() {
    const char* v = std::getenv("MMSCAN_FAULT_INJECT");
    return v && std::strcmp(v, "launch") == 0;
}

// Test hook for the device-side give-up path: with MMSCAN_FAULT_INJECT=stall
// the kernels that stage their inputs through bounded waits (the two forward
// scans, the backward, the SSD kernel) are launched with their producer told
// to issue nothing.  Nothing is then in flight; every wait runs out after its
// limit, the kernel returns, and mm_device_status reports
// MM_ERR_DEVICE_TIMEOUT.  The outputs of such a call are undefined.
int inject_stall() {
    const char* v = std::getenv("MMSCAN_FAULT_INJECT");
    return (v && std::strcmp(v, "stall") == 0) ? 1 : 0;
}

// Test hook for the sequence-split path's fallback: with
// MMSCAN_FAULT_INJECT=records its request for record memory asks for more
// than any device holds, fails, and the call runs the fused launch.
int inject_records_denied() {
    const char* v = std::getenv("MMSCAN_FAULT_INJECT");
    return (v && std::strcmp(v, "records") == 0) ? 1 : 0;
}

mm_status from_cuda(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return ok();
    return fail(MM_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

// Checks shared by the scan calls (sizes, dtype, scalars) and the byte
// sizes of their operands.
struct ScanSizes {
    int64_t esize;       // bytes of one io element
    int64_t seq_bytes;   // (batch, dim, L) io
    int64_t bc_bytes;    // (batch, dstate, L) io
    int64_t bcf_bytes;   // (batch, dstate, L) fp32
    int64_t a_bytes;     // (dim, dstate) fp32
    int64_t st_bytes;    // (batch, dim, dstate) fp32
    int64_t d_bytes;     // (dim) fp32
    int64_t ck_bytes;    // (batch, dim, ceil(L / 16), 2, dstate) fp32
};

// seqlen and batch * nheads (the grid) of the SSD calls within the 32-bit bounds.
mm_status check_ssd_range(const mm_ssd_dims* dims) {
    int64_t bh = 0;
    if (dims->seqlen > kMaxSeqlen || !mul_ok(dims->batch, dims->nheads, &bh) || bh > kMaxIndex)
        return fail(MM_ERR_UNSUPPORTED, "SSD seqlen=%lld batch=%lld nheads=%lld: seqlen must be <= 2^30 "
                    "and batch * nheads < 2^31", (long long)dims->seqlen, (long long)dims->batch,
                    (long long)dims->nheads);
    return MM_OK;
}

mm_status check_scan_dims(const mm_scan_dims* dims, float beta, float alpha, ScanSizes* z) {
    const int64_t bsz = dims->batch, L = dims->seqlen, D = dims->dim, N = dims->dstate;
    if (bsz < 1 || L < 1 || D < 1 || N < 1)
        return fail(MM_ERR_DIMS, "sizes must be >= 1 (batch=%lld seqlen=%lld dim=%lld dstate=%lld)",
                    (long long)bsz, (long long)L, (long long)D, (long long)N);
    if (N > 16) return fail(MM_ERR_UNSUPPORTED, "dstate=%lld > 16", (long long)N);
    if (L > kMaxSeqlen || bsz > kMaxIndex || D > kMaxIndex)
        return fail(MM_ERR_UNSUPPORTED, "seqlen=%lld batch=%lld dim=%lld: seqlen must be <= 2^30 and "
                    "batch, dim < 2^31", (long long)L, (long long)bsz, (long long)D);
    if (dims->io != MM_F32 && dims->io != MM_BF16)
        return fail(MM_ERR_DTYPE, "io=%d is not MM_F32 or MM_BF16", (int)dims->io);
    if (!std::isfinite(beta) || beta < 0.0f || beta >= 1.0f)
        return fail(MM_ERR_SCALAR, "beta=%g is outside [0, 1)", (double)beta);
    if (!std::isfinite(alpha) || alpha < 0.0f)
        return fail(MM_ERR_SCALAR, "alpha=%g must be finite and >= 0", (double)alpha);
    z->esize = dims->io == MM_F32 ? 4 : 2;
    const int64_t chunks = (L + MM_SCAN_CKPT_STEPS - 1) / MM_SCAN_CKPT_STEPS;
    int64_t bd, bdl, bn, bnl, dn, bdn, bdc, bdc2;
    if (!mul_ok(bsz, D, &bd) || !mul_ok(bd, L, &bdl) || !mul_ok(bdl, z->esize, &z->seq_bytes) ||
        !mul_ok(bsz, N, &bn) || !mul_ok(bn, L, &bnl) || !mul_ok(bnl, z->esize, &z->bc_bytes) ||
        !mul_ok(bnl, 4, &z->bcf_bytes) || !mul_ok(D, N, &dn) || !mul_ok(dn, 4, &z->a_bytes) ||
        !mul_ok(bd, N, &bdn) || !mul_ok(bdn, 4, &z->st_bytes) || !mul_ok(D, 4, &z->d_bytes) ||
        !mul_ok(bd, chunks, &bdc) || !mul_ok(bdc, 2 * N, &bdc2) || !mul_ok(bdc2, 4, &z->ck_bytes))
        return fail(MM_ERR_DIMS, "sizes overflow 64-bit byte counts");
    return MM_OK;
}

// Bytes of `segments` segment records of a split scan over (batch, dim);
// false when the count overflows 64 bits.
bool split_record_bytes(int64_t batch, int64_t dim, int64_t segments, int64_t* out) {
    const int64_t ch = mmscan::scan_seg_tile_channels();
    const int64_t tiles = dim / ch + (dim % ch != 0);
    int64_t per_seg = 0;
    return mul_ok(batch, tiles, &per_seg) && mul_ok(per_seg, mmscan::scan_seg_tile_record_bytes(), &per_seg) &&
           mul_ok(per_seg, segments, out);
}

// The checks the two launches of a split scan share: the segment length, the
// row rule of the tiled copies, and the piece's place in the whole sequence.
mm_status check_split(const mm_scan_dims* dims, const ScanSizes& zs, int64_t seg_len, int64_t seq_first,
                      int64_t seqlen_total) {
    const int64_t chunk = mmscan::scan_seg_chunk_steps(dims->io == MM_F32 ? 0 : 1);
    if (seg_len < chunk || seg_len > kMaxSeqlen || (seg_len & (seg_len - 1)) != 0)
        return fail(MM_ERR_UNSUPPORTED, "segment length %lld is not a power of two in [%lld, 2^30]",
                    (long long)seg_len, (long long)chunk);
    if ((dims->seqlen * zs.esize) % 16 != 0)
        return fail(MM_ERR_UNSUPPORTED, "rows of seqlen=%lld elements are not a whole number of 16-byte pieces",
                    (long long)dims->seqlen);
    if (seqlen_total < 1 || seqlen_total > kMaxSeqlen)
        return fail(MM_ERR_UNSUPPORTED, "seqlen_total=%lld is outside [1, 2^30]", (long long)seqlen_total);
    if (seq_first < 0 || seq_first % seg_len != 0 || seq_first > seqlen_total - dims->seqlen)
        return fail(MM_ERR_UNSUPPORTED, "a piece of %lld steps at step %lld does not start at a multiple of %lld "
                    "within %lld steps", (long long)dims->seqlen, (long long)seq_first, (long long)seg_len,
                    (long long)seqlen_total);
    if (seq_first + dims->seqlen < seqlen_total && dims->seqlen % seg_len != 0)
        return fail(MM_ERR_UNSUPPORTED, "a piece before the last must hold whole segments (seqlen=%lld, S=%lld)",
                    (long long)dims->seqlen, (long long)seg_len);
    return MM_OK;
}

}  // namespace

namespace mmscan {

mm_status report(mm_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

mm_status report_ok() { return ok(); }

}  // namespace mmscan

extern "C" {

const char* mm_status_string(mm_status s) {
    switch (s) {
        case MM_OK: return "ok";
        case MM_ERR_NULL: return "a required pointer is NULL";
        case MM_ERR_DIMS: return "invalid sizes";
        case MM_ERR_SCALAR: return "beta must be in [0, 1) and alpha finite and >= 0";
        case MM_ERR_DTYPE: return "unknown storage type";
        case MM_ERR_ALIGN: return "a base pointer is not 16-byte aligned";
        case MM_ERR_UNSUPPORTED: return "request outside what this build supports";
        case MM_ERR_CUDA: return "CUDA error";
        case MM_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait gave up";
        case MM_ERR_ALIAS: return "an output overlaps an input";
    }
    return "unknown status";
}

const char* mm_last_error(void) { return g_last_error.c_str(); }

int mm_version(void) { return 100; }

mm_status mm_device_status(void) {
    const cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return from_cuda(e, "mm_device_status: synchronize");
    const unsigned int w = mmscan::scan_read_and_clear_device_error() |
                           mmscan::scan_seg_read_and_clear_device_error() |
                           mmscan::scan_bwd_read_and_clear_device_error() |
                           mmscan::ssd_read_and_clear_device_error() |
                           mmscan::ssd_mom_tc_read_and_clear_device_error();
    if (w) return fail(MM_ERR_DEVICE_TIMEOUT, "a device-side wait ran past its limit (word 0x%x)", w);
    return ok();
}

mm_status mm_scan_set_tile(int spt, int warps, int time_lanes) {
    if (spt == 0 && warps == 0) {
        g_forced_spt = 0;
        g_forced_warps = 0;
        g_forced_ts = 1;
        return ok();
    }
    if (!mmscan::scan_tile_supported(spt, warps, time_lanes))
        return fail(MM_ERR_UNSUPPORTED, "scan tile spt=%d warps=%d time_lanes=%d is not built", spt,
                    warps, time_lanes);
    g_forced_spt = spt;
    g_forced_warps = warps;
    g_forced_ts = time_lanes;
    return ok();
}

mm_status mm_scan_set_path(int path, int64_t seg_len) {
    if (path < 0 || path > 3)
        return fail(MM_ERR_UNSUPPORTED, "scan path %d is not 0 (automatic), 1, 2 or 3", path);
    if (seg_len != 0 && (seg_len < 32 || seg_len > (int64_t(1) << 30) || seg_len % 32 != 0))
        return fail(MM_ERR_UNSUPPORTED, "segment length %lld is not 0 or a multiple of 32 in [32, 2^30]",
                    (long long)seg_len);
    g_forced_path = path;
    g_forced_seg_len = seg_len;
    return ok();
}

mm_status mm_scan_set_deterministic(int on) {
    if (on != 0 && on != 1) return fail(MM_ERR_UNSUPPORTED, "deterministic switch %d is not 0 or 1", on);
    g_deterministic = on;
    return ok();
}

mm_status mm_scan_segment_len(const mm_scan_dims* dims, int64_t* seg_len) {
    if (!dims || !seg_len) return fail(MM_ERR_NULL, "dims and seg_len are required");
    ScanSizes zs;
    if (mm_status st = check_scan_dims(dims, 0.0f, 1.0f, &zs)) return st;
    *seg_len = seg_len_for(dims->batch, dims->seqlen, dims->dim, dims->dstate, dims->io,
                           ((dims->seqlen * zs.esize) % 16) == 0);
    return ok();
}

mm_status mm_scan_split_maps_size(const mm_scan_dims* dims, int64_t segments, size_t* bytes) {
    if (!dims || !bytes) return fail(MM_ERR_NULL, "dims and bytes are required");
    ScanSizes zs;
    if (mm_status st = check_scan_dims(dims, 0.0f, 1.0f, &zs)) return st;
    if (segments < 0 || segments > kMaxSeqlen)
        return fail(MM_ERR_DIMS, "segments=%lld is outside [0, 2^30]", (long long)segments);
    int64_t total = 0;
    if (!split_record_bytes(dims->batch, dims->dim, segments, &total))
        return fail(MM_ERR_DIMS, "record bytes overflow 64 bits");
    *bytes = static_cast<size_t>(total);
    return ok();
}

mm_status mm_scan_fwd_split_maps(const void* x, const void* delta, const float* A, const void* B,
                                 const void* C, float beta, float alpha, void* y, void* maps,
                                 int64_t seg_len, const mm_scan_dims* dims, void* stream) {
    if (!dims) return fail(MM_ERR_NULL, "dims is NULL");
    if (!x || !delta || !A || !B || !C || !y || !maps)
        return fail(MM_ERR_NULL, "x, delta, A, B, C, y and maps are required");
    ScanSizes zs;
    if (mm_status st = check_scan_dims(dims, beta, alpha, &zs)) return st;
    // a piece is checked as the last one of a sequence that ends with it
    if (mm_status st = check_split(dims, zs, seg_len, 0, dims->seqlen)) return st;
    const void* ptrs[] = {x, delta, A, B, C, y, maps};
    const char* names[] = {"x", "delta", "A", "B", "C", "y", "maps"};
    for (int i = 0; i < 7; ++i)
        if (!aligned16(ptrs[i])) return fail(MM_ERR_ALIGN, "%s is not 16-byte aligned", names[i]);
    int64_t maps_bytes = 0;
    if (!split_record_bytes(dims->batch, dims->dim, (dims->seqlen + seg_len - 1) / seg_len, &maps_bytes))
        return fail(MM_ERR_DIMS, "record bytes overflow 64 bits");
    const Range ry = rng("y", y, zs.seq_bytes), rm = rng("maps", maps, maps_bytes);
    const Range ins[] = {rng("x", x, zs.seq_bytes), rng("delta", delta, zs.seq_bytes), rng("A", A, zs.a_bytes),
                         rng("B", B, zs.bc_bytes), rng("C", C, zs.bc_bytes)};
    for (const Range& in : ins) {
        if (overlap(ry, in)) return fail(MM_ERR_ALIAS, "y overlaps %s", in.name);
        if (overlap(rm, in)) return fail(MM_ERR_ALIAS, "maps overlaps %s", in.name);
    }
    if (overlap(rm, ry)) return fail(MM_ERR_ALIAS, "maps overlaps y");
    if (inject_launch_failure()) return fail(MM_ERR_CUDA, "injected launch failure (MMSCAN_FAULT_INJECT)");
    mmscan::ScanArgs a{};
    a.x = x; a.delta = delta; a.A = A; a.B = B; a.C = C; a.y = y;
    a.batch = dims->batch; a.seqlen = dims->seqlen; a.dim = dims->dim; a.dstate = (int)dims->dstate;
    a.beta = beta; a.alpha = alpha;
    a.vec_ok = 1;
    a.stall = inject_stall();
    return from_cuda(mmscan::launch_scan_seg_split(a, dims->io, seg_len, 1, maps, 0, dims->seqlen, nullptr, 0,
                                                   static_cast<cudaStream_t>(stream)),
                     "mm_scan_fwd_split_maps launch");
}

mm_status mm_scan_fwd_split_maps_peers(const void* x, const void* delta, const float* A, const void* B,
                                       const void* C, float beta, float alpha, void* y, void* const* dests,
                                       int ndest, int64_t seq_first, int64_t seg_len, int64_t seqlen_total,
                                       const mm_scan_dims* dims, void* stream) {
    if (!dims) return fail(MM_ERR_NULL, "dims is NULL");
    if (!x || !delta || !A || !B || !C || !y || !dests)
        return fail(MM_ERR_NULL, "x, delta, A, B, C, y and dests are required");
    if (ndest < 1 || ndest > MM_SPLIT_MAX_RANKS)
        return fail(MM_ERR_UNSUPPORTED, "ndest=%d is outside [1, %d]", ndest, MM_SPLIT_MAX_RANKS);
    ScanSizes zs;
    if (mm_status st = check_scan_dims(dims, beta, alpha, &zs)) return st;
    if (mm_status st = check_split(dims, zs, seg_len, seq_first, seqlen_total)) return st;
    const void* ptrs[] = {x, delta, A, B, C, y};
    const char* names[] = {"x", "delta", "A", "B", "C", "y"};
    for (int i = 0; i < 6; ++i)
        if (!aligned16(ptrs[i])) return fail(MM_ERR_ALIGN, "%s is not 16-byte aligned", names[i]);
    if ((reinterpret_cast<uintptr_t>(dests) & 7u) != 0) return fail(MM_ERR_ALIGN, "dests is not 8-byte aligned");
    const Range ry = rng("y", y, zs.seq_bytes);
    const Range ins[] = {rng("x", x, zs.seq_bytes), rng("delta", delta, zs.seq_bytes), rng("A", A, zs.a_bytes),
                         rng("B", B, zs.bc_bytes), rng("C", C, zs.bc_bytes)};
    for (const Range& in : ins)
        if (overlap(ry, in)) return fail(MM_ERR_ALIAS, "y overlaps %s", in.name);
    if (inject_launch_failure()) return fail(MM_ERR_CUDA, "injected launch failure (MMSCAN_FAULT_INJECT)");
    mmscan::ScanArgs a{};
    a.x = x; a.delta = delta; a.A = A; a.B = B; a.C = C; a.y = y;
    a.batch = dims->batch; a.seqlen = dims->seqlen; a.dim = dims->dim; a.dstate = (int)dims->dstate;
    a.beta = beta; a.alpha = alpha;
    a.vec_ok = 1;
    a.stall = inject_stall();
    return from_cuda(mmscan::launch_scan_seg_split(a, dims->io, seg_len, 1, nullptr, seq_first / seg_len,
                                                   seqlen_total, dests, ndest, static_cast<cudaStream_t>(stream)),
                     "mm_scan_fwd_split_maps_peers launch");
}

mm_status mm_scan_fwd_split_correct(const void* delta, const float* A, const void* C, const float* h0,
                                    const float* v0, float beta, float alpha, void* y, float* hT, float* vT,
                                    const void* maps_all, int64_t seg_len, int64_t seq_first,
                                    int64_t seqlen_total, const mm_scan_dims* dims, void* stream) {
    if (!dims) return fail(MM_ERR_NULL, "dims is NULL");
    if (!delta || !A || !C || !y || !maps_all)
        return fail(MM_ERR_NULL, "delta, A, C, y and maps_all are required");
    ScanSizes zs;
    if (mm_status st = check_scan_dims(dims, beta, alpha, &zs)) return st;
    if (mm_status st = check_split(dims, zs, seg_len, seq_first, seqlen_total)) return st;
    const void* ptrs[] = {delta, A, C, h0, v0, y, hT, vT, maps_all};
    const char* names[] = {"delta", "A", "C", "h0", "v0", "y", "hT", "vT", "maps_all"};
    for (int i = 0; i < 9; ++i)
        if (ptrs[i] && !aligned16(ptrs[i])) return fail(MM_ERR_ALIGN, "%s is not 16-byte aligned", names[i]);
    int64_t maps_bytes = 0;
    if (!split_record_bytes(dims->batch, dims->dim, (seqlen_total + seg_len - 1) / seg_len, &maps_bytes))
        return fail(MM_ERR_DIMS, "record bytes overflow 64 bits");
    const Range ry = rng("y", y, zs.seq_bytes), rhT = rng("hT", hT, zs.st_bytes), rvT = rng("vT", vT, zs.st_bytes);
    const Range ins[] = {rng("delta", delta, zs.seq_bytes), rng("A", A, zs.a_bytes), rng("C", C, zs.bc_bytes),
                         rng("h0", h0, zs.st_bytes), rng("v0", v0, zs.st_bytes),
                         rng("maps_all", maps_all, maps_bytes)};
    for (const Range* out : {&ry, &rhT, &rvT})
        for (const Range& in : ins)
            if (overlap(*out, in)) return fail(MM_ERR_ALIAS, "%s overlaps %s", out->name, in.name);
    if (overlap(rhT, ry) || overlap(rvT, ry) || overlap(rhT, rvT))
        return fail(MM_ERR_ALIAS, "hT, vT and y overlap");
    if (inject_launch_failure()) return fail(MM_ERR_CUDA, "injected launch failure (MMSCAN_FAULT_INJECT)");
    mmscan::ScanArgs a{};
    a.x = nullptr; a.delta = delta; a.A = A; a.B = nullptr; a.C = C; a.h0 = h0; a.v0 = v0;
    a.y = y; a.hT = hT; a.vT = vT;
    a.batch = dims->batch; a.seqlen = dims->seqlen; a.dim = dims->dim; a.dstate = (int)dims->dstate;
    a.beta = beta; a.alpha = alpha;
    a.vec_ok = 1;
    a.stall = inject_stall();
    return from_cuda(mmscan::launch_scan_seg_split(a, dims->io, seg_len, 2, const_cast<void*>(maps_all),
                                                   seq_first / seg_len, seqlen_total, nullptr, 0,
                                                   static_cast<cudaStream_t>(stream)),
                     "mm_scan_fwd_split_correct launch");
}

mm_status mm_scan_fwd(const void* x, const void* delta, const float* A, const void* B,
                      const void* C, const float* h0, const float* v0, float beta, float alpha,
                      void* y, float* hT, float* vT, const mm_scan_dims* dims, void* stream) {
    return mm_scan_fwd_gated(x, delta, A, B, C, nullptr, nullptr, nullptr, 0, h0, v0, beta, alpha,
                             y, hT, vT, nullptr, dims, stream);
}

mm_status mm_scan_fwd_gated(const void* x, const void* delta, const float* A, const void* B,
                            const void* C, const float* Dskip, const void* z, const float* delta_bias,
                            int delta_softplus, const float* h0, const float* v0, float beta,
                            float alpha, void* y, float* hT, float* vT, float* ckpt,
                            const mm_scan_dims* dims, void* stream) {
    if (!dims) return fail(MM_ERR_NULL, "dims is NULL");
    if (!x || !delta || !A || !B || !C || !y)
        return fail(MM_ERR_NULL, "x, delta, A, B, C and y are required");
    ScanSizes zs;
    if (mm_status st = check_scan_dims(dims, beta, alpha, &zs)) return st;
    const int64_t bsz = dims->batch, L = dims->seqlen, D = dims->dim, N = dims->dstate;
    const int64_t esize = zs.esize, seq_bytes = zs.seq_bytes, bc_bytes = zs.bc_bytes,
                  a_bytes = zs.a_bytes, st_bytes = zs.st_bytes, d_bytes = zs.d_bytes;
    const void* ptrs[] = {x, delta, A, B, C, h0, v0, y, hT, vT, Dskip, z, delta_bias, ckpt};
    const char* names[] = {"x", "delta", "A", "B", "C", "h0", "v0", "y", "hT", "vT", "D", "z",
                           "delta_bias", "ckpt"};
    for (int i = 0; i < 14; ++i)
        if (ptrs[i] && !aligned16(ptrs[i]))
            return fail(MM_ERR_ALIGN, "%s is not 16-byte aligned", names[i]);

    const Range rx = rng("x", x, seq_bytes), rd = rng("delta", delta, seq_bytes),
                rA = rng("A", A, a_bytes), rB = rng("B", B, bc_bytes), rC = rng("C", C, bc_bytes),
                rh0 = rng("h0", h0, st_bytes), rv0 = rng("v0", v0, st_bytes),
                ry = rng("y", y, seq_bytes), rhT = rng("hT", hT, st_bytes),
                rvT = rng("vT", vT, st_bytes), rD = rng("D", Dskip, d_bytes),
                rz = rng("z", z, seq_bytes), rbias = rng("delta_bias", delta_bias, d_bytes),
                rck = rng("ckpt", ckpt, zs.ck_bytes);
    const Range* inputs[] = {&rx, &rd, &rA, &rB, &rC, &rh0, &rv0, &rD, &rz, &rbias};
    for (const Range* in : inputs) {
        if (overlap(ry, *in)) return fail(MM_ERR_ALIAS, "y overlaps %s", in->name);
        if (overlap(rck, *in)) return fail(MM_ERR_ALIAS, "ckpt overlaps %s", in->name);
    }
    for (const Range* out : {&ry, &rhT, &rvT})
        if (overlap(rck, *out)) return fail(MM_ERR_ALIAS, "ckpt overlaps %s", out->name);
    for (const Range* out : {&rhT, &rvT}) {
        for (const Range* in : inputs) {
            const bool same_state = (out == &rhT && in == &rh0) || (out == &rvT && in == &rv0);
            if (!overlap(*out, *in)) continue;
            if (same_state && out->lo == in->lo) continue;   // in-place streaming
            return fail(MM_ERR_ALIAS, "%s overlaps %s", out->name, in->name);
        }
        if (overlap(*out, ry)) return fail(MM_ERR_ALIAS, "%s overlaps y", out->name);
    }
    if (overlap(rhT, rvT)) return fail(MM_ERR_ALIAS, "hT overlaps vT");
    if (inject_launch_failure()) return fail(MM_ERR_CUDA, "injected launch failure (MMSCAN_FAULT_INJECT)");

    mmscan::ScanArgs a{};
    a.x = x; a.delta = delta; a.A = A; a.B = B; a.C = C; a.h0 = h0; a.v0 = v0;
    a.y = y; a.hT = hT; a.vT = vT;
    a.batch = bsz; a.seqlen = L; a.dim = D; a.dstate = (int)N;
    a.beta = beta; a.alpha = alpha;
    a.vec_ok = ((L * esize) % 16) == 0;
    a.Dskip = Dskip; a.z = z; a.dbias = delta_bias; a.softplus = delta_softplus ? 1 : 0;
    a.ext = (Dskip || z || delta_bias || delta_softplus) ? 1 : 0;
    a.ckpt = ckpt;
    a.stall = inject_stall();
    a.deny_records = inject_records_denied();
    if (!a.ext && !ckpt) {
        const int64_t seg = seg_len_for(bsz, L, D, N, dims->io, a.vec_ok != 0);
        if (seg > 0) {
            // in-place streaming (hT = h0 or vT = v0) needs the fused launch, whose CTAs
            // all read the initial state before any writes the final one
            const bool fused = g_forced_path.load() == 3 || (hT && hT == h0) || (vT && vT == v0);
            return from_cuda(mmscan::launch_scan_seg(a, dims->io, seg, fused, static_cast<cudaStream_t>(stream)),
                             "mm_scan_fwd launch");
        }
    }
    const mmscan::ScanTileChoice t =
        mmscan::choose_scan_tile(bsz, D, N, dims->io, g_forced_spt.load(), g_forced_warps.load(),
                                 g_forced_ts.load());
    return from_cuda(mmscan::launch_scan_fwd(a, t, dims->io, static_cast<cudaStream_t>(stream)),
                     "mm_scan_fwd launch");
}

mm_status mm_scan_ckpt_size(const mm_scan_dims* dims, size_t* bytes) {
    if (!dims || !bytes) return fail(MM_ERR_NULL, "dims and bytes are required");
    ScanSizes zs;
    if (mm_status st = check_scan_dims(dims, 0.0f, 1.0f, &zs)) return st;
    *bytes = static_cast<size_t>(zs.ck_bytes);
    return ok();
}

mm_status mm_scan_bwd(const void* x, const void* delta, const float* A, const void* B, const void* C,
                      const float* h0, const float* v0, float beta, float alpha, const float* ckpt,
                      const void* dy, const float* dhT, const float* dvT, void* dx, void* ddelta,
                      float* dA, float* dB, float* dC, float* dh0, float* dv0,
                      const mm_scan_dims* dims, void* stream) {
    return mm_scan_bwd_gated(x, delta, A, B, C, nullptr, nullptr, nullptr, 0, h0, v0, beta, alpha, ckpt,
                             dy, dhT, dvT, dx, ddelta, dA, dB, dC, nullptr, nullptr, nullptr, dh0, dv0,
                             dims, stream);
}

mm_status mm_scan_bwd_gated(const void* x, const void* delta, const float* A, const void* B,
                            const void* C, const float* Dskip, const void* z, const float* delta_bias,
                            int delta_softplus, const float* h0, const float* v0, float beta, float alpha,
                            const float* ckpt, const void* dy, const float* dhT, const float* dvT,
                            void* dx, void* ddelta, float* dA, float* dB, float* dC, float* dD,
                            void* dz, float* ddelta_bias, float* dh0, float* dv0,
                            const mm_scan_dims* dims, void* stream) {
    if (!dims) return fail(MM_ERR_NULL, "dims is NULL");
    if (!x || !delta || !A || !B || !C || !dy || !dx || !ddelta || !dA || !dB || !dC)
        return fail(MM_ERR_NULL, "x, delta, A, B, C, dy, dx, ddelta, dA, dB and dC are required");
    ScanSizes zs;
    if (mm_status st = check_scan_dims(dims, beta, alpha, &zs)) return st;
    const int64_t L = dims->seqlen;
    if (!ckpt && L > MM_SCAN_CKPT_STEPS)
        return fail(MM_ERR_NULL, "ckpt is required when seqlen > %d", MM_SCAN_CKPT_STEPS);
    const void* ptrs[] = {x, delta, A, B, C, h0, v0, ckpt, dy, dhT, dvT, dx, ddelta, dA, dB, dC, dh0, dv0,
                          Dskip, z, delta_bias, dD, dz, ddelta_bias};
    const char* names[] = {"x", "delta", "A", "B", "C", "h0", "v0", "ckpt", "dy", "dhT", "dvT",
                           "dx", "ddelta", "dA", "dB", "dC", "dh0", "dv0", "D", "z", "delta_bias",
                           "dD", "dz", "ddelta_bias"};
    for (int i = 0; i < 24; ++i)
        if (ptrs[i] && !aligned16(ptrs[i]))
            return fail(MM_ERR_ALIGN, "%s is not 16-byte aligned", names[i]);
    const Range in_r[] = {rng("x", x, zs.seq_bytes), rng("delta", delta, zs.seq_bytes),
                          rng("A", A, zs.a_bytes), rng("B", B, zs.bc_bytes), rng("C", C, zs.bc_bytes),
                          rng("h0", h0, zs.st_bytes), rng("v0", v0, zs.st_bytes),
                          rng("ckpt", ckpt, zs.ck_bytes), rng("dy", dy, zs.seq_bytes),
                          rng("dhT", dhT, zs.st_bytes), rng("dvT", dvT, zs.st_bytes),
                          rng("D", Dskip, zs.d_bytes), rng("z", z, zs.seq_bytes),
                          rng("delta_bias", delta_bias, zs.d_bytes)};
    const Range out_r[] = {rng("dx", dx, zs.seq_bytes), rng("ddelta", ddelta, zs.seq_bytes),
                           rng("dA", dA, zs.a_bytes), rng("dB", dB, zs.bcf_bytes),
                           rng("dC", dC, zs.bcf_bytes), rng("dh0", dh0, zs.st_bytes),
                           rng("dv0", dv0, zs.st_bytes), rng("dD", dD, zs.d_bytes),
                           rng("dz", dz, zs.seq_bytes), rng("ddelta_bias", ddelta_bias, zs.d_bytes)};
    for (const Range& o : out_r) {
        for (const Range& in : in_r)
            if (overlap(o, in)) return fail(MM_ERR_ALIAS, "%s overlaps %s", o.name, in.name);
        for (const Range& o2 : out_r)
            if (&o2 != &o && overlap(o, o2)) return fail(MM_ERR_ALIAS, "%s overlaps %s", o.name, o2.name);
    }
    if (inject_launch_failure()) return fail(MM_ERR_CUDA, "injected launch failure (MMSCAN_FAULT_INJECT)");

    mmscan::ScanBwdArgs a{};
    a.x = x; a.delta = delta; a.A = A; a.B = B; a.C = C; a.h0 = h0; a.v0 = v0; a.ckpt = ckpt;
    a.dout = dy; a.dhT = dhT; a.dvT = dvT;
    a.dx = dx; a.ddelta = ddelta; a.dA = dA; a.dB = dB; a.dC = dC; a.dh0 = dh0; a.dv0 = dv0;
    a.batch = dims->batch; a.seqlen = L; a.dim = dims->dim; a.dstate = (int)dims->dstate;
    a.beta = beta; a.alpha = alpha;
    a.vec_ok = ((L * zs.esize) % 16) == 0;
    a.Dskip = Dskip; a.z = z; a.dbias = delta_bias; a.softplus = delta_softplus ? 1 : 0;
    a.ext = (Dskip || z || delta_bias || delta_softplus) ? 1 : 0;
    a.dD = a.ext ? dD : nullptr;
    a.dz = z ? dz : nullptr;
    a.ddbias = a.ext ? ddelta_bias : nullptr;
    a.stall = inject_stall();
    a.det = g_deterministic.load();
    if (a.det) {
        // the deterministic form allocates its workspace on the stream: not while
        // the stream is being captured into a graph
        if (mmscan::stream_capturing(static_cast<cudaStream_t>(stream)))
            return fail(MM_ERR_UNSUPPORTED, "the deterministic backward allocates its workspace on the stream; "
                                            "it does not run while the stream is being captured");
        if (mmscan::scan_bwd_det_workspace_bytes(a.batch, a.dim, a.dstate, L) < 0)
            return fail(MM_ERR_UNSUPPORTED, "the deterministic backward's workspace overflows 64 bits");
    }
    return from_cuda(mmscan::launch_scan_bwd(a, dims->io, static_cast<cudaStream_t>(stream)),
                     "mm_scan_bwd launch");
}

mm_status mm_scan_step(const void* x, const void* delta, const float* A, const void* B, const void* C,
                       const float* Dskip, const void* z, const float* delta_bias, int delta_softplus,
                       float* h, float* v, float beta, float alpha, void* y, const mm_scan_dims* dims,
                       void* stream) {
    if (!dims) return fail(MM_ERR_NULL, "dims is NULL");
    if (!x || !delta || !A || !B || !C || !h || !v || !y)
        return fail(MM_ERR_NULL, "x, delta, A, B, C, h, v and y are required");
    if (dims->seqlen != 1) return fail(MM_ERR_DIMS, "a decode step has seqlen 1 (got %lld)",
                                       (long long)dims->seqlen);
    ScanSizes zs;
    if (mm_status st = check_scan_dims(dims, beta, alpha, &zs)) return st;
    const void* ptrs[] = {x, delta, A, B, C, Dskip, z, delta_bias, h, v, y};
    const char* names[] = {"x", "delta", "A", "B", "C", "D", "z", "delta_bias", "h", "v", "y"};
    for (int i = 0; i < 11; ++i)
        if (ptrs[i] && !aligned16(ptrs[i]))
            return fail(MM_ERR_ALIGN, "%s is not 16-byte aligned", names[i]);
    const Range in_r[] = {rng("x", x, zs.seq_bytes), rng("delta", delta, zs.seq_bytes),
                          rng("A", A, zs.a_bytes), rng("B", B, zs.bc_bytes), rng("C", C, zs.bc_bytes),
                          rng("D", Dskip, zs.d_bytes), rng("z", z, zs.seq_bytes),
                          rng("delta_bias", delta_bias, zs.d_bytes)};
    const Range out_r[] = {rng("h", h, zs.st_bytes), rng("v", v, zs.st_bytes), rng("y", y, zs.seq_bytes)};
    for (const Range& o : out_r) {
        for (const Range& in : in_r)
            if (overlap(o, in)) return fail(MM_ERR_ALIAS, "%s overlaps %s", o.name, in.name);
        for (const Range& o2 : out_r)
            if (&o2 != &o && overlap(o, o2)) return fail(MM_ERR_ALIAS, "%s overlaps %s", o.name, o2.name);
    }
    if (inject_launch_failure()) return fail(MM_ERR_CUDA, "injected launch failure (MMSCAN_FAULT_INJECT)");
    mmscan::ScanStepArgs a{};
    a.x = x; a.delta = delta; a.A = A; a.B = B; a.C = C;
    a.Dskip = Dskip; a.z = z; a.dbias = delta_bias; a.softplus = delta_softplus ? 1 : 0;
    a.ext = (Dskip || z || delta_bias || delta_softplus) ? 1 : 0;
    a.h = h; a.v = v; a.y = y;
    a.batch = dims->batch; a.dim = dims->dim; a.dstate = (int)dims->dstate;
    a.vec = (dims->dstate % 4) == 0;
    a.beta = beta; a.alpha = alpha;
    return from_cuda(mmscan::launch_scan_step(a, dims->io, static_cast<cudaStream_t>(stream)),
                     "mm_scan_step launch");
}

mm_status mm_ssd_fwd(const void* x, const float* delta, const float* A, const void* B,
                     const void* C, const float* h0, float beta, float alpha, void* y, float* hT,
                     const mm_ssd_dims* dims, void* stream) {
    if (!dims) return fail(MM_ERR_NULL, "dims is NULL");
    if (!x || !delta || !A || !B || !C || !y)
        return fail(MM_ERR_NULL, "x, delta, A, B, C and y are required");
    if (dims->batch < 1 || dims->seqlen < 1 || dims->nheads < 1 || dims->headdim < 1 ||
        dims->dstate < 1 || dims->ngroups < 1 || dims->chunk < 1 ||
        dims->nheads % dims->ngroups != 0)
        return fail(MM_ERR_DIMS, "invalid SSD sizes");
    if (mm_status st = check_ssd_range(dims)) return st;
    if (!mmscan::ssd_shape_supported(dims->headdim, dims->dstate, dims->chunk))
        return fail(MM_ERR_UNSUPPORTED, "SSD with headdim=%lld dstate=%lld chunk=%lld is not built",
                    (long long)dims->headdim, (long long)dims->dstate, (long long)dims->chunk);
    if (!std::isfinite(beta) || beta < 0.0f || beta >= 1.0f)
        return fail(MM_ERR_SCALAR, "beta=%g is outside [0, 1)", (double)beta);
    if (beta != 0.0f)       // momentum: the chunked form with two carried states
        return mm_ssd_fwd_momentum(x, delta, A, B, C, h0, nullptr, beta, alpha, y, hT, nullptr, dims, stream);
    if (!std::isfinite(alpha) || alpha < 0.0f)
        return fail(MM_ERR_SCALAR, "alpha=%g must be finite and >= 0", (double)alpha);
    const int64_t bsz = dims->batch, L = dims->seqlen, H = dims->nheads, P = dims->headdim,
                  N = dims->dstate, G = dims->ngroups;
    int64_t blh, xy_bytes, bl, d_bytes, blg, bc_elems, bc_bytes, st_elems, st_bytes;
    int64_t bh, pn;
    if (!mul_ok(bsz, L, &bl) || !mul_ok(bl, H, &blh) || !mul_ok(blh, P * 2, &xy_bytes) ||
        !mul_ok(bl, H * 4, &d_bytes) || !mul_ok(bl, G, &blg) || !mul_ok(blg, N, &bc_elems) ||
        !mul_ok(bc_elems, 2, &bc_bytes) || !mul_ok(bsz, H, &bh) || !mul_ok(P, N, &pn) ||
        !mul_ok(bh, pn, &st_elems) || !mul_ok(st_elems, 4, &st_bytes))
        return fail(MM_ERR_DIMS, "sizes overflow 64-bit byte counts");
    const void* ptrs[] = {x, delta, A, B, C, h0, y, hT};
    const char* names[] = {"x", "delta", "A", "B", "C", "h0", "y", "hT"};
    for (int i = 0; i < 8; ++i)
        if (ptrs[i] && !aligned16(ptrs[i]))
            return fail(MM_ERR_ALIGN, "%s is not 16-byte aligned", names[i]);
    const Range rx = rng("x", x, xy_bytes), rd = rng("delta", delta, d_bytes),
                rA = rng("A", A, H * 4), rB = rng("B", B, bc_bytes), rC = rng("C", C, bc_bytes),
                rh0 = rng("h0", h0, st_bytes), ry = rng("y", y, xy_bytes),
                rhT = rng("hT", hT, st_bytes);
    const Range* inputs[] = {&rx, &rd, &rA, &rB, &rC, &rh0};
    for (const Range* out : {&ry, &rhT}) {
        for (const Range* in : inputs) {
            if (!overlap(*out, *in)) continue;
            if (out == &rhT && in == &rh0 && out->lo == in->lo) continue;
            return fail(MM_ERR_ALIAS, "%s overlaps %s", out->name, in->name);
        }
    }
    if (overlap(ry, rhT)) return fail(MM_ERR_ALIAS, "y overlaps hT");
    if (inject_launch_failure()) return fail(MM_ERR_CUDA, "injected launch failure (MMSCAN_FAULT_INJECT)");

    mmscan::SSDArgs a{};
    a.x = x; a.delta = delta; a.A = A; a.B = B; a.C = C; a.h0 = h0; a.y = y; a.hT = hT;
    a.batch = bsz; a.seqlen = L; a.nheads = H; a.headdim = P; a.dstate = N; a.ngroups = G;
    a.chunk = dims->chunk; a.alpha = alpha;
    a.stall = inject_stall();
    return from_cuda(mmscan::launch_ssd_fwd(a, static_cast<cudaStream_t>(stream)), "mm_ssd_fwd launch");
}

mm_status mm_ssd_fwd_momentum(const void* x, const float* delta, const float* A, const void* B,
                              const void* C, const float* h0, const float* v0, float beta, float alpha,
                              void* y, float* hT, float* vT, const mm_ssd_dims* dims, void* stream) {
    if (!dims) return fail(MM_ERR_NULL, "dims is NULL");
    if (!x || !delta || !A || !B || !C || !y)
        return fail(MM_ERR_NULL, "x, delta, A, B, C and y are required");
    const int64_t bsz = dims->batch, L = dims->seqlen, H = dims->nheads, P = dims->headdim,
                  N = dims->dstate, G = dims->ngroups;
    if (bsz < 1 || L < 1 || H < 1 || P < 1 || N < 1 || G < 1 || dims->chunk < 1 || H % G != 0)
        return fail(MM_ERR_DIMS, "sizes must be >= 1 and ngroups must divide nheads");
    if (mm_status st = check_ssd_range(dims)) return st;
    if (!mmscan::ssd_mom_shape_supported(P, N))
        return fail(MM_ERR_UNSUPPORTED, "momentum SSD needs headdim <= 64 and dstate <= 128 (got %lld, %lld)",
                    (long long)P, (long long)N);
    if (!std::isfinite(beta) || beta < 0.0f || beta >= 1.0f)
        return fail(MM_ERR_SCALAR, "beta=%g is outside [0, 1)", (double)beta);
    if (!std::isfinite(alpha) || alpha < 0.0f)
        return fail(MM_ERR_SCALAR, "alpha=%g must be finite and >= 0", (double)alpha);
    int64_t blh, xy_bytes, bl, d_bytes, blg, bc_elems, bc_bytes, st_elems, st_bytes;
    int64_t bh, pn;
    if (!mul_ok(bsz, L, &bl) || !mul_ok(bl, H, &blh) || !mul_ok(blh, P * 2, &xy_bytes) ||
        !mul_ok(bl, H * 4, &d_bytes) || !mul_ok(bl, G, &blg) || !mul_ok(blg, N, &bc_elems) ||
        !mul_ok(bc_elems, 2, &bc_bytes) || !mul_ok(bsz, H, &bh) || !mul_ok(P, N, &pn) ||
        !mul_ok(bh, pn, &st_elems) || !mul_ok(st_elems, 4, &st_bytes))
        return fail(MM_ERR_DIMS, "sizes overflow 64-bit byte counts");
    const void* ptrs[] = {x, delta, A, B, C, h0, v0, y, hT, vT};
    const char* names[] = {"x", "delta", "A", "B", "C", "h0", "v0", "y", "hT", "vT"};
    for (int i = 0; i < 10; ++i)
        if (ptrs[i] && !aligned16(ptrs[i]))
            return fail(MM_ERR_ALIGN, "%s is not 16-byte aligned", names[i]);
    const Range rx = rng("x", x, xy_bytes), rd = rng("delta", delta, d_bytes), rA = rng("A", A, H * 4),
                rB = rng("B", B, bc_bytes), rC = rng("C", C, bc_bytes), rh0 = rng("h0", h0, st_bytes),
                rv0 = rng("v0", v0, st_bytes), ry = rng("y", y, xy_bytes), rhT = rng("hT", hT, st_bytes),
                rvT = rng("vT", vT, st_bytes);
    const Range* inputs[] = {&rx, &rd, &rA, &rB, &rC, &rh0, &rv0};
    for (const Range* out : {&ry, &rhT, &rvT}) {
        for (const Range* in : inputs) {
            if (!overlap(*out, *in)) continue;
            const bool same_state = (out == &rhT && in == &rh0) || (out == &rvT && in == &rv0);
            if (same_state && out->lo == in->lo) continue;   // in-place streaming
            return fail(MM_ERR_ALIAS, "%s overlaps %s", out->name, in->name);
        }
    }
    if (overlap(ry, rhT) || overlap(ry, rvT) || overlap(rhT, rvT))
        return fail(MM_ERR_ALIAS, "outputs overlap");
    if (inject_launch_failure()) return fail(MM_ERR_CUDA, "injected launch failure (MMSCAN_FAULT_INJECT)");
    mmscan::SSDMomArgs a{};
    a.x = x; a.delta = delta; a.A = A; a.B = B; a.C = C; a.h0 = h0; a.v0 = v0;
    a.y = y; a.hT = hT; a.vT = vT;
    a.batch = bsz; a.seqlen = L; a.nheads = H; a.headdim = P; a.dstate = N; a.ngroups = G;
    a.beta = beta; a.alpha = alpha;
    a.stall = inject_stall();
    if (mmscan::ssd_mom_tc_shape_supported(P, N))
        return from_cuda(mmscan::launch_ssd_mom_tc(a, static_cast<cudaStream_t>(stream)),
                         "mm_ssd_fwd_momentum launch");
    return from_cuda(mmscan::launch_ssd_mom(a, static_cast<cudaStream_t>(stream)), "mm_ssd_fwd_momentum launch");
}

}  // extern "C"
