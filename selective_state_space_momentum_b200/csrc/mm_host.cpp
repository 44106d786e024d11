// mm_host.cpp -- the host-buffer entry points of libmmscan (mm_scan_fwd_host,
// mm_ssd_fwd_host and their workspace queries; declared in include/mm_scan.h).
//
// A call streams its tensors through a caller-provided device workspace in
// time chunks.  Chunk i's inputs are copied in on one stream, its device call
// (mm_scan_fwd_gated, mm_ssd_fwd or mm_ssd_fwd_momentum on device pointers)
// runs on the caller's stream, and its outputs are copied out on a third
// stream, so that with page-locked host memory the two directions of the
// host link and the kernels all overlap.  The chunks rotate through a ring of
// kSlots workspace slots.  The states carried from chunk to chunk stay on the
// device and are updated in place (the device calls allow hT == h0 and
// vT == v0), so a chunked call computes exactly what the streaming rule of
// the device call gives for the same split.
//
// Ordering (each arrow an event wait; K = slots):
//   copy-in(i)   after  device-call(i - K)   the slot's inputs were consumed
//   device-call(i) after copy-in(i)          its inputs have landed
//   device-call(i) after copy-out(i - K)     the slot's outputs were drained
//   copy-out(i)  after  device-call(i)       its outputs are complete
// plus a fork (the copy-in stream starts after the work queued on the
// caller's stream before the call; the copy-out stream only ever follows
// device calls queued after that) and a join (the caller's stream continues
// after the last copy-out).  Every copy is one cudaMemcpy2DAsync of a (rows, n steps)
// block of a (rows, L steps) host tensor, or one copy per row where a pitch is
// beyond what one 2D copy takes.
#include "mm_scan.h"

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "mm_internal.h"

namespace {

constexpr int kSlots = 3;
constexpr size_t kAlign = 256;
// Pitches of one 2D copy stay below 2^31 bytes; longer rows go one by one.
constexpr size_t kMaxPitch = (size_t(1) << 31) - 1;
// Automatic chunk length: about 1/32 of the call's streamed bytes per chunk,
// at least 32 MB (each chunk costs some tens of microseconds of copy and
// launch set-up), and host rows of at least 2 KB per copy.
constexpr int64_t kChunksTarget = 32;
constexpr int64_t kMinChunkBytes = int64_t(32) << 20;
constexpr int64_t kMinRowBytes = 2048;

bool mul(int64_t a, int64_t b, int64_t* out) {
    if (a < 0 || b < 0) return false;
    if (a != 0 && b > INT64_MAX / a) return false;
    *out = a * b;
    return true;
}

bool add(int64_t a, int64_t b, int64_t* out) {
    if (a < 0 || b < 0 || a > INT64_MAX - b) return false;
    *out = a + b;
    return true;
}

bool round_up(int64_t a, int64_t* out) {
    if (a < 0 || a > INT64_MAX - int64_t(kAlign)) return false;
    *out = (a + int64_t(kAlign) - 1) / int64_t(kAlign) * int64_t(kAlign);
    return true;
}

// One tensor streamed along time: on the host `rows` rows of L steps of
// `step` bytes (row pitch L * step); in a slot, a dense (rows, n, step) block.
struct Streamed {
    const char* name;
    char* host;
    int64_t rows, step;
    bool out;
    int64_t off;          // offset of its block inside a slot
};

// A tensor copied once: in before the first chunk and/or out after the last.
struct Held {
    const char* name;
    const void* in;       // host source, or null
    void* out;            // host destination, or null
    int64_t bytes;
    int64_t off;          // offset inside the fixed area
};

struct Plan {
    std::vector<Streamed> st;
    std::vector<Held> held;
    int64_t L = 0, chunk = 0, nchunks = 0;
    int slots = 0;
    int64_t fixed_bytes = 0, slot_bytes = 0, total = 0;
};

// Chunk length, slot count and workspace offsets.  `unit` is the step count
// the automatic chunk length is a multiple of; chunk_steps > 0 overrides it.
mm_status lay_out(Plan* p, int64_t L, int64_t chunk_steps, int64_t unit) {
    if (chunk_steps < 0)
        return mmscan::report(MM_ERR_DIMS, "chunk_steps=%lld must be >= 0 (0: automatic)", (long long)chunk_steps);
    int64_t per_step = 0, min_step = INT64_MAX;
    for (const Streamed& s : p->st) {
        int64_t b;
        if (!mul(s.rows, s.step, &b) || !add(per_step, b, &per_step))
            return mmscan::report(MM_ERR_DIMS, "sizes overflow 64-bit byte counts");
        if (s.step < min_step) min_step = s.step;
    }
    int64_t chunk = chunk_steps;
    if (chunk == 0) {
        int64_t total;
        if (!mul(per_step, L, &total)) return mmscan::report(MM_ERR_DIMS, "sizes overflow 64-bit byte counts");
        int64_t target = total / kChunksTarget;
        if (target < kMinChunkBytes) target = kMinChunkBytes;
        chunk = target / (per_step > 0 ? per_step : 1);
        const int64_t min_rows = (kMinRowBytes + min_step - 1) / min_step;
        if (chunk < min_rows) chunk = min_rows;
        chunk = (chunk + unit - 1) / unit * unit;
    }
    if (chunk > L) chunk = L;
    p->L = L;
    p->chunk = chunk;
    p->nchunks = (L + chunk - 1) / chunk;
    p->slots = p->nchunks < kSlots ? int(p->nchunks) : kSlots;
    int64_t off = 0;
    for (Held& h : p->held) {
        h.off = off;
        int64_t r;
        if (!round_up(h.bytes, &r) || !add(off, r, &off))
            return mmscan::report(MM_ERR_DIMS, "sizes overflow 64-bit byte counts");
    }
    p->fixed_bytes = off;
    off = 0;
    for (Streamed& s : p->st) {
        s.off = off;
        int64_t b, c, r;
        if (!mul(s.rows, s.step, &b) || !mul(b, chunk, &c) || !round_up(c, &r) || !add(off, r, &off))
            return mmscan::report(MM_ERR_DIMS, "sizes overflow 64-bit byte counts");
    }
    p->slot_bytes = off;
    int64_t ring;
    if (!mul(off, p->slots, &ring) || !add(p->fixed_bytes, ring, &p->total))
        return mmscan::report(MM_ERR_DIMS, "sizes overflow 64-bit byte counts");
    return MM_OK;
}

// Copy `rows` rows of `width` bytes between pitched buffers.
cudaError_t copy_rows(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width, int64_t rows,
                      cudaMemcpyKind kind, cudaStream_t s) {
    if (rows == 1 || (dpitch == width && spitch == width))
        return cudaMemcpyAsync(dst, src, width * size_t(rows), kind, s);
    if (dpitch <= kMaxPitch && spitch <= kMaxPitch)
        return cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, size_t(rows), kind, s);
    for (int64_t r = 0; r < rows; ++r) {
        const cudaError_t e = cudaMemcpyAsync(static_cast<char*>(dst) + size_t(r) * dpitch,
                                              static_cast<const char*>(src) + size_t(r) * spitch, width, kind, s);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// The side streams and events of the pipeline, created on first use and
// kept per host thread and device (thread_local below), so that a call pays
// no creation cost.  Reusing them across calls is safe: each call's first
// wait on the caller's stream orders it after the previous call's join.
struct Resources {
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    cudaEvent_t ev_in[kSlots] = {}, ev_comp[kSlots] = {}, ev_out[kSlots] = {};

    cudaError_t create() {
        cudaError_t e;
        if ((e = cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking)) != cudaSuccess) return e;
        for (cudaEvent_t* ev : {&fork, &join})
            if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return e;
        for (int k = 0; k < kSlots; ++k)
            for (cudaEvent_t* ev : {&ev_in[k], &ev_comp[k], &ev_out[k]})
                if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return e;
        return cudaSuccess;
    }

    // Destroying a stream or an event with work still pending is allowed:
    // the runtime frees it once that work completes.
    void release() {
        for (int k = 0; k < kSlots; ++k)
            for (cudaEvent_t* ev : {&ev_in[k], &ev_comp[k], &ev_out[k]})
                if (*ev) cudaEventDestroy(*ev), *ev = nullptr;
        for (cudaEvent_t* ev : {&fork, &join})
            if (*ev) cudaEventDestroy(*ev), *ev = nullptr;
        if (in) cudaStreamDestroy(in), in = nullptr;
        if (out) cudaStreamDestroy(out), out = nullptr;
    }
};

struct ThreadResources {
    struct Entry {
        int device;
        Resources* r;
    };
    std::vector<Entry> per_device;
    void release() {
        for (Entry& e : per_device) {
            e.r->release();
            delete e.r;
        }
        per_device.clear();
    }
    ~ThreadResources() { release(); }
};

thread_local ThreadResources t_resources;

cudaError_t resources(Resources** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    for (const ThreadResources::Entry& en : t_resources.per_device)
        if (en.device == dev) {
            *out = en.r;
            return cudaSuccess;
        }
    Resources* r = new Resources;
    if ((e = r->create()) != cudaSuccess) {
        r->release();
        delete r;
        return e;
    }
    t_resources.per_device.push_back({dev, r});
    *out = r;
    return cudaSuccess;
}

// The device call of one chunk: steps [t0, t0 + n) with the slot's block
// pointers (one per Streamed, in order), the fixed area and whether this is
// the first chunk (the carried states then come from the host, or are zero).
struct ChunkCall {
    virtual mm_status operator()(int64_t t0, int64_t n, char* const* blk, char* fixed, bool first,
                                 cudaStream_t s) const = 0;
    virtual ~ChunkCall() = default;
};

mm_status cuda_fail(cudaError_t e, const char* what) {
    return mmscan::report(MM_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

// Checks shared by both entries: the workspace is device memory, 16-byte
// aligned and large enough; every host pointer is not device memory.
mm_status check_buffers(const Plan& p, void* ws, size_t ws_bytes) {
    if (!ws) return mmscan::report(MM_ERR_NULL, "workspace is NULL");
    if ((reinterpret_cast<uintptr_t>(ws) & 15u) != 0)
        return mmscan::report(MM_ERR_ALIGN, "workspace is not 16-byte aligned");
    if (uint64_t(ws_bytes) < uint64_t(p.total))
        return mmscan::report(MM_ERR_DIMS, "workspace has %llu bytes, the call needs %lld", (unsigned long long)ws_bytes,
                              (long long)p.total);
    cudaPointerAttributes at;
    std::memset(&at, 0, sizeof(at));
    cudaError_t e = cudaPointerGetAttributes(&at, ws);
    if (e != cudaSuccess) return cuda_fail(e, "workspace attributes");
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
        return mmscan::report(MM_ERR_UNSUPPORTED, "workspace is not device memory");
    auto host_ok = [&](const char* name, const void* ptr) -> mm_status {
        if (!ptr) return MM_OK;
        cudaPointerAttributes a;
        std::memset(&a, 0, sizeof(a));
        const cudaError_t r = cudaPointerGetAttributes(&a, ptr);
        if (r != cudaSuccess) return cuda_fail(r, "host pointer attributes");
        if (a.type == cudaMemoryTypeDevice)
            return mmscan::report(MM_ERR_UNSUPPORTED, "%s is device memory: the host entry takes host buffers", name);
        return MM_OK;
    };
    for (const Streamed& s : p.st)
        if (mm_status st = host_ok(s.name, s.host)) return st;
    for (const Held& h : p.held) {
        if (mm_status st = host_ok(h.name, h.in)) return st;
        if (mm_status st = host_ok(h.name, h.out)) return st;
    }
    return MM_OK;
}

// Host ranges of the plan's tensors may not overlap, except a state's input
// and output at the same address (in-place streaming).
mm_status check_host_aliasing(const Plan& p) {
    struct R { const char* name; uintptr_t lo, hi; bool out; const void* pair; };
    std::vector<R> rs;
    for (const Streamed& s : p.st) {
        int64_t b = 0;
        mul(s.rows * s.step, p.L, &b);   // checked when the plan was laid out
        const uintptr_t lo = reinterpret_cast<uintptr_t>(s.host);
        rs.push_back({s.name, lo, lo + uintptr_t(b), s.out, nullptr});
    }
    for (const Held& h : p.held) {
        if (h.in) {
            const uintptr_t lo = reinterpret_cast<uintptr_t>(h.in);
            rs.push_back({h.name, lo, lo + uintptr_t(h.bytes), false, h.out});
        }
        if (h.out) {
            const uintptr_t lo = reinterpret_cast<uintptr_t>(h.out);
            rs.push_back({h.name, lo, lo + uintptr_t(h.bytes), true, h.in});
        }
    }
    for (size_t i = 0; i < rs.size(); ++i)
        for (size_t j = i + 1; j < rs.size(); ++j) {
            const R &a = rs[i], &b = rs[j];
            if (!a.out && !b.out) continue;                       // inputs may share memory
            if (a.lo >= b.hi || b.lo >= a.hi) continue;
            const bool same_state = a.pair && b.pair && a.lo == b.lo &&
                                    reinterpret_cast<uintptr_t>(a.pair) == b.lo;
            if (same_state) continue;
            return mmscan::report(MM_ERR_ALIAS, "host buffers %s and %s overlap", a.name, b.name);
        }
    return MM_OK;
}

// One chunk: everything on the caller's stream, in order.
mm_status run_single(const Plan& p, char* ws, cudaStream_t caller, const ChunkCall& call) {
    char* fixed = ws;
    char* slot = ws + p.fixed_bytes;
    std::vector<char*> blk(p.st.size());
    for (const Held& h : p.held) {
        if (!h.in) continue;
        const cudaError_t e = cudaMemcpyAsync(fixed + h.off, h.in, size_t(h.bytes), cudaMemcpyHostToDevice, caller);
        if (e != cudaSuccess) return cuda_fail(e, h.name);
    }
    for (size_t j = 0; j < p.st.size(); ++j) {
        const Streamed& s = p.st[j];
        blk[j] = slot + s.off;
        if (s.out) continue;
        const cudaError_t e = cudaMemcpyAsync(blk[j], s.host, size_t(s.rows * s.step * p.L), cudaMemcpyHostToDevice,
                                              caller);
        if (e != cudaSuccess) return cuda_fail(e, s.name);
    }
    if (mm_status st = call(0, p.L, blk.data(), fixed, true, caller)) return st;
    for (size_t j = 0; j < p.st.size(); ++j) {
        const Streamed& s = p.st[j];
        if (!s.out) continue;
        const cudaError_t e = cudaMemcpyAsync(s.host, blk[j], size_t(s.rows * s.step * p.L), cudaMemcpyDeviceToHost,
                                              caller);
        if (e != cudaSuccess) return cuda_fail(e, s.name);
    }
    for (const Held& h : p.held) {
        if (!h.out) continue;
        const cudaError_t e = cudaMemcpyAsync(h.out, fixed + h.off, size_t(h.bytes), cudaMemcpyDeviceToHost, caller);
        if (e != cudaSuccess) return cuda_fail(e, h.name);
    }
    return mmscan::report_ok();
}

mm_status run(const Plan& p, char* ws, cudaStream_t caller, const ChunkCall& call) {
    if (p.nchunks == 1) return run_single(p, ws, caller, call);
    Resources* rp = nullptr;
    cudaError_t e = resources(&rp);
    if (e != cudaSuccess) return cuda_fail(e, "host pipeline streams and events");
    Resources& r = *rp;
    char* fixed = ws;
    char* ring = ws + p.fixed_bytes;
    mm_status status = MM_OK;
    auto check = [&](cudaError_t err, const char* what) {
        if (err != cudaSuccess && status == MM_OK) status = cuda_fail(err, what);
        return err == cudaSuccess;
    };
    // fork: the copy-in stream starts after the caller's earlier work (the
    // copy-out stream waits for device calls queued after it anyway)
    bool ok = check(cudaEventRecord(r.fork, caller), "fork") &&
              check(cudaStreamWaitEvent(r.in, r.fork, 0), "fork");
    for (const Held& h : p.held) {
        if (!ok || !h.in) continue;
        ok = check(cudaMemcpyAsync(fixed + h.off, h.in, size_t(h.bytes), cudaMemcpyHostToDevice, r.in), h.name);
    }
    std::vector<char*> blk(p.st.size());
    for (int64_t i = 0; ok && i < p.nchunks; ++i) {
        const int k = int(i % p.slots);
        const int64_t t0 = i * p.chunk;
        const int64_t n = (p.L - t0) < p.chunk ? (p.L - t0) : p.chunk;
        char* slot = ring + k * p.slot_bytes;
        // copy-in
        if (i >= p.slots) ok = check(cudaStreamWaitEvent(r.in, r.ev_comp[k], 0), "copy-in wait");
        for (size_t j = 0; ok && j < p.st.size(); ++j) {
            const Streamed& s = p.st[j];
            blk[j] = slot + s.off;
            if (s.out) continue;
            ok = check(copy_rows(blk[j], size_t(n * s.step), s.host + t0 * s.step, size_t(p.L * s.step),
                                 size_t(n * s.step), s.rows, cudaMemcpyHostToDevice, r.in), s.name);
        }
        ok = ok && check(cudaEventRecord(r.ev_in[k], r.in), "copy-in record");
        // the chunk's device call, on the caller's stream
        ok = ok && check(cudaStreamWaitEvent(caller, r.ev_in[k], 0), "device-call wait");
        if (ok && i >= p.slots) ok = check(cudaStreamWaitEvent(caller, r.ev_out[k], 0), "device-call wait");
        if (ok) {
            const mm_status st = call(t0, n, blk.data(), fixed, i == 0, caller);
            if (st != MM_OK) {
                status = st;
                ok = false;
            }
        }
        ok = ok && check(cudaEventRecord(r.ev_comp[k], caller), "device-call record");
        // copy-out
        ok = ok && check(cudaStreamWaitEvent(r.out, r.ev_comp[k], 0), "copy-out wait");
        for (size_t j = 0; ok && j < p.st.size(); ++j) {
            const Streamed& s = p.st[j];
            if (!s.out) continue;
            ok = check(copy_rows(s.host + t0 * s.step, size_t(p.L * s.step), blk[j], size_t(n * s.step),
                                 size_t(n * s.step), s.rows, cudaMemcpyDeviceToHost, r.out), s.name);
        }
        ok = ok && check(cudaEventRecord(r.ev_out[k], r.out), "copy-out record");
    }
    for (const Held& h : p.held) {
        if (!ok || !h.out) continue;
        ok = check(cudaMemcpyAsync(h.out, fixed + h.off, size_t(h.bytes), cudaMemcpyDeviceToHost, r.out), h.name);
    }
    // join, also after a failure part-way, so that the caller's stream never
    // runs ahead of copies that were queued
    check(cudaEventRecord(r.join, r.out), "join");
    check(cudaStreamWaitEvent(caller, r.join, 0), "join");
    return status == MM_OK ? mmscan::report_ok() : status;
}

}  // namespace

namespace mmscan {
void host_pipeline_release() { t_resources.release(); }
}  // namespace mmscan

namespace {

int64_t scan_esize(const mm_scan_dims* d) { return d->io == MM_BF16 ? 2 : 4; }

// The plan of a scan call; host pointers may be null for a size query.
mm_status scan_plan(Plan* p, const mm_scan_dims* d, bool with_z, int64_t chunk_steps,
                    const void* x, const void* delta, const float* A, const void* B, const void* C,
                    const float* Dskip, const void* z, const float* bias, const float* h0, const float* v0,
                    void* y, float* hT, float* vT) {
    if (!d) return mmscan::report(MM_ERR_NULL, "dims is NULL");
    // the device call's size checks, on a call of the same sizes
    size_t ck;
    if (mm_status st = mm_scan_ckpt_size(d, &ck)) return st;
    const int64_t es = scan_esize(d), bsz = d->batch, D = d->dim, N = d->dstate;
    int64_t bd, bn, dn, bdn;
    if (!mul(bsz, D, &bd) || !mul(bsz, N, &bn) || !mul(D, N, &dn) || !mul(bd, N, &bdn))
        return mmscan::report(MM_ERR_DIMS, "sizes overflow 64-bit byte counts");
    char* cx = const_cast<char*>(static_cast<const char*>(x));
    p->st.push_back({"x", cx, bd, es, false, 0});
    p->st.push_back({"delta", const_cast<char*>(static_cast<const char*>(delta)), bd, es, false, 0});
    if (with_z) p->st.push_back({"z", const_cast<char*>(static_cast<const char*>(z)), bd, es, false, 0});
    p->st.push_back({"B", const_cast<char*>(static_cast<const char*>(B)), bn, es, false, 0});
    p->st.push_back({"C", const_cast<char*>(static_cast<const char*>(C)), bn, es, false, 0});
    p->st.push_back({"y", static_cast<char*>(y), bd, es, true, 0});
    p->held.push_back({"A", A, nullptr, dn * 4, 0});
    // D and delta_bias always have their place (2 * dim floats), used or not
    p->held.push_back({"D", Dskip, nullptr, D * 4, 0});
    p->held.push_back({"delta_bias", bias, nullptr, D * 4, 0});
    p->held.push_back({"h", h0, hT, bdn * 4, 0});
    p->held.push_back({"v", v0, vT, bdn * 4, 0});
    // chunks of whole 16-byte pieces keep every chunk on the vectorised path
    return lay_out(p, d->seqlen, chunk_steps, 32);
}

struct ScanChunk final : ChunkCall {
    const mm_scan_dims* d;
    const Plan* p;
    bool with_z, with_D, with_bias, has_h0, has_v0;
    int softplus;
    float beta, alpha;
    mm_status operator()(int64_t, int64_t n, char* const* blk, char* fixed, bool first,
                         cudaStream_t s) const override {
        mm_scan_dims cd = *d;
        cd.seqlen = n;
        int j = 0;
        const void* x = blk[j++];
        const void* delta = blk[j++];
        const void* z = with_z ? blk[j++] : nullptr;
        const void* B = blk[j++];
        const void* C = blk[j++];
        void* y = blk[j++];
        // held: A, D, delta_bias, h, v
        const float* A = reinterpret_cast<const float*>(fixed + p->held[0].off);
        const float* Dk = with_D ? reinterpret_cast<const float*>(fixed + p->held[1].off) : nullptr;
        const float* bias = with_bias ? reinterpret_cast<const float*>(fixed + p->held[2].off) : nullptr;
        float* hs = reinterpret_cast<float*>(fixed + p->held[3].off);
        float* vs = reinterpret_cast<float*>(fixed + p->held[4].off);
        const float* h0 = (!first || has_h0) ? hs : nullptr;
        const float* v0 = (!first || has_v0) ? vs : nullptr;
        return mm_scan_fwd_gated(x, delta, A, B, C, Dk, z, bias, softplus, h0, v0, beta, alpha, y, hs, vs, nullptr,
                                 &cd, s);
    }
};

mm_status ssd_plan(Plan* p, const mm_ssd_dims* d, bool momentum, int64_t chunk_steps, const void* x,
                   const float* delta, const float* A, const void* B, const void* C, const float* h0,
                   const float* v0, void* y, float* hT, float* vT) {
    if (!d) return mmscan::report(MM_ERR_NULL, "dims is NULL");
    const int64_t bsz = d->batch, H = d->nheads, P = d->headdim, N = d->dstate, G = d->ngroups;
    if (bsz < 1 || d->seqlen < 1 || H < 1 || P < 1 || N < 1 || G < 1 || d->chunk < 1 || H % G != 0)
        return mmscan::report(MM_ERR_DIMS, "sizes must be >= 1 and ngroups must divide nheads");
    int64_t hp, xs, gn, bs, bh, pn, st;
    if (!mul(H, P, &hp) || !mul(hp, 2, &xs) || !mul(G, N, &gn) || !mul(gn, 2, &bs) || !mul(bsz, H, &bh) ||
        !mul(P, N, &pn) || !mul(bh, pn, &st) || !mul(st, 4, &st) || H > INT64_MAX / 4)
        return mmscan::report(MM_ERR_DIMS, "sizes overflow 64-bit byte counts");
    if (d->seqlen > (int64_t(1) << 30) || bh > 0x7fffffffLL)
        return mmscan::report(MM_ERR_UNSUPPORTED, "SSD seqlen must be <= 2^30 and batch * nheads < 2^31");
    p->st.push_back({"x", const_cast<char*>(static_cast<const char*>(x)), bsz, xs, false, 0});
    p->st.push_back({"delta", reinterpret_cast<char*>(const_cast<float*>(delta)), bsz, H * 4, false, 0});
    p->st.push_back({"B", const_cast<char*>(static_cast<const char*>(B)), bsz, bs, false, 0});
    p->st.push_back({"C", const_cast<char*>(static_cast<const char*>(C)), bsz, bs, false, 0});
    p->st.push_back({"y", static_cast<char*>(y), bsz, xs, true, 0});
    p->held.push_back({"A", A, nullptr, H * 4, 0});
    p->held.push_back({"h", h0, hT, st, 0});
    if (momentum) p->held.push_back({"v", v0, vT, st, 0});
    return lay_out(p, d->seqlen, chunk_steps, d->chunk);
}

struct SSDChunk final : ChunkCall {
    const mm_ssd_dims* d;
    const Plan* p;
    bool momentum, has_h0, has_v0;
    float beta, alpha;
    mm_status operator()(int64_t, int64_t n, char* const* blk, char* fixed, bool first,
                         cudaStream_t s) const override {
        mm_ssd_dims cd = *d;
        cd.seqlen = n;
        const float* A = reinterpret_cast<const float*>(fixed + p->held[0].off);
        float* hs = reinterpret_cast<float*>(fixed + p->held[1].off);
        const float* h0 = (!first || has_h0) ? hs : nullptr;
        const float* delta = reinterpret_cast<const float*>(blk[1]);
        if (!momentum) return mm_ssd_fwd(blk[0], delta, A, blk[2], blk[3], h0, 0.0f, alpha, blk[4], hs, &cd, s);
        float* vs = reinterpret_cast<float*>(fixed + p->held[2].off);
        const float* v0 = (!first || has_v0) ? vs : nullptr;
        return mm_ssd_fwd_momentum(blk[0], delta, A, blk[2], blk[3], h0, v0, beta, alpha, blk[4], hs, vs, &cd, s);
    }
};

}  // namespace

extern "C" {

mm_status mm_scan_fwd_host_workspace_size(const mm_scan_dims* dims, int with_z, int64_t chunk_steps,
                                          size_t* bytes) {
    if (!bytes) return mmscan::report(MM_ERR_NULL, "bytes is NULL");
    Plan p;
    if (mm_status st = scan_plan(&p, dims, with_z != 0, chunk_steps, nullptr, nullptr, nullptr, nullptr, nullptr,
                                 nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr))
        return st;
    *bytes = size_t(p.total);
    return mmscan::report_ok();
}

mm_status mm_scan_fwd_host(const void* x, const void* delta, const float* A, const void* B, const void* C,
                           const float* Dskip, const void* z, const float* delta_bias, int delta_softplus,
                           const float* h0, const float* v0, float beta, float alpha, void* y, float* hT,
                           float* vT, void* workspace, size_t workspace_bytes, int64_t chunk_steps,
                           const mm_scan_dims* dims, void* stream) {
    if (!x || !delta || !A || !B || !C || !y)
        return mmscan::report(MM_ERR_NULL, "x, delta, A, B, C and y are required");
    if (!std::isfinite(beta) || beta < 0.0f || beta >= 1.0f)
        return mmscan::report(MM_ERR_SCALAR, "beta=%g is outside [0, 1)", (double)beta);
    if (!std::isfinite(alpha) || alpha < 0.0f)
        return mmscan::report(MM_ERR_SCALAR, "alpha=%g must be finite and >= 0", (double)alpha);
    Plan p;
    if (mm_status st = scan_plan(&p, dims, z != nullptr, chunk_steps, x, delta, A, B, C, Dskip, z, delta_bias, h0,
                                 v0, y, hT, vT))
        return st;
    if (mm_status st = check_buffers(p, workspace, workspace_bytes)) return st;
    if (mm_status st = check_host_aliasing(p)) return st;
    ScanChunk call;
    call.d = dims;
    call.p = &p;
    call.with_z = z != nullptr;
    call.with_D = Dskip != nullptr;
    call.with_bias = delta_bias != nullptr;
    call.has_h0 = h0 != nullptr;
    call.has_v0 = v0 != nullptr;
    call.softplus = delta_softplus ? 1 : 0;
    call.beta = beta;
    call.alpha = alpha;
    return run(p, static_cast<char*>(workspace), static_cast<cudaStream_t>(stream), call);
}

mm_status mm_ssd_fwd_host_workspace_size(const mm_ssd_dims* dims, int momentum, int64_t chunk_steps,
                                         size_t* bytes) {
    if (!bytes) return mmscan::report(MM_ERR_NULL, "bytes is NULL");
    Plan p;
    if (mm_status st = ssd_plan(&p, dims, momentum != 0, chunk_steps, nullptr, nullptr, nullptr, nullptr, nullptr,
                                nullptr, nullptr, nullptr, nullptr, nullptr))
        return st;
    *bytes = size_t(p.total);
    return mmscan::report_ok();
}

mm_status mm_ssd_fwd_host(const void* x, const float* delta, const float* A, const void* B, const void* C,
                          const float* h0, const float* v0, float beta, float alpha, void* y, float* hT, float* vT,
                          void* workspace, size_t workspace_bytes, int64_t chunk_steps, const mm_ssd_dims* dims,
                          void* stream) {
    if (!x || !delta || !A || !B || !C || !y)
        return mmscan::report(MM_ERR_NULL, "x, delta, A, B, C and y are required");
    if (!std::isfinite(beta) || beta < 0.0f || beta >= 1.0f)
        return mmscan::report(MM_ERR_SCALAR, "beta=%g is outside [0, 1)", (double)beta);
    if (!std::isfinite(alpha) || alpha < 0.0f)
        return mmscan::report(MM_ERR_SCALAR, "alpha=%g must be finite and >= 0", (double)alpha);
    // the velocity is carried when beta > 0 or when the caller passes one
    const bool momentum = beta != 0.0f || v0 != nullptr || vT != nullptr;
    Plan p;
    if (mm_status st = ssd_plan(&p, dims, momentum, chunk_steps, x, delta, A, B, C, h0, v0, y, hT, vT)) return st;
    if (!momentum && !mmscan::ssd_shape_supported(dims->headdim, dims->dstate, dims->chunk))
        return mmscan::report(MM_ERR_UNSUPPORTED, "SSD with headdim=%lld dstate=%lld chunk=%lld is not built",
                              (long long)dims->headdim, (long long)dims->dstate, (long long)dims->chunk);
    if (momentum && !mmscan::ssd_mom_shape_supported(dims->headdim, dims->dstate))
        return mmscan::report(MM_ERR_UNSUPPORTED, "momentum SSD needs headdim <= 64 and dstate <= 128");
    if (mm_status st = check_buffers(p, workspace, workspace_bytes)) return st;
    if (mm_status st = check_host_aliasing(p)) return st;
    SSDChunk call;
    call.d = dims;
    call.p = &p;
    call.momentum = momentum;
    call.has_h0 = h0 != nullptr;
    call.has_v0 = v0 != nullptr;
    call.beta = beta;
    call.alpha = alpha;
    return run(p, static_cast<char*>(workspace), static_cast<cudaStream_t>(stream), call);
}

}  // extern "C"
