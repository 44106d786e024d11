// host_pipeline_sanitized.cpp -- the host-buffer pipeline (mm_host.cpp) on a
// machine without CUDA, under AddressSanitizer and UndefinedBehaviorSanitizer.
//
// mm_host.cpp and mm_api.cpp are compiled against a stand-in CUDA runtime
// whose streams are queues of deferred operations.  A scheduler runs them in
// adversarial orders: every case is run under many seeds, each giving the
// streams random priorities, and only what CUDA guarantees is enforced
// (stream order, and a wait blocks until the record it saw when it was queued
// has run).  The kernel launchers are replaced by a plain CPU stand-in for
// the scan and the SSD recurrence (sequential per lane, so any time split
// gives the same bits), queued on the launch stream like a kernel.
//
// For every case the host entry point must reproduce, byte for byte, one
// device call over the whole problem; every copy and kernel operand must lie
// inside one registered buffer of the right kind (host or device).  The
// workspace is poisoned with NaN bytes before each run, the host inputs are
// written by an operation queued on the caller's stream just before the call
// (so the call must wait for it), and the outputs are read by an operation
// queued on that stream just after (so the call must be joined into it).
//
// Mutation check: for each wait the pipeline queues, dropping that one wait
// must make some seed fail -- no wait is redundant, and the harness can see
// the race each one prevents.  Exit status 0 and "host pipeline ok" when all
// hold.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <deque>
#include <functional>
#include <memory>
#include <random>
#include <string>
#include <vector>

#include "cuda_runtime.h"
#include "mm_internal.h"
#include "mm_scan.h"

// ---- registered buffers -------------------------------------------------------
namespace {

struct Region {
    uintptr_t lo, hi;
    bool device;
};
std::vector<Region> g_regions;
int g_bad = 0;
std::string g_first_bad;

void bad(const std::string& what) {
    if (g_bad++ == 0) g_first_bad = what;
}

const Region* find(const void* p, size_t n) {
    const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
    for (const Region& r : g_regions)
        if (lo >= r.lo && lo + n <= r.hi && lo + n >= lo) return &r;
    return nullptr;
}

void need(const void* p, size_t n, bool device, const char* what) {
    const Region* r = find(p, n);
    if (!r || r->device != device) bad(std::string(what) + ": range outside every " + (device ? "device" : "host") +
                                       " buffer");
}

struct Buf {
    std::unique_ptr<char, void (*)(void*)> mem{nullptr, std::free};
    size_t bytes = 0;
    Buf() = default;
    Buf(size_t n, bool device) : mem(static_cast<char*>(std::aligned_alloc(256, (n + 255) / 256 * 256 + 256)), std::free),
                                 bytes(n) {
        std::memset(mem.get(), 0, (n + 255) / 256 * 256 + 256);
        g_regions.push_back({reinterpret_cast<uintptr_t>(mem.get()), reinterpret_cast<uintptr_t>(mem.get()) + n, device});
    }
    char* p() const { return mem.get(); }
    ~Buf() {
        const uintptr_t lo = reinterpret_cast<uintptr_t>(mem.get());
        for (size_t i = 0; i < g_regions.size(); ++i)
            if (g_regions[i].lo == lo) {
                g_regions.erase(g_regions.begin() + long(i));
                break;
            }
    }
    Buf(const Buf&) = delete;
    Buf& operator=(const Buf&) = delete;
    template <class T> T* as() const { return reinterpret_cast<T*>(mem.get()); }
};

}  // namespace

// ---- the stand-in runtime -------------------------------------------------------
struct stub_event {
    uint64_t enq = 0, done = 0;
};

struct Op {
    enum Kind { RUN, RECORD, WAIT } kind;
    std::function<void()> fn;
    stub_event* ev = nullptr;
    uint64_t seq = 0;
};

struct stub_stream {
    std::deque<Op> q;
    int prio = 0;
};

namespace {
std::vector<std::unique_ptr<stub_stream>> g_streams;
std::vector<std::unique_ptr<stub_event>> g_events;
stub_stream g_default;
std::mt19937_64 g_rng(1);
long g_wait_calls = 0, g_drop_wait = -1;

stub_stream* S(cudaStream_t s) { return s ? s : &g_default; }

bool ready(const stub_stream& s) {
    if (s.q.empty()) return false;
    const Op& op = s.q.front();
    return op.kind != Op::WAIT || op.ev->done >= op.seq;
}

// Run one operation of some stream; false when nothing can run.
bool step() {
    std::vector<stub_stream*> r;
    if (ready(g_default)) r.push_back(&g_default);
    for (auto& s : g_streams)
        if (ready(*s)) r.push_back(s.get());
    if (r.empty()) return false;
    stub_stream* pick = r[0];
    if (g_rng() % 4 == 0) {
        pick = r[g_rng() % r.size()];
    } else {
        for (stub_stream* s : r)
            if (s->prio > pick->prio) pick = s;
    }
    Op op = std::move(pick->q.front());
    pick->q.pop_front();
    if (op.kind == Op::RUN) op.fn();
    if (op.kind == Op::RECORD) op.ev->done = std::max(op.ev->done, op.seq);
    return true;
}

bool pending() {
    if (!g_default.q.empty()) return true;
    for (auto& s : g_streams)
        if (!s->q.empty()) return true;
    return false;
}

void drain() {
    while (step()) {
    }
    if (pending()) bad("deadlock: queued operations that can never run");
}

void enqueue(cudaStream_t s, std::function<void()> fn) { S(s)->q.push_back(Op{Op::RUN, std::move(fn)}); }

}  // namespace

cudaError_t cudaStreamCreateWithFlags(cudaStream_t* s, unsigned) {
    g_streams.push_back(std::make_unique<stub_stream>());
    g_streams.back()->prio = int(g_rng() % 1000);
    *s = g_streams.back().get();
    return cudaSuccess;
}
cudaError_t cudaStreamDestroy(cudaStream_t) { return cudaSuccess; }   // freed when the case ends
cudaError_t cudaStreamSynchronize(cudaStream_t) {
    drain();
    return cudaSuccess;
}
cudaError_t cudaEventCreateWithFlags(cudaEvent_t* e, unsigned) {
    g_events.push_back(std::make_unique<stub_event>());
    *e = g_events.back().get();
    return cudaSuccess;
}
cudaError_t cudaEventDestroy(cudaEvent_t) { return cudaSuccess; }
cudaError_t cudaEventRecord(cudaEvent_t e, cudaStream_t s) {
    ++e->enq;
    S(s)->q.push_back(Op{Op::RECORD, nullptr, e, e->enq});
    return cudaSuccess;
}
cudaError_t cudaStreamWaitEvent(cudaStream_t s, cudaEvent_t e, unsigned) {
    if (g_wait_calls++ == g_drop_wait) return cudaSuccess;        // the planted mistake
    if (e->enq) S(s)->q.push_back(Op{Op::WAIT, nullptr, e, e->enq});
    return cudaSuccess;
}
cudaError_t cudaMemcpy2DAsync(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width,
                              size_t height, cudaMemcpyKind k, cudaStream_t s) {
    if (width > dpitch || width > spitch) return cudaErrorInvalidValue;
    const bool h2d = k == cudaMemcpyHostToDevice;
    for (size_t r = 0; r < height; ++r) {
        need(static_cast<const char*>(src) + r * spitch, width, !h2d, "copy source");
        need(static_cast<char*>(dst) + r * dpitch, width, h2d, "copy destination");
    }
    enqueue(s, [=] {
        for (size_t r = 0; r < height; ++r)
            std::memcpy(static_cast<char*>(dst) + r * dpitch, static_cast<const char*>(src) + r * spitch, width);
    });
    return cudaSuccess;
}
cudaError_t cudaMemcpyAsync(void* dst, const void* src, size_t n, cudaMemcpyKind k, cudaStream_t s) {
    return cudaMemcpy2DAsync(dst, n, src, n, n, 1, k, s);
}
cudaError_t cudaPointerGetAttributes(cudaPointerAttributes* a, const void* p) {
    std::memset(a, 0, sizeof(*a));
    const Region* r = find(p, 1);
    a->type = !r ? cudaMemoryTypeUnregistered : r->device ? cudaMemoryTypeDevice : cudaMemoryTypeHost;
    return cudaSuccess;
}
cudaError_t cudaDeviceSynchronize(void) {
    drain();
    return cudaSuccess;
}
cudaError_t cudaGetDevice(int* device) {
    *device = 0;
    return cudaSuccess;
}
const char* cudaGetErrorString(cudaError_t) { return "stub"; }
const char* cudaGetErrorName(cudaError_t) { return "stub"; }

// ---- CPU stand-ins for the kernels --------------------------------------------
namespace {

float bf16_to_f(uint16_t b) {
    uint32_t u = uint32_t(b) << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

uint16_t f_to_bf16(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return uint16_t((u >> 16) | 0x40);
    return uint16_t((u + 0x7fffu + ((u >> 16) & 1u)) >> 16);
}

float ld(const void* p, int64_t i, int io) {
    return io == 0 ? static_cast<const float*>(p)[i] : bf16_to_f(static_cast<const uint16_t*>(p)[i]);
}

void st(void* p, int64_t i, int io, float v) {
    if (io == 0) static_cast<float*>(p)[i] = v;
    else static_cast<uint16_t*>(p)[i] = f_to_bf16(v);
}

void scan_cpu(const mmscan::ScanArgs& a, int io) {
    const int64_t Bz = a.batch, L = a.seqlen, D = a.dim, N = a.dstate, es = io == 0 ? 4 : 2;
    need(a.x, size_t(Bz * D * L * es), true, "kernel x");
    need(a.delta, size_t(Bz * D * L * es), true, "kernel delta");
    need(a.B, size_t(Bz * N * L * es), true, "kernel B");
    need(a.C, size_t(Bz * N * L * es), true, "kernel C");
    need(a.y, size_t(Bz * D * L * es), true, "kernel y");
    need(a.A, size_t(D * N * 4), true, "kernel A");
    if (a.z) need(a.z, size_t(Bz * D * L * es), true, "kernel z");
    if (a.Dskip) need(a.Dskip, size_t(D * 4), true, "kernel D");
    if (a.dbias) need(a.dbias, size_t(D * 4), true, "kernel delta_bias");
    for (const float* s : {a.h0, a.v0, static_cast<const float*>(a.hT), static_cast<const float*>(a.vT)})
        if (s) need(s, size_t(Bz * D * N * 4), true, "kernel state");
    std::vector<float> h(N), v(N);
    for (int64_t b = 0; b < Bz; ++b)
        for (int64_t d = 0; d < D; ++d) {
            const int64_t row = (b * D + d) * L, srow = (b * D + d) * N;
            for (int64_t n = 0; n < N; ++n) {
                h[n] = a.h0 ? a.h0[srow + n] : 0.0f;
                v[n] = a.v0 ? a.v0[srow + n] : 0.0f;
            }
            for (int64_t t = 0; t < L; ++t) {
                float dt = ld(a.delta, row + t, io);
                if (a.dbias) dt += a.dbias[d];
                if (a.softplus) dt = std::log1p(std::exp(dt));
                const float u = ld(a.x, row + t, io);
                float acc = 0.0f;
                for (int64_t n = 0; n < N; ++n) {
                    const float Bt = ld(a.B, (b * N + n) * L + t, io), Ct = ld(a.C, (b * N + n) * L + t, io);
                    v[n] = a.beta * v[n] + a.alpha * dt * Bt * u;
                    h[n] = std::exp(dt * a.A[d * N + n]) * h[n] + v[n];
                    acc += Ct * h[n];
                }
                if (a.Dskip) acc += a.Dskip[d] * u;
                if (a.z) {
                    const float zz = ld(a.z, row + t, io);
                    acc *= zz / (1.0f + std::exp(-zz));
                }
                st(a.y, row + t, io, acc);
            }
            for (int64_t n = 0; n < N; ++n) {
                if (a.hT) a.hT[srow + n] = h[n];
                if (a.vT) a.vT[srow + n] = v[n];
            }
        }
}

// SSD: x, y (batch, L, H, P) bf16; delta (batch, L, H); B, C (batch, L, G, N) bf16.
void ssd_cpu(const void* x, const float* delta, const float* A, const void* B, const void* C, const float* h0,
             const float* v0, void* y, float* hT, float* vT, int64_t Bz, int64_t L, int64_t H, int64_t P, int64_t N,
             int64_t G, float beta, float alpha, bool momentum) {
    need(x, size_t(Bz * L * H * P * 2), true, "ssd x");
    need(y, size_t(Bz * L * H * P * 2), true, "ssd y");
    need(delta, size_t(Bz * L * H * 4), true, "ssd delta");
    need(B, size_t(Bz * L * G * N * 2), true, "ssd B");
    need(C, size_t(Bz * L * G * N * 2), true, "ssd C");
    need(A, size_t(H * 4), true, "ssd A");
    for (const float* s : {h0, v0, static_cast<const float*>(hT), static_cast<const float*>(vT)})
        if (s) need(s, size_t(Bz * H * P * N * 4), true, "ssd state");
    std::vector<float> h(N), v(N);
    for (int64_t b = 0; b < Bz; ++b)
        for (int64_t hh = 0; hh < H; ++hh)
            for (int64_t p = 0; p < P; ++p) {
                const int64_t g = hh / (H / G), srow = ((b * H + hh) * P + p) * N;
                for (int64_t n = 0; n < N; ++n) {
                    h[n] = h0 ? h0[srow + n] : 0.0f;
                    v[n] = (momentum && v0) ? v0[srow + n] : 0.0f;
                }
                for (int64_t t = 0; t < L; ++t) {
                    const float dt = delta[(b * L + t) * H + hh];
                    const float u = ld(x, ((b * L + t) * H + hh) * P + p, 1);
                    const float a = std::exp(dt * A[hh]);
                    float acc = 0.0f;
                    for (int64_t n = 0; n < N; ++n) {
                        const int64_t bc = ((b * L + t) * G + g) * N + n;
                        const float w = alpha * dt * ld(B, bc, 1) * u;
                        if (momentum) {
                            v[n] = beta * v[n] + w;
                            h[n] = a * h[n] + v[n];
                        } else {
                            h[n] = a * h[n] + w;
                        }
                        acc += ld(C, bc, 1) * h[n];
                    }
                    st(y, ((b * L + t) * H + hh) * P + p, 1, acc);
                }
                for (int64_t n = 0; n < N; ++n) {
                    if (hT) hT[srow + n] = h[n];
                    if (vT && momentum) vT[srow + n] = v[n];
                }
            }
}

int g_launches = 0;

}  // namespace

namespace mmscan {
bool scan_tile_supported(int spt, int warps, int time_lanes) {
    return (spt == 2 || spt == 4) && warps >= 1 && warps <= 8 && (time_lanes == 1 || time_lanes == 2);
}
ScanTileChoice choose_scan_tile(int64_t, int64_t, int64_t dstate, int, int, int, int) {
    return ScanTileChoice{dstate <= 2 ? 2 : dstate <= 4 ? 4 : dstate <= 8 ? 8 : 16, 2, 4, 1};
}
cudaError_t launch_scan_fwd(const ScanArgs& a, const ScanTileChoice&, int io, cudaStream_t s) {
    ++g_launches;
    enqueue(s, [a, io] { scan_cpu(a, io); });
    return cudaSuccess;
}
cudaError_t launch_scan_seg(const ScanArgs& a, int io, int64_t, bool, cudaStream_t s) {
    ++g_launches;
    enqueue(s, [a, io] { scan_cpu(a, io); });
    return cudaSuccess;
}
int64_t scan_seg_default_len(int64_t, int64_t) { return 64; }
cudaError_t launch_scan_bwd(const ScanBwdArgs&, int, cudaStream_t) { return cudaErrorInvalidValue; }
int64_t scan_bwd_det_workspace_bytes(int64_t, int64_t, int, int64_t) { return 1024; }
bool stream_capturing(cudaStream_t) { return false; }
cudaError_t launch_scan_step(const ScanStepArgs&, int, cudaStream_t) { return cudaErrorInvalidValue; }
cudaError_t launch_ssd_fwd(const SSDArgs& a, cudaStream_t s) {
    ++g_launches;
    enqueue(s, [a] {
        ssd_cpu(a.x, a.delta, a.A, a.B, a.C, a.h0, nullptr, a.y, a.hT, nullptr, a.batch, a.seqlen, a.nheads,
                a.headdim, a.dstate, a.ngroups, 0.0f, a.alpha, false);
    });
    return cudaSuccess;
}
cudaError_t launch_ssd_mom(const SSDMomArgs& a, cudaStream_t s) {
    ++g_launches;
    enqueue(s, [a] {
        ssd_cpu(a.x, a.delta, a.A, a.B, a.C, a.h0, a.v0, a.y, a.hT, a.vT, a.batch, a.seqlen, a.nheads, a.headdim,
                a.dstate, a.ngroups, a.beta, a.alpha, true);
    });
    return cudaSuccess;
}
int64_t scan_seg_chunk_steps(int io) { return io == 0 ? 32 : 64; }
int64_t scan_seg_tile_channels() { return 16; }
int64_t scan_seg_tile_record_bytes() { return 257 * 16; }
cudaError_t launch_scan_seg_split(const ScanArgs&, int, int64_t, int, void*, int64_t, int64_t, void* const*, int,
                                  cudaStream_t) {
    return cudaErrorInvalidValue;
}
unsigned int scan_seg_read_and_clear_device_error() { return 0; }
unsigned int scan_read_and_clear_device_error() { return 0; }
unsigned int scan_bwd_read_and_clear_device_error() { return 0; }
unsigned int ssd_read_and_clear_device_error() { return 0; }
bool ssd_shape_supported(int64_t headdim, int64_t dstate, int64_t chunk) {
    return headdim >= 1 && dstate >= 1 && chunk >= 1;
}
bool ssd_mom_shape_supported(int64_t headdim, int64_t dstate) { return headdim >= 1 && dstate >= 1; }
bool ssd_mom_tc_shape_supported(int64_t, int64_t) { return false; }
cudaError_t launch_ssd_mom_tc(const SSDMomArgs& a, cudaStream_t s) { return launch_ssd_mom(a, s); }
unsigned int ssd_mom_tc_read_and_clear_device_error() { return 0; }
}  // namespace mmscan

// ---- the driver ---------------------------------------------------------------
namespace {

void fill(Buf& b, int io_or_f32, uint64_t seed, float lo, float hi) {
    std::mt19937_64 r(seed);
    std::uniform_real_distribution<float> u(lo, hi);
    if (io_or_f32 == 0) {
        float* f = b.as<float>();
        for (size_t i = 0; i < b.bytes / 4; ++i) f[i] = u(r);
    } else {
        uint16_t* h = b.as<uint16_t>();
        for (size_t i = 0; i < b.bytes / 2; ++i) h[i] = f_to_bf16(u(r));
    }
}

// A tensor of a case: its source values, the host buffer the call reads or
// writes, and a device copy for the one-call reference.
struct T {
    Buf src, host, dev, seen;
    bool out = false;
    T(size_t n, bool is_out) : src(n, false), host(n, false), dev(n, true), seen(n, false), out(is_out) {}
};

struct ScanCase {
    const char* name;
    int64_t batch, L, dim, N;
    int io;
    bool z, Dk, bias, softplus, h0, v0, hT, vT, in_place;
    float beta, alpha;
    int64_t chunk_steps;
};

struct SSDCase {
    const char* name;
    int64_t batch, L, H, P, N, G, chunk;
    bool momentum, h0, v0, hT, vT;
    float beta, alpha;
    int64_t chunk_steps;
};

void reset_runtime(uint64_t seed) {
    mmscan::host_pipeline_release();   // the next call creates its streams under this seed
    g_rng.seed(seed);
    g_default.q.clear();
    g_default.prio = int(g_rng() % 1000);
    g_streams.clear();
    g_events.clear();
}

// Queue the inputs' producer on the caller's stream, call, then queue the
// outputs' consumer; drain and compare with the one-call result.  Returns
// false on a mismatch or a checker complaint.
template <class Call>
bool run_once(std::vector<T*>& ts, Buf& ws, uint64_t seed, long drop, Call call, const char* name,
              bool report) {
    reset_runtime(seed);
    g_wait_calls = 0;
    g_drop_wait = drop;
    const int bad0 = g_bad;
    std::memset(ws.p(), 0xff, ws.bytes);
    for (T* t : ts) {
        std::memset(t->host.p(), 0xff, t->host.bytes);
        std::memset(t->seen.p(), 0x5a, t->seen.bytes);
        if (!t->out) enqueue(nullptr, [t] { std::memcpy(t->host.p(), t->src.p(), t->src.bytes); });
        else if (t->src.bytes) enqueue(nullptr, [t] { std::memcpy(t->host.p(), t->src.p(), t->src.bytes); });
    }
    const mm_status st = call();
    for (T* t : ts)
        if (t->out) enqueue(nullptr, [t] { std::memcpy(t->seen.p(), t->host.p(), t->host.bytes); });
    drain();
    g_drop_wait = -1;
    if (st != MM_OK) {
        if (report) std::printf("%s: status %d (%s)\n", name, (int)st, mm_last_error());
        return false;
    }
    bool same = g_bad == bad0;
    for (T* t : ts)
        if (t->out && std::memcmp(t->seen.p(), t->dev.p(), t->dev.bytes) != 0) {
            same = false;
            if (report) std::printf("%s (seed %llu): output differs from one device call\n", name,
                                    (unsigned long long)seed);
            break;
        }
    if (!same && report && g_bad > bad0) std::printf("%s: %s\n", name, g_first_bad.c_str());
    g_bad = bad0;   // counted by the caller
    return same;
}

// Run a case under many schedules, then drop each of its waits in turn.
template <class Ref, class Call>
void check_case(std::vector<T*>& ts, Buf& ws, Ref ref, Call call, const char* name, int seeds, bool mutate) {
    // the one-call reference, on device copies
    reset_runtime(7);
    for (T* t : ts) std::memcpy(t->dev.p(), t->src.p(), t->src.bytes);
    if (ref() != MM_OK) {
        std::printf("%s: reference call failed: %s\n", name, mm_last_error());
        ++g_bad;
        return;
    }
    drain();
    for (int s = 0; s < seeds; ++s)
        if (!run_once(ts, ws, 1000 + s, -1, call, name, true)) {
            ++g_bad;
            return;
        }
    if (!mutate) return;
    run_once(ts, ws, 1, -1, call, name, false);
    const long waits = g_wait_calls;
    for (long k = 0; k < waits; ++k) {
        bool caught = false;
        for (int s = 0; s < 400 && !caught; ++s) caught = !run_once(ts, ws, 5000 + s, k, call, name, false);
        if (!caught) {
            std::printf("%s: dropping wait %ld of %ld went unnoticed\n", name, k, waits);
            ++g_bad;
        }
    }
}

void scan_case(const ScanCase& c, int seeds, bool mutate) {
    const int64_t es = c.io == 0 ? 4 : 2, seq = c.batch * c.dim * c.L * es, bc = c.batch * c.N * c.L * es,
                  stb = c.batch * c.dim * c.N * 4;
    T x(seq, false), dl(seq, false), A(c.dim * c.N * 4, false), B(bc, false), C(bc, false), y(seq, true);
    T z(c.z ? seq : 0, false), Dk(c.Dk ? c.dim * 4 : 0, false), bias(c.bias ? c.dim * 4 : 0, false);
    T h0(c.h0 ? stb : 0, false), v0(c.v0 ? stb : 0, false);
    T hT(c.hT && !c.in_place ? stb : 0, true), vT(c.vT && !c.in_place ? stb : 0, true);
    fill(x.src, c.io, 1, -1, 1);
    fill(dl.src, c.io, 2, 0.001f, 0.1f);
    fill(A.src, 0, 3, -2, -0.1f);
    fill(B.src, c.io, 4, -1, 1);
    fill(C.src, c.io, 5, -1, 1);
    if (c.z) fill(z.src, c.io, 6, -2, 2);
    if (c.Dk) fill(Dk.src, 0, 7, -1, 1);
    if (c.bias) fill(bias.src, 0, 8, -0.5f, 0.1f);
    if (c.h0) fill(h0.src, 0, 9, -1, 1);
    if (c.v0) fill(v0.src, 0, 10, -0.3f, 0.3f);
    if (c.in_place) {   // hT is h0 and vT is v0: the states are inputs and outputs at once
        h0.out = c.hT;
        v0.out = c.vT;
    }
    std::vector<T*> ts = {&x, &dl, &A, &B, &C, &y};
    for (T* t : {&z, &Dk, &bias, &h0, &v0, &hT, &vT})
        if (t->src.bytes) ts.push_back(t);
    mm_scan_dims d{c.batch, c.L, c.dim, c.N, c.io};
    size_t need_ws = 0;
    if (mm_scan_fwd_host_workspace_size(&d, c.z, c.chunk_steps, &need_ws) != MM_OK) {
        std::printf("%s: workspace size: %s\n", c.name, mm_last_error());
        ++g_bad;
        return;
    }
    Buf ws(need_ws, true);
    auto P = [](T& t, bool dev) -> void* { return t.src.bytes ? (dev ? t.dev.p() : t.host.p()) : nullptr; };
    auto args = [&](bool dev) {
        float* hout = c.in_place ? (c.hT ? static_cast<float*>(P(h0, dev)) : nullptr) : static_cast<float*>(P(hT, dev));
        float* vout = c.in_place ? (c.vT ? static_cast<float*>(P(v0, dev)) : nullptr) : static_cast<float*>(P(vT, dev));
        return std::make_pair(hout, vout);
    };
    auto ref = [&] {
        auto [ho, vo] = args(true);
        return mm_scan_fwd_gated(P(x, true), P(dl, true), static_cast<float*>(P(A, true)), P(B, true), P(C, true),
                                 static_cast<float*>(P(Dk, true)), P(z, true), static_cast<float*>(P(bias, true)),
                                 c.softplus, static_cast<float*>(P(h0, true)), static_cast<float*>(P(v0, true)),
                                 c.beta, c.alpha, P(y, true), ho, vo, nullptr, &d, nullptr);
    };
    auto call = [&] {
        auto [ho, vo] = args(false);
        return mm_scan_fwd_host(P(x, false), P(dl, false), static_cast<float*>(P(A, false)), P(B, false),
                                P(C, false), static_cast<float*>(P(Dk, false)), P(z, false),
                                static_cast<float*>(P(bias, false)), c.softplus, static_cast<float*>(P(h0, false)),
                                static_cast<float*>(P(v0, false)), c.beta, c.alpha, P(y, false), ho, vo, ws.p(),
                                ws.bytes, c.chunk_steps, &d, nullptr);
    };
    check_case(ts, ws, ref, call, c.name, seeds, mutate);
}

void ssd_case(const SSDCase& c, int seeds, bool mutate) {
    const int64_t xs = c.batch * c.L * c.H * c.P * 2, bcs = c.batch * c.L * c.G * c.N * 2,
                  stb = c.batch * c.H * c.P * c.N * 4;
    T x(xs, false), dl(c.batch * c.L * c.H * 4, false), A(c.H * 4, false), B(bcs, false), C(bcs, false),
        y(xs, true);
    T h0(c.h0 ? stb : 0, false), v0(c.v0 ? stb : 0, false), hT(c.hT ? stb : 0, true), vT(c.vT ? stb : 0, true);
    fill(x.src, 1, 11, -1, 1);
    fill(dl.src, 0, 12, 0.001f, 0.1f);
    fill(A.src, 0, 13, -2, -0.1f);
    fill(B.src, 1, 14, -1, 1);
    fill(C.src, 1, 15, -1, 1);
    if (c.h0) fill(h0.src, 0, 16, -1, 1);
    if (c.v0) fill(v0.src, 0, 17, -0.3f, 0.3f);
    std::vector<T*> ts = {&x, &dl, &A, &B, &C, &y};
    for (T* t : {&h0, &v0, &hT, &vT})
        if (t->src.bytes) ts.push_back(t);
    mm_ssd_dims d{c.batch, c.L, c.H, c.P, c.N, c.G, c.chunk};
    size_t need_ws = 0;
    if (mm_ssd_fwd_host_workspace_size(&d, c.momentum, c.chunk_steps, &need_ws) != MM_OK) {
        std::printf("%s: workspace size: %s\n", c.name, mm_last_error());
        ++g_bad;
        return;
    }
    Buf ws(need_ws, true);
    auto P = [](T& t, bool dev) -> void* { return t.src.bytes ? (dev ? t.dev.p() : t.host.p()) : nullptr; };
    auto F = [&](T& t, bool dev) { return static_cast<float*>(P(t, dev)); };
    auto ref = [&] {
        if (!c.momentum)
            return mm_ssd_fwd(P(x, true), F(dl, true), F(A, true), P(B, true), P(C, true), F(h0, true), 0.0f, c.alpha,
                              P(y, true), F(hT, true), &d, nullptr);
        return mm_ssd_fwd_momentum(P(x, true), F(dl, true), F(A, true), P(B, true), P(C, true), F(h0, true),
                                   F(v0, true), c.beta, c.alpha, P(y, true), F(hT, true), F(vT, true), &d, nullptr);
    };
    auto call = [&] {
        return mm_ssd_fwd_host(P(x, false), F(dl, false), F(A, false), P(B, false), P(C, false), F(h0, false),
                               F(v0, false), c.beta, c.alpha, P(y, false), F(hT, false), F(vT, false), ws.p(),
                               ws.bytes, c.chunk_steps, &d, nullptr);
    };
    check_case(ts, ws, ref, call, c.name, seeds, mutate);
}

void expect(mm_status got, mm_status want, const char* what) {
    if (got != want) {
        std::printf("%s: status %d, expected %d (%s)\n", what, (int)got, (int)want, mm_last_error());
        ++g_bad;
    }
}

// Argument checks that run before anything is queued.
void check_errors() {
    mm_scan_dims d{1, 64, 4, 4, MM_F32};
    Buf x(64 * 4 * 4, false), dl(64 * 4 * 4, false), A(16 * 4, false), B(64 * 4 * 4, false), C(64 * 4 * 4, false),
        y(64 * 4 * 4, false), dx(64 * 4 * 4, true);
    size_t need_ws = 0;
    expect(mm_scan_fwd_host_workspace_size(&d, 0, 0, &need_ws), MM_OK, "workspace query");
    expect(mm_scan_fwd_host_workspace_size(&d, 0, -1, &need_ws), MM_ERR_DIMS, "negative chunk_steps");
    expect(mm_scan_fwd_host_workspace_size(nullptr, 0, 0, &need_ws), MM_ERR_NULL, "NULL dims");
    Buf ws(need_ws, true), hws(need_ws, false);
    const int64_t n0 = int64_t(g_launches);
    auto call = [&](void* xp, void* yp, void* w, size_t wb, float beta) {
        reset_runtime(3);
        const mm_status st = mm_scan_fwd_host(xp, dl.p(), A.as<float>(), B.p(), C.p(), nullptr, nullptr, nullptr, 0,
                                              nullptr, nullptr, beta, 1.0f, yp, nullptr, nullptr, w, wb, 0, &d,
                                              nullptr);
        drain();
        return st;
    };
    expect(call(x.p(), y.p(), ws.p(), ws.bytes, 0.9f), MM_OK, "valid call");
    expect(call(x.p(), y.p(), ws.p(), ws.bytes - 1, 0.9f), MM_ERR_DIMS, "workspace one byte short");
    expect(call(x.p(), y.p(), nullptr, ws.bytes, 0.9f), MM_ERR_NULL, "NULL workspace");
    expect(call(x.p(), y.p(), ws.p() + 4, ws.bytes, 0.9f), MM_ERR_ALIGN, "unaligned workspace");
    expect(call(x.p(), y.p(), hws.p(), hws.bytes, 0.9f), MM_ERR_UNSUPPORTED, "workspace in host memory");
    expect(call(dx.p(), y.p(), ws.p(), ws.bytes, 0.9f), MM_ERR_UNSUPPORTED, "x in device memory");
    expect(call(x.p(), x.p(), ws.p(), ws.bytes, 0.9f), MM_ERR_ALIAS, "y is x");
    expect(call(x.p(), y.p(), ws.p(), ws.bytes, 1.0f), MM_ERR_SCALAR, "beta = 1");
    expect(call(nullptr, y.p(), ws.p(), ws.bytes, 0.9f), MM_ERR_NULL, "x NULL");
    if (int64_t(g_launches) != n0 + 1) {
        std::printf("rejected calls launched kernels\n");
        ++g_bad;
    }
    mm_scan_dims bad_dims{1, 0, 4, 4, MM_F32};
    expect(mm_scan_fwd_host_workspace_size(&bad_dims, 0, 0, &need_ws), MM_ERR_DIMS, "seqlen 0");
    mm_scan_dims huge{int64_t(1) << 40, int64_t(1) << 30, int64_t(1) << 30, 16, MM_F32};
    const mm_status hs = mm_scan_fwd_host_workspace_size(&huge, 1, 0, &need_ws);
    if (hs != MM_ERR_DIMS && hs != MM_ERR_UNSUPPORTED) {
        std::printf("huge sizes: status %d\n", (int)hs);
        ++g_bad;
    }
    mm_ssd_dims sd{1, 64, 2, 3, 4, 1, 16};
    expect(mm_ssd_fwd_host_workspace_size(&sd, 1, 0, &need_ws), MM_OK, "SSD workspace query");
    mm_ssd_dims sbad{1, 64, 3, 3, 4, 2, 16};
    expect(mm_ssd_fwd_host_workspace_size(&sbad, 1, 0, &need_ws), MM_ERR_DIMS, "SSD groups not dividing heads");
}

}  // namespace

int main() {
    const ScanCase scans[] = {
        // name, batch, L, dim, N, io, z, D, bias, softplus, h0, v0, hT, vT, in_place, beta, alpha, chunk_steps
        {"scan f32, 10 chunks", 2, 300, 5, 3, MM_F32, false, false, false, false, true, true, true, true, false,
         0.9f, 1.0f, 32},
        {"scan bf16, ragged chunks", 2, 301, 4, 4, MM_BF16, false, false, false, false, false, false, true, true,
         false, 0.5f, 2.0f, 64},
        {"scan gated, no states out", 1, 250, 6, 2, MM_F32, true, true, true, true, true, false, false, false,
         false, 0.99f, 1.0f, 32},
        {"scan in place, chunk 1", 1, 9, 3, 2, MM_F32, false, false, false, false, true, true, true, true, true,
         0.8f, 1.0f, 1},
        {"scan sequence-split chunks", 1, 640, 2, 16, MM_F32, false, true, false, false, true, true, true, true,
         false, 0.9f, 0.5f, 128},
        {"scan automatic chunk", 3, 100, 7, 5, MM_BF16, true, false, false, false, true, true, true, false, false,
         0.0f, 1.0f, 0},
    };
    const SSDCase ssds[] = {
        // name, batch, L, H, P, N, G, chunk, momentum, h0, v0, hT, vT, beta, alpha, chunk_steps
        {"ssd plain, 7 chunks", 2, 200, 4, 3, 5, 2, 16, false, true, false, true, false, 0.0f, 1.0f, 32},
        {"ssd momentum, ragged", 1, 150, 2, 2, 3, 1, 16, true, true, true, true, true, 0.9f, 0.5f, 48},
        {"ssd momentum from zero", 2, 96, 2, 4, 2, 2, 16, true, false, false, true, true, 0.5f, 1.0f, 16},
        {"ssd automatic chunk", 1, 64, 2, 2, 2, 1, 16, false, false, false, true, false, 0.0f, 1.0f, 0},
    };
    for (const ScanCase& c : scans) scan_case(c, 24, c.chunk_steps >= 32 && c.L / c.chunk_steps >= 4);
    for (const SSDCase& c : ssds) ssd_case(c, 24, c.chunk_steps > 0 && c.L / c.chunk_steps >= 4);
    check_errors();
    if (g_bad) {
        std::printf("%d problem(s)\n", g_bad);
        return 1;
    }
    std::printf("host pipeline ok (%d launches)\n", g_launches);
    return 0;
}
