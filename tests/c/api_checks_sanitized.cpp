// api_checks_sanitized.cpp -- the C ABI's host-side checks (mm_api.cpp) under
// AddressSanitizer and UndefinedBehaviorSanitizer, on a machine without CUDA.
//
// mm_api.cpp is compiled against a stand-in CUDA runtime (stub_cuda/) with
// the kernel launchers replaced by stubs that only count launches; the
// driver below calls every entry point with sizes at and past every limit
// (0, 1, 2^30, 2^31, 2^62, INT64_MAX, ...), non-finite and boundary scalars,
// and fake 16-byte-aligned pointers that are never dereferenced.  Every call
// must return one of the documented statuses without undefined behaviour
// (no signed overflow in a size product, no invalid shift or conversion),
// and the in-range calls must reach their launcher.  Exit status 0 and
// "api checks ok" when all hold.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <limits>
#include <vector>

#include "cuda_runtime.h"
#include "mm_scan.h"
#include "mm_internal.h"

// ---- the stand-in runtime and launchers --------------------------------------
cudaError_t cudaDeviceSynchronize(void) { return cudaSuccess; }
const char* cudaGetErrorString(cudaError_t) { return "stub"; }
const char* cudaGetErrorName(cudaError_t) { return "stub"; }

namespace {
int g_launches = 0;
}

namespace mmscan {
bool scan_tile_supported(int spt, int warps, int time_lanes) {
    return (spt == 2 || spt == 4 || spt == 8) && warps >= 1 && warps <= 8 && (time_lanes == 1 || time_lanes == 2);
}
ScanTileChoice choose_scan_tile(int64_t, int64_t, int64_t dstate, int, int, int, int) {
    return ScanTileChoice{dstate <= 2 ? 2 : dstate <= 4 ? 4 : dstate <= 8 ? 8 : 16, 2, 4, 1};
}
cudaError_t launch_scan_fwd(const ScanArgs&, const ScanTileChoice&, int, cudaStream_t) { ++g_launches; return cudaSuccess; }
cudaError_t launch_scan_bwd(const ScanBwdArgs&, int, cudaStream_t) { ++g_launches; return cudaSuccess; }
int64_t scan_bwd_det_workspace_bytes(int64_t, int64_t, int, int64_t) { return 1024; }
bool stream_capturing(cudaStream_t) { return false; }
cudaError_t launch_scan_step(const ScanStepArgs&, int, cudaStream_t) { ++g_launches; return cudaSuccess; }
cudaError_t launch_ssd_fwd(const SSDArgs&, cudaStream_t) { ++g_launches; return cudaSuccess; }
cudaError_t launch_ssd_mom(const SSDMomArgs&, cudaStream_t) { ++g_launches; return cudaSuccess; }
int64_t scan_seg_default_len(int64_t, int64_t) { return 16384; }
cudaError_t launch_scan_seg(const ScanArgs&, int, int64_t, bool, cudaStream_t) { ++g_launches; return cudaSuccess; }
int64_t scan_seg_chunk_steps(int io) { return io == 0 ? 32 : 64; }
int64_t scan_seg_tile_channels() { return 16; }
int64_t scan_seg_tile_record_bytes() { return 257 * 16; }
cudaError_t launch_scan_seg_split(const ScanArgs&, int, int64_t, int, void*, int64_t, int64_t, void* const*, int,
                                  cudaStream_t) {
    ++g_launches;
    return cudaSuccess;
}
unsigned int scan_seg_read_and_clear_device_error() { return 0; }
unsigned int scan_read_and_clear_device_error() { return 0; }
unsigned int scan_bwd_read_and_clear_device_error() { return 0; }
unsigned int ssd_read_and_clear_device_error() { return 0; }
bool ssd_shape_supported(int64_t headdim, int64_t dstate, int64_t chunk) {
    return headdim == 64 && dstate == 128 && (chunk == 128 || chunk == 256);
}
bool ssd_mom_tc_shape_supported(int64_t headdim, int64_t dstate) { return headdim == 64 && dstate == 128; }
cudaError_t launch_ssd_mom_tc(const SSDMomArgs&, cudaStream_t) { ++g_launches; return cudaSuccess; }
unsigned int ssd_mom_tc_read_and_clear_device_error() { return 0; }
bool ssd_mom_shape_supported(int64_t headdim, int64_t dstate) {
    return headdim >= 1 && headdim <= 64 && dstate >= 1 && dstate <= 128;
}
}  // namespace mmscan

// ---- the driver ---------------------------------------------------------------
namespace {

int g_bad = 0;

void* fake(int k) { return reinterpret_cast<void*>(static_cast<uintptr_t>(k + 1) << 40); }
float* ffake(int k) { return static_cast<float*>(fake(k)); }

void expect_status(mm_status st, const char* what) {
    if ((int)st < 0 || (int)st > 9) {
        if (g_bad < 10) std::printf("%s: undocumented status %d\n", what, (int)st);
        ++g_bad;
    }
}

const int64_t kSizes[] = {-1, 0, 1, 2, 3, 16, 17, 64, 129, int64_t(1) << 30, (int64_t(1) << 30) + 1,
                          (int64_t(1) << 31) - 1, int64_t(1) << 31, int64_t(1) << 40, int64_t(1) << 62,
                          std::numeric_limits<int64_t>::max()};
const float kScalars[] = {0.0f, -0.0f, 0.5f, 0.999999f, 1.0f, -1.0f, 1e30f, std::numeric_limits<float>::infinity(),
                          std::numeric_limits<float>::quiet_NaN(), std::numeric_limits<float>::denorm_min()};

void scan_calls(const mm_scan_dims& d, float beta, float alpha) {
    expect_status(mm_scan_fwd(fake(0), fake(1), ffake(2), fake(3), fake(4), ffake(5), ffake(6), beta, alpha,
                              fake(7), ffake(8), ffake(9), &d, nullptr), "mm_scan_fwd");
    expect_status(mm_scan_fwd_gated(fake(0), fake(1), ffake(2), fake(3), fake(4), ffake(10), fake(11), ffake(12), 1,
                                    nullptr, nullptr, beta, alpha, fake(7), nullptr, nullptr, ffake(13), &d, nullptr),
                  "mm_scan_fwd_gated");
    expect_status(mm_scan_bwd(fake(0), fake(1), ffake(2), fake(3), fake(4), ffake(5), ffake(6), beta, alpha,
                              ffake(13), fake(14), ffake(15), ffake(16), fake(17), fake(18), ffake(19), ffake(20),
                              ffake(21), ffake(22), ffake(23), &d, nullptr), "mm_scan_bwd");
    expect_status(mm_scan_bwd_gated(fake(0), fake(1), ffake(2), fake(3), fake(4), ffake(10), fake(11), ffake(12), 1,
                                    nullptr, nullptr, beta, alpha, ffake(13), fake(14), nullptr, nullptr, fake(17),
                                    fake(18), ffake(19), ffake(20), ffake(21), ffake(22), fake(23), ffake(24),
                                    nullptr, nullptr, &d, nullptr), "mm_scan_bwd_gated");
    mm_scan_dims one = d;
    one.seqlen = 1;
    expect_status(mm_scan_step(fake(0), fake(1), ffake(2), fake(3), fake(4), nullptr, nullptr, nullptr, 0, ffake(5),
                               ffake(6), beta, alpha, fake(7), &one, nullptr), "mm_scan_step");
    size_t bytes = 0;
    expect_status(mm_scan_ckpt_size(&d, &bytes), "mm_scan_ckpt_size");
    int64_t seg = 0;
    expect_status(mm_scan_segment_len(&d, &seg), "mm_scan_segment_len");
    // the split launches, with their segment length and the piece's place at extremes
    for (int64_t S : {int64_t(-1), int64_t(0), int64_t(32), int64_t(64), int64_t(1) << 30, int64_t(1) << 62})
        for (int64_t first : {int64_t(-64), int64_t(0), int64_t(64), int64_t(1) << 30, int64_t(1) << 62,
                              std::numeric_limits<int64_t>::max() - 1})
            for (int64_t total : {int64_t(0), int64_t(64), d.seqlen, int64_t(1) << 30, std::numeric_limits<int64_t>::max()}) {
                expect_status(mm_scan_fwd_split_correct(fake(1), ffake(2), fake(4), ffake(5), ffake(6), beta, alpha,
                                                        fake(7), ffake(8), ffake(9), fake(10), S, first, total, &d,
                                                        nullptr), "mm_scan_fwd_split_correct");
            }
    for (int64_t S : {int64_t(-1), int64_t(32), int64_t(64), int64_t(1) << 30, int64_t(1) << 62}) {
        expect_status(mm_scan_fwd_split_maps(fake(0), fake(1), ffake(2), fake(3), fake(4), beta, alpha, fake(7),
                                             fake(10), S, &d, nullptr), "mm_scan_fwd_split_maps");
        for (int nd : {0, 1, 65})
            for (int64_t first : {int64_t(0), int64_t(1) << 40})
                expect_status(mm_scan_fwd_split_maps_peers(fake(0), fake(1), ffake(2), fake(3), fake(4), beta, alpha,
                                                           fake(7), reinterpret_cast<void* const*>(fake(11)), nd,
                                                           first, S,
                                                           d.seqlen > INT64_MAX - first ? INT64_MAX : first + d.seqlen,
                                                           &d, nullptr),
                              "mm_scan_fwd_split_maps_peers");
    }
    for (int64_t n : {int64_t(-1), int64_t(0), int64_t(1), int64_t(1) << 30, int64_t(1) << 31})
        expect_status(mm_scan_split_maps_size(&d, n, &bytes), "mm_scan_split_maps_size");
}

void ssd_calls(const mm_ssd_dims& d, float beta, float alpha) {
    expect_status(mm_ssd_fwd(fake(0), ffake(1), ffake(2), fake(3), fake(4), ffake(5), beta, alpha, fake(6), ffake(7),
                             &d, nullptr), "mm_ssd_fwd");
    expect_status(mm_ssd_fwd_momentum(fake(0), ffake(1), ffake(2), fake(3), fake(4), ffake(5), ffake(9), beta, alpha,
                                      fake(6), ffake(7), ffake(10), &d, nullptr), "mm_ssd_fwd_momentum");
}

}  // namespace

int main() {
    // every scan size at every extreme, one field at a time, and all at once
    for (int field = 0; field < 5; ++field)
        for (int64_t v : kSizes) {
            mm_scan_dims d = {2, 64, 8, 16, MM_F32};
            int64_t* f[] = {&d.batch, &d.seqlen, &d.dim, &d.dstate};
            if (field < 4) *f[field] = v;
            else d.batch = d.seqlen = d.dim = v;
            for (int io : {0, 1, 7}) {
                d.io = static_cast<mm_dtype>(io);
                scan_calls(d, 0.9f, 1.0f);
            }
        }
    for (float b : kScalars)
        for (float a : kScalars) scan_calls(mm_scan_dims{1, 32, 4, 16, MM_BF16}, b, a);
    // the SSD sizes likewise
    for (int field = 0; field < 8; ++field)
        for (int64_t v : kSizes) {
            mm_ssd_dims d = {2, 256, 4, 64, 128, 1, 256};
            int64_t* f[] = {&d.batch, &d.seqlen, &d.nheads, &d.headdim, &d.dstate, &d.ngroups, &d.chunk};
            if (field < 7) *f[field] = v;
            else d.batch = d.seqlen = d.nheads = v;
            for (float b : {0.0f, 0.9f}) ssd_calls(d, b, 1.0f);
        }
    for (float b : kScalars)
        for (float a : kScalars) ssd_calls(mm_ssd_dims{1, 128, 2, 64, 128, 1, 128}, b, a);
    // in-range calls reach their launchers
    const int before = g_launches;
    const mm_scan_dims ok = {2, 64, 8, 16, MM_F32};
    if (mm_scan_fwd(fake(0), fake(1), ffake(2), fake(3), fake(4), nullptr, nullptr, 0.9f, 1.0f, fake(7), nullptr,
                    nullptr, &ok, nullptr) != MM_OK || g_launches != before + 1) {
        std::printf("an in-range scan call did not launch\n");
        ++g_bad;
    }
    const mm_ssd_dims sok = {1, 256, 2, 64, 128, 1, 256};
    if (mm_ssd_fwd(fake(0), ffake(1), ffake(2), fake(3), fake(4), nullptr, 0.0f, 1.0f, fake(6), nullptr,
                   &sok, nullptr) != MM_OK || g_launches != before + 2) {
        std::printf("an in-range SSD call did not launch\n");
        ++g_bad;
    }
    const mm_scan_dims piece = {2, 128, 8, 16, MM_F32};
    if (mm_scan_fwd_split_maps(fake(0), fake(1), ffake(2), fake(3), fake(4), 0.9f, 1.0f, fake(7), fake(10), 64,
                               &piece, nullptr) != MM_OK ||
        mm_scan_fwd_split_correct(fake(1), ffake(2), fake(4), nullptr, nullptr, 0.9f, 1.0f, fake(7), ffake(8),
                                  nullptr, fake(10), 64, 128, 300, &piece, nullptr) != MM_OK ||
        g_launches != before + 4) {
        std::printf("an in-range split call did not launch\n");
        ++g_bad;
    }
    expect_status(mm_device_status(), "mm_device_status");
    if (g_bad) return 1;
    std::printf("api checks ok (%d launches)\n", g_launches);
    return 0;
}
