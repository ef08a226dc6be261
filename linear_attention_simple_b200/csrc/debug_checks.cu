// debug_checks.cu -- input scans of the checking build (-DGLA_DEBUG_BOUNDS,
// libgla_debug.so).
//
// The normal build trusts the preconditions stated in gla.h (a_t <= 0 and
// finite, every input finite) and the index arithmetic of its kernels.  The
// checking build verifies both without faulting: every entry point first
// scans its inputs with the kernels below, and the kernels' direct global
// accesses are guarded by GLA_DCHECK.  A violation records
// GLA_ERR_INVALID_ARG in the device status word (read it with
// gla_get_device_status); the call itself still runs, so a caller sees the
// same outputs it would see from the normal build, plus the recorded status.
// In the normal build debug_scan() returns at once and launches nothing.
#include <cuda_bf16.h>

#include "gla_device.cuh"

namespace gla {
namespace {

#ifdef GLA_DEBUG_BOUNDS
constexpr int kScanThreads = 256;
constexpr int kScanBlocks = 592;   // four per SM of a B200

// a must be <= 0 and finite (NaN fails the first test, -inf the second).
__global__ void __launch_bounds__(kScanThreads) scan_decay_kernel(const float* __restrict__ a, int64_t n,
                                                                  int* __restrict__ status)
{
    bool bad = false;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float x = a[i];
        bad |= !(x <= 0.f) || isinf(x);
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) record_status(status, GLA_ERR_INVALID_ARG);
}

// rows of `width` bf16 values, `ld` elements apart: none may be inf or NaN
// (exponent field all ones).
__global__ void __launch_bounds__(kScanThreads) scan_bf16_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                                 int64_t ld, int64_t width, int* __restrict__ status)
{
    bool bad = false;
    const int64_t n = rows * width;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / width, c = i - r * width;
        bad |= (x[r * ld + c] & 0x7F80u) == 0x7F80u;
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) record_status(status, GLA_ERR_INVALID_ARG);
}

__global__ void __launch_bounds__(kScanThreads) scan_f32_kernel(const float* __restrict__ x, int64_t n,
                                                                int* __restrict__ status)
{
    bool bad = false;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        bad |= !isfinite(x[i]);
    if (__syncthreads_or(bad) && threadIdx.x == 0) record_status(status, GLA_ERR_INVALID_ARG);
}

unsigned blocks_for(int64_t n)
{
    const int64_t b = (n + kScanThreads - 1) / kScanThreads;
    return static_cast<unsigned>(b < kScanBlocks ? (b < 1 ? 1 : b) : kScanBlocks);
}
#endif

}  // namespace

gla_status debug_scan(const DebugScan& s, int* status, cudaStream_t st)
{
#ifdef GLA_DEBUG_BOUNDS
    if (s.a && s.na > 0) {
        scan_decay_kernel<<<blocks_for(s.na), kScanThreads, 0, st>>>(s.a, s.na, status);
        count_launch();
        if (check_launch("scan_decay_kernel") != GLA_OK) return GLA_ERR_CUDA;
    }
    for (int i = 0; i < DebugScan::kMaxBf16; ++i) {
        const DebugScan::Rows& t = s.bf16[i];
        if (!t.base || t.rows <= 0 || t.width <= 0) continue;
        scan_bf16_kernel<<<blocks_for(t.rows * t.width), kScanThreads, 0, st>>>(
            static_cast<const uint16_t*>(t.base), t.rows, t.ld, t.width, status);
        count_launch();
        if (check_launch("scan_bf16_kernel") != GLA_OK) return GLA_ERR_CUDA;
    }
    for (int i = 0; i < DebugScan::kMaxF32; ++i) {
        if (!s.f32[i] || s.nf32[i] <= 0) continue;
        scan_f32_kernel<<<blocks_for(s.nf32[i]), kScanThreads, 0, st>>>(s.f32[i], s.nf32[i], status);
        count_launch();
        if (check_launch("scan_f32_kernel") != GLA_OK) return GLA_ERR_CUDA;
    }
#else
    (void)s;
    (void)status;
    (void)st;
#endif
    return GLA_OK;
}

}  // namespace gla

extern "C" int gla_build_flags(void)
{
#ifdef GLA_DEBUG_BOUNDS
    return GLA_BUILD_DEBUG_BOUNDS;
#else
    return 0;
#endif
}
