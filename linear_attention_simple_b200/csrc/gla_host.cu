// gla_host.cu -- the exported C ABI of libgla (include/gla.h): argument
// validation, workspace sizing, status reporting and dispatch to the kernel
// launchers.  Nothing here allocates device memory or synchronises, except
// gla_get_device_status, which is documented to synchronise.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "gla_internal.h"

namespace gla {

// Device status word: kernels record the first error of a launch here
// (first writer wins).  One instance per device that loads the module.
__device__ int g_device_status;

namespace {

thread_local int t_last_cuda_error = 0;
std::atomic<unsigned long long> g_launches{0};
std::atomic<unsigned long long> g_wait_limit_ns{0};
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;  // 2 s
constexpr int kMaxDevices = 64;
int* g_status_addr[kMaxDevices] = {};
const void* g_status_ctx[kMaxDevices] = {};
std::mutex g_status_mu;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gla_status cuda_fail(cudaError_t e)
{
    t_last_cuda_error = static_cast<int>(e);
    return GLA_ERR_CUDA;
}

}  // namespace

// The driver context current on this thread (an opaque handle; null when it
// cannot be read), fetched through the runtime's driver entry point so that
// the library need not link the driver library.
const void* current_cu_context()
{
    typedef CUresult (*GetCtxFn)(CUcontext*);
    static GetCtxFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<GetCtxFn>(p);
    });
    CUcontext c = nullptr;
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

namespace {

int* status_addr_current(gla_status* err)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *err = cuda_fail(e == cudaSuccess ? cudaErrorInvalidDevice : e);
        return nullptr;
    }
    const void* ctx = current_cu_context();
    std::lock_guard<std::mutex> lk(g_status_mu);
    // looked up again whenever the device's current context is not the one
    // the cached address belongs to (a reset device, another context)
    if (!g_status_addr[dev] || g_status_ctx[dev] != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_device_status);
        if (e != cudaSuccess) {
            *err = cuda_fail(e);
            return nullptr;
        }
        g_status_addr[dev] = static_cast<int*>(p);
        g_status_ctx[dev] = ctx;
    }
    *err = GLA_OK;
    return g_status_addr[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Trace records: one (start, end, name) per launch while enabled.
struct TraceRec {
    cudaEvent_t start, end;
    const char* name;
};
std::atomic<bool> g_trace_on{false};
std::mutex g_trace_mu;
std::vector<TraceRec> g_trace;
std::vector<cudaEvent_t> g_event_pool;
thread_local cudaEvent_t t_pending_start = nullptr;

cudaEvent_t pool_event()
{
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

}  // namespace

void trace_begin(cudaStream_t st)
{
    if (!g_trace_on.load()) return;
    std::lock_guard<std::mutex> lk(g_trace_mu);
    t_pending_start = pool_event();
    if (t_pending_start) cudaEventRecord(t_pending_start, st);
}

void trace_end(cudaStream_t st, const char* name)
{
    if (!g_trace_on.load() || !t_pending_start) return;
    std::lock_guard<std::mutex> lk(g_trace_mu);
    cudaEvent_t e = pool_event();
    if (!e) return;
    cudaEventRecord(e, st);
    g_trace.push_back({t_pending_start, e, name});
    t_pending_start = nullptr;
}

WaitCtl wait_ctl_for_current_device(gla_status* err)
{
    WaitCtl c;
    c.status = status_addr_current(err);
    const unsigned long long lim = g_wait_limit_ns.load();
    c.limit_ns = lim ? lim : kDefaultWaitNs;
    return c;
}

gla_status status_of(cudaError_t e) { return e == cudaSuccess ? GLA_OK : cuda_fail(e); }

gla_status check_launch(const char* what)
{
    (void)what;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return GLA_OK;
}

void count_launch(unsigned n) { g_launches.fetch_add(n); }

gla_status make_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box, int elem_bytes,
                     int swizzle_bytes)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cuda_fail(cudaErrorNotSupported);
    cuuint64_t gd[5], gs[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        gd[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
        if (i > 0) gs[i - 1] = strides_bytes[i];
    }
    CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_NONE;
    if (swizzle_bytes == 32) sw = CU_TENSOR_MAP_SWIZZLE_32B;
    if (swizzle_bytes == 64) sw = CU_TENSOR_MAP_SWIZZLE_64B;
    if (swizzle_bytes == 128) sw = CU_TENSOR_MAP_SWIZZLE_128B;
    const CUtensorMapDataType dt =
        elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    CUresult r = fn(map, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), gd, gs, bx,
                    es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    return GLA_OK;
}

}  // namespace gla

using namespace gla;

namespace {

bool bad_scale(float s) { return !(s > 0.0f) || !std::isfinite(s); }

// Shared validation of the chunked entry points.  Returns GLA_OK or the
// first failing status; fills the token strides.
gla_status validate_chunk(const void* q, const void* k, const void* v, const float* a, int B,
                          int T, int H, int dk, int dv, int64_t ld_qkv, float scale,
                          gla_dtype dt, int64_t* ld_qk, int64_t* ld_v)
{
    if (B < 0 || T < 0 || H < 0) return GLA_ERR_INVALID_ARG;
    if (dt != GLA_BF16 && dt != GLA_F32) return GLA_ERR_INVALID_ARG;
    if (bad_scale(scale)) return GLA_ERR_INVALID_ARG;
    if (dk <= 0 || dv <= 0) return GLA_ERR_INVALID_ARG;
    if (dk != kDk || dv != kDv) return GLA_ERR_UNSUPPORTED;
    const int64_t esz = dt == GLA_BF16 ? 2 : 4;
    const int64_t packed_qk = static_cast<int64_t>(H) * dk;
    const int64_t packed_v = static_cast<int64_t>(H) * dv;
    if (ld_qkv < 0) return GLA_ERR_INVALID_ARG;
    if (ld_qkv == 0) {
        *ld_qk = packed_qk;
        *ld_v = packed_v;
    } else {
        if (ld_qkv < packed_qk || ld_qkv < packed_v) return GLA_ERR_INVALID_ARG;
        if ((ld_qkv * esz) % 16 != 0) return GLA_ERR_MISALIGNED;
        *ld_qk = ld_qkv;
        *ld_v = ld_qkv;
    }
    if (static_cast<int64_t>(B) * T * H == 0) return GLA_OK;
    if (!q || !k || !v || !a) return GLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(a)) return GLA_ERR_MISALIGNED;
    if (static_cast<int64_t>(T) * (*ld_v) * B > (int64_t(1) << 40)) return GLA_ERR_UNSUPPORTED;
    return GLA_OK;
}

// The checking build's scan of a chunked call's inputs (no-op otherwise):
// q, k [rows = B*T][H*96] and v [rows][H*192] at token stride ld, dO packed.
gla_status scan_chunk_inputs(const void* q, const void* k, const void* v, const float* a, const void* dO,
                             const float* s0, const float* s_extra, int B, int T, int H, int64_t ld_qk,
                             int64_t ld_v, int* status, cudaStream_t st)
{
    DebugScan d;
    const int64_t rows = static_cast<int64_t>(B) * T;
    d.a = a;
    d.na = rows * H;
    d.bf16[0] = {q, rows, ld_qk, static_cast<int64_t>(H) * kDk};
    d.bf16[1] = {k, rows, ld_qk, static_cast<int64_t>(H) * kDk};
    d.bf16[2] = {v, rows, ld_v, static_cast<int64_t>(H) * kDv};
    d.bf16[3] = {dO, rows, static_cast<int64_t>(H) * kDv, static_cast<int64_t>(H) * kDv};
    const int64_t ns = static_cast<int64_t>(B) * H * kDk * kDv;
    d.f32[0] = s0;
    d.nf32[0] = s0 ? ns : 0;
    d.f32[1] = s_extra;
    d.nf32[1] = s_extra ? ns : 0;
    return debug_scan(d, status, st);
}

}  // namespace

extern "C" {

const char* gla_status_string(gla_status s)
{
    switch (s) {
    case GLA_OK: return "GLA_OK";
    case GLA_ERR_INVALID_ARG: return "GLA_ERR_INVALID_ARG";
    case GLA_ERR_UNSUPPORTED: return "GLA_ERR_UNSUPPORTED";
    case GLA_ERR_MISALIGNED: return "GLA_ERR_MISALIGNED";
    case GLA_ERR_CUDA: return "GLA_ERR_CUDA";
    case GLA_ERR_TIMEOUT: return "GLA_ERR_TIMEOUT";
    }
    return "GLA_ERR_UNKNOWN";
}

int gla_last_cuda_error(void) { return t_last_cuda_error; }

unsigned long long gla_launch_count(void) { return g_launches.load(); }

size_t gla_chunk_workspace_bytes(int B, int T, int H, int dk, int dv, int for_bwd)
{
    if (B <= 0 || T <= 0 || H <= 0 || dk != kDk || dv != kDv) return 0;
    if (for_bwd == 2) return bwd_workspace_bytes(B, T, H, true);
    return for_bwd ? bwd_workspace_bytes(B, T, H) : fwd_workspace_bytes(B, T, H);
}

size_t gla_chunk_saved_state_bytes(int B, int T, int H, int dk, int dv)
{
    if (B <= 0 || T <= 0 || H <= 0 || dk != kDk || dv != kDv) return 0;
    const size_t NC = (static_cast<size_t>(T) + kChunk - 1) / kChunk;
    return static_cast<size_t>(B) * H * NC * 2 * kDk * kDv * 2;
}

gla_status gla_chunk_fwd(const void* q, const void* k, const void* v, const float* a,
                         const float* s0, void* o, float* s_final, void* ws, size_t ws_bytes,
                         int B, int T, int H, int dk, int dv, int64_t ld_qkv, float scale,
                         gla_dtype dt, cudaStream_t stream)
{
    int64_t ld_qk = 0, ld_v = 0;
    gla_status s = validate_chunk(q, k, v, a, B, T, H, dk, dv, ld_qkv, scale, dt, &ld_qk, &ld_v);
    if (s != GLA_OK) return s;
    if (!aligned16(s0) || !aligned16(s_final) || !aligned16(ws)) return GLA_ERR_MISALIGNED;
    if (static_cast<int64_t>(B) * H == 0) return GLA_OK;
    if (T == 0) {
        // Empty sequence: S_T = S_0.
        if (!s_final) return GLA_OK;
        const size_t bytes = static_cast<size_t>(B) * H * dk * dv * sizeof(float);
        cudaError_t e = s0 ? cudaMemcpyAsync(s_final, s0, bytes, cudaMemcpyDeviceToDevice, stream)
                           : cudaMemsetAsync(s_final, 0, bytes, stream);
        return e == cudaSuccess ? GLA_OK : cuda_fail(e);
    }
    if (!o) return GLA_ERR_INVALID_ARG;
    if (!aligned16(o)) return GLA_ERR_MISALIGNED;
    gla_status se;
    WaitCtl ctl = wait_ctl_for_current_device(&se);
    if (se != GLA_OK) return se;
    if (dt == GLA_F32)
        return launch_fwd_f32(static_cast<const float*>(q), static_cast<const float*>(k),
                              static_cast<const float*>(v), a, s0, static_cast<float*>(o),
                              s_final, B, T, H, ld_qk, ld_v, scale, ctl, stream);
    const size_t need = fwd_workspace_bytes(B, T, H);
    if (need > 0 && (!ws || ws_bytes < need)) return GLA_ERR_INVALID_ARG;
    if ((s = scan_chunk_inputs(q, k, v, a, nullptr, s0, nullptr, B, T, H, ld_qk, ld_v, ctl.status, stream)) !=
        GLA_OK)
        return s;
    ChunkProblem p{q, k, v, a, B, T, H, ld_qk, ld_v, scale};
    return run_chunk_fwd(p, s0, o, s_final, ws, ws_bytes, ctl, stream);
}

size_t gla_chunk_varlen_workspace_bytes(int N, int total_T, int H, int dk, int dv)
{
    if (N <= 0 || total_T <= 0 || H <= 0 || dk != kDk || dv != kDv) return 0;
    return varlen_workspace_bytes(N, total_T, H);
}

gla_status gla_chunk_fwd_train(const void* q, const void* k, const void* v, const float* a,
                               const float* s0, void* o, float* s_final, void* saved, size_t saved_bytes,
                               void* ws, size_t ws_bytes, int B, int T, int H, int dk, int dv, int64_t ld_qkv,
                               float scale, gla_dtype dt, cudaStream_t stream)
{
    int64_t ld_qk = 0, ld_v = 0;
    gla_status s = validate_chunk(q, k, v, a, B, T, H, dk, dv, ld_qkv, scale, dt, &ld_qk, &ld_v);
    if (s != GLA_OK) return s;
    if (dt != GLA_BF16) return GLA_ERR_UNSUPPORTED;
    if (!aligned16(s0) || !aligned16(s_final) || !aligned16(ws) || !aligned16(saved)) return GLA_ERR_MISALIGNED;
    if (static_cast<int64_t>(B) * T * H == 0) return gla_chunk_fwd(q, k, v, a, s0, o, s_final, ws, ws_bytes, B, T,
                                                                     H, dk, dv, ld_qkv, scale, dt, stream);
    if (!o || !saved || saved_bytes < gla_chunk_saved_state_bytes(B, T, H, dk, dv)) return GLA_ERR_INVALID_ARG;
    if (!aligned16(o)) return GLA_ERR_MISALIGNED;
    const size_t need = fwd_workspace_bytes(B, T, H);
    if (need > 0 && (!ws || ws_bytes < need)) return GLA_ERR_INVALID_ARG;
    gla_status se;
    WaitCtl ctl = wait_ctl_for_current_device(&se);
    if (se != GLA_OK) return se;
    if ((s = scan_chunk_inputs(q, k, v, a, nullptr, s0, nullptr, B, T, H, ld_qk, ld_v, ctl.status, stream)) !=
        GLA_OK)
        return s;
    ChunkProblem p{q, k, v, a, B, T, H, ld_qk, ld_v, scale};
    return run_chunk_fwd(p, s0, o, s_final, ws, ws_bytes, ctl, stream, saved);
}

gla_status gla_chunk_fwd_varlen(const void* q, const void* k, const void* v, const float* a,
                                const int32_t* cu_seqlens, int N, const float* s0, void* o, float* s_final,
                                void* ws, size_t ws_bytes, int total_T, int H, int dk, int dv, int64_t ld_qkv,
                                float scale, gla_dtype dt, cudaStream_t stream)
{
    if (N < 0 || N > 65535) return N < 0 ? GLA_ERR_INVALID_ARG : GLA_ERR_UNSUPPORTED;
    int64_t ld_qk = 0, ld_v = 0;
    gla_status s = validate_chunk(q, k, v, a, 1, total_T, H, dk, dv, ld_qkv, scale, dt, &ld_qk, &ld_v);
    if (s != GLA_OK) return s;
    if (dt != GLA_BF16) return GLA_ERR_UNSUPPORTED;
    if (!aligned16(s0) || !aligned16(s_final) || !aligned16(ws)) return GLA_ERR_MISALIGNED;
    if (N == 0 || H == 0) return GLA_OK;
    if (!cu_seqlens) return GLA_ERR_INVALID_ARG;
    if (total_T > 0 && !o) return GLA_ERR_INVALID_ARG;
    if (!aligned16(o)) return GLA_ERR_MISALIGNED;
    gla_status se;
    WaitCtl ctl = wait_ctl_for_current_device(&se);
    if (se != GLA_OK) return se;
    if ((s = scan_chunk_inputs(q, k, v, a, nullptr, nullptr, nullptr, 1, total_T, H, ld_qk, ld_v, ctl.status,
                               stream)) != GLA_OK)
        return s;
    ChunkProblem p{q, k, v, a, 1, total_T, H, ld_qk, ld_v, scale};
    return run_chunk_fwd_varlen(p, cu_seqlens, N, s0, o, s_final, ws, ws_bytes, ctl, stream);
}

gla_status gla_chunk_bwd(const void* q, const void* k, const void* v, const float* a,
                         const float* s0, const void* dO, const float* ds_final,
                         void* grad_q, void* grad_k, void* grad_v, float* grad_a,
                         float* grad_s0, void* ws, size_t ws_bytes, int B, int T, int H, int dk,
                         int dv, int64_t ld_qkv, float scale, gla_dtype dt, cudaStream_t stream)
{
    int64_t ld_qk = 0, ld_v = 0;
    gla_status s = validate_chunk(q, k, v, a, B, T, H, dk, dv, ld_qkv, scale, dt, &ld_qk, &ld_v);
    if (s != GLA_OK) return s;
    if (dt != GLA_BF16) return GLA_ERR_UNSUPPORTED;
    if (!aligned16(s0) || !aligned16(ds_final) || !aligned16(grad_s0) || !aligned16(ws))
        return GLA_ERR_MISALIGNED;
    if (static_cast<int64_t>(B) * H == 0) return GLA_OK;
    if (T == 0) {
        // Empty sequence: dL/dS_0 = dL/dS_T.
        if (!grad_s0) return GLA_OK;
        const size_t bytes = static_cast<size_t>(B) * H * dk * dv * sizeof(float);
        cudaError_t e = ds_final
                            ? cudaMemcpyAsync(grad_s0, ds_final, bytes, cudaMemcpyDeviceToDevice,
                                              stream)
                            : cudaMemsetAsync(grad_s0, 0, bytes, stream);
        return e == cudaSuccess ? GLA_OK : cuda_fail(e);
    }
    if (!dO || !grad_q || !grad_k || !grad_v || !grad_a) return GLA_ERR_INVALID_ARG;
    if (!aligned16(dO) || !aligned16(grad_q) || !aligned16(grad_k) || !aligned16(grad_v) ||
        !aligned16(grad_a))
        return GLA_ERR_MISALIGNED;
    const size_t need = bwd_workspace_bytes(B, T, H);
    if (need > 0 && (!ws || ws_bytes < need)) return GLA_ERR_INVALID_ARG;
    gla_status se;
    WaitCtl ctl = wait_ctl_for_current_device(&se);
    if (se != GLA_OK) return se;
    if ((s = scan_chunk_inputs(q, k, v, a, dO, s0, ds_final, B, T, H, ld_qk, ld_v, ctl.status, stream)) !=
        GLA_OK)
        return s;
    ChunkProblem p{q, k, v, a, B, T, H, ld_qk, ld_v, scale};
    return run_chunk_bwd(p, s0, dO, ds_final, grad_q, grad_k, grad_v, grad_a, grad_s0, ws,
                         ws_bytes, ctl, stream);
}

gla_status gla_chunk_bwd_saved(const void* q, const void* k, const void* v, const float* a, const void* saved,
                               size_t saved_bytes, const float* s_final, const void* dO, const float* ds_final,
                               void* grad_q, void* grad_k, void* grad_v, float* grad_a, float* grad_s0, void* ws,
                               size_t ws_bytes, int B, int T, int H, int dk, int dv, int64_t ld_qkv, float scale,
                               gla_dtype dt, cudaStream_t stream)
{
    int64_t ld_qk = 0, ld_v = 0;
    gla_status s = validate_chunk(q, k, v, a, B, T, H, dk, dv, ld_qkv, scale, dt, &ld_qk, &ld_v);
    if (s != GLA_OK) return s;
    if (dt != GLA_BF16) return GLA_ERR_UNSUPPORTED;
    if (!aligned16(saved) || !aligned16(s_final) || !aligned16(ds_final) || !aligned16(grad_s0) || !aligned16(ws))
        return GLA_ERR_MISALIGNED;
    if (static_cast<int64_t>(B) * H == 0) return GLA_OK;
    if (T == 0)   // no chunks, nothing saved: the plain backward's empty case
        return gla_chunk_bwd(q, k, v, a, nullptr, dO, ds_final, grad_q, grad_k, grad_v, grad_a, grad_s0, ws,
                             ws_bytes, B, T, H, dk, dv, ld_qkv, scale, dt, stream);
    if (!saved || saved_bytes < gla_chunk_saved_state_bytes(B, T, H, dk, dv)) return GLA_ERR_INVALID_ARG;
    if (ds_final && !s_final) return GLA_ERR_INVALID_ARG;   // <dS_T, S_T> needs the final state
    if (!dO || !grad_q || !grad_k || !grad_v || !grad_a) return GLA_ERR_INVALID_ARG;
    if (!aligned16(dO) || !aligned16(grad_q) || !aligned16(grad_k) || !aligned16(grad_v) || !aligned16(grad_a))
        return GLA_ERR_MISALIGNED;
    const size_t need = bwd_workspace_bytes(B, T, H, true);
    if (need > 0 && (!ws || ws_bytes < need)) return GLA_ERR_INVALID_ARG;
    gla_status se;
    WaitCtl ctl = wait_ctl_for_current_device(&se);
    if (se != GLA_OK) return se;
    if ((s = scan_chunk_inputs(q, k, v, a, dO, s_final, ds_final, B, T, H, ld_qk, ld_v, ctl.status, stream)) !=
        GLA_OK)
        return s;
    ChunkProblem p{q, k, v, a, B, T, H, ld_qk, ld_v, scale};
    return run_chunk_bwd(p, nullptr, dO, ds_final, grad_q, grad_k, grad_v, grad_a, grad_s0, ws, ws_bytes, ctl,
                         stream, saved, s_final);
}

size_t gla_segment_workspace_bytes(int B, int T, int H, int dk, int dv)
{
    if (B <= 0 || T <= 0 || H <= 0 || dk != kDk || dv != kDv) return 0;
    return segment_workspace_bytes(B, T, H);
}

}  // extern "C"

namespace {

// Shared by gla_segment_state_fwd / _bwd: u = k or q (dk wide, token stride
// ld_u), y = v or dO (dv wide, token stride ld_y).
gla_status segment_state(const void* u, const void* y, const float* a, float* s_seg, float* g_seg, void* ws,
                         size_t ws_bytes, int B, int T, int H, int dk, int dv, int64_t ld_u, int64_t ld_y,
                         float scale, bool reverse, cudaStream_t stream)
{
    if (static_cast<int64_t>(B) * H == 0) return GLA_OK;
    if (!s_seg) return GLA_ERR_INVALID_ARG;
    if (!aligned16(s_seg) || !aligned16(g_seg) || !aligned16(ws)) return GLA_ERR_MISALIGNED;
    if (T == 0) {
        // an empty segment contributes nothing and does not decay
        cudaError_t e = cudaMemsetAsync(s_seg, 0, static_cast<size_t>(B) * H * dk * dv * sizeof(float), stream);
        if (e == cudaSuccess && g_seg) e = cudaMemsetAsync(g_seg, 0, static_cast<size_t>(B) * H * sizeof(float), stream);
        return e == cudaSuccess ? GLA_OK : cuda_fail(e);
    }
    if (!ws || ws_bytes < segment_workspace_bytes(B, T, H)) return GLA_ERR_INVALID_ARG;
    gla_status se;
    WaitCtl ctl = wait_ctl_for_current_device(&se);
    if (se != GLA_OK) return se;
    DebugScan d;
    const int64_t rows = static_cast<int64_t>(B) * T;
    d.a = a;
    d.na = rows * H;
    d.bf16[0] = {u, rows, ld_u, static_cast<int64_t>(H) * dk};
    d.bf16[1] = {y, rows, ld_y, static_cast<int64_t>(H) * dv};
    gla_status s = debug_scan(d, ctl.status, stream);
    if (s != GLA_OK) return s;
    return run_segment_state(u, y, a, B, T, H, ld_u, ld_y, scale, reverse, s_seg, g_seg, ws, ctl, stream);
}

}  // namespace

extern "C" {

gla_status gla_segment_state_fwd(const void* k, const void* v, const float* a, float* s_seg, float* g_seg,
                                 void* ws, size_t ws_bytes, int B, int T, int H, int dk, int dv, int64_t ld_qkv,
                                 gla_dtype dt, cudaStream_t stream)
{
    int64_t ld_qk = 0, ld_v = 0;
    // q is not read: k stands in for it in the shared validation
    gla_status s = validate_chunk(k, k, v, a, B, T, H, dk, dv, ld_qkv, 1.0f, dt, &ld_qk, &ld_v);
    if (s != GLA_OK) return s;
    if (dt != GLA_BF16) return GLA_ERR_UNSUPPORTED;
    return segment_state(k, v, a, s_seg, g_seg, ws, ws_bytes, B, T, H, dk, dv, ld_qk, ld_v, 1.0f, false, stream);
}

gla_status gla_segment_state_bwd(const void* q, const void* dO, const float* a, float* ds_seg, float* g_seg,
                                 void* ws, size_t ws_bytes, int B, int T, int H, int dk, int dv, int64_t ld_qkv,
                                 float scale, gla_dtype dt, cudaStream_t stream)
{
    int64_t ld_qk = 0, ld_v = 0;
    // dO is contiguous; the shared validation checks it in v's place, and its
    // stride is the packed H*dv whatever ld_qkv is
    gla_status s = validate_chunk(q, q, dO, a, B, T, H, dk, dv, ld_qkv, scale, dt, &ld_qk, &ld_v);
    if (s != GLA_OK) return s;
    if (dt != GLA_BF16) return GLA_ERR_UNSUPPORTED;
    return segment_state(q, dO, a, ds_seg, g_seg, ws, ws_bytes, B, T, H, dk, dv, ld_qk,
                         static_cast<int64_t>(H) * dv, scale, true, stream);
}

gla_status gla_state_fold(const float* s, const float* g, int n, int reverse, const float* s_in, float* out,
                          int units, int dk, int dv, cudaStream_t stream)
{
    if (n < 0 || units < 0 || dk <= 0 || dv <= 0) return GLA_ERR_INVALID_ARG;
    if (dk != kDk || dv != kDv) return GLA_ERR_UNSUPPORTED;
    if (units == 0) return GLA_OK;
    if (!out || (n > 0 && (!s || !g))) return GLA_ERR_INVALID_ARG;
    // g is read one float at a time: 4-byte alignment suffices
    if (!aligned16(s) || !aligned16(s_in) || !aligned16(out) || (reinterpret_cast<uintptr_t>(g) & 3u))
        return GLA_ERR_MISALIGNED;
    return launch_state_fold(s, g, n, units, reverse ? 1 : 0, s_in, out, stream);
}

gla_status gla_decode_step(float* state, const int32_t* slot_idx, int n_slots, const void* q, const void* k,
                           const void* v, const float* a, float* o, int N, int H, int dk, int dv,
                           float scale, cudaStream_t stream)
{
    if (N < 0 || H < 0 || dk <= 0 || dv <= 0) return GLA_ERR_INVALID_ARG;
    if (n_slots < 0 || (!slot_idx && n_slots < N)) return GLA_ERR_INVALID_ARG;
    if (bad_scale(scale)) return GLA_ERR_INVALID_ARG;
    if (dk != kDk || dv != kDv) return GLA_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(N) * H == 0) return GLA_OK;
    if (!state || !q || !k || !v || !a || !o) return GLA_ERR_INVALID_ARG;
    if (!aligned16(state) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(a) ||
        !aligned16(o) || !aligned16(slot_idx))
        return GLA_ERR_MISALIGNED;
    gla_status se;
    WaitCtl ctl = wait_ctl_for_current_device(&se);
    if (se != GLA_OK) return se;
    DebugScan d;
    d.a = a;
    d.na = static_cast<int64_t>(N) * H;
    d.bf16[0] = {q, static_cast<int64_t>(N) * H, dk, dk};
    d.bf16[1] = {k, static_cast<int64_t>(N) * H, dk, dk};
    d.bf16[2] = {v, static_cast<int64_t>(N) * H, dv, dv};
    gla_status s = debug_scan(d, ctl.status, stream);
    if (s != GLA_OK) return s;
    return launch_decode(state, slot_idx, n_slots, q, k, v, a, o, N, H, scale, ctl.status, stream);
}

gla_status conv1d_silu_causal(const void* x, int apply_ln, const float* ln_gamma,
                              const float* ln_beta, float ln_eps, const float* w,
                              const float* bias, const float* conv_state_in,
                              float* conv_state_out, void* y, int B, int T, int D, int W,
                              cudaStream_t stream)
{
    if (B < 0 || T < 0 || D <= 0 || W <= 0) return GLA_ERR_INVALID_ARG;
    if (apply_ln && !(ln_eps > 0.0f && std::isfinite(ln_eps))) return GLA_ERR_INVALID_ARG;
    if (W != 4 || D % 8 != 0 || D > 4096) return GLA_ERR_UNSUPPORTED;
    if (!w) return GLA_ERR_INVALID_ARG;
    if (conv_state_in && conv_state_in == conv_state_out) return GLA_ERR_INVALID_ARG;
    if (B == 0) return GLA_OK;
    if (T == 0) {
        if (!conv_state_out) return GLA_OK;
        const size_t bytes = static_cast<size_t>(B) * (W - 1) * D * sizeof(float);
        cudaError_t e = conv_state_in ? cudaMemcpyAsync(conv_state_out, conv_state_in, bytes,
                                                        cudaMemcpyDeviceToDevice, stream)
                                      : cudaMemsetAsync(conv_state_out, 0, bytes, stream);
        return e == cudaSuccess ? GLA_OK : cuda_fail(e);
    }
    if (!x || !y) return GLA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y) || !aligned16(w) || !aligned16(ln_gamma) ||
        !aligned16(ln_beta) || !aligned16(bias) || !aligned16(conv_state_in) ||
        !aligned16(conv_state_out))
        return GLA_ERR_MISALIGNED;
    return launch_conv(x, apply_ln, ln_gamma, ln_beta, ln_eps, w, bias, conv_state_in,
                       conv_state_out, y, B, T, D, stream);
}

gla_status conv1d_silu_decode_step(const void* x, const int32_t* slot_idx, int n_slots, int apply_ln,
                                   const float* ln_gamma, const float* ln_beta, float ln_eps,
                                   const float* w, const float* bias, float* conv_state, void* y,
                                   int N, int D, int W, cudaStream_t stream)
{
    if (N < 0 || D <= 0 || W <= 0) return GLA_ERR_INVALID_ARG;
    if (n_slots < 0 || (!slot_idx && n_slots < N)) return GLA_ERR_INVALID_ARG;
    if (apply_ln && !(ln_eps > 0.0f && std::isfinite(ln_eps))) return GLA_ERR_INVALID_ARG;
    if (W != 4 || D % 8 != 0 || D > 4096) return GLA_ERR_UNSUPPORTED;
    if (N == 0) return GLA_OK;
    if (!x || !y || !w || !conv_state) return GLA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y) || !aligned16(w) || !aligned16(ln_gamma) || !aligned16(ln_beta) ||
        !aligned16(bias) || !aligned16(conv_state))
        return GLA_ERR_MISALIGNED;
    gla_status se;
    WaitCtl ctl = wait_ctl_for_current_device(&se);
    if (se != GLA_OK) return se;
    return launch_conv_decode(x, slot_idx, n_slots, apply_ln, ln_gamma, ln_beta, ln_eps, w, bias, conv_state, y, N,
                              D, ctl, stream);
}

size_t conv1d_silu_causal_bwd_workspace_bytes(int B, int T, int D, int W)
{
    if (B <= 0 || T <= 0 || W != 4 || D <= 0 || D % 8 != 0 || D > 4096) return 0;
    return conv_bwd_workspace_bytes(B, T, D);
}

gla_status conv1d_silu_causal_bwd(const void* x, int apply_ln, const float* ln_gamma, const float* ln_beta,
                                  float ln_eps, const float* w, const float* bias, const float* conv_state_in,
                                  const void* dy, void* dx, float* dw, float* dbias, float* dln_gamma,
                                  float* dln_beta, float* dconv_state_in, void* ws, size_t ws_bytes, int B, int T,
                                  int D, int W, cudaStream_t stream)
{
    if (B < 0 || T < 0 || D <= 0 || W <= 0) return GLA_ERR_INVALID_ARG;
    if (apply_ln && !(ln_eps > 0.0f && std::isfinite(ln_eps))) return GLA_ERR_INVALID_ARG;
    if (W != 4 || D % 8 != 0 || D > 4096) return GLA_ERR_UNSUPPORTED;
    if (!w || !dw) return GLA_ERR_INVALID_ARG;
    if (B > 65535) return GLA_ERR_UNSUPPORTED;
    if (!aligned16(w) || !aligned16(ln_gamma) || !aligned16(ln_beta) || !aligned16(bias) ||
        !aligned16(conv_state_in) || !aligned16(dw) || !aligned16(dbias) || !aligned16(dln_gamma) ||
        !aligned16(dln_beta) || !aligned16(dconv_state_in) || !aligned16(ws))
        return GLA_ERR_MISALIGNED;
    if (B == 0 || T == 0) {
        // no tokens: every gradient is zero
        cudaError_t e = cudaMemsetAsync(dw, 0, static_cast<size_t>(D) * W * sizeof(float), stream);
        if (e == cudaSuccess && dbias) e = cudaMemsetAsync(dbias, 0, D * sizeof(float), stream);
        if (e == cudaSuccess && dln_gamma) e = cudaMemsetAsync(dln_gamma, 0, D * sizeof(float), stream);
        if (e == cudaSuccess && dln_beta) e = cudaMemsetAsync(dln_beta, 0, D * sizeof(float), stream);
        if (e == cudaSuccess && dconv_state_in && B > 0)
            e = cudaMemsetAsync(dconv_state_in, 0, static_cast<size_t>(B) * (W - 1) * D * sizeof(float), stream);
        return e == cudaSuccess ? GLA_OK : cuda_fail(e);
    }
    if (!x || !dy || !dx) return GLA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dy) || !aligned16(dx)) return GLA_ERR_MISALIGNED;
    if (!ws || ws_bytes < conv_bwd_workspace_bytes(B, T, D)) return GLA_ERR_INVALID_ARG;
    return launch_conv_bwd(x, apply_ln, ln_gamma, ln_beta, ln_eps, w, bias, conv_state_in, dy, dx, dw, dbias,
                           dln_gamma, dln_beta, dconv_state_in, ws, B, T, D, stream);
}

gla_status gla_get_device_status(cudaStream_t stream, int* device_status)
{
    if (!device_status) return GLA_ERR_INVALID_ARG;
    gla_status err;
    int* addr = status_addr_current(&err);
    if (!addr) return err;
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e);
    int h = 0;
    e = cudaMemcpy(&h, addr, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e);
    const int zero = 0;
    e = cudaMemcpy(addr, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e);
    *device_status = h;
    return GLA_OK;
}

gla_status gla_trace_enable(int enable)
{
    std::lock_guard<std::mutex> lk(g_trace_mu);
    for (auto& r : g_trace) {
        cudaEventSynchronize(r.end);
        g_event_pool.push_back(r.start);
        g_event_pool.push_back(r.end);
    }
    g_trace.clear();
    g_trace_on.store(enable != 0);
    return GLA_OK;
}

int gla_trace_summary(const char** names, unsigned long long* launches, double* total_ms,
                      int max_entries)
{
    std::lock_guard<std::mutex> lk(g_trace_mu);
    int n = 0;
    for (auto& r : g_trace) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.end) != cudaSuccess ||
            cudaEventElapsedTime(&ms, r.start, r.end) != cudaSuccess)
            continue;
        int i = 0;
        while (i < n && std::strcmp(names[i], r.name) != 0) ++i;
        if (i == n) {
            if (n >= max_entries) continue;
            names[n] = r.name;
            launches[n] = 0;
            total_ms[n] = 0.0;
            ++n;
        }
        launches[i] += 1;
        total_ms[i] += ms;
    }
    return n;
}

gla_status gla_set_wait_limit_ns(unsigned long long ns)
{
    g_wait_limit_ns.store(ns);
    return GLA_OK;
}

gla_status gla_selftest_wait_timeout(cudaStream_t stream)
{
    gla_status se;
    WaitCtl ctl = wait_ctl_for_current_device(&se);
    if (se != GLA_OK) return se;
    return launch_wait_selftest(ctl, stream);
}

}  // extern "C"
