// chunk_fwd_noalloc.cu -- the chunked forward for callers that cannot
// allocate device memory.
//
// gla_chunk_fwd asks its caller for a workspace when a sequence is split into
// segments (few batch x heads, long T).  Some callers cannot provide one: a
// host runtime that has reserved all device memory for its own pool up
// front and forbids side allocations, an embedding framework whose plugins
// may not call cudaMalloc, or a latency-critical path that cannot afford the
// implicit device synchronisation of cudaMalloc/cudaFree.  For them
// gla_chunk_fwd_noalloc takes the same arguments minus the workspace and
// uses a fixed scratch array compiled into this library instead.  It calls
// no allocator of any kind.
//
// The scratch is a file-scope __device__ array: every GPU that loads the
// library holds GLA_NOALLOC_SCRATCH_BYTES of it until the process exits, and
// every call on that GPU shares it.  Calls that overlap on the GPU (two
// streams at once) race on it; callers must order them.  Nothing in it
// needs to start at zero: each call writes every scratch element before it
// reads it, so the previous call's leftovers are harmless.
//
// In host code the array's name is only a host-side stand-in, not a device
// address, so the host looks the device address up with
// cudaGetSymbolAddress, with that device current, on the first call made on
// it, and again whenever the device's current context is no longer the one
// the address was looked up in (after cudaDeviceReset, or from another
// context).  The first call on a device (and the first after such a change)
// must therefore come before any stream capture begins.
#include <mutex>

#include "gla_internal.h"

static __device__ __align__(256) unsigned char g_fwd_noalloc_scratch[GLA_NOALLOC_SCRATCH_BYTES];

namespace gla {
namespace {

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
const void* g_scratch_ctx[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device, looked up on
// the first call per device and again when the device's current context
// differs from the one the cached address belongs to.
gla_status scratch_for_current_device(void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return check_launch("cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return GLA_ERR_UNSUPPORTED;
    const void* ctx = current_cu_context();
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev] || g_scratch_ctx[dev] != ctx) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fwd_noalloc_scratch) != cudaSuccess || !p)
            return check_launch("cudaGetSymbolAddress");
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    *out = g_scratch_addr[dev];
    return GLA_OK;
}

}  // namespace
}  // namespace gla

extern "C" gla_status gla_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                            const float* a, const float* s0, void* o,
                                            float* s_final, int B, int T, int H, int dk, int dv,
                                            int64_t ld_qkv, float scale, gla_dtype dt,
                                            cudaStream_t stream)
{
    if (dt == GLA_BF16 && gla_chunk_workspace_bytes(B, T, H, dk, dv, 0) > GLA_NOALLOC_SCRATCH_BYTES)
        return GLA_ERR_UNSUPPORTED;   // this shape needs more scratch than the built-in array
    void* scratch = nullptr;
    const gla_status s = gla::scratch_for_current_device(&scratch);
    if (s != GLA_OK) return s;
    return gla_chunk_fwd(q, k, v, a, s0, o, s_final, scratch, GLA_NOALLOC_SCRATCH_BYTES, B, T, H,
                         dk, dv, ld_qkv, scale, dt, stream);
}
