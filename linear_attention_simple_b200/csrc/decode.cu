// decode.cu -- one-token Simple GLA decode step, in place on an fp32 state.
//
// For every (sequence n, head h):   S <- exp(a) S + k^T v ;  o = scale * q S
// (the fixed per-sequence recurrent state of "AWS serve Laplace 3B di i14 con
// uno stato fisso di 29,5 MB", section "Lo stato di Laplace 3B resta fisso
// durante l'inferenza").  The step is a pure stream over the 96 x 192 fp32
// state: 73,728 bytes read and written once per (sequence, head), about
// 0.5 flop per byte, so it is bound by HBM bandwidth.
//
// Mapping: one CTA of 192 threads per (n, h).  Thread t owns the float4
// column group c4 = t % 48 (columns 4*c4 .. 4*c4+3) and the rows
// r = t / 48 + 4 i, i = 0..23.  A warp's float4 accesses to one row are 512
// contiguous bytes, so every load and store is fully coalesced, and each
// thread keeps 24 independent 16-byte loads in flight before it computes.
// The column sums of q S are reduced over the four row groups in shared
// memory.  A slot outside [0, n_slots) is skipped (nothing read or written)
// and GLA_ERR_INVALID_ARG is recorded in the device status word.
#include <cuda_bf16.h>

#include "gla_internal.h"

namespace gla {
namespace {

constexpr int kThreads = 192;
constexpr int kC4 = kDv / 4;              // 48 float4 column groups
constexpr int kRowGroups = kThreads / kC4; // 4
constexpr int kRowsPerThread = kDk / kRowGroups;  // 24

__global__ void __launch_bounds__(kThreads, 2)
decode_step_kernel(float* __restrict__ state, const int32_t* __restrict__ slot_idx,
                   const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                   const __nv_bfloat16* __restrict__ v, const float* __restrict__ a,
                   float* __restrict__ o, int H, int n_slots, float scale, int* __restrict__ status)
{
    __shared__ float s_q[kDk];
    __shared__ float s_k[kDk];
    __shared__ float4 s_part[kRowGroups][kC4];

    const int unit = blockIdx.x;          // n * H + h
    const int n = unit / H;
    const int h = unit - n * H;
    const int t = threadIdx.x;
    const int c4 = t % kC4;
    const int rg = t / kC4;

    const int64_t slot = slot_idx ? static_cast<int64_t>(slot_idx[n]) : static_cast<int64_t>(n);
    if (slot < 0 || slot >= n_slots) {          // a slot outside the pool: touch nothing
        if (t == 0 && status) atomicCAS(status, 0, static_cast<int>(GLA_ERR_INVALID_ARG));
        return;
    }
    float4* S = reinterpret_cast<float4*>(state + (slot * H + h) * (int64_t)(kDk * kDv));

    // Issue the whole state slice of this thread first (24 x 16 B in flight).
    float4 s[kRowsPerThread];
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) {
        const int r = rg + kRowGroups * i;
        s[i] = __ldcs(S + r * kC4 + c4);
    }

    if (t < kDk) {
        s_q[t] = __bfloat162float(q[(int64_t)unit * kDk + t]);
        s_k[t] = __bfloat162float(k[(int64_t)unit * kDk + t]);
    }
    const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(v + (int64_t)unit * kDv);
    const float2 v01 = __bfloat1622float2(v2[2 * c4]);
    const float2 v23 = __bfloat1622float2(v2[2 * c4 + 1]);
    const float g = expf(a[unit]);
    __syncthreads();

    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) {
        const int r = rg + kRowGroups * i;
        const float kr = s_k[r];
        const float qr = s_q[r];
        float4 x = s[i];
        x.x = fmaf(g, x.x, kr * v01.x);
        x.y = fmaf(g, x.y, kr * v01.y);
        x.z = fmaf(g, x.z, kr * v23.x);
        x.w = fmaf(g, x.w, kr * v23.y);
        __stcs(S + r * kC4 + c4, x);
        acc.x = fmaf(qr, x.x, acc.x);
        acc.y = fmaf(qr, x.y, acc.y);
        acc.z = fmaf(qr, x.z, acc.z);
        acc.w = fmaf(qr, x.w, acc.w);
    }
    s_part[rg][c4] = acc;
    __syncthreads();
    if (t < kC4) {
        float4 r0 = s_part[0][t], r1 = s_part[1][t], r2 = s_part[2][t], r3 = s_part[3][t];
        float4 out;
        out.x = scale * ((r0.x + r1.x) + (r2.x + r3.x));
        out.y = scale * ((r0.y + r1.y) + (r2.y + r3.y));
        out.z = scale * ((r0.z + r1.z) + (r2.z + r3.z));
        out.w = scale * ((r0.w + r1.w) + (r2.w + r3.w));
        reinterpret_cast<float4*>(o + (int64_t)unit * kDv)[t] = out;
    }
}

}  // namespace

gla_status launch_decode(float* state, const int32_t* slot_idx, int n_slots, const void* q, const void* k,
                         const void* v, const float* a, float* o, int N, int H, float scale,
                         int* status, cudaStream_t st)
{
    const int64_t units = static_cast<int64_t>(N) * H;
    if (units == 0) return GLA_OK;
    if (units > 0x7FFFFFFF) return GLA_ERR_UNSUPPORTED;
    trace_begin(st);
    decode_step_kernel<<<static_cast<unsigned>(units), kThreads, 0, st>>>(
        state, slot_idx, static_cast<const __nv_bfloat16*>(q),
        static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), a, o, H,
        n_slots, scale, status);
    trace_end(st, "decode_step_kernel");
    count_launch();
    return check_launch("decode_step_kernel");
}

}  // namespace gla
