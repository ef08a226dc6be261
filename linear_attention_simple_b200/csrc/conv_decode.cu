// conv_decode.cu -- the per-layer front end at decode time: one token per
// sequence, the conv history of each sequence in a pool of slots.
//
// The front end of "Como i14 llevo Laplace 3B a AWS Trainium2", section
// "Diseno esencial de Laplace 3B" (LayerNorm, causal depthwise Conv1d of
// width 4, SiLU), taken one token at a time the way serving runs it; the
// history lives in a slot pool like the recurrent state ("AWS serve Laplace
// 3B di i14 con uno stato fisso di 29,5 MB", section "Lo stato di Laplace 3B
// resta fisso durante l'inferenza": the wrapper links the recurrent state to
// the serving memory pool).  For sequence n with slot s:
//
//   xn      = LayerNorm(x[n])                       (over D, fp32)
//   y[n,c]  = SiLU( w[c,0] h[s,0,c] + w[c,1] h[s,1,c] + w[c,2] h[s,2,c]
//                   + w[c,3] xn[c] + bias[c] )
//   h[s]   <- (h[s,1], h[s,2], xn)                  (in place)
//
// HBM-bound: per sequence x and y (2 B per channel each) and the history
// read and written (12 B each); the weights stay in L2 across sequences.
// One CTA per sequence, thread i owns channels 8i .. 8i+7: one 16-byte
// vector of x and y, two of each history row.  The history rows are loaded
// with x, before the LayerNorm, so their latency overlaps the moments (the
// weights and bias, L2-resident, come after); the two moments (sums of
// (x - x0) and (x - x0)^2, shifted by the row's first element x0 as the
// sequence front end does) come from one block reduction.
// A slot outside [0, n_slots) is skipped (nothing read or written) and
// GLA_ERR_INVALID_ARG is recorded in the device status word.
#include <cuda_bf16.h>

#include "gla_device.cuh"
#include "gla_internal.h"

namespace gla {
namespace {

constexpr int kMaxThreads = 512;   // D <= 4096

__device__ __forceinline__ float warp_sum_dec(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sums of a and b over the block; every thread gets both.
__device__ __forceinline__ float2 block_sum2(float a, float b, float2* red)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = (blockDim.x + 31) >> 5;
    a = warp_sum_dec(a);
    b = warp_sum_dec(b);
    if (lane == 0) red[warp] = make_float2(a, b);
    __syncthreads();
    float2 s = make_float2(0.f, 0.f);
    for (int i = 0; i < nw; ++i) {
        s.x += red[i].x;
        s.y += red[i].y;
    }
    return s;
}

// SiLU(x) = x sigmoid(x) with sigmoid(x) = (1 + tanh(x / 2)) / 2 on the
// hardware tanh approximation.
__device__ __forceinline__ float silu_dec(float x)
{
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return x * fmaf(0.5f, t, 0.5f);
}

__device__ __forceinline__ void load8(const float* p, float (&v)[8])
{
    const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// At most 80 registers, so that two CTAs of 384 threads (D = 3,072) share
// an SM.
__global__ void __maxnreg__(80) conv_decode_kernel(
    const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ slot_idx, int apply_ln,
    const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
    const float* __restrict__ w, const float* __restrict__ bias, float* __restrict__ hist,
    __nv_bfloat16* __restrict__ y, int D, int n_slots, int* __restrict__ status)
{
    __shared__ float2 red[kMaxThreads / 32];
    const int n = blockIdx.x, c0 = threadIdx.x * 8;
    const int s = slot_idx ? slot_idx[n] : n;
    if (s < 0 || s >= n_slots) {                // a slot outside the pool: touch nothing
        if (threadIdx.x == 0) record_status(status, GLA_ERR_INVALID_ARG);
        return;
    }
    // the loads from HBM first: x and the three history rows
    const uint4 xv = __ldcs(reinterpret_cast<const uint4*>(x + static_cast<int64_t>(n) * D + c0));
    float* hs = hist + static_cast<int64_t>(s) * 3 * D + c0;
    float4 hv[3][2];
#pragma unroll
    for (int r = 0; r < 3; ++r) {
        hv[r][0] = __ldcs(reinterpret_cast<const float4*>(hs + r * D));
        hv[r][1] = __ldcs(reinterpret_cast<const float4*>(hs + r * D + 4));
    }
    const float x0 = __bfloat162float(x[static_cast<int64_t>(n) * D]);

    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
    float v[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = bf16_lo(xw[i]);
        v[2 * i + 1] = bf16_hi(xw[i]);
    }
    if (apply_ln) {
        float s1 = 0.f, s2 = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float d = v[e] - x0;
            s1 += d;
            s2 = fmaf(d, d, s2);
        }
        const float2 m = block_sum2(s1, s2, red);
        const float m1 = m.x / D;
        const float var = fmaxf(m.y / D - m1 * m1, 0.f);
        const float mean = x0 + m1, rstd = rsqrtf(var + eps);
        float g[8], bt[8];
        if (gamma) load8(gamma + c0, g);
        if (beta) load8(beta + c0, bt);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float t = (v[e] - mean) * rstd;
            if (gamma) t *= g[e];
            if (beta) t += bt[e];
            v[e] = t;
        }
    }

    const float h0[8] = {hv[0][0].x, hv[0][0].y, hv[0][0].z, hv[0][0].w, hv[0][1].x, hv[0][1].y, hv[0][1].z, hv[0][1].w};
    const float h1[8] = {hv[1][0].x, hv[1][0].y, hv[1][0].z, hv[1][0].w, hv[1][1].x, hv[1][1].y, hv[1][1].z, hv[1][1].w};
    const float h2[8] = {hv[2][0].x, hv[2][0].y, hv[2][0].z, hv[2][0].w, hv[2][1].x, hv[2][1].y, hv[2][1].z, hv[2][1].w};
    // the weights and the bias are L2-resident across sequences
    float bi[8];
    if (bias) load8(bias + c0, bi);
    uint32_t out[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
        float r[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const float4 wc = *reinterpret_cast<const float4*>(w + static_cast<int64_t>(c0 + e + u) * 4);
            float acc = bias ? bi[e + u] : 0.f;
            acc = fmaf(wc.x, h0[e + u], acc);
            acc = fmaf(wc.y, h1[e + u], acc);
            acc = fmaf(wc.z, h2[e + u], acc);
            acc = fmaf(wc.w, v[e + u], acc);
            r[u] = silu_dec(acc);
        }
        out[e / 2] = pack_bf16(r[0], r[1]);
    }
    __stcs(reinterpret_cast<uint4*>(y + static_cast<int64_t>(n) * D + c0), make_uint4(out[0], out[1], out[2], out[3]));
    __stcs(reinterpret_cast<float4*>(hs), hv[1][0]);
    __stcs(reinterpret_cast<float4*>(hs + 4), hv[1][1]);
    __stcs(reinterpret_cast<float4*>(hs + D), hv[2][0]);
    __stcs(reinterpret_cast<float4*>(hs + D + 4), hv[2][1]);
    __stcs(reinterpret_cast<float4*>(hs + 2 * D), make_float4(v[0], v[1], v[2], v[3]));
    __stcs(reinterpret_cast<float4*>(hs + 2 * D + 4), make_float4(v[4], v[5], v[6], v[7]));
}

}  // namespace

gla_status launch_conv_decode(const void* x, const int32_t* slot_idx, int n_slots, int apply_ln, const float* g,
                              const float* b, float eps, const float* w, const float* bias, float* hist,
                              void* y, int N, int D, int* status, cudaStream_t st)
{
    trace_begin(st);
    conv_decode_kernel<<<N, D / 8, 0, st>>>(static_cast<const __nv_bfloat16*>(x), slot_idx, apply_ln, g, b, eps,
                                            w, bias, hist, static_cast<__nv_bfloat16*>(y), D, n_slots, status);
    trace_end(st, "conv_decode_kernel");
    count_launch();
    return check_launch("conv_decode_kernel");
}

}  // namespace gla
