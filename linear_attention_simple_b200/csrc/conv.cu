// conv.cu -- fused LayerNorm -> causal depthwise conv (width 4) -> SiLU.
//
// The per-layer front end of "Como i14 llevo Laplace 3B a AWS Trainium2",
// section "Diseno esencial de Laplace 3B": each residual vector x_t passes
// LayerNorm and a causal depthwise Conv1d of width k = 4 with SiLU (a 4-gram
// summary before the mixer).
//
//   xn[t]  = (x[t] - mean_t) / sqrt(var_t + eps) * gamma + beta   (over D)
//   y[t,c] = SiLU( sum_{j<4} w[c,j] xn[t-3+j, c] + bias[c] )
//
// HBM-bound: x is read once and y written once (2 x 2 bytes per element),
// about 20 flop per element.  One CTA owns a contiguous token range of one
// sequence and all D channels; thread i owns channels 8i .. 8i+7 (one 16-byte
// bf16 vector per token), so every row access is fully coalesced.  Tokens
// are processed in groups of G: the per-token mean and centred variance are
// block reductions (two-pass, so shifted inputs keep their precision), and
// the causal window of the previous three normalised tokens stays in
// registers.  A CTA recomputes the LayerNorm of the three tokens before its
// range (the halo) instead of exchanging them.
#include <cuda_bf16.h>

#include "gla_internal.h"

namespace gla {
namespace {

constexpr int kW = 4;
constexpr int kG = 4;            // tokens per group
constexpr int kMaxWarps = 16;   // up to 512 threads, D <= 4096

struct alignas(16) Bf16x8 {
    __nv_bfloat162 h[4];
};

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__global__ void __launch_bounds__(512, 1)
ln_conv_silu_kernel(const __nv_bfloat16* __restrict__ x, int apply_ln,
                    const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
                    const float* __restrict__ w, const float* __restrict__ bias,
                    const float* __restrict__ cs_in, float* __restrict__ cs_out,
                    __nv_bfloat16* __restrict__ y, int T, int D, int tokens_per_cta)
{
    __shared__ float red[2][kMaxWarps][kG];

    const int b = blockIdx.y;
    const int t_begin = blockIdx.x * tokens_per_cta;
    const int t_end = min(T, t_begin + tokens_per_cta);
    if (t_begin >= t_end) return;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int nwarps = blockDim.x >> 5;
    const int c0 = tid * 8;
    const bool active = c0 < D;
    const float invD = 1.0f / static_cast<float>(D);

    // Per-channel affine parameters and bias live in shared memory (read per
    // token); the conv taps stay in registers.
    extern __shared__ float s_par[];            // [3][D]: gamma, beta, bias
    for (int c = tid; c < D; c += blockDim.x) {
        s_par[c] = gamma ? gamma[c] : 1.f;
        s_par[D + c] = beta ? beta[c] : 0.f;
        s_par[2 * D + c] = bias ? bias[c] : 0.f;
    }
    float wr[8][kW];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const int ch = active ? c0 + c : 0;
#pragma unroll
        for (int j = 0; j < kW; ++j) wr[c][j] = active ? w[ch * kW + j] : 0.f;
    }
    __syncthreads();

    float win[kW - 1][8];   // xn of the three previous positions, oldest first
#pragma unroll
    for (int r = 0; r < kW - 1; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) win[r][c] = 0.f;

    const __nv_bfloat16* xb = x + static_cast<int64_t>(b) * T * D;
    __nv_bfloat16* yb = y + static_cast<int64_t>(b) * T * D;

    int stage = 0;
    for (int p0 = t_begin - (kW - 1); p0 < t_end; p0 += kG) {
        Bf16x8 xr[kG];
        float part[kG];
#pragma unroll
        for (int g = 0; g < kG; ++g) {
            const int p = p0 + g;
            if (active && p >= 0 && p < t_end) {
                xr[g] = *reinterpret_cast<const Bf16x8*>(xb + (int64_t)p * D + c0);
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) xr[g].h[c] = __floats2bfloat162_rn(0.f, 0.f);
            }
        }
#define XV(g, c) ((c) & 1 ? __high2float(xr[g].h[(c) >> 1]) : __low2float(xr[g].h[(c) >> 1]))
        float mean[kG], rstd[kG];
        if (apply_ln) {
            // pass 1: mean
#pragma unroll
            for (int g = 0; g < kG; ++g) {
                float s = 0.f;
#pragma unroll
                for (int c = 0; c < 8; ++c) s += XV(g, c);
                part[g] = warp_sum(s);
            }
            if (lane == 0)
#pragma unroll
                for (int g = 0; g < kG; ++g) red[stage][warp][g] = part[g];
            __syncthreads();
#pragma unroll
            for (int g = 0; g < kG; ++g) {
                float s = 0.f;
                for (int i = 0; i < nwarps; ++i) s += red[stage][i][g];
                mean[g] = s * invD;
            }
            stage ^= 1;
            // pass 2: centred variance
#pragma unroll
            for (int g = 0; g < kG; ++g) {
                float s = 0.f;
                if (active) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float d = XV(g, c) - mean[g];
                        s = fmaf(d, d, s);
                    }
                }
                part[g] = warp_sum(s);
            }
            if (lane == 0)
#pragma unroll
                for (int g = 0; g < kG; ++g) red[stage][warp][g] = part[g];
            __syncthreads();
#pragma unroll
            for (int g = 0; g < kG; ++g) {
                float s = 0.f;
                for (int i = 0; i < nwarps; ++i) s += red[stage][i][g];
                rstd[g] = 1.0f / sqrtf(s * invD + eps);
            }
            stage ^= 1;
        }

        // normalise, convolve, activate, store -- token by token
#pragma unroll
        for (int g = 0; g < kG; ++g) {
            const int p = p0 + g;
            if (p >= t_end) break;
            float xn[8];
            if (p < 0) {
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    xn[c] = (cs_in && active)
                                ? cs_in[((int64_t)b * (kW - 1) + (kW - 1) + p) * D + c0 + c]
                                : 0.f;
            } else if (apply_ln) {
                const float* ga = s_par + (active ? c0 : 0);
                const float* be = ga + D;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    xn[c] = fmaf((XV(g, c) - mean[g]) * rstd[g], ga[c], be[c]);
            } else {
#pragma unroll
                for (int c = 0; c < 8; ++c) xn[c] = XV(g, c);
            }
            if (p >= t_begin && active) {
                const float* bi = s_par + 2 * D + c0;
                Bf16x8 out;
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    float r[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        float acc = bi[c + e];
#pragma unroll
                        for (int j = 0; j < kW - 1; ++j) acc = fmaf(wr[c + e][j], win[j][c + e], acc);
                        acc = fmaf(wr[c + e][kW - 1], xn[c + e], acc);
                        r[e] = acc / (1.0f + expf(-acc));
                    }
                    out.h[c / 2] = __floats2bfloat162_rn(r[0], r[1]);
                }
                *reinterpret_cast<Bf16x8*>(yb + (int64_t)p * D + c0) = out;
            }
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                win[0][c] = win[1][c];
                win[1][c] = win[2][c];
                win[2][c] = xn[c];
            }
        }
    }

#undef XV
    // The CTA that owns the end of the sequence hands the window on.
    if (cs_out && t_end == T && active) {
#pragma unroll
        for (int r = 0; r < kW - 1; ++r)
#pragma unroll
            for (int c = 0; c < 8; ++c) cs_out[((int64_t)b * (kW - 1) + r) * D + c0 + c] = win[r][c];
    }
}

}  // namespace

gla_status launch_conv(const void* x, int apply_ln, const float* g, const float* b, float eps,
                       const float* w, const float* bias, const float* cs_in, float* cs_out,
                       void* y, int B, int T, int D, cudaStream_t st)
{
    if (B == 0 || T == 0) return GLA_OK;
    int threads = ((D / 8) + 31) / 32 * 32;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int target = 2 * sms;
    int nx = (target + B - 1) / B;
    const int max_nx = (T + 31) / 32;
    if (nx > max_nx) nx = max_nx;
    if (nx < 1) nx = 1;
    int per = (T + nx - 1) / nx;
    per = (per + kG - 1) / kG * kG;
    nx = (T + per - 1) / per;
    dim3 grid(nx, B);
    const size_t smem = static_cast<size_t>(3) * D * sizeof(float);
    trace_begin(st);
    ln_conv_silu_kernel<<<grid, threads, smem, st>>>(
        static_cast<const __nv_bfloat16*>(x), apply_ln, g, b, eps, w, bias, cs_in, cs_out,
        static_cast<__nv_bfloat16*>(y), T, D, per);
    trace_end(st, "ln_conv_silu_kernel");
    count_launch();
    return check_launch("ln_conv_silu_kernel");
}

}  // namespace gla
