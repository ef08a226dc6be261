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
// about 25 flop per element.  One CTA owns a contiguous token range of one
// sequence.  x rows reach shared memory through a ring of bulk asynchronous
// copies (cp.async.bulk, one copy of G contiguous rows per stage, completion
// on an mbarrier), so up to kStages x G rows are in flight while the CTA
// works; thread i owns CH consecutive channels (4, or 8 when D > 3072) and
// reads one vector per row from shared memory.  Per stage one block reduction
// gives every row's
// mean and variance: each thread accumulates sums of (x - x0) and (x - x0)^2
// with the row's first element x0 as shift, which keeps the one-pass
// variance free of cancellation for shifted inputs.  The causal window of the
// previous three normalised rows stays in registers; a CTA recomputes the
// LayerNorm of the three rows before its range instead of exchanging them.
// Every wait is bounded.
#include <cuda_bf16.h>

#include "gla_device.cuh"

namespace gla {
namespace {

constexpr int kW = 4;
constexpr int kG = 8;            // rows per stage
constexpr int kStages = 3;
constexpr int kMaxWarps = 32;    // up to 1024 threads

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// SiLU(x) = x * sigmoid(x), with sigmoid(x) = (1 + tanh(x / 2)) / 2 and the
// hardware tanh approximation: one special-function op per element.
__device__ __forceinline__ float silu(float x)
{
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return x * fmaf(0.5f, t, 0.5f);
}

// CH channels (one 2*CH-byte vector) per thread.
template <int CH>
struct Vec;
template <>
struct Vec<4> {
    using T = uint2;
};
template <>
struct Vec<8> {
    using T = uint4;
};

template <int CH>
__device__ __forceinline__ void unpack(const typename Vec<CH>::T& v, float* f)
{
    const uint32_t* w = reinterpret_cast<const uint32_t*>(&v);
#pragma unroll
    for (int i = 0; i < CH / 2; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

template <int CH>
__global__ void __launch_bounds__(CH == 4 ? 768 : 512, 1)
ln_conv_silu_kernel(const __nv_bfloat16* __restrict__ x, int apply_ln,
                    const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
                    const float* __restrict__ w, const float* __restrict__ bias,
                    const float* __restrict__ cs_in, float* __restrict__ cs_out,
                    __nv_bfloat16* __restrict__ y, int T, int D, int tokens_per_cta, WaitCtl ctl)
{
    using V = typename Vec<CH>::T;
    extern __shared__ __align__(16) uint8_t smem[];
    const size_t row_bytes = static_cast<size_t>(D) * 2;
    uint8_t* ring = smem;                                                     // [kStages][kG][D]
    float* red = reinterpret_cast<float*>(smem + kStages * kG * row_bytes);   // [kMaxWarps][kG][2]
    float* stats = red + kMaxWarps * kG * 2;                                  // [kG][2]: mean, rstd
    uint64_t* bars = reinterpret_cast<uint64_t*>(stats + kG * 2);

    const int b = blockIdx.y;
    const int t_begin = blockIdx.x * tokens_per_cta;
    const int t_end = min(T, t_begin + tokens_per_cta);
    if (t_begin >= t_end) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = blockDim.x >> 5;
    const int c0 = tid * CH;
    const bool active = c0 < D;
    const float invD = 1.0f / static_cast<float>(D);

    // positions p0 .. t_end-1 stream through the ring; p0 >= 0
    const int p0 = max(0, t_begin - (kW - 1));
    const int nstages = (t_end - p0 + kG - 1) / kG;
    const __nv_bfloat16* xb = x + static_cast<int64_t>(b) * T * D;
    __nv_bfloat16* yb = y + static_cast<int64_t>(b) * T * D;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(bars + s, 1);
        mbar_init_fence();
    }
    __syncthreads();
    auto issue = [&](int s) {
        const int pos = p0 + s * kG;
        const int rows = min(kG, t_end - pos);
        uint64_t* bar = bars + (s % kStages);
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(rows * row_bytes));
        bulk_load(ring + (s % kStages) * kG * row_bytes, xb + static_cast<int64_t>(pos) * D,
                  static_cast<uint32_t>(rows * row_bytes), bar);
    };
    if (tid == 0)
        for (int s = 0; s < min(kStages, nstages); ++s) issue(s);

    float wr[CH][kW], ga[CH], be[CH], bi[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
        const int ch = active ? c0 + c : 0;
#pragma unroll
        for (int j = 0; j < kW; ++j) wr[c][j] = active ? w[ch * kW + j] : 0.f;
        ga[c] = (gamma && active) ? gamma[ch] : 1.f;
        be[c] = (beta && active) ? beta[ch] : 0.f;
        bi[c] = (bias && active) ? bias[ch] : 0.f;
    }

    // window: the three positions before the stream start p0 (only negative
    // positions matter -- they come from the conv history; the others are
    // shifted out before any output uses them)
    float win[kW - 1][CH];
#pragma unroll
    for (int r = 0; r < kW - 1; ++r) {
        const int p = p0 - (kW - 1) + r;
#pragma unroll
        for (int c = 0; c < CH; ++c)
            win[r][c] = (p < 0 && cs_in && active)
                            ? cs_in[(static_cast<int64_t>(b) * (kW - 1) + (kW - 1) + p) * D + c0 + c]
                            : 0.f;
    }

    bool failed = false;
    for (int s = 0; s < nstages; ++s) {
        const int slot = s % kStages;
        const int pos0 = p0 + s * kG;
        const int rows = min(kG, t_end - pos0);
        if (!mbar_wait(bars + slot, (s / kStages) & 1, ctl)) failed = true;
        if (__syncthreads_or(failed)) break;
        const uint8_t* st = ring + slot * kG * row_bytes;

        if (apply_ln) {
            // per-row shifted sums -> warp partials -> one warp finalises
#pragma unroll
            for (int g = 0; g < kG; ++g) {
                float s1 = 0.f, s2 = 0.f;
                if (g < rows && active) {
                    const float x0 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(st + g * row_bytes));
                    float f[CH];
                    unpack<CH>(*reinterpret_cast<const V*>(st + g * row_bytes + c0 * 2), f);
#pragma unroll
                    for (int c = 0; c < CH; ++c) {
                        const float d = f[c] - x0;
                        s1 += d;
                        s2 = fmaf(d, d, s2);
                    }
                }
                s1 = warp_sum(s1);
                s2 = warp_sum(s2);
                if (lane == 0) {
                    red[(warp * kG + g) * 2] = s1;
                    red[(warp * kG + g) * 2 + 1] = s2;
                }
            }
            __syncthreads();
            if (warp == 0) {
                // lane = 2 g + k: row g, k = 0 sum, k = 1 sum of squares
                float v = 0.f;
                if (lane < 2 * kG)
                    for (int i = 0; i < nwarps; ++i) v += red[i * kG * 2 + lane];
                const float other = __shfl_xor_sync(0xffffffffu, v, 1);
                if (lane < 2 * kG && (lane & 1) == 0) {
                    const int g = lane >> 1;
                    const float x0 = g < rows
                                         ? __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(st + g * row_bytes))
                                         : 0.f;
                    const float m1 = v * invD;
                    const float var = fmaxf(other * invD - m1 * m1, 0.f);
                    stats[2 * g] = x0 + m1;
                    stats[2 * g + 1] = 1.0f / sqrtf(var + eps);
                }
            }
            __syncthreads();
        }

#pragma unroll
        for (int g = 0; g < kG; ++g) {
            if (g >= rows) break;
            const int p = pos0 + g;
            float xn[CH];
            if (active) {
                unpack<CH>(*reinterpret_cast<const V*>(st + g * row_bytes + c0 * 2), xn);
                if (apply_ln) {
                    const float mean = stats[2 * g], rstd = stats[2 * g + 1];
#pragma unroll
                    for (int c = 0; c < CH; ++c) xn[c] = fmaf((xn[c] - mean) * rstd, ga[c], be[c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < CH; ++c) xn[c] = 0.f;
            }
            if (p >= t_begin && active) {
                V out;
                uint32_t* ow = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
                for (int c = 0; c < CH; c += 2) {
                    float r[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        float acc = bi[c + e];
#pragma unroll
                        for (int j = 0; j < kW - 1; ++j) acc = fmaf(wr[c + e][j], win[j][c + e], acc);
                        r[e] = silu(fmaf(wr[c + e][kW - 1], xn[c + e], acc));
                    }
                    ow[c / 2] = pack_bf16(r[0], r[1]);
                }
                *reinterpret_cast<V*>(yb + static_cast<int64_t>(p) * D + c0) = out;
            }
#pragma unroll
            for (int c = 0; c < CH; ++c) {
                win[0][c] = win[1][c];
                win[1][c] = win[2][c];
                win[2][c] = xn[c];
            }
        }
        __syncthreads();                       // everyone is done with this slot
        if (tid == 0 && s + kStages < nstages) issue(s + kStages);
    }

    // The CTA that owns the end of the sequence hands the window on.
    if (!failed && cs_out && t_end == T && active) {
#pragma unroll
        for (int r = 0; r < kW - 1; ++r)
#pragma unroll
            for (int c = 0; c < CH; ++c) cs_out[(static_cast<int64_t>(b) * (kW - 1) + r) * D + c0 + c] = win[r][c];
    }
    if (failed && tid == 0) {
        // drain in-flight copies (bounded) before the shared memory is released
        for (int s = 0; s < kStages; ++s) mbar_wait(bars + s, 0, ctl) || mbar_wait(bars + s, 1, ctl);
    }
}

}  // namespace

gla_status launch_conv(const void* x, int apply_ln, const float* g, const float* b, float eps,
                       const float* w, const float* bias, const float* cs_in, float* cs_out,
                       void* y, int B, int T, int D, cudaStream_t st)
{
    if (B == 0 || T == 0) return GLA_OK;
    gla_status se;
    const WaitCtl ctl = wait_ctl_for_current_device(&se);
    if (se != GLA_OK) return se;
    // 4 channels per thread up to D = 3072 (768 threads), else 8 (512 threads)
    const int ch = D <= 3072 ? 4 : 8;
    const int threads = ((D / ch) + 31) / 32 * 32;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // one CTA per SM and sequence slice; at least a few stages per CTA
    int nx = (sms + B - 1) / B;
    const int max_nx = (T + 4 * kG - 1) / (4 * kG);
    if (nx > max_nx) nx = max_nx;
    if (nx < 1) nx = 1;
    int per = (T + nx - 1) / nx;
    nx = (T + per - 1) / per;
    const size_t smem = static_cast<size_t>(kStages) * kG * D * 2 +
                        (kMaxWarps * kG * 2 + kG * 2) * sizeof(float) + kStages * sizeof(uint64_t);
    auto kernel = ch == 4 ? ln_conv_silu_kernel<4> : ln_conv_silu_kernel<8>;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return check_launch("cudaFuncSetAttribute");
    dim3 grid(nx, B);
    trace_begin(st);
    kernel<<<grid, threads, smem, st>>>(static_cast<const __nv_bfloat16*>(x), apply_ln, g, b, eps, w,
                                        bias, cs_in, cs_out, static_cast<__nv_bfloat16*>(y), T, D, per,
                                        ctl);
    trace_end(st, "ln_conv_silu_kernel");
    count_launch();
    return check_launch("ln_conv_silu_kernel");
}

}  // namespace gla
