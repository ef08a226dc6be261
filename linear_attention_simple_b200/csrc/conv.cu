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
// about 12 instructions per element.  One CTA owns a contiguous token range
// of one sequence.  x rows reach shared memory through a ring of bulk
// asynchronous copies (cp.async.bulk, one copy of G contiguous rows per
// stage, completion on an mbarrier) issued by a producer warp, which refills
// a slot as soon as every worker has released it (a per-slot "free"
// mbarrier), so the workers meet at one block barrier per stage.  Per stage,
// warp g computes the LayerNorm moments of row g over all D channels (sums
// of (x - x0) and (x - x0)^2 with the row's first element x0 as shift, which
// keeps the one-pass variance free of cancellation for shifted inputs, then
// one warp reduction); then every worker thread, owning 8 consecutive
// channels, normalises, convolves and writes its channels of the G rows.  The causal window of the previous three
// normalised rows stays in registers; a CTA recomputes the LayerNorm of the
// three rows before its range instead of exchanging them.  Every wait is
// bounded.
#include <cuda_bf16.h>

#include "gla_device.cuh"

namespace gla {
namespace {

constexpr int kW = 4;
constexpr int kG = 8;            // rows per stage
constexpr int kMaxStages = 4;

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

// SiLU(u) = u sigmoid(u) = h + h tanh(h) with h = u / 2 (sigmoid(u) =
// (1 + tanh(u / 2)) / 2), on the hardware tanh approximation.  The kernel
// folds the 1/2 into the conv weights and bias, so it convolves straight to
// h: one special-function op and one FMA per element.
__device__ __forceinline__ float tanh_approx(float h)
{
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
    return t;
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

// OR of v over the n worker threads (named barrier 1; the producer warp is
// not among them).
__device__ __forceinline__ bool workers_or(bool v, int n)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %2, 0;\n\tbarrier.cta.red.or.pred q, 1, %1, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"(n), "r"(static_cast<uint32_t>(v)) : "memory");
    return r != 0;
}

// LayerNorm moments of one row of D bf16 values by one warp: (mean, rstd).
// The sums run on fp32 pairs (even and odd channels), added at the end.
__device__ __forceinline__ float2 row_moments(const uint8_t* row, int D, float eps, int lane)
{
    const float x0 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(row));
    const f2 x02 = f2_splat(x0);
    f2 s1 = f2_splat(0.f), s2 = f2_splat(0.f);
    for (int c = lane * 8; c < D; c += 256) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + c * 2);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const f2 d = f2_sub(f2_from_bf16x2(w[i]), x02);
            s1 = f2_add(s1, d);
            s2 = f2_fma(d, d, s2);
        }
    }
    const float2 a = f2_get(s1), b = f2_get(s2);
    const float t1 = warp_sum(a.x + a.y), t2 = warp_sum(b.x + b.y);
    const float invD = 1.0f / static_cast<float>(D);
    const float m1 = t1 * invD;
    const float var = fmaxf(t2 * invD - m1 * m1, 0.f);
    return make_float2(x0 + m1, 1.0f / sqrtf(var + eps));
}

// Block = D/8 worker threads (8 channels each, rounded up to whole warps) +
// one producer warp, at most MAXT threads: 13 warps up to D = 3,072 (four a
// sub-partition, so 128 registers a thread), 17 up to 4,096.  AFF: a
// LayerNorm affine or a conv bias is given (otherwise their registers are
// not needed).
constexpr int CH = 8;
// LN: the LayerNorm is applied (a template parameter, so that the row loop
// holds no test of it).
template <bool AFF, bool LN, int MAXT>
__global__ void __launch_bounds__(MAXT, 1)
ln_conv_silu_kernel(const __nv_bfloat16* __restrict__ x,
                    const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
                    const float* __restrict__ w, const float* __restrict__ bias,
                    const float* __restrict__ cs_in, float* __restrict__ cs_out,
                    __nv_bfloat16* __restrict__ y, int T, int D, int tokens_per_cta, int stages, WaitCtl ctl)
{
    using V = typename Vec<CH>::T;
    extern __shared__ __align__(16) uint8_t smem[];
    const size_t row_bytes = static_cast<size_t>(D) * 2;
    uint8_t* ring = smem;                                                        // [stages][kG][D]
    float2* stats = reinterpret_cast<float2*>(smem + stages * kG * row_bytes);   // [kMaxStages][kG]
    uint64_t* full = reinterpret_cast<uint64_t*>(stats + kMaxStages * kG);       // [kMaxStages]
    uint64_t* freeb = full + kMaxStages;                                         // [kMaxStages]

    const int b = blockIdx.y;
    const int t_begin = blockIdx.x * tokens_per_cta;
    const int t_end = min(T, t_begin + tokens_per_cta);
    if (t_begin >= t_end) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwork = blockDim.x - 32;                 // worker threads
    const int nwarps = nwork >> 5;
    const bool producer = warp == nwarps;
    const int c0 = tid * CH;
    const bool active = !producer && c0 < D;

    // positions p0 .. t_end-1 stream through the ring; p0 >= 0
    const int p0 = max(0, t_begin - (kW - 1));
    const int nstages = (t_end - p0 + kG - 1) / kG;
    const __nv_bfloat16* xb = x + static_cast<int64_t>(b) * T * D;
    __nv_bfloat16* yb = y + static_cast<int64_t>(b) * T * D;

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(freeb + s, nwork);
        }
        mbar_init_fence();
    }
    __syncthreads();

    if (producer) {
        // -------------------------------------------------------- producer
        if (lane == 0) {
            int issued[kMaxStages] = {0, 0, 0, 0};
            for (int s = 0; s < nstages; ++s) {
                const int slot = s % stages;
                // the slot's previous stage (s - stages) has been released by every worker
                if (s >= stages && !mbar_wait(freeb + slot, ((s - stages) / stages) & 1, ctl)) break;
                const int pos = p0 + s * kG;
                const int rows = min(kG, t_end - pos);
                mbar_arrive_expect_tx(full + slot, static_cast<uint32_t>(rows * row_bytes));
                bulk_load(ring + slot * kG * row_bytes, xb + static_cast<int64_t>(pos) * D,
                          static_cast<uint32_t>(rows * row_bytes), full + slot);
                ++issued[slot];
            }
            // every copy in flight lands before the shared memory is released
            for (int i = 0; i < stages; ++i)
                if (issued[i]) mbar_wait(full + i, (issued[i] - 1) & 1, ctl);
        }
        return;
    }

    // ----------------------------------------------------------- workers
    // channels in pairs (c0 + 2i, c0 + 2i + 1): every product below is one
    // fp32-pair instruction
    constexpr int NP = CH / 2;
    f2 wr[NP][kW], ga[AFF ? NP : 1], be[AFF ? NP : 1], bi[AFF ? NP : 1];
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        const int ch = active ? c0 + 2 * i : 0;
#pragma unroll
        for (int j = 0; j < kW; ++j)   // halved: see tanh_approx
            wr[i][j] = active ? f2_make(0.5f * w[ch * kW + j], 0.5f * w[(ch + 1) * kW + j]) : f2_splat(0.f);
        if constexpr (AFF) {
            ga[i] = (gamma && active) ? f2_make(gamma[ch], gamma[ch + 1]) : f2_splat(1.f);
            be[i] = (beta && active) ? f2_make(beta[ch], beta[ch + 1]) : f2_splat(0.f);
            bi[i] = (bias && active) ? f2_make(0.5f * bias[ch], 0.5f * bias[ch + 1]) : f2_splat(0.f);
        }
    }

    // window: the three positions before the stream start p0 (only negative
    // positions matter -- they come from the conv history; the others are
    // shifted out before any output uses them)
    f2 win[kW - 1][NP];
#pragma unroll
    for (int r = 0; r < kW - 1; ++r) {
        const int p = p0 - (kW - 1) + r;
        const float* src = cs_in + (static_cast<int64_t>(b) * (kW - 1) + (kW - 1) + p) * D + c0;
#pragma unroll
        for (int i = 0; i < NP; ++i)
            win[r][i] = (p < 0 && cs_in && active) ? f2_make(src[2 * i], src[2 * i + 1]) : f2_splat(0.f);
    }

    bool failed = false;
    for (int s = 0; s < nstages; ++s) {
        const int slot = s % stages;
        const int pos0 = p0 + s * kG;
        const int rows = min(kG, t_end - pos0);
        if (!failed && !mbar_wait(full + slot, (s / stages) & 1, ctl)) failed = true;
        const uint8_t* st = ring + slot * kG * row_bytes;
        float2* sst = stats + slot * kG;
        if (LN && !failed)
            for (int g = warp; g < rows; g += nwarps) {
                const float2 m = row_moments(st + g * row_bytes, D, eps, lane);
                if (lane == 0) sst[g] = m;
            }
        // moments visible to every worker; a timed-out wait stops the CTA
        if (workers_or(failed, nwork)) {
            failed = true;
            break;
        }

        // one row: normalise, convolve with the window, SiLU, write y (when the
        // row is an output of this CTA), shift the window
        auto do_row = [&](int g, int p, bool out) {
            f2 xn[NP];
            if (active) {
                const V xv = *reinterpret_cast<const V*>(st + g * row_bytes + c0 * 2);
                const uint32_t* xw = reinterpret_cast<const uint32_t*>(&xv);
#pragma unroll
                for (int i = 0; i < NP; ++i) xn[i] = f2_from_bf16x2(xw[i]);
                if constexpr (LN) {
                    const float2 m = sst[g];
                    if constexpr (AFF) {
                        const f2 mu = f2_splat(m.x), rs = f2_splat(m.y);
#pragma unroll
                        for (int i = 0; i < NP; ++i) xn[i] = f2_fma(f2_mul(f2_sub(xn[i], mu), rs), ga[i], be[i]);
                    } else {
                        const f2 rs = f2_splat(m.y), sh = f2_splat(-m.x * m.y);
#pragma unroll
                        for (int i = 0; i < NP; ++i) xn[i] = f2_fma(xn[i], rs, sh);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < NP; ++i) xn[i] = f2_splat(0.f);
            }
            if (out && GLA_DCHECK(p < T && c0 + CH <= D, ctl.status)) {
                V o;
                uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    f2 acc = AFF ? bi[AFF ? i : 0] : f2_splat(0.f);
#pragma unroll
                    for (int j = 0; j < kW - 1; ++j) acc = f2_fma(wr[i][j], win[j][i], acc);
                    const f2 h = f2_fma(wr[i][kW - 1], xn[i], acc);
                    const float2 hh = f2_get(h);
                    ow[i] = f2_to_bf16x2(f2_fma(h, f2_make(tanh_approx(hh.x), tanh_approx(hh.y)), h));
                }
                __stcs(reinterpret_cast<V*>(yb + static_cast<int64_t>(p) * D + c0), o);
            }
#pragma unroll
            for (int i = 0; i < NP; ++i) {
                win[0][i] = win[1][i];
                win[1][i] = win[2][i];
                win[2][i] = xn[i];
            }
        };
        if (rows == kG && pos0 >= t_begin && active) {
            // an interior stage: eight output rows and no branch between them,
            // so the rows' dependency chains interleave (and, unrolled, the
            // window rotation becomes register renaming)
#pragma unroll(MAXT <= 416 ? kG : 2)
            for (int g = 0; g < kG; ++g) do_row(g, pos0 + g, true);
        } else {
#pragma unroll 1
            for (int g = 0; g < rows; ++g) do_row(g, pos0 + g, pos0 + g >= t_begin && active);
        }
        mbar_arrive(freeb + slot);             // this worker is done with the slot
    }

    // The CTA that owns the end of the sequence hands the window on.
    if (!failed && cs_out && t_end == T && active) {
#pragma unroll
        for (int r = 0; r < kW - 1; ++r)
#pragma unroll
            for (int i = 0; i < NP; ++i) {
                const float2 v = f2_get(win[r][i]);
                float* dst = cs_out + (static_cast<int64_t>(b) * (kW - 1) + r) * D + c0 + 2 * i;
                dst[0] = v.x;
                dst[1] = v.y;
            }
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
    // 8 channels per worker thread (384 workers at D = 3,072); one more warp
    // issues the copies
    const int threads = ((D / CH) + 31) / 32 * 32 + 32;
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
    // as many ring stages (up to 4) as fit beside the moments and barriers
    const size_t stage_bytes = static_cast<size_t>(kG) * D * 2;
    const size_t fixed = kMaxStages * kG * sizeof(float2) + 2 * kMaxStages * sizeof(uint64_t);
    int stages = static_cast<int>((200 * 1024 - fixed) / stage_bytes);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) stages = 2;
    const size_t smem = stages * stage_bytes + fixed;
    const bool aff = g || b || bias;
    using KFn = decltype(&ln_conv_silu_kernel<true, true, 416>);
    static const KFn forms[2][2][2] = {
        {{ln_conv_silu_kernel<false, false, 416>, ln_conv_silu_kernel<false, false, 544>},
         {ln_conv_silu_kernel<false, true, 416>, ln_conv_silu_kernel<false, true, 544>}},
        {{ln_conv_silu_kernel<true, false, 416>, ln_conv_silu_kernel<true, false, 544>},
         {ln_conv_silu_kernel<true, true, 416>, ln_conv_silu_kernel<true, true, 544>}}};
    auto kernel = forms[aff][apply_ln != 0][threads > 416];
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return check_launch("cudaFuncSetAttribute");
    dim3 grid(nx, B);
    trace_begin(st);
    kernel<<<grid, threads, smem, st>>>(static_cast<const __nv_bfloat16*>(x), g, b, eps, w,
                                        bias, cs_in, cs_out, static_cast<__nv_bfloat16*>(y), T, D, per,
                                        stages, ctl);
    trace_end(st, "ln_conv_silu_kernel");
    count_launch();
    return check_launch("ln_conv_silu_kernel");
}

}  // namespace gla
