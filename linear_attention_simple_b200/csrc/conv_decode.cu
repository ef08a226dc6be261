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
// read and written (12 B each).  One CTA per SM walks the sequences
// blockIdx.x, + gridDim.x, ...: a producer warp brings each sequence's
// history rows and x row into a ring of shared-memory stages with bulk
// asynchronous copies (cp.async.bulk, completion on the stage's mbarrier)
// and refills a stage as soon as every worker has released it, so the loads
// of the next sequences are in flight while the workers finish this one.
// Worker thread i owns channels 8i .. 8i+7 and keeps their conv weights (and
// LayerNorm affine and bias) in registers for the whole launch.  The two
// moments (sums of (x - x0) and (x - x0)^2, shifted by the row's first
// element x0 as the sequence front end does) come from one reduction over
// the workers.  The outputs go out as streaming vector stores.
// A slot outside [0, n_slots) is skipped (nothing read or written) and
// GLA_ERR_INVALID_ARG is recorded in the device status word.  Every wait is
// bounded.
#include <cuda_bf16.h>

#include "gla_device.cuh"
#include "gla_internal.h"

namespace gla {
namespace {

// three stages: measured against two (24.6 us a launch), four (24.7) and
// five (26.6) at 1,280 sequences x D = 3,072 with inputs beyond L2: 23.9 us
constexpr int kMaxStages = 3;
constexpr int kSlotInts = (kMaxStages + 1) & ~1;   // the stages' slots, padded so the partials stay 8-byte aligned
constexpr int kCh = 8;

__device__ __forceinline__ float warp_sum_dec(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void bulk_load_dec(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Barrier over the n worker threads (named barrier 1) that also returns the
// OR of v over them.
__device__ __forceinline__ bool workers_or_dec(bool v, int n)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %2, 0;\n\tbarrier.cta.red.or.pred q, 1, %1, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"(n), "r"(static_cast<uint32_t>(v)) : "memory");
    return r != 0;
}

// SiLU(u) with h = u / 2 (the weights and bias are halved on load):
// u sigmoid(u) = h (1 + tanh h), on the hardware tanh approximation.
__device__ __forceinline__ float silu_of_half_dec(float h)
{
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
    return fmaf(h, t, h);
}

__device__ __forceinline__ void load8(const float* p, float (&v)[8])
{
    const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Stage layout: the slot's three history rows [3][D] fp32, then the x row
// [D] bf16 (14 D bytes, a multiple of 16 since D % 8 == 0).  After the
// stages: full[kMaxStages], free[kMaxStages] mbarriers, the slot of each
// stage (-1: skipped), and the moments' partials [2][warps] by parity.
// AFF: a LayerNorm affine or a conv bias is given (otherwise their
// registers are not needed).
template <bool AFF, int MAXT>
__global__ void __launch_bounds__(MAXT, 1) conv_decode_kernel(
    const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ slot_idx, int apply_ln,
    const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
    const float* __restrict__ w, const float* __restrict__ bias, float* __restrict__ hist,
    __nv_bfloat16* __restrict__ y, int N, int D, int n_slots, int stages, WaitCtl ctl)
{
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t hbytes = 12u * D, xbytes = 2u * D, stage_bytes = hbytes + xbytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(stages) * stage_bytes);
    uint64_t* freeb = full + kMaxStages;
    int* sslot = reinterpret_cast<int*>(freeb + kMaxStages);                 // [kMaxStages]
    float2* red = reinterpret_cast<float2*>(sslot + kSlotInts);               // [2][MAXT / 32]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwork = blockDim.x - 32, nwarps = nwork >> 5;
    const bool producer = warp == nwarps;
    const int c0 = tid * kCh;
    const bool active = !producer && c0 < D;
    const int nseq = blockIdx.x < N ? (N - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

    if (tid == 0) {
        for (int i = 0; i < stages; ++i) {
            mbar_init(full + i, 1);
            mbar_init(freeb + i, nwork);
        }
        mbar_init_fence();
    }
    __syncthreads();

    if (producer) {
        // -------------------------------------------------------- producer
        if (lane == 0) {
            int armed[kMaxStages] = {};
            for (int k = 0; k < nseq; ++k) {
                const int st = k % stages;
                // the stage's previous sequence has been released by every worker
                if (k >= stages && !mbar_wait(freeb + st, ((k - stages) / stages) & 1, ctl)) break;
                const int n = blockIdx.x + k * gridDim.x;
                const int s = slot_idx ? slot_idx[n] : n;
                const bool valid = s >= 0 && s < n_slots;
                sslot[st] = valid ? s : -1;
                uint8_t* base = smem + static_cast<size_t>(st) * stage_bytes;
                if (valid) {
                    mbar_arrive_expect_tx(full + st, stage_bytes);
                    bulk_load_dec(base, hist + static_cast<int64_t>(s) * 3 * D, hbytes, full + st);
                    bulk_load_dec(base + hbytes, x + static_cast<int64_t>(n) * D, xbytes, full + st);
                } else {
                    mbar_arrive(full + st);
                }
                ++armed[st];
            }
            // every copy in flight lands before the shared memory is released
            for (int i = 0; i < stages; ++i)
                if (armed[i]) mbar_wait(full + i, (armed[i] - 1) & 1, ctl);
        }
        return;
    }

    // ------------------------------------------------------------- workers
    float wr[kCh][4], ga[AFF ? kCh : 1], be[AFF ? kCh : 1], bi[AFF ? kCh : 1];
#pragma unroll
    for (int e = 0; e < kCh; ++e) {
        const float4 q = active ? *reinterpret_cast<const float4*>(w + static_cast<int64_t>(c0 + e) * 4)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
        wr[e][0] = 0.5f * q.x;      // halved: see silu_of_half_dec
        wr[e][1] = 0.5f * q.y;
        wr[e][2] = 0.5f * q.z;
        wr[e][3] = 0.5f * q.w;
    }
    if constexpr (AFF) {
        if (active && gamma) load8(gamma + c0, ga);
        else
            for (int e = 0; e < kCh; ++e) ga[e] = 1.f;
        if (active && beta) load8(beta + c0, be);
        else
            for (int e = 0; e < kCh; ++e) be[e] = 0.f;
        if (active && bias) {
            load8(bias + c0, bi);
            for (int e = 0; e < kCh; ++e) bi[e] *= 0.5f;
        } else {
            for (int e = 0; e < kCh; ++e) bi[e] = 0.f;
        }
    }
    const float invD = 1.0f / static_cast<float>(D);

    for (int k = 0; k < nseq; ++k) {
        const int st = k % stages;
        const bool got = mbar_wait(full + st, (k / stages) & 1, ctl);
        const uint8_t* base = smem + static_cast<size_t>(st) * stage_bytes;
        const int s = got ? sslot[st] : -1;
        float v[kCh];
        float s1 = 0.f, s2 = 0.f;
        if (s >= 0 && active) {
            const uint4 xv = *reinterpret_cast<const uint4*>(base + hbytes + c0 * 2);
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                v[2 * i] = bf16_lo(xw[i]);
                v[2 * i + 1] = bf16_hi(xw[i]);
            }
            if (apply_ln) {
                const float x0 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + hbytes));
#pragma unroll
                for (int e = 0; e < kCh; ++e) {
                    const float d = v[e] - x0;
                    s1 += d;
                    s2 = fmaf(d, d, s2);
                }
            }
        } else {
#pragma unroll
            for (int e = 0; e < kCh; ++e) v[e] = 0.f;
        }
        float2* rp = red + (k & 1) * (MAXT / 32);
        if (apply_ln) {
            s1 = warp_sum_dec(s1);
            s2 = warp_sum_dec(s2);
            if (lane == 0) rp[warp] = make_float2(s1, s2);
        }
        // the partials are visible to every worker (the buffer of this parity
        // was last read before the previous sequence's barrier); a timed-out
        // wait stops every worker here
        if (workers_or_dec(!got, nwork)) break;
        if (s < 0) {
            if (tid == 0) record_status(ctl.status, GLA_ERR_INVALID_ARG);
            mbar_arrive(freeb + st);
            continue;
        }
        if (apply_ln) {
            float m1 = 0.f, m2 = 0.f;
            for (int i = 0; i < nwarps; ++i) {
                m1 += rp[i].x;
                m2 += rp[i].y;
            }
            const float x0 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + hbytes));
            const float mu = m1 * invD;
            const float var = fmaxf(m2 * invD - mu * mu, 0.f);
            const float mean = x0 + mu, rstd = rsqrtf(var + eps);
#pragma unroll
            for (int e = 0; e < kCh; ++e) {
                const float t = (v[e] - mean) * rstd;
                if constexpr (AFF) v[e] = fmaf(t, ga[e], be[e]);
                else v[e] = t;
            }
        }
        if (active) {
            const float* hs = reinterpret_cast<const float*>(base);
            float h0[kCh], h1[kCh], h2[kCh];
            load8(hs + c0, h0);
            load8(hs + D + c0, h1);
            load8(hs + 2 * D + c0, h2);
            uint32_t out[4];
#pragma unroll
            for (int e = 0; e < kCh; e += 2) {
                float r[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    float acc = AFF ? bi[AFF ? e + u : 0] : 0.f;
                    acc = fmaf(wr[e + u][0], h0[e + u], acc);
                    acc = fmaf(wr[e + u][1], h1[e + u], acc);
                    acc = fmaf(wr[e + u][2], h2[e + u], acc);
                    r[u] = silu_of_half_dec(fmaf(wr[e + u][3], v[e + u], acc));
                }
                out[e / 2] = pack_bf16(r[0], r[1]);
            }
            const int n = blockIdx.x + k * gridDim.x;
            float* hg = hist + static_cast<int64_t>(s) * 3 * D + c0;
            __stcs(reinterpret_cast<uint4*>(y + static_cast<int64_t>(n) * D + c0),
                   make_uint4(out[0], out[1], out[2], out[3]));
            if ((reinterpret_cast<uintptr_t>(hist) & 31) == 0) {
                // each row's 8 channels as one 32-byte store: whole sectors
                // (c0 and the row stride 4 D are multiples of 32 bytes)
                uint32_t w8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) w8[i] = __float_as_uint(h1[i]);
                st_global_cs_v8(hg, w8);
#pragma unroll
                for (int i = 0; i < 8; ++i) w8[i] = __float_as_uint(h2[i]);
                st_global_cs_v8(hg + D, w8);
#pragma unroll
                for (int i = 0; i < 8; ++i) w8[i] = __float_as_uint(v[i]);
                st_global_cs_v8(hg + 2 * D, w8);
            } else {
                __stcs(reinterpret_cast<float4*>(hg), make_float4(h1[0], h1[1], h1[2], h1[3]));
                __stcs(reinterpret_cast<float4*>(hg + 4), make_float4(h1[4], h1[5], h1[6], h1[7]));
                __stcs(reinterpret_cast<float4*>(hg + D), make_float4(h2[0], h2[1], h2[2], h2[3]));
                __stcs(reinterpret_cast<float4*>(hg + D + 4), make_float4(h2[4], h2[5], h2[6], h2[7]));
                __stcs(reinterpret_cast<float4*>(hg + 2 * D), make_float4(v[0], v[1], v[2], v[3]));
                __stcs(reinterpret_cast<float4*>(hg + 2 * D + 4), make_float4(v[4], v[5], v[6], v[7]));
            }
        }
        mbar_arrive(freeb + st);             // this worker is done with the stage
    }
}

}  // namespace

gla_status launch_conv_decode(const void* x, const int32_t* slot_idx, int n_slots, int apply_ln, const float* g,
                              const float* b, float eps, const float* w, const float* bias, float* hist,
                              void* y, int N, int D, WaitCtl ctl, cudaStream_t st)
{
    // 8 channels per worker thread (384 workers at D = 3,072) and one warp
    // that issues the copies; one CTA per SM (or per sequence, if fewer)
    const int threads = ((D / kCh) + 31) / 32 * 32 + 32;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = N < sms ? N : sms;
    // as many stages (up to 3) as fit in 216 KB beside the barriers
    const size_t stage_bytes = static_cast<size_t>(14) * D;
    const size_t fixed = 2 * kMaxStages * sizeof(uint64_t) + kSlotInts * sizeof(int) + 2 * 32 * sizeof(float2);
    int stages = static_cast<int>((216 * 1024 - fixed) / stage_bytes);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages > N) stages = N > 1 ? N : 1;
    const size_t smem = stages * stage_bytes + fixed;
    const bool aff = g || b || bias;
    auto kernel = threads <= 416 ? (aff ? conv_decode_kernel<true, 416> : conv_decode_kernel<false, 416>)
                                 : (aff ? conv_decode_kernel<true, 544> : conv_decode_kernel<false, 544>);
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
        cudaSuccess)
        return check_launch("cudaFuncSetAttribute");
    trace_begin(st);
    kernel<<<grid, threads, smem, st>>>(static_cast<const __nv_bfloat16*>(x), slot_idx, apply_ln, g, b, eps, w, bias,
                                        hist, static_cast<__nv_bfloat16*>(y), N, D, n_slots, stages, ctl);
    trace_end(st, "conv_decode_kernel");
    count_launch();
    return check_launch("conv_decode_kernel");
}

}  // namespace gla
