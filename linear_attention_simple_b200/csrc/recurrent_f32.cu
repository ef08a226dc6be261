// recurrent_f32.cu -- fp32 Simple GLA forward on CUDA cores.
//
// The fp32 entry (dtype GLA_F32) serves small problems that want fp32
// inputs and outputs end to end (the tensor-core path takes bf16 operands).
// It evaluates the recurrence token by token, which is exact up to fp32
// rounding and needs no chunk machinery:
//     S_t = exp(a_t) S_{t-1} + k_t^T v_t ,   o_t = scale * q_t S_t
// ("AWS serve Laplace 3B di i14 con uno stato fisso di 29,5 MB", section
// "GLA sostituisce i token conservati con uno stato ricorrente").
//
// One CTA per (b, h) with dv = 192 threads; thread j keeps column j of S
// (dk = 96 values) in registers.  q_t and k_t for a block of 32 tokens are
// staged in shared memory and broadcast to all threads.  Work is
// O(T dk dv) per head on one SM, so this path is meant for small T*B*H.
#include "gla_internal.h"

namespace gla {
namespace {

constexpr int kTok = 32;

__global__ void __launch_bounds__(kDv)
fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
               const float* __restrict__ v, const float* __restrict__ a,
               const float* __restrict__ s0, float* __restrict__ o, float* __restrict__ s_final,
               int T, int H, int64_t ld_qk, int64_t ld_v, float scale)
{
    __shared__ float sq[kTok][kDk];
    __shared__ float sk[kTok][kDk];
    __shared__ float sa[kTok];

    const int bh = blockIdx.x;
    const int b = bh / H;
    const int h = bh - b * H;
    const int j = threadIdx.x;
    const int64_t tok0 = static_cast<int64_t>(b) * T;

    float S[kDk];
#pragma unroll
    for (int d = 0; d < kDk; ++d) S[d] = s0 ? s0[(static_cast<int64_t>(bh) * kDk + d) * kDv + j] : 0.f;

    for (int t0 = 0; t0 < T; t0 += kTok) {
        const int n = min(kTok, T - t0);
        __syncthreads();
        for (int e = j; e < n * kDk; e += kDv) {
            const int tt = e / kDk, d = e - tt * kDk;
            sq[tt][d] = q[(tok0 + t0 + tt) * ld_qk + (int64_t)h * kDk + d];
            sk[tt][d] = k[(tok0 + t0 + tt) * ld_qk + (int64_t)h * kDk + d];
        }
        if (j < n) sa[j] = expf(a[(tok0 + t0 + j) * H + h]);
        __syncthreads();
        for (int tt = 0; tt < n; ++tt) {
            const float vj = v[(tok0 + t0 + tt) * ld_v + (int64_t)h * kDv + j];
            const float g = sa[tt];
            float acc = 0.f;
#pragma unroll
            for (int d = 0; d < kDk; ++d) {
                S[d] = fmaf(g, S[d], sk[tt][d] * vj);
                acc = fmaf(sq[tt][d], S[d], acc);
            }
            o[((tok0 + t0 + tt) * H + h) * kDv + j] = scale * acc;
        }
    }
    if (s_final) {
#pragma unroll
        for (int d = 0; d < kDk; ++d) s_final[(static_cast<int64_t>(bh) * kDk + d) * kDv + j] = S[d];
    }
}

}  // namespace

gla_status launch_fwd_f32(const float* q, const float* k, const float* v, const float* a,
                          const float* s0, float* o, float* s_final, int B, int T, int H,
                          int64_t ld_qk, int64_t ld_v, float scale, const WaitCtl& ctl,
                          cudaStream_t st)
{
    (void)ctl;
    const int64_t units = static_cast<int64_t>(B) * H;
    if (units == 0) return GLA_OK;
    trace_begin(st);
    fwd_f32_kernel<<<static_cast<unsigned>(units), kDv, 0, st>>>(q, k, v, a, s0, o, s_final, T, H,
                                                                 ld_qk, ld_v, scale);
    trace_end(st, "fwd_f32_kernel");
    count_launch();
    return check_launch("fwd_f32_kernel");
}

}  // namespace gla
