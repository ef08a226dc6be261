// chunk_seg.cu -- a sequence cut into consecutive segments (one per rank of a
// sequence-parallel group): the state each segment contributes on its own,
// and the fold that turns those contributions into the state entering (or
// the state gradient leaving) any one segment.
//
// The state is linear in its inputs ("Como i14 llevo Laplace 3B a AWS
// Trainium2", section "Adaptaciones para AWS Trainium2", item 1: the chunked
// form is a regrouping of the one recurrence), so for segment r with total
// log-decay G_r = sum of a_t over its tokens:
//
//   forward   S_end(r) = e^{G_r} S_start(r) + L_r,
//             L_r = sum_t e^{A_end - A_t} k_t^T v_t   (the segment from a zero state)
//   reverse   dS_start(r) = e^{G_r} dS_end(r) + D_r,
//             D_r = sum_t scale e^{A_t - A_start} q_t^T dO_t  (zero gradient at its end)
//
// so the state entering segment r is the fold of (G_j, L_j) over j < r
// starting from S_0, and the gradient at its end the fold of (G_j, D_j) over
// j > r, right to left, starting from dS_T.  Each rank computes its (L_r,
// G_r) (and D_r) with the state-only pass kernel, the ranks exchange them
// (one all_gather of B*H*(dk*dv + 1) floats), and each folds the entries it
// needs with state_fold_kernel before running the ordinary chunked forward
// or backward on its own tokens with that carried state.
//
// Within a rank the segment is itself cut into sub-segments when B*H alone
// cannot fill the GPU (the same plan as the long-prefill forward), and the
// sub-segment results are folded by segment_finish_kernel.
#include <cstring>

#include "chunk_state.cuh"

namespace gla {
namespace {

constexpr int64_t kSS = static_cast<int64_t>(kDk) * kDv;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kFoldBatch = 8;      // entries whose loads are in flight together

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Fold of one unit's sub-segments, in order (forward) or right to left
// (reverse), from a zero state: out = the segment's L (or D); g_out = the
// segment's total natural-log decay.  parts [units][nseg][dk*dv], g2 [units][nseg] (log2).
// The loads of a batch of entries are issued before the dependent chain of
// FMAs that consumes them, so a thread waits once per batch, not per entry.
__global__ void __launch_bounds__(256) segment_finish_kernel(const float* __restrict__ parts,
                                                             const float* __restrict__ g2, int nseg, int units,
                                                             int reverse, float* __restrict__ out,
                                                             float* __restrict__ g_out)
{
    const int64_t n4 = kSS / 4;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= n4 * units) return;
    const int64_t unit = idx / n4, e4 = idx - unit * n4;
    const float4* src = reinterpret_cast<const float4*>(parts);
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    float gsum = 0.f;
    for (int i0 = 0; i0 < nseg; i0 += kFoldBatch) {
        float4 l[kFoldBatch];
        float e[kFoldBatch];
#pragma unroll
        for (int u = 0; u < kFoldBatch; ++u) {
            const int i = i0 + u, g = reverse ? nseg - 1 - i : i;
            if (i < nseg) {
                l[u] = src[(unit * nseg + g) * n4 + e4];
                e[u] = g2[unit * nseg + g];
            }
        }
#pragma unroll
        for (int u = 0; u < kFoldBatch; ++u) {
            if (i0 + u < nseg) {
                const float f = exp2f(e[u]);
                x.x = fmaf(f, x.x, l[u].x);
                x.y = fmaf(f, x.y, l[u].y);
                x.z = fmaf(f, x.z, l[u].z);
                x.w = fmaf(f, x.w, l[u].w);
                gsum += e[u];
            }
        }
    }
    reinterpret_cast<float4*>(out)[unit * n4 + e4] = x;
    if (g_out && e4 == 0) g_out[unit] = gsum * kLn2;
}

// out = fold over entries j of (g[j], s[j]) starting from s_in (zeros when
// null): x <- e^{g[j]} x + s[j], j = 0 .. n-1 (or n-1 .. 0 when reverse).
// s [n][units][dk*dv], g [n][units]; out may alias s_in.  Loads batched as in
// segment_finish_kernel.
__global__ void __launch_bounds__(256) state_fold_kernel(const float* __restrict__ s, const float* __restrict__ g,
                                                         int n, int units, int reverse, const float* s_in,
                                                         float* out)
{
    const int64_t n4 = kSS / 4;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= n4 * units) return;
    const int64_t unit = idx / n4;
    float4 x = s_in ? reinterpret_cast<const float4*>(s_in)[idx] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4* src = reinterpret_cast<const float4*>(s);
    for (int i0 = 0; i0 < n; i0 += kFoldBatch) {
        float4 l[kFoldBatch];
        float e[kFoldBatch];
#pragma unroll
        for (int u = 0; u < kFoldBatch; ++u) {
            const int i = i0 + u, j = reverse ? n - 1 - i : i;
            if (i < n) {
                l[u] = src[static_cast<int64_t>(j) * units * n4 + idx];
                e[u] = g[static_cast<int64_t>(j) * units + unit];
            }
        }
#pragma unroll
        for (int u = 0; u < kFoldBatch; ++u) {
            if (i0 + u < n) {
                const float f = expf(e[u]);
                x.x = fmaf(f, x.x, l[u].x);
                x.y = fmaf(f, x.y, l[u].y);
                x.z = fmaf(f, x.z, l[u].z);
                x.w = fmaf(f, x.w, l[u].w);
            }
        }
    }
    reinterpret_cast<float4*>(out)[idx] = x;
}

unsigned fold_blocks(int units) { return static_cast<unsigned>((units * (kSS / 4) + 255) / 256); }

}  // namespace

size_t segment_workspace_bytes(int B, int T, int H)
{
    const int units = B * H, NC = (T + kChunk - 1) / kChunk;
    int nseg, cps;
    chunk_segment_plan(units, NC, &nseg, &cps);
    return align256(static_cast<size_t>(units) * nseg * kSS * sizeof(float)) +
           align256(static_cast<size_t>(units) * nseg * sizeof(float));
}

gla_status run_segment_state(const void* u, const void* y, const float* a, int B, int T, int H, int64_t ld_u,
                             int64_t ld_y, float scale, bool reverse, float* s_seg, float* g_seg, void* ws,
                             const WaitCtl& ctl, cudaStream_t st)
{
    const int units = B * H, NC = (T + kChunk - 1) / kChunk;
    int nseg, cps;
    chunk_segment_plan(units, NC, &nseg, &cps);
    float* parts = static_cast<float*>(ws);
    float* g2 = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                         align256(static_cast<size_t>(units) * nseg * kSS * sizeof(float)));
    StateParams p;
    memset(&p, 0, sizeof(p));
    gla_status s;
    if ((s = make_token_map(&p.tm_u, u, kDk, H, T, B, ld_u, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&p.tm_y, y, kDv, H, T, B, ld_y, 64, 128)) != GLA_OK) return s;
    p.a = a;
    p.B = B;
    p.T = T;
    p.H = H;
    p.NC = NC;
    p.chunks_per_seg = cps;
    p.scale = scale;
    p.ctl = ctl;
    p.s_init = nullptr;
    p.s_out = parts;
    p.out_unit_stride = nseg * kSS;
    p.out_seg_stride = kSS;
    p.out_last_only = 0;
    p.g2_out = g2;
    p.g2_unit_stride = nseg;
    if ((s = launch_state_kernel(false, reverse, p, dim3(nseg, H, B), st)) != GLA_OK) return s;
    trace_begin(st);
    segment_finish_kernel<<<fold_blocks(units), 256, 0, st>>>(parts, g2, nseg, units, reverse ? 1 : 0, s_seg,
                                                              g_seg);
    trace_end(st, "segment_finish_kernel");
    count_launch();
    return check_launch("segment_finish_kernel");
}

gla_status launch_state_fold(const float* s, const float* g, int n, int units, int reverse, const float* s_in,
                             float* out, cudaStream_t st)
{
    trace_begin(st);
    state_fold_kernel<<<fold_blocks(units), 256, 0, st>>>(s, g, n, units, reverse, s_in, out);
    trace_end(st, "state_fold_kernel");
    count_launch();
    return check_launch("state_fold_kernel");
}

}  // namespace gla
