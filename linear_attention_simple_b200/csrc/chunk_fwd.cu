// chunk_fwd.cu -- host side of the chunked bf16 forward, plus the segment
// combine kernel.
//
// Work split.  The chunk recurrence is sequential per (batch, head), so with
// B*H units the fused kernel has B*H CTAs.  When B*H alone cannot fill the
// GPU (long prefill: T = 65,536 at B*H = 16), each unit's chunks are cut into
// nseg segments and processed in three steps:
//   1. state-only pass over segments 0..nseg-2 from a zero state: each
//      segment's local end state L_g (fp32) and total log2-decay G_g;
//   2. combine (CUDA cores, elementwise over dk x dv): the true state
//      entering each segment, S_{g+1} = 2^{G_g} S_g + L_g, S_0 = s0;
//   3. fused output pass over all segments from those states.
// This is exact (the state is linear in its inputs); it trades one extra
// read of k and v for nseg-fold parallelism.
#include <cstring>

#define GLA_CHUNK_KERNELS
#include "chunk_state.cuh"

namespace gla {
namespace {

constexpr int kTargetCtas = 148;                 // one wave of B200 SMs
constexpr int64_t kSS = static_cast<int64_t>(kDk) * kDv;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int num_chunks(int T) { return (T + kChunk - 1) / kChunk; }

// States entering every segment's sweep, in place (launch_seg_combine).
// The loads of a batch of segments are issued before the dependent chain that
// uses them.
__global__ void __launch_bounds__(256) seg_combine_kernel(float* __restrict__ states,
                                                          const float* __restrict__ g2,
                                                          const float* __restrict__ s_edge, int nseg,
                                                          int units, int reverse)
{
    constexpr int kBatch = 8;
    const int64_t n4 = kSS / 4;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= n4 * units) return;
    const int64_t unit = idx / n4, e4 = idx - unit * n4;
    float4* st = reinterpret_cast<float4*>(states);
    float4 x = s_edge ? reinterpret_cast<const float4*>(s_edge)[unit * n4 + e4] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = 0; i0 < nseg; i0 += kBatch) {
        float4 l[kBatch];
        float f[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u, g = reverse ? nseg - 1 - i : i;
            // the sweep's last segment only receives its entering state
            if (i < nseg - 1) {
                l[u] = st[(unit * nseg + g) * n4 + e4];
                f[u] = g2[unit * nseg + g];
            }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u, g = reverse ? nseg - 1 - i : i;
            if (i < nseg) {
                st[(unit * nseg + g) * n4 + e4] = x;
                if (i < nseg - 1) {
                    const float e = exp2f(f[u]);
                    x.x = fmaf(e, x.x, l[u].x);
                    x.y = fmaf(e, x.y, l[u].y);
                    x.z = fmaf(e, x.z, l[u].z);
                    x.w = fmaf(e, x.w, l[u].w);
                }
            }
        }
    }
}

// Segmented varlen forward: the state entering every segment of every
// sequence, in place over the scratch slots.  On entry slot(n, s) holds the
// pre-pass end state of segment s from zero (s < nseg_n - 1); on return it
// holds the state entering segment s (s >= 1; segment 0 starts from s0).
// One thread per (sequence, head, float4 of the state), walking the
// sequence's segments in order.
__global__ void __launch_bounds__(256) seg_combine_varlen_kernel(float* __restrict__ states,
                                                                 const float* __restrict__ g2,
                                                                 const float* __restrict__ s0,
                                                                 const int* __restrict__ cu, int N, int H,
                                                                 int total_T, const int* __restrict__ cps_dev)
{
    const int cps = *cps_dev;
    const int64_t n4 = kSS / 4;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= n4 * N * H) return;
    const int64_t u = idx / n4, e4 = idx - u * n4;
    const int n = static_cast<int>(u / H), h = static_cast<int>(u - static_cast<int64_t>(n) * H);
    const int tb = cu[n], Tn = cu[n + 1] - tb;
    if (tb < 0 || Tn < 0 || tb + Tn > total_T) return;   // reported by the pre-pass
    const int nseg = max(1, ((Tn + 127) / 128 + cps - 1) / cps);
    if (nseg == 1) return;
    float4* st = reinterpret_cast<float4*>(states);
    const int64_t slot0 = static_cast<int64_t>(n) + tb / (128 * cps);
    float4 x = s0 ? reinterpret_cast<const float4*>(s0)[u * n4 + e4] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sgm = 0; sgm < nseg - 1; ++sgm) {
        const int64_t at = ((slot0 + sgm) * H + h) * n4 + e4;
        const float4 l = st[at];
        const float f = exp2f(g2[(slot0 + sgm) * H + h]);
        if (sgm > 0) st[at] = x;
        x.x = fmaf(f, x.x, l.x);
        x.y = fmaf(f, x.y, l.y);
        x.z = fmaf(f, x.z, l.z);
        x.w = fmaf(f, x.w, l.w);
    }
    st[((slot0 + nseg - 1) * H + h) * n4 + e4] = x;
}

template <typename K>
gla_status launch_chunk_kernel(K kernel, uint32_t bytes, const char* name, const StateParams& p,
                               dim3 grid, cudaStream_t st, int threads = chunk::kThreads)
{
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return check_launch("cudaFuncSetAttribute");
    trace_begin(st);
    kernel<<<grid, threads, bytes, st>>>(p);
    trace_end(st, name);
    count_launch();
    return check_launch(name);
}

}  // namespace

void chunk_segment_plan(int units, int NC, int* nseg, int* cps)
{
    int n = units >= kTargetCtas / 2 ? 1 : kTargetCtas / units;
    n = n < 1 ? 1 : (n > NC ? NC : n);
    int c = (NC + n - 1) / n;
    *cps = c;
    *nseg = (NC + c - 1) / c;
}

gla_status launch_seg_combine(float* states, const float* g2, const float* s_edge, int nseg, int units,
                              bool reverse, cudaStream_t st)
{
    const int64_t n4 = static_cast<int64_t>(units) * (kSS / 4);
    trace_begin(st);
    seg_combine_kernel<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, st>>>(states, g2, s_edge, nseg, units,
                                                                               reverse ? 1 : 0);
    trace_end(st, "seg_combine_kernel");
    count_launch();
    return check_launch("seg_combine_kernel");
}

gla_status make_token_map(CUtensorMap* m, const void* base, int d, int H, int T, int B,
                          int64_t ld, int box_d, int swizzle, int box_rows)
{
    const uint64_t dims[4] = {static_cast<uint64_t>(d), static_cast<uint64_t>(H),
                              static_cast<uint64_t>(T), static_cast<uint64_t>(B)};
    const uint64_t strides[4] = {2, static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(ld) * 2,
                                 static_cast<uint64_t>(T) * ld * 2};
    const uint32_t box[4] = {static_cast<uint32_t>(box_d), 1, static_cast<uint32_t>(box_rows), 1};
    return make_tmap(m, base, 4, dims, strides, box, 2, swizzle);
}

gla_status make_state_map(CUtensorMap* m, void* base, int64_t nstates, int box_cols, int box_states)
{
    const uint64_t dims[3] = {static_cast<uint64_t>(kDv), static_cast<uint64_t>(kDk),
                              static_cast<uint64_t>(nstates)};
    const uint64_t strides[3] = {2, static_cast<uint64_t>(kDv) * 2,
                                 static_cast<uint64_t>(kDk) * kDv * 2};
    const uint32_t box[3] = {static_cast<uint32_t>(box_cols), static_cast<uint32_t>(kDk),
                             static_cast<uint32_t>(box_states)};
    return make_tmap(m, base, 3, dims, strides, box, 2, box_cols * 2);
}

gla_status launch_state_kernel(bool with_o, bool reverse, const StateParams& p, dim3 grid,
                               cudaStream_t st)
{
    if (with_o && !reverse)
        return p.cu_seqlens ? launch_chunk_kernel(gla_fwd_fused_kernel<true, false>, chunk::FusedSmem::BYTES,
                                                  "chunk_fwd_varlen_kernel", p, grid, st, chunk::kFusedThreads)
                            : launch_chunk_kernel(gla_fwd_fused_kernel<false, false>, chunk::FusedSmem::BYTES,
                                                  "chunk_fwd_fused_kernel", p, grid, st, chunk::kFusedThreads);
    if (!with_o && !reverse)
        return launch_chunk_kernel(gla_state_pass_kernel<false>, chunk::PassSmem::BYTES,
                                   "chunk_state_fwd_kernel", p, grid, st, chunk::kPassThreads);
    if (!with_o && reverse)
        return launch_chunk_kernel(gla_state_pass_kernel<true>, chunk::PassSmem::BYTES,
                                   "chunk_state_rev_kernel", p, grid, st, chunk::kPassThreads);
    // reverse sweep with the output fused in: the backward's D_c and dv
    return launch_chunk_kernel(gla_fwd_fused_kernel<false, true>, chunk::FusedSmem::BYTES, "chunk_rev_fused_kernel",
                               p, grid, st, chunk::kFusedThreads);
}

size_t fwd_workspace_bytes(int B, int T, int H)
{
    const int units = B * H, NC = num_chunks(T);
    int nseg, cps;
    chunk_segment_plan(units, NC, &nseg, &cps);
    if (nseg == 1) return 0;
    return align256(static_cast<size_t>(units) * nseg * kSS * sizeof(float)) +
           align256(static_cast<size_t>(units) * nseg * sizeof(float));
}

// Segment plan of the packed forward: chunks per segment such that the
// (sequence, head, segment) CTAs number about four per SM if the tokens were
// spread evenly (the lengths differ, so small pieces balance the waves; each
// extra segment costs a pre-pass sweep), at least 4 chunks; 0 when no
// sequence can be longer than one segment (total_T within it), i.e. no
// segmenting.
// Segment length of the packed forward: about one wave of CTAs over all the
// chunks (total_T H / (148 x 128) chunks a segment, at least 4).  Measured
// on 16,384 to 36,000 tokens at H = 16 with one or more long sequences,
// this length was within 10% of the best of 4 to 64 chunks (four waves of
// 4-chunk segments: up to 1.8x slower).  0: nothing to split.
int varlen_chunks_per_seg(int total_T, int H)
{
    const int64_t per_cta = (static_cast<int64_t>(total_T) * H + kTargetCtas - 1) / kTargetCtas;
    int cps = static_cast<int>((per_cta + 127) / 128);
    if (cps < 4) cps = 4;
    return static_cast<int64_t>(total_T) <= static_cast<int64_t>(cps) * 128 ? 0 : cps;
}

// Whether to split at all, decided on the device from the sequence lengths:
// the segment length above when the longest sequence has at least twice as
// many chunks, else a length no sequence reaches (one segment each: equal
// lengths gain nothing from the pre-pass).  The kernel also lists the
// (sequence, segment) items of the output pass and of the pre-pass (every
// segment but a sequence's last), so those grids hold only work.  One CTA;
// plan = {chunks per segment, output items, pre-pass items}.
constexpr int kNoSplit = 1 << 20;
constexpr int kPlanThreads = 1024;

// Upper bound of the items of either list: N + (all chunks + N) / cps + 1.
int64_t varlen_max_items(int N, int total_T, int cps)
{
    const int64_t chunks = (static_cast<int64_t>(total_T) + 127) / 128;
    return N + (chunks + N) / cps + 1;
}

__global__ void __launch_bounds__(kPlanThreads) varlen_plan_kernel(const int* __restrict__ cu, int N, int total_T,
                                                                   int cps, int* __restrict__ plan,
                                                                   int2* __restrict__ work_out,
                                                                   int2* __restrict__ work_pre)
{
    __shared__ int s_w[kPlanThreads / 32][2];
    __shared__ int s_cps, s_carry[2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto length = [&](int n) {
        const int tb = cu[n], Tn = cu[n + 1] - tb;
        return (tb >= 0 && Tn >= 0 && tb + Tn <= total_T) ? Tn : -1;   // -1: invalid (one item, reported later)
    };
    int m = 0;
    for (int n = tid; n < N; n += kPlanThreads) m = max(m, length(n));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s_w[warp][0] = m;
    __syncthreads();
    if (tid == 0) {
        int mm = 0;
        for (int w = 0; w < kPlanThreads / 32; ++w) mm = max(mm, s_w[w][0]);
        s_cps = (mm + 127) / 128 >= 2 * cps ? cps : kNoSplit;
        s_carry[0] = s_carry[1] = 0;
    }
    __syncthreads();
    const int c = s_cps;
    for (int base = 0; base < N; base += kPlanThreads) {
        const int n = base + tid;
        int segs = 0;
        if (n < N) {
            const int len = length(n);
            segs = len < 0 ? 1 : max(1, ((len + 127) / 128 + c - 1) / c);
        }
        const int pre = segs > 0 ? segs - 1 : 0;
        // inclusive scans of segs and pre over the block
        int a = segs, q = pre;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int ya = __shfl_up_sync(0xffffffffu, a, o), yq = __shfl_up_sync(0xffffffffu, q, o);
            if (lane >= o) {
                a += ya;
                q += yq;
            }
        }
        if (lane == 31) {
            s_w[warp][0] = a;
            s_w[warp][1] = q;
        }
        __syncthreads();
        int wa = 0, wq = 0;
        for (int w = 0; w < warp; ++w) {
            wa += s_w[w][0];
            wq += s_w[w][1];
        }
        const int off_a = s_carry[0] + wa + a - segs, off_q = s_carry[1] + wq + q - pre;
        for (int sg = 0; sg < segs; ++sg) work_out[off_a + sg] = make_int2(n, sg);
        for (int sg = 0; sg < pre; ++sg) work_pre[off_q + sg] = make_int2(n, sg);
        __syncthreads();
        if (tid == kPlanThreads - 1) {
            s_carry[0] = off_a + segs;
            s_carry[1] = off_q + pre;
        }
        __syncthreads();
    }
    if (tid == 0) {
        plan[0] = c;
        plan[1] = s_carry[0];
        plan[2] = s_carry[1];
    }
}

size_t varlen_workspace_bytes(int N, int total_T, int H)
{
    const int cps = varlen_chunks_per_seg(total_T, H);
    if (cps == 0) return 0;
    const int64_t L = static_cast<int64_t>(cps) * 128;
    const int64_t slots = N + (total_T + L - 1) / L + 1;
    const int64_t items = varlen_max_items(N, total_T, cps);
    return align256(static_cast<size_t>(slots) * H * kSS * sizeof(float)) +
           align256(static_cast<size_t>(slots) * H * sizeof(float)) + 256 +   // + the plan
           2 * align256(static_cast<size_t>(items) * sizeof(int2));            // + the two item lists
}

gla_status run_chunk_fwd_varlen(const ChunkProblem& pr, const int* cu_seqlens, int N, const float* s0, void* o,
                                float* s_final, void* ws, size_t ws_bytes, const WaitCtl& ctl, cudaStream_t st)
{
    // pr.B == 1, pr.T == total tokens; one CTA per (sequence, head, segment)
    const int cps = varlen_chunks_per_seg(pr.T, pr.H);
    const bool segmented = cps > 0 && ws && ws_bytes >= varlen_workspace_bytes(N, pr.T, pr.H);
    StateParams p;
    memset(&p, 0, sizeof(p));
    gla_status s;
    if ((s = make_token_map(&p.tm_q, pr.q, kDk, pr.H, pr.T, 1, pr.ld_qk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&p.tm_u, pr.k, kDk, pr.H, pr.T, 1, pr.ld_qk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&p.tm_y, pr.v, kDv, pr.H, pr.T, 1, pr.ld_v, 64, 128)) != GLA_OK) return s;
    if ((s = make_token_map(&p.tm_o, o, kDv, pr.H, pr.T, 1, static_cast<int64_t>(pr.H) * kDv, 64, 128)) != GLA_OK)
        return s;
    p.a = pr.a;
    p.B = N;
    p.T = pr.T;
    p.H = pr.H;
    p.NC = num_chunks(pr.T);
    p.chunks_per_seg = 1 << 30;
    p.scale = pr.scale;
    p.ctl = ctl;
    p.cu_seqlens = cu_seqlens;
    p.o_direct = o;
    p.s_init = s0;
    p.init_unit_stride = kSS;
    p.s_out = s_final;
    p.out_unit_stride = kSS;
    p.out_last_only = 1;
    if (!segmented) return launch_state_kernel(true, false, p, dim3(1, pr.H, N), st);

    // segments of cps chunks: state-only pre-pass from zero over every
    // segment but each sequence's last, the fold that leaves the state
    // entering each segment in its slot, then the fused pass per segment
    const int64_t L = static_cast<int64_t>(cps) * 128;
    const int64_t slots = N + (pr.T + L - 1) / L + 1;
    float* states = static_cast<float*>(ws);
    float* g2 = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                         align256(static_cast<size_t>(slots) * pr.H * kSS * sizeof(float)));
    int* plan = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(g2) +
                                       align256(static_cast<size_t>(slots) * pr.H * sizeof(float)));
    const int64_t items = varlen_max_items(N, pr.T, cps);
    int2* work_out = reinterpret_cast<int2*>(reinterpret_cast<uint8_t*>(plan) + 256);
    int2* work_pre = reinterpret_cast<int2*>(reinterpret_cast<uint8_t*>(work_out) +
                                             align256(static_cast<size_t>(items) * sizeof(int2)));
    const int* cps_dev = plan;
    trace_begin(st);
    varlen_plan_kernel<<<1, kPlanThreads, 0, st>>>(cu_seqlens, N, pr.T, cps, plan, work_out, work_pre);
    trace_end(st, "varlen_plan_kernel");
    count_launch();
    if ((s = check_launch("varlen_plan_kernel")) != GLA_OK) return s;
    StateParams pre = p;
    pre.chunks_per_seg = cps;
    pre.cps_dev = cps_dev;
    pre.work = work_pre;
    pre.work_count = plan + 2;
    pre.seg_states = states;
    pre.seg_g2 = g2;
    pre.varlen_segs = 1;
    pre.pre_pass = 1;
    pre.s_init = nullptr;
    pre.s_out = states;                 // written at each segment's slot
    pre.out_last_only = 0;
    if ((s = launch_state_kernel(false, false, pre, dim3(static_cast<unsigned>(items), pr.H, 1), st)) != GLA_OK)
        return s;
    {
        const int64_t n = static_cast<int64_t>(N) * pr.H * (kSS / 4);
        trace_begin(st);
        seg_combine_varlen_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(states, g2, s0, cu_seqlens,
                                                                                        N, pr.H, pr.T, cps_dev);
        trace_end(st, "seg_combine_varlen_kernel");
        count_launch();
        if ((s = check_launch("seg_combine_varlen_kernel")) != GLA_OK) return s;
    }
    p.chunks_per_seg = cps;
    p.cps_dev = cps_dev;
    p.work = work_out;
    p.work_count = plan + 1;
    p.seg_states = states;
    p.varlen_segs = 1;
    return launch_state_kernel(true, false, p, dim3(static_cast<unsigned>(items), pr.H, 1), st);
}

gla_status run_chunk_fwd(const ChunkProblem& pr, const float* s0, void* o, float* s_final,
                         void* ws, size_t ws_bytes, const WaitCtl& ctl, cudaStream_t st, void* h_save)
{
    (void)ws_bytes;
    const int units = pr.B * pr.H, NC = num_chunks(pr.T);
    int nseg, cps;
    chunk_segment_plan(units, NC, &nseg, &cps);

    StateParams p;
    memset(&p, 0, sizeof(p));
    gla_status s;
    if ((s = make_token_map(&p.tm_q, pr.q, kDk, pr.H, pr.T, pr.B, pr.ld_qk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&p.tm_u, pr.k, kDk, pr.H, pr.T, pr.B, pr.ld_qk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&p.tm_y, pr.v, kDv, pr.H, pr.T, pr.B, pr.ld_v, 64, 128)) != GLA_OK) return s;
    if ((s = make_token_map(&p.tm_o, o, kDv, pr.H, pr.T, pr.B, static_cast<int64_t>(pr.H) * kDv, 64, 128)) != GLA_OK)
        return s;
    p.a = pr.a;
    p.B = pr.B;
    p.T = pr.T;
    p.H = pr.H;
    p.NC = NC;
    p.chunks_per_seg = cps;
    p.scale = pr.scale;
    p.ctl = ctl;
    p.store_h = 0;
    p.h_save = h_save;
    // the hi plane of each saved state goes out from the kernel's bf16 state
    // copy ([3][96][64] SW128 in shared memory) by TMA
    if (h_save && (s = make_state_map(&p.tm_h, h_save, static_cast<int64_t>(units) * NC * 2, 64)) != GLA_OK)
        return s;

    if (nseg == 1) {
        p.s_init = s0;
        p.init_unit_stride = kSS;
        p.s_out = s_final;
        p.out_unit_stride = kSS;
        p.out_last_only = 1;
        return launch_state_kernel(true, false, p, dim3(1, pr.H, pr.B), st);
    }

    float* states = static_cast<float*>(ws);
    float* g2 = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                         align256(static_cast<size_t>(units) * nseg * kSS * sizeof(float)));
    // 1. local end states of segments 0..nseg-2
    StateParams pre = p;
    pre.h_save = nullptr;
    pre.s_init = nullptr;
    pre.s_out = states;
    pre.out_unit_stride = nseg * kSS;
    pre.out_seg_stride = kSS;
    pre.out_last_only = 0;
    pre.g2_out = g2;
    pre.g2_unit_stride = nseg;
    if ((s = launch_state_kernel(false, false, pre, dim3(nseg - 1, pr.H, pr.B), st)) != GLA_OK) return s;
    // 2. states entering every segment
    if ((s = launch_seg_combine(states, g2, s0, nseg, units, false, st)) != GLA_OK) return s;
    // 3. fused output pass
    p.s_init = states;
    p.init_unit_stride = nseg * kSS;
    p.init_seg_stride = kSS;
    p.s_out = s_final;
    p.out_unit_stride = kSS;
    p.out_seg_stride = 0;
    p.out_last_only = 1;
    return launch_state_kernel(true, false, p, dim3(nseg, pr.H, pr.B), st);
}

}  // namespace gla
