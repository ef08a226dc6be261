// conv_bwd.cu -- backward of the per-layer front end (LayerNorm -> causal
// depthwise conv of width 4 -> SiLU; "Como i14 llevo Laplace 3B a AWS
// Trainium2", section "Diseno esencial de Laplace 3B"), for training the
// mixer block.  With xn the conv inputs (history rows first), xhat the
// normalised rows, u the conv output before SiLU and s = sigmoid(u):
//
//   du[t,c]   = dy[t,c] * s (1 + u (1 - s))
//   dxn[p,c]  = sum_j w[c,j] du[p+3-j, c]             (rows p < 0: conv history)
//   dx[t]     = rstd_t (g - mean(g) - xhat mean(g xhat)),  g = dxn gamma
//   dw[c,j]   = sum_t du[t,c] xn[t-3+j, c]   dbias = sum du
//   dgamma    = sum dxn xhat                  dbeta = sum dxn
//
// One pass over the rows.  A cluster of CL CTAs (CL = 2 up to D = 3,072, 4
// above) owns a contiguous token range of one sequence, and CTA r of the
// cluster owns the r-th block of channels (whole 8-channel units).  Every
// per-channel quantity -- the conv weights, the windows of the last three
// rows' xn, xhat and du, the sums of dw, dbias, dgamma, dbeta -- stays in the
// registers of the thread that owns the channel (4 channels a thread, or 8
// for 2,048 < D <= 3,072) for the whole range.  A producer warp streams the rows of x and dy through a
// ring of shared-memory stages of kG rows (bulk asynchronous copies, one per
// row and tensor, completion on the stage's mbarrier).
//
// The LayerNorm needs two reductions over all D channels of a row: the
// moments of x (before the row can be normalised) and the sums of g and
// g xhat (before its dx can be written).  Per stage, each CTA reduces its
// channels' part of both (a 16-value butterfly in each warp, then the warps
// in a fixed order) and pushes the 24 numbers to every CTA of the cluster
// with st.async into their shared memory, completing bytes on their
// exchange mbarrier.  The exchange sent at stage s carries the g sums of the
// rows that stage finished (q = p - 3) and the moments of the rows two
// stages ahead; it is combined at stage s + 1, after that stage's rows are
// done, so the cluster round trip hides under a stage of work.  The rows'
// g and xhat wait in shared memory (fp32) for their dx until then.  The
// moments are taken about the first channel of CTA 0 (the row's first
// element, as the forward does), each CTA's shifted sums being moved to that
// shift before they are added.
//
// The channel sums go out as per-(range, CTA) partials [B * nx][7][D] that
// conv_bwd_reduce_kernel adds in a fixed order, so every output is
// deterministic.  The SiLU derivative runs on h = u / 2 with the hardware
// tanh (sigmoid(u) = (1 + tanh h) / 2); the kernel carries du2 = 2 du, so
// the conv weights are halved and dw, dbias halved at the end.  Every wait
// is bounded; on a timeout the CTAs record GLA_ERR_TIMEOUT and leave
// through the same final cluster barrier.
#include <cuda_bf16.h>

#include <algorithm>
#include <type_traits>

#include "gla_device.cuh"
#include "gla_internal.h"

namespace gla {
namespace {

constexpr int kW = 4;
constexpr int kG = 4;           // rows per stage
constexpr int kRing = 8;        // ring stages: s, s+1, s+2 (moments) and five in flight
// 8-channel workers hold half a row a CTA: four stages (s .. s+2 and one in
// flight) keep the ring and the g / xhat rows within shared memory; a stage
// takes microseconds, far longer than its load
constexpr int ring_stages(int np) { return np == 4 ? 4 : kRing; }
constexpr int kXch = 4;         // exchange buffers (a CTA runs at most two exchanges ahead)
constexpr int kMsg = 24;        // floats per CTA per exchange
constexpr int kStRing = 32;     // rows of LayerNorm statistics kept
constexpr int kParts = 7;       // dw (4 taps), dbias, dgamma, dbeta
constexpr int kMaxSlices = 128; // token ranges per sequence
constexpr int kMinRows = 64;    // rows per range at least

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

__device__ __forceinline__ void bulk_load_bwd(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Barrier over the n worker threads (named barrier 1) returning the OR of v.
__device__ __forceinline__ bool workers_or_bwd(bool v, int n)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %2, 0;\n\tbarrier.cta.red.or.pred q, 1, %1, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"(n), "r"(static_cast<uint32_t>(v)) : "memory");
    return r != 0;
}

__device__ __forceinline__ float tanh_hw(float h)
{
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
    return t;
}

// Sums over the 32 lanes of a warp of each of v[0..15], by halving: at each
// step a lane keeps one half of its values and adds the partner lane's copy
// of that half.  Lanes 2k and 2k+1 end with the total of value k (bits 4..1
// of the lane number are the value index).
__device__ __forceinline__ float warp_reduce16(float (&v)[16], int lane)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const bool up = lane & 16;
        const float send = up ? v[i] : v[i + 8], keep = up ? v[i + 8] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool up = lane & 8;
        const float send = up ? v[i] : v[i + 4], keep = up ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool up = lane & 4;
        const float send = up ? v[i] : v[i + 2], keep = up ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    {
        const bool up = lane & 2;
        const float send = up ? v[0] : v[1], keep = up ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

struct BwdArgs {
    const __nv_bfloat16* x;
    const __nv_bfloat16* dy;
    const float* gamma;
    const float* beta;
    const float* w;
    const float* bias;
    const float* cs_in;
    __nv_bfloat16* dx;
    float* part;       // [B * nx][7][D]
    float* dcs;        // [B][3][D] or null
    int T, D, nx, rps, upc, apply_ln;
    float eps;
    WaitCtl ctl;
};

// Shared-memory map (bytes), the same in every CTA of the cluster.
struct BwdSmem {
    uint32_t segb, ring, fin, red, xbuf, st, tot, bars, total;
    // np: fp32 pairs (channel pairs) a worker owns
    __host__ __device__ BwdSmem(int upc, int nwork, int np)
    {
        segb = 16u * upc;                                  // one row of a CTA's channels
        ring = 0;
        fin = ring + ring_stages(np) * 2 * kG * segb;     // [2][kG][nwork][4 np] fp32: g, xhat
        red = fin + 2 * kG * nwork * 16 * np;              // [2][warps][16] by stage parity
        xbuf = red + 2 * (nwork / 32) * 64;                // [kXch][CL max 4][kMsg]
        st = xbuf + kXch * 4 * kMsg * 4;                   // [kStRing] (mean, rstd)
        tot = st + kStRing * 8;                            // [2][kG] (mean g, mean g xhat) by stage parity
        bars = tot + 2 * kG * 8;                           // full[kRing], free[kRing], xbar[kXch]
        total = bars + (2 * kRing + kXch) * 8;
    }
};

// LN: the LayerNorm is applied (its statistics and row sums are exchanged).
// FULL: every worker thread of every CTA owns channels (the 8-channel units
// split evenly over the cluster into whole warps), so no thread is idle.
// Both are template parameters: their tests would otherwise be branches in
// the row loop (measured 9% of the kernel's time for the LayerNorm flag).
// NP: fp32 pairs a worker owns, 2 (4 channels: two workers an 8-channel
// unit) or 4 (the whole unit).
template <bool AFF, bool LN, bool FULL, int CL, int NP, int MAXT>
__global__ void __launch_bounds__(MAXT, 1) ln_conv_silu_bwd_kernel(const __grid_constant__ BwdArgs a)
{
    static_assert(CL >= 2 && CL <= 4, "the rows' channels are split over 2 to 4 CTAs");
    static_assert(NP == 2 || NP == 4, "a worker owns 4 or 8 channels");
    static_assert(kMsg == 16 + 2 * kG, "a message: 16 sums, then 2 kG first elements");
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwork = blockDim.x - 32, nwarps = nwork >> 5;
    const BwdSmem L(a.upc, nwork, NP);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* freeb = full + kRing;
    uint64_t* xbar = freeb + kRing;
    float* red = reinterpret_cast<float*>(smem + L.red);
    float* xbuf = reinterpret_cast<float*>(smem + L.xbuf);
    float2* st_ring = reinterpret_cast<float2*>(smem + L.st);
    float2* tot = reinterpret_cast<float2*>(smem + L.tot);
    const WaitCtl ctl = a.ctl;

    const int T = a.T, D = a.D, P = D / 8;
    const int rank = static_cast<int>(cluster_ctarank());
    const int ubase = (rank * P) / CL, nu = ((rank + 1) * P) / CL - ubase;
    const int slice = blockIdx.x / CL, b = blockIdx.y;
    const int t_b = slice * a.rps, t_e = min(T, t_b + a.rps);
    const int p_s = t_b - 3;                                   // stream rows p_s .. t_e + 2
    const int S = (t_e - t_b + 6 + kG - 1) / kG;
    const int p_load = min(T, t_e + 3);                        // rows [max(0, p_s), p_load) are loaded
    constexpr bool ln = LN;
    const int64_t row0 = static_cast<int64_t>(b) * T;

    if (tid == 0) {
        for (int i = 0; i < kRing; ++i) {
            mbar_init(full + i, 1);
            mbar_init(freeb + i, nwork);
        }
        for (int i = 0; i < kXch; ++i) mbar_init(xbar + i, 1);
        mbar_init_fence();
    }
    // every CTA's barriers exist before any CTA of the cluster sends to them
    cluster_sync_all();

    constexpr int RING = ring_stages(NP);
    auto ring_x = [&](int stage, int g) { return smem + L.ring + ((stage % RING) * 2 * kG + g) * L.segb; };
    auto ring_dy = [&](int stage, int g) { return smem + L.ring + ((stage % RING) * 2 * kG + kG + g) * L.segb; };

    if (warp == nwarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint32_t nbytes = 16u * nu;
            int armed[RING] = {};
            for (int s = 0; s < S; ++s) {
                const int slot = s % RING;
                if (s >= RING && !mbar_wait(freeb + slot, ((s - RING) / RING) & 1, ctl)) break;
                uint32_t bytes = 0;
#pragma unroll
                for (int g = 0; g < kG; ++g) {
                    const int p = p_s + s * kG + g;
                    if (nu > 0 && p >= 0 && p < p_load) bytes += (p >= t_b ? 2 : 1) * nbytes;
                }
                if (bytes == 0) {
                    mbar_arrive(full + slot);
                } else {
                    mbar_arrive_expect_tx(full + slot, bytes);
#pragma unroll
                    for (int g = 0; g < kG; ++g) {
                        const int p = p_s + s * kG + g;
                        if (nu > 0 && p >= 0 && p < p_load) {
                            const int64_t off = (row0 + p) * D + 8 * ubase;
                            bulk_load_bwd(ring_x(s, g), a.x + off, nbytes, full + slot);
                            if (p >= t_b) bulk_load_bwd(ring_dy(s, g), a.dy + off, nbytes, full + slot);
                        }
                    }
                }
                ++armed[slot];
            }
            for (int i = 0; i < RING; ++i)
                if (armed[i]) mbar_wait(full + i, (armed[i] - 1) & 1, ctl);
        }
    } else {
        // ------------------------------------------------------------- workers
        const int u = NP == 4 ? tid : tid >> 1, half = NP == 4 ? 0 : tid & 1;
        const bool active = FULL || u < nu;
        const int c = 8 * (ubase + u) + 4 * half;                // this thread's channels c .. c + 2 NP - 1
        const uint32_t seg_off = 16u * u + 8u * half;            // their bytes in a ring row

        f2 wr[NP][kW], ga[AFF ? NP : 1], be[AFF ? NP : 1], bi[AFF ? NP : 1];
#pragma unroll
        for (int i = 0; i < NP; ++i) {
            const int ch = active ? c + 2 * i : 0;
#pragma unroll
            for (int j = 0; j < kW; ++j)
                wr[i][j] = active ? f2_make(0.5f * a.w[ch * kW + j], 0.5f * a.w[(ch + 1) * kW + j]) : f2_splat(0.f);
            if constexpr (AFF) {
                ga[i] = (a.gamma && active) ? f2_make(a.gamma[ch], a.gamma[ch + 1]) : f2_splat(1.f);
                be[i] = (a.beta && active) ? f2_make(a.beta[ch], a.beta[ch + 1]) : f2_splat(0.f);
                bi[i] = (a.bias && active) ? f2_make(0.5f * a.bias[ch], 0.5f * a.bias[ch + 1]) : f2_splat(0.f);
            }
        }
        const f2 zero = f2_splat(0.f), one = f2_splat(1.f);
        f2 wxn[3][NP], wxh[3][NP], wdu[3][NP];     // windows: rows p-3, p-2, p-1
        f2 dw[kW][NP], db[NP], dg[NP], dbe[NP];
#pragma unroll
        for (int i = 0; i < NP; ++i) {
#pragma unroll
            for (int r = 0; r < 3; ++r) wxn[r][i] = wxh[r][i] = wdu[r][i] = zero;
#pragma unroll
            for (int j = 0; j < kW; ++j) dw[j][i] = zero;
            db[i] = dg[i] = dbe[i] = zero;
        }
        float gs[2 * kG] = {};                   // this thread's g and g xhat sums of the stage's output rows
        const float invD = 1.0f / static_cast<float>(D);
        float* fin = reinterpret_cast<float*>(smem + L.fin);
        auto fin_at = [&](int par, int g) { return fin + ((par * kG + g) * nwork + tid) * (4 * NP); };
        // this thread's channels of a ring row as NP fp32 pairs
        auto load_pairs = [&](const uint8_t* ring_row, f2 (&v)[NP]) {
            if constexpr (NP == 2) {
                const uint2 w = *reinterpret_cast<const uint2*>(ring_row + seg_off);
                v[0] = f2_from_bf16x2(w.x);
                v[1] = f2_from_bf16x2(w.y);
            } else {
                const uint4 w = *reinterpret_cast<const uint4*>(ring_row + seg_off);
                v[0] = f2_from_bf16x2(w.x);
                v[1] = f2_from_bf16x2(w.y);
                v[2] = f2_from_bf16x2(w.z);
                v[3] = f2_from_bf16x2(w.w);
            }
        };
        // NP pairs to global memory as bf16 (8 or 16 bytes) or fp32 (16 bytes a 2 pairs)
        auto store_bf16 = [&](__nv_bfloat16* dst, const f2 (&v)[NP]) {
            if constexpr (NP == 2)
                *reinterpret_cast<uint2*>(dst) = make_uint2(f2_to_bf16x2(v[0]), f2_to_bf16x2(v[1]));
            else
                *reinterpret_cast<uint4*>(dst) = make_uint4(f2_to_bf16x2(v[0]), f2_to_bf16x2(v[1]),
                                                            f2_to_bf16x2(v[2]), f2_to_bf16x2(v[3]));
        };
        auto store_f32 = [&](float* dst, const f2 (&v)[NP]) {
#pragma unroll
            for (int i = 0; i < NP; i += 2) {
                const float2 v0 = f2_get(v[i]), v1 = f2_get(v[i + 1]);
                *reinterpret_cast<float4*>(dst + 2 * i) = make_float4(v0.x, v0.y, v1.x, v1.y);
            }
        };

        // moments of this CTA's channels of stream row p about the row's
        // first element here: (sum d, sum d^2) for this thread's channels
        auto moments = [&](auto inner_tag, int stage, int g, int p, float& m1, float& m2) {
            constexpr bool INNER = decltype(inner_tag)::value;   // p is a loaded row
            m1 = m2 = 0.f;
            if (active && (INNER || (p >= 0 && p < p_load))) {
                const uint8_t* row = ring_x(stage, g);
                const f2 x0 = f2_splat(__bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(row)));
                f2 xv[NP];
                load_pairs(row, xv);
                f2 a1 = f2_sub(xv[0], x0), a2 = f2_mul(a1, a1);
#pragma unroll
                for (int i = 1; i < NP; ++i) {
                    const f2 d = f2_sub(xv[i], x0);
                    a1 = f2_add(a1, d);
                    a2 = f2_fma(d, d, a2);
                }
                const float2 s1 = f2_get(a1), s2 = f2_get(a2);
                m1 = s1.x + s1.y;
                m2 = s2.x + s2.y;
            }
        };
        // the row's first element of this CTA's channels (0 without channels)
        auto first_x = [&](int stage, int g, int p) {
            return (nu > 0 && p >= 0 && p < p_load)
                       ? __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(ring_x(stage, g)))
                       : 0.f;
        };
        auto xch_addr = [&](int e, int from, int k) { return xbuf + ((e % kXch) * 4 + from) * kMsg + k; };
        // value k of this CTA's message e, into every CTA of the cluster
        auto push = [&](int e, int k, float val) {
            const uint32_t la = smem_u32(xch_addr(e, rank, k)), lb = smem_u32(xbar + e % kXch);
#pragma unroll
            for (int r = 0; r < CL; ++r) st_async_f32(mapa_shared(la, r), val, mapa_shared(lb, r));
        };
        // LayerNorm statistics of a row from the CTAs' shifted sums
        auto combine_stats = [&](int e, int i_s1, int i_s2, int i_x0) {
            const float A = *xch_addr(e, 0, i_x0);
            float S1 = 0.f, S2 = 0.f;
            for (int r = 0; r < CL; ++r) {
                const float n = static_cast<float>(8 * (((r + 1) * P) / CL - (r * P) / CL));
                const float s1 = *xch_addr(e, r, i_s1), s2 = *xch_addr(e, r, i_s2);
                const float dlt = *xch_addr(e, r, i_x0) - A;
                S1 += fmaf(n, dlt, s1);
                S2 += fmaf(n * dlt, dlt, fmaf(2.f * dlt, s1, s2));
            }
            const float m1 = S1 * invD;
            const float var = fmaxf(S2 * invD - m1 * m1, 0.f);
            return make_float2(A + m1, 1.0f / sqrtf(var + a.eps));
        };
        // exchange e: armed once by this CTA for the bytes of all CL messages
        auto arm = [&](int e) {
            if (tid == 0) mbar_arrive_expect_tx(xbar + e % kXch, CL * kMsg * 4);
        };
        auto wait_x = [&](int e) { return mbar_wait_cluster(xbar + e % kXch, (e / kXch) & 1, ctl); };

        bool failed = false;

        // one stream row: xn, xhat, du (when p is a du row of this range),
        // the sums, and for q = p - 3 its dxn (g and xhat to fin, or dx).
        // INNER: a row with 0 <= p - 3, t_b <= p - 3 and p < min(T, t_e), so
        // that no range check is needed.
        auto do_row = [&](auto inner_tag, int stage, int g, int p) {
            constexpr bool INNER = decltype(inner_tag)::value;
            f2 xn[NP], xh[NP], du[NP];
            if (!INNER && p < 0) {
                const bool hv = active && a.cs_in;
                const float* src = a.cs_in + (static_cast<int64_t>(b) * 3 + p + 3) * D + c;
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    xn[i] = hv ? f2_make(src[2 * i], src[2 * i + 1]) : zero;
                    xh[i] = zero;
                }
            } else if ((INNER || p < T) && active) {
                load_pairs(ring_x(stage, g), xn);
                if (ln) {
                    const float2 m = st_ring[(p - p_s) & (kStRing - 1)];
                    if constexpr (AFF) {
                        const f2 mu = f2_splat(m.x), rs = f2_splat(m.y);
#pragma unroll
                        for (int i = 0; i < NP; ++i) {
                            xh[i] = f2_mul(f2_sub(xn[i], mu), rs);
                            xn[i] = f2_fma(xh[i], ga[i], be[i]);
                        }
                    } else {
                        const f2 rs = f2_splat(m.y), sh = f2_splat(-m.x * m.y);
#pragma unroll
                        for (int i = 0; i < NP; ++i) xh[i] = xn[i] = f2_fma(xn[i], rs, sh);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < NP; ++i) xh[i] = xn[i];
                }
            } else {
#pragma unroll
                for (int i = 0; i < NP; ++i) xn[i] = xh[i] = zero;
            }
            if ((INNER || (p >= t_b && p < T)) && active) {
                f2 dyv[NP];
                load_pairs(ring_dy(stage, g), dyv);
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    f2 acc = AFF ? bi[AFF ? i : 0] : zero;
#pragma unroll
                    for (int j = 0; j < kW - 1; ++j) acc = f2_fma(wr[i][j], wxn[j][i], acc);
                    const f2 h = f2_fma(wr[i][kW - 1], xn[i], acc);
                    const float2 hh = f2_get(h);
                    const f2 t = f2_make(tanh_hw(hh.x), tanh_hw(hh.y));
                    // du2 = 2 du = dy (1 + t) (1 + h (1 - t))
                    du[i] = f2_mul(f2_mul(dyv[i], f2_add(one, t)), f2_fma(h, f2_sub(one, t), one));
                }
                if (INNER || p < t_e) {
#pragma unroll
                    for (int i = 0; i < NP; ++i) {
#pragma unroll
                        for (int j = 0; j < kW - 1; ++j) dw[j][i] = f2_fma(du[i], wxn[j][i], dw[j][i]);
                        dw[kW - 1][i] = f2_fma(du[i], xn[i], dw[kW - 1][i]);
                        db[i] = f2_add(db[i], du[i]);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < NP; ++i) du[i] = zero;
            }
            const int q = p - 3;
            const bool out = INNER || (q >= t_b && q < t_e);
            const bool hist = !INNER && t_b == 0 && q < 0 && q >= -3 && a.dcs;
            if (out || hist) {
                f2 dxn[NP];
#pragma unroll
                for (int i = 0; i < NP; ++i)
                    dxn[i] = f2_fma(wr[i][0], du[i],
                                    f2_fma(wr[i][1], wdu[2][i], f2_fma(wr[i][2], wdu[1][i], f2_mul(wr[i][3], wdu[0][i]))));
                if (hist) {
                    if (active) {
                        store_f32(a.dcs + (static_cast<int64_t>(b) * 3 + q + 3) * D + c, dxn);
                    }
                } else if (ln) {
                    f2 gg[NP];
#pragma unroll
                    for (int i = 0; i < NP; ++i) {
                        gg[i] = AFF ? f2_mul(dxn[i], ga[AFF ? i : 0]) : dxn[i];
                        dg[i] = f2_fma(dxn[i], wxh[0][i], dg[i]);
                        dbe[i] = f2_add(dbe[i], dxn[i]);
                    }
                    f2 sg = gg[0], sgx = f2_mul(gg[0], wxh[0][0]);
#pragma unroll
                    for (int i = 1; i < NP; ++i) {
                        sg = f2_add(sg, gg[i]);
                        sgx = f2_fma(gg[i], wxh[0][i], sgx);
                    }
                    const float2 s1 = f2_get(sg), s2 = f2_get(sgx);
                    gs[g] += s1.x + s1.y;
                    gs[kG + g] += s2.x + s2.y;
                    float* fp = fin_at(stage & 1, g);
                    store_f32(fp, gg);
                    store_f32(fp + 2 * NP, wxh[0]);
                } else if (active) {
                    store_bf16(a.dx + (row0 + q) * D + c, dxn);
                }
            }
#pragma unroll
            for (int i = 0; i < NP; ++i) {
                wxn[0][i] = wxn[1][i];
                wxn[1][i] = wxn[2][i];
                wxn[2][i] = xn[i];
                wxh[0][i] = wxh[1][i];
                wxh[1][i] = wxh[2][i];
                wxh[2][i] = xh[i];
                wdu[0][i] = wdu[1][i];
                wdu[1][i] = wdu[2][i];
                wdu[2][i] = du[i];
            }
        };

        // dx of the output rows of stage s (their g, xhat in fin)
        auto finish = [&](int s) {
            auto one = [&](int g, int q) {
                const float rstd = st_ring[(q - p_s) & (kStRing - 1)].y;
                const float2 mt = tot[(s & 1) * kG + g];
                const f2 rs = f2_splat(rstd), na = f2_splat(-rstd * mt.x), nb = f2_splat(-rstd * mt.y);
                const float* fp = fin_at(s & 1, g);
                f2 o[NP];
#pragma unroll
                for (int i = 0; i < NP; i += 2) {
                    const float4 g4 = *reinterpret_cast<const float4*>(fp + 2 * i);
                    const float4 h4 = *reinterpret_cast<const float4*>(fp + 2 * NP + 2 * i);
                    o[i] = f2_fma(f2_make(h4.x, h4.y), nb, f2_fma(f2_make(g4.x, g4.y), rs, na));
                    o[i + 1] = f2_fma(f2_make(h4.z, h4.w), nb, f2_fma(f2_make(g4.z, g4.w), rs, na));
                }
                store_bf16(a.dx + (row0 + q) * D + c, o);
            };
            const int q0 = p_s + s * kG - 3;
            if (q0 >= t_b && q0 + kG <= t_e) {     // every row of the stage is an output row
                if (active) {
#pragma unroll
                    for (int g = 0; g < kG; ++g) one(g, q0 + g);
                }
            } else {
#pragma unroll
                for (int g = 0; g < kG; ++g)
                    if (q0 + g >= t_b && q0 + g < t_e && active) one(g, q0 + g);
            }
        };

        // ---- prologue: statistics of the rows of stages 0 and 1
        if (ln) {
            if (!mbar_wait(full + 0, 0, ctl)) failed = true;
            if (S > 1 && !failed && !mbar_wait(full + 1, 0, ctl)) failed = true;
            float v[16];
#pragma unroll
            for (int i = 0; i < 2 * kG; ++i) {
                const int p = p_s + i;
                if (!failed) moments(std::false_type{}, i / kG, i % kG, p, v[i], v[2 * kG + i]);
                else v[i] = v[2 * kG + i] = 0.f;
            }
            const float r = warp_reduce16(v, lane);
            if ((lane & 1) == 0) red[warp * 16 + (lane >> 1)] = r;
            if (!workers_or_bwd(failed, nwork)) {
                arm(0);
                if (tid < 16) {
                    float t = 0.f;
                    for (int w = 0; w < nwarps; ++w) t += red[w * 16 + tid];
                    push(0, tid, t);
                } else if (tid < kMsg) {
                    const int i = tid - 16;
                    push(0, tid, first_x(i / kG, i % kG, p_s + i));
                }
                if (warp == 0) {
                    if (!wait_x(0)) failed = true;
                    if (!failed && lane < 2 * kG) st_ring[lane] = combine_stats(0, lane, 2 * kG + lane, 16 + lane);
                }
            } else {
                failed = true;
            }
            if (workers_or_bwd(failed, nwork)) failed = true;
        }

        // ---- the stages (every exit from the loop follows a barrier, so
        // that all workers leave together)
        for (int s = 0; s < S && !failed; ++s) {
            const int pos0 = p_s + s * kG;
            if (ln && s >= 1 && warp == 0) {
                // exchange s (sent after stage s-1): the g sums of stage
                // s-1's output rows and the statistics of stage s+1's rows,
                // published to the other workers by this stage's barrier
                if (!wait_x(s)) failed = true;
                if (!failed) {
                    if (lane < kG) {
                        float sg = 0.f, sgx = 0.f;
                        for (int r2 = 0; r2 < CL; ++r2) {
                            sg += *xch_addr(s, r2, lane);
                            sgx += *xch_addr(s, r2, kG + lane);
                        }
                        tot[((s - 1) & 1) * kG + lane] = make_float2(sg * invD, sgx * invD);
                    } else if (lane < 2 * kG) {
                        const int g = lane - kG;
                        st_ring[(pos0 + kG + g - p_s) & (kStRing - 1)] =
                            combine_stats(s, 2 * kG + g, 3 * kG + g, 16 + g);
                    }
                }
            }
            const int slot = s % RING;
            bool ok = !failed && mbar_wait(full + slot, (s / RING) & 1, ctl);
            if (ln && ok && s + 2 < S) ok = mbar_wait(full + (s + 2) % RING, ((s + 2) / RING) & 1, ctl);
            if (!ok) failed = true;
#pragma unroll
            for (int i = 0; i < 2 * kG; ++i) gs[i] = 0.f;
            if (!failed) {
                if (pos0 >= t_b + 3 && pos0 + kG <= min(T, t_e)) {
#pragma unroll
                    for (int g = 0; g < kG; ++g) do_row(std::true_type{}, s, g, pos0 + g);
                } else {
#pragma unroll
                    for (int g = 0; g < kG; ++g)
                        if (pos0 + g <= t_e + 2) do_row(std::false_type{}, s, g, pos0 + g);
                }
            }
            mbar_arrive(freeb + slot);          // this worker is done with the stage's rows
            if constexpr (!LN) {
                if (workers_or_bwd(failed, nwork)) {
                    failed = true;
                    break;
                }
            } else {
                // moments of the rows two stages ahead, the g sums of this stage
                float v[16];
    #pragma unroll
                for (int i = 0; i < 2 * kG; ++i) v[i] = gs[i];
                    const int pm = pos0 + 2 * kG;           // the rows of stage s + 2
                if (!failed && s + 2 < S && pm >= 0 && pm + kG <= p_load) {
#pragma unroll
                    for (int g = 0; g < kG; ++g)
                        moments(std::true_type{}, s + 2, g, pm + g, v[2 * kG + g], v[3 * kG + g]);
                } else {
#pragma unroll
                    for (int g = 0; g < kG; ++g) {
                        if (!failed && s + 2 < S) moments(std::false_type{}, s + 2, g, pm + g, v[2 * kG + g], v[3 * kG + g]);
                        else v[2 * kG + g] = v[3 * kG + g] = 0.f;
                    }
                }
                float* rd = red + (s & 1) * nwarps * 16;
                const float r = warp_reduce16(v, lane);
                if ((lane & 1) == 0) rd[warp * 16 + (lane >> 1)] = r;
                if (workers_or_bwd(failed, nwork)) {
                    failed = true;
                    break;
                }
                arm(s + 1);
                if (tid < 16) {
                    float t = 0.f;
                    for (int w = 0; w < nwarps; ++w) t += rd[w * 16 + tid];
                    push(s + 1, tid, t);
                } else if (tid < kMsg) {
                    // every message is kMsg values (the arm counts them): the
                    // first elements of the rows two stages ahead, then zeros
                    const int g = tid - 16;
                    push(s + 1, tid, (g < kG && s + 2 < S) ? first_x(s + 2, g, pos0 + 2 * kG + g) : 0.f);
                }
                if (s >= 1) finish(s - 1);
            }
        }
        // the last stage's output rows
        if (ln && !failed && S > 0) {
            if (warp == 0) {
                if (!wait_x(S)) failed = true;
                if (!failed && lane < kG) {
                    float sg = 0.f, sgx = 0.f;
                    for (int r2 = 0; r2 < CL; ++r2) {
                        sg += *xch_addr(S, r2, lane);
                        sgx += *xch_addr(S, r2, kG + lane);
                    }
                    tot[((S - 1) & 1) * kG + lane] = make_float2(sg * invD, sgx * invD);
                }
            }
            if (!workers_or_bwd(failed, nwork)) finish(S - 1);
            else failed = true;
        }

        // per-(range, CTA) partial sums
        if (!failed && active) {
            float* pp = a.part + (static_cast<int64_t>(b) * a.nx + slice) * kParts * D + c;
            auto put = [&](int k, const f2 (&v)[NP]) { store_f32(pp + k * D, v); };
#pragma unroll
            for (int j = 0; j < kW; ++j) put(j, dw[j]);
            put(4, db);
            put(5, dg);
            put(6, dbe);
        }
    }
    // no CTA leaves while another may still write into its shared memory
    cluster_sync_all();
}

// Sum of the per-range partials in range order: thread per (part, channel).
// dw and dbias were summed from 2 du.
__global__ void __launch_bounds__(256) conv_bwd_reduce_kernel(const float* __restrict__ part, int nparts, int D,
                                                              float* __restrict__ dw, float* __restrict__ dbias,
                                                              float* __restrict__ dgamma, float* __restrict__ dbeta)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= kParts * D) return;
    const int k = i / D, ch = i - k * D;
    float s = 0.f;
    for (int n = 0; n < nparts; ++n) s += part[static_cast<int64_t>(n) * kParts * D + i];
    if (k < 4)
        dw[static_cast<int64_t>(ch) * 4 + k] = 0.5f * s;
    else if (k == 4) {
        if (dbias) dbias[ch] = 0.5f * s;
    } else if (k == 5) {
        if (dgamma) dgamma[ch] = s;
    } else if (dbeta) {
        dbeta[ch] = s;
    }
}

// At most 256 workers a CTA (4 channels each) and one producer warp, so
// that the per-channel registers fit without spilling.  (Workers of 2
// channels -- 13 warps a CTA at 128 registers -- measured slower at
// D = 3,072, 1.46 ms against 1.38 ms: the kernel is bound by instruction
// issue, and a narrower thread repeats the per-row work that does not
// scale with its channels.)
constexpr int kBwdThreads = 288;
constexpr int kBwdThreads8 = 224;   // 8-channel workers: at most 7 warps a CTA

struct BwdPlan {
    int CL, NP, upc, threads, nx, rps;
};

// Clusters of 2 CTAs where they fit: every SM can hold one (clusters of 4
// left 16 of 148 SMs idle, a GPC's SM count not being a multiple of 4).  Up
// to D = 2,048 a worker owns 4 channels; up to D = 3,072, 8 (at most 192
// workers + the producer: a thread may keep 255 registers, and the 4-stage
// ring and the g / xhat rows take 197 KB), which also spreads the per-row
// work that does not scale with the channels over twice as many; above,
// clusters of 4 CTAs with 4-channel workers.  clusters: how many clusters
// the device runs at once.
BwdPlan plan_bwd(int B, int T, int D, int clusters)
{
    BwdPlan pl;
    const int P = D / 8;
    pl.CL = D <= 3072 ? 2 : 4;
    pl.NP = D <= 2048 || D > 3072 ? 2 : 4;
    pl.upc = (P + pl.CL - 1) / pl.CL;
    pl.threads = ((pl.NP == 4 ? 1 : 2) * pl.upc + 31) / 32 * 32 + 32;
    int nx = clusters / (B > 0 ? B : 1);
    if (nx < 1) nx = 1;
    if (nx > kMaxSlices) nx = kMaxSlices;
    const int max_nx = (T + kMinRows - 1) / kMinRows;
    if (nx > max_nx) nx = max_nx;
    if (nx < 1) nx = 1;
    pl.rps = (T + nx - 1) / nx;
    pl.nx = (T + pl.rps - 1) / pl.rps;
    return pl;
}

}  // namespace

// part [B * nx][7][D] with nx at most min(128, ceil(T / 64)) ranges a sequence
size_t conv_bwd_workspace_bytes(int B, int T, int D)
{
    const size_t nx_max = std::min<size_t>(kMaxSlices, (static_cast<size_t>(T) + kMinRows - 1) / kMinRows);
    return align256(static_cast<size_t>(B) * (nx_max > 0 ? nx_max : 1) * kParts * D * sizeof(float));
}

gla_status launch_conv_bwd(const void* x, int apply_ln, const float* g, const float* be, float eps, const float* w,
                           const float* bias, const float* cs_in, const void* dy, void* dx, float* dw, float* dbias,
                           float* dgamma, float* dbeta, float* dcs, void* ws, int B, int T, int D, cudaStream_t st)
{
    gla_status se;
    const WaitCtl ctl = wait_ctl_for_current_device(&se);
    if (se != GLA_OK) return se;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    BwdPlan pl = plan_bwd(B, T, D, sms / (D <= 3072 ? 2 : 4));
    const int CL = pl.CL;
    const bool aff = g || be || bias;
    void (*kernel)(BwdArgs);
    const bool ln = apply_ln != 0;
    const int P = D / 8;
    const bool full = P % CL == 0 && ((pl.NP == 4 ? 1 : 2) * (P / CL)) % 32 == 0;
    // the 24 forms: affine or not, LayerNorm or not, every thread owning
    // channels or not; 4-channel workers in clusters of 2 or 4 CTAs, or
    // 8-channel workers in clusters of 2
    using KFn = void (*)(BwdArgs);
#define GLA_BWD_FORM(A, N, F)                                                                            \
    {ln_conv_silu_bwd_kernel<A, N, F, 2, 2, kBwdThreads>, ln_conv_silu_bwd_kernel<A, N, F, 4, 2, kBwdThreads>, \
     ln_conv_silu_bwd_kernel<A, N, F, 2, 4, kBwdThreads8>}
    static const KFn forms[2][2][2][3] = {
        {{GLA_BWD_FORM(false, false, false), GLA_BWD_FORM(false, false, true)},
         {GLA_BWD_FORM(false, true, false), GLA_BWD_FORM(false, true, true)}},
        {{GLA_BWD_FORM(true, false, false), GLA_BWD_FORM(true, false, true)},
         {GLA_BWD_FORM(true, true, false), GLA_BWD_FORM(true, true, true)}}};
#undef GLA_BWD_FORM
    kernel = forms[aff][ln][full][pl.NP == 4 ? 2 : (CL == 4 ? 1 : 0)];
    const BwdSmem L(pl.upc, pl.threads - 32, pl.NP);
    const size_t smem = L.total;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
        cudaSuccess)
        return check_launch("cudaFuncSetAttribute");
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.blockDim = dim3(pl.threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    // as many token ranges as clusters run at once (a GPC may hold a
    // number of SMs that is not a multiple of CL)
    cfg.gridDim = dim3(pl.nx * CL, B);
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, kernel, &cfg) == cudaSuccess && active > 0)
        pl = plan_bwd(B, T, D, active);
    else
        cudaGetLastError();
    cfg.gridDim = dim3(pl.nx * CL, B);
    BwdArgs a;
    a.x = static_cast<const __nv_bfloat16*>(x);
    a.dy = static_cast<const __nv_bfloat16*>(dy);
    a.gamma = g;
    a.beta = be;
    a.w = w;
    a.bias = bias;
    a.cs_in = cs_in;
    a.dx = static_cast<__nv_bfloat16*>(dx);
    a.part = static_cast<float*>(ws);
    a.dcs = dcs;
    a.T = T;
    a.D = D;
    a.nx = pl.nx;
    a.rps = pl.rps;
    a.upc = pl.upc;
    a.apply_ln = apply_ln;
    a.eps = eps;
    a.ctl = ctl;
    trace_begin(st);
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, a);
    trace_end(st, "ln_conv_silu_bwd_kernel");
    count_launch();
    if (e != cudaSuccess) return status_of(e);
    gla_status s;
    if ((s = check_launch("ln_conv_silu_bwd_kernel")) != GLA_OK) return s;
    trace_begin(st);
    conv_bwd_reduce_kernel<<<(kParts * D + 255) / 256, 256, 0, st>>>(a.part, B * pl.nx, D, dw, dbias, dgamma, dbeta);
    trace_end(st, "conv_bwd_reduce_kernel");
    count_launch();
    return check_launch("conv_bwd_reduce_kernel");
}

}  // namespace gla
