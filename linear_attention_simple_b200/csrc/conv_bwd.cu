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
// Three passes, none with a block-wide barrier per row:
//   ln_stats_kernel       mean and rstd of every row (a warp per row);
//   conv_bwd_tile_kernel<false>  tiles of 256 rows x 512 channels, a thread per
//                         2 channels walking the rows with register windows:
//                         u, du, dxn, the per-(tile, channel) sums of dw,
//                         dbias, dgamma, dbeta, the history gradient, and the
//                         per-row sums of g and g xhat over the tile's
//                         channels (dx itself when there is no LayerNorm);
//   conv_bwd_tile_kernel<true>   the same walk again, finishing dx from the
//                         row totals of those sums.
// conv_bwd_reduce_kernel adds the per-tile partials in a fixed order, so
// every output is deterministic.
#include <cuda_bf16.h>

#include "gla_device.cuh"
#include "gla_internal.h"

namespace gla {
namespace {

constexpr int kRows = 256;       // tokens per tile
constexpr int kTileThreads = 256;
constexpr int kTileCh = 2 * kTileThreads;   // channels per tile
constexpr int kParts = 7;        // dw (4 taps), dbias, dgamma, dbeta

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

__device__ __forceinline__ float warp_sum_bwd(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// stats[row] = (mean, rstd) of the row's D values; the moments are taken
// about the row's first element (shifted), as the forward does.
__global__ void __launch_bounds__(256) ln_stats_kernel(const __nv_bfloat16* __restrict__ x, int rows, int D,
                                                       float eps, float2* __restrict__ stats)
{
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (row >= rows) return;
    const __nv_bfloat16* xr = x + static_cast<int64_t>(row) * D;
    const float x0 = __bfloat162float(xr[0]);
    float s1 = 0.f, s2 = 0.f;
    for (int v = lane; v < D / 8; v += 32) {
        const uint4 q = *reinterpret_cast<const uint4*>(xr + v * 8);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float a = bf16_lo(w[i]) - x0, b = bf16_hi(w[i]) - x0;
            s1 += a + b;
            s2 = fmaf(a, a, fmaf(b, b, s2));
        }
    }
    s1 = warp_sum_bwd(s1);
    s2 = warp_sum_bwd(s2);
    if (lane == 0) {
        const float m1 = s1 / D;
        const float var = fmaxf(s2 / D - m1 * m1, 0.f);
        stats[row] = make_float2(x0 + m1, rsqrtf(var + eps));
    }
}

struct TileArgs {
    const __nv_bfloat16* x;
    const __nv_bfloat16* dy;
    const float* gamma;
    const float* beta;
    const float* w;
    const float* bias;
    const float* cs_in;
    const float2* stats;       // [B*T] (LayerNorm only)
    float2* psum;              // [B*T][CB] per-row sums of g and g xhat over a tile's channels
    float* part;               // [B * nrb][7][D]
    float* dcs;
    __nv_bfloat16* dx;
    int T, D, CB, nrb, apply_ln;
};

// FINISH = false: sums (and dx without LayerNorm); FINISH = true: dx.
template <bool FINISH>
__global__ void __launch_bounds__(kTileThreads) conv_bwd_tile_kernel(const TileArgs a)
{
    __shared__ float2 rowsum[kRows][kTileThreads / 32];
    __shared__ float2 total[kRows];
    __shared__ float2 st_s[kRows + 6];     // LayerNorm statistics of rows t0-3 .. t1+2
    const int rb = blockIdx.x, b = blockIdx.y, cb = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = cb * kTileCh + 2 * tid;
    const bool live = c < a.D;
    const int T = a.T, D = a.D;
    const int t0 = rb * kRows, t1 = min(T, t0 + kRows);
    const int64_t row0 = static_cast<int64_t>(b) * T;
    const bool ln = a.apply_ln != 0;

    for (int i = tid; i < t1 - t0 + 6; i += kTileThreads) {
        const int r = t0 - 3 + i;
        st_s[i] = (ln && r >= 0 && r < T) ? a.stats[row0 + r] : make_float2(0.f, 1.f);
    }
    if (FINISH) {
        // row totals of the tile's rows: the per-channel-block sums, in order
        for (int i = tid; i < t1 - t0; i += kTileThreads) {
            float sg = 0.f, sgh = 0.f;
            for (int k = 0; k < a.CB; ++k) {
                const float2 v = a.psum[(row0 + t0 + i) * a.CB + k];
                sg += v.x;
                sgh += v.y;
            }
            total[i] = make_float2(sg, sgh);
        }
    }
    __syncthreads();

    float wv[2][4], gm[2], bt[2], bi[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const float4 q = live ? *reinterpret_cast<const float4*>(a.w + static_cast<int64_t>(c + e) * 4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        wv[e][0] = q.x;
        wv[e][1] = q.y;
        wv[e][2] = q.z;
        wv[e][3] = q.w;
        gm[e] = (live && a.gamma) ? a.gamma[c + e] : 1.f;
        bt[e] = (live && a.beta) ? a.beta[c + e] : 0.f;
        bi[e] = (live && a.bias) ? a.bias[c + e] : 0.f;
    }
    float pdw[4][2] = {}, pdb[2] = {}, pdg[2] = {}, pdbe[2] = {};
    // windows over rows p-3 .. p (index 3 = row p)
    float xn[4][2] = {}, xh[4][2] = {}, du[4][2] = {}, rs[4] = {1.f, 1.f, 1.f, 1.f};

    // x and dy of a row (this thread's two channels), loaded a whole group of
    // kGroup rows ahead of their use: kGroup rows of loads stay in flight
    constexpr int kGroup = 4;
    auto fetch = [&](int r) {
        uint2 v = make_uint2(0u, 0u);
        if (live && r >= 0 && r < T) {
            v.x = *reinterpret_cast<const uint32_t*>(a.x + (row0 + r) * D + c);
            if (r >= t0) v.y = *reinterpret_cast<const uint32_t*>(a.dy + (row0 + r) * D + c);
        }
        return v;
    };
    uint2 cur[kGroup], nxt[kGroup];
#pragma unroll
    for (int i = 0; i < kGroup; ++i) cur[i] = fetch(t0 - 3 + i);

    auto row = [&](int p, const uint2 f0) {
        const float2 st = st_s[p - (t0 - 3)];
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            rs[j] = rs[j + 1];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                xn[j][e] = xn[j + 1][e];
                xh[j][e] = xh[j + 1][e];
                du[j][e] = du[j + 1][e];
            }
        }
        // (1) conv input of row p
        if (p < 0) {
            const bool hv = live && a.cs_in;
            const float* src = a.cs_in + (static_cast<int64_t>(b) * 3 + p + 3) * D + c;
            xn[3][0] = hv ? src[0] : 0.f;
            xn[3][1] = hv ? src[1] : 0.f;
            xh[3][0] = xh[3][1] = 0.f;
            rs[3] = 1.f;
        } else if (p < T) {
            const float v0 = bf16_lo(f0.x), v1 = bf16_hi(f0.x);
            if (ln) {
                xh[3][0] = (v0 - st.x) * st.y;
                xh[3][1] = (v1 - st.x) * st.y;
                xn[3][0] = fmaf(xh[3][0], gm[0], bt[0]);
                xn[3][1] = fmaf(xh[3][1], gm[1], bt[1]);
                rs[3] = st.y;
            } else {
                xh[3][0] = xn[3][0] = v0;
                xh[3][1] = xn[3][1] = v1;
                rs[3] = 1.f;
            }
        } else {
            xn[3][0] = xn[3][1] = xh[3][0] = xh[3][1] = 0.f;
            rs[3] = 1.f;
        }
        // (2) du of row p (rows t0 .. T-1; zero elsewhere)
        if (p >= t0 && p < T) {
            const float dyv[2] = {bf16_lo(f0.y), bf16_hi(f0.y)};
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float u = bi[e];
#pragma unroll
                for (int j = 0; j < 4; ++j) u = fmaf(wv[e][j], xn[j][e], u);
                // sigmoid with the fast exponential and division intrinsics:
                // about 2 ulp, far below the bf16 rounding of dx
                const float sg = __fdividef(1.f, 1.f + __expf(-u));
                du[3][e] = dyv[e] * sg * fmaf(u, 1.f - sg, 1.f);
            }
            if (!FINISH && p < t1) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    pdb[e] += du[3][e];
#pragma unroll
                    for (int j = 0; j < 4; ++j) pdw[j][e] = fmaf(du[3][e], xn[j][e], pdw[j][e]);
                }
            }
        } else {
            du[3][0] = du[3][1] = 0.f;
        }
        // (3) dxn of row q = p - 3, then its LayerNorm backward
        const int q = p - 3;
        const bool out_row = q >= t0 && q < t1;
        const bool hist_row = t0 == 0 && q < 0 && q >= -3;   // rows -3 .. -1: the history
        if (out_row || hist_row) {
            float dxn[2];
#pragma unroll
            for (int e = 0; e < 2; ++e)
                dxn[e] = wv[e][3] * du[0][e] + wv[e][2] * du[1][e] + wv[e][1] * du[2][e] + wv[e][0] * du[3][e];
            if (hist_row) {
                if (!FINISH && live && a.dcs) {
                    float* dst = a.dcs + (static_cast<int64_t>(b) * 3 + q + 3) * D + c;
                    dst[0] = dxn[0];
                    dst[1] = dxn[1];
                }
            } else if (ln) {
                const float g0 = dxn[0] * gm[0], g1 = dxn[1] * gm[1];
                if (!FINISH) {
                    const float sgv = warp_sum_bwd(g0 + g1);
                    const float sghv = warp_sum_bwd(fmaf(g0, xh[0][0], g1 * xh[0][1]));
                    if (lane == 0) rowsum[q - t0][warp] = make_float2(sgv, sghv);
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        pdg[e] = fmaf(dxn[e], xh[0][e], pdg[e]);
                        pdbe[e] += dxn[e];
                    }
                } else if (live) {
                    const float2 tt = total[q - t0];
                    const float mg = tt.x / D, mgh = tt.y / D;
                    const float o0 = rs[0] * (g0 - mg - xh[0][0] * mgh);
                    const float o1 = rs[0] * (g1 - mg - xh[0][1] * mgh);
                    *reinterpret_cast<uint32_t*>(a.dx + (row0 + q) * D + c) = pack_bf16(o0, o1);
                }
            } else if (!FINISH && live) {
                *reinterpret_cast<uint32_t*>(a.dx + (row0 + q) * D + c) = pack_bf16(dxn[0], dxn[1]);
            }
        }
    };

    for (int p0 = t0 - 3; p0 <= t1 + 2; p0 += kGroup) {
#pragma unroll
        for (int i = 0; i < kGroup; ++i) nxt[i] = fetch(p0 + kGroup + i);
#pragma unroll
        for (int i = 0; i < kGroup; ++i)
            if (p0 + i <= t1 + 2) row(p0 + i, cur[i]);
#pragma unroll
        for (int i = 0; i < kGroup; ++i) cur[i] = nxt[i];
    }

    if (!FINISH) {
        // per-row sums over this tile's channels, in warp order
        if (ln) {
            __syncthreads();
            for (int i = tid; i < t1 - t0; i += kTileThreads) {
                float sg = 0.f, sgh = 0.f;
#pragma unroll
                for (int k = 0; k < kTileThreads / 32; ++k) {
                    sg += rowsum[i][k].x;
                    sgh += rowsum[i][k].y;
                }
                a.psum[(row0 + t0 + i) * a.CB + cb] = make_float2(sg, sgh);
            }
        }
        // per-tile partials: dw taps 0..3, dbias, dgamma, dbeta
        if (live) {
            float* pp = a.part + (static_cast<int64_t>(b) * a.nrb + rb) * kParts * D + c;
#pragma unroll
            for (int j = 0; j < 4; ++j) *reinterpret_cast<float2*>(pp + j * D) = make_float2(pdw[j][0], pdw[j][1]);
            *reinterpret_cast<float2*>(pp + 4 * D) = make_float2(pdb[0], pdb[1]);
            *reinterpret_cast<float2*>(pp + 5 * D) = make_float2(pdg[0], pdg[1]);
            *reinterpret_cast<float2*>(pp + 6 * D) = make_float2(pdbe[0], pdbe[1]);
        }
    }
}

// Sum of the per-CTA partials in CTA order: thread per (part, channel).
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
        dw[static_cast<int64_t>(ch) * 4 + k] = s;
    else if (k == 4) {
        if (dbias) dbias[ch] = s;
    } else if (k == 5) {
        if (dgamma) dgamma[ch] = s;
    } else if (dbeta) {
        dbeta[ch] = s;
    }
}

}  // namespace

// part [B * nrb][7][D] | stats [B*T] float2 | psum [B*T][CB] float2
size_t conv_bwd_workspace_bytes(int B, int T, int D)
{
    const size_t nrb = static_cast<size_t>((T + kRows - 1) / kRows), CB = (D + kTileCh - 1) / kTileCh;
    const size_t rows = static_cast<size_t>(B) * T;
    return align256(static_cast<size_t>(B) * nrb * kParts * D * sizeof(float)) + align256(rows * sizeof(float2)) +
           align256(rows * CB * sizeof(float2));
}

gla_status launch_conv_bwd(const void* x, int apply_ln, const float* g, const float* be, float eps, const float* w,
                           const float* bias, const float* cs_in, const void* dy, void* dx, float* dw, float* dbias,
                           float* dgamma, float* dbeta, float* dcs, void* ws, int B, int T, int D, cudaStream_t st)
{
    const int nrb = (T + kRows - 1) / kRows, CB = (D + kTileCh - 1) / kTileCh;
    const size_t rows = static_cast<size_t>(B) * T;
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    TileArgs a;
    a.x = static_cast<const __nv_bfloat16*>(x);
    a.dy = static_cast<const __nv_bfloat16*>(dy);
    a.gamma = g;
    a.beta = be;
    a.w = w;
    a.bias = bias;
    a.cs_in = cs_in;
    a.part = reinterpret_cast<float*>(wsb);
    size_t off = align256(static_cast<size_t>(B) * nrb * kParts * D * sizeof(float));
    float2* stats = reinterpret_cast<float2*>(wsb + off);
    off += align256(rows * sizeof(float2));
    a.stats = stats;
    a.psum = reinterpret_cast<float2*>(wsb + off);
    a.dcs = dcs;
    a.dx = static_cast<__nv_bfloat16*>(dx);
    a.T = T;
    a.D = D;
    a.CB = CB;
    a.nrb = nrb;
    a.apply_ln = apply_ln;
    gla_status s;
    if (apply_ln) {
        trace_begin(st);
        ln_stats_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(a.x, static_cast<int>(rows), D, eps,
                                                                              stats);
        trace_end(st, "ln_stats_kernel");
        count_launch();
        if ((s = check_launch("ln_stats_kernel")) != GLA_OK) return s;
    }
    const dim3 grid(nrb, B, CB);
    trace_begin(st);
    conv_bwd_tile_kernel<false><<<grid, kTileThreads, 0, st>>>(a);
    trace_end(st, "conv_bwd_tile_kernel");
    count_launch();
    if ((s = check_launch("conv_bwd_tile_kernel")) != GLA_OK) return s;
    if (apply_ln) {
        trace_begin(st);
        conv_bwd_tile_kernel<true><<<grid, kTileThreads, 0, st>>>(a);
        trace_end(st, "conv_bwd_dx_kernel");
        count_launch();
        if ((s = check_launch("conv_bwd_dx_kernel")) != GLA_OK) return s;
    }
    trace_begin(st);
    conv_bwd_reduce_kernel<<<(kParts * D + 255) / 256, 256, 0, st>>>(a.part, B * nrb, D, dw, dbias, dgamma, dbeta);
    trace_end(st, "conv_bwd_reduce_kernel");
    count_launch();
    return check_launch("conv_bwd_reduce_kernel");
}

}  // namespace gla
