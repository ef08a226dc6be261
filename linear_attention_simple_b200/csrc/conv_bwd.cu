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
// conv_bwd_kernel: one CTA per (128-token range, sequence), thread i owns
// CH consecutive channels (4, or 8 when D > 3072) and walks the rows p = t0-3 .. t1+2 once: the
// LayerNorm of row p (one block reduction of the shifted first and second
// moments), then u and du of row p, then dxn and dx of row q = p-3 (one block
// reduction of sum g and sum g xhat).  The last four rows of xn, xhat and du
// sit in shared-memory rings private to each thread.  The sums over tokens
// go to per-CTA partials; conv_bwd_reduce_kernel adds them in a fixed order
// (deterministic).
#include <cuda_bf16.h>

#include "gla_device.cuh"
#include "gla_internal.h"

namespace gla {
namespace {

constexpr int kRows = 128;       // tokens per CTA
constexpr int kParts = 7;        // dw (4 taps), dbias, dgamma, dbeta

__device__ __forceinline__ float warp_sum_bwd(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Block sums of (a, b); every thread gets both.  Two buffers used in turn,
// so one barrier per reduction suffices.
__device__ __forceinline__ void block_sum2(float& a, float& b, float* red, int& turn)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = (blockDim.x + 31) >> 5;
    float* r = red + (turn & 1) * 64;
    ++turn;
    a = warp_sum_bwd(a);
    b = warp_sum_bwd(b);
    if (lane == 0) {
        r[warp] = a;
        r[32 + warp] = b;
    }
    __syncthreads();
    // every warp reduces the per-warp partials again (same order in each)
    a = warp_sum_bwd(lane < nw ? r[lane] : 0.f);
    b = warp_sum_bwd(lane < nw ? r[32 + lane] : 0.f);
}

// Raw bf16 words of CH channels (prefetched ahead of their use).
template <int CH>
struct RawRow {
    uint32_t w[CH / 2];
};

template <int CH>
__device__ __forceinline__ RawRow<CH> ld_raw(const __nv_bfloat16* p)
{
    RawRow<CH> r;
    if constexpr (CH == 4) {
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        r.w[0] = u.x;
        r.w[1] = u.y;
    } else {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        r.w[0] = u.x;
        r.w[1] = u.y;
        r.w[2] = u.z;
        r.w[3] = u.w;
    }
    return r;
}

template <int CH>
__device__ __forceinline__ void unpack_raw(const RawRow<CH>& r, float (&v)[CH])
{
#pragma unroll
    for (int i = 0; i < CH / 2; ++i) {
        v[2 * i] = bf16_lo(r.w[i]);
        v[2 * i + 1] = bf16_hi(r.w[i]);
    }
}

template <int CH>
__device__ __forceinline__ void stv_bf16(__nv_bfloat16* p, const float (&v)[CH])
{
    if constexpr (CH == 4) {
        *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]));
    } else {
        *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                                                  pack_bf16(v[6], v[7]));
    }
}

template <int CH>
__device__ __forceinline__ void ldv_f32(const float* p, float (&v)[CH])
{
#pragma unroll
    for (int i = 0; i < CH; i += 4) {
        const float4 q = *reinterpret_cast<const float4*>(p + i);
        v[i] = q.x;
        v[i + 1] = q.y;
        v[i + 2] = q.z;
        v[i + 3] = q.w;
    }
}

template <int CH>
__device__ __forceinline__ void stv_f32(float* p, const float (&v)[CH])
{
#pragma unroll
    for (int i = 0; i < CH; i += 4) *reinterpret_cast<float4*>(p + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
}

// CH channels per thread: 4 (at most 768 threads, D <= 3072) or 8 (D <= 4096).
template <int CH>
__global__ void __launch_bounds__(CH == 4 ? 768 : 512, 1) conv_bwd_kernel(
    const __nv_bfloat16* __restrict__ x, int apply_ln, const float* __restrict__ gamma,
    const float* __restrict__ beta, float eps, const float* __restrict__ w, const float* __restrict__ bias,
    const float* __restrict__ cs_in, const __nv_bfloat16* __restrict__ dy, __nv_bfloat16* __restrict__ dx,
    float* __restrict__ dcs, float* __restrict__ part, int T, int D)
{
    extern __shared__ float smf[];
    float* xn_r = smf;               // [4][D]
    float* xh_r = smf + 4 * D;       // [4][D]
    float* du_r = smf + 8 * D;       // [4][D]
    float* red = smf + 12 * D;       // [2][64]
    float* aff = red + 128;          // CH == 4: [3][D] gamma, beta, bias (fewer live registers)
    const int blk = blockIdx.x, b = blockIdx.y, c = threadIdx.x * CH;
    const int t0 = blk * kRows, t1 = min(T, t0 + kRows);
    const int64_t row0 = static_cast<int64_t>(b) * T;

    float wv[CH][4];
    float aff_r[3][CH == 4 ? 1 : CH];
#pragma unroll
    for (int e = 0; e < CH; ++e) {
        const float4 q = *reinterpret_cast<const float4*>(w + static_cast<int64_t>(c + e) * 4);
        wv[e][0] = q.x;
        wv[e][1] = q.y;
        wv[e][2] = q.z;
        wv[e][3] = q.w;
        const float gv = gamma ? gamma[c + e] : 1.f, bv = beta ? beta[c + e] : 0.f, iv = bias ? bias[c + e] : 0.f;
        if constexpr (CH == 4) {
            aff[c + e] = gv;
            aff[D + c + e] = bv;
            aff[2 * D + c + e] = iv;
        } else {
            aff_r[0][e] = gv;
            aff_r[1][e] = bv;
            aff_r[2][e] = iv;
        }
    }
    // gamma, beta, bias of channel c+e (thread-private in shared memory when
    // CH == 4, read as one 16-byte vector: conflict-free)
    auto affv = [&](int k, int e) {
        if constexpr (CH == 4) {
            const float4 q = *reinterpret_cast<const float4*>(aff + k * D + c);
            return e == 0 ? q.x : e == 1 ? q.y : e == 2 ? q.z : q.w;
        } else {
            return aff_r[k][e];
        }
    };
    auto g4 = [&](int e) { return affv(0, e); };
    auto be4 = [&](int e) { return affv(1, e); };
    auto bi4 = [&](int e) { return affv(2, e); };
    float pdw[4][CH] = {}, pdb[CH] = {}, pdg[CH] = {}, pdbe[CH] = {};
    float rs_r[4] = {1.f, 1.f, 1.f, 1.f};
    int turn = 0;

    // x (with its row's first element, the LayerNorm shift) and dy of rows
    // p, p+1 and p+2 in registers: loads go out two rows ahead of their use
    auto fetch = [&](int r, RawRow<CH>& xr, float& x0, RawRow<CH>& dr) {
        if (r >= 0 && r < T) {
            xr = ld_raw<CH>(x + (row0 + r) * D + c);
            x0 = __bfloat162float(x[(row0 + r) * D]);
            if (r >= t0) dr = ld_raw<CH>(dy + (row0 + r) * D + c);
        }
    };
    RawRow<CH> xr0 = {}, xr1 = {}, xr2 = {}, dr0 = {}, dr1 = {}, dr2 = {};
    float x00 = 0.f, x01 = 0.f, x02 = 0.f;
    fetch(t0 - 3, xr0, x00, dr0);
    fetch(t0 - 2, xr1, x01, dr1);

    for (int p = t0 - 3; p <= t1 + 2; ++p) {
        const int s = (p + 4) & 3;
        fetch(p + 2, xr2, x02, dr2);
        // (1) conv input of row p
        float xnv[CH] = {}, xhv[CH] = {};
        float rs = 1.f;
        if (p < 0) {
            if (cs_in) ldv_f32<CH>(cs_in + (static_cast<int64_t>(b) * 3 + p + 3) * D + c, xnv);
        } else if (p < T) {
            float v[CH];
            unpack_raw<CH>(xr0, v);
            if (apply_ln) {
                const float x0 = x00;   // shift: the row's first element
                float s1 = 0.f, s2 = 0.f;
#pragma unroll
                for (int e = 0; e < CH; ++e) {
                    s1 += v[e] - x0;
                    s2 = fmaf(v[e] - x0, v[e] - x0, s2);
                }
                block_sum2(s1, s2, red, turn);
                const float m1 = s1 / D;
                const float var = fmaxf(s2 / D - m1 * m1, 0.f);
                const float mean = x0 + m1;
                rs = rsqrtf(var + eps);
#pragma unroll
                for (int e = 0; e < CH; ++e) {
                    xhv[e] = (v[e] - mean) * rs;
                    xnv[e] = fmaf(xhv[e], g4(e), be4(e));
                }
            } else {
#pragma unroll
                for (int e = 0; e < CH; ++e) xnv[e] = xhv[e] = v[e];
            }
        }
        rs_r[s] = rs;
        stv_f32<CH>(xn_r + s * D + c, xnv);
        stv_f32<CH>(xh_r + s * D + c, xhv);

        // (2) du of row p (rows t0 .. T-1; zero elsewhere)
        float duv[CH] = {};
        if (p >= t0 && p < T) {
            float dyv[CH];
            unpack_raw<CH>(dr0, dyv);
            float win[4][CH];   // xn of rows p-3 .. p: vector loads, conflict-free
#pragma unroll
            for (int j = 0; j < 3; ++j) ldv_f32<CH>(xn_r + ((p + 1 + j) & 3) * D + c, win[j]);
#pragma unroll
            for (int e = 0; e < CH; ++e) win[3][e] = xnv[e];
#pragma unroll
            for (int e = 0; e < CH; ++e) {
                float u = bi4(e);
#pragma unroll
                for (int j = 0; j < 4; ++j) u = fmaf(wv[e][j], win[j][e], u);
                const float sg = 1.f / (1.f + expf(-u));
                duv[e] = dyv[e] * sg * fmaf(u, 1.f - sg, 1.f);
            }
            if (p < t1) {
#pragma unroll
                for (int e = 0; e < CH; ++e) {
                    pdb[e] += duv[e];
#pragma unroll
                    for (int j = 0; j < 4; ++j) pdw[j][e] = fmaf(duv[e], win[j][e], pdw[j][e]);
                }
            }
        }
        stv_f32<CH>(du_r + s * D + c, duv);

        // (3) dxn and dx of row q = p - 3
        const int q = p - 3;
        const bool out_row = q >= t0 && q < t1;
        const bool hist_row = t0 == 0 && q < 0 && q >= -3;   // rows -3 .. -1: the history
        if (out_row || hist_row) {
            float d4[3][CH];   // du of rows q .. q+2 (row q+3 = p is in registers)
#pragma unroll
            for (int j = 0; j < 3; ++j) ldv_f32<CH>(du_r + ((q + 4 + j) & 3) * D + c, d4[j]);
            float dxn[CH];
#pragma unroll
            for (int e = 0; e < CH; ++e)
                dxn[e] = wv[e][3] * d4[0][e] + wv[e][2] * d4[1][e] + wv[e][1] * d4[2][e] + wv[e][0] * duv[e];
            if (hist_row) {
                if (dcs) stv_f32<CH>(dcs + (static_cast<int64_t>(b) * 3 + q + 3) * D + c, dxn);
            } else {
                float o[CH];
                if (apply_ln) {
                    const int sq = (q + 4) & 3;
                    float xh[CH];
                    ldv_f32<CH>(xh_r + sq * D + c, xh);
                    float sg = 0.f, sgh = 0.f, gg[CH];
#pragma unroll
                    for (int e = 0; e < CH; ++e) {
                        gg[e] = dxn[e] * g4(e);
                        sg += gg[e];
                        sgh = fmaf(gg[e], xh[e], sgh);
                        pdg[e] = fmaf(dxn[e], xh[e], pdg[e]);
                        pdbe[e] += dxn[e];
                    }
                    block_sum2(sg, sgh, red, turn);
                    const float mg = sg / D, mgh = sgh / D, r = rs_r[sq];
#pragma unroll
                    for (int e = 0; e < CH; ++e) o[e] = r * (gg[e] - mg - xh[e] * mgh);
                } else {
#pragma unroll
                    for (int e = 0; e < CH; ++e) o[e] = dxn[e];
                }
                stv_bf16<CH>(dx + (row0 + q) * D + c, o);
            }
        }
        xr0 = xr1;
        xr1 = xr2;
        dr0 = dr1;
        dr1 = dr2;
        x00 = x01;
        x01 = x02;
    }

    // per-CTA partials: rows dw tap 0..3, dbias, dgamma, dbeta
    float* pp = part + (static_cast<int64_t>(b) * gridDim.x + blk) * kParts * D + c;
#pragma unroll
    for (int j = 0; j < 4; ++j) stv_f32<CH>(pp + j * D, pdw[j]);
    stv_f32<CH>(pp + 4 * D, pdb);
    stv_f32<CH>(pp + 5 * D, pdg);
    stv_f32<CH>(pp + 6 * D, pdbe);
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

size_t conv_bwd_workspace_bytes(int B, int T, int D)
{
    const size_t nblk = static_cast<size_t>((T + kRows - 1) / kRows);
    return static_cast<size_t>(B) * nblk * kParts * D * sizeof(float);
}

gla_status launch_conv_bwd(const void* x, int apply_ln, const float* g, const float* be, float eps, const float* w,
                           const float* bias, const float* cs_in, const void* dy, void* dx, float* dw, float* dbias,
                           float* dgamma, float* dbeta, float* dcs, void* ws, int B, int T, int D, cudaStream_t st)
{
    const int nblk = (T + kRows - 1) / kRows;
    const size_t smem = ((D <= 3072 ? 15 : 12) * static_cast<size_t>(D) + 128) * sizeof(float);
    const bool narrow = D <= 3072;
    auto kern = narrow ? conv_bwd_kernel<4> : conv_bwd_kernel<8>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return check_launch("cudaFuncSetAttribute");
    float* part = static_cast<float*>(ws);
    trace_begin(st);
    kern<<<dim3(nblk, B), D / (narrow ? 4 : 8), smem, st>>>(
        static_cast<const __nv_bfloat16*>(x), apply_ln, g, be, eps, w, bias, cs_in,
        static_cast<const __nv_bfloat16*>(dy), static_cast<__nv_bfloat16*>(dx), dcs, part, T, D);
    trace_end(st, "conv_bwd_kernel");
    count_launch();
    gla_status s = check_launch("conv_bwd_kernel");
    if (s != GLA_OK) return s;
    trace_begin(st);
    conv_bwd_reduce_kernel<<<(kParts * D + 255) / 256, 256, 0, st>>>(part, B * nblk, D, dw, dbias, dgamma, dbeta);
    trace_end(st, "conv_bwd_reduce_kernel");
    count_launch();
    return check_launch("conv_bwd_reduce_kernel");
}

}  // namespace gla
