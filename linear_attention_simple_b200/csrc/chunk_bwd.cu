// chunk_bwd.cu -- chunked Simple GLA backward on tcgen05.
//
// The backward of the chunked recurrence ("Como i14 llevo Laplace 3B a AWS
// Trainium2", section "Adaptaciones para AWS Trainium2", item 3: the backward
// walks the 16 chunks of a sequence in reverse).  For chunk c with tokens
// i, j, in-chunk cumulative log-decay b (gamma = b_last), h = S_{c-1} (state
// entering the chunk) and D = dL/dS_c (gradient of the state after it):
//
//   dP_ij = scale (dO_i . v_j) e^{b_i - b_j} [j <= i]
//   P_ij  = scale (q_i . k_j)  e^{b_i - b_j} [j <= i]
//   dq = diag(scale e^{b}) dO h^T + dP K
//   dk = dP^T Q + diag(e^{gamma - b}) V D^T
//   dv = P^T dO + diag(e^{gamma - b}) K D
//   da_t = sum_{m >= t} (q_m . dq_m - k_m . dk_m) + <dS_T, S_T>
//
// Passes (all on the caller's stream):
//   1. state kernel, forward, state-only: h_c (bf16) for every chunk, and
//      S_T when an upstream dS_T is given;
//   2. state kernel, reverse: D_c (bf16) for every chunk, dS_0 = D_{-1};
//   3. bwd_dqdk_kernel and bwd_dv_kernel: one CTA per (batch, head, chunk),
//      fully parallel, tcgen05 for every contraction; dP and P are split
//      into bf16 hi + lo terms; the row factors diag(...) are applied to
//      separate TMEM accumulators in the epilogue, so no operand needs a
//      scaled copy; the epilogue also emits q.dq - k.dk per token;
//   4. da_scan_kernel: reverse cumulative sum over T (plus <dS_T, S_T>).
#include <cstring>

#include "chunk_state.cuh"

namespace gla {
namespace {

constexpr int64_t kSS = static_cast<int64_t>(kDk) * kDv;
constexpr float kLog2e = 1.4426950408889634f;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
int num_chunks(int T) { return (T + kChunk - 1) / kChunk; }

struct BwdParams {
    CUtensorMap tm_q, tm_k, tm_v, tm_do;   // token tiles
    CUtensorMap tm_h, tm_d;                // per-chunk bf16 states
    CUtensorMap tm_dq, tm_dk, tm_dv;       // gradient stores
    CUtensorMap tm_do32, tm_d32, tm_dv32;  // 32-column SW64 boxes (dv kernel)
    const float* a;
    float* delta;                          // [B, T, H]: q.dq - k.dk per token
    int B, T, H, NC;
    float scale;
    WaitCtl ctl;
};

namespace bq {   // dq / dk kernel shared-memory map
constexpr uint32_t Q = 0, K = 24576, V = 49152, DO = 98304, HS = 147456, DS = 184320;
constexpr uint32_t MISC = 221184;
constexpr uint32_t BYTES = MISC + 2048 + 1024;
constexpr uint32_t TM_DP = 0, TM_X = 128, TM_W = 224, TM_Y = 320, TM_Z = 416;
}  // namespace bq


// Threads: warps 0-7 are workers; warp 8 only issues TMA and tcgen05.mma.
constexpr int kThreadsBwd = 288;

__device__ __forceinline__ void named_sync128()
{
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

// Inclusive cumulative log2-decay of the chunk's tokens, warps 0-3.
__device__ __forceinline__ void chunk_cumsum(float a, float* b2s, float* wsum, int tid, int warp,
                                             int lane)
{
    float x = a * kLog2e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    named_sync128();
    float pre = 0.f;
    for (int w = 0; w < warp; ++w) pre += wsum[w];
    b2s[tid] = x + pre;
}

// Masked, decayed 128x128 tile from TMEM (rows = this thread's lane, columns
// half*64 .. +63), split into bf16 hi and lo, written [i][j] as a K-major
// SW128 operand ([2][128][64]) at hi / lo.
__device__ __forceinline__ void masked_decay_tile(uint32_t tq, uint32_t col0, int row, int quad,
                                                  int half, const float* b2s, float scale,
                                                  uint8_t* hi_base, uint8_t* lo_base)
{
    const float b2r = b2s[row];
#pragma unroll
    for (int q2 = 0; q2 < 2; ++q2) {
        const int j0 = half * 64 + q2 * 32;
        uint32_t hi[16], lo[16];
        if (j0 > quad * 32 + 31) {
#pragma unroll
            for (int e = 0; e < 16; ++e) hi[e] = lo[e] = 0u;
        } else {
            uint32_t r[32];
            tmem_ld32(tq + col0 + j0, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
                const int j = j0 + e;
                const float v0 = (j <= row) ? scale * __uint_as_float(r[e]) * exp2f(b2r - b2s[j]) : 0.f;
                const float v1 = (j + 1 <= row) ? scale * __uint_as_float(r[e + 1]) * exp2f(b2r - b2s[j + 1]) : 0.f;
                const uint32_t h = pack_bf16(v0, v1);
                hi[e / 2] = h;
                lo[e / 2] = pack_bf16(v0 - bf16_lo(h), v1 - bf16_hi(h));
            }
        }
        uint8_t* hb = hi_base + half * 16384;
        uint8_t* lb = lo_base + half * 16384;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            const uint32_t off = swz_off(row, q2 * 4 + c4, 128);
            *reinterpret_cast<uint4*>(hb + off) = make_uint4(hi[c4 * 4], hi[c4 * 4 + 1], hi[c4 * 4 + 2], hi[c4 * 4 + 3]);
            *reinterpret_cast<uint4*>(lb + off) = make_uint4(lo[c4 * 4], lo[c4 * 4 + 1], lo[c4 * 4 + 2], lo[c4 * 4 + 3]);
        }
    }
}

__device__ __forceinline__ float bf16_at_sw64(const uint8_t* tile, int row, int d)
{
    const uint8_t* p = tile + (d >> 5) * 8192 + swz_off(row, (d & 31) >> 3, 64) + (d & 7) * 2;
    return __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(p)) << 16);
}

// ------------------------------------------------------------ dq, dk kernel

__global__ void __launch_bounds__(kThreadsBwd, 1) bwd_dqdk_kernel(const __grid_constant__ BwdParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(sm + bq::MISC);
    uint64_t* bar_m = bar_ld + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ld + 2);
    float* b2s = reinterpret_cast<float*>(sm + bq::MISC + 64);
    float* wsum = b2s + 128;
    float* dpart = wsum + 8;                 // [128]: delta partial of column half 1

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int unit = b * p.H + h;
    const int t0 = c * kChunk;
    const int quad = warp & 3, half = (warp >> 2) & 1, row = quad * 32 + lane;
    const bool worker = warp < 8;
    const bool issuer = warp == 8 && lane == 0;
    const WaitCtl ctl = p.ctl;

    if (issuer) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_m, 1);
        mbar_init_fence();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tq = tmem_addr(tmem, quad * 32, 0);
    bool failed = false;
    bool pend_ld = false, pend_m = false;
    float dsum = 0.f;                        // this thread's share of q.dq - k.dk

    if (issuer) {
        mbar_arrive_expect_tx(bar_ld, 2 * chunk::kTileQK + 2 * chunk::kTileV + 2 * 36864);
        for (int i = 0; i < 3; ++i) {
            tma_load_4d(sm + bq::Q + i * 8192, &p.tm_q, bar_ld, i * 32, h, t0, b);
            tma_load_4d(sm + bq::K + i * 8192, &p.tm_k, bar_ld, i * 32, h, t0, b);
            tma_load_4d(sm + bq::V + i * 16384, &p.tm_v, bar_ld, i * 64, h, t0, b);
            tma_load_4d(sm + bq::DO + i * 16384, &p.tm_do, bar_ld, i * 64, h, t0, b);
            tma_load_3d(sm + bq::HS + i * 12288, &p.tm_h, bar_ld, i * 64, 0, unit * p.NC + c);
            tma_load_3d(sm + bq::DS + i * 12288, &p.tm_d, bar_ld, i * 64, 0, unit * p.NC + c);
        }
        pend_ld = true;
        if (mbar_wait(bar_ld, 0, ctl)) {
            pend_ld = false;
            tc_fence_after();
            // dP_raw = dO V^T ; X = dO h^T ; W = V D^T
            for (int ks = 0; ks < 12; ++ks) {
                const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                const uint32_t soff = (ks >> 2) * 12288 + (ks & 3) * 32;
                const uint64_t ado = smem_desc(sb + bq::DO + off, 16, 1024, kLayoutSW128);
                const uint64_t av = smem_desc(sb + bq::V + off, 16, 1024, kLayoutSW128);
                umma_bf16(tmem + bq::TM_DP, ado, av, idesc_bf16_f32(128, 128, 0, 0), ks > 0);
                umma_bf16(tmem + bq::TM_X, ado, smem_desc(sb + bq::HS + soff, 16, 1024, kLayoutSW128),
                          idesc_bf16_f32(128, 96, 0, 0), ks > 0);
                umma_bf16(tmem + bq::TM_W, av, smem_desc(sb + bq::DS + soff, 16, 1024, kLayoutSW128),
                          idesc_bf16_f32(128, 96, 0, 0), ks > 0);
            }
            umma_commit(bar_m);
            pend_m = true;
        } else {
            failed = true;
        }
    }
    if (tid < 128) {
        const int t = t0 + tid;
        chunk_cumsum(t < p.T ? p.a[(static_cast<int64_t>(b) * p.T + t) * p.H + h] : 0.f, b2s, wsum,
                     tid, warp, lane);
    }
    if (!failed && !mbar_wait(bar_m, 0, ctl)) failed = true;
    tc_fence_before();
    if (__syncthreads_or(failed)) goto done;
    if (issuer) pend_m = false;
    tc_fence_after();
    // dP (hi -> h buffer, lo -> D buffer; both consumed by the MMAs above)
    if (worker) masked_decay_tile(tq, bq::TM_DP, row, quad, half, b2s, p.scale, sm + bq::HS, sm + bq::DS);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (issuer) {
        tc_fence_after();
        // Y = dP K (K as MN-major B, N = dk);  Z = dP^T Q (dP as MN-major A)
        for (int part = 0; part < 2; ++part) {
            const uint32_t pb = part ? bq::DS : bq::HS;
            for (int ks = 0; ks < 8; ++ks) {
                umma_bf16(tmem + bq::TM_Y,
                          smem_desc(sb + pb + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                          smem_desc(sb + bq::K + ks * 1024, 8192, 512, kLayoutSW64),
                          idesc_bf16_f32(128, 96, 0, 1), (part | ks) > 0);
                umma_bf16(tmem + bq::TM_Z, smem_desc(sb + pb + ks * 2048, 16384, 1024, kLayoutSW128),
                          smem_desc(sb + bq::Q + ks * 1024, 8192, 512, kLayoutSW64),
                          idesc_bf16_f32(128, 96, 1, 1), (part | ks) > 0);
            }
        }
        umma_commit(bar_m);
        pend_m = true;
    }
    if (!mbar_wait(bar_m, 1, ctl)) failed = true;
    tc_fence_before();
    if (__syncthreads_or(failed)) goto done;
    if (issuer) pend_m = false;
    tc_fence_after();
    if (worker) {
        // epilogue: dq = scale e^{b} X + Y ; dk = Z + e^{gamma - b} W ; delta
        const float b2r = b2s[row];
        const float fq = p.scale * exp2f(b2r);
        const float fk = exp2f(b2s[127] - b2r);
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const int d0 = half * 48 + j * 16;
            uint32_t x[16], y[16], z[16], w[16];
            tmem_ld16(tq + bq::TM_X + d0, x);
            tmem_ld16(tq + bq::TM_Y + d0, y);
            tmem_ld16(tq + bq::TM_Z + d0, z);
            tmem_ld16(tq + bq::TM_W + d0, w);
            tmem_ld_wait();
            float dq[16], dk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                dq[e] = fmaf(fq, __uint_as_float(x[e]), __uint_as_float(y[e]));
                dk[e] = fmaf(fk, __uint_as_float(w[e]), __uint_as_float(z[e]));
                dsum = fmaf(bf16_at_sw64(sm + bq::Q, row, d0 + e), dq[e], dsum);
                dsum = fmaf(-bf16_at_sw64(sm + bq::K, row, d0 + e), dk[e], dsum);
            }
            // staging in the dO buffer: dq [3][128][32] SW64, dk right after
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                const int d = d0 + g * 8;
                const uint32_t off = (d >> 5) * 8192 + swz_off(row, (d & 31) >> 3, 64);
                *reinterpret_cast<uint4*>(sm + bq::DO + off) =
                    make_uint4(pack_bf16(dq[g * 8], dq[g * 8 + 1]), pack_bf16(dq[g * 8 + 2], dq[g * 8 + 3]),
                               pack_bf16(dq[g * 8 + 4], dq[g * 8 + 5]), pack_bf16(dq[g * 8 + 6], dq[g * 8 + 7]));
                *reinterpret_cast<uint4*>(sm + bq::DO + 24576 + off) =
                    make_uint4(pack_bf16(dk[g * 8], dk[g * 8 + 1]), pack_bf16(dk[g * 8 + 2], dk[g * 8 + 3]),
                               pack_bf16(dk[g * 8 + 4], dk[g * 8 + 5]), pack_bf16(dk[g * 8 + 6], dk[g * 8 + 7]));
            }
        }
        if (half) dpart[row] = dsum;
        fence_async_smem();
        tc_fence_before();
    }
    __syncthreads();
    if (worker && !half && t0 + row < p.T)
        p.delta[(static_cast<int64_t>(b) * p.T + t0 + row) * p.H + h] = dsum + dpart[row];
    if (issuer) {
        for (int i = 0; i < 3; ++i) {
            tma_store_4d(&p.tm_dq, sm + bq::DO + i * 8192, i * 32, h, t0, b);
            tma_store_4d(&p.tm_dk, sm + bq::DO + 24576 + i * 8192, i * 32, h, t0, b);
        }
        tma_store_commit();
    }
done:
    if (issuer) {
        if (pend_ld) mbar_wait(bar_ld, 0, ctl);
        if (pend_m) mbar_wait(bar_m, 0, ctl) && mbar_wait(bar_m, 1, ctl);
        tma_store_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ----------------------------------------------------------------- dv kernel
//
// One CTA per (batch, head, chunk, half of dv), 94 KB of shared memory and
// 256 TMEM columns, so two CTAs share an SM and overlap each other's loads,
// tensor work and CUDA-core work.  With gamma the chunk's total log-decay:
//
//   dv_j = e^{gamma - b_j} ( sum_{i >= j} P~_ji dO_i + k_j D )
//   P~_ji = scale e^{b_i - gamma} (k_j . q_i)          (factorised path)
//
// scores^T = K Q^T lands in TMEM with lanes = j; each thread turns its own
// lane's 64 columns in place into the bf16 hi and lo halves of P~ (P~ as the
// A operand of a tcgen05.mma straight from tensor memory), and k_j D shares
// the accumulator because both terms carry the same row factor.  Chunks whose
// decay spans more than 2^100 take the exact path: P_ji = scale
// e^{b_i - b_j} (k_j . q_i), K rows scaled by e^{gamma - b_j} in place before
// K D, row factor 1.
//
// TMEM tile layout of P~ for one lane: K (token i) block kb = i / 32 holds
// the hi words in columns 32 kb .. +15 and the lo words in 32 kb + 16 .. +31
// (two bf16 per 32-bit column, even index in the low half).

namespace bv {   // dv kernel shared-memory map
constexpr uint32_t Q = 0, K = 24576, DO = 49152, DS = 73728;   // DO [3][128][32], DS [3][96][32] SW64
constexpr uint32_t MISC = 92160;
constexpr uint32_t BYTES = MISC + 1024 + 1024;
constexpr uint32_t TM_T = 0, TM_DV = 128, TMEM_COLS = 256;
}  // namespace bv

__device__ __forceinline__ uint32_t ts_hi(uint32_t base, int ks)
{
    return base + 32 * (ks >> 1) + 8 * (ks & 1);
}

__global__ void __launch_bounds__(kThreadsBwd, 2) bwd_dv_kernel(const __grid_constant__ BwdParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(sm + bv::MISC);
    uint64_t* bar_m = bar_ld + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ld + 2);
    float* b2s = reinterpret_cast<float*>(sm + bv::MISC + 64);
    float* cfs = b2s + 128;                  // [128] column factors scale 2^{b_i - gamma}
    float* wsum = cfs + 128;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x >> 1, dvh = blockIdx.x & 1, h = blockIdx.y, b = blockIdx.z;
    const int unit = b * p.H + h;
    const int t0 = c * kChunk;
    const int quad = warp & 3, half = (warp >> 2) & 1, row = quad * 32 + lane;
    const bool worker = warp < 8;
    const bool issuer = warp == 8 && lane == 0;
    const WaitCtl ctl = p.ctl;
    const uint32_t idT = idesc_bf16_f32(128, 128, 0, 0);
    const uint32_t idV = idesc_bf16_f32(128, 96, 0, 1);

    if (issuer) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_m, 1);
        mbar_init_fence();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, bv::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tq = tmem_addr(tmem, quad * 32, 0);
    bool failed = false, pend_ld = false, pend_m = false;
    uint32_t mph = 0;

    if (issuer) {
        mbar_arrive_expect_tx(bar_ld, 2 * chunk::kTileQK + 24576 + 18432);
        for (int i = 0; i < 3; ++i) {
            tma_load_4d(sm + bv::Q + i * 8192, &p.tm_q, bar_ld, i * 32, h, t0, b);
            tma_load_4d(sm + bv::K + i * 8192, &p.tm_k, bar_ld, i * 32, h, t0, b);
            tma_load_4d(sm + bv::DO + i * 8192, &p.tm_do32, bar_ld, dvh * 96 + i * 32, h, t0, b);
            tma_load_3d(sm + bv::DS + i * 6144, &p.tm_d32, bar_ld, dvh * 96 + i * 32, 0, unit * p.NC + c);
        }
        pend_ld = true;
    }
    if (tid < 128) {
        const int t = t0 + tid;
        chunk_cumsum(t < p.T ? p.a[(static_cast<int64_t>(b) * p.T + t) * p.H + h] : 0.f, b2s, wsum, tid, warp,
                     lane);
    }
    __syncthreads();
    const float g2 = b2s[127];
    const bool fast = -g2 <= chunk::kFactorRange;
    if (tid < 128) cfs[tid] = p.scale * exp2f(b2s[tid] - g2);

    // group 1: scores^T = K Q^T; on the factorised path also dv = K D
    if (issuer) {
        if (mbar_wait(bar_ld, 0, ctl)) {
            pend_ld = false;
            tc_fence_after();
            for (int ks = 0; ks < 6; ++ks) {
                const uint32_t off = (ks >> 1) * 8192 + (ks & 1) * 32;
                const uint64_t ak = smem_desc(sb + bv::K + off, 16, 512, kLayoutSW64);
                umma_bf16(tmem + bv::TM_T, ak, smem_desc(sb + bv::Q + off, 16, 512, kLayoutSW64), idT, ks > 0);
                if (fast)
                    umma_bf16(tmem + bv::TM_DV, ak, smem_desc(sb + bv::DS + ks * 1024, 6144, 512, kLayoutSW64), idV,
                              ks > 0);
            }
            umma_commit(bar_m);
            pend_m = true;
        } else {
            failed = true;
        }
    }
    if (!mbar_wait(bar_m, mph, ctl)) failed = true;
    tc_fence_before();
    if (__syncthreads_or(failed)) goto done;
    tc_fence_after();
    if (issuer) pend_m = false;
    mph ^= 1;

    if (worker) {
        // P~ (hi, lo) in place in tensor memory, this lane's 64 columns
        const float b2j = b2s[row];
#pragma unroll
        for (int kb2 = 0; kb2 < 2; ++kb2) {
            const int i0 = half * 64 + kb2 * 32;
            const uint32_t col = bv::TM_T + i0;
            uint32_t hi[16], lo[16];
            if (i0 + 31 < quad * 32) {            // every i < j here: masked
#pragma unroll
                for (int e = 0; e < 16; ++e) hi[e] = lo[e] = 0u;
            } else {
                uint32_t r[32];
                tmem_ld32(tq + col, r);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int i = i0 + e;
                    float v0, v1;
                    if (fast) {
                        v0 = (i >= row) ? __uint_as_float(r[e]) * cfs[i] : 0.f;
                        v1 = (i + 1 >= row) ? __uint_as_float(r[e + 1]) * cfs[i + 1] : 0.f;
                    } else {
                        v0 = (i >= row) ? p.scale * __uint_as_float(r[e]) * exp2f(b2s[i] - b2j) : 0.f;
                        v1 = (i + 1 >= row) ? p.scale * __uint_as_float(r[e + 1]) * exp2f(b2s[i + 1] - b2j) : 0.f;
                    }
                    const uint32_t hv = pack_bf16(v0, v1);
                    hi[e / 2] = hv;
                    lo[e / 2] = pack_bf16(v0 - bf16_lo(hv), v1 - bf16_hi(hv));
                }
            }
            tmem_st16(tq + col, hi);
            tmem_st16(tq + col + 16, lo);
        }
        tmem_st_wait();
        if (!fast) {
            // exact path: K rows scaled by e^{gamma - b_j} in place for K D
            for (int idx = tid; idx < 384; idx += 256) {
                const int r = idx & 127, blk = idx >> 7;
                chunk::scale_row_sw64(sm + bv::K, r, blk, exp2f(g2 - b2s[r]));
            }
            fence_async_smem();
        }
    }
    tc_fence_before();
    __syncthreads();

    // group 2: (exact path: dv = K~ D) ; dv += P~ dO  (A from tensor memory)
    if (issuer) {
        tc_fence_after();
        if (!fast)
            for (int ks = 0; ks < 6; ++ks) {
                const uint32_t off = (ks >> 1) * 8192 + (ks & 1) * 32;
                umma_bf16(tmem + bv::TM_DV, smem_desc(sb + bv::K + off, 16, 512, kLayoutSW64),
                          smem_desc(sb + bv::DS + ks * 1024, 6144, 512, kLayoutSW64), idV, ks > 0);
            }
        for (int part = 0; part < 2; ++part)
            for (int ks = 0; ks < 8; ++ks)
                umma_bf16_ts(tmem + bv::TM_DV, tmem + ts_hi(bv::TM_T, ks) + 16 * part,
                             smem_desc(sb + bv::DO + ks * 1024, 8192, 512, kLayoutSW64), idV, 1);
        umma_commit(bar_m);
        pend_m = true;
    }
    if (!mbar_wait(bar_m, mph, ctl)) failed = true;
    tc_fence_before();
    if (__syncthreads_or(failed)) goto done;
    tc_fence_after();
    if (issuer) pend_m = false;
    if (worker) {
        // epilogue: dv_j = f_j acc_j -> staging [3][128][32] SW64 in the dO buffer
        const float f = fast ? exp2f(g2 - b2s[row]) : 1.0f;
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const int n0 = half * 48 + j * 16;
            uint32_t u[16];
            tmem_ld16(tq + bv::TM_DV + n0, u);
            tmem_ld_wait();
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                const int n = n0 + g * 8;
                uint32_t pk[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    pk[e] = pack_bf16(f * __uint_as_float(u[g * 8 + 2 * e]), f * __uint_as_float(u[g * 8 + 2 * e + 1]));
                *reinterpret_cast<uint4*>(sm + bv::DO + (n >> 5) * 8192 + swz_off(row, (n & 31) >> 3, 64)) =
                    make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
        }
        fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (issuer) {
        for (int i = 0; i < 3; ++i)
            tma_store_4d(&p.tm_dv32, sm + bv::DO + i * 8192, dvh * 96 + i * 32, h, t0, b);
        tma_store_commit();
    }
done:
    if (issuer) {
        if (pend_ld) mbar_wait(bar_ld, 0, ctl);
        if (pend_m) mbar_wait(bar_m, mph, ctl);
        tma_store_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, bv::TMEM_COLS);
}

// ------------------------------------------------------------------ da scan
//
// da_t = sum_{m >= t} delta_m + <dS_T, S_T>, one CTA per (batch, head):
// each thread sums a contiguous span of tokens, the CTA scans the span
// totals from the end, then every thread rewrites its span.

constexpr int kScanThreads = 256;

__global__ void __launch_bounds__(kScanThreads) da_scan_kernel(float* __restrict__ da,
                                                               const float* __restrict__ dsT,
                                                               const float* __restrict__ sT,
                                                               int T, int H)
{
    __shared__ float tot[kScanThreads];
    __shared__ float red[kScanThreads / 32];
    const int unit = blockIdx.x;
    const int b = unit / H, h = unit - b * H;
    const int tid = threadIdx.x;
    float* col = da + static_cast<int64_t>(b) * T * H + h;
    float base = 0.f;
    if (dsT) {
        float s = 0.f;
        for (int64_t e = tid; e < kSS; e += kScanThreads) s = fmaf(dsT[unit * kSS + e], sT[unit * kSS + e], s);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if ((tid & 31) == 0) red[tid >> 5] = s;
        __syncthreads();
        for (int i = 0; i < kScanThreads / 32; ++i) base += red[i];
    }
    const int span = (T + kScanThreads - 1) / kScanThreads;
    const int lo = tid * span, hi = min(T, lo + span);
    float s = 0.f;
    for (int t = lo; t < hi; ++t) s += col[static_cast<int64_t>(t) * H];
    tot[tid] = s;
    __syncthreads();
    float after = base;   // sum of all spans after this one
    for (int i = tid + 1; i < kScanThreads; ++i) after += tot[i];
    for (int t = hi - 1; t >= lo; --t) {
        after += col[static_cast<int64_t>(t) * H];
        col[static_cast<int64_t>(t) * H] = after;
    }
}

template <typename K>
gla_status launch_bwd_kernel(K kernel, uint32_t bytes, const BwdParams& p, dim3 grid, cudaStream_t st,
                             const char* name)
{
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return check_launch(name);
    trace_begin(st);
    kernel<<<grid, kThreadsBwd, bytes, st>>>(p);
    trace_end(st, name);
    count_launch();
    return check_launch(name);
}

}  // namespace

size_t bwd_workspace_bytes(int B, int T, int H)
{
    const size_t units = static_cast<size_t>(B) * H, NC = num_chunks(T);
    const size_t states = align256(units * NC * kSS * 2);
    return 2 * states + align256(units * kSS * sizeof(float));
}

gla_status run_chunk_bwd(const ChunkProblem& pr, const float* s0, const void* dO,
                         const float* ds_final, void* dq, void* dk, void* dv, float* da,
                         float* ds0, void* ws, size_t ws_bytes, const WaitCtl& ctl,
                         cudaStream_t st)
{
    (void)ws_bytes;
    const int units = pr.B * pr.H, NC = num_chunks(pr.T);
    const size_t states = align256(static_cast<size_t>(units) * NC * kSS * 2);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    void* hbuf = wsb;
    void* dbuf = wsb + states;
    float* sT = reinterpret_cast<float*>(wsb + 2 * states);
    const int64_t ldo = static_cast<int64_t>(pr.H) * kDv;
    gla_status s;

    // 1. h_c for every chunk (and S_T when dS_T is given)
    StateParams sp;
    memset(&sp, 0, sizeof(sp));
    if ((s = make_token_map(&sp.tm_u, pr.k, kDk, pr.H, pr.T, pr.B, pr.ld_qk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&sp.tm_y, pr.v, kDv, pr.H, pr.T, pr.B, pr.ld_v, 64, 128)) != GLA_OK) return s;
    if ((s = make_state_map(&sp.tm_h, hbuf, static_cast<int64_t>(units) * NC)) != GLA_OK) return s;
    sp.a = pr.a;
    sp.s_init = s0;
    sp.init_unit_stride = kSS;
    sp.s_out = ds_final ? sT : nullptr;
    sp.out_unit_stride = kSS;
    sp.out_last_only = 1;
    sp.B = pr.B;
    sp.T = pr.T;
    sp.H = pr.H;
    sp.NC = NC;
    sp.chunks_per_seg = NC;
    sp.store_h = 1;
    sp.scale = pr.scale;
    sp.ctl = ctl;
    if ((s = launch_state_kernel(false, false, sp, dim3(1, pr.H, pr.B), st)) != GLA_OK) return s;

    // 2. D_c for every chunk, dS_0
    StateParams rp = sp;
    if ((s = make_token_map(&rp.tm_u, pr.q, kDk, pr.H, pr.T, pr.B, pr.ld_qk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&rp.tm_y, dO, kDv, pr.H, pr.T, pr.B, ldo, 64, 128)) != GLA_OK) return s;
    if ((s = make_state_map(&rp.tm_h, dbuf, static_cast<int64_t>(units) * NC)) != GLA_OK) return s;
    rp.s_init = ds_final;
    rp.s_out = ds0;
    if ((s = launch_state_kernel(false, true, rp, dim3(1, pr.H, pr.B), st)) != GLA_OK) return s;

    // 3. dq, dk (+ per-token delta into da) and dv
    BwdParams bp;
    memset(&bp, 0, sizeof(bp));
    const int64_t ldk = static_cast<int64_t>(pr.H) * kDk;
    if ((s = make_token_map(&bp.tm_q, pr.q, kDk, pr.H, pr.T, pr.B, pr.ld_qk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&bp.tm_k, pr.k, kDk, pr.H, pr.T, pr.B, pr.ld_qk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&bp.tm_v, pr.v, kDv, pr.H, pr.T, pr.B, pr.ld_v, 64, 128)) != GLA_OK) return s;
    if ((s = make_token_map(&bp.tm_do, dO, kDv, pr.H, pr.T, pr.B, ldo, 64, 128)) != GLA_OK) return s;
    if ((s = make_token_map(&bp.tm_dq, dq, kDk, pr.H, pr.T, pr.B, ldk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&bp.tm_dk, dk, kDk, pr.H, pr.T, pr.B, ldk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&bp.tm_dv, dv, kDv, pr.H, pr.T, pr.B, ldo, 64, 128)) != GLA_OK) return s;
    if ((s = make_state_map(&bp.tm_h, hbuf, static_cast<int64_t>(units) * NC)) != GLA_OK) return s;
    if ((s = make_state_map(&bp.tm_d, dbuf, static_cast<int64_t>(units) * NC)) != GLA_OK) return s;
    if ((s = make_token_map(&bp.tm_do32, dO, kDv, pr.H, pr.T, pr.B, ldo, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&bp.tm_dv32, dv, kDv, pr.H, pr.T, pr.B, ldo, 32, 64)) != GLA_OK) return s;
    if ((s = make_state_map(&bp.tm_d32, dbuf, static_cast<int64_t>(units) * NC, 32)) != GLA_OK) return s;
    bp.a = pr.a;
    bp.delta = da;
    bp.B = pr.B;
    bp.T = pr.T;
    bp.H = pr.H;
    bp.NC = NC;
    bp.scale = pr.scale;
    bp.ctl = ctl;
    const dim3 grid(NC, pr.H, pr.B);
    if ((s = launch_bwd_kernel(bwd_dqdk_kernel, bq::BYTES, bp, grid, st, "bwd_dqdk_kernel")) != GLA_OK) return s;
    if ((s = launch_bwd_kernel(bwd_dv_kernel, bv::BYTES, bp, dim3(2 * NC, pr.H, pr.B), st, "bwd_dv_kernel")) != GLA_OK)
        return s;

    // 4. da = reverse cumulative sum of delta (+ <dS_T, S_T>)
    trace_begin(st);
    da_scan_kernel<<<units, kScanThreads, 0, st>>>(da, ds_final, ds_final ? sT : nullptr, pr.T, pr.H);
    trace_end(st, "da_scan_kernel");
    count_launch();
    return check_launch("da_scan_kernel");
}

}  // namespace gla
