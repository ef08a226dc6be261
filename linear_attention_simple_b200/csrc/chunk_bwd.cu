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
//   1. state kernel, forward, state-only: h_c for every chunk (bf16 hi + lo
//      planes), and S_T when an upstream dS_T is given -- skipped when the
//      forward kept the states (gla_chunk_fwd_train / gla_chunk_bwd_saved);
//   2. the reverse sweep with dv fused in (the fused forward kernel run
//      backwards, chunk_state.cuh): D_c for every chunk (hi + lo), dS_0 =
//      D_{-1}, and dv = P^T dO + diag(e^{gamma - b}) K D (after a state-only
//      reverse pre-pass and a fold when a head's chunks are cut into
//      segments);
//   3. bwd_dqdk_persistent_kernel (dq and dk of a chunk in one CTA, one CTA
//      per SM), tcgen05 for every contraction; the masked, decayed dP tiles
//      stay in tensor memory as bf16 hi + lo and feed the next MMA from
//      there; the epilogues also emit q.dq and k.dk per token and per chunk;
//   4. da_finish_kernel: reverse cumulative sum over T (plus <dS_T, S_T>
//      from state_dot_kernel when dS_T is given), restarted every 16 chunks
//      from the closed form <dS_a, S_a> (da_anchor_kernel).
#include <cstring>
#include <type_traits>

#include "chunk_state.cuh"

namespace gla {
namespace {

constexpr int64_t kSS = static_cast<int64_t>(kDk) * kDv;
constexpr float kLog2e = 1.4426950408889634f;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
int num_chunks(int T) { return (T + kChunk - 1) / kChunk; }

struct BwdParams {
    CUtensorMap tm_q, tm_k;                // q, k tiles (32-column SW64 boxes)
    CUtensorMap tm_dq, tm_dk;              // gradient stores
    // 32-column SW64 boxes: dO, v; per-chunk states [units*NC][2][96][192]
    // (plane 0 hi, plane 1 lo) h and D, a state's two planes in one box
    CUtensorMap tm_do32, tm_v32, tm_h2, tm_d2;
    const float* a;
    float* delta;                          // [B*H, T]: q.dq per token (role 0), k.dk (role 1) after it
    float* ctot;                           // [B*H, NC, 2]: chunk totals of both halves
    int B, T, H, NC;
    float scale;
    WaitCtl ctl;
};




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

// TMEM column of the hi words of K step ks (16 tokens) of a tile kept as
// [32-token block: 16 hi columns, 16 lo columns]; the lo words are 16 further.
__device__ __forceinline__ uint32_t ts_hi(uint32_t base, int ks)
{
    return base + 32 * (ks >> 1) + 8 * (ks & 1);
}

// ------------------------------------------------------------ dq, dk kernel
//
// With gamma the chunk's total log-decay and T the masked tile of the dO / V
// products:
//
//   dq_i = s e^{b_i} ( dO_i h^T + sum_{j <= i} (dO_i . v_j) e^{-b_j} k_j )
//   dk_j = e^{gamma - b_j} ( v_j D^T + sum_{i >= j} s e^{b_i - gamma} (v_j . dO_i) q_i )
//
// The contraction over dv (T_q = dO V^T, T_k = V dO^T and the state products)
// streams in six 32-column slices; each slice carries h and D as their bf16
// hi and lo planes, both multiplied into the accumulators, so the state
// products keep the fp32 states' precision (q.dq and k.dk, and through them
// da, are sums that cancel to a small fraction of their terms).  The T tiles
// are then turned in place, in tensor memory, into the bf16 hi and lo halves
// of the decayed tiles and used as A operands against K (dq) and Q (dk); the
// row factors are applied in the epilogues.  Chunks whose decay spans more
// than 2^100 take the exact path: the tiles carry s e^{b_i - b_j}, the state
// products are scaled in place by the row factors first, row factor 1.  Each
// gradient also yields its half of the per-token delta of the da sum, q.dq
// or k.dk, and that half's chunk total.
//
// Persistent: both gradients of a chunk in one CTA, one CTA per SM walking
// the chunks blockIdx.x, + gridDim.x, ...: every input of a chunk is read
// into the SM once, and the next chunk's loads run under this chunk's
// conversion and epilogues.
//
//   producer warp   per chunk: the six dv slices into the ring as slots
//                   free, then Q and K once the previous chunk is done with
//                   them; every slice carries dO, V and the hi / lo planes
//                   of h and D (40 KB)
//   issuer thread   per slice: T_q += dO V^T, T_k += V dO^T, A_q += dO h^T
//                   (hi, lo), A_k += V D^T (hi, lo); then, once the tiles
//                   are converted and Q, K are in, A_q += dP K and
//                   A_k += dP^T Q (A from tensor memory, hi and lo)
//   workers 0-7     T_q -> dP in place (bf16 hi + lo), the dq epilogue and
//                   q.dq; workers 8-15 the same for T_k -> dP^T, dk, k.dk
// Tensor memory: T_q at 0, A_q at 128, T_k at 256, A_k at 384 (448 of 512
// columns): one chunk at a time, so a chunk's slice MMAs start once the
// previous chunk's accumulators are in the workers' registers (the "acc"
// barrier, at the start of the epilogue; the producer's next q, k load waits
// for the end of it, the "free" barrier).

// (A 4-slot ring, the gradients staged in place over the q, k tiles to make
// room, measured slower: 166 against 159 us per launch; the next chunk's
// q, k load then waits for each store to read its tile.)
namespace bqp {   // persistent dq / dk kernel shared-memory map
constexpr uint32_t SLOT = 40960;    // dO [128][32] | V [128][32] | h hi, lo | D hi, lo [96][32], SW64
constexpr uint32_t S_V = 8192, S_HH = 16384, S_HL = 22528, S_DH = 28672, S_DL = 34816;
constexpr int kSlots = 3, kSlices = 6;
constexpr uint32_t QT = kSlots * SLOT;          // q tile [3][128][32] SW64
constexpr uint32_t KT = QT + 24576;             // k tile
constexpr uint32_t SQ = KT + 24576;             // dq staging [3][128][32]
constexpr uint32_t SK = SQ + 24576;             // dk staging
constexpr uint32_t MISC = SK + 24576;          // barriers, tmem slot, decays, delta partials: 4,288 B
constexpr uint32_t BYTES = MISC + 4608 + 1024;
constexpr uint32_t TM_TQ = 0, TM_AQ = 128, TM_TK = 256, TM_AK = 384, TMEM_COLS = 512;
constexpr uint32_t kSliceBytes = 2 * 8192 + 4 * 6144;
constexpr int kWorkers = 512;
constexpr int kThreads = kWorkers + 64;
}  // namespace bqp

__global__ void __launch_bounds__(bqp::kThreads, 1) bwd_dqdk_persistent_kernel(const __grid_constant__ BwdParams p)
{
    using namespace bqp;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bar_full = reinterpret_cast<uint64_t*>(sm + MISC);   // [3] slot loaded
    uint64_t* bar_empty = bar_full + 3;                           // [3] slot's MMAs done
    uint64_t* bar_qk = bar_full + 6;                              // q, k tiles loaded
    uint64_t* bar_sl = bar_full + 7;                              // a chunk's slice MMAs done
    uint64_t* bar_cv = bar_full + 8;                              // both tiles converted (512)
    uint64_t* bar_tl = bar_full + 9;                              // tile MMAs done
    uint64_t* bar_free = bar_full + 10;                           // q, k tiles read (512)
    uint64_t* bar_acc = bar_full + 11;                            // accumulators read out of TMEM (512)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_full + 12);
    float* b2s = reinterpret_cast<float*>(sm + MISC + 128);       // [2][128] by chunk parity
    float* cfq = b2s + 256;                                       // [2][128] 2^{-b_j}
    float* cfk = cfq + 256;                                       // [2][128] s 2^{b_i - gamma}
    float* wsum = cfk + 256;                                      // [8]
    float* dpart = wsum + 8;                                      // [2][128] delta partial of column half 1
    float* rsum = dpart + 256;                                    // [2][4] chunk-total partials

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool worker = warp < 16;
    const bool issuer = warp == 16 && lane == 0;
    const bool producer = warp == 17 && lane == 0;
    const int role = (warp >> 3) & 1;                    // workers: 0 dq, 1 dk
    const int quad = warp & 3, half = (warp >> 2) & 1, row = quad * 32 + lane;
    const int wtid = tid & 255;                          // thread index within the role's 256
    const WaitCtl ctl = p.ctl;

    const int total = p.B * p.H * p.NC;
    const int first = blockIdx.x, stride = gridDim.x;
    const int n = first < total ? (total - first + stride - 1) / stride : 0;
    struct Item {
        int b, h, c, unit;
    };
    // chunk-major from chunk 0: the reverse state pass that runs just before
    // ends on the first chunks of every sequence, so the first items find
    // their D_c and q, dO tiles still in L2
    const int units = p.B * p.H;
    auto item = [&](int k) {
        const int it = first + k * stride;
        Item r;
        r.c = it / units;
        r.unit = it - r.c * units;
        r.b = r.unit / p.H;
        r.h = r.unit - r.b * p.H;
        return r;
    };

    if (issuer) {
        for (int i = 0; i < 12; ++i) mbar_init(bar_full + i, (i == 8 || i >= 10) ? kWorkers : 1);
        mbar_init_fence();
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_do32);
        tma_prefetch_desc(&p.tm_v32);
        tma_prefetch_desc(&p.tm_h2);
        tma_prefetch_desc(&p.tm_d2);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (producer) {
        // ----------------------------------------------------------- loads
        int n_full[kSlots] = {0, 0, 0}, n_qk = 0, sidx = 0;
        bool ok = true;
        auto load_slice = [&](const Item& w, int sl) {
            const int slot = sidx % kSlots;
            if (sidx >= kSlots && !mbar_wait(bar_empty + slot, ((sidx - kSlots) / kSlots) & 1, ctl)) return false;
            uint8_t* base = sm + slot * SLOT;
            const int t0 = w.c * kChunk, si = (w.unit * p.NC + w.c) * 2;
            mbar_arrive_expect_tx(bar_full + slot, kSliceBytes);
            tma_load_4d(base, &p.tm_do32, bar_full + slot, sl * 32, w.h, t0, w.b);
            tma_load_4d(base + S_V, &p.tm_v32, bar_full + slot, sl * 32, w.h, t0, w.b);
            tma_load_3d(base + S_HH, &p.tm_h2, bar_full + slot, sl * 32, 0, si);   // hi, then lo at S_HL
            tma_load_3d(base + S_DH, &p.tm_d2, bar_full + slot, sl * 32, 0, si);   // hi, then lo at S_DL
            ++n_full[slot];
            ++sidx;
            return true;
        };
        for (int k = 0; ok && k < n; ++k) {
            const Item w = item(k);
            // the slices first: they wait only for ring slots, and the slice
            // MMAs need nothing else
            for (int sl = 0; ok && sl < kSlices; ++sl) ok = load_slice(w, sl);
            // q, k of this chunk (needed from the tile MMAs on) once the
            // previous chunk's epilogue has read its tiles
            if (ok && k >= 1 && !mbar_wait(bar_free, (k - 1) & 1, ctl)) ok = false;
            if (ok) {
                const int t0 = w.c * kChunk;
                mbar_arrive_expect_tx(bar_qk, 2 * 24576);
                for (int i = 0; i < 3; ++i) {
                    tma_load_4d(sm + QT + i * 8192, &p.tm_q, bar_qk, i * 32, w.h, t0, w.b);
                    tma_load_4d(sm + KT + i * 8192, &p.tm_k, bar_qk, i * 32, w.h, t0, w.b);
                }
                ++n_qk;
            }
        }
        // at most one load per barrier is ever outstanding
        for (int i = 0; i < kSlots; ++i)
            if (n_full[i]) mbar_wait(bar_full + i, (n_full[i] - 1) & 1, ctl);
        if (n_qk) mbar_wait(bar_qk, (n_qk - 1) & 1, ctl);
    } else if (issuer) {
        // ------------------------------------------------------------ MMAs
        const uint32_t idT = idesc_bf16_f32(128, 128, 0, 0), idA = idesc_bf16_f32(128, 96, 0, 0);
        const uint32_t idB = idesc_bf16_f32(128, 96, 0, 1);
        int n_empty[kSlots] = {0, 0, 0}, n_sl = 0, n_tl = 0, sidx = 0;
        bool ok = true;
        for (int k = 0; ok && k < n; ++k) {
            // the previous chunk's accumulators have been read out
            if (k >= 1 && !mbar_wait(bar_acc, (k - 1) & 1, ctl)) break;
            tc_fence_after();
            for (int sl = 0; sl < kSlices; ++sl, ++sidx) {
                const int slot = sidx % kSlots;
                if (!mbar_wait(bar_full + slot, (sidx / kSlots) & 1, ctl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t base = sb + slot * SLOT;
                const uint64_t ddo = smem_desc(base, 16, 512, kLayoutSW64);
                const uint64_t dv = smem_desc(base + S_V, 16, 512, kLayoutSW64);
                const uint64_t dhh = smem_desc(base + S_HH, 16, 512, kLayoutSW64);
                const uint64_t dhl = smem_desc(base + S_HL, 16, 512, kLayoutSW64);
                const uint64_t ddh = smem_desc(base + S_DH, 16, 512, kLayoutSW64);
                const uint64_t ddl = smem_desc(base + S_DL, 16, 512, kLayoutSW64);
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    const uint32_t o = ks * 32, acc = (sl | ks) > 0;
                    umma_bf16(tmem + TM_TQ, desc_add(ddo, o), desc_add(dv, o), idT, acc);
                    umma_bf16(tmem + TM_TK, desc_add(dv, o), desc_add(ddo, o), idT, acc);
                    umma_bf16(tmem + TM_AQ, desc_add(ddo, o), desc_add(dhh, o), idA, acc);
                    umma_bf16(tmem + TM_AQ, desc_add(ddo, o), desc_add(dhl, o), idA, 1);
                    umma_bf16(tmem + TM_AK, desc_add(dv, o), desc_add(ddh, o), idA, acc);
                    umma_bf16(tmem + TM_AK, desc_add(dv, o), desc_add(ddl, o), idA, 1);
                }
                umma_commit(bar_empty + slot);
                ++n_empty[slot];
            }
            if (!ok) break;
            umma_commit(bar_sl);
            ++n_sl;
            // the tiles: dP (hi, lo) against K, dP^T against Q
            if (!mbar_wait(bar_cv, k & 1, ctl) || !mbar_wait(bar_qk, k & 1, ctl)) break;
            tc_fence_after();
            const uint64_t dk = smem_desc(sb + KT, 8192, 512, kLayoutSW64);
            const uint64_t dq = smem_desc(sb + QT, 8192, 512, kLayoutSW64);
#pragma unroll
            for (int part = 0; part < 2; ++part)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    umma_bf16_ts(tmem + TM_AQ, tmem + ts_hi(TM_TQ, ks) + 16 * part, desc_add(dk, ks * 1024), idB, 1);
                    umma_bf16_ts(tmem + TM_AK, tmem + ts_hi(TM_TK, ks) + 16 * part, desc_add(dq, ks * 1024), idB, 1);
                }
            umma_commit(bar_tl);
            ++n_tl;
        }
        // every commit's arrival has landed before the barriers go away
        for (int i = 0; i < kSlots; ++i)
            if (n_empty[i]) mbar_wait(bar_empty + i, (n_empty[i] - 1) & 1, ctl);
        if (n_sl) mbar_wait(bar_sl, (n_sl - 1) & 1, ctl);
        if (n_tl) mbar_wait(bar_tl, (n_tl - 1) & 1, ctl);
    } else if (worker) {
        // --------------------------------------------------------- workers
        const uint32_t tq = tmem_addr(tmem, quad * 32, 0);
        const uint32_t TT = role ? TM_TK : TM_TQ, TA = role ? TM_AK : TM_AQ;
        uint8_t* stg = sm + (role ? SK : SQ);
        const uint8_t* dot = sm + (role ? KT : QT);      // partner of the delta dot: k (dk) or q (dq)
        float* dp = dpart + role * 128;
        bool ok = true;
        for (int k = 0; ok && k < n; ++k) {
            const Item w = item(k);
            const int par = k & 1, t0 = w.c * kChunk;
            float* bz = b2s + par * 128;
            // decays of this chunk (warps 0-3); the buffers of parity par were
            // last read by chunk k-2, finished before chunk k-1's barriers
            if (tid < 128) {
                const int t = t0 + tid;
                chunk_cumsum(t < p.T ? p.a[(static_cast<int64_t>(w.b) * p.T + t) * p.H + w.h] : 0.f, bz, wsum, tid,
                             warp, lane);
                const float g2 = ((wsum[0] + wsum[1]) + wsum[2]) + wsum[3];
                cfq[par * 128 + tid] = exp2f(-bz[tid]);
                cfk[par * 128 + tid] = p.scale * exp2f(bz[tid] - g2);
            }
            chunk::named_sync(2, kWorkers);
            const float g2 = bz[127];
            const bool fast = -g2 <= chunk::kFactorRange;
            const float* cfs = (role ? cfk : cfq) + par * 128;
            const float b2r = bz[row];
            const float rowf = role ? exp2f(g2 - b2r) : p.scale * exp2f(b2r);

            // T -> decayed tile (hi, lo) in place; on the exact path also the
            // state product's row factor
            const bool got = mbar_wait(bar_sl, k & 1, ctl);
            if (chunk::bar_or(2, kWorkers, !got)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int kb2 = 0; kb2 < 2; ++kb2) {
                const int c0 = half * 64 + kb2 * 32;
                const uint32_t col = TT + c0;
                const bool dead = role ? (c0 + 31 < quad * 32) : (c0 > quad * 32 + 31);
                uint32_t hi[16], lo[16];
                if (dead) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) hi[e] = lo[e] = 0u;
                } else {
                    uint32_t r[32];
                    tmem_ld32(tq + col, r);
                    tmem_ld_wait();
                    // one loop per path (factorised or exact) and gradient, so
                    // that no element computes the factor of the other path
                    auto convert = [&](auto role_tag, auto fast_tag) {
                        constexpr bool DK = decltype(role_tag)::value, FAST = decltype(fast_tag)::value;
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            float v[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const int cc = c0 + e + u;
                                const bool keep = DK ? (cc >= row) : (cc <= row);
                                const float f = FAST ? cfs[cc] : p.scale * exp2f(DK ? bz[cc] - b2r : b2r - bz[cc]);
                                v[u] = keep ? __uint_as_float(r[e + u]) * f : 0.f;
                            }
                            const uint32_t hv = pack_bf16(v[0], v[1]);
                            hi[e / 2] = hv;
                            lo[e / 2] = pack_bf16(v[0] - bf16_lo(hv), v[1] - bf16_hi(hv));
                        }
                    };
                    if (role) {
                        if (fast) convert(std::true_type{}, std::true_type{});
                        else convert(std::true_type{}, std::false_type{});
                    } else {
                        if (fast) convert(std::false_type{}, std::true_type{});
                        else convert(std::false_type{}, std::false_type{});
                    }
                }
                tmem_st16(tq + col, hi);
                tmem_st16(tq + col + 16, lo);
            }
            if (!fast) {
#pragma unroll
                for (int j = 0; j < 3; ++j) {
                    const uint32_t col = TA + half * 48 + j * 16;
                    uint32_t u[16];
                    tmem_ld16(tq + col, u);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 16; ++e) u[e] = __float_as_uint(rowf * __uint_as_float(u[e]));
                    tmem_st16(tq + col, u);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(bar_cv);

            // epilogue: out = f acc -> staging; delta partial against q or k
            const bool got2 = mbar_wait(bar_tl, k & 1, ctl);
            if (wtid == 0) tma_store_wait_read();      // the staging's previous store has read it
            if (chunk::bar_or(2, kWorkers, !got2)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float f = fast ? rowf : 1.0f;
            uint32_t u[3][16];
#pragma unroll
            for (int j = 0; j < 3; ++j) tmem_ld16(tq + TA + half * 48 + j * 16, u[j]);
            tmem_ld_wait();
            // the accumulators are in registers: the next chunk's MMAs may start
            tc_fence_before();
            mbar_arrive(bar_acc);
            float dsum = 0.f;
#pragma unroll
            for (int j = 0; j < 3; ++j) {
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    const int nn = half * 48 + j * 16 + g * 8;
                    const uint32_t off = (nn >> 5) * 8192 + swz_off(row, (nn & 31) >> 3, 64);
                    const uint4 wv4 = *reinterpret_cast<const uint4*>(dot + off);
                    const uint32_t wv[4] = {wv4.x, wv4.y, wv4.z, wv4.w};
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float x0 = f * __uint_as_float(u[j][g * 8 + 2 * e]);
                        const float x1 = f * __uint_as_float(u[j][g * 8 + 2 * e + 1]);
                        dsum = fmaf(bf16_lo(wv[e]), x0, dsum);
                        dsum = fmaf(bf16_hi(wv[e]), x1, dsum);
                        pk[e] = pack_bf16(x0, x1);
                    }
                    *reinterpret_cast<uint4*>(stg + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
            // the q, k tiles are read: the producer may load the next chunk's
            mbar_arrive(bar_free);
            if (half) dp[row] = dsum;
            fence_async_smem();
            chunk::named_sync(3 + role, 256);
            if (!half) {
                const bool live = t0 + row < p.T;
                float x = live ? dsum + dp[row] : 0.f;
                if (live && GLA_DCHECK(w.unit < p.B * p.H && w.c < p.NC, ctl.status))
                    p.delta[(static_cast<int64_t>(role) * p.B * p.H + w.unit) * p.T + t0 + row] = x;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                if (lane == 0) rsum[role * 4 + quad] = x;
            }
            chunk::named_sync(3 + role, 256);
            if (wtid == 0) {
                if (GLA_DCHECK(w.unit < p.B * p.H && w.c < p.NC, ctl.status))
                    p.ctot[(static_cast<int64_t>(w.unit) * p.NC + w.c) * 2 + role] =
                        ((rsum[role * 4] + rsum[role * 4 + 1]) + rsum[role * 4 + 2]) + rsum[role * 4 + 3];
                const CUtensorMap* tm_out = role ? &p.tm_dk : &p.tm_dq;
                for (int i = 0; i < 3; ++i) tma_store_4d(tm_out, stg + i * 8192, i * 32, w.h, t0, w.b);
                tma_store_commit();
            }
        }
        if (wtid == 0) tma_store_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

// ------------------------------------------------------------------ da
//
// da_t = sum_{m >= t} (q_m . dq_m - k_m . dk_m) + <dS_T, S_T>.  One CTA of
// 128 threads per (chunk, batch x head): the reverse inclusive scan of the
// chunk's own tokens, plus the totals of the later chunks up to the next
// anchor, plus the anchor's value.
//
// Anchors.  Each chunk total carries the rounding of the bf16 state copies
// the gradient kernels read, and a sum over every later chunk would let that
// error grow like sqrt(T).  The sum over all tokens after chunk a has a
// closed form, <dS_a, S_a> (the gradient of the state after chunk a with that
// state: the same identity that gives <dS_T, S_T> for the tokens after T), so
// every kDaAnchor chunks the sum restarts from that inner product
// (da_anchor_kernel).  The last anchor is the dS_T term that state_dot_kernel
// wrote per (batch, head), or zero.

constexpr int kDaThreads = 128;
constexpr int kDaAnchor = 16;      // chunks between anchors (2,048 tokens)

__host__ __device__ inline int da_anchors(int NC) { return (NC - 1) / kDaAnchor; }

__global__ void __launch_bounds__(kDaThreads) da_finish_kernel(float* __restrict__ da,
                                                               const float* __restrict__ delta,
                                                               const float* __restrict__ ctot,
                                                               const float* __restrict__ base,
                                                               const float* __restrict__ anchor, int T, int H,
                                                               int NC, int units, int* __restrict__ status)
{
    __shared__ float wtot[kDaThreads / 32], wsuf[kDaThreads / 32];
    const int unit = blockIdx.x, c = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t = c * kChunk + tid;
    const float* cu = ctot + static_cast<int64_t>(unit) * NC * 2;
    // chunks c+1 .. last are summed; the anchor after `last` closes the sum
    const int na = da_anchors(NC), j = c / kDaAnchor;
    const int last = j < na ? (j + 1) * kDaAnchor - 1 : NC - 1;
    float suf = 0.f;
    for (int cc = c + 1 + tid; cc <= last; cc += kDaThreads) suf += cu[2 * cc] - cu[2 * cc + 1];
    float x = 0.f;
    if (t < T) x = delta[static_cast<int64_t>(unit) * T + t] - delta[(static_cast<int64_t>(units) + unit) * T + t];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += y;
        suf += __shfl_xor_sync(0xffffffffu, suf, o);
    }
    if (lane == 0) {
        wtot[warp] = x;
        wsuf[warp] = suf;
    }
    __syncthreads();
    float add = j < na ? anchor[static_cast<int64_t>(unit) * na + j] : (base ? base[unit] : 0.f);
    for (int w = 0; w < kDaThreads / 32; ++w) {
        add += wsuf[w];
        if (w > warp) add += wtot[w];
    }
    if (t < T && GLA_DCHECK(unit < units && c < NC, status)) da[(static_cast<int64_t>(unit / H) * T + t) * H + unit % H] = x + add;
}

// Both inner products below are a few hundred KB per CTA at most, read by
// 1,024 threads whose loads are all issued before the FMAs that use them, so
// each thread waits about once instead of once per vector.
constexpr int kDotThreads = 1024;

__device__ __forceinline__ float block_sum_dot(float s, float* red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
    __syncthreads();
    float r = 0.f;
    if (threadIdx.x == 0)
        for (int i = 0; i < kDotThreads / 32; ++i) r += red[i];
    return r;
}

// anchor[unit][j] = <D_a, h_{a+1}> for a = (j+1) kDaAnchor - 1: the
// gradient of the state after chunk a and the state after it (the state
// entering chunk a+1), each read as its bf16 hi + lo pair, in fp32.  One CTA
// per anchor.
__global__ void __launch_bounds__(kDotThreads) da_anchor_kernel(float* __restrict__ anchor,
                                                                const __nv_bfloat16* __restrict__ dbuf,
                                                                const __nv_bfloat16* __restrict__ hbuf, int NC)
{
    constexpr int kVec = static_cast<int>(kSS / 8);                       // 16-byte vectors per plane
    constexpr int kIt = (kVec + kDotThreads - 1) / kDotThreads;
    __shared__ float red[kDotThreads / 32];
    const int unit = blockIdx.x, j = blockIdx.y, tid = threadIdx.x;
    const int a = (j + 1) * kDaAnchor - 1;
    const uint4* x = reinterpret_cast<const uint4*>(dbuf + (static_cast<int64_t>(unit) * NC + a) * 2 * kSS);
    const uint4* y = reinterpret_cast<const uint4*>(hbuf + (static_cast<int64_t>(unit) * NC + a + 1) * 2 * kSS);
    uint4 xh[kIt], xl[kIt], yh[kIt], yl[kIt];
#pragma unroll
    for (int i = 0; i < kIt; ++i) {
        const int e = tid + i * kDotThreads;
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        xh[i] = e < kVec ? x[e] : z;
        xl[i] = e < kVec ? x[kVec + e] : z;
        yh[i] = e < kVec ? y[e] : z;
        yl[i] = e < kVec ? y[kVec + e] : z;
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kIt; ++i) {
        const uint32_t a0[4] = {xh[i].x, xh[i].y, xh[i].z, xh[i].w}, a1[4] = {xl[i].x, xl[i].y, xl[i].z, xl[i].w};
        const uint32_t b0[4] = {yh[i].x, yh[i].y, yh[i].z, yh[i].w}, b1[4] = {yl[i].x, yl[i].y, yl[i].z, yl[i].w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float u0 = bf16_lo(a0[w]) + bf16_lo(a1[w]), u1 = bf16_hi(a0[w]) + bf16_hi(a1[w]);
            const float v0 = bf16_lo(b0[w]) + bf16_lo(b1[w]), v1 = bf16_hi(b0[w]) + bf16_hi(b1[w]);
            s = fmaf(u0, v0, s);
            s = fmaf(u1, v1, s);
        }
    }
    const float r = block_sum_dot(s, red);
    if (tid == 0) anchor[static_cast<int64_t>(unit) * gridDim.y + j] = r;
}

// out[unit] = <dS_T, S_T> in fp32 (the da term of the tokens after T).
__global__ void __launch_bounds__(kDotThreads) state_dot_kernel(float* __restrict__ out,
                                                                const float* __restrict__ dsT,
                                                                const float* __restrict__ sT)
{
    constexpr int kVec = static_cast<int>(kSS / 4);                       // float4 per state
    constexpr int kIt = (kVec + kDotThreads - 1) / kDotThreads;
    __shared__ float red[kDotThreads / 32];
    const int unit = blockIdx.x, tid = threadIdx.x;
    const float4* x = reinterpret_cast<const float4*>(dsT + unit * kSS);
    const float4* y = reinterpret_cast<const float4*>(sT + unit * kSS);
    float4 u[kIt], v[kIt];
#pragma unroll
    for (int i = 0; i < kIt; ++i) {
        const int e = tid + i * kDotThreads;
        u[i] = e < kVec ? x[e] : make_float4(0.f, 0.f, 0.f, 0.f);
        v[i] = e < kVec ? y[e] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kIt; ++i)
        s = fmaf(u[i].x, v[i].x, fmaf(u[i].y, v[i].y, fmaf(u[i].z, v[i].z, fmaf(u[i].w, v[i].w, s))));
    const float r = block_sum_dot(s, red);
    if (tid == 0) out[unit] = r;
}

template <typename K>
gla_status launch_bwd_kernel(K kernel, uint32_t bytes, const BwdParams& p, dim3 grid, cudaStream_t st,
                             const char* name, int threads)
{
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return check_launch(name);
    trace_begin(st);
    kernel<<<grid, threads, bytes, st>>>(p);
    trace_end(st, name);
    count_launch();
    return check_launch(name);
}

}  // namespace

// Segment scratch of the state passes when B*H is too small to fill the GPU:
// per (unit, segment) an fp32 state and a log2-decay (none when nseg == 1).
size_t seg_scratch_bytes(int units, int nseg)
{
    if (nseg <= 1) return 0;
    return align256(static_cast<size_t>(units) * nseg * kSS * sizeof(float)) +
           align256(static_cast<size_t>(units) * nseg * sizeof(float));
}

// Layout: [h_c planes (not with saved states)] [D_c planes] [S_T (not with
// saved states)] [q.dq, k.dk] [chunk totals] [<dS_T, S_T>] [anchors]
// [segment scratch].
size_t bwd_workspace_bytes(int B, int T, int H, bool from_saved)
{
    const size_t units = static_cast<size_t>(B) * H, NC = num_chunks(T);
    const size_t states = align256(units * NC * kSS * 2 * 2);   // bf16 hi and lo planes
    int nseg, cps;
    chunk_segment_plan(static_cast<int>(units), static_cast<int>(NC), &nseg, &cps);
    const size_t own = from_saved ? 0 : states + align256(units * kSS * sizeof(float));
    return own + states + align256(2 * units * T * sizeof(float)) +
           align256(units * NC * 2 * sizeof(float)) + align256(units * sizeof(float)) +
           align256(units * da_anchors(static_cast<int>(NC)) * sizeof(float)) +
           seg_scratch_bytes(static_cast<int>(units), nseg);
}

gla_status run_chunk_bwd(const ChunkProblem& pr, const float* s0, const void* dO,
                         const float* ds_final, void* dq, void* dk, void* dv, float* da,
                         float* ds0, void* ws, size_t ws_bytes, const WaitCtl& ctl,
                         cudaStream_t st, const void* saved, const float* s_final)
{
    (void)ws_bytes;
    const int units = pr.B * pr.H, NC = num_chunks(pr.T);
    const size_t states = align256(static_cast<size_t>(units) * NC * kSS * 2 * 2);   // bf16 hi and lo planes
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    // with the forward's saved states (gla_chunk_fwd_train) h_c is read from
    // there and S_T is the forward's final state; otherwise both are computed
    // here by a state-only pass
    size_t off = 0;
    void* hbuf = saved ? const_cast<void*>(saved) : wsb;
    if (!saved) off += states;
    void* dbuf = wsb + off;
    off += states;
    float* sT = saved ? const_cast<float*>(s_final) : reinterpret_cast<float*>(wsb + off);
    if (!saved) off += align256(static_cast<size_t>(units) * kSS * sizeof(float));
    float* delta = reinterpret_cast<float*>(wsb + off);
    off += align256(2 * static_cast<size_t>(units) * pr.T * sizeof(float));
    float* ctot = reinterpret_cast<float*>(wsb + off);
    off += align256(static_cast<size_t>(units) * NC * 2 * sizeof(float));
    float* base = reinterpret_cast<float*>(wsb + off);
    off += align256(static_cast<size_t>(units) * sizeof(float));
    const int na = da_anchors(NC);
    float* anchor = reinterpret_cast<float*>(wsb + off);
    off += align256(static_cast<size_t>(units) * na * sizeof(float));
    // segments of chunks per unit, each swept by its own CTA, when B*H alone
    // cannot fill the GPU (long sequences, few heads); the state entering each
    // segment comes from a state-only pre-pass and a fold (launch_seg_combine)
    int nseg, cps;
    chunk_segment_plan(units, NC, &nseg, &cps);
    float* segst = reinterpret_cast<float*>(wsb + off);
    float* segg2 = reinterpret_cast<float*>(wsb + off + align256(static_cast<size_t>(units) * nseg * kSS * sizeof(float)));
    const int64_t ldo = static_cast<int64_t>(pr.H) * kDv;
    gla_status s;
    // state-only pass over `grid_segs` segments from zero into segst / segg2,
    // then the fold that leaves the state entering each segment's sweep there
    auto pre_pass = [&](const StateParams& base_p, bool reverse, int grid_segs, const float* edge) {
        StateParams pre = base_p;
        pre.store_h = 0;
        pre.h_out = nullptr;
        pre.s_init = nullptr;
        pre.s_out = segst;
        pre.out_unit_stride = static_cast<int64_t>(nseg) * kSS;
        pre.out_seg_stride = kSS;
        pre.out_last_only = 0;
        pre.g2_out = segg2;
        pre.g2_unit_stride = nseg;
        gla_status r = launch_state_kernel(false, reverse, pre, dim3(grid_segs, pr.H, pr.B), st);
        if (r != GLA_OK) return r;
        return launch_seg_combine(segst, segg2, edge, nseg, units, reverse, st);
    };

    // 1. h_c for every chunk (and S_T when dS_T is given)
    StateParams sp;
    memset(&sp, 0, sizeof(sp));
    if ((s = make_token_map(&sp.tm_u, pr.k, kDk, pr.H, pr.T, pr.B, pr.ld_qk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&sp.tm_y, pr.v, kDv, pr.H, pr.T, pr.B, pr.ld_v, 64, 128)) != GLA_OK) return s;
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
    sp.chunks_per_seg = cps;
    sp.store_h = 1;
    sp.h_out = hbuf;
    sp.scale = pr.scale;
    sp.ctl = ctl;
    if (!saved) {
        if (nseg > 1) {
            // local end states of segments 0 .. nseg-2 (the last one's is not needed)
            if ((s = pre_pass(sp, false, nseg - 1, s0)) != GLA_OK) return s;
            sp.s_init = segst;
            sp.init_unit_stride = static_cast<int64_t>(nseg) * kSS;
            sp.init_seg_stride = kSS;
        }
        if ((s = launch_state_kernel(false, false, sp, dim3(nseg, pr.H, pr.B), st)) != GLA_OK) return s;
    }

    // 2. D_c for every chunk, dS_0 (written by segment 0, where the reverse
    // sweep ends) and dv, in one reverse sweep: the fused forward kernel run
    // backwards (k in q's place, q in k's, dO in v's, dv out), D_c kept as hi
    // and lo planes like the forward's entering states.  With several
    // segments per head, a state-only reverse pre-pass from zero and the
    // right-to-left fold give each segment's sweep its entering D first.
    StateParams fp;
    memset(&fp, 0, sizeof(fp));
    if ((s = make_token_map(&fp.tm_q, pr.k, kDk, pr.H, pr.T, pr.B, pr.ld_qk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&fp.tm_u, pr.q, kDk, pr.H, pr.T, pr.B, pr.ld_qk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&fp.tm_y, dO, kDv, pr.H, pr.T, pr.B, ldo, 64, 128)) != GLA_OK) return s;
    if ((s = make_token_map(&fp.tm_o, dv, kDv, pr.H, pr.T, pr.B, ldo, 64, 128)) != GLA_OK) return s;
    if ((s = make_state_map(&fp.tm_h, dbuf, static_cast<int64_t>(units) * NC * 2, 64)) != GLA_OK) return s;
    fp.a = pr.a;
    fp.s_init = ds_final;
    fp.init_unit_stride = kSS;
    fp.s_out = ds0;
    fp.out_unit_stride = kSS;
    fp.out_last_only = 1;
    fp.B = pr.B;
    fp.T = pr.T;
    fp.H = pr.H;
    fp.NC = NC;
    fp.chunks_per_seg = cps;
    fp.h_save = dbuf;
    fp.scale = pr.scale;
    fp.ctl = ctl;
    if (nseg > 1) {
        // local gradients of every segment from zero (segment 0's is computed
        // and not used: its CTAs run beside the others'), then the fold
        StateParams rp = sp;
        if ((s = make_token_map(&rp.tm_u, pr.q, kDk, pr.H, pr.T, pr.B, pr.ld_qk, 32, 64)) != GLA_OK) return s;
        if ((s = make_token_map(&rp.tm_y, dO, kDv, pr.H, pr.T, pr.B, ldo, 64, 128)) != GLA_OK) return s;
        if ((s = pre_pass(rp, true, nseg, ds_final)) != GLA_OK) return s;
        fp.s_init = segst;
        fp.init_unit_stride = static_cast<int64_t>(nseg) * kSS;
        fp.init_seg_stride = kSS;
    }
    if ((s = launch_state_kernel(true, true, fp, dim3(nseg, pr.H, pr.B), st)) != GLA_OK) return s;

    // 3. dq, dk (+ per-token delta halves and chunk totals)
    BwdParams bp;
    memset(&bp, 0, sizeof(bp));
    const int64_t ldk = static_cast<int64_t>(pr.H) * kDk;
    if ((s = make_token_map(&bp.tm_q, pr.q, kDk, pr.H, pr.T, pr.B, pr.ld_qk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&bp.tm_k, pr.k, kDk, pr.H, pr.T, pr.B, pr.ld_qk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&bp.tm_dq, dq, kDk, pr.H, pr.T, pr.B, ldk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&bp.tm_dk, dk, kDk, pr.H, pr.T, pr.B, ldk, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&bp.tm_do32, dO, kDv, pr.H, pr.T, pr.B, ldo, 32, 64)) != GLA_OK) return s;
    if ((s = make_token_map(&bp.tm_v32, pr.v, kDv, pr.H, pr.T, pr.B, pr.ld_v, 32, 64)) != GLA_OK) return s;
    if ((s = make_state_map(&bp.tm_h2, hbuf, static_cast<int64_t>(units) * NC * 2, 32, 2)) != GLA_OK) return s;
    if ((s = make_state_map(&bp.tm_d2, dbuf, static_cast<int64_t>(units) * NC * 2, 32, 2)) != GLA_OK) return s;
    bp.a = pr.a;
    bp.delta = delta;
    bp.ctot = ctot;
    bp.B = pr.B;
    bp.T = pr.T;
    bp.H = pr.H;
    bp.NC = NC;
    bp.scale = pr.scale;
    bp.ctl = ctl;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    {
        // persistent: one CTA per SM over the (batch, head, chunk) items
        const int items = units * NC;
        const int grid = items < sms ? items : sms;
        if ((s = launch_bwd_kernel(bwd_dqdk_persistent_kernel, bqp::BYTES, bp, dim3(grid), st, "bwd_dqdk_kernel",
                                   bqp::kThreads)) != GLA_OK)
            return s;
    }

    // 4. da = reverse cumulative sum of delta (+ <dS_T, S_T>)
    if (ds_final) {
        trace_begin(st);
        state_dot_kernel<<<units, kDotThreads, 0, st>>>(base, ds_final, sT);
        trace_end(st, "state_dot_kernel");
        count_launch();
        if ((s = check_launch("state_dot_kernel")) != GLA_OK) return s;
    }
    if (na > 0) {
        trace_begin(st);
        da_anchor_kernel<<<dim3(units, na), kDotThreads, 0, st>>>(anchor, static_cast<const __nv_bfloat16*>(dbuf),
                                                          static_cast<const __nv_bfloat16*>(hbuf), NC);
        trace_end(st, "da_anchor_kernel");
        count_launch();
        if ((s = check_launch("da_anchor_kernel")) != GLA_OK) return s;
    }
    trace_begin(st);
    da_finish_kernel<<<dim3(units, NC), kDaThreads, 0, st>>>(da, delta, ctot, ds_final ? base : nullptr, anchor,
                                                             pr.T, pr.H, NC, units, ctl.status);
    trace_end(st, "da_finish_kernel");
    count_launch();
    return check_launch("da_finish_kernel");
}

}  // namespace gla
