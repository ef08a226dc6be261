// chunk_state.cuh -- the sequential-over-chunks Simple GLA kernels on tcgen05.
//
// A CTA owns one (batch, head, segment of chunks) and walks its chunks in
// order (or in reverse), keeping the fp32 dk x dv state in tensor memory as
// an MMA accumulator.  The chunked form ("Como i14 llevo Laplace 3B a AWS
// Trainium2", section "Adaptaciones para AWS Trainium2", item 1: chunks of
// 128 tokens; item 3: the backward walks the chunks sequentially), for a
// chunk with tokens i, j and in-chunk cumulative log-decay b (gamma = b_last):
//
//   forward  o_i  = scale ( e^{b_i} q_i S_prev + sum_{j<=i} e^{b_i-b_j} (q_i.k_j) v_j )
//            S    = e^{gamma} S_prev + sum_j e^{gamma-b_j} k_j^T v_j
//   reverse  D    = e^{gamma} D_next + sum_i (scale e^{b_i} q_i)^T dO_i
//
// Two kernels:
//
// gla_fwd_fused_kernel<VARLEN, REV> -- forward with the output fused in.
//   REV runs it as the backward's reverse sweep: chunks from the last, k in
//   q's place (the tile rows), q in k's (the scaled operand of the update
//   D = e^gamma D_next + (scale e^b q)^T dO), dO in v's and dv out:
//     dv_i = e^{gamma - b_i} ( k_i D_next + sum_{j >= i} scale e^{b_j - gamma} (k_i.q_j) dO_j )
//   i.e. the same tiles with the causal mask mirrored and the decay factors
//   of the two sides swapped.  Per chunk (forward names):
//   scores = Q K^T (tcgen05, 128x128x96); O = Q S_prev (128x192x96, against a
//   bf16 copy of the state); S += K~^T V (K~ = e^{gamma-b} K split into bf16
//   hi + lo, so the fp32 state keeps its precision); O += P V (P split into
//   bf16 hi + lo); epilogue o = r_i O_i.
//   Decay factorisation: while the chunk's total decay spans at most 2^100,
//   e^{b_i - b_j} = e^{b_i} e^{-b_j} is split into a column factor folded
//   into P (P'_ij = (q_i.k_j) 2^{-b_j}) and a row factor applied in the
//   epilogue (r_i = scale 2^{b_i}); every product stays finite and no
//   per-element exponential or scaled copy of Q is needed.  Chunks with a
//   steeper decay take the exact per-element path (P_ij with 2^{b_i - b_j},
//   Q scaled by scale e^{b_i} in place, r_i = 1).
//   Q tile row i = token i (natural order, three TMA boxes per tile: issuing
//   a tile as 24 permuted 16-row boxes kept the producer busy for about
//   2.5k cycles).  Each worker warp converts one 32-token block of P, so the
//   causal triangle's imbalance between lane quarters costs at most one
//   block per warp.
//
// gla_state_pass_kernel<REVERSE> -- state only: S (or D) = e^gamma S + U~^T Y
//   per chunk with U~ split into bf16 hi + lo, optionally storing the bf16
//   state before each chunk's update (the backward's h_c and D_c).  Twelve
//   warps hold S in registers (dk row, a quarter of dv each); per chunk they
//   write the next chunk's decayed U~^T (hi, lo) into one of two TMEM buffers
//   while the current chunk's dS = U~^T Y runs on the tensor core with A read
//   from TMEM, then fold dS into S and store the bf16 copy.  Warp 3 scans the
//   decays ahead into a ring of per-token factors, warp 11 issues the loads
//   (a three-stage ring) and warp 15 the MMAs.
//
// Operand layouts (validated against the hardware): q and k tiles are
// TMA-loaded as three 32-wide SW64 boxes ([3][128][32]; K-major for the
// scores; the k tile doubles as the MN-major A operand of the state product,
// whose fourth 32-row block -- the padding of dk = 96 to M = 128 -- only
// feeds TMEM lanes 96..127, which are never read); v tiles are three 64-wide
// SW128 boxes ([3][128][64], MN-major B); state copies are [3][96][64] SW128;
// P tiles are [2][128][64] SW128 (K-major A).
//
// Threads: warps 0-15 are workers (warp w reads TMEM lanes 32*(w%4) .. +31,
// column quarter w/4); warp 16 only issues tcgen05.mma, so the workers never
// stall behind the tensor core's issue queue, and warp 17 the TMA copies.  Every wait is
// bounded; on timeout the CTA stops at the next block-wide barrier, drains
// its in-flight copies and tensor-core work (bounded), frees its tensor
// memory and returns with GLA_ERR_TIMEOUT recorded.
#pragma once

#include <type_traits>

#include "gla_device.cuh"

namespace gla {

struct StateParams {
    CUtensorMap tm_q;       // tile rows of the fused kernel: q (forward) or k (reverse sweep)
    CUtensorMap tm_u;       // scaled operand: k (forward) or q (reverse)
    CUtensorMap tm_y;       // v (forward) or dO (reverse)
    CUtensorMap tm_o;       // output tile stores of the fused kernel: o (forward) or dv (reverse sweep)
    CUtensorMap tm_h;       // saved states, 64-column boxes of one plane (fused forward with h_save)
    const float* a;         // [B, T, H] log-decay
    const float* s_init;    // initial state per (unit, seg) or null (zeros)
    float* s_out;           // state after the segment, or null
    float* g2_out;          // total log2-decay of each segment, or null
    int64_t init_unit_stride, init_seg_stride;   // elements
    int64_t out_unit_stride, out_seg_stride;     // elements
    int B, T, H, NC, chunks_per_seg;
    int out_last_only;      // write s_out only from the segment that ends the sweep
                            // (the last one; segment 0 in the reverse pass)
    int g2_unit_stride;     // segments per unit in g2_out
    int store_h;            // store the state entering each chunk into h_out
    void* h_out;            // bf16 [B*H*NC][2][96][192]: plane 0 = bf16(S), plane 1 = bf16(S - plane 0)
    const int* cu_seqlens;  // varlen forward: [B+1] token offsets into batch row 0, or null
    void* o_direct;         // varlen forward: o, for the direct stores of a sequence's last chunk
    // varlen forward cut into segments of chunks_per_seg chunks: segment s of
    // sequence n owns scratch slot n + cu_seqlens[n] / (128 chunks_per_seg) + s
    // (distinct for every (n, s), fewer than N + total / (128 chunks_per_seg) + 1)
    float* seg_states;      // [slots][H][96][192] fp32: pre-pass end states, then entering states
    float* seg_g2;          // [slots][H] total log2-decay of each segment (pre-pass)
    int varlen_segs;        // 1: segmented varlen (chunks_per_seg chunks per segment)
    const int* cps_dev;     // segmented varlen: the chunks per segment the device planned
                            // (read instead of chunks_per_seg when set)
    const int2* work;       // segmented varlen: the (sequence, segment) of grid item x;
    const int* work_count;  // items past *work_count exit (null: the grid's own indices)
    int pre_pass;           // state pass: only segments 0 .. nseg_n - 2 of each sequence
    void* h_save;           // fused forward: the state entering each chunk, [B*H*NC][2][96][192]
                            // bf16 (hi, lo planes), for the backward; null = not saved
    float scale;
    WaitCtl ctl;
};

namespace chunk {

constexpr float kLog2e = 1.4426950408889634f;
// fused forward: 16 worker warps, warp w on TMEM lane quarter w % 4 and
// column quarter w / 4 (of the 128 score, 192 output and state columns)
constexpr int kWorkerWarps = 16;
constexpr int kWorkers = kWorkerWarps * 32;
constexpr int kThreads = kWorkers + 32;
constexpr int kFusedThreads = kThreads + 32;   // + a producer warp
// state pass: 16 warps; w % 4 < 3 for w < 15 are the 12 workers (TMEM lanes
// 0..95 = the dk rows, four column quarters), warp 15 issues
constexpr int kPassThreads = 512;
constexpr uint32_t kTileQK = 3 * 128 * 64;     // 24576 bytes
constexpr uint32_t kTileV = 3 * 128 * 128;     // 49152 bytes
constexpr float kFactorRange = 100.0f;         // max log2 span for the factorised decay

constexpr uint32_t kIdScores = idesc_bf16_f32(128, 128, 0, 0);
constexpr uint32_t kIdOut = idesc_bf16_f32(128, 192, 0, 1);
constexpr uint32_t kIdOutTs = idesc_bf16_f32(128, 192, 0, 1);   // A from tensor memory
constexpr uint32_t kIdState = idesc_bf16_f32(128, 192, 1, 1);
constexpr uint32_t kIdStateTs = idesc_bf16_f32(128, 192, 0, 1);   // A from tensor memory

// Shared-memory maps (bytes from a 1024-aligned base).
struct FusedSmem {
    static constexpr uint32_t Q = 0;          // q tile
    static constexpr uint32_t U = 24576;      // k tile, then K~ (its 4th M block is X: finite)
    static constexpr uint32_t X = 49152;      // bf16 state copy [3][96][64] SW128
    static constexpr uint32_t KL = 86016;     // lo half of K~ [3][128][32] SW64 (hi: K~ in place in U)
    static constexpr uint32_t KL_PAD = 110592;   // [8192] zeros: the 4th M block (dk 96..127) of KL
    static constexpr uint32_t Y0 = 122880;    // v tiles, double buffered
    static constexpr uint32_t Y1 = 172032;    // (the o staging of a chunk, once its P V is done)
    static constexpr uint32_t MISC = 221184;
    static constexpr uint32_t BYTES = MISC + 3072 + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_SC = 0, TM_O = 128, TM_S = 320;
};
struct PassSmem {
    // three stages of (U [3][128][32] SW64, Y [3][128][64] SW128)
    static constexpr uint32_t STAGE = 73728, Y = 24576;
    static constexpr int kStages = 3;
    static constexpr uint32_t MISC = kStages * STAGE;     // barriers, g2 ring
    static constexpr uint32_t FRING = MISC + 256;         // [4][128] per-token decay factors
    static constexpr uint32_t BYTES = FRING + 2048 + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    // dS accumulator [192 cols]; U~^T hi (64 cols) + lo (64 cols) per buffer, two buffers
    static constexpr uint32_t TM_DS = 0, TM_U = 256;
};

// Scratch slot of segment s of sequence n in the segmented varlen forward.
__device__ __forceinline__ int64_t varlen_slot(const int* cu, int n, int s, int chunks_per_seg)
{
    return static_cast<int64_t>(n) + cu[n] / (128 * chunks_per_seg) + s;
}

__device__ __forceinline__ void named_sync(int id, int n)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void bar_sync(int id, int n) { named_sync(id, n); }

// Named-barrier OR reduction over n threads (a __syncthreads_or on a subset).
__device__ __forceinline__ bool bar_or(int id, int n, bool v)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %3, 0;\n\tbarrier.cta.red.or.pred q, %1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"(id), "r"(n), "r"(static_cast<uint32_t>(v)) : "memory");
    return r != 0;
}

__device__ __forceinline__ uint4 scale8(uint4 v, float f)
{
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = pack_bf16(bf16_lo(w[i]) * f, bf16_hi(w[i]) * f);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// hi = bf16(f x), lo = bf16(f x - hi) for 8 bf16 elements.
__device__ __forceinline__ void scale8_split(uint4 v, float f, uint4& hi, uint4& lo)
{
    uint32_t w[4] = {v.x, v.y, v.z, v.w}, h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float a = bf16_lo(w[i]) * f, b = bf16_hi(w[i]) * f;
        h[i] = pack_bf16(a, b);
        l[i] = pack_bf16(a - bf16_lo(h[i]), b - bf16_hi(h[i]));
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Scale the 64-byte row segment `row` of block `blk` of a [3][128][32] SW64
// tile in place (the swizzle only permutes 16-byte chunks within a row).
__device__ __forceinline__ void scale_row_sw64(uint8_t* tile, int row, int blk, float f)
{
    uint4* p = reinterpret_cast<uint4*>(tile + blk * 8192 + row * 64);
#pragma unroll
    for (int c = 0; c < 4; ++c) p[c] = scale8(p[c], f);
}

// In-place hi / separate lo split of a scaled 64-byte row segment.
__device__ __forceinline__ void split_row_sw64(uint8_t* tile, uint8_t* lo_tile, int row, int blk, float f)
{
    uint4* p = reinterpret_cast<uint4*>(tile + blk * 8192 + row * 64);
    uint4* q = reinterpret_cast<uint4*>(lo_tile + blk * 8192 + row * 64);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 h, l;
        scale8_split(p[c], f, h, l);
        p[c] = h;
        q[c] = l;
    }
}

__device__ __forceinline__ uint4 pack8(const uint32_t* r)
{
    return make_uint4(pack_bf16(__uint_as_float(r[0]), __uint_as_float(r[1])),
                      pack_bf16(__uint_as_float(r[2]), __uint_as_float(r[3])),
                      pack_bf16(__uint_as_float(r[4]), __uint_as_float(r[5])),
                      pack_bf16(__uint_as_float(r[6]), __uint_as_float(r[7])));
}

// 8 fp32 values -> bf16 hi and lo (value - hi) terms.
__device__ __forceinline__ void pack8_split(const uint32_t* r, uint4& hi, uint4& lo)
{
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float a = __uint_as_float(r[2 * i]), b = __uint_as_float(r[2 * i + 1]);
        h[i] = pack_bf16(a, b);
        l[i] = pack_bf16(a - bf16_lo(h[i]), b - bf16_hi(h[i]));
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Inclusive cumulative log2-decay of the chunk's 128 tokens, warps 0-3
// (thread t holds token t's a).
__device__ __forceinline__ float chunk_cumsum(float a, float* wsum, int warp, int lane)
{
    float x = a * kLog2e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    named_sync(1, 128);
    float pre = 0.f;
    for (int w = 0; w < warp; ++w) pre += wsum[w];
    return x + pre;
}

// This thread's NCOL columns of its row of a [96][192] fp32 state (src
// points at the first; null = zeros) into TMEM.
template <int NCOL>
__device__ __forceinline__ void state_to_tmem(const float* src, uint32_t taddr)
{
#pragma unroll
    for (int j = 0; j < NCOL / 16; ++j) {
        uint32_t r[16];
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
            const float4 v = src ? *reinterpret_cast<const float4*>(src + j * 16 + e)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            r[e] = __float_as_uint(v.x);
            r[e + 1] = __float_as_uint(v.y);
            r[e + 2] = __float_as_uint(v.z);
            r[e + 3] = __float_as_uint(v.w);
        }
        tmem_st16(taddr + j * 16, r);
    }
    tmem_st_wait();
}

// This thread's NCOL columns of its row of the state, from TMEM to dst.
// Every thread writes a different row (rows 768 B apart), so whole 32-byte
// sectors go out where dst allows it: half the store transactions of
// 16-byte stores, none of them a partial sector.
template <int NCOL>
__device__ __forceinline__ void tmem_to_state(uint32_t taddr, float* dst)
{
    uint32_t r[NCOL / 16][16];
#pragma unroll
    for (int j = 0; j < NCOL / 16; ++j) tmem_ld16(taddr + j * 16, r[j]);
    tmem_ld_wait();
    if ((reinterpret_cast<uintptr_t>(dst) & 31) == 0) {
#pragma unroll
        for (int j = 0; j < NCOL / 16; ++j)
#pragma unroll
            for (int e = 0; e < 16; e += 8) {
                uint32_t w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) w[i] = r[j][e + i];
                st_global_v8(dst + j * 16 + e, w);
            }
    } else {
#pragma unroll
        for (int j = 0; j < NCOL / 16; ++j)
#pragma unroll
            for (int e = 0; e < 16; e += 4)
                *reinterpret_cast<float4*>(dst + j * 16 + e) =
                    make_float4(__uint_as_float(r[j][e]), __uint_as_float(r[j][e + 1]),
                                __uint_as_float(r[j][e + 2]), __uint_as_float(r[j][e + 3]));
    }
}

// State copy into [3][96][64] SW128 (row = dk index, n = dv column) of this
// thread's NCOL columns col0 .. col0+NCOL-1 of its row; then decay the state
// in TMEM by f.  The same values also go to global memory as a bf16 hi plane
// (ghi) and lo plane (glo, the remainder), 32-byte stores, where given.
template <int NCOL>
__device__ __forceinline__ void state_copy_and_decay(uint32_t taddr, int row, int col0, float f, uint8_t* copy,
                                                     uint8_t* ghi = nullptr, uint8_t* glo = nullptr)
{
    uint32_t r[NCOL / 16][16];
#pragma unroll
    for (int j = 0; j < NCOL / 16; ++j) tmem_ld16(taddr + j * 16, r[j]);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < NCOL / 16; ++j) {
        if (ghi || glo) {
            uint32_t w[8], l[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float x0 = __uint_as_float(r[j][2 * e]), x1 = __uint_as_float(r[j][2 * e + 1]);
                w[e] = pack_bf16(x0, x1);
                l[e] = pack_bf16(x0 - bf16_lo(w[e]), x1 - bf16_hi(w[e]));
            }
            if (ghi) st_global_v8(ghi + j * 32, w);
            if (glo) st_global_v8(glo + j * 32, l);
        }
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
            const int n = col0 + j * 16 + h8 * 8;
            *reinterpret_cast<uint4*>(copy + (n >> 6) * 12288 + swz_off(row, (n & 63) >> 3, 128)) =
                pack8(r[j] + h8 * 8);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) r[j][e] = __float_as_uint(__uint_as_float(r[j][e]) * f);
        tmem_st16(taddr + j * 16, r[j]);
    }
    tmem_st_wait();
}

}  // namespace chunk

// The kernels are defined only in the translation unit that launches them
// (chunk_fwd.cu defines GLA_CHUNK_KERNELS before including this header).
#ifdef GLA_CHUNK_KERNELS

// =====================================================================
// Fused forward.
// =====================================================================
template <bool VARLEN, bool REV>
__global__ void __launch_bounds__(chunk::kFusedThreads, 1) gla_fwd_fused_kernel(const __grid_constant__ StateParams p)
{
    using namespace chunk;
    using L = FusedSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bar_q = reinterpret_cast<uint64_t*>(sm + L::MISC);
    uint64_t* bar_u = bar_q + 1;
    uint64_t* bar_y = bar_q + 2;                                 // [2] v tile loaded
    uint64_t* bar_sc = bar_q + 4;                                // scores done
    uint64_t* bar_d = bar_q + 5;                                 // O = Q S_prev and the state update done
    uint64_t* bar_fo = bar_q + 6;                                // O += P V done
    uint64_t* bar_stg = bar_q + 7;                               // [2] o staged in the v buffer (256)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_q + 9);
    uint64_t* bar_xfree = bar_q + 10;                            // the saved-state store has read X
    float* b2s = reinterpret_cast<float*>(sm + L::MISC + 128);  // [2][128] by token, chunk parity
    float* cfac = b2s + 256;                                     // [2][128] 2^{-b_j}
    float* wsum = cfac + 256;                                    // [4]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y;
    int seg = blockIdx.x, b = blockIdx.z;
    if (VARLEN && p.work) {                        // the device-planned segment list
        if (static_cast<int>(blockIdx.x) >= *p.work_count) return;
        const int2 w = p.work[blockIdx.x];
        b = w.x;
        seg = w.y;
    }
    const int unit = b * p.H + h;
    // varlen: b is a sequence, its tokens tb .. tb+Tn-1 of batch row 0;
    // otherwise batch row b, tokens 0 .. T-1
    int tb = 0, Tn = p.T, NCn = p.NC;
    if constexpr (VARLEN) {
        tb = p.cu_seqlens[b];
        Tn = p.cu_seqlens[b + 1] - tb;
        NCn = (Tn + 127) / 128;
        if (tb < 0 || Tn < 0 || tb + Tn > p.T) {   // offsets out of range: touch nothing
            if (threadIdx.x == 0) record_status(p.ctl.status, GLA_ERR_INVALID_ARG);
            return;
        }
    }
    const int bc = VARLEN ? 0 : b;                 // batch coordinate of the token tensors
    const int cps = p.cps_dev ? *p.cps_dev : p.chunks_per_seg;
    const int c_begin = seg * cps;
    // segmented varlen: a grid slot past this sequence's last segment has
    // nothing to do (segment 0 always runs: an empty sequence still passes
    // its initial state on)
    if (VARLEN && seg > 0 && c_begin >= NCn) return;
    const int c_end = min(NCn, c_begin + cps);
    const int nchunks = c_end - c_begin;
    // the chunk of step it: forward in order; the reverse sweep from the last
    constexpr int dc = REV ? -1 : 1;          // chunk step
    const int c_first = REV ? c_end - 1 : c_begin;
    auto chunk_at = [c_first](int it) { return c_first + dc * it; };
    // the segment where the sweep ends (the reverse sweep ends on segment 0)
    const int last_seg = REV ? 0
                             : VARLEN ? max(1, (NCn + cps - 1) / cps) - 1
                                      : static_cast<int>(gridDim.x) - 1;
    const WaitCtl ctl = p.ctl;

    const int quad = warp & 3;
    const int row = quad * 32 + lane;         // TMEM lane = tile row = token in the chunk
    const int tok = row;
    const int cq = warp >> 2;                 // column quarter (workers)
    constexpr int kOC = kDv / 4;              // output and state columns per worker: 48
    const bool worker = warp < kWorkerWarps;
    const bool srow = worker && quad < 3;
    const bool issuer = warp == kWorkerWarps && lane == 0;
    const bool producer = warp == kWorkerWarps + 1 && lane == 0;   // TMA loads and o stores; outside the loop's barriers
    // this lane quarter's rows span tokens 32 quad .. +31: a 32-token column
    // block past them (forward) or before them (reverse) is masked whole
    const int quad_max_tok = quad * 32 + 31, quad_min_tok = quad * 32;

    if (issuer) {
        mbar_init(bar_q, 1);
        mbar_init(bar_u, 1);
        mbar_init(bar_y, 1);
        mbar_init(bar_y + 1, 1);
        mbar_init(bar_sc, 1);
        mbar_init(bar_d, 1);
        mbar_init(bar_fo, 1);
        mbar_init(bar_stg, kWorkers);
        mbar_init(bar_stg + 1, kWorkers);
        mbar_init(bar_xfree, 1);
        mbar_init_fence();
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_u);
        tma_prefetch_desc(&p.tm_y);
        tma_prefetch_desc(&p.tm_o);
        if (p.h_save) tma_prefetch_desc(&p.tm_h);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tq = tmem_addr(tmem, quad * 32, 0);

    auto load_a = [&](int c) {
        const int t = c * 128 + tid;
        return t < Tn ? p.a[(static_cast<int64_t>(bc) * p.T + tb + t) * p.H + h] : 0.f;
    };
    // this thread's row of the saved state entering chunk c (hi plane), or null
    constexpr int64_t kStatePlane = static_cast<int64_t>(kDk) * kDv * 2;
    auto save_row = [&](int c) -> uint8_t* {
        if (VARLEN || !p.h_save || !GLA_DCHECK(c < p.NC && unit < p.B * p.H, p.ctl.status)) return nullptr;
        return static_cast<uint8_t*>(p.h_save) + ((static_cast<int64_t>(unit) * p.NC + c) * 2) * kStatePlane +
               static_cast<int64_t>(row) * (kDv * 2) + cq * (kOC * 2);
    };
    // saved states: the lo plane from the workers' registers, the hi plane
    // from the bf16 copy X by the producer's TMA store
    const bool tma_save = !VARLEN && p.h_save != nullptr;
    // cumulative log2-decay b of a chunk and its column factors (warps 0-3):
    // 2^{-b_j} forward, scale 2^{b_i - gamma} in the reverse sweep
    auto decays = [&](float av, int par) {
        if (tid < 128) {
            const float x = chunk_cumsum(av, wsum, warp, lane);
            b2s[par * 128 + tid] = x;
            if constexpr (REV) {
                const float g = ((wsum[0] + wsum[1]) + wsum[2]) + wsum[3];
                cfac[par * 128 + tid] = p.scale * exp2f(x - g);
            } else {
                cfac[par * 128 + tid] = exp2f(-x);
            }
        }
    };

    // the rows dk 96..127 of the K~ lo operand (the padding of M to 128; they
    // feed only accumulator lanes that are never read): zeros
    for (int i = tid; i < 512; i += blockDim.x)
        reinterpret_cast<uint4*>(sm + L::KL_PAD)[i] = make_uint4(0u, 0u, 0u, 0u);

    // The producer's loads (q, k single, v double buffered).  Those of the
    // first chunks go out before the prologue: they fill Q, U, Y0 and Y1,
    // which the prologue does not touch (it writes KL_PAD, X and MISC).
    auto issue_qu = [&](int c) {
        const int t0 = c * 128;
        mbar_arrive_expect_tx(bar_q, kTileQK);
        for (int i = 0; i < 3; ++i) tma_load_4d(sm + L::Q + i * 8192, &p.tm_q, bar_q, i * 32, h, tb + t0, bc);
        mbar_arrive_expect_tx(bar_u, kTileQK);
        for (int i = 0; i < 3; ++i) tma_load_4d(sm + L::U + i * 8192, &p.tm_u, bar_u, i * 32, h, tb + t0, bc);
    };
    // q, k of a later chunk into L2, so that its load (issued only once the
    // current chunk's state update has released the tiles) hits L2
    auto prefetch_qu = [&](int c) {
        const int t0 = c * 128;
        for (int i = 0; i < 3; ++i) {
            tma_prefetch_l2_4d(&p.tm_q, i * 32, h, tb + t0, bc);
            tma_prefetch_l2_4d(&p.tm_u, i * 32, h, tb + t0, bc);
        }
    };
    auto issue_y = [&](int c, int s) {
        uint8_t* y = sm + (s ? L::Y1 : L::Y0);
        mbar_arrive_expect_tx(bar_y + s, kTileV);
        for (int i = 0; i < 3; ++i)
            tma_load_4d(y + i * 16384, &p.tm_y, bar_y + s, i * 64, h, tb + c * 128, bc);
    };
    if (producer) {
        if (nchunks > 1) prefetch_qu(chunk_at(1));
        if (nchunks > 0) {
            issue_qu(chunk_at(0));
            issue_y(chunk_at(0), 0);
            if (nchunks > 1) issue_y(chunk_at(1), 1);
        }
    }

    // prologue: decays and state copy of the first chunk
    float a_nx = (tid < 128 && nchunks > 1) ? load_a(chunk_at(1)) : 0.f;
    if (nchunks > 0) decays(tid < 128 ? load_a(chunk_at(0)) : 0.f, 0);
    if (srow) {
        const float* src = p.s_init ? p.s_init + unit * p.init_unit_stride + seg * p.init_seg_stride +
                                          row * kDv + cq * kOC
                                    : nullptr;
        if (VARLEN && seg > 0)    // a later segment of a sequence: the state the combine left for it
            src = p.seg_states + (varlen_slot(p.cu_seqlens, b, seg, cps) * p.H + h) * (kDk * kDv) +
                  row * kDv + cq * kOC;
        state_to_tmem<kOC>(src, tq + L::TM_S + cq * kOC);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (nchunks > 0 && srow) {
        uint8_t* g = save_row(chunk_at(0));
        state_copy_and_decay<kOC>(tq + L::TM_S + cq * kOC, row, cq * kOC, exp2f(b2s[127]), sm + L::X, g,
                                  g ? g + kStatePlane : nullptr);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (producer) {
        // ----------------------------------------------------------- producer
        // q, k of chunk it+1 once (D) of chunk it is done; the o tile of chunk
        // it from its v buffer once staged, then v of chunk it+2 into it
        // (loads issued so far: those of the first chunks, before the prologue)
        int n_qu = nchunks > 0 ? 1 : 0, n_y[2] = {nchunks > 0 ? 1 : 0, nchunks > 1 ? 1 : 0};
        for (int it = 0; it < nchunks; ++it) {
            const int c = chunk_at(it), ys = it & 1;
            if (it + 2 < nchunks) prefetch_qu(c + 2 * dc);
            if (it + 1 < nchunks) {
                if (!mbar_wait(bar_d, it & 1, ctl)) break;
                issue_qu(c + dc);
                ++n_qu;
            }
            if (!mbar_wait(bar_stg + ys, (it >> 1) & 1, ctl)) break;
            const bool direct = VARLEN && c * 128 + 128 > Tn;
            if (!direct) {
                uint8_t* y = sm + (ys ? L::Y1 : L::Y0);
                for (int i = 0; i < 3; ++i) tma_store_4d(&p.tm_o, y + i * 16384, i * 64, h, tb + c * 128, bc);
                tma_store_commit();
            }
            // the state entering chunk c+1, whose bf16 copy X the workers wrote
            // before this epilogue, goes out as its saved hi plane
            const bool save_x = tma_save && it + 1 < nchunks;
            if (save_x) {
                const int si = (unit * p.NC + c + dc) * 2;
                for (int i = 0; i < 3; ++i) tma_store_3d(&p.tm_h, sm + L::X + i * 12288, i * 64, 0, si);
                tma_store_commit();
            }
            if (it + 2 < nchunks || save_x) {
                tma_store_wait_read();
                if (save_x) mbar_arrive(bar_xfree);
                if (it + 2 < nchunks) {
                    issue_y(c + 2 * dc, ys);
                    ++n_y[ys];
                }
            }
        }
        tma_store_wait_all();
        // at most one load per barrier is ever outstanding
        if (n_qu) {
            mbar_wait(bar_q, (n_qu - 1) & 1, ctl);
            mbar_wait(bar_u, (n_qu - 1) & 1, ctl);
        }
        for (int i = 0; i < 2; ++i)
            if (n_y[i]) mbar_wait(bar_y + i, (n_y[i] - 1) & 1, ctl);
    }

    // -------------------------------------------------- workers and issuer
    uint32_t ph_q = 0, ph_u = 0, ph_y[2] = {0u, 0u};
    int n_sc = 0, n_d = 0, n_fo = 0;          // commits (issuer)
    bool failed = false, aborted = false;
    for (int it = 0; warp <= kWorkerWarps && it < nchunks; ++it) {
        const int c = chunk_at(it);
        const int ys = it & 1, par = it & 1;
        const uint32_t ya = ys ? L::Y1 : L::Y0;
        const float* b2c = b2s + par * 128;
        const float* cfc = cfac + par * 128;

        // (A) scores, once q and k are in and the last chunk's P V (which reads
        // its P from the scores columns) is done
        if (issuer) {
            if (mbar_wait(bar_q, ph_q, ctl) && mbar_wait(bar_u, ph_u, ctl) &&
                (it == 0 || mbar_wait(bar_fo, (it - 1) & 1, ctl))) {
                ph_q ^= 1;
                ph_u ^= 1;
                tc_fence_after();
                const uint64_t dq = smem_desc(sb + L::Q, 16, 512, kLayoutSW64);
                const uint64_t du = smem_desc(sb + L::U, 16, 512, kLayoutSW64);
#pragma unroll
                for (int ks = 0; ks < 6; ++ks) {
                    const uint32_t off = (ks >> 1) * 8192 + (ks & 1) * 32;
                    umma_bf16(tmem + L::TM_SC, desc_add(dq, off), desc_add(du, off), kIdScores, ks > 0);
                }
                umma_commit(bar_sc);
                ++n_sc;
            } else {
                failed = true;
            }
        }
        const float g2 = b2c[127];
        const bool fast = -g2 <= kFactorRange;   // uniform: the factorised path is safe

        // (C) K~ = e^{gamma - b} K as a bf16 pair: hi in place, lo (K~ - hi) in
        // KL, so that the state update keeps the fp32 state's precision; on
        // the exact path also Q~ = scale e^{b} Q
        if (worker && !failed && !mbar_wait(bar_sc, it & 1, ctl)) failed = true;
        if (!failed && worker) {
            const int live = Tn - c * 128;   // varlen: rows past the sequence (the next one's) add nothing
            // 16-byte chunk idx % 4 of row (idx / 4) % 128 of block idx / 512: a
            // warp covers 512 contiguous bytes, so no two lanes share a bank
            for (int idx = tid; idx < 1536; idx += kWorkers) {
                const int r = (idx >> 2) & 127, blk = idx >> 9, ch = idx & 3;
                uint4* u = reinterpret_cast<uint4*>(sm + L::U + blk * 8192 + r * 64) + ch;
                uint4 hi, lo;
                // forward K~ = 2^{gamma - b} K; reverse Q~ = scale 2^{b} Q (in the U tile)
                const float fu = REV ? p.scale * exp2f(b2c[r]) : exp2f(g2 - b2c[r]);
                scale8_split(*u, (!VARLEN || r < live) ? fu : 0.f, hi, lo);
                *u = hi;
                *(reinterpret_cast<uint4*>(sm + L::KL + blk * 8192 + r * 64) + ch) = lo;
                if (!fast) {
                    uint4* qq = reinterpret_cast<uint4*>(sm + L::Q + blk * 8192 + r * 64) + ch;
                    *qq = scale8(*qq, REV ? exp2f(g2 - b2c[r]) : p.scale * exp2f(b2c[r]));
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        if (bar_or(2, kThreads, failed)) { aborted = true; break; }
        tc_fence_after();

        // (D) O = Q S_prev, S += K~^T V (K~ as hi + lo)
        if (issuer) {
            if (mbar_wait(bar_y + ys, ph_y[ys], ctl)) {
                ph_y[ys] ^= 1;
                const uint64_t dq = smem_desc(sb + L::Q, 16, 512, kLayoutSW64);
                const uint64_t dx = smem_desc(sb + L::X, 12288, 1024, kLayoutSW128);
                const uint64_t dua = smem_desc(sb + L::U, 8192, 512, kLayoutSW64);
                const uint64_t dul = smem_desc(sb + L::KL, 8192, 512, kLayoutSW64);
                const uint64_t dy = smem_desc(sb + ya, 16384, 1024, kLayoutSW128);
#pragma unroll
                for (int ks = 0; ks < 6; ++ks)
                    umma_bf16(tmem + L::TM_O, desc_add(dq, (ks >> 1) * 8192 + (ks & 1) * 32),
                              desc_add(dx, ks * 2048), kIdOut, ks > 0);
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        umma_bf16(tmem + L::TM_S, desc_add(part ? dul : dua, ks * 1024), desc_add(dy, ks * 2048),
                                  kIdState, 1);
                umma_commit(bar_d);
                ++n_d;
            } else {
                failed = true;
            }
        }

        // (E) scores -> P (hi, lo) in place in tensor memory: lane = row i,
        // 32-token block kb holds hi in columns 32 kb .. +15 and lo in +16 .. +31.
        float rf = 1.0f;
        if (worker) {
            const float b2r = b2c[tok];
            if (fast) rf = REV ? exp2f(g2 - b2r) : p.scale * exp2f(b2r);
            {
                const int j0 = cq * 32;               // this warp's 32-token block
                const uint32_t col = L::TM_SC + j0;
                uint32_t hi[16], lo[16];
                if (REV ? j0 + 31 < quad_min_tok : j0 > quad_max_tok) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) hi[e] = lo[e] = 0u;
                } else {
                    uint32_t r[32];
                    tmem_ld32(tq + col, r);
                    tmem_ld_wait();
                    // one loop per path, so that no element computes the
                    // other path's factor
                    auto conv = [&](auto fast_tag) {
                        constexpr bool FAST = decltype(fast_tag)::value;
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const int j = j0 + e;
                            float v0, v1;
                            // causal: column j <= row (forward), j >= row (reverse)
                            if constexpr (FAST && !REV) {
                                v0 = (j <= tok) ? __uint_as_float(r[e]) * cfc[j] : 0.f;
                                v1 = (j + 1 <= tok) ? __uint_as_float(r[e + 1]) * cfc[j + 1] : 0.f;
                            } else if constexpr (!REV) {
                                v0 = (j <= tok) ? p.scale * __uint_as_float(r[e]) * exp2f(b2r - b2c[j]) : 0.f;
                                v1 = (j + 1 <= tok) ? p.scale * __uint_as_float(r[e + 1]) * exp2f(b2r - b2c[j + 1])
                                                    : 0.f;
                            } else if constexpr (FAST) {
                                v0 = (j >= tok) ? __uint_as_float(r[e]) * cfc[j] : 0.f;
                                v1 = (j + 1 >= tok) ? __uint_as_float(r[e + 1]) * cfc[j + 1] : 0.f;
                            } else {
                                v0 = (j >= tok) ? p.scale * __uint_as_float(r[e]) * exp2f(b2c[j] - b2r) : 0.f;
                                v1 = (j + 1 >= tok) ? p.scale * __uint_as_float(r[e + 1]) * exp2f(b2c[j + 1] - b2r)
                                                    : 0.f;
                            }
                            const uint32_t hv = pack_bf16(v0, v1);
                            hi[e / 2] = hv;
                            lo[e / 2] = pack_bf16(v0 - bf16_lo(hv), v1 - bf16_hi(hv));
                        }
                    };
                    if (fast) conv(std::true_type{});
                    else conv(std::false_type{});
                }
                tmem_st16(tq + col, hi);
                tmem_st16(tq + col + 16, lo);
            }
            tmem_st_wait();
        }
        tc_fence_before();
        if (bar_or(2, kThreads, failed)) { aborted = true; break; }

        // (F) O += P V with P from tensor memory
        if (issuer) {
            tc_fence_after();
            const uint64_t dy = smem_desc(sb + ya, 16384, 1024, kLayoutSW128);
#pragma unroll
            for (int part = 0; part < 2; ++part)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_bf16_ts(tmem + L::TM_O, tmem + L::TM_SC + 32 * (ks >> 1) + 8 * (ks & 1) + 16 * part,
                                 desc_add(dy, ks * 2048), kIdOutTs, 1);
            umma_commit(bar_fo);
            ++n_fo;
        }
        const float a_next = (tid < 128 && it + 2 < nchunks) ? load_a(c + 2 * dc) : 0.f;

        // (B) while P V runs: the next chunk's decays, then -- once (D) has
        // updated S and released the state copies -- its state copy and decay
        if (worker && it + 1 < nchunks) {
            decays(a_nx, par ^ 1);
            named_sync(3, kWorkers);             // the next chunk's total decay is in b2s
            if (!failed && !mbar_wait(bar_d, it & 1, ctl)) failed = true;
            // the producer's store of the last copy has read X
            if (!failed && tma_save && it >= 1 && !mbar_wait(bar_xfree, (it - 1) & 1, ctl)) failed = true;
            tc_fence_after();
            if (srow && !failed) {
                uint8_t* g = save_row(c + dc);
                state_copy_and_decay<kOC>(tq + L::TM_S + cq * kOC, row, cq * kOC, exp2f(b2s[(par ^ 1) * 128 + 127]),
                                          sm + L::X, tma_save ? nullptr : g, g ? g + kStatePlane : nullptr);
            }
            fence_async_smem();
        }

        // (G) epilogue: o = r_i O_i -> bf16 staging in this chunk's v buffer
        // (token order, [3][128][64] SW128) -> the producer's TMA store; a
        // varlen sequence's last chunk writes its rows itself
        if (worker) {
            if (!failed && !mbar_wait(bar_fo, it & 1, ctl)) failed = true;
            tc_fence_after();
            const bool direct = VARLEN && c * 128 + 128 > Tn;
            const bool mine = VARLEN && tok < Tn - c * 128;
            uint8_t* orow = VARLEN ? static_cast<uint8_t*>(p.o_direct) +
                                         ((static_cast<int64_t>(tb) + c * 128 + tok) * p.H + h) * (kDv * 2) + cq * (kOC * 2)
                                   : nullptr;
            if (!failed) {
                uint8_t* stg = sm + ya;
                uint32_t r[kOC / 16][16];
#pragma unroll
                for (int j = 0; j < kOC / 16; ++j) tmem_ld16(tq + L::TM_O + cq * kOC + j * 16, r[j]);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < kOC / 16; ++j) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) r[j][e] = __float_as_uint(__uint_as_float(r[j][e]) * rf);
#pragma unroll
                    for (int h8 = 0; h8 < 2; ++h8) {
                        const int n = cq * kOC + j * 16 + h8 * 8;
                        if (!direct)
                            *reinterpret_cast<uint4*>(stg + (n >> 6) * 16384 + swz_off(tok, (n & 63) >> 3, 128)) =
                                pack8(r[j] + h8 * 8);
                        else if (mine && GLA_DCHECK(tb + c * 128 + tok < p.T, p.ctl.status))
                            *reinterpret_cast<uint4*>(orow + (j * 16 + h8 * 8) * 2) = pack8(r[j] + h8 * 8);
                    }
                }
                fence_async_smem();
                mbar_arrive(bar_stg + ys);
            }
        }
        tc_fence_before();
        a_nx = a_next;
    }

    if (!aborted && warp <= kWorkerWarps) {
        // all MMAs are done (the epilogue waited for the last P V): S is final
        const bool write_state = p.s_out && (!p.out_last_only || seg == last_seg);
        if (write_state && srow && !failed && GLA_DCHECK(unit < p.B * p.H, p.ctl.status))
            tmem_to_state<kOC>(tq + L::TM_S + cq * kOC,
                               p.s_out + unit * p.out_unit_stride + seg * p.out_seg_stride + row * kDv + cq * kOC);
    }
    if (issuer) {
        // every commit's arrival has landed before the barriers go away: at
        // most one phase of each is outstanding, so wait for the last one
        if (n_sc) mbar_wait(bar_sc, (n_sc - 1) & 1, ctl);
        if (n_d) mbar_wait(bar_d, (n_d - 1) & 1, ctl);
        if (n_fo) mbar_wait(bar_fo, (n_fo - 1) & 1, ctl);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, L::TMEM_COLS);
}

// =====================================================================
// State-only pass (double-buffered tiles).
// =====================================================================
template <bool REVERSE>
__global__ void __launch_bounds__(chunk::kPassThreads, 1) gla_state_pass_kernel(const __grid_constant__ StateParams p)
{
    using namespace chunk;
    using L = PassSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(sm + L::MISC);   // [3] stage loaded
    uint64_t* bar_free = bar_ld + 3;                                // [3] stage's MMAs done
    uint64_t* bar_split = bar_ld + 6;                               // [2] U~^T buffer written (384)
    uint64_t* bar_mma = bar_ld + 8;                                 // [2] dS of chunk parity done
    uint64_t* bar_read = bar_ld + 10;                               // dS read by the workers (384)
    uint64_t* bar_f = bar_ld + 11;                                  // [4] decay factors ready (32)
    uint64_t* bar_fdone = bar_ld + 15;                              // [4] decay factors used (384)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ld + 19);
    float* g2s = reinterpret_cast<float*>(sm + L::MISC + 192);      // [4] chunk log2-decay
    float* fring = reinterpret_cast<float*>(sm + L::FRING);
    constexpr uint32_t kWork = 384;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y;
    int seg = blockIdx.x, b = blockIdx.z;
    if (p.cu_seqlens && p.work) {                  // the device-planned segment list
        if (static_cast<int>(blockIdx.x) >= *p.work_count) return;
        const int2 w = p.work[blockIdx.x];
        b = w.x;
        seg = w.y;
    }
    const int unit = b * p.H + h;
    const int cps = p.cps_dev ? *p.cps_dev : p.chunks_per_seg;
    // varlen (segmented pre-pass of the packed forward): b is a
    // sequence, its tokens tb .. tb+Tn-1 of batch row 0; the segments are
    // the sequence's own, and the pre-pass sweeps all but its last
    int tb = 0, Tn = p.T, NCn = p.NC;
    if (p.cu_seqlens) {
        tb = p.cu_seqlens[b];
        Tn = p.cu_seqlens[b + 1] - tb;
        if (tb < 0 || Tn < 0 || tb + Tn > p.T) {   // offsets out of range: touch nothing
            if (threadIdx.x == 0) record_status(p.ctl.status, GLA_ERR_INVALID_ARG);
            return;
        }
        NCn = (Tn + 127) / 128;
        const int nseg_n = max(1, (NCn + cps - 1) / cps);
        if (seg >= nseg_n - (p.pre_pass ? 1 : 0)) return;
    }
    const int bc = p.cu_seqlens ? 0 : b;         // batch coordinate of the token tensors
    const int c_begin = seg * cps;
    const int c_end = min(NCn, c_begin + cps);
    const int nchunks = c_end - c_begin;
    const WaitCtl ctl = p.ctl;
    const int quad = warp & 3, row = quad * 32 + lane, qt = warp >> 2;
    const bool worker = warp < 15 && quad < 3;     // TMEM lanes 0..95: row = dk index
    const bool issuer = warp == 15 && lane == 0;
    const bool producer = warp == 11 && lane == 0;
    const bool decay = warp == 3;

    if (issuer) {
        for (int i = 0; i < 3; ++i) {
            mbar_init(bar_ld + i, 1);
            mbar_init(bar_free + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_split + i, kWork);
            mbar_init(bar_mma + i, 1);
        }
        mbar_init(bar_read, kWork);
        for (int i = 0; i < 4; ++i) {
            mbar_init(bar_f + i, 32);
            mbar_init(bar_fdone + i, kWork);
        }
        mbar_init_fence();
        tma_prefetch_desc(&p.tm_u);
        tma_prefetch_desc(&p.tm_y);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto chunk_at = [&](int it) { return REVERSE ? (c_end - 1 - it) : (c_begin + it); };

    if (producer) {
        // -------------------------------------------------------- producer
        // chunk it goes to stage it % 3 as soon as the MMAs of chunk it-3,
        // the stage's previous user, are done
        int n_ld[3] = {0, 0, 0};
        for (int it = 0; it < nchunks; ++it) {
            const int st = it % 3;
            if (it >= 3 && !mbar_wait(bar_free + st, ((it - 3) / 3) & 1, ctl)) break;
            const int t0 = tb + chunk_at(it) * 128;
            uint8_t* base = sm + st * L::STAGE;
            mbar_arrive_expect_tx(bar_ld + st, kTileQK + kTileV);
            for (int i = 0; i < 3; ++i) {
                tma_load_4d(base + i * 8192, &p.tm_u, bar_ld + st, i * 32, h, t0, bc);
                tma_load_4d(base + L::Y + i * 16384, &p.tm_y, bar_ld + st, i * 64, h, t0, bc);
            }
            ++n_ld[st];
        }
        // at most one load per stage is ever outstanding: waiting for the last
        // one issued waits for everything in flight
        for (int i = 0; i < 3; ++i)
            if (n_ld[i]) mbar_wait(bar_ld + i, (n_ld[i] - 1) & 1, ctl);
    } else if (decay) {
        // ------------------------------------------------------ decay warp
        // per chunk: f_t (U~ = f U) for the 128 tokens and the chunk's total
        // log2-decay, into a four-slot ring; lane L scans tokens 4L .. 4L+3
        auto load_a = [&](int it, float (&x)[4]) {
            const int c = chunk_at(it);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int t = c * 128 + lane * 4 + e;
                x[e] = (it < nchunks && t < Tn) ? p.a[(static_cast<int64_t>(bc) * p.T + tb + t) * p.H + h] : 0.f;
            }
        };
        float xa[4];
        load_a(0, xa);
        for (int it = 0; it < nchunks; ++it) {
            float c4[4];
            c4[0] = xa[0] * kLog2e;
#pragma unroll
            for (int e = 1; e < 4; ++e) c4[e] = c4[e - 1] + xa[e] * kLog2e;
            load_a(it + 1, xa);
            float incl = c4[3];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const float up = __shfl_up_sync(0xffffffffu, incl, 1);
            const float pre = lane ? up : 0.f;
            const float g2 = __shfl_sync(0xffffffffu, incl, 31);
            float f[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) f[e] = REVERSE ? p.scale * exp2f(pre + c4[e]) : exp2f(g2 - (pre + c4[e]));
            if (p.cu_seqlens) {
                // rows past the sequence (the next sequence's tokens) add nothing
                const int t = chunk_at(it) * 128 + lane * 4;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (t + e >= Tn) f[e] = 0.f;
            }
            const int slot = it & 3;
            if (it >= 4 && !mbar_wait(bar_fdone + slot, ((it - 4) >> 2) & 1, ctl)) break;
            *reinterpret_cast<float4*>(fring + slot * 128 + lane * 4) = make_float4(f[0], f[1], f[2], f[3]);
            if (lane == 0) g2s[slot] = g2;
            __syncwarp();
            mbar_arrive(bar_f + slot);
        }
    } else if (issuer) {
        // ---------------------------------------------------------- issuer
        int n_mma[2] = {0, 0}, n_free[3] = {0, 0, 0};
        for (int it = 0; it < nchunks; ++it) {
            if (!mbar_wait(bar_split + (it & 1), (it >> 1) & 1, ctl)) break;
            if (it >= 1 && !mbar_wait(bar_read, (it - 1) & 1, ctl)) break;
            tc_fence_after();
            const uint32_t ya = sb + (it % 3) * L::STAGE + L::Y;
            const uint32_t ua = tmem + L::TM_U + (it & 1) * 128;
            const uint64_t yd = smem_desc(ya, 16384, 1024, kLayoutSW128);
#pragma unroll
            for (int part = 0; part < 2; ++part)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_bf16_ts(tmem + L::TM_DS, ua + part * 64 + ks * 8, desc_add(yd, ks * 2048), kIdStateTs,
                                 (part | ks) > 0);
            umma_commit(bar_mma + (it & 1));
            umma_commit(bar_free + it % 3);
            ++n_mma[it & 1];
            ++n_free[it % 3];
        }
        // at most one phase of each barrier is ever outstanding
        for (int i = 0; i < 2; ++i)
            if (n_mma[i]) mbar_wait(bar_mma + i, (n_mma[i] - 1) & 1, ctl);
        for (int i = 0; i < 3; ++i)
            if (n_free[i]) mbar_wait(bar_free + i, (n_free[i] - 1) & 1, ctl);
    } else if (worker) {
        // ---------- state in registers (row `row`, columns 48 qt .. +47)
        float S[48];
        const float* src = p.s_init ? p.s_init + unit * p.init_unit_stride + seg * p.init_seg_stride +
                                          row * kDv + qt * 48
                                    : nullptr;
#pragma unroll
        for (int e = 0; e < 48; e += 4) {
            const float4 v = src ? *reinterpret_cast<const float4*>(src + e) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[e] = v.x;
            S[e + 1] = v.y;
            S[e + 2] = v.z;
            S[e + 3] = v.w;
        }
        const uint32_t tq = tmem_addr(tmem, quad * 32, 0);
        // U~^T (row = dk index, columns = tokens 32 qt .. +31) -> TMEM buffer.
        // Element (t, d) of the [3][128][32] SW64 tile sits at block d/32, byte
        // 64 t + 16 ((d%32)/8 ^ (t/2)%4) + 2 (d%8); for t = 32 qt + 2 q the
        // xor term is q % 4, so every load has a constant offset.
        const uint32_t cb = lane >> 3;
        const uint32_t sw[4] = {(cb ^ 0u) * 16 + (lane & 7) * 2, (cb ^ 1u) * 16 + (lane & 7) * 2,
                                (cb ^ 2u) * 16 + (lane & 7) * 2, (cb ^ 3u) * 16 + (lane & 7) * 2};
        auto split = [&](int it) {
            const uint8_t* u = sm + (it % 3) * L::STAGE + quad * 8192 + qt * 32 * 64;
            const float* fs = fring + (it & 3) * 128 + qt * 32;
            const uint32_t dst = tq + L::TM_U + (it & 1) * 128 + qt * 16;
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                float f[16];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 v = *reinterpret_cast<const float4*>(fs + g * 16 + 4 * i);
                    f[4 * i] = v.x;
                    f[4 * i + 1] = v.y;
                    f[4 * i + 2] = v.z;
                    f[4 * i + 3] = v.w;
                }
                uint32_t hi[8], lo[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int tl = g * 16 + 2 * q;           // token within this quarter
                    const uint32_t o = sw[q & 3];
                    const float k0 = __uint_as_float(
                        static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(u + tl * 64 + o)) << 16);
                    const float k1 = __uint_as_float(
                        static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(u + tl * 64 + 64 + o)) << 16);
                    const float v0 = k0 * f[2 * q], v1 = k1 * f[2 * q + 1];
                    const uint32_t hv = pack_bf16(v0, v1);
                    hi[q] = hv;
                    lo[q] = pack_bf16(v0 - bf16_lo(hv), v1 - bf16_hi(hv));
                }
                tmem_st8(dst + g * 8, hi);
                tmem_st8(dst + 64 + g * 8, lo);
            }
            tmem_st_wait();
        };
        // S as a bf16 pair, hi = bf16(S) and lo = bf16(S - hi) (96 B of this
        // thread's row in each plane) -> h_out as 32-byte stores: whole
        // sectors, the row segments 32-byte aligned.  hi + lo carries S to
        // about 2^-17 of its size, so the gradient terms read against the
        // pair keep the precision of the fp32 state.
        auto store_h = [&](int it) {
            if (!GLA_DCHECK(chunk_at(it) >= 0 && chunk_at(it) < p.NC && unit < p.B * p.H, p.ctl.status)) return;
            uint8_t* dst = static_cast<uint8_t*>(p.h_out) +
                           (((static_cast<int64_t>(unit) * p.NC + chunk_at(it)) * 2) * kDk + row) * (kDv * 2) + qt * 96;
            constexpr int64_t kPlane = static_cast<int64_t>(kDk) * kDv * 2;
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                uint32_t w[8], l[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float x0 = S[16 * q + 2 * e], x1 = S[16 * q + 2 * e + 1];
                    w[e] = pack_bf16(x0, x1);
                    l[e] = pack_bf16(x0 - bf16_lo(w[e]), x1 - bf16_hi(w[e]));
                }
                st_global_v8(dst + 32 * q, w);
                st_global_v8(dst + kPlane + 32 * q, l);
            }
        };

        bool ok = true;
        float gsum2 = 0.f;
        float g2 = 0.f;
        // split of chunk it: its decay factors and tiles are ready and the
        // TMEM buffer's previous MMAs (chunk it-2) are done
        auto do_split = [&](int it) {
            if (!mbar_wait(bar_f + (it & 3), (it >> 2) & 1, ctl) || !mbar_wait(bar_ld + it % 3, (it / 3) & 1, ctl) ||
                (it >= 2 && !mbar_wait(bar_mma + (it & 1), ((it - 2) >> 1) & 1, ctl)))
                return false;
            tc_fence_after();
            split(it);
            g2 = g2s[it & 3];
            tc_fence_before();
            mbar_arrive(bar_split + (it & 1));
            mbar_arrive(bar_fdone + (it & 3));
            return true;
        };
        if (nchunks > 0) {
            if (p.store_h) store_h(0);
            ok = do_split(0);
        }
        for (int it = 0; ok && it < nchunks; ++it) {
            const float g2_cur = g2;
            if (it + 1 < nchunks && !do_split(it + 1)) {
                ok = false;
                break;
            }
            if (!mbar_wait(bar_mma + (it & 1), (it >> 1) & 1, ctl)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float fd = exp2f(g2_cur);
            gsum2 += g2_cur;
            {
                uint32_t r0[16], r1[16], r2[16];
                tmem_ld16(tq + L::TM_DS + qt * 48, r0);
                tmem_ld16(tq + L::TM_DS + qt * 48 + 16, r1);
                tmem_ld16(tq + L::TM_DS + qt * 48 + 32, r2);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    S[e] = fmaf(fd, S[e], __uint_as_float(r0[e]));
                    S[16 + e] = fmaf(fd, S[16 + e], __uint_as_float(r1[e]));
                    S[32 + e] = fmaf(fd, S[32 + e], __uint_as_float(r2[e]));
                }
            }
            tc_fence_before();
            mbar_arrive(bar_read);
            if (p.store_h && it + 1 < nchunks) store_h(it + 1);
        }
        if (ok) {
            const int sweep_end = REVERSE ? 0 : static_cast<int>(gridDim.x) - 1;
            const bool write_state = p.s_out && (!p.out_last_only || seg == sweep_end);
            if (write_state && GLA_DCHECK(unit < p.B * p.H && row < kDk, p.ctl.status)) {
                float* dst = p.cu_seqlens
                                 ? p.seg_states +
                                       (varlen_slot(p.cu_seqlens, b, seg, cps) * p.H + h) * (kDk * kDv) +
                                       row * kDv + qt * 48
                                 : p.s_out + unit * p.out_unit_stride + seg * p.out_seg_stride + row * kDv + qt * 48;
                if ((reinterpret_cast<uintptr_t>(dst) & 31) == 0) {
#pragma unroll
                    for (int e = 0; e < 48; e += 8) {
                        uint32_t w[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) w[i] = __float_as_uint(S[e + i]);
                        st_global_v8(dst + e, w);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 48; e += 4)
                        *reinterpret_cast<float4*>(dst + e) = make_float4(S[e], S[e + 1], S[e + 2], S[e + 3]);
                }
            }
            if (p.cu_seqlens && tid == 0)
                p.seg_g2[varlen_slot(p.cu_seqlens, b, seg, cps) * p.H + h] = gsum2;
            else if (p.g2_out && tid == 0)
                p.g2_out[static_cast<int64_t>(unit) * p.g2_unit_stride + seg] = gsum2;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, L::TMEM_COLS);
}

#endif  // GLA_CHUNK_KERNELS

}  // namespace gla
