// gla_internal.h -- declarations shared by the libgla translation units
// (host launchers, the wait-control block, tile constants).  Not part of the
// public ABI; the public ABI is include/gla.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime_api.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/gla.h"

namespace gla {

// Bounded-wait control passed by value to every kernel that waits.
struct WaitCtl {
    int* status;                   // device status word (first error wins)
    unsigned long long limit_ns;   // wall-time bound of each wait
};

// Chunk geometry of the tensor-core path.
constexpr int kChunk = 128;        // tokens per chunk (M of every MMA)
constexpr int kDk = 96;
constexpr int kDv = 192;

// Host-side helpers implemented in gla_host.cu.
WaitCtl wait_ctl_for_current_device(gla_status* err);
// The driver context current on this thread (opaque; null if unreadable):
// device addresses cached per device are valid only within it.
const void* current_cu_context();
gla_status check_launch(const char* what);
// GLA_ERR_CUDA for a failed runtime call, its code kept for gla_last_cuda_error.
gla_status status_of(cudaError_t e);
void count_launch(unsigned n = 1);

// Tracing: trace_begin() before a launch, trace_end() after it; both are
// no-ops unless tracing is enabled.  `name` must be a static string.
void trace_begin(cudaStream_t st);
void trace_end(cudaStream_t st, const char* name);

// Encode a tiled tensor map over a bf16 (or fp32) [d3][d2][d1][d0] tensor.
// dims[i] elements, strides_bytes[i] for i >= 1 (dim 0 contiguous), box[i].
gla_status make_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box, int elem_bytes,
                     int swizzle_bytes);

// ---- launchers (one per kernel family), all asynchronous on `st`.
gla_status launch_decode(float* state, const int32_t* slot_idx, int n_slots, const void* q, const void* k,
                         const void* v, const float* a, float* o, int N, int H, float scale,
                         int* status, cudaStream_t st);

gla_status launch_conv(const void* x, int apply_ln, const float* g, const float* b, float eps,
                       const float* w, const float* bias, const float* cs_in, float* cs_out,
                       void* y, int B, int T, int D, cudaStream_t st);

gla_status launch_conv_decode(const void* x, const int32_t* slot_idx, int n_slots, int apply_ln, const float* g,
                              const float* b, float eps, const float* w, const float* bias, float* hist,
                              void* y, int N, int D, WaitCtl ctl, cudaStream_t st);

size_t conv_bwd_workspace_bytes(int B, int T, int D);
gla_status launch_conv_bwd(const void* x, int apply_ln, const float* g, const float* be, float eps, const float* w,
                           const float* bias, const float* cs_in, const void* dy, void* dx, float* dw, float* dbias,
                           float* dgamma, float* dbeta, float* dcs, void* ws, int B, int T, int D, cudaStream_t st);

gla_status launch_fwd_f32(const float* q, const float* k, const float* v, const float* a,
                          const float* s0, float* o, float* s_final, int B, int T, int H,
                          int64_t ld_qk, int64_t ld_v, float scale, const WaitCtl& ctl,
                          cudaStream_t st);

// Chunked bf16 paths (chunk_fwd.cu / chunk_bwd.cu).
struct ChunkProblem {
    const void* q;
    const void* k;
    const void* v;
    const float* a;
    int B, T, H;
    int64_t ld_qk, ld_v;           // token strides in elements
    float scale;
};

size_t fwd_workspace_bytes(int B, int T, int H);
size_t bwd_workspace_bytes(int B, int T, int H, bool from_saved = false);

size_t varlen_workspace_bytes(int N, int total_T, int H);
gla_status run_chunk_fwd_varlen(const ChunkProblem& pr, const int* cu_seqlens, int N, const float* s0, void* o,
                                float* s_final, void* ws, size_t ws_bytes, const WaitCtl& ctl, cudaStream_t st);
// h_save (optional): the state entering each chunk as bf16 hi + lo planes,
// [B*H*NC][2][96][192], for gla_chunk_bwd from saved states.
gla_status run_chunk_fwd(const ChunkProblem& p, const float* s0, void* o, float* s_final,
                         void* ws, size_t ws_bytes, const WaitCtl& ctl, cudaStream_t st,
                         void* h_save = nullptr);

// saved / s_final (optional): the forward's saved states and final state;
// with them the forward state pass is skipped.
gla_status run_chunk_bwd(const ChunkProblem& p, const float* s0, const void* dO,
                         const float* ds_final, void* dq, void* dk, void* dv, float* da,
                         float* ds0, void* ws, size_t ws_bytes, const WaitCtl& ctl,
                         cudaStream_t st, const void* saved = nullptr, const float* s_final = nullptr);

gla_status launch_wait_selftest(const WaitCtl& ctl, cudaStream_t st);

// Inputs of one call for the checking build's precondition scan
// (debug_checks.cu): the decay a (<= 0 and finite), bf16 token tensors and
// fp32 states (finite).  debug_scan launches nothing in the normal build.
struct DebugScan {
    static constexpr int kMaxBf16 = 4, kMaxF32 = 2;
    struct Rows {
        const void* base;          // bf16; rows of `width` values, `ld` elements apart
        int64_t rows, ld, width;
    };
    const float* a = nullptr;
    int64_t na = 0;
    Rows bf16[kMaxBf16] = {};
    const float* f32[kMaxF32] = {};
    int64_t nf32[kMaxF32] = {};
};
gla_status debug_scan(const DebugScan& s, int* status, cudaStream_t st);

// Sequence split across ranks (chunk_seg.cu).
size_t segment_workspace_bytes(int B, int T, int H);
gla_status run_segment_state(const void* u, const void* y, const float* a, int B, int T, int H, int64_t ld_u,
                             int64_t ld_y, float scale, bool reverse, float* s_seg, float* g_seg, void* ws,
                             const WaitCtl& ctl, cudaStream_t st);
gla_status launch_state_fold(const float* s, const float* g, int n, int units, int reverse, const float* s_in,
                             float* out, cudaStream_t st);

// Shared by the forward and backward host code (chunk_fwd.cu).
struct StateParams;   // chunk_state.cuh
gla_status make_token_map(CUtensorMap* m, const void* base, int d, int H, int T, int B,
                          int64_t ld, int box_d, int swizzle, int box_rows = 128);
// [nstates][96][192] bf16 states; a box is box_states consecutive states
// (e.g. a state's hi and lo planes) of box_cols columns.
gla_status make_state_map(CUtensorMap* m, void* base, int64_t nstates, int box_cols = 64, int box_states = 1);
gla_status launch_state_kernel(bool with_o, bool reverse, const StateParams& p, dim3 grid,
                               cudaStream_t st);

// Segment plan of a unit's chunks when B*H alone cannot fill the GPU: nseg
// segments of cps chunks (the last may be shorter); nseg == 1 otherwise.
void chunk_segment_plan(int units, int NC, int* nseg, int* cps);
// In place over states [units][nseg][dk*dv]: slot g holds segment g's local
// state from zero on entry (L_g, or D_g in reverse) and, on return, the state
// entering segment g's sweep: S_0 folded forward over segments < g, or (reverse)
// dS_T folded right to left over segments > g.  s_edge (S_0 or dS_T) may be null.
gla_status launch_seg_combine(float* states, const float* g2, const float* s_edge, int nseg, int units,
                              bool reverse, cudaStream_t st);

}  // namespace gla
