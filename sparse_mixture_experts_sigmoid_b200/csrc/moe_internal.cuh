// Internal declarations shared by the CUDA translation units of libmoe.so.
// Not part of the public ABI (that is include/moe.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"  // include/ is on the include path

namespace moe {

// Device error flag bits (the flag lives in moe_api.cu; kernels get its address).
enum : uint32_t { kErrTimeout = 1u, kErrInput = 2u };

// ------------------------------------------------------------------ element helpers

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// Eight consecutive elements as fp32 from one 16-byte (bf16) or two 16-byte (fp32) loads.
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&v)[8]) {
    uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void load8(const float *p, float (&v)[8]) {
    float4 a = *reinterpret_cast<const float4 *>(p);
    float4 b = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
// Same, bypassing L1 (streamed once).
__device__ __forceinline__ void load8_stream(const __nv_bfloat16 *p, float (&v)[8]) {
    uint4 u = __ldcs(reinterpret_cast<const uint4 *>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void load8_stream(const float *p, float (&v)[8]) {
    float4 a = __ldcs(reinterpret_cast<const float4 *>(p));
    float4 b = __ldcs(reinterpret_cast<const float4 *>(p + 4));
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// silu(u) = u * sigmoid(u) = u / (1 + exp(-u)).  The fast divide is exact enough
// here: for u < -87 the denominator overflows to +inf or past 2^126 and the
// result flushes to zero, which is silu's limit there.
__device__ __forceinline__ float silu_f(float u) { return __fdividef(u, 1.0f + __expf(-u)); }

// Layout of the pre-activations a training forward keeps for the backward:
// rows (grouped rows, or tokens for the shared expert) of `words` 16-byte
// words (8 bf16 columns each: the gate columns, then the up columns), in
// blocks of 32 rows; inside a block, word j of its 32 rows is 512 contiguous
// bytes.  An epilogue warp holds 32 consecutive rows, one per thread, so each
// of its 16-byte stores (forward) and loads (backward) of one word covers
// whole lines.  Byte offset of word j of row r; the buffer holds rows rounded
// up to a multiple of 32.
__device__ __forceinline__ int64_t hpre_offset(int64_t r, int j, int words) {
    return (((r >> 5) * words + j) << 9) + ((r & 31) << 4);
}
inline int64_t hpre_rows(int64_t rows) { return (rows + 31) / 32 * 32; }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ------------------------------------------------------------------ kernel launchers
// Each returns the launch's cudaError_t (cudaGetLastError after the launch).

struct RouterArgs {
    const void *x, *w_router, *w_shared_gate;
    int64_t T;
    int d, E, k, norm_topk, score;
    int32_t *ids;
    float *gates, *probs, *shared_gate;
    float *zero_rows;   // optional [T, d] fp32 buffer to clear (the combine accumulator)
    uint32_t *err;      // device error word
    int32_t *hist;      // optional [B, E+1] block histogram for grouping (tensor-core router only)
    int hist_chunk;     // assignments per histogram block
    const float *bias;  // optional [E] balance bias: selection key = score + bias
    float *stats;       // optional [router_stats_rows(T), E] per-CTA score sums (fixed order)
    float *score_mean;  // optional [E] out: mean score per expert (needs stats)
    // optional, T == 1 only (the one-token router): the grouping of the token's
    // k assignments, written by the router itself (no separate grouping step)
    int32_t *counts, *offsets, *sorted_rows, *inv_rows;
};
// Rows of per-CTA score sums the routers write for the score-mean statistic:
// one per token for the one-token-per-CTA router (T <= 64), else at most one
// per 8 tokens.
inline int64_t router_stats_rows(int64_t T) { return T <= 64 ? T : (T + 7) / 8; }
// Sums the rows of a [rows, E] partial array in a fixed order and divides by
// T into score_mean (router_stats.cu).
cudaError_t launch_router_stats(const float *partial, int64_t rows, int E, int64_t T, float *score_mean,
                                cudaStream_t s);
// Router: the tensor-core logits GEMM + warp-per-token selection (router_tc.cu)
// when supported and scratch is given, else the CUDA-core routers (router.cu).
cudaError_t launch_router(const RouterArgs &a, int dtype, float *scratch, cudaStream_t s);
bool router_tc_supported(int64_t T, int E, int dtype);
size_t router_tc_workspace_bytes(int64_t T, int d, int E, bool shared);
cudaError_t launch_router_tc(const RouterArgs &a, float *scratch, cudaStream_t s);

struct PermuteArgs {
    const int32_t *ids;
    int R, E;
    int32_t *counts, *offsets, *sorted_rows, *inv_rows;
    uint32_t *err;
};
// table: scratch of permute_workspace_bytes(R, E) bytes, a [B, E+1] histogram of
// blocks of permute_chunk() assignments; table_ready: the router already filled it.
size_t permute_workspace_bytes(int64_t R, int E);
int permute_chunk();
cudaError_t launch_permute(const PermuteArgs &a, int32_t *table, bool table_ready, cudaStream_t s);

// A group of rows that one weight set serves: either the routed experts
// (offsets/sorted_rows give each expert's rows; the token of grouped row i is
// sorted_rows[i] / k) or one dense segment (the shared expert: row i is token i).
struct Segments {
    const int32_t *offsets;      // [E + 1]; NULL for the dense segment
    const int32_t *sorted_rows;  // [R]; NULL for the dense segment
    int E, k;                    // experts (1 for dense) and experts per token
    int64_t rows;                // R for routed, T for dense
};

struct SegGateUpArgs {
    const void *x, *w_gate, *w_up;   // x [T, d]; weights [E, hid, d]
    Segments seg;
    int64_t T;
    int d, hid;
    void *act;                       // [rows, hid]
};
cudaError_t launch_seg_gateup(const SegGateUpArgs &a, int dtype, cudaStream_t s, uint32_t *err);

struct SegDownArgs {
    const void *act, *w_down;        // act [rows, hid]; w_down [E, d, hid]
    Segments seg;
    int64_t T;
    int d, hid;
    const float *gates;              // routed: [R] gate per assignment; dense: [T] per token
    float *y_acc;                    // [T, d] fp32, accumulated into
    float *slots;                    // optional, routed only: [R, d] fp32 rows by assignment,
                                     // stored instead of added into y_acc (ordered combine)
};
cudaError_t launch_seg_down(const SegDownArgs &a, int dtype, cudaStream_t s, uint32_t *err);

// Small-batch down projection + combine written straight into y (no accumulator).
struct DownDirectArgs {
    const void *act, *w_down;          // act [R, h] grouped order; w_down [E, d, h]
    const int32_t *ids, *inv_rows;     // [T*k]
    const float *gates;                // [T*k]
    const void *act_shared, *sh_down;  // shared expert: act_shared [T, h_shared], sh_down [d, h_shared]; or null
    const float *shared_gate;          // [T]
    int64_t T;
    int d, h, E, k, h_shared;
    void *y;                           // [T, d]
};
cudaError_t launch_down_direct(const DownDirectArgs &a, int dtype, cudaStream_t s, uint32_t *err);

cudaError_t launch_finalize(const float *y_acc, void *y, int64_t n, cudaStream_t s);
// Ordered combine: y[t] = ((slots[t*k] + slots[t*k + 1]) + ... + slots[t*k + k-1]) (+ shared[t]),
// each row d floats; shared may be nullptr and may alias y (dtype MOE_F32).
cudaError_t launch_finalize_ordered(const float *slots, const float *shared, void *y, int64_t T, int d, int k,
                                    int dtype, cudaStream_t s);

// 4-bit routed experts on the small-batch path (segment_q4.cu).  A 4-bit
// weight matrix [rows, cols] is q [rows, cols / 2] (nibble code + 8, even
// element low) and scales [rows, cols / 64] (fp32, per group of 64).
struct SegGateUpQ4Args {
    const void *x;                       // [T, d] bf16
    const uint8_t *q_gate, *q_up;        // [E * hid, d / 2]
    const float *s_gate, *s_up;          // [E * hid, d / 64]
    Segments seg;
    int64_t T;
    int d, hid;
    void *act;                           // [rows, hid] bf16
};
struct DownDirectQ4Args {
    const void *act;                     // [R, h] bf16, grouped order
    const uint8_t *q_down;               // [E * d, h / 2]
    const float *s_down;                 // [E * d, h / 64]
    const int32_t *ids, *inv_rows;
    const float *gates;
    const void *act_shared, *sh_down;    // bf16 shared expert, or null
    const float *shared_gate;
    int64_t T;
    int d, h, E, k, h_shared;
    void *y;                             // [T, d] bf16
};
cudaError_t launch_quantize_q4(const void *w, int dtype, int64_t rows, int cols, uint8_t *q, float *scales,
                               cudaStream_t s);
cudaError_t launch_seg_gateup_q4(const SegGateUpQ4Args &a, cudaStream_t s, uint32_t *err);
// The same two steps with the codes streamed through a shared-memory ring by
// TMA (segment_q4_tma.cu), for d and h multiples of 256 and 16-byte aligned
// codes and scales; the down kernel writes y, adding shared_add [T, d] fp32
// (the shared expert's rows) when it is not null.
bool q4_tma_supported(int d, int h, const void *x, const void *q_gate, const float *s_gate, const void *q_up, const float *s_up,
                      const void *q_down, const float *s_down);
cudaError_t launch_q4t_gateup(const SegGateUpQ4Args &a, cudaStream_t s);
cudaError_t launch_down_direct_q4(const DownDirectQ4Args &a, cudaStream_t s, uint32_t *err);
cudaError_t launch_q4t_down(const DownDirectQ4Args &a, const float *shared_add, cudaStream_t s);

// Tensor-core grouped GEMM (grouped_gemm.cu).
struct GemmParams {
    const int32_t *offsets;      // [E + 1] grouped row offsets; nullptr: one dense segment of `rows` rows
    const int32_t *sorted_rows;  // grouped row -> assignment t*k + j (routed only)
    int E, k;
    int64_t rows;                // grouped rows (R routed, T dense)
    int64_t T;
    int K, N;                    // reduction length and output width
    const void *x;               // gather source [T, K] (gate/up of routed experts)
    void *act;                   // gate/up output [rows, N]
    float *y_acc;                // down output [T, N] fp32, accumulated into
    const float *gates;          // down: routed [R] by assignment, dense [T]
    uint32_t *err;
    bool stream_weights;         // each weight tile is read by one tile only: load it evict-first
    float *zero;                 // gate/up only, optional: [zero_floats] fp32 to clear (the
    int64_t zero_floats;         // down GEMM's accumulator), spread over the CTAs
    // kEarly* bits: what the kernel may read before the previous kernel in the
    // stream has completed (see pdl_wait).  Set only where every kernel between
    // the producer of that data and this one is known.
    int early;
    void *hpre;                  // gate/up only, optional: the pre-activations (gate | up, 2N
                                 // columns) kept for the backward pass, in the hpre_offset layout
    float *slot_out;             // down only, optional: [R, N] fp32 rows by assignment (routed) or
                                 // token (dense), stored instead of added into y_acc
    int n_groups;                // column tiles run in this many consecutive groups (decode_n); 0, 1: one
};
enum : int {
    kEarlyTiles = 1,   // offsets (and hence the tile list) and the weights
    kEarlyA = 2,       // the contiguous A operand
    // the weights of the tile each CTA would take first if every expert had
    // one row tile, fetched into L2 while the grouping kernels still run (a
    // wrong guess costs only the bandwidth)
    kEarlyPrefetch = 4,
};
struct GemmLaunch {
    int mode;             // 0: gate/up with SwiGLU epilogue, 1: down with gate-weighted combine
    bool gather;          // A rows gathered from x by index (routed gate/up); else TMA from a_src
    int dtype;            // MOE_BF16 or MOE_F32 (tf32 MMA)
    bool narrow;          // MMA N = 128 instead of N = 256
    bool pair;            // two SMs per tile (clusters of two CTAs, M = 256 MMAs)
    bool half;            // contiguous A only: 64-row tiles with 64-row A stages (few rows per group)
    GemmParams p;
    const void *a_src;    // contiguous A operand [rows, K] when !gather
    const void *b0, *b1;  // weights [E*N, K] (b1: up projection for gate/up)
};
cudaError_t launch_grouped_gemm(const GemmLaunch &L, cudaStream_t s);
cudaError_t launch_grouped_gemm_pair(const GemmLaunch &L, cudaStream_t s);

// Fused gate/up + SwiGLU + down + combine for layers whose experts average at
// most one 128-row tile (grouped_fused.cu).  y_acc must be zero on entry.
bool fused_expert_supported(const moe_config &c);
cudaError_t launch_fused_expert(const moe_config &c, const void *x, const void *wg, const void *wu, const void *wd,
                                const int32_t *offsets, const int32_t *srt, const float *gates, float *y_acc,
                                uint32_t *err, cudaStream_t s);

// Backward grouped GEMMs (grouped_bwd.cu).  An operand tensor: row-major
// [rows, cols] bf16 with a row stride of ld elements.
struct BwdOperand {
    const void *base;
    uint64_t rows, cols, ld;
};
struct BwdGemm {
    // SWIGLU: rows x N tiles, r = W^T dy with the SwiGLU-backward epilogue;
    // SCATTER: rows x N tiles added (weight 1) into acc[token];
    // WEIGHT: per group, M x N weight-gradient tiles reduced over the group's rows.
    enum Kind { SWIGLU, SCATTER, WEIGHT } kind;
    bool padded;                  // routed operands in the padded grouped layout (64-row aligned segments)
    BwdOperand a0, a1, b0, b1;    // TMA operands (a1/b1: second K range or second half)
    const int32_t *offsets, *sorted_rows;   // grouping (offsets == nullptr: one dense segment)
    int groups, k;
    int64_t rows, T;
    int nranges, Kr, N, M, halves;
    const void *hpre;             // SWIGLU: pre-activations (u | v, 2N columns), hpre_offset layout
    const float *gate;            // SWIGLU: routed [R] by assignment / dense [T]
    void *dh, *ga;                // SWIGLU out: [rows, 2N] du | dv, [rows, N] gate * a
    float *dgate;                 // SWIGLU: accumulated gate gradients
    float *acc;                   // SCATTER: [T, N] fp32
    void *out0, *out1;            // WEIGHT: [groups * M, N] per half
    bool out_f32;
    uint32_t *err;
};
cudaError_t launch_bwd_gemm(const BwdGemm &L, cudaStream_t s);

// Parts of the workspace (see moe_workspace_layout); the training parts exist
// only in the layout of a training step.
enum WsPart {
    P_IDS, P_GATES, P_SG, P_COUNTS, P_OFFSETS, P_SORTED, P_INV, P_ACT, P_ACTS, P_YACC, P_PERM, P_LOGITS,
    P_STATS,
    // training: kept by moe_forward_train for moe_backward, and the backward's scratch
    P_PROBS, P_HPRE, P_HPRES, P_DG, P_DSG, P_DH, P_DHS, P_GAS, P_DLB, P_DLS, P_XG, P_DYG, P_GA,
    P_SLOTS,   // ordered combine: [T*k, d] fp32 gate-weighted expert rows by assignment
    P_N
};
struct WsLayout {
    size_t off[P_N];
    size_t size[P_N];
    size_t total;
};
WsLayout ws_layout(const moe_config &c, bool train);
template <typename T>
T *ws_part(void *ws, const WsLayout &L, WsPart p) {
    return L.size[p] ? reinterpret_cast<T *>(static_cast<char *>(ws) + L.off[p]) : nullptr;
}
// Row stride (elements) of the bf16 router-gradient rows: E rounded up to 8.
inline int dl_stride(int E) { return (E + 7) / 8 * 8; }
// Rows of the backward's padded grouped layout (each expert's segment rounded
// up to a multiple of 64 rows): at most R + 63 E.
inline int64_t padded_rows(int64_t R, int E) { return R + 63LL * E; }

// Launch planning shared by the entry points (defined in moe_api.cu).
uint32_t *device_error_word();   // the library's device error word on the current device
// Down projection and combine of moe_combine / moe_combine_noalloc.  buf holds
// combine_scratch_floats(c) floats: the fp32 accumulator [T, d] (MOE_COMBINE_ADD
// with bf16; unused with f32, where y accumulates) or the slot rows [T*k, d]
// (MOE_COMBINE_ORDERED).
size_t combine_scratch_floats(const moe_config &c);
cudaError_t launch_combine(const moe_config &c, const void *act, const void *w_down, const int32_t *offsets,
                           const int32_t *srt, const float *gates, void *y, float *buf, cudaStream_t s,
                           uint32_t *err);

int num_sms();

// Counts one kernel launch (for moe_launch_count).
void note_launch();

// ------------------------------------------------------------------ programmatic dependent launch
// Every kernel of a pass is launched with programmatic stream serialization, so
// the next kernel in the stream can be scheduled (and run its prologue: barrier
// set-up, TMEM allocation, tensor-map prefetch) while this one drains.  Each
// kernel calls pdl_wait() before it touches data the previous kernel may still
// be writing (or reading) -- it returns once every earlier kernel of the
// stream has completed and its writes are visible -- and calls
// pdl_launch_dependents() only after its own pdl_wait() has returned and its
// TMEM (if any) is allocated.  Hence (a) a dependent CTA never holds TMEM that
// an earlier CTA on the same SM still has to allocate, and (b) when a kernel
// starts, every kernel two or more places back in the stream has completed,
// so data produced there (and the layer's inputs) may be read before
// pdl_wait().  Without the launch attribute both calls are no-ops.  MOE_PDL=0
// in the environment launches without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

bool pdl_enabled();

// Launches kern<<<grid, block, smem, s>>>(args...) with the attribute above and
// counts it.
template <typename... P, typename... A>
cudaError_t launch_kernel(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, A &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<A &&>(args)...);
    note_launch();
    return e;
}

// The same for a kernel launched in clusters of two CTAs along x.
template <typename... P, typename... A>
cudaError_t launch_kernel_pair(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                               A &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<A &&>(args)...);
    note_launch();
    return e;
}

}  // namespace moe
