// Grouping of the T*k (token, slot) assignments by expert: per-expert counts,
// their exclusive prefix sum, the stable permutation and its inverse.
//
// "Tutorial 11: Mixture of Experts (MoE)", section 3 "Expert Computation",
// Step 1 (argsort of the flattened expert ids groups each expert's rows; Step
// 3 unsorts with the inverse index); "Small MoE Architecture, in depth"
// (per-expert load by bincount).
//
// Over blocks of kChunk consecutive assignments:
//  1. histogram: per block and expert, the number of assignments, in a
//     [B, E+1] table (the last column counts out-of-range ids).  Either the
//     histogram kernel below builds it (each CTA counts its block in shared
//     memory; lanes holding the same expert are grouped with __match_any_sync
//     so one lane adds the group's size) or the router's selection kernel
//     accumulates it while it writes the ids.
//  2. scan + scatter: each CTA derives the per-expert counts, their exclusive
//     scan (the offsets) and its block's start for each expert from the table,
//     then ranks its assignments inside the block -- lane rank in the match
//     group plus the counts of earlier warps for the same expert -- so rows of
//     one expert keep increasing r order (a stable sort by expert).
// An out-of-range id anywhere reports MOE_ERR_DEVICE_INPUT, publishes empty
// experts and writes no permutation.  Up to kChunk assignments everything runs
// in one CTA.
#include "moe_internal.cuh"

namespace moe {
namespace {

#ifndef MOE_PERMUTE_CHUNK
#define MOE_PERMUTE_CHUNK 1024
#endif
constexpr int kChunk = MOE_PERMUTE_CHUNK;   // assignments per block
constexpr int kThreads = kChunk;            // one assignment per thread in the scatter
constexpr int kWarps = kThreads / 32;

__global__ void __launch_bounds__(256) hist_kernel(PermuteArgs a, int32_t *table) {
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ int32_t cnt[];   // [E + 1]
    const int b = blockIdx.x;
    for (int i = threadIdx.x; i <= a.E; i += blockDim.x) cnt[i] = 0;
    __syncthreads();
    const int beg = b * kChunk, end = min(a.R, beg + kChunk);
    for (int r0 = beg; r0 < end; r0 += blockDim.x) {
        const int r = r0 + threadIdx.x;
        int e = -1;
        if (r < end) {
            e = a.ids[r];
            if (e < 0 || e >= a.E) e = a.E;   // counted in the error column
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&cnt[e], __popc(peers));
    }
    __syncthreads();
    int32_t *row = table + (int64_t)b * (a.E + 1);
    for (int i = threadIdx.x; i <= a.E; i += blockDim.x) row[i] = cnt[i];
}

// Scan + stable scatter: every CTA reads the whole [B, E+1] histogram table,
// forms the per-expert totals, their exclusive scan (the offsets) and the
// start of its own block's rows of each expert, then ranks its assignments
// (lane rank in the match group plus the counts of earlier warps).  CTA 0
// publishes counts and offsets.  A non-zero error column anywhere reports
// MOE_ERR_DEVICE_INPUT, publishes empty experts and writes nothing else.
__global__ void __launch_bounds__(kThreads) scatter_kernel(PermuteArgs a, const int32_t *table, int nblocks) {
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ int32_t sm[];
    int32_t *wc = sm;                       // [kWarps][E]: per-warp counts, then per-warp starts
    int32_t *tot = wc + kWarps * a.E;       // [E]
    int32_t *base = tot + a.E;              // [E] start of this block's rows of each expert
    int32_t *off = base + a.E;              // [E + 1]
    __shared__ int bad;
    const int b = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < kWarps * a.E; i += kThreads) wc[i] = 0;
    if (threadIdx.x == 0) bad = 0;
    __syncthreads();
    for (int e = threadIdx.x; e <= a.E; e += kThreads) {
        int t = 0, before = 0;
#pragma unroll 4
        for (int q = 0; q < nblocks; ++q) {
            const int c = table[(int64_t)q * (a.E + 1) + e];
            t += c;
            before += q < b ? c : 0;
        }
        if (e < a.E) {
            tot[e] = t;
            base[e] = before;
        } else if (t) {
            bad = 1;
        }
    }
    __syncthreads();
    if (bad) {
        if (b == 0) {
            for (int i = threadIdx.x; i <= a.E; i += kThreads) {
                a.offsets[i] = 0;
                if (i < a.E) a.counts[i] = 0;
            }
            if (threadIdx.x == 0) atomicOr(a.err, kErrInput);
        }
        return;
    }
    if (warp == 0) {
        int carry = 0;
        for (int e0 = 0; e0 < a.E; e0 += 32) {
            const int e = e0 + lane;
            const int v = e < a.E ? tot[e] : 0;
            int in = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, in, o);
                if (lane >= o) in += u;
            }
            if (e < a.E) off[e] = carry + in - v;
            carry += __shfl_sync(0xffffffffu, in, 31);
        }
        if (lane == 0) off[a.E] = carry;
    }
    __syncthreads();
    if (b == 0)
        for (int e = threadIdx.x; e <= a.E; e += kThreads) {
            a.offsets[e] = off[e];
            if (e < a.E) a.counts[e] = tot[e];
        }
    const int r = b * kChunk + threadIdx.x;
    const int e = r < a.R ? a.ids[r] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && lane == __ffs(peers) - 1) wc[warp * a.E + e] = __popc(peers);
    __syncthreads();
    for (int x = threadIdx.x; x < a.E; x += kThreads) {
        int run = off[x] + base[x];
        for (int w = 0; w < kWarps; ++w) {
            const int c = wc[w * a.E + x];
            wc[w * a.E + x] = run;
            run += c;
        }
    }
    __syncthreads();
    if (e >= 0) {
        const int pos = wc[warp * a.E + e] + rank;
        a.sorted_rows[pos] = r;
        a.inv_rows[r] = pos;
    }
}

// All three steps in one CTA when every assignment fits in one block
// (R <= kChunk): per-warp counts, scans over warps and experts, scatter.
__global__ void __launch_bounds__(kThreads) permute_small_kernel(PermuteArgs a) {
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ int32_t sm[];
    int32_t *wc = sm;                       // [kWarps][E]
    int32_t *tot = sm + kWarps * a.E;       // [E]
    int32_t *off = tot + a.E;               // [E + 1]
    __shared__ int bad;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < kWarps * a.E; i += kThreads) wc[i] = 0;
    if (threadIdx.x == 0) bad = 0;
    __syncthreads();
    const int r = threadIdx.x;
    int e = r < a.R ? a.ids[r] : -1;
    if (r < a.R && (e < 0 || e >= a.E)) {
        bad = 1;
        e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && lane == __ffs(peers) - 1) wc[warp * a.E + e] = __popc(peers);
    __syncthreads();
    if (bad) {
        for (int i = threadIdx.x; i <= a.E; i += kThreads) {
            a.offsets[i] = 0;
            if (i < a.E) a.counts[i] = 0;
        }
        if (threadIdx.x == 0) atomicOr(a.err, kErrInput);
        return;
    }
    for (int x = threadIdx.x; x < a.E; x += kThreads) {
        int run = 0;
        for (int w = 0; w < kWarps; ++w) {
            const int c = wc[w * a.E + x];
            wc[w * a.E + x] = run;
            run += c;
        }
        tot[x] = run;
    }
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < a.E; base += 32) {
            const int x = base + lane;
            const int v = x < a.E ? tot[x] : 0;
            int in = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, in, o);
                if (lane >= o) in += u;
            }
            if (x < a.E) off[x] = carry + in - v;
            carry += __shfl_sync(0xffffffffu, in, 31);
        }
        if (lane == 0) off[a.E] = carry;
    }
    __syncthreads();
    for (int x = threadIdx.x; x <= a.E; x += kThreads) {
        a.offsets[x] = off[x];
        if (x < a.E) a.counts[x] = tot[x];
    }
    if (e >= 0) {
        const int pos = off[e] + wc[warp * a.E + e] + rank;
        a.sorted_rows[pos] = r;
        a.inv_rows[r] = pos;
    }
}

}  // namespace

size_t permute_workspace_bytes(int64_t R, int E) {
    const int64_t nblocks = (R + kChunk - 1) / kChunk;
    return sizeof(int32_t) * (size_t)nblocks * (E + 1);
}

cudaError_t launch_permute(const PermuteArgs &a, int32_t *table, bool table_ready, cudaStream_t s) {
    if (a.R <= 0) {
        // no assignments: every expert is empty
        cudaError_t e = cudaMemsetAsync(a.offsets, 0, sizeof(int32_t) * (a.E + 1), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(a.counts, 0, sizeof(int32_t) * a.E, s);
        return e;
    }
    if (a.R <= kChunk) {
        const size_t smem = sizeof(int32_t) * ((size_t)kWarps * a.E + 2 * (size_t)a.E + 1);
        cudaError_t e = cudaFuncSetAttribute(permute_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        return launch_kernel(permute_small_kernel, 1, kThreads, smem, s, a);
    }
    const int nblocks = (a.R + kChunk - 1) / kChunk;
    if (!table_ready) {
        const cudaError_t e = launch_kernel(hist_kernel, nblocks, 256, sizeof(int32_t) * (a.E + 1), s, a, table);
        if (e != cudaSuccess) return e;
    }
    const size_t smem = sizeof(int32_t) * ((size_t)kWarps * a.E + 3 * (size_t)a.E + 1);
    cudaError_t e = cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(scatter_kernel, nblocks, kThreads, smem, s, a, static_cast<const int32_t *>(table), nblocks);
}

int permute_chunk() { return kChunk; }

}  // namespace moe
