// Grouping of the T*k (token, slot) assignments by expert: per-expert counts,
// their exclusive prefix sum, the stable permutation and its inverse.
//
// "Tutorial 11: Mixture of Experts (MoE)", section 3 "Expert Computation",
// Step 1 (argsort of the flattened expert ids groups each expert's rows; Step
// 3 unsorts with the inverse index); "Small MoE Architecture, in depth"
// (per-expert load by bincount).
//
// One CTA of 32 warps.  Warp w owns the contiguous slice [w*S, (w+1)*S) of the
// assignments.  Pass 1 counts per (warp, expert) in shared memory; a 32-lane
// __match_any_sync groups the lanes holding the same expert so one lane adds
// the group's popcount (no atomics: a warp owns its counter row).  The counts
// are scanned over warps and over experts, so every (warp, expert) pair knows
// where its rows start.  Pass 2 walks the slice again in order; a lane's rank
// inside its match group plus the running per-(warp, expert) cursor is its
// position, which keeps the order of r inside each expert (stable).
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kWarps = 32;
constexpr int kThreads = kWarps * 32;

__global__ void __launch_bounds__(kThreads) permute_kernel(PermuteArgs a) {
    extern __shared__ int32_t sm[];
    int32_t *cnt = sm;                    // [kWarps][E]: counts, then start positions
    int32_t *tot = sm + kWarps * a.E;     // [E]
    int32_t *off = tot + a.E;             // [E + 1]
    __shared__ int32_t warp_tot[kWarps];
    __shared__ int bad;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < kWarps * a.E; i += kThreads) cnt[i] = 0;
    if (threadIdx.x == 0) bad = 0;
    __syncthreads();

    const int S = (a.R + kWarps - 1) / kWarps;
    const int beg = min(a.R, warp * S), end = min(a.R, beg + S);
    int32_t *mycnt = cnt + warp * a.E;

    // pass 1: per-warp counts
    for (int base = beg; base < end; base += 32) {
        const int r = base + lane;
        int e = r < end ? a.ids[r] : -1;
        if (r < end && (e < 0 || e >= a.E)) {
            bad = 1;
            e = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int leader = __ffs(peers) - 1;
        if (e >= 0 && lane == leader) mycnt[e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    if (bad) {
        // invalid input: report it and leave every expert empty so no later
        // stage reads through an out-of-range index
        for (int i = threadIdx.x; i <= a.E; i += kThreads) {
            a.offsets[i] = 0;
            if (i < a.E) a.counts[i] = 0;
        }
        if (threadIdx.x == 0) atomicOr(a.err, kErrInput);
        return;
    }
    // scan over warps for each expert
    for (int e = threadIdx.x; e < a.E; e += kThreads) {
        int run = 0;
        for (int w = 0; w < kWarps; ++w) {
            const int c = cnt[w * a.E + e];
            cnt[w * a.E + e] = run;
            run += c;
        }
        tot[e] = run;
    }
    __syncthreads();
    // exclusive scan over experts (E <= 1024 items, chunked per warp)
    {
        const int per = (a.E + kThreads - 1) / kThreads;   // items per thread (1 for E <= 1024)
        int local = 0;
        const int e0 = threadIdx.x * per;
        for (int i = 0; i < per; ++i)
            if (e0 + i < a.E) local += tot[e0 + i];
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int wv = warp_tot[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, wv, o);
                if (lane >= o) wv += v;
            }
            warp_tot[lane] = wv;   // inclusive over warps
        }
        __syncthreads();
        int run = incl - local + (warp > 0 ? warp_tot[warp - 1] : 0);
        for (int i = 0; i < per; ++i) {
            if (e0 + i < a.E) {
                off[e0 + i] = run;
                run += tot[e0 + i];
            }
        }
        if (threadIdx.x == kThreads - 1) off[a.E] = warp_tot[kWarps - 1];
    }
    __syncthreads();
    for (int e = threadIdx.x; e <= a.E; e += kThreads) {
        a.offsets[e] = off[e];
        if (e < a.E) a.counts[e] = tot[e];
    }
    // pass 2: stable scatter
    for (int base = beg; base < end; base += 32) {
        const int r = base + lane;
        const int e = r < end ? a.ids[r] : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int leader = __ffs(peers) - 1;
        const int rank = __popc(peers & ((1u << lane) - 1u));
        int pos = 0;
        if (e >= 0) pos = off[e] + mycnt[e] + rank;
        __syncwarp();
        if (e >= 0) {
            a.sorted_rows[pos] = r;
            a.inv_rows[r] = pos;
            if (lane == leader) mycnt[e] += __popc(peers);
        }
        __syncwarp();
    }
}

}  // namespace

cudaError_t launch_permute(const PermuteArgs &a, cudaStream_t s) {
    if (a.R <= 0) {
        // no assignments: every expert is empty
        cudaError_t e = cudaMemsetAsync(a.offsets, 0, sizeof(int32_t) * (a.E + 1), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(a.counts, 0, sizeof(int32_t) * a.E, s);
        return e;
    }
    const size_t smem = sizeof(int32_t) * ((size_t)kWarps * a.E + 2 * (size_t)a.E + 1);
    cudaError_t e = cudaFuncSetAttribute(permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    permute_kernel<<<1, kThreads, smem, s>>>(a);
    note_launch();
    return cudaGetLastError();
}

}  // namespace moe
