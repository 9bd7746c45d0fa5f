// Pieces shared by the small-batch (CUDA-core) expert kernels: the list of
// experts that own rows, and grid sizing by residency.
#pragma once

#include <mutex>
#include <unordered_map>

#include "moe_internal.cuh"

namespace moe {
namespace seg {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Builds, in shared memory, the list of experts that own at least one row.
__device__ inline int list_experts(const Segments &sg, int *list, int *beg, int *end) {
    __shared__ int s_n;
    if (sg.offsets == nullptr) {
        if (threadIdx.x == 0) {
            list[0] = 0;
            beg[0] = 0;
            end[0] = (int)sg.rows;
            s_n = 1;
        }
        __syncthreads();
        return s_n;
    }
    if (threadIdx.x == 0) s_n = 0;
    __syncthreads();
    // ordered compaction: each warp takes 32 experts at a time
    for (int base = 0; base < sg.E; base += kThreads) {
        const int e = base + threadIdx.x;
        int b = 0, en = 0;
        bool has = false;
        if (e < sg.E) {
            b = sg.offsets[e];
            en = sg.offsets[e + 1];
            has = en > b;
        }
        __shared__ int wcount[kWarps];
        const unsigned m = __ballot_sync(0xffffffffu, has);
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        if (lane == 0) wcount[warp] = __popc(m);
        __syncthreads();
        int before = s_n;
        for (int w = 0; w < warp; ++w) before += wcount[w];
        if (has) {
            const int pos = before + __popc(m & ((1u << lane) - 1u));
            list[pos] = e;
            beg[pos] = b;
            end[pos] = en;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int add = 0;
            for (int w = 0; w < kWarps; ++w) add += wcount[w];
            s_n += add;
        }
        __syncthreads();
    }
    return s_n;
}


// One warp per item, but no more CTAs than fit on the GPU at once: the
// kernels stream weights, so the warps resident per SM (and with them the
// bytes in flight) are what sets their rate.  The residency of each kernel is
// asked for once.
template <typename K>
inline int grid_for(K kern, int64_t items, size_t smem) {
    static std::mutex mu;
    static std::unordered_map<const void *, int> per_sm;
    int b = 0;
    {
        std::lock_guard<std::mutex> lk(mu);
        auto it = per_sm.find(reinterpret_cast<const void *>(kern));
        if (it != per_sm.end()) {
            b = it->second;
        } else {
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, kThreads, smem) != cudaSuccess || b < 1) b = 1;
            per_sm[reinterpret_cast<const void *>(kern)] = b;
        }
    }
    const int64_t cap = (int64_t)b * num_sms();
    const int64_t need = (items + kWarps - 1) / kWarps;
    return (int)(need < cap ? (need > 0 ? need : 1) : cap);
}


}  // namespace seg
}  // namespace moe
