// Small-batch grouped expert kernels (CUDA cores): one warp per (expert,
// output row).  The warp streams that weight row once with 16-byte loads and
// applies it to every grouped row of the expert, so weights are read once per
// call; this is the bandwidth-bound path for decode-sized batches, where an
// expert sees a handful of rows and a tensor-core tile would be mostly empty.
//
//   gate/up : act[i, n] = silu(W_gate[e, n] . x_t) * (W_up[e, n] . x_t)
//   down    : y_acc[t, n] += g_i * (W_down[e, n] . act[i])
//
// "Tutorial 11: Mixture of Experts (MoE)", section 3, Steps 2-3 (grouped
// expert linears, silu(gate) * up, weighted sum); "Small MoE Architecture, in
// depth", Expert.forward (the SwiGLU expert) and the batch-1 decode remarks in
// "Why small changes the MoE trade-off" (decode reads only the chosen experts).
#include <algorithm>

#include "segment_parts.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using seg::kThreads;
using seg::kWarps;
using seg::list_experts;
using seg::grid_for;
constexpr int RB = 4;  // grouped rows per pass over a weight row

__device__ __forceinline__ float dot8(const float (&a)[8], const float (&b)[8], float acc) {
#pragma unroll
    for (int u = 0; u < 8; ++u) acc = fmaf(a[u], b[u], acc);
    return acc;
}

// RG grouped rows per pass over a weight row pair: 4 in general, 1 for a
// single token (each chosen expert then owns exactly one row), where the
// smaller register footprint lets more warps, and so more weight bytes, be in
// flight per SM.
template <typename T, int RG>
__global__ void __launch_bounds__(kThreads) seg_gateup_kernel(SegGateUpArgs a, uint32_t *err) {
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ int sm[];
    int *list = sm, *beg = sm + a.seg.E, *end = sm + 2 * a.seg.E;
    const int ne = list_experts(a.seg, list, beg, end);
    const T *x = static_cast<const T *>(a.x);
    const T *wg = static_cast<const T *>(a.w_gate);
    const T *wu = static_cast<const T *>(a.w_up);
    T *act = static_cast<T *>(a.act);
    const int lane = threadIdx.x & 31;
    const int64_t nitems = (int64_t)ne * a.hid;
    const int64_t gw = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int64_t nw = (int64_t)gridDim.x * kWarps;
    for (int64_t item = gw; item < nitems; item += nw) {
        const int li = (int)(item / a.hid);
        const int n = (int)(item - (int64_t)li * a.hid);
        const int e = list[li];
        const T *grow = wg + ((int64_t)e * a.hid + n) * a.d;
        const T *urow = wu + ((int64_t)e * a.hid + n) * a.d;
        for (int r0 = beg[li]; r0 < end[li]; r0 += RG) {
            int64_t tok[RG];
#pragma unroll
            for (int b = 0; b < RG; ++b) {
                const int r = r0 + b;
                int64_t t = -1;
                if (r < end[li]) {
                    // range-check the assignment before deriving its token
                    const int v = a.seg.sorted_rows ? a.seg.sorted_rows[r] : r;
                    t = (v >= 0 && v < a.seg.rows) ? (a.seg.sorted_rows ? v / a.seg.k : v) : -1;
                    if (t < 0 || t >= a.T) {
                        if (lane == 0) atomicOr(err, kErrInput);
                        t = -1;
                    }
                }
                tok[b] = t;
            }
            float ag[RG], au[RG];
#pragma unroll
            for (int b = 0; b < RG; ++b) ag[b] = au[b] = 0.f;
            // four 256-column chunks per round: 8 weight loads in flight per lane
            int c = lane * 8;
            for (; c + 3 * 256 < a.d; c += 4 * 256) {
                float gv[4][8], uv[4][8];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    load8_stream(grow + c + u * 256, gv[u]);
                    load8_stream(urow + c + u * 256, uv[u]);
                }
#pragma unroll
                for (int b = 0; b < RG; ++b) {
                    if (tok[b] >= 0) {
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            float xv[8];
                            load8(x + tok[b] * a.d + c + u * 256, xv);
                            ag[b] = dot8(gv[u], xv, ag[b]);
                            au[b] = dot8(uv[u], xv, au[b]);
                        }
                    }
                }
            }
            for (; c < a.d; c += 256) {
                float gv[8], uv[8];
                load8_stream(grow + c, gv);
                load8_stream(urow + c, uv);
#pragma unroll
                for (int b = 0; b < RG; ++b) {
                    if (tok[b] >= 0) {
                        float xv[8];
                        load8(x + tok[b] * a.d + c, xv);
                        ag[b] = dot8(gv, xv, ag[b]);
                        au[b] = dot8(uv, xv, au[b]);
                    }
                }
            }
#pragma unroll
            for (int b = 0; b < RG; ++b) {
                const float g = warp_sum(ag[b]);
                const float u = warp_sum(au[b]);
                if (lane == b && tok[b] >= 0) act[(int64_t)(r0 + b) * a.hid + n] = from_f32<T>(silu_f(g) * u);
            }
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) seg_down_kernel(SegDownArgs a, uint32_t *err) {
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ int sm[];
    int *list = sm, *beg = sm + a.seg.E, *end = sm + 2 * a.seg.E;
    const int ne = list_experts(a.seg, list, beg, end);
    const T *act = static_cast<const T *>(a.act);
    const T *wd = static_cast<const T *>(a.w_down);
    const int lane = threadIdx.x & 31;
    const int64_t nitems = (int64_t)ne * a.d;
    const int64_t gw = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int64_t nw = (int64_t)gridDim.x * kWarps;
    for (int64_t item = gw; item < nitems; item += nw) {
        const int li = (int)(item / a.d);
        const int n = (int)(item - (int64_t)li * a.d);
        const int e = list[li];
        const T *row = wd + ((int64_t)e * a.d + n) * a.hid;
        for (int r0 = beg[li]; r0 < end[li]; r0 += RB) {
            float acc[RB];
#pragma unroll
            for (int b = 0; b < RB; ++b) acc[b] = 0.f;
            const int nb = min(RB, end[li] - r0);
            for (int c = lane * 8; c < a.hid; c += 256) {
                float wv[8];
                load8_stream(row + c, wv);
#pragma unroll
                for (int b = 0; b < RB; ++b) {
                    if (b < nb) {
                        float av[8];
                        load8(act + (int64_t)(r0 + b) * a.hid + c, av);
                        acc[b] = dot8(wv, av, acc[b]);
                    }
                }
            }
#pragma unroll
            for (int b = 0; b < RB; ++b) {
                const float v = warp_sum(acc[b]);
                if (lane == b && b < nb) {
                    const int r = r0 + b;
                    const int64_t slot = a.seg.sorted_rows ? a.seg.sorted_rows[r] : r;
                    const int64_t t = a.seg.sorted_rows ? slot / a.seg.k : r;
                    if (slot < 0 || t >= a.T) {
                        atomicOr(err, kErrInput);
                    } else if (a.slots) {
                        a.slots[slot * a.d + n] = a.gates[slot] * v;   // ordered combine: own slot row
                    } else {
                        atomicAdd(a.y_acc + t * a.d + n, a.gates[slot] * v);
                    }
                }
            }
        }
    }
}

// Down projection and combine for small batches, written straight into y:
// one warp per output element (t, n) sums the k selected experts' rows
//   y[t, n] = sum_j g[t, j] * (W_down[e_j, n] . act[inv(t*k + j)])
//           (+ sigmoid gate * (S_down[n] . act_shared[t]) with a shared expert),
// streaming each weight row once with 16-byte loads, four chunks per round.
// No accumulator, no atomics and no separate conversion pass.  (Eight chunks
// per round measured slower on the Mixtral decode shape: 54.4 vs 46.7 us.)
template <typename T>
__device__ __forceinline__ float row_dot(const T *w, const T *v, int n, int lane) {
    float acc = 0.f;
    int c = lane * 8;
    for (; c + 3 * 256 < n; c += 4 * 256) {
        float wv[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u) load8_stream(w + c + u * 256, wv[u]);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float av[8];
            load8(v + c + u * 256, av);
            acc = dot8(wv[u], av, acc);
        }
    }
    for (; c < n; c += 256) {
        float wv[8], av[8];
        load8_stream(w + c, wv);
        load8(v + c, av);
        acc = dot8(wv, av, acc);
    }
    return acc;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) down_direct_kernel(DownDirectArgs a, uint32_t *err) {
    pdl_wait();
    pdl_launch_dependents();
    const T *act = static_cast<const T *>(a.act);
    const T *wd = static_cast<const T *>(a.w_down);
    T *y = static_cast<T *>(a.y);
    const int lane = threadIdx.x & 31;
    const int64_t nitems = a.T * a.d;
    const int64_t gw = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int64_t nw = (int64_t)gridDim.x * kWarps;
    for (int64_t item = gw; item < nitems; item += nw) {
        const int64_t t = item / a.d;
        const int n = (int)(item - t * a.d);
        float acc = 0.f;
        for (int j = 0; j < a.k; ++j) {
            const int64_t slot = t * a.k + j;
            const int e = a.ids[slot];
            const int r = a.inv_rows[slot];
            if (e < 0 || e >= a.E || r < 0 || r >= a.T * a.k) {
                if (lane == 0) atomicOr(err, kErrInput);
                continue;
            }
            acc += a.gates[slot] * row_dot(wd + ((int64_t)e * a.d + n) * a.h, act + (int64_t)r * a.h, a.h, lane);
        }
        if (a.sh_down) {
            const T *sd = static_cast<const T *>(a.sh_down);
            const T *as = static_cast<const T *>(a.act_shared);
            acc += a.shared_gate[t] * row_dot(sd + (int64_t)n * a.h_shared, as + t * a.h_shared, a.h_shared, lane);
        }
        acc = warp_sum(acc);
        if (lane == 0) y[item] = from_f32<T>(acc);
    }
}

template <typename T>
__global__ void finalize_kernel(const float *y_acc, T *y, int64_t n) {
    pdl_wait();
    pdl_launch_dependents();
    const int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
    if (i + 8 <= n) {
        const float4 a = *reinterpret_cast<const float4 *>(y_acc + i);
        const float4 b = *reinterpret_cast<const float4 *>(y_acc + i + 4);
        __align__(16) __nv_bfloat16 o[8] = {__float2bfloat16_rn(a.x), __float2bfloat16_rn(a.y),
                                            __float2bfloat16_rn(a.z), __float2bfloat16_rn(a.w),
                                            __float2bfloat16_rn(b.x), __float2bfloat16_rn(b.y),
                                            __float2bfloat16_rn(b.z), __float2bfloat16_rn(b.w)};
        *reinterpret_cast<uint4 *>(y + i) = *reinterpret_cast<const uint4 *>(o);
    } else {
        for (int64_t j = i; j < n; ++j) y[j] = __float2bfloat16_rn(y_acc[j]);
    }
    // The accumulator is scratch that the next call clears before use: once the
    // four lanes sharing a 128-byte line have consumed their values, drop the
    // line from L2 instead of writing it back to HBM.  Only whole, aligned lines
    // inside [y_acc, y_acc + n) are dropped (a caller's workspace need only be
    // 16-byte aligned).
    __syncwarp();
    if ((threadIdx.x & 3) == 0 && i + 32 <= n && (reinterpret_cast<uintptr_t>(y_acc + i) & 127) == 0)
        tc::l2_discard_line(y_acc + i);
}

// Ordered combine: each thread adds eight columns of a token's k slot rows in
// slot order, then the shared expert's row, and writes y.  d % 8 == 0.
template <typename T>
__global__ void finalize_ordered_kernel(const float *slots, const float *shared, T *y, int64_t chunks, int d,
                                        int k) {
    pdl_wait();
    pdl_launch_dependents();
    const int cpr = d / 8;   // chunks per row
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunks; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / cpr;
        const int c = (int)(i - t * cpr) * 8;
        const float *src = slots + t * k * (int64_t)d + c;
        float4 a = *reinterpret_cast<const float4 *>(src);
        float4 b = *reinterpret_cast<const float4 *>(src + 4);
        for (int j = 1; j < k; ++j) {
            const float4 p = *reinterpret_cast<const float4 *>(src + (int64_t)j * d);
            const float4 q = *reinterpret_cast<const float4 *>(src + (int64_t)j * d + 4);
            a = make_float4(a.x + p.x, a.y + p.y, a.z + p.z, a.w + p.w);
            b = make_float4(b.x + q.x, b.y + q.y, b.z + q.z, b.w + q.w);
        }
        if (shared) {
            const float4 p = *reinterpret_cast<const float4 *>(shared + t * d + c);
            const float4 q = *reinterpret_cast<const float4 *>(shared + t * d + c + 4);
            a = make_float4(a.x + p.x, a.y + p.y, a.z + p.z, a.w + p.w);
            b = make_float4(b.x + q.x, b.y + q.y, b.z + q.z, b.w + q.w);
        }
        T *dst = y + t * d + c;
        if constexpr (sizeof(T) == 2) {
            __align__(16) __nv_bfloat16 o[8] = {__float2bfloat16_rn(a.x), __float2bfloat16_rn(a.y),
                                                __float2bfloat16_rn(a.z), __float2bfloat16_rn(a.w),
                                                __float2bfloat16_rn(b.x), __float2bfloat16_rn(b.y),
                                                __float2bfloat16_rn(b.z), __float2bfloat16_rn(b.w)};
            *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(o);
        } else {
            *reinterpret_cast<float4 *>(dst) = a;
            *reinterpret_cast<float4 *>(dst + 4) = b;
        }
    }
}

}  // namespace

cudaError_t launch_seg_gateup(const SegGateUpArgs &a, int dtype, cudaStream_t s, uint32_t *err) {
    if (a.seg.rows <= 0) return cudaSuccess;
    const size_t smem = sizeof(int) * 3 * (size_t)a.seg.E;
    const int64_t items = (int64_t)a.seg.E * a.hid;
    auto go = [&](auto kern) { return launch_kernel(kern, grid_for(kern, items, smem), kThreads, smem, s, a, err); };
    if (dtype == MOE_F32) return a.T == 1 ? go(seg_gateup_kernel<float, 1>) : go(seg_gateup_kernel<float, RB>);
    return a.T == 1 ? go(seg_gateup_kernel<__nv_bfloat16, 1>) : go(seg_gateup_kernel<__nv_bfloat16, RB>);
}

cudaError_t launch_seg_down(const SegDownArgs &a, int dtype, cudaStream_t s, uint32_t *err) {
    if (a.seg.rows <= 0) return cudaSuccess;
    const size_t smem = sizeof(int) * 3 * (size_t)a.seg.E;
    const int64_t items = (int64_t)a.seg.E * a.d;
    auto go = [&](auto kern) { return launch_kernel(kern, grid_for(kern, items, smem), kThreads, smem, s, a, err); };
    return dtype == MOE_F32 ? go(seg_down_kernel<float>) : go(seg_down_kernel<__nv_bfloat16>);
}

cudaError_t launch_down_direct(const DownDirectArgs &a, int dtype, cudaStream_t s, uint32_t *err) {
    if (a.T <= 0) return cudaSuccess;
    auto go = [&](auto kern) { return launch_kernel(kern, grid_for(kern, a.T * a.d, 0), kThreads, 0, s, a, err); };
    return dtype == MOE_F32 ? go(down_direct_kernel<float>) : go(down_direct_kernel<__nv_bfloat16>);
}

cudaError_t launch_finalize(const float *y_acc, void *y, int64_t n, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    const int threads = 256;
    const int64_t blocks = (n / 8 + threads) / threads + 1;
    return launch_kernel(finalize_kernel<__nv_bfloat16>, (unsigned)blocks, threads, 0, s, y_acc,
                         static_cast<__nv_bfloat16 *>(y), n);
}

cudaError_t launch_finalize_ordered(const float *slots, const float *shared, void *y, int64_t T, int d, int k,
                                    int dtype, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    const int64_t chunks = T * (d / 8);
    const int threads = 256;
    const unsigned blocks = (unsigned)std::min<int64_t>((chunks + threads - 1) / threads, 8 * num_sms());
    if (dtype == MOE_F32)
        return launch_kernel(finalize_ordered_kernel<float>, blocks, threads, 0, s, slots, shared,
                             static_cast<float *>(y), chunks, d, k);
    return launch_kernel(finalize_ordered_kernel<__nv_bfloat16>, blocks, threads, 0, s, slots, shared,
                         static_cast<__nv_bfloat16 *>(y), chunks, d, k);
}

}  // namespace moe
