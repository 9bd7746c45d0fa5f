// 4-bit routed experts for the small-batch (decode) path.
//
// "Small MoE Architecture, in depth": "Worked example: the batch-1 budget on
// a device" (4-bit weights, about half a byte per parameter: decode reads the
// k chosen experts' weights, so tokens/s follows the bytes per parameter) and
// "Running experts that do not fit: offloading and quantisation" (routed
// experts quantised more aggressively; shared expert and router kept at
// higher precision).  Format (this library's reading; the pages fix none):
// groups of 64 consecutive weights along a row (the reduction dimension),
// scale s = max|w| / 7 in fp32, code round(w / s) in [-7, 7] (ties to even),
// stored as nibble code + 8, two per byte, even element in the low nibble;
// the value represented is (nibble - 8) * s.
//
//   quantize_q4_kernel: one thread per group of 64 weights.
//   seg_gateup_q4_kernel: one warp per (expert, block of hidden rows): the
//     warp streams the 4-bit gate and up rows once (16 bytes = 32 weights per
//     lane per load, the group's scale alongside) and applies them to every
//     grouped row of the expert; act = silu(gate) * up in bf16.
//   down_direct_q4_kernel: one CTA per block of 4 output elements (t, n), the
//     reduction split over its warps: y = sum_j g_j (W_down[e_j, n] . act)
//     (+ the bf16 shared expert), written straight into y.
// The weights are dequantised in registers; accumulation is fp32.
#include <algorithm>

#include "segment_parts.cuh"

namespace moe {
namespace {

using seg::grid_for;
using seg::kThreads;
using seg::kWarps;
using seg::list_experts;

// One group of 64 weights -> 32 bytes of nibbles and one fp32 scale.  The
// code is decided in fp32: s = max|w| / 7 and w / s, each rounded once.
template <typename T>
__global__ void quantize_q4_kernel(const T *w, int64_t groups, int gpr, uint8_t *q, float *scales) {
    pdl_wait();
    pdl_launch_dependents();
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += (int64_t)gridDim.x * blockDim.x) {
        const T *src = w + g * 64;
        float v[64];
#pragma unroll
        for (int i = 0; i < 64; i += 8) {
            float t[8];
            load8(src + i, t);
#pragma unroll
            for (int j = 0; j < 8; ++j) v[i + j] = t[j];
        }
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) m = fmaxf(m, fabsf(v[i]));
        const float s = __fdiv_rn(m, 7.f);
        scales[g] = s;
        uint32_t out[8];
#pragma unroll
        for (int wd = 0; wd < 8; ++wd) {
            uint32_t word = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                int code = 0;
                if (s != 0.f) {
                    float c = rintf(__fdiv_rn(v[wd * 8 + j], s));
                    c = fminf(7.f, fmaxf(-7.f, c));
                    code = (int)c;
                }
                word |= (uint32_t)(code + 8) << (4 * j);
            }
            out[wd] = word;
        }
        uint4 *dst = reinterpret_cast<uint4 *>(q + g * 32);
        dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
        dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
        (void)gpr;
    }
}

// Dequantisation in the dot products: a nibble n placed in the low mantissa
// bits of 128.0f is the float 128 + n exactly, so for a 32-weight half group
// with scale s and activations x
//   sum_i (n_i - 8) s x_i = s (sum_i (128 + n_i) x_i - 136 sum_i x_i),
// and sum_i x_i is formed once per activation chunk and shared by every
// weight row that the chunk meets.  The products (128 + n) x are exact in
// fp32 (8 by 8 significant bits).  A 32-bit word of codes is split into its
// low nibbles (elements 0, 2, 4, 6, one per byte) and high nibbles (elements
// 1, 3, 5, 7) with one mask each, and a byte permute then builds each float
// from 0x43, the nibble's byte and two zero bytes.
__device__ __forceinline__ float nib_byte_f(uint32_t nibbles, int b) {
    return __uint_as_float(__byte_perm(nibbles, 0x43000000u, 0x7044u | ((uint32_t)b << 8)));
}

// 32 consecutive bf16 activations -> fp32 registers and their sum.
__device__ __forceinline__ float load32(const __nv_bfloat16 *v, float (&x)[32]) {
    float sum = 0.f;
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
        float t[8];
        load8(v + 8 * wd, t);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            x[8 * wd + j] = t[j];
            sum += t[j];
        }
    }
    return sum;
}

// sum_i (128 + n_i) x_i over the 32 nibbles of one 16-byte load (two
// accumulators, so the fma chain is half as long).
__device__ __forceinline__ float dot32_raw(const uint4 &qw, const float (&x)[32]) {
    const uint32_t words[4] = {qw.x, qw.y, qw.z, qw.w};
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
        const uint32_t lo = words[wd] & 0x0F0F0F0Fu;
        const uint32_t hi = (words[wd] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            acc0 = fmaf(nib_byte_f(lo, b), x[8 * wd + 2 * b], acc0);
            acc1 = fmaf(nib_byte_f(hi, b), x[8 * wd + 2 * b + 1], acc1);
        }
    }
    return acc0 + acc1;
}

// Grouped gate/up of the routed experts from 4-bit weights: one warp per
// (listed expert, block of NR hidden rows), RG grouped rows per pass; each
// activation chunk a lane loads (32 values) feeds the NR gate and NR up rows.
template <int RG, int NR>
__global__ void __launch_bounds__(kThreads) seg_gateup_q4_kernel(SegGateUpQ4Args a, uint32_t *err) {
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ int sm[];
    int *list = sm, *beg = sm + a.seg.E, *end = sm + 2 * a.seg.E;
    const int ne = list_experts(a.seg, list, beg, end);
    const __nv_bfloat16 *x = static_cast<const __nv_bfloat16 *>(a.x);
    __nv_bfloat16 *act = static_cast<__nv_bfloat16 *>(a.act);
    const int lane = threadIdx.x & 31;
    const int qpr = a.d / 2, spr = a.d / 64;   // bytes and scales per weight row
    const int nblk = (a.hid + NR - 1) / NR;
    const int64_t nitems = (int64_t)ne * nblk;
    const int64_t gw = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int64_t nw = (int64_t)gridDim.x * kWarps;
    for (int64_t item = gw; item < nitems; item += nw) {
        const int li = (int)(item / nblk);
        const int n0 = (int)(item - (int64_t)li * nblk) * NR;
        const int64_t wrow0 = (int64_t)list[li] * a.hid + n0;
        for (int r0 = beg[li]; r0 < end[li]; r0 += RG) {
            int64_t tok[RG];
#pragma unroll
            for (int b = 0; b < RG; ++b) {
                const int r = r0 + b;
                int64_t t = -1;
                if (r < end[li]) {
                    // range-check the assignment before deriving its token
                    const int v = a.seg.sorted_rows[r];
                    t = (v >= 0 && v < a.seg.rows) ? v / a.seg.k : -1;
                    if (t < 0 || t >= a.T) {
                        if (lane == 0) atomicOr(err, kErrInput);
                        t = -1;
                    }
                }
                tok[b] = t;
            }
            float ag[RG][NR], au[RG][NR];
#pragma unroll
            for (int b = 0; b < RG; ++b)
#pragma unroll
                for (int q = 0; q < NR; ++q) ag[b][q] = au[b][q] = 0.f;
            for (int c = lane * 32; c < a.d; c += 1024) {
                uint4 wg[NR], wu[NR];
                float sg[NR], su[NR];
#pragma unroll
                for (int q = 0; q < NR; ++q) {
                    const bool ok = n0 + q < a.hid;
                    const int64_t wr = ok ? wrow0 + q : wrow0;
                    wg[q] = __ldcs(reinterpret_cast<const uint4 *>(a.q_gate + wr * qpr + c / 2));
                    wu[q] = __ldcs(reinterpret_cast<const uint4 *>(a.q_up + wr * qpr + c / 2));
                    sg[q] = __ldg(a.s_gate + wr * spr + c / 64);
                    su[q] = __ldg(a.s_up + wr * spr + c / 64);
                }
#pragma unroll
                for (int b = 0; b < RG; ++b) {
                    if (tok[b] < 0) continue;
                    float xv[32];
                    const float xs = 136.f * load32(x + tok[b] * a.d + c, xv);
#pragma unroll
                    for (int q = 0; q < NR; ++q) {
                        ag[b][q] = fmaf(sg[q], dot32_raw(wg[q], xv) - xs, ag[b][q]);
                        au[b][q] = fmaf(su[q], dot32_raw(wu[q], xv) - xs, au[b][q]);
                    }
                }
            }
#pragma unroll
            for (int b = 0; b < RG; ++b) {
#pragma unroll
                for (int q = 0; q < NR; ++q) {
                    const float g = warp_sum(ag[b][q]);
                    const float u = warp_sum(au[b][q]);
                    if (lane == b * NR + q && tok[b] >= 0 && n0 + q < a.hid)
                        act[(int64_t)(r0 + b) * a.hid + n0 + q] = __float2bfloat16_rn(silu_f(g) * u);
                }
            }
        }
    }
}

// y[t, n] = sum_j g_j (W_down[e_j, n] . act[inv(t*k + j)]) (4-bit W_down)
//         (+ shared_gate[t] * (S_down[n] . act_shared[t]), bf16), for NR
// consecutive outputs n per CTA.  The reduction dimension is split over the
// CTA's warps (warp w takes the 1024-element steps w, w + 8, ...), each warp's
// NR rows share its activation chunks, and the warps' partial sums are added
// in warp order through shared memory: enough warps in flight to cover the
// weight loads' latency even at one token.
template <int NR>
__global__ void __launch_bounds__(kThreads) down_direct_q4_kernel(DownDirectQ4Args a, uint32_t *err) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ float red[kWarps][NR];
    const __nv_bfloat16 *act = static_cast<const __nv_bfloat16 *>(a.act);
    __nv_bfloat16 *y = static_cast<__nv_bfloat16 *>(a.y);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int qpr = a.h / 2, spr = a.h / 64;
    const int nblk = (a.d + NR - 1) / NR;
    const int64_t nitems = a.T * nblk;
    for (int64_t item = blockIdx.x; item < nitems; item += gridDim.x) {
        const int64_t t = item / nblk;
        const int n0 = (int)(item - t * nblk) * NR;
        float acc[NR];
#pragma unroll
        for (int q = 0; q < NR; ++q) acc[q] = 0.f;
        for (int j = 0; j < a.k; ++j) {
            const int64_t slot = t * a.k + j;
            const int e = a.ids[slot];
            const int r = a.inv_rows[slot];
            if (e < 0 || e >= a.E || r < 0 || r >= a.T * a.k) {
                if (threadIdx.x == 0) atomicOr(err, kErrInput);
                continue;
            }
            const float g = a.gates[slot];
            const int64_t wrow0 = (int64_t)e * a.d + n0;
            float part[NR];
#pragma unroll
            for (int q = 0; q < NR; ++q) part[q] = 0.f;
            for (int c = (warp * 32 + lane) * 32; c < a.h; c += kWarps * 1024) {
                uint4 w[NR];
                float sc[NR];
#pragma unroll
                for (int q = 0; q < NR; ++q) {
                    const int64_t wr = n0 + q < a.d ? wrow0 + q : wrow0;
                    w[q] = __ldcs(reinterpret_cast<const uint4 *>(a.q_down + wr * qpr + c / 2));
                    sc[q] = __ldg(a.s_down + wr * spr + c / 64);
                }
                float xv[32];
                const float xs = 136.f * load32(act + (int64_t)r * a.h + c, xv);
#pragma unroll
                for (int q = 0; q < NR; ++q) part[q] = fmaf(sc[q], dot32_raw(w[q], xv) - xs, part[q]);
            }
#pragma unroll
            for (int q = 0; q < NR; ++q) acc[q] = fmaf(g, part[q], acc[q]);
        }
        if (a.sh_down) {
            const __nv_bfloat16 *sd = static_cast<const __nv_bfloat16 *>(a.sh_down);
            const __nv_bfloat16 *as = static_cast<const __nv_bfloat16 *>(a.act_shared) + t * a.h_shared;
            const float sg = a.shared_gate[t];
#pragma unroll
            for (int q = 0; q < NR; ++q) {
                if (n0 + q >= a.d) continue;
                const __nv_bfloat16 *row = sd + (int64_t)(n0 + q) * a.h_shared;
                float p = 0.f;
                for (int c = (warp * 32 + lane) * 8; c < a.h_shared; c += kWarps * 256) {
                    float wv[8], av[8];
                    load8_stream(row + c, wv);
                    load8(as + c, av);
#pragma unroll
                    for (int u = 0; u < 8; ++u) p = fmaf(wv[u], av[u], p);
                }
                acc[q] = fmaf(sg, p, acc[q]);
            }
        }
#pragma unroll
        for (int q = 0; q < NR; ++q) {
            const float v = warp_sum(acc[q]);
            if (lane == 0) red[warp][q] = v;
        }
        __syncthreads();
        if (warp == 0 && lane < NR && n0 + lane < a.d) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) v += red[w][lane];
            y[t * a.d + n0 + lane] = __float2bfloat16_rn(v);
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_quantize_q4(const void *w, int dtype, int64_t rows, int cols, uint8_t *q, float *scales,
                               cudaStream_t s) {
    const int64_t groups = rows * (cols / 64);
    if (groups <= 0) return cudaSuccess;
    const unsigned blocks = (unsigned)std::min<int64_t>((groups + 255) / 256, 32LL * num_sms());
    if (dtype == MOE_F32)
        return launch_kernel(quantize_q4_kernel<float>, blocks, 256, 0, s, static_cast<const float *>(w), groups,
                             cols / 64, q, scales);
    return launch_kernel(quantize_q4_kernel<__nv_bfloat16>, blocks, 256, 0, s, static_cast<const __nv_bfloat16 *>(w),
                         groups, cols / 64, q, scales);
}

cudaError_t launch_seg_gateup_q4(const SegGateUpQ4Args &a, cudaStream_t s, uint32_t *err) {
    if (a.seg.rows <= 0) return cudaSuccess;
    const size_t smem = sizeof(int) * 3 * (size_t)a.seg.E;
    auto go = [&](auto kern, int nr) {
        const int64_t items = (int64_t)a.seg.E * ((a.hid + nr - 1) / nr);
        return launch_kernel(kern, grid_for(kern, items, smem), kThreads, smem, s, a, err);
    };
    // one token: two hidden rows per warp share each activation chunk; more
    // tokens: four grouped rows per pass share each weight load
    return a.T == 1 ? go(seg_gateup_q4_kernel<1, 2>, 2) : go(seg_gateup_q4_kernel<4, 1>, 1);
}

cudaError_t launch_down_direct_q4(const DownDirectQ4Args &a, cudaStream_t s, uint32_t *err) {
    if (a.T <= 0) return cudaSuccess;
    constexpr int NR = 4;
    auto kern = down_direct_q4_kernel<NR>;
    // one CTA per item (grid_for counts warps)
    const int64_t items = a.T * ((a.d + NR - 1) / NR);
    return launch_kernel(kern, grid_for(kern, items * kWarps, 0), kThreads, 0, s, a, err);
}

}  // namespace moe
