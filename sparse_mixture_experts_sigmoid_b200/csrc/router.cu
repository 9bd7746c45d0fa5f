// Router: fused GEMV (router logits), softmax or sigmoid scoring, register
// top-k with renormalisation.
//
// "Tutorial 11: Mixture of Experts (MoE)", section 2 "The Router" (route_topk:
// logits = x . W_router^T, softmax over all experts, top-k, gather, optional
// renormalisation); "Small MoE Architecture, in depth", SmallMoE.forward
// (sigmoid scores; top k of scores + balance_bias; gates are the kept raw
// scores) and the paragraph on auxiliary-loss-free balancing after it.
//
// Layout of the work: a CTA of 8 warps owns 8*TW consecutive tokens, each warp
// TW of them.  W_router (plus the shared-expert gate vector w_s as row E) is
// streamed through shared memory in chunks of KC columns with a two-stage
// cp.async pipeline, so every CTA reads W_router from L2 once.  Inside a warp,
// EL lanes span the experts (lane e % EL holds experts e, e + EL, ...) and
// CG = 32 / EL lane groups split the chunk's columns; the CG partial sums are
// folded with shuffles.  All arithmetic is fp32 on exact bf16/fp32 inputs.
// Selection is k rounds of a warp arg-max over (key, -index), so equal keys
// resolve to the lower expert index.  The key is the logit (it orders experts
// as either score function does), or the score plus the balance bias when one
// is given; gates always come from the unbiased scores.  With the score
// statistic requested, each CTA adds its tokens' score rows, in token order,
// into one partial row of a.stats.
#include <float.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int64_t kSmallT = 64;   // batches up to this many tokens use one CTA per token

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, int src_bytes) {
    uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

struct Geo {
    int Ep;     // rows staged: E (+1 for the shared gate)
    int EL;     // lanes across experts
    int KC;     // columns per chunk
    int ldw;    // staged row stride, elements
};

template <typename Tin>
__device__ __forceinline__ void stage_chunk(const RouterArgs &a, const Geo &g, Tin *ws, Tin *xs,
                                            int64_t t0, int NT, int c0) {
    constexpr int V = 16 / sizeof(Tin);  // elements per 16-byte vector
    const Tin *wr = static_cast<const Tin *>(a.w_router);
    const Tin *wsg = static_cast<const Tin *>(a.w_shared_gate);
    const Tin *x = static_cast<const Tin *>(a.x);
    const int vpr = g.KC / V;
    const int nw = g.Ep * vpr;
    for (int i = threadIdx.x; i < nw; i += kThreads) {
        int row = i / vpr, col = (i - row * vpr) * V;
        int gc = c0 + col;
        const Tin *src = row < a.E ? wr + (int64_t)row * a.d + gc : wsg + gc;
        bool ok = gc < a.d;
        cp_async16(ws + row * g.ldw + col, ok ? src : wr, ok ? 16 : 0);
    }
    const int nx = NT * vpr;
    for (int i = threadIdx.x; i < nx; i += kThreads) {
        int tok = i / vpr, col = (i - tok * vpr) * V;
        int gc = c0 + col;
        int64_t t = t0 + tok;
        bool ok = gc < a.d && t < a.T;
        cp_async16(xs + tok * g.KC + col, ok ? x + t * a.d + gc : x, ok ? 16 : 0);
    }
}

template <typename Tin, int TW, int EPL>
__global__ void __launch_bounds__(kThreads) router_kernel(RouterArgs a, Geo g) {
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ __align__(16) unsigned char smem_raw[];
    constexpr int NT = kWarps * TW;
    Tin *wbuf[2], *xbuf[2];
    {
        Tin *p = reinterpret_cast<Tin *>(smem_raw);
        const int wsz = g.Ep * g.ldw, xsz = NT * g.KC;
        wbuf[0] = p;
        wbuf[1] = p + wsz;
        xbuf[0] = p + 2 * wsz;
        xbuf[1] = p + 2 * wsz + xsz;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * NT;
    const int CG = 32 / g.EL;
    const int cg = lane / g.EL, le = lane % g.EL;
    const int nchunks = (a.d + g.KC - 1) / g.KC;
    const int NS = g.KC / 8;

    float acc[TW][EPL];
#pragma unroll
    for (int i = 0; i < TW; ++i)
#pragma unroll
        for (int q = 0; q < EPL; ++q) acc[i][q] = 0.f;

    stage_chunk<Tin>(a, g, wbuf[0], xbuf[0], t0, NT, 0);
    cp_async_commit();
    for (int c = 0; c < nchunks; ++c) {
        if (c + 1 < nchunks) {
            stage_chunk<Tin>(a, g, wbuf[(c + 1) & 1], xbuf[(c + 1) & 1], t0, NT, (c + 1) * g.KC);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const Tin *W = wbuf[c & 1];
        const Tin *X = xbuf[c & 1] + warp * TW * g.KC;
        for (int s = cg; s < NS; s += CG) {
            float xv[TW][8];
#pragma unroll
            for (int i = 0; i < TW; ++i) load8(X + i * g.KC + s * 8, xv[i]);
#pragma unroll
            for (int q = 0; q < EPL; ++q) {
                const int e = le + g.EL * q;
                if (e < g.Ep) {
                    float w[8];
                    load8(W + e * g.ldw + s * 8, w);
#pragma unroll
                    for (int i = 0; i < TW; ++i) {
                        float v = acc[i][q];
#pragma unroll
                        for (int u = 0; u < 8; ++u) v = fmaf(w[u], xv[i][u], v);
                        acc[i][q] = v;
                    }
                }
            }
        }
        __syncthreads();
    }
    // fold the column groups
    for (int o = g.EL; o < 32; o <<= 1)
#pragma unroll
        for (int i = 0; i < TW; ++i)
#pragma unroll
            for (int q = 0; q < EPL; ++q) acc[i][q] += __shfl_xor_sync(0xffffffffu, acc[i][q], o);

    // clear this CTA's rows of the combine accumulator
    if (a.zero_rows) {
        const int64_t tend = min(a.T, t0 + NT);
        const int64_t n4 = (tend - t0) * a.d / 4;
        float4 *z = reinterpret_cast<float4 *>(a.zero_rows + t0 * a.d);
        for (int64_t i = threadIdx.x; i < n4; i += kThreads) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }

    const bool sigm = a.score == MOE_SCORE_SIGMOID;
    const bool want_s = a.probs || a.stats || a.bias;
    float ssum[EPL];   // this warp's score sums per owned expert (score statistic)
#pragma unroll
    for (int q = 0; q < EPL; ++q) ssum[q] = 0.f;
#pragma unroll
    for (int i = 0; i < TW; ++i) {
        const int64_t t = t0 + warp * TW + i;
        if (t >= a.T) break;
        // softmax statistics over the E routed experts
        float m = -FLT_MAX;
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            const int e = le + g.EL * q;
            if (cg == 0 && e < a.E) m = fmaxf(m, acc[i][q]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float z = 0.f;
        if (!sigm) {
#pragma unroll
            for (int q = 0; q < EPL; ++q) {
                const int e = le + g.EL * q;
                if (cg == 0 && e < a.E) z += expf(acc[i][q] - m);
            }
            z = warp_sum(z);
        }
        float sc_e[EPL], key[EPL];
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            const int e = le + g.EL * q;
            const bool own = cg == 0 && e < a.E;
            sc_e[q] = 0.f;
            if (want_s && own) sc_e[q] = sigm ? 1.f / (1.f + expf(-acc[i][q])) : expf(acc[i][q] - m) / z;
            ssum[q] += sc_e[q];
            key[q] = acc[i][q];
            if (a.bias) key[q] = own ? sc_e[q] + a.bias[e] : -FLT_MAX;
        }

        uint32_t taken = 0;
        int my_e = 0;
        float my_l = 0.f;
        for (int j = 0; j < a.k; ++j) {
            float bk = -FLT_MAX;
            int be = 0x7fffffff;
            float bl = 0.f;
#pragma unroll
            for (int q = 0; q < EPL; ++q) {
                const int e = le + g.EL * q;
                const bool ok = cg == 0 && e < a.E && !((taken >> q) & 1u);
                if (ok && (key[q] > bk || (key[q] == bk && e < be))) {
                    bk = key[q];
                    be = e;
                    bl = acc[i][q];
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                float ok_ = __shfl_xor_sync(0xffffffffu, bk, o);
                int oe = __shfl_xor_sync(0xffffffffu, be, o);
                float ol = __shfl_xor_sync(0xffffffffu, bl, o);
                if (ok_ > bk || (ok_ == bk && oe < be)) {
                    bk = ok_;
                    be = oe;
                    bl = ol;
                }
            }
            if (be >= a.E) be = j;  // only reachable with non-finite logits; keeps ids in range
            if (le == be % g.EL && cg == 0) taken |= 1u << (be / g.EL);
            if (lane == j) {
                my_e = be;
                my_l = bl;
            }
        }
        float sc = 0.f;
        if (lane < a.k) sc = sigm ? 1.f / (1.f + expf(-my_l)) : expf(my_l - m) / z;
        if (a.norm_topk) {
            const float gsum = warp_sum(lane < a.k ? sc : 0.f);
            sc = sc / gsum;
        }
        if (lane < a.k) {
            a.ids[t * a.k + lane] = my_e;
            a.gates[t * a.k + lane] = sc;
        }
        if (a.probs) {
#pragma unroll
            for (int q = 0; q < EPL; ++q) {
                const int e = le + g.EL * q;
                if (cg == 0 && e < a.E) a.probs[t * a.E + e] = sc_e[q];
            }
        }
        if (a.shared_gate && a.w_shared_gate) {
#pragma unroll
            for (int q = 0; q < EPL; ++q) {
                const int e = le + g.EL * q;
                if (cg == 0 && e == a.E) a.shared_gate[t] = 1.f / (1.f + expf(-acc[i][q]));
            }
        }
    }
    if (a.stats) {
        // the staging buffers are idle (the chunk loop ended with a barrier):
        // per-warp score sums, then their sum in warp order
        float *ws = reinterpret_cast<float *>(smem_raw);   // [kWarps, E]
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            const int e = le + g.EL * q;
            if (cg == 0 && e < a.E) ws[warp * a.E + e] = ssum[q];
        }
        __syncthreads();
        for (int e = threadIdx.x; e < a.E; e += kThreads) {
            float v = 0.f;
            for (int w = 0; w < kWarps; ++w) v += ws[w * a.E + e];
            a.stats[(int64_t)blockIdx.x * a.E + e] = v;
        }
    }
}

// Router for small batches: one CTA of 8 warps per token.  The token's row is
// staged in shared memory as fp32; warp w computes the logits of experts w,
// w + 8, ... (lane l takes the 8-element slices l, l + 32, ... of the row with
// 16-byte loads, all issued before the reduction), so the router weights are
// streamed by the whole CTA at once.  Warp 0 then selects the top k with the
// same arg-max rounds as the batched router, over EPL experts per lane (the
// smallest power of two covering E / 32: the selection is the serial tail of
// a batch-1 step, and its code is fetched from memory each time).
template <typename Tin, int EPL>
__global__ void __launch_bounds__(kThreads) router_small_kernel(RouterArgs a) {
    {
        // The router rows are a layer input, not the previous kernel's output:
        // pull them into L2 (spread over the CTAs) before waiting for it, so
        // their DRAM latency overlaps its tail and the x row load below.  L2 is
        // coherent, so a row written by an earlier kernel is never read stale.
        const char *wb = static_cast<const char *>(a.w_router);
        const int64_t lines = ((int64_t)a.E * a.d * (int64_t)sizeof(Tin) + 127) / 128;
        for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < lines; i += (int64_t)gridDim.x * kThreads)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(wb + 128 * i));
    }
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ float sm[];
    float *sx = sm;              // [d] the token's row
    float *lg = sm + a.d;        // [E + 1] logits (shared gate last)
    const int64_t t = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Tin *wr = static_cast<const Tin *>(a.w_router);
    const int Ep = a.E + (a.w_shared_gate ? 1 : 0);
    auto row_of = [&](int e) { return e < a.E ? wr + (int64_t)e * a.d : static_cast<const Tin *>(a.w_shared_gate); };
    // the first kPre slices of this warp's first row (all of a row of up to
    // 4096 elements) are loaded before the x row is staged, so the two loads
    // overlap and the row arrives in one round trip
    constexpr int kPre = 16;
    float wpre[kPre][8];
    if (warp < Ep) {
        const Tin *row = row_of(warp);
#pragma unroll
        for (int i = 0; i < kPre; ++i)
            if (lane * 8 + 256 * i < a.d) load8(row + lane * 8 + 256 * i, wpre[i]);
    }
    const Tin *x = static_cast<const Tin *>(a.x) + t * a.d;
    for (int c = threadIdx.x * 8; c < a.d; c += kThreads * 8) {
        float v[8];
        load8(x + c, v);
#pragma unroll
        for (int u = 0; u < 8; ++u) sx[c + u] = v[u];
    }
    if (a.zero_rows) {
        float4 *z = reinterpret_cast<float4 *>(a.zero_rows + t * a.d);
        for (int i = threadIdx.x; i < a.d / 4; i += kThreads) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    for (int e = warp; e < Ep; e += kWarps) {
        const Tin *row = row_of(e);
        float acc = 0.f;
        int c = lane * 8;
        if (e == warp) {
#pragma unroll
            for (int i = 0; i < kPre; ++i, c += 256)
                if (c < a.d) {
#pragma unroll
                    for (int u = 0; u < 8; ++u) acc = fmaf(wpre[i][u], sx[c + u], acc);
                }
        }
#pragma unroll 4
        for (; c < a.d; c += 256) {
            float w[8];
            load8(row + c, w);
#pragma unroll
            for (int u = 0; u < 8; ++u) acc = fmaf(w[u], sx[c + u], acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) lg[e] = acc;
    }
    __syncthreads();
    if (warp != 0) return;
    const bool sigm = a.score == MOE_SCORE_SIGMOID;
    float l[EPL], key[EPL], sc_e[EPL];
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
        const int e = lane + 32 * q;
        l[q] = e < a.E ? lg[e] : -FLT_MAX;
    }
    float m = -FLT_MAX;
#pragma unroll
    for (int q = 0; q < EPL; ++q)
        if (lane + 32 * q < a.E) m = fmaxf(m, l[q]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float z = 0.f;
    if (!sigm) {
#pragma unroll
        for (int q = 0; q < EPL; ++q)
            if (lane + 32 * q < a.E) z += expf(l[q] - m);
        z = warp_sum(z);
    }
    // scores when needed; key = the logit, or the score plus the balance bias
    const bool want_s = a.probs || a.stats || a.bias;
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
        const int e = lane + 32 * q;
        sc_e[q] = (want_s && e < a.E) ? (sigm ? 1.f / (1.f + expf(-l[q])) : expf(l[q] - m) / z) : 0.f;
        key[q] = l[q];
        if (a.bias) key[q] = e < a.E ? sc_e[q] + a.bias[e] : -FLT_MAX;
    }
    uint32_t taken = 0;
    int my_e = 0;
    float my_l = 0.f;
    for (int j = 0; j < a.k; ++j) {
        float bk = -FLT_MAX, bl = 0.f;
        int be = 0x7fffffff;
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            const int e = lane + 32 * q;
            if (e < a.E && !((taken >> q) & 1u) && (key[q] > bk || (key[q] == bk && e < be))) {
                bk = key[q];
                be = e;
                bl = l[q];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ok_ = __shfl_xor_sync(0xffffffffu, bk, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            const float ol = __shfl_xor_sync(0xffffffffu, bl, o);
            if (ok_ > bk || (ok_ == bk && oe < be)) {
                bk = ok_;
                be = oe;
                bl = ol;
            }
        }
        if (be >= a.E) be = j;   // only reachable with non-finite logits; keeps ids in range
        if (lane == (be & 31)) taken |= 1u << (be >> 5);
        if (lane == j) {
            my_e = be;
            my_l = bl;
        }
    }
    float sc = 0.f;
    if (lane < a.k) sc = sigm ? 1.f / (1.f + expf(-my_l)) : expf(my_l - m) / z;
    if (a.norm_topk) {
        const float ssum = warp_sum(lane < a.k ? sc : 0.f);
        sc = sc / ssum;
    }
    if (lane < a.k) {
        a.ids[t * a.k + lane] = my_e;
        a.gates[t * a.k + lane] = sc;
    }
    if (a.counts && gridDim.x == 1) {
        // one token: its grouping directly (the k experts are distinct, so the
        // stable order by expert is the order of the expert ids)
        __shared__ int s_sel[32];
        if (lane < a.k) s_sel[lane] = my_e;
        __syncwarp();
        if (lane < a.k) {
            int pos = 0;
            for (int jj = 0; jj < a.k; ++jj) pos += s_sel[jj] < my_e;
            a.sorted_rows[pos] = lane;
            a.inv_rows[lane] = pos;
        }
        for (int e = lane; e <= a.E; e += 32) {
            int before = 0, has = 0;
            for (int jj = 0; jj < a.k; ++jj) {
                before += s_sel[jj] < e;
                has += s_sel[jj] == e;
            }
            a.offsets[e] = before;
            if (e < a.E) a.counts[e] = has;
        }
    }
    if (a.probs) {
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            const int e = lane + 32 * q;
            if (e < a.E) a.probs[t * a.E + e] = sc_e[q];
        }
    }
    if (a.stats) {
        // one token per CTA: its score row is the CTA's partial row
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            const int e = lane + 32 * q;
            if (e < a.E) a.stats[t * a.E + e] = sc_e[q];
        }
    }
    if (lane == 0 && a.shared_gate && a.w_shared_gate) a.shared_gate[t] = 1.f / (1.f + expf(-lg[a.E]));
}

int pow2ceil(int v) {
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

template <typename Tin, int TW, int EPL>
cudaError_t launch_t(const RouterArgs &a, const Geo &g, cudaStream_t s) {
    constexpr int NT = kWarps * TW;
    const size_t smem = sizeof(Tin) * (2 * (size_t)g.Ep * g.ldw + 2 * (size_t)NT * g.KC);
    auto kern = router_kernel<Tin, TW, EPL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((a.T + NT - 1) / NT);
    e = launch_kernel(kern, grid, kThreads, smem, s, a, g);
    if (e == cudaSuccess && a.stats && a.score_mean) e = launch_router_stats(a.stats, grid, a.E, a.T, a.score_mean, s);
    return e;
}

template <typename Tin, int EPL>
cudaError_t launch_e(const RouterArgs &a, const Geo &g, int TW, cudaStream_t s) {
    if constexpr (EPL <= 8) {
        if (TW >= 4) return launch_t<Tin, 4, EPL>(a, g, s);
    }
    if constexpr (EPL <= 16) {
        if (TW >= 2) return launch_t<Tin, 2, EPL>(a, g, s);
    }
    return launch_t<Tin, 1, EPL>(a, g, s);
}

template <typename Tin>
cudaError_t launch_dt(const RouterArgs &a, cudaStream_t s) {
    Geo g;
    g.Ep = a.E + (a.w_shared_gate ? 1 : 0);
    int EPL;
    if (g.Ep <= 32) {
        g.EL = pow2ceil(g.Ep < 4 ? 4 : g.Ep);
        EPL = 1;
    } else {
        g.EL = 32;
        EPL = pow2ceil((g.Ep + 31) / 32);
    }
    // chunk width: up to 512 columns while the staged router rows stay near 32 KB
    const int pad = 16 / (int)sizeof(Tin);
    int KC = 64;
    const int dpad = (a.d + 63) / 64 * 64;
    while (KC < 512 && KC * 2 <= dpad && (size_t)g.Ep * (KC * 2 + pad) * sizeof(Tin) <= 32768) KC *= 2;
    // wide fp32 rows with many experts: narrower chunks keep two stages under ~150 KB
    if (2 * (size_t)g.Ep * (KC + pad) * sizeof(Tin) > 150000) KC = 32;
    g.KC = KC;
    g.ldw = KC + pad;
    // tokens per warp: as many as keep at least ~2 CTAs per SM busy
    const int64_t target = 2LL * num_sms();
    int TW = 1;
    if ((a.T + 8 * 4 - 1) / (8 * 4) >= target) TW = 4;
    else if ((a.T + 8 * 2 - 1) / (8 * 2) >= target) TW = 2;
    switch (EPL) {
        case 1: return launch_e<Tin, 1>(a, g, TW, s);
        case 2: return launch_e<Tin, 2>(a, g, TW, s);
        case 4: return launch_e<Tin, 4>(a, g, TW, s);
        case 8: return launch_e<Tin, 8>(a, g, TW, s);
        case 16: return launch_e<Tin, 16>(a, g, TW, s);
        case 32: return launch_e<Tin, 32>(a, g, TW, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_router(const RouterArgs &a, int dtype, float *scratch, cudaStream_t s) {
    if (a.T <= 0) return cudaSuccess;
    if (scratch && router_tc_supported(a.T, a.E, dtype)) return launch_router_tc(a, scratch, s);
    if (a.T <= kSmallT) {
        const size_t smem = sizeof(float) * ((size_t)a.d + a.E + 1);
        const int epl = pow2ceil((a.E + 31) / 32);
        auto pick = [&](auto tin) -> void (*)(RouterArgs) {
            using Tin = decltype(tin);
            switch (epl) {
                case 1: return router_small_kernel<Tin, 1>;
                case 2: return router_small_kernel<Tin, 2>;
                case 4: return router_small_kernel<Tin, 4>;
                case 8: return router_small_kernel<Tin, 8>;
                default: return router_small_kernel<Tin, MOE_MAX_EXPERTS / 32>;
            }
        };
        auto kern = dtype == MOE_F32 ? pick(float{}) : pick(__nv_bfloat16{});
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess) e = launch_kernel(kern, (unsigned)a.T, kThreads, smem, s, a);
        if (e == cudaSuccess && a.stats && a.score_mean)
            e = launch_router_stats(a.stats, a.T, a.E, a.T, a.score_mean, s);
        return e;
    }
    return dtype == MOE_F32 ? launch_dt<float>(a, s) : launch_dt<__nv_bfloat16>(a, s);
}

}  // namespace moe
