// Router for bf16 batches, in two kernels:
//
//  1. router_logits_kernel: the router logits l = x . W_router^T (plus the
//     shared-expert gate logit w_s . x) as a tcgen05 GEMM over tiles of 128
//     tokens x BN logit columns x one chunk of the K range, fp32 accumulators
//     in TMEM.  Each tile writes its partial sums as fp32 rows of a
//     [S, T, LSP] scratch array (S chunks of K).  Splitting K across CTAs
//     puts ~256 CTAs (two per SM) on the layer, so the read of x is spread
//     over every SM however few token tiles there are.
//  2. router_select_kernel: one warp per token adds its S partial rows in
//     chunk order, forms softmax statistics or sigmoid scores, takes the top k
//     by k rounds of a warp arg-max over (key, -index) -- equal keys go to the
//     lower expert index -- and writes ids, gates (optionally renormalised),
//     the full score row and the shared gate.  The key is the logit (it
//     orders experts as either score does), or, with a balance bias, the
//     score plus the bias; the gates always come from the unbiased scores.
//     With the score statistic requested, the CTA's 8 score rows are added
//     in token order into one partial row per CTA.
//
// "Tutorial 11: Mixture of Experts (MoE)", section 2 "The Router" (route_topk:
// logits = x . W_router^T, softmax over all experts, top-k, gather of the kept
// scores, optional renormalisation); "Small MoE Architecture, in depth",
// SmallMoE.forward (sigmoid scores; top k of scores + balance_bias; gates are
// the kept raw scores) and the paragraph on auxiliary-loss-free balancing
// after it.
//
// Exactness: x and W_router are bf16, so every product is exact in fp32.  The
// K range is cut into S chunks (one per CTA) and, inside a CTA, k-block kb of
// the chunk accumulates into TMEM accumulator kb % G; the epilogue adds the G
// accumulators and the selection kernel the S chunks, both on the CUDA cores
// in a fixed order.  No accumulation chain inside the tensor core is longer
// than ceil(kpc / G) k-blocks of 64, which keeps the logits within ~1e-6 of a
// float64 sum (a single long chain measured 4e-6 on the gates).  Scores,
// selection and gates are fp32 on the CUDA cores.
//
// Logit columns: [0, E) are the router rows; when the shared expert is
// present its gate vector w_s is column nrw = E rounded up to 8 (so its 8-row
// TMA box lands on a 1024-byte swizzle atom).  BN is the smallest of 16..128
// covering the columns; LSP, the stored row length, is the column count
// rounded up to 16.
#include <float.h>

#include "moe_internal.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace rt {

using namespace tc;

constexpr int BM = 128;
constexpr int kThreads = 192;
constexpr int kTmaWarp = 4, kMmaWarp = 5;   // warps 0-3: epilogue
constexpr uint32_t kCols = 256;       // TMEM columns per CTA: two CTAs share an SM
#ifndef MOE_ROUTER_TARGET_CTAS
#define MOE_ROUTER_TARGET_CTAS 256
#endif
#ifndef MOE_ROUTER_MAX_BN
#define MOE_ROUTER_MAX_BN 128
#endif
constexpr int kTargetCtas = MOE_ROUTER_TARGET_CTAS;   // the K split aims at about this many CTAs
constexpr int kMaxBN = MOE_ROUTER_MAX_BN;
constexpr int kMaxChunks = 8;         // K chunks the selection kernel adds
constexpr int kABytes = BM * 128;     // 16 KB: 128 tokens x 64 bf16
constexpr int kMaxStages = 5;

template <int BN>
struct Shape {
    static constexpr int kBBytes = BN * 128;
    static constexpr int kStage = kABytes + kBBytes;
    // about 96 KB of ring per CTA, so two CTAs fit on an SM
    static constexpr int kStages = BN >= 128 ? 3 : (BN >= 64 ? 4 : kMaxStages);
    static constexpr int G = (int)kCols / BN > 8 ? 8 : (int)kCols / BN;   // K-split accumulators
};

struct LogitsArgs {
    int64_t T;
    int d, E, nrw, LSP;   // LSP: stored partial row length
    int n_tiles, S, kpc;  // column tiles, K chunks, k-blocks per chunk
    bool shared;
    float *partial;       // [S, T, LSP]
    uint32_t *err;
    int32_t *hist;        // grouping histogram to clear for the selection kernel (or null)
    int64_t hist_ints;
};

struct Ctrl {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tfull;
    uint32_t tmem_base;
    int abort;
};

// Sum of the ng partial accumulators (BN columns apart) for 16 columns.
template <int BN, int G>
__device__ __forceinline__ void load_logits(uint32_t taddr, int ng, float (&v)[16]) {
#pragma unroll
    for (int q = 0; q < 16; ++q) v[q] = 0.f;
#pragma unroll
    for (int g = 0; g < G; g += 2) {
        if (g < ng) {
            float p0[16], p1[16];
            tmem_ld16(taddr + g * BN, p0);
            if (g + 1 < ng) tmem_ld16(taddr + (g + 1) * BN, p1);
            tmem_wait_ld();
            if (g + 1 < ng) {
#pragma unroll
                for (int q = 0; q < 16; ++q) v[q] += p0[q] + p1[q];
            } else {
#pragma unroll
                for (int q = 0; q < 16; ++q) v[q] += p0[q];
            }
        }
    }
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 2)
    router_logits_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                         const __grid_constant__ CUtensorMap tmWB, const __grid_constant__ CUtensorMap tmS,
                         LogitsArgs a) {
    using Sh = Shape<BN>;
    constexpr int kStages = Sh::kStages, kStage = Sh::kStage, G = Sh::G;
    constexpr uint32_t kIdesc = instr_desc<__nv_bfloat16>(BM, BN);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctrl *ctrl = reinterpret_cast<Ctrl *>(smem + kStages * kStage);
    volatile int *abort = &ctrl->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ctrl->full[s], 1);
            mbar_init(&ctrl->empty[s], 1);
        }
        mbar_init(&ctrl->tfull, 1);
        ctrl->abort = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) tmem_alloc(&ctrl->tmem_base, kCols);
    if (warp == kTmaWarp && lane == 0) {
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmW);
        prefetch_tmap(&tmWB);
        if (a.shared) prefetch_tmap(&tmS);
    }
    pdl_wait();   // the prologue above overlaps the previous kernel's tail
    // clear the grouping histogram that the selection kernel accumulates into
    if (a.hist)
        for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < a.hist_ints; i += (int64_t)gridDim.x * kThreads)
            a.hist[i] = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch_dependents();   // this CTA's TMEM is allocated

    const uint32_t tmem = ctrl->tmem_base;
    const int nk = (a.d + 63) / 64;
    // one tile per CTA: id -> (token tile m, column tile n, K chunk c), chunks fastest
    const int per_m = a.n_tiles * a.S;
    const int id = blockIdx.x;
    const int m = id / per_m, rem = id - m * per_m, n = rem / a.S, c = rem - n * a.S;
    const int kb0 = c * a.kpc, kb1 = min(nk, kb0 + a.kpc);

    if (warp == kTmaWarp) {
        if (lane == 0) {
            // a tile of router rows only comes in one BN-row box per K block
            // (rows past E read as zeros); other tiles use 8-row boxes: router
            // rows below nrw, the shared gate row at nrw, and other rows are
            // never read
            const bool whole = a.E >= BN && !(a.shared && a.nrw >= n * BN && a.nrw < n * BN + BN);
            int nbox = 0;
            for (int j = 0; j < BN / 8; ++j) {
                const int r = n * BN + 8 * j;
                nbox += (r < a.nrw) || (a.shared && r == a.nrw);
            }
            if (whole) nbox = BN / 8;
            uint32_t it = 0;
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                const int s = it % kStages;
                if (!wait_bar(&ctrl->empty[s], ((it / kStages) & 1) ^ 1, abort, a.err)) {
                    ok = false;
                    break;
                }
                uint8_t *st = smem + s * kStage;
                mbar_expect_tx(&ctrl->full[s], kABytes + nbox * 1024);
                tma_load_2d(&tmX, st, &ctrl->full[s], kb * 64, m * BM);
                if (whole) {
                    tma_load_2d(&tmWB, st + kABytes, &ctrl->full[s], kb * 64, n * BN);
                    continue;
                }
                for (int j = 0; j < BN / 8; ++j) {
                    const int r = n * BN + 8 * j;
                    if (r < a.nrw)
                        tma_load_2d(&tmW, st + kABytes + j * 1024, &ctrl->full[s], kb * 64, r);
                    else if (a.shared && r == a.nrw)
                        tma_load_2d(&tmS, st + kABytes + j * 1024, &ctrl->full[s], kb * 64, 0);
                }
            }
            if (!ok) {
                // aborting: let the copies already issued land before the CTA exits
                for (uint32_t j = it > (uint32_t)kStages ? it - kStages : 0; j < it; ++j) {
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try_wait(&ctrl->full[j % kStages], (j / kStages) & 1) &&
                           globaltimer() - t0 < 100000000ull) {
                    }
                }
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb) {
                const uint32_t it = (uint32_t)(kb - kb0);
                const int s = it % kStages;
                if (!wait_bar(&ctrl->full[s], (it / kStages) & 1, abort, a.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = smem_desc(smem + s * kStage);
                const uint64_t bd = smem_desc(smem + s * kStage + kABytes);
                const int j = kb - kb0;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma<__nv_bfloat16>(tmem + (j % G) * BN, ad + 2 * kk, bd + 2 * kk, kIdesc,
                                       (j >= G || kk > 0) ? 1u : 0u);
                mma_commit(&ctrl->empty[s]);
            }
            if (ok) mma_commit(&ctrl->tfull);
        }
    } else {
        // epilogue: each warp takes its 32 TMEM lanes (tokens), adds the G
        // accumulators, stages the rows in the (now idle) ring and writes each
        // row with one coalesced warp store
        constexpr int kLd = BN + 4;   // staged row stride in floats (conflict-free float4 stores)
        float *stg = reinterpret_cast<float *>(smem) + warp * 32 * kLd;
        const uint32_t tb = tmem + ((uint32_t)(warp * 32) << 16);
        const int ng = kb1 - kb0 < G ? kb1 - kb0 : G;
        const int ncols = min(BN, a.LSP - n * BN);   // multiple of 16
        if (wait_bar(&ctrl->tfull, 0, abort, a.err)) {
            tc_fence_after();
#pragma unroll 1
            for (int col = 0; col < ncols; col += 16) {
                float v[16];
                load_logits<BN, G>(tb + col, ng, v);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<float4 *>(stg + lane * kLd + col + 4 * q) =
                        make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
            __syncwarp();
            const int64_t t0 = (int64_t)m * BM + warp * 32;
            float *dst = a.partial + ((int64_t)c * a.T + t0) * a.LSP + n * BN;
            for (int rr = 0; rr < 32 && t0 + rr < a.T; ++rr)
                for (int q = lane * 4; q < ncols; q += 128)
                    *reinterpret_cast<float4 *>(dst + (int64_t)rr * a.LSP + q) =
                        *reinterpret_cast<const float4 *>(stg + rr * kLd + q);
            tc_fence_before();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kCols);
}

// The selection for token t by one warp (see router_select_kernel).  With
// stat_row != NULL the lanes also write the token's score row there.
template <int EPL>
__device__ __forceinline__ void select_token(const RouterArgs &a, const float *partial, int LSP, int S, int nrw,
                                             int64_t t, int lane, float *stat_row) {
    const bool sigm = a.score == MOE_SCORE_SIGMOID;
    // the token's logits: lane owns experts lane * EPL .. + EPL - 1; its S
    // partial rows are read with vector loads, a group of chunks at a time with
    // all loads issued before the adds, and added in chunk order
    const int64_t slab = a.T * (int64_t)LSP;
    const float *row = partial + t * LSP;
    const int e0 = lane * EPL;
    const bool mine = e0 < LSP;   // then all EPL columns lie inside the row (LSP % 16 == 0)
    float l[EPL], key[EPL];
#pragma unroll
    for (int q = 0; q < EPL; ++q) l[q] = 0.f;
    constexpr int kGroup = EPL <= 8 ? 8 : 4;
#pragma unroll
    for (int c0 = 0; c0 < kMaxChunks; c0 += kGroup) {
        if (c0 < S) {
            float v[kGroup][EPL];
#pragma unroll
            for (int g = 0; g < kGroup; ++g) {
                const int c = c0 + g < S ? c0 + g : S - 1;   // clamped: always a valid row
                const float *src = row + c * slab + (mine ? e0 : 0);
#pragma unroll
                for (int q = 0; q < EPL; q += (EPL >= 4 ? 4 : EPL)) {
                    if constexpr (EPL >= 4) {
                        const float4 u = *reinterpret_cast<const float4 *>(src + q);
                        v[g][q] = u.x;
                        v[g][q + 1] = u.y;
                        v[g][q + 2] = u.z;
                        v[g][q + 3] = u.w;
                    } else {
                        const float2 u = *reinterpret_cast<const float2 *>(src + q);
                        v[g][q] = u.x;
                        v[g][q + 1] = u.y;
                    }
                }
            }
#pragma unroll
            for (int g = 0; g < kGroup; ++g)
                if (c0 + g < S)
#pragma unroll
                    for (int q = 0; q < EPL; ++q) l[q] += v[g][q];
        }
    }
#pragma unroll
    for (int q = 0; q < EPL; ++q)
        if (!mine || e0 + q >= a.E) l[q] = -FLT_MAX;
    if (a.zero_rows) {
        float4 *z = reinterpret_cast<float4 *>(a.zero_rows + t * a.d);
        for (int i = lane; i < a.d / 4; i += 32) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float m = -FLT_MAX;
#pragma unroll
    for (int q = 0; q < EPL; ++q)
        if (e0 + q < a.E) m = fmaxf(m, l[q]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float z = 0.f;
    if (!sigm) {
#pragma unroll
        for (int q = 0; q < EPL; ++q)
            if (e0 + q < a.E) z += expf(l[q] - m);
        z = warp_sum(z);
    }
    // every expert's score, when the score row, its statistic or a biased
    // key needs it
    float sc_e[EPL];
    if (a.probs || stat_row || a.bias) {
#pragma unroll
        for (int q = 0; q < EPL; ++q)
            sc_e[q] = e0 + q < a.E ? (sigm ? 1.f / (1.f + expf(-l[q])) : expf(l[q] - m) / z) : 0.f;
    }
    // selection key: the logit (monotone in the score under either function),
    // or the score plus the balance bias
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
        const int e = e0 + q;
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
            const int e = e0 + q;
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
        if (lane == be / EPL) taken |= 1u << (be % EPL);
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
        if (a.hist) {
            // per-block expert histogram for the grouping step
            const int64_t r = t * a.k + lane;
            atomicAdd(a.hist + (r / a.hist_chunk) * (a.E + 1) + my_e, 1);
        }
    }
    if (a.probs) {
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            const int e = e0 + q;
            if (e < a.E) a.probs[t * a.E + e] = sc_e[q];
        }
    }
    if (stat_row) {
#pragma unroll
        for (int q = 0; q < EPL; ++q)
            if (e0 + q < a.E) stat_row[e0 + q] = sc_e[q];
    }
    if (lane == 0 && a.shared_gate && a.w_shared_gate) {
        float ls = 0.f;
        for (int c = 0; c < S; ++c) ls += row[c * slab + nrw];
        a.shared_gate[t] = 1.f / (1.f + expf(-ls));
    }
}

// One warp per token: scoring, top-k and gates from a row of logits.  With
// the score statistic requested (a.stats), the 8 tokens' score rows are
// staged in shared memory and added in token order into row blockIdx.x of
// a.stats (tokens past T count as zero rows).
template <int EPL>
__global__ void __launch_bounds__(256) router_select_kernel(RouterArgs a, const float *partial, int LSP, int S,
                                                            int nrw) {
    extern __shared__ float s_rows[];   // [8, E] when a.stats
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * 8 + warp;
    float *stat_row = a.stats ? s_rows + warp * a.E : nullptr;
    if (t < a.T) {
        select_token<EPL>(a, partial, LSP, S, nrw, t, lane, stat_row);
    } else if (stat_row) {
        for (int e = lane; e < a.E; e += 32) stat_row[e] = 0.f;
    }
    if (a.stats) {
        __syncthreads();
        for (int e = threadIdx.x; e < a.E; e += 256) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) v += s_rows[w * a.E + e];
            a.stats[(int64_t)blockIdx.x * a.E + e] = v;
        }
    }
}

// Tiling of the logits GEMM for a batch (a pure function of the shape).
struct Plan {
    int nrw, L, BN, LSP, n_tiles, nk, S, kpc;
    int64_t m_tiles;
};
Plan plan(int64_t T, int d, int E, bool shared) {
    Plan p;
    p.nrw = (E + 7) / 8 * 8;
    p.L = p.nrw + (shared ? 1 : 0);
    p.BN = 16;
    while (p.BN < p.L && p.BN < kMaxBN) p.BN *= 2;
    p.n_tiles = (p.L + p.BN - 1) / p.BN;
    p.LSP = (p.L + 15) / 16 * 16;
    p.nk = (d + 63) / 64;
    p.m_tiles = (T + BM - 1) / BM;
    const int64_t tiles = p.m_tiles * p.n_tiles;
    int64_t S = kTargetCtas / tiles;
    S = S < 1 ? 1 : (S > p.nk ? p.nk : S);
    S = S > kMaxChunks ? kMaxChunks : S;
    p.kpc = (int)((p.nk + S - 1) / S);
    p.S = (p.nk + p.kpc - 1) / p.kpc;
    return p;
}

template <int BN>
cudaError_t launch_logits(const RouterArgs &a, const Plan &p, float *partial, cudaStream_t s) {
    const bool shared = a.w_shared_gate != nullptr;
    CUtensorMap mX, mW, mWB, mS;
    if (!make_map(&mX, a.x, false, (uint64_t)a.T, a.d, BM)) return cudaErrorInvalidValue;
    if (!make_map(&mW, a.w_router, false, (uint64_t)a.E, a.d, 8)) return cudaErrorInvalidValue;
    if (a.E >= BN) {
        if (!make_map(&mWB, a.w_router, false, (uint64_t)a.E, a.d, BN)) return cudaErrorInvalidValue;
    } else {
        mWB = mW;   // unused: tiles of fewer than BN router rows take 8-row boxes
    }
    if (shared) {
        if (!make_map(&mS, a.w_shared_gate, false, 1, a.d, 8)) return cudaErrorInvalidValue;
    } else {
        mS = mW;
    }
    const int64_t hist_ints = a.hist ? ((a.T * a.k + a.hist_chunk - 1) / a.hist_chunk) * (a.E + 1) : 0;
    LogitsArgs la{a.T, a.d, a.E, p.nrw, p.LSP, p.n_tiles, p.S, p.kpc, shared, partial, a.err, a.hist, hist_ints};
    const size_t smem = 1024 + (size_t)Shape<BN>::kStages * Shape<BN>::kStage + sizeof(Ctrl);
    auto kern = router_logits_kernel<BN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = p.m_tiles * p.n_tiles * p.S;   // one tile per CTA
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    return launch_kernel(kern, (unsigned)grid, kThreads, smem, s, mX, mW, mWB, mS, la);
}

}  // namespace rt

size_t router_tc_workspace_bytes(int64_t T, int d, int E, bool shared) {
    const rt::Plan p = rt::plan(T, d, E, shared);
    return sizeof(float) * (size_t)p.S * (size_t)T * p.LSP;
}

bool router_tc_supported(int64_t T, int E, int dtype) {
    return dtype == MOE_BF16 && T >= 128 && E <= MOE_MAX_EXPERTS;
}

cudaError_t launch_router_tc(const RouterArgs &a, float *scratch, cudaStream_t s) {
    using namespace rt;
    const Plan p = plan(a.T, a.d, a.E, a.w_shared_gate != nullptr);
    cudaError_t e;
    switch (p.BN) {
        case 16: e = launch_logits<16>(a, p, scratch, s); break;
        case 32: e = launch_logits<32>(a, p, scratch, s); break;
        case 64: e = launch_logits<64>(a, p, scratch, s); break;
        default: e = launch_logits<128>(a, p, scratch, s); break;
    }
    if (e != cudaSuccess) return e;
    const unsigned sgrid = (unsigned)((a.T + 7) / 8);
    const float *pt = scratch;
    const size_t ssm = a.stats ? sizeof(float) * 8 * (size_t)a.E : 0;
    if (a.E <= 64) e = launch_kernel(router_select_kernel<2>, sgrid, 256, ssm, s, a, pt, p.LSP, p.S, p.nrw);
    else if (a.E <= 128) e = launch_kernel(router_select_kernel<4>, sgrid, 256, ssm, s, a, pt, p.LSP, p.S, p.nrw);
    else if (a.E <= 256) e = launch_kernel(router_select_kernel<8>, sgrid, 256, ssm, s, a, pt, p.LSP, p.S, p.nrw);
    else e = launch_kernel(router_select_kernel<16>, sgrid, 256, ssm, s, a, pt, p.LSP, p.S, p.nrw);
    if (e == cudaSuccess && a.stats && a.score_mean) e = launch_router_stats(a.stats, sgrid, a.E, a.T, a.score_mean, s);
    return e;
}

}  // namespace moe
