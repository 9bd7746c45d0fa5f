// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05, TMEM
// accumulators, TMA), for the variable-size expert segments of a MoE layer.
//
//   GATEUP: act[i, n] = silu(W_gate[e, n] . a_i) * (W_up[e, n] . a_i)
//   DOWN  : y_acc[t_i, n] += g_i * (W_down[e, n] . a_i)
//
// where i runs over the grouped rows of expert e.  "Tutorial 11: Mixture of
// Experts (MoE)", section 3 "Expert Computation" (tokens grouped by expert, a
// grouped matrix multiply per projection, silu(gate) * up, weighted sum back
// in token order); "Small models, sparse experts", section "Dispatch decides
// everything" (read each token's expert weights in place, no gathered weight
// copies, no padding of groups to a common length).
//
// Design (sm_100a), one SM per tile (grouped_gemm2.cu holds the two-SM form):
//  * Persistent CTAs, one per SM, walk a tile list derived on the device from
//    the expert offsets: tiles are 128 grouped rows (64 with HALF) x (128 gate
//    + 128 up columns) for GATEUP, x 256 (or 128 when the output width is not
//    a multiple of 256) for DOWN; expert-major, and inside an expert the row
//    tiles vary fastest so CTAs running at the same time share one weight
//    tile through L2.  Partial row tiles at a segment's end are computed and
//    masked, never padded in memory.
//  * Warp roles: warps 0-3 epilogue (TMEM lane quarters 0-3), warp 4 TMA
//    producer, warp 5 TMEM allocator + single-thread MMA issuer, warps 6-13
//    token-row gather (routed gate/up).
//  * Weights (and contiguous A operands) arrive by TMA 2D tiles, 128-byte
//    swizzle, no multicast; weights read by one tile only carry an
//    evict-first L2 policy.  Token rows x[t] of the routed gate/up GEMM are
//    read in place by index: the gather warps issue 16-byte cp.async copies
//    straight into the 128-byte-swizzled K-major layout the MMA descriptor
//    reads, and signal each stage with a non-blocking
//    cp.async.mbarrier.arrive.noinc (the arrival lands when the thread's
//    copies have), so the gather runs as far ahead as the ring allows; no copy
//    of x is ever made.  (TMA tile::gather4 was measured 2.3x slower here.)  A
//    192 KB shared-memory ring (4 stages of 48 KB, 6 of 32 KB, 8 of 24 KB) is
//    guarded by full/empty mbarriers; the MMA thread frees a stage with
//    tcgen05.commit.
//  * One tcgen05.mma.cta_group::1 of M=128, N=BN per 32-byte K slice
//    (kind::f16 for bf16, kind::tf32 for fp32), fp32 accumulators in TMEM,
//    double-buffered (2 x 256 columns) so the epilogue of tile i overlaps the
//    main loop of tile i+1.
//  * Epilogues (grouped_parts.cuh): GATEUP reads gate and up columns of the
//    same row from TMEM (tcgen05.ld 32x32b), applies silu(g)*u and stores act;
//    DOWN scales each row by its gate and adds it into the fp32 accumulator
//    with 16-byte vector reductions (the combine over the k experts of a
//    token).
//  * With programmatic dependent launch the prologue overlaps the previous
//    kernel; when the offsets are known complete (two kernels back) the first
//    ring of weight tiles is issued before waiting for it.
//  * Every mbarrier wait is bounded (4 s of %globaltimer); on expiry the CTA
//    raises the device timeout flag, the other roles stop at their next wait,
//    outstanding copies are drained and TMEM is released before exit.
#include <algorithm>

#include "grouped_parts.cuh"

namespace moe {
namespace gg {

using namespace tc;

constexpr int BM = 128;
constexpr int kABytes = BM * 128;     // one A stage: 128 rows x 128 bytes
constexpr int kMaxStages = 8;
// Shared-memory ring depth for an MMA N of BN and A stages of a_bytes: as many
// stages as fit in 192 KB.
constexpr int stages_for(int BN, int a_bytes = kABytes) {
    const int s = 196608 / (a_bytes + BN * 128);
    return s > kMaxStages ? kMaxStages : s;
}
#ifndef MOE_GG_L2_PROMOTION
#define MOE_GG_L2_PROMOTION CU_TENSOR_MAP_L2_PROMOTION_L2_256B
#endif
constexpr int kEpiWarps = 4;
constexpr int kTmaWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kGatherWarp0 = 6;
#ifndef MOE_GATHER_THREADS
#define MOE_GATHER_THREADS 256
#endif
constexpr int kGatherThreads = MOE_GATHER_THREADS;   // 128 or 256
constexpr int kTmemCols = 512;

using Params = GemmParams;

struct Ctrl {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint32_t tmem_base;
    int abort;
    int n_mtiles;
    int pad;
};

// ------------------------------------------------------------------ kernel

// Pipeline trace of this kernel in a diagnostic build (-DMOE_PIPE_TRACE; read
// with moe_debug_fwd_trace): per variant (gate/up, down, 64-row down), SM
// cycles summed over CTAs for [0] the whole kernel, [1] the MMA issuer
// waiting for operands, [2] it waiting for a free accumulator, [3] the TMA
// producer waiting for a free stage, [4] epilogue warp 0 waiting for an
// accumulator, [5] it draining one, [6] the number of CTAs, [7] the first
// gather thread waiting for a free stage.
#ifdef MOE_PIPE_TRACE
__device__ unsigned long long g_fwd_trace[4][8];
#define FWD_SLOT(var, slot) (&g_fwd_trace[var][slot])
#else
#define FWD_SLOT(var, slot) nullptr
#endif

// HALF (contiguous A only): 64-row tiles whose A stage holds 64 rows, for
// experts of at most 64 rows, where the weights stream from HBM and the rows
// of a 128-row A stage would mostly sit empty.  The MMA still has M = 128: its
// rows 64-127 read the next 8 KB of shared memory (the following stage, or a
// pad after the last one) and land in TMEM lanes no epilogue thread reads.
// The smaller stages fit 8 in the ring instead of 6, a third more weight bytes
// in flight per SM.
template <int MODE, bool GATHER, typename T, int BN, bool HALF>
__global__ void __launch_bounds__(GATHER ? 192 + kGatherThreads : 192, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1, Params p) {
    constexpr int BK = 128 / (int)sizeof(T);   // elements per 128-byte K block
    constexpr int BN_OUT = MODE == GATEUP ? BN / 2 : BN;   // output columns per tile
    static_assert(!(HALF && GATHER), "half-height A tiles are loaded by TMA");
    constexpr int RB = HALF ? BM / 2 : BM;                 // grouped rows per tile
    constexpr int kAStage = RB * 128;                      // one A stage: RB rows x 128 bytes
    constexpr int kAPad = kABytes - kAStage;               // room for the MMA's reads past the last stage
    constexpr int kStages = stages_for(BN, kAStage);
    constexpr int kBBytes = BN * 128;                      // one B stage: BN rows x 128 bytes
    constexpr uint32_t kIdesc = instr_desc<T>(BM, BN);
    constexpr int kStageBytes = MODE == DOWN ? kEpiWarps * kEpiStageBytes : 0;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + kStages * kAStage + kAPad;
    uint8_t *sEpi = sB + kStages * kBBytes;                // DOWN epilogue staging
    Ctrl *ctrl = reinterpret_cast<Ctrl *>(sEpi + kStageBytes);
    int *tile_start = reinterpret_cast<int *>(ctrl + 1);
    int *seg_off = tile_start + (p.E + 1);
    int *seg_end = seg_off + (p.E + 1);
    volatile int *abort = &ctrl->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ctrl->full[s], GATHER ? 1 + kGatherThreads : 1);
            mbar_init(&ctrl->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&ctrl->tfull[a], 1);
            mbar_init(&ctrl->tempty[a], kEpiWarps * 32);
        }
        ctrl->abort = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) tmem_alloc(&ctrl->tmem_base, kTmemCols);
    if (warp == kTmaWarp && lane == 0) {
        prefetch_tmap(&tmB0);
        if (MODE == GATEUP) prefetch_tmap(&tmB1);
        if (!GATHER) prefetch_tmap(&tmA);
    }
    // everything above overlaps the previous kernel's tail.  Data the previous
    // kernel may still be writing (act, sorted rows, offsets right after the
    // grouping step) is read only after pdl_wait(); what p.early marks as
    // complete already (weights, the layer input, offsets from further back)
    // is read before it, so the first weight tiles are in flight early.
    const bool early_tiles = (p.early & kEarlyTiles) != 0;
    if (!early_tiles && (p.early & kEarlyPrefetch) && warp == kTmaWarp && lane == 0) {
        // with one row tile per expert and every expert active, tile id is
        // (expert id / n_tiles, column tile id % n_tiles)
        const int nt = (p.N + BN_OUT - 1) / BN_OUT, e = blockIdx.x / nt;
        if (e < p.E) {
            const int b_row = e * p.N + (blockIdx.x - e * nt) * BN_OUT;
            for (int kb = 0; kb < (p.K + BK - 1) / BK; ++kb) {
                tma_prefetch_2d(&tmB0, kb * BK, b_row);
                if (MODE == GATEUP) tma_prefetch_2d(&tmB1, kb * BK, b_row);
            }
        }
    }
    if (!early_tiles) pdl_wait();
    if (warp == kTmaWarp) build_tiles<RB>(p, tile_start, seg_off, seg_end, &ctrl->n_mtiles);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // dependents are released only after this CTA's TMEM is allocated and after
    // the wait.  With early loads the producer warp skips the wait here (a warp
    // waits as a whole) and its issuing lane waits once it has issued them.
    if (!early_tiles) {
        pdl_launch_dependents();
    } else if (warp != kTmaWarp) {
        pdl_wait();
        pdl_launch_dependents();
    }

    const uint32_t tmem = ctrl->tmem_base;
    const int n_tiles = (p.N + BN_OUT - 1) / BN_OUT;
    const int total = ctrl->n_mtiles * n_tiles;
    const int nk = (p.K + BK - 1) / BK;
    const int nE = p.offsets ? p.E : 1;
    constexpr int kPtVar = MODE == GATEUP ? 0 : (HALF ? 2 : 1);
    PipeClock ck_total, ck_a, ck_b;
    ck_total.start();

    if (warp == kTmaWarp) {
        if (lane == 0) {
            // weights that no other tile reads again stream through L2 with an
            // evict-first policy, so what is reused from L2 (prefetched weights,
            // the gathered rows, act, the combine accumulator) stays
            const uint64_t wpol = l2_evict_first_policy();
            auto load_b = [&](int s, int kb, int b_row) {
                if (p.stream_weights) {
                    tma_load_2d_hint(&tmB0, sB + s * kBBytes, &ctrl->full[s], kb * BK, b_row, wpol);
                    if (MODE == GATEUP)
                        tma_load_2d_hint(&tmB1, sB + s * kBBytes + kBBytes / 2, &ctrl->full[s], kb * BK, b_row, wpol);
                } else {
                    tma_load_2d(&tmB0, sB + s * kBBytes, &ctrl->full[s], kb * BK, b_row);
                    if (MODE == GATEUP)
                        tma_load_2d(&tmB1, sB + s * kBBytes + kBBytes / 2, &ctrl->full[s], kb * BK, b_row);
                }
            };
            const bool early_a = !GATHER && (p.early & kEarlyA) != 0;
            // the first kStages stages are free: fill them with weight tiles (and
            // the A tiles, when they are complete already) before waiting
            uint32_t pre = 0;
            if (early_tiles) {
                for (int id = blockIdx.x; id < total && pre < (uint32_t)kStages; id += gridDim.x) {
                    const Tile tl = decode_n(id, n_tiles, p.n_groups, ctrl->n_mtiles, tile_start, nE);
                    const int a_row = seg_off[tl.e] + tl.m * RB;
                    const int b_row = tl.e * p.N + tl.n * BN_OUT;
                    for (int kb = 0; kb < nk && pre < (uint32_t)kStages; ++kb, ++pre) {
                        mbar_expect_tx(&ctrl->full[pre], kBBytes + (GATHER ? 0 : kAStage));
                        if (early_a) tma_load_2d(&tmA, sA + pre * kAStage, &ctrl->full[pre], kb * BK, a_row);
                        load_b((int)pre, kb, b_row);
                    }
                }
                pdl_wait();
                pdl_launch_dependents();
            }
            uint32_t it = 0;
            bool ok = true;
            for (int id = blockIdx.x; id < total && ok; id += gridDim.x) {
                const Tile tl = decode_n(id, n_tiles, p.n_groups, ctrl->n_mtiles, tile_start, nE);
                const int a_row = seg_off[tl.e] + tl.m * RB;
                const int b_row = tl.e * p.N + tl.n * BN_OUT;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (it < pre) {
                        // issued above; only the A tile may still be missing
                        if (!GATHER && !early_a) tma_load_2d(&tmA, sA + s * kAStage, &ctrl->full[s], kb * BK, a_row);
                        continue;
                    }
                    ck_a.start();
                    const bool got = wait_bar(&ctrl->empty[s], ph ^ 1, abort, p.err);
                    ck_a.stop();
                    if (!got) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&ctrl->full[s], kBBytes + (GATHER ? 0 : kAStage));
                    if (!GATHER) tma_load_2d(&tmA, sA + s * kAStage, &ctrl->full[s], kb * BK, a_row);
                    load_b(s, kb, b_row);
                }
            }
            ck_a.flush(FWD_SLOT(kPtVar, 3));
            if (!ok) {
                // aborting: let the copies already issued land before the CTA exits
                for (uint32_t j = it > kStages ? it - kStages : 0; j < it; ++j) {
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try_wait(&ctrl->full[j % kStages], (j / kStages) & 1) &&
                           globaltimer() - t0 < 100000000ull) {
                    }
                }
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int id = blockIdx.x; id < total && ok; id += gridDim.x, ++tc) {
                const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
                ck_b.start();
                const bool free_acc = wait_bar(&ctrl->tempty[acc], aph ^ 1, abort, p.err);
                ck_b.stop();
                if (!free_acc) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + acc * BN;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    ck_a.start();
                    const bool got = wait_bar(&ctrl->full[s], ph, abort, p.err);
                    ck_a.stop();
                    if (!got) {
                        ok = false;
                        break;
                    }
                    // gathered rows were written by cp.async (generic proxy); the
                    // MMA reads them through the async proxy
                    if constexpr (GATHER) fence_proxy_async();
                    tc_fence_after();
                    const uint64_t ad = smem_desc(sA + s * kAStage);
                    const uint64_t bd = smem_desc(sB + s * kBBytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)   // four 32-byte K slices per 128-byte block
                        mma<T>(d_tmem, ad + 2 * kk, bd + 2 * kk, kIdesc, (kb | kk) != 0);
                    mma_commit(&ctrl->empty[s]);
                }
                if (ok) mma_commit(&ctrl->tfull[acc]);
            }
            ck_a.flush(FWD_SLOT(kPtVar, 1));
            ck_b.flush(FWD_SLOT(kPtVar, 2));
        }
    } else if (warp < kEpiWarps) {
        if (MODE == GATEUP && p.zero) {
            // clear this CTA's share of the down GEMM's accumulator while the
            // first tile's operands stream in
            const int64_t n4 = p.zero_floats / 4;
            const int64_t per = (n4 + gridDim.x - 1) / gridDim.x;
            const int64_t b = (int64_t)blockIdx.x * per, e = min(n4, b + per);
            float4 *z = reinterpret_cast<float4 *>(p.zero);
            for (int64_t i = b + threadIdx.x; i < e; i += kEpiWarps * 32) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        uint32_t tc = 0;
        const int row = warp * 32 + lane;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        for (int id = blockIdx.x; id < total; id += gridDim.x, ++tc) {
            const Tile tl = decode_n(id, n_tiles, p.n_groups, ctrl->n_mtiles, tile_start, nE);
            const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
            ck_a.start();
            const bool ready = wait_bar(&ctrl->tfull[acc], aph, abort, p.err);
            ck_a.stop();
            if (!ready) break;
            tc_fence_after();
            ck_b.start();
            const int64_t r = (int64_t)seg_off[tl.e] + (int64_t)tl.m * RB + row;
            epilogue_row<MODE, T, BN>(p, tl.n, r, row < RB && r < seg_end[tl.e], tmem + acc * BN + lane_base,
                                      reinterpret_cast<float *>(sEpi + warp * kEpiStageBytes));
            ck_b.stop();
            tc_fence_before();
            mbar_arrive(&ctrl->tempty[acc]);
        }
        if (threadIdx.x == 0) {
            ck_a.flush(FWD_SLOT(kPtVar, 4));
            ck_b.flush(FWD_SLOT(kPtVar, 5));
        }
    } else if (GATHER && warp >= kGatherWarp0) {
        PipeClock ck_g;
        gather_rows<T, kStages, RB, kGatherThreads>(p, threadIdx.x - kGatherWarp0 * 32, blockIdx.x, gridDim.x, total, n_tiles,
                                    tile_start, seg_off, seg_end, nE, nk, 0, sA, ctrl->full, ctrl->empty, abort,
                                    &ck_g);
        if (threadIdx.x == kGatherWarp0 * 32) ck_g.flush(FWD_SLOT(kPtVar, 7));
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
    ck_total.stop();
    if (threadIdx.x == 0) {
        ck_total.flush(FWD_SLOT(kPtVar, 0));
#ifdef MOE_PIPE_TRACE
        atomicAdd(&g_fwd_trace[kPtVar][6], 1ull);
#endif
    }
}

// ------------------------------------------------------------------ host side

template <int MODE, bool GATHER, typename T, int BN, bool HALF>
cudaError_t launch_t(const GemmLaunch &L, cudaStream_t s) {
    const Params &p = L.p;
    constexpr int BN_OUT = MODE == GATEUP ? BN / 2 : BN;
    constexpr int RB = HALF ? BM / 2 : BM;
    constexpr int kStages = stages_for(BN, RB * 128);
    const bool f32 = sizeof(T) == 4;
    CUtensorMap mA, mB0, mB1;
    const int nE = p.offsets ? p.E : 1;
    const CUtensorMapL2promotion wp = MOE_GG_L2_PROMOTION;
    if (!make_map(&mB0, L.b0, f32, (uint64_t)nE * p.N, p.K, BN_OUT, wp)) return cudaErrorInvalidValue;
    if (MODE == GATEUP) {
        if (!make_map(&mB1, L.b1, f32, (uint64_t)nE * p.N, p.K, BN_OUT, wp)) return cudaErrorInvalidValue;
    } else {
        mB1 = mB0;
    }
    if (!GATHER) {
        if (!make_map(&mA, L.a_src, f32, (uint64_t)p.rows, p.K, RB)) return cudaErrorInvalidValue;
    } else {
        mA = mB0;   // unused: gather mode reads x with cp.async
    }
    const int n_tiles = (p.N + BN_OUT - 1) / BN_OUT;
    const int64_t max_m = p.rows / RB + nE;
    const int64_t max_tiles = max_m * n_tiles;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms(), max_tiles));
    const size_t smem = 1024 + (size_t)kStages * (RB * 128 + BN * 128) + (kABytes - RB * 128) +
                        (MODE == DOWN ? kEpiWarps * kEpiStageBytes : 0) + sizeof(Ctrl) + 3 * sizeof(int) * (p.E + 1);
    auto kern = grouped_gemm_kernel<MODE, GATHER, T, BN, HALF>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(kern, grid, GATHER ? 192 + kGatherThreads : 192, smem, s, mA, mB0, mB1, p);
}

template <int MODE, bool GATHER, typename T>
cudaError_t launch_bn(const GemmLaunch &L, cudaStream_t s) {
    if constexpr (!GATHER) {
        if (L.half)
            return L.narrow ? launch_t<MODE, GATHER, T, 128, true>(L, s) : launch_t<MODE, GATHER, T, 256, true>(L, s);
    }
    return L.narrow ? launch_t<MODE, GATHER, T, 128, false>(L, s) : launch_t<MODE, GATHER, T, 256, false>(L, s);
}

}  // namespace gg

cudaError_t launch_grouped_gemm(const GemmLaunch &L, cudaStream_t s) {
    const GemmParams &p = L.p;
    if (p.rows <= 0) return cudaSuccess;
    if (L.pair) return launch_grouped_gemm_pair(L, s);
    const bool f32 = L.dtype == MOE_F32;
    if (L.mode == gg::GATEUP) {
        if (L.gather)
            return f32 ? gg::launch_bn<gg::GATEUP, true, float>(L, s)
                       : gg::launch_bn<gg::GATEUP, true, __nv_bfloat16>(L, s);
        return f32 ? gg::launch_bn<gg::GATEUP, false, float>(L, s)
                   : gg::launch_bn<gg::GATEUP, false, __nv_bfloat16>(L, s);
    }
    return f32 ? gg::launch_bn<gg::DOWN, false, float>(L, s) : gg::launch_bn<gg::DOWN, false, __nv_bfloat16>(L, s);
}

}  // namespace moe

#ifdef MOE_PIPE_TRACE
// Diagnostic build only: copies the forward pipeline trace (4 x 8 counters,
// see above) to host memory and optionally clears it.
extern "C" int moe_debug_fwd_trace(unsigned long long *out, int reset) {
    if (cudaDeviceSynchronize() != cudaSuccess) return 1;
    if (cudaMemcpyFromSymbol(out, moe::gg::g_fwd_trace, sizeof(moe::gg::g_fwd_trace)) != cudaSuccess) return 1;
    if (reset) {
        static const unsigned long long zero[4][8] = {};
        if (cudaMemcpyToSymbol(moe::gg::g_fwd_trace, zero, sizeof(zero)) != cudaSuccess) return 1;
    }
    return 0;
}
#endif
