// Grouped expert GEMMs on two SMs per tile (tcgen05.mma.cta_group::2), for
// layers whose experts hold many rows (the tensor-bound regime).
//
// Same math and tile order as grouped_gemm.cu ("Tutorial 11: Mixture of
// Experts (MoE)", section 3 "Expert Computation"), with the tiles doubled in
// M: a cluster of two CTAs computes 256 grouped rows x BN columns.  Each CTA
// stages its own 128 rows of A and its own half of the B columns (for gate/up:
// CTA 0 the gate rows, CTA 1 the up rows), so per K block a CTA moves 32 KB
// into shared memory for the same MMA work that costs 48 KB on one SM: the
// operand traffic per FLOP, which bounds the one-SM kernel on these layers,
// drops by a third.  The even CTA issues M=256 MMAs that read both CTAs'
// shared memory and write each CTA's half of D into its own TMEM.  The
// gathered gate/up runs with wide tiles (two MMAs per K slice, see W below).
//
// Synchronisation across the pair:
//  * both CTAs' TMA loads complete on the even CTA's full[s] barrier (the
//    even CTA posts the expected bytes of both); gathered token rows of the
//    odd CTA are signalled by a relay thread that waits for the local cp.async
//    arrivals and arrives on the even CTA's full[s];
//  * tcgen05.commit multicasts the stage release (empty[s]) and the
//    accumulator-ready signal (tfull) to both CTAs;
//  * each CTA's epilogue warps release the accumulator on the even CTA's
//    tempty barrier (the odd CTA's by remote arrive);
//  * cluster barriers after set-up and before exit keep every barrier and
//    shared buffer alive while the peer may still touch it.
// Every mbarrier wait is bounded as in the one-SM kernel.
#include <algorithm>
#include <mutex>

#include "grouped_parts.cuh"

namespace moe {
namespace gg {
namespace {

constexpr int BM2 = 256;                  // grouped rows per pair tile
constexpr int kHalfRows = 128;            // rows per CTA
constexpr int kABytes = kHalfRows * 128;  // one A stage: 128 rows x 128 bytes
constexpr int kMaxStages = 8;
// Warp roles: epilogue warps 0 .. EW-1, then the TMA producer, the MMA issuer
// (the gather relay in the odd CTA) and the gather warps.  Gate/up drains a
// half accumulator while the MMAs of its tile's other half, or of the next
// tile's first K blocks, run: with eight epilogue warps (two per TMEM lane
// quarter, each half of the columns) the drain is short enough that the MMA
// issuer rarely waits for it.
#ifndef MOE_GG2_GATEUP_EPI_WARPS
#define MOE_GG2_GATEUP_EPI_WARPS 8
#endif
#ifndef MOE_GG2_GATHER_THREADS
#define MOE_GG2_GATHER_THREADS 128
#endif
constexpr int kGatherThreads = MOE_GG2_GATHER_THREADS;
static_assert(kGatherThreads == 128 || kGatherThreads == 256, "8 threads per row, 128 rows in whole passes");
template <int MODE>
constexpr int epi_warps() {
    return MODE == GATEUP ? MOE_GG2_GATEUP_EPI_WARPS : 4;
}
static_assert(MOE_GG2_GATEUP_EPI_WARPS == 4 || MOE_GG2_GATEUP_EPI_WARPS == 8, "one or two warps per lane quarter");
template <int MODE, bool GATHER>
constexpr int pair_threads() {
    return (epi_warps<MODE>() + 2) * 32 + (GATHER ? kGatherThreads : 0);
}
constexpr int kTmemCols = 512;

// Ring depth for an MMA N of BN (each CTA holds BN / 2 rows of B per stage).
constexpr int pair_stages(int BN) {
    const int s = 196608 / (kABytes + BN * 64);
    return s > kMaxStages ? kMaxStages : s;
}

struct Ctrl2 {
    uint64_t full[kMaxStages];    // even CTA: operands of a K block landed (both CTAs)
    uint64_t empty[kMaxStages];   // both: the MMAs of a K block are done
    uint64_t gfull[kMaxStages];   // odd CTA: its gathered rows landed (relayed to the even CTA)
    uint64_t tfull[2];            // both: accumulator ready
    uint64_t tempty[2];           // even CTA: accumulator released by both epilogues
    uint64_t done;                // both: all MMAs of the CTA pair completed
    uint32_t tmem_base;
    int abort;
    int n_mtiles;
    int pad;
};

// W = 2 (gathered gate/up): each pair tile issues two N = BN MMAs per K slice
// into one 2 x BN column accumulator, so every gathered token row feeds twice
// the output columns and the gather, which bounds this GEMM, is needed at half
// the rate per FLOP.  The accumulator then fills TMEM, so instead of two
// accumulators its two halves (MMA j = 0 and 1) are handed over separately:
// in a tile's last ring of K blocks the MMAs of half 0 run first and half 0
// goes to the epilogue while half 1 finishes, and in the next tile's first
// ring of K blocks half 0 is started while the epilogue still drains half 1.
// Pipeline trace of this kernel in a diagnostic build (-DMOE_PIPE_TRACE; read
// with moe_debug_fwd2_trace): per variant (gathered gate/up, contiguous
// gate/up, down), SM cycles summed over CTAs for [0] the whole kernel, [1] the
// MMA issuer waiting for operands, [2] it waiting for an accumulator, [3] the
// TMA producers waiting for a free stage, [4] epilogue warp 0 waiting for an
// accumulator, [5] it draining one, [6] the number of CTAs, [7] the first
// gather thread waiting for a free stage.
#ifdef MOE_PIPE_TRACE
__device__ unsigned long long g_fwd2_trace[4][8];
#define FWD2_SLOT(var, slot) (&g_fwd2_trace[var][slot])
#else
#define FWD2_SLOT(var, slot) nullptr
#endif

template <int MODE, bool GATHER, typename T, int BN, int W>
__global__ void __launch_bounds__(pair_threads<MODE, GATHER>(), 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                             const __grid_constant__ CUtensorMap tmB1, GemmParams p) {
    constexpr int kEpiWarps = epi_warps<MODE>(), kTmaWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1,
                  kGatherWarp0 = kEpiWarps + 2;
    constexpr int BK = 128 / (int)sizeof(T);
    static_assert(W == 1 || (W == 2 && MODE == GATEUP), "wide tiles are for gate/up");
    constexpr int BN_OUT = MODE == GATEUP ? W * BN / 2 : BN;   // output columns per tile
    constexpr int kStages = pair_stages(W * BN);
    constexpr int kBSub = BN * 64;                   // this CTA's half of one MMA's B
    constexpr int kBBytes = W * kBSub;               // this CTA's B per stage
    constexpr uint32_t kIdesc = instr_desc<T>(BM2, BN);
    constexpr int kStageBytes = MODE == DOWN ? kEpiWarps * kEpiStageBytes : 0;
    static_assert(MODE == GATEUP || kEpiWarps == 4, "the down epilogue stages 4 warps' rows");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + kStages * kABytes;
    uint8_t *sEpi = sB + kStages * kBBytes;                // DOWN epilogue staging
    Ctrl2 *ctrl = reinterpret_cast<Ctrl2 *>(sEpi + kStageBytes);
    int *tile_start = reinterpret_cast<int *>(ctrl + 1);
    int *seg_off = tile_start + (p.E + 1);
    int *seg_end = seg_off + (p.E + 1);
    volatile int *abort = &ctrl->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool lead = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            // the even CTA's expect_tx arrival (+ its 128 gather threads and the
            // odd CTA's relay when the rows are gathered)
            mbar_init(&ctrl->full[s], GATHER ? 1 + kGatherThreads + 1 : 1);
            mbar_init(&ctrl->empty[s], 1);
            mbar_init(&ctrl->gfull[s], kGatherThreads);
        }
        // W = 1: two accumulators; W = 2: the two halves of one
        for (int a = 0; a < 2; ++a) {
            mbar_init(&ctrl->tfull[a], 1);
            mbar_init(&ctrl->tempty[a], 2 * kEpiWarps);
        }
        mbar_init(&ctrl->done, 1);
        ctrl->abort = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) tmem_alloc2(&ctrl->tmem_base, kTmemCols);
    if (warp == kTmaWarp && lane == 0) {
        prefetch_tmap(&tmB0);
        if (MODE == GATEUP) prefetch_tmap(&tmB1);
        if (!GATHER) prefetch_tmap(&tmA);
    }
    pdl_wait();
    if (warp == kTmaWarp) build_tiles<BM2>(p, tile_start, seg_off, seg_end, &ctrl->n_mtiles);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync_all();   // both CTAs' barriers exist before any remote arrive
    pdl_launch_dependents();
    [[maybe_unused]] constexpr int kPtVar = MODE == GATEUP ? (GATHER ? 0 : 1) : 2;
    PipeClock ck_total, ck_a, ck_b;
    ck_total.start();

    const uint32_t tmem = ctrl->tmem_base;
    const int n_tiles = (p.N + BN_OUT - 1) / BN_OUT;
    const int total = ctrl->n_mtiles * n_tiles;
    const int nk = (p.K + BK - 1) / BK;
    const int nE = p.offsets ? p.E : 1;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int row_off = (int)rank * kHalfRows;   // this CTA's rows inside a 256-row tile

    if (warp == kTmaWarp) {
        if (lane == 0) {
            // this CTA's A rows (when contiguous) and its half of the B columns,
            // completing on the even CTA's full[s]; the even CTA posts the bytes
            // of both CTAs
            constexpr uint32_t kTx = 2u * (uint32_t)(kBBytes + (GATHER ? 0 : kABytes));
            const uint32_t full_lead = mapa_shared(&ctrl->full[0], 0);   // the even CTA's full[0]
            const CUtensorMap *mb = (MODE == GATEUP && !lead) ? &tmB1 : &tmB0;
            uint32_t it = 0;
            bool ok = true;
            for (int id = pair; id < total && ok; id += npairs) {
                const Tile tl = decode_n(id, n_tiles, p.n_groups, ctrl->n_mtiles, tile_start, nE);
                const int a_row = seg_off[tl.e] + tl.m * BM2 + row_off;
                // gate/up: the gate rows from CTA 0, the up rows from CTA 1 (W x
                // BN / 2 of them, one box); down: the first and second half of
                // the BN weight rows
                const int b_row = tl.e * p.N + tl.n * BN_OUT + (MODE == GATEUP ? 0 : (int)rank * (BN / 2));
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    ck_a.start();
                    const bool free_stage = wait_bar(&ctrl->empty[s], ((it / kStages) & 1) ^ 1, abort, p.err);
                    ck_a.stop();
                    if (!free_stage) {
                        ok = false;
                        break;
                    }
                    if (lead) mbar_expect_tx(&ctrl->full[s], kTx);
                    const uint32_t fb = full_lead + s * (uint32_t)sizeof(uint64_t);
                    if (!GATHER) tma_load_2d_pair(&tmA, sA + s * kABytes, fb, kb * BK, a_row);
                    tma_load_2d_pair(mb, sB + s * kBBytes, fb, kb * BK, b_row);
                }
            }
            if (!ok) {
                // aborting: let this CTA's copies land before it leaves (the last
                // stages it filled are released by the MMAs or time out)
                for (uint32_t j = it > (uint32_t)kStages ? it - kStages : 0; j < it; ++j) {
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try_wait(&ctrl->empty[j % kStages], (j / kStages) & 1) &&
                           globaltimer() - t0 < 100000000ull) {
                    }
                }
            }
        }
        if (lane == 0) ck_a.flush(FWD2_SLOT(kPtVar, 3));
    } else if (warp == kMmaWarp) {
        if (lane == 0 && lead) {
            uint32_t it = 0, tc = 0;
            bool ok = true;
            // the operands of ring position i have landed (both CTAs)
            auto wait_full = [&](uint32_t i) -> bool {
                const int s = i % kStages;
                const uint32_t ph = (i / kStages) & 1;
                ck_a.start();
                bool got = mbar_try_wait_cluster(&ctrl->full[s], ph);
                if (!got) got = wait_bar(&ctrl->full[s], ph, abort, p.err) && mbar_try_wait_cluster(&ctrl->full[s], ph);
                ck_a.stop();
                if (got) {
                    if constexpr (GATHER) fence_proxy_async();
                    tc_fence_after();
                }
                return got;
            };
            // MMA j of K block kb from ring position i into accumulator columns d
            auto issue = [&](uint32_t i, int kb, int j, uint32_t d) {
                const int s = i % kStages;
                const uint64_t ad = smem_desc(sA + s * kABytes);
                // B rows j * BN / 2 .. of each CTA
                const uint64_t bd = smem_desc(sB + s * kBBytes + j * kBSub);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma2<T>(d + j * BN, ad + 2 * kk, bd + 2 * kk, kIdesc, (kb | kk) != 0);
            };
            auto release = [&](uint32_t i) { mma_commit2(&ctrl->empty[i % kStages], 0x3); };
            for (int id = pair; id < total && ok; id += npairs, ++tc) {
                if constexpr (W == 1) {
                    const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
                    ck_b.start();
                    const bool free_acc = wait_bar(&ctrl->tempty[acc], aph ^ 1, abort, p.err);
                    ck_b.stop();
                    if (!free_acc) break;
                    tc_fence_after();
                    for (int kb = 0; kb < nk; ++kb, ++it) {
                        if (!wait_full(it)) {
                            ok = false;
                            break;
                        }
                        issue(it, kb, 0, tmem + acc * BN);
                        release(it);
                    }
                    if (ok) mma_commit2(&ctrl->tfull[acc], 0x3);
                } else {
                    const uint32_t aph = tc & 1;
                    const int H = nk < kStages ? nk : kStages;                      // head K blocks
                    const int Tb = nk - H < kStages ? nk - H : kStages;            // tail K blocks
                    // head: half 0 over the first ring once the epilogue has
                    // released it, then half 1 once that is released too
                    ck_b.start();
                    const bool free_half0 = wait_bar(&ctrl->tempty[0], aph ^ 1, abort, p.err);
                    ck_b.stop();
                    if (!free_half0) break;
                    tc_fence_after();
                    for (int kb = 0; kb < H && ok; ++kb) {
                        if (wait_full(it + kb)) issue(it + kb, kb, 0, tmem);
                        else ok = false;
                    }
                    if (!ok) break;
                    if (H == nk) mma_commit2(&ctrl->tfull[0], 0x3);
                    ck_b.start();
                    const bool free_half1 = wait_bar(&ctrl->tempty[1], aph ^ 1, abort, p.err);
                    ck_b.stop();
                    if (!free_half1) break;
                    tc_fence_after();
                    for (int kb = 0; kb < H; ++kb) {
                        issue(it + kb, kb, 1, tmem);
                        release(it + kb);
                    }
                    it += H;
                    // body: both halves per K block
                    for (int kb = H; kb < nk - Tb; ++kb, ++it) {
                        if (!wait_full(it)) {
                            ok = false;
                            break;
                        }
                        issue(it, kb, 0, tmem);
                        issue(it, kb, 1, tmem);
                        release(it);
                    }
                    if (!ok) break;
                    // tail: half 0 over the last ring, handed to the epilogue,
                    // then half 1
                    if (Tb > 0) {
                        for (int q = 0; q < Tb && ok; ++q) {
                            if (wait_full(it + q)) issue(it + q, nk - Tb + q, 0, tmem);
                            else ok = false;
                        }
                        if (!ok) break;
                        mma_commit2(&ctrl->tfull[0], 0x3);
                        for (int q = 0; q < Tb; ++q) {
                            issue(it + q, nk - Tb + q, 1, tmem);
                            release(it + q);
                        }
                        it += Tb;
                    }
                    mma_commit2(&ctrl->tfull[1], 0x3);
                }
            }
            mma_commit2(&ctrl->done, 0x3);
            ck_a.flush(FWD2_SLOT(kPtVar, 1));
            ck_b.flush(FWD2_SLOT(kPtVar, 2));
        } else if (lane == 0 && GATHER) {
            // odd CTA: relay its gathered rows of each K block to the even CTA
            uint32_t it = 0;
            bool ok = true;
            for (int id = pair; id < total && ok; id += npairs) {
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    if (!wait_bar(&ctrl->gfull[s], (it / kStages) & 1, abort, p.err)) {
                        ok = false;
                        break;
                    }
                    // the rows sit in this CTA's shared memory: the fence makes the
                    // cp.async writes visible to the async proxy that the MMAs read
                    // them through, and the MMAs are issued only after this arrival.
                    // (A release arrive stalls the relay ~1 us per K block, which
                    // measured 1.6x slower on the whole kernel.)
                    fence_proxy_async();
                    mbar_arrive_remote_relaxed(mapa_shared(&ctrl->full[s], 0));   // the even CTA's full[s]
                }
            }
        }
    } else if (warp < kEpiWarps) {
        if (MODE == GATEUP && p.zero) {
            const int64_t n4 = p.zero_floats / 4;
            const int64_t per = (n4 + gridDim.x - 1) / gridDim.x;
            const int64_t b = (int64_t)blockIdx.x * per, e = min(n4, b + per);
            float4 *z = reinterpret_cast<float4 *>(p.zero);
            for (int64_t i = b + threadIdx.x; i < e; i += kEpiWarps * 32) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        uint32_t tc = 0;
        const int row = (warp & 3) * 32 + lane;   // TMEM lane quarter warp % 4
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        // this warp's part of the output columns of one accumulator (half)
        constexpr int kParts = kEpiWarps / 4, kPartCols = (MODE == GATEUP ? BN / 2 : BN) / kParts;
        const int c_lo = (warp >> 2) * kPartCols;
        const uint32_t tempty_lead = mapa_shared(&ctrl->tempty[0], 0);
        bool ok = true;
        for (int id = pair; id < total && ok; id += npairs, ++tc) {
            const Tile tl = decode_n(id, n_tiles, p.n_groups, ctrl->n_mtiles, tile_start, nE);
            const int64_t r = (int64_t)seg_off[tl.e] + (int64_t)tl.m * BM2 + row_off + row;
#pragma unroll 1
            for (int j = 0; j < W; ++j) {
                // W = 1: accumulator tc % 2; W = 2: half j of the one accumulator
                const uint32_t b = W == 1 ? (tc & 1) : (uint32_t)j;
                const uint32_t ph = W == 1 ? ((tc >> 1) & 1) : (tc & 1);
                ck_a.start();
                const bool ready = wait_bar(&ctrl->tfull[b], ph, abort, p.err);
                ck_a.stop();
                if (!ready) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                ck_b.start();
                epilogue_row<MODE, T, BN>(p, tl.n * W + j, r, r < seg_end[tl.e], tmem + b * BN + lane_base,
                                          reinterpret_cast<float *>(sEpi + warp * kEpiStageBytes), c_lo,
                                          c_lo + kPartCols);
                ck_b.stop();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (lead) mbar_arrive(&ctrl->tempty[b]);
                    else mbar_arrive_remote(tempty_lead + b * (uint32_t)sizeof(uint64_t));
                }
            }
        }
        if (threadIdx.x == 0) {
            ck_a.flush(FWD2_SLOT(kPtVar, 4));
            ck_b.flush(FWD2_SLOT(kPtVar, 5));
        }
    } else if (GATHER && warp >= kGatherWarp0) {
        PipeClock ck_g;
        gather_rows<T, kStages, BM2, kGatherThreads>(p, threadIdx.x - kGatherWarp0 * 32, pair, npairs, total, n_tiles, tile_start,
                                     seg_off, seg_end, nE, nk, row_off, sA, lead ? ctrl->full : ctrl->gfull,
                                     ctrl->empty, abort, &ck_g);
        if (threadIdx.x == kGatherWarp0 * 32) ck_g.flush(FWD2_SLOT(kPtVar, 7));
    }

    // every MMA of the pair has completed (its arrivals on this CTA's barriers
    // included) before the pair meets for the last time and frees TMEM
    if (threadIdx.x == 0) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(&ctrl->done, 0) && globaltimer() - t0 < kWaitLimitNs) {
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc2(tmem, kTmemCols);
    ck_total.stop();
    if (threadIdx.x == 0) {
        ck_total.flush(FWD2_SLOT(kPtVar, 0));
#ifdef MOE_PIPE_TRACE
        atomicAdd(&g_fwd2_trace[kPtVar][6], 1ull);
#endif
    }
}

}  // namespace

// ------------------------------------------------------------------ host side

template <int MODE, bool GATHER, typename T, int BN, int W>
cudaError_t launch_pair_t(const GemmLaunch &L, cudaStream_t s) {
    const GemmParams &p = L.p;
    constexpr int BN_OUT = MODE == GATEUP ? W * BN / 2 : BN;
    constexpr int kStages = pair_stages(W * BN);
    const bool f32 = sizeof(T) == 4;
    CUtensorMap mA, mB0, mB1;
    const int nE = p.offsets ? p.E : 1;
    // B boxes hold this CTA's half of the tile's weight rows
    if (!make_map(&mB0, L.b0, f32, (uint64_t)nE * p.N, p.K, W * BN / 2)) return cudaErrorInvalidValue;
    if (MODE == GATEUP) {
        if (!make_map(&mB1, L.b1, f32, (uint64_t)nE * p.N, p.K, W * BN / 2)) return cudaErrorInvalidValue;
    } else {
        mB1 = mB0;
    }
    if (!GATHER) {
        if (!make_map(&mA, L.a_src, f32, (uint64_t)p.rows, p.K, kHalfRows)) return cudaErrorInvalidValue;
    } else {
        mA = mB0;   // unused: gather mode reads x with cp.async
    }
    const size_t smem = 1024 + (size_t)kStages * (kABytes + W * BN * 64) + (MODE == DOWN ? 4 * kEpiStageBytes : 0) +
                        sizeof(Ctrl2) + 3 * sizeof(int) * (p.E + 1);
    auto kern = grouped_gemm_pair_kernel<MODE, GATHER, T, BN, W>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // as many CTA pairs as can be resident at once (one CTA per SM), capped by
    // the tile count
    static std::mutex mu;
    static int max_pairs[8] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 8) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!max_pairs[dev]) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(2 * (unsigned)(num_sms() / 2));
            cfg.blockDim = dim3(pair_threads<MODE, GATHER>());
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n = 0;
            e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
            if (e != cudaSuccess) return e;
            max_pairs[dev] = n > 0 ? n : 1;
        }
    }
    const int n_tiles = (p.N + BN_OUT - 1) / BN_OUT;
    const int64_t max_tiles = (p.rows / BM2 + nE) * (int64_t)n_tiles;
    const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(max_pairs[dev], max_tiles));
    return launch_kernel_pair(kern, 2 * pairs, pair_threads<MODE, GATHER>(), smem, s, mA, mB0, mB1, p);
}

template <int MODE, bool GATHER, typename T>
cudaError_t launch_pair_bn(const GemmLaunch &L, cudaStream_t s) {
    if (L.narrow) return launch_pair_t<MODE, GATHER, T, 128, 1>(L, s);
#ifndef MOE_GG_WIDE
#define MOE_GG_WIDE 1
#endif
    if constexpr (MODE == GATEUP && GATHER && MOE_GG_WIDE)
        if (L.p.N >= 256) return launch_pair_t<MODE, GATHER, T, 256, 2>(L, s);
    return launch_pair_t<MODE, GATHER, T, 256, 1>(L, s);
}

}  // namespace gg

cudaError_t launch_grouped_gemm_pair(const GemmLaunch &L, cudaStream_t s) {
    const GemmParams &p = L.p;
    if (p.rows <= 0) return cudaSuccess;
    const bool f32 = L.dtype == MOE_F32;
    if (L.mode == gg::GATEUP) {
        if (L.gather)
            return f32 ? gg::launch_pair_bn<gg::GATEUP, true, float>(L, s)
                       : gg::launch_pair_bn<gg::GATEUP, true, __nv_bfloat16>(L, s);
        return f32 ? gg::launch_pair_bn<gg::GATEUP, false, float>(L, s)
                   : gg::launch_pair_bn<gg::GATEUP, false, __nv_bfloat16>(L, s);
    }
    return f32 ? gg::launch_pair_bn<gg::DOWN, false, float>(L, s)
               : gg::launch_pair_bn<gg::DOWN, false, __nv_bfloat16>(L, s);
}

}  // namespace moe

#ifdef MOE_PIPE_TRACE
// Diagnostic build only: copies the two-SM forward pipeline trace (4 x 8
// counters, see above) to host memory and optionally clears it.
extern "C" int moe_debug_fwd2_trace(unsigned long long *out, int reset) {
    if (cudaDeviceSynchronize() != cudaSuccess) return 1;
    if (cudaMemcpyFromSymbol(out, moe::gg::g_fwd2_trace, sizeof(moe::gg::g_fwd2_trace)) != cudaSuccess) return 1;
    if (reset) {
        static const unsigned long long zero[4][8] = {};
        if (cudaMemcpyToSymbol(moe::gg::g_fwd2_trace, zero, sizeof(zero)) != cudaSuccess) return 1;
    }
    return 0;
}
#endif
