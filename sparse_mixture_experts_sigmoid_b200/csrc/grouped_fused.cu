// Fused expert kernel for layers whose experts hold about one row tile each
// (T * k <= 128 * E, e.g. 2048 tokens over 256 experts, 32 rows per expert):
// the gate/up projection, SwiGLU, the down projection and the gate-weighted
// combine of one expert slice in one persistent kernel, act kept on chip.
//
//   unit (e, m, q):  rows m*128.. of expert e's segment, hidden columns
//                    q*64 .. q*64+63
//   phase 1: G|U = X_rows . [W_gate[e][q-slice]; W_up[e][q-slice]]^T   (K = d)
//            act = silu(G) * U  -> shared memory (bf16, K-major)
//   phase 2: for each 128-column chunk c of d:
//            y_acc[t_i, c-chunk] += g_i * act . W_down[e][c-chunk, q-slice]^T   (K = 64)
//
// "Tutorial 11: Mixture of Experts (MoE)", section 3 "Expert Computation"
// (grouped gate/up, silu(gate) * up, down projection, weighted sum in token
// order); "Small models, sparse experts", "Dispatch decides everything"
// (expert weights read in place, no padding of groups).
//
// In this regime every weight tile is read by one unit only, so the layer is
// a stream of its weights (2/3 gate/up, 1/3 down).  Two separate kernels each
// pay a ramp and a tail, and the down kernel re-reads act from L2 once per
// output tile; here each unit streams its gate/up slice and then the matching
// W_down slice through one ring, and act never leaves the SM.
//
// Roles: warps 0-3 epilogue (TMEM lane quarters), warp 4 TMA producer (weights,
// evict-first), warp 5 TMEM allocator + MMA issuer, warps 6-13 gather the token
// rows (cp.async into the 128-byte-swizzled K-major layout).  Rings: token rows
// (3 stages of 16 KB) and weights (7 stages of 16 KB: a gate|up K block of
// 64 + 64 rows, or a 128 x 64 W_down block).  TMEM: two gate|up accumulators
// and two down accumulators of 128 columns each.  The MMA thread runs one
// unit ahead: it issues unit i+1's gate|up before unit i's down, so while the
// epilogue turns unit i's gate|up into act the tensor core already streams the
// next unit, and act (double-buffered) never idles it.  Ordering: the down
// MMAs of unit i wait for act (an mbarrier the epilogue arrives on after
// writing it); act buffer i % 2 is rewritten for unit i+2 only after unit
// i+2's gate|up accumulator is complete, and that commit tracks every earlier
// MMA of the issuing thread, unit i's down included.  The combine
// accumulator must be zero when the kernel starts (the router clears it).
// Every mbarrier wait is bounded as in the other kernels.
#include <algorithm>

#include "grouped_parts.cuh"

namespace moe {
namespace gf {

using namespace tc;
using gg::build_tiles;
using gg::decode;
using gg::Tile;

constexpr int BM = 128;
constexpr int HQ = 64;                    // hidden columns per unit
constexpr int DC = 128;                   // output columns per down chunk
constexpr int BK = 64;
constexpr int kAStage = BM * 128;         // 16 KB of token rows per K block
constexpr int kAStages = 3;
constexpr int kBStage = 16384;            // gate|up K block (64 + 64 rows x 128 B) or W_down block (128 rows x 128 B)
constexpr int kBStages = 7;
constexpr int kActBytes = BM * 128;       // act: 128 rows x 64 hidden columns, one K block
constexpr int kEpiWarps = 4;
constexpr int kTmaWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kGatherWarp0 = 6;
constexpr int kGatherThreads = 256;
constexpr int kTmemCols = 512;
constexpr uint32_t kAcc1 = 0, kAcc2 = 256;   // TMEM: two gate|up accumulators, two down accumulators

struct Ctrl {
    uint64_t a_full[kAStages], a_empty[kAStages];
    uint64_t full[kBStages], empty[kBStages];
    uint64_t tfull1[2], tempty1[2], act_full[2];
    uint64_t tfull2[2], tempty2[2];
    uint32_t tmem_base;
    int abort;
    int n_mtiles;
    int pad;
};

__global__ void __launch_bounds__(192 + kGatherThreads, 1)
    fused_expert_kernel(const __grid_constant__ CUtensorMap tmWg, const __grid_constant__ CUtensorMap tmWu,
                        const __grid_constant__ CUtensorMap tmWd, GemmParams p, int h) {
    constexpr uint32_t kId1 = instr_desc<__nv_bfloat16>(BM, 2 * HQ);
    constexpr uint32_t kId2 = instr_desc<__nv_bfloat16>(BM, DC);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = sA + kAStages * kAStage;
    uint8_t *sAct = sB + kBStages * kBStage;   // two act buffers
    uint8_t *sEpi = sAct + 2 * kActBytes;
    Ctrl *ctrl = reinterpret_cast<Ctrl *>(sEpi + kEpiWarps * gg::kEpiStageBytes);
    int *tile_start = reinterpret_cast<int *>(ctrl + 1);
    int *seg_off = tile_start + (p.E + 1);
    int *seg_end = seg_off + (p.E + 1);
    volatile int *abort = &ctrl->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&ctrl->a_full[s], kGatherThreads);
            mbar_init(&ctrl->a_empty[s], 1);
        }
        for (int s = 0; s < kBStages; ++s) {
            mbar_init(&ctrl->full[s], 1);
            mbar_init(&ctrl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctrl->tfull1[b], 1);
            mbar_init(&ctrl->tempty1[b], kEpiWarps * 32);
            mbar_init(&ctrl->act_full[b], kEpiWarps * 32);
            mbar_init(&ctrl->tfull2[b], 1);
            mbar_init(&ctrl->tempty2[b], kEpiWarps * 32);
        }
        ctrl->abort = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) tmem_alloc(&ctrl->tmem_base, kTmemCols);
    if (warp == kTmaWarp && lane == 0) {
        prefetch_tmap(&tmWg);
        prefetch_tmap(&tmWu);
        prefetch_tmap(&tmWd);
    }
    pdl_wait();
    if (warp == kTmaWarp) build_tiles<BM>(p, tile_start, seg_off, seg_end, &ctrl->n_mtiles);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch_dependents();

    const uint32_t tmem = ctrl->tmem_base;
    const int nq = h / HQ;                       // hidden slices per expert
    const int total = ctrl->n_mtiles * nq;
    const int nk1 = (p.K + BK - 1) / BK;         // gate|up K blocks (K = d)
    const int nc = (p.N + DC - 1) / DC;          // down chunks (N = d)
    // this CTA's units: id = blockIdx.x + u * gridDim.x, u = 0 .. nu-1
    const int nu = blockIdx.x < total ? (total - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    auto unit_id = [&](int u) { return (int)blockIdx.x + u * (int)gridDim.x; };

    if (warp == kTmaWarp) {
        if (lane == 0) {
            // weight stages in the MMA thread's order: gate|up of unit u, then down of unit u-1
            const uint64_t pol = l2_evict_first_policy();
            uint32_t it = 0;
            bool ok = true;
            auto next = [&]() -> int {
                const int s = it % kBStages;
                if (!wait_bar(&ctrl->empty[s], ((it / kBStages) & 1) ^ 1, abort, p.err)) return -1;
                mbar_expect_tx(&ctrl->full[s], kBStage);
                return s;
            };
            for (int u = 0; u <= nu && ok; ++u) {
                if (u < nu) {
                    const Tile tl = decode(unit_id(u), nq, tile_start, p.E);
                    const int wrow = tl.e * h + tl.n * HQ;
                    for (int kb = 0; kb < nk1; ++kb, ++it) {
                        const int s = next();
                        if (s < 0) {
                            ok = false;
                            break;
                        }
                        tma_load_2d_hint(&tmWg, sB + s * kBStage, &ctrl->full[s], kb * BK, wrow, pol);
                        tma_load_2d_hint(&tmWu, sB + s * kBStage + kBStage / 2, &ctrl->full[s], kb * BK, wrow, pol);
                    }
                }
                if (u >= 1 && ok) {
                    const Tile tl = decode(unit_id(u - 1), nq, tile_start, p.E);
                    for (int c = 0; c < nc; ++c, ++it) {
                        const int s = next();
                        if (s < 0) {
                            ok = false;
                            break;
                        }
                        tma_load_2d_hint(&tmWd, sB + s * kBStage, &ctrl->full[s], tl.n * HQ, tl.e * p.N + c * DC, pol);
                    }
                }
            }
            if (!ok) {
                for (uint32_t j = it > kBStages ? it - kBStages : 0; j < it; ++j) {
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try_wait(&ctrl->full[j % kBStages], (j / kBStages) & 1) &&
                           globaltimer() - t0 < 100000000ull) {
                    }
                }
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            uint32_t it = 0, ia = 0, cc = 0;
            bool ok = true;
            for (int u = 0; u <= nu && ok; ++u) {
                if (u < nu) {
                    // gate|up of unit u into acc1[u % 2]
                    const uint32_t b = u & 1;
                    if (!wait_bar(&ctrl->tempty1[b], ((u >> 1) & 1) ^ 1, abort, p.err)) break;
                    tc_fence_after();
                    for (int kb = 0; kb < nk1; ++kb, ++it, ++ia) {
                        const int s = it % kBStages, sa = ia % kAStages;
                        if (!wait_bar(&ctrl->a_full[sa], (ia / kAStages) & 1, abort, p.err) ||
                            !wait_bar(&ctrl->full[s], (it / kBStages) & 1, abort, p.err)) {
                            ok = false;
                            break;
                        }
                        fence_proxy_async();   // gathered rows were written by cp.async
                        tc_fence_after();
                        const uint64_t ad = smem_desc(sA + sa * kAStage);
                        const uint64_t bd = smem_desc(sB + s * kBStage);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma<__nv_bfloat16>(tmem + kAcc1 + b * 2 * HQ, ad + 2 * kk, bd + 2 * kk, kId1, (kb | kk) != 0);
                        mma_commit(&ctrl->a_empty[sa]);
                        mma_commit(&ctrl->empty[s]);
                    }
                    if (!ok) break;
                    mma_commit(&ctrl->tfull1[b]);
                }
                if (u >= 1) {
                    // down of unit u-1: act buffer (u-1) % 2 times its W_down chunks
                    const uint32_t ab = (u - 1) & 1;
                    if (!wait_bar(&ctrl->act_full[ab], ((u - 1) >> 1) & 1, abort, p.err)) break;
                    tc_fence_after();
                    const uint64_t ad = smem_desc(sAct + ab * kActBytes);
                    for (int c = 0; c < nc; ++c, ++it, ++cc) {
                        const uint32_t b = cc & 1;
                        const int s = it % kBStages;
                        if (!wait_bar(&ctrl->tempty2[b], ((cc >> 1) & 1) ^ 1, abort, p.err) ||
                            !wait_bar(&ctrl->full[s], (it / kBStages) & 1, abort, p.err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t bd = smem_desc(sB + s * kBStage);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma<__nv_bfloat16>(tmem + kAcc2 + b * DC, ad + 2 * kk, bd + 2 * kk, kId2, kk != 0);
                        mma_commit(&ctrl->empty[s]);
                        mma_commit(&ctrl->tfull2[b]);
                    }
                }
            }
        }
    } else if (warp < kEpiWarps) {
        const int row = warp * 32 + lane;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        uint32_t cc = 0;
        bool ok = true;
        for (int u = 0; u <= nu && ok; ++u) {
            if (u < nu) {
                // epilogue 1 of unit u: act = silu(gate) * up -> act buffer u % 2
                const uint32_t b = u & 1;
                const Tile tl = decode(unit_id(u), nq, tile_start, p.E);
                const int64_t r = (int64_t)seg_off[tl.e] + (int64_t)tl.m * BM + row;
                const bool valid = r < seg_end[tl.e];
                if (!wait_bar(&ctrl->tfull1[b], (u >> 1) & 1, abort, p.err)) break;
                tc_fence_after();
                uint8_t *blk = sAct + b * kActBytes + row * 128;
#pragma unroll 1
                for (int c = 0; c < HQ; c += 32) {
                    float g[2][16], v[2][16];
                    const uint32_t ta = tmem + kAcc1 + b * 2 * HQ + lane_base;
                    tmem_ld16(ta + c, g[0]);
                    tmem_ld16(ta + c + 16, g[1]);
                    tmem_ld16(ta + HQ + c, v[0]);
                    tmem_ld16(ta + HQ + c + 16, v[1]);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t w[4];
#pragma unroll
                        for (int z = 0; z < 4; ++z) {
                            const int i = 8 * q + 2 * z;
                            const float a0 = valid ? silu_f(g[i >> 4][i & 15]) * v[i >> 4][i & 15] : 0.f;
                            const float a1 = valid ? silu_f(g[(i + 1) >> 4][(i + 1) & 15]) * v[(i + 1) >> 4][(i + 1) & 15]
                                                   : 0.f;
                            __nv_bfloat162 b2 = __floats2bfloat162_rn(a0, a1);
                            w[z] = *reinterpret_cast<uint32_t *>(&b2);
                        }
                        const int chunk = (c >> 3) + q;
                        *reinterpret_cast<uint4 *>(blk + ((chunk ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
                fence_proxy_async();   // act is read by the tensor core (async proxy)
                tc_fence_before();
                mbar_arrive(&ctrl->act_full[b]);
                mbar_arrive(&ctrl->tempty1[b]);
            }
            if (u >= 1) {
                // epilogue 2 of unit u-1: each down chunk, gate-scaled, into the combine accumulator
                const Tile tl = decode(unit_id(u - 1), nq, tile_start, p.E);
                const int64_t r = (int64_t)seg_off[tl.e] + (int64_t)tl.m * BM + row;
                const bool valid = r < seg_end[tl.e];
                for (int c = 0; c < nc; ++c, ++cc) {
                    const uint32_t b = cc & 1;
                    if (!wait_bar(&ctrl->tfull2[b], (cc >> 1) & 1, abort, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    gg::epilogue_row<gg::DOWN, __nv_bfloat16, DC>(p, c, r, valid, tmem + kAcc2 + b * DC + lane_base,
                                                                  reinterpret_cast<float *>(sEpi + warp * gg::kEpiStageBytes));
                    tc_fence_before();
                    mbar_arrive(&ctrl->tempty2[b]);
                }
            }
        }
    } else if (warp >= kGatherWarp0) {
        // the token rows of each unit's gate|up (K = d), one A stage per K block
        gg::gather_rows<__nv_bfloat16, kAStages, BM, kGatherThreads>(p, threadIdx.x - kGatherWarp0 * 32, blockIdx.x,
                                                                     gridDim.x, total, nq, tile_start, seg_off,
                                                                     seg_end, p.E, nk1, 0, sA, ctrl->a_full,
                                                                     ctrl->a_empty, abort);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace gf

bool fused_expert_supported(const moe_config &c) {
    return c.dtype == MOE_BF16 && c.h % gf::HQ == 0 && (int64_t)c.T * c.k <= 128LL * c.E;
}

// x [T, d]; weights [E, h, d] (gate, up) and [E, d, h] (down); offsets/sorted_rows
// of the grouping; y_acc [T, d] fp32 (zero on entry).
cudaError_t launch_fused_expert(const moe_config &c, const void *x, const void *wg, const void *wu, const void *wd,
                                const int32_t *offsets, const int32_t *srt, const float *gates, float *y_acc,
                                uint32_t *err, cudaStream_t s) {
    using namespace gf;
    CUtensorMap mg, mu, md;
    if (!make_map(&mg, wg, false, (uint64_t)c.E * c.h, c.d, HQ)) return cudaErrorInvalidValue;
    if (!make_map(&mu, wu, false, (uint64_t)c.E * c.h, c.d, HQ)) return cudaErrorInvalidValue;
    if (!make_map(&md, wd, false, (uint64_t)c.E * c.d, c.h, DC)) return cudaErrorInvalidValue;
    GemmParams p{offsets, srt, c.E, c.k, c.T * c.k, c.T, c.d, c.d, x, nullptr, y_acc, gates, err};
    const int nq = c.h / HQ;
    const int64_t max_units = ((int64_t)c.T * c.k / BM + c.E) * nq;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms(), max_units));
    const size_t smem = 1024 + (size_t)kAStages * kAStage + (size_t)kBStages * kBStage + 2 * kActBytes +
                        kEpiWarps * gg::kEpiStageBytes + sizeof(Ctrl) + 3 * sizeof(int) * (c.E + 1);
    cudaError_t e = cudaFuncSetAttribute(fused_expert_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(fused_expert_kernel, grid, 192 + kGatherThreads, smem, s, mg, mu, md, p, c.h);
}

}  // namespace moe
