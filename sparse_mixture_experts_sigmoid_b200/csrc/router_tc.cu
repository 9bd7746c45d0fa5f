// Router for bf16 batches, in two kernels:
//
//  1. router_logits_kernel: the router logits l = x . W_router^T (plus the
//     shared-expert gate logit w_s . x) as a tcgen05 GEMM over tiles of 128
//     tokens x 64 logit columns, fp32 accumulators in TMEM, stored as fp32
//     rows of a [T, LS] scratch matrix.
//  2. router_select_kernel: one warp per token reads its row of logits, forms
//     softmax statistics or sigmoid scores, takes the top k by k rounds of a
//     warp arg-max over (key, -index) -- equal keys go to the lower expert
//     index -- and writes ids, gates (optionally renormalised), the full score
//     row and the shared gate.
//
// "Tutorial 11: Mixture of Experts (MoE)", section 2 "The Router" (route_topk:
// logits = x . W_router^T, softmax over all experts, top-k, gather of the kept
// scores, optional renormalisation); "Small MoE Architecture, in depth",
// SmallMoE.forward (sigmoid scores; gates are the kept raw scores).
//
// Exactness: x and W_router are bf16, so every product is exact in fp32.  The
// K loop is split over 8 TMEM accumulators (k-block kb accumulates into
// kb % 8) that the epilogue adds on the CUDA cores, so no accumulation chain
// inside the tensor core is longer than ceil(d / 512) k-blocks; this keeps
// the logits within ~1e-6 of a float64 sum (a single long chain measured 4e-6
// on the gates).  Scores, selection and gates are fp32 on the CUDA cores.
//
// Logit columns: [0, E) are the router rows; when the shared expert is
// present its gate vector w_s is column nrw = E rounded up to 8 (so its 8-row
// TMA box lands on a 1024-byte swizzle atom); LS = columns rounded up to 64.
#include <float.h>

#include "moe_internal.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace rt {

using namespace tc;

constexpr int BM = 128;
constexpr int BN = 64;
constexpr int kStages = 8;
constexpr int G = 8;                      // K-split accumulators: 8 x 64 = 512 TMEM columns
constexpr int kABytes = BM * 128;         // 16 KB
constexpr int kBBytes = BN * 128;         // 8 KB
constexpr int kStage = kABytes + kBBytes;
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4, kTmaWarp = 4, kMmaWarp = 5;
constexpr uint32_t kCols = 512;

struct LogitsArgs {
    int64_t T;
    int d, E, nrw, LS;
    bool shared;
    float *logits;   // [T, LS]
    uint32_t *err;
    int32_t *hist;   // grouping histogram to clear for the selection kernel (or null)
    int64_t hist_ints;
};

struct Ctrl {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tfull, tempty;
    uint32_t tmem_base;
    int abort;
};

// Sum of the ng partial accumulators (BN columns apart) for 16 columns.
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

__global__ void __launch_bounds__(kThreads, 1)
    router_logits_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                         const __grid_constant__ CUtensorMap tmS, LogitsArgs a) {
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
        mbar_init(&ctrl->tempty, kEpiWarps * 32);
        ctrl->abort = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) tmem_alloc(&ctrl->tmem_base, kCols);
    if (warp == kTmaWarp && lane == 0) {
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmW);
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
    const int n_tiles = a.LS / BN;
    const int total = (int)((a.T + BM - 1) / BM) * n_tiles;
    const int nk = (a.d + 63) / 64;

    if (warp == kTmaWarp) {
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int id = blockIdx.x; id < total && ok; id += gridDim.x) {
                const int m = id / n_tiles, n = id - m * n_tiles;
                // 8-row boxes of the tile's logit rows: router rows below nrw, the
                // shared gate row at nrw; other rows are never read
                int nbox = 0;
                for (int j = 0; j < BN / 8; ++j) {
                    const int r = n * BN + 8 * j;
                    nbox += (r < a.nrw) || (a.shared && r == a.nrw);
                }
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    if (!wait_bar(&ctrl->empty[s], ((it / kStages) & 1) ^ 1, abort, a.err)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + s * kStage;
                    mbar_expect_tx(&ctrl->full[s], kABytes + nbox * 1024);
                    tma_load_2d(&tmX, st, &ctrl->full[s], kb * 64, m * BM);
                    for (int j = 0; j < BN / 8; ++j) {
                        const int r = n * BN + 8 * j;
                        if (r < a.nrw)
                            tma_load_2d(&tmW, st + kABytes + j * 1024, &ctrl->full[s], kb * 64, r);
                        else if (a.shared && r == a.nrw)
                            tma_load_2d(&tmS, st + kABytes + j * 1024, &ctrl->full[s], kb * 64, 0);
                    }
                }
            }
            if (!ok) {
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
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int id = blockIdx.x; id < total && ok; id += gridDim.x, ++tc) {
                if (!wait_bar(&ctrl->tempty, (tc & 1) ^ 1, abort, a.err)) break;
                tc_fence_after();
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    if (!wait_bar(&ctrl->full[s], (it / kStages) & 1, abort, a.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = smem_desc(smem + s * kStage);
                    const uint64_t bd = smem_desc(smem + s * kStage + kABytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma<__nv_bfloat16>(tmem + (kb % G) * BN, ad + 2 * kk, bd + 2 * kk, kIdesc,
                                           (kb >= G || kk > 0) ? 1u : 0u);
                    mma_commit(&ctrl->empty[s]);
                }
                if (ok) mma_commit(&ctrl->tfull);
            }
        }
    } else {
        const int row = warp * 32 + lane;
        const uint32_t tb = tmem + ((uint32_t)(warp * 32) << 16);
        const int ng = nk < G ? nk : G;
        uint32_t tc = 0;
        for (int id = blockIdx.x; id < total; id += gridDim.x, ++tc) {
            const int m = id / n_tiles, n = id - m * n_tiles;
            if (!wait_bar(&ctrl->tfull, tc & 1, abort, a.err)) break;
            tc_fence_after();
            const int64_t t = (int64_t)m * BM + row;
            float *dst = a.logits + t * a.LS + n * BN;
#pragma unroll 1
            for (int c = 0; c < BN; c += 16) {
                float v[16];
                load_logits(tb + c, ng, v);
                if (t < a.T) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<float4 *>(dst + c + 4 * q) =
                            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                }
            }
            tc_fence_before();
            mbar_arrive(&ctrl->tempty);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kCols);
}

// One warp per token: scoring, top-k and gates from a row of logits.
template <int EPL>
__global__ void __launch_bounds__(256) router_select_kernel(RouterArgs a, const float *logits, int LS, int nrw) {
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * 8 + warp;
    if (t >= a.T) return;
    const float *row = logits + t * LS;
    const bool sigm = a.score == MOE_SCORE_SIGMOID;
    float l[EPL], key[EPL];
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
        const int e = lane + 32 * q;
        l[q] = e < a.E ? row[e] : -FLT_MAX;
        key[q] = sigm ? 1.f / (1.f + expf(-l[q])) : l[q];
    }
    if (a.zero_rows) {
        float4 *z = reinterpret_cast<float4 *>(a.zero_rows + t * a.d);
        for (int i = lane; i < a.d / 4; i += 32) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
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
        if (a.hist) {
            // per-block expert histogram for the grouping step
            const int64_t r = t * a.k + lane;
            atomicAdd(a.hist + (r / a.hist_chunk) * (a.E + 1) + my_e, 1);
        }
    }
    if (a.probs) {
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            const int e = lane + 32 * q;
            if (e < a.E) a.probs[t * a.E + e] = sigm ? key[q] : expf(l[q] - m) / z;
        }
    }
    if (lane == 0 && a.shared_gate && a.w_shared_gate) a.shared_gate[t] = 1.f / (1.f + expf(-row[nrw]));
}

struct Geometry {
    int nrw, LS;
};
Geometry geometry(int E, bool shared) {
    Geometry g;
    g.nrw = (E + 7) / 8 * 8;
    g.LS = (g.nrw + (shared ? 1 : 0) + BN - 1) / BN * BN;
    return g;
}

}  // namespace rt

size_t router_tc_workspace_bytes(int64_t T, int E, bool shared) {
    return sizeof(float) * (size_t)T * rt::geometry(E, shared).LS;
}

bool router_tc_supported(int64_t T, int E, int dtype) {
    return dtype == MOE_BF16 && T >= 128 && E <= MOE_MAX_EXPERTS;
}

cudaError_t launch_router_tc(const RouterArgs &a, float *scratch, cudaStream_t s) {
    using namespace rt;
    const bool shared = a.w_shared_gate != nullptr;
    const Geometry g = geometry(a.E, shared);
    CUtensorMap mX, mW, mS;
    if (!tc::make_map(&mX, a.x, false, (uint64_t)a.T, a.d, BM)) return cudaErrorInvalidValue;
    if (!tc::make_map(&mW, a.w_router, false, (uint64_t)a.E, a.d, 8)) return cudaErrorInvalidValue;
    if (shared) {
        if (!tc::make_map(&mS, a.w_shared_gate, false, 1, a.d, 8)) return cudaErrorInvalidValue;
    } else {
        mS = mW;
    }
    const int64_t hist_ints = a.hist ? ((a.T * a.k + a.hist_chunk - 1) / a.hist_chunk) * (a.E + 1) : 0;
    LogitsArgs la{a.T, a.d, a.E, g.nrw, g.LS, shared, scratch, a.err, a.hist, hist_ints};
    const size_t smem = 1024 + (size_t)kStages * kStage + sizeof(Ctrl);
    cudaError_t e = cudaFuncSetAttribute(router_logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int total = (int)((a.T + BM - 1) / BM) * (g.LS / BN);
    const int grid = total < num_sms() ? total : num_sms();
    e = launch_kernel(router_logits_kernel, grid, kThreads, smem, s, mX, mW, mS, la);
    if (e != cudaSuccess) return e;
    const unsigned sgrid = (unsigned)((a.T + 7) / 8);
    const float *lg = scratch;
    if (a.E <= 64) return launch_kernel(router_select_kernel<2>, sgrid, 256, 0, s, a, lg, g.LS, g.nrw);
    if (a.E <= 128) return launch_kernel(router_select_kernel<4>, sgrid, 256, 0, s, a, lg, g.LS, g.nrw);
    if (a.E <= 256) return launch_kernel(router_select_kernel<8>, sgrid, 256, 0, s, a, lg, g.LS, g.nrw);
    return launch_kernel(router_select_kernel<16>, sgrid, 256, 0, s, a, lg, g.LS, g.nrw);
}

}  // namespace moe
