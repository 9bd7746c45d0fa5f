// Router on the tensor cores for bf16 inputs: router logits as a tcgen05 GEMM
// (128 tokens x E experts per tile, fp32 accumulators in TMEM), then softmax
// or sigmoid scoring, top-k and gates in a thread-per-token epilogue.
//
// "Tutorial 11: Mixture of Experts (MoE)", section 2 "The Router" (route_topk:
// logits = x . W_router^T, softmax over all experts, top-k by score, gather,
// optional renormalisation); "Small MoE Architecture, in depth", SmallMoE
// .forward (sigmoid scores; gates are the kept raw scores).
//
// Exactness: x and W_router are bf16, so every product is exact in fp32 and
// the logits differ from a float64 sum only by fp32 accumulation rounding
// (~1e-6 relative), far below the selection margins this library is checked
// with; the scores, selection and gates are then computed in fp32 exactly as
// in the CUDA-core router.
//
// K-split: k-block kb goes to TMEM accumulator kb % G (G up to 8, limited by
// the 512 TMEM columns) and the epilogue adds the partial logits, so no
// accumulation chain inside the tensor core is longer than ceil(d / 64 / G)
// k-blocks; this keeps the logits within ~1e-6 of a float64 sum.
//
// Layout: the B operand tile holds the router rows (rows >= E zero-filled by
// TMA) followed, when the shared expert is present, by an 8-row box whose
// first row is w_s, so the shared-gate logit is one more TMEM column.  The
// epilogue thread of token t reads its row of logits 16 columns at a time
// (tcgen05.ld 32x32b), keeps an online softmax (running max and sum) and a
// sorted register list of the k best (key, expert); a new key enters only if
// strictly larger, and experts arrive in increasing index, so equal keys keep
// the lower index first.
#include <float.h>

#include "moe_internal.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace rt {

using namespace tc;

constexpr int BM = 128;
constexpr int kEpiWarps = 4;
constexpr int kTmaWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 192;
constexpr int kABytes = BM * 128;

struct Ctrl {
    uint64_t full[8];
    uint64_t empty[8];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint32_t tmem_base;
    int abort;
};

constexpr int stages_for(int NR) {
    const int s = 196608 / (kABytes + NR * 128);
    return s > 8 ? 8 : s;
}
// K-split: k-block kb accumulates into TMEM accumulator kb % G, and the
// epilogue adds the G partial logits on the CUDA cores, which shortens every
// sequential accumulation chain inside the tensor core by a factor of G.
constexpr int ksplit_for(int NR) {
    const int g = 512 / NR;
    return g > 8 ? 8 : g;
}
constexpr uint32_t tmem_cols_for(int NR) {
    uint32_t c = 32;
    while (c < (uint32_t)(ksplit_for(NR) * NR)) c <<= 1;
    return c;
}

template <int KMAX>
__device__ __forceinline__ void topk_insert(float (&key)[KMAX], int (&id)[KMAX], float &kth, int k, float nk,
                                            int ni) {
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        const bool sw = j < k && nk > key[j];
        const float tk = key[j];
        const int ti = id[j];
        key[j] = sw ? nk : tk;
        id[j] = sw ? ni : ti;
        nk = sw ? tk : nk;
        ni = sw ? ti : ni;
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
        if (j == k - 1) kth = key[j];
}

// Sum of the ng partial accumulators (NR columns apart) for 16 columns; two
// partials are loaded per round and added to the running sum.
template <int G>
__device__ __forceinline__ void load_logits(uint32_t taddr, int ng, int NR, float (&v)[16]) {
#pragma unroll
    for (int q = 0; q < 16; ++q) v[q] = 0.f;
#pragma unroll
    for (int g = 0; g < G; g += 2) {
        if (g < ng) {
            float p0[16], p1[16];
            tmem_ld16(taddr + g * NR, p0);
            if (g + 1 < ng) tmem_ld16(taddr + (g + 1) * NR, p1);
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

template <int NR, int KMAX>
__global__ void __launch_bounds__(kThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const __grid_constant__ CUtensorMap tmS, RouterArgs a, int nrw) {
    uint32_t *err = a.err;
    constexpr int kStages = stages_for(NR);
    constexpr int kBBytes = NR * 128;
    constexpr int kStage = kABytes + kBBytes;
    constexpr uint32_t kCols = tmem_cols_for(NR);
    constexpr int G = ksplit_for(NR);
    constexpr uint32_t kIdesc = instr_desc<__nv_bfloat16>(BM, NR);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctrl *ctrl = reinterpret_cast<Ctrl *>(smem + kStages * kStage);
    volatile int *abort = &ctrl->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool shared = a.w_shared_gate != nullptr;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ctrl->full[s], 1);
            mbar_init(&ctrl->empty[s], 1);
        }
        for (int q = 0; q < 2; ++q) {
            mbar_init(&ctrl->tfull[q], 1);
            mbar_init(&ctrl->tempty[q], kEpiWarps * 32);
        }
        ctrl->abort = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) tmem_alloc(&ctrl->tmem_base, kCols);
    if (warp == kTmaWarp && lane == 0) {
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmW);
        if (shared) prefetch_tmap(&tmS);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = ctrl->tmem_base;
    const int ntiles = (int)((a.T + BM - 1) / BM);
    const int nk = (a.d + 63) / 64;

    if (warp == kTmaWarp) {
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            const uint32_t bytes = kABytes + nrw * 128 + (shared ? 8 * 128 : 0);
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    if (!wait_bar(&ctrl->empty[s], ((it / kStages) & 1) ^ 1, abort, err)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + s * kStage;
                    mbar_expect_tx(&ctrl->full[s], bytes);
                    tma_load_2d(&tmX, st, &ctrl->full[s], kb * 64, tile * BM);
                    tma_load_2d(&tmW, st + kABytes, &ctrl->full[s], kb * 64, 0);
                    if (shared) tma_load_2d(&tmS, st + kABytes + nrw * 128, &ctrl->full[s], kb * 64, 0);
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
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++tc) {
                if (!wait_bar(&ctrl->tempty[0], (tc & 1) ^ 1, abort, err)) break;
                tc_fence_after();
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    if (!wait_bar(&ctrl->full[s], (it / kStages) & 1, abort, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = smem_desc(smem + s * kStage);
                    const uint64_t bd = smem_desc(smem + s * kStage + kABytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma<__nv_bfloat16>(tmem + (kb % G) * NR, ad + 2 * kk, bd + 2 * kk, kIdesc,
                                           (kb >= G || kk > 0) ? 1u : 0u);
                    mma_commit(&ctrl->empty[s]);
                }
                if (ok) mma_commit(&ctrl->tfull[0]);
            }
        }
    } else {
        // epilogue: warps 0-3, one token row per thread
        const int row = warp * 32 + lane;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const bool sigm = a.score == MOE_SCORE_SIGMOID;
        uint32_t tc = 0;
        const int ng = nk < G ? nk : G;   // accumulators that received k-blocks
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tc) {
            if (!wait_bar(&ctrl->tfull[0], tc & 1, abort, err)) break;
            tc_fence_after();
            const uint32_t tb = tmem + lane_base;
            float m = -FLT_MAX, z = 0.f, sl = 0.f, kth = -FLT_MAX;
            float key[KMAX];
            int id[KMAX];
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                key[j] = -FLT_MAX;
                id[j] = 0;
            }
#pragma unroll 1
            for (int c = 0; c < NR; c += 16) {
                float v[16];
                load_logits<G>(tb + c, ng, NR, v);
                if (shared && c <= nrw && nrw < c + 16) {
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        if (c + q == nrw) sl = v[q];
                }
                if (c >= a.E) continue;
                float cm = -FLT_MAX;
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    if (c + q < a.E) cm = fmaxf(cm, v[q]);
                if (!sigm) {
                    if (cm > m) {
                        z *= expf(m - cm);
                        m = cm;
                    }
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        if (c + q < a.E) z += expf(v[q] - m);
                }
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    if (c + q < a.E) {
                        const float kq = sigm ? 1.f / (1.f + expf(-v[q])) : v[q];
                        if (kq > kth) topk_insert<KMAX>(key, id, kth, a.k, kq, c + q);
                    }
                }
            }
            const int64_t t = (int64_t)tile * BM + row;
            if (a.probs) {
                // second pass over the logits for the full score row (loads are warp-wide)
#pragma unroll 1
                for (int c = 0; c < NR && c < a.E; c += 16) {
                    float v[16];
                    load_logits<G>(tb + c, ng, NR, v);
                    if (t < a.T) {
#pragma unroll
                        for (int q = 0; q < 16; ++q)
                            if (c + q < a.E)
                                a.probs[t * a.E + c + q] = sigm ? 1.f / (1.f + expf(-v[q])) : expf(v[q] - m) / z;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&ctrl->tempty[0]);
            if (t < a.T) {
                float gsum = 0.f;
                float gate[KMAX];
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    gate[j] = sigm ? key[j] : expf(key[j] - m) / z;
                    if (j < a.k) gsum += gate[j];
                }
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    if (j < a.k) {
                        a.ids[t * a.k + j] = id[j];
                        a.gates[t * a.k + j] = a.norm_topk ? gate[j] / gsum : gate[j];
                    }
                }
                if (shared && a.shared_gate) a.shared_gate[t] = 1.f / (1.f + expf(-sl));
            }
            if (a.zero_rows) {
                const int64_t t0 = (int64_t)tile * BM;
                const int64_t n4 = (min(a.T, t0 + BM) - t0) * a.d / 4;
                float4 *zr = reinterpret_cast<float4 *>(a.zero_rows + t0 * a.d);
                for (int64_t i = row; i < n4; i += kEpiWarps * 32) zr[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kCols);
}

template <int NR, int KMAX>
cudaError_t launch_t(const RouterArgs &a, int nrw, cudaStream_t s) {
    CUtensorMap mX, mW, mS;
    if (!make_map(&mX, a.x, false, (uint64_t)a.T, a.d, BM)) return cudaErrorInvalidValue;
    if (!make_map(&mW, a.w_router, false, (uint64_t)a.E, a.d, nrw)) return cudaErrorInvalidValue;
    if (a.w_shared_gate) {
        if (!make_map(&mS, a.w_shared_gate, false, 1, a.d, 8)) return cudaErrorInvalidValue;
    } else {
        mS = mW;
    }
    constexpr int kStages = stages_for(NR);
    const size_t smem = 1024 + (size_t)kStages * (kABytes + NR * 128) + sizeof(Ctrl);
    auto kern = router_tc_kernel<NR, KMAX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int ntiles = (int)((a.T + BM - 1) / BM);
    const int grid = ntiles < num_sms() ? ntiles : num_sms();
    kern<<<grid, kThreads, smem, s>>>(mX, mW, mS, a, nrw);
    note_launch();
    return cudaGetLastError();
}

template <int NR>
cudaError_t launch_nr(const RouterArgs &a, int nrw, cudaStream_t s) {
    if (a.k <= 4) return launch_t<NR, 4>(a, nrw, s);
    if (a.k <= 8) return launch_t<NR, 8>(a, nrw, s);
    return launch_t<NR, 16>(a, nrw, s);
}

}  // namespace rt

bool router_tc_supported(const RouterArgs &a, int dtype) {
    const int nrw = (a.E + 7) / 8 * 8;
    return dtype == MOE_BF16 && nrw + (a.w_shared_gate ? 8 : 0) <= 256 && a.T >= 2 * rt::BM && a.k <= MOE_MAX_TOPK;
}

cudaError_t launch_router_tc(const RouterArgs &a, cudaStream_t s) {
    const int nrw = (a.E + 7) / 8 * 8;
    const int n = nrw + (a.w_shared_gate ? 8 : 0);
    if (n <= 16) return rt::launch_nr<16>(a, nrw, s);
    if (n <= 32) return rt::launch_nr<32>(a, nrw, s);
    if (n <= 64) return rt::launch_nr<64>(a, nrw, s);
    if (n <= 128) return rt::launch_nr<128>(a, nrw, s);
    return rt::launch_nr<256>(a, nrw, s);
}

}  // namespace moe
