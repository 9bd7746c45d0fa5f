// Down projection and combine of the small-batch (decode) path for bf16
// weights, with the weight rows streamed through a shared-memory ring by TMA:
//
//   y[t, n] = sum_j g[t, j] * (W_down[e_j, n] . act[inv(t*k + j)])
//
// summed in slot order j and written straight into y (no accumulator, no
// atomics).  "Tutorial 11: Mixture of Experts (MoE)", section 3, Step 3 (the
// gate-weighted sum of a token's k expert outputs); "Small MoE Architecture,
// in depth", "Why small changes the MoE trade-off" (decode reads only the
// chosen experts' weights).
//
// Decode reads every chosen weight row once, so its time is set by the bytes
// each SM keeps in flight.  A warp that streams its own row with 16-byte
// loads keeps about 2 KB in flight, and a batch-1 down projection has only
// d such rows per expert; here one producer thread per CTA keeps a 145 KB
// ring full instead (five stages; on the Mixtral decode shape four stages
// measured the same, seven 2 us slower).  A stage holds 28 weight rows x 512
// reduction elements (one 2D TMA box, 28 KB) and the 512 activations they
// meet (one bulk copy).  The first stages' weight rows are requested before
// the wait on the previous kernel (they depend only on the routing), which
// took 2.5 us off the Mixtral decode step.
// Fourteen consumer warps take two rows each: a lane reads elements
// [8 lane, 8 lane + 8) and [256 + 8 lane, 256 + 8 lane + 8) of each row (two
// conflict-free 16-byte shared loads per row) and the matching activations,
// widens the bf16 pairs to fp32 pairs and accumulates with packed fp32 FMAs.
// Work items are (token, block of 28 output rows); one CTA per SM at most.
// Rows of an item past d belong to the next expert (or TMA's zero fill) and
// are not stored; reduction elements past h are zero-filled by TMA and met by
// zeroed activations.  Every mbarrier wait is bounded.
#include <algorithm>
#include <cstdlib>

#include "moe_internal.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace tc;

constexpr int kWarps = 14;                           // consumer warps
constexpr int kRW = 2;                               // weight rows per consumer warp
constexpr int kRows = kRW * kWarps;                  // rows per work item
constexpr int kThreads = (kWarps + 1) * 32;          // + the producer warp
#ifndef MOE_DTMA_CHUNK
#define MOE_DTMA_CHUNK 512
#endif
#ifndef MOE_DTMA_RING_KB
#define MOE_DTMA_RING_KB 150
#endif
#ifndef MOE_DTMA_EARLY
#define MOE_DTMA_EARLY 1
#endif
constexpr int kChunk = MOE_DTMA_CHUNK;               // reduction elements per stage (256 or 512)
constexpr int kRowBytes = kChunk * 2;
constexpr int kHalves = kChunk / 256;                // 256-element runs a warp reads per row and stage
constexpr int kWBytes = kRows * kRowBytes;           // weight rows of a stage
constexpr int kStageBytes = kWBytes + kRowBytes;     // + one activation chunk
constexpr int kStages = (MOE_DTMA_RING_KB * 1024) / kStageBytes;
static_assert(kChunk == 256 || kChunk == 512, "a stage row is one TMA box of at most 256 words");
static_assert(kWBytes % 128 == 0 && kStageBytes % 128 == 0, "TMA destinations stay 128-byte aligned");
static_assert(kStages >= 2 && kStages <= 16, "ring depth");

struct Ctrl {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    int abort;
};

struct DownTma {
    const __nv_bfloat16 *act;   // [R, h] grouped order
    const int32_t *ids, *inv_rows;
    const float *gates;
    int64_t T;
    int d, h, E, k;
    __nv_bfloat16 *y;
};

// Packed pairs of fp32 values (sm_100's .f32x2 arithmetic: one instruction
// for two fused multiply-adds).
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2_fma(uint64_t &acc, uint64_t a, uint64_t b) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
__device__ __forceinline__ float f2_sum(uint64_t v) {
    float a, b;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
    return a + b;
}
// The two bf16 values of a 32-bit word as an fp32 pair, lower element first
// (a bf16 value is the high half of its fp32 bits).
__device__ __forceinline__ uint64_t widen(uint32_t w) {
    return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

__global__ void __launch_bounds__(kThreads, 1)
    down_tma_kernel(const __grid_constant__ CUtensorMap mw, DownTma a, uint32_t *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctrl *c = reinterpret_cast<Ctrl *>(ring + kStages * kStageBytes);
    volatile int *abort = &c->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&c->full[s], 1);
            mbar_init(&c->empty[s], kWarps);
        }
        c->abort = 0;
        fence_barrier_init();
    }
    __syncthreads();

    const int nrb = (a.d + kRows - 1) / kRows;
    const int64_t nitems = a.T * nrb;
    const int nch = (a.h + kChunk - 1) / kChunk;
    const int R = (int)(a.T * a.k);
    // slot j of token t: its expert, or -1 when the routing entry is invalid
    auto expert_of = [&](int64_t t, int j, int *r) -> int {
        const int64_t slot = t * a.k + j;
        const int e = a.ids[slot];
        *r = a.inv_rows[slot];
        return (e < 0 || e >= a.E || *r < 0 || *r >= R) ? -1 : e;
    };

    // The routing (ids, inv_rows) was written two kernels back and is complete
    // when this grid starts, act (the previous kernel's output) only after the
    // wait: the weight rows of the first kStages stages are requested before
    // it, their activation chunks after it.
    uint32_t pre = 0;
    if (warp == kWarps && lane == 0) {
        prefetch_tmap(&mw);
        if (MOE_DTMA_EARLY) {
            for (int64_t item = blockIdx.x; item < nitems && pre < (uint32_t)kStages; item += gridDim.x) {
                const int64_t t = item / nrb;
                const int nb = (int)(item - t * nrb);
                for (int j = 0; j < a.k && pre < (uint32_t)kStages; ++j) {
                    int r;
                    const int e = expert_of(t, j, &r);
                    if (e < 0) continue;
                    for (int ch = 0; ch < nch && pre < (uint32_t)kStages; ++ch, ++pre) {
                        const int k0 = ch * kChunk;
                        mbar_expect_tx(&c->full[pre], kWBytes + 2u * (uint32_t)min(kChunk, a.h - k0));
                        tma_load_2d(&mw, ring + pre * kStageBytes, &c->full[pre], k0 / 2, e * a.d + nb * kRows);
                    }
                }
            }
        }
    }
    pdl_wait();
    pdl_launch_dependents();

    if (warp == kWarps) {
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int64_t item = blockIdx.x; item < nitems && ok; item += gridDim.x) {
                const int64_t t = item / nrb;
                const int nb = (int)(item - t * nrb);
                for (int j = 0; j < a.k && ok; ++j) {
                    int r;
                    const int e = expert_of(t, j, &r);
                    if (e < 0) continue;
                    const int row0 = e * a.d + nb * kRows;
                    for (int ch = 0; ch < nch; ++ch, ++it) {
                        const int s = it % kStages;
                        uint8_t *st = ring + s * kStageBytes;
                        const int k0 = ch * kChunk;
                        const uint32_t xbytes = 2u * (uint32_t)min(kChunk, a.h - k0);
                        if (it < pre) {
                            // weights requested before the wait
                            bulk_load(st + kWBytes, a.act + (int64_t)r * a.h + k0, xbytes, &c->full[s]);
                            continue;
                        }
                        if (!wait_bar(&c->empty[s], ((it / kStages) & 1) ^ 1, abort, err)) {
                            ok = false;
                            break;
                        }
                        mbar_expect_tx(&c->full[s], kWBytes + xbytes);
                        tma_load_2d(&mw, st, &c->full[s], k0 / 2, row0);
                        bulk_load(st + kWBytes, a.act + (int64_t)r * a.h + k0, xbytes, &c->full[s]);
                    }
                }
            }
            if (!ok) {
                // let the copies already issued land before the CTA exits
                for (uint32_t j = it > (uint32_t)kStages ? it - kStages : 0; j < it; ++j) {
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try_wait(&c->full[j % kStages], (j / kStages) & 1) &&
                           globaltimer() - t0 < 100000000ull) {
                    }
                }
            }
        }
    } else {
        const int rr0 = kRW * warp;
        uint32_t it = 0;
        bool ok = true;
        for (int64_t item = blockIdx.x; item < nitems && ok; item += gridDim.x) {
            const int64_t t = item / nrb;
            const int nb = (int)(item - t * nrb);
            float acc[kRW];
#pragma unroll
            for (int q = 0; q < kRW; ++q) acc[q] = 0.f;
            for (int j = 0; j < a.k && ok; ++j) {
                int r;
                const int e = expert_of(t, j, &r);
                if (e < 0) {
                    if (warp == 0 && lane == 0) atomicOr(err, kErrInput);
                    continue;
                }
                const float g = a.gates[t * a.k + j];
                uint64_t part[kRW];
#pragma unroll
                for (int q = 0; q < kRW; ++q) part[q] = 0;
                for (int ch = 0; ch < nch; ++ch, ++it) {
                    const int s = it % kStages;
                    if (!wait_bar(&c->full[s], (it / kStages) & 1, abort, err)) {
                        ok = false;
                        break;
                    }
                    const uint8_t *st = ring + s * kStageBytes;
                    const int lim = a.h - ch * kChunk;   // elements of this chunk inside h (a multiple of 8)
                    uint4 w[kRW][kHalves], xr[kHalves];
#pragma unroll
                    for (int hf = 0; hf < kHalves; ++hf) {
                        const int el = 256 * hf + 8 * lane;
                        xr[hf] = el < lim ? *reinterpret_cast<const uint4 *>(st + kWBytes + 2 * el) : make_uint4(0, 0, 0, 0);
#pragma unroll
                        for (int q = 0; q < kRW; ++q)
                            w[q][hf] = *reinterpret_cast<const uint4 *>(st + (rr0 + q) * kRowBytes + 2 * el);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&c->empty[s]);   // the stage's values are in registers
#pragma unroll
                    for (int hf = 0; hf < kHalves; ++hf) {
                        const uint64_t x2[4] = {widen(xr[hf].x), widen(xr[hf].y), widen(xr[hf].z), widen(xr[hf].w)};
#pragma unroll
                        for (int q = 0; q < kRW; ++q) {
                            f2_fma(part[q], widen(w[q][hf].x), x2[0]);
                            f2_fma(part[q], widen(w[q][hf].y), x2[1]);
                            f2_fma(part[q], widen(w[q][hf].z), x2[2]);
                            f2_fma(part[q], widen(w[q][hf].w), x2[3]);
                        }
                    }
                }
                if (!ok) break;
#pragma unroll
                for (int q = 0; q < kRW; ++q) acc[q] = fmaf(g, f2_sum(part[q]), acc[q]);
            }
            if (!ok) break;
            const int n0 = nb * kRows + rr0;
#pragma unroll
            for (int q = 0; q < kRW; ++q) {
                const float v = warp_sum(acc[q]);
                if (lane == 0 && n0 + q < a.d) a.y[t * a.d + n0 + q] = __float2bfloat16_rn(v);
            }
        }
    }
}

// W_down [E * d, h] bf16 viewed as 32-bit words (pairs of elements), box 256
// words (one 512-element chunk) x 28 rows, no swizzle: a row's chunk is
// contiguous in the stage.  Elements past h and rows past E * d read as zero.
bool weight_map(CUtensorMap *m, const void *w, int64_t rows, int h) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)h / 2, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)h * 2};
    cuuint32_t box[2] = {kChunk / 2, kRows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(w), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// The ring kernel serves bf16 layers without a shared expert whose rows are
// 16-byte strides (h a multiple of 8) from 16-byte aligned bases;
// MOE_DOWN_TMA=0 keeps the warp-per-row kernel.
bool down_tma_supported(const DownDirectArgs &a, int dtype) {
    static const bool on = [] {
        const char *v = std::getenv("MOE_DOWN_TMA");
        return !(v && v[0] == '0');
    }();
    const uintptr_t al = reinterpret_cast<uintptr_t>(a.act) | reinterpret_cast<uintptr_t>(a.w_down);
    return on && dtype == MOE_BF16 && a.sh_down == nullptr && a.h % 8 == 0 && a.h > 0 && a.d > 0 &&
           (al & 15) == 0;
}

cudaError_t launch_down_tma(const DownDirectArgs &a, cudaStream_t s, uint32_t *err) {
    if (a.T <= 0) return cudaSuccess;
    CUtensorMap mw;
    if (!weight_map(&mw, a.w_down, (int64_t)a.E * a.d, a.h)) return cudaErrorInvalidValue;
    DownTma p{static_cast<const __nv_bfloat16 *>(a.act), a.ids, a.inv_rows, a.gates, a.T, a.d, a.h, a.E, a.k,
              static_cast<__nv_bfloat16 *>(a.y)};
    const size_t smem = 1024 + (size_t)kStages * kStageBytes + sizeof(Ctrl);
    cudaError_t e = cudaFuncSetAttribute(down_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t items = a.T * ((a.d + kRows - 1) / kRows);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(items, num_sms()));
    return launch_kernel(down_tma_kernel, grid, kThreads, smem, s, mw, p, err);
}

}  // namespace moe
