// 4-bit routed experts on the small-batch (decode) path, with the weights
// streamed through a shared-memory ring by TMA.
//
// Same format and arithmetic as segment_q4.cu ("Small MoE Architecture, in
// depth": "Worked example: the batch-1 budget on a device" and "Running
// experts that do not fit: offloading and quantisation"): groups of 64 codes
// along the reduction dimension with one fp32 scale, nibble n standing for
// (n - 8) * s, dequantised in the dot products as (128 + n) with 136 * sum(x)
// subtracted once per activation chunk.
//
// Decode reads every chosen weight once, so the kernels are bound by how many
// bytes each SM keeps in flight.  Loading the codes into registers ties that
// to the register file (the warps that fit and the loads each can have
// outstanding); here one producer thread per CTA streams the codes and scales
// of 28 weight rows x 1024 reduction elements per stage (14 KB of codes per
// matrix), with the activation chunks they meet (contiguous bulk copies),
// into a ~180 KB ring, and fourteen consumer warps read them from shared
// memory, two rows per warp, each lane 32 codes of a row per stage (one
// 16-byte shared load).  The activation chunk a lane needs (32 values) is
// read once per stage and shared by its rows.
//
//   q4t_gateup_kernel: work items (expert pass, block of 28 hidden rows); a
//     pass holds up to two of the expert's grouped rows, whose activations
//     meet the staged gate and up codes; act = silu(gate) * up in bf16.
//   q4t_down_kernel: work items (token, block of 28 output rows); the stages
//     walk the k chosen experts' W_down rows in slot order, so
//     y = sum_j g_j (W_down[e_j] . act_j) is summed in a fixed order, plus the
//     shared expert's row (computed beforehand in fp32) when there is one.
// Every mbarrier wait is bounded (error flag, then the CTA leaves).
#include <algorithm>
#include <mutex>

#include "segment_parts.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace tc;

#ifndef MOE_Q4_WARPS
#define MOE_Q4_WARPS 14
#endif
constexpr int kQWarps = MOE_Q4_WARPS;                  // consumer warps
static_assert(kQWarps == 8 || kQWarps == 14 || kQWarps == 16, "consumer warps per CTA");
constexpr int kQThreads = (kQWarps + 1) * 32;          // + the producer warp
constexpr int kQRW = 2;                                // weight rows per consumer warp
// weight rows per work item: 28 makes the Mixtral shapes' item counts fit
// the 148 SMs (1024 gate/up items, 6.9 per SM; 147 down items) where 32
// left a seventh gate/up item on 8 SMs and 20 SMs without a down item; the
// last item of a matrix may be partial (its extra rows are computed from
// the next rows or TMA's zero fill, and not stored)
constexpr int kQRows = kQRW * kQWarps;
constexpr int kQChunk = 1024;                          // reduction elements per stage
constexpr int kQCodeBytes = kQRows * kQChunk / 2;      // codes per matrix (14 KB for 28 rows)
constexpr int kQScaleBytes = kQRows * (kQChunk / 64) * 4;   // scales per matrix
static_assert(kQCodeBytes % 128 == 0 && kQScaleBytes % 128 == 0, "TMA destinations stay 128-byte aligned");
constexpr int kQRing = 180 * 1024;                     // shared-memory ring
constexpr int kQTok = 2;                               // grouped rows per gate/up pass
constexpr int kQMaxPasses = 64;                        // at most kDecodeMaxRows rows

constexpr int kQActBytes = kQChunk * 2;                // one activation row chunk (bf16)

// A stage: the codes of each matrix, their scales, then NACT activation row
// chunks (gate/up: the pass's token rows; down: the expert's act row).
template <int NMAT>
constexpr int q_nact() {
    return NMAT == 2 ? kQTok : 1;
}
template <int NMAT>
constexpr int q_stage_bytes() {
    return NMAT * (kQCodeBytes + kQScaleBytes) + q_nact<NMAT>() * kQActBytes;
}
template <int NMAT>
constexpr int q_stages() {
    return kQRing / q_stage_bytes<NMAT>();
}

static_assert(q_stages<1>() <= 12 && q_stages<2>() <= 12, "ring stages fit the barrier arrays");
struct QCtrl {
    uint64_t full[12];
    uint64_t empty[12];
    int abort;
    int n_pass;
    int pe[kQMaxPasses], pb[kQMaxPasses], pn[kQMaxPasses];   // pass: expert, first grouped row, rows
};

// Packed pairs of fp32 values (the .f32x2 arithmetic of sm_100: one
// instruction for two fused multiply-adds).
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2_fma(uint64_t &acc, uint64_t a, uint64_t b) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
__device__ __forceinline__ void f2_add(uint64_t &acc, uint64_t a) {
    asm("add.rn.f32x2 %0, %0, %1;" : "+l"(acc) : "l"(a));
}
__device__ __forceinline__ float f2_sum(uint64_t v) {
    float a, b;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
    return a + b;
}

// 32 consecutive bf16 activations of a staged chunk in shared memory, from
// element idx, as 16 packed pairs (elements 2i, 2i + 1), and their sum (zero
// past `limit`, where the copy stopped).  A bf16 value is the high half of
// its fp32 bits.  Each lane converts its own chunk: one conversion shared by
// the warps needs a barrier per stage, which measured 2x slower.
__device__ __forceinline__ float load32_smem(const uint8_t *chunk, int idx, int limit, uint64_t (&x2)[16]) {
    uint64_t s2 = 0;
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
        uint4 raw = make_uint4(0, 0, 0, 0);
        if (8 * wd < limit) raw = *reinterpret_cast<const uint4 *>(chunk + 2 * (idx + 8 * wd));
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            x2[4 * wd + j] = f2_pack(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xFFFF0000u));
            f2_add(s2, x2[4 * wd + j]);
        }
    }
    return f2_sum(s2);
}

// The float 128 + n for the nibble in byte b of `nibbles` (0x43, the nibble
// byte, two zero bytes).
__device__ __forceinline__ float q_nib(uint32_t nibbles, int b) {
    return __uint_as_float(__byte_perm(nibbles, 0x43000000u, 0x7044u | ((uint32_t)b << 8)));
}
// sum_i (128 + n_i) x_i over the 32 codes of one 16-byte word group: the low
// nibble of byte b of a word is element 2b of its eight, the high nibble
// element 2b + 1, so each byte meets one packed activation pair.
__device__ __forceinline__ float q_dot32(const uint4 &qw, const uint64_t (&x2)[16]) {
    const uint32_t words[4] = {qw.x, qw.y, qw.z, qw.w};
    uint64_t a0 = 0, a1 = 0;
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
        const uint32_t lo = words[wd] & 0x0F0F0F0Fu, hi = (words[wd] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int b = 0; b < 4; ++b) f2_fma(b & 1 ? a1 : a0, f2_pack(q_nib(lo, b), q_nib(hi, b)), x2[4 * wd + b]);
    }
    f2_add(a0, a1);
    return f2_sum(a0);
}

// Warp 0 lists the gate/up passes: each expert's grouped rows in runs of at
// most kQTok, in expert order.  Offsets outside [0, rows] are reported.
__device__ void q_build_passes(const Segments &sg, QCtrl *c, uint32_t *err) {
    const int lane = threadIdx.x & 31;
    int n = 0;
    for (int base = 0; base < sg.E; base += 32) {
        const int e = base + lane;
        int b = 0, cnt = 0;
        if (e < sg.E) {
            b = sg.offsets[e];
            const int en = sg.offsets[e + 1];
            if (b < 0 || en < b || en > sg.rows) {
                atomicOr(err, kErrInput);
            } else {
                cnt = en - b;
            }
        }
        const int np = (cnt + kQTok - 1) / kQTok;
        int incl = np;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += v;
        }
        for (int q = 0; q < np; ++q) {
            const int idx = n + incl - np + q;
            if (idx < kQMaxPasses) {
                c->pe[idx] = e;
                c->pb[idx] = b + q * kQTok;
                c->pn[idx] = min(kQTok, cnt - q * kQTok);
            }
        }
        n += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) c->n_pass = min(n, kQMaxPasses);
}

struct Q4GateUpTma {
    const __nv_bfloat16 *x;
    Segments seg;
    int64_t T;
    int d, hid;
    __nv_bfloat16 *act;
};

// Offsets of the activation chunks in a gate/up and a down stage.
constexpr int kQXOff2 = 2 * (kQCodeBytes + kQScaleBytes);
constexpr int kQXOff1 = kQCodeBytes + kQScaleBytes;

// The tokens of pass ps (-1: no row, or an assignment out of range, which is
// reported when err is given).
__device__ __forceinline__ void q_pass_tokens(const Q4GateUpTma &a, const QCtrl *c, int ps, int64_t (&tok)[kQTok],
                                              uint32_t *err) {
#pragma unroll
    for (int b = 0; b < kQTok; ++b) {
        tok[b] = -1;
        if (b < c->pn[ps]) {
            const int v = a.seg.sorted_rows[c->pb[ps] + b];
            const int64_t t = (v >= 0 && v < a.seg.rows) ? v / a.seg.k : -1;
            if (t < 0 || t >= a.T) {
                if (err) atomicOr(err, kErrInput);
            } else {
                tok[b] = t;
            }
        }
    }
}

// Ring position it of this CTA: stage it % S, phase (it / S) & 1.
__global__ void __launch_bounds__(kQThreads, 1)
    q4t_gateup_kernel(const __grid_constant__ CUtensorMap mqg, const __grid_constant__ CUtensorMap mqu,
                      const __grid_constant__ CUtensorMap msg, const __grid_constant__ CUtensorMap msu,
                      Q4GateUpTma a, uint32_t *err) {
    constexpr int S = q_stages<2>();
    constexpr int SB = q_stage_bytes<2>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    QCtrl *c = reinterpret_cast<QCtrl *>(ring + S * SB);
    volatile int *abort = &c->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&c->full[s], 1);
            mbar_init(&c->empty[s], kQWarps);
        }
        c->abort = 0;
        fence_barrier_init();
    }
    if (warp == kQWarps && lane == 0) {
        prefetch_tmap(&mqg);
        prefetch_tmap(&mqu);
        prefetch_tmap(&msg);
        prefetch_tmap(&msu);
    }
    pdl_wait();
    if (warp == 0) q_build_passes(a.seg, c, err);
    __syncthreads();
    pdl_launch_dependents();

    const int nrb = (a.hid + kQRows - 1) / kQRows;
    const int nitems = c->n_pass * nrb;
    const int nch = (a.d + kQChunk - 1) / kQChunk;

    if (warp == kQWarps) {
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < nitems && ok; item += gridDim.x) {
                const int ps = item / nrb, rb = item - ps * nrb;
                const int row0 = c->pe[ps] * a.hid + rb * kQRows;
                int64_t tok[kQTok];
                q_pass_tokens(a, c, ps, tok, nullptr);
                for (int ch = 0; ch < nch; ++ch, ++it) {
                    const int s = it % S;
                    if (!wait_bar(&c->empty[s], ((it / S) & 1) ^ 1, abort, err)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = ring + s * SB;
                    const int k0 = ch * kQChunk;
                    const uint32_t xbytes = 2u * (uint32_t)min(kQChunk, a.d - k0);
                    uint32_t tx = 2 * (kQCodeBytes + kQScaleBytes);
#pragma unroll
                    for (int b = 0; b < kQTok; ++b) tx += tok[b] >= 0 ? xbytes : 0;
                    mbar_expect_tx(&c->full[s], tx);
                    tma_load_2d(&mqg, st, &c->full[s], ch * (kQChunk / 8), row0);
                    tma_load_2d(&mqu, st + kQCodeBytes, &c->full[s], ch * (kQChunk / 8), row0);
                    tma_load_2d(&msg, st + 2 * kQCodeBytes, &c->full[s], ch * (kQChunk / 64), row0);
                    tma_load_2d(&msu, st + 2 * kQCodeBytes + kQScaleBytes, &c->full[s], ch * (kQChunk / 64), row0);
#pragma unroll
                    for (int b = 0; b < kQTok; ++b)
                        if (tok[b] >= 0)
                            bulk_load(st + kQXOff2 + b * kQActBytes, a.x + tok[b] * a.d + k0, xbytes, &c->full[s]);
                }
            }
            if (!ok) {
                // aborting: let the copies already issued land before the CTA exits
                for (uint32_t j = it > (uint32_t)S ? it - S : 0; j < it; ++j) {
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try_wait(&c->full[j % S], (j / S) & 1) && globaltimer() - t0 < 100000000ull) {
                    }
                }
            }
        }
    } else {
        uint32_t it = 0;
        for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
            const int ps = item / nrb, rb = item - ps * nrb;
            int64_t tok[kQTok];
            q_pass_tokens(a, c, ps, tok, warp == 0 && lane == 0 ? err : nullptr);
            float ag[kQTok][kQRW], au[kQTok][kQRW];
#pragma unroll
            for (int b = 0; b < kQTok; ++b)
#pragma unroll
                for (int q = 0; q < kQRW; ++q) ag[b][q] = au[b][q] = 0.f;
            bool ok = true;
            for (int ch = 0; ch < nch; ++ch, ++it) {
                const int s = it % S;
                if (!wait_bar(&c->full[s], (it / S) & 1, abort, err)) {
                    ok = false;
                    break;
                }
                const uint8_t *st = ring + s * SB;
                const int k0 = ch * kQChunk + 32 * lane;   // this lane's first reduction index
                uint4 wg[kQRW], wu[kQRW];
                float sg[kQRW], su[kQRW];
#pragma unroll
                for (int q = 0; q < kQRW; ++q) {
                    const int r = kQRW * warp + q;
                    wg[q] = *reinterpret_cast<const uint4 *>(st + r * (kQChunk / 2) + 16 * lane);
                    wu[q] = *reinterpret_cast<const uint4 *>(st + kQCodeBytes + r * (kQChunk / 2) + 16 * lane);
                    sg[q] = reinterpret_cast<const float *>(st + 2 * kQCodeBytes)[r * (kQChunk / 64) + lane / 2];
                    su[q] = reinterpret_cast<const float *>(st + 2 * kQCodeBytes + kQScaleBytes)[r * (kQChunk / 64) + lane / 2];
                }
#pragma unroll
                for (int b = 0; b < kQTok; ++b) {
                    if (tok[b] < 0) continue;
                    uint64_t xv[16];
                    const float xs = 136.f * load32_smem(st + kQXOff2 + b * kQActBytes, 32 * lane, a.d - k0, xv);
#pragma unroll
                    for (int q = 0; q < kQRW; ++q) {
                        ag[b][q] = fmaf(sg[q], q_dot32(wg[q], xv) - xs, ag[b][q]);
                        au[b][q] = fmaf(su[q], q_dot32(wu[q], xv) - xs, au[b][q]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&c->empty[s]);   // this warp is done with the stage
            }
            if (!ok) break;
            const int n0 = rb * kQRows + kQRW * warp;
#pragma unroll
            for (int b = 0; b < kQTok; ++b) {
#pragma unroll
                for (int q = 0; q < kQRW; ++q) {
                    const float g = warp_sum(ag[b][q]);
                    const float u = warp_sum(au[b][q]);
                    if (lane == 0 && tok[b] >= 0 && n0 + q < a.hid)
                        a.act[(int64_t)(c->pb[ps] + b) * a.hid + n0 + q] = __float2bfloat16_rn(silu_f(g) * u);
                }
            }
        }
    }
}

struct Q4DownTma {
    const __nv_bfloat16 *act;   // [R, h] grouped order
    const int32_t *ids, *inv_rows;
    const float *gates;
    const float *shared_add;    // [T, d] fp32 shared-expert rows, or null
    int64_t T;
    int d, h, E, k;
    __nv_bfloat16 *y;
};

__global__ void __launch_bounds__(kQThreads, 1)
    q4t_down_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap ms, Q4DownTma a,
                    uint32_t *err) {
    constexpr int S = q_stages<1>();
    constexpr int SB = q_stage_bytes<1>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    QCtrl *c = reinterpret_cast<QCtrl *>(ring + S * SB);
    volatile int *abort = &c->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&c->full[s], 1);
            mbar_init(&c->empty[s], kQWarps);
        }
        c->abort = 0;
        fence_barrier_init();
    }
    __syncthreads();

    const int nrb = (a.d + kQRows - 1) / kQRows;
    const int64_t nitems = a.T * nrb;
    const int nch = (a.h + kQChunk - 1) / kQChunk;
    const int R = (int)(a.T * a.k);
    // slot j of token t: its expert, or -1 when the routing entry is invalid
    auto expert_of = [&](int64_t t, int j, int *r) -> int {
        const int64_t slot = t * a.k + j;
        const int e = a.ids[slot];
        *r = a.inv_rows[slot];
        return (e < 0 || e >= a.E || *r < 0 || *r >= R) ? -1 : e;
    };

    // The routing was written two or more kernels back and is complete when
    // this grid starts; act (the gate/up output) and the shared expert's rows
    // only after the wait.  The codes and scales of the first S stages are
    // requested before it, their activation chunks after it.
    uint32_t pre = 0;
    if (warp == kQWarps && lane == 0) {
        prefetch_tmap(&mq);
        prefetch_tmap(&ms);
        for (int64_t item = blockIdx.x; item < nitems && pre < (uint32_t)S; item += gridDim.x) {
            const int64_t t = item / nrb;
            const int nb = (int)(item - t * nrb);
            for (int j = 0; j < a.k && pre < (uint32_t)S; ++j) {
                int r;
                const int e = expert_of(t, j, &r);
                if (e < 0) continue;
                for (int ch = 0; ch < nch && pre < (uint32_t)S; ++ch, ++pre) {
                    uint8_t *st = ring + pre * SB;
                    mbar_expect_tx(&c->full[pre],
                                   kQCodeBytes + kQScaleBytes + 2u * (uint32_t)min(kQChunk, a.h - ch * kQChunk));
                    tma_load_2d(&mq, st, &c->full[pre], ch * (kQChunk / 8), e * a.d + nb * kQRows);
                    tma_load_2d(&ms, st + kQCodeBytes, &c->full[pre], ch * (kQChunk / 64), e * a.d + nb * kQRows);
                }
            }
        }
    }
    pdl_wait();
    pdl_launch_dependents();

    if (warp == kQWarps) {
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
                    const int row0 = e * a.d + nb * kQRows;
                    for (int ch = 0; ch < nch; ++ch, ++it) {
                        const int s = it % S;
                        uint8_t *st = ring + s * SB;
                        const int k0 = ch * kQChunk;
                        const uint32_t xbytes = 2u * (uint32_t)min(kQChunk, a.h - k0);
                        if (it < pre) {
                            // codes and scales requested before the wait
                            bulk_load(st + kQXOff1, a.act + (int64_t)r * a.h + k0, xbytes, &c->full[s]);
                            continue;
                        }
                        if (!wait_bar(&c->empty[s], ((it / S) & 1) ^ 1, abort, err)) {
                            ok = false;
                            break;
                        }
                        mbar_expect_tx(&c->full[s], kQCodeBytes + kQScaleBytes + xbytes);
                        tma_load_2d(&mq, st, &c->full[s], ch * (kQChunk / 8), row0);
                        tma_load_2d(&ms, st + kQCodeBytes, &c->full[s], ch * (kQChunk / 64), row0);
                        bulk_load(st + kQXOff1, a.act + (int64_t)r * a.h + k0, xbytes, &c->full[s]);
                    }
                }
            }
            if (!ok) {
                for (uint32_t j = it > (uint32_t)S ? it - S : 0; j < it; ++j) {
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try_wait(&c->full[j % S], (j / S) & 1) && globaltimer() - t0 < 100000000ull) {
                    }
                }
            }
        }
    } else {
        uint32_t it = 0;
        bool ok = true;
        for (int64_t item = blockIdx.x; item < nitems && ok; item += gridDim.x) {
            const int64_t t = item / nrb;
            const int nb = (int)(item - t * nrb);
            float acc[kQRW];
#pragma unroll
            for (int q = 0; q < kQRW; ++q) acc[q] = 0.f;
            for (int j = 0; j < a.k && ok; ++j) {
                int r;
                const int e = expert_of(t, j, &r);
                if (e < 0) {
                    if (warp == 0 && lane == 0) atomicOr(err, kErrInput);
                    continue;
                }
                const float g = a.gates[t * a.k + j];
                float part[kQRW];
#pragma unroll
                for (int q = 0; q < kQRW; ++q) part[q] = 0.f;
                for (int ch = 0; ch < nch; ++ch, ++it) {
                    const int s = it % S;
                    if (!wait_bar(&c->full[s], (it / S) & 1, abort, err)) {
                        ok = false;
                        break;
                    }
                    const uint8_t *st = ring + s * SB;
                    const int k0 = ch * kQChunk + 32 * lane;
                    uint4 w[kQRW];
                    float sc[kQRW];
#pragma unroll
                    for (int q = 0; q < kQRW; ++q) {
                        const int rr = kQRW * warp + q;
                        w[q] = *reinterpret_cast<const uint4 *>(st + rr * (kQChunk / 2) + 16 * lane);
                        sc[q] = reinterpret_cast<const float *>(st + kQCodeBytes)[rr * (kQChunk / 64) + lane / 2];
                    }
                    uint64_t xv[16];
                    const float xs = 136.f * load32_smem(st + kQXOff1, 32 * lane, a.h - k0, xv);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&c->empty[s]);   // codes, scales and act are in registers
#pragma unroll
                    for (int q = 0; q < kQRW; ++q) part[q] = fmaf(sc[q], q_dot32(w[q], xv) - xs, part[q]);
                }
#pragma unroll
                for (int q = 0; q < kQRW; ++q) acc[q] = fmaf(g, part[q], acc[q]);
            }
            if (!ok) break;
            const int n0 = nb * kQRows + kQRW * warp;
#pragma unroll
            for (int q = 0; q < kQRW; ++q) {
                float v = warp_sum(acc[q]);
                if (lane == 0 && n0 + q < a.d) {
                    if (a.shared_add) v += a.shared_add[t * a.d + n0 + q];
                    a.y[t * a.d + n0 + q] = __float2bfloat16_rn(v);
                }
            }
        }
    }
}

// Codes [rows, K / 2] bytes as 32-bit words, box 128 words x 32 rows; scales
// [rows, K / 64] fp32, box 16 x 32.  No swizzle: a row's bytes are contiguous
// in the stage.
bool q_maps(CUtensorMap *mq, CUtensorMap *ms, const uint8_t *q, const float *s, int64_t rows, int K) {
    auto fn = encode_fn();
    if (!fn) return false;
    {
        cuuint64_t dims[2] = {(cuuint64_t)K / 8, (cuuint64_t)rows};
        cuuint64_t strides[1] = {(cuuint64_t)K / 2};
        cuuint32_t box[2] = {kQChunk / 8, kQRows};
        cuuint32_t estr[2] = {1, 1};
        if (fn(mq, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint8_t *>(q), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    cuuint64_t dims[2] = {(cuuint64_t)K / 64, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K / 64 * 4};
    cuuint32_t box[2] = {kQChunk / 64, kQRows};
    cuuint32_t estr[2] = {1, 1};
    return fn(ms, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(s), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NMAT>
size_t q_smem() {
    return 1024 + (size_t)q_stages<NMAT>() * q_stage_bytes<NMAT>() + sizeof(QCtrl);
}

// Persistent grid: one CTA per SM at most, no more than the items.
int q_grid(int64_t items) { return (int)std::max<int64_t>(1, std::min<int64_t>(items, num_sms())); }

}  // namespace

bool q4_tma_supported(int d, int h, const void *x, const void *q_gate, const float *s_gate, const void *q_up, const float *s_up,
                      const void *q_down, const float *s_down) {
    // rows of scales must be 16-byte strides (K / 64 a multiple of 4) and
    // every base 16-byte aligned
    const uintptr_t al = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(q_gate) |
                         reinterpret_cast<uintptr_t>(s_gate) |
                         reinterpret_cast<uintptr_t>(q_up) | reinterpret_cast<uintptr_t>(s_up) |
                         reinterpret_cast<uintptr_t>(q_down) | reinterpret_cast<uintptr_t>(s_down);
    return d % 256 == 0 && h % 256 == 0 && (al & 15) == 0;
}

cudaError_t launch_q4t_gateup(const SegGateUpQ4Args &a, cudaStream_t s) {
    if (a.seg.rows <= 0) return cudaSuccess;
    CUtensorMap mqg, mqu, msg, msu;
    const int64_t rows = (int64_t)a.seg.E * a.hid;
    if (!q_maps(&mqg, &msg, a.q_gate, a.s_gate, rows, a.d) || !q_maps(&mqu, &msu, a.q_up, a.s_up, rows, a.d))
        return cudaErrorInvalidValue;
    Q4GateUpTma p{static_cast<const __nv_bfloat16 *>(a.x), a.seg, a.T, a.d, a.hid,
                  static_cast<__nv_bfloat16 *>(a.act)};
    const size_t smem = q_smem<2>();
    cudaError_t e = cudaFuncSetAttribute(q4t_gateup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // passes are at most the grouped rows; items = passes x row blocks
    const int64_t items = std::min<int64_t>(a.seg.rows, kQMaxPasses) * ((a.hid + kQRows - 1) / kQRows);
    return launch_kernel(q4t_gateup_kernel, q_grid(items), kQThreads, smem, s, mqg, mqu, msg, msu, p,
                         device_error_word());
}

cudaError_t launch_q4t_down(const DownDirectQ4Args &a, const float *shared_add, cudaStream_t s) {
    if (a.T <= 0) return cudaSuccess;
    CUtensorMap mq, ms;
    if (!q_maps(&mq, &ms, a.q_down, a.s_down, (int64_t)a.E * a.d, a.h)) return cudaErrorInvalidValue;
    Q4DownTma p{static_cast<const __nv_bfloat16 *>(a.act), a.ids, a.inv_rows, a.gates, shared_add, a.T, a.d, a.h,
                a.E, a.k, static_cast<__nv_bfloat16 *>(a.y)};
    const size_t smem = q_smem<1>();
    cudaError_t e = cudaFuncSetAttribute(q4t_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(q4t_down_kernel, q_grid(a.T * ((a.d + kQRows - 1) / kQRows)), kQThreads, smem, s, mq, ms, p,
                         device_error_word());
}

}  // namespace moe
