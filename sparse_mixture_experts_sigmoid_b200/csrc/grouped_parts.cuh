// Pieces shared by the one-SM and the two-SM grouped GEMM kernels: the
// epilogue of one accumulator row and the token-row gather producer.
//
//   GATEUP: act[i, n] = silu(W_gate[e, n] . a_i) * (W_up[e, n] . a_i)
//   DOWN  : y_acc[t_i, n] += g_i * (W_down[e, n] . a_i)
//           (ordered combine: slot_out[v_i, n] = g_i * (W_down[e, n] . a_i),
//            v_i the row's assignment)
//
// "Tutorial 11: Mixture of Experts (MoE)", section 3 "Expert Computation"
// (silu(gate) * up; the weighted sum back in token order).
#pragma once

#include "grouped_tiles.cuh"
#include "moe_internal.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace gg {

using namespace tc;

enum { GATEUP = 0, DOWN = 1 };

// Row exchange through shared memory.  An epilogue thread owns one row of
// the accumulator (TMEM lane = row), so a thread-per-row store makes each warp
// instruction touch 32 rows, 16 bytes each.  Instead a warp moves 64-byte
// pieces of its 32 rows through 2 KB of its own shared memory and writes
// global memory as 8 rows x 64 contiguous bytes per instruction (4 threads
// per row).  The 16-byte word j of row i sits at i * 64 + 16 * (j ^ ((i >> 1)
// & 3)), so both the row-wise and the column-wise shared accesses are free of
// bank conflicts (each group of 8 threads covers all 32 banks once).
constexpr int kXBytes = 32 * 64;   // one warp's exchange buffer

__device__ __forceinline__ uint32_t x_slot(int i, int j) { return (uint32_t)(i * 64 + ((j ^ ((i >> 1) & 3)) << 4)); }

// Row-wise -> global: in[j] is word j of row `lane`; row i = 8 t + lane / 4
// goes to base + (row0 + i) * ld (bytes) when i < nrows, word j = lane & 3
// only when j < nwords.
__device__ __forceinline__ void x_store_rows(uint8_t *buf, const uint4 (&in)[4], uint8_t *base, int64_t row0,
                                             int64_t ld, int nrows, int nwords) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < 4; ++j) *reinterpret_cast<uint4 *>(buf + x_slot(lane, j)) = in[j];
    __syncwarp();
    const int j = lane & 3;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int i = 8 * t + (lane >> 2);
        const uint4 w = *reinterpret_cast<const uint4 *>(buf + x_slot(i, j));
        if (i < nrows && j < nwords) *reinterpret_cast<uint4 *>(base + (row0 + i) * ld + 16 * j) = w;
    }
    __syncwarp();
}

// shared-memory staging of the DOWN epilogue: 32 rows x 32 fp32 per warp
constexpr int kEpiStageBytes = 32 * 32 * 4;

// Epilogue of one grouped row r (valid: r lies inside its expert's segment)
// of a tile in column tile n, whose fp32 accumulator row starts at TMEM
// address tbase (this thread's lane).  GATEUP holds BN/2 gate columns then
// BN/2 up columns and stores silu(g) * u into act; DOWN scales the BN
// columns by the row's gate and adds them into y_acc with 16-byte reductions,
// through the warp's 4 KB shared-memory staging block `stage`.  Several TMEM
// loads are in flight per wait.  Called by all 32 lanes of an epilogue warp;
// GATEUP drains only output columns c_lo .. c_hi of the tile (two warps per
// TMEM lane quarter split them).
template <int MODE, typename T, int BN>
__device__ __forceinline__ void epilogue_row(const GemmParams &p, int n, int64_t r, bool valid, uint32_t tbase,
                                             float *stage, int c_lo = 0, int c_hi = BN) {
    constexpr int BN_OUT = MODE == GATEUP ? BN / 2 : BN;
    if constexpr (MODE == GATEUP) {
        if (!__any_sync(0xffffffffu, valid)) return;   // no row of this warp lies in the segment
        T *act = static_cast<T *>(p.act);
        // silu(g) * u for 16 output columns from column c of the tile (and, in
        // training, g and u themselves into the pre-activation rows)
        auto store16 = [&](int c, const float(&g)[16], const float(&u)[16]) {
            const int col = n * BN_OUT + c;
            if (!valid || col >= p.N) return;
            T *dst = act + r * p.N + col;
            if constexpr (sizeof(T) == 2) {
                if (p.hpre) {
                    uint8_t *hp = static_cast<uint8_t *>(p.hpre);
                    const int words = p.N / 4, j0 = col / 8;
#pragma unroll
                    for (int h8 = 0; h8 < 2; ++h8) {
                        if (col + 8 * h8 >= p.N) continue;
                        uint32_t wg[4], wu[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int i0 = 8 * h8 + 2 * q;
                            __nv_bfloat162 a2 = __floats2bfloat162_rn(g[i0], g[i0 + 1]);
                            __nv_bfloat162 b2 = __floats2bfloat162_rn(u[i0], u[i0 + 1]);
                            wg[q] = *reinterpret_cast<uint32_t *>(&a2);
                            wu[q] = *reinterpret_cast<uint32_t *>(&b2);
                        }
                        *reinterpret_cast<uint4 *>(hp + hpre_offset(r, j0 + h8, words)) =
                            make_uint4(wg[0], wg[1], wg[2], wg[3]);
                        *reinterpret_cast<uint4 *>(hp + hpre_offset(r, p.N / 8 + j0 + h8, words)) =
                            make_uint4(wu[0], wu[1], wu[2], wu[3]);
                    }
                }
            }
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                if (col + 8 * h8 >= p.N) continue;
                if constexpr (sizeof(T) == 2) {
                    uint32_t w[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int i0 = 8 * h8 + 2 * q;
                        __nv_bfloat162 b2 =
                            __floats2bfloat162_rn(silu_f(g[i0]) * u[i0], silu_f(g[i0 + 1]) * u[i0 + 1]);
                        w[q] = *reinterpret_cast<uint32_t *>(&b2);
                    }
                    *reinterpret_cast<uint4 *>(dst + 8 * h8) = make_uint4(w[0], w[1], w[2], w[3]);
                } else {
                    float o[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) o[q] = silu_f(g[8 * h8 + q]) * u[8 * h8 + q];
                    float *fd = reinterpret_cast<float *>(dst + 8 * h8);
                    *reinterpret_cast<float4 *>(fd) = make_float4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<float4 *>(fd + 4) = make_float4(o[4], o[5], o[6], o[7]);
                }
            }
        };
        // 32 output columns per TMEM wait: four loads in flight at a time;
        // output columns c_lo .. c_hi of the tile (gate/up: of BN_OUT)
#pragma unroll 1
        for (int c = c_lo; c < min(BN_OUT, c_hi); c += 32) {
            float g[2][16], u[2][16];
            tmem_ld16(tbase + c, g[0]);
            tmem_ld16(tbase + c + 16, g[1]);
            tmem_ld16(tbase + BN_OUT + c, u[0]);
            tmem_ld16(tbase + BN_OUT + c + 16, u[1]);
            tmem_wait_ld();
            store16(c, g[0], u[0]);
            store16(c + 16, g[1], u[1]);
        }
    } else {
        // t: the destination row, the token (accumulated into y_acc) or, with
        // slot_out, the assignment (stored into its own slot row)
        int t = -1;
        float gate = 0.f;
        if (valid) {
            // gates == nullptr: every row is added with weight 1
            if (p.sorted_rows) {
                // range-check the assignment before deriving its token: a value in
                // (-k, 0) would otherwise truncate to token 0
                const int v = p.sorted_rows[r];
                if (v >= 0 && v < p.rows) {
                    t = p.slot_out ? v : v / p.k;
                    gate = p.gates ? p.gates[v] : 1.f;
                } else {
                    t = -2;   // reported below
                }
            } else {
                t = (int)r;
                gate = p.gates ? p.gates[r] : 1.f;
            }
            if (t < 0 || t >= (p.slot_out ? p.rows : p.T)) {
                atomicOr(p.err, kErrInput);
                t = -1;
            }
        }
        if (!__any_sync(0xffffffffu, t >= 0)) return;   // no row of this warp lies in the segment
        // The gate-scaled rows go through a 32 x 32 fp32 staging block so that
        // each reduction instruction covers four whole 128-byte row segments of
        // y_acc instead of 16 bytes in each of 32 rows: lane l reduces the
        // 16-byte chunk l % 8 of staged row 4i + l / 8 in pass i.  Chunk q of
        // row w is stored at slot q ^ (w % 8), so neither the row-wise writes
        // nor the column-wise reads hit a shared-memory bank twice per phase.
        const int lane = threadIdx.x & 31;
        const int j = lane & 7;
        int tok[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) tok[i] = __shfl_sync(0xffffffffu, t, 4 * i + (lane >> 3));
        float4 *st = reinterpret_cast<float4 *>(stage);
        // the accumulator is reduced into k times per token, by tiles far apart in
        // time: keep its lines in L2 over the streamed weights and activations
        const uint64_t acc_pol = l2_evict_last_policy();
        // 32 columns per TMEM wait: two loads in flight at a time
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
            float v[2][16];
            tmem_ld16(tbase + c, v[0]);
            tmem_ld16(tbase + c + 16, v[1]);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 8; ++q)
                st[lane * 8 + (q ^ (lane & 7))] =
                    make_float4(gate * v[q >> 2][4 * (q & 3)], gate * v[q >> 2][4 * (q & 3) + 1],
                                gate * v[q >> 2][4 * (q & 3) + 2], gate * v[q >> 2][4 * (q & 3) + 3]);
            __syncwarp();
            const int col = n * BN + c + 4 * j;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int w = 4 * i + (lane >> 3);
                const float4 val = st[w * 8 + (j ^ (w & 7))];
                if (tok[i] >= 0 && col < p.N) {
                    if (p.slot_out)
                        *reinterpret_cast<float4 *>(p.slot_out + (int64_t)tok[i] * p.N + col) = val;
                    else
                        red_add_v4_hint(p.y_acc + (int64_t)tok[i] * p.N + col, val, acc_pol);
                }
            }
            __syncwarp();
        }
    }
}

// Gather producer (NG threads, g = 0..NG-1): the token rows x[t] of the routed
// gate/up GEMM, read in place by index with 16-byte cp.async into the
// 128-byte-swizzled K-major layout the MMA descriptor reads (8 threads per
// row, NG / 8 rows per pass).  Tile id runs from `first` in steps of `stride`;
// the rows of a tile start `row_off` rows into its RB-row block.  Stage s of
// the S-deep ring is written once empty[s] shows the previous use consumed,
// and its arrival lands on full[s] when the thread's copies have (non-blocking
// cp.async.mbarrier.arrive.noinc).  The assignment ids are loaded one tile
// ahead so their loads overlap the copies.  Returns false on abort.
template <typename T, int S, int RB, int NG = 128>
__device__ bool gather_rows(const GemmParams &p, int g, int first, int stride, int total, int n_tiles,
                            const int *tile_start, const int *seg_off, const int *seg_end, int nE, int nk,
                            int row_off, uint8_t *sA, uint64_t *full, uint64_t *empty, volatile int *abort,
                            PipeClock *ck = nullptr) {
    constexpr int BK = 128 / (int)sizeof(T);
    constexpr int V = 16 / (int)sizeof(T);
    constexpr int kABytes = 128 * 128;
    constexpr int RG = NG / 8;                       // rows per pass (a multiple of 8)
    constexpr int RPT = 128 / RG;                    // rows per thread
    const int c = g & 7;                             // 16-byte chunk of the 128-byte row
    const int rg = g >> 3;                           // rows rg, rg + RG, ..., of the 128
    const int swz = (c ^ (rg & 7)) << 4;             // 128-byte swizzle: chunk ^ (row mod 8)
    const T *x = static_cast<const T *>(p.x);
    auto load_ids = [&](int id, int (&v)[RPT]) {
        if (id >= total) return;
        const Tile tl = decode(id, n_tiles, tile_start, nE);
        const int64_t row0 = (int64_t)seg_off[tl.e] + (int64_t)tl.m * RB + row_off;
        const int64_t rend = seg_end[tl.e];
#pragma unroll
        for (int q = 0; q < RPT; ++q) {
            const int64_t r = row0 + rg + RG * q;
            v[q] = r < rend ? p.sorted_rows[r] : -1;
        }
    };
    int vnext[RPT];
    load_ids(first, vnext);
    uint32_t it = 0;
    bool ok = true;
    for (int id = first; id < total && ok; id += stride) {
        int vcur[RPT];
#pragma unroll
        for (int q = 0; q < RPT; ++q) vcur[q] = vnext[q];
        load_ids(id + stride, vnext);
        const T *src[RPT];
        uint32_t okmask = 0;
#pragma unroll
        for (int q = 0; q < RPT; ++q) {
            src[q] = x;
            const int v = vcur[q];
            if (v != -1) {
                const int64_t t = v / p.k;
                if (v >= 0 && t < p.T) {
                    src[q] = x + t * p.K + c * V;
                    okmask |= 1u << q;
                } else {
                    atomicOr(p.err, kErrInput);
                }
            }
        }
        for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = it % S;
            const uint32_t ph = (it / S) & 1;
            if (ck) ck->start();
            const bool got = wait_bar(&empty[s], ph ^ 1, abort, p.err);
            if (ck) ck->stop();
            if (!got) {
                ok = false;
                break;
            }
            uint8_t *dst = sA + s * kABytes + rg * 128 + swz;
            const bool colok = kb * BK + c * V < p.K;
#pragma unroll
            for (int q = 0; q < RPT; ++q)
                if (okmask & (1u << q))
                    cp_async16(dst + q * RG * 128, colok ? (const void *)(src[q] + kb * BK) : (const void *)x,
                               colok ? 16 : 0);
            cp_async_commit();
            // the barrier receives this thread's arrival once its copies have landed
            cp_async_arrive_noinc(&full[s]);
        }
    }
    cp_async_wait<0>();
    return ok;
}

}  // namespace gg
}  // namespace moe
