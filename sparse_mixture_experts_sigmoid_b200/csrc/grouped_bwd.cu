// Backward grouped GEMMs of the MoE layer on the 5th-generation tensor cores
// (tcgen05, TMEM accumulators, TMA), bf16 operands, fp32 accumulation.
//
// The layer's backward (chain rule through the forward's steps; "Small models,
// sparse experts", "Dispatch decides everything" trains this layer and quotes
// training tokens/s; "Small MoE Architecture, in depth", SmallMoE):
//
//   r_i  = W_down[e]^T dy_t                      (ROWS, SWIGLU epilogue)
//          dgate_i += r_i . a_i,  da = g_i r_i,  du = da v silu'(u),
//          dv = da silu(u),  ga_i = g_i a_i       (a = silu(u) v from the kept u, v)
//   dx_t += W_gate[e]^T du_i + W_up[e]^T dv_i    (ROWS, SCATTER epilogue)
//   dW_down[e] = sum_i dy_t (x) ga_i             (WGRAD)
//   dW_gate[e] = sum_i du_i (x) x_t, dW_up[e] = sum_i dv_i (x) x_t   (WGRAD)
//
// and the same for the shared expert (one dense segment, gate sigmoid(w_s.x))
// and for the router (dx += dl W_router, dW_router = dl^T x).
//
// Every operand comes by TMA.  The routed rows live in a padded grouped
// layout: expert e's rows start at row 64 * (sum over e' < e of
// ceil(count_e' / 64)), and the rows from the end of its segment to the next
// multiple of 64 are zero (x and dy are copied into that layout by the
// backward's first kernel; du | dv and gate * a are written into it by the
// SWIGLU epilogue).  So a weight-gradient tile reads whole 64-row K blocks of
// both operands and the rows past a segment's end add nothing.
//
// Two tile schemes share one persistent kernel (one CTA per SM; epilogue
// warps first -- eight, two per TMEM lane quarter, or four for the scatter
// epilogue -- then the TMA producer warp and the TMEM allocator + MMA issuer
// warp), and a two-SM variant of it (see bwd_gemm_pair_kernel):
//  * ROWS: tiles of 128 grouped rows x 256 output columns, K over the
//    weight's reduction dimension in blocks of 64, split into up to two K
//    ranges (the gate half and the up half of [du | dv]).  A is K-major; B is
//    a weight read MN-major (its rows are the K index, contiguous along N),
//    one 3D TMA box of 64-column atoms per K block.
//  * WGRAD: tiles of 128 weight rows x 256 weight columns of one expert, K
//    over that expert's (padded) rows in blocks of 64.  Both operands are
//    MN-major: each row contributes one 128-byte k-row per 64 columns.  An
//    expert without rows writes a zero gradient.
// MN-major shared-memory operands use the canonical 128-byte-swizzled layout:
// 64-element atoms along M/N 8 KB apart (leading offset), 8-row k groups
// 1 KB apart (stride offset); a K slice of 16 advances the start by 2 KB.
// The instruction descriptor marks each operand's major-ness.
// Every mbarrier wait is bounded as in the forward kernels.
#include <algorithm>
#include <cstdlib>

#include "grouped_parts.cuh"

namespace moe {
namespace gb {

using namespace tc;
using gg::build_tiles;
using gg::decode;
using gg::Tile;

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;                    // bf16 elements per 128-byte k slice
constexpr int kAStage = BM * 128;         // 16 KB
constexpr int kBStage = BN * 128;         // 32 KB
constexpr int kStages = 4;
constexpr int kAtom = 8192;               // one MN-major atom column: 64 k-rows x 128 bytes
// Warp roles: epilogue warps first, then the TMA producer and the MMA issuer.
// The SwiGLU and weight-gradient epilogues run on eight warps (warp w drains
// TMEM lanes 32 (w mod 4) .. + 31, columns 128 (w / 4) .. + 127 of the 256),
// the scatter epilogue, which is not the bottleneck and needs 4 KB of
// staging per warp, on four.
constexpr int kScatterEpiWarps = 4;
constexpr int kTmemCols = 512;

enum { ROWS = 0, WGRAD = 1 };

// Pipeline trace of the backward kernels, compiled in only with
// -DMOE_PIPE_TRACE (a diagnostic build): per kernel variant (rows 0-2: the
// one-SM kernel's ROWS/SWIGLU, ROWS/SCATTER and WGRAD; rows 4-6: the same for
// the two-SM kernel, summed over both CTAs of a pair), SM cycles summed over CTAs for [0] the whole kernel, [1] the MMA
// issuer waiting for operands, [2] the MMA issuer waiting for a free
// accumulator, [3] the producer waiting for a free stage, [4] epilogue warp 0
// waiting for an accumulator, [5] epilogue warp 0 draining one, and [6] the
// number of CTAs.  Read with moe_debug_pipe_trace (same build only).
#ifdef MOE_PIPE_TRACE
__device__ unsigned long long g_pipe_trace[8][8];
#define PIPE_SLOT(var, slot) (&g_pipe_trace[var][slot])
#else
#define PIPE_SLOT(var, slot) nullptr
#endif
enum { EPI_SWIGLU = 0, EPI_SCATTER = 1, EPI_STORE = 2 };
template <int EPI>
constexpr int epi_warps() {
    return EPI == EPI_SCATTER ? kScatterEpiWarps : 8;
}
template <int EPI>
constexpr int kernel_threads() {
    return (epi_warps<EPI>() + 2) * 32;
}

struct Ctrl {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint32_t tmem_base;
    int abort;
    int n_mtiles;
    int pad;
};

// Shared-memory descriptor of an MN-major operand (128-byte swizzle): atoms of
// 64 elements along M/N `lbo` bytes apart, 8-row k groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_mn(const void *p, uint32_t lbo) {
    const uint32_t a = smem_u32(p);
    return (uint64_t)((a & 0x3FFFF) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor: bf16 A and B, fp32 D, M = 128, N = 256, A K-major
// (ROWS) or MN-major (WGRAD), B MN-major.
template <int MODE>
constexpr uint32_t idesc_bwd() {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(MODE == WGRAD) << 15) | (1u << 16) |
           ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

struct Params {
    GemmParams g;            // grouping (offsets, sorted_rows, E = groups, k, rows, T, err) and, for
                             // SCATTER, N = output width, y_acc, gates (nullptr: weight 1)
    bool padded;             // routed operands in the padded grouped layout (see the top of the file)
    int nranges;             // ROWS: K ranges (1 or 2)
    int Kr;                  // ROWS: K extent of each range (weight rows per group per range)
    int N;                   // output columns (ROWS) / weight columns (WGRAD)
    int M;                   // WGRAD: weight rows per group per half
    int halves;              // WGRAD: 1 or 2 (gate | up)
    // SWIGLU epilogue
    const __nv_bfloat16 *hpre;   // [rows, 2N] kept pre-activations (u | v), unpadded grouped rows
    const float *gate;           // routed: [R] by assignment; dense: [T]
    __nv_bfloat16 *dh;           // [rows (padded), 2N] out: du | dv
    __nv_bfloat16 *ga;           // [rows (padded), N] out: gate * a
    float *dgate;                // routed: [R] by assignment; dense: [T]; accumulated
    // STORE epilogue: row-major [groups * M, N] per half
    void *out0, *out1;
    bool out_f32;
    // WGRAD on one SM, fp32 output of one dense group (the router's weight
    // gradient: few output tiles, a long K): its K blocks split into ksplit
    // consecutive ranges, each range's product added into the zeroed output
    // (1: stored whole)
    int ksplit;
    // the MN-major operands (B; A too in WGRAD) come through 3D tensor maps
    // {64 columns, rows, 64-column blocks}: one TMA instruction fetches all
    // of a stage's 64-column atoms of an operand
    bool mn3d;
};

// ------------------------------------------------------------------ epilogues

using gg::kXBytes;
using gg::x_slot;
using gg::x_store_rows;

// x_store_rows with fp32 reductions into global memory instead of stores.
__device__ __forceinline__ void x_reduce_rows(uint8_t *buf, const uint4 (&in)[4], uint8_t *base, int64_t row0,
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
        if (i < nrows && j < nwords) {
            float *dst = reinterpret_cast<float *>(base + (row0 + i) * ld + 16 * j);
            asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};"
                         ::"l"(dst), "f"(__uint_as_float(w.x)), "f"(__uint_as_float(w.y)), "f"(__uint_as_float(w.z)),
                           "f"(__uint_as_float(w.w))
                         : "memory");
        }
    }
    __syncwarp();
}

// Shared memory of the epilogue warps: the scatter's row staging, else the
// exchange buffers (16 KB either way).
template <int EPI>
constexpr int epi_stage_bytes() {
    return EPI == EPI_SCATTER ? kScatterEpiWarps * gg::kEpiStageBytes : epi_warps<EPI>() * kXBytes;
}

// ROWS / SWIGLU: the kept pre-activations u | v of 32 columns from col0 of
// this thread's grouped row r (the row's 16-byte words; not read when ok is
// false).  In the pre-activation layout one word of the warp's 32 rows spans
// at most two 512-byte runs.
struct UV {
    uint4 u[4], v[4];
};
__device__ __forceinline__ void load_uv(const Params &p, int64_t r, bool ok, int col0, UV &b) {
    if (!ok) return;
    const uint8_t *hp = reinterpret_cast<const uint8_t *>(p.hpre);
    const int words = p.N / 4, j0 = col0 / 8;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        if (col0 + 8 * q < p.N) {
            b.u[q] = __ldg(reinterpret_cast<const uint4 *>(hp + hpre_offset(r, j0 + q, words)));
            b.v[q] = __ldg(reinterpret_cast<const uint4 *>(hp + hpre_offset(r, p.N / 8 + j0 + q, words)));
        }
    }
}

// ROWS / SWIGLU epilogue of column tile nt for the warp's grouped rows r0 ..
// r0 + 31 (the first nrows valid; this thread's row is r0 + lane, gidx its
// assignment, or token for the dense expert, -1 if not valid; g its gate);
// D = r_i from TMEM.  The outputs go to rows ro0 .. (r in the padded
// layout).  buf holds the first 32 columns' u | v already (loaded before the
// accumulator was ready); once a chunk's outputs are computed the next
// chunk's loads are issued into buf, so they are in flight while the chunk is
// stored.  With two warps per row each adds its partial dot product into the
// row's gate gradient.  This warp drains NC columns from column c0 of the
// tile (tbase points at column c0); xb is its exchange buffer.
template <int NC>
__device__ __forceinline__ void epilogue_swiglu(const Params &p, int nt, int c0, int64_t r0, int64_t ro0, int nrows,
                                                int64_t gidx, float g, uint32_t tbase, UV &buf, uint8_t *xb) {
    const int N = p.N;
    const int lane = threadIdx.x & 31;
    float dot = 0.f;
#pragma unroll 1
    for (int ci = 0; ci < NC / 32; ++ci) {
        const int col0 = nt * BN + c0 + 32 * ci;
        float v[2][16];
        tmem_ld16(tbase + 32 * ci, v[0]);
        tmem_ld16(tbase + 32 * ci + 16, v[1]);
        tmem_wait_ld();
        const uint4 *ur = buf.u, *vr = buf.v;
        uint4 dur[4], dvr[4], gar[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const __nv_bfloat162 *u2 = reinterpret_cast<const __nv_bfloat162 *>(&ur[q]);
            const __nv_bfloat162 *w2 = reinterpret_cast<const __nv_bfloat162 *>(&vr[q]);
            uint32_t *du2 = reinterpret_cast<uint32_t *>(&dur[q]), *dv2 = reinterpret_cast<uint32_t *>(&dvr[q]),
                     *ga2 = reinterpret_cast<uint32_t *>(&gar[q]);
            const bool in = col0 + 8 * q < N;
#pragma unroll
            for (int z2 = 0; z2 < 4; ++z2) {
                const float2 uf = __bfloat1622float2(u2[z2]);
                const float2 wf = __bfloat1622float2(w2[z2]);
                const float uu[2] = {uf.x, uf.y}, ww[2] = {wf.x, wf.y};
                float du[2], dv[2], ga[2];
#pragma unroll
                for (int z = 0; z < 2; ++z) {
                    const int i = 8 * q + 2 * z2 + z;   // column within the 32-column chunk
                    const float rv = v[i >> 4][i & 15];
                    const float sg = __fdividef(1.f, 1.f + __expf(-uu[z]));   // sigmoid(u), as the forward
                    const float su = uu[z] * sg;   // silu(u)
                    const float a = su * ww[z];
                    if (in) dot = fmaf(rv, a, dot);
                    const float da = g * rv;
                    du[z] = da * ww[z] * sg * (1.f + uu[z] * (1.f - sg));
                    dv[z] = da * su;
                    ga[z] = g * a;
                }
                __nv_bfloat162 bb;
                bb = __floats2bfloat162_rn(du[0], du[1]);
                du2[z2] = *reinterpret_cast<uint32_t *>(&bb);
                bb = __floats2bfloat162_rn(dv[0], dv[1]);
                dv2[z2] = *reinterpret_cast<uint32_t *>(&bb);
                bb = __floats2bfloat162_rn(ga[0], ga[1]);
                ga2[z2] = *reinterpret_cast<uint32_t *>(&bb);
            }
        }
        if (ci + 1 < NC / 32) {
            int64_t r = r0;
            asm volatile("" : "+l"(r));
            load_uv(p, r + lane, lane < nrows, col0 + 32, buf);
        }
        const int nw = min(4, (N - col0) / 8);
        // the row addresses are worked out afresh for each chunk rather than
        // held in registers across the loop
        int64_t ro = ro0;
        asm volatile("" : "+l"(ro));
        uint8_t *dh = reinterpret_cast<uint8_t *>(p.dh + col0);
        x_store_rows(xb, dur, dh, ro, 4 * (int64_t)N, nrows, nw);
        x_store_rows(xb, dvr, dh + 2 * (int64_t)N, ro, 4 * (int64_t)N, nrows, nw);
        x_store_rows(xb, gar, reinterpret_cast<uint8_t *>(p.ga + col0), ro, 2 * (int64_t)N, nrows, nw);
    }
    if (gidx >= 0) atomicAdd(p.dgate + gidx, dot);
}

// WGRAD / STORE: the warp's weight rows m0 .. m0 + 31 (of M, in half `half`)
// of group e, NC columns from n0 (TMEM from tbase); zero when the group had
// no rows.  xb: the warp's exchange buffer.
template <int NC>
__device__ __forceinline__ void epilogue_store(const Params &p, int e, int half, int m0, int n0, bool has_rows,
                                               uint32_t tbase, uint8_t *xb) {
    const int nrows = min(32, p.M - m0);
    if (nrows <= 0 || (p.ksplit > 1 && !has_rows)) return;   // split K: an empty range adds nothing
    const int64_t orow0 = (int64_t)e * p.M + m0;
    uint8_t *out = static_cast<uint8_t *>(half ? p.out1 : p.out0);
#pragma unroll 1
    for (int c = 0; c < NC; c += 32) {
        const int col0 = n0 + c;
        if (col0 >= p.N) break;
        float v[2][16];
        if (has_rows) {
            tmem_ld16(tbase + c, v[0]);
            tmem_ld16(tbase + c + 16, v[1]);
            tmem_wait_ld();
        } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) v[0][q] = v[1][q] = 0.f;
        }
        if (p.out_f32) {
            // two 16-column halves of 64 bytes per row
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint4 w[4];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    w[q] = make_uint4(__float_as_uint(v[h][4 * q]), __float_as_uint(v[h][4 * q + 1]),
                                      __float_as_uint(v[h][4 * q + 2]), __float_as_uint(v[h][4 * q + 3]));
                const int c16 = col0 + 16 * h;
                if (c16 >= p.N) continue;
                if (p.ksplit > 1)
                    x_reduce_rows(xb, w, out + 4 * (int64_t)c16, orow0, 4 * (int64_t)p.N, nrows, min(4, (p.N - c16) / 4));
                else
                    x_store_rows(xb, w, out + 4 * (int64_t)c16, orow0, 4 * (int64_t)p.N, nrows, min(4, (p.N - c16) / 4));
            }
        } else {
            uint4 w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t *wq = reinterpret_cast<uint32_t *>(&w[q]);
#pragma unroll
                for (int z = 0; z < 4; ++z) {
                    const int i = 8 * q + 2 * z;
                    __nv_bfloat162 b = __floats2bfloat162_rn(v[i >> 4][i & 15], v[i >> 4][(i & 15) + 1]);
                    wq[z] = *reinterpret_cast<uint32_t *>(&b);
                }
            }
            x_store_rows(xb, w, out + 2 * (int64_t)col0, orow0, 2 * (int64_t)p.N, nrows, min(4, (p.N - col0) / 8));
        }
    }
}

// ------------------------------------------------------------------ kernel

// WGRAD tile id -> (group, half, m tile, n tile); m tiles vary fastest.
struct WTile {
    int e, half, mt, nt;
};
__device__ __forceinline__ WTile wdecode(int id, int mtiles, int ntiles, int halves) {
    WTile w;
    const int per = mtiles * halves * ntiles;
    w.e = id / per;
    int rem = id - w.e * per;
    w.nt = rem / (mtiles * halves);
    rem -= w.nt * mtiles * halves;
    w.half = rem / mtiles;
    w.mt = rem - w.half * mtiles;
    return w;
}

// A tile's operand coordinates, worked out once per tile by the producer
// (the tile decode walks the tile table in shared memory, too slow to repeat
// for every K block): ROWS: the first A row and the weights' first row and
// column; WGRAD: the A map, the weight row and column of the tile and the
// expert's first K row.
struct TileAt {
    int a_row, b_row, b_col;   // ROWS
    int half, m0, n0, krow0;   // WGRAD
};

template <int MODE, int EPI>
__global__ void __launch_bounds__(kernel_threads<EPI>(), 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                    const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1, Params p) {
    constexpr uint32_t kIdesc = idesc_bwd<MODE>();
    constexpr int kEpiWarps = epi_warps<EPI>(), kTmaWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1;
    constexpr int kCols = BN / (kEpiWarps / 4);   // columns one epilogue warp drains
    constexpr int kEpiStage = epi_stage_bytes<EPI>();

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + kStages * kAStage;
    uint8_t *sEpi = sB + kStages * kBStage;
    Ctrl *ctrl = reinterpret_cast<Ctrl *>(sEpi + kEpiStage);
    int *tile_start = reinterpret_cast<int *>(ctrl + 1);
    int *seg_off = tile_start + (p.g.E + 1);
    int *seg_end = seg_off + (p.g.E + 1);
    int *blk64 = seg_end + (p.g.E + 1);   // padded layout: group e starts at row 64 * blk64[e]
    volatile int *abort = &ctrl->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ctrl->full[s], 1);
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
        prefetch_tmap(&tmA0);
        prefetch_tmap(&tmB0);
    }
    pdl_wait();
    if (warp == kTmaWarp) {
        int blocks64;
        build_tiles<64>(p.g, blk64, seg_off, seg_end, &blocks64);
        if (MODE == ROWS) build_tiles<BM>(p.g, tile_start, seg_off, seg_end, &ctrl->n_mtiles);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch_dependents();
    [[maybe_unused]] constexpr int kPtVar = MODE == WGRAD ? 2 : EPI;
    PipeClock ck_total, ck_a, ck_b;
    ck_total.start();

    const uint32_t tmem = ctrl->tmem_base;
    const int nE = p.g.offsets ? p.g.E : 1;
    const int ntiles = (p.N + BN - 1) / BN;
    const int mtiles = MODE == WGRAD ? (p.M + BM - 1) / BM : 0;
    const int wbase = nE * p.halves * mtiles * ntiles;   // WGRAD tiles per K range
    const int total = MODE == ROWS ? ctrl->n_mtiles * ntiles : wbase * p.ksplit;
    const int kpr = (p.Kr + BK - 1) / BK;   // ROWS: K blocks per range
    // first row of group e in the operands' layout
    auto op_row0 = [&](int e) -> int { return p.padded ? 64 * blk64[e] : seg_off[e]; };
    // WGRAD: tile id -> its weight tile and its K range's first K block and
    // K block count (ranges of whole 64-row blocks; a range may be empty)
    auto wtile = [&](int id, int *kb0, int *nk) -> WTile {
        const int ks = id / wbase;
        const WTile w = wdecode(id - ks * wbase, mtiles, ntiles, p.halves);
        const int blocks = (seg_end[w.e] - seg_off[w.e] + 63) / 64;
        const int per = (blocks + p.ksplit - 1) / p.ksplit;
        *kb0 = ks * per;
        *nk = max(0, min(per, blocks - *kb0));
        return w;
    };
    // K blocks of a tile
    auto tile_nk = [&](int id) -> int {
        if constexpr (MODE == ROWS) {
            return p.nranges * kpr;
        } else {
            int kb0, nk;
            wtile(id, &kb0, &nk);
            return nk;
        }
    };

    if (warp == kTmaWarp) {
        if (lane == 0) {
            // the boxes of K block kb of tile id, into stage s
            auto boxes = [&](const TileAt &t, int kb, int s) {
                uint8_t *a = sA + s * kAStage, *b = sB + s * kBStage;
                uint64_t *bar = &ctrl->full[s];
                auto box = [&](const CUtensorMap *m, uint8_t *dst, int c0, int c1) { tma_load_2d(m, dst, bar, c0, c1); };
                // an MN-major operand: `blocks` 64-column atoms from column c, k-rows from krow
                auto mn = [&](const CUtensorMap *m, uint8_t *dst, int c, int krow, int blocks) {
                    if (p.mn3d) {
                        tma_load_3d(m, dst, bar, 0, krow, c / 64);
                    } else {
                        for (int j = 0; j < blocks; ++j) box(m, dst + j * kAtom, c + 64 * j, krow);
                    }
                };
                if constexpr (MODE == ROWS) {
                    const int range = kb >= kpr, kr = kb - range * kpr;
                    box(range ? &tmA1 : &tmA0, a, kr * BK, t.a_row);
                    mn(range ? &tmB1 : &tmB0, b, t.b_col, t.b_row + kr * BK, BN / 64);
                } else {
                    const int krow = t.krow0 + kb * 64;
                    mn(t.half ? &tmA1 : &tmA0, a, t.m0, krow, BM / 64);
                    mn(&tmB0, b, t.n0, krow, BN / 64);
                }
            };
            uint32_t it = 0;
            bool ok = true;
            for (int id = blockIdx.x; id < total && ok; id += gridDim.x) {
                const int nk = tile_nk(id);
                TileAt t{};
                if constexpr (MODE == ROWS) {
                    const Tile tl = decode(id, ntiles, tile_start, nE);
                    t.a_row = op_row0(tl.e) + tl.m * BM;
                    t.b_row = tl.e * p.Kr;
                    t.b_col = tl.n * BN;
                } else {
                    int kb0, nkw;
                    const WTile w = wtile(id, &kb0, &nkw);
                    t.half = w.half;
                    t.m0 = w.mt * BM;
                    t.n0 = w.nt * BN;
                    t.krow0 = op_row0(w.e) + 64 * kb0;
                }
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    ck_a.start();
                    const bool got = wait_bar(&ctrl->empty[s], ((it / kStages) & 1) ^ 1, abort, p.g.err);
                    ck_a.stop();
                    if (!got) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&ctrl->full[s], kAStage + kBStage);
                    boxes(t, kb, s);
                }
            }
            ck_a.flush(PIPE_SLOT(kPtVar, 3));
            if (!ok) {
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
                const bool free_acc = wait_bar(&ctrl->tempty[acc], aph ^ 1, abort, p.g.err);
                ck_b.stop();
                if (!free_acc) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + acc * BN;
                const int nk = tile_nk(id);
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    ck_a.start();
                    const bool got = wait_bar(&ctrl->full[s], (it / kStages) & 1, abort, p.g.err);
                    ck_a.stop();
                    if (!got) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = MODE == ROWS ? smem_desc(sA + s * kAStage) + 2 * kk
                                                         : desc_mn(sA + s * kAStage + kk * 2048, kAtom);
                        const uint64_t bd = desc_mn(sB + s * kBStage + kk * 2048, kAtom);
                        mma<__nv_bfloat16>(d_tmem, ad, bd, kIdesc, (kb | kk) != 0);
                    }
                    mma_commit(&ctrl->empty[s]);
                }
                if (ok) mma_commit(&ctrl->tfull[acc]);
            }
            ck_a.flush(PIPE_SLOT(kPtVar, 1));
            ck_b.flush(PIPE_SLOT(kPtVar, 2));
        }
    } else if (warp < kEpiWarps) {
        uint32_t tc = 0;
        const int row = (warp & 3) * 32 + lane;
        const int c0 = (warp >> 2) * kCols;   // this warp's first column of the tile
        const uint32_t lane_base = ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)c0;
        for (int id = blockIdx.x; id < total; id += gridDim.x, ++tc) {
            const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
            if constexpr (MODE == ROWS && EPI == EPI_SWIGLU) {
                // the row's gate and first pre-activation columns are read while
                // the accumulator is still being computed
                const Tile tl = decode(id, ntiles, tile_start, nE);
                const int64_t local = (int64_t)tl.m * BM + row;
                const int64_t r = (int64_t)seg_off[tl.e] + local;
                const bool valid = r < seg_end[tl.e];
                int64_t gidx = -1;
                float g = 0.f;
                if (valid) {
                    gidx = p.g.sorted_rows ? (int64_t)p.g.sorted_rows[r] : r;
                    if (gidx < 0 || gidx >= (p.g.sorted_rows ? p.g.rows : p.g.T)) {
                        atomicOr(p.g.err, kErrInput);
                        gidx = -1;
                    } else {
                        g = p.gate[gidx];
                    }
                }
                const int64_t r0 = r - lane;   // the warp's first row
                const int64_t left = seg_end[tl.e] - r0;
                const int nrows = left <= 0 ? 0 : (left >= 32 ? 32 : (int)left);
                UV buf;
                load_uv(p, r, lane < nrows, tl.n * BN + c0, buf);
                ck_a.start();
                const bool ready = wait_bar(&ctrl->tfull[acc], aph, abort, p.g.err);
                ck_a.stop();
                if (!ready) break;
                tc_fence_after();
                ck_b.start();
                if (nrows > 0)
                    epilogue_swiglu<kCols>(p, tl.n, c0, r0, op_row0(tl.e) + local - lane, nrows, gidx, g,
                                           tmem + acc * BN + lane_base, buf, sEpi + warp * kXBytes);
                ck_b.stop();
                tc_fence_before();
                mbar_arrive(&ctrl->tempty[acc]);
                continue;
            }
            ck_a.start();
            const bool ready = wait_bar(&ctrl->tfull[acc], aph, abort, p.g.err);
            ck_a.stop();
            if (!ready) break;
            tc_fence_after();
            ck_b.start();
            const uint32_t tb = tmem + acc * BN + lane_base;
            if constexpr (MODE == ROWS) {
                const Tile tl = decode(id, ntiles, tile_start, nE);
                const int64_t local = (int64_t)tl.m * BM + row;
                const int64_t r = (int64_t)seg_off[tl.e] + local;
                const bool valid = r < seg_end[tl.e];
                if constexpr (EPI == EPI_SWIGLU) {
                    // handled above
                } else {
                    gg::epilogue_row<gg::DOWN, __nv_bfloat16, BN>(
                        p.g, tl.n, r, valid, tb, reinterpret_cast<float *>(sEpi + warp * gg::kEpiStageBytes));
                }
            } else {
                int kb0, nkw;
                const WTile w = wtile(id, &kb0, &nkw);
                epilogue_store<kCols>(p, w.e, w.half, w.mt * BM + row - lane, w.nt * BN + c0, nkw > 0, tb,
                                      sEpi + warp * kXBytes);
            }
            ck_b.stop();
            tc_fence_before();
            mbar_arrive(&ctrl->tempty[acc]);
        }
        if (threadIdx.x == 0) {
            ck_a.flush(PIPE_SLOT(kPtVar, 4));
            ck_b.flush(PIPE_SLOT(kPtVar, 5));
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
    ck_total.stop();
    if (threadIdx.x == 0) {
        ck_total.flush(PIPE_SLOT(kPtVar, 0));
#ifdef MOE_PIPE_TRACE
        atomicAdd(&g_pipe_trace[kPtVar][6], 1ull);
#endif
    }
}

// ------------------------------------------------------------------ two-SM kernel
//
// The same tile schemes with tiles doubled in M, on clusters of two CTAs
// (tcgen05.mma.cta_group::2, M = 256): each CTA stages its own 128 rows of A
// (ROWS: 128 grouped rows; WGRAD: 128 weight rows) and its own 128 of the 256
// output columns of B, so per K block a CTA moves 32 KB into shared memory
// for the MMA work that costs 48 KB on one SM, and the ring holds six K
// blocks instead of four.  The even CTA issues the MMAs; each CTA's half of D
// lands in its own TMEM and its epilogue warps drain it.  Synchronisation as
// in the forward two-SM kernel: both CTAs' loads complete on the even CTA's
// full[s]; tcgen05.commit multicasts stage releases and accumulator-ready
// signals to both; the epilogue warps of both release an accumulator on the
// even CTA's tempty; cluster barriers after set-up and before exit.
#ifndef MOE_BWD_PSTAGES
#define MOE_BWD_PSTAGES 6
#endif
constexpr int kPStages = MOE_BWD_PSTAGES;
constexpr int kPStage = 128 * 128;   // 16 KB: this CTA's A (or B) of one K block

struct Ctrl2 {
    uint64_t full[kPStages];   // even CTA: operands of a K block landed (both CTAs)
    uint64_t empty[kPStages];  // both: the MMAs of a K block are done
    uint64_t tfull[2];         // both: accumulator ready
    uint64_t tempty[2];        // even CTA: accumulator released by both CTAs' epilogue warps
    uint64_t done;             // both: all MMAs of the pair completed
    uint32_t tmem_base;
    int abort;
    int n_mtiles;
    int pad;
};

template <int MODE>
constexpr uint32_t idesc_bwd2() {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(MODE == WGRAD) << 15) | (1u << 16) |
           ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

template <int MODE, int EPI>
__global__ void __launch_bounds__(kernel_threads<EPI>(), 1)
    bwd_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                         const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                         Params p) {
    constexpr uint32_t kIdesc = idesc_bwd2<MODE>();
    constexpr int kEpiWarps = epi_warps<EPI>(), kTmaWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1;
    constexpr int kCols = BN / (kEpiWarps / 4);   // columns one epilogue warp drains
    constexpr int kEpiStage = epi_stage_bytes<EPI>();
    constexpr int BM2 = 256;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sB = smem;                          // B stages first, then A
    uint8_t *sA = smem + kPStages * kPStage;
    uint8_t *sEpi = sA + kPStages * kPStage;
    Ctrl2 *ctrl = reinterpret_cast<Ctrl2 *>(sEpi + kEpiStage);
    int *tile_start = reinterpret_cast<int *>(ctrl + 1);
    int *seg_off = tile_start + (p.g.E + 1);
    int *seg_end = seg_off + (p.g.E + 1);
    int *blk64 = seg_end + (p.g.E + 1);
    volatile int *abort = &ctrl->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool lead = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&ctrl->full[s], 1);
            mbar_init(&ctrl->empty[s], 1);
        }
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
        prefetch_tmap(&tmA0);
        prefetch_tmap(&tmB0);
    }
    pdl_wait();
    if (warp == kTmaWarp) {
        int blocks64;
        build_tiles<64>(p.g, blk64, seg_off, seg_end, &blocks64);
        if (MODE == ROWS) build_tiles<BM2>(p.g, tile_start, seg_off, seg_end, &ctrl->n_mtiles);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync_all();   // both CTAs' barriers exist before any remote arrive
    pdl_launch_dependents();
    [[maybe_unused]] constexpr int kPtVar = 4 + (MODE == WGRAD ? 2 : EPI);   // two-SM kernels: rows 4-6
    PipeClock ck_total, ck_a, ck_b;
    ck_total.start();

    const uint32_t tmem = ctrl->tmem_base;
    const int nE = p.g.offsets ? p.g.E : 1;
    const int ntiles = (p.N + BN - 1) / BN;
    const int mtiles = MODE == WGRAD ? (p.M + BM2 - 1) / BM2 : 0;
    const int total = MODE == ROWS ? ctrl->n_mtiles * ntiles : nE * p.halves * mtiles * ntiles;
    const int kpr = (p.Kr + BK - 1) / BK;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int half_off = (int)rank * 128;   // this CTA's rows of A / columns of B inside a tile
    auto op_row0 = [&](int e) -> int { return p.padded ? 64 * blk64[e] : seg_off[e]; };
    auto tile_nk = [&](int id) -> int {
        if constexpr (MODE == ROWS) {
            return p.nranges * kpr;
        } else {
            const WTile w = wdecode(id, mtiles, ntiles, p.halves);
            return (seg_end[w.e] - seg_off[w.e] + 63) / 64;
        }
    };

    if (warp == kTmaWarp) {
        if (lane == 0) {
            constexpr uint32_t kTx = 2u * 2u * kPStage;   // A and B of both CTAs
            const uint32_t full_lead = mapa_shared(&ctrl->full[0], 0);
            // this CTA's boxes of K block kb of tile id, into stage s
            auto boxes = [&](const TileAt &t, int kb, int s) {
                uint8_t *a = sA + s * kPStage, *b = sB + s * kPStage;
                const uint32_t fb = full_lead + s * (uint32_t)sizeof(uint64_t);
                auto box = [&](const CUtensorMap *m, uint8_t *dst, int c0, int c1) {
                    tma_load_2d_pair(m, dst, fb, c0, c1);
                };
                // an MN-major operand: this CTA's two 64-column atoms from column c
                auto mn = [&](const CUtensorMap *m, uint8_t *dst, int c, int krow) {
                    if (p.mn3d) {
                        tma_load_3d_pair(m, dst, fb, 0, krow, c / 64);
                    } else {
                        for (int j = 0; j < 2; ++j) box(m, dst + j * kAtom, c + 64 * j, krow);
                    }
                };
                if constexpr (MODE == ROWS) {
                    const int range = kb >= kpr, kr = kb - range * kpr;
                    box(range ? &tmA1 : &tmA0, a, kr * BK, t.a_row);
                    mn(range ? &tmB1 : &tmB0, b, t.b_col, t.b_row + kr * BK);
                } else {
                    const int krow = t.krow0 + kb * 64;
                    mn(t.half ? &tmA1 : &tmA0, a, t.m0, krow);
                    mn(&tmB0, b, t.n0, krow);
                }
            };
            uint32_t it = 0;
            bool ok = true;
            for (int id = pair; id < total && ok; id += npairs) {
                const int nk = tile_nk(id);
                TileAt t{};
                if constexpr (MODE == ROWS) {
                    const Tile tl = decode(id, ntiles, tile_start, nE);
                    t.a_row = op_row0(tl.e) + tl.m * BM2 + half_off;
                    t.b_row = tl.e * p.Kr;
                    t.b_col = tl.n * BN + half_off;
                } else {
                    const WTile w = wdecode(id, mtiles, ntiles, p.halves);
                    t.half = w.half;
                    t.m0 = w.mt * BM2 + half_off;
                    t.n0 = w.nt * BN + half_off;
                    t.krow0 = op_row0(w.e);
                }
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kPStages;
                    ck_a.start();
                    const bool free_stage = wait_bar(&ctrl->empty[s], ((it / kPStages) & 1) ^ 1, abort, p.g.err);
                    ck_a.stop();
                    if (!free_stage) {
                        ok = false;
                        break;
                    }
                    if (lead) mbar_expect_tx(&ctrl->full[s], kTx);
                    boxes(t, kb, s);
                }
            }
            if (!ok) {
                // aborting: let this CTA's copies land before it leaves
                for (uint32_t j = it > (uint32_t)kPStages ? it - kPStages : 0; j < it; ++j) {
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try_wait(&ctrl->empty[j % kPStages], (j / kPStages) & 1) &&
                           globaltimer() - t0 < 100000000ull) {
                    }
                }
            }
            ck_a.flush(PIPE_SLOT(kPtVar, 3));
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0 && lead) {
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int id = pair; id < total && ok; id += npairs, ++tc) {
                const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
                ck_b.start();
                const bool free_acc = wait_bar(&ctrl->tempty[acc], aph ^ 1, abort, p.g.err);
                ck_b.stop();
                if (!free_acc) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + acc * BN;
                const int nk = tile_nk(id);
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kPStages;
                    const uint32_t ph = (it / kPStages) & 1;
                    // the operands of both CTAs have landed (acquire at cluster scope)
                    ck_a.start();
                    bool got = mbar_try_wait_cluster(&ctrl->full[s], ph);
                    if (!got)
                        got = wait_bar(&ctrl->full[s], ph, abort, p.g.err) && mbar_try_wait_cluster(&ctrl->full[s], ph);
                    ck_a.stop();
                    if (!got) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = MODE == ROWS ? smem_desc(sA + s * kPStage) + 2 * kk
                                                         : desc_mn(sA + s * kPStage + kk * 2048, kAtom);
                        const uint64_t bd = desc_mn(sB + s * kPStage + kk * 2048, kAtom);
                        mma2<__nv_bfloat16>(d_tmem, ad, bd, kIdesc, (kb | kk) != 0);
                    }
                    mma_commit2(&ctrl->empty[s], 0x3);
                }
                if (ok) mma_commit2(&ctrl->tfull[acc], 0x3);
            }
            mma_commit2(&ctrl->done, 0x3);
            ck_a.flush(PIPE_SLOT(kPtVar, 1));
            ck_b.flush(PIPE_SLOT(kPtVar, 2));
        }
    } else if (warp < kEpiWarps) {
        uint32_t tc = 0;
        const int row = (warp & 3) * 32 + lane;
        const int c0 = (warp >> 2) * kCols;   // this warp's first column of the tile
        const uint32_t lane_base = ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)c0;
        const uint32_t tempty_lead = mapa_shared(&ctrl->tempty[0], 0);
        for (int id = pair; id < total; id += npairs, ++tc) {
            const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
            const uint32_t tb = tmem + acc * BN + lane_base;
            bool got;
            if constexpr (MODE == ROWS) {
                const Tile tl = decode(id, ntiles, tile_start, nE);
                const int64_t local = (int64_t)tl.m * BM2 + half_off + row;
                const int64_t r = (int64_t)seg_off[tl.e] + local;
                const bool valid = r < seg_end[tl.e];
                if constexpr (EPI == EPI_SWIGLU) {
                    int64_t gidx = -1;
                    float g = 0.f;
                    if (valid) {
                        gidx = p.g.sorted_rows ? (int64_t)p.g.sorted_rows[r] : r;
                        if (gidx < 0 || gidx >= (p.g.sorted_rows ? p.g.rows : p.g.T)) {
                            atomicOr(p.g.err, kErrInput);
                            gidx = -1;
                        } else {
                            g = p.gate[gidx];
                        }
                    }
                    const int64_t r0 = r - lane;   // the warp's first row
                    const int64_t left = seg_end[tl.e] - r0;
                    const int nrows = left <= 0 ? 0 : (left >= 32 ? 32 : (int)left);
                    UV buf;
                    load_uv(p, r, lane < nrows, tl.n * BN + c0, buf);
                    ck_a.start();
                    got = wait_bar(&ctrl->tfull[acc], aph, abort, p.g.err);
                    ck_a.stop();
                    if (!got) break;
                    tc_fence_after();
                    ck_b.start();
                    if (nrows > 0)
                        epilogue_swiglu<kCols>(p, tl.n, c0, r0, op_row0(tl.e) + local - lane, nrows, gidx, g, tb, buf,
                                               sEpi + warp * kXBytes);
                    ck_b.stop();
                } else {
                    ck_a.start();
                    got = wait_bar(&ctrl->tfull[acc], aph, abort, p.g.err);
                    ck_a.stop();
                    if (!got) break;
                    tc_fence_after();
                    ck_b.start();
                    gg::epilogue_row<gg::DOWN, __nv_bfloat16, BN>(
                        p.g, tl.n, r, valid, tb, reinterpret_cast<float *>(sEpi + warp * gg::kEpiStageBytes));
                    ck_b.stop();
                }
            } else {
                ck_a.start();
                got = wait_bar(&ctrl->tfull[acc], aph, abort, p.g.err);
                ck_a.stop();
                if (!got) break;
                tc_fence_after();
                const WTile w = wdecode(id, mtiles, ntiles, p.halves);
                ck_b.start();
                epilogue_store<kCols>(p, w.e, w.half, w.mt * BM2 + half_off + row - lane, w.nt * BN + c0,
                                      seg_end[w.e] > seg_off[w.e], tb, sEpi + warp * kXBytes);
                ck_b.stop();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (lead) mbar_arrive(&ctrl->tempty[acc]);
                else mbar_arrive_remote(tempty_lead + acc * (uint32_t)sizeof(uint64_t));
            }
        }
        if (threadIdx.x == 0) {
            ck_a.flush(PIPE_SLOT(kPtVar, 4));
            ck_b.flush(PIPE_SLOT(kPtVar, 5));
        }
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
        ck_total.flush(PIPE_SLOT(kPtVar, 0));
#ifdef MOE_PIPE_TRACE
        atomicAdd(&g_pipe_trace[kPtVar][6], 1ull);
#endif
    }
}

}  // namespace gb

// ------------------------------------------------------------------ host side

namespace {

// Row-major [rows, cols] bf16 tensor with a row stride of `ld` elements (a
// multiple of 8), box of box_rows x 64 columns, 128-byte swizzle, zero fill.
bool map_bf16(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows) {
    auto fn = tc::encode_fn();
    if (!fn || ld % 8 || (reinterpret_cast<uintptr_t>(base) & 15)) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same tensor viewed as {64 columns, rows, cols / 64 blocks} (block stride
// 128 bytes), box of 64 x box_rows x box_blocks: one box holds box_blocks
// 64-column atoms of box_rows rows, each atom 64 * box_rows * 2 bytes after
// the previous one in shared memory.  Needs cols % 64 == 0, so that every
// in-range coordinate is an element of the tensor.
bool map_bf16_3d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows,
                 uint32_t box_blocks) {
    auto fn = tc::encode_fn();
    if (!fn || ld % 8 || cols % 64 || (reinterpret_cast<uintptr_t>(base) & 15)) return false;
    cuuint64_t dims[3] = {64, rows, cols / 64};
    cuuint64_t strides[2] = {ld * 2, 128};
    cuuint32_t box[3] = {64, box_rows, box_blocks};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor maps of a backward GEMM: A (K-major boxes of a_box rows in ROWS, else
// MN-major) and B (MN-major), 3D for the MN-major operands when every one of
// them allows it (p.mn3d), else 2D boxes of one 64-column atom.
template <int MODE>
bool bwd_maps(const BwdOperand &a0, const BwdOperand &a1, const BwdOperand &b0, const BwdOperand &b1, uint32_t a_box,
              uint32_t mn_blocks_a, uint32_t mn_blocks_b, CUtensorMap *mA0, CUtensorMap *mA1, CUtensorMap *mB0,
              CUtensorMap *mB1, bool *mn3d) {
    const BwdOperand *ops[4] = {&a0, &a1, &b0, &b1};
    CUtensorMap *maps[4] = {mA0, mA1, mB0, mB1};
    for (int pass = 0; pass < 2; ++pass) {
        const bool three = pass == 0;
        bool ok = true;
        for (int i = 0; i < 4 && ok; ++i) {
            const BwdOperand &o = *ops[i];
            if (!o.base) {
                *maps[i] = *maps[i & 2];   // a1 / b1 absent: the first map of the pair
                continue;
            }
            const bool mn_major = i >= 2 || MODE == gb::WGRAD;
            if (!mn_major) ok = map_bf16(maps[i], o.base, o.rows, o.cols, o.ld, a_box);
            else if (three) ok = map_bf16_3d(maps[i], o.base, o.rows, o.cols, o.ld, 64, i >= 2 ? mn_blocks_b : mn_blocks_a);
            else ok = map_bf16(maps[i], o.base, o.rows, o.cols, o.ld, 64);
        }
        if (ok) {
            *mn3d = three;
            return true;
        }
    }
    return false;
}

template <int MODE, int EPI>
cudaError_t launch_bwd(const BwdOperand &a0, const BwdOperand &a1, const BwdOperand &b0, const BwdOperand &b1,
                       const gb::Params &p, cudaStream_t s) {
    using namespace gb;
    CUtensorMap mA0, mA1, mB0, mB1;
    Params q = p;
    // ROWS: A K-major boxes of 128 rows; otherwise MN-major boxes of 64 k-rows
    if (!bwd_maps<MODE>(a0, a1, b0, b1, MODE == ROWS ? BM : 64, BM / 64, BN / 64, &mA0, &mA1, &mB0, &mB1, &q.mn3d))
        return cudaErrorInvalidValue;
    const int nE = p.g.offsets ? p.g.E : 1;
    const int ntiles = (p.N + BN - 1) / BN;
    int64_t max_tiles;
    if (MODE == ROWS) max_tiles = (p.g.rows / BM + nE) * (int64_t)ntiles;
    else max_tiles = (int64_t)nE * p.halves * ((p.M + BM - 1) / BM) * ntiles * p.ksplit;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms(), max_tiles));
    const size_t smem = 1024 + (size_t)kStages * (kAStage + kBStage) +
                        epi_stage_bytes<EPI>() + sizeof(Ctrl) +
                        4 * sizeof(int) * (p.g.E + 1);
    auto kern = bwd_gemm_kernel<MODE, EPI>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(kern, grid, kernel_threads<EPI>(), smem, s, mA0, mA1, mB0, mB1, q);
}

template <int MODE, int EPI>
cudaError_t launch_bwd_pair(const BwdOperand &a0, const BwdOperand &a1, const BwdOperand &b0, const BwdOperand &b1,
                            const gb::Params &p, cudaStream_t s) {
    using namespace gb;
    CUtensorMap mA0, mA1, mB0, mB1;
    Params q = p;
    // each CTA of the pair: 128 rows of A (ROWS), two 64-column atoms of each MN-major operand
    if (!bwd_maps<MODE>(a0, a1, b0, b1, MODE == ROWS ? 128 : 64, 2, 2, &mA0, &mA1, &mB0, &mB1, &q.mn3d))
        return cudaErrorInvalidValue;
    const size_t smem = 1024 + (size_t)kPStages * 2 * kPStage + epi_stage_bytes<EPI>() +
                        sizeof(Ctrl2) + 4 * sizeof(int) * (p.g.E + 1);
    auto kern = bwd_gemm_pair_kernel<MODE, EPI>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // as many CTA pairs as can be resident at once, capped by the tile count
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (unsigned)(num_sms() / 2));
    cfg.blockDim = dim3(kernel_threads<EPI>());
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int max_pairs = 0;
    e = cudaOccupancyMaxActiveClusters(&max_pairs, kern, &cfg);
    if (e != cudaSuccess) return e;
    const int nE = p.g.offsets ? p.g.E : 1;
    const int ntiles = (p.N + BN - 1) / BN;
    int64_t max_tiles;
    if (MODE == ROWS) max_tiles = (p.g.rows / 256 + nE) * (int64_t)ntiles;
    else max_tiles = (int64_t)nE * p.halves * ((p.M + 255) / 256) * ntiles;
    const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(std::max(max_pairs, 1), max_tiles));
    return launch_kernel_pair(kern, 2 * pairs, kernel_threads<EPI>(), smem, s, mA0, mA1, mB0, mB1, q);
}

// Two-SM tiles where there is enough work for them: ROWS when the groups
// average at least 512 rows (as in the forward), WGRAD when a group's weight
// has at least 512 rows and the groups average at least 256 rows (the K
// extent of its tiles).  Measured on training steps: the two-SM weight
// gradients take olmoe_zipf's backward from 3.09 to 2.95 ms and
// mixtral_prefill's from 8.64 to 8.15 ms; on gemma_upcycle (32 rows per
// expert) they were slower (0.71 vs 0.51 ms).  MOE_BWD_PAIR=1 / 0 forces them
// on / off.
bool bwd_pair(const BwdGemm &L) {
    static const int force = [] {
        const char *v = std::getenv("MOE_BWD_PAIR");
        return v ? (v[0] == '1' ? 1 : 0) : -1;
    }();
    if (force >= 0) return force == 1;
    const int64_t groups = L.offsets ? L.groups : 1;
    if (L.kind == BwdGemm::WEIGHT) return L.M >= 512 && L.rows >= 256LL * groups;
    return L.rows >= 512LL * groups;
}

}  // namespace

cudaError_t launch_bwd_gemm(const BwdGemm &L, cudaStream_t s) {
    using namespace gb;
    Params p{};
    p.g = GemmParams{L.offsets, L.sorted_rows, L.groups, L.k, L.rows, L.T, 0, L.N, nullptr, nullptr, L.acc,
                     nullptr, L.err};
    p.padded = L.padded;
    p.nranges = L.nranges;
    p.Kr = L.Kr;
    p.N = L.N;
    p.M = L.M;
    p.halves = L.halves;
    p.hpre = static_cast<const __nv_bfloat16 *>(L.hpre);
    p.gate = L.gate;
    p.dh = static_cast<__nv_bfloat16 *>(L.dh);
    p.ga = static_cast<__nv_bfloat16 *>(L.ga);
    p.dgate = L.dgate;
    p.out0 = L.out0;
    p.out1 = L.out1;
    p.out_f32 = L.out_f32;
    p.ksplit = 1;
    if (L.rows <= 0 && L.kind != BwdGemm::WEIGHT) return cudaSuccess;
    if (bwd_pair(L)) {
        switch (L.kind) {
            case BwdGemm::SWIGLU: return launch_bwd_pair<ROWS, EPI_SWIGLU>(L.a0, L.a1, L.b0, L.b1, p, s);
            case BwdGemm::SCATTER: return launch_bwd_pair<ROWS, EPI_SCATTER>(L.a0, L.a1, L.b0, L.b1, p, s);
            default: return launch_bwd_pair<WGRAD, EPI_STORE>(L.a0, L.a1, L.b0, L.b1, p, s);
        }
    }
    if (L.kind == BwdGemm::WEIGHT && !L.offsets && L.out_f32 && L.rows > 0) {
        // one dense group with an fp32 output (the router's weight gradient:
        // E x d outputs, K = T rows): split K so that about one tile runs per
        // SM, each range adding into the zeroed output (at least 4 K blocks
        // per range)
        const int64_t tiles = (int64_t)L.halves * ((L.M + BM - 1) / BM) * ((L.N + BN - 1) / BN);
        const int64_t blocks = (L.rows + 63) / 64;
        const int64_t split = std::min<int64_t>(num_sms() / std::max<int64_t>(tiles, 1), blocks / 4);
        if (split > 1) {
            p.ksplit = (int)split;
            const size_t bytes = sizeof(float) * (size_t)L.M * (size_t)L.N;
            cudaError_t e = cudaMemsetAsync(L.out0, 0, bytes, s);
            if (e == cudaSuccess && L.halves > 1) e = cudaMemsetAsync(L.out1, 0, bytes, s);
            if (e != cudaSuccess) return e;
        }
    }
    switch (L.kind) {
        case BwdGemm::SWIGLU: return launch_bwd<ROWS, EPI_SWIGLU>(L.a0, L.a1, L.b0, L.b1, p, s);
        case BwdGemm::SCATTER: return launch_bwd<ROWS, EPI_SCATTER>(L.a0, L.a1, L.b0, L.b1, p, s);
        default: return launch_bwd<WGRAD, EPI_STORE>(L.a0, L.a1, L.b0, L.b1, p, s);
    }
}

}  // namespace moe

#ifdef MOE_PIPE_TRACE
// Diagnostic build only: copies the pipeline trace (4 x 8 counters, see
// above) to host memory and optionally clears it.
extern "C" int moe_debug_pipe_trace(unsigned long long *out, int reset) {
    if (cudaDeviceSynchronize() != cudaSuccess) return 1;
    if (cudaMemcpyFromSymbol(out, moe::gb::g_pipe_trace, sizeof(moe::gb::g_pipe_trace)) != cudaSuccess) return 1;
    if (reset) {
        static const unsigned long long zero[8][8] = {};
        if (cudaMemcpyToSymbol(moe::gb::g_pipe_trace, zero, sizeof(zero)) != cudaSuccess) return 1;
    }
    return 0;
}
#endif
