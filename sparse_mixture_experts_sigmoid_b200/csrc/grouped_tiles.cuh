// Device-side tile list of the grouped GEMMs: per-expert row-block counts and
// their prefix sum, built from the expert offsets by one warp, and the mapping
// of a tile id to (expert, column block, row block).  Tiles are expert-major;
// inside an expert the row blocks vary fastest, so CTAs running at the same
// time share one weight tile through L2.
#pragma once

#include "moe_internal.cuh"

namespace moe {
namespace gg {

// One warp: per-expert counts of RB-row blocks and their prefix sum
// (tile_start), the validated segment bounds (seg_off, seg_end), and the total
// (n_mtiles).  Lane l owns the C = ceil(E / 32) consecutive experts starting
// at l * C, so all offsets are read with one round of independent loads.
// Offsets outside [0, rows] or decreasing are reported and treated as empty
// segments.
template <int RB>
__device__ void build_tiles(const GemmParams &p, int *tile_start, int *seg_off, int *seg_end, int *n_mtiles) {
    const int lane = threadIdx.x & 31;
    if (p.offsets == nullptr) {
        if (lane == 0) {
            seg_off[0] = 0;
            seg_end[0] = (int)p.rows;
            tile_start[0] = 0;
            tile_start[1] = (int)((p.rows + RB - 1) / RB);
            *n_mtiles = tile_start[1];
        }
        return;
    }
    constexpr int kMaxC = (MOE_MAX_EXPERTS + 31) / 32;
    const int C = (p.E + 31) / 32;
    const int e0 = lane * C;
    int o[kMaxC + 1];
#pragma unroll
    for (int j = 0; j <= kMaxC; ++j)
        if (j <= C && e0 + j <= p.E) o[j] = p.offsets[e0 + j];
    int mt[kMaxC];
    int sum = 0;
    bool bad = false;
#pragma unroll
    for (int j = 0; j < kMaxC; ++j) {
        mt[j] = 0;
        if (j < C && e0 + j < p.E) {
            int b = o[j], en = o[j + 1];
            if (b < 0 || en < b || en > p.rows) {
                bad = true;
                en = b = 0;
            }
            seg_off[e0 + j] = b;
            seg_end[e0 + j] = en;
            mt[j] = (en - b + RB - 1) / RB;
            sum += mt[j];
        }
    }
    int incl = sum;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
    }
    int run = incl - sum;
#pragma unroll
    for (int j = 0; j < kMaxC; ++j)
        if (j < C && e0 + j < p.E) {
            tile_start[e0 + j] = run;
            run += mt[j];
        }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.err, kErrInput);
    if (lane == 31) {
        tile_start[p.E] = incl;
        *n_mtiles = incl;
    }
}

struct Tile {
    int e, m, n;
};

__device__ __forceinline__ Tile decode(int id, int n_tiles, const int *tile_start, int E) {
    const int q = id / n_tiles;
    int lo = 0, hi = E;  // first j in [0, E] with tile_start[j] > q, minus one
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tile_start[mid] <= q) lo = mid;
        else hi = mid - 1;
    }
    // lo = the last index with tile_start[lo] <= q; a run of empty experts shares
    // its start with the next non-empty one, so lo lands on the expert owning q
    Tile t;
    t.e = lo;
    const int mt = tile_start[lo + 1] - tile_start[lo];
    const int local = id - tile_start[lo] * n_tiles;
    t.n = local / mt;
    t.m = local - t.n * mt;
    return t;
}

// The same tiles with the column tiles split into G consecutive groups that
// run one after another: all tiles of columns [0, gs) (expert-major as in
// decode), then all of [gs, 2 gs), ... (gs = ceil(n_tiles / G)).  For the down
// GEMM this bounds the part of the combine accumulator that the CTAs running
// at one time reduce into (T x gs columns), so it stays in L2 across the k
// experts of a token; each row of act is then read once per group.  G <= 1 is
// decode.
__device__ __forceinline__ Tile decode_n(int id, int n_tiles, int G, int n_mtiles, const int *tile_start, int E) {
    if (G <= 1) return decode(id, n_tiles, tile_start, E);
    const int gs = (n_tiles + G - 1) / G;
    const int per = n_mtiles * gs;
    const int g = id / per;
    const int gsz = min(gs, n_tiles - g * gs);
    Tile t = decode(id - g * per, gsz, tile_start, E);
    t.n += g * gs;
    return t;
}

}  // namespace gg
}  // namespace moe
