// C ABI of libmoe.so: argument validation, workspace layout and the launch
// sequence of the MoE layer forward pass.  Declarations and contracts are in
// include/moe.h.
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <mutex>
#include <vector>

#include "moe_internal.cuh"

namespace moe {
namespace {

// Device error word: kernels OR kErrTimeout / kErrInput into it.
__device__ uint32_t g_device_error;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint32_t *g_err_ptr[kMaxDevices];
int g_sms[kMaxDevices];

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

int current_device() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) return -1;
    return d;
}

// Device address of g_device_error on the current device (looked up once per device).
uint32_t *err_ptr() {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_err_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        g_err_ptr[dev] = static_cast<uint32_t *>(p);
    }
    return g_err_ptr[dev];
}

using Layout = WsLayout;
using Part = WsPart;

// Scratch of the tensor-core router (fp32 logits), 0 when the CUDA-core router runs.
size_t router_scratch_bytes(const moe_config &c) {
    return router_tc_supported(c.T, c.E, c.dtype) ? router_tc_workspace_bytes(c.T, c.d, c.E, c.h_shared > 0) : 0;
}
// Per-CTA score sums of the score-mean statistic.
size_t router_stats_bytes(const moe_config &c) { return sizeof(float) * (size_t)router_stats_rows(c.T) * c.E; }
// moe_route's scratch: the logits part, then (256-byte aligned) the statistic part.
size_t route_ws_total(const moe_config &c) { return align256(router_scratch_bytes(c)) + router_stats_bytes(c); }

Layout make_layout(const moe_config &c, bool train = false) {
    Layout L{};
    const size_t R = (size_t)c.T * c.k, esz = c.dtype == MOE_F32 ? 4 : 2;
    L.size[P_IDS] = R * 4;
    L.size[P_GATES] = R * 4;
    L.size[P_SG] = c.h_shared > 0 ? (size_t)c.T * 4 : 0;
    L.size[P_COUNTS] = (size_t)c.E * 4;
    L.size[P_OFFSETS] = ((size_t)c.E + 1) * 4;
    L.size[P_SORTED] = R * 4;
    L.size[P_INV] = R * 4;
    L.size[P_ACT] = R * (size_t)c.h * esz;
    L.size[P_ACTS] = c.h_shared > 0 ? (size_t)c.T * c.h_shared * esz : 0;
    L.size[P_YACC] = c.dtype == MOE_BF16 ? (size_t)c.T * c.d * 4 : 0;
    L.size[P_PERM] = permute_workspace_bytes((int64_t)R, c.E);
    L.size[P_LOGITS] = router_scratch_bytes(c);
    L.size[P_STATS] = router_stats_bytes(c);
    L.size[P_SLOTS] = c.combine == MOE_COMBINE_ORDERED ? R * (size_t)c.d * 4 : 0;
    if (train) {
        // kept for the backward pass, and the backward's scratch (the dx accumulator reuses y_acc)
        const size_t hs = (size_t)c.h_shared;
        L.size[P_PROBS] = (size_t)c.T * c.E * 4;
        L.size[P_HPRE] = (size_t)hpre_rows((int64_t)R) * 2 * (size_t)c.h * esz;
        L.size[P_HPRES] = (size_t)hpre_rows(c.T) * 2 * hs * esz;
        const size_t Rp = (size_t)padded_rows((int64_t)R, c.E);
        L.size[P_DG] = R * 4;
        L.size[P_DSG] = hs ? (size_t)c.T * 4 : 0;
        L.size[P_DH] = Rp * 2 * (size_t)c.h * esz;
        L.size[P_XG] = Rp * (size_t)c.d * esz;
        L.size[P_DYG] = Rp * (size_t)c.d * esz;
        L.size[P_GA] = Rp * (size_t)c.h * esz;
        L.size[P_DHS] = (size_t)c.T * 2 * hs * esz;
        L.size[P_GAS] = (size_t)c.T * hs * esz;
        L.size[P_DLB] = (size_t)c.T * dl_stride(c.E) * 2;
        L.size[P_DLS] = hs ? (size_t)c.T * 4 : 0;
        if (c.dtype == MOE_BF16 && L.size[P_YACC] == 0) L.size[P_YACC] = (size_t)c.T * c.d * 4;
    }
    size_t o = 0;
    for (int i = 0; i < P_N; ++i) {
        L.off[i] = o;
        o += align256(L.size[i]);
    }
    L.total = o;
    return L;
}

template <typename T>
T *part(void *ws, const Layout &L, Part p) {
    return ws_part<T>(ws, L, p);
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

std::atomic<int64_t> g_launches{0};

// Per-thread profiling events (moe_profile_events).
thread_local cudaEvent_t t_events[MOE_STAGE_COUNT + 1];
thread_local bool t_profile = false;

// Per-thread NVTX stage ranges (moe_profile_nvtx).
thread_local bool t_nvtx = false;
const char *const kStageNames[MOE_STAGE_COUNT] = {"moe route",      "moe permute",     "moe gate_up",
                                                  "moe shared gate_up", "moe down", "moe shared down",
                                                  "moe finalize"};

// Boundary i of a forward call: 0 before the first launch, 1 + s after stage s.
void mark(int i, cudaStream_t s) {
    if (t_profile) cudaEventRecord(t_events[i], s);
    if (t_nvtx) {
        if (i > 0) nvtxRangePop();
        if (i < MOE_STAGE_COUNT) nvtxRangePushA(kStageNames[i]);
    }
}

// The tensor-core grouped GEMM serves batches above this many assignments;
// smaller ones (decode) use the CUDA-core segment kernels.
constexpr int32_t kDecodeMaxRows = 64;

// MMA N of the expert GEMMs: 256 unless the output width is not a multiple of
// the wide tile (128 output columns for gate/up, 256 for down), where the last
// column tile would load weight rows of the next expert for nothing; then 128.
bool narrow_gateup(const moe_config &c) { return c.h % 128 != 0; }
bool narrow_down(const moe_config &c) { return c.d % 256 != 0; }

// Experts average at most one 128-row tile: every weight tile is read once.
bool one_tile_per_expert(const moe_config &c) { return (int64_t)c.T * c.k <= 128LL * c.E; }

// Two SMs per tile (M = 256 across a CTA pair) for GEMMs whose groups average
// at least 512 rows: the layer is tensor-bound and the operand traffic per SM
// drops by a third (measured: mixtral_prefill down 874 -> 732 us, the shared
// expert's gate/up and down of qwen_shared -17%).  With gathered token rows
// the pair pays only with its wide tiles (two MMAs of N = 256 per K slice, so
// the gather is needed at half the rate per FLOP), which want the output width
// to be a multiple of 256; with fewer rows the 256-row tiles waste work.
// MOE_GG_PAIR=1 / 0 forces it on / off.
#ifndef MOE_GG_PAIR_GATHER
#define MOE_GG_PAIR_GATHER 1
#endif
bool pair_tiles(int64_t rows, int groups, bool gather, int64_t out_cols) {
    static const int force = [] {
        const char *v = std::getenv("MOE_GG_PAIR");
        return v ? (v[0] == '1' ? 1 : 0) : -1;
    }();
    if (force >= 0) return force == 1;
    if (gather) return MOE_GG_PAIR_GATHER && out_cols % 256 == 0 && rows >= 512LL * groups;
    return rows >= 512LL * groups;
}

// 64-row tiles for a contiguous A when the groups average at most 64 rows
// (the weights stream from HBM; see grouped_gemm.cu).  MOE_GG_HALF=1 / 0
// forces it on / off.
bool half_tiles(int64_t rows, int groups) {
    static const int force = [] {
        const char *v = std::getenv("MOE_GG_HALF");
        return v ? (v[0] == '1' ? 1 : 0) : -1;
    }();
    if (force >= 0) return force == 1;
    return rows <= 64LL * groups;
}

GemmLaunch gemm_gateup(const moe_config &c, const void *x, const void *wg, const void *wu, const int32_t *offsets,
                       const int32_t *srt, void *act, uint32_t *err) {
    GemmLaunch L{};
    L.mode = 0;
    L.gather = true;
    L.dtype = c.dtype;
    L.p = GemmParams{offsets, srt, c.E, c.k, c.T * c.k, c.T, c.d, c.h, x, act, nullptr, nullptr, err};
    L.narrow = narrow_gateup(c);
    L.p.stream_weights = one_tile_per_expert(c);
    L.pair = pair_tiles(c.T * c.k, c.E, true, c.h);
    L.b0 = wg;
    L.b1 = wu;
    return L;
}
GemmLaunch gemm_gateup_dense(const moe_config &c, const void *x, const void *wg, const void *wu, void *act,
                             uint32_t *err) {
    GemmLaunch L{};
    L.mode = 0;
    L.gather = false;
    L.dtype = c.dtype;
    L.p = GemmParams{nullptr, nullptr, 1, 1, c.T, c.T, c.d, c.h_shared, x, act, nullptr, nullptr, err};
    L.pair = pair_tiles(c.T, 1, false, c.h_shared);
    L.a_src = x;
    L.b0 = wg;
    L.b1 = wu;
    return L;
}
// Column groups of the routed down GEMM (see decode_n).  Two groups halve the
// part of the fp32 accumulator [T, d] that the CTAs reduce into at one time,
// so that it stays in L2 while the k experts of each token add into it, at
// the price of reading act twice: taken when the accumulator is larger than
// 48 MB and act at most 2.5 times its size.  MOE_DOWN_GROUPS=n forces n.
int down_groups(const moe_config &c, int n_tiles) {
    static const int force = [] {
        const char *v = std::getenv("MOE_DOWN_GROUPS");
        return v ? std::atoi(v) : 0;
    }();
    const int64_t acc = (int64_t)c.T * c.d * 4;
    const int64_t act = (int64_t)c.T * c.k * c.h * (c.dtype == MOE_F32 ? 4 : 2);
    int g = force > 0 ? force : (acc > (48LL << 20) && 2 * act <= 5 * acc ? 2 : 1);
    return g < 1 ? 1 : (g > n_tiles ? n_tiles : g);
}

GemmLaunch gemm_down(const moe_config &c, const void *act, const void *wd, const int32_t *offsets,
                     const int32_t *srt, const float *gates, float *acc, uint32_t *err) {
    GemmLaunch L{};
    L.mode = 1;
    L.gather = false;
    L.dtype = c.dtype;
    L.p = GemmParams{offsets, srt, c.E, c.k, c.T * c.k, c.T, c.h, c.d, nullptr, nullptr, acc, gates, err};
    L.narrow = narrow_down(c);
    L.p.stream_weights = one_tile_per_expert(c);
    L.pair = pair_tiles(c.T * c.k, c.E, false, c.d);
    L.half = !L.pair && half_tiles(c.T * c.k, c.E);
    L.p.n_groups = down_groups(c, (c.d + (L.narrow ? 127 : 255)) / (L.narrow ? 128 : 256));
    L.a_src = act;
    L.b0 = wd;
    return L;
}
GemmLaunch gemm_down_dense(const moe_config &c, const void *act, const void *wd, const float *sg, float *acc,
                           uint32_t *err) {
    GemmLaunch L{};
    L.mode = 1;
    L.gather = false;
    L.dtype = c.dtype;
    L.p = GemmParams{nullptr, nullptr, 1, 1, c.T, c.T, c.h_shared, c.d, nullptr, nullptr, acc, sg, err};
    L.pair = pair_tiles(c.T, 1, false, c.d);
    L.a_src = act;
    L.b0 = wd;
    return L;
}
bool use_gemm(const moe_config &c) { return c.T * c.k > kDecodeMaxRows; }

// The fused expert kernel (gate/up, SwiGLU, down and combine in one pass over
// the weights) only when MOE_FUSED=1 asks for it (where the shape allows):
// on the layers it targets (experts of about one 128-row tile) it measured
// slower than the two grouped GEMMs (gemma_upcycle: 150 us against ~104 us),
// so the two-kernel path is the default.
// The speculative L2 prefetch of each CTA's first gate/up weight tile
// (kEarlyPrefetch); MOE_PREFETCH=0 turns it off.
bool prefetch_first_tiles() {
    static const bool on = [] {
        const char *v = std::getenv("MOE_PREFETCH");
        return !(v && v[0] == '0');
    }();
    return on;
}

bool use_fused(const moe_config &c) {
    static const bool on = [] {
        const char *v = std::getenv("MOE_FUSED");
        return v && v[0] == '1';
    }();
    return on && c.dtype == MOE_BF16 && c.h % 64 == 0;
}


}  // namespace

uint32_t *device_error_word() { return err_ptr(); }
WsLayout ws_layout(const moe_config &c, bool train) { return make_layout(c, train); }
size_t combine_scratch_floats(const moe_config &c) {
    if (c.combine == MOE_COMBINE_ORDERED) return (size_t)c.T * c.k * c.d;
    return c.dtype == MOE_BF16 ? (size_t)c.T * c.d : 0;
}

cudaError_t launch_combine(const moe_config &c, const void *act, const void *w_down, const int32_t *offsets,
                           const int32_t *srt, const float *gates, void *y, float *buf, cudaStream_t s,
                           uint32_t *err) {
    const bool ordered = c.combine == MOE_COMBINE_ORDERED;
    // ordered: every slot row is stored once, so nothing needs clearing
    float *acc = ordered ? nullptr : (c.dtype == MOE_BF16 ? buf : static_cast<float *>(y));
    cudaError_t e = ordered ? cudaSuccess : cudaMemsetAsync(acc, 0, (size_t)c.T * c.d * sizeof(float), s);
    if (e != cudaSuccess) return e;
    if (use_gemm(c)) {
        GemmLaunch dl = gemm_down(c, act, w_down, offsets, srt, gates, acc, err);
        dl.p.slot_out = ordered ? buf : nullptr;
        e = launch_grouped_gemm(dl, s);
    } else {
        SegDownArgs a{};
        a.act = act;
        a.w_down = w_down;
        a.seg = Segments{offsets, srt, c.E, c.k, c.T * c.k};
        a.T = c.T;
        a.d = c.d;
        a.hid = c.h;
        a.gates = gates;
        a.y_acc = acc;
        a.slots = ordered ? buf : nullptr;
        e = launch_seg_down(a, c.dtype, s, err);
    }
    if (e != cudaSuccess) return e;
    if (ordered) return launch_finalize_ordered(buf, nullptr, y, c.T, c.d, c.k, c.dtype, s);
    return c.dtype == MOE_BF16 ? launch_finalize(acc, y, c.T * c.d, s) : cudaSuccess;
}

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

bool pdl_enabled() {
    static const bool on = [] {
        const char *v = std::getenv("MOE_PDL");
        return !(v && v[0] == '0');
    }();
    return on;
}

int num_sms() {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return 148;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_sms[dev]) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        g_sms[dev] = v;
    }
    return g_sms[dev];
}

}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: null pointer, bad size, k outside [1, E] or bad enum";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape outside the library's limits";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace null, misaligned or too small";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call or kernel launch failed";
        case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT: a kernel's bounded wait ran out";
        case MOE_ERR_DEVICE_INPUT: return "MOE_ERR_DEVICE_INPUT: a kernel met an invalid device input";
    }
    return "unknown moe_status";
}

moe_status moe_validate(const moe_config *c) {
    if (!c) return MOE_ERR_INVALID_ARG;
    if (c->T < 0 || c->d < 1 || c->E < 1 || c->h < 1 || c->k < 1 || c->k > c->E || c->h_shared < 0)
        return MOE_ERR_INVALID_ARG;
    if (c->score != MOE_SCORE_SOFTMAX && c->score != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
    if (c->dtype != MOE_BF16 && c->dtype != MOE_F32) return MOE_ERR_INVALID_ARG;
    if (c->combine != MOE_COMBINE_ADD && c->combine != MOE_COMBINE_ORDERED) return MOE_ERR_INVALID_ARG;
    if (c->E > MOE_MAX_EXPERTS || c->k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
    if (c->d % 8 || c->h % 8 || c->h_shared % 8) return MOE_ERR_UNSUPPORTED;
    if (c->T * (int64_t)c->k >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
    int64_t w = c->d > c->h ? c->d : c->h;
    if (c->h_shared > w) w = c->h_shared;
    if (c->T * w >= (int64_t)1 << 40) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status moe_workspace_size(const moe_config *c, size_t *bytes) {
    if (!bytes) return MOE_ERR_INVALID_ARG;
    const moe_status st = moe_validate(c);
    if (st != MOE_OK) return st;
    *bytes = make_layout(*c).total;
    return MOE_OK;
}

moe_status moe_workspace_layout(const moe_config *c, void *ws, size_t ws_bytes, moe_workspace_views *v) {
    if (!v) return MOE_ERR_INVALID_ARG;
    const moe_status st = moe_validate(c);
    if (st != MOE_OK) return st;
    const Layout L = make_layout(*c);
    if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255)) return MOE_ERR_WORKSPACE;
    v->ids = part<int32_t>(ws, L, P_IDS);
    v->gates = part<float>(ws, L, P_GATES);
    v->shared_gate = part<float>(ws, L, P_SG);
    v->counts = part<int32_t>(ws, L, P_COUNTS);
    v->offsets = part<int32_t>(ws, L, P_OFFSETS);
    v->sorted_rows = part<int32_t>(ws, L, P_SORTED);
    v->inv_rows = part<int32_t>(ws, L, P_INV);
    v->act = part<void>(ws, L, P_ACT);
    v->act_shared = part<void>(ws, L, P_ACTS);
    v->y_acc = part<float>(ws, L, P_YACC);
    v->y_slots = part<float>(ws, L, P_SLOTS);
    return MOE_OK;
}

int32_t moe_decode_max_rows(void) { return kDecodeMaxRows; }

moe_status moe_route_workspace_size(const moe_config *c, size_t *bytes) {
    if (!bytes) return MOE_ERR_INVALID_ARG;
    const moe_status st = moe_validate(c);
    if (st != MOE_OK) return st;
    *bytes = route_ws_total(*c);
    return MOE_OK;
}

moe_status moe_route(const moe_config *c, const moe_route_opts *opts, const void *x, const void *w_router,
                     const void *w_shared_gate, int32_t *ids, float *gates, float *probs, float *shared_gate,
                     void *ws, size_t ws_bytes, void *stream) {
    moe_status st = moe_validate(c);
    if (st != MOE_OK) return st;
    if (c->T == 0) return MOE_OK;
    if (!x || !w_router || !ids || !gates) return MOE_ERR_INVALID_ARG;
    if (shared_gate && !w_shared_gate) return MOE_ERR_INVALID_ARG;
    const bool stats = opts && opts->score_mean;
    const size_t logits = router_scratch_bytes(*c);
    // the statistic part is needed only when the statistic is asked for
    const size_t need = stats ? route_ws_total(*c) : logits;
    if (need && (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255))) return MOE_ERR_WORKSPACE;
    RouterArgs a{};
    a.x = x;
    a.w_router = w_router;
    a.w_shared_gate = shared_gate ? w_shared_gate : nullptr;
    a.T = c->T;
    a.d = c->d;
    a.E = c->E;
    a.k = c->k;
    a.norm_topk = c->norm_topk != 0;
    a.score = c->score;
    a.ids = ids;
    a.gates = gates;
    a.probs = probs;
    a.shared_gate = shared_gate;
    a.zero_rows = nullptr;
    a.bias = opts ? opts->balance_bias : nullptr;
    a.score_mean = stats ? opts->score_mean : nullptr;
    a.stats = stats ? reinterpret_cast<float *>(static_cast<char *>(ws) + align256(logits)) : nullptr;
    a.err = err_ptr();
    if (!a.err) return MOE_ERR_CUDA;
    return cuda_status(launch_router(a, c->dtype, logits ? static_cast<float *>(ws) : nullptr,
                                     static_cast<cudaStream_t>(stream)));
}

moe_status moe_permute_workspace_size(const moe_config *c, size_t *bytes) {
    if (!bytes) return MOE_ERR_INVALID_ARG;
    const moe_status st = moe_validate(c);
    if (st != MOE_OK) return st;
    *bytes = permute_workspace_bytes(c->T * c->k, c->E);
    return MOE_OK;
}

moe_status moe_permute(const moe_config *c, const int32_t *ids, int32_t *counts, int32_t *offsets,
                       int32_t *sorted_rows, int32_t *inv_rows, void *ws, size_t ws_bytes, void *stream) {
    moe_status st = moe_validate(c);
    if (st != MOE_OK) return st;
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    if (c->T > 0 && (!ids || !sorted_rows || !inv_rows)) return MOE_ERR_INVALID_ARG;
    if (c->T > 0 && (!ws || ws_bytes < permute_workspace_bytes(c->T * c->k, c->E) ||
                     (reinterpret_cast<uintptr_t>(ws) & 15)))
        return MOE_ERR_WORKSPACE;
    uint32_t *err = err_ptr();
    if (!err) return MOE_ERR_CUDA;
    PermuteArgs a{ids, (int)(c->T * c->k), c->E, counts, offsets, sorted_rows, inv_rows, err};
    return cuda_status(launch_permute(a, static_cast<int32_t *>(ws), false, static_cast<cudaStream_t>(stream)));
}

moe_status moe_grouped_swiglu(const moe_config *c, const void *x, const void *w_gate, const void *w_up,
                              const int32_t *offsets, const int32_t *sorted_rows, void *act, void *stream) {
    moe_status st = moe_validate(c);
    if (st != MOE_OK) return st;
    if (c->T == 0) return MOE_OK;
    if (!x || !w_gate || !w_up || !offsets || !sorted_rows || !act) return MOE_ERR_INVALID_ARG;
    uint32_t *err = err_ptr();
    if (!err) return MOE_ERR_CUDA;
    SegGateUpArgs a{};
    a.x = x;
    a.w_gate = w_gate;
    a.w_up = w_up;
    a.seg = Segments{offsets, sorted_rows, c->E, c->k, c->T * c->k};
    a.T = c->T;
    a.d = c->d;
    a.hid = c->h;
    a.act = act;
    if (use_gemm(*c))
        return cuda_status(launch_grouped_gemm(gemm_gateup(*c, x, w_gate, w_up, offsets, sorted_rows, act, err),
                                               static_cast<cudaStream_t>(stream)));
    return cuda_status(launch_seg_gateup(a, c->dtype, static_cast<cudaStream_t>(stream), err));
}

moe_status moe_combine(const moe_config *c, const void *act, const void *w_down, const int32_t *offsets,
                       const int32_t *sorted_rows, const float *gates, void *y, void *ws, size_t ws_bytes,
                       void *stream) {
    moe_status st = moe_validate(c);
    if (st != MOE_OK) return st;
    if (c->T == 0) return MOE_OK;
    if (!act || !w_down || !offsets || !sorted_rows || !gates || !y) return MOE_ERR_INVALID_ARG;
    const size_t need = combine_scratch_floats(*c) * 4;
    if (need && (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 15))) return MOE_ERR_WORKSPACE;
    uint32_t *err = err_ptr();
    if (!err) return MOE_ERR_CUDA;
    return cuda_status(launch_combine(*c, act, w_down, offsets, sorted_rows, gates, y, static_cast<float *>(ws),
                                      static_cast<cudaStream_t>(stream), err));
}

}  // extern "C"

namespace moe {
// bf16 batch-1 down projection with the weight rows streamed by TMA through a
// shared-memory ring (segment_tma.cu); the warp-per-row kernel serves the rest.
bool down_tma_supported(const DownDirectArgs &a, int dtype);
cudaError_t launch_down_tma(const DownDirectArgs &a, cudaStream_t s, uint32_t *err);

// The forward pass; `train` also keeps what moe_backward needs (the full score
// rows and the pre-activations of every grouped row) and always takes the
// tensor-core path, whose gate/up epilogue writes them.
moe_status forward_impl(const moe_config *c, const moe_route_opts *opts, const void *x, const void *w_router,
                        const void *w_gate, const void *w_up, const void *w_down, const void *sh_gate,
                        const void *sh_up, const void *sh_down, const void *w_shared_gate, void *y, void *ws,
                        size_t ws_bytes, void *stream, bool train) {
    moe_status st = moe_validate(c);
    if (st != MOE_OK) return st;
    if (train && c->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (c->T == 0) return MOE_OK;
    if (!x || !w_router || !w_gate || !w_up || !w_down || !y) return MOE_ERR_INVALID_ARG;
    const bool shared = c->h_shared > 0;
    if (shared && (!sh_gate || !sh_up || !sh_down || !w_shared_gate)) return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(*c, train);
    if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255)) return MOE_ERR_WORKSPACE;
    uint32_t *err = err_ptr();
    if (!err) return MOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool bf16 = c->dtype == MOE_BF16;

    int32_t *ids = part<int32_t>(ws, L, P_IDS);
    float *gates = part<float>(ws, L, P_GATES);
    float *sg = part<float>(ws, L, P_SG);
    int32_t *counts = part<int32_t>(ws, L, P_COUNTS);
    int32_t *offsets = part<int32_t>(ws, L, P_OFFSETS);
    int32_t *srt = part<int32_t>(ws, L, P_SORTED);
    int32_t *inv = part<int32_t>(ws, L, P_INV);
    void *act = part<void>(ws, L, P_ACT);
    void *acts = part<void>(ws, L, P_ACTS);
    float *acc = bf16 ? part<float>(ws, L, P_YACC) : static_cast<float *>(y);

    RouterArgs ra{};
    ra.x = x;
    ra.w_router = w_router;
    ra.w_shared_gate = shared ? w_shared_gate : nullptr;
    ra.T = c->T;
    ra.d = c->d;
    ra.E = c->E;
    ra.k = c->k;
    ra.norm_topk = c->norm_topk != 0;
    ra.score = c->score;
    ra.ids = ids;
    ra.gates = gates;
    ra.probs = train ? part<float>(ws, L, P_PROBS) : nullptr;
    ra.shared_gate = sg;
    const bool gemm = train || use_gemm(*c);
    // ordered combine: the routed rows go to their slot rows and a last pass adds
    // them in slot order (the small-batch path already sums in slot order)
    const bool ordered = gemm && c->combine == MOE_COMBINE_ORDERED;
    float *slots = ordered ? part<float>(ws, L, P_SLOTS) : nullptr;
    const bool fused = gemm && !train && !ordered && use_fused(*c);
    // the fused expert kernel adds into the accumulator from its first unit on, so
    // the router clears it; otherwise the gate/up GEMM does (the small-batch path writes y)
    ra.zero_rows = fused ? acc : nullptr;
    ra.err = err;
    ra.bias = opts ? opts->balance_bias : nullptr;
    ra.score_mean = opts ? opts->score_mean : nullptr;
    ra.stats = ra.score_mean ? part<float>(ws, L, P_STATS) : nullptr;
    // the tensor-core router also builds the grouping histogram
    const bool fused_hist = L.size[P_LOGITS] && c->T * c->k > permute_chunk();
    ra.hist = fused_hist ? part<int32_t>(ws, L, P_PERM) : nullptr;
    ra.hist_chunk = permute_chunk();
    // one token (decode): the router writes the grouping itself
    const bool one_token = c->T == 1 && !L.size[P_LOGITS];
    if (one_token) {
        ra.counts = counts;
        ra.offsets = offsets;
        ra.sorted_rows = srt;
        ra.inv_rows = inv;
    }
    mark(0, s);
    cudaError_t e = launch_router(ra, c->dtype, part<float>(ws, L, P_LOGITS), s);
    mark(1 + MOE_STAGE_ROUTE, s);

    const int R = (int)(c->T * c->k);
    if (e == cudaSuccess && !one_token) {
        PermuteArgs pa{ids, R, c->E, counts, offsets, srt, inv, err};
        e = launch_permute(pa, part<int32_t>(ws, L, P_PERM), fused_hist, s);
    }
    mark(1 + MOE_STAGE_PERMUTE, s);
    const Segments routed{offsets, srt, c->E, c->k, (int64_t)R};
    const Segments dense{nullptr, nullptr, 1, 1, c->T};
    if (e == cudaSuccess && fused) {
        e = launch_fused_expert(*c, x, w_gate, w_up, w_down, offsets, srt, gates, acc, err, s);
    } else if (e == cudaSuccess) {
        SegGateUpArgs ga{x, w_gate, w_up, routed, c->T, c->d, c->h, act};
        GemmLaunch gl = gemm_gateup(*c, x, w_gate, w_up, offsets, srt, act, err);
        if (gl.p.stream_weights && prefetch_first_tiles()) gl.p.early |= kEarlyPrefetch;
        // the down GEMMs accumulate into it two kernels later (ordered: only the shared one)
        gl.p.zero = !ordered || shared ? acc : nullptr;
        gl.p.zero_floats = c->T * c->d;
        gl.p.hpre = train ? part<void>(ws, L, P_HPRE) : nullptr;
        e = gemm ? launch_grouped_gemm(gl, s) : launch_seg_gateup(ga, c->dtype, s, err);
    }
    mark(1 + MOE_STAGE_GATE_UP, s);
    if (e == cudaSuccess && shared) {
        SegGateUpArgs ga{x, sh_gate, sh_up, dense, c->T, c->d, c->h_shared, acts};
        GemmLaunch gl = gemm_gateup_dense(*c, x, sh_gate, sh_up, acts, err);
        gl.p.early = kEarlyTiles | kEarlyA;   // x and the weights are layer inputs
        gl.p.hpre = train ? part<void>(ws, L, P_HPRES) : nullptr;
        e = gemm ? launch_grouped_gemm(gl, s) : launch_seg_gateup(ga, c->dtype, s, err);
    }
    mark(1 + MOE_STAGE_SHARED_GATE_UP, s);
    if (!gemm) {
        // small batch: down projection, gate-weighted combine and the shared
        // expert in one pass that writes y
        if (e == cudaSuccess) {
            DownDirectArgs da{act, w_down, ids, inv, gates, shared ? acts : nullptr, shared ? sh_down : nullptr,
                              sg, c->T, c->d, c->h, c->E, c->k, c->h_shared, y};
            e = down_tma_supported(da, c->dtype) ? launch_down_tma(da, s, err)
                                                 : launch_down_direct(da, c->dtype, s, err);
        }
        mark(1 + MOE_STAGE_DOWN, s);
        mark(1 + MOE_STAGE_SHARED_DOWN, s);
        mark(1 + MOE_STAGE_FINALIZE, s);
        return cuda_status(e);
    }
    // the grouping step ran two or more kernels back, so the offsets are
    // complete when the down GEMM starts; act is read after the wait
    GemmLaunch dl = gemm_down(*c, act, w_down, offsets, srt, gates, acc, err);
    dl.p.early = kEarlyTiles;
    dl.p.slot_out = slots;
    if (e == cudaSuccess && !fused) e = launch_grouped_gemm(dl, s);   // fused: done in the gate/up stage
    mark(1 + MOE_STAGE_DOWN, s);
    // the shared expert's act came from the kernel before the routed down GEMM
    // (with the fused expert kernel, from the kernel right before this one)
    GemmLaunch sdl = gemm_down_dense(*c, acts, sh_down, sg, acc, err);
    sdl.p.early = fused ? kEarlyTiles : (kEarlyTiles | kEarlyA);
    if (e == cudaSuccess && shared) e = launch_grouped_gemm(sdl, s);
    mark(1 + MOE_STAGE_SHARED_DOWN, s);
    // ordered: y = the slot rows in slot order, then the shared expert's row (its
    // down GEMM is the only writer of each accumulator element, so that sum is exact)
    if (e == cudaSuccess && ordered)
        e = launch_finalize_ordered(slots, shared ? acc : nullptr, y, c->T, c->d, c->k, c->dtype, s);
    else if (e == cudaSuccess && bf16)
        e = launch_finalize(acc, y, c->T * c->d, s);
    mark(1 + MOE_STAGE_FINALIZE, s);
    return cuda_status(e);
}
}  // namespace moe

extern "C" {

moe_status moe_forward(const moe_config *c, const moe_route_opts *opts, const void *x, const void *w_router,
                       const void *w_gate, const void *w_up, const void *w_down, const void *sh_gate,
                       const void *sh_up, const void *sh_down, const void *w_shared_gate, void *y, void *ws,
                       size_t ws_bytes, void *stream) {
    return forward_impl(c, opts, x, w_router, w_gate, w_up, w_down, sh_gate, sh_up, sh_down, w_shared_gate, y, ws,
                        ws_bytes, stream, false);
}

namespace {

constexpr int64_t kMaxHostPieces = 256;   // moe_forward_host: events per call stay few

// Pieces of moe_forward_host: n = min(chunks, T, 256); with n >= 3 the first
// and last pieces carry half the tokens of the others (the first piece's copy
// in and the last piece's copy back are the parts no layer overlaps), so
// piece i spans tokens [T c_i / (2n - 2), T c_{i+1} / (2n - 2)) with c_0 = 0,
// c_i = 2i - 1 (0 < i < n), c_n = 2n - 2 (integer division); with n <= 2 the
// pieces are T c_i / n with c_i = i.
int64_t host_pieces(int64_t T, int32_t chunks) {
    int64_t n = chunks > T ? T : chunks;
    return n > kMaxHostPieces ? kMaxHostPieces : n;
}
int64_t host_bound(int64_t T, int64_t n, int64_t i) {
    if (n <= 2) return T * i / n;
    const int64_t c = i == 0 ? 0 : (i == n ? 2 * n - 2 : 2 * i - 1);
    return T * c / (2 * n - 2);
}

// Workspace of moe_forward_host: the device copies of x and y, then the
// layer's workspace for its largest piece.
struct HostLayout {
    size_t x_off, y_off, ws_off, total;
    int64_t n;   // pieces
};
moe_status host_layout(const moe_config &c, int32_t chunks, HostLayout *h) {
    if (chunks <= 0) return MOE_ERR_INVALID_ARG;
    const moe_status st = moe_validate(&c);
    if (st != MOE_OK) return st;
    const size_t esz = c.dtype == MOE_F32 ? 4 : 2;
    h->n = host_pieces(c.T, chunks);
    int64_t largest = 0;
    for (int64_t i = 0; i < h->n; ++i)
        largest = std::max<int64_t>(largest, host_bound(c.T, h->n, i + 1) - host_bound(c.T, h->n, i));
    moe_config pc = c;
    pc.T = largest;
    const size_t rows = (size_t)c.T * c.d * esz;
    h->x_off = 0;
    h->y_off = align256(rows);
    h->ws_off = h->y_off + align256(rows);
    h->total = h->ws_off + (pc.T > 0 ? make_layout(pc).total : 0);
    return MOE_OK;
}

}  // namespace

moe_status moe_forward_host_workspace_size(const moe_config *c, int32_t chunks, size_t *bytes) {
    if (!c || !bytes) return MOE_ERR_INVALID_ARG;
    HostLayout h;
    const moe_status st = host_layout(*c, chunks, &h);
    if (st == MOE_OK) *bytes = h.total;
    return st;
}

moe_status moe_forward_host(const moe_config *c, const void *x_host, const void *w_router, const void *w_gate,
                            const void *w_up, const void *w_down, const void *sh_gate, const void *sh_up,
                            const void *sh_down, const void *w_shared_gate, void *y_host, int32_t chunks, void *ws,
                            size_t ws_bytes, void *stream, void *copy_stream) {
    if (!c) return MOE_ERR_INVALID_ARG;
    HostLayout h;
    moe_status st = host_layout(*c, chunks, &h);
    if (st != MOE_OK) return st;
    if (c->T == 0) return MOE_OK;
    if (!x_host || !y_host || !w_router || !w_gate || !w_up || !w_down) return MOE_ERR_INVALID_ARG;
    if (c->h_shared > 0 && (!sh_gate || !sh_up || !sh_down || !w_shared_gate)) return MOE_ERR_INVALID_ARG;
    if (!ws || ws_bytes < h.total || (reinterpret_cast<uintptr_t>(ws) & 255)) return MOE_ERR_WORKSPACE;
    const size_t row_bytes = (size_t)c->d * (c->dtype == MOE_F32 ? 4 : 2);
    char *xd = static_cast<char *>(ws) + h.x_off;
    char *yd = static_cast<char *>(ws) + h.y_off;
    void *lws = static_cast<char *>(ws) + h.ws_off;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaStream_t cs = copy_stream ? static_cast<cudaStream_t>(copy_stream) : s;
    const int64_t n = h.n;
    // events order the two streams: start (earlier work on stream is done
    // with the device copies), in[i] (piece i is on the device), out[i]
    // (piece i's y is ready), done (the last copy back has landed)
    std::vector<cudaEvent_t> ev((size_t)(2 * n + 2), nullptr);
    cudaError_t e = cudaSuccess;
    for (auto &v : ev)
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&v, cudaEventDisableTiming);
    cudaEvent_t &start = ev[0], &done = ev[1];
    auto ev_in = [&](int64_t i) { return ev[2 + i]; };
    auto ev_out = [&](int64_t i) { return ev[2 + n + i]; };
    if (e == cudaSuccess && cs != s) e = cudaEventRecord(start, s);
    if (e == cudaSuccess && cs != s) e = cudaStreamWaitEvent(cs, start, 0);
    // every piece's rows in first (one copy each), so that no copy to the
    // device waits behind a copy back on the copy stream
    for (int64_t i = 0; i < n && e == cudaSuccess; ++i) {
        const int64_t t0 = host_bound(c->T, n, i), rows = host_bound(c->T, n, i + 1) - t0;
        if (rows <= 0) continue;
        e = cudaMemcpyAsync(xd + t0 * row_bytes, static_cast<const char *>(x_host) + t0 * row_bytes,
                            (size_t)rows * row_bytes, cudaMemcpyHostToDevice, cs);
        if (e == cudaSuccess) e = cudaEventRecord(ev_in(i), cs);
    }
    for (int64_t i = 0; i < n && e == cudaSuccess && st == MOE_OK; ++i) {
        const int64_t t0 = host_bound(c->T, n, i), rows = host_bound(c->T, n, i + 1) - t0;
        if (rows <= 0) continue;
        moe_config pc = *c;
        pc.T = rows;
        e = cudaStreamWaitEvent(s, ev_in(i), 0);
        if (e != cudaSuccess) break;
        st = forward_impl(&pc, nullptr, xd + t0 * row_bytes, w_router, w_gate, w_up, w_down, sh_gate, sh_up,
                          sh_down, w_shared_gate, yd + t0 * row_bytes, lws, ws_bytes - h.ws_off, stream, false);
        if (st != MOE_OK) break;
        e = cudaEventRecord(ev_out(i), s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, ev_out(i), 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(static_cast<char *>(y_host) + t0 * row_bytes, yd + t0 * row_bytes,
                                (size_t)rows * row_bytes, cudaMemcpyDeviceToHost, cs);
    }
    // the caller waits on `stream` alone
    if (e == cudaSuccess && st == MOE_OK && cs != s) e = cudaEventRecord(done, cs);
    if (e == cudaSuccess && st == MOE_OK && cs != s) e = cudaStreamWaitEvent(s, done, 0);
    for (auto &v : ev)
        if (v) cudaEventDestroy(v);   // released once the recorded work completes
    if (st != MOE_OK) return st;
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_forward_train(const moe_config *c, const moe_route_opts *opts, const void *x, const void *w_router,
                             const void *w_gate, const void *w_up, const void *w_down, const void *sh_gate,
                             const void *sh_up, const void *sh_down, const void *w_shared_gate, void *y, void *ws,
                             size_t ws_bytes, void *stream) {
    return forward_impl(c, opts, x, w_router, w_gate, w_up, w_down, sh_gate, sh_up, sh_down, w_shared_gate, y, ws,
                        ws_bytes, stream, true);
}

moe_status moe_quantize_q4(const void *w, int32_t dtype, int64_t rows, int32_t cols, uint8_t *q, float *scales,
                           void *stream) {
    if ((dtype != MOE_BF16 && dtype != MOE_F32) || rows < 0 || cols <= 0) return MOE_ERR_INVALID_ARG;
    if (cols % 64) return MOE_ERR_UNSUPPORTED;
    if (rows == 0) return MOE_OK;
    if (!w || !q || !scales) return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(q)) & 15) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_quantize_q4(w, dtype, rows, cols, q, scales, static_cast<cudaStream_t>(stream)));
}

moe_status moe_forward_q4(const moe_config *c, const moe_route_opts *opts, const void *x, const void *w_router,
                          const uint8_t *q_gate, const float *s_gate, const uint8_t *q_up, const float *s_up,
                          const uint8_t *q_down, const float *s_down, const void *sh_gate, const void *sh_up,
                          const void *sh_down, const void *w_shared_gate, void *y, void *ws, size_t ws_bytes,
                          void *stream) {
    moe_status st = moe_validate(c);
    if (st != MOE_OK) return st;
    if (c->dtype != MOE_BF16 || c->d % 64 || c->h % 64 || c->T * c->k > kDecodeMaxRows) return MOE_ERR_UNSUPPORTED;
    if (c->T == 0) return MOE_OK;
    if (!x || !w_router || !q_gate || !s_gate || !q_up || !s_up || !q_down || !s_down || !y)
        return MOE_ERR_INVALID_ARG;
    const uintptr_t qa = reinterpret_cast<uintptr_t>(q_gate) | reinterpret_cast<uintptr_t>(q_up) |
                         reinterpret_cast<uintptr_t>(q_down);
    if (qa & 15) return MOE_ERR_INVALID_ARG;
    const bool shared = c->h_shared > 0;
    if (shared && (!sh_gate || !sh_up || !sh_down || !w_shared_gate)) return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(*c);
    if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255)) return MOE_ERR_WORKSPACE;
    uint32_t *err = err_ptr();
    if (!err) return MOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t *ids = part<int32_t>(ws, L, P_IDS);
    float *gates = part<float>(ws, L, P_GATES);
    float *sg = part<float>(ws, L, P_SG);
    int32_t *counts = part<int32_t>(ws, L, P_COUNTS);
    int32_t *offsets = part<int32_t>(ws, L, P_OFFSETS);
    int32_t *srt = part<int32_t>(ws, L, P_SORTED);
    int32_t *inv = part<int32_t>(ws, L, P_INV);
    void *act = part<void>(ws, L, P_ACT);
    void *acts = part<void>(ws, L, P_ACTS);

    RouterArgs ra{};
    ra.x = x;
    ra.w_router = w_router;
    ra.w_shared_gate = shared ? w_shared_gate : nullptr;
    ra.T = c->T;
    ra.d = c->d;
    ra.E = c->E;
    ra.k = c->k;
    ra.norm_topk = c->norm_topk != 0;
    ra.score = c->score;
    ra.ids = ids;
    ra.gates = gates;
    ra.shared_gate = sg;
    ra.err = err;
    ra.bias = opts ? opts->balance_bias : nullptr;
    ra.score_mean = opts ? opts->score_mean : nullptr;
    ra.stats = ra.score_mean ? part<float>(ws, L, P_STATS) : nullptr;
    ra.hist_chunk = permute_chunk();
    const bool one_token = c->T == 1 && !L.size[P_LOGITS];
    if (one_token) {
        ra.counts = counts;
        ra.offsets = offsets;
        ra.sorted_rows = srt;
        ra.inv_rows = inv;
    }
    mark(0, s);
    cudaError_t e = launch_router(ra, c->dtype, part<float>(ws, L, P_LOGITS), s);
    mark(1 + MOE_STAGE_ROUTE, s);
    const int R = (int)(c->T * c->k);
    if (e == cudaSuccess && !one_token) {
        PermuteArgs pa{ids, R, c->E, counts, offsets, srt, inv, err};
        e = launch_permute(pa, part<int32_t>(ws, L, P_PERM), false, s);
    }
    mark(1 + MOE_STAGE_PERMUTE, s);
    // the ring-streamed kernels where the shapes and alignments allow them
    const bool tma = q4_tma_supported(c->d, c->h, x, q_gate, s_gate, q_up, s_up, q_down, s_down);
    if (e == cudaSuccess) {
        SegGateUpQ4Args ga{x, q_gate, q_up, s_gate, s_up, Segments{offsets, srt, c->E, c->k, (int64_t)R}, c->T, c->d,
                           c->h, act};
        e = tma ? launch_q4t_gateup(ga, s) : launch_seg_gateup_q4(ga, s, err);
    }
    mark(1 + MOE_STAGE_GATE_UP, s);
    if (e == cudaSuccess && shared) {
        SegGateUpArgs ga{x, sh_gate, sh_up, Segments{nullptr, nullptr, 1, 1, c->T}, c->T, c->d, c->h_shared, acts};
        e = launch_seg_gateup(ga, c->dtype, s, err);
    }
    mark(1 + MOE_STAGE_SHARED_GATE_UP, s);
    if (e == cudaSuccess) {
        DownDirectQ4Args da{act, q_down, s_down, ids, inv, gates, shared ? acts : nullptr, shared ? sh_down : nullptr,
                            sg, c->T, c->d, c->h, c->E, c->k, c->h_shared, y};
        if (!tma) {
            e = launch_down_direct_q4(da, s, err);
        } else {
            // the shared expert's gated rows first, into the (cleared) fp32
            // accumulator, one contribution per element; the 4-bit kernel adds
            // them after the routed experts
            float *acc = shared ? part<float>(ws, L, P_YACC) : nullptr;
            if (shared) {
                e = cudaMemsetAsync(acc, 0, (size_t)c->T * c->d * sizeof(float), s);
                SegDownArgs sa{};
                sa.act = acts;
                sa.w_down = sh_down;
                sa.seg = Segments{nullptr, nullptr, 1, 1, c->T};
                sa.T = c->T;
                sa.d = c->d;
                sa.hid = c->h_shared;
                sa.gates = sg;
                sa.y_acc = acc;
                if (e == cudaSuccess) e = launch_seg_down(sa, c->dtype, s, err);
            }
            if (e == cudaSuccess) e = launch_q4t_down(da, acc, s);
        }
    }
    mark(1 + MOE_STAGE_DOWN, s);
    mark(1 + MOE_STAGE_SHARED_DOWN, s);
    mark(1 + MOE_STAGE_FINALIZE, s);
    return cuda_status(e);
}

moe_status moe_train_workspace_size(const moe_config *c, size_t *bytes) {
    if (!bytes) return MOE_ERR_INVALID_ARG;
    const moe_status st = moe_validate(c);
    if (st != MOE_OK) return st;
    if (c->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    *bytes = make_layout(*c, true).total;
    return MOE_OK;
}

moe_status moe_profile_events(void *const *events, int32_t n) {
    if (!events) {
        t_profile = false;
        return MOE_OK;
    }
    if (n != MOE_STAGE_COUNT + 1) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i <= MOE_STAGE_COUNT; ++i) {
        if (!events[i]) return MOE_ERR_INVALID_ARG;
        t_events[i] = static_cast<cudaEvent_t>(events[i]);
    }
    t_profile = true;
    return MOE_OK;
}

moe_status moe_profile_nvtx(int32_t on) {
    t_nvtx = on != 0;
    return MOE_OK;
}

int64_t moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

moe_status moe_device_status(void *stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    uint32_t v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof v) != cudaSuccess) return MOE_ERR_CUDA;
    if (v && cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero) != cudaSuccess) return MOE_ERR_CUDA;
    if (v & kErrTimeout) return MOE_ERR_DEVICE_TIMEOUT;
    if (v & kErrInput) return MOE_ERR_DEVICE_INPUT;
    return MOE_OK;
}

}  // extern "C"
