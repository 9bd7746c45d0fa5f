// moe_backward: the gradient of the MoE layer after moe_forward_train.
//
// The chain rule through the forward's steps (the layer of "Tutorial 11:
// Mixture of Experts (MoE)", sections 2-4, with the sigmoid scores, shared
// expert and balance bias of "Small MoE Architecture, in depth", SmallMoE;
// "Small models, sparse experts", "Dispatch decides everything" trains it):
//
//   0. x and dy rows copied into the padded grouped layout the backward GEMMs
//      read by TMA (gather_pad_kernel)
//   1. routed experts, rows grouped by expert:  r = W_down^T dy;  the gate
//      gradient r . a;  du, dv through silu(u) * v;  gate * a kept for dW_down
//      (grouped_bwd.cu, SWIGLU)
//   2. the shared expert, the same on one dense segment with gate sigmoid(w_s.x)
//   3. router: the gate gradients through the (renormalised) softmax or the
//      sigmoid to the logits (router_bwd_kernel, one warp per token)
//   4. dx: W_gate^T du + W_up^T dv added into token order (SCATTER), the
//      shared expert's, and dl W_router; then fp32 -> bf16 with the shared
//      gate's w_s term (finalize_dx_kernel)
//   5. weight gradients: dW_down, dW_gate / dW_up per expert over its rows,
//      the shared expert's over all tokens, dW_router = dl^T x (WEIGHT), and
//      dw_s = sum_t dl_s x_t (shared_gate_grad_kernel, fixed summation order)
//
// The top-k selection (and the balance bias) passes no gradient.
#include <algorithm>

#include "grouped_tiles.cuh"
#include "moe_internal.cuh"

namespace moe {
namespace {

// The routed rows of x and dy copied into the padded grouped layout of the
// backward GEMMs (expert e's rows from row 64 * sum_{e' < e} ceil(count_e' /
// 64), in grouped order), with the padding rows -- past each segment's end up
// to the next multiple of 64 -- zeroed in x_g, dy_g, dH and ga.  CTA-strided
// over (64-row block, 1024-column slice) units; 16-byte copies.
struct GatherPadArgs {
    const __nv_bfloat16 *x, *dy;
    const int32_t *offsets, *sorted_rows;
    int E, k, d, h;
    int64_t T, R;
    __nv_bfloat16 *xg, *dyg, *dh, *ga;
    uint32_t *err;
};
__global__ void __launch_bounds__(256) gather_pad_kernel(GatherPadArgs a) {
    __shared__ int blk[MOE_MAX_EXPERTS + 1], off[MOE_MAX_EXPERTS + 1], end[MOE_MAX_EXPERTS + 1];
    __shared__ int nblk;
    pdl_wait();
    pdl_launch_dependents();
    if (threadIdx.x < 32) {
        GemmParams g{};
        g.offsets = a.offsets;
        g.E = a.E;
        g.rows = a.R;
        g.err = a.err;
        int n = 0;
        gg::build_tiles<64>(g, blk, off, end, &n);
        if (threadIdx.x == 31) nblk = n;
    }
    __syncthreads();
    const int cpr = a.d / 8;                 // 16-byte chunks per x / dy row
    const int S = (cpr + 127) / 128;         // column slices of 128 chunks
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int u = blockIdx.x; u < nblk * S; u += gridDim.x) {
        const int b = u / S, sl = u - b * S;
        const gg::Tile tl = gg::decode(b, 1, blk, a.E);
        const int64_t pr0 = (int64_t)b * 64;               // first padded row of the block
        const int64_t r0 = (int64_t)off[tl.e] + tl.m * 64;  // its first grouped row
        // x_g and dy_g: one warp per row (its token looked up once), each lane
        // four 16-byte chunks of the slice of x and of dy in flight before it
        // stores them
        for (int q = warp; q < 64; q += 8) {
            const int64_t r = r0 + q;
            int64_t t = -1;
            if (lane == 0 && r < end[tl.e]) {
                const int v = a.sorted_rows[r];
                t = (v >= 0 && v < a.R) ? v / a.k : -1;
                if (t < 0 || t >= a.T) {
                    atomicOr(a.err, kErrInput);
                    t = -1;
                }
            }
            t = __shfl_sync(0xffffffffu, t, 0);
            uint4 *xo = reinterpret_cast<uint4 *>(a.xg + (pr0 + q) * a.d);
            uint4 *dyo = reinterpret_cast<uint4 *>(a.dyg + (pr0 + q) * a.d);
            const uint4 *xi = reinterpret_cast<const uint4 *>(a.x + (t < 0 ? 0 : t) * a.d);
            const uint4 *dyi = reinterpret_cast<const uint4 *>(a.dy + (t < 0 ? 0 : t) * a.d);
            const int c0 = sl * 128 + lane;
            uint4 vx[4], vd[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + 32 * j;
                vx[j] = vd[j] = make_uint4(0, 0, 0, 0);
                if (t >= 0 && c < cpr) {
                    vx[j] = xi[c];
                    vd[j] = dyi[c];
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + 32 * j;
                if (c < cpr) {
                    __stcs(xo + c, vx[j]);
                    __stcs(dyo + c, vd[j]);
                }
            }
        }
        // dH and ga: zero the padding rows (the SWIGLU epilogue writes the
        // others), the block's share of them
        const int64_t rem = (int64_t)end[tl.e] - r0;
        const int64_t valid = rem < 64 ? rem : 64;
        const int hc = a.h / 8;
        for (int64_t q = valid; q < 64; ++q) {
            uint4 *dh = reinterpret_cast<uint4 *>(a.dh + (pr0 + q) * 2 * a.h);
            uint4 *ga = reinterpret_cast<uint4 *>(a.ga + (pr0 + q) * a.h);
            for (int i = sl * blockDim.x + threadIdx.x; i < 3 * hc; i += S * blockDim.x) {
                if (i < 2 * hc) dh[i] = make_uint4(0, 0, 0, 0);
                else ga[i - 2 * hc] = make_uint4(0, 0, 0, 0);
            }
        }
    }
}

struct RouterBwdArgs {
    int64_t T;
    int E, k, norm_topk, score, ep;   // ep: row stride of dl
    const int32_t *ids;
    const float *gates, *probs, *dgate;
    const float *sg, *dsg;            // shared gate and its gradient (or null)
    __nv_bfloat16 *dl;                // [T, ep] out, zero past E
    float *dls;                       // [T] out: gradient of the shared gate's logit (or null)
};

// One warp per token.  q_j = s_{ids_j} are the kept raw scores; with
// renormalisation g_j = q_j / Q and dq_j = (dg_j - sum_i dg_i g_i) / Q, else
// dq_j = dg_j.  ds is dq on the kept experts and 0 elsewhere; softmax:
// dl_e = s_e (ds_e - sum_e' s_e' ds_e'), sigmoid: dl_e = ds_e s_e (1 - s_e).
__global__ void __launch_bounds__(256) router_bwd_kernel(RouterBwdArgs a) {
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * 8 + warp;
    if (t >= a.T) return;
    const float *s = a.probs + t * a.E;
    int id = -1;
    float dg = 0.f, g = 0.f, q = 0.f;
    if (lane < a.k) {
        id = a.ids[t * a.k + lane];
        if (id < 0 || id >= a.E) id = -1;
        dg = a.dgate[t * a.k + lane];
        g = a.gates[t * a.k + lane];
        q = id >= 0 ? s[id] : 0.f;
    }
    const float Q = warp_sum(q);
    const float dot = warp_sum(dg * g);
    const float dq = a.norm_topk ? (dg - dot) / Q : dg;
    const bool sigm = a.score == MOE_SCORE_SIGMOID;
    const float sd = sigm ? 0.f : warp_sum(id >= 0 ? q * dq : 0.f);   // sum_e s_e ds_e
    // every lane takes the k (id, dq) pairs (a uniform loop, so all lanes shuffle)
    int idj[MOE_MAX_TOPK];
    float dqj[MOE_MAX_TOPK];
#pragma unroll
    for (int j = 0; j < MOE_MAX_TOPK; ++j) {
        idj[j] = -1;
        dqj[j] = 0.f;
        if (j < a.k) {
            idj[j] = __shfl_sync(0xffffffffu, id, j);
            dqj[j] = __shfl_sync(0xffffffffu, dq, j);
        }
    }
    for (int e = lane; e < a.ep; e += 32) {
        float ds = 0.f;
#pragma unroll
        for (int j = 0; j < MOE_MAX_TOPK; ++j)
            if (idj[j] == e) ds = dqj[j];
        float dl = 0.f;
        if (e < a.E) dl = sigm ? ds * s[e] * (1.f - s[e]) : s[e] * (ds - sd);
        a.dl[t * a.ep + e] = __float2bfloat16_rn(dl);
    }
    if (lane == 0 && a.dls) a.dls[t] = a.dsg[t] * a.sg[t] * (1.f - a.sg[t]);
}

// dx[t, i] = bf16(acc[t, i] + dls[t] * w_s[i]) (the w_s term only with a
// shared expert), eight elements per thread step (d % 8 == 0): two 16-byte
// loads and one 16-byte store.
__global__ void finalize_dx_kernel(const float *acc, const float *dls, const __nv_bfloat16 *ws, __nv_bfloat16 *dx,
                                   int64_t T, int d) {
    pdl_wait();
    pdl_launch_dependents();
    const int cpr = d / 8;
    const int64_t chunks = T * cpr;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunks;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float4 a = *reinterpret_cast<const float4 *>(acc + 8 * i);
        const float4 b = *reinterpret_cast<const float4 *>(acc + 8 * i + 4);
        float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        if (dls) {
            const int64_t t = i / cpr;
            const int c = (int)(i - t * cpr) * 8;
            const float g = dls[t];
            float w[8];
            load8(ws + c, w);
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = fmaf(g, w[j], v[j]);
        }
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
            o[j] = *reinterpret_cast<uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(dx + 8 * i) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// dw_s[i] = sum over t of dls[t] * x[t, i], in a fixed order: a CTA takes 32
// columns (one per lane); warp w of its 32 sums the w-th 32nd of the tokens
// in increasing order, eight loads in flight at a time, and the 32 partial
// sums are added in warp order.
__global__ void __launch_bounds__(1024) shared_gate_grad_kernel(const float *dls, const __nv_bfloat16 *x, float *dws,
                                                                int64_t T, int d) {
    __shared__ float part[32][33];
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int i = blockIdx.x * 32 + lane;
    const int64_t per = (T + 31) / 32, t0 = warp * per, t1 = t0 + per < T ? t0 + per : T;
    float s = 0.f;
    if (i < d) {
        int64_t t = t0;
        for (; t + 8 <= t1; t += 8) {
            float xv[8], g[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                xv[u] = __bfloat162float(x[(t + u) * d + i]);
                g[u] = dls[t + u];
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) s = fmaf(g[u], xv[u], s);
        }
        for (; t < t1; ++t) s = fmaf(dls[t], __bfloat162float(x[t * d + i]), s);
    }
    part[warp][lane] = s;
    __syncthreads();
    if (warp == 0 && i < d) {
        float r = 0.f;
#pragma unroll
        for (int w = 0; w < 32; ++w) r += part[w][lane];
        dws[i] = r;
    }
}

cudaError_t set0(void *p, size_t bytes, cudaStream_t s) { return p && bytes ? cudaMemsetAsync(p, 0, bytes, s) : cudaSuccess; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_backward(const moe_config *c, const void *x, const void *w_router, const void *w_gate,
                                   const void *w_up, const void *w_down, const void *sh_gate, const void *sh_up,
                                   const void *sh_down, const void *w_shared_gate, const void *dy, void *ws,
                                   size_t ws_bytes, void *dx, float *dw_router, void *dw_gate, void *dw_up,
                                   void *dw_down, void *dsh_gate, void *dsh_up, void *dsh_down,
                                   float *dw_shared_gate, void *stream) {
    moe_status st = moe_validate(c);
    if (st != MOE_OK) return st;
    if (c->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (!dw_router || !dw_gate || !dw_up || !dw_down || !w_router || !w_gate || !w_up || !w_down)
        return MOE_ERR_INVALID_ARG;
    const bool shared = c->h_shared > 0;
    if (shared && (!sh_gate || !sh_up || !sh_down || !w_shared_gate || !dsh_gate || !dsh_up || !dsh_down ||
                   !dw_shared_gate))
        return MOE_ERR_INVALID_ARG;
    if (c->T > 0 && (!x || !dy || !dx)) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*c, true);
    if (c->T > 0 && (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255))) return MOE_ERR_WORKSPACE;
    uint32_t *err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t T = c->T, R = T * c->k;
    const int d = c->d, E = c->E, h = c->h, hs = c->h_shared, ep = dl_stride(E);
    if (T == 0) {
        // no tokens: every weight gradient is zero
        cudaError_t e = set0(dw_router, sizeof(float) * (size_t)E * d, s);
        if (e == cudaSuccess) e = set0(dw_gate, 2 * (size_t)E * h * d, s);
        if (e == cudaSuccess) e = set0(dw_up, 2 * (size_t)E * h * d, s);
        if (e == cudaSuccess) e = set0(dw_down, 2 * (size_t)E * d * h, s);
        if (shared) {
            if (e == cudaSuccess) e = set0(dsh_gate, 2 * (size_t)hs * d, s);
            if (e == cudaSuccess) e = set0(dsh_up, 2 * (size_t)hs * d, s);
            if (e == cudaSuccess) e = set0(dsh_down, 2 * (size_t)d * hs, s);
            if (e == cudaSuccess) e = set0(dw_shared_gate, sizeof(float) * d, s);
        }
        return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    }

    const int32_t *ids = ws_part<int32_t>(ws, L, P_IDS);
    const float *gates = ws_part<float>(ws, L, P_GATES);
    const float *sg = ws_part<float>(ws, L, P_SG);
    const int32_t *offsets = ws_part<int32_t>(ws, L, P_OFFSETS);
    const int32_t *srt = ws_part<int32_t>(ws, L, P_SORTED);
    const float *probs = ws_part<float>(ws, L, P_PROBS);
    char *hpre = ws_part<char>(ws, L, P_HPRE);
    char *hpres = ws_part<char>(ws, L, P_HPRES);
    float *dg = ws_part<float>(ws, L, P_DG);
    float *dsg = ws_part<float>(ws, L, P_DSG);
    char *dh = ws_part<char>(ws, L, P_DH);
    char *dhs = ws_part<char>(ws, L, P_DHS);
    void *ga = ws_part<void>(ws, L, P_GA);       // gate * a of the routed rows, padded layout
    void *xg = ws_part<void>(ws, L, P_XG);       // x and dy rows in the padded grouped layout
    void *dyg = ws_part<void>(ws, L, P_DYG);
    const uint64_t Rp = (uint64_t)padded_rows(R, E);
    void *gas = ws_part<void>(ws, L, P_GAS);
    void *dlb = ws_part<void>(ws, L, P_DLB);
    float *dls = ws_part<float>(ws, L, P_DLS);
    float *acc = ws_part<float>(ws, L, P_YACC);  // the dx accumulator

    cudaError_t e = set0(dg, sizeof(float) * R, s);
    if (e == cudaSuccess) e = set0(dsg, shared ? sizeof(float) * T : 0, s);
    if (e == cudaSuccess) e = set0(acc, sizeof(float) * T * d, s);

    auto base = [](const BwdGemm::Kind kind) {
        BwdGemm g{};
        g.kind = kind;
        return g;
    };
    // 0. x and dy rows into the padded grouped layout; zero padding rows
    if (e == cudaSuccess) {
        GatherPadArgs a{static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(dy), offsets, srt,
                        E, c->k, d, h, T, R, static_cast<__nv_bfloat16 *>(xg), static_cast<__nv_bfloat16 *>(dyg),
                        reinterpret_cast<__nv_bfloat16 *>(dh), static_cast<__nv_bfloat16 *>(ga), err};
        // one CTA per 64-row block and slice of 1024 columns, so that enough
        // copies are in flight for HBM (at most 32 CTAs per SM, grid-strided)
        const int64_t slices = ((int64_t)d / 8 + 127) / 128;
        const unsigned blocks = (unsigned)std::min<int64_t>((int64_t)(Rp / 64) * slices, 32LL * num_sms());
        e = launch_kernel(gather_pad_kernel, std::max(1u, blocks), 256, 0, s, a);
    }
    // 1. routed: r = W_down^T dy over grouped rows
    if (e == cudaSuccess) {
        BwdGemm g = base(BwdGemm::SWIGLU);
        g.padded = true;
        g.a0 = {dyg, Rp, (uint64_t)d, (uint64_t)d};
        g.b0 = {w_down, (uint64_t)E * d, (uint64_t)h, (uint64_t)h};
        g.offsets = offsets;
        g.sorted_rows = srt;
        g.groups = E;
        g.k = c->k;
        g.rows = R;
        g.T = T;
        g.nranges = 1;
        g.Kr = d;
        g.N = h;
        g.hpre = hpre;
        g.gate = gates;
        g.dh = dh;
        g.ga = ga;
        g.dgate = dg;
        g.err = err;
        e = launch_bwd_gemm(g, s);
    }
    // 2. shared expert: the same on the dense segment (gate sigmoid(w_s . x))
    if (e == cudaSuccess && shared) {
        BwdGemm g = base(BwdGemm::SWIGLU);
        g.a0 = {dy, (uint64_t)T, (uint64_t)d, (uint64_t)d};
        g.b0 = {sh_down, (uint64_t)d, (uint64_t)hs, (uint64_t)hs};
        g.groups = 1;
        g.k = 1;
        g.rows = T;
        g.T = T;
        g.nranges = 1;
        g.Kr = d;
        g.N = hs;
        g.hpre = hpres;
        g.gate = sg;
        g.dh = dhs;
        g.ga = gas;
        g.dgate = dsg;
        g.err = err;
        e = launch_bwd_gemm(g, s);
    }
    // 3. router: gate gradients -> logit gradients
    if (e == cudaSuccess) {
        RouterBwdArgs a{T, E, c->k, c->norm_topk, c->score, ep, ids, gates, probs, dg, shared ? sg : nullptr,
                        shared ? dsg : nullptr, static_cast<__nv_bfloat16 *>(dlb), shared ? dls : nullptr};
        e = launch_kernel(router_bwd_kernel, (unsigned)((T + 7) / 8), 256, 0, s, a);
    }
    // 4. dx: the routed experts' gate/up (two K ranges: du with W_gate, dv with W_up), the shared expert's,
    //    and the router's
    if (e == cudaSuccess) {
        BwdGemm g = base(BwdGemm::SCATTER);
        g.padded = true;
        g.a0 = {dh, Rp, (uint64_t)h, 2 * (uint64_t)h};
        g.a1 = {dh + (size_t)h * 2, Rp, (uint64_t)h, 2 * (uint64_t)h};
        g.b0 = {w_gate, (uint64_t)E * h, (uint64_t)d, (uint64_t)d};
        g.b1 = {w_up, (uint64_t)E * h, (uint64_t)d, (uint64_t)d};
        g.offsets = offsets;
        g.sorted_rows = srt;
        g.groups = E;
        g.k = c->k;
        g.rows = R;
        g.T = T;
        g.nranges = 2;
        g.Kr = h;
        g.N = d;
        g.acc = acc;
        g.err = err;
        e = launch_bwd_gemm(g, s);
    }
    if (e == cudaSuccess && shared) {
        BwdGemm g = base(BwdGemm::SCATTER);
        g.a0 = {dhs, (uint64_t)T, (uint64_t)hs, 2 * (uint64_t)hs};
        g.a1 = {dhs + (size_t)hs * 2, (uint64_t)T, (uint64_t)hs, 2 * (uint64_t)hs};
        g.b0 = {sh_gate, (uint64_t)hs, (uint64_t)d, (uint64_t)d};
        g.b1 = {sh_up, (uint64_t)hs, (uint64_t)d, (uint64_t)d};
        g.groups = 1;
        g.k = 1;
        g.rows = T;
        g.T = T;
        g.nranges = 2;
        g.Kr = hs;
        g.N = d;
        g.acc = acc;
        g.err = err;
        e = launch_bwd_gemm(g, s);
    }
    if (e == cudaSuccess) {
        BwdGemm g = base(BwdGemm::SCATTER);
        g.a0 = {dlb, (uint64_t)T, (uint64_t)E, (uint64_t)ep};
        g.b0 = {w_router, (uint64_t)E, (uint64_t)d, (uint64_t)d};
        g.groups = 1;
        g.k = 1;
        g.rows = T;
        g.T = T;
        g.nranges = 1;
        g.Kr = E;
        g.N = d;
        g.acc = acc;
        g.err = err;
        e = launch_bwd_gemm(g, s);
    }
    if (e == cudaSuccess) {
        const int64_t n = T * (d / 8);
        const unsigned blocks = (unsigned)std::min<int64_t>((n + 255) / 256, 4LL * num_sms() * 8);
        e = launch_kernel(finalize_dx_kernel, blocks, 256, 0, s, static_cast<const float *>(acc),
                          static_cast<const float *>(shared ? dls : nullptr),
                          static_cast<const __nv_bfloat16 *>(shared ? w_shared_gate : nullptr),
                          static_cast<__nv_bfloat16 *>(dx), T, d);
    }
    // 5. weight gradients
    if (e == cudaSuccess) {
        // dW_down[e] = sum over the expert's rows of dy_t (x) (gate * a)
        BwdGemm g = base(BwdGemm::WEIGHT);
        g.padded = true;
        g.a0 = {dyg, Rp, (uint64_t)d, (uint64_t)d};
        g.b0 = {ga, Rp, (uint64_t)h, (uint64_t)h};
        g.offsets = offsets;
        g.sorted_rows = srt;
        g.groups = E;
        g.k = c->k;
        g.rows = R;
        g.T = T;
        g.M = d;
        g.halves = 1;
        g.N = h;
        g.out0 = dw_down;
        g.err = err;
        e = launch_bwd_gemm(g, s);
    }
    if (e == cudaSuccess) {
        // dW_gate[e] / dW_up[e] = sum over the expert's rows of du / dv (x) x_t
        BwdGemm g = base(BwdGemm::WEIGHT);
        g.padded = true;
        g.a0 = {dh, Rp, (uint64_t)h, 2 * (uint64_t)h};
        g.a1 = {dh + (size_t)h * 2, Rp, (uint64_t)h, 2 * (uint64_t)h};
        g.b0 = {xg, Rp, (uint64_t)d, (uint64_t)d};
        g.offsets = offsets;
        g.sorted_rows = srt;
        g.groups = E;
        g.k = c->k;
        g.rows = R;
        g.T = T;
        g.M = h;
        g.halves = 2;
        g.N = d;
        g.out0 = dw_gate;
        g.out1 = dw_up;
        g.err = err;
        e = launch_bwd_gemm(g, s);
    }
    if (e == cudaSuccess && shared) {
        BwdGemm g = base(BwdGemm::WEIGHT);
        g.a0 = {dy, (uint64_t)T, (uint64_t)d, (uint64_t)d};
        g.b0 = {gas, (uint64_t)T, (uint64_t)hs, (uint64_t)hs};
        g.groups = 1;
        g.k = 1;
        g.rows = T;
        g.T = T;
        g.M = d;
        g.halves = 1;
        g.N = hs;
        g.out0 = dsh_down;
        g.err = err;
        e = launch_bwd_gemm(g, s);
    }
    if (e == cudaSuccess && shared) {
        BwdGemm g = base(BwdGemm::WEIGHT);
        g.a0 = {dhs, (uint64_t)T, (uint64_t)hs, 2 * (uint64_t)hs};
        g.a1 = {dhs + (size_t)hs * 2, (uint64_t)T, (uint64_t)hs, 2 * (uint64_t)hs};
        g.b0 = {x, (uint64_t)T, (uint64_t)d, (uint64_t)d};
        g.groups = 1;
        g.k = 1;
        g.rows = T;
        g.T = T;
        g.M = hs;
        g.halves = 2;
        g.N = d;
        g.out0 = dsh_gate;
        g.out1 = dsh_up;
        g.err = err;
        e = launch_bwd_gemm(g, s);
    }
    if (e == cudaSuccess) {
        // dW_router = dl^T x
        BwdGemm g = base(BwdGemm::WEIGHT);
        g.a0 = {dlb, (uint64_t)T, (uint64_t)E, (uint64_t)ep};
        g.b0 = {x, (uint64_t)T, (uint64_t)d, (uint64_t)d};
        g.groups = 1;
        g.k = 1;
        g.rows = T;
        g.T = T;
        g.M = E;
        g.halves = 1;
        g.N = d;
        g.out0 = dw_router;
        g.out_f32 = true;
        g.err = err;
        e = launch_bwd_gemm(g, s);
    }
    if (e == cudaSuccess && shared)
        e = launch_kernel(shared_gate_grad_kernel, (unsigned)((d + 31) / 32), 1024, 0, s,
                          static_cast<const float *>(dls), static_cast<const __nv_bfloat16 *>(x), dw_shared_gate, T, d);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
