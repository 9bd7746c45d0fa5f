// Load-balancing machinery of the routing step, for training:
//
//  * router_stats_kernel: P_e, the mean score of expert e over the T tokens,
//    from the per-CTA partial rows the routers write (rows added in a fixed
//    order, so the result is bit-identical from call to call);
//  * update_bias_kernel: the auxiliary-loss-free balance bias after a step,
//    bias_e += lr * sign(mean load - load_e), from the per-expert counts of
//    the grouping step;
//  * balance_loss_kernel: the Switch load-balancing term
//    alpha * E * sum_e f_e * P_e with f_e = counts_e / T.
//
// "Small MoE Architecture, in depth", section "A small MoE layer in PyTorch"
// (SmallMoE.forward: the balance bias is added to the scores only to choose
// the top k; in training the load is the bincount of the chosen ids and the
// bias moves by bias_lr * sign(mean load - load)) and the paragraph on
// auxiliary-loss-free balancing after it; "Mixture-of-Experts -- more capacity
// per byte of weight", section "What's wired today" (the auxiliary loss
// alpha * N * sum_e f_e * P_e, the Switch recipe).
//
// All three are single-pass, allocation-free and stream-ordered; none waits
// on another CTA.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kStatCols = 32;    // experts per CTA of the statistic
constexpr int kStatPhases = 32;  // row phases per CTA

// score_mean[e] = (sum over rows r of partial[r, e]) / T.  CTA b owns experts
// 32b .. 32b + 31; thread (phase p, column c) adds rows p, p + 32, ... of its
// column in increasing order (each warp reads 128 contiguous bytes per row),
// then the 32 phase sums of a column are added in phase order.
__global__ void __launch_bounds__(kStatCols * kStatPhases)
    router_stats_kernel(const float *partial, int64_t rows, int E, int64_t T, float *score_mean) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ float part[kStatPhases][kStatCols + 1];
    const int c = threadIdx.x & (kStatCols - 1), ph = threadIdx.x / kStatCols;
    const int e = blockIdx.x * kStatCols + c;
    float v = 0.f;
    if (e < E) {
#pragma unroll 4
        for (int64_t r = ph; r < rows; r += kStatPhases) v += partial[r * E + e];
    }
    part[ph][c] = v;
    __syncthreads();
    if (ph == 0 && e < E) {
        float s = 0.f;
        for (int p = 0; p < kStatPhases; ++p) s += part[p][c];
        score_mean[e] = T > 0 ? __fdiv_rn(s, (float)T) : 0.f;
    }
}

// One CTA of MOE_MAX_EXPERTS threads.  The mean load is compared exactly in
// integers: mean > load_e  <=>  sum(counts) > E * load_e.
__global__ void __launch_bounds__(MOE_MAX_EXPERTS) update_bias_kernel(const int32_t *counts, int E, float lr,
                                                                        float *bias) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ long long wsum[MOE_MAX_EXPERTS / 32];
    const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
    const long long load = e < E ? (long long)counts[e] : 0;
    long long s = load;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) wsum[warp] = s;
    __syncthreads();
    long long total = 0;
    for (int w = 0; w < MOE_MAX_EXPERTS / 32; ++w) total += wsum[w];
    if (e < E) {
        const long long scaled = (long long)E * load;
        const float sign = total > scaled ? 1.f : (total < scaled ? -1.f : 0.f);
        bias[e] = __fadd_rn(bias[e], __fmul_rn(lr, sign));
    }
}

// One CTA of MOE_MAX_EXPERTS threads: f_e = counts_e / T, and the sum of
// f_e * P_e by a fixed shared-memory tree, times alpha * E.
__global__ void __launch_bounds__(MOE_MAX_EXPERTS)
    balance_loss_kernel(const int32_t *counts, const float *score_mean, int E, int64_t T, float alpha, float *frac,
                        float *loss) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ float prod[MOE_MAX_EXPERTS];
    const int e = threadIdx.x;
    float f = 0.f;
    if (e < E && T > 0) f = __fdiv_rn((float)counts[e], (float)T);
    if (e < E && frac) frac[e] = f;
    prod[e] = e < E ? __fmul_rn(f, score_mean[e]) : 0.f;
    __syncthreads();
    for (int half = MOE_MAX_EXPERTS / 2; half > 0; half >>= 1) {
        if (e < half) prod[e] = __fadd_rn(prod[e], prod[e + half]);
        __syncthreads();
    }
    if (e == 0) *loss = __fmul_rn(__fmul_rn(alpha, (float)E), prod[0]);
}

}  // namespace

cudaError_t launch_router_stats(const float *partial, int64_t rows, int E, int64_t T, float *score_mean,
                                cudaStream_t s) {
    const unsigned grid = (unsigned)((E + kStatCols - 1) / kStatCols);
    return launch_kernel(router_stats_kernel, grid, kStatCols * kStatPhases, 0, s, partial, rows, E, T, score_mean);
}

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_update_bias(const moe_config *c, const int32_t *counts, float lr, float *bias,
                                      void *stream) {
    const moe_status st = moe_validate(c);
    if (st != MOE_OK) return st;
    if (!counts || !bias || !(lr == lr) || lr - lr != 0.f) return MOE_ERR_INVALID_ARG;   // null or lr not finite
    const cudaError_t e = launch_kernel(update_bias_kernel, 1, MOE_MAX_EXPERTS, 0, static_cast<cudaStream_t>(stream),
                                        counts, c->E, lr, bias);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status moe_balance_loss(const moe_config *c, const int32_t *counts, const float *score_mean,
                                       float alpha, float *frac, float *loss, void *stream) {
    const moe_status st = moe_validate(c);
    if (st != MOE_OK) return st;
    if (!counts || !score_mean || !loss || !(alpha == alpha) || alpha - alpha != 0.f) return MOE_ERR_INVALID_ARG;
    const cudaError_t e = launch_kernel(balance_loss_kernel, 1, MOE_MAX_EXPERTS, 0, static_cast<cudaStream_t>(stream),
                                        counts, score_mean, c->E, c->T, alpha, frac, loss);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
