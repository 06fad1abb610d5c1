// moe_route_grouped: per-group candidates, then a global top-k ("Crate
// ferrox_moe", Functions, route_top_k_grouped).
//
// Definition: the E experts form n_groups contiguous groups; each group keeps
// its k_per_group best experts by score; of those candidates, the k_max best
// are selected, in descending score order, ties to the lower id; weights as
// moe_route (unbiased score, renormalise, route_scale; gpt-oss: softmax over
// the selected logits).  Every score function is monotone in the logit, so
// ranking by score is ranking by logit, and the kernel ranks fp32 logits
// exactly.
//
// B200 design: one warp per token row, lane l holding experts l, l+32, ...
// (coalesced 128-byte loads).  Each expert's rank inside its group is counted
// against the row's 64-bit selection words staged in shared memory (word =
// order-preserving image of the logit above a descending id, so words are
// unique and a larger word is the better expert); the final choice is k_max
// rounds of a two-step warp max (redux.sync on the high, then the low half).
#include "common.cuh"

namespace moe {
namespace {

constexpr int kGrWarps = 8;
constexpr int kGrMaxE = 512;

__device__ __forceinline__ uint64_t sel_word(float l, int e) {
    return ((uint64_t)order_key(l) << 32) | (uint64_t)(0xffffffffu - (uint32_t)e);
}

template <int VPL>
__global__ void __launch_bounds__(kGrWarps * 32)
    route_grouped_kernel(const float *__restrict__ logits, int64_t T, int E, int k_max, int score,
                         int G, int kpg, int renorm, float scale, int32_t *__restrict__ ids,
                         float *__restrict__ wout, int32_t *status) {
    __shared__ uint64_t words[kGrWarps][kGrMaxE];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t *sw = words[warp];
    const int gsz = E / G;
    const int64_t nw = (int64_t)gridDim.x * kGrWarps;
    bool nan = false;
    for (int64_t t = (int64_t)blockIdx.x * kGrWarps + warp; t < T; t += nw) {
        const float *row = logits + t * E;
        float l[VPL];
        uint64_t wd[VPL];
        float m = -INFINITY;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int e = i * 32 + lane;
            l[i] = e < E ? ld_stream(row + e) : -INFINITY;
            wd[i] = e < E ? sel_word(l[i], e) : 0ull;
            if (e < E) {
                nan |= l[i] != l[i];
                m = fmaxf(m, l[i]);
            }
        }
        __syncwarp();  // the previous row's readers are done with sw
#pragma unroll
        for (int i = 0; i < VPL; ++i)
            if (i * 32 + lane < E) sw[i * 32 + lane] = wd[i];
        __syncwarp();
        // Candidates: rank inside the group below k_per_group.
        if (kpg < gsz) {
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int e = i * 32 + lane;
                if (e >= E) continue;
                const int g0 = (e / gsz) * gsz;
                int rank = 0;
                for (int q = 0; q < gsz && rank < kpg; ++q) rank += sw[g0 + q] > wd[i] ? 1 : 0;
                if (rank >= kpg) wd[i] = 0ull;
            }
        }
        // Softmax over the whole row needs its max and denominator.
        float z = 0.0f;
        if (score == MOE_SCORE_SOFTMAX) {
            m = warp_max(m);
#pragma unroll
            for (int i = 0; i < VPL; ++i)
                if (i * 32 + lane < E) z += expf(l[i] - m);
            z = warp_sum(z);
        }
        // k_max rounds of the warp-wide best word; lane j keeps pick j.
        int my_id = -1;
        float my_l = 0.0f;
        for (int j = 0; j < k_max; ++j) {
            uint64_t best = 0ull;
#pragma unroll
            for (int i = 0; i < VPL; ++i) best = wd[i] > best ? wd[i] : best;
            const uint32_t hi = __reduce_max_sync(MOE_FULL_MASK, (uint32_t)(best >> 32));
            const uint32_t lo = __reduce_max_sync(
                MOE_FULL_MASK, (uint32_t)(best >> 32) == hi ? (uint32_t)best : 0u);
            if (hi == 0u) break;  // no candidate left (cannot happen when k_max <= G*kpg)
            const int e = (int)(0xffffffffu - lo);
            float le = 0.0f;
#pragma unroll
            for (int i = 0; i < VPL; ++i)
                if (i * 32 + lane == e) {
                    le = l[i];
                    wd[i] = 0ull;
                }
            le = __shfl_sync(MOE_FULL_MASK, le, e & 31);
            if (lane == j) {
                my_id = e;
                my_l = le;
            }
        }
        // Weights of the picks (lanes < k_max).
        const bool act = my_id >= 0;
        float v = 0.0f;
        if (score == MOE_SCORE_TOPK_SOFTMAX) {
            const float ms = warp_max(act ? my_l : -INFINITY);
            v = act ? expf(my_l - ms) : 0.0f;
        } else if (act) {
            if (score == MOE_SCORE_SOFTMAX)
                v = expf(my_l - m) / z;
            else if (score == MOE_SCORE_SIGMOID)
                v = sigmoid_score(my_l);
            else
                v = sqrt_softplus_score(my_l);
        }
        const float sum = warp_sum(v);
        if (renorm || score == MOE_SCORE_TOPK_SOFTMAX) v = sum > 0.0f ? v / sum : v;
        if (lane < k_max) {
            ids[t * k_max + lane] = my_id;
            wout[t * k_max + lane] = act ? v * scale : 0.0f;
        }
    }
    if (nan) report(status, MOE_ERR_NAN_LOGIT);
}

template <int VPL>
void launch_grouped(const float *logits, int64_t T, int E, int k_max, int score, int G, int kpg,
                    int renorm, float scale, int32_t *ids, float *w, int32_t *status,
                    cudaStream_t s) {
    int64_t blocks = (T + kGrWarps - 1) / kGrWarps;
    const int64_t most = (int64_t)sm_count() * 6;
    blocks = blocks < most ? blocks : most;
    route_grouped_kernel<VPL><<<(unsigned)blocks, kGrWarps * 32, 0, s>>>(
        logits, T, E, k_max, score, G, kpg, renorm, scale, ids, w, status);
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_route_grouped(const float *logits, const moe_route_params *p,
                                        int32_t k_per_group, int64_t T, int32_t *topk_ids,
                                        float *topk_w, int32_t *d_status, moe_stream_t stream) {
    using namespace moe;
    if (!p || T < 0) return MOE_ERR_INVALID_ARG;
    const int E = p->num_experts, G = p->n_groups, k = p->k_max;
    if (E < 1 || E > kGrMaxE || G < 1 || E % G != 0 || k_per_group < 1 || k_per_group > E / G ||
        k < 0 || k > 32 || (int64_t)k > (int64_t)G * k_per_group)
        return MOE_ERR_INVALID_ARG;
    if (p->score < MOE_SCORE_SOFTMAX || p->score > MOE_SCORE_TOPK_SOFTMAX)
        return MOE_ERR_INVALID_ARG;
    if (T == 0 || k == 0) return MOE_OK;
    if (!logits || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
    if (T * (int64_t)E >= ((int64_t)1 << 40)) return MOE_ERR_UNSUPPORTED;
    const int renorm = p->renormalize ? 1 : 0;
    cudaStream_t s = as_cuda(stream);
    if (E <= 64)
        launch_grouped<2>(logits, T, E, k, p->score, G, k_per_group, renorm, p->route_scale,
                          topk_ids, topk_w, d_status, s);
    else if (E <= 128)
        launch_grouped<4>(logits, T, E, k, p->score, G, k_per_group, renorm, p->route_scale,
                          topk_ids, topk_w, d_status, s);
    else if (E <= 256)
        launch_grouped<8>(logits, T, E, k, p->score, G, k_per_group, renorm, p->route_scale,
                          topk_ids, topk_w, d_status, s);
    else
        launch_grouped<16>(logits, T, E, k, p->score, G, k_per_group, renorm, p->route_scale,
                           topk_ids, topk_w, d_status, s);
    return launch_status();
}
