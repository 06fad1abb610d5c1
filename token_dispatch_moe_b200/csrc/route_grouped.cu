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

// ---------------------------------------------------------------- quad path --
// Rows of whole 16-expert chunks, groups of whole chunks, k_per_group and
// k_max <= 8: four lanes (a quad) route one row, a warp 8 rows at a time.  Lane
// j reads, in each chunk c of its row, the 4-expert vector 16c + 4j (float4
// loads; a quad reads 64 contiguous bytes).  Per group every lane keeps its P1
// best words with an insertion network; two shuffle rounds merge the quad's
// lists into the group's k_per_group best, which are the group's candidates
// (words are unique, so "fewer than k_per_group better words in the group" is
// "among its k_per_group best").  Lane g % 4 feeds group g's candidates into
// its list of the P2 best; two more shuffle rounds give the row's k_max picks.
// The words are the same 64-bit words as above, so the selection, NaN's last
// place and the lower-id rule on equal keys are the same.
constexpr int kGqThreads = 256;

template <int P>
__device__ __forceinline__ void gq_insert(uint64_t (&L)[P], uint64_t v) {
#pragma unroll
    for (int p = 0; p < P; ++p) {
        const uint64_t hi = L[p] > v ? L[p] : v;
        v = L[p] > v ? v : L[p];
        L[p] = hi;
    }
}

// Both lanes end with the P best words of their two lists, in descending order.
template <int P>
__device__ __forceinline__ void gq_merge(uint64_t (&L)[P], int mask) {
    uint64_t B[P];
#pragma unroll
    for (int p = 0; p < P; ++p) B[p] = __shfl_xor_sync(MOE_FULL_MASK, L[P - 1 - p], mask);
#pragma unroll
    for (int p = 0; p < P; ++p) L[p] = L[p] > B[p] ? L[p] : B[p];  // a bitonic sequence
#pragma unroll
    for (int st = P / 2; st >= 1; st >>= 1)
#pragma unroll
        for (int i = 0; i < P; ++i)
            if ((i & st) == 0) {
                const uint64_t hi = L[i] > L[i + st] ? L[i] : L[i + st];
                const uint64_t lo = L[i] > L[i + st] ? L[i + st] : L[i];
                L[i] = hi;
                L[i + st] = lo;
            }
}

__device__ __forceinline__ float gq_max(float v) {
    v = fmaxf(v, __shfl_xor_sync(MOE_FULL_MASK, v, 1));
    return fmaxf(v, __shfl_xor_sync(MOE_FULL_MASK, v, 2));
}
__device__ __forceinline__ float gq_sum(float v) {
    v += __shfl_xor_sync(MOE_FULL_MASK, v, 1);
    return v + __shfl_xor_sync(MOE_FULL_MASK, v, 2);
}

template <int P1, int P2>
__global__ void __launch_bounds__(kGqThreads)
    route_grouped_quad_kernel(const float *__restrict__ logits, int64_t T, int E, int k_max,
                              int score, int G, int kpg, int renorm, float scale,
                              int32_t *__restrict__ ids, float *__restrict__ wout,
                              int32_t *status) {
    const int lane = threadIdx.x & 31, j = lane & 3;
    const int cpg = E / G / 16;  // chunks a group
    const int64_t step = (int64_t)gridDim.x * (kGqThreads / 4);
    for (int64_t base = (int64_t)blockIdx.x * (kGqThreads / 4) + (threadIdx.x >> 5) * 8; base < T;
         base += step) {
        const int64_t row = base + (lane >> 2);
        const bool valid = row < T;
        const float *src = logits + (valid ? row : 0) * E;
        auto vec = [&](int c) -> float4 {
            return valid ? __ldg(reinterpret_cast<const float4 *>(src + 16 * c + 4 * j))
                         : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        };
        // Softmax over the whole row needs its max and denominator.
        float m = -INFINITY, z = 0.0f;
        bool nan = false;
        if (score == MOE_SCORE_SOFTMAX) {
            for (int c = 0; c < E / 16; ++c) {
                const float4 v = vec(c);
                m = fmaxf(fmaxf(m, v.x), fmaxf(v.y, fmaxf(v.z, v.w)));
            }
            m = gq_max(m);
            for (int c = 0; c < E / 16; ++c) {
                const float4 v = vec(c);
                z += expf(v.x - m) + expf(v.y - m) + expf(v.z - m) + expf(v.w - m);
            }
            z = gq_sum(z);
        }
        // Candidates of each group, then the row's picks.
        uint64_t R[P2];
#pragma unroll
        for (int p = 0; p < P2; ++p) R[p] = 0ull;
        for (int g = 0; g < G; ++g) {
            uint64_t L[P1];
#pragma unroll
            for (int p = 0; p < P1; ++p) L[p] = 0ull;
            for (int cc = 0; cc < cpg; ++cc) {
                const int c = g * cpg + cc;
                const int e0 = 16 * c + 4 * j;
                const float4 v = vec(c);
                nan |= (v.x != v.x) | (v.y != v.y) | (v.z != v.z) | (v.w != v.w);
                if (valid) {
                    gq_insert<P1>(L, sel_word(v.x, e0));
                    gq_insert<P1>(L, sel_word(v.y, e0 + 1));
                    gq_insert<P1>(L, sel_word(v.z, e0 + 2));
                    gq_insert<P1>(L, sel_word(v.w, e0 + 3));
                }
            }
            gq_merge<P1>(L, 1);
            gq_merge<P1>(L, 2);
            if ((g & 3) == j) {
#pragma unroll
                for (int p = 0; p < P1; ++p)
                    if (p < kpg) gq_insert<P2>(R, L[p]);
            }
        }
        gq_merge<P2>(R, 1);
        gq_merge<P2>(R, 2);
        nan = gq_sum(nan ? 1.0f : 0.0f) > 0.0f;
        if (valid && nan && j == 0) report(status, MOE_ERR_NAN_LOGIT);

        // Weights of the picks: lane j takes slots j and j + 4.
        constexpr int NS = (P2 + 3) / 4;
        int pid[NS];
        float pl[NS], v[NS];
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const int sl = j + 4 * i;
            uint64_t w = 0ull;
#pragma unroll
            for (int p = 0; p < P2; ++p)
                if (p == sl) w = R[p];
            pid[i] = (valid && sl < k_max && (w >> 32) != 0ull) ? (int)(0xffffffffu - (uint32_t)w)
                                                                  : -1;
            pl[i] = pid[i] >= 0 ? __ldg(src + pid[i]) : 0.0f;
        }
        float ms = -INFINITY;
        if (score == MOE_SCORE_TOPK_SOFTMAX) {
#pragma unroll
            for (int i = 0; i < NS; ++i)
                if (pid[i] >= 0) ms = fmaxf(ms, pl[i]);
            ms = gq_max(ms);
        }
        float part = 0.0f;
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            float x = 0.0f;
            if (pid[i] >= 0) {
                if (score == MOE_SCORE_TOPK_SOFTMAX)
                    x = expf(pl[i] - ms);
                else if (score == MOE_SCORE_SOFTMAX)
                    x = expf(pl[i] - m) / z;
                else if (score == MOE_SCORE_SIGMOID)
                    x = sigmoid_score(pl[i]);
                else
                    x = sqrt_softplus_score(pl[i]);
            }
            v[i] = x;
            part += x;
        }
        const float sum = gq_sum(part);
        if (valid) {
#pragma unroll
            for (int i = 0; i < NS; ++i) {
                const int sl = j + 4 * i;
                if (sl < k_max) {
                    float x = v[i];
                    if (renorm || score == MOE_SCORE_TOPK_SOFTMAX) x = sum > 0.0f ? x / sum : x;
                    ids[row * k_max + sl] = pid[i];
                    wout[row * k_max + sl] = pid[i] >= 0 ? x * scale : 0.0f;
                }
            }
        }
    }
}

template <int P1>
void *gq_fn_p(int P2) {
    switch (P2) {
        case 1: return (void *)route_grouped_quad_kernel<P1, 1>;
        case 2: return (void *)route_grouped_quad_kernel<P1, 2>;
        case 4: return (void *)route_grouped_quad_kernel<P1, 4>;
        default: return (void *)route_grouped_quad_kernel<P1, 8>;
    }
}

void *gq_fn(int P1, int P2) {
    switch (P1) {
        case 1: return gq_fn_p<1>(P2);
        case 2: return gq_fn_p<2>(P2);
        case 4: return gq_fn_p<4>(P2);
        default: return gq_fn_p<8>(P2);
    }
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
    if (E % 16 == 0 && (E / G) % 16 == 0 && k <= 8 && k_per_group <= 8 && aligned16(logits)) {
        int P1 = 1, P2 = 1;
        while (P1 < k_per_group) P1 *= 2;
        while (P2 < k) P2 *= 2;
        void *fn = gq_fn(P1, P2);
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kGqThreads, 0) !=
                cudaSuccess ||
            per_sm < 1) {
            cudaGetLastError();
            per_sm = 1;
        }
        const int64_t need = (T + kGqThreads / 4 - 1) / (kGqThreads / 4);
        const int64_t cap = (int64_t)sm_count() * per_sm;
        const unsigned grid = (unsigned)(need < cap ? need : cap);
        int score = p->score, kk = k, kp = k_per_group;
        float sc = p->route_scale;
        void *args[] = {&logits, &T, (void *)&E, &kk, &score, (void *)&G, &kp, (void *)&renorm, &sc,
                        &topk_ids, &topk_w, &d_status};
        if (cudaLaunchKernel(fn, dim3(grid), dim3(kGqThreads), args, 0, s) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        return launch_status();
    }
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
