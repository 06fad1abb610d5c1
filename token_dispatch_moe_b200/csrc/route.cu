// moe_route and moe_hash_route: scoring, selection-only bias, group limit,
// per-token top-k and weights, one warp per token row, in one pass.
//
// Method ("DeepSeek-V3.2-Exp - Select experts", Explanation and gate forward;
// "Crate ferrox_moe", route_top_k_* and route_hash; "Feature Request: dynamic
// number of experts", k per request):
//   key_e = score(l_e) + bias_e; group score = sum of the group_topn largest
//   keys of each contiguous group; keep topk_groups groups; take the k_t
//   largest keys (equal keys -> lower id); weight = unbiased score, optionally
//   renormalised, times route_scale.
//
// B200 design: a row of E <= 512 fp32 logits is spread over the 32 lanes of a
// warp (128-bit loads when E % 4 == 0: lane l holds experts 128c + 4l .. +3 of
// chunk c).  Selection keys are order-preserving uint32 images of the fp32
// keys, so a round of top-k is two single-instruction warp reductions
// (redux.sync max over keys, min over the ids that hold the max).  When no
// bias is given and the group score is an amax, every score function is
// monotone in the logit, so selection runs on the raw logits and only the k
// selected experts are ever scored.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kRouteWarps = 8;  // warps per block
constexpr int kMaxE = 512;

struct RouteArgs {
    const float *logits;
    const float *bias;
    const int32_t *kpt;
    int32_t *ids;
    float *w;
    int32_t *status;
    int64_t T;
    int E, k_max, score, G, TG, topn, renorm;
    float scale;
    int gsz, lpg, strip;      // group size, lanes per group, experts per lane strip
    int keys_from_scores;     // 0: select on the logit (monotone case)
};

template <bool VEC>
__device__ __forceinline__ int slot_expert(int s, int lane) {
    return VEC ? (s >> 2) * 128 + lane * 4 + (s & 3) : s * 32 + lane;
}

// Keep the two largest finite-or-infinite values seen (NaN never enters).
__device__ __forceinline__ void top2_insert(float v, float &t1, float &t2) {
    if (v > t1) {
        t2 = t1;
        t1 = v;
    } else if (v > t2) {
        t2 = v;
    }
}

template <bool VEC, int VPL>
__global__ void __launch_bounds__(kRouteWarps * 32) route_kernel(const RouteArgs a) {
    __shared__ float sh_keys[kRouteWarps][kMaxE];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int E = a.E;

    // Per-lane constants: which expert each slot holds, its group, its bias.
    int eid[VPL];
    int gidx[VPL];
    float biasr[VPL];
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        int e = slot_expert<VEC>(s, lane);
        eid[s] = e < E ? e : -1;
        gidx[s] = (e < E && a.G > 1) ? e / a.gsz : 0;
        biasr[s] = (a.bias && e < E) ? a.bias[e] : 0.0f;
    }
    const int my_g = lane / a.lpg;
    const int my_p = lane % a.lpg;

    for (int64_t row = (int64_t)blockIdx.x * kRouteWarps + warp; row < a.T;
         row += (int64_t)gridDim.x * kRouteWarps) {
        const float *lrow = a.logits + row * E;
        float l[VPL];
        if (VEC) {
#pragma unroll
            for (int c = 0; c < VPL / 4; ++c) {
                const int e0 = c * 128 + lane * 4;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (e0 < E) v = ld_stream(reinterpret_cast<const float4 *>(lrow + e0));
                l[4 * c + 0] = v.x;
                l[4 * c + 1] = v.y;
                l[4 * c + 2] = v.z;
                l[4 * c + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int s = 0; s < VPL; ++s) l[s] = eid[s] >= 0 ? ld_stream(lrow + eid[s]) : 0.0f;
        }

        int kt = a.k_max;
        if (a.kpt) {
            kt = a.kpt[row];
            if (kt < 0 || kt > a.k_max) {
                if (lane == 0) report(a.status, MOE_ERR_DEVICE_INDEX);
                kt = kt < 0 ? 0 : a.k_max;
            }
        }

        bool has_nan = false;
#pragma unroll
        for (int s = 0; s < VPL; ++s) has_nan |= (eid[s] >= 0) && (l[s] != l[s]);
        if (__any_sync(MOE_FULL_MASK, has_nan) && lane == 0) report(a.status, MOE_ERR_NAN_LOGIT);

        // Softmax statistics of the whole row, only when a weight or a key
        // needs the full-row denominator.
        float m = -INFINITY, z = 1.0f;
        const bool need_z =
            a.score == MOE_SCORE_SOFTMAX && (a.keys_from_scores || !a.renorm);
        if (need_z) {
            float lm = -INFINITY;
#pragma unroll
            for (int s = 0; s < VPL; ++s)
                if (eid[s] >= 0) lm = fmaxf(lm, l[s]);
            m = warp_max(lm);
            float ls = 0.0f;
#pragma unroll
            for (int s = 0; s < VPL; ++s)
                if (eid[s] >= 0) ls += expf(l[s] - m);
            z = warp_sum(ls);
        }

        // Selection keys.
        uint32_t key[VPL];
        float *kb = sh_keys[warp];
#pragma unroll
        for (int s = 0; s < VPL; ++s) {
            float v = l[s];
            if (a.keys_from_scores) {
                if (a.score == MOE_SCORE_SOFTMAX)
                    v = expf(l[s] - m) / z;
                else if (a.score == MOE_SCORE_SIGMOID)
                    v = sigmoid_score(l[s]);
                else if (a.score == MOE_SCORE_SQRT_SOFTPLUS)
                    v = sqrt_softplus_score(l[s]);
                v += biasr[s];
            }
            key[s] = eid[s] >= 0 ? order_key(v) : 0u;
            if (a.G > 1 && eid[s] >= 0) kb[eid[s]] = v;
        }

        // Group limit: per-group top-n sum over a lane strip, merged across
        // the lanes of the group, then topk_groups rounds of warp argmax.
        if (a.G > 1) {
            __syncwarp();
            float t1 = -INFINITY, t2 = -INFINITY;
            if (my_g < a.G) {
                const int lo = my_g * a.gsz + my_p * a.strip;
                const int hi = min(lo + a.strip, (my_g + 1) * a.gsz);
                for (int e = lo; e < hi; ++e) top2_insert(kb[e], t1, t2);
            }
            for (int o = 1; o < a.lpg; o <<= 1) {
                const float b1 = __shfl_xor_sync(MOE_FULL_MASK, t1, o);
                const float b2 = __shfl_xor_sync(MOE_FULL_MASK, t2, o);
                const float n1 = fmaxf(t1, b1);
                const float n2 = fmaxf(fminf(t1, b1), fmaxf(t2, b2));
                t1 = n1;
                t2 = n2;
            }
            __syncwarp();
            const float gs = a.topn == 1 ? t1 : t1 + t2;
            uint32_t gk = (my_g < a.G && my_p == 0) ? order_key(gs) : 0u;
            uint32_t kept = 0;
            for (int r = 0; r < a.TG; ++r) {
                const uint32_t mx = __reduce_max_sync(MOE_FULL_MASK, gk);
                const uint32_t cand = (gk == mx) ? (uint32_t)my_g : 0xffffffffu;
                const uint32_t win = __reduce_min_sync(MOE_FULL_MASK, cand);
                kept |= 1u << win;
                if ((uint32_t)my_g == win) gk = 0u;
            }
#pragma unroll
            for (int s = 0; s < VPL; ++s)
                if (!((kept >> gidx[s]) & 1u)) key[s] = 0u;
        }

        // Top-k_t: each round takes the largest key, lowest id among equals.
        uint32_t bk = 0u;
        int bid = 0x7fffffff;
#pragma unroll
        for (int s = 0; s < VPL; ++s)
            if (key[s] > bk) {
                bk = key[s];
                bid = eid[s];
            }
        int my_id = -1;
        float my_l = 0.0f;
        int nsel = 0;
        for (int r = 0; r < kt; ++r) {
            const uint32_t mx = __reduce_max_sync(MOE_FULL_MASK, bk);
            if (mx == 0u) break;
            const uint32_t cand = (bk == mx) ? (uint32_t)bid : 0xffffffffu;
            const int win = (int)__reduce_min_sync(MOE_FULL_MASK, cand);
            const int owner = VEC ? ((win & 127) >> 2) : (win & 31);
            float lw = 0.0f;
            if (lane == owner) {
                bk = 0u;
                bid = 0x7fffffff;
#pragma unroll
                for (int s = 0; s < VPL; ++s) {
                    if (eid[s] == win) {
                        lw = l[s];
                        key[s] = 0u;
                    }
                    if (key[s] > bk) {
                        bk = key[s];
                        bid = eid[s];
                    }
                }
            }
            lw = __shfl_sync(MOE_FULL_MASK, lw, owner);
            if (lane == r) {
                my_id = win;
                my_l = lw;
            }
            ++nsel;
        }

        // Weights of the selected experts, one per lane.
        const bool act = lane < nsel;
        float s = 0.0f;
        if (a.score == MOE_SCORE_SOFTMAX && !a.renorm) {
            s = act ? expf(my_l - m) / z : 0.0f;
        } else if (a.score == MOE_SCORE_SOFTMAX || a.score == MOE_SCORE_TOPK_SOFTMAX) {
            const float msel = warp_max(act ? my_l : -INFINITY);
            s = act ? expf(my_l - msel) : 0.0f;
        } else if (a.score == MOE_SCORE_SIGMOID) {
            s = act ? sigmoid_score(my_l) : 0.0f;
        } else {
            s = act ? sqrt_softplus_score(my_l) : 0.0f;
        }
        if (a.renorm || a.score == MOE_SCORE_TOPK_SOFTMAX) {
            const float sum = warp_sum(s);
            if (act && sum > 0.0f) s = s / sum;
        }
        if (lane < a.k_max) {
            a.ids[row * a.k_max + lane] = act ? my_id : -1;
            a.w[row * a.k_max + lane] = act ? s * a.scale : 0.0f;
        }
    }
}

template <bool VEC>
cudaError_t launch_route(const RouteArgs &a, int vpl, dim3 grid, cudaStream_t st) {
    switch (vpl) {
        case 4: route_kernel<VEC, 4><<<grid, kRouteWarps * 32, 0, st>>>(a); break;
        case 8: route_kernel<VEC, 8><<<grid, kRouteWarps * 32, 0, st>>>(a); break;
        case 12: route_kernel<VEC, 12><<<grid, kRouteWarps * 32, 0, st>>>(a); break;
        default: route_kernel<VEC, 16><<<grid, kRouteWarps * 32, 0, st>>>(a); break;
    }
    return cudaSuccess;
}

// ------------------------------------------------------------- hash route --
struct HashArgs {
    const int32_t *tok;
    const int32_t *table;
    const float *logits;
    int32_t *ids;
    float *w;
    int32_t *status;
    int64_t T;
    int vocab, k, E, score, renorm;
    float scale;
};

__global__ void __launch_bounds__(256) hash_route_kernel(const HashArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < a.T;
         row += warps) {
        const int v = a.tok[row];
        const bool row_ok = v >= 0 && v < a.vocab;
        if (!row_ok && lane == 0) report(a.status, MOE_ERR_DEVICE_INDEX);
        int id = -1;
        if (row_ok && lane < a.k) {
            id = a.table[(int64_t)v * a.k + lane];
            if (id < 0 || id >= a.E) {
                report(a.status, MOE_ERR_DEVICE_INDEX);
                id = -1;
            }
        }
        const bool act = id >= 0;
        float s;
        if (a.logits) {
            const float *lrow = a.logits + row * a.E;
            const float l = act ? lrow[id] : 0.0f;
            if (l != l) report(a.status, MOE_ERR_NAN_LOGIT);
            if (a.score == MOE_SCORE_SOFTMAX && !a.renorm) {
                float lm = -INFINITY;
                for (int e = lane; e < a.E; e += 32) lm = fmaxf(lm, lrow[e]);
                const float m = warp_max(lm);
                float ls = 0.0f;
                for (int e = lane; e < a.E; e += 32) ls += expf(lrow[e] - m);
                const float z = warp_sum(ls);
                s = act ? expf(l - m) / z : 0.0f;
            } else if (a.score == MOE_SCORE_SOFTMAX || a.score == MOE_SCORE_TOPK_SOFTMAX) {
                const float msel = warp_max(act ? l : -INFINITY);
                s = act ? expf(l - msel) : 0.0f;
            } else if (a.score == MOE_SCORE_SIGMOID) {
                s = act ? sigmoid_score(l) : 0.0f;
            } else {
                s = act ? sqrt_softplus_score(l) : 0.0f;
            }
            if (a.renorm || a.score == MOE_SCORE_TOPK_SOFTMAX) {
                const float sum = warp_sum(s);
                if (act && sum > 0.0f) s = s / sum;
            }
            s *= a.scale;
        } else {
            s = act ? a.scale / (float)a.k : 0.0f;
        }
        if (lane < a.k) {
            a.ids[row * a.k + lane] = id;
            a.w[row * a.k + lane] = act ? s : 0.0f;
        }
    }
}

bool valid_score(int s) {
    return s == MOE_SCORE_SOFTMAX || s == MOE_SCORE_SIGMOID || s == MOE_SCORE_SQRT_SOFTPLUS ||
           s == MOE_SCORE_TOPK_SOFTMAX;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_route(const float *logits, const float *bias, const int32_t *k_per_token,
                                const moe_route_params *p, int64_t T, int32_t *topk_ids,
                                float *topk_w, int32_t *d_status, moe_stream_t stream) {
    using namespace moe;
    if (!p || T < 0) return MOE_ERR_INVALID_ARG;
    const int E = p->num_experts, G = p->n_groups;
    if (E < 1 || E > kMaxE || p->k_max < 0 || p->k_max > E || p->k_max > 32)
        return MOE_ERR_INVALID_ARG;
    if (!valid_score(p->score) || G < 1 || E % G != 0) return MOE_ERR_INVALID_ARG;
    if (G > 32) return MOE_ERR_UNSUPPORTED;
    if (G > 1 && (p->topk_groups < 1 || p->topk_groups > G || p->group_topn < 1 ||
                  p->group_topn > 2 || p->group_topn > E / G || p->k_max > p->topk_groups * (E / G)))
        return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!logits || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
    if (T > (int64_t)INT32_MAX / (p->k_max > 0 ? p->k_max : 1)) return MOE_ERR_UNSUPPORTED;

    RouteArgs a;
    a.logits = logits;
    a.bias = bias;
    a.kpt = k_per_token;
    a.ids = topk_ids;
    a.w = topk_w;
    a.status = d_status;
    a.T = T;
    a.E = E;
    a.k_max = p->k_max;
    a.score = p->score;
    a.G = G;
    a.TG = G > 1 ? p->topk_groups : 1;
    a.topn = G > 1 ? p->group_topn : 1;
    a.renorm = p->renormalize ? 1 : 0;
    a.scale = p->route_scale;
    a.gsz = E / G;
    int lpg = 1;
    while (lpg * 2 * G <= 32) lpg *= 2;
    a.lpg = lpg;
    a.strip = (a.gsz + lpg - 1) / lpg;
    a.keys_from_scores = (bias != nullptr) || (G > 1 && a.topn > 1);

    const bool vec = (E % 4 == 0) && aligned16(logits);
    const int vpl_need = vec ? 4 * ((E + 127) / 128) : (E + 31) / 32;
    const int vpl = vpl_need <= 4 ? 4 : vpl_need <= 8 ? 8 : vpl_need <= 12 ? 12 : 16;
    const int64_t blocks_needed = (T + kRouteWarps - 1) / kRouteWarps;
    const int64_t cap = (int64_t)sm_count() * 8;
    dim3 grid((unsigned)(blocks_needed < cap ? blocks_needed : cap));
    cudaStream_t st = as_cuda(stream);
    if (vec)
        launch_route<true>(a, vpl, grid, st);
    else
        launch_route<false>(a, vpl, grid, st);
    return launch_status();
}

extern "C" moe_status moe_hash_route(const int32_t *token_ids, const int32_t *tid2eid,
                                     int32_t vocab, int32_t k, const float *logits,
                                     const moe_route_params *p, int64_t T, int32_t *topk_ids,
                                     float *topk_w, int32_t *d_status, moe_stream_t stream) {
    using namespace moe;
    if (!p || T < 0 || vocab < 1 || k < 1 || k > 32) return MOE_ERR_INVALID_ARG;
    if (p->num_experts < 1 || p->num_experts > kMaxE || !valid_score(p->score))
        return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!token_ids || !tid2eid || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
    if (T > (int64_t)INT32_MAX / k) return MOE_ERR_UNSUPPORTED;
    HashArgs a;
    a.tok = token_ids;
    a.table = tid2eid;
    a.logits = logits;
    a.ids = topk_ids;
    a.w = topk_w;
    a.status = d_status;
    a.T = T;
    a.vocab = vocab;
    a.k = k;
    a.E = p->num_experts;
    a.score = p->score;
    a.renorm = p->renormalize ? 1 : 0;
    a.scale = p->route_scale;
    const int64_t blocks_needed = (T + 7) / 8;
    const int64_t cap = (int64_t)sm_count() * 8;
    hash_route_kernel<<<(unsigned)(blocks_needed < cap ? blocks_needed : cap), 256, 0,
                        as_cuda(stream)>>>(a);
    return launch_status();
}
