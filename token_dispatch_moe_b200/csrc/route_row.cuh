// The per-row router shared by moe_route's kernel and the gate GEMM's
// routing epilogue (moe_gate_route): one warp routes one token row held in
// shared memory.  Internal to libmoe_dispatch.
//
// Keys are 64-bit words: the order-preserving image of the fp32 key (NaN
// lowest, -0 = +0) above 511 - id, so words are unique and a larger word is
// the better expert (ties go to the lower id).  Each lane sorts its <= 16
// words with a compile-time Batcher network (every register index constant);
// a top-k round is then two warp reductions (redux.sync max of hi, then max
// of lo among the lanes holding that hi) and a register shift in the one lane
// that owned the winner.  Monotone shortcut: with no bias and an amax group
// score, every score function orders experts like their logits, so keys are
// the logits and only the selected experts are ever scored.  Groups: when
// groups align with the 4-expert lane vectors and the 128-wide chunks, a
// group's top-2 is merged with register shuffles; otherwise each lane scans a
// strip of the group in shared memory.
#pragma once

#include "common.cuh"

namespace moe {
namespace {

constexpr int kRouteMaxE = 512;

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
    int gsz;                  // group size E / G
    int lpg, strip;           // shared-memory group path: lanes per group, strip length
    int group_mode;           // 0 none, 1 shuffle (gsz <= 128), 2 shuffle (gsz multiple of 128), 3 smem
    int keys_from_scores;     // 0: select on the logit (monotone case)
    int R;                    // rows per tile (multiple of 8)
    int64_t ntiles;
    int red_width;            // power of two >= k_max (width of the weight reductions)
    // quad-per-row kernel (moe_route): padded row stride in floats, ring depth,
    // values per lane of the warp-per-row routine (rows it takes over), row
    // chunks of 16 experts, chunks per group
    int rs, nstage, vpl, nch, cpg;
};

// Everything of RouteArgs that follows from the call's parameters (not the
// tiling of the kernel that uses it).
inline void fill_route_args(RouteArgs &a, const float *logits, const float *bias,
                            const int32_t *k_per_token, const moe_route_params &p, int64_t T,
                            int32_t *topk_ids, float *topk_w, int32_t *d_status) {
    const int E = p.num_experts, G = p.n_groups;
    a.logits = logits;
    a.bias = bias;
    a.kpt = k_per_token;
    a.ids = topk_ids;
    a.w = topk_w;
    a.status = d_status;
    a.T = T;
    a.E = E;
    a.k_max = p.k_max;
    a.score = p.score;
    a.G = G;
    a.TG = G > 1 ? p.topk_groups : 1;
    a.topn = G > 1 ? p.group_topn : 1;
    a.renorm = p.renormalize ? 1 : 0;
    a.scale = p.route_scale;
    a.gsz = E / G;
    int lpg = 1;
    while (lpg * 2 * G <= 32) lpg *= 2;
    a.lpg = lpg;
    a.strip = (a.gsz + lpg - 1) / lpg;
    a.keys_from_scores = (bias != nullptr) || (G > 1 && a.topn > 1);
    const bool vec = (E % 4 == 0);
    if (G == 1)
        a.group_mode = 0;
    else if (vec && a.gsz % 4 == 0 && 128 % a.gsz == 0)
        a.group_mode = 1;
    else if (vec && a.gsz % 128 == 0)
        a.group_mode = 2;
    else
        a.group_mode = 3;
    int width = 1;
    while (width < p.k_max) width *= 2;
    a.red_width = width;
    a.R = 0;
    a.ntiles = 0;
    a.vpl = vec ? 4 * ((E + 127) / 128) : (E + 31) / 32;
    a.vpl = a.vpl <= 4 ? 4 : a.vpl <= 8 ? 8 : a.vpl <= 12 ? 12 : 16;
    a.nch = (E + 15) / 16;
    a.cpg = a.gsz % 16 == 0 ? a.gsz / 16 : 0;
    a.rs = 0;
    a.nstage = 0;
}

template <bool VEC>
__device__ __forceinline__ int slot_expert(int s, int lane) {
    return VEC ? (s >> 2) * 128 + lane * 4 + (s & 3) : s * 32 + lane;
}

// Order-preserving image of an fp32 key: larger float -> larger word; -0 and
// +0 equal; NaN -> 1 (below -inf, whose image is 0x007fffff); 0 is reserved.
__device__ __forceinline__ uint32_t key_bits(float v) {
    uint32_t u = __float_as_uint(v);
    u = (v == 0.0f) ? 0u : u;
    const uint32_t o = u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
    return (v != v) ? 1u : o;
}

// Keep the two largest values seen (NaN never enters).
__device__ __forceinline__ void top2_insert(float v, float &t1, float &t2) {
    if (v > t1) {
        t2 = t1;
        t1 = v;
    } else if (v > t2) {
        t2 = v;
    }
}

__device__ __forceinline__ void top2_merge(float &t1, float &t2, float b1, float b2) {
    const float n1 = fmaxf(t1, b1);
    const float n2 = fmaxf(fminf(t1, b1), fmaxf(t2, b2));
    t1 = n1;
    t2 = n2;
}

// Width-limited butterfly reductions (lanes >= width contribute the identity).
__device__ __forceinline__ float sum_width(float v, int width) {
    for (int o = 1; o < width; o <<= 1) v += __shfl_xor_sync(MOE_FULL_MASK, v, o);
    return v;
}
__device__ __forceinline__ float max_width(float v, int width) {
    for (int o = 1; o < width; o <<= 1) v = fmaxf(v, __shfl_xor_sync(MOE_FULL_MASK, v, o));
    return v;
}

// Descending compare-exchange on (hi, lo) words.
__device__ __forceinline__ void cas_desc(uint32_t &ah, uint32_t &al, uint32_t &bh, uint32_t &bl) {
    const bool swap = (bh > ah) || (bh == ah && bl > al);
    const uint32_t th = swap ? bh : ah, tl = swap ? bl : al;
    bh = swap ? ah : bh;
    bl = swap ? al : bl;
    ah = th;
    al = tl;
}

// Comparators of Batcher's odd-even merge sort of N (power of two) elements,
// listed at compile time so that every register index is a constant.
struct Comparators {
    int n;
    int a[80];
    int b[80];
};

__host__ __device__ constexpr Comparators batcher(int N) {
    Comparators c{};
    for (int p = 1; p < N; p <<= 1)
        for (int k = p; k >= 1; k >>= 1)
            for (int j = k % p; j + k < N; j += 2 * k)
                for (int i = 0; i < k; ++i)
                    if (i + j + k < N && (i + j) / (2 * p) == (i + j + k) / (2 * p)) {
                        c.a[c.n] = i + j;
                        c.b[c.n] = i + j + k;
                        ++c.n;
                    }
    return c;
}

// Sorts N (power of two) words in descending order.
template <int N>
__device__ __forceinline__ void sort_desc(uint32_t (&h)[N], uint32_t (&l)[N]) {
    constexpr Comparators net = batcher(N);
#pragma unroll
    for (int c = 0; c < net.n; ++c) cas_desc(h[net.a[c]], l[net.a[c]], h[net.b[c]], l[net.b[c]]);
}

template <int V>
struct Pow2 {
    static constexpr int value = V <= 1 ? 1 : V <= 2 ? 2 : V <= 4 ? 4 : V <= 8 ? 8 : 16;
};

template <bool VEC, int VPL>
__device__ __forceinline__ void load_row(const float *src, int lane, int E, float (&l)[VPL]) {
    if (VEC) {
#pragma unroll
        for (int c = 0; c < VPL / 4; ++c) {
            const int e0 = c * 128 + lane * 4;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (e0 < E) v = *reinterpret_cast<const float4 *>(src + e0);
            l[4 * c + 0] = v.x;
            l[4 * c + 1] = v.y;
            l[4 * c + 2] = v.z;
            l[4 * c + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int s = 0; s < VPL; ++s) {
            const int e = s * 32 + lane;
            l[s] = e < E ? src[e] : 0.0f;
        }
    }
}

// One token row: keys, group limit, top-k_t, weights, stores.
template <bool VEC, int VPL>
__device__ __forceinline__ void route_row(const RouteArgs &a, const float *src, int kt,
                                          int64_t row, int lane, const float (&biasr)[VPL],
                                          const int (&gidx)[VPL], float *kscratch) {
    constexpr int NP = Pow2<VPL>::value;
    const int E = a.E;
    float l[VPL];
    load_row<VEC, VPL>(src, lane, E, l);

    if (kt < 0 || kt > a.k_max) {
        if (lane == 0) report(a.status, MOE_ERR_DEVICE_INDEX);
        kt = kt < 0 ? 0 : a.k_max;
    }

    bool has_nan = false;
#pragma unroll
    for (int s = 0; s < VPL; ++s) has_nan |= (slot_expert<VEC>(s, lane) < E) && (l[s] != l[s]);
    if (__any_sync(MOE_FULL_MASK, has_nan) && lane == 0) report(a.status, MOE_ERR_NAN_LOGIT);

    // Full-row softmax statistics, only where a key or a weight needs them.
    float m = -INFINITY, z = 1.0f;
    if (a.score == MOE_SCORE_SOFTMAX && (a.keys_from_scores || !a.renorm)) {
        float lm = -INFINITY;
#pragma unroll
        for (int s = 0; s < VPL; ++s)
            if (slot_expert<VEC>(s, lane) < E) lm = fmaxf(lm, l[s]);
        m = warp_max(lm);
        float ls = 0.0f;
#pragma unroll
        for (int s = 0; s < VPL; ++s)
            if (slot_expert<VEC>(s, lane) < E) ls += expf(l[s] - m);
        z = warp_sum(ls);
    }

    // Selection keys as fp32 values.
    float v[VPL];
    if (a.keys_from_scores) {
        const float zinv = 1.0f / z;
#pragma unroll
        for (int s = 0; s < VPL; ++s) v[s] = l[s];
        score_keys<VPL>(a.score, v, m, zinv);
#pragma unroll
        for (int s = 0; s < VPL; ++s) v[s] += biasr[s];
    } else {
#pragma unroll
        for (int s = 0; s < VPL; ++s) v[s] = l[s];
    }

    // Group limit -> bit mask of kept groups.
    uint32_t kept = 0xffffffffu;
    if (a.group_mode != 0) {
        float my_gs = -INFINITY;
        if (a.group_mode == 1) {
            const int lg = a.gsz >> 2;     // lanes per group within a chunk
            const int gpc = 128 / a.gsz;   // groups per chunk
#pragma unroll
            for (int c = 0; c < VPL / 4; ++c) {
                float t1 = -INFINITY, t2 = -INFINITY;
                if (c * 128 + lane * 4 < E)
#pragma unroll
                    for (int j = 0; j < 4; ++j) top2_insert(v[4 * c + j], t1, t2);
                for (int o = 1; o < lg; o <<= 1) {
                    const float b1 = __shfl_xor_sync(MOE_FULL_MASK, t1, o);
                    const float b2 = __shfl_xor_sync(MOE_FULL_MASK, t2, o);
                    top2_merge(t1, t2, b1, b2);
                }
                const float gs = a.topn == 1 ? t1 : t1 + t2;
                const float got = __shfl_sync(MOE_FULL_MASK, gs, (lane % gpc) * lg);
                if (lane / gpc == c) my_gs = got;
            }
        } else if (a.group_mode == 2) {
            const int cpg = a.gsz / 128;  // chunks per group
#pragma unroll
            for (int g = 0; g < VPL / 4; ++g) {
                if (g >= a.G) break;
                float t1 = -INFINITY, t2 = -INFINITY;
#pragma unroll
                for (int c = 0; c < VPL / 4; ++c)
                    if (c / cpg == g && c * 128 + lane * 4 < E)
#pragma unroll
                        for (int j = 0; j < 4; ++j) top2_insert(v[4 * c + j], t1, t2);
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float b1 = __shfl_xor_sync(MOE_FULL_MASK, t1, o);
                    const float b2 = __shfl_xor_sync(MOE_FULL_MASK, t2, o);
                    top2_merge(t1, t2, b1, b2);
                }
                if (lane == g) my_gs = a.topn == 1 ? t1 : t1 + t2;
            }
        } else {
            // Strip scan in shared memory: lane (g, p) takes part p of group g.
#pragma unroll
            for (int s = 0; s < VPL; ++s) {
                const int e = slot_expert<VEC>(s, lane);
                if (e < E) kscratch[e] = v[s];
            }
            __syncwarp();
            const int g = lane / a.lpg, p = lane % a.lpg;
            float t1 = -INFINITY, t2 = -INFINITY;
            if (g < a.G) {
                const int lo = g * a.gsz + p * a.strip;
                const int hi = min(lo + a.strip, (g + 1) * a.gsz);
                for (int e = lo; e < hi; ++e) top2_insert(kscratch[e], t1, t2);
            }
            for (int o = 1; o < a.lpg; o <<= 1) {
                const float b1 = __shfl_xor_sync(MOE_FULL_MASK, t1, o);
                const float b2 = __shfl_xor_sync(MOE_FULL_MASK, t2, o);
                top2_merge(t1, t2, b1, b2);
            }
            __syncwarp();
            const float gs = a.topn == 1 ? t1 : t1 + t2;
            const float got = __shfl_sync(MOE_FULL_MASK, gs, (lane < a.G ? lane : 0) * a.lpg);
            my_gs = got;
        }
        uint32_t gk = lane < a.G ? key_bits(my_gs) : 0u;
        if (lane < a.G && gk == 0u) gk = 1u;
        kept = 0u;
        for (int r = 0; r < a.TG; ++r) {
            const uint32_t mx = __reduce_max_sync(MOE_FULL_MASK, gk);
            const uint32_t cand = (gk == mx) ? (uint32_t)lane : 32u;
            const uint32_t win = __reduce_min_sync(MOE_FULL_MASK, cand);
            kept |= 1u << win;
            if ((uint32_t)lane == win) gk = 0u;
        }
    }

    // 64-bit selection words, sorted per lane.
    uint32_t kh[NP], kl[NP];
#pragma unroll
    for (int s = 0; s < NP; ++s) {
        kh[s] = 0u;
        kl[s] = 0u;
    }
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const int e = slot_expert<VEC>(s, lane);
        const bool ok = e < E && ((kept >> gidx[s]) & 1u);
        kh[s] = ok ? key_bits(v[s]) : 0u;
        kl[s] = ok ? (uint32_t)(511 - e) : 0u;
    }
    sort_desc<NP>(kh, kl);

    // Top-k_t rounds.
    uint32_t sel_lo = 0u;
    int nsel = 0;
    for (; nsel < kt; ++nsel) {
        const uint32_t mh = __reduce_max_sync(MOE_FULL_MASK, kh[0]);
        if (mh == 0u) break;
        const bool hit = kh[0] == mh;
        const uint32_t ml = __reduce_max_sync(MOE_FULL_MASK, hit ? kl[0] : 0u);
        const bool pop = hit && kl[0] == ml;
#pragma unroll
        for (int i = 0; i + 1 < NP; ++i) {
            kh[i] = pop ? kh[i + 1] : kh[i];
            kl[i] = pop ? kl[i + 1] : kl[i];
        }
        kh[NP - 1] = pop ? 0u : kh[NP - 1];
        kl[NP - 1] = pop ? 0u : kl[NP - 1];
        if (lane == nsel) sel_lo = ml;
    }

    // Weights of the selected experts, one per lane.
    const bool act = lane < nsel;
    const int my_id = 511 - (int)sel_lo;
    const float my_l = act ? src[my_id] : 0.0f;
    float s = 0.0f;
    if (a.score == MOE_SCORE_SOFTMAX && !a.renorm) {
        s = act ? expf(my_l - m) / z : 0.0f;
    } else if (a.score == MOE_SCORE_SOFTMAX || a.score == MOE_SCORE_TOPK_SOFTMAX) {
        const float msel = max_width(act ? my_l : -INFINITY, a.red_width);
        s = act ? expf(my_l - msel) : 0.0f;
    } else if (a.score == MOE_SCORE_SIGMOID) {
        s = act ? sigmoid_score(my_l) : 0.0f;
    } else {
        s = act ? sqrt_softplus_score(my_l) : 0.0f;
    }
    if (a.renorm || a.score == MOE_SCORE_TOPK_SOFTMAX) {
        const float sum = sum_width(s, a.red_width);
        if (act && sum > 0.0f) s = s / sum;
    }
    if (lane < a.k_max) {
        a.ids[row * a.k_max + lane] = act ? my_id : -1;
        a.w[row * a.k_max + lane] = act ? s * a.scale : 0.0f;
    }
}

// k_max == 1 without groups: the argmax of the keys (lowest id among equal
// keys) and its weight; no per-lane sort and a single warp round.
template <bool VEC, int VPL>
__device__ __forceinline__ void route_row_top1(const RouteArgs &a, const float *src, int kt,
                                               int64_t row, int lane, const float (&biasr)[VPL]) {
    const int E = a.E;
    float l[VPL];
    load_row<VEC, VPL>(src, lane, E, l);
    if (kt < 0 || kt > 1) {
        if (lane == 0) report(a.status, MOE_ERR_DEVICE_INDEX);
        kt = kt < 0 ? 0 : 1;
    }
    float m = -INFINITY, z = 1.0f;
    bool has_nan = false;
#pragma unroll
    for (int s = 0; s < VPL; ++s)
        if (slot_expert<VEC>(s, lane) < E) {
            has_nan |= l[s] != l[s];
            m = fmaxf(m, l[s]);
        }
    if (__any_sync(MOE_FULL_MASK, has_nan) && lane == 0) report(a.status, MOE_ERR_NAN_LOGIT);
    if (a.score == MOE_SCORE_SOFTMAX && (a.keys_from_scores || !a.renorm)) {
        m = warp_max(m);
        float ls = 0.0f;
#pragma unroll
        for (int s = 0; s < VPL; ++s)
            if (slot_expert<VEC>(s, lane) < E) ls += expf(l[s] - m);
        z = warp_sum(ls);
    }
    // Lane's best key (the first slot wins ties: slots ascend in expert id).
    uint32_t bk = 0u;
    int be = 0x7fffffff;
    const float zinv = 1.0f / z;
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const int e = slot_expert<VEC>(s, lane);
        float v = l[s];
        if (a.keys_from_scores) {
            if (a.score == MOE_SCORE_SOFTMAX)
                v = expf(l[s] - m) * zinv;
            else if (a.score == MOE_SCORE_SIGMOID)
                v = sigmoid_key(l[s]);
            else if (a.score == MOE_SCORE_SQRT_SOFTPLUS)
                v = sqrt_softplus_score(l[s]);
            v += biasr[s];
        }
        const uint32_t k = e < E ? key_bits(v) : 0u;
        if (k > bk) {
            bk = k;
            be = e;
        }
    }
    const uint32_t mx = __reduce_max_sync(MOE_FULL_MASK, bk);
    const int win = (int)__reduce_min_sync(MOE_FULL_MASK, bk == mx ? (uint32_t)be : 0xffffffffu);
    if (lane == 0) {
        const bool act = kt == 1 && mx != 0u;
        float s = 0.0f;
        if (act) {
            const float lw = src[win];
            if (a.score == MOE_SCORE_SOFTMAX && !a.renorm)
                s = expf(lw - m) / z;
            else if (a.score == MOE_SCORE_SOFTMAX || a.score == MOE_SCORE_TOPK_SOFTMAX)
                s = 1.0f;  // softmax over the single selected expert
            else if (a.score == MOE_SCORE_SIGMOID)
                s = sigmoid_score(lw);
            else
                s = sqrt_softplus_score(lw);
            if (a.renorm && s > 0.0f) s = s / s;
        }
        a.ids[row] = act ? win : -1;
        a.w[row] = act ? s * a.scale : 0.0f;
    }
}

}  // namespace
}  // namespace moe
