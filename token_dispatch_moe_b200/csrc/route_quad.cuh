// The quad-per-row route kernel (moe_route's path for 128-bit rows, k_max <=
// 8 and groups of whole 16-expert chunks).  Its instances are compiled in two
// files: route_quad.cu (selection words from the float image of the key) and
// route_quad_fixed.cu (fixed-point words, for sigmoid and softmax keys), so
// that the two sets build in parallel.  route.cu includes the constants and
// the two lookups only (MOE_ROUTE_QUAD_HOST_ONLY).
#pragma once

#include "common.cuh"
#include "tc.cuh"
#include "route_row.cuh"

namespace moe {

// The kernel for P selection slots (1, 2, 4, 8) and rows of nch chunks of 16
// experts, with float-image or fixed-point selection words.
void *route_quad_fn_float(int P, int nch);
void *route_quad_fn_fixed(int P, int nch);

namespace {

// ------------------------------------------------- quad-per-row route kernel --
// Four lanes (a quad) route one token row; a warp routes 8 rows at a time.
// Lane j of the quad owns, in every chunk of 16 experts, the 4-expert vector
// 16c + 4j.  Each lane copies its own vectors of the row straight into its
// own slots of the warp's shared-memory buffer with cp.async (16 bytes each,
// buffer layout [chunk][lane], so every 128-bit access of the warp is
// contiguous and free of bank conflicts); no other thread touches them, so no
// barrier is needed, and without tiles or a TMA ring many warps per SM stay
// resident to hide the latency of the per-row arithmetic.
//
// Per row (quad-cooperative, no warp-wide step):
//   stats    row max and softmax denominator, only where a key or a weight
//            needs them (quad reductions);
//   keys     with a bias or a top-2 group score, key = score + bias is
//            computed once and written over the logits;
//   groups   each group's top-2 (or amax) merged over the quad with
//            shuffles; the kept groups by topk_groups rounds of an exact
//            argmax over (group score, lower group id);
//   select   a key enters the selection as one 32-bit word: a 23-bit key
//            prefix above 511 - id.  The prefix is the top of the key's
//            order-preserving float image (sign, exponent, 14 mantissa bits),
//            or, for sigmoid and softmax keys, which lie in [min bias,
//            1 + max bias], the key in 23-bit fixed point over that range
//            (the FIX instances).  Words are unique and a larger word is a
//            larger key prefix, then a lower id, so each lane keeps its P
//            largest words with a branch-free umax/umin insertion network
//            (two integer ops a step), and two shuffle rounds merge the
//            quad's four lists (bitonic: the partner's list reversed,
//            elementwise max, then a half-cleaner).  The first k_t words are
//            the selection in output order when the prefixes decide it;
//   check    they do unless two keys share a prefix where it matters: the
//            network also keeps the largest word it pushed out, so the
//            (k_t+1)-th word is known, and the row is settled here when the
//            k_t selected prefixes are distinct and the (k_t+1)-th word's
//            prefix is below the k_t-th (then the word order is the key
//            order and the set is the key set);
//   weights  each lane finishes the slots j, j+4, ... from the logits.
// A row that fails the check (two keys sharing a prefix at the selection:
// within 2^-14 of each other for float prefixes, within 2^-23 of the key range
// for fixed-point ones; exact ties included), or that holds a NaN or infinite
// key (or, with keys that are the logits, logit), is handed to the
// warp-per-row routine (route_row), whose 64-bit keys order equal keys by id
// and NaN below every number.  The fewer rows reach it the better: it is a
// long chain of warp reductions, and a warp that takes one finishes late.
constexpr int kQuadThreads = 256;           // 8 warps, 64 quads
constexpr int kQuadWarps = kQuadThreads / 32;
constexpr int kQuadGroupStride = 33;        // per-quad group-score slots (padded)
constexpr uint32_t kPrefixMask = 0xfffffe00u;

#ifndef MOE_ROUTE_QUAD_HOST_ONLY
__device__ __forceinline__ float quad_max(float v) {
    v = fmaxf(v, __shfl_xor_sync(MOE_FULL_MASK, v, 1));
    return fmaxf(v, __shfl_xor_sync(MOE_FULL_MASK, v, 2));
}
__device__ __forceinline__ float quad_sum(float v) {
    v += __shfl_xor_sync(MOE_FULL_MASK, v, 1);
    return v + __shfl_xor_sync(MOE_FULL_MASK, v, 2);
}

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Selection word of a key that is not NaN: order-preserving image (v + 0
// turns -0 into +0), its low 9 bits replaced by 511 - id.
__device__ __forceinline__ uint32_t sel_word(float v, int id) {
    const uint32_t u = __float_as_uint(v + 0.0f);
    const uint32_t img = u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
    return (img & kPrefixMask) | (uint32_t)(511 - id);
}

// Insert v into the descending list; ext keeps the largest word pushed out
// (the (P+1)-th largest seen so far).
template <int P>
__device__ __forceinline__ void net_insert(uint32_t (&L)[P], uint32_t &ext, uint32_t v) {
#pragma unroll
    for (int p = 0; p < P; ++p) {
        const uint32_t hi = max(L[p], v);
        v = min(L[p], v);
        L[p] = hi;
    }
    ext = max(ext, v);
}

// Insert four words: sorted among themselves (five compare-exchanges), set
// against the list's tail in reverse (elementwise max: the larger halves form
// a bitonic sequence, the smaller ones are pushed out), then sorted back by a
// half-cleaner cascade.
template <int P>
__device__ __forceinline__ void net_insert4(uint32_t (&L)[P], uint32_t &ext, uint32_t a0,
                                            uint32_t a1, uint32_t a2, uint32_t a3) {
    if (P < 4) {
        net_insert<P>(L, ext, a0);
        net_insert<P>(L, ext, a1);
        net_insert<P>(L, ext, a2);
        net_insert<P>(L, ext, a3);
        return;
    }
    uint32_t s[4] = {a0, a1, a2, a3};
    auto cx = [](uint32_t &x, uint32_t &y) {
        const uint32_t hi = max(x, y);
        y = min(x, y);
        x = hi;
    };
    cx(s[0], s[1]);
    cx(s[2], s[3]);
    cx(s[0], s[2]);
    cx(s[1], s[3]);
    cx(s[1], s[2]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int p = P - 4 + i;
        if (p >= 0) {
            ext = max(ext, min(L[p], s[3 - i]));
            L[p] = max(L[p], s[3 - i]);
        }
    }
#pragma unroll
    for (int st = P / 2; st >= 1; st >>= 1)
#pragma unroll
        for (int i = 0; i < P; ++i)
            if ((i & st) == 0) cx(L[i], L[i + st]);
}

// Merge with the list of the lane `mask` away: both lanes end with the P
// largest words of the two lists, descending, and ext with the largest word
// of both lanes that is not among them.
template <int P>
__device__ __forceinline__ void net_merge(uint32_t (&L)[P], uint32_t &ext, int mask) {
    uint32_t B[P];
#pragma unroll
    for (int p = 0; p < P; ++p) B[p] = __shfl_xor_sync(MOE_FULL_MASK, L[P - 1 - p], mask);
    ext = max(ext, __shfl_xor_sync(MOE_FULL_MASK, ext, mask));
#pragma unroll
    for (int p = 0; p < P; ++p) {  // the larger halves form a bitonic sequence
        ext = max(ext, min(L[p], B[p]));
        L[p] = max(L[p], B[p]);
    }
#pragma unroll
    for (int s = P / 2; s >= 1; s >>= 1)
#pragma unroll
        for (int i = 0; i < P; ++i)
            if ((i & s) == 0) {
                const uint32_t hi = max(L[i], L[i + s]);
                const uint32_t lo = min(L[i], L[i + s]);
                L[i] = hi;
                L[i + s] = lo;
            }
}

// fma(v, 0, acc) turns acc into NaN for a NaN or infinite v.
__device__ __forceinline__ float finite_acc(float acc, const float4 &v) {
    acc = fmaf(v.x, 0.0f, acc);
    acc = fmaf(v.y, 0.0f, acc);
    acc = fmaf(v.z, 0.0f, acc);
    return fmaf(v.w, 0.0f, acc);
}

// A row the quad path does not settle: the warp-per-row routine routes it from
// the logits in global memory (and writes the row's outputs itself).
template <int VPL>
__device__ __forceinline__ void slow_row_t(const RouteArgs &a, int64_t row, int kt, int lane,
                                           float *kscratch) {
    int gidx[VPL];
    float biasr[VPL];
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const int e = slot_expert<true>(s, lane);
        gidx[s] = (e < a.E && a.G > 1) ? e / a.gsz : 0;
        biasr[s] = (a.bias && e < a.E) ? a.bias[e] : 0.0f;
    }
    route_row<true, VPL>(a, a.logits + row * a.E, kt, row, lane, biasr, gidx, kscratch);
}

__device__ __noinline__ void slow_row(const RouteArgs &a, int64_t row, int kt, int lane,
                                      float *kscratch) {
    switch (a.vpl) {
        case 4: slow_row_t<4>(a, row, kt, lane, kscratch); break;
        case 8: slow_row_t<8>(a, row, kt, lane, kscratch); break;
        case 12: slow_row_t<12>(a, row, kt, lane, kscratch); break;
        default: slow_row_t<16>(a, row, kt, lane, kscratch); break;
    }
}

template <int P, int NCH, bool FIX>
__global__ void __launch_bounds__(kQuadThreads, 3) route_quad_kernel(const __grid_constant__ RouteArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int j = lane & 3;            // lane within the quad
    const int qd = threadIdx.x >> 2;   // quad of the block
    const int E = a.E;
    constexpr int nch = NCH;  // chunks of 16 experts (E <= 16 * NCH)
    // [warps x NCH x 32 lanes float4 rows][bias E][group scores 64 x 33]
    // [warp scratch 8 x 512 (group mode 3 only)]
    float4 *buf = reinterpret_cast<float4 *>(smem) + (size_t)warp * nch * 32 + lane;
    float *bias_s = reinterpret_cast<float *>(smem) + (size_t)kQuadWarps * nch * 128;
    float *gsc = bias_s + ((E + 3) & ~3) + qd * kQuadGroupStride;
    float *kscratch = bias_s + ((E + 3) & ~3) + (kQuadThreads / 4) * kQuadGroupStride +
                      (size_t)warp * kRouteMaxE;
    griddep_wait();  // the logits' producer (e.g. the gate GEMM) has completed
    for (int e = threadIdx.x; e < E; e += blockDim.x) bias_s[e] = a.bias ? a.bias[e] : 0.0f;
    __syncthreads();
    // Sigmoid and softmax scores lie in [0, 1], so their keys lie in
    // [min bias, 1 + max bias]: there the selection word's 23-bit prefix is the
    // key in fixed point over that range (about 2^-23 of it a step), far finer
    // than the 14 mantissa bits of the float image and so far fewer prefix
    // ties.  fmaf(key, fx_scale, fx_off) lands in [2^23 + 32, 2^24 - 32], one
    // binade, whose mantissa is the fixed-point key (monotone in the key).
    // (FIX: the launch has sigmoid or softmax keys, a compile-time choice so
    // that the other instances keep the float-image code alone)
    float fx_scale = 0.0f, fx_off = 0.0f;
    if constexpr (FIX) {
        float bmin = 0.0f, bmax = 0.0f;
        if (a.bias) {
            bmin = INFINITY;
            bmax = -INFINITY;
            for (int e = lane; e < E; e += 32) {
                bmin = fminf(bmin, bias_s[e]);
                bmax = fmaxf(bmax, bias_s[e]);
            }
            bmin = -warp_max(-bmin);
            bmax = warp_max(bmax);
        }
        fx_scale = (8388608.0f - 64.0f) / ((1.0f + bmax) - bmin);
        fx_off = 8388608.0f + 32.0f - bmin * fx_scale;
    }

    const bool mono = !a.keys_from_scores;
    const bool grouped = a.G > 1;
    const bool need_stats = a.score == MOE_SCORE_SOFTMAX && (a.keys_from_scores || !a.renorm);
    const bool norm = a.renorm || a.score == MOE_SCORE_TOPK_SOFTMAX;
    const int cpg = grouped ? a.cpg : nch;
    const int64_t step = (int64_t)gridDim.x * kQuadThreads / 4;
    for (int64_t base = (int64_t)blockIdx.x * (kQuadThreads / 4) + warp * 8; base < a.T;
         base += step) {
        const int64_t row = base + (lane >> 2);
        const bool valid = row < a.T;
        const float *src = a.logits + (valid ? row : 0) * E;
        // This lane's vectors of the row, straight into its own slots.
#pragma unroll
        for (int c = 0; c < nch; ++c) {
            const int e0 = 16 * c + 4 * j;
            if (valid && e0 < E) cp_async16(buf + c * 32, src + e0);
        }
        int kraw = a.k_max;
        if (a.kpt && valid) kraw = a.kpt[row];
        int kt = kraw;
        if (kt < 0 || kt > a.k_max) {
            if (valid && j == 0) report(a.status, MOE_ERR_DEVICE_INDEX);
            kt = kt < 0 ? 0 : a.k_max;
        }
        if (!valid) kt = 0;
        cp_async_wait_all();

        float fin = 0.0f;  // NaN once a NaN or infinite logit or key is seen
        float m = -INFINITY, z = 1.0f;
        if (need_stats) {
            float lm = -INFINITY;
#pragma unroll
            for (int c = 0; c < nch; ++c)
                if (16 * c + 4 * j < E) {
                    const float4 v = buf[c * 32];
                    lm = fmaxf(fmaxf(lm, v.x), fmaxf(v.y, fmaxf(v.z, v.w)));
                }
            m = quad_max(lm);
            float ls = 0.0f;
#pragma unroll
            for (int c = 0; c < nch; ++c)
                if (16 * c + 4 * j < E) {
                    const float4 v = buf[c * 32];
                    ls += expf(v.x - m) + expf(v.y - m) + expf(v.z - m) + expf(v.w - m);
                }
            z = quad_sum(ls);
        }
        const float zinv = 1.0f / z;

        // keys (written over the logits) and group scores
        // (a NaN logit gives a NaN key under every score, and an infinite one
        // a key that is infinite or that the warp routine computes alike, so
        // scored rows check their keys only)
        auto make_keys = [&](float4 &v, int e0) {
            if (mono) fin = finite_acc(fin, v);
            if (!mono) {
                const float4 b = *reinterpret_cast<const float4 *>(bias_s + e0);
                float x[4] = {v.x, v.y, v.z, v.w};
                score_keys<4>(a.score, x, m, zinv);  // the same arithmetic as route_row
                v = make_float4(x[0] + b.x, x[1] + b.y, x[2] + b.z, x[3] + b.w);
                fin = finite_acc(fin, v);
            }
        };
        uint32_t kept = 0xffffffffu;
        if (!grouped) {
            if (!mono) {
#pragma unroll
                for (int c = 0; c < nch; ++c) {
                    const int e0 = 16 * c + 4 * j;
                    if (e0 < E) {
                        float4 v = buf[c * 32];
                        make_keys(v, e0);
                        buf[c * 32] = v;
                    }
                }
            }
        } else {
            for (int g = 0; g < a.G; ++g) {
                float t1 = -INFINITY, t2 = -INFINITY;
                for (int cc = 0; cc < cpg; ++cc) {
                    const int c = g * cpg + cc;
                    const int e0 = 16 * c + 4 * j;
                    if (e0 < E) {
                        float4 v = buf[c * 32];
                        make_keys(v, e0);
                        if (!mono) buf[c * 32] = v;
                        // top two by min/max (no NaN reaches a settled row)
                        t2 = fmaxf(t2, fminf(t1, v.x));
                        t1 = fmaxf(t1, v.x);
                        t2 = fmaxf(t2, fminf(t1, v.y));
                        t1 = fmaxf(t1, v.y);
                        t2 = fmaxf(t2, fminf(t1, v.z));
                        t1 = fmaxf(t1, v.z);
                        t2 = fmaxf(t2, fminf(t1, v.w));
                        t1 = fmaxf(t1, v.w);
                    }
                }
#pragma unroll
                for (int o = 1; o <= 2; o <<= 1) {
                    const float b1 = __shfl_xor_sync(MOE_FULL_MASK, t1, o);
                    const float b2 = __shfl_xor_sync(MOE_FULL_MASK, t2, o);
                    top2_merge(t1, t2, b1, b2);
                }
                if (j == 0) gsc[g] = a.topn == 1 ? t1 : t1 + t2;
            }
            // topk_groups rounds of an exact argmax over (score, lower id);
            // lane j weighs the groups j, j+4, ...
            __syncwarp();
            kept = 0u;
            for (int r = 0; r < a.TG; ++r) {
                float bs = -INFINITY;
                int bg = 64;
                for (int g = j; g < a.G; g += 4) {
                    const float sc = gsc[g];
                    if (!((kept >> g) & 1u) && (sc > bs || (sc == bs && g < bg))) {
                        bs = sc;
                        bg = g;
                    }
                }
#pragma unroll
                for (int o = 1; o <= 2; o <<= 1) {
                    const float os = __shfl_xor_sync(MOE_FULL_MASK, bs, o);
                    const int og = __shfl_xor_sync(MOE_FULL_MASK, bg, o);
                    if (os > bs || (os == bs && og < bg)) {
                        bs = os;
                        bg = og;
                    }
                }
                kept |= 1u << (bg & 31);
            }
            __syncwarp();
        }

        // the selection word of key x of expert id: a fixed-point (FIX) or
        // float-image prefix above 511 - id
        auto word = [&](float x, int id) -> uint32_t {
            if constexpr (FIX)
                return (__float_as_uint(fmaf(x, fx_scale, fx_off)) << 9) | (uint32_t)(511 - id);
            else
                return sel_word(x, id);
        };
        // f(keys, first expert) over this lane's vectors of the kept experts
        auto each_kept = [&](auto &&f) {
            if (!grouped) {
#pragma unroll
                for (int c = 0; c < nch; ++c) {
                    const int e0 = 16 * c + 4 * j;
                    if (e0 < E) f(buf[c * 32], e0);
                }
            } else {
                uint32_t mk = kept;
                for (int gi = 0; gi < a.TG; ++gi) {
                    const int g = __ffs(mk) - 1;
                    mk &= mk - 1u;
                    for (int cc = 0; cc < cpg; ++cc) {
                        const int c = g * cpg + cc;
                        const int e0 = 16 * c + 4 * j;
                        if (e0 < E) f(buf[c * 32], e0);
                    }
                }
            }
        };
        // select: the P largest words of the kept experts, and the largest
        // word beyond them
        uint32_t L[P];
        uint32_t ext = 0u;
#pragma unroll
        for (int p = 0; p < P; ++p) L[p] = 0u;
        each_kept([&](const float4 &v, int e0) {
            if (mono && !grouped) fin = finite_acc(fin, v);  // (other keys were checked above)
            net_insert4<P>(L, ext, word(v.x, e0), word(v.y, e0 + 1), word(v.z, e0 + 2),
                           word(v.w, e0 + 3));
        });
        net_merge<P>(L, ext, 1);
        net_merge<P>(L, ext, 2);
        // check: distinct selected prefixes, and the next word's prefix below
        // the k_t-th's
        uint32_t tp = 0u, nxt = ext;
        bool dup = false;
#pragma unroll
        for (int p = 0; p < P; ++p) {
            if (p == kt - 1) tp = L[p] & kPrefixMask;
            if (p == kt) nxt = L[p];
            if (p > 0 && p < kt && ((L[p] ^ L[p - 1]) & kPrefixMask) == 0u) dup = true;
        }
        fin += __shfl_xor_sync(MOE_FULL_MASK, fin, 1);
        fin += __shfl_xor_sync(MOE_FULL_MASK, fin, 2);
        const bool slow = valid && (fin != fin || dup || (kt > 0 && (nxt & kPrefixMask) == tp));

        // weights of the slots j, j+4, ...
        constexpr int NS = (P + 3) / 4;
        float lsel[NS];
        int isel[NS];
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const int sl = j + 4 * i;
            uint32_t wv = 0u;
#pragma unroll
            for (int p = 0; p < P; ++p)
                if (p == sl) wv = L[p];
            isel[i] = (sl < kt && !slow) ? 511 - (int)(wv & 0x1ffu) : -1;
            lsel[i] = isel[i] >= 0 ? __ldg(src + isel[i]) : 0.0f;
        }
        float msel = -INFINITY;
#pragma unroll
        for (int i = 0; i < NS; ++i)
            if (isel[i] >= 0) msel = fmaxf(msel, lsel[i]);
        msel = quad_max(msel);
        float sv[NS];
        float part = 0.0f;
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            float x = 0.0f;
            if (isel[i] >= 0) {
                const float l = lsel[i];
                if (a.score == MOE_SCORE_SOFTMAX && !a.renorm)
                    x = expf(l - m) / z;
                else if (a.score == MOE_SCORE_SOFTMAX || a.score == MOE_SCORE_TOPK_SOFTMAX)
                    x = expf(l - msel);
                else if (a.score == MOE_SCORE_SIGMOID)
                    x = sigmoid_score(l);
                else
                    x = sqrt_softplus_score(l);
            }
            sv[i] = x;
            part += x;
        }
        const float sum = quad_sum(part);
        if (valid && !slow) {
            int32_t *orow = a.ids + row * a.k_max;
            float *wrow = a.w + row * a.k_max;
#pragma unroll
            for (int i = 0; i < NS; ++i) {
                const int sl = j + 4 * i;
                if (isel[i] >= 0) {
                    orow[sl] = isel[i];
                    wrow[sl] = (norm && sum > 0.0f ? sv[i] / sum : sv[i]) * a.scale;
                }
            }
            for (int sl = kt + j; sl < a.k_max; sl += 4) {
                orow[sl] = -1;
                wrow[sl] = 0.0f;
            }
        }

        // rows the quad path did not settle
        unsigned sm = __ballot_sync(MOE_FULL_MASK, slow && j == 0);
        while (sm) {
            const int src_lane = __ffs(sm) - 1;
            sm &= sm - 1u;
            const int kr = __shfl_sync(MOE_FULL_MASK, kraw, src_lane);
            slow_row(a, base + src_lane / 4, kr, lane, kscratch);
        }
        __syncwarp();  // every lane is done with its slots before the next rows land
    }
    griddep_launch_dependents();
}

template <int NCH, bool FIX>
void *quad_fn_p(int P) {
    switch (P) {
        case 1: return (void *)route_quad_kernel<1, NCH, FIX>;
        case 2: return (void *)route_quad_kernel<2, NCH, FIX>;
        case 4: return (void *)route_quad_kernel<4, NCH, FIX>;
        default: return (void *)route_quad_kernel<8, NCH, FIX>;
    }
}

// The instance for P selection slots and rows of nch chunks of 16 experts.
template <bool FIX>
void *quad_fn(int P, int nch) {
    if (nch <= 8) return quad_fn_p<8, FIX>(P);
    if (nch <= 16) return quad_fn_p<16, FIX>(P);
    if (nch <= 24) return quad_fn_p<24, FIX>(P);
    return quad_fn_p<32, FIX>(P);
}

#endif  // MOE_ROUTE_QUAD_HOST_ONLY

}  // namespace
}  // namespace moe
