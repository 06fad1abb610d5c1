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
// B200 design.
//  * Memory: the kernel is persistent; each block streams tiles of R logits
//    rows (contiguous in memory) into a ring of shared-memory stages with 1-D
//    TMA bulk copies (cp.async.bulk, completion on an mbarrier), so several
//    tiles per SM are in flight while warps compute on an earlier one.
//  * Layout: a row of E <= 512 keys is spread over the 32 lanes of a warp;
//    when E % 4 == 0 lane l holds experts 128c + 4l .. 128c + 4l + 3 of chunk
//    c (128-bit shared loads), otherwise experts 32s + l.
//  * Keys: a selection key is one 64-bit word, hi = order-preserving image of
//    the fp32 key (larger float -> larger word, -0 == +0, NaN below every
//    number, 0 = not selectable), lo = 511 - expert id.  Every word is
//    distinct, a larger word is a better expert, and equal keys rank the lower
//    id first, so selection is exact.  Each lane sorts its words once
//    (Batcher's odd-even merge network); a top-k round is then two warp
//    reductions (redux.sync max of hi, then max of lo among the lanes holding
//    that hi) and a register shift in the one lane that owned the winner.
//  * Monotone shortcut: with no bias and an amax group score, every score
//    function orders experts like their logits, so keys are the logits and
//    only the selected experts are ever scored.
//  * Groups: when groups align with the 4-expert lane vectors and the 128-wide
//    chunks, a group's top-2 is merged with register shuffles; otherwise each
//    lane scans a strip of the group in shared memory.
#include "common.cuh"
#include "tc.cuh"
#include "route_row.cuh"

namespace moe {
namespace {

constexpr int kRouteWarps = 8;  // warps per block
constexpr int kMaxE = kRouteMaxE;
constexpr int kStages = 3;

// ---------------------------------------------------------------- helpers --
// Copies `bytes` (a multiple of 16, may be 0) from global src to shared dst;
// completion is counted on the mbarrier's transaction count.
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
    if (bytes)
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                dst),
            "l"(src), "r"(bytes), "r"(bar)
            : "memory");
}

template <bool VEC, int VPL, bool TOP1>
__global__ void __launch_bounds__(kRouteWarps * 32) route_kernel(const RouteArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    griddep_wait();  // the logits' producer (e.g. the gate GEMM) has completed
    const int E = a.E;
    const int R = a.R;
    const size_t stage_floats = (size_t)R * E;
    // [stages x R x E logits][stages x R k_per_token][stages mbarriers]
    float *stages = reinterpret_cast<float *>(smem);
    int32_t *kstages = reinterpret_cast<int32_t *>(stages + kStages * stage_floats);
    uint64_t *bars = reinterpret_cast<uint64_t *>(kstages + kStages * R);
    float *kscratch = reinterpret_cast<float *>(bars + kStages) + (size_t)warp * kMaxE;
    // Per-lane constants: group of each slot, bias of each slot.
    int gidx[VPL];
    float biasr[VPL];
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const int e = slot_expert<VEC>(s, lane);
        gidx[s] = (e < E && a.G > 1) ? e / a.gsz : 0;
        biasr[s] = (a.bias && e < E) ? a.bias[e] : 0.0f;
    }

    auto tile_rows = [&](int64_t t) -> int {
        const int64_t r0 = t * R;
        return (int)(a.T - r0 < R ? a.T - r0 : R);
    };
    // Bytes of a tile that one bulk copy can carry (a multiple of 16).
    auto tile_bytes = [&](int64_t t) -> uint32_t {
        return (uint32_t)(((uint64_t)tile_rows(t) * E * sizeof(float)) & ~uint64_t(15));
    };
    // Bytes of the tile's k_per_token that one bulk copy can carry.
    auto kpt_bytes = [&](int64_t t) -> uint32_t {
        return a.kpt ? (uint32_t)(((uint32_t)tile_rows(t) * sizeof(int32_t)) & ~15u) : 0u;
    };
    auto issue = [&](int64_t t, int stage) {
        const uint32_t bar = smem_u32(&bars[stage]);
        const uint32_t lb = tile_bytes(t), kb = kpt_bytes(t);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                     "r"(lb + kb)
                     : "memory");
        bulk_copy(smem_u32(stages + stage * stage_floats), a.logits + t * R * (int64_t)E, lb, bar);
        bulk_copy(smem_u32(kstages + stage * R), a.kpt + t * R, kb, bar);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars[s])) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int s = 0; s < kStages; ++s) {
            const int64_t t = blockIdx.x + (int64_t)s * gridDim.x;
            if (t < a.ntiles) issue(t, s);
        }
    }
    __syncthreads();

    const int rpw = R / kRouteWarps;
    int it = 0;
    for (int64_t t = blockIdx.x; t < a.ntiles; t += gridDim.x, ++it) {
        const int stage = it % kStages;
        const bool ok = mbar_wait(smem_u32(&bars[stage]), (uint32_t)(it / kStages) & 1u, a.status);
        if (!__syncthreads_and(ok)) break;
        const int rows = tile_rows(t);
        const int covered = (int)(tile_bytes(t) / ((uint32_t)E * sizeof(float)));
        const int kcovered = (int)(kpt_bytes(t) / sizeof(int32_t));
        const float *tile = stages + stage * stage_floats;
        const int32_t *ktile = kstages + stage * R;
        for (int i = 0; i < rpw; ++i) {
            const int r = warp * rpw + i;
            if (r >= rows) break;
            const int64_t row = t * R + r;
            const int kt = !a.kpt ? a.k_max : (r < kcovered ? ktile[r] : a.kpt[row]);
            const float *src = r < covered ? tile + (size_t)r * E : a.logits + row * E;
            if (TOP1)
                route_row_top1<VEC, VPL>(a, src, kt, row, lane, biasr);
            else
                route_row<VEC, VPL>(a, src, kt, row, lane, biasr, gidx, kscratch);
        }
        __syncthreads();  // every warp is done with this stage
        if (threadIdx.x == 0) {
            const int64_t nt = t + (int64_t)kStages * gridDim.x;
            if (nt < a.ntiles) issue(nt, stage);
        }
    }
    // A wait that timed out leaves later tiles unconsumed: let their copies land.
    if (threadIdx.x == 0) {
        for (int64_t t = blockIdx.x + (int64_t)it * gridDim.x, j = it;
             t < a.ntiles && j < it + kStages; t += gridDim.x, ++j)
            if (!mbar_wait(smem_u32(&bars[j % kStages]), (uint32_t)(j / kStages) & 1u, a.status))
                break;
    }
    griddep_launch_dependents();
}

template <bool VEC>
void *route_fn(int vpl, bool top1) {
    if (top1) {
        switch (vpl) {
            case 4: return (void *)route_kernel<VEC, 4, true>;
            case 8: return (void *)route_kernel<VEC, 8, true>;
            case 12: return (void *)route_kernel<VEC, 12, true>;
            default: return (void *)route_kernel<VEC, 16, true>;
        }
    }
    switch (vpl) {
        case 4: return (void *)route_kernel<VEC, 4, false>;
        case 8: return (void *)route_kernel<VEC, 8, false>;
        case 12: return (void *)route_kernel<VEC, 12, false>;
        default: return (void *)route_kernel<VEC, 16, false>;
    }
}

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
//   select   a key enters the selection as one 32-bit word: the top 23 bits
//            of its order-preserving image (sign, exponent, 14 mantissa
//            bits) above 511 - id.  Words are unique and a larger word is a
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
// A row that fails the check (two keys within 2^-14 of each other at the
// selection, exact ties included), or that holds a NaN or infinite logit or
// key, is handed to the warp-per-row routine (route_row), whose 64-bit keys
// order equal keys by id and NaN below every number.
constexpr int kQuadThreads = 256;           // 8 warps, 64 quads
constexpr int kQuadWarps = kQuadThreads / 32;
constexpr int kQuadGroupStride = 33;        // per-quad group-score slots (padded)
constexpr uint32_t kPrefixMask = 0xfffffe00u;

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

template <int P, int NCH>
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
        auto make_keys = [&](float4 &v, int e0) {
            fin = finite_acc(fin, v);
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

        // select: the P largest words of the kept experts, and the largest
        // word beyond them
        uint32_t L[P];
        uint32_t ext = 0u;
#pragma unroll
        for (int p = 0; p < P; ++p) L[p] = 0u;
        auto insert4 = [&](const float4 &v, int e0) {
            net_insert4<P>(L, ext, sel_word(v.x, e0), sel_word(v.y, e0 + 1),
                           sel_word(v.z, e0 + 2), sel_word(v.w, e0 + 3));
        };
        if (!grouped) {
#pragma unroll
            for (int c = 0; c < nch; ++c) {
                const int e0 = 16 * c + 4 * j;
                if (e0 < E) {
                    const float4 v = buf[c * 32];
                    if (mono) fin = finite_acc(fin, v);  // (keys were checked above)
                    insert4(v, e0);
                }
            }
        } else {
            uint32_t mk = kept;
            for (int gi = 0; gi < a.TG; ++gi) {
                const int g = __ffs(mk) - 1;
                mk &= mk - 1u;
                for (int cc = 0; cc < cpg; ++cc) {
                    const int c = g * cpg + cc;
                    const int e0 = 16 * c + 4 * j;
                    if (e0 < E) insert4(buf[c * 32], e0);
                }
            }
        }
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

template <int NCH>
void *quad_fn_p(int P) {
    switch (P) {
        case 1: return (void *)route_quad_kernel<1, NCH>;
        case 2: return (void *)route_quad_kernel<2, NCH>;
        case 4: return (void *)route_quad_kernel<4, NCH>;
        default: return (void *)route_quad_kernel<8, NCH>;
    }
}

// The instance for P selection slots and rows of nch chunks of 16 experts.
void *quad_fn(int P, int nch) {
    if (nch <= 8) return quad_fn_p<8>(P);
    if (nch <= 16) return quad_fn_p<16>(P);
    if (nch <= 24) return quad_fn_p<24>(P);
    return quad_fn_p<32>(P);
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

// W lanes per token, 32 / W tokens a warp (W = the power of two >= k, at most
// 32): every token's dependent loads (token id, table row, logits of the
// looked-up experts) are in flight together with those of the warp's other
// tokens.  Scores that need only the looked-up logits; a softmax over the
// whole row without renormalisation takes hash_route_kernel.
template <int W>
__global__ void __launch_bounds__(256) hash_route_grouped_kernel(const HashArgs a) {
    const int lane = threadIdx.x & 31;
    const int sl = lane & (W - 1);  // slot of this lane in its token
    constexpr int TPW = 32 / W;     // tokens per warp
    const int64_t step = (int64_t)gridDim.x * (blockDim.x >> 5) * TPW;
    griddep_wait();
    for (int64_t row0 = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * TPW;
         row0 < a.T; row0 += step) {
        const int64_t row = row0 + lane / W;
        const bool live = row < a.T;
        const int v = live ? a.tok[row] : 0;
        const bool row_ok = live && v >= 0 && v < a.vocab;
        if (live && !row_ok && sl == 0) report(a.status, MOE_ERR_DEVICE_INDEX);
        int id = -1;
        if (row_ok && sl < a.k) {
            id = a.table[(int64_t)v * a.k + sl];
            if (id < 0 || id >= a.E) {
                report(a.status, MOE_ERR_DEVICE_INDEX);
                id = -1;
            }
        }
        const bool act = id >= 0;
        float s;
        if (a.logits) {
            const float l = act ? a.logits[row * a.E + id] : 0.0f;
            if (l != l) report(a.status, MOE_ERR_NAN_LOGIT);
            if (a.score == MOE_SCORE_SOFTMAX || a.score == MOE_SCORE_TOPK_SOFTMAX) {
                float msel = act ? l : -INFINITY;
#pragma unroll
                for (int o = 1; o < W; o <<= 1)
                    msel = fmaxf(msel, __shfl_xor_sync(MOE_FULL_MASK, msel, o));
                s = act ? expf(l - msel) : 0.0f;
            } else if (a.score == MOE_SCORE_SIGMOID) {
                s = act ? sigmoid_score(l) : 0.0f;
            } else {
                s = act ? sqrt_softplus_score(l) : 0.0f;
            }
            if (a.renorm || a.score == MOE_SCORE_TOPK_SOFTMAX) {
                float sum = s;
#pragma unroll
                for (int o = 1; o < W; o <<= 1) sum += __shfl_xor_sync(MOE_FULL_MASK, sum, o);
                if (act && sum > 0.0f) s = s / sum;
            }
            s *= a.scale;
        } else {
            s = act ? a.scale / (float)a.k : 0.0f;
        }
        if (live && sl < a.k) {
            a.ids[row * a.k + sl] = id;
            a.w[row * a.k + sl] = act ? s : 0.0f;
        }
    }
    griddep_launch_dependents();
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
    if (!logits || !topk_ids || !topk_w || !aligned16(logits) ||
        (k_per_token && !aligned16(k_per_token)))
        return MOE_ERR_INVALID_ARG;
    if (T > (int64_t)INT32_MAX / (p->k_max > 0 ? p->k_max : 1)) return MOE_ERR_UNSUPPORTED;

    RouteArgs a;
    fill_route_args(a, logits, bias, k_per_token, *p, T, topk_ids, topk_w, d_status);
    const bool vec = (E % 4 == 0);
    const int sms = sm_count();

    // Quad-per-row kernel: 128-bit rows, k_max <= 8, groups of whole 16-expert
    // chunks.  A larger k_max keeps the warp-per-row kernel, whose top-k rounds
    // follow each token's own k: with per-request k of 4, 8 or 16 over 128
    // experts (qwen3_dynk) a network sized for 16 measured 30.7 against 20.5 us.
    if (vec && p->k_max >= 1 && p->k_max <= 8 && (G == 1 || a.cpg > 0)) {
        const int nch_t = a.nch <= 8 ? 8 : a.nch <= 16 ? 16 : a.nch <= 24 ? 24 : 32;
        const size_t smem = (size_t)kQuadWarps * nch_t * 512 + (size_t)((E + 3) & ~3) * 4 +
                            (size_t)(kQuadThreads / 4) * kQuadGroupStride * 4 +
                            (a.group_mode == 3 ? (size_t)kQuadWarps * kRouteMaxE * 4 : 0);
        int P = 1;
        while (P < p->k_max) P *= 2;
        void *fn = quad_fn(P, a.nch);
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kQuadThreads, smem) !=
                cudaSuccess ||
            per_sm < 1) {
            cudaGetLastError();
            per_sm = 1;
        }
        const int64_t need = (T + kQuadThreads / 4 - 1) / (kQuadThreads / 4);
        const int64_t cap = (int64_t)sms * per_sm;
        const unsigned grid = (unsigned)(need < cap ? need : cap);
        void *args[] = {&a};
        cudaLaunchAttribute attr[1];
        const cudaLaunchConfig_t cfg =
            pdl_config(dim3(grid), dim3(kQuadThreads), smem, as_cuda(stream), attr);
        if (cudaLaunchKernelExC(&cfg, fn, args) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        return launch_status();
    }

    // Rows per tile: about 8 KB of logits (16 KB for top-1, whose rows are
    // short), and small enough that every SM gets at least two tiles (each row
    // is a serial chain of warp reductions, so the rows are spread over as
    // many resident warps as possible).
    int R = ((p->k_max == 1 && G == 1 ? 4096 : 2048) / E) / 8 * 8;
    const int64_t spread = ((T + 2 * sms - 1) / (2 * sms) + 7) / 8 * 8;
    if (spread < R) R = (int)spread;
    R = R < 8 ? 8 : (R > 256 ? 256 : R);
    a.R = R;
    a.ntiles = (T + R - 1) / R;

    const int vpl_need = vec ? 4 * ((E + 127) / 128) : (E + 31) / 32;
    const int vpl = vpl_need <= 4 ? 4 : vpl_need <= 8 ? 8 : vpl_need <= 12 ? 12 : 16;
    const bool top1 = p->k_max == 1 && G == 1;
    void *fn = vec ? route_fn<true>(vpl, top1) : route_fn<false>(vpl, top1);
    const size_t smem = (size_t)kStages * R * E * sizeof(float) + (size_t)kStages * R * sizeof(int32_t) +
                        kStages * sizeof(uint64_t) +
                        (a.group_mode == 3 ? (size_t)kRouteWarps * kMaxE * sizeof(float) : 0);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kRouteWarps * 32, smem) !=
            cudaSuccess ||
        per_sm < 1) {
        cudaGetLastError();
        per_sm = 1;
    }
    const int64_t cap = (int64_t)sms * per_sm;
    const unsigned grid = (unsigned)(a.ntiles < cap ? a.ntiles : cap);
    void *args[] = {&a};
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg =
        pdl_config(dim3(grid), dim3(kRouteWarps * 32), smem, as_cuda(stream), attr);
    if (cudaLaunchKernelExC(&cfg, fn, args) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
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
    const int64_t cap = (int64_t)sm_count() * 8;
    if (logits && p->score == MOE_SCORE_SOFTMAX && !p->renormalize) {
        // full-row softmax statistics: one warp a token
        const int64_t blocks_needed = (T + 7) / 8;
        hash_route_kernel<<<(unsigned)(blocks_needed < cap ? blocks_needed : cap), 256, 0,
                            as_cuda(stream)>>>(a);
        return launch_status();
    }
    const int W = k <= 4 ? 4 : k <= 8 ? 8 : k <= 16 ? 16 : 32;
    const int64_t per_block = 8 * (32 / W);
    const int64_t blocks_needed = (T + per_block - 1) / per_block;
    const unsigned grid = (unsigned)(blocks_needed < cap ? blocks_needed : cap);
    cudaError_t err;
    switch (W) {
        case 4: err = launch_pdl(hash_route_grouped_kernel<4>, dim3(grid), dim3(256), 0, as_cuda(stream), a); break;
        case 8: err = launch_pdl(hash_route_grouped_kernel<8>, dim3(grid), dim3(256), 0, as_cuda(stream), a); break;
        case 16: err = launch_pdl(hash_route_grouped_kernel<16>, dim3(grid), dim3(256), 0, as_cuda(stream), a); break;
        default: err = launch_pdl(hash_route_grouped_kernel<32>, dim3(grid), dim3(256), 0, as_cuda(stream), a); break;
    }
    if (err != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return launch_status();
}
