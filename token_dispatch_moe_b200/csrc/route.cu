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
#define MOE_ROUTE_QUAD_HOST_ONLY
#include "route_quad.cuh"

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
    // follow each token's own k.  With per-request k of 4, 8 or 16 over 128
    // experts (qwen3_dynk) a 16-word network measured 30.7 us, two passes of 8
    // (the second only where a row needs it) 22.8 us, and this kernel 21.9 us.
    if (vec && p->k_max >= 1 && p->k_max <= 8 && (G == 1 || a.cpg > 0)) {
        const int nch_t = a.nch <= 8 ? 8 : a.nch <= 16 ? 16 : a.nch <= 24 ? 24 : 32;
        const size_t smem = (size_t)kQuadWarps * nch_t * 512 + (size_t)((E + 3) & ~3) * 4 +
                            (size_t)(kQuadThreads / 4) * kQuadGroupStride * 4 +
                            (a.group_mode == 3 ? (size_t)kQuadWarps * kRouteMaxE * 4 : 0);
        int P = 1;
        while (P < p->k_max) P *= 2;
        const bool fixed_words = a.keys_from_scores && (p->score == MOE_SCORE_SIGMOID ||
                                                         p->score == MOE_SCORE_SOFTMAX);
        void *fn = fixed_words ? route_quad_fn_fixed(P, a.nch) : route_quad_fn_float(P, a.nch);
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
