// moe_dispatch: per-expert histogram, exclusive scan and stable scatter of the
// T*k_max routing slots into expert-contiguous order.
//
// Definition: counts[e] = #slots with id e; offsets = exclusive scan of counts;
// walking the slots in flat order a = t*k_max + j, slot a with id e gets
// pos = offsets[e] + (number of earlier slots with id e); sorted_token[pos] = t,
// dest_pos[a] = pos (-1 for empty slots).
//
// B200 design: a batch of at most 1024 slots is one block in one launch
// (dispatch_single_kernel).  Larger batches take two short launches with no
// inter-block waiting.  The slots are cut
// into S block segments of 8 warps x ITEMS items x 32 lanes, each warp owning a
// contiguous sub-segment.
//   1. count:   every block builds its segment's histogram in shared memory
//               with warp-aggregated updates (__match_any_sync: one leader per
//               distinct id adds the popcount of its peers) and stores it.
//   2. scatter: every warp loads its sub-segment's ids into registers while
//               the block loads the segment totals of the whole grid (16-byte
//               loads, all in flight together), so the kernel waits on memory
//               once.  The block sums all S totals (for counts) and those
//               before it (for its own base), scans counts into offsets
//               (block 0 writes counts and offsets), rebuilds its warps'
//               histograms from the ids in registers, and every warp walks
//               its ids in order, ranking each slot among its peers with the
//               same id (popcount of lower lanes in the match mask), writing
//               sorted_token and dest_pos.
// Above 296 segments of 16 items a lane (1,212,416 slots) each segment takes
// several rounds of 4096 slots (its block carries per-expert running counts
// from round to round), so S stays at most 296 and the totals each scatter
// block sums stay bounded (without rounds, 8 M slots measured 2.4x the time
// of 4 M, from re-summing S x E totals).
// Workspace: seg_total [S][Ep] int32, Ep = E rounded up to a multiple of 4.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kDispWarps = 8;
constexpr int kMaxE = 512;
constexpr int kSumUnroll = 16;  // independent 16-byte segment-total loads in flight per thread
constexpr int kMaxPad = 4096;   // largest block padding of moe_dispatch_limited

int warp_items(int64_t n_flat) {
    int items = 4;
    while ((int64_t)items * 32 * kDispWarps * 148 < n_flat && items < 16) items *= 2;
    return items;
}

// Above kMaxSegments segments of 16 items a lane (1,212,416 slots) a segment
// takes several rounds of 8 warps x 16 items x 32 lanes, so that the totals
// every scatter block sums (segments x experts) stay bounded.
constexpr int64_t kMaxSegments = 2 * 148;

int seg_rounds(int64_t n_flat, int items) {
    const int64_t seg = (int64_t)items * 32 * kDispWarps;
    const int64_t s1 = (n_flat + seg - 1) / seg;
    return s1 <= kMaxSegments ? 1 : (int)((s1 + kMaxSegments - 1) / kMaxSegments);
}

int64_t num_segments(int64_t n_flat, int items) {
    const int64_t seg = (int64_t)items * 32 * kDispWarps * seg_rounds(n_flat, items);
    return (n_flat + seg - 1) / seg;
}

// Row stride of seg_total: whole 16-byte quads per segment.
int seg_stride(int E) { return (E + 3) / 4 * 4; }

__device__ __forceinline__ int load_id(const int32_t *ids, int64_t a, int64_t n_flat, int E,
                                       bool &bad) {
    int e = a < n_flat ? ids[a] : -1;
    if (e < -1 || e >= E) {
        bad = true;
        e = -1;
    }
    return e;
}

// The first slot of warp `warp`'s sub-segment in round r of segment s.
template <int ITEMS>
__device__ __forceinline__ int64_t round_base(int64_t s, int rounds, int r, int warp) {
    return ((s * rounds + r) * kDispWarps + warp) * (int64_t)ITEMS * 32;
}

template <int ITEMS>
__global__ void __launch_bounds__(kDispWarps * 32)
    dispatch_count_kernel(const int32_t *__restrict__ ids, int64_t n_flat, int E, int Ep,
                          int rounds, int32_t *__restrict__ seg_total, int32_t *status) {
    __shared__ int32_t hist[kMaxE];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t s = blockIdx.x;
    for (int e = threadIdx.x; e < Ep; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    griddep_wait();
    bool bad = false;
    for (int r = 0; r < rounds; ++r) {
        const int64_t base = round_base<ITEMS>(s, rounds, r, warp);
        int eb[ITEMS];  // every load of the sub-segment is issued before any is used
#pragma unroll
        for (int j = 0; j < ITEMS; ++j)
            eb[j] = load_id(ids, base + (int64_t)j * 32 + lane, n_flat, E, bad);
#pragma unroll
        for (int j = 0; j < ITEMS; ++j) {
            const int e = eb[j];
            const unsigned peers = __match_any_sync(MOE_FULL_MASK, e);
            if (e >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[e], __popc(peers));
        }
    }
    if (__any_sync(MOE_FULL_MASK, bad) && lane == 0) report(status, MOE_ERR_DEVICE_INDEX);
    __syncthreads();
    for (int e = threadIdx.x; e < Ep; e += blockDim.x) seg_total[s * Ep + e] = hist[e];
    griddep_launch_dependents();
}

// A per-expert capacity and block padding (moe_dispatch_limited); the plain
// dispatch is cap = INT32_MAX, pad = 1 with LIMITED = false.
struct Limits {
    int32_t cap;       // slots kept per expert, in flat order
    int32_t pad;       // expert blocks rounded up to a multiple of this many rows
    int32_t *dropped;  // nullable: number of slots over capacity
};

// Shared memory of a block that scatters one segment.
struct ScatterSmem {
    int32_t total[kMaxE];              // totals per expert, then the expert blocks' offsets
    int32_t before[kMaxE];             // slots of each expert in earlier segments
    int32_t hist[kDispWarps][kMaxE];   // per-warp histograms, then each warp's first rank
    int32_t wsum[kDispWarps];
    int32_t kept[kMaxE];               // with limits: kept slots per expert
    int32_t racc[kMaxE];               // slots of each expert in this segment's earlier rounds
    int32_t drop;
};

// Segment s (of S) once sh.total holds the per-expert totals: exclusive scan
// of the expert blocks (the totals, or with limits the kept slots rounded up
// to the padding) into offsets, left in sh.total; segment 0 writes counts,
// offsets and the dropped count; with padding, the padding rows of the expert
// blocks (experts shared out over the segments).
template <bool LIMITED>
__device__ __forceinline__ void scatter_offsets(ScatterSmem &sh, int64_t s, int64_t S, int E,
                                                int32_t *__restrict__ counts,
                                                int32_t *__restrict__ offsets,
                                                int32_t *__restrict__ sorted_token,
                                                const Limits &lim) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // Exclusive scan of the block sizes (the totals, or with limits the kept
    // slots rounded up to the padding) into offsets: thread i owns experts 2i,
    // 2i+1.
    {
        const int i0 = 2 * threadIdx.x, i1 = i0 + 1;
        const int32_t n0 = i0 < E ? sh.total[i0] : 0;
        const int32_t n1 = i1 < E ? sh.total[i1] : 0;
        int32_t c0 = n0, c1 = n1;
        if (LIMITED) {
            if (threadIdx.x == 0) sh.drop = 0;
            const int32_t k0 = min(n0, lim.cap), k1 = min(n1, lim.cap);
            if (i0 < E) sh.kept[i0] = k0;
            if (i1 < E) sh.kept[i1] = k1;
            c0 = (k0 + lim.pad - 1) / lim.pad * lim.pad;
            c1 = (k1 + lim.pad - 1) / lim.pad * lim.pad;
            __syncthreads();
            const int32_t over = (n0 - k0) + (n1 - k1);
            if (s == 0 && over) atomicAdd(&sh.drop, over);
        }
        const int32_t v = c0 + c1;
        int32_t incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t n = __shfl_up_sync(MOE_FULL_MASK, incl, o);
            if (lane >= o) incl += n;
        }
        if (lane == 31) sh.wsum[warp] = incl;
        __syncthreads();
        int32_t pre = 0;
        for (int w = 0; w < warp; ++w) pre += sh.wsum[w];
        const int32_t excl = pre + incl - v;
        if (s == 0) {
            if (i0 < E) {
                counts[i0] = n0;
                offsets[i0] = excl;
            }
            if (i1 < E) {
                counts[i1] = n1;
                offsets[i1] = excl + c0;
            }
            if (threadIdx.x == 0) {
                int32_t all = 0;
                for (int w = 0; w < kDispWarps; ++w) all += sh.wsum[w];
                offsets[E] = all;
                if (LIMITED && lim.dropped) *lim.dropped = sh.drop;
            }
        }
        __syncthreads();
        if (i0 < E) sh.total[i0] = excl;
        if (i1 < E) sh.total[i1] = excl + c0;
        __syncthreads();
    }
    if (LIMITED) {
        // The padding rows of expert blocks (experts shared out over blocks).
        for (int e = (int)s; e < E; e += (int)S) {
            const int32_t lo = sh.total[e] + sh.kept[e];
            const int32_t hi = sh.total[e] + (sh.kept[e] + lim.pad - 1) / lim.pad * lim.pad;
            for (int32_t p = lo + (int32_t)threadIdx.x; p < hi; p += (int32_t)blockDim.x)
                sorted_token[p] = -1;
        }
    }
}

// One round of a segment once the warps' histograms of the round are in
// place: each warp's first rank per expert (earlier segments, earlier rounds
// of this segment, earlier warps of this round; without limits the block
// offset as well), then the stable scatter of the warp's slots (ids eb, peer
// masks pm, in registers).  Leaves sh.racc counting this round too.
template <int ITEMS, bool LIMITED>
__device__ __forceinline__ void scatter_round(ScatterSmem &sh, int64_t base, int64_t n_flat,
                                              int k_max, int E, const int (&eb)[ITEMS],
                                              const unsigned (&pm)[ITEMS],
                                              int32_t *__restrict__ sorted_token,
                                              int32_t *__restrict__ dest_pos, const Limits &lim) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t b = (LIMITED ? 0 : sh.total[e]) + sh.before[e] + sh.racc[e];
        int32_t here = 0;
#pragma unroll
        for (int w = 0; w < kDispWarps; ++w) {
            const int32_t h = sh.hist[w][e];
            sh.hist[w][e] = b;
            b += h;
            here += h;
        }
        sh.racc[e] += here;
    }
    __syncthreads();

    int32_t *run = sh.hist[warp];
    const unsigned lower = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < ITEMS; ++j) {
        const int64_t a = base + (int64_t)j * 32 + lane;
        const int e = eb[j];
        const unsigned peers = pm[j];
        if (e >= 0) {
            int32_t pos = run[e] + __popc(peers & lower);
            if (LIMITED) pos = pos < lim.cap ? sh.total[e] + pos : -1;
            if (pos >= 0) sorted_token[pos] = (int32_t)(a / k_max);
            dest_pos[a] = pos;
        } else if (a < n_flat) {
            dest_pos[a] = -1;
        }
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) run[e] += __popc(peers);
        __syncwarp();
    }
}

template <int ITEMS, bool LIMITED>
__global__ void __launch_bounds__(kDispWarps * 32)
    dispatch_scatter_kernel(const int32_t *__restrict__ ids, int64_t n_flat, int k_max, int E,
                            int Ep, int64_t S, int rounds, const int32_t *__restrict__ seg_total,
                            int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                            int32_t *__restrict__ sorted_token, int32_t *__restrict__ dest_pos,
                            Limits lim) {
    __shared__ ScatterSmem sh;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t s = blockIdx.x;

    for (int e = threadIdx.x; e < Ep; e += blockDim.x) {
        sh.total[e] = 0;
        sh.before[e] = 0;
        sh.racc[e] = 0;
    }
    for (int i = threadIdx.x; i < kDispWarps * Ep; i += blockDim.x) sh.hist[i / Ep][i % Ep] = 0;
    __syncthreads();
    griddep_wait();

    // This warp's ids of the first round, loaded while the totals below are
    // summed.  An id outside [-1, E) counts as empty here; the count kernel
    // reported it.
    int64_t base = round_base<ITEMS>(s, rounds, 0, warp);
    bool bad = false;
    int eb[ITEMS];
#pragma unroll
    for (int j = 0; j < ITEMS; ++j) eb[j] = load_id(ids, base + (int64_t)j * 32 + lane, n_flat, E, bad);

    // Per-expert totals over all segments and over the segments before this
    // one.  Thread = (quad q of 4 experts, segment residue r); nsr residues
    // walk the segments in steps of nsr, kSumUnroll 16-byte loads in flight.
    {
        const int Q = Ep / 4;
        const int nsr = (int)blockDim.x / Q;
        const int q = (int)threadIdx.x % Q, r = (int)threadIdx.x / Q;
        if (r < nsr) {
            const int4 *st4 = reinterpret_cast<const int4 *>(seg_total);
            int4 at = make_int4(0, 0, 0, 0), ab = make_int4(0, 0, 0, 0);
            for (int64_t sp0 = r; sp0 < S; sp0 += (int64_t)nsr * kSumUnroll) {
                int4 v[kSumUnroll];
#pragma unroll
                for (int u = 0; u < kSumUnroll; ++u) {
                    const int64_t sp = sp0 + (int64_t)u * nsr;
                    v[u] = sp < S ? st4[sp * Q + q] : make_int4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < kSumUnroll; ++u) {
                    at.x += v[u].x;
                    at.y += v[u].y;
                    at.z += v[u].z;
                    at.w += v[u].w;
                    if (sp0 + (int64_t)u * nsr < s) {
                        ab.x += v[u].x;
                        ab.y += v[u].y;
                        ab.z += v[u].z;
                        ab.w += v[u].w;
                    }
                }
            }
            atomicAdd(&sh.total[4 * q + 0], at.x);
            atomicAdd(&sh.total[4 * q + 1], at.y);
            atomicAdd(&sh.total[4 * q + 2], at.z);
            atomicAdd(&sh.total[4 * q + 3], at.w);
            atomicAdd(&sh.before[4 * q + 0], ab.x);
            atomicAdd(&sh.before[4 * q + 1], ab.y);
            atomicAdd(&sh.before[4 * q + 2], ab.z);
            atomicAdd(&sh.before[4 * q + 3], ab.w);
        }
    }

    __syncthreads();
    scatter_offsets<LIMITED>(sh, s, S, E, counts, offsets, sorted_token, lim);

    for (int r = 0; r < rounds; ++r) {
        if (r > 0) {
            base = round_base<ITEMS>(s, rounds, r, warp);
#pragma unroll
            for (int j = 0; j < ITEMS; ++j)
                eb[j] = load_id(ids, base + (int64_t)j * 32 + lane, n_flat, E, bad);
            // the last round's running ranks are done with: fresh histograms
            for (int i = threadIdx.x; i < kDispWarps * Ep; i += blockDim.x)
                sh.hist[i / Ep][i % Ep] = 0;
            __syncthreads();
        }
        // This warp's histogram of the round, from the ids in registers (one
        // leader per id).
        unsigned pm[ITEMS];
#pragma unroll
        for (int j = 0; j < ITEMS; ++j) {
            const int e = eb[j];
            pm[j] = __match_any_sync(MOE_FULL_MASK, e);
            if (e >= 0 && lane == __ffs(pm[j]) - 1) sh.hist[warp][e] += __popc(pm[j]);
            __syncwarp();
        }
        __syncthreads();
        scatter_round<ITEMS, LIMITED>(sh, base, n_flat, k_max, E, eb, pm, sorted_token, dest_pos,
                                      lim);
        __syncthreads();
    }
    griddep_launch_dependents();
}

// ------------------------------------------------------ one-block dispatch
// A batch whose slots fit one segment of 4 items a lane (at most 1024 slots: a
// decode-sized batch) is dispatched by a single block in one launch: its histogram is the
// whole histogram, no segment comes before it, and the scatter follows
// directly; no workspace is touched.
template <int ITEMS, bool LIMITED>
__global__ void __launch_bounds__(kDispWarps * 32)
    dispatch_single_kernel(const int32_t *__restrict__ ids, int64_t n_flat, int k_max, int E,
                           int Ep, int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                           int32_t *__restrict__ sorted_token, int32_t *__restrict__ dest_pos,
                           Limits lim, int32_t *status) {
    __shared__ ScatterSmem sh;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < kDispWarps * Ep; i += blockDim.x) sh.hist[i / Ep][i % Ep] = 0;
    __syncthreads();
    griddep_wait();
    const int64_t base = (int64_t)warp * ITEMS * 32;
    bool bad = false;
    int eb[ITEMS];
#pragma unroll
    for (int j = 0; j < ITEMS; ++j) eb[j] = load_id(ids, base + (int64_t)j * 32 + lane, n_flat, E, bad);
    if (__any_sync(MOE_FULL_MASK, bad) && lane == 0) report(status, MOE_ERR_DEVICE_INDEX);
    unsigned pm[ITEMS];
#pragma unroll
    for (int j = 0; j < ITEMS; ++j) {
        const int e = eb[j];
        pm[j] = __match_any_sync(MOE_FULL_MASK, e);
        if (e >= 0 && lane == __ffs(pm[j]) - 1) sh.hist[warp][e] += __popc(pm[j]);
        __syncwarp();
    }
    __syncthreads();
    for (int e = threadIdx.x; e < Ep; e += blockDim.x) {
        int32_t c = 0;
#pragma unroll
        for (int w = 0; w < kDispWarps; ++w) c += sh.hist[w][e];
        sh.total[e] = c;
        sh.before[e] = 0;
        sh.racc[e] = 0;
    }
    __syncthreads();
    scatter_offsets<LIMITED>(sh, 0, 1, E, counts, offsets, sorted_token, lim);
    scatter_round<ITEMS, LIMITED>(sh, base, n_flat, k_max, E, eb, pm, sorted_token, dest_pos, lim);
    griddep_launch_dependents();
}

// Launches the dispatch: one block when every slot fits one segment of 4
// items a lane (1024 slots: 8.3 against 11.4 us at 512 slots, while at 4096
// slots, 16 items a lane in one block measured 14.4 against 11.6 us for four
// blocks and two launches), else count + scatter over S segments of `items`
// items a lane (segment totals in the workspace).
template <bool LIMITED>
cudaError_t launch_dispatch(int items, int rounds, int64_t S, cudaStream_t cs, const int32_t *ids,
                            int64_t n_flat, int k_max, int E, int32_t *seg_total,
                            int32_t *counts, int32_t *offsets, int32_t *sorted_token,
                            int32_t *dest_pos, int32_t *d_status, Limits lim) {
    const int Ep = seg_stride(E);
    const dim3 block(kDispWarps * 32);
    if (n_flat <= 4 * 32 * kDispWarps)
        return launch_pdl(dispatch_single_kernel<4, LIMITED>, dim3(1), block, 0, cs, ids, n_flat,
                          k_max, E, Ep, counts, offsets, sorted_token, dest_pos, lim, d_status);
    const dim3 grid((unsigned)S);
    cudaError_t err;
#define MOE_DISPATCH_CASE(IT)                                                                     \
    case IT:                                                                                      \
        err = launch_pdl(dispatch_count_kernel<IT>, grid, block, 0, cs, ids, n_flat, E, Ep,       \
                         rounds, seg_total, d_status);                                            \
        if (err != cudaSuccess) return err;                                                       \
        return launch_pdl(dispatch_scatter_kernel<IT, LIMITED>, grid, block, 0, cs, ids, n_flat,  \
                          k_max, E, Ep, S, rounds, (const int32_t *)seg_total, counts, offsets,   \
                          sorted_token, dest_pos, lim);
    switch (items) {
        MOE_DISPATCH_CASE(4)
        MOE_DISPATCH_CASE(8)
        MOE_DISPATCH_CASE(16)
        default:
            return cudaErrorInvalidValue;
    }
#undef MOE_DISPATCH_CASE
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_dispatch_workspace_size(int64_t T, int32_t k_max, int32_t E,
                                                  size_t *bytes) {
    using namespace moe;
    if (!bytes || T < 0 || k_max < 0 || k_max > 32 || E < 1 || E > kMaxE)
        return MOE_ERR_INVALID_ARG;
    const int64_t n_flat = T * (int64_t)k_max;
    if (n_flat >= (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
    const int64_t S = num_segments(n_flat, warp_items(n_flat));
    const size_t b = (size_t)S * (size_t)seg_stride(E) * sizeof(int32_t);
    *bytes = (b + 255) / 256 * 256;
    return MOE_OK;
}

extern "C" moe_status moe_dispatch(const int32_t *topk_ids, int64_t T, int32_t k_max, int32_t E,
                                   int32_t *counts, int32_t *offsets, int32_t *sorted_token,
                                   int32_t *dest_pos, void *workspace, size_t ws_bytes,
                                   int32_t *d_status, moe_stream_t stream) {
    using namespace moe;
    size_t need = 0;
    moe_status st = moe_dispatch_workspace_size(T, k_max, E, &need);
    if (st != MOE_OK) return st;
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    const int64_t n_flat = T * (int64_t)k_max;
    if (n_flat > 0 && (!topk_ids || !sorted_token || !dest_pos || !workspace))
        return MOE_ERR_INVALID_ARG;
    if (n_flat > 0 && ((reinterpret_cast<uintptr_t>(workspace) & 255u) || ws_bytes < need))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t cs = as_cuda(stream);
    const int items = warp_items(n_flat);
    const int64_t S = num_segments(n_flat, items);
    if (S > 0) {
        if (launch_dispatch<false>(items, seg_rounds(n_flat, items), S, cs, topk_ids, n_flat, (int)k_max, (int)E,
                                   static_cast<int32_t *>(workspace), counts, offsets,
                                   sorted_token, dest_pos, d_status,
                                   Limits{INT32_MAX, 1, nullptr}) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
    } else {
        // No slots: every count and every offset is 0.
        if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, cs) != cudaSuccess ||
            cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), cs) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
    }
    return launch_status();
}

// ------------------------------------------- dispatch with capacity/padding
extern "C" moe_status moe_dispatch_limited_rows(int64_t T, int32_t k_max, int32_t E,
                                                int32_t capacity, int32_t pad, int64_t *rows) {
    using namespace moe;
    if (!rows || T < 0 || k_max < 0 || k_max > 32 || E < 1 || E > kMaxE || capacity < 0 ||
        pad < 1 || pad > kMaxPad)
        return MOE_ERR_INVALID_ARG;
    const int64_t n_flat = T * (int64_t)k_max;
    int64_t kept = n_flat;
    if (capacity > 0 && (int64_t)capacity * E < kept) kept = (int64_t)capacity * E;
    const int64_t r = kept + (int64_t)E * (pad - 1);
    if (n_flat >= (int64_t)INT32_MAX || r >= (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
    *rows = r;
    return MOE_OK;
}

extern "C" moe_status moe_dispatch_limited(const int32_t *topk_ids, int64_t T, int32_t k_max,
                                           int32_t E, int32_t capacity, int32_t pad,
                                           int32_t *counts, int32_t *offsets,
                                           int32_t *sorted_token, int64_t sorted_rows,
                                           int32_t *dest_pos, int32_t *dropped, void *workspace,
                                           size_t ws_bytes, int32_t *d_status,
                                           moe_stream_t stream) {
    using namespace moe;
    int64_t bound = 0;
    moe_status st = moe_dispatch_limited_rows(T, k_max, E, capacity, pad, &bound);
    if (st != MOE_OK) return st;
    size_t need = 0;
    st = moe_dispatch_workspace_size(T, k_max, E, &need);
    if (st != MOE_OK) return st;
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    const int64_t n_flat = T * (int64_t)k_max;
    if (n_flat > 0 && (!topk_ids || !sorted_token || !dest_pos || !workspace))
        return MOE_ERR_INVALID_ARG;
    if (n_flat > 0 && ((reinterpret_cast<uintptr_t>(workspace) & 255u) || ws_bytes < need ||
                       sorted_rows < bound))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t cs = as_cuda(stream);
    const int items = warp_items(n_flat);
    const int64_t S = num_segments(n_flat, items);
    if (S > 0) {
        const Limits lim{capacity > 0 ? capacity : INT32_MAX, pad, dropped};
        if (launch_dispatch<true>(items, seg_rounds(n_flat, items), S, cs, topk_ids, n_flat, (int)k_max, (int)E,
                                  static_cast<int32_t *>(workspace), counts, offsets, sorted_token,
                                  dest_pos, d_status, lim) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
    } else {
        if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, cs) != cudaSuccess ||
            cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), cs) != cudaSuccess ||
            (dropped && cudaMemsetAsync(dropped, 0, sizeof(int32_t), cs) != cudaSuccess)) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
    }
    return launch_status();
}

// ------------------------------------------------- dispatch, no caller scratch
// A variant of moe_dispatch for callers that cannot allocate device memory
// themselves.  Its scratch is this file-scope device array: every GPU that
// loads the library holds these 4 MiB until the process exits.  Host code must
// not pass the array's name to a kernel (on the host it is only a stand-in);
// the device address is fetched with cudaGetSymbolAddress in the calling
// thread's current context and cached under that context's unique id, so a
// context that is destroyed and created again (cudaDeviceReset, a primary
// context released and retained again) is looked up afresh instead of reusing
// an address of the old one.
namespace moe {
namespace {
// The most moe_dispatch_workspace_size() returns for any size it accepts:
// kMaxSegments segments of 512 experts (606,208 bytes), so no accepted size is
// refused for want of scratch.
constexpr size_t kStaticScratchBytes = size_t(kMaxSegments) * kMaxE * sizeof(int32_t);
static_assert(kStaticScratchBytes % 256 == 0, "workspace sizes are rounded to 256 bytes");
constexpr int kScratchCacheSlots = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

template <typename Fn>
Fn driver_fn(const char *name) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return reinterpret_cast<Fn>(p);
}

// Unique id (for the life of the process) of the calling thread's current
// context; false when no context is current or the driver cannot tell.
bool current_context_id(unsigned long long &id) {
    static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    CUcontext ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, &id) == CUDA_SUCCESS;
}

// (context id -> scratch address) of the contexts seen so far; a full table
// overwrites its oldest entry.  Context ids are never reused, so an entry of a
// destroyed context can only go unused, never match a new one.
struct ScratchCache {
    std::mutex mu;
    unsigned long long ctx[kScratchCacheSlots] = {};
    void *addr[kScratchCacheSlots] = {};
    int next = 0;
};
ScratchCache g_scratch_cache;
}  // namespace
}  // namespace moe

static __device__ __align__(256) int32_t g_dispatch_scratch[moe::kStaticScratchBytes / sizeof(int32_t)];

namespace moe {
namespace {
// Device address of g_dispatch_scratch in the current context (looked up on
// the first call in each context, with cudaGetSymbolAddress; that lookup may
// create the device's primary context, so it must not run inside a stream
// capture), or nullptr on a CUDA error.
void *static_scratch() {
    unsigned long long id = 0;
    bool have_id = current_context_id(id);
    if (have_id) {
        std::lock_guard<std::mutex> lock(g_scratch_cache.mu);
        for (int i = 0; i < kScratchCacheSlots; ++i)
            if (g_scratch_cache.ctx[i] == id && g_scratch_cache.addr[i]) return g_scratch_cache.addr[i];
    }
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_dispatch_scratch) != cudaSuccess || !addr) {
        cudaGetLastError();
        return nullptr;
    }
    // The lookup makes the device's primary context current if none was.
    if (!have_id) have_id = current_context_id(id);
    if (have_id) {
        std::lock_guard<std::mutex> lock(g_scratch_cache.mu);
        const int i = g_scratch_cache.next;
        g_scratch_cache.ctx[i] = id;
        g_scratch_cache.addr[i] = addr;
        g_scratch_cache.next = (i + 1) % kScratchCacheSlots;
    }
    return addr;
}
}  // namespace
}  // namespace moe

extern "C" moe_status moe_dispatch_static(const int32_t *topk_ids, int64_t T, int32_t k_max,
                                          int32_t E, int32_t *counts, int32_t *offsets,
                                          int32_t *sorted_token, int32_t *dest_pos,
                                          int32_t *d_status, moe_stream_t stream) {
    using namespace moe;
    size_t need = 0;
    moe_status st = moe_dispatch_workspace_size(T, k_max, E, &need);
    if (st != MOE_OK) return st;
    if (need > kStaticScratchBytes) return MOE_ERR_UNSUPPORTED;  // (cannot happen: see above)
    void *addr = static_scratch();
    if (!addr) return MOE_ERR_CUDA;
    // Every scratch entry a dispatch reads is written earlier by the same
    // dispatch, so the array needs no clearing between calls.
    return moe_dispatch(topk_ids, T, k_max, E, counts, offsets, sorted_token, dest_pos, addr,
                        kStaticScratchBytes, d_status, stream);
}
