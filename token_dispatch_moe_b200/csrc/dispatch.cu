// moe_dispatch: per-expert histogram, exclusive scan and stable scatter of the
// T*k_max routing slots into expert-contiguous order.
//
// Definition: counts[e] = #slots with id e; offsets = exclusive scan of counts;
// walking the slots in flat order a = t*k_max + j, slot a with id e gets
// pos = offsets[e] + (number of earlier slots with id e); sorted_token[pos] = t,
// dest_pos[a] = pos (-1 for empty slots).
//
// B200 design: two short launches, no inter-block waiting.  The slots are cut
// into S block segments of 8 warps x W items x 32 lanes, each warp owning a
// contiguous sub-segment.
//   1. count:   every warp builds its sub-segment's histogram in shared memory
//               with warp-aggregated updates (__match_any_sync: one leader per
//               distinct id adds the popcount of its peers) and stores it; the
//               block also stores its segment's total per expert.
//   2. scatter: each block sums the segment totals of the whole grid (all S,
//               for counts; those before it, for its own base) straight from
//               L2, scans counts into offsets (block 0 writes counts and
//               offsets), adds the per-warp histograms of the earlier warps of
//               its segment, then every warp walks its sub-segment again in
//               order, ranks each slot among its peers with the same id
//               (popcount of lower lanes in the match mask) and writes
//               sorted_token and dest_pos.
// Workspace: seg_total [S][E] and warp_hist [S][8][E], int32.
#include <atomic>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kDispWarps = 8;
constexpr int kMaxE = 512;
constexpr int kBatch = 4;  // slot loads issued together per lane (items is a multiple)
constexpr int kSumUnroll = 16;  // independent segment-total loads in flight per thread
constexpr int kMaxPad = 4096;   // largest block padding of moe_dispatch_limited

int warp_items(int64_t n_flat) {
    int items = 4;
    while ((int64_t)items * 32 * kDispWarps * 148 < n_flat && items < 16) items *= 2;
    return items;
}

int64_t num_segments(int64_t n_flat, int items) {
    const int64_t seg = (int64_t)items * 32 * kDispWarps;
    return (n_flat + seg - 1) / seg;
}

__device__ __forceinline__ int load_id(const int32_t *ids, int64_t a, int64_t n_flat, int E,
                                       bool &bad) {
    int e = a < n_flat ? ids[a] : -1;
    if (e < -1 || e >= E) {
        bad = true;
        e = -1;
    }
    return e;
}

__global__ void __launch_bounds__(kDispWarps * 32)
    dispatch_count_kernel(const int32_t *__restrict__ ids, int64_t n_flat, int E, int items,
                          int32_t *__restrict__ seg_total, int32_t *__restrict__ warp_hist,
                          int32_t *status) {
    __shared__ int32_t hist[kDispWarps][kMaxE];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t s = blockIdx.x;
    for (int e = lane; e < E; e += 32) hist[warp][e] = 0;
    __syncwarp();
    griddep_wait();
    const int64_t base = (s * kDispWarps + warp) * (int64_t)items * 32;
    bool bad = false;
    for (int i0 = 0; i0 < items; i0 += kBatch) {
        int eb[kBatch];  // loads of a batch are issued before any of them is used
#pragma unroll
        for (int j = 0; j < kBatch; ++j)
            eb[j] = load_id(ids, base + (int64_t)(i0 + j) * 32 + lane, n_flat, E, bad);
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const int e = eb[j];
            const unsigned peers = __match_any_sync(MOE_FULL_MASK, e);
            if (e >= 0 && lane == __ffs(peers) - 1) hist[warp][e] += __popc(peers);
            __syncwarp();
        }
    }
    if (__any_sync(MOE_FULL_MASK, bad) && lane == 0) report(status, MOE_ERR_DEVICE_INDEX);
    int32_t *wh = warp_hist + (s * kDispWarps + warp) * E;
    for (int e = lane; e < E; e += 32) wh[e] = hist[warp][e];
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t t = 0;
#pragma unroll
        for (int w = 0; w < kDispWarps; ++w) t += hist[w][e];
        seg_total[s * E + e] = t;
    }
    griddep_launch_dependents();
}

// A per-expert capacity and block padding (moe_dispatch_limited); the plain
// dispatch is cap = INT32_MAX, pad = 1 with LIMITED = false.
struct Limits {
    int32_t cap;       // slots kept per expert, in flat order
    int32_t pad;       // expert blocks rounded up to a multiple of this many rows
    int32_t *dropped;  // nullable: number of slots over capacity
};

template <bool LIMITED>
__global__ void __launch_bounds__(kDispWarps * 32)
    dispatch_scatter_kernel(const int32_t *__restrict__ ids, int64_t n_flat, int k_max, int E,
                            int items, int64_t S, const int32_t *__restrict__ seg_total,
                            const int32_t *__restrict__ warp_hist, int32_t *__restrict__ counts,
                            int32_t *__restrict__ offsets, int32_t *__restrict__ sorted_token,
                            int32_t *__restrict__ dest_pos, Limits lim) {
    __shared__ int32_t total[kMaxE + 1];
    __shared__ int32_t before[kMaxE];
    __shared__ int32_t run[kDispWarps][kMaxE];
    __shared__ int32_t wsum[kDispWarps];
    __shared__ int32_t kept_s[LIMITED ? kMaxE : 1];
    __shared__ int32_t drop_s;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t s = blockIdx.x;

    // Per-expert totals over all segments and over the segments before this one.
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        total[e] = 0;
        before[e] = 0;
    }
    __syncthreads();
    griddep_wait();
    // Lane = expert within a 32-wide chunk, warp = every 8th segment: each
    // load is a coalesced 128-byte line, and kSumUnroll of them are in flight
    // per thread before any is added.
    for (int c = 0; c < E; c += 32) {
        const int e = c + lane;
        int32_t acc_t = 0, acc_b = 0;
        for (int64_t sp0 = warp; sp0 < S; sp0 += (int64_t)kDispWarps * kSumUnroll) {
            int32_t v[kSumUnroll];
#pragma unroll
            for (int u = 0; u < kSumUnroll; ++u) {
                const int64_t sp = sp0 + (int64_t)u * kDispWarps;
                v[u] = (e < E && sp < S) ? seg_total[sp * E + e] : 0;
            }
#pragma unroll
            for (int u = 0; u < kSumUnroll; ++u) {
                acc_t += v[u];
                acc_b += (sp0 + (int64_t)u * kDispWarps < s) ? v[u] : 0;
            }
        }
        if (e < E) {
            atomicAdd(&total[e], acc_t);
            atomicAdd(&before[e], acc_b);
        }
    }
    __syncthreads();

    // Exclusive scan of the block sizes (the totals, or with limits the kept
    // slots rounded up to the padding) into offsets: thread i owns experts 2i,
    // 2i+1.
    {
        const int i0 = 2 * threadIdx.x, i1 = i0 + 1;
        const int32_t n0 = i0 < E ? total[i0] : 0;
        const int32_t n1 = i1 < E ? total[i1] : 0;
        int32_t c0 = n0, c1 = n1;
        if (LIMITED) {
            if (threadIdx.x == 0) drop_s = 0;
            const int32_t k0 = min(n0, lim.cap), k1 = min(n1, lim.cap);
            if (i0 < E) kept_s[i0] = k0;
            if (i1 < E) kept_s[i1] = k1;
            c0 = (k0 + lim.pad - 1) / lim.pad * lim.pad;
            c1 = (k1 + lim.pad - 1) / lim.pad * lim.pad;
            __syncthreads();
            const int32_t over = (n0 - k0) + (n1 - k1);
            if (blockIdx.x == 0 && over) atomicAdd(&drop_s, over);
        }
        const int32_t v = c0 + c1;
        int32_t incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t n = __shfl_up_sync(MOE_FULL_MASK, incl, o);
            if (lane >= o) incl += n;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        int32_t pre = 0;
        for (int w = 0; w < warp; ++w) pre += wsum[w];
        const int32_t excl = pre + incl - v;
        if (blockIdx.x == 0) {
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
                for (int w = 0; w < kDispWarps; ++w) all += wsum[w];
                offsets[E] = all;
                if (LIMITED && lim.dropped) *lim.dropped = drop_s;
            }
        }
        // Each warp's starting position per expert: offset + earlier segments +
        // earlier warps of this segment.
        __syncthreads();
        if (i0 < E) total[i0] = excl;
        if (i1 < E) total[i1] = excl + c0;
        __syncthreads();
    }
    if (LIMITED) {
        // The padding rows of expert blocks (experts shared out over blocks).
        for (int e = (int)blockIdx.x; e < E; e += (int)gridDim.x) {
            const int32_t lo = total[e] + kept_s[e];
            const int32_t hi = total[e] + (kept_s[e] + lim.pad - 1) / lim.pad * lim.pad;
            for (int32_t p = lo + (int32_t)threadIdx.x; p < hi; p += (int32_t)blockDim.x)
                sorted_token[p] = -1;
        }
    }
    // Each warp's first rank per expert (earlier segments + earlier warps of
    // this segment); without limits the block offset is folded in as well.
    const int32_t *wh = warp_hist + s * kDispWarps * E;
    int32_t *r = run[warp];
    for (int e = lane; e < E; e += 32) {
        int32_t v[kDispWarps];
#pragma unroll
        for (int w = 0; w < kDispWarps; ++w) v[w] = w < warp ? wh[w * E + e] : 0;
        int32_t b = (LIMITED ? 0 : total[e]) + before[e];
#pragma unroll
        for (int w = 0; w < kDispWarps; ++w) b += v[w];
        r[e] = b;
    }
    __syncwarp();

    const int64_t base = (s * kDispWarps + warp) * (int64_t)items * 32;
    const unsigned lower = (1u << lane) - 1u;
    bool bad = false;
    for (int i0 = 0; i0 < items; i0 += kBatch) {
        int eb[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j)
            eb[j] = load_id(ids, base + (int64_t)(i0 + j) * 32 + lane, n_flat, E, bad);
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const int64_t a = base + (int64_t)(i0 + j) * 32 + lane;
            const int e = eb[j];
            const unsigned peers = __match_any_sync(MOE_FULL_MASK, e);
            if (e >= 0) {
                int32_t pos = r[e] + __popc(peers & lower);
                if (LIMITED) pos = pos < lim.cap ? total[e] + pos : -1;
                if (pos >= 0) sorted_token[pos] = (int32_t)(a / k_max);
                dest_pos[a] = pos;
            } else if (a < n_flat) {
                dest_pos[a] = -1;
            }
            __syncwarp();
            if (e >= 0 && lane == __ffs(peers) - 1) r[e] += __popc(peers);
            __syncwarp();
        }
    }
    griddep_launch_dependents();
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
    const size_t b = (size_t)S * (size_t)E * sizeof(int32_t) * (1 + kDispWarps);
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
        int32_t *seg_total = static_cast<int32_t *>(workspace);
        int32_t *warp_hist = seg_total + S * E;
        if (launch_pdl(dispatch_count_kernel, dim3((unsigned)S), dim3(kDispWarps * 32), 0, cs,
                       topk_ids, n_flat, (int)E, items, seg_total, warp_hist, d_status) !=
            cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        if (launch_pdl(dispatch_scatter_kernel<false>, dim3((unsigned)S), dim3(kDispWarps * 32), 0,
                       cs, topk_ids, n_flat, (int)k_max, (int)E, items, S,
                       (const int32_t *)seg_total, (const int32_t *)warp_hist, counts, offsets,
                       sorted_token, dest_pos, Limits{INT32_MAX, 1, nullptr}) != cudaSuccess) {
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
        int32_t *seg_total = static_cast<int32_t *>(workspace);
        int32_t *warp_hist = seg_total + S * E;
        if (launch_pdl(dispatch_count_kernel, dim3((unsigned)S), dim3(kDispWarps * 32), 0, cs,
                       topk_ids, n_flat, (int)E, items, seg_total, warp_hist, d_status) !=
            cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        const Limits lim{capacity > 0 ? capacity : INT32_MAX, pad, dropped};
        if (launch_pdl(dispatch_scatter_kernel<true>, dim3((unsigned)S), dim3(kDispWarps * 32), 0,
                       cs, topk_ids, n_flat, (int)k_max, (int)E, items, S,
                       (const int32_t *)seg_total, (const int32_t *)warp_hist, counts, offsets,
                       sorted_token, dest_pos, lim) != cudaSuccess) {
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
// the device address is fetched with cudaGetSymbolAddress once per device and
// cached.
namespace moe {
namespace {
constexpr size_t kStaticScratchBytes = size_t(4) << 20;
constexpr int kMaxDevices = 64;
std::atomic<void *> g_static_scratch_addr[kMaxDevices];
}  // namespace
}  // namespace moe

static __device__ __align__(256) int32_t g_dispatch_scratch[moe::kStaticScratchBytes / sizeof(int32_t)];

extern "C" moe_status moe_dispatch_static(const int32_t *topk_ids, int64_t T, int32_t k_max,
                                          int32_t E, int32_t *counts, int32_t *offsets,
                                          int32_t *sorted_token, int32_t *dest_pos,
                                          int32_t *d_status, moe_stream_t stream) {
    using namespace moe;
    size_t need = 0;
    moe_status st = moe_dispatch_workspace_size(T, k_max, E, &need);
    if (st != MOE_OK) return st;
    if (need > kStaticScratchBytes) return MOE_ERR_UNSUPPORTED;  // beyond the fixed scratch
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    void *addr = g_static_scratch_addr[dev].load(std::memory_order_acquire);
    if (!addr) {
        // First call on this device (with it current): resolve the array's
        // device address.  Two threads racing here store the same value.
        if (cudaGetSymbolAddress(&addr, g_dispatch_scratch) != cudaSuccess || !addr) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        g_static_scratch_addr[dev].store(addr, std::memory_order_release);
    }
    // Every scratch entry a dispatch reads is written earlier by the same
    // dispatch, so the array needs no clearing between calls.
    return moe_dispatch(topk_ids, T, k_max, E, counts, offsets, sorted_token, dest_pos, addr,
                        kStaticScratchBytes, d_status, stream);
}
