// moe_dispatch: per-expert histogram, exclusive scan and stable scatter of the
// T*k_max routing slots into expert-contiguous order.
//
// Definition: counts[e] = #slots with id e; offsets = exclusive scan of counts;
// walking the slots in flat order a = t*k_max + j, slot a with id e gets
// pos = offsets[e] + (number of earlier slots with id e); sorted_token[pos] = t,
// dest_pos[a] = pos (-1 for empty slots).
//
// B200 design: three short launches and no inter-block waiting.
//   1. count:   each warp owns a segment of SEG consecutive slots and builds its
//               segment's histogram in shared memory with warp-aggregated
//               updates (__match_any_sync: one leader per distinct id adds the
//               popcount of its peers) -> seg[s][e] in the workspace.
//   2. scan:    per expert, exclusive prefix of seg[.][e] over segments (in
//               place) and the total counts[e]; 32 experts per block so every
//               row access is a coalesced 128-byte line.
//   3. scatter: each block scans counts into offsets in shared memory (block 0
//               also writes them out); each warp walks its segment again in
//               order, ranks every slot among its peers with the same id
//               (popcount of lower lanes in the match mask) and writes
//               sorted_token and dest_pos.
// The workspace is seg: S x E int32, S = ceil(T*k_max / SEG).
#include <atomic>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kDispWarps = 8;
constexpr int kMaxE = 512;

int seg_items(int64_t n_flat) {
    int items = 4;
    while (n_flat > (int64_t)items * 32 * 1024 && items < 64) items *= 2;
    return items;
}

int64_t num_segments(int64_t n_flat, int items) { return (n_flat + items * 32 - 1) / (items * 32); }

__global__ void __launch_bounds__(kDispWarps * 32)
    dispatch_count_kernel(const int32_t *__restrict__ ids, int64_t n_flat, int E, int items,
                          int64_t S, int32_t *__restrict__ seg, int32_t *status) {
    __shared__ int32_t hist[kDispWarps][kMaxE];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t s = (int64_t)blockIdx.x * kDispWarps + warp;
    if (s >= S) return;  // whole warp leaves together
    int32_t *h = hist[warp];
    for (int e = lane; e < E; e += 32) h[e] = 0;
    __syncwarp();
    const int64_t base = s * items * 32;
    bool bad = false;
    for (int i = 0; i < items; ++i) {
        const int64_t a = base + (int64_t)i * 32 + lane;
        int e = a < n_flat ? ids[a] : -1;
        if (e < -1 || e >= E) {
            bad = true;
            e = -1;
        }
        const unsigned peers = __match_any_sync(MOE_FULL_MASK, e);
        if (e >= 0 && lane == __ffs(peers) - 1) h[e] += __popc(peers);
        __syncwarp();
    }
    if (__any_sync(MOE_FULL_MASK, bad) && lane == 0) report(status, MOE_ERR_DEVICE_INDEX);
    int32_t *out = seg + s * E;
    for (int e = lane; e < E; e += 32) out[e] = h[e];
}

// Block b handles experts 32b .. 32b+31 (lane = expert), warp w a contiguous
// chunk of segments.
__global__ void __launch_bounds__(1024)
    dispatch_scan_kernel(int32_t *__restrict__ seg, int64_t S, int E, int32_t *__restrict__ counts) {
    __shared__ int32_t part[32][33];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = blockIdx.x * 32 + lane;
    const int64_t chunk = (S + 31) / 32;
    const int64_t s0 = warp * chunk;
    const int64_t s1 = s0 + chunk < S ? s0 + chunk : S;
    int32_t sum = 0;
    if (e < E)
        for (int64_t s = s0; s < s1; ++s) sum += seg[s * E + e];
    part[warp][lane] = sum;
    __syncthreads();
    int32_t run = 0;
    for (int w = 0; w < warp; ++w) run += part[w][lane];
    if (e < E) {
        for (int64_t s = s0; s < s1; ++s) {
            const int32_t v = seg[s * E + e];
            seg[s * E + e] = run;
            run += v;
        }
        if (warp == 31) counts[e] = run;
    }
}

__global__ void __launch_bounds__(kDispWarps * 32)
    dispatch_scatter_kernel(const int32_t *__restrict__ ids, int64_t n_flat, int k_max, int E,
                            int items, int64_t S, const int32_t *__restrict__ seg,
                            const int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                            int32_t *__restrict__ sorted_token, int32_t *__restrict__ dest_pos) {
    __shared__ int32_t off[kMaxE + 1];
    __shared__ int32_t run[kDispWarps][kMaxE];
    __shared__ int32_t wsum[kDispWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    // Block-wide exclusive scan of counts: thread i owns experts 2i, 2i+1.
    {
        const int i0 = 2 * threadIdx.x, i1 = i0 + 1;
        const int32_t c0 = i0 < E ? counts[i0] : 0;
        const int32_t c1 = i1 < E ? counts[i1] : 0;
        int32_t v = c0 + c1, incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t n = __shfl_up_sync(MOE_FULL_MASK, incl, o);
            if (lane >= o) incl += n;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        int32_t before = 0;
        for (int w = 0; w < warp; ++w) before += wsum[w];
        const int32_t excl = before + incl - v;
        if (i0 < E) off[i0] = excl;
        if (i1 < E) off[i1] = excl + c0;
        if (threadIdx.x == 0) {
            int32_t total = 0;
            for (int w = 0; w < kDispWarps; ++w) total += wsum[w];
            off[E] = total;
        }
        __syncthreads();
        if (blockIdx.x == 0)
            for (int e = threadIdx.x; e <= E; e += blockDim.x) offsets[e] = off[e];
    }

    const int64_t s = (int64_t)blockIdx.x * kDispWarps + warp;
    if (s >= S) return;
    int32_t *r = run[warp];
    const int32_t *sb = seg + s * E;
    for (int e = lane; e < E; e += 32) r[e] = off[e] + sb[e];
    __syncwarp();
    const int64_t base = s * items * 32;
    const unsigned lower = (1u << lane) - 1u;
    for (int i = 0; i < items; ++i) {
        const int64_t a = base + (int64_t)i * 32 + lane;
        int e = a < n_flat ? ids[a] : -1;
        if (e < -1 || e >= E) e = -1;
        const unsigned peers = __match_any_sync(MOE_FULL_MASK, e);
        if (e >= 0) {
            const int32_t pos = r[e] + __popc(peers & lower);
            sorted_token[pos] = (int32_t)(a / k_max);
            dest_pos[a] = pos;
        } else if (a < n_flat) {
            dest_pos[a] = -1;
        }
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) r[e] += __popc(peers);
        __syncwarp();
    }
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
    const int64_t S = num_segments(n_flat, seg_items(n_flat));
    const size_t b = (size_t)S * (size_t)E * sizeof(int32_t);
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
    const int items = seg_items(n_flat);
    const int64_t S = num_segments(n_flat, items);
    int32_t *seg = static_cast<int32_t *>(workspace);
    if (S > 0) {
        const unsigned blocks = (unsigned)((S + kDispWarps - 1) / kDispWarps);
        dispatch_count_kernel<<<blocks, kDispWarps * 32, 0, cs>>>(topk_ids, n_flat, E, items, S,
                                                                  seg, d_status);
        dispatch_scan_kernel<<<(E + 31) / 32, 1024, 0, cs>>>(seg, S, E, counts);
        dispatch_scatter_kernel<<<blocks, kDispWarps * 32, 0, cs>>>(
            topk_ids, n_flat, k_max, E, items, S, seg, counts, offsets, sorted_token, dest_pos);
    } else {
        // No slots: every count is 0 and every offset is 0.
        if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, cs) != cudaSuccess ||
            cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), cs) != cudaSuccess) {
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
