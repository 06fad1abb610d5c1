// Expert-parallel exchange: the permute and the combine of ranks that each own
// E/G of the experts, moving rows straight over peer memory.
//
// Placement: expert e lives on rank e / (E/G).  Rank d's receive buffer holds
// its experts in ascending order; inside an expert, the rows sent by rank 0,
// then rank 1, ...; inside one source, that rank's slots in flat order
// a = t*k_max + j (the order of its local moe_dispatch).  So every expert's
// rows are contiguous on its owner, as a grouped expert GEMM wants them.
//
// Steps on each rank (the exchange of counts is the caller's collective):
//   moe_dispatch   -> counts[E], offsets, dest_pos (local, as on one GPU)
//   all-gather of counts over the ranks -> all_counts[G][E]
//   moe_ep_layout  -> dest_rank / dest_row of every slot, recv_offsets
//   moe_ep_permute -> x rows stored into the owners' receive buffers
//   (barrier; experts run on the receive buffers; barrier)
//   moe_ep_combine -> out[t] from the owners' expert outputs, read remotely
//
// B200 design: no separate all-to-all.  The permute's row stores and the
// combine's row loads go straight to the peer GPU's HBM over NVLink (peer
// pointers through NVSwitch), so the transfer is the row movement itself: one
// read of x and one write per slot, each crossing NVLink once.  Plain 16-byte
// loads and stores only; no TMA with cluster-wide delivery touches peer memory.
#include "common.cuh"
#include "rows.cuh"

namespace moe {
namespace {

constexpr int kEpWarps = 8;
constexpr int kMaxRanks = 64;
constexpr int kLayoutThreads = 512;  // one per expert (E <= 512)

// Per-expert first row of this rank's block on the owner, in shared memory;
// block 0 also writes this rank's own receive offsets.
__global__ void __launch_bounds__(kLayoutThreads)
    ep_layout_kernel(const int32_t *__restrict__ all_counts, const int32_t *__restrict__ ids,
                     const int32_t *__restrict__ dest_pos, const int32_t *__restrict__ offsets,
                     int G, int rank, int64_t n_flat, int E, int32_t *__restrict__ dest_rank,
                     int32_t *__restrict__ dest_row, int32_t *__restrict__ recv_offsets,
                     int32_t *status) {
    __shared__ int32_t excl[kLayoutThreads + 1];
    __shared__ int32_t base[kLayoutThreads];
    __shared__ int32_t mine[kLayoutThreads];
    __shared__ int32_t wsum[kLayoutThreads / 32];
    const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
    const int el = E / G;
    int32_t demand = 0, before = 0;
    if (e < E) {
        for (int r = 0; r < G; ++r) {
            const int32_t c = all_counts[(int64_t)r * E + e];
            demand += c;
            before += r < rank ? c : 0;
        }
        mine[e] = all_counts[(int64_t)rank * E + e];
    }
    // Exclusive scan of the demand over all experts.
    int32_t incl = demand;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(MOE_FULL_MASK, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int32_t pre = 0;
    for (int w = 0; w < warp; ++w) pre += wsum[w];
    excl[e] = pre + incl - demand;
    if (e == kLayoutThreads - 1) excl[kLayoutThreads] = pre + incl;
    __syncthreads();
    // The owner's blocks start at its first expert: subtract that expert's prefix.
    if (e < E) base[e] = excl[e] - excl[(e / el) * el] + before;
    if (blockIdx.x == 0 && e <= el) {
        const int first = rank * el;
        recv_offsets[e] = excl[first + e] - excl[first];
    }
    __syncthreads();

    bool bad = false;
    for (int64_t a = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; a < n_flat;
         a += (int64_t)gridDim.x * blockDim.x) {
        const int32_t id = ids[a];
        int32_t rk = -1, row = -1;
        if (id >= 0 && id < E) {
            const int32_t r_in = dest_pos[a] - offsets[id];  // rank among this rank's slots of id
            if (r_in >= 0 && r_in < mine[id]) {
                rk = id / el;
                row = base[id] + r_in;
            } else {
                bad = true;
            }
        } else if (id != -1) {
            bad = true;
        }
        dest_rank[a] = rk;
        dest_row[a] = row;
    }
    if (bad) report(status, MOE_ERR_DEVICE_INDEX);
}

// The owner's row of slot j of a token, or nullptr when the slot is empty or
// its (rank, row) falls outside the receive buffers (or the buffer pointer is
// null or not 16-byte aligned).
__device__ __forceinline__ uint4 *peer_row(uint4 *const *peers, int G, int64_t cap, int nvec,
                                           int rk, int row, bool &bad) {
    if (rk < 0) return nullptr;
    if (rk >= G || row < 0 || row >= cap) {
        bad = true;
        return nullptr;
    }
    uint4 *p = peers[rk];
    if (p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) != 0) {
        bad = true;
        return nullptr;
    }
    return p + (int64_t)row * nvec;
}

template <int U>
__global__ void __launch_bounds__(kEpWarps * 32)
    ep_permute_kernel(const uint4 *__restrict__ x, const int32_t *__restrict__ dest_rank,
                      const int32_t *__restrict__ dest_row, uint4 *const *__restrict__ peers,
                      int G, int64_t cap, int64_t T, int k_max, int nvec, int32_t *status) {
    const int lane = threadIdx.x & 31;
    const int64_t nw = (int64_t)gridDim.x * kEpWarps;
    bool bad = false;
    for (int64_t t = (int64_t)blockIdx.x * kEpWarps + (threadIdx.x >> 5); t < T; t += nw) {
        uint4 *dst_l = nullptr;  // lane j holds slot j's destination row
        if (lane < k_max)
            dst_l = peer_row(peers, G, cap, nvec, dest_rank[t * k_max + lane],
                             dest_row[t * k_max + lane], bad);
        const uint4 *src = x + t * nvec;
        for (int v0 = 0; v0 < nvec; v0 += 32 * U) {
            uint4 buf[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v < nvec) buf[u] = ld_stream(src + v);
            }
            for (int j = 0; j < k_max; ++j) {
                uint4 *dst = reinterpret_cast<uint4 *>(
                    __shfl_sync(MOE_FULL_MASK, reinterpret_cast<unsigned long long>(dst_l), j));
                if (dst == nullptr) continue;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec) dst[v] = buf[u];
                }
            }
        }
    }
    if (bad) report(status, MOE_ERR_DEVICE_INDEX);
}

template <int U>
__global__ void __launch_bounds__(kEpWarps * 32)
    ep_combine_kernel(uint4 *const *__restrict__ peers, const int32_t *__restrict__ dest_rank,
                      const int32_t *__restrict__ dest_row, const float *__restrict__ w,
                      const uint4 *__restrict__ shared, int G, int64_t cap, int64_t T, int k_max,
                      int nvec, uint4 *__restrict__ out, int32_t *status) {
    constexpr int J = 4;  // slots whose loads are issued together
    const int lane = threadIdx.x & 31;
    const int64_t nw = (int64_t)gridDim.x * kEpWarps;
    bool bad = false;
    for (int64_t t = (int64_t)blockIdx.x * kEpWarps + (threadIdx.x >> 5); t < T; t += nw) {
        const uint4 *src_l = nullptr;
        float wl = 0.0f;
        if (lane < k_max) {
            src_l = peer_row(peers, G, cap, nvec, dest_rank[t * k_max + lane],
                             dest_row[t * k_max + lane], bad);
            wl = w[t * k_max + lane];
        }
        for (int v0 = 0; v0 < nvec; v0 += 32 * U) {
            float acc[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
            for (int j0 = 0; j0 < k_max; j0 += J) {
                const uint4 *src[J];
                float wt[J];
                uint4 tv[J][U];
#pragma unroll
                for (int q = 0; q < J; ++q) {
                    const int j = j0 + q;
                    src[q] = reinterpret_cast<const uint4 *>(__shfl_sync(
                        MOE_FULL_MASK, reinterpret_cast<unsigned long long>(src_l), j & 31));
                    wt[q] = __shfl_sync(MOE_FULL_MASK, wl, j & 31);
                    if (j >= k_max) src[q] = nullptr;
                }
#pragma unroll
                for (int q = 0; q < J; ++q)
                    if (src[q] != nullptr)
#pragma unroll
                        for (int u = 0; u < U; ++u) {
                            const int v = v0 + u * 32 + lane;
                            tv[q][u] = v < nvec ? ld_stream(src[q] + v) : make_uint4(0, 0, 0, 0);
                        }
#pragma unroll
                for (int q = 0; q < J; ++q)
                    if (src[q] != nullptr)
#pragma unroll
                        for (int u = 0; u < U; ++u) fma_bf16x8(acc[u], wt[q], tv[q][u]);
            }
            if (shared) {
                const uint4 *s = shared + t * nvec;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec) add_bf16x8(acc[u], ld_stream(s + v));
                }
            }
            uint4 *dst = out + t * nvec;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v < nvec) dst[v] = pack_bf16x8(acc[u]);
            }
        }
    }
    if (bad) report(status, MOE_ERR_DEVICE_INDEX);
}

unsigned ep_grid(int64_t T) {
    const int64_t need = (T + kEpWarps - 1) / kEpWarps;
    const int64_t cap = (int64_t)sm_count() * 32;
    return (unsigned)(need < cap ? need : cap);
}

moe_status check_ep(int32_t G, int64_t cap, int64_t T, int32_t k_max, int32_t d) {
    if (G < 1 || G > kMaxRanks || cap < 0 || cap >= (int64_t)INT32_MAX || T < 0 || k_max < 0 ||
        k_max > 32 || d < 8 || d % 8 != 0)
        return MOE_ERR_INVALID_ARG;
    if (T * (int64_t)k_max >= (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_ep_layout(const int32_t *all_counts, const int32_t *topk_ids,
                                    const int32_t *dest_pos, const int32_t *offsets, int32_t G,
                                    int32_t rank, int64_t T, int32_t k_max, int32_t E,
                                    int32_t *dest_rank, int32_t *dest_row, int32_t *recv_offsets,
                                    int32_t *d_status, moe_stream_t stream) {
    using namespace moe;
    if (G < 1 || G > kMaxRanks || rank < 0 || rank >= G || E < 1 || E > kLayoutThreads ||
        E % G != 0 || T < 0 || k_max < 0 || k_max > 32)
        return MOE_ERR_INVALID_ARG;
    const int64_t n_flat = T * (int64_t)k_max;
    if (n_flat >= (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
    if (!all_counts || !recv_offsets) return MOE_ERR_INVALID_ARG;
    if (n_flat > 0 && (!topk_ids || !dest_pos || !offsets || !dest_rank || !dest_row))
        return MOE_ERR_INVALID_ARG;
    int64_t blocks = (n_flat + kLayoutThreads - 1) / kLayoutThreads;
    const int64_t most = (int64_t)sm_count() * 4;
    blocks = blocks < 1 ? 1 : (blocks > most ? most : blocks);
    ep_layout_kernel<<<(unsigned)blocks, kLayoutThreads, 0, as_cuda(stream)>>>(
        all_counts, topk_ids, dest_pos, offsets, G, rank, n_flat, E, dest_rank, dest_row,
        recv_offsets, d_status);
    return launch_status();
}

extern "C" moe_status moe_ep_permute(const moe_bf16_t *x, const int32_t *dest_rank,
                                     const int32_t *dest_row, moe_bf16_t *const *peer_recv,
                                     int32_t G, int64_t recv_capacity, int64_t T, int32_t k_max,
                                     int32_t d, int32_t *d_status, moe_stream_t stream) {
    using namespace moe;
    moe_status st = check_ep(G, recv_capacity, T, k_max, d);
    if (st != MOE_OK) return st;
    if (T == 0 || k_max == 0) return MOE_OK;
    if (!x || !dest_rank || !dest_row || !peer_recv || !aligned16(x)) return MOE_ERR_INVALID_ARG;
    // Vectors per lane as in moe_permute: sixteen on rows of at least 4096
    // elements (deepseek_v3 over 8 emulated ranks: 1444 -> 1393 us), eight below.
    const uint4 *x4 = reinterpret_cast<const uint4 *>(x);
    uint4 *const *peers = reinterpret_cast<uint4 *const *>(peer_recv);
    if (d / 8 >= 512)
        ep_permute_kernel<16><<<ep_grid(T), kEpWarps * 32, 0, as_cuda(stream)>>>(
            x4, dest_rank, dest_row, peers, G, recv_capacity, T, k_max, d / 8, d_status);
    else
        ep_permute_kernel<8><<<ep_grid(T), kEpWarps * 32, 0, as_cuda(stream)>>>(
            x4, dest_rank, dest_row, peers, G, recv_capacity, T, k_max, d / 8, d_status);
    return launch_status();
}

extern "C" moe_status moe_ep_combine(moe_bf16_t *const *peer_y, const int32_t *dest_rank,
                                     const int32_t *dest_row, const float *topk_w,
                                     const moe_bf16_t *shared, int32_t G, int64_t recv_capacity,
                                     int64_t T, int32_t k_max, int32_t d, moe_bf16_t *out,
                                     int32_t *d_status, moe_stream_t stream) {
    using namespace moe;
    moe_status st = check_ep(G, recv_capacity, T, k_max, d);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    if (!out || !aligned16(out) || (shared && !aligned16(shared))) return MOE_ERR_INVALID_ARG;
    if (k_max > 0 && (!peer_y || !dest_rank || !dest_row || !topk_w)) return MOE_ERR_INVALID_ARG;
    // Two vectors per lane per slot at every width: four (the rule of
    // moe_combine) measured slower here, e.g. 1287 -> 1628 us for gptoss_top4
    // over 8 emulated ranks, as the peer-row lookups add registers.
    ep_combine_kernel<2><<<ep_grid(T), kEpWarps * 32, 0, as_cuda(stream)>>>(
        reinterpret_cast<uint4 *const *>(peer_y), dest_rank, dest_row, topk_w,
        reinterpret_cast<const uint4 *>(shared), G, recv_capacity, T, k_max, d / 8,
        reinterpret_cast<uint4 *>(out), d_status);
    return launch_status();
}
