// moe_permute and moe_combine: the two HBM-bound row movers of the path.
//
// permute: xs[dest_pos[t][j]] = x[t]   (bit-exact copy into expert order)
// combine: out[t] = bf16_rne( sum_j w[t][j] * y[dest_pos[t][j]] + shared[t] ),
//          fp32 accumulation in slot order, the shared expert ("Crate
//          ferrox_moe", combine_expert_outputs: routed + shared) added last.
//
// B200 design: both kernels are token-major, one warp per token row, 16-byte
// vector accesses.  permute reads each row of x once and writes it to its k_t
// destinations (T*d*2 + N*d*2 bytes: the algorithmic minimum; a gather loop
// over destination rows would re-read x k times) with streaming stores, which
// measured 3 % faster than plain ones for the permuted rows.  combine gathers the k_t
// expert rows of a token and writes one row; loads of four slots are issued
// before their FMAs so that enough bytes are in flight per warp (four vectors
// per lane per slot where the row has them: at d = 2048 that took combine from
// 104.6 to 102.2 us against two).
#include "common.cuh"
#include "rows.cuh"

namespace moe {
namespace {

constexpr int kRowWarps = 8;

// CHECK: every dest_pos outside [-1, rows) is skipped and reported (the
// bounded entry points, and every launch of a MOE_CHECKED build).
template <bool CHECK>
__device__ __forceinline__ int checked_pos(int dp, int64_t rows, int32_t *status) {
    if (CHECK && (dp < -1 || (int64_t)dp >= rows)) {
        report(status, MOE_ERR_DEVICE_INDEX);
        return -1;
    }
    return dp;
}

template <int U, bool CHECK>
__global__ void __launch_bounds__(kRowWarps * 32)
    permute_kernel(const uint4 *__restrict__ x, const int32_t *__restrict__ dest_pos, int64_t T,
                   int k_max, int nvec, uint4 *__restrict__ xs, int64_t rows, int32_t *status) {
    const int lane = threadIdx.x & 31;
    const int64_t nw = (int64_t)gridDim.x * kRowWarps;
    griddep_wait();
    for (int64_t row = (int64_t)blockIdx.x * kRowWarps + (threadIdx.x >> 5); row < T; row += nw) {
        const int dp = checked_pos<CHECK>(lane < k_max ? dest_pos[row * k_max + lane] : -1, rows,
                                          status);
        const uint4 *src = x + row * nvec;
        for (int v0 = 0; v0 < nvec; v0 += 32 * U) {
            uint4 buf[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v < nvec) buf[u] = ld_stream(src + v);
            }
            for (int j = 0; j < k_max; ++j) {
                const int pos = __shfl_sync(MOE_FULL_MASK, dp, j);
                if (pos < 0) continue;
                uint4 *dst = xs + (int64_t)pos * nvec;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec) __stcs(dst + v, buf[u]);  // written once, read later
                }
            }
        }
    }
    griddep_launch_dependents();
}

// SHG: the call has a shared row and k_max % J != 0 (the host checks), so the
// shared row travels in the last slot group's free slot.
template <int U, bool CHECK, bool SHG>
__global__ void __launch_bounds__(kRowWarps * 32)
    combine_kernel(const uint4 *__restrict__ y, const float *__restrict__ w,
                   const int32_t *__restrict__ dest_pos, const uint4 *__restrict__ shared,
                   int64_t T, int k_max, int nvec, uint4 *__restrict__ out, int64_t rows,
                   int32_t *status) {
    constexpr int J = 4;  // slots whose loads are issued together
    const int lane = threadIdx.x & 31;
    const int64_t nw = (int64_t)gridDim.x * kRowWarps;
    griddep_wait();
    for (int64_t row = (int64_t)blockIdx.x * kRowWarps + (threadIdx.x >> 5); row < T; row += nw) {
        const int dp = checked_pos<CHECK>(lane < k_max ? dest_pos[row * k_max + lane] : -1, rows,
                                          status);
        const float wl = lane < k_max ? w[row * k_max + lane] : 0.0f;
        for (int v0 = 0; v0 < nvec; v0 += 32 * U) {
            float acc[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
            // With k_max not a multiple of J the last group has a free slot qs:
            // the shared row's loads go out with that group's (one wait, not
            // two), and it is still added after every slot.
            const int qs = k_max % J;
            constexpr bool sh_in_group = SHG;
            for (int j0 = 0; j0 < k_max; j0 += J) {
                int pos[J];
                float wt[J];
                uint4 t[J][U];
                const bool sh_here = sh_in_group && j0 + J > k_max;
#pragma unroll
                for (int q = 0; q < J; ++q) {
                    const int j = j0 + q;
                    pos[q] = __shfl_sync(MOE_FULL_MASK, dp, j & 31);
                    wt[q] = __shfl_sync(MOE_FULL_MASK, wl, j & 31);
                    if (j >= k_max) pos[q] = -1;
                }
#pragma unroll
                for (int q = 0; q < J; ++q) {
                    const uint4 *src = pos[q] >= 0 ? y + (int64_t)pos[q] * nvec
                                       : (SHG && sh_here && q == qs) ? shared + row * nvec
                                                                     : nullptr;
                    if (src) {
#pragma unroll
                        for (int u = 0; u < U; ++u) {
                            const int v = v0 + u * 32 + lane;
                            t[q][u] = v < nvec ? ld_stream(src + v) : make_uint4(0, 0, 0, 0);
                        }
                    }
                }
#pragma unroll
                for (int q = 0; q < J; ++q)
                    if (pos[q] >= 0)
#pragma unroll
                        for (int u = 0; u < U; ++u) fma_bf16x8(acc[u], wt[q], t[q][u]);
                if (SHG && sh_here) {
#pragma unroll
                    for (int q = 1; q < J; ++q)
                        if (q == qs)
#pragma unroll
                            for (int u = 0; u < U; ++u)
                                if (v0 + u * 32 + lane < nvec) add_bf16x8(acc[u], t[q][u]);
                }
            }
            if (shared && !sh_in_group) {
                const uint4 *src = shared + row * nvec;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec) add_bf16x8(acc[u], ld_stream(src + v));
                }
            }
            uint4 *dst = out + row * nvec;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v < nvec) dst[v] = pack_bf16x8(acc[u]);
            }
        }
    }
    griddep_launch_dependents();
}

unsigned row_grid(int64_t T) {
    const int64_t need = (T + kRowWarps - 1) / kRowWarps;
    const int64_t cap = (int64_t)sm_count() * 32;
    return (unsigned)(need < cap ? need : cap);
}

// Launches a row kernel; a grid of at most one block per SM (a decode-sized
// batch) is launched as a programmatic dependent of the kernel before it, so
// its launch overlaps that kernel's tail.  Larger grids use plain launches:
// there the early-resident waiting blocks measured slower (0.3 % at 2048
// blocks), while at 32 blocks the overlap gave 6 %.
template <typename... KArgs, typename... Args>
cudaError_t launch_rows(void (*kernel)(KArgs...), unsigned grid, cudaStream_t s, Args... args) {
    if (grid <= (unsigned)sm_count())
        return launch_pdl(kernel, dim3(grid), dim3(kRowWarps * 32), 0, s, args...);
    kernel<<<grid, kRowWarps * 32, 0, s>>>(static_cast<KArgs>(args)...);
    return cudaGetLastError();
}

// Both row movers with the dest_pos check switched on (CHECK) or off.
template <bool CHECK>
moe_status run_permute(const moe_bf16_t *x, const int32_t *dest_pos, int64_t T, int32_t k_max,
                       int32_t d, moe_bf16_t *xs, int64_t rows, int32_t *d_status,
                       moe_stream_t stream) {
    if (T < 0 || k_max < 0 || k_max > 32 || d < 8 || d % 8 != 0 || rows < 0)
        return MOE_ERR_INVALID_ARG;
    if (T == 0 || k_max == 0) return MOE_OK;
    if (!x || !dest_pos || !xs || !aligned16(x) || !aligned16(xs)) return MOE_ERR_INVALID_ARG;
    if (T * (int64_t)k_max >= (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
    // Sixteen vectors per lane on rows of more than 256 vectors (d > 2048): more
    // bytes in flight per warp measured 0.6-1.1 % faster at d >= 4096, and at
    // d = 2880 (360 vectors) one round of sixteen instead of a full round of
    // eight and a third of one measured 1289 -> 1225 us; eight elsewhere.
    // Rows of 769-896 vectors (d = 7168: deepseek-v3/v4) take twenty-eight, the
    // whole row in one round (133 registers, one block an SM): 1343 -> 1312 us
    // and 1048 -> 1026 us; capped at 128 registers for two blocks an SM it
    // spilled and measured 1331 us; twenty at d = 5120 gained nothing.
    const uint4 *x4 = reinterpret_cast<const uint4 *>(x);
    uint4 *xs4 = reinterpret_cast<uint4 *>(xs);
    const cudaError_t err =
        (d / 8 > 768 && d / 8 <= 896)
            ? launch_rows(permute_kernel<28, CHECK>, row_grid(T), as_cuda(stream), x4, dest_pos, T,
                          (int)k_max, d / 8, xs4, rows, d_status)
        : d / 8 > 256 ? launch_rows(permute_kernel<16, CHECK>, row_grid(T), as_cuda(stream), x4,
                                   dest_pos, T, (int)k_max, d / 8, xs4, rows, d_status)
                     : launch_rows(permute_kernel<8, CHECK>, row_grid(T), as_cuda(stream), x4,
                                   dest_pos, T, (int)k_max, d / 8, xs4, rows, d_status);
    if (err != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return launch_status();
}

template <bool CHECK>
moe_status run_combine(const moe_bf16_t *y, const float *topk_w, const int32_t *dest_pos,
                       const moe_bf16_t *shared, int64_t T, int32_t k_max, int32_t d,
                       moe_bf16_t *out, int64_t rows, int32_t *d_status, moe_stream_t stream) {
    if (T < 0 || k_max < 0 || k_max > 32 || d < 8 || d % 8 != 0 || rows < 0)
        return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!out || !aligned16(out) || (shared && !aligned16(shared))) return MOE_ERR_INVALID_ARG;
    if (k_max > 0 && (!y || !topk_w || !dest_pos || !aligned16(y))) return MOE_ERR_INVALID_ARG;
    if (T * (int64_t)k_max >= (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
    // Vectors per lane per slot: as many as the row has for the whole warp, up
    // to four (short rows would leave lanes idle).
    const int nvec = d / 8;
    const uint4 *y4 = reinterpret_cast<const uint4 *>(y);
    const uint4 *s4 = reinterpret_cast<const uint4 *>(shared);
    uint4 *o4 = reinterpret_cast<uint4 *>(out);
    const unsigned grid = row_grid(T);
    cudaStream_t cs = as_cuda(stream);
    // The shared row in a free slot of the last group of four (k_max % 4 != 0):
    // llama4_top1 (k = 1, a shared expert) combine 1331 -> 1225 us.
    const bool shg = shared && k_max % 4 != 0;
#define MOE_COMBINE(UU, SH)                                                                         \
    launch_rows(combine_kernel<UU, CHECK, SH>, grid, cs, y4, topk_w, dest_pos, s4, T, (int)k_max, \
                nvec, o4, rows, d_status)
    const cudaError_t err = nvec >= 128 ? (shg ? MOE_COMBINE(4, true) : MOE_COMBINE(4, false))
                            : nvec >= 64 ? (shg ? MOE_COMBINE(2, true) : MOE_COMBINE(2, false))
                                         : (shg ? MOE_COMBINE(1, true) : MOE_COMBINE(1, false));
#undef MOE_COMBINE
    if (err != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return launch_status();
}

// A MOE_CHECKED build checks the plain entry points too, against T * k_max
// rows (the most a dispatch of T tokens can fill); their signatures carry no
// status word, so a skipped slot there is not reported.
#ifdef MOE_CHECKED
constexpr bool kCheckedBuild = true;
#else
constexpr bool kCheckedBuild = false;
#endif

}  // namespace
}  // namespace moe

extern "C" moe_status moe_permute(const moe_bf16_t *x, const int32_t *dest_pos, int64_t T,
                                  int32_t k_max, int32_t d, moe_bf16_t *xs, moe_stream_t stream) {
    return moe::run_permute<moe::kCheckedBuild>(x, dest_pos, T, k_max, d, xs, T * (int64_t)k_max,
                                                nullptr, stream);
}

extern "C" moe_status moe_combine(const moe_bf16_t *y, const float *topk_w,
                                  const int32_t *dest_pos, const moe_bf16_t *shared, int64_t T,
                                  int32_t k_max, int32_t d, moe_bf16_t *out, moe_stream_t stream) {
    return moe::run_combine<moe::kCheckedBuild>(y, topk_w, dest_pos, shared, T, k_max, d, out,
                                                T * (int64_t)k_max, nullptr, stream);
}

extern "C" moe_status moe_permute_bounded(const moe_bf16_t *x, const int32_t *dest_pos, int64_t T,
                                          int32_t k_max, int32_t d, moe_bf16_t *xs,
                                          int64_t xs_rows, int32_t *d_status,
                                          moe_stream_t stream) {
    return moe::run_permute<true>(x, dest_pos, T, k_max, d, xs, xs_rows, d_status, stream);
}

extern "C" moe_status moe_combine_bounded(const moe_bf16_t *y, const float *topk_w,
                                          const int32_t *dest_pos, const moe_bf16_t *shared,
                                          int64_t T, int32_t k_max, int32_t d, int64_t y_rows,
                                          moe_bf16_t *out, int32_t *d_status,
                                          moe_stream_t stream) {
    return moe::run_combine<true>(y, topk_w, dest_pos, shared, T, k_max, d, out, y_rows, d_status,
                                  stream);
}
