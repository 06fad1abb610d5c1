// moe_expert_gate_up and moe_expert_down: the routed experts' SwiGLU FFN as
// two grouped GEMMs over the expert-ordered rows that moe_permute writes.
//
// Method ("Crate ferrox_moe", Functions: run_expert, run_expert_oai,
// swiglu_oai; Constants: SWIGLU_OAI_ALPHA, SWIGLU_OAI_LIMIT): one expert's FFN
// is gate and up projections of the hidden row, a gated activation, and a
// down projection; the gpt-oss form adds a bias to each of the three products
// and uses the clamped SwiGLU with alpha = 1.702 and limit 7.0.
//   gate_up: h[r] = act(xs[r] . W1[e]^T + b1[e], xs[r] . W3[e]^T + b3[e])
//   down:    y[r] = h[r] . W2[e]^T + b2[e]
// with e the expert whose block holds row r (offsets, padded to 128 rows as
// moe_dispatch_limited writes them with pad = 128), h and y rounded to bf16.
//   swiglu:     act(g, u) = g * sigmoid(g) * u
//   swiglu_oai: g' = min(g, limit), u' = clamp(u, -limit, limit),
//               act = g' * sigmoid(alpha * g') * (u' + 1)
//
// sm_100a design: one 128-row M tile of one expert per CTA (expert blocks are
// 128-row aligned, so a tile never straddles two experts) and one N tile of
// BN output columns; grid (N tiles, M tiles), N fastest so CTAs that share an
// A tile run together and find it in L2.  Warp 0 issues TMA loads (A tile and,
// for gate_up, the W1 and W3 tiles of the same columns), one thread of warp 1
// issues tcgen05.mma into TMEM (gate_up: two accumulators side by side), warp
// 2 owns the TMEM columns, warps 4..7 run the epilogue (tcgen05.ld, bias,
// activation, bf16 stores of the CTA's rows).  Tiles past the last expert
// block exit at once.  Every mbarrier wait is bounded.
#include "common.cuh"
#include "tc.cuh"

namespace moe {
namespace {

constexpr int kFBM = 128;
constexpr int kFBK = 64;
constexpr int kFUmmaK = 16;
constexpr int kFATile = kFBM * kFBK * 2;
constexpr int kFThreads = 256;
constexpr int kFMaxE = 4096;
constexpr float kOaiAlpha = 1.702f;
constexpr float kOaiLimit = 7.0f;

struct FfnArgs {
    const int32_t *offsets;  // [E+1], multiples of 128
    const float *bias0;      // gate_up: b1 [E][N]; down: b2 [E][N]
    const float *bias1;      // gate_up: b3 [E][N]
    moe_bf16_t *out;         // [rows][N]
    int32_t *status;
    int64_t rows;            // rows of the A and out buffers
    int E, N, BN, num_kb, stages, tmem_cols, act;
    uint32_t stage_bytes, idesc;
};

__device__ __forceinline__ float silu_gate(float g) { return g / (1.0f + expf(-g)); }

__device__ __forceinline__ float activation(int act, float g, float u) {
    if (act == MOE_ACT_SWIGLU_OAI) {
        const float gc = fminf(g, kOaiLimit);
        const float uc = fminf(fmaxf(u, -kOaiLimit), kOaiLimit);
        return gc / (1.0f + expf(-kOaiAlpha * gc)) * (uc + 1.0f);
    }
    return silu_gate(g) * u;
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

// GATE_UP: A = xs, B0 = W1, B1 = W3, out = h.  Otherwise A = h, B0 = W2, out = y.
template <bool GATE_UP>
__global__ void __launch_bounds__(kFThreads, 1)
    expert_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                       const __grid_constant__ CUtensorMap tmap_b0,
                       const __grid_constant__ CUtensorMap tmap_b1, const FfnArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ int expert_s;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * a.BN;
    const int64_t m0 = (int64_t)blockIdx.y * kFBM;

    // Which expert block holds this tile (last e with offsets[e] <= m0).
    if (threadIdx.x == 0) {
        int e = -1;
        const int64_t total = a.offsets[a.E];
        if (m0 < total && total <= a.rows) {
            int lo = 0, hi = a.E - 1;
            while (lo < hi) {  // offsets ascend; find the last e with offsets[e] <= m0
                const int mid = (lo + hi + 1) >> 1;
                if ((int64_t)a.offsets[mid] <= m0) lo = mid; else hi = mid - 1;
            }
            e = lo;
            if ((a.offsets[e] & (kFBM - 1)) != 0 || m0 + kFBM > (int64_t)a.offsets[e + 1]) {
                report(a.status, MOE_ERR_DEVICE_INDEX);  // blocks not 128-row aligned
                e = -1;
            }
        } else if (total > a.rows) {
            report(a.status, MOE_ERR_DEVICE_INDEX);
        }
        expert_s = e;
    }
    __syncthreads();
    const int e = expert_s;
    if (e < 0) return;  // past the last block (or bad offsets): nothing to do

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const gbase = smem_raw + (base - raw);
    const int S = a.stages;
    const uint32_t bar0 = base + (uint32_t)S * a.stage_bytes;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    const uint32_t tmem_full_bar = bar0 + 8u * (2 * S);
    uint32_t *tmem_slot =
        reinterpret_cast<uint32_t *>(gbase + (size_t)S * a.stage_bytes + 8u * (2 * S + 1));
    const uint32_t btile = (uint32_t)a.BN * 128u;  // bytes of one BN x 64 operand tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(tmem_full_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(a.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int brow = e * a.N + n0;  // first weight row of this tile in the [E*N][K] view

    if (warp == 0 && lane == 0) {
        int issued = 0;
        for (int kb = 0; kb < a.num_kb; ++kb) {
            const int s = kb % S;
            const uint32_t ph = (uint32_t)(kb / S) & 1u;
            if (!mbar_wait(empty_bar(s), ph ^ 1u, a.status)) break;
            const uint32_t st = base + (uint32_t)s * a.stage_bytes;
            mbar_arrive_expect_tx(full_bar(s), a.stage_bytes);
            tma_load_2d(st, &tmap_a, full_bar(s), kb * kFBK, (int)m0);
            tma_load_2d(st + kFATile, &tmap_b0, full_bar(s), kb * kFBK, brow);
            if (GATE_UP) tma_load_2d(st + kFATile + btile, &tmap_b1, full_bar(s), kb * kFBK, brow);
            issued = kb + 1;
        }
        for (int kb = issued - S < 0 ? 0 : issued - S; kb < issued; ++kb)
            if (!mbar_wait(full_bar(kb % S), (uint32_t)(kb / S) & 1u, a.status)) break;
    } else if (warp == 1 && lane == 0) {
        for (int kb = 0; kb < a.num_kb; ++kb) {
            const int s = kb % S;
            const uint32_t ph = (uint32_t)(kb / S) & 1u;
            if (!mbar_wait(full_bar(s), ph, a.status)) break;
            tc_fence_after();
            const uint32_t st = base + (uint32_t)s * a.stage_bytes;
#pragma unroll
            for (int k = 0; k < kFBK / kFUmmaK; ++k) {
                const uint32_t koff = (uint32_t)(k * kFUmmaK * 2);
                const uint64_t adesc = sw128_desc(st + koff);
                const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
                umma_bf16(tmem_base, adesc, sw128_desc(st + kFATile + koff), a.idesc, acc);
                if (GATE_UP)
                    umma_bf16(tmem_base + (uint32_t)a.BN, adesc,
                              sw128_desc(st + kFATile + btile + koff), a.idesc, acc);
            }
            umma_commit(empty_bar(s));
        }
        umma_commit(tmem_full_bar);
    } else if (warp >= 4) {
        const int q = warp & 3;
        const bool ok = __all_sync(MOE_FULL_MASK, mbar_wait(tmem_full_bar, 0u, a.status));
        tc_fence_after();
        const int64_t row = m0 + q * 32 + lane;
        const uint32_t trow = tmem_base + ((uint32_t)(q * 32) << 16);
        if (ok) {
            const float *b0 = a.bias0 ? a.bias0 + (int64_t)e * a.N + n0 : nullptr;
            const float *b1 = a.bias1 ? a.bias1 + (int64_t)e * a.N + n0 : nullptr;
            moe_bf16_t *dst = a.out + row * a.N + n0;
            for (int c0 = 0; c0 < a.BN; c0 += 16) {
                uint32_t g[16];
                tmem_ld16(trow + (uint32_t)c0, g);
                float v[16];
                if (GATE_UP) {
                    uint32_t u[16];
                    tmem_ld16(trow + (uint32_t)(a.BN + c0), u);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float gv = __uint_as_float(g[i]) + (b0 ? b0[c0 + i] : 0.0f);
                        const float uv = __uint_as_float(u[i]) + (b1 ? b1[c0 + i] : 0.0f);
                        v[i] = activation(a.act, gv, uv);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        v[i] = __uint_as_float(g[i]) + (b0 ? b0[c0 + i] : 0.0f);
                }
                if (row < a.rows) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst + c0);
                    d4[0] = make_uint4(pack2(v[0], v[1]), pack2(v[2], v[3]), pack2(v[4], v[5]),
                                       pack2(v[6], v[7]));
                    d4[1] = make_uint4(pack2(v[8], v[9]), pack2(v[10], v[11]),
                                       pack2(v[12], v[13]), pack2(v[14], v[15]));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(a.tmem_cols)
                     : "memory");
    }
}

// Widest N tile (multiple of 16, <= cap) that divides N; 0 if none of the list does.
int pick_bn(int N, bool gate_up) {
    static const int gu[] = {128, 96, 64, 32, 16};
    static const int dn[] = {256, 192, 128, 64, 32, 16};
    const int *list = gate_up ? gu : dn;
    const int n = gate_up ? 5 : 6;
    for (int i = 0; i < n; ++i)
        if (N % list[i] == 0) return list[i];
    return 0;
}

template <bool GATE_UP>
moe_status launch_expert_gemm(const moe_bf16_t *A, const moe_bf16_t *B0, const moe_bf16_t *B1,
                              int K, FfnArgs a, int64_t rows, moe_stream_t stream) {
    a.BN = pick_bn(a.N, GATE_UP);
    if (a.BN == 0) return MOE_ERR_UNSUPPORTED;
    a.num_kb = (K + kFBK - 1) / kFBK;
    const int ncols = GATE_UP ? 2 * a.BN : a.BN;
    int cols = 32;
    while (cols < ncols) cols *= 2;
    a.tmem_cols = cols;
    a.stage_bytes = (uint32_t)(kFATile + (GATE_UP ? 2 : 1) * a.BN * 128);
    a.idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(a.BN >> 3) << 17) |
              ((uint32_t)(kFBM >> 4) << 24);
    int dev = 0, max_smem = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    const int overhead = 1024 + 256;
    int stages = (int)((max_smem - overhead) / (int)a.stage_bytes);
    if (stages > 6) stages = 6;
    if (stages < 2) return MOE_ERR_UNSUPPORTED;
    a.stages = stages;
    const size_t smem = (size_t)stages * a.stage_bytes + overhead;
    CUtensorMap ma, mb0, mb1;
    const int64_t brows = (int64_t)a.E * a.N;
    if (!make_map(&ma, A, rows, K, kFBM) || !make_map(&mb0, B0, brows, K, a.BN) ||
        !make_map(&mb1, GATE_UP ? B1 : B0, brows, K, a.BN))
        return MOE_ERR_CUDA;
    if (cudaFuncSetAttribute(expert_gemm_kernel<GATE_UP>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    const dim3 grid((unsigned)(a.N / a.BN), (unsigned)((rows + kFBM - 1) / kFBM));
    expert_gemm_kernel<GATE_UP><<<grid, kFThreads, smem, as_cuda(stream)>>>(ma, mb0, mb1, a);
    return launch_status();
}

moe_status check_ffn(const void *A, const int32_t *offsets, int32_t E, int32_t d, int32_t F,
                     int64_t rows, const void *out) {
    if (E < 1 || E > kFMaxE || d < 16 || d % 16 != 0 || F < 16 || F % 16 != 0 || rows < 0)
        return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (!A || !offsets || !out || !aligned16(A) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    if ((rows + kFBM - 1) / kFBM > 65535 || (int64_t)E * (d > F ? d : F) >= (int64_t)INT32_MAX)
        return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_expert_gate_up(const moe_bf16_t *xs, const int32_t *offsets,
                                         const moe_bf16_t *w1, const moe_bf16_t *w3,
                                         const float *b1, const float *b3, int32_t E, int32_t d,
                                         int32_t F, int64_t rows, int32_t act, moe_bf16_t *h,
                                         int32_t *d_status, moe_stream_t stream) {
    using namespace moe;
    moe_status st = check_ffn(xs, offsets, E, d, F, rows, h);
    if (st != MOE_OK || rows == 0) return st;
    if (act != MOE_ACT_SWIGLU && act != MOE_ACT_SWIGLU_OAI) return MOE_ERR_INVALID_ARG;
    if (!w1 || !w3 || !aligned16(w1) || !aligned16(w3)) return MOE_ERR_INVALID_ARG;
    FfnArgs a{};
    a.offsets = offsets;
    a.bias0 = b1;
    a.bias1 = b3;
    a.out = h;
    a.status = d_status;
    a.rows = rows;
    a.E = E;
    a.N = F;
    a.act = act;
    return launch_expert_gemm<true>(xs, w1, w3, d, a, rows, stream);
}

extern "C" moe_status moe_expert_down(const moe_bf16_t *h, const int32_t *offsets,
                                      const moe_bf16_t *w2, const float *b2, int32_t E, int32_t d,
                                      int32_t F, int64_t rows, moe_bf16_t *y, int32_t *d_status,
                                      moe_stream_t stream) {
    using namespace moe;
    moe_status st = check_ffn(h, offsets, E, d, F, rows, y);
    if (st != MOE_OK || rows == 0) return st;
    if (!w2 || !aligned16(w2)) return MOE_ERR_INVALID_ARG;
    FfnArgs a{};
    a.offsets = offsets;
    a.bias0 = b2;
    a.out = y;
    a.status = d_status;
    a.rows = rows;
    a.E = E;
    a.N = d;
    a.act = MOE_ACT_SWIGLU;
    return launch_expert_gemm<false>(h, w2, nullptr, F, a, rows, stream);
}
