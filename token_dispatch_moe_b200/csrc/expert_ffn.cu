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
// sm_100a design: a persistent grid, two CTAs per SM, walks output tiles of
// 128 rows of one expert (expert blocks are 128-row aligned, so a tile never
// straddles two experts) by BN columns, N tile fastest so the CTAs running
// together share their A tile in L2.  Warp 0 issues TMA loads (the A tile and,
// for gate_up, the W1 and W3 tiles of the same columns) into a stage ring that
// runs on across tiles; one thread of warp 1 issues tcgen05.mma into the
// CTA's TMEM accumulator (gate_up: gate and up side by side); warp 2 owns the
// TMEM columns; warps 4..7 run the epilogue (tcgen05.ld, bias, activation,
// bf16 stores of the tile's rows).  The epilogue of one tile overlaps a
// mainloop: the other CTA's on the same SM (two CTAs per SM, one accumulator
// each) or, with one CTA per SM, the CTA's own next tile in its second
// accumulator.  Every mbarrier wait is bounded; a wait that
// gives up stops every role, and the CTA drains its copies and MMAs before it
// frees the TMEM.
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
// Two CTAs per SM, one TMEM accumulator each: one CTA's epilogue overlaps the
// other's mainloop, and two producers keep more loads in flight.  Against one
// CTA per SM with two accumulators: gpt-oss shape 10 % faster, qwen3 shape equal.
constexpr int kFfnCtasPerSm = 2;
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
    int nbuf;                // TMEM accumulators per CTA: 2 (one CTA per SM) or 1 (two per SM)
    uint32_t stage_bytes, idesc;
};

// The activations, in the epilogue of every gate_up tile.  h is rounded to
// bf16 (8 significant bits), so the exponential and the quotient use the fast
// intrinsics (__expf, __fdividef: a few fp32 ulps, about 1e-6 relative here,
// far below h's rounding).  A quotient by 1 + e^-x that overflows to inf
// gives 0, the limit of x * sigmoid(x) for very negative x.
__device__ __forceinline__ float silu_gate(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

__device__ __forceinline__ float swiglu_oai(float g, float u) {
    const float gc = fminf(g, kOaiLimit);
    const float uc = fminf(fmaxf(u, -kOaiLimit), kOaiLimit);
    return __fdividef(gc, 1.0f + __expf(-kOaiAlpha * gc)) * (uc + 1.0f);
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

// The expert whose 128-row-aligned block holds the M tile starting at row m0
// (off = the offsets, staged in shared memory), or -1 when the tile lies past
// the last block or straddles two blocks (offsets not 128-aligned).  Every
// role of the CTA walks the same tiles through this function.
__device__ __forceinline__ int tile_expert(const int32_t *off, int E, int64_t total, int64_t m0) {
    if (m0 >= total) return -1;
    int lo = 0, hi = E - 1;
    while (lo < hi) {  // the last e with off[e] <= m0 (offsets ascend)
        const int mid = (lo + hi + 1) >> 1;
        if ((int64_t)off[mid] <= m0) lo = mid; else hi = mid - 1;
    }
    if ((off[lo] & (kFBM - 1)) != 0 || m0 + kFBM > (int64_t)off[lo + 1]) return -1;
    return lo;
}

// GATE_UP: A = xs, B0 = W1, B1 = W3, out = h.  Otherwise A = h, B0 = W2, out = y.
// Persistent: each CTA walks tiles blockIdx.x, +gridDim.x, ...; the
// shared-memory stage ring runs on across tiles; the a.nbuf TMEM accumulators
// are used in turn (tile j in accumulator j % nbuf).
template <bool GATE_UP>
__global__ void __launch_bounds__(kFThreads, 1)
    expert_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                       const __grid_constant__ CUtensorMap tmap_b0,
                       const __grid_constant__ CUtensorMap tmap_b1, const FfnArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ int abort_s;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    griddep_wait();  // offsets and the A rows come from the kernels before this one
    const int n_tiles = a.N / a.BN;
    const int64_t total = __ldg(a.offsets + a.E);
    const int64_t m_tiles = total > 0 && total <= a.rows ? (total + kFBM - 1) / kFBM : 0;
    const int64_t num_tiles = m_tiles * n_tiles;
    if (threadIdx.x == 0 && blockIdx.x == 0 && total > a.rows)
        report(a.status, MOE_ERR_DEVICE_INDEX);  // blocks reach past the buffers: no tile runs
    if ((int64_t)blockIdx.x >= num_tiles) return;  // nothing for this CTA

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const gbase = smem_raw + (base - raw);
    const int S = a.stages;
    // [stages][full[S]][empty[S]][tmem_full[2]][tmem_empty[2]][drain][tmem slot]
    const uint32_t bar0 = base + (uint32_t)S * a.stage_bytes;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * S + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * S + 2 + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * S + 4);
    uint32_t *tmem_slot =
        reinterpret_cast<uint32_t *>(gbase + (size_t)S * a.stage_bytes + 8u * (2 * S + 5));
    int32_t *off = reinterpret_cast<int32_t *>(gbase + (size_t)S * a.stage_bytes + 256);
    const uint32_t btile = (uint32_t)a.BN * 128u;  // bytes of one BN x 64 operand tile
    const uint32_t acc_cols = GATE_UP ? 2u * a.BN : (uint32_t)a.BN;

    if (threadIdx.x == 0) {
        abort_s = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 4);  // one arrival per epilogue warp
        }
        mbar_init(drain_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int i = threadIdx.x; i <= a.E; i += blockDim.x) off[i] = __ldg(a.offsets + i);
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
    volatile int *abort_v = &abort_s;
    griddep_launch_dependents();  // the next kernel may be scheduled; it waits for this grid

    if (warp == 0 && lane == 0) {
        // TMA producer: the stage ring runs on across tiles.
        uint32_t it = 0;
        for (int64_t t = blockIdx.x; t < num_tiles && !*abort_v; t += gridDim.x) {
            const int64_t m0 = (t / n_tiles) * kFBM;
            const int e = tile_expert(off, a.E, total, m0);
            if (e < 0) continue;
            const int brow = e * a.N + (int)(t % n_tiles) * a.BN;
            for (int kb = 0; kb < a.num_kb; ++kb, ++it) {
                const int s = (int)(it % (uint32_t)S);
                const uint32_t ph = (it / (uint32_t)S) & 1u;
                if (!mbar_wait(empty_bar(s), ph ^ 1u, a.status)) {
                    *abort_v = 1;
                    break;
                }
                const uint32_t st = base + (uint32_t)s * a.stage_bytes;
                mbar_arrive_expect_tx(full_bar(s), a.stage_bytes);
                tma_load_2d(st, &tmap_a, full_bar(s), kb * kFBK, (int)m0);
                tma_load_2d(st + kFATile, &tmap_b0, full_bar(s), kb * kFBK, brow);
                if (GATE_UP)
                    tma_load_2d(st + kFATile + btile, &tmap_b1, full_bar(s), kb * kFBK, brow);
            }
        }
        // Drain: the last load into every stage has landed before the CTA exits.
        const uint32_t first = it > (uint32_t)S ? it - (uint32_t)S : 0u;
        for (uint32_t i = first; i < it; ++i)
            if (!mbar_wait(full_bar((int)(i % (uint32_t)S)), (i / (uint32_t)S) & 1u, a.status))
                break;
    } else if (warp == 1 && lane == 0) {
        // MMA issuer: accumulator b = j & 1 of the j-th tile this CTA computes.
        uint32_t it = 0, j = 0;
        for (int64_t t = blockIdx.x; t < num_tiles && !*abort_v; t += gridDim.x) {
            if (tile_expert(off, a.E, total, (t / n_tiles) * kFBM) < 0) continue;
            const uint32_t b = j % (uint32_t)a.nbuf;
            if (!mbar_wait(tempty_bar((int)b), ((j / (uint32_t)a.nbuf) & 1u) ^ 1u, a.status)) {
                *abort_v = 1;
                break;
            }
            tc_fence_after();
            const uint32_t acc = tmem_base + b * acc_cols;
            for (int kb = 0; kb < a.num_kb; ++kb, ++it) {
                const int s = (int)(it % (uint32_t)S);
                const uint32_t ph = (it / (uint32_t)S) & 1u;
                if (!mbar_wait(full_bar(s), ph, a.status)) {
                    *abort_v = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t st = base + (uint32_t)s * a.stage_bytes;
#pragma unroll
                for (int k = 0; k < kFBK / kFUmmaK; ++k) {
                    const uint32_t koff = (uint32_t)(k * kFUmmaK * 2);
                    const uint64_t adesc = sw128_desc(st + koff);
                    const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
                    umma_bf16(acc, adesc, sw128_desc(st + kFATile + koff), a.idesc, accum);
                    if (GATE_UP)
                        umma_bf16(acc + (uint32_t)a.BN, adesc,
                                  sw128_desc(st + kFATile + btile + koff), a.idesc, accum);
                }
                umma_commit(empty_bar(s));
            }
            if (*abort_v) break;
            umma_commit(tfull_bar((int)b));
            ++j;
        }
        // Every MMA issued above has completed before the columns are freed.
        umma_commit(drain_bar);
        mbar_wait(drain_bar, 0u, a.status);
    } else if (warp >= 4) {
        // Epilogue: warp w reads TMEM lanes 32*(w%4).. = rows of the tile.
        const int q = warp & 3;
        uint32_t j = 0;
        for (int64_t t = blockIdx.x; t < num_tiles; t += gridDim.x) {
            const int64_t m0 = (t / n_tiles) * kFBM;
            const int e = tile_expert(off, a.E, total, m0);
            if (e < 0) {  // a tile straddling two blocks: skipped by every role, reported here
                if (q == 0 && lane == 0) report(a.status, MOE_ERR_DEVICE_INDEX);
                continue;
            }
            const uint32_t b = j % (uint32_t)a.nbuf;
            const bool ok = __all_sync(MOE_FULL_MASK,
                                       !*abort_v && mbar_wait(tfull_bar((int)b), (j / (uint32_t)a.nbuf) & 1u,
                                                              a.status));
            if (!ok) {
                if (lane == 0) *abort_v = 1;
                break;
            }
            tc_fence_after();
            const int n0 = (int)(t % n_tiles) * a.BN;
            const int64_t row = m0 + q * 32 + lane;
            const uint32_t trow = tmem_base + b * acc_cols + ((uint32_t)(q * 32) << 16);
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
                    float gv[16], uv[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        gv[i] = __uint_as_float(g[i]) + (b0 ? b0[c0 + i] : 0.0f);
                        uv[i] = __uint_as_float(u[i]) + (b1 ? b1[c0 + i] : 0.0f);
                    }
                    // the activation chosen once per 16 columns, not once per value
                    if (a.act == MOE_ACT_SWIGLU_OAI) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = swiglu_oai(gv[i], uv[i]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = silu_gate(gv[i]) * uv[i];
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
            // This warp's reads of accumulator b are done: the MMA may reuse it.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar((int)b));
            ++j;
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
    // One CTA per SM with two TMEM accumulators, or two CTAs per SM with one each.
    a.nbuf = kFfnCtasPerSm == 1 ? 2 : 1;
    const int ncols = a.nbuf * (GATE_UP ? 2 * a.BN : a.BN);
    int cols = 32;
    while (cols < ncols) cols *= 2;
    if (cols > 512) return MOE_ERR_UNSUPPORTED;
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
    // alignment slack, barriers and TMEM slot, the staged offsets
    const int overhead = 1024 + 256 + ((a.E + 1) * 4 + 15) / 16 * 16;
    int budget = max_smem;
    if (kFfnCtasPerSm == 2) {
        int per_sm = 0;
        if (cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
            cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        budget = per_sm / 2 - 1024;  // 1 KB per block is reserved by the system
    }
    int stages = (int)((budget - 1024 - overhead) / (int)a.stage_bytes);  // 1 KB static
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
    // Persistent: kFfnCtasPerSm CTAs per SM, never more than the largest tile count.
    const int64_t most = (int64_t)(a.N / a.BN) * ((rows + kFBM - 1) / kFBM);
    const int64_t slots = (int64_t)sm_count() * kFfnCtasPerSm;
    const int64_t grid = most < slots ? most : slots;
    if (launch_pdl(expert_gemm_kernel<GATE_UP>, dim3((unsigned)grid), dim3(kFThreads), smem,
                   as_cuda(stream), ma, mb0, mb1, a) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return launch_status();
}

moe_status check_ffn(const void *A, const int32_t *offsets, int32_t E, int32_t d, int32_t F,
                     int64_t rows, const void *out) {
    if (E < 1 || E > kFMaxE || d < 16 || d % 16 != 0 || F < 16 || F % 16 != 0 || rows < 0)
        return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (!A || !offsets || !out || !aligned16(A) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    if (rows >= (int64_t)INT32_MAX || (int64_t)E * (d > F ? d : F) >= (int64_t)INT32_MAX)
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
