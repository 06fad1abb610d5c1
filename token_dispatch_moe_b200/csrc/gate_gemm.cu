// moe_gate_gemm: fp32 gate logits = x . W^T on Blackwell tensor cores.
//
// Method ("DeepSeek-V3.2-Exp - Select experts", gate forward): the gate is a
// bias-free linear layer evaluated in fp32 on inputs up-cast from the model
// dtype.  bf16 x bf16 products are exact in fp32, so a bf16 tcgen05 MMA with an
// fp32 accumulator computes the same quantity (up to summation order).
//
// sm_100a design (one 128-row M tile per CTA, the whole expert dimension as N):
//   warp 0      TMA producer: 128x64 tile of x and Npad x64 tile of W per
//               k-block into a ring of shared-memory stages, 128-byte swizzle,
//               completion counted on a "full" mbarrier per stage;
//   warp 1      MMA issuer (one thread): tcgen05.mma kind::f16, M=128, N=BN,
//               K=16, A and B from shared memory through matrix descriptors,
//               accumulator in TMEM; tcgen05.commit frees the stage ("empty"
//               mbarrier) and, after the last k-block, signals the epilogue;
//   warp 2      allocates / frees the TMEM accumulator columns;
//   warps 4..7  epilogue: tcgen05.ld (32 lanes x 16 columns per load), fp32
//               stores of the logits rows.
// E <= 256 is one accumulator of N = round16(E) columns; 256 < E <= 512 is two
// of N = round16(E/2) side by side (UMMA N <= 256).  Rows beyond T and experts
// beyond E are zero-filled by TMA and not stored.
// Every mbarrier wait is bounded (about 2 s of %globaltimer); on expiry the
// kernel records MOE_ERR_TIMEOUT, drains, frees its TMEM and returns.
#include <cuda.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;           // rows of x per CTA (UMMA M)
constexpr int kBK = 64;            // bf16 elements per k-block = one 128-byte swizzle row
constexpr int kUmmaK = 16;         // K of one kind::f16 MMA
constexpr int kATileBytes = kBM * kBK * 2;
constexpr int kThreads = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct GemmArgs {
    float *logits;
    int32_t *status;
    int64_t T;
    int E, num_kb, BN, NC, stages, tmem_cols;
    uint32_t stage_bytes;
    uint32_t idesc;
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase of the given parity; false (and a recorded
// MOE_ERR_TIMEOUT) if it has not completed within the limit.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int32_t *status) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try(bar, parity)) return true;
        if ((it & 255u) == 0u && global_timer_ns() - t0 > kWaitLimitNs) {
            report(status, MOE_ERR_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor, K-major operand with 128-byte swizzle:
// start address >> 4 in bits [0,14), leading byte offset (unused by this
// layout, set to 16 B) in [16,30), stride byte offset = 1024 B (one 8-row
// swizzle atom) in [32,46), descriptor version 1 in [46,48), base offset 0,
// layout type 2 (128-byte swizzle) in [61,64).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3fffu);
    d |= (uint64_t)(16u >> 4) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
    gate_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                     const __grid_constant__ CUtensorMap tmap_w, const GemmArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;  // 128-byte swizzle atoms need 1 KB alignment
    uint8_t *const gbase = smem_raw + (base - raw);
    const int S = a.stages;
    // [stages x stage_bytes tiles][full[S]][empty[S]][tmem_full][tmem slot]
    const uint32_t bar0 = base + (uint32_t)S * a.stage_bytes;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    const uint32_t tmem_full_bar = bar0 + 8u * (2 * S);
    uint32_t *tmem_slot =
        reinterpret_cast<uint32_t *>(gbase + (size_t)S * a.stage_bytes + 8u * (2 * S + 1));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * kBM;

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

    if (warp == 0 && lane == 0) {
        // TMA producer.
        int issued = 0;
        for (int kb = 0; kb < a.num_kb; ++kb) {
            const int s = kb % S;
            const uint32_t ph = (uint32_t)(kb / S) & 1u;
            if (!mbar_wait(empty_bar(s), ph ^ 1u, a.status)) break;
            const uint32_t st = base + (uint32_t)s * a.stage_bytes;
            mbar_arrive_expect_tx(full_bar(s), a.stage_bytes);
            tma_load_2d(st, &tmap_x, full_bar(s), kb * kBK, m0);
            for (int c = 0; c < a.NC; ++c)
                tma_load_2d(st + kATileBytes + (uint32_t)(c * a.BN * 128), &tmap_w, full_bar(s),
                            kb * kBK, c * a.BN);
            issued = kb + 1;
        }
        // Drain: every stage's last issued load has landed before the CTA exits.
        for (int kb = issued - S < 0 ? 0 : issued - S; kb < issued; ++kb)
            if (!mbar_wait(full_bar(kb % S), (uint32_t)(kb / S) & 1u, a.status)) break;
    } else if (warp == 1 && lane == 0) {
        // MMA issuer.
        for (int kb = 0; kb < a.num_kb; ++kb) {
            const int s = kb % S;
            const uint32_t ph = (uint32_t)(kb / S) & 1u;
            if (!mbar_wait(full_bar(s), ph, a.status)) break;
            tc_fence_after();
            const uint32_t st = base + (uint32_t)s * a.stage_bytes;
#pragma unroll
            for (int k = 0; k < kBK / kUmmaK; ++k) {
                const uint64_t adesc = sw128_desc(st + (uint32_t)(k * kUmmaK * 2));
                for (int c = 0; c < a.NC; ++c) {
                    const uint64_t bdesc = sw128_desc(st + kATileBytes +
                                                      (uint32_t)(c * a.BN * 128 + k * kUmmaK * 2));
                    umma_bf16(tmem_base + (uint32_t)(c * a.BN), adesc, bdesc, a.idesc,
                              (kb > 0 || k > 0) ? 1u : 0u);
                }
            }
            umma_commit(empty_bar(s));
        }
        // Signals the epilogue once every MMA issued above has completed (also
        // on the timeout path, so the epilogue never reads a TMEM in use).
        umma_commit(tmem_full_bar);
    } else if (warp >= 4) {
        // Epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = tile rows.
        const int q = warp & 3;
        const bool ok = mbar_wait(tmem_full_bar, 0u, a.status);
        tc_fence_after();
        const int64_t row = (int64_t)m0 + q * 32 + lane;
        const bool vec = (a.E & 3) == 0;
        if (ok) {
            const int ncols = a.NC * a.BN;
            for (int c0 = 0; c0 < ncols; c0 += 16) {
                uint32_t r[16];
                tmem_ld16(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, r);
                // Accumulator chunks sit side by side, so TMEM column j is expert j.
                const int e0 = c0;
                if (row < a.T) {
                    float *dst = a.logits + row * a.E;
                    if (vec && e0 + 16 <= a.E) {
#pragma unroll
                        for (int i = 0; i < 16; i += 4)
                            *reinterpret_cast<float4 *>(dst + e0 + i) =
                                make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]),
                                            __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (e0 + i < a.E) dst[e0 + i] = __uint_as_float(r[i]);
                    }
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

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    }
    return fn;
}

// 2-D bf16 K-major tensor [rows][cols], box = box_rows x 64 columns, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *ptr, int64_t rows, int64_t cols, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_gate_gemm(const moe_bf16_t *x, const moe_bf16_t *w, float *logits,
                                    int64_t T, int32_t d, int32_t E, int32_t *d_status,
                                    moe_stream_t stream) {
    using namespace moe;
    if (T < 0 || E < 1 || E > 512 || d < 8 || d % 8 != 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !w || !logits || !aligned16(x) || !aligned16(w)) return MOE_ERR_INVALID_ARG;
    if (T * (int64_t)E >= (int64_t)INT32_MAX || T >= (int64_t)INT32_MAX)
        return MOE_ERR_UNSUPPORTED;

    GemmArgs a;
    a.logits = logits;
    a.status = d_status;
    a.T = T;
    a.E = E;
    a.num_kb = (d + kBK - 1) / kBK;
    a.NC = E <= 256 ? 1 : 2;
    const int per = (E + a.NC - 1) / a.NC;
    a.BN = (per + 15) / 16 * 16;
    if (a.BN < 16) a.BN = 16;
    const int npad = a.NC * a.BN;
    int cols = 32;
    while (cols < npad) cols *= 2;
    a.tmem_cols = cols;
    a.stage_bytes = (uint32_t)(kATileBytes + npad * 128);
    // D fp32, A and B bf16, both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
    a.idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(a.BN >> 3) << 17) |
              ((uint32_t)(kBM >> 4) << 24);

    int dev = 0, max_smem = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    const int overhead = 1024 + 256;  // alignment slack + barriers and TMEM slot
    int stages = (max_smem - overhead) / (int)a.stage_bytes;
    if (stages > 8) stages = 8;
    if (stages < 2) return MOE_ERR_UNSUPPORTED;
    a.stages = stages;
    const size_t smem = (size_t)stages * a.stage_bytes + overhead;

    CUtensorMap mx, mw;
    if (!make_map(&mx, x, T, d, kBM) || !make_map(&mw, w, E, d, a.BN)) return MOE_ERR_CUDA;
    if (cudaFuncSetAttribute(gate_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    const unsigned grid = (unsigned)((T + kBM - 1) / kBM);
    gate_gemm_kernel<<<grid, kThreads, smem, as_cuda(stream)>>>(mx, mw, a);
    return launch_status();
}
