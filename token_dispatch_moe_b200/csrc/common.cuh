// Internal helpers of libmoe_dispatch (device side and launch plumbing).
// Every kernel of the library includes this; nothing outside the library does.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_dispatch.h"

#define MOE_FULL_MASK 0xffffffffu

namespace moe {

inline cudaStream_t as_cuda(moe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// Map the outcome of the launches just issued to a status, clearing the error.
inline moe_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

inline int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return n > 0 ? n : 148;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Programmatic dependent launch: the kernel may be scheduled while the kernel
// before it on the stream finishes.  Such a kernel calls griddep_wait() before
// it touches global memory (that wait returns once the previous grid has
// completed and its writes are visible), and griddep_launch_dependents() once
// its own main work is issued, so the next kernel's launch overlaps its tail.
inline cudaLaunchConfig_t pdl_config(dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                     cudaLaunchAttribute *attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args... args) {
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pdl_config(grid, block, smem, s, attr);
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// First device-side problem wins; later ones are dropped.
__device__ __forceinline__ void report(int32_t *status, int32_t code) {
    if (status) atomicCAS(status, 0, code);
}

// Order-preserving map of an fp32 value to uint32: a larger float gives a
// larger key; -0 and +0 give the same key; NaN gives 1, below every number
// (-inf maps to 0x007fffff); 0 is reserved for "not selectable".
__device__ __forceinline__ uint32_t order_key(float v) {
    if (v != v) return 1u;
    uint32_t u = __float_as_uint(v == 0.0f ? 0.0f : v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(MOE_FULL_MASK, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(MOE_FULL_MASK, v, o));
    return v;
}

// Selection key of the sigmoid score, shared by every routing kernel so that
// they agree bit for bit: 1 / (1 + e^-l) with accurate expf and the hardware
// reciprocal (rcp.approx: at most 1 ulp from the correctly rounded value, a
// relative 6e-8, far inside the 1e-6 band within which the parity rule lets
// near-tied experts swap; its argument is >= 1 and its result in (0, 1], so
// flushing subnormals changes nothing).  Weights use sigmoid_score below.
__device__ __forceinline__ float sigmoid_key(float l) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + expf(-l)));
    return r;
}

// Per-expert scores that do not depend on the rest of the row.
__device__ __forceinline__ float sigmoid_score(float l) { return 1.0f / (1.0f + expf(-l)); }
__device__ __forceinline__ float sqrt_softplus_score(float l) {
    return sqrtf(fmaxf(l, 0.0f) + log1pf(expf(-fabsf(l))));
}

// Selection keys of N logits in place, before the bias: the score function is
// chosen once for the whole array (a branch per logit costs more than the key
// itself).  m and zinv are the row's max and 1 / softmax denominator (read for
// softmax only); the gpt-oss score and monotone keys leave the logits as they are.
template <int N>
__device__ __forceinline__ void score_keys(int score, float (&x)[N], float m, float zinv) {
    if (score == MOE_SCORE_SIGMOID) {
#pragma unroll
        for (int i = 0; i < N; ++i) x[i] = sigmoid_key(x[i]);
    } else if (score == MOE_SCORE_SQRT_SOFTPLUS) {
#pragma unroll
        for (int i = 0; i < N; ++i) x[i] = sqrt_softplus_score(x[i]);
    } else if (score == MOE_SCORE_SOFTMAX) {
#pragma unroll
        for (int i = 0; i < N; ++i) x[i] = expf(x[i] - m) * zinv;
    }
}

// Streaming loads for data read exactly once.
__device__ __forceinline__ float4 ld_stream(const float4 *p) { return __ldcs(p); }
__device__ __forceinline__ float ld_stream(const float *p) { return __ldcs(p); }
__device__ __forceinline__ uint4 ld_stream(const uint4 *p) { return __ldcs(p); }

}  // namespace moe
