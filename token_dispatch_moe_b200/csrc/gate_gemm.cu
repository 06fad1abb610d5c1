// moe_gate_gemm: fp32 gate logits = x . W^T on Blackwell tensor cores.
//
// Method ("DeepSeek-V3.2-Exp - Select experts", gate forward): the gate is a
// bias-free linear layer evaluated in fp32 on inputs up-cast from the model
// dtype.  bf16 x bf16 products are exact in fp32, so a bf16 tcgen05 MMA with an
// fp32 accumulator computes the same quantity (up to summation order).
//
// sm_100a design: CTA pairs (clusters of two CTAs on two SMs, tcgen05
// cta_group::2), one 256-row M tile per pair, the whole expert dimension as N.
// CTA r of a pair stages rows 128r .. 128r + 127 of the tile's x and half of
// the experts of each accumulator chunk, so each SM stages half of W per
// k-block (deepseek_v3's gate: 250 -> 216 us against one 128-row tile per
// CTA; qwen3_dynk's: 32.0 -> 27.5 us).
//   warp 0      TMA producer (both CTAs): the x tile (128 x 64) and W halves
//               (BN/2 x 64 per chunk) of each k-block into a ring of
//               shared-memory stages, 128-byte swizzle; both CTAs' loads
//               complete on the leader's "full" mbarrier of the stage;
//   warp 1      MMA issuer (the leader's one thread): tcgen05.mma kind::f16,
//               M=256, N=BN, K=16, A and B from both CTAs' shared memory
//               through matrix descriptors (same offsets), each CTA's 128
//               rows of the accumulator in its own TMEM; tcgen05.commit
//               (multicast to both CTAs) frees the stage ("empty" mbarrier)
//               and, after the last k-block, signals both epilogues;
//   warp 2      allocates / frees the TMEM accumulator columns (both CTAs);
//   warps 4..7  epilogue: tcgen05.ld (32 lanes x 16 columns per load), fp32
//               stores of the logits rows, or the route of each row
//               (moe_gate_route).
// E <= 256 is one accumulator of N = round16(E) columns; 256 < E <= 512 is two
// of N = round16(E/2) side by side (UMMA N <= 256).  Rows beyond T and experts
// beyond E are zero-filled by TMA and not stored.
// Every mbarrier wait is bounded (about 2 s of %globaltimer); on expiry the
// kernel records MOE_ERR_TIMEOUT, drains, frees its TMEM and returns.  No TMA
// load uses a cluster-wide multicast.
#include <cuda.h>

#include "common.cuh"
#include "tc.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;           // rows of x per CTA (UMMA M)
constexpr int kBK = 64;            // bf16 elements per k-block = one 128-byte swizzle row
constexpr int kUmmaK = 16;         // K of one kind::f16 MMA
constexpr int kATileBytes = kBM * kBK * 2;
constexpr int kThreads = 256;

struct GemmArgs {
    float *logits;
    int32_t *status;
    int64_t T;
    int E, num_kb, BN, NC, stages, tmem_cols;
    uint32_t stage_bytes;
    uint32_t idesc;
};

// ------------------------------------------------------- fused route epilogue --
// moe_gate_route: the route of moe_route computed in the GEMM epilogue.  A
// TMEM lane holds one token's whole logits row, so each epilogue thread routes
// its own row without any warp-wide step:
//   pass 1  (optional) logits out, NaN flag, row max; softmax denominator when
//           a key or a weight needs it; group scores (top-2 or amax of each
//           contiguous group, in expert order) and the kept groups;
//   pass 2  the P largest keys of kept experts with a branch-free max/min
//           network on fp32 values (fmaxf/fminf are exact), which gives the
//           exact k_t-th largest key tau and how many keys exceed it;
//   pass 3  in expert-id order, every key > tau and the first (k_t - #(> tau))
//           keys == tau (equal keys -> lower id) are appended to a per-thread
//           list in shared memory;
//   then the k_t entries are sorted by (key desc, id asc) and weighted.
// Keys are recomputed from the logits in each pass (for the monotone case the
// key is the logit itself).  NaN keys rank below every number: they enter only
// if fewer than k_t other experts remain.
struct FusedArgs {
    const float *bias;
    const int32_t *kpt;
    int32_t *ids;
    float *w;
    float *logits;  // optional copy of the logits
    int k_max, score, G, TG, topn, renorm, keys_from_scores, gsz;
    float scale;
};

struct RowStats {
    float m, z;  // row max and softmax denominator (when needed)
};

// Keys of the 16 experts c0 .. c0 + 15 from their logits (the same arithmetic
// as the route kernels); experts past E get -inf.
template <bool MONO>
__device__ __forceinline__ void fused_keys16(const FusedArgs &f, const float (&l)[16], int c0,
                                             int E, const RowStats &st, float zinv,
                                             float (&x)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = l[i];
    if (!MONO) {
        score_keys<16>(f.score, x, st.m, zinv);
        if (f.bias) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (c0 + i < E) x[i] += __ldg(f.bias + c0 + i);
        }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i)
        if (c0 + i >= E) x[i] = -INFINITY;
}

__device__ __forceinline__ uint32_t fkey_bits(float v) {
    uint32_t u = __float_as_uint(v);
    u = (v == 0.0f) ? 0u : u;
    const uint32_t o = u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
    return (v != v) ? 1u : o;
}

// Bit i set when expert c0 + i exists and its group is kept.
template <bool GROUPED>
__device__ __forceinline__ uint32_t chunk_mask(uint32_t kept, int c0, int E, int gsz) {
    const uint32_t valid = E - c0 >= 16 ? 0xffffu : (E > c0 ? (1u << (E - c0)) - 1u : 0u);
    if (!GROUPED) return valid;
    uint32_t m = 0u;
    int g = c0 / gsz;
    for (int start = g * gsz; start < c0 + 16 && start < E; ++g, start += gsz) {
        if ((kept >> g) & 1u) {
            const int lo = start > c0 ? start - c0 : 0;
            const int hi = start + gsz < c0 + 16 ? start + gsz - c0 : 16;
            m |= ((hi >= 32 ? 0xffffffffu : (1u << hi) - 1u)) & ~((1u << lo) - 1u);
        }
    }
    return m & valid;
}

// Loads 16 columns of values (keys when keys sit in TMEM, else logits) and
// converts them to keys.
template <bool MONO>
__device__ __forceinline__ void chunk_keys(const FusedArgs &f, uint32_t trow, uint32_t koff,
                                           bool keys_in_tmem, int c0, int E, const RowStats &st,
                                           float zinv, float (&x)[16], float (&l)[16],
                                           bool need_logits) {
    uint32_t r[16], q[16];
    if (MONO || !keys_in_tmem) {
        tmem_ld16_nowait(trow + (uint32_t)c0, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) l[i] = __uint_as_float(r[i]);
        fused_keys16<MONO>(f, l, c0, E, st, zinv, x);
    } else {
        tmem_ld16_nowait(trow + koff + (uint32_t)c0, q);
        if (need_logits) tmem_ld16_nowait(trow + (uint32_t)c0, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            x[i] = __uint_as_float(q[i]);
            l[i] = need_logits ? __uint_as_float(r[i]) : 0.0f;
        }
    }
}

template <int P, bool MONO, bool GROUPED>
__device__ __forceinline__ void route_epilogue(const GemmArgs &g, const FusedArgs &f,
                                               uint32_t trow, int64_t row, bool valid, int tid,
                                               float *gs_s, float *lk, int32_t *li, float *ll) {
    const int E = g.E;
    const int ncols = g.NC * g.BN;
    const uint32_t koff = (uint32_t)ncols;  // key columns follow the logits when stored
    const bool keys_in_tmem = !MONO && 2 * ncols <= g.tmem_cols;
    int kt = f.k_max;
    if (valid && f.kpt) {
        kt = f.kpt[row];
        if (kt < 0 || kt > f.k_max) {
            report(g.status, MOE_ERR_DEVICE_INDEX);
            kt = kt < 0 ? 0 : f.k_max;
        }
    }
    if (!valid) kt = 0;

    // Pass 1: logits out, NaN, row max.
    bool nan = false;
    RowStats st{-INFINITY, 1.0f};
    const bool vec = (E & 3) == 0;
    for (int c0 = 0; c0 < ncols; c0 += 16) {
        uint32_t r[16];
        tmem_ld16_nowait(trow + (uint32_t)c0, r);
        tmem_wait_ld();
        if (valid && f.logits) {
            float *dst = f.logits + row * E + c0;
            if (vec && c0 + 16 <= E) {
#pragma unroll
                for (int i = 0; i < 16; i += 4)
                    *reinterpret_cast<float4 *>(dst + i) =
                        make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]),
                                    __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (c0 + i < E) dst[i] = __uint_as_float(r[i]);
            }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (c0 + i < E) {
                const float v = __uint_as_float(r[i]);
                nan |= v != v;
                st.m = fmaxf(st.m, v);
            }
    }
    if (valid && nan) report(g.status, MOE_ERR_NAN_LOGIT);
    if (f.score == MOE_SCORE_SOFTMAX && (!MONO || !f.renorm)) {
        float z = 0.0f;
        for (int c0 = 0; c0 < ncols; c0 += 16) {
            uint32_t r[16];
            tmem_ld16_nowait(trow + (uint32_t)c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (c0 + i < E) z += expf(__uint_as_float(r[i]) - st.m);
        }
        st.z = z;
    }
    const float zinv = 1.0f / st.z;

    // Keys into spare TMEM columns (score keys only), group scores, kept groups.
    if (!MONO && keys_in_tmem) {
        for (int c0 = 0; c0 < ncols; c0 += 16) {
            uint32_t r[16];
            tmem_ld16_nowait(trow + (uint32_t)c0, r);
            tmem_wait_ld();
            float l[16], x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) l[i] = __uint_as_float(r[i]);
            fused_keys16<MONO>(f, l, c0, E, st, zinv, x);
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(x[i]);
            tmem_st16(trow + koff + (uint32_t)c0, r);
        }
        tmem_wait_st();
    }
    uint32_t kept = 0xffffffffu;
    if (GROUPED) {
        float t1 = -INFINITY, t2 = -INFINITY;
        int gpos = 0, gidx = 0;  // position within the current group, group index
        for (int c0 = 0; c0 < ncols; c0 += 16) {
            float x[16], l[16];
            chunk_keys<MONO>(f, trow, koff, keys_in_tmem, c0, E, st, zinv, x, l, false);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if (c0 + i < E) {
                    if (x[i] > t1) {
                        t2 = t1;
                        t1 = x[i];
                    } else if (x[i] > t2) {
                        t2 = x[i];
                    }
                    if (++gpos == f.gsz) {
                        gs_s[gidx * 128 + tid] = f.topn == 1 ? t1 : t1 + t2;
                        t1 = t2 = -INFINITY;
                        gpos = 0;
                        ++gidx;
                    }
                }
            }
        }
        kept = 0u;
        for (int r = 0; r < f.TG; ++r) {
            uint32_t bk = 0u;
            int bg = 0;
            for (int gg = 0; gg < f.G; ++gg) {
                const uint32_t k = ((kept >> gg) & 1u) ? 0u : fkey_bits(gs_s[gg * 128 + tid]);
                if (k > bk) {
                    bk = k;
                    bg = gg;
                }
            }
            kept |= 1u << bg;
        }
    }

    // Pass 2: the P largest keys (values only; NaN counts as -inf here).
    float L[P];
#pragma unroll
    for (int p = 0; p < P; ++p) L[p] = -INFINITY;
    for (int c0 = 0; c0 < ncols; c0 += 16) {
        float x[16], l[16];
        chunk_keys<MONO>(f, trow, koff, keys_in_tmem, c0, E, st, zinv, x, l, false);
        const uint32_t cm = chunk_mask<GROUPED>(kept, c0, E, f.gsz);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float v = ((cm >> i) & 1u) ? x[i] : -INFINITY;
            v = (v != v) ? -INFINITY : v;
#pragma unroll
            for (int p = 0; p < P; ++p) {
                const float hi = fmaxf(L[p], v);
                v = fminf(L[p], v);
                L[p] = hi;
            }
        }
    }
    float tau = -INFINITY;
    int n_gt = 0;
#pragma unroll
    for (int p = 0; p < P; ++p)
        if (p == kt - 1) tau = L[p];
#pragma unroll
    for (int p = 0; p < P; ++p) n_gt += (p < kt && L[p] > tau) ? 1 : 0;
    const int need_eq = kt - n_gt;

    // Pass 3: collect the selected experts in id order.
    int cnt = 0, eq_seen = 0;
    if (__any_sync(MOE_FULL_MASK, kt > 0)) {
        for (int c0 = 0; c0 < ncols; c0 += 16) {
            float x[16], l[16];
            chunk_keys<MONO>(f, trow, koff, keys_in_tmem, c0, E, st, zinv, x, l, true);
            const uint32_t cm = kt > 0 ? chunk_mask<GROUPED>(kept, c0, E, f.gsz) : 0u;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if ((cm >> i) & 1u) {
                    const bool eq = x[i] == tau;
                    const bool sel = x[i] > tau || (eq && eq_seen < need_eq);
                    eq_seen += eq ? 1 : 0;
                    if (sel && cnt < P) {
                        lk[cnt * 128 + tid] = x[i];
                        li[cnt * 128 + tid] = c0 + i;
                        ll[cnt * 128 + tid] = l[i];
                        ++cnt;
                    }
                }
            }
        }
    }
    // NaN keys fill what is left, in id order (only rows that need it).
    if (__any_sync(MOE_FULL_MASK, nan && cnt < kt)) {
        for (int c0 = 0; c0 < ncols; c0 += 16) {
            float x[16], l[16];
            chunk_keys<MONO>(f, trow, koff, keys_in_tmem, c0, E, st, zinv, x, l, true);
            const uint32_t cm = chunk_mask<GROUPED>(kept, c0, E, f.gsz);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if (((cm >> i) & 1u) && nan && cnt < kt && x[i] != x[i]) {
                    lk[cnt * 128 + tid] = x[i];
                    li[cnt * 128 + tid] = c0 + i;
                    ll[cnt * 128 + tid] = l[i];
                    ++cnt;
                }
            }
        }
    }

    // Order the selected by (key desc, id asc).
    uint32_t sk[P];
    int32_t sid[P];
    float sl[P];
#pragma unroll
    for (int p = 0; p < P; ++p) {
        const bool in = p < cnt;
        sk[p] = in ? fkey_bits(lk[p * 128 + tid]) : 0u;
        sid[p] = in ? li[p * 128 + tid] : 0x7fffffff;
        sl[p] = in ? ll[p * 128 + tid] : 0.0f;
    }
#pragma unroll
    for (int i = 1; i < P; ++i)
#pragma unroll
        for (int j = i; j > 0; --j) {
            const bool sw = sk[j] > sk[j - 1] || (sk[j] == sk[j - 1] && sid[j] < sid[j - 1]);
            const uint32_t tk = sw ? sk[j - 1] : sk[j];
            const int32_t ti = sw ? sid[j - 1] : sid[j];
            const float tl = sw ? sl[j - 1] : sl[j];
            sk[j - 1] = sw ? sk[j] : sk[j - 1];
            sid[j - 1] = sw ? sid[j] : sid[j - 1];
            sl[j - 1] = sw ? sl[j] : sl[j - 1];
            sk[j] = tk;
            sid[j] = ti;
            sl[j] = tl;
        }

    // Weights.
    float sv[P];
    float msel = -INFINITY;
#pragma unroll
    for (int p = 0; p < P; ++p)
        if (p < cnt) msel = fmaxf(msel, sl[p]);
    float sum = 0.0f;
#pragma unroll
    for (int p = 0; p < P; ++p) {
        float x = 0.0f;
        if (p < cnt) {
            if (f.score == MOE_SCORE_SOFTMAX && !f.renorm)
                x = expf(sl[p] - st.m) / st.z;
            else if (f.score == MOE_SCORE_SOFTMAX || f.score == MOE_SCORE_TOPK_SOFTMAX)
                x = expf(sl[p] - msel);
            else if (f.score == MOE_SCORE_SIGMOID)
                x = sigmoid_score(sl[p]);
            else
                x = sqrt_softplus_score(sl[p]);
        }
        sv[p] = x;
        sum += x;
    }
    const bool norm = f.renorm || f.score == MOE_SCORE_TOPK_SOFTMAX;
    if (valid) {
        int32_t *orow = f.ids + row * f.k_max;
        float *wrow = f.w + row * f.k_max;
#pragma unroll
        for (int p = 0; p < P; ++p)
            if (p < f.k_max) {
                const bool act = p < cnt;
                orow[p] = act ? sid[p] : -1;
                wrow[p] = act ? (norm && sum > 0.0f ? sv[p] / sum : sv[p]) * f.scale : 0.0f;
            }
    }
}

// MODE 0: the epilogue stores the logits.  MODE 1: it routes each row (and
// stores the logits only if f.logits is set); MONO: keys are the logits;
// GROUPED: a group limit applies.
// The kernel runs as clusters of two CTAs on two SMs (tcgen05 cta_group::2,
// M = 256 a pair).  CTA r of a pair holds rows 128r ..
// 128r + 127 of the pair's 256 rows of x and, for each accumulator chunk c,
// experts c*BN + r*BN/2 .. c*BN + (r+1)*BN/2 - 1 of W, at the same
// shared-memory offsets in both CTAs, and its own 128 rows of the
// accumulator in its own TMEM: each SM stages half of W per k-block.
//   warp 0 (both CTAs)  waits for its own "empty" stage, then loads its x rows
//                       and its halves of W; both CTAs' loads complete on the
//                       leader's (rank 0) "full" barrier, which the leader
//                       arms with the bytes of both;
//   warp 1 (leader)     issues the MMAs; each commit arrives on that stage's
//                       "empty" barrier in both CTAs, the last one on both
//                       CTAs' "accumulator ready" barrier;
//   warp 2 (both)       allocates the pair's TMEM (cta_group::2);
//   warps 4..7 (both)   the epilogue on the CTA's own 128 rows.
// A cluster barrier follows the barrier set-up (no commit or remote load
// reaches a barrier before it is initialised) and precedes the TMEM free and
// exit (no CTA leaves while the other may still read its shared memory or
// signal its barriers).
template <int MODE, int P, bool MONO, bool GROUPED, int NC>
__global__ void __launch_bounds__(kThreads, 1)
    gate_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                const GemmArgs a, const FusedArgs f) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;  // 128-byte swizzle atoms need 1 KB alignment
    uint8_t *const gbase = smem_raw + (base - raw);
    const int S = a.stages;
    // [stages x stage_bytes tiles][full[S]][empty[S]][tmem_full][tmem slot][epilogue scratch]
    const uint32_t bar0 = base + (uint32_t)S * a.stage_bytes;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    const uint32_t tmem_full_bar = bar0 + 8u * (2 * S);
    uint32_t *tmem_slot =
        reinterpret_cast<uint32_t *>(gbase + (size_t)S * a.stage_bytes + 8u * (2 * S + 1));
    float *epi = reinterpret_cast<float *>(gbase + (size_t)S * a.stage_bytes + 256);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_cta_rank();
    const bool leader = rank == 0;
    const int m0 = (int)(blockIdx.x >> 1) * (2 * kBM) + (int)rank * kBM;
    const int half = a.BN / 2;  // experts of each accumulator chunk staged by each CTA

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(tmem_full_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(a.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    griddep_wait();  // inputs and outputs are free of the previous kernel

    if (warp == 0 && lane == 0) {
        // TMA producer; the loads complete on the leader's barriers.
        const uint32_t lead_full0 = cluster_map(full_bar(0), 0);
        int issued = 0;
        for (int kb = 0; kb < a.num_kb; ++kb) {
            const int s = kb % S;
            const uint32_t ph = (uint32_t)(kb / S) & 1u;
            if (!mbar_wait(empty_bar(s), ph ^ 1u, a.status)) break;
            const uint32_t st = base + (uint32_t)s * a.stage_bytes;
            if (leader) mbar_arrive_expect_tx(full_bar(s), 2u * a.stage_bytes);
            tma_load_2d_pair(st, &tmap_x, lead_full0 + 8u * s, kb * kBK, m0);
            for (int c = 0; c < NC; ++c)
                tma_load_2d_pair(st + kATileBytes + (uint32_t)(c * half * 128), &tmap_w,
                                 lead_full0 + 8u * s, kb * kBK, c * a.BN + (int)rank * half);
            issued = kb + 1;
        }
        // Drain (leader: its full barriers count both CTAs' bytes).
        if (leader)
            for (int kb = issued - S < 0 ? 0 : issued - S; kb < issued; ++kb)
                if (!mbar_wait(full_bar(kb % S), (uint32_t)(kb / S) & 1u, a.status)) break;
    } else if (warp == 1 && lane == 0) {
        // MMA issuer: the leader alone, M = 256, N = BN per chunk.
        if (leader) {
            for (int kb = 0; kb < a.num_kb; ++kb) {
                const int s = kb % S;
                const uint32_t ph = (uint32_t)(kb / S) & 1u;
                if (!mbar_wait(full_bar(s), ph, a.status)) break;
                tc_fence_after();
                const uint32_t st = base + (uint32_t)s * a.stage_bytes;
#pragma unroll
                for (int k = 0; k < kBK / kUmmaK; ++k) {
                    const uint64_t adesc = sw128_desc(st + (uint32_t)(k * kUmmaK * 2));
                    for (int c = 0; c < NC; ++c)
                        umma_bf16_pair(tmem_base + (uint32_t)(c * a.BN), adesc,
                                       sw128_desc(st + kATileBytes +
                                                  (uint32_t)(c * half * 128 + k * kUmmaK * 2)),
                                       a.idesc, (kb > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit_pair(empty_bar(s));
            }
            // Both epilogues go once every MMA above has completed (also after
            // a timeout, so that no epilogue reads a TMEM still being written).
            umma_commit_pair(tmem_full_bar);
        }
    } else if (warp >= 4) {
        // Epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = tile rows.
        const int q = warp & 3;
        // TMEM loads are warp-collective: the whole warp reads or none of it.
        const bool ok = __all_sync(MOE_FULL_MASK, mbar_wait(tmem_full_bar, 0u, a.status));
        tc_fence_after();
        const int64_t row = (int64_t)m0 + q * 32 + lane;
        const uint32_t trow = tmem_base + ((uint32_t)(q * 32) << 16);
        if (MODE == 0) {
            const bool vec = (a.E & 3) == 0;
            if (ok) {
                const int ncols = NC * a.BN;
                for (int c0 = 0; c0 < ncols; c0 += 16) {
                    uint32_t r[16];
                    tmem_ld16(trow + (uint32_t)c0, r);
                    // Accumulator chunks sit side by side, so TMEM column j is expert j.
                    const int e0 = c0;
                    if (row < a.T) {
                        float *dst = a.logits + row * a.E;
                        if (vec && e0 + 16 <= a.E) {
#pragma unroll
                            for (int i = 0; i < 16; i += 4)
                                *reinterpret_cast<float4 *>(dst + e0 + i) = make_float4(
                                    __uint_as_float(r[i]), __uint_as_float(r[i + 1]),
                                    __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
                        } else {
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                if (e0 + i < a.E) dst[e0 + i] = __uint_as_float(r[i]);
                        }
                    }
                }
            }
        } else if (ok) {
            const int tid = q * 32 + lane;  // 0..127
            float *gs_s = epi;              // [32][128] group scores
            float *lk = gs_s + 32 * 128;    // [P][128] selected keys
            int32_t *li = reinterpret_cast<int32_t *>(lk + P * 128);
            float *ll = reinterpret_cast<float *>(li + P * 128);
            route_epilogue<P, MONO, GROUPED>(a, f, trow, row, row < a.T, tid, gs_s, lk, li, ll);
        }
    }

    tc_fence_before();
    cluster_sync();
    griddep_launch_dependents();
    if (warp == 2) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(a.tmem_cols)
                     : "memory");
    }
}

// Shapes, stage count and shared-memory size of one launch.
moe_status plan_gemm(int64_t T, int32_t d, int32_t E, size_t epi_bytes, GemmArgs &a,
                     size_t &smem) {
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
    // Each CTA of a pair stages its 128 rows of x and half of each chunk's experts.
    a.stage_bytes = (uint32_t)(kATileBytes + a.NC * (a.BN / 2) * 128);
    // D fp32, A and B bf16, both K-major, N >> 3 at bit 17, M >> 4 at bit 24
    // (M = 256: the pair's two 128-row halves).
    a.idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(a.BN >> 3) << 17) |
              ((uint32_t)((2 * kBM) >> 4) << 24);
    int dev = 0, max_smem = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    const int overhead = 1024 + 256;  // alignment slack + barriers and TMEM slot
    const int static_smem = 1024;     // the kernel's own __shared__ alignment block
    int stages = (int)((max_smem - static_smem - overhead - (int64_t)epi_bytes) /
                       (int)a.stage_bytes);
    if (stages > 8) stages = 8;
    if (stages < 2) return MOE_ERR_UNSUPPORTED;
    // More CTAs than SMs (several waves), a plain epilogue and at most half of
    // the TMEM: two CTAs per SM, so that one's epilogue and pipeline fill
    // overlap the other's mainloop, with as many stages as half of the SM's
    // shared memory holds.
    const int64_t tiles = 2 * ((T + 2 * kBM - 1) / (2 * kBM));
    int per_sm_smem = 0;
    if (epi_bytes == 0 && a.tmem_cols <= 256 && tiles > sm_count() &&
        cudaDeviceGetAttribute(&per_sm_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) ==
            cudaSuccess) {
        const int half = per_sm_smem / 2 - 1024;  // 1 KB per block is reserved by the system
        const int s2 = (half - static_smem - overhead) / (int)a.stage_bytes;
        if (s2 >= 2) stages = s2 < stages ? s2 : stages;
    }
    cudaGetLastError();
    a.stages = stages;
    smem = (size_t)stages * a.stage_bytes + overhead + epi_bytes;
    return MOE_OK;
}

// The chunk count is a template argument: a runtime loop over it in the MMA
// issue measured 5 us slower at qwen3_dynk (30.6 against 26.5 us).
template <int MODE, int P, bool MONO, bool GROUPED, int NC>
moe_status launch_gate_nc(const moe_bf16_t *x, const moe_bf16_t *w, const GemmArgs &a,
                       const FusedArgs &f, size_t smem, int32_t d, moe_stream_t stream) {
    CUtensorMap mx, mw;
    if (!make_map(&mx, x, a.T, d, kBM) || !make_map(&mw, w, a.E, d, a.BN / 2)) return MOE_ERR_CUDA;
    if (cudaFuncSetAttribute(gate_kernel<MODE, P, MONO, GROUPED, NC>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    // One pair of CTAs (a cluster of two) per 256 rows.
    const unsigned grid = (unsigned)(2 * ((a.T + 2 * kBM - 1) / (2 * kBM)));
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = pdl_config(dim3(grid), dim3(kThreads), smem, as_cuda(stream), attr);
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, gate_kernel<MODE, P, MONO, GROUPED, NC>, mx, mw, a, f) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return launch_status();
}

template <int MODE, int P, bool MONO = true, bool GROUPED = false>
moe_status launch_gate(const moe_bf16_t *x, const moe_bf16_t *w, const GemmArgs &a,
                       const FusedArgs &f, size_t smem, int32_t d, moe_stream_t stream) {
    return a.NC == 1 ? launch_gate_nc<MODE, P, MONO, GROUPED, 1>(x, w, a, f, smem, d, stream)
                     : launch_gate_nc<MODE, P, MONO, GROUPED, 2>(x, w, a, f, smem, d, stream);
}

template <bool MONO, bool GROUPED>
moe_status launch_fused_p(int P, const moe_bf16_t *x, const moe_bf16_t *w, const GemmArgs &a,
                          const FusedArgs &f, size_t smem, int32_t d, moe_stream_t stream) {
    switch (P) {
        case 1: return launch_gate<1, 1, MONO, GROUPED>(x, w, a, f, smem, d, stream);
        case 2: return launch_gate<1, 2, MONO, GROUPED>(x, w, a, f, smem, d, stream);
        case 4: return launch_gate<1, 4, MONO, GROUPED>(x, w, a, f, smem, d, stream);
        case 8: return launch_gate<1, 8, MONO, GROUPED>(x, w, a, f, smem, d, stream);
        default: return launch_gate<1, 16, MONO, GROUPED>(x, w, a, f, smem, d, stream);
    }
}

moe_status launch_fused(int P, bool mono, bool grouped, const moe_bf16_t *x, const moe_bf16_t *w,
                        const GemmArgs &a, const FusedArgs &f, size_t smem, int32_t d,
                        moe_stream_t stream) {
    if (mono)
        return grouped ? launch_fused_p<true, true>(P, x, w, a, f, smem, d, stream)
                       : launch_fused_p<true, false>(P, x, w, a, f, smem, d, stream);
    return grouped ? launch_fused_p<false, true>(P, x, w, a, f, smem, d, stream)
                   : launch_fused_p<false, false>(P, x, w, a, f, smem, d, stream);
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
    size_t smem = 0;
    moe_status st = plan_gemm(T, d, E, 0, a, smem);
    if (st != MOE_OK) return st;
    FusedArgs f{};
    return launch_gate<0, 1>(x, w, a, f, smem, d, stream);
}

extern "C" moe_status moe_gate_route(const moe_bf16_t *x, const moe_bf16_t *w, const float *bias,
                                     const int32_t *k_per_token, const moe_route_params *p,
                                     int64_t T, int32_t d, int32_t *topk_ids, float *topk_w,
                                     float *logits, int32_t *d_status, moe_stream_t stream) {
    using namespace moe;
    if (!p || T < 0 || d < 8 || d % 8 != 0) return MOE_ERR_INVALID_ARG;
    const int E = p->num_experts, G = p->n_groups;
    if (E < 1 || E > 512 || p->k_max < 0 || p->k_max > E) return MOE_ERR_INVALID_ARG;
    if (p->score < MOE_SCORE_SOFTMAX || p->score > MOE_SCORE_TOPK_SOFTMAX || G < 1 || E % G != 0)
        return MOE_ERR_INVALID_ARG;
    if (G > 32 || p->k_max > 16) return MOE_ERR_UNSUPPORTED;
    if (G > 1 && (p->topk_groups < 1 || p->topk_groups > G || p->group_topn < 1 ||
                  p->group_topn > 2 || p->group_topn > E / G || p->k_max > p->topk_groups * (E / G)))
        return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !w || !topk_ids || !topk_w || !aligned16(x) || !aligned16(w))
        return MOE_ERR_INVALID_ARG;
    if (T * (int64_t)E >= (int64_t)INT32_MAX || T >= (int64_t)INT32_MAX / 16)
        return MOE_ERR_UNSUPPORTED;
    int P = 1;
    while (P < p->k_max) P *= 2;
    GemmArgs a;
    a.logits = logits;
    a.status = d_status;
    FusedArgs f;
    f.bias = bias;
    f.kpt = k_per_token;
    f.ids = topk_ids;
    f.w = topk_w;
    f.logits = logits;
    f.k_max = p->k_max;
    f.score = p->score;
    f.G = G;
    f.TG = G > 1 ? p->topk_groups : 1;
    f.topn = G > 1 ? p->group_topn : 1;
    f.renorm = p->renormalize ? 1 : 0;
    f.keys_from_scores = (bias != nullptr) || (G > 1 && f.topn > 1);
    f.gsz = E / G;
    f.scale = p->route_scale;
    const size_t epi = (size_t)32 * 128 * 4 + (size_t)P * 128 * 12;
    size_t smem = 0;
    moe_status st = plan_gemm(T, d, E, epi, a, smem);
    if (st != MOE_OK) return st;
    // Score keys keep a copy in spare TMEM columns when the accumulator uses at
    // most half of the 512 columns.
    if (f.keys_from_scores && a.NC * a.BN <= 256) a.tmem_cols = 512;
    const bool mono = !f.keys_from_scores;
    const bool grouped = G > 1;
    return launch_fused(P, mono, grouped, x, w, a, f, smem, d, stream);
}
