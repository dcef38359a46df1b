// Device-side building blocks shared by the MSA kernels (sm_100a only).
//
//  - bf16 <-> fp32 unpacking of 16-byte vectors,
//  - mbarrier + cp.async.bulk (TMA bulk copy) helpers with bounded waits,
//  - programmatic dependent launch (PDL) controls,
//  - the selection order of TopK (higher score first, ties to the lower
//    block id) and warp-cooperative sorted top-k lists.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "msa_internal.h"

namespace msa {

constexpr unsigned FULL = 0xffffffffu;

// ---------------------------------------------------------------- elements
// A 16-byte vector of stored elements widened to fp32.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int N = 4;
    __device__ static inline void unpack(const uint4 &u, float (&f)[4]) {
        f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    // a bf16 is the high half of an IEEE fp32: widening is a shift / mask
    __device__ static inline void unpack(const uint4 &u, float (&f)[8]) {
        f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
        f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
        f[4] = __uint_as_float(u.z << 16); f[5] = __uint_as_float(u.z & 0xffff0000u);
        f[6] = __uint_as_float(u.w << 16); f[7] = __uint_as_float(u.w & 0xffff0000u);
    }
};

// FP8 E4M3 codes of MXFP8 index keys: unpacked without their block scale (the scan applies it)
struct e4m3_t {
    uint8_t v;
};
template <> struct Vec16<e4m3_t> {
    static constexpr int N = 16;
    __device__ static inline void unpack(const uint4 &u, float (&f)[16]) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                // two codes, the lower byte first, to two halves, then to fp32 (both exact)
                const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] >> (16 * h)), __NV_E4M3);
                const float2 p = __half22float2(*reinterpret_cast<const __half2 *>(&r));
                f[4 * i + 2 * h] = p.x;
                f[4 * i + 2 * h + 1] = p.y;
            }
    }
};
// An E8M0 scale byte as fp32: 2^(e - 127); 0 gives the subnormal 2^-127, 255 NaN.
__device__ inline float e8m0_to_float(uint32_t e) {
    return e == 0 ? __uint_as_float(0x00400000u) : (e == 255 ? __uint_as_float(0x7fc00000u) : __uint_as_float(e << 23));
}

__device__ inline float load_elem(const float *p) { return *p; }
__device__ inline float load_elem(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ inline void store_elem(float *p, float v) { *p = v; }
__device__ inline void store_elem(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

// ---------------------------------------------------------------- smem / mbarrier / bulk copy
__device__ inline uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ inline void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ inline void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ inline void mbar_arrive_local(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ inline void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ inline bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ inline uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Limit of a bounded wait: the workspace header's wait-limit field (bytes
// 8..15 after the status word, set by msa_set_wait_limit) when it is non-zero,
// else kWaitLimitNs.  Read only once a wait has not completed at once.
__device__ inline uint64_t wait_limit_ns(const int *status) {
    if (status == nullptr) return kWaitLimitNs;
    const uint64_t v = *reinterpret_cast<const volatile uint64_t *>(status + kWaitLimitWord);
    return v != 0 ? v : kWaitLimitNs;
}

// Wait for phase `parity` of an mbarrier for at most wait_limit_ns(status).
// On timeout the workspace status word is set to MSA_ERR_TIMEOUT and false is
// returned; the caller then stops issuing work and drains what it issued.
__device__ inline bool mbar_wait(uint64_t *bar, uint32_t parity, int *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    const uint64_t limit = wait_limit_ns(status);
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit) {
            if (status) atomicExch(status, (int)MSA_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// L2 policy for data read exactly once per call (streamed caches).
__device__ inline uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// L2 policy for data read again soon by other CTAs.
__device__ inline uint64_t l2_evict_normal_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// TMA bulk copy global -> shared (contiguous bytes, 16-byte aligned, size a
// multiple of 16), completion counted on `bar`.
__device__ inline void bulk_g2s(void *smem_dst, const void *gmem_src, uint32_t bytes, uint64_t *bar,
                                uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// ---------------------------------------------------------------- PDL
__device__ inline void pdl_wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ inline void pdl_allow_next_grid() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ inline void named_barrier(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------- selection order
// TopK keeps the best blocks in the order: higher score first, then lower id.
// Empty slots hold (-inf, -1) and lose to every finite score.
__device__ inline bool better(float s1, int i1, float s2, int i2) {
    return s1 > s2 || (s1 == s2 && (unsigned)i1 < (unsigned)i2);
}

// Warp-distributed sorted list of the k best (score, id) pairs, k <= 32:
// lane i holds the i-th best.  (thr_s, thr_i) mirror slot k-1 in every lane
// so that a losing candidate costs one comparison.
struct WarpTopK {
    float s; int id; float thr_s; int thr_i;
    __device__ inline void reset() { s = -INFINITY; id = -1; thr_s = -INFINITY; thr_i = -1; }
    // cs/ci must be warp-uniform.
    __device__ inline void insert(float cs, int ci, int k, int lane) {
        if (!better(cs, ci, thr_s, thr_i)) return;
        const unsigned m = __ballot_sync(FULL, lane < k && better(cs, ci, s, id));
        const int p = __ffs(m) - 1;
        const float us = __shfl_up_sync(FULL, s, 1);
        const int ui = __shfl_up_sync(FULL, id, 1);
        if (lane == p) { s = cs; id = ci; }
        else if (lane > p && lane < k) { s = us; id = ui; }
        thr_s = __shfl_sync(FULL, s, k - 1);
        thr_i = __shfl_sync(FULL, id, k - 1);
    }
};

// insert(cs[g], ci, ...) into l[g] for every g, the N lists in lockstep: one candidate id
// with N scores (the block's max for each of N groups), so that the shuffles of different
// lists are independent instructions.  cs/ci must be warp-uniform.
template <int N>
__device__ inline void warp_topk_insert_all(WarpTopK (&l)[N], const float (&cs)[N], int ci, int k, int lane) {
    bool any = false;
#pragma unroll
    for (int g = 0; g < N; ++g) any |= better(cs[g], ci, l[g].thr_s, l[g].thr_i);
    if (!any) return;
    unsigned m[N];
    float us[N];
    int ui[N];
#pragma unroll
    for (int g = 0; g < N; ++g) {
        m[g] = __ballot_sync(FULL, lane < k && better(cs[g], ci, l[g].s, l[g].id));
        us[g] = __shfl_up_sync(FULL, l[g].s, 1);
        ui[g] = __shfl_up_sync(FULL, l[g].id, 1);
    }
#pragma unroll
    for (int g = 0; g < N; ++g) {
        const int p = m[g] != 0 ? __ffs(m[g]) - 1 : 32;
        if (lane == p) { l[g].s = cs[g]; l[g].id = ci; }
        else if (lane > p && lane < k) { l[g].s = us[g]; l[g].id = ui[g]; }
    }
#pragma unroll
    for (int g = 0; g < N; ++g) {
        l[g].thr_s = __shfl_sync(FULL, l[g].s, k - 1);
        l[g].thr_i = __shfl_sync(FULL, l[g].id, k - 1);
    }
}

// (score, block id) as one 64-bit key whose unsigned order is the selection
// order (higher score first, then lower id): the score's bits made
// order-preserving in the high word, the complemented id in the low word.
__device__ inline unsigned long long sel_key(float s, int id) {
    uint32_t u = __float_as_uint(s + 0.0f);  // -0 -> +0: equal scores compare by id
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)u << 32) | (uint32_t)~(uint32_t)id;
}
__device__ inline void sel_unkey(unsigned long long key, float &s, int &id) {
    uint32_t u = (uint32_t)(key >> 32);
    u = (u & 0x80000000u) ? (u & 0x7fffffffu) : ~u;
    s = __uint_as_float(u);
    id = (int)~(uint32_t)key;
}

// Descending bitonic sort of keys[0, P) (P a power of two) by the whole CTA.
__device__ inline void block_sort_desc(unsigned long long *keys, int P) {
    for (int size = 2; size <= P; size <<= 1)
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < P / 2; i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1)), hi = lo + stride;
                const unsigned long long x = keys[lo], y = keys[hi];
                const bool desc = (lo & size) == 0;
                if (desc ? x < y : x > y) {
                    keys[lo] = y;
                    keys[hi] = x;
                }
            }
            __syncthreads();
        }
}

// The 32 best of two lists of distinct keys, each held descending one key per lane: the
// elementwise max of one list and the other reversed is a bitonic sequence holding the 32
// largest keys, which five half-cleaner steps sort descending.
__device__ inline unsigned long long warp_merge_top32(unsigned long long a, unsigned long long b, int lane) {
    const unsigned long long br = __shfl_sync(FULL, b, 31 - lane);
    unsigned long long c = a > br ? a : br;
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
        const unsigned long long o = __shfl_xor_sync(FULL, c, d);
        c = (lane & d) ? (c < o ? c : o) : (c > o ? c : o);
    }
    return c;
}

// Warp argmax of (s, i) under `better`; every lane receives the winner.
__device__ inline void warp_best(float &s, int &i) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float os = __shfl_xor_sync(FULL, s, off);
        const int oi = __shfl_xor_sync(FULL, i, off);
        if (better(os, oi, s, i)) { s = os; i = oi; }
    }
}

// Merge of n_lists sorted lists (each `len` long, padded with (-inf, -1))
// into the k best, by one warp: lane l owns lists l, l+32, ... (at most
// kMaxOwnedLists each).  Lists live at ls[list * stride + j] / li[...].
// Writes out_s/out_i[0..k) (padded with (-inf, -1)).  Ids must be unique.
template <int kMaxOwned>
__device__ inline void warp_merge_sorted_lists(const float *ls, const int *li, int n_lists, int len, int stride,
                                               int k, float *out_s, int *out_i, int lane) {
    int head[kMaxOwned];
#pragma unroll
    for (int o = 0; o < kMaxOwned; ++o) head[o] = 0;
    for (int r = 0; r < k; ++r) {
        float bs = -INFINITY; int bi = -1; int bo = -1;
#pragma unroll
        for (int o = 0; o < kMaxOwned; ++o) {
            const int l = lane + 32 * o;
            if (l < n_lists && head[o] < len) {
                const float s = ls[(size_t)l * stride + head[o]];
                const int i = li[(size_t)l * stride + head[o]];
                if (i >= 0 && better(s, i, bs, bi)) { bs = s; bi = i; bo = o; }
            }
        }
        float ws = bs; int wi = bi;
        warp_best(ws, wi);
        if (wi >= 0 && wi == bi) {
#pragma unroll
            for (int o = 0; o < kMaxOwned; ++o) if (o == bo) head[o] += 1;
        }
        if (lane == 0) { out_s[r] = ws; out_i[r] = wi; }
    }
}

// ---------------------------------------------------------------- mma.sync fragments
// ldmatrix of four 8x8 b16 matrices (plain and transposed), the bf16
// m16n8k16 MMA with fp32 accumulation, and the byte offset of 16-byte chunk c
// of row `row` in a 128-byte-swizzled tile of 128-byte rows.
__device__ inline void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ inline void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ inline void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// the same product without volatile: a pure function of its registers, which the compiler may
// schedule freely among the operand loads
__device__ inline void mma_16816_pure(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// byte offset of 16-byte vector c (0..7) of row `row` in a 128-byte-swizzled tile of 128-byte rows
__device__ inline uint32_t sw128(int row, int c) { return (uint32_t)(row * 128 + ((c ^ (row & 7)) << 4)); }

}  // namespace msa
