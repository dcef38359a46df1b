// Step 2 of MSA for a causal prefill chunk on the tensor cores: every query
// head attends over its group's selected blocks of the real K/V.
//
// Page "MiniMax wird duenn" (atlascloud.ai), section 1, Step 2: the heads of
// a group share one block list, so one set of KV blocks serves all of them
// (Q1/Q2/Q3 -> I1, Q4/Q5/Q6 -> I2).  In prefill every token has its own list;
// a work unit packs TQ = 128 / r consecutive tokens x the r heads of group g
// into one 128-row query tile (row = token * r + head) and walks the sorted
// union of the TQ tokens' lists.  Per union block:
//   S = Q K^T      tcgen05.mma (M=128, N=block, K=16 steps over head_dim),
//                  fp32 accumulator in TMEM (double-buffered);
//   softmax        two warps per TMEM lane quadrant, each on half of the
//                  block's columns: tcgen05.ld of S, mask (block not in this
//                  token's list, or key after the token), row max exchanged
//                  between the two warps through shared memory, running max
//                  with lazy rescaling (the output is rescaled in TMEM only
//                  when the max grows by more than 2^8), P = 2^(z*c - m) as
//                  bf16 into shared memory in the 128-byte swizzle layout;
//   O += P V       tcgen05.mma with V as an MN-major operand, O in TMEM.
// K and V tiles have their own stages: a K stage is refilled as soon as its
// Q K^T has completed, a V stage once its P V has.
// Warp roles: 0 TMA producer of Q and K, 1 MMA issuer and TMEM owner, 2
// builds the per-unit block union and per-token membership masks, 3 TMA
// producer of V, 4-11 softmax and the final normalisation.
#include "tcgen05.cuh"

namespace msa {

namespace {

constexpr int kPaThreads = 384;
constexpr int kPaRows = 128;
constexpr int kPaSm0 = 4;    // first softmax warp
constexpr int kPaSmWarps = 8;
constexpr int kHalf = 16384; // one 128-row x 128-byte operand tile

struct PaBars {
    uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full, pv_done;
    uint64_t q_full, q_empty;
    uint64_t u_full[2], u_empty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
    int u_count[2];
    float red_m[2][2][kPaRows];  // [block parity][column half][row]: raw row max of the half
    float red_l[2][kPaRows];     // [column half][row]: row sum of the half
};

__device__ inline void mbar_arrive1(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ inline void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ inline void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ inline void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 2^x with the hardware approximation (2^-inf = +0).
__device__ __forceinline__ float exp2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Barrier over the two softmax warps of one lane quadrant (64 threads) that
// also ANDs a per-thread flag across them, so both warps leave a loop at the
// same barrier when either has given up a wait.
__device__ inline bool pair_sync_and(int id, bool ok) {
    uint32_t r;
    __syncwarp();
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, 64, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)ok), "r"(id)
        : "memory");
    return r != 0;
}

// Shared-memory descriptor of an MN-major operand in the 128-byte swizzle
// layout: 64-element rows of 128 bytes along N, consecutive K rows 128 bytes
// apart, 8-row groups 1024 bytes apart (stride byte offset), the next 64
// elements of N `lbo` bytes further (leading byte offset).
__device__ inline uint64_t sw128_mnmajor_desc(uint32_t smem_addr, uint32_t lbo) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3fff);
    d |= (uint64_t)((lbo >> 4) & 0x3fff) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

template <int D, int BK>
__global__ void __launch_bounds__(kPaThreads, 1)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap, const PrefillAttnArgs a) {
    constexpr int NH = D / 64;        // 64-dim halves of a row
    constexpr int PH = BK / 64;       // 64-key halves of a P row
    constexpr int KVH = BK * 128;     // bytes of one 64-dim half of a K or V block tile
    constexpr int STAGE = 2 * NH * KVH;
    constexpr uint32_t TMEM_COLS = (2 * BK + D) <= 256 ? 256 : 512;
    constexpr uint32_t O_COL = 2 * BK;
    constexpr int CW = BK / 2;        // S columns of one softmax warp
    constexpr int DW = D / 2;         // O columns of one softmax warp

    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    unsigned char *smQ = base;                       // [NH][128 rows][128 B]
    unsigned char *smP = smQ + NH * kHalf;           // [PH][128 rows][128 B]
    unsigned char *smKV = smP + PH * kHalf;          // [2 stages][K halves | V halves]
    PaBars &S = *reinterpret_cast<PaBars *>(smKV + 2 * STAGE);
    int *u_ids = reinterpret_cast<int *>(&S + 1);    // [2][max_union]
    uint32_t *u_mask = reinterpret_cast<uint32_t *>(u_ids + 2 * a.max_union);  // [2][max_union][MW]
    uint32_t *bitmap = u_mask + 2 * a.max_union * a.mask_words;               // [bitmap_words]
    int *prefix = reinterpret_cast<int *>(bitmap + a.bitmap_words);           // [bitmap_words]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = a.r, TQ = kPaRows / r, MW = a.mask_words;
    const int n_tiles = (a.T + TQ - 1) / TQ;
    const int n_units = a.B * a.G * n_tiles;

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.k_full[i], 1); mbar_init(&S.k_empty[i], 1);
            mbar_init(&S.v_full[i], 1); mbar_init(&S.v_empty[i], 1);
            mbar_init(&S.s_full[i], 1); mbar_init(&S.s_empty[i], kPaSmWarps);
            // K producer, V producer, MMA issuer and the softmax warps release a union slot
            mbar_init(&S.u_full[i], 1); mbar_init(&S.u_empty[i], 3 + kPaSmWarps);
        }
        mbar_init(&S.p_full, kPaSmWarps);
        mbar_init(&S.pv_done, 1);
        mbar_init(&S.q_full, 1);
        mbar_init(&S.q_empty, 1);
        mbar_init(&S.mma_done, 1);
        S.abort_flag = 0;
        fence_mbar_init();
        tc::prefetch_tmap(&qmap);
        tc::prefetch_tmap(&kmap);
        tc::prefetch_tmap(&vmap);
    }
    if (warp == 1) {
        tc::tmem_alloc(&S.tmem_base, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = S.tmem_base;
    volatile int *abort_flag = &S.abort_flag;

    auto unit_of = [&](int u, int &b, int &g, int &t0) {
        const int tile = u % n_tiles;
        const int bg = u / n_tiles;
        b = bg / a.G;
        g = bg % a.G;
        t0 = tile * TQ;
    };

    if (warp == 2) {
        // ------------------------------------------------ union of the tile's block lists
        int ui = 0;
        for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++ui) {
            int b, g, t0;
            unit_of(u, b, g, t0);
            const int slot = ui & 1;
            bool ok = true;
            if (lane == 0) ok = tc::wait_or_abort(&S.u_empty[slot], ((ui >> 1) & 1) ^ 1, abort_flag, a.status);
            if (!__shfl_sync(FULL, ok, 0)) break;
            const int nv = a.T - t0 < TQ ? a.T - t0 : TQ;
            const int nbits = (a.q_start + t0 + nv - 1) / a.Bk + 1;
            const int words = (nbits + 31) >> 5;
            for (int i = lane; i < words; i += 32) bitmap[i] = 0;
            __syncwarp();
            const int *ids = a.ids + (((size_t)b * a.T + t0) * a.G + g) * a.k;
            const size_t tok_stride = (size_t)a.G * a.k;
            for (int i = lane; i < nv * a.k; i += 32) {
                const int tq = i / a.k;
                const int id = ids[tq * tok_stride + i % a.k];
                if (id >= 0 && id * a.Bk <= a.q_start + t0 + tq) atomicOr(&bitmap[id >> 5], 1u << (id & 31));
            }
            __syncwarp();
            int carry = 0;
            for (int w0 = 0; w0 < words; w0 += 32) {
                const int wi = w0 + lane;
                const int c = wi < words ? __popc(bitmap[wi]) : 0;
                int incl = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int v = __shfl_up_sync(FULL, incl, o);
                    if (lane >= o) incl += v;
                }
                if (wi < words) prefix[wi] = carry + incl - c;
                carry += __shfl_sync(FULL, incl, 31);
            }
            const int U = carry;
            __syncwarp();
            int *uid = u_ids + slot * a.max_union;
            uint32_t *um = u_mask + (size_t)slot * a.max_union * MW;
            for (int wi = lane; wi < words; wi += 32) {
                uint32_t bits = bitmap[wi];
                int at = prefix[wi];
                while (bits) {
                    const int bit = __ffs(bits) - 1;
                    uid[at++] = wi * 32 + bit;
                    bits &= bits - 1;
                }
            }
            for (int i = lane; i < U * MW; i += 32) um[i] = 0;
            __syncwarp();
            for (int i = lane; i < nv * a.k; i += 32) {
                const int tq = i / a.k;
                const int id = ids[tq * tok_stride + i % a.k];
                if (id >= 0 && id * a.Bk <= a.q_start + t0 + tq) {
                    const int wi = id >> 5;
                    const int at = prefix[wi] + __popc(bitmap[wi] & ((1u << (id & 31)) - 1u));
                    atomicOr(&um[at * MW + (tq >> 5)], 1u << (tq & 31));
                }
            }
            __syncwarp();
            if (lane == 0) {
                S.u_count[slot] = U;
                mbar_arrive1(&S.u_full[slot]);
            }
        }
    } else if (warp == 0 || warp == 3) {
        // ------------------------------------------------ TMA producers: warp 0 the Q tile and K tiles, warp 3 V tiles
        if (lane == 0) {
            const bool is_k = warp == 0;
            const CUtensorMap *map = is_k ? &kmap : &vmap;
            uint64_t *full = is_k ? S.k_full : S.v_full;
            uint64_t *empty = is_k ? S.k_empty : S.v_empty;
            const int off = is_k ? 0 : NH * KVH;
            int ui = 0, it = 0;
            for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++ui) {
                int b, g, t0;
                unit_of(u, b, g, t0);
                const int slot = ui & 1;
                if (!tc::wait_or_abort(&S.u_full[slot], (ui >> 1) & 1, abort_flag, a.status)) break;
                const int U = S.u_count[slot];
                if (is_k) {
                    if (!tc::wait_or_abort(&S.q_empty, (ui & 1) ^ 1, abort_flag, a.status)) break;
                    mbar_arrive_expect_tx(&S.q_full, NH * kHalf);
                    for (int h = 0; h < NH; ++h)
                        tc::tma_load_3d(smQ + h * kHalf, &qmap, h * 64, g * r, b * a.T + t0, &S.q_full);
                }
                const int *uid = u_ids + slot * a.max_union;
                bool ok = true;
                for (int j = 0; j < U; ++j, ++it) {
                    const int st = it & 1;
                    if (!tc::wait_or_abort(&empty[st], ((it >> 1) & 1) ^ 1, abort_flag, a.status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[st], NH * KVH);
                    const int row = (b * a.G + g) * a.L_max + uid[j] * a.Bk;
                    unsigned char *dst = smKV + st * STAGE + off;
                    for (int h = 0; h < NH; ++h) tc::tma_load_2d(dst + h * KVH, map, h * 64, row, &full[st]);
                }
                mbar_arrive1(&S.u_empty[slot]);
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_qk = tc::idesc_bf16_f32(kPaRows, BK);
            const uint32_t idesc_pv = tc::idesc_bf16_f32(kPaRows, D) | (1u << 16);  // B (V) is MN-major
            int ui = 0, it = 0, sc = 0, pc = 0;
            for (int u = blockIdx.x; u < n_units && !*abort_flag; u += gridDim.x, ++ui) {
                const int slot = ui & 1;
                if (!tc::wait_or_abort(&S.u_full[slot], (ui >> 1) & 1, abort_flag, a.status)) break;
                const int U = S.u_count[slot];
                if (!tc::wait_or_abort(&S.q_full, ui & 1, abort_flag, a.status)) break;
                tc::fence_after_sync();
                const uint32_t q_addr = smem_u32(smQ);
                bool ok = true;
                // Q K^T of block j into S buffer (sc + j) & 1; its K stage is free once it completes
                auto qk = [&](int j) -> bool {
                    const int st = (it + j) & 1;
                    const int sb = (sc + j) & 1;
                    if (!tc::wait_or_abort(&S.k_full[st], ((it + j) >> 1) & 1, abort_flag, a.status)) return false;
                    if (!tc::wait_or_abort(&S.s_empty[sb], (((sc + j) >> 1) & 1) ^ 1, abort_flag, a.status)) return false;
                    tc::fence_after_sync();
                    const uint32_t k_addr = smem_u32(smKV + st * STAGE);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks)
                        tc::mma_bf16_ss(tmem + sb * BK, tc::sw128_kmajor_desc(q_addr + (ks >> 2) * kHalf + (ks & 3) * 32),
                                        tc::sw128_kmajor_desc(k_addr + (ks >> 2) * KVH + (ks & 3) * 32), idesc_qk, ks > 0);
                    tc::mma_commit(&S.k_empty[st]);
                    tc::mma_commit(&S.s_full[sb]);
                    return true;
                };
                if (U > 0 && !qk(0)) break;
                for (int j = 0; j < U; ++j) {
                    if (j + 1 < U && !qk(j + 1)) { ok = false; break; }
                    if (!tc::wait_or_abort(&S.p_full, pc & 1, abort_flag, a.status)) { ok = false; break; }
                    ++pc;
                    const int st = (it + j) & 1;
                    if (!tc::wait_or_abort(&S.v_full[st], ((it + j) >> 1) & 1, abort_flag, a.status)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t v_addr = smem_u32(smKV + st * STAGE + NH * KVH);
                    const uint32_t p_addr = smem_u32(smP);
#pragma unroll
                    for (int ks = 0; ks < BK / 16; ++ks)
                        tc::mma_bf16_ss(tmem + O_COL, tc::sw128_kmajor_desc(p_addr + (ks >> 2) * kHalf + (ks & 3) * 32),
                                        sw128_mnmajor_desc(v_addr + ks * 2048, KVH), idesc_pv, (j > 0 || ks > 0) ? 1u : 0u);
                    tc::mma_commit(&S.v_empty[st]);
                    tc::mma_commit(&S.pv_done);
                }
                if (!ok) break;
                it += U;
                sc += U;
                tc::mma_commit(&S.q_empty);
                mbar_arrive1(&S.u_empty[slot]);
            }
            tc::mma_commit(&S.mma_done);
            mbar_wait(&S.mma_done, 0, a.status);
        }
    } else {
        // ------------------------------------------------ softmax / epilogue
        // Warps w and w + 4 share TMEM lane quadrant w % 4 (one query row per
        // lane); warp half hf takes S columns [hf*CW, hf*CW + CW) and O
        // columns [hf*DW, hf*DW + DW).  Every wait result is made uniform over
        // the pair through pair_sync_and before either warp acts on it, so the
        // two always execute the same sequence of pair barriers.
        const int sw = warp - kPaSm0;
        const int qd = sw & 3, hf = sw >> 2;
        const int pair_bar = 1 + qd;
        const int row = qd * 32 + lane;
        const int tq = row / r, hh = row % r;
        const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
        int ui = 0, sc = 0, pv_waits = 0;
        bool p_zero = false;  // this warp's part of P already holds zeros
        for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++ui) {
            int b, g, t0;
            unit_of(u, b, g, t0);
            const int slot = ui & 1;
            bool ok = __all_sync(FULL, tc::wait_or_abort(&S.u_full[slot], (ui >> 1) & 1, abort_flag, a.status));
            if (!pair_sync_and(pair_bar, ok)) break;
            const int U = S.u_count[slot];
            const int *uid = u_ids + slot * a.max_union;
            const uint32_t *um = u_mask + (size_t)slot * a.max_union * MW;
            const int t = t0 + tq;
            const bool row_live = t < a.T;
            const int pos = a.q_start + t;
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < U; ++j, ++sc) {
                const int sb = sc & 1;
                if (ok) ok = __all_sync(FULL, tc::wait_or_abort(&S.s_full[sb], (sc >> 1) & 1, abort_flag, a.status));
                const int id = uid[j];
                const bool member = row_live && ((um[j * MW + (tq >> 5)] >> (tq & 31)) & 1u);
                const bool active = __any_sync(FULL, member);
                uint32_t zr[CW];
                float mb = -INFINITY;
                if (ok) {
                    if (active) {
                        tc::fence_after_sync();
#pragma unroll
                        for (int c = 0; c < CW / 32; ++c)
                            tc::tmem_ld32(tmem + lane_addr + sb * BK + hf * CW + c * 32,
                                          *reinterpret_cast<uint32_t(*)[32]>(&zr[c * 32]));
                        tc::tmem_ld_wait();
                        tc::fence_before_sync();
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive1(&S.s_empty[sb]);
                    if (active) {
                        // only the block holding the query needs the causal mask
                        const int kb = id * a.Bk + hf * CW;
                        if (member && kb + CW - 1 > pos) {
#pragma unroll
                            for (int c = 0; c < CW; ++c)
                                if (kb + c > pos) zr[c] = __float_as_uint(-INFINITY);
                        }
                        float mx[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) mx[i] = -INFINITY;
#pragma unroll
                        for (int c = 0; c < CW; c += 8)
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                mx[i] = tc::fmax3(mx[i], __uint_as_float(zr[c + 2 * i]), __uint_as_float(zr[c + 2 * i + 1]));
                        mb = member ? fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) : -INFINITY;
                    }
                }
                S.red_m[sc & 1][hf][row] = mb;
                ok = pair_sync_and(pair_bar, ok);
                if (!ok) break;
                // row max of the block (raw scores), then the running max in the log2 domain
                const float mraw = fmaxf(mb, S.red_m[sc & 1][hf ^ 1][row]);
                const float m_new = fmaxf(m, mraw * a.scale_log2);
                const bool grow = m_new > m + 8.f;  // rescale only when the max grows by more than 2^8
                const float alpha = grow ? exp2_approx(m - m_new) : 1.f;
                if (grow) m = m_new;
                // P = 2^(z*c - m) as packed bf16 pairs; rows whose token did not select the block get 0
                uint32_t pk[CW / 2];
                float ps = 0.f;
                if (active) {
                    const float cz = member ? a.scale_log2 : 0.f;
                    const float off = member ? -m : -INFINITY;
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int e = 0; e < CW / 2; ++e) {
                        const float p0 = exp2_approx(fmaf(__uint_as_float(zr[2 * e]), cz, off));
                        const float p1 = exp2_approx(fmaf(__uint_as_float(zr[2 * e + 1]), cz, off));
                        acc[e & 3] += p0 + p1;
                        const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                        pk[e] = *reinterpret_cast<const uint32_t *>(&pb);
                    }
                    ps = (acc[0] + acc[1]) + (acc[2] + acc[3]);
                }
                // the P buffer and O are free once the previous block's P.V has completed
                if (j > 0) {
                    ok = __all_sync(FULL, tc::wait_or_abort(&S.pv_done, pv_waits & 1, abort_flag, a.status));
                    ++pv_waits;
                    if (!ok) continue;  // both warps of the pair leave at the next pair barrier
                    tc::fence_after_sync();
                    if (__any_sync(FULL, alpha != 1.f)) {
#pragma unroll 1
                        for (int c = 0; c < DW / 32; ++c) {
                            uint32_t ov[32];
                            const uint32_t ta = tmem + lane_addr + O_COL + hf * DW + c * 32;
                            tc::tmem_ld32(ta, ov);
                            tc::tmem_ld_wait();
#pragma unroll
                            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                            tmem_st32(ta, ov);
                        }
                        tmem_st_wait();
                    }
                }
                if (active || !p_zero) {
                    if (!active) {
#pragma unroll
                        for (int e = 0; e < CW / 2; ++e) pk[e] = 0u;
                    }
                    p_zero = !active;
                    // this warp's CW keys of the row: 16-byte chunks of P half-tile (hf*CW)/64
#pragma unroll
                    for (int c16 = 0; c16 < CW / 8; ++c16) {
                        const int kc = hf * CW + c16 * 8;  // first key of the chunk
                        unsigned char *dst = smP + (kc >> 6) * kHalf + row * 128 + ((((kc & 63) >> 3) ^ (row & 7)) << 4);
                        *reinterpret_cast<uint4 *>(dst) =
                            make_uint4(pk[c16 * 4], pk[c16 * 4 + 1], pk[c16 * 4 + 2], pk[c16 * 4 + 3]);
                    }
                    fence_proxy_async_smem();
                }
                l = l * alpha + ps;
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive1(&S.p_full);
            }
            // final normalisation once the last P.V has completed
            if (ok && U > 0) {
                ok = __all_sync(FULL, tc::wait_or_abort(&S.pv_done, pv_waits & 1, abort_flag, a.status));
                ++pv_waits;
            }
            S.red_l[hf][row] = l;
            if (!pair_sync_and(pair_bar, ok)) break;
            const float l_row = l + S.red_l[hf ^ 1][row];
            float o_scale = 0.f;
            if (U > 0) {
                tc::fence_after_sync();
                o_scale = l_row > 0.f ? 1.f / l_row : 0.f;
            }
            const int hq = g * r + hh;
            __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(a.o) + (((size_t)b * a.T + t) * a.Hq + hq) * D + hf * DW;
#pragma unroll
            for (int c = 0; c < DW / 32; ++c) {
                uint32_t ov[32];
                if (U > 0) {
                    tc::tmem_ld32(tmem + lane_addr + O_COL + hf * DW + c * 32, ov);
                    tc::tmem_ld_wait();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] = 0u;
                }
                if (row_live) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t pk[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(ov[q * 8 + 2 * e]) * o_scale,
                                                                            __uint_as_float(ov[q * 8 + 2 * e + 1]) * o_scale);
                            pk[e] = *reinterpret_cast<const uint32_t *>(&v2);
                        }
                        *reinterpret_cast<uint4 *>(o + c * 32 + q * 8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                }
            }
            if (hf == 0 && row_live && a.lse != nullptr)
                a.lse[((size_t)b * a.T + t) * a.Hq + hq] = l_row > 0.f ? (m + log2f(l_row)) * 0.69314718055994531f : -INFINITY;
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive1(&S.u_empty[slot]);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <int D, int BK>
cudaError_t launch_pa(const PrefillAttnArgs &a, const CUtensorMap &qm, const CUtensorMap &km, const CUtensorMap &vm,
                      int grid, cudaStream_t s) {
    constexpr int NH = D / 64, PH = BK / 64;
    const size_t smem = 1024 + (size_t)NH * kHalf + (size_t)PH * kHalf + 2 * (2 * NH * BK * 128) + sizeof(PaBars) +
                        (size_t)2 * a.max_union * 4 + (size_t)2 * a.max_union * a.mask_words * 4 +
                        (size_t)a.bitmap_words * 8 + 64;
    if (smem > 232448) return cudaErrorInvalidValue;
    static size_t attr_bytes = 0;
    if (smem > attr_bytes) {
        cudaError_t e =
            cudaFuncSetAttribute(prefill_attn_kernel<D, BK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_bytes = smem;
    }
    prefill_attn_kernel<D, BK><<<grid, kPaThreads, smem, s>>>(qm, km, vm, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_attn(PrefillAttnArgs a, const void *q, const void *k_cache, const void *v_cache, int n_sm,
                                cudaStream_t s, const char **why) {
    const int TQ = kPaRows / a.r;
    a.max_union = TQ * a.k;
    a.mask_words = (TQ + 31) / 32;
    const int nb_all = (a.L_max + a.Bk - 1) / a.Bk;
    a.bitmap_words = (nb_all + 31) / 32;
    CUtensorMap qm, km, vm;
    const unsigned long long qdim[3] = {(unsigned long long)a.D, (unsigned long long)a.Hq,
                                        (unsigned long long)a.B * a.T};
    const unsigned long long qstr[2] = {(unsigned long long)a.D * 2, (unsigned long long)a.Hq * a.D * 2};
    const unsigned qbox[3] = {64, (unsigned)a.r, (unsigned)TQ};
    *why = "encoding the prefill attention tensor maps failed";
    if (!encode_3d(&qm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void *>(q), qdim, qstr, qbox,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const unsigned long long rows = (unsigned long long)a.B * a.G * a.L_max;
    if (!encode_2d(&km, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void *>(k_cache), a.D, rows,
                   (unsigned long long)a.D * 2, 64, a.Bk, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&vm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void *>(v_cache), a.D, rows,
                   (unsigned long long)a.D * 2, 64, a.Bk, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int n_units = a.B * a.G * ((a.T + TQ - 1) / TQ);
    const int grid = n_units < n_sm ? n_units : n_sm;
    *why = "prefill attention launch (shared memory or shape out of range)";
    if (a.D == 128) return a.Bk == 128 ? launch_pa<128, 128>(a, qm, km, vm, grid, s) : launch_pa<128, 64>(a, qm, km, vm, grid, s);
    return a.Bk == 128 ? launch_pa<64, 128>(a, qm, km, vm, grid, s) : launch_pa<64, 64>(a, qm, km, vm, grid, s);
}

}  // namespace msa
