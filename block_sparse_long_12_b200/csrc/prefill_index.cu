// Step 1 of MSA for a causal prefill chunk on the tensor cores: index scores,
// block max pool and TopK, fused (scores never leave the SM).
//
// Page "MiniMax wird duenn" (atlascloud.ai), section 1, Step 1: the group's
// index query scores every visible token (Q_idx . K_idx^T), the scores are
// max-pooled per fixed block and TopK keeps the best blocks of the group.
// In prefill every query row has its own index query, so Step 1 is a causal
// GEMM with a reduction epilogue; section 3 of the page notes that this scan
// of the full input remains in prefill.
//
// A work unit is (sequence b, group g, 256 query rows) against all the key
// tiles its rows can see.  When the units alone would leave the last wave of
// CTAs part-empty, each unit's keys are cut into n_seg segments (whole
// blocks); the pieces are taken segment by segment, heaviest unit first, so
// the CTAs running at the same time read the same keys of a group (shared in
// L2), and the SMs finish together.  A unit cut into segments leaves one
// per-row list per segment in the workspace; the CTA that finishes its last
// segment merges them (same order: higher score, then lower block id).
// Warp roles:
//   warp 0      TMA producer: the unit's two 128-row index-query tiles, then
//               the index-key tiles (128 keys x 64 dims, 128-byte swizzle)
//               through a kStages ring;
//   warp 1      owns 512 TMEM columns and issues tcgen05.mma (M=128, N=128,
//               K=16, bf16 in, fp32 accumulate) for both row tiles into a
//               double-buffered pair of accumulators;
//   warps 4-19  epilogue, one TMEM lane (= query row) per thread, in two
//               groups of 8 warps that take alternate blocks of tiles:
//               tcgen05.ld of the scores, causal mask on diagonal tiles,
//               3-input max per 32 columns, block max, and a sorted top-k per
//               row in shared memory; the groups' lists are merged per row
//               when the piece ends.  For k beyond the lists (large k) the
//               epilogue stores every visible block's score instead, and a
//               radix select per row (large_topk.cu) keeps the k best.
// The next tile's MMAs overlap the epilogue of the current one.
#include "tcgen05.cuh"

namespace msa {

namespace {

constexpr int kRows = 128;              // rows per accumulator (one TMEM lane each)
constexpr int kAccs = 2;                // row tiles per unit
constexpr int kUnitRows = kRows * kAccs;
constexpr int kKeys = 128;              // keys per tile (N)
constexpr int kThreads = 640;           // 4 control warps + 16 epilogue warps
constexpr int kEpiWarp0 = 4;
constexpr int kEpiThreads = 512;
// ring stages: the per-row lists take K x 512 x 8 bytes of shared memory (K = 0: no lists, the
// block scores are stored for a radix select)
template <int K> struct PiShape { static constexpr int S = K >= 32 ? 4 : 6; };
constexpr int kMaxStages = 6;
constexpr int kTileBytes = kKeys * 128; // 128 rows of 64 bf16
constexpr int kABytes = kRows * 128;
constexpr uint32_t kTmemCols = 512;     // 2 buffers x 2 accumulators x 128 columns

struct Smem {
    // 1024-byte aligned operand tiles come first (set up by hand in the kernel)
    uint64_t full[kMaxStages], empty[kMaxStages];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t a_full, a_empty, mma_done;
    uint32_t tmem_base;
    int abort_flag;
    int merge_here;  // this CTA finished the last segment of a split unit
};

// One piece of work: segment s of unit u = i * (B*G) + bg, key tiles [n0, n1)
// of the unit's nt, which has n_parts non-empty segments.
struct Piece {
    int u, i, bg, s, n0, n1, nt, n_parts;
};

__device__ inline void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Row-wise sorted top-K (score desc, id asc) kept in shared memory, entry i of
// list j at [i * kEpiThreads + j] (consecutive threads, consecutive words); the
// K-th entry is mirrored in registers so that a losing block costs one compare.
// K = 0 (large k): block scores are staged per row in shared memory, 32 blocks per window and
// two windows, rows padded to kStageRow floats (16-byte reads of different rows stay clear of
// each other's banks), and written to the workspace a window at a time as whole 64-byte runs.
constexpr int kStageRow = 36;
constexpr int kStageFloats = kUnitRows * kStageRow;  // one window
template <int K> constexpr size_t stage_bytes() { return K == 0 ? (size_t)2 * kStageFloats * 4 : 0; }

template <int K>
struct SmemTopK {
    float *s;
    int *id;
    int j;
    float thr_s;
    int thr_i;
    float *store = nullptr;  // K = 0: this row in window buffer 0 of the stage
    __device__ inline void reset() {
        if constexpr (K == 0) return;
#pragma unroll
        for (int i = 0; i < K; ++i) { s[i * kEpiThreads + j] = -INFINITY; id[i * kEpiThreads + j] = 0x7fffffff; }
        thr_s = -INFINITY;
        thr_i = 0x7fffffff;
    }
    __device__ inline void insert(float cs, int ci) {
        if constexpr (K == 0) {
            store[((ci >> 5) & 1) * kStageFloats + (ci & 31)] = cs;
            return;
        }
        if (!better(cs, ci, thr_s, thr_i)) return;
#pragma unroll
        for (int i = 0; i < K; ++i) {
            const float ts = s[i * kEpiThreads + j];
            const int ti = id[i * kEpiThreads + j];
            if (better(cs, ci, ts, ti)) {
                s[i * kEpiThreads + j] = cs;
                id[i * kEpiThreads + j] = ci;
                cs = ts;
                ci = ti;
            }
        }
        thr_s = s[(K - 1) * kEpiThreads + j];
        thr_i = id[(K - 1) * kEpiThreads + j];
    }
};

// Barrier over nthreads threads (named barrier id) that also ANDs a per-thread flag across them.
__device__ inline bool epi_sync_and(int id, int nthreads, bool ok) {
    uint32_t r;
    __syncwarp();
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)ok), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// Max over the 32 keys j0..j0+31 of one row, counting only keys j <= pos.
__device__ inline float chunk_max_masked(const uint32_t (&r)[32], int j0, int pos) {
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < 32; ++i) m = (j0 + i <= pos) ? fmaxf(m, __uint_as_float(r[i])) : m;
    return m;
}

template <int K, int BK>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_index_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                         const PrefillIdxArgs a) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    unsigned char *base = smem_raw + ((1024 - (raw & 1023)) & 1023);
    unsigned char *smA = base;                               // [kAccs][128 rows][128 B]
    constexpr int kStages = PiShape<K>::S;
    unsigned char *smB = base + kAccs * kABytes;             // [kStages][128 keys][128 B]
    float *list_s = reinterpret_cast<float *>(smB + kStages * kTileBytes);  // [K][512]
    int *list_i = reinterpret_cast<int *>(list_s + K * kEpiThreads);        // [K][512]
    float *stage = reinterpret_cast<float *>(list_i + K * kEpiThreads);     // K = 0: [2][256][kStageRow]
    Smem &S = *reinterpret_cast<Smem *>(reinterpret_cast<unsigned char *>(stage) + stage_bytes<K>());

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int BG = a.B * a.G;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) { mbar_init(&S.full[i], 1); mbar_init(&S.empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&S.acc_full[i], 1); mbar_init(&S.acc_empty[i], 8); }
        mbar_init(&S.a_full, 1);
        mbar_init(&S.a_empty, 1);
        mbar_init(&S.mma_done, 1);
        S.abort_flag = 0;
        fence_mbar_init();
        tc::prefetch_tmap(&qmap);
        tc::prefetch_tmap(&kmap);
    }
    if (warp == 1) {
        tc::tmem_alloc(&S.tmem_base, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = S.tmem_base;
    volatile int *abort_flag = &S.abort_flag;

    // every role takes the same pieces (segment-major, heaviest unit first) and skips the empty ones
    const int n_units = a.n_mt * BG;
    const int n_pieces = n_units * a.n_seg;
    auto piece_of = [&](int p, Piece &w) -> bool {
        w.s = p / n_units;
        w.u = p - w.s * n_units;
        w.i = w.u / BG;
        w.bg = w.u - w.i * BG;
        w.nt = prefill_unit_tiles(w.i, a.n_mt, a.T, a.q_start, a.Bk);
        const int len = a.n_seg > 1 ? prefill_seg_tiles(w.nt, a.n_seg, a.Bk) : w.nt;
        w.n0 = w.s * len;
        w.n1 = w.n0 + len < w.nt ? w.n0 + len : w.nt;
        w.n_parts = (w.nt + len - 1) / len;
        return w.n0 < w.nt;
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int it = 0, pc = 0;
            Piece w;
            for (int p = blockIdx.x; p < n_pieces; p += gridDim.x) {
                if (!piece_of(p, w)) continue;
                const int b = w.bg / a.G, g = w.bg % a.G, m0 = (a.n_mt - 1 - w.i) * kUnitRows;
                if (!tc::wait_or_abort(&S.a_empty, (pc++ & 1) ^ 1, abort_flag, a.status)) break;
                mbar_arrive_expect_tx(&S.a_full, kAccs * kABytes);
                for (int acc = 0; acc < kAccs; ++acc)
                    tc::tma_load_3d(smA + acc * kABytes, &qmap, 0, g, b * a.T + m0 + acc * kRows, &S.a_full);
                const int hik = g % a.Hik;
                bool ok = true;
                for (int n = w.n0; n < w.n1; ++n, ++it) {
                    const int st = it % kStages;
                    if (!tc::wait_or_abort(&S.empty[st], ((it / kStages) & 1) ^ 1, abort_flag, a.status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&S.full[st], kTileBytes);
                    // a 128-key tile lies inside one page (paged caches have pages of a multiple of 128 keys)
                    tc::tma_load_2d(smB + st * kTileBytes, &kmap, 0, a.cache.row(b, hik, a.Hik, a.L_max, n * kKeys),
                                    &S.full[st]);
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_bf16_f32(kRows, kKeys);
            // descriptor bases (the issue loop only adds offsets: see tc::desc_add)
            const uint64_t ad0 = tc::sw128_kmajor_desc(smem_u32(smA)), bd0 = tc::sw128_kmajor_desc(smem_u32(smB));
            int it = 0, ti = 0, pc = 0;
            Piece w;
            for (int p = blockIdx.x; p < n_pieces && !*abort_flag; p += gridDim.x) {
                if (!piece_of(p, w)) continue;
                if (!tc::wait_or_abort(&S.a_full, pc++ & 1, abort_flag, a.status)) break;
                tc::fence_after_sync();
                bool ok = true;
                for (int n = w.n0; n < w.n1; ++n, ++it, ++ti) {
                    const int st = it % kStages;
                    const int buf = ti & 1;
                    if (!tc::wait_or_abort(&S.full[st], (it / kStages) & 1, abort_flag, a.status) ||
                        !tc::wait_or_abort(&S.acc_empty[buf], ((ti >> 1) & 1) ^ 1, abort_flag, a.status)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint64_t bd = tc::desc_add(bd0, (uint32_t)(st * kTileBytes));
                    const uint32_t d0 = tmem + (uint32_t)(buf * kAccs * kKeys);
#pragma unroll
                    for (int acc = 0; acc < kAccs; ++acc) {
                        const uint64_t ad = tc::desc_add(ad0, acc * kABytes);
                        const uint32_t d = d0 + acc * kKeys;
                        tc::mma_bf16_ss_c<false>(d, ad, bd, idesc);
#pragma unroll
                        for (int ks = 1; ks < 4; ++ks)
                            tc::mma_bf16_ss_c<true>(d, tc::desc_add(ad, ks * 32), tc::desc_add(bd, ks * 32), idesc);
                    }
                    tc::mma_commit(&S.empty[st]);
                    tc::mma_commit(&S.acc_full[buf]);
                }
                if (!ok) break;
                tc::mma_commit(&S.a_empty);
            }
            // every MMA issued by this thread has completed before TMEM is released
            tc::mma_commit(&S.mma_done);
            mbar_wait(&S.mma_done, 0, a.status);
        }
    } else if (warp >= kEpiWarp0) {
        // ------------------------------------------------ epilogue: one query row per thread
        // two groups of 8 warps take alternate blocks of tiles; each keeps its own list per row and
        // the two lists are merged when the piece ends
        const int e = warp - kEpiWarp0;
        const int grp = e >> 3;
        const int q4 = warp & 3, acc = (e >> 2) & 1;
        const int rl = acc * kRows + q4 * 32 + lane;  // row within the unit
        const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
        // With blocks of at most one tile, group n & 1 takes tile n, so within a piece each group
        // consumes the phases of one accumulator buffer in order (the piece-end barriers keep the
        // groups in step across pieces).  Blocks spanning two tiles go to group 0 alone: a group
        // skipping tiles of its own buffer could otherwise wait on a phase two steps ahead.
        constexpr bool two_groups = BK <= kKeys;
        SmemTopK<K> top{list_s, list_i, e * 32 + lane};
        int ti = 0;
        bool ok = true;
        Piece w;
        for (int p = blockIdx.x; p < n_pieces; p += gridDim.x) {
            if (!piece_of(p, w)) continue;
            const int b = w.bg / a.G, g = w.bg % a.G, m0 = (a.n_mt - 1 - w.i) * kUnitRows;
            const int t = m0 + rl;
            const int pos = a.q_start + t;
            const int pos_min = a.q_start + m0;  // smallest position of the unit
            // MSA_FORCE_SINK_LOCAL: block 0 and the row's own block rank above every score (large
            // k: the radix select applies it to the stored scores)
            auto forced = [&](int blk) { return K > 0 && a.force && (blk == 0 || blk == pos / BK); };
            top.reset();
            if constexpr (K == 0) top.store = stage + rl * kStageRow;
            // K = 0: the piece's blocks, and the stage written to the workspace after each window's
            // last block (every epilogue thread takes part, so no thread leaves the tile loop early)
            const int blk_lo = w.n0 * kKeys / BK, blk_hi = (w.n1 * kKeys + BK - 1) / BK - 1;
            auto flush = [&](int win) {
                const int te = e * 32 + lane, r = te >> 1, h = te & 1, tr = m0 + r;
                const int c0 = win * 32 + h * 16;
                if (tr >= a.T) return;
                const float *src = stage + (win & 1) * kStageFloats + r * kStageRow + h * 16;
                float *dst = a.blk_scores + (((long long)b * a.T + tr) * a.G + g) * a.blk_stride + c0;
                if (c0 >= blk_lo && c0 + 15 <= blk_hi) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        reinterpret_cast<float4 *>(dst)[q] = reinterpret_cast<const float4 *>(src)[q];
                } else {
                    for (int i = 0; i < 16; ++i)
                        if (c0 + i >= blk_lo && c0 + i <= blk_hi) dst[i] = src[i];
                }
            };
            float bm = -INFINITY;
            // one tile of this group: scores from TMEM, causal mask on diagonal tiles, maxima per 32
            // columns, block maxima into the row's list (or the stage); false when a wait gave up
            auto do_tile = [&](int n, int ti_) -> bool {
                const int buf = ti_ & 1;
                if (!__all_sync(FULL, tc::wait_or_abort(&S.acc_full[buf], (ti_ >> 1) & 1, abort_flag, a.status)))
                    return false;
                tc::fence_after_sync();
                const uint32_t col = tmem + lane_addr + (uint32_t)((buf * kAccs + acc) * kKeys);
                const int kb = n * kKeys;
                const bool diag = kb + kKeys - 1 > pos_min;
                float cm[4];
                {
                    uint32_t r0[32], r1[32];
                    tc::tmem_ld32(col, r0);
                    tc::tmem_ld32(col + 32, r1);
                    tc::tmem_ld_wait();
                    cm[0] = diag ? chunk_max_masked(r0, kb, pos) : tc::max32(r0);
                    cm[1] = diag ? chunk_max_masked(r1, kb + 32, pos) : tc::max32(r1);
                    tc::tmem_ld32(col + 64, r0);
                    tc::tmem_ld32(col + 96, r1);
                    tc::tmem_ld_wait();
                    cm[2] = diag ? chunk_max_masked(r0, kb + 64, pos) : tc::max32(r0);
                    cm[3] = diag ? chunk_max_masked(r1, kb + 96, pos) : tc::max32(r1);
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.acc_empty[buf]);
                // block maxima (BK is a compile-time block size: the block ends fold away); only the
                // diagonal tiles can hold blocks that start after the row
                if constexpr (BK >= kKeys) {
                    bm = fmaxf(bm, tc::fmax3(cm[0], cm[1], fmaxf(cm[2], cm[3])));
                    if ((n + 1) % (BK / kKeys) == 0) {  // last tile of block n / (BK / kKeys)
                        const int blk = n / (BK / kKeys);
                        if (!diag || blk * BK <= pos) top.insert(forced(blk) ? INFINITY : bm, blk);
                        bm = -INFINITY;
                    }
                } else {
                    constexpr int CPB = BK / 32;  // 32-column chunks per block
#pragma unroll
                    for (int q = 0; q < 4 / CPB; ++q) {
                        float v = cm[q * CPB];
#pragma unroll
                        for (int c = 1; c < CPB; ++c) v = fmaxf(v, cm[q * CPB + c]);
                        const int blk = n * (kKeys / BK) + q;
                        if (!diag || blk * BK <= pos) top.insert(forced(blk) ? INFINITY : v, blk);
                    }
                }
                return true;
            };
            if constexpr (K == 0) {
                // every epilogue thread walks every tile of the piece (no thread leaves early), so that
                // all of them meet at each window's end: a window ends with its 32nd block or the piece
                for (int n = w.n0; n < w.n1; ++n, ++ti) {
                    const int last_blk = BK >= kKeys ? ((n + 1) % (BK / kKeys) == 0 ? n / (BK / kKeys) : -1)
                                                     : (n + 1) * (kKeys / BK) - 1;
                    const bool win_end = last_blk >= 0 && ((last_blk & 31) == 31 || n == w.n1 - 1);
                    if (ok && (two_groups ? (n & 1) : 0) == grp) ok = do_tile(n, ti);
                    if (win_end) {
                        ok = epi_sync_and(3, kEpiThreads, ok);
                        if (ok) flush(last_blk >> 5);
                    }
                }
            } else {
                for (int n = w.n0; n < w.n1 && ok; ++n, ++ti) {
                    if ((two_groups ? (n & 1) : 0) != grp) continue;  // the other group's tile
                    if (!do_tile(n, ti)) {
                        ok = false;
                        break;
                    }
                }
            }
            // After an abort every warp still runs every barrier of every piece (its waits fail fast).
            const bool whole = w.n_parts == 1;
            named_barrier(1, kEpiThreads);
            if (K > 0 && grp == 0) {
                // merge the two groups' lists of each row (disjoint block sets)
                const int ja = e * 32 + lane, jb = ja + 8 * 32;
                const size_t o = (((size_t)b * a.T + t) * a.G + g) * a.k;
                const size_t po = ((size_t)w.u * a.n_seg + w.s) * K * kUnitRows + rl;
                int ia = 0, ib = 0;
                const int n_out = whole ? a.k : K;
                for (int i = 0; ok && i < n_out; ++i) {
                    const float sa = list_s[ia * kEpiThreads + ja], sb = list_s[ib * kEpiThreads + jb];
                    const int da = list_i[ia * kEpiThreads + ja], db = list_i[ib * kEpiThreads + jb];
                    const bool take_a = ib >= K || (ia < K && better(sa, da, sb, db));
                    const float sv = take_a ? sa : sb;
                    const int dv = take_a ? da : db;
                    if (take_a) ++ia; else ++ib;
                    if (whole) {
                        if (t < a.T) {
                            a.ids_out[o + i] = sv > -INFINITY ? dv : -1;
                            if (a.top_scores_out != nullptr) a.top_scores_out[o + i] = sv;
                        }
                    } else {
                        a.part_s[po + (size_t)i * kUnitRows] = sv;
                        a.part_i[po + (size_t)i * kUnitRows] = dv;
                    }
                }
                if (!whole) {
                    // the CTA that finishes the unit's last segment merges every segment's lists
                    __threadfence();
                    named_barrier(2, kEpiThreads / 2);
                    if (e == 0 && lane == 0) S.merge_here = ok && atomicAdd(&a.counters[w.u], 1) == w.n_parts - 1;
                    named_barrier(2, kEpiThreads / 2);
                    if (S.merge_here) {
                        __threadfence();
                        top.reset();
                        for (int sg = 0; sg < w.n_parts; ++sg) {
                            const size_t q = ((size_t)w.u * a.n_seg + sg) * K * kUnitRows + rl;
                            for (int i = 0; i < K; ++i) {
                                const float cs = __ldcg(a.part_s + q + (size_t)i * kUnitRows);
                                const int ci = __ldcg(a.part_i + q + (size_t)i * kUnitRows);
                                if (!better(cs, ci, top.thr_s, top.thr_i)) break;  // the rest of this list is worse
                                top.insert(cs, ci);
                            }
                        }
                        if (t < a.T) {
                            for (int i = 0; i < a.k; ++i) {
                                const float sv = list_s[i * kEpiThreads + ja];
                                a.ids_out[o + i] = sv > -INFINITY ? list_i[i * kEpiThreads + ja] : -1;
                                if (a.top_scores_out != nullptr) a.top_scores_out[o + i] = sv;
                            }
                        }
                    }
                }
            }
            named_barrier(1, kEpiThreads);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

template <int K, int BK>
cudaError_t launch_k(const PrefillIdxArgs &a, const CUtensorMap &qm, const CUtensorMap &km, int grid,
                     cudaStream_t s) {
    const size_t smem = 1024 + kAccs * kABytes + PiShape<K>::S * kTileBytes + (size_t)K * kEpiThreads * 8 +
                        stage_bytes<K>() + sizeof(Smem) + 64;
    static bool attr = false;
    if (!attr) {
        cudaError_t e =
            cudaFuncSetAttribute(prefill_index_kernel<K, BK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    prefill_index_kernel<K, BK><<<grid, kThreads, smem, s>>>(qm, km, a);
    return cudaGetLastError();
}

template <int K>
cudaError_t launch_kb(const PrefillIdxArgs &a, const CUtensorMap &qm, const CUtensorMap &km, int grid, cudaStream_t s) {
    switch (a.Bk) {
        case 32: return launch_k<K, 32>(a, qm, km, grid, s);
        case 64: return launch_k<K, 64>(a, qm, km, grid, s);
        case 128: return launch_k<K, 128>(a, qm, km, grid, s);
        case 256: return launch_k<K, 256>(a, qm, km, grid, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_prefill_index(const PrefillIdxArgs &a, const void *q_idx, const void *k_idx, int n_sm,
                                 cudaStream_t s, const char **why) {
    CUtensorMap qm, km;
    // q_idx [B*T, G, 64] bf16: box of 64 dims x 1 group x 128 rows
    const unsigned long long qdim[3] = {64, (unsigned long long)a.G, (unsigned long long)a.B * a.T};
    const unsigned long long qstr[2] = {64 * 2, (unsigned long long)a.G * 64 * 2};
    const unsigned qbox[3] = {64, 1, kRows};
    if (!encode_3d(&qm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void *>(q_idx), qdim, qstr, qbox,
                   CU_TENSOR_MAP_SWIZZLE_128B)) {
        *why = "encoding the index-query tensor map failed";
        return cudaErrorInvalidValue;
    }
    // k_idx [B*Hik*Lmax, 64] bf16: box of 64 dims x 128 keys
    if (!encode_2d(&km, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void *>(k_idx), 64,
                   a.cache.rows(a.B, a.Hik, a.L_max), 128, 64, kKeys, CU_TENSOR_MAP_SWIZZLE_128B)) {
        *why = "encoding the index-key tensor map failed";
        return cudaErrorInvalidValue;
    }
    const int grid = n_sm;  // the plan's CTA count (at most one per SM)
    *why = "prefill index kernel launch";
    if (a.blk_scores != nullptr) return launch_kb<0>(a, qm, km, grid, s);
    return a.k <= 8 ? launch_kb<8>(a, qm, km, grid, s) : a.k <= 16 ? launch_kb<16>(a, qm, km, grid, s)
                                                             : launch_kb<32>(a, qm, km, grid, s);
}

}  // namespace msa
