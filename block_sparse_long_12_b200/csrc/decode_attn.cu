// Step 2 of MSA for decode: exact softmax attention over the selected blocks.
//
// Page "MiniMax wird duenn" (atlascloud.ai), section 1, Step 2: every query
// head of a GQA group uses the group's single TopK list (Q1/Q2/Q3 -> I1,
// Q4/Q5/Q6 -> I2) and attends over only those blocks of the full, real K/V
// cache, so one group loads one set of KV blocks for all its heads.
//
// Grid (split s, group g, sequence b); split s owns list positions
// [s * blocks_per_split, ...).  In the fused decode step a CTA first finishes
// Step 1 for its group (select_group_topk: the scan's per-piece sorted
// candidate lists are staged in shared memory and the k best kept).  Then it
// streams its blocks' K/V tiles through a TMA ring and keeps an online
// softmax for all r heads of the group.  Each split writes a normalised
// partial output and its log2 normaliser; the last split of a group to
// finish (atomic arrival count) merges them by log-sum-exp.  With MSA_DENSE
// the splits cover every visible block: plain GQA decode.
//
// bf16: decode_attn_mma_kernel runs both products on mma.sync tensor-core
// fragments (the r <= 16 heads padded to 16 rows), K/V tiles in the 128-byte
// swizzle layout written by TMA tensor copies; splits of many tiles (large k,
// MSA_DENSE) take decode_attn_wide_kernel, whose warps run their own tiles
// without barriers.  fp32: decode_attn_kernel on CUDA cores (exact fp32
// products).
#include "tcgen05.cuh"

namespace msa {

namespace {

template <typename T, int N>
__device__ inline void load_row(const T *p, float (&f)[N]) {
    constexpr int BYTES = N * (int)sizeof(T);
    if constexpr (BYTES == 16) {
        const uint4 u = *reinterpret_cast<const uint4 *>(p);
        if constexpr (sizeof(T) == 4) {
            f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
            f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
        } else {
            float g[8];
            Vec16<__nv_bfloat16>::unpack(u, g);
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = g[i];
        }
    } else if constexpr (BYTES == 8) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        if constexpr (sizeof(T) == 4) {
            f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        } else {
            f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
            f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
        }
    } else if constexpr (BYTES == 4) {
        const uint32_t u = *reinterpret_cast<const uint32_t *>(p);
        if constexpr (sizeof(T) == 4) {
            f[0] = __uint_as_float(u);
        } else {
            f[0] = __uint_as_float(u << 16); f[1] = __uint_as_float(u & 0xffff0000u);
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i) f[i] = load_elem(p + i);
    }
}

// Sum over the 32 lanes of x[0..R) such that every lane ends with the total
// of one head; returns it and sets `head`.  Lanes (lane & (32/R - 1)) == 0
// hold distinct heads.
template <int R>
__device__ inline float reduce_scatter(float (&x)[R], int lane, int &head) {
    head = 0;
#pragma unroll
    for (int lvl = 0; lvl < 5; ++lvl) {
        const int o = 16 >> lvl;
        const int cnt = R >> lvl;
        const bool upper = (lane & o) != 0;
        if (cnt >= 2) {
            const int half = cnt / 2;
#pragma unroll
            for (int i = 0; i < half; ++i) {
                const float send = upper ? x[i] : x[i + half];
                const float keep = upper ? x[i + half] : x[i];
                x[i] = keep + __shfl_xor_sync(FULL, send, o);
            }
            if (upper) head += half;
        } else {
            x[0] += __shfl_xor_sync(FULL, x[0], o);
        }
    }
    return x[0];
}


// Descending bitonic sort of 64 keys held by one warp, element lane + 32 * j
// in v[j]; the element of rank r ends in lane r % 32, v[r / 32].
__device__ inline void warp_sort64_desc(unsigned long long (&v)[2], int lane) {
#pragma unroll
    for (int size = 2; size <= 64; size <<= 1)
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            if (stride == 32) {
                if (v[0] < v[1]) {  // size 64: one descending run
                    const unsigned long long t = v[0];
                    v[0] = v[1];
                    v[1] = t;
                }
            } else {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int idx = lane + 32 * j;
                    const unsigned long long o = __shfl_xor_sync(FULL, v[j], stride);
                    const bool keep_max = ((idx & stride) == 0) == ((idx & size) == 0);
                    v[j] = keep_max ? (v[j] > o ? v[j] : o) : (v[j] < o ? v[j] : o);
                }
            }
        }
}

constexpr int kSortCap = 512;  // survivors sorted at once; more go the counting way

// The scan's pieces of segment (b, hik): which CTA's list comes first and how
// many CTAs hold one.  The same split the scan makes (equal ranges over the
// streams' first nb - scan_tail_blocks(nb) blocks), recomputed from seq_lens
// so that it is known before the scan has finished.  Called by every thread.
__device__ SegInfo seg_pieces(const AttnArgs &a, int b, int hik) {
    __shared__ long long red[2][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    long long tot = 0, pre = 0;
    for (int bb = threadIdx.x; bb < a.B; bb += blockDim.x) {
        int L = a.seq_lens[bb];
        L = L < 0 ? 0 : (L > a.L_max ? a.L_max : L);
        const int nb = (L + a.Bk - 1) / a.Bk;
        const long long na = (long long)(nb - scan_tail_blocks(nb)) * a.Hik;
        tot += na;
        if (bb < b) pre += na;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        tot += __shfl_xor_sync(FULL, tot, o);
        pre += __shfl_xor_sync(FULL, pre, o);
    }
    if (lane == 0) {
        red[0][warp] = tot;
        red[1][warp] = pre;
    }
    __syncthreads();
    tot = 0;
    pre = 0;
    for (int w2 = 0; w2 < nwarps; ++w2) {
        tot += red[0][w2];
        pre += red[1][w2];
    }
    int L = a.seq_lens[b];
    L = L < 0 ? 0 : (L > a.L_max ? a.L_max : L);
    const int nb = (L + a.Bk - 1) / a.Bk, nba = nb - scan_tail_blocks(nb);
    __syncthreads();  // red is free again
    SegInfo si{-1, 0};
    const long long per = tot > 0 ? (tot + a.n_cta - 1) / a.n_cta : 1;
    if (nba > 0) {
        const long long st = pre + (long long)hik * nba;
        si.first_cta = (int)(st / per);
        si.n_pieces = (int)((st + nba - 1) / per) - si.first_cta + 1;
    }
    return si;
}

// Final TopK of group g of sequence b (the fused decode step) from the scan's
// per-piece sorted lists and the block scores of the stream's tail.  The
// lists are staged in `scratch` (select_scratch_bytes) by the whole CTA.  The
// k-th best of a subset of the candidates (the first entries of some lists)
// is a floor that the final k all reach: the list entries and tail blocks at
// or above it are sorted as 64-bit keys and the first k kept.  If too many
// reach the floor, counting ranks take over.  Leaves the list in sel_s /
// sel_i[0..32), padded with (-inf, -1).  Called by every thread of the CTA.
__device__ void select_group_topk(const AttnArgs &a, int b, int g, const SegInfo info, unsigned char *scratch,
                                  float *sel_s, int *sel_i) {
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int cap = a.n_cta * a.k;
    // scratch: lists [cap] scores | [cap] ids | 32 state words | one region for the survivors
    // (sort keys, or scores and ids) and for the tail merge's lists
    float *ls = reinterpret_cast<float *>(scratch);
    int *li = reinterpret_cast<int *>(ls + cap);
    int *st = li + cap;  // [0] survivors, [1] threshold id, [2] threshold score (bits), [4..] per-warp floors
    float *ss = reinterpret_cast<float *>(st + 32);
    int *si = reinterpret_cast<int *>(ss + cap);
    const int gps = a.G / a.Hik;
    const int seg = b * a.Hik + g % a.Hik, gl = g / a.Hik;
    // the first batch of the tail's block scores (merged at the end) is loaded now, so that its
    // latency overlaps the work on the ranges' lists
    constexpr int kBatch = 16;  // loads in flight per lane
    const int lane = tid & 31, warp = tid >> 5, nwarps = nthr >> 5;
    int L = a.seq_lens[b];
    L = L < 0 ? 0 : (L > a.L_max ? a.L_max : L);
    const int nb = (L + a.Bk - 1) / a.Bk, nt = a.tail_scores != nullptr ? scan_tail_blocks(nb) : 0;
    const float *tsc = a.tail_scores + ((size_t)b * a.G + g) * ((a.L_max + a.Bk - 1) / a.Bk);
    const int base0 = nb - nt + warp * 32 * kBatch;
    float v0[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
        const int n = base0 + u * 32 + lane;
        v0[u] = n < nb ? tsc[n] : -INFINITY;
    }
    // the pieces' lists into shared memory, kLists loads in flight per thread and array
    constexpr int kLists = 8;
    const int k = a.k, np = info.n_pieces, n = np * k;
    for (int i0 = tid; i0 < n; i0 += nthr * kLists) {
        float sv[kLists];
        int iv[kLists];
#pragma unroll
        for (int u = 0; u < kLists; ++u) {
            const int i = i0 + u * nthr;
            if (i < n) {
                const size_t src = (((size_t)seg * a.n_cta + i / k) * gps + gl) * k + i % k;
                sv[u] = a.cand_s[src];
                iv[u] = a.cand_i[src];
            }
        }
#pragma unroll
        for (int u = 0; u < kLists; ++u) {
            const int i = i0 + u * nthr;
            if (i < n) {
                ls[i] = sv[u];
                li[i] = iv[u];
            }
        }
    }
    if (tid == 0) {
        st[0] = 0;
        st[1] = -1;
        st[2] = __float_as_int(-INFINITY);
    }
    if (tid < 32) {
        sel_s[tid] = -INFINITY;
        sel_i[tid] = -1;
    }
    __syncthreads();
    {
        // floor: the k-th best of the first J entries of up to 64 / J lists, sorted by one warp;
        // the k-th best of any subset is no better than the k-th best of all candidates
        if (warp == 0) {
            const int J = np > 0 ? min(k, max(1, (2 * k + np - 1) / np)) : 1;
            const int nl = min(np, 64 / J);
            unsigned long long v[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int e = lane + 32 * j, l = e / J, pos = e - l * J;
                v[j] = 0ull;
                if (l < nl && li[l * k + pos] >= 0) v[j] = sel_key(ls[l * k + pos], li[l * k + pos]);
            }
            warp_sort64_desc(v, lane);
            const unsigned long long kth = __shfl_sync(FULL, (k - 1) < 32 ? v[0] : v[1], (k - 1) & 31);
            if (lane == 0) {
                st[4] = (int)(uint32_t)kth;
                st[5] = (int)(uint32_t)(kth >> 32);
            }
        }
        __syncthreads();
        // 0 (fewer than k entries in the subset): no floor
        const unsigned long long fk = ((unsigned long long)(uint32_t)st[5] << 32) | (uint32_t)st[4];
        // survivors: list prefixes and tail blocks at or above the floor, as sort keys
        unsigned long long *keys = reinterpret_cast<unsigned long long *>(ss);  // [max(cap, kSortCap)]
        const int key_cap = cap > kSortCap ? cap : kSortCap;
        for (int l = tid; l < np; l += nthr)
            for (int j = 0; j < k; ++j) {
                const int id = li[l * k + j];
                if (id < 0) break;
                const unsigned long long key = sel_key(ls[l * k + j], id);
                if (key < fk) break;
                const int at = atomicAdd(&st[0], 1);
                if (at < key_cap) keys[at] = key;
            }
        for (int base = base0; base < nb; base += nwarps * 32 * kBatch) {
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int n = base + u * 32 + lane;
                const float v = base == base0 ? v0[u] : (n < nb ? tsc[n] : -INFINITY);
                const unsigned long long key = sel_key(v, n);
                if (n < nb && key >= fk) {
                    const int at = atomicAdd(&st[0], 1);
                    if (at < key_cap) keys[at] = key;
                }
            }
        }
        __syncthreads();
        const int m = st[0];
        if (m <= 64) {
            // one warp sorts them in registers
            if (warp == 0) {
                unsigned long long v[2];
#pragma unroll
                for (int j = 0; j < 2; ++j) v[j] = lane + 32 * j < m ? keys[lane + 32 * j] : 0ull;
                warp_sort64_desc(v, lane);
                if (lane < k && lane < m) sel_unkey(v[0], sel_s[lane], sel_i[lane]);
            }
            __syncthreads();
            return;
        }
        if (m <= kSortCap) {
            int P = 32;
            while (P < m) P <<= 1;
            for (int i = m + tid; i < P; i += nthr) keys[i] = 0ull;  // below every real key
            __syncthreads();
            block_sort_desc(keys, P);
            if (tid < k && tid < m) sel_unkey(keys[tid], sel_s[tid], sel_i[tid]);
            __syncthreads();
            return;
        }
        // too many at the floor: the counting way below (its state starts afresh)
        if (tid == 0) st[0] = 0;
        __syncthreads();
    }
    // Threshold: the k-th best among the first J entries of every piece.  The k-th best of any
    // subset is no better than the k-th best of all candidates, so the whole top-k passes it;
    // taking each piece's head makes it tight, and few candidates survive.
    const int J = np > 0 ? min(k, 2 * ((k + np - 1) / np)) : 0;
    for (int t = tid; t < np * J; t += nthr) {
        const int e = (t / J) * k + t % J;
        const float s = ls[e];
        const int id = li[e];
        if (id < 0) continue;
        int rank = 0;
        for (int pc = 0; pc < np; ++pc)
            for (int j = 0; j < J; ++j) {
                const int f = pc * k + j;
                rank += (li[f] >= 0 && better(ls[f], li[f], s, id)) ? 1 : 0;
            }
        if (rank == k - 1) {
            st[1] = id;
            st[2] = __float_as_int(s);
        }
    }
    __syncthreads();
    // survivors: candidates at least as good as the threshold (all valid ones when the subset
    // holds fewer than k), then their exact ranks (ids are unique, so ranks are distinct)
    const float ts = __int_as_float(st[2]);
    const int ti = st[1];
    for (int i = tid; i < n; i += nthr) {
        if (li[i] >= 0 && !better(ts, ti, ls[i], li[i])) {
            const int at = atomicAdd(&st[0], 1);
            ss[at] = ls[i];
            si[at] = li[i];
        }
    }
    __syncthreads();
    const int m = st[0];
    for (int i = tid; i < m; i += nthr) {
        const float s = ss[i];
        const int id = si[i];
        int rank = 0;
        for (int j = 0; j < m; ++j) rank += better(ss[j], si[j], s, id) ? 1 : 0;
        if (rank < k) {
            sel_s[rank] = s;
            sel_i[rank] = id;
        }
    }
    __syncthreads();
    if (a.tail_scores == nullptr) return;
    // The tail of the stream (blocks [nb - nt, nb)) left block scores only: every warp keeps
    // the k best of its share of those that beat the k-th entry so far (the others cost one
    // comparison), and one warp merges these lists with the ranges' k best.
    WarpTopK t;
    t.reset();
    // floor: a tail block must beat the k-th entry of the ranges' list (while the warp's own
    // list is not full its threshold is below that)
    const float fl_s = sel_s[k - 1];
    const int fl_i = sel_i[k - 1];
    for (int base = base0; base < nb; base += nwarps * 32 * kBatch) {
        float v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int n = base + u * 32 + lane;
            v[u] = base == base0 ? v0[u] : (n < nb ? tsc[n] : -INFINITY);
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int n0 = base + u * 32;
            unsigned msk = __ballot_sync(FULL, n0 + lane < nb && better(v[u], n0 + lane, fl_s, fl_i) &&
                                                   better(v[u], n0 + lane, t.thr_s, t.thr_i));
            while (msk) {
                const int l = __ffs(msk) - 1;
                msk &= msk - 1;
                t.insert(__shfl_sync(FULL, v[u], l), n0 + l, k, lane);
            }
        }
    }
    float *tl_s = ss;  // [1 + nwarps][32] lists (the survivors are ranked by now)
    int *tl_i = reinterpret_cast<int *>(tl_s + 9 * 32);
    tl_s[(1 + warp) * 32 + lane] = t.s;
    tl_i[(1 + warp) * 32 + lane] = t.id;
    if (warp == 0) {
        tl_s[lane] = sel_s[lane];
        tl_i[lane] = sel_i[lane];
    }
    __syncthreads();
    if (warp == 0) warp_merge_sorted_lists<1>(tl_s, tl_i, 1 + nwarps, k, 32, k, sel_s, sel_i, lane);
    __syncthreads();
}

// Descending bitonic sort of 32 keys held one per lane.
__device__ inline unsigned long long warp_sort32_desc(unsigned long long v, int lane) {
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const unsigned long long o = __shfl_xor_sync(FULL, v, stride);
            const bool keep_max = ((lane & stride) == 0) == ((lane & size) == 0);
            v = keep_max ? (v > o ? v : o) : (v < o ? v : o);
        }
    return v;
}

// Final TopK of group g of sequence b from the block scores of every block of
// its stream.  Groups that share one index-K stream take this way: the scan
// keeps no per-piece lists for them (every CTA of the scan would hold a piece
// of the one stream) and leaves every block's score.  The scores are staged
// in shared memory by one bulk copy (chunks of what the scratch holds), so
// that both passes read shared memory: every thread's best block of its
// share (blocks tid, tid + nthr, ...) is one of the candidates, so the k-th
// best of the threads' bests is a floor that the final k all reach; the
// second pass gathers the blocks at or above it and one warp (or the CTA)
// sorts them.  If more than kSortCap reach the floor, every warp keeps the k
// best of its share that do and one warp merges the warps' lists.  Leaves the
// list in sel_s / sel_i[0..32), padded with (-inf, -1).  Called by every
// thread of the CTA.
constexpr int kScoreStageOff = 12352;  // scratch bytes before the staged scores (16-byte aligned)
// Every thread's shared-memory writes before the tensor copies (async proxy) that reuse the
// scratch for K/V tiles, then a CTA barrier.
__device__ inline void fence_scratch_for_tma() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
}
__device__ void select_from_scores(const AttnArgs &a, int b, int g, unsigned char *scratch, float *sel_s, int *sel_i) {
    const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5, nwarps = nthr >> 5;
    const int k = a.k;
    int L = a.seq_lens[b];
    L = L < 0 ? 0 : (L > a.L_max ? a.L_max : L);
    const int nb = (L + a.Bk - 1) / a.Bk;
    const float *tsc = a.tail_scores + ((size_t)b * a.G + g) * ((a.L_max + a.Bk - 1) / a.Bk);
    // scratch: survivors [kSortCap] | the warps' sorted bests [nwarps][32] | floor | barrier | count | staged scores
    unsigned long long *keys = reinterpret_cast<unsigned long long *>(scratch);
    unsigned long long *wl = keys + kSortCap;
    unsigned long long *floor_key = wl + nwarps * 32;
    uint64_t *bar = reinterpret_cast<uint64_t *>(floor_key + 1);
    int *cnt = reinterpret_cast<int *>(bar + 1);
    float *stage = reinterpret_cast<float *>(scratch + kScoreStageOff);
    // floats per chunk (a multiple of 4, 3 spare for the alignment shift)
    const int cap = ((a.ring_bytes - kScoreStageOff) / 4 - 3) / 4 * 4;
    // the bulk copy starts at the first 16-byte aligned score; the h scores before it and the
    // ragged end are loaded by the threads; score i of a chunk sits at stage[i + sh]
    const int h = (int)(((16u - ((uint32_t)reinterpret_cast<uintptr_t>(tsc) & 15u)) & 15u) >> 2);
    const int sh = (4 - h) & 3;
    if (tid == 0) {
        *cnt = 0;
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    if (tid < 32) {
        sel_s[tid] = -INFINITY;
        sel_i[tid] = -1;
    }
    __syncthreads();
    uint32_t phase = 0;
    auto stage_chunk = [&](int c0, int cn) {
        const int hh = h < cn ? h : cn;
        const int body = (cn - hh) / 4 * 4;
        if (tid == 0 && body > 0) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // earlier reads of the stage first
            mbar_arrive_expect_tx(bar, (uint32_t)body * 4);
            bulk_g2s(stage + hh + sh, tsc + c0 + hh, (uint32_t)body * 4, bar, l2_evict_normal_policy());
        }
        for (int i = tid; i < cn; i += nthr)
            if (i < hh || i >= hh + body) stage[i + sh] = tsc[c0 + i];
        if (body > 0) {
            mbar_wait(bar, phase, a.status);
            phase ^= 1u;
        }
        __syncthreads();
    };
    unsigned long long best = 0ull;  // below every real key
    for (int c0 = 0; c0 < nb; c0 += cap) {
        const int cn = nb - c0 < cap ? nb - c0 : cap;
        stage_chunk(c0, cn);
        for (int i = tid; i < cn; i += nthr) {
            const unsigned long long key = sel_key(stage[i + sh], c0 + i);
            best = key > best ? key : best;
        }
        if (c0 + cap < nb) __syncthreads();  // the next chunk overwrites the stage
    }
    wl[warp * 32 + lane] = warp_sort32_desc(best, lane);
    __syncthreads();
    if (warp == 0) {
        unsigned long long t = wl[lane];
        for (int w2 = 1; w2 < nwarps; ++w2) t = warp_merge_top32(t, wl[w2 * 32 + lane], lane);
        // 0 when fewer than k threads hold a block (nb < k): every block survives
        const unsigned long long fk = __shfl_sync(FULL, t, k - 1);
        if (lane == 0) *floor_key = fk;
    }
    __syncthreads();
    const unsigned long long fk = *floor_key;
    for (int c0 = 0; c0 < nb; c0 += cap) {
        const int cn = nb - c0 < cap ? nb - c0 : cap;
        if (nb > cap) stage_chunk(c0, cn);  // one chunk: its scores are still staged
        for (int i0 = 0; i0 < cn; i0 += nthr) {
            const int i = i0 + tid;
            const unsigned long long key = i < cn ? sel_key(stage[i + sh], c0 + i) : 0ull;
            const bool keep = i < cn && key >= fk;
            const unsigned msk = __ballot_sync(FULL, keep);
            if (msk != 0u) {
                int at = 0;
                if (lane == 0) at = atomicAdd(cnt, __popc(msk));
                at = __shfl_sync(FULL, at, 0) + __popc(msk & ((1u << lane) - 1u));
                if (keep && at < kSortCap) keys[at] = key;
            }
        }
        __syncthreads();
    }
    if (tid == 0) asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
    const int m = *cnt;
    if (m <= 64) {
        if (warp == 0) {
            unsigned long long v[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) v[j] = lane + 32 * j < m ? keys[lane + 32 * j] : 0ull;
            warp_sort64_desc(v, lane);
            if (lane < k && lane < m) sel_unkey(v[0], sel_s[lane], sel_i[lane]);
        }
        fence_scratch_for_tma();
        return;
    }
    if (m <= kSortCap) {
        int P = 128;
        while (P < m) P <<= 1;
        for (int i = m + tid; i < P; i += nthr) keys[i] = 0ull;
        __syncthreads();
        block_sort_desc(keys, P);
        if (tid < k) sel_unkey(keys[tid], sel_s[tid], sel_i[tid]);
        fence_scratch_for_tma();
        return;
    }
    // many blocks at the floor: the k best of each warp's share that reach it, then one merge
    WarpTopK t;
    t.reset();
    for (int base = warp * 32; base < nb; base += nwarps * 32) {
        const int n = base + lane;
        const float v = n < nb ? tsc[n] : -INFINITY;
        unsigned msk = __ballot_sync(FULL, n < nb && sel_key(v, n) >= fk && better(v, n, t.thr_s, t.thr_i));
        while (msk) {
            const int l = __ffs(msk) - 1;
            msk &= msk - 1;
            t.insert(__shfl_sync(FULL, v, l), base + l, k, lane);
        }
    }
    __syncthreads();  // every thread is done with the survivors' keys
    float *tl_s = reinterpret_cast<float *>(keys);  // [nwarps][32]
    int *tl_i = reinterpret_cast<int *>(tl_s + nwarps * 32);
    tl_s[warp * 32 + lane] = t.s;
    tl_i[warp * 32 + lane] = t.id;
    __syncthreads();
    if (warp == 0) warp_merge_sorted_lists<1>(tl_s, tl_i, nwarps, k, 32, k, sel_s, sel_i, lane);
    fence_scratch_for_tma();
}

// Scratch bytes the selection needs: select_group_topk's lists of n_cta pieces of k entries and
// its survivors, or select_from_scores' survivors and per-warp lists.
__host__ __device__ inline size_t select_scratch_bytes(int n_cta, int k) {
    const size_t cap = (size_t)n_cta * k;
    const size_t lists = cap * 8 + 32 * 4 + (cap > (size_t)kSortCap ? cap : (size_t)kSortCap) * 8;
    const size_t scores = (size_t)kScoreStageOff + 16384;  // chunks of 4,096 scores at least
    return lists > scores ? lists : scores;
}

// The last split CTA of (b, g) merges the normalised partial outputs of all
// splits by log-sum-exp (weights staged in `wgt`, S * r floats).
template <typename T>
__device__ void merge_splits(const AttnArgs &a, int b, int g, float *wgt) {
    const int tid = threadIdx.x, nthr = blockDim.x, r = a.r, D = a.D;
    const size_t bg = (size_t)b * a.G + g;
    __threadfence();
    for (int i = tid; i < a.S * r; i += nthr) wgt[i] = __ldcg(a.part_lse + bg * a.S * r + i);
    __syncthreads();
    if (tid < r) {
        float M = -INFINITY;
        for (int j = 0; j < a.S; ++j) M = fmaxf(M, wgt[j * r + tid]);
        float den = 0.f;
        for (int j = 0; j < a.S; ++j) {
            const float e = M > -INFINITY ? exp2f(wgt[j * r + tid] - M) : 0.f;
            wgt[j * r + tid] = e;
            den += e;
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
        for (int j = 0; j < a.S; ++j) wgt[j * r + tid] *= inv;
        if (a.lse != nullptr)
            a.lse[(size_t)b * a.Hq + (size_t)g * r + tid] =
                den > 0.f ? (M + log2f(den)) * 0.69314718055994531f : -INFINITY;
    }
    __syncthreads();
    // every thread owns up to 4 float4 groups of outputs and keeps 4 splits x 4 groups of loads in
    // flight, so the merge costs a few L2 round trips rather than one per split
    T *o = reinterpret_cast<T *>(a.o) + ((size_t)b * a.Hq + (size_t)g * r) * D;
    const float4 *po = reinterpret_cast<const float4 *>(a.part_o + bg * a.S * r * D);
    const int n4 = r * D / 4, split4 = r * D / 4;
    for (int f0 = tid; f0 < n4; f0 += 4 * nthr) {
        float4 acc[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j0 = 0; j0 < a.S; j0 += 4) {
            float4 v[4][4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int f = f0 + u * nthr;
                    v[jj][u] = (j0 + jj < a.S && f < n4) ? __ldcg(po + (size_t)(j0 + jj) * split4 + f)
                                                         : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int f = f0 + u * nthr;
                    if (j0 + jj < a.S && f < n4) {
                        const float wj = wgt[(j0 + jj) * r + (f * 4) / D];
                        acc[u].x = fmaf(wj, v[jj][u].x, acc[u].x);
                        acc[u].y = fmaf(wj, v[jj][u].y, acc[u].y);
                        acc[u].z = fmaf(wj, v[jj][u].z, acc[u].z);
                        acc[u].w = fmaf(wj, v[jj][u].w, acc[u].w);
                    }
                }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int f = f0 + u * nthr;
            if (f < n4) {
                store_elem(o + 4 * f, acc[u].x);
                store_elem(o + 4 * f + 1, acc[u].y);
                store_elem(o + 4 * f + 2, acc[u].z);
                store_elem(o + 4 * f + 3, acc[u].w);
            }
        }
    }
    if (tid == 0) a.counters[bg] = 0;  // ready for the next call
}

// True in every thread of the CTA that finished last among the S splits of (b, g).
__device__ inline bool last_split(const AttnArgs &a, int b, int g, int *flag) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) *flag = (atomicAdd(&a.counters[(size_t)b * a.G + g], 1) == a.S - 1) ? 1 : 0;
    __syncthreads();
    return *flag != 0;
}

// Obtain the group's list: fused selection from the scan, or a given ids tensor.
// MSA_FORCE_SINK_LOCAL applied to a finished selection: block 0 and the sequence's last block
// first (by id, score +inf), then the list's other blocks in their order.  The list holds the k
// best of all blocks, so its other blocks, in order, are the best of the others.  Called by
// every thread of the CTA; sel_s / sel_i stay padded with (-inf, -1).
__device__ inline void force_sink_local(const AttnArgs &a, int b, float *sel_s, int *sel_i) {
    int L = a.seq_lens[b];
    L = L < 0 ? 0 : (L > a.L_max ? a.L_max : L);
    const int nb = (L + a.Bk - 1) / a.Bk, nf = nb < 2 ? nb : 2, k = a.k;
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const float s = sel_s[lane];
        const int id = sel_i[lane];
        const bool keep = lane < k && id >= 0 && id != 0 && id != nb - 1;
        const unsigned m = __ballot_sync(FULL, keep);
        const int dst = nf + __popc(m & ((1u << lane) - 1u));
        const int n_keep = __popc(m);
        __syncwarp();
        if (keep && dst < k) {
            sel_s[dst] = s;
            sel_i[dst] = id;
        }
        if (lane < nf && lane < k) {
            sel_s[lane] = INFINITY;
            sel_i[lane] = lane == 0 ? 0 : nb - 1;
        }
        if (lane >= nf + n_keep || lane >= k) {
            sel_s[lane] = -INFINITY;
            sel_i[lane] = -1;
        }
    }
    __syncthreads();
}

// SO: the stream's groups share one index-K head (a.scores_only): the selection reads every
// block's score instead of the scan's per-piece lists
template <bool SO>
__device__ inline void group_list(const AttnArgs &a, int b, int g, const SegInfo info, unsigned char *scratch,
                                  float *sel_s, int *sel_i) {
    if (a.dense) return;
    if (a.cand_s != nullptr) {
        if constexpr (SO)
            select_from_scores(a, b, g, scratch, sel_s, sel_i);
        else
            select_group_topk(a, b, g, info, scratch, sel_s, sel_i);
        if (a.force) force_sink_local(a, b, sel_s, sel_i);
        if (blockIdx.x == 0 && threadIdx.x < a.k) {
            const size_t o = ((size_t)b * a.G + g) * a.k + threadIdx.x;
            if (a.ids_out != nullptr) a.ids_out[o] = sel_i[threadIdx.x];
            if (a.top_scores_out != nullptr) a.top_scores_out[o] = sel_s[threadIdx.x];
        }
    } else {
        if (threadIdx.x < a.k && a.k <= kMaxTopKList)
            sel_i[threadIdx.x] = a.ids_in[((size_t)b * a.G + g) * a.k + threadIdx.x];
        __syncthreads();
    }
}

template <typename T, int D, int R>
struct AttnCfg {
    static constexpr int ES = (int)sizeof(T);
    static constexpr int KT_MAX = (65536 / (2 * D * ES)) > 256 ? 256 : (65536 / (2 * D * ES)); // keys per tile
    static constexpr int DPL = D / 32;                                  // dims per lane (scores)
    static constexpr int DPT = (R * D / kAttnThreads) > 0 ? (R * D / kAttnThreads) : 1; // dims per thread (P.V)
    static constexpr int NST = 2;
};

template <typename T, int D, int R>
__global__ void __launch_bounds__(kAttnThreads) decode_attn_kernel(const AttnArgs a) {
    using Cfg = AttnCfg<T, D, R>;
    constexpr int ES = Cfg::ES, DPL = Cfg::DPL, DPT = Cfg::DPT, NST = Cfg::NST;
    const int KT = a.Bk < Cfg::KT_MAX ? a.Bk : Cfg::KT_MAX;
    const size_t tile_bytes = (size_t)KT * D * ES;

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *ring = smem;  // [NST][K tile | V tile]; also the selection scratch
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring + a.ring_bytes);  // [NST]
    float *sel_s = reinterpret_cast<float *>(bars + NST);                   // [32]
    int *sel_i = reinterpret_cast<int *>(sel_s + 32);                       // [32]
    float *m_s = reinterpret_cast<float *>(sel_i + 32);                     // running max (log2 domain)
    float *l_s = m_s + R;                                                   // running sum
    float *al_s = l_s + R;                                                  // rescale of this tile
    float *p_s = al_s + R;                                                  // [R][KT]

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int r = a.r;

    if (tid < NST) mbar_init(&bars[tid], 1);
    if (tid < R) { m_s[tid] = -INFINITY; l_s[tid] = 0.f; }
    fence_mbar_init();

    // query slice of every head of the group (input, independent of the scan)
    float qreg[R][DPL];
    {
        const T *qg = reinterpret_cast<const T *>(a.q) + ((size_t)b * a.Hq + (size_t)g * r) * D + lane * DPL;
#pragma unroll
        for (int h = 0; h < R; ++h) {
            if (h < r) {
                load_row<T, DPL>(qg + (size_t)h * D, qreg[h]);
            } else {
#pragma unroll
                for (int d = 0; d < DPL; ++d) qreg[h][d] = 0.f;
            }
        }
    }
    int L = a.seq_lens[b];
    L = L < 0 ? 0 : (L > a.L_max ? a.L_max : L);
    const int pos = L - 1;
    const int nb = (L + a.Bk - 1) / a.Bk;

    // where the scan leaves this group's lists is known from seq_lens alone
    const SegInfo info = (!a.dense && a.cand_s != nullptr) ? seg_pieces(a, b, g % a.Hik) : SegInfo{-1, 0};
    pdl_wait_prior_grid();  // the scan's candidates are complete from here on
    pdl_allow_next_grid();
    __shared__ int last_flag;
    group_list<false>(a, b, g, info, ring, sel_s, sel_i);

    // this split's blocks: list positions [j0, j1)
    const int bps = a.blocks_per_split;
    const int j0 = s * bps;
    int j1 = j0 + bps;
    const int jmax = a.dense ? nb : a.k;
    if (j1 > jmax) j1 = jmax;

    auto block_at = [&](int j) -> int {
        // more than 32 given ids stay in global memory (each split reads its own range)
        const int id = a.dense ? j : (a.k > kMaxTopKList ? a.ids_in[((size_t)b * a.G + g) * a.k + j] : sel_i[j]);
        return (id >= 0 && id < nb) ? id : -1;
    };
    auto tiles_of = [&](int id) -> int {
        if (id < 0) return 0;
        int keys = pos + 1 - id * a.Bk;
        keys = keys < a.Bk ? keys : a.Bk;
        return (keys + KT - 1) / KT;
    };

    // producer (thread 0): walks (list position, tile) pairs
    int pj = j0, pt = 0;
    while (pj < j1 && tiles_of(block_at(pj)) == 0) ++pj;
    const unsigned char *kb = reinterpret_cast<const unsigned char *>(a.k_cache);
    const unsigned char *vb = reinterpret_cast<const unsigned char *>(a.v_cache);

    int issued = 0;
    bool failed = false;
    auto issue = [&]() {
        const int id = block_at(pj);
        const int key0 = id * a.Bk + pt * KT;
        int nk = pos + 1 - key0;
        nk = nk < KT ? nk : KT;
        const int in_block = (id + 1) * a.Bk - key0;
        nk = nk < in_block ? nk : in_block;
        const int slot = issued % NST;
        if (tid == 0) {
            const uint32_t bytes = (uint32_t)nk * D * ES;
            mbar_arrive_expect_tx(&bars[slot], 2 * bytes);
            const size_t src = (size_t)a.cache.row(b, g, a.G, a.L_max, key0) * D * ES;
            unsigned char *dst = ring + (size_t)slot * 2 * tile_bytes;
            bulk_g2s(dst, kb + src, bytes, &bars[slot], l2_evict_first_policy());
            bulk_g2s(dst + tile_bytes, vb + src, bytes, &bars[slot], l2_evict_first_policy());
        }
        ++issued;
        if (++pt >= tiles_of(id)) {
            pt = 0;
            ++pj;
            while (pj < j1 && tiles_of(block_at(pj)) == 0) ++pj;
        }
    };
    __syncthreads();  // barrier init visible before the first copy
    for (int i = 0; i < NST && pj < j1; ++i) issue();

    float acc[DPT];
#pragma unroll
    for (int d = 0; d < DPT; ++d) acc[d] = 0.f;
    const int flat = tid * DPT;
    const int ch = flat / D, cd = flat % D;  // P.V output owned by this thread
    const bool c_live = ch < r && flat < R * D;

    int consumed = 0;
    for (int j = j0; j < j1; ++j) {
        const int id = block_at(j);
        const int nt = tiles_of(id);
        for (int t = 0; t < nt; ++t) {
            const int key0 = id * a.Bk + t * KT;
            int nk = pos + 1 - key0;
            nk = nk < KT ? nk : KT;
            const int in_block = (id + 1) * a.Bk - key0;
            nk = nk < in_block ? nk : in_block;
            const int slot = consumed % NST;
            if (!failed && !mbar_wait(&bars[slot], (consumed / NST) & 1, a.status)) {
                failed = true;
                for (int q2 = consumed; q2 < issued; ++q2) mbar_wait(&bars[q2 % NST], (q2 / NST) & 1, nullptr);
            }
            const T *ks = reinterpret_cast<const T *>(ring + (size_t)slot * 2 * tile_bytes);
            const T *vs = reinterpret_cast<const T *>(ring + (size_t)slot * 2 * tile_bytes + tile_bytes);

            // scores z[h][key] = scale*log2e * q_h . k_key
            for (int key = w; key < nk; key += kAttnThreads / 32) {
                float kf[DPL];
                load_row<T, DPL>(ks + (size_t)key * D + lane * DPL, kf);
                float part[R];
#pragma unroll
                for (int h = 0; h < R; ++h) {
                    float acc_h = 0.f;
#pragma unroll
                    for (int d = 0; d < DPL; ++d) acc_h = fmaf(qreg[h][d], kf[d], acc_h);
                    part[h] = acc_h;
                }
                int head;
                const float z = reduce_scatter<R>(part, lane, head);
                if ((lane & (32 / R - 1)) == 0) p_s[head * KT + key] = z * a.scale_log2;
            }
            __syncthreads();
            // online softmax update, one warp per head
            for (int h = w; h < r; h += kAttnThreads / 32) {
                float mt = -INFINITY;
                for (int key = lane; key < nk; key += 32) mt = fmaxf(mt, p_s[h * KT + key]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, o));
                const float m_old = m_s[h];
                const float m_new = fmaxf(m_old, mt);
                float sum = 0.f;
                for (int key = lane; key < nk; key += 32) {
                    const float e = exp2f(p_s[h * KT + key] - m_new);
                    p_s[h * KT + key] = e;
                    sum += e;
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(FULL, sum, o);
                if (lane == 0) {
                    const float alpha = exp2f(m_old - m_new);  // 0 on the first tile (m_old = -inf)
                    al_s[h] = alpha;
                    l_s[h] = l_s[h] * alpha + sum;
                    m_s[h] = m_new;
                }
            }
            __syncthreads();
            if (c_live) {
                const float alpha = al_s[ch];
#pragma unroll
                for (int d = 0; d < DPT; ++d) acc[d] *= alpha;
                const float *ph = p_s + ch * KT;
                for (int key = 0; key < nk; ++key) {
                    float vf[DPT];
                    load_row<T, DPT>(vs + (size_t)key * D + cd, vf);
                    const float pk = ph[key];
#pragma unroll
                    for (int d = 0; d < DPT; ++d) acc[d] = fmaf(pk, vf[d], acc[d]);
                }
            }
            __syncthreads();  // stage and p_s free
            ++consumed;
            if (pj < j1 && !failed) issue();
        }
    }

    // normalised partial output and log2 normaliser of this split
    const size_t bg = (size_t)b * a.G + g;
    const size_t split = bg * a.S + s;
    if (c_live) {
        const float l = l_s[ch];
        const float inv = l > 0.f ? 1.f / l : 0.f;
        float *dst = a.part_o + (split * r + ch) * D + cd;
#pragma unroll
        for (int d = 0; d < DPT; ++d) dst[d] = acc[d] * inv;
    }
    if (tid < r) {
        const float l = l_s[tid];
        a.part_lse[split * r + tid] = l > 0.f ? m_s[tid] + log2f(l) : -INFINITY;
    }

    if (!last_split(a, b, g, &last_flag)) return;
    merge_splits<T>(a, b, g, p_s);  // p_s holds R * max(KT, kMaxSplits) floats
}


// ---------------------------------------------------------------- bf16: mma.sync tensor-core fragments

// thread-block cluster helpers (distributed shared memory)
__device__ inline void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ inline int cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return (int)r;
}
// store a float into the shared memory of CTA `rank` of the cluster, at the same offset as `local`
__device__ inline void st_peer(float *local, int rank, float v) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

constexpr int kMmaThreads = 128;  // 4 warps
constexpr int kMaxStages = 4;     // K/V ring stages (mbarriers reserved)
constexpr int kMmaRows = 16;      // query rows of the fragment (heads of the group, padded)
constexpr int kMaxCluster = 8;    // splits of a group that form one cluster

template <int D, bool SO>
__global__ void __launch_bounds__(kMmaThreads, 1) decode_attn_mma_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                      const __grid_constant__ CUtensorMap vmap,
                                                                      const AttnArgs a) {
    constexpr int NH = D / 64;     // 64-dim halves of a K/V row
    constexpr int KS = D / 16;     // k-steps of Q.K^T
    constexpr int DT = D / 8 / 4;  // 8-dim output tiles per warp
    const int KT = a.Bk < 128 ? a.Bk : 128;  // keys per tile
    const int KVH = KT * 128;                // bytes of one 64-dim half tile
    const int STAGE = 2 * NH * KVH;
    const int PST = KT + 8;                  // P row stride (bf16 elements), padded against bank conflicts

    extern __shared__ unsigned char smem_raw[];
    unsigned char *ring = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    __nv_bfloat16 *Ps = reinterpret_cast<__nv_bfloat16 *>(ring + a.ring_bytes);   // [16][PST]
    float *red_m = reinterpret_cast<float *>(Ps + kMmaRows * PST);                 // [4][16]
    float *red_l = red_m + 64;                                                     // [4][16]
    float *sel_s = red_l + 64;                                                     // [32]
    int *sel_i = reinterpret_cast<int *>(sel_s + 32);                              // [32]
    float *red_s = reinterpret_cast<float *>(sel_i + 32);                          // [32]
    int *red_i = reinterpret_cast<int *>(red_s + 32);                              // [32]
    int *misc = red_i + 32;                                                        // [4]
    uint64_t *bars = reinterpret_cast<uint64_t *>(misc + 4);                       // [kMaxStages]
    float *recv = reinterpret_cast<float *>(bars + kMaxStages);  // [cluster][slice] partials pushed to this CTA
    float *recv_l = recv + kMmaRows * D + kMaxCluster;   // [cluster][16] their log2 normalisers

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int grp = lane >> 2, tig = lane & 3;  // fragment row group / thread in group
    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int r = a.r;
    const int nst = a.nst;

    if (tid == 0) {
        for (int i = 0; i < nst; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        tc::prefetch_tmap(&kmap);
        tc::prefetch_tmap(&vmap);
    }
    // Q fragments (rows = heads of the group; rows >= r are zero), independent of Step 1
    uint32_t qa[KS][4];
    {
        const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(a.q) + ((size_t)b * a.Hq + (size_t)g * r) * D;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            const int c0 = ks * 16 + tig * 2;
            qa[ks][0] = grp < r ? *reinterpret_cast<const uint32_t *>(qg + (size_t)grp * D + c0) : 0u;
            qa[ks][1] = grp + 8 < r ? *reinterpret_cast<const uint32_t *>(qg + (size_t)(grp + 8) * D + c0) : 0u;
            qa[ks][2] = grp < r ? *reinterpret_cast<const uint32_t *>(qg + (size_t)grp * D + c0 + 8) : 0u;
            qa[ks][3] = grp + 8 < r ? *reinterpret_cast<const uint32_t *>(qg + (size_t)(grp + 8) * D + c0 + 8) : 0u;
        }
    }
    int L = a.seq_lens[b];
    L = L < 0 ? 0 : (L > a.L_max ? a.L_max : L);
    const int pos = L - 1;
    const int nb = (L + a.Bk - 1) / a.Bk;

    // where the scan leaves this group's lists is known from seq_lens alone
    const SegInfo info = (!SO && !a.dense && a.cand_s != nullptr) ? seg_pieces(a, b, g % a.Hik) : SegInfo{-1, 0};
    pdl_wait_prior_grid();  // the scan's candidates are complete from here on
    pdl_allow_next_grid();
    group_list<SO>(a, b, g, info, ring, sel_s, sel_i);

    // this split's blocks: list positions [j0, j1), each cut into tiles of KT keys
    const int j0 = s * a.blocks_per_split;
    int j1 = j0 + a.blocks_per_split;
    const int jmax = a.dense ? nb : a.k;
    if (j1 > jmax) j1 = jmax;
    auto block_at = [&](int j) -> int {
        // more than 32 given ids stay in global memory (each split reads its own range)
        const int id = a.dense ? j : (a.k > kMaxTopKList ? a.ids_in[((size_t)b * a.G + g) * a.k + j] : sel_i[j]);
        return (id >= 0 && id < nb) ? id : -1;
    };
    auto tiles_of = [&](int id) -> int {
        if (id < 0) return 0;
        int keys = pos + 1 - id * a.Bk;
        keys = keys < a.Bk ? keys : a.Bk;
        return (keys + KT - 1) / KT;
    };
    int pj = j0, pt = 0, issued = 0;
    while (pj < j1 && tiles_of(block_at(pj)) == 0) ++pj;
    auto issue = [&]() {
        const int id = block_at(pj);
        const int slot = issued % nst;
        if (tid == 0) {
            unsigned char *dst = ring + slot * STAGE;
            mbar_arrive_expect_tx(&bars[slot], STAGE);
            const int row = a.cache.row(b, g, a.G, a.L_max, id * a.Bk + pt * KT);
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                tc::tma_load_2d(dst + h * KVH, &kmap, h * 64, row, &bars[slot]);
                tc::tma_load_2d(dst + (NH + h) * KVH, &vmap, h * 64, row, &bars[slot]);
            }
        }
        ++issued;
        if (++pt >= tiles_of(id)) {
            pt = 0;
            ++pj;
            while (pj < j1 && tiles_of(block_at(pj)) == 0) ++pj;
        }
    };
    __syncthreads();  // barrier init and the list visible; the selection scratch is free
    for (int i = 0; i < nst && pj < j1; ++i) issue();

    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    float oacc[DT][4];
#pragma unroll
    for (int t = 0; t < DT; ++t) oacc[t][0] = oacc[t][1] = oacc[t][2] = oacc[t][3] = 0.f;
    const uint32_t ps_addr = smem_u32(Ps);
    int consumed = 0;
    bool failed = false;
    for (int j = j0; j < j1; ++j) {
        const int id = block_at(j);
        const int ntl = tiles_of(id);
        for (int t = 0; t < ntl; ++t) {
            const int key0 = id * a.Bk + t * KT;
            int nk = pos + 1 - key0;
            nk = nk < KT ? nk : KT;
            const int slot = consumed % nst;
            if (!failed && !mbar_wait(&bars[slot], (consumed / nst) & 1, a.status)) {
                failed = true;
                for (int q2 = consumed; q2 < issued; ++q2) mbar_wait(&bars[q2 % nst], (q2 / nst) & 1, nullptr);
            }
            const uint32_t k_addr = smem_u32(ring + slot * STAGE);
            const uint32_t v_addr = k_addr + NH * KVH;
            // S = Q K^T for this warp's 8-key tiles kn = w, w+4, ...
            float mx[2] = {-INFINITY, -INFINITY};
            float sv[4][4];
            const int n_kt = KT / 8;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int kn = w + 4 * i;
                sv[i][0] = sv[i][1] = sv[i][2] = sv[i][3] = 0.f;
                if (kn < n_kt) {
#pragma unroll
                    for (int ks = 0; ks < KS; ks += 2) {
                        const int mi = lane >> 3;
                        const int key = kn * 8 + (lane & 7);
                        const int d0 = (ks + (mi >> 1)) * 16 + (mi & 1) * 8;
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(k_addr + (d0 >> 6) * KVH + sw128(key, (d0 & 63) >> 3), b0, b1, b2, b3);
                        mma_16816(sv[i], qa[ks], b0, b1);
                        mma_16816(sv[i], qa[ks + 1], b2, b3);
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int key = kn * 8 + tig * 2 + (e & 1);
                        sv[i][e] = key < nk ? sv[i][e] * a.scale_log2 : -INFINITY;
                        mx[e >> 1] = fmaxf(mx[e >> 1], sv[i][e]);
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(FULL, mx[h], 1));
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(FULL, mx[h], 2));
            }
            if (tig == 0) { red_m[w * 16 + grp] = mx[0]; red_m[w * 16 + grp + 8] = mx[1]; }
            __syncthreads();
            float alpha[2], m_new[2], ls[2] = {0.f, 0.f};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = grp + 8 * h;
                const float mb = fmaxf(fmaxf(red_m[row], red_m[16 + row]), fmaxf(red_m[32 + row], red_m[48 + row]));
                m_new[h] = fmaxf(m_run[h], mb);
                alpha[h] = m_run[h] > -INFINITY ? exp2f(m_run[h] - m_new[h]) : 0.f;
            }
            // P = exp2(S - m) as bf16 into shared memory
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int kn = w + 4 * i;
                if (kn < n_kt) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float p0 = sv[i][2 * h] > -INFINITY ? exp2f(sv[i][2 * h] - m_new[h]) : 0.f;
                        const float p1 = sv[i][2 * h + 1] > -INFINITY ? exp2f(sv[i][2 * h + 1] - m_new[h]) : 0.f;
                        const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                        ls[h] += __low2float(pb) + __high2float(pb);
                        *reinterpret_cast<__nv_bfloat162 *>(Ps + (grp + 8 * h) * PST + kn * 8 + tig * 2) = pb;
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                ls[h] += __shfl_xor_sync(FULL, ls[h], 1);
                ls[h] += __shfl_xor_sync(FULL, ls[h], 2);
            }
            if (tig == 0) { red_l[w * 16 + grp] = ls[0]; red_l[w * 16 + grp + 8] = ls[1]; }
            __syncthreads();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = grp + 8 * h;
                const float lb = red_l[row] + red_l[16 + row] + red_l[32 + row] + red_l[48 + row];
                l_run[h] = l_run[h] * alpha[h] + lb;
                m_run[h] = m_new[h];
            }
#pragma unroll
            for (int dt = 0; dt < DT; ++dt) {
                oacc[dt][0] *= alpha[0]; oacc[dt][1] *= alpha[0];
                oacc[dt][2] *= alpha[1]; oacc[dt][3] *= alpha[1];
            }
            // O += P V: this warp's 8-dim output tiles dn = w, w+4, ...
            for (int ks = 0; ks < KT / 16; ++ks) {
                uint32_t pa[4];
                {
                    const int mi = lane >> 3;
                    const int row = (mi & 1) * 8 + (lane & 7);
                    const int key = ks * 16 + (mi >> 1) * 8;
                    ldsm_x4(ps_addr + (uint32_t)(row * PST + key) * 2, pa[0], pa[1], pa[2], pa[3]);
                }
#pragma unroll
                for (int dp = 0; dp < DT; dp += 2) {
                    const int mi = lane >> 3;
                    const int dn = w + 4 * (dp + (mi >> 1));
                    const int key = ks * 16 + (mi & 1) * 8 + (lane & 7);
                    const int d0 = dn * 8;
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(v_addr + (d0 >> 6) * KVH + sw128(key, (d0 & 63) >> 3), b0, b1, b2, b3);
                    mma_16816(oacc[dp], pa, b0, b1);
                    mma_16816(oacc[dp + 1], pa, b2, b3);
                }
            }
            __syncthreads();  // stage and P free
            ++consumed;
            if (pj < j1 && !failed) issue();
        }
    }

    if (a.cluster > 1) {
        // The splits of (b, g) form one thread-block cluster.  CTA c owns a slice of the r * D
        // outputs; every CTA stores its normalised partial of each slice, and its log2
        // normalisers, straight into the owner's shared memory, and after one cluster barrier
        // each owner merges its slice from local memory (nothing is read remotely).
        const int cs = a.cluster, rank = cluster_rank();
        const int n_out = r * D, per = (n_out + cs - 1) / cs;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int row = grp + 8 * h;
            if (row >= r) continue;
            const float inv = l_run[h] > 0.f ? 1.f / l_run[h] : 0.f;
#pragma unroll
            for (int dt = 0; dt < DT; ++dt) {
                const int f = row * D + (w + 4 * dt) * 8 + tig * 2;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int owner = (f + e) / per;
                    st_peer(recv + rank * per + (f + e - owner * per), owner, oacc[dt][2 * h + e] * inv);
                }
            }
            if (w == 0 && tig == 0) {
                const float lse2 = l_run[h] > 0.f ? m_run[h] + log2f(l_run[h]) : -INFINITY;
                for (int c = 0; c < cs; ++c) st_peer(recv_l + rank * kMmaRows + row, c, lse2);
            }
        }
        cluster_sync_all();
        const int f_end = (rank + 1) * per < n_out ? (rank + 1) * per : n_out;
        __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(a.o) + ((size_t)b * a.Hq + (size_t)g * r) * D;
        for (int f = rank * per + tid; f < f_end; f += kMmaThreads) {
            const int h = f / D;
            float M = -INFINITY;
            for (int c = 0; c < cs; ++c) M = fmaxf(M, recv_l[c * kMmaRows + h]);
            float num = 0.f, den = 0.f;
            for (int c = 0; c < cs; ++c) {
                const float lc = recv_l[c * kMmaRows + h];
                if (lc > -INFINITY) {
                    const float wgt = exp2f(lc - M);
                    den += wgt;
                    num = fmaf(wgt, recv[c * per + (f - rank * per)], num);
                }
            }
            o[f] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
            if (a.lse != nullptr && f % D == 0)
                a.lse[(size_t)b * a.Hq + (size_t)g * r + h] =
                    den > 0.f ? (M + log2f(den)) * 0.69314718055994531f : -INFINITY;
        }
        return;  // no peer touches this CTA's shared memory after the barrier
    }

    // normalised partial output and log2 normaliser of this split
    const size_t split = ((size_t)b * a.G + g) * a.S + s;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int row = grp + 8 * h;
        if (row < r) {
            const float inv = l_run[h] > 0.f ? 1.f / l_run[h] : 0.f;
            float *dst = a.part_o + (split * r + row) * D;
#pragma unroll
            for (int dt = 0; dt < DT; ++dt) {
                const int d = (w + 4 * dt) * 8 + tig * 2;
                *reinterpret_cast<float2 *>(dst + d) = make_float2(oacc[dt][2 * h] * inv, oacc[dt][2 * h + 1] * inv);
            }
            if (w == 0 && tig == 0)
                a.part_lse[split * r + row] = l_run[h] > 0.f ? m_run[h] + log2f(l_run[h]) : -INFINITY;
        }
    }
    if (!last_split(a, b, g, &misc[1])) return;
    merge_splits<__nv_bfloat16>(a, b, g, reinterpret_cast<float *>(ring));
}

template <typename T, int D, int R>
cudaError_t launch_attn_t(AttnArgs a, cudaStream_t s, bool pdl) {
    using Cfg = AttnCfg<T, D, R>;
    const int KT = a.Bk < Cfg::KT_MAX ? a.Bk : Cfg::KT_MAX;
    const size_t ring = (size_t)Cfg::NST * 2 * KT * D * Cfg::ES;
    const size_t scratch = a.cand_s != nullptr ? select_scratch_bytes(a.n_cta, a.k) : 0;
    a.ring_bytes = (int)((ring > scratch ? ring : scratch) + 15) / 16 * 16;
    // p_s doubles as the [S][r] merge weights of the last split: R * max(KT, kMaxSplits) floats
    const size_t smem = (size_t)a.ring_bytes + Cfg::NST * 8 + 64 * 4 + 3 * R * 4 +
                        (size_t)R * (KT > kMaxSplits ? KT : kMaxSplits) * 4 + 16;
    static size_t attr_bytes = 0;
    if (smem > attr_bytes) {
        cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<T, D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        attr_bytes = smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.S, a.G, a.B);
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode_attn_kernel<T, D, R>, a);
}

template <typename T, int D>
cudaError_t launch_attn_r(const AttnArgs &a, cudaStream_t s, bool pdl) {
    const int r = a.r;
    if (r <= 1) return launch_attn_t<T, D, 1>(a, s, pdl);
    if (r <= 2) return launch_attn_t<T, D, 2>(a, s, pdl);
    if (r <= 4) return launch_attn_t<T, D, 4>(a, s, pdl);
    if (r <= 8) return launch_attn_t<T, D, 8>(a, s, pdl);
    return launch_attn_t<T, D, 16>(a, s, pdl);
}

template <int D, bool SO>
cudaError_t launch_mma_t(AttnArgs a, cudaStream_t s, bool pdl) {
    a.cluster = (!a.dense && a.S <= kMaxCluster) ? a.S : 1;
    const int KT = a.Bk < 128 ? a.Bk : 128;
    const size_t stage = (size_t)2 * (D / 64) * KT * 128;
    // one stage when every split is a single tile; three for long splits of small tiles (large
    // k, 64-key blocks: two CTAs per SM then keep 192 KB of K/V in flight per SM), two otherwise
    const bool one_tile = a.blocks_per_split == 1 && a.Bk <= 128;
    const int tiles = a.blocks_per_split * ((a.Bk + KT - 1) / KT);
    a.nst = one_tile ? 1 : (stage <= 32768 && tiles >= 3 ? 3 : 2);
    const size_t ring = a.nst * stage;
    const size_t scratch = a.cand_s != nullptr ? select_scratch_bytes(a.n_cta, a.k) : 0;
    const size_t wgt = (size_t)a.S * a.r * 4 > (size_t)kMmaRows * D * 4 + 64 ? (size_t)a.S * a.r * 4
                                                                            : (size_t)kMmaRows * D * 4 + 64;
    size_t rb = ring > scratch ? ring : scratch;
    rb = rb > wgt ? rb : wgt;
    a.ring_bytes = (int)((rb + 1023) / 1024 * 1024);
    const size_t smem = 1024 + (size_t)a.ring_bytes + (size_t)kMmaRows * (KT + 8) * 2 + (64 + 64 + 32 * 4 + 4) * 4 + kMaxStages * 8 +
                        ((size_t)kMmaRows * D + kMaxCluster + (size_t)kMaxCluster * kMmaRows) * 4 + 64;
    static size_t attr_bytes = 0;
    if (smem > attr_bytes) {
        cudaError_t e = cudaFuncSetAttribute(decode_attn_mma_kernel<D, SO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        attr_bytes = smem;
    }
    CUtensorMap km, vm;
    const unsigned long long rows = a.cache.rows(a.B, a.G, a.L_max);
    if (!encode_2d(&km, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void *>(a.k_cache), D, rows, D * 2, 64, KT,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&vm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void *>(a.v_cache), D, rows, D * 2, 64, KT,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.S, a.G, a.B);
    cfg.blockDim = dim3(kMmaThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (a.cluster > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = a.cluster;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, decode_attn_mma_kernel<D, SO>, km, vm, a);
}

template <int D>
cudaError_t launch_mma(const AttnArgs &a, cudaStream_t s, bool pdl) {
    return a.scores_only ? launch_mma_t<D, true>(a, s, pdl) : launch_mma_t<D, false>(a, s, pdl);
}


// ---------------------------------------------------------------- bf16, many tiles per split
// Large k and MSA_DENSE give every split tens to hundreds of key tiles.  One CTA per SM; each of
// its NW warps owns SPW ring stages (K and V of TK keys each) and runs its own tiles
// t = w, w + NW, ... from copy to output with no barrier: while it works on one tile its next
// one is on the way.  S = Q K^T on mma.sync fragments, the online softmax on the quad's
// registers, P handed to P V straight from the S accumulators (the accumulator layout of two
// 8-key tiles is the A-fragment layout of one 16-key step).  NW x SPW stages keep ~192 KB of
// K/V in flight per SM.  The warps' (m, l, O) are combined in shared memory at the end; splits
// merge by log-sum-exp as in the other kernels.
constexpr int kWideRing = 196608;  // bytes of ring per CTA

template <int D> struct WideShape {
    static constexpr int TK = D == 128 ? 32 : 64;        // keys per tile
    static constexpr int STAGE = 2 * D * TK * 2;         // K and V of one tile, bf16 (16 KB)
    static constexpr int SPW = 2;                        // stages per warp
    static constexpr int NW = kWideRing / (STAGE * SPW); // warps
};

template <int D>
__global__ void __launch_bounds__(WideShape<D>::NW * 32, 1)
    decode_attn_wide_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                            const AttnArgs a) {
    constexpr int NW = WideShape<D>::NW, STAGE = WideShape<D>::STAGE, SPW = WideShape<D>::SPW;
    constexpr int TK = WideShape<D>::TK;
    constexpr int NH = D / 64;          // 64-dim halves of a K/V row
    constexpr int KS = D / 16;          // k-steps of Q.K^T
    constexpr int NT = TK / 8;          // 8-key tiles of S
    constexpr int DN = D / 8;           // 8-dim output tiles
    constexpr int KVH = TK * 128;       // bytes of one 64-dim half tile
    extern __shared__ unsigned char smem_raw[];
    unsigned char *ring = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring + NW * SPW * STAGE);  // [NW][SPW]
    float *cm = reinterpret_cast<float *>(bars + NW * SPW);                   // [NW][16] warps' row maxima
    float *cl = cm + NW * 16;                                                 // [NW][16] warps' row sums
    int *misc = reinterpret_cast<int *>(cl + NW * 16);                        // [4]
    int *sid = misc + 4;                                                      // [kMaxTopK] the split's ids

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int grp = lane >> 2, tig = lane & 3;
    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int r = a.r;
    uint64_t *my_bars = bars + w * SPW;
    if (lane < SPW) mbar_init(&my_bars[lane], 1);
    if (tid == 0) {
        tc::prefetch_tmap(&kmap);
        tc::prefetch_tmap(&vmap);
    }
    fence_mbar_init();
    __syncwarp();
    uint32_t qa[KS][4];
    {
        const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(a.q) + ((size_t)b * a.Hq + (size_t)g * r) * D;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            const int c0 = ks * 16 + tig * 2;
            qa[ks][0] = grp < r ? *reinterpret_cast<const uint32_t *>(qg + (size_t)grp * D + c0) : 0u;
            qa[ks][1] = grp + 8 < r ? *reinterpret_cast<const uint32_t *>(qg + (size_t)(grp + 8) * D + c0) : 0u;
            qa[ks][2] = grp < r ? *reinterpret_cast<const uint32_t *>(qg + (size_t)grp * D + c0 + 8) : 0u;
            qa[ks][3] = grp + 8 < r ? *reinterpret_cast<const uint32_t *>(qg + (size_t)(grp + 8) * D + c0 + 8) : 0u;
        }
    }
    int L = a.seq_lens[b];
    L = L < 0 ? 0 : (L > a.L_max ? a.L_max : L);
    const int pos = L - 1;
    const int nb = (L + a.Bk - 1) / a.Bk;
    pdl_wait_prior_grid();  // the selection (large k) is complete from here on
    pdl_allow_next_grid();

    // this split's list positions [j0, j1), each block cut into TPB tiles of TK keys
    const int TPB = (a.Bk + TK - 1) / TK;
    const int j0 = s * a.blocks_per_split;
    int j1 = j0 + a.blocks_per_split;
    const int jmax = a.dense ? nb : a.k;
    if (j1 > jmax) j1 = jmax;
    const int n_tiles = j1 > j0 ? (j1 - j0) * TPB : 0;
    if (!a.dense) {
        // the split's ids into shared memory once (a global load per tile would sit on the
        // issue path of every copy)
        const int *ids = a.ids_in + ((size_t)b * a.G + g) * a.k;
        for (int j = j0 + tid; j < j1; j += NW * 32) sid[j - j0] = ids[j];
        __syncthreads();
    }
    // first key and visible key count of tile t of the split (0 keys: nothing to do)
    auto tile_of = [&](int t, int &key0) -> int {
        const int j = j0 + t / TPB;
        const int id = a.dense ? j : sid[j - j0];
        if (id < 0 || id >= nb) return 0;
        key0 = id * a.Bk + (t % TPB) * TK;
        const int blk_end = (id + 1) * a.Bk < pos + 1 ? (id + 1) * a.Bk : pos + 1;
        const int nk = blk_end - key0;
        return nk < TK ? (nk > 0 ? nk : 0) : TK;
    };
    unsigned char *my_ring = ring + (size_t)w * SPW * STAGE;
    // the warp's tiles in order: the next one with keys is copied into the next stage
    int t_next = w, issued = 0, consumed = 0;
    int nk_slot[SPW];
#pragma unroll
    for (int i = 0; i < SPW; ++i) nk_slot[i] = 0;
    auto issue = [&]() {
        int key0 = 0, nk = 0;
        for (; t_next < n_tiles; t_next += NW) {
            nk = tile_of(t_next, key0);
            if (nk > 0) break;
        }
        if (t_next >= n_tiles) return;
        t_next += NW;
        const int slot = issued % SPW;
#pragma unroll
        for (int i = 0; i < SPW; ++i)
            if (i == slot) nk_slot[i] = nk;
        if (lane == 0) {
            unsigned char *st = my_ring + (size_t)slot * STAGE;
            mbar_arrive_expect_tx(&my_bars[slot], STAGE);
            const int row = a.cache.row(b, g, a.G, a.L_max, key0);
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                tc::tma_load_2d(st + h * KVH, &kmap, h * 64, row, &my_bars[slot]);
                tc::tma_load_2d(st + (NH + h) * KVH, &vmap, h * 64, row, &my_bars[slot]);
            }
        }
        ++issued;
    };
#pragma unroll
    for (int i = 0; i < SPW; ++i) issue();

    float m_run[2] = {-INFINITY, -INFINITY}, l_part[2] = {0.f, 0.f};
    float oacc[DN][4];
#pragma unroll
    for (int dn = 0; dn < DN; ++dn) oacc[dn][0] = oacc[dn][1] = oacc[dn][2] = oacc[dn][3] = 0.f;
    bool failed = false;
    while (consumed < issued) {
        const int slot = consumed % SPW;
        if (!mbar_wait(&my_bars[slot], (consumed / SPW) & 1, a.status)) {
            // give up: wait (bounded) for the warp's copies in flight, issue nothing more
            failed = true;
            for (int q2 = consumed; q2 < issued; ++q2) mbar_wait(&my_bars[q2 % SPW], (q2 / SPW) & 1, nullptr);
            break;
        }
        int nk = 0;
#pragma unroll
        for (int i = 0; i < SPW; ++i)
            if (i == slot) nk = nk_slot[i];
        const uint32_t k_addr = smem_u32(my_ring + (size_t)slot * STAGE), v_addr = k_addr + NH * KVH;
        // S = Q K^T (scaled to the log2 domain), keys past the row masked
        float sv[NT][4];
#pragma unroll
        for (int kn = 0; kn < NT; ++kn) sv[kn][0] = sv[kn][1] = sv[kn][2] = sv[kn][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ks += 2) {
            const int mi = lane >> 3;
            const int d0 = (ks + (mi >> 1)) * 16 + (mi & 1) * 8;
#pragma unroll
            for (int kn = 0; kn < NT; ++kn) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(k_addr + (d0 >> 6) * KVH + sw128(kn * 8 + (lane & 7), (d0 & 63) >> 3), b0, b1, b2, b3);
                mma_16816(sv[kn], qa[ks], b0, b1);
                mma_16816(sv[kn], qa[ks + 1], b2, b3);
            }
        }
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int kn = 0; kn < NT; ++kn)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = kn * 8 + tig * 2 + (e & 1);
                sv[kn][e] = key < nk ? sv[kn][e] * a.scale_log2 : -INFINITY;
                mx[e >> 1] = fmaxf(mx[e >> 1], sv[kn][e]);
            }
        float alpha[2], m_new[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(FULL, mx[h], 1));
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(FULL, mx[h], 2));
            m_new[h] = fmaxf(m_run[h], mx[h]);
            alpha[h] = m_run[h] > -INFINITY ? exp2f(m_run[h] - m_new[h]) : 0.f;
            m_run[h] = m_new[h];
            l_part[h] *= alpha[h];
        }
#pragma unroll
        for (int dn = 0; dn < DN; ++dn) {
            oacc[dn][0] *= alpha[0]; oacc[dn][1] *= alpha[0];
            oacc[dn][2] *= alpha[1]; oacc[dn][3] *= alpha[1];
        }
        // O += P V, 16 keys per step; P's A fragments come from the S accumulators of two 8-key tiles
#pragma unroll
        for (int kc = 0; kc < TK / 16; ++kc) {
            uint32_t pa[4];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {      // the two 8-key tiles of the step
#pragma unroll
                for (int h = 0; h < 2; ++h) {     // rows grp, grp + 8
                    const float x0 = sv[2 * kc + hh][2 * h], x1 = sv[2 * kc + hh][2 * h + 1];
                    const float p0 = x0 > -INFINITY ? exp2f(x0 - m_new[h]) : 0.f;
                    const float p1 = x1 > -INFINITY ? exp2f(x1 - m_new[h]) : 0.f;
                    const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                    l_part[h] += __low2float(pb) + __high2float(pb);
                    pa[hh * 2 + h] = *reinterpret_cast<const uint32_t *>(&pb);
                }
            }
#pragma unroll
            for (int dp = 0; dp < DN; dp += 2) {
                const int mi = lane >> 3;
                const int d0 = (dp + (mi >> 1)) * 8;
                const int key = kc * 16 + (mi & 1) * 8 + (lane & 7);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(v_addr + (d0 >> 6) * KVH + sw128(key, (d0 & 63) >> 3), b0, b1, b2, b3);
                mma_16816(oacc[dp], pa, b0, b1);
                mma_16816(oacc[dp + 1], pa, b2, b3);
            }
        }
        __syncwarp();  // every lane is done with the stage before it is refilled
        ++consumed;
        issue();
    }
    (void)failed;

    // the warp's rows: quad sums, then every warp's (m, l, O) combined in shared memory
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l_part[h] += __shfl_xor_sync(FULL, l_part[h], 1);
        l_part[h] += __shfl_xor_sync(FULL, l_part[h], 2);
    }
    __syncthreads();  // every warp is done with the ring: it holds the warps' O now
    float *co = reinterpret_cast<float *>(ring);  // [NW][16][D]
    if (tig == 0) {
        cm[w * 16 + grp] = m_run[0];
        cm[w * 16 + grp + 8] = m_run[1];
        cl[w * 16 + grp] = l_part[0];
        cl[w * 16 + grp + 8] = l_part[1];
    }
#pragma unroll
    for (int dn = 0; dn < DN; ++dn) {
        const int d = dn * 8 + tig * 2;
        *reinterpret_cast<float2 *>(co + ((size_t)w * 16 + grp) * D + d) = make_float2(oacc[dn][0], oacc[dn][1]);
        *reinterpret_cast<float2 *>(co + ((size_t)w * 16 + grp + 8) * D + d) = make_float2(oacc[dn][2], oacc[dn][3]);
    }
    __syncthreads();
    const size_t split = ((size_t)b * a.G + g) * a.S + s;
    for (int f = tid; f < r * D; f += NW * 32) {
        const int row = f / D, d = f % D;
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < NW; ++ww) M = fmaxf(M, cm[ww * 16 + row]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int ww = 0; ww < NW; ++ww) {
            const float mw = cm[ww * 16 + row];
            if (mw > -INFINITY) {
                const float e = exp2f(mw - M);
                num = fmaf(e, co[((size_t)ww * 16 + row) * D + d], num);
                den = fmaf(e, cl[ww * 16 + row], den);
            }
        }
        a.part_o[(split * r + row) * D + d] = den > 0.f ? num / den : 0.f;
        if (d == 0) a.part_lse[split * r + row] = den > 0.f ? M + log2f(den) : -INFINITY;
    }
    if (!last_split(a, b, g, &misc[0])) return;
    merge_splits<__nv_bfloat16>(a, b, g, reinterpret_cast<float *>(ring));
}

template <int D>
cudaError_t launch_wide(const AttnArgs &a, cudaStream_t s, bool pdl) {
    constexpr int NW = WideShape<D>::NW, STAGE = WideShape<D>::STAGE, SPW = WideShape<D>::SPW;
    constexpr int TK = WideShape<D>::TK;
    const size_t smem = 1024 + (size_t)NW * SPW * STAGE + NW * SPW * 8 + (size_t)NW * 16 * 4 * 2 + 16 + kMaxTopK * 4;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(decode_attn_wide_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    CUtensorMap km, vm;
    const unsigned long long rows = a.cache.rows(a.B, a.G, a.L_max);
    if (!encode_2d(&km, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void *>(a.k_cache), D, rows, D * 2, 64, TK,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&vm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void *>(a.v_cache), D, rows, D * 2, 64, TK,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.S, a.G, a.B);
    cfg.blockDim = dim3(NW * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode_attn_wide_kernel<D>, km, vm, a);
}
}  // namespace

// bf16 splits of many tiles (large k, MSA_DENSE) take the warp-per-stage kernel; the sparse step
// with k <= kMaxTopKList (a few blocks per split, the selection inside) takes decode_attn_mma_kernel.
bool wide_attention(const msa_params_t &p) {
    return p.dtype == MSA_BF16 && ((p.flags & MSA_DENSE) || p.top_k > kMaxTopKList);
}

cudaError_t launch_decode_attn(const AttnArgs &a, int dtype, cudaStream_t s, bool pdl) {
    if (dtype == MSA_BF16 && (a.dense || a.k > kMaxTopKList))
        return a.D == 64 ? launch_wide<64>(a, s, pdl) : launch_wide<128>(a, s, pdl);
    if (dtype == MSA_BF16) return a.D == 64 ? launch_mma<64>(a, s, pdl) : launch_mma<128>(a, s, pdl);
    return a.D == 64 ? launch_attn_r<float, 64>(a, s, pdl) : launch_attn_r<float, 128>(a, s, pdl);
}

}  // namespace msa
