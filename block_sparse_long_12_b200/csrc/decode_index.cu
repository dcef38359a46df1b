// Step 1 of MSA for decode: index scores, block max pool, per-piece TopK.
//
// Page "MiniMax wird duenn" (atlascloud.ai), section 1, Step 1: the group's
// index query scores every cached token against its index key, the scores
// are max-pooled per fixed-size block, and TopK keeps the best blocks of the
// group.  For decode this is a single query against the whole cache, so the
// kernel is a stream of k_idx from HBM: each byte is read once.
//
// Work split: the first three quarters of the index-K streams of all
// (sequence b, index-K head) pairs are concatenated (block granularity) and
// cut into n_cta ranges of equal length (the last one shorter), one per
// persistent CTA (one CTA per SM), so ragged lengths stay balanced.  SMs do
// not stream equally fast, so the last quarter of every stream is a shared
// tail: each warp that is done with its range takes tail blocks one at a
// time from a few interleaved counters in the workspace, and the faster SMs
// take more of them.  Tail blocks leave only their block scores; the
// attention kernel's select merges them with the ranges' candidate lists.  Inside a CTA every warp owns a private two-stage
// ring of 8 KB shared-memory tiles filled by TMA tensor copies
// (cp.async.bulk.tensor, 128-byte swizzle) and consumes the blocks w, w+W, ...
// of the CTA's range.  One lane owns one index-key row: the swizzle makes the
// 32 lanes' 16-byte reads of the same vector position hit distinct banks, so
// the fp32 dot product against the index query (registers) needs no
// cross-lane reduction; a warp max per block gives the block score and a
// warp-distributed sorted list keeps the warp's best blocks.  At the end of
// each piece the warp lists are merged into one sorted candidate list per
// group; decode_select_kernel merges the pieces of a segment.
#include <type_traits>

#include "tcgen05.cuh"

namespace msa {

namespace {

struct Piece {
    int b, hik, nb, n0, n1, idx;  // segment (b, hik) with nb blocks; this CTA's blocks [n0, n1); piece index
    long long seg_start;
};

// CTA i owns the global blocks [i*per, (i+1)*per) (clipped to the total), so
// every CTA below ceil(total/per) has a non-empty range and the CTAs that
// touch a segment are consecutive and all write a piece.
__device__ inline int cta_of(long long x, long long per) { return (int)(x / per); }

// Enumerates the pieces of the range [x, x1) in order.
struct PieceWalker {
    long long x, x1;
    __device__ inline bool next(const long long *off, const int *nbs, int B, int Hik, Piece &p) {
        if (x >= x1) return false;
        int lo = 0, hi = B - 1;  // largest b with off[b] <= x (never an empty sequence since x < off[B])
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (off[mid] <= x) lo = mid; else hi = mid - 1;
        }
        p.b = lo;
        p.nb = nbs[lo];
        p.hik = (int)((x - off[lo]) / p.nb);
        p.seg_start = off[lo] + (long long)p.hik * p.nb;
        p.n0 = (int)(x - p.seg_start);
        const long long end = x1 - p.seg_start;
        p.n1 = end < p.nb ? (int)end : p.nb;
        p.idx = 0;
        x = p.seg_start + p.n1;
        return true;
    }
};

// The chunk sequence one warp consumes: its blocks n0+w, n0+w+W, ... of every
// piece, each block cut into chunks of at most kScanChunkBytes.
struct ChunkCursor {
    PieceWalker pw;
    Piece p;
    int n, c, nch, valid;
    int w, W, Bk, ct;  // warp, warps per CTA, block size, tokens per chunk
    __device__ inline int block_tokens(const int *lens) const {
        const int L = lens[p.b];
        const int t = L - n * Bk;
        return t < Bk ? t : Bk;
    }
    __device__ inline bool next_piece(const long long *off, const int *nbs, const int *lens, int B, int Hik) {
        while (pw.next(off, nbs, B, Hik, p)) {
            n = p.n0 + w;
            if (n < p.n1) {
                c = 0;
                nch = (block_tokens(lens) + ct - 1) / ct;
                return true;
            }
        }
        return false;
    }
    __device__ inline void start(const long long *off, const int *nbs, const int *lens, int B, int Hik) {
        valid = next_piece(off, nbs, lens, B, Hik);
    }
    __device__ inline void advance(const long long *off, const int *nbs, const int *lens, int B, int Hik) {
        if (++c < nch) return;
        n += W;
        if (n < p.n1) {
            c = 0;
            nch = (block_tokens(lens) + ct - 1) / ct;
            return;
        }
        valid = next_piece(off, nbs, lens, B, Hik);
    }
};

// MXFP8 keys: the E8M0 scales of a chunk's rows are copied beside its codes, at most 256 bytes
constexpr int kScaleStage = 256;
template <typename T> constexpr bool is_fp8() { return sizeof(T) == 1; }
// several groups on one bf16 stream of 128- or 256-byte rows are scored on tensor cores
template <typename T, int GPS, int ROWB> constexpr bool scan_mma() { return GPS > 1 && sizeof(T) == 2 && ROWB >= 128; }
// Warps per CTA (W): one index-K head per stream (GPS 1) keeps the index query in registers and
// affords 12 warps; several groups on one stream read it from shared memory (CUDA cores, 8 warps)
// or hold it as mma fragments (8 warps with three ring stages each while the batch's bookkeeping
// leaves the shared memory, two beyond: measured at 1M with one shared head, 57.0 us per step
// against 58.3 with 12 warps of two stages, the same bytes in flight).

// S: ring stages per warp (2)
template <typename T, int GPS, int ROWB, int S, int W>
__global__ void __launch_bounds__(W * 32, 1)
    decode_scan_kernel(const __grid_constant__ CUtensorMap kmap, const ScanArgs a) {
    constexpr int ES = (int)sizeof(T);
    constexpr int EPV = Vec16<T>::N;      // elements per 16-byte vector
    constexpr int NCH = ROWB / 16;        // 16-byte vectors per index-key row
    constexpr int DI = ROWB / ES;         // index dim
    constexpr bool QREG = GPS == 1 && DI <= 64;
    // several groups on one bf16 stream: the scores of a chunk are a small GEMM (the chunk's keys
    // times the groups' index queries, padded to 8 columns) on mma.sync tensor-core fragments
    constexpr bool MMA = scan_mma<T, GPS, ROWB>();
    constexpr int KS = DI / 16;           // k-steps of 16 index dims
    constexpr bool FP8 = is_fp8<T>();     // MXFP8 keys: E4M3 codes, one E8M0 scale per 32 dims
    constexpr int SPR = FP8 ? DI / 32 : 0;  // scale bytes per row
    const int CT = a.chunk_tokens;        // tokens per chunk (<= block size, 8 KB at most)

    extern __shared__ unsigned char smem_raw[];
    unsigned char *ring = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);  // [W][S][8 KB]
    unsigned char *sring = ring + (size_t)W * S * kScanChunkBytes;                    // FP8: [W][S][256]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sring + (FP8 ? (size_t)W * S * kScaleStage : 0));
    float *lists_s = reinterpret_cast<float *>(bars + W * S);                 // [W][GPS][32]
    int *lists_i = reinterpret_cast<int *>(lists_s + W * GPS * 32);
    float *q_s = reinterpret_cast<float *>(lists_i + W * GPS * 32);           // [GPS][DI] (QREG: unused)
    int4 *trec = reinterpret_cast<int4 *>(q_s + GPS * DI);                    // [W][4] tail blocks in flight
    float *q_w = reinterpret_cast<float *>(trec + W * 4);                     // [W][GPS][DI] (QREG: unused)
    long long *off = reinterpret_cast<long long *>(q_w + (QREG || MMA ? 0 : W * GPS * DI));  // [B+1] ranges' prefix
    long long *offt = off + a.B + 1;                                          // [B+1] tail pool prefix
    int *nbs = reinterpret_cast<int *>(offt + a.B + 1);                       // [B] blocks
    int *lens = nbs + a.B;                                                    // [B] clamped lengths
    int *nba = lens + a.B;                                                    // [B] blocks before the tail
    int *exh = nba + a.B;                                                     // [kTailPools] pool is empty
    int *arrived = exh + kTailPools;                                          // warps done with their pieces

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int B = a.B, Hik = a.Hik, Bk = a.Bk, C = a.n_cta;

    // per-sequence block counts and their prefix over (b, index-K head)
    for (int b = tid; b < B; b += blockDim.x) {
        int L = a.seq_lens[b];
        L = L < 0 ? 0 : (L > a.L_max ? a.L_max : L);
        lens[b] = L;
        nbs[b] = (L + Bk - 1) / Bk;
        nba[b] = nbs[b] - scan_tail_blocks(nbs[b]);
    }
    if (tid < kTailPools) exh[tid] = 0;
    if (tid == 0) *arrived = 0;
    if (tid < W * S) mbar_init(&bars[tid], 1);
    if (tid == 0) tc::prefetch_tmap(&kmap);
    fence_mbar_init();
    __syncthreads();
    if (w < 2) {
        // warp 0: prefix of the ranges' blocks (nba), warp 1: of the tails' blocks
        long long *dst = w == 0 ? off : offt;
        long long carry = 0;
        for (int b0 = 0; b0 < B; b0 += 32) {
            const int b = b0 + lane;
            long long v = b < B ? (long long)(w == 0 ? nba[b] : nbs[b] - nba[b]) * Hik : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const long long u = __shfl_up_sync(FULL, v, o);
                if (lane >= o) v += u;
            }
            if (b < B) dst[b + 1] = carry + v;
            carry += __shfl_sync(FULL, v, 31);
        }
        if (lane == 0) dst[0] = 0;
    }
    __syncthreads();
    const long long total = off[B];
    const long long per = total > 0 ? (total + C - 1) / C : 1;  // blocks per CTA
    long long x0 = per * blockIdx.x, x1 = x0 + per;
    x0 = x0 < total ? x0 : total;
    x1 = x1 < total ? x1 : total;

    if (blockIdx.x == 0 && a.counters != nullptr)
        for (int i = tid; i < B * a.G; i += blockDim.x) a.counters[i] = 0;  // the attention's split counters
    if (blockIdx.x == 0 && a.seg_info != nullptr) {
        for (int s = tid; s < B * Hik; s += blockDim.x) {
            const int b = s / Hik, h = s % Hik;
            SegInfo si{-1, 0};
            if (nba[b] > 0) {
                const long long st = off[b] + (long long)h * nba[b];
                si.first_cta = cta_of(st, per);
                si.n_pieces = cta_of(st + nba[b] - 1, per) - si.first_cta + 1;
            }
            a.seg_info[s] = si;
        }
    }
    // the next grid may start its prologue while this grid runs
    pdl_allow_next_grid();

    // the index query: the keys' type, or bf16 beside MXFP8 keys
    using QT = typename std::conditional<is_fp8<T>(), __nv_bfloat16, T>::type;
    const QT *qg = reinterpret_cast<const QT *>(a.q_idx);
    unsigned char *my_ring = ring + (size_t)w * S * kScanChunkBytes;
    unsigned char *my_sring = sring + (size_t)w * S * kScaleStage;
    uint64_t *my_bars = bars + w * S;
    const bool want_cand = a.cand_s != nullptr;
    const uint32_t chunk_bytes = (uint32_t)CT * ROWB;
    // the index keys are read once: evict-first in L2, so that the stream does not push out what
    // the attention kernel reads next (the lists, block scores and counters this kernel writes);
    // evict-normal for very long streams, whose own rate the hint lowers
    const uint64_t stream_pol = a.stream_evict_first ? l2_evict_first_policy() : l2_evict_normal_policy();

    // The shared tail (the last quarter of every stream's blocks): every warp takes tail blocks,
    // one at a time, until the pools are empty; a tail block leaves only its scores
    // (block_scores).  The pools hold the tail positions i * kTailPools + pool of the tails
    // concatenated over (b, index-K head); a warp turns to the next pool after each block.
    const long long total_t = a.sched != nullptr ? offt[B] : 0;
    int pool = (int)(((long long)blockIdx.x * W + w) % kTailPools);
    auto grab = [&]() -> long long {
        long long x = -1;
        if (lane == 0) {
            for (int t = 0; t < kTailPools && x < 0; ++t, pool = (pool + 1) % kTailPools) {
                if (*reinterpret_cast<volatile int *>(&exh[pool])) continue;
                const long long y = (long long)atomicAdd(&a.sched[pool], 1u) * kTailPools + pool;
                if (y < total_t)
                    x = y;
                else
                    *reinterpret_cast<volatile int *>(&exh[pool]) = 1;
            }
        }
        return __shfl_sync(FULL, x, 0);
    };
    // tail position -> (b, index-K head, block, chunks)
    auto locate = [&](long long x) -> int4 {
        int lo = 0, hi = B - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (offt[mid] <= x) lo = mid; else hi = mid - 1;
        }
        const int nt = nbs[lo] - nba[lo];
        const int r = (int)(x - offt[lo]);
        const int hik = r / nt;
        const int n = nba[lo] + (r - hik * nt);
        int bt = lens[lo] - n * Bk;
        bt = bt < Bk ? bt : Bk;
        return make_int4(lo, hik, n, (bt + CT - 1) / CT);
    };

    // One producer per warp (lane 0 issues, every lane tracks it to stay uniform) keeps the
    // warp's ring full: first the chunks of the warp's blocks of its CTA's range, then, with no
    // gap, chunks of tail blocks, so that the copies of the first tail blocks are in flight
    // while the range's last chunks are scored.
    ChunkCursor prod;
    prod.pw = PieceWalker{x0, x1};
    prod.w = w; prod.W = W; prod.Bk = Bk; prod.ct = CT;
    prod.start(off, nba, lens, B, Hik);
    bool failed = false;
    int issued = 0, consumed = 0;
    int4 *my_rec = trec + w * 4;  // tail blocks with chunks issued, in order (at most S + 1 live)
    int t_head = 0, t_tail = 0, pc = 0;
    bool more = total_t > 0, have = false;
    int4 pr = make_int4(0, 0, 0, 0);
    auto refill = [&]() {
        while (!failed && issued - consumed < S) {
            int row;
            if (prod.valid) {
                row = a.cache.row(prod.p.b, prod.p.hik, Hik, a.L_max, prod.n * Bk + prod.c * CT);
                prod.advance(off, nba, lens, B, Hik);
            } else {
                if (!more) break;
                if (!have) {
                    const long long x = grab();
                    if (x < 0) {
                        more = false;
                        break;
                    }
                    pr = locate(x);
                    if (lane == 0) my_rec[t_tail & 3] = pr;
                    __syncwarp();
                    ++t_tail;
                    have = true;
                    pc = 0;
                }
                row = a.cache.row(pr.x, pr.y, Hik, a.L_max, pr.z * Bk + pc * CT);
                if (++pc == pr.w) have = false;
            }
            if (lane == 0) {
                const int slot = issued % S;
                unsigned char *dst = my_ring + (size_t)slot * kScanChunkBytes;
                if constexpr (FP8) {
                    // the chunk's scales, clipped to the scale tensor (its row count is a multiple of 16,
                    // chunks start at multiples of 16 rows: whole 16-byte units)
                    const long long left = a.k_scale_rows - row;
                    const uint32_t sb = (uint32_t)((left < CT ? left : CT) * SPR);
                    mbar_arrive_expect_tx(&my_bars[slot], chunk_bytes + sb);
                    bulk_g2s(my_sring + (size_t)slot * kScaleStage, a.k_scale + (size_t)row * SPR, sb, &my_bars[slot],
                             l2_evict_first_policy());
                } else {
                    mbar_arrive_expect_tx(&my_bars[slot], chunk_bytes);
                }
                tc::tma_load_2d_hint(dst, &kmap, 0, row, &my_bars[slot], stream_pol);
                if constexpr (ROWB == 256)
                    tc::tma_load_2d_hint(dst + CT * 128, &kmap, 128 / ES, row, &my_bars[slot], stream_pol);
            }
            ++issued;
        }
    };
    refill();

    // B fragments of the groups' index queries (columns = the GPS groups of the stream, zero columns
    // up to 8; rows = index dims), loaded when the warp moves to another stream
    uint32_t qb[MMA ? KS : 1][2];
    auto load_qa = [&](int b, int hik) {
        if constexpr (MMA) {
            const int grp = lane >> 2, tig = lane & 3;
            const uint16_t *src = reinterpret_cast<const uint16_t *>(a.q_idx) +
                                  ((size_t)b * a.G + hik + (size_t)Hik * (grp < GPS ? grp : 0)) * DI;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                const int c0 = ks * 16 + tig * 2;
                qb[ks][0] = grp < GPS ? *reinterpret_cast<const uint32_t *>(src + c0) : 0u;
                qb[ks][1] = grp < GPS ? *reinterpret_cast<const uint32_t *>(src + c0 + 8) : 0u;
            }
        }
    };

    // one chunk of nt index-key rows of segment (b, hik) starting at token tok_base: fp32 dot
    // products with the index query (qv in registers, or qsrc in shared memory, or the qa
    // fragments on tensor cores), running max m
    auto scan_chunk = [&](const unsigned char *base, const unsigned char *sbase, int nt, int b, int hik, int tok_base,
                          const float *qv_, const float *qsrc, float *m) {
        if constexpr (MMA) {
            // S^T = K Q_idx^T, 16 keys (rows) by the 8 group columns per tile, so no MMA row is
            // padding; lane (grp, tig) holds the scores of keys grp and grp + 8 of each tile for
            // groups 2 tig and 2 tig + 1, and keeps their running maxima in m[0], m[1] (reduced
            // over the lanes at the block end).  Every tile's A fragments are loaded before its
            // MMAs; the tiles' accumulators are independent.
            constexpr int NKT = kScanChunkBytes / ROWB / 16;  // key tiles of a full chunk
            const uint32_t tile = smem_u32(base);
            const int grp = lane >> 2, tig = lane & 3;
            const int arow = (lane & 7) + ((lane >> 3) & 1) * 8, ahalf = lane >> 4;
            float sv[NKT][4];
#pragma unroll
            for (int kt = 0; kt < NKT; ++kt) {
                sv[kt][0] = sv[kt][1] = sv[kt][2] = sv[kt][3] = 0.f;
                if (kt * 16 < nt) {
                    uint32_t af[KS][4];
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks) {
                        const int d0 = ks * 16 + ahalf * 8;
                        ldsm_x4(tile + (d0 >> 6) * (CT * 128) + sw128(kt * 16 + arow, (d0 & 63) >> 3), af[ks][0], af[ks][1],
                                af[ks][2], af[ks][3]);
                    }
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks) mma_16816_pure(sv[kt], af[ks], qb[ks][0], qb[ks][1]);
                }
            }
            float c0 = m[0], c1 = m[1];
#pragma unroll
            for (int kt = 0; kt < NKT; ++kt) {
                const int k0 = kt * 16 + grp, k1 = k0 + 8;
                const bool v0 = k0 < nt && !failed, v1 = k1 < nt && !failed;
                c0 = tc::fmax3(c0, v0 ? sv[kt][0] : -INFINITY, v1 ? sv[kt][2] : -INFINITY);
                c1 = tc::fmax3(c1, v0 ? sv[kt][1] : -INFINITY, v1 ? sv[kt][3] : -INFINITY);
                if (a.token_scores != nullptr && !failed) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int gl = 2 * tig + h;
                        if (gl < GPS) {
                            float *ts = a.token_scores + ((size_t)b * a.G + hik + Hik * gl) * a.L_max + tok_base;
                            if (v0) ts[k0] = sv[kt][h];
                            if (v1) ts[k1] = sv[kt][2 + h];
                        }
                    }
                }
            }
            m[0] = c0;
            m[1] = c1;
        } else {
            for (int t0 = 0; t0 < nt; t0 += 32) {
                const int tok = t0 + lane;  // one index-key row per lane
                const bool live = tok < nt && !failed;
                float dot[GPS];
#pragma unroll
                for (int gl = 0; gl < GPS; ++gl) dot[gl] = 0.f;
                // position of 16-byte vector c16 of row `tok` in the swizzled tile
                auto vec_at = [&](int c16) -> uint4 {
                    int o;
                    if constexpr (ROWB == 64) {
                        o = tok * 64 + ((c16 ^ ((tok >> 1) & 3)) << 4);
                    } else {
                        o = (c16 >> 3) * (CT * 128) + tok * 128 + (((c16 & 7) ^ (tok & 7)) << 4);
                    }
                    return *reinterpret_cast<const uint4 *>(base + o);
                };
                if (live && FP8) {
                    // per 32 dims (two vectors): the code products, then their E8M0 scale
#pragma unroll
                    for (int j = 0; j < (FP8 ? SPR : 1); ++j) {
                        const float sc = e8m0_to_float(sbase[tok * SPR + j]);
                        float part[GPS];
#pragma unroll
                        for (int gl = 0; gl < GPS; ++gl) part[gl] = 0.f;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int c16 = 2 * j + h;
                            float f[EPV];
                            Vec16<T>::unpack(vec_at(c16), f);
                            if constexpr (QREG) {
#pragma unroll
                                for (int e = 0; e < EPV; ++e) part[0] = fmaf(qv_[c16 * EPV + e], f[e], part[0]);
                            } else {
#pragma unroll
                                for (int gl = 0; gl < GPS; ++gl) {
                                    const float *qq = qsrc + gl * DI + c16 * EPV;
#pragma unroll
                                    for (int e = 0; e < EPV; ++e) part[gl] = fmaf(qq[e], f[e], part[gl]);
                                }
                            }
                        }
#pragma unroll
                        for (int gl = 0; gl < GPS; ++gl) dot[gl] = fmaf(sc, part[gl], dot[gl]);
                    }
                } else if (live) {
#pragma unroll
                    for (int c16 = 0; c16 < NCH; ++c16) {
                        const uint4 u = vec_at(c16);
                        float f[EPV];
                        Vec16<T>::unpack(u, f);
                        if constexpr (QREG) {
#pragma unroll
                            for (int e = 0; e < EPV; ++e) dot[0] = fmaf(qv_[c16 * EPV + e], f[e], dot[0]);
                        } else {
#pragma unroll
                            for (int gl = 0; gl < GPS; ++gl) {
                                const float *qq = qsrc + gl * DI + c16 * EPV;
#pragma unroll
                                for (int e = 0; e < EPV; ++e) dot[gl] = fmaf(qq[e], f[e], dot[gl]);
                            }
                        }
                    }
                }
#pragma unroll
                for (int gl = 0; gl < GPS; ++gl) {
                    const float sc = live ? dot[gl] : -INFINITY;
                    m[gl] = fmaxf(m[gl], sc);
                    if (a.token_scores != nullptr && live) {
                        const int g = hik + Hik * gl;
                        a.token_scores[((size_t)b * a.G + g) * a.L_max + tok_base + tok] = sc;
                    }
                }
            }
        }
    };

    // every lane ends with the block's max of each group: a butterfly over the lanes, or, with
    // tensor-core scores (the 8 lanes of one tig hold groups 2 tig and 2 tig + 1), a reduction
    // over those 8 lanes and one broadcast per group
    auto block_max = [&](float *m) {
        if constexpr (MMA) {
            float c0 = m[0], c1 = m[1];
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                c0 = fmaxf(c0, __shfl_xor_sync(FULL, c0, o));
                c1 = fmaxf(c1, __shfl_xor_sync(FULL, c1, o));
            }
#pragma unroll
            for (int gl = 0; gl < GPS; ++gl) m[gl] = __shfl_sync(FULL, (gl & 1) ? c1 : c0, gl >> 1);
        } else {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int gl = 0; gl < GPS; ++gl) m[gl] = fmaxf(m[gl], __shfl_xor_sync(FULL, m[gl], o));
        }
    };

    float qv[QREG ? DI : 1];
    int q_b = -1, q_h = -1;
    WarpTopK lst[GPS];
    bool merged = false;
    int def_seg = -1, def_piece = 0;  // the piece whose merge waits for the kernel's end
    // group w's W lists pairwise, the pairs' results pairwise, ... (a tree of top-32 merges
    // whose merges of one level are independent) into the candidates of piece `piece` of
    // segment `seg`
    auto merge_piece = [&](int seg, int piece) {
        const int gl = GPS == 1 ? 0 : w;
        unsigned long long key[W];
#pragma unroll
        for (int j = 0; j < W; ++j)
            key[j] = sel_key(lists_s[(j * GPS + gl) * 32 + lane], lists_i[(j * GPS + gl) * 32 + lane]);
#pragma unroll
        for (int st = 1; st < W; st *= 2)
#pragma unroll
            for (int j = 0; j + st < W; j += 2 * st) key[j] = warp_merge_top32(key[j], key[j + st], lane);
        const size_t o = (((size_t)seg * C + piece) * GPS + gl) * a.k;
        if (lane < a.k) sel_unkey(key[0], a.cand_s[o + lane], a.cand_i[o + lane]);
    };
    PieceWalker pw{x0, x1};
    Piece p;
    while (pw.next(off, nba, B, Hik, p)) {
        if (p.b != q_b || p.hik != q_h) {
            q_b = p.b; q_h = p.hik;
            if constexpr (QREG) {
                const QT *src = qg + ((size_t)p.b * a.G + p.hik) * DI;
#pragma unroll
                for (int e = 0; e < DI; ++e) qv[e] = load_elem(src + e);
            } else if constexpr (MMA) {
                load_qa(p.b, p.hik);
            } else {
                __syncthreads();  // every warp is done with the previous segment's query
                for (int i = tid; i < GPS * DI; i += blockDim.x) {
                    const int g = p.hik + Hik * (i / DI);
                    q_s[i] = load_elem(qg + ((size_t)p.b * a.G + g) * DI + i % DI);
                }
                __syncthreads();
            }
        }
#pragma unroll
        for (int gl = 0; gl < GPS; ++gl) lst[gl].reset();
        const int L = lens[p.b];
        for (int n = p.n0 + w; n < p.n1; n += W) {
            int bt = L - n * Bk;
            bt = bt < Bk ? bt : Bk;
            const int nch = (bt + CT - 1) / CT;
            float m[GPS];
#pragma unroll
            for (int gl = 0; gl < GPS; ++gl) m[gl] = -INFINITY;
            for (int c = 0; c < nch; ++c) {
                const int slot = consumed % S;
                const uint32_t parity = (consumed / S) & 1;
                if (!failed && !mbar_wait(&my_bars[slot], parity, a.status)) {
                    // give up: wait (bounded) for this warp's copies still in flight, then
                    // run the loop to its end without waiting or issuing again
                    failed = true;
                    for (int q2 = consumed; q2 < issued; ++q2) mbar_wait(&my_bars[q2 % S], (q2 / S) & 1, nullptr);
                }
                int nt = bt - c * CT;
                nt = nt < CT ? nt : CT;
                scan_chunk(my_ring + (size_t)slot * kScanChunkBytes, my_sring + (size_t)slot * kScaleStage, nt, p.b, p.hik,
                           n * Bk + c * CT, qv, q_s, m);
                __syncwarp();
                ++consumed;
                refill();
            }
            block_max(m);
            if (a.block_scores != nullptr && lane == 0)
#pragma unroll
                for (int gl = 0; gl < GPS; ++gl)
                    a.block_scores[((size_t)p.b * a.G + p.hik + Hik * gl) * a.nb_max + n] = m[gl];
            if (want_cand) warp_topk_insert_all<GPS>(lst, m, n, a.k, lane);
        }
        if (want_cand) {
            // The warps' sorted lists of this piece merge into its candidates.  One group: the
            // warp that finishes last merges them, and no warp waits for another.  Several
            // groups: one warp per group, after every warp is done; for the CTA's last piece
            // that is at the kernel's end, so that no warp waits before it goes on to the tail.
            if (merged) __syncthreads();  // the previous piece's merge has read the lists
#pragma unroll
            for (int gl = 0; gl < GPS; ++gl) {
                lists_s[(w * GPS + gl) * 32 + lane] = lst[gl].s;
                lists_i[(w * GPS + gl) * 32 + lane] = lst[gl].id;
            }
            const int seg = p.b * Hik + p.hik;
            const int piece = blockIdx.x - cta_of(p.seg_start, per);
            if constexpr (GPS == 1) {
                __syncwarp();
                int ticket = 0;
                if (lane == 0) {
                    __threadfence_block();  // this warp's list before its arrival
                    ticket = atomicAdd(arrived, 1);
                }
                ticket = __shfl_sync(FULL, ticket, 0);
                if (ticket % W == W - 1) {
                    __threadfence_block();  // every warp's list after their arrivals
                    merge_piece(seg, piece);
                }
                merged = true;
            } else if (pw.x >= pw.x1) {
                def_seg = seg;
                def_piece = piece;
            } else {
                __syncthreads();
                if (w < GPS) merge_piece(seg, piece);
                merged = true;
            }
        }
    }

    // ------------------------------------------------ the shared tail, one block at a time
    {
        float *my_q = q_w + (QREG || MMA ? 0 : w * GPS * DI);
        int qb = -1, qh = -1;
        refill();
        while (t_head < t_tail) {
            const int4 r = my_rec[t_head & 3];
            if (r.x != qb || r.y != qh) {
                qb = r.x;
                qh = r.y;
                if constexpr (QREG) {
                    const QT *src = qg + ((size_t)qb * a.G + qh) * DI;
#pragma unroll
                    for (int e = 0; e < DI; ++e) qv[e] = load_elem(src + e);
                } else if constexpr (MMA) {
                    load_qa(qb, qh);
                } else {
                    __syncwarp();
                    for (int i = lane; i < GPS * DI; i += 32) {
                        const int g = qh + Hik * (i / DI);
                        my_q[i] = load_elem(qg + ((size_t)qb * a.G + g) * DI + i % DI);
                    }
                    __syncwarp();
                }
            }
            int bt = lens[r.x] - r.z * Bk;
            bt = bt < Bk ? bt : Bk;
            float m[GPS];
#pragma unroll
            for (int gl = 0; gl < GPS; ++gl) m[gl] = -INFINITY;
            for (int c = 0; c < r.w; ++c) {
                const int slot = consumed % S;
                if (!failed && !mbar_wait(&my_bars[slot], (consumed / S) & 1, a.status)) {
                    failed = true;
                    for (int q2 = consumed; q2 < issued; ++q2) mbar_wait(&my_bars[q2 % S], (q2 / S) & 1, nullptr);
                }
                int nt = bt - c * CT;
                nt = nt < CT ? nt : CT;
                scan_chunk(my_ring + (size_t)slot * kScanChunkBytes, my_sring + (size_t)slot * kScaleStage, nt, r.x, r.y,
                           r.z * Bk + c * CT, qv, my_q, m);
                __syncwarp();
                ++consumed;
                refill();
            }
            block_max(m);
            if (a.block_scores != nullptr && lane == 0)
#pragma unroll
                for (int gl = 0; gl < GPS; ++gl)
                    a.block_scores[((size_t)r.x * a.G + r.y + Hik * gl) * a.nb_max + r.z] = m[gl];
            ++t_head;
            refill();
        }
    }

    __syncthreads();
    if (def_seg >= 0 && w < GPS) merge_piece(def_seg, def_piece);
    // the CTA that finishes last returns the pool counters to zero for the next call
    if (a.sched != nullptr && tid == 0) {
        __threadfence();
        if (atomicAdd(&a.sched[kTailPools], 1u) == gridDim.x - 1) {
            for (int i = 0; i < kTailPools; ++i) a.sched[i] = 0;
            __threadfence();
            a.sched[kTailPools] = 0;
        }
    }
}

__global__ void fill_neg_inf_kernel(const FillArgs a) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < a.n; i += (long long)gridDim.x * blockDim.x)
        a.scores[i] = -INFINITY;
}

template <typename T, int GPS, int ROWB, int S, int W>
size_t scan_smem_bytes(int B) {
    constexpr bool MMA = scan_mma<T, GPS, ROWB>();
    constexpr int DI = ROWB / (int)sizeof(T);
    constexpr bool QREG = GPS == 1 && DI <= 64;
    return 1024 + (size_t)W * S * kScanChunkBytes + (is_fp8<T>() ? (size_t)W * S * kScaleStage : 0) + W * S * 8 +
           (size_t)W * GPS * 32 * 8 + (size_t)GPS * DI * 4 +
           (size_t)W * 4 * 16 + (QREG || MMA ? 0 : (size_t)W * GPS * DI * 4) + (size_t)(B + 1) * 16 + (size_t)B * 12 +
           kTailPools * 4 + 4 + 64;
}

template <typename T, int GPS, int ROWB, int S, int W>
cudaError_t launch_scan_s(const ScanArgs &a, const CUtensorMap &km, cudaStream_t s, bool pdl) {
    const size_t smem = scan_smem_bytes<T, GPS, ROWB, S, W>(a.B);
    static size_t attr_bytes = 0;  // opt-in raised on demand (smem grows with the batch)
    if (smem > attr_bytes) {
        cudaError_t e = cudaFuncSetAttribute(decode_scan_kernel<T, GPS, ROWB, S, W>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_bytes = smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.n_cta);
    cfg.blockDim = dim3(W * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode_scan_kernel<T, GPS, ROWB, S, W>, km, a);
}

template <typename T, int GPS, int ROWB>
cudaError_t launch_scan_t(const ScanArgs &a, const CUtensorMap &km, cudaStream_t s, bool pdl) {
    if constexpr (GPS == 1) {
        return launch_scan_s<T, GPS, ROWB, 2, 12>(a, km, s, pdl);
    } else {
        if constexpr (scan_mma<T, GPS, ROWB>()) {
            if (scan_smem_bytes<T, GPS, ROWB, 3, 8>(a.B) <= 232448) return launch_scan_s<T, GPS, ROWB, 3, 8>(a, km, s, pdl);
        }
        return launch_scan_s<T, GPS, ROWB, 2, 8>(a, km, s, pdl);
    }
}

template <typename T, int ROWB>
cudaError_t launch_scan_g(const ScanArgs &a, const CUtensorMap &km, int gps, cudaStream_t s, bool pdl) {
    switch (gps) {
        case 1: return launch_scan_t<T, 1, ROWB>(a, km, s, pdl);
        case 2: return launch_scan_t<T, 2, ROWB>(a, km, s, pdl);
        case 4: return launch_scan_t<T, 4, ROWB>(a, km, s, pdl);
        case 8: return launch_scan_t<T, 8, ROWB>(a, km, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t launch_scan_r(const ScanArgs &a, const CUtensorMap &km, int rowb, int gps, cudaStream_t s, bool pdl) {
    switch (rowb) {
        case 64: return launch_scan_g<T, 64>(a, km, gps, s, pdl);
        case 128: return launch_scan_g<T, 128>(a, km, gps, s, pdl);
        case 256: return launch_scan_g<T, 256>(a, km, gps, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

// Streams up to this many bytes (the index-key cache's rows times the row size) load evict-first:
// measured on B200, the hint kept the attention kernel's inputs in L2 and shortened the 1 GB
// decode steps by 1-4 us, and slowed a 4.3 GB scan (batch 4 at 1M) by 3 %.
constexpr double kEvictFirstMaxBytes = 2147483648.0;

cudaError_t launch_decode_scan(ScanArgs a, int dtype, int row_bytes, int gps, cudaStream_t s, bool pdl) {
    a.stream_evict_first = (double)a.cache.rows(a.B, a.Hik, a.L_max) * row_bytes <= kEvictFirstMaxBytes;
    // MXFP8 keys (a.k_scale set): one byte per index dim
    const bool fp8 = a.k_scale != nullptr;
    const int es = fp8 ? 1 : dtype == MSA_F32 ? 4 : 2;
    int ct = kScanChunkBytes / row_bytes;
    if (ct > a.Bk) ct = a.Bk;
    a.chunk_tokens = ct;
    // index keys as a 2D tensor [B * Hik * Lmax rows, di]; one box = ct rows x 128 bytes
    // (64 for 64-byte rows), swizzled so that one lane per row reads without bank conflicts
    const int box_x = (row_bytes >= 128 ? 128 : 64) / es;
    CUtensorMap km;
    const CUtensorMapDataType ty = fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                   : dtype == MSA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!encode_2d(&km, ty, const_cast<void *>(a.k_idx), row_bytes / es, a.cache.rows(a.B, a.Hik, a.L_max), row_bytes,
                   box_x, ct, row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (fp8) return launch_scan_r<e4m3_t>(a, km, row_bytes, gps, s, pdl);
    return dtype == MSA_F32 ? launch_scan_r<float>(a, km, row_bytes, gps, s, pdl)
                            : launch_scan_r<__nv_bfloat16>(a, km, row_bytes, gps, s, pdl);
}

cudaError_t launch_fill_neg_inf(float *p, long long n, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    long long blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    fill_neg_inf_kernel<<<(unsigned)blocks, 256, 0, s>>>(FillArgs{p, n});
    return cudaGetLastError();
}

}  // namespace msa
