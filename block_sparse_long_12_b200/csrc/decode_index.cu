// Step 1 of MSA for decode: index scores, block max pool, per-piece TopK.
//
// Page "MiniMax wird duenn" (atlascloud.ai), section 1, Step 1: the group's
// index query scores every cached token against its index key, the scores
// are max-pooled per fixed-size block, and TopK keeps the best blocks of the
// group.  For decode this is a single query against the whole cache, so the
// kernel is a stream of k_idx from HBM: each byte is read once.
//
// Work split: the index-K streams of all (sequence b, index-K head) pairs are
// concatenated (block granularity) and cut into n_cta ranges of equal length
// (the last one shorter), one per persistent CTA (one CTA per SM), so ragged
// lengths stay balanced.  Inside a
// CTA every warp owns a private ring of kScanStages 8 KB shared-memory stages
// filled by TMA bulk copies (cp.async.bulk, L2 evict-first) and consumes the
// blocks w, w+8, ... of the CTA's range.  For one 16-byte vector of a key row
// a lane does the fp32 dot-product part against its slice of the index query
// (held in registers); a butterfly over the lanes of the row completes the
// token score, a running max gives the block score, and a warp-distributed
// sorted list keeps the warp's best blocks.  At the end of each piece the
// eight warp lists are merged into one sorted candidate list per group; the
// attention kernel merges the pieces of a segment into the final TopK.
#include "msa_device.cuh"

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
    int w, Bk, row_bytes, ct;  // ct = tokens per chunk
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
        n += kScanWarps;
        if (n < p.n1) {
            c = 0;
            nch = (block_tokens(lens) + ct - 1) / ct;
            return;
        }
        valid = next_piece(off, nbs, lens, B, Hik);
    }
};

template <typename T, int GPS, int LPT>
__global__ void __launch_bounds__(kScanWarps * 32, 1) decode_scan_kernel(const ScanArgs a) {
    constexpr int EPV = Vec16<T>::N;          // elements per 16-byte vector
    constexpr int ROW = LPT * 16;             // bytes per index-key row
    constexpr int CT = kScanChunkBytes / ROW; // tokens per chunk
    constexpr int TPI = 32 / LPT;             // tokens per warp step

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *ring = smem;                                             // [W][S][chunk]
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring + (size_t)kScanWarps * kScanStages * kScanChunkBytes);
    float *lists_s = reinterpret_cast<float *>(bars + kScanWarps * kScanStages); // [W][GPS][32]
    int *lists_i = reinterpret_cast<int *>(lists_s + kScanWarps * GPS * 32);
    long long *off = reinterpret_cast<long long *>(lists_i + kScanWarps * GPS * 32); // [B+1]
    int *nbs = reinterpret_cast<int *>(off + a.B + 1);                   // [B]
    int *lens = nbs + a.B;                                               // [B] clamped lengths

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int B = a.B, Hik = a.Hik, Bk = a.Bk, C = a.n_cta;

    // per-sequence block counts and their prefix over (b, index-K head)
    for (int b = tid; b < B; b += blockDim.x) {
        int L = a.seq_lens[b];
        L = L < 0 ? 0 : (L > a.L_max ? a.L_max : L);
        lens[b] = L;
        nbs[b] = (L + Bk - 1) / Bk;
    }
    if (tid < kScanWarps * kScanStages) mbar_init(&bars[tid], 1);
    fence_mbar_init();
    __syncthreads();
    if (w == 0) {
        long long carry = 0;
        for (int b0 = 0; b0 < B; b0 += 32) {
            const int b = b0 + lane;
            long long v = b < B ? (long long)nbs[b] * Hik : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const long long u = __shfl_up_sync(FULL, v, o);
                if (lane >= o) v += u;
            }
            if (b < B) off[b + 1] = carry + v;
            carry += __shfl_sync(FULL, v, 31);
        }
        if (lane == 0) off[0] = 0;
    }
    __syncthreads();
    const long long total = off[B];
    const long long per = total > 0 ? (total + C - 1) / C : 1;  // blocks per CTA
    long long x0 = per * blockIdx.x, x1 = x0 + per;
    x0 = x0 < total ? x0 : total;
    x1 = x1 < total ? x1 : total;

    if (blockIdx.x == 0 && a.seg_info != nullptr) {
        for (int s = tid; s < B * Hik; s += blockDim.x) {
            const int b = s / Hik, h = s % Hik;
            SegInfo si{-1, 0};
            if (nbs[b] > 0) {
                const long long st = off[b] + (long long)h * nbs[b];
                si.first_cta = cta_of(st, per);
                si.n_pieces = cta_of(st + nbs[b] - 1, per) - si.first_cta + 1;
            }
            a.seg_info[s] = si;
        }
    }
    // the attention grid may start its prologue while this grid runs
    pdl_allow_next_grid();

    const T *qg = reinterpret_cast<const T *>(a.q_idx);
    const unsigned char *kg = reinterpret_cast<const unsigned char *>(a.k_idx);
    const uint64_t pol = l2_evict_first_policy();
    unsigned char *my_ring = ring + (size_t)w * kScanStages * kScanChunkBytes;
    uint64_t *my_bars = bars + w * kScanStages;
    const bool want_cand = a.cand_s != nullptr;

    // producer cursor (lane 0 issues, every lane tracks it to stay uniform)
    ChunkCursor prod;
    prod.pw = PieceWalker{x0, x1};
    prod.w = w; prod.Bk = Bk; prod.row_bytes = ROW; prod.ct = CT;
    prod.start(off, nbs, lens, B, Hik);
    bool failed = false;
    int issued = 0;
    auto issue = [&](int slot) {
        const int tok0 = prod.n * Bk + prod.c * CT;
        int nt = lens[prod.p.b] - tok0;
        nt = nt < CT ? nt : CT;
        if (nt > Bk - prod.c * CT) nt = Bk - prod.c * CT;
        const uint32_t bytes = (uint32_t)nt * ROW;
        if (lane == 0) {
            const unsigned char *src =
                kg + (((size_t)prod.p.b * Hik + prod.p.hik) * (size_t)a.L_max + (size_t)tok0) * ROW;
            mbar_arrive_expect_tx(&my_bars[slot], bytes);
            bulk_g2s(my_ring + (size_t)slot * kScanChunkBytes, src, bytes, &my_bars[slot], pol);
        }
        ++issued;
        prod.advance(off, nbs, lens, B, Hik);
    };
    for (int s = 0; s < kScanStages && prod.valid; ++s) issue(s);

    int consumed = 0;
    float qv[GPS][EPV];
    int q_b = -1, q_h = -1;
    WarpTopK lst[GPS];
    PieceWalker pw{x0, x1};
    Piece p;
    while (pw.next(off, nbs, B, Hik, p)) {
        if (p.b != q_b || p.hik != q_h) {
            q_b = p.b; q_h = p.hik;
#pragma unroll
            for (int gl = 0; gl < GPS; ++gl) {
                const int g = p.hik + Hik * gl;
                const T *src = qg + ((size_t)p.b * a.G + g) * a.di + (lane % LPT) * EPV;
#pragma unroll
                for (int e = 0; e < EPV; ++e) qv[gl][e] = load_elem(src + e);
            }
        }
#pragma unroll
        for (int gl = 0; gl < GPS; ++gl) lst[gl].reset();
        const int L = lens[p.b];
        for (int n = p.n0 + w; n < p.n1; n += kScanWarps) {
            int bt = L - n * Bk;
            bt = bt < Bk ? bt : Bk;
            const int nch = (bt + CT - 1) / CT;
            float m[GPS];
#pragma unroll
            for (int gl = 0; gl < GPS; ++gl) m[gl] = -INFINITY;
            for (int c = 0; c < nch; ++c) {
                const int slot = consumed % kScanStages;
                const uint32_t parity = (consumed / kScanStages) & 1;
                if (!failed && !mbar_wait(&my_bars[slot], parity, a.status)) {
                    // give up: wait (bounded) for this warp's copies still in flight, then
                    // run the loop to its end without waiting or issuing again
                    failed = true;
                    for (int q2 = consumed + 1; q2 < issued; ++q2)
                        mbar_wait(&my_bars[q2 % kScanStages], (q2 / kScanStages) & 1, nullptr);
                }
                int nt = bt - c * CT;
                nt = nt < CT ? nt : CT;
                const unsigned char *base = my_ring + (size_t)slot * kScanChunkBytes;
                const int tok_base = n * Bk + c * CT;
#pragma unroll 4
                for (int it = 0; it < CT / TPI; ++it) {
                    const int tok = it * TPI + lane / LPT;
                    const bool live = tok < nt && !failed;
                    float dot[GPS];
#pragma unroll
                    for (int gl = 0; gl < GPS; ++gl) dot[gl] = 0.f;
                    if (live) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(base + tok * ROW + (lane % LPT) * 16);
                        float f[EPV];
                        Vec16<T>::unpack(u, f);
#pragma unroll
                        for (int gl = 0; gl < GPS; ++gl)
#pragma unroll
                            for (int e = 0; e < EPV; ++e) dot[gl] = fmaf(qv[gl][e], f[e], dot[gl]);
                    }
#pragma unroll
                    for (int o = LPT / 2; o > 0; o >>= 1)
#pragma unroll
                        for (int gl = 0; gl < GPS; ++gl) dot[gl] += __shfl_xor_sync(FULL, dot[gl], o);
#pragma unroll
                    for (int gl = 0; gl < GPS; ++gl) {
                        const float sc = live ? dot[gl] : -INFINITY;
                        m[gl] = fmaxf(m[gl], sc);
                        if (a.token_scores != nullptr && live && (lane % LPT) == 0) {
                            const int g = p.hik + Hik * gl;
                            a.token_scores[((size_t)p.b * a.G + g) * a.L_max + tok_base + tok] = sc;
                        }
                    }
                }
                __syncwarp();
                ++consumed;
                if (prod.valid && !failed) issue(slot);
            }
#pragma unroll
            for (int o = LPT; o < 32; o <<= 1)
#pragma unroll
                for (int gl = 0; gl < GPS; ++gl) m[gl] = fmaxf(m[gl], __shfl_xor_sync(FULL, m[gl], o));
#pragma unroll
            for (int gl = 0; gl < GPS; ++gl) {
                if (a.block_scores != nullptr && lane == 0) {
                    const int g = p.hik + Hik * gl;
                    a.block_scores[((size_t)p.b * a.G + g) * a.nb_max + n] = m[gl];
                }
                if (want_cand) lst[gl].insert(m[gl], n, a.k, lane);
            }
        }
        if (want_cand) {
            // merge the warps' sorted lists into this piece's candidates
#pragma unroll
            for (int gl = 0; gl < GPS; ++gl) {
                lists_s[(w * GPS + gl) * 32 + lane] = lst[gl].s;
                lists_i[(w * GPS + gl) * 32 + lane] = lst[gl].id;
            }
            __syncthreads();
            if (w < GPS) {
                const int gl = w;
                const int seg = p.b * Hik + p.hik;
                const int piece = blockIdx.x - cta_of(p.seg_start, per);
                const size_t o = (((size_t)seg * C + piece) * GPS + gl) * a.k;
                warp_merge_sorted_lists<1>(lists_s + gl * 32, lists_i + gl * 32, kScanWarps, a.k, GPS * 32, a.k,
                                           a.cand_s + o, a.cand_i + o, lane);
            }
            __syncthreads();
        }
    }
}

__global__ void fill_neg_inf_kernel(const FillArgs a) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < a.n; i += (long long)gridDim.x * blockDim.x)
        a.scores[i] = -INFINITY;
}

template <typename T, int GPS, int LPT>
cudaError_t launch_scan_t(const ScanArgs &a, cudaStream_t s, bool pdl) {
    const size_t smem = (size_t)kScanWarps * kScanStages * kScanChunkBytes + kScanWarps * kScanStages * 8 +
                        (size_t)kScanWarps * GPS * 32 * 8 + (size_t)(a.B + 1) * 8 + (size_t)a.B * 8;
    static size_t attr_bytes = 0;  // opt-in raised on demand (smem grows with the batch)
    if (smem > attr_bytes) {
        cudaError_t e = cudaFuncSetAttribute(decode_scan_kernel<T, GPS, LPT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_bytes = smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.n_cta);
    cfg.blockDim = dim3(kScanWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode_scan_kernel<T, GPS, LPT>, a);
}

template <typename T, int LPT>
cudaError_t launch_scan_g(const ScanArgs &a, int gps, cudaStream_t s, bool pdl) {
    switch (gps) {
        case 1: return launch_scan_t<T, 1, LPT>(a, s, pdl);
        case 2: return launch_scan_t<T, 2, LPT>(a, s, pdl);
        case 4: return launch_scan_t<T, 4, LPT>(a, s, pdl);
        case 8: return launch_scan_t<T, 8, LPT>(a, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t launch_scan_l(const ScanArgs &a, int lpt, int gps, cudaStream_t s, bool pdl) {
    switch (lpt) {
        case 4: return launch_scan_g<T, 4>(a, gps, s, pdl);
        case 8: return launch_scan_g<T, 8>(a, gps, s, pdl);
        case 16: return launch_scan_g<T, 16>(a, gps, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode_scan(const ScanArgs &a, int dtype, int lpt, int gps, cudaStream_t s, bool pdl) {
    return dtype == MSA_F32 ? launch_scan_l<float>(a, lpt, gps, s, pdl)
                            : launch_scan_l<__nv_bfloat16>(a, lpt, gps, s, pdl);
}

cudaError_t launch_fill_neg_inf(float *p, long long n, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    long long blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    fill_neg_inf_kernel<<<(unsigned)blocks, 256, 0, s>>>(FillArgs{p, n});
    return cudaGetLastError();
}

}  // namespace msa
