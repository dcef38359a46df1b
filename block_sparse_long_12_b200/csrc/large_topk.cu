// Steps 1b + 1c of MSA for large k (more blocks than a warp-distributed list holds): the k best
// block scores of every row.
//
// Page "MiniMax wird duenn" (atlascloud.ai), section 1, Step 1: block scores (the block maxima
// of the index scores) go through TopK per group.  Section 3 back-calculates that a query
// touches about 6-7 % of the blocks at 1M tokens (k near 1000 of 16,384 blocks of 64 tokens),
// far beyond what per-warp sorted lists hold.  One CTA per row forms every block's 64-bit key
// (the score's order-preserving bits above the complemented id: all distinct, ordered as the
// selection), finds the k-th largest key exactly by a radix select (a shared histogram per pass:
// digits of 12, 12 and 8 bits over the score bits, the same over the id bits only when blocks tie
// at the k-th score), takes the k keys at or above it and sorts them once (bitonic).  Rows of
// up to 16,384 blocks keep their keys in registers; longer rows re-read the scores from global
// memory in every pass (L2 keeps them).  Prefill rows with k up to 256 take one warp per row
// instead (warp_topk_kernel).
#include "msa_device.cuh"

namespace msa {

namespace {

constexpr int kLargeThreads = 1024;  // = kMaxTopK: one sorted slot per thread

// order-preserving image of a float: larger score, larger unsigned value (-0 taken as +0)
__device__ inline uint32_t score_bits(float v) {
    const uint32_t u = __float_as_uint(v + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ inline float bits_score(uint32_t u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// Inclusive sum over the CTA of one value per thread; `tot` receives the total.
__device__ inline int block_inclusive_sum(int v, int *warp_sums, int &tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(FULL, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) warp_sums[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int x = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(FULL, x, o);
            if (lane >= o) x += u;
        }
        if (lane < nw) warp_sums[lane] = x;
    }
    __syncthreads();
    tot = warp_sums[nw - 1];
    const int before = warp > 0 ? warp_sums[warp - 1] : 0;
    __syncthreads();  // warp_sums free again
    return v + before;
}

constexpr int kHistBins = 4096;  // the widest digit: 12 bits

__global__ void __launch_bounds__(kLargeThreads) large_topk_kernel(const LargeTopkArgs a) {
    constexpr int KPT = 16;  // keys per thread held in registers (rows of up to 16,384 blocks)
    __shared__ unsigned hist[kHistBins];
    __shared__ int warp_sums[32];
    __shared__ unsigned long long keys[kMaxTopK];
    __shared__ int st[4];  // [0] chosen digit, [1] remaining rank, [2] taken blocks, [3] prefix all taken
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nthr = blockDim.x;
    const int row = blockIdx.x;
    const int t = (row / a.G) % a.q_len, b = row / (a.G * a.q_len);
    int pos;
    if (a.prefill) {
        pos = a.q_start + t;
    } else {
        int L = a.seq_lens[b];
        L = L < 0 ? 0 : (L > a.L_max ? a.L_max : L);
        pos = L - 1;
    }
    if (pos >= a.L_max) pos = a.L_max - 1;
    const int nb = pos >= 0 ? pos / a.Bk + 1 : 0;
    const int kk = a.k < nb ? a.k : nb;
    const float *src = a.scores + (size_t)row * a.stride;
    // the selection key of block n: score bits above the complemented id, so that keys are
    // distinct and their order is the selection order (higher score, then lower id)
    auto key_of = [&](int n) -> unsigned long long {
        // MSA_FORCE_SINK_LOCAL: block 0 and the row's own block rank above every score
        const float v = (a.force && (n == 0 || n == nb - 1)) ? INFINITY : src[n];
        return ((unsigned long long)score_bits(v) << 32) | (uint32_t)~(uint32_t)n;
    };
    const bool in_regs = nb <= KPT * nthr;
    unsigned long long kr[KPT];
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const int n = tid + j * nthr;
        kr[j] = (in_regs && n < nb) ? key_of(n) : 0ull;
    }

    // the kk-th largest key T (exactly): digits of 12, 12 and 8 bits from the top, first over the
    // score bits, then over the id bits when the k-th score is tied.  12-bit digits spread the
    // first pass (sign, exponent and 3 mantissa bits) over more bins than 8 would.
    unsigned long long prefix = 0, mask = 0;
    int rem = kk;  // rank of T among the keys that match the prefix so far
    if (kk < nb) {
#pragma unroll 1
        for (int ps = 0; ps < 6; ++ps) {
            // passes 0-2: bits 63-52, 51-40, 39-32 (score); passes 3-5: bits 31-20, 19-8, 7-0 (id)
            const int within = ps % 3;
            const int shift = 32 * (1 - ps / 3) + (within == 0 ? 20 : within == 1 ? 8 : 0);
            const int nbins = within == 2 ? 256 : 4096;
            const unsigned dmask = (unsigned)nbins - 1u;
            for (int i = tid; i < nbins; i += nthr) hist[i] = 0;
            __syncthreads();
            // lanes with the same digit add once (the high digits of nearby scores coincide, and
            // one atomic per lane would serialise on a few bins)
            auto count = [&](unsigned long long u, bool valid) {
                const unsigned d = valid && (u & mask) == prefix ? ((unsigned)(u >> shift) & dmask) : 0xffffffffu;
                const unsigned peers = __match_any_sync(FULL, d);
                if (d != 0xffffffffu && lane == __ffs(peers) - 1) atomicAdd(&hist[d], (unsigned)__popc(peers));
            };
            if (in_regs) {
#pragma unroll
                for (int j = 0; j < KPT; ++j) count(kr[j], tid + j * nthr < nb);
            } else {
                for (int n0 = 0; n0 < nb; n0 += nthr) {
                    const int n = n0 + tid;
                    count(n < nb ? key_of(n) : 0ull, n < nb);
                }
            }
            __syncthreads();
            // thread t sums the bins nbins - 1 - (t * bpt ... t * bpt + bpt - 1) (from the top); the
            // thread whose running count crosses rem holds T's digit
            const int bpt = nbins > nthr ? nbins / nthr : 1;
            unsigned c[kHistBins / kLargeThreads];
            unsigned sum = 0;
#pragma unroll
            for (int i = 0; i < kHistBins / kLargeThreads; ++i) {
                const int bin = nbins - 1 - (tid * bpt + i);
                c[i] = (i < bpt && bin >= 0) ? hist[bin] : 0u;
                sum += c[i];
            }
            int tot = 0;
            const unsigned incl = (unsigned)block_inclusive_sum((int)sum, warp_sums, tot);
            const unsigned excl = incl - sum;
            if (sum > 0 && excl < (unsigned)rem && (unsigned)rem <= incl) {
                unsigned above = excl;
                int d = nbins - 1 - tid * bpt;
#pragma unroll
                for (int i = 0; i < kHistBins / kLargeThreads; ++i) {
                    if (i < bpt && above + c[i] >= (unsigned)rem) {
                        d = nbins - 1 - (tid * bpt + i);
                        st[3] = c[i] == (unsigned)rem - above;  // every key with this prefix is taken
                        break;
                    }
                    above += c[i];
                }
                st[0] = d;
                st[1] = rem - (int)above;
            }
            __syncthreads();
            prefix |= (unsigned long long)st[0] << shift;
            mask |= (unsigned long long)dmask << shift;
            rem = st[1];
            const bool all_taken = st[3] != 0;
            __syncthreads();
            // once the score bits are fixed and every block with that score is taken, the id bits
            // need no passes: T is that score with the lowest id bits
            if (shift == 32 && all_taken) break;
        }
    }
    // keys are distinct, so exactly kk of them are >= T (with kk == nb, T = 0 takes every block)
    const unsigned long long T = prefix;
    if (tid == 0) st[2] = 0;
    __syncthreads();
    auto take = [&](unsigned long long u) {
        if (u >= T) {
            const int at = atomicAdd(&st[2], 1);
            if (at < kMaxTopK) keys[at] = u;
        }
    };
    if (in_regs) {
#pragma unroll
        for (int j = 0; j < KPT; ++j)
            if (tid + j * nthr < nb) take(kr[j]);
    } else {
        for (int n = tid; n < nb; n += nthr) take(key_of(n));
    }
    __syncthreads();
    // descending bitonic sort of the kMaxTopK slots (one per thread, zero padding below every
    // real key): strides below 32 exchange through shuffles, larger ones through shared memory
    unsigned long long v = tid < kk ? keys[tid] : 0ull;
    if (kk > 1) {
        for (int size = 2; size <= kMaxTopK; size <<= 1)
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                unsigned long long o;
                if (stride >= 32) {
                    __syncthreads();
                    keys[tid] = v;
                    __syncthreads();
                    o = keys[tid ^ stride];
                } else {
                    o = __shfl_xor_sync(FULL, v, stride);
                }
                const bool keep_max = ((tid & stride) == 0) == ((tid & size) == 0);
                v = keep_max ? (v > o ? v : o) : (v < o ? v : o);
            }
    }
    if (tid < a.k) {  // thread i holds the i-th key (a.k <= kMaxTopK = blockDim.x)
        const size_t o = (size_t)row * a.k + tid;
        const int id = tid < kk ? (int)~(uint32_t)v : -1;
        a.ids_out[o] = id;
        if (a.ids_copy != nullptr) a.ids_copy[o] = id;
        if (a.top_scores_out != nullptr) a.top_scores_out[o] = tid < kk ? bits_score((uint32_t)(v >> 32)) : -INFINITY;
    }
}

// Prefill rows (one list per query row: many rows, each of at most a few thousand blocks) with
// k <= kWarpRowMaxK: one warp per row.  The k-th largest score is found exactly by a radix select
// over the 32 order-preserving score bits (four passes of 8-bit digits, a 256-bin histogram per
// warp in shared memory, the scores re-read from L2 in each pass); every block above that score
// is taken, and of the blocks at it the lowest ids, scanned in id order.  The k keys are then
// ranked by counting (keys are distinct: score bits above the complemented id).
constexpr int kWarpRowMaxK = 256;
constexpr int kWarpRows = 8;  // rows (warps) per CTA

__global__ void __launch_bounds__(kWarpRows * 32) warp_topk_kernel(const LargeTopkArgs a) {
    __shared__ unsigned hist[kWarpRows][256];
    __shared__ unsigned long long cand[kWarpRows][kWarpRowMaxK];
    const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kWarpRows + wib;
    if (row >= a.rows) return;  // whole warps only; no CTA-wide barrier below
    const int t = (int)((row / a.G) % a.q_len);
    int pos = a.q_start + t;
    if (pos >= a.L_max) pos = a.L_max - 1;
    const int nb = pos / a.Bk + 1;
    const int kk = a.k < nb ? a.k : nb;
    const float *src = a.scores + row * a.stride;
    const unsigned lt = (1u << lane) - 1u;  // lanes below this one
    auto bits_of = [&](int n) -> uint32_t {
        // MSA_FORCE_SINK_LOCAL: block 0 and the row's own block rank above every score
        return score_bits((a.force && (n == 0 || n == nb - 1)) ? INFINITY : src[n]);
    };
    unsigned *H = hist[wib];
    uint32_t prefix = 0, mask = 0;
    int rem = kk;  // rank of the k-th score among the scores that match the prefix so far
    if (kk < nb) {
#pragma unroll 1
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = lane; i < 256; i += 32) H[i] = 0;
            __syncwarp();
            for (int n0 = 0; n0 < nb; n0 += 32) {
                const int n = n0 + lane;
                const uint32_t u = n < nb ? bits_of(n) : 0u;
                const unsigned d = (n < nb && (u & mask) == prefix) ? ((u >> shift) & 255u) : 0xffffffffu;
                const unsigned peers = __match_any_sync(FULL, d);
                if (d != 0xffffffffu && lane == __ffs(peers) - 1) atomicAdd(&H[d], (unsigned)__popc(peers));
            }
            __syncwarp();
            // lane l sums bins 255 - 8 l .. 248 - 8 l (from the top); the lane whose running count
            // reaches rem holds the digit
            unsigned c[8], sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                c[i] = H[255 - 8 * lane - i];
                sum += c[i];
            }
            unsigned incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned v = __shfl_up_sync(FULL, incl, o);
                if (lane >= o) incl += v;
            }
            int dsel = -1, rsel = 0;
            if (incl - sum < (unsigned)rem && (unsigned)rem <= incl) {
                unsigned above = incl - sum;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (dsel < 0 && above + c[i] >= (unsigned)rem) {
                        dsel = 255 - 8 * lane - i;
                        rsel = rem - (int)above;
                    }
                    above += c[i];
                }
            }
            const int from = __ffs(__ballot_sync(FULL, dsel >= 0)) - 1;
            dsel = __shfl_sync(FULL, dsel, from);
            rsel = __shfl_sync(FULL, rsel, from);
            prefix |= (uint32_t)dsel << shift;
            mask |= 255u << shift;
            rem = rsel;
            __syncwarp();  // H is read before the next pass clears it
        }
    }
    // kk < nb: every score above `prefix` is taken, and `rem` of the scores equal to it, lowest ids
    // first; kk == nb: every block
    unsigned long long *C = cand[wib];
    int taken = 0, eq_seen = 0;
    for (int n0 = 0; n0 < nb; n0 += 32) {
        const int n = n0 + lane;
        const uint32_t u = n < nb ? bits_of(n) : 0u;
        const bool gt = n < nb && (kk == nb || u > prefix);
        const bool eq = n < nb && kk < nb && u == prefix;
        const unsigned be = __ballot_sync(FULL, eq);
        const bool take = gt || (eq && eq_seen + __popc(be & lt) < rem);
        const unsigned bt = __ballot_sync(FULL, take);
        if (take) C[taken + __popc(bt & lt)] = ((unsigned long long)u << 32) | (uint32_t)~(uint32_t)n;
        taken += __popc(bt);
        eq_seen += __popc(be);
    }
    __syncwarp();
    // rank of each key among the kk (distinct) keys: its slot in the list
    for (int i = lane; i < kk; i += 32) {
        const unsigned long long key = C[i];
        int rank = 0;
        for (int j = 0; j < kk; ++j) rank += C[j] > key ? 1 : 0;
        const size_t o = (size_t)row * a.k + rank;
        const int id = (int)~(uint32_t)key;
        a.ids_out[o] = id;
        if (a.ids_copy != nullptr) a.ids_copy[o] = id;
        if (a.top_scores_out != nullptr) a.top_scores_out[o] = bits_score((uint32_t)(key >> 32));
    }
    for (int i = kk + lane; i < a.k; i += 32) {
        const size_t o = (size_t)row * a.k + i;
        a.ids_out[o] = -1;
        if (a.ids_copy != nullptr) a.ids_copy[o] = -1;
        if (a.top_scores_out != nullptr) a.top_scores_out[o] = -INFINITY;
    }
}

// Block maxima of stored token scores (rows of L_max) over the visible tokens of every block,
// one warp per (row, block), for the large-k TopK that reads block scores.
__global__ void __launch_bounds__(256) token_block_max_kernel(const LargeTopkArgs a, const float *tok,
                                                              float *blk) {
    const int lane = threadIdx.x & 31;
    const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    const long long total = (long long)a.rows * a.stride;
    for (long long x = wid; x < total; x += nw) {
        const int row = (int)(x / a.stride), n = (int)(x % a.stride);
        const int t = (row / a.G) % a.q_len, b = row / (a.G * a.q_len);
        int pos;
        if (a.prefill) {
            pos = a.q_start + t;
        } else {
            int L = a.seq_lens[b];
            L = L < 0 ? 0 : (L > a.L_max ? a.L_max : L);
            pos = L - 1;
        }
        if (pos >= a.L_max) pos = a.L_max - 1;
        const int lo = n * a.Bk, hi = (n + 1) * a.Bk - 1 < pos ? (n + 1) * a.Bk - 1 : pos;
        float m = -INFINITY;
        for (int j = lo + lane; j <= hi; j += 32) m = fmaxf(m, tok[(size_t)row * a.L_max + j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
        if (lane == 0) blk[x] = m;
    }
}

}  // namespace

cudaError_t launch_large_topk(const LargeTopkArgs &a, cudaStream_t s) {
    if (a.rows <= 0) return cudaSuccess;
    if (a.prefill && a.k <= kWarpRowMaxK) {
        warp_topk_kernel<<<(unsigned)((a.rows + kWarpRows - 1) / kWarpRows), kWarpRows * 32, 0, s>>>(a);
        return cudaGetLastError();
    }
    large_topk_kernel<<<(unsigned)a.rows, kLargeThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_token_block_max(const LargeTopkArgs &a, const float *tok, float *blk, cudaStream_t s) {
    const long long warps = (long long)a.rows * a.stride;
    if (warps <= 0) return cudaSuccess;
    long long blocks = (warps + 7) / 8;
    if (blocks > 4096) blocks = 4096;
    token_block_max_kernel<<<(unsigned)blocks, 256, 0, s>>>(a, tok, blk);
    return cudaGetLastError();
}

}  // namespace msa
