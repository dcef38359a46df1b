// Steps 1b + 1c of MSA for large k (more blocks than a warp-distributed list holds): the k best
// block scores of every row.
//
// Page "MiniMax wird duenn" (atlascloud.ai), section 1, Step 1: block scores (the block maxima
// of the index scores) go through TopK per group.  Section 3 back-calculates that a query
// touches about 6-7 % of the blocks at 1M tokens (k near 1000 of 16,384 blocks of 64 tokens),
// far beyond what per-warp sorted lists hold.  One CTA per row finds the k-th best score by a
// radix select on the scores' order-preserving bits (four passes of 8 bits, a shared histogram
// each), takes every block above it and, among the blocks equal to it, the lowest ids (an
// ordered block-wide count), then sorts the k taken blocks once (bitonic, 64-bit keys: score
// bits above the complemented id).  The row's scores are read from global memory in every pass
// (L2 keeps them), so the number of blocks is not bounded by shared memory.
#include "msa_device.cuh"

namespace msa {

namespace {

constexpr int kLargeThreads = 1024;

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

__global__ void __launch_bounds__(kLargeThreads) large_topk_kernel(const LargeTopkArgs a) {
    __shared__ unsigned hist[256];
    __shared__ unsigned long long keys[kMaxTopK];
    __shared__ int warp_sums[32];
    __shared__ int st[4];  // [0] chosen digit, [1] remaining rank, [2] taken blocks
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
    auto key_of = [&](int n) -> uint32_t {
        // MSA_FORCE_SINK_LOCAL: block 0 and the row's own block rank above every score
        const float v = (a.force && (n == 0 || n == nb - 1)) ? INFINITY : src[n];
        return score_bits(v);
    };

    // the kk-th largest key T (exactly): one 8-bit digit per pass, from the top
    uint32_t prefix = 0, mask = 0;
    int rem = kk;  // rank of T among the keys that match the prefix so far
    if (kk < nb) {
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += nthr) hist[i] = 0;
            __syncthreads();
            for (int n = tid; n < nb; n += nthr) {
                const uint32_t u = key_of(n);
                if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
            }
            __syncthreads();
            if (warp == 0) {
                // lane l holds digits 255 - 8 l .. 248 - 8 l (from the top)
                unsigned c[8];
                unsigned sum = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    c[j] = hist[255 - 8 * lane - j];
                    sum += c[j];
                }
                unsigned incl = sum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const unsigned u = __shfl_up_sync(FULL, incl, o);
                    if (lane >= o) incl += u;
                }
                const unsigned excl = incl - sum;
                const bool here = excl < (unsigned)rem && (unsigned)rem <= incl;
                if (here) {
                    unsigned above = excl;
                    int d = 255 - 8 * lane;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if (above + c[j] >= (unsigned)rem) {
                            d = 255 - 8 * lane - j;
                            break;
                        }
                        above += c[j];
                    }
                    st[0] = d;
                    st[1] = rem - (int)above;
                }
            }
            __syncthreads();
            prefix |= (uint32_t)st[0] << shift;
            mask |= 255u << shift;
            rem = st[1];
            __syncthreads();
        }
    }
    const uint32_t T = prefix;  // with kk == nb every block is taken (mask 0 keeps all)

    // take every key above T and the `rem` lowest ids equal to T: each thread scans a contiguous
    // range of ids, so an inclusive sum of the per-thread counts ranks the equal keys by id
    if (tid == 0) st[2] = 0;
    const int chunk = (nb + nthr - 1) / nthr;
    const int n0 = tid * chunk, n1 = n0 + chunk < nb ? n0 + chunk : nb;
    int eq = 0;
    if (kk < nb)
        for (int n = n0; n < n1; ++n) eq += key_of(n) == T;
    int tot = 0;
    const int eq_incl = block_inclusive_sum(eq, warp_sums, tot);
    int rank = eq_incl - eq;  // equal keys with lower ids
    for (int n = n0; n < n1; ++n) {
        const uint32_t u = key_of(n);
        bool take;
        if (kk == nb) {
            take = true;
        } else if (u > T) {
            take = true;
        } else if (u == T) {
            take = rank < rem;
            ++rank;
        } else {
            take = false;
        }
        if (take) {
            const int at = atomicAdd(&st[2], 1);
            if (at < kMaxTopK) keys[at] = ((unsigned long long)u << 32) | (uint32_t)~(uint32_t)n;
        }
    }
    __syncthreads();
    int P = 1;
    while (P < kk) P <<= 1;
    for (int i = kk + tid; i < P; i += nthr) keys[i] = 0ull;  // below every real key
    __syncthreads();
    if (P > 1) block_sort_desc(keys, P);
    for (int i = tid; i < a.k; i += nthr) {
        const size_t o = (size_t)row * a.k + i;
        const unsigned long long key = i < kk ? keys[i] : 0ull;
        const int id = i < kk ? (int)~(uint32_t)key : -1;
        a.ids_out[o] = id;
        if (a.ids_copy != nullptr) a.ids_copy[o] = id;
        if (a.top_scores_out != nullptr) a.top_scores_out[o] = i < kk ? bits_score((uint32_t)(key >> 32)) : -INFINITY;
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
