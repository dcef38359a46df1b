// Steps 1b + 1c of MSA from stored scores: block max pool and TopK per row.
//
// Page "MiniMax wird duenn" (atlascloud.ai), section 1, Step 1: token scores
// are reduced to one score per fixed-size block by their maximum, then TopK
// keeps the best blocks for the group.  This entry works on scores that an
// earlier call stored (token or block granularity), one CTA per
// (sequence, query row, group); eight warps take blocks round-robin, keep
// warp-distributed sorted lists, and warp 0 merges them.  With
// MSA_FORCE_SINK_LOCAL block 0 and the row's own block take the score +inf.
#include "msa_device.cuh"

namespace msa {

namespace {

__global__ void __launch_bounds__(256) pool_topk_kernel(const PoolTopkArgs a) {
    __shared__ float ls[8 * 32];
    __shared__ int li[8 * 32];
    __shared__ float out_s[32];
    __shared__ int out_i[32];
    const int row = blockIdx.x;
    const int t = (row / a.G) % a.q_len, b = row / (a.G * a.q_len);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
    WarpTopK lst;
    lst.reset();
    const float *src = a.scores + (size_t)row * (a.is_block ? a.nb_max : a.L_max);
    for (int n = w; n < nb; n += 8) {
        float m;
        if (a.is_block) {
            m = src[n];  // same address in every lane
        } else {
            m = -INFINITY;
            const int hi = (n + 1) * a.Bk - 1 < pos ? (n + 1) * a.Bk - 1 : pos;
            for (int j = n * a.Bk + lane; j <= hi; j += 32) m = fmaxf(m, src[j]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
        }
        // forced sink / local blocks rank above every score
        if (a.force && (n == 0 || n == nb - 1)) m = INFINITY;
        lst.insert(m, n, a.k, lane);
    }
    ls[w * 32 + lane] = lst.s;
    li[w * 32 + lane] = lst.id;
    __syncthreads();
    if (w == 0) {
        warp_merge_sorted_lists<1>(ls, li, 8, a.k, 32, a.k, out_s, out_i, lane);
        __syncwarp();
        if (lane < a.k) {
            a.ids_out[(size_t)row * a.k + lane] = out_i[lane];
            if (a.top_scores_out != nullptr) a.top_scores_out[(size_t)row * a.k + lane] = out_s[lane];
        }
    }
}

}  // namespace

cudaError_t launch_pool_topk(const PoolTopkArgs &a, cudaStream_t s) {
    const long long rows = (long long)a.B * a.q_len * a.G;
    if (rows <= 0) return cudaSuccess;
    pool_topk_kernel<<<(unsigned)rows, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace msa
