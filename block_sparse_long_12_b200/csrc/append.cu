// The serving step before a decode: the new token's K, V and index key of every sequence go to
// its position seq_lens[b] - 1 in the caches (contiguous or paged), 16 bytes per thread.
#include "msa_device.cuh"

namespace msa {

namespace {

struct AppendArgs {
    const uint4 *k_new, *v_new, *ki_new;  // [B, Hkv, D], [B, Hkv, D], [B, Hik, di] elements
    uint4 *k, *v, *ki;
    const int *seq_lens;
    int B, Hkv, Hik, L_max;
    int kv_vecs, ki_vecs;                 // 16-byte vectors per row: D * es / 16, di * es / 16
    CacheMap cache;
};

__global__ void append_kernel(const AppendArgs a) {
    const int per_b = 2 * a.Hkv * a.kv_vecs + a.Hik * a.ki_vecs;
    const long long n = (long long)a.B * per_b;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const int b = (int)(i / per_b);
        int e = (int)(i - (long long)b * per_b);
        int pos = a.seq_lens[b] - 1;
        pos = pos < 0 ? 0 : (pos >= a.L_max ? a.L_max - 1 : pos);
        if (e < 2 * a.Hkv * a.kv_vecs) {
            const bool is_v = e >= a.Hkv * a.kv_vecs;
            if (is_v) e -= a.Hkv * a.kv_vecs;
            const int h = e / a.kv_vecs, c = e - h * a.kv_vecs;
            const size_t dst = (size_t)a.cache.row(b, h, a.Hkv, a.L_max, pos) * a.kv_vecs + c;
            const size_t src = ((size_t)b * a.Hkv + h) * a.kv_vecs + c;
            if (is_v) a.v[dst] = a.v_new[src];
            else a.k[dst] = a.k_new[src];
        } else {
            e -= 2 * a.Hkv * a.kv_vecs;
            const int h = e / a.ki_vecs, c = e - h * a.ki_vecs;
            a.ki[(size_t)a.cache.row(b, h, a.Hik, a.L_max, pos) * a.ki_vecs + c] =
                a.ki_new[((size_t)b * a.Hik + h) * a.ki_vecs + c];
        }
    }
}

}  // namespace

cudaError_t launch_append(const msa_params_t &p, const CacheMap &cache, const void *k_new, const void *v_new,
                          const void *ki_new, void *k, void *v, void *ki, cudaStream_t s) {
    const int es = p.dtype == MSA_F32 ? 4 : 2;
    AppendArgs a{};
    a.k_new = static_cast<const uint4 *>(k_new);
    a.v_new = static_cast<const uint4 *>(v_new);
    a.ki_new = static_cast<const uint4 *>(ki_new);
    a.k = static_cast<uint4 *>(k);
    a.v = static_cast<uint4 *>(v);
    a.ki = static_cast<uint4 *>(ki);
    a.seq_lens = p.seq_lens;
    a.B = p.batch; a.Hkv = p.n_kv_heads; a.Hik = p.n_idx_k_heads; a.L_max = p.max_seq_len;
    a.kv_vecs = p.head_dim * es / 16;
    // MXFP8 index keys are quantised into their cache by launch_mxfp8_append instead
    a.ki_vecs = p.idx_format == MSA_IDX_MXFP8 ? 0 : p.idx_dim * es / 16;
    a.cache = cache;
    const long long n = (long long)p.batch * (2 * a.Hkv * a.kv_vecs + a.Hik * a.ki_vecs);
    const int grid = (int)((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
    append_kernel<<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace msa
