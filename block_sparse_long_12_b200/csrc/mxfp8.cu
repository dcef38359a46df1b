// MXFP8 storage of index keys: the quantiser.
//
// The pages name MXFP8 as the format of the official quantised checkpoints (docs.clore.ai
// "MiniMax M3", deployment table and checkpoint list); read as the microscaling format, every 32
// consecutive index dimensions of a token's key share one E8M0 scale 2^shared, with shared =
// floor(log2 max|v|) - 8 (8: the exponent of E4M3's largest normal, 448 = 1.75 * 2^8) clamped to
// [-127, 127], and every element is v / 2^shared rounded to the nearest FP8 E4M3 value (ties to
// even, saturating at 448).  One warp per 32-element block, one element per lane: the block's
// maximum magnitude by a warp reduction over the fp32 bit patterns (non-negative floats order as
// unsigned integers), the exponent by ilogbf, the scaling by ldexpf (exact: a power of two), the
// rounding by the hardware conversion to E4M3 with saturation.
#include "msa_device.cuh"

namespace msa {

namespace {

struct QuantArgs {
    const __nv_bfloat16 *src;  // [rows, di]
    uint8_t *codes;            // plain: [rows, di]; append: the code cache
    uint8_t *scales;           // plain: [rows, di / 32]; append: the scale cache
    long long n_blocks;        // rows * di / 32
    int di;
    // append: source row r = b * Hik + h goes to position seq_lens[b] - 1 of head h's cache rows
    int append;
    const int *seq_lens;
    int Hik, L_max;
    CacheMap cache;
};

__global__ void __launch_bounds__(256) mxfp8_quantize_kernel(const QuantArgs a) {
    const int lane = threadIdx.x & 31;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    const int bpr = a.di / 32;  // blocks per row
    for (long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < a.n_blocks; i += nw) {
        const long long r = i / bpr;
        const int j = (int)(i - r * bpr);
        const float v = __bfloat162float(a.src[r * a.di + j * 32 + lane]);
        const float amax = __uint_as_float(__reduce_max_sync(FULL, __float_as_uint(fabsf(v))));
        int shared = -127;
        if (amax > 0.f) {
            shared = ilogbf(amax) - 8;
            shared = shared < -127 ? -127 : (shared > 127 ? 127 : shared);
        }
        const uint8_t code = (uint8_t)__nv_cvt_float_to_fp8(ldexpf(v, -shared), __NV_SATFINITE, __NV_E4M3);
        long long row = r;
        if (a.append) {
            const int b = (int)(r / a.Hik), h = (int)(r - (long long)b * a.Hik);
            int pos = a.seq_lens[b] - 1;
            pos = pos < 0 ? 0 : (pos >= a.L_max ? a.L_max - 1 : pos);
            row = a.cache.row(b, h, a.Hik, a.L_max, pos);
        }
        a.codes[row * a.di + j * 32 + lane] = code;
        if (lane == 0) a.scales[row * bpr + j] = (uint8_t)(shared + 127);
    }
}

cudaError_t launch(const QuantArgs &a, cudaStream_t s) {
    if (a.n_blocks <= 0) return cudaSuccess;
    long long blocks = (a.n_blocks + 7) / 8;  // 8 warps per CTA
    if (blocks > 4096) blocks = 4096;
    mxfp8_quantize_kernel<<<(unsigned)blocks, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mxfp8_quantize(const void *src, long long rows, int di, uint8_t *codes, uint8_t *scales,
                                  cudaStream_t s) {
    QuantArgs a{};
    a.src = static_cast<const __nv_bfloat16 *>(src);
    a.codes = codes;
    a.scales = scales;
    a.di = di;
    a.n_blocks = rows * (di / 32);
    return launch(a, s);
}

cudaError_t launch_mxfp8_append(const msa_params_t &p, const CacheMap &cache, const void *ki_new, uint8_t *codes,
                                uint8_t *scales, cudaStream_t s) {
    QuantArgs a{};
    a.src = static_cast<const __nv_bfloat16 *>(ki_new);
    a.codes = codes;
    a.scales = scales;
    a.di = p.idx_dim;
    a.n_blocks = (long long)p.batch * p.n_idx_k_heads * (p.idx_dim / 32);
    a.append = 1;
    a.seq_lens = p.seq_lens;
    a.Hik = p.n_idx_k_heads;
    a.L_max = p.max_seq_len;
    a.cache = cache;
    return launch(a, s);
}

}  // namespace msa
