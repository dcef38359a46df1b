// Step 2 of MSA for decode: exact softmax attention over the selected blocks.
//
// Page "MiniMax wird duenn" (atlascloud.ai), section 1, Step 2: every query
// head of a GQA group uses the group's single TopK list (Q1/Q2/Q3 -> I1,
// Q4/Q5/Q6 -> I2) and attends over only those blocks of the full, real K/V
// cache, so one group loads one set of KV blocks for all its heads.
//
// decode_select_kernel finishes Step 1: one CTA per (sequence, group) stages
// the scan's per-piece sorted candidate lists in shared memory and selects
// the group's final TopK list from them.
//
// decode_attn_kernel, grid (split s, group g, sequence b): a CTA reads the
// group's list, streams the K/V tiles of its share of the blocks through a
// two-stage TMA bulk-copy ring and keeps an online softmax for all r heads
// of the group: scores with one warp per key (lanes split the head
// dimension, a reduce-scatter butterfly finishes the r dot products), then
// per-head max/exp2/sum, then P.V with each thread owning a few output
// elements.  Each split writes a normalised partial output and its log2
// normaliser; the last split of a group to finish (atomic arrival count)
// merges them by log-sum-exp into the output.  With MSA_DENSE the splits
// cover every visible block: plain GQA decode.
#include "msa_device.cuh"

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
    unsigned char *ring = smem;                                             // [NST][K tile | V tile]
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring + NST * 2 * tile_bytes); // [NST]
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

    pdl_wait_prior_grid();  // the selection is complete from here on
    pdl_allow_next_grid();
    if (!a.dense && tid < a.k) sel_i[tid] = a.ids_in[((size_t)b * a.G + g) * a.k + tid];
    __syncthreads();

    // this split's blocks: list positions [j0, j1)
    const int bps = a.blocks_per_split;
    const int j0 = s * bps;
    int j1 = j0 + bps;
    const int jmax = a.dense ? nb : a.k;
    if (j1 > jmax) j1 = jmax;

    auto block_at = [&](int j) -> int {
        const int id = a.dense ? j : sel_i[j];
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
    const size_t head_off = ((size_t)b * a.G + g) * (size_t)a.L_max;
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
            const size_t src = (head_off + (size_t)key0) * D * ES;
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
                for (int q2 = consumed + 1; q2 < issued; ++q2) mbar_wait(&bars[q2 % NST], (q2 / NST) & 1, nullptr);
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

    // the last split of (b, g) to arrive merges all splits
    __threadfence();
    __syncthreads();
    if (tid == 0) sel_s[0] = (atomicAdd(&a.counters[bg], 1) == a.S - 1) ? 1.f : 0.f;
    __syncthreads();
    if (sel_s[0] == 0.f) return;
    __threadfence();
    float *wgt = p_s;  // [S][r] merge weights (S <= max(k, kMaxSplits))
    for (int i = tid; i < a.S * r; i += kAttnThreads) wgt[i] = __ldcg(a.part_lse + bg * a.S * r + i);
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
    T *o = reinterpret_cast<T *>(a.o) + ((size_t)b * a.Hq + (size_t)g * r) * D;
    const float *po = a.part_o + bg * a.S * r * D;
    for (int f = tid; f < r * D; f += kAttnThreads) {
        const int h = f / D;
        float num = 0.f;
#pragma unroll 4
        for (int j = 0; j < a.S; ++j) num = fmaf(wgt[j * r + h], __ldcg(po + ((size_t)j * r) * D + f), num);
        store_elem(o + f, num);
    }
    if (tid == 0) a.counters[bg] = 0;  // ready for the next call
}

// Final TopK of a group from the scan's per-piece sorted lists.  All
// candidates are staged in shared memory; any candidate worse than the k-th
// entry of some full list cannot be in the final k (that list alone already
// has k better ones), so only the survivors are ranked, each by counting the
// survivors that beat it.
__global__ void __launch_bounds__(256) decode_select_kernel(const SelectArgs a) {
    extern __shared__ __align__(16) unsigned char sm_raw[];
    const int cap = a.n_cta * a.k;
    float *ls = reinterpret_cast<float *>(sm_raw);
    int *li = reinterpret_cast<int *>(ls + cap);
    float *ss = reinterpret_cast<float *>(li + cap);   // survivors
    int *si_ = reinterpret_cast<int *>(ss + cap);
    float *out_s = reinterpret_cast<float *>(si_ + cap);
    int *out_i = reinterpret_cast<int *>(out_s + 32);
    __shared__ float thr_s[8];
    __shared__ int thr_i[8];
    __shared__ int n_surv;
    const int g = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait_prior_grid();
    pdl_allow_next_grid();
    const int gps = a.G / a.Hik;
    const int seg = b * a.Hik + g % a.Hik, gl = g / a.Hik;
    const SegInfo si = a.seg_info[seg];
    const int n = si.n_pieces * a.k;
    for (int i = tid; i < n; i += blockDim.x) {
        const size_t src = (((size_t)seg * a.n_cta + i / a.k) * gps + gl) * a.k + i % a.k;
        ls[i] = a.cand_s[src];
        li[i] = a.cand_i[src];
    }
    if (tid < 32) { out_s[tid] = -INFINITY; out_i[tid] = -1; }
    if (tid == 0) n_surv = 0;
    __syncthreads();
    // threshold: the best k-th entry over all lists
    float ts = -INFINITY;
    int ti = -1;
    for (int l = tid; l < si.n_pieces; l += blockDim.x) {
        const float s = ls[l * a.k + a.k - 1];
        const int i = li[l * a.k + a.k - 1];
        if (i >= 0 && better(s, i, ts, ti)) { ts = s; ti = i; }
    }
    warp_best(ts, ti);
    if (lane == 0) { thr_s[warp] = ts; thr_i[warp] = ti; }
    __syncthreads();
    ts = thr_s[0];
    ti = thr_i[0];
    for (int w2 = 1; w2 < 8; ++w2)
        if (better(thr_s[w2], thr_i[w2], ts, ti)) { ts = thr_s[w2]; ti = thr_i[w2]; }
    for (int i = tid; i < n; i += blockDim.x) {
        if (li[i] >= 0 && !better(ts, ti, ls[i], li[i])) {
            const int at = atomicAdd(&n_surv, 1);
            ss[at] = ls[i];
            si_[at] = li[i];
        }
    }
    __syncthreads();
    const int m = n_surv;
    for (int i = tid; i < m; i += blockDim.x) {
        const float s = ss[i];
        const int id = si_[i];
        int rank = 0;
        for (int j = 0; j < m; ++j) rank += better(ss[j], si_[j], s, id) ? 1 : 0;
        if (rank < a.k) { out_s[rank] = s; out_i[rank] = id; }
    }
    __syncthreads();
    if (tid < a.k) {
        const size_t o = ((size_t)b * a.G + g) * a.k + tid;
        a.sel_ids[o] = out_i[tid];
        if (a.ids_out != nullptr) a.ids_out[o] = out_i[tid];
        if (a.top_scores_out != nullptr) a.top_scores_out[o] = out_s[tid];
    }
    if (tid == 0) a.counters[(size_t)b * a.G + g] = 0;
}

template <typename T, int D, int R>
cudaError_t launch_attn_t(const AttnArgs &a, cudaStream_t s, bool pdl) {
    using Cfg = AttnCfg<T, D, R>;
    const int KT = a.Bk < Cfg::KT_MAX ? a.Bk : Cfg::KT_MAX;
    // p_s doubles as the [S][r] merge weights of the last split: R * max(KT, kMaxSplits) floats
    const size_t smem = (size_t)Cfg::NST * 2 * KT * D * Cfg::ES + Cfg::NST * 8 + 64 * 4 + 3 * R * 4 +
                        (size_t)R * (KT > kMaxSplits ? KT : kMaxSplits) * 4 + 16;
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<T, D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             160 * 1024);
        if (e != cudaSuccess) return e;
        attr_done = true;
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

template <typename T>
cudaError_t launch_attn_d(const AttnArgs &a, cudaStream_t s, bool pdl) {
    return a.D == 64 ? launch_attn_r<T, 64>(a, s, pdl) : launch_attn_r<T, 128>(a, s, pdl);
}

}  // namespace

cudaError_t launch_decode_attn(const AttnArgs &a, int dtype, cudaStream_t s, bool pdl) {
    return dtype == MSA_F32 ? launch_attn_d<float>(a, s, pdl) : launch_attn_d<__nv_bfloat16>(a, s, pdl);
}

cudaError_t launch_decode_select(const SelectArgs &a, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.G, a.B);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = (size_t)a.n_cta * a.k * 16 + 256;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    static size_t attr_bytes = 48 * 1024;
    if (cfg.dynamicSmemBytes > attr_bytes) {
        cudaError_t e = cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)cfg.dynamicSmemBytes);
        if (e != cudaSuccess) return e;
        attr_bytes = cfg.dynamicSmemBytes;
    }
    return cudaLaunchKernelEx(&cfg, decode_select_kernel, a);
}

}  // namespace msa
