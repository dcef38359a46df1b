// Host side of the MSA C ABI: argument checks, workspace layout, launches.
// Every check runs before anything is enqueued; the library never allocates,
// frees or synchronises (except msa_get_device_status, which reads back one
// word on request).
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "msa_internal.h"

#include <nvtx3/nvToolsExt.h>

namespace msa {
namespace {

thread_local std::string g_err;
thread_local cudaEvent_t g_stage_ev[3];
thread_local int g_n_stage_ev = 0;

msa_status_t fail(msa_status_t st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return st;
}

msa_status_t cuda_fail(cudaError_t e, const char *what) {
    return fail(MSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int elem_size(int dtype) { return dtype == MSA_F32 ? 4 : 2; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

struct DevCache {
    int checked = 0, ok = 0, sms = 0;
};
DevCache g_dev[64];

msa_status_t check_device(int *n_sm) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(MSA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    DevCache &c = g_dev[dev];
    if (!c.checked) {
        int major = 0, minor = 0, sms = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute");
        c.ok = (major == 10 && minor == 0);
        c.sms = sms;
        c.checked = 1;
        if (!c.ok) return fail(MSA_ERR_UNSUPPORTED, "compute capability %d.%d: this library runs on sm_100 only",
                               major, minor);
    }
    if (!c.ok) return fail(MSA_ERR_UNSUPPORTED, "this library runs on sm_100 (B200) only");
    *n_sm = c.sms;
    return MSA_OK;
}

enum Mode { DECODE_ONLY, PREFILL_ONLY, ANY_ROWS };

// bytes of one index-key row: idx_dim elements of params.dtype, or one E4M3 byte each (MXFP8)
int idx_row_bytes(const msa_params_t &p) {
    return p.idx_dim * (p.idx_format == MSA_IDX_MXFP8 ? 1 : elem_size(p.dtype));
}

msa_status_t check_params(const msa_params_t *p, Mode mode) {
    if (p == nullptr) return fail(MSA_ERR_INVALID_ARG, "params is NULL");
    if (p->dtype != MSA_F32 && p->dtype != MSA_BF16) return fail(MSA_ERR_INVALID_ARG, "dtype %d unknown", p->dtype);
    if (p->batch < 1) return fail(MSA_ERR_INVALID_ARG, "batch %d < 1", p->batch);
    if (p->batch > kMaxBatch) return fail(MSA_ERR_UNSUPPORTED, "batch %d > %d", p->batch, kMaxBatch);
    if (p->n_kv_heads < 1 || p->n_q_heads < 1 || p->n_q_heads % p->n_kv_heads != 0)
        return fail(MSA_ERR_INVALID_ARG, "n_q_heads %d must be a positive multiple of n_kv_heads %d", p->n_q_heads,
                    p->n_kv_heads);
    if (p->n_q_heads / p->n_kv_heads > 16)
        return fail(MSA_ERR_UNSUPPORTED, "group size %d > 16", p->n_q_heads / p->n_kv_heads);
    if (p->n_idx_k_heads != 1 && p->n_idx_k_heads != p->n_kv_heads)
        return fail(MSA_ERR_INVALID_ARG, "n_idx_k_heads %d must be 1 or n_kv_heads %d", p->n_idx_k_heads,
                    p->n_kv_heads);
    const int gps = p->n_kv_heads / p->n_idx_k_heads;
    if (gps > kMaxGroupsPerSeg || !pow2(gps))
        return fail(MSA_ERR_UNSUPPORTED, "%d groups sharing one index-K head (supported: 1, 2, 4, 8)", gps);
    if (p->head_dim != 64 && p->head_dim != 128) return fail(MSA_ERR_UNSUPPORTED, "head_dim %d (64 or 128)", p->head_dim);
    if (p->idx_format != MSA_IDX_PLAIN && p->idx_format != MSA_IDX_MXFP8)
        return fail(MSA_ERR_INVALID_ARG, "idx_format %d unknown", p->idx_format);
    const int row = idx_row_bytes(*p);
    if (p->idx_dim < 1 || (row != 64 && row != 128 && row != 256))
        return fail(MSA_ERR_UNSUPPORTED, "idx_dim %d: an index-key row must be 64, 128 or 256 bytes", p->idx_dim);
    if (p->idx_format == MSA_IDX_MXFP8) {
        if (p->dtype != MSA_BF16) return fail(MSA_ERR_UNSUPPORTED, "MXFP8 index keys go with bf16 tensors");
        if (mode != DECODE_ONLY && !(mode == ANY_ROWS && p->q_len == 1))
            return fail(MSA_ERR_UNSUPPORTED, "MXFP8 index keys are read by the decode entries only");
        if (p->k_idx_scale == nullptr) return fail(MSA_ERR_INVALID_ARG, "k_idx_scale is NULL with MXFP8 index keys");
        if (!aligned16(p->k_idx_scale)) return fail(MSA_ERR_INVALID_ARG, "k_idx_scale is not 16-byte aligned");
        if (p->block_table == nullptr && p->max_seq_len % 16 != 0)
            return fail(MSA_ERR_UNSUPPORTED, "MXFP8 index keys need max_seq_len a multiple of 16");
    }
    if (!pow2(p->block_size) || p->block_size < 16 || p->block_size > 256)
        return fail(MSA_ERR_UNSUPPORTED, "block_size %d (a power of two in [16, 256])", p->block_size);
    if (p->top_k < 1) return fail(MSA_ERR_INVALID_ARG, "top_k %d < 1", p->top_k);
    if (p->top_k > kMaxTopK) return fail(MSA_ERR_UNSUPPORTED, "top_k %d > %d", p->top_k, kMaxTopK);
    if (p->max_seq_len < 1) return fail(MSA_ERR_INVALID_ARG, "max_seq_len %d < 1", p->max_seq_len);
    if ((long long)p->batch * p->n_kv_heads * p->max_seq_len >= (1LL << 31))
        return fail(MSA_ERR_UNSUPPORTED, "batch * n_kv_heads * max_seq_len must stay below 2^31 cache rows");
    if (!(p->softmax_scale > 0.f) || !std::isfinite(p->softmax_scale))
        return fail(MSA_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
    if (p->flags & ~(MSA_SCORES_TOKEN | MSA_SCORES_BLOCKMAX | MSA_DENSE | MSA_FORCE_SINK_LOCAL))
        return fail(MSA_ERR_INVALID_ARG, "unknown flags 0x%x", p->flags);
    if (p->q_len < 1) return fail(MSA_ERR_INVALID_ARG, "q_len %d < 1", p->q_len);
    if (mode == DECODE_ONLY && p->q_len != 1) return fail(MSA_ERR_INVALID_ARG, "decode entries take q_len = 1");
    if (mode == PREFILL_ONLY || (mode == ANY_ROWS && p->q_len > 1)) {
        if (p->q_start < 0 || (long long)p->q_start + p->q_len > p->max_seq_len)
            return fail(MSA_ERR_INVALID_ARG, "prefill rows [%d, %d) outside max_seq_len %d", p->q_start,
                        p->q_start + p->q_len, p->max_seq_len);
    }
    if (mode == DECODE_ONLY || (mode == ANY_ROWS && p->q_len == 1)) {
        if (p->seq_lens == nullptr) return fail(MSA_ERR_INVALID_ARG, "seq_lens is NULL");
    }
    if (p->block_table != nullptr) {
        if ((reinterpret_cast<uintptr_t>(p->block_table) & 3u) != 0)
            return fail(MSA_ERR_INVALID_ARG, "block_table is not 4-byte aligned");
        if (p->n_pages < 1) return fail(MSA_ERR_INVALID_ARG, "n_pages %d < 1 with a block table", p->n_pages);
        const int hmax = p->n_kv_heads > p->n_idx_k_heads ? p->n_kv_heads : p->n_idx_k_heads;
        if ((long long)p->n_pages * hmax * p->block_size >= (1LL << 31))
            return fail(MSA_ERR_UNSUPPORTED, "n_pages * heads * block_size must stay below 2^31 cache rows");
    }
    return MSA_OK;
}

// MXFP8 index keys: the scan reads their scales beside the codes.
void set_scales(ScanArgs &a, const msa_params_t &p) {
    if (p.idx_format != MSA_IDX_MXFP8) return;
    a.k_scale = p.k_idx_scale;
    a.k_scale_rows = (long long)a.cache.rows(p.batch, p.n_idx_k_heads, p.max_seq_len);
}

// Layout of the caches a call reads: contiguous, or pages named by the block table.
CacheMap cache_of(const msa_params_t &p) {
    CacheMap c{};
    if (p.block_table != nullptr) {
        c.table = p.block_table;
        c.nbt = (p.max_seq_len + p.block_size - 1) / p.block_size;
        c.n_pages = p.n_pages;
        c.page_log2 = __builtin_ctz((unsigned)p.block_size);
    }
    return c;
}

msa_status_t check_ptr(const void *ptr, const char *name, bool nullable = false) {
    if (ptr == nullptr) {
        if (nullable) return MSA_OK;
        return fail(MSA_ERR_INVALID_ARG, "%s is NULL", name);
    }
    if (!aligned16(ptr)) return fail(MSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return MSA_OK;
}

#define MSA_TRY(x)                          \
    do {                                    \
        msa_status_t st_ = (x);             \
        if (st_ != MSA_OK) return st_;      \
    } while (0)

int nb_max_of(const msa_params_t &p) { return (p.max_seq_len + p.block_size - 1) / p.block_size; }

}  // namespace

int num_sms() {
    int n = 0;
    return check_device(&n) == MSA_OK ? n : 0;
}

msa_status_t set_error(msa_status_t st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return st;
}

msa_status_t decode_fused_scratch_bytes(const msa_params_t *p, size_t *bytes) {
    MSA_TRY(check_params(p, DECODE_ONLY));
    int n_sm = 0;
    MSA_TRY(check_device(&n_sm));
    *bytes = decode_ws_layout(*p, true, true, n_sm).total;
    return MSA_OK;
}

// Groups that share one index-K stream, bf16 K/V (the tensor-core attention kernel): the scan
// keeps no per-piece lists and the attention kernel selects from every block's score.
static bool shared_stream_scores(const msa_params_t &p) {
    return p.n_kv_heads > p.n_idx_k_heads && p.dtype == MSA_BF16 && !(p.flags & MSA_DENSE);
}

DecodeWs decode_ws_layout(const msa_params_t &p, bool scan, bool attend, int n_sm) {
    DecodeWs L{};
    L.n_cta = n_sm < 256 ? n_sm : 256;
    if (L.n_cta < 1) L.n_cta = 1;
    const int n_seg = p.batch * p.n_idx_k_heads, gps = p.n_kv_heads / p.n_idx_k_heads;
    const int r = p.n_q_heads / p.n_kv_heads;
    size_t off = kStatusBytes;
    const bool large = p.top_k > kMaxTopKList;
    if (scan) {
        L.seg_info = off;
        off += round256((size_t)n_seg * sizeof(SegInfo));
        // large k: no per-piece lists; the scan leaves every block's score and a radix select
        // writes the ids.  Groups that share one index-K stream: no lists either; the attention
        // kernel selects from every block's score
        const size_t cand = (large || shared_stream_scores(p)) ? 0 : (size_t)n_seg * L.n_cta * gps * p.top_k * 4;
        L.cand_s = off;
        off += round256(cand);
        L.cand_i = off;
        off += round256(cand);
        L.tail_scores = off;
        off += round256((size_t)p.batch * p.n_kv_heads * nb_max_of(p) * 4);
        L.large_ids = off;
        off += round256(large ? (size_t)p.batch * p.n_kv_heads * p.top_k * 4 : 0);
    }
    if (attend) {
        if ((p.flags & MSA_DENSE) || large) {
            // many blocks per group: one CTA per SM (the bf16 warp-per-stage kernel) or about two
            // (fp32) over all (sequence, group) pairs
            const int nb = (p.flags & MSA_DENSE) ? nb_max_of(p) : p.top_k;
            const long long bg = (long long)p.batch * p.n_kv_heads;
            // one CTA per SM: no more splits than fill one wave (a second, short wave would
            // double the kernel's time); two per SM: round up
            long long S = wide_attention(p) ? n_sm / bg : (2LL * n_sm + bg - 1) / bg;
            if (S < 1) S = 1;
            if (S > kMaxSplits) S = kMaxSplits;
            if (S > nb) S = nb;
            L.blocks_per_split = (int)((nb + S - 1) / S);
            L.S = (nb + L.blocks_per_split - 1) / L.blocks_per_split;
        } else {
            // the splits of a (sequence, group) form one cluster; as many as one wave of CTAs holds:
            // the largest power of two <= kSparseSplits with batch * groups * S <= SMs (a second
            // wave of clusters would double the kernel's time)
            const long long bg = (long long)p.batch * p.n_kv_heads;
            int S = kSparseSplits;
            while (S > 1 && bg * S > n_sm) S >>= 1;
            L.S = p.top_k < S ? p.top_k : S;
            L.blocks_per_split = (p.top_k + L.S - 1) / L.S;
        }
        L.counters = off;
        off += round256((size_t)p.batch * p.n_kv_heads * 4);
        const size_t parts = (size_t)p.batch * p.n_kv_heads * L.S * r;
        L.part_o = off;
        off += round256(parts * p.head_dim * 4);
        L.part_lse = off;
        off += round256(parts * 4);
    }
    L.total = off;
    return L;
}

PrefillIdxPlan prefill_index_plan(const msa_params_t &p, int n_sm) {
    PrefillIdxPlan L{};
    L.n_mt = (p.q_len + 255) / 256;
    L.kt = p.top_k <= 8 ? 8 : p.top_k <= 16 ? 16 : p.top_k <= kMaxTopKList ? 32 : 0;
    // a row's block scores padded to whole 32-block windows (the stage writes them 16 at a time)
    L.blk_stride = ((p.q_start + p.q_len - 1) / p.block_size + 1 + 31) / 32 * 32;
    const long long units = (long long)L.n_mt * p.batch * p.n_kv_heads;
    const int max_tiles = prefill_unit_tiles(0, L.n_mt, p.q_len, p.q_start, p.block_size);
    const int gran = p.block_size > 128 ? p.block_size / 128 : 1;
    // segments per unit: the fewest that fill whole waves of CTAs (to within ~2 %), never
    // shorter than 64 tiles or one block
    L.n_seg = 1;
    double best = 0.0;
    for (int sgm = 1; sgm <= 16; ++sgm) {
        if (sgm > 1 && (max_tiles / sgm < 64 || max_tiles / sgm < gran)) break;
        const long long pieces = units * sgm;
        const long long waves = (pieces + n_sm - 1) / n_sm;
        const double eff = (double)pieces / ((double)waves * n_sm);
        if (eff > best + 0.02) {
            best = eff;
            L.n_seg = sgm;
        }
    }
    const long long pieces = units * L.n_seg;
    L.grid = (int)(pieces < n_sm ? pieces : n_sm);
    size_t off = kStatusBytes;
    L.counters = off;
    off += round256((size_t)units * 4);
    const size_t part = L.n_seg > 1 ? (size_t)units * L.n_seg * L.kt * 256 * 4 : 0;
    L.part_s = off;
    off += round256(part);
    L.part_i = off;
    off += round256(part);
    L.blk_scores = off;
    if (L.kt == 0) off += round256((size_t)p.batch * p.q_len * p.n_kv_heads * L.blk_stride * 4);
    L.total = off;
    return L;
}

// The stand-alone TopK keeps warp lists up to kMaxTopKList; beyond, a radix select per row reads
// block scores, which token scores first become in the workspace.
size_t maxpool_topk_ws_bytes(const msa_params_t &p) {
    if (p.top_k <= kMaxTopKList || (p.flags & MSA_SCORES_BLOCKMAX)) return kStatusBytes;
    return kStatusBytes + round256((size_t)p.batch * p.q_len * p.n_kv_heads * nb_max_of(p) * 4);
}

}  // namespace msa

using namespace msa;

// An NVTX range over one entry's launches, named after the entry (Nsight Systems / Compute show
// it; without a tool attached the calls return at once).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

extern "C" {

const char *msa_last_error_string(void) { return g_err.c_str(); }

const char *msa_status_string(msa_status_t s) {
    switch (s) {
        case MSA_OK: return "MSA_OK";
        case MSA_ERR_INVALID_ARG: return "MSA_ERR_INVALID_ARG";
        case MSA_ERR_UNSUPPORTED: return "MSA_ERR_UNSUPPORTED";
        case MSA_ERR_WORKSPACE: return "MSA_ERR_WORKSPACE";
        case MSA_ERR_CUDA: return "MSA_ERR_CUDA";
        case MSA_ERR_TIMEOUT: return "MSA_ERR_TIMEOUT";
    }
    return "unknown status";
}

size_t msa_workspace_size(const msa_params_t *p, int entry) {
    int n_sm = 0;
    switch (entry) {
        case MSA_ENTRY_INDEX_SCORE:
            if (check_params(p, ANY_ROWS) != MSA_OK) return (size_t)-1;
            return kStatusBytes;
        case MSA_ENTRY_MAXPOOL_TOPK:
            if (check_params(p, ANY_ROWS) != MSA_OK) return (size_t)-1;
            return maxpool_topk_ws_bytes(*p);
        case MSA_ENTRY_ATTN_DECODE:
            if (check_params(p, DECODE_ONLY) != MSA_OK || check_device(&n_sm) != MSA_OK) return (size_t)-1;
            return decode_ws_layout(*p, false, true, n_sm).total;
        case MSA_ENTRY_DECODE_FUSED:
            if (check_params(p, DECODE_ONLY) != MSA_OK || check_device(&n_sm) != MSA_OK) return (size_t)-1;
            return decode_ws_layout(*p, true, true, n_sm).total;
        case MSA_ENTRY_ATTN_PREFILL:
            if (check_params(p, PREFILL_ONLY) != MSA_OK) return (size_t)-1;
            return prefill_attn_plan(*p).total;
        case MSA_ENTRY_PREFILL_INDEX_TOPK:
            if (check_params(p, PREFILL_ONLY) != MSA_OK || check_device(&n_sm) != MSA_OK) return (size_t)-1;
            return prefill_index_plan(*p, n_sm).total;
        default:
            fail(MSA_ERR_INVALID_ARG, "unknown entry %d", entry);
            return (size_t)-1;
    }
}

msa_status_t msa_set_stage_events(void *const *events, int n_events) {
    if (n_events == 0) {
        g_n_stage_ev = 0;
        return MSA_OK;
    }
    if (n_events != 3 || events == nullptr) return fail(MSA_ERR_INVALID_ARG, "n_events must be 0 or 3");
    for (int i = 0; i < 3; ++i) {
        if (events[i] == nullptr) return fail(MSA_ERR_INVALID_ARG, "event %d is NULL", i);
        g_stage_ev[i] = (cudaEvent_t)events[i];
    }
    g_n_stage_ev = 3;
    return MSA_OK;
}

static cudaError_t stage_mark(int i, cudaStream_t s) {
    return g_n_stage_ev == 3 ? cudaEventRecord(g_stage_ev[i], s) : cudaSuccess;
}

msa_status_t msa_get_device_status(const void *ws, int *status, msa_stream_t stream) {
    if (ws == nullptr || status == nullptr) return fail(MSA_ERR_INVALID_ARG, "ws or status is NULL");
    cudaError_t e = cudaMemcpyAsync(status, ws, sizeof(int), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
    return MSA_OK;
}

msa_status_t msa_clear_device_status(void *ws, msa_stream_t stream) {
    if (ws == nullptr) return fail(MSA_ERR_INVALID_ARG, "ws is NULL");
    // the status word, the wait limit and the scan's counters (left non-zero by a scan that did not
    // end normally)
    cudaError_t e = cudaMemsetAsync(ws, 0, (kSchedWord + kTailPools + 1) * sizeof(unsigned), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
    return MSA_OK;
}

msa_status_t msa_set_wait_limit(void *ws, uint64_t limit_ns, msa_stream_t stream) {
    if (ws == nullptr) return fail(MSA_ERR_INVALID_ARG, "ws is NULL");
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(MSA_ERR_INVALID_ARG, "ws is not 256-byte aligned");
    cudaError_t e = launch_set_wait_limit(reinterpret_cast<int *>(ws), (unsigned long long)limit_ns, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "setting the wait limit");
    return MSA_OK;
}

msa_status_t msa_diag_wait_timeout(void *ws, size_t ws_bytes, msa_stream_t stream) {
    MSA_TRY(check_ptr(ws, "ws"));
    if (ws_bytes < kStatusBytes) return fail(MSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, kStatusBytes);
    int n_sm = 0;
    MSA_TRY(check_device(&n_sm));
    cudaError_t e = launch_wait_never(reinterpret_cast<int *>(ws), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "diagnostic wait launch");
    return MSA_OK;
}

msa_status_t msa_index_score(const msa_params_t *p, const void *q_idx, const void *k_idx, float *scores_out,
                             void *ws, size_t ws_bytes, msa_stream_t stream) {
    NvtxRange nvtx_range("msa_index_score");
    MSA_TRY(check_params(p, ANY_ROWS));
    const int mode = p->flags & (MSA_SCORES_TOKEN | MSA_SCORES_BLOCKMAX);
    if (mode != MSA_SCORES_TOKEN && mode != MSA_SCORES_BLOCKMAX)
        return fail(MSA_ERR_INVALID_ARG, "exactly one of MSA_SCORES_TOKEN / MSA_SCORES_BLOCKMAX must be set");
    if (p->flags & (MSA_DENSE | MSA_FORCE_SINK_LOCAL))
        return fail(MSA_ERR_INVALID_ARG, "MSA_DENSE and MSA_FORCE_SINK_LOCAL do not apply to index scores");
    MSA_TRY(check_ptr(q_idx, "q_idx"));
    MSA_TRY(check_ptr(k_idx, "k_idx"));
    MSA_TRY(check_ptr(scores_out, "scores_out"));
    MSA_TRY(check_ptr(ws, "ws"));
    if (ws_bytes < kStatusBytes) return fail(MSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, kStatusBytes);
    if (p->q_len != 1)
        return fail(MSA_ERR_UNSUPPORTED, "stored prefill index scores are not available; use msa_prefill_index_topk");
    int n_sm = 0;
    MSA_TRY(check_device(&n_sm));
    const cudaStream_t s = (cudaStream_t)stream;
    const int nb_max = nb_max_of(*p);
    const long long n_out = (long long)p->batch * p->n_kv_heads * (mode == MSA_SCORES_TOKEN ? p->max_seq_len : nb_max);
    cudaError_t e = launch_fill_neg_inf(scores_out, n_out, s);
    if (e != cudaSuccess) return cuda_fail(e, "fill");
    ScanArgs a{};
    a.q_idx = q_idx; a.k_idx = k_idx; a.seq_lens = p->seq_lens;
    a.B = p->batch; a.G = p->n_kv_heads; a.Hik = p->n_idx_k_heads; a.di = p->idx_dim; a.Bk = p->block_size;
    a.k = p->top_k; a.L_max = p->max_seq_len; a.nb_max = nb_max;
    a.n_cta = decode_ws_layout(*p, true, false, n_sm).n_cta;
    a.token_scores = mode == MSA_SCORES_TOKEN ? scores_out : nullptr;
    a.block_scores = mode == MSA_SCORES_BLOCKMAX ? scores_out : nullptr;
    a.sched = reinterpret_cast<unsigned *>(ws) + kSchedWord;
    a.status = reinterpret_cast<int *>(ws);
    a.cache = cache_of(*p);
    set_scales(a, *p);
    e = launch_decode_scan(a, p->dtype, idx_row_bytes(*p), p->n_kv_heads / p->n_idx_k_heads, s, false);
    if (e != cudaSuccess) return cuda_fail(e, "index scan launch");
    return MSA_OK;
}

msa_status_t msa_block_maxpool_topk(const msa_params_t *p, const float *scores_in, int32_t *ids_out,
                                    float *top_scores_out, void *ws, size_t ws_bytes, msa_stream_t stream) {
    NvtxRange nvtx_range("msa_block_maxpool_topk");
    MSA_TRY(check_params(p, ANY_ROWS));
    if (p->flags & (MSA_SCORES_TOKEN | MSA_DENSE))
        return fail(MSA_ERR_INVALID_ARG,
                    "only MSA_SCORES_BLOCKMAX and MSA_FORCE_SINK_LOCAL may be set for msa_block_maxpool_topk");
    MSA_TRY(check_ptr(scores_in, "scores_in"));
    MSA_TRY(check_ptr(ids_out, "ids_out"));
    MSA_TRY(check_ptr(top_scores_out, "top_scores_out", true));
    MSA_TRY(check_ptr(ws, "ws"));
    const size_t need = maxpool_topk_ws_bytes(*p);
    if (ws_bytes < need) return fail(MSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
    int n_sm = 0;
    MSA_TRY(check_device(&n_sm));
    if (p->top_k > kMaxTopKList) {
        LargeTopkArgs la{};
        la.seq_lens = p->seq_lens; la.rows = p->batch * p->q_len * p->n_kv_heads; la.q_len = p->q_len;
        la.q_start = p->q_start; la.G = p->n_kv_heads; la.Bk = p->block_size; la.k = p->top_k;
        la.L_max = p->max_seq_len; la.prefill = p->q_len > 1; la.force = (p->flags & MSA_FORCE_SINK_LOCAL) != 0;
        la.ids_out = ids_out; la.top_scores_out = top_scores_out;
        la.stride = nb_max_of(*p);
        cudaError_t e;
        if (p->flags & MSA_SCORES_BLOCKMAX) {
            la.scores = scores_in;
        } else {
            float *blk = reinterpret_cast<float *>(static_cast<unsigned char *>(ws) + kStatusBytes);
            if ((e = launch_token_block_max(la, scores_in, blk, (cudaStream_t)stream)) != cudaSuccess)
                return cuda_fail(e, "block max launch");
            la.scores = blk;
        }
        if ((e = launch_large_topk(la, (cudaStream_t)stream)) != cudaSuccess) return cuda_fail(e, "topk launch");
        return MSA_OK;
    }
    PoolTopkArgs a{};
    a.scores = scores_in; a.seq_lens = p->seq_lens; a.ids_out = ids_out; a.top_scores_out = top_scores_out;
    a.B = p->batch; a.q_len = p->q_len; a.q_start = p->q_start; a.G = p->n_kv_heads; a.Bk = p->block_size;
    a.k = p->top_k; a.L_max = p->max_seq_len; a.nb_max = nb_max_of(*p);
    a.is_block = (p->flags & MSA_SCORES_BLOCKMAX) != 0;
    a.force = (p->flags & MSA_FORCE_SINK_LOCAL) != 0;
    a.prefill = p->q_len > 1;
    cudaError_t e = launch_pool_topk(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "pool/topk launch");
    return MSA_OK;
}

static msa_status_t attend_decode(const msa_params_t *p, const void *q, const void *k_cache, const void *v_cache,
                                  const int32_t *ids, bool after_scan, const DecodeWs &L, unsigned char *wsb,
                                  void *o, int32_t *ids_out, float *lse, cudaStream_t s) {
    AttnArgs a{};
    a.q = q; a.k_cache = k_cache; a.v_cache = v_cache; a.seq_lens = p->seq_lens;
    a.ids_in = ids;
    if (after_scan && ids == nullptr) {  // select the group's list inside the attention kernel
        a.cand_s = reinterpret_cast<const float *>(wsb + L.cand_s);
        a.cand_i = reinterpret_cast<const int *>(wsb + L.cand_i);
        a.tail_scores = reinterpret_cast<const float *>(wsb + L.tail_scores);
        a.ids_out = ids_out;
        a.scores_only = shared_stream_scores(*p);
    }
    a.n_cta = L.n_cta;
    a.part_o = reinterpret_cast<float *>(wsb + L.part_o);
    a.part_lse = reinterpret_cast<float *>(wsb + L.part_lse);
    a.counters = reinterpret_cast<int *>(wsb + L.counters);
    a.o = o; a.lse = lse;
    a.B = p->batch; a.Hq = p->n_q_heads; a.G = p->n_kv_heads; a.Hik = p->n_idx_k_heads; a.D = p->head_dim;
    a.Bk = p->block_size; a.k = p->top_k; a.L_max = p->max_seq_len; a.r = p->n_q_heads / p->n_kv_heads;
    a.S = L.S; a.blocks_per_split = L.blocks_per_split; a.dense = (p->flags & MSA_DENSE) != 0;
    a.force = (p->flags & MSA_FORCE_SINK_LOCAL) != 0;
    a.scale_log2 = p->softmax_scale * 1.4426950408889634f;
    a.status = reinterpret_cast<int *>(wsb);
    a.cache = cache_of(*p);
    cudaError_t e;
    if (!after_scan) {  // the scan zeroes the counters in the fused path
        e = cudaMemsetAsync(a.counters, 0, (size_t)p->batch * p->n_kv_heads * 4, s);
        if (e != cudaSuccess) return cuda_fail(e, "clearing the split counters");
    }
    e = launch_decode_attn(a, p->dtype, s, after_scan);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    if (after_scan && (e = stage_mark(2, s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    return MSA_OK;
}

msa_status_t msa_sparse_attn_decode(const msa_params_t *p, const void *q, const void *k_cache, const void *v_cache,
                                    const int32_t *ids, void *o, float *lse, void *ws, size_t ws_bytes,
                                    msa_stream_t stream) {
    NvtxRange nvtx_range("msa_sparse_attn_decode");
    MSA_TRY(check_params(p, DECODE_ONLY));
    if (p->flags & (MSA_SCORES_TOKEN | MSA_SCORES_BLOCKMAX | MSA_FORCE_SINK_LOCAL))
        return fail(MSA_ERR_INVALID_ARG, "score and selection flags do not apply to attention from given ids");
    const bool dense = (p->flags & MSA_DENSE) != 0;
    MSA_TRY(check_ptr(q, "q"));
    MSA_TRY(check_ptr(k_cache, "k_cache"));
    MSA_TRY(check_ptr(v_cache, "v_cache"));
    MSA_TRY(check_ptr(ids, "ids", dense));
    MSA_TRY(check_ptr(o, "o"));
    MSA_TRY(check_ptr(lse, "lse", true));
    MSA_TRY(check_ptr(ws, "ws"));
    int n_sm = 0;
    MSA_TRY(check_device(&n_sm));
    const DecodeWs L = decode_ws_layout(*p, false, true, n_sm);
    if (ws_bytes < L.total) return fail(MSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
    return attend_decode(p, q, k_cache, v_cache, dense ? nullptr : ids, false, L,
                         reinterpret_cast<unsigned char *>(ws), o, nullptr, lse, (cudaStream_t)stream);
}

msa_status_t msa_decode_fused(const msa_params_t *p, const void *q, const void *q_idx, const void *k_cache,
                              const void *v_cache, const void *k_idx, void *o, int32_t *ids_out, float *lse, void *ws,
                              size_t ws_bytes, msa_stream_t stream) {
    NvtxRange nvtx_range("msa_decode_fused");
    MSA_TRY(check_params(p, DECODE_ONLY));
    if (p->flags & ~MSA_FORCE_SINK_LOCAL)
        return fail(MSA_ERR_INVALID_ARG,
                    "msa_decode_fused takes only MSA_FORCE_SINK_LOCAL (dense decode: msa_sparse_attn_decode + MSA_DENSE)");
    MSA_TRY(check_ptr(q, "q"));
    MSA_TRY(check_ptr(q_idx, "q_idx"));
    MSA_TRY(check_ptr(k_cache, "k_cache"));
    MSA_TRY(check_ptr(v_cache, "v_cache"));
    MSA_TRY(check_ptr(k_idx, "k_idx"));
    MSA_TRY(check_ptr(o, "o"));
    MSA_TRY(check_ptr(ids_out, "ids_out", true));
    MSA_TRY(check_ptr(lse, "lse", true));
    MSA_TRY(check_ptr(ws, "ws"));
    int n_sm = 0;
    MSA_TRY(check_device(&n_sm));
    const DecodeWs L = decode_ws_layout(*p, true, true, n_sm);
    if (ws_bytes < L.total) return fail(MSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
    unsigned char *wsb = reinterpret_cast<unsigned char *>(ws);
    const cudaStream_t s = (cudaStream_t)stream;
    ScanArgs a{};
    a.q_idx = q_idx; a.k_idx = k_idx; a.seq_lens = p->seq_lens;
    a.B = p->batch; a.G = p->n_kv_heads; a.Hik = p->n_idx_k_heads; a.di = p->idx_dim; a.Bk = p->block_size;
    a.k = p->top_k; a.L_max = p->max_seq_len; a.nb_max = nb_max_of(*p);
    a.n_cta = L.n_cta;
    a.cand_s = reinterpret_cast<float *>(wsb + L.cand_s);
    a.cand_i = reinterpret_cast<int *>(wsb + L.cand_i);
    a.seg_info = reinterpret_cast<SegInfo *>(wsb + L.seg_info);
    a.block_scores = reinterpret_cast<float *>(wsb + L.tail_scores);  // read back for the tails' blocks
    a.sched = reinterpret_cast<unsigned *>(wsb) + kSchedWord;
    a.counters = reinterpret_cast<int *>(wsb + L.counters);
    a.status = reinterpret_cast<int *>(wsb);
    a.cache = cache_of(*p);
    const bool large = p->top_k > kMaxTopKList;
    if (large || shared_stream_scores(*p)) {
        // every block's score (static ranges and tails alike) into the block-score region: for
        // the radix select (large k), or for the attention kernel's selection when groups share
        // one index-K stream (every scan CTA would hold a piece of it: too many lists to merge)
        a.cand_s = nullptr;
        a.cand_i = nullptr;
    }
    cudaError_t e = stage_mark(0, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    set_scales(a, *p);
    e = launch_decode_scan(a, p->dtype, idx_row_bytes(*p), p->n_kv_heads / p->n_idx_k_heads, s, false);
    if (e != cudaSuccess) return cuda_fail(e, "index scan launch");
    if (large) {
        if ((e = stage_mark(1, s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
        int32_t *ids = reinterpret_cast<int32_t *>(wsb + L.large_ids);
        LargeTopkArgs la{};
        la.scores = reinterpret_cast<const float *>(wsb + L.tail_scores);
        la.stride = nb_max_of(*p);
        la.seq_lens = p->seq_lens; la.rows = p->batch * p->n_kv_heads; la.q_len = 1; la.q_start = 0;
        la.G = p->n_kv_heads; la.Bk = p->block_size; la.k = p->top_k; la.L_max = p->max_seq_len;
        la.prefill = 0; la.force = (p->flags & MSA_FORCE_SINK_LOCAL) != 0;
        la.ids_out = ids;
        la.ids_copy = ids_out;
        if ((e = launch_large_topk(la, s)) != cudaSuccess) return cuda_fail(e, "topk launch");
        return attend_decode(p, q, k_cache, v_cache, ids, true, L, wsb, o, nullptr, lse, s);
    }
    if ((e = stage_mark(1, s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    return attend_decode(p, q, k_cache, v_cache, nullptr, true, L, wsb, o, ids_out, lse, s);
}

msa_status_t msa_decode_append(const msa_params_t *p, const void *k_new, const void *v_new, const void *k_idx_new,
                               void *k_cache, void *v_cache, void *k_idx, msa_stream_t stream) {
    NvtxRange nvtx_range("msa_decode_append");
    MSA_TRY(check_params(p, DECODE_ONLY));
    MSA_TRY(check_ptr(k_new, "k_new"));
    MSA_TRY(check_ptr(v_new, "v_new"));
    MSA_TRY(check_ptr(k_idx_new, "k_idx_new"));
    MSA_TRY(check_ptr(k_cache, "k_cache"));
    MSA_TRY(check_ptr(v_cache, "v_cache"));
    MSA_TRY(check_ptr(k_idx, "k_idx"));
    int n_sm = 0;
    MSA_TRY(check_device(&n_sm));
    cudaError_t e = launch_append(*p, cache_of(*p), k_new, v_new, k_idx_new, k_cache, v_cache, k_idx, (cudaStream_t)stream);
    if (e == cudaSuccess && p->idx_format == MSA_IDX_MXFP8)
        e = launch_mxfp8_append(*p, cache_of(*p), k_idx_new, static_cast<uint8_t *>(k_idx),
                                const_cast<uint8_t *>(p->k_idx_scale), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
    return MSA_OK;
}

msa_status_t msa_quantize_index_k(const msa_params_t *p, const void *src, long long rows, uint8_t *codes,
                                  uint8_t *scales, msa_stream_t stream) {
    NvtxRange nvtx_range("msa_quantize_index_k");
    if (p == nullptr) return fail(MSA_ERR_INVALID_ARG, "params is NULL");
    if (p->idx_dim != 64 && p->idx_dim != 128 && p->idx_dim != 256)
        return fail(MSA_ERR_UNSUPPORTED, "idx_dim %d: MXFP8 index keys take 64, 128 or 256 dims", p->idx_dim);
    if (rows < 0) return fail(MSA_ERR_INVALID_ARG, "rows %lld < 0", rows);
    MSA_TRY(check_ptr(src, "src"));
    MSA_TRY(check_ptr(codes, "codes"));
    MSA_TRY(check_ptr(scales, "scales"));
    int n_sm = 0;
    MSA_TRY(check_device(&n_sm));
    cudaError_t e = launch_mxfp8_quantize(src, rows, p->idx_dim, codes, scales, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "quantise launch");
    return MSA_OK;
}

msa_status_t msa_sparse_attn_prefill(const msa_params_t *p, const void *q, const void *k_cache, const void *v_cache,
                                     const int32_t *ids, void *o, float *lse, void *ws, size_t ws_bytes,
                                     msa_stream_t stream) {
    NvtxRange nvtx_range("msa_sparse_attn_prefill");
    MSA_TRY(check_params(p, PREFILL_ONLY));
    if (p->flags != 0) return fail(MSA_ERR_INVALID_ARG, "msa_sparse_attn_prefill takes no flags");
    if (p->dtype != MSA_BF16) return fail(MSA_ERR_UNSUPPORTED, "prefill entries take bf16 only");
    if (p->block_size != 64 && p->block_size != 128)
        return fail(MSA_ERR_UNSUPPORTED, "prefill attention takes block_size 64 or 128");
    const int r = p->n_q_heads / p->n_kv_heads;
    if (128 % r != 0) return fail(MSA_ERR_UNSUPPORTED, "prefill attention needs a group size dividing 128");
    if ((long long)p->batch * p->q_len * p->n_q_heads >= (1LL << 31))
        return fail(MSA_ERR_UNSUPPORTED, "prefill attention: batch * q_len * n_q_heads must stay below 2^31 rows");
    MSA_TRY(check_ptr(q, "q"));
    MSA_TRY(check_ptr(k_cache, "k_cache"));
    MSA_TRY(check_ptr(v_cache, "v_cache"));
    MSA_TRY(check_ptr(ids, "ids"));
    MSA_TRY(check_ptr(o, "o"));
    MSA_TRY(check_ptr(lse, "lse", true));
    MSA_TRY(check_ptr(ws, "ws"));
    const PrefillAttnPlan L = prefill_attn_plan(*p);
    if (ws_bytes < L.total) return fail(MSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
    int n_sm = 0;
    MSA_TRY(check_device(&n_sm));
    PrefillAttnArgs a{};
    a.ids = ids; a.o = o; a.lse = lse;
    a.B = p->batch; a.T = p->q_len; a.Hq = p->n_q_heads; a.G = p->n_kv_heads; a.D = p->head_dim;
    a.Bk = p->block_size; a.k = p->top_k; a.q_start = p->q_start; a.L_max = p->max_seq_len; a.r = r;
    a.scale_log2 = p->softmax_scale * 1.4426950408889634f;
    a.status = reinterpret_cast<int *>(ws);
    a.cache = cache_of(*p);
    unsigned char *w = static_cast<unsigned char *>(ws);
    a.counts = reinterpret_cast<int *>(w + L.counts);
    a.offsets = reinterpret_cast<int *>(w + L.offsets);
    a.n_tiles = reinterpret_cast<int *>(w + L.n_tiles);
    a.block_sums = reinterpret_cast<int *>(w + L.block_sums);
    a.rank = reinterpret_cast<int *>(w + L.rank);
    a.members = reinterpret_cast<int *>(w + L.members);
    a.tiles = reinterpret_cast<int4 *>(w + L.tiles);
    a.part_lse = reinterpret_cast<float *>(w + L.part_lse);
    a.part_o = reinterpret_cast<__nv_bfloat16 *>(w + L.part_o);
    const char *why = "";
    cudaError_t e = launch_prefill_attn(a, q, k_cache, v_cache, n_sm, (cudaStream_t)stream, &why);
    if (e != cudaSuccess) return cuda_fail(e, why);
    return MSA_OK;
}

msa_status_t msa_prefill_index_topk(const msa_params_t *p, const void *q_idx, const void *k_idx, int32_t *ids_out,
                                    float *top_scores_out, void *ws, size_t ws_bytes, msa_stream_t stream) {
    NvtxRange nvtx_range("msa_prefill_index_topk");
    MSA_TRY(check_params(p, PREFILL_ONLY));
    if (p->flags & ~MSA_FORCE_SINK_LOCAL)
        return fail(MSA_ERR_INVALID_ARG, "msa_prefill_index_topk takes only MSA_FORCE_SINK_LOCAL");
    if (p->dtype != MSA_BF16) return fail(MSA_ERR_UNSUPPORTED, "prefill entries take bf16 only");
    if (p->idx_dim != 64) return fail(MSA_ERR_UNSUPPORTED, "prefill index scoring takes idx_dim 64");
    if (p->block_size < 32) return fail(MSA_ERR_UNSUPPORTED, "prefill index scoring takes block_size >= 32");
    if (p->block_table != nullptr && p->block_size < 128)
        return fail(MSA_ERR_UNSUPPORTED, "prefill index scoring of a paged cache takes block_size >= 128");
    MSA_TRY(check_ptr(q_idx, "q_idx"));
    MSA_TRY(check_ptr(k_idx, "k_idx"));
    MSA_TRY(check_ptr(ids_out, "ids_out"));
    MSA_TRY(check_ptr(top_scores_out, "top_scores_out", true));
    MSA_TRY(check_ptr(ws, "ws"));
    int n_sm = 0;
    MSA_TRY(check_device(&n_sm));
    const PrefillIdxPlan L = prefill_index_plan(*p, n_sm);
    if (ws_bytes < L.total) return fail(MSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
    PrefillIdxArgs a{};
    a.B = p->batch; a.T = p->q_len; a.G = p->n_kv_heads; a.Hik = p->n_idx_k_heads; a.Bk = p->block_size;
    a.k = p->top_k; a.q_start = p->q_start; a.L_max = p->max_seq_len;
    a.force = (p->flags & MSA_FORCE_SINK_LOCAL) != 0;
    a.n_mt = L.n_mt;
    a.n_seg = L.n_seg;
    a.ids_out = ids_out; a.top_scores_out = top_scores_out;
    unsigned char *w = static_cast<unsigned char *>(ws);
    a.counters = reinterpret_cast<int *>(w + L.counters);
    a.part_s = reinterpret_cast<float *>(w + L.part_s);
    a.part_i = reinterpret_cast<int *>(w + L.part_i);
    a.status = reinterpret_cast<int *>(ws);
    a.cache = cache_of(*p);
    if (L.kt == 0) {
        a.blk_scores = reinterpret_cast<float *>(w + L.blk_scores);
        a.blk_stride = L.blk_stride;
    }
    const char *why = "clearing the prefill index piece counters";
    cudaError_t e = cudaMemsetAsync(a.counters, 0, (size_t)L.n_mt * p->batch * p->n_kv_heads * 4, (cudaStream_t)stream);
    if (e == cudaSuccess) e = launch_prefill_index(a, q_idx, k_idx, L.grid, (cudaStream_t)stream, &why);
    if (e == cudaSuccess && L.kt == 0) {
        // large k: the k best of each row's stored block scores
        LargeTopkArgs la{};
        la.scores = a.blk_scores; la.stride = L.blk_stride;
        la.rows = p->batch * p->q_len * p->n_kv_heads; la.q_len = p->q_len; la.q_start = p->q_start;
        la.G = p->n_kv_heads; la.Bk = p->block_size; la.k = p->top_k; la.L_max = p->max_seq_len;
        la.prefill = 1; la.force = a.force;
        la.ids_out = ids_out; la.top_scores_out = top_scores_out;
        why = "prefill large-k TopK launch";
        e = launch_large_topk(la, (cudaStream_t)stream);
    }
    if (e != cudaSuccess) return cuda_fail(e, why);
    return MSA_OK;
}

}  // extern "C"
