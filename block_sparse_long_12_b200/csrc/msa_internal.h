// Internal declarations shared by the MSA translation units (host + device).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "msa.h"
#include "scan_args.h"

namespace msa {

// Bounded device-side waits give up after this long and report MSA_ERR_TIMEOUT,
// unless the workspace header holds another limit (msa_set_wait_limit).
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr int kWaitLimitWord = 2;  // int words 2..3 of the workspace header: wait limit in ns (0: default)

constexpr int kMaxBatch = 1024;
constexpr int kMaxTopK = 1024;          // largest top_k (decode entries and the stand-alone TopK)
constexpr int kMaxTopKList = 32;        // largest top_k of the warp-list paths (fused prefill index, its attention)
constexpr int kMaxGroupsPerSeg = 8;   // n_kv_heads / n_idx_k_heads handled by one index-K stream
constexpr int kMaxPiecesPerSeg = 256; // lists merged per (segment, group) by one warp (8 per lane)

// ---- decode sparse attention (Step 2 for decode)
constexpr int kAttnThreads = 256;
constexpr int kMaxSplits = 64;           // dense decode: splits per (sequence, group)
constexpr int kSparseSplits = 8;         // sparse decode: splits (= cluster size) per (sequence, group)

struct AttnArgs {
    const void *q;
    const void *k_cache;
    const void *v_cache;
    const int *seq_lens;
    const int *ids_in;         // [B, 1, G, k] given selection (unused with dense or cand_s)
    const float *cand_s;       // scan candidates [n_seg, n_cta, G/Hik, k]: select in the kernel (fused decode)
    const int *cand_i;
    const float *tail_scores;  // [B, G, nb_max] block scores of the segments' tails (fused decode)
    int scores_only;           // groups share one index-K stream: no lists, every block's score in tail_scores
    int n_cta;
    int *ids_out;              // nullable (fused decode)
    float *top_scores_out;     // nullable (fused decode)
    float *part_o;             // [B, G, S, r, D] fp32, normalised per split
    float *part_lse;           // [B, G, S, r] log2-domain normaliser
    int *counters;             // [B, G] arrival counts, zero on entry; reset by the last split
    void *o;                   // [B, 1, Hq, D]
    float *lse;                // nullable, natural log
    int B, Hq, G, Hik, D, Bk, k, L_max, r;
    int S, blocks_per_split, dense;
    float scale_log2;          // softmax_scale * log2(e)
    int ring_bytes, nst;       // set by the launcher
    int cluster;               // > 1: the S splits of a (b, g) form one cluster and merge in shared memory
    int force;                 // MSA_FORCE_SINK_LOCAL: the selection keeps block 0 and the last block
    int *status;
    CacheMap cache;            // K/V cache layout (contiguous or paged)
};

struct PoolTopkArgs {
    const float *scores;       // token [rows, L_max] or block [rows, nb_max]
    const int *seq_lens;
    int32_t *ids_out;
    float *top_scores_out;
    int B, q_len, q_start, G, Bk, k, L_max, nb_max, is_block, prefill;
    int force;                 // MSA_FORCE_SINK_LOCAL: block 0 and the row's own block rank first
};

// Large-k TopK of stored block scores, one CTA per row (b, t, g).
struct LargeTopkArgs {
    const float *scores;       // block scores: row r at scores + r * stride
    long long stride;          // nb_max
    const int *seq_lens;       // decode rows: pos = seq_lens[b] - 1
    int rows, q_len, q_start, G, Bk, k, L_max, prefill, force;
    int32_t *ids_out;          // [rows, k]
    int32_t *ids_copy;         // nullable: a second copy of ids_out
    float *top_scores_out;     // nullable
};

struct PrefillIdxArgs {
    int B, T, G, Hik, Bk, k, q_start, L_max;
    int force;                 // MSA_FORCE_SINK_LOCAL: block 0 and the row's own block rank first
    int n_mt;                  // 256-row query tiles per (b, g)
    int n_seg;                 // key segments per unit
    int32_t *ids_out;          // [B, T, G, k]
    float *top_scores_out;     // nullable
    int *counters;             // [units] segments finished (zeroed before the launch)
    float *part_s;             // [units][n_seg][Kt][256] per-segment row lists of split units
    int *part_i;
    int *status;
    CacheMap cache;            // index-key cache layout (paged: pages of a multiple of 128 tokens)
    // large k: every visible block's score, row (b * T + t) * G + g at blk_scores + row * blk_stride
    // (the radix select takes the k best afterwards); null when the epilogue keeps the lists
    float *blk_scores;
    long long blk_stride;      // blocks visible to the call's last row
};

// Key tiles (128 keys) of the i-th prefill index unit in processing order:
// query rows [m0, m0 + 256) of tile mt = n_mt - 1 - i (latest rows first)
// see keys up to the end of the block holding their last position.
__host__ __device__ inline int prefill_unit_tiles(int i, int n_mt, int T, int q_start, int Bk) {
    const int m0 = (n_mt - 1 - i) * 256;
    const int last = m0 + 255 < T - 1 ? m0 + 255 : T - 1;
    const int nb_last = (q_start + last) / Bk;
    return ((nb_last + 1) * Bk + 127) / 128;
}

// Key tiles of one segment of a unit with nt tiles cut into n_seg segments
// (a whole number of blocks of Bk keys).
__host__ __device__ inline int prefill_seg_tiles(int nt, int n_seg, int Bk) {
    const int gran = Bk > 128 ? Bk / 128 : 1;
    const int per = (nt + n_seg - 1) / n_seg;
    return (per + gran - 1) / gran * gran;
}

// How a prefill index call splits its work and where its scratch lives.
struct PrefillIdxPlan {
    int n_mt, n_seg, grid, kt;  // kt 0: large k (block scores stored, then the radix select)
    long long blk_stride;
    size_t counters, part_s, part_i, blk_scores, total;
};
PrefillIdxPlan prefill_index_plan(const msa_params_t &p, int n_sm);

// Prefill sparse attention, block-major: the (row, selected block) pairs of up to
// kPrefillRowsPerPass query rows are bucketed by block; a tile is up to 128 / r member
// rows' r heads against one block, giving one partial output per pair that a merge
// combines per row by log-sum-exp.
constexpr int kPrefillRowsPerPass = 8192;
// Rows per pass for top_k blocks per row: kPrefillRowsPerPass up to kMaxTopKList, fewer beyond
// so that a pass's (row, block) pairs -- and its per-pair partials -- stay within those of
// kPrefillRowsPerPass rows of kMaxTopKList blocks.
__host__ __device__ inline int prefill_rows_per_pass(int top_k) {
    return top_k <= kMaxTopKList ? kPrefillRowsPerPass : kPrefillRowsPerPass * kMaxTopKList / top_k;
}
// A tile member is (row of the pass << kSlotBits) | slot of the row's list (slot < kMaxTopK).
constexpr int kSlotBits = 10;

struct PrefillAttnArgs {
    const int *ids;            // [B, T, G, k]
    void *o;                   // [B, T, Hq, D] bf16
    float *lse;                // [B, T, Hq] nullable
    int B, T, Hq, G, D, Bk, k, q_start, L_max, r;
    float scale_log2;
    int *status;
    CacheMap cache;            // K/V cache layout (contiguous or paged)
    // one pass over query rows [t0, t0 + Tn)
    int t0, Tn;
    int nbv;                   // blocks visible to the pass's last row: buckets per (b, g)
    int tt;                    // member rows per tile, 128 / r
    int *counts;               // [B*G*nbv] pairs per bucket (zeroed before the pass)
    int *offsets;              // [B*G*nbv] first member of each bucket
    int *rank;                 // [B*Tn*G*k] rank of each pair in its bucket (-1: not attended)
    int *members;              // [pairs] member (tt << kSlotBits) | slot, grouped by bucket
    int4 *tiles;               // [max_tiles] (bucket, first member, member count, 0)
    int *n_tiles;
    int *block_sums;           // [2 * scan blocks] pairs and tiles of each scan block's buckets
    __nv_bfloat16 *part_o;     // [B*Tn*G*k][D/8][r][8] per-pair output (chunk-major), normalised by the pair's sum
    float *part_lse;           // [B*Tn*G*k][r] per-pair log2 normaliser
};

// Workspace of one prefill attention call (offsets in bytes).
struct PrefillAttnPlan {
    int rows, nbv_max, max_tiles;
    size_t counts, offsets, n_tiles, block_sums, rank, members, tiles, part_lse, part_o, total;
};
PrefillAttnPlan prefill_attn_plan(const msa_params_t &p);

struct FillArgs {
    float *scores;
    long long n;
};

// Workspace layout of the decode entries (offsets in bytes from ws).
struct DecodeWs {
    size_t seg_info, cand_s, cand_i, tail_scores, large_ids, counters, part_o, part_lse, total;
    int n_cta, S, blocks_per_split;
};
DecodeWs decode_ws_layout(const msa_params_t &p, bool scan, bool attend, int n_sm);
bool wide_attention(const msa_params_t &p);  // bf16 and (MSA_DENSE or top_k > kMaxTopKList)

// launchers (return cudaError_t of the launch)
cudaError_t launch_fill_neg_inf(float *p, long long n, cudaStream_t s);
cudaError_t launch_decode_scan(ScanArgs a, int dtype, int row_bytes, int gps, cudaStream_t s, bool pdl);
cudaError_t launch_decode_attn(const AttnArgs &a, int dtype, cudaStream_t s, bool pdl);
cudaError_t launch_pool_topk(const PoolTopkArgs &a, cudaStream_t s);
cudaError_t launch_large_topk(const LargeTopkArgs &a, cudaStream_t s);
cudaError_t launch_token_block_max(const LargeTopkArgs &a, const float *tok, float *blk, cudaStream_t s);
cudaError_t launch_prefill_attn(PrefillAttnArgs a, const void *q, const void *k_cache, const void *v_cache, int n_sm,
                                cudaStream_t s, const char **why);
cudaError_t launch_prefill_index(const PrefillIdxArgs &a, const void *q_idx, const void *k_idx, int n_sm,
                                 cudaStream_t s, const char **why);
cudaError_t launch_set_wait_limit(int *ws, unsigned long long limit_ns, cudaStream_t s);
cudaError_t launch_mxfp8_quantize(const void *src, long long rows, int di, uint8_t *codes, uint8_t *scales,
                                  cudaStream_t s);
cudaError_t launch_mxfp8_append(const msa_params_t &p, const CacheMap &cache, const void *ki_new, uint8_t *codes,
                                uint8_t *scales, cudaStream_t s);
cudaError_t launch_append(const msa_params_t &p, const CacheMap &cache, const void *k_new, const void *v_new,
                          const void *ki_new, void *k, void *v, void *ki, cudaStream_t s);
cudaError_t launch_wait_never(int *ws, cudaStream_t s);

int num_sms();

// set the calling thread's error string and return `st`
msa_status_t set_error(msa_status_t st, const char *fmt, ...);
// scratch bytes msa_decode_fused needs for these params (checks params and device first)
msa_status_t decode_fused_scratch_bytes(const msa_params_t *p, size_t *bytes);

// TMA tensor maps (host); false if the driver cannot encode the map
bool encode_2d(CUtensorMap *map, CUtensorMapDataType dt, void *base, unsigned long long inner,
               unsigned long long rows, unsigned long long row_stride_bytes, unsigned box_x, unsigned box_y,
               CUtensorMapSwizzle swizzle);
bool encode_3d(CUtensorMap *map, CUtensorMapDataType dt, void *base, const unsigned long long dims[3],
               const unsigned long long strides_bytes[2], const unsigned box[3], CUtensorMapSwizzle swizzle);

}  // namespace msa
