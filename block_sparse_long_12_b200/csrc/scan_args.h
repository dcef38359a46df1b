// Declarations of the decode index scan (Step 1 for decode) shared by the
// scan kernel, its callers and the attention kernel that reads its results.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace msa {

constexpr size_t kStatusBytes = 256;  // workspace head: device status word, scan counters, padding
constexpr int kSchedWord = 4;          // ws words 4..4+kTailPools: tail-pool counters, then finished CTAs
constexpr int kTailPools = 4;          // interleaved pools (counters) of the scan's shared tail

// Blocks of a segment of nb blocks that the index scan hands out dynamically
// (the last quarter); the first nb - scan_tail_blocks(nb) are split equally
// between the CTAs.
__host__ __device__ inline int scan_tail_blocks(int nb) { return nb / 4; }

// Where token `tok` of head h of sequence b sits in a cache of H heads (rows of head_dim or idx_dim
// elements): contiguous [B, H, L_max, row], or paged [n_pages, H, page, row] where a block table of
// nbt entries per sequence names the page of each block of page (= block_size) tokens.  Page ids
// outside [0, n_pages) are out of contract; they are clamped so that nothing is read outside the
// pool.
struct CacheMap {
    const int *table;  // nullptr: contiguous
    int nbt;           // table entries per sequence
    int n_pages;
    int page_log2;     // log2 of the tokens per page
    __host__ __device__ inline int row(int b, int h, int H, int L_max, int tok) const {
        if (table == nullptr) return (b * H + h) * L_max + tok;
        int pg = table[b * nbt + (tok >> page_log2)];
        pg = pg < 0 ? 0 : (pg >= n_pages ? n_pages - 1 : pg);
        return ((pg * H + h) << page_log2) + (tok & ((1 << page_log2) - 1));
    }
    // rows of the tensor a TMA map covers
    __host__ __device__ inline unsigned long long rows(int B, int H, int L_max) const {
        return table == nullptr ? (unsigned long long)B * H * L_max : ((unsigned long long)n_pages * H) << page_log2;
    }
};

// ---- decode index scan (Step 1 for decode): persistent, 1 CTA per SM
constexpr int kScanChunkBytes = 8192;   // ring stage: bytes of index keys per TMA copy

// A segment is the index-K stream of one (sequence b, index-K head): blocks
// 0..nb_b-1 of k_idx[b, hik].  The scan splits the concatenation of all
// segments' first nb_b - scan_tail_blocks(nb_b) blocks evenly over its CTAs;
// a CTA's share of one segment is a piece.
struct SegInfo {
    int first_cta;  // CTA holding the segment's first block (-1: empty segment)
    int n_pieces;   // CTAs that touched it
};

struct ScanArgs {
    const void *q_idx;
    const void *k_idx;
    const int *seq_lens;
    int B, G, Hik, di, Bk, k, L_max, nb_max;
    int n_cta;
    int chunk_tokens;      // tokens per bulk copy (set by the launcher)
    float *cand_s;  // [n_seg, n_cta, G/Hik, k] per-piece sorted top-k (nullable)
    int *cand_i;
    SegInfo *seg_info;     // [n_seg] (written by CTA 0 when cand_s != nullptr)
    unsigned *sched;       // [kTailPools + 1] tail-pool counters and finished CTAs (workspace head)
    float *token_scores;   // [B, 1, G, L_max] (nullable)
    float *block_scores;   // [B, 1, G, nb_max] (nullable)
    int *counters;         // [B, G] attention arrival counters, zeroed by CTA 0 (nullable)
    int *status;
    CacheMap cache;        // index-key cache layout (contiguous or paged)
    // MXFP8 index keys: E8M0 scales [rows, di / 32] beside the E4M3 codes (nullptr: plain keys);
    // rows = the code tensor's rows, a multiple of 16
    const uint8_t *k_scale;
    long long k_scale_rows;
    // the stream's TMA loads evict-first in L2 (set by the launcher for streams of at most
    // kEvictFirstMaxBytes; evict-normal beyond)
    int stream_evict_first;
};

}  // namespace msa
