/*
 * msa.h -- C ABI of the B200 (sm_100a) MiniMax Sparse Attention hot path.
 *
 * The method (page "MiniMax wird duenn: M3-Attention anhand eines einzigen
 * Diagramms entschluesselt", atlascloud.ai, section 1 and Figure 1) is a GQA
 * attention block in two steps:
 *   Step 1, index branch: each KV group g has one small index query q_idx;
 *     every cached token j carries an index key k_idx[j]; token scores
 *     s_j = q_idx . k_idx[j] are reduced per fixed block of block_size tokens
 *     by their maximum ("Block Max Pool"), and TopK keeps the top_k blocks of
 *     the group.
 *   Step 2, sparse branch: every query head of the group (contiguous heads:
 *     head h belongs to group h / (n_q_heads / n_kv_heads)) runs exact softmax
 *     attention over only the selected blocks of the real, uncompressed K/V.
 *
 * Readings taken where the page is silent (its formulas were lost):
 *   - index score: raw dot product, no scale, no activation, fp32 accumulate;
 *   - causality: a query at position pos sees tokens 0..pos; a block is
 *     eligible if it holds any visible token, its score is the max over its
 *     visible tokens only, and attention masks keys after pos;
 *   - decode: pos = seq_lens[b] - 1 (the new token's K/V and index key are
 *     already in the cache); prefill chunk: pos = q_start + t;
 *   - top-k order: higher score first, ties to the lower block id; with fewer
 *     than top_k valid blocks all are taken and ids are padded with -1;
 *   - index-K head of group g: g mod n_idx_k_heads (1 shared head, or one per
 *     KV group);
 *   - softmax: z = softmax_scale * q . k, no bias, sink or soft-cap.
 *
 * Layouts (all contiguous, row-major, element type = params.dtype):
 *   q      [B, q_len, n_q_heads, head_dim]
 *   q_idx  [B, q_len, G, idx_dim]                       G = n_kv_heads
 *   k, v   [B, n_kv_heads, max_seq_len, head_dim]       (caches)
 *   k_idx  [B, n_idx_k_heads, max_seq_len, idx_dim]     (index-key cache)
 *   ids    int32 [B, q_len, G, top_k]
 *   o      [B, q_len, n_q_heads, head_dim]               (params.dtype)
 *   lse    fp32 [B, q_len, n_q_heads]   natural-log softmax normaliser
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are caller-owned device memory, 16-byte aligned.
 *     The library never allocates, frees or synchronises: work is enqueued on
 *     `stream` and returns immediately.
 *   - Scratch memory comes from the caller: `ws` of at least
 *     msa_workspace_size(params, entry) bytes (256-byte aligned).  Each call
 *     overwrites the workspace; calls that share a workspace must not overlap.
 *     Its first 256 bytes hold the device status word, the limit of the
 *     kernels' bounded waits (msa_set_wait_limit; 0 = one second) and the
 *     index scan's work counters (msa_index_score, msa_decode_fused), which
 *     the scan returns to zero when it ends: zero-fill a workspace once before
 *     its first use (a cudaMemset or a zeroed allocation).
 *   - Arguments are checked before anything is enqueued; on error nothing is
 *     launched and the call returns the status (text: msa_last_error_string).
 *   - A CUDA launch error returns MSA_ERR_CUDA.  Devices other than
 *     compute capability 10.0 return MSA_ERR_UNSUPPORTED.
 *   - seq_lens is a device pointer; values outside [1, max_seq_len] are out of
 *     contract: kernels clamp them and never read outside the caches.
 *   - Non-finite inputs are out of contract (results undefined, no fault).
 *   - Each compute entry encloses its launches in an NVTX range named after it
 *     (seen by Nsight tools; a no-op without one attached).
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

typedef struct CUstream_st *msa_stream_t; /* same type as cudaStream_t */

typedef enum {
    MSA_OK = 0,
    MSA_ERR_INVALID_ARG = 1, /* null pointer, bad shape, misalignment        */
    MSA_ERR_UNSUPPORTED = 2, /* valid but not implemented (dims, dtype, GPU)  */
    MSA_ERR_WORKSPACE = 3,   /* ws_bytes < msa_workspace_size(...)           */
    MSA_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed          */
    MSA_ERR_TIMEOUT = 5      /* a bounded device-side wait ran out            */
} msa_status_t;

typedef enum { MSA_F32 = 0, MSA_BF16 = 1 } msa_dtype_t;

/* params.idx_format: storage of the index-key cache k_idx */
typedef enum {
    MSA_IDX_PLAIN = 0,   /* params.dtype, like every other tensor                    */
    MSA_IDX_MXFP8 = 1    /* MXFP8: E4M3 codes plus one E8M0 scale per 32 dims (below) */
} msa_idx_format_t;

/* params.flags */
enum {
    MSA_SCORES_TOKEN = 1,    /* token scores s_j  [B, q_len, G, max_seq_len]  */
    MSA_SCORES_BLOCKMAX = 2, /* block scores S_n  [B, q_len, G, nb_max]       */
    MSA_DENSE = 8,           /* attend every visible block (plain GQA), ids unused */
    MSA_FORCE_SINK_LOCAL = 16 /* TopK always keeps block 0 and the query's own block */
};
/*
 * MSA_FORCE_SINK_LOCAL (accepted by msa_decode_fused, msa_decode_fused_noalloc,
 * msa_block_maxpool_topk and msa_prefill_index_topk): the selection of a query at
 * position pos always holds the sink block 0 and the local block floor(pos / Bk),
 * the block of the query itself.  They rank above every other block, between
 * themselves by block id (sink first), and their reported score is +inf; the
 * remaining top_k - 2 places (top_k - 1 when pos < Bk, where the two are one
 * block) go to the best other blocks in the usual order.  With top_k = 1 only
 * the sink is kept.  No page fixes such a rule: the atlascloud.ai page, section 2
 * ("Drei bewusste Abgrenzungen", third point), only guesses that an attention
 * sink and positional encoding stand in for NSA's dropped sliding window.  It is
 * offered here as an option, off by default.
 */

/* entry ids for msa_workspace_size */
enum {
    MSA_ENTRY_INDEX_SCORE = 0,
    MSA_ENTRY_MAXPOOL_TOPK = 1,
    MSA_ENTRY_ATTN_DECODE = 2,
    MSA_ENTRY_ATTN_PREFILL = 3,
    MSA_ENTRY_DECODE_FUSED = 4,
    MSA_ENTRY_PREFILL_INDEX_TOPK = 5
};

typedef struct {
    int batch;            /* B >= 1                                            */
    int n_q_heads;        /* multiple of n_kv_heads                            */
    int n_kv_heads;       /* G, the number of GQA groups                      */
    int n_idx_k_heads;    /* 1 or n_kv_heads                                   */
    int head_dim;         /* D: 64 or 128                                      */
    int idx_dim;          /* di: idx_dim * sizeof(elem) in {64, 128, 256} bytes */
    int block_size;       /* Bk: 16..256, power of two                         */
    int top_k;            /* 1..1024                                           */
    int q_len;            /* decode entries: 1; prefill: chunk length          */
    int q_start;          /* prefill: absolute position of query row 0         */
    int max_seq_len;      /* Lmax, the caches' token stride                    */
    const int32_t *seq_lens; /* device int32[B]: cached length incl. current token(s) */
    float softmax_scale;  /* > 0; 1/sqrt(head_dim) in the usual attention      */
    int dtype;            /* msa_dtype_t; prefill entries take MSA_BF16 only   */
    int flags;            /* MSA_SCORES_* / MSA_DENSE / MSA_FORCE_SINK_LOCAL   */
    const int32_t *block_table; /* NULL: contiguous caches; else paged, see below */
    int n_pages;          /* pages in each pool when block_table != NULL       */
    int idx_format;       /* msa_idx_format_t (0: plain)                       */
    const uint8_t *k_idx_scale; /* MSA_IDX_MXFP8: the index keys' scales, below */
} msa_params_t;
/*
 * MXFP8 index keys (idx_format = MSA_IDX_MXFP8; decode entries and
 * msa_index_score with q_len 1, dtype MSA_BF16, idx_dim 64, 128 or 256): k_idx
 * holds one FP8 E4M3 code per index dimension (uint8, [.., idx_dim]) and
 * k_idx_scale one E8M0 byte per 32 of them ([.., idx_dim / 32], same row
 * order as k_idx, contiguous or paged alike); key value = 2^(scale - 127) *
 * E4M3(code).  The index query stays bf16 and the scores accumulate in fp32.
 * The pages name MXFP8 only as the format of the official quantised checkpoints
 * (docs.clore.ai "MiniMax M3", deployment table and checkpoint list); reading
 * it as the microscaling format, it is offered here as the storage of the
 * index-key cache, the stream the decode scan reads: 66 bytes per 64-dim row
 * instead of 128.  msa_quantize_index_k writes it; msa_decode_append quantises
 * the new token's key when idx_format says so.
 */
/*
 * Paged caches (block_table != NULL): the K, V and index-K caches are pools of
 * n_pages pages of block_size tokens each, page-major and head-major inside a
 * page:
 *   k, v   [n_pages, n_kv_heads, block_size, head_dim]
 *   k_idx  [n_pages, n_idx_k_heads, block_size, idx_dim]
 * and block_table (device int32 [B, ceil(max_seq_len / block_size)]) names the
 * page that holds block n of sequence b (tokens n*block_size ..) in all three
 * pools.  One MSA block is one page, so a selected block is fetched from one
 * place and a serving loop can hand out pages as sequences grow.  Entries for
 * blocks a call can see must lie in [0, n_pages) (others are out of contract:
 * kernels clamp them and never read outside the pools).  All entries take it
 * except msa_prefill_index_topk with block_size < 128 (its 128-key tiles must
 * lie inside one page), which returns MSA_ERR_UNSUPPORTED.
 */

/*
 * Step 1a (+1b): index scores.  Exactly one of MSA_SCORES_TOKEN or
 * MSA_SCORES_BLOCKMAX must be set in params->flags.
 *   TOKEN:    scores_out [B, q_len, G, max_seq_len] fp32, s_j for j <= pos,
 *             -inf for j > pos.
 *   BLOCKMAX: scores_out [B, q_len, G, nb_max] fp32 with
 *             nb_max = ceil(max_seq_len / block_size); S_n for visible blocks,
 *             -inf for blocks after pos.
 * Decode (q_len == 1) streams k_idx once per index-K head.
 */
MSA_API msa_status_t msa_index_score(const msa_params_t *params, const void *q_idx, const void *k_idx,
                             float *scores_out, void *ws, size_t ws_bytes, msa_stream_t stream);

/*
 * Step 1b + 1c: block max pool and TopK from stored scores.  scores_in holds
 * token scores ([B, q_len, G, max_seq_len], default) or, with
 * MSA_SCORES_BLOCKMAX, block scores ([B, q_len, G, nb_max]); only entries of
 * visible tokens/blocks are read.  ids_out [B, q_len, G, top_k] int32 in
 * selection order; top_scores_out (nullable) the matching fp32 scores
 * (-inf for padding).  top_k up to 32 keeps warp-distributed lists; larger
 * top_k (the atlascloud.ai page, section 3: about 6-7 % of 16,384 blocks at
 * 1M tokens) takes a radix select per row, and token scores then need
 * msa_workspace_size(params, MSA_ENTRY_MAXPOOL_TOPK) bytes of ws for the
 * rows' block maxima.
 */
MSA_API msa_status_t msa_block_maxpool_topk(const msa_params_t *params, const float *scores_in,
                                    int32_t *ids_out, float *top_scores_out, void *ws,
                                    size_t ws_bytes, msa_stream_t stream);

/*
 * Step 2 for decode (q_len == 1): o = softmax attention of each query head
 * over the keys j <= pos of its group's listed blocks (ids entries of -1 are
 * skipped; with MSA_DENSE every visible block, ids may be NULL).
 * lse (nullable) receives the log normaliser.
 */
MSA_API msa_status_t msa_sparse_attn_decode(const msa_params_t *params, const void *q, const void *k_cache,
                                    const void *v_cache, const int32_t *ids, void *o, float *lse,
                                    void *ws, size_t ws_bytes, msa_stream_t stream);

/*
 * Step 2 for a causal prefill chunk: query rows t = 0..q_len-1 at positions
 * q_start + t, each with its own list ids[b, t, g, :].  bf16 only; block_size
 * 64 or 128.  Work is by block: every (row, listed block) pair leaves a partial
 * output in ws that a merge combines per row, in passes of 8192 rows (fewer
 * when top_k > 32: 8192 * 32 / top_k, so that ws does not grow with top_k).
 * Entries of ids that are -1 or name a block after the row are skipped.
 */
MSA_API msa_status_t msa_sparse_attn_prefill(const msa_params_t *params, const void *q, const void *k_cache,
                                     const void *v_cache, const int32_t *ids, void *o, float *lse,
                                     void *ws, size_t ws_bytes, msa_stream_t stream);

/*
 * One decode step, Steps 1 and 2 fused into back-to-back kernels on `stream`
 * (the block list never leaves the device).  ids_out and lse are nullable.
 * top_k up to 32: the scan keeps per-range candidate lists and the attention
 * kernel finishes the TopK (bf16 caches whose groups share one index-K head,
 * n_idx_k_heads < n_kv_heads: no lists, the scan stores every block's score in
 * ws and the attention kernel selects from those); larger top_k: the scan
 * stores every block's score in ws, a radix select per (sequence, group)
 * writes the list, and the attention splits each group's blocks over about
 * two CTAs per SM.  The index-key loads are marked evict-first in L2 when the
 * index-key cache is at most 2 GiB.
 */
MSA_API msa_status_t msa_decode_fused(const msa_params_t *params, const void *q, const void *q_idx,
                              const void *k_cache, const void *v_cache, const void *k_idx, void *o,
                              int32_t *ids_out, float *lse, void *ws, size_t ws_bytes,
                              msa_stream_t stream);

/*
 * msa_decode_fused for callers that cannot allocate device memory.  The
 * pages have no counterpart to this entry; it exists for callers that are
 * handed only their input and output buffers -- plugin or foreign-function
 * hosts whose calling convention has no slot for scratch memory, or serving
 * loops that reserve all device memory at start-up and allocate nothing
 * afterwards -- and so cannot supply msa_decode_fused's workspace.
 * Scratch comes from a fixed 8 MiB array that the library keeps in device
 * memory on every GPU that loads it, for as long as it stays loaded.
 *   - Shapes whose scratch (msa_workspace_size(params, MSA_ENTRY_DECODE_FUSED))
 *     exceeds 8 MiB are rejected with MSA_ERR_WORKSPACE before any launch;
 *     1M-token decode at batch 1 needs well under 1 MiB.
 *   - The array is shared by every call on a device: calls whose work
 *     overlaps on the GPU (other streams, other host threads) race on it
 *     and must be ordered by the caller.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current, and again after the
 *     device's context was replaced (cudaDeviceReset); make it before
 *     capturing any stream.
 *   - Nothing is allocated or freed; results equal msa_decode_fused's.
 *   - A bounded wait that ran out is reported only through the fixed
 *     scratch's status word: msa_noalloc_get_status / msa_noalloc_clear_status.
 */
MSA_API msa_status_t msa_decode_fused_noalloc(const msa_params_t *params, const void *q, const void *q_idx,
                                              const void *k_cache, const void *v_cache, const void *k_idx, void *o,
                                              int32_t *ids_out, float *lse, msa_stream_t stream);

/*
 * Status of msa_decode_fused_noalloc's fixed scratch on the current device:
 * its device status word works like a workspace's (see msa_get_device_status),
 * and a call whose bounded wait ran out still returns MSA_OK (the kernels are
 * asynchronous), so read it here after the calls.  msa_noalloc_get_status
 * synchronises `stream`; msa_noalloc_clear_status resets the status word and
 * the scan's counters of the fixed scratch, asynchronously on `stream`.
 */
MSA_API msa_status_t msa_noalloc_get_status(int *status, msa_stream_t stream);
MSA_API msa_status_t msa_noalloc_clear_status(msa_stream_t stream);

/*
 * MXFP8 quantisation of `rows` index-key rows (src bf16 [rows, idx_dim], device):
 * per 32 consecutive dims the shared exponent floor(log2 max|v|) - 8 clamped to
 * [-127, 127] (an all-zero block takes -127), stored as E8M0 (exponent + 127) in
 * scales [rows, idx_dim / 32]; each v / 2^shared rounded to the nearest E4M3
 * value, ties to even, saturating at 448, stored in codes [rows, idx_dim].
 * params gives idx_dim (64, 128 or 256); idx_format is not read.
 */
MSA_API msa_status_t msa_quantize_index_k(const msa_params_t *params, const void *src, long long rows,
                                          uint8_t *codes, uint8_t *scales, msa_stream_t stream);

/*
 * Serving step before msa_decode_fused (not part of the method): the new token
 * of every sequence -- k_new and v_new [B, n_kv_heads, head_dim], k_idx_new
 * [B, n_idx_k_heads, idx_dim], params.dtype, contiguous -- is written to its
 * position seq_lens[b] - 1 of the K, V and index-K caches (contiguous or paged,
 * as params say).  With idx_format MSA_IDX_MXFP8, k_idx_new is bf16 and is
 * quantised as msa_quantize_index_k does into k_idx (codes) and
 * params.k_idx_scale.  With the new token's q and q_idx it is all one decode
 * step takes from the host, so a caller can bring them in one copy; the caches
 * are otherwise untouched.
 */
MSA_API msa_status_t msa_decode_append(const msa_params_t *params, const void *k_new, const void *v_new,
                                       const void *k_idx_new, void *k_cache, void *v_cache, void *k_idx,
                                       msa_stream_t stream);

/*
 * Step 1 for a causal prefill chunk, fused: index scores on tensor cores,
 * block max pool and TopK in the epilogue; token scores are never stored.
 * ids_out [B, q_len, G, top_k]; top_scores_out nullable.  bf16 only.
 * The work (every query row against every key it can see) is cut into equal
 * ranges, one per SM; ws holds the per-row lists of rows whose keys were
 * split between ranges until they are merged (msa_workspace_size(params,
 * MSA_ENTRY_PREFILL_INDEX_TOPK) bytes, contents need no initialisation).
 * top_k up to 32 keeps sorted lists per row in the epilogue; above 32 the
 * epilogue stores every visible block score of every row in ws (B * q_len *
 * G * ((q_start + q_len - 1) / block_size + 1) floats) and a radix select
 * per row keeps the k best, in the same order.
 */
MSA_API msa_status_t msa_prefill_index_topk(const msa_params_t *params, const void *q_idx, const void *k_idx,
                                    int32_t *ids_out, float *top_scores_out, void *ws, size_t ws_bytes,
                                    msa_stream_t stream);

/*
 * Measurement hook (not part of the method): while set, msa_decode_fused
 * records events[0] before its first kernel, events[1] after the index scan
 * and events[2] after the attention kernel (TopK merge, sparse attention and
 * split merge) on the call's stream, so a caller can time each kernel with
 * cudaEventElapsedTime.  events are cudaEvent_t handles owned by the caller;
 * n_events must be 0 (unset) or 3.  Per calling thread.  Recording between
 * the kernels removes their launch overlap, so time whole steps without it.
 */
MSA_API msa_status_t msa_set_stage_events(void *const *events, int n_events);

/* Scratch bytes an entry needs for these params (0 if none); queries the
 * current device.  Returns (size_t)-1 for invalid params. */
MSA_API size_t msa_workspace_size(const msa_params_t *params, int entry);

/* Text of the last error on the calling thread ("" if none). */
MSA_API const char *msa_last_error_string(void);

/* Fixed text of a status code. */
MSA_API const char *msa_status_string(msa_status_t status);

/* Device status word kept in a workspace (first 4 bytes): MSA_OK, or
 * MSA_ERR_TIMEOUT after a bounded wait ran out.  Copies it to *status after
 * synchronising `stream`; msa_clear_device_status resets it asynchronously,
 * together with the wait limit (back to the default) and the scan's work
 * counters (left non-zero by a scan that did not end normally).  A kernel that
 * timed out stops issuing work, waits (bounded) for its own copies in flight
 * and returns; its outputs are then undefined, the context stays usable. */
MSA_API msa_status_t msa_get_device_status(const void *ws, int *status, msa_stream_t stream);
MSA_API msa_status_t msa_clear_device_status(void *ws, msa_stream_t stream);

/* Limit of every bounded device wait of the kernels that use this workspace,
 * in nanoseconds (bytes 8..15 of the workspace header, written on `stream`);
 * 0 restores the default of one second.  ws: 256-byte aligned device memory. */
MSA_API msa_status_t msa_set_wait_limit(void *ws, uint64_t limit_ns, msa_stream_t stream);

/* Failure-detection diagnostic (not part of the method): launches one thread
 * that waits, bounded by the workspace's wait limit, for an mbarrier phase
 * that nothing completes, so the wait runs out and the status word becomes
 * MSA_ERR_TIMEOUT without any fault.  Lets a caller check that timeouts reach
 * msa_get_device_status and that the workspace works again after
 * msa_clear_device_status.  ws_bytes >= 256. */
MSA_API msa_status_t msa_diag_wait_timeout(void *ws, size_t ws_bytes, msa_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MSA_H */
