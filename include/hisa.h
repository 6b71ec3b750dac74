/*
 * hisa.h — C ABI of the HISA hierarchical top-k indexer for B200 (sm_100a).
 *
 * HISA (HISA: Efficient Hierarchical Indexing for Fine-Grained Sparse
 * Attention; gptget.net English summary, "Methodology"; Chinese summary,
 * "方法详解" method details; arXiv abstract) replaces the flat indexer scan of
 * token-level sparse attention with two stages:
 *   1. block-level coarse filter: the key prefix is cut into contiguous
 *      blocks of B tokens, each block is mean-pooled into a representative,
 *      the representatives are scored with the same indexer and the top-m
 *      blocks are kept;
 *   2. token-level refinement: the m*B tokens of the kept blocks are scored
 *      with the indexer and the exact top-k token indices are emitted for the
 *      downstream sparse attention operator.
 * The flat scan it replaces (blog "Hierarchical Indexing Makes Sparse
 * Attention Actually Fast", "How Fine-Grained Sparse Attention Works Today")
 * scores every prefix token and keeps the top-k; it is exported as
 * dsa_flat_select for comparison.
 *
 * Indexer score of key x for query row i (H indexer heads, head dim d):
 *     score(i, x) = sum_h w[i,h] * max(0, q[i,h,:] . x)
 * Keys are visible to a query at position t iff their position s <= t.
 * The block holding t is always kept and counts inside m.  Ties go to the
 * lower token index (and the lower block id).
 *
 * Conventions for every entry point
 *   - All array arguments are DEVICE pointers to caller-owned memory, unless
 *     stated otherwise.  The library allocates nothing: scratch space is the
 *     caller's workspace buffer (size from the *_workspace_bytes queries).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  The return value only reports argument checks and
 *     launch errors.  Conditions found on the device (a query position
 *     outside its sequence, an append past capacity, a bounded wait that ran
 *     out) set bits in the cache's device status word; read it after the
 *     stream has synchronised.
 *   - Calls that share a cache or workspace must be ordered on one stream.
 *   - Arrays are row-major and densely packed.  Pointers must be 16-byte
 *     aligned; the workspace must be 256-byte aligned.
 */
#ifndef HISA_H_
#define HISA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* hisa_stream_t;   /* same handle as cudaStream_t */

/* Key storage formats. */
enum hisa_key_dtype {
    HISA_KEY_BF16 = 0,   /* bf16 keys */
    HISA_KEY_E4M3 = 1    /* OCP e4m3 codes + one fp32 scale (> 0) per token;
                            the key value is fp32(e4m3 value * scale) */
};

/* Block representatives.  MEAN: the mean of the block's valid keys (HISA
 * Methodology: mean pooling).  MAX: their elementwise maximum (blog
 * "Hierarchical Indexing Makes Sparse Attention Actually Fast", "HISA's
 * Approach": summary nodes pool a token group by mean or by max). */
enum hisa_pool_mode {
    HISA_POOL_MEAN = 0,
    HISA_POOL_MAX = 1
};

/* Return codes. */
enum hisa_status {
    HISA_OK = 0,
    HISA_E_INVAL = 1,        /* a NULL, misaligned or out-of-range argument */
    HISA_E_UNSUPPORTED = 2,  /* a size outside the built kernels (d, B, H) */
    HISA_E_WORKSPACE = 3,    /* workspace too small or misaligned */
    HISA_E_CUDA = 4,         /* a CUDA call or launch failed */
    HISA_E_SCRATCH_LIMIT = 5 /* hisa_select_static: the call needs more than
                                HISA_STATIC_SCRATCH_BYTES of scratch */
};

/* Bits of the device status word (sticky: the library only ORs bits in). */
#define HISA_DEV_BAD_QUERY 0x1u  /* a query's position is not inside its prefix;
                                    that row's output is all -1 */
#define HISA_DEV_CAPACITY  0x2u  /* hisa_append found len == cap; nothing appended
                                    for that sequence */
#define HISA_DEV_BAD_LEN   0x4u  /* a len[] entry outside [0, cap] */
#define HISA_DEV_TIMEOUT   0x8u  /* a bounded in-kernel wait ran out; outputs of
                                    that launch are undefined */

/*
 * The indexer key cache and its block index ("hierarchical index").
 *
 *   keys       [batch, cap, d]   bf16, or e4m3 bytes (dtype)
 *   key_scale  [batch, cap]      fp32 > 0, E4M3 only (NULL for BF16)
 *   pooled     [batch, nblk, d]  fp32 block means, nblk = ceil(cap / B)
 *   pooled_hl  [batch, nblk, 2*d] bf16: row j holds hi = bf16(pooled[j])
 *                                 then lo = bf16(pooled[j] - hi), the
 *                                 tensor-core form of the block means
 *   len        [batch]           int32 valid prefix length per sequence
 *   status     [1]               uint32 device status word (see HISA_DEV_*)
 *
 * Block representatives are the means (or, with pool = HISA_POOL_MAX, the
 * elementwise maxima) of the visible keys of each block (HISA Methodology:
 * mean pooling generates the block representatives).  The trailing partial
 * block is pooled over its len - j*B valid keys.
 *
 * Sizes: d in {64, 128}.  Pooling and append take any B >= 1; the select
 * calls need B in {8, 16, 32, 64} or a multiple of 128 up to 1024.
 */
typedef struct hisa_kv {
    void* keys;
    float* key_scale;
    float* pooled;
    uint16_t* pooled_hl;
    int32_t* len;
    uint32_t* status;
    int32_t batch;
    int32_t cap;
    int32_t d;
    int32_t B;
    int32_t dtype;   /* enum hisa_key_dtype */
    int32_t pool;    /* enum hisa_pool_mode */
} hisa_kv;

/*
 * hisa_pool_blocks — build the block index from scratch.
 * HISA Chinese summary, method details (first step): the length-L prefix is
 * split into contiguous blocks of size B and each block is mean-pooled.
 * For every sequence b and block j with j*B < len[b], writes pooled[b, j, :]
 * (fp32 mean of keys j*B .. min((j+1)*B, len[b]) - 1, summed in fp32) and
 * pooled_hl[b, j, :].  Rows of blocks at or past len[b] are not written.
 * One streaming pass over the keys.
 */
int hisa_pool_blocks(const hisa_kv* kv, hisa_stream_t stream);

/*
 * hisa_append — append one key per sequence and keep the index current.
 * Blog "Hierarchical Indexing Makes Sparse Attention Actually Fast", "HISA's
 * Approach": the summary structure is maintained incrementally as tokens are
 * appended.  In the two-stage form only the trailing block changes.
 *   tok        [batch, d]  the new key rows (bf16 or e4m3, as kv->dtype)
 *   tok_scale  [batch]     fp32 scales (E4M3) or NULL
 * For each sequence b with len[b] < cap: writes the key at position len[b],
 * recomputes the trailing block's mean over its valid keys (O(B*d) work, the
 * same arithmetic as hisa_pool_blocks, so the result equals a full re-pool
 * bit for bit), then len[b] += 1.  A full sequence sets HISA_DEV_CAPACITY and
 * is left unchanged.
 */
int hisa_append(const hisa_kv* kv, const void* tok, const float* tok_scale,
                hisa_stream_t stream);

/*
 * hisa_select — the two-stage HISA selection for n_q query rows.
 * HISA arXiv abstract, stages (1) and (2); gptget.net summary, "Methodology"
 * (top-m blocks by pooled score, then token scoring inside them); Chinese
 * summary, method details (the final k tokens feed sparse attention).
 *   Q      [n_q, H, d] bf16  indexer queries
 *   w      [n_q, H]    fp32  per-row head weights
 *   q_seq  [n_q]       int32 sequence of each row
 *   q_pos  [n_q]       int32 position t of each row (keys s <= t visible);
 *                            NULL = each row's last position len[q_seq] - 1
 *   m      blocks kept per row (the own block included); m >= #blocks keeps
 *          every block, which makes the result equal dsa_flat_select
 *   k      tokens kept per row
 *   idx    [n_q, k] int32 out: selected positions within the row's sequence,
 *          ascending, then -1 padding when fewer than k are visible
 *   scores [n_q, k] fp32 out (or NULL): the indexer score of each idx entry
 *          (NaN under -1 padding)
 *   ws     workspace of at least hisa_select_workspace_bytes(...) bytes
 * H in 1..128.  The pooled index must be current for every row (built by
 * hisa_pool_blocks / hisa_append); the own block's representative may cover
 * keys past t — it is kept whatever its score.
 * e4m3 keys with d = 128 are scored on the fp8 tensor cores: every query head
 * is scaled by a power of two and split into two e4m3 parts whose sum is the
 * bf16 value, except for the parts of an element below e4m3's smallest step
 * after scaling (under 2^-17 of the head's largest |q|), which are dropped.
 */
size_t hisa_select_workspace_bytes(const hisa_kv* kv, int n_q, int H, int m, int k);
int hisa_select(const hisa_kv* kv, const uint16_t* Q, const float* w, const int32_t* q_seq,
                const int32_t* q_pos, int n_q, int H, int m, int k, int32_t* idx,
                float* scores, void* ws, size_t ws_bytes, hisa_stream_t stream);

/*
 * hisa_decode_step — one decode step of a batch: hisa_append, then
 * hisa_select for every sequence's new last position, in one call.
 * HISA blog "Hierarchical Indexing Makes Sparse Attention Actually Fast",
 * "HISA's Approach" (the summary is kept current as tokens are appended) and
 * the two stages of hisa_select (arXiv abstract, stages (1) and (2)).
 *   tok        [batch, d]  the new key of each sequence (bf16 or e4m3 codes)
 *   tok_scale  [batch]     fp32 scales (E4M3) or NULL
 *   Q [batch, H, d] bf16, w [batch, H] fp32: query row b belongs to sequence b
 *   idx [batch, k] int32 out, scores [batch, k] fp32 out or NULL: as hisa_select
 *   ws  workspace of at least hisa_decode_step_workspace_bytes(...) bytes
 * Results (idx, scores, keys, key scales, pooled, pooled_hl, len, status) are
 * those of hisa_append(kv, tok, tok_scale) followed by hisa_select(kv, Q, w,
 * q_seq = 0..batch-1, q_pos = NULL, m, k), bit for bit.  Rows of at most
 * 4 x 128 blocks and batches of at most two rows per SM run the append and
 * the block scoring (one CTA per row, top-m kept in the same kernel) side by
 * side: the block scoring does not read the appended block (the row's own
 * block, kept without a score) and publishes the new lengths once the append
 * kernel has finished.  Other sizes run the two calls' launches.  A full sequence is left
 * as it is (HISA_DEV_CAPACITY) and selects for position cap - 1; a len[]
 * outside [0, cap] sets HISA_DEV_BAD_LEN and HISA_DEV_BAD_QUERY and gives a
 * -1 row.  Errors as hisa_append and hisa_select.
 */
size_t hisa_decode_step_workspace_bytes(const hisa_kv* kv, int H, int m, int k);
int hisa_decode_step(const hisa_kv* kv, const void* tok, const float* tok_scale, const uint16_t* Q,
                     const float* w, int H, int m, int k, int32_t* idx, float* scores, void* ws,
                     size_t ws_bytes, hisa_stream_t stream);

/*
 * hisa_select_inspect — hisa_select plus its intermediate results, for
 * verification of the two stages separately.
 *   blocks  [n_q, min(m, nblk)] int32 out (or NULL): kept block ids per row,
 *           ascending, -1 padded
 *   nblocks [n_q] int32 out (or NULL): number of kept blocks per row
 *   counts  [n_q, 2] uint64 out (or NULL), zeroed by the call: per row the
 *           number of block representatives scored and of token slots scored
 *           (HISA Methodology: O(L/B + mB) indexer work per query)
 */
int hisa_select_inspect(const hisa_kv* kv, const uint16_t* Q, const float* w,
                        const int32_t* q_seq, const int32_t* q_pos, int n_q, int H, int m,
                        int k, int32_t* idx, float* scores, int32_t* blocks, int32_t* nblocks,
                        uint64_t* counts, void* ws, size_t ws_bytes, hisa_stream_t stream);

/*
 * hisa_tree_select — three-level search: superblocks, blocks, tokens.
 * Blog "Hierarchical Indexing Makes Sparse Attention Actually Fast", "HISA's
 * Approach": a multi-level summary of the cache searched top down, keeping
 * the best branches at every level.
 *   kv2    a second index over the same keys (keys, key_scale, len, batch,
 *          cap, d, dtype and pool equal to kv's) whose block size is
 *          bf = kv2->B / kv->B first-level blocks (a superblock); its own
 *          pooled / pooled_hl, built by hisa_pool_blocks(kv2) and kept
 *          current after each hisa_append(kv, ...) by hisa_pool_tail(kv2)
 *   W      superblocks kept per row: the own superblock plus the best W - 1
 *   m, k   blocks kept among the visible blocks under the kept superblocks
 *          (the own block plus the best m - 1), then tokens, as hisa_select
 *   sblocks [n_q, min(W, kv2 blocks)] out (or NULL): kept superblocks,
 *          ascending, -1 padded; nsblocks [n_q] out (or NULL)
 *   blocks [n_q, min(m, kv blocks)], nblocks [n_q]: out (or NULL), as
 *          hisa_select_inspect
 *   counts [n_q, 3] out (or NULL), zeroed by the call: superblocks scored,
 *          blocks scored, token slots scored
 * W covering every superblock gives hisa_select's result.  kv2 may hold up to
 * 32768 superblocks per sequence (HISA_E_UNSUPPORTED beyond).  The block
 * level reads and scores only the kept superblocks' children when they are
 * at most a quarter of the blocks, W * bf <= 512, bf is a power of two from
 * 8 to 128 and there are at most two rows per SM; otherwise it scores every
 * visible block and masks the others.  Either way the results and the
 * counters (which count the children below the own block, plus the own
 * block) are the same.
 */
size_t hisa_tree_workspace_bytes(const hisa_kv* kv, const hisa_kv* kv2, int n_q, int H, int W,
                                 int m, int k);
int hisa_tree_select(const hisa_kv* kv, const hisa_kv* kv2, const uint16_t* Q, const float* w,
                     const int32_t* q_seq, const int32_t* q_pos, int n_q, int H, int W, int m,
                     int k, int32_t* idx, float* scores, int32_t* sblocks, int32_t* nsblocks,
                     int32_t* blocks, int32_t* nblocks, uint64_t* counts, void* ws,
                     size_t ws_bytes, hisa_stream_t stream);

/*
 * hisa_pool_tail — re-pool each sequence's trailing block (the block that
 * holds key len[b] - 1) from the keys.  For a coarser index over keys that
 * hisa_append on a finer index sharing them has just grown; len is read,
 * not changed.
 */
int hisa_pool_tail(const hisa_kv* kv, hisa_stream_t stream);

/*
 * hisa_levels_select — search of any depth: n_levels levels of blocks, then
 * tokens.  Blog "Hierarchical Indexing Makes Sparse Attention Actually
 * Fast", "HISA's Approach" and "The Complexity Win": the cache summarised as
 * a tree, searched from the root down with the best branches kept at every
 * level, so that the summaries a query scores grow with the depth of the
 * tree rather than with L/B.
 *   kv      [n_levels] host array of indexes over the same keys (keys,
 *           key_scale, len, batch, cap, d, dtype and pool equal to kv[0]'s),
 *           finest first: kv[0] is the block index (its B is the token
 *           block size, as hisa_select), kv[l]->B a multiple of kv[l-1]->B;
 *           each built by hisa_pool_blocks and, after hisa_append on kv[0],
 *           kept current by hisa_pool_tail(kv[l]); kv[l] for l >= 1 may hold
 *           up to 32768 units per sequence (HISA_E_UNSUPPORTED beyond)
 *   n_levels 1 .. HISA_MAX_LEVELS (1: hisa_select_inspect's result)
 *   keep    [n_levels] host array, each >= 1: units kept per row at level l,
 *           the own unit (the one holding the query position) plus the best
 *           keep[l] - 1 candidates by (score desc, id asc); keep[0] is m
 *   The candidates are every visible unit at the top level and, below it,
 *   the visible units inside the units kept one level up (the own unit
 *   apart).  A level reads and scores only those children when
 *   hisa_tree_select's gathered conditions hold for it (branching factor a
 *   power of two from 8 to 128, the kept units above times it at most 512
 *   and at most a quarter of the level's units, at most two rows per SM);
 *   otherwise it scores every visible unit and masks the others, with the
 *   same results.
 *   k, idx, scores  as hisa_select
 *   kept    NULL, or a host array of n_levels device pointers, each NULL or
 *           [n_q, min(keep[l], units of kv[l])] out: the kept units ascending,
 *           -1 padded
 *   nkept   NULL, or a host array of n_levels device pointers, each NULL or
 *           [n_q] out: the units kept at level l
 *   counts  [n_q, n_levels + 1] out (or NULL), zeroed by the call: the units
 *           of each level scored (candidates plus the own unit), then the
 *           token slots scored
 * Two levels give hisa_tree_select's result (with its counts columns in
 * the other order).  Errors: HISA_E_INVAL for a level that does not match
 * kv[0] or a unit size that is not a multiple of the one below;
 * HISA_E_WORKSPACE for ws smaller than hisa_levels_workspace_bytes (0 for
 * invalid arguments); the other codes as hisa_select.
 */
#define HISA_MAX_LEVELS 8
size_t hisa_levels_workspace_bytes(const hisa_kv* const* kv, int n_levels, const int* keep, int n_q,
                                   int H, int k);
int hisa_levels_select(const hisa_kv* const* kv, int n_levels, const int* keep, const uint16_t* Q,
                       const float* w, const int32_t* q_seq, const int32_t* q_pos, int n_q, int H,
                       int k, int32_t* idx, float* scores, int32_t* const* kept,
                       int32_t* const* nkept, uint64_t* counts, void* ws, size_t ws_bytes,
                       hisa_stream_t stream);

/*
 * Context parallelism: one sequence longer than a GPU holds, split by token
 * range over R ranks.  The pages motivate contexts of 64K to 1M tokens and
 * beyond (blog "What This Means for Long-Context Inference"; gptget.net
 * summary, limitations: texts beyond millions of tokens) but give no
 * multi-GPU design; this decomposition is this library's.  Each rank's
 * hisa_kv is a shard: keys[b, s] holds global position tok_off + s of
 * sequence b, for every sequence, with tok_off and cap multiples of B and
 * len[b] the shard's own length (a shard before the one holding the end of
 * a sequence is full).  q_pos are GLOBAL positions and are required.
 * The result equals hisa_select on the whole sequence:
 *   1. hisa_cp_blocks on every rank: the shard's candidates, [n_q, m]
 *      (global block id, score) pairs, ascending in id, -1 / NaN padded:
 *      the best m - 1 blocks visible to the row other than its own block,
 *      then, on the rank holding the query position, the own block with
 *      score +inf.
 *   2. all-gather the pairs in rank order (ranks own ascending ranges) into
 *      [R, n_q, m], and hisa_merge_topk(lists = R, n = m, k = m): the kept
 *      global block ids [n_q, m] (the own block always among them).
 *   3. hisa_cp_tokens on every rank with those ids: the top-k of the
 *      shard's tokens in the kept blocks, as (global index, score) pairs.
 *   4. all-gather [R, n_q, k] and hisa_merge_topk(lists = R, n = k, k).
 * Exactness: every block and token is scored by the same kernel as in
 * hisa_select, and the best kk of a union of lists is the best kk of the
 * union of each list's best kk, so each merge is exact (ties: lower id).
 * Rows the shard cannot see (query before the shard) give no candidates.
 * An invalid row (bad sequence, a position past the sequence end) gives -1
 * rows and sets HISA_DEV_BAD_QUERY: in hisa_cp_blocks on a shard that sees
 * it, and in hisa_cp_tokens on every shard (a valid row always has its own
 * block, global id q_pos / B, among the merged kept blocks).
 * Limits: at most 24576 blocks per shard; lists * n <= 24576 in a merge.
 * Errors as hisa_select; HISA_E_INVAL also for a missing q_pos, or tok_off
 * or cap not on block boundaries.  Workspace: hisa_cp_workspace_bytes,
 * reused by both calls of one rank.
 */
size_t hisa_cp_workspace_bytes(const hisa_kv* kv, int32_t tok_off, int n_q, int H, int m, int k);
int hisa_cp_blocks(const hisa_kv* kv, int32_t tok_off, const uint16_t* Q, const float* w,
                   const int32_t* q_seq, const int32_t* q_pos, int n_q, int H, int m,
                   int32_t* cand_ids, float* cand_scores, void* ws, size_t ws_bytes,
                   hisa_stream_t stream);
int hisa_cp_tokens(const hisa_kv* kv, int32_t tok_off, const uint16_t* Q, const float* w,
                   const int32_t* q_seq, const int32_t* q_pos, int n_q, int H, int m, int k,
                   const int32_t* kept, int32_t* idx, float* scores, void* ws, size_t ws_bytes,
                   hisa_stream_t stream);

/*
 * hisa_sparse_attn — the consumer of the selection: attention of each query
 * row over the tokens it selected (HISA blog, "How Fine-Grained Sparse
 * Attention Works Today": the second stage attends only to the top-K tokens;
 * arXiv abstract: the indices feed the sparse attention operator).  A
 * synthetic multi-query operator: Ha query heads (1..128) of d = 128 share
 * one key head and one value head.  For row i (sequence b = q_seq[i]) and
 * head h, over the entries j with 0 <= idx[i, j] < len[b]:
 *     s_j = scale * Qa[i, h] . Kc[b, idx[i, j]]
 *     out[i, h] = sum_j exp(s_j) Vc[b, idx[i, j]] / sum_j exp(s_j)
 *     lse[i, h] = log sum_j exp(s_j)
 * Other entries (-1 padding, or past len[b]) are skipped; a repeated index
 * counts once per entry.  A row with no valid entry gives out = 0 and
 * lse = -inf.
 *   Qa [n_q, Ha, 128] bf16; Kc, Vc [batch, cap, 128] bf16 (16-byte aligned);
 *   len [batch] int32; q_seq [n_q]; idx [n_q, k] (hisa_select's output);
 *   out [n_q, Ha, 128] fp32 (16-byte aligned); lse [n_q, Ha] or NULL;
 *   status: a device word for HISA_DEV_TIMEOUT; all device memory, caller
 *   owned.  Workspace: hisa_sparse_attn_workspace_bytes(n_q, k).
 * Numerics: Qa Kc^T on the bf16 tensor cores into fp32; softmax weights in
 * fp32 (hardware 2^x, about 2^-22 relative), rounded to bf16 for the
 * weights-times-values product (fp32 accumulate); the normalising sum is
 * taken over the fp32 weights.  Each output is then within 2^-9 (plus fp32
 * rounding) of max |v| over the row's entries of the exact value.
 * Errors: HISA_E_INVAL (sizes, pointers, alignment, scale not finite and
 * positive), HISA_E_UNSUPPORTED (d != 128, Ha outside 1..128),
 * HISA_E_WORKSPACE, HISA_E_CUDA.
 */
size_t hisa_sparse_attn_workspace_bytes(int n_q, int k);
int hisa_sparse_attn(const uint16_t* Qa, int Ha, const uint16_t* Kc, const uint16_t* Vc, const int32_t* len,
                     int batch, int cap, int d, const int32_t* q_seq, const int32_t* idx, int n_q, int k,
                     float scale, float* out, float* lse, uint32_t* status, void* ws, size_t ws_bytes,
                     hisa_stream_t stream);

/*
 * hisa_merge_topk — top-k of several (id, score) lists per row, by (score
 * desc, id asc): the exchange step of context parallelism.  ids and scores
 * are [lists, rows, n] (device, row-major; the layout an all-gather in list
 * order produces); id -1 marks an empty entry (its score is ignored).  The
 * concatenation of a row's lists must ascend in id (each list ascending and
 * the lists' id ranges ascending), which is what makes the lower-id rule the
 * lower-slot rule.  Out: idx [rows, k] ascending then -1, out_scores
 * [rows, k] (NaN under padding) or NULL.  Scores must not be NaN for
 * non-empty entries.  HISA_E_UNSUPPORTED if lists * n > 24576.
 */
int hisa_merge_topk(const int32_t* ids, const float* scores, int lists, int rows, int n, int k,
                    int32_t* idx, float* out_scores, hisa_stream_t stream);

/*
 * hisa_select_static — hisa_select without a caller workspace.  The pages
 * have no counterpart: this is a deployment convenience of this library.
 * The scratch hisa_select keeps in `ws` lives instead in one fixed device
 * array inside the library, HISA_STATIC_SCRATCH_BYTES (8 MiB) per device, so
 * the call allocates no device or host memory at all.  It is meant for
 * callers that cannot allocate on their selection path: an engine whose
 * device memory is fully reserved up front (KV cache pages fill what is
 * left), or a C caller with no allocator of its own that should not own a
 * workspace's lifetime.
 *   Arguments, outputs and results are those of hisa_select (same kernels,
 *   same arithmetic: results are identical to hisa_select's).
 *   Limit: hisa_select_workspace_bytes(kv, n_q, H, m, k) must be at most
 *   HISA_STATIC_SCRATCH_BYTES, else HISA_E_SCRATCH_LIMIT and nothing is
 *   launched (64 decode rows over 32K keys with B = 128, m = 64 need about
 *   2.2 MB; a 4096-row prefill chunk does not fit — use hisa_select).
 *   Setup: the first call on a device, with that device current, looks up
 *   the array's device address (cudaGetSymbolAddress, which loads the
 *   library's device code if it is not loaded yet); later calls on that
 *   device reuse it while the device's context lives.  The address is kept
 *   with the context's unique id: after a cudaDeviceReset the next call is a
 *   first call again and looks the address up anew.  Make the first call on
 *   a device (and the first after a reset) before any stream capture.
 *   Contents: nothing in the array needs to start at zero; every byte a call
 *   reads was written earlier in the same call.
 *   Races: all calls on one device share the one array.  Two calls whose
 *   kernels may overlap (different streams, or host threads without
 *   ordering) race on it and give undefined results; order them on one
 *   stream.
 */
#define HISA_STATIC_SCRATCH_BYTES ((size_t)8 << 20)
int hisa_select_static(const hisa_kv* kv, const uint16_t* Q, const float* w,
                       const int32_t* q_seq, const int32_t* q_pos, int n_q, int H, int m,
                       int k, int32_t* idx, float* scores, hisa_stream_t stream);

/*
 * dsa_flat_select — the flat indexer scan HISA replaces: every visible key
 * s <= t is scored and the top-k kept (blog "How Fine-Grained Sparse
 * Attention Works Today"; HISA abstract: the indexer scans the entire
 * prefix).  Arguments as hisa_select without m.  Scores come from the same
 * scoring kernel as hisa_select, so both paths give the same fp32 score to
 * the same key.
 */
size_t dsa_flat_workspace_bytes(const hisa_kv* kv, int n_q, int H, int k);
int dsa_flat_select(const hisa_kv* kv, const uint16_t* Q, const float* w, const int32_t* q_seq,
                    const int32_t* q_pos, int n_q, int H, int k, int32_t* idx, float* scores,
                    void* ws, size_t ws_bytes, hisa_stream_t stream);

/*
 * hisa_topk_f32 — the selection rule alone: for each of `rows` rows of n
 * fp32 values x[r, :], the k largest (ties: lower index), indices ascending
 * then -1 padding, into idx[rows, k].  NaN inputs are not allowed; -0.0 and
 * +0.0 are equal.  The same routine selects blocks and tokens inside
 * hisa_select and dsa_flat_select (HISA Chinese summary, method details:
 * final k tokens; gptget.net summary: top-m blocks).
 */
int hisa_topk_f32(const float* x, int rows, int n, int k, int32_t* idx, hisa_stream_t stream);

/*
 * Phase timing for measurement tools (no counterpart on the pages).  While
 * enabled, every call records a CUDA event pair around each kernel it
 * launches, on the call's stream.  hisa_profile_read waits for the recorded
 * events, adds up their durations per phase (milliseconds) and launch counts,
 * and with reset != 0 starts a new accumulation.  Phases:
 */
enum hisa_phase {
    HISA_PHASE_BLOCK_SCORE = 0,   /* stage 1: score block representatives */
    HISA_PHASE_BLOCK_SELECT = 1,  /* stage 1: keep top-m blocks */
    HISA_PHASE_TOKEN_SCORE = 2,   /* stage 2: gather + score candidate tokens */
    HISA_PHASE_TOKEN_SELECT = 3,  /* stage 2: keep top-k tokens */
    HISA_PHASE_FLAT_SCORE = 4,    /* flat scan: score every visible token */
    HISA_PHASE_FLAT_SELECT = 5,   /* flat scan: keep top-k */
    HISA_PHASE_POOL = 6,          /* hisa_pool_blocks */
    HISA_PHASE_APPEND = 7,        /* hisa_append */
    HISA_PHASE_TOPK = 8,          /* hisa_topk_f32 */
    HISA_PHASE_QSPLIT = 9,        /* query heads split for fp8 scoring (e4m3 keys, d = 128) */
    HISA_PHASE_MERGE = 10,        /* hisa_merge_topk */
    HISA_PHASE_ATTN = 11,         /* hisa_sparse_attn */
    HISA_NUM_PHASES = 12
};
int hisa_profile_enable(int on);
int hisa_profile_read(float* ms, int* launches, int reset);

/*
 * hisa_selftest_wait — failure detection check (no counterpart on the pages).
 * Launches one warp that waits on an mbarrier nothing completes, with the
 * same bounded wait every library kernel uses: after its 2 s limit the wait
 * gives up, HISA_DEV_TIMEOUT is OR-ed into the device word `status`, and the
 * kernel returns, leaving the context usable.  No fault, trap or hang is
 * involved.  HISA_E_INVAL for a NULL or unaligned status.
 */
int hisa_selftest_wait(uint32_t* status, hisa_stream_t stream);

/* Human-readable name of a return code. */
const char* hisa_status_string(int code);

/* The CUDA runtime's description of the error behind the calling thread's
 * last HISA_E_CUDA from a launch ("no error" if there was none). */
const char* hisa_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* HISA_H_ */
