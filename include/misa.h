/*
 * misa.h -- C ABI of the B200 (sm_100a) token-indexer library libmisa.so.
 *
 * The library implements the indexer that sits in front of sparse attention in
 * three forms:
 *   - MISA: a router reads mean-pooled key blocks and keeps h of the H indexer
 *     heads per query (block); only those heads score every prefix token; a
 *     per-query top-k follows.
 *     ["MISA: Mixture of Indexer Sparse Attention for Long-Context LLM
 *     Inference" (gist.science), technical summary, "Methodology: MISA".]
 *   - MISA-dagger (hierarchical MISA): the routed pass keeps k' candidates, all
 *     H heads rescore them, top-k over the candidates.
 *     [same page, "Hierarchical variant (MISA-dagger)".]
 *   - HISA: mean-pooled B-token blocks are scored with all heads, the top-m
 *     blocks are kept, the token indexer runs inside them, top-k.
 *     ["HISA：为什么长文本理解的关键，藏在图书馆的分类索引里？" (zhichai.net),
 *     section 三, Stage 1 and Stage 2.]
 *   - the dense DSA indexer (all H heads score every token) is the same calls
 *     with heads == NULL.  [MISA page, "Problem statement".]
 * The decode step in one call: misa_index_decode (router and routed scoring in
 * one kernel, the top-k behind it).  HISA's token stage straight from the
 * chosen blocks: misa_index_score_blocks.
 * Around the indexer: block statistics (mean or max pooling, plain blocks or
 * overlapping windows: the *_ex calls) kept current as keys are appended
 * (misa_append_keys); the sparse attention that consumes the k indices
 * (misa_sparse_mla) [HISA page, sections 二 and 四]; and two small steps of
 * the key-sharded (context-parallel) indexer (misa_shard_prefix,
 * misa_gather_candidates).
 *
 * Indexer score (the pages print no formula; this is the library's definition):
 *     S[t, s] = sum over active heads h (ascending id) of w[t, h] * ReLU(q[t, h] . k[s])
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Head dimension d is fixed at MISA_HEAD_DIM (128).
 *  - bf16 arrays are passed as uint16_t bit patterns.  Layouts are row-major with
 *    the innermost dimension contiguous:
 *        q        [T][H][128]            bf16
 *        w        [T][H]                 fp32
 *        keys     row s of sequence b at keys + b * key_seq_stride + s * 128 (bf16)
 *        means    block j of sequence b at means + b * means_seq_stride + j * 128 (fp32);
 *                 its optional bf16 split means_hi / means_lo at the same offsets
 *        seq_of   [T] int32   which sequence (key cache) query t reads
 *        prefix_len [T] int32 query t may see keys 0 <= s < prefix_len[t]
 *  - Every pointer argument is a DEVICE pointer owned by the caller (except
 *    where a comment says "host").  The library allocates no device memory,
 *    keeps no pointer after a call returns and holds no global state apart from
 *    constant tables, the cached address of the driver's tensor-map encoder and
 *    the fixed scratch array of misa_route_heads_noalloc.
 *  - Every compute call is asynchronous on `stream` and never synchronises.
 *    Only misa_error_query() synchronises (on the given stream).
 *  - Arguments are checked on the host before anything is launched; a bad
 *    argument returns MISA_ERR_INVALID_ARG (or MISA_ERR_UNSUPPORTED for a
 *    well-formed request outside what the kernels implement, or
 *    MISA_ERR_WORKSPACE for a workspace smaller than misa_workspace_bytes()).
 *    Such a call has no effect.  A CUDA launch error returns MISA_ERR_CUDA.
 *  - Device-side checks: an out-of-range seq_of[t], head id or token index, and a pipeline
 *    wait that gives up (a bounded wait of about two seconds), are recorded as
 *    bits in the error word at the start of the workspace (MISA_DEVERR_*); the
 *    kernel then skips the affected work and returns.  Read the word with
 *    misa_error_query(); clear it with misa_error_reset().
 *  - Top-k order: larger score first, ties to the lower position; -0.0 ranks
 *    equal to +0.0; entries equal to -inf (masked) are never selected.  The
 *    selected positions are written in ascending order; when fewer than k
 *    entries are valid the row is padded with -1.
 *  - Visibility: key s is visible to query t iff 0 <= s < min(prefix_len[t], L).
 *    A routing decision (and a HISA block score) sees block j iff the whole
 *    block lies inside the prefix: min((j + 1) * B, L) <= prefix_len; HISA also
 *    keeps the one block a prefix cuts (see hisa_block_filter).
 */
#ifndef MISA_H
#define MISA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols of libmisa.so (the library is built with hidden default
 * visibility; only the functions declared here are exported). */
#if defined(__GNUC__)
#define MISA_API __attribute__((visibility("default")))
#else
#define MISA_API
#endif

#define MISA_HEAD_DIM 128
#define MISA_MAX_HEADS 128     /* H limit */
#define MISA_MAX_TOPK 16384    /* k (and k') limit of misa_topk */
#define MISA_MAX_TOPK_ROWS 65535 /* rows (T) limit of the calls that run a top-k */
#define MISA_ABI_VERSION 1
#define MISA_MLA_DQK 576       /* misa_sparse_mla: latent KV row (512 latent + 64 rotary) */
#define MISA_MLA_DV 512        /* misa_sparse_mla: value part (the first 512 entries of a row) */

/* Same object as cudaStream_t (a CUDA runtime stream handle); NULL is the
 * legacy default stream. */
typedef struct CUstream_st* misa_stream_t;

typedef enum misa_status {
  MISA_OK = 0,
  MISA_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or combination */
  MISA_ERR_UNSUPPORTED = 2,  /* valid request the kernels do not implement */
  MISA_ERR_WORKSPACE = 3,    /* workspace NULL or smaller than required */
  MISA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  MISA_ERR_DEVICE = 5        /* misa_error_query: the device recorded an error */
} misa_status;

/* Bits of the device error word (first 4 bytes of every workspace). */
#define MISA_DEVERR_TIMEOUT 1u    /* a bounded pipeline wait gave up */
#define MISA_DEVERR_BAD_SEQ 2u    /* seq_of[t] outside [0, nseq) */
#define MISA_DEVERR_BAD_HEAD 4u   /* a head id outside [0, H) */
#define MISA_DEVERR_BAD_LEN 8u    /* misa_append_keys: len[b] < 0 or len[b] + n_new > L_cap */
#define MISA_DEVERR_BAD_INDEX 16u /* misa_sparse_mla: an index outside [-1, L) (treated as empty) */

/* Static description of a status code (never NULL). */
MISA_API const char* misa_status_string(int status);

/* MISA_ABI_VERSION of the loaded library. */
MISA_API int misa_abi_version(void);

/* Operation ids for misa_workspace_bytes. */
#define MISA_OP_ROUTE_HEADS 1
#define MISA_OP_INDEX_SCORE 2
#define MISA_OP_TOPK 3
#define MISA_OP_HIER_RERANK 4
#define MISA_OP_HISA_BLOCK_FILTER 5
#define MISA_OP_APPEND_KEYS 6
#define MISA_OP_SPARSE_MLA 7
#define MISA_OP_INDEX_DECODE 8

/* Bytes of device workspace the operation needs for these sizes (>= 256: the
 * first 256 bytes hold the device error word).  Arguments an operation does not
 * use are ignored:
 *   ROUTE_HEADS: T, H, L, B;  INDEX_SCORE: none;  TOPK: none;
 *   HIER_RERANK: T, kp;  HISA_BLOCK_FILTER: T, L, B;  APPEND_KEYS: none;
 *   SPARSE_MLA: T, H (= Hq), k;  INDEX_DECODE: T, L.
 * Returns 0 for an unknown op or negative sizes. */
MISA_API size_t misa_workspace_bytes(int op, int T, int H, int64_t L, int B, int k, int kp);

/* Set the device error word of `workspace` to 0 (asynchronous on stream). */
MISA_API misa_status misa_error_reset(void* workspace, misa_stream_t stream);

/* Synchronise `stream`, copy the device error word to *host_bits (host
 * pointer) and return MISA_OK if it is 0, MISA_ERR_DEVICE otherwise. */
MISA_API misa_status misa_error_query(const void* workspace, misa_stream_t stream, uint32_t* host_bits);

/*
 * misa_block_stats -- mean-pooled key blocks (the router's block statistics).
 *   [MISA page, "Methodology: MISA": the prefix is split into M = ceil(L/B)
 *   blocks summarised by their mean-pooled indexer keys; HISA page, Stage 1:
 *   one mean-pooled representative per B-token block.]
 * keys: nseq caches of L keys (row stride 128, sequence stride key_seq_stride
 * elements; key_seq_stride may be 0 when nseq == 1).  Writes
 *   means[b * M * 128 + j * 128 + c] = mean over s in block j of keys[b][s][c]
 * as fp32 (fp32 accumulation of the bf16 inputs), M = ceil(L / B); the last,
 * partial block averages the L - (M-1)*B keys it holds.
 * means_hi, means_lo: both NULL, or both [nseq][M][128] bf16 at the same
 * element offsets as means, receiving the split of each mean m into
 * hi = bf16(m) and lo = bf16(m - hi) (round to nearest even), the two operands
 * the tensor-core router multiplies (about 16 significant bits together).
 * Passing them to misa_route_heads / hisa_block_filter saves the per-call split.
 * Limits: 1 <= B <= 4096, L >= 1, nseq >= 1.  keys, means, means_hi, means_lo
 * 16-byte aligned, key_seq_stride % 8 == 0.
 */
MISA_API misa_status misa_block_stats(const uint16_t* keys, int64_t nseq, int64_t L, int64_t key_seq_stride,
                             int B, float* means, uint16_t* means_hi, uint16_t* means_lo,
                             misa_stream_t stream);

/*
 * Block statistics over overlapping windows, and max pooling.
 *   [HISA page (zhichai.net), section 七 (局限与未来方向), 潜在改进: overlapping
 *   blocks to soften block-boundary effects, and max pooling in place of mean
 *   pooling, as ways around the information a block mean loses.  The pages give
 *   no layout; the library's reading:]
 * Window j of a cache of L keys covers keys [j*S, min(j*S + B, L)), for a window
 * length B and a stride 1 <= S <= B; there are
 *     M = misa_num_windows(L, B, S) = 1 + ceil(max(L - B, 0) / S)
 * windows, so every key is covered and no window lies inside another one's
 * extent.  S = B gives the plain blocks (M = ceil(L / B)) of the calls above.
 * The statistic of a window is the mean of its keys (MISA_POOL_MEAN) or their
 * coordinate-wise maximum (MISA_POOL_MAX; keys must be finite).  The _ex calls
 * below take (B, S, pool); the plain calls are the same with S = B and
 * MISA_POOL_MEAN.  Visibility generalises to windows: a routing decision (and a
 * HISA window score) sees window j iff min(j*S + B, L) <= prefix_len; HISA keeps
 * every window the prefix cuts (j*S < prefix_len < min(j*S + B, L)).
 * Workspace sizes: misa_workspace_bytes with S passed as B is enough for the
 * windows of stride S (ceil(L / S) >= M).
 */
#define MISA_POOL_MEAN 0
#define MISA_POOL_MAX 1

/* M = 1 + ceil(max(L - B, 0) / S) (host; 0 for L < 1, B < 1, S < 1 or S > B). */
MISA_API int64_t misa_num_windows(int64_t L, int B, int S);

/*
 * misa_block_stats_ex -- misa_block_stats over windows of B keys every S keys,
 * mean or max pooled.  means (and means_hi / means_lo) are [nseq][M][128] with
 * M = misa_num_windows(L, B, S); the bf16 split of a max is (max, 0) exactly.
 * Limits as misa_block_stats, and 1 <= S <= B, pool in {MISA_POOL_MEAN,
 * MISA_POOL_MAX}.
 */
MISA_API misa_status misa_block_stats_ex(const uint16_t* keys, int64_t nseq, int64_t L, int64_t key_seq_stride,
                                         int B, int S, int pool, float* means, uint16_t* means_hi,
                                         uint16_t* means_lo, misa_stream_t stream);

/*
 * misa_append_keys_ex -- misa_append_keys for windowed / max-pooled
 * statistics: every window the new rows [len[b], len[b] + n_new) touch (those
 * reaching past len[b], up to the last window of the longer cache) is
 * recomputed over the longer cache, bit for bit what misa_block_stats_ex
 * computes on it.  means_seq_stride >= misa_num_windows(L_cap, B, S) * 128.
 */
MISA_API misa_status misa_append_keys_ex(uint16_t* keys, int64_t nseq, int64_t key_seq_stride, int64_t L_cap,
                                         const int32_t* len, const uint16_t* new_keys, int n_new, int B, int S,
                                         int pool, float* means, uint16_t* means_hi, uint16_t* means_lo,
                                         int64_t means_seq_stride, void* workspace, size_t workspace_bytes,
                                         misa_stream_t stream);

/*
 * misa_append_keys -- append indexer keys to nseq caches and keep their block
 * statistics current (the step before the indexer on every decode step).
 *   [MISA page, "Methodology: MISA": the router reads mean-pooled blocks of the
 *   indexer keys; HISA page, Stage 1: one mean-pooled representative per block.
 *   How the statistics are maintained as the cache grows is not described; this
 *   call recomputes the blocks the new keys touch.]
 * keys: nseq caches of capacity L_cap rows (row stride 128, sequence stride
 *   key_seq_stride >= L_cap * 128 elements when nseq > 1), device, in/out.
 * len: [nseq] int32, device: keys already in each cache (not modified; the
 *   caller advances it by n_new).
 * new_keys: [nseq][n_new][128] bf16, device: copied to rows
 *   [len[b], len[b] + n_new) of cache b.
 * means: [nseq] x means_seq_stride fp32, device, in/out; means_seq_stride >=
 *   ceil(L_cap / B) * 128, a multiple of 128.  Every block j that the new rows
 *   touch is rewritten as the mean of rows [j*B, min((j+1)*B, len[b] + n_new)),
 *   bit for bit what misa_block_stats computes on the longer cache; other
 *   blocks are untouched.
 * means_hi, means_lo: both NULL, or both bf16 at the same element offsets as
 *   means (stride means_seq_stride), in/out: the touched blocks' split is
 *   rewritten as misa_block_stats writes it.
 * A sequence with len[b] < 0 or len[b] + n_new > L_cap is skipped and sets
 * MISA_DEVERR_BAD_LEN in the workspace error word.
 * Limits: 1 <= B <= 4096, 1 <= n_new, nseq >= 1; keys, new_keys, means,
 *   means_hi, means_lo 16-byte aligned; key_seq_stride % 8 == 0.
 * workspace: >= 256 bytes (the error word).
 */
MISA_API misa_status misa_append_keys(uint16_t* keys, int64_t nseq, int64_t key_seq_stride, int64_t L_cap,
                             const int32_t* len, const uint16_t* new_keys, int n_new, int B, float* means,
                             uint16_t* means_hi, uint16_t* means_lo, int64_t means_seq_stride,
                             void* workspace, size_t workspace_bytes, misa_stream_t stream);

/*
 * misa_route_heads -- block-aggregated head router (MISA).
 *   [MISA page, "Methodology: MISA": per-head affinities against the block
 *   statistics, aggregated into an importance per head, top-h heads kept; cost
 *   O(H * M) per query.  MISA forum thread (zingnex.cn), "核心架构：轻量级路由器",
 *   step 2: 8 of 64 heads kept per query.]
 * Affinity A[t, h, j] = w[t, h] * ReLU(q[t, h] . means[seq_of[t]][j]).
 * Queries [g*q_block, min((g+1)*q_block, T)) form routing decision g; block j is
 * visible to it iff min((j+1)*B, L) <= prefix_len[g*q_block].
 * importance[g][h] = sum over the decision's queries t and visible blocks j of
 * A[t, h, j]; heads[g][0..h) = the h heads of largest importance (ties: lower
 * head id), written in ascending id order.
 *   means: nseq sequences of [M][128] fp32 at sequence stride means_seq_stride
 *          elements (as written by misa_block_stats: M * 128); 16-byte aligned,
 *          means_seq_stride % 128 == 0; seq_of values must lie in [0, nseq).
 *   means_hi, means_lo: both NULL, or both the bf16 split misa_block_stats
 *          writes, laid out like means.  When given they are read instead of
 *          means (which may then be NULL) and the results are bit-identical.
 *   heads: [ceil(T/q_block)][h] int32 out.  importance: [ceil(T/q_block)][H]
 *          fp32 out, may be NULL.
 * Limits: 1 <= H <= 128, 1 <= h <= H, 1 <= q_block, T >= 1.
 * workspace: >= misa_workspace_bytes(MISA_OP_ROUTE_HEADS, T, H, L, B, 0, 0);
 *   its contents on entry do not matter (the call clears the scratch it relies
 *   on with an asynchronous memset on `stream`), apart from the error word.
 */
MISA_API misa_status misa_route_heads(const uint16_t* q, const float* w, const float* means,
                             const uint16_t* means_hi, const uint16_t* means_lo, int64_t nseq, int64_t means_seq_stride, const int32_t* seq_of,
                             const int32_t* prefix_len, int T, int H, int64_t L, int B,
                             int q_block, int h, int32_t* heads, float* importance,
                             void* workspace, size_t workspace_bytes, misa_stream_t stream);

/*
 * misa_route_heads_ex -- misa_route_heads over window statistics of stride S
 * (means [nseq][M][128], M = misa_num_windows(L, B, S), as misa_block_stats_ex
 * writes them, mean or max pooled: the router reads whatever statistic it is
 * given).  Window j is visible iff min(j*S + B, L) <= prefix_len[g*q_block].
 * 1 <= S <= B.  workspace: >= misa_workspace_bytes(MISA_OP_ROUTE_HEADS, T, H,
 * L, S, 0, 0).
 */
MISA_API misa_status misa_route_heads_ex(const uint16_t* q, const float* w, const float* means,
                                         const uint16_t* means_hi, const uint16_t* means_lo, int64_t nseq,
                                         int64_t means_seq_stride, const int32_t* seq_of, const int32_t* prefix_len,
                                         int T, int H, int64_t L, int B, int S, int q_block, int h, int32_t* heads,
                                         float* importance, void* workspace, size_t workspace_bytes,
                                         misa_stream_t stream);

/*
 * misa_route_heads_noalloc -- misa_route_heads without a caller workspace.
 *   The papers have no counterpart to this call; it is a library convenience.
 * For callers that cannot allocate device memory at the point where they route:
 * an inference engine that reserved all device memory up front and gives its
 * plug-ins no allocator, or a serving loop that must not call cudaMalloc /
 * cudaFree because they can synchronise the whole device.  Inputs (fp32 means
 * only, no bf16 split), outputs and results are exactly those of
 * misa_route_heads (same kernels); only the
 * router's per-chunk partial importances move from the workspace into a fixed
 * array of MISA_ROUTE_NOALLOC_SCRATCH_BYTES bytes compiled into the library,
 * which every device that loads the library holds until the process exits.
 *  - Calls with T * ceil(ceil(L/B) / 32) * H * 4 (rounded up to 256) +
 *    4 * ceil(T / q_block) > MISA_ROUTE_NOALLOC_SCRATCH_BYTES are rejected with
 *    MISA_ERR_UNSUPPORTED before anything is launched.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - All calls on one device share the array and it keeps the last call's
 *    contents; each call clears the per-decision counters it uses (an
 *    asynchronous memset on `stream`, no allocation).  Calls whose kernels can
 *    overlap on the GPU (unordered streams) race on it and give wrong results:
 *    order them on one stream or with events.
 *  - There is no device error word: an out-of-range seq_of is clamped to 0
 *    without being reported, and a pipeline wait that gives up (about two
 *    seconds, which only a stalled GPU reaches) stops the kernel with the
 *    affected heads left unwritten, also unreported.
 *  - The cached address is only valid in the CUDA context it was looked up
 *    in: do not call this function again after cudaDeviceReset.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
#define MISA_ROUTE_NOALLOC_SCRATCH_BYTES (2u << 20)
MISA_API misa_status misa_route_heads_noalloc(const uint16_t* q, const float* w, const float* means,
                                              int64_t nseq, int64_t means_seq_stride, const int32_t* seq_of,
                                              const int32_t* prefix_len, int T, int H, int64_t L, int B,
                                              int q_block, int h, int32_t* heads, float* importance,
                                              misa_stream_t stream);

/*
 * misa_index_score -- indexer scores of the active heads (the hot loop).
 *   [MISA page, "Methodology: MISA": only the h active heads score every
 *   prefix token; "Problem statement": the dense DSA indexer scores every prefix
 *   token with all H_I heads.  HISA page, Stage 2: the token indexer runs only
 *   inside the selected blocks (candidate mode).]
 * Active heads of query t: heads[(t / q_block) * h + i], i < h (any order; the
 * sum runs in ascending i), or all H heads when heads == NULL (dense indexer; h
 * is then ignored and taken as H).
 *   cand == NULL: scores[t * scores_row_stride + s] for 0 <= s < L, -inf where
 *     s >= prefix_len[t].
 *   cand != NULL: cand is [T][n_cand] int32 token ids (-1 = empty slot);
 *     scores[t * scores_row_stride + p] for 0 <= p < n_cand is the score of token
 *     cand[t][p], or -inf if that id is < 0 or >= min(prefix_len[t], L).
 * keys: nkeyseq caches (seq_of values must lie in [0, nkeyseq)); key_seq_stride
 *   must be 0 when nkeyseq == 1 and queries share the cache.
 * Limits: 1 <= H <= 128, 1 <= h <= 128, L >= 1, keys 16-byte aligned,
 *   key_seq_stride % 128 == 0, scores_row_stride >= (cand ? n_cand : L).
 * workspace: >= 256 bytes (error word).
 */
MISA_API misa_status misa_index_score(const uint16_t* q, const float* w, const uint16_t* keys,
                             int64_t nkeyseq, int64_t key_seq_stride, const int32_t* seq_of,
                             const int32_t* prefix_len, int T, int H, int64_t L,
                             const int32_t* heads, int h, int q_block,
                             const int32_t* cand, int n_cand,
                             float* scores, int64_t scores_row_stride,
                             void* workspace, size_t workspace_bytes, misa_stream_t stream);

/*
 * misa_index_score_blocks -- the dense indexer (all H heads) over the tokens of
 * chosen key blocks, read block by block.
 *   [HISA page, section 三, Stage 2: inside the m chosen blocks the token-level
 *   indexer scores every token; the candidates are the blocks' tokens.]
 * blocks: [T][m] int32 block ids of B keys each (B = 64 or 128), -1 = empty
 * slot (as hisa_block_filter writes them with stride B).  scores[t][i*B + r] =
 * sum over h of w[t,h] * ReLU(q[t,h] . keys[blocks[t][i]*B + r]) when the
 * block slot is filled and the token is inside the prefix (< min(prefix_len,
 * L)), -inf otherwise -- bit for bit what misa_index_score computes on the
 * candidate list cand[t][i*B + r] = blocks[t][i]*B + r (-1 past the prefix).
 * Each block's keys are read as whole tiles (no per-row gather).  A block id
 * at or past ceil(L / B) records MISA_DEVERR_BAD_INDEX and scores -inf.
 * Limits: as misa_index_score (heads NULL), m*B < 2^31, scores_row_stride >=
 * m*B.  workspace: >= 256 bytes (error word).
 */
MISA_API misa_status misa_index_score_blocks(const uint16_t* q, const float* w, const uint16_t* keys,
                                             int64_t nkeyseq, int64_t key_seq_stride, const int32_t* seq_of,
                                             const int32_t* prefix_len, int T, int H, int64_t L,
                                             const int32_t* blocks, int m, int B, float* scores,
                                             int64_t scores_row_stride, void* workspace, size_t workspace_bytes,
                                             misa_stream_t stream);

/*
 * misa_index_decode -- one whole MISA decode step in one call: the router and
 * the routed token scoring in one persistent kernel, the per-query top-k in a
 * second kernel that starts while the first one's last CTAs finish.
 *   [MISA page (gist.science), "Methodology: MISA": the router reads the
 *   mean-pooled block statistics and keeps h of the H heads per query; only
 *   those heads score every prefix token; the top-k tokens are kept.]
 * Computes exactly what misa_route_heads (q_block = 1, bf16 split means),
 * misa_index_score (with those heads) and misa_topk (row_valid = prefix_len)
 * compute one after the other, with one query per routing decision:
 *   heads [T][h] out (ascending ids), importance [T][H] out (may be NULL),
 *   scores [T] rows of L fp32 out (row stride scores_row_stride; -inf past the
 *     prefix; the top-k reads them back from L2, so they are also an output),
 *   idx [T][k] out (ascending positions, -1 padded), or NULL: no top-k, the
 *     call ends with the scores (k is still checked).
 * The importances are summed in another order than misa_route_heads sums them
 * (a per-block reduction on the tensor-core accumulator), so they can differ
 * in the last bits and a head choice can differ where two importances are that
 * close; given the heads, the scores equal misa_index_score's bit for bit and
 * idx is misa_topk's of the scores written.
 * means_hi / means_lo: the bf16 split misa_block_stats writes (block size B,
 * nmeanseq sequences of ceil(L/B) rows at stride means_seq_stride, a multiple
 * of 128).  Keys as misa_index_score.
 * Limits: 1 <= H <= 64, 1 <= h <= 16, h <= H, 1 <= L <= 65536, 1 <= k <=
 *   MISA_MAX_TOPK, T <= MISA_MAX_TOPK_ROWS; other shapes return
 *   MISA_ERR_UNSUPPORTED (use the separate calls).  q, keys, means_hi,
 *   means_lo, scores 16-byte aligned, scores_row_stride >= L and a multiple
 *   of 4.
 * workspace: >= misa_workspace_bytes(MISA_OP_INDEX_DECODE, T, H, L, B, k, 0)
 *   (the error word).
 */
MISA_API misa_status misa_index_decode(const uint16_t* q, const float* w, const uint16_t* keys, int64_t nkeyseq,
                                       int64_t key_seq_stride, const uint16_t* means_hi, const uint16_t* means_lo,
                                       int64_t nmeanseq, int64_t means_seq_stride, const int32_t* seq_of,
                                       const int32_t* prefix_len, int T, int H, int64_t L, int B, int h, int k,
                                       int32_t* heads, float* importance, float* scores, int64_t scores_row_stride,
                                       int32_t* idx, void* workspace, size_t workspace_bytes, misa_stream_t stream);

/*
 * misa_topk -- per-row top-k of fp32 scores (fused radix select).
 *   [MISA forum thread, "DeepSeek稀疏注意力（DSA）的突破": the indexer keeps the
 *   most relevant token subset; HISA page, section 二: top-k tokens per query;
 *   section 四: the output is k token indices.]
 * Row t is scores[t * row_stride + p], 0 <= p < n_t, with n_t = n, or
 * min(n, row_valid[t]) when row_valid != NULL.  idx[t * k + i] receives the
 * selected positions in ascending order (translated through
 * id_map[t * id_map_stride + p] when id_map != NULL), -1 padded.
 * Limits: 1 <= k <= MISA_MAX_TOPK, 1 <= T <= MISA_MAX_TOPK_ROWS, 1 <= n < 2^31,
 *   row_stride % 4 == 0 and >= n, scores 16-byte aligned.
 * workspace: >= 256 bytes.
 */
MISA_API misa_status misa_topk(const float* scores, int T, int64_t n, int64_t row_stride,
                      const int32_t* row_valid, const int32_t* id_map, int64_t id_map_stride,
                      int k, int32_t* idx, void* workspace, size_t workspace_bytes,
                      misa_stream_t stream);

/*
 * misa_hier_rerank -- fine stage of MISA-dagger: all H heads rescore each
 * query's k' candidates and the top-k of them are kept.
 *   [MISA page, "Hierarchical variant (MISA-dagger)": the original DSA indexer
 *   (all H_I heads) rescores only the candidate set; the final top-k is taken
 *   among the candidates.]
 * cand: [T][kp] int32 token ids (typically the coarse misa_topk output, -1 =
 * empty).  cand_scores: [T][kp] fp32 out, may be NULL.  idx: [T][k] out
 * (token ids, ascending candidate position order, -1 padded).
 * Limits: as misa_index_score and misa_topk; 1 <= k <= kp.
 * workspace: >= misa_workspace_bytes(MISA_OP_HIER_RERANK, T, H, L, B, k, kp).
 */
MISA_API misa_status misa_hier_rerank(const uint16_t* q, const float* w, const uint16_t* keys,
                             int64_t nkeyseq, int64_t key_seq_stride, const int32_t* seq_of,
                             const int32_t* prefix_len, int T, int H, int64_t L,
                             const int32_t* cand, int kp, int k, float* cand_scores,
                             int32_t* idx, void* workspace, size_t workspace_bytes,
                             misa_stream_t stream);

/*
 * hisa_block_filter -- HISA Stage 1: block scores with all heads, top-m blocks,
 * candidate token list.
 *   [HISA page, section 三, Stage 1: the query is scored against the
 *   mean-pooled block representatives only and the top-m blocks are kept, cost
 *   O(L/B); Stage 2 then looks at the at most m*B tokens inside them.]
 * block score bs[t][j] = sum over all H heads of w[t,h] * ReLU(q[t,h] . means_j)
 * for wholly visible blocks (min((j+1)*B, L) <= prefix_len[t]); +inf for the
 * block the prefix cuts (j*B < prefix_len[t] < min((j+1)*B, L): a causal
 * query's own block, whose mean would include future keys, is always kept and
 * masked token by token below); -inf otherwise.
 * blocks[t][0..m): chosen block ids ascending, -1 padded.
 * cand[t][i*B + r] = blocks[t][i]*B + r, or -1 if that block slot is empty or the
 * id is >= min(prefix_len[t], L).  block_scores: [T][M] fp32 out, may be NULL.
 * means / means_hi / means_lo / nseq / seq_of as for misa_route_heads
 * (means_seq_stride % 128 == 0).
 * Limits: 1 <= H <= 128, 1 <= m <= MISA_MAX_TOPK, 1 <= B.
 * workspace: >= misa_workspace_bytes(MISA_OP_HISA_BLOCK_FILTER, T, H, L, B, m, 0).
 */
MISA_API misa_status hisa_block_filter(const uint16_t* q, const float* w, const float* means,
                              const uint16_t* means_hi, const uint16_t* means_lo, int64_t nseq, int64_t means_seq_stride, const int32_t* seq_of,
                              const int32_t* prefix_len, int T, int H, int64_t L, int B, int m,
                              int32_t* blocks, int32_t* cand, float* block_scores,
                              void* workspace, size_t workspace_bytes, misa_stream_t stream);

/*
 * hisa_block_filter_ex -- hisa_block_filter over window statistics of stride S
 * (overlapping windows when S < B; mean or max pooled, as misa_block_stats_ex
 * writes them).  bs[t][j] over the M = misa_num_windows(L, B, S) windows, with
 * the visibility and cut rules above.  blocks[t][0..m): chosen window ids
 * ascending, -1 padded.  cand[t][i*B + r] = blocks[t][i]*S + r, or -1 if the
 * slot is empty, the id is >= min(prefix_len[t], L), or an earlier chosen
 * window already lists it (id < blocks[t][i-1]*S + B): each token appears at
 * most once and the listed ids ascend.  block_scores: [T][M] fp32 out, may be
 * NULL.  1 <= S <= B.
 * workspace: >= misa_workspace_bytes(MISA_OP_HISA_BLOCK_FILTER, T, H, L, S, m, 0).
 */
MISA_API misa_status hisa_block_filter_ex(const uint16_t* q, const float* w, const float* means,
                                          const uint16_t* means_hi, const uint16_t* means_lo, int64_t nseq,
                                          int64_t means_seq_stride, const int32_t* seq_of,
                                          const int32_t* prefix_len, int T, int H, int64_t L, int B, int S, int m,
                                          int32_t* blocks, int32_t* cand, float* block_scores, void* workspace,
                                          size_t workspace_bytes, misa_stream_t stream);

/*
 * misa_selftest_wait_timeout -- failure-detection self-test (no counterpart in
 * the pages).  Launches one CTA that waits, through the bounded wait every
 * pipeline of the library uses, on an mbarrier that nothing completes.  After
 * the wait's limit (about two seconds) the kernel records MISA_DEVERR_TIMEOUT
 * in the workspace error word, writes 0 to the word after it (1 would mean the
 * wait wrongly succeeded) and returns; the context stays usable.  Read the
 * outcome with misa_error_query.  workspace: >= 256 bytes, device.
 */
MISA_API misa_status misa_selftest_wait_timeout(void* workspace, size_t workspace_bytes, misa_stream_t stream);

/*
 * misa_shard_prefix -- prefix lengths of one key shard (context parallelism).
 *   [MISA page (gist.science), "Methodology: MISA": the head importance sums
 *   over visible blocks and the scores are per token, so a key shard can be
 *   indexed on its own.  The pages do not shard; this is the library's
 *   key-sharded form.]
 * A rank holds keys [s0, s0 + L_shard) of every sequence; its key at local
 * position s is visible to query t iff s < out[t] = clamp(prefix_len[t] - s0,
 * 0, L_shard).  Pass out as the prefix_len of misa_route_heads /
 * misa_index_score / misa_topk (row_valid) over the shard (s0 a multiple of B,
 * so the shard's blocks are the global blocks).
 * prefix_len, out: [T] int32, device.  T >= 1, s0 >= 0, L_shard >= 1.
 */
MISA_API misa_status misa_shard_prefix(const int32_t* prefix_len, int T, int64_t s0, int64_t L_shard, int32_t* out,
                             misa_stream_t stream);

/*
 * misa_gather_candidates -- (score, global token id) pairs of a shard's local
 * top-k, for the exchange that merges the shards.
 *   out_scores[t][i] = scores[t * row_stride + idx[t][i]] and
 *   out_ids[t][i] = idx[t][i] + id_offset when 0 <= idx[t][i] < n; otherwise
 *   (-inf, -1), which misa_topk never selects.  The top-k of the union of the
 *   shards' candidate lists (misa_topk with id_map = the gathered ids, shards
 *   in ascending s0 order) is the top-k of the whole row, ties included: the
 *   lists are ascending, so the lower position is the lower token id.
 * scores: [T] rows of n fp32 (row stride row_stride); idx: [T][k] int32 local
 * positions; out_scores [T][k] fp32, out_ids [T][k] int32; all device.
 * Limits: T >= 1, 1 <= k, n >= 1, row_stride >= n, 0 <= id_offset and
 *   id_offset + n < 2^31.
 */
MISA_API misa_status misa_gather_candidates(const float* scores, int T, int64_t n, int64_t row_stride,
                             const int32_t* idx, int k, int64_t id_offset, float* out_scores,
                             int32_t* out_ids, misa_stream_t stream);

/*
 * misa_sparse_mla -- attention of every query head over its query's k selected
 * tokens (the operator the indexer feeds).
 *   [HISA page (zhichai.net), section 二 (DSA 的工作原理): after the indexer
 *   picks k tokens per query, attention is computed over those tokens only;
 *   section 四 (Drop-in Replacement): that operator (Sparse MLA) takes the k
 *   token indices over the unchanged KV cache.  The pages print no formula;
 *   this is textbook softmax attention in the multi-query latent form a
 *   DeepSeek-V3.2-shaped model decodes with.]
 * kv: nseq caches of L latent rows of MISA_MLA_DQK bf16 (row stride 576,
 *   sequence stride kv_seq_stride elements, 0 allowed when nseq == 1), shared by
 *   all query heads: keys are whole rows, values their first MISA_MLA_DV entries.
 * q: [T][Hq][576] bf16 (the queries with the key up-projection absorbed).
 * idx: [T] rows of k int32 slots (row stride idx_stride >= k): token ids in
 *   [0, L) of cache seq_of[t]; -1 = empty slot (the indexer's padding).  Other
 *   values set MISA_DEVERR_BAD_INDEX and are treated as empty.  Each listed slot
 *   takes part once.
 *   out[t][h] = sum_i p_i v_i / sum_i p_i over the listed slots i, with
 *   p_i = exp(scale * q[t][h] . k_i - max); bf16 [T][Hq][512].  A query with no
 *   valid slot gets zeros.
 * lse: [T][Hq] fp32 natural-log sum_i exp(scale * q . k_i) (-inf when empty),
 *   may be NULL.
 * Precision: scores fp32 (bf16 inputs), weights rounded to bf16 for the value
 *   product, fp32 accumulation, bf16 output.
 * Limits: 1 <= Hq <= 128, 1 <= k <= MISA_MAX_TOPK, T >= 1; q, kv, out 16-byte
 *   aligned; kv_seq_stride % 8 == 0 and >= L * 576 when nseq > 1.
 * workspace: >= misa_workspace_bytes(MISA_OP_SPARSE_MLA, T, Hq, 0, 0, k, 0)
 *   (per-chunk partial results: T * ceil(k / 256) * Hq * 514 * 4 bytes + 256).
 */
MISA_API misa_status misa_sparse_mla(const uint16_t* q, const uint16_t* kv, int64_t nseq, int64_t kv_seq_stride,
                             int64_t L, const int32_t* seq_of, int T, int Hq, const int32_t* idx, int k,
                             int64_t idx_stride, float scale, uint16_t* out, float* lse, void* workspace,
                             size_t workspace_bytes, misa_stream_t stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif /* MISA_H */
