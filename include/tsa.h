/*
 * tsa.h -- C ABI of libtsa: top-k context-sparse attention at decode, B200 (sm_100a).
 *
 * The operation (one decode step of one attention layer, GQA):
 *   1. score  every cached key against the current query group
 *             ("inference-time context sparsity: illusion or opportunity?",
 *             sec. 2, oracle Top-K: the k most important tokens are chosen
 *             exactly, with no approximate indexer; "Flash Attention vs Sparse
 *             Attention", DeepSeek Sparse Attention stage 1, the indexer pass);
 *   2. select the top-k token (or 128-token block) indices per sequence and
 *             kv-head (same sections);
 *   3. attend exactly, with softmax, over only the selected K/V rows
 *             (HyLRA sec. 2.3 hybrid inference: attention limited to the
 *             subset; DSA stage 2 selective attention), computed as split-K
 *             flash decoding with an online softmax ("Flash Attention vs Sparse
 *             Attention", tiling + online softmax).
 * A layer may instead reuse the previous layer's indices (HyLRA sec. 2.1/2.3
 * tolerant layers; IndexCache in "Flash Attention vs Sparse Attention") or run
 * full attention (Flux Attention sec. 1/3 hard per-layer routing; HyLRA
 * sensitive layers).  Block mode scores 128-token blocks by q . (block-mean key)
 * (HyLRA sec. 2.4, block-level sparsity).
 *
 * Conventions (every entry point):
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, never frees and never synchronises (except
 *    tsa_check_device_status).  Work is enqueued on `stream` (a cudaStream_t;
 *    NULL = the legacy default stream) and runs asynchronously.
 *  - Shapes: Q [B, Hq, d] bf16; K, V [B, Hkv, Ncap, d] bf16 (row-major,
 *    contiguous); seq_lens [B] int32 with 0 <= len_b <= Ncap; d must be 128;
 *    Hq must be g * Hkv with g in {1, 2, 4, 8}.  Kv-head kvh serves query heads
 *    kvh*g .. kvh*g+g-1.  Q, K, V, Kmean, O must be 16-byte aligned.
 *  - "Unit" = (b, kvh).  In token mode a unit has n_b = len_b rows; in block
 *    mode (block > 1) it has n_b = ceil(len_b / block) blocks.
 *  - k_per_seq [B] int32 (device) or NULL (= k_max for every sequence);
 *    k_b = min(k_per_seq[b], n_b) and must not exceed k_max.
 *  - idx [B, Hkv, k_max] int32: the k_b selected rows (or blocks) in ascending
 *    order, then -1.
 *  - scale must be finite and > 0 (scores are stored scaled).
 *  - Errors: an argument error returns a status before anything is enqueued
 *    (tsa_last_error_string() says which).  A failed launch returns
 *    TSA_ERR_CUDA.  Errors only the device can see (a len_b above Ncap, a k_b
 *    above k_max, an index out of range) skip the offending work, never fault,
 *    and set a flag in the first 256 bytes of `ws`, read by
 *    tsa_check_device_status.  No C++ exception crosses this boundary.
 *  - Workspace: `ws` is caller-owned device memory of at least
 *    tsa_workspace_size(...) bytes, 256-byte aligned, set to zero once with
 *    tsa_workspace_init before first use.  Calls that share a workspace must be
 *    ordered on one stream; calls that overlap on the GPU with the same `ws` race.
 *    Between its scorer and its top-k a SELECT decode step keeps per-unit
 *    counts in the workspace, which the top-k returns to zero; after any call
 *    that returned TSA_ERR_CUDA, run tsa_workspace_init again before reusing it.
 */
#ifndef TSA_H
#define TSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TSA_OK = 0,
    TSA_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or value */
    TSA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (d != 128, g not in {1,2,4,8}) */
    TSA_ERR_WORKSPACE = 3,     /* ws NULL or smaller than tsa_workspace_size() */
    TSA_ERR_CUDA = 4,          /* a CUDA launch or query failed */
    TSA_ERR_DEVICE_BOUNDS = 5, /* device saw a length / k / index out of range */
    TSA_ERR_DEVICE_TIMEOUT = 6 /* a bounded device-side wait gave up */
} tsa_status;

typedef enum { TSA_FULL = 0, TSA_SELECT = 1, TSA_REUSE = 2 } tsa_mode;

typedef struct {
    int32_t B;    /* sequences in the batch */
    int32_t Hq;   /* query heads */
    int32_t Hkv;  /* kv heads (Hq = g * Hkv) */
    int32_t Ncap; /* cache capacity in tokens (rows of K and V per unit) */
    int32_t d;    /* head dimension (must be 128) */
} tsa_shape;

/* ------------------------------------------------------------------ sizing */

/* Bytes of workspace that tsa_decode_step needs for (shape, k_max, block, mode);
 * enough for every other entry point called with the same arguments.  Layers of
 * different modes may share one workspace sized with the largest of their
 * sizes: every layout keeps the regions that must stay zero between calls (the
 * top-digit histograms, the split counters) at the same offsets.  Returns 0 on
 * invalid arguments (see tsa_last_error_string). */
size_t tsa_workspace_size(tsa_shape shape, int32_t k_max, int32_t block, int32_t mode);

/* Zero a workspace (enqueued memset).  Call once after allocating it. */
tsa_status tsa_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ stages */

/* Block summaries for block mode (HyLRA sec. 2.4): Kmean[b,kvh,beta,:] = fp32
 * mean of the valid K rows [beta*block, min(beta*block+block, len_b)).  Kmean is
 * [B, Hkv, ceil(Ncap/block), d] fp32; blocks past ceil(len_b/block) are not
 * written.  Run when the cache is appended to, outside the decode step. */
tsa_status tsa_block_summarize(const void* K, const int32_t* seq_lens, tsa_shape shape,
                               int32_t block, float* Kmean, void* ws, size_t ws_bytes,
                               void* stream);

/* Step 1, score (oracle Top-K criterion; DSA indexer pass):
 *   scores[b,kvh,j] = max over the group's heads h of scale * <q_h, key_j>,
 * bf16 products accumulated in fp32.  block == 1: keys = K (bf16, rows Ncap);
 * block > 1: keys = Kmean (fp32, rows ceil(Ncap/block)).  scores is
 * [B, Hkv, rows] fp32; only rows j < n_b are written. */
tsa_status sparse_decode_score(const void* Q, const void* keys, const int32_t* seq_lens,
                               tsa_shape shape, int32_t block, float scale, float* scores,
                               void* ws, size_t ws_bytes, void* stream);

/* Step 2, exact top-k per unit over scores [B, Hkv, rows] (rows as in
 * sparse_decode_score): the k_b largest, ties to the lower index, written to
 * idx in ascending order and padded with -1 (oracle Top-K, exact selection). */
tsa_status topk_select(const float* scores, const int32_t* seq_lens, const int32_t* k_per_seq,
                       int32_t k_max, tsa_shape shape, int32_t block, int32_t* idx, void* ws,
                       size_t ws_bytes, void* stream);

/* Step 3, exact softmax attention over the selected rows (selective attention;
 * split-K flash decoding with an online softmax, then a combine of the splits).
 *   idx == NULL : every valid row [0, len_b) (a full-attention layer);
 *   block == 1  : rows idx[b,kvh,0:k_b] (entries < 0 skipped);
 *   block  > 1  : idx holds block numbers; each expands to its valid rows.
 * O is [B, Hq, d] fp32; a head with no attended row gets O = 0.
 * Index reuse (HyLRA tolerant layers, IndexCache) is this call with a previous
 * layer's idx and no score/select. */
tsa_status sparse_decode_attn(const void* Q, const void* K, const void* V,
                              const int32_t* seq_lens, const int32_t* idx,
                              const int32_t* k_per_seq, int32_t k_max, int32_t block,
                              tsa_shape shape, float scale, float* O, void* ws, size_t ws_bytes,
                              void* stream);

/* Step 3 without a workspace.  The pages have no counterpart to this entry
 * point: it exists for callers that cannot allocate device memory for a
 * workspace (a plugin host that passes an operator only its inputs and outputs,
 * a runtime whose device memory all belongs to another allocator, a serving loop
 * that must not call cudaMalloc or cudaFree, which can block or synchronise the
 * device).  Same arguments, meaning and result as sparse_decode_attn, minus
 * ws/ws_bytes.  Its scratch (split counters and split partials) is a fixed
 * 8 MiB device array inside the library, which every GPU that loads the library
 * holds until the process exits.  It allocates nothing (no cudaMalloc, cudaFree
 * or allocating library routine).
 *  - Every call looks up that array's device address on the current device.
 *    The first call on a device loads the library's device code there (with
 *    CUDA's lazy module loading), which commits the array and may block: make
 *    it during warm-up, before any stream capture.
 *  - Every call clears the counters it needs, then launches: all calls share the
 *    one array, so calls that overlap on the GPU (different streams, or other
 *    host threads, on the same device) race and must be ordered by the caller.
 *  - A shape whose scratch exceeds 8 MiB returns TSA_ERR_WORKSPACE with the
 *    bytes it needs (use sparse_decode_attn with a workspace instead).  The
 *    array holds about 15,880 split partials of (d + 4) * 4 = 528 bytes (one
 *    per unit, split and query head); the 128K-token shape (8 units, 8 splits,
 *    4 heads) uses 135 KB of it.
 *  - Nothing the device detects is reported: the device flag lives in the
 *    shared array and the next call clears it.  Range errors skip the offending
 *    rows, as in sparse_decode_attn; a bounded wait that gives up (contiguous
 *    128-row tiles: idx == NULL, or block == 128) leaves O unspecified, and that
 *    goes unreported too.  A caller that must know uses sparse_decode_attn and
 *    tsa_check_device_status. */
tsa_status sparse_decode_attn_noalloc(const void* Q, const void* K, const void* V,
                                      const int32_t* seq_lens, const int32_t* idx,
                                      const int32_t* k_per_seq, int32_t k_max, int32_t block,
                                      tsa_shape shape, float scale, float* O, void* stream);

/* ------------------------------------------------------------------ one step */

typedef struct {
    tsa_shape shape;          /* as for the stage calls */
    const void* Q;            /* [B, Hq, d] bf16 */
    const void* K;            /* [B, Hkv, Ncap, d] bf16 */
    const void* V;            /* [B, Hkv, Ncap, d] bf16 */
    const float* Kmean;       /* block mode SELECT (and FULL with idx_out): from tsa_block_summarize */
    const int32_t* seq_lens;  /* [B] */
    const int32_t* k_per_seq; /* [B] or NULL (= k_max) */
    int32_t k_max;            /* columns of idx; TSA_FULL: used only with idx_out */
    int32_t block;            /* 1 = token mode, > 1 = block mode (128 in the pages) */
    int32_t mode;             /* TSA_FULL, TSA_SELECT or TSA_REUSE */
    float scale;              /* softmax scale, > 0 (1/sqrt(d) usually) */
    const int32_t* idx_in;    /* TSA_REUSE: the earlier layer's idx [B, Hkv, k_max] */
    int32_t* idx_out;         /* TSA_SELECT: this layer's idx [B, Hkv, k_max];
                               * TSA_FULL: NULL, or where the layer's own top-k goes */
    float* O;                 /* [B, Hq, d] fp32 */
    void* ws;                 /* workspace */
    size_t ws_bytes;
    uint32_t flags;           /* 0, or TSA_KV_HOST and/or TSA_EARLY_INPUTS */
} tsa_step_args;

/* tsa_step_args.flags: K and V live in page-locked host memory that the device
 * reads at the same address (cudaHostAlloc; or cudaHostRegister'd and mapped):
 * a cache larger than HBM, offloaded.  The attention then fetches only the
 * selected rows (or 128-token blocks) across the host link, with plain loads
 * through the device's mapping of the pages (index-guided offload, HyLRA sec.
 * 2.4: the block indices say which blocks to bring in).  Layers that select must
 * score block means (block > 1, Kmean in device memory), since token-mode
 * scoring reads every K row; TSA_SELECT or a TSA_FULL layer with idx_out in
 * token mode returns TSA_ERR_UNSUPPORTED.  TSA_REUSE works in either mode; a
 * TSA_FULL layer reads all of K and V across the link.  A K or V pointer that is
 * not such memory returns TSA_ERR_INVALID_ARG (pageable memory would fault). */
#define TSA_KV_HOST 1u

/* tsa_step_args.flags: the caller's promise that the kernel enqueued on
 * `stream` just before this step (the end of the previous layer, say) writes
 * none of seq_lens, k_per_seq, K, V and (TSA_REUSE) idx_in: they were written
 * two or more launches earlier, or are constant for the step.  The step's first
 * kernel may then read them before that kernel has finished (programmatic
 * dependent launch): a TSA_REUSE or TSA_FULL layer reads its index list and
 * issues the loads of its first K/V tiles, and a TSA_SELECT layer's scorer
 * requests its first K tiles, while the previous kernel runs.  Q, the
 * workspace, idx_out and O are still touched only after it has finished, so Q
 * may come from the kernel just before.  Breaking the promise gives results
 * computed from stale inputs (no fault).  Without the flag every kernel waits
 * for its predecessor before its first read. */
#define TSA_EARLY_INPUTS 2u

/* One decode step of one layer: TSA_SELECT = score -> top-k -> attention;
 * TSA_REUSE = attention over idx_in; TSA_FULL = attention over every valid row.
 * A TSA_FULL layer given idx_out (and k_max > 0) also writes the top-k that a
 * SELECT step would have chosen, so that the tolerant layers after it can reuse
 * it (HyLRA, sec. 2.3: the indices of a sensitive, fully attended layer are
 * handed on).  Token mode: the full attention writes each row's group-max
 * scaled score as it forms the logits, then the top-k runs on those; block
 * mode: the block means (Kmean) are scored first.  O is unchanged by idx_out;
 * the workspace must then be sized with tsa_workspace_size(shape, k_max,
 * block, TSA_FULL), k_max > 0. */
tsa_status tsa_decode_step(const tsa_step_args* args, void* stream);

/* ------------------------------------------------------------------ sequence sharding */

/* One sequence's cache split by rows across R ranks (R <= 64): shard r holds rows
 * [row0_r, row0_r + Ncap_r) of every unit, with row0 increasing with r (rank
 * order = row order), as K_shard, V_shard [B, Hkv, Ncap_r, d] and its own
 * lengths shard_lens[b] = clamp(len_b - row0_r, 0, Ncap_r).  A SELECT layer then
 * runs as: tsa_shard_select on every rank; an all-gather of the candidates (rank
 * order); tsa_shard_merge (every rank, same result); tsa_shard_attend on every
 * rank; an all-gather of the parts; tsa_shard_combine.  The result is the
 * single-GPU SELECT step's: the same indices (every row of the global top-k is
 * among its shard's top-k, and rank order keeps the lower-index tie rule) and
 * the same attention up to rounding (split-K over shards, as flash decoding
 * splits a sequence).  shard_shape is (B, Hq, Hkv, Ncap_r, d); `shape` in the
 * merge and combine calls is the same with any Ncap.  Workspace: at least
 * tsa_shard_workspace_size(shard_shape, k_max, n_shards), shared by the four
 * calls of a rank, initialised with tsa_workspace_init. */
size_t tsa_shard_workspace_size(tsa_shape shard_shape, int32_t k_max, int32_t n_shards);

/* This shard's top-k (score -> select, as in a SELECT step, with
 * k_b = min(k_per_seq[b], shard_lens[b])) as candidates: cand_scores
 * [B, Hkv, k_max] fp32 and cand_rows [B, Hkv, k_max] int32 GLOBAL rows
 * (row0 + local row), ascending, then (-inf, -1). */
tsa_status tsa_shard_select(const void* Q, const void* K_shard, const int32_t* shard_lens, tsa_shape shard_shape,
                            const int32_t* k_per_seq, int32_t k_max, float scale, int32_t row0,
                            float* cand_scores, int32_t* cand_rows, void* ws, size_t ws_bytes, void* stream);

/* The exact global top-k from the gathered candidates of all shards:
 * cand_scores, cand_rows [n_shards, B, Hkv, k_max] (rank order) -> idx
 * [B, Hkv, k_max] global rows, ascending, then -1.  Candidates out of row
 * order across shards set the device bounds flag. */
tsa_status tsa_shard_merge(const float* cand_scores, const int32_t* cand_rows, int32_t n_shards, tsa_shape shape,
                           const int32_t* k_per_seq, int32_t k_max, int32_t* idx, void* ws, size_t ws_bytes,
                           void* stream);

/* This shard's part of the attention over the global idx: the rows of idx in
 * [row0, row0 + Ncap_r).  O_part [B, Hq, d] fp32 is the softmax-normalised
 * output over those rows (0 if none) and lse_part [B, Hq] fp32 the base-2
 * log-sum-exp of their scaled logits, log2(sum_j 2^(scale*log2(e)*q.k_j)), or
 * -inf if the shard holds none of them. */
tsa_status tsa_shard_attend(const void* Q, const void* K_shard, const void* V_shard, const int32_t* shard_lens,
                            tsa_shape shard_shape, const int32_t* idx, const int32_t* k_per_seq, int32_t k_max,
                            int32_t row0, float scale, float* O_part, float* lse_part, void* ws, size_t ws_bytes,
                            void* stream);

/* O [B, Hq, d] = sum_r 2^(lse_r - M) O_r / sum_r 2^(lse_r - M), M = max_r lse_r
 * (0 where every lse_r is -inf), from O_parts [n_shards, B, Hq, d] and
 * lse_parts [n_shards, B, Hq].  O_parts and O 16-byte aligned. */
tsa_status tsa_shard_combine(const float* O_parts, const float* lse_parts, int32_t n_shards, tsa_shape shape,
                             float* O, void* stream);

/* ------------------------------------------------------------------ reuse profiling */

/* Overlap of the top-k index sets of n_layers layers: the similarity matrix
 * that HyLRA's offline policy search runs on (HyLRA sec. 2.2; M[i][j] there is
 * the overlap ratio of the top-k indices of source layer i and target layer j).
 *  - idx [n_layers, units, k_max] int32 (device): layer l's index lists for the
 *    units (b, kvh), units = B * Hkv, each in the form of `idx` above
 *    (ascending, then -1), e.g. the idx_out of n_layers decode steps.
 *  - counts [n_layers, n_layers, units] int32 (device) or NULL:
 *    counts[(i*n_layers + j)*units + u] = |I_i(u) ∩ I_j(u)| for every i, j
 *    (symmetric; the diagonal holds the list lengths |I_i(u)|).  Exact.
 *  - M [n_layers, n_layers] double (device) or NULL: for source i <= target j,
 *    M[j*n_layers + i] = the mean over the units with |I_j(u)| > 0 of
 *    |I_i(u) ∩ I_j(u)| / |I_j(u)| (the share of the target layer's top-k that
 *    reusing layer i's indices keeps), summed in unit order; 1 when every
 *    target list is empty; M[i*n_layers + j] = 0 for i < j.  So M is lower
 *    triangular with row = target layer, column = source layer.
 *  - Not both counts and M NULL; 1 <= n_layers <= 1024; ws: the first 256
 *    bytes (the device flag) are used.
 *  - A list that is not strictly ascending before its first -1, or holds
 *    anything but -1 after it, sets the device bounds flag
 *    (tsa_check_device_status); the results for that pair are then unspecified. */
tsa_status tsa_index_overlap(const int32_t* idx, int32_t n_layers, int32_t units, int32_t k_max,
                             int32_t* counts, double* M, void* ws, size_t ws_bytes, void* stream);

/* HyLRA's offline reuse policy (HyLRA sec. 2.2, dynamic programming over M).
 * HOST function: M, force_full, source, n_full and total_sim are host pointers;
 * nothing is enqueued and no GPU is needed.
 *  - M [n_layers, n_layers] double, the layout tsa_index_overlap writes:
 *    M[j*n_layers + i] = the similarity of source layer i to target layer j, i < j
 *    (entries on and above the diagonal are not read).
 *  - A policy gives every layer j a source s_j <= j: s_j = j is a full layer
 *    (a reset: full attention that hands on its top-k, TSA_FULL with idx_out);
 *    s_j = s_{j-1} < j reuses that source's indices (TSA_REUSE), allowed only
 *    if M[j][s_j] > theta (strictly).  Layer 0, and every layer with
 *    force_full[j] != 0 (force_full may be NULL), is a full layer.
 *  - The policy returned has the fewest full layers, then the largest sum over
 *    the reusing layers j of M[j][s_j] (added in layer order); among policies
 *    equal in both, the smallest source sequence compared from the last layer
 *    backwards.  source [n_layers] int32 receives it; n_full and total_sim (may
 *    be NULL) its two costs.
 *  - 1 <= n_layers <= 4096; theta not NaN (NaN entries of M never allow reuse). */
tsa_status tsa_reuse_policy(const double* M, int32_t n_layers, double theta, const uint8_t* force_full,
                            int32_t* source, int32_t* n_full, double* total_sim);

/* ------------------------------------------------------------------ status */

/* Wait for `stream`, then read and clear the device error flag in `ws`:
 * TSA_OK, TSA_ERR_DEVICE_BOUNDS or TSA_ERR_DEVICE_TIMEOUT (or TSA_ERR_CUDA). */
tsa_status tsa_check_device_status(void* ws, void* stream);

/* Text of the last error on this thread ("" if none). */
const char* tsa_last_error_string(void);

/* Kernels this library has launched in this process (all entry points). */
uint64_t tsa_launch_count(void);

/* ------------------------------------------------------------------ measurement */

/* HBM roofline probe: dst[0:bytes] = src[0:bytes] with 16-byte vector loads
 * and stores over a grid sized to the SM count.  bytes must be a multiple of 16. */
tsa_status tsa_hbm_copy(const void* src, void* dst, size_t bytes, void* stream);

/* HBM read probe: reads src[0:bytes] with the copy probe's 16-byte loads over a
 * grid of 16 CTAs an SM, and stores nothing (a fold of the words lands in the workspace's flag block only
 * for a value no buffer of repeated bytes gives).  Its bandwidth is the ceiling
 * of a read-only stream, above the copy's.  src and bytes must be multiples of
 * 16 bytes; ws >= 256 bytes (its first 8 bytes are the flag and that word). */
tsa_status tsa_hbm_read(const void* src, size_t bytes, void* ws, size_t ws_bytes, void* stream);

/* Random-row gather probe: fetch the 256-byte rows base[rows[i]*256 .. +256)
 * (rows[] on the device, nrows of them) into shared memory with bulk copies and
 * drop them.  Its bandwidth is the ceiling of a gather-bound stage (the
 * attention stage reads the selected K/V rows at random).  base_bytes must be a
 * multiple of 256; a row number outside [0, base_bytes/256) is skipped and sets
 * the device flag in ws (>= 256 bytes). */
tsa_status tsa_hbm_gather(const void* base, size_t base_bytes, const int32_t* rows, int32_t nrows, void* ws,
                          size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TSA_H */
