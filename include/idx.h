/*
 * idx.h -- C ABI of the B200 lightning-indexer + top-k library (libidx.so).
 *
 * The operation (PIVOT: "Efficient Query-Group Indexing for Token-Level
 * Sparse Attention", Method, first paragraph, Eq. (1); the equation text is
 * missing from the page, the DSA lightning-indexer form is used):
 *
 *     I[t,s] = sum_j w[t,j] * max(0, q[t,j] . k[s]),     0 <= s <= t,
 *
 * with t, s positions inside one request, followed by a per-query top-k:
 * the k keys of highest score, ties to the lower position, listed in
 * ascending position and padded with -1 when the prefix holds fewer than k.
 *
 * Grouped form (same page, Method, grouping paragraph; Experimental setup;
 * Abstract): each request is cut into contiguous groups of g queries (the
 * last one may be shorter, none crosses a request).  A group's proxy query
 * is the mean of its members' queries (fp32 sum in member order, IEEE
 * division, rounded to bf16 for bf16 inputs) and its proxy weight the mean
 * of their w (fp32).  One scan of the group's full prefix (up to its last
 * member) with the proxy gives
 *   - IDX_MODE_REUSE:  each member takes the proxy ranking restricted to its
 *                      own prefix (s <= t_member), first k entries;
 *   - IDX_MODE_REFINE: the proxy's top-c positions form the candidate set C;
 *                      each member re-scores C with its own q and w, masks
 *                      s > t_member and takes its own top-k.
 *   - IDX_MODE_BLOCK:  Refine over a candidate set from block summaries
 *                      instead of the token scan (pages "Not All Tokens
 *                      Deserve Equal Resolution", abstract: chunk summaries
 *                      first, exact token scores inside the chosen chunks;
 *                      "Uncertainty-gated selection for block-sparse
 *                      attention", Sec. 3.1: a 64-key block is summarised by
 *                      its mean key).  Each complete 64-token block of the
 *                      request that ends at or before the group's last
 *                      member t_last gets a mean key (fp32 sum in key order,
 *                      IEEE division, bf16 rounding for bf16 keys) and a
 *                      proxy score (the indexer score against that key).  C
 *                      is the tokens of the top c/64 blocks by (score desc,
 *                      block asc), one block fewer when t_last+1 is not a
 *                      multiple of 64, plus the partial block that holds
 *                      t_last.  Members then re-score C as in Refine.  No
 *                      key after t_last takes part.  c must be a multiple of
 *                      64 and >= topk.
 *   - IDX_MODE_QUEST:  IDX_MODE_BLOCK with the blocks ranked by the Quest
 *                      bound instead of the mean key (same page, Sec. 3.1,
 *                      Eq. (2)): a block is summarised by the per-dimension
 *                      minimum and maximum of its keys, and its proxy score
 *                      is sum_h wbar_h * max(0, sum_i max(qbar_hi * kmax_i,
 *                      qbar_hi * kmin_i)), the indexer's weighted ReLU of
 *                      each head's upper bound of q . k over the block.
 *                      Scored on CUDA cores in fp32; H * d * 8 bytes must fit
 *                      in one block's shared memory (else
 *                      IDX_ERR_UNSUPPORTED).  The workspace holds one fp32
 *                      score per (scored proxy, block of the longest
 *                      request): 4 * (T / g) * (T / 64) bytes for one
 *                      request of T tokens, bounded by row-range calls.
 *
 * Decode form (same page, Method, decode paragraph): the G queries of one
 * MTP step form one group; query m of request b sits at position
 * kv_len[b] - G + m and the cache already holds the keys of the group.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers, row-major and contiguous.
 *     bf16 tensors hold IEEE bfloat16; fp32 tensors IEEE binary32.
 *   - The caller owns every buffer.  The library never allocates device
 *     memory on these paths: scratch space is the caller's workspace `ws`
 *     of at least `*_workspace_size(...)` bytes, 256-byte aligned.
 *   - Every call is asynchronous on `stream` (NULL = legacy default stream).
 *     Argument errors are returned synchronously and nothing is launched.
 *     Device-side anomalies (a bounded wait that ran out, a scratch overflow)
 *     set a status word inside `ws`; read it with idx_device_status().
 *   - Indices are request-local positions (int32).  Selected scores, when
 *     requested, are the fp32 scores the selection used; padding slots get
 *     index -1 and score -INFINITY.
 *   - A workspace may be used by one call at a time; calls that share a
 *     workspace must be ordered on one stream.
 */
#ifndef IDX_H
#define IDX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *idx_stream_t; /* same object as cudaStream_t */

typedef enum {
    IDX_OK = 0,
    IDX_ERR_INVALID = 1,     /* bad argument (shape, pointer, k > c, ...) */
    IDX_ERR_UNSUPPORTED = 2, /* valid but not supported (e.g. a request longer than 2^20) */
    IDX_ERR_WORKSPACE = 3,   /* ws NULL, misaligned or smaller than *_workspace_size() */
    IDX_ERR_CUDA = 4,        /* a CUDA runtime call failed (launch, memset, ...) */
    IDX_ERR_TIMEOUT = 5,     /* device: a bounded wait ran out; the results are invalid */
    IDX_ERR_OVERFLOW = 6     /* device: a scratch buffer overflowed; the results are invalid */
} idx_status;

typedef enum { IDX_BF16 = 0, IDX_F32 = 1 } idx_dtype;

typedef enum {
    IDX_MODE_DENSE = 0,
    IDX_MODE_REUSE = 1,
    IDX_MODE_REFINE = 2,
    IDX_MODE_BLOCK = 3,
    IDX_MODE_QUEST = 4
} idx_mode;

/* ------------------------------------------------------------ prefill */

/* Workspace bytes for idx_dense_topk.  T = total tokens of the packed batch,
 * num_seqs = number of requests.  Returns 0 for invalid arguments. */
size_t idx_dense_workspace_size(int T, int H, int d, int topk, int num_seqs, idx_dtype dtype);

/* Dense indexer + top-k over a packed batch of requests (PIVOT page,
 * Method, first paragraph: every query scores its whole causal prefix).
 *   q          [T, H, d]  dtype       query of row t, head j
 *   k          [T, d]     dtype       key of row s (shared by all heads)
 *   w          [T, H]     fp32        head weights of row t
 *   cu_seqlens [num_seqs+1] int32     device; request b is rows
 *                                     cu_seqlens[b] .. cu_seqlens[b+1]-1,
 *                                     cu_seqlens[0] = 0, cu_seqlens[num_seqs] = T
 *   out_idx    [T, topk]  int32       selected request-local positions
 *   out_score  [T, topk]  fp32 or NULL
 * Requirements: T >= 1, H >= 1, d >= 1 and d % 8 == 0, topk >= 1,
 * every request no longer than 2^20 tokens (else IDX_ERR_UNSUPPORTED). */
idx_status idx_dense_topk(const void *q, const void *k, const float *w, const int *cu_seqlens,
                          int num_seqs, int T, int H, int d, int topk, idx_dtype dtype,
                          int *out_idx, float *out_score, void *ws, size_t ws_bytes,
                          idx_stream_t stream);

/* Workspace bytes for idx_adaptive_topk; 0 for arguments it would reject
 * (including rho*topk above 8192). */
size_t idx_adaptive_workspace_size(int T, int H, int d, int topk, int rho, int num_seqs, idx_dtype dtype);

/* Dense indexer + top-k with an adaptive budget ("Uncertainty-gated
 * selection for block-sparse attention", Section 3 Method, steps 3-5, and
 * Appendix A, steps (A.5)-(A.9)), on the indexer's per-query scores:
 *   sigma[t] = (s_(k-1) - s_(k)) / (s_(0) - s_(k))   (fp32; s_(i) = the row's
 *              i-th largest score; 0 when the first k+1 scores are equal;
 *              NaN when the row has at most k positions);
 *   tau      = the ceil(q n)-th smallest defined sigma over all T rows
 *              (n = rows with a defined sigma, q n formed in fp64; no row
 *              triggers when ceil(q n) = 0);
 *   trigger  = sigma[t] <= tau;
 * a triggered row lists its top-(rho topk); any other row its top-topk,
 * padded with -1 to rho*topk entries.  Positions ascending, ties to the lower
 * position, as in idx_dense_topk.
 *   q, k, w, cu_seqlens  as in idx_dense_topk
 *   rho          budget expansion, >= 2 (the page uses 2)
 *   qfrac        trigger quantile in [0, 1] (the page uses 0.4)
 *   out_idx      [T, rho*topk] int32
 *   out_score    [T, rho*topk] fp32 or NULL (-inf on padding)
 *   out_sigma    [T] fp32 or NULL
 *   out_trigger  [T] uint8 or NULL (1 = the row kept rho*topk)
 * Errors: rho < 2, qfrac outside [0, 1] or NaN -> IDX_ERR_INVALID;
 * rho*topk above 8192 -> IDX_ERR_UNSUPPORTED; otherwise as idx_dense_topk. */
idx_status idx_adaptive_topk(const void *q, const void *k, const float *w, const int *cu_seqlens,
                             int num_seqs, int T, int H, int d, int topk, int rho, double qfrac,
                             idx_dtype dtype, int *out_idx, float *out_score, float *out_sigma,
                             uint8_t *out_trigger, void *ws, size_t ws_bytes, idx_stream_t stream);

/* Workspace bytes for idx_pivot_topk (mode REUSE, REFINE, BLOCK or QUEST) with the
 * same dense_below; 0 for arguments idx_pivot_topk would reject. */
size_t idx_pivot_workspace_size(int T, int H, int d, int topk, int num_seqs, idx_dtype dtype, int g,
                                int c, idx_mode mode, int dense_below);

/* PIVOT grouped indexer + top-k (Reuse, Refine or block pre-filter Refine)
 * over a packed batch.  Same tensors and layouts as idx_dense_topk, plus
 *   g     group size (>= 1); groups are request-local [m*g, min((m+1)*g, n))
 *   c     candidate budget in tokens for REFINE, BLOCK and QUEST (c >= topk;
 *         BLOCK, QUEST: a multiple of 64); ignored for REUSE
 *   mode  IDX_MODE_REUSE, IDX_MODE_REFINE, IDX_MODE_BLOCK or IDX_MODE_QUEST
 *   dense_below  the guardrail (PIVOT page, Results, indexer speed: PIVOT
 *         falls back to a dense scan for short groups, so that it is never
 *         slower than the dense indexer; the page gives no threshold).  A
 *         group whose last member's prefix holds at most dense_below keys
 *         (t_last + 1 <= dense_below) is not grouped: each member takes its
 *         dense top-k, exactly as idx_dense_topk would.  Those groups are
 *         the first min(n, floor(dense_below / g) * g) tokens of a request
 *         (all n when n <= dense_below); the other groups are unchanged.
 *         0 turns it off.  REUSE and REFINE only (BLOCK, QUEST:
 *         IDX_ERR_UNSUPPORTED for dense_below > 0).  For REFINE a threshold of at most c changes
 *         no result: such a group's candidate set is its whole prefix.
 * IDX_ERR_INVALID for g < 1, dense_below < 0, an unknown mode or a c these
 * rules reject. */
idx_status idx_pivot_topk(const void *q, const void *k, const float *w, const int *cu_seqlens,
                          int num_seqs, int T, int H, int d, int topk, idx_dtype dtype, int g, int c,
                          idx_mode mode, int dense_below, int *out_idx, float *out_score, void *ws,
                          size_t ws_bytes, idx_stream_t stream);

/* Output rows [row_lo, row_hi) only (packed token rows, 0 <= row_lo <= row_hi
 * <= T): the same result as idx_dense_topk / idx_pivot_topk for those rows,
 * computed without the work of the others; the other rows of out_idx and
 * out_score are left as they are.  Every key of each request is still read
 * (a row needs its whole prefix), so q, k and w are passed whole.  Uses:
 *   - one request split across GPUs: each rank passes the ranges it owns
 *     (zig-zag chunks of equal causal work, groups whole; see the multi-GPU
 *     partition in the Python package) and writes disjoint rows;
 *   - a long prefill in row chunks with a bounded workspace: the per-row
 *     scratch covers the call's rows only, so a call whose range spans at
 *     most max_rows rows needs *_workspace_size_rows(..., max_rows) bytes.
 * PIVOT rows: a group is computed when one of its members is in the range,
 * so a range that cuts a group recomputes that group on both sides.  Same
 * errors as the full calls, plus IDX_ERR_INVALID for a bad range and
 * IDX_ERR_WORKSPACE for a workspace smaller than the size for the range's
 * length; an empty range launches nothing.  (The debug score export reads
 * the member scores of full calls only.) */
size_t idx_dense_workspace_size_rows(int T, int H, int d, int topk, int num_seqs, idx_dtype dtype,
                                     int max_rows);
size_t idx_pivot_workspace_size_rows(int T, int H, int d, int topk, int num_seqs, idx_dtype dtype, int g,
                                     int c, idx_mode mode, int dense_below, int max_rows);
idx_status idx_dense_topk_rows(const void *q, const void *k, const float *w, const int *cu_seqlens,
                               int num_seqs, int T, int H, int d, int topk, idx_dtype dtype, int row_lo,
                               int row_hi, int *out_idx, float *out_score, void *ws, size_t ws_bytes,
                               idx_stream_t stream);
idx_status idx_pivot_topk_rows(const void *q, const void *k, const float *w, const int *cu_seqlens,
                               int num_seqs, int T, int H, int d, int topk, idx_dtype dtype, int g, int c,
                               idx_mode mode, int dense_below, int row_lo, int row_hi, int *out_idx,
                               float *out_score, void *ws, size_t ws_bytes, idx_stream_t stream);

/* ------------------------------------------------------------- decode */

/* Workspace bytes for idx_decode_topk. */
size_t idx_decode_workspace_size(int B, int G, int n_max, int H, int d, int topk, int c, idx_mode mode,
                                 idx_dtype dtype);

/* One decode step of the indexer for B requests of G MTP queries each
 * (PIVOT page, Method, decode paragraph).
 *   q       [B, G, H, d]  dtype   query m of request b (position kv_len[b]-G+m)
 *   kcache  [B, n_max, d] dtype   keys of request b at rows 0 .. kv_len[b]-1
 *   kv_len  [B] int32             device; G <= kv_len[b] <= n_max (else the
 *                                 request's rows are written as all -1 and
 *                                 the status word records IDX_ERR_INVALID)
 *   w       [B, G, H] fp32
 *   mode    DENSE (each query scans its own prefix), REUSE or REFINE (the G
 *           queries are one group; c as in idx_pivot_topk)
 *   out_idx [B, G, topk] int32, out_score [B, G, topk] fp32 or NULL */
idx_status idx_decode_topk(const void *q, const void *kcache, const int *kv_len, const float *w,
                           int B, int G, int n_max, int H, int d, int topk, int c, idx_mode mode,
                           idx_dtype dtype, int *out_idx, float *out_score, void *ws,
                           size_t ws_bytes, idx_stream_t stream);

/* idx_decode_topk over a paged key cache (the block-table layout of
 * paged-attention serving engines; the pages describe a contiguous cache
 * and leave its storage open).  Same queries, weights, modes, outputs and
 * status as idx_decode_topk; only the key addressing differs:
 *   kpool        [num_pages, page, d] dtype   device pages of keys
 *   block_table  [B, max_pages] int32          device; position s of request
 *                b is row s % page of page block_table[b, s / page].
 *                Entries covering only positions >= kv_len[b] may hold any
 *                value and never change a result.  An entry outside
 *                [0, num_pages) is read as page 0.
 *   page         keys per page: a divisor of 128 (1, 2, 4, ..., 128) or a
 *                multiple of 128, else IDX_ERR_UNSUPPORTED.  Pages of 8 keys
 *                or more use the tensor-core scan; smaller ones the CUDA-core
 *                scan.
 *   kv_len[b] <= max_pages * page <= 2^20; num_pages * page < 2^31.
 * Workspace: idx_decode_workspace_size(B, G, max_pages * page, ...).
 * Returns IDX_ERR_INVALID for a NULL block_table or a non-positive size. */
idx_status idx_decode_paged_topk(const void *q, const void *kpool, const int *block_table,
                                 const int *kv_len, const float *w, int B, int G, int max_pages,
                                 int page, long long num_pages, int H, int d, int topk, int c,
                                 idx_mode mode, idx_dtype dtype, int *out_idx, float *out_score,
                                 void *ws, size_t ws_bytes, idx_stream_t stream);

/* --------------------------------------------- decode block pre-filter */

/* Decode with the block pre-filter as the candidate generator (page
 * "Uncertainty-gated selection for block-sparse attention", Sec. 3.1, step
 * 1: a block of 64 keys is summarised by its mean key, Eq. (1), or by its
 * per-dimension key minimum and maximum, Eq. (2), after Quest; page "Not All Tokens
 * Deserve Equal Resolution", abstract: chunk summaries are scored first, the
 * tokens of the chosen chunks are then scored exactly).  The decode group of
 * request b (its G queries, PIVOT page, Method, decode paragraph) is one
 * group: its proxy (mean query, mean w) scores the complete blocks below
 * kv_len[b] -- rule 0: the indexer score of the proxy against the block's
 * mean key; rule 1 (Quest): sum_h wbar_h * max(0, sum_i max(qbar_hi * kmax_i,
 * qbar_hi * kmin_i)), the indexer's weighted ReLU of each head's upper
 * bound of q . k over the block -- and the c / 64 best blocks (one fewer when
 * kv_len[b] ends inside a block, whose partial block is then always taken),
 * ties to the lower block, give the candidate positions; each query
 * re-scores the candidates inside its own prefix and keeps its top-k.  This
 * is the prefill block mode (idx_pivot_topk with IDX_MODE_BLOCK) applied to
 * the decode group.
 *
 * The block summaries are a cache the caller keeps beside the key cache,
 * so a decode step reads them (n / 64 rows per request) and the chosen
 * blocks' keys instead of the whole cache:
 *   rule 0: kbar [B, n_max / 64, d] dtype   row b * (n_max / 64) + j = the
 *         mean of rows 64 j .. 64 j + 63 of request b's cache: fp32 sum in
 *         row order, one IEEE fp32 division by 64, round-to-nearest-even to
 *         bf16 for bf16 keys (the same rule as the group proxy);
 *         idx_decode_block_means writes it;
 *   rule 1: kminmax [B, n_max / 64, 2, d] dtype   for block j of request b,
 *         the per-dimension minimum of its 64 rows, then their maximum;
 *         idx_decode_block_minmax writes it.
 * Blocks at or past kv_len[b] / 64 are never read. */

/* kbar rows of the blocks j >= first_block (j < n_max / 64) of every request
 * from kcache [B, n_max, d]; first_block = 0 fills all of it, and after keys
 * are appended, the first newly completed block updates only the rest.
 * n_max must be a positive multiple of 64 (else IDX_ERR_INVALID); d % 8 ==
 * 0.  Asynchronous on `stream`; kbar is caller-owned device memory. */
idx_status idx_decode_block_means(const void *kcache, int B, int n_max, int d, idx_dtype dtype,
                                  int first_block, void *kbar, idx_stream_t stream);

/* The same for rule 1: kminmax rows of blocks j >= first_block (exact: every
 * value is a key element). */
idx_status idx_decode_block_minmax(const void *kcache, int B, int n_max, int d, idx_dtype dtype,
                                   int first_block, void *kminmax, idx_stream_t stream);

/* Workspace bytes for idx_decode_block_topk (0 for arguments it rejects). */
size_t idx_decode_block_workspace_size(int B, int G, int n_max, int H, int d, int topk, int c, int rule,
                                       idx_dtype dtype);

/* One decode step with the block pre-filter.  q, kcache, kv_len, w, out_idx,
 * out_score and the status word as in idx_decode_topk; ksum = kbar (rule 0)
 * or kminmax (rule 1) as above.
 *   c  candidate budget in tokens: a multiple of 64, >= 64 and >= topk
 *   n_max a multiple of 64
 * Argument errors (a rule other than 0 or 1 included) return
 * IDX_ERR_INVALID before any launch; G > 8, n_max > 2^20, a shape neither
 * score path serves, or rule 1 with H * d * 8 bytes above the shared memory
 * of one block return IDX_ERR_UNSUPPORTED. */
idx_status idx_decode_block_topk(const void *q, const void *kcache, const void *ksum, int rule,
                                 const int *kv_len, const float *w, int B, int G, int n_max, int H, int d,
                                 int topk, int c, idx_dtype dtype, int *out_idx, float *out_score, void *ws,
                                 size_t ws_bytes, idx_stream_t stream);

/* ----------------------------------------------- no-allocation variant */

/* The pages have no counterpart of this entry point; it exists for callers
 * that cannot allocate device memory, such as a plugin inside another
 * runtime that owns all device memory and hands out no workspace, or a
 * serving loop that must not allocate once decoding runs.
 *
 * Same result as idx_decode_topk with mode IDX_MODE_DENSE (c unused), same
 * tensors and layouts, but no workspace argument: the scratch is a fixed
 * 32 MiB device array inside the library, reserved on every GPU that loads
 * the library until the process exits.  Nothing is allocated by the call.
 *   - Limit: 256 + 4*B*G*n_max bytes must fit in 32 MiB (B*G*n_max <=
 *     8388544, e.g. 32 requests x 2 queries x 131071 tokens); larger calls
 *     return IDX_ERR_UNSUPPORTED with a message on stderr and launch nothing.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *     The address is kept per device together with the id of the context it
 *     came from, and looked up again when the current context differs (after
 *     cudaDeviceReset the module, and with it the array, is loaded anew).
 *   - Every call uses the same array, which keeps the last call's contents
 *     (the status word is cleared at the start of each call): calls whose
 *     kernels overlap on the GPU -- other streams, other host threads --
 *     race and corrupt each other's results.  Order them on one stream.
 *   - Arguments idx_decode_topk rejects are rejected with the same code.
 *   - The device status word lives in the shared array; read it with
 *     idx_decode_noalloc_status() after the call (requests whose kv_len is
 *     out of range come back as rows of -1 and IDX_ERR_INVALID there; a
 *     bounded wait that ran out gives IDX_ERR_TIMEOUT and invalid rows). */
idx_status idx_decode_topk_noalloc(const void *q, const void *kcache, const int *kv_len, const float *w,
                                   int B, int G, int n_max, int H, int d, int topk, idx_dtype dtype,
                                   int *out_idx, float *out_score, idx_stream_t stream);

/* Device status of the last idx_decode_topk_noalloc call on the current
 * device, as idx_device_status() reports it for a workspace: synchronises
 * `stream` (the stream of that call), then reads the status word out of the
 * library's fixed array.  Allocates nothing. */
idx_status idx_decode_noalloc_status(idx_stream_t stream);

/* --------------------------------------------- token-sparse attention */

/* Workspace bytes for idx_sparse_attn (its status word). */
size_t idx_sparse_attn_workspace_size(void);

/* Attention of each query row restricted to its selected positions: the
 * consumer of the top-k sets (PIVOT page, introduction: the selected set
 * feeds sparse MLA attention).  The pages give no formula; the reading is
 * softmax attention over the listed keys in the absorbed-MLA form of the
 * production models that page names: one latent row per key is the key
 * (all Dqk dims) and its first Dv dims the value, shared by all heads.
 *   z_j      = scale * q[r,h,:] . kv[cu_kv[b] + idx[r,j], :]   (idx[r,j] >= 0)
 *   out[r,h] = sum_j softmax_j(z) * kv[cu_kv[b] + idx[r,j], :Dv]
 *   lse[r,h] = log sum_j exp(z_j)   (natural log; -inf for a row with no entry)
 * where b is the request of query row r (cu_q[b] <= r < cu_q[b+1]).
 *   q       [R, H, Dqk] bf16        query rows
 *   kv      [Nkv, Dqk] bf16         latent rows of all requests
 *   idx     [R, topk] int32         positions inside the row's request; -1 =
 *                                   no entry (anywhere in the row); an entry
 *                                   listed twice counts twice.  The output of
 *                                   idx_dense_topk / idx_pivot_topk (cu_q =
 *                                   cu_kv = cu_seqlens) or idx_decode_topk
 *                                   (cu_q = [0, G, 2G, ..], cu_kv = [0, n_max,
 *                                   2 n_max, ..]) fits as is.
 *   cu_q, cu_kv [num_seqs+1] int32  device request boundaries
 *   out     [R, H, Dv] bf16; lse [R, H] fp32 or NULL
 * Supported: bf16, Dqk = 576, Dv = 512, 1 <= H <= 128 (tensor cores);
 * other shapes return IDX_ERR_UNSUPPORTED.  Positions >= the request's kv
 * length and malformed boundaries are skipped and flagged as
 * IDX_ERR_INVALID in the device status word of ws. */
idx_status idx_sparse_attn(const void *q, const void *kv, const int *idx, const int *cu_q,
                           const int *cu_kv, int num_seqs, int R, long long Nkv, int H, int Dqk,
                           int Dv, int topk, float scale, idx_dtype dtype, void *out, float *lse,
                           void *ws, size_t ws_bytes, idx_stream_t stream);

/* ------------------------------------------------------ status, debug */

/* Synchronises `stream`, returns the device status recorded in `ws` by the
 * last call that used it (IDX_OK, IDX_ERR_TIMEOUT, IDX_ERR_OVERFLOW or
 * IDX_ERR_INVALID), or IDX_ERR_CUDA if the synchronisation itself failed. */
idx_status idx_device_status(const void *ws, idx_stream_t stream);

/* A static, human-readable name of a status code. */
const char *idx_status_string(idx_status s);

/* Test hook: the fp32 scores the selection of the preceding call used, for
 * a list of scored rows, written as out[i * ld + s] for s = 0 .. bound(i)
 * (other entries untouched).  `stage` selects what is exported:
 *   0: dense query rows (rows[] = global query rows; same arguments as
 *      idx_dense_topk),
 *   1: PIVOT proxy rows (rows[] = proxy indices in request order; same
 *      arguments as idx_pivot_topk),
 *   2: PIVOT Refine member re-scores over the candidate set (rows[] = global
 *      member rows; out[i * ld + j] is the score of candidate j of the
 *      member's group, j < c; requires that idx_pivot_topk ran on `ws`),
 *   3: block mode proxy rows against the block mean keys (rows[] = proxy
 *      indices; out[i * ld + j] for blocks j = 0 .. (t_last+1)/64 - 1),
 *   4: like 2 for a preceding idx_pivot_topk call in IDX_MODE_BLOCK; the
 *      candidate j of a group is slot j/64, position j%64 of that slot (the
 *      selected blocks in ascending order, -1 slots, the partial block in
 *      the last slot).
 * rows is a DEVICE int32 array of DISTINCT rows (a row listed twice gets one
 * of its output rows written).  The scores come from the same kernels and
 * arithmetic as the selection, so re-selecting on them reproduces out_idx. */
idx_status idx_debug_scores(int stage, const void *q, const void *k, const float *w,
                            const int *cu_seqlens, int num_seqs, int T, int H, int d, idx_dtype dtype,
                            int g, int c, int topk, const int *rows, int nrows, float *out, long long ld,
                            void *ws, size_t ws_bytes, idx_stream_t stream);

/* Test hook for decode: stage 0 = dense query scores (row i = b*G+m, over
 * s < kv_len[b]-G+m+1), stage 1 = proxy scores of request b (row i = b),
 * stage 2 = Refine member re-scores over C (row i = b*G+m, j < c). */
idx_status idx_debug_decode_scores(int stage, const void *q, const void *kcache, const int *kv_len,
                                   const float *w, int B, int G, int n_max, int H, int d, int topk,
                                   int c, idx_mode mode, idx_dtype dtype, float *out, long long ld,
                                   void *ws, size_t ws_bytes, idx_stream_t stream);

/* Test hook for failure detection: launches one thread that waits, with the
 * bounded wait every tensor-core kernel uses, on a barrier nothing completes.
 * After limit_ms milliseconds (1..10000) the wait gives up and records
 * IDX_ERR_TIMEOUT in the status word of `ws` (at least 4 bytes); read it
 * with idx_device_status().  Nothing faults and the context stays usable. */
idx_status idx_debug_wait_probe(void *ws, unsigned limit_ms, idx_stream_t stream);

/* Per-kernel device timing.  idx_trace_enable(1) clears the record and
 * starts bracketing every kernel launch of the library with two CUDA events
 * on its stream; idx_trace_enable(0) stops (the record is kept).
 * idx_trace_report() waits for the recorded events and writes one line per
 * kernel, "<phase>/<kernel> <launches> <total milliseconds>", into buf
 * (NUL-terminated, truncated to len); it returns the number of launches
 * recorded, or -1 if an event could not be read.  Host-side state shared by
 * all threads; meant for benchmarks, off by default. */
int idx_trace_enable(int on);
long long idx_trace_report(char *buf, size_t len);

/* Which score kernel serves a shape: 1 = tcgen05 tensor-core kernel,
 * 0 = SIMT kernel.  (bf16 with H = 64 and d = 128 uses the tensor cores.) */
int idx_uses_tensor_cores(int H, int d, idx_dtype dtype);

#ifdef __cplusplus
}
#endif

#endif /* IDX_H */
