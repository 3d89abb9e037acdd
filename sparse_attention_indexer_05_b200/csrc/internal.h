// internal.h -- launch-side declarations shared by the libidx sources.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace idx {

constexpr int RB = 8;           // scored rows per row block (score kernels)
constexpr int KT = 128;         // keys per key tile
constexpr int kMaxLen = 1 << 20;  // longest supported request / cache

// Plan area (int32 words at the start of a prefill workspace plan region):
//   [0] valid flag (1 = cu_seqlens passed the device checks)
//   [1] number of row blocks scheduled (those with a member in [row_lo, row_hi))
//   [2] number of scored rows
//   [3] work counter (persistent score kernels)
//   [4] row_lo  [5] row_hi: the output rows (packed token rows) of the call
//   [6] p_lo    [7] p_hi: the scored rows with a member in [row_lo, row_hi);
//       per-row scratch (candidate buffers, counts, floors, candidate sets,
//       packed keys) is indexed from p_lo
//   [8] m_lo: the first member of scored row p_lo; member scores (every
//       member of the call's groups) are indexed from it
//   [9 .. 9+S]          rp[b]: first scored row of request b (S = num_seqs)
//   [10+S .. 10+2S]     bp[b]: first row block of request b
//   [11+2S .. +maxblk)  order: scheduled row blocks, longest key range first
//   then (maxtiles+1)   per-tile-count histogram (plan scratch)
struct PlanLayout {
    int S, maxblk, maxtiles;
    __host__ __device__ size_t words() const {
        return (size_t)11 + 2 * (size_t)S + (size_t)maxblk + (size_t)maxtiles + 1;
    }
    __host__ __device__ int rp() const { return 9; }
    __host__ __device__ int bp() const { return 10 + S; }
    __host__ __device__ int order() const { return 11 + 2 * S; }
    __host__ __device__ int hist() const { return 11 + 2 * S + maxblk; }
};

enum Sink { SINK_FILTER = 0, SINK_SPILL = 1 };

// A prefill score pass: rows of `q` (queries, or PIVOT proxies when g > 1)
// against the keys of their request, streamed into a sink.
// block pre-filter: keys summarised per complete block of kBlockN tokens
constexpr int kBlockShift = 6;
constexpr int kBlockN = 1 << kBlockShift;

struct ScoreArgs {
    const void *q;       // [R, H, d] scored rows
    const void *k;       // [T, d] keys (kshift = 0), or block mean keys (kshift > 0)
    const float *w;      // [R, H]
    const int *cu;       // cu_seqlens [S+1] (device)
    int S, T, H, d, g;   // g = 1: row i of request b is query i; g > 1: proxy i
    int db;              // guardrail: short groups scored member by member (plan.cuh)
    long long R;         // rows allocated in q / w
    // kshift > 0: keys are the complete 2^kshift-token blocks of each request,
    // block i of request b at key row (cu[b] >> kshift) + i; a row whose token
    // bound is t sees blocks 0 .. ((t + 1) >> kshift) - 1
    int kshift;
    const int *plan;     // plan area
    PlanLayout pl;
    int sink;
    // SINK_FILTER: candidate buffers [R, cap] and counts [R]
    unsigned long long *buf;
    unsigned cap, ksel;
    unsigned ksel_dense;  // guardrail: rows of short-group members keep their top-k only
    unsigned *cnt;
    unsigned *floor_out;  // per row: keys with a lower ord cannot be selected
    // SINK_SPILL: out[slot * ld + s] for rows with slot_of_row[row] >= 0
    float *spill;
    long long ld;
    const int *slot_of_row;
    unsigned *status;
};

// decode score pass (one row block = the G queries of one request, or its proxy)
struct DecodeArgs {
    const void *q;       // [B, Gq, H, d] rows scored (Gq = G queries, or 1 proxy)
    const void *kc;      // [B, n_max, d]
    const float *w;      // [B, Gq, H]
    const int *kv_len;   // [B]
    int B, G, Gq, n_max, H, d;
    int chunk_tiles;     // key tiles per work item
    float *spill;        // [B*Gq, n_max]
    unsigned *status;
    unsigned *work;
    // paged cache (bt != NULL): kc is [num_pages, page, d]; position s of
    // request b sits at row bt[b * max_pages + s / page] * page + s % page
    const int *bt;
    int page, max_pages;
    long long num_pages;
};

// Refine re-score pass: member rows against the gathered candidate keys.
struct GatherArgs {
    const void *q;       // [rows, H, d] member queries
    const void *k;       // [*, d] keys (prefill: packed keys; decode: cache)
    const float *w;      // [rows, H]
    const int *cand;     // [P, c] candidate positions (ascending, -1 padded)
    int c, H, d;
    int nitems;          // work items (one per group, members <= RB)
    // mapping of a work item -> (first member row, members, candidate row, key base)
    int mode;            // 0: prefill (cu, g, plan rp of proxies), 1: decode (B, G, n_max)
    const int *cu;
    int S, g, db;
    int cu_T;            // prefill: rows of q and k (total tokens)
    const int *plan;
    PlanLayout pl;
    int G, n_max;
    const int *kv_len;
    float *out;          // [rows, c] member scores (prefill: rows from the call's first member)
    void *ckeys;         // [groups, c_pad, d] packed candidate keys (tensor-core path; prefill: groups
                         // from the call's first scored row)
    long long ckey_groups;  // groups the packed-key area holds
    int c_pad;           // c rounded up to a multiple of 128
    unsigned *status;
    const int *bt;       // decode: paged cache, as in DecodeArgs
    int page, max_pages;
    long long num_pages;
};

// Row of the key cache holding position s of request b: contiguous
// [B, n_max, d] when bt is NULL, else paged through the block table (an
// entry outside [0, num_pages) reads row 0; positions past the request are
// masked by the callers).
__host__ __device__ inline long long cache_row(const int *bt, int page, int max_pages, long long num_pages,
                                               long long n_max, int b, int s) {
    if (!bt) return (long long)b * n_max + s;
    const int j = s / page;
    long long pg = j < max_pages ? bt[(long long)b * max_pages + j] : 0;
    if (pg < 0 || pg >= num_pages) pg = 0;
    return pg * page + s % page;
}

// select pass descriptors
enum SelKind {
    SEL_DENSE_CAND = 0,     // out row = query row; candidates of that row
    SEL_REUSE_CAND = 1,     // out row = member; candidates of its group's proxy row
    SEL_PROXY_TO_C = 2,     // out = candidate set of proxy row (k = c), positions only
    SEL_MEMBER_SCORES = 3,  // out row = member; scores over its group's candidate set
    SEL_DEC_DENSE = 4,      // decode: spill row (b, m)
    SEL_DEC_REUSE = 5,      // decode: proxy spill row b restricted to member m
    SEL_DEC_PROXY_TO_C = 6, // decode: candidate set of request b
    SEL_DEC_MEMBER = 7,     // decode: member scores over the candidate set
    SEL_PROXY_TO_BLOCKS = 8, // block pre-filter: complete blocks of a proxy row (k = c / kBlockN, one
                             // fewer when the row's prefix ends inside a block), block indices only
    SEL_DEC_PROXY_TO_BLOCKS = 9, // decode block mode: the same over request b's block-score spill row
    SEL_PROXY_SPILL_TO_BLOCKS = 10 // prefill block mode, Quest rule: the same over a proxy's block-score
                                   // spill row (scores, ld), into cand = the selected blocks [R, k]
};

struct SelectArgs {
    int kind;
    int nrows;               // CTAs / output rows
    int k;                   // entries selected per row
    int *out_idx;            // [nrows, k]
    float *out_score;        // [nrows, k] or NULL
    // prefill context
    const int *cu;
    int S, g, db;
    const int *plan;
    PlanLayout pl;
    const unsigned long long *buf;
    unsigned cap;
    const unsigned *cnt;
    const unsigned *floor;   // per candidate row (NULL: no floor)
    int stage_cap;           // set by launch_select
    // score-row sources
    const float *scores;     // spill or member scores
    long long ld;
    const int *cand;         // candidate sets [P, c]
    int c;
    // decode context
    const int *kv_len;
    int G, n_max;
    int bitmap_words;        // shared bitmap capacity (words)
    unsigned *status;
    // dense candidate rows only: the cutoff margin of the top-kmargin inside
    // the row's top-k (adaptive budget), per output row; kmargin = 0: none
    int kmargin;
    float *m_sigma;
    unsigned *m_vk;
    int *m_need;
    // SEL_MEMBER_SCORES in select_fast_kernel: the member rows are selected by
    // member_select_kernel; only the guardrail's own rows are left here
    int skip_members;
};

// adaptive.cu: the adaptive budget from the cutoff margin over the rows of a
// top-(rho k) result (in place).
constexpr int kAdaptiveMaxWidth = 8192;  // rho * k: the final select's staging room stays in shared memory
struct AdaptiveArgs {
    long long T;
    int k, width;             // width = rho * k
    int *idx;                 // [T, width] ascending positions, -1 padded (in/out)
    float *score;             // [T, width] their scores (in/out)
    float *sigma;             // [T] cutoff margins (out)
    unsigned *vk;             // [T] ord of s_(k-1) (scratch)
    int *need;                // [T] ties of s_(k-1) the top-k keeps (scratch)
    unsigned char *trigger;   // [T] or null (out)
    unsigned *tau;            // [2] {tau defined, ord of tau} (scratch)
    double q;                 // trigger quantile
    unsigned *status;
};

// ---- tracing (trace.cu): a TraceScope around a launch records two events
// on its stream while tracing is enabled; TracePhase names the entry-point
// phase that prefixes the kernel names in the report.
struct TracePhase {
    explicit TracePhase(const char *p);
    ~TracePhase();
    const char *prev;
};
struct TraceScope {
    TraceScope(const char *name, cudaStream_t st);
    ~TraceScope();
    cudaStream_t st_;
    int idx_;
};

// ---- launchers (each returns cudaSuccess or the launch error)
cudaError_t launch_plan(const int *cu, int S, int T, int g, int db, int row_lo, int row_hi, int *plan,
                        const PlanLayout &pl, unsigned *status, cudaStream_t st);
cudaError_t launch_score_simt(const ScoreArgs &a, int dtype, cudaStream_t st);
cudaError_t launch_score_tc(const ScoreArgs &a, cudaStream_t st);
cudaError_t launch_decode_simt(const DecodeArgs &a, int dtype, cudaStream_t st);
cudaError_t launch_decode_tc(const DecodeArgs &a, cudaStream_t st);
cudaError_t launch_gather_simt(const GatherArgs &a, int dtype, cudaStream_t st);
cudaError_t launch_gather_tc(const GatherArgs &a, cudaStream_t st);
cudaError_t launch_select(const SelectArgs &a, cudaStream_t st);
// dec_select.cu: the decode score rows (SEL_DEC_DENSE, _REUSE, _PROXY_TO_C),
// one cluster of CTAs per row
bool dec_select_kind(int kind);
cudaError_t launch_dec_select(const SelectArgs &a, cudaStream_t st);
// member_select.cu: Refine member rows (SEL_MEMBER_SCORES, SEL_DEC_MEMBER)
// whose candidate lists fit in shared memory, one 128-thread CTA per row
bool member_select_fits(const SelectArgs &a);
cudaError_t launch_member_select(const SelectArgs &a, cudaStream_t st);
cudaError_t launch_adaptive(const AdaptiveArgs &a, cudaStream_t st);
cudaError_t launch_proxy(const void *q, const float *w, const int *cu, int S, int T, int H, int d,
                         int g, int db, int dtype, const int *plan, const PlanLayout &pl, void *qbar,
                         float *wbar, int max_proxies, cudaStream_t st);
// token-sparse attention over selected positions (absorbed-MLA shapes)
struct SparseAttnArgs {
    const void *q;        // [R, H, 576] bf16
    const void *kv;       // [Nkv, 576] bf16: key = all dims, value = dims [0, 512)
    const int *idx;       // [R, topk] positions inside the row's request, -1 = none
    const int *cu_q;      // [S+1] request boundaries over query rows
    const int *cu_kv;     // [S+1] request boundaries over kv rows
    int S, R, H, topk;
    long long Nkv;
    float scale;          // logit = scale * q . k
    void *out;            // [R, H, 512] bf16
    float *lse;           // [R, H] natural-log softmax denominators, or NULL
    unsigned *status;
};
bool attn_tc_supported(int H, int Dqk, int Dv, int dtype);
cudaError_t launch_sparse_attn_tc(const SparseAttnArgs &a, cudaStream_t st);

// block pre-filter: mean keys of the complete blocks of every request
cudaError_t launch_block_means(const void *k, const int *cu, int S, int T, int d, int dtype, void *kb,
                               cudaStream_t st);
// block pre-filter: candidate positions [R, c] from the selected blocks [R, c / kBlockN]
// plus the partial block that holds each proxy's last member
cudaError_t launch_block_expand(const int *cu, int S, int g, const int *plan, const PlanLayout &pl,
                                const int *cblk, int *cand, int c, int R, cudaStream_t st);
cudaError_t launch_decode_proxy(const void *q, const float *w, int B, int G, int H, int d, int dtype,
                                void *qbar, float *wbar, cudaStream_t st);
// decode block mode: block means of a cache [B, n_max, d] (blocks >= first_block),
// the complete blocks per request, and candidate positions from the selected blocks
cudaError_t launch_decode_block_means(const void *kc, int B, int n_max, int d, int dtype, int first_block,
                                      void *kbar, cudaStream_t st);
cudaError_t launch_decode_block_len(const int *kv_len, int B, int G, int n_max, int *nlen, cudaStream_t st);
// decode block mode with the Quest bound: per-block key minimum and maximum
// [B, n_max / 64, 2, d], and the proxy's bound scores of the complete blocks
cudaError_t launch_decode_block_minmax(const void *kc, int B, int n_max, int d, int dtype, int first_block,
                                       void *kq, cudaStream_t st);
size_t quest_scan_smem(int H, int d);
// prefill block mode with the Quest bound: per-block key min/max of every
// request ([T / 64, 2, d], placed as the block means), and the proxy rows'
// bound scores of their complete blocks into spill rows (stride ld)
cudaError_t launch_block_minmax(const void *k, const int *cu, int S, int T, int d, int dtype, void *kq,
                                cudaStream_t st);
cudaError_t launch_prefill_quest_scan(const void *qbar, const float *wbar, const void *kq, const int *cu, int S,
                                      int g, const int *plan, const PlanLayout &pl, int R, int nbmax, int H, int d,
                                      int dtype, float *spill, long long ld, cudaStream_t st);
cudaError_t launch_decode_quest_scan(const void *qbar, const float *wbar, const void *kq, const int *nlen, int B,
                                     int nb, int H, int d, int dtype, float *spill, cudaStream_t st);
cudaError_t launch_decode_block_expand(const int *kv_len, int B, int G, int n_max, const int *cblk, int *cand,
                                       int c, cudaStream_t st);
size_t simt_smem_bytes(int H, int d, int dtype);
bool tc_supported(int H, int d, int dtype);
bool tc_decode_supported(int H, int d, int dtype, int rows_per_request);
bool tc_gather_supported(int H, int d, int dtype, int group, int c);

}  // namespace idx
