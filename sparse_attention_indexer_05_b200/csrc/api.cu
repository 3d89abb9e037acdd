// api.cu -- the C ABI of libidx (include/idx.h): argument checks, workspace
// layout and the launch sequence of each entry point.  No entry point
// allocates device memory; every call is asynchronous on its stream.
#include <math.h>
#include <string.h>

#include "../../include/idx.h"
#include "common.cuh"
#include "internal.h"

using namespace idx;

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kMaxSmem = 232448;  // opt-in shared memory per block on sm_100

size_t up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

// Candidate buffer capacity per scored row for a streaming top-ksel over
// rows of at most n keys.  A random key order appends about
// ksel * (1 + ln(n / ksel)) keys; 1.5x that leaves room for the histogram's
// coarse threshold.  At least 2*ksel + 1024 so that a compaction (cut to
// ksel) always frees more than the appends that can arrive between two
// upkeeps (8 tiles of 128 keys); never more than n, which cannot overflow.
unsigned cap_for(long long ksel, long long n) {
    if (n < 1) n = 1;
    const long long nn = (long long)up((size_t)n, 32);
    if (n <= ksel) return (unsigned)nn;
    const double est = 1.5 * (double)ksel * (1.0 + log((double)n / (double)ksel));
    long long cap = (long long)up((size_t)ceil(est), 256);
    if (cap < 2 * ksel + 1024) cap = 2 * ksel + 1024;
    if (cap > nn) cap = nn;
    return (unsigned)cap;
}

struct Carve {
    size_t off = 0;
    size_t take(size_t bytes) {
        const size_t o = off;
        off = up(off + bytes);
        return o;
    }
};

size_t esize(idx_dtype dt) { return dt == IDX_F32 ? 4 : 2; }

int c_pad_of(int c) { return (c + KT - 1) / KT * KT; }

long long nbound(int T) { return T < kMaxLen ? T : kMaxLen; }

struct PrefillWs {
    PlanLayout pl;
    long long R;          // scored rows (queries or proxies, upper bound)
    long long Rb;         // scored rows of one call's output rows (per-row scratch)
    long long Mb;         // members of one call's groups (member scores)
    unsigned cap, ksel;
    size_t status, plan, slot, qbar, wbar, cnt, floor, buf, cand, msc, ckeys, kblk, cblk, qspill, total;
    long long nbmax;      // Quest: blocks of the longest request (spill row stride)
};

// the block pre-filter, blocks ranked by their mean key or by the Quest bound
bool blocky(idx_mode m) { return m == IDX_MODE_BLOCK || m == IDX_MODE_QUEST; }
bool refines(idx_mode m) { return m == IDX_MODE_REFINE || blocky(m); }

long long block_rows(int T) { return (T >> kBlockShift) > 0 ? (T >> kBlockShift) : 1; }

// Workspace of a prefill call whose output rows span at most max_rows rows
// (max_rows <= 0 or >= T: any call).  The plan, proxies and the debug slot
// map cover the whole batch; the per-row scratch only the call's rows.
PrefillWs prefill_ws(int T, int H, int d, int topk, int S, idx_dtype dt, int g, int c, idx_mode mode,
                     int db = 0, long long max_rows = 0) {
    PrefillWs L{};
    const bool pivot = mode != IDX_MODE_DENSE;
    const long long m = (max_rows <= 0 || max_rows >= T) ? T : max_rows;
    L.R = pivot ? ((long long)T + (long long)S * (g - 1)) / g : T;
    long long extra = 0;
    if (pivot && db > 0 && g > 1) {
        // members of short groups are scored rows of their own: at most
        // min(n, db) per request
        extra = (long long)S * db < T ? (long long)S * db : T;
        L.R = L.R + extra < T ? L.R + extra : T;
    }
    L.Rb = L.R;
    L.Mb = T;
    if (m < T) {
        // a run of m output rows meets at most m / g + 2 groups per request it
        // touches (partial groups at both ends), plus the short groups'
        // members; those groups hold at most m + 2 (g - 1) members per request
        long long rb = pivot ? m / g + 2LL * S + (extra < m ? extra : m) : m;
        if (rb > m) rb = m;
        L.Rb = rb < L.R ? rb : L.R;
        const long long mb = pivot ? m + 2LL * (g - 1) * S : m;
        L.Mb = mb < T ? mb : T;
    }
    L.pl.S = S;
    L.pl.maxblk = (int)((L.R + RB - 1) / RB + S);
    L.pl.maxtiles = (int)(nbound(T) / KT + 1);
    L.ksel = mode == IDX_MODE_REUSE    ? (unsigned)(topk + g - 1)
             : mode == IDX_MODE_REFINE ? (unsigned)c
             : blocky(mode)            ? (unsigned)(c >> kBlockShift)
                                       : (unsigned)topk;
    L.cap = blocky(mode) ? cap_for(L.ksel, (nbound(T) >> kBlockShift) + 1) : cap_for(L.ksel, nbound(T));
    L.nbmax = (nbound(T) >> kBlockShift) + 1;
    Carve cv;
    L.status = cv.take(16);
    L.plan = cv.take(L.pl.words() * 4);
    L.slot = cv.take((size_t)(L.R > T ? L.R : T) * 4);
    L.qbar = pivot ? cv.take((size_t)L.R * H * d * esize(dt)) : 0;
    L.wbar = pivot ? cv.take((size_t)L.R * H * 4) : 0;
    L.cnt = cv.take((size_t)L.Rb * 4);
    L.floor = cv.take((size_t)L.Rb * 4);
    L.buf = cv.take((size_t)L.Rb * L.cap * 8);
    L.cand = refines(mode) ? cv.take((size_t)L.Rb * c * 4) : 0;
    L.msc = refines(mode) ? cv.take((size_t)L.Mb * c * 4) : 0;
    L.ckeys = (refines(mode) && tc_gather_supported(H, d, (int)dt, g, c))
                  ? cv.take((size_t)L.Rb * c_pad_of(c) * d * esize(dt))
                  : 0;
    // block means [T / 64, d], or the Quest rule's per-block min and max [T / 64, 2, d]
    L.kblk = blocky(mode) ? cv.take((size_t)block_rows(T) * d * esize(dt) * (mode == IDX_MODE_QUEST ? 2 : 1)) : 0;
    L.cblk = blocky(mode) ? cv.take((size_t)L.Rb * (c >> kBlockShift) * 4) : 0;
    // Quest: the proxies' block scores, one row of nbmax per scored proxy
    L.qspill = mode == IDX_MODE_QUEST ? cv.take((size_t)L.Rb * L.nbmax * 4) : 0;
    L.total = cv.off;
    return L;
}

struct AdaptiveWs {
    PrefillWs P;   // the dense top-(rho k) pass
    size_t score, sigma, vk, need, tau, total;
};

AdaptiveWs adaptive_ws(int T, int H, int d, int topk, int rho, int S, idx_dtype dt) {
    AdaptiveWs L{};
    const int width = topk * rho;
    L.P = prefill_ws(T, H, d, width, S, dt, 1, width, IDX_MODE_DENSE);
    Carve cv;
    cv.off = L.P.total;
    L.score = cv.take((size_t)T * width * 4);
    L.sigma = cv.take((size_t)T * 4);
    L.vk = cv.take((size_t)T * 4);
    L.need = cv.take((size_t)T * 4);
    L.tau = cv.take(16);
    L.total = cv.off;
    return L;
}

struct DecodeWs {
    size_t status, qbar, wbar, spill, cand, msc, ckeys, nlen, cblk, total;
};

// mode BLOCK: the decode block pre-filter (the proxy scans block means, then
// the members re-score the chosen blocks' keys as in Refine)
DecodeWs decode_ws(int B, int G, int n_max, int H, int d, int c, idx_mode mode, idx_dtype dt) {
    DecodeWs L{};
    Carve cv;
    const bool blocks = mode == IDX_MODE_BLOCK, sets = mode == IDX_MODE_REFINE || blocks;
    const int rows = mode == IDX_MODE_DENSE ? B * G : B;
    L.status = cv.take(16);
    L.qbar = mode != IDX_MODE_DENSE ? cv.take((size_t)B * H * d * esize(dt)) : 0;
    L.wbar = mode != IDX_MODE_DENSE ? cv.take((size_t)B * H * 4) : 0;
    L.spill = cv.take((size_t)rows * (blocks ? n_max >> kBlockShift : n_max) * 4);
    L.cand = sets ? cv.take((size_t)B * c * 4) : 0;
    L.msc = sets ? cv.take((size_t)B * G * c * 4) : 0;
    L.ckeys = (sets && tc_gather_supported(H, d, (int)dt, G, c)) ? cv.take((size_t)B * c_pad_of(c) * d * esize(dt))
                                                                 : 0;
    L.nlen = blocks ? cv.take((size_t)B * 4) : 0;
    L.cblk = blocks ? cv.take((size_t)B * (c >> kBlockShift) * 4) : 0;
    L.total = cv.off;
    return L;
}

bool shape_ok(int H, int d, idx_dtype dt) {
    if (H < 1 || d < 8 || d % 8 != 0 || (dt != IDX_BF16 && dt != IDX_F32)) return false;
    return true;
}

bool path_ok(int H, int d, idx_dtype dt) {
    return tc_supported(H, d, (int)dt) || simt_smem_bytes(H, d, (int)dt) <= kMaxSmem;
}

idx_status cuda_st(cudaError_t e) { return e == cudaSuccess ? IDX_OK : IDX_ERR_CUDA; }

#define TRY_CUDA(x)                                  \
    do {                                             \
        cudaError_t e_ = (x);                        \
        if (e_ != cudaSuccess) return IDX_ERR_CUDA;  \
    } while (0)

__global__ void scatter_slots(const int *rows, int nrows, int R, int *slot, unsigned *status) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nrows) return;
    const int r = rows[i];
    if (r < 0 || r >= R) {
        atomicOr(status, ST_INVALID);
        return;
    }
    slot[r] = i;
}

__global__ void copy_rows(const float *src, long long src_ld, const int *rows, int nrows, int R, int ncols,
                          float *dst, long long ld, unsigned *status) {
    const int i = blockIdx.y;
    if (i >= nrows) return;
    const int r = rows[i];
    if (r < 0 || r >= R) {
        if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(status, ST_INVALID);
        return;
    }
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < ncols; j += gridDim.x * blockDim.x)
        dst[(long long)i * ld + j] = src[(long long)r * src_ld + j];
}

struct Prefill {
    const void *q, *k;
    const float *w;
    const int *cu;
    int S, T, H, d, topk;
    idx_dtype dt;
    int g, c;
    idx_mode mode;
    char *ws;
    PrefillWs L;
    cudaStream_t st;
    int db = 0;  // guardrail threshold (PIVOT modes)
    int row_lo = 0, row_hi = -1;  // output rows of the call (-1: up to T)

    unsigned *status() const { return reinterpret_cast<unsigned *>(ws + L.status); }
    int *plan() const { return reinterpret_cast<int *>(ws + L.plan); }

    ScoreArgs score_args(bool proxies) const {
        ScoreArgs a{};
        const bool blocks = proxies && mode == IDX_MODE_BLOCK;
        a.q = proxies ? (const void *)(ws + L.qbar) : q;
        a.k = blocks ? (const void *)(ws + L.kblk) : k;
        a.kshift = blocks ? kBlockShift : 0;
        a.w = proxies ? reinterpret_cast<const float *>(ws + L.wbar) : w;
        a.cu = cu;
        a.S = S; a.T = T; a.H = H; a.d = d;
        a.g = proxies ? g : 1;
        a.db = proxies ? db : 0;
        a.R = proxies ? L.R : T;
        a.plan = plan();
        a.pl = L.pl;
        a.sink = SINK_FILTER;
        a.buf = reinterpret_cast<unsigned long long *>(ws + L.buf);
        a.cap = L.cap;
        a.ksel = L.ksel;
        a.ksel_dense = (unsigned)topk < L.ksel ? (unsigned)topk : L.ksel;
        a.cnt = reinterpret_cast<unsigned *>(ws + L.cnt);
        a.floor_out = reinterpret_cast<unsigned *>(ws + L.floor);
        a.status = status();
        return a;
    }

    cudaError_t score(const ScoreArgs &a) const {
        // the persistent score kernels pull row blocks from plan[3]
        cudaError_t e = cudaMemsetAsync(plan() + 3, 0, 4, st);
        if (e != cudaSuccess) return e;
        return tc_supported(H, d, (int)dt) ? launch_score_tc(a, st) : launch_score_simt(a, (int)dt, st);
    }

    cudaError_t prepare() const {
        cudaError_t e = cudaMemsetAsync(status(), 0, 4, st);
        if (e != cudaSuccess) return e;
        e = launch_plan(cu, S, T, mode == IDX_MODE_DENSE ? 1 : g, mode == IDX_MODE_DENSE ? 0 : db, row_lo,
                        row_hi < 0 ? T : row_hi, plan(), L.pl, status(), st);
        if (e != cudaSuccess) return e;
        if (mode != IDX_MODE_DENSE)
            e = launch_proxy(q, w, cu, S, T, H, d, g, db, (int)dt, plan(), L.pl, ws + L.qbar,
                             reinterpret_cast<float *>(ws + L.wbar), (int)L.R, st);
        if (e == cudaSuccess && mode == IDX_MODE_BLOCK)
            e = launch_block_means(k, cu, S, T, d, (int)dt, ws + L.kblk, st);
        if (e == cudaSuccess && mode == IDX_MODE_QUEST)
            e = launch_block_minmax(k, cu, S, T, d, (int)dt, ws + L.kblk, st);
        return e;
    }

    SelectArgs select_args(int kind, int nrows, int kk, int *oi, float *os) const {
        SelectArgs s{};
        s.kind = kind;
        s.nrows = nrows;
        s.k = kk;
        s.out_idx = oi;
        s.out_score = os;
        s.cu = cu;
        s.S = S;
        s.g = mode == IDX_MODE_DENSE ? 1 : g;
        s.db = mode == IDX_MODE_DENSE ? 0 : db;
        s.plan = plan();
        s.pl = L.pl;
        s.buf = reinterpret_cast<const unsigned long long *>(ws + L.buf);
        s.cap = L.cap;
        s.cnt = reinterpret_cast<const unsigned *>(ws + L.cnt);
        s.floor = reinterpret_cast<const unsigned *>(ws + L.floor);
        s.c = c;
        s.cand = reinterpret_cast<const int *>(ws + L.cand);
        s.scores = reinterpret_cast<const float *>(ws + L.msc);
        s.ld = c;
        s.bitmap_words = (int)(nbound(T) / 32 + 1);
        s.status = status();
        return s;
    }

    GatherArgs gather_args() const {
        GatherArgs a{};
        a.q = q; a.k = k; a.w = w;
        a.cand = reinterpret_cast<const int *>(ws + L.cand);
        a.c = c; a.H = H; a.d = d;
        a.nitems = (int)L.R;
        a.mode = 0;
        a.cu = cu; a.S = S; a.g = g; a.db = db; a.cu_T = T;
        a.plan = plan(); a.pl = L.pl;
        a.out = reinterpret_cast<float *>(ws + L.msc);
        a.ckeys = ws + L.ckeys;
        a.ckey_groups = L.Rb;
        a.c_pad = c_pad_of(c);
        a.status = status();
        return a;
    }
};

idx_status check_prefill(const void *q, const void *k, const float *w, const int *cu, int S, int T, int H,
                         int d, int topk, idx_dtype dt, const int *out_idx, void *ws, size_t ws_bytes,
                         size_t need) {
    if (!q || !k || !w || !cu || !out_idx) return IDX_ERR_INVALID;
    if (S < 1 || T < 1 || topk < 1 || !shape_ok(H, d, dt)) return IDX_ERR_INVALID;
    if (!path_ok(H, d, dt)) return IDX_ERR_UNSUPPORTED;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 || ws_bytes < need) return IDX_ERR_WORKSPACE;
    return IDX_OK;
}

}  // namespace

extern "C" {

const char *idx_status_string(idx_status s) {
    switch (s) {
    case IDX_OK: return "IDX_OK";
    case IDX_ERR_INVALID: return "IDX_ERR_INVALID";
    case IDX_ERR_UNSUPPORTED: return "IDX_ERR_UNSUPPORTED";
    case IDX_ERR_WORKSPACE: return "IDX_ERR_WORKSPACE";
    case IDX_ERR_CUDA: return "IDX_ERR_CUDA";
    case IDX_ERR_TIMEOUT: return "IDX_ERR_TIMEOUT";
    case IDX_ERR_OVERFLOW: return "IDX_ERR_OVERFLOW";
    }
    return "IDX_ERR_UNKNOWN";
}

int idx_uses_tensor_cores(int H, int d, idx_dtype dtype) { return tc_supported(H, d, (int)dtype) ? 1 : 0; }

size_t idx_dense_workspace_size_rows(int T, int H, int d, int topk, int num_seqs, idx_dtype dtype, int max_rows) {
    if (T < 1 || num_seqs < 1 || topk < 1 || max_rows < 0 || !shape_ok(H, d, dtype)) return 0;
    return prefill_ws(T, H, d, topk, num_seqs, dtype, 1, topk, IDX_MODE_DENSE, 0, max_rows).total;
}

size_t idx_dense_workspace_size(int T, int H, int d, int topk, int num_seqs, idx_dtype dtype) {
    return idx_dense_workspace_size_rows(T, H, d, topk, num_seqs, dtype, 0);
}

idx_status idx_dense_topk_rows(const void *q, const void *k, const float *w, const int *cu_seqlens, int num_seqs,
                               int T, int H, int d, int topk, idx_dtype dtype, int row_lo, int row_hi, int *out_idx,
                               float *out_score, void *ws, size_t ws_bytes, idx_stream_t stream) {
    if (row_lo < 0 || row_hi < row_lo || row_hi > T) return IDX_ERR_INVALID;
    const int m = row_hi - row_lo > 0 ? row_hi - row_lo : 1;
    const size_t need = idx_dense_workspace_size_rows(T, H, d, topk, num_seqs, dtype, m);
    idx_status s = check_prefill(q, k, w, cu_seqlens, num_seqs, T, H, d, topk, dtype, out_idx, ws, ws_bytes,
                                 need);
    if (s != IDX_OK) return s;
    if (row_lo == row_hi) return IDX_OK;
    TracePhase phase("dense");
    Prefill P{q, k, w, cu_seqlens, num_seqs, T, H, d, topk, dtype, 1, topk, IDX_MODE_DENSE,
              static_cast<char *>(ws), prefill_ws(T, H, d, topk, num_seqs, dtype, 1, topk, IDX_MODE_DENSE, 0, m),
              reinterpret_cast<cudaStream_t>(stream)};
    P.row_lo = row_lo;
    P.row_hi = row_hi;
    TRY_CUDA(P.prepare());
    TRY_CUDA(P.score(P.score_args(false)));
    return cuda_st(launch_select(P.select_args(SEL_DENSE_CAND, T, topk, out_idx, out_score), P.st));
}

idx_status idx_dense_topk(const void *q, const void *k, const float *w, const int *cu_seqlens, int num_seqs,
                          int T, int H, int d, int topk, idx_dtype dtype, int *out_idx, float *out_score,
                          void *ws, size_t ws_bytes, idx_stream_t stream) {
    return idx_dense_topk_rows(q, k, w, cu_seqlens, num_seqs, T, H, d, topk, dtype, 0, T > 0 ? T : 0, out_idx,
                               out_score, ws, ws_bytes, stream);
}

size_t idx_adaptive_workspace_size(int T, int H, int d, int topk, int rho, int num_seqs, idx_dtype dtype) {
    if (T < 1 || num_seqs < 1 || topk < 1 || rho < 2 || !shape_ok(H, d, dtype)) return 0;
    if ((long long)topk * rho > kAdaptiveMaxWidth) return 0;
    return adaptive_ws(T, H, d, topk, rho, num_seqs, dtype).total;
}

idx_status idx_adaptive_topk(const void *q, const void *k, const float *w, const int *cu_seqlens, int num_seqs,
                             int T, int H, int d, int topk, int rho, double qfrac, idx_dtype dtype, int *out_idx,
                             float *out_score, float *out_sigma, uint8_t *out_trigger, void *ws, size_t ws_bytes,
                             idx_stream_t stream) {
    if (rho < 2 || !(qfrac >= 0.0 && qfrac <= 1.0) || topk < 1 || (long long)topk * rho > 0x7FFFFFFFLL)
        return IDX_ERR_INVALID;
    if ((long long)topk * rho > kAdaptiveMaxWidth) return IDX_ERR_UNSUPPORTED;
    const int width = topk * rho;
    const size_t need = idx_adaptive_workspace_size(T, H, d, topk, rho, num_seqs, dtype);
    idx_status s = check_prefill(q, k, w, cu_seqlens, num_seqs, T, H, d, width, dtype, out_idx, ws, ws_bytes,
                                 need);
    if (s != IDX_OK) return s;
    TracePhase phase("adaptive");
    const AdaptiveWs L = adaptive_ws(T, H, d, topk, rho, num_seqs, dtype);
    char *base = static_cast<char *>(ws);
    Prefill P{q, k, w, cu_seqlens, num_seqs, T, H, d, width, dtype, 1, width, IDX_MODE_DENSE, base, L.P,
              reinterpret_cast<cudaStream_t>(stream)};
    TRY_CUDA(P.prepare());
    TRY_CUDA(P.score(P.score_args(false)));
    float *sc = out_score ? out_score : reinterpret_cast<float *>(base + L.score);
    AdaptiveArgs a{};
    a.T = T;
    a.k = topk;
    a.width = width;
    a.idx = out_idx;
    a.score = sc;
    a.sigma = out_sigma ? out_sigma : reinterpret_cast<float *>(base + L.sigma);
    a.vk = reinterpret_cast<unsigned *>(base + L.vk);
    a.need = reinterpret_cast<int *>(base + L.need);
    // the final select ranks each row's top-(rho k) and, from the same staged
    // keys, its cutoff margin at k (sigma, the ord of s_(k-1), its ties kept)
    SelectArgs sa = P.select_args(SEL_DENSE_CAND, T, width, out_idx, sc);
    sa.kmargin = topk;
    sa.m_sigma = a.sigma;
    sa.m_vk = a.vk;
    sa.m_need = a.need;
    TRY_CUDA(launch_select(sa, P.st));
    a.trigger = out_trigger;
    a.tau = reinterpret_cast<unsigned *>(base + L.tau);
    a.q = qfrac;
    a.status = P.status();
    return cuda_st(launch_adaptive(a, P.st));
}

size_t idx_pivot_workspace_size_rows(int T, int H, int d, int topk, int num_seqs, idx_dtype dtype, int g, int c,
                                     idx_mode mode, int dense_below, int max_rows) {
    if (T < 1 || num_seqs < 1 || topk < 1 || g < 1 || dense_below < 0 || max_rows < 0 || !shape_ok(H, d, dtype))
        return 0;
    if (mode != IDX_MODE_REUSE && mode != IDX_MODE_REFINE && !blocky(mode)) return 0;
    if (mode == IDX_MODE_REUSE) c = topk;
    if (refines(mode) && c < topk) return 0;
    if (blocky(mode) && (c < kBlockN || c % kBlockN != 0 || dense_below > 0)) return 0;
    if (mode == IDX_MODE_QUEST && quest_scan_smem(H, d) > kMaxSmem) return 0;
    return prefill_ws(T, H, d, topk, num_seqs, dtype, g, c, mode, dense_below, max_rows).total;
}

size_t idx_pivot_workspace_size(int T, int H, int d, int topk, int num_seqs, idx_dtype dtype, int g, int c,
                                idx_mode mode, int dense_below) {
    return idx_pivot_workspace_size_rows(T, H, d, topk, num_seqs, dtype, g, c, mode, dense_below, 0);
}

idx_status idx_pivot_topk_rows(const void *q, const void *k, const float *w, const int *cu_seqlens, int num_seqs,
                               int T, int H, int d, int topk, idx_dtype dtype, int g, int c, idx_mode mode,
                               int dense_below, int row_lo, int row_hi, int *out_idx, float *out_score, void *ws,
                               size_t ws_bytes, idx_stream_t stream) {
    if (g < 1 || dense_below < 0 || (mode != IDX_MODE_REUSE && mode != IDX_MODE_REFINE && !blocky(mode)))
        return IDX_ERR_INVALID;
    if (row_lo < 0 || row_hi < row_lo || row_hi > T) return IDX_ERR_INVALID;
    if (refines(mode) && c < topk) return IDX_ERR_INVALID;
    if (blocky(mode) && (c < kBlockN || c % kBlockN != 0)) return IDX_ERR_INVALID;
    if (blocky(mode) && dense_below > 0) return IDX_ERR_UNSUPPORTED;
    if (mode == IDX_MODE_QUEST && quest_scan_smem(H, d) > kMaxSmem) return IDX_ERR_UNSUPPORTED;
    // every request is at most T tokens long: with dense_below >= T every
    // group is short and the call is the dense call (the same rows, without
    // the grouped pipeline's extra work)
    if (g > 1 && dense_below >= T && T > 0) {
        if (!ws || ws_bytes < idx_pivot_workspace_size_rows(T, H, d, topk, num_seqs, dtype, g,
                                                             mode == IDX_MODE_REUSE ? topk : c, mode, dense_below,
                                                             row_hi - row_lo > 0 ? row_hi - row_lo : 1))
            return IDX_ERR_WORKSPACE;
        return idx_dense_topk_rows(q, k, w, cu_seqlens, num_seqs, T, H, d, topk, dtype, row_lo, row_hi, out_idx,
                                   out_score, ws, ws_bytes, stream);
    }
    if (mode == IDX_MODE_REUSE) c = topk;
    const int m = row_hi - row_lo > 0 ? row_hi - row_lo : 1;
    const size_t need = idx_pivot_workspace_size_rows(T, H, d, topk, num_seqs, dtype, g, c, mode, dense_below, m);
    idx_status s = check_prefill(q, k, w, cu_seqlens, num_seqs, T, H, d, topk, dtype, out_idx, ws, ws_bytes,
                                 need);
    if (s != IDX_OK) return s;
    if (row_lo == row_hi) return IDX_OK;
    TracePhase phase(mode == IDX_MODE_REUSE    ? "reuse"
                     : mode == IDX_MODE_REFINE ? "refine"
                     : mode == IDX_MODE_BLOCK  ? "block"
                                               : "quest");
    Prefill P{q, k, w, cu_seqlens, num_seqs, T, H, d, topk, dtype, g, c, mode, static_cast<char *>(ws),
              prefill_ws(T, H, d, topk, num_seqs, dtype, g, c, mode, dense_below, m),
              reinterpret_cast<cudaStream_t>(stream)};
    P.db = g > 1 ? dense_below : 0;
    P.row_lo = row_lo;
    P.row_hi = row_hi;
    TRY_CUDA(P.prepare());
    int *cand = reinterpret_cast<int *>(P.ws + P.L.cand);
    if (mode == IDX_MODE_QUEST) {
        // the proxies' Quest bounds of their complete blocks, the top blocks
        // of each, then the candidate positions as in the block-mean rule
        float *qsp = reinterpret_cast<float *>(P.ws + P.L.qspill);
        int *cblk = reinterpret_cast<int *>(P.ws + P.L.cblk);
        TRY_CUDA(launch_prefill_quest_scan(P.ws + P.L.qbar, reinterpret_cast<const float *>(P.ws + P.L.wbar),
                                           P.ws + P.L.kblk, cu_seqlens, num_seqs, g, P.plan(), P.L.pl, (int)P.L.R,
                                           (int)P.L.nbmax, H, d, (int)dtype, qsp, P.L.nbmax, P.st));
        SelectArgs sa = P.select_args(SEL_PROXY_SPILL_TO_BLOCKS, (int)P.L.R, c >> kBlockShift, cblk, nullptr);
        sa.scores = qsp;
        sa.ld = P.L.nbmax;
        TRY_CUDA(launch_select(sa, P.st));
        TRY_CUDA(launch_block_expand(cu_seqlens, num_seqs, g, P.plan(), P.L.pl, cblk, cand, c, (int)P.L.R, P.st));
        const GatherArgs ga = P.gather_args();
        TRY_CUDA(tc_gather_supported(H, d, (int)dtype, g, c) ? launch_gather_tc(ga, P.st)
                                                           : launch_gather_simt(ga, (int)dtype, P.st));
        return cuda_st(launch_select(P.select_args(SEL_MEMBER_SCORES, T, topk, out_idx, out_score), P.st));
    }
    TRY_CUDA(P.score(P.score_args(true)));
    if (mode == IDX_MODE_REUSE)
        return cuda_st(launch_select(P.select_args(SEL_REUSE_CAND, T, topk, out_idx, out_score), P.st));
    if (mode == IDX_MODE_BLOCK) {
        int *cblk = reinterpret_cast<int *>(P.ws + P.L.cblk);
        TRY_CUDA(launch_select(P.select_args(SEL_PROXY_TO_BLOCKS, (int)P.L.R, c >> kBlockShift, cblk, nullptr),
                               P.st));
        TRY_CUDA(launch_block_expand(cu_seqlens, num_seqs, g, P.plan(), P.L.pl, cblk, cand, c, (int)P.L.R, P.st));
    } else {
        TRY_CUDA(launch_select(P.select_args(SEL_PROXY_TO_C, (int)P.L.R, c, cand, nullptr), P.st));
    }
    const GatherArgs ga = P.gather_args();
    TRY_CUDA(tc_gather_supported(H, d, (int)dtype, g, c) ? launch_gather_tc(ga, P.st)
                                                       : launch_gather_simt(ga, (int)dtype, P.st));
    return cuda_st(launch_select(P.select_args(SEL_MEMBER_SCORES, T, topk, out_idx, out_score), P.st));
}

idx_status idx_pivot_topk(const void *q, const void *k, const float *w, const int *cu_seqlens, int num_seqs,
                          int T, int H, int d, int topk, idx_dtype dtype, int g, int c, idx_mode mode,
                          int dense_below, int *out_idx, float *out_score, void *ws, size_t ws_bytes,
                          idx_stream_t stream) {
    return idx_pivot_topk_rows(q, k, w, cu_seqlens, num_seqs, T, H, d, topk, dtype, g, c, mode, dense_below, 0,
                               T > 0 ? T : 0, out_idx, out_score, ws, ws_bytes, stream);
}

size_t idx_decode_workspace_size(int B, int G, int n_max, int H, int d, int topk, int c, idx_mode mode,
                                 idx_dtype dtype) {
    if (B < 1 || G < 1 || G > RB || n_max < G || n_max > kMaxLen || topk < 1 || !shape_ok(H, d, dtype))
        return 0;
    if (mode != IDX_MODE_DENSE && mode != IDX_MODE_REUSE && mode != IDX_MODE_REFINE) return 0;
    if (mode == IDX_MODE_REFINE && c < topk) return 0;
    return decode_ws(B, G, n_max, H, d, c, mode, dtype).total;
}

namespace {

struct Decode {
    const void *q, *kc;
    const int *kv;
    const float *w;
    int B, G, n_max, H, d, topk, c;
    idx_mode mode;
    idx_dtype dt;
    char *ws;
    DecodeWs L;
    cudaStream_t st;
    const int *bt = nullptr;  // paged cache: block table [B, max_pages], else NULL
    int page = 0, max_pages = 0;
    long long num_pages = 0;
    const void *kbar = nullptr;  // block mode: block means [B, n_max / 64, d], or
    int rule = 0;                // (rule 1, Quest) per-block key min and max [B, n_max / 64, 2, d]

    unsigned *status() const { return reinterpret_cast<unsigned *>(ws + L.status); }

    DecodeArgs dargs(bool proxy, float *spill) const {
        DecodeArgs a{};
        a.q = proxy ? (const void *)(ws + L.qbar) : q;
        a.kc = kc;
        a.w = proxy ? reinterpret_cast<const float *>(ws + L.wbar) : w;
        a.kv_len = kv;
        a.B = B; a.G = G; a.Gq = proxy ? 1 : G; a.n_max = n_max; a.H = H; a.d = d;
        a.chunk_tiles = 64;
        a.spill = spill;
        a.status = status();
        a.bt = bt; a.page = page; a.max_pages = max_pages; a.num_pages = num_pages;
        return a;
    }
    cudaError_t scan(const DecodeArgs &a) const {
        // the tensor-core scan loads a paged tile as 128 / page boxes; a box of
        // fewer than 8 rows would break the 1 KB alignment of its swizzled slice
        const bool tc = tc_decode_supported(H, d, (int)dt, a.Gq) && (!bt || page >= 8);
        return tc ? launch_decode_tc(a, st) : launch_decode_simt(a, (int)dt, st);
    }
    SelectArgs sargs(int kind, int nrows, int kk, int *oi, float *os, const float *scores, long long ld) const {
        SelectArgs s{};
        s.kind = kind; s.nrows = nrows; s.k = kk; s.out_idx = oi; s.out_score = os;
        s.scores = scores; s.ld = ld;
        s.cand = reinterpret_cast<const int *>(ws + L.cand);
        s.c = c;
        s.kv_len = kv; s.G = G; s.n_max = n_max;
        s.bitmap_words = n_max / 32 + 1;
        s.status = status();
        return s;
    }
    GatherArgs gargs() const {
        GatherArgs a{};
        a.q = q; a.k = kc; a.w = w;
        a.cand = reinterpret_cast<const int *>(ws + L.cand);
        a.c = c; a.H = H; a.d = d;
        a.nitems = B;
        a.mode = 1;
        a.G = G; a.n_max = n_max; a.kv_len = kv;
        a.out = reinterpret_cast<float *>(ws + L.msc);
        a.ckeys = ws + L.ckeys;
        a.ckey_groups = B;
        a.c_pad = c_pad_of(c);
        a.status = status();
        a.bt = bt; a.page = page; a.max_pages = max_pages; a.num_pages = num_pages;
        return a;
    }
    idx_status run(int *out_idx, float *out_score) const;
};

idx_status Decode::run(int *out_idx, float *out_score) const {
    TRY_CUDA(cudaMemsetAsync(status(), 0, 4, st));
    float *spill = reinterpret_cast<float *>(ws + L.spill);
    if (mode == IDX_MODE_DENSE) {
        TRY_CUDA(scan(dargs(false, spill)));
        return cuda_st(launch_select(sargs(SEL_DEC_DENSE, B * G, topk, out_idx, out_score, spill, n_max), st));
    }
    TRY_CUDA(launch_decode_proxy(q, w, B, G, H, d, (int)dt, ws + L.qbar, reinterpret_cast<float *>(ws + L.wbar), st));
    int *cand = reinterpret_cast<int *>(ws + L.cand);
    if (mode == IDX_MODE_BLOCK) {
        // the proxy against the block means of the complete blocks, then the
        // chosen blocks (and the partial block) become the candidate set
        int *nlen = reinterpret_cast<int *>(ws + L.nlen);
        int *cblk = reinterpret_cast<int *>(ws + L.cblk);
        TRY_CUDA(launch_decode_block_len(kv, B, G, n_max, nlen, st));
        if (rule == 1) {
            TRY_CUDA(launch_decode_quest_scan(ws + L.qbar, reinterpret_cast<const float *>(ws + L.wbar), kbar, nlen,
                                              B, n_max >> kBlockShift, H, d, (int)dt, spill, st));
        } else {
            DecodeArgs a = dargs(true, spill);
            a.kc = kbar;
            a.kv_len = nlen;
            a.G = 1;
            a.n_max = n_max >> kBlockShift;
            TRY_CUDA(scan(a));
        }
        TRY_CUDA(launch_select(sargs(SEL_DEC_PROXY_TO_BLOCKS, B, c >> kBlockShift, cblk, nullptr, spill,
                                     n_max >> kBlockShift),
                               st));
        TRY_CUDA(launch_decode_block_expand(kv, B, G, n_max, cblk, cand, c, st));
    } else {
        TRY_CUDA(scan(dargs(true, spill)));
        if (mode == IDX_MODE_REUSE)
            return cuda_st(launch_select(sargs(SEL_DEC_REUSE, B * G, topk, out_idx, out_score, spill, n_max), st));
        TRY_CUDA(launch_select(sargs(SEL_DEC_PROXY_TO_C, B, c, cand, nullptr, spill, n_max), st));
    }
    const GatherArgs ga = gargs();
    TRY_CUDA(tc_gather_supported(H, d, (int)dt, G, c) ? launch_gather_tc(ga, st)
                                                     : launch_gather_simt(ga, (int)dt, st));
    const float *msc = reinterpret_cast<const float *>(ws + L.msc);
    return cuda_st(launch_select(sargs(SEL_DEC_MEMBER, B * G, topk, out_idx, out_score, msc, c), st));
}

idx_status check_decode(const void *q, const void *kc, const int *kv, const float *w, int B, int G, int n_max,
                        int H, int d, int topk, int c, idx_mode mode, idx_dtype dt, const int *out_idx,
                        void *ws, size_t ws_bytes) {
    if (!q || !kc || !kv || !w || !out_idx) return IDX_ERR_INVALID;
    if (B < 1 || G < 1 || n_max < G || topk < 1 || !shape_ok(H, d, dt)) return IDX_ERR_INVALID;
    if (mode != IDX_MODE_DENSE && mode != IDX_MODE_REUSE && mode != IDX_MODE_REFINE) return IDX_ERR_INVALID;
    if (mode == IDX_MODE_REFINE && c < topk) return IDX_ERR_INVALID;
    if (G > RB || n_max > kMaxLen || !path_ok(H, d, dt)) return IDX_ERR_UNSUPPORTED;
    const size_t need = idx_decode_workspace_size(B, G, n_max, H, d, topk, c, mode, dt);
    if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 || ws_bytes < need) return IDX_ERR_WORKSPACE;
    return IDX_OK;
}

}  // namespace

idx_status idx_decode_topk(const void *q, const void *kcache, const int *kv_len, const float *w, int B, int G,
                           int n_max, int H, int d, int topk, int c, idx_mode mode, idx_dtype dtype,
                           int *out_idx, float *out_score, void *ws, size_t ws_bytes, idx_stream_t stream) {
    idx_status s = check_decode(q, kcache, kv_len, w, B, G, n_max, H, d, topk, c, mode, dtype, out_idx, ws,
                                ws_bytes);
    if (s != IDX_OK) return s;
    TracePhase phase(mode == IDX_MODE_DENSE ? "decode_dense" : mode == IDX_MODE_REUSE ? "decode_reuse" : "decode_refine");
    Decode D{q, kcache, kv_len, w, B, G, n_max, H, d, topk, c, mode, dtype, static_cast<char *>(ws),
             decode_ws(B, G, n_max, H, d, c, mode, dtype), reinterpret_cast<cudaStream_t>(stream)};
    return D.run(out_idx, out_score);
}

idx_status idx_decode_paged_topk(const void *q, const void *kpool, const int *block_table, const int *kv_len,
                                 const float *w, int B, int G, int max_pages, int page, long long num_pages, int H,
                                 int d, int topk, int c, idx_mode mode, idx_dtype dtype, int *out_idx,
                                 float *out_score, void *ws, size_t ws_bytes, idx_stream_t stream) {
    if (!block_table || max_pages < 1 || page < 1 || num_pages < 1) return IDX_ERR_INVALID;
    if ((long long)max_pages * page > kMaxLen) return IDX_ERR_UNSUPPORTED;
    if (KT % page != 0 && page % KT != 0) return IDX_ERR_UNSUPPORTED;
    if (num_pages > (long long)0x7FFFFFFF / page) return IDX_ERR_UNSUPPORTED;
    const int n_max = max_pages * page;
    idx_status s = check_decode(q, kpool, kv_len, w, B, G, n_max, H, d, topk, c, mode, dtype, out_idx, ws,
                                ws_bytes);
    if (s != IDX_OK) return s;
    TracePhase phase(mode == IDX_MODE_DENSE ? "decode_paged_dense"
                     : mode == IDX_MODE_REUSE ? "decode_paged_reuse"
                                              : "decode_paged_refine");
    Decode D{q, kpool, kv_len, w, B, G, n_max, H, d, topk, c, mode, dtype, static_cast<char *>(ws),
             decode_ws(B, G, n_max, H, d, c, mode, dtype), reinterpret_cast<cudaStream_t>(stream)};
    D.bt = block_table;
    D.page = page;
    D.max_pages = max_pages;
    D.num_pages = num_pages;
    return D.run(out_idx, out_score);
}

namespace {

idx_status check_decode_block(int B, int G, int n_max, int H, int d, int topk, int c, int rule, idx_dtype dt) {
    if (B < 1 || G < 1 || n_max < G || topk < 1 || !shape_ok(H, d, dt)) return IDX_ERR_INVALID;
    if (n_max % kBlockN != 0 || c < topk || c < kBlockN || c % kBlockN != 0 || (rule != 0 && rule != 1))
        return IDX_ERR_INVALID;
    if (G > RB || n_max > kMaxLen || !path_ok(H, d, dt)) return IDX_ERR_UNSUPPORTED;
    if (rule == 1 && quest_scan_smem(H, d) > kMaxSmem) return IDX_ERR_UNSUPPORTED;
    return IDX_OK;
}

}  // namespace

size_t idx_decode_block_workspace_size(int B, int G, int n_max, int H, int d, int topk, int c, int rule,
                                       idx_dtype dtype) {
    if (check_decode_block(B, G, n_max, H, d, topk, c, rule, dtype) != IDX_OK) return 0;
    return decode_ws(B, G, n_max, H, d, c, IDX_MODE_BLOCK, dtype).total;
}

idx_status idx_decode_block_means(const void *kcache, int B, int n_max, int d, idx_dtype dtype, int first_block,
                                  void *kbar, idx_stream_t stream) {
    if (!kcache || !kbar || B < 1 || n_max < kBlockN || n_max % kBlockN != 0 || first_block < 0 ||
        !shape_ok(1, d, dtype))
        return IDX_ERR_INVALID;
    if (n_max > kMaxLen) return IDX_ERR_UNSUPPORTED;
    TracePhase phase("decode_block");
    return cuda_st(launch_decode_block_means(kcache, B, n_max, d, (int)dtype, first_block, kbar,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

idx_status idx_decode_block_minmax(const void *kcache, int B, int n_max, int d, idx_dtype dtype, int first_block,
                                   void *kminmax, idx_stream_t stream) {
    if (!kcache || !kminmax || B < 1 || n_max < kBlockN || n_max % kBlockN != 0 || first_block < 0 ||
        !shape_ok(1, d, dtype))
        return IDX_ERR_INVALID;
    if (n_max > kMaxLen) return IDX_ERR_UNSUPPORTED;
    TracePhase phase("decode_quest");
    return cuda_st(launch_decode_block_minmax(kcache, B, n_max, d, (int)dtype, first_block, kminmax,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

idx_status idx_decode_block_topk(const void *q, const void *kcache, const void *ksum, int rule, const int *kv_len,
                                 const float *w, int B, int G, int n_max, int H, int d, int topk, int c,
                                 idx_dtype dtype, int *out_idx, float *out_score, void *ws, size_t ws_bytes,
                                 idx_stream_t stream) {
    if (!q || !kcache || !ksum || !kv_len || !w || !out_idx) return IDX_ERR_INVALID;
    idx_status s = check_decode_block(B, G, n_max, H, d, topk, c, rule, dtype);
    if (s != IDX_OK) return s;
    const size_t need = decode_ws(B, G, n_max, H, d, c, IDX_MODE_BLOCK, dtype).total;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 || ws_bytes < need) return IDX_ERR_WORKSPACE;
    TracePhase phase(rule == 1 ? "decode_quest" : "decode_block");
    Decode D{q, kcache, kv_len, w, B, G, n_max, H, d, topk, c, IDX_MODE_BLOCK, dtype, static_cast<char *>(ws),
             decode_ws(B, G, n_max, H, d, c, IDX_MODE_BLOCK, dtype), reinterpret_cast<cudaStream_t>(stream)};
    D.kbar = ksum;
    D.rule = rule;
    return D.run(out_idx, out_score);
}

size_t idx_sparse_attn_workspace_size(void) { return kAlign; }

idx_status idx_sparse_attn(const void *q, const void *kv, const int *idx, const int *cu_q, const int *cu_kv,
                           int num_seqs, int R, long long Nkv, int H, int Dqk, int Dv, int topk, float scale,
                           idx_dtype dtype, void *out, float *lse, void *ws, size_t ws_bytes, idx_stream_t stream) {
    if (!q || !kv || !idx || !cu_q || !cu_kv || !out) return IDX_ERR_INVALID;
    if (num_seqs < 1 || R < 0 || Nkv < 1 || H < 1 || Dqk < 1 || Dv < 1 || Dv > Dqk || topk < 1 || !isfinite(scale))
        return IDX_ERR_INVALID;
    if (dtype != IDX_BF16 && dtype != IDX_F32) return IDX_ERR_INVALID;
    if (!attn_tc_supported(H, Dqk, Dv, (int)dtype) || (long long)R * 128 > 0x7FFFFFFFLL) return IDX_ERR_UNSUPPORTED;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 || ws_bytes < kAlign) return IDX_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    TracePhase phase("sparse_attn");
    unsigned *status = static_cast<unsigned *>(ws);
    TRY_CUDA(cudaMemsetAsync(status, 0, 4, st));
    if (R == 0) return IDX_OK;
    SparseAttnArgs a{};
    a.q = q; a.kv = kv; a.idx = idx; a.cu_q = cu_q; a.cu_kv = cu_kv;
    a.S = num_seqs; a.R = R; a.H = H; a.topk = topk; a.Nkv = Nkv; a.scale = scale;
    a.out = out; a.lse = lse; a.status = status;
    return cuda_st(launch_sparse_attn_tc(a, st));
}

idx_status idx_device_status(const void *ws, idx_stream_t stream) {
    if (!ws) return IDX_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    unsigned h = 0;
    if (cudaMemcpyAsync(&h, ws, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess) return IDX_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return IDX_ERR_CUDA;
    if (h & ST_TIMEOUT) return IDX_ERR_TIMEOUT;
    if (h & ST_OVERFLOW) return IDX_ERR_OVERFLOW;
    if (h & ST_INVALID) return IDX_ERR_INVALID;
    return IDX_OK;
}

idx_status idx_debug_scores(int stage, const void *q, const void *k, const float *w, const int *cu_seqlens,
                            int num_seqs, int T, int H, int d, idx_dtype dtype, int g, int c, int topk,
                            const int *rows, int nrows, float *out, long long ld, void *ws, size_t ws_bytes,
                            idx_stream_t stream) {
    if (!rows || !out || nrows < 0 || ld < 1 || stage < 0 || stage > 4) return IDX_ERR_INVALID;
    const idx_mode mode = stage == 0   ? IDX_MODE_DENSE
                          : stage >= 3 ? IDX_MODE_BLOCK
                                       : (stage == 2 || c > 0 ? IDX_MODE_REFINE : IDX_MODE_REUSE);
    const int gg = stage == 0 ? 1 : g;
    const int cc = refines(mode) ? c : topk;
    if (gg < 1 || (refines(mode) && cc < topk)) return IDX_ERR_INVALID;
    if (mode == IDX_MODE_BLOCK && (cc < kBlockN || cc % kBlockN != 0)) return IDX_ERR_INVALID;
    const size_t need = mode == IDX_MODE_DENSE
                            ? idx_dense_workspace_size(T, H, d, topk, num_seqs, dtype)
                            : idx_pivot_workspace_size(T, H, d, topk, num_seqs, dtype, gg, cc, mode, 0);
    int dummy = 0;
    idx_status s = check_prefill(q, k, w, cu_seqlens, num_seqs, T, H, d, topk, dtype, &dummy, ws, ws_bytes, need);
    if (s != IDX_OK) return s;
    Prefill P{q, k, w, cu_seqlens, num_seqs, T, H, d, topk, dtype, gg, cc, mode, static_cast<char *>(ws),
              prefill_ws(T, H, d, topk, num_seqs, dtype, gg, cc, mode), reinterpret_cast<cudaStream_t>(stream)};
    if (nrows == 0) return IDX_OK;
    if (stage == 2 || stage == 4) {
        TRY_CUDA(cudaMemsetAsync(P.status(), 0, 4, P.st));
        for (int r0 = 0; r0 < nrows; r0 += 65535) {
            const int nr = nrows - r0 < 65535 ? nrows - r0 : 65535;
            dim3 grid((c + 255) / 256 < 64 ? (c + 255) / 256 : 64, nr);
            copy_rows<<<grid, 256, 0, P.st>>>(reinterpret_cast<const float *>(P.ws + P.L.msc), c, rows + r0, nr,
                                              T, c, out + (long long)r0 * ld, ld, P.status());
            TRY_CUDA(cudaGetLastError());
        }
        return IDX_OK;
    }
    TRY_CUDA(P.prepare());
    int *slot = reinterpret_cast<int *>(P.ws + P.L.slot);
    const long long R = stage == 0 ? T : P.L.R;
    TRY_CUDA(cudaMemsetAsync(slot, 0xFF, (size_t)R * 4, P.st));
    scatter_slots<<<(nrows + 255) / 256, 256, 0, P.st>>>(rows, nrows, (int)R, slot, P.status());
    TRY_CUDA(cudaGetLastError());
    ScoreArgs a = P.score_args(stage == 1 || stage == 3);
    a.sink = SINK_SPILL;
    a.spill = out;
    a.ld = ld;
    a.slot_of_row = slot;
    return cuda_st(P.score(a));
}

idx_status idx_debug_decode_scores(int stage, const void *q, const void *kcache, const int *kv_len, const float *w,
                                   int B, int G, int n_max, int H, int d, int topk, int c, idx_mode mode,
                                   idx_dtype dtype, float *out, long long ld, void *ws, size_t ws_bytes,
                                   idx_stream_t stream) {
    if (!out || ld < 1 || stage < 0 || stage > 2) return IDX_ERR_INVALID;
    if (stage == 0) mode = IDX_MODE_DENSE;
    if (stage == 2 && mode != IDX_MODE_REFINE) return IDX_ERR_INVALID;
    if (stage == 1 && mode == IDX_MODE_DENSE) return IDX_ERR_INVALID;
    int dummy = 0;
    idx_status s = check_decode(q, kcache, kv_len, w, B, G, n_max, H, d, topk, c, mode, dtype, &dummy, ws, ws_bytes);
    if (s != IDX_OK) return s;
    Decode D{q, kcache, kv_len, w, B, G, n_max, H, d, topk, c, mode, dtype, static_cast<char *>(ws),
             decode_ws(B, G, n_max, H, d, c, mode, dtype), reinterpret_cast<cudaStream_t>(stream)};
    TRY_CUDA(cudaMemsetAsync(D.status(), 0, 4, D.st));
    if (stage == 2) {
        // member re-scores of the preceding Refine call: rows b*G+m
        const float *msc = reinterpret_cast<const float *>(D.ws + D.L.msc);
        for (int r = 0; r < B * G; ++r)
            TRY_CUDA(cudaMemcpyAsync(out + (long long)r * ld, msc + (long long)r * c, (size_t)c * 4,
                                     cudaMemcpyDeviceToDevice, D.st));
        return IDX_OK;
    }
    if (stage == 1)
        TRY_CUDA(launch_decode_proxy(q, w, B, G, H, d, (int)dtype, D.ws + D.L.qbar,
                                     reinterpret_cast<float *>(D.ws + D.L.wbar), D.st));
    DecodeArgs a = D.dargs(stage == 1, out);
    a.spill = out;
    // the scan kernels write row r at spill + r * n_max; a separate ld needs a staging copy
    if (ld == n_max) return cuda_st(D.scan(a));
    float *spill = reinterpret_cast<float *>(D.ws + D.L.spill);
    a.spill = spill;
    TRY_CUDA(D.scan(a));
    const int rows = stage == 1 ? B : B * G;
    for (int r = 0; r < rows; ++r)
        TRY_CUDA(cudaMemcpyAsync(out + (long long)r * ld, spill + (long long)r * n_max, (size_t)n_max * 4,
                                 cudaMemcpyDeviceToDevice, D.st));
    return IDX_OK;
}

}  // extern "C"
