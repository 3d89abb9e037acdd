// proxy.cu -- PIVOT group proxies (PIVOT page, Experimental setup: the proxy
// is the mean of the group's queries; the mean of w is the reading used for
// the proxy's head weights).
//
// Per head and dimension: fp32 sum of the members in member order, one IEEE
// fp32 division by the group size, then round-to-nearest-even to bf16 for
// bf16 queries.  Loads are 16-byte vectors along the contiguous H*d axis.
#include "common.cuh"
#include "plan.cuh"

namespace idx {

namespace {

constexpr int kProxyThreads = 256;

template <typename T>
struct Vec;  // 8 elements per 16-byte load
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void load(const __nv_bfloat16 *p, float *f) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 t = __bfloat1622float2(h[i]);
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    }
    __device__ static void store(__nv_bfloat16 *p, const float *f) {
        uint4 v;
        __nv_bfloat16 *h = reinterpret_cast<__nv_bfloat16 *>(&v);
#pragma unroll
        for (int i = 0; i < 8; ++i) h[i] = __float2bfloat16_rn(f[i]);
        *reinterpret_cast<uint4 *>(p) = v;
    }
};
template <>
struct Vec<float> {
    static constexpr int N = 8;
    __device__ static void load(const float *p, float *f) {
        const float4 a = reinterpret_cast<const float4 *>(p)[0];
        const float4 b = reinterpret_cast<const float4 *>(p)[1];
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
    __device__ static void store(float *p, const float *f) {
        reinterpret_cast<float4 *>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
        reinterpret_cast<float4 *>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
};

// mean of cnt consecutive rows (row stride HD) -> one row
template <typename T>
__device__ void mean_rows(const T *src, const float *wsrc, int cnt, int HD, int H, T *dst, float *wdst) {
    const float fc = (float)cnt;
    for (int e = threadIdx.x * 8; e < HD; e += blockDim.x * 8) {
        float acc[8], v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        for (int m = 0; m < cnt; ++m) {
            Vec<T>::load(src + (long long)m * HD + e, v);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], v[i]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = __fdiv_rn(acc[i], fc);
        Vec<T>::store(dst + e, acc);
    }
    for (int j = threadIdx.x; j < H; j += blockDim.x) {
        float s = 0.0f;
        for (int m = 0; m < cnt; ++m) s = __fadd_rn(s, wsrc[(long long)m * H + j]);
        wdst[j] = __fdiv_rn(s, fc);
    }
}

template <typename T>
__global__ void __launch_bounds__(kProxyThreads) proxy_kernel(const T *q, const float *w, const int *cu, int S,
                                                              int H, int d, int g, int db, const int *plan,
                                                              PlanLayout pl, T *qbar, float *wbar) {
    const int p = blockIdx.x;
    if (!plan[0] || p >= plan[2]) return;
    const int *rp = plan + pl.rp();
    const int b = find_seg(rp, S, p);
    const int i = p - rp[b];
    const int n = cu[b + 1] - cu[b];
    // a member scored on its own (guardrail) is a group of one: its mean is
    // the member itself, bit for bit
    const int lo = group_start(i, n, g, db);
    const int cnt = group_size(i, n, g, db);
    const int HD = H * d;
    const long long m0 = (long long)cu[b] + lo;
    mean_rows(q + m0 * HD, w + m0 * H, cnt, HD, H, qbar + (long long)p * HD, wbar + (long long)p * H);
}

template <typename T>
__global__ void __launch_bounds__(kProxyThreads) decode_proxy_kernel(const T *q, const float *w, int G, int H,
                                                                     int d, T *qbar, float *wbar) {
    const int b = blockIdx.x;
    const int HD = H * d;
    mean_rows(q + (long long)b * G * HD, w + (long long)b * G * H, G, HD, H, qbar + (long long)b * HD,
              wbar + (long long)b * H);
}

// Block pre-filter (page "Uncertainty-gated selection for block-sparse
// attention", Sec. 3.1: a block of 64 keys is summarised by its mean key;
// page "Not All Tokens Deserve Equal Resolution", abstract: coarse chunk
// summaries first, exact token scores inside the chosen chunks next).  The
// mean of each complete block of a request: fp32 sum in key order, one IEEE
// division by the block size, bf16 round-to-nearest-even for bf16 keys.
// Block i of request b goes to row (cu[b] >> kBlockShift) + i; rows that
// belong to no complete block are zero.  One thread per 8 dimensions of one
// block row.
template <typename T>
__global__ void __launch_bounds__(kProxyThreads) block_mean_kernel(const T *k, const int *cu, int S, int T_,
                                                                   int d, long long nrows, T *kb) {
    const int per_row = d / 8;
    const long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= nrows * per_row) return;
    const long long x = u / per_row;
    const int e = (int)(u - x * per_row) * 8;
    // the request whose block rows start at or before x (last such b)
    int lo = 0, hi = S;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if ((long long)(cu[mid] >> kBlockShift) <= x) lo = mid; else hi = mid;
    }
    const long long i = x - (cu[lo] >> kBlockShift);
    // malformed cu_seqlens (the plan flags them) read nothing
    const bool ok = cu[lo] >= 0 && cu[lo] <= cu[lo + 1] && cu[lo + 1] <= T_;
    const int nfull = ok ? (cu[lo + 1] - cu[lo]) >> kBlockShift : 0;
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
    if (i < nfull) {
        const T *src = k + ((long long)cu[lo] + i * kBlockN) * d + e;
        float v[8];
        for (int r = 0; r < kBlockN; ++r) {
            Vec<T>::load(src + (long long)r * d, v);
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = __fadd_rn(acc[j], v[j]);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = __fdiv_rn(acc[j], (float)kBlockN);
    }
    Vec<T>::store(kb + x * d + e, acc);
}

// Block means of a decode cache kc [B, n_max, d] (n_max a multiple of 64):
// block j of request b (rows 64 j .. 64 j + 63) to row b * (n_max / 64) + j
// of kbar, for blocks j >= first_block only (an update after appends), with
// the same arithmetic as block_mean_kernel.  Rows past a request's kv_len
// take part like any other: only the blocks below kv_len / 64 are ever read
// by the decode block scan.  One thread per 8 dimensions of one block row.
template <typename T>
__global__ void __launch_bounds__(kProxyThreads) decode_block_mean_kernel(const T *kc, int B, int n_max, int d,
                                                                          int first_block, T *kbar) {
    const int per_row = d / 8;
    const int nb = n_max >> kBlockShift, nu = nb - first_block;
    const long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (nu <= 0 || u >= (long long)B * nu * per_row) return;
    const long long x = u / per_row;  // (request, block) pair
    const int e = (int)(u - x * per_row) * 8;
    const int b = (int)(x / nu), j = first_block + (int)(x - (long long)b * nu);
    const T *src = kc + ((long long)b * n_max + (long long)j * kBlockN) * d + e;
    float acc[8], v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int r = 0; r < kBlockN; ++r) {
        Vec<T>::load(src + (long long)r * d, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], v[i]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = __fdiv_rn(acc[i], (float)kBlockN);
    Vec<T>::store(kbar + ((long long)b * nb + j) * d + e, acc);
}

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }

// Block summaries for the Quest bound ("Uncertainty-gated selection for
// block-sparse attention", Sec. 3.1, Eq. (2)): the per-dimension minimum and
// maximum of the 64 keys of block j of request b, to rows 2 (b * nb + j) and
// 2 (b * nb + j) + 1 of kq [B, nb, 2, d] (exact: they are keys), blocks j >=
// first_block only.  One thread per 8 dimensions of one block.
template <typename T>
__global__ void __launch_bounds__(kProxyThreads) decode_block_minmax_kernel(const T *kc, int B, int n_max, int d,
                                                                            int first_block, T *kq) {
    const int per_row = d / 8;
    const int nb = n_max >> kBlockShift, nu = nb - first_block;
    const long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (nu <= 0 || u >= (long long)B * nu * per_row) return;
    const long long x = u / per_row;
    const int e = (int)(u - x * per_row) * 8;
    const int b = (int)(x / nu), j = first_block + (int)(x - (long long)b * nu);
    const T *src = kc + ((long long)b * n_max + (long long)j * kBlockN) * d + e;
    float lo[8], hi[8], v[8];
    Vec<T>::load(src, lo);
#pragma unroll
    for (int i = 0; i < 8; ++i) hi[i] = lo[i];
    for (int r = 1; r < kBlockN; ++r) {
        Vec<T>::load(src + (long long)r * d, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            lo[i] = fminf(lo[i], v[i]);
            hi[i] = fmaxf(hi[i], v[i]);
        }
    }
    T *dst = kq + ((long long)b * nb + j) * 2 * d + e;
    Vec<T>::store(dst, lo);
    Vec<T>::store(dst + d, hi);
}

// Block scores by the Quest bound ("Uncertainty-gated selection for
// block-sparse attention", Sec. 3.1, Eq. (2)): for one proxy (qbar [H, d],
// wbar [H]) and each complete block j < nl of its request,
//     bound_h = sum_i max(q_hi * kmax_i, q_hi * kmin_i)   (i ascending, fp32)
//     score   = sum_h wbar_h * max(bound_h, 0)           (h ascending)
// to out[j].  max(q a, q b) with a >= b is q a for q >= 0 and q b otherwise,
// so the bound is accumulated as two FMAs with q+ = max(q, 0) and q- =
// min(q, 0) (the zero product adds nothing).  The proxy's q+ and q- sit in
// shared memory as fp32 (H * d * 8 bytes) and are read as broadcasts; each
// thread scores four blocks (kQuestPer), so every shared load feeds four
// blocks' FMAs and four independent FMA chains run per head, with heads in
// chunks of 16 whose partial bounds stay in registers.  kq holds the
// request's blocks from block 0: [*, 2, d] (kmin, kmax).
constexpr int kQuestThreads = 128;
constexpr int kQuestPer = 4;
constexpr int kQuestHeads = 16;  // heads per register chunk

template <typename T>
__device__ void quest_load_proxy(const T *qbar, int HD, float *qs) {
    for (int i = threadIdx.x; i < HD; i += blockDim.x) {
        const float v = to_float(qbar[i]);
        qs[i] = v > 0.0f ? v : 0.0f;
        qs[HD + i] = v < 0.0f ? v : 0.0f;
    }
}

template <typename T>
__device__ void quest_block_scores(const float *qs, const float *wbar, const T *kq, int nl, int j0, int H, int d,
                                   float *out) {
    const int HD = H * d;
    const T *row[kQuestPer];  // a block past nl repeats the first (not stored)
#pragma unroll
    for (int u = 0; u < kQuestPer; ++u) {
        const int j = j0 + u * kQuestThreads < nl ? j0 + u * kQuestThreads : j0;
        row[u] = kq + (long long)j * 2 * d;
    }
    float total[kQuestPer];
#pragma unroll
    for (int u = 0; u < kQuestPer; ++u) total[u] = 0.0f;
    for (int h0 = 0; h0 < H; h0 += kQuestHeads) {
        float acc[kQuestPer][kQuestHeads];
#pragma unroll
        for (int u = 0; u < kQuestPer; ++u)
#pragma unroll
            for (int hh = 0; hh < kQuestHeads; ++hh) acc[u][hh] = 0.0f;
        for (int e = 0; e < d; e += 8) {
            float lo[kQuestPer][8], hi[kQuestPer][8];
#pragma unroll
            for (int u = 0; u < kQuestPer; ++u) {
                Vec<T>::load(row[u] + e, lo[u]);
                Vec<T>::load(row[u] + d + e, hi[u]);
            }
#pragma unroll
            for (int hh = 0; hh < kQuestHeads; ++hh) {
                if (h0 + hh < H) {
                    const float4 *pp = reinterpret_cast<const float4 *>(qs + (h0 + hh) * d + e);
                    const float4 *pn = reinterpret_cast<const float4 *>(qs + HD + (h0 + hh) * d + e);
                    const float4 p0 = pp[0], p1 = pp[1], n0 = pn[0], n1 = pn[1];
                    const float qp[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
                    const float qn[8] = {n0.x, n0.y, n0.z, n0.w, n1.x, n1.y, n1.z, n1.w};
#pragma unroll
                    for (int u = 0; u < kQuestPer; ++u) {
                        float a = acc[u][hh];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            a = fmaf(qp[i], hi[u][i], a);
                            a = fmaf(qn[i], lo[u][i], a);
                        }
                        acc[u][hh] = a;
                    }
                }
            }
        }
#pragma unroll
        for (int hh = 0; hh < kQuestHeads; ++hh) {
            if (h0 + hh < H) {
                const float wh = wbar[h0 + hh];
#pragma unroll
                for (int u = 0; u < kQuestPer; ++u) total[u] = fmaf(wh, fmaxf(acc[u][hh], 0.0f), total[u]);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < kQuestPer; ++u)
        if (j0 + u * kQuestThreads < nl) out[j0 + u * kQuestThreads] = total[u];
}

// Decode: the proxy of request b against its complete blocks j < nlen[b];
// kq [B, nb, 2, d], scores to spill [b * nb + j].
template <typename T>
__global__ void __launch_bounds__(kQuestThreads, 3) decode_quest_scan_kernel(const T *qbar, const float *wbar,
                                                                          const T *kq, const int *nlen, int nb,
                                                                          int H, int d, float *spill) {
    extern __shared__ __align__(16) float qs[];  // [H][d] q+, then [H][d] q-
    const int b = blockIdx.x;  // request (grid x: no 65535 limit); block chunk on grid y
    const int j0 = blockIdx.y * (kQuestThreads * kQuestPer) + threadIdx.x;
    const int nl = nlen[b];
    if (blockIdx.y * (kQuestThreads * kQuestPer) >= nl) return;
    quest_load_proxy(qbar + (long long)b * H * d, H * d, qs);
    __syncthreads();
    if (j0 >= nl) return;
    quest_block_scores(qs, wbar + (long long)b * H, kq + (long long)b * nb * 2 * d, nl, j0, H, d,
                       spill + (long long)b * nb);
}

// Prefill block mode with the Quest bound: proxy row p (its request b, its
// group's last member t_last) against the complete blocks j < (t_last + 1) /
// 64 of its request; kq [T / 64, 2, d] with request b's blocks from row
// cu[b] / 64; scores to spill [(p - plan[6]) * ld + j] (the call's scratch
// rows, as the other per-row scratch).  One CTA per proxy walks all of its
// blocks, so the proxy is loaded into shared memory once.
template <typename T>
__global__ void __launch_bounds__(kQuestThreads, 3) prefill_quest_scan_kernel(const T *qbar, const float *wbar,
                                                                           const T *kq, const int *cu, int S,
                                                                           int g, const int *plan, PlanLayout pl,
                                                                           int H, int d, float *spill, long long ld) {
    extern __shared__ __align__(16) float qs[];
    // proxy row, the last first (a request's later proxies have the longer
    // prefixes, so the grid's tail holds the short ones)
    const int p = (int)(gridDim.x - 1 - blockIdx.x);
    if (!plan[0] || p >= plan[2] || !scored_in_range(plan, p)) return;
    const int *rp = plan + pl.rp();
    const int b = find_seg(rp, S, p);
    const int i = p - rp[b];
    const int n = cu[b + 1] - cu[b];
    const int tl = row_bound(i, n, g);
    const int nl = (tl + 1) >> kBlockShift;
    if (nl <= 0) return;
    quest_load_proxy(qbar + (long long)p * H * d, H * d, qs);
    __syncthreads();
    const T *kb = kq + (long long)(cu[b] >> kBlockShift) * 2 * d;
    float *out = spill + ((long long)p - plan[6]) * ld;
    for (int base = 0; base < nl; base += kQuestThreads * kQuestPer) {
        const int j0 = base + threadIdx.x;
        if (j0 < nl) quest_block_scores(qs, wbar + (long long)p * H, kb, nl, j0, H, d, out);
    }
}

// Prefill block summaries for the Quest bound: the per-dimension minimum and
// maximum of each complete block of each request, block i of request b to
// rows 2 x and 2 x + 1 of kq, x = (cu[b] >> 6) + i (as block_mean_kernel
// places its means); rows that belong to no complete block are zero.
template <typename T>
__global__ void __launch_bounds__(kProxyThreads) block_minmax_kernel(const T *k, const int *cu, int S, int T_,
                                                                     int d, long long nrows, T *kq) {
    const int per_row = d / 8;
    const long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= nrows * per_row) return;
    const long long x = u / per_row;
    const int e = (int)(u - x * per_row) * 8;
    int lo = 0, hi = S;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if ((long long)(cu[mid] >> kBlockShift) <= x) lo = mid; else hi = mid;
    }
    const long long i = x - (cu[lo] >> kBlockShift);
    const bool ok = cu[lo] >= 0 && cu[lo] <= cu[lo + 1] && cu[lo + 1] <= T_;
    const int nfull = ok ? (cu[lo + 1] - cu[lo]) >> kBlockShift : 0;
    float mn[8], mx[8], v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) mn[j] = mx[j] = 0.0f;
    if (i < nfull) {
        const T *src = k + ((long long)cu[lo] + i * kBlockN) * d + e;
        Vec<T>::load(src, mn);
#pragma unroll
        for (int j = 0; j < 8; ++j) mx[j] = mn[j];
        for (int r = 1; r < kBlockN; ++r) {
            Vec<T>::load(src + (long long)r * d, v);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                mn[j] = fminf(mn[j], v[j]);
                mx[j] = fmaxf(mx[j], v[j]);
            }
        }
    }
    Vec<T>::store(kq + x * 2 * d + e, mn);
    Vec<T>::store(kq + x * 2 * d + d + e, mx);
}

// Decode block mode: the complete blocks each request's proxy scans,
// kv_len[b] / 64 (0 for a request whose kv_len is out of range; the block
// select flags it).
__global__ void decode_block_len_kernel(const int *kv_len, int B, int G, int n_max, int *nlen) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    const int kv = kv_len[b];
    nlen[b] = (kv < G || kv > n_max) ? 0 : kv >> kBlockShift;
}

// Decode block mode: candidate set of request b from its selected blocks
// cblk [B, c / 64] (ascending, -1 padded) and the partial block that holds
// the last query (position kv_len[b] - 1), as block_expand_kernel does for
// a prefill proxy.
__global__ void __launch_bounds__(kProxyThreads) decode_block_expand_kernel(const int *kv_len, int G, int n_max,
                                                                            const int *cblk, int *cand, int c) {
    const int b = blockIdx.x;
    const int kv = kv_len[b];
    int *out = cand + (long long)b * c;
    const int nb = c >> kBlockShift;
    const bool ok = kv >= G && kv <= n_max;
    const int tl = kv - 1;
    const int part0 = (tl + 1) & ~(kBlockN - 1);
    const bool partial = ok && part0 <= tl;
    const int *sel = cblk + (long long)b * nb;
    for (int j = threadIdx.x; j < c; j += blockDim.x) {
        const int slot = j >> kBlockShift, r = j & (kBlockN - 1);
        int v = -1;
        if (ok) {
            if (partial && slot == nb - 1) {
                v = part0 + r <= tl ? part0 + r : -1;
            } else {
                const int blk = sel[slot];
                v = blk >= 0 ? blk * kBlockN + r : -1;
            }
        }
        out[j] = v;
    }
}

// Candidate set of each proxy row in block mode: slot j of cblk [R, nb]
// (a selected block, or -1) expands to the 64 positions of that block; the
// partial block that holds the proxy's last member t_last fills the last
// slot, which the block selection leaves empty whenever such a block exists.
__global__ void __launch_bounds__(kProxyThreads) block_expand_kernel(const int *cu, int S, int g, const int *plan,
                                                                     PlanLayout pl, const int *cblk, int *cand,
                                                                     int c) {
    const int p = blockIdx.x;
    // scratch rows (selected blocks, candidate sets) start at the call's
    // first scored row; a proxy with no output member has none
    if (!plan[0] || p >= plan[2] || !scored_in_range(plan, p)) return;
    const long long sp = (long long)p - plan[6];
    int *out = cand + sp * c;
    const int nb = c >> kBlockShift;
    const int *rp = plan + pl.rp();
    const int b = find_seg(rp, S, p);
    const int i = p - rp[b];
    const int n = cu[b + 1] - cu[b];
    const int tl = row_bound(i, n, g);
    const int part0 = (tl + 1) & ~(kBlockN - 1);
    const bool partial = part0 <= tl;
    const int *sel = cblk + sp * nb;
    for (int j = threadIdx.x; j < c; j += blockDim.x) {
        const int slot = j >> kBlockShift, r = j & (kBlockN - 1);
        int v;
        if (partial && slot == nb - 1) {
            v = part0 + r <= tl ? part0 + r : -1;
        } else {
            const int blk = sel[slot];
            v = blk >= 0 ? blk * kBlockN + r : -1;
        }
        out[j] = v;
    }
}

}  // namespace

cudaError_t launch_block_means(const void *k, const int *cu, int S, int T, int d, int dtype, void *kb,
                               cudaStream_t st) {
    const long long nrows = (T >> kBlockShift) > 0 ? (T >> kBlockShift) : 1;
    const long long units = nrows * (d / 8);
    TraceScope ts("block_means", st);
    const unsigned grid = (unsigned)((units + kProxyThreads - 1) / kProxyThreads);
    if (dtype == 1)
        block_mean_kernel<float><<<grid, kProxyThreads, 0, st>>>((const float *)k, cu, S, T, d, nrows,
                                                                 (float *)kb);
    else
        block_mean_kernel<__nv_bfloat16><<<grid, kProxyThreads, 0, st>>>(
            (const __nv_bfloat16 *)k, cu, S, T, d, nrows, (__nv_bfloat16 *)kb);
    return cudaGetLastError();
}

cudaError_t launch_block_expand(const int *cu, int S, int g, const int *plan, const PlanLayout &pl,
                                const int *cblk, int *cand, int c, int R, cudaStream_t st) {
    if (R <= 0) return cudaSuccess;
    TraceScope ts("block_expand", st);
    block_expand_kernel<<<R, kProxyThreads, 0, st>>>(cu, S, g, plan, pl, cblk, cand, c);
    return cudaGetLastError();
}

cudaError_t launch_proxy(const void *q, const float *w, const int *cu, int S, int T, int H, int d, int g,
                         int db, int dtype, const int *plan, const PlanLayout &pl, void *qbar, float *wbar,
                         int max_proxies, cudaStream_t st) {
    (void)T;
    if (max_proxies <= 0) return cudaSuccess;
    TraceScope ts("proxy", st);
    if (dtype == 1)
        proxy_kernel<float><<<max_proxies, kProxyThreads, 0, st>>>(
            (const float *)q, w, cu, S, H, d, g, db, plan, pl, (float *)qbar, wbar);
    else
        proxy_kernel<__nv_bfloat16><<<max_proxies, kProxyThreads, 0, st>>>(
            (const __nv_bfloat16 *)q, w, cu, S, H, d, g, db, plan, pl, (__nv_bfloat16 *)qbar, wbar);
    return cudaGetLastError();
}

cudaError_t launch_decode_block_means(const void *kc, int B, int n_max, int d, int dtype, int first_block,
                                      void *kbar, cudaStream_t st) {
    const int nu = (n_max >> kBlockShift) - first_block;
    if (B <= 0 || nu <= 0) return cudaSuccess;
    const long long units = (long long)B * nu * (d / 8);
    const unsigned grid = (unsigned)((units + kProxyThreads - 1) / kProxyThreads);
    TraceScope ts("block_means", st);
    if (dtype == 1)
        decode_block_mean_kernel<float><<<grid, kProxyThreads, 0, st>>>((const float *)kc, B, n_max, d, first_block,
                                                                        (float *)kbar);
    else
        decode_block_mean_kernel<__nv_bfloat16><<<grid, kProxyThreads, 0, st>>>(
            (const __nv_bfloat16 *)kc, B, n_max, d, first_block, (__nv_bfloat16 *)kbar);
    return cudaGetLastError();
}

cudaError_t launch_decode_block_minmax(const void *kc, int B, int n_max, int d, int dtype, int first_block,
                                       void *kq, cudaStream_t st) {
    const int nu = (n_max >> kBlockShift) - first_block;
    if (B <= 0 || nu <= 0) return cudaSuccess;
    const long long units = (long long)B * nu * (d / 8);
    const unsigned grid = (unsigned)((units + kProxyThreads - 1) / kProxyThreads);
    TraceScope ts("block_minmax", st);
    if (dtype == 1)
        decode_block_minmax_kernel<float><<<grid, kProxyThreads, 0, st>>>((const float *)kc, B, n_max, d,
                                                                          first_block, (float *)kq);
    else
        decode_block_minmax_kernel<__nv_bfloat16><<<grid, kProxyThreads, 0, st>>>(
            (const __nv_bfloat16 *)kc, B, n_max, d, first_block, (__nv_bfloat16 *)kq);
    return cudaGetLastError();
}

size_t quest_scan_smem(int H, int d) { return (size_t)H * d * 8; }

cudaError_t launch_decode_quest_scan(const void *qbar, const float *wbar, const void *kq, const int *nlen, int B,
                                     int nb, int H, int d, int dtype, float *spill, cudaStream_t st) {
    const size_t smem = quest_scan_smem(H, d);
    cudaError_t e = dtype == 1 ? cudaFuncSetAttribute(decode_quest_scan_kernel<float>,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
                               : cudaFuncSetAttribute(decode_quest_scan_kernel<__nv_bfloat16>,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int per_cta = kQuestThreads * kQuestPer;
    const dim3 grid((unsigned)B, (unsigned)((nb + per_cta - 1) / per_cta));
    TraceScope ts("quest_scan", st);
    if (dtype == 1)
        decode_quest_scan_kernel<float><<<grid, kQuestThreads, smem, st>>>((const float *)qbar, wbar,
                                                                           (const float *)kq, nlen, nb, H, d, spill);
    else
        decode_quest_scan_kernel<__nv_bfloat16><<<grid, kQuestThreads, smem, st>>>(
            (const __nv_bfloat16 *)qbar, wbar, (const __nv_bfloat16 *)kq, nlen, nb, H, d, spill);
    return cudaGetLastError();
}

cudaError_t launch_block_minmax(const void *k, const int *cu, int S, int T, int d, int dtype, void *kq,
                                cudaStream_t st) {
    const long long nrows = (T >> kBlockShift) > 0 ? (T >> kBlockShift) : 1;
    const long long units = nrows * (d / 8);
    TraceScope ts("block_minmax", st);
    const unsigned grid = (unsigned)((units + kProxyThreads - 1) / kProxyThreads);
    if (dtype == 1)
        block_minmax_kernel<float><<<grid, kProxyThreads, 0, st>>>((const float *)k, cu, S, T, d, nrows,
                                                                   (float *)kq);
    else
        block_minmax_kernel<__nv_bfloat16><<<grid, kProxyThreads, 0, st>>>((const __nv_bfloat16 *)k, cu, S, T, d,
                                                                           nrows, (__nv_bfloat16 *)kq);
    return cudaGetLastError();
}

cudaError_t launch_prefill_quest_scan(const void *qbar, const float *wbar, const void *kq, const int *cu, int S,
                                      int g, const int *plan, const PlanLayout &pl, int R, int nbmax, int H, int d,
                                      int dtype, float *spill, long long ld, cudaStream_t st) {
    if (R <= 0 || nbmax <= 0) return cudaSuccess;
    const size_t smem = quest_scan_smem(H, d);
    cudaError_t e = dtype == 1 ? cudaFuncSetAttribute(prefill_quest_scan_kernel<float>,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
                               : cudaFuncSetAttribute(prefill_quest_scan_kernel<__nv_bfloat16>,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)R;
    TraceScope ts("quest_scan", st);
    if (dtype == 1)
        prefill_quest_scan_kernel<float><<<grid, kQuestThreads, smem, st>>>(
            (const float *)qbar, wbar, (const float *)kq, cu, S, g, plan, pl, H, d, spill, ld);
    else
        prefill_quest_scan_kernel<__nv_bfloat16><<<grid, kQuestThreads, smem, st>>>(
            (const __nv_bfloat16 *)qbar, wbar, (const __nv_bfloat16 *)kq, cu, S, g, plan, pl, H, d, spill, ld);
    return cudaGetLastError();
}

cudaError_t launch_decode_block_len(const int *kv_len, int B, int G, int n_max, int *nlen, cudaStream_t st) {
    decode_block_len_kernel<<<(B + 127) / 128, 128, 0, st>>>(kv_len, B, G, n_max, nlen);
    return cudaGetLastError();
}

cudaError_t launch_decode_block_expand(const int *kv_len, int B, int G, int n_max, const int *cblk, int *cand,
                                       int c, cudaStream_t st) {
    TraceScope ts("block_expand", st);
    decode_block_expand_kernel<<<B, kProxyThreads, 0, st>>>(kv_len, G, n_max, cblk, cand, c);
    return cudaGetLastError();
}

cudaError_t launch_decode_proxy(const void *q, const float *w, int B, int G, int H, int d, int dtype,
                                void *qbar, float *wbar, cudaStream_t st) {
    TraceScope ts("proxy", st);
    if (dtype == 1)
        decode_proxy_kernel<float><<<B, kProxyThreads, 0, st>>>((const float *)q, w, G, H, d, (float *)qbar,
                                                                wbar);
    else
        decode_proxy_kernel<__nv_bfloat16><<<B, kProxyThreads, 0, st>>>(
            (const __nv_bfloat16 *)q, w, G, H, d, (__nv_bfloat16 *)qbar, wbar);
    return cudaGetLastError();
}

}  // namespace idx
