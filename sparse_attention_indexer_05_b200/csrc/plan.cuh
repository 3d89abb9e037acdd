// plan.cuh -- device helpers that map row blocks and rows to requests.
#pragma once

#include "internal.h"

namespace idx {

// first index i in a[0..n] (sorted, non-decreasing) with a[i] > v, minus 1:
// the last i with a[i] <= v (callers guarantee a[0] <= v < a[n]).
__device__ __forceinline__ int find_seg(const int *a, int n, long long v) {
    int lo = 0, hi = n;  // answer in [0, n-1]
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if ((long long)a[mid] <= v) lo = mid; else hi = mid;
    }
    return lo;
}

// Grouping of a request of n tokens into scored rows.  Groups are the
// request-local [m*g, min((m+1)*g, n)).  Under the guardrail (db > 0, the
// PIVOT page's dense fallback for short groups) every group whose last
// member's prefix holds at most db keys is not grouped: each of its members
// is a scored row of its own.  Those groups form a prefix of the request,
// its first dense_rows() tokens; the groups after it are unchanged, so
// scored row i is member i for i < nd and proxy i - nd of the rest.
__device__ __forceinline__ int dense_rows(int n, int g, int db) {
    if (db <= 0 || g == 1) return 0;
    return n <= db ? n : (db / g) * g;
}

// Number of scored rows of a request of n tokens: queries (g = 1) or proxies.
__device__ __forceinline__ int rows_of(int n, int g, int db = 0) {
    if (g == 1) return n;
    const int nd = dense_rows(n, g, db);
    return nd + (n - nd + g - 1) / g;
}

// First member (request-local) and member count of scored row i.
__device__ __forceinline__ int group_start(int i, int n, int g, int db = 0) {
    const int nd = dense_rows(n, g, db);
    return i < nd ? i : nd + (i - nd) * g;
}
__device__ __forceinline__ int group_size(int i, int n, int g, int db = 0) {
    const int nd = dense_rows(n, g, db);
    if (i < nd) return 1;
    const int lo = nd + (i - nd) * g;
    return (lo + g < n ? lo + g : n) - lo;
}

// Scored row that holds member t.
__device__ __forceinline__ int group_of(int t, int n, int g, int db = 0) {
    const int nd = dense_rows(n, g, db);
    return t < nd ? t : nd + (t - nd) / g;
}

// Causal bound (request-local, inclusive) of scored row i of a request of n
// tokens: a query sees s <= i; a proxy sees the prefix of its last member.
__device__ __forceinline__ int row_bound(int i, int n, int g, int db = 0) {
    if (g == 1) return i;
    const int nd = dense_rows(n, g, db);
    if (i < nd) return i;
    const long long e = nd + (long long)(i - nd + 1) * g;
    return (int)((e < n ? e : n) - 1);
}

// Does scored row i of request b (n tokens) have a member among the call's
// output rows [plan[4], plan[5]) (packed token rows)?  Rows without one are
// neither scored (unless their row block is) nor selected.
__device__ __forceinline__ bool row_in_range(const int *plan, const int *cu, int b, int i, int n, int g,
                                             int db = 0) {
    const long long lo = (long long)cu[b] + group_start(i, n, g, db);
    const long long hi = lo + group_size(i, n, g, db);
    return hi > plan[4] && lo < plan[5];
}

// Is scored row p one of the call's (a member in [row_lo, row_hi))?  Its
// per-row scratch then sits at row p - plan[6].
__device__ __forceinline__ bool scored_in_range(const int *plan, long long p) {
    return p >= plan[6] && p < plan[7];
}

struct BlockInfo {
    int b;        // request
    int row0;     // first scored row (global index into the scored tensor)
    int nrows;    // valid rows in the block (<= RB)
    long long key0;  // first key row of the request
    int n;        // request length
    int i0;       // request-local index of the first scored row
    int maxbound; // bound of the last valid row
    int ntiles;   // key tiles covering 0..maxbound
};

// Row bound in key units: keys are tokens (kshift = 0) or complete blocks of
// 2^kshift tokens (a row whose token bound is t sees the blocks that end at
// or before t); -1 when no key is visible.
__device__ __forceinline__ int key_bound(int t, int kshift) { return ((t + 1) >> kshift) - 1; }

__device__ __forceinline__ BlockInfo block_info(const int *plan, const PlanLayout &pl, const int *cu,
                                                int g, int blk, int kshift = 0, int db = 0) {
    BlockInfo bi;
    const int *rp = plan + pl.rp();
    const int *bp = plan + pl.bp();
    bi.b = find_seg(bp, pl.S, blk);
    const int j = blk - bp[bi.b];
    bi.n = cu[bi.b + 1] - cu[bi.b];
    const int R = rows_of(bi.n, g, db);
    bi.i0 = j * RB;
    bi.row0 = rp[bi.b] + bi.i0;
    int e = bi.i0 + RB;
    if (e > R) e = R;
    bi.nrows = e - bi.i0;
    bi.key0 = kshift ? (long long)(cu[bi.b] >> kshift) : (long long)cu[bi.b];
    bi.maxbound = key_bound(row_bound(e - 1, bi.n, g, db), kshift);
    bi.ntiles = bi.maxbound < 0 ? 1 : bi.maxbound / KT + 1;
    return bi;
}

}  // namespace idx
