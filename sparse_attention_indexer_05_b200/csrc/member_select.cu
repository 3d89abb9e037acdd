// member_select.cu -- the top-k of Refine member rows: a member's c scores
// over its group's candidate list (ascending positions, -1 = none), masked to
// positions <= the member's own, prefill and decode alike.
//
// One CTA of 128 threads per row, up to ten CTAs an SM (48 registers).  A row needs only
// the scores' ords: its candidates' positions ascend with their index, so
// among equal scores the lower position is the lower index, and the top-k
// by (score, then lower position) is
//     every entry with ord > V, plus the first `need` entries with ord == V
// (V the k-th largest ord, `need` = k minus the entries above V).
//   1. the valid entries' ords go to shared memory (0 marks an invalid slot:
//      no arithmetic result has ord 0), with their count and range;
//   2. V by a radix over ord - lo: a first 10-bit digit spanning [lo, hi]
//      exactly, then 8-bit digits inside the k-th entry's bin, until a bin is
//      all selected or V is exact;
//   3. an ordered compaction: each warp counts its part's entries above V and
//      equal to V, a block scan gives each part's offsets, and every selected
//      entry writes its position (and score) at
//          (entries above V before it) + min(entries equal to V before it, need).
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "plan.cuh"

namespace idx {

namespace {

constexpr int kMT = 128;               // threads per CTA
constexpr int kMWarps = kMT / 32;
constexpr int kMBits = 10;             // first radix digit
constexpr int kMBins = 1 << kMBits;
constexpr int kMemberMaxC = 12288;     // candidates a row keeps in shared memory (48 KB of ords)

struct __align__(16) MemShared {
    unsigned hist[kMBins];
    unsigned wtot[kMWarps];
    unsigned wgt[kMWarps], weq[kMWarps];
    unsigned lo, hi, nv;
    int dgt;
    unsigned above, inbin;
};

// Block-wide: over hist[0..nbins) (nbins = per * kMT), the largest bin b with
// sum(hist[b..]) >= need; writes b (-1 if none), the sum above it and its
// count to sh.
template <int per>
__device__ void member_find_bin(MemShared &sh, unsigned need) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b0 = tid * per;
    unsigned loc[per];
    unsigned sum = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) {
        loc[i] = sh.hist[b0 + i];
        sum += loc[i];
    }
    unsigned suf = sum;  // inclusive suffix over the warp's threads
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned v = __shfl_down_sync(0xFFFFFFFFu, suf, o);
        if (lane + o < 32) suf += v;
    }
    if (lane == 0) sh.wtot[warp] = suf;
    if (tid == 0) sh.dgt = -1;
    __syncthreads();
    unsigned after = 0;
#pragma unroll
    for (int w = 0; w < kMWarps; ++w) after += w > warp ? sh.wtot[w] : 0u;
    suf += after;
    if (suf >= need && suf - sum < need) {
        unsigned run = suf - sum;
        for (int i = per - 1; i >= 0; --i) {
            if (run + loc[i] >= need) {
                sh.dgt = b0 + i;
                sh.above = run;
                sh.inbin = loc[i];
                break;
            }
            run += loc[i];
        }
    }
    __syncthreads();
}

// One member row: its scores and candidate positions, its bound, its output.
struct MemRow {
    bool active;   // this kernel selects the row
    bool invalid;  // decode kv_len out of range: -1 row, status raised
    const float *sc;
    const int *pos;
    int c, bound;
};

__device__ MemRow member_row(const SelectArgs &a, int row) {
    MemRow r{};
    if (a.kind == SEL_DEC_MEMBER) {
        const int b = row / a.G, m = row % a.G;
        const int kv = a.kv_len[b];
        if (kv < a.G || kv > a.n_max) {
            r.invalid = true;
            return r;
        }
        r.active = true;
        r.sc = a.scores + (long long)row * a.ld;
        r.pos = a.cand + (long long)b * a.c;
        r.c = a.c;
        r.bound = kv - a.G + m;
        return r;
    }
    // SEL_MEMBER_SCORES: output rows of the call whose member is not scored on
    // its own (the guardrail's rows take the candidate-buffer select)
    if (row < a.plan[4] || row >= a.plan[5]) return r;
    const int b = find_seg(a.cu, a.S, row);
    const int t = row - a.cu[b];
    const int n = a.cu[b + 1] - a.cu[b];
    if (t < dense_rows(n, a.g, a.db)) return r;
    const int p = a.plan[a.pl.rp() + b] + group_of(t, n, a.g, a.db);
    r.active = true;
    r.sc = a.scores + ((long long)row - a.plan[8]) * a.ld;
    r.pos = a.cand + ((long long)p - a.plan[6]) * a.c;
    r.c = a.c;
    r.bound = t;
    return r;
}

__device__ __forceinline__ void member_pad(int from, int k, int *oi, float *os) {
    for (int i = from + (int)threadIdx.x; i < k; i += kMT) {
        oi[i] = -1;
        if (os) os[i] = -INFINITY;
    }
}

// Step 1 for one candidate: its ord (0 when invalid) and the range counters.
__device__ __forceinline__ unsigned member_ord(float s, int p, int bound, unsigned &mn, unsigned &mx, unsigned &cnt) {
    if (p < 0 || p > bound) return 0u;
    const unsigned o = score_ord(s);
    mn = o < mn ? o : mn;
    mx = o > mx ? o : mx;
    ++cnt;
    return o;
}

__global__ void __launch_bounds__(kMT, 10) member_select_kernel(SelectArgs a) {
    extern __shared__ __align__(16) unsigned mem_ords[];
    __shared__ MemShared sh;
    const int row = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = a.k;
    int *oi = a.out_idx + (long long)row * k;
    float *os = a.out_score ? a.out_score + (long long)row * k : nullptr;
    if (a.kind == SEL_MEMBER_SCORES && !a.plan[0]) {  // the call's inputs failed the device checks
        member_pad(0, k, oi, os);
        return;
    }
    const MemRow r = member_row(a, row);
    if (r.invalid) {
        if (tid == 0) raise_status(a.status, ST_INVALID);
        member_pad(0, k, oi, os);
        return;
    }
    if (!r.active) return;
    const int c = r.c;
    if (tid == 0) {
        sh.lo = 0xFFFFFFFFu;
        sh.hi = 0u;
        sh.nv = 0u;
    }
    __syncthreads();

    // 1. ords of the valid candidates (four runs of 4 per thread in flight
    // when the rows are 16-byte aligned)
    unsigned mn = 0xFFFFFFFFu, mx = 0u, cnt = 0u;
    const bool vec = (c & 3) == 0 &&
                     ((reinterpret_cast<uintptr_t>(r.sc) | reinterpret_cast<uintptr_t>(r.pos)) & 15u) == 0;
    if (vec) {
        const int n4 = c >> 2;
        const float4 *s4 = reinterpret_cast<const float4 *>(r.sc);
        const int4 *p4 = reinterpret_cast<const int4 *>(r.pos);
        for (int i0 = tid; i0 < n4; i0 += 4 * kMT) {
            float4 sv[4];
            int4 pv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * kMT;
                sv[u] = i < n4 ? s4[i] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                pv[u] = i < n4 ? p4[i] : make_int4(-1, -1, -1, -1);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * kMT;
                if (i < n4) {
                    uint4 o;
                    o.x = member_ord(sv[u].x, pv[u].x, r.bound, mn, mx, cnt);
                    o.y = member_ord(sv[u].y, pv[u].y, r.bound, mn, mx, cnt);
                    o.z = member_ord(sv[u].z, pv[u].z, r.bound, mn, mx, cnt);
                    o.w = member_ord(sv[u].w, pv[u].w, r.bound, mn, mx, cnt);
                    reinterpret_cast<uint4 *>(mem_ords)[i] = o;
                }
            }
        }
    } else {
        for (int i = tid; i < c; i += kMT) mem_ords[i] = member_ord(r.sc[i], r.pos[i], r.bound, mn, mx, cnt);
    }
    mn = __reduce_min_sync(0xFFFFFFFFu, mn);
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    cnt = __reduce_add_sync(0xFFFFFFFFu, cnt);
    if (lane == 0 && cnt) {
        atomicMin(&sh.lo, mn);
        atomicMax(&sh.hi, mx);
        atomicAdd(&sh.nv, cnt);
    }
    __syncthreads();
    const unsigned nv = sh.nv, lo = sh.lo, hi = sh.hi;

    // 2. the k-th largest ord V and how many entries equal to it are taken
    unsigned V = 0u, need_eq = 0u;  // nv <= k: every valid entry (ord > 0)
    if (nv > (unsigned)k) {
        const unsigned span = hi - lo;
        const int bl = 32 - __clz(span);
        int s = bl > kMBits ? bl - kMBits : 0;  // first digit (ord - lo) >> s < 1024
        for (int i = tid; i < kMBins; i += kMT) sh.hist[i] = 0u;
        __syncthreads();
        for (int j = tid; j < c; j += kMT) {
            const unsigned o = mem_ords[j];
            if (o) atomicAdd(&sh.hist[(o - lo) >> s], 1u);
        }
        __syncthreads();
        member_find_bin<kMBins / kMT>(sh, (unsigned)k);
        unsigned need = (unsigned)k - sh.above;
        unsigned prefix = (unsigned)sh.dgt << s, mask = 0xFFFFFFFFu << s;
        bool closed = sh.inbin == need;
        while (!closed && s > 0) {
            const int bits = s >= 8 ? 8 : s;
            s -= bits;
            const unsigned dm = (1u << bits) - 1u;
            for (int i = tid; i < 256; i += kMT) sh.hist[i] = 0u;
            __syncthreads();
            for (int j = tid; j < c; j += kMT) {
                const unsigned o = mem_ords[j];
                if (o && ((o - lo) & mask) == prefix) atomicAdd(&sh.hist[((o - lo) >> s) & dm], 1u);
            }
            __syncthreads();
            member_find_bin<256 / kMT>(sh, need);
            need -= sh.above;
            prefix |= (unsigned)sh.dgt << s;
            mask |= dm << s;
            closed = sh.inbin == need;
        }
        if (closed) {  // everything from the bin's lower edge: ord > edge - 1
            V = lo + prefix - 1u;
            need_eq = 0u;
        } else {  // s == 0: the bin is the single ord V, `need` of its entries taken
            V = lo + prefix;
            need_eq = need;
        }
    }

    // 3. ordered compaction, each warp over a contiguous part of the row
    const int wseg = ((c + kMWarps - 1) / kMWarps + 31) & ~31;
    const int j0 = warp * wseg, j1 = j0 + wseg < c ? j0 + wseg : c;
    unsigned ngt = 0u, neq = 0u;
    for (int j = j0; j < j1; j += 32) {
        const int jj = j + lane;
        const unsigned o = jj < j1 ? mem_ords[jj] : 0u;
        ngt += __popc(__ballot_sync(0xFFFFFFFFu, o > V));
        neq += __popc(__ballot_sync(0xFFFFFFFFu, o != 0u && o == V));
    }
    if (lane == 0) {
        sh.wgt[warp] = ngt;
        sh.weq[warp] = neq;
    }
    __syncthreads();
    unsigned gt_run = 0u, eq_run = 0u, gt_all = 0u, eq_all = 0u;
#pragma unroll
    for (int w = 0; w < kMWarps; ++w) {
        gt_run += w < warp ? sh.wgt[w] : 0u;
        eq_run += w < warp ? sh.weq[w] : 0u;
        gt_all += sh.wgt[w];
        eq_all += sh.weq[w];
    }
    for (int j = j0; j < j1; j += 32) {
        const int jj = j + lane;
        const unsigned o = jj < j1 ? mem_ords[jj] : 0u;
        const bool gt = o > V, eq = o != 0u && o == V;
        const unsigned gm = __ballot_sync(0xFFFFFFFFu, gt), em = __ballot_sync(0xFFFFFFFFu, eq);
        const unsigned er = eq_run + __popc(em & lanemask_lt());
        if (gt || (eq && er < need_eq)) {
            const unsigned rank = gt_run + __popc(gm & lanemask_lt()) + (er < need_eq ? er : need_eq);
            if (rank < (unsigned)k) {  // never past the row
                oi[rank] = r.pos[jj];
                if (os) os[rank] = ord_score(o);
            }
        }
        gt_run += __popc(gm);
        eq_run += __popc(em);
    }
    const unsigned nsel = gt_all + (eq_all < need_eq ? eq_all : need_eq);
    member_pad((int)(nsel < (unsigned)k ? nsel : (unsigned)k), k, oi, os);
}

}  // namespace

// Decode calls with few member rows keep select_fast_kernel's 256 threads a
// row: 128 rows of 128-thread CTAs leave the GPU emptier (0.082 against
// 0.076 ms for the 64 x 2 rows of the decode bench step).
bool member_select_fits(const SelectArgs &a) {
    if (a.c <= 0 || a.c > kMemberMaxC) return false;
    return a.kind == SEL_MEMBER_SCORES || (a.kind == SEL_DEC_MEMBER && a.nrows >= 1024);
}

cudaError_t launch_member_select(const SelectArgs &a, cudaStream_t st) {
    if (a.nrows <= 0) return cudaSuccess;
    const size_t smem = ((size_t)a.c * 4 + 15) & ~(size_t)15;
    cudaError_t e = cudaFuncSetAttribute(member_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    TraceScope ts("select", st);
    member_select_kernel<<<a.nrows, kMT, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace idx
