// adaptive.cu -- adaptive top-k budget from the cutoff margin
// ("Uncertainty-gated selection for block-sparse attention", Section 3
// Method, steps 3-5, and Appendix A, steps (A.5)-(A.9)), applied to the
// indexer's per-query scores.
//
// Input: the dense top-(rho k) of every row (ascending positions, -1 padded)
// with its fp32 scores.  Three launches:
//   1. margin   (one CTA per row, keys in registers): s_(0), s_(k-1), s_(k)
//      of the row, s_(k-1) by a bitwise search over the orderable score bits
//      (32 block counts, no atomics); sigma =
//      (s_(k-1) - s_(k)) / (s_(0) - s_(k)) in fp32 (0 when 0/0, NaN when the
//      row has at most k positions); also the ord of s_(k-1) and how many of
//      its ties the top-k keeps (lowest positions first);
//   2. quantile (one CTA): tau = the ceil(q n)-th smallest defined sigma of the
//      call (q n in fp64), by the same radix select over all rows;
//   3. finalize (one warp per row): trigger = sigma <= tau; rows that do not
//      trigger are cut in place to their top-k (score desc, position asc),
//      still in ascending positions (ballot scans, no block barriers), and
//      padded with -1 / -inf to rho k.
// Every row's data is a few KB; the stage is small next to the score pass
// that produced its input.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace idx {

namespace {

constexpr int kAdThreads = 256;
constexpr int kAdWarps = kAdThreads / 32;
constexpr int kTauThreads = 1024;
constexpr int kTauWarps = kTauThreads / 32;

struct __align__(16) RadixSmem {
    unsigned hist[256];
    unsigned red[32];
    unsigned bcast[4];
};

// Block-wide sum / max of one value per thread (any block size up to 1024).
template <int NW>
__device__ __forceinline__ unsigned block_sum(unsigned v, unsigned *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    const int w = threadIdx.x >> 5;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[w] = v;
    __syncthreads();
    unsigned s = 0;
#pragma unroll
    for (int i = 0; i < NW; ++i) s += red[i];
    return s;
}
// The element of descending rank r (0-based) among the keys produced by
// key_of(i) for i < n (the key is valid when key_of returns true).  Returns
// its value; *gt = how many keys are strictly greater, *eq = how many equal.
template <int NT, int NW, class KeyOf>
__device__ unsigned radix_select_desc(int n, unsigned r, KeyOf key_of, RadixSmem &sm, unsigned *gt,
                                      unsigned *eq) {
    unsigned prefix = 0u, mask = 0u, rem = r, last_bin_count = 0u;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += NT) sm.hist[i] = 0u;
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += NT) {
            unsigned key;
            if (key_of(i, &key) && (key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 0xFFu], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            unsigned above = 0;
            const int b = warp_find_bin(sm.hist, rem + 1u, &above);
            if (threadIdx.x == 0) {
                sm.bcast[0] = (unsigned)b;
                sm.bcast[1] = above;
                sm.bcast[2] = b >= 0 ? sm.hist[b] : 0u;
            }
        }
        __syncthreads();
        const unsigned b = sm.bcast[0], above = sm.bcast[1];
        last_bin_count = sm.bcast[2];
        __syncthreads();
        rem -= above;
        prefix |= b << shift;
        mask |= 0xFFu << shift;
    }
    *gt = r - rem;
    *eq = last_bin_count;
    return prefix;
}

// Block-wide sum with one barrier: the two halves of red[] alternate between
// calls (parity p), so a call's writes never race the previous call's reads.
__device__ __forceinline__ unsigned block_sum1(unsigned v, unsigned (*red)[kAdWarps], int &p) {
    v = __reduce_add_sync(0xFFFFFFFFu, v);
    if ((threadIdx.x & 31) == 0) red[p][threadIdx.x >> 5] = v;
    __syncthreads();
    unsigned s = 0;
#pragma unroll
    for (int i = 0; i < kAdWarps; ++i) s += red[p][i];
    p ^= 1;
    return s;
}
__device__ __forceinline__ unsigned block_max1(unsigned v, unsigned (*red)[kAdWarps], int &p) {
    v = __reduce_max_sync(0xFFFFFFFFu, v);
    if ((threadIdx.x & 31) == 0) red[p][threadIdx.x >> 5] = v;
    __syncthreads();
    unsigned m = 0;
#pragma unroll
    for (int i = 0; i < kAdWarps; ++i) m = red[p][i] > m ? red[p][i] : m;
    p ^= 1;
    return m;
}

// Three block-wide sums with one barrier (same parity scheme, red3[p][c][w]).
__device__ __forceinline__ void block_sum3(unsigned &a0, unsigned &a1, unsigned &a2,
                                           unsigned (*red3)[3][kAdWarps], int &p) {
    a0 = __reduce_add_sync(0xFFFFFFFFu, a0);
    a1 = __reduce_add_sync(0xFFFFFFFFu, a1);
    a2 = __reduce_add_sync(0xFFFFFFFFu, a2);
    if ((threadIdx.x & 31) == 0) {
        red3[p][0][threadIdx.x >> 5] = a0;
        red3[p][1][threadIdx.x >> 5] = a1;
        red3[p][2][threadIdx.x >> 5] = a2;
    }
    __syncthreads();
    a0 = a1 = a2 = 0u;
#pragma unroll
    for (int i = 0; i < kAdWarps; ++i) {
        a0 += red3[p][0][i];
        a1 += red3[p][1][i];
        a2 += red3[p][2][i];
    }
    p ^= 1;
}

// One CTA per row; the row's orderable keys sit in registers (KPT per
// thread, 0 for padding, below every finite score's key).  s_(k-1) is the
// largest v with #{key >= v} >= k.  It lies between the row's smallest and
// largest key, so it shares their common leading bits; the bits below are
// found from the top, two per block count (three candidates, one barrier).
template <int KPT>
__global__ void __launch_bounds__(kAdThreads) adaptive_margin_kernel(AdaptiveArgs a) {
    __shared__ unsigned red[2][kAdWarps];
    __shared__ unsigned red3[2][3][kAdWarps];
    int p = 0, p3 = 0;
    const int W = a.width;
    const unsigned k = (unsigned)a.k;
    for (long long t = blockIdx.x; t < a.T; t += gridDim.x) {
        const int *ix = a.idx + t * W;
        const float *sc = a.score + t * W;
        unsigned key[KPT];
        unsigned cnt = 0u, mx = 0u, mn = 0xFFFFFFFFu;
        // both arrays are read unconditionally (in bounds for i < W), so
        // that all 2 KPT loads of a thread are in flight together
        int pos[KPT];
#pragma unroll
        for (int j = 0; j < KPT; ++j) {
            const int i = j * kAdThreads + threadIdx.x;
            pos[j] = i < W ? ix[i] : -1;
            key[j] = i < W ? __float_as_uint(sc[i]) : 0u;
        }
#pragma unroll
        for (int j = 0; j < KPT; ++j) {
            key[j] = pos[j] >= 0 ? score_ord(__uint_as_float(key[j])) : 0u;
            if (key[j] != 0u) {
                ++cnt;
                mx = key[j] > mx ? key[j] : mx;
                mn = key[j] < mn ? key[j] : mn;
            }
        }
        const unsigned n = block_sum1(cnt, red, p);
        mx = block_max1(mx, red, p);
        mn = ~block_max1(~mn, red, p);
        if (n < k + 1u) {
            if (threadIdx.x == 0) {
                a.sigma[t] = __uint_as_float(0x7FC00000u);  // quiet NaN: no (k+1)-th score
                a.vk[t] = 0u;
                a.need[t] = 0;
            }
            continue;
        }
        unsigned v = mx;  // all keys equal: s_(k-1) = the key
        if (mn != mx) {
            int bit = 31 - __clz(mn ^ mx);  // highest bit where the keys differ
            v = mx & ~((2u << bit) - 1u);   // common leading bits, zeros below: #{key >= v} = n >= k
            for (; bit >= 1; bit -= 2) {
                const unsigned c1 = v | (1u << (bit - 1)), c2 = v | (2u << (bit - 1)), c3 = v | (3u << (bit - 1));
                unsigned n1 = 0u, n2 = 0u, n3 = 0u;
#pragma unroll
                for (int j = 0; j < KPT; ++j) {
                    n1 += key[j] >= c1 ? 1u : 0u;
                    n2 += key[j] >= c2 ? 1u : 0u;
                    n3 += key[j] >= c3 ? 1u : 0u;
                }
                block_sum3(n1, n2, n3, red3, p3);
                v = n3 >= k ? c3 : (n2 >= k ? c2 : (n1 >= k ? c1 : v));
            }
            if (bit == 0) {
                const unsigned cand = v | 1u;
                unsigned c = 0u;
#pragma unroll
                for (int j = 0; j < KPT; ++j) c += key[j] >= cand ? 1u : 0u;
                if (block_sum1(c, red, p) >= k) v = cand;
            }
        }
        const unsigned v1 = v;  // s_(k-1)
        unsigned gt = 0u, eq = 0u;
#pragma unroll
        for (int j = 0; j < KPT; ++j) {
            gt += key[j] > v1 ? 1u : 0u;
            eq += key[j] == v1 ? 1u : 0u;
        }
        gt = block_sum1(gt, red, p);
        eq = block_sum1(eq, red, p);
        unsigned v2 = v1;  // s_(k): a tie of s_(k-1) if one is left over, else the largest key below it
        if (gt + eq < k + 1u) {
            unsigned below = 0u;
#pragma unroll
            for (int j = 0; j < KPT; ++j) below = (key[j] < v1 && key[j] > below) ? key[j] : below;
            v2 = block_max1(below, red, p);
        }
        if (threadIdx.x == 0) {
            const float f0 = ord_score(mx), f1 = ord_score(v1), f2 = ord_score(v2);
            const float num = f1 - f2, den = f0 - f2;
            a.sigma[t] = den > 0.0f ? num / den : 0.0f;
            a.vk[t] = v1;
            a.need[t] = (int)(k - gt);
        }
    }
}

__global__ void __launch_bounds__(kTauThreads) adaptive_quantile_kernel(AdaptiveArgs a) {
    __shared__ RadixSmem sm;
    unsigned cnt = 0u;
    for (long long t = threadIdx.x; t < a.T; t += kTauThreads) cnt += isnan(a.sigma[t]) ? 0u : 1u;
    const unsigned n = block_sum<kTauWarps>(cnt, sm.red);
    double rq = ceil(a.q * (double)n);
    if (rq > (double)n) rq = (double)n;
    const unsigned r = rq > 0.0 ? (unsigned)rq : 0u;
    if (r == 0u) {
        if (threadIdx.x == 0) {
            a.tau[0] = 0u;
            a.tau[1] = 0u;
        }
        return;
    }
    // the r-th smallest = descending rank n - r; sigma >= +0, so its ord is monotone
    auto key_of = [&](int i, unsigned *key) {
        const float s = a.sigma[i];
        *key = score_ord(s);
        return !isnan(s);
    };
    unsigned gt = 0u, eq = 0u;
    const unsigned v = radix_select_desc<kTauThreads, kTauWarps>(a.T, n - r, key_of, sm, &gt, &eq);
    if (threadIdx.x == 0) {
        a.tau[0] = 1u;
        a.tau[1] = v;
    }
}

__global__ void __launch_bounds__(kAdThreads) adaptive_finalize_kernel(AdaptiveArgs a) {
    const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = a.width;
    const bool has_tau = a.tau[0] != 0u;
    const unsigned tau = a.tau[1];
    for (long long t = (long long)blockIdx.x * kAdWarps + wid; t < a.T; t += (long long)gridDim.x * kAdWarps) {
        const float sg = a.sigma[t];
        const bool defined = !isnan(sg);
        const bool trig = defined && has_tau && score_ord(sg) <= tau;
        if (lane == 0 && a.trigger) a.trigger[t] = trig ? 1 : 0;
        if (!defined || trig) continue;  // whole prefix (<= k) or the full rho k stay
        int *ix = a.idx + t * W;
        float *sc = a.score + t * W;
        const unsigned v1 = a.vk[t];
        const unsigned need = (unsigned)a.need[t];
        const unsigned lt = lanemask_lt();
        unsigned eq_before = 0u, kept = 0u;
        constexpr int U = 4;  // chunks of 32 read ahead of their ballots
        for (int base = 0; base < W && kept < (unsigned)a.k; base += 32 * U) {
            float s[U];
            int p[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = base + u * 32 + lane;
                p[u] = i < W ? ix[i] : -1;
                s[u] = i < W ? sc[i] : 0.0f;  // not conditional on p[u]: the loads go out together
            }
            // writes go to positions below every entry still to be read
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const bool valid = p[u] >= 0;
                const unsigned o = valid ? score_ord(s[u]) : 0u;
                const bool is_eq = valid && o == v1;
                const unsigned meq = __ballot_sync(0xFFFFFFFFu, is_eq);
                const bool keep = valid && (o > v1 || (is_eq && eq_before + __popc(meq & lt) < need));
                const unsigned mk = __ballot_sync(0xFFFFFFFFu, keep);
                if (keep) {
                    const unsigned pos = kept + __popc(mk & lt);
                    ix[pos] = p[u];
                    sc[pos] = s[u];
                }
                eq_before += __popc(meq);
                kept += __popc(mk);
            }
        }
        __syncwarp();
        for (int i = (int)kept + lane; i < W; i += 32) {
            ix[i] = -1;
            sc[i] = -INFINITY;
        }
        if (lane == 0 && kept != (unsigned)a.k) raise_status(a.status, ST_OVERFLOW);
    }
}

}  // namespace

cudaError_t launch_adaptive(const AdaptiveArgs &a, cudaStream_t st) {
    if (a.T <= 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long blocks = (a.T + kAdWarps - 1) / kAdWarps, cap = (long long)sms * 8;
    const unsigned grid = (unsigned)(blocks < cap ? blocks : cap);
    const int kpt = (a.width + kAdThreads - 1) / kAdThreads;
    const unsigned mgrid = (unsigned)(a.T < cap ? a.T : cap);
    {
        TraceScope ts("margin", st);
        if (kpt <= 4)
            adaptive_margin_kernel<4><<<mgrid, kAdThreads, 0, st>>>(a);
        else if (kpt <= 8)
            adaptive_margin_kernel<8><<<mgrid, kAdThreads, 0, st>>>(a);
        else if (kpt <= 16)
            adaptive_margin_kernel<16><<<mgrid, kAdThreads, 0, st>>>(a);
        else if (kpt <= 32)
            adaptive_margin_kernel<32><<<mgrid, kAdThreads, 0, st>>>(a);
        else
            return cudaErrorInvalidValue;  // rho * k above 8192: rejected on the host first
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    {
        TraceScope ts("quantile", st);
        adaptive_quantile_kernel<<<1, kTauThreads, 0, st>>>(a);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    TraceScope ts("finalize", st);
    adaptive_finalize_kernel<<<grid, kAdThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace idx
