// adaptive.cu -- adaptive top-k budget from the cutoff margin ("Read the
// Cutoff", the sparse-attention router page: Section 3, steps 3-5, and
// Appendix A, steps (A.5)-(A.9)), applied to the indexer's per-query scores.
//
// Input: the dense top-(rho k) of every row (ascending positions, -1 padded)
// with its fp32 scores.  Three launches:
//   1. margin   (one CTA per row): s_(0), s_(k-1), s_(k) of the row by an
//      8-bit radix select over the orderable score bits; sigma =
//      (s_(k-1) - s_(k)) / (s_(0) - s_(k)) in fp32 (0 when 0/0, NaN when the
//      row has at most k positions); also the ord of s_(k-1) and how many of
//      its ties the top-k keeps (lowest positions first);
//   2. quantile (one CTA): tau = the ceil(q n)-th smallest defined sigma of the
//      call (q n in fp64), by the same radix select over all rows;
//   3. finalize (one CTA per row): trigger = sigma <= tau; rows that do not
//      trigger are cut in place to their top-k (score desc, position asc),
//      still in ascending positions, and padded with -1 / -inf to rho k.
// Every row's data is a few KB, read from L2; the whole stage is small next
// to the score pass that produced its input.
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
template <int NW>
__device__ __forceinline__ unsigned block_max(unsigned v, unsigned *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned u = __shfl_xor_sync(0xFFFFFFFFu, v, o);
        v = u > v ? u : v;
    }
    const int w = threadIdx.x >> 5;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[w] = v;
    __syncthreads();
    unsigned m = 0;
#pragma unroll
    for (int i = 0; i < NW; ++i) m = red[i] > m ? red[i] : m;
    return m;
}

// Exclusive prefix sum of a 0/1 flag over the block, plus the block total.
template <int NW>
__device__ __forceinline__ unsigned block_excl_scan(unsigned f, unsigned *red, unsigned *total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const unsigned m = __ballot_sync(0xFFFFFFFFu, f != 0u);
    const unsigned in_warp = __popc(m & lanemask_lt());
    __syncthreads();
    if (lane == 0) red[w] = __popc(m);
    __syncthreads();
    unsigned before = 0, all = 0;
#pragma unroll
    for (int i = 0; i < NW; ++i) {
        before += i < w ? red[i] : 0u;
        all += red[i];
    }
    *total = all;
    return before + in_warp;
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

__global__ void __launch_bounds__(kAdThreads) adaptive_margin_kernel(AdaptiveArgs a) {
    __shared__ RadixSmem sm;
    const int W = a.width;
    for (long long t = blockIdx.x; t < a.T; t += gridDim.x) {
        const int *ix = a.idx + t * W;
        const float *sc = a.score + t * W;
        unsigned cnt = 0u, mx = 0u;
        for (int i = threadIdx.x; i < W; i += kAdThreads) {
            if (ix[i] >= 0) {
                ++cnt;
                const unsigned o = score_ord(sc[i]);
                mx = o > mx ? o : mx;
            }
        }
        const unsigned n = block_sum<kAdWarps>(cnt, sm.red);
        mx = block_max<kAdWarps>(mx, sm.red);
        if (n < (unsigned)a.k + 1u) {
            if (threadIdx.x == 0) {
                a.sigma[t] = __uint_as_float(0x7FC00000u);  // quiet NaN: no (k+1)-th score
                a.vk[t] = 0u;
                a.need[t] = 0;
            }
            __syncthreads();
            continue;
        }
        // valid entries are the first n (the select pads at the end)
        auto key_of = [&](int i, unsigned *key) {
            *key = score_ord(sc[i]);
            return true;
        };
        unsigned gt = 0u, eq = 0u;
        const unsigned v1 = radix_select_desc<kAdThreads, kAdWarps>((int)n, (unsigned)a.k - 1u, key_of, sm, &gt, &eq);
        unsigned v2 = v1;  // s_(k): a tie of s_(k-1) if one is left over, else the largest key below it
        if (gt + eq < (unsigned)a.k + 1u) {
            unsigned below = 0u;
            for (int i = threadIdx.x; i < (int)n; i += kAdThreads) {
                const unsigned o = score_ord(sc[i]);
                if (o < v1 && o > below) below = o;
            }
            v2 = block_max<kAdWarps>(below, sm.red);
        }
        if (threadIdx.x == 0) {
            const float f0 = ord_score(mx), f1 = ord_score(v1), f2 = ord_score(v2);
            const float num = f1 - f2, den = f0 - f2;
            a.sigma[t] = den > 0.0f ? num / den : 0.0f;
            a.vk[t] = v1;
            a.need[t] = a.k - (int)gt;
        }
        __syncthreads();
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
    __shared__ RadixSmem sm;
    const int W = a.width;
    const bool has_tau = a.tau[0] != 0u;
    const unsigned tau = a.tau[1];
    for (long long t = blockIdx.x; t < a.T; t += gridDim.x) {
        const float sg = a.sigma[t];
        const bool defined = !isnan(sg);
        const bool trig = defined && has_tau && score_ord(sg) <= tau;
        if (threadIdx.x == 0 && a.trigger) a.trigger[t] = trig ? 1 : 0;
        if (!defined || trig) continue;  // whole prefix (<= k) or the full rho k stay
        int *ix = a.idx + t * W;
        float *sc = a.score + t * W;
        const unsigned v1 = a.vk[t];
        const unsigned need = (unsigned)a.need[t];
        unsigned eq_before = 0u, kept = 0u;
        for (int base = 0; base < W; base += kAdThreads) {
            const int i = base + threadIdx.x;
            const bool valid = i < W && ix[i] >= 0;
            const float s = valid ? sc[i] : 0.0f;
            const int p = valid ? ix[i] : -1;
            const unsigned o = valid ? score_ord(s) : 0u;
            const bool is_eq = valid && o == v1;
            unsigned eq_total = 0u;
            const unsigned eq_rank = eq_before + block_excl_scan<kAdWarps>(is_eq ? 1u : 0u, sm.red, &eq_total);
            const bool keep = valid && (o > v1 || (is_eq && eq_rank < need));
            unsigned keep_total = 0u;
            const unsigned pos = kept + block_excl_scan<kAdWarps>(keep ? 1u : 0u, sm.red, &keep_total);
            __syncthreads();  // every read of this chunk precedes the writes (pos <= i)
            if (keep) {
                ix[pos] = p;
                sc[pos] = s;
            }
            eq_before += eq_total;
            kept += keep_total;
        }
        __syncthreads();
        for (int i = (int)kept + threadIdx.x; i < W; i += kAdThreads) {
            ix[i] = -1;
            sc[i] = -INFINITY;
        }
        if (threadIdx.x == 0 && kept != (unsigned)a.k) raise_status(a.status, ST_OVERFLOW);
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_adaptive(const AdaptiveArgs &a, cudaStream_t st) {
    if (a.T <= 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long cap = (long long)sms * 8;
    const unsigned grid = (unsigned)(a.T < cap ? a.T : cap);
    {
        TraceScope ts("margin", st);
        adaptive_margin_kernel<<<grid, kAdThreads, 0, st>>>(a);
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
