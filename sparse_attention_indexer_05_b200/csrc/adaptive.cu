// adaptive.cu -- adaptive top-k budget from the cutoff margin
// ("Uncertainty-gated selection for block-sparse attention", Section 3
// Method, steps 3-5, and Appendix A, steps (A.5)-(A.9)), applied to the
// indexer's per-query scores.
//
// Input: the dense top-(rho k) of every row (ascending positions, -1 padded)
// with its fp32 scores, and each row's cutoff margin at k, which the final
// select computes from the same staged keys (select.cu, fast_margin: sigma =
// (s_(k-1) - s_(k)) / (s_(0) - s_(k)) in fp32, 0 when 0/0, NaN when the row
// has at most k positions; the ord of s_(k-1) and how many of its ties the
// top-k keeps).  Two launches here:
//   1. quantile (one CTA): tau = the ceil(q n)-th smallest defined sigma of the
//      call (q n in fp64), by a radix select over all rows;
//   2. finalize (one warp per row): trigger = sigma <= tau; rows that do not
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
    {
        TraceScope ts("quantile", st);
        adaptive_quantile_kernel<<<1, kTauThreads, 0, st>>>(a);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    TraceScope ts("finalize", st);
    adaptive_finalize_kernel<<<grid, kAdThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace idx
