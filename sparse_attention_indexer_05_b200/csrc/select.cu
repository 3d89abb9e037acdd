// select.cu -- exact final top-k of one row per CTA.
//
// The entries of a row (candidate keys from a score pass, or dense fp32
// scores) are ranked by key = (ord(score) << 32) | (0xFFFFFFFF - s), so the
// top-k is "highest score first, ties to the lower position".  An MSB-first
// radix select with 8-bit digits finds the k-th largest key K; the selected
// positions (key >= K) are marked in a shared bitmap over 0..bound, and
// each selected entry writes itself at its rank among the marked bits,
// which lists the top-k in ascending position without a sort.
#include <math.h>

#include "common.cuh"
#include "plan.cuh"

namespace idx {

namespace {

constexpr int kSelThreads = 512;

struct CandSrc {
    const unsigned long long *buf;
    int n;
    int bound;
    __device__ unsigned long long key(int i) const {
        const unsigned long long kk = buf[i];
        return key_pos(kk) <= bound ? kk : 0ull;
    }
};

struct ScoreSrc {
    const float *sc;
    const int *pos;  // NULL: position = i
    int n;
    int bound;
    __device__ unsigned long long key(int i) const {
        const int p = pos ? pos[i] : i;
        if (p < 0 || p > bound) return 0ull;
        return make_key(score_ord(sc[i]), p);
    }
};

__device__ unsigned block_sum(unsigned v, unsigned *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    unsigned t = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    __syncthreads();
    return t;
}

constexpr int kMaxBins = 4096;  // widest radix digit: 12 bits

struct SelShared {
    unsigned hist[kMaxBins];
    unsigned red[32];
    unsigned red2[32];
    int dgt;
    unsigned above;
    unsigned inbin;
};

// Digits of the 64-bit key, most significant first: 12 + 12 + 8 bits of the
// score's ord (the first digit separates exponents, so the k-th key's bin is
// already narrow), then 12 + 12 + 8 bits of the position part (ties only).
__device__ __forceinline__ int digit_bits(int pass) { return (pass % 3 == 2) ? 8 : 12; }

// Block-wide: the largest bin b of hist[0..nbins) with sum(hist[b..]) >= need;
// writes b, sum(hist[b+1..]) and hist[b] to sh.  nbins is a multiple of 8
// and at most 8 * blockDim.x.
__device__ void block_find_bin(SelShared &sh, int nbins, unsigned need) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int per = 8;
    const bool own = tid * per < nbins;
    unsigned loc[per];
    unsigned sum = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) {
        loc[i] = own ? sh.hist[tid * per + i] : 0u;
        sum += loc[i];
    }
    // inclusive suffix sum over threads: suf(t) = sum of threads >= t
    unsigned suf = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned v = __shfl_down_sync(0xFFFFFFFFu, suf, o);
        if (lane + o < 32) suf += v;
    }
    if (lane == 0) sh.red2[warp] = suf;  // warp total
    __syncthreads();
    unsigned after = 0;  // totals of the warps above this one
    for (int w2 = warp + 1; w2 < nw; ++w2) after += sh.red2[w2];
    suf += after;
    if (suf >= need && suf - sum < need) {
        unsigned run = suf - sum;
        for (int i = per - 1; i >= 0; --i) {
            if (run + loc[i] >= need) {
                sh.dgt = tid * per + i;
                sh.above = run;
                sh.inbin = loc[i];
                break;
            }
            run += loc[i];
        }
    }
    __syncthreads();
}

template <class Src>
__device__ void block_select(const Src &src, int k, int *out_idx, float *out_score, SelShared &sh,
                             unsigned *bm, unsigned *gpre, int wcap, unsigned *status) {
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31;
    unsigned long long K = 1ull;
    unsigned nv = 0;
    {
        unsigned long long prefix = 0ull, mask = 0ull;
        unsigned need = (unsigned)k;
        int shift = 64;
        for (int pass = 0; pass < 6; ++pass) {
            const int bits = digit_bits(pass);
            shift -= bits;
            const unsigned dmask = (1u << bits) - 1u;
            for (int i = tid; i < (1 << bits); i += nt) sh.hist[i] = 0u;
            if (tid == 0) sh.dgt = -1;
            __syncthreads();
            unsigned nvl = 0;
            for (int base = 0; base < src.n; base += nt) {
                const int i = base + tid;
                unsigned long long key = i < src.n ? src.key(i) : 0ull;
                const bool act = key != 0ull && (key & mask) == prefix;
                nvl += key != 0ull;
                const unsigned dg = act ? (unsigned)(key >> shift) & dmask : 0xFFFFFFFFu;
                const unsigned m = __match_any_sync(0xFFFFFFFFu, dg);
                if (act && lane == __ffs(m) - 1) atomicAdd(&sh.hist[dg], (unsigned)__popc(m));
            }
            if (pass == 0) {
                nv = block_sum(nvl, sh.red);  // also orders the histogram updates
                if (nv <= (unsigned)k) break;  // every valid entry is selected
            } else {
                __syncthreads();
            }
            block_find_bin(sh, 1 << bits, need);
            const int d = sh.dgt;
            const unsigned above = sh.above, inbin = sh.inbin;
            __syncthreads();
            if (d < 0) break;  // unreachable when nv > k
            need -= above;
            prefix |= (unsigned long long)d << shift;
            mask |= (unsigned long long)dmask << shift;
            K = prefix;
            if (inbin == need) break;  // the whole bin is selected
        }
        if (nv <= (unsigned)k) K = 1ull;
    }
    const int nsel = (int)(nv < (unsigned)k ? nv : (unsigned)k);
    if (nsel > 0) {
        const int W = src.bound / 32 + 1;
        if (W > wcap) {
            raise_status(status, ST_INVALID);
            for (int r = tid; r < k; r += nt) {
                out_idx[r] = -1;
                if (out_score) out_score[r] = -INFINITY;
            }
            return;
        }
        for (int i = tid; i < W; i += nt) bm[i] = 0u;
        __syncthreads();
        for (int i = tid; i < src.n; i += nt) {
            const unsigned long long key = src.key(i);
            if (key != 0ull && key >= K) {
                const int p = key_pos(key);
                atomicOr(&bm[p >> 5], 1u << (p & 31));
            }
        }
        __syncthreads();
        // per group of 32 words: exclusive prefix of the set bits
        const int NG = (W + 31) / 32;
        for (int gi = tid; gi < NG; gi += nt) {
            unsigned s = 0;
            const int e = (gi + 1) * 32 < W ? (gi + 1) * 32 : W;
            for (int w = gi * 32; w < e; ++w) s += __popc(bm[w]);
            gpre[gi] = s;
        }
        __syncthreads();
        if (tid == 0) {
            unsigned run = 0;
            for (int gi = 0; gi < NG; ++gi) {
                const unsigned s = gpre[gi];
                gpre[gi] = run;
                run += s;
            }
        }
        __syncthreads();
        for (int i = tid; i < src.n; i += nt) {
            const unsigned long long key = src.key(i);
            if (key != 0ull && key >= K) {
                const int p = key_pos(key);
                const int w = p >> 5;
                unsigned r = gpre[w >> 5];
                for (int w2 = w & ~31; w2 < w; ++w2) r += __popc(bm[w2]);
                r += __popc(bm[w] & ((1u << (p & 31)) - 1u));
                out_idx[r] = p;
                if (out_score) out_score[r] = ord_score(key_ord(key));
            }
        }
    }
    for (int r = nsel + tid; r < k; r += nt) {
        out_idx[r] = -1;
        if (out_score) out_score[r] = -INFINITY;
    }
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectArgs a) {
    extern __shared__ unsigned sel_smem[];
    __shared__ SelShared sh;
    const int row = blockIdx.x;
    const int wcap = a.bitmap_words;
    unsigned *bm = sel_smem;
    unsigned *gpre = sel_smem + wcap;
    int *oi = a.out_idx + (long long)row * a.k;
    float *os = a.out_score ? a.out_score + (long long)row * a.k : nullptr;
    auto pad_all = [&]() {
        for (int r = threadIdx.x; r < a.k; r += blockDim.x) {
            oi[r] = -1;
            if (os) os[r] = -INFINITY;
        }
    };
    switch (a.kind) {
    case SEL_DENSE_CAND:
    case SEL_REUSE_CAND:
    case SEL_MEMBER_SCORES: {
        if (!a.plan[0]) { pad_all(); return; }
        const int b = find_seg(a.cu, a.S, row);
        const int t = row - a.cu[b];
        if (a.kind == SEL_DENSE_CAND) {
            unsigned n = a.cnt[row];
            CandSrc src{a.buf + (long long)row * a.cap, (int)(n < a.cap ? n : a.cap), t};
            block_select(src, a.k, oi, os, sh, bm, gpre, wcap, a.status);
        } else {
            const int p = a.plan[a.pl.rp() + b] + t / a.g;
            if (a.kind == SEL_REUSE_CAND) {
                unsigned n = a.cnt[p];
                CandSrc src{a.buf + (long long)p * a.cap, (int)(n < a.cap ? n : a.cap), t};
                block_select(src, a.k, oi, os, sh, bm, gpre, wcap, a.status);
            } else {
                ScoreSrc src{a.scores + (long long)row * a.ld, a.cand + (long long)p * a.c, a.c, t};
                block_select(src, a.k, oi, os, sh, bm, gpre, wcap, a.status);
            }
        }
        return;
    }
    case SEL_PROXY_TO_C: {
        if (!a.plan[0]) { pad_all(); return; }
        if (row >= a.plan[2]) return;
        const int *rp = a.plan + a.pl.rp();
        const int b = find_seg(rp, a.S, row);
        const int i = row - rp[b];
        const int n = a.cu[b + 1] - a.cu[b];
        const int bound = row_bound(i, n, a.g);
        unsigned cn = a.cnt[row];
        CandSrc src{a.buf + (long long)row * a.cap, (int)(cn < a.cap ? cn : a.cap), bound};
        block_select(src, a.k, oi, nullptr, sh, bm, gpre, wcap, a.status);
        return;
    }
    default: {  // decode kinds
        const bool per_member = a.kind != SEL_DEC_PROXY_TO_C;
        const int b = per_member ? row / a.G : row;
        const int m = per_member ? row % a.G : 0;
        const int kv = a.kv_len[b];
        if (kv < a.G || kv > a.n_max) {
            if (threadIdx.x == 0) raise_status(a.status, ST_INVALID);
            pad_all();
            return;
        }
        if (a.kind == SEL_DEC_DENSE) {
            const int bound = kv - a.G + m;
            ScoreSrc src{a.scores + (long long)row * a.ld, nullptr, bound + 1, bound};
            block_select(src, a.k, oi, os, sh, bm, gpre, wcap, a.status);
        } else if (a.kind == SEL_DEC_REUSE) {
            const int bound = kv - a.G + m;
            ScoreSrc src{a.scores + (long long)b * a.ld, nullptr, bound + 1, bound};
            block_select(src, a.k, oi, os, sh, bm, gpre, wcap, a.status);
        } else if (a.kind == SEL_DEC_PROXY_TO_C) {
            ScoreSrc src{a.scores + (long long)b * a.ld, nullptr, kv, kv - 1};
            block_select(src, a.k, oi, nullptr, sh, bm, gpre, wcap, a.status);
        } else {  // SEL_DEC_MEMBER
            const int bound = kv - a.G + m;
            ScoreSrc src{a.scores + (long long)row * a.ld, a.cand + (long long)b * a.c, a.c, bound};
            block_select(src, a.k, oi, os, sh, bm, gpre, wcap, a.status);
        }
        return;
    }
    }
}

}  // namespace

cudaError_t launch_select(const SelectArgs &a, cudaStream_t st) {
    if (a.nrows <= 0) return cudaSuccess;
    const size_t smem = ((size_t)a.bitmap_words + (size_t)(a.bitmap_words + 31) / 32 + 1) * 4;
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    TraceScope ts("select", st);
    select_kernel<<<a.nrows, kSelThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace idx
