// select.cu -- exact final top-k of one row per CTA.
//
// The entries of a row (candidate keys from a score pass, or fp32 scores)
// are ranked by key = (ord(score) << 32) | (0xFFFFFFFF - s), so the top-k is
// "highest score first, ties to the lower position".
//
// Two kernels here (the decode score rows, a full fp32 row per query or
// proxy over its whole cache, take a cluster of CTAs per row: dec_select.cu):
//  - select_kernel: the block-score rows of the block pre-filter (a proxy's
//    scores over the complete blocks of its prefix, prefill Quest rule and
//    decode), below;
//  - select_fast_kernel: candidate buffers with a floor (dense, Reuse,
//    proxy -> C, proxy -> blocks) and Refine member rows over a candidate
//    set, further down.
//
// select_kernel:
// 1. One pass over the row in global memory counts the valid entries and
//    builds a histogram of the key's top 12 bits (1/16-octave score bins);
//    the bin D holding the k-th largest key follows.
// 2. A second global pass copies every entry whose top bits are >= D into
//    shared memory: the k-th key and everything above it, a few thousand
//    entries at most for the workloads here.
// 3. An MSB-first radix select (12/12/8-bit digits over the score part, the
//    position part only for ties) over the staged keys finds the exact k-th
//    largest key K.
// 4. The selected positions (key >= K) are marked in a shared bitmap over
//    0..bound; each selected entry writes itself at its rank among the
//    marked bits, which lists the top-k in ascending position without a sort.
// When the staged set would not fit, steps 3-4 read the row from global
// memory instead (same arithmetic).
#include <math.h>

#include "common.cuh"
#include "plan.cuh"

namespace idx {

namespace {

constexpr int kSelThreads = 512;
constexpr int kMaxBins = 4096;  // widest radix digit: 12 bits

// dense fp32 scores with their positions (NULL: position = index)
struct ScoreSrc {
    static constexpr bool kShared = false;
    const float *sc;
    const int *pos;
    int n;
    int bound;
    __device__ unsigned long long key(int i) const {
        const int p = pos ? pos[i] : i;
        if (p < 0 || p > bound) return 0ull;
        return make_key(score_ord(sc[i]), p);
    }
};

// keys staged in shared memory (all valid)
struct StageSrc {
    static constexpr bool kShared = true;  // cheap to read: no unrolled prefetch needed
    const unsigned long long *st;
    int n;
    int bound;
    __device__ unsigned long long key(int i) const { return st[i]; }
};

struct SelShared {
    unsigned hist[kMaxBins];
    unsigned red[32];
    unsigned red2[32];
    int dgt;
    unsigned above;
    unsigned inbin;
    unsigned nstage;
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

// Digits of the 64-bit key, most significant first: 12 + 12 + 8 bits of the
// score's ord, then 12 + 12 + 8 bits of the position part (ties only).
__device__ __forceinline__ int digit_bits(int pass) { return (pass % 3 == 2) ? 8 : 12; }

// Block-wide: the largest bin b of hist[0..nbins) with sum(hist[b..]) >= need;
// writes b, sum(hist[b+1..]) and hist[b] to sh (sh.dgt stays -1 if none).
// nbins is a multiple of 8 and at most 8 * blockDim.x.
__device__ void block_find_bin(SelShared &sh, int nbins, unsigned need) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    constexpr int per = 8;
    const bool own = tid * per < nbins;
    unsigned loc[per];
    unsigned sum = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) {
        loc[i] = own ? sh.hist[tid * per + i] : 0u;
        sum += loc[i];
    }
    unsigned suf = sum;  // inclusive suffix sum over the warp's threads
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned v = __shfl_down_sync(0xFFFFFFFFu, suf, o);
        if (lane + o < 32) suf += v;
    }
    if (lane == 0) sh.red2[warp] = suf;
    __syncthreads();
    unsigned after = 0;
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

// Histogram of digit (key >> shift) & dmask over entries matching `prefix`
// under `mask`; warp-aggregated increments (equal digits add once per warp).
// Returns the number of valid entries seen by this thread.
// Entries are read kUnroll at a time per thread, all loads issued before any
// is used, so that a warp keeps several memory requests in flight.
constexpr int kUnroll = 8;

template <class Src>
__device__ unsigned hist_pass(const Src &src, SelShared &sh, int shift, unsigned dmask, unsigned long long prefix,
                              unsigned long long mask) {
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31;
    unsigned nvl = 0;
    if constexpr (Src::kShared) {
        for (int base = 0; base < src.n; base += nt) {
            const int i = base + tid;
            const unsigned long long key = i < src.n ? src.key(i) : 0ull;
            nvl += key != 0ull;
            const bool act = key != 0ull && (key & mask) == prefix;
            const unsigned dg = act ? (unsigned)(key >> shift) & dmask : 0xFFFFFFFFu;
            const unsigned m = __match_any_sync(0xFFFFFFFFu, dg);
            if (act && lane == __ffs(m) - 1) atomicAdd(&sh.hist[dg], (unsigned)__popc(m));
        }
    } else {
        for (int base = 0; base < src.n; base += nt * kUnroll) {
            unsigned long long key[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int i = base + u * nt + tid;
                key[u] = i < src.n ? src.key(i) : 0ull;
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                nvl += key[u] != 0ull;
                const bool act = key[u] != 0ull && (key[u] & mask) == prefix;
                const unsigned dg = act ? (unsigned)(key[u] >> shift) & dmask : 0xFFFFFFFFu;
                const unsigned m = __match_any_sync(0xFFFFFFFFu, dg);
                if (act && lane == __ffs(m) - 1) atomicAdd(&sh.hist[dg], (unsigned)__popc(m));
            }
        }
    }
    return nvl;
}

// Exact k-th largest valid key of src, refining a known prefix from digit
// pass `pass0` on; `need` = how many keys matching the prefix to select.
template <class Src>
__device__ unsigned long long radix_kth(const Src &src, SelShared &sh, unsigned need, int pass0,
                                        unsigned long long prefix, unsigned long long mask) {
    const int tid = threadIdx.x, nt = blockDim.x;
    int shift = 64;
    for (int p = 0; p < pass0; ++p) shift -= digit_bits(p);
    unsigned long long K = prefix;
    for (int pass = pass0; pass < 6; ++pass) {
        const int bits = digit_bits(pass);
        shift -= bits;
        const unsigned dmask = (1u << bits) - 1u;
        for (int i = tid; i < (1 << bits); i += nt) sh.hist[i] = 0u;
        if (tid == 0) sh.dgt = -1;
        __syncthreads();
        hist_pass(src, sh, shift, dmask, prefix, mask);
        __syncthreads();
        block_find_bin(sh, 1 << bits, need);
        const int d = sh.dgt;
        const unsigned above = sh.above, inbin = sh.inbin;
        __syncthreads();
        if (d < 0) break;  // unreachable when more than `need` keys match
        need -= above;
        prefix |= (unsigned long long)d << shift;
        mask |= (unsigned long long)dmask << shift;
        K = prefix;
        if (inbin == need) break;  // the whole bin is selected
    }
    return K;
}

// write the nsel keys >= K of src in ascending position, then pad to k
template <class Src>
__device__ void emit(const Src &src, unsigned long long K, int nsel, int k, int *out_idx, float *out_score,
                     unsigned *bm, unsigned *gpre, int wcap, unsigned *status) {
    const int tid = threadIdx.x, nt = blockDim.x;
    if (nsel > 0) {
        const int W = src.bound / 32 + 1;
        if (W > wcap) {
            raise_status(status, ST_INVALID);
            nsel = 0;
        } else {
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
            // exclusive prefix of the set bits per word: each thread owns a
            // contiguous run of words; a block scan of the runs' totals
            const int per = (W + nt - 1) / nt;
            const int w0 = tid * per, w1 = w0 + per < W ? w0 + per : W;
            unsigned run = 0;
            for (int w = w0; w < w1; ++w) run += __popc(bm[w]);
            unsigned inc = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned v = __shfl_up_sync(0xFFFFFFFFu, inc, o);
                if ((tid & 31) >= o) inc += v;
            }
            if ((tid & 31) == 31) gpre[W + (tid >> 5)] = inc;  // warp totals after the words
            __syncthreads();
            unsigned before = 0;
            for (int w2 = 0; w2 < (tid >> 5); ++w2) before += gpre[W + w2];
            unsigned acc = before + inc - run;
            for (int w = w0; w < w1; ++w) {
                const unsigned c = __popc(bm[w]);
                gpre[w] = acc;
                acc += c;
            }
            __syncthreads();
            for (int i = tid; i < src.n; i += nt) {
                const unsigned long long key = src.key(i);
                if (key != 0ull && key >= K) {
                    const int p = key_pos(key);
                    const int w = p >> 5;
                    const unsigned r = gpre[w] + __popc(bm[w] & ((1u << (p & 31)) - 1u));
                    out_idx[r] = p;
                    if (out_score) out_score[r] = ord_score(key_ord(key));
                }
            }
        }
    }
    for (int r = nsel + tid; r < k; r += nt) {
        out_idx[r] = -1;
        if (out_score) out_score[r] = -INFINITY;
    }
}

// Append the keys of src that are valid and >= lo to the shared stage
// (order not kept); returns how many there were (the stage holds the first
// stage_cap of them).
template <class Src>
__device__ unsigned stage_keys(const Src &src, SelShared &sh, unsigned long long lo, unsigned long long *stage,
                               int stage_cap) {
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31;
    if (tid == 0) sh.nstage = 0;
    __syncthreads();
    for (int base = 0; base < src.n; base += nt * kUnroll) {
        unsigned long long key[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = base + u * nt + tid;
            key[u] = i < src.n ? src.key(i) : 0ull;
        }
        // one reservation per warp for all kept keys of the round
        unsigned cnt = 0;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) cnt += (key[u] != 0ull && key[u] >= lo) ? 1u : 0u;
        unsigned inc = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned v = __shfl_up_sync(0xFFFFFFFFu, inc, o);
            if (lane >= o) inc += v;
        }
        const unsigned total = __shfl_sync(0xFFFFFFFFu, inc, 31);
        if (total) {
            unsigned b = 0;
            if (lane == 31) b = atomicAdd(&sh.nstage, total);
            b = __shfl_sync(0xFFFFFFFFu, b, 31) + inc - cnt;
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                if (key[u] != 0ull && key[u] >= lo) {
                    if (b < (unsigned)stage_cap) stage[b] = key[u];
                    ++b;
                }
            }
        }
    }
    __syncthreads();
    return sh.nstage;
}

template <class Src>
__device__ void block_select(const Src &src, int k, int *out_idx, float *out_score, SelShared &sh,
                             unsigned long long *stage, int stage_cap, unsigned *bm, unsigned *gpre, int wcap,
                             unsigned *status) {
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31;
    if (src.n <= stage_cap) {
        // short rows: one pass stages them all
        const unsigned ns = stage_keys(src, sh, 1ull, stage, stage_cap);
        if (ns <= (unsigned)stage_cap) {
            const StageSrc ss{stage, (int)ns, src.bound};
            if (ns <= (unsigned)k) {
                emit(ss, 1ull, (int)ns, k, out_idx, out_score, bm, gpre, wcap, status);
            } else {
                const unsigned long long K = radix_kth(ss, sh, (unsigned)k, 0, 0ull, 0ull);
                emit(ss, K, k, k, out_idx, out_score, bm, gpre, wcap, status);
            }
            return;
        }
        __syncthreads();  // too many: select over the row in global memory
    }
    // pass 1: valid count and the top-12-bit histogram
    for (int i = tid; i < kMaxBins; i += nt) sh.hist[i] = 0u;
    if (tid == 0) {
        sh.dgt = -1;
        sh.nstage = 0;
    }
    __syncthreads();
    const unsigned nv = block_sum(hist_pass(src, sh, 52, 0xFFFu, 0ull, 0ull), sh.red);
    if (nv <= (unsigned)k) {  // every valid entry is selected
        emit(src, 1ull, (int)nv, k, out_idx, out_score, bm, gpre, wcap, status);
        return;
    }
    block_find_bin(sh, kMaxBins, (unsigned)k);
    const int d0 = sh.dgt;
    const unsigned above0 = sh.above, inbin0 = sh.inbin;
    __syncthreads();
    const unsigned long long pre0 = (unsigned long long)d0 << 52, mask0 = 0xFFFull << 52;
    const unsigned need = (unsigned)k - above0;
    if (inbin0 == need) {  // the k-th key closes its bin: select everything >= the bin
        emit(src, pre0, k, k, out_idx, out_score, bm, gpre, wcap, status);
        return;
    }
    if (above0 + inbin0 <= (unsigned)stage_cap) {
        // pass 2: stage the keys of bin d0 and above
        const unsigned ns = stage_keys(src, sh, pre0, stage, stage_cap);
        const StageSrc ss{stage, (int)ns, src.bound};
        const unsigned long long K = radix_kth(ss, sh, need, 1, pre0, mask0);
        emit(ss, K, k, k, out_idx, out_score, bm, gpre, wcap, status);
        return;
    }
    const unsigned long long K = radix_kth(src, sh, need, 1, pre0, mask0);
    emit(src, K, k, k, out_idx, out_score, bm, gpre, wcap, status);
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectArgs a) {
    extern __shared__ __align__(16) unsigned long long sel_smem[];
    __shared__ SelShared sh;
    const int row = blockIdx.x;
    const int wcap = a.bitmap_words;
    unsigned long long *stage = sel_smem;
    unsigned *bm = reinterpret_cast<unsigned *>(sel_smem + a.stage_cap);
    unsigned *gpre = bm + wcap;
    int *oi = a.out_idx + (long long)row * a.k;
    float *os = a.out_score ? a.out_score + (long long)row * a.k : nullptr;
    auto pad_all = [&]() {
        for (int r = threadIdx.x; r < a.k; r += blockDim.x) {
            oi[r] = -1;
            if (os) os[r] = -INFINITY;
        }
    };
    switch (a.kind) {
    case SEL_PROXY_SPILL_TO_BLOCKS: {
        // prefill block mode (Quest rule): proxy row p's top blocks among the
        // complete blocks of its prefix (t_last + 1) / 64, k = c / 64 slots,
        // one of them kept for the partial block when the prefix ends inside
        // a block; rows of the call's scratch from plan[6]
        const int p = row;
        if (!a.plan[0] || p >= a.plan[2] || !scored_in_range(a.plan, p)) return;
        const long long sp = (long long)p - a.plan[6];
        int *ob = a.out_idx + sp * a.k;
        const int *rp = a.plan + a.pl.rp();
        const int b = find_seg(rp, a.S, p);
        const int i = p - rp[b];
        const int n = a.cu[b + 1] - a.cu[b];
        const int tl = row_bound(i, n, a.g);
        const int nfull = (tl + 1) >> kBlockShift;
        const int want = a.k - (((tl + 1) & (kBlockN - 1)) != 0 ? 1 : 0);
        const int take = want < nfull ? want : nfull;
        if (take > 0) {
            ScoreSrc src{a.scores + sp * a.ld, nullptr, nfull, nfull - 1};
            block_select(src, take, ob, nullptr, sh, stage, a.stage_cap, bm, gpre, wcap, a.status);
        }
        for (int r = (take > 0 ? take : 0) + threadIdx.x; r < a.k; r += blockDim.x) ob[r] = -1;
        return;
    }
    case SEL_DEC_PROXY_TO_BLOCKS: {
        // the proxy's top blocks among request b's complete blocks: k = c / 64
        // slots, one of them kept for the partial block when kv_len[b] ends
        // inside a block; the slots not taken are -1
        const int b = row;
        const int kv = a.kv_len[b];
        if (kv < a.G || kv > a.n_max) {
            if (threadIdx.x == 0) raise_status(a.status, ST_INVALID);
            pad_all();
            return;
        }
        const int nfull = kv >> kBlockShift;
        const int want = a.k - ((kv & (kBlockN - 1)) != 0 ? 1 : 0);
        const int take = want < nfull ? want : nfull;
        if (take > 0) {
            ScoreSrc src{a.scores + (long long)b * a.ld, nullptr, nfull, nfull - 1};
            block_select(src, take, oi, nullptr, sh, stage, a.stage_cap, bm, gpre, wcap, a.status);
        }
        for (int r = (take > 0 ? take : 0) + threadIdx.x; r < a.k; r += blockDim.x) oi[r] = -1;
        return;
    }
    default:  // the other kinds run in select_fast_kernel
        return;
    }
}

// ===================================================================
// select_fast_kernel: the final top-k of rows whose entries are few or
// filtered -- candidate buffers with a floor (dense, Reuse, proxy -> C,
// proxy -> blocks) and Refine member score rows over a candidate set.
//
// One CTA of 256 threads per row, several CTAs per SM (the row's work is a
// chain of short, barrier-separated steps, so rows in flight hide each
// other's latency):
// 1. one global pass stages every valid entry at or above the row's floor
//    into shared memory (16-byte loads, one reservation per warp and round);
//    member rows stage entry i at slot i, which keeps their order;
// 2. an MSB-first radix select with 8-bit digits over the staged keys finds
//    the exact k-th largest key K, starting right below the leading bits all
//    staged scores share (they lie between the floor and the largest staged
//    score), two barriers per digit (double-buffered histograms);
// 3. the selected entries (key >= K) are listed in ascending position:
//    member rows by an ordered compaction of the stage (their candidate
//    positions ascend), candidate rows by a bitmap over the prefix, in
//    chunks of 131072 positions (16 KB), walked word by word.
// A row whose floor admits more entries than the stage holds takes the same
// steps reading its entries from global memory instead.
// ===================================================================
constexpr int kFT = 256;                          // threads of select_fast_kernel
constexpr int kFWarps = kFT / 32;
constexpr int kChunkBits = 1 << 17;               // positions per bitmap chunk
constexpr int kChunkWords = kChunkBits / 32;      // 4096 words = 16 KB

struct __align__(16) FastShared {
    unsigned hist[2][256];
    unsigned wtot[kFWarps];
    unsigned blkpre[kFT];           // emit: chunk-local rank of each lane block's first bit
    unsigned short blkmid[kFT];     // emit: rank of its ninth word's first bit within the block
    unsigned nstage;
    unsigned maxord;
    unsigned minord;
    int dgt;
    unsigned above;
    unsigned inbin;
};

// Block-wide exclusive prefix of one value per thread; *total = the sum.
__device__ __forceinline__ unsigned fast_excl_scan(unsigned v, unsigned *wtot, unsigned *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned u = __shfl_up_sync(0xFFFFFFFFu, inc, o);
        if (lane >= o) inc += u;
    }
    if (lane == 31) wtot[warp] = inc;
    __syncthreads();
    unsigned before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < kFWarps; ++w) {
        const unsigned t = wtot[w];
        before += w < warp ? t : 0u;
        all += t;
    }
    __syncthreads();  // wtot may be reused right after
    *total = all;
    return before + inc - v;
}

// Source: candidate keys in global memory, filtered by floor and bound.
struct GCand {
    const unsigned long long *buf;
    int n;
    unsigned long long lo;  // keys below lo (ord < floor) are out
    unsigned pmin;          // low word >= pmin <=> position <= bound
    __device__ __forceinline__ unsigned long long key(int i) const {
        const unsigned long long kk = buf[i];
        return (kk >= lo && (unsigned)kk >= pmin) ? kk : 0ull;
    }
};
// Source: score row over a list of positions (NULL: position = index).
struct GScore {
    const float *sc;
    const int *pos;
    int n;
    int bound;
    __device__ __forceinline__ unsigned long long key(int i) const {
        const int p = pos ? pos[i] : i;
        if (p < 0 || p > bound) return 0ull;
        return make_key(score_ord(sc[i]), p);
    }
};
// Source: keys staged in shared memory (0 = empty slot).
struct SStage {
    const unsigned long long *st;
    int n;
    __device__ __forceinline__ unsigned long long key(int i) const { return st[i]; }
};

// MSB-first radix with 8-bit digits below a known prefix: the `need`-th
// largest of the nonzero keys of src matching `prefix` under `mask`, the
// digits below bit `shift`.  Pass p builds its histogram in sh.hist[p & 1],
// which is clear on entry (p = p0), and clears the other one for the next
// pass.  Returns the key K with exactly `need` matching keys >= K (plus the
// keys above the prefix the caller already counted).
template <class Src>
__device__ unsigned long long fast_kth_run(const Src &src, FastShared &sh, unsigned need,
                                           unsigned long long prefix, unsigned long long mask, int shift, int p) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    while (shift > 0) {
        const int bits = shift >= 8 ? 8 : shift;
        shift -= bits;
        const unsigned dmask = (1u << bits) - 1u;
        unsigned *h = sh.hist[p & 1];
        sh.hist[(p + 1) & 1][tid] = 0u;  // the next digit's histogram
        for (int i = tid; i < src.n; i += kFT) {
            const unsigned long long kk = src.key(i);
            if (kk != 0ull && (kk & mask) == prefix) atomicAdd(&h[(unsigned)(kk >> shift) & dmask], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            unsigned above;
            const int b = warp_find_bin(h, need, &above);
            if (lane == 0) {
                sh.dgt = b;
                sh.above = above;
                sh.inbin = b >= 0 ? h[b] : 0u;
            }
        }
        __syncthreads();
        const int d = sh.dgt;
        const unsigned above = sh.above, inbin = sh.inbin;
        ++p;
        if (d < 0) break;  // unreachable: more than `need` keys match the prefix
        need -= above;
        prefix |= (unsigned long long)d << shift;
        mask |= (unsigned long long)dmask << shift;
        if (inbin == need) break;  // the whole bin is selected
    }
    // leave hist[0] clear for the next user
    sh.hist[0][tid] = 0u;
    __syncthreads();
    return prefix;
}

// Exact k-th largest nonzero key of src (more than `need` nonzero keys,
// all with ords in [lo_ord, hi_ord]): the radix from the first bit where
// lo_ord and hi_ord differ; sh.hist[0] is clear on entry (and sh.hist[1] is
// cleared here).
template <class Src>
__device__ unsigned long long fast_kth(const Src &src, FastShared &sh, unsigned need, unsigned lo_ord,
                                       unsigned hi_ord) {
    const unsigned diff = lo_ord ^ hi_ord;
    const int lead = diff ? __clz(diff) : 32;  // leading ord bits every key shares
    const unsigned long long mask = lead ? (~0ull << (64 - lead)) : 0ull;
    const unsigned long long prefix = ((unsigned long long)hi_ord << 32) & mask;
    return fast_kth_run(src, sh, need, prefix, mask, 64 - lead, 0);
}

// Keys staged in shared memory, read relative to a base ord: key - base << 32.
// A key whose ord is at or above the base gives a nonzero result; a key below
// it (or an empty slot) wraps around to a value whose top bits are set, which
// matches none of the prefixes the callers search.
struct SStageOff {
    const unsigned long long *st;
    int n;
    unsigned long long base;
    __device__ __forceinline__ unsigned long long key(int i) const { return st[i] - base; }
};

// First digit of a staged candidate key, built while staging: its ord above
// the floor in 1/128-octave steps (2^16 ord units; the scores near the k-th
// of these rows put about a hundred keys in a step), 255 = that far or more.
constexpr int kFirstShift = 16;
__device__ __forceinline__ unsigned first_digit(unsigned ord, unsigned floor_ord) {
    const unsigned x = (ord - floor_ord) >> kFirstShift;
    return x < 255u ? x : 255u;
}

// Copy n entries from shared memory to a row in global memory with 16-byte
// accesses when both sides are 16-byte aligned.
template <typename T>
__device__ __forceinline__ void fast_copy_out(const T *src, T *dst, int n) {
    if (((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src)) & 15u) == 0) {
        const int n4 = n >> 2;
        const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
        uint4 *d4 = reinterpret_cast<uint4 *>(dst);
        for (int i = threadIdx.x; i < n4; i += kFT) d4[i] = s4[i];
        for (int i = (n4 << 2) + threadIdx.x; i < n; i += kFT) dst[i] = src[i];
    } else {
        for (int i = threadIdx.x; i < n; i += kFT) dst[i] = src[i];
    }
}

// Bitmap layout of the emit.  The chunk's words (word L covers positions
// 32L .. 32L+31) are split between the warps in contiguous ranges of
// 32 * per words, and within a warp's range between the lanes in contiguous
// blocks of `per` words (per a power of two), so that each lane ranks its
// block in order with one warp scan.  Word L is stored transposed: the j-th
// word of lane i's block at (warp range) + 32 j + i, so that a warp reading
// the j-th word of every lane's block touches 32 consecutive words.
__device__ __forceinline__ int emit_per(int nwords) {
    const int per = (nwords + kFWarps * 32 - 1) / (kFWarps * 32);  // 1 .. kChunkWords / kFT
    return per <= 1 ? 1 : 1 << (32 - __clz(per - 1));
}
__device__ __forceinline__ int emit_word(int L, int per) {
    const int range = 32 * per;
    const int m = L & (range - 1);
    return (L - m) + ((m & (per - 1)) << 5) + (m >> (31 - __clz(per)));
}

// List the nonzero keys >= K of src in ascending position through a bitmap
// (chunks of kChunkBits positions over 0..bound); returns how many.  Each
// chunk: the selected keys set their bits; each lane block's count is ranked
// by a warp scan and a block scan; then every selected key is placed at its
// rank = its lane block's first rank + the bits before it in the block.  The
// bits before it in its word come from one popcount, those of the block's
// earlier words from a per-word table (8 bits a word: the rank of the word's
// first bit within its run of 8 words; the second run's offset is kept per
// block) in `buf` when it has room, else from popcounts of those words.  The
// lists are built in `buf` after the table and copied out with coalesced
// stores; without room they are written directly.
template <class Src>
__device__ int fast_emit_bitmap(const Src &src, unsigned long long K, int bound, int k, int *out_idx,
                                float *out_score, FastShared &sh, unsigned *bm, unsigned *buf, int buf_words,
                                bool bm_clear = false) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // the first chunk is the widest: its table size serves every chunk
    const int tw0 = kFT * emit_per(bound / 32 + 1 < kChunkWords ? bound / 32 + 1 : kChunkWords);
    const bool tab = buf_words >= tw0 / 4;
    unsigned char *rk = reinterpret_cast<unsigned char *>(buf);
    unsigned *lst = buf + (tab ? tw0 / 4 : 0);
    const int lw = buf_words - (tab ? tw0 / 4 : 0);
    const bool via_smem = lw >= (out_score ? 2 * k : k);
    int *pi = via_smem ? reinterpret_cast<int *>(lst) : out_idx;
    float *ps = via_smem ? reinterpret_cast<float *>(lst + k) : out_score;
    int base = 0;
    for (int c0 = 0; c0 <= bound; c0 += kChunkBits) {
        const int nwords = (bound - c0) / 32 + 1 < kChunkWords ? (bound - c0) / 32 + 1 : kChunkWords;
        const int per = emit_per(nwords), lg = 31 - __clz(per);
        if (!(bm_clear && c0 == 0)) {  // the caller may have cleared it for the first chunk
            for (int j = tid; j < kFT * per; j += kFT) bm[j] = 0u;
            __syncthreads();
        }
        for (int i = tid; i < src.n; i += kFT) {
            const unsigned long long kk = src.key(i);
            if (kk != 0ull && kk >= K) {
                const int p = key_pos(kk) - c0;
                if (p >= 0 && p < kChunkBits) atomicOr(&bm[emit_word(p >> 5, per)], 1u << (p & 31));
            }
        }
        __syncthreads();
        // lane `lane` of warp `warp` owns logical words wb + lane * per .. + per - 1,
        // stored at wb + 32 j + lane; the table entry of a word sits at its
        // storage index
        const int wb = warp * 32 * per;
        unsigned cnt = 0, run = 0;
        for (int j = 0; j < per; ++j) {
            const int w = wb + 32 * j + lane;
            if (j == 8) {  // per <= kChunkWords / kFT = 16: at most two runs
                sh.blkmid[tid] = (unsigned short)cnt;
                run = 0;
            }
            if (tab) rk[w] = (unsigned char)run;  // at most 7 * 32 = 224
            const unsigned c = __popc(bm[w]);
            cnt += c;
            run += c;
        }
        unsigned inc = cnt;  // inclusive warp prefix of the lanes' counts
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned v = __shfl_up_sync(0xFFFFFFFFu, inc, o);
            if (lane >= o) inc += v;
        }
        if (lane == 31) sh.wtot[warp] = inc;
        __syncthreads();
        unsigned before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < kFWarps; ++w) {
            const unsigned t = sh.wtot[w];
            before += w < warp ? t : 0u;
            total += t;
        }
        sh.blkpre[tid] = before + inc - cnt;  // chunk-local rank of the lane block's first bit
        __syncthreads();
        for (int i = tid; i < src.n; i += kFT) {
            const unsigned long long kk = src.key(i);
            if (kk != 0ull && kk >= K) {
                const int p = key_pos(kk) - c0;
                if (p >= 0 && p < kChunkBits) {
                    const int L = p >> 5, w = emit_word(L, per), j = L & (per - 1);
                    unsigned r = sh.blkpre[L >> lg] + __popc(bm[w] & ((1u << (p & 31)) - 1u));
                    if (tab) {
                        r += rk[w] + (j >= 8 ? sh.blkmid[L >> lg] : 0u);
                    } else {  // the block's earlier words sit 32, 64, .. words below
                        for (int t = 1; t <= j; ++t) r += __popc(bm[w - 32 * t]);
                    }
                    const int at = base + (int)r;
                    if (at < k) {  // never past the row
                        pi[at] = c0 + p;
                        if (out_score) ps[at] = ord_score(key_ord(kk));
                    }
                }
            }
        }
        base += (int)total;
        if (base > k) base = k;
        __syncthreads();  // the bitmap and the table are rewritten by the next chunk
    }
    if (via_smem) {
        fast_copy_out(pi, out_idx, base);
        if (out_score) fast_copy_out(ps, out_score, base);
    }
    return base;
}

// Member rows: the staged entries are in candidate order (ascending
// position); list the nonzero keys >= K in that order.  Warp w owns a
// contiguous segment of the stage and walks it 32 entries at a time (lane i
// reads entry base + i: conflict-free), placing its selected entries by a
// ballot prefix; a block scan of the warps' counts gives each segment's
// offset.  The list is built in shared memory (`buf`, room for 2 * k words)
// and then copied out with coalesced stores; without room it is written
// directly.
__device__ int fast_emit_ordered(const unsigned long long *st, int n, unsigned long long K, int k, int *out_idx,
                                 float *out_score, FastShared &sh, unsigned *buf, int buf_words) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int seg = ((n + kFWarps - 1) / kFWarps + 31) & ~31;
    const int i0 = warp * seg, i1 = i0 + seg < n ? i0 + seg : n;
    unsigned cnt = 0;
    for (int b = i0; b < i1; b += 32) {
        const int i = b + lane;
        const unsigned long long kk = i < i1 ? st[i] : 0ull;
        cnt += __popc(__ballot_sync(0xFFFFFFFFu, kk != 0ull && kk >= K));
    }
    // exclusive prefix over warps (lane 0 holds each warp's count)
    if (lane == 0) sh.wtot[warp] = cnt;
    __syncthreads();
    unsigned before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kFWarps; ++w) {
        const unsigned t = sh.wtot[w];
        before += w < warp ? t : 0u;
        total += t;
    }
    __syncthreads();  // wtot may be reused right after
    const bool via_smem = 2 * k <= buf_words;
    int *pi = via_smem ? reinterpret_cast<int *>(buf) : out_idx;
    float *ps = via_smem ? reinterpret_cast<float *>(buf + k) : out_score;
    unsigned r = before;
    for (int b = i0; b < i1; b += 32) {
        const int i = b + lane;
        const unsigned long long kk = i < i1 ? st[i] : 0ull;
        const bool sel = kk != 0ull && kk >= K;
        const unsigned m = __ballot_sync(0xFFFFFFFFu, sel);
        const unsigned at = r + __popc(m & lanemask_lt());
        if (sel && at < (unsigned)k) {  // never past the row
            pi[at] = key_pos(kk);
            if (out_score) ps[at] = ord_score(key_ord(kk));
        }
        r += __popc(m);
    }
    const int nsel = (int)total < k ? (int)total : k;
    if (via_smem) {
        __syncthreads();
        fast_copy_out(pi, out_idx, nsel);
        if (out_score) fast_copy_out(ps, out_score, nsel);
    }
    return nsel;
}

__device__ __forceinline__ void fast_pad(int nsel, int k, int *out_idx, float *out_score) {
    for (int r = nsel + (int)threadIdx.x; r < k; r += kFT) {
        out_idx[r] = -1;
        if (out_score) out_score[r] = -INFINITY;
    }
}

__device__ __forceinline__ unsigned warp_max_u(unsigned v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned u = __shfl_xor_sync(0xFFFFFFFFu, v, o);
        v = u > v ? u : v;
    }
    return v;
}
__device__ __forceinline__ unsigned warp_min_u(unsigned v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned u = __shfl_xor_sync(0xFFFFFFFFu, v, o);
        v = u < v ? u : v;
    }
    return v;
}

// Outputs of the cutoff margin of a row (adaptive budget), or km = 0.
struct MarginOut {
    int km;          // the budget k whose margin is taken (< the row's k_sel)
    float *sigma;    // this row's sigma
    unsigned *vk;    // ord of s_(km-1)
    int *need;       // ties of s_(km-1) the top-km keeps
};

// Cutoff margin over the row's top-k_sel (the nsel keys >= K of src, every
// key of src at or above lo_ord, the largest hi_ord) ("Uncertainty-gated
// selection for block-sparse attention", Section 3 Method, steps 3-4):
// s_(0) = the largest score, s_(km-1) = the km-th largest, s_(km) = the
// (km+1)-th; sigma = (s_(km-1) - s_(km)) / (s_(0) - s_(km)) in fp32, 0 when
// the denominator is 0, NaN when the row has at most km entries.  Also the
// ord of s_(km-1) and how many of its ties the top-km keeps (the lowest
// positions, as the top-k rule ranks them).
template <class Src>
__device__ void fast_margin(const Src &src, unsigned long long K, int nsel, unsigned lo_ord, unsigned hi_ord,
                            const MarginOut &m, FastShared &sh) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (nsel < m.km + 1) {
        if (tid == 0) {
            *m.sigma = __uint_as_float(0x7FC00000u);  // quiet NaN: no (km+1)-th score
            *m.vk = 0u;
            *m.need = 0;
        }
        return;
    }
    sh.hist[0][tid] = 0u;
    __syncthreads();
    // the key with exactly km keys >= it (a bin edge, not always a key)
    const unsigned long long Km = fast_kth(src, sh, (unsigned)m.km, lo_ord, hi_ord);
    // one pass over the top-k_sel: among the top-km, the smallest ord
    // (s_(km-1)) and how many keys hold it (the ties the top-km keeps); below
    // them, the largest ord (s_(km): the (km+1)-th key, a tie or not)
    unsigned mn = 0xFFFFFFFFu, nmn = 0u, below = 0u;
    for (int i = tid; i < src.n; i += kFT) {
        const unsigned long long kk = src.key(i);
        if (kk != 0ull && kk >= K) {
            const unsigned o = key_ord(kk);
            if (kk >= Km) {
                nmn = o < mn ? 1u : (o == mn ? nmn + 1u : nmn);
                mn = o < mn ? o : mn;
            } else {
                below = o > below ? o : below;
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const unsigned om = __shfl_xor_sync(0xFFFFFFFFu, mn, off);
        const unsigned on = __shfl_xor_sync(0xFFFFFFFFu, nmn, off);
        nmn = om < mn ? on : (om == mn ? nmn + on : nmn);
        mn = om < mn ? om : mn;
    }
    below = __reduce_max_sync(0xFFFFFFFFu, below);
    if (lane == 0) {
        sh.hist[1][warp] = mn;
        sh.hist[1][kFWarps + warp] = nmn;
        sh.hist[1][2 * kFWarps + warp] = below;
    }
    __syncthreads();
    if (tid == 0) {
        unsigned v1 = 0xFFFFFFFFu, ties = 0u, v2 = 0u;
#pragma unroll
        for (int w = 0; w < kFWarps; ++w) {
            const unsigned om = sh.hist[1][w], on = sh.hist[1][kFWarps + w], ob = sh.hist[1][2 * kFWarps + w];
            ties = om < v1 ? on : (om == v1 ? ties + on : ties);
            v1 = om < v1 ? om : v1;
            v2 = ob > v2 ? ob : v2;
        }
        const float f0 = ord_score(hi_ord), f1 = ord_score(v1), f2 = ord_score(v2);
        const float num = f1 - f2, den = f0 - f2;
        *m.sigma = den > 0.0f ? num / den : 0.0f;
        *m.vk = v1;
        *m.need = (int)ties;
    }
}

// Staging pass of a candidate row: every key with ord >= max(floor_ord, 1)
// (ord 0 is the empty key; no arithmetic result has it) goes to the stage,
// and the first radix digit of each is counted in sh.hist[0].  kPos: the
// buffer may hold positions past the bound (a Reuse member reading its
// proxy's buffer), which are dropped too; without it every buffered position
// is within the bound (the score pass appends only keys the row may see).
// Returns this thread's largest staged ord (0: none).
template <bool kPos>
__device__ unsigned stage_cand(const GCand &g, unsigned floor_ord, FastShared &sh, unsigned long long *stage,
                               int stage_cap) {
    const int tid = threadIdx.x, lane = tid & 31, n = g.n;
    const unsigned f1 = floor_ord > 0u ? floor_ord : 1u;
    unsigned mx = 0u;
    // 8 keys per thread and round, as four 16-byte loads (rows start 2 KB
    // aligned); the next round's loads are issued before this round's keys
    // are filtered, so their latency overlaps the work
    const ulonglong2 *b2 = reinterpret_cast<const ulonglong2 *>(g.buf);
    ulonglong2 nx[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = u * (kFT * 2) + tid * 2;
        nx[u] = i < n ? b2[i >> 1] : make_ulonglong2(0ull, 0ull);
    }
    for (int base = 0; base < n; base += kFT * 8) {
        unsigned long long kv[8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + u * (kFT * 2) + tid * 2;
            kv[2 * u] = i < n ? nx[u].x : 0ull;
            kv[2 * u + 1] = (i + 1 < n) ? nx[u].y : 0ull;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + kFT * 8 + u * (kFT * 2) + tid * 2;
            if (i < n) nx[u] = b2[i >> 1];
        }
        unsigned okm = 0u;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const unsigned o = key_ord(kv[u]);
            bool ok = o >= f1;
            if (kPos) {
                ok = ok && (unsigned)kv[u] >= g.pmin;
                mx = max(mx, ok ? o : 0u);
            } else {
                mx = max(mx, o);
            }
            okm |= ok ? 1u << u : 0u;
        }
        const unsigned cnt = __popc(okm);
        unsigned inc = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned v = __shfl_up_sync(0xFFFFFFFFu, inc, o);
            if (lane >= o) inc += v;
        }
        const unsigned wt = __shfl_sync(0xFFFFFFFFu, inc, 31);
        if (wt) {
            unsigned b = 0;
            if (lane == 31) b = atomicAdd(&sh.nstage, wt);
            b = __shfl_sync(0xFFFFFFFFu, b, 31) + inc - cnt;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (okm & (1u << u)) {
                    if (b < (unsigned)stage_cap) stage[b] = kv[u];
                    ++b;
                    // the radix's first digit, counted here
                    atomicAdd(&sh.hist[0][first_digit(key_ord(kv[u]), floor_ord)], 1u);
                }
            }
        }
    }
    // without kPos the largest ord is staged exactly when it reaches f1
    if (!kPos && mx < f1) mx = 0u;
    return mx;
}

// Top-k of a candidate row (keys at or above `floor_ord`, positions <= bound),
// and its cutoff margin when m.km > 0.
__device__ void fast_cand_row(const unsigned long long *buf, int n, unsigned floor_ord, int bound, int k,
                              int *out_idx, float *out_score, FastShared &sh, unsigned long long *stage,
                              int stage_cap, unsigned *bm, const MarginOut &m, bool pos_check) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const GCand g{buf, n, (unsigned long long)floor_ord << 32, 0xFFFFFFFFu - (unsigned)bound};
    if (tid == 0) {
        sh.nstage = 0u;
        sh.maxord = 0u;
    }
    sh.hist[0][tid] = 0u;
    sh.hist[1][tid] = 0u;
    __syncthreads();
    // the emit's bitmap (first chunk, the words the walk reads), cleared here
    // (ordered before it by the barrier below)
    {
        const int nw = bound / 32 + 1 < kChunkWords ? bound / 32 + 1 : kChunkWords;
        const int nclr = kFT * emit_per(nw);
        for (int j = tid; j < nclr; j += kFT) bm[j] = 0u;
    }
    unsigned mx = pos_check ? stage_cand<true>(g, floor_ord, sh, stage, stage_cap)
                            : stage_cand<false>(g, floor_ord, sh, stage, stage_cap);
    mx = warp_max_u(mx);
    if (lane == 0 && mx) atomicMax(&sh.maxord, mx);
    __syncthreads();
    const int ns = (int)sh.nstage;
    const unsigned hi = sh.maxord;
    int nsel;
    // free stage room after the staged keys, from a 16-byte boundary
    const int used = ((ns < stage_cap ? ns : stage_cap) + 1) & ~1;
    unsigned *tail = reinterpret_cast<unsigned *>(stage + used);
    const int tail_words = used < stage_cap ? 2 * (stage_cap - used) : 0;
    if (ns <= k) {
        const SStage s{stage, ns};
        nsel = fast_emit_bitmap(s, 1ull, bound, k, out_idx, out_score, sh, bm, tail, tail_words, true);
        if (m.km) fast_margin(s, 1ull, nsel, floor_ord, hi, m, sh);
    } else if (ns <= stage_cap) {
        const SStage s{stage, ns};
        // the first digit's histogram is in hist[0]: find its bin, then refine
        // inside it relative to the floor (keys - floor << 32)
        if (warp == 0) {
            unsigned above;
            const int b = warp_find_bin(sh.hist[0], (unsigned)k, &above);
            if (lane == 0) {
                sh.dgt = b;
                sh.above = above;
                sh.inbin = b >= 0 ? sh.hist[0][b] : 0u;
            }
        }
        __syncthreads();
        const int b1 = sh.dgt;
        const unsigned above1 = sh.above, inbin1 = sh.inbin;
        const unsigned long long fl = (unsigned long long)floor_ord << 32;
        const unsigned long long edge = (unsigned long long)floor_ord + ((unsigned long long)(b1 > 0 ? b1 : 0) << kFirstShift);
        unsigned long long K;
        if (b1 >= 0 && inbin1 == (unsigned)k - above1 && edge <= 0xFFFFFFFFull) {
            K = edge << 32;  // everything from the bin's lower edge up
            sh.hist[0][tid] = 0u;
            __syncthreads();
        } else if (b1 >= 0 && b1 < 255) {
            // x = ord - floor has its top 16 bits = b1 (bits 48..63 of key - fl)
            const SStageOff so{stage, ns, fl};
            K = fast_kth_run(so, sh, (unsigned)k - above1, (unsigned long long)b1 << 48, 0xFFFFull << 48, 48, 1) + fl;
        } else {  // the k-th key is far above the floor: the plain radix
            sh.hist[0][tid] = 0u;
            sh.hist[1][tid] = 0u;
            __syncthreads();
            K = fast_kth(s, sh, (unsigned)k, floor_ord, hi);
        }
        nsel = fast_emit_bitmap(s, K, bound, k, out_idx, out_score, sh, bm, tail, tail_words, true);
        if (m.km) fast_margin(s, K, nsel, floor_ord, hi, m, sh);
    } else {
        // more entries at or above the floor than the stage holds: the same
        // steps over the row in global memory (the whole stage is free)
        sh.hist[0][tid] = 0u;
        __syncthreads();
        const unsigned long long K = fast_kth(g, sh, (unsigned)k, floor_ord, hi);
        nsel = fast_emit_bitmap(g, K, bound, k, out_idx, out_score, sh, bm, reinterpret_cast<unsigned *>(stage),
                                2 * stage_cap);
        if (m.km) fast_margin(g, K, nsel, floor_ord, hi, m, sh);
    }
    fast_pad(nsel, k, out_idx, out_score);
}

// Top-k of a member score row over its candidate list (positions ascending,
// -1 = none), masked to positions <= bound.
__device__ void fast_member_row(const float *sc, const int *pos, int n, int bound, int k, int *out_idx,
                                float *out_score, FastShared &sh, unsigned long long *stage, int stage_cap,
                                unsigned *bm) {
    const int tid = threadIdx.x, lane = tid & 31;
    const GScore g{sc, pos, n, bound};
    if (tid == 0) {
        sh.nstage = 0u;
        sh.maxord = 0u;
        sh.minord = 0xFFFFFFFFu;
    }
    sh.hist[0][tid] = 0u;
    __syncthreads();
    unsigned mx = 0u, mn = 0xFFFFFFFFu, cnt = 0;
    const bool staged = n <= stage_cap;
    const bool vec = staged && pos != nullptr &&
                     ((reinterpret_cast<uintptr_t>(sc) | reinterpret_cast<uintptr_t>(pos)) & 15u) == 0;
    // 8 entries per thread and round, every load issued before any is used:
    // with 16-byte aligned rows as two runs of 4 (16-byte loads and stores),
    // else one entry at a time
    if (vec) {
        for (int base = 0; base < n; base += kFT * 8) {
            float4 sv[2];
            int4 pv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int i = base + (u * kFT + tid) * 4;
                if (i + 3 < n) {
                    sv[u] = *reinterpret_cast<const float4 *>(sc + i);
                    pv[u] = *reinterpret_cast<const int4 *>(pos + i);
                } else {
                    sv[u] = make_float4(i < n ? sc[i] : 0.0f, i + 1 < n ? sc[i + 1] : 0.0f,
                                        i + 2 < n ? sc[i + 2] : 0.0f, 0.0f);
                    pv[u] = make_int4(i < n ? pos[i] : -1, i + 1 < n ? pos[i + 1] : -1, i + 2 < n ? pos[i + 2] : -1,
                                      -1);
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int i = base + (u * kFT + tid) * 4;
                const float s4[4] = {sv[u].x, sv[u].y, sv[u].z, sv[u].w};
                const int p4[4] = {pv[u].x, pv[u].y, pv[u].z, pv[u].w};
                unsigned long long kk[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    kk[j] = (p4[j] >= 0 && p4[j] <= bound) ? make_key(score_ord(s4[j]), p4[j]) : 0ull;
                    if (kk[j] != 0ull) {
                        const unsigned o = key_ord(kk[j]);
                        mx = o > mx ? o : mx;
                        mn = o < mn ? o : mn;
                        ++cnt;
                    }
                }
                if (i + 3 < n) {
                    ulonglong2 *d2 = reinterpret_cast<ulonglong2 *>(stage + i);
                    d2[0] = make_ulonglong2(kk[0], kk[1]);
                    d2[1] = make_ulonglong2(kk[2], kk[3]);
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (i + j < n) stage[i + j] = kk[j];
                }
            }
        }
    } else {
        for (int base = 0; base < n; base += kFT * 8) {
            int pv[8];
            float sv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = base + u * kFT + tid;
                pv[u] = i < n ? (pos ? pos[i] : i) : -1;
                sv[u] = i < n ? sc[i] : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = base + u * kFT + tid;
                const unsigned long long kk =
                    (pv[u] >= 0 && pv[u] <= bound) ? make_key(score_ord(sv[u]), pv[u]) : 0ull;
                if (staged && i < n) stage[i] = kk;
                if (kk != 0ull) {
                    const unsigned o = key_ord(kk);
                    mx = o > mx ? o : mx;
                    mn = o < mn ? o : mn;
                    ++cnt;
                }
            }
        }
    }
    mx = warp_max_u(mx);
    mn = warp_min_u(mn);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, o);
    if (lane == 0) {
        if (cnt) {
            atomicMax(&sh.maxord, mx);
            atomicMin(&sh.minord, mn);
        }
        atomicAdd(&sh.nstage, cnt);
    }
    __syncthreads();
    const unsigned nv = sh.nstage, hi = sh.maxord, lo = sh.minord;
    int nsel;
    if (staged) {
        const SStage s{stage, n};
        const unsigned long long K = nv <= (unsigned)k ? 1ull : fast_kth(s, sh, (unsigned)k, lo, hi);
        nsel = fast_emit_ordered(stage, n, K, k, out_idx, out_score, sh, bm, kChunkWords);
    } else {
        const unsigned long long K = nv <= (unsigned)k ? 1ull : fast_kth(g, sh, (unsigned)k, lo, hi);
        nsel = fast_emit_bitmap(g, K, bound, k, out_idx, out_score, sh, bm, reinterpret_cast<unsigned *>(stage),
                                2 * stage_cap);
    }
    fast_pad(nsel, k, out_idx, out_score);
}

__global__ void __launch_bounds__(kFT, 4) select_fast_kernel(SelectArgs a) {
    extern __shared__ __align__(16) unsigned long long fast_smem[];
    __shared__ FastShared sh;
    const int row = blockIdx.x;
    unsigned *bm = reinterpret_cast<unsigned *>(fast_smem);
    unsigned long long *stage = fast_smem + kChunkWords / 2;
    const int scap = a.stage_cap;
    int *oi = a.out_idx + (long long)row * a.k;
    float *os = a.out_score ? a.out_score + (long long)row * a.k : nullptr;
    // per-row scratch of prefill calls starts at the call's first scored row
    // (plan[6]); member scores at the first member of that row (plan[8])
    const long long p0 = a.kind == SEL_DEC_MEMBER ? 0 : a.plan[6];
    // the cutoff margin of dense rows (adaptive budget), per output row
    const MarginOut mo = a.kind == SEL_DENSE_CAND && a.kmargin > 0
                             ? MarginOut{a.kmargin, a.m_sigma + row, a.m_vk + row, a.m_need + row}
                             : MarginOut{0, nullptr, nullptr, nullptr};
    // own: the buffer is the output row's own (scored with the same bound)
    auto cand = [&](long long r, int bound, int k, const MarginOut &m, bool own) {
        const long long sr = r - p0;
        const unsigned n = a.cnt[sr];
        fast_cand_row(a.buf + sr * a.cap, (int)(n < a.cap ? n : a.cap), a.floor ? a.floor[sr] : 0u, bound, k, oi, os,
                      sh, stage, scap, bm, m, !own);
    };
    const MarginOut none{0, nullptr, nullptr, nullptr};
    switch (a.kind) {
    case SEL_DENSE_CAND:
    case SEL_REUSE_CAND:
    case SEL_MEMBER_SCORES: {
        if (!a.plan[0]) {
            fast_pad(0, a.k, oi, os);
            if (mo.km && threadIdx.x == 0) {
                *mo.sigma = __uint_as_float(0x7FC00000u);
                *mo.vk = 0u;
                *mo.need = 0;
            }
            return;
        }
        if (row < a.plan[4] || row >= a.plan[5]) return;  // not an output row of this call
        const int b = find_seg(a.cu, a.S, row);
        const int t = row - a.cu[b];
        if (a.kind == SEL_DENSE_CAND) {
            cand(row, t, a.k, mo, true);
        } else {
            const int n = a.cu[b + 1] - a.cu[b];
            const int p = a.plan[a.pl.rp() + b] + group_of(t, n, a.g, a.db);
            // Reuse, and members scored on their own (guardrail): the top-k of
            // the scored row's candidates inside the member's prefix
            if (a.kind == SEL_REUSE_CAND || t < dense_rows(n, a.g, a.db))
                cand(p, t, a.k, none, false);
            else if (!a.skip_members)
                fast_member_row(a.scores + ((long long)row - a.plan[8]) * a.ld, a.cand + (p - p0) * a.c, a.c, t,
                                a.k, oi, os, sh, stage, scap, bm);
        }
        return;
    }
    case SEL_PROXY_TO_C:
    case SEL_PROXY_TO_BLOCKS: {
        // output: the proxy's scratch row (candidate set, or selected blocks);
        // a proxy with no output member has none
        if (!a.plan[0] || row >= a.plan[2] || !scored_in_range(a.plan, row)) return;
        const int *rp = a.plan + a.pl.rp();
        const int b = find_seg(rp, a.S, row);
        const int i = row - rp[b];
        const int n = a.cu[b + 1] - a.cu[b];
        int *po = a.out_idx + ((long long)row - p0) * a.k;
        if (a.kind == SEL_PROXY_TO_C) {
            // a member scored on its own needs no candidate set (nothing reads its row)
            if (i < dense_rows(n, a.g, a.db)) return;
            oi = po;
            os = nullptr;
            cand(row, row_bound(i, n, a.g, a.db), a.k, none, true);
            return;
        }
        const int tl = row_bound(i, n, a.g);
        // the partial block holding the last member takes one slot of the budget
        const int kr = a.k - (((tl + 1) & (kBlockN - 1)) ? 1 : 0);
        if (kr > 0) {
            oi = po;
            os = nullptr;
            cand(row, key_bound(tl, kBlockShift), kr, none, false);
        }
        for (int r = (kr > 0 ? kr : 0) + (int)threadIdx.x; r < a.k; r += kFT) po[r] = -1;
        return;
    }
    case SEL_DEC_MEMBER: {
        const int b = row / a.G, m = row % a.G;
        const int kv = a.kv_len[b];
        if (kv < a.G || kv > a.n_max) {
            if (threadIdx.x == 0) raise_status(a.status, ST_INVALID);
            fast_pad(0, a.k, oi, os);
            return;
        }
        fast_member_row(a.scores + (long long)row * a.ld, a.cand + (long long)b * a.c, a.c, kv - a.G + m, a.k, oi,
                        os, sh, stage, scap, bm);
        return;
    }
    default:
        return;
    }
}


// Staging room (keys) of select_fast_kernel: room for the top-k plus the
// entries the floor lets through beyond it, and for every entry of a member
// row (c); at least the room that still fits four CTAs per SM.
constexpr int kFastMinRoom = 4608;

bool fast_kind(int kind) {
    return kind == SEL_DENSE_CAND || kind == SEL_REUSE_CAND || kind == SEL_PROXY_TO_C ||
           kind == SEL_PROXY_TO_BLOCKS || kind == SEL_MEMBER_SCORES || kind == SEL_DEC_MEMBER;
}

cudaError_t launch_select_fast(const SelectArgs &a, cudaStream_t st) {
    SelectArgs b = a;
    const bool member = a.kind == SEL_MEMBER_SCORES || a.kind == SEL_DEC_MEMBER;
    // candidate rows stage about 1.2 k keys (at most 1.7 k measured): 1.5 k + 512
    long long room = a.k + a.k / 2 + 512;
    if (member && a.c > room) room = a.c;
    if (room < kFastMinRoom) room = kFastMinRoom;
    room = (room + 255) / 256 * 256;
    const size_t limit = 232448 - sizeof(FastShared) - 1024 - (size_t)kChunkWords * 4;
    if ((size_t)room * 8 > limit) room = (long long)(limit / 8) & ~1LL;
    b.stage_cap = (int)room;
    const size_t smem = (size_t)kChunkWords * 4 + (size_t)room * 8;
    cudaError_t e = cudaFuncSetAttribute(select_fast_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    TraceScope ts("select", st);
    select_fast_kernel<<<a.nrows, kFT, smem, st>>>(b);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const SelectArgs &a, cudaStream_t st) {
    if (a.nrows <= 0) return cudaSuccess;
    if (member_select_fits(a)) {
        const cudaError_t e = launch_member_select(a, st);
        if (e != cudaSuccess || a.kind != SEL_MEMBER_SCORES || a.db <= 0 || a.g <= 1) return e;
        SelectArgs b = a;  // the guardrail's members scored on their own
        b.skip_members = 1;
        return launch_select_fast(b, st);
    }
    if (fast_kind(a.kind)) return launch_select_fast(a, st);
    if (dec_select_kind(a.kind)) return launch_dec_select(a, st);
    SelectArgs b = a;
    const size_t tail = ((size_t)a.bitmap_words * 2 + 32) * 4;  // bitmap + per-word prefix + warp totals
    const size_t limit = 232448 - sizeof(SelShared) - 1024;
    // staging room: the k-th key's 1/16-octave bin and everything above it
    long long cap = 2LL * a.k + 2048;
    if ((size_t)cap * 8 + tail > limit) cap = ((long long)limit - (long long)tail) / 8;
    if (cap < 0) cap = 0;
    b.stage_cap = (int)cap;
    const size_t smem = (size_t)cap * 8 + tail;
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    TraceScope ts("select", st);
    select_kernel<<<a.nrows, kSelThreads, smem, st>>>(b);
    return cudaGetLastError();
}

}  // namespace idx

