// dec_select.cu -- the top-k of decode score rows (one fp32 score per cached
// position, up to 2^20 of them per row) by a cluster of 8 CTAs per row.
//
// The row's positions 0..bound are split into 8 contiguous segments, one per
// CTA of the cluster; a CTA keeps its segment's score ords in shared memory.
// The CTAs agree on the exact k-th largest key K (score ord, then the lower
// position first, as everywhere in this library) through the cluster's
// distributed shared memory:
//   1. the segment minima and maxima give the row's ord range [LO, HI];
//   2. radix rounds over x = key - LO<<32 with 11-bit digits, the first
//      spanning [LO, HI] exactly: every CTA counts its segment's digits, CTA r
//      sums bin slice r over the cluster, and every CTA reads the summed slices
//      and finds the bin holding the k-th key.  Rounds go on while that bin
//      holds more than kList keys (after one round it holds a few dozen: the
//      digits spread the row's range over 2048 bins);
//   3. the CTAs copy the bin's keys from every segment into one short list and
//      each finishes the radix on it (8-bit digits), all reaching the same K.
//      The pass that collects a segment's keys of the bin also counts, per
//      warp, the keys above the bin; with the bin's keys >= K (from the list)
//      that gives each warp's count of selected keys without another pass;
//   4. a prefix over the cluster's counts gives each CTA its offset, and it
//      writes its selected positions in ascending order.
// Cluster barriers separate the steps.  Every decision between them comes
// from values all CTAs of a cluster share (the row's bound and k, the summed
// histogram), so all CTAs take the same barriers; the last barrier keeps each
// CTA's shared memory alive until the others have read it.
#include <cooperative_groups.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace idx {

namespace {

constexpr int kDC = 8;              // CTAs per row (one cluster)
constexpr int kDT = 512;            // threads per CTA (two CTAs per SM: 32 warps hide the latencies)
constexpr int kDWarps = kDT / 32;
constexpr int kDBits = 11;          // radix digit of the cluster rounds
constexpr int kDBins = 1 << kDBits;
constexpr int kDSlice = kDBins / kDC;
constexpr int kList = 1024;         // keys of the k-th key's bin resolved in one CTA
constexpr int kSegCache = 16384;    // segment entries whose ords stay in shared memory

struct __align__(16) DecShared {
    unsigned hist[kDBins];
    unsigned red[kDSlice];                 // this CTA's slice of the cluster's histogram
    unsigned long long list[kList];        // this segment's keys of the k-th key's bin
    unsigned long long merged[kList];      // the bin's keys from every segment
    unsigned wtot[kDWarps];
    unsigned lo, hi;                       // segment ord range (published)
    unsigned nlist;                        // list entries (published)
    unsigned nsel;                         // selected entries (published)
    int dgt;
    unsigned above, inbin;
};

// One decode row: the scores, the positions 0..bound, and where the result goes.
struct DecRow {
    bool valid;
    const float *sc;
    int n;          // bound + 1 positions
    int k;
    int *oi;
    float *os;
};

__device__ DecRow dec_row(const SelectArgs &a, int row) {
    DecRow r{};
    const bool per_member = a.kind != SEL_DEC_PROXY_TO_C;
    const int b = per_member ? row / a.G : row;
    const int m = per_member ? row % a.G : 0;
    const int kv = a.kv_len[b];
    r.k = a.k;
    r.oi = a.out_idx + (long long)row * a.k;
    r.os = a.out_score && a.kind != SEL_DEC_PROXY_TO_C ? a.out_score + (long long)row * a.k : nullptr;
    r.valid = kv >= a.G && kv <= a.n_max;
    if (!r.valid) return r;
    if (a.kind == SEL_DEC_DENSE) {
        r.sc = a.scores + (long long)row * a.ld;
        r.n = kv - a.G + m + 1;
    } else if (a.kind == SEL_DEC_REUSE) {
        r.sc = a.scores + (long long)b * a.ld;
        r.n = kv - a.G + m + 1;
    } else {
        r.sc = a.scores + (long long)b * a.ld;
        r.n = kv;
    }
    return r;
}

// Block-wide: over the 2048 summed bins (slice s of them in CTA s of the
// cluster), the largest bin b with sum(bins >= b) >= need; writes b, the sum
// above it and its count to sh.
__device__ void find_bin_cluster(cg::cluster_group &cl, DecShared &sh, unsigned need) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int per = kDBins / kDT;  // consecutive bins per thread
    const int b0 = tid * per;
    const unsigned *src = cl.map_shared_rank(sh.red, b0 / kDSlice);
    unsigned loc[per];
    unsigned sum = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) {
        loc[i] = src[(b0 % kDSlice) + i];
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
    for (int w = warp + 1; w < kDWarps; ++w) after += sh.wtot[w];
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

// The need-th largest of the n keys of `keys` whose x = key - base matches
// prefix under mask, digits below bit `shift` (8 bits a pass); one CTA.
__device__ unsigned long long local_kth(const unsigned long long *keys, int n, unsigned long long base,
                                        unsigned long long prefix, unsigned long long mask, int shift,
                                        unsigned need, DecShared &sh) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    while (shift > 0) {
        const int bits = shift >= 8 ? 8 : shift;
        shift -= bits;
        const unsigned dmask = (1u << bits) - 1u;
        if (tid < 256) sh.hist[tid] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += kDT) {
            const unsigned long long x = keys[i] - base;
            if ((x & mask) == prefix) atomicAdd(&sh.hist[(unsigned)(x >> shift) & dmask], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            unsigned above;
            const int b = warp_find_bin(sh.hist, need, &above);
            if (lane == 0) {
                sh.dgt = b;
                sh.above = above;
                sh.inbin = b >= 0 ? sh.hist[b] : 0u;
            }
        }
        __syncthreads();
        const int d = sh.dgt;
        const unsigned above = sh.above, inbin = sh.inbin;
        __syncthreads();  // sh.hist and sh.dgt are rewritten by the next pass
        if (d < 0) break;  // unreachable: more than `need` keys match the prefix
        need -= above;
        prefix |= (unsigned long long)d << shift;
        mask |= (unsigned long long)dmask << shift;
        if (inbin == need) break;  // the whole bin is selected
    }
    return prefix;
}

__global__ void __cluster_dims__(kDC, 1, 1) __launch_bounds__(kDT, 2) dec_select_kernel(SelectArgs a, int seg,
                                                                                   int cached) {
    extern __shared__ __align__(16) unsigned dec_ords[];
    __shared__ DecShared sh;
    cg::cluster_group cl = cg::this_cluster();
    const int rank = (int)cl.block_rank();
    const int row = blockIdx.x / kDC;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const DecRow r = dec_row(a, row);
    if (!r.valid) {  // the same for every CTA of the cluster: no cluster barrier is taken
        if (rank == 0) {
            if (tid == 0) raise_status(a.status, ST_INVALID);
            for (int i = tid; i < r.k; i += kDT) {
                r.oi[i] = -1;
                if (r.os) r.os[i] = -INFINITY;
            }
        }
        return;
    }
    const int s0 = rank * seg < r.n ? rank * seg : r.n;
    const int s1 = s0 + seg < r.n ? s0 + seg : r.n;
    const int len = s1 - s0;
    const float *sc = r.sc + s0;
    auto ord_at = [&](int j) -> unsigned { return cached ? dec_ords[j] : score_ord(sc[j]); };
    auto key_at = [&](int j) -> unsigned long long { return make_key(ord_at(j), s0 + j); };

    // 1. segment ords to shared memory, and their range
    unsigned mn = 0xFFFFFFFFu, mx = 0u;
    const bool vec = ((reinterpret_cast<uintptr_t>(sc)) & 15u) == 0;
    if (vec) {
        // eight 16-byte loads per thread in flight before any is used: one
        // at a time, every load would wait out the full memory latency
        const int n4 = len >> 2;
        const float4 *s4 = reinterpret_cast<const float4 *>(sc);
        for (int i0 = tid; i0 < n4; i0 += 8 * kDT) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + u * kDT;
                v[u] = i < n4 ? s4[i] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + u * kDT;
                if (i < n4) {
                    const unsigned o0 = score_ord(v[u].x), o1 = score_ord(v[u].y), o2 = score_ord(v[u].z),
                                   o3 = score_ord(v[u].w);
                    if (cached) reinterpret_cast<uint4 *>(dec_ords)[i] = make_uint4(o0, o1, o2, o3);
                    mn = min(mn, min(min(o0, o1), min(o2, o3)));
                    mx = max(mx, max(max(o0, o1), max(o2, o3)));
                }
            }
        }
        for (int j = (n4 << 2) + tid; j < len; j += kDT) {
            const unsigned o = score_ord(sc[j]);
            if (cached) dec_ords[j] = o;
            mn = min(mn, o);
            mx = max(mx, o);
        }
    } else {
        for (int j0 = tid; j0 < len; j0 += 8 * kDT) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + u * kDT;
                v[u] = j < len ? sc[j] : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + u * kDT;
                if (j < len) {
                    const unsigned o = score_ord(v[u]);
                    if (cached) dec_ords[j] = o;
                    mn = min(mn, o);
                    mx = max(mx, o);
                }
            }
        }
    }
    // warp w's part of the segment in steps 3 and 4: [wj0, wj1)
    const int wseg = ((len + kDWarps - 1) / kDWarps + 31) & ~31;
    const int wj0 = warp * wseg, wj1 = wj0 + wseg < len ? wj0 + wseg : len;
    bool counted = false;  // sh.wtot holds each warp's count of keys >= K
    unsigned long long K = 1ull;  // n <= k: every position
    if (r.n > r.k) {
        mn = __reduce_min_sync(0xFFFFFFFFu, mn);
        mx = __reduce_max_sync(0xFFFFFFFFu, mx);
        if (tid == 0) {
            sh.lo = 0xFFFFFFFFu;
            sh.hi = 0u;
        }
        __syncthreads();
        if (lane == 0) {
            atomicMin(&sh.lo, mn);
            atomicMax(&sh.hi, mx);
        }
        cl.sync();
        unsigned LO = 0xFFFFFFFFu, HI = 0u;
#pragma unroll
        for (int c = 0; c < kDC; ++c) {
            const DecShared *o = cl.map_shared_rank(&sh, c);
            LO = min(LO, o->lo);
            HI = max(HI, o->hi);
        }
        const unsigned long long base = (unsigned long long)LO << 32;
        const unsigned span = HI - LO;
        // `shift` is the lowest bit of the current digit.  The first digit,
        // bits [32 + sh1, 43 + sh1) of x, covers ord - LO exactly: it is
        // (ord - LO) >> sh1, 32-bit arithmetic on the ord alone; each later
        // round takes the next (up to) 11 bits below it
        const int sh1 = span >= (unsigned)kDBins ? 32 - kDBits - __clz(span) : 0;
        int shift = 32 + sh1;
        unsigned long long prefix = 0ull, mask = 0ull;
        unsigned need = (unsigned)r.k;
        bool done = false, one_round = true;
        // 2. cluster rounds
        for (int round = 0;; ++round) {
            const int bits = round == 0 ? kDBits : (shift >= kDBits ? kDBits : shift);
            if (round > 0) shift -= bits;
            const unsigned dmask = (1u << bits) - 1u;
            for (int i = tid; i < kDBins; i += kDT) sh.hist[i] = 0u;
            __syncthreads();
            if (round == 0) {
                for (int j = tid; j < len; j += kDT) atomicAdd(&sh.hist[(ord_at(j) - LO) >> sh1], 1u);
            } else {
                for (int j = tid; j < len; j += kDT) {
                    const unsigned long long x = key_at(j) - base;
                    if ((x & mask) == prefix) atomicAdd(&sh.hist[(unsigned)(x >> shift) & dmask], 1u);
                }
            }
            cl.sync();  // every segment's histogram is complete
            for (int i = tid; i < kDSlice; i += kDT) {
                unsigned s = 0;
#pragma unroll
                for (int c = 0; c < kDC; ++c) s += cl.map_shared_rank(sh.hist, c)[rank * kDSlice + i];
                sh.red[i] = s;
            }
            cl.sync();  // every slice is summed
            find_bin_cluster(cl, sh, need);
            const int d = sh.dgt;
            const unsigned above = sh.above, inbin = sh.inbin;
            if (d < 0) break;  // unreachable: more than `need` keys remain
            need -= above;
            prefix |= (unsigned long long)d << shift;
            mask |= (unsigned long long)dmask << shift;
            if (inbin == need || shift == 0) {  // the whole bin is selected
                done = true;
                break;
            }
            if (inbin <= (unsigned)kList) break;
            one_round = false;
        }
        if (!done) {
            // 3. the bin's keys from every segment, resolved in each CTA; the
            // same pass counts each warp's keys above the bin, all selected
            if (tid == 0) sh.nlist = 0u;
            __syncthreads();
            const unsigned b1 = (unsigned)(prefix >> shift);  // the first digit, when it is the only one
            unsigned above_cnt = 0;
            for (int j0 = wj0; j0 < wj1; j0 += 32) {
                const int j = j0 + lane;
                bool in = false, up = false;
                if (j < wj1) {
                    const unsigned o = ord_at(j);
                    if (one_round) {
                        const unsigned d1 = (o - LO) >> sh1;
                        in = d1 == b1;
                        up = d1 > b1;
                    } else {
                        const unsigned long long xm = (make_key(o, s0 + j) - base) & mask;
                        in = xm == prefix;
                        up = xm > prefix;
                    }
                }
                above_cnt += __popc(__ballot_sync(0xFFFFFFFFu, up));
                const unsigned m = __ballot_sync(0xFFFFFFFFu, in);
                if (m) {
                    unsigned at = 0;
                    if (lane == 0) at = atomicAdd(&sh.nlist, (unsigned)__popc(m));
                    at = __shfl_sync(0xFFFFFFFFu, at, 0) + __popc(m & lanemask_lt());
                    if (in && at < (unsigned)kList) sh.list[at] = key_at(j);
                }
            }
            cl.sync();  // every list is complete
            // the eight list lengths in one round of remote reads, then every
            // entry copied by its own thread
            int end[kDC];
            int off = 0;
#pragma unroll
            for (int c = 0; c < kDC; ++c) end[c] = (int)cl.map_shared_rank(&sh, c)->nlist;
#pragma unroll
            for (int c = 0; c < kDC; ++c) {
                off += end[c];
                end[c] = off;
            }
            const int nm = off < kList ? off : kList;
            for (int i = tid; i < nm; i += kDT) {
                int c = 0, first = 0;  // the list holding entry i (the ends ascend)
#pragma unroll
                for (int c2 = 0; c2 < kDC - 1; ++c2) {
                    if (i >= end[c2]) {
                        c = c2 + 1;
                        first = end[c2];
                    }
                }
                sh.merged[i] = cl.map_shared_rank(sh.list, c)[i - first];
            }
            __syncthreads();
            prefix = local_kth(sh.merged, nm, base, prefix, mask, shift, need, sh);
            // each warp's count: its keys above the bin, plus its keys of the
            // bin (all in this CTA's list) that reach K
            const unsigned long long Kb = prefix + base;
            if (lane == 0) sh.wtot[warp] = above_cnt;
            __syncthreads();
            const int nown = (int)(sh.nlist < (unsigned)kList ? sh.nlist : (unsigned)kList);
            for (int i = tid; i < nown; i += kDT) {
                const unsigned long long kk = sh.list[i];
                if (kk >= Kb) atomicAdd(&sh.wtot[(key_pos(kk) - s0) / wseg], 1u);
            }
            __syncthreads();
            counted = true;
        }
        K = prefix + base;
    }

    // 4. this segment's selected keys, at the cluster offset, in ascending position
    const int j0 = wj0, j1 = wj1;
    // key >= K  <=>  ord > Kord, or ord == Kord and position <= Kpos
    const unsigned Kord = (unsigned)(K >> 32), Kpos = 0xFFFFFFFFu - (unsigned)K;
    auto selected = [&](int j) {
        const unsigned o = ord_at(j);
        return o > Kord || (o == Kord && (unsigned)(s0 + j) <= Kpos);
    };
    if (!counted) {  // the bin closed at K, or every position is selected
        unsigned cnt = 0;
        for (int j = j0; j < j1; j += 32) {
            const int jj = j + lane;
            const bool sel = jj < j1 && selected(jj);
            cnt += __popc(__ballot_sync(0xFFFFFFFFu, sel));
        }
        if (lane == 0) sh.wtot[warp] = cnt;
        __syncthreads();
    }
    unsigned wbefore = 0, own = 0;
    for (int w = 0; w < kDWarps; ++w) {
        wbefore += w < warp ? sh.wtot[w] : 0u;
        own += sh.wtot[w];
    }
    if (tid == 0) sh.nsel = own;
    cl.sync();  // every count is published
    unsigned before = 0, total = 0;
#pragma unroll
    for (int c = 0; c < kDC; ++c) {
        const unsigned nc = cl.map_shared_rank(&sh, c)->nsel;
        before += c < rank ? nc : 0u;
        total += nc;
    }
    unsigned at = before + wbefore;
    for (int j = j0; j < j1; j += 32) {
        const int jj = j + lane;
        const bool sel = jj < j1 && selected(jj);
        const unsigned m = __ballot_sync(0xFFFFFFFFu, sel);
        const unsigned p = at + __popc(m & lanemask_lt());
        if (sel && p < (unsigned)r.k) {  // never past the row
            r.oi[p] = s0 + jj;
            if (r.os) r.os[p] = ord_score(ord_at(jj));
        }
        at += __popc(m);
    }
    if (rank == kDC - 1) {
        for (int i = (int)(total < (unsigned)r.k ? total : (unsigned)r.k) + tid; i < r.k; i += kDT) {
            r.oi[i] = -1;
            if (r.os) r.os[i] = -INFINITY;
        }
    }
    cl.sync();  // no CTA leaves while another may still read its shared memory
}

}  // namespace

bool dec_select_kind(int kind) {
    return kind == SEL_DEC_DENSE || kind == SEL_DEC_REUSE || kind == SEL_DEC_PROXY_TO_C;
}

cudaError_t launch_dec_select(const SelectArgs &a, cudaStream_t st) {
    if (a.nrows <= 0) return cudaSuccess;
    // segments: multiples of 32 positions, 8 per row of up to n_max positions
    const int seg = ((a.n_max + kDC - 1) / kDC + 31) & ~31;
    const int cached = seg <= kSegCache ? 1 : 0;
    const size_t smem = cached ? (size_t)seg * 4 : 0;
    cudaError_t e = cudaFuncSetAttribute(dec_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    TraceScope ts("select", st);
    dec_select_kernel<<<a.nrows * kDC, kDT, smem, st>>>(a, seg, cached);
    return cudaGetLastError();
}

}  // namespace idx
