// common.cuh -- shared device helpers of libidx: score keys, status word,
// bounded waits, and the streaming per-row candidate filter used by every
// score kernel.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace idx {

// ------------------------------------------------------------- status word
// Bits OR-ed into the device status word (first 4 bytes of a workspace).
enum : unsigned { ST_TIMEOUT = 1u, ST_OVERFLOW = 2u, ST_INVALID = 4u };

__device__ __forceinline__ void raise_status(unsigned *status, unsigned bits) {
    if (status) atomicOr(status, bits);
}

// ----------------------------------------------------------------- keys
// A score is ranked by an unsigned "ord" that orders like the float
// (larger ord = larger score, -0 folded onto +0).  A candidate key packs
// (ord << 32) | (0xFFFFFFFF - s): larger key = better; equal scores rank
// the lower position higher (ties go to the lower index).  Key 0 never
// occurs for a finite score and marks an empty slot.
__device__ __forceinline__ unsigned score_ord(float f) {
    if (f == 0.0f) f = 0.0f;  // -0 -> +0
    unsigned u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord_score(unsigned o) {
    unsigned u = (o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o;
    return __uint_as_float(u);
}
__device__ __forceinline__ unsigned long long make_key(unsigned ord, int s) {
    return ((unsigned long long)ord << 32) | (unsigned long long)(0xFFFFFFFFu - (unsigned)s);
}
__device__ __forceinline__ int key_pos(unsigned long long key) {
    return (int)(0xFFFFFFFFu - (unsigned)(key & 0xFFFFFFFFull));
}
__device__ __forceinline__ unsigned key_ord(unsigned long long key) { return (unsigned)(key >> 32); }

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// ----------------------------------------------------------- bounded waits
// Every spin in this library ends: after ~kWaitNs nanoseconds of polling
// the wait gives up, the caller records ST_TIMEOUT and unwinds.
constexpr unsigned long long kWaitNs = 1000ull * 1000ull * 1000ull;  // 1 s

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// --------------------------------------------------- streaming candidate filter
// Each scored row keeps, in global memory, an append-only buffer of
// candidate keys of capacity `cap` and, in shared memory, a count, an
// admission threshold `thr` (a key is appended iff its ord >= thr) and a
// 256-bin histogram of the ords appended so far.
//
// Invariant (exactness): every key that can still be among the row's
// final top-`ksel` has ord >= thr when it is offered, so it is appended.
// Two rules raise thr and both keep the invariant:
//   (a) histogram: if >= ksel appended keys lie in bins >= b, every later
//       key whose ord is below bin b's lower edge is beaten by ksel keys;
//   (b) compaction: when the buffer nears capacity it is cut to its exact
//       top-ksel keys K_1 > ... > K_ksel; keys arrive in increasing
//       position, so a later key whose ord equals ord(K_ksel) loses the
//       tie, and thr = ord(K_ksel) + 1.
// The histogram bins are 1/16-octave slices of ord (ord >> 19) in a window
// placed once per row, when the first ksel keys have been appended, from
// the largest of them; bin 0 collects everything below the window and bin
// 255 everything above it.
constexpr int kBins = 256;
constexpr int kBinShift = 19;
constexpr int kBaseUnset = -0x40000000;  // histogram window not placed yet

struct RowSel {
    unsigned cnt;
    unsigned thr;
    int base;           // histogram window base, in units of ord >> kBinShift
    unsigned last_cnt;  // cnt at the last histogram threshold update
    unsigned floor;     // an ord that >= ksel offered keys reach: keys below it are out
};

__device__ __forceinline__ int sel_bin(unsigned ord, int base) {
    int b = (int)(ord >> kBinShift) - base + 1;
    return b < 0 ? 0 : (b > kBins - 1 ? kBins - 1 : b);
}
// lower edge (as an ord) of histogram bin b
__device__ __forceinline__ unsigned sel_bin_edge(int b, int base) {
    if (b <= 0) return 0u;
    int e = base + (b > kBins - 2 ? kBins - 2 : b) - 1;
    if (e < 0) e = 0;
    if (e > (int)(0xFFFFFFFFu >> kBinShift)) e = (int)(0xFFFFFFFFu >> kBinShift);
    return (unsigned)e << kBinShift;
}

// Warp-cooperative offer of one key per lane for row `r` (all 32 lanes of
// the warp call it with the same r).  buf_row = row's buffer in global.
__device__ __forceinline__ void sel_offer(RowSel &st, unsigned *hist, unsigned long long *buf_row,
                                          unsigned cap, bool valid, float score, int s,
                                          unsigned *status) {
    const unsigned ord = score_ord(score);
    const bool ok = valid && ord >= st.thr;
    const unsigned m = __ballot_sync(0xFFFFFFFFu, ok);
    if (m == 0u) return;
    const int lane = threadIdx.x & 31;
    const int leader = __ffs(m) - 1;
    unsigned base = 0;
    if (lane == leader) base = atomicAdd(&st.cnt, (unsigned)__popc(m));
    base = __shfl_sync(0xFFFFFFFFu, base, leader);
    if (ok) {
        const unsigned pos = base + (unsigned)__popc(m & lanemask_lt());
        if (pos < cap) buf_row[pos] = make_key(ord, s);
        else raise_status(status, ST_OVERFLOW);
        if (st.base != kBaseUnset) atomicAdd(&hist[sel_bin(ord, st.base)], 1u);
    }
}

// Warp-level suffix search over a 256-entry histogram h (16-byte aligned;
// lane l owns bins 8l..8l+7): returns the largest bin b with sum(h[b..255]) >= need (or -1
// if the total is below need) and, through *above, sum(h[b+1..255]).
__device__ __forceinline__ int warp_find_bin(const unsigned *h, unsigned need, unsigned *above) {
    const int lane = threadIdx.x & 31;
    unsigned loc[8];
    // two 16-byte loads per lane: 4 wavefronts each, no bank conflicts
    const uint4 *h4 = reinterpret_cast<const uint4 *>(h) + lane * 2;
    const uint4 x0 = h4[0], x1 = h4[1];
    loc[0] = x0.x; loc[1] = x0.y; loc[2] = x0.z; loc[3] = x0.w;
    loc[4] = x1.x; loc[5] = x1.y; loc[6] = x1.z; loc[7] = x1.w;
    unsigned sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) sum += loc[i];
    // inclusive suffix sum over lanes: suf(l) = sum of lanes >= l
    unsigned suf = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        unsigned v = __shfl_down_sync(0xFFFFFFFFu, suf, o);
        if (lane + o < 32) suf += v;
    }
    const unsigned ge = __ballot_sync(0xFFFFFFFFu, suf >= need);
    if (ge == 0u) {
        *above = 0;
        return -1;
    }
    const int L = 31 - __clz(ge);  // highest lane whose suffix reaches need
    int bin = -1;
    unsigned ab = 0;
    if (lane == L) {
        unsigned run = suf - sum;  // sum of lanes > L
        for (int i = 7; i >= 0; --i) {
            if (run + loc[i] >= need) {
                bin = L * 8 + i;
                ab = run;
                break;
            }
            run += loc[i];
        }
    }
    bin = __shfl_sync(0xFFFFFFFFu, bin, L);
    ab = __shfl_sync(0xFFFFFFFFu, ab, L);
    *above = ab;
    return bin;
}

// Rule (a): raise thr from the histogram (one warp per row).
__device__ __forceinline__ void sel_update_threshold(RowSel &st, const unsigned *hist, unsigned ksel) {
    const unsigned c = st.cnt;
    if (c < ksel) return;
    if (st.thr != 0u && c - st.last_cnt < 32u) return;
    unsigned above;
    const int b = warp_find_bin(hist, ksel, &above);
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
        st.last_cnt = c;
        if (b >= 0) {
            const unsigned e = sel_bin_edge(b, st.base);
            if (e > st.thr) st.thr = e;
            if (e > st.floor) st.floor = e;
        }
    }
    __syncwarp();
}

// Exact k-th largest key among buf[0..n) (keys unique, n >= k >= 1), by
// an MSB-first radix select with 8-bit digits.  One warp; scratch = 256
// words of shared memory owned by the warp.  Returns K such that exactly k
// keys of buf are >= K.
__device__ __forceinline__ unsigned long long warp_kth_key(const unsigned long long *buf, unsigned n,
                                                           unsigned k, unsigned *scratch) {
    const int lane = threadIdx.x & 31;
    unsigned long long prefix = 0ull, mask = 0ull;
    unsigned need = k;
    for (int shift = 56; shift >= 0; shift -= 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) scratch[lane * 8 + i] = 0u;
        __syncwarp();
        for (unsigned i = lane; i < n; i += 32) {
            const unsigned long long key = buf[i];
            if ((key & mask) == prefix) atomicAdd(&scratch[(unsigned)(key >> shift) & 255u], 1u);
        }
        __syncwarp();
        unsigned above;
        const int dgt = warp_find_bin(scratch, need, &above);
        const unsigned inbin = scratch[dgt < 0 ? 0 : dgt];
        __syncwarp();
        if (dgt < 0) return 0ull;  // fewer than k keys: cannot happen when n >= k
        need -= above;
        prefix |= (unsigned long long)dgt << shift;
        mask |= 0xFFull << shift;
        if (inbin == need) return prefix;  // the whole bin is selected
    }
    return prefix;
}

// Rule (b): compact row buffer to its exact top-ksel (one warp per row).
__device__ __forceinline__ void sel_compact(RowSel &st, unsigned long long *buf_row, unsigned cap,
                                            unsigned ksel, unsigned *scratch) {
    const int lane = threadIdx.x & 31;
    unsigned n = st.cnt;
    if (n > cap) n = cap;
    if (n <= ksel) return;
    const unsigned long long K = warp_kth_key(buf_row, n, ksel, scratch);
    unsigned wpos = 0;
    unsigned minord = 0xFFFFFFFFu;
    for (unsigned b0 = 0; b0 < n; b0 += 32) {
        const unsigned i = b0 + lane;
        unsigned long long key = 0ull;
        if (i < n) key = buf_row[i];
        const bool keep = (i < n) && key >= K;
        const unsigned m = __ballot_sync(0xFFFFFFFFu, keep);
        __syncwarp();
        if (keep) {
            buf_row[wpos + __popc(m & lanemask_lt())] = key;
            const unsigned o = key_ord(key);
            minord = o < minord ? o : minord;
        }
        wpos += __popc(m);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned v = __shfl_xor_sync(0xFFFFFFFFu, minord, o);
        minord = v < minord ? v : minord;
    }
    __syncwarp();
    if (lane == 0) {
        st.cnt = wpos;
        const unsigned t = minord + 1u;
        if (t > st.thr) st.thr = t;
        if (minord > st.floor) st.floor = minord;
    }
    __syncwarp();
}

// Per-tile upkeep of one row (one warp): place the histogram window once
// ksel keys have been appended (from the largest appended ord, 12 octaves
// below it to 4 above), cut the buffer when it is close to full, and raise
// the admission threshold.  Called only between tiles, when no warp offers.
// `slack` = the most keys one row can be offered before the next upkeep.
__device__ __forceinline__ void sel_maintain(RowSel &st, unsigned *hist, unsigned long long *buf_row,
                                             unsigned cap, unsigned ksel, unsigned *scratch, int slack) {
    const int lane = threadIdx.x & 31;
    __syncwarp();  // the warp's appends (buffer, counts) are visible to all its lanes
    if (st.base == kBaseUnset && st.cnt >= ksel) {
        const unsigned n = st.cnt < cap ? st.cnt : cap;
        unsigned mx = 0u;
        for (unsigned i = lane; i < n; i += 32) {
            const unsigned o = key_ord(buf_row[i]);
            mx = o > mx ? o : mx;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned v = __shfl_xor_sync(0xFFFFFFFFu, mx, o);
            mx = v > mx ? v : mx;
        }
        const int base = (int)(mx >> kBinShift) - 192;
        for (unsigned i = lane; i < n; i += 32) atomicAdd(&hist[sel_bin(key_ord(buf_row[i]), base)], 1u);
        __syncwarp();
        if (lane == 0) st.base = base;
        __syncwarp();
    }
    if ((int)st.cnt > (int)cap - slack) sel_compact(st, buf_row, cap, ksel, scratch);
    if (st.base != kBaseUnset) sel_update_threshold(st, hist, ksel);
}

__device__ __forceinline__ void sel_init(RowSel &st, unsigned *hist) {
    const int lane = threadIdx.x & 31;
    for (int i = lane; i < kBins; i += 32) hist[i] = 0u;
    if (lane == 0) {
        st.cnt = 0u;
        st.thr = 0u;
        st.base = kBaseUnset;
        st.last_cnt = 0u;
        st.floor = 0u;
    }
    __syncwarp();
}

}  // namespace idx
