// simt.cu -- CUDA-core (FFMA) score kernels: any dtype, H and d that fit in
// shared memory.  They serve fp32 inputs and shapes the tensor-core kernels
// do not cover, and share the streaming filter and the select pass with the
// tensor-core path.
//
// Score of one (row, key) pair, in this order:
//     dot_j = sum_i q[j,i] * k[i]          (fp32 fma, i ascending)
//     acc   = fma(w_j, max(dot_j, 0), acc) (j ascending)
#include "common.cuh"
#include "plan.cuh"

namespace idx {

namespace {

constexpr int kSimtThreads = 256;  // 8 warps: one warp per row of a block

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

__host__ __device__ constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// shared-memory carve-up common to the three kernels
template <typename T>
struct SimtSmem {
    size_t q_off, k_off, w_off, sel_off, hist_off, scr_off, total;
    __host__ __device__ SimtSmem(int H, int d) {
        q_off = 0;
        k_off = align_up(q_off + (size_t)RB * H * d * sizeof(T), 16);
        w_off = align_up(k_off + (size_t)KT * (d + 1) * sizeof(float), 16);
        sel_off = align_up(w_off + (size_t)RB * H * sizeof(float), 16);
        hist_off = align_up(sel_off + (size_t)RB * sizeof(RowSel), 16);
        scr_off = hist_off + (size_t)RB * kBins * sizeof(unsigned);
        total = scr_off + (size_t)(kSimtThreads / 32) * 256 * sizeof(unsigned);
    }
};

// copy n_rows rows of H*d elements (row stride H*d) into shared memory,
// zero-filling rows >= valid
template <typename T>
__device__ void load_rows(T *dst, const T *src, int valid, int HD) {
    const int per = HD * (int)sizeof(T) / 16;  // 16-byte chunks per row (d % 8 == 0)
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
    for (int i = threadIdx.x; i < RB * per; i += blockDim.x) {
        const int r = i / per;
        d4[i] = r < valid ? s4[i] : make_uint4(0, 0, 0, 0);
    }
}

// keys[i] for i < KT of the tile, fp32, row stride d+1; rows past `valid` = 0
template <typename T>
__device__ void load_keys(float *ks, const T *k0, int valid, int d) {
    for (int idx = threadIdx.x; idx < KT * d; idx += blockDim.x) {
        const int i = idx / d, e = idx - i * d;
        ks[i * (d + 1) + e] = i < valid ? to_f(k0[(long long)i * d + e]) : 0.0f;
    }
}

// scores of the row in qs/ws against keys kb*32+lane (kb < 4) of the tile
template <typename T>
__device__ __forceinline__ void tile_scores(const T *qs, const float *ws, const float *ks, int H, int d,
                                            float sc[4]) {
    const int lane = threadIdx.x & 31;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < H; ++j) {
        float dot[4] = {0.f, 0.f, 0.f, 0.f};
        const T *qj = qs + j * d;
        for (int i = 0; i < d; ++i) {
            const float qv = to_f(qj[i]);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) dot[kb] = fmaf(qv, ks[(kb * 32 + lane) * (d + 1) + i], dot[kb]);
        }
        const float wj = ws[j];
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) acc[kb] = fmaf(wj, fmaxf(dot[kb], 0.0f), acc[kb]);
    }
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) sc[kb] = acc[kb];
}

template <typename T>
__global__ void __launch_bounds__(kSimtThreads) score_simt_kernel(ScoreArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const SimtSmem<T> L(a.H, a.d);
    T *qs = reinterpret_cast<T *>(smem + L.q_off);
    float *ks = reinterpret_cast<float *>(smem + L.k_off);
    float *wsm = reinterpret_cast<float *>(smem + L.w_off);
    RowSel *sel = reinterpret_cast<RowSel *>(smem + L.sel_off);
    unsigned *hist = reinterpret_cast<unsigned *>(smem + L.hist_off);
    unsigned *scr = reinterpret_cast<unsigned *>(smem + L.scr_off);
    __shared__ int s_item;
    const int warp = threadIdx.x >> 5;
    const int HD = a.H * a.d;
    int *plan = const_cast<int *>(a.plan);
    if (!plan[0]) return;
    const int nblocks = plan[1];
    unsigned *work = reinterpret_cast<unsigned *>(plan + 3);
    const T *q = reinterpret_cast<const T *>(a.q);
    const T *k = reinterpret_cast<const T *>(a.k);
    for (;;) {
        __syncthreads();
        if (threadIdx.x == 0) s_item = (int)atomicAdd(work, 1u);
        __syncthreads();
        const int item = s_item;
        if (item >= nblocks) break;
        const BlockInfo bi = block_info(plan, a.pl, a.cu, a.g, plan[a.pl.order() + item], a.kshift, a.db);
        load_rows(qs, q + (long long)bi.row0 * HD, bi.nrows, HD);
        for (int i = threadIdx.x; i < RB * a.H; i += blockDim.x)
            wsm[i] = (i / a.H) < bi.nrows ? a.w[(long long)bi.row0 * a.H + i] : 0.0f;
        if (a.sink == SINK_FILTER && warp < RB) sel_init(sel[warp], hist + warp * kBins);
        const int r = warp;
        const long long grow = (long long)bi.row0 + r;
        // a filtered row whose members are all outside the call's output rows
        // is not ranked (it has no scratch row)
        const bool row_ok = r < bi.nrows && (a.sink != SINK_FILTER || scored_in_range(plan, grow));
        const int bound = row_ok ? key_bound(row_bound(bi.i0 + r, bi.n, a.g, a.db), a.kshift) : -1;
        const long long srow = grow - plan[6];  // scratch row
        int slot = -1;
        if (a.sink == SINK_SPILL && row_ok && a.slot_of_row) slot = a.slot_of_row[grow];
        for (int tile = 0; tile < bi.ntiles; ++tile) {
            __syncthreads();
            const int s0 = tile * KT;
            int nvk = bi.maxbound + 1 - s0;
            nvk = nvk > KT ? KT : nvk;
            load_keys(ks, k + (bi.key0 + s0) * a.d, nvk, a.d);
            __syncthreads();
            if (row_ok && s0 <= bound) {
                float sc[4];
                tile_scores(qs + r * HD, wsm + r * a.H, ks, a.H, a.d, sc);
#pragma unroll
                for (int kb = 0; kb < 4; ++kb) {
                    const int s = s0 + kb * 32 + (threadIdx.x & 31);
                    const bool valid = s <= bound;
                    if (a.sink == SINK_FILTER) {
                        sel_offer(sel[r], hist + r * kBins, a.buf + srow * a.cap, a.cap, valid, sc[kb], s,
                                  a.status);
                    } else if (slot >= 0 && valid) {
                        a.spill[(long long)slot * a.ld + s] = sc[kb];
                    }
                }
            }
            if (a.sink == SINK_FILTER && row_ok)
                sel_maintain(sel[r], hist + r * kBins, a.buf + srow * a.cap, a.cap,
                             bi.i0 + r < dense_rows(bi.n, a.g, a.db) ? a.ksel_dense : a.ksel, scr + warp * 256, KT);
        }
        if (a.sink == SINK_FILTER && row_ok && (threadIdx.x & 31) == 0) {
            a.cnt[srow] = sel[r].cnt;
            if (a.floor_out) a.floor_out[srow] = sel[r].floor;
        }
    }
}

// decode: work item = (request b, chunk of key tiles); rows = the Gq scored
// rows of the request (G queries, or its single proxy); scores spill.
template <typename T>
__global__ void __launch_bounds__(kSimtThreads) decode_simt_kernel(DecodeArgs a, int nchunks, long long ld) {
    extern __shared__ __align__(16) unsigned char smem[];
    const SimtSmem<T> L(a.H, a.d);
    T *qs = reinterpret_cast<T *>(smem + L.q_off);
    float *ks = reinterpret_cast<float *>(smem + L.k_off);
    float *wsm = reinterpret_cast<float *>(smem + L.w_off);
    const int HD = a.H * a.d;
    const int b = blockIdx.x / nchunks, ch = blockIdx.x % nchunks;
    const int kv = a.kv_len[b];
    if (kv < a.G || kv > a.n_max) return;  // the select pass flags the request
    const T *q = reinterpret_cast<const T *>(a.q) + (long long)b * a.Gq * HD;
    const T *kc = reinterpret_cast<const T *>(a.kc);
    load_rows(qs, q, a.Gq, HD);
    for (int i = threadIdx.x; i < RB * a.H; i += blockDim.x)
        wsm[i] = (i / a.H) < a.Gq ? a.w[(long long)b * a.Gq * a.H + i] : 0.0f;
    const int r = threadIdx.x >> 5;
    const bool row_ok = r < a.Gq;
    const int bound = !row_ok ? -1 : (a.Gq == 1 ? kv - 1 : kv - a.G + r);
    const int ntiles = (kv - 1) / KT + 1;
    const int t0 = ch * a.chunk_tiles;
    const int t1 = t0 + a.chunk_tiles < ntiles ? t0 + a.chunk_tiles : ntiles;
    float *out = a.spill + ((long long)b * a.Gq + r) * ld;
    for (int tile = t0; tile < t1; ++tile) {
        __syncthreads();
        const int s0 = tile * KT;
        int nvk = kv - s0;
        nvk = nvk > KT ? KT : nvk;
        for (int idx = threadIdx.x; idx < KT * a.d; idx += blockDim.x) {
            const int i = idx / a.d, e = idx - i * a.d;
            ks[i * (a.d + 1) + e] =
                i < nvk ? to_f(kc[cache_row(a.bt, a.page, a.max_pages, a.num_pages, a.n_max, b, s0 + i) * a.d + e])
                        : 0.0f;
        }
        __syncthreads();
        if (row_ok && s0 <= bound) {
            float sc[4];
            tile_scores(qs + r * HD, wsm + r * a.H, ks, a.H, a.d, sc);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                const int s = s0 + kb * 32 + (threadIdx.x & 31);
                if (s <= bound) out[s] = sc[kb];
            }
        }
    }
}

// Refine: work item = (group, chunk of up to RB members); the keys are the
// group's candidate positions; member scores go to out[member_row * c + j].
template <typename T>
__global__ void __launch_bounds__(kSimtThreads) gather_simt_kernel(GatherArgs a, int mchunks) {
    extern __shared__ __align__(16) unsigned char smem[];
    const SimtSmem<T> L(a.H, a.d);
    T *qs = reinterpret_cast<T *>(smem + L.q_off);
    float *ks = reinterpret_cast<float *>(smem + L.k_off);
    float *wsm = reinterpret_cast<float *>(smem + L.w_off);
    __shared__ int s_pos[KT];
    const int HD = a.H * a.d;
    const int grp = blockIdx.x / mchunks, mc = blockIdx.x % mchunks;
    long long mrow0, key0, sgrp, orow0;
    int nmem;
    if (a.mode == 0) {
        if (!a.plan[0] || grp >= a.plan[2]) return;
        const int *rp = a.plan + a.pl.rp();
        const int b = find_seg(rp, a.S, grp);
        const int i = grp - rp[b];
        const int n = a.cu[b + 1] - a.cu[b];
        // a member scored on its own needs no re-score; a group with no
        // output member has no candidate set
        if (i < dense_rows(n, a.g, a.db) || !row_in_range(a.plan, a.cu, b, i, n, a.g, a.db)) return;
        const int lo = group_start(i, n, a.g, a.db);
        const int cnt = group_size(i, n, a.g, a.db);
        mrow0 = (long long)a.cu[b] + lo + mc * RB;
        nmem = cnt - mc * RB;
        key0 = a.cu[b];
        sgrp = (long long)grp - a.plan[6];   // scratch rows of the call
        orow0 = mrow0 - a.plan[8];
    } else {
        const int kv = a.kv_len[grp];
        if (kv < a.G || kv > a.n_max) return;
        mrow0 = (long long)grp * a.G + mc * RB;
        nmem = a.G - mc * RB;
        key0 = (long long)grp * a.n_max;
        sgrp = grp;
        orow0 = mrow0;
    }
    if (nmem <= 0) return;
    if (nmem > RB) nmem = RB;
    const T *q = reinterpret_cast<const T *>(a.q) + mrow0 * HD;
    const T *k = reinterpret_cast<const T *>(a.k);
    load_rows(qs, q, nmem, HD);
    for (int i = threadIdx.x; i < RB * a.H; i += blockDim.x)
        wsm[i] = (i / a.H) < nmem ? a.w[mrow0 * a.H + i] : 0.0f;
    const int *cand = a.cand + sgrp * a.c;
    const int r = threadIdx.x >> 5;
    for (int j0 = 0; j0 < a.c; j0 += KT) {
        __syncthreads();
        for (int i = threadIdx.x; i < KT; i += blockDim.x) s_pos[i] = j0 + i < a.c ? cand[j0 + i] : -1;
        __syncthreads();
        for (int idx = threadIdx.x; idx < KT * a.d; idx += blockDim.x) {
            const int i = idx / a.d, e = idx - i * a.d;
            const int p = s_pos[i];
            const long long row = a.mode == 0 ? key0 + p
                                              : cache_row(a.bt, a.page, a.max_pages, a.num_pages, a.n_max, grp, p);
            ks[i * (a.d + 1) + e] = p >= 0 ? to_f(k[row * a.d + e]) : 0.0f;
        }
        __syncthreads();
        if (r < nmem) {
            float sc[4];
            tile_scores(qs + r * HD, wsm + r * a.H, ks, a.H, a.d, sc);
            float *out = a.out + (orow0 + r) * a.c;
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                const int j = j0 + kb * 32 + (threadIdx.x & 31);
                if (j < a.c) out[j] = sc[kb];
            }
        }
    }
}

template <typename K>
cudaError_t set_smem(K kern, size_t bytes) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

size_t simt_smem_bytes(int H, int d, int dtype) {
    return dtype == 1 ? SimtSmem<float>(H, d).total : SimtSmem<__nv_bfloat16>(H, d).total;
}

cudaError_t launch_score_simt(const ScoreArgs &a, int dtype, cudaStream_t st) {
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = simt_smem_bytes(a.H, a.d, dtype);
    cudaError_t e;
    TraceScope ts("score_simt", st);
    if (dtype == 1) {
        if ((e = set_smem(score_simt_kernel<float>, smem)) != cudaSuccess) return e;
        score_simt_kernel<float><<<sms * 2, kSimtThreads, smem, st>>>(a);
    } else {
        if ((e = set_smem(score_simt_kernel<__nv_bfloat16>, smem)) != cudaSuccess) return e;
        score_simt_kernel<__nv_bfloat16><<<sms * 2, kSimtThreads, smem, st>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_decode_simt(const DecodeArgs &a, int dtype, cudaStream_t st) {
    const int ntiles = (a.n_max + KT - 1) / KT;
    const int nchunks = (ntiles + a.chunk_tiles - 1) / a.chunk_tiles;
    const size_t smem = simt_smem_bytes(a.H, a.d, dtype);
    const long long ld = a.n_max;
    cudaError_t e;
    TraceScope ts("decode_simt", st);
    if (dtype == 1) {
        if ((e = set_smem(decode_simt_kernel<float>, smem)) != cudaSuccess) return e;
        decode_simt_kernel<float><<<a.B * nchunks, kSimtThreads, smem, st>>>(a, nchunks, ld);
    } else {
        if ((e = set_smem(decode_simt_kernel<__nv_bfloat16>, smem)) != cudaSuccess) return e;
        decode_simt_kernel<__nv_bfloat16><<<a.B * nchunks, kSimtThreads, smem, st>>>(a, nchunks, ld);
    }
    return cudaGetLastError();
}

cudaError_t launch_gather_simt(const GatherArgs &a, int dtype, cudaStream_t st) {
    const int gmax = a.mode == 0 ? a.g : a.G;
    const int mchunks = (gmax + RB - 1) / RB;
    const size_t smem = simt_smem_bytes(a.H, a.d, dtype);
    cudaError_t e;
    if (a.nitems <= 0) return cudaSuccess;
    TraceScope ts("gather_simt", st);
    if (dtype == 1) {
        if ((e = set_smem(gather_simt_kernel<float>, smem)) != cudaSuccess) return e;
        gather_simt_kernel<float><<<a.nitems * mchunks, kSimtThreads, smem, st>>>(a, mchunks);
    } else {
        if ((e = set_smem(gather_simt_kernel<__nv_bfloat16>, smem)) != cudaSuccess) return e;
        gather_simt_kernel<__nv_bfloat16><<<a.nitems * mchunks, kSimtThreads, smem, st>>>(a, mchunks);
    }
    return cudaGetLastError();
}

}  // namespace idx
