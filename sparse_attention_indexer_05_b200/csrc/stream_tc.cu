// stream_tc.cu -- tensor-core kernels that score up to 4 query rows (N =
// 64*m <= 256 columns) against a stream of key tiles and write every score:
//   * decode scan: the keys are the request's cache, streamed once by TMA
//     in 128-key tiles; rows = the request's G MTP queries (or its proxy);
//   * Refine re-score: the keys are a group's candidate set C, first packed
//     into a contiguous [c_pad, d] block per group by compact_keys_kernel
//     (coalesced 16-byte copies), then streamed by TMA like the decode
//     cache; rows = up to 4 members of the group.
// Same MMA shape as the prefill score kernel (keys on M, (row, head) on N,
// bf16 -> fp32 in TMEM, fused ReLU + w-weighted head sum), with the two
// 256-column TMEM buffers used alternately by consecutive key tiles.
#include <cudaTypedefs.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "plan.cuh"
#include "tc.cuh"

namespace idx {

namespace {

constexpr int S_H = 64;
constexpr int S_D = 128;
constexpr int kEpiWarps = 16;                    // 4 per TMEM lane quarter, one scored row each
constexpr int kThreads = 64 + 32 * kEpiWarps;    // + producer warp + MMA warp
constexpr int kStages = 4;
constexpr uint32_t kQSlice = 256 * 128;          // 256 rows x 64 bf16 (32 KB)
constexpr uint32_t kQBytes = 2 * kQSlice;        // 2 K slices
constexpr uint32_t kASlice = KT * 128;           // 128 keys x 64 bf16 (16 KB)
constexpr uint32_t kAStage = 2 * kASlice;        // one key tile (32 KB)
constexpr int kDecodeChunkTiles = 64;            // decode: key tiles per work item

struct __align__(8) StShared {
    uint64_t afull[kStages], aempty[kStages], qfull, tfull[2], tempty[2], drain;
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kOffQ = 0;
constexpr size_t kOffA = kOffQ + kQBytes;
constexpr int kMaxPageBoxes = kDecodeChunkTiles * (KT / 8);  // paged decode: boxes of >= 8 rows per item
constexpr size_t kOffW = kOffA + (size_t)kStages * kAStage;
constexpr size_t kOffPg = kOffW + 4 * S_H * 4;
constexpr size_t kOffCtl = kOffPg + (size_t)kMaxPageBoxes * 4;
constexpr size_t kSmemBytes = kOffCtl + sizeof(StShared) + 1024;

struct Item {
    bool valid;
    int m;              // rows scored (<= 4)
    long long qrow0;    // first query row (rows of [*, 64, 128])
    long long key0;     // first key row of the request
    int t0, nt;         // key tiles [t0, t0 + nt) of the item
    // outputs
    long long out_row0; // output row of scored row 0
    int bound0, bstep;  // decode: causal bound of row r = bound0 + bstep * r (inclusive)
};

template <bool GATHER>
__device__ __forceinline__ Item item_info(const GatherArgs &g, const DecodeArgs &dd, int item) {
    Item it{};
    it.valid = false;
    if (GATHER) {
        const int mchunks = ((g.mode == 0 ? g.g : g.G) + 3) / 4;
        const int grp = item / mchunks, mc = item % mchunks;
        long long m0, key0;
        int cnt;
        if (g.mode == 0) {
            if (!g.plan[0] || grp >= g.plan[2]) return it;
            const int *rp = g.plan + g.pl.rp();
            const int b = find_seg(rp, g.S, grp);
            const int i = grp - rp[b];
            const int n = g.cu[b + 1] - g.cu[b];
            // a member scored on its own needs no re-score; a group with no
            // output member has no candidate set
            if (i < dense_rows(n, g.g, g.db) || !row_in_range(g.plan, g.cu, b, i, n, g.g, g.db)) return it;
            const int lo = group_start(i, n, g.g, g.db);
            cnt = group_size(i, n, g.g, g.db);
            m0 = (long long)g.cu[b] + lo;
            key0 = g.cu[b];
        } else {
            const int kv = g.kv_len[grp];
            if (kv < g.G || kv > g.n_max) return it;
            cnt = g.G;
            m0 = (long long)grp * g.G;
            key0 = (long long)grp * g.n_max;
        }
        const int m = cnt - mc * 4;
        if (m <= 0) return it;
        (void)key0;
        it.valid = true;
        it.m = m < 4 ? m : 4;
        it.qrow0 = m0 + mc * 4;
        // prefill scratch: member scores from the call's first member,
        // packed keys from its first scored row
        it.out_row0 = it.qrow0 - (g.mode == 0 ? g.plan[8] : 0);
        it.key0 = ((long long)grp - (g.mode == 0 ? g.plan[6] : 0)) * g.c_pad;  // the group's packed keys
        it.t0 = 0;
        it.nt = g.c_pad / KT;
    } else {
        const int ntiles_max = (dd.n_max + KT - 1) / KT;
        const int nch = (ntiles_max + kDecodeChunkTiles - 1) / kDecodeChunkTiles;
        const int b = item / nch, ch = item % nch;
        const int kv = dd.kv_len[b];
        if (kv < dd.G || kv > dd.n_max) return it;
        const int ntiles = (kv - 1) / KT + 1;
        const int t0 = ch * kDecodeChunkTiles;
        if (t0 >= ntiles) return it;
        it.valid = true;
        it.m = dd.Gq;
        it.qrow0 = (long long)b * dd.Gq;
        it.out_row0 = it.qrow0;
        it.key0 = (long long)b * dd.n_max;
        it.t0 = t0;
        it.nt = (t0 + kDecodeChunkTiles < ntiles ? t0 + kDecodeChunkTiles : ntiles) - t0;
        it.bound0 = dd.Gq == 1 ? kv - 1 : kv - dd.G;
        it.bstep = dd.Gq == 1 ? 0 : 1;
    }
    return it;
}

// Packed (2 x fp32) fused multiply-add: acc.{x,y} = w.{x,y} * r.{x,y} + acc.{x,y},
// each lane of the pair rounded separately (the sm_100 fma.rn.f32x2).
__device__ __forceinline__ unsigned long long ffma2(unsigned long long acc, float w0, float w1, float r0, float r1) {
    unsigned long long wp, rp;
    asm("mov.b64 %0, {%1, %2};" : "=l"(wp) : "f"(w0), "f"(w1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(rp) : "f"(r0), "f"(r1));
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(wp), "l"(rp));
    return acc;
}

// v + |v| = 2 max(v, 0), exactly for every finite v below FLT_MAX / 2; an
// fp32 add on the FMA pipe instead of a max on the half-rate ALU pipe.
__device__ __forceinline__ float twice_relu(uint32_t x) {
    const float f = __uint_as_float(x);
    return f + fabsf(f);
}

// sum_j w[j] * max(v[j], 0) over 32 heads, given w2 = w / 2 (read as float4,
// 16-byte aligned): each term is w2[j] * (v[j] + |v[j]|), the same fp32
// product.  8 independent partial sums kept as 4 packed pairs, so each two
// heads cost two adds and one packed fma.
__device__ __forceinline__ float reduce32(const uint32_t (&v)[32], const float *w2) {
    const float4 *w4 = reinterpret_cast<const float4 *>(w2);
    unsigned long long a[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int j4 = 0; j4 < 8; ++j4) {
        const float4 wv = w4[j4];
        a[(2 * j4) & 3] = ffma2(a[(2 * j4) & 3], wv.x, wv.y, twice_relu(v[4 * j4 + 0]), twice_relu(v[4 * j4 + 1]));
        a[(2 * j4 + 1) & 3] =
            ffma2(a[(2 * j4 + 1) & 3], wv.z, wv.w, twice_relu(v[4 * j4 + 2]), twice_relu(v[4 * j4 + 3]));
    }
    float s[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) asm("mov.b64 {%0, %1}, %2;" : "=f"(s[2 * i]), "=f"(s[2 * i + 1]) : "l"(a[i]));
    return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
}

template <bool GATHER>
__global__ void __launch_bounds__(kThreads, 1)
    stream_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                     GatherArgs g, DecodeArgs dd, int nitems) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t *qs = smem + kOffQ;
    uint8_t *as = smem + kOffA;
    float *wsm = reinterpret_cast<float *>(smem + kOffW);
    int *pg_rows = reinterpret_cast<int *>(smem + kOffPg);  // paged decode: first pool row of each box
    StShared &sh = *reinterpret_cast<StShared *>(smem + kOffCtl);
    volatile int *abort = &sh.abort;
    unsigned *status = GATHER ? g.status : dd.status;
    const float *wsrc = GATHER ? g.w : dd.w;
    float *out = GATHER ? g.out : dd.spill;
    const long long ld = GATHER ? (long long)g.c : (long long)dd.n_max;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(&sh.afull[s], 1);
            tc::mbar_init(&sh.aempty[s], 1);
        }
        tc::mbar_init(&sh.qfull, 1);
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&sh.tfull[b], 1);
            tc::mbar_init(&sh.tempty[b], kEpiWarps);
        }
        tc::mbar_init(&sh.drain, 1);
        sh.abort = 0;
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tmap_q);
        tc::prefetch_tmap(&tmap_k);
    }
    if (warp == 1) {
        tc::tmem_alloc(&sh.tmem_base, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sh.tmem_base;

    uint32_t t = 0;     // key tiles consumed by this CTA (all roles agree)
    uint32_t nq = 0;    // query loads so far
    uint32_t mma_issued = 0;

    for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
        const Item it = item_info<GATHER>(g, dd, item);
        if (!it.valid) continue;
        __syncthreads();
        // the halved head weights (exact) of the item's rows, for reduce32
        for (int i = threadIdx.x; i < 4 * S_H; i += kThreads)
            wsm[i] = (i / S_H) < it.m ? 0.5f * wsrc[it.qrow0 * S_H + i] : 0.0f;
        __syncthreads();
        const uint32_t idesc = tc::idesc_bf16_f32(128, 64 * it.m);

        if (warp == 0) {
            bool ok = !*abort;
            const bool paged = !GATHER && dd.bt;
            const int box = paged && dd.page < KT ? dd.page : KT;  // rows per TMA box
            if (paged) {
                // the item's block-table lookups in one coalesced pass, off the issue path
                const int n = it.nt * (KT / box);
                const int b = (int)(it.qrow0 / dd.Gq);
                for (int i = lane; i < n; i += 32)
                    pg_rows[i] = (int)cache_row(dd.bt, dd.page, dd.max_pages, dd.num_pages, dd.n_max, b,
                                                it.t0 * KT + i * box);
                __syncwarp();
            }
            if (lane == 0 && ok) {
                tc::mbar_arrive_expect_tx(&sh.qfull, kQBytes);
                for (int kh = 0; kh < 2; ++kh)
                    tc::tma_load_2d(qs + kh * kQSlice, &tmap_q, kh * 64, (int)(it.qrow0 * S_H), &sh.qfull);
            }
            for (int j = 0; j < it.nt && ok; ++j) {
                const uint32_t tt = t + j, st = tt % kStages, ph = (tt / kStages) & 1u;
                if (lane == 0) ok = tc::mbar_wait(&sh.aempty[st], ph ^ 1u, abort, status);
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) break;
                uint8_t *dst = as + st * kAStage;
                if (lane == 0) {
                    tc::mbar_arrive_expect_tx(&sh.afull[st], kAStage);
                    if (!paged) {
                        const int row = (int)(it.key0 + (long long)(it.t0 + j) * KT);
                        for (int kh = 0; kh < 2; ++kh)
                            tc::tma_load_2d(dst + kh * kASlice, &tmap_k, kh * 64, row, &sh.afull[st]);
                    } else {
                        // paged cache: the tile's 128 positions are 128 / box boxes of whole pages
                        // (or one box inside a page); each box lands at its row offset in the stage
                        const int per = KT / box;
                        for (int i = 0; i < per; ++i)
                            for (int kh = 0; kh < 2; ++kh)
                                tc::tma_load_2d(dst + kh * kASlice + i * box * 128, &tmap_k, kh * 64,
                                                pg_rows[j * per + i], &sh.afull[st]);
                    }
                }
            }
        } else if (warp == 1) {
            if (lane == 0) {
                bool ok = tc::mbar_wait(&sh.qfull, nq & 1u, abort, status);
                const uint32_t qbase = tc::smem_u32(qs);
                for (int j = 0; j < it.nt && ok; ++j) {
                    const uint32_t tt = t + j, st = tt % kStages, ph = (tt / kStages) & 1u, buf = tt & 1u;
                    if (!(ok = tc::mbar_wait(&sh.afull[st], ph, abort, status))) break;
                    if (!(ok = tc::mbar_wait(&sh.tempty[buf], ((tt >> 1) & 1u) ^ 1u, abort, status))) break;
                    tc::fence_after_sync();
                    const uint32_t abase = tc::smem_u32(as + st * kAStage);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off_a = (kk >> 2) * kASlice + (kk & 3) * 32;
                        const uint32_t off_q = (kk >> 2) * kQSlice + (kk & 3) * 32;
                        tc::mma_bf16(tmem + buf * 256, tc::sw128_desc(abase + off_a), tc::sw128_desc(qbase + off_q),
                                     idesc, kk > 0 ? 1u : 0u);
                    }
                    ++mma_issued;
                    tc::mma_commit(&sh.tfull[buf]);
                    tc::mma_commit(&sh.aempty[st]);
                }
            }
        } else {
            const int quarter = warp & 3;
            const int r = (warp - 2) >> 2;  // the scored row of this warp
            const bool mine = r < it.m;
            bool ok = true;
            for (int j = 0; j < it.nt; ++j) {
                const uint32_t tt = t + j, buf = tt & 1u;
                if (ok) ok = tc::mbar_wait(&sh.tfull[buf], (tt >> 1) & 1u, abort, status);
                if (ok) {
                    tc::fence_after_sync();
                    const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + buf * 256 + r * 64;
                    // two 32-column halves, to keep the register footprint small
                    float part[2] = {0.0f, 0.0f};
                    if (mine) {
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            uint32_t v[32];
                            tc::tmem_ld32(taddr + hh * 32, v);
                            tc::tmem_wait_ld_all();
                            tc::reg_fence(v);
                            part[hh] = reduce32(v, wsm + r * S_H + hh * 32);
                        }
                    }
                    tc::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&sh.tempty[buf]);
                    if (mine) {
                        const float sc = part[0] + part[1];
                        const int kidx = quarter * 32 + lane;
                        if (GATHER) {
                            const int jj = j * KT + kidx;
                            if (jj < g.c) out[(it.out_row0 + r) * ld + jj] = sc;
                        } else {
                            const int s = (it.t0 + j) * KT + kidx;
                            if (s <= it.bound0 + it.bstep * r) out[(it.out_row0 + r) * ld + s] = sc;
                        }
                    }
                }
            }
        }
        t += it.nt;
        ++nq;
    }

    __syncthreads();
    if (*abort) {
        if (warp == 1 && lane == 0 && mma_issued) {
            tc::mma_commit(&sh.drain);
            tc::mbar_wait_drain(&sh.drain, 0);
        }
        if (warp == 0 && lane == 0) {
            for (uint32_t tt = t > kStages ? t - kStages : 0; tt < t; ++tt)
                tc::mbar_wait_drain(&sh.afull[tt % kStages], (tt / kStages) & 1u);
            if (nq) tc::mbar_wait_drain(&sh.qfull, (nq - 1) & 1u);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// Packs the key rows of every group's candidate set into a contiguous block
// of c_pad rows (padding slots and the -1 pads of short sets copy the
// request's row 0; their scores are written but never selected).
// Grid (groups, c_pad / 128); each CTA copies 128 rows of d bf16.
__global__ void __launch_bounds__(256) compact_keys_kernel(GatherArgs a) {
    const int grp = blockIdx.x;
    const int j0 = blockIdx.y * KT;
    long long key0;
    if (a.mode == 0) {
        if (!a.plan[0] || grp >= a.plan[2]) return;
        const int *rp = a.plan + a.pl.rp();
        const int b = find_seg(rp, a.S, grp);
        const int i = grp - rp[b], n = a.cu[b + 1] - a.cu[b];
        if (i < dense_rows(n, a.g, a.db) || !row_in_range(a.plan, a.cu, b, i, n, a.g, a.db)) return;  // no set
        key0 = a.cu[b];
    } else {
        const int kv = a.kv_len[grp];
        if (kv < a.G || kv > a.n_max) return;
        key0 = -1;  // decode: rows through cache_row
    }
    const long long sg = (long long)grp - (a.mode == 0 ? a.plan[6] : 0);  // the group's scratch row
    const int *cand = a.cand + sg * a.c;
    const int per_row = a.d * 2 / 16;  // 16-byte chunks per key row
    const uint4 *src = reinterpret_cast<const uint4 *>(a.k);
    uint4 *dst = reinterpret_cast<uint4 *>(a.ckeys) + (sg * a.c_pad + j0) * per_row;
    for (int u = threadIdx.x; u < KT * per_row; u += blockDim.x) {
        const int r = u / per_row, part = u - r * per_row;
        const int j = j0 + r;
        const int pos = j < a.c ? cand[j] : -1;
        const int p = pos >= 0 ? pos : 0;
        const long long row =
            key0 >= 0 ? key0 + p : cache_row(a.bt, a.page, a.max_pages, a.num_pages, a.n_max, grp, p);
        dst[u] = src[row * per_row + part];
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn2() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

bool map2d(CUtensorMap *m, const void *base, unsigned long long rows, unsigned box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn2();
    if (!fn) return false;
    memset(m, 0, sizeof(*m));
    cuuint64_t dims[2] = {(cuuint64_t)S_D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)S_D * 2};
    cuuint32_t box[2] = {64u, box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    return sms;
}

}  // namespace

bool tc_decode_supported(int H, int d, int dtype, int rows_per_request) {
    return H == S_H && d == S_D && dtype == 0 && rows_per_request >= 1 && rows_per_request <= 4;
}
bool tc_gather_supported(int H, int d, int dtype, int group, int c) {
    (void)group;
    return H == S_H && d == S_D && dtype == 0 && c >= 1;
}

cudaError_t launch_decode_tc(const DecodeArgs &a, cudaStream_t st) {
    if (a.bt && (a.page < 8 || (KT % a.page != 0 && a.page % KT != 0))) return cudaErrorInvalidValue;
    CUtensorMap mq, mk;
    const unsigned long long krows = a.bt ? (unsigned long long)a.num_pages * a.page : (unsigned long long)a.B * a.n_max;
    const unsigned box = a.bt && a.page < KT ? (unsigned)a.page : (unsigned)KT;
    if (!map2d(&mq, a.q, (unsigned long long)a.B * a.Gq * S_H, 256) || !map2d(&mk, a.kc, krows, box))
        return cudaErrorInvalidValue;
    const int ntiles_max = (a.n_max + KT - 1) / KT;
    const int nitems = a.B * ((ntiles_max + kDecodeChunkTiles - 1) / kDecodeChunkTiles);
    const size_t smem = kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(stream_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    GatherArgs g{};
    TraceScope ts("decode_tc", st);
    const int grid = nitems < sm_count() ? nitems : sm_count();
    stream_tc_kernel<false><<<grid, kThreads, smem, st>>>(mq, mk, g, a, nitems);
    return cudaGetLastError();
}

cudaError_t launch_gather_tc(const GatherArgs &a, cudaStream_t st) {
    const long long qrows = a.mode == 0 ? (long long)a.cu_T : (long long)a.G * a.nitems;
    const long long krows = a.ckey_groups * a.c_pad;  // packed candidate keys
    CUtensorMap mq, mk;
    if (!map2d(&mq, a.q, (unsigned long long)qrows * S_H, 256) || !map2d(&mk, a.ckeys, (unsigned long long)krows, KT))
        return cudaErrorInvalidValue;
    {
        TraceScope tsc("pack_keys", st);
        dim3 cgrid(a.nitems, a.c_pad / KT);
        compact_keys_kernel<<<cgrid, 256, 0, st>>>(a);
        cudaError_t ce = cudaGetLastError();
        if (ce != cudaSuccess) return ce;
    }
    const int mchunks = ((a.mode == 0 ? a.g : a.G) + 3) / 4;
    const int nitems = a.nitems * mchunks;
    const size_t smem = kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(stream_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    DecodeArgs dd{};
    TraceScope ts("gather_tc", st);
    const int grid = nitems < sm_count() ? nitems : sm_count();
    if (grid <= 0) return cudaSuccess;
    stream_tc_kernel<true><<<grid, kThreads, smem, st>>>(mq, mk, a, dd, nitems);
    return cudaGetLastError();
}

}  // namespace idx
