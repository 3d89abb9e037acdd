// score_tc.cu -- tensor-core score kernel for bf16 inputs with H = 64 heads
// and d = 128: the contraction Q(H*d) x K^T on tcgen05 with the per-head
// ReLU and the w-weighted head sum fused into the epilogue, so the L x L x H
// tensor of per-head dot products never leaves the SM.
//
// Layout of one MMA: keys on M (128 keys of a key tile, one TMEM lane per
// key) and (query, head) pairs on N (4 queries x 64 heads = 256 columns),
// K = d = 128 in 8 steps of 16.  A row block holds 8 scored rows split in
// two halves of 4; the two halves use the two 256-column halves of TMEM and
// share every key tile that TMA brings in, so each key byte fetched feeds
// 8 queries.  The epilogue of one half overlaps the MMA of the other.
//
// Roles (576 threads): warp 0 = TMA producer (one lane), warp 1 = MMA issuer
// (one lane; the whole warp allocates TMEM), warps 2..17 = epilogue in four
// roles of four warps, one warp per TMEM lane quarter (warp % 4: keys
// 32*(warp%4) .. +31 of the tile).  Role p owns rows 2p, 2p+1, two queries
// of half p/2, so half-0 and half-1 roles run offset by one MMA half and
// their ALU-heavy reductions interleave with the other half's waits and
// loads.  Each thread reduces, per row, the 64 head dot products of its key:
//     I = sum_j w_j * max(dot_j, 0)      (8 partial sums, fixed order),
// computed as (w_j / 2) * (dot_j + |dot_j|), the same value bit for bit
// (dot + |dot| is 2 max(dot, 0) exactly; halving w is exact), which keeps the
// max off the ALU pipe.
// The scores go to the same sinks as the CUDA-core kernel: the streaming
// candidate filter (common.cuh) or a spill of full score rows (debug export).
#include <cudaTypedefs.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "plan.cuh"
#include "tc.cuh"

namespace idx {

namespace {

constexpr int TC_H = 64;
constexpr int TC_D = 128;
constexpr int kEpiWarps = 16;                         // 4 per TMEM lane quarter, one query each per half
constexpr int kThreads = 64 + 32 * kEpiWarps;         // + TMA warp + MMA warp
constexpr int kMaintEvery = 8;                        // tiles between candidate-filter upkeeps
constexpr int kStages = 2;                            // key-tile stages
constexpr uint32_t kQHalfBytes = 256 * 128;           // one half, one 64-column K slice (32 KB)
constexpr uint32_t kQBytes = 4 * kQHalfBytes;         // 2 halves x 2 K slices (128 KB)
constexpr uint32_t kKSliceBytes = KT * 128;           // 128 keys x 64 bf16 (16 KB)
constexpr uint32_t kKStageBytes = 2 * kKSliceBytes;   // one key tile (32 KB)
constexpr uint32_t kIdesc = tc::idesc_bf16_f32(128, 256);

struct __align__(8) TcShared {
    uint64_t kfull[kStages], kempty[kStages], qfull, tfull[2], tempty[2], drain;
    uint32_t tmem_base;
    int item;
    int abort;
    int row0, nrows, i0, n, ntiles;
    long long key0;
    int bound[RB];
    int slot[RB];
    RowSel sel[RB];
};

constexpr size_t kOffQ = 0;
constexpr size_t kOffK = kOffQ + kQBytes;
constexpr size_t kOffW = kOffK + (size_t)kStages * kKStageBytes;
constexpr size_t kOffHist = kOffW + (size_t)RB * TC_H * 4;
constexpr size_t kOffScr = kOffHist + (size_t)RB * kBins * 4;
constexpr size_t kOffCtl = kOffScr + (size_t)RB * 256 * 4;
constexpr size_t kSmemBytes = kOffCtl + sizeof(TcShared) + 1024;  // + alignment slack

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

// sum_j w[j] * max(v[j], 0) over 64 heads held in two 32-register groups,
// given w2 = w / 2 (read as float4, 16-byte aligned): each term is
// w2[j] * (v[j] + |v[j]|), the same fp32 product.  8 independent partial sums
// kept as 4 packed pairs, so each two heads cost two adds and one packed fma.
__device__ __forceinline__ float head_reduce(const uint32_t (&v0)[32], const uint32_t (&v1)[32], const float *w2) {
    const float4 *w4 = reinterpret_cast<const float4 *>(w2);
    unsigned long long a[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int j4 = 0; j4 < 8; ++j4) {
        const float4 wv = w4[j4];
        a[(2 * j4) & 3] = ffma2(a[(2 * j4) & 3], wv.x, wv.y, twice_relu(v0[4 * j4 + 0]), twice_relu(v0[4 * j4 + 1]));
        a[(2 * j4 + 1) & 3] =
            ffma2(a[(2 * j4 + 1) & 3], wv.z, wv.w, twice_relu(v0[4 * j4 + 2]), twice_relu(v0[4 * j4 + 3]));
    }
#pragma unroll
    for (int j4 = 0; j4 < 8; ++j4) {
        const float4 wv = w4[8 + j4];
        a[(2 * j4) & 3] = ffma2(a[(2 * j4) & 3], wv.x, wv.y, twice_relu(v1[4 * j4 + 0]), twice_relu(v1[4 * j4 + 1]));
        a[(2 * j4 + 1) & 3] =
            ffma2(a[(2 * j4 + 1) & 3], wv.z, wv.w, twice_relu(v1[4 * j4 + 2]), twice_relu(v1[4 * j4 + 3]));
    }
    float s[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) asm("mov.b64 {%0, %1}, %2;" : "=f"(s[2 * i]), "=f"(s[2 * i + 1]) : "l"(a[i]));
    return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
}

__global__ void __launch_bounds__(kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                    ScoreArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t *qs = smem + kOffQ;
    uint8_t *ks = smem + kOffK;
    float *wsm = reinterpret_cast<float *>(smem + kOffW);
    unsigned *hist = reinterpret_cast<unsigned *>(smem + kOffHist);
    unsigned *scr = reinterpret_cast<unsigned *>(smem + kOffScr);
    TcShared &sh = *reinterpret_cast<TcShared *>(smem + kOffCtl);
    volatile int *abort = &sh.abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    int *plan = const_cast<int *>(a.plan);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(&sh.kfull[s], 1);
            tc::mbar_init(&sh.kempty[s], 1);
        }
        tc::mbar_init(&sh.qfull, 1);
        for (int h = 0; h < 2; ++h) {
            tc::mbar_init(&sh.tfull[h], 1);
            tc::mbar_init(&sh.tempty[h], kEpiWarps / 2);
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

    const bool valid_plan = plan[0] != 0;
    const int nblocks = valid_plan ? plan[1] : 0;
    unsigned *work = reinterpret_cast<unsigned *>(plan + 3);

    uint32_t kt = 0;   // key tiles processed by this CTA so far (all roles agree)
    uint32_t nb = 0;   // row blocks processed so far
    // producer bookkeeping for the teardown drain
    uint32_t issued_q = 0;
    uint32_t mma_issued = 0;

    for (;;) {
        __syncthreads();
        if (threadIdx.x == 0) sh.item = (int)atomicAdd(work, 1u);
        __syncthreads();
        const int item = sh.item;
        if (item >= nblocks) break;
        const BlockInfo bi = block_info(plan, a.pl, a.cu, a.g, plan[a.pl.order() + item], a.kshift, a.db);
        const int ntiles = bi.ntiles;

        if (warp >= 2) {
            const int e = warp - 2;
            // halved head weights of the block's rows, zero for rows past the request
            for (int i = threadIdx.x - 64; i < RB * TC_H; i += kEpiWarps * 32)
                wsm[i] = (i / TC_H) < bi.nrows ? 0.5f * a.w[(long long)bi.row0 * TC_H + i] : 0.0f;
            if (e < RB) {
                if (lane == 0) {
                    // a filtered row whose members are all outside the call's
                    // output rows is not ranked (it has no scratch row)
                    const bool act = e < bi.nrows && (a.sink != SINK_FILTER || scored_in_range(plan, bi.row0 + e));
                    sh.bound[e] = act ? key_bound(row_bound(bi.i0 + e, bi.n, a.g, a.db), a.kshift) : -1;
                    sh.slot[e] = -1;
                    if (a.sink == SINK_SPILL && e < bi.nrows && a.slot_of_row)
                        sh.slot[e] = a.slot_of_row[bi.row0 + e];
                }
                if (a.sink == SINK_FILTER) sel_init(sh.sel[e], hist + e * kBins);
            }
        }
        __syncthreads();

        if (warp == 0) {
            if (lane == 0 && !*abort) {
                // queries of the block: 8 rows x 64 heads = 512 rows of the [R*64, 128] view
                tc::mbar_arrive_expect_tx(&sh.qfull, kQBytes);
                for (int h = 0; h < 2; ++h)
                    for (int kh = 0; kh < 2; ++kh)
                        tc::tma_load_2d(qs + (h * 2 + kh) * kQHalfBytes, &tmap_q, kh * 64,
                                        (bi.row0 + 4 * h) * TC_H, &sh.qfull);
                ++issued_q;
                for (int j = 0; j < ntiles; ++j) {
                    const uint32_t t = kt + j, st = t % kStages, ph = (t / kStages) & 1u;
                    if (!tc::mbar_wait(&sh.kempty[st], ph ^ 1u, abort, a.status)) break;
                    tc::mbar_arrive_expect_tx(&sh.kfull[st], kKStageBytes);
                    for (int kh = 0; kh < 2; ++kh)
                        tc::tma_load_2d(ks + st * kKStageBytes + kh * kKSliceBytes, &tmap_k, kh * 64,
                                        (int)(bi.key0 + (long long)j * KT), &sh.kfull[st]);
                }
            }
        } else if (warp == 1) {
            if (lane == 0) {
                bool ok = tc::mbar_wait(&sh.qfull, nb & 1u, abort, a.status);
                for (int j = 0; j < ntiles && ok; ++j) {
                    const uint32_t t = kt + j, st = t % kStages, ph = (t / kStages) & 1u;
                    if (!(ok = tc::mbar_wait(&sh.kfull[st], ph, abort, a.status))) break;
                    tc::fence_after_sync();
                    const uint32_t kbase = tc::smem_u32(ks + st * kKStageBytes);
                    for (int h = 0; h < 2; ++h) {
                        if (!(ok = tc::mbar_wait(&sh.tempty[h], (t & 1u) ^ 1u, abort, a.status))) break;
                        tc::fence_after_sync();
                        const uint32_t qbase = tc::smem_u32(qs + h * 2 * kQHalfBytes);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t koff = (kk >> 2) * kKSliceBytes + (kk & 3) * 32;
                            const uint32_t qoff = (kk >> 2) * kQHalfBytes + (kk & 3) * 32;
                            tc::mma_bf16(tmem + h * 256, tc::sw128_desc(kbase + koff), tc::sw128_desc(qbase + qoff),
                                         kIdesc, kk > 0 ? 1u : 0u);
                        }
                        ++mma_issued;
                        tc::mma_commit(&sh.tfull[h]);
                    }
                    if (!ok) break;
                    tc::mma_commit(&sh.kempty[st]);
                }
            }
        } else {
            // epilogue role: warps 2+4*role .. 5+4*role (one per TMEM lane
            // quarter) own rows 2*role, 2*role+1 -- two queries of half role/2
            const int e = warp - 2;
            const int role = e >> 2;
            const int h = role >> 1;
            const int ra = 2 * role;             // first of the role's two rows (h*4 + query)
            const int quarter = warp & 3;
            const int key_in_tile = quarter * 32 + lane;
            const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(ra * 64);
            const bool filter = a.sink == SINK_FILTER;
            const int mrow = ra + (e & 1);       // row this warp maintains (warps with e & 3 < 2)
            const bool maint = (e & 3) < 2 && mrow < bi.nrows && (!filter || scored_in_range(plan, bi.row0 + mrow));
            // scratch rows start at the call's first scored row
            unsigned long long *buf0 = filter ? a.buf + ((long long)bi.row0 - plan[6]) * a.cap : nullptr;
            const long long srow0 = (long long)bi.row0 - plan[6];
            bool ok = true;
            for (int j = 0; j < ntiles; ++j) {
                const uint32_t t = kt + j;
                const int s = j * KT + key_in_tile;
                if (ok) ok = tc::mbar_wait(&sh.tfull[h], t & 1u, abort, a.status);
                if (ok) tc::fence_after_sync();
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    float score = 0.0f;
                    const int r = ra + q;
                    if (ok) {
                        uint32_t v0[32], v1[32];
                        tc::tmem_ld32(tbase + q * 64, v0);
                        tc::tmem_ld32(tbase + q * 64 + 32, v1);
                        tc::tmem_wait_ld_all();
                        tc::reg_fence(v0);
                        tc::reg_fence(v1);
                        if (q == 1) {
                            tc::fence_before_sync();
                            __syncwarp();
                            tc::mbar_arrive_if(&sh.tempty[h], lane == 0);
                        }
                        score = head_reduce(v0, v1, wsm + r * TC_H);
                    }
                    const bool valid = ok && s <= sh.bound[r];
                    if (filter) {
                        sel_offer(sh.sel[r], hist + r * kBins, buf0 + (long long)r * a.cap, a.cap, valid, score, s,
                                  a.status);
                    } else if (valid && sh.slot[r] >= 0) {
                        a.spill[(long long)sh.slot[r] * a.ld + s] = score;
                    }
                }
                if (filter && ((j % kMaintEvery) == kMaintEvery - 1 || j == ntiles - 1)) {
                    tc::named_bar_sync(1 + role, 128);
                    if (maint)
                        sel_maintain(sh.sel[mrow], hist + mrow * kBins, buf0 + (long long)mrow * a.cap, a.cap,
                                     bi.i0 + mrow < dense_rows(bi.n, a.g, a.db) ? a.ksel_dense : a.ksel,
                                     scr + mrow * 256, KT * kMaintEvery);
                    tc::named_bar_sync(1 + role, 128);
                }
            }
            if (filter && maint && lane == 0) {
                a.cnt[srow0 + mrow] = sh.sel[mrow].cnt;
                if (a.floor_out) a.floor_out[srow0 + mrow] = sh.sel[mrow].floor;
            }
        }
        kt += ntiles;
        ++nb;
    }

    // teardown: after a timeout let every copy and MMA in flight finish
    // (bounded), then release TMEM.
    __syncthreads();
    if (*abort) {
        if (warp == 0 && lane == 0) {
            // the last armed phase of every barrier TMA completes
            if (issued_q) tc::mbar_wait_drain(&sh.qfull, (nb - 1) & 1u);
            for (uint32_t t = kt > kStages ? kt - kStages : 0; t < kt; ++t)
                tc::mbar_wait_drain(&sh.kfull[t % kStages], (t / kStages) & 1u);
        }
        if (warp == 1 && lane == 0 && mma_issued) {
            tc::mma_commit(&sh.drain);
            tc::mbar_wait_drain(&sh.drain, 0);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// [rows, 128] bf16 row-major, boxes of 64 columns x box_rows rows, 128 B swizzle
bool make_map(CUtensorMap *m, const void *base, unsigned long long rows, unsigned box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return false;
    memset(m, 0, sizeof(*m));
    cuuint64_t dims[2] = {(cuuint64_t)TC_D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)TC_D * 2};
    cuuint32_t box[2] = {64u, box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int num_sms() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    return sms;
}

}  // namespace

bool tc_supported(int H, int d, int dtype) { return H == TC_H && d == TC_D && dtype == 0; }

cudaError_t launch_score_tc(const ScoreArgs &a, cudaStream_t st) {
    // the scored tensor [R, 64, 128] viewed as [R*64, 128]; keys [T, 128]
    CUtensorMap mq, mk;
    const unsigned long long krows =
        a.kshift ? ((a.T >> a.kshift) > 0 ? (unsigned long long)(a.T >> a.kshift) : 1ull) : (unsigned long long)a.T;
    if (!make_map(&mq, a.q, (unsigned long long)a.R * TC_H, 256) || !make_map(&mk, a.k, krows, KT))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(score_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    TraceScope ts("score_tc", st);
    score_tc_kernel<<<num_sms(), kThreads, kSmemBytes, st>>>(mq, mk, a);
    return cudaGetLastError();
}


}  // namespace idx
