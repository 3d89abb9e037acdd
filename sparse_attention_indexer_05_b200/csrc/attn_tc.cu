// attn_tc.cu -- token-sparse attention over the selected positions, the
// consumer of the indexer's top-k sets (PIVOT page, introduction: the chosen
// set feeds sparse MLA attention).  Absorbed-MLA form: one latent row per key
// (Dqk = 576 dims) is the key and its first Dv = 512 dims the value, shared
// by all heads:
//     z_j   = scale * q[r,h] . kv[row_j],   row_j = cu_kv[b] + idx[r, j] (idx >= 0)
//     o[r,h] = sum_j softmax_j(z) * kv[row_j, :Dv],   lse[r,h] = log sum_j exp(z_j)
//
// A cluster of two CTAs per query row.  The 128 heads of the row are the
// MMA's M.  The 576 key dims are split between the pair: CTA 0 holds Q and
// gathers the keys of 64-dim slices 0..4, CTA 1 holds Q of slices 5..8 and
// gathers key slices 4..8, so that each also holds the value dims of its
// output half (CTA c writes value dims [256c, 256c+256)).  Per chunk of 32
// selected keys, in each CTA:
//   S_c = Q_c K_c^T   tcgen05, M=128, N=32, K=320 or 256   -> TMEM, 2 buffers
//   the partial S_c goes to the peer's shared memory (DSMEM) and the peer's
//   partial comes back; both add own + peer (the same fp32 sum on both sides)
//   P  = exp2(S*scale*log2e - m), m a running row maximum that is only moved
//        (and O rescaled in TMEM) when it grows by more than 8, so that P <= 2^8
//   O_c += P V_c      tcgen05, M=128, N=256, K=32            -> TMEM, 256 cols
// Both CTAs run the same softmax on the same S, so m, l and P agree.
// The key rows are gathered by TMA (tile::gather4: four rows of one 64-dim
// slice per request, 40 requests per chunk and CTA) into the
// 128-byte-swizzled K-major layout; the value operand is read from the same
// buffer through an MN-major descriptor.  Entries that are -1 or out of
// range load the request's first row (finite data) and get weight 0.  P goes
// to tensor memory as bf16 pairs and is the A operand of the second MMA there.
//
// Roles (512 threads per CTA): warp 0 = MMA issuer (one lane) and TMEM owner;
// warps 1..4 = receive, softmax and epilogue, one head row per thread (TMEM
// lane quarter = warp % 4); warps 5..8 = send (this CTA's partial S from TMEM
// to the staging buffer, ahead of the softmax); warps 9..13 = gather, one
// slice each; warp 14 = courier (send), warp 15 = courier (hand back)
// (one lane): one bulk shared-to-peer copy per chunk moves the staged partial
// S, and the buffer hand-back to the peer is one remote arrive.  Every wait
// is bounded; a cluster barrier after set-up and another before exit keep
// each CTA's shared memory alive while its peer may still write to it.
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace idx {

namespace {

constexpr int A_H = 128;                    // head rows on M (fewer heads: the rest is computed, not stored)
constexpr int A_DQK = 576;
constexpr int A_DV = 512;
constexpr int A_DVH = 256;                  // value dims per CTA
constexpr int A_KC = 32;                    // keys per chunk
constexpr int A_LS = 5;                     // 64-dim key slices gathered per CTA
constexpr int A_STAGES = 4;
constexpr uint32_t kQSlice = A_H * 128;              // 16 KB
constexpr uint32_t kQBytesMax = A_LS * kQSlice;      // 80 KB (CTA 0: 5 slices, CTA 1: 4)
constexpr uint32_t kKSlice = A_KC * 128;             // 4 KB
constexpr uint32_t kKStage = A_LS * kKSlice;         // 20 KB
constexpr uint32_t kXBytes = A_H * A_KC * 4;         // 16 KB: one chunk's partial S
constexpr int kSoftWarps = 4;   // receive, softmax, epilogue
constexpr int kSendWarps = 4;   // this CTA's partial S: TMEM -> staging buffer
constexpr int kGatherWarps = A_LS;
constexpr int kCourierWarp = 1 + kSoftWarps + kSendWarps + kGatherWarps;  // copies partial S to the peer
constexpr int kReturnWarp = kCourierWarp + 1;                                // hands receive buffers back
constexpr int kThreads = 32 * (kReturnWarp + 1);
constexpr uint32_t kColS = 0;               // S buffers: columns [0, 64)
constexpr uint32_t kColP = 64;              // P buffers (bf16 pairs): columns [64, 96)
constexpr uint32_t kColO = 256;             // O: columns [256, 512)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.0f;            // move the running max only past this growth (log2 units)

struct __align__(8) AttnShared {
    uint64_t qfull, kfull[A_STAGES], kempty[A_STAGES], sfull[2], sfree[2], pfull[2], pdone[2], drain;
    // exchange: xfull[b] = the peer's partial landed in xin[b] (transaction bytes);
    // xfree[b] = the peer read what this CTA sent into its xin[b] (remote arrive);
    // xready[b] = xout[b] holds this CTA's next partial; xout_free[b] = the copy
    // read xout[b]; xused[b] = this CTA's softmax threads read xin[b]
    uint64_t xfull[2], xfree[2], xready[2], xout_free[2], xused[2];
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kOffQ = 0;
constexpr size_t kOffK = kOffQ + kQBytesMax;
constexpr size_t kOffX = kOffK + (size_t)A_STAGES * kKStage;   // xin[2]: partials from the peer
constexpr size_t kOffXo = kOffX + 2 * (size_t)kXBytes;          // xout[2]: this CTA's partials, staged
constexpr size_t kOffCtl = kOffXo + 2 * (size_t)kXBytes;
constexpr size_t kSmemBytes = kOffCtl + sizeof(AttnShared) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory of one CTA");
static_assert(A_KC == 32, "one chunk position per lane of a gather warp");

// MN-major operand in the 128-byte swizzle: rows of 128 bytes along MN (64
// elements), 8 K-rows per 1024-byte atom; `lbo` = stride between 64-element
// MN blocks, 1024 B between 8-row K groups.
__device__ __forceinline__ uint64_t mnmajor_sw128_desc(uint32_t saddr, uint32_t lbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// four rows (r0..r3) of the 64-column box at column x, 128 bytes each, to
// four consecutive 128-byte rows at dst (tensor map box: 64 x 1)
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap *map, int x, int r0, int r1, int r2,
                                            int r3, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(tc::smem_u32(bar)), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
        : "memory");
}
// non-blocking test of an mbarrier phase (polling two barriers in turn)
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(tc::smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
// 16 consecutive 32-bit columns of the warp's 32 TMEM lanes (one lane per thread)
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
// D[tmem] (+)= A[tmem] * B: A (M x 16, bf16 pairs per 32-bit column, row = lane)
// in tensor memory, B by a shared-memory descriptor
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 2^x by the hardware approximation (ex2.approx.ftz: relative error far below
// the bf16 rounding of P that follows; 2^-inf = 0)
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// ------------------------------------------------ cluster (DSMEM) helpers
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of this CTA's shared address `saddr` in CTA `rank`
__device__ __forceinline__ uint32_t peer_addr(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
// arrive on an mbarrier of the peer CTA, releasing this thread's earlier writes at cluster scope
__device__ __forceinline__ void mbar_arrive_remote(uint32_t caddr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(tc::smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// bounded wait for a phase completed by the peer CTA (acquire at cluster scope)
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, volatile int *abort,
                                                  unsigned *status) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (unsigned it = 1;; ++it) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort) return false;
        if ((it & 31u) == 0u && globaltimer_ns() - t0 > kWaitNs) {
            *abort = 1;
            raise_status(status, ST_TIMEOUT);
            return false;
        }
    }
}
// this CTA's shared bytes [src, src+bytes) into the peer's shared memory at
// `dst`, completing `bytes` of transaction count on the peer's barrier `bar`
// (dst and bar are shared::cluster addresses)
__device__ __forceinline__ void bulk_to_peer(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "r"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until the committed bulk copies have read their source
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// wait until the committed bulk copies have completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The request of query row r and its key range; false for malformed
// boundaries (the row is then written as zeros and flagged).
__device__ __forceinline__ bool locate(const int *cu_q, const int *cu_kv, int S, int R, long long Nkv, int r,
                                      long long &kv0, int &nkv) {
    int lo = 0, hi = S;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cu_q[mid] <= r) lo = mid; else hi = mid;
    }
    const bool ok = cu_q[lo] <= r && r < cu_q[lo + 1] && cu_q[S] <= R && cu_kv[lo] >= 0 &&
                    cu_kv[lo] <= cu_kv[lo + 1] && (long long)cu_kv[lo + 1] <= Nkv;
    kv0 = ok ? cu_kv[lo] : 0;
    nkv = ok ? cu_kv[lo + 1] - cu_kv[lo] : 0;
    return ok;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_kv,
                   SparseAttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    // the same offset in both CTAs of the pair (same kernel, same shared layout)
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t *qs = smem + kOffQ;
    uint8_t *ks = smem + kOffK;
    uint8_t *xs = smem + kOffX;
    AttnShared &sh = *reinterpret_cast<AttnShared *>(smem + kOffCtl);
    volatile int *abort = &sh.abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t crank = cluster_rank();
    const uint32_t peer = crank ^ 1u;
    const int r = blockIdx.x >> 1;
    const int half = (int)crank;                 // value dims [256 * half, +256) are written here
    const int nq = crank == 0 ? 5 : 4;           // Q slices held here = key slices in this CTA's logits
    const int gq0 = crank == 0 ? 0 : 5;          // global slice of Q slot 0
    const int gk0 = crank == 0 ? 0 : 4;          // global slice of local key slice 0
    const int qk0 = crank == 0 ? 0 : 1;          // local key slice of Q slot 0
    const int nch = (a.topk + A_KC - 1) / A_KC;
    long long kv0;
    int nkv;
    const bool row_ok = locate(a.cu_q, a.cu_kv, a.S, a.R, a.Nkv, r, kv0, nkv);
    const int *ix = a.idx + (long long)r * a.topk;

    if (threadIdx.x == 0) {
        tc::mbar_init(&sh.qfull, 1);
        for (int s = 0; s < A_STAGES; ++s) {
            tc::mbar_init(&sh.kfull[s], kGatherWarps);
            tc::mbar_init(&sh.kempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&sh.sfull[b], 1);
            tc::mbar_init(&sh.sfree[b], 32 * (kSoftWarps + kSendWarps));  // both read S
            tc::mbar_init(&sh.xfull[b], 1);      // this CTA's courier (expected bytes) + the peer's copy
            tc::mbar_init(&sh.xfree[b], 1);      // the peer's courier
            tc::mbar_init(&sh.xused[b], 32 * kSoftWarps);
            tc::mbar_init(&sh.xready[b], 32 * kSendWarps);
            tc::mbar_init(&sh.xout_free[b], 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&sh.pfull[b], 32 * kSoftWarps);
            tc::mbar_init(&sh.pdone[b], 1);
        }
        tc::mbar_init(&sh.drain, 1);
        sh.abort = 0;
        tc::fence_mbar_init();
        // the first use of each receive buffer expects one partial (before the peer may send)
        for (int b = 0; b < 2; ++b)
            if (b < nch) tc::mbar_arrive_expect_tx(&sh.xfull[b], kXBytes);
        if (!row_ok && crank == 0) raise_status(a.status, ST_INVALID);
    }
    if (warp == 0) {
        tc::tmem_alloc(&sh.tmem_base, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before any remote arrive
    tc::fence_after_sync();
    const uint32_t tmem = sh.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            tc::prefetch_tmap(&tmap_q);
            tc::mbar_arrive_expect_tx(&sh.qfull, (uint32_t)nq * kQSlice);
            for (int s = 0; s < nq; ++s)
                tc::tma_load_2d(qs + s * kQSlice, &tmap_q, (gq0 + s) * 64, r * a.H, &sh.qfull);
            const uint32_t idesc_s = tc::idesc_bf16_f32(A_H, A_KC);
            const uint32_t idesc_o = tc::idesc_bf16_f32(A_H, A_DVH) | (1u << 16);  // value operand MN-major
            const uint32_t qa = tc::smem_u32(qs), ka = tc::smem_u32(ks);
            bool ok = tc::mbar_wait(&sh.qfull, 0, abort, a.status);
            // two independent streams: the partial logits of chunk jq (its keys have
            // landed and an S buffer is free) and O += P V of chunk jp (its P is
            // written); whichever is ready is issued
            int jq = 0, jp = 0;
            unsigned idle = 0;
            unsigned long long t_idle = 0;
            while (ok && jp < nch) {
                bool progressed = false;
                if (jq < nch) {
                    const int st = jq % A_STAGES, sb = jq & 1;
                    if (mbar_test(&sh.kfull[st], (jq / A_STAGES) & 1u) &&
                        mbar_test(&sh.sfree[sb], ((jq >> 1) & 1u) ^ 1u)) {
                        tc::fence_after_sync();
                        for (int kk = 0; kk < nq * 4; ++kk) {
                            const uint32_t off = (kk & 3) * 32u;  // 16-element K step inside the 128-byte row
                            const uint64_t ad = tc::sw128_desc(qa + (kk >> 2) * kQSlice + off);
                            const uint64_t bd =
                                tc::sw128_desc(ka + st * kKStage + (qk0 + (kk >> 2)) * kKSlice + off);
                            tc::mma_bf16(tmem + kColS + sb * A_KC, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                        }
                        tc::mma_commit(&sh.sfull[sb]);
                        ++jq;
                        progressed = true;
                    }
                }
                if (jp < jq && mbar_test(&sh.pfull[jp & 1], (jp >> 1) & 1u)) {
                    const int st = jp % A_STAGES;
                    tc::fence_after_sync();
                    const uint32_t vbase = ka + st * kKStage;  // local key slices 0..3 = this CTA's value dims
                    for (int kk = 0; kk < A_KC / 16; ++kk) {
                        // P (keys 16kk .. 16kk+15) = 8 columns of bf16 pairs in TMEM
                        const uint32_t at = tmem + kColP + (jp & 1) * (A_KC / 2) + kk * 8;
                        const uint64_t bd = mnmajor_sw128_desc(vbase + kk * 16u * 128u, kKSlice);
                        mma_bf16_ts(tmem + kColO, at, bd, idesc_o, (jp > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(&sh.kempty[st]);
                    tc::mma_commit(&sh.pdone[jp & 1]);
                    ++jp;
                    progressed = true;
                }
                if (progressed) {
                    idle = 0;
                } else if (*abort) {
                    ok = false;
                } else if (idle++ == 0) {
                    t_idle = globaltimer_ns();
                } else if ((idle & 63u) == 0 && globaltimer_ns() - t_idle > kWaitNs) {
                    *abort = 1;
                    raise_status(a.status, ST_TIMEOUT);
                    ok = false;
                }
            }
            // drain: every MMA issued so far has completed before TMEM is released
            tc::mma_commit(&sh.drain);
            tc::mbar_wait_drain(&sh.drain, 0);
            tc::mbar_wait_drain(&sh.qfull, 0);
        }
        __syncwarp();
    } else if (warp <= kSoftWarps) {
        // ------------------------------ exchange, softmax and epilogue
        const int quarter = warp & 3;
        const int h = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const float sl2 = a.scale * kLog2e;
        float m_used = -INFINITY, l = 0.0f;
        bool ok = true;
        uint32_t own[32];
        // the chunk's positions are loaded one chunk ahead (off the wait for S)
        int pos_next = lane < a.topk ? ix[lane] : -1;
        for (int j = 0; ok && j < nch; ++j) {
            const int xb = j & 1;
            const uint32_t use = (uint32_t)(j >> 1);  // use of exchange buffer xb
            const int pos = pos_next;
            if ((j + 1) * A_KC + lane < a.topk) pos_next = ix[(j + 1) * A_KC + lane];
            else pos_next = -1;
            // the peer's partial of chunk j and this CTA's own (read again from TMEM);
            // the sum is the same fp32 addition on both sides
            if (lane == 0)
                ok = tc::mbar_wait(&sh.xfull[xb], use & 1u, abort, a.status) &&
                     tc::mbar_wait(&sh.sfull[xb], use & 1u, abort, a.status);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) break;
            tc::fence_after_sync();
            tc::tmem_ld32(tmem + lane_off + kColS + xb * A_KC, own);
            tc::tmem_wait_ld(own);
            tc::fence_before_sync();
            tc::mbar_arrive(&sh.sfree[xb]);
            const uint4 *xr = reinterpret_cast<const uint4 *>(xs + xb * kXBytes + h * 128);
            float st_[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 v = xr[c ^ (h & 7)];
                st_[4 * c + 0] = __uint_as_float(own[4 * c + 0]) + __uint_as_float(v.x);
                st_[4 * c + 1] = __uint_as_float(own[4 * c + 1]) + __uint_as_float(v.y);
                st_[4 * c + 2] = __uint_as_float(own[4 * c + 2]) + __uint_as_float(v.z);
                st_[4 * c + 3] = __uint_as_float(own[4 * c + 3]) + __uint_as_float(v.w);
            }
            tc::mbar_arrive(&sh.xused[xb]);  // the courier tells the peer this buffer is free
            // which keys of the chunk are listed and inside the request
            const bool bad = pos >= nkv;
            if (bad && crank == 0 && quarter == 0) raise_status(a.status, ST_INVALID);
            const unsigned valid = __ballot_sync(0xFFFFFFFFu, row_ok && pos >= 0 && !bad);
            float x[32];
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                x[c] = (valid >> c) & 1u ? st_[c] * sl2 : -INFINITY;
                mx = fmaxf(mx, x[c]);
            }
            const bool need = mx > m_used + kRescale;
            const float factor = need ? fast_exp2(m_used - mx) : 1.0f;  // 0 while nothing was listed yet
            const float m_new = need ? mx : m_used;
            // masked entries are -inf and give 0; with nothing listed yet every
            // entry is masked and any finite reference serves
            const float m_ref = m_new == -INFINITY ? 0.0f : m_new;
            // weights and their bf16 packing do not depend on the previous chunk's P V
            uint32_t pk[16];
            float psum = 0.0f;
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
                const float p0 = fast_exp2(x[c] - m_ref);
                const float p1 = fast_exp2(x[c + 1] - m_ref);
                psum += p0 + p1;
                pk[c >> 1] = pack_bf16(p0, p1);
            }
            // P buffer j&1 is free once P V of chunk j-2 completed
            if (j >= 2) {
                if (lane == 0) ok = tc::mbar_wait(&sh.pdone[j & 1], ((j - 2) >> 1) & 1u, abort, a.status);
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) break;
            }
            const bool resc = j >= 1 && __any_sync(0xFFFFFFFFu, need);
            if (resc) {
                // O is rescaled only after every earlier P V completed (that of chunk j-1 last)
                if (lane == 0) ok = tc::mbar_wait(&sh.pdone[(j - 1) & 1], ((j - 1) >> 1) & 1u, abort, a.status);
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) break;
            }
            tc::fence_after_sync();
            if (resc) {
                uint32_t o[32];
                for (int b = 0; b < A_DVH / 32; ++b) {
                    tc::tmem_ld32(tmem + lane_off + kColO + b * 32, o);
                    tc::tmem_wait_ld(o);
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * factor);
                    tmem_st32(tmem + lane_off + kColO + b * 32, o);
                }
                tmem_wait_st();
            }
            l = l * factor + psum;
            m_used = m_new;
            // P row h into TMEM lane h: column i holds keys 2i, 2i+1 (bf16 pair)
            tmem_st16(tmem + lane_off + kColP + (j & 1) * (A_KC / 2), pk);
            tmem_wait_st();
            tc::fence_before_sync();
            tc::mbar_arrive(&sh.pfull[j & 1]);
        }
        // epilogue: O / l for this half of the value dims, lse from CTA 0
        if (ok && nch > 0) {
            if (lane == 0) ok = tc::mbar_wait(&sh.pdone[(nch - 1) & 1], ((nch - 1) >> 1) & 1u, abort, a.status);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        }
        if (ok) {
            tc::fence_after_sync();
            const float inv = l > 0.0f ? 1.0f / l : 0.0f;
            __nv_bfloat16 *orow =
                reinterpret_cast<__nv_bfloat16 *>(a.out) + ((long long)r * a.H + h) * A_DV + half * A_DVH;
            uint32_t o[32];
            for (int b = 0; b < A_DVH / 32; ++b) {
                tc::tmem_ld32(tmem + lane_off + kColO + b * 32, o);
                tc::tmem_wait_ld(o);
                if (h < a.H) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + b * 32);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint4 v;
                        v.x = pack_bf16(__uint_as_float(o[8 * q4 + 0]) * inv, __uint_as_float(o[8 * q4 + 1]) * inv);
                        v.y = pack_bf16(__uint_as_float(o[8 * q4 + 2]) * inv, __uint_as_float(o[8 * q4 + 3]) * inv);
                        v.z = pack_bf16(__uint_as_float(o[8 * q4 + 4]) * inv, __uint_as_float(o[8 * q4 + 5]) * inv);
                        v.w = pack_bf16(__uint_as_float(o[8 * q4 + 6]) * inv, __uint_as_float(o[8 * q4 + 7]) * inv);
                        dst[q4] = v;
                    }
                }
            }
            if (crank == 0 && h < a.H && a.lse)
                a.lse[(long long)r * a.H + h] = l > 0.0f ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
        }
    } else if (warp <= kSoftWarps + kSendWarps) {
        // --------------------- send: this CTA's partial S into the staging buffer
        // (runs ahead of the softmax, bounded by the two S buffers)
        const int quarter = warp & 3;
        const int h = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        // 16-byte piece c of row h stored at piece c ^ (h & 7): conflict-free row-per-thread access
        uint8_t *xo_row = smem + kOffXo + h * 128;  // + b * kXBytes
        bool ok = true;
        uint32_t own[32];
        for (int j = 0; ok && j < nch; ++j) {
            const int b = j & 1;
            if (lane == 0) ok = tc::mbar_wait(&sh.sfull[b], (j >> 1) & 1u, abort, a.status);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) break;
            tc::fence_after_sync();
            tc::tmem_ld32(tmem + lane_off + kColS + b * A_KC, own);
            tc::tmem_wait_ld(own);
            tc::fence_before_sync();
            tc::mbar_arrive(&sh.sfree[b]);
            // staging buffer b is free once the copy of chunk j-2 has read it
            if (lane == 0) ok = tc::mbar_wait(&sh.xout_free[b], ((j >> 1) & 1u) ^ 1u, abort, a.status);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) break;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4 *>(xo_row + b * kXBytes + ((c ^ (h & 7)) << 4)) =
                    make_uint4(own[4 * c], own[4 * c + 1], own[4 * c + 2], own[4 * c + 3]);
            fence_proxy_async();  // the copy reads the staging buffer through the async proxy
            tc::mbar_arrive(&sh.xready[b]);
        }
    } else if (warp < kCourierWarp) {
        // --------------------------------------- gather (TMA), one slice per warp
        const int gw = warp - (1 + kSoftWarps + kSendWarps);  // local key slice
        const int xcol = (gk0 + gw) * 64;         // its first column in the latent rows
        bool ok = true;
        int issued = 0;
        int pos_next = lane < a.topk ? ix[lane] : -1;  // positions one chunk ahead
        for (int j = 0; j < nch; ++j) {
            const int st = j % A_STAGES;
            const int pos = pos_next;
            pos_next = (j + 1) * A_KC + lane < a.topk ? ix[(j + 1) * A_KC + lane] : -1;
            if (lane == 0) ok = tc::mbar_wait(&sh.kempty[st], ((j / A_STAGES) & 1u) ^ 1u, abort, a.status);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) break;
            // lane i: row of chunk position i (the request's first row for entries not used)
            const bool valid = row_ok && pos >= 0 && pos < nkv;
            const int row = (int)(valid ? kv0 + pos : kv0);
            if (lane == 0) tc::mbar_arrive_expect_tx(&sh.kfull[st], kKSlice);
            __syncwarp();
            const int r0 = __shfl_sync(0xFFFFFFFFu, row, (lane & 7) * 4 + 0);
            const int r1 = __shfl_sync(0xFFFFFFFFu, row, (lane & 7) * 4 + 1);
            const int r2 = __shfl_sync(0xFFFFFFFFu, row, (lane & 7) * 4 + 2);
            const int r3 = __shfl_sync(0xFFFFFFFFu, row, (lane & 7) * 4 + 3);
            if (lane < 8)  // rows 4*lane .. 4*lane+3 of this slice
                tma_gather4(tc::smem_u32(ks + st * kKStage + gw * kKSlice) + lane * 4 * 128, &tmap_kv, xcol, r0, r1,
                            r2, r3, &sh.kfull[st]);
            issued = j + 1;
        }
        // teardown: the copies issued last land before shared memory is released
        if (lane == 0) {
            for (int j = (issued > A_STAGES ? issued - A_STAGES : 0); j < issued; ++j)
                tc::mbar_wait_drain(&sh.kfull[j % A_STAGES], (j / A_STAGES) & 1u);
        }
        __syncwarp();
    } else if (warp == kCourierWarp) {
        // ------------------------------------------- courier (one lane): send
        // each staged partial goes to the peer in one bulk DSMEM transfer
        if (lane == 0) {
            bool ok = true;
            for (int j = 0; ok && j < nch; ++j) {
                const int b = j & 1;
                const uint32_t u = (uint32_t)(j >> 1);
                if (!(ok = tc::mbar_wait(&sh.xready[b], u & 1u, abort, a.status))) break;
                // the peer read what was sent into its buffer b two chunks ago
                if (!(ok = mbar_wait_cluster(&sh.xfree[b], (u & 1u) ^ 1u, abort, a.status))) break;
                bulk_to_peer(peer_addr(tc::smem_u32(xs + b * kXBytes), peer), tc::smem_u32(smem + kOffXo + b * kXBytes),
                             kXBytes, peer_addr(tc::smem_u32(&sh.xfull[b]), peer));
                bulk_commit();
                bulk_wait_read_all();
                tc::mbar_arrive(&sh.xout_free[b]);
            }
            bulk_wait_all();  // this CTA's copies have landed in the peer
        }
        __syncwarp();
    } else {
        // ------------------------------------- courier (one lane): hand back
        // once this CTA's threads read a receive buffer, its next partial is
        // announced and the peer may send into it again
        if (lane == 0) {
            bool ok = true;
            for (int j = 0; ok && j < nch; ++j) {
                const int b = j & 1;
                if (!(ok = tc::mbar_wait(&sh.xused[b], (j >> 1) & 1u, abort, a.status))) break;
                if (j + 2 < nch) tc::mbar_arrive_expect_tx(&sh.xfull[b], kXBytes);
                mbar_arrive_remote(peer_addr(tc::smem_u32(&sh.xfree[b]), peer));
            }
        }
        __syncwarp();
    }

    tc::fence_before_sync();
    __syncthreads();
    cluster_sync();  // the peer no longer writes into this CTA's shared memory
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host
PFN_cuTensorMapEncodeTiled_v12000 encode_fn_attn() {
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

}  // namespace

bool attn_tc_supported(int H, int Dqk, int Dv, int dtype) {
    return H >= 1 && H <= A_H && Dqk == A_DQK && Dv == A_DV && dtype == 0;
}

cudaError_t launch_sparse_attn_tc(const SparseAttnArgs &a, cudaStream_t st) {
    if (a.R <= 0) return cudaSuccess;
    if (!attn_tc_supported(a.H, A_DQK, A_DV, 0)) return cudaErrorInvalidValue;
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn_attn();
    if (!fn) return cudaErrorInvalidValue;
    // q [R * H, 576] bf16 rows, boxes of 64 columns x 128 rows (one row's heads,
    // and for H < 128 rows of the next query or the zero fill past the end)
    CUtensorMap mq;
    memset(&mq, 0, sizeof(mq));
    cuuint64_t dims[2] = {(cuuint64_t)A_DQK, (cuuint64_t)a.R * a.H};
    cuuint64_t strides[1] = {(cuuint64_t)A_DQK * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)A_H};
    cuuint32_t estr[2] = {1u, 1u};
    if (fn(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(a.q), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    // kv [Nkv, 576] bf16 rows, gather boxes of 64 columns x 1 row
    CUtensorMap mkv;
    memset(&mkv, 0, sizeof(mkv));
    cuuint64_t kdims[2] = {(cuuint64_t)A_DQK, (cuuint64_t)a.Nkv};
    cuuint32_t kbox[2] = {64u, 1u};
    if (fn(&mkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(a.kv), kdims, strides, kbox, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    TraceScope ts("attn_tc", st);
    // a cluster of two CTAs per query row (compile-time cluster shape)
    attn_tc_kernel<<<(unsigned)(2LL * a.R), kThreads, kSmemBytes, st>>>(mq, mkv, a);
    return cudaGetLastError();
}

}  // namespace idx
