// plan.cu -- validates cu_seqlens on the device and lays out the row blocks
// of a prefill score pass, ordered longest key range first so that the
// persistent score kernels finish together (longest-processing-time order).
#include "common.cuh"
#include "plan.cuh"

namespace idx {

namespace {

constexpr int kPlanThreads = 1024;

// block-wide inclusive scan of one int per thread (kPlanThreads threads)
__device__ int block_incl_scan(int v, int *warp_tot, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int u = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int t = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int u = __shfl_up_sync(0xFFFFFFFFu, t, o);
            if (lane >= o) t += u;
        }
        warp_tot[lane] = t;  // inclusive over warps
    }
    __syncthreads();
    if (warp > 0) v += warp_tot[warp - 1];
    *total = warp_tot[31];
    __syncthreads();
    return v;
}

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int *cu, int S, int T, int g, int db,
                                                            int row_lo, int row_hi, int *plan, PlanLayout pl,
                                                            unsigned *status) {
    __shared__ int s_bad;
    __shared__ int warp_tot[32];
    __shared__ int warp_tot2[32];
    const int tid = threadIdx.x;
    if (tid == 0) s_bad = (cu[0] != 0 || cu[S] != T) ? 1 : 0;
    __syncthreads();
    for (int b = tid; b < S; b += kPlanThreads) {
        const int n = cu[b + 1] - cu[b];
        if (n < 0 || n > kMaxLen) atomicOr(&s_bad, 1);
    }
    __syncthreads();
    if (s_bad) {
        if (tid == 0) {
            plan[0] = 0; plan[1] = 0; plan[2] = 0; plan[3] = 0; plan[4] = 0; plan[5] = 0;
            plan[6] = 0; plan[7] = 0; plan[8] = 0;
            raise_status(status, ST_INVALID);
        }
        return;
    }
    if (tid == 0) {
        plan[4] = row_lo;
        plan[5] = row_hi;
    }
    int *rp = plan + pl.rp();
    int *bp = plan + pl.bp();
    int carry_r = 0, carry_b = 0;
    for (int base = 0; base < S; base += kPlanThreads) {
        const int b = base + tid;
        const int r = b < S ? rows_of(cu[b + 1] - cu[b], g, db) : 0;
        const int nb = (r + RB - 1) / RB;
        int tot_r, tot_b;
        const int ir = block_incl_scan(r, warp_tot, &tot_r);
        const int ib = block_incl_scan(nb, warp_tot2, &tot_b);
        if (b < S) {
            rp[b] = carry_r + ir - r;
            bp[b] = carry_b + ib - nb;
        }
        carry_r += tot_r;
        carry_b += tot_b;
    }
    const int nblocks = carry_b;
    __syncthreads();  // every rp[b] is written
    if (tid == 0) {
        rp[S] = carry_r;
        bp[S] = carry_b;
        plan[2] = carry_r;
        plan[3] = 0;
        // the scored rows holding the first and the last output row
        int plo = 0, phi = 0, mlo = 0;
        if (row_lo < row_hi) {
            const int b0 = find_seg(cu, S, row_lo), b1 = find_seg(cu, S, row_hi - 1);
            const int n0 = cu[b0 + 1] - cu[b0];
            const int i0 = group_of(row_lo - cu[b0], n0, g, db);
            plo = rp[b0] + i0;
            mlo = cu[b0] + group_start(i0, n0, g, db);
            phi = rp[b1] + group_of(row_hi - 1 - cu[b1], cu[b1 + 1] - cu[b1], g, db) + 1;
        }
        plan[6] = plo;
        plan[7] = phi;
        plan[8] = mlo;
    }
    int *hist = plan + pl.hist();
    for (int i = tid; i <= pl.maxtiles; i += kPlanThreads) hist[i] = 0;
    __syncthreads();
    // a row block is scheduled when the members of its scored rows (a
    // contiguous run of tokens) meet [row_lo, row_hi)
    auto scheduled = [&](const BlockInfo &bi) {
        const int il = bi.i0 + bi.nrows - 1;
        const long long lo = (long long)cu[bi.b] + group_start(bi.i0, bi.n, g, db);
        const long long hi = (long long)cu[bi.b] + group_start(il, bi.n, g, db) + group_size(il, bi.n, g, db);
        return bi.nrows > 0 && hi > row_lo && lo < row_hi;
    };
    for (int blk = tid; blk < nblocks; blk += kPlanThreads) {
        const BlockInfo bi = block_info(plan, pl, cu, g, blk, 0, db);
        if (!scheduled(bi)) continue;
        const int t = bi.ntiles < pl.maxtiles ? bi.ntiles : pl.maxtiles;
        atomicAdd(&hist[t], 1);
    }
    __syncthreads();
    // start[t] = number of blocks with more tiles than t (descending order)
    if (tid == 0) {
        int run = 0;
        for (int t = pl.maxtiles; t >= 0; --t) {
            const int h = hist[t];
            hist[t] = run;
            run += h;
        }
        plan[1] = run;
    }
    __syncthreads();
    int *order = plan + pl.order();
    for (int blk = tid; blk < nblocks; blk += kPlanThreads) {
        const BlockInfo bi = block_info(plan, pl, cu, g, blk, 0, db);
        if (!scheduled(bi)) continue;
        const int t = bi.ntiles < pl.maxtiles ? bi.ntiles : pl.maxtiles;
        order[atomicAdd(&hist[t], 1)] = blk;
    }
    if (tid == 0) plan[0] = 1;
}

}  // namespace

cudaError_t launch_plan(const int *cu, int S, int T, int g, int db, int row_lo, int row_hi, int *plan,
                        const PlanLayout &pl, unsigned *status, cudaStream_t st) {
    TraceScope ts("plan", st);
    plan_kernel<<<1, kPlanThreads, 0, st>>>(cu, S, T, g, db, row_lo, row_hi, plan, pl, status);
    return cudaGetLastError();
}

}  // namespace idx
