// proxy.cu -- PIVOT group proxies (PIVOT page, Experimental setup: the proxy
// is the mean of the group's queries; the mean of w is the reading used for
// the proxy's head weights).
//
// Per head and dimension: fp32 sum of the members in member order, one IEEE
// fp32 division by the group size, then round-to-nearest-even to bf16 for
// bf16 queries.  Loads are 16-byte vectors along the contiguous H*d axis.
#include "common.cuh"
#include "plan.cuh"

namespace idx {

namespace {

constexpr int kProxyThreads = 256;

template <typename T>
struct Vec;  // 8 elements per 16-byte load
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void load(const __nv_bfloat16 *p, float *f) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 t = __bfloat1622float2(h[i]);
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    }
    __device__ static void store(__nv_bfloat16 *p, const float *f) {
        uint4 v;
        __nv_bfloat16 *h = reinterpret_cast<__nv_bfloat16 *>(&v);
#pragma unroll
        for (int i = 0; i < 8; ++i) h[i] = __float2bfloat16_rn(f[i]);
        *reinterpret_cast<uint4 *>(p) = v;
    }
};
template <>
struct Vec<float> {
    static constexpr int N = 8;
    __device__ static void load(const float *p, float *f) {
        const float4 a = reinterpret_cast<const float4 *>(p)[0];
        const float4 b = reinterpret_cast<const float4 *>(p)[1];
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
    __device__ static void store(float *p, const float *f) {
        reinterpret_cast<float4 *>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
        reinterpret_cast<float4 *>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
};

// mean of cnt consecutive rows (row stride HD) -> one row
template <typename T>
__device__ void mean_rows(const T *src, const float *wsrc, int cnt, int HD, int H, T *dst, float *wdst) {
    const float fc = (float)cnt;
    for (int e = threadIdx.x * 8; e < HD; e += blockDim.x * 8) {
        float acc[8], v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        for (int m = 0; m < cnt; ++m) {
            Vec<T>::load(src + (long long)m * HD + e, v);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], v[i]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = __fdiv_rn(acc[i], fc);
        Vec<T>::store(dst + e, acc);
    }
    for (int j = threadIdx.x; j < H; j += blockDim.x) {
        float s = 0.0f;
        for (int m = 0; m < cnt; ++m) s = __fadd_rn(s, wsrc[(long long)m * H + j]);
        wdst[j] = __fdiv_rn(s, fc);
    }
}

template <typename T>
__global__ void __launch_bounds__(kProxyThreads) proxy_kernel(const T *q, const float *w, const int *cu, int S,
                                                              int H, int d, int g, const int *plan,
                                                              PlanLayout pl, T *qbar, float *wbar) {
    const int p = blockIdx.x;
    if (!plan[0] || p >= plan[2]) return;
    const int *rp = plan + pl.rp();
    const int b = find_seg(rp, S, p);
    const int i = p - rp[b];
    const int n = cu[b + 1] - cu[b];
    const int lo = i * g;
    const int cnt = (lo + g < n ? lo + g : n) - lo;
    const int HD = H * d;
    const long long m0 = (long long)cu[b] + lo;
    mean_rows(q + m0 * HD, w + m0 * H, cnt, HD, H, qbar + (long long)p * HD, wbar + (long long)p * H);
}

template <typename T>
__global__ void __launch_bounds__(kProxyThreads) decode_proxy_kernel(const T *q, const float *w, int G, int H,
                                                                     int d, T *qbar, float *wbar) {
    const int b = blockIdx.x;
    const int HD = H * d;
    mean_rows(q + (long long)b * G * HD, w + (long long)b * G * H, G, HD, H, qbar + (long long)b * HD,
              wbar + (long long)b * H);
}

}  // namespace

cudaError_t launch_proxy(const void *q, const float *w, const int *cu, int S, int T, int H, int d, int g,
                         int dtype, const int *plan, const PlanLayout &pl, void *qbar, float *wbar,
                         int max_proxies, cudaStream_t st) {
    (void)T;
    if (max_proxies <= 0) return cudaSuccess;
    TraceScope ts("proxy", st);
    if (dtype == 1)
        proxy_kernel<float><<<max_proxies, kProxyThreads, 0, st>>>(
            (const float *)q, w, cu, S, H, d, g, plan, pl, (float *)qbar, wbar);
    else
        proxy_kernel<__nv_bfloat16><<<max_proxies, kProxyThreads, 0, st>>>(
            (const __nv_bfloat16 *)q, w, cu, S, H, d, g, plan, pl, (__nv_bfloat16 *)qbar, wbar);
    return cudaGetLastError();
}

cudaError_t launch_decode_proxy(const void *q, const float *w, int B, int G, int H, int d, int dtype,
                                void *qbar, float *wbar, cudaStream_t st) {
    TraceScope ts("proxy", st);
    if (dtype == 1)
        decode_proxy_kernel<float><<<B, kProxyThreads, 0, st>>>((const float *)q, w, G, H, d, (float *)qbar,
                                                                wbar);
    else
        decode_proxy_kernel<__nv_bfloat16><<<B, kProxyThreads, 0, st>>>(
            (const __nv_bfloat16 *)q, w, G, H, d, (__nv_bfloat16 *)qbar, wbar);
    return cudaGetLastError();
}

}  // namespace idx
