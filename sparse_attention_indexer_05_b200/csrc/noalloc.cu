// noalloc.cu -- a decode entry point for callers that cannot allocate device
// memory.
//
// Some callers only ever see input and output buffers: a plugin running
// inside another runtime that owns all device memory and hands out no
// workspace, or a serving loop whose memory plan forbids any allocation
// once decoding has started.  They cannot call cudaMalloc (or a caching
// allocator) to obtain the workspace that idx_decode_topk needs.
// idx_decode_topk_noalloc serves them: its scratch (the status word and
// the per-query score rows of the dense decode scan) lives in the
// file-scope device array below, which the CUDA runtime reserves on every
// GPU that loads this library, for as long as the process lives.
#include <stdio.h>

#include "../../include/idx.h"
#include "internal.h"

namespace {

// The whole scratch of one call: 256 bytes of status/padding, then
// B*G*n_max fp32 score rows (see decode_ws in api.cu for the layout).
constexpr size_t kNoAllocScratchBytes = (size_t)32 << 20;  // 32 MiB per GPU

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices] = {nullptr};

// The device address of g_noalloc_scratch on the current device.  In host
// code the array's name is only a host-side handle, so the address is
// asked from the runtime once per device (with that device current) and
// kept.  Returns nullptr on failure.
void *scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_scratch_addr[dev] = p;
    }
    return g_scratch_addr[dev];
}

}  // namespace

extern "C" idx_status idx_decode_topk_noalloc(const void *q, const void *kcache, const int *kv_len,
                                              const float *w, int B, int G, int n_max, int H, int d,
                                              int topk, idx_dtype dtype, int *out_idx, float *out_score,
                                              idx_stream_t stream) {
    const size_t need = idx_decode_workspace_size(B, G, n_max, H, d, topk, 0, IDX_MODE_DENSE, dtype);
    if (need == 0) return IDX_ERR_INVALID;
    if (need > kNoAllocScratchBytes) {
        fprintf(stderr,
                "idx_decode_topk_noalloc: B*G*n_max = %lld score rows need %zu bytes of scratch, "
                "more than the fixed %zu bytes; use idx_decode_topk with a workspace\n",
                (long long)B * G * n_max, need, kNoAllocScratchBytes);
        return IDX_ERR_UNSUPPORTED;
    }
    void *ws = scratch_address();
    if (!ws) return IDX_ERR_CUDA;
    // idx_decode_topk clears the status word before its kernels run; every
    // score the select pass reads is written by the scan first.
    return idx_decode_topk(q, kcache, kv_len, w, B, G, n_max, H, d, topk, 0, IDX_MODE_DENSE, dtype, out_idx,
                           out_score, ws, kNoAllocScratchBytes, stream);
}
