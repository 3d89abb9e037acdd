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
#include <cuda.h>
#include <stdio.h>

#include <mutex>

#include "../../include/idx.h"
#include "internal.h"

namespace {

// The whole scratch of one call: 256 bytes of status/padding, then
// B*G*n_max fp32 score rows (see decode_ws in api.cu for the layout).
constexpr size_t kNoAllocScratchBytes = (size_t)32 << 20;  // 32 MiB per GPU

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch, per device ordinal, together with
// the id of the context it was looked up in.  The array belongs to the
// module loaded into a context: after a device reset (or any teardown of
// the primary context) the module is loaded again and the array may sit
// elsewhere, so a cached address is used only while the current context
// is the one it came from.  All of it is guarded by one mutex, so first
// calls from several host threads do not race.
constexpr int kMaxDevices = 64;
struct ScratchSlot {
    unsigned long long ctx_id;
    void *addr;
};
std::mutex g_scratch_mu;
ScratchSlot g_scratch[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;
bool g_ctx_fns_tried = false;

// Driver entry points for the current context and its unique id (called
// with g_scratch_mu held).
void resolve_ctx_fns() {
    if (g_ctx_fns_tried) return;
    g_ctx_fns_tried = true;
    cudaDriverEntryPointQueryResult q;
    void *p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(p);
}

// Id of the calling thread's current context; false when there is none yet
// (or the driver calls are unavailable).
bool current_ctx_id(unsigned long long *id) {
    if (!g_ctx_get_current || !g_ctx_get_id) return false;
    CUcontext ctx = nullptr;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return g_ctx_get_id(ctx, id) == CUDA_SUCCESS;
}

// The device address of g_noalloc_scratch on the current device.  In host
// code the array's name is only a host-side handle, so the address is
// asked from the runtime (with the device current) and kept until the
// context changes.  Returns nullptr on failure.
void *scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    resolve_ctx_fns();
    unsigned long long id = 0;
    const bool have_id = current_ctx_id(&id);
    ScratchSlot &s = g_scratch[dev];
    if (have_id && s.addr && s.ctx_id == id) return s.addr;
    void *p = nullptr;
    // also makes the device's primary context current if it was not yet
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    if (have_id || current_ctx_id(&id)) {
        s.ctx_id = id;
        s.addr = p;
    } else {
        s.addr = nullptr;  // no context id to key on: look the address up again next call
    }
    return p;
}

}  // namespace

extern "C" idx_status idx_decode_topk_noalloc(const void *q, const void *kcache, const int *kv_len,
                                              const float *w, int B, int G, int n_max, int H, int d,
                                              int topk, idx_dtype dtype, int *out_idx, float *out_score,
                                              idx_stream_t stream) {
    const size_t need = idx_decode_workspace_size(B, G, n_max, H, d, topk, 0, IDX_MODE_DENSE, dtype);
    if (need == 0) {
        // arguments idx_decode_topk rejects before it looks at a workspace:
        // let it return its own code (nothing is launched)
        return idx_decode_topk(q, kcache, kv_len, w, B, G, n_max, H, d, topk, 0, IDX_MODE_DENSE, dtype, out_idx,
                               out_score, nullptr, 0, stream);
    }
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

extern "C" idx_status idx_decode_noalloc_status(idx_stream_t stream) {
    void *ws = scratch_address();
    if (!ws) return IDX_ERR_CUDA;
    return idx_device_status(ws, stream);
}
