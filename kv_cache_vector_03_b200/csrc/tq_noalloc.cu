// tq_logits_noalloc: tq_logits for callers that cannot allocate device memory.
//
// Some callers are not allowed to call cudaMalloc or any allocating routine: code that
// runs inside a host framework whose memory pool owns all of the device memory, plugins
// that may only use the buffers they are handed, and latency-critical loops under a
// no-allocation policy. This entry point takes the same inputs and outputs as tq_logits
// but no workspace: its scratch (status word, query fragments, per-head constants) lives
// in a fixed array in device memory that every GPU loading the library keeps until exit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "tq.h"

// tq_logits_est behind its argument checks (tq_api.cu); clear_status clears the status word
// on the stream once every check has passed
int tq_logits_run(const tq_codec* c, const void* packed, int64_t n_seq, int n_kv, int64_t n_tok, const void* q,
                  tq_dtype q_dtype, int g, const void* tail, int n_tail, float scale, float* out, void* ws,
                  size_t ws_bytes, int estimator, int clear_status, void* stream);

namespace {

constexpr size_t kScratchBytes = TQ_NOALLOC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Host code must not pass g_scratch to a kernel: on the host it names a shadow, not a
// device address. The address belongs to the module as loaded in one CUDA context, so it is
// resolved (cudaGetSymbolAddress, with that context current) on the first call in a context
// and again whenever the current context of a device changes, e.g. after cudaDeviceReset
// reloaded the module. Contexts are told apart by the driver's unique context ID.
constexpr int kMaxDevices = 64;
struct Slot {
    unsigned long long ctx_id;   // 0: not resolved
    void* ptr;
};
Slot g_slot[kMaxDevices];
std::mutex g_lock;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_get_current = nullptr;
CtxGetIdFn g_get_id = nullptr;

// driver entry points through the runtime (the library does not link libcuda itself)
bool resolve_driver_calls() {
    if (g_get_current && g_get_id) return true;
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &a, 12000, cudaEnableDefault, &qa) != cudaSuccess ||
        qa != cudaDriverEntryPointSuccess || !a)
        return false;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &b, 12000, cudaEnableDefault, &qb) != cudaSuccess ||
        qb != cudaDriverEntryPointSuccess || !b)
        return false;
    g_get_current = reinterpret_cast<CtxGetCurrentFn>(a);
    g_get_id = reinterpret_cast<CtxGetIdFn>(b);
    return true;
}

// ID of the context the runtime uses for `dev` on this thread (made current if need be)
bool current_context_id(int dev, unsigned long long* id) {
    CUcontext ctx = nullptr;
    if (g_get_current(&ctx) != CUDA_SUCCESS) return false;
    if (!ctx) {
        // the runtime makes its context current lazily; cudaSetDevice initialises it
        if (cudaSetDevice(dev) != cudaSuccess || g_get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    }
    return g_get_id(ctx, id) == CUDA_SUCCESS && *id != 0;
}

int scratch_of_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TQ_ERR_CUDA;
    std::lock_guard<std::mutex> guard(g_lock);
    unsigned long long id = 0;
    if (!resolve_driver_calls() || !current_context_id(dev, &id)) return TQ_ERR_CUDA;
    Slot& s = g_slot[dev];
    if (s.ctx_id != id || !s.ptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) {
            s.ctx_id = 0;
            s.ptr = nullptr;
            return TQ_ERR_CUDA;
        }
        s.ctx_id = id;
        s.ptr = p;
    }
    *out = s.ptr;
    return TQ_OK;
}

}  // namespace

extern "C" int tq_logits_noalloc(const tq_codec* codec, const void* packed, int64_t n_seq, int n_kv, int64_t n_tok,
                                 const void* q, tq_dtype q_dtype, int g, const void* tail, int n_tail, float scale,
                                 float* out, void* stream) {
    const size_t need = tq_workspace_bytes(codec, TQ_OP_LOGITS, n_seq, n_kv, g);
    if (need == 0) return TQ_ERR_ARG;
    if (need > kScratchBytes) return TQ_ERR_WORKSPACE;
    void* ws = nullptr;
    const int st = scratch_of_current_device(&ws);
    if (st != TQ_OK) return st;
    // every argument is checked before the status word is cleared and the kernels are
    // enqueued: a rejected call leaves the stream and the shared array untouched
    return tq_logits_run(codec, packed, n_seq, n_kv, n_tok, q, q_dtype, g, tail, n_tail, scale, out, ws,
                         kScratchBytes, TQ_EST_QJL, 1, stream);
}
