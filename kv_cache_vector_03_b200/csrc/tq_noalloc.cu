// tq_logits_noalloc: tq_logits for callers that cannot allocate device memory.
//
// Some callers are not allowed to call cudaMalloc or any allocating routine: code that
// runs inside a host framework whose memory pool owns all of the device memory, plugins
// that may only use the buffers they are handed, and latency-critical loops under a
// no-allocation policy. This entry point takes the same inputs and outputs as tq_logits
// but no workspace: its scratch (status word, query fragments, per-head constants) lives
// in a fixed array in device memory that every GPU loading the library keeps until exit.
#include <cuda_runtime.h>

#include <mutex>

#include "tq.h"

namespace {

constexpr size_t kScratchBytes = TQ_NOALLOC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Host code must not pass g_scratch to a kernel: on the host it names a shadow, not a
// device address. The address is resolved once per device, with that device current.
constexpr int kMaxDevices = 64;
void* g_ptr[kMaxDevices];
std::mutex g_lock;

int scratch_of_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TQ_ERR_CUDA;
    std::lock_guard<std::mutex> guard(g_lock);
    if (!g_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return TQ_ERR_CUDA;
        g_ptr[dev] = p;
    }
    *out = g_ptr[dev];
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
    // the status word starts at zero for every call; the rest is written before it is read
    if (cudaMemsetAsync(ws, 0, 4, static_cast<cudaStream_t>(stream)) != cudaSuccess) return TQ_ERR_CUDA;
    return tq_logits(codec, packed, n_seq, n_kv, n_tok, q, q_dtype, g, tail, n_tail, scale, out, ws, kScratchBytes,
                     stream);
}
