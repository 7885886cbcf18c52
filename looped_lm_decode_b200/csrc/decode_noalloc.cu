// loopvq_decode_attn_noalloc: decode attention whose split scratch lives in a fixed
// device array compiled into the library, for callers that cannot allocate device
// memory.  It runs the same kernels as loopvq_decode_attn; only where the scratch
// comes from differs.
#include <cstdio>
#include <mutex>

#include "loopvq_internal.cuh"

namespace {

// Split-partial scratch shared by every call in this process, one copy per GPU that loads the library.
static __device__ __align__(256) unsigned char g_decode_scratch[LOOPVQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};


// Device address of the scratch array on the current device; looked up once per device.
// (In host code the symbol names a host-side stand-in, not device memory.)
cudaError_t scratch_for_current_device(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

size_t loopvq_noalloc_scratch_bytes(void) { return (size_t)LOOPVQ_NOALLOC_SCRATCH_BYTES; }

loopvq_status loopvq_decode_attn_noalloc(const loopvq_cache *cache, int layer, int t, const uint16_t *q,
                                         const int32_t *lens, int max_len, float scale, float *out, float *lse,
                                         void *stream) {
    // 0 for an invalid shape or max_len: loopvq_decode_attn below then rejects the call with the precise message
    const size_t need = loopvq_decode_workspace_bytes(cache, max_len);
    if (need > (size_t)LOOPVQ_NOALLOC_SCRATCH_BYTES) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "loopvq_decode_attn_noalloc: this call needs %zu bytes of scratch, the built-in array holds %zu "
                 "(use loopvq_decode_attn with a caller workspace)", need, (size_t)LOOPVQ_NOALLOC_SCRATCH_BYTES);
        loopvq::set_last_error(msg);
        return LOOPVQ_ERR_WORKSPACE;
    }
    void *ws = nullptr;
    cudaError_t e = scratch_for_current_device(&ws);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof(msg), "loopvq_decode_attn_noalloc: scratch address lookup failed: %s",
                 cudaGetErrorString(e));
        loopvq::set_last_error(msg);
        return LOOPVQ_ERR_CUDA;
    }
    return loopvq_decode_attn(cache, layer, t, q, lens, max_len, scale, out, lse, ws,
                              (size_t)LOOPVQ_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
