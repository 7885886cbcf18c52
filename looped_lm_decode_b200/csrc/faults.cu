// Device-side fault reporting: a word per GPU that kernels set when they cannot do their job (a bounded
// wait of the tensor-core encoder ran out, or a window roll found the coded cache full), and the entry
// points that bound those waits and read the word back.  Calls stay asynchronous; only
// loopvq_fault_check synchronises.
#include <atomic>
#include <cstdio>
#include <mutex>

#include "loopvq_internal.cuh"

namespace {

// Fault bits of this process, one word per GPU that loads the library (kFault* in loopvq_internal.cuh).
static __device__ unsigned int g_fault_word;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned int *g_fault_ptr[kMaxDevices] = {};
std::atomic<unsigned long long> g_wait_ns{2000000000ull};

}  // namespace

namespace loopvq {

cudaError_t fault_word_for_current_device(unsigned int **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_fault_ptr[dev] == nullptr) {
        void *p = nullptr;
        // in host code the symbol is a host-side stand-in; the kernels get the device address
        e = cudaGetSymbolAddress(&p, g_fault_word);
        if (e != cudaSuccess) return e;
        g_fault_ptr[dev] = static_cast<unsigned int *>(p);
    }
    *out = g_fault_ptr[dev];
    return cudaSuccess;
}

unsigned long long wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

}  // namespace loopvq

extern "C" {

void loopvq_set_wait_limit_ns(uint64_t ns) { g_wait_ns.store(ns, std::memory_order_relaxed); }

uint64_t loopvq_wait_limit_ns(void) { return g_wait_ns.load(std::memory_order_relaxed); }

loopvq_status loopvq_fault_check(void *stream) {
    unsigned int *word = nullptr;
    cudaError_t e = loopvq::fault_word_for_current_device(&word);
    unsigned int bits = 0;
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaMemcpy(&bits, word, sizeof(bits), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && bits != 0) e = cudaMemset(word, 0, sizeof(bits));
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof(msg), "loopvq_fault_check: %s", cudaGetErrorString(e));
        loopvq::set_last_error(msg);
        return LOOPVQ_ERR_CUDA;
    }
    if (bits & loopvq::kFaultEncodeWait) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "a tensor-core encode gave up waiting for its own contraction (wait limit %llu ns); the codes that "
                 "encode call wrote are undefined%s",
                 (unsigned long long)loopvq::wait_limit_ns(),
                 (bits & loopvq::kFaultWindowFull) ? "; also a window roll found the coded cache full" : "");
        loopvq::set_last_error(msg);
        return LOOPVQ_ERR_TIMEOUT;
    }
    if (bits & loopvq::kFaultWindowFull) {
        loopvq::set_last_error(
            "a window advance found a sequence's coded cache full (coded_end + 8 > Nmax): that sequence did not roll, "
            "and its newest window slot was overwritten by the next append");
        return LOOPVQ_ERR_OVERFLOW;
    }
    return LOOPVQ_OK;
}

}  // extern "C"
