// kda_noalloc.cu -- kda_chunk_fwd_noalloc: the chunkwise prefill for callers
// that cannot allocate device memory themselves.
//
// Some hosts give a plugin its input and output buffers but no way to obtain
// device scratch: the host owns every allocation (a memory pool that already
// holds all free memory, a runtime that forbids cudaMalloc on its hot path
// because cudaMalloc can synchronise the device, or an embedding that only
// exposes tensors it created).  This entry point serves them: its scratch is a
// fixed-size array in the library's own device memory, so the call needs no
// workspace argument and allocates nothing.
//
// The array lives in this file's module; the driver reserves it on a device
// when that module is loaded there and keeps it until the process exits.  In
// host code the symbol is only a stand-in, never a device address: its device
// address is looked up once per device with cudaGetSymbolAddress (with that
// device current) and that address is what the kernels receive.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/kda.h"

namespace {

static __device__ __align__(256) uint8_t g_kda_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
// Device address of the array per device.  Host threads may call concurrently:
// each entry is an atomic, and two threads that look up the same device at once
// both store the same address.  A cudaDeviceReset unloads the module, so a cached
// address is stale afterwards (documented in kda.h).
std::atomic<void*> g_scratch_dev_ptr[kMaxDevices];

// Device address of the scratch array on the current device (looked up once
// per device, with that device current).  Returns nullptr on failure.
void* scratch_on_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    void* p = g_scratch_dev_ptr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
        if (cudaGetSymbolAddress(&p, g_kda_noalloc_scratch) != cudaSuccess) return nullptr;
        g_scratch_dev_ptr[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace

extern "C" kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const void* log_alpha,
                                            const void* beta, const float* init_state, void* o, float* final_state,
                                            int B, int64_t T, int H, int dk, int dv, const int32_t* cu_seqlens,
                                            int n_seqs, int64_t max_seqlen, kda_dtype in_dtype,
                                            kda_dtype out_dtype, float scale, const void* gate,
                                            const float* norm_weight, float eps, void* stream) {
    // size check first, so an oversized problem is rejected before any CUDA call
    const int n = cu_seqlens ? n_seqs : B;
    const int64_t maxlen = cu_seqlens ? max_seqlen : T;
    size_t need = 0;
    const kda_status st = kda_chunk_fwd_workspace_size(cu_seqlens ? T : (int64_t)B * T, H, dk, dv, n, maxlen,
                                                       &need, nullptr);
    if (st != KDA_OK) return st;
    if (need > (size_t)KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_WORKSPACE;
    void* scratch = scratch_on_current_device();
    if (scratch == nullptr) return KDA_ERR_CUDA;
    return kda_chunk_fwd(q, k, v, log_alpha, beta, init_state, o, final_state, B, T, H, dk, dv, cu_seqlens, n_seqs,
                         max_seqlen, in_dtype, out_dtype, scale, gate, norm_weight, eps, scratch,
                         (size_t)KDA_NOALLOC_SCRATCH_BYTES, stream);
}

// The device status word of the last kda_chunk_fwd_noalloc call on the current
// device sits at the start of the static array (the layout every prefill
// workspace has); kda_query_status reads and clears it.
extern "C" kda_status kda_chunk_fwd_noalloc_query_status(void* stream) {
    void* scratch = scratch_on_current_device();
    if (scratch == nullptr) return KDA_ERR_CUDA;
    return kda_query_status(scratch, stream);
}
