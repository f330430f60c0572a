// moe_trellis_gemv for callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc (or any allocator) when they run
// the layer: a serving runtime whose device memory is one pool carved up at start-up,
// an engine that runs inside a sandbox or plugin host which hands it only the tensors
// of the call, or a latency-critical path where an allocation (and the device
// synchronisation it can imply) is not allowed.  moe_trellis_gemv needs a workspace
// for the SwiGLU activations h and their rotation h'; this entry point takes that
// workspace from a fixed array compiled into the library instead.
#include "tq_common.cuh"

#include <atomic>

namespace tq {

// Scratch for the GEMV's workspace (gate/up partial sums, fixed-point h' and x'): at most
// 4 MiB (T <= 25 tokens at k = 8, D = 4096, F = 1024).  Every GPU that loads the library
// holds this array until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
static std::atomic<void *> g_noalloc_ptr[kNoAllocMaxDevices];

// Device address of the scratch array on the current device (in host code the array's
// name is only a host-side stand-in, never a device address).  Looked up once per
// device, by the first call with that device current, and kept for the life of the
// process's context on that device: after cudaDeviceReset the library must be
// reloaded before this entry point is called again.  Threads that race on the first
// lookup all store the same address.
static int noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return record_cuda_error("cudaGetDevice");
    if (dev < 0 || dev >= kNoAllocMaxDevices) return TQ_ERR_UNSUPPORTED;
    void *p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
            return record_cuda_error("cudaGetSymbolAddress");
        g_noalloc_ptr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return TQ_OK;
}

int run_moe_gemv(const tq_moe_layer *L, const __half *x_rot, const int32_t *offsets, const int32_t *perm,
                 const int32_t *active_ids, const int32_t *n_active, int T, int k, float *y_perm,
                 void *ws, cudaStream_t s);

}  // namespace tq

int moe_validate_args(const tq_moe_layer *layer, const uint16_t *x_rot, const int32_t *offsets,
                      const int32_t *perm, const int32_t *active_ids, const int32_t *n_active, int T,
                      int k, float *y_perm);

TQ_API int moe_trellis_gemv_noalloc(const tq_moe_layer *layer, const uint16_t *x_rot,
                                    const int32_t *offsets, const int32_t *perm,
                                    const int32_t *active_ids, const int32_t *n_active, int T, int k,
                                    float *y_perm, tq_stream stream) {
    // the same argument statuses as moe_trellis_gemv, then the size of the call
    int st = moe_validate_args(layer, x_rot, offsets, perm, active_ids, n_active, T, k, y_perm);
    if (st || T == 0) return st;
    if (layer->codebook != TQ_CODEBOOK_T16) return TQ_ERR_UNSUPPORTED;   // as moe_trellis_gemv
    if (tq::workspace_bytes(layer, T, k) > tq::kNoAllocScratchBytes) return TQ_ERR_WORKSPACE;
    void *scratch = nullptr;
    st = tq::noalloc_scratch(&scratch);
    if (st) return st;
    return tq::run_moe_gemv(layer, reinterpret_cast<const __half *>(x_rot), offsets, perm, active_ids,
                            n_active, T, k, y_perm, scratch, (cudaStream_t)stream);
}
