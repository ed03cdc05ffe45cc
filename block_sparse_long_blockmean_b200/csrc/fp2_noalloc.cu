// fp2_noalloc.cu -- fp2_prefill_noalloc: the whole prefill path with its
// scratch (block means, scores, masks, error word) in a fixed device array
// owned by the library, for callers that cannot allocate device memory.
//
// Some hosts hand a kernel only its inputs and outputs and have no device
// allocator to offer it (plugin-style integrations), and some serving
// runtimes reserve all device memory up front, so that a cudaMalloc on the
// request path would fail or stall the device.  Such callers cannot provide
// the workspace fp2_prefill needs; this entry point takes the same inputs and
// output and uses FP2_NOALLOC_SCRATCH_BYTES of library-owned device memory
// instead.  It allocates nothing and calls no allocating routine.
#include <mutex>

#include "fp2.h"

namespace fp2 {
// fp2_prefill's argument checks, without queuing anything (fp2_api.cu)
fp2_status validate_prefill(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* page_table, const int32_t* cu_seqlens, float tau,
                            int block, fp2_dtype dtype, const void* out,
                            const fp2_params* params);
}  // namespace fp2

namespace {

// The scratch.  Every GPU that loads the library holds this much device
// memory until the process exits.  Calls share it: the contents left by one
// call are there for the next, and two calls whose work overlaps on the GPU
// (different streams, or different host threads) race on it.
static __device__ __align__(256) unsigned char g_scratch[FP2_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_mutex;

// Device address of g_scratch on the current device.  In host code the name
// g_scratch is a host-side stand-in, not a device address; the address comes
// from cudaGetSymbolAddress, taken once per device with that device current.
fp2_status scratch_on_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FP2_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FP2_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return FP2_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return FP2_OK;
}

}  // namespace

extern "C" fp2_status fp2_prefill_noalloc(const void* q, const void* k_cache,
                                          const void* v_cache, const int32_t* page_table,
                                          const int32_t* cu_seqlens, float tau, int block,
                                          fp2_dtype dtype, void* out, const fp2_params* params) {
    if (!params) return FP2_ERR_INVALID_ARG;
    const size_t need = fp2_workspace_size(params, block);
    if (need == 0) return FP2_ERR_INVALID_ARG;
    if (need > (size_t)FP2_NOALLOC_SCRATCH_BYTES) return FP2_ERR_WORKSPACE;
    // every argument check first, against the array's size (the checks never
    // dereference the workspace): a call that is going to be rejected must
    // not touch the shared array, which another call may still be using
    fp2_params p = *params;
    p.workspace = reinterpret_cast<void*>(static_cast<uintptr_t>(256));
    p.workspace_bytes = FP2_NOALLOC_SCRATCH_BYTES;
    fp2_status st = fp2::validate_prefill(q, k_cache, v_cache, page_table, cu_seqlens, tau,
                                          block, dtype, out, &p);
    if (st != FP2_OK) return st;
    void* scratch = nullptr;
    if ((st = scratch_on_current_device(&scratch)) != FP2_OK) return st;
    p.workspace = scratch;
    // the error word must start at zero; the rest is fully written before it is read
    st = fp2_workspace_init(&p);
    if (st != FP2_OK) return st;
    return fp2_prefill(q, k_cache, v_cache, page_table, cu_seqlens, tau, block, dtype, out, &p);
}

extern "C" fp2_status fp2_noalloc_get_status(void* stream, uint32_t* detail) {
    void* scratch = nullptr;
    fp2_status st = scratch_on_current_device(&scratch);
    if (st != FP2_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t w[2] = {0, 0};
    if (cudaStreamSynchronize(s) != cudaSuccess) return FP2_ERR_CUDA;
    if (cudaMemcpy(w, scratch, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess)
        return FP2_ERR_CUDA;
    if (w[0] != 0) {
        if (cudaMemsetAsync(scratch, 0, sizeof(w), s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return FP2_ERR_CUDA;
    }
    if (detail) *detail = w[1];
    return static_cast<fp2_status>(w[0]);
}
