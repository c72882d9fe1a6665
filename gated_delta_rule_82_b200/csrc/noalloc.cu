// noalloc.cu -- ckda_fwd_chunked_noalloc: the chunked forward with library-owned scratch.
//
// Some callers cannot call cudaMalloc at the point where they run the forward: code running
// while a stream is being captured into a CUDA graph, runtimes that hand out device memory only
// from a pool sized at start-up, or real-time paths where any allocation (and the device-wide
// synchronisation cudaFree can imply) is forbidden.  For them this entry point takes the same
// inputs and outputs as ckda_fwd_chunked but keeps its scratch in a fixed, file-scope device
// array, so it allocates nothing.
//
// The array is CKDA_NOALLOC_MAX_WORKSPACE bytes; every GPU that loads the library holds it until
// the process exits.  Host code cannot use the array's name as a device address, so the first call
// on each device looks the address up with cudaGetSymbolAddress (with that device current) and
// caches it.  Every call shares the array: calls whose kernels overlap on the GPU (different
// streams, or host threads racing) corrupt each other's scratch.  No byte of the scratch has to
// start at zero: every call clears the chunk-heads' ready flags itself, and the chunk-factor work
// writes every other byte the state pass later reads.  That holds for the whole forward (stages 0
// and 3); the profiling stages 1 and 2, which split it across calls, are refused.
#include <mutex>

#include "internal.cuh"

namespace {

constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[CKDA_NOALLOC_MAX_WORKSPACE];

void* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_lock;

// Device address of the scratch array on the current device, or nullptr on failure.
void* scratch_address(int device) {
    std::lock_guard<std::mutex> guard(g_scratch_lock);
    if (!g_scratch_addr[device]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_scratch_addr[device] = p;
    }
    return g_scratch_addr[device];
}

}  // namespace

extern "C" CKDA_API ckda_status ckda_fwd_chunked_noalloc(
    const void* q, const void* k, const void* v, const void* alpha, const float* beta,
    const float* h0, void* out, float* hT, int B, int T, int H, int dk, int dv, int chunk,
    ckda_flags flags, ckda_dtype dtype, long long pos_offset, ckda_stream_t stream) {
    // the profiling stages 1 and 2 would leave or read images of the shared array across calls
    if (flags.stages != 0 && flags.stages != 3) return CKDA_ERR_ARG;
    const size_t need = ckda_fwd_workspace_bytes(B, T, H, dk, dv, chunk, dtype, flags.path);
    if (need != (size_t)-1 && need > (size_t)CKDA_NOALLOC_MAX_WORKSPACE) return CKDA_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need != (size_t)-1 && need > 0) {
        int device = 0;
        if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxDevices)
            return CKDA_ERR_CUDA;
        scratch = scratch_address(device);
        if (!scratch) return CKDA_ERR_CUDA;
    }
    return ckda_fwd_chunked(q, k, v, alpha, beta, h0, out, hT, B, T, H, dk, dv, chunk, flags, dtype,
                            pos_offset, scratch, scratch ? (size_t)CKDA_NOALLOC_MAX_WORKSPACE : 0,
                            stream);
}
