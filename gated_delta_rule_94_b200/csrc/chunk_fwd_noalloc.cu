// chunk_fwd_noalloc.cu -- gdn_chunk_fwd for callers that cannot allocate
// device memory.
//
// Some callers cannot call cudaMalloc at all: code running inside another
// runtime's memory pool or a framework that forbids allocations on its hot
// path, or a process that has handed its whole device memory to a caching
// allocator it does not control.  gdn_chunk_fwd wants a caller-provided
// workspace; this entry point supplies it from a fixed scratch array that the
// library holds in device memory, so the caller passes only inputs and
// outputs.
//
// The scratch is a file-scope __device__ array: every GPU that loads the
// library holds its kNoAllocScratchBytes until the process exits.  The CUDA
// runtime loads this file's module -- and so reserves the array -- the first
// time the array is used on a device (lazy module loading, the default since
// CUDA 12.2; with CUDA_MODULE_LOADING=EAGER it happens when the context is
// created).  A call that has no work (B = 0 or H = 0) performs only that
// set-up: a caller makes it once per device at start-up, before its own
// framework takes the device memory and before any stream capture, so that no
// later call reserves anything.
//
// The array is shared by every call on a device and keeps the last call's
// contents; the forward writes every workspace byte it reads before reading
// it, so nothing needs clearing between calls.  Calls whose work overlaps on
// the GPU (different streams, or concurrent host threads without ordering)
// race on the array.
#include <mutex>

#include "common.cuh"
#include "gdn.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(128) << 20;   // 128 MiB

static __device__ __align__(256) unsigned char gdn_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device, looked up once
// per device with that device current.  Host code must not use the array's
// name as a device pointer: on the host it names a stand-in, not device memory.
// A failed lookup (for instance out of memory while the module loads) clears
// the runtime's last-error state, so that no later, unrelated call reports it.
void* scratch_address() {
    static std::mutex mu;
    static void* cache[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        (void)cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, gdn_noalloc_scratch) != cudaSuccess) {
            (void)cudaGetLastError();
            return nullptr;
        }
        cache[dev] = ptr;
    }
    return cache[dev];
}

}  // namespace

extern "C" {

size_t gdn_chunk_fwd_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

gdn_status gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const void* beta,
                                 const void* g, gdn_gate gate_kind, const float* initial_state,
                                 void* o, float* final_state, int B, int T, int H, int Dk, int Dv,
                                 int chunk, gdn_dtype dtype, gdn_stream_t stream) {
    const size_t need = gdn_chunk_fwd_workspace_min_bytes(B, T, H, Dk, Dv, chunk, dtype, gate_kind);
    if ((B == 0 || H == 0) && need != (size_t)-1) {
        // No work: only the set-up of the current device (module load and the
        // array's address), so that later calls reserve nothing.
        return scratch_address() ? GDN_OK : GDN_ERR_CUDA;
    }
    if (need == (size_t)-1 || need > kNoAllocScratchBytes) {
        // Let the regular entry point report the argument error, or
        // GDN_ERR_WORKSPACE when the shape needs more than the scratch holds;
        // with no workspace it returns before anything is enqueued.
        return gdn_chunk_fwd(q, k, v, beta, g, gate_kind, initial_state, o, final_state, B, T,
                             H, Dk, Dv, chunk, dtype, nullptr, 0, stream);
    }
    void* scratch = nullptr;
    if (need > 0) {
        scratch = scratch_address();
        if (!scratch) return GDN_ERR_CUDA;
    }
    return gdn_chunk_fwd(q, k, v, beta, g, gate_kind, initial_state, o, final_state, B, T, H,
                         Dk, Dv, chunk, dtype, scratch, need > 0 ? kNoAllocScratchBytes : 0,
                         stream);
}

}  // extern "C"
