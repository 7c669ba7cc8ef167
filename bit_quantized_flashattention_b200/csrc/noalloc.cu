// Attention entry point for callers that cannot allocate device memory.
//
// hifa4_attention_fwd needs a small device workspace (a status word and a
// work counter) that the caller allocates. Some callers cannot call
// cudaMalloc at all: a plugin running inside a host runtime that owns every
// byte of device memory and hands out no allocator, or a latency-critical
// path where cudaMalloc's implicit device-wide synchronisation is not
// acceptable. hifa4_attention_fwd_noalloc serves them: its scratch is a
// fixed-size array in the library's own device image, so the call allocates
// nothing (no cudaMalloc, cudaFree or allocating library routine).
//
// The array lives in every GPU that loads the library until the process
// exits. Its device address is looked up once per device with
// cudaGetSymbolAddress; the host-side name of the array is only a stand-in
// and must never be handed to a kernel directly.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/hifa4.h"

// Upper bound of the scratch one call may use (hifa4_workspace_bytes of the
// problem). Calls that would need more are rejected.
static constexpr size_t kNoAllocScratchBytes = 4096;

// Shared by every call on a device; keeps the last call's contents.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on the
// first call per device).
hifa4_status scratch_on_current_device(void** addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HIFA4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) return HIFA4_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return HIFA4_OK;
}

}  // namespace

extern "C" hifa4_status hifa4_attention_fwd_noalloc(const hifa4_packed* in, int B, int Hq, int Hkv, int Nq, int Nkv,
                                                    int D, float sm_scale, unsigned flags, hifa4_norm_mode norm,
                                                    void* o, hifa4_dtype o_dtype, float* lse,
                                                    hifa4_stream_t stream) {
    const size_t need = hifa4_workspace_bytes(B, Hq, Hkv, Nq, Nkv, D);
    if (need == 0 || need > kNoAllocScratchBytes) return HIFA4_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    const hifa4_status st = scratch_on_current_device(&scratch);
    if (st != HIFA4_OK) return st;
    // the status word and the work counter must start at zero
    if (cudaMemsetAsync(scratch, 0, need, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return HIFA4_ERR_CUDA;
    return hifa4_attention_fwd(in, B, Hq, Hkv, Nq, Nkv, D, sm_scale, flags, norm, o, o_dtype, lse, scratch, stream);
}
