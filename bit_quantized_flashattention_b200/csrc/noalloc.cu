// Attention entry point for callers that cannot allocate device memory.
//
// hifa4_attention_fwd needs a small device workspace (a status word) that the
// caller allocates. Some callers cannot call cudaMalloc at all: a plugin
// running inside a host runtime that owns every byte of device memory and
// hands out no allocator, or a latency-critical path where cudaMalloc's
// implicit device-wide synchronisation is not acceptable.
// hifa4_attention_fwd_noalloc serves them: its scratch is a fixed-size array
// in the library's own device image, so the call allocates nothing (no
// cudaMalloc, cudaFree or allocating library routine).
//
// The array lives in every GPU that loads the library until the process
// exits. Its device address is looked up with cudaGetSymbolAddress on the
// first call on a device, and again whenever that device's context has been
// re-created since (cudaDeviceReset reloads the module, so an address taken in
// the old context is stale). The host-side name of the array is only a
// stand-in and is never handed to a kernel.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "../../include/hifa4.h"
#include "api_internal.h"

// Upper bound of the scratch one call may use (hifa4_workspace_bytes of the
// problem). Calls that would need more are rejected.
static constexpr size_t kNoAllocScratchBytes = 4096;

// Shared by every call on a device; keeps the last call's contents.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;

struct ScratchSlot {
    void* addr = nullptr;
    unsigned long long ctx_id = 0;   // context the address belongs to (0: unknown)
};

std::mutex g_setup_mutex;
ScratchSlot g_slots[kMaxDevices];

// Unique id of the calling thread's current context (never reused within the
// process), or 0 when it cannot be determined.
unsigned long long current_context_id() {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
        looked_up = true;
    }
    if (get_current == nullptr || get_id == nullptr) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the scratch array on the current device, set up on the
// first call per device and again after its context was re-created.
hifa4_status scratch_on_current_device(void** addr) {
    int dev = -1;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return hifa4::from_cuda(e);
    if (dev < 0 || dev >= kMaxDevices) return HIFA4_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    ScratchSlot& slot = g_slots[dev];
    const unsigned long long id = current_context_id();
    if (slot.addr == nullptr || id == 0 || slot.ctx_id != id) {
        void* p = nullptr;
        const cudaError_t e2 = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e2 != cudaSuccess) return hifa4::from_cuda(e2);
        if (p == nullptr) return hifa4::from_cuda(cudaErrorInvalidSymbol);
        slot.addr = p;
        slot.ctx_id = current_context_id();   // the lookup may have created the context
    }
    *addr = slot.addr;
    return HIFA4_OK;
}

}  // namespace

extern "C" hifa4_status hifa4_attention_fwd_noalloc(const hifa4_packed* in, int B, int Hq, int Hkv, int Nq, int Nkv,
                                                    int D, float sm_scale, unsigned flags, hifa4_norm_mode norm,
                                                    void* o, hifa4_dtype o_dtype, float* lse,
                                                    hifa4_stream_t stream) {
    // every host-side check first: a rejected call leaves nothing on the stream
    const hifa4_status chk =
        hifa4::check_attention_args(in, B, Hq, Hkv, Nq, Nkv, D, sm_scale, flags, norm, o, o_dtype, lse);
    if (chk != HIFA4_OK) return chk;
    const size_t need = hifa4_workspace_bytes(B, Hq, Hkv, Nq, Nkv, D);
    if (need == 0 || need > kNoAllocScratchBytes) return HIFA4_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    const hifa4_status st = scratch_on_current_device(&scratch);
    if (st != HIFA4_OK) return st;
    // the status word must start at zero
    const cudaError_t e = cudaMemsetAsync(scratch, 0, need, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return hifa4::from_cuda(e);
    return hifa4_attention_fwd(in, B, Hq, Hkv, Nq, Nkv, D, sm_scale, flags, norm, o, o_dtype, lse, scratch, stream);
}
