// tam_mass_select_noalloc: pass 2 for callers that cannot allocate device memory.
//
// Some callers have no way to provide a workspace: a plugin inside a serving
// engine whose memory planner owns every device allocation and hands the plugin
// only its input and output tensors, or a process that must not call cudaMalloc
// once it is running (cudaMalloc can synchronise the device and can fail under
// fragmentation in the middle of serving).  This entry point serves them with a
// fixed scratch area that lives in the library itself: a file-scope static
// __device__ array of kStaticScratchBytes.  The caller still passes every input
// and output buffer; nothing here calls cudaMalloc, cudaFree or any allocating
// library routine.
//
// The array is ordinary module memory: it is reserved on a device whenever the
// library's module is loaded there (at the first launch of any of its kernels
// under lazy loading, at context creation under eager loading), whether or not
// this entry point is ever called, and the device keeps it until the process
// exits.  In host code its name is only a host-side stand-in, so every call looks
// up its device address with cudaGetSymbolAddress, with the caller's device
// current, and that address is what the kernels receive.  Nothing is cached: a
// torn-down and re-created context (cudaDeviceReset) may load the module at
// another address, and a cached pointer would then point at unmapped memory.
#include <cuda_runtime.h>

#include "../../include/tam.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;   // 64 MiB per device
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of the static scratch on the current device, or null if the
// lookup fails.  The lookup is a host-side query (no stream work).
void* scratch_for_current_device() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
    return p;
}

}  // namespace

extern "C" int tam_mass_select_noalloc(int64_t N, int Hq, int Hkv, int d, int dtype,
                                       const void* q, const void* k, const float* lse,
                                       int budget_k, int block_q, int32_t* sup_idx,
                                       int32_t* sup_len, float* sup_mass, void* stream) {
    const size_t need = tam_mass_workspace_min(N, Hq, Hkv, d, dtype, budget_k, block_q);
    if (need == 0) {
        // let the regular entry point name the argument error (it returns before any launch)
        return tam_mass_select(N, Hq, Hkv, d, dtype, q, k, lse, budget_k, block_q, sup_idx,
                               sup_len, sup_mass, nullptr, 0, stream);
    }
    if (need > kStaticScratchBytes) return TAM_ERR_WORKSPACE;
    void* scratch = scratch_for_current_device();
    if (scratch == nullptr) return TAM_ERR_CUDA;
    // The regular entry point clears the status block at the start of the scratch,
    // and every other byte it uses is written before it is read.
    const int rc = tam_mass_select(N, Hq, Hkv, d, dtype, q, k, lse, budget_k, block_q, sup_idx,
                                   sup_len, sup_mass, scratch, kStaticScratchBytes, stream);
    if (rc != TAM_OK) return rc;
    return tam_check_status(scratch, stream, nullptr);
}
