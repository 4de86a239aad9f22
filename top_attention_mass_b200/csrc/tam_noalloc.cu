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
// The array is ordinary module memory: a GPU on which it has been used keeps it
// until the process exits.  In host code its name is only a host-side stand-in,
// so its device address is looked up once per device with cudaGetSymbolAddress
// (on the first call on that device, with that device current) and that address
// is what the kernels receive.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/tam.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;   // 64 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the static scratch on the current device; looked up once per
// device.  Returns null if the device index is out of range or the lookup fails.
void* scratch_for_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
            return nullptr;
        g_scratch_addr[dev] = p;
    }
    return g_scratch_addr[dev];
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
