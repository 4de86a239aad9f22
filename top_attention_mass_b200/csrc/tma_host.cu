// Host helpers: TMA tensor maps, wait deadline, debug switches.
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "tma_host.h"

namespace tam {

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

int env_int(const char* name, int dflt) {
    const char* s = std::getenv(name);
    if (!s || !*s) return dflt;
    return std::atoi(s);
}

}  // namespace

bool make_tmap_3d_bf16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0,
                       uint32_t box1, uint32_t box2) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    std::memset(map, 0, sizeof(*map));
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    cuuint32_t box[3] = {box0, box1, box2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

uint64_t wait_timeout_ns() {
    return (debug_flags() & kDebugForceTimeout) ? 20000000ull : 2000000000ull;
}

bool pair_path_disabled() { return env_int("TAM_DISABLE_PAIR_KERNELS", 0) != 0; }

bool block_tc_disabled() { return env_int("TAM_DISABLE_BLOCK_TC", 0) != 0; }

bool materialise_rows() { return env_int("TAM_MATERIALISE_ROWS", 0) != 0; }

bool dense_pair_tiles_selected() { return env_int("TAM_DENSE_PAIR_TILES", 0) != 0; }

int debug_force_fallback() {
    const int v = env_int("TAM_DEBUG_FORCE_FALLBACK", 0);
    return (v == 1 || v == 2) ? v : 0;
}

uint64_t debug_extent(uint64_t cap) {
    return env_int("TAM_DEBUG_SHRINK_EXTENTS", 0) ? (cap < 64 ? cap : 64) : cap;
}

int debug_flags() { return env_int("TAM_DEBUG_FORCE_TIMEOUT", 0) ? kDebugForceTimeout : 0; }

}  // namespace tam
