// Host helpers: TMA tensor-map encoding (through the runtime's driver entry point,
// so the library needs no link-time libcuda) and the wait deadline / debug switches.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tam {

// Encodes a 3-D bf16 tensor map with a 128-byte swizzle.  Dimensions innermost
// first; strides in bytes for dims 1 and 2 (multiples of 16); box sizes in
// elements (box0 * 2 must be 128).  Returns false if the driver rejects it.
bool make_tmap_3d_bf16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0,
                       uint32_t box1, uint32_t box2);

// Deadline of every bounded device wait (ns).  2 s normally; with the debug
// variable TAM_DEBUG_FORCE_TIMEOUT=1 in the environment a short deadline is used
// and kernels that support it park one role on a barrier nobody arrives on, so the
// timeout path can be exercised without faulting anything.
uint64_t wait_timeout_ns();
int debug_flags();

constexpr int kDebugForceTimeout = 1;

// TAM_DISABLE_PAIR_KERNELS=1 routes pass 2 to the single-CTA kernel (A/B comparisons).
bool pair_path_disabled();
// TAM_DISABLE_BLOCK_TC=1 routes block-shared pass 3 to the mma.sync kernel (A/B comparisons).
bool block_tc_disabled();
// TAM_MATERIALISE_ROWS=1 routes the per-query selection (mass and indexer) through
// materialised score rows and the row top-k instead of the streamed candidates
// (A/B comparisons).
bool materialise_rows();
// TAM_DENSE_PAIR_TILES=1 runs dense attention on the block-shared pass-3 pipeline (two
// query tiles per CTA) instead of the single-tile kernel (A/B comparisons).
bool dense_pair_tiles_selected();
// TAM_DEBUG_FORCE_FALLBACK=1 (threshold above every key) or =2 (threshold below every
// key) sends every row the streamed selection would sample to the fallback path, so
// that path can be tested on ordinary inputs.
int debug_force_fallback();
// Extent handed to a launch for its debug-checks: `cap`, or at most 64 entries when
// TAM_DEBUG_SHRINK_EXTENTS is set (so that the checks of the debug-checks build fire
// while every store still lands inside the real buffer, which they then skip).
uint64_t debug_extent(uint64_t cap);

}  // namespace tam
