// Shared device helpers: status block, dtype loads, block scans and the exact
// block-level top-k selection used by the CUDA-core kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tam.h"

namespace tam {

// ---------------------------------------------------------------- status block
// The first 256 bytes of every workspace.  word[0] = first error code (0 = none),
// word[1] = id of the kernel that set it, word[2..7] = kernel-specific detail.
constexpr size_t kStatusBytes = 256;

enum KernelId : int32_t {
    KID_LSE_SIMT = 1, KID_MASS_SIMT = 2, KID_ATTN_SIMT = 3, KID_INDEXER_SIMT = 4,
    KID_LSE_TC = 11, KID_MASS_TC = 12, KID_TOPK_FINAL = 13, KID_ATTN_GATHER = 14,
    KID_DENSE_TC = 15, KID_INDEXER_TC = 16, KID_BLOCK_MASS_TC = 17, KID_BLOCK_ATTN = 18,
};

__device__ __forceinline__ void report_error(int32_t* status, int32_t code, int32_t kid,
                                             int32_t a = 0, int32_t b = 0, int32_t c = 0) {
    if (status == nullptr) return;
    if (atomicCAS(status, 0, code) == 0) {
        status[1] = kid;
        status[2] = a;
        status[3] = b;
        status[4] = c;
        status[5] = blockIdx.x;
        status[6] = threadIdx.x;
    }
}

// ---------------------------------------------------------------- debug-checks build
// Built with -DTAM_DEBUG_CHECKS (libtam_debug.so), the pass-2 kernels check the index
// of every slab row, candidate and block-mass store against the extent the host gave
// the launch (MassArgs::out_cap) and, instead of an out-of-range store, record
// TAM_ERR_OVERFLOW (detail: the site, the index and the extent, truncated to 32 bits)
// and skip it.  The release build compiles the checks away.
#ifdef TAM_DEBUG_CHECKS
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
enum DebugSite : int32_t { kSiteRows = 1, kSiteCand = 2, kSiteBlockMass = 3 };

__device__ __forceinline__ bool in_bounds(int32_t* status, int32_t kid, int32_t site, uint64_t idx,
                                          uint64_t extent) {
    if constexpr (!kDebugChecks) return true;
    if (idx < extent) return true;
    report_error(status, TAM_ERR_OVERFLOW, kid, site, (int32_t)idx, (int32_t)extent);
    return false;
}

// ---------------------------------------------------------------- element loads
template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------- warp / block reductions
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Exclusive prefix sum of one int per thread over the whole block (blockDim.x a
// multiple of 32, at most 1024).  `warp_tot` is shared scratch of 33 ints.
// Returns the exclusive prefix; *total receives the block sum.  Contains barriers:
// every thread of the block must call it.
__device__ __forceinline__ int block_exclusive_scan(int x, int* warp_tot, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int t = (lane < nw) ? warp_tot[lane] : 0;
        int ti = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, ti, o);
            if (lane >= o) ti += y;
        }
        if (lane < nw) warp_tot[lane] = ti - t;   // exclusive warp offsets
        if (lane == nw - 1) warp_tot[32] = ti;
    }
    __syncthreads();
    int r = warp_tot[warp] + incl - x;
    *total = warp_tot[32];
    __syncthreads();
    return r;
}

// Order-preserving map float -> uint32 (a < b  <=>  key(a) < key(b); +0 above -0).
__device__ __forceinline__ uint32_t order_key(float v) {
    uint32_t b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct SelectSmem {
    int hist[256];
    int warp_tot[33];
    int digit;
    int rem;
};

// Exact top-min(k, n) of vals[0..n) (global or shared memory, visible to the whole
// block), ranked by value descending, ties by smaller index.  Writes the chosen
// indices ascending to out_idx[0..m) with their values, pads out_idx/out_val up to
// k with -1 / 0 and sets *out_len = m.  A 4 x 8-bit MSB-first radix select finds
// the k-th key T; the selection pass walks the row in index order, so the output
// comes out sorted.  All threads of the block must call it.
__device__ inline void block_select_topk(const float* vals, int n, int k, int32_t* out_idx,
                                  float* out_val, int32_t* out_len, SelectSmem& sm) {
    const int tid = threadIdx.x, nt = blockDim.x;
    const int m = min(k, n);
    const bool take_all = (n <= k);
    uint32_t T = 0;
    int take_eq = 0;
    if (!take_all) {
        uint32_t prefix = 0, mask = 0;
        int remaining = k;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int b = tid; b < 256; b += nt) sm.hist[b] = 0;
            __syncthreads();
            for (int j = tid; j < n; j += nt) {
                const uint32_t key = order_key(vals[j]);
                if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 255u], 1);
            }
            __syncthreads();
            if (tid == 0) {
                int cum = 0;
                for (int b = 255; b >= 0; --b) {
                    const int c = sm.hist[b];
                    if (cum + c >= remaining) {
                        sm.digit = b;
                        sm.rem = remaining - cum;
                        break;
                    }
                    cum += c;
                }
            }
            __syncthreads();
            prefix |= (uint32_t)sm.digit << shift;
            mask |= 255u << shift;
            remaining = sm.rem;
            __syncthreads();
        }
        T = prefix;
        take_eq = remaining;
    }
    int base_sel = 0, base_eq = 0;
    for (int j0 = 0; j0 < n; j0 += nt) {
        const int j = j0 + tid;
        bool gt = false, eq = false;
        float v = 0.f;
        if (j < n) {
            v = vals[j];
            if (take_all) {
                gt = true;
            } else {
                const uint32_t key = order_key(v);
                gt = key > T;
                eq = key == T;
            }
        }
        int eq_tot, sel_tot;
        const int eq_excl = block_exclusive_scan(eq ? 1 : 0, sm.warp_tot, &eq_tot);
        const bool sel = gt || (eq && (base_eq + eq_excl) < take_eq);
        const int sel_excl = block_exclusive_scan(sel ? 1 : 0, sm.warp_tot, &sel_tot);
        if (sel) {
            out_idx[base_sel + sel_excl] = j;
            out_val[base_sel + sel_excl] = v;
        }
        base_eq += eq_tot;
        base_sel += sel_tot;
    }
    for (int t = m + tid; t < k; t += nt) {
        out_idx[t] = -1;
        out_val[t] = 0.f;
    }
    if (tid == 0) *out_len = m;
    __syncthreads();
}

}  // namespace tam
