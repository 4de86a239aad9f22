// Warp-level pieces of the streaming exact top-k used by the pass-2 and indexer
// kernels: order-preserving keys, a batched 4 x 8-bit radix select of the k-th key
// over a candidate buffer, and stable compaction / emission.
#pragma once

#include <stdint.h>

namespace tam {
namespace sel {

// Order-preserving map float -> uint32 and back (a < b <=> key(a) < key(b)), so
// candidate keys of any sign sort as unsigned integers.
__device__ __forceinline__ uint32_t key_of(float v) {
    const uint32_t b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float value_of(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

struct SelWarpSmem {
    int hist[256];
};

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Candidate buffer of one query: keys[cap] (key_of(value)) followed by idx[cap],
// in ascending key index order.  Every pass over it batches kBatch loads per lane so the L2 latency
// is paid once per batch, not once per entry.
constexpr int kBatch = 8;

// k-th largest of keys[0..n) by an MSB-first 4 x 8-bit radix select over the warp.
// Returns the key T and how many entries equal to T belong to the top k (the
// earliest ones in buffer order).
// With passes < 4 the result is the k-th key's leading 8*passes bits (low bits zero):
// every key >= T is then at least the k-th largest's bin, and there are >= k of them.
__device__ __forceinline__ void warp_kth(const uint32_t* keys, int n, int k, int* hist,
                                         uint32_t& T, int& take_eq, int passes = 4) {
    const int lane = threadIdx.x & 31;
    uint32_t prefix = 0, mask = 0;
    int remaining = k;
#pragma unroll 1
    for (int shift = 24; shift >= 32 - 8 * passes; shift -= 8) {
        for (int b = lane; b < 256; b += 32) hist[b] = 0;
        __syncwarp();
        for (int base = 0; base < n; base += 32 * kBatch) {
            uint32_t kv[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int e = base + u * 32 + lane;
                kv[u] = e < n ? keys[e] : 0u;
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int e = base + u * 32 + lane;
                if (e < n && (kv[u] & mask) == prefix) atomicAdd(&hist[(kv[u] >> shift) & 255u], 1);
            }
        }
        __syncwarp();
        int c8[8], sum = 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            c8[t] = hist[255 - 8 * lane - t];
            sum += c8[t];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const int excl = incl - sum;
        const uint32_t who = __ballot_sync(0xffffffffu, excl < remaining && remaining <= incl);
        const int src = __ffs(who) - 1;
        int digit = -1, rem = 0, cum = excl;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            if (digit < 0 && cum + c8[t] >= remaining) {
                digit = 255 - 8 * lane - t;
                rem = remaining - cum;
            }
            cum += c8[t];
        }
        digit = __shfl_sync(0xffffffffu, digit, src);
        rem = __shfl_sync(0xffffffffu, rem, src);
        prefix |= (uint32_t)digit << shift;
        mask |= 255u << shift;
        remaining = rem;
        __syncwarp();
    }
    T = prefix;
    take_eq = remaining;
}

// Stable selection of the entries with key > T plus the first take_eq entries with
// key == T (select_all: every entry).  Kept entries go, in order, either back into
// the buffer (out_idx == null; positions never pass the read position, and a whole
// batch is read before any of it is written) or to the output row, where the value
// is written as float.  Returns the kept count.
__device__ __forceinline__ int warp_select(uint32_t* keys, uint32_t* idx, int n, uint32_t T,
                                           int take_eq, bool select_all, int32_t* out_idx,
                                           float* out_mass) {
    const int lane = threadIdx.x & 31;
    const uint32_t lt = lanemask_lt();
    int kept = 0, eq_seen = 0;
    for (int base = 0; base < n; base += 32 * kBatch) {
        uint32_t kv[kBatch], iv[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int e = base + u * 32 + lane;
            kv[u] = e < n ? keys[e] : 0u;
            iv[u] = e < n ? idx[e] : 0u;
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int e = base + u * 32 + lane;
            const bool in = e < n;
            const bool gt = in && (select_all || kv[u] > T);
            const bool eq = in && !select_all && kv[u] == T;
            const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
            const bool keep = gt || (eq && eq_seen + __popc(eqb & lt) < take_eq);
            const uint32_t kb = __ballot_sync(0xffffffffu, keep);
            if (keep) {
                const int pos = kept + __popc(kb & lt);
                if (out_idx) {
                    out_idx[pos] = (int32_t)iv[u];
                    out_mass[pos] = value_of(kv[u]);
                } else {
                    keys[pos] = kv[u];
                    idx[pos] = iv[u];
                }
            }
            kept += __popc(kb);
            eq_seen += __popc(eqb);
        }
        __syncwarp();
    }
    return kept;
}


}  // namespace sel
}  // namespace tam
