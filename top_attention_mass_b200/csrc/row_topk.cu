// Exact per-row top-k over materialised score rows: the selection step of the
// per-query oracle and of the indexer.
//
//   S_i = top-min(k, i+1) of row i (values x_i[0..i]),
//   ties at the k-th value broken toward the smaller key index,
//   emitted in ascending key index with their values.
//
// (arXiv 2606.07703, Abstract: the per-query oracle keeps the keys of largest
// head-averaged mass; gist.science technical report §2.1 "Selektion" and §2.2 for
// the indexer's top-k of its scores.)
//
// Row i lives in a triangular slab: it starts tri(i) - tri(row0) floats after the
// slab base, tri(i) = i (i + 1) / 2, and holds i + 1 values.  The producing kernel
// has just written it, so the passes below read it from L2.
//
// One CTA per row (longest rows first).  Values are compared as order-preserving
// 32-bit keys, so any float (negative indexer scores included) orders exactly.
//   1. threshold guess: the r-th largest of 512 evenly spaced samples, r chosen so
//      that about 1.25 k + 64 keys of the row are expected at or above it;
//   2. count the keys >= guess (per warp segment); if the count is outside
//      [k, kCap] bisect the key range with further counting passes;
//   3. ordered compaction of the keys >= guess into shared memory (at most kCap);
//   4. exact k-th key T of the candidates by a 4 x 8-bit radix select, and how
//      many keys equal to T are taken (the earliest ones);
//   5. ordered emission of the candidates > T and the first of those == T.
// If no guess has a count in [k, kCap] (more than kCap keys tie at the k-th value)
// the bisection ends with the exact k-th key and step 5 runs over the row itself.
#include "common.cuh"
#include "launch.h"

namespace tam {
namespace {

constexpr int kRtThreads = 512;
constexpr int kRtWarps = kRtThreads / 32;
constexpr int kCap = 8192;     // candidates staged in shared memory

__device__ __forceinline__ uint32_t okey(float v) {
    const uint32_t b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float oval(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
__device__ __forceinline__ int64_t tri(int64_t i) { return i * (i + 1) / 2; }
__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

struct RowSmem {
    uint32_t ckey[kCap];
    int32_t cidx[kCap];
    int hist[256];
    int wa[kRtWarps];       // per warp segment: count of the first predicate
    int wb[kRtWarps];       // per warp segment: count of keys equal to the threshold
    int scal[4];
};

// Source of a pass: the row in global memory or the staged candidates.
struct RowSrc {
    const float* row;
    __device__ __forceinline__ uint32_t key(int e) const { return okey(__ldg(row + e)); }
    __device__ __forceinline__ int32_t idx(int e) const { return e; }
};
struct CandSrc {
    const RowSmem* s;
    __device__ __forceinline__ uint32_t key(int e) const { return s->ckey[e]; }
    __device__ __forceinline__ int32_t idx(int e) const { return s->cidx[e]; }
};

// Warp w owns the contiguous segment [w * seg, min(n, (w + 1) * seg)).
__device__ __forceinline__ int seg_len(int n) { return (((n + kRtWarps - 1) / kRtWarps) + 31) & ~31; }

// Per warp segment: wa = #(key >= T) (GE) or #(key > T) (!GE); wb = #(key == T).
// Returns the block totals through scal[0] / scal[1].  Contains barriers.
template <class Src, bool GE>
__device__ void seg_count(const Src& src, int n, uint32_t T, RowSmem& s, int& tot_a, int& tot_b) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seg = seg_len(n);
    const int beg = warp * seg, end = min(n, beg + seg);
    int ca = 0, cb = 0;
    constexpr int U = 8;
    for (int base = beg; base < end; base += 32 * U) {
        uint32_t kv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = base + u * 32 + lane;
            kv[u] = e < end ? src.key(e) : 0u;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = base + u * 32 + lane;
            if (e < end) {
                ca += GE ? (kv[u] >= T) : (kv[u] > T);
                cb += kv[u] == T;
            }
        }
    }
    ca = __reduce_add_sync(0xffffffffu, ca);
    cb = __reduce_add_sync(0xffffffffu, cb);
    __syncthreads();                       // previous readers of wa / wb are done
    if (lane == 0) {
        s.wa[warp] = ca;
        s.wb[warp] = cb;
    }
    __syncthreads();
    tot_a = 0;
    tot_b = 0;
#pragma unroll
    for (int w = 0; w < kRtWarps; ++w) {
        tot_a += s.wa[w];
        tot_b += s.wb[w];
    }
}

// Ordered compaction after seg_count over the same (src, n, T).
//   GE:  keep key >= T                     -> candidates (ckey / cidx)
//   !GE: keep key > T, or key == T among the first `quota` such keys -> output row
// Positions follow source order, so the kept keys stay in ascending index order.
template <class Src, bool GE>
__device__ void seg_emit(const Src& src, int n, uint32_t T, int quota, RowSmem& s,
                         int32_t* out_idx, float* out_val) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seg = seg_len(n);
    const int beg = warp * seg, end = min(n, beg + seg);
    int gt_before = 0, eq_before = 0;
    for (int w = 0; w < warp; ++w) {
        gt_before += s.wa[w];
        eq_before += s.wb[w];
    }
    const uint32_t lt = lanemask_lt();
    constexpr int U = 8;
    for (int base = beg; base < end; base += 32 * U) {
        uint32_t kv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = base + u * 32 + lane;
            kv[u] = e < end ? src.key(e) : 0u;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = base + u * 32 + lane;
            const bool in = e < end;
            const bool gt = in && (GE ? kv[u] >= T : kv[u] > T);
            const bool eq = in && !GE && kv[u] == T;
            const uint32_t gb = __ballot_sync(0xffffffffu, gt);
            const uint32_t eb = __ballot_sync(0xffffffffu, eq);
            const int g_pre = gt_before + __popc(gb & lt);
            const int e_pre = eq_before + __popc(eb & lt);
            if (GE) {
                if (gt) {
                    s.ckey[g_pre] = kv[u];
                    s.cidx[g_pre] = src.idx(e);
                }
            } else if (gt || (eq && e_pre < quota)) {
                const int pos = g_pre + min(e_pre, quota);
                out_idx[pos] = src.idx(e);
                out_val[pos] = oval(kv[u]);
            }
            gt_before += __popc(gb);
            eq_before += __popc(eb);
        }
    }
}

// Exact k-th largest key of the c candidates (k <= c): returns T and how many of
// the keys equal to T belong to the top k.  Contains barriers.
__device__ void cand_kth(RowSmem& s, int c, int k, uint32_t& T, int& take_eq) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t prefix = 0, mask = 0;
    int remaining = k;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = threadIdx.x; b < 256; b += blockDim.x) s.hist[b] = 0;
        __syncthreads();
        for (int e = threadIdx.x; e < c; e += blockDim.x) {
            const uint32_t kv = s.ckey[e];
            if ((kv & mask) == prefix) atomicAdd(&s.hist[(kv >> shift) & 255u], 1);
        }
        __syncthreads();
        if (warp == 0) {
            // lane l holds bins 255 - 8l .. 248 - 8l (descending)
            int c8[8], sum = 0;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                c8[t] = s.hist[255 - 8 * lane - t];
                sum += c8[t];
            }
            int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int excl = incl - sum;
            if (excl < remaining && remaining <= incl) {
                int cum = excl;
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    if (cum + c8[t] >= remaining) {
                        s.scal[0] = 255 - 8 * lane - t;
                        s.scal[1] = remaining - cum;
                        break;
                    }
                    cum += c8[t];
                }
            }
        }
        __syncthreads();
        prefix |= (uint32_t)s.scal[0] << shift;
        mask |= 255u << shift;
        remaining = s.scal[1];
        __syncthreads();
    }
    T = prefix;
    take_eq = remaining;
}

struct RowTopkParams {
    const float* slab;
    int64_t row0;
    int n_rows, budget;
    int32_t* sup_idx;
    int32_t* sup_len;
    float* sup_val;
};

__global__ void __launch_bounds__(kRtThreads) k_row_topk(const RowTopkParams p) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    RowSmem& s = *reinterpret_cast<RowSmem*>(smem_raw);
    const int64_t i = p.row0 + (p.n_rows - 1 - (int)blockIdx.x);
    const int n = (int)i + 1;
    const int k = p.budget;
    const RowSrc row{p.slab + (tri(i) - tri(p.row0))};
    int32_t* oi = p.sup_idx + i * (int64_t)k;
    float* ov = p.sup_val + i * (int64_t)k;

    if (n <= k) {           // the whole causal prefix is the support
        for (int t = threadIdx.x; t < k; t += blockDim.x) {
            oi[t] = t < n ? t : -1;
            ov[t] = t < n ? __ldg(row.row + t) : 0.f;
        }
        if (threadIdx.x == 0) p.sup_len[i] = n;
        return;
    }

    // ---- 1-2: a threshold G with k <= #(key >= G) <= kCap
    uint64_t lo = 0, hi = 1ull << 32;   // #(key >= lo) >= k;  #(key >= hi) < k
    int c_hi = 0;                       // #(key >= hi)
    uint32_t G = 0;
    int cnt = n, dummy;
    bool found = n <= kCap;             // G = 0 takes the whole row
    if (!found) {
        // r-th largest of the samples, r so that about 1.25 k + 64 keys are expected >= it
        const int sidx = (int)(((int64_t)threadIdx.x * n) / kRtThreads);
        const uint32_t sk = row.key(sidx);
        const double want = 1.25 * k + 64.0;
        int r = (int)ceil(want * kRtThreads / n);
        r = max(1, min(kRtThreads, r));
        uint32_t t = 0;
        for (int b = 31; b >= 0; --b) {
            const uint32_t c = t | (1u << b);
            if (__syncthreads_count(sk >= c) >= r) t = c;
        }
        G = t;
        for (int probe = 0; probe < 40; ++probe) {
            seg_count<RowSrc, true>(row, n, G, s, cnt, dummy);
            if (cnt >= k && cnt <= kCap) {
                found = true;
                break;
            }
            if (cnt < k) {
                hi = G;
                c_hi = cnt;
            } else {
                lo = G;
            }
            if (hi - lo <= 1) break;
            G = (uint32_t)((lo + hi) >> 1);
        }
    }
    if (found) {
        // ---- 3: ordered candidates (keys >= G); seg_count above left their warp counts
        if (G == 0u) seg_count<RowSrc, true>(row, n, 0u, s, cnt, dummy);
        seg_emit<RowSrc, true>(row, n, G, 0, s, nullptr, nullptr);
        __syncthreads();
        // ---- 4: exact k-th key of the candidates
        uint32_t T;
        int take_eq;
        cand_kth(s, cnt, k, T, take_eq);
        // ---- 5: ordered emission of the top k
        const CandSrc cs{&s};
        seg_count<CandSrc, false>(cs, cnt, T, s, dummy, dummy);
        seg_emit<CandSrc, false>(cs, cnt, T, take_eq, s, oi, ov);
    } else {
        // more than kCap keys tie at the k-th value: lo is that value, exactly
        const uint32_t T = (uint32_t)lo;
        seg_count<RowSrc, false>(row, n, T, s, dummy, dummy);
        seg_emit<RowSrc, false>(row, n, T, k - c_hi, s, oi, ov);
    }
    if (threadIdx.x == 0) p.sup_len[i] = k;
}

}  // namespace

size_t row_topk_smem_bytes() { return sizeof(RowSmem); }

cudaError_t row_topk(const float* slab, int64_t row0, int64_t row1, int budget, int32_t* sup_idx,
                     int32_t* sup_len, float* sup_val, cudaStream_t st) {
    if (row1 <= row0) return cudaSuccess;
    RowTopkParams p{slab, row0, (int)(row1 - row0), budget, sup_idx, sup_len, sup_val};
    const int smem = (int)sizeof(RowSmem);
    cudaError_t e = cudaFuncSetAttribute(k_row_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k_row_topk<<<(unsigned)(row1 - row0), kRtThreads, smem, st>>>(p);
    note_launch();
    return cudaGetLastError();
}

}  // namespace tam
