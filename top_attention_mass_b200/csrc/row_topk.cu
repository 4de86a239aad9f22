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
//   1. threshold guess: the r-th largest of s evenly spaced samples (s = 512, plus
//      256 per 2^17 keys of the row, at most 4096), r = mu + 3 sqrt(mu) + 4, mu = s k / n
//      the expected sample count at or above the k-th key, so that the guess lies
//      below the k-th key unless the samples are three deviations off; rows of at
//      most 2k + 256 keys take every key instead;
//   2-3. one pass over the row, chunk by chunk: each thread takes 8 consecutive
//      keys, a block-wide scan of the per-thread counts places the keys >= guess in
//      index order in shared memory (at most cap = max(4096, 2k + 2048); beyond
//      that they are only counted).  If the count is outside [k, cap], counting
//      passes bisect the key range for a threshold that fits and the pass repeats;
//   4. exact k-th key T of the candidates by a radix select over the bits below
//      their common prefix (8 bits per pass), and how many keys equal to T are
//      taken (the earliest ones);
//   5. ordered emission of the candidates > T and the first of those == T.
// If no threshold has a count in [k, cap] (more than cap keys tie at the k-th
// value) the bisection ends with the exact k-th key and step 5 runs over the row.
#include <algorithm>
#include <climits>

#include "common.cuh"
#include "launch.h"

namespace tam {
namespace {

constexpr int kRtThreads = 256;
constexpr int kRtWarps = kRtThreads / 32;
constexpr int kChunkKeys = 8;  // consecutive keys per thread in one chunk of the row

// Candidates staged in shared memory for budget k.
__host__ __device__ constexpr int cand_cap(int k) { return 2 * k + 2048 > 4096 ? 2 * k + 2048 : 4096; }

__device__ __forceinline__ uint32_t okey(float v) {
    const uint32_t b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float oval(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
__device__ __forceinline__ int64_t tri(int64_t i) { return i * (i + 1) / 2; }
__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }
__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Shared memory of one row: this header, then ckey[cap] and cidx[cap].
struct RowSmem {
    int hist[256];
    int wa[kRtWarps];       // per warp segment: count of the first predicate
    int wb[kRtWarps];       // per warp segment: count of keys equal to the threshold
    int wsc[2][kRtWarps];   // per warp totals of a chunk (double-buffered)
    int scal[4];
    unsigned int cmax;      // largest candidate key
    uint32_t* ckey;
    int32_t* cidx;
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
// Returns the block totals in tot_a / tot_b.  Contains barriers.
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

// Ordered emission after seg_count<Src, false> over the same (src, n, T): keeps
// key > T, or key == T among the first `quota` such keys, into the output row.
// Positions follow source order, so the kept keys stay in ascending index order.
template <class Src>
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
            const bool gt = in && kv[u] > T;
            const bool eq = in && kv[u] == T;
            const uint32_t gb = __ballot_sync(0xffffffffu, gt);
            const uint32_t eb = __ballot_sync(0xffffffffu, eq);
            const int g_pre = gt_before + __popc(gb & lt);
            const int e_pre = eq_before + __popc(eb & lt);
            if (gt || (eq && e_pre < quota)) {
                const int pos = g_pre + min(e_pre, quota);
                out_idx[pos] = src.idx(e);
                out_val[pos] = oval(kv[u]);
            }
            gt_before += __popc(gb);
            eq_before += __popc(eb);
        }
    }
}

// One pass over the row: the keys >= G, in index order, go to ckey / cidx (at most
// cap of them; beyond that they are only counted).  Thread t takes the 8
// consecutive keys at chunk + 8t; a warp scan plus the warp totals of the chunk
// give every thread its output position.  Returns the count; s.cmax receives the
// largest key >= G.  Contains barriers.
__device__ int compact_ge(const RowSrc& row, int n, uint32_t G, RowSmem& s, int cap) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int kStep = kRtThreads * kChunkKeys;
    int base = 0, buf = 0;
    uint32_t kmax = 0;
    // the next chunk's loads are issued before this chunk's scan and barrier
    float nx[kChunkKeys];
#pragma unroll
    for (int u = 0; u < kChunkKeys; ++u) {
        const int e = threadIdx.x * kChunkKeys + u;
        nx[u] = e < n ? __ldg(row.row + e) : 0.f;
    }
    for (int c0 = 0; c0 < n; c0 += kStep, buf ^= 1) {
        const int e0 = c0 + threadIdx.x * kChunkKeys;
        uint32_t kv[kChunkKeys];
        int cnt = 0;
#pragma unroll
        for (int u = 0; u < kChunkKeys; ++u) {
            kv[u] = okey(nx[u]);
            cnt += (e0 + u < n && kv[u] >= G) ? 1 : 0;
        }
#pragma unroll
        for (int u = 0; u < kChunkKeys; ++u) {
            const int e = e0 + kStep + u;
            nx[u] = e < n ? __ldg(row.row + e) : 0.f;
        }
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) s.wsc[buf][warp] = incl;
        __syncthreads();
        // exclusive prefix of the warp totals (lanes 0..15 hold one warp each)
        const int wt = lane < kRtWarps ? s.wsc[buf][lane] : 0;
        int wincl = wt;
#pragma unroll
        for (int o = 1; o < kRtWarps; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, wincl, o);
            if (lane >= o) wincl += y;
        }
        const int before = __shfl_sync(0xffffffffu, wincl - wt, warp);
        const int tot = __shfl_sync(0xffffffffu, wincl, kRtWarps - 1);
        if (cnt) {
            int pos = base + before + incl - cnt;
#pragma unroll
            for (int u = 0; u < kChunkKeys; ++u) {
                if (e0 + u < n && kv[u] >= G) {
                    if (pos < cap) {
                        s.ckey[pos] = kv[u];
                        s.cidx[pos] = e0 + u;
                    }
                    ++pos;
                    kmax = max(kmax, kv[u]);
                }
            }
        }
        base += tot;
    }
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) atomicMax(&s.cmax, kmax);
    return base;
}

// Exact k-th largest key of the c candidates (k <= c), all >= G and <= s.cmax:
// returns T and how many of the keys equal to T belong to the top k.  The bits
// above the highest bit where G and cmax differ are common to every candidate, so
// the radix passes start below them.  Contains barriers.
__device__ void cand_kth(RowSmem& s, int c, int k, uint32_t G, uint32_t& T, int& take_eq) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t diff = G ^ s.cmax;
    if (diff == 0u) {           // every candidate equals G
        T = G;
        take_eq = k;
        return;
    }
    int hi_bit = 31 - __clz(diff);
    uint32_t mask = ~(uint32_t)((2ull << hi_bit) - 1ull);
    uint32_t prefix = G & mask;
    int remaining = k;
#pragma unroll 1
    while (hi_bit >= 0) {
        const int width = min(8, hi_bit + 1);
        const int shift = hi_bit + 1 - width;
        const uint32_t dmask = (1u << width) - 1u;
        for (int b = threadIdx.x; b < 256; b += blockDim.x) s.hist[b] = 0;
        __syncthreads();
        for (int e = threadIdx.x; e < c; e += blockDim.x) {
            const uint32_t kv = s.ckey[e];
            if ((kv & mask) == prefix) atomicAdd(&s.hist[(kv >> shift) & dmask], 1);
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
        mask |= dmask << shift;
        remaining = s.scal[1];
        hi_bit = shift - 1;
        __syncthreads();
    }
    T = prefix;
    take_eq = remaining;
}

struct RowTopkParams {
    const float* slab;
    int64_t row0;
    int n_rows, budget, cap;
    int32_t* sup_idx;
    int32_t* sup_len;
    float* sup_val;
};

__global__ void __launch_bounds__(kRtThreads, 6) k_row_topk(const RowTopkParams p) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    RowSmem& s = *reinterpret_cast<RowSmem*>(smem_raw);
    const int64_t i = p.row0 + (p.n_rows - 1 - (int)blockIdx.x);
    const int n = (int)i + 1;
    const int k = p.budget, cap = p.cap;
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
    if (threadIdx.x == 0) {
        s.ckey = reinterpret_cast<uint32_t*>(smem_raw + sizeof(RowSmem));
        s.cidx = reinterpret_cast<int32_t*>(s.ckey + cap);
        s.cmax = 0u;
    }
    __syncthreads();

    // ---- 1: threshold guess G (rows of at most 2k + 256 keys: G = 0, every key)
    uint32_t G = 0;
    if (!(n <= 2 * k + 256 && n <= cap)) {
        // m samples per thread, evenly spaced over the row, staged in the (still
        // unused) candidate buffer; warp 0 then finds the r-th largest
        const int m = min(16, 2 + (n >> 17));
        const int s_tot = kRtThreads * m;
        const float step = (float)n / (float)s_tot;
        for (int u = 0; u < m; ++u) {
            const int t = threadIdx.x + u * kRtThreads;
            s.ckey[t] = row.key(min(n - 1, (int)((float)t * step)));
        }
        __syncthreads();
        if (warp_id() == 0) {
            const float mu = (float)s_tot * (float)k / (float)n;
            const int r = max(1, min(s_tot, (int)ceilf(mu + 3.f * sqrtf(mu) + 4.f)));
            const int lane = threadIdx.x & 31;
            // bits above the highest one where the smallest and largest sample differ
            // are common to all samples
            // the first 512 samples sit in registers (16 per lane), the rest are re-read
            uint32_t v[16];
            uint32_t mn = 0xffffffffu, mx = 0u;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                v[u] = s.ckey[lane + 32 * u];
                mn = min(mn, v[u]);
                mx = max(mx, v[u]);
            }
            for (int e = 512 + lane; e < s_tot; e += 32) {
                mn = min(mn, s.ckey[e]);
                mx = max(mx, s.ckey[e]);
            }
            mn = __reduce_min_sync(0xffffffffu, mn);
            mx = __reduce_max_sync(0xffffffffu, mx);
            uint32_t t = mn;
            if (mn != mx) {
                const int top = 31 - __clz(mn ^ mx);
                t = mn & ~(uint32_t)((2ull << top) - 1ull);
                for (int b = top; b >= 0; --b) {
                    const uint32_t c = t | (1u << b);
                    int cl = 0;
#pragma unroll
                    for (int u = 0; u < 16; ++u) cl += v[u] >= c ? 1 : 0;
                    for (int e = 512 + lane; e < s_tot; e += 32) cl += s.ckey[e] >= c ? 1 : 0;
                    if (__reduce_add_sync(0xffffffffu, cl) >= r) t = c;
                }
            }
            if (lane == 0) s.scal[2] = (int)t;
        }
        __syncthreads();
        G = (uint32_t)s.scal[2];
    }
    // ---- 2-3: ordered candidates (keys >= G)
    int cnt = compact_ge(row, n, G, s, cap), dummy;
    bool found = cnt >= k && cnt <= cap;
    uint64_t lo = 0, hi = 1ull << 32;   // #(key >= lo) >= k;  #(key >= hi) < k
    int c_hi = 0;                       // #(key >= hi)
    if (!found) {
        if (cnt < k) {
            hi = G;
            c_hi = cnt;
        } else {
            lo = G;
        }
        while (hi - lo > 1) {
            G = (uint32_t)((lo + hi) >> 1);
            seg_count<RowSrc, true>(row, n, G, s, cnt, dummy);
            if (cnt >= k && cnt <= cap) {
                found = true;
                break;
            }
            if (cnt < k) {
                hi = G;
                c_hi = cnt;
            } else {
                lo = G;
            }
        }
        if (found) {
            if (threadIdx.x == 0) s.cmax = 0u;
            __syncthreads();
            cnt = compact_ge(row, n, G, s, cap);
        }
    }
    if (found) {
        __syncthreads();
        // ---- 4: exact k-th key of the candidates
        uint32_t T;
        int take_eq;
        cand_kth(s, cnt, k, G, T, take_eq);
        // ---- 5: ordered emission of the top k
        const CandSrc cs{&s};
        seg_count<CandSrc, false>(cs, cnt, T, s, dummy, dummy);
        seg_emit<CandSrc>(cs, cnt, T, take_eq, s, oi, ov);
    } else {
        // more than cap keys tie at the k-th value: lo is that value, exactly
        const uint32_t T = (uint32_t)lo;
        seg_count<RowSrc, false>(row, n, T, s, dummy, dummy);
        seg_emit<RowSrc>(row, n, T, k - c_hi, s, oi, ov);
    }
    if (threadIdx.x == 0) p.sup_len[i] = k;
}

// ---------------------------------------------------------------- streamed selection
// Threshold of each row from its sampled keys (a lower bound of the row's k-th
// value unless the samples are z deviations off; cand_select checks it).
struct SampleTauParams {
    const float* slab;
    int64_t row0;
    int n_rows, S, budget, take_all, force;
    float z;
    float* tau;
};

__global__ void __launch_bounds__(kRtThreads) k_sample_tau(const SampleTauParams p) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    RowSmem& s = *reinterpret_cast<RowSmem*>(smem_raw);
    const int64_t i = p.row0 + (p.n_rows - 1 - (int)blockIdx.x);
    const int n = (int)i + 1;
    if (n <= p.take_all) {
        if (threadIdx.x == 0) p.tau[i] = -INFINITY;
        return;
    }
    if (p.force) {
        if (threadIdx.x == 0) p.tau[i] = p.force == 1 ? INFINITY : -INFINITY;
        return;
    }
    const int ns = (int)(i / p.S) + 1;
    const float* row = p.slab + (sample_offset(i, p.S) - sample_offset(p.row0, p.S));
    if (threadIdx.x == 0) {
        s.ckey = reinterpret_cast<uint32_t*>(smem_raw + sizeof(RowSmem));
        s.cmax = 0u;
        s.scal[3] = -1;                       // smallest key, as ~x to use atomicMax
    }
    __syncthreads();
    uint32_t mx = 0u, mn = 0xffffffffu;
    for (int t = threadIdx.x; t < ns; t += blockDim.x) {
        const uint32_t kv = okey(__ldg(row + t));
        s.ckey[t] = kv;
        mx = max(mx, kv);
        mn = min(mn, kv);
    }
    mx = __reduce_max_sync(0xffffffffu, mx);
    mn = __reduce_min_sync(0xffffffffu, mn);
    if ((threadIdx.x & 31) == 0) {
        atomicMax(&s.cmax, mx);
        atomicMin(reinterpret_cast<unsigned int*>(&s.scal[3]), mn);
    }
    __syncthreads();
    const int k = min(p.budget, n);
    const float mu = (float)ns * (float)k / (float)n;
    const int r = max(1, min(ns, (int)ceilf(mu + p.z * sqrtf(mu) + 4.f)));
    uint32_t T;
    int take_eq;
    cand_kth(s, ns, r, (uint32_t)s.scal[3], T, take_eq);
    if (threadIdx.x == 0) p.tau[i] = oval(T);
}

// Exact top-k of a row from its candidate segments.  The k-th key T is found by the
// same radix select as for materialised rows; the kept keys are then marked in a
// bitmap over the row's key indices (one bit per key 0..i), whose word-wise prefix
// popcount gives every kept key its place in ascending index order.  Equal values at T
// keep the smallest indices: when more keys equal T than are taken, the equal keys
// are marked in a second bitmap and the cut-off index is the take-th set bit.
struct CandSelParams {
    const uint2* cand;
    const int32_t* cnt;
    int64_t row0;
    int n_rows, nseg, seg_cap, budget, max_words;
    int32_t* sup_idx;
    int32_t* sup_len;
    float* sup_val;
    int32_t* fb;
};

constexpr int kMaxSegments = 8;

// Exclusive prefix of the popcounts of words [0, nw) into pre[]: thread t sums a
// contiguous range, one block scan (s.hist as its scratch, so not during a radix
// pass), then each thread writes its range.  Contains barriers.  Returns the total.
__device__ int word_prefix(const uint32_t* bits, int* pre, int nw, RowSmem& s) {
    const int per = (nw + kRtThreads - 1) / kRtThreads;
    const int w0 = min(nw, (int)threadIdx.x * per), w1 = min(nw, w0 + per);
    int c = 0;
    for (int w = w0; w < w1; ++w) c += __popc(bits[w]);
    int tot;
    int run = block_exclusive_scan(c, s.hist, &tot);        // hist: free scratch here
    for (int w = w0; w < w1; ++w) {
        pre[w] = run;
        run += __popc(bits[w]);
    }
    __syncthreads();
    return tot;
}

__global__ void __launch_bounds__(kRtThreads) k_cand_select(const CandSelParams p) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    RowSmem& s = *reinterpret_cast<RowSmem*>(smem_raw);
    __shared__ int soff[kMaxSegments + 1];
    __shared__ int sflag, s_ceq, s_cut, s_badidx;
    const int64_t i = p.row0 + (p.n_rows - 1 - (int)blockIdx.x);
    const int n = (int)i + 1;
    const int k = min(p.budget, n);
    const int cap = p.nseg * p.seg_cap;
    const int nw = (n + 31) >> 5;
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem_raw + sizeof(RowSmem)) + 2 * cap;
    int* pre = reinterpret_cast<int*>(bits + p.max_words);
    if (threadIdx.x == 0) {
        s.ckey = reinterpret_cast<uint32_t*>(smem_raw + sizeof(RowSmem));
        s.cidx = reinterpret_cast<int32_t*>(s.ckey + cap);
        s.cmax = 0u;
        s.scal[3] = -1;
        s_ceq = 0;
        s_cut = 0x7fffffff;
        s_badidx = 0;
        const int32_t* c = p.cnt + (i - p.row0) * p.nseg;
        int tot = 0;
        bool bad = false;
        for (int g = 0; g < p.nseg; ++g) {
            const int cg = c[g];
            bad = bad || cg < 0 || cg > p.seg_cap;
            soff[g] = tot;
            tot += max(0, min(cg, p.seg_cap));
        }
        soff[p.nseg] = tot;
        // overflowed segments lost keys; fewer than k keys means the threshold was
        // above the k-th value: either way the row goes to the fallback
        sflag = bad || tot < k;
        if (sflag) {
            const int t = atomicAdd(p.fb, 1);
            p.fb[1 + t] = (int32_t)i;
        }
    }
    __syncthreads();
    if (sflag) return;
    const int tot = soff[p.nseg];
    // the segments back to back, and a clear bitmap
    const uint2* base = p.cand + (i - p.row0) * (int64_t)cap;
    uint32_t mx = 0u, mn = 0xffffffffu;
    for (int t = threadIdx.x; t < tot; t += blockDim.x) {
        int g = 0;
        while (g + 1 < p.nseg && soff[g + 1] <= t) ++g;
        const uint2 e = base[g * p.seg_cap + (t - soff[g])];
        const uint32_t kv = okey(__uint_as_float(e.x));
        // a key outside [0, i] can only come from a scan that did not finish (a wait
        // that gave up): the row is left to the fallback and never indexes the bitmap
        if (e.y > (uint32_t)i) s_badidx = 1;
        s.ckey[t] = kv;
        s.cidx[t] = (int32_t)e.y;
        mx = max(mx, kv);
        mn = min(mn, kv);
    }
    for (int w = threadIdx.x; w < nw; w += blockDim.x) bits[w] = 0u;
    mx = __reduce_max_sync(0xffffffffu, mx);
    mn = __reduce_min_sync(0xffffffffu, mn);
    if ((threadIdx.x & 31) == 0) {
        atomicMax(&s.cmax, mx);
        atomicMin(reinterpret_cast<unsigned int*>(&s.scal[3]), mn);
    }
    __syncthreads();
    if (s_badidx) {
        if (threadIdx.x == 0) {
            const int t = atomicAdd(p.fb, 1);
            p.fb[1 + t] = (int32_t)i;
        }
        return;
    }
    uint32_t T = 0u;
    int take_eq = 0;
    if (tot > k) cand_kth(s, tot, k, (uint32_t)s.scal[3], T, take_eq);  // else keep them all
    // keys above T; count the keys equal to T
    int ceq = 0;
    for (int t = threadIdx.x; t < tot; t += blockDim.x) {
        const uint32_t kv = s.ckey[t];
        if (kv > T) {
            const int x = s.cidx[t];
            atomicOr(&bits[x >> 5], 1u << (x & 31));
        }
        ceq += kv == T && tot > k;
    }
    ceq = __reduce_add_sync(0xffffffffu, ceq);
    if ((threadIdx.x & 31) == 0 && ceq) atomicAdd(&s_ceq, ceq);
    __syncthreads();
    if (take_eq > 0 && s_ceq > take_eq) {
        // more keys tie at T than are taken: the cut-off is the take_eq-th smallest index
        uint32_t* eqb = reinterpret_cast<uint32_t*>(pre);
        for (int w = threadIdx.x; w < nw; w += blockDim.x) eqb[w] = 0u;
        __syncthreads();
        for (int t = threadIdx.x; t < tot; t += blockDim.x)
            if (s.ckey[t] == T) atomicOr(&eqb[s.cidx[t] >> 5], 1u << (s.cidx[t] & 31));
        __syncthreads();
        const int per = (nw + kRtThreads - 1) / kRtThreads;
        const int w0 = min(nw, (int)threadIdx.x * per), w1 = min(nw, w0 + per);
        int c = 0;
        for (int w = w0; w < w1; ++w) c += __popc(eqb[w]);
        int tot_eq;
        int run = block_exclusive_scan(c, s.hist, &tot_eq);
        for (int w = w0; w < w1; ++w) {
            const uint32_t word = eqb[w];
            const int pc = __popc(word);
            if (run < take_eq && take_eq <= run + pc) {
                uint32_t m = word;
                for (int r = take_eq - run; r > 1; --r) m &= m - 1;   // drop the lower bits
                s_cut = w * 32 + (__ffs(m) - 1);
            }
            run += pc;
        }
        __syncthreads();
    }
    if (take_eq > 0) {
        const int cut = s_cut;
        for (int t = threadIdx.x; t < tot; t += blockDim.x) {
            const int x = s.cidx[t];
            if (s.ckey[t] == T && x <= cut) atomicOr(&bits[x >> 5], 1u << (x & 31));
        }
    }
    __syncthreads();
    word_prefix(bits, pre, nw, s);
    int32_t* oi = p.sup_idx + i * (int64_t)p.budget;
    float* ov = p.sup_val + i * (int64_t)p.budget;
    for (int t = threadIdx.x; t < tot; t += blockDim.x) {
        const int x = s.cidx[t];
        const uint32_t word = bits[x >> 5];
        const uint32_t bit = 1u << (x & 31);
        if (word & bit) {
            const int pos = pre[x >> 5] + __popc(word & (bit - 1u));
            oi[pos] = x;
            ov[pos] = oval(s.ckey[t]);
        }
    }
    for (int t = k + threadIdx.x; t < p.budget; t += blockDim.x) {
        oi[t] = -1;
        ov[t] = 0.f;
    }
    if (threadIdx.x == 0) p.sup_len[i] = k;
}

}  // namespace

cudaError_t sample_tau(const float* slab, int64_t row0, int64_t row1, int S, int budget,
                       int take_all, float z, int force, float* tau, cudaStream_t st) {
    if (row1 <= row0) return cudaSuccess;
    SampleTauParams p{slab, row0, (int)(row1 - row0), S, budget, take_all, force, z, tau};
    const int max_samples = (int)((row1 - 1) / S) + 1;
    const int smem = (int)sizeof(RowSmem) + max_samples * 4;
    cudaError_t e = cudaFuncSetAttribute(k_sample_tau, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k_sample_tau<<<(unsigned)(row1 - row0), kRtThreads, smem, st>>>(p);
    note_launch();
    return cudaGetLastError();
}

int cand_select_smem(int64_t max_row_keys, int cap) {
    const int64_t words = (max_row_keys + 31) / 32;
    return (int)std::min<int64_t>(INT32_MAX, (int64_t)sizeof(RowSmem) + (int64_t)cap * 8 + words * 8);
}

cudaError_t cand_select(const void* cand, const int32_t* cnt, int64_t row0, int64_t row1,
                        int nseg, int seg_cap, int budget, int32_t* sup_idx, int32_t* sup_len,
                        float* sup_val, int32_t* fb, cudaStream_t st) {
    if (row1 <= row0) return cudaSuccess;
    if (nseg < 1 || nseg > kMaxSegments) return cudaErrorInvalidValue;
    const int max_words = (int)((row1 + 31) / 32);
    CandSelParams p{reinterpret_cast<const uint2*>(cand), cnt, row0, (int)(row1 - row0), nseg,
                    seg_cap, budget, max_words, sup_idx, sup_len, sup_val, fb};
    const int smem = cand_select_smem(row1, nseg * seg_cap);
    if (smem > kCandSelectMaxSmem) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(k_cand_select, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k_cand_select<<<(unsigned)(row1 - row0), kRtThreads, smem, st>>>(p);
    note_launch();
    return cudaGetLastError();
}

cudaError_t row_topk(const float* slab, int64_t row0, int64_t row1, int budget, int32_t* sup_idx,
                     int32_t* sup_len, float* sup_val, cudaStream_t st) {
    if (row1 <= row0) return cudaSuccess;
    const int cap = cand_cap(budget);
    RowTopkParams p{slab, row0, (int)(row1 - row0), budget, cap, sup_idx, sup_len, sup_val};
    const int smem = (int)sizeof(RowSmem) + cap * 8;
    cudaError_t e = cudaFuncSetAttribute(k_row_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k_row_topk<<<(unsigned)(row1 - row0), kRtThreads, smem, st>>>(p);
    note_launch();
    return cudaGetLastError();
}

}  // namespace tam
