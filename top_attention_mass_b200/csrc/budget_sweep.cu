// Budget sweep from one pass-2 run: each support row's mass at several budgets.
//
//   m_r(k) = sum of the k largest values of row r of a top-k_max support (k <= k_max),
//            = the support mass of the top-k support, since the top-k of a row is the
//            top-k of its top-k_max for every k <= k_max;  k >= len_r: the whole row.
//
// (gist.science technical report §3.1, "Budget-Sensitivitaet": the oracle compared at
// top-k budgets of 256 to 2048 over 4K-100K contexts; the sparsity at a budget is the
// closed form 1 - sum_i min(k, i+1) / sum_i (i+1) and needs no kernel.)
//
// One CTA per row: the row's values go to shared memory as order-preserving keys
// (masses are non-negative, so the float bits already order them); for each budget a
// 4 x 8-bit radix select finds the k-th largest key T and how many entries equal to
// T are taken, and a block reduction sums the entries above T plus those.
#include "common.cuh"
#include "launch.h"

namespace tam {
namespace {

constexpr int kSwThreads = 256;

struct SweepParams {
    const float* val;
    const int32_t* len;
    int kmax, nk;
    int ks[kMaxSweepBudgets];
    float* out;             // [rows, nk]
};

__global__ void __launch_bounds__(kSwThreads) k_support_mass_curve(const SweepParams p) {
    extern __shared__ uint32_t s_key[];                      // kmax keys
    __shared__ int hist[256];
    __shared__ int s_digit, s_rem;
    __shared__ float s_red[kSwThreads / 32];
    const int r = blockIdx.x;
    const int n = min(max(p.len[r], 0), p.kmax);
    const float* row = p.val + (size_t)r * p.kmax;
    for (int e = threadIdx.x; e < n; e += kSwThreads) s_key[e] = __float_as_uint(fmaxf(row[e], 0.f));
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int t = 0; t < p.nk; ++t) {
        const int kb = p.ks[t];
        uint32_t T = 0;
        int take_eq = 0;
        const bool all = kb >= n;
        if (!all) {
            uint32_t prefix = 0, mask = 0;
            int remaining = kb;
            for (int shift = 24; shift >= 0; shift -= 8) {
                for (int b = threadIdx.x; b < 256; b += kSwThreads) hist[b] = 0;
                __syncthreads();
                for (int e = threadIdx.x; e < n; e += kSwThreads) {
                    const uint32_t key = s_key[e];
                    if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
                }
                __syncthreads();
                if (warp == 0) {
                    // lane l scans bins 255 - 8l .. 248 - 8l; a shuffle scan finds the lane
                    // whose bins hold the remaining-th largest key
                    int c8[8], sum = 0;
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        c8[u] = hist[255 - 8 * lane - u];
                        sum += c8[u];
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
                        for (int u = 0; u < 8; ++u) {
                            if (cum + c8[u] >= remaining) {
                                s_digit = 255 - 8 * lane - u;
                                s_rem = remaining - cum;
                                break;
                            }
                            cum += c8[u];
                        }
                    }
                }
                __syncthreads();
                prefix |= (uint32_t)s_digit << shift;
                mask |= 255u << shift;
                remaining = s_rem;
                __syncthreads();
            }
            T = prefix;
            take_eq = remaining;
        }
        float acc = 0.f;
        for (int e = threadIdx.x; e < n; e += kSwThreads) {
            const uint32_t key = s_key[e];
            if (all || key > T) acc += __uint_as_float(key);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) s_red[warp] = acc;
        __syncthreads();
        if (threadIdx.x == 0) {
            float sum = (float)take_eq * __uint_as_float(T);
            for (int w = 0; w < kSwThreads / 32; ++w) sum += s_red[w];
            p.out[(size_t)r * p.nk + t] = sum;
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t support_mass_curve(const float* val, const int32_t* len, int64_t rows, int kmax,
                               const int32_t* ks, int nk, float* out, cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    SweepParams p{};
    p.val = val;
    p.len = len;
    p.kmax = kmax;
    p.nk = nk;
    for (int t = 0; t < nk; ++t) p.ks[t] = ks[t];
    p.out = out;
    const int smem = kmax * (int)sizeof(uint32_t);
    k_support_mass_curve<<<(unsigned)rows, kSwThreads, smem, st>>>(p);
    note_launch();
    return cudaGetLastError();
}

}  // namespace tam
