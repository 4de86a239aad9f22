// The indexer's distillation target: per query, the KL divergence of the indexer's
// distribution from the head-averaged attention mass.
//
//   KL_i = sum_{j <= i} P_i[j] log(P_i[j] / q_i[j]),  q_i = softmax_{j <= i}(t_i),
//        = sum_j P_i[j] log P_i[j] - sum_j P_i[j] t_ij + log sum_j exp(t_ij)
//   (sum_j P_i[j] = 1; 0 log 0 = 0), t_ij = q_idx_i . k_idx_j (scale 1)
//
// (gist.science technical report §2.2, "Trainingsziel": the head-collapsed indexer is
// trained by KL distillation from the dense attention-mass distribution.)
//
// Both rows come from the row slabs the per-query mass kernel and the indexer score
// kernel wrote for the same chunk of queries (row i starts tri(i) - tri(row0) floats
// in).  One 256-thread CTA per row makes one pass over both: a running max and
// rescaled exp-sum for the log-sum-exp of t, and the two P-weighted sums; the block
// combines them.  The work is two streams of reads, so exp and log use the MUFU
// intrinsics.
#include "common.cuh"
#include "launch.h"

namespace tam {
namespace {

constexpr int kKlThreads = 256;

struct KlParams {
    const float* mass;      // slab of P rows
    const float* score;     // slab of t rows
    int64_t row0;
    int n_rows;
    float* kl;              // [N], indexed by the absolute row
};

__global__ void __launch_bounds__(kKlThreads) k_row_kl(const KlParams p) {
    __shared__ float s_m[kKlThreads / 32], s_l[kKlThreads / 32], s_a[kKlThreads / 32];
    const int64_t i = p.row0 + (p.n_rows - 1 - (int)blockIdx.x);
    const int n = (int)i + 1;
    const int64_t off = (i * (i + 1) - p.row0 * (p.row0 + 1)) / 2;
    const float* P = p.mass + off;
    const float* t = p.score + off;
    float m = -INFINITY, l = 0.f, a = 0.f;   // max of t, sum exp(t - m), sum P (log P - t)
    for (int j = threadIdx.x; j < n; j += kKlThreads) {
        const float pj = __ldg(P + j), tj = __ldg(t + j);
        if (tj > m) {
            l = l * __expf(m - tj) + 1.f;
            m = tj;
        } else {
            l += __expf(tj - m);
        }
        if (pj > 0.f) a += pj * (__logf(pj) - tj);
    }
    // warp, then block combination of (m, l) and a
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
        a += __shfl_xor_sync(0xffffffffu, a, o);
        const float mm = fmaxf(m, m2);
        l = (mm == -INFINITY) ? 0.f : l * __expf(m - mm) + l2 * __expf(m2 - mm);
        m = mm;
    }
    if (lane == 0) {
        s_m[warp] = m;
        s_l[warp] = l;
        s_a[warp] = a;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float M = -INFINITY;
        for (int w = 0; w < kKlThreads / 32; ++w) M = fmaxf(M, s_m[w]);
        float L = 0.f, A = 0.f;
        for (int w = 0; w < kKlThreads / 32; ++w) {
            if (s_m[w] > -INFINITY) L += s_l[w] * __expf(s_m[w] - M);
            A += s_a[w];
        }
        p.kl[i] = A + M + __logf(L);
    }
}

}  // namespace

cudaError_t row_kl(const float* mass, const float* score, int64_t row0, int64_t row1, float* kl,
                   cudaStream_t st) {
    if (row1 <= row0) return cudaSuccess;
    KlParams p{mass, score, row0, (int)(row1 - row0), kl};
    k_row_kl<<<(unsigned)(row1 - row0), kKlThreads, 0, st>>>(p);
    note_launch();
    return cudaGetLastError();
}

}  // namespace tam
