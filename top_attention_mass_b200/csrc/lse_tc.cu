// Pass 1 on the tensor cores: per-head log-sum-exp of the causal scores.
//
//   lse[h, i] = log sum_{j <= i} exp(scale * q[i,h] . k[j,g(h)])
//
// (arXiv 2606.07703, Abstract and gist.science technical report §2.1: the dense
// attention distribution of every head, whose normaliser pass 2 needs before the
// head average can be taken.)
//
// One CTA owns one KV group g and one tile of 128/G queries: its G query heads
// are packed as 128 rows (row = query*G + head), so a single M=128 UMMA computes
// the scores of all heads that share K.  Roles:
//   warp 4      TMA producer: the Q tile once, then K tiles of 128 keys into a
//               2-stage ring (128-byte swizzle, K-major);
//   warp 5      one thread issues tcgen05.mma (M=128, N=128, K=16 steps) into one
//               of two TMEM accumulators (128 columns each) and commits to mbarriers;
//   warps 0-3   one thread per row: tcgen05.ld the 128 scores, causal mask on the
//               diagonal tile, online max / sum of 2^(scale*log2e*s - m).
// Tiles are issued heaviest first (last query tile first).
#include "launch.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace tam {
namespace {

constexpr int kStages = 2;
constexpr int kHalfBytes = 128 * 64 * 2;   // one 128-row x 64-element swizzle half
constexpr int kThreads = 192;

template <int D>
constexpr int lse_smem_bytes() {
    return 1024 + (D / 64) * kHalfBytes * (1 + kStages) + 256;
}

template <int G, int D>
__global__ void __launch_bounds__(kThreads, 2)
k_lse_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
         const __grid_constant__ SeqTable seqs, int Hq, int Hkv, float sl2,
         float* __restrict__ lse, int32_t* status, uint64_t timeout_ns, int dbg) {
    constexpr int BQ = 128 / G;
    constexpr int NH = D / 64;
    constexpr uint32_t kTileBytes = NH * kHalfBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sQ = base;
    uint8_t* sK = base + kTileBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sK + kStages * kTileBytes);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = k_full + kStages;
    uint64_t* s_full = k_empty + kStages;
    uint64_t* s_empty = s_full + 2;
    uint64_t* mma_done = s_empty + 2;
    uint64_t* never = mma_done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int sq, qt;
    seq_tile<BQ>(seqs, (int)(blockIdx.x / Hkv), sq, qt);
    const int g = (int)(blockIdx.x % Hkv);
    const int tok0 = seqs.cu[sq], N = seqs.cu[sq + 1] - tok0;   // this tile's sequence
    const int q0 = qt * BQ;                                     // positions within it
    const int q_last = min(N, q0 + BQ) - 1;
    const int n_kt = q_last / 128 + 1;

    if (threadIdx.x == 0) {
        tc::mbar_init(q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(&k_full[s], 1);
            tc::mbar_init(&k_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&s_full[b], 1);
            tc::mbar_init(&s_empty[b], 128);
        }
        tc::mbar_init(mma_done, 1);
        tc::mbar_init(never, 1);
        *abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 256);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const tc::Guard gd{abort_flag, status, KID_LSE_TC, timeout_ns};

    if (warp == 4) {
        if (lane == 0) {
            tc::prefetch_tmap(&tmQ);
            tc::prefetch_tmap(&tmK);
            tc::mbar_arrive_expect_tx(q_full, kTileBytes);
            for (int h = 0; h < NH; ++h) tc::tma_load_3d(sQ + h * kHalfBytes, &tmQ, q_full, h * 64, g * G, tok0 + q0);
            int issued = 0;
            for (int t = 0; t < n_kt; ++t) {
                const int s = t % kStages;
                const uint32_t ph = (t / kStages) & 1;
                if (!tc::wait(&k_empty[s], ph ^ 1, gd, 1)) break;
                tc::mbar_arrive_expect_tx(&k_full[s], kTileBytes);
                for (int h = 0; h < NH; ++h)
                    tc::tma_load_3d(sK + (s * NH + h) * kHalfBytes, &tmK, &k_full[s], h * 64, g,
                                    tok0 + t * 128);
                ++issued;
            }
            // let the last loads of every stage land before the CTA may exit
            int zero = 0;
            const tc::Guard drain_noabort{&zero, nullptr, KID_LSE_TC, timeout_ns};
            for (int t = max(0, issued - kStages); t < issued; ++t)
                tc::wait(&k_full[t % kStages], (t / kStages) & 1, drain_noabort, 0);
            tc::wait(q_full, 0, drain_noabort, 0);
        }
    } else if (warp == 5) {
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_bf16_f32(128, 128);
            bool ok = tc::wait(q_full, 0, gd, 2);
            const uint32_t aq = tc::smem_u32(sQ);
            for (int t = 0; ok && t < n_kt; ++t) {
                const int s = t % kStages;
                const uint32_t ph = (t / kStages) & 1;
                const int b = t & 1;
                const uint32_t bph = (t >> 1) & 1;
                if (!tc::wait(&k_full[s], ph, gd, 3)) break;
                if (!tc::wait(&s_empty[b], bph ^ 1, gd, 4)) break;
                tc::fence_after_sync();
                const uint32_t ak = tc::smem_u32(sK + s * kTileBytes);
#pragma unroll
                for (int kk = 0; kk < NH * 4; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                    tc::mma_bf16_ss(tmem + b * 128, tc::desc_kmajor_sw128(aq + off),
                                    tc::desc_kmajor_sw128(ak + off), idesc, kk > 0 ? 1u : 0u);
                }
                tc::mma_commit(&k_empty[s]);
                tc::mma_commit(&s_full[b]);
            }
            tc::mma_commit(mma_done);
            int zero = 0;
            const tc::Guard drain{&zero, nullptr, KID_LSE_TC, timeout_ns};
            tc::wait(mma_done, 0, drain, 0);
        }
    } else {
        // softmax warps 0..3: thread = TMEM lane = row (query*G + head)
        const int r = threadIdx.x;
        const int i = q0 + r / G;
        const int h = g * G + r % G;
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        if (dbg & kDebugForceTimeout) ok = tc::wait(never, 0, gd, 9);
        for (int t = 0; ok && t < n_kt; ++t) {
            const int b = t & 1;
            const uint32_t bph = (t >> 1) & 1;
            if (!tc::wait(&s_full[b], bph, gd, 5)) { ok = false; break; }
            tc::fence_after_sync();
            uint32_t v[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tc::tmem_ld32(lane_addr + b * 128 + c * 32, v[c]);
#pragma unroll
            for (int c = 0; c < 4; ++c) tc::tmem_wait_ld(v[c]);
            tc::fence_before_sync();
            tc::mbar_arrive(&s_empty[b]);
            const int j0 = t * 128;
            const bool diag = (j0 + 127 > q0);
            if (diag) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (j0 + c * 32 + e > i) v[c][e] = __float_as_uint(-INFINITY);
            }
            // row max: two independent chains of 3-input max
            float tm[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    tm[c & 1] = tc::max3(tm[c & 1], __uint_as_float(v[c][e]),
                                         __uint_as_float(v[c][e + 1]));
            const float m_new = fmaxf(m, fmaxf(tm[0], tm[1]) * sl2);
            const float neg = -m_new;
            // exponentials of column pairs: packed scale-and-shift, packed sums in two chains
            const uint64_t sl2x2 = tc::f2_pack(sl2, sl2), negx2 = tc::f2_pack(neg, neg);
            uint64_t sum2[2] = {0ull, 0ull};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const uint64_t x2 = tc::f2_fma(tc::f2_pack(__uint_as_float(v[c][e]),
                                                               __uint_as_float(v[c][e + 1])),
                                                   sl2x2, negx2);
                    float x0, x1, y0, y1;
                    tc::f2_unpack(x2, x0, x1);
                    // one pair in four on the FMA pipe (packed polynomial), the rest on MUFU
                    if ((e & 7) == 6) {
                        tc::ex2_fma2(x0, x1, y0, y1);
                    } else {
                        y0 = tc::ex2(x0);
                        y1 = tc::ex2(x1);
                    }
                    sum2[c & 1] = tc::f2_add(sum2[c & 1], tc::f2_pack(y0, y1));
                }
            }
            float s0, s1, s2, s3;
            tc::f2_unpack(sum2[0], s0, s1);
            tc::f2_unpack(sum2[1], s2, s3);
            l = l * tc::ex2(m - m_new) + ((s0 + s1) + (s2 + s3));
            m = m_new;
        }
        if (ok && i < N && !*abort_flag)
            lse[(size_t)Hq * tok0 + (size_t)h * N + i] = (m + __log2f(l)) * kLn2;
    }
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 256);
    }
}

template <int G, int D>
cudaError_t launch_lse_tc(const LseArgs& a, cudaStream_t st) {
    constexpr int BQ = 128 / G;
    CUtensorMap tq, tk;
    const uint64_t d = a.d;
    if (!make_tmap_3d_bf16(&tq, a.q, d, a.Hq, a.N, d * 2, (uint64_t)a.Hq * d * 2, 64, G, BQ) ||
        !make_tmap_3d_bf16(&tk, a.k, d, a.Hkv, a.N, d * 2, (uint64_t)a.Hkv * d * 2, 64, 1, 128))
        return cudaErrorInvalidValue;
    constexpr int smem = lse_smem_bytes<D>();
    auto kern = k_lse_tc<G, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return with_table(a.N, a.seqs, [&](SeqTable& t) {
        const int n_tiles = seq_table_tiles(t, BQ);
        if (n_tiles == 0) return cudaSuccess;
        kern<<<(unsigned)(n_tiles * a.Hkv), kThreads, smem, st>>>(
            tq, tk, t, a.Hq, a.Hkv, a.sl2, a.lse, a.status, wait_timeout_ns(), debug_flags());
        note_launch();
        return cudaGetLastError();
    });
}

template <int D>
cudaError_t dispatch_g(const LseArgs& a, cudaStream_t st) {
    switch (a.Hq / a.Hkv) {
        case 1: return launch_lse_tc<1, D>(a, st);
        case 2: return launch_lse_tc<2, D>(a, st);
        case 4: return launch_lse_tc<4, D>(a, st);
        case 8: return launch_lse_tc<8, D>(a, st);
        case 16: return launch_lse_tc<16, D>(a, st);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace

bool tc_lse_supported(const LseArgs& a) {
    const int G = a.Hq / a.Hkv;
    return a.dtype == TAM_BF16 && (a.d == 64 || a.d == 128 || a.d == 256) &&
           (G == 1 || G == 2 || G == 4 || G == 8 || G == 16);
}

cudaError_t tc_lse(const LseArgs& a, cudaStream_t st) {
    switch (a.d) {
        case 64: return dispatch_g<64>(a, st);
        case 128: return dispatch_g<128>(a, st);
        default: return dispatch_g<256>(a, st);
    }
}

}  // namespace tam
