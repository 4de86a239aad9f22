// Dense causal GQA prefill on the tensor cores (the comparator of the sparse pass).
//
//   out[i,h] = softmax_{j <= i}(scale * q[i,h].k[j,g(h)]) v[j,g(h)],  lse optional
//
// (arXiv 2606.07703, Abstract: sparse serving is measured against a dense
// FlashAttention-2 baseline; this is that baseline written for sm_100a.)
//
// One CTA owns one KV group g and 128/G queries: the G query heads are packed as
// the 128 UMMA rows (row = query*G + head).  Per key tile of 128:
//   S = Q K^T           tcgen05.mma into one of two TMEM score buffers;
//   softmax warps       tcgen05.ld their row, causal mask, exp2 against a lazily
//                       raised row max (O is rescaled in TMEM only when the max grew
//                       by more than 2^8), P written as bf16 into a 128-byte-swizzled
//                       shared tile (K-major A operand) and fenced to the async proxy;
//   O += P V            tcgen05.mma with V as an MN-major B operand; O stays in TMEM.
// Roles: warps 0-3 softmax (thread = row), warp 4 TMA producer (Q once; K and V in
// separate 2-stage rings so K for tile t+2 loads as soon as S of tile t is done),
// warp 5 MMA issuer (issues S of tile t+1 before P V of tile t).
#include "launch.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace tam {
namespace {

constexpr int kHalf = 128 * 64 * 2;     // one 128-row x 64-element swizzled half
constexpr int kThreads = 192;
constexpr float kRescaleLog2 = 8.f;     // lazy rescale threshold (factor 256)

// K and V ring depth: two tiles each, one at d = 256 (a 256-wide tile is 64 KB)
template <int D>
constexpr int dense_stages() { return D == 256 ? 1 : 2; }

template <int D>
constexpr int dense_smem_bytes() {
    // Q + K ring + V ring + P + barriers
    return 1024 + (D / 64) * kHalf * (1 + 2 * dense_stages<D>()) + 2 * kHalf + 512;
}

template <int G, int D>
__global__ void __launch_bounds__(kThreads, 1)
k_dense_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ SeqTable seqs, int Hq,
           int Hkv, float sl2, __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
           int32_t* status, uint64_t timeout_ns) {
    constexpr int BQ = 128 / G;
    constexpr int kStages = dense_stages<D>();
    constexpr int NH = D / 64;
    constexpr uint32_t kTile = NH * kHalf;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sQ = base;
    uint8_t* sK = sQ + kTile;
    uint8_t* sV = sK + kStages * kTile;
    uint8_t* sP = sV + kStages * kTile;                 // 2 halves of 64 keys
    uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * kHalf);
    uint64_t* q_full = bars;
    uint64_t* k_full = q_full + 1;
    uint64_t* k_empty = k_full + kStages;
    uint64_t* v_full = k_empty + kStages;
    uint64_t* v_empty = v_full + kStages;
    uint64_t* s_full = v_empty + kStages;
    uint64_t* s_empty = s_full + 2;
    uint64_t* p_full = s_empty + 2;
    uint64_t* o_done = p_full + 1;
    uint64_t* mma_done = o_done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
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
            tc::mbar_init(&v_full[s], 1);
            tc::mbar_init(&v_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&s_full[b], 1);
            tc::mbar_init(&s_empty[b], 128);
        }
        tc::mbar_init(p_full, 128);
        tc::mbar_init(o_done, 1);
        tc::mbar_init(mma_done, 1);
        *abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_o = tmem + 256;           // O accumulator: columns 256..256+D
    const tc::Guard gd{abort_flag, status, KID_DENSE_TC, timeout_ns};

    if (warp == 4) {
        if (lane == 0) {
            tc::prefetch_tmap(&tmQ);
            tc::prefetch_tmap(&tmK);
            tc::prefetch_tmap(&tmV);
            tc::mbar_arrive_expect_tx(q_full, kTile);
            for (int h = 0; h < NH; ++h) tc::tma_load_3d(sQ + h * kHalf, &tmQ, q_full, h * 64, g * G, tok0 + q0);
            // K runs up to kStages tiles ahead of S; V up to kStages tiles ahead of P V.
            int nk = 0, nv = 0;
            bool ok = true;
            while (ok && (nk < n_kt || nv < n_kt)) {
                if (nk < n_kt && (nk <= nv || nv == n_kt)) {
                    const int s = nk % kStages;
                    if (!tc::wait(&k_empty[s], ((nk / kStages) & 1) ^ 1, gd, 1)) { ok = false; break; }
                    tc::mbar_arrive_expect_tx(&k_full[s], kTile);
                    for (int h = 0; h < NH; ++h)
                        tc::tma_load_3d(sK + s * kTile + h * kHalf, &tmK, &k_full[s], h * 64, g, tok0 + nk * 128);
                    ++nk;
                } else {
                    const int s = nv % kStages;
                    if (!tc::wait(&v_empty[s], ((nv / kStages) & 1) ^ 1, gd, 2)) { ok = false; break; }
                    tc::mbar_arrive_expect_tx(&v_full[s], kTile);
                    for (int h = 0; h < NH; ++h)
                        tc::tma_load_3d(sV + s * kTile + h * kHalf, &tmV, &v_full[s], h * 64, g, tok0 + nv * 128);
                    ++nv;
                }
            }
            int zero = 0;
            const tc::Guard drain{&zero, nullptr, 0, timeout_ns};
            for (int t = max(0, nk - kStages); t < nk; ++t) tc::wait(&k_full[t % kStages], (t / kStages) & 1, drain, 0);
            for (int t = max(0, nv - kStages); t < nv; ++t) tc::wait(&v_full[t % kStages], (t / kStages) & 1, drain, 0);
            tc::wait(q_full, 0, drain, 0);
        }
    } else if (warp == 5) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, 128);
            constexpr uint32_t idesc_o = tc::idesc_bf16_f32(128, D, false, true);
            const uint32_t aq = tc::smem_u32(sQ);
            const uint32_t ap = tc::smem_u32(sP);
            bool ok = tc::wait(q_full, 0, gd, 3);
            auto issue_s = [&](int t) -> bool {
                const int s = t % kStages, b = t & 1;
                if (!tc::wait(&k_full[s], (t / kStages) & 1, gd, 4)) return false;
                if (!tc::wait(&s_empty[b], ((t >> 1) & 1) ^ 1, gd, 5)) return false;
                tc::fence_after_sync();
                const uint32_t ak = tc::smem_u32(sK + s * kTile);
#pragma unroll
                for (int kk = 0; kk < NH * 4; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
                    tc::mma_bf16_ss(tmem + b * 128, tc::desc_kmajor_sw128(aq + off),
                                    tc::desc_kmajor_sw128(ak + off), idesc_s, kk > 0 ? 1u : 0u);
                }
                tc::mma_commit(&k_empty[s]);
                tc::mma_commit(&s_full[b]);
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int t = 0; ok && t < n_kt; ++t) {
                if (t + 1 < n_kt && !issue_s(t + 1)) break;
                const int s = t % kStages;
                if (!tc::wait(&v_full[s], (t / kStages) & 1, gd, 6)) break;
                if (!tc::wait(p_full, t & 1, gd, 7)) break;
                tc::fence_after_sync();
                const uint32_t av = tc::smem_u32(sV + s * kTile);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {   // 128 keys in steps of 16
                    const uint32_t offp = (kk >> 2) * kHalf + (kk & 3) * 32;
                    tc::mma_bf16_ss(tmem_o, tc::desc_kmajor_sw128(ap + offp),
                                    tc::desc_mnmajor_sw128(av + kk * 16 * 128, kHalf), idesc_o,
                                    (t > 0 || kk > 0) ? 1u : 0u);
                }
                tc::mma_commit(&v_empty[s]);
                tc::mma_commit(o_done);
            }
            tc::mma_commit(mma_done);
            int zero = 0;
            const tc::Guard drain{&zero, nullptr, 0, timeout_ns};
            tc::wait(mma_done, 0, drain, 0);
        }
    } else {
        // softmax warps: thread = row (query*G + head) = TMEM lane
        const int r = threadIdx.x;
        const int i = q0 + r / G;
        const int h = g * G + r % G;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        uint8_t* prow0 = sP + r * 128;               // row r of half 0
        for (int t = 0; ok && t < n_kt; ++t) {
            const int b = t & 1;
            if (!tc::wait(&s_full[b], (t >> 1) & 1, gd, 8)) { ok = false; break; }
            tc::fence_after_sync();
            uint32_t v[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tc::tmem_ld32(tmem + lane_off + b * 128 + c * 32, v[c]);
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
            // row max of the raw scores: two chains of 3-input max
            float tm[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    tm[c & 1] = tc::max3(tm[c & 1], __uint_as_float(v[c][e]),
                                         __uint_as_float(v[c][e + 1]));
            const float tmax = fmaxf(tm[0], tm[1]) * sl2;
            const bool raise = tmax > m_used + kRescaleLog2;
            const float m_new = raise ? tmax : m_used;
            const float corr = tc::ex2(m_used - m_new);     // 0 on the first tile
            const uint64_t sl2x2 = tc::f2_pack(sl2, sl2), negm2 = tc::f2_pack(-m_new, -m_new);
            uint64_t sum2[2] = {0ull, 0ull};
            // P in bf16, row r of the swizzled tile (16-byte chunks XOR row%8); column
            // pairs: packed scale-and-shift and sums, one pair in four on the FMA pipe
#pragma unroll
            for (int c8 = 0; c8 < 16; ++c8) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int col = c8 * 8 + 2 * e;
                    const uint64_t x2 = tc::f2_fma(
                        tc::f2_pack(__uint_as_float(v[col / 32][col % 32]),
                                    __uint_as_float(v[(col + 1) / 32][(col + 1) % 32])),
                        sl2x2, negm2);
                    float x0, x1, p0, p1;
                    tc::f2_unpack(x2, x0, x1);
                    if (e == 3) {
                        tc::ex2_fma2(x0, x1, p0, p1);
                    } else {
                        p0 = tc::ex2(x0);
                        p1 = tc::ex2(x1);
                    }
                    sum2[e & 1] = tc::f2_add(sum2[e & 1], tc::f2_pack(p0, p1));
                    __nv_bfloat162 pk = __floats2bfloat162_rn(p0, p1);
                    w[e] = *reinterpret_cast<uint32_t*>(&pk);
                }
                const int half = c8 >> 3, chunk = c8 & 7;
                // P V of tile t-1 must have finished reading the P tile before it is
                // overwritten (single P buffer); wait once, before the first store.
                if (c8 == 0 && t > 0) {
                    if (!tc::wait(o_done, (t - 1) & 1, gd, 9)) { ok = false; break; }
                }
                uint4* dst = reinterpret_cast<uint4*>(prow0 + half * kHalf + ((chunk ^ (r & 7)) << 4));
                *dst = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (!ok) break;
            float s0, s1, s2, s3;
            tc::f2_unpack(sum2[0], s0, s1);
            tc::f2_unpack(sum2[1], s2, s3);
            l = l * corr + ((s0 + s1) + (s2 + s3));
            // rescale O in TMEM when this warp's rows raised their max (after P V t-1)
            const bool any_raise = __any_sync(0xffffffffu, raise && t > 0);
            if (any_raise) {
                tc::fence_after_sync();
                const float f = (raise && t > 0) ? corr : 1.f;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tc::tmem_ld32(tmem_o + lane_off + c * 32, o);
                    tc::tmem_wait_ld(o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
                    tc::tmem_st32(tmem_o + lane_off + c * 32, o);
                }
                tc::tmem_wait_st();
            }
            m_used = m_new;
            tc::fence_proxy_async_smem();
            tc::fence_before_sync();
            tc::mbar_arrive(p_full);
        }
        // epilogue: wait for the last P V, normalise, store bf16 rows
        if (ok && tc::wait(o_done, (n_kt - 1) & 1, gd, 10)) {
            tc::fence_after_sync();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16* orow = out + ((size_t)(tok0 + i) * Hq + h) * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tc::tmem_ld32(tmem_o + lane_off + c * 32, o);
                tc::tmem_wait_ld(o);
                if (i < N) {
#pragma unroll
                    for (int e8 = 0; e8 < 4; ++e8) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            __nv_bfloat162 pk = __floats2bfloat162_rn(
                                __uint_as_float(o[e8 * 8 + 2 * e]) * inv,
                                __uint_as_float(o[e8 * 8 + 2 * e + 1]) * inv);
                            w[e] = *reinterpret_cast<uint32_t*>(&pk);
                        }
                        *reinterpret_cast<uint4*>(orow + c * 32 + e8 * 8) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
            if (lse && i < N) lse[(size_t)Hq * tok0 + (size_t)h * N + i] = (m_used + __log2f(l)) * kLn2;
        }
    }
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

template <int G, int D>
cudaError_t launch_dense(const AttnArgs& a, cudaStream_t st) {
    constexpr int BQ = 128 / G;
    CUtensorMap tq, tk, tv;
    const uint64_t d = a.d;
    if (!make_tmap_3d_bf16(&tq, a.q, d, a.Hq, a.N, d * 2, (uint64_t)a.Hq * d * 2, 64, G, BQ) ||
        !make_tmap_3d_bf16(&tk, a.k, d, a.Hkv, a.N, d * 2, (uint64_t)a.Hkv * d * 2, 64, 1, 128) ||
        !make_tmap_3d_bf16(&tv, a.v, d, a.Hkv, a.N, d * 2, (uint64_t)a.Hkv * d * 2, 64, 1, 128))
        return cudaErrorInvalidValue;
    constexpr int smem = dense_smem_bytes<D>();
    static_assert(smem <= 227 * 1024, "dense tile layout exceeds shared memory");
    auto kern = k_dense_tc<G, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return with_table(a.N, a.seqs, [&](SeqTable& t) {
        const int n_tiles = seq_table_tiles(t, BQ);
        if (n_tiles == 0) return cudaSuccess;
        kern<<<(unsigned)(n_tiles * a.Hkv), kThreads, smem, st>>>(
            tq, tk, tv, t, a.Hq, a.Hkv, a.sl2, (__nv_bfloat16*)a.out, a.lse, a.status,
            wait_timeout_ns());
        note_launch();
        return cudaGetLastError();
    });
}

template <int D>
cudaError_t dispatch_g(const AttnArgs& a, cudaStream_t st) {
    switch (a.Hq / a.Hkv) {
        case 1: return launch_dense<1, D>(a, st);
        case 2: return launch_dense<2, D>(a, st);
        case 4: return launch_dense<4, D>(a, st);
        case 8: return launch_dense<8, D>(a, st);
        case 16: return launch_dense<16, D>(a, st);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace

bool tc_dense_supported(const AttnArgs& a) {
    const int G = a.Hq / a.Hkv;
    return a.dtype == TAM_BF16 && (a.d == 64 || a.d == 128 || a.d == 256) &&
           (G == 1 || G == 2 || G == 4 || G == 8 || G == 16);
}

cudaError_t tc_dense(const AttnArgs& a, cudaStream_t st) {
    switch (a.d) {
        case 64: return dispatch_g<64>(a, st);
        case 128: return dispatch_g<128>(a, st);
        default: return dispatch_g<256>(a, st);
    }
}

}  // namespace tam
