// Block-shared pass 3 on the tensor cores: attention recomputed on a block's support.
//
//   out[i,h] = sum_{j in T_i} softmax_{T_i}(scale * q[i,h].k[j,g(h)]) v[j,g(h)],
//   T_i = S_b intersected with [0, i], b = i / block_q
//
// (arXiv 2606.07703, Abstract: "recomputes attention only on that support";
// gist.science technical report §2.1 "Ausführung" and "Granularität": the support is
// selected once for a block of consecutive queries.)
//
// The flash-style pipeline of the dense kernel over gathered keys.  One CTA owns one
// KV group g and TT tiles of 128/G queries of block b (TT = 2 when the block has an
// even number of tiles; the G query heads packed as the 128 UMMA rows of a tile,
// row = query*G + head); its keys are the entries of S_b up to its last query, in
// chunks of 64 in a four-stage ring, gathered once for all of its tiles:
//   gather warps        cp.async the K and V rows of the chunk (whole rows per warp
//                       instruction, zero-filled past the support) into 128-byte-swizzled shared
//                       tiles laid out as a TMA tile load would leave them, stage the
//                       key indices for the mask; a chunk is signalled (fence to the async
//                       proxy, arrive) once the copies of the two chunks after it are in
//                       flight, so three chunks of rows travel at once;
//   TMA warp            the Q tiles (once);
//   MMA warp            per chunk, S = Q K^T of every tile into one of its two TMEM
//                       buffers, then O += P V per tile, S of chunk t+1 issued before
//                       P V of chunk t;
//   softmax warpgroups  one per tile (warps 4tt..4tt+3), thread = row: mask (key not in
//                       [0, i] or past the support), lazy online softmax in exp2 as in
//                       the dense kernel, P as bf16 into the tile's swizzled shared
//                       tile; rows with no key get a zero output row and lse = -inf.
// With two tiles the softmax of one overlaps the MMAs of the other, and every gathered
// key row serves twice the queries.
#include "launch.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace tam {
namespace {

constexpr int kKeys = 64;                   // keys per chunk
constexpr int kHalf = 128 * 64 * 2;         // one 128-row x 64-element swizzled half (Q, P)
constexpr int kHalfKV = kKeys * 64 * 2;     // one 64-key x 64-element swizzled half (K, V)
// K/V ring depth and gather lag (chunks in flight behind the one being signalled): four
// and two; at d = 256, where one chunk of K and V is 64 KB, two and none.
template <int D>
__host__ __device__ constexpr int kv_stages() { return D == 256 ? 2 : 4; }
template <int D>
__host__ __device__ constexpr int gather_lag() { return D == 256 ? 0 : 2; }
constexpr int kGatherThreads = 64;          // two gather warps
constexpr float kRescaleLog2 = 8.f;

// TT softmax warpgroups, then the TMA warp, the MMA warp and the two gather warps.
__host__ __device__ constexpr int block_threads(int TT) { return 32 * (4 * TT + 4); }

template <int D, int TT>
constexpr int block_tc_smem_bytes() {
    // slack + Q tiles + K ring + V ring + P tiles + staged key indices + barriers
    return 1024 + (D / 64) * (TT * kHalf + 2 * kv_stages<D>() * kHalfKV) + TT * kHalf +
           kv_stages<D>() * kKeys * 4 + 256;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    const int n = valid ? 16 : 0;           // n = 0 writes 16 zero bytes
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

struct BlockTcParams {
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    int N, Hq, Hkv, tiles_per_block, n_ctas_per_group;
    int block_q, kmax;
    float sl2;
    const int32_t* sup_idx;
    const int32_t* sup_len;
    __nv_bfloat16* out;
    float* lse;
    int32_t* status;
    uint64_t timeout_ns;
};

// DENSE: the same pipeline over every key 0..q_last (the dense comparator): the TMA
// warp also streams the K and V chunks (tmK, tmV with 64-row boxes) and the mask is the
// causal one; the gather warps stay idle.
template <int G, int D, int TT, bool DENSE>
__global__ void __launch_bounds__(block_threads(TT), 1)
k_attn_block_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const BlockTcParams p) {
    constexpr int kThreads = block_threads(TT);
    constexpr int kStages = kv_stages<D>(), kLag = gather_lag<D>();
    static_assert(kLag < kStages - 1, "the gather may run at most kStages - 2 chunks ahead");
    static_assert(256 + 128 * (TT - 1) + D <= 512, "TMEM columns: O of tile tt at 256 + 128 tt");
    constexpr int kTmaWarp = 4 * TT, kMmaWarp = 4 * TT + 1, kGatherWarp0 = 4 * TT + 2;
    constexpr int BQ = 128 / G;
    constexpr int NH = D / 64;
    constexpr uint32_t kTile = NH * kHalf;        // Q of one tile
    constexpr uint32_t kTileKV = NH * kHalfKV;    // one chunk of K (or V)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sQ = base;                                 // TT tiles
    uint8_t* sK = sQ + TT * kTile;
    uint8_t* sV = sK + kStages * kTileKV;
    uint8_t* sP = sV + kStages * kTileKV;               // TT tiles of 128 rows x 64 keys
    int32_t* sIdx = reinterpret_cast<int32_t*>(sP + TT * kHalf);   // kStages x kKeys
    uint64_t* bars = reinterpret_cast<uint64_t*>(sIdx + kStages * kKeys);
    uint64_t* q_full = bars;
    uint64_t* kv_full = q_full + 1;
    uint64_t* kv_empty = kv_full + kStages;
    uint64_t* s_full = kv_empty + kStages;              // [tile][buffer]
    uint64_t* s_empty = s_full + 2 * TT;                // [tile][buffer]
    uint64_t* p_full = s_empty + 2 * TT;                // [tile]
    uint64_t* o_done = p_full + TT;                     // [tile]
    uint64_t* mma_done = o_done + TT;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = (int)(blockIdx.x % p.Hkv);
    // the CTA's TT consecutive tiles (within one block: tiles_per_block % TT == 0)
    const int tile0 = (p.n_ctas_per_group - 1 - (int)(blockIdx.x / p.Hkv)) * TT;  // later first
    const int b = tile0 / p.tiles_per_block;
    const int q0 = b * p.block_q + (tile0 % p.tiles_per_block) * BQ;
    if (q0 >= p.N) return;                                          // uniform for the CTA
    const int q_last = min(p.N, q0 + TT * BQ) - 1;
    const int32_t* srow = p.sup_idx + (size_t)b * p.kmax;
    // n_t = 1 + the last position of the (ascending) support row holding a key <= q_last:
    // one round of independent loads across the CTA and a max-reduction, instead of a
    // chain of dependent loads; the first chunk's indices are staged on the way.
    __shared__ int s_last[kThreads / 32];
    if (DENSE) {
        if (threadIdx.x < kThreads / 32) s_last[threadIdx.x] = q_last + 1;
    } else {
        const int len = min(p.sup_len[b], p.kmax);
        int last = 0;
#pragma unroll 4
        for (int c = threadIdx.x; c < len; c += kThreads) {
            const int j = srow[c];
            if (j <= q_last) last = c + 1;
            if (c < kKeys) sIdx[c] = j;
        }
        if (threadIdx.x < kKeys && (int)threadIdx.x >= len) sIdx[threadIdx.x] = -1;
        last = __reduce_max_sync(0xffffffffu, last);
        if (lane == 0) s_last[warp] = last;
    }
    __syncthreads();
    int n_t = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) n_t = max(n_t, s_last[w]);
    const int n_ch = (n_t + kKeys - 1) / kKeys;

    if (n_ch == 0) {
        // no support key at or before any query of the tiles: zero rows, lse = -inf
        if (threadIdx.x < 128 * TT) {
            const int r = threadIdx.x % 128, tt = threadIdx.x / 128;
            const int i = q0 + tt * BQ + r / G, h = g * G + r % G;
            if (i < p.N) {
                __nv_bfloat16* orow = p.out + ((size_t)i * p.Hq + h) * D;
                for (int c = 0; c < D; ++c) orow[c] = __float2bfloat16_rn(0.f);
                if (p.lse) p.lse[(size_t)h * p.N + i] = -INFINITY;
            }
        }
        return;
    }

    if (threadIdx.x == 0) {
        tc::mbar_init(q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(&kv_full[s], DENSE ? 1 : kGatherThreads);   // TMA, or every gather thread
            tc::mbar_init(&kv_empty[s], 1);
        }
        for (int x = 0; x < 2 * TT; ++x) {
            tc::mbar_init(&s_full[x], 1);
            tc::mbar_init(&s_empty[x], 128);
        }
        for (int tt = 0; tt < TT; ++tt) {
            tc::mbar_init(&p_full[tt], 128);
            tc::mbar_init(&o_done[tt], 1);
        }
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
    // tile tt: S buffers at columns 128 tt + {0, 64}, O accumulator at 256 + 128 tt
    const tc::Guard gd{abort_flag, p.status, DENSE ? KID_DENSE_TC : KID_BLOCK_ATTN, p.timeout_ns};

    if (warp >= kGatherWarp0) {
      if constexpr (!DENSE) {
        // ---------------------------------------------------------------- gather
        // Warp gw copies key rows [64 gw, 64 gw + 64) of each chunk.  Lane l owns the
        // indices of rows 64 gw + l and 64 gw + 32 + l; the copies go row-contiguous:
        // PR lanes share one row (lane % PR = its 16-byte piece), so one warp
        // instruction moves 32 / PR whole rows with every sector fully used.
        const int gw = warp - kGatherWarp0;
        constexpr int PR = D / 8;                          // 16-byte pieces per row
        constexpr int RPI = 32 / PR;                       // rows per warp instruction
        constexpr int RPW = kKeys / (kGatherThreads / 32); // rows per gather warp
        constexpr int RR = RPW / 32;                       // index registers per lane
        static_assert(RR * 32 == RPW && RPI * PR == 32, "gather tiling");
        const int piece = lane % PR, sub = lane / PR;
        const uint32_t half_off = (uint32_t)(piece / 8) * kHalfKV;
        const int pc = piece % 8;
        const __nv_bfloat16* kbase = p.k + (size_t)g * D + piece * 8;
        const __nv_bfloat16* vbase = p.v + (size_t)g * D + piece * 8;
        const size_t row_stride = (size_t)p.Hkv * D;
        int jn[RR];                                        // indices of the next chunk
#pragma unroll
        for (int rr = 0; rr < RR; ++rr) {
            const int r = gw * RPW + rr * 32 + lane;
            jn[rr] = r < n_t ? sIdx[r] : -1;              // chunk 0, staged above
        }
        int signalled = 0;                                  // chunks announced so far
        for (int t = 0; t < n_ch; ++t) {
            const int s = t % kStages;
            if (!tc::wait(&kv_empty[s], ((t / kStages) & 1) ^ 1, gd, 1)) break;
            const uint32_t dk = tc::smem_u32(sK + s * kTileKV), dv = tc::smem_u32(sV + s * kTileKV);
            int js[RR];
#pragma unroll
            for (int rr = 0; rr < RR; ++rr) {
                const int j = jn[rr];
                js[rr] = (j >= 0 && j < p.N) ? j : -1;
                sIdx[s * kKeys + gw * RPW + rr * 32 + lane] = js[rr];
                // the next chunk's indices load while this chunk's rows are in flight
                const int c = (t + 1) * kKeys + gw * RPW + rr * 32 + lane;
                jn[rr] = c < n_t ? srow[c] : -1;
            }
#pragma unroll
            for (int it = 0; it < RPW / RPI; ++it) {
                const int rl = it * RPI + sub;             // row within the warp's share
                const int j = __shfl_sync(0xffffffffu, js[(it * RPI) >> 5], rl & 31);
                const int r = gw * RPW + rl;
                const bool valid = j >= 0;
                const size_t off = valid ? (size_t)j * row_stride : 0;
                const uint32_t o = half_off + r * 128 + ((pc ^ (r & 7)) << 4);
                cp_async16(dk + o, kbase + off, valid);
                cp_async16(dv + o, vbase + off, valid);
            }
            cp_async_commit();
            // chunk t - kLag has landed once at most kLag newer groups are pending:
            // make it visible to the tensor core and signal it
            if (t >= kLag) {
                cp_async_wait<kLag>();
                tc::fence_proxy_async_smem();
                tc::mbar_arrive(&kv_full[(t - kLag) % kStages]);
                signalled = t - kLag + 1;
            }
        }
        cp_async_wait<0>();
        tc::fence_proxy_async_smem();
        // the last chunks (every chunk issued, or stopped early: whatever was issued)
        for (int t = signalled; t < n_ch; ++t) {
            if (*abort_flag) break;
            tc::mbar_arrive(&kv_full[t % kStages]);
        }
      }
    } else if (warp == kTmaWarp) {
        // ---------------------------------------------------------------- Q (TMA)
        if (lane == 0) {
            tc::prefetch_tmap(&tmQ);
            tc::mbar_arrive_expect_tx(q_full, TT * kTile);
            for (int tt = 0; tt < TT; ++tt)
                for (int h = 0; h < NH; ++h)
                    tc::tma_load_3d(sQ + tt * kTile + h * kHalf, &tmQ, q_full, h * 64, g * G,
                                    q0 + tt * BQ);
            if (DENSE) {
                // K and V chunks of keys 64 t .. 64 t + 63 (past N the box reads zeros,
                // and the causal mask drops those keys)
                tc::prefetch_tmap(&tmK);
                tc::prefetch_tmap(&tmV);
                int issued = 0;
                for (int t = 0; t < n_ch; ++t) {
                    const int s = t % kStages;
                    if (!tc::wait(&kv_empty[s], ((t / kStages) & 1) ^ 1, gd, 1)) break;
                    tc::mbar_arrive_expect_tx(&kv_full[s], 2 * kTileKV);
                    for (int h = 0; h < NH; ++h) {
                        tc::tma_load_3d(sK + s * kTileKV + h * kHalfKV, &tmK, &kv_full[s], h * 64, g,
                                        t * kKeys);
                        tc::tma_load_3d(sV + s * kTileKV + h * kHalfKV, &tmV, &kv_full[s], h * 64, g,
                                        t * kKeys);
                    }
                    issued = t + 1;
                }
                int zero0 = 0;
                const tc::Guard drain0{&zero0, nullptr, 0, p.timeout_ns};
                for (int t = max(0, issued - kStages); t < issued; ++t)
                    tc::wait(&kv_full[t % kStages], (t / kStages) & 1, drain0, 0);
            }
            int zero = 0;
            const tc::Guard drain{&zero, nullptr, 0, p.timeout_ns};
            tc::wait(q_full, 0, drain, 0);
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, kKeys);
            constexpr uint32_t idesc_o = tc::idesc_bf16_f32(128, D, false, true);
            const uint32_t aq = tc::smem_u32(sQ);
            const uint32_t ap = tc::smem_u32(sP);
            bool ok = tc::wait(q_full, 0, gd, 3);
            auto issue_s = [&](int t) -> bool {
                const int s = t % kStages, bb = t & 1;
                if (!tc::wait(&kv_full[s], (t / kStages) & 1, gd, 4)) return false;
                for (int tt = 0; tt < TT; ++tt)
                    if (!tc::wait(&s_empty[tt * 2 + bb], ((t >> 1) & 1) ^ 1, gd, 5)) return false;
                tc::fence_after_sync();
                const uint32_t ak = tc::smem_u32(sK + s * kTileKV);
#pragma unroll
                for (int tt = 0; tt < TT; ++tt) {
#pragma unroll
                    for (int kk = 0; kk < NH * 4; ++kk) {
                        const uint32_t offq = tt * kTile + (kk >> 2) * kHalf + (kk & 3) * 32;
                        const uint32_t offk = (kk >> 2) * kHalfKV + (kk & 3) * 32;
                        tc::mma_bf16_ss(tmem + tt * 128 + bb * kKeys, tc::desc_kmajor_sw128(aq + offq),
                                        tc::desc_kmajor_sw128(ak + offk), idesc_s, kk > 0 ? 1u : 0u);
                    }
                    tc::mma_commit(&s_full[tt * 2 + bb]);
                }
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int t = 0; ok && t < n_ch; ++t) {
                if (t + 1 < n_ch && !issue_s(t + 1)) break;
                const int s = t % kStages;
                const uint32_t av = tc::smem_u32(sV + s * kTileKV);
                for (int tt = 0; ok && tt < TT; ++tt) {
                    if (!tc::wait(&p_full[tt], t & 1, gd, 7)) { ok = false; break; }
                    tc::fence_after_sync();
#pragma unroll
                    for (int kk = 0; kk < kKeys / 16; ++kk) {   // the chunk's keys in steps of 16
                        tc::mma_bf16_ss(tmem + 256 + tt * 128,
                                        tc::desc_kmajor_sw128(ap + tt * kHalf + kk * 32),
                                        tc::desc_mnmajor_sw128(av + kk * 16 * 128, kHalfKV), idesc_o,
                                        (t > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(&o_done[tt]);
                }
                if (!ok) break;
                tc::mma_commit(&kv_empty[s]);
            }
            tc::mma_commit(mma_done);
            int zero = 0;
            const tc::Guard drain{&zero, nullptr, 0, p.timeout_ns};
            tc::wait(mma_done, 0, drain, 0);
        }
    } else {
        // ---------------------------------------------------------------- softmax
        const int tt = warp >> 2;                    // this warpgroup's tile
        const int r = threadIdx.x & 127;
        const int i = q0 + tt * BQ + r / G;
        const int h = g * G + r % G;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tmem_s = tmem + tt * 128;     // the tile's two S buffers
        const uint32_t tmem_o = tmem + 256 + tt * 128;
        uint64_t* my_s_full = s_full + tt * 2;
        uint64_t* my_s_empty = s_empty + tt * 2;
        uint64_t* my_p_full = p_full + tt;
        uint64_t* my_o_done = o_done + tt;
        const float sl2 = p.sl2;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        uint8_t* prow0 = sP + tt * kHalf + r * 128;  // row r of the tile's P
        for (int t = 0; ok && t < n_ch; ++t) {
            const int bb = t & 1, s = t % kStages;
            if (!tc::wait(&my_s_full[bb], (t >> 1) & 1, gd, 8)) { ok = false; break; }
            tc::fence_after_sync();
            constexpr int NC = kKeys / 32;            // 32-column loads of a chunk
            uint32_t v[NC][32];
#pragma unroll
            for (int c = 0; c < NC; ++c) tc::tmem_ld32(tmem_s + lane_off + bb * kKeys + c * 32, v[c]);
#pragma unroll
            for (int c = 0; c < NC; ++c) tc::tmem_wait_ld(v[c]);
            tc::fence_before_sync();
            tc::mbar_arrive(&my_s_empty[bb]);
            // mask: keys past the support (index -1) or after query i
            if (DENSE) {
                if ((t + 1) * kKeys - 1 > i) {           // only the chunks that reach past i
#pragma unroll
                    for (int c = 0; c < NC; ++c)
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (t * kKeys + c * 32 + e > i) v[c][e] = __float_as_uint(-INFINITY);
                }
            } else {
                // support rows are ascending: a chunk whose first and last keys lie in
                // [0, the tile's first query] needs no mask (most chunks: the keys before
                // the block); otherwise one unsigned compare drops both -1 and keys > i
                const int jf = sIdx[s * kKeys], jl = sIdx[s * kKeys + kKeys - 1];
                if (!(jf >= 0 && jl >= 0 && jl <= q0 + tt * BQ)) {
                    const int4* ix4 = reinterpret_cast<const int4*>(sIdx + s * kKeys);
#pragma unroll
                    for (int c = 0; c < NC; ++c)
#pragma unroll
                        for (int e4 = 0; e4 < 8; ++e4) {
                            const int4 jj = ix4[c * 8 + e4];
                            const int js[4] = {jj.x, jj.y, jj.z, jj.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                if ((unsigned)js[e] > (unsigned)i)
                                    v[c][e4 * 4 + e] = __float_as_uint(-INFINITY);
                        }
                }
            }
            float tm[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < NC; ++c)
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    tm[c & 1] = tc::max3(tm[c & 1], __uint_as_float(v[c][e]),
                                         __uint_as_float(v[c][e + 1]));
            const float tmax = fmaxf(tm[0], tm[1]) * sl2;
            const bool raise = tmax > m_used + kRescaleLog2;
            const float m_new = raise ? tmax : m_used;
            // a row with no key so far keeps l = 0 and a zero P row
            const bool none = m_new == -INFINITY;
            const float corr = none ? 1.f : tc::ex2(m_used - m_new);     // 0 on the first key
            const uint64_t sl2x2 = tc::f2_pack(sl2, sl2);
            const uint64_t negm2 = tc::f2_pack(none ? 0.f : -m_new, none ? 0.f : -m_new);
            uint64_t sum2[2] = {0ull, 0ull};
#pragma unroll
            for (int c8 = 0; c8 < kKeys / 8; ++c8) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int col = c8 * 8 + 2 * e;
                    const float s0 = __uint_as_float(v[col / 32][col % 32]);
                    const float s1 = __uint_as_float(v[(col + 1) / 32][(col + 1) % 32]);
                    const uint64_t x2 = tc::f2_fma(tc::f2_pack(s0, s1), sl2x2, negm2);
                    float x0, x1, p0, p1;
                    tc::f2_unpack(x2, x0, x1);
                    if (e == 3) {
                        tc::ex2_fma2(x0, x1, p0, p1);
                    } else {
                        p0 = tc::ex2(x0);
                        p1 = tc::ex2(x1);
                    }
                    // masked keys are exactly 0 (the polynomial path would leave ~2^-125)
                    p0 = s0 == -INFINITY ? 0.f : p0;
                    p1 = s1 == -INFINITY ? 0.f : p1;
                    sum2[e & 1] = tc::f2_add(sum2[e & 1], tc::f2_pack(p0, p1));
                    __nv_bfloat162 pk = __floats2bfloat162_rn(p0, p1);
                    w[e] = *reinterpret_cast<uint32_t*>(&pk);
                }
                // P V of chunk t-1 must have finished reading the P tile before it is
                // overwritten; wait once, before the first store
                if (c8 == 0 && t > 0) {
                    if (!tc::wait(my_o_done, (t - 1) & 1, gd, 9)) { ok = false; break; }
                }
                uint4* dst = reinterpret_cast<uint4*>(prow0 + ((c8 ^ (r & 7)) << 4));
                *dst = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (!ok) break;
            float a0, a1, a2, a3;
            tc::f2_unpack(sum2[0], a0, a1);
            tc::f2_unpack(sum2[1], a2, a3);
            l = l * corr + ((a0 + a1) + (a2 + a3));
            const bool any_raise = __any_sync(0xffffffffu, raise && t > 0 && !none);
            if (any_raise) {
                tc::fence_after_sync();
                const float f = (raise && t > 0 && !none) ? corr : 1.f;
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
            tc::mbar_arrive(my_p_full);
        }
        // epilogue: wait for the last P V, normalise, store bf16 rows
        if (ok && tc::wait(my_o_done, (n_ch - 1) & 1, gd, 10)) {
            tc::fence_after_sync();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16* orow = p.out + ((size_t)i * p.Hq + h) * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tc::tmem_ld32(tmem_o + lane_off + c * 32, o);
                tc::tmem_wait_ld(o);
                if (i < p.N) {
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
            if (p.lse && i < p.N) p.lse[(size_t)h * p.N + i] = (m_used + __log2f(l)) * kLn2;
        }
    }
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

template <int G, int D, int TT, bool DENSE>
cudaError_t launch_block_tc(const AttnArgs& a, cudaStream_t st) {
    constexpr int BQ = 128 / G;
    CUtensorMap tq, tk, tv;
    const uint64_t d = a.d;
    if (!make_tmap_3d_bf16(&tq, a.q, d, a.Hq, a.N, d * 2, (uint64_t)a.Hq * d * 2, 64, G, BQ))
        return cudaErrorInvalidValue;
    if (DENSE) {
        if (!make_tmap_3d_bf16(&tk, a.k, d, a.Hkv, a.N, d * 2, (uint64_t)a.Hkv * d * 2, 64, 1, kKeys) ||
            !make_tmap_3d_bf16(&tv, a.v, d, a.Hkv, a.N, d * 2, (uint64_t)a.Hkv * d * 2, 64, 1, kKeys))
            return cudaErrorInvalidValue;
    } else {
        tk = tq;                                // unused by the gathering form
        tv = tq;
    }
    BlockTcParams p{};
    p.k = (const __nv_bfloat16*)a.k;
    p.v = (const __nv_bfloat16*)a.v;
    p.N = (int)a.N;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    if (DENSE) {
        // one "block" per CTA: TT query tiles, keys 0 .. the last of their queries
        p.block_q = TT * BQ;
        p.kmax = 0;
        p.tiles_per_block = TT;
        p.n_ctas_per_group = (int)((a.N + TT * BQ - 1) / (TT * BQ));
    } else {
        p.block_q = a.block_q;
        p.kmax = a.kmax;
        p.tiles_per_block = a.block_q / BQ;
        const int nb = (int)((a.N + a.block_q - 1) / a.block_q);
        p.n_ctas_per_group = nb * p.tiles_per_block / TT;
    }
    p.sl2 = a.sl2;
    p.sup_idx = a.sup_idx;
    p.sup_len = a.sup_len;
    p.out = (__nv_bfloat16*)a.out;
    p.lse = a.lse;
    p.status = a.status;
    p.timeout_ns = wait_timeout_ns();
    constexpr int smem = block_tc_smem_bytes<D, TT>();
    static_assert(smem <= 227 * 1024, "block pass 3 shared memory");
    auto kern = k_attn_block_tc<G, D, TT, DENSE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(p.n_ctas_per_group * a.Hkv), block_threads(TT), smem, st>>>(tq, tk, tv, p);
    note_launch();
    return cudaGetLastError();
}

// Two tiles per CTA when the block has an even number of tiles, else one (dense: two).
template <int G, int D, bool DENSE>
cudaError_t launch_tt(const AttnArgs& a, cudaStream_t st) {
    if constexpr (D == 256) {
        // one tile (its O takes TMEM columns 256..511); no dense form
        return DENSE ? cudaErrorNotSupported : launch_block_tc<G, D, 1, false>(a, st);
    } else {
        if (DENSE) return launch_block_tc<G, D, 2, true>(a, st);
        return (a.block_q / (128 / G)) % 2 == 0 ? launch_block_tc<G, D, 2, false>(a, st)
                                                 : launch_block_tc<G, D, 1, false>(a, st);
    }
}

template <int D, bool DENSE>
cudaError_t dispatch_g(const AttnArgs& a, cudaStream_t st) {
    switch (a.Hq / a.Hkv) {
        case 1: return launch_tt<1, D, DENSE>(a, st);
        case 2: return launch_tt<2, D, DENSE>(a, st);
        case 4: return launch_tt<4, D, DENSE>(a, st);
        case 8: return launch_tt<8, D, DENSE>(a, st);
        case 16: return launch_tt<16, D, DENSE>(a, st);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace

bool block_tc_supported(const AttnArgs& a) {
    const int G = a.Hq / a.Hkv;
    if (a.dtype != TAM_BF16 || (a.d != 64 && a.d != 128 && a.d != 256) || a.block_q <= 1)
        return false;
    if (!(G == 1 || G == 2 || G == 4 || G == 8 || G == 16)) return false;
    return a.block_q % (128 / G) == 0 && a.sup_idx != nullptr;
}

cudaError_t block_attention_tc(const AttnArgs& a, cudaStream_t st) {
    switch (a.d) {
        case 64: return dispatch_g<64, false>(a, st);
        case 128: return dispatch_g<128, false>(a, st);
        default: return dispatch_g<256, false>(a, st);
    }
}

bool dense_pair_tiles_supported(const AttnArgs& a) {
    const int G = a.Hq / a.Hkv;
    if (a.dtype != TAM_BF16 || (a.d != 64 && a.d != 128)) return false;
    return G == 1 || G == 2 || G == 4 || G == 8 || G == 16;
}

cudaError_t dense_pair_tiles(const AttnArgs& a, cudaStream_t st) {
    return a.d == 64 ? dispatch_g<64, true>(a, st) : dispatch_g<128, true>(a, st);
}

}  // namespace tam
