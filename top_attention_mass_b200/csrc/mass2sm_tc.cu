// Pass 2 on CTA pairs: head-averaged mass and its top-k with 2-SM UMMA.
//
//   P_i[j] = (1/Hq) sum_h exp(scale * q[i,h].k[j,g(h)] - lse[h,i]),  j <= i
//   rows:    the rows P_i (or, with a key stride 2^L, their values at the sampled
//            keys j = m 2^L only), written to a triangular slab;
//   stream:  per query, only the keys with P_i[j] >= tau_i are kept: each mass warp
//            appends them to its own segment of the row's candidate buffer, so the
//            N x N mass never reaches memory (the exact top-k over the candidates
//            is row_topk.cu's cand_select);
//   block:   M_b[j] = sum_{i in b, j <= i} P_i[j], as in mass_tc.cu
//
// (arXiv 2606.07703, Abstract; gist.science technical report §2.1 "Selektion",
// "Granularität".)
//
// Same orientation as the single-CTA kernel (S^T = K_g Q_g^T, the key-row thread
// sums every head of a query in registers), but a cluster of two CTAs issues one
// M = 256, N = 128 UMMA per KV group: each CTA holds 128 of the 256 keys (A) and
// the Q rows of 16 of the pair's 32 queries for all heads (its half of B), and each
// CTA's TMEM receives its 128 keys x all 128 (query, head) columns.  Every K row
// read from L2 then serves 32 queries instead of 16, and each CTA reads half as many
// operand bytes per unit of work - the two things that bounded the single-CTA pass.
//
// Roles in each CTA (W = 8 mass warps per query, 16 block-shared; W + 2 warps):
//   warp W      TMA producer: this CTA's Q half (once) and its 128 keys of each
//               256-key tile, counted on CTA 0's barriers;
//   warp W+1    CTA 0 only: issues the pair MMAs into a ring of four 128-column TMEM
//               slots and commits to the barriers of both CTAs;
//   warps 0..W-1 mass warps: thread = key row (warp w reads TMEM lanes 32 (w % 4) ..),
//               column part w / 4 of W / 4 parts, i.e. the (query, head) columns of
//               that share of the pair's queries; exp2 against the pass-1 LSE, sum
//               over heads -> mass of those queries for 128 keys.  Several warps per
//               TMEM lane quarter keep several exp streams per scheduler.  Rows mode
//               stores the mass to the row slab (one coalesced 128-byte store per warp
//               and query); stream mode ballots the keys at or above the query's
//               threshold and appends them (value, key) to the warp's segment of the
//               row (a warp-uniform running count, no atomics; segments stay in key
//               order); block-shared mass goes to the fixed-point block sums.
// Every wait is bounded; the pair shakes hands before it frees TMEM and exits so
// that no remote arrive or MMA of one CTA can land after the other left.
#include "launch.h"
#include "mass_exp.cuh"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace tam {
namespace {

constexpr int kModeRows = 0, kModeBlock = 1, kModeStream = 2;
// K ring of two key tiles (deeper rings, up to four tiles where Q leaves room, measured
// no faster: the pipeline is not waiting on K)
constexpr int kStages = 2;
// Mass warps: 16 (four per TMEM lane quarter, each on a quarter of the columns), in
// every mode: with the packed head sums, 16 warps measured 10 % faster per query than 8
// (7.25 vs 8.02 ms at 32K, same results) and 5 % faster block-shared.  Then the TMA
// producer and the MMA issuer.
__host__ __device__ constexpr int mass_warps(bool) { return 16; }
__host__ __device__ constexpr int pair_threads(bool block) { return 32 * (mass_warps(block) + 2); }
constexpr int kNQ = 128;                // MMA N: (query, head) columns of the pair
constexpr int kHalfRows = 64;           // B rows held by each CTA
constexpr int kR = 512 / kNQ;           // TMEM accumulator slots
constexpr int kTileKeys = 256;          // keys per pair tile (128 per CTA)

constexpr int kMaxDynSmem = 227 * 1024;
__host__ __device__ constexpr int pair_smem_bytes(int D, int Hkv) {
    // alignment slack + Q half + K ring + lse of all 128 columns + thresholds + barriers
    return 1024 + Hkv * kHalfRows * D * 2 + kStages * 128 * D * 2 + Hkv * kNQ * 4 + 128 + 512;
}

struct PairParams {
    int N, Hq, Hkv, pair0, n_pairs, block_q;
    int64_t row0, row1;       // per query: the rows [row0, row1) of this launch
    int kst;                  // rows mode: key m of the K map sits at position m * kst
    uint64_t out_cap;         // entries of rows / cand / bmass (debug-checks build)
    int seg_cap;              // stream mode: entries per candidate segment
    float sl2, inv_hq;
    const float* lse;
    float* rows;
    const float* tau;         // stream mode: threshold of every query [N]
    uint2* cand;              // stream mode: (value bits, key) of rows [row0, row1)
    int32_t* cnt;             // stream mode: appended count per (row, segment)
    unsigned long long* bmass;
    int32_t* status;
    uint64_t timeout_ns;
    int dbg;
};

// Adds a block-mass column sum in 2^-40 fixed point (one 64-bit atomic per (block, key)
// and warp part).
__device__ __forceinline__ void block_mass_add(const PairParams& p, int64_t at, float sum) {
    if (in_bounds(p.status, KID_BLOCK_MASS_TC, kSiteBlockMass, (uint64_t)at, p.out_cap))
        atomicAdd(&p.bmass[at], (unsigned long long)__float2ll_rn(sum * p.inv_hq * 1099511627776.0f));
}

__host__ __device__ __forceinline__ int64_t bmass_row(int64_t b, int block_q) {
    return (int64_t)block_q * b * (b + 1) / 2;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

template <int G, int D, int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair_threads(MODE == kModeBlock), 1)
k_mass_pair(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
            const PairParams p) {
    constexpr bool BLOCK = MODE == kModeBlock;
    constexpr bool STREAM = MODE == kModeStream;
    constexpr int kMassWarps = mass_warps(BLOCK);
    constexpr int kProducerWarp = kMassWarps, kMmaWarp = kMassWarps + 1;
    constexpr int BQP = kNQ / G;              // queries of the pair
    constexpr int BQC = kHalfRows / G;        // queries of one column half
    constexpr int NH = D / 64;
    constexpr uint32_t kQHalf = kHalfRows * 128;   // one 64-element half of a group's B rows
    constexpr uint32_t kKHalf = 128 * 128;
    constexpr uint32_t kKTile = NH * kKHalf;
    const int Hkv = p.Hkv;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sQ = base;
    uint8_t* sK = sQ + Hkv * NH * kQHalf;
    float* sLse = reinterpret_cast<float*>(sK + kStages * kKTile);     // Hkv * 128
    float* sTau = sLse + Hkv * kNQ;                                      // 32 (stream)
    uint64_t* bars = reinterpret_cast<uint64_t*>(sTau + 32);
    uint64_t* q_full = bars;                 // CTA 0's counts both CTAs' Q bytes
    uint64_t* k_full = q_full + 1;           // CTA 0's counts both CTAs' K bytes
    uint64_t* k_empty = k_full + kStages;    // both (pair commits)
    uint64_t* s_full = k_empty + kStages;    // both (pair commits)
    uint64_t* s_empty = s_full + kR;         // CTA 0's: both CTAs' mass threads
    uint64_t* mma_done = s_empty + kR;       // both (pair commit)
    uint64_t* exit_bar = mma_done + 1;       // each: the peer's arrival at the end
    uint64_t* never = exit_bar + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = tc::cluster_rank();
    const uint32_t peer = rank ^ 1u;
    const int pt = p.pair0 + p.n_pairs - 1 - (int)(blockIdx.x >> 1);   // heaviest pair first
    const int q0 = pt * BQP;
    const int q_last = min(p.N, q0 + BQP) - 1;
    const int n_kt = (q_last / p.kst) / kTileKeys + 1;
    const int n_units = n_kt * Hkv;
    const int my_q0 = q0 + (int)rank * BQC;
    const int64_t slab0 = sample_offset(p.row0, p.kst);

    if (threadIdx.x == 0) {
        tc::mbar_init(q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(&k_full[s], 1);
            tc::mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < kR; ++s) {
            tc::mbar_init(&s_full[s], 1);
            tc::mbar_init(&s_empty[s], 2 * kMassWarps);   // every mass warp of both CTAs
        }
        tc::mbar_init(mma_done, 1);
        tc::mbar_init(exit_bar, 1);
        tc::mbar_init(never, 1);
        *abort_flag = 0;
        tc::fence_barrier_init();
    }
    for (int t = threadIdx.x; t < Hkv * kNQ; t += blockDim.x) {
        const int g = t / kNQ, c = t % kNQ;
        const int i = q0 + c / G, h = g * G + c % G;
        sLse[t] = (i < p.N) ? -p.lse[(size_t)h * p.N + i] * kLog2e : -INFINITY;   // negated
    }
    if constexpr (STREAM) {
        for (int c = threadIdx.x; c < BQP; c += blockDim.x) {
            const int64_t i = q0 + c;
            sTau[c] = (i < p.row1) ? p.tau[i] : INFINITY;
        }
    }
    if (warp == 0) {
        tc::tmem_alloc_pair(tmem_slot, 512);
        tc::tmem_relinquish_pair();
    }
    tc::fence_before_sync();
    __syncthreads();
    // both CTAs' barriers must be initialised before either CTA signals the other
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // a timeout in either CTA aborts both (the flag of the peer is raised over DSMEM)
    const tc::Guard gd{abort_flag, p.status, BLOCK ? KID_BLOCK_MASS_TC : KID_MASS_TC, p.timeout_ns,
                       tc::map_to_cta(tc::smem_u32(abort_flag), peer)};
    int zero = 0;
    const tc::Guard drain{&zero, nullptr, 0, p.timeout_ns};
    // the exit handshake outlasts any skew between the two CTAs' wind-down
    const tc::Guard handshake{&zero, nullptr, 0, 16 * p.timeout_ns};

    if (warp == kProducerWarp) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            tc::prefetch_tmap(&tmQ);
            tc::prefetch_tmap(&tmK);
            if (rank == 0) tc::mbar_arrive_expect_tx(q_full, 2u * Hkv * NH * kQHalf);
            for (int g = 0; g < Hkv; ++g)
                for (int h = 0; h < NH; ++h)
                    tc::tma_load_3d_pair(sQ + (g * NH + h) * kQHalf, &tmQ, q_full, h * 64, g * G,
                                         my_q0);
            int issued = 0;
            for (int u = 0; u < n_units; ++u) {
                const int s = u % kStages;
                if (!tc::wait(&k_empty[s], ((u / kStages) & 1) ^ 1, gd, 1)) break;
                const int kt = u / Hkv, g = u % Hkv;
                if (rank == 0) tc::mbar_arrive_expect_tx(&k_full[s], 2u * kKTile);
                for (int h = 0; h < NH; ++h)
                    tc::tma_load_3d_pair(sK + s * kKTile + h * kKHalf, &tmK, &k_full[s], h * 64, g,
                                         kt * kTileKeys + (int)rank * 128);
                ++issued;
            }
            // the last pair commits on k_empty must have landed before this CTA exits
            // (when aborting, the MMAs behind them may never have been issued; the
            // completion of every issued MMA is covered by mma_done)
            for (int u = max(0, issued - kStages); u < issued && !*abort_flag; ++u)
                tc::wait(&k_empty[u % kStages], (u / kStages) & 1, drain, 0);
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------------- MMA issuer (CTA 0)
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = tc::idesc_bf16_f32(256, kNQ);
            bool ok = tc::wait(q_full, 0, gd, 2);
            int done = 0;
            for (int u = 0; ok && u < n_units; ++u) {
                const int s = u % kStages, slot = u % kR, g = u % Hkv;
                if (!tc::wait(&k_full[s], (u / kStages) & 1, gd, 3)) break;
                if (!tc::wait(&s_empty[slot], ((u / kR) & 1) ^ 1, gd, 4)) break;
                tc::fence_after_sync();
                const uint32_t ak = tc::smem_u32(sK + s * kKTile);
                const uint32_t bq = tc::smem_u32(sQ + g * NH * kQHalf);
#pragma unroll
                for (int kk = 0; kk < NH * 4; ++kk) {
                    const uint32_t offk = (kk >> 2) * kKHalf + (kk & 3) * 32;
                    const uint32_t offq = (kk >> 2) * kQHalf + (kk & 3) * 32;
                    tc::mma_bf16_ss_pair(tmem + slot * kNQ, tc::desc_kmajor_sw128(ak + offk),
                                         tc::desc_kmajor_sw128(bq + offq), idesc, kk > 0 ? 1u : 0u);
                }
                tc::mma_commit_pair(&k_empty[s], 0x3);
                tc::mma_commit_pair(&s_full[slot], 0x3);
                done = u + 1;
            }
            tc::mma_commit_pair(mma_done, 0x3);
            // the peer's last slot releases must have landed before CTA 0 exits (when
            // aborting, the exit handshake stands in for them)
            for (int u = max(0, done - kR); u < done && !*abort_flag; ++u)
                tc::wait_cluster(&s_empty[u % kR], (u / kR) & 1, drain, 0);
        }
    } else if (warp < kMassWarps) {
        // ---------------------------------------------------------------- mass warps
        constexpr int kParts = kMassWarps / 4;         // warps per TMEM lane quarter
        constexpr int kCols = kNQ / kParts;            // columns of one part
        constexpr int kQP = kCols / G;                 // queries of one part
        const int quarter = warp & 3, part = warp >> 2;
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(part * kCols);
        const uint32_t s_empty_leader = tc::map_to_cta(tc::smem_u32(s_empty), 0);
        // stream mode: this warp's segment of every row and its running counts; the
        // candidates of (query qbase + ql, this segment) start at entry off0 + ql * qstride
        // (32-bit: the host keeps a chunk's candidate buffer below 2^32 entries)
        const int seg = (int)rank * 4 + quarter;
        const int qbase = q0 + part * kQP;
        const uint32_t qstride = 8u * (uint32_t)p.seg_cap;
        const uint32_t off0 = (uint32_t)(qbase - (int)p.row0) * qstride + (uint32_t)(seg * p.seg_cap);
        const int qend = STREAM ? min(kQP, (int)(p.row1 - qbase)) : 0;   // queries in the launch
        int cnt[STREAM ? kQP : 1];
#pragma unroll
        for (int q = 0; q < (STREAM ? kQP : 1); ++q) cnt[q] = 0;
        bool ok = true;
        if (p.dbg & kDebugForceTimeout) ok = tc::wait(never, 0, gd, 9);
        const uint64_t sl2x2 = tc::f2_pack(p.sl2, p.sl2);
        for (int kt = 0; ok && kt < n_kt; ++kt) {
            MassAcc<G, kQP> acc2;
            acc2.clear();
            for (int g = 0; g < Hkv; ++g) {
                const int u = kt * Hkv + g;
                const int slot = u % kR;
                if (!tc::wait(&s_full[slot], (u / kR) & 1, gd, 5)) { ok = false; break; }
                tc::fence_after_sync();
                const uint32_t col0 = lane_addr + slot * kNQ;
                uint32_t va[32], vb[32];
                tc::tmem_ld32(col0, va);
                tc::tmem_wait_ld(va);
#pragma unroll
                for (int c = 0; c < kCols / 32; ++c) {
                    uint32_t (&cur)[32] = (c & 1) ? vb : va;
                    uint32_t (&nxt)[32] = (c & 1) ? va : vb;
                    if (c + 1 < kCols / 32) tc::tmem_ld32(col0 + (c + 1) * 32, nxt);
                    const ulonglong2* nl =
                        reinterpret_cast<const ulonglong2*>(sLse + g * kNQ + part * kCols + c * 32);
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const ulonglong2 L = nl[c4];
                        mass_columns4<G, kQP>(acc2, c * 32 + c4 * 4, cur[c4 * 4], cur[c4 * 4 + 1],
                                              cur[c4 * 4 + 2], cur[c4 * 4 + 3], L.x, L.y, sl2x2,
                                              (c4 & 1) != 0);
                    }
                    if (c + 1 < kCols / 32) tc::tmem_wait_ld(nxt);
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) {
                    if (rank == 0) tc::mbar_arrive(&s_empty[slot]);
                    else tc::mbar_arrive_remote_relaxed(s_empty_leader + (uint32_t)slot * 8u);
                }
            }
            if (!ok) break;
            float acc[kQP];
#pragma unroll
            for (int q = 0; q < kQP; ++q) acc[q] = acc2.get(q);
            const int m = kt * kTileKeys + (int)rank * 128 + row;   // key (or sample) index
            if constexpr (MODE == kModeRows) {
                // row i of the slab starts off(i) - off(row0) floats in (32-bit: the host
                // keeps a chunk's slab below 2^32 floats) and holds i / S + 1 values; the
                // offsets of this part's rows follow from the first one by adding
                // i / S + 1, so no division runs per key tile.  Lanes store consecutive
                // keys of one query; key m sits at position m S <= i iff m <= i / S.
                int a = qbase / p.kst, b = qbase - a * p.kst;   // first row's i / S, i % S
                uint32_t off = (uint32_t)(qbase + (int64_t)p.kst * ((int64_t)a * (a - 1) / 2) +
                                          (int64_t)a * b - slab0);
#pragma unroll
                for (int ql = 0; ql < kQP; ++ql) {
                    if (m <= a && qbase + ql < p.row1 &&
                        in_bounds(p.status, KID_MASS_TC, kSiteRows, off + (uint32_t)m, p.out_cap))
                        p.rows[off + (uint32_t)m] = acc[ql] * p.inv_hq;
                    off += (uint32_t)a + 1u;
                    if (++b == p.kst) { b = 0; ++a; }
                }
            } else if constexpr (STREAM) {
                // keys at or above the query's threshold, appended in key order to this
                // warp's segment (positions past the capacity are only counted); no
                // warp-uniform branch, so the queries' ballot chains interleave
                const uint32_t lt = lanemask_lt();
                const bool below = m <= qbase;        // key at or before every query here
#pragma unroll
                for (int ql = 0; ql < kQP; ++ql) {
                    const float v = acc[ql] * p.inv_hq;
                    const bool pass = ql < qend && (below || m <= qbase + ql) &&
                                      v >= sTau[part * kQP + ql];
                    const uint32_t bal = __ballot_sync(0xffffffffu, pass);
                    const int pos = cnt[ql] + __popc(bal & lt);
                    const uint32_t at = off0 + (uint32_t)ql * qstride + (uint32_t)pos;
                    if (pass && pos < p.seg_cap && in_bounds(p.status, KID_MASS_TC, kSiteCand, at, p.out_cap))
                        p.cand[at] = make_uint2(__float_as_uint(v), (uint32_t)m);
                    cnt[ql] += __popc(bal);
                }
            } else {
                const int j = m;
                const int qh = q0 + part * kQP;
                int cur_b = qh / p.block_q;
                float sum = 0.f;
#pragma unroll
                for (int q = 0; q < kQP; ++q) {
                    const int i = qh + q;
                    if (i < p.N) {
                        const int b = i / p.block_q;
                        if (b != cur_b) {
                            if (sum > 0.f)
                                block_mass_add(p, bmass_row(cur_b, p.block_q) + j, sum);
                            sum = 0.f;
                            cur_b = b;
                        }
                        if (j <= i) sum += acc[q];
                    }
                }
                if (sum > 0.f) block_mass_add(p, bmass_row(cur_b, p.block_q) + j, sum);
            }
        }
        if constexpr (STREAM) {
            if (ok && lane == 0) {
#pragma unroll
                for (int ql = 0; ql < kQP; ++ql) {
                    const int64_t i = q0 + part * kQP + ql;
                    if (i < p.row1) p.cnt[(i - p.row0) * 8 + seg] = cnt[ql];
                }
            }
        }
    }
    // every CTA waits for the pair MMAs (they write into both CTAs' TMEM)
    if (threadIdx.x == 0) tc::wait(mma_done, 0, drain, 0);
    __syncthreads();
    // pair handshake: neither CTA frees TMEM or exits while the other may still touch it
    if (threadIdx.x == 0) {
        tc::mbar_arrive_remote(tc::map_to_cta(tc::smem_u32(exit_bar), peer));
        tc::wait_cluster(exit_bar, 0, handshake, 0);
    }
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc_pair(tmem, 512);
    }
}

template <int G, int D, int MODE>
cudaError_t launch_pair(const MassArgs& a, cudaStream_t st) {
    constexpr bool BLOCK = MODE == kModeBlock;
    constexpr int BQP = kNQ / G, BQC = kHalfRows / G;
    CUtensorMap tq, tk;
    const uint64_t d = a.d;
    // rows mode with a key stride reads every S-th key row: the same K with an S-fold
    // longer row pitch and (N - 1) / S + 1 rows
    const int S = (MODE == kModeRows && a.kst > 1) ? a.kst : 1;
    const uint64_t n_keys = (uint64_t)((a.N - 1) / S) + 1;
    if (!make_tmap_3d_bf16(&tq, a.q, d, a.Hq, a.N, d * 2, (uint64_t)a.Hq * d * 2, 64, G, BQC) ||
        !make_tmap_3d_bf16(&tk, a.k, d, a.Hkv, n_keys, d * 2, (uint64_t)a.Hkv * d * 2 * S, 64,
                           1, 128))
        return cudaErrorInvalidValue;
    PairParams p{};
    p.N = (int)a.N;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    // per query the launch covers the queries [row0, row1) (row0 a multiple of BQP)
    const int64_t r0 = BLOCK ? 0 : a.row0, r1 = BLOCK ? a.N : a.row1;
    p.pair0 = (int)(r0 / BQP);
    p.n_pairs = (int)((r1 + BQP - 1) / BQP) - p.pair0;
    p.row0 = r0;
    p.row1 = r1;
    p.kst = S;
    p.seg_cap = a.seg_cap;
    p.block_q = a.block_q;
    p.sl2 = a.sl2;
    p.inv_hq = 1.f / (float)a.Hq;
    p.lse = a.lse;
    p.rows = a.rows;
    p.tau = a.tau;
    p.cand = reinterpret_cast<uint2*>(a.cand);
    p.cnt = a.cnt;
    p.bmass = reinterpret_cast<unsigned long long*>(a.bmass);
    p.status = a.status;
    p.out_cap = a.out_cap;
    p.timeout_ns = wait_timeout_ns();
    p.dbg = debug_flags();
    if (p.n_pairs <= 0) return cudaSuccess;
    const int smem = pair_smem_bytes(D, a.Hkv);
    auto kern = k_mass_pair<G, D, MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (BLOCK) {
        const int64_t nb = (a.N + a.block_q - 1) / a.block_q;
        e = cudaMemsetAsync(a.bmass, 0, (size_t)bmass_row(nb, a.block_q) * 8, st);
        if (e != cudaSuccess) return e;
    }
    kern<<<(unsigned)(2 * p.n_pairs), pair_threads(BLOCK), smem, st>>>(tq, tk, p);
    note_launch();
    return cudaGetLastError();
}

template <int D, int MODE>
cudaError_t dispatch_g(const MassArgs& a, cudaStream_t st) {
    switch (a.Hq / a.Hkv) {
        case 4: return launch_pair<4, D, MODE>(a, st);
        case 8: return launch_pair<8, D, MODE>(a, st);
        case 16: return launch_pair<16, D, MODE>(a, st);
        default: return cudaErrorNotSupported;
    }
}

template <int D>
cudaError_t dispatch_mode(const MassArgs& a, cudaStream_t st) {
    if (a.block_q > 1) return dispatch_g<D, kModeBlock>(a, st);
    return a.stream ? dispatch_g<D, kModeStream>(a, st) : dispatch_g<D, kModeRows>(a, st);
}

}  // namespace

bool pair_mass_supported(const MassArgs& a) {
    const int G = a.Hq / a.Hkv;
    if (a.dtype != TAM_BF16 || (a.d != 64 && a.d != 128)) return false;
    if (G != 4 && G != 8 && G != 16) return false;
    if (a.block_q > 1 && a.block_q > (1 << 20)) return false;
    return pair_smem_bytes(a.d, a.Hkv) <= kMaxDynSmem;
}

// Launches the pair kernel only: per query it fills the slab rows [row0, row1) (rows
// mode) or their candidate segments (stream mode); per block the caller runs the
// block top-k after it.
cudaError_t pair_mass(const MassArgs& a, cudaStream_t st) {
    return a.d == 64 ? dispatch_mode<64>(a, st) : dispatch_mode<128>(a, st);
}

}  // namespace tam
