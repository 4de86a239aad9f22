// Pass 2 on the tensor cores: head-averaged token mass (and the indexer's scores).
//
//   P_i[j] = (1/Hq) sum_h exp(scale * q[i,h].k[j,g(h)] - lse[h,i]),  j <= i
//   per query:  the rows P_i, written to a triangular slab (with a key stride S
//               only the sampled keys j = m S); row_topk.cu then selects
//               S_i = top-min(k, i+1) of each row (value desc, index asc);
//               or, streamed, only the keys with P_i[j] >= tau_i, appended to the
//               row's candidate segments (one per mass warp) for cand_select
//   per block:  M_b[j] = sum_{i in block b, i >= j} P_i[j]  -> top-k in k_block_select
//   indexer:    the rows s_i[j] = q_idx[i] . k_idx[j] (one head, no exponentials),
//               as rows, sample rows or streamed candidates like the mass
//
// (arXiv 2606.07703, Abstract: "selects head-averaged token support"; gist.science
// technical report §2.1, "Mechanismus", "Selektion" and "Granularität", §2.2 for
// the indexer.)
//
// Orientation: one UMMA per KV group computes S^T = K_g Q_g^T with M = 128 keys
// and N = NQ columns (BQ queries x G heads of that group).  A CTA keeps Q of its
// BQ queries for *all* heads resident in shared memory, so the thread that owns a
// key row adds the probabilities of every head of a query in registers - the head
// average needs no cross-thread reduction.
// Roles (320 threads):
//   warp 8      TMA producer: Q (once, all groups), then K_g tiles in a 2-stage ring;
//   warp 9      MMA issuer: for each key tile, one UMMA chain per group into a ring
//               of 512/NQ TMEM slots;
//   warps 0-7   mass warps: thread = key row (warp w reads TMEM lanes 32 (w % 4) ..),
//               half w / 4 of the columns; exp2 against the pass-1 LSE, sum over
//               heads -> mass of BQ / 2 queries; causal mask; then either the mass
//               goes to the row slab (per query, indexer: lanes store consecutive keys
//               of one query), or the keys at or above the query's threshold are
//               appended to segment w % 4 of the query's row (streamed: a warp ballot
//               and a warp-uniform running count, no atomics; each segment has one
//               writer, so it stays in key order), or the block column sum is added
//               in 2^-40 fixed point (block-shared).
#include "launch.h"
#include "mass_exp.cuh"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace tam {
namespace {

// K ring depth: two tiles; one where the Q of every group at d = 256 leaves no room
// for a second 64 KB tile.
// Eight mass warps (two per TMEM lane quarter, each on half of the columns), then the
// TMA producer and the MMA issuer.
constexpr int kMassWarps = 8;
constexpr int kThreads = 32 * (kMassWarps + 2);

// Kernel modes: head-averaged mass rows, block-shared mass sums, the
// head-collapsed indexer's score rows (one score per (query, key), no exponentials),
// and the streamed (threshold-filtered) forms of the mass and indexer rows.
constexpr int kModeQuery = 0, kModeBlock = 1, kModeIndexer = 2, kModeQueryStream = 3,
              kModeIndexerStream = 4;

// alignment slack + Q (all groups) + K ring + lse2 + thresholds + barriers
__host__ __device__ constexpr int mass_smem_bytes(int NQ, int D, int Hkv, int stages = 2) {
    return 1024 + Hkv * NQ * D * 2 + stages * 128 * D * 2 + Hkv * NQ * 4 + 128 + 512;
}
constexpr int kMaxDynSmem = 227 * 1024;

struct MassParams {
    int N, Hq, Hkv, ct0, n_ctiles, block_q;
    int64_t row0, row1;              // per query / indexer: the rows [row0, row1)
    int kst;                         // rows modes: key m of the K map is at m * kst
    uint64_t out_cap;                // entries of rows / cand / bmass (debug-checks build)
    int seg_cap;                     // stream modes: entries per candidate segment
    float sl2, inv_hq;
    const float* lse;
    float* rows;                     // triangular row slab (per query / indexer)
    const float* tau;                // stream modes: threshold of every query [N]
    uint2* cand;                     // stream modes: (value bits, key) of rows [row0, row1)
    int32_t* cnt;                    // stream modes: appended count per (row, segment)
    unsigned long long* bmass;       // triangular block mass (block mode)
    int32_t* status;
    uint64_t timeout_ns;
    int dbg;
};

// Offset of block b's row in the triangular block-mass buffer.
__host__ __device__ __forceinline__ int64_t bmass_offset(int64_t b, int block_q) {
    return (int64_t)block_q * b * (b + 1) / 2;
}

// Adds a block-mass column sum in 2^-40 fixed point.
__device__ __forceinline__ void block_mass_add(const MassParams& p, int64_t at, float sum) {
    if (in_bounds(p.status, KID_BLOCK_MASS_TC, kSiteBlockMass, (uint64_t)at, p.out_cap))
        atomicAdd(&p.bmass[at], (unsigned long long)__float2ll_rn(sum * p.inv_hq * 1099511627776.0f));
}

template <int G, int D, int NQ, int MODE, int kStages>
__global__ void __launch_bounds__(kThreads, 1)
k_mass_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const MassParams p) {
    constexpr int BQ = NQ / G;            // queries per CTA
    constexpr int NH = D / 64;
    constexpr int R = 512 / NQ;           // TMEM accumulator slots
    constexpr uint32_t kQHalf = NQ * 128; // bytes of one 64-element half of a group's Q
    constexpr uint32_t kKHalf = 128 * 128;
    constexpr uint32_t kKTile = NH * kKHalf;
    constexpr bool BLOCK = MODE == kModeBlock;
    constexpr bool INDEXER = MODE == kModeIndexer || MODE == kModeIndexerStream;
    constexpr bool STREAM = MODE == kModeQueryStream || MODE == kModeIndexerStream;
    const int Hkv = p.Hkv;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sQ = base;                                   // Hkv * NH * kQHalf
    uint8_t* sK = sQ + Hkv * NH * kQHalf;                 // kStages * kKTile
    float* sLse = reinterpret_cast<float*>(sK + kStages * kKTile);   // Hkv * NQ
    float* sTau = sLse + Hkv * NQ;                                   // 32 (stream)
    uint64_t* bars = reinterpret_cast<uint64_t*>(sTau + 32);
    uint64_t* q_full = bars;
    uint64_t* k_full = q_full + 1;
    uint64_t* k_empty = k_full + kStages;
    uint64_t* s_full = k_empty + kStages;
    uint64_t* s_empty = s_full + R;
    uint64_t* mma_done = s_empty + R;
    uint64_t* never = mma_done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ct = p.ct0 + p.n_ctiles - 1 - (int)blockIdx.x;   // heaviest tile first
    const int q0 = ct * BQ;
    const int q_last = min(p.N, q0 + BQ) - 1;
    const int n_kt = (q_last / p.kst) / 128 + 1;
    const int n_units = n_kt * Hkv;
    const int64_t slab0 = sample_offset(p.row0, p.kst);

    if (threadIdx.x == 0) {
        tc::mbar_init(q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(&k_full[s], 1);
            tc::mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < R; ++s) {
            tc::mbar_init(&s_full[s], 1);
            tc::mbar_init(&s_empty[s], 32 * kMassWarps);
        }
        tc::mbar_init(mma_done, 1);
        tc::mbar_init(never, 1);
        *abort_flag = 0;
        tc::fence_barrier_init();
    }
    // log2-domain LSE of every column of every group (+inf for padding queries)
    if constexpr (!INDEXER) {
        for (int t = threadIdx.x; t < Hkv * NQ; t += blockDim.x) {
            const int g = t / NQ, c = t % NQ;
            const int i = q0 + c / G, h = g * G + c % G;
            sLse[t] = (i < p.N) ? -p.lse[(size_t)h * p.N + i] * kLog2e : -INFINITY;   // negated
        }
    }
    if constexpr (STREAM) {
        for (int c = threadIdx.x; c < BQ; c += blockDim.x) {
            const int64_t i = q0 + c;
            sTau[c] = (i < p.row1) ? p.tau[i] : INFINITY;
        }
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const tc::Guard gd{abort_flag, p.status,
                       BLOCK ? KID_BLOCK_MASS_TC : (INDEXER ? KID_INDEXER_TC : KID_MASS_TC),
                       p.timeout_ns};

    if (warp == kMassWarps) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            tc::prefetch_tmap(&tmQ);
            tc::prefetch_tmap(&tmK);
            tc::mbar_arrive_expect_tx(q_full, Hkv * NH * kQHalf);
            for (int g = 0; g < Hkv; ++g)
                for (int h = 0; h < NH; ++h)
                    tc::tma_load_3d(sQ + (g * NH + h) * kQHalf, &tmQ, q_full, h * 64, g * G, q0);
            int issued = 0;
            for (int u = 0; u < n_units; ++u) {
                const int s = u % kStages;
                const uint32_t ph = (u / kStages) & 1;
                if (!tc::wait(&k_empty[s], ph ^ 1, gd, 1)) break;
                const int kt = u / Hkv, g = u % Hkv;
                tc::mbar_arrive_expect_tx(&k_full[s], kKTile);
                for (int h = 0; h < NH; ++h)
                    tc::tma_load_3d(sK + s * kKTile + h * kKHalf, &tmK, &k_full[s], h * 64, g,
                                    kt * 128);
                ++issued;
            }
            int zero = 0;
            const tc::Guard drain{&zero, nullptr, 0, p.timeout_ns};
            for (int u = max(0, issued - kStages); u < issued; ++u)
                tc::wait(&k_full[u % kStages], (u / kStages) & 1, drain, 0);
            tc::wait(q_full, 0, drain, 0);
        }
    } else if (warp == kMassWarps + 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_bf16_f32(128, NQ);
            bool ok = tc::wait(q_full, 0, gd, 2);
            for (int u = 0; ok && u < n_units; ++u) {
                const int s = u % kStages;
                const uint32_t ph = (u / kStages) & 1;
                const int slot = u % R;
                const uint32_t sph = (u / R) & 1;
                const int g = u % Hkv;
                if (!tc::wait(&k_full[s], ph, gd, 3)) break;
                if (!tc::wait(&s_empty[slot], sph ^ 1, gd, 4)) break;
                tc::fence_after_sync();
                const uint32_t ak = tc::smem_u32(sK + s * kKTile);
                const uint32_t bq = tc::smem_u32(sQ + g * NH * kQHalf);
#pragma unroll
                for (int kk = 0; kk < NH * 4; ++kk) {
                    const uint32_t offk = (kk >> 2) * kKHalf + (kk & 3) * 32;
                    const uint32_t offq = (kk >> 2) * kQHalf + (kk & 3) * 32;
                    tc::mma_bf16_ss(tmem + slot * NQ, tc::desc_kmajor_sw128(ak + offk),
                                    tc::desc_kmajor_sw128(bq + offq), idesc, kk > 0 ? 1u : 0u);
                }
                tc::mma_commit(&k_empty[s]);
                tc::mma_commit(&s_full[slot]);
            }
            tc::mma_commit(mma_done);
            int zero = 0;
            const tc::Guard drain{&zero, nullptr, 0, p.timeout_ns};
            tc::wait(mma_done, 0, drain, 0);
        }
    } else if (warp < kMassWarps) {
        // ---------------------------------------------------------------- mass warps
        constexpr int kParts = kMassWarps / 4;         // warps per TMEM lane quarter
        constexpr int kCols = NQ / kParts;             // columns of one part
        constexpr int kQP = kCols / G;                 // queries of one part
        constexpr int CW = kCols < 32 ? kCols : 32;    // columns per TMEM load
        const int quarter = warp & 3, part = warp >> 2;
        const int row = quarter * 32 + lane;           // key row of the tile
        const uint32_t lane_addr =
            tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(part * kCols);
        // stream modes: the quarter-q warps write segment q of their queries' rows, with
        // running counts; the candidates of (query qbase + q, segment) start at entry
        // off0 + q * qstride (32-bit: the host keeps a chunk below 2^32 entries)
        const int qbase = q0 + part * kQP;
        const uint32_t qstride = 4u * (uint32_t)p.seg_cap;
        const uint32_t off0 =
            (uint32_t)(qbase - (int)p.row0) * qstride + (uint32_t)(quarter * p.seg_cap);
        const int qend = STREAM ? min(kQP, (int)(p.row1 - qbase)) : 0;
        int cnt[STREAM ? kQP : 1];
#pragma unroll
        for (int q = 0; q < (STREAM ? kQP : 1); ++q) cnt[q] = 0;
        bool ok = true;
        if (p.dbg & kDebugForceTimeout) ok = tc::wait(never, 0, gd, 9);
        const uint64_t sl2x2 = tc::f2_pack(p.sl2, p.sl2);
        for (int kt = 0; ok && kt < n_kt; ++kt) {
            float acc[kQP];
            MassAcc<G, kQP> acc2;
            acc2.clear();
            for (int g = 0; g < Hkv; ++g) {
                const int u = kt * Hkv + g;
                const int slot = u % R;
                if (!tc::wait(&s_full[slot], (u / R) & 1, gd, 5)) { ok = false; break; }
                tc::fence_after_sync();
                // stream this part's columns in CW-column chunks, loading chunk c+1
                // while chunk c is exponentiated
                const uint32_t col0 = lane_addr + slot * NQ;
                uint32_t va[CW], vb[CW];
                if constexpr (CW == 32) tc::tmem_ld32(col0, va); else tc::tmem_ld16(col0, va);
                tc::tmem_wait_ld(va);
#pragma unroll
                for (int c = 0; c < kCols / CW; ++c) {
                    uint32_t (&cur)[CW] = (c & 1) ? vb : va;
                    uint32_t (&nxt)[CW] = (c & 1) ? va : vb;
                    if (c + 1 < kCols / CW) {
                        if constexpr (CW == 32) tc::tmem_ld32(col0 + (c + 1) * CW, nxt);
                        else tc::tmem_ld16(col0 + (c + 1) * CW, nxt);
                    }
                    if constexpr (INDEXER) {
                        // one column per query: the raw indexer score
#pragma unroll
                        for (int e = 0; e < CW; ++e) acc[c * CW + e] = __uint_as_float(cur[e]);
                    } else {
                        const ulonglong2* nl = reinterpret_cast<const ulonglong2*>(
                            sLse + g * NQ + part * kCols + c * CW);
#pragma unroll
                        for (int c4 = 0; c4 < CW / 4; ++c4) {
                            const ulonglong2 L = nl[c4];
                            mass_columns4<G, kQP>(acc2, c * CW + c4 * 4, cur[c4 * 4],
                                                  cur[c4 * 4 + 1], cur[c4 * 4 + 2],
                                                  cur[c4 * 4 + 3], L.x, L.y, sl2x2,
                                                  (c4 & 1) != 0);
                        }
                    }
                    if (c + 1 < kCols / CW) tc::tmem_wait_ld(nxt);
                }
                tc::fence_before_sync();
                tc::mbar_arrive(&s_empty[slot]);
            }
            if (!ok) break;
            if constexpr (!INDEXER) {
#pragma unroll
                for (int q = 0; q < kQP; ++q) acc[q] = acc2.get(q);
            }
            const int j = kt * 128 + row;                     // key (or sample) index
            const int qp0 = q0 + part * kQP;                  // first query of this part
            if constexpr (STREAM) {
                // keys at or above the query's threshold, appended in key order to this
                // warp's segment (positions past the capacity are only counted); no
                // warp-uniform branch, so the queries' ballot chains interleave
                uint32_t lt;
                asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt));
                const bool below = j <= qbase;        // key at or before every query here
#pragma unroll
                for (int q = 0; q < kQP; ++q) {
                    const float v = INDEXER ? acc[q] : acc[q] * p.inv_hq;
                    const bool pass = q < qend && (below || j <= qbase + q) &&
                                      v >= sTau[part * kQP + q];
                    const uint32_t bal = __ballot_sync(0xffffffffu, pass);
                    const int pos = cnt[q] + __popc(bal & lt);
                    const uint32_t at = off0 + (uint32_t)q * qstride + (uint32_t)pos;
                    if (pass && pos < p.seg_cap &&
                        in_bounds(p.status, INDEXER ? KID_INDEXER_TC : KID_MASS_TC, kSiteCand, at,
                                  p.out_cap))
                        p.cand[at] = make_uint2(__float_as_uint(v), (uint32_t)j);
                    cnt[q] += __popc(bal);
                }
            } else if constexpr (!BLOCK) {
                // row i of the slab starts off(i) - off(row0) floats in (32-bit: the host
                // keeps a chunk's slab below 2^32 floats) and holds i / S + 1 values; the
                // offsets of this part's rows follow from the first one by adding
                // i / S + 1, so no division runs per key tile.  Lanes store consecutive
                // keys of one query; key j sits at position j S <= i iff j <= i / S.
                int a = qbase / p.kst, b = qbase - a * p.kst;   // first row's i / S, i % S
                uint32_t off = (uint32_t)(qbase + (int64_t)p.kst * ((int64_t)a * (a - 1) / 2) +
                                          (int64_t)a * b - slab0);
#pragma unroll
                for (int q = 0; q < kQP; ++q) {
                    if (j <= a && qbase + q < p.row1 &&
                        in_bounds(p.status, KID_MASS_TC, kSiteRows, off + (uint32_t)j, p.out_cap))
                        p.rows[off + (uint32_t)j] = INDEXER ? acc[q] : acc[q] * p.inv_hq;
                    off += (uint32_t)a + 1u;
                    if (++b == p.kst) { b = 0; ++a; }
                }
            } else {
                // block column sums of this part's queries, 2^-40 fixed point, one add
                // per (block, key, part)
                int cur_b = qp0 / p.block_q;
                float sum = 0.f;
#pragma unroll
                for (int q = 0; q < kQP; ++q) {
                    const int i = qp0 + q;
                    if (i < p.N) {
                        const int b = i / p.block_q;
                        if (b != cur_b) {
                            if (sum > 0.f)
                                block_mass_add(p, bmass_offset(cur_b, p.block_q) + j, sum);
                            sum = 0.f;
                            cur_b = b;
                        }
                        if (j <= i) sum += acc[q];
                    }
                }
                if (sum > 0.f) block_mass_add(p, bmass_offset(cur_b, p.block_q) + j, sum);
            }
        }
        if constexpr (STREAM) {
            if (ok && lane == 0) {
#pragma unroll
                for (int q = 0; q < kQP; ++q) {
                    const int64_t i = q0 + part * kQP + q;
                    if (i < p.row1) p.cnt[(i - p.row0) * 4 + quarter] = cnt[q];
                }
            }
        }
    }
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- block top-k
// One CTA per block: exact top-min(k, e_b+1) of the fixed-point block mass row
// (64-bit keys, 8 x 8-bit radix select), written ascending with the mass as fp32.
__global__ void __launch_bounds__(256) k_block_select(const unsigned long long* __restrict__ bmass,
                                                      int N, int block_q, int budget,
                                                      int32_t* __restrict__ sup_idx,
                                                      int32_t* __restrict__ sup_len,
                                                      float* __restrict__ sup_mass) {
    __shared__ int hist[256];
    __shared__ int warp_tot[33];
    __shared__ int s_digit, s_rem;
    const int b = blockIdx.x;
    const int n = min(N, (b + 1) * block_q);     // keys 0..e_b
    const unsigned long long* row = bmass + bmass_offset(b, block_q);
    const int tid = threadIdx.x, nt = blockDim.x;
    int32_t* oi = sup_idx + (size_t)b * budget;
    float* om = sup_mass + (size_t)b * budget;
    const bool all = n <= budget;
    unsigned long long T = 0;
    int take_eq = 0;
    if (!all) {
        unsigned long long prefix = 0, mask = 0;
        int remaining = budget;
        for (int shift = 56; shift >= 0; shift -= 8) {
            for (int x = tid; x < 256; x += nt) hist[x] = 0;
            __syncthreads();
            for (int j = tid; j < n; j += nt) {
                const unsigned long long key = row[j];
                if ((key & mask) == prefix) atomicAdd(&hist[(int)((key >> shift) & 255ull)], 1);
            }
            __syncthreads();
            if (tid == 0) {
                int cum = 0;
                for (int x = 255; x >= 0; --x) {
                    if (cum + hist[x] >= remaining) {
                        s_digit = x;
                        s_rem = remaining - cum;
                        break;
                    }
                    cum += hist[x];
                }
            }
            __syncthreads();
            prefix |= (unsigned long long)s_digit << shift;
            mask |= 255ull << shift;
            remaining = s_rem;
            __syncthreads();
        }
        T = prefix;
        take_eq = remaining;
    }
    int base_sel = 0, base_eq = 0;
    for (int j0 = 0; j0 < n; j0 += nt) {
        const int j = j0 + tid;
        unsigned long long key = 0;
        bool gt = false, eq = false;
        if (j < n) {
            key = row[j];
            gt = all || key > T;
            eq = !all && key == T;
        }
        int eq_tot, sel_tot;
        const int eq_excl = block_exclusive_scan(eq ? 1 : 0, warp_tot, &eq_tot);
        const bool sel = gt || (eq && base_eq + eq_excl < take_eq);
        const int sel_excl = block_exclusive_scan(sel ? 1 : 0, warp_tot, &sel_tot);
        if (sel) {
            oi[base_sel + sel_excl] = j;
            om[base_sel + sel_excl] = (float)((double)key * (1.0 / 1099511627776.0));
        }
        base_eq += eq_tot;
        base_sel += sel_tot;
    }
    const int m = min(n, budget);
    for (int t = m + tid; t < budget; t += nt) {
        oi[t] = -1;
        om[t] = 0.f;
    }
    if (tid == 0) sup_len[b] = m;
}

template <int G, int D, int NQ, int MODE, int KS>
cudaError_t launch_mass(const MassArgs& a, cudaStream_t st) {
    constexpr int BQ = NQ / G;
    constexpr bool BLOCK = MODE == kModeBlock;
    constexpr bool ROWS = MODE == kModeQuery || MODE == kModeIndexer;
    CUtensorMap tq, tk;
    const uint64_t d = a.d;
    // rows modes with a key stride read every S-th key row: the same K with an
    // S-fold longer row pitch and (N - 1) / S + 1 rows
    const int S = (ROWS && a.kst > 1) ? a.kst : 1;
    const uint64_t n_keys = (uint64_t)((a.N - 1) / S) + 1;
    if (!make_tmap_3d_bf16(&tq, a.q, d, a.Hq, a.N, d * 2, (uint64_t)a.Hq * d * 2, 64, G, BQ) ||
        !make_tmap_3d_bf16(&tk, a.k, d, a.Hkv, n_keys, d * 2, (uint64_t)a.Hkv * d * 2 * S, 64,
                           1, 128))
        return cudaErrorInvalidValue;
    MassParams p{};
    p.N = (int)a.N;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    // per query / indexer the launch covers the queries [row0, row1) (row0 a
    // multiple of BQ)
    const int64_t r0 = BLOCK ? 0 : a.row0, r1 = BLOCK ? a.N : a.row1;
    p.ct0 = (int)(r0 / BQ);
    p.n_ctiles = (int)((r1 + BQ - 1) / BQ) - p.ct0;
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
    if (p.n_ctiles <= 0) return cudaSuccess;
    const int smem = mass_smem_bytes(NQ, D, a.Hkv, KS);
    auto kern = k_mass_tc<G, D, NQ, MODE, KS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (BLOCK) {
        const int64_t nb = (a.N + a.block_q - 1) / a.block_q;
        e = cudaMemsetAsync(a.bmass, 0, (size_t)bmass_offset(nb, a.block_q) * 8, st);
        if (e != cudaSuccess) return e;
    }
    kern<<<(unsigned)p.n_ctiles, kThreads, smem, st>>>(tq, tk, p);
    note_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess || !BLOCK) return e;
    const int nb = (int)((a.N + a.block_q - 1) / a.block_q);
    k_block_select<<<nb, 256, 0, st>>>(p.bmass, p.N, a.block_q, a.budget, a.sup_idx, a.sup_len,
                                       a.sup_mass);
    note_launch();
    return cudaGetLastError();
}

// Only (G, NQ) pairs with 4..32 queries per CTA are instantiated (at d = 256, NQ <= 64:
// the wider Q of every group does not fit in shared memory beside the K ring).
template <int G, int D, int NQ, int MODE>
cudaError_t launch_if_valid(const MassArgs& a, cudaStream_t st) {
    if constexpr (NQ / G >= 4 && NQ / G <= 32 && (D < 256 || NQ <= 64)) {
        if constexpr (D == 256) {
            if (mass_smem_bytes(NQ, D, a.Hkv, 2) > kMaxDynSmem)
                return launch_mass<G, D, NQ, MODE, 1>(a, st);
        }
        return launch_mass<G, D, NQ, MODE, 2>(a, st);
    }
    else
        return cudaErrorNotSupported;
}

template <int D, int NQ, int MODE>
cudaError_t dispatch_g(const MassArgs& a, cudaStream_t st) {
    switch (a.Hq / a.Hkv) {
        case 1: return launch_if_valid<1, D, NQ, MODE>(a, st);
        case 2: return launch_if_valid<2, D, NQ, MODE>(a, st);
        case 4: return launch_if_valid<4, D, NQ, MODE>(a, st);
        case 8: return launch_if_valid<8, D, NQ, MODE>(a, st);
        case 16: return launch_if_valid<16, D, NQ, MODE>(a, st);
        default: return cudaErrorNotSupported;
    }
}

template <int D, int MODE>
cudaError_t dispatch_nq(const MassArgs& a, cudaStream_t st) {
    switch (tc_mass_columns(a)) {
        case 128: return dispatch_g<D, 128, MODE>(a, st);
        case 64: return dispatch_g<D, 64, MODE>(a, st);
        case 32: return dispatch_g<D, 32, MODE>(a, st);
        default: return cudaErrorNotSupported;
    }
}

template <int MODE>
cudaError_t dispatch(const MassArgs& a, cudaStream_t st) {
    switch (a.d) {
        case 64: return dispatch_nq<64, MODE>(a, st);
        case 128: return dispatch_nq<128, MODE>(a, st);
        default: return dispatch_nq<256, MODE>(a, st);
    }
}

// The indexer runs as a single-head problem: Hq = Hkv = 1, d = d_idx, 32 queries per CTA.
cudaError_t launch_indexer_tc(const MassArgs& a, cudaStream_t st) {
    if (a.stream)
        return a.d == 64 ? launch_mass<1, 64, 32, kModeIndexerStream, 2>(a, st)
                         : launch_mass<1, 128, 32, kModeIndexerStream, 2>(a, st);
    return a.d == 64 ? launch_mass<1, 64, 32, kModeIndexer, 2>(a, st)
                     : launch_mass<1, 128, 32, kModeIndexer, 2>(a, st);
}

}  // namespace

int tc_mass_columns(const MassArgs& a) {
    // NQ columns per group: 128 (twice the queries per CTA, half the K re-reads) when
    // the Q of all groups plus the rest of the layout fits in shared memory, else 64.
    const int G = a.Hq / a.Hkv;
    // (queries per CTA NQ/G kept within [4, 32] so the per-thread accumulators stay
    // in registers)
    if (a.Hkv > 64 || G < 1) return 0;
    for (int nq = a.d == 256 ? 64 : 128; nq >= 32; nq >>= 1) {
        const int bq = nq / G;
        if (bq < 4 || bq > 32) continue;
        if (mass_smem_bytes(nq, a.d, a.Hkv, a.d == 256 ? 1 : 2) <= kMaxDynSmem) return nq;
    }
    return 0;
}

bool tc_mass_supported(const MassArgs& a) {
    const int G = a.Hq / a.Hkv;
    const int nq = tc_mass_columns(a);
    if (a.dtype != TAM_BF16 || (a.d != 64 && a.d != 128 && a.d != 256) || nq == 0) return false;
    if (!(G == 1 || G == 2 || G == 4 || G == 8 || G == 16)) return false;
    if (a.block_q > 1 && a.block_q > (1 << 20)) return false;
    return true;
}

size_t tc_mass_block_bytes(int64_t N, int block_q) {
    const int64_t nb = (N + block_q - 1) / block_q;
    return (size_t)bmass_offset(nb, block_q) * 8;
}

cudaError_t tc_mass_pass(const MassArgs& a, cudaStream_t st) {
    if (pair_mass_supported(a) && !pair_path_disabled()) {
        cudaError_t e = pair_mass(a, st);
        if (e != cudaSuccess || a.block_q == 1) return e;
        const int nb = (int)((a.N + a.block_q - 1) / a.block_q);
        k_block_select<<<nb, 256, 0, st>>>(reinterpret_cast<unsigned long long*>(a.bmass), (int)a.N,
                                           a.block_q, a.budget, a.sup_idx, a.sup_len, a.sup_mass);
        note_launch();
        return cudaGetLastError();
    }
    if (a.block_q > 1) return dispatch<kModeBlock>(a, st);
    return a.stream ? dispatch<kModeQueryStream>(a, st) : dispatch<kModeQuery>(a, st);
}

int tc_mass_segments(const MassArgs& a) {
    return (pair_mass_supported(a) && !pair_path_disabled()) ? 8 : 4;
}

bool tc_indexer_supported(int64_t N, int d_idx, int dtype, int block_q) {
    return dtype == TAM_BF16 && (d_idx == 64 || d_idx == 128) && block_q == 1 && N >= 1;
}

cudaError_t tc_indexer_rows(const IndexerArgs& ia, cudaStream_t st) {
    MassArgs a{};
    a.N = ia.N;
    a.Hq = 1;
    a.Hkv = 1;
    a.d = ia.d_idx;
    a.dtype = ia.dtype;
    a.q = ia.q_idx;
    a.k = ia.k_idx;
    a.budget = ia.budget;
    a.block_q = 1;
    a.rows = ia.rows;
    a.row0 = ia.row0;
    a.row1 = ia.row1;
    a.kst = ia.kst;
    a.stream = ia.stream;
    a.tau = ia.tau;
    a.cand = ia.cand;
    a.cnt = ia.cnt;
    a.seg_cap = ia.seg_cap;
    a.out_cap = ia.out_cap;
    a.status = ia.status;
    return launch_indexer_tc(a, st);
}

}  // namespace tam
