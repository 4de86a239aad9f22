// Pass 3: attention recomputed on the selected support (bf16 inputs, fp32 softmax).
//
//   out[i,h] = sum_{j in T_i} softmax_{T_i}(scale * q[i,h].k[j,g(h)]) v[j,g(h)]
//
// (arXiv 2606.07703, Abstract: "recomputes attention only on that support";
// gist.science technical report §2.1 "Ausführung": original Q, K, V restricted to
// the selected tokens, softmax renormalised over them.)
//
// The work is a gather: every selected key costs one K row and one V row per KV
// group (2 x 256 B at d = 128) against only G = Hq/Hkv query heads, so the kernels
// stream rows through shared memory with cp.async (16-byte pieces, rows XOR-
// swizzled so ldmatrix reads are conflict-free, invalid slots zero-filled) and use
// warp-level mma.sync m16n8k16 for the two small products; the tensor pipe is far
// from the bound here, the memory system is.
//
// k_attn_gather   per query:     one warp per (query i, KV group g); the G heads are
//                                the rows of one 16-row MMA tile; keys in chunks of 16.
// k_attn_block    block-shared:  one CTA per (block, group, slice of 256 rows); the
//                                chunk of gathered rows is shared by 16 warps, each
//                                owning 16 (query, head) rows, causal mask j <= i.
#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "tma_host.h"

namespace tam {
namespace {

constexpr int kChunk = 16;    // keys per chunk
// per-query kernel: warps per CTA (one CTA per SM) and cp.async ring depth per warp
constexpr int kGatherWarps = 12, kGatherStages = 2;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    const int n = valid ? 16 : 0;   // n = 0 writes 16 zero bytes
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Byte offset of 16-byte piece `pc` of row `r` in a chunk buffer with RB-byte rows.
template <int RB>
__device__ __forceinline__ uint32_t swz(int r, int pc) {
    return (uint32_t)(r * RB + ((pc ^ (r & 7)) << 4));
}

// Issue the cp.async copies of one chunk (kChunk K rows then kChunk V rows of KV
// group g) into `buf`; `nthr` threads starting at `t0` cooperate.  Rows whose slot
// is past `n`, or whose key is outside [0, N), are zero-filled.
template <int D>
__device__ __forceinline__ void issue_chunk(uint32_t buf, const __nv_bfloat16* k,
                                            const __nv_bfloat16* v, int N, int Hkv, int g,
                                            const int32_t* srow, int t_base, int n, int tid,
                                            int nthr) {
    constexpr int RB = D * 2;
    constexpr int PC = RB / 16;
    constexpr int PIECES = kChunk * PC;   // per matrix
    for (int p = tid; p < 2 * PIECES; p += nthr) {
        const int mat = p / PIECES;          // 0 = K, 1 = V
        const int r = (p % PIECES) / PC, pc = p % PC;
        const int t = t_base + r;
        const int jr = t < n ? srow[t] : -1;
        const bool valid = (unsigned)jr < (unsigned)N;    // keys outside [0, N) are never read
        const int j = valid ? jr : 0;
        const __nv_bfloat16* src = (mat == 0 ? k : v) + ((size_t)j * Hkv + g) * D + pc * 8;
        cp_async16(buf + mat * kChunk * RB + swz<RB>(r, pc), src, valid);
    }
}

// Warp version of issue_chunk: the chunk's kChunk support indices are read once
// (one lane each) and broadcast; every lane keeps one 16-byte column `pc` of the
// rows and issues the K and V copies of each of its rows from one row offset.  Keys
// outside [0, jmax] (jmax = the query's position: negative, later or past the sequence)
// are not read; their rows are zero-filled.  Returns the chunk's valid slots as bits.
template <int D>
__device__ __forceinline__ uint32_t issue_chunk_warp(uint32_t buf, const __nv_bfloat16* k,
                                                     const __nv_bfloat16* v, int Hkv, int g,
                                                     const int32_t* srow, int t_base, int n,
                                                     int jmax, int tok0) {
    constexpr int RB = D * 2;
    constexpr int PC = RB / 16;          // 16-byte pieces per row
    constexpr int RPP = 32 / PC;         // rows covered by one pass of the warp
    const int lane = threadIdx.x & 31;
    const int pc = lane % PC, r0 = lane / PC;
    int jl = -1;
    if (lane < kChunk && t_base + lane < n) {
        const int j = srow[t_base + lane];
        jl = (unsigned)j <= (unsigned)jmax ? j : -1;
    }
    const uint32_t bits = __ballot_sync(0xffffffffu, jl >= 0);
#pragma unroll
    for (int u = 0; u < kChunk / RPP; ++u) {
        const int r = u * RPP + r0;
        const int j = __shfl_sync(0xffffffffu, jl, r);
        const bool valid = j >= 0;
        const size_t off = valid ? ((size_t)(tok0 + j) * Hkv + g) * D + pc * 8 : 0;
        const uint32_t dst = buf + swz<RB>(r, pc);
        cp_async16(dst, k + off, valid);
        cp_async16(dst + kChunk * RB, v + off, valid);
    }
    return bits;
}

// One chunk of keys for one 16-row MMA tile: S = Q K^T (2 n-tiles of 8 keys),
// masked online softmax (base 2), O += P V.  qa: A fragments of Q (a0..a3 per
// k-step).  valid(key slot r, row half) decides the mask.  ROW8: rows 8..15 live.
template <int D, bool ROW8, typename MaskFn>
__device__ __forceinline__ void chunk_step(uint32_t kbuf, const uint32_t (&qa)[D / 16][4],
                                           float sl2, float (&m)[2], float (&l)[2],
                                           float (&o)[D / 8][4], MaskFn valid) {
    constexpr int RB = D * 2;
    const int lane = threadIdx.x & 31;
    const int c = lane & 3;
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    // ldmatrix row address of this lane for the K tile (non-transposed B fragments)
    const int krow = ((lane >> 4) << 3) + (lane & 7);
    const int kpc = (lane >> 3) & 1;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kbuf + swz<RB>(krow, 2 * kk + kpc), b0, b1, b2, b3);
        mma16816(s[0], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
        mma16816(s[1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b2, b3);
    }
    // mask and scale to the log2 domain
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int r = nt * 8 + 2 * c + (e & 1);
            s[nt][e] = valid(r, e >> 1) ? s[nt][e] * sl2 : -INFINITY;
        }
    float p[2][4];
#pragma unroll
    for (int hf = 0; hf < (ROW8 ? 2 : 1); ++hf) {
        float mx = fmaxf(fmaxf(s[0][2 * hf], s[0][2 * hf + 1]), fmaxf(s[1][2 * hf], s[1][2 * hf + 1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(m[hf], mx);
        const float base = (m_new == -INFINITY) ? 0.f : m_new;
        // rescale only when some row of the warp raised its max (else every factor is 1)
        if (__any_sync(0xffffffffu, m_new != m[hf])) {
            const float corr = ex2f(m[hf] - base);
            l[hf] *= corr;
#pragma unroll
            for (int nd = 0; nd < D / 8; ++nd) {
                o[nd][2 * hf] *= corr;
                o[nd][2 * hf + 1] *= corr;
            }
        }
        m[hf] = m_new;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float pv = ex2f(s[nt][2 * hf + e] - base);
                p[nt][2 * hf + e] = pv;
                l[hf] += pv;
            }
    }
    if (!ROW8) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) p[nt][2] = p[nt][3] = 0.f;
    }
    const uint32_t a0 = pack_bf16(p[0][0], p[0][1]);
    const uint32_t a1 = pack_bf16(p[0][2], p[0][3]);
    const uint32_t a2 = pack_bf16(p[1][0], p[1][1]);
    const uint32_t a3 = pack_bf16(p[1][2], p[1][3]);
    // V tile: transposed fragments; matrix mi of x4 = (keys (mi&1)*8.., dims (nd+mi/2)*8..)
    const uint32_t vbuf = kbuf + kChunk * RB;
    const int vrow = ((lane >> 3) & 1) * 8 + (lane & 7);
    const int vdt = lane >> 4;
#pragma unroll
    for (int nd = 0; nd < D / 8; nd += 2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vbuf + swz<RB>(vrow, nd + vdt), b0, b1, b2, b3);
        mma16816(o[nd], a0, a1, a2, a3, b0, b1);
        mma16816(o[nd + 1], a0, a1, a2, a3, b2, b3);
    }
}

// Q A-fragments of the 16-row tile whose row r maps to query row pointer qrow(r)
// (null = zero row): a0 = row gq, cols 2c..; a1 = row gq+8; a2/a3 = cols +8.
template <int D, typename RowFn>
__device__ __forceinline__ void load_q_frags(uint32_t (&qa)[D / 16][4], RowFn qrow) {
    const int lane = threadIdx.x & 31;
    const int gq = lane >> 2, c = lane & 3;
    const __nv_bfloat16* r0 = qrow(gq);
    const __nv_bfloat16* r1 = qrow(gq + 8);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int col = kk * 16 + 2 * c;
        qa[kk][0] = r0 ? *reinterpret_cast<const uint32_t*>(r0 + col) : 0u;
        qa[kk][1] = r1 ? *reinterpret_cast<const uint32_t*>(r1 + col) : 0u;
        qa[kk][2] = r0 ? *reinterpret_cast<const uint32_t*>(r0 + col + 8) : 0u;
        qa[kk][3] = r1 ? *reinterpret_cast<const uint32_t*>(r1 + col + 8) : 0u;
    }
}

// Row sums across the 4 lanes of a row, then write rows < nrows of the tile.
template <int D, typename OutFn>
__device__ __forceinline__ void write_rows(const float (&m)[2], float (&l)[2],
                                           const float (&o)[D / 8][4], OutFn sink) {
    const int lane = threadIdx.x & 31;
    const int gq = lane >> 2, c = lane & 3;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        l[hf] += __shfl_xor_sync(0xffffffffu, l[hf], 1);
        l[hf] += __shfl_xor_sync(0xffffffffu, l[hf], 2);
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int row = gq + 8 * hf;
        const float inv = l[hf] > 0.f ? 1.f / l[hf] : 0.f;
        __nv_bfloat16* dst;
        float* lse_dst;
        if (!sink(row, dst, lse_dst)) continue;
#pragma unroll
        for (int nd = 0; nd < D / 8; ++nd)
            *reinterpret_cast<uint32_t*>(dst + nd * 8 + 2 * c) =
                pack_bf16(o[nd][2 * hf] * inv, o[nd][2 * hf + 1] * inv);
        if (lse_dst && c == 0)
            *lse_dst = l[hf] > 0.f ? (m[hf] + __log2f(l[hf])) * kLn2 : -INFINITY;
    }
}

// Key of slot t of a support row for the causal mask: the index when it is a key of the
// sequence, else INT32_MAX (never <= a query: the slot is skipped).
__device__ __forceinline__ int slot_key(const int32_t* row, int t, int n, int N) {
    const int j = t < n ? row[t] : -1;
    return (unsigned)j < (unsigned)N ? j : INT32_MAX;
}

// Number of leading entries of an ascending support row that are <= limit.
__device__ __forceinline__ int count_le(const int32_t* row, int n, int limit) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (row[mid] <= limit && row[mid] >= 0) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

// ---------------------------------------------------------------- per query
template <int D, int G, int STAGES, int W>
__global__ void __launch_bounds__(32 * W, 1)
k_attn_gather(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
              const __nv_bfloat16* __restrict__ v, const __grid_constant__ SeqTable seqs, int Hq,
              int Hkv, float sl2, const int32_t* __restrict__ sup_idx,
              const int32_t* __restrict__ sup_len, int kmax, int block_q,
              __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
    constexpr int RB = D * 2;
    constexpr int STAGE = 2 * kChunk * RB;
    constexpr bool ROW8 = G > 8;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const uint32_t wbuf = smem_addr(smem) + warp * STAGES * STAGE;
    // the table's rows (packed tokens); per query, selection row = token row
    const int rows = seqs.cu[seqs.n_seq] - seqs.cu[0];
    const int64_t total = (int64_t)rows * Hkv;
    for (int64_t item = (int64_t)blockIdx.x * W + warp; item < total; item += (int64_t)gridDim.x * W) {
        // KV groups in two halves when Hkv is even: all queries of the first half of the
        // groups, then the second, so that each half's K/V (67 MB at the 32K layer) stays
        // in L2 while it is gathered
        const int gh = (Hkv % 2 == 0) ? Hkv / 2 : Hkv;
        const int64_t per_half = (int64_t)rows * gh;
        const int64_t rem = item % per_half;
        const int i = seqs.cu[0] + (int)(rem / gh), g = (int)(item / per_half) * gh + (int)(rem % gh);
        // the query's sequence sq: keys are positions within it, from token tok0 on
        int sq = 0;
        if (seqs.n_seq > 1) {
            int hi = seqs.n_seq - 1;                  // the last s with cu[s] <= i
            while (sq < hi) {
                const int mid = (sq + hi + 1) >> 1;
                if (seqs.cu[mid] <= i) sq = mid;
                else hi = mid - 1;
            }
        }
        const int tok0 = seqs.cu[sq];
        const int32_t* srow;
        int n;
        if (block_q == 1) {
            srow = sup_idx + (size_t)i * kmax;
            n = min(sup_len[i], kmax);
        } else {
            const int b = (i - tok0) / block_q;
            srow = sup_idx + (size_t)b * kmax;
            n = count_le(srow, min(sup_len[b], kmax), i - tok0);
        }
        uint32_t qa[D / 16][4];
        load_q_frags<D>(qa, [&](int r) -> const __nv_bfloat16* {
            return r < G ? q + ((size_t)i * Hq + g * G + r) * D : nullptr;
        });
        float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
        float o[D / 8][4];
#pragma unroll
        for (int nd = 0; nd < D / 8; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
        static_assert(STAGES == 2, "one chunk in flight beside the one computed");
        const int nch = (n + kChunk - 1) / kChunk;
        const int jmax = i - tok0;                    // keys after the query are skipped
        uint32_t bits = 0;                            // valid slots of the chunk computed next
        if (nch > 0) bits = issue_chunk_warp<D>(wbuf, k, v, Hkv, g, srow, 0, n, jmax, tok0);
        cp_async_commit();
        for (int ch = 0; ch < nch; ++ch) {
            uint32_t next = 0;
            if (ch + 1 < nch)
                next = issue_chunk_warp<D>(wbuf + ((ch + 1) & 1) * STAGE, k, v, Hkv, g, srow,
                                           (ch + 1) * kChunk, n, jmax, tok0);
            cp_async_commit();
            cp_async_wait<1>();
            __syncwarp();
            chunk_step<D, ROW8>(wbuf + (ch & 1) * STAGE, qa, sl2, m, l, o,
                                [&](int r, int) { return (bits >> r) & 1u; });
            __syncwarp();
            bits = next;
        }
        cp_async_wait<0>();
        write_rows<D>(m, l, o, [&](int row, __nv_bfloat16*& dst, float*& ld) {
            if (row >= G) return false;
            const int h = g * G + row;
            dst = out + ((size_t)i * Hq + h) * D;
            const int len = seqs.cu[sq + 1] - tok0;
            ld = lse ? lse + (size_t)Hq * tok0 + (size_t)h * len + (i - tok0) : nullptr;
            return true;
        });
    }
}

// ---------------------------------------------------------------- block-shared
// CTA = (block b, group g, slice of 256 rows of the block's B_q x G rows).
template <int D, int G, int STAGES>
__global__ void __launch_bounds__(512, 1)
k_attn_block(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
             const __nv_bfloat16* __restrict__ v, int N, int Hq, int Hkv, float sl2,
             const int32_t* __restrict__ sup_idx, const int32_t* __restrict__ sup_len, int kmax,
             int block_q, int slices, __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
    constexpr int RB = D * 2;
    constexpr int STAGE = 2 * kChunk * RB;
    constexpr bool ROW8 = true;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const uint32_t buf0 = smem_addr(smem);
    const int b = blockIdx.x / slices, sl = blockIdx.x % slices;
    const int g = blockIdx.y;
    const int i0 = b * block_q;
    const int rows_in_block = (min(N, i0 + block_q) - i0) * G;
    const int row0 = sl * 256 + warp * 16;             // first tile row of this warp
    const int slice_last_row = min(rows_in_block, (sl + 1) * 256) - 1;
    if (sl * 256 >= rows_in_block) return;             // uniform for the CTA
    const int i_last = i0 + slice_last_row / G;        // last query of the slice
    const int32_t* srow = sup_idx + (size_t)b * kmax;
    const int n = count_le(srow, min(sup_len[b], kmax), i_last);
    const bool active = row0 < rows_in_block;
    uint32_t qa[D / 16][4];
    load_q_frags<D>(qa, [&](int r) -> const __nv_bfloat16* {
        const int rr = row0 + r;
        if (!active || rr >= rows_in_block) return nullptr;
        return q + ((size_t)(i0 + rr / G) * Hq + g * G + rr % G) * D;
    });
    const int lane = threadIdx.x & 31;
    const int qrow0 = i0 + (row0 + (lane >> 2)) / G;       // query of tile row gq
    const int qrow1 = i0 + (row0 + (lane >> 2) + 8) / G;   // query of tile row gq + 8
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    float o[D / 8][4];
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
    __shared__ int32_t s_idx[STAGES][kChunk];
    const int nch = (n + kChunk - 1) / kChunk;
#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) {
        if (s < nch) {
            issue_chunk<D>(buf0 + s * STAGE, k, v, N, Hkv, g, srow, s * kChunk, n, threadIdx.x, 512);
            if (threadIdx.x < kChunk) s_idx[s][threadIdx.x] = slot_key(srow, s * kChunk + (int)threadIdx.x, n, N);
        }
        cp_async_commit();
    }
    for (int ch = 0; ch < nch; ++ch) {
        const int nx = ch + STAGES - 1;
        if (nx < nch) {
            issue_chunk<D>(buf0 + (nx % STAGES) * STAGE, k, v, N, Hkv, g, srow, nx * kChunk, n,
                           threadIdx.x, 512);
            if (threadIdx.x < kChunk)
                s_idx[nx % STAGES][threadIdx.x] = slot_key(srow, nx * kChunk + (int)threadIdx.x, n, N);
        }
        cp_async_commit();
        cp_async_wait<STAGES - 1>();
        __syncthreads();
        const int32_t* keys = s_idx[ch % STAGES];
        if (active)
            chunk_step<D, ROW8>(buf0 + (ch % STAGES) * STAGE, qa, sl2, m, l, o,
                                [&](int r, int half) { return keys[r] <= (half ? qrow1 : qrow0); });
        __syncthreads();
    }
    cp_async_wait<0>();
    if (!active) return;
    write_rows<D>(m, l, o, [&](int row, __nv_bfloat16*& dst, float*& ld) {
        const int rr = row0 + row;
        if (rr >= rows_in_block) return false;
        const int i = i0 + rr / G, h = g * G + rr % G;
        dst = out + ((size_t)i * Hq + h) * D;
        ld = lse ? lse + (size_t)h * N + i : nullptr;
        return true;
    });
}

template <int D, int G>
cudaError_t launch_gather(const AttnArgs& a, cudaStream_t st) {
    // d = 256: six warps (a 32 KB ring each, and twice the registers per warp)
    constexpr int STAGES = kGatherStages, W = D == 256 ? 6 : kGatherWarps;
    constexpr int smem = W * STAGES * 2 * kChunk * D * 2;
    auto kern = k_attn_gather<D, G, STAGES, W>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int sms = 148;
    int dev;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return with_table(a.N, a.seqs, [&](SeqTable& t) {
        if (t.cu[t.n_seq] == t.cu[0]) return cudaSuccess;
        kern<<<sms, 32 * W, smem, st>>>((const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.k,
                                     (const __nv_bfloat16*)a.v, t, a.Hq, a.Hkv, a.sl2, a.sup_idx,
                                     a.sup_len, a.kmax, a.block_q, (__nv_bfloat16*)a.out, a.lse);
        note_launch();
        return cudaGetLastError();
    });
}

template <int D, int G>
cudaError_t launch_block(const AttnArgs& a, cudaStream_t st) {
    constexpr int STAGES = 3;
    constexpr int smem = STAGES * 2 * kChunk * D * 2;
    auto kern = k_attn_block<D, G, STAGES>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int nb = (int)((a.N + a.block_q - 1) / a.block_q);
    const int slices = (a.block_q * G + 255) / 256;
    dim3 grid((unsigned)(nb * slices), (unsigned)a.Hkv);
    kern<<<grid, 512, smem, st>>>((const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.k,
                                  (const __nv_bfloat16*)a.v, (int)a.N, a.Hq, a.Hkv, a.sl2,
                                  a.sup_idx, a.sup_len, a.kmax, a.block_q, slices,
                                  (__nv_bfloat16*)a.out, a.lse);
    note_launch();
    return cudaGetLastError();
}

template <int D>
cudaError_t dispatch(const AttnArgs& a, cudaStream_t st, bool block) {
    if constexpr (D == 256) {
        // one warp per (query, group) only: 16 warps of 256-wide accumulators do not fit
        switch (a.Hq / a.Hkv) {
            case 1: return launch_gather<D, 1>(a, st);
            case 2: return launch_gather<D, 2>(a, st);
            case 4: return launch_gather<D, 4>(a, st);
            case 8: return launch_gather<D, 8>(a, st);
            case 16: return launch_gather<D, 16>(a, st);
            default: return cudaErrorNotSupported;
        }
    } else {
        switch (a.Hq / a.Hkv) {
            case 1: return block ? launch_block<D, 1>(a, st) : launch_gather<D, 1>(a, st);
            case 2: return block ? launch_block<D, 2>(a, st) : launch_gather<D, 2>(a, st);
            case 4: return block ? launch_block<D, 4>(a, st) : launch_gather<D, 4>(a, st);
            case 8: return block ? launch_block<D, 8>(a, st) : launch_gather<D, 8>(a, st);
            case 16: return block ? launch_block<D, 16>(a, st) : launch_gather<D, 16>(a, st);
            default: return cudaErrorNotSupported;
        }
    }
}

}  // namespace

bool gather_supported(const AttnArgs& a) {
    const int G = a.Hq / a.Hkv;
    return a.dtype == TAM_BF16 && a.sup_idx != nullptr && (a.d == 64 || a.d == 128 || a.d == 256) &&
           (G == 1 || G == 2 || G == 4 || G == 8 || G == 16);
}

cudaError_t gather_attention(const AttnArgs& a, cudaStream_t st) {
    // block-shared supports: tcgen05 over gathered chunks where the query tiles fit the
    // blocks (attn_block_tc.cu), else the shared-chunk kernel when blocks have enough
    // rows, else one warp per (query, group)
    if (a.block_q > 1 && block_tc_supported(a) && !block_tc_disabled())
        return block_attention_tc(a, st);
    const bool block = a.block_q > 1 && (int64_t)a.block_q * (a.Hq / a.Hkv) >= 64;
    switch (a.d) {
        case 64: return dispatch<64>(a, st, block);
        case 128: return dispatch<128>(a, st, block);
        default: return dispatch<256>(a, st, false);
    }
}

}  // namespace tam
