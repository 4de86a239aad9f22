// C ABI of libtam.so: argument checks, workspace layout and kernel dispatch.
// Declarations and their contracts: include/tam.h.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>

#include "common.cuh"
#include "launch.h"
#include "tma_host.h"

using namespace tam;

namespace {
std::atomic<uint64_t> g_launches{0};
}  // namespace

void tam::note_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr int kMaxBudget = 4096;
constexpr int kSimtPersistentCtas = 1024;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
// Packed LSE of a whole batch ([Hq, N_s] per sequence) kept at the end of the workspace,
// with slack to start it on a 256-byte boundary.
inline size_t packed_lse_bytes(int64_t T, int Hq) { return align256((size_t)Hq * T * 4) + 256; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by every attention-shaped call.
int check_shape(int64_t N, int Hq, int Hkv, int d, int dtype) {
    if (N < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return TAM_ERR_INVALID_ARG;
    if (dtype != TAM_BF16 && dtype != TAM_F32) return TAM_ERR_INVALID_ARG;
    // bf16 runs on the tensor cores (d = 256 where its tiles fit), fp32 on the CUDA cores
    if (d != 64 && d != 128 && d != 256) return TAM_ERR_UNSUPPORTED;
    if (N >= (int64_t(1) << 31) - 1) return TAM_ERR_UNSUPPORTED;
    // the CUDA-core kernels stage one query row (all heads) in shared memory
    if ((size_t)(Hq * d + Hq) * sizeof(float) > 200 * 1024) return TAM_ERR_UNSUPPORTED;
    return TAM_OK;
}

int check_budget(int64_t N, int budget_k, int block_q) {
    if (budget_k < 1 || block_q < 1) return TAM_ERR_INVALID_ARG;
    if (budget_k > kMaxBudget) return TAM_ERR_UNSUPPORTED;
    if (N * (int64_t)budget_k >= (int64_t(1) << 31)) return TAM_ERR_UNSUPPORTED;
    return TAM_OK;
}

inline int64_t n_selection_units(int64_t N, int block_q) {
    return block_q == 1 ? N : (N + block_q - 1) / block_q;
}

// Per-query selection on the tensor cores (pass 2 and the indexer) streams: a sample
// pass scores every S-th key of each row and sets the row's threshold tau_i, then
// the scoring kernel keeps only the keys at or above tau_i, in fixed candidate
// segments, and an exact select runs over those; rows whose candidates fall short
// or overflow are recomputed whole on the CUDA cores.  Nothing of size N x N is
// written.  With TAM_MATERIALISE_ROWS=1 the rows are written instead, to a
// triangular slab, and selected from there (A/B comparisons).  Both forms run in
// chunks of queries sized by the workspace; chunks start at multiples of 64 queries
// (a multiple of every kernel's query tile).
constexpr size_t kSlabPrefBytes = size_t(4) << 30;
constexpr int64_t kChunkRows = 64;
constexpr int kMaxSamplesPerRow = 4096;   // sets the sample stride
constexpr float kTauSigmas = 5.f;         // margin of the sampled threshold
constexpr int kFallbackCtas = 148;

size_t slab_pref_bytes(int64_t N) {
    return std::min(kSlabPrefBytes, (size_t)tri(N) * sizeof(float));
}
size_t slab_min_bytes(int64_t N) {
    return (size_t)std::min(tri(N), kChunkRows * N) * sizeof(float);
}

// End of the chunk that starts at r0 (a multiple of 64) for a buffer of cap floats,
// where rows [r0, r1) take off(r1) - off(r0) floats (off non-decreasing, and 64 rows
// always fit): the whole rest if it fits, else the most 64-row steps that do.
template <class Off>
int64_t chunk_end_by(int64_t r0, int64_t N, int64_t cap, Off off) {
    if (off(N) - off(r0) <= cap) return N;
    int64_t lo = 1, hi = (N - r0) / kChunkRows + 1;
    while (hi - lo > 1) {
        const int64_t mid = (lo + hi) / 2;
        if (off(std::min(N, r0 + mid * kChunkRows)) - off(r0) <= cap) lo = mid; else hi = mid;
    }
    return std::min(N, r0 + lo * kChunkRows);
}

int64_t chunk_end(int64_t r0, int64_t N, int64_t cap) {
    return chunk_end_by(r0, N, cap, [](int64_t i) { return tri(i); });
}

// Layout and sizes of the streamed selection, after the caller's other regions:
//   tau [N] f32 | fallback list [1 + N] i32 | counts [N * nseg] i32 | region
// The region holds, one after the other, the sample rows of a chunk, the candidate
// segments of a chunk, and finally the fallback rows' scratch (or, materialised,
// the row slab of a chunk).
struct StreamPlan {
    bool materialise = false;     // rows written and selected instead (see below)
    int S = 1;                    // sample stride: every S-th key is scored
    int nseg = 0, seg_cap = 0;    // candidate segments per row and entries per segment
    int cap = 0;                  // nseg * seg_cap: rows of at most cap keys keep every key
    size_t off_tau = 0, off_fb = 0, off_cnt = 0, off_region = 0;
    size_t region_pref = 0, region_min = 0;
};

// Sample stride: the smallest prime of at least 17 that leaves at most
// kMaxSamplesPerRow sampled keys per row.  A prime stride does not line up with
// power-of-two structure in the key positions (a document or chunk grid, tokens
// planted every N/32 positions), which would put such keys in every row's sample.
int sample_stride(int64_t N) {
    int64_t S = std::max<int64_t>(17, (N + kMaxSamplesPerRow - 1) / kMaxSamplesPerRow);
    auto prime = [](int64_t x) {
        for (int64_t f = 2; f * f <= x; ++f)
            if (x % f == 0) return false;
        return true;
    };
    while (!prime(S) || ((N - 1) / S) + 1 > kMaxSamplesPerRow) ++S;
    return (int)S;
}

// Threshold rank r = ceil(mu + z sqrt(mu) + 4) of mu = k / S expected sampled keys
// at or above the k-th value; about S (r + 1) keys of a row then pass, and the
// segments hold half as many again (plus 32 each) before they overflow.
int segment_capacity(int budget, int S, int nseg) {
    const double mu = (double)budget / (double)S;
    const double r = std::ceil(mu + kTauSigmas * std::sqrt(mu) + 4.0);
    const double expect = (double)S * (r + 1.0);
    const int per = (int)std::ceil(1.5 * expect / nseg) + 32;
    return (per + 31) & ~31;
}

StreamPlan plan_stream(int64_t N, int budget, int nseg, size_t off) {
    StreamPlan sp;
    sp.S = sample_stride(N);
    sp.nseg = nseg;
    sp.seg_cap = segment_capacity(budget, sp.S, nseg);
    sp.cap = nseg * sp.seg_cap;
    sp.off_tau = off;
    sp.off_fb = sp.off_tau + align256((size_t)N * 4);
    sp.off_cnt = sp.off_fb + align256((size_t)(N + 1) * 4);
    sp.off_region = sp.off_cnt + align256((size_t)N * nseg * 4);
    const size_t samples_all = (size_t)sample_offset(N, sp.S) * 4;
    const size_t cand_all = (size_t)N * sp.cap * 8;
    const size_t fb_pref = (size_t)std::min<int64_t>(N, kFallbackCtas) * N * 4;
    sp.region_pref = std::max({samples_all, cand_all, fb_pref});
    // the select keeps a bitmap of the row's keys in shared memory: rows too long for it
    // (N beyond about 800K keys) are materialised and selected from the slab instead
    sp.materialise = materialise_rows() || cand_select_smem(N, sp.cap) > kCandSelectMaxSmem;
    if (sp.materialise) sp.region_pref = std::max(sp.region_pref, slab_pref_bytes(N));
    const int64_t s_max = (N - 1) / sp.S + 1;
    sp.region_min = std::max({(size_t)std::min<int64_t>(N, kChunkRows) * s_max * 4,
                              (size_t)std::min<int64_t>(N, kChunkRows) * sp.cap * 8,
                              slab_min_bytes(N)});
    return sp;
}

// The streamed per-query selection over a region of `region_bytes` (>= region_min).
// sample(r0, r1, S, slab) scores the sampled keys of rows [r0, r1) into slab;
// scan(c0, c1) writes the candidate segments and counts of rows [c0, c1) to the
// region; fallback(fb, scratch, n_ctas) redoes the listed rows.
template <class Sample, class Scan, class Fallback>
cudaError_t run_stream_select(const StreamPlan& sp, char* ws, size_t region_bytes, int64_t N,
                              int budget, int32_t* sup_idx, int32_t* sup_len, float* sup_val,
                              cudaStream_t st, Sample sample, Scan scan, Fallback fallback) {
    float* tau = (float*)(ws + sp.off_tau);
    int32_t* fb = (int32_t*)(ws + sp.off_fb);
    int32_t* cnt = (int32_t*)(ws + sp.off_cnt);
    char* region = ws + sp.off_region;
    cudaError_t e = cudaMemsetAsync(fb, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return e;
    // rows of at most cap keys keep every key: no samples needed below r_start
    const int64_t r_start = std::min<int64_t>(N, (sp.cap / kChunkRows) * kChunkRows);
    const int force = debug_force_fallback();
    if ((e = sample_tau(nullptr, 0, r_start, sp.S, budget, sp.cap, kTauSigmas, force, tau, st)))
        return e;
    const int S = sp.S;
    // slab offsets within a chunk are 32-bit in the scoring kernels
    const int64_t slab_cap = std::min<int64_t>((int64_t)(region_bytes / 4), (int64_t(1) << 32) - 1);
    for (int64_t r0 = r_start; r0 < N;) {
        const int64_t r1 = chunk_end_by(r0, N, slab_cap, [S](int64_t i) { return sample_offset(i, S); });
        if ((e = sample(r0, r1, S, (float*)region))) return e;
        if ((e = sample_tau((const float*)region, r0, r1, S, budget, sp.cap, kTauSigmas, force, tau,
                            st)))
            return e;
        r0 = r1;
    }
    // candidate offsets within a chunk are 32-bit in the scan kernels
    const int64_t fit = std::min<int64_t>((int64_t)(region_bytes / ((size_t)sp.cap * 8)),
                                          (int64_t(1) << 32) / sp.cap - kChunkRows);
    const int64_t rows_per_chunk = std::max<int64_t>(kChunkRows, fit / kChunkRows * kChunkRows);
    for (int64_t c0 = 0; c0 < N; c0 += rows_per_chunk) {
        const int64_t c1 = std::min(N, c0 + rows_per_chunk);
        if ((e = scan(c0, c1, tau, (void*)region, cnt))) return e;
        if ((e = cand_select(region, cnt, c0, c1, sp.nseg, sp.seg_cap, budget, sup_idx, sup_len,
                             sup_val, fb, st)))
            return e;
    }
    const int n_ctas = (int)std::min<int64_t>(
        {(int64_t)kFallbackCtas, N, (int64_t)(region_bytes / ((size_t)N * 4))});
    return fallback(fb, (float*)region, std::max(1, n_ctas));
}

// Workspace layout of tam_mass_oracle_prefill / tam_mass_select: status block, lse
// (when the caller passes none), then the pass-2 scratch of whichever kernel runs:
// the streamed selection (tensor cores, per query), fixed-point block mass (tensor
// cores, block-shared) or staged mass rows (CUDA cores).  `total` is the preferred
// size, `min_total` the smallest accepted (a smaller region only means more chunks).
struct MassPlan {
    size_t off_lse, off_work, total, min_total;
    bool tc, stream;
    int n_ctas;
    StreamPlan sp;
};

MassArgs mass_shape(int64_t N, int Hq, int Hkv, int d, int dtype, int budget_k, int block_q) {
    MassArgs a{};
    a.N = N; a.Hq = Hq; a.Hkv = Hkv; a.d = d; a.dtype = dtype;
    a.budget = budget_k; a.block_q = block_q;
    return a;
}

MassPlan plan_mass(int64_t N, int Hq, int Hkv, int d, int dtype, int budget_k, int block_q) {
    MassPlan p{};
    const int64_t n_sel = n_selection_units(N, block_q);
    const MassArgs shape = mass_shape(N, Hq, Hkv, d, dtype, budget_k, block_q);
    p.tc = tc_mass_supported(shape);
    p.n_ctas = (int)std::min<int64_t>(n_sel, kSimtPersistentCtas);
    p.stream = p.tc && block_q == 1;
    p.off_lse = kStatusBytes;
    p.off_work = p.off_lse + align256((size_t)Hq * N * sizeof(float));
    size_t work, min_work;
    if (!p.tc) {
        work = min_work = (size_t)p.n_ctas * N * sizeof(float);
    } else if (p.stream) {
        p.sp = plan_stream(N, budget_k, tc_mass_segments(shape), p.off_work);
        p.total = p.sp.off_region + align256(p.sp.region_pref);
        p.min_total = p.sp.off_region + align256(p.sp.region_min);
        return p;
    } else {
        work = min_work = tc_mass_block_bytes(N, block_q);
    }
    p.total = p.off_work + align256(work);
    p.min_total = p.off_work + align256(min_work);
    return p;
}

// Workspace of tam_indexer_topk: status block, then the streamed selection of the
// tensor-core path or the staged score rows of the CUDA-core path.
struct IndexerPlan {
    size_t off_scratch, total, min_total;
    bool tc;
    int n_ctas;
    StreamPlan sp;
};

IndexerPlan plan_indexer(int64_t N, int d_idx, int dtype, int budget_k, int block_q) {
    IndexerPlan p{};
    p.tc = tc_indexer_supported(N, d_idx, dtype, block_q);
    p.n_ctas = (int)std::min<int64_t>(N, kSimtPersistentCtas);
    p.off_scratch = kStatusBytes;
    if (p.tc) {
        p.sp = plan_stream(N, budget_k, kIndexerSegments, p.off_scratch);
        p.total = p.sp.off_region + align256(p.sp.region_pref);
        p.min_total = p.sp.off_region + align256(p.sp.region_min);
    } else {
        const size_t simt = (size_t)p.n_ctas * N * sizeof(float);
        p.total = p.min_total = p.off_scratch + align256(simt);
    }
    return p;
}

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? TAM_OK : TAM_ERR_CUDA; }

// Pass 3 with the gathered-row MMA kernels where built, else on the CUDA cores.
cudaError_t run_sparse_attention(const AttnArgs& a, cudaStream_t st) {
    return gather_supported(a) ? gather_attention(a, st) : simt_attention(a, st);
}

// Dense causal attention: the single-tile tensor-core kernel (128-key tiles), or with
// TAM_DENSE_PAIR_TILES=1 the block-shared pass-3 pipeline over all keys (two query
// tiles per CTA, 64-key chunks; measured 10 % slower at 32K, kept for A/B comparisons),
// or the CUDA cores for other shapes.
cudaError_t run_dense(const AttnArgs& a, cudaStream_t st) {
    if (dense_pair_tiles_supported(a) && dense_pair_tiles_selected()) return dense_pair_tiles(a, st);
    return tc_dense_supported(a) ? tc_dense(a, st) : simt_attention(a, st);
}

// Pass 1 on the tensor cores where the shape is built, else on the CUDA cores.
cudaError_t run_lse(const LseArgs& a, cudaStream_t st) {
    return tc_lse_supported(a) ? tc_lse(a, st) : simt_lse(a, st);
}

inline float score_log2_scale(int d) { return (float)(1.0 / std::sqrt((double)d)) * kLog2e; }

int start_call(void* workspace, cudaStream_t st) {
    return cuda_status(cudaMemsetAsync(workspace, 0, kStatusBytes, st));
}

// Pass 2 on an already computed lse, into the workspace laid out by plan_mass
// (ws_bytes >= plan.min_total).
int launch_mass_select(int64_t N, int Hq, int Hkv, int d, int dtype, const void* q, const void* k,
                       const float* lse, int budget_k, int block_q, int32_t* sup_idx,
                       int32_t* sup_len, float* sup_mass, char* ws, size_t ws_bytes,
                       const MassPlan& plan, cudaStream_t st, float sl2) {
    MassArgs ma = mass_shape(N, Hq, Hkv, d, dtype, budget_k, block_q);
    ma.q = q; ma.k = k; ma.lse = lse; ma.sl2 = sl2;
    ma.n_sel = (int)n_selection_units(N, block_q);
    ma.n_ctas = plan.n_ctas;
    ma.scratch = (float*)(ws + plan.off_work);
    ma.rows = (float*)(ws + plan.off_work);
    ma.bmass = ws + plan.off_work;
    ma.sup_idx = sup_idx; ma.sup_len = sup_len; ma.sup_mass = sup_mass;
    ma.status = (int32_t*)ws;
    if (!plan.tc) return cuda_status(simt_mass_select(ma, st));
    ma.out_cap = debug_extent((ws_bytes - plan.off_work) / 8);   // block mass (u64)
    if (!plan.stream) return cuda_status(tc_mass_pass(ma, st));
    const StreamPlan& sp = plan.sp;
    char* region = ws + sp.off_region;
    const size_t region_bytes = ws_bytes - sp.off_region;
    if (sp.materialise) {
        // mass rows of a chunk of queries, then their top-k, chunk by chunk
        const int64_t cap = std::min<int64_t>((int64_t)(region_bytes / sizeof(float)),
                                              (int64_t(1) << 32) - 1);   // 32-bit row offsets
        ma.rows = (float*)region;
        ma.out_cap = debug_extent((uint64_t)cap);
        for (int64_t r0 = 0; r0 < N;) {
            const int64_t r1 = chunk_end(r0, N, cap);
            ma.row0 = r0;
            ma.row1 = r1;
            cudaError_t e = tc_mass_pass(ma, st);
            if (e == cudaSuccess)
                e = row_topk(ma.rows, r0, r1, budget_k, sup_idx, sup_len, sup_mass, st);
            if (e != cudaSuccess) return TAM_ERR_CUDA;
            r0 = r1;
        }
        return TAM_OK;
    }
    auto sample = [&](int64_t r0, int64_t r1, int S, float* slab) {
        MassArgs a = ma;
        a.row0 = r0; a.row1 = r1; a.kst = S; a.rows = slab;
        a.out_cap = debug_extent(region_bytes / 4);
        return tc_mass_pass(a, st);
    };
    auto scan = [&](int64_t c0, int64_t c1, const float* tau, void* cand, int32_t* cnt) {
        MassArgs a = ma;
        a.row0 = c0; a.row1 = c1; a.stream = true; a.tau = tau; a.cand = cand; a.cnt = cnt;
        a.out_cap = debug_extent(region_bytes / 8);
        a.seg_cap = sp.seg_cap;
        return tc_mass_pass(a, st);
    };
    auto fallback = [&](const int32_t* fb, float* scratch, int n_ctas) {
        return fallback_mass_rows(ma, fb, scratch, n_ctas, st);
    };
    return cuda_status(run_stream_select(sp, ws, region_bytes, N, budget_k, sup_idx, sup_len,
                                         sup_mass, st, sample, scan, fallback));
}

// Null and alignment checks of the prefill entry points.
int check_prefill_ptrs(const void* q, const void* k, const void* v, const void* sup_idx,
                       const void* sup_len, const void* sup_mass, const void* lse,
                       const void* out, const void* workspace) {
    if (!q || !k || !sup_idx || !sup_len || !sup_mass || !workspace) return TAM_ERR_INVALID_ARG;
    if (out && !v) return TAM_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, sup_idx, sup_len, sup_mass, lse, out, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return TAM_ERR_INVALID_ARG;
    return TAM_OK;
}

// Passes 1-3 of one causal sequence of N tokens (the status block is already cleared).
int run_prefill(int64_t N, int Hq, int Hkv, int d, int dtype, const void* q, const void* k,
                const void* v, int budget_k, int block_q, int32_t* sup_idx, int32_t* sup_len,
                float* sup_mass, float* lse, void* out, char* ws, size_t ws_bytes,
                const MassPlan& plan, cudaStream_t st) {
    int32_t* status = (int32_t*)ws;
    float* lse_buf = lse ? lse : (float*)(ws + plan.off_lse);
    const float sl2 = score_log2_scale(d);
    int rc;
    LseArgs la{N, Hq, Hkv, d, dtype, q, k, sl2, lse_buf, status};
    if ((rc = cuda_status(run_lse(la, st)))) return rc;

    if ((rc = launch_mass_select(N, Hq, Hkv, d, dtype, q, k, lse_buf, budget_k, block_q, sup_idx,
                                 sup_len, sup_mass, ws, ws_bytes, plan, st, sl2)))
        return rc;

    if (out) {
        AttnArgs aa{N, Hq, Hkv, d, dtype, q, k, v, sl2, sup_idx, sup_len, budget_k, block_q,
                    out, nullptr, status};
        if ((rc = cuda_status(run_sparse_attention(aa, st)))) return rc;
    }
    return TAM_OK;
}

// Host-side cumulative lengths of a packed batch: cu[0] = 0, non-decreasing, total
// below 2^31 tokens.  Empty sequences are allowed.
int check_cu_seqlens(int n_seq, const int64_t* cu, int64_t* max_len) {
    if (n_seq < 1 || !cu || cu[0] != 0) return TAM_ERR_INVALID_ARG;
    int64_t mx = 0;
    for (int s = 0; s < n_seq; ++s) {
        const int64_t n = cu[s + 1] - cu[s];
        if (n < 0) return TAM_ERR_INVALID_ARG;
        mx = std::max(mx, n);
    }
    if (cu[n_seq] >= (int64_t(1) << 31) - 1) return TAM_ERR_UNSUPPORTED;
    *max_len = mx;
    return TAM_OK;
}

inline size_t elt_bytes(int dtype) { return dtype == TAM_F32 ? 4 : 2; }

// A packed batch as tables of up to kMaxSeqPerLaunch sequences (one launch per kernel
// each); tables of empty sequences only are skipped.
template <class F>
int for_seq_tables(int n_seq, const int64_t* cu, F&& fn) {
    for (int s0 = 0; s0 < n_seq; s0 += kMaxSeqPerLaunch) {
        SeqTable t{};
        t.n_seq = std::min(kMaxSeqPerLaunch, n_seq - s0);
        for (int s = 0; s <= t.n_seq; ++s) t.cu[s] = (int)cu[s0 + s];
        for (int s = 0; s < t.n_seq; ++s) t.max_len = std::max(t.max_len, t.cu[s + 1] - t.cu[s]);
        if (t.max_len == 0) continue;
        seq_table_order(t);
        const int rc = fn(t);
        if (rc) return rc;
    }
    return TAM_OK;
}

// Range checks of the indexer entry points (dtype and d_idx >= 1 checked by the caller).
int check_indexer_args(int64_t N, int d_idx, int dtype, int budget_k, int block_q) {
    if (d_idx != 16 && d_idx != 32 && d_idx != 64 && d_idx != 128) return TAM_ERR_UNSUPPORTED;
    if (N >= (int64_t(1) << 31) - 1) return TAM_ERR_UNSUPPORTED;
    int rc = check_budget(N, budget_k, block_q);
    if (rc) return rc;
    // block-shared: the indexer head runs as a one-head layer (tensor-core head dims)
    if (block_q > 1) return check_shape(N, 1, 1, d_idx, dtype);
    return TAM_OK;
}

int check_indexer_ptrs(const void* q_idx, const void* k_idx, const void* sup_idx,
                       const void* sup_len, const void* sup_score, const void* workspace) {
    if (!q_idx || !k_idx || !sup_idx || !sup_len || !sup_score || !workspace)
        return TAM_ERR_INVALID_ARG;
    const void* ptrs[] = {q_idx, k_idx, sup_idx, sup_len, sup_score, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return TAM_ERR_INVALID_ARG;
    return TAM_OK;
}

size_t indexer_min_bytes(int64_t N, int d_idx, int dtype, int budget_k, int block_q) {
    if (block_q > 1) return plan_mass(N, 1, 1, d_idx, dtype, budget_k, block_q).min_total;
    return plan_indexer(N, d_idx, dtype, budget_k, block_q).min_total;
}

// Indexer support of one sequence of N tokens (arguments checked, status cleared).
int run_indexer(int64_t N, int d_idx, int dtype, const void* q_idx, const void* k_idx,
                int budget_k, int block_q, int32_t* sup_idx, int32_t* sup_len, float* sup_score,
                char* ws, size_t ws_bytes, cudaStream_t st) {
    int rc;
    if (block_q > 1) {
        // Block-shared: softmax of the indexer scores per query (scale 1), summed over
        // the block, top-k of the sums: pass 1 and the block-mass pass 2 of a one-head
        // layer whose query and key are q_idx and k_idx.
        const MassPlan plan = plan_mass(N, 1, 1, d_idx, dtype, budget_k, block_q);
        float* lse_buf = (float*)(ws + plan.off_lse);
        LseArgs la{N, 1, 1, d_idx, dtype, q_idx, k_idx, kLog2e, lse_buf, (int32_t*)ws};
        if ((rc = cuda_status(run_lse(la, st)))) return rc;
        return launch_mass_select(N, 1, 1, d_idx, dtype, q_idx, k_idx, lse_buf, budget_k, block_q,
                                  sup_idx, sup_len, sup_score, ws, ws_bytes, plan, st, kLog2e);
    }
    const IndexerPlan plan = plan_indexer(N, d_idx, dtype, budget_k, block_q);
    IndexerArgs ia{};
    ia.N = N; ia.d_idx = d_idx; ia.dtype = dtype; ia.q_idx = q_idx; ia.k_idx = k_idx;
    ia.budget = budget_k; ia.n_ctas = plan.n_ctas; ia.scratch = (float*)(ws + plan.off_scratch);
    ia.rows = (float*)(ws + plan.off_scratch);
    ia.sup_idx = sup_idx; ia.sup_len = sup_len; ia.sup_score = sup_score;
    ia.status = (int32_t*)ws;
    if (!plan.tc) return cuda_status(simt_indexer_select(ia, st));
    const StreamPlan& sp = plan.sp;
    char* region = ws + sp.off_region;
    const size_t region_bytes = ws_bytes - sp.off_region;
    if (sp.materialise) {
        // score rows of a chunk of queries, then their top-k, chunk by chunk
        const int64_t cap = std::min<int64_t>((int64_t)(region_bytes / sizeof(float)),
                                              (int64_t(1) << 32) - 1);   // 32-bit row offsets
        ia.rows = (float*)region;
        ia.out_cap = debug_extent((uint64_t)cap);
        for (int64_t r0 = 0; r0 < N;) {
            const int64_t r1 = chunk_end(r0, N, cap);
            ia.row0 = r0;
            ia.row1 = r1;
            cudaError_t e = tc_indexer_rows(ia, st);
            if (e == cudaSuccess)
                e = row_topk(ia.rows, r0, r1, budget_k, sup_idx, sup_len, sup_score, st);
            if (e != cudaSuccess) return TAM_ERR_CUDA;
            r0 = r1;
        }
        return TAM_OK;
    }
    auto sample = [&](int64_t r0, int64_t r1, int S, float* slab) {
        IndexerArgs a = ia;
        a.row0 = r0; a.row1 = r1; a.kst = S; a.rows = slab;
        a.out_cap = debug_extent(region_bytes / 4);
        return tc_indexer_rows(a, st);
    };
    auto scan = [&](int64_t c0, int64_t c1, const float* tau, void* cand, int32_t* cnt) {
        IndexerArgs a = ia;
        a.row0 = c0; a.row1 = c1; a.stream = true; a.tau = tau; a.cand = cand; a.cnt = cnt;
        a.out_cap = debug_extent(region_bytes / 8);
        a.seg_cap = sp.seg_cap;
        return tc_indexer_rows(a, st);
    };
    auto fallback = [&](const int32_t* fb, float* scratch, int n_ctas) {
        return fallback_indexer_rows(ia, fb, scratch, n_ctas, st);
    };
    return cuda_status(run_stream_select(sp, ws, region_bytes, N, budget_k, sup_idx, sup_len,
                                         sup_score, st, sample, scan, fallback));
}

}  // namespace

extern "C" {

int tam_version(void) { return kVersion; }

uint64_t tam_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char* tam_status_string(int s) {
    switch (s) {
        case TAM_OK: return "ok";
        case TAM_ERR_INVALID_ARG: return "invalid argument";
        case TAM_ERR_UNSUPPORTED: return "unsupported shape or option";
        case TAM_ERR_WORKSPACE: return "workspace too small";
        case TAM_ERR_CUDA: return "CUDA error";
        case TAM_ERR_TIMEOUT: return "device wait timed out";
        case TAM_ERR_OVERFLOW: return "buffer overflow";
        default: return "unknown status";
    }
}

size_t tam_mass_oracle_workspace(int64_t N, int Hq, int Hkv, int d, int dtype, int budget_k,
                                 int block_q) {
    if (check_shape(N, Hq, Hkv, d, dtype) != TAM_OK) return 0;
    if (check_budget(N, budget_k, block_q) != TAM_OK) return 0;
    return plan_mass(N, Hq, Hkv, d, dtype, budget_k, block_q).total;
}

int tam_mass_oracle_prefill(int64_t N, int Hq, int Hkv, int d, int dtype, const void* q,
                            const void* k, const void* v, int budget_k, int block_q,
                            int32_t* sup_idx, int32_t* sup_len, float* sup_mass, float* lse,
                            void* out, void* workspace, size_t ws_bytes, void* stream) {
    int rc = check_shape(N, Hq, Hkv, d, dtype);
    if (rc) return rc;
    rc = check_budget(N, budget_k, block_q);
    if (rc) return rc;
    if ((rc = check_prefill_ptrs(q, k, v, sup_idx, sup_len, sup_mass, lse, out, workspace)))
        return rc;
    const MassPlan plan = plan_mass(N, Hq, Hkv, d, dtype, budget_k, block_q);
    if (ws_bytes < plan.min_total) return TAM_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    if ((rc = start_call(workspace, st))) return rc;
    return run_prefill(N, Hq, Hkv, d, dtype, q, k, v, budget_k, block_q, sup_idx, sup_len,
                       sup_mass, lse, out, (char*)workspace, ws_bytes, plan, st);
}

size_t tam_mass_oracle_workspace_varlen(int n_seq, const int64_t* cu_seqlens, int Hq, int Hkv,
                                        int d, int dtype, int budget_k, int block_q) {
    int64_t max_len = 0;
    if (check_cu_seqlens(n_seq, cu_seqlens, &max_len) != TAM_OK) return 0;
    if (check_shape(std::max<int64_t>(max_len, 1), Hq, Hkv, d, dtype) != TAM_OK) return 0;
    if (check_budget(std::max<int64_t>(max_len, 1), budget_k, block_q) != TAM_OK) return 0;
    size_t total = kStatusBytes;
    for (int s = 0; s < n_seq; ++s) {
        const int64_t n = cu_seqlens[s + 1] - cu_seqlens[s];
        if (n > 0) total = std::max(total, plan_mass(n, Hq, Hkv, d, dtype, budget_k, block_q).total);
    }
    // room for the packed LSE of the whole batch (used when the caller passes no lse)
    return total + packed_lse_bytes(cu_seqlens[n_seq], Hq);
}

int tam_mass_oracle_prefill_varlen(int n_seq, const int64_t* cu_seqlens, int Hq, int Hkv, int d,
                                   int dtype, const void* q, const void* k, const void* v,
                                   int budget_k, int block_q, int32_t* sup_idx, int32_t* sup_len,
                                   float* sup_mass, float* lse, void* out, void* workspace,
                                   size_t ws_bytes, void* stream) {
    int64_t max_len = 0;
    int rc = check_cu_seqlens(n_seq, cu_seqlens, &max_len);
    if (rc) return rc;
    if ((rc = check_shape(std::max<int64_t>(max_len, 1), Hq, Hkv, d, dtype))) return rc;
    if ((rc = check_budget(std::max<int64_t>(max_len, 1), budget_k, block_q))) return rc;
    if ((rc = check_prefill_ptrs(q, k, v, sup_idx, sup_len, sup_mass, lse, out, workspace)))
        return rc;
    if (ws_bytes < kStatusBytes) return TAM_ERR_WORKSPACE;
    const int64_t T = cu_seqlens[n_seq];
    const float sl2 = score_log2_scale(d);
    cudaStream_t st = (cudaStream_t)stream;
    const size_t qrow = (size_t)Hq * d * elt_bytes(dtype), krow = (size_t)Hkv * d * elt_bytes(dtype);
    LseArgs lall{T, Hq, Hkv, d, dtype, q, k, sl2, lse, (int32_t*)workspace};
    if (T > 0 && tc_lse_supported(lall)) {
        // Pass 1 of every sequence in one launch per table, into lse or (when the caller
        // passes none) the packed-LSE area at the end of the workspace; then pass 2 of each
        // sequence on its slice; then, for per-query supports, pass 3 of every sequence in
        // one launch per table.
        size_t ws2 = ws_bytes;
        if (!lse) {
            const size_t lb = packed_lse_bytes(T, Hq);
            if (ws_bytes < lb + kStatusBytes) return TAM_ERR_WORKSPACE;
            ws2 = (ws_bytes - lb) & ~size_t(255);
            lall.lse = (float*)((char*)workspace + ws2);
        }
        for (int s = 0; s < n_seq; ++s) {
            const int64_t n = cu_seqlens[s + 1] - cu_seqlens[s];
            if (n > 0 && ws2 < plan_mass(n, Hq, Hkv, d, dtype, budget_k, block_q).min_total)
                return TAM_ERR_WORKSPACE;
        }
        if ((rc = start_call(workspace, st))) return rc;
        rc = for_seq_tables(n_seq, cu_seqlens, [&](const SeqTable& t) {
            LseArgs la = lall;
            la.seqs = &t;
            return cuda_status(tc_lse(la, st));
        });
        if (rc) return rc;
        int64_t sel0 = 0;
        for (int s = 0; s < n_seq; ++s) {
            const int64_t t0 = cu_seqlens[s], n = cu_seqlens[s + 1] - t0;
            if (n == 0) continue;
            const MassPlan plan = plan_mass(n, Hq, Hkv, d, dtype, budget_k, block_q);
            rc = launch_mass_select(n, Hq, Hkv, d, dtype, (const char*)q + t0 * qrow,
                                    (const char*)k + t0 * krow, lall.lse + (size_t)Hq * t0,
                                    budget_k, block_q, sup_idx + sel0 * budget_k, sup_len + sel0,
                                    sup_mass + sel0 * budget_k, (char*)workspace, ws2, plan, st,
                                    sl2);
            if (rc) return rc;
            sel0 += n_selection_units(n, block_q);
        }
        if (!out) return TAM_OK;
        AttnArgs aall{T, Hq, Hkv, d, dtype, q, k, v, sl2, sup_idx, sup_len, budget_k, block_q,
                      out, nullptr, (int32_t*)workspace};
        if (block_q == 1 && gather_supported(aall))
            return for_seq_tables(n_seq, cu_seqlens, [&](const SeqTable& t) {
                AttnArgs aa = aall;
                aa.seqs = &t;
                return cuda_status(gather_attention(aa, st));
            });
        sel0 = 0;
        for (int s = 0; s < n_seq; ++s) {
            const int64_t t0 = cu_seqlens[s], n = cu_seqlens[s + 1] - t0;
            if (n == 0) continue;
            AttnArgs aa{n, Hq, Hkv, d, dtype, (const char*)q + t0 * qrow,
                        (const char*)k + t0 * krow, (const char*)v + t0 * krow, sl2,
                        sup_idx + sel0 * budget_k, sup_len + sel0, budget_k, block_q,
                        (char*)out + t0 * qrow, nullptr, (int32_t*)workspace};
            if ((rc = cuda_status(run_sparse_attention(aa, st)))) return rc;
            sel0 += n_selection_units(n, block_q);
        }
        return TAM_OK;
    }
    for (int s = 0; s < n_seq; ++s) {
        const int64_t n = cu_seqlens[s + 1] - cu_seqlens[s];
        if (n > 0 && ws_bytes < plan_mass(n, Hq, Hkv, d, dtype, budget_k, block_q).min_total)
            return TAM_ERR_WORKSPACE;
    }
    if ((rc = start_call(workspace, st))) return rc;
    // CUDA-core shapes: each sequence runs the single-sequence path on its slice of the
    // packed tensors, one after another on `stream`, reusing the workspace (stream order
    // separates them).
    int64_t sel0 = 0;
    for (int s = 0; s < n_seq; ++s) {
        const int64_t t0 = cu_seqlens[s], n = cu_seqlens[s + 1] - t0;
        if (n == 0) continue;
        const MassPlan plan = plan_mass(n, Hq, Hkv, d, dtype, budget_k, block_q);
        rc = run_prefill(n, Hq, Hkv, d, dtype, (const char*)q + t0 * qrow,
                         (const char*)k + t0 * krow, v ? (const char*)v + t0 * krow : nullptr,
                         budget_k, block_q, sup_idx + sel0 * budget_k, sup_len + sel0,
                         sup_mass + sel0 * budget_k, lse ? lse + (size_t)Hq * t0 : nullptr,
                         out ? (char*)out + t0 * qrow : nullptr, (char*)workspace, ws_bytes, plan,
                         st);
        if (rc) return rc;
        sel0 += n_selection_units(n, block_q);
    }
    return TAM_OK;
}

size_t tam_mass_workspace_min(int64_t N, int Hq, int Hkv, int d, int dtype, int budget_k,
                              int block_q) {
    if (check_shape(N, Hq, Hkv, d, dtype) != TAM_OK) return 0;
    if (check_budget(N, budget_k, block_q) != TAM_OK) return 0;
    return plan_mass(N, Hq, Hkv, d, dtype, budget_k, block_q).min_total;
}

size_t tam_attention_lse_workspace(int64_t N, int Hq, int Hkv, int d, int dtype) {
    if (check_shape(N, Hq, Hkv, d, dtype) != TAM_OK) return 0;
    return kStatusBytes;
}

int tam_attention_lse(int64_t N, int Hq, int Hkv, int d, int dtype, const void* q, const void* k,
                      float* lse, void* workspace, size_t ws_bytes, void* stream) {
    int rc = check_shape(N, Hq, Hkv, d, dtype);
    if (rc) return rc;
    if (!q || !k || !lse || !workspace) return TAM_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, lse, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return TAM_ERR_INVALID_ARG;
    if (ws_bytes < kStatusBytes) return TAM_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    if ((rc = start_call(workspace, st))) return rc;
    LseArgs la{N, Hq, Hkv, d, dtype, q, k, score_log2_scale(d), lse, (int32_t*)workspace};
    return cuda_status(run_lse(la, st));
}

size_t tam_mass_select_workspace(int64_t N, int Hq, int Hkv, int d, int dtype, int budget_k,
                                 int block_q) {
    return tam_mass_oracle_workspace(N, Hq, Hkv, d, dtype, budget_k, block_q);
}

int tam_mass_select(int64_t N, int Hq, int Hkv, int d, int dtype, const void* q, const void* k,
                    const float* lse, int budget_k, int block_q, int32_t* sup_idx,
                    int32_t* sup_len, float* sup_mass, void* workspace, size_t ws_bytes,
                    void* stream) {
    int rc = check_shape(N, Hq, Hkv, d, dtype);
    if (rc) return rc;
    rc = check_budget(N, budget_k, block_q);
    if (rc) return rc;
    if (!q || !k || !lse || !sup_idx || !sup_len || !sup_mass || !workspace)
        return TAM_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, lse, sup_idx, sup_len, sup_mass, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return TAM_ERR_INVALID_ARG;
    const MassPlan plan = plan_mass(N, Hq, Hkv, d, dtype, budget_k, block_q);
    if (ws_bytes < plan.min_total) return TAM_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    if ((rc = start_call(workspace, st))) return rc;
    return launch_mass_select(N, Hq, Hkv, d, dtype, q, k, lse, budget_k, block_q, sup_idx, sup_len,
                              sup_mass, (char*)workspace, ws_bytes, plan, st, score_log2_scale(d));
}

size_t tam_indexer_workspace(int64_t N, int d_idx, int dtype, int budget_k, int block_q) {
    if (N < 1 || d_idx < 1 || (dtype != TAM_BF16 && dtype != TAM_F32)) return 0;
    if (check_indexer_args(N, d_idx, dtype, budget_k, block_q) != TAM_OK) return 0;
    // block-shared: the indexer head as a one-head layer (lse, block mass)
    if (block_q > 1) return plan_mass(N, 1, 1, d_idx, dtype, budget_k, block_q).total;
    return plan_indexer(N, d_idx, dtype, budget_k, block_q).total;
}

size_t tam_indexer_workspace_min(int64_t N, int d_idx, int dtype, int budget_k, int block_q) {
    if (tam_indexer_workspace(N, d_idx, dtype, budget_k, block_q) == 0) return 0;
    return indexer_min_bytes(N, d_idx, dtype, budget_k, block_q);
}

int tam_indexer_topk(int64_t N, int d_idx, int dtype, const void* q_idx, const void* k_idx,
                     int budget_k, int block_q, int32_t* sup_idx, int32_t* sup_len,
                     float* sup_score, void* workspace, size_t ws_bytes, void* stream) {
    if (N < 1 || d_idx < 1 || (dtype != TAM_BF16 && dtype != TAM_F32)) return TAM_ERR_INVALID_ARG;
    int rc = check_indexer_args(N, d_idx, dtype, budget_k, block_q);
    if (rc) return rc;
    if ((rc = check_indexer_ptrs(q_idx, k_idx, sup_idx, sup_len, sup_score, workspace))) return rc;
    if (ws_bytes < indexer_min_bytes(N, d_idx, dtype, budget_k, block_q)) return TAM_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    if ((rc = start_call(workspace, st))) return rc;
    return run_indexer(N, d_idx, dtype, q_idx, k_idx, budget_k, block_q, sup_idx, sup_len,
                       sup_score, (char*)workspace, ws_bytes, st);
}

size_t tam_indexer_workspace_varlen(int n_seq, const int64_t* cu_seqlens, int d_idx, int dtype,
                                    int budget_k, int block_q) {
    int64_t max_len = 0;
    if (check_cu_seqlens(n_seq, cu_seqlens, &max_len) != TAM_OK) return 0;
    if (d_idx < 1 || (dtype != TAM_BF16 && dtype != TAM_F32)) return 0;
    if (check_indexer_args(std::max<int64_t>(max_len, 1), d_idx, dtype, budget_k, block_q)) return 0;
    size_t total = kStatusBytes;
    for (int s = 0; s < n_seq; ++s) {
        const int64_t n = cu_seqlens[s + 1] - cu_seqlens[s];
        if (n > 0) total = std::max(total, tam_indexer_workspace(n, d_idx, dtype, budget_k, block_q));
    }
    return total;
}

int tam_indexer_topk_varlen(int n_seq, const int64_t* cu_seqlens, int d_idx, int dtype,
                            const void* q_idx, const void* k_idx, int budget_k, int block_q,
                            int32_t* sup_idx, int32_t* sup_len, float* sup_score, void* workspace,
                            size_t ws_bytes, void* stream) {
    int64_t max_len = 0;
    int rc = check_cu_seqlens(n_seq, cu_seqlens, &max_len);
    if (rc) return rc;
    if (d_idx < 1 || (dtype != TAM_BF16 && dtype != TAM_F32)) return TAM_ERR_INVALID_ARG;
    if ((rc = check_indexer_args(std::max<int64_t>(max_len, 1), d_idx, dtype, budget_k, block_q)))
        return rc;
    if ((rc = check_indexer_ptrs(q_idx, k_idx, sup_idx, sup_len, sup_score, workspace))) return rc;
    if (ws_bytes < kStatusBytes) return TAM_ERR_WORKSPACE;
    for (int s = 0; s < n_seq; ++s) {
        const int64_t n = cu_seqlens[s + 1] - cu_seqlens[s];
        if (n > 0 && ws_bytes < indexer_min_bytes(n, d_idx, dtype, budget_k, block_q))
            return TAM_ERR_WORKSPACE;
    }
    cudaStream_t st = (cudaStream_t)stream;
    if ((rc = start_call(workspace, st))) return rc;
    const size_t row = (size_t)d_idx * elt_bytes(dtype);
    int64_t sel0 = 0;
    for (int s = 0; s < n_seq; ++s) {
        const int64_t t0 = cu_seqlens[s], n = cu_seqlens[s + 1] - t0;
        if (n == 0) continue;
        rc = run_indexer(n, d_idx, dtype, (const char*)q_idx + t0 * row,
                         (const char*)k_idx + t0 * row, budget_k, block_q,
                         sup_idx + sel0 * budget_k, sup_len + sel0, sup_score + sel0 * budget_k,
                         (char*)workspace, ws_bytes, st);
        if (rc) return rc;
        sel0 += n_selection_units(n, block_q);
    }
    return TAM_OK;
}

namespace {
// Workspace of tam_distill_kl: status block, then two row slabs of equal size (mass
// rows of the layer, score rows of the indexer) for a chunk of queries.
struct KlPlan {
    size_t off_slab, total, min_total;
    bool ok;
};

KlPlan plan_kl(int64_t N, int Hq, int Hkv, int d, int dtype, int d_idx) {
    KlPlan p{};
    MassArgs a = mass_shape(N, Hq, Hkv, d, dtype, 1, 1);
    p.ok = tc_mass_supported(a) && tc_indexer_supported(N, d_idx, dtype, 1);
    p.off_slab = kStatusBytes;
    p.total = p.off_slab + 2 * align256(slab_pref_bytes(N));
    p.min_total = p.off_slab + 2 * align256(slab_min_bytes(N));
    return p;
}
}  // namespace

size_t tam_distill_kl_workspace(int64_t N, int Hq, int Hkv, int d, int dtype, int d_idx) {
    if (check_shape(N, Hq, Hkv, d, dtype) != TAM_OK) return 0;
    const KlPlan p = plan_kl(N, Hq, Hkv, d, dtype, d_idx);
    return p.ok ? p.total : 0;
}

size_t tam_distill_kl_workspace_min(int64_t N, int Hq, int Hkv, int d, int dtype, int d_idx) {
    if (tam_distill_kl_workspace(N, Hq, Hkv, d, dtype, d_idx) == 0) return 0;
    return plan_kl(N, Hq, Hkv, d, dtype, d_idx).min_total;
}

int tam_distill_kl(int64_t N, int Hq, int Hkv, int d, int dtype, const void* q, const void* k,
                   const float* lse, int d_idx, const void* q_idx, const void* k_idx, float* kl,
                   void* workspace, size_t ws_bytes, void* stream) {
    int rc = check_shape(N, Hq, Hkv, d, dtype);
    if (rc) return rc;
    if (!q || !k || !lse || !q_idx || !k_idx || !kl || !workspace) return TAM_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, lse, q_idx, k_idx, kl, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return TAM_ERR_INVALID_ARG;
    const KlPlan plan = plan_kl(N, Hq, Hkv, d, dtype, d_idx);
    if (!plan.ok) return TAM_ERR_UNSUPPORTED;
    if (ws_bytes < plan.min_total) return TAM_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    if ((rc = start_call(workspace, st))) return rc;
    // two slabs of equal size share what follows the status block
    const size_t half = ((ws_bytes - plan.off_slab) / 2) & ~size_t(255);
    float* mass_rows = (float*)(ws + plan.off_slab);
    float* score_rows = (float*)(ws + plan.off_slab + half);
    MassArgs ma = mass_shape(N, Hq, Hkv, d, dtype, 1, 1);
    ma.q = q; ma.k = k; ma.lse = lse; ma.sl2 = score_log2_scale(d);
    ma.n_sel = (int)N;
    ma.rows = mass_rows;
    ma.status = (int32_t*)ws;
    IndexerArgs ia{};
    ia.N = N; ia.d_idx = d_idx; ia.dtype = dtype; ia.q_idx = q_idx; ia.k_idx = k_idx;
    ia.budget = 1; ia.rows = score_rows; ia.status = (int32_t*)ws;
    const int64_t cap = std::min<int64_t>((int64_t)(half / sizeof(float)),
                                          (int64_t(1) << 32) - 1);       // 32-bit row offsets
    ma.out_cap = ia.out_cap = debug_extent((uint64_t)cap);
    for (int64_t r0 = 0; r0 < N;) {
        const int64_t r1 = chunk_end(r0, N, cap);
        ma.row0 = ia.row0 = r0;
        ma.row1 = ia.row1 = r1;
        cudaError_t e = tc_mass_pass(ma, st);
        if (e == cudaSuccess) e = tc_indexer_rows(ia, st);
        if (e == cudaSuccess) e = row_kl(mass_rows, score_rows, r0, r1, kl, st);
        if (e != cudaSuccess) return TAM_ERR_CUDA;
        r0 = r1;
    }
    return TAM_OK;
}

int tam_support_mass_curve(int64_t n_rows, int kmax, const float* sup_val, const int32_t* sup_len,
                           const int32_t* budgets, int n_budgets, float* out, void* stream) {
    if (n_rows < 0 || kmax < 1 || !budgets || n_budgets < 1) return TAM_ERR_INVALID_ARG;
    if (kmax > kMaxBudget || n_budgets > kMaxSweepBudgets) return TAM_ERR_UNSUPPORTED;
    for (int t = 0; t < n_budgets; ++t)
        if (budgets[t] < 1) return TAM_ERR_INVALID_ARG;
    if (n_rows == 0) return TAM_OK;
    if (!sup_val || !sup_len || !out) return TAM_ERR_INVALID_ARG;
    const void* ptrs[] = {sup_val, sup_len, out};
    for (const void* p : ptrs)
        if (!aligned16(p)) return TAM_ERR_INVALID_ARG;
    return cuda_status(support_mass_curve(sup_val, sup_len, n_rows, kmax, budgets, n_budgets, out,
                                          (cudaStream_t)stream));
}

size_t tam_sparse_attention_workspace(int64_t N, int Hq, int Hkv, int d, int dtype) {
    if (check_shape(N, Hq, Hkv, d, dtype) != TAM_OK) return 0;
    return kStatusBytes;
}

int tam_sparse_support_attention(int64_t N, int Hq, int Hkv, int d, int dtype, const void* q,
                                 const void* k, const void* v, const int32_t* sup_idx,
                                 const int32_t* sup_len, int kmax, int block_q, void* out,
                                 float* lse, void* workspace, size_t ws_bytes, void* stream) {
    int rc = check_shape(N, Hq, Hkv, d, dtype);
    if (rc) return rc;
    rc = check_budget(N, kmax, block_q);
    if (rc) return rc;
    if (!q || !k || !v || !sup_idx || !sup_len || !out || !workspace) return TAM_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, sup_idx, sup_len, out, lse, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return TAM_ERR_INVALID_ARG;
    if (ws_bytes < kStatusBytes) return TAM_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    if ((rc = start_call(workspace, st))) return rc;
    AttnArgs aa{N, Hq, Hkv, d, dtype, q, k, v, score_log2_scale(d), sup_idx, sup_len, kmax,
                block_q, out, lse, (int32_t*)workspace};
    return cuda_status(run_sparse_attention(aa, st));
}

int tam_sparse_support_attention_varlen(int n_seq, const int64_t* cu_seqlens, int Hq, int Hkv,
                                        int d, int dtype, const void* q, const void* k,
                                        const void* v, const int32_t* sup_idx,
                                        const int32_t* sup_len, int kmax, int block_q, void* out,
                                        float* lse, void* workspace, size_t ws_bytes,
                                        void* stream) {
    int64_t max_len = 0;
    int rc = check_cu_seqlens(n_seq, cu_seqlens, &max_len);
    if (rc) return rc;
    if ((rc = check_shape(std::max<int64_t>(max_len, 1), Hq, Hkv, d, dtype))) return rc;
    if ((rc = check_budget(std::max<int64_t>(max_len, 1), kmax, block_q))) return rc;
    if (!q || !k || !v || !sup_idx || !sup_len || !out || !workspace) return TAM_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, sup_idx, sup_len, out, lse, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return TAM_ERR_INVALID_ARG;
    if (ws_bytes < kStatusBytes) return TAM_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    if ((rc = start_call(workspace, st))) return rc;
    const size_t qrow = (size_t)Hq * d * elt_bytes(dtype), krow = (size_t)Hkv * d * elt_bytes(dtype);
    // per-query supports: every sequence in one launch per table
    AttnArgs aall{cu_seqlens[n_seq], Hq, Hkv, d, dtype, q, k, v, score_log2_scale(d), sup_idx,
                  sup_len, kmax, block_q, out, lse, (int32_t*)workspace};
    if (block_q == 1 && gather_supported(aall))
        return for_seq_tables(n_seq, cu_seqlens, [&](const SeqTable& t) {
            AttnArgs aa = aall;
            aa.seqs = &t;
            return cuda_status(gather_attention(aa, st));
        });
    int64_t sel0 = 0;
    for (int s = 0; s < n_seq; ++s) {
        const int64_t t0 = cu_seqlens[s], n = cu_seqlens[s + 1] - t0;
        if (n == 0) continue;
        AttnArgs aa{n, Hq, Hkv, d, dtype, (const char*)q + t0 * qrow, (const char*)k + t0 * krow,
                    (const char*)v + t0 * krow, score_log2_scale(d), sup_idx + sel0 * kmax,
                    sup_len + sel0, kmax, block_q, (char*)out + t0 * qrow,
                    lse ? lse + (size_t)Hq * t0 : nullptr, (int32_t*)workspace};
        if ((rc = cuda_status(run_sparse_attention(aa, st)))) return rc;
        sel0 += n_selection_units(n, block_q);
    }
    return TAM_OK;
}

size_t tam_dense_workspace(int64_t N, int Hq, int Hkv, int d, int dtype) {
    if (check_shape(N, Hq, Hkv, d, dtype) != TAM_OK) return 0;
    return kStatusBytes;
}

int tam_dense_gqa_prefill(int64_t N, int Hq, int Hkv, int d, int dtype, const void* q,
                          const void* k, const void* v, void* out, float* lse, void* workspace,
                          size_t ws_bytes, void* stream) {
    int rc = check_shape(N, Hq, Hkv, d, dtype);
    if (rc) return rc;
    if (!q || !k || !v || !out || !workspace) return TAM_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, out, lse, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return TAM_ERR_INVALID_ARG;
    if (ws_bytes < kStatusBytes) return TAM_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    if ((rc = start_call(workspace, st))) return rc;
    AttnArgs aa{N, Hq, Hkv, d, dtype, q, k, v, score_log2_scale(d), nullptr, nullptr, 0, 1,
                out, lse, (int32_t*)workspace};
    return cuda_status(run_dense(aa, st));
}

int tam_dense_gqa_prefill_varlen(int n_seq, const int64_t* cu_seqlens, int Hq, int Hkv, int d,
                                 int dtype, const void* q, const void* k, const void* v,
                                 void* out, float* lse, void* workspace, size_t ws_bytes,
                                 void* stream) {
    int64_t max_len = 0;
    int rc = check_cu_seqlens(n_seq, cu_seqlens, &max_len);
    if (rc) return rc;
    if ((rc = check_shape(std::max<int64_t>(max_len, 1), Hq, Hkv, d, dtype))) return rc;
    if (!q || !k || !v || !out || !workspace) return TAM_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, out, lse, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return TAM_ERR_INVALID_ARG;
    if (ws_bytes < kStatusBytes) return TAM_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    if ((rc = start_call(workspace, st))) return rc;
    const size_t qrow = (size_t)Hq * d * elt_bytes(dtype), krow = (size_t)Hkv * d * elt_bytes(dtype);
    // tensor-core shapes: every sequence in one launch per table
    AttnArgs aall{cu_seqlens[n_seq], Hq, Hkv, d, dtype, q, k, v, score_log2_scale(d), nullptr,
                  nullptr, 0, 1, out, lse, (int32_t*)workspace};
    if (tc_dense_supported(aall))
        return for_seq_tables(n_seq, cu_seqlens, [&](const SeqTable& t) {
            AttnArgs aa = aall;
            aa.seqs = &t;
            return cuda_status(tc_dense(aa, st));
        });
    for (int s = 0; s < n_seq; ++s) {
        const int64_t t0 = cu_seqlens[s], n = cu_seqlens[s + 1] - t0;
        if (n == 0) continue;
        AttnArgs aa{n, Hq, Hkv, d, dtype, (const char*)q + t0 * qrow, (const char*)k + t0 * krow,
                    (const char*)v + t0 * krow, score_log2_scale(d), nullptr, nullptr, 0, 1,
                    (char*)out + t0 * qrow, lse ? lse + (size_t)Hq * t0 : nullptr,
                    (int32_t*)workspace};
        if ((rc = cuda_status(run_dense(aa, st))))
            return rc;
    }
    return TAM_OK;
}

namespace {
int64_t read_fallback_count(const void* workspace, size_t off_fb, void* stream) {
    if (!workspace) return -1;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return -1;
    int32_t c = 0;
    if (cudaMemcpy(&c, (const char*)workspace + off_fb, sizeof(c), cudaMemcpyDeviceToHost) !=
        cudaSuccess)
        return -1;
    return c;
}
}  // namespace

int64_t tam_mass_fallback_rows(int64_t N, int Hq, int Hkv, int d, int dtype, int budget_k,
                               const void* workspace, void* stream) {
    if (check_shape(N, Hq, Hkv, d, dtype) != TAM_OK || check_budget(N, budget_k, 1) != TAM_OK)
        return -1;
    const MassPlan plan = plan_mass(N, Hq, Hkv, d, dtype, budget_k, 1);
    if (!plan.stream || plan.sp.materialise) return -1;
    return read_fallback_count(workspace, plan.sp.off_fb, stream);
}

int64_t tam_indexer_fallback_rows(int64_t N, int d_idx, int dtype, int budget_k,
                                  const void* workspace, void* stream) {
    if (N < 1 || d_idx < 1 || (dtype != TAM_BF16 && dtype != TAM_F32)) return -1;
    if (check_indexer_args(N, d_idx, dtype, budget_k, 1) != TAM_OK) return -1;
    const IndexerPlan plan = plan_indexer(N, d_idx, dtype, budget_k, 1);
    if (!plan.tc || plan.sp.materialise) return -1;
    return read_fallback_count(workspace, plan.sp.off_fb, stream);
}

int tam_check_status(const void* workspace, void* stream, int32_t* detail) {
    if (!workspace) return TAM_ERR_INVALID_ARG;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return TAM_ERR_CUDA;
    int32_t w[8];
    if (cudaMemcpy(w, workspace, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess)
        return TAM_ERR_CUDA;
    if (detail) std::memcpy(detail, w, sizeof(w));
    return w[0];
}

}  // extern "C"
