// Internal launcher interface between the C ABI (tam_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace tam {

// Packed batches in one launch: sequence s of the table owns the tokens
// [cu[s], cu[s+1]) of the packed q/k/v rows (a single-sequence call is the table
// {1, N, {0, N}}).  The kernels that take a table number their query tiles of BQ rows
// sequence by sequence, longest sequence first (`order`), each sequence's tiles
// heaviest (last) first, so that the machine works through the long sequences while
// the short ones fill the tail, and the CTAs in flight share one or two sequences' K/V
// in L2.  Larger batches run as several tables.
constexpr int kMaxSeqPerLaunch = 128;
struct SeqTable {
    int n_seq;
    int max_len;                        // longest sequence of the table
    int cu[kMaxSeqPerLaunch + 1];       // absolute token offsets, non-decreasing
    int order[kMaxSeqPerLaunch];        // sequences by length, longest first
    int tile0[kMaxSeqPerLaunch + 1];    // first tile of order[r] (set per launch for its BQ)
};

// Sorts the table's sequences by length (longest first, ties in order).
inline void seq_table_order(SeqTable& t) {
    for (int s = 0; s < t.n_seq; ++s) t.order[s] = s;
    for (int a = 1; a < t.n_seq; ++a) {            // insertion sort: at most 128 entries
        const int s = t.order[a], n = t.cu[s + 1] - t.cu[s];
        int b = a;
        for (; b > 0 && t.cu[t.order[b - 1] + 1] - t.cu[t.order[b - 1]] < n; --b)
            t.order[b] = t.order[b - 1];
        t.order[b] = s;
    }
}

// Fills tile0 for tiles of BQ rows; returns the table's tile count.
inline int seq_table_tiles(SeqTable& t, int BQ) {
    t.tile0[0] = 0;
    for (int r = 0; r < t.n_seq; ++r) {
        const int s = t.order[r];
        t.tile0[r + 1] = t.tile0[r] + (t.cu[s + 1] - t.cu[s] + BQ - 1) / BQ;
    }
    return t.tile0[t.n_seq];
}

// Runs fn on a copy of the launch's table: *seqs, or the single sequence [0, N) when
// seqs is null (the copy is the launch's own, so it may fill tile0).
template <class F>
cudaError_t with_table(int64_t N, const SeqTable* seqs, F&& fn) {
    SeqTable t{};
    if (seqs) {
        t = *seqs;
    } else {
        t.n_seq = 1;
        t.max_len = (int)N;
        t.cu[0] = 0;
        t.cu[1] = (int)N;
        t.order[0] = 0;
    }
    return fn(t);
}

// (sequence, local tile) of the b-th tile of the table in the order above, for tiles of
// BQ rows; any thread may call it (and the host, to check the order).
__host__ __device__ inline void seq_tile_of(const SeqTable& t, int BQ, int b, int& s_out,
                                            int& L_out) {
    int lo = 0, hi = t.n_seq - 1;                  // the last r with tile0[r] <= b
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (t.tile0[mid] <= b) lo = mid;
        else hi = mid - 1;
    }
    const int s = t.order[lo];
    s_out = s;
    L_out = (t.cu[s + 1] - t.cu[s] + BQ - 1) / BQ - 1 - (b - t.tile0[lo]);
}

#ifdef __CUDACC__
template <int BQ>
__device__ __forceinline__ void seq_tile(const SeqTable& t, int b, int& s_out, int& L_out) {
    seq_tile_of(t, BQ, b, s_out, L_out);
}
#endif

struct LseArgs {
    int64_t N;
    int Hq, Hkv, d, dtype;
    const void* q;
    const void* k;
    float sl2;            // scale * log2(e)
    float* lse;           // [Hq, N] natural log (packed batch: [Hq, N_s] per sequence s,
                          // starting at element Hq * cu[s])
    int32_t* status;
    const SeqTable* seqs = nullptr;   // packed batch on the N = T packed rows (tensor cores)
};

struct MassArgs {
    int64_t N;
    int Hq, Hkv, d, dtype;
    const void* q;
    const void* k;
    const float* lse;     // [Hq, N] from pass 1
    float sl2;
    int budget, block_q, n_sel;
    int n_ctas;           // persistent blocks (CUDA-core path)
    float* scratch;       // n_ctas * N floats (CUDA-core path)
    float* rows;          // triangular slab of mass rows (tensor-core path, per query)
    int64_t row0, row1;   // the queries whose rows this launch writes (per query)
    int kst;              // rows mode: only the keys j = m * kst (sample rows); 1 = every key
    bool stream;          // per query: threshold-filtered candidates instead of rows
    const float* tau;     // stream: threshold of every query [N]
    void* cand;           // stream: candidate segments of the rows [row0, row1)
    int32_t* cnt;         // stream: appended count per (row, segment)
    int seg_cap;          // stream: entries per segment
    void* bmass;          // fixed-point block mass (tensor-core path, block-shared)
    int32_t* sup_idx;
    int32_t* sup_len;
    float* sup_mass;
    int32_t* status;
    // entries of rows (floats), cand (pairs) or bmass (u64) the launch may write: checked
    // by the debug-checks build only
    uint64_t out_cap = ~uint64_t(0);
};

struct AttnArgs {
    int64_t N;
    int Hq, Hkv, d, dtype;
    const void* q;
    const void* k;
    const void* v;
    float sl2;
    const int32_t* sup_idx;   // null = dense causal
    const int32_t* sup_len;
    int kmax, block_q;
    void* out;
    float* lse;
    int32_t* status;
    const SeqTable* seqs = nullptr;   // packed batch on the N = T packed rows (see LseArgs)
};

struct IndexerArgs {
    int64_t N;
    int d_idx, dtype;
    const void* q_idx;
    const void* k_idx;
    int budget;
    int n_ctas;
    float* scratch;       // n_ctas * N floats (CUDA-core path)
    float* rows;          // triangular slab of score rows (tensor-core path)
    int64_t row0, row1;   // the queries whose rows this launch writes
    int kst;              // rows mode: only the keys j = m * kst (sample rows); 1 = every key
    bool stream;          // threshold-filtered candidates instead of rows
    const float* tau;
    void* cand;
    int32_t* cnt;
    int seg_cap;
    int32_t* sup_idx;
    int32_t* sup_len;
    float* sup_score;
    int32_t* status;
    uint64_t out_cap = ~uint64_t(0);   // as MassArgs::out_cap
};

// Counts one kernel launch (read back by tam_kernel_launches).
void note_launch(int n = 1);

// Tensor-core kernels (bf16, sm_100a).  *_supported says whether a shape is built.
bool tc_lse_supported(const LseArgs& a);
cudaError_t tc_lse(const LseArgs& a, cudaStream_t st);
int tc_mass_columns(const MassArgs& a);
bool tc_mass_supported(const MassArgs& a);
size_t tc_mass_block_bytes(int64_t N, int block_q);
// Per query: writes the mass rows [row0, row1) to the slab (select with row_topk);
// block-shared: block sums and the block top-k, the whole of pass 2.
cudaError_t tc_mass_pass(const MassArgs& a, cudaStream_t st);
bool pair_mass_supported(const MassArgs& a);
cudaError_t pair_mass(const MassArgs& a, cudaStream_t st);
bool tc_indexer_supported(int64_t N, int d_idx, int dtype, int block_q);
// Writes the indexer score rows [row0, row1) to the slab (select with row_topk), or
// with a.stream their threshold-filtered candidate segments (select with cand_select).
cudaError_t tc_indexer_rows(const IndexerArgs& a, cudaStream_t st);
// Candidate segments per row written by the per-query kernel tc_mass_pass would run
// for this shape (8 on CTA pairs, 4 on single CTAs; the indexer always 4).
int tc_mass_segments(const MassArgs& a);
constexpr int kIndexerSegments = 4;

// Row slabs: row i (i + 1 values) starts tri(i) - tri(row0) floats after the base.
inline int64_t tri(int64_t i) { return i * (i + 1) / 2; }
// Exact top-min(k, i+1) of each slab row i in [row0, row1), ascending key index,
// ties toward the smaller index; sup_* are indexed by the absolute row i.
cudaError_t row_topk(const float* slab, int64_t row0, int64_t row1, int budget, int32_t* sup_idx,
                     int32_t* sup_len, float* sup_val, cudaStream_t st);
// Rows sampled every S keys: row i' holds i' / S + 1 values, so the rows before
// i = a S + b hold i + S a (a - 1) / 2 + a b (tri(i) for S = 1); row i starts
// sample_offset(i, S) - sample_offset(row0, S) floats after the slab base.
__host__ __device__ inline int64_t sample_offset(int64_t i, int S) {
    const int64_t a = i / S, b = i - a * S;
    return i + S * (a * (a - 1) / 2) + a * b;
}
// Per-row thresholds from a sample slab: for rows of at most `take_all` keys
// tau = -inf (every key is a candidate); otherwise the r-th largest of the row's
// s = i / S + 1 samples, r = ceil(mu + z sqrt(mu) + 4), mu = s min(k, i+1) / (i+1),
// clamped to [1, s].  `force` (debug): 1 sets tau = +inf, 2 tau = -inf on the
// sampled rows, so that every such row falls back.
cudaError_t sample_tau(const float* slab, int64_t row0, int64_t row1, int S, int budget,
                       int take_all, float z, int force, float* tau, cudaStream_t st);
// Exact top-min(k, i+1) of each row i in [row0, row1) from its candidate segments
// (nseg per row, seg_cap entries each, (value bits, key) in key order, counts in cnt),
// written like row_topk.  A row whose segments overflowed or hold fewer than
// min(k, i+1) keys is appended to the fallback list fb (fb[0] = count, fb[1 + t] = row)
// and its outputs are left to the fallback.
// Shared memory cand_select needs for rows of up to max_row_keys keys and cap
// candidates each; it runs only when that is at most kCandSelectMaxSmem.
int cand_select_smem(int64_t max_row_keys, int cap);
constexpr int kCandSelectMaxSmem = 227 * 1024;
cudaError_t cand_select(const void* cand, const int32_t* cnt, int64_t row0, int64_t row1,
                        int nseg, int seg_cap, int budget, int32_t* sup_idx, int32_t* sup_len,
                        float* sup_val, int32_t* fb, cudaStream_t st);
// The rows on a fallback list, computed whole on the CUDA cores and selected exactly
// (n_ctas persistent blocks, each with an N-float row of scratch).
cudaError_t fallback_mass_rows(const MassArgs& a, const int32_t* fb, float* scratch, int n_ctas,
                               cudaStream_t st);
cudaError_t fallback_indexer_rows(const IndexerArgs& a, const int32_t* fb, float* scratch,
                                  int n_ctas, cudaStream_t st);
// out[r, t] = sum of the ks[t] largest values of support row r (rows of a top-kmax
// support: val [rows, kmax], len [rows]); nk <= kMaxSweepBudgets, kmax <= 4096.
constexpr int kMaxSweepBudgets = 16;
cudaError_t support_mass_curve(const float* val, const int32_t* len, int64_t rows, int kmax,
                               const int32_t* ks, int nk, float* out, cudaStream_t st);

// kl[i] = KL(P_i || softmax(t_i)) for the rows [row0, row1) of a mass slab and a score
// slab laid out alike.
cudaError_t row_kl(const float* mass, const float* score, int64_t row0, int64_t row1, float* kl,
                   cudaStream_t st);
bool tc_dense_supported(const AttnArgs& a);
cudaError_t tc_dense(const AttnArgs& a, cudaStream_t st);
bool gather_supported(const AttnArgs& a);
cudaError_t gather_attention(const AttnArgs& a, cudaStream_t st);
bool block_tc_supported(const AttnArgs& a);
cudaError_t block_attention_tc(const AttnArgs& a, cudaStream_t st);
// Dense causal attention on the block kernel's two-tile pipeline (TMA K/V chunks of 64
// keys, two query tiles per CTA); used with TAM_DENSE_PAIR_TILES=1.
bool dense_pair_tiles_supported(const AttnArgs& a);
cudaError_t dense_pair_tiles(const AttnArgs& a, cudaStream_t st);

// CUDA-core kernels (any dtype, any supported shape).
cudaError_t simt_lse(const LseArgs& a, cudaStream_t st);
cudaError_t simt_mass_select(const MassArgs& a, cudaStream_t st);
cudaError_t simt_attention(const AttnArgs& a, cudaStream_t st);
cudaError_t simt_indexer_select(const IndexerArgs& a, cudaStream_t st);

}  // namespace tam
