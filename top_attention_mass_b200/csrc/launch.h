// Internal launcher interface between the C ABI (tam_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace tam {

struct LseArgs {
    int64_t N;
    int Hq, Hkv, d, dtype;
    const void* q;
    const void* k;
    float sl2;            // scale * log2(e)
    float* lse;           // [Hq, N] natural log
    int32_t* status;
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
    void* bmass;          // fixed-point block mass (tensor-core path, block-shared)
    int32_t* sup_idx;
    int32_t* sup_len;
    float* sup_mass;
    int32_t* status;
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
    int32_t* sup_idx;
    int32_t* sup_len;
    float* sup_score;
    int32_t* status;
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
// Writes the indexer score rows [row0, row1) to the slab (select with row_topk).
cudaError_t tc_indexer_rows(const IndexerArgs& a, cudaStream_t st);

// Row slabs: row i (i + 1 values) starts tri(i) - tri(row0) floats after the base.
inline int64_t tri(int64_t i) { return i * (i + 1) / 2; }
// Exact top-min(k, i+1) of each slab row i in [row0, row1), ascending key index,
// ties toward the smaller index; sup_* are indexed by the absolute row i.
cudaError_t row_topk(const float* slab, int64_t row0, int64_t row1, int budget, int32_t* sup_idx,
                     int32_t* sup_len, float* sup_val, cudaStream_t st);
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

// CUDA-core kernels (any dtype, any supported shape).
cudaError_t simt_lse(const LseArgs& a, cudaStream_t st);
cudaError_t simt_mass_select(const MassArgs& a, cudaStream_t st);
cudaError_t simt_attention(const AttnArgs& a, cudaStream_t st);
cudaError_t simt_indexer_select(const IndexerArgs& a, cudaStream_t st);

}  // namespace tam
