/*
 * tam.h - C ABI of the B200 attention-mass top-k library (libtam.so).
 *
 * The method (arXiv 2606.07703, "How Much Dense Attention is Necessary?
 * Oracle-Guided Sparse Prefill for Full/GQA Layers in Hybrid Long-Context
 * Models"): for each query position of a causal GQA prefill layer, compute
 * dense attention, average the per-head probabilities over all query heads
 * into one token-mass row, keep the top-k tokens of that row (per query, or
 * once for a block of consecutive queries), and recompute attention for every
 * head only on that support, with the softmax renormalised over it
 * (Abstract; gist.science technical report §2.1 "Der Attention-Mass Top-k
 * Oracle").  A head-collapsed indexer picks the support from one shared
 * low-dimensional score instead (report §2.2).
 *
 * Notation.  N query/key positions (batch 1, causal: query i sees keys j <= i),
 * Hq query heads, Hkv KV heads (Hq % Hkv == 0), head dim d, G = Hq / Hkv.
 * Query head h reads KV head g(h) = h / G (consecutive heads share a KV head).
 * scale = 1/sqrt(d).
 *
 * Layouts (all row-major, contiguous, device memory unless stated):
 *   q   [N, Hq, d]    element (i,h,c) at (i*Hq + h)*d + c
 *   k,v [N, Hkv, d]   element (j,g,c) at (j*Hkv + g)*d + c
 *   out [N, Hq, d]    same dtype as q
 *   lse [Hq, N] fp32  natural-log sum of exp(scale * q.k) over the keys used
 *   sup_idx  [n_sel, budget_k] int32, each row ascending, padded with -1
 *   sup_len  [n_sel] int32,   sup_mass / sup_score [n_sel, budget_k] fp32 (0 in the padding)
 *   n_sel = N for per-query support (block_q == 1), ceil(N / block_q) otherwise.
 *
 * dtype: TAM_BF16 (bf16 storage, fp32 accumulation; tensor cores) or TAM_F32
 * (fp32 storage and arithmetic on CUDA cores).  Head dim d: 64, 128 or 256.  bf16
 * runs on the tensor cores at every d, except pass 2 at d = 256 when the Q tile of
 * every KV group does not fit in shared memory (more than 8 KV groups, or more than 4
 * with 16 query heads per group: CUDA cores, same results), and the indexer, whose
 * head is 16..128 wide.
 *
 * Packed batches ("_varlen" entry points).  n_seq independent causal sequences
 * are packed along the token axis: sequence s owns tokens [cu[s], cu[s+1]) of
 * q/k/v/out (T = cu[n_seq] rows in the layouts above, positions restarting at 0
 * in every sequence).  cu_seqlens is a HOST array of n_seq + 1 int64 with
 * cu[0] = 0, non-decreasing (empty sequences are allowed), T < 2^31.  Per
 * sequence the results are exactly those of the single-sequence call on its
 * slice: key indices in sup_idx are positions within the sequence; selection
 * rows are packed in sequence order (sequence s starts at row
 * sum_{s'<s} n_sel(N_s')); lse is packed as one [Hq, N_s] block per sequence,
 * block s starting at element Hq * cu[s].
 *
 * Ownership.  The caller allocates and frees every buffer, including the
 * workspace; the library never allocates device memory.  Every launch goes to
 * `stream` (a cudaStream_t; NULL = the legacy default stream) and the calls
 * return right after enqueueing.
 *
 * Errors.  Argument errors are detected on the host before anything is
 * enqueued and returned directly: TAM_ERR_INVALID_ARG (null pointer, bad
 * shape, pointer not 16-byte aligned, k < 1, block_q < 1, bad cu_seqlens),
 * TAM_ERR_UNSUPPORTED (d not 64/128/256, k > 4096, N*k >= 2^31, combination not
 * built), TAM_ERR_WORKSPACE
 * (ws_bytes below the smallest accepted size).  A failed launch returns TAM_ERR_CUDA.
 * Errors found on the device (a bounded wait that gave up) are recorded in a
 * status block at the start of the workspace and are read by tam_check_status.
 * No call traps and no call prints.
 */
#ifndef TAM_H
#define TAM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TAM_OK = 0,
    TAM_ERR_INVALID_ARG = 1,
    TAM_ERR_UNSUPPORTED = 2,
    TAM_ERR_WORKSPACE = 3,
    TAM_ERR_CUDA = 4,
    TAM_ERR_TIMEOUT = 5,
    TAM_ERR_OVERFLOW = 6    /* debug-checks build only: a store outside its buffer, skipped */
} tam_status;

typedef enum { TAM_BF16 = 0, TAM_F32 = 1 } tam_dtype;

/* Library version as 10000*major + 100*minor + patch. */
int tam_version(void);

/* Human-readable name of a status code (static string; never NULL). */
const char* tam_status_string(int status);

/*
 * Workspace bytes tam_mass_oracle_prefill prefers for this problem (always a
 * multiple of 256).  Returns 0 for arguments that the call would reject.
 * Per query on the tensor cores, pass 2 selects without writing the mass rows:
 *   1. a sample pass scores every S-th key of each row (S the smallest prime of
 *      at least 17 that leaves at most 4096 sampled keys per row; a prime stride
 *      does not line up with power-of-two structure in the key positions) and sets
 *      the row's threshold tau_i = the r-th largest sampled mass,
 *      r = ceil(mu + 5 sqrt(mu) + 4) with mu = s min(k, i+1) / (i+1) the expected
 *      number of sampled keys at or above the k-th value among the row's
 *      s = i / S + 1 samples (rows of at most `cap` keys keep every key:
 *      tau_i = -inf);
 *   2. the scoring pass keeps only the keys with P_i[j] >= tau_i, in nseg
 *      candidate segments per row (8 on CTA pairs, 4 otherwise) of seg_cap
 *      entries each, seg_cap = 32 * ceil((ceil(1.5 * S * (r0 + 1) / nseg) + 32)
 *      / 32), r0 the threshold rank for mu = k / S, cap = nseg * seg_cap;
 *   3. an exact select runs over each row's candidates; a row whose candidates
 *      fell short of min(k, i+1) or overflowed a segment is recomputed whole on
 *      the CUDA cores and selected exactly (the results are the same).
 * Layout after the status block (256 B) and lse (Hq*N floats, 256-aligned):
 * tau [N] f32, fallback list [1 + N] i32, counts [N * nseg] i32 (each
 * 256-aligned), then a region that holds in turn the sample rows of a chunk of
 * queries, the candidates of a chunk (cap entries of 8 bytes per row) and the
 * fallback rows' scratch.  The preferred region takes every row at once (and at
 * least min(N, 148) rows of N floats); any size down to tam_mass_workspace_min()
 * is accepted and only means more chunks.  Otherwise the two sizes are equal.
 */
size_t tam_mass_oracle_workspace(int64_t N, int Hq, int Hkv, int d, int dtype, int budget_k,
                                 int block_q);

/*
 * Smallest workspace tam_mass_oracle_prefill, tam_mass_select and
 * tam_mass_select_noalloc accept for this problem (a multiple of 256; 0 for
 * arguments the calls would reject).  Per query on the tensor cores the region
 * then holds the largest of 64 rows of samples, 64 rows of candidates and 64 rows
 * of N floats (enough for the materialised rows below, and for one fallback row).
 */
size_t tam_mass_workspace_min(int64_t N, int Hq, int Hkv, int d, int dtype, int budget_k,
                              int block_q);

/*
 * The attention-mass top-k oracle for one causal GQA prefill layer
 * (Abstract; technical report §2.1):
 *   pass 1  lse[h,i]  = log sum_{j<=i} exp(scale * q[i,h].k[j,g(h)])
 *   pass 2  P_i[j]    = (1/Hq) sum_h exp(scale * q[i,h].k[j,g(h)] - lse[h,i]),   j <= i
 *           block_q == 1: S_i = top-min(k, i+1) of P_i                     (n_sel = N)
 *           block_q  > 1: M_b[j] = sum_{i in block b, i >= j} P_i[j] for j <= e_b,
 *                         e_b = min(N, (b+1)*block_q) - 1, S_b = top-min(k, e_b+1) of M_b
 *           ranking: larger value first, equal values -> smaller index first;
 *           sup_idx rows are written ascending, sup_mass holds P_i[j] (or M_b[j]).
 *   pass 3  (only if out != NULL) for every head h of query i,
 *           out[i,h] = sum_{j in T_i} softmax_{T_i}(scale * q[i,h].k[j,g(h)]) v[j,g(h)],
 *           T_i = S_i (per query) or S_b intersected with [0, i] (block), output in q's dtype.
 * lse may be NULL (then it lives in the workspace).  Per query, no mass row P_i
 * is written: only the keys at or above a sampled threshold are kept and selected
 * from (see tam_mass_oracle_workspace); block-shared, only the block sums M_b are
 * written.  With TAM_MATERIALISE_ROWS=1 in the environment the per-query rows are
 * written to the workspace region chunk by chunk and selected from there instead
 * (same results; for A/B comparisons).  budget_k in [1, 4096]; block_q in [1, N].
 * A workspace smaller than tam_mass_workspace_min() gives TAM_ERR_WORKSPACE before
 * anything is enqueued.
 */
int tam_mass_oracle_prefill(int64_t N, int Hq, int Hkv, int d, int dtype, const void* q,
                            const void* k, const void* v, int budget_k, int block_q,
                            int32_t* sup_idx, int32_t* sup_len, float* sup_mass, float* lse,
                            void* out, void* workspace, size_t ws_bytes, void* stream);

/*
 * Workspace bytes tam_mass_oracle_prefill_varlen prefers: the largest of
 * tam_mass_oracle_workspace over the batch's sequences (their pass 2 runs one after
 * another and shares it), plus Hq * T * 4 bytes rounded up to 256, plus 256, for the
 * packed LSE of the whole batch when the caller passes lse = NULL.  0 for arguments
 * the call would reject.
 */
size_t tam_mass_oracle_workspace_varlen(int n_seq, const int64_t* cu_seqlens, int Hq, int Hkv,
                                        int d, int dtype, int budget_k, int block_q);

/*
 * tam_mass_oracle_prefill over a packed batch of independent sequences (layout in
 * the header comment, "Packed batches").  Each sequence runs passes 1-3 on its own
 * causal prefix, with the same budget_k and block_q; sup_idx/sup_len/sup_mass hold
 * sum_s n_sel(N_s) rows, lse (or NULL) Hq * T floats, out (or NULL) [T, Hq, d].
 * Launches (bf16 tensor-core shapes): pass 1 of every sequence in one launch per
 * table of up to 128 sequences (query tiles ordered heaviest first over the whole
 * table), pass 2 sequence by sequence, and pass 3 for per-query supports again one
 * launch per table (block-shared: sequence by sequence).  ws_bytes must reach the
 * largest sequence's tam_mass_workspace_min (plus the packed-LSE bytes above when
 * lse is NULL), else TAM_ERR_WORKSPACE before anything is enqueued.
 */
int tam_mass_oracle_prefill_varlen(int n_seq, const int64_t* cu_seqlens, int Hq, int Hkv, int d,
                                   int dtype, const void* q, const void* k, const void* v,
                                   int budget_k, int block_q, int32_t* sup_idx, int32_t* sup_len,
                                   float* sup_mass, float* lse, void* out, void* workspace,
                                   size_t ws_bytes, void* stream);

/*
 * Pass 1 alone: per-head log-sum-exp of the causal scores, lse [Hq, N] fp32
 * (technical report §2.1: the dense distribution each head's probabilities come from).
 */
size_t tam_attention_lse_workspace(int64_t N, int Hq, int Hkv, int d, int dtype);
int tam_attention_lse(int64_t N, int Hq, int Hkv, int d, int dtype, const void* q, const void* k,
                      float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * Pass 2 alone: head-averaged mass and its top-k support, given pass 1's lse [Hq, N]
 * (technical report §2.1, "Selektion" and "Granularität").  Same support semantics,
 * ranking and output layout as tam_mass_oracle_prefill; lse is read, not written.
 */
size_t tam_mass_select_workspace(int64_t N, int Hq, int Hkv, int d, int dtype, int budget_k,
                                 int block_q);
int tam_mass_select(int64_t N, int Hq, int Hkv, int d, int dtype, const void* q, const void* k,
                    const float* lse, int budget_k, int block_q, int32_t* sup_idx,
                    int32_t* sup_len, float* sup_mass, void* workspace, size_t ws_bytes,
                    void* stream);

/*
 * Pass 2 without a caller-provided workspace.  The paper has no counterpart: this
 * is a library service for callers that cannot allocate device memory (a plugin
 * whose host engine owns all device memory and hands it only its input and output
 * tensors; a process that must not call cudaMalloc while serving, because it can
 * synchronise the device and fail under fragmentation).
 * Same arguments, semantics and outputs as tam_mass_select, minus the workspace:
 * the scratch is a 64 MiB static device array inside the library.  Problems whose
 * tam_mass_workspace_min() exceeds 64 MiB are rejected with TAM_ERR_WORKSPACE
 * before anything is enqueued; a problem whose preferred workspace is larger than
 * 64 MiB but whose minimum fits runs in more chunks.  Nothing is allocated.  Every
 * call looks up the array's device address on the current device (a host-side
 * query), so the call works again after the context is torn down and re-created.
 * The call blocks: it waits for `stream` and returns the device status (TAM_OK or
 * TAM_ERR_TIMEOUT), so it cannot be used inside a stream capture.  All calls in
 * the process share the one array per device and it keeps the last call's
 * contents: calls that can overlap on the GPU (other streams, other threads) race
 * and must be serialised by the caller.  The 64 MiB are reserved on every device
 * where the library's module is loaded, whether or not this call is used, and are
 * held until the process exits.
 */
int tam_mass_select_noalloc(int64_t N, int Hq, int Hkv, int d, int dtype, const void* q,
                            const void* k, const float* lse, int budget_k, int block_q,
                            int32_t* sup_idx, int32_t* sup_len, float* sup_mass, void* stream);

/*
 * Head-collapsed indexer support (technical report §2.2 "Head-Collapsed Indexer":
 * one token score shared by all heads, top-k of it):
 *   score[i,j] = q_idx[i] . k_idx[j] for j <= i (no scale: ranking only),
 *   block_q == 1: S_i = top-min(k, i+1) of score_i with the same ranking and output
 *                 layout as above; sup_score holds the scores of the chosen keys.
 *   block_q  > 1: the fused, selection-block-shared path (Abstract; technical report
 *                 §3.2): q_i = softmax_{j <= i}(score_i) per query (scale 1),
 *                 M_b[j] = sum_{i in block b, i >= j} q_i[j], S_b = top-min(k, e_b+1) of
 *                 M_b; rows [n_sel = ceil(N / block_q), k], sup_score holds M_b of the
 *                 chosen keys.  Pass 3 on it: tam_sparse_support_attention(block_q).
 * q_idx, k_idx: [N, d_idx] in `dtype` (bf16 or fp32), d_idx in {16, 32, 64, 128}
 * (block_q > 1: d_idx in {64, 128}).
 * On the tensor cores the per-query selection streams as in tam_mass_oracle_prefill
 * (sampled thresholds, 4 candidate segments per row, fallback rows on the CUDA cores;
 * same workspace layout after the status block, with no lse);
 * tam_indexer_workspace() is the preferred size (every row at once),
 * tam_indexer_workspace_min() the smallest accepted.
 */
size_t tam_indexer_workspace(int64_t N, int d_idx, int dtype, int budget_k, int block_q);
size_t tam_indexer_workspace_min(int64_t N, int d_idx, int dtype, int budget_k, int block_q);
int tam_indexer_topk(int64_t N, int d_idx, int dtype, const void* q_idx, const void* k_idx,
                     int budget_k, int block_q, int32_t* sup_idx, int32_t* sup_len,
                     float* sup_score, void* workspace, size_t ws_bytes, void* stream);

/*
 * tam_indexer_topk over a packed batch (layout in the header comment, "Packed
 * batches"): q_idx, k_idx [T, d_idx]; each sequence selects among its own keys;
 * sup_* hold sum_s n_sel(N_s) rows with positions local to the sequence.  The
 * workspace query returns the largest single-sequence size (0 for rejected
 * arguments); ws_bytes must reach the largest sequence's tam_indexer_workspace_min.
 */
size_t tam_indexer_workspace_varlen(int n_seq, const int64_t* cu_seqlens, int d_idx, int dtype,
                                    int budget_k, int block_q);
int tam_indexer_topk_varlen(int n_seq, const int64_t* cu_seqlens, int d_idx, int dtype,
                            const void* q_idx, const void* k_idx, int budget_k, int block_q,
                            int32_t* sup_idx, int32_t* sup_len, float* sup_score, void* workspace,
                            size_t ws_bytes, void* stream);

/*
 * The indexer's distillation target (technical report §2.2, "Trainingsziel": the
 * head-collapsed indexer is trained by KL divergence from the dense attention-mass
 * distribution), per query, without returning the N x N distributions:
 *   kl[i] = sum_{j <= i} P_i[j] log(P_i[j] / q_i[j]),  0 log 0 = 0,
 *   P_i as in pass 2 (needs pass 1's lse [Hq, N]), q_i = softmax_{j <= i}(q_idx[i] . k_idx[j])
 *   (scale 1, as for the block-shared indexer).
 * q, k: as for tam_mass_select (bf16, tensor-core shapes); q_idx, k_idx: [N, d_idx] bf16,
 * d_idx in {64, 128}; kl: [N] fp32.  Other dtypes or shapes: TAM_ERR_UNSUPPORTED.
 * The mass rows and the indexer score rows of a chunk of queries go through two slabs
 * in the workspace: tam_distill_kl_workspace() is the preferred size (every row at
 * once, up to 2 x 4 GiB), tam_distill_kl_workspace_min() the smallest accepted.
 */
size_t tam_distill_kl_workspace(int64_t N, int Hq, int Hkv, int d, int dtype, int d_idx);
size_t tam_distill_kl_workspace_min(int64_t N, int Hq, int Hkv, int d, int dtype, int d_idx);
int tam_distill_kl(int64_t N, int Hq, int Hkv, int d, int dtype, const void* q, const void* k,
                   const float* lse, int d_idx, const void* q_idx, const void* k_idx, float* kl,
                   void* workspace, size_t ws_bytes, void* stream);

/*
 * Budget sweep from one pass-2 run (technical report §3.1, "Budget-Sensitivitaet":
 * the oracle compared at top-k budgets of 256 to 2048): for each row r of a top-kmax
 * support (sup_val [n_rows, kmax] fp32 values >= 0, e.g. sup_mass of tam_mass_select,
 * sup_len [n_rows]) and each budget budgets[t] (host array, 1 <= n_budgets <= 16),
 *   out[r, t] = sum of the budgets[t] largest values of row r   (the whole row if
 *               budgets[t] >= sup_len[r]),
 * which is the support mass of the top-budgets[t] support whenever budgets[t] <= kmax.
 * out: [n_rows, n_budgets] fp32, device.  kmax <= 4096.  No workspace; argument errors
 * return before anything is enqueued.  The sparsity at a budget is a closed form
 * (1 - sum_i min(k, i+1) / sum_i (i+1)) and needs no call.
 */
int tam_support_mass_curve(int64_t n_rows, int kmax, const float* sup_val, const int32_t* sup_len,
                           const int32_t* budgets, int n_budgets, float* out, void* stream);

/*
 * Pass 3 alone: attention recomputed on a given support (technical report §2.1,
 * "Ausführung": original Q, K, V restricted to the selected tokens).
 * block_q == 1: row i of sup_idx (first sup_len[i] entries) is query i's support.
 * block_q  > 1: row b = i / block_q is shared by the block's queries; query i uses the
 *               entries j <= i.  Entries < 0 or > i are skipped.  kmax = row stride of
 *               sup_idx (>= every sup_len).  A query whose support is empty gets a zero
 *               output row and lse = -inf.
 */
size_t tam_sparse_attention_workspace(int64_t N, int Hq, int Hkv, int d, int dtype);
int tam_sparse_support_attention(int64_t N, int Hq, int Hkv, int d, int dtype, const void* q,
                                 const void* k, const void* v, const int32_t* sup_idx,
                                 const int32_t* sup_len, int kmax, int block_q, void* out,
                                 float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * tam_sparse_support_attention over a packed batch (layout in the header comment,
 * "Packed batches"): the support rows of sequence s (positions local to it) start at
 * row sum_{s'<s} n_sel(N_s'), as tam_mass_oracle_prefill_varlen and
 * tam_indexer_topk_varlen write them.  Per-query supports (block_q = 1) run as one
 * launch per table of up to 128 sequences.  Workspace: tam_sparse_attention_workspace
 * bytes.
 */
int tam_sparse_support_attention_varlen(int n_seq, const int64_t* cu_seqlens, int Hq, int Hkv,
                                        int d, int dtype, const void* q, const void* k,
                                        const void* v, const int32_t* sup_idx,
                                        const int32_t* sup_len, int kmax, int block_q, void* out,
                                        float* lse, void* workspace, size_t ws_bytes,
                                        void* stream);

/*
 * Dense causal GQA prefill (the FlashAttention-2 comparator the abstract measures
 * against): out[i,h] = softmax_{j<=i}(scale * q[i,h].k[j,g(h)]) v[j,g(h)], lse optional.
 */
size_t tam_dense_workspace(int64_t N, int Hq, int Hkv, int d, int dtype);
int tam_dense_gqa_prefill(int64_t N, int Hq, int Hkv, int d, int dtype, const void* q,
                          const void* k, const void* v, void* out, float* lse, void* workspace,
                          size_t ws_bytes, void* stream);

/*
 * tam_dense_gqa_prefill over a packed batch of independent causal sequences (layout
 * in the header comment, "Packed batches"): out [T, Hq, d], lse (or NULL) one
 * [Hq, N_s] block per sequence.  bf16 runs as one launch per table of up to 128
 * sequences, query tiles ordered heaviest first over the table.  Workspace:
 * tam_dense_workspace bytes (any N).
 */
int tam_dense_gqa_prefill_varlen(int n_seq, const int64_t* cu_seqlens, int Hq, int Hkv, int d,
                                 int dtype, const void* q, const void* k, const void* v,
                                 void* out, float* lse, void* workspace, size_t ws_bytes,
                                 void* stream);

/*
 * Diagnostics of the streamed per-query selection: how many rows of the last
 * per-query tam_mass_oracle_prefill / tam_mass_select (or tam_indexer_topk) call
 * that used `workspace` for this problem went to the fallback path (their sampled
 * threshold was above the k-th value, or a candidate segment overflowed).  Waits
 * for `stream`.  Returns -1 for arguments those calls would reject, for problems
 * that do not stream (CUDA-core path, block_q > 1) and with TAM_MATERIALISE_ROWS=1.
 */
int64_t tam_mass_fallback_rows(int64_t N, int Hq, int Hkv, int d, int dtype, int budget_k,
                               const void* workspace, void* stream);
int64_t tam_indexer_fallback_rows(int64_t N, int d_idx, int dtype, int budget_k,
                                  const void* workspace, void* stream);

/*
 * Number of CUDA kernels this library has launched in this process so far (all
 * devices, all entry points; status-block clears are not kernels and do not count).
 */
uint64_t tam_kernel_launches(void);

/*
 * Waits for `stream`, then reads the device status block at the start of
 * `workspace` that the last call using this workspace wrote.  Returns TAM_OK,
 * TAM_ERR_TIMEOUT or TAM_ERR_CUDA (and, from the debug-checks build libtam_debug.so,
 * TAM_ERR_OVERFLOW).  `detail` (may be NULL) receives 8 int32 words: [0] status,
 * [1] kernel id, [2..7] kernel-specific (overflow: [2] site 1 slab row / 2 candidate /
 * 3 block mass, [3] index, [4] extent, truncated to 32 bits).
 *
 * Debug-checks build: compiled with -DTAM_DEBUG_CHECKS (same symbols), the pass-2
 * kernels check every slab-row, candidate and block-mass store against the extent the
 * host planned for the launch; instead of an out-of-range store they record
 * TAM_ERR_OVERFLOW here and skip it.  With the environment variable
 * TAM_DEBUG_SHRINK_EXTENTS set, the host plans extents of at most 64 entries, so that
 * the checks fire on stores that still land inside the real buffers.
 */
int tam_check_status(const void* workspace, void* stream, int32_t* detail);

#ifdef __cplusplus
}
#endif

#endif /* TAM_H */
