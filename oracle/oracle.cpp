// Plain fp64 CPU oracle of the attention-mass top-k path for causal GQA prefill.
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
// this file: only the tests, the package smoke check and the benchmark's CPU
// baseline leg use it.  It shares no code with the CUDA kernels.
//
// What it follows (page titles and sections of the sources on arXiv 2606.07703,
// "How Much Dense Attention is Necessary? Oracle-Guided Sparse Prefill for
// Full/GQA Layers in Hybrid Long-Context Models"):
//   * Abstract (arXiv listing): for each layer and query position the oracle
//     computes dense attention, selects head-averaged token support and
//     recomputes attention only on that support.
//   * gist.science technical report, section 2.1 "Der Attention-Mass Top-k
//     Oracle": dense distribution per query, aggregated over the query heads
//     into a head-averaged token-importance distribution P_{l,t}; the top-k
//     token indices of P are selected either per query (b_sel = 1) or once for
//     a selection block of consecutive queries (b_sel = 64); attention is then
//     recomputed on the selected support with the original Q, K, V.
//   * same report, section 2.2 "Head-Collapsed Indexer": one shared token
//     score across heads, top-k of it, sparse GQA recompute on that support;
//     Abstract and section 3.2: the fused, selection-block-shared indexer path;
//     section 2.2 "Trainingsziel": the indexer's KL-distillation target;
//     section 3.1 "Budget-Sensitivitaet": support mass at several budgets.
//
// Readings where the pages are silent (each listed in the design notes):
//   * query head h reads KV head g(h) = floor(h / (Hq/Hkv)) (consecutive grouping);
//   * score scale 1/sqrt(d), no soft-cap; the head average is the mean over all Hq heads;
//   * per-query support size min(k, i+1) over causal keys j <= i;
//   * ties are broken by the smaller key index;
//   * a block's mass is the sum of P_i over its causally valid queries; query i of a
//     block attends over S_b intersected with [0, i];
//   * the recompute renormalises the softmax over the support;
//   * the indexer score is the plain dot product q_idx . k_idx;
//   * block-shared indexer: each query's scores turned into softmax_{j <= i} (no
//     scale, the indexer being trained toward a distribution), summed over the block.
//
// Every input arrives as fp32 (bf16 and fp32 inputs are exactly representable)
// and is widened to double before any arithmetic.  All arithmetic is double.
// Rows (or blocks) are independent, so the outer loops run in parallel with
// OpenMP; nothing else is blocked, fused or reordered.

#include <algorithm>
#include <functional>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// Planted-mistake switch, used only by the oracle's own mutation tests to show
// that its pins catch plausible mistakes.  0 = the oracle as specified.
int g_mutation = 0;

inline int kv_head_of(int h, int Hq, int Hkv) {
    if (g_mutation == 2) return h % Hkv;          // planted: interleaved head map
    return h / (Hq / Hkv);
}

// s[j] = q_{i,h} . k_{j,g(h)} / sqrt(d) for j = 0..i.
void head_scores(const float* q, const float* k, int Hq, int Hkv, int d, int64_t i, int h,
                 double* s) {
    const int g = kv_head_of(h, Hq, Hkv);
    const float* qi = q + (i * Hq + h) * (int64_t)d;
    const double scale = (g_mutation == 1) ? 1.0 : 1.0 / std::sqrt((double)d);  // planted: no scale
    for (int64_t j = 0; j <= i; ++j) {
        const float* kj = k + (j * Hkv + g) * (int64_t)d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += (double)qi[c] * (double)kj[c];
        s[j] = acc * scale;
    }
}

// log sum_j exp(s[j]) with the maximum taken out first.
double log_sum_exp(const double* s, int64_t n) {
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) m = std::max(m, s[j]);
    double sum = 0.0;
    for (int64_t j = 0; j < n; ++j) sum += std::exp(s[j] - m);
    return m + std::log(sum);
}

// Head-averaged token mass of query i: P[j] = (1/Hq) sum_h exp(s_{h,i,j} - lse_{h,i}), j <= i.
void mass_row(const float* q, const float* k, int Hq, int Hkv, int d, int64_t i, double* P,
              double* s) {
    std::fill(P, P + i + 1, 0.0);
    for (int h = 0; h < Hq; ++h) {
        head_scores(q, k, Hq, Hkv, d, i, h, s);
        const double lse = log_sum_exp(s, i + 1);
        for (int64_t j = 0; j <= i; ++j) P[j] += std::exp(s[j] - lse);
    }
    const double inv = (g_mutation == 3) ? 1.0 : 1.0 / Hq;   // planted: sum instead of mean
    for (int64_t j = 0; j <= i; ++j) P[j] *= inv;
}

// Top-min(k, n) of val[0..n) ordered by (value descending, index ascending);
// the chosen indices are written in ascending order.  Returns the count.
int select_top(const double* val, int64_t n, int k, int32_t* out_idx) {
    const int64_t m = std::min<int64_t>(k, n);
    std::vector<int32_t> ord(n);
    std::iota(ord.begin(), ord.end(), 0);
    auto better = [val](int32_t a, int32_t b) {
        if (val[a] != val[b]) return val[a] > val[b];
        return (g_mutation == 4) ? a > b : a < b;     // planted: reversed tie rule
    };
    std::partial_sort(ord.begin(), ord.begin() + m, ord.end(), better);
    std::sort(ord.begin(), ord.begin() + m);
    std::copy(ord.begin(), ord.begin() + m, out_idx);
    return (int)m;
}

// Attention of query i, head h, over the support entries j with 0 <= j <= i,
// softmax renormalised over those entries.  Writes o[d] and returns the lse.
double support_attention(const float* q, const float* k, const float* v, int Hq, int Hkv, int d,
                         int64_t i, int h, const int32_t* sup, int64_t nsup, double* o,
                         std::vector<double>& s, std::vector<int32_t>& js) {
    const int g = kv_head_of(h, Hq, Hkv);
    const float* qi = q + (i * Hq + h) * (int64_t)d;
    const double scale = (g_mutation == 1) ? 1.0 : 1.0 / std::sqrt((double)d);
    js.clear();
    s.clear();
    for (int64_t t = 0; t < nsup; ++t) {
        const int32_t j = sup[t];
        if (j < 0 || j > i) continue;
        const float* kj = k + ((int64_t)j * Hkv + g) * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += (double)qi[c] * (double)kj[c];
        js.push_back(j);
        s.push_back(acc * scale);
    }
    std::fill(o, o + d, 0.0);
    if (js.empty()) return -INFINITY;
    const double lse = log_sum_exp(s.data(), (int64_t)s.size());
    for (size_t t = 0; t < js.size(); ++t) {
        const double p = std::exp(s[t] - lse);
        const float* vj = v + ((int64_t)js[t] * Hkv + g) * d;
        for (int c = 0; c < d; ++c) o[c] += p * (double)vj[c];
    }
    return lse;
}

bool shape_ok(int64_t N, int Hq, int Hkv, int d) {
    return N > 0 && Hq > 0 && Hkv > 0 && d > 0 && Hq % Hkv == 0;
}

}  // namespace

extern "C" {

void orc_set_mutation(int m) { g_mutation = m; }

void orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int orc_get_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

// Per-head log-sum-exp of the causal scores of each listed row: lse[r*Hq + h].
int orc_lse_rows(int64_t N, int Hq, int Hkv, int d, const float* q, const float* k,
                 const int64_t* rows, int64_t nrows, double* lse) {
    if (!shape_ok(N, Hq, Hkv, d)) return 1;
#pragma omp parallel
    {
        std::vector<double> s(N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            const int64_t i = rows[r];
            for (int h = 0; h < Hq; ++h) {
                head_scores(q, k, Hq, Hkv, d, i, h, s.data());
                lse[r * Hq + h] = log_sum_exp(s.data(), i + 1);
            }
        }
    }
    return 0;
}

// Head-averaged mass rows: P[r*N + j] for j <= rows[r], zero beyond.
int orc_mass_rows(int64_t N, int Hq, int Hkv, int d, const float* q, const float* k,
                  const int64_t* rows, int64_t nrows, double* P) {
    if (!shape_ok(N, Hq, Hkv, d)) return 1;
#pragma omp parallel
    {
        std::vector<double> s(N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            double* Pr = P + r * N;
            std::fill(Pr, Pr + N, 0.0);
            mass_row(q, k, Hq, Hkv, d, rows[r], Pr, s.data());
        }
    }
    return 0;
}

// Per-query support: S_i = top-min(k, i+1) of P_i.  idx[r*k ..] ascending, -1 padded;
// len[r]; mass[r*k + t] = P_i[idx[r*k + t]] (0 in the padding).
int orc_topk_rows(int64_t N, int Hq, int Hkv, int d, const float* q, const float* k,
                  const int64_t* rows, int64_t nrows, int budget, int32_t* idx, int32_t* len,
                  double* mass) {
    if (!shape_ok(N, Hq, Hkv, d) || budget < 1) return 1;
#pragma omp parallel
    {
        std::vector<double> s(N), P(N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            const int64_t i = rows[r];
            mass_row(q, k, Hq, Hkv, d, i, P.data(), s.data());
            int32_t* ir = idx + r * budget;
            std::fill(ir, ir + budget, -1);
            const int n = select_top(P.data(), i + 1, budget, ir);
            len[r] = n;
            for (int t = 0; t < budget; ++t) mass[r * budget + t] = (t < n) ? P[ir[t]] : 0.0;
        }
    }
    return 0;
}

// Block mass M_b[j] = sum_{i = max(j, b*Bq)}^{e_b} P_i[j] for j <= e_b, e_b = min(N, (b+1)Bq) - 1.
// M[r*N + j], zero beyond e_b.
int orc_block_mass(int64_t N, int Hq, int Hkv, int d, const float* q, const float* k, int block_q,
                   const int64_t* blocks, int64_t nblocks, double* M) {
    if (!shape_ok(N, Hq, Hkv, d) || block_q < 1) return 1;
#pragma omp parallel
    {
        std::vector<double> s(N), P(N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nblocks; ++r) {
            const int64_t b0 = blocks[r] * block_q;
            const int64_t e = std::min<int64_t>(N, b0 + block_q) - 1;
            double* Mr = M + r * N;
            std::fill(Mr, Mr + N, 0.0);
            for (int64_t i = b0; i <= e; ++i) {
                mass_row(q, k, Hq, Hkv, d, i, P.data(), s.data());
                for (int64_t j = 0; j <= i; ++j) Mr[j] += P[j];
            }
        }
    }
    return 0;
}

// Block-shared support: S_b = top-min(k, e_b+1) of M_b.  Layout as orc_topk_rows, with
// mass[r*k + t] = M_b[idx].
int orc_block_topk(int64_t N, int Hq, int Hkv, int d, const float* q, const float* k, int block_q,
                   const int64_t* blocks, int64_t nblocks, int budget, int32_t* idx, int32_t* len,
                   double* mass) {
    if (!shape_ok(N, Hq, Hkv, d) || block_q < 1 || budget < 1) return 1;
    std::vector<double> M((size_t)nblocks * N);
    int rc = orc_block_mass(N, Hq, Hkv, d, q, k, block_q, blocks, nblocks, M.data());
    if (rc) return rc;
    for (int64_t r = 0; r < nblocks; ++r) {
        const int64_t e = std::min<int64_t>(N, (blocks[r] + 1) * block_q) - 1;
        int32_t* ir = idx + r * budget;
        std::fill(ir, ir + budget, -1);
        const int n = select_top(M.data() + r * N, e + 1, budget, ir);
        len[r] = n;
        for (int t = 0; t < budget; ++t) mass[r * budget + t] = (t < n) ? M[r * N + ir[t]] : 0.0;
    }
    return 0;
}

// Attention recomputed on a support: for each listed row i and head h, softmax over
// T_i = {j in sup row : 0 <= j <= i}, renormalised, times V.  sup == NULL means the
// dense causal row T_i = [0, i].  out[(r*Hq + h)*d + c]; lse[r*Hq + h] (may be NULL),
// -inf when T_i is empty (the output row is then zero).
int orc_attn_rows(int64_t N, int Hq, int Hkv, int d, const float* q, const float* k,
                  const float* v, const int64_t* rows, int64_t nrows, const int32_t* sup,
                  const int32_t* sup_len, int64_t sup_stride, double* out, double* lse) {
    if (!shape_ok(N, Hq, Hkv, d)) return 1;
#pragma omp parallel
    {
        std::vector<double> s;
        std::vector<int32_t> js, dense;
        s.reserve(N);
        js.reserve(N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            const int64_t i = rows[r];
            const int32_t* srow;
            int64_t n;
            if (sup) {
                srow = sup + r * sup_stride;
                n = sup_len ? sup_len[r] : sup_stride;
            } else {
                dense.resize(i + 1);
                std::iota(dense.begin(), dense.end(), 0);
                srow = dense.data();
                n = i + 1;
            }
            for (int h = 0; h < Hq; ++h) {
                const double l = support_attention(q, k, v, Hq, Hkv, d, i, h, srow, n,
                                                   out + (r * Hq + h) * (int64_t)d, s, js);
                if (lse) lse[r * Hq + h] = l;
            }
        }
    }
    return 0;
}

// Head-collapsed indexer support: score_ij = q_idx_i . k_idx_j (j <= i); top-min(k, i+1)
// with the same order and tie rule; score[r*k + t] = score of idx.
int orc_indexer_topk_rows(int64_t N, int d_idx, const float* qx, const float* kx,
                          const int64_t* rows, int64_t nrows, int budget, int32_t* idx,
                          int32_t* len, double* score) {
    if (N <= 0 || d_idx <= 0 || budget < 1) return 1;
#pragma omp parallel
    {
        std::vector<double> s(N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            const int64_t i = rows[r];
            const float* qi = qx + i * d_idx;
            for (int64_t j = 0; j <= i; ++j) {
                const float* kj = kx + j * d_idx;
                double acc = 0.0;
                for (int c = 0; c < d_idx; ++c) acc += (double)qi[c] * (double)kj[c];
                s[j] = acc;
            }
            int32_t* ir = idx + r * budget;
            std::fill(ir, ir + budget, -1);
            const int n = select_top(s.data(), i + 1, budget, ir);
            len[r] = n;
            for (int t = 0; t < budget; ++t) score[r * budget + t] = (t < n) ? s[ir[t]] : 0.0;
        }
    }
    return 0;
}

// Block-shared indexer support ("fused selection-block-shared support", Abstract;
// technical report section 3.2, per-query vs fused path): the indexer's scores define
// one distribution per query, q_i[j] = softmax_{j <= i}(q_idx_i . k_idx_j) (no scale),
// and a block of consecutive queries shares the top-k of their sum, exactly as the
// block-shared oracle does with the head-averaged mass:
//   M_b[j] = sum_{i in block b, i >= j} q_i[j],  S_b = top-min(k, e_b+1) of M_b.
// M[r*N + j] for the listed blocks (0 beyond e_b).
int orc_indexer_block_mass(int64_t N, int d_idx, const float* qx, const float* kx, int block_q,
                           const int64_t* blocks, int64_t nblocks, double* M) {
    if (N <= 0 || d_idx <= 0 || block_q < 1) return 1;
#pragma omp parallel
    {
        std::vector<double> s(N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nblocks; ++r) {
            const int64_t b0 = blocks[r] * block_q;
            const int64_t e = std::min<int64_t>(N, b0 + block_q) - 1;
            double* Mr = M + r * N;
            std::fill(Mr, Mr + N, 0.0);
            for (int64_t i = b0; i <= e; ++i) {
                const float* qi = qx + i * d_idx;
                for (int64_t j = 0; j <= i; ++j) {
                    const float* kj = kx + j * d_idx;
                    double acc = 0.0;
                    for (int c = 0; c < d_idx; ++c) acc += (double)qi[c] * (double)kj[c];
                    s[j] = acc;
                }
                const double lse = log_sum_exp(s.data(), i + 1);
                for (int64_t j = 0; j <= i; ++j) Mr[j] += std::exp(s[j] - lse);
            }
        }
    }
    return 0;
}

// S_b for the listed blocks; layout as orc_block_topk (mass[r*k + t] = M_b[idx]).
int orc_indexer_block_topk(int64_t N, int d_idx, const float* qx, const float* kx, int block_q,
                           const int64_t* blocks, int64_t nblocks, int budget, int32_t* idx,
                           int32_t* len, double* mass) {
    if (budget < 1) return 1;
    std::vector<double> M((size_t)nblocks * N);
    int rc = orc_indexer_block_mass(N, d_idx, qx, kx, block_q, blocks, nblocks, M.data());
    if (rc) return rc;
    for (int64_t r = 0; r < nblocks; ++r) {
        const int64_t e = std::min<int64_t>(N, (blocks[r] + 1) * block_q) - 1;
        int32_t* ir = idx + r * budget;
        std::fill(ir, ir + budget, -1);
        const int n = select_top(M.data() + r * N, e + 1, budget, ir);
        len[r] = n;
        for (int t = 0; t < budget; ++t) mass[r * budget + t] = (t < n) ? M[r * N + ir[t]] : 0.0;
    }
    return 0;
}

// Distillation target of the indexer (technical report section 2.2, "Trainingsziel":
// the indexer is trained by KL divergence from the dense attention-mass distribution):
//   KL_i = sum_{j <= i} P_i[j] * log(P_i[j] / q_i[j]),
//   q_i[j] = softmax_{j <= i}(q_idx_i . k_idx_j)   (scale 1, as for the fused indexer),
// with 0 * log 0 = 0.  kl[r] for the listed rows.
int orc_distill_kl_rows(int64_t N, int Hq, int Hkv, int d, const float* q, const float* k,
                        int d_idx, const float* qx, const float* kx, const int64_t* rows,
                        int64_t nrows, double* kl) {
    if (!shape_ok(N, Hq, Hkv, d) || d_idx <= 0) return 1;
#pragma omp parallel
    {
        std::vector<double> s(N), P(N), t(N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            const int64_t i = rows[r];
            mass_row(q, k, Hq, Hkv, d, i, P.data(), s.data());
            const float* qi = qx + i * d_idx;
            for (int64_t j = 0; j <= i; ++j) {
                const float* kj = kx + j * d_idx;
                double acc = 0.0;
                for (int c = 0; c < d_idx; ++c) acc += (double)qi[c] * (double)kj[c];
                t[j] = acc;
            }
            const double lse = log_sum_exp(t.data(), i + 1);
            double sum = 0.0;
            for (int64_t j = 0; j <= i; ++j)
                if (P[j] > 0.0) sum += P[j] * (std::log(P[j]) - (t[j] - lse));
            kl[r] = sum;
        }
    }
    return 0;
}

// Budget sweep (technical report section 3.1, "Budget-Sensitivitaet": top-k budgets of
// 256 to 2048 compared on the same oracle): the support mass of query i at budget k is
// the sum of its k largest mass values, sum over S_i(k) of P_i[j].  out[r*nk + t] for
// budget ks[t], for the listed rows.
int orc_support_mass_curve(int64_t N, int Hq, int Hkv, int d, const float* q, const float* k,
                           const int64_t* rows, int64_t nrows, const int32_t* ks, int nk,
                           double* out) {
    if (!shape_ok(N, Hq, Hkv, d) || nk < 1) return 1;
    for (int t = 0; t < nk; ++t)
        if (ks[t] < 1) return 1;
#pragma omp parallel
    {
        std::vector<double> s(N), P(N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            const int64_t i = rows[r];
            mass_row(q, k, Hq, Hkv, d, i, P.data(), s.data());
            std::sort(P.begin(), P.begin() + i + 1, std::greater<double>());
            for (int t = 0; t < nk; ++t) {
                const int64_t n = std::min<int64_t>(ks[t], i + 1);
                double acc = 0.0;
                for (int64_t j = 0; j < n; ++j) acc += P[j];
                out[r * nk + t] = acc;
            }
        }
    }
    return 0;
}

}  // extern "C"
