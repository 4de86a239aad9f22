// Stand-alone self-test of the fp64 oracle (test infrastructure only).
//
// Built with g++ together with oracle.cpp and run by tests/test_oracle_cpp.py.
// Each check ties the oracle to something other than itself: a direct evaluation
// written out here (exp and sum without a log-sum-exp), a closed form, or an
// invariant of the method (arXiv 2606.07703, Abstract; gist.science technical
// report §2.1: dense attention -> head-averaged mass -> top-k support -> attention
// recomputed on the support).  Exit status 0 and "all passed" on success; with a
// planted mistake (argument 1..4) it must report failures.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <vector>

extern "C" {
void orc_set_mutation(int m);
int orc_mass_rows(int64_t N, int Hq, int Hkv, int d, const float* q, const float* k,
                  const int64_t* rows, int64_t nrows, double* P);
int orc_topk_rows(int64_t N, int Hq, int Hkv, int d, const float* q, const float* k,
                  const int64_t* rows, int64_t nrows, int budget, int32_t* idx, int32_t* len,
                  double* mass);
int orc_block_topk(int64_t N, int Hq, int Hkv, int d, const float* q, const float* k, int block_q,
                   const int64_t* blocks, int64_t nblocks, int budget, int32_t* idx, int32_t* len,
                   double* mass);
int orc_attn_rows(int64_t N, int Hq, int Hkv, int d, const float* q, const float* k,
                  const float* v, const int64_t* rows, int64_t nrows, const int32_t* sup,
                  const int32_t* sup_len, int64_t sup_stride, double* out, double* lse);
}

namespace {

int g_failed = 0;

void expect(bool ok, const char* what, int64_t a = -1, int64_t b = -1) {
    if (!ok) {
        std::printf("FAILED: %s (%lld, %lld)\n", what, (long long)a, (long long)b);
        ++g_failed;
    }
}

// Deterministic N(0,1) draws: a 64-bit LCG (Knuth's MMIX constants) and Box-Muller.
struct Gauss {
    uint64_t s;
    explicit Gauss(uint64_t seed) : s(seed * 2862933555777941757ull + 3037000493ull) {}
    double uniform() {
        s = s * 6364136223846793005ull + 1442695040888963407ull;
        return ((s >> 11) + 0.5) * (1.0 / 9007199254740992.0);
    }
    float next() {
        const double u1 = uniform(), u2 = uniform();
        return (float)(std::sqrt(-2.0 * std::log(u1)) * std::cos(6.283185307179586 * u2));
    }
};

std::vector<float> draw(size_t n, uint64_t seed) {
    Gauss g(seed);
    std::vector<float> x(n);
    for (auto& e : x) e = g.next();
    return x;
}

std::vector<int64_t> all_rows(int64_t n) {
    std::vector<int64_t> r(n);
    for (int64_t i = 0; i < n; ++i) r[i] = i;
    return r;
}

// Head-averaged mass written out directly: exp of each score over the sum of exps
// (scores are O(1) here, so no shift is needed), averaged over the query heads.
void direct_mass(int N, int Hq, int Hkv, int d, const std::vector<float>& q,
                 const std::vector<float>& k, std::vector<double>& P) {
    const int G = Hq / Hkv;
    P.assign((size_t)N * N, 0.0);
    for (int i = 0; i < N; ++i)
        for (int h = 0; h < Hq; ++h) {
            std::vector<double> e(i + 1);
            double z = 0;
            for (int j = 0; j <= i; ++j) {
                double s = 0;
                for (int c = 0; c < d; ++c)
                    s += (double)q[((size_t)i * Hq + h) * d + c] *
                         (double)k[((size_t)j * Hkv + h / G) * d + c];
                e[j] = std::exp(s / std::sqrt((double)d));
                z += e[j];
            }
            for (int j = 0; j <= i; ++j) P[(size_t)i * N + j] += e[j] / z / Hq;
        }
}

}  // namespace

// argv[1] (optional): plant one of the oracle's known mistakes first; the run must fail.
int main(int argc, char** argv) {
    if (argc > 1) orc_set_mutation(std::atoi(argv[1]));
    const int N = 40, Hq = 4, Hkv = 2, d = 8;
    auto q = draw((size_t)N * Hq * d, 1), k = draw((size_t)N * Hkv * d, 2),
         v = draw((size_t)N * Hkv * d, 3);
    const auto rows = all_rows(N);

    // 1. mass against the direct evaluation; rows sum to one; nothing after the query
    std::vector<double> P((size_t)N * N), Pd;
    expect(orc_mass_rows(N, Hq, Hkv, d, q.data(), k.data(), rows.data(), N, P.data()) == 0,
           "mass_rows accepted");
    direct_mass(N, Hq, Hkv, d, q, k, Pd);
    for (int i = 0; i < N; ++i) {
        double sum = 0;
        for (int j = 0; j < N; ++j) {
            const double p = P[(size_t)i * N + j];
            expect(std::fabs(p - Pd[(size_t)i * N + j]) <= 1e-12, "mass = direct", i, j);
            if (j > i) expect(p == 0.0, "no mass after the query", i, j);
            sum += p;
        }
        expect(std::fabs(sum - 1.0) <= 1e-12, "row sums to 1", i);
    }

    // 2. supports: the k largest by value (ties -> smaller index), ascending, and
    //    nested in k with non-decreasing support mass
    double prev_mass[N] = {};
    std::vector<int32_t> prev_idx;
    std::vector<int32_t> prev_len;
    for (int budget = 1; budget <= 6; ++budget) {
        std::vector<int32_t> idx((size_t)N * budget), len(N);
        std::vector<double> ms((size_t)N * budget);
        orc_topk_rows(N, Hq, Hkv, d, q.data(), k.data(), rows.data(), N, budget, idx.data(),
                      len.data(), ms.data());
        for (int i = 0; i < N; ++i) {
            const int n = len[i];
            expect(n == std::min(budget, i + 1), "support size min(k, i+1)", i, budget);
            double smass = 0, m_k = 1e300;
            for (int t = 0; t < n; ++t) {
                const int j = idx[(size_t)i * budget + t];
                if (t) expect(j > idx[(size_t)i * budget + t - 1], "ascending", i, t);
                smass += P[(size_t)i * N + j];
                m_k = std::min(m_k, P[(size_t)i * N + j]);
            }
            // every key left out has mass <= the smallest kept one
            for (int j = 0; j <= i; ++j) {
                bool in = false;
                for (int t = 0; t < n; ++t) in |= idx[(size_t)i * budget + t] == j;
                if (!in) expect(P[(size_t)i * N + j] <= m_k, "left-out key below the support", i, j);
            }
            expect(smass + 1e-15 >= prev_mass[i], "support mass non-decreasing in k", i, budget);
            prev_mass[i] = smass;
            if (budget > 1)   // S(k-1) is contained in S(k)
                for (int t = 0; t < prev_len[i]; ++t) {
                    const int j = prev_idx[(size_t)i * (budget - 1) + t];
                    bool in = false;
                    for (int u = 0; u < n; ++u) in |= idx[(size_t)i * budget + u] == j;
                    expect(in, "supports nested in k", i, j);
                }
        }
        prev_idx = idx;
        prev_len = len;
    }

    // 3. block of one query equals per query
    {
        const int budget = 5;
        std::vector<int32_t> a((size_t)N * budget), la(N), b((size_t)N * budget), lb(N);
        std::vector<double> ma((size_t)N * budget), mb((size_t)N * budget);
        orc_topk_rows(N, Hq, Hkv, d, q.data(), k.data(), rows.data(), N, budget, a.data(),
                      la.data(), ma.data());
        orc_block_topk(N, Hq, Hkv, d, q.data(), k.data(), 1, rows.data(), N, budget, b.data(),
                       lb.data(), mb.data());
        for (size_t t = 0; t < a.size(); ++t) expect(a[t] == b[t], "block of one = per query", t);
    }

    // 4. a budget covering the prefix reproduces dense attention
    {
        const int budget = N;
        std::vector<int32_t> idx((size_t)N * budget), len(N);
        std::vector<double> ms((size_t)N * budget);
        orc_topk_rows(N, Hq, Hkv, d, q.data(), k.data(), rows.data(), N, budget, idx.data(),
                      len.data(), ms.data());
        std::vector<double> o1((size_t)N * Hq * d), l1((size_t)N * Hq), o2(o1.size()), l2(l1.size());
        orc_attn_rows(N, Hq, Hkv, d, q.data(), k.data(), v.data(), rows.data(), N, idx.data(),
                      len.data(), budget, o1.data(), l1.data());
        orc_attn_rows(N, Hq, Hkv, d, q.data(), k.data(), v.data(), rows.data(), N, nullptr,
                      nullptr, 0, o2.data(), l2.data());
        for (size_t t = 0; t < o1.size(); ++t)
            expect(std::fabs(o1[t] - o2[t]) <= 1e-12, "k >= i+1 equals dense", t);
    }

    // 5. Q = 0: every key of the prefix has mass 1/(i+1), the support is the first k keys
    //    (ties -> smaller index), and the output is the mean of V over them
    {
        std::vector<float> z(q.size(), 0.f);
        const int budget = 7;
        std::vector<int32_t> idx((size_t)N * budget), len(N);
        std::vector<double> ms((size_t)N * budget);
        orc_topk_rows(N, Hq, Hkv, d, z.data(), k.data(), rows.data(), N, budget, idx.data(),
                      len.data(), ms.data());
        std::vector<double> o((size_t)N * Hq * d), l((size_t)N * Hq);
        orc_attn_rows(N, Hq, Hkv, d, z.data(), k.data(), v.data(), rows.data(), N, idx.data(),
                      len.data(), budget, o.data(), l.data());
        const int G = Hq / Hkv;
        for (int i = 0; i < N; ++i) {
            const int n = std::min(budget, i + 1);
            for (int t = 0; t < n; ++t) {
                expect(idx[(size_t)i * budget + t] == t, "Q=0 support = first keys", i, t);
                expect(std::fabs(ms[(size_t)i * budget + t] - 1.0 / (i + 1)) <= 1e-15,
                       "Q=0 mass = 1/(i+1)", i, t);
            }
            for (int h = 0; h < Hq; ++h)
                for (int c = 0; c < d; ++c) {
                    double mean = 0;
                    for (int j = 0; j < n; ++j) mean += v[((size_t)j * Hkv + h / G) * d + c];
                    mean /= n;
                    expect(std::fabs(o[((size_t)i * Hq + h) * d + c] - mean) <= 1e-12,
                           "Q=0 output = mean of V", i, h);
                }
        }
    }

    if (g_failed) {
        std::printf("%d checks failed\n", g_failed);
        return 1;
    }
    std::printf("all passed\n");
    return 0;
}
