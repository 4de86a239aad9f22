// Shared step of the pass-2 mass kernels (mass2sm_tc.cu, mass_tc.cu): the head-summed
// probabilities of one key row over four consecutive (query, head) columns,
//
//   acc[query] += exp2(score * scale*log2(e) - lse[head, query] * log2(e)),
//
// in packed f32x2 arithmetic (one fma.rn.f32x2 per column pair for the scale-and-shift,
// one add.rn.f32x2 per pair into the accumulators), with one column pair in four
// exponentiated on the FMA pipe and the rest on MUFU.  Both kernels use it so that they
// give the same mass bit for bit.
//
// Columns are (query, head) with the head fastest.  For G >= 4 heads per KV group the
// four columns are heads of one query: the two pairs are added packed and the pair's
// halves into the query's fp32 sum.  For G = 2 a pair holds two heads of one query and
// the query's packed accumulator keeps two partial sums (lo, hi), added at the end; for
// G = 1 a pair holds two queries and its accumulator their two sums.
#pragma once

#include "tc_ptx.cuh"

namespace tam {

// head sums of kQP queries (fp32 for G >= 4, packed pairs below)
template <int G, int kQP>
struct MassAcc {
    static constexpr int N = G >= 4 ? 1 : (G >= 2 ? kQP : kQP / 2);
    uint64_t v[N];
    float s[G >= 4 ? kQP : 1];
    __device__ __forceinline__ void clear() {
#pragma unroll
        for (int a = 0; a < N; ++a) v[a] = 0ull;
#pragma unroll
        for (int a = 0; a < (G >= 4 ? kQP : 1); ++a) s[a] = 0.f;
    }
    __device__ __forceinline__ float get(int q) const {
        float lo, hi;
        if constexpr (G >= 4) {
            return s[q];
        } else if constexpr (G >= 2) {
            tc::f2_unpack(v[q], lo, hi);
            return lo + hi;
        } else {
            tc::f2_unpack(v[q >> 1], lo, hi);
            return (q & 1) ? hi : lo;
        }
    }
};

// Columns col .. col+3 (col a multiple of 4): raw scores s0..s3 (fp32 bits), the negated
// log2-domain lse of the four columns as two packed pairs, sl2x2 = (scale*log2e) twice.
// `poly`: this group of four sends its second pair through the FMA-pipe exp2.
template <int G, int kQP>
__device__ __forceinline__ void mass_columns4(MassAcc<G, kQP>& acc, int col, uint32_t s0,
                                              uint32_t s1, uint32_t s2, uint32_t s3,
                                              uint64_t nl01, uint64_t nl23, uint64_t sl2x2,
                                              bool poly) {
    const uint64_t x01 = tc::f2_fma(tc::f2_pack(__uint_as_float(s0), __uint_as_float(s1)),
                                    sl2x2, nl01);
    const uint64_t x23 = tc::f2_fma(tc::f2_pack(__uint_as_float(s2), __uint_as_float(s3)),
                                    sl2x2, nl23);
    float x0, x1, x2, x3, y0, y1, y2, y3;
    tc::f2_unpack(x01, x0, x1);
    tc::f2_unpack(x23, x2, x3);
    y0 = tc::ex2(x0);
    y1 = tc::ex2(x1);
    if (poly) {
        tc::ex2_fma2(x2, x3, y2, y3);
    } else {
        y2 = tc::ex2(x2);
        y3 = tc::ex2(x3);
    }
    const uint64_t p01 = tc::f2_pack(y0, y1), p23 = tc::f2_pack(y2, y3);
    if constexpr (G >= 4) {
        // all four columns belong to query col / G
        const int q = col / G;
        float lo, hi;
        tc::f2_unpack(tc::f2_add(p01, p23), lo, hi);
        acc.s[q] += lo + hi;
    } else {
        // G = 2: one query per pair; G = 1: two queries per pair (accumulator col / 2
        // holds columns col, col + 1 either way)
        acc.v[col / 2] = tc::f2_add(acc.v[col / 2], p01);
        acc.v[col / 2 + 1] = tc::f2_add(acc.v[col / 2 + 1], p23);
    }
}

}  // namespace tam
