// CUDA-core kernels of every step of the path, for any storage dtype.
//
// They are the fp32 path (fp32 inputs keep fp32 arithmetic: no tensor-core
// rounding), and they cover any shape the tensor-core kernels do not.  Each
// step is written the plain way: one warp or block per query row, exact block
// radix select over a staged mass row.
//
// Method: arXiv 2606.07703, Abstract and gist.science technical report §2.1
// (dense attention -> head-averaged mass -> top-k support -> recompute on the
// support) and §2.2 (head-collapsed indexer score -> top-k).
#include "common.cuh"
#include "launch.h"

namespace tam {

// ---------------------------------------------------------------- pass 1: per-head LSE
// One warp per (query row i, head h).  Lanes stride over keys; each keeps an online
// (max, sum) in the base-2 domain; the warp merges them at the end.
template <typename T>
__global__ void __launch_bounds__(256) k_lse_simt(const T* __restrict__ q, const T* __restrict__ k,
                                                  int N, int Hq, int Hkv, int d, float sl2,
                                                  float* __restrict__ lse) {
    extern __shared__ float sq[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const int i = blockIdx.x * 8 + warp;
    if (i >= N) return;
    const int g = h / (Hq / Hkv);
    float* qs = sq + warp * d;
    for (int c = lane; c < d; c += 32) qs[c] = to_f(q[((size_t)i * Hq + h) * d + c]);
    __syncwarp();
    float m = -INFINITY, l = 0.f;
    for (int j = lane; j <= i; j += 32) {
        const T* kj = k + ((size_t)j * Hkv + g) * d;
        float s = 0.f;
        for (int c = 0; c < d; ++c) s = fmaf(qs[c], to_f(kj[c]), s);
        s *= sl2;
        const float mn = fmaxf(m, s);
        l = l * exp2f(m - mn) + exp2f(s - mn);
        m = mn;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
        const float mn = fmaxf(m, m2);
        if (mn == -INFINITY) continue;
        l = (m == -INFINITY ? 0.f : l * exp2f(m - mn)) + (m2 == -INFINITY ? 0.f : l2 * exp2f(m2 - mn));
        m = mn;
    }
    if (lane == 0) lse[(size_t)h * N + i] = (m + log2f(l)) * kLn2;
}

// ---------------------------------------------------------------- pass 2: mass row + select
// Persistent blocks walk the selection units (query rows, or blocks of block_q rows)
// from the most expensive down.  For each unit the block stages the head-averaged
// mass row (or the block's summed mass row) in its private scratch row, then runs
// the exact block selection on it.
template <typename T>
__global__ void __launch_bounds__(256) k_mass_select_simt(
    const T* __restrict__ q, const T* __restrict__ k, const float* __restrict__ lse, int N, int Hq,
    int Hkv, int d, float sl2, int budget, int block_q, int n_sel, float* __restrict__ scratch,
    int32_t* __restrict__ sup_idx, int32_t* __restrict__ sup_len, float* __restrict__ sup_mass) {
    extern __shared__ float smem[];
    __shared__ SelectSmem sel;
    float* qs = smem;              // Hq * d
    float* lse2 = smem + Hq * d;   // Hq
    float* row = scratch + (size_t)blockIdx.x * N;
    const int G = Hq / Hkv;
    const float inv_hq = 1.f / (float)Hq;
    for (int u = n_sel - 1 - (int)blockIdx.x; u >= 0; u -= gridDim.x) {
        const int i0 = u * block_q;
        const int i1 = min(N, i0 + block_q) - 1;
        const int len = i1 + 1;
        for (int j = threadIdx.x; j < len; j += blockDim.x) row[j] = 0.f;
        for (int i = i0; i <= i1; ++i) {
            __syncthreads();
            for (int t = threadIdx.x; t < Hq * d; t += blockDim.x) qs[t] = to_f(q[(size_t)i * Hq * d + t]);
            for (int h = threadIdx.x; h < Hq; h += blockDim.x) lse2[h] = lse[(size_t)h * N + i] * kLog2e;
            __syncthreads();
            for (int j = threadIdx.x; j <= i; j += blockDim.x) {
                float p = 0.f;
                for (int h = 0; h < Hq; ++h) {
                    const T* kj = k + ((size_t)j * Hkv + h / G) * d;
                    const float* qh = qs + h * d;
                    float s = 0.f;
                    for (int c = 0; c < d; ++c) s = fmaf(qh[c], to_f(kj[c]), s);
                    p += exp2f(s * sl2 - lse2[h]);
                }
                row[j] += p * inv_hq;
            }
        }
        __syncthreads();
        block_select_topk(row, len, budget, sup_idx + (size_t)u * budget,
                          sup_mass + (size_t)u * budget, sup_len + u, sel);
    }
}

// ---------------------------------------------------------------- pass 3 / dense: row attention
// One block per query row; warp w takes heads w, w+8, ...  Each warp streams the row's
// support (or 0..i when sup_idx is null) in chunks of 32 keys with an online softmax;
// lanes own d/32 output channels.
template <typename T, int DPL>
__global__ void __launch_bounds__(256) k_attn_rows_simt(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, int N, int Hq,
    int Hkv, int d, float sl2, const int32_t* __restrict__ sup_idx,
    const int32_t* __restrict__ sup_len, int kmax, int block_q, T* __restrict__ out,
    float* __restrict__ lse) {
    extern __shared__ float qs[];   // Hq * d
    const int i = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = Hq / Hkv;
    for (int t = threadIdx.x; t < Hq * d; t += blockDim.x) qs[t] = to_f(q[(size_t)i * Hq * d + t]);
    __syncthreads();
    const int32_t* srow = nullptr;
    int n;
    if (sup_idx) {
        const int r = (block_q > 1) ? i / block_q : i;
        srow = sup_idx + (size_t)r * kmax;
        n = sup_len ? min(sup_len[r], kmax) : kmax;
    } else {
        n = i + 1;
    }
    for (int h = warp; h < Hq; h += 8) {
        const int g = h / G;
        const float* qh = qs + h * d;
        float m = -INFINITY, l = 0.f, acc[DPL];
#pragma unroll
        for (int c = 0; c < DPL; ++c) acc[c] = 0.f;
        for (int t0 = 0; t0 < n; t0 += 32) {
            const int t = t0 + lane;
            int j = -1;
            if (t < n) j = srow ? srow[t] : t;
            const bool valid = (j >= 0) && (j <= i);
            float s = -INFINITY;
            if (valid) {
                const T* kj = k + ((size_t)j * Hkv + g) * d;
                float a = 0.f;
                for (int c = 0; c < d; ++c) a = fmaf(qh[c], to_f(kj[c]), a);
                s = a * sl2;
            }
            const float mn = fmaxf(m, warp_max(s));
            if (mn == -INFINITY) continue;
            const float corr = (m == -INFINITY) ? 0.f : exp2f(m - mn);
            const float p = valid ? exp2f(s - mn) : 0.f;
            l = l * corr + warp_sum(p);
#pragma unroll
            for (int c = 0; c < DPL; ++c) acc[c] *= corr;
            for (int tt = 0; tt < 32; ++tt) {
                const float pt = __shfl_sync(0xffffffffu, p, tt);
                const int jt = __shfl_sync(0xffffffffu, j, tt);
                const int vt = __shfl_sync(0xffffffffu, valid ? 1 : 0, tt);
                if (!vt) continue;
                const T* vj = v + ((size_t)jt * Hkv + g) * d;
#pragma unroll
                for (int c = 0; c < DPL; ++c) acc[c] = fmaf(pt, to_f(vj[lane + 32 * c]), acc[c]);
            }
            m = mn;
        }
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        T* oh = out + ((size_t)i * Hq + h) * d;
#pragma unroll
        for (int c = 0; c < DPL; ++c) oh[lane + 32 * c] = from_f<T>(acc[c] * inv);
        if (lse && lane == 0) lse[(size_t)h * N + i] = (l > 0.f) ? (m + log2f(l)) * kLn2 : -INFINITY;
    }
}

// ---------------------------------------------------------------- indexer: score row + select
template <typename T>
__global__ void __launch_bounds__(256) k_indexer_select_simt(
    const T* __restrict__ qx, const T* __restrict__ kx, int N, int dx, int budget,
    float* __restrict__ scratch, int32_t* __restrict__ sup_idx, int32_t* __restrict__ sup_len,
    float* __restrict__ sup_score) {
    extern __shared__ float qs[];   // dx
    __shared__ SelectSmem sel;
    float* row = scratch + (size_t)blockIdx.x * N;
    for (int i = N - 1 - (int)blockIdx.x; i >= 0; i -= gridDim.x) {
        __syncthreads();
        for (int c = threadIdx.x; c < dx; c += blockDim.x) qs[c] = to_f(qx[(size_t)i * dx + c]);
        __syncthreads();
        for (int j = threadIdx.x; j <= i; j += blockDim.x) {
            const T* kj = kx + (size_t)j * dx;
            float s = 0.f;
            for (int c = 0; c < dx; ++c) s = fmaf(qs[c], to_f(kj[c]), s);
            row[j] = s;
        }
        __syncthreads();
        block_select_topk(row, i + 1, budget, sup_idx + (size_t)i * budget,
                          sup_score + (size_t)i * budget, sup_len + i, sel);
    }
}

// ---------------------------------------------------------------- fallback rows
// Rows whose streamed candidates could not be used (a threshold above the k-th value,
// or a full candidate segment): each persistent block takes rows off the list
// fb (fb[0] = count, fb[1 + t] = row), computes the whole row into its scratch row
// and selects from it exactly.
// Eight consecutive elements of a row as floats (one 16-byte load for bf16, two for fp32).
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&x)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
    }
}
__device__ __forceinline__ void load8(const float* p, float (&x)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// Thread = key: for each KV group it reads the key row in 16-byte pieces and adds the
// dot products of all G query heads of the group (at most kMaxG) at once, the query
// row staged in shared memory as fp32 (read as broadcasts).
constexpr int kMaxG = 16;

template <typename T>
__global__ void __launch_bounds__(256) k_mass_rows_fallback(
    const T* __restrict__ q, const T* __restrict__ k, const float* __restrict__ lse, int N, int Hq,
    int Hkv, int d, float sl2, int budget, const int32_t* __restrict__ fb,
    float* __restrict__ scratch, int32_t* __restrict__ sup_idx, int32_t* __restrict__ sup_len,
    float* __restrict__ sup_mass) {
    extern __shared__ float smem[];
    __shared__ SelectSmem sel;
    float* qs = smem;              // Hq * d
    float* lse2 = smem + Hq * d;   // Hq
    float* row = scratch + (size_t)blockIdx.x * N;
    const int G = Hq / Hkv;
    const float inv_hq = 1.f / (float)Hq;
    const int n_fb = fb[0];
    for (int t = blockIdx.x; t < n_fb; t += gridDim.x) {
        const int i = fb[1 + t];
        __syncthreads();
        for (int x = threadIdx.x; x < Hq * d; x += blockDim.x) qs[x] = to_f(q[(size_t)i * Hq * d + x]);
        for (int h = threadIdx.x; h < Hq; h += blockDim.x) lse2[h] = lse[(size_t)h * N + i] * kLog2e;
        __syncthreads();
        for (int j = threadIdx.x; j <= i; j += blockDim.x) {
            float p = 0.f;
            for (int g = 0; g < Hkv; ++g) {
                const T* kj = k + ((size_t)j * Hkv + g) * d;
                const float* qg = qs + (size_t)g * G * d;
                float dot[kMaxG];
#pragma unroll
                for (int hh = 0; hh < kMaxG; ++hh) dot[hh] = 0.f;
                for (int c = 0; c < d; c += 8) {
                    float kv[8];
                    load8(kj + c, kv);
#pragma unroll
                    for (int hh = 0; hh < kMaxG; ++hh) {
                        if (hh < G) {
                            const float* qh = qg + hh * d + c;
#pragma unroll
                            for (int e = 0; e < 8; ++e) dot[hh] = fmaf(qh[e], kv[e], dot[hh]);
                        }
                    }
                }
#pragma unroll
                for (int hh = 0; hh < kMaxG; ++hh)
                    if (hh < G) p += exp2f(dot[hh] * sl2 - lse2[g * G + hh]);
            }
            row[j] = p * inv_hq;
        }
        __syncthreads();
        block_select_topk(row, i + 1, budget, sup_idx + (size_t)i * budget,
                          sup_mass + (size_t)i * budget, sup_len + i, sel);
    }
}

template <typename T>
__global__ void __launch_bounds__(256) k_indexer_rows_fallback(
    const T* __restrict__ qx, const T* __restrict__ kx, int dx, int budget,
    const int32_t* __restrict__ fb, int N, float* __restrict__ scratch,
    int32_t* __restrict__ sup_idx, int32_t* __restrict__ sup_len, float* __restrict__ sup_score) {
    extern __shared__ float qs[];   // dx
    __shared__ SelectSmem sel;
    float* row = scratch + (size_t)blockIdx.x * N;
    const int n_fb = fb[0];
    for (int t = blockIdx.x; t < n_fb; t += gridDim.x) {
        const int i = fb[1 + t];
        __syncthreads();
        for (int c = threadIdx.x; c < dx; c += blockDim.x) qs[c] = to_f(qx[(size_t)i * dx + c]);
        __syncthreads();
        for (int j = threadIdx.x; j <= i; j += blockDim.x) {
            const T* kj = kx + (size_t)j * dx;
            float sc = 0.f;
            for (int c = 0; c < dx; c += 8) {
                float kv[8];
                load8(kj + c, kv);
#pragma unroll
                for (int e = 0; e < 8; ++e) sc = fmaf(qs[c + e], kv[e], sc);
            }
            row[j] = sc;
        }
        __syncthreads();
        block_select_topk(row, i + 1, budget, sup_idx + (size_t)i * budget,
                          sup_score + (size_t)i * budget, sup_len + i, sel);
    }
}

// ---------------------------------------------------------------- launchers
template <typename T>
static cudaError_t launch_lse(const LseArgs& a, cudaStream_t st) {
    dim3 grid((unsigned)((a.N + 7) / 8), (unsigned)a.Hq);
    k_lse_simt<T><<<grid, 256, 8 * a.d * sizeof(float), st>>>(
        (const T*)a.q, (const T*)a.k, (int)a.N, a.Hq, a.Hkv, a.d, a.sl2, a.lse);
    note_launch();
    return cudaGetLastError();
}

cudaError_t simt_lse(const LseArgs& a, cudaStream_t st) {
    return a.dtype == TAM_F32 ? launch_lse<float>(a, st) : launch_lse<__nv_bfloat16>(a, st);
}

template <typename T>
static cudaError_t launch_mass(const MassArgs& a, cudaStream_t st) {
    const size_t smem = (size_t)(a.Hq * a.d + a.Hq) * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_mass_select_simt<T>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k_mass_select_simt<T><<<a.n_ctas, 256, smem, st>>>(
        (const T*)a.q, (const T*)a.k, a.lse, (int)a.N, a.Hq, a.Hkv, a.d, a.sl2, a.budget, a.block_q,
        a.n_sel, a.scratch, a.sup_idx, a.sup_len, a.sup_mass);
    note_launch();
    return cudaGetLastError();
}

cudaError_t simt_mass_select(const MassArgs& a, cudaStream_t st) {
    return a.dtype == TAM_F32 ? launch_mass<float>(a, st) : launch_mass<__nv_bfloat16>(a, st);
}

template <typename T, int DPL>
static cudaError_t launch_attn_t(const AttnArgs& a, cudaStream_t st) {
    const size_t smem = (size_t)a.Hq * a.d * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_attn_rows_simt<T, DPL>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k_attn_rows_simt<T, DPL><<<(unsigned)a.N, 256, smem, st>>>(
        (const T*)a.q, (const T*)a.k, (const T*)a.v, (int)a.N, a.Hq, a.Hkv, a.d, a.sl2, a.sup_idx,
        a.sup_len, a.kmax, a.block_q, (T*)a.out, a.lse);
    note_launch();
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st) {
    switch (a.d) {
        case 64: return launch_attn_t<T, 2>(a, st);
        case 128: return launch_attn_t<T, 4>(a, st);
        case 256: return launch_attn_t<T, 8>(a, st);
        default: return cudaErrorNotSupported;
    }
}

cudaError_t simt_attention(const AttnArgs& a, cudaStream_t st) {
    return a.dtype == TAM_F32 ? launch_attn<float>(a, st) : launch_attn<__nv_bfloat16>(a, st);
}

template <typename T>
static cudaError_t launch_indexer(const IndexerArgs& a, cudaStream_t st) {
    k_indexer_select_simt<T><<<a.n_ctas, 256, a.d_idx * sizeof(float), st>>>(
        (const T*)a.q_idx, (const T*)a.k_idx, (int)a.N, a.d_idx, a.budget, a.scratch, a.sup_idx,
        a.sup_len, a.sup_score);
    note_launch();
    return cudaGetLastError();
}

cudaError_t simt_indexer_select(const IndexerArgs& a, cudaStream_t st) {
    return a.dtype == TAM_F32 ? launch_indexer<float>(a, st) : launch_indexer<__nv_bfloat16>(a, st);
}

template <typename T>
static cudaError_t launch_mass_fallback(const MassArgs& a, const int32_t* fb, float* scratch,
                                        int n_ctas, cudaStream_t st) {
    const size_t smem = (size_t)(a.Hq * a.d + a.Hq) * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_mass_rows_fallback<T>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k_mass_rows_fallback<T><<<n_ctas, 256, smem, st>>>(
        (const T*)a.q, (const T*)a.k, a.lse, (int)a.N, a.Hq, a.Hkv, a.d, a.sl2, a.budget, fb,
        scratch, a.sup_idx, a.sup_len, a.sup_mass);
    note_launch();
    return cudaGetLastError();
}

cudaError_t fallback_mass_rows(const MassArgs& a, const int32_t* fb, float* scratch, int n_ctas,
                               cudaStream_t st) {
    // the fallback reads rows in 8-element pieces and holds one dot product per head of a group
    if (n_ctas < 1 || a.d % 8 != 0 || a.Hq / a.Hkv > kMaxG) return cudaErrorInvalidValue;
    return a.dtype == TAM_F32 ? launch_mass_fallback<float>(a, fb, scratch, n_ctas, st)
                              : launch_mass_fallback<__nv_bfloat16>(a, fb, scratch, n_ctas, st);
}

template <typename T>
static cudaError_t launch_indexer_fallback(const IndexerArgs& a, const int32_t* fb,
                                           float* scratch, int n_ctas, cudaStream_t st) {
    k_indexer_rows_fallback<T><<<n_ctas, 256, a.d_idx * sizeof(float), st>>>(
        (const T*)a.q_idx, (const T*)a.k_idx, a.d_idx, a.budget, fb, (int)a.N, scratch, a.sup_idx,
        a.sup_len, a.sup_score);
    note_launch();
    return cudaGetLastError();
}

cudaError_t fallback_indexer_rows(const IndexerArgs& a, const int32_t* fb, float* scratch,
                                  int n_ctas, cudaStream_t st) {
    if (n_ctas < 1 || a.d_idx % 8 != 0) return cudaErrorInvalidValue;
    return a.dtype == TAM_F32 ? launch_indexer_fallback<float>(a, fb, scratch, n_ctas, st)
                              : launch_indexer_fallback<__nv_bfloat16>(a, fb, scratch, n_ctas, st);
}

}  // namespace tam
