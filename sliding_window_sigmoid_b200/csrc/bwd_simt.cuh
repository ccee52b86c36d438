// bwd_simt.cuh — CUDA-core backward (exact fp32 arithmetic; any even d <= 128).
//
// Gradients of the SWAT attention equation ("SWAT" page, "Balanced ALiBi"),
// derived by calculus (the pages print no backward):
//   dv_j = sum_i p_ij dO_i,      dP_ij = dO_i . v_j
//   sigmoid: dS_ij = dP_ij p_ij (1 - p_ij)
//   softmax: dS_ij = p_ij (dP_ij - D_i), D_i = dO_i . o_i
//   dq'_i = sum_j dS_ij k'_j / sqrt(d),  dk'_j = sum_i dS_ij q'_i / sqrt(d)
//   dq = R_i^T dq',  dk = R_j^T dk'
// Two kernels, no atomics: a query-stationary one for dq, a key-stationary
// one for dk and dv (which sums the query heads of a KV group).
#pragma once
#include "common.cuh"
#include "fwd_simt.cuh"

namespace swat {

struct BwdArgs {
    const void *q, *k, *v, *o, *dout;
    const float *lse;
    void *dq, *dk, *dv;
    float *Dws;          // [B,H,N] fp32, softmax mode
    const float *slopes;
    int B, H, Hkv, N, d, window, n_sink, mode;
    double log2_base;
    int use_rope;
    float scale;
};

// D_i = dO_i . o_i (softmax mode), one warp per row.
template <typename T>
__global__ void swat_bwd_dot_do_o_kernel(BwdArgs a)
{
    long long row = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    int lane = threadIdx.x % 32;
    long long total = (long long)a.B * a.N * a.H;
    if (row >= total) return;
    // row enumerates (b, i, h) in BSHD order
    const T *o = (const T *)a.o + (size_t)row * a.d;
    const T *dO = (const T *)a.dout + (size_t)row * a.d;
    float s = 0.f;
    for (int c = lane; c < a.d; c += 32) s = fmaf(to_f(o[c]), to_f(dO[c]), s);
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) {
        long long h = row % a.H, bi = row / a.H, i = bi % a.N, b = bi / a.N;
        a.Dws[((size_t)b * a.H + h) * a.N + i] = s;
    }
}

__device__ __forceinline__ float simt_weight(float s, float lse_or_zero, int mode)
{
    return mode == SWAT_MODE_SIGMOID_ ? sigmoid_exact(s) : expf(s - lse_or_zero);
}

__device__ __forceinline__ float simt_dscore(float p, float dP, float D, int mode)
{
    return mode == SWAT_MODE_SIGMOID_ ? dP * p * (1.f - p) : p * (dP - D);
}

// Raw (unrotated) rows into smem as fp32.
template <typename T>
__device__ void simt_load_plain(float *dst, int ld, const T *src, long long p0, int rows, int N,
                                size_t rs, int d)
{
    for (int e = threadIdx.x; e < rows * d; e += blockDim.x) {
        int r = e / d, c = e % d;
        long long p = p0 + r;
        dst[r * ld + c] = (p < N) ? to_f(src[(size_t)p * rs + c]) : 0.f;
    }
}

template <typename T>
__global__ void __launch_bounds__(SIMT_THREADS)
swat_bwd_dq_simt_kernel(BwdArgs a)
{
    extern __shared__ float smem[];
    const int d = a.d, ld = SIMT_DMAX + 1;
    float *Qs = smem;                   // rotated q
    float *dOs = Qs + SIMT_BQ * ld;
    float *Ks = dOs + SIMT_BQ * ld;     // rotated k
    float *Vs = Ks + SIMT_BK * ld;
    float *dSs = Vs + SIMT_BK * ld;     // [BQ][BK+1]
    float *rowA = dSs + SIMT_BQ * (SIMT_BK + 1);  // lse
    float *rowD = rowA + SIMT_BQ;

    const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int G = a.H / a.Hkv, kvh = h / G;
    const long long i0 = (long long)qb * SIMT_BQ;
    const size_t rsq = (size_t)a.H * d, rsk = (size_t)a.Hkv * d;
    const T *q = (const T *)a.q + ((size_t)b * a.N * a.H + h) * d;
    const T *dO = (const T *)a.dout + ((size_t)b * a.N * a.H + h) * d;
    const T *k = (const T *)a.k + ((size_t)b * a.N * a.Hkv + kvh) * d;
    const T *v = (const T *)a.v + ((size_t)b * a.N * a.Hkv + kvh) * d;
    const float slope = a.slopes ? a.slopes[h] : 0.f;

    simt_load_rows<T>(Qs, ld, q, i0, SIMT_BQ, a.N, rsq, d, a.use_rope, a.log2_base);
    simt_load_plain<T>(dOs, ld, dO, i0, SIMT_BQ, a.N, rsq, d);
    if (threadIdx.x < SIMT_BQ) {
        long long i = i0 + threadIdx.x;
        bool ok = i < a.N && a.mode == SWAT_MODE_SOFTMAX_;
        rowA[threadIdx.x] = ok ? a.lse[((size_t)b * a.H + h) * a.N + i] : 0.f;
        rowD[threadIdx.x] = ok ? a.Dws[((size_t)b * a.H + h) * a.N + i] : 0.f;
    }
    const int r_o = threadIdx.x / 8, c_o = threadIdx.x % 8;
    float acc[SIMT_DMAX / 8];
#pragma unroll
    for (int u = 0; u < SIMT_DMAX / 8; ++u) acc[u] = 0.f;

    const long long i_last = min((long long)a.N - 1, i0 + SIMT_BQ - 1);
    const long long kstart = max(0LL, i0 - a.window + 1);
    const long long kstart_al = (kstart / SIMT_BK) * SIMT_BK;
    const long long sink_end = min((long long)a.n_sink, kstart_al);
    const long long n_sink_tiles = (sink_end + SIMT_BK - 1) / SIMT_BK;
    const long long n_band_tiles = (i_last - kstart_al) / SIMT_BK + 1;
    __syncthreads();

    for (long long tt = 0; tt < n_sink_tiles + n_band_tiles; ++tt) {
        const long long j0 = tt < n_sink_tiles ? tt * SIMT_BK : kstart_al + (tt - n_sink_tiles) * SIMT_BK;
        simt_load_rows<T>(Ks, ld, k, j0, SIMT_BK, a.N, rsk, d, a.use_rope, a.log2_base);
        simt_load_plain<T>(Vs, ld, v, j0, SIMT_BK, a.N, rsk, d);
        __syncthreads();
        for (int e = threadIdx.x; e < SIMT_BQ * SIMT_BK; e += blockDim.x) {
            int r = e / SIMT_BK, c = e % SIMT_BK;
            long long i = i0 + r, j = j0 + c;
            float ds = 0.f;
            if (i < a.N && in_keyset(i, j, a.window, a.n_sink)) {
                float dot = 0.f, dp = 0.f;
                for (int x = 0; x < d; ++x) {
                    dot = fmaf(Qs[r * ld + x], Ks[c * ld + x], dot);
                    dp = fmaf(dOs[r * ld + x], Vs[c * ld + x], dp);
                }
                float s = dot * a.scale + slope * (float)(i - j);
                float p = simt_weight(s, rowA[r], a.mode);
                ds = simt_dscore(p, dp, rowD[r], a.mode);
            }
            dSs[r * (SIMT_BK + 1) + c] = ds;
        }
        __syncthreads();
        for (int c = 0; c < SIMT_BK; ++c) {
            float ds = dSs[r_o * (SIMT_BK + 1) + c];
#pragma unroll
            for (int u = 0; u < SIMT_DMAX / 8; ++u) {
                int col = c_o + 8 * u;
                if (col < d) acc[u] = fmaf(ds, Ks[c * ld + col], acc[u]);
            }
        }
        __syncthreads();
    }
    // rotated-space dq' -> smem, then R^T per pair
#pragma unroll
    for (int u = 0; u < SIMT_DMAX / 8; ++u) {
        int col = c_o + 8 * u;
        if (col < d) Qs[r_o * ld + col] = acc[u] * a.scale;
    }
    __syncthreads();
    T *dq = (T *)a.dq + ((size_t)b * a.N * a.H + h) * d;
    const int half = d / 2;
    for (int e = threadIdx.x; e < SIMT_BQ * half; e += blockDim.x) {
        int r = e / half, t = e % half;
        long long i = i0 + r;
        if (i >= a.N) continue;
        float x0 = Qs[r * ld + 2 * t], x1 = Qs[r * ld + 2 * t + 1], y0 = x0, y1 = x1;
        if (a.use_rope) {
            float c, s;
            rope_cos_sin(i, rope_theta(t, d, a.log2_base), c, s);
            rope_pair_inv(x0, x1, c, s, y0, y1);
        }
        dq[(size_t)i * rsq + 2 * t] = from_f<T>(y0);
        dq[(size_t)i * rsq + 2 * t + 1] = from_f<T>(y1);
    }
}

template <typename T>
__global__ void __launch_bounds__(SIMT_THREADS)
swat_bwd_dkdv_simt_kernel(BwdArgs a)
{
    extern __shared__ float smem[];
    const int d = a.d, ld = SIMT_DMAX + 1;
    float *Ks = smem;                   // rotated k (this CTA's keys)
    float *Vs = Ks + SIMT_BK * ld;
    float *Qs = Vs + SIMT_BK * ld;      // rotated q (current query tile)
    float *dOs = Qs + SIMT_BQ * ld;
    float *Pt = dOs + SIMT_BQ * ld;     // [BK][BQ+1]  p_ij transposed
    float *dSt = Pt + SIMT_BK * (SIMT_BQ + 1);
    float *rowA = dSt + SIMT_BK * (SIMT_BQ + 1);
    float *rowD = rowA + SIMT_BQ;

    const int kb = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int G = a.H / a.Hkv;
    const long long j0 = (long long)kb * SIMT_BK;
    const size_t rsq = (size_t)a.H * d, rsk = (size_t)a.Hkv * d;
    const T *k = (const T *)a.k + ((size_t)b * a.N * a.Hkv + kvh) * d;
    const T *v = (const T *)a.v + ((size_t)b * a.N * a.Hkv + kvh) * d;

    simt_load_rows<T>(Ks, ld, k, j0, SIMT_BK, a.N, rsk, d, a.use_rope, a.log2_base);
    simt_load_plain<T>(Vs, ld, v, j0, SIMT_BK, a.N, rsk, d);
    const int r_o = threadIdx.x / 8, c_o = threadIdx.x % 8;   // r_o = key row
    float accK[SIMT_DMAX / 8], accV[SIMT_DMAX / 8];
#pragma unroll
    for (int u = 0; u < SIMT_DMAX / 8; ++u) { accK[u] = 0.f; accV[u] = 0.f; }

    const long long j_last = min((long long)a.N - 1, j0 + SIMT_BK - 1);
    // queries that can see any of these keys
    long long q_end = (j0 < a.n_sink) ? (long long)a.N : min((long long)a.N, j_last + a.window);
    const long long n_qt = (q_end - j0 + SIMT_BQ - 1) / SIMT_BQ;

    for (int g = 0; g < G; ++g) {
        const int h = kvh * G + g;
        const float slope = a.slopes ? a.slopes[h] : 0.f;
        const T *q = (const T *)a.q + ((size_t)b * a.N * a.H + h) * d;
        const T *dO = (const T *)a.dout + ((size_t)b * a.N * a.H + h) * d;
        for (long long qt = 0; qt < n_qt; ++qt) {
            const long long i0 = j0 + qt * SIMT_BQ;
            __syncthreads();
            simt_load_rows<T>(Qs, ld, q, i0, SIMT_BQ, a.N, rsq, d, a.use_rope, a.log2_base);
            simt_load_plain<T>(dOs, ld, dO, i0, SIMT_BQ, a.N, rsq, d);
            if (threadIdx.x < SIMT_BQ) {
                long long i = i0 + threadIdx.x;
                bool ok = i < a.N && a.mode == SWAT_MODE_SOFTMAX_;
                rowA[threadIdx.x] = ok ? a.lse[((size_t)b * a.H + h) * a.N + i] : 0.f;
                rowD[threadIdx.x] = ok ? a.Dws[((size_t)b * a.H + h) * a.N + i] : 0.f;
            }
            __syncthreads();
            for (int e = threadIdx.x; e < SIMT_BK * SIMT_BQ; e += blockDim.x) {
                int c = e / SIMT_BQ, r = e % SIMT_BQ;   // c = key, r = query
                long long i = i0 + r, j = j0 + c;
                float p = 0.f, ds = 0.f;
                if (i < a.N && j < a.N && in_keyset(i, j, a.window, a.n_sink)) {
                    float dot = 0.f, dp = 0.f;
                    for (int x = 0; x < d; ++x) {
                        dot = fmaf(Qs[r * ld + x], Ks[c * ld + x], dot);
                        dp = fmaf(dOs[r * ld + x], Vs[c * ld + x], dp);
                    }
                    float s = dot * a.scale + slope * (float)(i - j);
                    p = simt_weight(s, rowA[r], a.mode);
                    ds = simt_dscore(p, dp, rowD[r], a.mode);
                }
                Pt[c * (SIMT_BQ + 1) + r] = p;
                dSt[c * (SIMT_BQ + 1) + r] = ds;
            }
            __syncthreads();
            for (int r = 0; r < SIMT_BQ; ++r) {
                float p = Pt[r_o * (SIMT_BQ + 1) + r], ds = dSt[r_o * (SIMT_BQ + 1) + r];
#pragma unroll
                for (int u = 0; u < SIMT_DMAX / 8; ++u) {
                    int col = c_o + 8 * u;
                    if (col < d) {
                        accV[u] = fmaf(p, dOs[r * ld + col], accV[u]);
                        accK[u] = fmaf(ds, Qs[r * ld + col], accK[u]);
                    }
                }
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < SIMT_DMAX / 8; ++u) {
        int col = c_o + 8 * u;
        if (col < d) Ks[r_o * ld + col] = accK[u] * a.scale;
    }
    __syncthreads();
    T *dk = (T *)a.dk + ((size_t)b * a.N * a.Hkv + kvh) * d;
    T *dv = (T *)a.dv + ((size_t)b * a.N * a.Hkv + kvh) * d;
    const int half = d / 2;
    for (int e = threadIdx.x; e < SIMT_BK * half; e += blockDim.x) {
        int r = e / half, t = e % half;
        long long j = j0 + r;
        if (j >= a.N) continue;
        float x0 = Ks[r * ld + 2 * t], x1 = Ks[r * ld + 2 * t + 1], y0 = x0, y1 = x1;
        if (a.use_rope) {
            float c, s;
            rope_cos_sin(j, rope_theta(t, d, a.log2_base), c, s);
            rope_pair_inv(x0, x1, c, s, y0, y1);
        }
        dk[(size_t)j * rsk + 2 * t] = from_f<T>(y0);
        dk[(size_t)j * rsk + 2 * t + 1] = from_f<T>(y1);
    }
    if (j0 + r_o < a.N) {
#pragma unroll
        for (int u = 0; u < SIMT_DMAX / 8; ++u) {
            int col = c_o + 8 * u;
            if (col < d) dv[(size_t)(j0 + r_o) * rsk + col] = from_f<T>(accV[u]);
        }
    }
}

inline size_t simt_bwd_dq_smem_bytes()
{
    return sizeof(float) * (size_t)(4 * SIMT_BQ * (SIMT_DMAX + 1) + SIMT_BQ * (SIMT_BK + 1) + 2 * SIMT_BQ);
}
inline size_t simt_bwd_dkdv_smem_bytes()
{
    return sizeof(float) * (size_t)(4 * SIMT_BQ * (SIMT_DMAX + 1) + 2 * SIMT_BK * (SIMT_BQ + 1) + 2 * SIMT_BQ);
}

}  // namespace swat
