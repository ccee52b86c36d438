// fwd_simt.cuh — CUDA-core forward (exact fp32 arithmetic; any even d <= 128).
//
// This is the fp32 path of the ABI (dtype SWAT_F32), whose outputs must match
// the oracle to 1e-5. One CTA takes 32 query rows of one (b, h) and walks the
// 32-key tiles that hold any key of those rows: the sink tiles below the
// window, then the band [i0 - window + 1, i0 + 31]. All other tiles are
// skipped ("Sliding Window Attention" glossary, flash-attention entry: blocks
// outside the window are skipped entirely).
#pragma once
#include "common.cuh"

namespace swat {

constexpr int SIMT_BQ = 32;
constexpr int SIMT_BK = 32;
constexpr int SIMT_DMAX = 128;
constexpr int SIMT_THREADS = 256;

struct FwdArgs {
    const void *q, *k, *v;
    void *o;
    float *lse;
    const float *slopes;
    int B, H, Hkv, N, d, window, n_sink, mode;
    double log2_base;   // log2(rope_base); rope off when use_rope == 0
    int use_rope;
    float scale;        // 1/sqrt(d)
};

// Loads `rows` rows of a BSHD tensor (row stride `rs` elements) starting at
// position p0, rotates them by their absolute position, and stores fp32 into
// smem [rows][ld]. Rows at positions >= N are zero.
template <typename T>
__device__ void simt_load_rows(float *dst, int ld, const T *src, long long p0, int rows, int N,
                               size_t rs, int d, int rotate, double log2_base)
{
    const int half = d / 2;
    for (int e = threadIdx.x; e < rows * half; e += blockDim.x) {
        int r = e / half, t = e % half;
        long long p = p0 + r;
        float y0 = 0.f, y1 = 0.f;
        if (p < N && p >= 0) {
            const T *row = src + (size_t)p * rs;
            float x0 = to_f(row[2 * t]), x1 = to_f(row[2 * t + 1]);
            if (rotate) {
                float c, s;
                rope_cos_sin(p, rope_theta(t, d, log2_base), c, s);
                rope_pair(x0, x1, c, s, y0, y1);
            } else {
                y0 = x0; y1 = x1;
            }
        }
        dst[r * ld + 2 * t] = y0;
        dst[r * ld + 2 * t + 1] = y1;
    }
}

template <typename T>
__global__ void __launch_bounds__(SIMT_THREADS)
swat_fwd_simt_kernel(FwdArgs a)
{
    extern __shared__ float smem[];
    const int d = a.d;
    const int ldq = SIMT_DMAX + 1;
    float *Qs = smem;                          // [BQ][ldq]
    float *Ks = Qs + SIMT_BQ * ldq;            // [BK][ldq]
    float *Vs = Ks + SIMT_BK * ldq;            // [BK][ldq]
    float *Ps = Vs + SIMT_BK * ldq;            // [BQ][BK+1]
    float *row_m = Ps + SIMT_BQ * (SIMT_BK + 1);
    float *row_l = row_m + SIMT_BQ;
    float *row_scale = row_l + SIMT_BQ;

    const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int G = a.H / a.Hkv, kvh = h / G;
    const long long i0 = (long long)qb * SIMT_BQ;
    const T *q = (const T *)a.q + ((size_t)b * a.N * a.H + h) * d;
    const T *k = (const T *)a.k + ((size_t)b * a.N * a.Hkv + kvh) * d;
    const T *v = (const T *)a.v + ((size_t)b * a.N * a.Hkv + kvh) * d;
    const float slope = a.slopes ? a.slopes[h] : 0.f;

    simt_load_rows<T>(Qs, ldq, q, i0, SIMT_BQ, a.N, (size_t)a.H * d, d, a.use_rope, a.log2_base);
    if (threadIdx.x < SIMT_BQ) {
        row_m[threadIdx.x] = -INFINITY;
        row_l[threadIdx.x] = 0.f;
    }
    // each thread owns row r_o and columns c_o + 8u of the output tile
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
        simt_load_rows<T>(Ks, ldq, k, j0, SIMT_BK, a.N, (size_t)a.Hkv * d, d, a.use_rope, a.log2_base);
        simt_load_rows<T>(Vs, ldq, v, j0, SIMT_BK, a.N, (size_t)a.Hkv * d, d, 0, 0.0);
        __syncthreads();
        // scores: 32x32, 4 per thread
        for (int e = threadIdx.x; e < SIMT_BQ * SIMT_BK; e += blockDim.x) {
            int r = e / SIMT_BK, c = e % SIMT_BK;
            long long i = i0 + r, j = j0 + c;
            float s = -INFINITY;
            if (i < a.N && in_keyset(i, j, a.window, a.n_sink)) {
                float dot = 0.f;
                for (int x = 0; x < d; ++x) dot = fmaf(Qs[r * ldq + x], Ks[c * ldq + x], dot);
                s = dot * a.scale + slope * (float)(i - j);
            }
            if (a.mode == SWAT_MODE_SIGMOID_) s = (s == -INFINITY) ? 0.f : sigmoid_exact(s);
            Ps[r * (SIMT_BK + 1) + c] = s;
        }
        __syncthreads();
        if (a.mode == SWAT_MODE_SOFTMAX_) {
            if (threadIdx.x < SIMT_BQ) {
                int r = threadIdx.x;
                float m_old = row_m[r], mx = m_old;
                for (int c = 0; c < SIMT_BK; ++c) mx = fmaxf(mx, Ps[r * (SIMT_BK + 1) + c]);
                float sc = (mx == -INFINITY) ? 1.f : expf(m_old - mx);   // m_old = -inf -> 0
                float sum = 0.f;
                for (int c = 0; c < SIMT_BK; ++c) {
                    float s = Ps[r * (SIMT_BK + 1) + c];
                    float p = (s == -INFINITY) ? 0.f : expf(s - mx);
                    Ps[r * (SIMT_BK + 1) + c] = p;
                    sum += p;
                }
                row_m[r] = mx;
                row_l[r] = row_l[r] * sc + sum;
                row_scale[r] = sc;
            }
            __syncthreads();
            float sc = row_scale[r_o];
#pragma unroll
            for (int u = 0; u < SIMT_DMAX / 8; ++u) acc[u] *= sc;
        }
        // O += P V
        for (int c = 0; c < SIMT_BK; ++c) {
            float p = Ps[r_o * (SIMT_BK + 1) + c];
#pragma unroll
            for (int u = 0; u < SIMT_DMAX / 8; ++u) {
                int col = c_o + 8 * u;
                if (col < d) acc[u] = fmaf(p, Vs[c * ldq + col], acc[u]);
            }
        }
        __syncthreads();
    }
    const long long i = i0 + r_o;
    if (i < a.N) {
        float inv = 1.f;
        if (a.mode == SWAT_MODE_SOFTMAX_) {
            float l = row_l[r_o];
            inv = 1.f / l;
            if (c_o == 0) a.lse[((size_t)b * a.H + h) * a.N + i] = row_m[r_o] + logf(l);
        }
        T *o = (T *)a.o + (((size_t)b * a.N + i) * a.H + h) * d;
#pragma unroll
        for (int u = 0; u < SIMT_DMAX / 8; ++u) {
            int col = c_o + 8 * u;
            if (col < d) o[col] = from_f<T>(acc[u] * inv);
        }
    }
}

inline size_t simt_fwd_smem_bytes()
{
    return sizeof(float) * (size_t)(3 * SIMT_BQ * (SIMT_DMAX + 1) + SIMT_BQ * (SIMT_BK + 1) + 3 * SIMT_BQ);
}

}  // namespace swat
