// decode.cuh — ring-buffer KV cache: fill, write-new-token, attention, combine.
//
// "Sliding Window Attention" glossary, ring-buffer paragraph: w slots,
// position i lives in slot i mod w, overwriting the oldest entry; "Attention
// sink" entry: the first tokens stay beside the window. The cache holds keys
// already rotated at their absolute position, so a step rotates only the new
// key and the query.
//
// A step is three launches on one stream (so the write precedes every read):
//   1. decode_write:   rotate k_new at pos, store k/v into slot pos mod w
//                      (and into sink slot pos when pos < n_sink);
//   2. decode_attn:    each CTA streams one chunk of slots of one
//                      (b, kv head) for all G query heads of the group and
//                      writes a partial (sum, max, denominator) per head;
//   3. decode_combine: merges the partials of each (b, h).
// Step 2 is the HBM-bound hot loop: it reads the whole ring once per step.
#pragma once
#include "common.cuh"

namespace swat {

// Ring slots per CTA of the decode attention: long enough that the per-CTA
// set-up (query rotation, final reduction) is small next to the streaming;
// measured on B200 (batch 64, w 4096, sigmoid, no L2 prefetch): 512 -> 67 %,
// 1024 -> 74 %, 2048 -> 76 % of the copy bandwidth; with the L2 prefetch
// below, 1024 -> 85 % and 2048 -> 88 %.
#ifndef SWAT_DEC_SLOTS
#define SWAT_DEC_SLOTS 2048
#endif
constexpr int DEC_SLOTS_PER_SPLIT = SWAT_DEC_SLOTS;
// Iterations of K/V rows the streaming kernel keeps on their way into L2
// ahead of its own loads (bulk L2 prefetches of contiguous slot ranges).
// Measured on B200 (batch 64, w 4096, 2048 slots per CTA): 0 -> 76 % / 72 %,
// 1 to 3 -> 88 % / 79 %, 4 -> 85 % / 78 %, 8 -> 61 % / 58 % of the copy
// bandwidth (sigmoid / softmax with sinks).
#ifndef SWAT_DEC_PFD
#define SWAT_DEC_PFD 2
#endif
constexpr int DEC_PREFETCH_ITERS = SWAT_DEC_PFD;
constexpr int DEC_THREADS = 256;
constexpr int DEC_MAX_G = 8;

inline int decode_nsplit(int window) { return (window + DEC_SLOTS_PER_SPLIT - 1) / DEC_SLOTS_PER_SPLIT; }

struct DecArgs {
    const void *q, *k_new, *v_new;
    void *k_cache, *v_cache, *k_sink, *v_sink;
    const long long *pos;
    void *o;
    float *part_o, *part_m, *part_l;   // [B*H][nsplit][d], [B*H][nsplit] x2
    const float *slopes;
    int B, H, Hkv, d, window, n_sink, mode, nsplit;
    double log2_base;
    int use_rope;
    float scale;
};

struct FillArgs {
    const void *k, *v;
    void *k_cache, *v_cache, *k_sink, *v_sink;
    int B, Hkv, n_tok, d, window, n_sink;
    long long p0;
    double log2_base;
    int use_rope;
};

// Writes one raw token (k rotated at position p) into ring slot p mod w and,
// if p < n_sink, into sink slot p. Threads stride over (kv head, pair). The
// rotation's (cos, sin) of pair t come from cs[t] when given (one table per
// token, shared by its kv heads), else are computed here.
template <typename T>
__device__ void ring_store_token(const T *k_tok, const T *v_tok, T *kc, T *vc, T *ks, T *vs,
                                 int b, int Hkv, int d, int window, int n_sink, long long p,
                                 bool write_ring, int use_rope, double log2_base, const float2 *cs = nullptr)
{
    const int half = d / 2;
    const long long slot = p % window;
    for (int e = threadIdx.x; e < Hkv * half; e += blockDim.x) {
        int kvh = e / half, t = e % half;
        float x0 = to_f(k_tok[(size_t)kvh * d + 2 * t]), x1 = to_f(k_tok[(size_t)kvh * d + 2 * t + 1]);
        float y0 = x0, y1 = x1;
        if (use_rope) {
            float c, s;
            if (cs) {
                c = cs[t].x;
                s = cs[t].y;
            } else {
                rope_cos_sin(p, rope_theta(t, d, log2_base), c, s);
            }
            rope_pair(x0, x1, c, s, y0, y1);
        }
        T v0 = v_tok[(size_t)kvh * d + 2 * t], v1 = v_tok[(size_t)kvh * d + 2 * t + 1];
        if (write_ring) {
            size_t base = (((size_t)b * Hkv + kvh) * window + (size_t)slot) * d + 2 * t;
            kc[base] = from_f<T>(y0); kc[base + 1] = from_f<T>(y1);
            vc[base] = v0; vc[base + 1] = v1;
        }
        if (p < n_sink) {
            size_t sb = (((size_t)b * Hkv + kvh) * n_sink + (size_t)p) * d + 2 * t;
            ks[sb] = from_f<T>(y0); ks[sb + 1] = from_f<T>(y1);
            vs[sb] = v0; vs[sb + 1] = v1;
        }
    }
}

// grid (n_tok, B): token t of sequence b sits at position p0 + t. Only the
// latest position of each slot is written, so the result does not depend on
// the order in which CTAs run.
template <typename T>
__global__ void swa_cache_fill_kernel(FillArgs a)
{
    __shared__ float2 cs[64];          // (cos, sin) of p theta_t, d <= 128
    const int t = blockIdx.x, b = blockIdx.y;
    const long long p = a.p0 + t;
    const long long p_end = a.p0 + a.n_tok;
    const bool latest = p + a.window >= p_end;
    if (!latest && p >= a.n_sink) return;   // overwritten later in the ring, not a sink
    if (a.use_rope) {
        for (int i = threadIdx.x; i < a.d / 2; i += blockDim.x) {
            float c, s;
            rope_cos_sin(p, rope_theta(i, a.d, a.log2_base), c, s);
            cs[i] = make_float2(c, s);
        }
        __syncthreads();
    }
    const T *kt = (const T *)a.k + ((size_t)b * a.n_tok + t) * a.Hkv * a.d;
    const T *vt = (const T *)a.v + ((size_t)b * a.n_tok + t) * a.Hkv * a.d;
    ring_store_token<T>(kt, vt, (T *)a.k_cache, (T *)a.v_cache, (T *)a.k_sink, (T *)a.v_sink, b,
                        a.Hkv, a.d, a.window, a.n_sink, p, latest, a.use_rope, a.log2_base, cs);
}

// grid (B): the new token of sequence b.
template <typename T>
__global__ void swa_decode_write_kernel(DecArgs a)
{
    const int b = blockIdx.x;
    const long long p = a.pos[b];
    if (p < 0) {                       // positions are absolute and >= 0
        if (threadIdx.x == 0) record_status(-1);
        return;
    }
    const T *kt = (const T *)a.k_new + (size_t)b * a.Hkv * a.d;
    const T *vt = (const T *)a.v_new + (size_t)b * a.Hkv * a.d;
    ring_store_token<T>(kt, vt, (T *)a.k_cache, (T *)a.v_cache, (T *)a.k_sink, (T *)a.v_sink, b,
                        a.Hkv, a.d, a.window, a.n_sink, p, true, a.use_rope, a.log2_base);
}

// Per-(head) running state of one lane group.
struct DecHeadState { float m, l; };

// grid (nsplit, B*Hkv), DEC_THREADS threads. Generic element type and d
// (lanes stride over the d elements of a row; one row per warp at a time).
template <typename T>
__global__ void __launch_bounds__(DEC_THREADS)
swa_decode_attn_generic_kernel(DecArgs a)
{
    __shared__ float qs[DEC_MAX_G][128];
    __shared__ float red_acc[DEC_THREADS / 32][DEC_MAX_G][128];
    __shared__ float red_m[DEC_THREADS / 32][DEC_MAX_G], red_l[DEC_THREADS / 32][DEC_MAX_G];
    const int split = blockIdx.x, bk = blockIdx.y;
    const int b = bk / a.Hkv, kvh = bk % a.Hkv;
    const int G = a.H / a.Hkv, d = a.d;
    const long long P = a.pos[b];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nwarps = blockDim.x / 32;
    // rotated queries of the group
    for (int e = threadIdx.x; e < G * (d / 2); e += blockDim.x) {
        int g = e / (d / 2), t = e % (d / 2);
        const T *qrow = (const T *)a.q + ((size_t)b * a.H + kvh * G + g) * d;
        float x0 = to_f(qrow[2 * t]), x1 = to_f(qrow[2 * t + 1]), y0 = x0, y1 = x1;
        if (a.use_rope) {
            float c, s;
            rope_cos_sin(P, rope_theta(t, d, a.log2_base), c, s);
            rope_pair(x0, x1, c, s, y0, y1);
        }
        qs[g][2 * t] = y0; qs[g][2 * t + 1] = y1;
    }
    __syncthreads();
    float acc[DEC_MAX_G][4];
    DecHeadState st[DEC_MAX_G];
    float slope[DEC_MAX_G];
    for (int g = 0; g < G; ++g) {
        st[g].m = -INFINITY; st[g].l = 0.f;
        slope[g] = a.slopes ? a.slopes[kvh * G + g] : 0.f;
        for (int u = 0; u < 4; ++u) acc[g][u] = 0.f;
    }
    const T *kc = (const T *)a.k_cache + ((size_t)b * a.Hkv + kvh) * a.window * d;
    const T *vc = (const T *)a.v_cache + ((size_t)b * a.Hkv + kvh) * a.window * d;
    const int s0 = split * DEC_SLOTS_PER_SPLIT;
    const int s1 = min(a.window, s0 + DEC_SLOTS_PER_SPLIT);
    // rows: ring slots of this split, then (split 0) the sinks before the window
    const long long sink_lim = (split == 0) ? min((long long)a.n_sink, P - a.window + 1) : 0;
    const int n_ring = s1 - s0;
    const int n_rows = n_ring + (int)max(0LL, sink_lim);
    for (int r = warp; r < n_rows; r += nwarps) {
        const T *krow, *vrow;
        long long delta;
        if (r < n_ring) {
            int slot = s0 + r;
            delta = ((P - slot) % a.window + a.window) % a.window;
            if (P - delta < 0) continue;
            krow = kc + (size_t)slot * d; vrow = vc + (size_t)slot * d;
        } else {
            int j = r - n_ring;
            delta = P - j;
            krow = (const T *)a.k_sink + (((size_t)b * a.Hkv + kvh) * a.n_sink + j) * d;
            vrow = (const T *)a.v_sink + (((size_t)b * a.Hkv + kvh) * a.n_sink + j) * d;
        }
        float kv_[4], vv_[4];
        for (int u = 0; u < 4; ++u) {
            int c = lane + 32 * u;
            kv_[u] = c < d ? to_f(krow[c]) : 0.f;
            vv_[u] = c < d ? to_f(vrow[c]) : 0.f;
        }
        for (int g = 0; g < G; ++g) {
            float dot = 0.f;
            for (int u = 0; u < 4; ++u) {
                int c = lane + 32 * u;
                if (c < d) dot = fmaf(qs[g][c], kv_[u], dot);
            }
            for (int off = 16; off; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
            float s = dot * a.scale + slope[g] * (float)delta;
            float p;
            if (a.mode == SWAT_MODE_SIGMOID_) {
                p = sigmoid_exact(s);
            } else {
                if (s > st[g].m) {
                    float sc = expf(st[g].m - s);
                    st[g].l *= sc;
                    for (int u = 0; u < 4; ++u) acc[g][u] *= sc;
                    st[g].m = s;
                }
                p = expf(s - st[g].m);
                st[g].l += p;
            }
            for (int u = 0; u < 4; ++u) acc[g][u] = fmaf(p, vv_[u], acc[g][u]);
        }
    }
    for (int g = 0; g < G; ++g) {
        for (int u = 0; u < 4; ++u) {
            int c = lane + 32 * u;
            if (c < d) red_acc[warp][g][c] = acc[g][u];
        }
        if (lane == 0) { red_m[warp][g] = st[g].m; red_l[warp][g] = st[g].l; }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < G * d; e += blockDim.x) {
        int g = e / d, c = e % d;
        float M = -INFINITY;
        if (a.mode == SWAT_MODE_SOFTMAX_)
            for (int w = 0; w < nwarps; ++w) M = fmaxf(M, red_m[w][g]);
        float sum = 0.f, L = 0.f;
        for (int w = 0; w < nwarps; ++w) {
            float f = 1.f;
            if (a.mode == SWAT_MODE_SOFTMAX_) f = (red_m[w][g] == -INFINITY) ? 0.f : expf(red_m[w][g] - M);
            sum = fmaf(red_acc[w][g][c], f, sum);
            L = fmaf(red_l[w][g], f, L);
        }
        size_t row = (size_t)b * a.H + kvh * G + g;
        a.part_o[(row * a.nsplit + split) * d + c] = sum;
        if (c == 0) {
            a.part_m[row * a.nsplit + split] = M;
            a.part_l[row * a.nsplit + split] = L;
        }
    }
}

// grid (B*H), d threads (<= 128 rounded up to a warp multiple).
template <typename T>
__global__ void swa_decode_combine_kernel(DecArgs a)
{
    const size_t row = blockIdx.x;
    const int c = threadIdx.x;
    if (c >= a.d) return;
    float M = -INFINITY;
    if (a.mode == SWAT_MODE_SOFTMAX_)
        for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, a.part_m[row * a.nsplit + s]);
    float sum = 0.f, L = 0.f;
    for (int s = 0; s < a.nsplit; ++s) {
        float f = 1.f;
        if (a.mode == SWAT_MODE_SOFTMAX_) {
            float m = a.part_m[row * a.nsplit + s];
            f = (m == -INFINITY) ? 0.f : expf(m - M);
            L = fmaf(a.part_l[row * a.nsplit + s], f, L);
        }
        sum = fmaf(a.part_o[(row * a.nsplit + s) * a.d + c], f, sum);
    }
    if (a.mode == SWAT_MODE_SOFTMAX_) sum /= L;
    ((T *)a.o)[row * a.d + c] = from_f<T>(sum);
}

}  // namespace swat
