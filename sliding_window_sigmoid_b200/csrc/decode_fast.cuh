// decode_fast.cuh — bf16 ring-buffer decode attention, HBM streaming kernel.
//
// One step reads the whole ring of every (b, kv head): 2 * window * d * 2
// bytes, the bound of the decode ("Sliding Window Attention" glossary,
// ring-buffer paragraph: the cache holds the last w keys and values). Each
// CTA streams DEC_SLOTS_PER_SPLIT consecutive slots of one (b, kv head) for
// the G query heads that share it, with 16-byte loads: a group of d/8 lanes
// covers one cache row (each lane owns 8 dimensions), and the loads of four
// rows per row group are issued before their arithmetic. One thread of the
// CTA keeps the next DEC_PREFETCH_ITERS iterations of K and V rows (two
// contiguous ranges) on their way into L2 with bulk prefetches, so those
// loads mostly hit L2 and the warps need fewer bytes in flight to cover HBM
// latency. Split 0 also takes the sink rows. Partial sums (and, in softmax
// mode, the running maximum and denominator per head) go to the workspace;
// decode_combine merges them.
#pragma once
#include "common.cuh"
#include "decode.cuh"
#include "sm100.cuh"

namespace swat {

// Two CTAs per SM (registers capped at 128) keep 16 warps of loads in
// flight; a group of 8 heads needs the full register file of one CTA.
template <int D, int G, int MODE>
__global__ void __launch_bounds__(256, (G <= 4) ? 2 : 1)
swa_decode_attn_bf16_kernel(DecArgs a)
{
    constexpr int LPR = D / 8;        // lanes per cache row
    constexpr int RPW = 32 / LPR;     // rows per warp per iteration
    constexpr int NW = 8;             // warps
    constexpr int U = 4;              // iterations whose loads are in flight together
    constexpr int PAIRS = 4;          // RoPE pairs per lane (8 dims)
    __shared__ float red[NW][G][D];
    __shared__ float red_m[NW][G], red_l[NW][G];

    const int split = blockIdx.x, bk = blockIdx.y;
    const int b = bk / a.Hkv, kvh = bk % a.Hkv;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int grp = lane / LPR, li = lane % LPR;
    const long long P = a.pos[b];
    const int w = a.window;
    const int s0 = split * DEC_SLOTS_PER_SPLIT;
    const int s1 = min(w, s0 + DEC_SLOTS_PER_SPLIT);
    const __nv_bfloat16 *kc = reinterpret_cast<const __nv_bfloat16 *>(a.k_cache) + ((size_t)b * a.Hkv + kvh) * (size_t)w * D;
    const __nv_bfloat16 *vc = reinterpret_cast<const __nv_bfloat16 *>(a.v_cache) + ((size_t)b * a.Hkv + kvh) * (size_t)w * D;

    // The new token first: the CTA whose slot range holds slot P mod w rotates
    // k_new at P and stores it and v_new there (and in sink slot P when
    // P < n_sink), the same values the separate write kernel stores, then
    // syncs so that its own reads below see them. No other CTA reads that slot.
    if (P < 0) {
        if (split == 0 && threadIdx.x == 0) record_status(-1);   // positions are absolute, >= 0
    } else if ((int)(P % w) >= s0 && (int)(P % w) < s1) {
        const int slot = (int)(P % w);
        const __nv_bfloat16 *kt = reinterpret_cast<const __nv_bfloat16 *>(a.k_new) + ((size_t)b * a.Hkv + kvh) * D;
        const __nv_bfloat16 *vt = reinterpret_cast<const __nv_bfloat16 *>(a.v_new) + ((size_t)b * a.Hkv + kvh) * D;
        __nv_bfloat16 *kw = const_cast<__nv_bfloat16 *>(kc) + (size_t)slot * D;
        __nv_bfloat16 *vw = const_cast<__nv_bfloat16 *>(vc) + (size_t)slot * D;
        for (int t = threadIdx.x; t < D / 2; t += blockDim.x) {
            const float x0 = __bfloat162float(kt[2 * t]), x1 = __bfloat162float(kt[2 * t + 1]);
            float y0 = x0, y1 = x1;
            if (a.use_rope) {
                float c, sn;
                rope_cos_sin(P, rope_theta(t, D, a.log2_base), c, sn);
                rope_pair(x0, x1, c, sn, y0, y1);
            }
            const __nv_bfloat16 k0 = __float2bfloat16(y0), k1 = __float2bfloat16(y1);
            kw[2 * t] = k0; kw[2 * t + 1] = k1;
            vw[2 * t] = vt[2 * t]; vw[2 * t + 1] = vt[2 * t + 1];
            if (P < a.n_sink) {
                const size_t sb = (((size_t)b * a.Hkv + kvh) * a.n_sink + (size_t)P) * D + 2 * t;
                __nv_bfloat16 *ks = reinterpret_cast<__nv_bfloat16 *>(a.k_sink), *vs = reinterpret_cast<__nv_bfloat16 *>(a.v_sink);
                ks[sb] = k0; ks[sb + 1] = k1;
                vs[sb] = vt[2 * t]; vs[sb + 1] = vt[2 * t + 1];
            }
        }
        __syncthreads();
    }

    // ---- L2 prefetch: one thread keeps the CTA's next PFD iterations of K and
    // V rows (contiguous slot ranges) on their way into L2 with bulk
    // prefetches, so the warps' own loads mostly hit L2 and fewer bytes need
    // to be in flight per warp; the first PFD go out before the query rotation.
    constexpr int CROWS = U * NW * RPW;                // slots the CTA consumes per iteration
    constexpr int PFD = DEC_PREFETCH_ITERS;            // iterations prefetched ahead
    auto prefetch_rows = [&](int r0) {
        if (r0 < s1) {
            const uint32_t bytes = (uint32_t)(min(CROWS, s1 - r0) * D * 2);
            sm100::bulk_prefetch_l2(kc + (size_t)r0 * D, bytes);
            sm100::bulk_prefetch_l2(vc + (size_t)r0 * D, bytes);
        }
    };
    if (PFD > 0 && threadIdx.x == 0)
        for (int i = 0; i < PFD; ++i) prefetch_rows(s0 + i * CROWS);

    // ---- rotated queries of the group, this lane's 8 dimensions
    float q[G][8];
    {
        float cs[PAIRS], sn[PAIRS];
#pragma unroll
        for (int p = 0; p < PAIRS; ++p) {
            if (a.use_rope) {
                const int t = 4 * li + p;
                rope_cos_sin(P, rope_theta(t, D, a.log2_base), cs[p], sn[p]);
            } else {
                cs[p] = 1.f; sn[p] = 0.f;
            }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const uint4 raw = *reinterpret_cast<const uint4 *>(
                reinterpret_cast<const __nv_bfloat16 *>(a.q) + ((size_t)b * a.H + kvh * G + g) * D + 8 * li);
            const uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int p = 0; p < PAIRS; ++p) {
                const float x0 = sm100::bf16lo(wds[p]), x1 = sm100::bf16hi(wds[p]);
                q[g][2 * p] = (x0 * cs[p] - x1 * sn[p]) * a.scale;      // 1/sqrt(d) folded into q
                q[g][2 * p + 1] = (x0 * sn[p] + x1 * cs[p]) * a.scale;
            }
        }
    }
    float acc[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;

    const int pm = (int)(P % w);                      // slot of position P

    // Reduction of the G per-head partial dots over the LPR lanes of a row
    // group, exchanging halves: after log2(G) levels each lane holds the full
    // score of one head, hh = li / (LPR / G); the remaining levels are plain.
    constexpr int HSPAN = LPR / G;                    // lanes per head after the exchange
    const int hh = li / HSPAN;
    const float my_slope = a.slopes ? __ldg(a.slopes + kvh * G + hh) : 0.f;
    float mh = -INFINITY, lh = 0.f;                   // softmax state of head hh (this lane's copy)

    // Score of one cache row for head hh (this lane's head after the exchange).
    auto score = [&](const uint4 &kr, int delta) -> float {
        const uint32_t kw[4] = {kr.x, kr.y, kr.z, kr.w};
        sm100::f2 kf[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) kf[p] = {sm100::bf16lo(kw[p]), sm100::bf16hi(kw[p])};
        float s[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            sm100::f2 d = {0.f, 0.f};
#pragma unroll
            for (int p = 0; p < 4; ++p) d = sm100::fma2({q[g][2 * p], q[g][2 * p + 1]}, kf[p], d);
            s[g] = d.x + d.y;
        }
        // exchange levels
        int n = G;
#pragma unroll
        for (int off = LPR / 2; off >= HSPAN; off >>= 1) {
            const bool hi = (li & off) != 0;
            n >>= 1;
#pragma unroll
            for (int i = 0; i < G / 2; ++i) {
                if (i < n) {
                    const float keep = hi ? s[i + n] : s[i];
                    const float send = hi ? s[i] : s[i + n];
                    s[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
            }
        }
        float x = s[0];
#pragma unroll
        for (int off = HSPAN / 2; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        return x + my_slope * (float)delta;
    };
    // acc[g] += p_g v for one cache row, p_g taken from a lane of head g.
    auto accumulate = [&](const uint4 &vr, float pw) {
        const uint32_t vw[4] = {vr.x, vr.y, vr.z, vr.w};
        sm100::f2 vf[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) vf[p] = {sm100::bf16lo(vw[p]), sm100::bf16hi(vw[p])};
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float pg = __shfl_sync(0xffffffffu, pw, grp * LPR + g * HSPAN);
            const sm100::f2 p2 = {pg, pg};
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const sm100::f2 r = sm100::fma2(p2, vf[p], {acc[g][2 * p], acc[g][2 * p + 1]});
                acc[g][2 * p] = r.x;
                acc[g][2 * p + 1] = r.y;
            }
        }
    };
    // Rescales the accumulators of the heads whose running maximum moved.
    auto rescale = [&](float f) {
        if (__any_sync(0xffffffffu, f != 1.f)) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float fg = __shfl_sync(0xffffffffu, f, grp * LPR + g * HSPAN);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[g][e] *= fg;
            }
        }
    };
    // One row: score, weight, accumulate. In softmax mode the running maximum
    // is raised lazily (only when a score exceeds it by 8).
    auto consume = [&](const uint4 &kr, const uint4 &vr, int delta, bool valid) {
        const float x = score(kr, delta);
        float pw;
        if (MODE == SWAT_MODE_SIGMOID_) {
            pw = valid ? fmaf(0.5f, sm100::tanh_approx(0.5f * x), 0.5f) : 0.f;
        } else {
            float f = 1.f;
            if (valid && x > mh + 8.f) {
                f = (mh == -INFINITY) ? 0.f : __expf(mh - x);
                mh = x;
                lh *= f;
            }
            pw = valid ? __expf(x - mh) : 0.f;
            lh += pw;
            rescale(f);
        }
        accumulate(vr, pw);
    };

    // ---- ring slots of this split. Loop bounds are warp-uniform (the row
    // groups of a warp must take the same trip count: consume() shuffles
    // across the whole warp); a row past the split loads an in-bounds row and
    // is masked.
    constexpr int STRIDE = NW * RPW;
    for (int base = s0 + warp * RPW; base < s1; base += U * STRIDE) {
        if (PFD > 0 && threadIdx.x == 0) prefetch_rows(base + PFD * CROWS);
        uint4 kr[U], vr[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int slot = base + u * STRIDE + grp;
            const int sl = slot < s1 ? slot : s0;
            kr[u] = __ldg(reinterpret_cast<const uint4 *>(kc + (size_t)sl * D + 8 * li));
            vr[u] = __ldg(reinterpret_cast<const uint4 *>(vc + (size_t)sl * D + 8 * li));
        }
        if constexpr (MODE == SWAT_MODE_SIGMOID_) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int slot = base + u * STRIDE + grp;
                const int delta = (slot <= pm) ? pm - slot : pm - slot + w;   // distance of the position held
                const bool valid = slot < s1 && (long long)delta <= P;
                consume(kr[u], vr[u], delta, valid);
            }
        } else {
            // softmax: the U rows are scored first and the running maximum is
            // raised at most once for the group (by its largest valid score),
            // so the rows do not wait on one another through a branch
            float x[U], xm = -INFINITY;
            bool valid[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int slot = base + u * STRIDE + grp;
                const int delta = (slot <= pm) ? pm - slot : pm - slot + w;
                valid[u] = slot < s1 && (long long)delta <= P;
                x[u] = score(kr[u], delta);
                xm = valid[u] ? fmaxf(xm, x[u]) : xm;
            }
            float f = 1.f;
            if (xm > mh + 8.f) {
                f = (mh == -INFINITY) ? 0.f : __expf(mh - xm);
                mh = xm;
                lh *= f;
            }
            rescale(f);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const float pw = valid[u] ? __expf(x[u] - mh) : 0.f;
                lh += pw;
                accumulate(vr[u], pw);
            }
        }
    }
    // ---- sinks before the window (split 0)
    if (split == 0 && a.n_sink > 0) {
        const long long lim = min((long long)a.n_sink, P - w + 1);
        const __nv_bfloat16 *ks = reinterpret_cast<const __nv_bfloat16 *>(a.k_sink) + ((size_t)b * a.Hkv + kvh) * a.n_sink * D;
        const __nv_bfloat16 *vs = reinterpret_cast<const __nv_bfloat16 *>(a.v_sink) + ((size_t)b * a.Hkv + kvh) * a.n_sink * D;
        for (int jb = warp * RPW; jb < a.n_sink; jb += STRIDE) {
            const int j = jb + grp;
            const int jl = j < a.n_sink ? j : 0;
            const uint4 kr = __ldg(reinterpret_cast<const uint4 *>(ks + (size_t)jl * D + 8 * li));
            const uint4 vr = __ldg(reinterpret_cast<const uint4 *>(vs + (size_t)jl * D + 8 * li));
            consume(kr, vr, (int)(P - j), (long long)j < lim);
        }
    }

    // ---- reduce: the RPW row groups of a warp, then the warps. In softmax
    // mode the running maximum and denominator of head g live in the lanes
    // with hh == g; they are fetched from lane g * HSPAN of each group.
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float mg = 0.f, lg = 0.f;
        if (MODE == SWAT_MODE_SOFTMAX_) {
            mg = __shfl_sync(0xffffffffu, mh, grp * LPR + g * HSPAN);
            lg = __shfl_sync(0xffffffffu, lh, grp * LPR + g * HSPAN);
            float mm = mg;
#pragma unroll
            for (int off = 16; off >= LPR; off >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, off));
            const float f = (mg == -INFINITY) ? 0.f : __expf(mg - mm);
            lg *= f;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[g][e] *= f;
            mg = mm;
        }
#pragma unroll
        for (int off = 16; off >= LPR; off >>= 1) {
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], off);
            if (MODE == SWAT_MODE_SOFTMAX_) lg += __shfl_xor_sync(0xffffffffu, lg, off);
        }
        if (grp == 0) {
#pragma unroll
            for (int e = 0; e < 8; ++e) red[warp][g][8 * li + e] = acc[g][e];
            if (li == 0) { red_m[warp][g] = mg; red_l[warp][g] = lg; }
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
        const int g = e / D, c = e % D;
        float M = -INFINITY;
        if (MODE == SWAT_MODE_SOFTMAX_)
            for (int ww = 0; ww < NW; ++ww) M = fmaxf(M, red_m[ww][g]);
        float sum = 0.f, L = 0.f;
        for (int ww = 0; ww < NW; ++ww) {
            float f = 1.f;
            if (MODE == SWAT_MODE_SOFTMAX_) f = (red_m[ww][g] == -INFINITY) ? 0.f : __expf(red_m[ww][g] - M);
            sum = fmaf(red[ww][g][c], f, sum);
            L = fmaf(red_l[ww][g], f, L);
        }
        const size_t row = (size_t)b * a.H + kvh * G + g;
        a.part_o[(row * a.nsplit + split) * D + c] = sum;
        if (c == 0) {
            a.part_m[row * a.nsplit + split] = M;
            a.part_l[row * a.nsplit + split] = L;
        }
    }
}

template <int D, int MODE>
inline bool launch_decode_attn_dg(const DecArgs &a, cudaStream_t stream, int G)
{
    if (G > D / 8) return false;   // the head exchange needs G <= lanes per row
    dim3 grid(a.nsplit, a.B * a.Hkv);
    switch (G) {
        case 1: swa_decode_attn_bf16_kernel<D, 1, MODE><<<grid, 256, 0, stream>>>(a); return true;
        case 2: swa_decode_attn_bf16_kernel<D, 2, MODE><<<grid, 256, 0, stream>>>(a); return true;
        case 4: swa_decode_attn_bf16_kernel<D, 4, MODE><<<grid, 256, 0, stream>>>(a); return true;
        case 8: swa_decode_attn_bf16_kernel<D, 8, MODE><<<grid, 256, 0, stream>>>(a); return true;
        default: return false;
    }
}

// bf16 decode step up to the combine: the streaming kernel (which also stores
// the new token) for d in {64, 128} and a group of 1, 2, 4 or 8 query heads
// per KV head; the write kernel and the generic kernel otherwise. Returns the
// number of kernels launched.
inline int launch_decode_attn_fast(const DecArgs &a, cudaStream_t stream)
{
    const int G = a.H / a.Hkv;
    bool done = false;
    if (a.d == 128)
        done = a.mode == SWAT_MODE_SIGMOID_ ? launch_decode_attn_dg<128, SWAT_MODE_SIGMOID_>(a, stream, G)
                                            : launch_decode_attn_dg<128, SWAT_MODE_SOFTMAX_>(a, stream, G);
    else if (a.d == 64)
        done = a.mode == SWAT_MODE_SIGMOID_ ? launch_decode_attn_dg<64, SWAT_MODE_SIGMOID_>(a, stream, G)
                                            : launch_decode_attn_dg<64, SWAT_MODE_SOFTMAX_>(a, stream, G);
    if (!done) {   // the generic kernel expects the new token already in the ring
        swa_decode_write_kernel<__nv_bfloat16><<<a.B, 128, 0, stream>>>(a);
        dim3 grid(a.nsplit, a.B * a.Hkv);
        swa_decode_attn_generic_kernel<__nv_bfloat16><<<grid, DEC_THREADS, 0, stream>>>(a);
        return 2;
    }
    return 1;
}

}  // namespace swat
