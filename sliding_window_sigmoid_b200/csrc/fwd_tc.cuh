// fwd_tc.cuh — bf16 SWAT forward on 5th-generation tensor cores (sm_100a).
//
// Computes, for one (b, h) and a 128-row query tile, the SWAT attention of
// "SWAT: Sliding Window Attention Training" (section "Balanced ALiBi", the
// attention equation): o_m = sum over the key set of act(s_mn) v_n with
// s_mn = (R_m q_m).(R_n k_n)/sqrt(d) + slope_h (m - n); act = sigmoid
// (element-wise, section "Sigmoid") or, in softmax mode, the SWA(w, s)
// softmax over the window plus sink tokens ("Sliding-window beats linear
// attention"). Only 128-key tiles that hold a key of the tile's queries are
// visited (the band, plus the sink tile): the "Sliding Window Attention"
// glossary's flash-attention entry (blocks outside the window are skipped).
//
// CTA layout (320 threads, one CTA per SM: it owns all 512 TMEM columns):
//   warps 0-3  activation: tcgen05.ld S (one query row per thread, TMEM lane
//              = row), add the ALiBi term, mask edge tiles, apply the
//              activation, pack P to bf16 and tcgen05.st it over S; epilogue.
//   warps 4-7  RoPE prep: rotate the TMA-staged Q tile and each K tile in
//              place in shared memory (SWIZZLE_128B layout), then
//              fence.proxy.async so the tensor core sees the rotated values.
//   warp 8     MMA issue (one thread): S_b = Q K^T into TMEM buffer b = t%2,
//              then O += P_b V with P read from TMEM (A operand in TMEM).
//   warp 9     TMA producer (one thread): Q once, K/V tiles into a ring of
//              NST stages.
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D). P_b aliases the
// first 64 columns of S_b (bf16 pairs).
#pragma once
#include "common.cuh"
#include "sm100.cuh"
#include "fwd_simt.cuh"
#include "bwd_simt.cuh"

namespace swat {

using TcFwdArgs = FwdArgs;

template <int D>
struct FwdTcCfg {
    static constexpr int BM = 128, BN = 128;
    static constexpr int NST = (D == 64) ? 3 : 2;            // K/V pipeline stages
    static constexpr int TILE_BYTES = 128 * D * 2;            // one 128-row bf16 tile
    static constexpr int HALF_BYTES = 128 * 128;              // one 64-column SW128 box
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + TILE_BYTES;
    static constexpr int OFF_V = OFF_K + NST * TILE_BYTES;
    static constexpr int OFF_W = OFF_V + NST * TILE_BYTES;    // float2 [D/2][32]
    static constexpr int OFF_E = OFF_W + (D / 2) * 32 * 8;    // float2 [2][4][D/2]
    static constexpr int OFF_TH = OFF_E + 2 * 4 * (D / 2) * 8;   // double [D/2]
    static constexpr int OFF_BAR = OFF_TH + (D / 2) * 8;
    static constexpr int NBAR = 2 + 4 * NST + 4 + 3;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;         // + slack for 1024-B alignment
    static constexpr int THREADS = 320;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_O = 256;
};

constexpr int FWD_ACT_WARP0 = 0, FWD_PREP_WARP0 = 4, FWD_MMA_WARP = 8, FWD_TMA_WARP = 9;
constexpr int FWD_PREP_BAR = 1;   // named barrier of the 128 prep threads

// Key tiles of a query tile: optional sink tile (keys 0..127) when the band
// starts above it, then the band tiles from floor(max(0,i0-w+1)/128) to the
// tile holding min(N-1, i0+127).
struct TileRange {
    int n_tiles, has_sink, j0_first;
};

__device__ __forceinline__ TileRange fwd_tile_range(int i0, int N, int window, int n_sink)
{
    long long kstart = (long long)i0 - window + 1;
    if (kstart < 0) kstart = 0;
    int jf = (int)(kstart / 128) * 128;
    int jl = (min(N - 1, i0 + 127) / 128) * 128;
    int hs = (n_sink > 0 && jf > 0) ? 1 : 0;
    return {hs + (jl - jf) / 128 + 1, hs, jf};
}

__device__ __forceinline__ int fwd_tile_j0(const TileRange &r, int t)
{
    return (r.has_sink && t == 0) ? 0 : r.j0_first + (t - r.has_sink) * 128;
}

__device__ __forceinline__ bool named_bar_or(int id, int n, bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// Waits bounded by time only (used to drain in-flight async work before exit).
__device__ __forceinline__ bool mbar_wait_drain(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = sm100::globaltimer();
    while (!sm100::mbar_try_wait(bar, parity)) {
        if (sm100::globaltimer() - t0 > SWAT_WAIT_NS) {
            record_status(-4);
            return false;
        }
    }
    return true;
}

// (cos, sin) of pos * theta with the angle reduced modulo 2*pi in fp64.
__device__ __forceinline__ float2 rope_cs(double pos_theta)
{
    const double two_pi = 6.283185307179586476925286766559;
    const double inv_two_pi = 0.15915494309189533576888376337251;
    double r = pos_theta - rint(pos_theta * inv_two_pi) * two_pi;
    float s, c;
    sincosf((float)r, &s, &c);
    return make_float2(c, s);
}

// Rotate a 128-row tile in place (SW128 layout, D/64 boxes of [128 rows][128 B]).
// Thread (w, l) owns row r = 32 w + l. The angle of row r, pair t is
// (pos0 + 32 w + l) theta_t = base angle Eb[w][t] plus table angle W[t][l].
template <int D>
__device__ __forceinline__ void rope_rotate_tile(uint8_t *tile, const float2 *W, const float2 *Eb, int w,
                                                 int l)
{
    const int r = 32 * w + l;
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh) {
        uint8_t *rowp = tile + hh * 16384 + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint4 *p = reinterpret_cast<uint4 *>(rowp + ((c ^ (r & 7)) << 4));
            uint4 v = *p;
            uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const int t = hh * 32 + 4 * c + qq;
                const float2 e = Eb[w * (D / 2) + t];
                const float2 wt = W[t * 32 + l];
                const float cs = e.x * wt.x - e.y * wt.y;
                const float sn = e.y * wt.x + e.x * wt.y;
                const float x0 = sm100::bf16lo(w4[qq]), x1 = sm100::bf16hi(w4[qq]);
                w4[qq] = sm100::pack_bf16x2(x0 * cs - x1 * sn, x0 * sn + x1 * cs);
            }
            *p = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
    }
}

template <int D, int MODE>
__global__ void __launch_bounds__(320, 1)
swat_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdArgs a)
{
    using C = FwdTcCfg<D>;
    constexpr int NST = C::NST;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + C::OFF_Q;
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    float2 *sW = reinterpret_cast<float2 *>(smem + C::OFF_W);
    float2 *sE = reinterpret_cast<float2 *>(smem + C::OFF_E);
    double *sTh = reinterpret_cast<double *>(smem + C::OFF_TH);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *q_full = bars + 0, *q_ready = bars + 1;
    uint64_t *k_full = bars + 2, *k_ready = k_full + NST, *v_full = k_ready + NST, *kv_empty = v_full + NST;
    uint64_t *s_full = kv_empty + NST, *p_full = s_full + 2;
    uint64_t *o_full = p_full + 2, *o_upd = o_full + 1, *drain = o_upd + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int G = a.H / a.Hkv, kvh = h / G;
    const int i0 = qt * 128;
    const TileRange tr = fwd_tile_range(i0, a.N, a.window, a.n_sink);
    const int T = tr.n_tiles;

    if (threadIdx.x == 0) {
        sm100::mbar_init(q_full, 1);
        sm100::mbar_init(q_ready, 128);
        for (int s = 0; s < NST; ++s) {
            sm100::mbar_init(k_full + s, 1);
            sm100::mbar_init(k_ready + s, 128);
            sm100::mbar_init(v_full + s, 1);
            sm100::mbar_init(kv_empty + s, 1);
        }
        for (int s = 0; s < 2; ++s) {
            sm100::mbar_init(s_full + s, 1);
            sm100::mbar_init(p_full + s, 128);
        }
        sm100::mbar_init(o_full, 1);
        sm100::mbar_init(o_upd, 1);
        sm100::mbar_init(drain, 1);
        *abort_flag = 0;
        sm100::fence_mbar_init();
    }
    if (warp == FWD_MMA_WARP) {
        sm100::tmem_alloc(tmem_slot, C::TMEM_COLS);
        sm100::tmem_relinquish();
    }
    if (warp == FWD_TMA_WARP && lane == 0) {
        sm100::prefetch_tmap(&tm_q);
        sm100::prefetch_tmap(&tm_k);
        sm100::prefetch_tmap(&tm_v);
    }
    const int ptid = threadIdx.x - 32 * FWD_PREP_WARP0;   // 0..127 inside the prep group
    const bool is_prep = warp >= FWD_PREP_WARP0 && warp < FWD_PREP_WARP0 + 4;
    if (is_prep && a.use_rope) {
        if (ptid < D / 2) sTh[ptid] = exp2(-2.0 * (double)ptid / (double)D * a.log2_base);
        sm100::named_bar_sync(FWD_PREP_BAR, 128);
        for (int e = ptid; e < (D / 2) * 32; e += 128) {
            int t = e / 32, l = e % 32;
            sW[e] = rope_cs((double)l * sTh[t]);
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == FWD_TMA_WARP) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int last_n[NST];
            for (int s = 0; s < NST; ++s) last_n[s] = -1;
            sm100::mbar_arrive_expect_tx(q_full, C::TILE_BYTES);
            for (int hh = 0; hh < D / 64; ++hh)
                sm100::tma_load_4d(sQ + hh * C::HALF_BYTES, &tm_q, q_full, hh * 64, h, i0, b);
            for (int t = 0; t < T; ++t) {
                const int st = t % NST, n = t / NST;
                if (n > 0 && !sm100::mbar_wait(kv_empty + st, (n - 1) & 1, abort_flag)) break;
                const int j0 = fwd_tile_j0(tr, t);
                sm100::mbar_arrive_expect_tx(k_full + st, C::TILE_BYTES);
                for (int hh = 0; hh < D / 64; ++hh)
                    sm100::tma_load_4d(sK + st * C::TILE_BYTES + hh * C::HALF_BYTES, &tm_k, k_full + st,
                                       hh * 64, kvh, j0, b);
                sm100::mbar_arrive_expect_tx(v_full + st, C::TILE_BYTES);
                for (int hh = 0; hh < D / 64; ++hh)
                    sm100::tma_load_4d(sV + st * C::TILE_BYTES + hh * C::HALF_BYTES, &tm_v, v_full + st,
                                       hh * 64, kvh, j0, b);
                last_n[st] = n;
            }
            // every issued copy must have landed before the CTA may exit
            mbar_wait_drain(q_full, 0);
            for (int s = 0; s < NST; ++s)
                if (last_n[s] >= 0) {
                    mbar_wait_drain(k_full + s, last_n[s] & 1);
                    mbar_wait_drain(v_full + s, last_n[s] & 1);
                }
        }
    } else if (is_prep) {
        // ------------------------------------------------------------ RoPE prep
        const int w = ptid / 32, l = ptid % 32;
        auto make_bases = [&](int buf, int pos0) {
            if (!a.use_rope) return;
            for (int e = ptid; e < 4 * (D / 2); e += 128) {
                int ww = e / (D / 2), t = e % (D / 2);
                sE[buf * 4 * (D / 2) + e] = rope_cs((double)(pos0 + 32 * ww) * sTh[t]);
            }
        };
        make_bases(0, i0);
        bool ok = sm100::mbar_wait(q_full, 0, abort_flag);
        if (!named_bar_or(FWD_PREP_BAR, 128, !ok || *abort_flag)) {
            if (a.use_rope) rope_rotate_tile<D>(sQ, sW, sE, w, l);
            sm100::fence_proxy_async_smem();
            sm100::mbar_arrive(q_ready);
            for (int t = 0; t < T; ++t) {
                const int st = t % NST, n = t / NST, buf = (t + 1) & 1;
                make_bases(buf, fwd_tile_j0(tr, t));
                ok = sm100::mbar_wait(k_full + st, n & 1, abort_flag);
                if (named_bar_or(FWD_PREP_BAR, 128, !ok || *abort_flag)) break;
                if (a.use_rope) rope_rotate_tile<D>(sK + st * C::TILE_BYTES, sW, sE + buf * 4 * (D / 2), w, l);
                sm100::fence_proxy_async_smem();
                sm100::mbar_arrive(k_ready + st);
            }
        }
    } else if (warp == FWD_MMA_WARP) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            constexpr uint32_t IDESC_S = sm100::idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t IDESC_PV = sm100::idesc_bf16_f32(128, D, 0, 1);
            const uint32_t qa = sm100::smem_u32(sQ);
            auto issue_pv = [&](int u) -> bool {
                const int st = u % NST, bb = u & 1;
                if (!sm100::mbar_wait(p_full + bb, (u >> 1) & 1, abort_flag)) return false;
                if (!sm100::mbar_wait(v_full + st, (u / NST) & 1, abort_flag)) return false;
                sm100::tc_fence_after();
                const uint32_t va = sm100::smem_u32(sV + st * C::TILE_BYTES);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t bd = sm100::sdesc_sw128(va + ks * 2048, C::HALF_BYTES, 1024);
                    sm100::umma_ts(tmem + C::COL_O, tmem + bb * 128 + ks * 8, bd, IDESC_PV,
                                   (u > 0 || ks > 0) ? 1u : 0u);
                }
                sm100::umma_commit(kv_empty + st);
                if (MODE == SWAT_MODE_SOFTMAX_) sm100::umma_commit(o_upd);
                return true;
            };
            bool ok = sm100::mbar_wait(q_ready, 0, abort_flag);
            for (int t = 0; ok && t < T; ++t) {
                const int st = t % NST, n = t / NST, bb = t & 1;
                if (!sm100::mbar_wait(k_ready + st, n & 1, abort_flag)) { ok = false; break; }
                sm100::tc_fence_after();
                const uint32_t ka = sm100::smem_u32(sK + st * C::TILE_BYTES);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks / 4) * C::HALF_BYTES + (ks % 4) * 32;
                    const uint64_t ad = sm100::sdesc_sw128(qa + off, 16, 1024);
                    const uint64_t bd = sm100::sdesc_sw128(ka + off, 16, 1024);
                    sm100::umma_ss(tmem + bb * 128, ad, bd, IDESC_S, ks > 0 ? 1u : 0u);
                }
                sm100::umma_commit(s_full + bb);
                if (t >= 1 && !issue_pv(t - 1)) { ok = false; break; }
            }
            if (ok) ok = issue_pv(T - 1);
            if (ok) sm100::umma_commit(o_full);
            sm100::umma_commit(drain);
            mbar_wait_drain(drain, 0);   // nothing of ours is in flight past this point
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ activation
        const int r = 32 * warp + lane;                  // query row inside the tile (= TMEM lane)
        const int i = i0 + r;
        const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
        const float slope = a.slopes ? a.slopes[h] : 0.f;
        float m_used = -INFINITY, l_sum = 0.f;           // softmax state (log2 domain)
        bool ok = true;
        for (int t = 0; t < T; ++t) {
            const int bb = t & 1;
            ok = sm100::mbar_wait(s_full + bb, (t >> 1) & 1, abort_flag);
            if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
            sm100::tc_fence_after();
            const int j0 = fwd_tile_j0(tr, t);
            const bool need_mask = !(j0 + 127 <= i0 && (i0 + 127 - j0 < a.window || j0 + 127 < a.n_sink));
            const int rd = i - j0;                       // i - j at column 0
            const uint32_t s_addr = tmem + lane_base + bb * 128;
            if (MODE == SWAT_MODE_SIGMOID_) {
                // sigma(x) = 0.5 + 0.5 tanh(x / 2), x = acc/sqrt(d) + slope (i - j)
                const float hs = 0.5f * a.scale, hsl = 0.5f * slope, hb0 = hsl * (float)rd;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint32_t v[32];
                    sm100::tmem_ld32(s_addr + 32 * k, v);
                    sm100::tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int c0 = 32 * k + 2 * e, c1 = c0 + 1;
                        float x0 = fmaf(__uint_as_float(v[2 * e]), hs, fmaf(-hsl, (float)c0, hb0));
                        float x1 = fmaf(__uint_as_float(v[2 * e + 1]), hs, fmaf(-hsl, (float)c1, hb0));
                        float p0 = fmaf(0.5f, sm100::tanh_approx(x0), 0.5f);
                        float p1 = fmaf(0.5f, sm100::tanh_approx(x1), 0.5f);
                        if (need_mask) {
                            const int d0 = rd - c0, d1 = rd - c1;
                            if (!(d0 >= 0 && (d0 < a.window || j0 + c0 < a.n_sink))) p0 = 0.f;
                            if (!(d1 >= 0 && (d1 < a.window || j0 + c1 < a.n_sink))) p1 = 0.f;
                        }
                        pk[e] = sm100::pack_bf16x2(p0, p1);
                    }
                    sm100::tmem_st16(s_addr + 16 * k, pk);
                }
            } else {
                // softmax in the log2 domain: x2 = log2(e) * s
                const float LOG2E = 1.4426950408889634f;
                const float sc2 = a.scale * LOG2E, sl2 = slope * LOG2E, b2 = sl2 * (float)rd;
                float mx = -INFINITY;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint32_t v[32];
                    sm100::tmem_ld32(s_addr + 32 * k, v);
                    sm100::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int c = 32 * k + e;
                        float x = fmaf(__uint_as_float(v[e]), sc2, fmaf(-sl2, (float)c, b2));
                        if (need_mask) {
                            const int dd = rd - c;
                            if (!(dd >= 0 && (dd < a.window || j0 + c < a.n_sink))) x = -INFINITY;
                        }
                        mx = fmaxf(mx, x);
                    }
                }
                // keep a stale maximum while the new one exceeds it by at most 8
                // (weights stay <= 2^8); otherwise rescale this row of O and l
                const bool need = mx > m_used + 8.0f;
                const bool need_o = need && m_used != -INFINITY;
                if (__any_sync(0xffffffffu, need_o)) {
                    if (!sm100::mbar_wait(o_upd, (t - 1) & 1, abort_flag)) ok = false;
                    if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
                    sm100::tc_fence_after();
                    const float f = need_o ? sm100::ex2_approx(m_used - mx) : 1.f;
#pragma unroll
                    for (int k = 0; k < D / 32; ++k) {
                        uint32_t v[32];
                        sm100::tmem_ld32(tmem + lane_base + C::COL_O + 32 * k, v);
                        sm100::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * f);
                        sm100::tmem_st32(tmem + lane_base + C::COL_O + 32 * k, v);
                    }
                    if (need_o) l_sum *= f;
                }
                if (need) m_used = mx;
                float lsum = 0.f;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint32_t v[32];
                    sm100::tmem_ld32(s_addr + 32 * k, v);
                    sm100::tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int c0 = 32 * k + 2 * e, c1 = c0 + 1;
                        float x0 = fmaf(__uint_as_float(v[2 * e]), sc2, fmaf(-sl2, (float)c0, b2));
                        float x1 = fmaf(__uint_as_float(v[2 * e + 1]), sc2, fmaf(-sl2, (float)c1, b2));
                        float p0 = (m_used == -INFINITY) ? 0.f : sm100::ex2_approx(x0 - m_used);
                        float p1 = (m_used == -INFINITY) ? 0.f : sm100::ex2_approx(x1 - m_used);
                        if (need_mask) {
                            const int d0 = rd - c0, d1 = rd - c1;
                            if (!(d0 >= 0 && (d0 < a.window || j0 + c0 < a.n_sink))) p0 = 0.f;
                            if (!(d1 >= 0 && (d1 < a.window || j0 + c1 < a.n_sink))) p1 = 0.f;
                        }
                        lsum += p0 + p1;
                        pk[e] = sm100::pack_bf16x2(p0, p1);
                    }
                    sm100::tmem_st16(s_addr + 16 * k, pk);
                }
                l_sum += lsum;
            }
            sm100::tmem_wait_st();
            sm100::tc_fence_before();
            sm100::mbar_arrive(p_full + bb);
        }
        // ---- epilogue: O (TMEM) -> registers -> global, one row per thread
        if (ok) ok = sm100::mbar_wait(o_full, 0, abort_flag);
        if (!__any_sync(0xffffffffu, !ok)) {
            sm100::tc_fence_after();
            float inv = 1.f;
            if (MODE == SWAT_MODE_SOFTMAX_) inv = 1.f / l_sum;
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(a.o) + (((size_t)b * a.N + i) * a.H + h) * D;
#pragma unroll
            for (int k = 0; k < D / 32; ++k) {
                uint32_t v[32];
                sm100::tmem_ld32(tmem + lane_base + C::COL_O + 32 * k, v);
                sm100::tmem_wait_ld();
                if (i < a.N) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = sm100::pack_bf16x2(__uint_as_float(v[2 * e]) * inv, __uint_as_float(v[2 * e + 1]) * inv);
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * k);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                }
            }
            if (MODE == SWAT_MODE_SOFTMAX_ && i < a.N)
                a.lse[((size_t)b * a.H + h) * a.N + i] = (m_used + log2f(l_sum)) * 0.6931471805599453f;
        }
    }

    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    if (warp == FWD_MMA_WARP) sm100::tmem_dealloc(tmem, C::TMEM_COLS);
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------
typedef CUresult (*PFN_tmapEncodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                         const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                         const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                         CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline PFN_tmapEncodeTiled tmap_encoder()
{
    static PFN_tmapEncodeTiled fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_tmapEncodeTiled>(p);
    }
    return fn;
}

// bf16 tensor [B, N, Hx, D] (BSHD) as a 4-D map (D, Hx, N, B); box = 64 x 1 x 128 x 1, SW128.
inline bool make_tmap_bshd(CUtensorMap *m, const void *ptr, int B, int N, int Hx, int D)
{
    PFN_tmapEncodeTiled enc = tmap_encoder();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)Hx, (cuuint64_t)N, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)Hx * D * 2, (cuuint64_t)N * Hx * D * 2};
    cuuint32_t box[4] = {64, 1, 128, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int MODE>
inline int launch_fwd_tc_t(const FwdArgs &a, cudaStream_t stream)
{
    using C = FwdTcCfg<D>;
    CUtensorMap tq, tk, tv;
    if (!make_tmap_bshd(&tq, a.q, a.B, a.N, a.H, D) || !make_tmap_bshd(&tk, a.k, a.B, a.N, a.Hkv, D) ||
        !make_tmap_bshd(&tv, a.v, a.B, a.N, a.Hkv, D))
        return -1;
    auto kern = swat_fwd_tc_kernel<D, MODE>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess) return -1;
    dim3 grid((a.N + 127) / 128, a.H, a.B);
    kern<<<grid, C::THREADS, C::SMEM, stream>>>(tq, tk, tv, a);
    return 1;
}

// Returns the number of kernels launched, or -1 on a launch-configuration error.
inline int launch_fwd_tc(const TcFwdArgs &a, cudaStream_t stream)
{
    if (a.d == 64)
        return a.mode == SWAT_MODE_SIGMOID_ ? launch_fwd_tc_t<64, SWAT_MODE_SIGMOID_>(a, stream)
                                            : launch_fwd_tc_t<64, SWAT_MODE_SOFTMAX_>(a, stream);
    if (a.d == 128)
        return a.mode == SWAT_MODE_SIGMOID_ ? launch_fwd_tc_t<128, SWAT_MODE_SIGMOID_>(a, stream)
                                            : launch_fwd_tc_t<128, SWAT_MODE_SOFTMAX_>(a, stream);
    return -1;
}

// ---------------------------------------------------------------------------
// bf16 backward (CUDA-core kernels for now)
// ---------------------------------------------------------------------------
inline size_t tc_bwd_extra_workspace(int B, int H, int Hkv, int N, int d)
{
    (void)B; (void)H; (void)Hkv; (void)N; (void)d;
    return 0;
}

inline int launch_bwd_tc(const BwdArgs &a, void *extra_ws, cudaStream_t stream)
{
    (void)extra_ws;
    size_t smem_q = simt_bwd_dq_smem_bytes(), smem_k = simt_bwd_dkdv_smem_bytes();
    cudaFuncSetAttribute(swat_bwd_dq_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_q);
    cudaFuncSetAttribute(swat_bwd_dkdv_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_k);
    dim3 gq((a.N + SIMT_BQ - 1) / SIMT_BQ, a.H, a.B);
    dim3 gk((a.N + SIMT_BK - 1) / SIMT_BK, a.Hkv, a.B);
    swat_bwd_dq_simt_kernel<__nv_bfloat16><<<gq, SIMT_THREADS, smem_q, stream>>>(a);
    swat_bwd_dkdv_simt_kernel<__nv_bfloat16><<<gk, SIMT_THREADS, smem_k, stream>>>(a);
    return 2;
}

}  // namespace swat
