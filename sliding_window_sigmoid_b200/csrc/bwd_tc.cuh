// bwd_tc.cuh — bf16 SWAT backward on 5th-generation tensor cores (sm_100a).
//
// Gradients of the attention equation of "SWAT: Sliding Window Attention
// Training" (section "Balanced ALiBi"), derived by calculus (the pages train
// SWAT from scratch but print no backward):
//   dv_j = sum_i p_ij dO_i,  dP_ij = dO_i . v_j,
//   sigmoid: dS_ij = dP_ij p_ij (1 - p_ij);  softmax: dS_ij = p_ij (dP_ij - D_i)
//   dq'_i = sum_j dS_ij k'_j / sqrt(d),  dk'_j = sum_i dS_ij q'_i / sqrt(d),
//   dq = R_i^T dq', dk = R_j^T dk'.
// One persistent kernel template, three roles (no atomics: every output row
// has one owner, results are deterministic):
//   DQ    item = (b, h, 128-query tile); stationary Q', dO; streamed K', V tiles:
//         S = Q'K'^T, dP = dO V^T, dS element-wise, dQ' += dS K'.
//   DKDV  item = (b, kv head, 128-key tile); stationary K', V; streamed Q', dO
//         tiles of every query head of the group: S^T = K'Q'^T, dP^T = V dO^T,
//         dV += P^T dO, dK' += dS^T Q'.
//   DSUM  (softmax) the DQ products without dQ': D_i = sum_j p_ij dP_ij.
// Each streamed tile is processed as two 64-column half-steps; half-step
// hs goes to TMEM buffer hs % NBUF and activation warpgroup hs % NWG
// (NWG = NBUF: 3 where three 128-column buffers fit beside the accumulators
// -- dq, and dk/dv at d 64 -- else 2), so the element-wise pass of one
// half-step overlaps the MMAs of the next ones.
// Warp roles (512 threads, one CTA per SM):
//   warp 0     issues S / dP of each half-step (X MMAs) into its TMEM buffer.
//   warp 1     TMA: stationary tile pair per item, streamed pairs into a ring.
//   warp 3     issues the gradient MMAs (dV, dK', dQ') of each half-step.
//   warps 4..  NWG activation warpgroups (one TMEM lane = one row per
//              thread); the epilogue of an item runs in one of them:
//              deferred until after its next half-step where two
//              accumulator sets fit, else right after the item's last
//              half-step, releasing the accumulators after its last TMEM load.
//   others     set-up only. Q and K arrive RoPE-rotated: a small kernel
//              writes rotated copies into the workspace first, or the
//              forward's copies are reused (swat_attn_bwd_rotated).
// TMEM columns: buffer b = [128 b, 128 b + 128): S half, then dP half (bf16
// P and dS over their first 32 columns, or in columns of their own);
// accumulators after the buffers.
#pragma once
#include "fwd_tc.cuh"
#include "rope_rows.cuh"

namespace swat {

enum { BWD_ROLE_DQ = 0, BWD_ROLE_DKDV = 1, BWD_ROLE_DSUM = 2 };

constexpr int BWD_X_WARP = 0, BWD_TMA_WARP = 1, BWD_G_WARP = 3, BWD_ACT_WARP0 = 4, BWD_PREP_WARP0 = 12;
constexpr int BWD_THREADS = 512;

template <int D, int ROLE>
struct BwdCfg {
    static constexpr int TILE = 128 * D * 2;                   // one 128-row bf16 tile
    static constexpr int HALF_BYTES = 128 * 128;               // one 64-column SW128 box
    static constexpr int NSTAT = (D == 64) ? 2 : 1;            // stationary tile pairs
    static constexpr int NST = (D == 64) ? 4 : 2;              // streamed tile pairs
    static constexpr int ACC_COLS = (ROLE == BWD_ROLE_DKDV) ? 2 * D : (ROLE == BWD_ROLE_DQ ? D : 0);
    // bf16 P / dS of each buffer: in columns of their own when they fit next
    // to two accumulator sets (the next S / dP MMA into the buffer then waits
    // only for the element-wise pass, not for the gradient MMAs), else over
    // the S / dP halves.
    // TMEM buffers of S / dP halves (128 columns each) in flight: three where
    // they fit next to one accumulator set (the dependency chain of a buffer
    // -- S / dP MMAs, element-wise pass, gradient MMAs -- then spans three
    // half-steps), else two.
    static constexpr int NBUF = (ROLE != BWD_ROLE_DSUM && 3 * 128 + ACC_COLS <= 512) ? 3 : 2;
    // activation warpgroups: one per buffer (half-step hs goes to warpgroup
    // hs % NWG and buffer hs % NBUF, so a warpgroup always meets the same
    // buffer and waits on its barriers in order)
    static constexpr int NWG = NBUF;
    static constexpr int PD_COLS = (ROLE == BWD_ROLE_DKDV) ? 64 : (ROLE == BWD_ROLE_DQ ? 32 : 0);
    static constexpr bool SEP_PD = NBUF == 2 && PD_COLS > 0 && 256 + 2 * PD_COLS + 2 * ACC_COLS <= 512;
    static constexpr int ACC_BASE = NBUF * 128 + (SEP_PD ? 2 * PD_COLS : 0);
    static constexpr int NACC = (ACC_COLS == 0) ? 1 : ((ACC_BASE + 2 * ACC_COLS <= 512) ? 2 : 1);
    static constexpr int OFF_A1 = 0;                           // stationary tiles [NSTAT]
    static constexpr int OFF_A2 = OFF_A1 + NSTAT * TILE;
    static constexpr int OFF_B1 = OFF_A2 + NSTAT * TILE;       // streamed tiles [NST]
    static constexpr int OFF_B2 = OFF_B1 + NST * TILE;
    static constexpr int OFF_ROT = OFF_B2 + NST * TILE;        // float2 [2][D/2] prep bases
    static constexpr int OFF_TH = OFF_ROT + 2 * (D / 2) * 8;   // double [D/2]
    static constexpr int OFF_THF = OFF_TH + (D / 2) * 8;       // float [D/2]
    static constexpr int OFF_A0 = OFF_THF + (D / 2) * 4;       // float [3 wg][4 warps][D/2] epilogue base angles
    static constexpr int OFF_ROWS = OFF_A0 + 12 * (D / 2) * 4; // float [3 wg][2 buf][128]: lse, D of 64 queries
    static constexpr int OFF_DSUM = OFF_ROWS + 3 * 2 * 128 * 4; // float [2 item][3 wg][128]
    static constexpr int OFF_BAR = OFF_DSUM + 2 * 3 * 128 * 4;
    static constexpr int NBAR = 3 * 2 + 4 * 4 + 3 * 3 + 4 * 2 + 2;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;          // + slack for 1024-B alignment
    static_assert(OFF_BAR % 8 == 0, "barrier alignment");
    static_assert(SMEM <= 232448, "shared memory per CTA");
    static_assert(NST <= 4 && NBUF <= 3, "barrier arrays");
    static_assert(ROLE != BWD_ROLE_DSUM || NWG == 2, "D_i partials: one half per warpgroup per step");
};

// Inverse RoPE of one accumulator row held in TMEM (fp32, D columns), for a
// row at absolute position pos0 + r; the angle is A0[t] + r theta_t (A0 is the
// position pos0 reduced in fp64), reduced again in fp32 before __sincosf.
// release: when non-null, arrived on (once per thread) as soon as the last
// TMEM load has landed, so the accumulator can be reused during the stores.
template <int D>
__device__ __forceinline__ void unrotate_store_row(uint32_t taddr, int r, const float *A0, const float *THF,
                                                   bool use_rope, __nv_bfloat16 *dst, bool store, float mul = 1.f,
                                                   uint64_t *release = nullptr)
{
    const float two_pi = 6.2831853071795865f, inv_two_pi = 0.15915494309189534f;
#pragma unroll
    for (int k = 0; k < D / 32; ++k) {
        uint32_t v[32];
        sm100::tmem_ld32(taddr + 32 * k, v);
        sm100::tmem_wait_ld_dep(v);
        if (release && k == D / 32 - 1) {
            sm100::tc_fence_before();
            sm100::mbar_arrive(release);
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            float x0 = __uint_as_float(v[2 * e]) * mul, x1 = __uint_as_float(v[2 * e + 1]) * mul;
            if (use_rope) {
                const int t = 16 * k + e;
                float ang = fmaf((float)r, THF[t], A0[t]);
                ang = fmaf(-rintf(ang * inv_two_pi), two_pi, ang);
                float sn, cs;
                __sincosf(ang, &sn, &cs);
                const float y0 = x0 * cs + x1 * sn, y1 = -x0 * sn + x1 * cs;
                x0 = y0; x1 = y1;
            }
            pk[e] = sm100::pack_bf16x2(x0, x1);
        }
        if (store) {
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + 32 * k);
#pragma unroll
            for (int e = 0; e < 4; ++e) d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
    }
}

template <int D>
__device__ __forceinline__ void store_row_bf16_plain(uint32_t taddr, __nv_bfloat16 *dst, bool store)
{
#pragma unroll
    for (int k = 0; k < D / 32; ++k) {
        uint32_t v[32];
        sm100::tmem_ld32(taddr + 32 * k, v);
        sm100::tmem_wait_ld_dep(v);
        if (store) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = sm100::pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + 32 * k);
#pragma unroll
            for (int e = 0; e < 4; ++e) d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
    }
}

// Last query tile whose key set meets key tile kt.
__device__ __forceinline__ int bwd_q_last(int kt, int nQT, int window, int n_sink)
{
    if (kt == 0 && n_sink > 0) return nQT - 1;            // sink keys are seen by every later query
    const long long last = ((long long)kt * 128 + 126 + (long long)window) / 128;
    return (int)min((long long)nQT - 1, last);
}

// Bits c0 .. c0+31 of the column interval [lo, hi] (bit e = column c0 + e).
__device__ __forceinline__ uint32_t interval_bits32(int lo, int hi, int c0)
{
    const int a = max(lo - c0, 0), z = min(hi - c0, 31);
    return (a <= z) ? ((0xFFFFFFFFu >> (31 - z)) & (0xFFFFFFFFu << a)) : 0u;
}

// One work item of a persistent backward CTA and its streamed tiles.
//   DQ / DSUM: u = ((b Hkv + kvh) nQT + qt) G + g; stationary rows are the
//              queries of (b, h = kvh G + g, qt); step t streams key tile t of
//              the query tile's key range (fwd_tile_range).
//   DKDV:      u = (b Hkv + kvh) nQT + kt; stationary rows are the keys of
//              (b, kvh, kt); step t streams query tile q_first + t % per_head
//              of query head kvh G + t / per_head.
struct BwdItem {
    int b, kvh, h, row0, T;
    int q_first, per_head;     // DKDV
    TileRange tr;              // DQ / DSUM
};

template <int ROLE>
__device__ __forceinline__ BwdItem bwd_item(const BwdArgs &a, int u)
{
    BwdItem it;
    const int G = a.H / a.Hkv, nQT = (a.N + 127) / 128;
    const unsigned v = (unsigned)u;
    if (ROLE == BWD_ROLE_DKDV) {
        const unsigned kt = v % (unsigned)nQT, sq = v / (unsigned)nQT;
        it.kvh = (int)(sq % (unsigned)a.Hkv);
        it.b = (int)(sq / (unsigned)a.Hkv);
        it.h = it.kvh * G;
        it.row0 = (int)kt * 128;
        it.q_first = (int)kt;
        it.per_head = bwd_q_last((int)kt, nQT, a.window, a.n_sink) - (int)kt + 1;
        it.T = G * it.per_head;
        it.tr = TileRange{0, 0, 0};
    } else {
        const unsigned g = v % (unsigned)G, r = v / (unsigned)G;
        const unsigned qt = r % (unsigned)nQT, sq = r / (unsigned)nQT;
        it.kvh = (int)(sq % (unsigned)a.Hkv);
        it.b = (int)(sq / (unsigned)a.Hkv);
        it.h = it.kvh * G + (int)g;
        it.row0 = (int)qt * 128;
        it.tr = fwd_tile_range(it.row0, a.N, a.window, a.n_sink);
        it.T = it.tr.n_tiles;
        it.q_first = 0; it.per_head = 1;
    }
    return it;
}

// Streamed tile of step t: its head index in the streamed tensor (K/V: kv
// head, Q/dO: query head) and its first row.
template <int ROLE>
__device__ __forceinline__ void bwd_stream(const BwdItem &it, int G, int t, int &head, int &pos0)
{
    if (ROLE == BWD_ROLE_DKDV) {
        head = it.kvh * G + t / it.per_head;
        pos0 = (it.q_first + t % it.per_head) * 128;
    } else {
        head = it.kvh;
        pos0 = fwd_tile_j0(it.tr, t);
    }
}

// Element-wise work of one 64-column half-step for one row (thread):
// reads the S and dP halves from TMEM (x_addr, x_addr + 64), writes bf16 P
// to p_addr (WRITE_P) and bf16 g to ds_addr (WRITE_DS), 32 columns each, and
// returns sum_c p dP (DSUM). The score of column c is
//   sigmoid: x = s hs + hb0 + hstep c   (hs = scale/2, bias halved), t = tanh x,
//            p = (1 + t)/2, g = dP p (1 - p);
//   softmax: x = s sc2 + b0 + bstep c - L_c  (log2 units), p = 2^x,
//            g = p (dP - D_c),
// with L_c, D_c per row (colL == nullptr: lrow, drow) or per column (colL,
// colD in shared memory); dS = g scale, the factor applied to the dQ' / dK'
// accumulators in the epilogue. Columns whose bit in m[] is clear get
// x = -inf, hence P = 0 and g = 0. Each 32-column block computes all its
// scores, then all its MUFU results, then the rest, so the MUFU work of one
// column overlaps the FMA work of others.
template <int MODE, bool WRITE_P, bool WRITE_DS, bool DSUM>
__device__ __forceinline__ float bwd_half_step(uint32_t x_addr, uint32_t p_addr, uint32_t ds_addr, float xs, float b0,
                                               float bstep, const uint32_t (&m)[2], float lrow, float drow,
                                               const float *colL, const float *colD)
{
    float dsum = 0.f;
#pragma unroll 1
    for (int cc = 0; cc < 2; ++cc) {
        uint32_t s0[16], s1[16], d0[16], d1[16];
        sm100::tmem_ld16(x_addr + 32 * cc, s0);
        sm100::tmem_ld16(x_addr + 32 * cc + 16, s1);
        sm100::tmem_ld16(x_addr + 64 + 32 * cc, d0);
        sm100::tmem_ld16(x_addr + 64 + 32 * cc + 16, d1);
        const int c0 = 32 * cc;
        const uint32_t mb = m[cc];
        const sm100::f2 xs2 = {xs, xs};
        const sm100::f2 step2 = {2.f * bstep, 2.f * bstep};
        sm100::f2 bias2 = {fmaf(bstep, (float)c0, b0), fmaf(bstep, (float)(c0 + 1), b0)};
        sm100::tmem_wait_ld_dep16(s0);
        sm100::tmem_wait_ld_dep16(s1);
        sm100::tmem_wait_ld_dep16(d0);
        sm100::tmem_wait_ld_dep16(d1);
        // scores (masked columns: -inf)
        float x[32];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const uint32_t *sv = e < 8 ? s0 : s1;
            const int k = e & 7;
            const sm100::f2 xx = sm100::fma2({__uint_as_float(sv[2 * k]), __uint_as_float(sv[2 * k + 1])}, xs2, bias2);
            bias2 = sm100::add2(bias2, step2);
            x[2 * e] = xx.x;
            x[2 * e + 1] = xx.y;
        }
        if (MODE != SWAT_MODE_SIGMOID_) {
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] -= colL ? colL[c0 + e] : lrow;
        }
        if (!__all_sync(0xffffffffu, mb == 0xFFFFFFFFu)) {
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = (mb & (1u << e)) ? x[e] : -INFINITY;
        }
        // MUFU: t = tanh x (sigmoid) or p = 2^x (softmax)
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = (MODE == SWAT_MODE_SIGMOID_) ? sm100::tanh_approx(x[e]) : sm100::ex2_approx(x[e]);
        uint32_t pk[16], gk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const uint32_t *dv = e < 8 ? d0 : d1;
            const int k = e & 7;
            const sm100::f2 dp = {__uint_as_float(dv[2 * k]), __uint_as_float(dv[2 * k + 1])};
            sm100::f2 p, g;
            if (MODE == SWAT_MODE_SIGMOID_) {
                const sm100::f2 t = {x[2 * e], x[2 * e + 1]};
                p = sm100::fma2(t, {0.5f, 0.5f}, {0.5f, 0.5f});
                const sm100::f2 q = sm100::fma2(t, {-0.5f, -0.5f}, {0.5f, 0.5f});
                g = sm100::mul2(dp, sm100::mul2(p, q));
            } else {
                p = {x[2 * e], x[2 * e + 1]};
                if (DSUM) {
                    dsum = fmaf(p.x, dp.x, dsum);
                    dsum = fmaf(p.y, dp.y, dsum);
                    g = {0.f, 0.f};
                } else {
                    const int c = c0 + 2 * e;
                    const sm100::f2 dd = {colD ? colD[c] : drow, colD ? colD[c + 1] : drow};
                    g = sm100::mul2(p, sm100::add2(dp, {-dd.x, -dd.y}));
                }
            }
            if (WRITE_P) pk[e] = sm100::pack_bf16x2(p.x, p.y);
            if (WRITE_DS) gk[e] = sm100::pack_bf16x2(g.x, g.y);
        }
        if (WRITE_P) sm100::tmem_st16(p_addr + 16 * cc, pk);
        if (WRITE_DS) sm100::tmem_st16(ds_addr + 16 * cc, gk);
    }
    return dsum;
}

// ===========================================================================
// The persistent backward kernel.
// tm_a1/tm_a2: stationary tensors (DQ, DSUM: Q, dO; DKDV: K, V);
// tm_b1/tm_b2: streamed tensors (DQ, DSUM: K, V; DKDV: Q, dO). Tiles a1 and
// b1 are RoPE-rotated in shared memory.
// ===========================================================================
template <int D, int MODE, int ROLE>
__global__ void __launch_bounds__(BWD_THREADS, 1)
swat_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_a2,
                   const __grid_constant__ CUtensorMap tm_b1, const __grid_constant__ CUtensorMap tm_b2,
                   const BwdArgs a)
{
    using C = BwdCfg<D, ROLE>;
    constexpr int NST = C::NST, NSTAT = C::NSTAT, NACC = C::NACC;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA1 = smem + C::OFF_A1, *sA2 = smem + C::OFF_A2, *sB1 = smem + C::OFF_B1, *sB2 = smem + C::OFF_B2;
    double *sTh = reinterpret_cast<double *>(smem + C::OFF_TH);
    float *sThf = reinterpret_cast<float *>(smem + C::OFF_THF);
    float *sA0 = reinterpret_cast<float *>(smem + C::OFF_A0);
    float *sRows = reinterpret_cast<float *>(smem + C::OFF_ROWS);
    float *sDsum = reinterpret_cast<float *>(smem + C::OFF_DSUM);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *stat_full = bars, *stat_ready = bars + 2, *stat_free = bars + 4;
    uint64_t *b1_full = bars + 6, *b2_full = b1_full + 4, *st_ready = b2_full + 4, *st_free = st_ready + 4;
    uint64_t *x_full = st_free + 4, *p_full = x_full + 3, *buf_free = p_full + 3, *acc_full = buf_free + 3;
    uint64_t *acc_free = acc_full + 2, *dsum_full = acc_free + 2, *dsum_free = dsum_full + 2;
    uint64_t *drain_x = dsum_free + 2, *drain_g = drain_x + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int G = a.H / a.Hkv, nQT = (a.N + 127) / 128;
    const long long U = (ROLE == BWD_ROLE_DKDV) ? (long long)a.B * a.Hkv * nQT : (long long)a.B * a.H * nQT;
    const int u_begin = (int)(U * blockIdx.x / gridDim.x), u_end = (int)(U * (blockIdx.x + 1) / gridDim.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            sm100::mbar_init(stat_full + s, 1);
            sm100::mbar_init(stat_ready + s, 128);
            sm100::mbar_init(stat_free + s, 1);
            sm100::mbar_init(acc_full + s, 1);
            sm100::mbar_init(acc_free + s, 128);
            sm100::mbar_init(dsum_full + s, 128 * C::NWG);
            sm100::mbar_init(dsum_free + s, 128);
        }
        for (int s = 0; s < 3; ++s) {
            sm100::mbar_init(x_full + s, 1);
            sm100::mbar_init(p_full + s, 128);
            sm100::mbar_init(buf_free + s, 1);
        }
        for (int s = 0; s < 4; ++s) {
            sm100::mbar_init(b1_full + s, 1);
            sm100::mbar_init(b2_full + s, 1);
            sm100::mbar_init(st_ready + s, 128);
            sm100::mbar_init(st_free + s, 1);
        }
        sm100::mbar_init(drain_x, 1);
        sm100::mbar_init(drain_g, 1);
        *abort_flag = 0;
        sm100::fence_mbar_init();
    }
    if (warp == BWD_X_WARP) {
        sm100::tmem_alloc(tmem_slot, 512);
        sm100::tmem_relinquish();
    }
    if (warp == BWD_TMA_WARP && lane == 0) {
        sm100::prefetch_tmap(&tm_a1);
        sm100::prefetch_tmap(&tm_a2);
        sm100::prefetch_tmap(&tm_b1);
        sm100::prefetch_tmap(&tm_b2);
    }
    const bool is_prep = warp >= BWD_PREP_WARP0;
    const int ptid = threadIdx.x - 32 * BWD_PREP_WARP0;
    if (is_prep && ptid < D / 2) {   // RoPE frequencies for the epilogue's inverse rotation
        const double th = exp2(-2.0 * (double)ptid / (double)D * a.log2_base);
        sTh[ptid] = th;
        sThf[ptid] = (float)th;
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == BWD_TMA_WARP) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stat_par[2] = {-1, -1}, st_par[4] = {-1, -1, -1, -1};
            int ts = 0, k = 0;
            bool ok = true;
            for (int u = u_begin; ok && u < u_end; ++u, ++k) {
                const BwdItem it = bwd_item<ROLE>(a, u);
                const int sb = k % NSTAT;
                if (k >= NSTAT && !sm100::mbar_wait(stat_free + sb, ((k / NSTAT) - 1) & 1, abort_flag)) break;
                const int head_a = (ROLE == BWD_ROLE_DKDV) ? it.kvh : it.h;
                sm100::mbar_arrive_expect_tx(stat_full + sb, 2 * C::TILE);
                for (int hh = 0; hh < D / 64; ++hh) {
                    sm100::tma_load_4d(sA1 + sb * C::TILE + hh * C::HALF_BYTES, &tm_a1, stat_full + sb, hh * 64, head_a, it.row0, it.b);
                    sm100::tma_load_4d(sA2 + sb * C::TILE + hh * C::HALF_BYTES, &tm_a2, stat_full + sb, hh * 64, head_a, it.row0, it.b);
                }
                stat_par[sb] = (k / NSTAT) & 1;
                for (int t = 0; t < it.T; ++t, ++ts) {
                    const int s = ts % NST;
                    if (ts >= NST && !sm100::mbar_wait(st_free + s, ((ts / NST) - 1) & 1, abort_flag)) { ok = false; break; }
                    int head, pos0;
                    bwd_stream<ROLE>(it, G, t, head, pos0);
                    sm100::mbar_arrive_expect_tx(b1_full + s, C::TILE);
                    for (int hh = 0; hh < D / 64; ++hh)
                        sm100::tma_load_4d(sB1 + s * C::TILE + hh * C::HALF_BYTES, &tm_b1, b1_full + s, hh * 64, head, pos0, it.b);
                    sm100::mbar_arrive_expect_tx(b2_full + s, C::TILE);
                    for (int hh = 0; hh < D / 64; ++hh)
                        sm100::tma_load_4d(sB2 + s * C::TILE + hh * C::HALF_BYTES, &tm_b2, b2_full + s, hh * 64, head, pos0, it.b);
                    st_par[s] = (ts / NST) & 1;
                }
            }
            // every issued copy must have landed before the CTA may exit
            for (int s = 0; s < 2; ++s)
                if (stat_par[s] >= 0) mbar_wait_drain(stat_full + s, stat_par[s]);
            for (int s = 0; s < 4; ++s)
                if (st_par[s] >= 0) { mbar_wait_drain(b1_full + s, st_par[s]); mbar_wait_drain(b2_full + s, st_par[s]); }
        }
    } else if (warp == BWD_X_WARP) {
        // ------------------------------------------------------------ X MMAs: S half and dP half
        if (lane == 0) {
            constexpr uint32_t IDESC_X = sm100::idesc_bf16_f32(128, 64, 0, 0);
            const uint64_t d0 = sm100::sdesc_sw128(sm100::smem_u32(smem), 16, 1024);
            const uint32_t hi = (uint32_t)(d0 >> 32), lo0 = (uint32_t)d0;   // lo0 + (byte offset >> 4)
            auto dsc = [&](uint32_t off_bytes) { return ((uint64_t)hi << 32) | (lo0 + (off_bytes >> 4)); };
            int ts = 0, k = 0, hs = 0;
            bool ok = true;
            for (int u = u_begin; ok && u < u_end; ++u, ++k) {
                const BwdItem it = bwd_item<ROLE>(a, u);
                const int sb = k % NSTAT;
                if (!sm100::mbar_wait(stat_full + sb, (k / NSTAT) & 1, abort_flag)) break;
                const uint32_t a1 = C::OFF_A1 + sb * C::TILE, a2 = C::OFF_A2 + sb * C::TILE;
                for (int t = 0; ok && t < it.T; ++t, ++ts) {
                    const int s = ts % NST;
                    if (!sm100::mbar_wait(b1_full + s, (ts / NST) & 1, abort_flag) ||
                        !sm100::mbar_wait(b2_full + s, (ts / NST) & 1, abort_flag)) { ok = false; break; }
                    const uint32_t b1 = C::OFF_B1 + s * C::TILE, b2 = C::OFF_B2 + s * C::TILE;
                    for (int h = 0; h < 2; ++h, ++hs) {
                        // buffer h is free again once its previous half-step's S / dP were
                        // consumed: by the element-wise pass (P, dS elsewhere) or, when
                        // P / dS overlay S / dP, by the gradient MMAs
                        constexpr int NB = C::NBUF;
                        const int bf = hs % NB;
                        if (hs >= NB && !sm100::mbar_wait(C::SEP_PD ? p_full + bf : buf_free + bf, ((hs / NB) - 1) & 1,
                                                         abort_flag)) { ok = false; break; }
                        sm100::tc_fence_after();
                        const uint32_t dx = tmem + bf * 128;
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint32_t off = (ks / 4) * C::HALF_BYTES + (ks % 4) * 32;
                            sm100::umma_ss(dx, dsc(a1 + off), dsc(b1 + h * 8192 + off), IDESC_X, ks > 0 ? 1u : 0u);
                        }
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint32_t off = (ks / 4) * C::HALF_BYTES + (ks % 4) * 32;
                            sm100::umma_ss(dx + 64, dsc(a2 + off), dsc(b2 + h * 8192 + off), IDESC_X, ks > 0 ? 1u : 0u);
                        }
                        sm100::umma_commit(x_full + bf);
                    }
                }
                if (ok) sm100::umma_commit(stat_free + sb);   // the item's stationary tiles are read
            }
            sm100::umma_commit(drain_x);
            mbar_wait_drain(drain_x, 0);
        }
        __syncwarp();
    } else if (warp == BWD_G_WARP) {
        // ------------------------------------------------------------ gradient MMAs
        if (lane == 0) {
            constexpr uint32_t IDESC_G = sm100::idesc_bf16_f32(128, D, 0, 1);
            const uint64_t d0 = sm100::sdesc_sw128(sm100::smem_u32(smem), C::HALF_BYTES, 1024);   // MN-major B
            const uint32_t hi = (uint32_t)(d0 >> 32), lo0 = (uint32_t)d0;
            auto dsc = [&](uint32_t off_bytes) { return ((uint64_t)hi << 32) | (lo0 + (off_bytes >> 4)); };
            int ts = 0, k = 0, hs = 0;
            bool ok = true;
            for (int u = u_begin; ok && u < u_end; ++u, ++k) {
                const BwdItem it = bwd_item<ROLE>(a, u);
                const int ab = k % NACC;
                const uint32_t acc = tmem + C::ACC_BASE + ab * C::ACC_COLS;
                for (int t = 0; ok && t < it.T; ++t, ++ts) {
                    const int s = ts % NST;
                    const uint32_t b1 = C::OFF_B1 + s * C::TILE, b2 = C::OFF_B2 + s * C::TILE;
                    for (int h = 0; h < 2; ++h, ++hs) {
                        constexpr int NB = C::NBUF;
                        const int bf = hs % NB;
                        if (!sm100::mbar_wait(p_full + bf, (hs / NB) & 1, abort_flag)) { ok = false; break; }
                        if (ROLE != BWD_ROLE_DSUM) {
                            const bool first = (t == 0 && h == 0);
                            if (first && k >= NACC && !sm100::mbar_wait(acc_free + ab, ((k / NACC) - 1) & 1, abort_flag)) {
                                ok = false;
                                break;
                            }
                            sm100::tc_fence_after();
                            const uint32_t pa = C::SEP_PD ? tmem + C::NBUF * 128 + bf * C::PD_COLS : tmem + bf * 128;
                            const uint32_t da = C::SEP_PD ? pa + (ROLE == BWD_ROLE_DKDV ? 32 : 0) : tmem + bf * 128 + 64;
                            if (ROLE == BWD_ROLE_DKDV) {
#pragma unroll
                                for (int ks = 0; ks < 4; ++ks)    // dV += P^T dO
                                    sm100::umma_ts(acc, pa + ks * 8, dsc(b2 + h * 8192 + ks * 2048), IDESC_G,
                                                   (first && ks == 0) ? 0u : 1u);
#pragma unroll
                                for (int ks = 0; ks < 4; ++ks)    // dK' += dS^T Q'
                                    sm100::umma_ts(acc + D, da + ks * 8, dsc(b1 + h * 8192 + ks * 2048), IDESC_G,
                                                   (first && ks == 0) ? 0u : 1u);
                            } else {
#pragma unroll
                                for (int ks = 0; ks < 4; ++ks)    // dQ' += dS K'
                                    sm100::umma_ts(acc, da + ks * 8, dsc(b1 + h * 8192 + ks * 2048), IDESC_G,
                                                   (first && ks == 0) ? 0u : 1u);
                            }
                        }
                        sm100::umma_commit(buf_free + bf);
                        if (h == 1) sm100::umma_commit(st_free + s);   // the step's streamed tiles are read
                        if (ROLE != BWD_ROLE_DSUM && h == 1 && t == it.T - 1) sm100::umma_commit(acc_full + ab);
                    }
                }
            }
            sm100::umma_commit(drain_g);
            mbar_wait_drain(drain_g, 0);
        }
        __syncwarp();
    } else if (warp >= BWD_ACT_WARP0 && warp < BWD_ACT_WARP0 + 4 * C::NWG) {
        // ------------------------------------------------------------ activation + epilogue
        constexpr int NWG = C::NWG;
        const int w = (warp - BWD_ACT_WARP0) / 4;                 // warpgroup: half-steps hs = w mod NWG
        const int r = 32 * (warp % 4) + lane;                     // stationary row (= TMEM lane)
        const int wtid = threadIdx.x - 32 * (BWD_ACT_WARP0 + 4 * w);   // 0..127
        const uint32_t lane_base = (uint32_t)(32 * (warp % 4)) << 16;
        const float LOG2E = 1.4426950408889634f;
        const bool sig = (MODE == SWAT_MODE_SIGMOID_);
        const float xs = sig ? 0.5f * a.scale : a.scale * LOG2E;
        const float bmul = sig ? 0.5f : LOG2E;                    // bias units
        struct PendE { int k, b, h, kvh, row0; };
        PendE pend{};
        bool has_pend = false;
        int nmine = 0;                                            // half-steps done here
        // Stop decisions (abort) are taken per warp, except where the warpgroup
        // meets at a named barrier after them (dk/dv softmax: per-column rows).
        constexpr bool WG_BAR = (ROLE == BWD_ROLE_DKDV && MODE == SWAT_MODE_SOFTMAX_);
        auto stop_any = [&](bool v) -> bool {
            return WG_BAR ? named_bar_or(2 + w, 128, v) : (__any_sync(0xffffffffu, v) != 0);
        };
        auto epilogue = [&](const PendE &p) -> bool {
            if (ROLE == BWD_ROLE_DSUM) {
                const int ib = p.k & 1;
                const bool ok = sm100::mbar_wait(dsum_full + ib, (p.k >> 1) & 1, abort_flag);
                if (stop_any(!ok)) return false;
                float dsum = 0.f;
#pragma unroll
                for (int j = 0; j < NWG; ++j) dsum += sDsum[(ib * NWG + j) * 128 + r];
                const int i = p.row0 + r;
                if (i < a.N) a.Dws[((size_t)p.b * a.H + p.h) * a.N + i] = dsum;
                sm100::mbar_arrive(dsum_free + ib);
                return true;
            }
            const int ab = p.k % NACC;
            const bool ok = sm100::mbar_wait(acc_full + ab, (p.k / NACC) & 1, abort_flag);
            if (stop_any(!ok)) return false;
            sm100::tc_fence_after();
            // base angles of the item's rows, one copy per warp (no warpgroup barrier)
            float *A0 = sA0 + (w * 4 + (warp % 4)) * (D / 2);
            if (a.use_rope) {
                __syncwarp();   // the previous epilogue's reads of this copy are done
                for (int t = lane; t < D / 2; t += 32) {
                    const double two_pi = 6.283185307179586476925286766559;
                    const double x = (double)p.row0 * sTh[t];
                    A0[t] = (float)(x - rint(x / two_pi) * two_pi);
                }
                __syncwarp();
            }
            const uint32_t acc = tmem + lane_base + C::ACC_BASE + ab * C::ACC_COLS;
            const int row = p.row0 + r;
            if (ROLE == BWD_ROLE_DQ) {
                __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(a.dq) + (((size_t)p.b * a.N + row) * a.H + p.h) * D;
                unrotate_store_row<D>(acc, r, A0, sThf, a.use_rope, dst, row < a.N, a.scale);   // dS = g scale
            } else {
                const size_t o = (((size_t)p.b * a.N + row) * a.Hkv + p.kvh) * D;
                store_row_bf16_plain<D>(acc, reinterpret_cast<__nv_bfloat16 *>(a.dv) + o, row < a.N);
                // dK' is read last: the accumulators are released after its final TMEM load
                unrotate_store_row<D>(acc + D, r, A0, sThf, a.use_rope, reinterpret_cast<__nv_bfloat16 *>(a.dk) + o,
                                      row < a.N, a.scale, acc_free + ab);
                return true;
            }
            sm100::tc_fence_before();
            sm100::mbar_arrive(acc_free + ab);
            return true;
        };
        int ts = 0, k = 0;
        bool good = true;
        for (int u = u_begin; good && u < u_end; ++u, ++k) {
            const BwdItem it = bwd_item<ROLE>(a, u);
            const int row = it.row0 + r;
            // per-row softmax terms (DQ, DSUM: the row is a query)
            float lrow = 0.f, drow = 0.f;
            if (!sig && ROLE != BWD_ROLE_DKDV && row < a.N) {
                lrow = a.lse[((size_t)it.b * a.H + it.h) * a.N + row] * LOG2E;
                if (ROLE == BWD_ROLE_DQ) drow = a.Dws[((size_t)it.b * a.H + it.h) * a.N + row];
            }
            float dsum = 0.f;
            // epilogue of this item: the warpgroup of its last half-step (2 groups: by item parity)
            const int ep_w = (NWG == 2) ? (k & 1) : ((2 * (ts + it.T - 1) + 1) % NWG);
            // ALiBi slope of each step's query head, loaded one step ahead
            int head_n, pos_n;
            bwd_stream<ROLE>(it, G, 0, head_n, pos_n);
            float slope_n = a.slopes ? __ldg(a.slopes + (ROLE == BWD_ROLE_DKDV ? head_n : it.h)) : 0.f;
            for (int t = 0; good && t < it.T; ++t, ++ts) {
                int head, pos0;
                bwd_stream<ROLE>(it, G, t, head, pos0);
                const float slope = slope_n;
                if (ROLE == BWD_ROLE_DKDV && t + 1 < it.T && a.slopes) {
                    bwd_stream<ROLE>(it, G, t + 1, head_n, pos_n);
                    slope_n = __ldg(a.slopes + head_n);
                }
                for (int h = 0; h < 2; ++h) {
                const int hsm = 2 * ts + h;                           // this half-step
                if (hsm % NWG != w) continue;
                const int cb = pos0 + 64 * h;                         // first streamed row of this half
                const float *colL = nullptr, *colD = nullptr;
                if (!sig && ROLE == BWD_ROLE_DKDV) {
                    // lse (log2 units) and D of the 64 queries of this half
                    float *rows = sRows + (w * 2 + (nmine & 1)) * 128;
                    const int c = wtid & 63, iq = cb + c;
                    float val = 0.f;
                    if (iq < a.N) {
                        const size_t o = ((size_t)it.b * a.H + head) * a.N + iq;
                        val = (wtid < 64) ? a.lse[o] * LOG2E : a.Dws[o];
                    }
                    rows[wtid] = val;
                    sm100::named_bar_sync(2 + w, 128);
                    colL = rows;
                    colD = rows + 64;
                }

                // column masks and ALiBi bias of this half
                uint32_t m[2];
                float b0, bstep;
                if (ROLE == BWD_ROLE_DKDV) {
                    const int lo = row - cb;                          // column of query i = j
                    int hi = (row < a.n_sink) ? 63 : lo + a.window - 1;
                    hi = min(hi, a.N - 1 - cb);
                    m[0] = interval_bits32(lo, hi, 0);
                    m[1] = interval_bits32(lo, hi, 32);
                    b0 = -slope * (float)lo * bmul;                   // slope (i - j), i = cb + c
                    bstep = slope * bmul;
                } else {
                    const int rd = row - cb;                          // i - j for column 0
                    const RowMask mk = row_mask(rd, cb, a.window, a.n_sink);
                    m[0] = col_bits32(mk, 0);
                    m[1] = col_bits32(mk, 32);
                    b0 = slope * (float)rd * bmul;
                    bstep = -slope * bmul;
                }
                const int bf = hsm % C::NBUF;                         // its TMEM buffer
                const bool ok = sm100::mbar_wait(x_full + bf, (hsm / C::NBUF) & 1, abort_flag);
                if (stop_any(!ok)) { good = false; break; }
                sm100::tc_fence_after();
                if (C::SEP_PD && hsm >= C::NBUF) {
                    // P / dS columns of this buffer: read by the previous half-step's gradient MMAs
                    const bool okp = sm100::mbar_wait(buf_free + bf, ((hsm / C::NBUF) - 1) & 1, abort_flag);
                    if (stop_any(!okp)) { good = false; break; }
                    sm100::tc_fence_after();
                }
                const uint32_t x_addr = tmem + lane_base + bf * 128;
                const uint32_t p_addr = C::SEP_PD ? tmem + lane_base + C::NBUF * 128 + bf * C::PD_COLS : x_addr;
                const uint32_t ds_addr = C::SEP_PD ? p_addr + (ROLE == BWD_ROLE_DKDV ? 32 : 0) : x_addr + 64;
                if (ROLE == BWD_ROLE_DSUM)
                    dsum += bwd_half_step<MODE, false, false, true>(x_addr, p_addr, ds_addr, xs, b0, bstep, m, lrow,
                                                                    drow, colL, colD);
                else if (ROLE == BWD_ROLE_DQ)
                    bwd_half_step<MODE, false, true, false>(x_addr, p_addr, ds_addr, xs, b0, bstep, m, lrow, drow,
                                                            colL, colD);
                else
                    bwd_half_step<MODE, true, true, false>(x_addr, p_addr, ds_addr, xs, b0, bstep, m, lrow, drow,
                                                           colL, colD);
                sm100::tmem_wait_st();
                sm100::tc_fence_before();
                sm100::mbar_arrive(p_full + bf);
                ++nmine;
                if (has_pend) {
                    has_pend = false;
                    if (!epilogue(pend)) { good = false; break; }
                }
                if (t == it.T - 1) {
                    if (ROLE == BWD_ROLE_DSUM) {
                        const int ib = k & 1;
                        if (k >= 2) {
                            const bool okf = sm100::mbar_wait(dsum_free + ib, ((k >> 1) - 1) & 1, abort_flag);
                            if (stop_any(!okf)) { good = false; break; }
                        }
                        sDsum[(ib * NWG + w) * 128 + r] = dsum;
                        sm100::mbar_arrive(dsum_full + ib);
                    }
                    if (w == ep_w) {
                        pend = PendE{k, it.b, it.h, it.kvh, it.row0};
                        has_pend = true;
                        if (NACC == 1) {   // one accumulator set: the next item's MMAs wait for it, so now
                            has_pend = false;
                            if (!epilogue(pend)) { good = false; break; }
                        }
                    }
                }
                }   // half
            }
        }
        if (good && has_pend) epilogue(pend);
    }

    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    if (warp == BWD_X_WARP) sm100::tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// Host launch: persistent grids (one CTA per SM, at most one per item).
// Softmax: DSUM (D_i into the workspace) first, then DQ and DKDV.
// ---------------------------------------------------------------------------
template <int D, int MODE, int ROLE>
inline bool launch_bwd_role(const BwdArgs &a, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                            const CUtensorMap &tdo, cudaStream_t stream)
{
    using C = BwdCfg<D, ROLE>;
    auto kern = swat_bwd_tc_kernel<D, MODE, ROLE>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess) return false;
    const long long nQT = (a.N + 127) / 128;
    const long long U = (ROLE == BWD_ROLE_DKDV) ? (long long)a.B * a.Hkv * nQT : (long long)a.B * a.H * nQT;
    if (U >= (1LL << 31)) return false;   // item indices are decoded in 32 bits
    const int grid = (int)std::min<long long>(U, (long long)num_sms());
    if (ROLE == BWD_ROLE_DKDV)
        kern<<<grid, BWD_THREADS, C::SMEM, stream>>>(tk, tv, tq, tdo, a);
    else
        kern<<<grid, BWD_THREADS, C::SMEM, stream>>>(tq, tdo, tk, tv, a);
    return true;
}

template <int D, int MODE>
inline int launch_bwd_tc_t(const BwdArgs &a, void *extra_ws, const void *qk_rot, cudaStream_t stream)
{
    int n = 0;
    const void *qr = a.q, *kr = a.k;
    if (a.use_rope && qk_rot) {   // the forward's rotated copies (same layout)
        qr = qk_rot;
        kr = reinterpret_cast<const char *>(qk_rot) + align256((size_t)a.B * a.N * a.H * D * 2);
    } else if (a.use_rope) {      // rotated copies of Q and K in the workspace
        n += launch_rope_copies<D>(a.q, a.k, extra_ws, a.B, a.H, a.Hkv, a.N, a.log2_base, stream, &qr, &kr);
    }
    CUtensorMap tq, tk, tv, tdo;
    if (!make_tmap_bshd(&tq, qr, a.B, a.N, a.H, D) || !make_tmap_bshd(&tk, kr, a.B, a.N, a.Hkv, D) ||
        !make_tmap_bshd(&tv, a.v, a.B, a.N, a.Hkv, D) || !make_tmap_bshd(&tdo, a.dout, a.B, a.N, a.H, D))
        return -1;
    if (MODE == SWAT_MODE_SOFTMAX_) {
        if (!launch_bwd_role<D, MODE, BWD_ROLE_DSUM>(a, tq, tk, tv, tdo, stream)) return -1;
        ++n;
    }
    if (!launch_bwd_role<D, MODE, BWD_ROLE_DQ>(a, tq, tk, tv, tdo, stream)) return -1;
    if (!launch_bwd_role<D, MODE, BWD_ROLE_DKDV>(a, tq, tk, tv, tdo, stream)) return -1;
    return n + 2;
}

// Workspace after the softmax D_i: RoPE-rotated copies of Q and K (bf16).
inline size_t tc_bwd_extra_workspace(int B, int H, int Hkv, int N, int d)
{
    return rope_copies_bytes(B, H, Hkv, N, d);
}

// Returns the number of kernels launched, or -1 on a launch-configuration error.
// qk_rot: NULL, or the rotated copies a swat_attn_fwd_ws call wrote for
// the same q and k (skips the rotation kernels).
inline int launch_bwd_tc(const BwdArgs &a, void *extra_ws, const void *qk_rot, cudaStream_t stream)
{
    if (a.d == 64)
        return a.mode == SWAT_MODE_SIGMOID_ ? launch_bwd_tc_t<64, SWAT_MODE_SIGMOID_>(a, extra_ws, qk_rot, stream)
                                            : launch_bwd_tc_t<64, SWAT_MODE_SOFTMAX_>(a, extra_ws, qk_rot, stream);
    if (a.d == 128)
        return a.mode == SWAT_MODE_SIGMOID_ ? launch_bwd_tc_t<128, SWAT_MODE_SIGMOID_>(a, extra_ws, qk_rot, stream)
                                            : launch_bwd_tc_t<128, SWAT_MODE_SOFTMAX_>(a, extra_ws, qk_rot, stream);
    return -1;
}

}  // namespace swat
