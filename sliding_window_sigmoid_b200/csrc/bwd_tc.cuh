// bwd_tc.cuh — bf16 SWAT backward on 5th-generation tensor cores (sm_100a).
//
// Gradients of the attention equation of "SWAT: Sliding Window Attention
// Training" (section "Balanced ALiBi"), derived by calculus (the pages train
// SWAT from scratch but print no backward):
//   dv_j = sum_i p_ij dO_i,  dP_ij = dO_i . v_j,
//   sigmoid: dS_ij = dP_ij p_ij (1 - p_ij);  softmax: dS_ij = p_ij (dP_ij - D_i)
//   dq'_i = sum_j dS_ij k'_j / sqrt(d),  dk'_j = sum_i dS_ij q'_i / sqrt(d),
//   dq = R_i^T dq', dk = R_j^T dk'.
// Two kernels, no atomics (every output row has one owner, results are
// deterministic):
//   dq kernel   (query tile per CTA):  S = Q'K'^T, dP = dO V^T, dS in registers,
//                                     dQ' += dS K'          (dS as TMEM A operand)
//   dkdv kernel (key tile per CTA, all query heads of the KV group):
//                S^T = K'Q'^T, dP^T = V dO^T, P^T and dS^T in registers,
//                dV += P^T dO, dK' += dS^T Q'            (TMEM A operands)
// Roles (384 threads): warp 0 issues MMAs, warp 1 TMA copies, warps 4-7 the
// element-wise math and the epilogue (one tile row per thread = TMEM lane),
// warps 8-11 rotate the streamed Q or K tiles (RoPE) in shared memory.
// TMEM: [0,128) S (its first 64 columns then hold the bf16 dS or P),
// [128,256) dP (then dS^T in the dkdv kernel), accumulators from 256.
#pragma once
#include "fwd_tc.cuh"

namespace swat {

constexpr int BWD_MMA_WARP = 0, BWD_TMA_WARP = 1, BWD_ACT_WARP0 = 4, BWD_PREP_WARP0 = 8;
constexpr int BWD_THREADS = 384;

template <int D>
struct BwdTcCfg {
    static constexpr int TILE_BYTES = 128 * D * 2;
    static constexpr int HALF_BYTES = 128 * 128;
    static constexpr int NST = (D == 64) ? 3 : 2;          // streamed-tile stages
    // fixed tiles (A, B) + streamed pairs (C[NST], E[NST])
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + TILE_BYTES;
    static constexpr int OFF_C = OFF_B + TILE_BYTES;
    static constexpr int OFF_E = OFF_C + NST * TILE_BYTES;
    static constexpr int OFF_ROT = OFF_E + NST * TILE_BYTES;  // float2 [2][D/2] bases
    static constexpr int OFF_TH = OFF_ROT + 2 * (D / 2) * 8;  // double [D/2]
    static constexpr int OFF_A0 = OFF_TH + (D / 2) * 8;       // float [D/2] epilogue base angle
    static constexpr int OFF_THF = OFF_A0 + (D / 2) * 4;      // float [D/2]
    static constexpr int OFF_ROWS = OFF_THF + (D / 2) * 4;    // float [NST][2][128] (lse, D per query)
    static constexpr int OFF_BAR = OFF_ROWS + NST * 2 * 128 * 4;
    static constexpr int NBAR = 2 + 4 * NST + 4;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
};

// Inverse RoPE of one accumulator row held in TMEM (fp32, D columns), for a
// row at absolute position pos0 + r; the angle is A0[t] + r theta_t (A0 is the
// position pos0 reduced in fp64), reduced again in fp32 before __sincosf.
template <int D>
__device__ __forceinline__ void unrotate_store_row(uint32_t taddr, int r, const float *A0, const float *THF,
                                                   bool use_rope, __nv_bfloat16 *dst, bool store)
{
    const float two_pi = 6.2831853071795865f, inv_two_pi = 0.15915494309189534f;
#pragma unroll
    for (int k = 0; k < D / 32; ++k) {
        uint32_t v[32];
        sm100::tmem_ld32(taddr + 32 * k, v);
        sm100::tmem_wait_ld_dep(v);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            float x0 = __uint_as_float(v[2 * e]), x1 = __uint_as_float(v[2 * e + 1]);
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

__device__ __forceinline__ void store_row_bf16_plain(uint32_t taddr, int D, __nv_bfloat16 *dst, bool store)
{
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

// dS of one 128x128 tile, one row per thread: reads S and dP (TMEM, fp32),
// writes bf16 dS (scaled by 1/sqrt(d)) over the first 64 columns of the S
// buffer (at `out_addr`), and, when `p_addr` != 0, bf16 P over another
// buffer's first 64 columns (WRITE_P). `valid(c)` masks column c. Element-wise:
//   sigmoid: x = s/sqrt(d) + bias_c, t = tanh(x/2), p = (1+t)/2,
//            dS = dP (1 - t^2) / 4 / sqrt(d)
//   softmax: p = exp(x - lse), dS = p (dP - Dr) / sqrt(d)
template <int MODE, bool MASKED, bool WRITE_P, typename BiasF, typename ValidF, typename RowVal>
__device__ __forceinline__ void bwd_ds_tile(uint32_t s_addr, uint32_t dp_addr, uint32_t out_addr, uint32_t p_addr,
                                            float scale, BiasF bias_of, ValidF valid, RowVal rowval)
{
#pragma unroll 1
    for (int k = 0; k < 8; ++k) {
        uint32_t sv[16], dv[16];
        sm100::tmem_ld16(s_addr + 16 * k, sv);
        sm100::tmem_ld16(dp_addr + 16 * k, dv);
        sm100::tmem_wait_ld_dep16(sv);
        sm100::tmem_wait_ld_dep16(dv);
        uint32_t dk[8], pkk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float ds[2], pp[2];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int c = 16 * k + 2 * e + h2;
                const float s = __uint_as_float(sv[2 * e + h2]), dp = __uint_as_float(dv[2 * e + h2]);
                float lse_or_zero, Dr;
                rowval(c, lse_or_zero, Dr);
                const float x = fmaf(s, scale, bias_of(c));
                float p, g;
                if (MODE == SWAT_MODE_SIGMOID_) {
                    const float th = sm100::tanh_approx(0.5f * x);
                    p = fmaf(0.5f, th, 0.5f);
                    g = dp * fmaf(-th, th, 1.f) * (0.25f * scale);
                } else {
                    p = __expf(x - lse_or_zero);
                    g = p * (dp - Dr) * scale;
                }
                if (MASKED && !valid(c)) { p = 0.f; g = 0.f; }
                ds[h2] = g; pp[h2] = p;
            }
            dk[e] = sm100::pack_bf16x2(ds[0], ds[1]);
            pkk[e] = sm100::pack_bf16x2(pp[0], pp[1]);
        }
        sm100::tmem_st8(out_addr + 8 * k, dk);
        if (WRITE_P) sm100::tmem_st8(p_addr + 8 * k, pkk);
    }
}

// Softmax row term D_i = sum_j p_ij dP_ij of one tile (fp32, masked), the
// exact form of dO_i . o_i (it does not depend on the rounding of o).
template <bool MASKED, typename BiasF, typename ValidF>
__device__ __forceinline__ float bwd_rowsum_tile(uint32_t s_addr, uint32_t dp_addr, float scale, float lse,
                                                 BiasF bias_of, ValidF valid)
{
    float acc = 0.f;
#pragma unroll 1
    for (int k = 0; k < 8; ++k) {
        uint32_t sv[16], dv[16];
        sm100::tmem_ld16(s_addr + 16 * k, sv);
        sm100::tmem_ld16(dp_addr + 16 * k, dv);
        sm100::tmem_wait_ld_dep16(sv);
        sm100::tmem_wait_ld_dep16(dv);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int c = 16 * k + e;
            float p = __expf(fmaf(__uint_as_float(sv[e]), scale, bias_of(c)) - lse);
            if (MASKED && !valid(c)) p = 0.f;
            acc = fmaf(p, __uint_as_float(dv[e]), acc);
        }
    }
    return acc;
}

// ===========================================================================
// dq kernel: one CTA per (b, h, 128-row query tile); key tiles streamed.
// With DPASS (softmax mode, launched first) it only computes D_i into the
// workspace: the same S and dP, no dQ' product.
// smem A = Q (rotated), B = dO, C[] = K (rotated), E[] = V.
// ===========================================================================
template <int D, int MODE, bool DPASS>
__global__ void __launch_bounds__(BWD_THREADS, 1)
swat_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const BwdArgs a, float *dq_f32_unused)
{
    (void)dq_f32_unused;
    using C = BwdTcCfg<D>;
    constexpr int NST = C::NST;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + C::OFF_A, *sDO = smem + C::OFF_B, *sK = smem + C::OFF_C, *sV = smem + C::OFF_E;
    float2 *sRot = reinterpret_cast<float2 *>(smem + C::OFF_ROT);
    double *sTh = reinterpret_cast<double *>(smem + C::OFF_TH);
    float *sA0 = reinterpret_cast<float *>(smem + C::OFF_A0);
    float *sThf = reinterpret_cast<float *>(smem + C::OFF_THF);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *q_full = bars, *q_ready = bars + 1;
    uint64_t *k_full = bars + 2, *k_ready = k_full + NST, *v_full = k_ready + NST, *release = v_full + NST;
    uint64_t *s_full = release + NST, *p_full = s_full + 1, *o_full = p_full + 1, *drain = o_full + 1;
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
            sm100::mbar_init(release + s, 1);
        }
        sm100::mbar_init(s_full, 1);
        sm100::mbar_init(p_full, 128);
        sm100::mbar_init(o_full, 1);
        sm100::mbar_init(drain, 1);
        *abort_flag = 0;
        sm100::fence_mbar_init();
    }
    if (warp == BWD_MMA_WARP) {
        sm100::tmem_alloc(tmem_slot, 512);
        sm100::tmem_relinquish();
    }
    const bool is_prep = warp >= BWD_PREP_WARP0;
    const int ptid = threadIdx.x - 32 * BWD_PREP_WARP0;
    RotThread rot;
    if (is_prep && a.use_rope) {
        if (ptid < D / 2) {
            const double th = exp2(-2.0 * (double)ptid / (double)D * a.log2_base);
            sTh[ptid] = th;
            sThf[ptid] = (float)th;
            const double two_pi = 6.283185307179586476925286766559;
            const double x = (double)i0 * th;
            sA0[ptid] = (float)(x - rint(x / two_pi) * two_pi);
        }
        sm100::named_bar_sync(FWD_PREP_BAR, 128);
        constexpr int CPR = D / 8, RS = 128 / CPR;
        const int c = ptid % CPR, r0 = ptid / CPR;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const double th = sTh[4 * c + q];
            const float2 w0 = rope_cs((double)r0 * th), stp = rope_cs((double)RS * th);
            rot.w0c[q] = w0.x; rot.w0s[q] = w0.y; rot.stc[q] = stp.x; rot.sts[q] = stp.y;
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == BWD_TMA_WARP) {
        if (lane == 0) {
            int last_par[NST];
            for (int s = 0; s < NST; ++s) last_par[s] = -1;
            sm100::mbar_arrive_expect_tx(q_full, 2 * C::TILE_BYTES);
            for (int hh = 0; hh < D / 64; ++hh) {
                sm100::tma_load_4d(sQ + hh * C::HALF_BYTES, &tm_q, q_full, hh * 64, h, i0, b);
                sm100::tma_load_4d(sDO + hh * C::HALF_BYTES, &tm_do, q_full, hh * 64, h, i0, b);
            }
            for (int t = 0; t < T; ++t) {
                const int st = t % NST, n = t / NST;
                if (n > 0 && !sm100::mbar_wait(release + st, (n - 1) & 1, abort_flag)) break;
                const int j0 = fwd_tile_j0(tr, t);
                sm100::mbar_arrive_expect_tx(k_full + st, C::TILE_BYTES);
                for (int hh = 0; hh < D / 64; ++hh)
                    sm100::tma_load_4d(sK + st * C::TILE_BYTES + hh * C::HALF_BYTES, &tm_k, k_full + st, hh * 64, kvh, j0, b);
                sm100::mbar_arrive_expect_tx(v_full + st, C::TILE_BYTES);
                for (int hh = 0; hh < D / 64; ++hh)
                    sm100::tma_load_4d(sV + st * C::TILE_BYTES + hh * C::HALF_BYTES, &tm_v, v_full + st, hh * 64, kvh, j0, b);
                last_par[st] = n & 1;
            }
            mbar_wait_drain(q_full, 0);
            for (int s = 0; s < NST; ++s)
                if (last_par[s] >= 0) { mbar_wait_drain(k_full + s, last_par[s]); mbar_wait_drain(v_full + s, last_par[s]); }
        }
    } else if (is_prep) {
        int ebuf = 0;
        auto make_bases = [&](int pos0) {
            ebuf ^= 1;
            if (a.use_rope && ptid < D / 2) sRot[ebuf * (D / 2) + ptid] = rope_cs((double)pos0 * sTh[ptid]);
        };
        make_bases(i0);
        bool ok = sm100::mbar_wait(q_full, 0, abort_flag);
        if (!named_bar_or(FWD_PREP_BAR, 128, !ok || *abort_flag)) {
            if (a.use_rope) rope_rotate_tile<D>(sQ, sRot + ebuf * (D / 2), rot, ptid);
            sm100::fence_proxy_async_smem();
            sm100::mbar_arrive(q_ready);
            for (int t = 0; t < T; ++t) {
                const int st = t % NST, n = t / NST;
                make_bases(fwd_tile_j0(tr, t));
                ok = sm100::mbar_wait(k_full + st, n & 1, abort_flag);
                if (named_bar_or(FWD_PREP_BAR, 128, !ok || *abort_flag)) break;
                if (a.use_rope) rope_rotate_tile<D>(sK + st * C::TILE_BYTES, sRot + ebuf * (D / 2), rot, ptid);
                sm100::fence_proxy_async_smem();
                sm100::mbar_arrive(k_ready + st);
            }
        }
    } else if (warp == BWD_MMA_WARP) {
        if (lane == 0) {
            constexpr uint32_t IDESC_S = sm100::idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t IDESC_DQ = sm100::idesc_bf16_f32(128, D, 0, 1);
            const uint32_t qa = sm100::smem_u32(sQ), doa = sm100::smem_u32(sDO);
            bool ok = sm100::mbar_wait(q_ready, 0, abort_flag);
            for (int t = 0; ok && t < T; ++t) {
                const int st = t % NST, n = t / NST;
                if (!sm100::mbar_wait(k_ready + st, n & 1, abort_flag) || !sm100::mbar_wait(v_full + st, n & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                sm100::tc_fence_after();
                const uint32_t ka = sm100::smem_u32(sK + st * C::TILE_BYTES), va = sm100::smem_u32(sV + st * C::TILE_BYTES);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks / 4) * C::HALF_BYTES + (ks % 4) * 32;
                    sm100::umma_ss(tmem + 0, sm100::sdesc_sw128(qa + off, 16, 1024), sm100::sdesc_sw128(ka + off, 16, 1024),
                                   IDESC_S, ks > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks / 4) * C::HALF_BYTES + (ks % 4) * 32;
                    sm100::umma_ss(tmem + 128, sm100::sdesc_sw128(doa + off, 16, 1024), sm100::sdesc_sw128(va + off, 16, 1024),
                                   IDESC_S, ks > 0 ? 1u : 0u);
                }
                sm100::umma_commit(s_full);
                if (!sm100::mbar_wait(p_full, t & 1, abort_flag)) { ok = false; break; }
                sm100::tc_fence_after();
                if (!DPASS) {
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        sm100::umma_ts(tmem + 256, tmem + 0 + ks * 8, sm100::sdesc_sw128(ka + ks * 2048, C::HALF_BYTES, 1024),
                                       IDESC_DQ, (t > 0 || ks > 0) ? 1u : 0u);
                }
                sm100::umma_commit(release + st);
            }
            if (ok) sm100::umma_commit(o_full);
            sm100::umma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
        __syncwarp();
    } else if (warp >= BWD_ACT_WARP0) {
        const int r = 32 * (warp % 4) + lane;
        const int i = i0 + r;
        const uint32_t lane_base = (uint32_t)(32 * (warp % 4)) << 16;
        const float slope = a.slopes ? __ldg(a.slopes + h) : 0.f;
        float lse = 0.f, Dr = 0.f, dsum = 0.f;
        if (MODE == SWAT_MODE_SOFTMAX_ && i < a.N) {
            lse = a.lse[((size_t)b * a.H + h) * a.N + i];
            if (!DPASS) Dr = a.Dws[((size_t)b * a.H + h) * a.N + i];
        }
        bool ok = sm100::mbar_wait(q_ready, 0, abort_flag);   // (also orders the epilogue's base angles)
        for (int t = 0; ok && t < T; ++t) {
            ok = sm100::mbar_wait(s_full, t & 1, abort_flag);
            if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
            sm100::tc_fence_after();
            const int j0 = fwd_tile_j0(tr, t);
            const bool masked = !(j0 + 127 <= i0 && (i0 + 127 - j0 < a.window || j0 + 127 < a.n_sink));
            const int rd = i - j0;
            const RowMask mk = row_mask(rd, j0, a.window, a.n_sink);
            auto bias_of = [&](int c) { return slope * (float)(rd - c); };
            auto valid = [&](int c) { return col_valid(mk, c); };
            auto rowval = [&](int, float &l_, float &d_) { l_ = lse; d_ = Dr; };
            const uint32_t s_addr = tmem + lane_base, dp_addr = tmem + lane_base + 128;
            if (DPASS) {
                dsum += masked ? bwd_rowsum_tile<true>(s_addr, dp_addr, a.scale, lse, bias_of, valid)
                               : bwd_rowsum_tile<false>(s_addr, dp_addr, a.scale, lse, bias_of, valid);
            } else if (masked) {
                bwd_ds_tile<MODE, true, false>(s_addr, dp_addr, s_addr, 0u, a.scale, bias_of, valid, rowval);
            } else {
                bwd_ds_tile<MODE, false, false>(s_addr, dp_addr, s_addr, 0u, a.scale, bias_of, valid, rowval);
            }
            sm100::tmem_wait_st();
            sm100::tc_fence_before();
            sm100::mbar_arrive(p_full);
        }
        if (DPASS) {
            if (ok && i < a.N) a.Dws[((size_t)b * a.H + h) * a.N + i] = dsum;
        } else {
            if (ok) ok = sm100::mbar_wait(o_full, 0, abort_flag);
            if (!__any_sync(0xffffffffu, !ok)) {
                sm100::tc_fence_after();
                __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(a.dq) + (((size_t)b * a.N + i) * a.H + h) * D;
                unrotate_store_row<D>(tmem + lane_base + 256, r, sA0, sThf, a.use_rope, dst, i < a.N);
            }
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    if (warp == BWD_MMA_WARP) sm100::tmem_dealloc(tmem, 512);
}

// ===========================================================================
// dkdv kernel: one CTA per (b, kv head, 128-row key tile); for each query
// head of the group, the query tiles whose key set meets this key tile.
// smem A = K (rotated), B = V, C[] = Q (rotated), E[] = dO.
// ===========================================================================
__device__ __forceinline__ int bwd_q_last(int kt, int nQT, int window, int n_sink)
{
    if (kt == 0 && n_sink > 0) return nQT - 1;            // sink keys are seen by every later query
    const long long last = ((long long)kt * 128 + 126 + (long long)window) / 128;
    return (int)min((long long)nQT - 1, last);
}

template <int D, int MODE>
__global__ void __launch_bounds__(BWD_THREADS, 1)
swat_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const BwdArgs a)
{
    using C = BwdTcCfg<D>;
    constexpr int NST = C::NST;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sK = smem + C::OFF_A, *sV = smem + C::OFF_B, *sQ = smem + C::OFF_C, *sDO = smem + C::OFF_E;
    float2 *sRot = reinterpret_cast<float2 *>(smem + C::OFF_ROT);
    double *sTh = reinterpret_cast<double *>(smem + C::OFF_TH);
    float *sA0 = reinterpret_cast<float *>(smem + C::OFF_A0);
    float *sThf = reinterpret_cast<float *>(smem + C::OFF_THF);
    float *sRows = reinterpret_cast<float *>(smem + C::OFF_ROWS);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *k_full = bars, *k_ready = bars + 1;
    uint64_t *q_full = bars + 2, *q_ready = q_full + NST, *do_full = q_ready + NST, *release = do_full + NST;
    uint64_t *s_full = release + NST, *p_full = s_full + 1, *o_full = p_full + 1, *drain = o_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int kt = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int G = a.H / a.Hkv;
    const int j0 = kt * 128;
    const int nQT = (a.N + 127) / 128;
    const int q_first = kt, q_last = bwd_q_last(kt, nQT, a.window, a.n_sink);
    const int per_head = q_last - q_first + 1;
    const int T = G * per_head;                           // steps: (g, query tile)

    if (threadIdx.x == 0) {
        sm100::mbar_init(k_full, 1);
        sm100::mbar_init(k_ready, 128);
        for (int s = 0; s < NST; ++s) {
            sm100::mbar_init(q_full + s, 1);
            sm100::mbar_init(q_ready + s, 128);
            sm100::mbar_init(do_full + s, 1);
            sm100::mbar_init(release + s, 1);
        }
        sm100::mbar_init(s_full, 1);
        sm100::mbar_init(p_full, 128);
        sm100::mbar_init(o_full, 1);
        sm100::mbar_init(drain, 1);
        *abort_flag = 0;
        sm100::fence_mbar_init();
    }
    if (warp == BWD_MMA_WARP) {
        sm100::tmem_alloc(tmem_slot, 512);
        sm100::tmem_relinquish();
    }
    const bool is_prep = warp >= BWD_PREP_WARP0;
    const int ptid = threadIdx.x - 32 * BWD_PREP_WARP0;
    RotThread rot;
    if (is_prep && a.use_rope) {
        if (ptid < D / 2) {
            const double th = exp2(-2.0 * (double)ptid / (double)D * a.log2_base);
            sTh[ptid] = th;
            sThf[ptid] = (float)th;
            const double two_pi = 6.283185307179586476925286766559;
            const double x = (double)j0 * th;
            sA0[ptid] = (float)(x - rint(x / two_pi) * two_pi);
        }
        sm100::named_bar_sync(FWD_PREP_BAR, 128);
        constexpr int CPR = D / 8, RS = 128 / CPR;
        const int c = ptid % CPR, r0 = ptid / CPR;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const double th = sTh[4 * c + q];
            const float2 w0 = rope_cs((double)r0 * th), stp = rope_cs((double)RS * th);
            rot.w0c[q] = w0.x; rot.w0s[q] = w0.y; rot.stc[q] = stp.x; rot.sts[q] = stp.y;
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == BWD_TMA_WARP) {
        if (lane == 0) {
            int last_par[NST];
            for (int s = 0; s < NST; ++s) last_par[s] = -1;
            sm100::mbar_arrive_expect_tx(k_full, 2 * C::TILE_BYTES);
            for (int hh = 0; hh < D / 64; ++hh) {
                sm100::tma_load_4d(sK + hh * C::HALF_BYTES, &tm_k, k_full, hh * 64, kvh, j0, b);
                sm100::tma_load_4d(sV + hh * C::HALF_BYTES, &tm_v, k_full, hh * 64, kvh, j0, b);
            }
            for (int t = 0; t < T; ++t) {
                const int st = t % NST, n = t / NST;
                if (n > 0 && !sm100::mbar_wait(release + st, (n - 1) & 1, abort_flag)) break;
                const int g = t / per_head, qt = q_first + t % per_head, h = kvh * G + g;
                sm100::mbar_arrive_expect_tx(q_full + st, C::TILE_BYTES);
                for (int hh = 0; hh < D / 64; ++hh)
                    sm100::tma_load_4d(sQ + st * C::TILE_BYTES + hh * C::HALF_BYTES, &tm_q, q_full + st, hh * 64, h, qt * 128, b);
                sm100::mbar_arrive_expect_tx(do_full + st, C::TILE_BYTES);
                for (int hh = 0; hh < D / 64; ++hh)
                    sm100::tma_load_4d(sDO + st * C::TILE_BYTES + hh * C::HALF_BYTES, &tm_do, do_full + st, hh * 64, h, qt * 128, b);
                last_par[st] = n & 1;
            }
            mbar_wait_drain(k_full, 0);
            for (int s = 0; s < NST; ++s)
                if (last_par[s] >= 0) { mbar_wait_drain(q_full + s, last_par[s]); mbar_wait_drain(do_full + s, last_par[s]); }
        }
    } else if (is_prep) {
        int ebuf = 0;
        auto make_bases = [&](int pos0) {
            ebuf ^= 1;
            if (a.use_rope && ptid < D / 2) sRot[ebuf * (D / 2) + ptid] = rope_cs((double)pos0 * sTh[ptid]);
        };
        make_bases(j0);
        bool ok = sm100::mbar_wait(k_full, 0, abort_flag);
        if (!named_bar_or(FWD_PREP_BAR, 128, !ok || *abort_flag)) {
            if (a.use_rope) rope_rotate_tile<D>(sK, sRot + ebuf * (D / 2), rot, ptid);
            sm100::fence_proxy_async_smem();
            sm100::mbar_arrive(k_ready);
            for (int t = 0; t < T; ++t) {
                const int st = t % NST, n = t / NST;
                const int qt = q_first + t % per_head;
                make_bases(qt * 128);
                ok = sm100::mbar_wait(q_full + st, n & 1, abort_flag);
                if (named_bar_or(FWD_PREP_BAR, 128, !ok || *abort_flag)) break;
                if (a.use_rope) rope_rotate_tile<D>(sQ + st * C::TILE_BYTES, sRot + ebuf * (D / 2), rot, ptid);
                sm100::fence_proxy_async_smem();
                sm100::mbar_arrive(q_ready + st);
            }
        }
    } else if (warp == BWD_MMA_WARP) {
        if (lane == 0) {
            constexpr uint32_t IDESC_S = sm100::idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t IDESC_ACC = sm100::idesc_bf16_f32(128, D, 0, 1);
            const uint32_t ka = sm100::smem_u32(sK), va = sm100::smem_u32(sV);
            bool ok = sm100::mbar_wait(k_ready, 0, abort_flag);
            for (int t = 0; ok && t < T; ++t) {
                const int st = t % NST, n = t / NST;
                if (!sm100::mbar_wait(q_ready + st, n & 1, abort_flag) || !sm100::mbar_wait(do_full + st, n & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                sm100::tc_fence_after();
                const uint32_t qa = sm100::smem_u32(sQ + st * C::TILE_BYTES), doa = sm100::smem_u32(sDO + st * C::TILE_BYTES);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks / 4) * C::HALF_BYTES + (ks % 4) * 32;
                    sm100::umma_ss(tmem + 0, sm100::sdesc_sw128(ka + off, 16, 1024), sm100::sdesc_sw128(qa + off, 16, 1024),
                                   IDESC_S, ks > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks / 4) * C::HALF_BYTES + (ks % 4) * 32;
                    sm100::umma_ss(tmem + 128, sm100::sdesc_sw128(va + off, 16, 1024), sm100::sdesc_sw128(doa + off, 16, 1024),
                                   IDESC_S, ks > 0 ? 1u : 0u);
                }
                sm100::umma_commit(s_full);
                if (!sm100::mbar_wait(p_full, t & 1, abort_flag)) { ok = false; break; }
                sm100::tc_fence_after();
                // dV += P^T dO  (P^T over S columns 0..63),  dK' += dS^T Q'  (dS^T over dP columns 0..63)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    sm100::umma_ts(tmem + 256, tmem + 0 + ks * 8, sm100::sdesc_sw128(doa + ks * 2048, C::HALF_BYTES, 1024),
                                   IDESC_ACC, (t > 0 || ks > 0) ? 1u : 0u);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    sm100::umma_ts(tmem + 256 + D, tmem + 128 + ks * 8, sm100::sdesc_sw128(qa + ks * 2048, C::HALF_BYTES, 1024),
                                   IDESC_ACC, (t > 0 || ks > 0) ? 1u : 0u);
                sm100::umma_commit(release + st);
            }
            if (ok) sm100::umma_commit(o_full);
            sm100::umma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
        __syncwarp();
    } else if (warp >= BWD_ACT_WARP0) {
        const int r = 32 * (warp % 4) + lane;             // key row in the tile (= TMEM lane)
        const int j = j0 + r;
        const uint32_t lane_base = (uint32_t)(32 * (warp % 4)) << 16;
        const int atid = threadIdx.x - 32 * BWD_ACT_WARP0;   // 0..127
        bool ok = sm100::mbar_wait(k_ready, 0, abort_flag);
        for (int t = 0; ok && t < T; ++t) {
            const int g = t / per_head, qt = q_first + t % per_head, h = kvh * G + g;
            const int i0 = qt * 128;
            float *rows = sRows + (t & 1) * 256;          // lse / D of the 128 queries of this step
            if (MODE == SWAT_MODE_SOFTMAX_) {
                const int iq = i0 + atid;
                rows[atid] = iq < a.N ? a.lse[((size_t)b * a.H + h) * a.N + iq] : 0.f;
                rows[128 + atid] = iq < a.N ? a.Dws[((size_t)b * a.H + h) * a.N + iq] : 0.f;
                sm100::named_bar_sync(2, 128);
            }
            ok = sm100::mbar_wait(s_full, t & 1, abort_flag);
            if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
            sm100::tc_fence_after();
            const float slope = a.slopes ? __ldg(a.slopes + h) : 0.f;
            // column c is query i0 + c; valid iff 0 <= i - j < window, or j is a sink (j < n_sink, i >= j), and i < N
            const int lo = j - i0;
            const int hi = (j < a.n_sink) ? 127 : lo + a.window - 1;
            const int hi_n = min(hi, a.N - 1 - i0);
            const bool masked = __any_sync(0xffffffffu, !(lo <= 0 && hi_n >= 127));   // warp-uniform
            auto bias_of = [&](int c) { return slope * (float)(c - lo); };
            auto valid = [&](int c) { return (c >= lo) & (c <= hi_n); };
            auto rowval = [&](int c, float &l_, float &d_) {
                if (MODE == SWAT_MODE_SOFTMAX_) { l_ = rows[c]; d_ = rows[128 + c]; } else { l_ = 0.f; d_ = 0.f; }
            };
            const uint32_t s_addr = tmem + lane_base, dp_addr = tmem + lane_base + 128;
            // dS^T over the dP buffer, P^T over the S buffer
            if (masked) bwd_ds_tile<MODE, true, true>(s_addr, dp_addr, dp_addr, s_addr, a.scale, bias_of, valid, rowval);
            else bwd_ds_tile<MODE, false, true>(s_addr, dp_addr, dp_addr, s_addr, a.scale, bias_of, valid, rowval);
            sm100::tmem_wait_st();
            sm100::tc_fence_before();
            sm100::mbar_arrive(p_full);
        }
        if (ok) ok = sm100::mbar_wait(o_full, 0, abort_flag);
        if (!__any_sync(0xffffffffu, !ok)) {
            sm100::tc_fence_after();
            const size_t row = ((size_t)b * a.N + j) * a.Hkv + kvh;
            store_row_bf16_plain(tmem + lane_base + 256, D, reinterpret_cast<__nv_bfloat16 *>(a.dv) + row * D, j < a.N);
            unrotate_store_row<D>(tmem + lane_base + 256 + D, r, sA0, sThf, a.use_rope,
                                  reinterpret_cast<__nv_bfloat16 *>(a.dk) + row * D, j < a.N);
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    if (warp == BWD_MMA_WARP) sm100::tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// Host launch
// ---------------------------------------------------------------------------
template <int D, int MODE>
inline int launch_bwd_tc_t(const BwdArgs &a, cudaStream_t stream)
{
    using C = BwdTcCfg<D>;
    CUtensorMap tq, tk, tv, tdo;
    if (!make_tmap_bshd(&tq, a.q, a.B, a.N, a.H, D) || !make_tmap_bshd(&tk, a.k, a.B, a.N, a.Hkv, D) ||
        !make_tmap_bshd(&tv, a.v, a.B, a.N, a.Hkv, D) || !make_tmap_bshd(&tdo, a.dout, a.B, a.N, a.H, D))
        return -1;
    auto kq = swat_bwd_dq_tc_kernel<D, MODE, false>;
    auto kk = swat_bwd_dkdv_tc_kernel<D, MODE>;
    if (cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess) return -1;
    if (cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess) return -1;
    const int nQT = (a.N + 127) / 128;
    int n = 0;
    if (MODE == SWAT_MODE_SOFTMAX_) {   // D_i = sum_j p_ij dP_ij first (workspace), used by both kernels
        auto kd = swat_bwd_dq_tc_kernel<D, MODE, true>;
        if (cudaFuncSetAttribute(kd, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess) return -1;
        kd<<<dim3(nQT, a.H, a.B), BWD_THREADS, C::SMEM, stream>>>(tq, tk, tv, tdo, a, nullptr);
        ++n;
    }
    kq<<<dim3(nQT, a.H, a.B), BWD_THREADS, C::SMEM, stream>>>(tq, tk, tv, tdo, a, nullptr);
    kk<<<dim3(nQT, a.Hkv, a.B), BWD_THREADS, C::SMEM, stream>>>(tq, tk, tv, tdo, a);
    return n + 2;
}

inline size_t tc_bwd_extra_workspace(int B, int H, int Hkv, int N, int d)
{
    (void)B; (void)H; (void)Hkv; (void)N; (void)d;
    return 0;
}

inline int launch_bwd_tc(const BwdArgs &a, void *extra_ws, cudaStream_t stream)
{
    (void)extra_ws;
    if (a.d == 64)
        return a.mode == SWAT_MODE_SIGMOID_ ? launch_bwd_tc_t<64, SWAT_MODE_SIGMOID_>(a, stream)
                                            : launch_bwd_tc_t<64, SWAT_MODE_SOFTMAX_>(a, stream);
    if (a.d == 128)
        return a.mode == SWAT_MODE_SIGMOID_ ? launch_bwd_tc_t<128, SWAT_MODE_SIGMOID_>(a, stream)
                                            : launch_bwd_tc_t<128, SWAT_MODE_SOFTMAX_>(a, stream);
    return -1;
}

}  // namespace swat
