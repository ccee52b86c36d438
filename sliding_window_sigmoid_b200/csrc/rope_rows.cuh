// rope_rows.cuh — RoPE-rotated copies of Q / K rows ("SWAT" page, RoPE
// section; RoFormer pairs (2t, 2t+1), theta_t = base^(-2t/d)).
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace swat {

// ===========================================================================
// RoPE of Q or K rows into a copy (workspace), once per call: the tensor-core
// kernels then load rotated tiles directly. x, y: [B, N, Hx, D] bf16. CTA =
// 128 positions of one (b, head); the angle of pair t at position n0 + r is
// A_t + r theta_t, A_t = n0 theta_t reduced mod 2 pi in fp64, the sum reduced
// again in fp32 before __sincosf (|error| ~ 1e-6 rad).
// ===========================================================================
template <int D>
__global__ void __launch_bounds__(256)
swat_rope_rows_kernel(const __nv_bfloat16 *__restrict__ x, __nv_bfloat16 *__restrict__ y, int N, int Hx,
                      double log2_base)
{
    __shared__ float sA[D / 2], sT[D / 2];
    const int n0 = blockIdx.x * 128, hx = blockIdx.y, b = blockIdx.z;
    if (threadIdx.x < D / 2) {
        const double th = exp2(-2.0 * (double)threadIdx.x / (double)D * log2_base);
        const double two_pi = 6.283185307179586476925286766559;
        const double an = (double)n0 * th;
        sA[threadIdx.x] = (float)(an - rint(an / two_pi) * two_pi);
        sT[threadIdx.x] = (float)th;
    }
    __syncthreads();
    const float two_pi = 6.2831853071795865f, inv_two_pi = 0.15915494309189534f;
    constexpr int CH = D / 8;                      // 16-byte chunks per row (4 pairs each)
    for (int idx = threadIdx.x; idx < 128 * CH; idx += blockDim.x) {
        const int r = idx / CH, c = idx % CH, n = n0 + r;
        if (n >= N) break;
        const size_t off = (((size_t)b * N + n) * Hx + hx) * D + 8 * c;
        const uint4 in = *reinterpret_cast<const uint4 *>(x + off);
        const uint32_t w[4] = {in.x, in.y, in.z, in.w};
        uint32_t o[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const int t = 4 * c + p;
            float ang = fmaf((float)r, sT[t], sA[t]);
            ang = fmaf(-rintf(ang * inv_two_pi), two_pi, ang);
            float sn, cs;
            __sincosf(ang, &sn, &cs);
            const float x0 = sm100::bf16lo(w[p]), x1 = sm100::bf16hi(w[p]);
            o[p] = sm100::pack_bf16x2(x0 * cs - x1 * sn, x0 * sn + x1 * cs);
        }
        *reinterpret_cast<uint4 *>(y + off) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Bytes of the rotated copies of Q [B,N,H,d] and K [B,N,Hkv,d] (bf16).
inline size_t rope_copies_bytes(int B, int H, int Hkv, int N, int d)
{
    return align256((size_t)B * N * H * d * 2) + align256((size_t)B * N * Hkv * d * 2);
}

// Writes R q and R k into ws (layout as rope_copies_bytes); returns launches.
template <int D>
inline int launch_rope_copies(const void *q, const void *k, void *ws, int B, int H, int Hkv, int N, double log2_base,
                              cudaStream_t stream, const void **qr, const void **kr)
{
    __nv_bfloat16 *wq = reinterpret_cast<__nv_bfloat16 *>(ws);
    __nv_bfloat16 *wk = reinterpret_cast<__nv_bfloat16 *>(reinterpret_cast<char *>(ws) +
                                                           align256((size_t)B * N * H * D * 2));
    const unsigned nqt = (unsigned)((N + 127) / 128);
    swat_rope_rows_kernel<D><<<dim3(nqt, H, B), 256, 0, stream>>>(reinterpret_cast<const __nv_bfloat16 *>(q), wq, N, H,
                                                                   log2_base);
    swat_rope_rows_kernel<D><<<dim3(nqt, Hkv, B), 256, 0, stream>>>(reinterpret_cast<const __nv_bfloat16 *>(k), wk, N,
                                                                     Hkv, log2_base);
    *qr = wq;
    *kr = wk;
    return 2;
}

}  // namespace swat
