// common.cuh — device helpers shared by the libswat kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#define SWAT_MODE_SIGMOID_ 0
#define SWAT_MODE_SOFTMAX_ 1

namespace swat {

// Device status word (SWAT_ERR_TIMEOUT is recorded here by a kernel that gave
// up on a bounded wait). One per device; read and cleared by the host API.
__device__ int g_status;

__device__ __forceinline__ void record_status(int code) { atomicCAS(&g_status, 0, code); }

// ---------------------------------------------------------------------------
// I/O element conversions
// ---------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// ---------------------------------------------------------------------------
// RoPE ("SWAT" page, RoPE section; RoFormer convention): pair (2t, 2t+1) at
// absolute position p is rotated by p * theta_t, theta_t = base^(-2t/d).
// The angle is formed and reduced modulo 2*pi in fp64, so positions up to
// 2^16 and beyond keep full fp32 accuracy in cos/sin.
// ---------------------------------------------------------------------------
__device__ __forceinline__ double rope_theta(int t, int d, double log2_base)
{
    return exp2(-2.0 * (double)t / (double)d * log2_base);
}

__device__ __forceinline__ void rope_cos_sin(long long pos, double theta, float &c, float &s)
{
    const double two_pi = 6.283185307179586476925286766559;
    const double inv_two_pi = 0.15915494309189533576888376337251;
    double a = (double)pos * theta;
    double r = a - rint(a * inv_two_pi) * two_pi;   // |r| <= pi (up to rounding)
    sincosf((float)r, &s, &c);
}

// Rotate one pair in fp32.
__device__ __forceinline__ void rope_pair(float x0, float x1, float c, float s, float &y0, float &y1)
{
    y0 = x0 * c - x1 * s;
    y1 = x0 * s + x1 * c;
}

// Inverse (transposed) rotation of one pair.
__device__ __forceinline__ void rope_pair_inv(float x0, float x1, float c, float s, float &y0, float &y1)
{
    y0 = x0 * c + x1 * s;
    y1 = -x0 * s + x1 * c;
}

// Key-set predicate: j <= i and (i - j < window or j < n_sink).
__device__ __forceinline__ bool in_keyset(long long i, long long j, int window, int n_sink)
{
    return j <= i && (i - j < (long long)window || j < (long long)n_sink);
}

__device__ __forceinline__ float sigmoid_exact(float x) { return 1.0f / (1.0f + expf(-x)); }

}  // namespace swat
