// fwd_tc.cuh — bf16 forward / backward launchers.
#pragma once
#include "common.cuh"
#include "fwd_simt.cuh"
#include "bwd_simt.cuh"

namespace swat {

using TcFwdArgs = FwdArgs;

// Returns the number of kernels launched, or -1 on a launch-configuration error.
inline int launch_fwd_tc(const TcFwdArgs &a, cudaStream_t stream)
{
    if (a.H > 65535 || a.B > 65535) return -1;
    dim3 grid((a.N + SIMT_BQ - 1) / SIMT_BQ, a.H, a.B);
    size_t smem = simt_fwd_smem_bytes();
    cudaFuncSetAttribute(swat_fwd_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    swat_fwd_simt_kernel<__nv_bfloat16><<<grid, SIMT_THREADS, smem, stream>>>(a);
    return 1;
}

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
