// decode_fast.cuh — bf16 decode attention launcher.
#pragma once
#include "decode.cuh"

namespace swat {

inline int launch_decode_attn_fast(const DecArgs &a, cudaStream_t stream)
{
    dim3 grid(a.nsplit, a.B * a.Hkv);
    swa_decode_attn_generic_kernel<__nv_bfloat16><<<grid, DEC_THREADS, 0, stream>>>(a);
    return 1;
}

}  // namespace swat
