// api.cu — the C ABI of libswat.so (declared in include/swat.h).
//
// Host side only: argument validation (before any launch), kernel selection,
// launch on the caller's stream, error mapping. Every call is asynchronous.
#include <math.h>
#include <stdio.h>
#include <atomic>
#include <mutex>

#include "swat.h"
#include "common.cuh"
#include "fwd_simt.cuh"
#include "bwd_simt.cuh"
#include "decode.cuh"
#include "fwd_tc.cuh"
#include "bwd_tc.cuh"
#include "decode_fast.cuh"

namespace {

std::atomic<long long> g_launches{0};

inline cudaStream_t S(void *s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int after_launch(int n_launched)
{
    g_launches += n_launched;
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SWAT_OK : SWAT_ERR_CUDA;
}

// Common shape checks of fwd/bwd.
int check_attn_shapes(int B, int H, int Hkv, int N, int d, int window, int n_sink, int mode,
                      int dtype)
{
    if (B < 1 || N < 1 || H < 1 || Hkv < 1 || H % Hkv != 0) return SWAT_ERR_INVALID_ARG;
    if (B > 65535 || H > 65535) return SWAT_ERR_INVALID_ARG;   // grid y/z limits
    if (window < 1 || n_sink < 0 || n_sink > 64) return SWAT_ERR_INVALID_ARG;
    if (mode != SWAT_MODE_SIGMOID && mode != SWAT_MODE_SOFTMAX) return SWAT_ERR_INVALID_ARG;
    if (dtype != SWAT_BF16 && dtype != SWAT_F32) return SWAT_ERR_INVALID_ARG;
    if (d < 2 || d % 2 != 0 || d > 128) return SWAT_ERR_INVALID_ARG;
    if (dtype == SWAT_BF16 && d != 64 && d != 128) return SWAT_ERR_UNSUPPORTED;
    if ((long long)B * N * H * d > (1LL << 40)) return SWAT_ERR_INVALID_ARG;
    return SWAT_OK;
}

inline double log2_base_of(float rope_base) { return rope_base > 0.f ? log2((double)rope_base) : 0.0; }

}  // namespace

extern "C" {

const char *swat_status_string(int status)
{
    switch (status) {
        case SWAT_OK: return "SWAT_OK";
        case SWAT_ERR_INVALID_ARG: return "SWAT_ERR_INVALID_ARG";
        case SWAT_ERR_UNSUPPORTED: return "SWAT_ERR_UNSUPPORTED";
        case SWAT_ERR_CUDA: return "SWAT_ERR_CUDA";
        case SWAT_ERR_TIMEOUT: return "SWAT_ERR_TIMEOUT";
        case SWAT_ERR_SCRATCH_LIMIT: return "SWAT_ERR_SCRATCH_LIMIT";
        default: return "SWAT_ERR_UNKNOWN";
    }
}

long long swat_launch_count(void) { return g_launches.load(); }

int swat_get_device_status(void *stream)
{
    int h = 0, zero = 0;
    if (cudaMemcpyFromSymbolAsync(&h, swat::g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, S(stream)) != cudaSuccess)
        return SWAT_ERR_CUDA;
    if (cudaMemcpyToSymbolAsync(swat::g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, S(stream)) != cudaSuccess)
        return SWAT_ERR_CUDA;
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return SWAT_ERR_CUDA;
    return h;
}

}  // extern "C"

namespace {
// One thread waits, bounded by limit_ns of %globaltimer, for the first phase
// of an mbarrier that nothing arrives on: the same bounded-wait path every
// tensor-core kernel takes, ending in SWAT_ERR_TIMEOUT in the status word.
__global__ void swat_wait_timeout_kernel(long long limit_ns)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        swat::sm100::mbar_init(&bar, 1);
        swat::sm100::fence_mbar_init();
        const uint64_t t0 = swat::sm100::globaltimer();
        while (!swat::sm100::mbar_try_wait(&bar, 0)) {
            if (swat::sm100::globaltimer() - t0 > (uint64_t)limit_ns) {
                swat::record_status(SWAT_ERR_TIMEOUT);
                break;
            }
        }
    }
}
}  // namespace

extern "C" int swat_check_wait_timeout(long long limit_ns, void *stream)
{
    if (limit_ns < 1000 || limit_ns > 2000000000LL) return SWAT_ERR_INVALID_ARG;
    swat_wait_timeout_kernel<<<1, 32, 0, S(stream)>>>(limit_ns);
    return after_launch(1);
}

namespace {
// The forward with an optional workspace for RoPE-rotated copies of Q and K.
int attn_fwd_impl(const void *q, const void *k, const void *v, void *o, float *lse, void *workspace,
                  int B, int H, int Hkv, int N, int d, int window, int n_sink, int mode,
                  const float *slopes, float rope_base, int dtype, void *stream)
{
    int st = check_attn_shapes(B, H, Hkv, N, d, window, n_sink, mode, dtype);
    if (st != SWAT_OK) return st;
    if (!q || !k || !v || !o) return SWAT_ERR_INVALID_ARG;
    if (mode == SWAT_MODE_SOFTMAX && !lse) return SWAT_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SWAT_ERR_INVALID_ARG;
    if ((lse && !aligned16(lse)) || (slopes && (reinterpret_cast<uintptr_t>(slopes) & 3u)))
        return SWAT_ERR_INVALID_ARG;

    if (window > N) window = N;   // a window of N already covers every earlier key
    if (dtype == SWAT_BF16) {
        swat::TcFwdArgs a{};
        a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse; a.slopes = slopes;
        a.B = B; a.H = H; a.Hkv = Hkv; a.N = N; a.d = d; a.window = window; a.n_sink = n_sink;
        a.mode = mode; a.use_rope = rope_base > 0.f; a.log2_base = log2_base_of(rope_base);
        a.scale = (float)(1.0 / sqrt((double)d));
        int n = swat::launch_fwd_tc(a, workspace, S(stream));
        if (n < 0) return SWAT_ERR_CUDA;
        return after_launch(n);
    }
    swat::FwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse; a.slopes = slopes;
    a.B = B; a.H = H; a.Hkv = Hkv; a.N = N; a.d = d; a.window = window; a.n_sink = n_sink;
    a.mode = mode; a.use_rope = rope_base > 0.f; a.log2_base = log2_base_of(rope_base);
    a.scale = (float)(1.0 / sqrt((double)d));
    dim3 grid((N + swat::SIMT_BQ - 1) / swat::SIMT_BQ, H, B);
    size_t smem = swat::simt_fwd_smem_bytes();
    cudaFuncSetAttribute(swat::swat_fwd_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    swat::swat_fwd_simt_kernel<float><<<grid, swat::SIMT_THREADS, smem, S(stream)>>>(a);
    return after_launch(1);
}
}  // namespace

extern "C" {

int swat_attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                  int B, int H, int Hkv, int N, int d, int window, int n_sink, int mode,
                  const float *slopes, float rope_base, int dtype, void *stream)
{
    return attn_fwd_impl(q, k, v, o, lse, nullptr, B, H, Hkv, N, d, window, n_sink, mode, slopes, rope_base,
                         dtype, stream);
}

size_t swat_attn_fwd_workspace_bytes(int B, int H, int Hkv, int N, int d, int dtype)
{
    if (B < 1 || H < 1 || Hkv < 1 || N < 1 || d < 2 || dtype != SWAT_BF16) return 0;
    return swat::rope_copies_bytes(B, H, Hkv, N, d);
}

int swat_attn_fwd_ws(const void *q, const void *k, const void *v, void *o, float *lse, void *workspace,
                     int B, int H, int Hkv, int N, int d, int window, int n_sink, int mode,
                     const float *slopes, float rope_base, int dtype, void *stream)
{
    if (dtype == SWAT_BF16 && (!workspace || !aligned16(workspace))) return SWAT_ERR_INVALID_ARG;
    return attn_fwd_impl(q, k, v, o, lse, dtype == SWAT_BF16 ? workspace : nullptr, B, H, Hkv, N, d, window,
                         n_sink, mode, slopes, rope_base, dtype, stream);
}

size_t swat_attn_bwd_workspace_bytes(int B, int H, int Hkv, int N, int d, int dtype)
{
    (void)Hkv;
    if (B < 1 || H < 1 || N < 1 || d < 2) return 0;
    size_t D = (size_t)B * H * N * sizeof(float);
    D = (D + 255) & ~(size_t)255;
    size_t extra = 0;
    if (dtype == SWAT_BF16) extra = swat::tc_bwd_extra_workspace(B, H, Hkv, N, d);
    return D + extra;
}

}  // extern "C"

namespace {
int attn_bwd_impl(const void *q, const void *k, const void *v, const void *o, const float *lse,
                  const void *dout, void *dq, void *dk, void *dv, void *workspace, const void *qk_rot,
                  int B, int H, int Hkv, int N, int d, int window, int n_sink, int mode,
                  const float *slopes, float rope_base, int dtype, void *stream)
{
    int st = check_attn_shapes(B, H, Hkv, N, d, window, n_sink, mode, dtype);
    if (st != SWAT_OK) return st;
    if (!q || !k || !v || !dout || !dq || !dk || !dv || !workspace) return SWAT_ERR_INVALID_ARG;
    if (mode == SWAT_MODE_SOFTMAX && (!o || !lse)) return SWAT_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, dout, dq, dk, dv, workspace};
    for (const void *p : ptrs) if (!aligned16(p)) return SWAT_ERR_INVALID_ARG;
    if (o && !aligned16(o)) return SWAT_ERR_INVALID_ARG;

    if (window > N) window = N;
    swat::BwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.o = o; a.dout = dout; a.lse = lse;
    a.dq = dq; a.dk = dk; a.dv = dv; a.Dws = (float *)workspace; a.slopes = slopes;
    a.B = B; a.H = H; a.Hkv = Hkv; a.N = N; a.d = d; a.window = window; a.n_sink = n_sink;
    a.mode = mode; a.use_rope = rope_base > 0.f; a.log2_base = log2_base_of(rope_base);
    a.scale = (float)(1.0 / sqrt((double)d));
    int n = 0;
    if (mode == SWAT_MODE_SOFTMAX && dtype == SWAT_F32) {   // (the bf16 path computes D_i itself)
        long long rows = (long long)B * N * H;
        int threads = 256, rpb = threads / 32;
        swat::swat_bwd_dot_do_o_kernel<float><<<(unsigned)((rows + rpb - 1) / rpb), threads, 0, S(stream)>>>(a);
        ++n;
    }
    if (dtype == SWAT_BF16) {
        size_t D = ((size_t)B * H * N * sizeof(float) + 255) & ~(size_t)255;
        int m = swat::launch_bwd_tc(a, (char *)workspace + D, qk_rot, S(stream));
        if (m < 0) return SWAT_ERR_CUDA;
        return after_launch(n + m);
    }
    size_t smem_q = swat::simt_bwd_dq_smem_bytes(), smem_k = swat::simt_bwd_dkdv_smem_bytes();
    cudaFuncSetAttribute(swat::swat_bwd_dq_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_q);
    cudaFuncSetAttribute(swat::swat_bwd_dkdv_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_k);
    dim3 gq((N + swat::SIMT_BQ - 1) / swat::SIMT_BQ, H, B);
    dim3 gk((N + swat::SIMT_BK - 1) / swat::SIMT_BK, Hkv, B);
    swat::swat_bwd_dq_simt_kernel<float><<<gq, swat::SIMT_THREADS, smem_q, S(stream)>>>(a);
    swat::swat_bwd_dkdv_simt_kernel<float><<<gk, swat::SIMT_THREADS, smem_k, S(stream)>>>(a);
    return after_launch(n + 2);
}
}  // namespace

extern "C" {

int swat_attn_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
                  const void *dout, void *dq, void *dk, void *dv, void *workspace,
                  int B, int H, int Hkv, int N, int d, int window, int n_sink, int mode,
                  const float *slopes, float rope_base, int dtype, void *stream)
{
    return attn_bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, workspace, nullptr, B, H, Hkv, N, d, window, n_sink,
                         mode, slopes, rope_base, dtype, stream);
}

int swat_attn_bwd_rotated(const void *q, const void *k, const void *v, const void *o, const float *lse,
                          const void *dout, void *dq, void *dk, void *dv, void *workspace, const void *qk_rot,
                          int B, int H, int Hkv, int N, int d, int window, int n_sink, int mode,
                          const float *slopes, float rope_base, int dtype, void *stream)
{
    if (dtype == SWAT_BF16 && rope_base > 0.f && (!qk_rot || !aligned16(qk_rot))) return SWAT_ERR_INVALID_ARG;
    return attn_bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, workspace, dtype == SWAT_BF16 ? qk_rot : nullptr,
                         B, H, Hkv, N, d, window, n_sink, mode, slopes, rope_base, dtype, stream);
}

int swa_cache_fill(const void *k, const void *v, void *k_cache, void *v_cache,
                   void *k_sink, void *v_sink, int B, int Hkv, int n_tok, int d,
                   int window, int n_sink, long long p0, float rope_base, int dtype,
                   void *stream)
{
    if (B < 1 || Hkv < 1 || n_tok < 0 || window < 1 || n_sink < 0 || n_sink > 64 || p0 < 0)
        return SWAT_ERR_INVALID_ARG;
    if (d < 2 || d % 2 || d > 128) return SWAT_ERR_INVALID_ARG;
    if (dtype != SWAT_BF16 && dtype != SWAT_F32) return SWAT_ERR_INVALID_ARG;
    if (!k || !v || !k_cache || !v_cache) return SWAT_ERR_INVALID_ARG;
    if (n_sink > 0 && (!k_sink || !v_sink)) return SWAT_ERR_INVALID_ARG;
    if (n_tok == 0) return SWAT_OK;
    if (n_tok > 65535 * 64) return SWAT_ERR_INVALID_ARG;
    swat::FillArgs a{};
    a.k = k; a.v = v; a.k_cache = k_cache; a.v_cache = v_cache; a.k_sink = k_sink; a.v_sink = v_sink;
    a.B = B; a.Hkv = Hkv; a.n_tok = n_tok; a.d = d; a.window = window; a.n_sink = n_sink; a.p0 = p0;
    a.use_rope = rope_base > 0.f; a.log2_base = log2_base_of(rope_base);
    if (B > 65535) return SWAT_ERR_INVALID_ARG;
    dim3 grid(n_tok, B);
    if (dtype == SWAT_BF16)
        swat::swa_cache_fill_kernel<__nv_bfloat16><<<grid, 128, 0, S(stream)>>>(a);
    else
        swat::swa_cache_fill_kernel<float><<<grid, 128, 0, S(stream)>>>(a);
    return after_launch(1);
}

size_t swa_decode_workspace_bytes(int B, int H, int Hkv, int d, int window)
{
    (void)Hkv;
    if (B < 1 || H < 1 || d < 2 || window < 1) return 0;
    size_t ns = (size_t)swat::decode_nsplit(window);
    size_t rows = (size_t)B * H;
    size_t po = rows * ns * d * sizeof(float);
    po = (po + 255) & ~(size_t)255;
    size_t pm = (rows * ns * sizeof(float) + 255) & ~(size_t)255;
    return po + 2 * pm;
}

int swa_decode_step(const void *q, const void *k_new, const void *v_new,
                    void *k_cache, void *v_cache, void *k_sink, void *v_sink,
                    const long long *pos, void *o, void *workspace,
                    int B, int H, int Hkv, int d, int window, int n_sink, int mode,
                    const float *slopes, float rope_base, int dtype, void *stream)
{
    int st = check_attn_shapes(B, H, Hkv, 1, d, window, n_sink, mode, dtype);
    if (st != SWAT_OK) return st;
    if (H / Hkv > swat::DEC_MAX_G) return SWAT_ERR_UNSUPPORTED;
    if (!q || !k_new || !v_new || !k_cache || !v_cache || !pos || !o || !workspace)
        return SWAT_ERR_INVALID_ARG;
    if (n_sink > 0 && (!k_sink || !v_sink)) return SWAT_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k_new, v_new, k_cache, v_cache, o, workspace};
    for (const void *p : ptrs) if (!aligned16(p)) return SWAT_ERR_INVALID_ARG;
    if (B > 65535) return SWAT_ERR_INVALID_ARG;

    swat::DecArgs a{};
    a.q = q; a.k_new = k_new; a.v_new = v_new; a.k_cache = k_cache; a.v_cache = v_cache;
    a.k_sink = k_sink; a.v_sink = v_sink; a.pos = pos; a.o = o; a.slopes = slopes;
    a.B = B; a.H = H; a.Hkv = Hkv; a.d = d; a.window = window; a.n_sink = n_sink; a.mode = mode;
    a.nsplit = swat::decode_nsplit(window);
    a.use_rope = rope_base > 0.f; a.log2_base = log2_base_of(rope_base);
    a.scale = (float)(1.0 / sqrt((double)d));
    size_t rows = (size_t)B * H, ns = (size_t)a.nsplit;
    size_t po = (rows * ns * d * sizeof(float) + 255) & ~(size_t)255;
    size_t pm = (rows * ns * sizeof(float) + 255) & ~(size_t)255;
    a.part_o = (float *)workspace;
    a.part_m = (float *)((char *)workspace + po);
    a.part_l = (float *)((char *)workspace + po + pm);
    int threads_c = ((d + 31) / 32) * 32;
    if (dtype == SWAT_BF16) {
        int m = swat::launch_decode_attn_fast(a, S(stream));
        if (m < 0) return SWAT_ERR_CUDA;
        swat::swa_decode_combine_kernel<__nv_bfloat16><<<(unsigned)rows, threads_c, 0, S(stream)>>>(a);
        return after_launch(1 + m);
    }
    swat::swa_decode_write_kernel<float><<<B, 128, 0, S(stream)>>>(a);
    dim3 grid(a.nsplit, B * Hkv);
    swat::swa_decode_attn_generic_kernel<float><<<grid, swat::DEC_THREADS, 0, S(stream)>>>(a);
    swat::swa_decode_combine_kernel<float><<<(unsigned)rows, threads_c, 0, S(stream)>>>(a);
    return after_launch(3);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode step with library-owned scratch (no workspace argument, no allocation)
//
// The split partials that swa_decode_step keeps in the caller's workspace live
// here in one file-scope device buffer instead. Its device address is looked
// up once per device (cudaGetSymbolAddress with that device current) and then
// reused; the decode kernels themselves are the ones swa_decode_step runs.
// Every partial is written by the attention pass before the combine pass reads
// it, so the buffer's contents never need to start at zero.
static __device__ __align__(256) unsigned char g_decode_scratch[SWA_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxScratchDevices = 64;
std::atomic<void *> g_decode_scratch_ptr[kMaxScratchDevices];
std::mutex g_decode_scratch_mu;

// Device address of g_decode_scratch on the current device (set-up on first use).
int decode_scratch_current_device(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return SWAT_ERR_CUDA; }
    if (dev < 0 || dev >= kMaxScratchDevices) return SWAT_ERR_UNSUPPORTED;
    void *p = g_decode_scratch_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_decode_scratch_mu);
        p = g_decode_scratch_ptr[dev].load(std::memory_order_relaxed);
        if (!p) {
            cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
            if (e != cudaSuccess || !p) { cudaGetLastError(); return SWAT_ERR_CUDA; }
            g_decode_scratch_ptr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return SWAT_OK;
}

}  // namespace

extern "C" int swa_decode_step_noalloc(const void *q, const void *k_new, const void *v_new,
                                       void *k_cache, void *v_cache, void *k_sink, void *v_sink,
                                       const long long *pos, void *o,
                                       int B, int H, int Hkv, int d, int window, int n_sink,
                                       int mode, const float *slopes, float rope_base, int dtype,
                                       void *stream)
{
    int st = check_attn_shapes(B, H, Hkv, 1, d, window, n_sink, mode, dtype);
    if (st != SWAT_OK) return st;
    const size_t need = swa_decode_workspace_bytes(B, H, Hkv, d, window);
    if (need == 0) return SWAT_ERR_INVALID_ARG;
    if (need > (size_t)SWA_DECODE_NOALLOC_SCRATCH_BYTES) return SWAT_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    st = decode_scratch_current_device(&scratch);
    if (st != SWAT_OK) return st;
    return swa_decode_step(q, k_new, v_new, k_cache, v_cache, k_sink, v_sink, pos, o, scratch,
                           B, H, Hkv, d, window, n_sink, mode, slopes, rope_base, dtype, stream);
}
