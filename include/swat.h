/*
 * swat.h — C ABI of libswat.so: SWAT sliding-window attention on B200 (sm_100a).
 *
 * The operations are defined on these pages:
 *   [SWAT]  "SWAT: Sliding Window Attention Training" (explainer of
 *           arXiv 2502.18845): section "Balanced ALiBi" (the attention
 *           equation and the slope rule), section "Sigmoid: Dense Attention
 *           Without Suppression" (element-wise sigmoid), section "RoPE:
 *           Stabilizing Sigmoid Attention Training" and the Symbol Map.
 *   [SWA]   "Sliding Window Attention" glossary (Ultralytics): section "How
 *           the window grows with depth" (the causal window mask), the
 *           ring-buffer paragraph (slot = position mod w) and the "Attention
 *           sink" entry.
 *   [SINK]  "Sliding-window beats linear attention": SWA(w, s), softmax
 *           attention over the first s tokens plus the last w.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Tensors are row-major "BSHD": q/o [B, N, H, d], k/v [B, N, Hkv, d], d
 *   contiguous. Query head h reads KV head h / (H / Hkv).
 * - Key set of query i: { j <= i : i - j < window  or  j < n_sink }
 *   ([SWA] window mask: the token itself plus window-1 predecessors; [SINK]
 *   the first n_sink tokens, counted once if already inside the window).
 * - Score s_ij = (R_i q_i) . (R_j k_j) / sqrt(d) + slopes[h] * (i - j)
 *   ([SWAT] attention equation). R_p is RoPE at absolute position p:
 *   pair (2t, 2t+1) rotated by p * rope_base^(-2t/d); rope_base <= 0 turns
 *   RoPE off. slopes == NULL means all zero.
 * - mode SWAT_MODE_SIGMOID: o_i = sum_j sigmoid(s_ij) v_j, no normalisation
 *   ([SWAT] sigmoid section). mode SWAT_MODE_SOFTMAX: o_i = sum_j
 *   softmax_j(s_ij) v_j over the key set, and lse_i = log sum_j exp(s_ij)
 *   ([SINK]).
 * - dtype SWAT_BF16: bf16 tensors, fp32 accumulation (tensor cores, d must be
 *   64 or 128). dtype SWAT_F32: fp32 tensors on the exact fp32 CUDA-core
 *   path, any even d <= 128. slopes, lse and workspaces are always fp32.
 * - Every pointer is a DEVICE pointer unless stated; the caller owns all
 *   memory (the library allocates nothing); pointers must be 16-byte
 *   aligned. Calls are asynchronous on `stream` (a cudaStream_t passed as
 *   void*; NULL = legacy default stream) and never synchronise the host.
 * - Errors: the return value is a swat_status_t. Invalid arguments return
 *   SWAT_ERR_INVALID_ARG (or SWAT_ERR_UNSUPPORTED for a valid but
 *   unimplemented combination) before anything is launched; a failed launch
 *   returns SWAT_ERR_CUDA. Kernel-side waits are bounded: if one gives up,
 *   the kernel records SWAT_ERR_TIMEOUT in a device status word that
 *   swat_get_device_status() returns. No call aborts the process.
 */
#ifndef SWAT_H_
#define SWAT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SWAT_API __attribute__((visibility("default")))
#else
#define SWAT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SWAT_OK = 0,
    SWAT_ERR_INVALID_ARG = -1,
    SWAT_ERR_UNSUPPORTED = -2,
    SWAT_ERR_CUDA = -3,
    SWAT_ERR_TIMEOUT = -4,
    SWAT_ERR_SCRATCH_LIMIT = -5
} swat_status_t;

typedef enum { SWAT_MODE_SIGMOID = 0, SWAT_MODE_SOFTMAX = 1 } swat_mode_t;
typedef enum { SWAT_BF16 = 0, SWAT_F32 = 1 } swat_dtype_t;

/* Forward attention ([SWAT] "Balanced ALiBi" equation; [SINK] in softmax mode).
 *   q [B,N,H,d], k, v [B,N,Hkv,d]   inputs (raw, un-rotated Q and K)
 *   o [B,N,H,d]                      output, same dtype as the inputs
 *   lse [B,H,N] fp32                 softmax mode: required, receives
 *                                    log-sum-exp of each row; sigmoid mode:
 *                                    may be NULL (unused)
 *   B, N >= 1; H % Hkv == 0; window >= 1 (window >= N is full causal);
 *   0 <= n_sink <= 64; slopes [H] fp32 or NULL; rope_base <= 0 disables RoPE. */
SWAT_API int swat_attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                  int B, int H, int Hkv, int N, int d, int window, int n_sink, int mode,
                  const float *slopes, float rope_base, int dtype, void *stream);

/* Bytes of device workspace swat_attn_fwd_ws needs: RoPE-rotated copies of Q
 * and K (bf16 [B,N,H,d] and [B,N,Hkv,d], each padded to 256 bytes) for the
 * bf16 path; 0 for fp32 or invalid sizes. */
SWAT_API size_t swat_attn_fwd_workspace_bytes(int B, int H, int Hkv, int N, int d, int dtype);

/* swat_attn_fwd with a workspace: same operation, arguments, layouts and
 * results. With bf16 and RoPE on, Q and K are first rotated into the
 * workspace by a small element-wise kernel and the attention kernel loads
 * rotated tiles, instead of rotating each staged tile in shared memory.
 *   workspace: swat_attn_fwd_workspace_bytes() bytes of device memory,
 *              16-byte aligned (required for bf16; ignored for fp32); its
 *              contents on entry do not matter, and it may be reused as
 *              soon as the call's work on `stream` has finished.
 * Returns SWAT_ERR_INVALID_ARG for a missing or misaligned bf16 workspace;
 * otherwise as swat_attn_fwd. */
SWAT_API int swat_attn_fwd_ws(const void *q, const void *k, const void *v, void *o, float *lse, void *workspace,
                  int B, int H, int Hkv, int N, int d, int window, int n_sink, int mode,
                  const float *slopes, float rope_base, int dtype, void *stream);

/* Bytes of device workspace swat_attn_bwd needs for these sizes: the softmax
 * row terms D_i ([B,H,N] fp32) and, for bf16, RoPE-rotated copies of Q and K. */
SWAT_API size_t swat_attn_bwd_workspace_bytes(int B, int H, int Hkv, int N, int d, int dtype);

/* Backward of swat_attn_fwd (derived by calculus from the [SWAT] equation;
 * the pages train SWAT from scratch, so the gradient is part of the method).
 *   o, lse: the forward's outputs (softmax mode needs both; sigmoid mode
 *           reads neither and accepts NULL)
 *   dout [B,N,H,d]: gradient of the loss w.r.t. o
 *   dq [B,N,H,d], dk, dv [B,N,Hkv,d]: outputs (overwritten; for grouped KV
 *           heads the G query heads of a group are summed into one dk/dv)
 *   workspace: device buffer of swat_attn_bwd_workspace_bytes() bytes,
 *           16-byte aligned; its contents on entry do not matter.
 * No gradient is produced for slopes or rope_base. Other arguments as in
 * swat_attn_fwd. */
SWAT_API int swat_attn_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
                  const void *dout, void *dq, void *dk, void *dv, void *workspace,
                  int B, int H, int Hkv, int N, int d, int window, int n_sink, int mode,
                  const float *slopes, float rope_base, int dtype, void *stream);

/* swat_attn_bwd reusing the forward's rotated copies: qk_rot is the
 * workspace of a swat_attn_fwd_ws call on the same q and k with the same
 * B, H, Hkv, N, d and rope_base (bf16), and must still hold what that call
 * wrote; the backward then skips its own RoPE pass (a training step rotates
 * Q and K once). Same operation, arguments and results as swat_attn_bwd
 * otherwise; `workspace` is still required. SWAT_ERR_INVALID_ARG for a
 * missing or misaligned qk_rot (bf16 with RoPE on). */
SWAT_API int swat_attn_bwd_rotated(const void *q, const void *k, const void *v, const void *o, const float *lse,
                  const void *dout, void *dq, void *dk, void *dv, void *workspace, const void *qk_rot,
                  int B, int H, int Hkv, int N, int d, int window, int n_sink, int mode,
                  const float *slopes, float rope_base, int dtype, void *stream);

/* Ring-buffer KV cache ([SWA] ring-buffer paragraph, [SWA] "Attention sink"):
 *   k_cache, v_cache [B, Hkv, window, d]: slot s holds the token whose
 *           position p satisfies p mod window == s (the newest such p); keys
 *           are stored already RoPE-rotated at their absolute position.
 *   k_sink, v_sink [B, Hkv, n_sink, d]: positions 0 .. n_sink-1, rotated,
 *           never evicted (NULL when n_sink == 0).
 *
 * swa_cache_fill writes a prefill into the cache: k, v [B, n_tok, Hkv, d]
 * are the raw tokens at positions p0 .. p0+n_tok-1 (same p0 for every
 * sequence). Where several positions map to one slot, the latest wins, as if
 * they had been decoded one by one. Positions < n_sink also go to the sinks. */
SWAT_API int swa_cache_fill(const void *k, const void *v, void *k_cache, void *v_cache,
                   void *k_sink, void *v_sink, int B, int Hkv, int n_tok, int d,
                   int window, int n_sink, long long p0, float rope_base, int dtype,
                   void *stream);

/* One decode step over the ring cache.
 *   q [B,H,d], k_new, v_new [B,Hkv,d]: the new token of each sequence (raw)
 *   pos [B] int64 (device): its absolute position; the cache must hold the
 *           sequence's positions max(0, pos-window) .. pos-1 (and the sinks)
 *   o [B,H,d]: output
 *   workspace: swa_decode_workspace_bytes() bytes of device memory.
 * The new key is rotated at pos and written to slot pos mod window (and to
 * sink slot pos when pos < n_sink) BEFORE attention, so the token attends to
 * itself. Key set: the slots holding positions max(0, pos-window+1) .. pos,
 * plus the sinks j < min(n_sink, pos-window+1). The ALiBi distance of a slot
 * is pos minus the position it holds. */
SWAT_API int swa_decode_step(const void *q, const void *k_new, const void *v_new,
                    void *k_cache, void *v_cache, void *k_sink, void *v_sink,
                    const long long *pos, void *o, void *workspace,
                    int B, int H, int Hkv, int d, int window, int n_sink, int mode,
                    const float *slopes, float rope_base, int dtype, void *stream);

/* Bytes of device workspace swa_decode_step needs. */
SWAT_API size_t swa_decode_workspace_bytes(int B, int H, int Hkv, int d, int window);

/* Size of the library's own decode scratch buffer (16 MiB of device memory
 * per device, reserved when the library's device code is loaded). A decode
 * step fits iff swa_decode_workspace_bytes(B, H, Hkv, d, window) is at most
 * this: e.g. 64 sequences x 32 query heads, d 128, window 4096 need 2.1 MiB. */
#define SWA_DECODE_NOALLOC_SCRATCH_BYTES (16u << 20)

/* swa_decode_step without a workspace argument: the same decode step, same
 * kernels and same results, with the split partials kept in the library's
 * own static device buffer (SWA_DECODE_NOALLOC_SCRATCH_BYTES). It allocates
 * no device memory, ever. This entry point has no counterpart in the pages:
 * it exists for callers that cannot hand over a workspace, such as a C host
 * with no device allocator of its own, or a serving loop that must not call
 * cudaMalloc/cudaFree between steps because those calls synchronise the
 * device and stall its other streams.
 *
 * Arguments, layouts, ownership and the key set are those of swa_decode_step
 * (minus `workspace`).
 *
 * - The first call on each device does a one-time set-up: with that device
 *   current it looks up the buffer's device address. Make that first call
 *   before any stream capture begins. Call with the device that owns the
 *   buffers and `stream` current.
 * - Nothing in the buffer has to start at zero: each step writes every
 *   partial before it reads it.
 * - There is ONE buffer per device: two calls whose work can overlap on the
 *   device (different streams without ordering between them, or concurrent
 *   host threads) race on it and corrupt each other's results. Order such
 *   calls on one stream or with events.
 * - Returns SWAT_ERR_SCRATCH_LIMIT, before any launch, when the step needs
 *   more than SWA_DECODE_NOALLOC_SCRATCH_BYTES (use swa_decode_step with a
 *   workspace for such shapes); SWAT_ERR_CUDA if the set-up lookup fails;
 *   otherwise whatever swa_decode_step returns. */
SWAT_API int swa_decode_step_noalloc(const void *q, const void *k_new, const void *v_new,
                    void *k_cache, void *v_cache, void *k_sink, void *v_sink,
                    const long long *pos, void *o,
                    int B, int H, int Hkv, int d, int window, int n_sink, int mode,
                    const float *slopes, float rope_base, int dtype, void *stream);

/* Human-readable name of a status code (static string, never NULL). */
SWAT_API const char *swat_status_string(int status);

/* Reads and clears the device status word of the current device: SWAT_OK;
 * SWAT_ERR_TIMEOUT if a kernel gave up on a bounded wait since the last call;
 * SWAT_ERR_INVALID_ARG if a kernel rejected a device-resident argument (a
 * negative decode position: that sequence's step is skipped). Synchronises
 * `stream`. Returns SWAT_ERR_CUDA if the read fails. */
SWAT_API int swat_get_device_status(void *stream);

/* Failure-path check (no counterpart in the pages): launches one kernel
 * whose thread waits for an mbarrier phase that nothing completes, bounded
 * by limit_ns of device time, exactly as the attention kernels bound their
 * waits. It then records SWAT_ERR_TIMEOUT in the device status word and
 * returns; the context stays usable. Read the result with
 * swat_get_device_status(). limit_ns in [1e3, 2e9], else SWAT_ERR_INVALID_ARG
 * before any launch. */
SWAT_API int swat_check_wait_timeout(long long limit_ns, void *stream);

/* Number of kernel launches the library has issued in this process (host
 * counter; lets a caller count device work done through this ABI). */
SWAT_API long long swat_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SWAT_H_ */
