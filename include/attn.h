/*
 * attn.h -- C ABI of the B200 (sm_100a) exact-attention library.
 *
 * The operation (per head, Q, K, V each T x d_h):
 *     O = softmax(mask(scale * Q K^T)) V,   lse_i = log sum_j exp(scale * q_i . k_j)
 * with the causal mask "key j visible to query i iff j <= i".
 * Defined in "Why Attention Is Difficult to Optimize" (section "The Attention
 * Computation Flow": Q, K, V of shape T x d_h, scores divided by sqrt(d_h),
 * causal mask to -inf, row softmax, O = P V) and in "Attention Mechanism:
 * Computation & Memory Patterns" (section 1, the three steps S = QK^T,
 * P = softmax(S / sqrt(d_k)), O = PV).  The fused entry point is the
 * IO-aware single-kernel form of section 3 of the latter page ("Tiling" +
 * "Online Softmax"); the unfused entry point is the materialised three-kernel
 * form of "Storing and Rereading Large Intermediate Matrices".
 *
 * Conventions shared by every entry point:
 *  - Layout: q, k, v, o are bf16, [B, H, T, d_h] contiguous (row = token,
 *    d_h values contiguous); lse is fp32, [B, H, T].  Head (b, h) starts at
 *    element ((b * H + h) * T) * d_h.
 *  - Pointers are device pointers unless the name says host.  Tensor and
 *    workspace pointers must be 16-byte aligned (tensor-memory-accelerator
 *    rule); lse pointers need only float (4-byte) alignment, since every
 *    kernel reads and writes lse one value at a time.  The caller owns all
 *    memory; no entry point allocates device memory.
 *  - Per-device set-up (kernel attributes, the library's own streams and
 *    events, the static workspace's address) is done on the first call in a
 *    CUDA context and redone when the device's current context changes (for
 *    example after cudaDeviceReset), so no handle outlives its context.
 *  - d_h must be 64 or 128.  B, H, T >= 1.  B * H * T must fit in 2^31 - 1
 *    and T in 2^31 / 256.  scale must be finite and > 0 (configs use
 *    1 / sqrt(d_h)).  causal is 0 or 1 (top-left aligned, Tq = Tk = T).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  The return value reports host-side validation and
 *    launch errors only; device-side failures (a bounded wait that ran out)
 *    are read with attn_last_error().
 *  - Results are deterministic run to run.  The library is thread-compatible,
 *    not thread-safe: serialise concurrent calls from several host threads.
 *  - attn_fwd, attn_fwd_gqa, attn_fwd_decode, attn_bwd, attn_fwd_unfused and
 *    attn_fwd_host may be captured into a CUDA graph (stream capture) once a
 *    first call has done the device set-up in that context: they then only
 *    launch kernels and copies on `stream` (attn_fwd_host: on its own two
 *    streams, forked from and joined back to `stream` through events).
 *    attn_last_error synchronises and must not be captured.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_NULL = 1,           /* a required pointer is NULL                         */
    ATTN_ERR_UNSUPPORTED_DH = 2, /* d_h not in {64, 128}                               */
    ATTN_ERR_BAD_SHAPE = 3,      /* B, H or T < 1, or sizes overflow the limits above  */
    ATTN_ERR_ALIGN = 4,          /* a pointer is under-aligned (see the conventions)   */
    ATTN_ERR_BAD_SCALE = 5,      /* scale not finite or <= 0                           */
    ATTN_ERR_LAUNCH = 6,         /* a CUDA runtime/driver call failed                  */
    ATTN_ERR_TIMEOUT = 7,        /* device: a bounded wait ran out; the kernel returned */
    ATTN_ERR_NO_DEVICE = 8,      /* no usable sm_100 device is current                 */
    ATTN_ERR_BAD_ARG = 9,        /* another argument is out of range                   */
    ATTN_ERR_WORKSPACE_LIMIT = 10 /* problem too large for the library's static workspace */
} attn_status;

/*
 * Fused attention forward (one kernel; the T x T score and probability
 * matrices never reach device memory).
 *   q, k, v : in,  bf16 [B, H, T, d_h]
 *   o       : out, bf16 [B, H, T, d_h], each element written once
 *   lse     : out, fp32 [B, H, T], natural-log log-sum-exp of the scaled,
 *             masked scores of each query row
 * Returns ATTN_OK or an attn_status; nothing is launched on error.
 */
int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int T,
             int d_h, int causal, float scale, void *stream);

/*
 * Fused forward with grouped-query attention: the H query heads of a batch
 * entry share H_kv K/V heads, query head h reading K/V head h / (H / H_kv)
 * ("FlashAttention -- avoid writing the giant intermediate", "Return to the
 * incident": grouped-query attention changes how the head structure sizes the
 * persistent K/V state).
 *   q, o : bf16 [B, H, T, d_h];  k, v : bf16 [B, H_kv, T, d_h];  lse : fp32 [B, H, T]
 *   H_kv >= 1 and H % H_kv == 0 (H_kv = H is attn_fwd, H_kv = 1 multi-query).
 * Other arguments, errors and asynchrony as attn_fwd.
 */
int attn_fwd_gqa(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
                 int H_kv, int T, int d_h, int causal, float scale, void *stream);

/*
 * Decode forward: Tq new queries against a K/V cache of Tk >= Tq tokens,
 * query i at position Tk - Tq + i (causal: it sees keys 0 .. Tk - Tq + i;
 * "FlashAttention -- avoid writing the giant intermediate": persistent K/V
 * state in cached decoding, measured apart from prefill).  Grouped-query heads
 * as attn_fwd_gqa.  The key range is split across CTAs (split-KV) and the
 * pieces' partial results are merged by their log-sum-exp.
 *   q, o   : bf16 [B, H, Tq, d_h];  k, v : bf16 [B, H_kv, Tk, d_h]
 *   lse    : out, fp32 [B, H, Tq]
 *   ws     : caller-owned device workspace of attn_decode_workspace_bytes()
 *            bytes for the same sizes and splits (partial outputs)
 *   splits : > 0: every head's keys cut into that many equal ranges (clamped
 *            to [1, ceil(Tk / 128)]), one CTA each;  < 0: balanced -- one CTA
 *            per SM, all heads' 128-key tiles dealt out in equal contiguous
 *            ranges (a head may span several CTAs, a CTA several heads);
 *            0: automatic -- the split that fills one wave of one CTA per SM
 *            when that keeps at least 85 % of the SMs busy, else balanced
 * (H / H_kv) * Tq <= 65535 * 128.  Other arguments, errors and asynchrony as
 * attn_fwd.
 */
int attn_fwd_decode(const void *q, const void *k, const void *v, void *o, float *lse, void *ws,
                    int B, int H, int H_kv, int Tq, int Tk, int d_h, int causal, float scale,
                    int splits, void *stream);

/* Bytes of attn_fwd_decode's workspace for these sizes and splits; 0 on bad
 * sizes (or, with splits <= 0, without a device). */
size_t attn_decode_workspace_bytes(int B, int H, int H_kv, int Tq, int Tk, int d_h, int splits);

/*
 * Backward pass (gradients) of the fused forward, recomputing S and P from Q,
 * K and the forward's lse instead of reading stored intermediates
 * ("Attention Mechanism: Computation & Memory Patterns", section 4):
 *   dV = P^T dO,  dS = P o (dP - D) with dP = dO V^T and D_i = sum_c dO_ic O_ic,
 *   dQ = scale dS K,  dK = scale dS^T Q   (K/V heads sum over their group).
 *   q, o, dout : in,  bf16 [B, H, T, d_h]   (o, lse: the forward's outputs)
 *   k, v       : in,  bf16 [B, H_kv, T, d_h]
 *   lse        : in,  fp32 [B, H, T]
 *   dq         : out, bf16 [B, H, T, d_h];  dk, dv : out, bf16 [B, H_kv, T, d_h]
 *   ws         : caller-owned device workspace of attn_bwd_workspace_bytes()
 *                bytes (per-row statistics; contents on return unspecified)
 * Any T >= 1 (a ragged last block of 128 rows is padded internally);
 * H % H_kv == 0; B * H <= 65535; B * H * Tp < 2^31 with Tp = T rounded up to
 * a multiple of 128.  Other arguments, errors and asynchrony as attn_fwd.
 */
int attn_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
             const void *dout, void *dq, void *dk, void *dv, void *ws, int B, int H, int H_kv,
             int T, int d_h, int causal, float scale, void *stream);

/* Bytes of attn_bwd's workspace: B * H * Tp * 8, Tp = T rounded up to a
 * multiple of 128 (one pair of fp32 row statistics per padded row).  0 on bad
 * sizes. */
size_t attn_bwd_workspace_bytes(int B, int H, int T);

/*
 * Unfused attention forward: three kernels with the T x T intermediates in
 * device memory, as in the materialised path ("Storing and Rereading Large
 * Intermediate Matrices"):
 *   K1 writes S = Q K^T (raw, unscaled) to s_ws;
 *   K2 reads S, scales, masks, applies the row softmax, writes P to p_ws and
 *      the row log-sum-exp to lse;
 *   K3 reads P and V and writes O = P V.
 *   s_ws, p_ws : caller-owned bf16 [B, H, T, T] workspaces (2 bytes per
 *                entry, the pages' convention), attn_unfused_workspace_bytes()
 *                bytes each; contents on return are S and P -- under the
 *                causal mask only what the mask leaves visible is computed and
 *                moved: the 128 x 128 tiles of S at or below the diagonal, and
 *                each row of P up to the end of its 128-row block (zeros past
 *                the diagonal); the other entries are left as they were.
 * T must be a multiple of 128 on this path.  Other arguments as attn_fwd.
 */
int attn_fwd_unfused(const void *q, const void *k, const void *v, void *o, float *lse, void *s_ws,
                     void *p_ws, int B, int H, int T, int d_h, int causal, float scale,
                     void *stream);

/* Bytes of one unfused workspace (S or P): B * H * T * T * 2.  0 on bad sizes. */
size_t attn_unfused_workspace_bytes(int B, int H, int T);

/*
 * Unfused forward that allocates nothing and takes no workspace: S and P live
 * in a static device array inside the library (64 MiB, 32 MiB each for S and
 * P, reserved on every GPU that loads the library until the process exits).
 * The pages have no counterpart; this entry point exists for callers that
 * cannot call cudaMalloc -- for instance a plug-in inside a host application
 * that owns all device memory through its own pool, where a foreign
 * allocation can fail or break the host's accounting, or code that must not
 * risk the device synchronisation an allocation or free can cause.
 *   Sizes: as attn_fwd_unfused, plus B * H * T * T <= 16,777,216 (for
 *   example one head at T = 4096, or 16 heads at T = 1024); larger problems
 *   return ATTN_ERR_WORKSPACE_LIMIT and launch nothing.
 *   The first call on a device (and the first after a change of its CUDA
 *   context) looks up the array's device address (cudaGetSymbolAddress) for
 *   that device; make that first call before any stream capture.
 *   Every call on a device shares the one array and leaves its S and P there;
 *   nothing in it needs to start at zero (each call writes every entry of S
 *   and P that it later reads).  Calls whose work overlaps on the GPU (several
 *   streams, or several host threads) race on the array: serialise them.
 */
int attn_fwd_unfused_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                             int B, int H, int T, int d_h, int causal, float scale, void *stream);

/*
 * Fused forward with HOST buffers: copies q/k/v host -> device into the
 * caller's device buffers dq/dk/dv, runs attn_fwd into do_/dlse, and copies
 * O and lse back to o_host/lse_host.  The B * H heads are cut into up to 8
 * chunks so that the host -> device copy of one chunk, the attention of the
 * previous one (on `stream`) and the copy back of the one before run at the
 * same time (two library-owned streams, created on the first call per
 * device, carry the copies; they wait for the work already on `stream` and
 * `stream` waits for them at the end).  Host buffers should be pinned
 * (cudaHostAlloc) for asynchronous copies.  The call returns once everything
 * is enqueued; synchronise `stream` before reading o_host.  Not for
 * concurrent use from several host threads.
 */
int attn_fwd_host(const void *q_host, const void *k_host, const void *v_host, void *o_host,
                  float *lse_host, void *dq, void *dk, void *dv, void *do_, float *dlse, int B,
                  int H, int T, int d_h, int causal, float scale, void *stream);

/*
 * Device status word: synchronises the current device, returns the first
 * device-side error recorded since the previous call (ATTN_OK if none) and
 * clears it.  ATTN_ERR_LAUNCH if the synchronisation itself fails.
 */
int attn_last_error(void);

/* Static description of a status code. */
const char *attn_status_str(int status);

/*
 * CTAs the persistent fused kernel launches for this problem on the current
 * device: min(SMs, work items) CTAs of 384 threads, where a work item is a
 * block of 256 query rows of one head (causal: a pair of such blocks).
 * 0 on bad sizes or without a device.
 */
int attn_fused_grid_ctas(int B, int H, int T, int d_h, int causal);

/* Library version, "major.minor.patch". */
const char *attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
