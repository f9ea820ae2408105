/*
 * attn_selftest.h -- diagnostic entry points of the B200 attention library.
 *
 * These exercise, on one tile, the building blocks the attention kernels are
 * made of, so that a wrong bit in a descriptor shows up as a wrong number in
 * a small test rather than inside the full kernel.  They follow the same
 * conventions as attn.h (device pointers, 16-byte alignment, asynchronous on
 * `stream`, device errors via attn_last_error()).
 *
 * The tile products are the two matrix multiplications of scaled
 * dot-product attention ("Attention Mechanism: Computation & Memory
 * Patterns", section 1: S = Q K^T and O = P V), restricted to one 128-row
 * tile as in the tiled algorithm of section 3 of that page.
 */
#ifndef ATTN_B200_SELFTEST_H
#define ATTN_B200_SELFTEST_H

#ifdef __cplusplus
extern "C" {
#endif

/*
 * One score tile on the tensor cores: s[i][j] = sum_c q[i][c] * k[j][c]
 * for i, j in [0, 128), fp32 accumulation.
 *   q, k : in,  bf16 [128, d_h] row-major (d_h in {64, 128})
 *   s    : out, fp32 [128, 128] row-major
 */
int attn_selftest_qk_tile(const void *q, const void *k, float *s, int d_h, void *stream);

/*
 * One output tile with the probabilities held in tensor memory:
 * o[i][c] = sum_j p[i][j] * v[j][c] for i, j in [0, 128), c in [0, d_h).
 *   p : in,  bf16 [128, 128] row-major
 *   v : in,  bf16 [128, d_h] row-major
 *   o : out, fp32 [128, d_h] row-major
 */
int attn_selftest_pv_tile(const void *p, const void *v, float *o, int d_h, void *stream);

/*
 * Failure detection: launches one CTA that waits on a barrier nothing ever
 * completes, with a wait limit of `limit_us` microseconds (1 .. 10^6).  The
 * wait gives up, the kernel records ATTN_ERR_TIMEOUT in the status word and
 * returns normally, leaving the context usable.  attn_last_error() then
 * reports ATTN_ERR_TIMEOUT.
 */
int attn_selftest_timeout(int limit_us, void *stream);

/*
 * Scheduling order of the fused kernel's MMA warp.
 *   mode 0 (default): the next score MMA of a query tile is issued right
 *     after the PV MMA of that tile, in the tensor core's issue order;
 *   mode 1: the MMA warp waits for the PV MMA to complete before issuing the
 *     next score MMA into the same tensor-memory columns.
 * Both compute the same arithmetic in the same order; the tests compare them
 * bit for bit.  Returns the previous mode, or -1 for a bad mode.
 */
int attn_selftest_set_mma_order(int mode);

/*
 * Share of the softmax exponentials evaluated on the FMA pipe instead of the
 * special-function unit, in column pairs out of every 8: 0, 2, 3 or 4; -1
 * restores the per-head-size default.  Only tiles without masked keys use
 * the FMA-pipe form; results differ from the all-MUFU form by rounding only.
 * Returns the previous setting, or -2 for a value not built.
 */
int attn_selftest_set_exp_split(int pairs_of_8);

/*
 * Which wait gave up (an internal site code, 0 if none), as read by the most
 * recent attn_last_error() call; for diagnostics only.
 */
int attn_selftest_last_wait_site(void);

/*
 * Host only (no device needed): the work units the fused forward would run
 * for these sizes on a device with `sms` SMs, computed by the kernel's own
 * unit function.  A unit is 256 query rows of one query head: two 128-row
 * tiles that see n0 and n1 key tiles of 128.
 *   units : up to `cap` records of 7 ints (cta, k-th unit of that CTA, query
 *           head b * H + h, K/V head, first query row, n0, n1)
 *   ctas  : the grid the launch would use
 * Returns the number of units (records beyond `cap` are not written), or -1
 * for bad sizes.
 */
int attn_selftest_fused_plan(int B, int H, int H_kv, int T, int causal, int sms, int *units,
                             int cap, int *ctas);

/*
 * Host only (no device needed): the work plan attn_fwd_decode would launch
 * for these sizes and `splits` on a device with `sms` SMs, computed by the
 * same code the kernel runs.  A head is (batch * H_kv + K/V head, block of 128
 * packed query rows), numbered w = kvbh * ceil((H / H_kv) * Tq / 128) + block.
 *   segs   : up to seg_cap records of 8 ints
 *            (cta.x, cta.y, cta.z, kvbh, row block, first key tile, tiles, slot)
 *            -- one per segment, a segment being one head's key tiles in one
 *            CTA, its partial results going to partial slots slot .. slot +
 *            copies - 1 of that head (one per copy of the packed rows)
 *   nseg   : for heads w < nseg_cap, how many partial slots the merge reads
 *   slots  : the workspace's partial slots per query row
 *   copies : copies of the packed query rows in the 128-row tile (4, 2, 1)
 * Returns the number of segments (records beyond seg_cap are not written),
 * or -1 for bad sizes.
 */
int attn_selftest_decode_plan(int B, int H, int H_kv, int Tq, int Tk, int splits, int sms,
                              int *segs, int seg_cap, int *nseg, int nseg_cap, int *slots,
                              int *copies);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_SELFTEST_H */
