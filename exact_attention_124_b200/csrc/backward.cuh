// backward.cuh -- attention backward pass for B200 (sm_100a), recomputing S
// and P from Q, K and the forward's row log-sum-exp instead of storing them
// ("Attention Mechanism: Computation & Memory Patterns", section 4: the scores
// that were never saved are recomputed in the backward pass).
//
// Gradients (per head, scale s, P the masked row softmax of s Q K^T):
//   dV = P^T dO,  dP = dO V^T,  dS = P o (dP - D),  D_i = sum_c dO_ic O_ic,
//   dQ = s dS K,  dK = s dS^T Q.
// Three kernels, no atomics:
//   bwd_stats_kernel  per query row: (lse * log2 e, D) -- one warp per row
//   bwd_dkdv_kernel   one CTA per (K/V head, 128 keys): loops over the query
//                     heads of its group and the query blocks that see these
//                     keys; S^T = K Q^T and dP^T = V dO^T on tcgen05 into TMEM,
//                     P^T and dS^T written back over them as bf16, then
//                     dV += P^T dO and dK += dS^T Q accumulate in TMEM
//   bwd_dq_kernel     one CTA per (query head, 128 queries): loops over the key
//                     blocks it sees; S and dP into TMEM, dS back as bf16,
//                     dQ += dS K in TMEM (its own schedule: see DqCfg below)
// Both gradient kernels: warps 0-3 / 4-7 are elementwise warpgroups 0 / 1
// (thread = TMEM lane = the stationary block's row), warp 8 issues MMAs,
// warp 9 issues TMA copies.
// At d_h = 64 the dK/dV pass runs bwd_dkdv64_kernel (the dQ kernel's
// schedule: 128-wide score MMAs, two S^T buffers).  dK/dV kernel at d_h =
// 128: each 128-wide block of queries is taken as two 64-wide
// halves, half h in TMEM buffer h and handled by elementwise warpgroup h, so
// the tensor cores compute one half's S/dP and accumulate the other's
// gradient while a warpgroup does the elementwise step (a two-buffer
// ping-pong; TMEM has room for two 64-column S/dP pairs next to the 2 d_h
// accumulator columns, not for two 128-column ones).  TMEM: buffer h = S/P
// [128h, 128h + 64), dP/dS [128h + 64, 128h + 128); accumulators from 256.
#pragma once

#include "sm100.cuh"

namespace attn {

struct BwdParams {
    const float2 *stats;  // [B*H, Tp] (lse * log2 e, D); rows T .. Tp-1 of a head: (+inf, 0)
    __nv_bfloat16 *out_a; // dkdv: dK [B*H_kv, T, D];  dq: dQ [B*H, T, D]
    __nv_bfloat16 *out_b; // dkdv: dV [B*H_kv, T, D]
    int H, H_kv, group, T, nq, causal;
    int Tp;               // T rounded up to the 128-row block: 128 * nq
    float c_log2;         // scale * log2 e
    float scale;
    unsigned long long limit_ns;
};

enum : unsigned int { W_B_KV = 96, W_B_STFULL, W_B_STEMPTY, W_B_SFULL, W_B_PFULL, W_B_DONE, W_B_DRAIN };

template <int D>
struct BwdCfg {
    static_assert(D == 64 || D == 128, "d_h must be 64 or 128");
    static constexpr int KB = D / 64;
    static constexpr int SUB = 128 * 128;       // 128 rows x 128 bytes
    static constexpr int TILE = 128 * D * 2;    // one 128-row tile
    static constexpr int NST = 2;               // ring stages
    static constexpr int STAGE = 2 * TILE + 1024;  // two tiles + 128 row statistics
    static constexpr int OFF_FIX = 0;           // the stationary pair of tiles
    static constexpr int OFF_RING = 2 * TILE;
    static constexpr int OFF_BAR = OFF_RING + NST * STAGE;
    static constexpr int NBAR = 1 + 2 * NST + 4 + 2;
    static constexpr int SMEM = 1024 + OFF_BAR + NBAR * 8 + 16;
    static constexpr int THREADS = 320;
    static constexpr int MMA_WARP = 8, TMA_WARP = 9;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_ACC0 = 256, TM_ACC1 = 256 + D;
    static constexpr int HALF = 64 * 128;       // 64 rows x 128 bytes of a SW128 block
    __host__ __device__ static constexpr uint32_t tm_s(int h) { return 128u * h; }
    __host__ __device__ static constexpr uint32_t tm_dp(int h) { return 128u * h + 64u; }
    static constexpr uint32_t IDESC_SQ = idesc_bf16_f32(128, 64, false);   // N = 64 rows of B
    static constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, D, true);    // B MN-major, N = d_h
};

// ---------------------------------------------------------------- preprocess
// stats[h * Tp + t] = (lse * log2 e, sum_c dO[c] O[c]) of row t of head h, one
// warp per row; rows t >= T (padding up to the 128-row block) get (+inf, 0):
// their probabilities 2^(s - inf) are exactly 0 and their dS = P (dP - 0) too,
// so the zero rows the tensor maps read there add nothing to the gradients.
template <int D>
__global__ void __launch_bounds__(256)
    bwd_stats_kernel(const __nv_bfloat16 *__restrict__ O, const __nv_bfloat16 *__restrict__ dO,
                     const float *__restrict__ lse, float2 *__restrict__ stats, long long prow,
                     int T, int Tp)
{
    const long long pr = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (pr >= prow) return;
    const long long head = pr / Tp;
    const int t = (int)(pr - head * Tp);
    if (t >= T) {
        if (lane == 0) stats[pr] = make_float2(INFINITY, 0.f);
        return;
    }
    const long long r = head * T + t;
    constexpr int PER = D / 32;  // bf16 values per lane: 4 (8 bytes) or 2 (4 bytes)
    const __nv_bfloat16 *o = O + r * D + lane * PER;
    const __nv_bfloat16 *g = dO + r * D + lane * PER;
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) acc = fmaf(__bfloat162float(o[i]), __bfloat162float(g[i]), acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) stats[pr] = make_float2(lse[r] * 1.4426950408889634f, acc);
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}

// Common CTA set-up of both gradient kernels: shared-memory carve-up,
// barrier init, TMEM allocation.  Returns the TMEM base.
template <int D>
struct BwdSmem {
    uint32_t base, fix, ring, bar;
    uint8_t *gbase;
    uint32_t b_fix, b_full, b_empty, b_sfull, b_pfull, b_done, b_drain;
    uint32_t *tmem_slot;
    volatile int *abort_flag;
    __device__ __forceinline__ void init(uint8_t *smem_raw)
    {
        using C = BwdCfg<D>;
        const uint32_t raw = smem_addr(smem_raw);
        base = (raw + 1023u) & ~1023u;
        gbase = smem_raw + (base - raw);
        fix = base + C::OFF_FIX;
        ring = base + C::OFF_RING;
        bar = base + C::OFF_BAR;
        b_fix = bar;
        b_full = bar + 8;                 // [NST]
        b_empty = b_full + 8 * C::NST;    // [NST]
        b_sfull = b_empty + 8 * C::NST;   // [2]: S/dP of buffer h computed
        b_pfull = b_sfull + 16;           // [2]: P/dS of buffer h written
        b_done = b_pfull + 16;
        b_drain = b_done + 8;
        tmem_slot = reinterpret_cast<uint32_t *>(gbase + C::OFF_BAR + C::NBAR * 8);
        abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    }
};

template <int D>
__device__ __forceinline__ uint32_t bwd_setup(BwdSmem<D> &sm, int warp)
{
    using C = BwdCfg<D>;
    if (threadIdx.x == 0) {
        mbar_init(sm.b_fix, 1);
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(sm.b_full + 8 * s, 1);
            mbar_init(sm.b_empty + 8 * s, 1);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(sm.b_sfull + 8 * h, 1);
            mbar_init(sm.b_pfull + 8 * h, 128);
        }
        mbar_init(sm.b_done, 1);
        mbar_init(sm.b_drain, 1);
        *sm.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc(smem_addr(sm.tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    return *sm.tmem_slot;
}

// Elementwise step of both kernels on one 128 x 64 half block, one row per
// thread, 32 columns at a time: p = 2^(s c - lse2) (0 where masked) and
// ds = p (dp - D).  With WRITE_P, P (bf16 pairs) goes over the first 32 S
// columns of the buffer; dS goes to tDS (over the dP columns in the dK/dV
// kernel, over the S columns in the dQ kernel).  Chunk c writes columns
// [16c, 16c + 16), all of which this or the earlier chunk has already read.
// PER_COLUMN: rows are keys and the statistics come per query column from
// shared memory; else rows are queries and the row's own statistics are
// st_row.  The buffer is signalled on b_pfull once all of it is in TMEM.
template <bool PER_COLUMN, bool WRITE_P>
__device__ __forceinline__ void bwd_elementwise(uint32_t tS, uint32_t tDP, float cl2,
                                                const float2 *st_col, float2 st_row,
                                                bool need_mask, int row_idx, int col0,
                                                uint32_t tDS, uint32_t b_pfull)
{
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        uint32_t rs[32], rd[32];
        tmem_ld32(tS + 32 * c, rs);
        tmem_ld32(tDP + 32 * c, rd);
        tmem_wait_ld_regs(rs);
        tmem_wait_ld_regs(rd);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int q = 0; q < 32; q += 2) {
            float pr[2], dsr[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int cc = 32 * c + q + e;
                const float2 sd = PER_COLUMN ? st_col[cc] : st_row;
                float pv = fast_exp2(fmaf(__uint_as_float(rs[q + e]), cl2, -sd.x));
                if (need_mask) {
                    // PER_COLUMN: rows are keys, columns queries; else the reverse
                    const int key = PER_COLUMN ? row_idx : col0 + cc;
                    const int qry = PER_COLUMN ? col0 + cc : row_idx;
                    if (key > qry) pv = 0.f;
                }
                pr[e] = pv;
                dsr[e] = pv * (__uint_as_float(rd[q + e]) - sd.y);
            }
            pk[q >> 1] = pack_bf16x2(pr[0], pr[1]);
            dk[q >> 1] = pack_bf16x2(dsr[0], dsr[1]);
        }
        if (WRITE_P) tmem_st16(tS + 16 * c, pk);
        tmem_st16(tDS + 16 * c, dk);
    }
    tmem_wait_st();
    tc_fence_before_sync();
    mbar_arrive(b_pfull);
}

// Epilogue: 32-column chunks [C0, C1) of the rows of a TMEM accumulator times
// `mul`, as bf16; a lane whose row is padding (`store` false) reads its TMEM
// lane like the others -- tcgen05.ld is a whole-warp instruction -- and writes
// nothing.
template <int C0, int C1>
__device__ __forceinline__ void store_rows(uint32_t tacc, float mul, __nv_bfloat16 *dst, bool store)
{
#pragma unroll
    for (int c = C0; c < C1; ++c) {
        uint32_t r[32];
        tmem_ld32(tacc + 32 * c, r);
        tmem_wait_ld_regs(r);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * mul, __uint_as_float(r[2 * i + 1]) * mul);
        if (store) {
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + 32 * c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
    }
}

// MMA issue order of both kernels, iteration n of the moving operand, halves
// 0 and 1 in buffers 0 and 1:
//   sdp(0,0) sdp(0,1) | acc(n,0) sdp(n+1,0) acc(n,1) [stage free] sdp(n+1,1) | ...
// where sdp(n,h) computes S/dP of half h into buffer h (signalled on
// b_sfull[h]) and acc(n,h) waits for warpgroup h's P/dS (b_pfull[h]) and
// accumulates from it.  The tensor pipe runs in issue order, so sdp(n+1,h)
// overwrites buffer h only after acc(n,h) has read it.  Each of the four
// barriers completes once per iteration and its waiter has passed the
// previous completion before the next can start, so parity n & 1 is exact.
template <typename Sdp, typename Acc, typename Full>
__device__ __forceinline__ bool bwd_mma_loop(int niter, uint32_t b_pfull, uint32_t b_empty,
                                             uint64_t lim, volatile int *abort_flag, Sdp sdp,
                                             Acc acc, Full wait_full, int nst)
{
    if (niter <= 0) return true;
    if (!wait_full(0)) return false;
    tc_fence_after_sync();
    sdp(0, 0);
    sdp(0, 1);
    for (int n = 0; n < niter; ++n) {
        const uint32_t par = (uint32_t)n & 1u;
        if (!mbar_wait(b_pfull, par, lim, W_B_PFULL, abort_flag)) return false;
        tc_fence_after_sync();
        acc(n, 0);
        const bool more = n + 1 < niter;
        if (more) {
            if (!wait_full(n + 1)) return false;
            tc_fence_after_sync();
            sdp(n + 1, 0);
        }
        if (!mbar_wait(b_pfull + 8, par, lim, W_B_PFULL, abort_flag)) return false;
        tc_fence_after_sync();
        acc(n, 1);
        tc_commit(b_empty + 8 * (n % nst));
        if (more) sdp(n + 1, 1);
    }
    return true;
}

// ---------------------------------------------------------------- dK, dV
// grid: (T / 128 key blocks, B * H_kv); key block j = blockIdx.x (causal:
// the lowest keys see the most queries, so the longest CTAs start first).
template <int D>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const BwdParams p)
{
    static_assert(D == 128, "d_h = 64 runs bwd_dkdv64_kernel");
    using C = BwdCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    BwdSmem<D> sm;
    sm.init(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t tmem = bwd_setup<D>(sm, warp);
    const uint64_t lim = p.limit_ns;
    const int j = blockIdx.x;
    const int kvbh = blockIdx.y;
    const int b = kvbh / p.H_kv, kvl = kvbh % p.H_kv;
    const int i0 = p.causal ? j : 0;
    const int per_head = p.nq - i0;
    const int niter = p.group * per_head;
    const uint32_t sK = sm.fix, sV = sm.fix + C::TILE;

    if (warp == C::TMA_WARP) {
        if (lane == 0) {  // TMA: K_j, V_j once; then Q_i, dO_i, stats per iteration
            const uint64_t pol = policy_evict_last();
            mbar_arrive_expect_tx(sm.b_fix, 2 * C::TILE);
            for (int kb = 0; kb < C::KB; ++kb) {
                tma_load_3d(sK + kb * C::SUB, &tmK, sm.b_fix, 64 * kb, 128 * j, kvbh, pol);
                tma_load_3d(sV + kb * C::SUB, &tmV, sm.b_fix, 64 * kb, 128 * j, kvbh, pol);
            }
            uint32_t armed = 0, armed_par = 0;
            bool ok = true;
            for (int n = 0; n < niter; ++n) {
                const int s = n % C::NST;
                const uint32_t par = (uint32_t)(n / C::NST) & 1u;
                if (!mbar_wait(sm.b_empty + 8 * s, par ^ 1u, lim, W_B_STEMPTY, sm.abort_flag)) {
                    ok = false;
                    break;
                }
                const int g = n / per_head, i = i0 + n % per_head;
                const int bh = b * (p.H_kv * p.group) + kvl * p.group + g;
                const uint32_t st = sm.ring + s * C::STAGE;
                mbar_arrive_expect_tx(sm.b_full + 8 * s, 2 * C::TILE + 1024);
                armed |= 1u << s;
                armed_par = (armed_par & ~(1u << s)) | (par << s);
                for (int kb = 0; kb < C::KB; ++kb) {
                    tma_load_3d(st + kb * C::SUB, &tmQ, sm.b_full + 8 * s, 64 * kb, 128 * i, bh, pol);
                    tma_load_3d(st + C::TILE + kb * C::SUB, &tmdO, sm.b_full + 8 * s, 64 * kb,
                                128 * i, bh, pol);
                }
                bulk_load(st + 2 * C::TILE, p.stats + (size_t)bh * p.Tp + 128 * i, 1024,
                          sm.b_full + 8 * s);
            }
            if (!ok) {
                *sm.abort_flag = 1;
                mbar_wait(sm.b_fix, 0, lim, W_B_KV);
                for (int s = 0; s < C::NST; ++s)
                    if ((armed >> s) & 1u) mbar_wait(sm.b_full + 8 * s, (armed_par >> s) & 1u, lim, W_B_STFULL);
            }
        }
    } else if (warp == C::MMA_WARP) {
        if (lane == 0) {  // MMA issuer
            bool ok = mbar_wait(sm.b_fix, 0, lim, W_B_KV, sm.abort_flag);
            tc_fence_after_sync();
            const uint32_t kl = sw128_desc_lo(sK, 16), vl = sw128_desc_lo(sV, 16);
            auto wait_full = [&](int n) {
                return mbar_wait(sm.b_full + 8 * (n % C::NST), (uint32_t)(n / C::NST) & 1u, lim,
                                 W_B_STFULL, sm.abort_flag);
            };
            auto sdp = [&](int n, int h) {  // S^T = K Q_h^T, dP^T = V dO_h^T (64 queries)
                const uint32_t st = sm.ring + (n % C::NST) * C::STAGE + h * C::HALF;
                const uint32_t ql = sw128_desc_lo(st, 16), gl = sw128_desc_lo(st + C::TILE, 16);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::SUB + (kk & 3) * 32) >> 4;
                    mma_ss(tmem + C::tm_s(h), sw128_desc_join(kl + off, 1024),
                           sw128_desc_join(ql + off, 1024), C::IDESC_SQ, kk > 0 ? 1u : 0u);
                    mma_ss(tmem + C::tm_dp(h), sw128_desc_join(vl + off, 1024),
                           sw128_desc_join(gl + off, 1024), C::IDESC_SQ, kk > 0 ? 1u : 0u);
                }
                tc_commit(sm.b_sfull + 8 * h);
            };
            auto acc = [&](int n, int h) {  // dV += P_h^T dO_h, dK += dS_h^T Q_h (16 queries each)
                const uint32_t st = sm.ring + (n % C::NST) * C::STAGE;
                const uint32_t qm = sw128_desc_lo(st, C::SUB), gm = sw128_desc_lo(st + C::TILE, C::SUB);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t a = (n > 0 || h > 0 || kk > 0) ? 1u : 0u;
                    const uint32_t boff = (uint32_t)(4 * h + kk) * (2048 >> 4);
                    mma_ts(tmem + C::TM_ACC0, tmem + C::tm_s(h) + 8 * kk,
                           sw128_desc_join(gm + boff, 1024), C::IDESC_ACC, a);
                    mma_ts(tmem + C::TM_ACC1, tmem + C::tm_dp(h) + 8 * kk,
                           sw128_desc_join(qm + boff, 1024), C::IDESC_ACC, a);
                }
            };
            ok = ok && bwd_mma_loop(niter, sm.b_pfull, sm.b_empty, lim, sm.abort_flag, sdp, acc,
                                    wait_full, C::NST);
            if (!ok) *sm.abort_flag = 1;
            tc_commit(sm.b_done);  // fires when every MMA issued above has completed
        }
    } else if (warp < 8) {  // elementwise warpgroup h: thread = key row, queries of half h
        const int h = warp >> 2;
        const int kr = (warp & 3) * 32 + lane;
        const int key = 128 * j + kr;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        bool ok = true;
        for (int n = 0; ok && n < niter; ++n) {
            const int s = n % C::NST;
            const uint32_t par = (uint32_t)(n / C::NST) & 1u;
            const int i = i0 + n % per_head;
            bool w = mbar_wait(sm.b_full + 8 * s, par, lim, W_B_STFULL, sm.abort_flag);
            w = w && mbar_wait(sm.b_sfull + 8 * h, (uint32_t)n & 1u, lim, W_B_SFULL, sm.abort_flag);
            if (!(ok = __all_sync(0xffffffffu, w))) break;
            tc_fence_after_sync();
            const float2 *stc = reinterpret_cast<const float2 *>(sm.gbase + C::OFF_RING +
                                                                 s * C::STAGE + 2 * C::TILE) +
                                64 * h;
            const bool need_mask = p.causal && i == j;
            bwd_elementwise<true, true>(tmem + lane_off + C::tm_s(h), tmem + lane_off + C::tm_dp(h),
                                        p.c_log2, stc, make_float2(0.f, 0.f), need_mask, key,
                                        128 * i + 64 * h, tmem + lane_off + C::tm_dp(h),
                                        sm.b_pfull + 8 * h);
        }
        const bool w = ok && mbar_wait(sm.b_done, 0, lim, W_B_DONE, sm.abort_flag);
        if (__all_sync(0xffffffffu, w) && !*sm.abort_flag) {
            tc_fence_after_sync();
            const size_t orow = ((size_t)kvbh * p.T + key) * D;
            const bool real = key < p.T;  // padding rows of the last key block store nothing
            if (h == 0)
                store_rows<0, D / 32>(tmem + lane_off + C::TM_ACC1, p.scale, p.out_a + orow, real);  // dK
            else
                store_rows<0, D / 32>(tmem + lane_off + C::TM_ACC0, 1.f, p.out_b + orow, real);  // dV
        } else {
            *sm.abort_flag = 1;
        }
    }
    if (warp == C::MMA_WARP && lane == 0 && *sm.abort_flag) {
        tc_commit(sm.b_drain);
        mbar_wait(sm.b_drain, 0, lim, W_B_DRAIN);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == C::MMA_WARP) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ---------------------------------------------------------------- dK, dV at d_h = 64
// At d_h = 64 the two accumulators take 128 TMEM columns, which leaves room
// for the dQ kernel's schedule with 128-wide score MMAs: two S^T buffers, one
// dP^T buffer, and per query block n
//   dP^T(n+1) [once both warpgroups hold dP^T(n) in registers]
//   dV += P^T(n) dO_n, dK += dS^T(n) Q_n [once P^T, dS^T are written]
//   S^T(n+2) [into the buffer just read]
// Warpgroup h takes queries [64h, 64h + 64) of every block and writes its
// P^T and dS^T as bf16 pairs over its own 64 S^T columns (P^T first 32,
// dS^T last 32).  TMEM: S^T buffer b [128b, 128b + 128), dP^T [256, 384),
// dV [384, 448), dK [448, 512).
struct Dkdv64Cfg {
    static constexpr int D = 64;
    static constexpr int TILE = 128 * D * 2;        // 16 KB
    static constexpr int NST = 5;                   // stages: Q, dO and statistics of a block
    static constexpr int STAGE = 2 * TILE + 1024;
    static constexpr int OFF_FIX = 0;               // K, V
    static constexpr int OFF_RING = 2 * TILE;
    static constexpr int OFF_BAR = OFF_RING + NST * STAGE;
    // fix, full/empty[NST], sfull[2], dpfull, dpfree, pfull[2], done, drain
    static constexpr int NBAR = 1 + 2 * NST + 2 + 1 + 1 + 2 + 1 + 1;
    static constexpr int SMEM = 1024 + OFF_BAR + NBAR * 8 + 16;
    static constexpr int THREADS = 320;
    static constexpr int MMA_WARP = 8, TMA_WARP = 9;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_DP = 256, TM_DV = 384, TM_DK = 448;  // S^T buffer b at 128 b
    static constexpr uint32_t IDESC_SQ = idesc_bf16_f32(128, 128, false);
    static constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, D, true);
};

// grid: (T / 128 key blocks, B * H_kv), as bwd_dkdv_kernel.
__global__ void __launch_bounds__(Dkdv64Cfg::THREADS, 1)
    bwd_dkdv64_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                      const BwdParams p)
{
    using C = Dkdv64Cfg;
    constexpr int D = C::D;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t sK = base + C::OFF_FIX, sV = sK + C::TILE, ring = base + C::OFF_RING;
    const uint32_t b_fix = base + C::OFF_BAR;
    const uint32_t b_full = b_fix + 8, b_empty = b_full + 8 * C::NST;
    const uint32_t b_sfull = b_empty + 8 * C::NST;  // [2] S^T(n) in buffer n & 1
    const uint32_t b_dpfull = b_sfull + 16;         // dP^T(n) computed
    const uint32_t b_dpfree = b_dpfull + 8;         // both warpgroups hold dP^T(n) in registers
    const uint32_t b_pfull = b_dpfree + 8;          // [2] P^T(n), dS^T(n) written over buffer n & 1
    const uint32_t b_done = b_pfull + 16;
    const uint32_t b_drain = b_done + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + C::OFF_BAR + C::NBAR * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(b_fix, 1);
        for (int s2 = 0; s2 < C::NST; ++s2) {
            mbar_init(b_full + 8 * s2, 1);
            mbar_init(b_empty + 8 * s2, 1);
        }
        for (int b2 = 0; b2 < 2; ++b2) {
            mbar_init(b_sfull + 8 * b2, 1);
            mbar_init(b_pfull + 8 * b2, 256);
        }
        mbar_init(b_dpfull, 1);
        mbar_init(b_dpfree, 256);
        mbar_init(b_done, 1);
        mbar_init(b_drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint64_t lim = p.limit_ns;
    const int j = blockIdx.x;
    const int kvbh = blockIdx.y;
    const int b = kvbh / p.H_kv, kvl = kvbh % p.H_kv;
    const int i0 = p.causal ? j : 0;
    const int per_head = p.nq - i0;
    const int niter = p.group * per_head;

    if (warp == C::TMA_WARP) {
        if (lane == 0) {  // TMA: K_j, V_j once; then Q_i, dO_i, statistics per query block
            const uint64_t pol = policy_evict_last();
            mbar_arrive_expect_tx(b_fix, 2 * C::TILE);
            tma_load_3d(sK, &tmK, b_fix, 0, 128 * j, kvbh, pol);
            tma_load_3d(sV, &tmV, b_fix, 0, 128 * j, kvbh, pol);
            uint32_t armed = 0, armed_par = 0;
            bool ok = true;
            for (int n = 0; n < niter; ++n) {
                const int s2 = n % C::NST;
                const uint32_t par = (uint32_t)(n / C::NST) & 1u;
                if (!mbar_wait(b_empty + 8 * s2, par ^ 1u, lim, W_B_STEMPTY, abort_flag)) {
                    ok = false;
                    break;
                }
                const int g = n / per_head, i = i0 + n % per_head;
                const int bh = b * (p.H_kv * p.group) + kvl * p.group + g;
                const uint32_t st = ring + s2 * C::STAGE;
                mbar_arrive_expect_tx(b_full + 8 * s2, 2 * C::TILE + 1024);
                armed |= 1u << s2;
                armed_par = (armed_par & ~(1u << s2)) | (par << s2);
                tma_load_3d(st, &tmQ, b_full + 8 * s2, 0, 128 * i, bh, pol);
                tma_load_3d(st + C::TILE, &tmdO, b_full + 8 * s2, 0, 128 * i, bh, pol);
                bulk_load(st + 2 * C::TILE, p.stats + (size_t)bh * p.Tp + 128 * i, 1024, b_full + 8 * s2);
            }
            if (!ok) {
                *abort_flag = 1;
                mbar_wait(b_fix, 0, lim, W_B_KV);
                for (int s2 = 0; s2 < C::NST; ++s2)
                    if ((armed >> s2) & 1u) mbar_wait(b_full + 8 * s2, (armed_par >> s2) & 1u, lim, W_B_STFULL);
            }
        }
    } else if (warp == C::MMA_WARP) {
        if (lane == 0) {  // MMA issuer
            bool ok = mbar_wait(b_fix, 0, lim, W_B_KV, abort_flag);
            tc_fence_after_sync();
            const uint32_t kl = sw128_desc_lo(sK, 16), vl = sw128_desc_lo(sV, 16);
            auto stage = [&](int n) { return ring + (n % C::NST) * C::STAGE; };
            auto wait_full = [&](int n) {
                return mbar_wait(b_full + 8 * (n % C::NST), (uint32_t)(n / C::NST) & 1u, lim, W_B_STFULL,
                                 abort_flag);
            };
            auto s_mma = [&](int n) {  // S^T(n) = K Q_n^T into buffer n & 1
                const uint32_t ql = sw128_desc_lo(stage(n), 16);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (uint32_t)(kk * 32) >> 4;
                    mma_ss(tmem + 128u * (n & 1), sw128_desc_join(kl + off, 1024),
                           sw128_desc_join(ql + off, 1024), C::IDESC_SQ, kk > 0 ? 1u : 0u);
                }
                tc_commit(b_sfull + 8 * (n & 1));
            };
            auto dp_mma = [&](int n) {  // dP^T(n) = V dO_n^T
                const uint32_t gl = sw128_desc_lo(stage(n) + C::TILE, 16);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (uint32_t)(kk * 32) >> 4;
                    mma_ss(tmem + C::TM_DP, sw128_desc_join(vl + off, 1024),
                           sw128_desc_join(gl + off, 1024), C::IDESC_SQ, kk > 0 ? 1u : 0u);
                }
                tc_commit(b_dpfull);
            };
            if (ok && (ok = wait_full(0))) {
                tc_fence_after_sync();
                s_mma(0);
                dp_mma(0);
            }
            if (ok && niter > 1 && (ok = wait_full(1))) {
                tc_fence_after_sync();
                s_mma(1);
            }
            for (int n = 0; ok && n < niter; ++n) {
                if (n + 1 < niter) {  // dP^T(n+1) once dP^T(n) is out of TMEM (stage n+1 is in)
                    if (!(ok = mbar_wait(b_dpfree, (uint32_t)n & 1u, lim, W_B_PFULL, abort_flag))) break;
                    tc_fence_after_sync();
                    dp_mma(n + 1);
                }
                if (!(ok = mbar_wait(b_pfull + 8 * (n & 1), (uint32_t)(n >> 1) & 1u, lim, W_B_PFULL,
                                     abort_flag)))
                    break;
                tc_fence_after_sync();
                // dV += P^T dO_n, dK += dS^T Q_n: queries [64h, 64h + 64) at columns 64h + [0, 32)
                // (P^T) and 64h + [32, 64) (dS^T) as bf16 pairs
                const uint32_t st = stage(n);
                const uint32_t qm = sw128_desc_lo(st, 16384), gm = sw128_desc_lo(st + C::TILE, 16384);
                const uint32_t tb = tmem + 128u * (n & 1);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a = (n > 0 || kk > 0) ? 1u : 0u;
                    const uint32_t col = 64u * (kk >> 2) + 8u * (kk & 3);
                    const uint32_t boff = (uint32_t)kk * (2048 >> 4);
                    mma_ts(tmem + C::TM_DV, tb + col, sw128_desc_join(gm + boff, 1024), C::IDESC_ACC, a);
                    mma_ts(tmem + C::TM_DK, tb + col + 32, sw128_desc_join(qm + boff, 1024), C::IDESC_ACC, a);
                }
                tc_commit(b_empty + 8 * (n % C::NST));  // Q_n, dO_n and the statistics are used up
                if (n + 2 < niter) {  // S^T(n+2) into the buffer just read (in issue order)
                    if (!(ok = wait_full(n + 2))) break;
                    tc_fence_after_sync();
                    s_mma(n + 2);
                }
            }
            if (!ok) *abort_flag = 1;
            tc_commit(b_done);
        }
    } else if (warp < 8) {  // elementwise warpgroup h: thread = key row, queries [64h, 64h + 64)
        const int h = warp >> 2;
        const int kr = (warp & 3) * 32 + lane;
        const int key = 128 * j + kr;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const float cl2 = p.c_log2;
        bool ok = true;
        for (int n = 0; ok && n < niter; ++n) {
            const int s2 = n % C::NST;
            const int i = i0 + n % per_head;
            bool w = mbar_wait(b_full + 8 * s2, (uint32_t)(n / C::NST) & 1u, lim, W_B_STFULL, abort_flag);
            w = w && mbar_wait(b_sfull + 8 * (n & 1), (uint32_t)(n >> 1) & 1u, lim, W_B_SFULL, abort_flag);
            w = w && mbar_wait(b_dpfull, (uint32_t)n & 1u, lim, W_B_SFULL, abort_flag);
            if (!(ok = __all_sync(0xffffffffu, w))) break;
            tc_fence_after_sync();
            const uint32_t tS = tmem + lane_off + 128u * (n & 1) + 64 * h;
            const uint32_t tD = tmem + lane_off + C::TM_DP + 64 * h;
            uint32_t rs[64], rd[64];
            {
                uint32_t a0[32], a1[32], d0[32], d1[32];
                tmem_ld32(tS, a0);
                tmem_ld32(tS + 32, a1);
                tmem_ld32(tD, d0);
                tmem_ld32(tD + 32, d1);
                tmem_wait_ld_regs(a0);
                tmem_wait_ld_regs(a1);
                tmem_wait_ld_regs(d0);
                tmem_wait_ld_regs(d1);
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    rs[x] = a0[x];
                    rs[32 + x] = a1[x];
                    rd[x] = d0[x];
                    rd[32 + x] = d1[x];
                }
            }
            tc_fence_before_sync();
            mbar_arrive(b_dpfree);  // dP^T(n) is in registers: dP^T(n+1) may overwrite it
            const float2 *stc =
                reinterpret_cast<const float2 *>(gbase + C::OFF_RING + s2 * C::STAGE + 2 * C::TILE) + 64 * h;
            const bool need_mask = p.causal && i == j;
            const int q0 = 128 * i + 64 * h;
            uint32_t pk[32], dk[32];
#pragma unroll
            for (int q = 0; q < 64; q += 2) {
                float pr[2], dsr[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float2 sd = stc[q + e];
                    float pv = fast_exp2(fmaf(__uint_as_float(rs[q + e]), cl2, -sd.x));
                    if (need_mask && key > q0 + q + e) pv = 0.f;
                    pr[e] = pv;
                    dsr[e] = pv * (__uint_as_float(rd[q + e]) - sd.y);
                }
                pk[q >> 1] = pack_bf16x2(pr[0], pr[1]);
                dk[q >> 1] = pack_bf16x2(dsr[0], dsr[1]);
            }
            tmem_st32(tS, pk);
            tmem_st32(tS + 32, dk);
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(b_pfull + 8 * (n & 1));
        }
        const bool w = ok && mbar_wait(b_done, 0, lim, W_B_DONE, abort_flag);
        if (__all_sync(0xffffffffu, w) && !*abort_flag) {
            tc_fence_after_sync();
            const size_t orow = ((size_t)kvbh * p.T + key) * D;
            const bool real = key < p.T;  // padding rows of the last key block store nothing
            if (h == 0)
                store_rows<0, D / 32>(tmem + lane_off + C::TM_DK, p.scale, p.out_a + orow, real);  // dK
            else
                store_rows<0, D / 32>(tmem + lane_off + C::TM_DV, 1.f, p.out_b + orow, real);  // dV
        } else {
            *abort_flag = 1;
        }
    }
    if (warp == C::MMA_WARP && lane == 0 && *abort_flag) {
        tc_commit(b_drain);
        mbar_wait(b_drain, 0, lim, W_B_DRAIN);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == C::MMA_WARP) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ---------------------------------------------------------------- dQ
// The dQ kernel keeps 128-wide score MMAs (64-wide ones run at 2/3 of the
// rate): TMEM holds two S buffers, one dP buffer and dQ (2 x 128 + 128 + d_h
// <= 512 columns), K and V stream through separate rings, and the MMA issue
// order per key block n is
//   dP(n+1) [once both warpgroups hold dP(n) in registers]
//   dQ += dS(n) K_n [once dS(n) is written]  S(n+2) [into dS(n)'s buffer]
// so the tensor pipe computes the next blocks' S and dP during the
// elementwise step of block n.  Warpgroup h takes keys [64h, 64h + 64) of
// every block and writes its dS as bf16 pairs over the first 32 of its own
// 64 S columns.
template <int D>
struct DqCfg {
    static constexpr int KB = D / 64;
    static constexpr int SUB = 128 * 128;
    static constexpr int TILE = 128 * D * 2;
    static constexpr int NK = (D == 128) ? 3 : 4;   // K ring slots
    static constexpr int NV = (D == 128) ? 2 : 3;   // V ring slots
    static constexpr int OFF_FIX = 0;               // Q, dO
    static constexpr int OFF_K = 2 * TILE;
    static constexpr int OFF_V = OFF_K + NK * TILE;
    static constexpr int OFF_BAR = OFF_V + NV * TILE;
    // fix, kfull/kempty[NK], vfull/vempty[NV], sfull[2], dpfull, dpfree, dsfull[2], done, drain
    static constexpr int NBAR = 1 + 2 * NK + 2 * NV + 2 + 1 + 1 + 2 + 1 + 1;
    static constexpr int SMEM = 1024 + OFF_BAR + NBAR * 8 + 16;
    static constexpr int THREADS = 320;
    static constexpr int MMA_WARP = 8, TMA_WARP = 9;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_DP = 256, TM_DQ = 384;  // S buffer b at 128 b
    static constexpr uint32_t IDESC_SQ = idesc_bf16_f32(128, 128, false);
    static constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, D, true);
};

enum : unsigned int { W_Q_FIX = 112, W_Q_KFULL, W_Q_KEMPTY, W_Q_VFULL, W_Q_VEMPTY, W_Q_SFULL,
                      W_Q_DPFULL, W_Q_DPFREE, W_Q_DSFULL, W_Q_DONE, W_Q_DRAIN };

// grid: (T / 128 query blocks, B * H); causal: the highest query block sees
// the most keys and starts first.
template <int D>
__global__ void __launch_bounds__(DqCfg<D>::THREADS, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const BwdParams p)
{
    using C = DqCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t sQ = base + C::OFF_FIX, sG = sQ + C::TILE;
    const uint32_t sK = base + C::OFF_K, sV = base + C::OFF_V;
    const uint32_t b_fix = base + C::OFF_BAR;
    const uint32_t b_kfull = b_fix + 8, b_kempty = b_kfull + 8 * C::NK;
    const uint32_t b_vfull = b_kempty + 8 * C::NK, b_vempty = b_vfull + 8 * C::NV;
    const uint32_t b_sfull = b_vempty + 8 * C::NV;  // [2] S(n) in buffer n & 1
    const uint32_t b_dpfull = b_sfull + 16;         // dP(n) computed
    const uint32_t b_dpfree = b_dpfull + 8;         // both warpgroups hold dP(n) in registers
    const uint32_t b_dsfull = b_dpfree + 8;         // [2] dS(n) written over buffer n & 1
    const uint32_t b_done = b_dsfull + 16;
    const uint32_t b_drain = b_done + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + C::OFF_BAR + C::NBAR * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(b_fix, 1);
        for (int s = 0; s < C::NK; ++s) {
            mbar_init(b_kfull + 8 * s, 1);
            mbar_init(b_kempty + 8 * s, 1);
        }
        for (int s = 0; s < C::NV; ++s) {
            mbar_init(b_vfull + 8 * s, 1);
            mbar_init(b_vempty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(b_sfull + 8 * b, 1);
            mbar_init(b_dsfull + 8 * b, 256);
        }
        mbar_init(b_dpfull, 1);
        mbar_init(b_dpfree, 256);
        mbar_init(b_done, 1);
        mbar_init(b_drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint64_t lim = p.limit_ns;
    const int i = p.causal ? p.nq - 1 - (int)blockIdx.x : (int)blockIdx.x;
    const int bh = blockIdx.y;
    const int Hq = p.H_kv * p.group;
    const int kvbh = (bh / Hq) * p.H_kv + (bh % Hq) / p.group;
    const int nkb = p.causal ? i + 1 : p.nq;

    if (warp == C::TMA_WARP) {
        if (lane == 0) {  // TMA: Q_i, dO_i once; then K_0, V_0, K_1, V_1, K_2, ... (consumption order)
            const uint64_t pol = policy_evict_last();
            mbar_arrive_expect_tx(b_fix, 2 * C::TILE);
            for (int kb = 0; kb < C::KB; ++kb) {
                tma_load_3d(sQ + kb * C::SUB, &tmQ, b_fix, 64 * kb, 128 * i, bh, pol);
                tma_load_3d(sG + kb * C::SUB, &tmdO, b_fix, 64 * kb, 128 * i, bh, pol);
            }
            uint32_t karmed = 0, karmed_par = 0, varmed = 0, varmed_par = 0;
            bool ok = true;
            auto load = [&](bool is_k, int jj) -> bool {
                const int nsl = is_k ? C::NK : C::NV;
                const int s = jj % nsl;
                const uint32_t par = (uint32_t)(jj / nsl) & 1u;
                const uint32_t full = (is_k ? b_kfull : b_vfull) + 8 * s;
                if (!mbar_wait((is_k ? b_kempty : b_vempty) + 8 * s, par ^ 1u, lim,
                               is_k ? W_Q_KEMPTY : W_Q_VEMPTY, abort_flag))
                    return false;
                mbar_arrive_expect_tx(full, C::TILE);
                uint32_t &armed = is_k ? karmed : varmed, &apar = is_k ? karmed_par : varmed_par;
                armed |= 1u << s;
                apar = (apar & ~(1u << s)) | (par << s);
                const uint32_t dst = (is_k ? sK : sV) + s * C::TILE;
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_3d(dst + kb * C::SUB, is_k ? &tmK : &tmV, full, 64 * kb, 128 * jj, kvbh, pol);
                return true;
            };
            // the MMA warp takes K_0, V_0, K_1, then V_n before K_{n+1} for n >= 1
            ok = load(true, 0) && load(false, 0);
            if (ok && nkb > 1) ok = load(true, 1);
            for (int jj = 1; ok && jj < nkb; ++jj) {
                ok = load(false, jj);
                if (ok && jj + 1 < nkb) ok = load(true, jj + 1);
            }
            if (!ok) {
                *abort_flag = 1;
                mbar_wait(b_fix, 0, lim, W_Q_FIX);
                for (int s = 0; s < C::NK; ++s)
                    if ((karmed >> s) & 1u) mbar_wait(b_kfull + 8 * s, (karmed_par >> s) & 1u, lim, W_Q_KFULL);
                for (int s = 0; s < C::NV; ++s)
                    if ((varmed >> s) & 1u) mbar_wait(b_vfull + 8 * s, (varmed_par >> s) & 1u, lim, W_Q_VFULL);
            }
        }
    } else if (warp == C::MMA_WARP) {
        if (lane == 0) {  // MMA issuer
            bool ok = mbar_wait(b_fix, 0, lim, W_Q_FIX, abort_flag);
            tc_fence_after_sync();
            const uint32_t ql = sw128_desc_lo(sQ, 16), gl = sw128_desc_lo(sG, 16);
            auto wait_k = [&](int jj) {
                return mbar_wait(b_kfull + 8 * (jj % C::NK), (uint32_t)(jj / C::NK) & 1u, lim, W_Q_KFULL,
                                 abort_flag);
            };
            auto wait_v = [&](int jj) {
                return mbar_wait(b_vfull + 8 * (jj % C::NV), (uint32_t)(jj / C::NV) & 1u, lim, W_Q_VFULL,
                                 abort_flag);
            };
            auto s_mma = [&](int jj) {  // S(jj) = Q K_jj^T into buffer jj & 1
                const uint32_t kl = sw128_desc_lo(sK + (jj % C::NK) * C::TILE, 16);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::SUB + (kk & 3) * 32) >> 4;
                    mma_ss(tmem + 128u * (jj & 1), sw128_desc_join(ql + off, 1024),
                           sw128_desc_join(kl + off, 1024), C::IDESC_SQ, kk > 0 ? 1u : 0u);
                }
                tc_commit(b_sfull + 8 * (jj & 1));
            };
            auto dp_mma = [&](int jj) {  // dP(jj) = dO V_jj^T
                const int vs = jj % C::NV;
                const uint32_t vl = sw128_desc_lo(sV + vs * C::TILE, 16);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::SUB + (kk & 3) * 32) >> 4;
                    mma_ss(tmem + C::TM_DP, sw128_desc_join(gl + off, 1024),
                           sw128_desc_join(vl + off, 1024), C::IDESC_SQ, kk > 0 ? 1u : 0u);
                }
                tc_commit(b_dpfull);
                tc_commit(b_vempty + 8 * vs);  // V_jj is free once dP(jj) has run
            };
            if (ok && (ok = wait_k(0))) { tc_fence_after_sync(); s_mma(0); }
            if (ok && (ok = wait_v(0))) { tc_fence_after_sync(); dp_mma(0); }
            if (ok && nkb > 1 && (ok = wait_k(1))) { tc_fence_after_sync(); s_mma(1); }
            for (int n = 0; ok && n < nkb; ++n) {
                if (n + 1 < nkb) {  // dP(n+1) once dP(n) is out of TMEM
                    if (!(ok = mbar_wait(b_dpfree, (uint32_t)n & 1u, lim, W_Q_DPFREE, abort_flag))) break;
                    if (!(ok = wait_v(n + 1))) break;
                    tc_fence_after_sync();
                    dp_mma(n + 1);
                }
                if (!(ok = mbar_wait(b_dsfull + 8 * (n & 1), (uint32_t)(n >> 1) & 1u, lim, W_Q_DSFULL,
                                     abort_flag)))
                    break;
                tc_fence_after_sync();
                // dQ += dS(n) K_n: keys [64h, 64h + 64) sit at columns 64h + [0, 32) as bf16 pairs
                const uint32_t km = sw128_desc_lo(sK + (n % C::NK) * C::TILE, C::SUB);
                const uint32_t tds = tmem + 128u * (n & 1);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + C::TM_DQ, tds + 64 * (kk >> 2) + 8 * (kk & 3),
                           sw128_desc_join(km + kk * (2048 >> 4), 1024), C::IDESC_ACC,
                           (n > 0 || kk > 0) ? 1u : 0u);
                tc_commit(b_kempty + 8 * (n % C::NK));  // K_n's last use
                if (n + 2 < nkb) {  // S(n+2) into the buffer dQ just read (in issue order)
                    if (!(ok = wait_k(n + 2))) break;
                    tc_fence_after_sync();
                    s_mma(n + 2);
                }
            }
            if (!ok) *abort_flag = 1;
            tc_commit(b_done);  // fires when every MMA issued above has completed
        }
    } else if (warp < 8) {  // elementwise warpgroup h: thread = query row, keys [64h, 64h + 64)
        const int h = warp >> 2;
        const int qr = (warp & 3) * 32 + lane;
        const int row = 128 * i + qr;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const float2 st = p.stats[(size_t)bh * p.Tp + row];
        const float cl2 = p.c_log2;
        bool ok = true;
        for (int n = 0; ok && n < nkb; ++n) {
            bool w = mbar_wait(b_sfull + 8 * (n & 1), (uint32_t)(n >> 1) & 1u, lim, W_Q_SFULL, abort_flag);
            w = w && mbar_wait(b_dpfull, (uint32_t)n & 1u, lim, W_Q_DPFULL, abort_flag);
            if (!(ok = __all_sync(0xffffffffu, w))) break;
            tc_fence_after_sync();
            const uint32_t tS = tmem + lane_off + 128u * (n & 1) + 64 * h;
            const uint32_t tD = tmem + lane_off + C::TM_DP + 64 * h;
            uint32_t rs[64], rd[64];
            {
                uint32_t a[32], b2[32], c[32], d[32];
                tmem_ld32(tS, a);
                tmem_ld32(tS + 32, b2);
                tmem_ld32(tD, c);
                tmem_ld32(tD + 32, d);
                tmem_wait_ld_regs(a);
                tmem_wait_ld_regs(b2);
                tmem_wait_ld_regs(c);
                tmem_wait_ld_regs(d);
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    rs[x] = a[x];
                    rs[32 + x] = b2[x];
                    rd[x] = c[x];
                    rd[32 + x] = d[x];
                }
            }
            tc_fence_before_sync();
            mbar_arrive(b_dpfree);  // dP(n) is in registers: dP(n+1) may overwrite it
            const bool need_mask = p.causal && n == i;
            const int key0 = 128 * n + 64 * h;
            uint32_t dk[32];
#pragma unroll
            for (int q = 0; q < 64; q += 2) {
                float dsr[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float pv = fast_exp2(fmaf(__uint_as_float(rs[q + e]), cl2, -st.x));
                    if (need_mask && key0 + q + e > row) pv = 0.f;
                    dsr[e] = pv * (__uint_as_float(rd[q + e]) - st.y);
                }
                dk[q >> 1] = pack_bf16x2(dsr[0], dsr[1]);
            }
            tmem_st32(tS, dk);
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(b_dsfull + 8 * (n & 1));
        }
        const bool w = ok && mbar_wait(b_done, 0, lim, W_Q_DONE, abort_flag);
        if (__all_sync(0xffffffffu, w) && !*abort_flag) {
            tc_fence_after_sync();
            __nv_bfloat16 *dst = p.out_a + ((size_t)bh * p.T + row) * D;
            const bool real = row < p.T;  // padding rows of the last query block store nothing
            if (h == 0)  // the two warpgroups store the two halves of the d_h columns
                store_rows<0, D / 64>(tmem + lane_off + C::TM_DQ, p.scale, dst, real);
            else
                store_rows<D / 64, D / 32>(tmem + lane_off + C::TM_DQ, p.scale, dst, real);
        } else {
            *abort_flag = 1;
        }
    }
    if (warp == C::MMA_WARP && lane == 0 && *abort_flag) {
        tc_commit(b_drain);
        mbar_wait(b_drain, 0, lim, W_Q_DRAIN);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == C::MMA_WARP) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace attn
