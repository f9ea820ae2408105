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
//                     dQ += dS K in TMEM
// Warps: 0-3 elementwise (thread = TMEM lane = the stationary block's row),
// warp 4 issues MMAs, warp 5 issues TMA copies, warps 6-7 idle.
// TMEM: S/P [0,128), dP/dS [128,256), accumulators from 256.
#pragma once

#include "sm100.cuh"

namespace attn {

struct BwdParams {
    const float2 *stats;  // [B*H, T] (lse * log2 e, D)
    __nv_bfloat16 *out_a; // dkdv: dK [B*H_kv, T, D];  dq: dQ [B*H, T, D]
    __nv_bfloat16 *out_b; // dkdv: dV [B*H_kv, T, D]
    int H, H_kv, group, T, nq, causal;
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
    static constexpr int NBAR = 1 + 2 * NST + 4 + 1;
    static constexpr int SMEM = 1024 + OFF_BAR + NBAR * 8 + 16;
    static constexpr int THREADS = 256;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_ACC0 = 256, TM_ACC1 = 256 + D;
    static constexpr uint32_t IDESC_SQ = idesc_bf16_f32(128, 128, false);  // N = 128 rows of B
    static constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, D, true);    // B MN-major, N = d_h
};

// ---------------------------------------------------------------- preprocess
// stats[r] = (lse[r] * log2 e, sum_c dO[r][c] O[r][c]); one warp per row.
template <int D>
__global__ void __launch_bounds__(256)
    bwd_stats_kernel(const __nv_bfloat16 *__restrict__ O, const __nv_bfloat16 *__restrict__ dO,
                     const float *__restrict__ lse, float2 *__restrict__ stats, long long rows)
{
    const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    constexpr int PER = D / 32;  // bf16 values per lane: 4 (8 bytes) or 2 (4 bytes)
    const __nv_bfloat16 *o = O + r * D + lane * PER;
    const __nv_bfloat16 *g = dO + r * D + lane * PER;
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) acc = fmaf(__bfloat162float(o[i]), __bfloat162float(g[i]), acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) stats[r] = make_float2(lse[r] * 1.4426950408889634f, acc);
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
        b_sfull = b_empty + 8 * C::NST;
        b_pfull = b_sfull + 8;            // [2]: columns 0-63 / 64-127 written
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
        mbar_init(sm.b_sfull, 1);
        mbar_init(sm.b_pfull, 128);
        mbar_init(sm.b_pfull + 8, 128);
        mbar_init(sm.b_done, 1);
        mbar_init(sm.b_drain, 1);
        *sm.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 4) {
        tmem_alloc(smem_addr(sm.tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    return *sm.tmem_slot;
}

// Elementwise step of both kernels on one 128 x 128 block, one row per
// thread, 32 columns at a time: p = 2^(s c - lse2) (0 where masked) and
// ds = p (dp - D).  With WRITE_P, P (bf16 pairs) goes over the first 64 S
// columns; dS goes to tDS (over the dP columns in the dK/dV kernel, over the
// S columns in the dQ kernel).  Chunk c writes columns [16c, 16c + 16), all of
// which earlier chunks (or this one) have already read.  PER_COLUMN: rows are
// keys and the statistics come per query column from shared memory; else rows
// are queries and the row's own statistics are st_row.  Each half of the
// columns is signalled on its own barrier (b_half, b_half + 8) as soon as it
// is in TMEM, so the MMAs that consume it can start.
template <bool PER_COLUMN, bool WRITE_P>
__device__ __forceinline__ void bwd_elementwise(uint32_t tS, uint32_t tDP, float cl2,
                                                const float2 *st_col, float2 st_row,
                                                bool need_mask, int row_idx, int col0,
                                                uint32_t tDS, uint32_t b_half)
{
#pragma unroll
    for (int c = 0; c < 4; ++c) {
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
        if (c & 1) {  // columns [0, 64) after chunk 1, [64, 128) after chunk 3
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(b_half + 8 * (c >> 1));
        }
    }
}

// Epilogue: rows of a TMEM accumulator (D fp32 columns) times `mul`, as bf16.
template <int D>
__device__ __forceinline__ void store_rows(uint32_t tacc, float mul, __nv_bfloat16 *dst)
{
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tacc + 32 * c, r);
        tmem_wait_ld_regs(r);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * mul, __uint_as_float(r[2 * i + 1]) * mul);
        uint4 *d4 = reinterpret_cast<uint4 *>(dst + 32 * c);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    }
}

// ---------------------------------------------------------------- dK, dV
// grid: (T / 128 key blocks, B * H_kv); key block j = blockIdx.x (causal:
// the lowest keys see the most queries, so the longest CTAs start first).
template <int D>
__global__ void __launch_bounds__(256, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const BwdParams p)
{
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

    if (warp == 5) {
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
                bulk_load(st + 2 * C::TILE, p.stats + (size_t)bh * p.T + 128 * i, 1024,
                          sm.b_full + 8 * s);
            }
            if (!ok) {
                *sm.abort_flag = 1;
                mbar_wait(sm.b_fix, 0, lim, W_B_KV);
                for (int s = 0; s < C::NST; ++s)
                    if ((armed >> s) & 1u) mbar_wait(sm.b_full + 8 * s, (armed_par >> s) & 1u, lim, W_B_STFULL);
            }
        }
    } else if (warp == 4) {
        if (lane == 0) {  // MMA issuer
            bool ok = mbar_wait(sm.b_fix, 0, lim, W_B_KV, sm.abort_flag);
            tc_fence_after_sync();
            const uint32_t kl = sw128_desc_lo(sK, 16), vl = sw128_desc_lo(sV, 16);
            for (int n = 0; ok && n < niter; ++n) {
                const int s = n % C::NST;
                const uint32_t par = (uint32_t)(n / C::NST) & 1u;
                if (!(ok = mbar_wait(sm.b_full + 8 * s, par, lim, W_B_STFULL, sm.abort_flag))) break;
                tc_fence_after_sync();
                const uint32_t st = sm.ring + s * C::STAGE;
                const uint32_t ql = sw128_desc_lo(st, 16), gl = sw128_desc_lo(st + C::TILE, 16);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {  // S^T = K Q^T, dP^T = V dO^T
                    const uint32_t off = ((kk >> 2) * C::SUB + (kk & 3) * 32) >> 4;
                    mma_ss(tmem + C::TM_S, sw128_desc_join(kl + off, 1024),
                           sw128_desc_join(ql + off, 1024), C::IDESC_SQ, kk > 0 ? 1u : 0u);
                    mma_ss(tmem + C::TM_DP, sw128_desc_join(vl + off, 1024),
                           sw128_desc_join(gl + off, 1024), C::IDESC_SQ, kk > 0 ? 1u : 0u);
                }
                tc_commit(sm.b_sfull);
                const uint32_t qm = sw128_desc_lo(st, C::SUB), gm = sw128_desc_lo(st + C::TILE, C::SUB);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {  // each half of the queries as soon as it is ready
                    if (!(ok = mbar_wait(sm.b_pfull + 8 * hh, (uint32_t)n & 1u, lim, W_B_PFULL,
                                         sm.abort_flag)))
                        break;
                    tc_fence_after_sync();
#pragma unroll
                    for (int kk = 4 * hh; kk < 4 * hh + 4; ++kk) {  // dV += P^T dO, dK += dS^T Q
                        const uint32_t acc = (n > 0 || kk > 0) ? 1u : 0u;
                        mma_ts(tmem + C::TM_ACC0, tmem + C::TM_S + 8 * kk,
                               sw128_desc_join(gm + kk * (2048 >> 4), 1024), C::IDESC_ACC, acc);
                        mma_ts(tmem + C::TM_ACC1, tmem + C::TM_DP + 8 * kk,
                               sw128_desc_join(qm + kk * (2048 >> 4), 1024), C::IDESC_ACC, acc);
                    }
                }
                if (!ok) break;
                tc_commit(sm.b_empty + 8 * s);
            }
            if (!ok) *sm.abort_flag = 1;
            tc_commit(sm.b_done);  // fires when every MMA issued above has completed
        }
    } else if (warp < 4) {  // elementwise: thread = key row
        const int kr = warp * 32 + lane;
        const int key = 128 * j + kr;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        bool ok = true;
        for (int n = 0; ok && n < niter; ++n) {
            const int s = n % C::NST;
            const uint32_t par = (uint32_t)(n / C::NST) & 1u;
            const int i = i0 + n % per_head;
            bool w = mbar_wait(sm.b_full + 8 * s, par, lim, W_B_STFULL, sm.abort_flag);
            w = w && mbar_wait(sm.b_sfull, (uint32_t)n & 1u, lim, W_B_SFULL, sm.abort_flag);
            if (!(ok = __all_sync(0xffffffffu, w))) break;
            tc_fence_after_sync();
            const float2 *stc =
                reinterpret_cast<const float2 *>(sm.gbase + C::OFF_RING + s * C::STAGE + 2 * C::TILE);
            const bool need_mask = p.causal && i == j;
            bwd_elementwise<true, true>(tmem + lane_off + C::TM_S, tmem + lane_off + C::TM_DP,
                                        p.c_log2, stc, make_float2(0.f, 0.f), need_mask, key,
                                        128 * i, tmem + lane_off + C::TM_DP, sm.b_pfull);
        }
        const bool w = ok && mbar_wait(sm.b_done, 0, lim, W_B_DONE, sm.abort_flag);
        if (__all_sync(0xffffffffu, w) && !*sm.abort_flag) {
            tc_fence_after_sync();
            const size_t orow = ((size_t)kvbh * p.T + key) * D;
            store_rows<D>(tmem + lane_off + C::TM_ACC1, p.scale, p.out_a + orow);  // dK
            store_rows<D>(tmem + lane_off + C::TM_ACC0, 1.f, p.out_b + orow);      // dV
        } else {
            *sm.abort_flag = 1;
        }
    }
    if (warp == 4 && lane == 0 && *sm.abort_flag) {
        tc_commit(sm.b_drain);
        mbar_wait(sm.b_drain, 0, lim, W_B_DRAIN);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 4) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ---------------------------------------------------------------- dQ
// grid: (T / 128 query blocks, B * H); causal: the highest query block sees
// the most keys and starts first.
template <int D>
__global__ void __launch_bounds__(256, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const BwdParams p)
{
    using C = BwdCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    BwdSmem<D> sm;
    sm.init(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t tmem = bwd_setup<D>(sm, warp);
    const uint64_t lim = p.limit_ns;
    const int i = p.causal ? p.nq - 1 - (int)blockIdx.x : (int)blockIdx.x;
    const int bh = blockIdx.y;
    const int Hq = p.H_kv * p.group;
    const int kvbh = (bh / Hq) * p.H_kv + (bh % Hq) / p.group;
    const int nkb = p.causal ? i + 1 : p.nq;
    const uint32_t sQ = sm.fix, sG = sm.fix + C::TILE;

    if (warp == 5) {
        if (lane == 0) {  // TMA: Q_i, dO_i once; then K_j, V_j per iteration
            const uint64_t pol = policy_evict_last();
            mbar_arrive_expect_tx(sm.b_fix, 2 * C::TILE);
            for (int kb = 0; kb < C::KB; ++kb) {
                tma_load_3d(sQ + kb * C::SUB, &tmQ, sm.b_fix, 64 * kb, 128 * i, bh, pol);
                tma_load_3d(sG + kb * C::SUB, &tmdO, sm.b_fix, 64 * kb, 128 * i, bh, pol);
            }
            uint32_t armed = 0, armed_par = 0;
            bool ok = true;
            for (int jj = 0; jj < nkb; ++jj) {
                const int s = jj % C::NST;
                const uint32_t par = (uint32_t)(jj / C::NST) & 1u;
                if (!mbar_wait(sm.b_empty + 8 * s, par ^ 1u, lim, W_B_STEMPTY, sm.abort_flag)) {
                    ok = false;
                    break;
                }
                const uint32_t st = sm.ring + s * C::STAGE;
                mbar_arrive_expect_tx(sm.b_full + 8 * s, 2 * C::TILE);
                armed |= 1u << s;
                armed_par = (armed_par & ~(1u << s)) | (par << s);
                for (int kb = 0; kb < C::KB; ++kb) {
                    tma_load_3d(st + kb * C::SUB, &tmK, sm.b_full + 8 * s, 64 * kb, 128 * jj, kvbh, pol);
                    tma_load_3d(st + C::TILE + kb * C::SUB, &tmV, sm.b_full + 8 * s, 64 * kb,
                                128 * jj, kvbh, pol);
                }
            }
            if (!ok) {
                *sm.abort_flag = 1;
                mbar_wait(sm.b_fix, 0, lim, W_B_KV);
                for (int s = 0; s < C::NST; ++s)
                    if ((armed >> s) & 1u) mbar_wait(sm.b_full + 8 * s, (armed_par >> s) & 1u, lim, W_B_STFULL);
            }
        }
    } else if (warp == 4) {
        if (lane == 0) {  // MMA issuer
            bool ok = mbar_wait(sm.b_fix, 0, lim, W_B_KV, sm.abort_flag);
            tc_fence_after_sync();
            const uint32_t ql = sw128_desc_lo(sQ, 16), gl = sw128_desc_lo(sG, 16);
            for (int jj = 0; ok && jj < nkb; ++jj) {
                const int s = jj % C::NST;
                const uint32_t par = (uint32_t)(jj / C::NST) & 1u;
                if (!(ok = mbar_wait(sm.b_full + 8 * s, par, lim, W_B_STFULL, sm.abort_flag))) break;
                tc_fence_after_sync();
                const uint32_t st = sm.ring + s * C::STAGE;
                const uint32_t kl = sw128_desc_lo(st, 16), vl = sw128_desc_lo(st + C::TILE, 16);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {  // S = Q K^T, dP = dO V^T
                    const uint32_t off = ((kk >> 2) * C::SUB + (kk & 3) * 32) >> 4;
                    mma_ss(tmem + C::TM_S, sw128_desc_join(ql + off, 1024),
                           sw128_desc_join(kl + off, 1024), C::IDESC_SQ, kk > 0 ? 1u : 0u);
                    mma_ss(tmem + C::TM_DP, sw128_desc_join(gl + off, 1024),
                           sw128_desc_join(vl + off, 1024), C::IDESC_SQ, kk > 0 ? 1u : 0u);
                }
                tc_commit(sm.b_sfull);
                const uint32_t km = sw128_desc_lo(st, C::SUB);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {  // each half of the keys as soon as it is ready
                    if (!(ok = mbar_wait(sm.b_pfull + 8 * hh, (uint32_t)jj & 1u, lim, W_B_PFULL,
                                         sm.abort_flag)))
                        break;
                    tc_fence_after_sync();
#pragma unroll
                    for (int kk = 4 * hh; kk < 4 * hh + 4; ++kk)  // dQ += dS K (16 keys each)
                        mma_ts(tmem + C::TM_ACC0, tmem + C::TM_S + 8 * kk,
                               sw128_desc_join(km + kk * (2048 >> 4), 1024), C::IDESC_ACC,
                               (jj > 0 || kk > 0) ? 1u : 0u);
                }
                if (!ok) break;
                tc_commit(sm.b_empty + 8 * s);
            }
            if (!ok) *sm.abort_flag = 1;
            tc_commit(sm.b_done);
        }
    } else if (warp < 4) {  // elementwise: thread = query row
        const int qr = warp * 32 + lane;
        const int row = 128 * i + qr;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const float2 st_row = p.stats[(size_t)bh * p.T + row];
        bool ok = true;
        for (int jj = 0; ok && jj < nkb; ++jj) {
            const bool w = mbar_wait(sm.b_sfull, (uint32_t)jj & 1u, lim, W_B_SFULL, sm.abort_flag);
            if (!(ok = __all_sync(0xffffffffu, w))) break;
            tc_fence_after_sync();
            const bool need_mask = p.causal && jj == i;
            bwd_elementwise<false, false>(tmem + lane_off + C::TM_S, tmem + lane_off + C::TM_DP,
                                          p.c_log2, nullptr, st_row, need_mask, row, 128 * jj,
                                          tmem + lane_off + C::TM_S, sm.b_pfull);
        }
        const bool w = ok && mbar_wait(sm.b_done, 0, lim, W_B_DONE, sm.abort_flag);
        if (__all_sync(0xffffffffu, w) && !*sm.abort_flag) {
            tc_fence_after_sync();
            store_rows<D>(tmem + lane_off + C::TM_ACC0, p.scale, p.out_a + ((size_t)bh * p.T + row) * D);
        } else {
            *sm.abort_flag = 1;
        }
    }
    if (warp == 4 && lane == 0 && *sm.abort_flag) {
        tc_commit(sm.b_drain);
        mbar_wait(sm.b_drain, 0, lim, W_B_DRAIN);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 4) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace attn
