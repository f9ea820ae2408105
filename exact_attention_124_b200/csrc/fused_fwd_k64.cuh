// fused_fwd_k64.cuh -- variant of the fused forward (fused_fwd.cuh) that walks
// the keys in tiles of 64 and double-buffers each query tile's score tile in
// TMEM.  Same arithmetic, same work units, same roles; what changes is the
// schedule ("Tiling and an incremental normalization": the tile sizes are a
// free choice of the method).
//
// With 128-key tiles, P_t is written over S_t and the next score MMA of a
// query tile can only start after P_t V has read it, so every softmax
// warpgroup waits for P V + Q K^T between two tiles.  With 64-key tiles two
// score buffers fit per query tile:
//   TMEM  tile t: S_t[0] / P_t[0] [128t, 128t + 64), S_t[1] / P_t[1]
//         [128t + 64, 128t + 128); O_t [256 + d_h t, 256 + d_h (t + 1))
// and the MMA warp issues, per key tile j,
//   P_t(j) V_j for both tiles, then S_t(j+2) = Q_t K_{j+2}^T into the buffer
//   P_t(j) V_j just read (the tensor pipe runs in issue order)
// so S_t(j+1) is computed while the softmax works on S_t(j).  The cost: the
// 64-wide score MMAs run at 2/3 of the 128-wide rate (they read 6 KB of
// shared memory per 16-deep step for half the work).
//
// Barriers whose waits could see two completions in flight are per buffer
// (sfull, pfull); the lazy O rescale at tile j waits for P_t(j-1) V on a
// per-tile barrier (only that one can be outstanding: P_t(j-2) V was issued
// before S_t(j), whose completion the softmax has seen); the epilogue waits
// on a barrier committed once per unit.
#pragma once

#include "fused_fwd.cuh"

namespace attn {

template <int D>
struct FusedK64Cfg {
    static_assert(D == 64 || D == 128, "d_h must be 64 or 128");
    static constexpr int KB = D / 64;
    static constexpr int SUBQ = 128 * 128;       // one 128-row x 128-byte block (Q)
    static constexpr int SUBK = 64 * 128;        // one 64-row x 128-byte block (K, V)
    static constexpr int TILEQ = 128 * D * 2;
    static constexpr int TILEK = 64 * D * 2;
    static constexpr int NSTAGE = (D == 64) ? 16 : 8;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = 2 * TILEQ;
    static constexpr int OFF_BAR = OFF_KV + NSTAGE * TILEK;
    // qfull[2] qempty[2] kvfull[N] kvempty[N] sfull[2][2] pfull[2][2] pvdone[2] pvlast[2] drain
    static constexpr int NBAR = 2 + 2 + 2 * NSTAGE + 4 + 4 + 2 + 2 + 1;
    static constexpr int SMEM = 1024 + OFF_BAR + NBAR * 8 + 16;
    static constexpr int THREADS = 384;
    static constexpr int REGS_LAUNCH = 168;
    static constexpr int REGS_CTRL = 88;
    static constexpr int REGS_SOFTMAX = 208;
    static_assert(128 * REGS_CTRL + 256 * REGS_SOFTMAX <= THREADS * REGS_LAUNCH,
                  "register split exceeds the launch's registers");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_O = 256;
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 64, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);
};

enum : unsigned int { W_K64_PVLAST = 32, W_K64_PVDONE };

// key tiles of 64 that query tile t of unit u sees (0 if the tile is past T)
__device__ __forceinline__ int k64_tiles(const FusedParams &p, const UnitInfo &u, int t)
{
    const int r0 = u.i0 + 128 * t;
    if (r0 >= p.T) return 0;
    const int nkv = (p.T + 63) >> 6;
    if (!p.causal) return nkv;
    const int n = (r0 + 127) / 64 + 1;
    return n < nkv ? n : nkv;
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_fused_k64_kernel(const __grid_constant__ CUtensorMap tmQ,
                              const __grid_constant__ CUtensorMap tmK,
                              const __grid_constant__ CUtensorMap tmV, const FusedParams p)
{
    using C = FusedK64Cfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);

    const uint32_t sQ = base + C::OFF_Q;
    const uint32_t sKV = base + C::OFF_KV;
    const uint32_t bar0 = base + C::OFF_BAR;
    const uint32_t b_qfull = bar0;                        // [2]
    const uint32_t b_qempty = bar0 + 16;                  // [2]
    const uint32_t b_kvfull = bar0 + 32;                  // [NSTAGE]
    const uint32_t b_kvempty = b_kvfull + 8 * C::NSTAGE;  // [NSTAGE]
    const uint32_t b_sfull = b_kvempty + 8 * C::NSTAGE;   // [tile][buffer]
    const uint32_t b_pfull = b_sfull + 32;                // [tile][buffer]
    const uint32_t b_pvdone = b_pfull + 32;               // [tile] every P V
    const uint32_t b_pvlast = b_pvdone + 16;              // [tile] a unit's last P V
    const uint32_t b_drain = b_pvlast + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + C::OFF_BAR + C::NBAR * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(b_qfull + 8 * t, 1);
            mbar_init(b_qempty + 8 * t, 1);
            for (int b = 0; b < 2; ++b) {
                mbar_init(b_sfull + 16 * t + 8 * b, 1);
                mbar_init(b_pfull + 16 * t + 8 * b, 128);
            }
            mbar_init(b_pvdone + 8 * t, 1);
            mbar_init(b_pvlast + 8 * t, 1);
        }
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(b_kvfull + 8 * s, 1);
            mbar_init(b_kvempty + 8 * s, 1);
        }
        mbar_init(b_drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 8) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 9 && lane == 0) {
        tma_prefetch_map(&tmQ);
        tma_prefetch_map(&tmK);
        tma_prefetch_map(&tmV);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint64_t lim = p.limit_ns;

    if (warp >= 8) {
      reg_dealloc<C::REGS_CTRL>();
      if (warp == 9) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_q = policy_evict_first();
            const uint64_t pol_kv = policy_evict_last();
            Ring ring;
            uint32_t qph[2] = {0u, 0u};
            uint32_t armed = 0u, armed_par = 0u;
            uint32_t q_armed = 0u, q_armed_par = 0u;
            bool ok = true;
            auto load_kv = [&](const CUtensorMap *map, int j, int bh) -> bool {
                const uint32_t s = ring.idx;
                if (!mbar_wait(b_kvempty + 8 * s, ring.phase ^ 1u, lim, W_KVEMPTY, abort_flag)) return false;
                mbar_arrive_expect_tx(b_kvfull + 8 * s, C::TILEK);
                armed |= 1u << s;
                armed_par = (armed_par & ~(1u << s)) | (ring.phase << s);
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_3d(sKV + s * C::TILEK + kb * C::SUBK, map, b_kvfull + 8 * s, 64 * kb,
                                64 * j, bh, pol_kv);
                ring.advance<C::NSTAGE>();
                return true;
            };
            for (int k = 0; ok; ++k) {
                UnitInfo u;
                const int r = unit_of(p, k, u);
                if (r < 0) break;
                if (r == 0) continue;
                if (*abort_flag) { ok = false; break; }
                const int n0 = k64_tiles(p, u, 0), n1 = k64_tiles(p, u, 1);
                const int niter = n0 > n1 ? n0 : n1;
#pragma unroll
                for (int t = 0; t < 2 && ok; ++t) {
                    if ((t == 0 ? n0 : n1) == 0) continue;
                    if (!mbar_wait(b_qempty + 8 * t, qph[t] ^ 1u, lim, W_QEMPTY, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(b_qfull + 8 * t, C::TILEQ);
                    q_armed |= 1u << t;
                    q_armed_par = (q_armed_par & ~(1u << t)) | (qph[t] << t);
#pragma unroll
                    for (int kb = 0; kb < C::KB; ++kb)
                        tma_load_3d(sQ + t * C::TILEQ + kb * C::SUBQ, &tmQ, b_qfull + 8 * t, 64 * kb,
                                    u.i0 + 128 * t, u.bh, pol_q);
                    qph[t] ^= 1u;
                }
                if (!ok) break;
                // consumption order: K_0, K_1, then V_j, K_{j+2} for j = 0, 1, ...
                ok = load_kv(&tmK, 0, u.kvh);
                if (ok && niter > 1) ok = load_kv(&tmK, 1, u.kvh);
                for (int j = 0; ok && j < niter; ++j) {
                    ok = load_kv(&tmV, j, u.kvh);
                    if (ok && j + 2 < niter) ok = load_kv(&tmK, j + 2, u.kvh);
                }
            }
            if (!ok) {
                *abort_flag = 1;
                for (int s = 0; s < C::NSTAGE; ++s)
                    if ((armed >> s) & 1u)
                        mbar_wait(b_kvfull + 8 * s, (armed_par >> s) & 1u, lim, W_KVFULL);
                for (int t = 0; t < 2; ++t)
                    if ((q_armed >> t) & 1u)
                        mbar_wait(b_qfull + 8 * t, (q_armed_par >> t) & 1u, lim, W_QFULL);
            }
        }
      } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            Ring ring;
            uint32_t qph[2] = {0u, 0u};
            uint32_t pph = 0u;  // bit 2t + b: phase of pfull[t][b]
            bool ok = true;
            auto next_kv = [&](uint32_t &slot) -> bool {
                slot = ring.idx;
                const bool r = mbar_wait(b_kvfull + 8 * slot, ring.phase, lim, W_KVFULL, abort_flag);
                ring.advance<C::NSTAGE>();
                tc_fence_after_sync();
                return r;
            };
            // S_t[b] = Q_t K^T (64 keys)
            auto qk = [&](int t, int b, uint32_t kslot) {
                const uint32_t qa = sw128_desc_lo(sQ + t * C::TILEQ, 16);
                const uint32_t ka = sw128_desc_lo(sKV + kslot * C::TILEK, 16);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t qo = ((kk >> 2) * C::SUBQ + (kk & 3) * 32) >> 4;
                    const uint32_t ko = ((kk >> 2) * C::SUBK + (kk & 3) * 32) >> 4;
                    mma_ss(tmem + 128u * t + 64u * b, sw128_desc_join(qa + qo, 1024),
                           sw128_desc_join(ka + ko, 1024), C::IDESC_QK, kk > 0 ? 1u : 0u);
                }
                tc_commit(b_sfull + 16 * t + 8 * b);
            };
            for (int k = 0; ok; ++k) {
                UnitInfo u;
                const int r = unit_of(p, k, u);
                if (r < 0) break;
                if (r == 0) continue;
                const int n[2] = {k64_tiles(p, u, 0), k64_tiles(p, u, 1)};
                const int niter = n[0] > n[1] ? n[0] : n[1];
#pragma unroll
                for (int t = 0; t < 2 && ok; ++t) {
                    if (n[t] == 0) continue;
                    ok = mbar_wait(b_qfull + 8 * t, qph[t], lim, W_QFULL, abort_flag);
                    qph[t] ^= 1u;
                }
                if (!ok) break;
                for (int j = 0; ok && j < 2 && j < niter; ++j) {  // S_t(0), S_t(1)
                    uint32_t ks;
                    if (!(ok = next_kv(ks))) break;
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        if (j >= n[t]) continue;
                        qk(t, j, ks);
                        if (j == n[t] - 1) tc_commit(b_qempty + 8 * t);
                    }
                    tc_commit(b_kvempty + 8 * ks);
                }
                for (int j = 0; ok && j < niter; ++j) {
                    const int b = j & 1;
                    uint32_t vs;
                    if (!(ok = next_kv(vs))) break;
                    const uint32_t va = sw128_desc_lo(sKV + vs * C::TILEK, C::SUBK);
#pragma unroll
                    for (int t = 0; t < 2; ++t) {  // O_t (+)= P_t(j) V_j
                        if (j >= n[t]) continue;
                        const uint32_t bit = 1u << (2 * t + b);
                        if (!(ok = mbar_wait(b_pfull + 16 * t + 8 * b, (pph & bit) ? 1u : 0u, lim, W_PFULL,
                                             abort_flag)))
                            break;
                        pph ^= bit;
                        tc_fence_after_sync();
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_ts(tmem + C::TM_O + D * t, tmem + 128u * t + 64u * b + 8 * kk,
                                   sw128_desc_join(va + kk * (2048 >> 4), 1024), C::IDESC_PV,
                                   (j > 0 || kk > 0) ? 1u : 0u);
                        tc_commit(b_pvdone + 8 * t);
                        if (j == n[t] - 1) tc_commit(b_pvlast + 8 * t);
                    }
                    if (!ok) break;
                    tc_commit(b_kvempty + 8 * vs);
                    if (j + 2 < niter) {  // S_t(j+2) into the buffer P_t(j) V just read
                        uint32_t ks;
                        if (!(ok = next_kv(ks))) break;
#pragma unroll
                        for (int t = 0; t < 2; ++t) {
                            if (j + 2 >= n[t]) continue;
                            qk(t, b, ks);
                            if (j + 2 == n[t] - 1) tc_commit(b_qempty + 8 * t);
                        }
                        tc_commit(b_kvempty + 8 * ks);
                    }
                }
            }
            if (!ok) {
                *abort_flag = 1;
                tc_commit(b_drain);
                mbar_wait(b_drain, 0, lim, W_DRAIN);
            }
        }
      }
    } else {
        // ------------------------------------------------------------ softmax warpgroups
        reg_alloc<C::REGS_SOFTMAX>();
        const int t = warp >> 2;
        const int wq = warp & 3;
        const int rit = wq * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t tO = tmem + lane_off + C::TM_O + D * t;
        const float cl2 = p.c_log2;
        uint32_t sph = 0u, lph = 0u;  // sph bit b: phase of sfull[t][b]; lph: pvlast[t]
        uint32_t pvbase = 0u;         // P V MMAs of this tile in earlier units
        bool ok = true;
        for (int k = 0; ok; ++k) {
            UnitInfo u;
            const int r = unit_of(p, k, u);
            if (r < 0) break;
            if (r == 0) continue;
            const int nt = k64_tiles(p, u, t);
            if (nt == 0) continue;
            const int r0 = u.i0 + 128 * t;
            const int row = r0 + rit;
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < nt; ++j) {
                const int b = j & 1;
                bool w = mbar_wait(b_sfull + 16 * t + 8 * b, (sph >> b) & 1u, lim, W_SFULL, abort_flag);
                if (!(ok = __all_sync(0xffffffffu, w))) break;
                sph ^= 1u << b;
                tc_fence_after_sync();
                const uint32_t tS = tmem + lane_off + 128u * t + 64u * b;
                float s[64];
                {
                    uint32_t ra[32], rb[32];
                    tmem_ld32(tS, ra);
                    tmem_ld32(tS + 32, rb);
                    tmem_wait_ld_regs(ra);
                    tmem_wait_ld_regs(rb);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        s[i] = __uint_as_float(ra[i]);
                        s[32 + i] = __uint_as_float(rb[i]);
                    }
                }
                const int key0 = 64 * j;
                const bool need_mask = (p.causal && key0 + 63 > r0) || (key0 + 64 > p.T);
                if (need_mask) {
                    const int lim_key = p.causal ? min(row, p.T - 1) : p.T - 1;
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (key0 + c > lim_key) s[c] = -INFINITY;
                }
                float mx[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) mx[i] = s[i];
#pragma unroll
                for (int c = 4; c < 60; c += 8) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) mx[i] = max3(mx[i], s[c + 2 * i], s[c + 2 * i + 1]);
                }
                const float cand = max3(max3(mx[0], mx[1], s[60]), max3(mx[2], mx[3], s[61]),
                                        fmaxf(s[62], s[63])) * cl2;
                float alpha = 1.f;
                bool resc = false;
                if (j == 0) {
                    m = cand;
                } else if (cand > m + RESCALE_TAU) {
                    alpha = fast_exp2(m - cand);
                    m = cand;
                    resc = true;
                }
                if (__any_sync(0xffffffffu, resc)) {
                    // O_t may still be accumulating P_t(j-1) V: wait for it
                    w = mbar_wait(b_pvdone + 8 * t, (pvbase + (uint32_t)j - 1u) & 1u, lim, W_K64_PVDONE,
                                  abort_flag);
                    if (!(ok = __all_sync(0xffffffffu, w))) break;
                    tc_fence_after_sync();
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t rr[32];
                        tmem_ld32(tO + 32 * c, rr);
                        tmem_wait_ld_regs(rr);
#pragma unroll
                        for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
                        tmem_st32(tO + 32 * c, rr);
                    }
                }
                l *= alpha;
                const float neg_m = (m == -INFINITY) ? 0.f : -m;
                const float2 c2 = make_float2(cl2, cl2), nm2 = make_float2(neg_m, neg_m);
                float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float2 x = __ffma2_rn(make_float2(s[2 * i], s[2 * i + 1]), c2, nm2);
                    const float2 pr = make_float2(fast_exp2(x.x), fast_exp2(x.y));
                    ls[i & 1] = __fadd2_rn(ls[i & 1], pr);
                    pk[i] = pack_bf16x2(pr.x, pr.y);
                }
                tmem_st32(tS, pk);
                tmem_wait_st();
                tc_fence_before_sync();
                mbar_arrive(b_pfull + 16 * t + 8 * b);
                l += (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y);
            }
            if (!ok) break;
            pvbase += (uint32_t)nt;
            // epilogue: O = acc / l, lse = (m + log2 l) ln 2
            bool w = mbar_wait(b_pvlast + 8 * t, lph, lim, W_K64_PVLAST, abort_flag);
            if (!(ok = __all_sync(0xffffffffu, w))) break;
            lph ^= 1u;
            tc_fence_after_sync();
            const float inv_l = 1.f / l;
            const size_t orow = (size_t)u.bh * (size_t)p.T + (size_t)row;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t rr[32];
                tmem_ld32(tO + 32 * c, rr);
                tmem_wait_ld_regs(rr);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(rr[2 * i]) * inv_l,
                                        __uint_as_float(rr[2 * i + 1]) * inv_l);
                if (row < p.T) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.o + orow * D + 32 * c);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
            if (row < p.T) p.lse[orow] = (m + fast_log2(l)) * 0.69314718055994530942f;
            tc_fence_before_sync();
        }
        if (!ok) *abort_flag = 1;
    }

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 8) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace attn
