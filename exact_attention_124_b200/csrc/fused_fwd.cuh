// fused_fwd.cuh -- fused exact attention forward for B200 (sm_100a).
//
// What it computes (per head, Q/K/V of T x d_h): O = softmax(mask(scale*QK^T)) V
// and the row log-sum-exp, as defined in "Why Attention Is Difficult to
// Optimize" ("The Attention Computation Flow") and "Attention Mechanism:
// Computation & Memory Patterns" (section 1).  How: the IO-aware form of that
// page's section 3 -- Q/K/V tiles staged on chip, each score tile scaled and
// causally masked in place from query/key indices ("From a Score Tile to
// Probabilities"), and an online softmax that carries a running maximum, a
// running normaliser and a consistently rescaled P.V accumulator ("FlashAttention
// -- avoid writing the giant intermediate", "Tiling and an incremental
// normalization").  The T x T matrices S and P never leave the SM: S lives in
// tensor memory (TMEM), P is written back over it as bf16 and read from there
// by the second MMA.
//
// B200 mapping (one persistent CTA per SM, 384 threads = 3 warpgroups):
//   warps 0-3  softmax warpgroup for query tile 0 (thread = query row = TMEM lane)
//   warps 4-7  softmax warpgroup for query tile 1 (the two tiles ping-pong, so one
//              tile's exponentials overlap the other tile's MMAs)
//   warp 8     MMA issuer (one thread): tcgen05.mma S_t = Q_t K_j^T (smem x smem)
//              and O_t += P_t V_j (tmem x smem); allocates/frees TMEM
//   warp 9     TMA producer (one thread): Q tiles, then K_j / V_j into an
//              NSTAGE-deep shared-memory ring, in the order the MMA consumes them
//   warps 10-11 idle (they complete the third warpgroup, whose registers
//              setmaxnreg hands to the softmax warpgroups)
// A work unit is (head, 256 query rows).  Causal: query block q of a head is
// paired with block nqb-1-q, so every pair costs the same; pairs are dealt
// round-robin to CTAs in head-major order, so the CTAs running at one time
// share a few heads' K/V through L2.  Non-causal: units head-major.
// Grouped-query attention: query head h of batch entry b reads K/V head
// b * (H / group) + h / group; the head-major order keeps a group's query
// heads on neighbouring CTAs, which then share that K/V head through L2.
//
// TMEM (512 columns x 128 lanes x 32 bit):
//   S_0 / P_0 : columns [0, 128)     S_1 / P_1 : [128, 256)
//   O_0       : [256, 256 + d_h)     O_1       : [256 + d_h, 256 + 2 d_h)
// Online softmax in the log2 domain: s2 = s * scale * log2(e); the running
// maximum m only moves when a row's new maximum exceeds it by more than
// RESCALE_TAU = 32, so the O rescale (a TMEM read-modify-write of the whole
// warp's rows, done when any of its 32 rows needs it) is rare; the final
// O = acc / l and lse = (m + log2 l) ln 2 are exact for any m, stale or not.
// A stale m only makes the weights larger, p <= 2^32: far inside the range of
// bf16 P and of the fp32 O and l (2^32 x 2^31 keys x |v| < 2^127), and
// floating point keeps its relative precision at any scale.
#pragma once

#include "sm100.cuh"

namespace attn {

constexpr float RESCALE_TAU = 32.0f;

// 2^x on the FMA pipe for two values at once (x <= RESCALE_TAU).  Range
// reduction x = n + f, n = round(x) (adding 1.5 * 2^23 rounds to an integer in
// the low mantissa bits, |n| < 256), f in [-1/2, 1/2]; 2^f by a degree-3 polynomial whose
// coefficients minimise the maximum relative error on [-1/2, 1/2] (Remez
// exchange, computed by gen_exp2_poly.py next to this file; max relative
// error 7.5e-5, far below the bf16 rounding of P); 2^n by adding n to the
// exponent field.  x is clamped to -125 first so the result stays a normal
// number (anything that small is negligible next to the row's terms >= 2^-8).
constexpr float EXP2_C0 = 0.99992806f;
constexpr float EXP2_C1 = 0.69326097f;
constexpr float EXP2_C2 = 0.24261113f;
constexpr float EXP2_C3 = 0.05517167f;

__device__ __forceinline__ float2 exp2_poly2(float2 x)
{
    x.x = fmaxf(x.x, -125.f);
    x.y = fmaxf(x.y, -125.f);
    const float2 t = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));   // 1.5 * 2^23 + n
    const float2 n = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f)); // n, exactly
    const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);            // x - n, exactly
    float2 q = __ffma2_rn(make_float2(EXP2_C3, EXP2_C3), f, make_float2(EXP2_C2, EXP2_C2));
    q = __ffma2_rn(q, f, make_float2(EXP2_C1, EXP2_C1));
    q = __ffma2_rn(q, f, make_float2(EXP2_C0, EXP2_C0));
    // the low 9 bits of t's pattern hold n (two's complement): shift them into
    // the exponent field and add
    const uint32_t ex = __float_as_uint(t.x) << 23, ey = __float_as_uint(t.y) << 23;
    return make_float2(__uint_as_float(__float_as_uint(q.x) + ex),
                       __uint_as_float(__float_as_uint(q.y) + ey));
}

// Which of every 8 consecutive column pairs go to the FMA pipe: the EMU pairs
// spread evenly over the 8 (EMU = 0 .. 8).
template <int EMU>
__device__ __forceinline__ constexpr bool emu_pair(int i)
{
    return ((i & 7) * EMU) % 8 + EMU >= 8;
}

struct FusedParams {
    __nv_bfloat16 *o;
    float *lse;
    int BH;        // query heads B * H
    int H;         // query heads per batch entry
    int group;     // query heads per K/V head (1 = multi-head, H = multi-query)
    int T;
    int causal;
    float c_log2;  // scale * log2(e)
    int nqb;       // query blocks of 256 rows per head
    int units;     // BH * nqb
    int nkv;       // key/value tiles of 128 per head
    int order_mode;
    unsigned long long limit_ns;
};

template <int D>
struct FusedCfg {
    static_assert(D == 64 || D == 128, "d_h must be 64 or 128");
    static constexpr int BM = 128;                 // query rows per tile (TMEM lanes)
    static constexpr int BN = 128;                 // keys per K/V tile
    static constexpr int KB = D / 64;              // 128-byte column blocks per row
    static constexpr int SUB = 128 * 128;          // one 128-row x 128-byte block
    static constexpr int TILE = BN * D * 2;        // bytes of one Q, K or V tile
    static constexpr int NSTAGE = (D == 64) ? 8 : 4;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = 2 * TILE;
    static constexpr int OFF_BAR = OFF_KV + NSTAGE * TILE;
    static constexpr int NBAR = 2 + 2 + 2 * NSTAGE + 2 + 4 + 2 + 1;
    static constexpr int SMEM = 1024 + OFF_BAR + NBAR * 8 + 16;
    // non-causal instance: O staged through 4 KB per softmax warp, after the barriers
    static constexpr int OFF_EPI = (OFF_BAR + NBAR * 8 + 16 + 1023) / 1024 * 1024;
    static constexpr int SMEM_NC = 1024 + OFF_EPI + 8 * 4096;
    static constexpr int THREADS = 384;
    // setmaxnreg split: the launch gets 168 registers per thread (384 x 168 =
    // 64512); the control warpgroup gives back down to 88, the two softmax
    // warpgroups take 208: 128 x 88 + 256 x 208 = 64512.
    static constexpr int REGS_LAUNCH = 168;
    static constexpr int REGS_CTRL = 88;
    static constexpr int REGS_SOFTMAX = 208;
    static_assert(128 * REGS_CTRL + 256 * REGS_SOFTMAX <= THREADS * REGS_LAUNCH,
                  "register split exceeds the launch's registers");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_S = 0;            // + 128 * t
    static constexpr uint32_t TM_O = 256;          // + D * t
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);
};

// Wait codes recorded with a timeout (which barrier gave up).
enum : unsigned int {
    W_QFULL = 1, W_QEMPTY, W_KVFULL, W_KVEMPTY, W_SFULL, W_PFULL, W_PVDONE, W_DRAIN
};

// Row maximum of 128 scores: eight independent running maxima (two new
// columns each per step), then a short tree.
__device__ __forceinline__ float row_max(const float (&s)[128])
{
    float mx[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) mx[i] = s[i];
#pragma unroll
    for (int c = 8; c < 120; c += 16) {  // columns 8 .. 119
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = max3(mx[i], s[c + 2 * i], s[c + 2 * i + 1]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) mx[i] = max3(mx[i], s[120 + 2 * i], s[121 + 2 * i]);
    return max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
}

// p = 2^(s * c - m) for column pairs P0 .. P0+NP-1, packed to bf16 pairs in pk;
// the fp32 p are summed into ls (two packed accumulators).
template <int EMU, int P0, int NP, int N>
__device__ __forceinline__ void exp_pairs(const float (&s)[N], float2 c2, float2 nm2,
                                          uint32_t (&pk)[NP], float2 (&ls)[2])
{
    static_assert(2 * (P0 + NP) <= N, "pairs past the array");
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        const int pi = P0 + i;
        const float2 x = __ffma2_rn(make_float2(s[2 * pi], s[2 * pi + 1]), c2, nm2);
        float2 pr;
        if (emu_pair<EMU>(pi)) {
            pr = exp2_poly2(x);
        } else {
            pr.x = fast_exp2(x.x);
            pr.y = fast_exp2(x.y);
        }
        ls[i & 1] = __fadd2_rn(ls[i & 1], pr);
        pk[i] = pack_bf16x2(pr.x, pr.y);
    }
}

struct UnitInfo {
    int bh, kvh, i0;  // query head, its K/V head, first query row
    int n[2];
    int niter;
};

// Pairs per head in causal mode (query block q with nqb-1-q).
__host__ __device__ __forceinline__ int pairs_per_head(const FusedParams &p) { return (p.nqb + 1) >> 1; }

// The k-th unit of CTA c of a grid of G CTAs.  Returns 1 with `u` filled, 0
// for a hole (the middle block of an odd nqb appears once per pair list), -1
// when the CTA has no more work.  Every role of the CTA walks the same
// sequence.  Also run on the host by attn_selftest_fused_plan().
__host__ __device__ __forceinline__ int unit_of_cta(const FusedParams &p, int G, int c, int k,
                                                    UnitInfo &u)
{
    int qb;
    if (p.causal) {
        const int npp = pairs_per_head(p);
        const int pid = c + G * (k >> 1);   // < BH * npp + G < 2^31 (host-checked sizes)
        if (pid >= p.BH * npp) return -1;
        u.bh = pid / npp;
        const int pp = pid - u.bh * npp;
        if ((k & 1) == 0) {
            qb = p.nqb - 1 - pp;
        } else {
            qb = pp;
            if (qb == p.nqb - 1 - pp) return 0;
        }
    } else {
        const int pid = c + G * k;
        if (pid >= p.units) return -1;
        u.bh = pid / p.nqb;
        qb = pid - u.bh * p.nqb;
    }
    u.kvh = (u.bh / p.H) * (p.H / p.group) + (u.bh % p.H) / p.group;
    u.i0 = qb * 256;
    const int r1 = u.i0 + 128;
    if (p.causal) {
        const int l0 = r1 / 128;           // = i0/128 + 1
        u.n[0] = l0 < p.nkv ? l0 : p.nkv;
        u.n[1] = r1 >= p.T ? 0 : (l0 + 1 < p.nkv ? l0 + 1 : p.nkv);
    } else {
        u.n[0] = p.nkv;
        u.n[1] = r1 >= p.T ? 0 : p.nkv;
    }
    u.niter = u.n[0] > u.n[1] ? u.n[0] : u.n[1];
    return 1;
}

__device__ __forceinline__ int unit_of(const FusedParams &p, int k, UnitInfo &u)
{
    return unit_of_cta(p, (int)gridDim.x, (int)blockIdx.x, k, u);
}

struct Ring {
    uint32_t idx = 0, phase = 0;
    template <int N>
    __device__ __forceinline__ void advance()
    {
        if (++idx == (uint32_t)N) {
            idx = 0;
            phase ^= 1u;
        }
    }
};

template <int D, int EMU, bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_fused_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const FusedParams p)
{
    using C = FusedCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzled tiles
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);

    const uint32_t sQ = base + C::OFF_Q;
    const uint32_t sKV = base + C::OFF_KV;
    const uint32_t bar0 = base + C::OFF_BAR;
    const uint32_t b_qfull = bar0;                          // [2]
    const uint32_t b_qempty = bar0 + 16;                    // [2]
    const uint32_t b_kvfull = bar0 + 32;                    // [NSTAGE]
    const uint32_t b_kvempty = b_kvfull + 8 * C::NSTAGE;    // [NSTAGE]
    const uint32_t b_sfull = b_kvempty + 8 * C::NSTAGE;     // [2]
    const uint32_t b_pfull = b_sfull + 16;                  // [2 tiles][2 halves]
    const uint32_t b_pvdone = b_pfull + 32;                 // [2]
    const uint32_t b_drain = b_pvdone + 16;                 // [1]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + C::OFF_BAR + C::NBAR * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(b_qfull, 1);
        mbar_init(b_qfull + 8, 1);
        mbar_init(b_qempty, 1);
        mbar_init(b_qempty + 8, 1);
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(b_kvfull + 8 * s, 1);
            mbar_init(b_kvempty + 8 * s, 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(b_sfull + 8 * t, 1);
            mbar_init(b_pfull + 16 * t, 128);      // keys 0-63 of P_t written
            mbar_init(b_pfull + 16 * t + 8, 128);  // keys 64-127 of P_t written
            mbar_init(b_pvdone + 8 * t, 1);
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
            uint32_t armed = 0u, armed_par = 0u;      // bit s: slot s has a load in flight / its parity
            uint32_t q_armed = 0u, q_armed_par = 0u;  // bit t: same for the Q tiles
            bool ok = true;
            auto load_kv = [&](const CUtensorMap *map, int j, int bh) -> bool {
                const uint32_t s = ring.idx;
                if (!mbar_wait(b_kvempty + 8 * s, ring.phase ^ 1u, lim, W_KVEMPTY, abort_flag)) return false;
                mbar_arrive_expect_tx(b_kvfull + 8 * s, C::TILE);
                armed |= 1u << s;
                armed_par = (armed_par & ~(1u << s)) | (ring.phase << s);
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_3d(sKV + s * C::TILE + kb * C::SUB, map, b_kvfull + 8 * s, 64 * kb,
                                128 * j, bh, pol_kv);
                ring.advance<C::NSTAGE>();
                return true;
            };
            for (int k = 0; ok; ++k) {
                UnitInfo u;
                const int r = unit_of(p, k, u);
                if (r < 0) break;
                if (r == 0) continue;
                if (*abort_flag) { ok = false; break; }
                #pragma unroll
                for (int t = 0; t < 2 && ok; ++t) {
                    if (u.n[t] == 0) continue;
                    if (!mbar_wait(b_qempty + 8 * t, qph[t] ^ 1u, lim, W_QEMPTY, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(b_qfull + 8 * t, C::TILE);
                    q_armed |= 1u << t;
                    q_armed_par = (q_armed_par & ~(1u << t)) | (qph[t] << t);
#pragma unroll
                    for (int kb = 0; kb < C::KB; ++kb)
                        tma_load_3d(sQ + t * C::TILE + kb * C::SUB, &tmQ, b_qfull + 8 * t, 64 * kb,
                                    u.i0 + 128 * t, u.bh, pol_q);
                    qph[t] ^= 1u;
                }
                if (!ok) break;
                ok = load_kv(&tmK, 0, u.kvh);
                for (int j = 1; ok && j < u.niter; ++j) {
                    ok = load_kv(&tmK, j, u.kvh);
                    if (ok) ok = load_kv(&tmV, j - 1, u.kvh);
                }
                if (ok) ok = load_kv(&tmV, u.niter - 1, u.kvh);
            }
            if (!ok) {
                *abort_flag = 1;
                // let every copy still in flight land before the CTA exits
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
            uint32_t pph[2] = {0u, 0u};
            uint32_t drain_ph = 0;
            bool issued_any = false;
            bool ok = true;
            const uint32_t tS[2] = {tmem + C::TM_S, tmem + C::TM_S + 128};
            const uint32_t tO[2] = {tmem + C::TM_O, tmem + C::TM_O + D};

            auto drain = [&]() -> bool {  // wait for every MMA issued so far
                tc_commit(b_drain);
                const bool r = mbar_wait(b_drain, drain_ph, lim, W_DRAIN);
                drain_ph ^= 1u;
                return r;
            };
            // descriptor low words advance by (byte offset >> 4); high words are fixed
            auto qk = [&](int t, uint32_t kslot) {
                const uint32_t qa = sw128_desc_lo(sQ + t * C::TILE, 16);
                const uint32_t ka = sw128_desc_lo(sKV + kslot * C::TILE, 16);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::SUB + (kk & 3) * 32) >> 4;
                    mma_ss(tS[t], sw128_desc_join(qa + off, 1024), sw128_desc_join(ka + off, 1024),
                           C::IDESC_QK, kk > 0 ? 1u : 0u);
                }
            };
            // O_t (+)= P_t V: each half of P (64 keys) is consumed as soon as the
            // softmax warpgroup has written it, so the first half of the MMA
            // overlaps the exponentials of the second half.
            auto pv = [&](int t, uint32_t vslot, bool acc) -> bool {
                const uint32_t va = sw128_desc_lo(sKV + vslot * C::TILE, C::SUB);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (!mbar_wait(b_pfull + 16 * t + 8 * h, pph[t], lim, W_PFULL, abort_flag))
                        return false;
                    tc_fence_after_sync();
#pragma unroll
                    for (int kk = 4 * h; kk < 4 * h + 4; ++kk)
                        mma_ts(tO[t], tS[t] + 8 * kk, sw128_desc_join(va + kk * (2048 >> 4), 1024),
                               C::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
                }
                pph[t] ^= 1u;
                return true;
            };

            for (int k = 0; ok; ++k) {
                UnitInfo u;
                const int r = unit_of(p, k, u);
                if (r < 0) break;
                if (r == 0) continue;
#pragma unroll
                for (int t = 0; t < 2 && ok; ++t) {
                    if (u.n[t] == 0) continue;
                    ok = mbar_wait(b_qfull + 8 * t, qph[t], lim, W_QFULL, abort_flag);
                    qph[t] ^= 1u;
                }
                if (!ok) break;
                // K_0: first score tiles
                uint32_t ks = ring.idx;
                if (!(ok = mbar_wait(b_kvfull + 8 * ks, ring.phase, lim, W_KVFULL, abort_flag))) break;
                ring.advance<C::NSTAGE>();
                tc_fence_after_sync();
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (u.n[t] == 0) continue;
                    if (p.order_mode == 1 && issued_any && !(ok = drain())) break;
                    qk(t, ks);
                    issued_any = true;
                    tc_commit(b_sfull + 8 * t);
                    if (u.n[t] == 1) tc_commit(b_qempty + 8 * t);
                }
                if (!ok) break;
                tc_commit(b_kvempty + 8 * ks);
                for (int j = 1; ok && j < u.niter; ++j) {
                    ks = ring.idx;
                    if (!(ok = mbar_wait(b_kvfull + 8 * ks, ring.phase, lim, W_KVFULL, abort_flag))) break;
                    ring.advance<C::NSTAGE>();
                    const uint32_t vs = ring.idx;
                    if (!(ok = mbar_wait(b_kvfull + 8 * vs, ring.phase, lim, W_KVFULL, abort_flag))) break;
                    ring.advance<C::NSTAGE>();
                    tc_fence_after_sync();
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        if (j - 1 < u.n[t]) {  // O_t += P_t(j-1) V_{j-1}
                            if (!(ok = pv(t, vs, j - 1 > 0))) break;
                            if (j - 1 == u.n[t] - 1) tc_commit(b_pvdone + 8 * t);
                        }
                        if (j < u.n[t]) {      // S_t = Q_t K_j^T
                            if (p.order_mode == 1 && !(ok = drain())) break;
                            qk(t, ks);
                            tc_commit(b_sfull + 8 * t);
                            if (j == u.n[t] - 1) tc_commit(b_qempty + 8 * t);
                        }
                    }
                    if (!ok) break;
                    tc_commit(b_kvempty + 8 * ks);
                    tc_commit(b_kvempty + 8 * vs);
                }
                if (!ok) break;
                const uint32_t vs = ring.idx;
                if (!(ok = mbar_wait(b_kvfull + 8 * vs, ring.phase, lim, W_KVFULL, abort_flag))) break;
                ring.advance<C::NSTAGE>();
                tc_fence_after_sync();
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (u.niter - 1 < u.n[t]) {
                        if (!(ok = pv(t, vs, u.niter - 1 > 0))) break;
                        tc_commit(b_pvdone + 8 * t);
                    }
                }
                if (!ok) break;
                tc_commit(b_kvempty + 8 * vs);
            }
            if (!ok) {
                *abort_flag = 1;
                drain();  // every issued MMA finishes before TMEM is freed
            }
        }
      }
    } else {
        // ------------------------------------------------------------ softmax warpgroups
        reg_alloc<C::REGS_SOFTMAX>();
        const int t = warp >> 2;          // query tile 0 or 1
        const int wq = warp & 3;          // TMEM lane quarter
        const int rit = wq * 32 + lane;   // row in tile == TMEM lane
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + lane_off + C::TM_S + 128 * t;
        const uint32_t tO = tmem + lane_off + C::TM_O + D * t;
        const float cl2 = p.c_log2;
        uint32_t sph = 0, oph = 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
            UnitInfo u;
            const int r = unit_of(p, k, u);
            if (r < 0) break;
            if (r == 0) continue;
            const int nt = u.n[t];
            if (nt == 0) continue;
            const int r0 = u.i0 + 128 * t;
            const int row = r0 + rit;
            float m = -INFINITY;  // running max, log2 units
            float l = 0.f;        // running normaliser (fp32 weights)
            float lcor = 0.f;     // bf16 rounding of each tile's largest weight
            for (int j = 0; j < nt; ++j) {
                bool w = mbar_wait(b_sfull + 8 * t, sph, lim, W_SFULL, abort_flag);
                ok = __all_sync(0xffffffffu, w);
                if (!ok) break;
                sph ^= 1u;
                tc_fence_after_sync();
                float s[128];
                {
                    uint32_t r[128];
                    tmem_ld128(tS, r);
                    tmem_wait_ld_regs128(r);
#pragma unroll
                    for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(r[i]);
                }
                const int key0 = 128 * j;
                const bool need_mask = (CAUSAL && key0 + 127 > r0) || (key0 + 128 > p.T);
                if (need_mask) {
                    const int lim_key = CAUSAL ? min(row, p.T - 1) : p.T - 1;
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (key0 + c > lim_key) s[c] = -INFINITY;
                }
                const float smax = row_max(s);
                const float cand = smax * cl2;
                // Does the tile's largest score sit in a pair whose exponential the
                // FMA pipe evaluates?  Its weight for the correction below must
                // come from the same evaluation (variants with EMU > 0 only).
                bool max_emu = false;
                if constexpr (EMU > 0) {
                    if (!need_mask) {
#pragma unroll
                        for (int i = 0; i < 64; ++i)
                            if (emu_pair<EMU>(i)) max_emu |= (s[2 * i] == smax) | (s[2 * i + 1] == smax);
                    }
                }
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
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld32(tO + 32 * c, r);
                        tmem_wait_ld_regs(r);
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                        tmem_st32(tO + 32 * c, r);
                    }
                }
                l *= alpha;
                lcor *= alpha;
                const float neg_m = (m == -INFINITY) ? 0.f : -m;
                const float2 c2 = make_float2(cl2, cl2);
                float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                // p = 2^(s * scale * log2e - m).  On tiles without masked keys a
                // fixed share of the pairs (EMU of every 8) is evaluated on the
                // FMA pipe, the rest by MUFU.EX2.
                uint32_t pk0[32];
                if (EMU > 0 && !need_mask)
                    exp_pairs<EMU, 0, 32>(s, c2, make_float2(neg_m, neg_m), pk0, ls);
                else
                    exp_pairs<0, 0, 32>(s, c2, make_float2(neg_m, neg_m), pk0, ls);
                tmem_st32(tS, pk0);
                tmem_wait_st();
                tc_fence_before_sync();
                mbar_arrive(b_pfull + 16 * t);  // keys 0-63 of P are in TMEM
                uint32_t pk1[32];
                if (EMU > 0 && !need_mask)
                    exp_pairs<EMU, 32, 32>(s, c2, make_float2(neg_m, neg_m), pk1, ls);
                else
                    exp_pairs<0, 32, 32>(s, c2, make_float2(neg_m, neg_m), pk1, ls);
                tmem_st32(tS + 32, pk1);
                tmem_wait_st();
                tc_fence_before_sync();
                mbar_arrive(b_pfull + 16 * t + 8);  // keys 64-127
                l += (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y);
                // The P.V MMA multiplies bf16-rounded weights while l sums the
                // fp32 ones.  On a row dominated by one key that mismatch would
                // scale O by up to 1 +- 2^-9; the dominant key is its tile's
                // largest score, so the normaliser of O takes that element's
                // rounding error (its p recomputed bit for bit: the same fma,
                // and the same ex2 or polynomial, as above -- two evaluations
                // 7.5e-5 apart can round to neighbouring bf16 values, an error
                // of 2^-8 that the correction would then add instead of
                // removing).  lse keeps the fp32 sum.
                const float xmax = fmaf(smax, cl2, neg_m);
                const float pmax = max_emu ? exp2_poly2(make_float2(xmax, xmax)).x : fast_exp2(xmax);
                lcor += bf16_round(pmax) - pmax;
            }
            if (!ok) break;
            // epilogue: O = acc / l, lse = (m + log2 l) ln 2
            bool w = mbar_wait(b_pvdone + 8 * t, oph, lim, W_PVDONE, abort_flag);
            ok = __all_sync(0xffffffffu, w);
            if (!ok) break;
            oph ^= 1u;
            tc_fence_after_sync();
            const float inv_l = 1.f / (l + lcor);
            const size_t orow = (size_t)u.bh * (size_t)p.T + (size_t)row;
            if constexpr (CAUSAL) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tO + 32 * c, r);
                tmem_wait_ld_regs(r);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l,
                                        __uint_as_float(r[2 * i + 1]) * inv_l);
                if (row < p.T) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.o + orow * D + 32 * c);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
            } else {
            // non-causal: O rows through this warp's 4 KB of shared memory, 64
            // columns at a time, so that each store instruction writes four whole
            // 128-byte lines (4 rows x 64 columns) instead of 32 scattered
            // 16-byte pieces; 16-byte chunk j of a staged row sits at j ^ (row & 7)
            uint8_t *stg = gbase + C::OFF_EPI + warp * 4096;
            const int r0w = r0 + wq * 32;  // the warp's first row
#pragma unroll
            for (int hh = 0; hh < D / 64; ++hh) {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    uint32_t rr[32];
                    tmem_ld32(tO + 64 * hh + 32 * cc, rr);
                    tmem_wait_ld_regs(rr);
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int j = 4 * cc + jj;
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(rr[8 * jj + 0]) * inv_l, __uint_as_float(rr[8 * jj + 1]) * inv_l);
                        v.y = pack_bf16x2(__uint_as_float(rr[8 * jj + 2]) * inv_l, __uint_as_float(rr[8 * jj + 3]) * inv_l);
                        v.z = pack_bf16x2(__uint_as_float(rr[8 * jj + 4]) * inv_l, __uint_as_float(rr[8 * jj + 5]) * inv_l);
                        v.w = pack_bf16x2(__uint_as_float(rr[8 * jj + 6]) * inv_l, __uint_as_float(rr[8 * jj + 7]) * inv_l);
                        *reinterpret_cast<uint4 *>(stg + lane * 128 + 16 * (j ^ (lane & 7))) = v;
                    }
                }
                __syncwarp();
#pragma unroll
                for (int k4 = 0; k4 < 8; ++k4) {
                    const int rw = 4 * k4 + (lane >> 3), j = lane & 7;
                    const uint4 v = *reinterpret_cast<const uint4 *>(stg + rw * 128 + 16 * (j ^ (rw & 7)));
                    if (r0w + rw < p.T)
                        *reinterpret_cast<uint4 *>(p.o + ((size_t)u.bh * (size_t)p.T + (size_t)(r0w + rw)) * D +
                                                   64 * hh + 8 * j) = v;
                }
                __syncwarp();
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
