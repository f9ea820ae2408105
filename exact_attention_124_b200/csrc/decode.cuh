// decode.cuh -- decode attention for B200 (sm_100a): Tq new queries against a
// K/V cache of Tk tokens (query i at position Tk - Tq + i; causal: it sees
// keys up to its own position).  "FlashAttention -- avoid writing the giant
// intermediate", "Exact attention has limits": the persistent K/V state of
// cached decoding; "Apply it at the right layer": decode is measured apart
// from prefill.
//
// Decode is bound by reading the cache, so the keys are spread over every SM.
// The work is the list of (K/V head, block of 128 packed query rows) "heads"
// times their ceil(Tk / 128) key tiles; a CTA takes a contiguous range of
// that list, cut into segments at head boundaries (one segment = one head's
// tiles in this CTA), and writes one partial result per segment:
//   balanced (automatic): one CTA per SM, the list cut into equal ranges, so
//            every SM streams the same number of tiles (a head may span
//            several CTAs and a CTA several heads);
//   fixed:   every head cut into `splits` equal key ranges, one CTA each.
//   decode_partial_kernel  the rows packed into the M = 128 tile are (query
//                          head of the K/V head's group, query) pairs, so a
//                          grouped-query group shares each K/V tile.  With
//                          R = group * Tq <= 32 (64) real rows, the tile holds
//                          CP = 4 (2) copies of them, one per 128 / CP lanes,
//                          and copy c takes only keys [c W, c W + W) of every
//                          tile (W = 128 / CP; P is zero elsewhere in its
//                          rows): each softmax thread does W instead of 128
//                          exponentials and the copies are merged like
//                          further key splits.  Online
//                          softmax over a segment's tiles exactly as the
//                          prefill kernel (S = Q K^T and O += P V on tcgen05, S
//                          double buffered in TMEM so the next score tile is
//                          computed during this one's softmax, Q double
//                          buffered in shared memory across segments); writes
//                          each segment's O (fp32, normalised by its own l)
//                          and lse.
//   decode_combine_kernel  per query row: lse = log sum_s exp(lse_s),
//                          O = sum_s exp(lse_s - lse) O_s, as bf16 / fp32.
#pragma once

#include "sm100.cuh"

namespace attn {

struct DecodeParams {
    float *part_o;    // [slots, B*H*Tq, D]
    float *part_lse;  // [slots, B*H*Tq]
    long long nrows;  // B * H * Tq
    int H, H_kv, group, Tq, Tk, causal;
    int rows;         // packed query rows per K/V head: group * Tq
    int nrb;          // blocks of 128 packed rows per K/V head
    int nkt;          // key tiles of 128
    int copies;       // CP: copies of the packed rows in the 128-row tile
    int balanced;     // 1: balanced ranges over G CTAs; 0: fixed splits
    int chunk;        // fixed: key tiles per split
    int splits;       // fixed: splits per head (= partial slots)
    long long tot;    // balanced: heads * nkt tiles in all
    int G;            // balanced: CTAs
    float c_log2;
    unsigned long long limit_ns;
};

constexpr float DEC_RESCALE_TAU = 32.0f;  // lazy rescale threshold, log2 units (as prefill)

enum : unsigned int {
    W_D_Q = 128, W_D_KVFULL, W_D_KVEMPTY, W_D_SFULL, W_D_PFULL, W_D_PVDONE, W_D_DRAIN, W_D_QEMPTY,
    W_D_OFREE
};

// Balanced mode: CTA c covers tiles [c tot / G, (c + 1) tot / G) of the list;
// the CTA that holds tile g.
__host__ __device__ __forceinline__ long long dec_cta_of(long long g, long long tot, int G)
{
    return ((g + 1) * G - 1) / tot;
}

// Partial slots a head needs in balanced mode (segments it is cut into).
__host__ __device__ __forceinline__ int dec_nseg(long long w, int nkt, long long tot, int G)
{
    return (int)(dec_cta_of(w * nkt + nkt - 1, tot, G) - dec_cta_of(w * nkt, tot, G) + 1);
}

struct DecSeg {
    int kvbh, qt;  // K/V head (batch * H_kv + kv head), block of packed rows
    int t0, n;     // first key tile, tiles
    int slot;      // partial slot of this head
};

// The idx-th segment of CTA (bx, by, bz); false when there is none.  Also
// run on the host by attn_selftest_decode_segments().
__host__ __device__ __forceinline__ bool dec_segment(const DecodeParams &p, int bx, int by, int bz,
                                                     int idx, DecSeg &sg)
{
    if (!p.balanced) {
        if (idx > 0) return false;
        sg.kvbh = by;
        sg.qt = bz;
        sg.t0 = bx * p.chunk;
        sg.n = (p.nkt < sg.t0 + p.chunk ? p.nkt : sg.t0 + p.chunk) - sg.t0;  // >= 1 by the host's choice
        sg.slot = bx;
        return true;
    }
    const long long c = bx;
    const long long lo = c * p.tot / p.G, hi = (c + 1) * p.tot / p.G;
    const long long w = lo / p.nkt + idx;
    const long long start = lo > w * p.nkt ? lo : w * p.nkt;
    if (start >= hi) return false;
    const long long end = hi < (w + 1) * p.nkt ? hi : (w + 1) * p.nkt;
    sg.kvbh = (int)(w / p.nrb);
    sg.qt = (int)(w % p.nrb);
    sg.t0 = (int)(start - w * p.nkt);
    sg.n = (int)(end - start);
    sg.slot = (int)(c - dec_cta_of(w * p.nkt, p.tot, p.G));
    return true;
}

template <int D>
struct DecCfg {
    static constexpr int KB = D / 64;
    static constexpr int SUB = 128 * 128;
    static constexpr int TILE = 128 * D * 2;
    static constexpr int NSTAGE = (D == 64) ? 8 : 4;
    static constexpr int OFF_Q = 0;                // [2] Q tiles
    static constexpr int OFF_KV = 2 * TILE;
    static constexpr int OFF_BAR = OFF_KV + NSTAGE * TILE;
    static constexpr int NBAR = 2 + 2 + 2 * NSTAGE + 2 + 2 + 1 + 1 + 1 + 1;
    static constexpr int SMEM = 1024 + OFF_BAR + NBAR * 8 + 16;
    static constexpr int THREADS = 192;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_S = 0;    // + 128 * buffer
    static constexpr uint32_t TM_O = 256;
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);
};

template <int D, int CP>
__global__ void __launch_bounds__(192, 1)
    decode_partial_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const DecodeParams p)
{
    using C = DecCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t sQ = base + C::OFF_Q, sKV = base + C::OFF_KV;
    const uint32_t bar0 = base + C::OFF_BAR;
    const uint32_t b_qfull = bar0;                       // [2]
    const uint32_t b_qempty = b_qfull + 16;              // [2]
    const uint32_t b_kvfull = b_qempty + 16;             // [NSTAGE]
    const uint32_t b_kvempty = b_kvfull + 8 * C::NSTAGE;  // [NSTAGE]
    const uint32_t b_sfull = b_kvempty + 8 * C::NSTAGE;  // [2]
    // one P barrier per S buffer: a single one could complete twice (two
    // tiles) before the MMA warp waits on the first, aliasing its phase
    const uint32_t b_pfull = b_sfull + 16;  // [2]
    // b_pvdone completes after every P V (the lazy rescale waits for the
    // previous one: only that one can be outstanding there).  The epilogue
    // waits on b_pvlast, completed once per segment after its last P V: with
    // the per-tile barrier the last P V's parity could alias the one before
    // it while both are still in flight.
    const uint32_t b_pvdone = b_pfull + 16;
    const uint32_t b_pvlast = b_pvdone + 8;
    const uint32_t b_ofree = b_pvlast + 8;  // the softmax warps have read a segment's O
    const uint32_t b_drain = b_ofree + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + C::OFF_BAR + C::NBAR * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t lim = p.limit_ns;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(b_qfull + 8 * i, 1);
            mbar_init(b_qempty + 8 * i, 1);
            mbar_init(b_sfull + 8 * i, 1);
            mbar_init(b_pfull + 8 * i, 128);
        }
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(b_kvfull + 8 * s, 1);
            mbar_init(b_kvempty + 8 * s, 1);
        }
        mbar_init(b_pvdone, 1);
        mbar_init(b_pvlast, 1);
        mbar_init(b_ofree, 128);
        mbar_init(b_drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 4) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 5) {
        if (lane == 0) {  // TMA: per segment Q, then K_0, K_1, V_0, K_2, V_1, ... (consumption order)
            const uint64_t pol_q = policy_evict_first(), pol_kv = policy_evict_first();
            uint32_t idx = 0, ph = 0, armed = 0, armed_par = 0, qarmed = 0, qarmed_par = 0;
            bool ok = true;
            DecSeg sg;
            for (int si = 0; ok && dec_segment(p, blockIdx.x, blockIdx.y, blockIdx.z, si, sg); ++si) {
                const int qb = si & 1;
                const uint32_t qpar = (uint32_t)(si >> 1) & 1u;
                if (!mbar_wait(b_qempty + 8 * qb, qpar ^ 1u, lim, W_D_QEMPTY, abort_flag)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(b_qfull + 8 * qb, C::TILE);
                qarmed |= 1u << qb;
                qarmed_par = (qarmed_par & ~(1u << qb)) | (qpar << qb);
                const int b = sg.kvbh / p.H_kv, kvl = sg.kvbh % p.H_kv;
                const int qrow0 = (b * p.H + kvl * p.group) * p.Tq + sg.qt * 128;
                // CP copies of the R = 128 / CP rows (the map's box is R rows)
                for (int kb = 0; kb < C::KB; ++kb)
#pragma unroll
                    for (int cp = 0; cp < CP; ++cp)
                        tma_load_3d(sQ + qb * C::TILE + kb * C::SUB + cp * (128 / CP) * 128, &tmQ,
                                    b_qfull + 8 * qb, 64 * kb, qrow0, 0, pol_q);
                auto load = [&](const CUtensorMap *map, int tile) -> bool {
                    if (!mbar_wait(b_kvempty + 8 * idx, ph ^ 1u, lim, W_D_KVEMPTY, abort_flag)) return false;
                    mbar_arrive_expect_tx(b_kvfull + 8 * idx, C::TILE);
                    armed |= 1u << idx;
                    armed_par = (armed_par & ~(1u << idx)) | (ph << idx);
                    for (int kb = 0; kb < C::KB; ++kb)
                        tma_load_3d(sKV + idx * C::TILE + kb * C::SUB, map, b_kvfull + 8 * idx, 64 * kb,
                                    128 * (sg.t0 + tile), sg.kvbh, pol_kv);
                    if (++idx == (uint32_t)C::NSTAGE) { idx = 0; ph ^= 1u; }
                    return true;
                };
                ok = load(&tmK, 0);
                if (ok && sg.n > 1) ok = load(&tmK, 1);
                for (int j = 0; ok && j < sg.n; ++j) {
                    ok = load(&tmV, j);
                    if (ok && j + 2 < sg.n) ok = load(&tmK, j + 2);
                }
            }
            if (!ok) {
                *abort_flag = 1;
                for (int i = 0; i < 2; ++i)
                    if ((qarmed >> i) & 1u) mbar_wait(b_qfull + 8 * i, (qarmed_par >> i) & 1u, lim, W_D_Q);
                for (int s = 0; s < C::NSTAGE; ++s)
                    if ((armed >> s) & 1u) mbar_wait(b_kvfull + 8 * s, (armed_par >> s) & 1u, lim, W_D_KVFULL);
            }
        }
    } else if (warp == 4) {
        if (lane == 0) {  // MMA issuer
            uint32_t idx = 0, ph = 0;
            bool ok = true;
            auto next = [&](uint32_t &slot) -> bool {
                slot = idx;
                const bool r = mbar_wait(b_kvfull + 8 * idx, ph, lim, W_D_KVFULL, abort_flag);
                if (++idx == (uint32_t)C::NSTAGE) { idx = 0; ph ^= 1u; }
                tc_fence_after_sync();
                return r;
            };
            uint32_t ql = 0;
            auto qk = [&](int buf, uint32_t slot) {
                const uint32_t kl = sw128_desc_lo(sKV + slot * C::TILE, 16);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::SUB + (kk & 3) * 32) >> 4;
                    mma_ss(tmem + C::TM_S + 128 * buf, sw128_desc_join(ql + off, 1024),
                           sw128_desc_join(kl + off, 1024), C::IDESC_QK, kk > 0 ? 1u : 0u);
                }
                tc_commit(b_sfull + 8 * buf);
                tc_commit(b_kvempty + 8 * slot);
            };
            uint32_t u = 0;  // tiles of earlier segments: global tile u + j uses S buffer (u + j) & 1
            DecSeg sg;
            for (int si = 0; ok && dec_segment(p, blockIdx.x, blockIdx.y, blockIdx.z, si, sg); ++si) {
                const int qb = si & 1;
                if (!(ok = mbar_wait(b_qfull + 8 * qb, (uint32_t)(si >> 1) & 1u, lim, W_D_Q, abort_flag)))
                    break;
                tc_fence_after_sync();
                ql = sw128_desc_lo(sQ + qb * C::TILE, 16);
                const int n = sg.n;
                uint32_t slot = 0;
                if ((ok = next(slot))) qk(u & 1, slot);
                if (ok && n > 1) {
                    if ((ok = next(slot))) qk((u + 1) & 1, slot);
                }
                for (int j = 0; ok && j < n; ++j) {
                    const uint32_t t = u + j;
                    uint32_t vs = 0;
                    if (!(ok = next(vs))) break;
                    if (!(ok = mbar_wait(b_pfull + 8 * (t & 1), (t >> 1) & 1u, lim, W_D_PFULL, abort_flag)))
                        break;
                    // the first P V of a segment overwrites O: the previous
                    // segment's O must have been read out
                    if (j == 0 && si > 0 &&
                        !(ok = mbar_wait(b_ofree, (uint32_t)(si - 1) & 1u, lim, W_D_OFREE, abort_flag)))
                        break;
                    tc_fence_after_sync();
                    const uint32_t vl = sw128_desc_lo(sKV + vs * C::TILE, C::SUB);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts(tmem + C::TM_O, tmem + C::TM_S + 128 * (t & 1) + 8 * kk,
                               sw128_desc_join(vl + kk * (2048 >> 4), 1024), C::IDESC_PV,
                               (j > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(b_pvdone);
                    if (j == n - 1) tc_commit(b_pvlast);
                    tc_commit(b_kvempty + 8 * vs);
                    if (j + 2 < n) {  // the next score tile into the buffer just consumed
                        if (!(ok = next(slot))) break;
                        qk(t & 1, slot);
                    }
                }
                if (!ok) break;
                tc_commit(b_qempty + 8 * qb);  // fires once this segment's Q K^T are done
                u += n;
            }
            if (!ok) {
                *abort_flag = 1;
                tc_commit(b_drain);
                mbar_wait(b_drain, 0, lim, W_D_DRAIN);
            }
        }
    } else if (warp < 4) {  // softmax: thread = packed query row of one copy
        constexpr int W = 128 / CP;  // rows per copy, and keys per copy in each tile
        const int r = warp * 32 + lane;
        const int cp = r / W, rr = r % W;  // copy (warp-uniform), row within the copy
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const float cl2 = p.c_log2;
        bool ok = true;
        uint32_t u = 0;
        DecSeg sg;
        for (int si = 0; ok && dec_segment(p, blockIdx.x, blockIdx.y, blockIdx.z, si, sg); ++si) {
            const int n = sg.n;
            const int pr = sg.qt * 128 + rr;
            const bool valid = pr < p.rows;
            const int g = valid ? pr / p.Tq : 0, qi = valid ? pr % p.Tq : 0;
            const int pos = p.Tk - p.Tq + qi;
            const int lim_key = p.causal ? pos : p.Tk - 1;
            float m = -INFINITY, l = 0.f;
            float lcor = 0.f;  // bf16 rounding of each tile's largest weight (normaliser of O only)
            for (int j = 0; ok && j < n; ++j) {
                const uint32_t t = u + j;
                const int buf = t & 1;
                const bool w = mbar_wait(b_sfull + 8 * buf, (t >> 1) & 1u, lim, W_D_SFULL, abort_flag);
                if (!(ok = __all_sync(0xffffffffu, w))) break;
                tc_fence_after_sync();
                const uint32_t tS = tmem + lane_off + C::TM_S + 128 * buf;
                float s[W];
                if constexpr (W == 128) {
                    uint32_t rg[128];
                    tmem_ld128(tS, rg);
                    tmem_wait_ld_regs128(rg);
#pragma unroll
                    for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(rg[i]);
                } else {
#pragma unroll
                    for (int c = 0; c < W / 32; ++c) {
                        uint32_t rg[32];
                        tmem_ld32(tS + cp * W + 32 * c, rg);
                        tmem_wait_ld_regs(rg);
#pragma unroll
                        for (int i = 0; i < 32; ++i) s[32 * c + i] = __uint_as_float(rg[i]);
                    }
                }
                const int key0 = 128 * (sg.t0 + j) + cp * W;  // key of s[0]
                const bool need_mask = (key0 + W > p.Tk) || (p.causal && key0 + W - 1 > p.Tk - p.Tq);
                if (need_mask) {
#pragma unroll
                    for (int c = 0; c < W; ++c)
                        if (key0 + c > lim_key) s[c] = -INFINITY;
                }
                float mx = s[0];
#pragma unroll
                for (int c = 1; c < W; ++c) mx = fmaxf(mx, s[c]);
                const float cand = mx * cl2;
                float alpha = 1.f;
                bool resc = false;
                if (m == -INFINITY) {
                    m = cand;  // first visible key: the accumulator holds zeros so far
                } else if (cand > m + DEC_RESCALE_TAU) {
                    alpha = fast_exp2(m - cand);
                    m = cand;
                    resc = true;
                }
                if (__any_sync(0xffffffffu, resc)) {  // wait for the previous PV, then rescale O
                    const bool w2 = mbar_wait(b_pvdone, (t - 1) & 1u, lim, W_D_PVDONE, abort_flag);
                    if (!(ok = __all_sync(0xffffffffu, w2))) break;
                    tc_fence_after_sync();
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t rg[32];
                        tmem_ld32(tmem + lane_off + C::TM_O + 32 * c, rg);
                        tmem_wait_ld_regs(rg);
#pragma unroll
                        for (int i = 0; i < 32; ++i) rg[i] = __float_as_uint(__uint_as_float(rg[i]) * alpha);
                        tmem_st32(tmem + lane_off + C::TM_O + 32 * c, rg);
                    }
                }
                l *= alpha;
                lcor *= alpha;
                const float neg_m = (m == -INFINITY) ? 0.f : -m;
                {  // the P.V MMA sees bf16 weights; see the fused kernel's softmax
                    const float pmax = fast_exp2(fmaf(mx, cl2, neg_m));
                    lcor += bf16_round(pmax) - pmax;
                }
                float ls = 0.f;
                // P over the first 64 S columns (bf16 pairs): this copy's W keys
                // at pair columns [cp W / 2, cp W / 2 + W / 2), zeros elsewhere
#pragma unroll
                for (int h = 0; h < (W + 63) / 64; ++h) {
                    constexpr int NP = W < 64 ? W / 2 : 32;  // pairs in this store
                    uint32_t pk[NP];
#pragma unroll
                    for (int i = 0; i < NP; ++i) {
                        const float p0 = fast_exp2(fmaf(s[64 * h + 2 * i], cl2, neg_m));
                        const float p1 = fast_exp2(fmaf(s[64 * h + 2 * i + 1], cl2, neg_m));
                        ls += p0 + p1;
                        pk[i] = pack_bf16x2(p0, p1);
                    }
                    if constexpr (NP == 32) tmem_st32(tS + cp * (W / 2) + 32 * h, pk);
                    else tmem_st16(tS + cp * (W / 2), pk);
                }
                if constexpr (CP == 2) {
                    uint32_t z[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) z[i] = 0u;
                    tmem_st32(tS + (1 - cp) * 32, z);
                } else if constexpr (CP == 4) {
                    uint32_t z[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) z[i] = 0u;
#pragma unroll
                    for (int o = 1; o < 4; ++o) tmem_st16(tS + ((cp + o) & 3) * 16, z);
                }
                l += ls;
                tmem_wait_st();
                tc_fence_before_sync();
                mbar_arrive(b_pfull + 8 * buf);
            }
            if (!ok) break;
            u += n;
            const bool w = mbar_wait(b_pvlast, (uint32_t)si & 1u, lim, W_D_PVDONE, abort_flag);
            if (!(ok = __all_sync(0xffffffffu, w))) break;
            tc_fence_after_sync();
            const int b = sg.kvbh / p.H_kv, kvl = sg.kvbh % p.H_kv;
            const size_t row = (size_t)(b * p.H + kvl * p.group + g) * p.Tq + qi;
            // each copy's result is one more partial of this row
            const size_t at = ((size_t)sg.slot * CP + cp) * (size_t)p.nrows + row;
            const float inv = l > 0.f ? 1.f / (l + lcor) : 0.f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t rg[32];
                tmem_ld32(tmem + lane_off + C::TM_O + 32 * c, rg);
                tmem_wait_ld_regs(rg);
                if (valid) {
                    float4 *dst = reinterpret_cast<float4 *>(p.part_o + at * D + 32 * c);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[i] = make_float4(__uint_as_float(rg[4 * i]) * inv, __uint_as_float(rg[4 * i + 1]) * inv,
                                             __uint_as_float(rg[4 * i + 2]) * inv, __uint_as_float(rg[4 * i + 3]) * inv);
                }
            }
            tc_fence_before_sync();
            mbar_arrive(b_ofree);  // O of this segment is in registers / memory: it may be overwritten
            if (valid) p.part_lse[at] = l > 0.f ? (m + fast_log2(l)) * 0.69314718055994530942f : -INFINITY;
        }
        if (!ok) *abort_flag = 1;
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 4) tmem_dealloc(tmem, C::TMEM_COLS);
}

// The merge: 128 threads per CTA, 128 / D query rows per CTA, one thread per
// output column.  Every thread walks the row's partials with loads that depend
// on nothing loaded before them (the lse reads are the same address across
// the row's threads: one broadcast each), so a row costs about two memory
// round trips, and there are as many CTAs as rows x D / 128.
template <int D>
__global__ void __launch_bounds__(128)
    decode_combine_kernel(const DecodeParams p, __nv_bfloat16 *__restrict__ o, float *__restrict__ lse)
{
    // launched as a programmatic dependent of decode_partial_kernel: wait
    // until that grid has finished and its writes are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    constexpr int ROWS = 128 / D;
    const long long nrows = p.nrows;
    const float *__restrict__ part_o = p.part_o;
    const float *__restrict__ part_lse = p.part_lse;
    const long long r = (long long)blockIdx.x * ROWS + threadIdx.x / D;
    const int c = threadIdx.x % D;
    if (r >= nrows) return;
    int splits = p.splits;
    if (p.balanced) {  // row (b, h, query) -> its head (K/V head, packed row block)
        const long long b = r / ((long long)p.H * p.Tq), h = (r / p.Tq) % p.H, tq = r % p.Tq;
        const long long pr = (h % p.group) * p.Tq + tq;
        const long long w = (b * p.H_kv + h / p.group) * p.nrb + pr / 128;
        splits = dec_nseg(w, p.nkt, p.tot, p.G);
    }
    splits *= p.copies;  // every segment wrote one partial per copy of the rows
    float mx = -INFINITY;
#pragma unroll 8
    for (int s = 0; s < splits; ++s) mx = fmaxf(mx, part_lse[(size_t)s * nrows + r]);
    float acc = 0.f, sum = 0.f;
    if (mx != -INFINITY) {
        // a partial with lse = -inf (no visible key) gets weight 0; its O was
        // written as exactly 0
#pragma unroll 8
        for (int s = 0; s < splits; ++s) {
            const float ls = part_lse[(size_t)s * nrows + r];
            const float w = ls == -INFINITY ? 0.f : expf(ls - mx);
            sum += w;
            acc = fmaf(w, part_o[((size_t)s * nrows + r) * D + c], acc);
        }
    }
    o[r * D + c] = __float2bfloat16_rn(sum > 0.f ? acc / sum : 0.f);
    if (c == 0) lse[r] = sum > 0.f ? mx + logf(sum) : -INFINITY;
}

}  // namespace attn
