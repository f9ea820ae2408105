// decode.cuh -- decode attention for B200 (sm_100a): Tq new queries against a
// K/V cache of Tk tokens (query i at position Tk - Tq + i; causal: it sees
// keys up to its own position).  "FlashAttention -- avoid writing the giant
// intermediate", "Exact attention has limits": the persistent K/V state of
// cached decoding; "Apply it at the right layer": decode is measured apart
// from prefill.
//
// Decode is bound by reading the cache, so the key range is split across
// CTAs (split-KV) to put every SM on it:
//   decode_partial_kernel  one CTA per (key split, batch x K/V head, block of
//                          128 packed query rows).  The rows packed into the
//                          M = 128 tile are (query head of the K/V head's
//                          group, query) pairs, so a grouped-query group
//                          shares each K/V tile.  Online softmax over the
//                          split's key tiles exactly as the prefill kernel
//                          (S = Q K^T and O += P V on tcgen05, S double
//                          buffered in TMEM so the next score tile is computed
//                          during this one's softmax); writes the split's O
//                          (fp32, normalised by the split's own l) and lse.
//   decode_combine_kernel  per query row: lse = log sum_s exp(lse_s),
//                          O = sum_s exp(lse_s - lse) O_s, as bf16 / fp32.
#pragma once

#include "sm100.cuh"

namespace attn {

struct DecodeParams {
    float *part_o;    // [splits, B*H*Tq, D]
    float *part_lse;  // [splits, B*H*Tq]
    int H, H_kv, group, Tq, Tk, causal;
    int rows;         // packed query rows per K/V head: group * Tq
    int nkt;          // key tiles of 128
    int chunk;        // key tiles per split
    int splits;
    float c_log2;
    unsigned long long limit_ns;
};

constexpr float DEC_RESCALE_TAU = 8.0f;  // lazy rescale threshold, log2 units (as prefill)

enum : unsigned int { W_D_Q = 128, W_D_KVFULL, W_D_KVEMPTY, W_D_SFULL, W_D_PFULL, W_D_PVDONE, W_D_DRAIN };

template <int D>
struct DecCfg {
    static constexpr int KB = D / 64;
    static constexpr int SUB = 128 * 128;
    static constexpr int TILE = 128 * D * 2;
    static constexpr int NSTAGE = (D == 64) ? 8 : 4;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = TILE;
    static constexpr int OFF_BAR = OFF_KV + NSTAGE * TILE;
    static constexpr int NBAR = 1 + 2 * NSTAGE + 2 + 2 + 1 + 1;
    static constexpr int SMEM = 1024 + OFF_BAR + NBAR * 8 + 16;
    static constexpr int THREADS = 192;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_S = 0;    // + 128 * buffer
    static constexpr uint32_t TM_O = 256;
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);
};

template <int D>
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
    const uint32_t b_q = bar0;
    const uint32_t b_kvfull = bar0 + 8;
    const uint32_t b_kvempty = b_kvfull + 8 * C::NSTAGE;
    const uint32_t b_sfull = b_kvempty + 8 * C::NSTAGE;  // [2]
    // one P barrier per S buffer: a single one could complete twice (two
    // tiles) before the MMA warp waits on the first, aliasing its phase
    const uint32_t b_pfull = b_sfull + 16;  // [2]
    const uint32_t b_pvdone = b_pfull + 16;
    const uint32_t b_drain = b_pvdone + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + C::OFF_BAR + C::NBAR * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int split = blockIdx.x;
    const int kvbh = blockIdx.y;
    const int qt = blockIdx.z;
    const int b = kvbh / p.H_kv, kvl = kvbh % p.H_kv;
    const int t0 = split * p.chunk;
    const int n = min(p.nkt, t0 + p.chunk) - t0;  // >= 1 by the host's choice of splits
    const uint64_t lim = p.limit_ns;

    if (threadIdx.x == 0) {
        mbar_init(b_q, 1);
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(b_kvfull + 8 * s, 1);
            mbar_init(b_kvempty + 8 * s, 1);
        }
        mbar_init(b_sfull, 1);
        mbar_init(b_sfull + 8, 1);
        mbar_init(b_pfull, 128);
        mbar_init(b_pfull + 8, 128);
        mbar_init(b_pvdone, 1);
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
        if (lane == 0) {  // TMA: Q once, then K_0, K_1, V_0, K_2, V_1, ... (consumption order)
            const uint64_t pol_q = policy_evict_first(), pol_kv = policy_evict_first();
            mbar_arrive_expect_tx(b_q, C::TILE);
            const int qrow0 = (b * p.H + kvl * p.group) * p.Tq + qt * 128;
            for (int kb = 0; kb < C::KB; ++kb)
                tma_load_3d(sQ + kb * C::SUB, &tmQ, b_q, 64 * kb, qrow0, 0, pol_q);
            uint32_t idx = 0, ph = 0, armed = 0, armed_par = 0;
            bool ok = true;
            auto load = [&](const CUtensorMap *map, int tile) -> bool {
                if (!mbar_wait(b_kvempty + 8 * idx, ph ^ 1u, lim, W_D_KVEMPTY, abort_flag)) return false;
                mbar_arrive_expect_tx(b_kvfull + 8 * idx, C::TILE);
                armed |= 1u << idx;
                armed_par = (armed_par & ~(1u << idx)) | (ph << idx);
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_3d(sKV + idx * C::TILE + kb * C::SUB, map, b_kvfull + 8 * idx, 64 * kb,
                                128 * (t0 + tile), kvbh, pol_kv);
                if (++idx == (uint32_t)C::NSTAGE) { idx = 0; ph ^= 1u; }
                return true;
            };
            ok = load(&tmK, 0);
            if (ok && n > 1) ok = load(&tmK, 1);
            for (int j = 0; ok && j < n; ++j) {
                ok = load(&tmV, j);
                if (ok && j + 2 < n) ok = load(&tmK, j + 2);
            }
            if (!ok) {
                *abort_flag = 1;
                mbar_wait(b_q, 0, lim, W_D_Q);
                for (int s = 0; s < C::NSTAGE; ++s)
                    if ((armed >> s) & 1u) mbar_wait(b_kvfull + 8 * s, (armed_par >> s) & 1u, lim, W_D_KVFULL);
            }
        }
    } else if (warp == 4) {
        if (lane == 0) {  // MMA issuer
            uint32_t idx = 0, ph = 0;
            bool ok = mbar_wait(b_q, 0, lim, W_D_Q, abort_flag);
            const uint32_t ql = sw128_desc_lo(sQ, 16);
            auto next = [&](uint32_t &slot) -> bool {
                slot = idx;
                const bool r = mbar_wait(b_kvfull + 8 * idx, ph, lim, W_D_KVFULL, abort_flag);
                if (++idx == (uint32_t)C::NSTAGE) { idx = 0; ph ^= 1u; }
                tc_fence_after_sync();
                return r;
            };
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
            uint32_t slot = 0;
            if (ok) ok = next(slot);
            if (ok) qk(0, slot);
            if (ok && n > 1) {
                if ((ok = next(slot))) qk(1, slot);
            }
            for (int j = 0; ok && j < n; ++j) {
                uint32_t vs = 0;
                if (!(ok = next(vs))) break;
                if (!(ok = mbar_wait(b_pfull + 8 * (j & 1), (uint32_t)(j >> 1) & 1u, lim, W_D_PFULL,
                                     abort_flag)))
                    break;
                tc_fence_after_sync();
                const uint32_t vl = sw128_desc_lo(sKV + vs * C::TILE, C::SUB);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + C::TM_O, tmem + C::TM_S + 128 * (j & 1) + 8 * kk,
                           sw128_desc_join(vl + kk * (2048 >> 4), 1024), C::IDESC_PV,
                           (j > 0 || kk > 0) ? 1u : 0u);
                tc_commit(b_pvdone);
                tc_commit(b_kvempty + 8 * vs);
                if (j + 2 < n) {  // the next score tile into the buffer just consumed
                    if (!(ok = next(slot))) break;
                    qk(j & 1, slot);
                }
            }
            if (!ok) {
                *abort_flag = 1;
                tc_commit(b_drain);
                mbar_wait(b_drain, 0, lim, W_D_DRAIN);
            }
        }
    } else if (warp < 4) {  // softmax: thread = packed query row
        const int r = warp * 32 + lane;
        const int pr = qt * 128 + r;
        const bool valid = pr < p.rows;
        const int g = valid ? pr / p.Tq : 0, qi = valid ? pr % p.Tq : 0;
        const int pos = p.Tk - p.Tq + qi;
        const int lim_key = p.causal ? pos : p.Tk - 1;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const float cl2 = p.c_log2;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; ok && j < n; ++j) {
            const int buf = j & 1;
            const bool w = mbar_wait(b_sfull + 8 * buf, (uint32_t)(j >> 1) & 1u, lim, W_D_SFULL, abort_flag);
            if (!(ok = __all_sync(0xffffffffu, w))) break;
            tc_fence_after_sync();
            const uint32_t tS = tmem + lane_off + C::TM_S + 128 * buf;
            float s[128];
            {
                uint32_t rr[128];
                tmem_ld128(tS, rr);
                tmem_wait_ld_regs128(rr);
#pragma unroll
                for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(rr[i]);
            }
            const int key0 = 128 * (t0 + j);
            const bool need_mask = (key0 + 128 > p.Tk) || (p.causal && key0 + 127 > p.Tk - p.Tq);
            if (need_mask) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (key0 + c > lim_key) s[c] = -INFINITY;
            }
            float mx = s[0];
#pragma unroll
            for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
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
                const bool w2 = mbar_wait(b_pvdone, (uint32_t)(j - 1) & 1u, lim, W_D_PVDONE, abort_flag);
                if (!(ok = __all_sync(0xffffffffu, w2))) break;
                tc_fence_after_sync();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t rr[32];
                    tmem_ld32(tmem + lane_off + C::TM_O + 32 * c, rr);
                    tmem_wait_ld_regs(rr);
#pragma unroll
                    for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
                    tmem_st32(tmem + lane_off + C::TM_O + 32 * c, rr);
                }
            }
            l *= alpha;
            const float neg_m = (m == -INFINITY) ? 0.f : -m;
            float ls = 0.f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float p0 = fast_exp2(fmaf(s[64 * h + 2 * i], cl2, neg_m));
                    const float p1 = fast_exp2(fmaf(s[64 * h + 2 * i + 1], cl2, neg_m));
                    ls += p0 + p1;
                    pk[i] = pack_bf16x2(p0, p1);
                }
                tmem_st32(tS + 32 * h, pk);
            }
            l += ls;
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(b_pfull + 8 * buf);
        }
        const bool w = ok && mbar_wait(b_pvdone, (uint32_t)(n - 1) & 1u, lim, W_D_PVDONE, abort_flag);
        if (__all_sync(0xffffffffu, w)) {
            tc_fence_after_sync();
            const size_t row = (size_t)(b * p.H + kvl * p.group + g) * p.Tq + qi;
            const size_t nrows = (size_t)gridDim.y / p.H_kv * p.H * p.Tq;  // B * H * Tq
            const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t rr[32];
                tmem_ld32(tmem + lane_off + C::TM_O + 32 * c, rr);
                tmem_wait_ld_regs(rr);
                if (valid) {
                    float4 *dst = reinterpret_cast<float4 *>(p.part_o + ((size_t)split * nrows + row) * D + 32 * c);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[i] = make_float4(__uint_as_float(rr[4 * i]) * inv, __uint_as_float(rr[4 * i + 1]) * inv,
                                             __uint_as_float(rr[4 * i + 2]) * inv, __uint_as_float(rr[4 * i + 3]) * inv);
                }
            }
            if (valid)
                p.part_lse[(size_t)split * nrows + row] =
                    l > 0.f ? (m + fast_log2(l)) * 0.69314718055994530942f : -INFINITY;
        } else {
            *abort_flag = 1;
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 4) tmem_dealloc(tmem, C::TMEM_COLS);
}

// One warp per query row: merge the splits' (O_s, lse_s).
template <int D>
__global__ void __launch_bounds__(256)
    decode_combine_kernel(const float *__restrict__ part_o, const float *__restrict__ part_lse,
                          __nv_bfloat16 *__restrict__ o, float *__restrict__ lse, long long nrows,
                          int splits)
{
    const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= nrows) return;
    float mx = -INFINITY;
    for (int s = 0; s < splits; ++s) mx = fmaxf(mx, part_lse[(size_t)s * nrows + r]);
    constexpr int PER = D / 32;
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
    float sum = 0.f;
    if (mx != -INFINITY) {
        for (int s = 0; s < splits; ++s) {
            const float ls = part_lse[(size_t)s * nrows + r];
            if (ls == -INFINITY) continue;
            const float w = expf(ls - mx);
            sum += w;
            const float *src = part_o + ((size_t)s * nrows + r) * D + lane * PER;
#pragma unroll
            for (int i = 0; i < PER; ++i) acc[i] = fmaf(w, src[i], acc[i]);
        }
    }
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
    __nv_bfloat16 *dst = o + r * D + lane * PER;
#pragma unroll
    for (int i = 0; i < PER; ++i) dst[i] = __float2bfloat16_rn(acc[i] * inv);
    if (lane == 0) lse[r] = sum > 0.f ? mx + logf(sum) : -INFINITY;
}

}  // namespace attn
