// unfused.cuh -- the materialised three-kernel attention forward.
//
// "Why Attention Is Difficult to Optimize", section "Storing and Rereading
// Large Intermediate Matrices": the kernel computing QK^T stores the score
// matrix S and finishes; the next kernel reads S, scales, masks and applies
// softmax and stores P; the last kernel reads P and multiplies it by V.  S and
// P are T x T per head at 2 bytes per value (bf16), so this path moves
// 2 * 2 * T^2 * 2 bytes per head through device memory that the fused kernel
// never touches.  It exists to measure that traffic.
//
//   K1 s_gemm_kernel     S = Q K^T   (tcgen05, 128x128 tiles, TMA operands;
//                        persistent, one CTA per SM over the tiles)
//   K2 softmax_kernel    P = softmax(mask(scale * S)), lse   (one warp per row,
//                        warp-shuffle reduction of (max, sum) pairs)
//   K3 pv_gemm_kernel    O = P V     (tcgen05, 128 x d_h tiles, 4-stage TMA ring)
// Causal: what the mask hides is neither computed nor moved.  K1 skips the
// 128 x 128 score tiles above the diagonal, K2 reads a row's scores only up
// to the row itself and writes its probabilities up to the end of the row's
// 128-row block (zeros past the diagonal), and K3 stops at each query
// block's diagonal; the rest of S and P is left untouched.
#pragma once

#include "sm100.cuh"

namespace attn {

// TMA store helpers (only K1 stores through TMA).
// 3-D tiled store of a box from shared memory at `src` to the tensor at
// (x, y, z): x a multiple of 8 elements, every coordinate >= 0.  Tracked by
// the issuing thread's bulk-async group (tma_store_commit / _wait_read).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, uint32_t src, int x, int y,
                                             int z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(src), "r"(x), "r"(y), "r"(z)
        : "memory");
}

__device__ __forceinline__ void tma_store_commit()
{
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until at most the most recently committed store group has not yet
// read its shared memory (every older group's source may be reused).
__device__ __forceinline__ void tma_store_wait_read_1()
{
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// Waits until every committed store has completed.
__device__ __forceinline__ void tma_store_wait_all()
{
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Orders this thread's ordinary shared-memory writes before later accesses by
// the asynchronous (TMA) proxy.
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

struct UnfusedParams {
    int BH, T, causal;
    float c_log2;
    unsigned long long limit_ns;
};

enum : unsigned int { W_K1 = 32, W_K3_FULL, W_K3_EMPTY, W_K3_DONE };

// ---------------------------------------------------------------------------
// K1: S = Q K^T, raw (unscaled) bf16, as a persistent kernel: one CTA per SM
// walks the 128 x 128 tiles of S (all of them, or under the causal mask the
// tiles at or below the diagonal), tile k*G + c for CTA c of G.  192 threads:
//   warp 0     TMA producer: Q_m and K_n of each tile into a ring of NST
//              stages (4 at d_h = 64, 2 at d_h = 128)
//   warp 1     MMA issuer: S into one of two 128-column TMEM buffers
//   warps 2-5  epilogue (thread = row = TMEM lane): TMEM -> bf16 -> one of two
//              shared-memory staging tiles (128-byte swizzled, two 64-key
//              boxes) -> two TMA stores, whole 128-byte lines
// so loading tile k+1, computing it and storing tile k overlap.
// ---------------------------------------------------------------------------
template <int D>
struct K1Cfg {
    static constexpr int KB = D / 64;
    static constexpr int SUB = 128 * 128;           // 128 rows x 128 bytes
    static constexpr int TILE = 128 * D * 2;        // one Q or K tile
    static constexpr int NST = D == 64 ? 4 : 2;  // Q/K stages: 4 x 32 KB at d_h = 64, 2 x 64 KB at 128
    static constexpr int STAGE = 2 * TILE;          // Q_m and K_n
    static constexpr int STG = 128 * 128 * 2;       // one S tile (bf16)
    static constexpr int OFF_STG = NST * STAGE;
    static constexpr int OFF_BAR = OFF_STG + 2 * STG;
    static constexpr int NBAR = 2 * NST + 5;        // full, empty, tfull[2], tempty[2], drain
    static constexpr int SMEM = 1024 + OFF_BAR + NBAR * 8 + 16;
    static constexpr int THREADS = 192;
    static constexpr uint32_t TMEM_COLS = 256;
};

// Tile l of a head's list -> (query block m, key block n).  Causal: the
// lower triangle row by row, n <= m.
__device__ __forceinline__ void k1_tile(const UnfusedParams &p, long long l, int nt, int &m, int &n)
{
    if (!p.causal) {
        m = (int)(l / nt);
        n = (int)(l - (long long)m * nt);
        return;
    }
    int mm = (int)((sqrtf(8.f * (float)l + 1.f) - 1.f) * 0.5f);
    while ((long long)(mm + 1) * (mm + 2) / 2 <= l) ++mm;
    while ((long long)mm * (mm + 1) / 2 > l) --mm;
    m = mm;
    n = (int)(l - (long long)mm * (mm + 1) / 2);
}

// All 128 epilogue threads: true iff every one of them passes true.
__device__ __forceinline__ bool epi_all(bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(v ? 1u : 0u)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int D>
__global__ void __launch_bounds__(192, 1)
    s_gemm_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmS, const UnfusedParams p)
{
    using C = K1Cfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t b_full = base + C::OFF_BAR;          // [NST]
    const uint32_t b_empty = b_full + 8 * C::NST;       // [NST]
    const uint32_t b_tfull = b_empty + 8 * C::NST;      // [2] S of TMEM buffer b computed
    const uint32_t b_tempty = b_tfull + 16;             // [2] TMEM buffer b read out
    const uint32_t b_drain = b_tempty + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + C::OFF_BAR + C::NBAR * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = (int)gridDim.x;
    const int nt = p.T / 128;
    const long long tph = p.causal ? (long long)nt * (nt + 1) / 2 : (long long)nt * nt;
    const long long total = tph * p.BH;
    const uint64_t lim = p.limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(b_full + 8 * s, 1);
            mbar_init(b_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(b_tfull + 8 * b, 1);
            mbar_init(b_tempty + 8 * b, 128);
        }
        mbar_init(b_drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {  // TMA producer
            const uint64_t pol = policy_evict_last();
            uint32_t armed = 0, armed_par = 0;
            bool ok = true;
            int k = 0;
            for (long long i = blockIdx.x; i < total; i += G, ++k) {
                const int s = k % C::NST;
                const uint32_t par = (uint32_t)(k / C::NST) & 1u;
                if (!mbar_wait(b_empty + 8 * s, par ^ 1u, lim, W_K1, abort_flag)) { ok = false; break; }
                const int bh = (int)(i / tph);
                int m, n;
                k1_tile(p, i - (long long)bh * tph, nt, m, n);
                const uint32_t st = base + s * C::STAGE;
                mbar_arrive_expect_tx(b_full + 8 * s, C::STAGE);
                armed |= 1u << s;
                armed_par = (armed_par & ~(1u << s)) | (par << s);
                for (int kb = 0; kb < C::KB; ++kb) {
                    tma_load_3d(st + kb * C::SUB, &tmQ, b_full + 8 * s, 64 * kb, 128 * m, bh, pol);
                    tma_load_3d(st + C::TILE + kb * C::SUB, &tmK, b_full + 8 * s, 64 * kb, 128 * n, bh, pol);
                }
            }
            if (!ok) {
                *abort_flag = 1;
                for (int s = 0; s < C::NST; ++s)
                    if ((armed >> s) & 1u) mbar_wait(b_full + 8 * s, (armed_par >> s) & 1u, lim, W_K1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {  // MMA issuer
            constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
            bool ok = true;
            int k = 0;
            for (long long i = blockIdx.x; i < total; i += G, ++k) {
                const int s = k % C::NST, b = k & 1;
                if (!(ok = mbar_wait(b_full + 8 * s, (uint32_t)(k / C::NST) & 1u, lim, W_K1, abort_flag)))
                    break;
                if (!(ok = mbar_wait(b_tempty + 8 * b, ((uint32_t)(k >> 1) & 1u) ^ 1u, lim, W_K1, abort_flag)))
                    break;
                tc_fence_after_sync();
                const uint32_t sq = base + s * C::STAGE, sk = sq + C::TILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::SUB + (kk & 3) * 32;
                    mma_ss(tmem + 128 * b, sw128_desc(sq + off, 16, 1024), sw128_desc(sk + off, 16, 1024),
                           idesc, kk > 0 ? 1u : 0u);
                }
                tc_commit(b_empty + 8 * s);
                tc_commit(b_tfull + 8 * b);
            }
            if (!ok) *abort_flag = 1;
            tc_commit(b_drain);  // every MMA issued above has completed before TMEM is freed
            mbar_wait(b_drain, 0, lim, W_K1);
        }
    } else {  // epilogue warpgroup: warps 2-5, TMEM lane quarter warp & 3
        const int r = (warp & 3) * 32 + lane;  // row of the tile
        const uint32_t taddr_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const bool storer = (warp == 2 && lane == 0);
        int k = 0;
        for (long long i = blockIdx.x; i < total; i += G, ++k) {
            const int b = k & 1;
            const bool w = mbar_wait(b_tfull + 8 * b, (uint32_t)(k >> 1) & 1u, lim, W_K1, abort_flag);
            if (!epi_all(w)) {
                if (threadIdx.x == 64) *abort_flag = 1;
                break;
            }
            tc_fence_after_sync();
            uint32_t pk[64];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t rg[32];
                tmem_ld32(taddr_lane + 128 * b + 32 * c, rg);
                tmem_wait_ld_regs(rg);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[16 * c + e] = pack_bf16x2(__uint_as_float(rg[2 * e]), __uint_as_float(rg[2 * e + 1]));
            }
            tc_fence_before_sync();
            mbar_arrive(b_tempty + 8 * b);  // TMEM buffer b may take the next tile
            // staging buffer b: the store issued from it two tiles ago has read it
            if (storer) tma_store_wait_read_1();
            epi_sync();
            uint8_t *stg = gbase + C::OFF_STG + b * C::STG;
#pragma unroll
            for (int c = 0; c < 16; ++c) {  // 16-byte chunk c: keys 8c .. 8c+7, box c / 8
                uint8_t *row_base = stg + (c >> 3) * C::SUB + r * 128;
                *reinterpret_cast<uint4 *>(row_base + 16 * ((c & 7) ^ (r & 7))) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            }
            fence_proxy_async_smem();
            epi_sync();
            if (storer) {
                const int bh = (int)(i / tph);
                int m, n;
                k1_tile(p, i - (long long)bh * tph, nt, m, n);
                const uint32_t sa = base + C::OFF_STG + b * C::STG;
                tma_store_3d(&tmS, sa, 128 * n, 128 * m, bh);
                tma_store_3d(&tmS, sa + C::SUB, 128 * n + 64, 128 * m, bh);
                tma_store_commit();
            }
        }
        if (storer) tma_store_wait_all();  // the staging tiles stay valid until the stores finish
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ---------------------------------------------------------------------------
// K2: row softmax, one warp per query row, 8 rows per 256-thread CTA.
// Pass 1 reads the row once (16-byte loads) and keeps a per-lane running
// (max, sum) in the log2 domain; a butterfly of warp shuffles merges the 32
// pairs.  Pass 2 re-reads the row (L2-resident by then) and writes
// P = exp2(s * scale * log2e - m) / l, exactly 0 where masked.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void merge_ml(float &m, float &l, float m2, float l2)
{
    const float mn = fmaxf(m, m2);
    if (mn == -INFINITY) return;  // both empty
    l = l * fast_exp2(m - mn) + l2 * fast_exp2(m2 - mn);
    m = mn;
}

__global__ void __launch_bounds__(256)
    softmax_kernel(const __nv_bfloat16 *__restrict__ S, __nv_bfloat16 *__restrict__ P,
                   float *__restrict__ lse, const UnfusedParams p)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long grow = (long long)blockIdx.x * 8 + warp;  // flat row over B*H*T
    if (grow >= (long long)p.BH * p.T) return;
    const int row = (int)(grow % p.T);
    const int T = p.T;
    const float c = p.c_log2;
    const int lim_key = p.causal ? row : T - 1;
    const uint4 *src = reinterpret_cast<const uint4 *>(S + grow * (long long)T);
    uint4 *dst = reinterpret_cast<uint4 *>(P + grow * (long long)T);
    const int nchunk = T / 8;
    // causal: scores are read up to the row itself, probabilities written up
    // to the end of the row's 128-row block (what K3 multiplies)
    const int rd_chunks = p.causal ? min(nchunk, (row >> 3) + 1) : nchunk;
    const int wr_chunks = p.causal ? min(nchunk, ((row | 127) + 1) >> 3) : nchunk;

    // Each lane has U 16-byte loads in flight per step (the row's memory
    // parallelism, not the exponentials, bounds this kernel).  Pass 1: the
    // lane's online (max, sum) over its chunks; the second read of S is its
    // last use (evict first).
    constexpr int U = 4;
    float m = -INFINITY, l = 0.f;
    for (int base = lane; base < rd_chunks; base += 32 * U) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int ch = base + 32 * u;
            v[u] = ch < rd_chunks ? src[ch] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int ch = base + 32 * u;
            if (ch >= rd_chunks) break;
            const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            float x[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                x[2 * i] = __uint_as_float(w[i] << 16) * c;
                x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u) * c;
            }
            float cm = -INFINITY;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (ch * 8 + i > lim_key) x[i] = -INFINITY;
                cm = fmaxf(cm, x[i]);
            }
            if (cm == -INFINITY) continue;
            const float mn = fmaxf(m, cm);
            float add = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) add += fast_exp2(x[i] - mn);
            l = l * fast_exp2(m - mn) + add;
            m = mn;
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
        const float l2 = __shfl_xor_sync(0xffffffffu, l, off);
        merge_ml(m, l, m2, l2);
    }
    const float inv_l = 1.f / l;
    // Pass 2: P, and zeros from the diagonal to the end of the row's block.
    for (int base = lane; base < wr_chunks; base += 32 * U) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int ch = base + 32 * u;
            v[u] = ch < rd_chunks ? __ldcs(src + ch) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int ch = base + 32 * u;
            if (ch >= wr_chunks) break;
            if (ch >= rd_chunks) {
                dst[ch] = make_uint4(0u, 0u, 0u, 0u);
                continue;
            }
            const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int k0 = ch * 8 + 2 * i;
                const float a = (k0 > lim_key)
                                    ? 0.f
                                    : fast_exp2(__uint_as_float(w[i] << 16) * c - m) * inv_l;
                const float b = (k0 + 1 > lim_key)
                                    ? 0.f
                                    : fast_exp2(__uint_as_float(w[i] & 0xFFFF0000u) * c - m) * inv_l;
                o[i] = pack_bf16x2(a, b);
            }
            dst[ch] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
    if (lane == 0) lse[grow] = (m + fast_log2(l)) * 0.69314718055994530942f;
}

// ---------------------------------------------------------------------------
// K3: O = P V, one CTA per 128 query rows of one head (grid: T/128, B*H);
// 128 threads: thread 0 produces (TMA), thread 32 issues MMAs, all four warps
// run the epilogue.  Keys advance 64 at a time through a 4-stage ring of
// (P chunk 128 x 64, V chunk 64 x d_h).
// ---------------------------------------------------------------------------
template <int D>
struct PvCfg {
    static constexpr int KB = D / 64;
    static constexpr int P_BYTES = 128 * 128;    // 128 rows x 64 keys x 2 B
    static constexpr int V_SUB = 64 * 128;       // 64 keys x 64 d x 2 B
    static constexpr int V_BYTES = KB * V_SUB;
    static constexpr int STAGE = P_BYTES + V_BYTES;
    static constexpr int NST = 4;
    static constexpr int SMEM = 1024 + NST * STAGE + 2 * NST * 8 + 8 + 16;
};

template <int D>
__global__ void __launch_bounds__(128)
    pv_gemm_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmV,
                   __nv_bfloat16 *O, const UnfusedParams p)
{
    using C = PvCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t b_full = base + C::NST * C::STAGE;
    const uint32_t b_empty = b_full + 8 * C::NST;
    const uint32_t b_done = b_empty + 8 * C::NST;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + C::NST * C::STAGE + 16 * C::NST + 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * 128, bh = blockIdx.y;
    // causal: the 64-key chunks up to this query block's diagonal
    const int nchunks = p.causal ? min(p.T / 64, (m0 + 128) / 64) : p.T / 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(b_full + 8 * s, 1);
            mbar_init(b_empty + 8 * s, 1);
        }
        mbar_init(b_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(smem_addr(tmem_slot), D < 32 ? 32 : D);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (threadIdx.x == 0) {  // producer
        const uint64_t pol_p = policy_evict_first(), pol_v = policy_evict_last();
        uint32_t idx = 0, ph = 0;
        bool ok = true;
        bool armed[C::NST] = {};
        uint32_t armed_ph[C::NST] = {};
        for (int ch = 0; ch < nchunks; ++ch) {
            if (!mbar_wait(b_empty + 8 * idx, ph ^ 1u, p.limit_ns, W_K3_EMPTY, abort_flag)) {
                ok = false;
                break;
            }
            const uint32_t st = base + idx * C::STAGE;
            mbar_arrive_expect_tx(b_full + 8 * idx, C::STAGE);
            armed[idx] = true;
            armed_ph[idx] = ph;
            tma_load_3d(st, &tmP, b_full + 8 * idx, 64 * ch, m0, bh, pol_p);
            for (int kb = 0; kb < C::KB; ++kb)
                tma_load_3d(st + C::P_BYTES + kb * C::V_SUB, &tmV, b_full + 8 * idx, 64 * kb, 64 * ch,
                            bh, pol_v);
            if (++idx == (uint32_t)C::NST) { idx = 0; ph ^= 1u; }
        }
        if (!ok) {
            *abort_flag = 1;
            for (int s = 0; s < C::NST; ++s)
                if (armed[s]) mbar_wait(b_full + 8 * s, armed_ph[s], p.limit_ns, W_K3_FULL);
        }
    } else if (threadIdx.x == 32) {  // MMA issuer
        constexpr uint32_t idesc = idesc_bf16_f32(128, D, true);
        uint32_t idx = 0, ph = 0;
        bool ok = true;
        for (int ch = 0; ch < nchunks; ++ch) {
            if (!mbar_wait(b_full + 8 * idx, ph, p.limit_ns, W_K3_FULL, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            const uint32_t st = base + idx * C::STAGE;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ss(tmem, sw128_desc(st + kk * 32, 16, 1024),
                       sw128_desc(st + C::P_BYTES + kk * 2048, C::V_SUB, 1024), idesc,
                       (ch > 0 || kk > 0) ? 1u : 0u);
            tc_commit(b_empty + 8 * idx);
            if (++idx == (uint32_t)C::NST) { idx = 0; ph ^= 1u; }
        }
        if (!ok) *abort_flag = 1;
        tc_commit(b_done);  // fires once every MMA above has completed
    }
    __syncwarp();
    const bool w = mbar_wait(b_done, 0, p.limit_ns, W_K3_DONE);
    const bool good = __syncthreads_and((w && !*abort_flag) ? 1 : 0) != 0;
    if (good) {
        tc_fence_after_sync();
        const int row = m0 + warp * 32 + lane;
        const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
        __nv_bfloat16 *dst_row = O + ((size_t)bh * p.T + row) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(taddr + 32 * c, r);
            tmem_wait_ld_regs(r);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
            uint4 *d4 = reinterpret_cast<uint4 *>(dst_row + 32 * c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, D < 32 ? 32 : D);
}

}  // namespace attn
