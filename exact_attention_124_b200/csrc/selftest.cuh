// selftest.cuh -- one-tile kernels that check the tcgen05 building blocks the
// attention kernels use (descriptor bits, swizzle, TMEM packing), plus a
// bounded-wait failure check.  Each is one CTA of 128 threads.
//
// The two tile products are the matrix multiplications of scaled dot-product
// attention ("Attention Mechanism: Computation & Memory Patterns", section 1:
// S = QK^T and O = PV) on a single 128-row tile.
#pragma once

#include "sm100.cuh"

namespace attn {

enum : unsigned int { W_ST_LOAD = 64, W_ST_MMA, W_ST_NEVER };

// s[i][j] = sum_c q[i][c] k[j][c]: TMA loads (128-byte swizzle), an SS MMA
// exactly like the fused kernel's score MMA, then a TMEM read-back.
template <int D>
__global__ void __launch_bounds__(128)
    selftest_qk_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK, float *s,
                       unsigned long long limit_ns)
{
    constexpr int KB = D / 64, SUB = 128 * 128, TILE = 128 * D * 2;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t sQ = base, sK = base + TILE, b_load = base + 2 * TILE, b_mma = b_load + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + 2 * TILE + 16);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(b_load, 1);
        mbar_init(b_mma, 1);
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(smem_addr(tmem_slot), 128);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    int ok = 1;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(b_load, 2 * TILE);
        for (int kb = 0; kb < KB; ++kb) {
            tma_load_3d(sQ + kb * SUB, &tmQ, b_load, 64 * kb, 0, 0, policy_evict_first());
            tma_load_3d(sK + kb * SUB, &tmK, b_load, 64 * kb, 0, 0, policy_evict_first());
        }
        ok = mbar_wait(b_load, 0, limit_ns, W_ST_LOAD);
        if (ok) {
            tc_fence_after_sync();
            constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk >> 2) * SUB + (kk & 3) * 32;
                mma_ss(tmem, sw128_desc(sQ + off, 16, 1024), sw128_desc(sK + off, 16, 1024), idesc,
                       kk > 0 ? 1u : 0u);
            }
        }
        tc_commit(b_mma);
    }
    __syncwarp();
    const bool w = mbar_wait(b_mma, 0, limit_ns, W_ST_MMA);
    ok = __syncthreads_and((w && __shfl_sync(0xffffffffu, ok, 0)) ? 1 : 0);
    if (ok) {
        tc_fence_after_sync();
        const int row = warp * 32 + lane;
        for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 32 * c, r);
            tmem_wait_ld_regs(r);
            for (int i = 0; i < 32; ++i) s[row * 128 + 32 * c + i] = __uint_as_float(r[i]);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

// o[i][c] = sum_j p[i][j] v[j][c]: each thread writes its row of P into TMEM
// as packed bf16 pairs (tcgen05.st, exactly as the fused softmax does), V
// arrives by TMA, and a TS MMA (A from TMEM, B MN-major) accumulates.
template <int D>
__global__ void __launch_bounds__(128)
    selftest_pv_kernel(const __nv_bfloat16 *__restrict__ P, const __grid_constant__ CUtensorMap tmV,
                       float *o, unsigned long long limit_ns)
{
    constexpr int KB = D / 64, SUB = 128 * 128, TILE = 128 * D * 2;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t sV = base, b_load = base + TILE, b_mma = b_load + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + TILE + 16);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(b_load, 1);
        mbar_init(b_mma, 1);
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(smem_addr(tmem_slot), 256);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;       // P at columns [0, 64), O at [128, 128 + D)
    const int row = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    {
        const uint32_t *prow = reinterpret_cast<const uint32_t *>(P + row * 128);
        for (int h = 0; h < 2; ++h) {
            uint32_t pk[32];
            for (int i = 0; i < 32; ++i) pk[i] = prow[32 * h + i];
            tmem_st32(tmem + lane_off + 32 * h, pk);
        }
        tmem_wait_st();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    int ok = 1;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(b_load, TILE);
        for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(sV + kb * SUB, &tmV, b_load, 64 * kb, 0, 0, policy_evict_first());
        ok = mbar_wait(b_load, 0, limit_ns, W_ST_LOAD);
        if (ok) {
            tc_fence_after_sync();
            constexpr uint32_t idesc = idesc_bf16_f32(128, D, true);
            for (int kk = 0; kk < 8; ++kk)
                mma_ts(tmem + 128, tmem + 8 * kk, sw128_desc(sV + kk * 2048, SUB, 1024), idesc,
                       kk > 0 ? 1u : 0u);
        }
        tc_commit(b_mma);
    }
    __syncwarp();
    const bool w = mbar_wait(b_mma, 0, limit_ns, W_ST_MMA);
    ok = __syncthreads_and((w && __shfl_sync(0xffffffffu, ok, 0)) ? 1 : 0);
    if (ok) {
        tc_fence_after_sync();
        for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_off + 128 + 32 * c, r);
            tmem_wait_ld_regs(r);
            for (int i = 0; i < 32; ++i) o[row * D + 32 * c + i] = __uint_as_float(r[i]);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// A barrier nobody arrives on: the bounded wait must give up and record
// ATTN_ERR_TIMEOUT, and the kernel must return normally.
__global__ void selftest_timeout_kernel(unsigned long long limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_addr(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(b, 0, limit_ns, W_ST_NEVER);
    __syncthreads();
}

}  // namespace attn
