// Diagnostic kernel for the UMMA operand formats the tensor-core path relies on.
// It multiplies two 128x128 bf16 matrices four ways, each exercising a different
// pairing of shared-memory layouts (TMA-written / thread-written, K-major /
// MN-major), so a descriptor or swizzle mistake shows up in one product only:
//   r0[t][s] = sum_k X1[t][k] X2[s][k]   A: TMA K-major,    B: TMA K-major   (N=128)
//   r1[t][p] = sum_k X1[t][k] X2[k][p]   A: thread K-major, B: TMA MN-major  (N=64)
//   r2[m][p] = sum_k X1[k][m] X2[k][p]   A: TMA MN-major,   B: thread MN-major
//   r3[t][p] = sum_k X1[t][k] X2[k][p]   A: TMA K-major,    B: thread MN-major
//   r4[t][p] = sum_k X1[t][k] X2[k][p]   A: thread-written TMEM, B: TMA MN-major
// out is [5][128][128] fp32; columns >= 64 of r1..r4 are written as zero.
#pragma once

#include "ssd_tc_ptx.cuh"

namespace ssd {
namespace tc {

constexpr int kSelftestSmem = 4 * 32768 + 1024 + 64;

__global__ void __launch_bounds__(128)
k_umma_selftest(const __grid_constant__ CUtensorMap map1, const __grid_constant__ CUtensorMap map2,
                const __nv_bfloat16* __restrict__ X1, const __nv_bfloat16* __restrict__ X2,
                float* __restrict__ out) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* x1t = sm;                 // [2][128][64] bf16, TMA
    uint8_t* x2t = sm + 32768;         // [2][128][64] bf16, TMA
    uint8_t* twa = sm + 65536;         // [2][128][64] bf16, thread-written K-major copy of X1
    uint8_t* twb = sm + 98304;         // [128][64]   bf16, thread-written MN-major copy of X2[:, :64]
    __shared__ uint64_t bar_tma, bar_mma;
    __shared__ uint32_t tmem_slot;
    const int tid = threadIdx.x, warp = tid >> 5;

    if (tid == 0) {
        mbar_init(&bar_tma, 1);
        mbar_init(&bar_mma, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_slot;

    if (tid == 0) {
        mbar_arrive_expect_tx(&bar_tma, 4 * 16384);
        tma_load_3d(x1t, &map1, &bar_tma, 0, 0, 0);
        tma_load_3d(x1t + 16384, &map1, &bar_tma, 64, 0, 0);
        tma_load_3d(x2t, &map2, &bar_tma, 0, 0, 0);
        tma_load_3d(x2t + 16384, &map2, &bar_tma, 64, 0, 0);
    }
    // Thread-written operands.
    {
        const int r = tid;
        const uint4* src1 = reinterpret_cast<const uint4*>(X1 + r * 128);
        const uint4* src2 = reinterpret_cast<const uint4*>(X2 + r * 128);
        for (int j = 0; j < 2; ++j)
            for (int c = 0; c < 8; ++c) {
                uint4 v = src1[j * 8 + c];
                st_shared_v4(smem_u32(twa) + j * 16384 + swz(r, c), v.x, v.y, v.z, v.w);
            }
        for (int c = 0; c < 8; ++c) {
            uint4 v = src2[c];
            st_shared_v4(smem_u32(twb) + swz(r, c), v.x, v.y, v.z, v.w);
        }
    }
    // A operand of r4 in TMEM: row r (lane r) = X1[r][:], bf16 pairs per column 320..383.
    {
        const int r = tid;
        const uint32_t* src = reinterpret_cast<const uint32_t*>(X1 + r * 128);
        for (int q = 0; q < 2; ++q) {
            uint32_t v[32];
            for (int j = 0; j < 32; ++j) v[j] = src[q * 32 + j];
            tmem_st32(tmem_addr(tbase, warp * 32, 320 + q * 32), v);
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    bool ok = __syncthreads_and(mbar_wait(&bar_tma, 0));

    if (tid == 0 && ok) {
        tc_fence_after();
        const uint32_t a1 = smem_u32(x1t), a2 = smem_u32(x2t), ta = smem_u32(twa), tb = smem_u32(twb);
        for (int k = 0; k < 8; ++k)
            umma_bf16(tbase + 0, desc_kmajor(a1, 128, k), desc_kmajor(a2, 128, k), idesc_bf16(128, 128, 0, 0), k > 0);
        for (int k = 0; k < 8; ++k)
            umma_bf16(tbase + 128, desc_kmajor(ta, 128, k), desc_mnmajor(a2, k, 16384), idesc_bf16(128, 64, 0, 1),
                      k > 0);
        for (int k = 0; k < 8; ++k)
            umma_bf16(tbase + 192, desc_mnmajor(a1, k, 16384), desc_mnmajor(tb, k, 16384),
                      idesc_bf16(128, 64, 1, 1), k > 0);
        for (int k = 0; k < 8; ++k)
            umma_bf16(tbase + 256, desc_kmajor(a1, 128, k), desc_mnmajor(tb, k, 16384), idesc_bf16(128, 64, 0, 1),
                      k > 0);
        for (int k = 0; k < 8; ++k)
            umma_bf16_ts(tbase + 384, tbase + 320 + 8 * k, desc_mnmajor(a2, k, 16384), idesc_bf16(128, 64, 0, 1),
                         k > 0);
        umma_commit(&bar_mma);
    }
    __syncwarp();
    if (ok) ok = mbar_wait(&bar_mma, 0);
    ok = __syncthreads_and(ok);
    tc_fence_after();
    const int row = warp * 32 + (tid & 31);
    const uint32_t lane_base = tmem_addr(tbase, warp * 32, 0);
    uint32_t r[32];
    for (int q = 0; q < 4; ++q) {
        tmem_ld32(lane_base + q * 32, r);
        tmem_wait_ld();
        for (int j = 0; j < 32; ++j) out[(0 * 128 + row) * 128 + q * 32 + j] = ok ? __uint_as_float(r[j]) : 0.f;
    }
    for (int m = 1; m < 5; ++m) {
        const uint32_t col = m < 4 ? 128 + (m - 1) * 64 : 384;
        for (int q = 0; q < 2; ++q) {
            tmem_ld32(lane_base + col + q * 32, r);
            tmem_wait_ld();
            for (int j = 0; j < 32; ++j)
                out[(m * 128 + row) * 128 + q * 32 + j] = ok ? __uint_as_float(r[j]) : 0.f;
        }
        for (int j = 64; j < 128; ++j) out[(m * 128 + row) * 128 + j] = 0.f;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

}  // namespace tc
}  // namespace ssd
