// Decode: one recurrent state update per sequence and token (RL-Kernel issue page, §1:
// rollout decode advances the SSM state one token at a time; §2: the upstream decode
// path is the conv-state update followed by the selective state update).
//
//   dt = softplus(dt_raw + dt_bias[h]);  h <- exp(dt*A[h]) h + dt x B^T;  y = h.C + D x
//
// The FP32 state ([nseq,H,P,N], 2 MiB per sequence at H=64, P=64, N=128) dominates
// the traffic: every step reads and rewrites it once, so the kernel is an HBM stream.
// One block per (sequence, head); a state row of N floats is read with 16-byte
// vector loads by N/4 lanes, several rows are loaded before any is written back
// (memory-level parallelism), and the row's y is a shuffle reduction.
#pragma once

#include "ssd_common.cuh"

namespace ssd {

constexpr int kDecodeThreads = 128;

template <typename T, int P, int N>
__global__ void __launch_bounds__(kDecodeThreads)
k_state_update(float* __restrict__ state, const T* __restrict__ x, const float* __restrict__ dt_raw,
               const float* __restrict__ dt_bias, const float* __restrict__ A,
               const T* __restrict__ B, const T* __restrict__ C, const float* __restrict__ D,
               T* __restrict__ y, int H, int G) {
    constexpr int NV = N / 4;              // lanes per state row
    constexpr int RPW = 32 / NV;           // rows per warp per pass
    constexpr int WARPS = kDecodeThreads / 32;
    constexpr int ROWS_PER_PASS = RPW * WARPS;
    constexpr int PASSES = (P + ROWS_PER_PASS - 1) / ROWS_PER_PASS;
    constexpr int U = PASSES < 4 ? PASSES : 4;   // rows in flight per thread

    const int sh = blockIdx.x;
    const int s = sh / H, h = sh % H, g = h / (H / G);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c4 = lane % NV, roff = lane / NV;

    const float a = A[h];
    if (!(a <= 0.f) || isinf(a)) latch_error(SSD_ERR_INVALID_ARG);
    const float dt = softplus_f32(dt_raw[(int64_t)s * H + h] + dt_bias[h]);
    const float decay = expf(dt * a);
    const float Dh = D[h];
    const float4 bv = load4(B + ((int64_t)s * G + g) * N + 4 * c4);
    const float4 cv = load4(C + ((int64_t)s * G + g) * N + 4 * c4);
    const T* xh = x + ((int64_t)s * H + h) * P;
    float* st = state + ((int64_t)s * H + h) * P * N;
    T* yh = y + ((int64_t)s * H + h) * P;

    for (int pass = 0; pass < PASSES; pass += U) {
        float4 v[U];
        float xv[U];
        int prow[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            prow[u] = (pass + u) * ROWS_PER_PASS + warp * RPW + roff;
            if (prow[u] < P && pass + u < PASSES) {
                v[u] = __ldcs(reinterpret_cast<const float4*>(st + prow[u] * N + 4 * c4));
                xv[u] = to_f32(xh[prow[u]]);
            } else {
                v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                xv[u] = 0.f;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const float dx = dt * xv[u];
            float4 w;
            w.x = fmaf(decay, v[u].x, dx * bv.x);
            w.y = fmaf(decay, v[u].y, dx * bv.y);
            w.z = fmaf(decay, v[u].z, dx * bv.z);
            w.w = fmaf(decay, v[u].w, dx * bv.w);
            const bool live = prow[u] < P && pass + u < PASSES;
            if (live) __stcs(reinterpret_cast<float4*>(st + prow[u] * N + 4 * c4), w);
            float part = w.x * cv.x + w.y * cv.y + w.z * cv.z + w.w * cv.w;
#pragma unroll
            for (int off = NV / 2; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
            if (live && c4 == 0) yh[prow[u]] = from_f32<T>(part + Dh * xv[u]);
        }
    }
}

}  // namespace ssd
