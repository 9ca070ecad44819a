// Gated group RMSNorm, the stage after the SSD scan in a Mamba-2 block (RL-Kernel issue
// page, Figure 2: the scan output y is gated by SiLU of the z branch and normalised over
// groups of 512 channels; the JAX Nemotron 3 Nano page's configuration gives the RMSNorm
// epsilon). Per token t and channel c of group G(c):
//   g[t][c]   = y[t][c] * silu(z[t][c])
//   out[t][c] = g[t][c] * rsqrt(mean_{c' in G(c)} g[t][c']^2 + eps) * weight[c]
// in FP32, rounded to the input dtype. HBM-bound: y and z read once, out written once.
// One warp per (token, group): a lane holds group/32 consecutive channels, the group's
// sum of squares is a warp reduction; a warp keeps its weight slice in registers over a
// run of tokens.
#pragma once

#include "ssd_common.cuh"

namespace ssd {

constexpr int kNormTokens = 16;      // tokens per warp
constexpr int kNormWarps = 8;        // warps per block

__device__ __forceinline__ void norm_load8(const float* p, float (&o)[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
__device__ __forceinline__ void norm_load8(const __nv_bfloat16* p, float (&o)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = __uint_as_float(w[i] << 16);
        o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void norm_store8(float* p, const float (&v)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void norm_store8(__nv_bfloat16* p, const float (&v)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// silu(z) with the hardware base-2 exponential and reciprocal.
__device__ __forceinline__ float norm_silu(float v) {
    float e, r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-v * 1.4426950408889634f));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.f + e));
    return v * r;
}

// VPL = 8-channel vectors per lane (group = 256 * VPL channels).
template <typename T, int VPL>
__global__ void __launch_bounds__(32 * kNormWarps)
k_gated_rmsnorm(const T* __restrict__ y, const T* __restrict__ z, const float* __restrict__ weight,
                T* __restrict__ out, int64_t ntok, int channels, float eps) {
    constexpr int GS = 256 * VPL;
    const int lane = threadIdx.x & 31;
    const int64_t wid = (int64_t)blockIdx.x * kNormWarps + (threadIdx.x >> 5);
    const int ngroups = channels / GS;
    const int grp = (int)(wid % ngroups);
    const int64_t t0 = (wid / ngroups) * kNormTokens;
    if (t0 >= ntok) return;
    const int64_t t1 = t0 + kNormTokens < ntok ? t0 + kNormTokens : ntok;
    const int cb = grp * GS + lane * 8 * VPL;           // this lane's first channel
    float wv[VPL][8];
#pragma unroll
    for (int v = 0; v < VPL; ++v) norm_load8(weight + cb + 8 * v, wv[v]);
    const float inv = 1.f / (float)GS;
    for (int64_t t = t0; t < t1; ++t) {
        float g[VPL][8];
        float ss = 0.f;
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            float yv[8], zv[8];
            norm_load8(y + t * channels + cb + 8 * v, yv);
            norm_load8(z + t * channels + cb + 8 * v, zv);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                g[v][j] = yv[j] * norm_silu(zv[j]);
                ss = fmaf(g[v][j], g[v][j], ss);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float rstd = rsqrtf(fmaf(ss, inv, eps));
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            float o[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) o[j] = g[v][j] * rstd * wv[v][j];
            norm_store8(out + t * channels + cb + 8 * v, o);
        }
    }
}

}  // namespace ssd
