// Shared device helpers and the host-side plan of one ssd_scan_fwd call.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd.h"

namespace ssd {

// ---------------------------------------------------------------------------------
// Device error word: the first error a kernel finds is latched here (0 = none);
// ssd_get_device_status() reads and clears it.
__device__ int g_device_error = 0;

__device__ __forceinline__ void latch_error(int code) { atomicCAS(&g_device_error, 0, code); }

// ---------------------------------------------------------------------------------
// Element access for the two input dtypes.
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// Four consecutive elements starting at p (16-byte aligned for float, 8-byte for bf16).
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
}

// 16-byte asynchronous global -> shared copies (cp.async): the issuing thread does not
// wait for them; cp_async_wait<n>() waits until at most n committed groups are pending.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gsrc) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// softplus(z) = log(1 + e^z), written so that neither branch overflows.
__device__ __forceinline__ float softplus_f32(float z) {
    return z > 0.f ? z + log1pf(expf(-z)) : log1pf(expf(z));
}

// ---------------------------------------------------------------------------------
// Chunk table: one entry per chunk of the call, anchored at sequence starts.
struct ChunkEntry {
    int32_t seq;     // sequence index
    int32_t start;   // first packed token row of the chunk
    int32_t len;     // tokens in the chunk (1..Q)
    int32_t pad;
};

// Host-side plan: validated dims and the carving of the workspace.
struct Plan {
    int64_t T = 0;        // tokens in the call
    int32_t nseq = 0;
    int32_t H = 0, P = 0, G = 0, N = 0, Q = 0;
    bool varlen = false;
    bool bf16 = false;
    int64_t seqlen = 0;   // dense mode
    int64_t max_chunks = 0;
    // workspace byte offsets
    size_t off_table = 0, off_first = 0, off_count = 0, off_dt = 0, off_acum = 0, off_states = 0;
    size_t bytes = 0;
    // tensor-core pipeline (tc): segment length (tokens), segment slots, state slots
    bool tc = false;
    int Ls = 0;
    int64_t max_segs = 0;
    size_t off_seg_acum = 0;
    size_t off_order = 0;     // packed varlen: CTA order over the segments, longest first
    // state snapshots every `snap` tokens of each sequence (0: none), written to
    // snap_out; per-sequence index of the first snapshot in the workspace
    int64_t snap = 0;
    size_t off_snap_first = 0;
    float* snap_out = nullptr;
    // tc with snapshots: segments cut at the snapshot positions into sub-segments, one
    // state slot each (at most max_segs + T / snap); per-sequence first sub-segment and
    // each sub-segment's end (tokens from its sequence's start)
    int64_t max_subs = 0;
    size_t off_sub_first = 0, off_sub_end = 0;
};

}  // namespace ssd
