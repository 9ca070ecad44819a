// Chunked SSD prefill on the sm_100a tensor cores (bf16 x/B/C, headdim 64, dstate 128,
// heads per B/C group a multiple of 4).
//
// The chunked SSD algorithm (JAX Nemotron 3 Nano page, "Key Components" 1; RL-Kernel
// issue page, Figure 2) runs here as a two-level scan. Every sequence is cut into
// segments of Ls tokens (a multiple of the 128-token MMA tile), anchored at the
// sequence start, and every segment into 128-token chunks:
//
//   ssd_chunk_state (pass A): per (segment, 4 heads) the segment's zero-start state
//       S_seg = sum_{s in seg} exp(Acum_end - Acum_s) dt_s x_s B_s^T,
//       accumulated over the segment's chunks in TMEM by UMMA (A = B^T from the TMA
//       tile, B = w*X written by the threads as a bf16 hi/lo pair, so the product
//       keeps ~16 mantissa bits: the FP32 final state is held to 1e-3). dt =
//       softplus(dt_raw + dt_bias) and the in-chunk cumulative sums of dt*A
//       (ssd_chunk_cumsum) are computed in the same kernel.
//   ssd_state_passing (chain): per (sequence, head, state element), sequentially over
//       the sequence's segments, h_in(seg+1) = exp(sum_seg dt*A) h_in(seg) + S_seg,
//       starting from the initial state; the last value is the final state.
//   ssd_chunk_scan (pass B): per (segment, 4 heads), chunk by chunk, starting from
//       h_in(seg) held in TMEM (FP32):
//         CB   = C B^T                                  (UMMA, once per chunk)
//         M    = CB o exp(Acum_t - Acum_s) dt_s, s <= t (threads, bf16 to smem)
//         Y    = M X,  Z = C h^T                        (UMMA)
//         y_t  = Y_t + exp(Acum_t) Z_t + D x_t          (threads, bf16 to HBM)
//         h   <- exp(Acum_end) h + B^T (w X)            (TMEM rescale + UMMA accumulate)
//
// All exponents are <= 0 since A <= 0. TMA boxes that run past a sequence's end read
// the next sequence's rows: their dt is forced to 0 and their y rows are not stored.
#pragma once

#include "ssd_tc_ptx.cuh"

namespace ssd {
namespace tc {

constexpr int kTile = 128;       // tokens per MMA tile (chunk)
constexpr int kP = 64;           // headdim
constexpr int kN = 128;          // dstate
constexpr int kHeads = 4;        // heads per CTA
constexpr float kLog2e = 1.4426950408889634f;

// Per-tile dt / cumulative decay for this CTA's 4 heads, computed by 128 threads
// (thread s = token s of the tile). acs2[h][s] = log2(e) * sum_{r<=s} dt_r A[h];
// dts[h][s] = dt_s (0 past the tile's valid length).
__device__ __forceinline__ void tile_cumsum(const float* __restrict__ dt_raw, const float* __restrict__ dt_bias,
                                            const float* __restrict__ A, int H, int h0, int64_t t0, int tl,
                                            float (*acs2)[kTile], float (*dts)[kTile], float (*wsum)[kHeads]) {
    const int s = threadIdx.x, lane = s & 31, warp = s >> 5;
    float a[kHeads], dtv[kHeads];
#pragma unroll
    for (int hh = 0; hh < kHeads; ++hh) {
        const float Ah = A[h0 + hh];
        if (s == 0 && (!(Ah <= 0.f) || isinf(Ah))) latch_error(SSD_ERR_INVALID_ARG);
        dtv[hh] = s < tl ? softplus_f32(dt_raw[(t0 + s) * H + h0 + hh] + dt_bias[h0 + hh]) : 0.f;
        a[hh] = dtv[hh] * Ah;
    }
#pragma unroll
    for (int hh = 0; hh < kHeads; ++hh) {
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float v = __shfl_up_sync(0xffffffffu, a[hh], off);
            if (lane >= off) a[hh] += v;
        }
    }
    if (lane == 31) {
#pragma unroll
        for (int hh = 0; hh < kHeads; ++hh) wsum[warp][hh] = a[hh];
    }
    __syncthreads();
#pragma unroll
    for (int hh = 0; hh < kHeads; ++hh) {
        float pre = 0.f;
        for (int w = 0; w < warp; ++w) pre += wsum[w][hh];
        acs2[hh][s] = (a[hh] + pre) * kLog2e;
        dts[hh][s] = dtv[hh];
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------------
// Pass A: zero-start segment states S_seg (fp32, layout [seg][H][N][P]) and the
// segment's total sum of dt*A (seg_acum[seg][H]).
constexpr int kSmemA = 128 * 1024 + 1024;

__global__ void __launch_bounds__(128, 1)
k_tc_segment_state(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_b,
                   const float* __restrict__ dt_raw, const float* __restrict__ dt_bias,
                   const float* __restrict__ A, const ChunkEntry* __restrict__ segs,
                   const int32_t* __restrict__ nsegs, int H, int G, float* __restrict__ seg_state,
                   float* __restrict__ seg_acum) {
    const int sg = blockIdx.x;
    if (sg >= *nsegs) return;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sB = sm;                       // [2][128 s][64 n]
    uint8_t* sX = sm + 32768;               // [4][128 s][64 p]
    uint8_t* sHi = sm + 98304;              // [128 s][64 p]
    uint8_t* sLo = sm + 114688;             // [128 s][64 p]
    __shared__ float acs2[kHeads][kTile], dts[kHeads][kTile], wsum[4][kHeads];
    __shared__ uint64_t bar_load, bar_mma;
    __shared__ uint32_t tmem_slot;

    const int tid = threadIdx.x, warp = tid >> 5;
    const int h0 = blockIdx.y * kHeads, g = h0 / (H / G);
    const ChunkEntry seg = segs[sg];
    const int ntiles = (seg.len + kTile - 1) / kTile;

    if (tid == 0) {
        mbar_init(&bar_load, 1);
        mbar_init(&bar_mma, 1);
        fence_barrier_init();
        prefetch_tmap(&map_x);
        prefetch_tmap(&map_b);
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tS = tmem_slot;            // S_seg for head hh at columns [64*hh, 64*hh + 64)

    float suffix[kHeads] = {0.f, 0.f, 0.f, 0.f};   // log2-scaled sum of dt*A over later tiles
    uint32_t ph_load = 0, ph_mma = 0;
    bool ok = true, first_mma = true;
    for (int it = ntiles - 1; it >= 0 && ok; --it) {
        const int64_t t0 = seg.start + (int64_t)it * kTile;
        const int tl = min(kTile, seg.len - it * kTile);
        if (tid == 0) {
            mbar_arrive_expect_tx(&bar_load, 32768 + kHeads * 16384);
            tma_load_3d(sB, &map_b, &bar_load, 0, g, (int)t0);
            tma_load_3d(sB + 16384, &map_b, &bar_load, 64, g, (int)t0);
            for (int hh = 0; hh < kHeads; ++hh) tma_load_3d(sX + hh * 16384, &map_x, &bar_load, 0, h0 + hh, (int)t0);
        }
        tile_cumsum(dt_raw, dt_bias, A, H, h0, t0, tl, acs2, dts, wsum);
        ok = __syncthreads_and(mbar_wait(&bar_load, ph_load));
        ph_load ^= 1;
        const int s = tid;
        for (int hh = 0; hh < kHeads && ok; ++hh) {
            // w_s = exp(sum of dt*A after s up to the segment end) * dt_s
            const float w = exp2f(suffix[hh] + acs2[hh][kTile - 1] - acs2[hh][s]) * dts[hh][s];
            const uint32_t xrow = smem_u32(sX + hh * 16384);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 v = ld_shared_v4(xrow + swz(s, c));
                const uint32_t in[4] = {v.x, v.y, v.z, v.w};
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 f = bf16x2_to_f2(in[q]);
                    const float p0 = f.x * w, p1 = f.y * w;
                    const __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
                    const float2 hf = __bfloat1622float2(hb);
                    hi[q] = *reinterpret_cast<const uint32_t*>(&hb);
                    lo[q] = pack_bf16(p0 - hf.x, p1 - hf.y);
                }
                st_shared_v4(smem_u32(sHi) + swz(s, c), hi[0], hi[1], hi[2], hi[3]);
                st_shared_v4(smem_u32(sLo) + swz(s, c), lo[0], lo[1], lo[2], lo[3]);
            }
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                const uint32_t idesc = idesc_bf16(128, 64, 1, 1);
                const uint32_t aB = smem_u32(sB), aHi = smem_u32(sHi), aLo = smem_u32(sLo);
                const uint32_t d = tS + hh * 64;
                for (int k = 0; k < 8; ++k)
                    umma_bf16(d, desc_mnmajor(aB, k, 16384), desc_mnmajor(aHi, k, 16384), idesc,
                              !(first_mma && k == 0));
                for (int k = 0; k < 8; ++k)
                    umma_bf16(d, desc_mnmajor(aB, k, 16384), desc_mnmajor(aLo, k, 16384), idesc, true);
                umma_commit(&bar_mma);
            }
            __syncwarp();
            ok = __syncthreads_and(mbar_wait(&bar_mma, ph_mma));
            ph_mma ^= 1;
        }
        first_mma = false;
#pragma unroll
        for (int hh = 0; hh < kHeads; ++hh) suffix[hh] += acs2[hh][kTile - 1];
        __syncthreads();
    }

    // Write S_seg: thread = TMEM lane = state row n; 64 fp32 columns p per head.
    tc_fence_after();
    const int n = tid;
    for (int hh = 0; hh < kHeads; ++hh) {
        float* dst = seg_state + (((int64_t)sg * H + h0 + hh) * kN + n) * kP;
        for (int q = 0; q < 2; ++q) {
            uint32_t r[32];
            tmem_ld32(tmem_addr(tS, warp * 32, hh * 64 + q * 32), r);
            tmem_wait_ld();
            float4* d4 = reinterpret_cast<float4*>(dst + q * 32);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                d4[j] = ok ? make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                         __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (tid == 0) seg_acum[(int64_t)sg * H + h0 + hh] = ntiles > 0 ? suffix[hh] / kLog2e : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tS, 256);
}

// ---------------------------------------------------------------------------------
// Chain over segments. Element e = n*P + p of head h; seg_state slots are replaced
// by the state entering each segment (h_in, layout [seg][H][N][P]); final_state and
// init use the API layout [nseq][H][P][N].
__global__ void __launch_bounds__(256)
k_tc_segment_passing(float* __restrict__ seg_state, const float* __restrict__ seg_acum,
                     const int32_t* __restrict__ first, const float* __restrict__ init,
                     float* __restrict__ final_state, int H) {
    const int s = blockIdx.x, h = blockIdx.y;
    const int e = blockIdx.z * 256 + threadIdx.x;
    if (e >= kP * kN) return;
    const int n = e / kP, p = e % kP;
    const int64_t api = (((int64_t)s * H + h) * kP + p) * kN + n;
    float hv = init ? init[api] : 0.f;
    const int c0 = first[s], c1 = first[s + 1];
    constexpr int U = 4;
    for (int c = c0; c < c1; c += U) {
        float sv[U], dec[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (c + u < c1) {
                sv[u] = seg_state[((int64_t)(c + u) * H + h) * (kP * kN) + e];
                dec[u] = expf(seg_acum[(int64_t)(c + u) * H + h]);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (c + u < c1) {
                seg_state[((int64_t)(c + u) * H + h) * (kP * kN) + e] = hv;
                hv = fmaf(dec[u], hv, sv[u]);
            }
        }
    }
    if (final_state) final_state[api] = hv;
}

// ---------------------------------------------------------------------------------
// Pass B: outputs y for one (segment, 4 heads), chunk by chunk.
constexpr int kSmemB = 192 * 1024 + 1024;

__global__ void __launch_bounds__(128, 1)
k_tc_chunk_scan(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_b,
                const __grid_constant__ CUtensorMap map_c, const float* __restrict__ dt_raw,
                const float* __restrict__ dt_bias, const float* __restrict__ A, const float* __restrict__ D,
                const ChunkEntry* __restrict__ segs, const int32_t* __restrict__ nsegs, int H, int G,
                const float* __restrict__ hin, __nv_bfloat16* __restrict__ y) {
    const int sg = blockIdx.x;
    if (sg >= *nsegs) return;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sC = sm;                       // [2][128 t][64 n]   K-major
    uint8_t* sB = sm + 32768;               // [2][128 s][64 n]   K-major for CB, MN-major for B^T
    uint8_t* sX = sm + 65536;               // [4][128 s][64 p]   MN-major
    uint8_t* sM = sm + 131072;              // [2][128 t][64 s]   K-major
    uint8_t* sW = sm + 163840;              // [128 s][64 p]      MN-major (w * X)
    uint8_t* sH = sm + 180224;              // [128 n][64 p]      MN-major (bf16 h_in)
    __shared__ float acs2[kHeads][kTile], dts[kHeads][kTile], wsum[4][kHeads];
    __shared__ uint64_t bar_load, bar_mma;
    __shared__ uint32_t tmem_slot;

    const int tid = threadIdx.x, warp = tid >> 5;
    const int h0 = blockIdx.y * kHeads, g = h0 / (H / G);
    const ChunkEntry seg = segs[sg];
    const int ntiles = (seg.len + kTile - 1) / kTile;

    if (tid == 0) {
        mbar_init(&bar_load, 1);
        mbar_init(&bar_mma, 1);
        fence_barrier_init();
        prefetch_tmap(&map_x);
        prefetch_tmap(&map_b);
        prefetch_tmap(&map_c);
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tH = tmem_slot;            // running state, head hh at columns [64*hh, +64)
    const uint32_t tCB = tmem_slot + 256;     // C B^T, 128 columns
    const uint32_t tY = tmem_slot + 384;      // M X, 64 columns
    const uint32_t tZ = tmem_slot + 448;      // C h^T, 64 columns
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    // Running state <- h_in(seg): thread = TMEM lane = state row n.
    {
        const int n = tid;
        for (int hh = 0; hh < kHeads; ++hh) {
            const float* src = hin + (((int64_t)sg * H + h0 + hh) * kN + n) * kP;
            for (int q = 0; q < 2; ++q) {
                uint32_t r[32];
                const float4* s4 = reinterpret_cast<const float4*>(src + q * 32);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 v = s4[j];
                    r[4 * j] = __float_as_uint(v.x);
                    r[4 * j + 1] = __float_as_uint(v.y);
                    r[4 * j + 2] = __float_as_uint(v.z);
                    r[4 * j + 3] = __float_as_uint(v.w);
                }
                tmem_st32(tH + lane_off + hh * 64 + q * 32, r);
            }
        }
        tmem_wait_st();
    }

    uint32_t ph_load = 0, ph_mma = 0;
    bool ok = true;
    const int me = tid;   // tile row (token t / state row n / source s, by phase)
    for (int it = 0; it < ntiles && ok; ++it) {
        const int64_t t0 = seg.start + (int64_t)it * kTile;
        const int tl = min(kTile, seg.len - it * kTile);
        if (tid == 0) {
            mbar_arrive_expect_tx(&bar_load, 2 * 32768 + kHeads * 16384);
            tma_load_3d(sC, &map_c, &bar_load, 0, g, (int)t0);
            tma_load_3d(sC + 16384, &map_c, &bar_load, 64, g, (int)t0);
            tma_load_3d(sB, &map_b, &bar_load, 0, g, (int)t0);
            tma_load_3d(sB + 16384, &map_b, &bar_load, 64, g, (int)t0);
            for (int hh = 0; hh < kHeads; ++hh) tma_load_3d(sX + hh * 16384, &map_x, &bar_load, 0, h0 + hh, (int)t0);
        }
        tile_cumsum(dt_raw, dt_bias, A, H, h0, t0, tl, acs2, dts, wsum);
        ok = __syncthreads_and(mbar_wait(&bar_load, ph_load));
        ph_load ^= 1;
        if (!ok) break;
        // CB = C B^T
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t aC = smem_u32(sC), aB = smem_u32(sB);
            for (int k = 0; k < 8; ++k)
                umma_bf16(tCB, desc_kmajor(aC, 128, k), desc_kmajor(aB, 128, k), idesc_bf16(128, 128, 0, 0), k > 0);
            umma_commit(&bar_mma);
        }
        __syncwarp();
        ok = __syncthreads_and(mbar_wait(&bar_mma, ph_mma));
        ph_mma ^= 1;
        tc_fence_after();

        for (int hh = 0; hh < kHeads && ok; ++hh) {
            const float* ac = acs2[hh];
            const float* dv = dts[hh];
            const float a_end = ac[kTile - 1];
            // (a) h_in of this chunk -> bf16 operand; state <- exp(Acum_end) * state.
            {
                const float decay = exp2f(a_end);
                for (int q = 0; q < 2; ++q) {
                    uint32_t r[32];
                    tmem_ld32(tH + lane_off + hh * 64 + q * 32, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t pk[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            pk[j] = pack_bf16(__uint_as_float(r[8 * c + 2 * j]), __uint_as_float(r[8 * c + 2 * j + 1]));
                        st_shared_v4(smem_u32(sH) + swz(me, q * 4 + c), pk[0], pk[1], pk[2], pk[3]);
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * decay);
                    tmem_st32(tH + lane_off + hh * 64 + q * 32, r);
                }
                tmem_wait_st();
            }
            // (b) w X (w_s = exp(Acum_end - Acum_s) dt_s) -> bf16 operand.
            {
                const float w = exp2f(a_end - ac[me]) * dv[me];
                const uint32_t xrow = smem_u32(sX + hh * 16384);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = ld_shared_v4(xrow + swz(me, c));
                    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
                    uint32_t o[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 f = bf16x2_to_f2(in[q]);
                        o[q] = pack_bf16(f.x * w, f.y * w);
                    }
                    st_shared_v4(smem_u32(sW) + swz(me, c), o[0], o[1], o[2], o[3]);
                }
            }
            // (c) M[t][s] = CB[t][s] exp(Acum_t - Acum_s) dt_s for s <= t.
            {
                const int t = me;
                const float at = ac[t];
                for (int q = 0; q < 4; ++q) {
                    uint32_t r[32];
                    tmem_ld32(tCB + lane_off + q * 32, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t pk[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int s0 = q * 32 + c * 8 + 2 * j;
                            const float m0 = s0 <= t ? __uint_as_float(r[c * 8 + 2 * j]) * exp2f(at - ac[s0]) * dv[s0] : 0.f;
                            const float m1 = s0 + 1 <= t ? __uint_as_float(r[c * 8 + 2 * j + 1]) * exp2f(at - ac[s0 + 1]) * dv[s0 + 1] : 0.f;
                            pk[j] = pack_bf16(m0, m1);
                        }
                        // column s -> sub-tile s / 64, chunk (s % 64) / 8
                        const int sc = q * 32 + c * 8;
                        st_shared_v4(smem_u32(sM) + (sc >> 6) * 16384 + swz(t, (sc & 63) >> 3), pk[0], pk[1], pk[2], pk[3]);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                const uint32_t aC = smem_u32(sC), aB = smem_u32(sB), aX = smem_u32(sX + hh * 16384);
                const uint32_t aM = smem_u32(sM), aW = smem_u32(sW), aH = smem_u32(sH);
                const uint32_t id64_km = idesc_bf16(128, 64, 0, 1), id64_mm = idesc_bf16(128, 64, 1, 1);
                for (int k = 0; k < 8; ++k)
                    umma_bf16(tY, desc_kmajor(aM, 128, k), desc_mnmajor(aX, k, 16384), id64_km, k > 0);
                for (int k = 0; k < 8; ++k)
                    umma_bf16(tZ, desc_kmajor(aC, 128, k), desc_mnmajor(aH, k, 16384), id64_km, k > 0);
                for (int k = 0; k < 8; ++k)
                    umma_bf16(tH + hh * 64, desc_mnmajor(aB, k, 16384), desc_mnmajor(aW, k, 16384), id64_mm, true);
                umma_commit(&bar_mma);
            }
            __syncwarp();
            ok = __syncthreads_and(mbar_wait(&bar_mma, ph_mma));
            ph_mma ^= 1;
            tc_fence_after();
            // (d) y_t = Y_t + exp(Acum_t) Z_t + D x_t
            if (ok) {
                const int t = me;
                const float et = exp2f(ac[t]);
                const float Dh = D[h0 + hh];
                const uint32_t xrow = smem_u32(sX + hh * 16384);
                __nv_bfloat16* yrow = y + ((t0 + t) * H + h0 + hh) * kP;
                for (int q = 0; q < 2; ++q) {
                    uint32_t ry[32], rz[32];
                    tmem_ld32(tY + lane_off + q * 32, ry);
                    tmem_ld32(tZ + lane_off + q * 32, rz);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 xv = ld_shared_v4(xrow + swz(t, q * 4 + c));
                        const uint32_t xin[4] = {xv.x, xv.y, xv.z, xv.w};
                        uint32_t o[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float2 xf = bf16x2_to_f2(xin[j]);
                            const int k0 = c * 8 + 2 * j;
                            const float v0 = __uint_as_float(ry[k0]) + et * __uint_as_float(rz[k0]) + Dh * xf.x;
                            const float v1 = __uint_as_float(ry[k0 + 1]) + et * __uint_as_float(rz[k0 + 1]) + Dh * xf.y;
                            o[j] = pack_bf16(v0, v1);
                        }
                        if (t < tl)
                            *reinterpret_cast<uint4*>(yrow + q * 32 + c * 8) = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
            }
            tc_fence_before();
            __syncthreads();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem_slot, 512);
}

}  // namespace tc
}  // namespace ssd
