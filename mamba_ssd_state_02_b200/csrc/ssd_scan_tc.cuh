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
//
// One CTA per (segment, 2 heads). Warp roles (320 threads): warp 0 issues the TMA
// loads, warp 1 issues the UMMAs, warps 2..9 form two compute warpgroups (cw = 0, 1)
// that split every row's columns in halves. Compute thread (cw, r) owns TMEM lane r = 32*(warp%4) + lane and holds
// the FP32 running state h[head][n = r][p in its half] in registers.
// Shared memory: two C/B stages (tile i+1 loads while tile i computes), a two-slot
// ring of X tiles (one per head), and one w*X and one bf16 h operand tile.
// TMEM: C B^T (128 cols), two M buffers (A operands, bf16 pairs, 64 cols each), and
// the Y, Z, S accumulators (64 cols each). Per head the compute warps build M for
// head hh while the UMMAs of head hh-1 run, then drain head hh-1 (y rows, state
// update) and write the h / w*X operands of head hh.
constexpr int kThreadsB = 320;
constexpr int kHeadsB = 2;          // heads per pass-B CTA
constexpr int kSmemB = 192 * 1024 + 1024;

__device__ __forceinline__ void compute_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Wait with a shared abort flag: once any wait has timed out, every later wait
// returns at once, so all roles run to the end without blocking each other.
__device__ __forceinline__ void wait_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return;
        if (clock64() - t0 > kWaitBudgetCycles) {
            latch_error(SSD_ERR_TIMEOUT);
            *abort_flag = 1;
            return;
        }
    }
}

__global__ void __launch_bounds__(kThreadsB, 1)
k_tc_chunk_scan(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_b,
                const __grid_constant__ CUtensorMap map_c, const float* __restrict__ dt_raw,
                const float* __restrict__ dt_bias, const float* __restrict__ A, const float* __restrict__ D,
                const ChunkEntry* __restrict__ segs, const int32_t* __restrict__ nsegs, int H, int G,
                const float* __restrict__ hin, __nv_bfloat16* __restrict__ y) {
    const int sg = blockIdx.x;
    if (sg >= *nsegs) return;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sCB = sm;                      // stage st: C at st*65536 ([2][128 t][64 n]), B at +32768
    uint8_t* sX = sm + 131072;              // slot j: [128 s][64 p] at j*16384
    uint8_t* sW = sm + 163840;              // [128 s][64 p]  w * X
    uint8_t* sH = sm + 180224;              // [128 n][64 p]  bf16 h_in
    __shared__ float ac2[kHeadsB][kTile], dts[kHeadsB][kTile], uw[kHeadsB][kTile], ww[kHeadsB][kTile];
    __shared__ float wpart[2][4];
    __shared__ uint64_t full_cb[2], empty_cb[2], full_x[2], empty_x[2], cb_done, ops_ready, mma_done;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h0 = blockIdx.y * kHeadsB, g = h0 / (H / G);
    const ChunkEntry seg = segs[sg];
    const int ntiles = (seg.len + kTile - 1) / kTile;

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&full_cb[i], 1);
            mbar_init(&empty_cb[i], 1);
            mbar_init(&full_x[i], 1);
            mbar_init(&empty_x[i], 8);
        }
        mbar_init(&cb_done, 1);
        mbar_init(&ops_ready, 8);
        mbar_init(&mma_done, 1);
        abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&map_x);
        prefetch_tmap(&map_b);
        prefetch_tmap(&map_c);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_slot;
    const uint32_t tCB = tbase, tM = tbase + 128, tY = tbase + 256, tZ = tbase + 320, tS = tbase + 384;
    volatile int* abort_p = &abort_flag;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            for (int it = 0; it < ntiles; ++it) {
                const int t0 = seg.start + it * kTile, st = it & 1;
                if (it >= 2) wait_abort(&empty_cb[st], ((it - 2) >> 1) & 1, abort_p);
                mbar_arrive_expect_tx(&full_cb[st], 65536);
                uint8_t* cbuf = sCB + st * 65536;
                tma_load_3d(cbuf, &map_c, &full_cb[st], 0, g, t0);
                tma_load_3d(cbuf + 16384, &map_c, &full_cb[st], 64, g, t0);
                tma_load_3d(cbuf + 32768, &map_b, &full_cb[st], 0, g, t0);
                tma_load_3d(cbuf + 49152, &map_b, &full_cb[st], 64, g, t0);
                for (int hh = 0; hh < kHeadsB; ++hh) {
                    const int j = it * kHeadsB + hh, slot = j & 1;
                    if (j >= 2) wait_abort(&empty_x[slot], ((j - 2) >> 1) & 1, abort_p);
                    mbar_arrive_expect_tx(&full_x[slot], 16384);
                    tma_load_3d(sX + slot * 16384, &map_x, &full_x[slot], 0, h0 + hh, t0);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ UMMA issuer
        if (lane == 0) {
            const uint32_t id_cb = idesc_bf16(128, 128, 0, 0);
            const uint32_t id_km = idesc_bf16(128, 64, 0, 1), id_mm = idesc_bf16(128, 64, 1, 1);
            const uint32_t aW = smem_u32(sW), aH = smem_u32(sH);
            for (int it = 0; it < ntiles; ++it) {
                const int st = it & 1;
                wait_abort(&full_cb[st], (it >> 1) & 1, abort_p);
                tc_fence_after();
                const uint32_t aC = smem_u32(sCB + st * 65536), aB = aC + 32768;
                for (int k = 0; k < 8; ++k)
                    umma_bf16(tCB, desc_kmajor(aC, 128, k), desc_kmajor(aB, 128, k), id_cb, k > 0);
                umma_commit(&cb_done);
                for (int hh = 0; hh < kHeadsB; ++hh) {
                    const int j = it * kHeadsB + hh;
                    wait_abort(&ops_ready, j & 1, abort_p);
                    tc_fence_after();
                    const uint32_t aX = smem_u32(sX + (hh & 1) * 16384), tMh = tM + (hh & 1) * 64;
                    for (int k = 0; k < 8; ++k) umma_bf16_ts(tY, tMh + 8 * k, desc_mnmajor(aX, k, 16384), id_km, k > 0);
                    for (int k = 0; k < 8; ++k)
                        umma_bf16(tZ, desc_kmajor(aC, 128, k), desc_mnmajor(aH, k, 16384), id_km, k > 0);
                    for (int k = 0; k < 8; ++k)
                        umma_bf16(tS, desc_mnmajor(aB, k, 16384), desc_mnmajor(aW, k, 16384), id_mm, k > 0);
                    umma_commit(&mma_done);
                    if (hh == kHeadsB - 1) umma_commit(&empty_cb[st]);
                }
            }
        }
    } else {
        // ------------------------------------------------------------ compute warpgroups
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int r = q * 32 + lane;            // row: token t, source s or state row n
        const int cw = (warp - 2) >> 2;         // column half
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        float h[kHeadsB][32];                    // h[head][n = r][p = 32*cw + j]
#pragma unroll
        for (int hh = 0; hh < kHeadsB; ++hh) {
            const float4* src =
                reinterpret_cast<const float4*>(hin + (((int64_t)sg * H + h0 + hh) * kN + r) * kP + 32 * cw);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 v = src[j];
                h[hh][4 * j] = v.x;
                h[hh][4 * j + 1] = v.y;
                h[hh][4 * j + 2] = v.z;
                h[hh][4 * j + 3] = v.w;
            }
        }

        // Epilogue of head e: y rows (this thread's token r, its 32 columns) and the
        // state update h <- exp(Acum_end) h + S (this thread's state row r).
        auto drain = [&](int e, int64_t t0, int tl) {
            const float et = exp2f(ac2[e][r]);
            const float Dh = D[h0 + e];
            const uint32_t xrow = smem_u32(sX + (e & 1) * 16384);
            uint32_t ry[32], rz[32];
            tmem_ld32(tY + lane_off + 32 * cw, ry);
            tmem_ld32(tZ + lane_off + 32 * cw, rz);
            tmem_wait_ld();
            uint32_t o[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 xv = ld_shared_v4(xrow + swz(r, 4 * cw + c));
                const uint32_t xin[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const float2 xf = bf16x2_to_f2(xin[jj]);
                    const int k0 = c * 8 + 2 * jj;
                    const float v0 = fmaf(et, __uint_as_float(rz[k0]), __uint_as_float(ry[k0])) + Dh * xf.x;
                    const float v1 = fmaf(et, __uint_as_float(rz[k0 + 1]), __uint_as_float(ry[k0 + 1])) + Dh * xf.y;
                    o[c * 4 + jj] = pack_bf16(v0, v1);
                }
            }
            if (r < tl) {
                uint4* dst = reinterpret_cast<uint4*>(y + ((t0 + r) * H + h0 + e) * kP + 32 * cw);
#pragma unroll
                for (int c = 0; c < 4; ++c) dst[c] = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
            }
            uint32_t rs[32];
            tmem_ld32(tS + lane_off + 32 * cw, rs);
            tmem_wait_ld();
            const float decay = exp2f(ac2[e][kTile - 1]);
#pragma unroll
            for (int j = 0; j < 32; ++j) h[e][j] = fmaf(decay, h[e][j], __uint_as_float(rs[j]));
        };

        for (int it = 0; it < ntiles; ++it) {
            const int64_t t0 = seg.start + (int64_t)it * kTile;
            const int tl = min(kTile, seg.len - it * kTile);
            // -------- dt, log2-scaled cumulative dt*A, and the decay weights of this tile
            compute_bar();
            {
                const int hh = cw;
                const float Ah = A[h0 + hh];
                if (r == 0 && it == 0 && (!(Ah <= 0.f) || isinf(Ah))) latch_error(SSD_ERR_INVALID_ARG);
                const float dtv = r < tl ? softplus_f32(dt_raw[(t0 + r) * H + h0 + hh] + dt_bias[h0 + hh]) : 0.f;
                float a = dtv * Ah;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float v = __shfl_up_sync(0xffffffffu, a, off);
                    if (lane >= off) a += v;
                }
                if (lane == 31) wpart[cw][q] = a;
                compute_bar();
                float pre = 0.f;
                for (int w = 0; w < q; ++w) pre += wpart[cw][w];
                const float av = (a + pre) * kLog2e;
                ac2[hh][r] = av;
                dts[hh][r] = dtv;
                compute_bar();
                uw[hh][r] = exp2f(ac2[hh][(r | 31)] - av) * dtv;
                ww[hh][r] = exp2f(ac2[hh][kTile - 1] - av) * dtv;
                compute_bar();
            }
            wait_abort(&cb_done, it & 1, abort_p);
            tc_fence_after();

#pragma unroll
            for (int hh = 0; hh < kHeadsB; ++hh) {
                const int j = it * kHeadsB + hh;
                // -------- (c) M[t][s] for head hh, t = r, s in [64 cw, 64 cw + 64) -> TMEM
                {
                    const float* ac = ac2[hh];
                    const float at = ac[r];
                    const int bt = r >> 5;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int sb = 2 * cw + half;              // 32-wide source block
                        uint32_t pk[16];
                        if (sb > bt) {
#pragma unroll
                            for (int k = 0; k < 16; ++k) pk[k] = 0u;
                        } else {
                            uint32_t rc[32];
                            tmem_ld32(tCB + lane_off + 32 * sb, rc);
                            tmem_wait_ld();
                            if (sb < bt) {
                                const float v = exp2f(at - ac[32 * sb + 31]);
#pragma unroll
                                for (int k = 0; k < 16; ++k) {
                                    const int s0 = 32 * sb + 2 * k;
                                    pk[k] = pack_bf16(__uint_as_float(rc[2 * k]) * v * uw[hh][s0],
                                                      __uint_as_float(rc[2 * k + 1]) * v * uw[hh][s0 + 1]);
                                }
                            } else {
#pragma unroll
                                for (int k = 0; k < 16; ++k) {
                                    const int s0 = 32 * sb + 2 * k;
                                    const float m0 = s0 <= r ? __uint_as_float(rc[2 * k]) * exp2f(at - ac[s0]) * dts[hh][s0] : 0.f;
                                    const float m1 = s0 + 1 <= r ? __uint_as_float(rc[2 * k + 1]) * exp2f(at - ac[s0 + 1]) * dts[hh][s0 + 1] : 0.f;
                                    pk[k] = pack_bf16(m0, m1);
                                }
                            }
                        }
                        // 16 packed columns at tM[hh&1] + 16*sb
                        tmem_st16(tM + (hh & 1) * 64 + lane_off + 16 * sb, pk);
                    }
                    tmem_wait_st();
                }
                // -------- drain head hh-1 (its UMMAs overlapped the M build above)
                if (hh > 0) {
                    wait_abort(&mma_done, (j - 1) & 1, abort_p);
                    tc_fence_after();
                    drain(hh - 1, t0, tl);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty_x[(hh - 1) & 1]);
                }
                // -------- (a) bf16 h_in of head hh, (b) w * X of head hh
                {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t pk[4];
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) pk[jj] = pack_bf16(h[hh][8 * c + 2 * jj], h[hh][8 * c + 2 * jj + 1]);
                        st_shared_v4(smem_u32(sH) + swz(r, 4 * cw + c), pk[0], pk[1], pk[2], pk[3]);
                    }
                    wait_abort(&full_x[hh & 1], (j >> 1) & 1, abort_p);
                    const float w = ww[hh][r];
                    const uint32_t xrow = smem_u32(sX + (hh & 1) * 16384);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 v = ld_shared_v4(xrow + swz(r, 4 * cw + c));
                        const uint32_t in[4] = {v.x, v.y, v.z, v.w};
                        uint32_t o[4];
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
                            const float2 f = bf16x2_to_f2(in[jj]);
                            o[jj] = pack_bf16(f.x * w, f.y * w);
                        }
                        st_shared_v4(smem_u32(sW) + swz(r, 4 * cw + c), o[0], o[1], o[2], o[3]);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ops_ready);
            }
            wait_abort(&mma_done, (it * kHeadsB + kHeadsB - 1) & 1, abort_p);
            tc_fence_after();
            drain(kHeadsB - 1, t0, tl);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_x[(kHeadsB - 1) & 1]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tbase, 512);
}

}  // namespace tc
}  // namespace ssd
