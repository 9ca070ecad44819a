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
//       softplus(dt_raw + dt_bias) and the cumulative sums of dt*A (ssd_chunk_cumsum)
//       are computed in the same kernel.
//   ssd_state_passing (chain): per (sequence, head, state element), sequentially over
//       the sequence's segments, h_in(seg+1) = exp(sum_seg dt*A) h_in(seg) + S_seg,
//       starting from the initial state; the last value is the final state.
//   ssd_chunk_scan (pass B): per (segment, 2 heads), chunk by chunk, starting from
//       h_in(seg) held in the compute threads' registers (FP32):
//         CB   = C B^T                                      (UMMA, once per chunk)
//         M    = CB o exp(Acum_t - Acum_s) dt_s, s <= t, + D on the diagonal
//                                                           (threads, bf16 in TMEM)
//         Y    = M X + exp(Acum_t) C h^T                    (UMMA; scaled sum by threads)
//         h   <- exp(Acum_end) h + B^T (w X)                (UMMA + threads)
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

// ---------------------------------------------------------------------------------
// Shared by both passes.
constexpr int kRoleWarps = 2;                    // warp 0: TMA producer, warp 1: UMMA issuer
constexpr int kComputeWarps = 16;                // four compute warpgroups (cw = 0..3)
constexpr int kThreadsTc = 32 * (kRoleWarps + kComputeWarps);

// Bounded waits with a CTA-wide abort flag. A wait that runs out latches SSD_ERR_TIMEOUT
// and raises the flag, after which every wait in the CTA returns at once. The compute
// and scan warps then run to the end on whatever the buffers hold: they issue no copy or
// MMA, and the barriers they arrive on carry no transaction counts. The two issuing
// roles stop at the first wait after the flag is up (wait_issue: an arrival made after
// its warp saw the flag reaches them through the barrier's release/acquire, so they
// never act on it), and at the end the TMA producer waits for the loads it has issued
// and the UMMA warp for its MMAs (both bounded), so that no copy or MMA is in flight
// when TMEM is freed and the CTA exits.
__device__ __forceinline__ bool wait_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait_sleep(bar, parity)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > kWaitBudgetCycles) {
            latch_error(SSD_ERR_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

// For an issuing role: true if the phase completed and no abort has been raised.
__device__ __forceinline__ bool wait_issue(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    return wait_abort(bar, parity, abort_flag) && !*abort_flag;
}

// The same for a whole warp (all lanes call it), warp-uniform.
__device__ __forceinline__ bool wait_issue_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    return __all_sync(0xffffffffu, wait_issue(bar, parity, abort_flag));
}

// ---------------------------------------------------------------------------------
// Pass A: zero-start segment states S_seg (fp32, layout [slot][H][P][N]) and the
// segment's total sum of dt*A (seg_acum[slot][H]). One CTA per (segment, 4 heads); the
// chunks run from the segment end backwards so the decay to the end is a running sum.
// With snapshots, one state and sum per piece of the segment between snapshot positions.
//
// Warp 0 issues the TMA loads, warp 1 the UMMAs, warps 18 and 19 scan dt of heads
// 0-1 and 2-3 (up to four chunks ahead; w_s = exp(sum_{r > s in seg} dt_r A) dt_s), and
// the 16 compute warps write w*X as a bf16 hi/lo pair (hi in place over x, lo next to
// it), so the product keeps ~16 mantissa bits: the FP32 final state is held to 1e-3.
// Heads go in pairs: per pair 8 UMMAs with N = 256 ([hi|hi|lo|lo] of the two heads side
// by side, B^T read once) accumulate S_hi and S_lo of the two heads in TMEM, issued in
// two batches of 4, one per 64-token half of the chunk; while they run the compute warps
// prepare the other half or pair. At the end S = S_hi + S_lo. Compute thread (cw, r)
// owns token row r (half r / 64) and column quarter cw of every head's w*X.
//
// Shared memory: two B stages; per head pair [x/hi h0 | x/hi h1 | lo h0 | lo h1], each
// half of a pair's rows reloaded as soon as that half's UMMAs are done. TMEM: per pair p,
// columns 256p + [S_hi h0 | S_hi h1 | S_lo h0 | S_lo h1] (64 each).
constexpr int kSmemA = 192 * 1024 + 1024;
constexpr int kXParts = 2;                    // x slot parts per chunk (2 or 4; 4 measured slower)
constexpr int kXRows = kTile / kXParts;       // token rows per part
constexpr int kScanWarpA = kRoleWarps + kComputeWarps;         // warps 18, 19: dt scan
constexpr int kThreadsA = 32 * (kScanWarpA + 2);

__global__ void __launch_bounds__(kThreadsA, 1)
k_tc_segment_state(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_b,
                   const float* __restrict__ dt_raw, const float* __restrict__ dt_bias,
                   const float* __restrict__ A, ChunkEntry* __restrict__ segs,
                   int32_t* __restrict__ nsegs, int H, int G, float* __restrict__ seg_state,
                   float* __restrict__ seg_acum, const int32_t* __restrict__ order,
                   int32_t* __restrict__ first, int64_t snap, int stall, int nseq, int64_t dense_len, int Ls) {
    const int nq = H / kHeads;
    // A dense batch without snapshots needs no table kernel: segment sg is piece sg % nps of
    // sequence sg / nps (nps = segments per sequence), computed here from the grid (one CTA
    // per (segment, 4 heads), exactly), and the first head quad's CTA writes the segment's
    // table entry, the sequence's first segment and the count for the kernels that follow.
    ChunkEntry dseg{0, 0, 0, 0};
    if (dense_len > 0) {
        const int nps = (int)((dense_len + Ls - 1) / Ls), sgd = (int)(blockIdx.x / nq);
        const int sq = sgd / nps, k = sgd % nps;
        dseg.seq = sq;
        dseg.start = (int32_t)((int64_t)sq * dense_len + (int64_t)k * Ls);
        dseg.len = (int32_t)min((int64_t)Ls, dense_len - (int64_t)k * Ls);
        dseg.pad = sgd;
        if (blockIdx.x % nq == 0 && threadIdx.x == 0) {
            segs[sgd] = dseg;
            if (k == 0) first[sq] = sgd;
            if (sgd == nseq * nps - 1) {
                first[nseq] = nseq * nps;
                *nsegs = nseq * nps;
            }
        }
    } else if ((int)(blockIdx.x / nq) >= *nsegs) {
        return;
    }
    const int sg = order ? order[blockIdx.x / nq] : (int)(blockIdx.x / nq);   // longest segments first
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sB = sm;                       // stage st at st*32768: [2][128 s][64 n]
    uint8_t* sP = sm + 65536;               // pair p at p*65536: x/hi of its heads, then lo; [128 s][64 p] each
    auto xs = [&](int hh) { return sP + (hh >> 1) * 65536 + (hh & 1) * 16384; };           // x, then hi
    auto los = [&](int hh) { return sP + (hh >> 1) * 65536 + 32768 + (hh & 1) * 16384; };  // lo
    __shared__ __align__(16) float wts[4][kHeads][kTile];
    // x slots by (head pair, part of kXParts token rows): a part's rows are loaded, formed
    // into hi/lo and read by its K-steps on barriers of their own, so a part is reloaded for
    // the next chunk while the later parts' UMMAs still run.
    __shared__ uint64_t full_b[2], empty_b[2], full_x[2][kXParts], pair_done[2][kXParts], ops_ready[2][kXParts],
        w_ready[4], w_free[4], all_done,
        drained, stall_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h0 = (blockIdx.x % nq) * kHeads, g = h0 / (H / G);
    const ChunkEntry seg = dense_len > 0 ? dseg : segs[sg];
    const int ntiles = (seg.len + kTile - 1) / kTile;
    // State slots. Without snapshots the segment has one (seg.pad). With snapshots every
    // snap tokens the segment is cut at the multiples of snap inside it (counted from the
    // sequence start) and each piece (sub-segment) gets its own zero-start state, in slots
    // seg.pad, seg.pad + 1, ... in token order. Step k of the reverse walk takes chunk
    // ntiles-1-k: it opens a piece at the piece's last chunk and closes it at its first.
    // In 128-token chunks (segments start and snapshots fall on chunk boundaries): rc0 =
    // the segment's first chunk within its sequence, sc = chunks per snapshot interval
    // (0: none; capped where no sequence reaches a second interval).
    const int sc = snap > 0 ? (int)min((int64_t)1 << 30, snap / kTile) : 0;
    const int rc0 = sc ? (seg.start - segs[first[seg.seq]].start) / kTile : 0;
    auto slot_of = [&](int it) -> int { return sc ? seg.pad + (rc0 + it) / sc - rc0 / sc : seg.pad; };
    // chunk it ends a piece / starts one
    auto opens = [&](int k) { const int it = ntiles - 1 - k; return k == 0 || (sc && (rc0 + it + 1) % sc == 0); };
    auto closes = [&](int k) { const int it = ntiles - 1 - k; return it == 0 || (sc && (rc0 + it) % sc == 0); };

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&full_b[i], 1);
            mbar_init(&empty_b[i], 1);
            for (int hf = 0; hf < kXParts; ++hf) {
                mbar_init(&full_x[i][hf], 1);
                mbar_init(&pair_done[i][hf], 1);
                mbar_init(&ops_ready[i][hf], kComputeWarps / kXParts);
            }
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(&w_ready[i], 2);
            mbar_init(&w_free[i], kComputeWarps);
        }
        mbar_init(&all_done, 1);
        mbar_init(&drained, 1);
        mbar_init(&stall_bar, 1);
        abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&map_x);
        prefetch_tmap(&map_b);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tS = tmem_slot;
    volatile int* abort_p = &abort_flag;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            auto t0_of = [&](int k) { return seg.start + (ntiles - 1 - k) * kTile; };   // k-th chunk processed
            int nb0 = 0, nb1 = 0, nx[2][kXParts] = {};      // phases issued on full_b[.], full_x[.][.]
            bool ok = true;
            for (int k = 0; k < ntiles && ok; ++k) {
                const int t0 = t0_of(k), st = k & 1;
                if (k >= 2 && !wait_issue(&empty_b[st], ((k - 2) >> 1) & 1, abort_p)) break;
                mbar_arrive_expect_tx(&full_b[st], 32768);
                tma_load_3d(sB + st * 32768, &map_b, &full_b[st], 0, g, t0);
                tma_load_3d(sB + st * 32768 + 16384, &map_b, &full_b[st], 64, g, t0);
                if (st) ++nb1; else ++nb0;
                if (k + 1 < ntiles) {               // next chunk's B and X into L2 meanwhile
                    const int tn = t0_of(k + 1);
                    tma_prefetch_3d(&map_b, 0, g, tn);
                    tma_prefetch_3d(&map_b, 64, g, tn);
                    for (int hh = 0; hh < kHeads; ++hh)
                        for (int hf = 0; hf < kXParts; ++hf) tma_prefetch_3d(&map_x, 0, h0 + hh, tn + hf * kXRows);
                }
                for (int pr = 0; pr < 2 && ok; ++pr) {
                    for (int hf = 0; hf < kXParts; ++hf) {
                        // the part's slot rows (x, then hi) and lo rows are free
                        if (k >= 1 && !wait_issue(&pair_done[pr][hf], (k - 1) & 1, abort_p)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&full_x[pr][hf], 2 * kXRows * 128);
                        for (int hh = 2 * pr; hh < 2 * pr + 2; ++hh)
                            tma_load_3d(xs(hh) + hf * kXRows * 128, &map_x, &full_x[pr][hf], 0, h0 + hh,
                                        t0 + hf * kXRows);
                        ++nx[pr][hf];
                    }
                }
            }
            // The last phase issued on each barrier completes once its bytes have landed
            // (a phase is issued only after the previous one has been consumed).
            if (nb0) mbar_wait(&full_b[0], (nb0 - 1) & 1);
            if (nb1) mbar_wait(&full_b[1], (nb1 - 1) & 1);
            for (int pr = 0; pr < 2; ++pr)
                for (int hf = 0; hf < kXParts; ++hf)
                    if (nx[pr][hf]) mbar_wait(&full_x[pr][hf], (nx[pr][hf] - 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ UMMA issuer
        // [S_hi|S_lo] of a head pair += B^T [hi h0|hi h1|lo h0|lo h1]: A = B^T (MN-major),
        // B MN-major with its four 64-column blocks 16 KB apart, N = 256.
        const uint32_t idesc = idesc_bf16(128, 256, 1, 1);
        const uint64_t dP = smem_desc(smem_u32(sP), 16384, 1024);
        bool ok = true;
        for (int k = 0; k < ntiles && ok; ++k) {
            const int st = k & 1;
            if (!wait_issue_warp(&full_b[st], (k >> 1) & 1, abort_p)) break;
            const uint64_t dB = smem_desc(smem_u32(sB + st * 32768), 16384, 1024);
            const bool fresh = opens(k);            // first chunk of a piece: overwrite the accumulator
            for (int pr = 0; pr < 2 && ok; ++pr) {
                for (int hf = 0; hf < kXParts; ++hf) {
                    // test hook (stall): before the first head pair's UMMAs, a wait that runs out
                    if ((stall && k == 0 && hf == 0 && !wait_issue_warp(&stall_bar, 0, abort_p)) ||
                        !wait_issue_warp(&ops_ready[pr][hf], k & 1, abort_p)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d = tS + pr * 256;
                    const uint64_t dp = desc_add(dP, pr * 65536);
                    if (elect_one()) {
#pragma unroll
                        for (int kk = hf * (8 / kXParts); kk < (hf + 1) * (8 / kXParts); ++kk)
                            umma_bf16(d, desc_add(dB, kk * kMnStep), desc_add(dp, kk * kMnStep), idesc,
                                      !(kk == 0 && fresh));
                        umma_commit(&pair_done[pr][hf]);
                        if (pr == 1 && hf == kXParts - 1) umma_commit(&empty_b[st]);
                        if (pr == 1 && hf == kXParts - 1 && k == ntiles - 1) umma_commit(&all_done);
                    }
                    __syncwarp();
                }
            }
        }
        // Every MMA issued above has completed once this commit arrives.
        if (elect_one()) umma_commit(&drained);
        __syncwarp();
        mbar_wait(&drained, 0);
    } else if (warp >= kScanWarpA) {
        // ------------------------------------------------------------ dt scan
        // Warp 18 + i scans heads 2i, 2i+1. Lane l holds tokens 4l..4l+3 of a chunk; the
        // dt_raw of the next chunk is loaded while this one is scanned. suf[e] = sum of
        // dt*A after the current chunk (log2 units).
        const int hb = 2 * (warp - kScanWarpA);
        float bias[2], Ah[2], suf[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            bias[e] = dt_bias[h0 + hb + e];
            Ah[e] = A[h0 + hb + e] * kLog2e;
            suf[e] = 0.f;
            if (lane == 0 && (!(A[h0 + hb + e] <= 0.f) || isinf(A[h0 + hb + e]))) latch_error(SSD_ERR_INVALID_ARG);
        }
        float z[2][4], zn[2][4];
        auto load_dt = [&](int k, float (&zz)[2][4]) {
            const int it = ntiles - 1 - k;
            const int tlk = min(kTile, seg.len - it * kTile);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int64_t row = ((int64_t)seg.start + (int64_t)it * kTile + 4 * lane + i) * H + h0 + hb;
#pragma unroll
                for (int e = 0; e < 2; ++e) zz[e][i] = 4 * lane + i < tlk ? dt_raw[row + e] : 0.f;
            }
        };
        load_dt(0, zn);
        for (int k = 0; k < ntiles; ++k) {
            const int bf = k % 4, it = ntiles - 1 - k;
            const int tlk = min(kTile, seg.len - it * kTile);
            if (opens(k)) suf[0] = suf[1] = 0.f;
#pragma unroll
            for (int e = 0; e < 2; ++e)
#pragma unroll
                for (int i = 0; i < 4; ++i) z[e][i] = zn[e][i];
            if (k + 1 < ntiles) load_dt(k + 1, zn);
            if (k >= 4) wait_abort(&w_free[bf], ((k >> 2) - 1) & 1, abort_p);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float dtv[4], p[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    dtv[i] = 4 * lane + i < tlk ? softplus_fast(z[e][i] + bias[e]) : 0.f;
                    p[i] = (i ? p[i - 1] : 0.f) + dtv[i] * Ah[e];
                }
                float incl = p[3];
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float v = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += v;
                }
                const float tot = __shfl_sync(0xffffffffu, incl, 31);
                const float base = suf[e] + tot - (incl - p[3]);    // decay exponent of token 4l, plus p[i] below
                float w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) w[i] = fast_exp2(base - p[i]) * dtv[i];
                *reinterpret_cast<float4*>(&wts[bf][hb + e][4 * lane]) = make_float4(w[0], w[1], w[2], w[3]);
                suf[e] += tot;
            }
            if (closes(k) && lane < 2)                          // total decay exponent of the piece
                seg_acum[(int64_t)slot_of(it) * H + h0 + hb + lane] = (lane ? suf[1] : suf[0]) / kLog2e;
            __syncwarp();
            if (lane == 0) mbar_arrive(&w_ready[bf]);
        }
    } else {
        // ------------------------------------------------------------ compute warps
        const int cw = (warp - kRoleWarps) >> 2, q = warp & 3, r = q * 32 + lane;
        // Warpgroup cw writes the state of head cw into a slot: thread = state row n.
        auto store_state = [&](int slot) {
            // layout [slot][H][P][N]: for each p the warp writes 32 consecutive n
            float* dst = seg_state + ((int64_t)slot * H + h0 + cw) * kP * kN + r;
            const uint32_t thi = tS + ((uint32_t)(q * 32) << 16) + (cw >> 1) * 256 + (cw & 1) * 64;
            for (int half = 0; half < 2; ++half) {
                uint32_t vh[32], vl[32];
                tmem_ld32(thi + half * 32, vh);
                tmem_ld32(thi + 128 + half * 32, vl);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    dst[(half * 32 + e) * kN] = __uint_as_float(vh[e]) + __uint_as_float(vl[e]);
            }
        };
        for (int k = 0; k < ntiles; ++k) {
            const int bf = k % 4;
            if (k > 0 && opens(k)) {
                // Step k-1 closed a piece: once its UMMAs are done, store the piece's state
                // before this step's operands are handed over (the UMMA warp waits for them
                // and then overwrites the accumulator).
                wait_abort(&pair_done[cw >> 1][kXParts - 1], (k - 1) & 1, abort_p);   // covers earlier MMAs
                tc_fence_after();
                store_state(slot_of(ntiles - k));
                tc_fence_before();
                // Every compute warp has read the accumulators before any of them hands over
                // a half's operands (that half's first UMMA overwrites the whole accumulator).
                named_barrier(1, 32 * kComputeWarps);
            }
            wait_abort(&w_ready[bf], (k >> 2) & 1, abort_p);
            for (int pr = 0; pr < 2; ++pr) {
                wait_abort(&full_x[pr][q / (4 / kXParts)], k & 1, abort_p);   // rows r = 32 q + lane
#pragma unroll
                for (int hh = 2 * pr; hh < 2 * pr + 2; ++hh) {
                    const float w = wts[bf][hh][r];
                    const float2 w2 = make_float2(w, w);
                    const uint32_t xrow = smem_u32(xs(hh)), lrow = smem_u32(los(hh));
#pragma unroll
                    for (int c = 2 * cw; c < 2 * cw + 2; ++c) {
                        const uint4 v = ld_shared_v4(xrow + swz(r, c));
                        const uint32_t in[4] = {v.x, v.y, v.z, v.w};
                        uint32_t oh[4], ol[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 pw = fmul2(bf16x2_to_f2(in[e]), w2);
                            oh[e] = pack_bf16(pw);
                            ol[e] = pack_bf16(fsub2(pw, bf16x2_to_f2(oh[e])));
                        }
                        st_shared_v4(xrow + swz(r, c), oh[0], oh[1], oh[2], oh[3]);     // hi in place of x
                        st_shared_v4(lrow + swz(r, c), ol[0], ol[1], ol[2], ol[3]);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ops_ready[pr][q / (4 / kXParts)]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&w_free[bf]);
        }
        // Wait for the last UMMAs, then write the state of the segment's first piece.
        wait_abort(&all_done, 0, abort_p);
        tc_fence_after();
        store_state(slot_of(0));
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tS, 512);
}

// ---------------------------------------------------------------------------------
// Chain over state slots: a sequence's segments, or with snapshots the pieces its
// segments are cut into (slots first[s] .. first[s+1]-1, in token order). The slot of
// each segment's first piece is replaced by the state entering the segment (h_in), which
// the chunk scan reads. Slots, init, final_state and the snapshots all use the layout
// [.][H][P][N]. A CTA owns kPassElems consecutive elements of one (sequence, head);
// thread t walks elements t + 256 i (i < 4) down the slots, up to eight slots' loads
// in flight, every access coalesced.
constexpr int kPassE = 4;                        // elements per thread
constexpr int kPassElems = 256 * kPassE;         // elements per CTA

__global__ void __launch_bounds__(256, 4)
k_tc_segment_passing(float* __restrict__ seg_state, const float* __restrict__ seg_acum,
                     const int32_t* __restrict__ first, const float* __restrict__ init,
                     float* __restrict__ final_state, int H, int Ls, int64_t snap,
                     const int32_t* __restrict__ sub_end, const int32_t* __restrict__ snap_first,
                     float* __restrict__ snap_out) {
    constexpr int E = kPassE, PN = kP * kN;
    const int s = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int64_t e0 = (int64_t)blockIdx.z * kPassElems + tid;       // element of thread's i = 0
    auto at = [&](int64_t slot) { return ((int64_t)slot * H + h) * PN + e0; };
    float hv[E];
#pragma unroll
    for (int i = 0; i < E; ++i) hv[i] = init ? init[at(s) + 256 * i] : 0.f;
    const int c0 = first[s], c1 = first[s + 1];
    // Snapshot positions and segment starts, in tokens from the sequence start (int32: a
    // sequence holds fewer than 2^31 tokens, so an interval beyond that never comes up).
    const int sn = snap > 0 && snap <= INT32_MAX ? (int)snap : 0;
    int prev_end = 0;                                       // where the current slot starts
    // Groups of U slots, double-buffered: the next group's loads are in flight while
    // this one is applied.
    constexpr int U = 4;
    struct Group {
        float sv[U][E], ac[U];
        int end[U];
    };
    auto load = [&](int c, Group& g) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (c + u < c1) {
#pragma unroll
                for (int i = 0; i < E; ++i) g.sv[u][i] = seg_state[at(c + u) + 256 * i];
                g.ac[u] = seg_acum[(int64_t)(c + u) * H + h];
                g.end[u] = sub_end ? sub_end[c + u] : 0;
            }
        }
    };
    auto apply = [&](int c, const Group& g) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (c + u < c1) {
                // Only a segment's first slot is read by the chunk scan.
                if (!sub_end || prev_end % Ls == 0) {
#pragma unroll
                    for (int i = 0; i < E; ++i) seg_state[at(c + u) + 256 * i] = hv[i];
                }
                const float dec = expf(g.ac[u]);
#pragma unroll
                for (int i = 0; i < E; ++i) hv[i] = fmaf(dec, hv[i], g.sv[u][i]);
                if (sub_end) {                            // state after a multiple of snap tokens
                    prev_end = g.end[u];
                    if (sn && g.end[u] % sn == 0) {
                        float* dst = snap_out + ((int64_t)(snap_first[s] + g.end[u] / sn - 1) * H + h) * PN + e0;
#pragma unroll
                        for (int i = 0; i < E; ++i) dst[256 * i] = hv[i];
                    }
                }
            }
        }
    };
    Group ga, gb;
    if (c0 < c1) load(c0, ga);
    for (int c = c0; c < c1; c += 2 * U) {
        if (c + U < c1) load(c + U, gb);
        apply(c, ga);
        if (c + U >= c1) break;
        if (c + 2 * U < c1) load(c + 2 * U, ga);
        apply(c + U, gb);
    }
    if (final_state) {
#pragma unroll
        for (int i = 0; i < E; ++i) final_state[at(s) + 256 * i] = hv[i];
    }
}

// ---------------------------------------------------------------------------------
// Pass B: outputs y for one (segment, 2 heads), chunk by chunk.
//
// Warp 0 issues the TMA loads and the y stores, warp 1 the UMMAs, and four compute
// warpgroups (cw = 0..3) split every row's 64 columns in quarters. Compute thread
// (cw, r) owns TMEM lane r = 32*(warp%4) + lane and keeps the FP32 running state
// h[head][n = r][p in its quarter] in registers.
//
// Per chunk j: CB = C B^T (UMMA, into the M columns) -> the compute warps turn it into
// M for both heads in place (D_h joins M on the diagonal, so y = M X + exp(Acum_t) Z
// carries the skip term) -> UMMA batch: S = B^T [wX0|wX1] then Z = C [h0|h1]^T (N = 128
// each, so C and B are read once for both heads), then Y_hh = M_hh X_hh. When S is done
// the compute warps write w*X of chunk j+1; when Z is done they update h and write bf16
// h of chunk j+1 (while the Y UMMAs run); when Y is done they drain y into the chunk's
// X slot (full chunks) and warp 0 stores the tile with one TMA store per head, then
// loads chunk j+2's X into the slot (prefetched into L2 a chunk earlier). The UMMA warp
// issues chunk j+1's C B^T as soon as the Y UMMAs have read M, so it overlaps the
// drain. Warp 18 scans dt*A up to four chunks ahead; while S and Z run, the compute
// warps tabulate chunk j+1's diagonal-block decays.
//
// M of row block q (TMEM lane quarter q) has source blocks 0..q-1 below the diagonal,
// written as CB * exp2(Acum_t - Acum_e) * exp2(Acum_e - Acum_s) dt_s with e the last
// row of the source block (both exponents <= 0), the diagonal block as CB times the
// tabulated exp2(Acum_t - Acum_s) dt_s (fp16, shared memory), and zeros above. Warp
// (cw, q) takes block cw when cw != q; the warps with cw >= q share the diagonal block
// by 16-source halves.
//
// TMEM: Z (cols 0..127), S (128..255), Y0, Y1 (256..383), C B^T then M (384..511; M of
// head hh for sources 16k..16k+15 in columns 384 + 16k + 8hh). Shared memory: one C/B
// stage (reloaded as soon as the Z/S UMMAs are done), two X slots (chunk j uses slot
// j & 1; its y tile replaces x there), bf16 h and w*X for both heads, the diagonal-block
// decay table (16 KB).
constexpr int kHeadsB = 2;
constexpr int kSmemB = 208 * 1024 + 1024;
constexpr int kScanWarp = kRoleWarps + kComputeWarps;          // warp 18: dt scan
constexpr int kThreadsB = 32 * (kScanWarp + 1);

__global__ void __launch_bounds__(kThreadsB, 1)
k_tc_chunk_scan(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_b,
                const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_y,
                const float* __restrict__ dt_raw, const float* __restrict__ dt_bias, const float* __restrict__ A,
                const float* __restrict__ D, const ChunkEntry* __restrict__ segs, const int32_t* __restrict__ nsegs,
                int H, int G, const float* __restrict__ hin, __nv_bfloat16* __restrict__ y,
                const int32_t* __restrict__ order, int stall) {
    const int nhp = H / kHeadsB;
    if ((int)(blockIdx.x / nhp) >= *nsegs) return;
    const int sg = order ? order[blockIdx.x / nhp] : (int)(blockIdx.x / nhp);   // longest segments first
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sC = sm;                       // [2][128 t][64 n]   K-major
    uint8_t* sB = sm + 32768;               // [2][128 s][64 n]   K-major for C B^T, MN-major for B^T
    uint8_t* sX = sm + 65536;               // slot sl, head hh at sl*32768 + hh*16384: [128 s][64 p]
    uint8_t* sH = sm + 131072;              // head hh block at hh*16384: [128 n][64 p]  bf16 h_in
    uint8_t* sW = sm + 163840;              // head hh block at hh*16384: [128 s][64 p]  w * X
    uint8_t* sL = sm + 196608;              // head hh at hh*8192: [128 t][32] fp16 diagonal-block decays
    __shared__ __align__(16) float ac2[4][kHeadsB][kTile];
    __shared__ __align__(16) float dts[4][kHeadsB][kTile];
    __shared__ __align__(16) float uw[4][kHeadsB][kTile];
    __shared__ __align__(16) float ww[4][kHeadsB][kTile];
    __shared__ uint64_t full_b, full_c[2], s_done, zs_done, full_x[2], cb_done, ops_ready, y0_done, mma_done, l_ready,
        dt_ready[4], dt_free[4], y_staged, drained, stall_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h0 = (blockIdx.x % nhp) * kHeadsB, g = h0 / (H / G);
    const ChunkEntry seg = segs[sg];
    const int ntiles = (seg.len + kTile - 1) / kTile;

    if (tid == 0) {
        mbar_init(&full_b, 1);
        mbar_init(&full_c[0], 1);
        mbar_init(&full_c[1], 1);
        mbar_init(&y0_done, 1);
        mbar_init(&s_done, 1);
        mbar_init(&zs_done, 1);
        for (int sl = 0; sl < 2; ++sl) mbar_init(&full_x[sl], 1);
        mbar_init(&y_staged, kComputeWarps);
        mbar_init(&cb_done, 1);
        mbar_init(&ops_ready, kComputeWarps);
        mbar_init(&mma_done, 1);
        for (int i = 0; i < 4; ++i) {
            mbar_init(&dt_ready[i], 1);
            mbar_init(&dt_free[i], kComputeWarps);
        }
        mbar_init(&l_ready, kComputeWarps);
        mbar_init(&drained, 1);
        mbar_init(&stall_bar, 1);
        abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&map_x);
        prefetch_tmap(&map_b);
        prefetch_tmap(&map_c);
        prefetch_tmap(&map_y);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_slot;
    const uint32_t tZ = tbase, tS = tbase + 128, tY = tbase + 256, tM = tbase + 384;
    volatile int* abort_p = &abort_flag;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int nx0 = 0, nx1 = 0, nb = 0, nc = 0;  // phases issued on full_x[0/1], full_b, full_c[.]
            auto load_x = [&](int j) {              // X of chunk j (both heads) into slot j & 1
                const int sl = j & 1;
                if (sl) ++nx1; else ++nx0;
                mbar_arrive_expect_tx(&full_x[sl], 32768);
                for (int hh = 0; hh < kHeadsB; ++hh)
                    tma_load_3d(sX + sl * 32768 + hh * 16384, &map_x, &full_x[sl], 0, h0 + hh, seg.start + j * kTile);
            };
            // B of chunk j (once the S UMMAs of chunk j-1 are done) and the two halves of
            // C (once Z is done), on separate barriers, so C B^T can start on the first
            // half. B, C and X of chunk j+1 are prefetched into L2 meanwhile.
            auto load_b = [&](int j) {
                const int t0 = seg.start + j * kTile;
                ++nb;
                mbar_arrive_expect_tx(&full_b, 32768);
                tma_load_3d(sB, &map_b, &full_b, 0, g, t0);
                tma_load_3d(sB + 16384, &map_b, &full_b, 64, g, t0);
            };
            auto load_c = [&](int j) {
                const int t0 = seg.start + j * kTile;
                ++nc;
                for (int hf = 0; hf < 2; ++hf) {
                    mbar_arrive_expect_tx(&full_c[hf], 16384);
                    tma_load_3d(sC + hf * 16384, &map_c, &full_c[hf], 64 * hf, g, t0);
                }
                if (j + 1 < ntiles) {
                    tma_prefetch_3d(&map_c, 0, g, t0 + kTile);
                    tma_prefetch_3d(&map_c, 64, g, t0 + kTile);
                    tma_prefetch_3d(&map_b, 0, g, t0 + kTile);
                    tma_prefetch_3d(&map_b, 64, g, t0 + kTile);
                    for (int hh = 0; hh < kHeadsB; ++hh) tma_prefetch_3d(&map_x, 0, h0 + hh, t0 + kTile);
                }
            };
            // y tile of chunk j, staged by the compute warps in the chunk's X slot (full
            // chunks only; a partial last chunk is written by the threads).
            auto store_y = [&](int j) -> bool {
                if (!wait_issue(&y_staged, j & 1, abort_p)) return false;
                if (seg.len - j * kTile >= kTile) {
                    for (int hh = 0; hh < kHeadsB; ++hh)
                        tma_store_3d(&map_y, sX + (j & 1) * 32768 + hh * 16384, 0, h0 + hh, seg.start + j * kTile);
                    bulk_commit_group();
                }
                return true;
            };
            if (ntiles > 0) {
                load_x(0);
                if (ntiles > 1) load_x(1);
                load_b(0);
                load_c(0);
            }
            bool ok = true;
            for (int j = 1; j < ntiles && ok; ++j) {
                ok = wait_issue(&s_done, (j - 1) & 1, abort_p);     // B of chunk j-1 read
                if (!ok) break;
                load_b(j);
                ok = wait_issue(&zs_done, (j - 1) & 1, abort_p);    // C of chunk j-1 read
                if (!ok) break;
                load_c(j);
                ok = store_y(j - 1);
                if (ok && j + 1 < ntiles) {
                    bulk_wait_read_all();                           // slot (j+1) & 1 read by the store
                    load_x(j + 1);
                }
            }
            if (ok && ntiles > 0) store_y(ntiles - 1);
            bulk_wait_all();
            // The last phase issued on each barrier completes once its bytes have landed
            // (a phase is issued only after the previous one has been consumed).
            if (nx0) mbar_wait(&full_x[0], (nx0 - 1) & 1);
            if (nx1) mbar_wait(&full_x[1], (nx1 - 1) & 1);
            if (nb) mbar_wait(&full_b, (nb - 1) & 1);
            if (nc) {
                mbar_wait(&full_c[0], (nc - 1) & 1);
                mbar_wait(&full_c[1], (nc - 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ UMMA issuer
        // The whole warp runs the loop (warp-uniform descriptors), one elected lane issues.
        const uint32_t id_cb = idesc_bf16(128, 128, 0, 0), id_z = idesc_bf16(128, 128, 0, 1);
        const uint32_t id_s = idesc_bf16(128, 128, 1, 1), id_y = idesc_bf16(128, 64, 0, 1);
        const uint64_t dCk = smem_desc(smem_u32(sC), 16, 1024), dBk = smem_desc(smem_u32(sB), 16, 1024);
        const uint64_t dBm = smem_desc(smem_u32(sB), 16384, 1024);
        const uint64_t dH = smem_desc(smem_u32(sH), 16384, 1024), dW = smem_desc(smem_u32(sW), 16384, 1024);
        const uint64_t dX = smem_desc(smem_u32(sX), 16384, 1024);
        // C B^T of chunk j into the M columns (fp32): dstate columns 0..63 once B and the
        // first half of C have landed, 64..127 once the second half has.
        auto issue_cb = [&](int j) -> bool {
            if (!wait_issue_warp(&full_b, j & 1, abort_p)) return false;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                if (!wait_issue_warp(&full_c[hf], j & 1, abort_p)) return false;
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int k = 4 * hf; k < 4 * hf + 4; ++k)
                        umma_bf16(tM, desc_add(dCk, kmajor_step(128, k)), desc_add(dBk, kmajor_step(128, k)), id_cb,
                                  k > 0);
                    if (hf == 1) umma_commit(&cb_done);
                }
                __syncwarp();
            }
            return true;
        };
        // test hook (stall): before the first UMMAs, a wait that runs out
        bool ok = !(stall && !wait_issue_warp(&stall_bar, 0, abort_p)) && (ntiles == 0 || issue_cb(0));
        for (int it = 0; it < ntiles && ok; ++it) {
            if (!wait_issue_warp(&ops_ready, it & 1, abort_p)) break;
            tc_fence_after();
            const uint64_t dX0 = desc_add(dX, (it & 1) * 32768), dX1 = desc_add(dX0, 16384);
            if (elect_one()) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    umma_bf16(tS, desc_add(dBm, k * kMnStep), desc_add(dW, k * kMnStep), id_s, k > 0);
                umma_commit(&s_done);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    umma_bf16(tZ, desc_add(dCk, kmajor_step(128, k)), desc_add(dH, k * kMnStep), id_z, k > 0);
                umma_commit(&zs_done);
                // M of head hh, sources 16k..16k+15: TMEM columns 16k + 8hh of the M block.
#pragma unroll
                for (int k = 0; k < 8; ++k) umma_bf16_ts(tY, tM + 16 * k, desc_add(dX0, k * kMnStep), id_y, k > 0);
                umma_commit(&y0_done);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    umma_bf16_ts(tY + 64, tM + 16 * k + 8, desc_add(dX1, k * kMnStep), id_y, k > 0);
                umma_commit(&mma_done);
            }
            __syncwarp();
            if (it + 1 < ntiles) {
                if (!wait_issue_warp(&mma_done, it & 1, abort_p)) break;   // the Y UMMAs have read M
                ok = issue_cb(it + 1);
            }
        }
        // Every MMA issued above has completed once this commit arrives.
        if (elect_one()) umma_commit(&drained);
        __syncwarp();
        mbar_wait(&drained, 0);
    } else if (warp == kScanWarp) {
        // ------------------------------------------------------------ dt scan
        // Chunk by chunk, up to four ahead of the compute warps: dt, the log2-scaled
        // cumulative dt*A and the decay weights of both heads into buffer j % 4. Lane l
        // holds tokens 4l..4l+3; the dt_raw of chunk j+1 is loaded while chunk j is scanned.
        float bias[kHeadsB], Ah[kHeadsB];
#pragma unroll
        for (int hh = 0; hh < kHeadsB; ++hh) {
            bias[hh] = dt_bias[h0 + hh];
            Ah[hh] = A[h0 + hh];
            if (lane == 0 && (!(Ah[hh] <= 0.f) || isinf(Ah[hh]))) latch_error(SSD_ERR_INVALID_ARG);
        }
        float z[kHeadsB][4], zn[kHeadsB][4];       // dt_raw of chunk j and of chunk j+1
        auto load_dt = [&](int j, float (&zz)[kHeadsB][4]) {
            const int tlj = min(kTile, seg.len - j * kTile);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int64_t row = ((int64_t)seg.start + (int64_t)j * kTile + 4 * lane + i) * H + h0;
#pragma unroll
                for (int hh = 0; hh < kHeadsB; ++hh) zz[hh][i] = 4 * lane + i < tlj ? dt_raw[row + hh] : 0.f;
            }
        };
        if (ntiles > 0) load_dt(0, zn);
        for (int j = 0; j < ntiles; ++j) {
            const int bf = j % 4;
#pragma unroll
            for (int hh = 0; hh < kHeadsB; ++hh)
#pragma unroll
                for (int i = 0; i < 4; ++i) z[hh][i] = zn[hh][i];
            if (j + 1 < ntiles) load_dt(j + 1, zn);
            if (j >= 4) wait_abort(&dt_free[bf], ((j >> 2) - 1) & 1, abort_p);
            const int tlj = min(kTile, seg.len - j * kTile);
#pragma unroll
            for (int hh = 0; hh < kHeadsB; ++hh) {
                float dtv[4], p[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    dtv[i] = 4 * lane + i < tlj ? softplus_fast(z[hh][i] + bias[hh]) : 0.f;
                    p[i] = (i ? p[i - 1] : 0.f) + dtv[i] * Ah[hh];
                }
                float incl = p[3];
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float v = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += v;
                }
                const float excl = incl - p[3];
                float av[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) av[i] = (excl + p[i]) * kLog2e;
                const float a_blk = __shfl_sync(0xffffffffu, av[3], (lane & ~7) | 7);    // token 32b + 31
                const float a_end = __shfl_sync(0xffffffffu, av[3], 31);                 // token 127
                float u[4], w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    u[i] = fast_exp2(a_blk - av[i]) * dtv[i];
                    w[i] = fast_exp2(a_end - av[i]) * dtv[i];
                }
                *reinterpret_cast<float4*>(&ac2[bf][hh][4 * lane]) = make_float4(av[0], av[1], av[2], av[3]);
                *reinterpret_cast<float4*>(&dts[bf][hh][4 * lane]) = make_float4(dtv[0], dtv[1], dtv[2], dtv[3]);
                *reinterpret_cast<float4*>(&uw[bf][hh][4 * lane]) = make_float4(u[0], u[1], u[2], u[3]);
                *reinterpret_cast<float4*>(&ww[bf][hh][4 * lane]) = make_float4(w[0], w[1], w[2], w[3]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&dt_ready[bf]);
        }
    } else {
        // ------------------------------------------------------------ compute warpgroups
        const int q = warp & 3;                     // TMEM lane quarter of this warp
        const int r = q * 32 + lane;                // row: token t, source s or state row n
        const int cw = (warp - kRoleWarps) >> 2;    // column quarter / source block
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        float h[kHeadsB][16];                       // h[head][n = r][p = 16*cw + j]
#pragma unroll
        for (int hh = 0; hh < kHeadsB; ++hh) {
            // layout [slot][H][P][N]: for each p the warp reads 32 consecutive n
            const float* src = hin + (((int64_t)seg.pad * H + h0 + hh) * kP + 16 * cw) * kN + r;
#pragma unroll
            for (int j = 0; j < 16; ++j) h[hh][j] = src[j * kN];
        }
        const float Dh0 = D[h0], Dh1 = D[h0 + 1];
        // Decays of the diagonal 32x32 blocks of chunk j, L[t][s] = exp2(Acum_t - Acum_s)
        // dt_s for s <= t in t's block (fp16). Thread (cw, r) writes row t = r of head
        // cw & 1, sources 16 (cw >> 1) .. +15 of the block. 16-byte chunk c of a row sits
        // at chunk c ^ ((t >> 1) & 3).
        auto diag_decays = [&](int j) {
            const int bf = j % 4, hd = cw & 1, c0 = 2 * (cw >> 1);
            wait_abort(&dt_ready[bf], (j / 4) & 1, abort_p);
            const float at = ac2[bf][hd][r];
            const float4* a4 = reinterpret_cast<const float4*>(&ac2[bf][hd][32 * q + 8 * c0]);
            const float4* d4 = reinterpret_cast<const float4*>(&dts[bf][hd][32 * q + 8 * c0]);
            const uint32_t row = smem_u32(sL + hd * 8192 + r * 64);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t o[4];
#pragma unroll
                for (int k2 = 0; k2 < 2; ++k2) {
                    const float4 as = a4[2 * c + k2], dv = d4[2 * c + k2];
                    const int s0 = 8 * (c0 + c) + 4 * k2;   // source offset within the block
                    const float l0 = s0 <= lane ? fast_exp2(at - as.x) * dv.x : 0.f;
                    const float l1 = s0 + 1 <= lane ? fast_exp2(at - as.y) * dv.y : 0.f;
                    const float l2 = s0 + 2 <= lane ? fast_exp2(at - as.z) * dv.z : 0.f;
                    const float l3 = s0 + 3 <= lane ? fast_exp2(at - as.w) * dv.w : 0.f;
                    o[2 * k2] = pack_f16(l0, l1);
                    o[2 * k2 + 1] = pack_f16(l2, l3);
                }
                st_shared_v4(row + (((c0 + c) ^ ((r >> 1) & 3)) << 4), o[0], o[1], o[2], o[3]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&l_ready);
        };
        // w*X of chunk j for both heads into shared memory.
        auto stage_wx = [&](int j) {
            const int bf = j % 4, sl = j & 1;
            wait_abort(&dt_ready[bf], (j / 4) & 1, abort_p);
            wait_abort(&full_x[sl], (j >> 1) & 1, abort_p);
#pragma unroll
            for (int hh = 0; hh < kHeadsB; ++hh) {
                const float w = ww[bf][hh][r];
                const uint32_t w2 = pack_bf16(w, w);
                const uint32_t xrow = smem_u32(sX + sl * 32768 + hh * 16384), wrow = smem_u32(sW + hh * 16384);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const uint4 v = ld_shared_v4(xrow + swz(r, 2 * cw + c));
                    st_shared_v4(wrow + swz(r, 2 * cw + c), hmul2_bf16(v.x, w2), hmul2_bf16(v.y, w2),
                                 hmul2_bf16(v.z, w2), hmul2_bf16(v.w, w2));
                }
            }
        };
        // bf16 h (from the registers) for both heads into shared memory.
        auto stage_h = [&]() {
#pragma unroll
            for (int hh = 0; hh < kHeadsB; ++hh) {
                const uint32_t hrow = smem_u32(sH + hh * 16384);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t pk[4];
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) pk[jj] = pack_bf16(h[hh][8 * c + 2 * jj], h[hh][8 * c + 2 * jj + 1]);
                    st_shared_v4(hrow + swz(r, 2 * cw + c), pk[0], pk[1], pk[2], pk[3]);
                }
            }
        };

        diag_decays(0);
        stage_h();
        stage_wx(0);

        for (int it = 0; it < ntiles; ++it) {
            const int64_t t0 = seg.start + (int64_t)it * kTile;
            const int tl = min(kTile, seg.len - it * kTile);
            const int bf = it % 4;
            wait_abort(&dt_ready[bf], (it / 4) & 1, abort_p);
            wait_abort(&l_ready, it & 1, abort_p);
            wait_abort(&cb_done, it & 1, abort_p);
            tc_fence_after();
            // -------- M[t][s] of both heads, t = r, in place over C B^T. Source block b
            // (32 sources) keeps its 32 columns: half j (sources 16j..16j+15 of the
            // block) becomes M of head 0 in its first 8 columns and of head 1 in the
            // next 8. The diagonal block q is done half by half (both heads) by the warps
            // of lane quarter q that have no block below the diagonal (cw >= q): warp
            // cw takes the halves j = cw - q, cw - q + (4 - q), ... < 2. Each half is read
            // and overwritten by one warp only.
            auto diag_half = [&](int jh) {
                const int sd = 32 * q + 16 * jh;
                uint32_t rc[16];
                tmem_ld16(tM + lane_off + sd, rc);
                tmem_wait_ld();
                const int jd = r - sd;              // D joins M on the diagonal (s = t)
#pragma unroll
                for (int hd = 0; hd < kHeadsB; ++hd) {
                    const uint32_t lrow = smem_u32(sL + hd * 8192 + r * 64);
                    const int c0 = 2 * jh;
                    const uint4 la = ld_shared_v4(lrow + ((c0 ^ ((r >> 1) & 3)) << 4));
                    const uint4 lb = ld_shared_v4(lrow + (((c0 + 1) ^ ((r >> 1) & 3)) << 4));
                    const uint32_t lw[8] = {la.x, la.y, la.z, la.w, lb.x, lb.y, lb.z, lb.w};
                    const float Dd = hd ? Dh1 : Dh0;
                    uint32_t pk[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        float2 m = fmul2(f16x2_to_f2(lw[k]),
                                         make_float2(__uint_as_float(rc[2 * k]), __uint_as_float(rc[2 * k + 1])));
                        if (jd == 2 * k) m.x += Dd;
                        if (jd == 2 * k + 1) m.y += Dd;
                        pk[k] = pack_bf16(m);
                    }
                    tmem_st8(tM + lane_off + sd + 8 * hd, pk);
                }
            };
            if (cw >= q && cw - q < 2) diag_half(cw - q);
            if (q == 3 && cw == 3) diag_half(1);    // lane quarter 3: warp cw = 3 takes both halves
            if (cw < q) {                          // below the diagonal: factorized
                float2 v[kHeadsB];
#pragma unroll
                for (int hh = 0; hh < kHeadsB; ++hh) {
                    const float vv = fast_exp2(ac2[bf][hh][r] - ac2[bf][hh][32 * cw + 31]);
                    v[hh] = make_float2(vv, vv);
                }
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const uint32_t col = lane_off + 32 * cw + 16 * half;
                    uint32_t rc[16];
                    tmem_ld16(tM + col, rc);
                    tmem_wait_ld();
#pragma unroll
                    for (int hh = 0; hh < kHeadsB; ++hh) {
                        const float4* u4 = reinterpret_cast<const float4*>(&uw[bf][hh][32 * cw + 16 * half]);
                        uint32_t pk[8];
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            const float4 u = u4[k4];
                            const float2 m01 = fmul2(make_float2(__uint_as_float(rc[4 * k4]), __uint_as_float(rc[4 * k4 + 1])),
                                                     fmul2(v[hh], make_float2(u.x, u.y)));
                            const float2 m23 = fmul2(make_float2(__uint_as_float(rc[4 * k4 + 2]), __uint_as_float(rc[4 * k4 + 3])),
                                                     fmul2(v[hh], make_float2(u.z, u.w)));
                            pk[2 * k4] = pack_bf16(m01);
                            pk[2 * k4 + 1] = pack_bf16(m23);
                        }
                        tmem_st8(tM + col + 8 * hh, pk);
                    }
                }
            } else if (cw > q) {                   // above the diagonal: zero
                const uint32_t zero[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) tmem_st8(tM + lane_off + 32 * cw + 8 * c8, zero);
            }
            tmem_wait_st();
            fence_proxy_async_smem();              // bf16 h and w*X of this chunk
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ops_ready);
            // -------- while S and Z run: all compute warps tabulate chunk it+1's diagonal
            // decays once every warp has read chunk it's (ops_ready complete).
            if (it + 1 < ntiles) {
                wait_abort(&ops_ready, it & 1, abort_p);
                diag_decays(it + 1);
            }
            // -------- S done: w*X of the next chunk (its buffer was read by this chunk's S).
            // Z done (the Y UMMAs may still run): state update, then bf16 h of the next
            // chunk (its buffer was read by this chunk's Z).
            if (it + 1 < ntiles) {
                wait_abort(&s_done, it & 1, abort_p);
                stage_wx(it + 1);
            }
            wait_abort(&zs_done, it & 1, abort_p);
            tc_fence_after();
#pragma unroll
            for (int hh = 0; hh < kHeadsB; ++hh) {
                uint32_t rs[16];
                tmem_ld16(tS + hh * 64 + lane_off + 16 * cw, rs);
                tmem_wait_ld();
                const float decay = fast_exp2(ac2[bf][hh][kTile - 1]);
                const float2 dc = make_float2(decay, decay);
#pragma unroll
                for (int j = 0; j < 16; j += 2) {
                    const float2 hn = ffma2(dc, make_float2(h[hh][j], h[hh][j + 1]),
                                            make_float2(__uint_as_float(rs[j]), __uint_as_float(rs[j + 1])));
                    h[hh][j] = hn.x;
                    h[hh][j + 1] = hn.y;
                }
            }
            if (it + 1 < ntiles) stage_h();
            // -------- drain: y rows (into the chunk's X slot for a full chunk, else
            // straight to HBM). The TMEM loads of the next 8-column piece are issued before the
            // current one is consumed.
            wait_abort(&y0_done, it & 1, abort_p);
            tc_fence_after();
            {
                const bool staged = tl == kTile;
                uint32_t ry[2][8], rz[2][8];
                tmem_ld8(tY + lane_off + 16 * cw, ry[0]);
                tmem_ld8(tZ + lane_off + 16 * cw, rz[0]);
                const float et0 = fast_exp2(ac2[bf][0][r]), et1 = fast_exp2(ac2[bf][1][r]);
                const float2 e20 = make_float2(et0, et0), e21 = make_float2(et1, et1);
#pragma unroll
                for (int piece = 0; piece < 4; ++piece) {           // (head, half) = (piece/2, piece%2)
                    const int hh = piece >> 1, half = piece & 1, cur = piece & 1;
                    tmem_wait_ld();
                    if (piece == 1) {                               // head 1's Y needs all Y UMMAs
                        wait_abort(&mma_done, it & 1, abort_p);
                        tc_fence_after();
                    }
                    if (piece < 3) {
                        const int nh = (piece + 1) >> 1, nf = (piece + 1) & 1;
                        tmem_ld8(tY + nh * 64 + lane_off + 16 * cw + 8 * nf, ry[cur ^ 1]);
                        tmem_ld8(tZ + nh * 64 + lane_off + 16 * cw + 8 * nf, rz[cur ^ 1]);
                    }
                    const float2 et = hh ? e21 : e20;
                    uint32_t o[4];
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj)
                        o[jj] = pack_bf16(ffma2(et, make_float2(__uint_as_float(rz[cur][2 * jj]), __uint_as_float(rz[cur][2 * jj + 1])),
                                                make_float2(__uint_as_float(ry[cur][2 * jj]), __uint_as_float(ry[cur][2 * jj + 1]))));
                    if (staged) {
                        st_shared_v4(smem_u32(sX + (it & 1) * 32768 + hh * 16384) + swz(r, 2 * cw + half), o[0], o[1],
                                     o[2], o[3]);
                    } else if (r < tl) {
                        *reinterpret_cast<uint4*>(y + ((t0 + r) * H + h0 + hh) * kP + 16 * cw + 8 * half) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&y_staged);
                mbar_arrive(&dt_free[bf]);          // this chunk's dt buffer is no longer read
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tbase, 512);
}

}  // namespace tc
}  // namespace ssd
