// Chunked SSD prefill, CUDA-core FP32 pipeline (all dtypes and supported dims).
//
// The chunked SSD algorithm (JAX Nemotron 3 Nano page, "Key Components" 1; RL-Kernel
// issue page, Figure 2, the chunked-scan box) splits each sequence into chunks of Q
// tokens anchored at the sequence start and evaluates the recurrence as:
//
//   chunk_cumsum   dt_s = softplus(dt_raw_s + dt_bias), Acum_s = sum_{r<=s in chunk} dt_r A
//   chunk_state    S_c = sum_{s in c} exp(Acum_last - Acum_s) dt_s x_s B_s^T     (zero-start
//                  state at the chunk's end)
//   state_passing  h_in(first chunk) = init; h_in(c+1) = exp(Acum_last(c)) h_in(c) + S_c;
//                  final_state = the value after the sequence's last chunk
//   chunk_scan     y_t = sum_{s<=t in c} (C_t.B_s) exp(Acum_t - Acum_s) dt_s x_s
//                        + exp(Acum_t) C_t.h_in(c) + D x_t
//
// Every exponent above is <= 0 because A <= 0, so nothing overflows; decays that
// underflow are true zeros to within float precision.
#pragma once

#include "ssd_common.cuh"

namespace ssd {

// ---------------------------------------------------------------------------------
// Chunk table (one block). Builds one entry per chunk and first[s] = index of the
// first chunk of sequence s (first[nseq] = number of chunks). Packed mode validates
// cu_seqlens (cu[0] == 0, non-decreasing, cu[nseq] == T); on failure it latches
// SSD_ERR_INVALID_ARG and emits an empty table, so later kernels touch nothing.
// With `order` (entries of at most 128 chunks of 128 tokens), order[k] is the entry the
// k-th CTA of a pass takes: longest entries first (by 128-token chunks), so that CTAs of
// unequal length finish together (longest-processing-time-first scheduling).
// An entry's `pad` holds its index in the table. With `sub_first` (entries of the
// tensor-core pipeline and state snapshots every `snap` tokens, snap a multiple of 128),
// every entry is further cut at the multiples of snap that fall inside it (positions
// counted from its sequence's start) into sub-segments, numbered in token order over the
// whole call: `pad` becomes the number of the entry's first sub-segment, sub_first[s] that
// of sequence s's first one (sub_first[nseq] = their count), and sub_end[k] is where
// sub-segment k ends, counted from its sequence's start.
constexpr int kTableThreads = 1024;

// Exclusive prefix sum of v over the kTableThreads threads of the block (warp shuffles,
// then the 32 warp totals); *total = the sum over the block. wsum: 32 shared slots, free
// again after the next barrier.
__device__ __forceinline__ int32_t table_scan(int32_t v, int32_t* wsum, int32_t* total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int32_t x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) wsum[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int32_t w = wsum[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
        }
        wsum[lane] = w;
    }
    __syncthreads();
    *total = wsum[31];
    return (wid ? wsum[wid - 1] : 0) + x - v;
}

__global__ void __launch_bounds__(kTableThreads)
k_chunk_table(const int32_t* __restrict__ cu, int32_t nseq, int64_t T, int64_t seqlen, int Q,
              ChunkEntry* __restrict__ table, int32_t* __restrict__ first,
              int32_t* __restrict__ count, int64_t snap, int32_t* __restrict__ snap_first,
              int32_t* __restrict__ order = nullptr, int32_t* __restrict__ sub_first = nullptr,
              int32_t* __restrict__ sub_end = nullptr) {
    static_assert(kTableThreads == 32 * 32, "table_scan assumes 32 warps");
    __shared__ int32_t wsum[3][32];
    const int tid = threadIdx.x;
    const int per = (nseq + kTableThreads - 1) / kTableThreads;
    const int s0 = min(nseq, tid * per), s1 = min(nseq, s0 + per);
    auto seq_begin = [&](int s) -> int64_t { return cu ? (int64_t)cu[s] : (int64_t)s * seqlen; };

    int bad = 0;
    if (cu) {
        for (int s = s0; s < s1; ++s) bad |= (cu[s + 1] < cu[s]);
        if (tid == 0) bad |= (cu[0] != 0) || ((int64_t)cu[nseq] != T);
    }
    bad = __syncthreads_or(bad);
    if (bad) {
        if (tid == 0) latch_error(SSD_ERR_INVALID_ARG);
        for (int s = tid; s <= nseq; s += kTableThreads) first[s] = 0;
        if (tid == 0) *count = 0;
        return;
    }
    int32_t local = 0;
    for (int s = s0; s < s1; ++s) {
        int64_t len = seq_begin(s + 1) - seq_begin(s);
        local += (int32_t)((len + Q - 1) / Q);
    }
    int32_t nent = 0;
    int32_t run = table_scan(local, wsum[0], &nent);
    for (int s = s0; s < s1; ++s) {
        first[s] = run;
        const int64_t b = seq_begin(s), len = seq_begin(s + 1) - b;
        const int32_t nc = (int32_t)((len + Q - 1) / Q);
        for (int32_t j = 0; j < nc; ++j) {
            ChunkEntry e;
            e.seq = s;
            e.start = (int32_t)(b + (int64_t)j * Q);
            { const int64_t rem = len - (int64_t)j * Q; e.len = (int32_t)(rem < Q ? rem : Q); }
            e.pad = run + j;
            table[run + j] = e;
        }
        run += nc;
    }
    if (tid == kTableThreads - 1) {
        first[nseq] = nent;
        *count = nent;
    }
    if (order) {                                          // counting sort by chunks, descending
        __shared__ int32_t hist[129];
        __syncthreads();                                  // every entry is written
        const int32_t n = nent;
        for (int b = tid; b < 129; b += kTableThreads) hist[b] = 0;
        __syncthreads();
        for (int32_t i = tid; i < n; i += kTableThreads) atomicAdd(&hist[min(128, (table[i].len + 127) / 128)], 1);
        __syncthreads();
        if (tid == 0) {
            int32_t r = 0;
            for (int b = 128; b >= 0; --b) {
                const int32_t c = hist[b];
                hist[b] = r;
                r += c;
            }
        }
        __syncthreads();
        for (int32_t i = tid; i < n; i += kTableThreads)
            order[atomicAdd(&hist[min(128, (table[i].len + 127) / 128)], 1)] = i;
    }
    if (snap > 0) {                                       // snapshots: floor(len / snap) per sequence
        int32_t nsnap = 0, tot = 0;
        for (int s = s0; s < s1; ++s) nsnap += (int32_t)((seq_begin(s + 1) - seq_begin(s)) / snap);
        int32_t r2 = table_scan(nsnap, wsum[1], &tot);
        for (int s = s0; s < s1; ++s) {
            snap_first[s] = r2;
            r2 += (int32_t)((seq_begin(s + 1) - seq_begin(s)) / snap);
        }
        if (tid == kTableThreads - 1) snap_first[nseq] = tot;
    }
    if (snap > 0 && sub_first) {                          // sub-segments cut at multiples of snap
        int32_t nsub = 0, tot = 0;
        for (int s = s0; s < s1; ++s) {                   // entries plus the cuts strictly inside them
            const int64_t len = seq_begin(s + 1) - seq_begin(s);
            int64_t cut = snap;
            for (int64_t r0 = 0; r0 < len; r0 += Q) {
                const int64_t r1 = r0 + Q < len ? r0 + Q : len;
                for (++nsub; cut < r1; cut += snap) ++nsub;
                if (cut == r1) cut += snap;
            }
        }
        int32_t k = table_scan(nsub, wsum[2], &tot);
        for (int s = s0; s < s1; ++s) {
            sub_first[s] = k;
            const int64_t len = seq_begin(s + 1) - seq_begin(s);
            int32_t c = first[s];
            int64_t cut = snap;                                   // next multiple of snap
            for (int64_t r0 = 0; r0 < len; r0 += Q, ++c) {
                const int64_t r1 = r0 + Q < len ? r0 + Q : len;
                table[c].pad = k;
                for (; cut < r1; cut += snap) sub_end[k++] = (int32_t)cut;
                sub_end[k++] = (int32_t)r1;
                if (cut == r1) cut += snap;
            }
        }
        if (tid == kTableThreads - 1) sub_first[nseq] = tot;
    }
}

// ---------------------------------------------------------------------------------
// chunk_cumsum: dt and the in-chunk inclusive cumulative sum of dt*A, per (chunk,
// head), as [chunk][H][Q] arrays. Positions past the chunk's end get dt = 0 and
// a flat Acum. One block = one chunk x 32 heads; a warp scans one head at a time.
template <int Q>
__global__ void __launch_bounds__(256)
k_chunk_cumsum(const float* __restrict__ dt_raw, const float* __restrict__ dt_bias,
               const float* __restrict__ A, const ChunkEntry* __restrict__ table,
               const int32_t* __restrict__ count, int H, float* __restrict__ dt_out,
               float* __restrict__ acum_out) {
    __shared__ float raw[Q][33];
    const int c = blockIdx.x;
    if (c >= *count) return;
    const ChunkEntry e = table[c];
    const int h0 = blockIdx.y * 32;
    for (int i = threadIdx.x; i < Q * 32; i += 256) {
        const int r = i >> 5, col = i & 31, h = h0 + col;
        raw[r][col] = (r < e.len && h < H) ? dt_raw[(int64_t)(e.start + r) * H + h] : 0.f;
    }
    __syncthreads();
    constexpr int PER = Q / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int col = warp; col < 32; col += 8) {
        const int h = h0 + col;
        if (h >= H) break;
        const float bias = dt_bias[h], a = A[h];
        if (!(a <= 0.f) || isinf(a)) latch_error(SSD_ERR_INVALID_ARG);
        float dtv[PER], cum[PER];
        float run = 0.f;
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int r = lane * PER + k;
            dtv[k] = r < e.len ? softplus_f32(raw[r][col] + bias) : 0.f;
            run += dtv[k] * a;
            cum[k] = run;
        }
        float incl = run;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            float v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        const float excl = incl - run;
        const int64_t base = ((int64_t)c * H + h) * Q + lane * PER;
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            dt_out[base + k] = dtv[k];
            acum_out[base + k] = excl + cum[k];
        }
    }
}

// ---------------------------------------------------------------------------------
// chunk_state: S_c[p][n] = sum_s w_s x_s[p] B_s[n], w_s = exp(Acum_last - Acum_s) dt_s.
// One block = one (chunk, head); thread owns column n = tid % N and rows
// p = tid / N + k * (256 / N).
template <typename T, int Q, int P, int N>
__global__ void __launch_bounds__(256)
k_chunk_state_simt(const T* __restrict__ x, const T* __restrict__ B,
                   const float* __restrict__ dtc, const float* __restrict__ acum,
                   const ChunkEntry* __restrict__ table, const int32_t* __restrict__ count,
                   int H, int G, float* __restrict__ states) {
    constexpr int NOUT = P * N / 256;
    constexpr int PSTEP = 256 / N;
    __shared__ float w[Q];
    __shared__ float xs[32][P];
    __shared__ float bs[32][N];
    const int c = blockIdx.x;
    if (c >= *count) return;
    const int h = blockIdx.y, g = h / (H / G), tid = threadIdx.x;
    const ChunkEntry e = table[c];
    const float* ac = acum + ((int64_t)c * H + h) * Q;
    const float* dv = dtc + ((int64_t)c * H + h) * Q;
    const float last = ac[e.len - 1];
    for (int s = tid; s < Q; s += 256) w[s] = expf(last - ac[s]) * dv[s];
    const int n = tid % N, p0 = tid / N;
    float acc[NOUT];
#pragma unroll
    for (int k = 0; k < NOUT; ++k) acc[k] = 0.f;
    __syncthreads();
    for (int s0 = 0; s0 < e.len; s0 += 32) {
        for (int i = tid; i < 32 * P; i += 256) {
            const int r = i / P, pp = i % P;
            const int64_t t = e.start + s0 + r;
            xs[r][pp] = (s0 + r < e.len) ? w[s0 + r] * to_f32(x[(t * H + h) * P + pp]) : 0.f;
        }
        for (int i = tid; i < 32 * N; i += 256) {
            const int r = i / N, nn = i % N;
            const int64_t t = e.start + s0 + r;
            bs[r][nn] = (s0 + r < e.len) ? to_f32(B[(t * G + g) * N + nn]) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int r = 0; r < 32; ++r) {
            const float bv = bs[r][n];
#pragma unroll
            for (int k = 0; k < NOUT; ++k) acc[k] = fmaf(xs[r][p0 + k * PSTEP], bv, acc[k]);
        }
        __syncthreads();
    }
    float* out = states + ((int64_t)c * H + h) * P * N;
#pragma unroll
    for (int k = 0; k < NOUT; ++k) out[(p0 + k * PSTEP) * N + n] = acc[k];
}

// ---------------------------------------------------------------------------------
// state_passing: sequential over the chunks of one sequence, parallel over (head,
// state element). Overwrites each chunk's S_c with the state entering that chunk,
// h_in(c), and writes final_state.
template <int Q>
__global__ void __launch_bounds__(256)
k_state_passing(float* __restrict__ states, const float* __restrict__ acum,
                const ChunkEntry* __restrict__ table, const int32_t* __restrict__ first,
                const float* __restrict__ init, float* __restrict__ final_state, int H, int PN,
                int64_t snap, const int32_t* __restrict__ snap_first, float* __restrict__ snap_out) {
    const int s = blockIdx.x, h = blockIdx.y;
    const int i = blockIdx.z * 256 + threadIdx.x;
    if (i >= PN) return;
    float hv = init ? init[((int64_t)s * H + h) * PN + i] : 0.f;
    const int c0 = first[s], c1 = first[s + 1];
    const int64_t seq0 = c1 > c0 ? table[c0].start : 0;
    for (int c = c0; c < c1; ++c) {
        const ChunkEntry e = table[c];
        const float decay = expf(acum[((int64_t)c * H + h) * Q + e.len - 1]);
        float* slot = states + ((int64_t)c * H + h) * PN + i;
        const float sv = *slot;
        *slot = hv;
        hv = fmaf(decay, hv, sv);
        if (snap > 0) {                                   // state after a multiple of snap tokens
            const int64_t end = (int64_t)e.start + e.len - seq0;
            if (end % snap == 0) snap_out[((int64_t)(snap_first[s] + end / snap - 1) * H + h) * PN + i] = hv;
        }
    }
    if (final_state) final_state[((int64_t)s * H + h) * PN + i] = hv;
}

// ---------------------------------------------------------------------------------
// chunk_scan: y for 32 rows of one (chunk, head). Thread owns column p = tid % P and
// rows t = tid / P + k * (256 / P).
template <typename T, int Q, int P, int N>
__global__ void __launch_bounds__(256)
k_chunk_scan_simt(const T* __restrict__ x, const T* __restrict__ B, const T* __restrict__ C,
                  const float* __restrict__ D, const float* __restrict__ dtc,
                  const float* __restrict__ acum, const float* __restrict__ hin,
                  const ChunkEntry* __restrict__ table, const int32_t* __restrict__ count,
                  int H, int G, T* __restrict__ y) {
    constexpr int NOUT = 32 * P / 256;
    constexpr int TSTEP = 256 / P;
    extern __shared__ float smem[];
    float* acs = smem;                    // [Q]
    float* dts = acs + Q;                 // [Q]
    float* cs = dts + Q;                  // [32][N+1]
    float* bs = cs + 32 * (N + 1);        // [32][N+1]
    float* xs = bs + 32 * (N + 1);        // [32][P]
    float* ms = xs + 32 * P;              // [32][33]
    float* hs = ms + 32 * 33;             // [P][33]
    const int c = blockIdx.x;
    if (c >= *count) return;
    const ChunkEntry e = table[c];
    const int tb = blockIdx.z;
    if (tb * 32 >= e.len) return;
    const int h = blockIdx.y, g = h / (H / G), tid = threadIdx.x;
    const int64_t cbase = ((int64_t)c * H + h) * Q;
    for (int i = tid; i < Q; i += 256) {
        acs[i] = acum[cbase + i];
        dts[i] = dtc[cbase + i];
    }
    const int t0 = tb * 32;
    for (int i = tid; i < 32 * N; i += 256) {
        const int r = i / N, nn = i % N;
        const int64_t t = e.start + t0 + r;
        cs[r * (N + 1) + nn] = (t0 + r < e.len) ? to_f32(C[(t * G + g) * N + nn]) : 0.f;
    }
    const int p = tid % P, r0 = tid / P;
    float acc[NOUT];
#pragma unroll
    for (int k = 0; k < NOUT; ++k) acc[k] = 0.f;
    __syncthreads();

    // (1) C_t . h_in over N, in slices of 32 state columns.
    const float* hp = hin + ((int64_t)c * H + h) * P * N;
    for (int n0 = 0; n0 < N; n0 += 32) {
        for (int i = tid; i < P * 32; i += 256) {
            const int pp = i / 32, j = i % 32;
            hs[pp * 33 + j] = (n0 + j < N) ? hp[pp * N + n0 + j] : 0.f;
        }
        __syncthreads();
        const int jmax = min(32, N - n0);
        for (int j = 0; j < jmax; ++j) {
            const float hv = hs[p * 33 + j];
#pragma unroll
            for (int k = 0; k < NOUT; ++k)
                acc[k] = fmaf(cs[(r0 + k * TSTEP) * (N + 1) + n0 + j], hv, acc[k]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int k = 0; k < NOUT; ++k) acc[k] *= expf(acs[t0 + r0 + k * TSTEP]);

    // (2) intra-chunk causal part over 32-token source tiles s <= t.
    for (int s0 = 0; s0 <= t0; s0 += 32) {
        for (int i = tid; i < 32 * N; i += 256) {
            const int r = i / N, nn = i % N;
            const int64_t t = e.start + s0 + r;
            bs[r * (N + 1) + nn] = (s0 + r < e.len) ? to_f32(B[(t * G + g) * N + nn]) : 0.f;
        }
        for (int i = tid; i < 32 * P; i += 256) {
            const int r = i / P, pp = i % P;
            const int64_t t = e.start + s0 + r;
            xs[r * P + pp] = (s0 + r < e.len) ? to_f32(x[(t * H + h) * P + pp]) : 0.f;
        }
        __syncthreads();
        for (int q = tid; q < 32 * 32; q += 256) {
            const int tt = q >> 5, ss = q & 31;
            const int ta = t0 + tt, sa = s0 + ss;
            float v = 0.f;
            if (sa <= ta && sa < e.len) {
                float dot = 0.f;
                for (int nn = 0; nn < N; ++nn) dot = fmaf(cs[tt * (N + 1) + nn], bs[ss * (N + 1) + nn], dot);
                v = dot * expf(acs[ta] - acs[sa]) * dts[sa];
            }
            ms[tt * 33 + ss] = v;
        }
        __syncthreads();
        for (int ss = 0; ss < 32; ++ss) {
            const float xv = xs[ss * P + p];
#pragma unroll
            for (int k = 0; k < NOUT; ++k) acc[k] = fmaf(ms[(r0 + k * TSTEP) * 33 + ss], xv, acc[k]);
        }
        __syncthreads();
    }

    // (3) D skip and store.
    const float Dh = D[h];
#pragma unroll
    for (int k = 0; k < NOUT; ++k) {
        const int tt = t0 + r0 + k * TSTEP;
        if (tt < e.len) {
            const int64_t o = ((int64_t)(e.start + tt) * H + h) * P + p;
            y[o] = from_f32<T>(acc[k] + Dh * to_f32(x[o]));
        }
    }
}

template <int Q, int P, int N>
constexpr size_t chunk_scan_simt_smem() {
    return sizeof(float) * (2 * Q + 2 * 32 * (N + 1) + 32 * P + 32 * 33 + P * 33);
}

}  // namespace ssd
