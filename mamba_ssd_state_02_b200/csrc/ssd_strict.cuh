// Strict mode: a chunked SSD prefill and a chunk-emulating decode step that give the
// same bits for the same token however the sequence was split between them.
//
// The RL-Kernel issue page (§4.1, batch invariance: a token's output must not depend on
// whether it came from training, prefill of any length or decode at any step; §7: train,
// prefill and decode of the Mamba-2 mixer share device functions, and the decode emulates
// the chunked arithmetic) asks for this with a fixed reduction order, fixed FP32
// accumulation and no fast-math reassociation.
//
// How it is met here. Both paths evaluate the chunked algorithm (chunks of Q tokens
// anchored at the sequence start) through the functions in `namespace strict` below,
// each a fixed sequence of correctly rounded FP32 operations (__fadd_rn, __fmul_rn,
// __fmaf_rn: never contracted or reordered by the compiler) and deterministic exponentials
// (strict_exp for the decays and weights, library expf/log1pf for softplus):
//
//   dt_s      = softplus(dt_raw_s + dt_bias)
//   Acum_s    = Acum_{s-1} + dt_s A            (left to right from Acum_{-1} = 0)
//   w(t, s)   = exp(Acum_t - Acum_s) dt_s
//   y_t[p]    = D x_t[p] + ( exp(Acum_t) (C_t . h_in[p]) + sum_{s=0..t} (C_t . B_s) w(t,s) x_s[p] )
//   S[p][n]   = sum_{s=0..Q-1} (w(last, s) x_s[p]) B_s[n]
//   h_in'     = exp(Acum_last) h_in + S
//
// with every dot product and every sum taken left to right over its index. The decode
// keeps, per sequence, the state at the start of its open chunk and the open chunk's
// x, B, dt and Acum (the chunk cache); a decode step computes the new token's y with the
// same functions over the same operands in the same order as the prefill would for that
// chunk position, and when the chunk fills it folds the chunk into the state exactly as
// the prefill's chunk-state and state-passing kernels do. The result is bitwise
// independent of batch size, batch position and the split between prefill and decode at
// any token; a prefill may resume from a cache whose open chunk is empty (a split at a
// chunk boundary) and fails closed otherwise.
#pragma once

#include "ssd_common.cuh"

namespace ssd {
namespace strict {

// ---------------------------------------------------------------------------------
// The arithmetic shared by the strict prefill and the chunk-emulating decode.
__device__ __forceinline__ float dt_of(float raw, float bias) {
    const float z = __fadd_rn(raw, bias);
    return z > 0.f ? __fadd_rn(z, log1pf(expf(-z))) : log1pf(expf(z));
}
// exp(x) of the decays and weights: one correctly rounded multiply by log2(e), then the
// hardware base-2 exponential (relative error ~2^-21). Deterministic, and the same function
// on every path, which is all bitwise invariance needs.
__device__ __forceinline__ float strict_exp(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(__fmul_rn(x, 1.4426950408889634f)));
    return y;
}
__device__ __forceinline__ float acum_next(float prev, float dt, float a) {
    return __fadd_rn(prev, __fmul_rn(dt, a));
}
// w(t, s) = exp(Acum_t - Acum_s) dt_s
__device__ __forceinline__ float src_weight(float acum_t, float acum_s, float dt_s) {
    return __fmul_rn(strict_exp(__fsub_rn(acum_t, acum_s)), dt_s);
}
// one step of a left-to-right dot product
__device__ __forceinline__ float dot_step(float acc, float u, float v) { return __fmaf_rn(u, v, acc); }
// coefficient of x_s in y_t: (C_t . B_s) w(t, s)
__device__ __forceinline__ float mix_coef(float cb, float acum_t, float acum_s, float dt_s) {
    return __fmul_rn(cb, src_weight(acum_t, acum_s, dt_s));
}
// y accumulator: start from the incoming-state term, add sources left to right, add D x_t
__device__ __forceinline__ float y_begin(float c_dot_h, float acum_t) { return __fmul_rn(c_dot_h, strict_exp(acum_t)); }
__device__ __forceinline__ float y_step(float acc, float coef, float xs) { return __fmaf_rn(coef, xs, acc); }
__device__ __forceinline__ float y_end(float acc, float Dh, float xt) { return __fmaf_rn(Dh, xt, acc); }
// chunk state: source term w(last, s) x_s[p], accumulated left to right against B_s[n]
__device__ __forceinline__ float state_src(float w, float xs) { return __fmul_rn(w, xs); }
__device__ __forceinline__ float state_step(float acc, float wx, float b) { return __fmaf_rn(wx, b, acc); }
// state passing across a chunk boundary
__device__ __forceinline__ float pass(float h, float acum_last, float S) { return __fmaf_rn(strict_exp(acum_last), h, S); }
// Two independent steps of the sums above at once: per component the same correctly
// rounded FMA (u v + acc) as the scalar steps, so a tile that packs its outputs in pairs
// produces the same bits as one that does not. Halves the issued FMA instructions.
__device__ __forceinline__ float2 step2(float2 acc, float2 u, float2 v) { return __ffma2_rn(u, v, acc); }
__device__ __forceinline__ float2 splat(float v) { return make_float2(v, v); }

__device__ __forceinline__ bool bad_A(float a) { return !(a <= 0.f) || isinf(a); }

constexpr int kThreads = 256;

// The register tile of a chunk-state sum S[p][n] = sum_s wx_s[p] b_s[n], sources left to
// right, with NOUT = P N / 256 outputs per thread. When NOUT is a multiple of 4 a thread
// owns R = NOUT / 4 consecutive rows p0.. and 4 consecutive columns n0.. (per source one
// 16-byte load of b and R/4 of wx for 4R FMAs); otherwise one column n0 and NOUT rows.
// Rows are held in pairs (acc[i / 2][j], component i % 2), so that four rows of a source
// update with packed FMAs; at(i, j) is output (p0 + i, n0 + j).
template <int NOUT>
struct StateTile {
    static constexpr bool kWide = NOUT % 4 == 0;
    static constexpr int R = kWide ? NOUT / 4 : NOUT, CN = kWide ? 4 : 1;
    float2 acc[(R + 1) / 2][CN];
    int p0, n0;
    __device__ __forceinline__ float& at(int i, int j) { return (i & 1) ? acc[i >> 1][j].y : acc[i >> 1][j].x; }
    __device__ __forceinline__ StateTile(int tid, int N) {
        if (kWide) {
            n0 = (tid % (N / 4)) * 4;
            p0 = (tid / (N / 4)) * R;
        } else {
            n0 = tid % N;
            p0 = (tid / N) * NOUT;
        }
#pragma unroll
        for (int i = 0; i < (R + 1) / 2; ++i)
#pragma unroll
            for (int j = 0; j < CN; ++j) acc[i][j] = make_float2(0.f, 0.f);
    }
    // One source: xr = its wx row [P], br = its b row [N] (shared memory).
    __device__ __forceinline__ void row(const float* xr, const float* br) {
        float bv[CN];
        if constexpr (kWide) {
            const float4 b = *reinterpret_cast<const float4*>(br + n0);
            bv[0] = b.x;
            bv[1] = b.y;
            bv[2] = b.z;
            bv[3] = b.w;
        } else {
            bv[0] = br[n0];
        }
        if constexpr (R % 4 == 0) {
            float2 bb[CN];
#pragma unroll
            for (int j = 0; j < CN; ++j) bb[j] = splat(bv[j]);
#pragma unroll
            for (int i = 0; i < R; i += 4) {
                const float4 v = *reinterpret_cast<const float4*>(xr + p0 + i);
                const float2 va[2] = {make_float2(v.x, v.y), make_float2(v.z, v.w)};
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                    for (int j = 0; j < CN; ++j) acc[i / 2 + a][j] = step2(acc[i / 2 + a][j], va[a], bb[j]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const float v = xr[p0 + i];
#pragma unroll
                for (int j = 0; j < CN; ++j) at(i, j) = state_step(at(i, j), v, bv[j]);
            }
        }
    }
};

// A tile of raw rows (n elements, rows of P) to FP32 in shared memory, 16 bytes per step:
// dst[i] = state_src(scale[i / P], src[i]), or src[i] when scale is null. P is a power of
// two and a multiple of the step's element count; src and dst are 16-byte aligned.
template <typename T>
__device__ __forceinline__ void tile_to_f32(float* dst, const T* src, int n, int P, const float* scale, int tid) {
    constexpr int V = 16 / (int)sizeof(T);
    const int lp = __ffs(P) - 1;
    for (int v = tid; v < n / V; v += kThreads) {
        const int i = v * V;
        const uint4 u = *reinterpret_cast<const uint4*>(src + i);
        float f[V];
        if constexpr (V == 8) {
            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                f[2 * k] = __uint_as_float(w4[k] << 16);
                f[2 * k + 1] = __uint_as_float(w4[k] & 0xffff0000u);
            }
        } else {
            f[0] = __uint_as_float(u.x);
            f[1] = __uint_as_float(u.y);
            f[2] = __uint_as_float(u.z);
            f[3] = __uint_as_float(u.w);
        }
        if (scale) {
            const float sc = scale[i >> lp];
#pragma unroll
            for (int k = 0; k < V; ++k) f[k] = state_src(sc, f[k]);
        }
#pragma unroll
        for (int k = 0; k < V; k += 4)
            *reinterpret_cast<float4*>(dst + i + k) = make_float4(f[k], f[k + 1], f[k + 2], f[k + 3]);
    }
}

// ---------------------------------------------------------------------------------
// Prefill stage 1: dt and Acum per (chunk, head), left to right, [chunk][H][Q] (past the
// chunk's end dt is zero and Acum holds its value at the last token). One thread per
// (chunk, head); 16 tokens' raw dt are loaded before their 16 dependent steps, and dt, Acum
// go out as 16-byte stores (Q is a multiple of 32).
__global__ void __launch_bounds__(128)
k_strict_cumsum(const float* __restrict__ dt_raw, const float* __restrict__ dt_bias, const float* __restrict__ A,
                const ChunkEntry* __restrict__ table, const int32_t* __restrict__ count, int H, int Q,
                float* __restrict__ dt_out, float* __restrict__ acum_out) {
    const int c = blockIdx.x;
    const int h = blockIdx.y * 128 + threadIdx.x;
    if (c >= *count || h >= H) return;
    const ChunkEntry e = table[c];
    const float bias = dt_bias[h], a = A[h];
    if (bad_A(a)) latch_error(SSD_ERR_INVALID_ARG);
    const int64_t base = ((int64_t)c * H + h) * Q;
    float run = 0.f;
    constexpr int U = 16;
    for (int r0 = 0; r0 < Q; r0 += U) {
        float raw[U], dv[U], av[U];
#pragma unroll
        for (int u = 0; u < U; ++u) raw[u] = r0 + u < e.len ? dt_raw[(int64_t)(e.start + r0 + u) * H + h] : 0.f;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float d = 0.f;
            if (r0 + u < e.len) {
                d = dt_of(raw[u], bias);
                run = acum_next(run, d, a);
            }
            dv[u] = d;
            av[u] = run;
        }
#pragma unroll
        for (int u = 0; u < U; u += 4) {
            *reinterpret_cast<float4*>(dt_out + base + r0 + u) = make_float4(dv[u], dv[u + 1], dv[u + 2], dv[u + 3]);
            *reinterpret_cast<float4*>(acum_out + base + r0 + u) = make_float4(av[u], av[u + 1], av[u + 2], av[u + 3]);
        }
    }
}

// ---------------------------------------------------------------------------------
// Prefill stage 2: chunk states S_c[p][n] (zero-start state at the chunk's last token).
// One block per (chunk, head); a thread owns a StateTile of NOUT = P N / 256 outputs.
// The chunk is walked in tiles of 32
// tokens: the raw x and B rows of tile t+1 are copied into shared memory (16-byte
// asynchronous copies) while tile t is used; each tile is converted once to FP32 (x
// scaled by w(last, s)).
template <typename T, int NOUT>
__global__ void __launch_bounds__(kThreads)
k_strict_chunk_state(const T* __restrict__ x, const T* __restrict__ B, const float* __restrict__ dtc,
                     const float* __restrict__ acum, const ChunkEntry* __restrict__ table,
                     const int32_t* __restrict__ count, int H, int G, int P, int N, int Q,
                     float* __restrict__ states) {
    extern __shared__ __align__(16) float sm[];
    float* w = sm;                       // [Q]
    float* xs = w + Q;                   // [32][P]   w(last, s) x_s
    float* bs = xs + 32 * P;             // [32][N]
    T* raw = reinterpret_cast<T*>(bs + 32 * N);   // [2][32 (P + N)] raw x rows, then B rows, of a tile
    // Block b: head b % H of chunk b / H, so the heads of one chunk run side by side (B in L2).
    const int c = (int)(blockIdx.x / (unsigned)H);
    if (c >= *count) return;
    const int h = (int)(blockIdx.x % (unsigned)H), g = h / (H / G), tid = threadIdx.x;
    const ChunkEntry e = table[c];
    constexpr int V = 16 / (int)sizeof(T);                 // elements per 16-byte copy
    const int tile_elems = 32 * (P + N), ntile = (e.len + 31) / 32;
    auto fetch = [&](int t) {                               // rows of tile t into buffer t & 1
        T* dst = raw + (t & 1) * tile_elems;
        const int rows = min(32, e.len - 32 * t), xp = P / V, bp = N / V;
        for (int i = tid; i < rows * xp; i += kThreads) {
            const int r = i / xp, k = i % xp;
            cp_async16(dst + r * P + k * V, x + ((int64_t)(e.start + 32 * t + r) * H + h) * P + k * V);
        }
        for (int i = tid; i < rows * bp; i += kThreads) {
            const int r = i / bp, k = i % bp;
            cp_async16(dst + 32 * P + r * N + k * V, B + ((int64_t)(e.start + 32 * t + r) * G + g) * N + k * V);
        }
        cp_async_commit();
    };
    fetch(0);
    const float* ac = acum + ((int64_t)c * H + h) * Q;
    const float* dv = dtc + ((int64_t)c * H + h) * Q;
    const float last = ac[e.len - 1];
    for (int s = tid; s < e.len; s += kThreads) w[s] = src_weight(last, ac[s], dv[s]);
    StateTile<NOUT> tile(tid, N);
    for (int t = 0; t < ntile; ++t) {
        if (t + 1 < ntile) {
            fetch(t + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();                                    // tile t landed (all threads' copies); w
        const int rows = min(32, e.len - 32 * t);
        const T* rx = raw + (t & 1) * tile_elems;
        const T* rb = rx + 32 * P;
        tile_to_f32(xs, rx, rows * P, P, w + 32 * t, tid);
        tile_to_f32(bs, rb, rows * N, N, static_cast<const float*>(nullptr), tid);
        __syncthreads();
        for (int r = 0; r < rows; ++r) tile.row(xs + r * P, bs + r * N);
        __syncthreads();                                    // xs, bs and buffer t & 1 free again
    }
    float* out = states + ((int64_t)c * H + h) * P * N;
#pragma unroll
    for (int i = 0; i < StateTile<NOUT>::R; ++i)
#pragma unroll
        for (int j = 0; j < StateTile<NOUT>::CN; ++j) out[(tile.p0 + i) * N + tile.n0 + j] = tile.at(i, j);
}

// ---------------------------------------------------------------------------------
// Prefill stage 3: state passing, sequential over a sequence's chunks, parallel over
// (head, state element), four consecutive elements per thread. Overwrites S_c with
// h_in(c), writes the final state and the cache state (the state entering the sequence's
// open chunk: h_in of a partial last chunk, else the final state). `resume`: start from
// cache_state, whose open chunk must be empty (cache_len == 0), else SSD_ERR_UNSUPPORTED is
// latched (fail closed).
__global__ void __launch_bounds__(kThreads, 4)
k_strict_passing(float* __restrict__ states, const float* __restrict__ acum, const ChunkEntry* __restrict__ table,
                 const int32_t* __restrict__ first, int resume, float* __restrict__ cache_state,
                 const int32_t* __restrict__ cache_len, float* __restrict__ final_state, int H, int PN, int Q) {
    const int s = blockIdx.x, h = blockIdx.y;
    const int i = (blockIdx.z * kThreads + threadIdx.x) * 4;     // elements i .. i + 3 (PN % 4 == 0)
    if (i >= PN) return;
    const int64_t slot0 = ((int64_t)s * H + h) * PN + i;
    float hv[4] = {0.f, 0.f, 0.f, 0.f};
    if (resume) {
        if (cache_len[(int64_t)s * H + h] != 0) latch_error(SSD_ERR_UNSUPPORTED);
#pragma unroll
        for (int k = 0; k < 4; ++k) hv[k] = cache_state[slot0 + k];
    }
    const int c0 = first[s], c1 = first[s + 1];
    float open[4] = {hv[0], hv[1], hv[2], hv[3]};
    // Groups of four chunks, double-buffered: the next group's loads are in flight while
    // this one is applied (same arithmetic per element).
    constexpr int U = 4;
    struct Group {
        float4 sv[U];
        float al[U];
        int len[U];
    };
    auto load = [&](int c, Group& g) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (c + u < c1) {
                g.len[u] = table[c + u].len;
                g.sv[u] = *reinterpret_cast<const float4*>(states + ((int64_t)(c + u) * H + h) * PN + i);
                g.al[u] = acum[((int64_t)(c + u) * H + h) * Q + g.len[u] - 1];
            }
        }
    };
    auto apply = [&](int c, const Group& g) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (c + u < c1) {
                *reinterpret_cast<float4*>(states + ((int64_t)(c + u) * H + h) * PN + i) =
                    make_float4(hv[0], hv[1], hv[2], hv[3]);
                const float sv[4] = {g.sv[u].x, g.sv[u].y, g.sv[u].z, g.sv[u].w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    open[k] = hv[k];
                    hv[k] = pass(hv[k], g.al[u], sv[k]);
                    if (g.len[u] == Q) open[k] = hv[k];
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
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        cache_state[slot0 + k] = open[k];
        if (final_state) final_state[slot0 + k] = hv[k];
    }
}

// ---------------------------------------------------------------------------------
// Prefill stage 4: y for 32 rows of one chunk and every head of one group. One block per
// (chunk, group, 32-row tile), 256 threads:
//   1. C_t . B_s for the tile's rows and every source s <= t, once for the group
//      (2x2 (t, s) pairs per thread, 16-byte shared loads along n);
//   2. per head: the coefficients (C_t . B_s) w(t, s); the incoming-state term
//      C_t . h_in[p] (TA x TB (t, p) outputs per thread, 16-byte loads along n); the
//      sources s = 0..t left to right; D x_t; store.
// Thread (rg, pg) owns rows rg*TA + i and columns pg + j*PG (PG = P / TB).
template <int P> struct ScanTile;
template <> struct ScanTile<16> { static constexpr int TA = 2, TB = 1; };
template <> struct ScanTile<32> { static constexpr int TA = 2, TB = 2; };
template <> struct ScanTile<64> { static constexpr int TA = 4, TB = 2; };
template <> struct ScanTile<128> { static constexpr int TA = 4, TB = 4; };

constexpr int kHPad = 36;    // row stride of the h_in slice [P][32 + 4]

__host__ __device__ inline int scan_cb_region(int N, int Q) { return 32 * (Q > N + 4 ? Q : N + 4); }

template <typename T, int P>
__global__ void __launch_bounds__(kThreads)
k_strict_chunk_scan(const T* __restrict__ x, const T* __restrict__ B, const T* __restrict__ C,
                    const float* __restrict__ D, const float* __restrict__ dtc, const float* __restrict__ acum,
                    const float* __restrict__ hin, const ChunkEntry* __restrict__ table,
                    const int32_t* __restrict__ count, int H, int G, int N, int Q, T* __restrict__ y) {
    constexpr int TA = ScanTile<P>::TA, TB = ScanTile<P>::TB, PG = P / TB;
    static_assert((32 / TA) * PG == kThreads, "tile covers 32 rows x P columns");
    extern __shared__ __align__(16) float sm[];
    const int NS = N + 4;                 // row stride of C and B tiles
    float* cs = sm;                       // [32][N+4]   C rows of the tile
    float* ms = cs + 32 * NS;             // [32][Q] coefficients (aliases the B slice [32][N+4])
    float* bs = ms;
    float* cbm = ms + scan_cb_region(N, Q);   // [32][Q]  C_t . B_s
    float* acs = cbm + 32 * Q;            // [Q]
    float* dts = acs + Q;                 // [Q]
    float* hs = dts + Q;                  // [P][36]
    float* xs = hs + P * kHPad;           // [32][P]
    // Block b: tile b % (Q/32), group (b / (Q/32)) % G, chunk b / ((Q/32) G): the tiles of
    // one (chunk, group) run side by side and share its B, incoming states and x in L2.
    const int ntile = Q / 32;
    const int c = (int)(blockIdx.x / (unsigned)(ntile * G));
    if (c >= *count) return;
    const ChunkEntry e = table[c];
    const int t0 = (int)(blockIdx.x % (unsigned)ntile) * 32;
    if (t0 >= e.len) return;
    const int g = (int)((blockIdx.x / (unsigned)ntile) % (unsigned)G), hpg = H / G, tid = threadIdx.x;
    const int rows = min(32, e.len - t0);
    for (int i = tid; i < 32 * N; i += kThreads) {
        const int r = i / N, nn = i % N;
        cs[r * NS + nn] = r < rows ? to_f32(C[((int64_t)(e.start + t0 + r) * G + g) * N + nn]) : 0.f;
    }

    // (1) C_t . B_s, left to right over n, for s <= t (source slices of 32).
    {
        const int ti = 2 * (tid >> 4), sj = tid & 15;     // rows ti, ti+1; sources sj, sj+16
        for (int s0 = 0; s0 <= t0; s0 += 32) {
            const int srows = min(32, e.len - s0);
            __syncthreads();
            for (int i = tid; i < 32 * N; i += kThreads) {
                const int r = i / N, nn = i % N;
                bs[r * NS + nn] = r < srows ? to_f32(B[((int64_t)(e.start + s0 + r) * G + g) * N + nn]) : 0.f;
            }
            __syncthreads();
            float d[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
            for (int n = 0; n < N; n += 4) {
                const float4 c0 = *reinterpret_cast<const float4*>(cs + ti * NS + n);
                const float4 c1 = *reinterpret_cast<const float4*>(cs + (ti + 1) * NS + n);
                const float4 b0 = *reinterpret_cast<const float4*>(bs + sj * NS + n);
                const float4 b1 = *reinterpret_cast<const float4*>(bs + (sj + 16) * NS + n);
                const float cv[2][4] = {{c0.x, c0.y, c0.z, c0.w}, {c1.x, c1.y, c1.z, c1.w}};
                const float bv[2][4] = {{b0.x, b0.y, b0.z, b0.w}, {b1.x, b1.y, b1.z, b1.w}};
#pragma unroll
                for (int k = 0; k < 4; ++k)
#pragma unroll
                    for (int a = 0; a < 2; ++a)
#pragma unroll
                        for (int b = 0; b < 2; ++b) d[a][b] = dot_step(d[a][b], cv[a][k], bv[b][k]);
            }
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b) cbm[(ti + a) * Q + s0 + sj + 16 * b] = d[a][b];
        }
    }
    const int rg = tid / PG, pg = tid % PG;
    const float* hbase = hin + (int64_t)c * H * P * N;
    for (int hh = 0; hh < hpg; ++hh) {
        const int h = g * hpg + hh;
        const int64_t cbase = ((int64_t)c * H + h) * Q;
        __syncthreads();                  // previous head done with ms, xs, hs, acs
        for (int i = tid; i < Q; i += kThreads) {
            acs[i] = acum[cbase + i];
            dts[i] = dtc[cbase + i];
        }
        __syncthreads();
        // (2a) coefficients of the tile's rows (only s <= t, s < len are used).
        for (int i = tid; i < 32 * (t0 + 32); i += kThreads) {
            const int tt = i / (t0 + 32), sa = i % (t0 + 32), ta = t0 + tt;
            if (sa <= ta && sa < e.len && tt < rows) ms[tt * Q + sa] = mix_coef(cbm[tt * Q + sa], acs[ta], acs[sa], dts[sa]);
        }
        // (2b) C_t . h_in[p], left to right over n, in slices of 32 columns.
        float acc[TA][TB];
#pragma unroll
        for (int i = 0; i < TA; ++i)
#pragma unroll
            for (int j = 0; j < TB; ++j) acc[i][j] = 0.f;
        const float* hp = hbase + (int64_t)h * P * N;
        for (int n0 = 0; n0 < N; n0 += 32) {
            const int cols = min(32, N - n0);
            __syncthreads();
            for (int i = tid; i < P * 32; i += kThreads) {
                const int pp = i / 32, jj = i % 32;
                hs[pp * kHPad + jj] = jj < cols ? hp[(int64_t)pp * N + n0 + jj] : 0.f;
            }
            __syncthreads();
            for (int q = 0; q < cols; q += 4) {
                float cv[TA][4], hv[TB][4];
#pragma unroll
                for (int i = 0; i < TA; ++i) {
                    const float4 v = *reinterpret_cast<const float4*>(cs + (rg * TA + i) * NS + n0 + q);
                    cv[i][0] = v.x; cv[i][1] = v.y; cv[i][2] = v.z; cv[i][3] = v.w;
                }
#pragma unroll
                for (int j = 0; j < TB; ++j) {
                    const float4 v = *reinterpret_cast<const float4*>(hs + (pg + j * PG) * kHPad + q);
                    hv[j][0] = v.x; hv[j][1] = v.y; hv[j][2] = v.z; hv[j][3] = v.w;
                }
#pragma unroll
                for (int k = 0; k < 4; ++k)
#pragma unroll
                    for (int i = 0; i < TA; ++i)
#pragma unroll
                        for (int j = 0; j < TB; ++j) acc[i][j] = dot_step(acc[i][j], cv[i][k], hv[j][k]);
            }
        }
#pragma unroll
        for (int i = 0; i < TA; ++i)
#pragma unroll
            for (int j = 0; j < TB; ++j) acc[i][j] = y_begin(acc[i][j], acs[t0 + rg * TA + i]);

        // (2c) sources s = 0..t, left to right, in 32-token slices.
        for (int s0 = 0; s0 <= t0; s0 += 32) {
            const int srows = min(32, e.len - s0);
            __syncthreads();
            for (int i = tid; i < 32 * P; i += kThreads) {
                const int r = i / P, pp = i % P;
                xs[i] = r < srows ? to_f32(x[((int64_t)(e.start + s0 + r) * H + h) * P + pp]) : 0.f;
            }
            __syncthreads();
            // Coefficients of four consecutive sources are read with one 16-byte load per
            // row; the sources are still added one at a time, left to right.
            if (s0 < t0) {                // every row of the tile sees all 32 sources
                for (int s4 = 0; s4 < 32; s4 += 4) {
                    float4 cf4[TA];
#pragma unroll
                    for (int i = 0; i < TA; ++i) cf4[i] = *reinterpret_cast<const float4*>(ms + (rg * TA + i) * Q + s0 + s4);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        float xv[TB];
#pragma unroll
                        for (int j = 0; j < TB; ++j) xv[j] = xs[(s4 + k) * P + pg + j * PG];
#pragma unroll
                        for (int i = 0; i < TA; ++i) {
                            const float cf = k == 0 ? cf4[i].x : k == 1 ? cf4[i].y : k == 2 ? cf4[i].z : cf4[i].w;
#pragma unroll
                            for (int j = 0; j < TB; ++j) acc[i][j] = y_step(acc[i][j], cf, xv[j]);
                        }
                    }
                }
            } else {                      // diagonal slice: sources s <= t, s < len
                for (int s4 = 0; s4 < srows; s4 += 4) {
                    float4 cf4[TA];
#pragma unroll
                    for (int i = 0; i < TA; ++i) cf4[i] = *reinterpret_cast<const float4*>(ms + (rg * TA + i) * Q + s0 + s4);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int ss = s4 + k;
                        if (ss >= srows) break;
                        float xv[TB];
#pragma unroll
                        for (int j = 0; j < TB; ++j) xv[j] = xs[ss * P + pg + j * PG];
#pragma unroll
                        for (int i = 0; i < TA; ++i) {
                            if (ss > rg * TA + i) continue;
                            const float cf = k == 0 ? cf4[i].x : k == 1 ? cf4[i].y : k == 2 ? cf4[i].z : cf4[i].w;
#pragma unroll
                            for (int j = 0; j < TB; ++j) acc[i][j] = y_step(acc[i][j], cf, xv[j]);
                        }
                    }
                }
            }
        }

        // (2d) D skip and store.
        const float Dh = D[h];
#pragma unroll
        for (int i = 0; i < TA; ++i) {
            const int tt = rg * TA + i;
            if (tt >= rows) continue;
#pragma unroll
            for (int j = 0; j < TB; ++j) {
                const int64_t o = ((int64_t)(e.start + t0 + tt) * H + h) * P + pg + j * PG;
                y[o] = from_f32<T>(y_end(acc[i][j], Dh, to_f32(x[o])));
            }
        }
    }
}

// Prefill stage 4 with wide register tiles, for P = 64 and heads per group a multiple of
// 4: the same outputs, operations and order as k_strict_chunk_scan. One block per (chunk,
// group, 32-row tile), 256 threads:
//   1. C_t . B_s for the tile's rows and every source s < min(len, t0 + 32), once for the
//      group, in 64-source slices (B rows transposed into shared memory; 4 x 2 (t, s) pairs
//      per thread), kept s-major;
//   2. the group's heads four at a time, 64 threads per head; thread (rg, pg) owns rows
//      8 rg .. 8 rg + 7 and columns 4 pg .. 4 pg + 3 (32 outputs): C_t . h_in[p] in 16-wide
//      slices of n (h_in transposed into shared memory by 4-byte asynchronous copies, the
//      next slice in flight while one is used), then the sources in 32-wide slices (the
//      head's coefficients (C_t . B_s) w(t, s) from its Acum and dt rows, staged once per
//      head, and the raw x rows, the next slice's copies in flight), then D x_t and the store.
constexpr int kWideHS = 68;   // row stride of a transposed h_in slice (16-byte rows)

// Floats of the work region: the B^T slice of (1), two h_in^T slices per head, or the
// coefficients and two raw x slices per head.
template <typename T>
__host__ __device__ inline int wide_work_floats(int N) {
    const int a = N * 64, b = 2 * 4 * 16 * kWideHS, c = 4 * 32 * 32 + 2 * 4 * 32 * 64 * (int)sizeof(T) / 4;
    return a > b ? (a > c ? a : c) : (b > c ? b : c);
}

// One 16-column slice of a head's h_in, transposed: hT[nn][p] = h_in[p][n0 + nn].
__device__ __forceinline__ void wide_h_slice(float* hT, const float* hsrc, int N, int n0, int u) {
    for (int i = u; i < 64 * 16; i += 64) {
        const int p = i / 16, nn = i % 16;
        cp_async4(hT + nn * kWideHS + p, hsrc + (int64_t)p * N + n0 + nn);
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 2)
k_strict_chunk_scan_wide(const T* __restrict__ x, const T* __restrict__ B, const T* __restrict__ C,
                         const float* __restrict__ D, const float* __restrict__ dtc, const float* __restrict__ acum,
                         const float* __restrict__ hin, const ChunkEntry* __restrict__ table,
                         const int32_t* __restrict__ count, int H, int G, int N, int Q, T* __restrict__ y) {
    constexpr int P = 64;
    constexpr int V = 16 / (int)sizeof(T);                 // elements per 16-byte copy
    extern __shared__ __align__(16) float sm[];
    float* cbs = sm;                      // [Q][32]  C_t . B_s: row s, column t (row of the tile)
    float* ct = cbs + Q * 32;             // [N][32]  the tile's C rows, transposed
    float* work = ct + N * 32;            // B^T slice [N][64]; or h_in^T slices [2][4 heads][16][68];
                                          // or coefficients [4 heads][32][32], then raw x [2][4 heads][32][64]
    float* acs = work + wide_work_floats<T>(N);   // [4 heads][Q] Acum
    float* dvs = acs + 4 * Q;                     // [4 heads][Q] dt
    const int ntile = Q / 32;
    const int c = (int)(blockIdx.x / (unsigned)(ntile * G));
    if (c >= *count) return;
    const ChunkEntry e = table[c];
    const int t0 = (int)(blockIdx.x % (unsigned)ntile) * 32;
    if (t0 >= e.len) return;
    const int g = (int)((blockIdx.x / (unsigned)ntile) % (unsigned)G), hpg = H / G, tid = threadIdx.x;
    const int rows = min(32, e.len - t0);
    const int nsrc = min(e.len, t0 + 32);                  // sources the tile's rows use: 0 .. nsrc-1
    const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);

    // (0) The tile's C rows, transposed (zero past the chunk's end).
    for (int i = tid; i < 32 * (N / 4); i += kThreads) {
        const int t = i % 32, n0 = (i / 32) * 4;
        const float4 v = t < rows ? load4(C + ((int64_t)(e.start + t0 + t) * G + g) * N + n0) : zero4;
        ct[(n0 + 0) * 32 + t] = v.x;
        ct[(n0 + 1) * 32 + t] = v.y;
        ct[(n0 + 2) * 32 + t] = v.z;
        ct[(n0 + 3) * 32 + t] = v.w;
    }

    // (1) C_t . B_s, left to right over n, 64 sources at a time.
    {
        const int ta = (tid % 8) * 4, sb = (tid / 8) * 2;   // rows ta..ta+3, slice sources sb, sb+1
        for (int s0 = 0; s0 < nsrc; s0 += 64) {
            __syncthreads();                                 // ct written; work free
            for (int i = tid; i < 64 * (N / 4); i += kThreads) {
                const int sl = i % 64, n0 = (i / 64) * 4;
                const float4 v = s0 + sl < nsrc ? load4(B + ((int64_t)(e.start + s0 + sl) * G + g) * N + n0) : zero4;
                work[(n0 + 0) * 64 + sl] = v.x;
                work[(n0 + 1) * 64 + sl] = v.y;
                work[(n0 + 2) * 64 + sl] = v.z;
                work[(n0 + 3) * 64 + sl] = v.w;
            }
            __syncthreads();
            float2 d[2][2];                                  // d[a][b]: rows ta + 2a, ta + 2a + 1; source sb + b
#pragma unroll
            for (int a = 0; a < 2; ++a) d[a][0] = d[a][1] = make_float2(0.f, 0.f);
            for (int n = 0; n < N; ++n) {
                const float4 cv = *reinterpret_cast<const float4*>(ct + n * 32 + ta);
                const float2 bv = *reinterpret_cast<const float2*>(work + n * 64 + sb);
                const float2 cva[2] = {make_float2(cv.x, cv.y), make_float2(cv.z, cv.w)};
                const float2 bx = splat(bv.x), by = splat(bv.y);
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    d[a][0] = step2(d[a][0], cva[a], bx);
                    d[a][1] = step2(d[a][1], cva[a], by);
                }
            }
#pragma unroll
            for (int b = 0; b < 2; ++b)
                if (s0 + sb + b < nsrc)
                    *reinterpret_cast<float4*>(cbs + (s0 + sb + b) * 32 + ta) = make_float4(d[0][b].x, d[0][b].y, d[1][b].x, d[1][b].y);
        }
    }

    // (2) The group's heads, four at a time.
    const int hl = tid / 64, u = tid % 64, r0 = (u / 16) * 8, p0 = (u % 16) * 4;
    float* cf = work + hl * (32 * 32);
    const float* ac = acs + hl * Q;
    const float* dv = dvs + hl * Q;
    auto hT = [&](int buf) { return work + (buf * 4 + hl) * (16 * kWideHS); };
    auto xs = [&](int buf) { return reinterpret_cast<T*>(work + 4 * 32 * 32) + (buf * 4 + hl) * (32 * P); };
    for (int hp = 0; hp < hpg; hp += 4) {
        const int h = g * hpg + hp + hl;
        const float* hsrc = hin + ((int64_t)c * H + h) * P * N;
        __syncthreads();                                     // work, acs and dvs free
        for (int i = u; i < Q / 4; i += 64) {
            cp_async16(acs + hl * Q + 4 * i, acum + ((int64_t)c * H + h) * Q + 4 * i);
            cp_async16(dvs + hl * Q + 4 * i, dtc + ((int64_t)c * H + h) * Q + 4 * i);
        }
        wide_h_slice(hT(0), hsrc, N, 0, u);
        cp_async_commit();
        float2 acc[4][4];                                    // rows r0 + 2i, r0 + 2i + 1; column p0 + j
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = make_float2(0.f, 0.f);
        // (2a) C_t . h_in[p], left to right over n, 16 at a time.
        for (int k = 0; k < N / 16; ++k) {
            if (k > 0) __syncthreads();                      // slice k - 1 used: its buffer is free
            if (k + 1 < N / 16) wide_h_slice(hT((k + 1) & 1), hsrc, N, 16 * (k + 1), u);
            cp_async_commit();
            cp_async_wait<1>();                              // slice k (and the Acum, dt rows) landed
            __syncthreads();
            const float* hb = hT(k & 1);
            const int n0 = 16 * k;
#pragma unroll 4
            for (int nn = 0; nn < 16; ++nn) {
                const float4 c0 = *reinterpret_cast<const float4*>(ct + (n0 + nn) * 32 + r0);
                const float4 c1 = *reinterpret_cast<const float4*>(ct + (n0 + nn) * 32 + r0 + 4);
                const float4 hv = *reinterpret_cast<const float4*>(hb + nn * kWideHS + p0);
                const float2 cva[4] = {make_float2(c0.x, c0.y), make_float2(c0.z, c0.w), make_float2(c1.x, c1.y),
                                       make_float2(c1.z, c1.w)};
                const float2 hva[4] = {splat(hv.x), splat(hv.y), splat(hv.z), splat(hv.w)};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = step2(acc[i][j], cva[i], hva[j]);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float a0 = ac[t0 + r0 + 2 * i], a1 = ac[t0 + r0 + 2 * i + 1];
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = make_float2(y_begin(acc[i][j].x, a0), y_begin(acc[i][j].y, a1));
        }
        // (2b) Sources s = 0..t, left to right, 32 at a time.
        const int nxs = t0 / 32 + 1;
        auto x_slice = [&](int k) {
            T* dst = xs(k & 1);
            const int s0 = 32 * k;
            for (int i = u; i < 32 * (P / V); i += 64) {
                const int r = i / (P / V), q = i % (P / V);
                if (s0 + r < e.len)
                    cp_async16(dst + r * P + q * V, x + ((int64_t)(e.start + s0 + r) * H + h) * P + q * V);
            }
        };
        __syncthreads();                                     // (2a) done: its buffers hold cf and x now
        x_slice(0);
        cp_async_commit();
        for (int k = 0; k < nxs; ++k) {
            const int s0 = 32 * k;
            if (k > 0) __syncthreads();                      // slice k - 1 used: cf and its x buffer free
            if (k + 1 < nxs) x_slice(k + 1);
            cp_async_commit();
            for (int i = u; i < 32 * 32; i += 64) {
                const int sl = i / 32, tl = i % 32, s_ = s0 + sl, t = t0 + tl;
                cf[i] = s_ <= t && s_ < e.len ? mix_coef(cbs[s_ * 32 + tl], ac[t], ac[s_], dv[s_]) : 0.f;
            }
            cp_async_wait<1>();                              // x of slice k landed
            __syncthreads();
            const T* xb = xs(k & 1);
            if (s0 < t0) {                                   // every row of the tile sees all 32 sources
#pragma unroll 4
                for (int kk = 0; kk < 32; ++kk) {
                    const float4 f0 = *reinterpret_cast<const float4*>(cf + kk * 32 + r0);
                    const float4 f1 = *reinterpret_cast<const float4*>(cf + kk * 32 + r0 + 4);
                    const float4 xv = load4(xb + kk * P + p0);
                    const float2 fva[4] = {make_float2(f0.x, f0.y), make_float2(f0.z, f0.w), make_float2(f1.x, f1.y),
                                           make_float2(f1.z, f1.w)};
                    const float2 xva[4] = {splat(xv.x), splat(xv.y), splat(xv.z), splat(xv.w)};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int j = 0; j < 4; ++j) acc[i][j] = step2(acc[i][j], fva[i], xva[j]);
                }
            } else {                                         // diagonal slice: sources s <= t
                // Source kk reaches the thread's rows r0 .. r0 + 7 while kk <= r0 + 7, and all
                // of them while kk <= r0.
                for (int kk = 0; kk < r0 + 8; ++kk) {
                    const float4 f0 = *reinterpret_cast<const float4*>(cf + kk * 32 + r0);
                    const float4 f1 = *reinterpret_cast<const float4*>(cf + kk * 32 + r0 + 4);
                    const float4 xv = load4(xb + kk * P + p0);
                    const float2 fva[4] = {make_float2(f0.x, f0.y), make_float2(f0.z, f0.w), make_float2(f1.x, f1.y),
                                           make_float2(f1.z, f1.w)};
                    const float xva[4] = {xv.x, xv.y, xv.z, xv.w};
                    if (kk <= r0) {
                        const float2 xs2[4] = {splat(xv.x), splat(xv.y), splat(xv.z), splat(xv.w)};
#pragma unroll
                        for (int i = 0; i < 4; ++i)
#pragma unroll
                            for (int j = 0; j < 4; ++j) acc[i][j] = step2(acc[i][j], fva[i], xs2[j]);
                        continue;
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        // rows r0 + 2i (takes source kk while kk <= r0 + 2i) and r0 + 2i + 1
                        if (kk > r0 + 2 * i + 1) continue;
                        if (kk == r0 + 2 * i + 1) {
#pragma unroll
                            for (int j = 0; j < 4; ++j) acc[i][j].y = y_step(acc[i][j].y, fva[i].y, xva[j]);
                        } else {
#pragma unroll
                            for (int j = 0; j < 4; ++j) acc[i][j] = step2(acc[i][j], fva[i], splat(xva[j]));
                        }
                    }
                }
            }
        }
        // (2c) D skip and store. x_t of the tile's rows is the last (diagonal) source slice,
        // still in shared memory (it starts at t0).
        const float Dh = D[h];
        const T* xl = xs((nxs - 1) & 1);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int tt = r0 + i;
            if (tt >= rows) continue;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t o = ((int64_t)(e.start + t0 + tt) * H + h) * P + p0 + j;
                const float a = (i & 1) ? acc[i >> 1][j].y : acc[i >> 1][j].x;
                y[o] = from_f32<T>(y_end(a, Dh, to_f32(xl[tt * P + p0 + j])));
            }
        }
    }
}

template <typename T>
inline size_t chunk_scan_wide_smem(int N, int Q) {
    return sizeof(float) * (Q * 32 + N * 32 + wide_work_floats<T>(N) + 8 * Q);
}

inline size_t chunk_scan_smem(int P, int N, int Q) {
    return sizeof(float) * (32 * (N + 4) + scan_cb_region(N, Q) + 32 * Q + 2 * Q + P * kHPad + 32 * P);
}
template <typename T>
inline size_t chunk_state_smem(int P, int N, int Q) {
    return sizeof(float) * (Q + 32 * P + 32 * N) + sizeof(T) * 2 * 32 * (P + N);
}

// ---------------------------------------------------------------------------------
// Prefill stage 5: the chunk cache's open chunk (a partial last chunk's tokens) and its
// length. One block per (sequence, head); the group's first head writes the B rows.
template <typename T>
__global__ void __launch_bounds__(kThreads)
k_strict_cache_fill(const T* __restrict__ x, const T* __restrict__ B, const float* __restrict__ dtc,
                    const float* __restrict__ acum, const ChunkEntry* __restrict__ table,
                    const int32_t* __restrict__ first, int H, int G, int P, int N, int Q, T* __restrict__ cx,
                    T* __restrict__ cB, float* __restrict__ cdt, float* __restrict__ cacum,
                    int32_t* __restrict__ clen) {
    const int s = blockIdx.x, h = blockIdx.y, g = h / (H / G), tid = threadIdx.x;
    const int c0 = first[s], c1 = first[s + 1];
    int open = 0;
    ChunkEntry e{0, 0, 0, 0};
    if (c1 > c0) {
        e = table[c1 - 1];
        open = e.len < Q ? e.len : 0;
    }
    if (tid == 0) clen[(int64_t)s * H + h] = open;
    if (open == 0) return;
    const int c = c1 - 1;
    for (int i = tid; i < open * P; i += kThreads) {
        const int r = i / P, pp = i % P;
        cx[(((int64_t)s * H + h) * Q + r) * P + pp] = x[((int64_t)(e.start + r) * H + h) * P + pp];
    }
    if (h % (H / G) == 0)
        for (int i = tid; i < open * N; i += kThreads) {
            const int r = i / N, nn = i % N;
            cB[(((int64_t)s * G + g) * Q + r) * N + nn] = B[((int64_t)(e.start + r) * G + g) * N + nn];
        }
    for (int r = tid; r < open; r += kThreads) {
        cdt[((int64_t)s * H + h) * Q + r] = dtc[((int64_t)c * H + h) * Q + r];
        cacum[((int64_t)s * H + h) * Q + r] = acum[((int64_t)c * H + h) * Q + r];
    }
}

// ---------------------------------------------------------------------------------
// Chunk-emulating decode step. One block per (sequence, group): its H/G heads share
// C_t and the cached B rows, so the dots C_t . B_s are taken once per group. With j =
// the open chunk's length (equal across the heads), the new token is position j of the
// open chunk: y is the prefill's y_t for t = j over sources 0..j (cached 0..j-1, the new
// token j), and the token is appended to the cache (len -> j + 1). A chunk that this
// fills (len == Q) is folded into the state by k_strict_fold, launched right after in
// the same call. Threads take the dots one source each, then the coefficients
// (C_t . B_s) w(j, s) of every head, then y[h][p] one (head, p) each.
//
// The incoming-state term C_t . h_in[p] reads each state row left to right in one thread.
// The group's state rows are contiguous, and they reach shared memory as slices of 16
// columns of up to 512 rows (64 bytes per row, four 16-byte asynchronous copies; a warp
// copies 8 whole row pieces per instruction) through a ring of three slices, the first two
// issued before the dots and coefficients are taken. In a slice, 16-byte chunk c of row r
// sits at chunk c ^ ((r >> 1) & 3), so that eight consecutive threads reading the same chunk
// of their own rows hit eight different bank groups.
constexpr int kDecThreads = 512;
constexpr int kDecSlice = 16;         // state columns per staged slice
constexpr int kDecStages = 3;

// Left-to-right dot of the float row c[0..N) with the row b[0..N) of T, 16-byte loads.
template <typename T>
__device__ __forceinline__ float row_dot(const float* c, const T* b, int N);
template <>
__device__ __forceinline__ float row_dot<__nv_bfloat16>(const float* c, const __nv_bfloat16* b, int N) {
    float d = 0.f;
    for (int n = 0; n < N; n += 8) {
        const uint4 u = *reinterpret_cast<const uint4*>(b + n);
        d = dot_step(d, c[n], __uint_as_float(u.x << 16));
        d = dot_step(d, c[n + 1], __uint_as_float(u.x & 0xffff0000u));
        d = dot_step(d, c[n + 2], __uint_as_float(u.y << 16));
        d = dot_step(d, c[n + 3], __uint_as_float(u.y & 0xffff0000u));
        d = dot_step(d, c[n + 4], __uint_as_float(u.z << 16));
        d = dot_step(d, c[n + 5], __uint_as_float(u.z & 0xffff0000u));
        d = dot_step(d, c[n + 6], __uint_as_float(u.w << 16));
        d = dot_step(d, c[n + 7], __uint_as_float(u.w & 0xffff0000u));
    }
    return d;
}
template <>
__device__ __forceinline__ float row_dot<float>(const float* c, const float* b, int N) {
    float d = 0.f;
    for (int n = 0; n < N; n += 4) {
        const float4 v = *reinterpret_cast<const float4*>(b + n);
        d = dot_step(d, c[n], v.x);
        d = dot_step(d, c[n + 1], v.y);
        d = dot_step(d, c[n + 2], v.z);
        d = dot_step(d, c[n + 3], v.w);
    }
    return d;
}

// Stage q: column slice q % nsl of the row batch q / nsl (rows 512 (q / nsl) ..), into
// ring slot q % 3. Every thread commits one group per stage (empty past the last).
__device__ __forceinline__ void decode_stage(float* ring, const float* st0, int q, int nst, int nsl, int rows,
                                             int N, int tid) {
    if (q < nst) {
        const int rb = (q / nsl) * kDecThreads, n0 = (q % nsl) * kDecSlice, nr = min(kDecThreads, rows - rb);
        float* dst = ring + (q % kDecStages) * (kDecThreads * kDecSlice);
        for (int i = tid; i < nr * 4; i += kDecThreads) {
            const int r = i >> 2, c = i & 3;
            cp_async16(dst + r * kDecSlice + ((c ^ ((r >> 1) & 3)) << 2), st0 + (int64_t)(rb + r) * N + n0 + (c << 2));
        }
    }
    cp_async_commit();
}

template <typename T>
__global__ void __launch_bounds__(kDecThreads, 2)
k_strict_decode(const float* __restrict__ cstate, T* __restrict__ cx, T* __restrict__ cB, float* __restrict__ cdt,
                float* __restrict__ cacum, int32_t* __restrict__ clen, const T* __restrict__ x,
                const float* __restrict__ dt_raw, const float* __restrict__ dt_bias, const float* __restrict__ A,
                const T* __restrict__ B, const T* __restrict__ C, const float* __restrict__ D, T* __restrict__ y,
                int H, int G, int P, int N, int Q) {
    extern __shared__ __align__(16) float sm[];
    const int hpg = H / G;
    float* ring = sm;                     // [3][512][16] state slices
    float* cs = ring + kDecStages * kDecThreads * kDecSlice;   // [N]       C_t
    float* dots = cs + N;                 // [Q]       C_t . B_s
    float* coef = dots + Q;               // [hpg][Q]  (C_t . B_s) w(j, s) per head
    float* hdt = coef + hpg * Q;          // [hpg]     the token's dt per head
    float* hac = hdt + hpg;               // [hpg]     the token's Acum per head
    __shared__ int s_j, s_bad;
    const int s = blockIdx.x / G, g = blockIdx.x % G, h0 = g * hpg, tid = threadIdx.x;
    const int rows = hpg * P, nsl = N / kDecSlice, nst = ((rows + kDecThreads - 1) / kDecThreads) * nsl;
    const float* st0 = cstate + ((int64_t)s * H + h0) * P * N;   // row r = hl P + p
    decode_stage(ring, st0, 0, nst, nsl, rows, N, tid);
    decode_stage(ring, st0, 1, nst, nsl, rows, N, tid);
    if (tid == 0) {
        s_j = clen[(int64_t)s * H + h0];
        s_bad = 0;
    }
    __syncthreads();
    const int j = s_j;
    for (int hl = tid; hl < hpg; hl += kDecThreads) {
        const int h = h0 + hl;
        const int64_t sh = (int64_t)s * H + h;
        const float a = A[h];
        if (clen[sh] != j || j < 0 || j >= Q || bad_A(a)) {   // not a cache this step can continue
            atomicOr(&s_bad, 1);
            continue;
        }
        const float d = dt_of(dt_raw[sh], dt_bias[h]);
        hdt[hl] = d;
        hac[hl] = acum_next(j > 0 ? cacum[sh * Q + j - 1] : 0.f, d, a);
    }
    const T* Bt = B + ((int64_t)s * G + g) * N;
    const T* Ct = C + ((int64_t)s * G + g) * N;
    const T* brow = cB + ((int64_t)s * G + g) * Q * N;     // cached B rows [Q][N]
    for (int n = tid; n < N; n += kDecThreads) cs[n] = to_f32(Ct[n]);
    __syncthreads();
    if (s_bad) {
        if (tid == 0) latch_error(SSD_ERR_INVALID_ARG);
        cp_async_wait<0>();                                  // no copy left in flight at exit
        return;
    }

    // C_t . B_s of sources 0..j (B_j: the token's B).
    for (int sidx = tid; sidx <= j; sidx += kDecThreads)
        dots[sidx] = row_dot<T>(cs, sidx < j ? brow + (int64_t)sidx * N : Bt, N);
    __syncthreads();
    // Coefficients of every head.
    for (int i = tid; i < hpg * (j + 1); i += kDecThreads) {
        const int hl = i / (j + 1), sidx = i % (j + 1);
        const int64_t sh = (int64_t)s * H + h0 + hl;
        const float acj = hac[hl];
        const float acs = sidx < j ? cacum[sh * Q + sidx] : acj;
        const float dts = sidx < j ? cdt[sh * Q + sidx] : hdt[hl];
        coef[hl * Q + sidx] = mix_coef(dots[sidx], acj, acs, dts);
    }
    __syncthreads();

    // y[h][p]: incoming-state term, sources left to right, D skip. Thread tid owns row
    // 512 b + tid of each row batch b.
    for (int rb = 0; rb < rows; rb += kDecThreads) {
        const int i = rb + tid;
        float dot = 0.f;
        for (int k = 0; k < nsl; ++k) {
            const int q = (rb / kDecThreads) * nsl + k;
            cp_async_wait<1>();                              // this thread's copies of stage q
            __syncthreads();                                 // everyone's; slot (q + 2) % 3 free again
            decode_stage(ring, st0, q + 2, nst, nsl, rows, N, tid);
            if (i < rows) {
                const float* src = ring + (q % kDecStages) * (kDecThreads * kDecSlice) + tid * kDecSlice;
                const float* cn = cs + k * kDecSlice;
                const int sw = (tid >> 1) & 3;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float4 v = *reinterpret_cast<const float4*>(src + ((c ^ sw) << 2));
                    dot = dot_step(dot, cn[4 * c], v.x);
                    dot = dot_step(dot, cn[4 * c + 1], v.y);
                    dot = dot_step(dot, cn[4 * c + 2], v.z);
                    dot = dot_step(dot, cn[4 * c + 3], v.w);
                }
            }
        }
        if (i >= rows) continue;
        const int hl = i / P, p = i % P, h = h0 + hl;
        const int64_t sh = (int64_t)s * H + h;
        const float* cf = coef + hl * Q;
        float acc = y_begin(dot, hac[hl]);
        const T* xp = cx + sh * Q * P + p;                  // cached x rows [Q][P]
        int sidx = 0;
        for (; sidx + 4 <= j; sidx += 4) {
            const float x0 = to_f32(xp[(int64_t)sidx * P]), x1 = to_f32(xp[(int64_t)(sidx + 1) * P]);
            const float x2 = to_f32(xp[(int64_t)(sidx + 2) * P]), x3 = to_f32(xp[(int64_t)(sidx + 3) * P]);
            acc = y_step(acc, cf[sidx], x0);
            acc = y_step(acc, cf[sidx + 1], x1);
            acc = y_step(acc, cf[sidx + 2], x2);
            acc = y_step(acc, cf[sidx + 3], x3);
        }
        for (; sidx < j; ++sidx) acc = y_step(acc, cf[sidx], to_f32(xp[(int64_t)sidx * P]));
        const float xv = to_f32(x[sh * P + p]);
        acc = y_step(acc, cf[j], xv);
        y[sh * P + p] = from_f32<T>(y_end(acc, D[h], xv));
    }

    // Append the token to the open chunk.
    for (int i = tid; i < hpg * P; i += kDecThreads) {
        const int64_t sh = (int64_t)s * H + h0 + i / P;
        cx[(sh * Q + j) * P + i % P] = x[sh * P + i % P];
    }
    T* bdst = cB + (((int64_t)s * G + g) * Q + j) * N;
    for (int n = tid; n < N; n += kDecThreads) bdst[n] = Bt[n];
    for (int hl = tid; hl < hpg; hl += kDecThreads) {
        const int64_t sh = (int64_t)s * H + h0 + hl;
        cdt[sh * Q + j] = hdt[hl];
        cacum[sh * Q + j] = hac[hl];
        clen[sh] = j + 1;
    }
}

inline size_t decode_smem(int H, int G, int N, int Q) {
    return sizeof(float) * (kDecStages * kDecThreads * kDecSlice + N + Q + (H / G) * (Q + 2));
}

// ---------------------------------------------------------------------------------
// Fold of a full open chunk (len == Q) into the cache state: the prefill's chunk-state
// and passing arithmetic, sources left to right; then len -> 0. The grid is a few blocks
// per SM; block b looks at its stretch of at most 32 (sequence, head) pairs (one load and
// one vote) and folds the full ones one after the other, so a step that fills no chunk
// costs one small launch. A fold walks the chunk in tiles of 32 sources: the raw x and B
// rows of tile t+1 are copied into shared memory (16-byte asynchronous copies) while tile
// t is used; each tile is converted once to FP32 (x scaled by w(last, s)). A thread owns a
// StateTile of NOUT = P N / 256 outputs.

template <typename T, int NOUT>
__global__ void __launch_bounds__(kThreads)
k_strict_fold(float* __restrict__ cstate, const T* __restrict__ cx, const T* __restrict__ cB,
              const float* __restrict__ cdt, const float* __restrict__ cacum, int32_t* __restrict__ clen, int H,
              int G, int P, int N, int Q, int npairs, int per_block) {
    extern __shared__ __align__(16) float sm[];
    float* wv = sm;                       // [Q]      w(last, s)
    float* xs = wv + Q;                   // [32][P]  w(last, s) x_s
    float* bs = xs + 32 * P;              // [32][N]
    T* raw = reinterpret_cast<T*>(bs + 32 * N);   // [2][32 (P + N)] raw x rows, then B rows, of a tile
    __shared__ int full[32], nfull;
    const int tid = threadIdx.x;
    if (tid < 32) {                       // per_block <= 32
        const int pr = blockIdx.x * per_block + tid;
        const bool f = tid < per_block && pr < npairs && clen[pr] == Q;
        const unsigned m = __ballot_sync(0xffffffffu, f);
        if (f) full[__popc(m & ((1u << tid) - 1u))] = pr;
        if (tid == 0) nfull = __popc(m);
    }
    __syncthreads();
    constexpr int V = 16 / (int)sizeof(T);                 // elements per 16-byte copy
    const int tile_elems = 32 * (P + N);
    auto fold_one = [&](int64_t sh) {
        const int s = (int)(sh / H), h = (int)(sh % H), g = h / (H / G);
        const T* xrow = cx + sh * Q * P;
        const T* brow = cB + ((int64_t)s * G + g) * Q * N;
        auto fetch = [&](int t) {                           // raw rows of tile t into buffer t & 1
            T* dst = raw + (t & 1) * tile_elems;
            for (int i = tid; i < 32 * P / V; i += kThreads) cp_async16(dst + i * V, xrow + (int64_t)t * 32 * P + i * V);
            for (int i = tid; i < 32 * N / V; i += kThreads)
                cp_async16(dst + 32 * P + i * V, brow + (int64_t)t * 32 * N + i * V);
            cp_async_commit();
        };
        fetch(0);
        const float last = cacum[sh * Q + Q - 1];
        for (int sidx = tid; sidx < Q; sidx += kThreads)
            wv[sidx] = src_weight(last, cacum[sh * Q + sidx], cdt[sh * Q + sidx]);
        StateTile<NOUT> tile(tid, N);
        const int ntile = Q / 32;
        for (int t = 0; t < ntile; ++t) {
            if (t + 1 < ntile) {
                fetch(t + 1);
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            __syncthreads();                                // tile t landed (all threads' copies); wv
            const T* rx = raw + (t & 1) * tile_elems;
            const T* rb = rx + 32 * P;
            tile_to_f32(xs, rx, 32 * P, P, wv + 32 * t, tid);
            tile_to_f32(bs, rb, 32 * N, N, static_cast<const float*>(nullptr), tid);
            __syncthreads();
            for (int r = 0; r < 32; ++r) tile.row(xs + r * P, bs + r * N);
            __syncthreads();                                // xs, bs and buffer t & 1 free again
        }
        float* hout = cstate + sh * P * N;
#pragma unroll
        for (int i = 0; i < StateTile<NOUT>::R; ++i)
#pragma unroll
            for (int j = 0; j < StateTile<NOUT>::CN; ++j) {
                const int64_t o = (int64_t)(tile.p0 + i) * N + tile.n0 + j;
                hout[o] = pass(hout[o], last, tile.at(i, j));
            }
        if (tid == 0) clen[sh] = 0;
    };
    for (int f = 0; f < nfull; ++f) fold_one(full[f]);
}

template <typename T>
inline size_t fold_smem(int P, int N, int Q) {
    return sizeof(float) * (Q + 32 * P + 32 * N) + sizeof(T) * 2 * 32 * (P + N);
}

}  // namespace strict
}  // namespace ssd
