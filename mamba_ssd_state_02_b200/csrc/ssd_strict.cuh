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
// __fmaf_rn: never contracted or reordered by the compiler):
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
__device__ __forceinline__ float acum_next(float prev, float dt, float a) {
    return __fadd_rn(prev, __fmul_rn(dt, a));
}
// w(t, s) = exp(Acum_t - Acum_s) dt_s
__device__ __forceinline__ float src_weight(float acum_t, float acum_s, float dt_s) {
    return __fmul_rn(expf(__fsub_rn(acum_t, acum_s)), dt_s);
}
// one step of a left-to-right dot product
__device__ __forceinline__ float dot_step(float acc, float u, float v) { return __fmaf_rn(u, v, acc); }
// coefficient of x_s in y_t: (C_t . B_s) w(t, s)
__device__ __forceinline__ float mix_coef(float cb, float acum_t, float acum_s, float dt_s) {
    return __fmul_rn(cb, src_weight(acum_t, acum_s, dt_s));
}
// y accumulator: start from the incoming-state term, add sources left to right, add D x_t
__device__ __forceinline__ float y_begin(float c_dot_h, float acum_t) { return __fmul_rn(c_dot_h, expf(acum_t)); }
__device__ __forceinline__ float y_step(float acc, float coef, float xs) { return __fmaf_rn(coef, xs, acc); }
__device__ __forceinline__ float y_end(float acc, float Dh, float xt) { return __fmaf_rn(Dh, xt, acc); }
// chunk state: source term w(last, s) x_s[p], accumulated left to right against B_s[n]
__device__ __forceinline__ float state_src(float w, float xs) { return __fmul_rn(w, xs); }
__device__ __forceinline__ float state_step(float acc, float wx, float b) { return __fmaf_rn(wx, b, acc); }
// state passing across a chunk boundary
__device__ __forceinline__ float pass(float h, float acum_last, float S) { return __fmaf_rn(expf(acum_last), h, S); }

__device__ __forceinline__ bool bad_A(float a) { return !(a <= 0.f) || isinf(a); }

constexpr int kThreads = 256;

// ---------------------------------------------------------------------------------
// Prefill stage 1: dt and Acum per (chunk, head), left to right, [chunk][H][Q] (zero past
// the chunk's end). One thread per (chunk, head).
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
    for (int r = 0; r < Q; ++r) {
        float d = 0.f;
        if (r < e.len) {
            d = dt_of(dt_raw[(int64_t)(e.start + r) * H + h], bias);
            run = acum_next(run, d, a);
        }
        dt_out[base + r] = d;
        acum_out[base + r] = run;
    }
}

// ---------------------------------------------------------------------------------
// Prefill stage 2: chunk states S_c[p][n] (zero-start state at the chunk's last token).
// One block per (chunk, head); thread owns column n = tid % N and rows tid / N + k (256 / N).
template <typename T>
__global__ void __launch_bounds__(kThreads)
k_strict_chunk_state(const T* __restrict__ x, const T* __restrict__ B, const float* __restrict__ dtc,
                     const float* __restrict__ acum, const ChunkEntry* __restrict__ table,
                     const int32_t* __restrict__ count, int H, int G, int P, int N, int Q,
                     float* __restrict__ states) {
    extern __shared__ float sm[];
    float* w = sm;                       // [Q]
    float* xs = w + Q;                   // [32][P]   w(last, s) x_s
    float* bs = xs + 32 * P;             // [32][N]
    const int c = blockIdx.x;
    if (c >= *count) return;
    const int h = blockIdx.y, g = h / (H / G), tid = threadIdx.x;
    const ChunkEntry e = table[c];
    const float* ac = acum + ((int64_t)c * H + h) * Q;
    const float* dv = dtc + ((int64_t)c * H + h) * Q;
    const float last = ac[e.len - 1];
    for (int s = tid; s < e.len; s += kThreads) w[s] = src_weight(last, ac[s], dv[s]);
    const int n = tid % N, p0 = tid / N, pstep = kThreads / N;
    const int nout = P * N / kThreads;   // 1..64
    float acc[64];
#pragma unroll
    for (int k = 0; k < 64; ++k) acc[k] = 0.f;
    __syncthreads();
    for (int s0 = 0; s0 < e.len; s0 += 32) {
        const int rows = min(32, e.len - s0);
        for (int i = tid; i < rows * P; i += kThreads) {
            const int r = i / P, pp = i % P;
            const int64_t t = e.start + s0 + r;
            xs[r * P + pp] = state_src(w[s0 + r], to_f32(x[(t * H + h) * P + pp]));
        }
        for (int i = tid; i < rows * N; i += kThreads) {
            const int r = i / N, nn = i % N;
            const int64_t t = e.start + s0 + r;
            bs[r * N + nn] = to_f32(B[(t * G + g) * N + nn]);
        }
        __syncthreads();
        for (int r = 0; r < rows; ++r) {
            const float bv = bs[r * N + n];
#pragma unroll
            for (int k = 0; k < 64; ++k)
                if (k < nout) acc[k] = state_step(acc[k], xs[r * P + p0 + k * pstep], bv);
        }
        __syncthreads();
    }
    float* out = states + ((int64_t)c * H + h) * P * N;
#pragma unroll
    for (int k = 0; k < 64; ++k)
        if (k < nout) out[(p0 + k * pstep) * N + n] = acc[k];
}

// ---------------------------------------------------------------------------------
// Prefill stage 3: state passing, sequential over a sequence's chunks, parallel over
// (head, state element). Overwrites S_c with h_in(c), writes the final state and the
// cache state (the state entering the sequence's open chunk: h_in of a partial last
// chunk, else the final state). `resume`: start from cache_state, whose open chunk
// must be empty (cache_len == 0), else SSD_ERR_UNSUPPORTED is latched (fail closed).
__global__ void __launch_bounds__(kThreads)
k_strict_passing(float* __restrict__ states, const float* __restrict__ acum, const ChunkEntry* __restrict__ table,
                 const int32_t* __restrict__ first, int resume, float* __restrict__ cache_state,
                 const int32_t* __restrict__ cache_len, float* __restrict__ final_state, int H, int PN, int Q) {
    const int s = blockIdx.x, h = blockIdx.y;
    const int i = blockIdx.z * kThreads + threadIdx.x;
    if (i >= PN) return;
    const int64_t slot0 = ((int64_t)s * H + h) * PN + i;
    float hv = 0.f;
    if (resume) {
        if (cache_len[(int64_t)s * H + h] != 0) latch_error(SSD_ERR_UNSUPPORTED);
        hv = cache_state[slot0];
    }
    const int c0 = first[s], c1 = first[s + 1];
    float open = hv;
    for (int c = c0; c < c1; ++c) {
        const ChunkEntry e = table[c];
        float* slot = states + ((int64_t)c * H + h) * PN + i;
        const float sv = *slot;
        *slot = hv;
        open = hv;
        hv = pass(hv, acum[((int64_t)c * H + h) * Q + e.len - 1], sv);
        if (e.len == Q) open = hv;
    }
    cache_state[slot0] = open;
    if (final_state) final_state[slot0] = hv;
}

// ---------------------------------------------------------------------------------
// Prefill stage 4: y for 32 rows of one (chunk, head). Thread owns column p = tid % P and
// rows tid / P + k (256 / P).
template <typename T>
__global__ void __launch_bounds__(kThreads)
k_strict_chunk_scan(const T* __restrict__ x, const T* __restrict__ B, const T* __restrict__ C,
                    const float* __restrict__ D, const float* __restrict__ dtc, const float* __restrict__ acum,
                    const float* __restrict__ hin, const ChunkEntry* __restrict__ table,
                    const int32_t* __restrict__ count, int H, int G, int P, int N, int Q, T* __restrict__ y) {
    extern __shared__ float sm[];
    const int NP = N + 1;
    float* acs = sm;                      // [Q]
    float* dts = acs + Q;                 // [Q]
    float* cs = dts + Q;                  // [32][N+1]
    float* bs = cs + 32 * NP;             // [32][N+1]
    float* xs = bs + 32 * NP;             // [32][P]
    float* ms = xs + 32 * P;              // [32][33]
    float* hs = ms + 32 * 33;             // [P][33]
    const int c = blockIdx.x;
    if (c >= *count) return;
    const ChunkEntry e = table[c];
    const int t0 = blockIdx.z * 32;
    if (t0 >= e.len) return;
    const int h = blockIdx.y, g = h / (H / G), tid = threadIdx.x;
    const int64_t cbase = ((int64_t)c * H + h) * Q;
    for (int i = tid; i < Q; i += kThreads) {
        acs[i] = acum[cbase + i];
        dts[i] = dtc[cbase + i];
    }
    const int rows = min(32, e.len - t0);
    for (int i = tid; i < 32 * N; i += kThreads) {
        const int r = i / N, nn = i % N;
        cs[r * NP + nn] = r < rows ? to_f32(C[((int64_t)(e.start + t0 + r) * G + g) * N + nn]) : 0.f;
    }
    const int p = tid % P, r0 = tid / P, tstep = kThreads / P;
    const int nout = 32 * P / kThreads;   // 2..16
    float acc[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) acc[k] = 0.f;
    __syncthreads();

    // (1) C_t . h_in[p], left to right over n (in slices of 32 columns).
    const float* hp = hin + ((int64_t)c * H + h) * P * N;
    for (int n0 = 0; n0 < N; n0 += 32) {
        const int cols = min(32, N - n0);
        for (int i = tid; i < P * 32; i += kThreads) {
            const int pp = i / 32, j = i % 32;
            hs[pp * 33 + j] = j < cols ? hp[pp * N + n0 + j] : 0.f;
        }
        __syncthreads();
        for (int j = 0; j < cols; ++j) {
            const float hv = hs[p * 33 + j];
#pragma unroll
            for (int k = 0; k < 16; ++k)
                if (k < nout) acc[k] = dot_step(acc[k], cs[(r0 + k * tstep) * NP + n0 + j], hv);
        }
        __syncthreads();
    }
#pragma unroll
    for (int k = 0; k < 16; ++k)
        if (k < nout) acc[k] = y_begin(acc[k], acs[min(t0 + r0 + k * tstep, Q - 1)]);

    // (2) sources s = 0..t, left to right, in 32-token slices.
    for (int s0 = 0; s0 <= t0; s0 += 32) {
        const int srows = min(32, e.len - s0);
        for (int i = tid; i < 32 * N; i += kThreads) {
            const int r = i / N, nn = i % N;
            bs[r * NP + nn] = r < srows ? to_f32(B[((int64_t)(e.start + s0 + r) * G + g) * N + nn]) : 0.f;
        }
        for (int i = tid; i < 32 * P; i += kThreads) {
            const int r = i / P, pp = i % P;
            xs[r * P + pp] = r < srows ? to_f32(x[((int64_t)(e.start + s0 + r) * H + h) * P + pp]) : 0.f;
        }
        __syncthreads();
        for (int q = tid; q < 32 * 32; q += kThreads) {
            const int tt = q >> 5, ss = q & 31;
            const int ta = t0 + tt, sa = s0 + ss;
            float v = 0.f;
            if (sa <= ta && ss < srows && tt < rows) {
                float dot = 0.f;
                for (int nn = 0; nn < N; ++nn) dot = dot_step(dot, cs[tt * NP + nn], bs[ss * NP + nn]);
                v = mix_coef(dot, acs[ta], acs[sa], dts[sa]);
            }
            ms[tt * 33 + ss] = v;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            if (k >= nout) break;
            const int tt = r0 + k * tstep;
            const int smax = min(min(31, t0 + tt - s0), srows - 1);
            for (int ss = 0; ss <= smax; ++ss) acc[k] = y_step(acc[k], ms[tt * 33 + ss], xs[ss * P + p]);
        }
        __syncthreads();
    }

    // (3) D skip and store.
    const float Dh = D[h];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        if (k >= nout) break;
        const int tt = r0 + k * tstep;
        if (tt < rows) {
            const int64_t o = ((int64_t)(e.start + t0 + tt) * H + h) * P + p;
            y[o] = from_f32<T>(y_end(acc[k], Dh, to_f32(x[o])));
        }
    }
}

inline size_t chunk_scan_smem(int P, int N, int Q) {
    return sizeof(float) * (2 * Q + 2 * 32 * (N + 1) + 32 * P + 32 * 33 + P * 33);
}
inline size_t chunk_state_smem(int P, int N, int Q) { return sizeof(float) * (Q + 32 * P + 32 * N); }

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
// Chunk-emulating decode step. One block per (sequence, head). With j = the open chunk's
// length, the new token is position j of the open chunk:
//   y   = the prefill's y_t for t = j over sources 0..j (cached 0..j-1, the new token j),
//   the new token is appended to the cache, and when j = Q-1 the full chunk is folded into
//   the cache state with the prefill's chunk-state and passing arithmetic (length -> 0).
// Shared memory: C_t [N], coefficients [Q], and for the fold w(last,s) x_s [32][P] and
// B_s [32][N] slices.
template <typename T>
__global__ void __launch_bounds__(kThreads)
k_strict_decode(float* __restrict__ cstate, T* __restrict__ cx, T* __restrict__ cB, float* __restrict__ cdt,
                float* __restrict__ cacum, int32_t* __restrict__ clen, const T* __restrict__ x,
                const float* __restrict__ dt_raw, const float* __restrict__ dt_bias, const float* __restrict__ A,
                const T* __restrict__ B, const T* __restrict__ C, const float* __restrict__ D, T* __restrict__ y,
                int H, int G, int P, int N, int Q) {
    extern __shared__ float sm[];
    float* cs = sm;                       // [N]
    float* coef = cs + N;                 // [Q]
    float* wv = coef + Q;                 // [Q]  w(last, s) for the fold
    float* xs = wv + Q;                   // [32][P]
    float* bs = xs + 32 * P;              // [32][N]
    __shared__ float s_dt, s_acum;
    const int bid = blockIdx.x;
    const int s = bid / H, h = bid % H, g = h / (H / G), tid = threadIdx.x;
    const int64_t sh = (int64_t)s * H + h;
    const int j = clen[sh];
    if (j < 0 || j >= Q) {                 // not a cache this step can continue
        if (tid == 0) latch_error(SSD_ERR_INVALID_ARG);
        return;
    }
    const float a = A[h];
    if (tid == 0) {
        if (bad_A(a)) latch_error(SSD_ERR_INVALID_ARG);
        const float d = dt_of(dt_raw[sh], dt_bias[h]);
        s_dt = d;
        s_acum = acum_next(j > 0 ? cacum[sh * Q + j - 1] : 0.f, d, a);
    }
    const T* xt = x + sh * P;
    const T* Bt = B + ((int64_t)s * G + g) * N;
    const T* Ct = C + ((int64_t)s * G + g) * N;
    const T* xrow = cx + sh * Q * P;                       // cached x rows [Q][P]
    const T* brow = cB + ((int64_t)s * G + g) * Q * N;     // cached B rows [Q][N]
    for (int n = tid; n < N; n += kThreads) cs[n] = to_f32(Ct[n]);
    __syncthreads();
    const float dtj = s_dt, acj = s_acum;

    // Coefficients of sources 0..j: (C_t . B_s) w(j, s).
    for (int sidx = tid; sidx <= j; sidx += kThreads) {
        const T* bsrc = sidx < j ? brow + (int64_t)sidx * N : Bt;
        float dot = 0.f;
        for (int n = 0; n < N; ++n) dot = dot_step(dot, cs[n], to_f32(bsrc[n]));
        const float acs = sidx < j ? cacum[sh * Q + sidx] : acj;
        const float dts = sidx < j ? cdt[sh * Q + sidx] : dtj;
        coef[sidx] = mix_coef(dot, acj, acs, dts);
    }
    __syncthreads();

    // y[p]: incoming-state term, sources left to right, D skip.
    const float* hrow = cstate + sh * P * N;
    for (int p = tid; p < P; p += kThreads) {
        float dot = 0.f;
        const float* hp = hrow + (int64_t)p * N;
        for (int n = 0; n < N; n += 4) {
            const float4 v = *reinterpret_cast<const float4*>(hp + n);
            dot = dot_step(dot, cs[n], v.x);
            dot = dot_step(dot, cs[n + 1], v.y);
            dot = dot_step(dot, cs[n + 2], v.z);
            dot = dot_step(dot, cs[n + 3], v.w);
        }
        float acc = y_begin(dot, acj);
        for (int sidx = 0; sidx < j; ++sidx) acc = y_step(acc, coef[sidx], to_f32(xrow[(int64_t)sidx * P + p]));
        const float xv = to_f32(xt[p]);
        acc = y_step(acc, coef[j], xv);
        y[sh * P + p] = from_f32<T>(y_end(acc, D[h], xv));
    }

    // Append the token to the open chunk.
    T* xdst = cx + (sh * Q + j) * P;
    for (int p = tid; p < P; p += kThreads) xdst[p] = xt[p];
    if (h % (H / G) == 0) {
        T* bdst = cB + (((int64_t)s * G + g) * Q + j) * N;
        for (int n = tid; n < N; n += kThreads) bdst[n] = Bt[n];
    }
    if (tid == 0) {
        cdt[sh * Q + j] = dtj;
        cacum[sh * Q + j] = acj;
    }
    if (j + 1 < Q) {
        if (tid == 0) clen[sh] = j + 1;
        return;
    }

    // The chunk is full: fold it into the cache state (the prefill's chunk-state and
    // passing arithmetic, sources left to right), then empty the open chunk.
    for (int sidx = tid; sidx < Q; sidx += kThreads) {
        const float acs = sidx < j ? cacum[sh * Q + sidx] : acj;
        const float dts = sidx < j ? cdt[sh * Q + sidx] : dtj;
        wv[sidx] = src_weight(acj, acs, dts);
    }
    const int n = tid % N, p0 = tid / N, pstep = kThreads / N;
    const int nout = P * N / kThreads;
    float acc[64];
#pragma unroll
    for (int k = 0; k < 64; ++k) acc[k] = 0.f;
    __syncthreads();
    for (int s0 = 0; s0 < Q; s0 += 32) {
        for (int i = tid; i < 32 * P; i += kThreads) {
            const int r = i / P, pp = i % P, sidx = s0 + r;
            const float xv = sidx < j ? to_f32(xrow[(int64_t)sidx * P + pp]) : to_f32(xt[pp]);
            xs[r * P + pp] = state_src(wv[sidx], xv);
        }
        for (int i = tid; i < 32 * N; i += kThreads) {
            const int r = i / N, nn = i % N, sidx = s0 + r;
            bs[r * N + nn] = sidx < j ? to_f32(brow[(int64_t)sidx * N + nn]) : to_f32(Bt[nn]);
        }
        __syncthreads();
        for (int r = 0; r < 32; ++r) {
            const float bv = bs[r * N + n];
#pragma unroll
            for (int k = 0; k < 64; ++k)
                if (k < nout) acc[k] = state_step(acc[k], xs[r * P + p0 + k * pstep], bv);
        }
        __syncthreads();
    }
    float* hout = cstate + sh * P * N;
#pragma unroll
    for (int k = 0; k < 64; ++k)
        if (k < nout) {
            const int64_t o = (int64_t)(p0 + k * pstep) * N + n;
            hout[o] = pass(hout[o], acj, acc[k]);
        }
    if (tid == 0) clen[sh] = 0;
}

inline size_t decode_smem(int P, int N, int Q) { return sizeof(float) * (N + 2 * Q + 32 * P + 32 * N); }

}  // namespace strict
}  // namespace ssd
