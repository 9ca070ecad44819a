// Causal depthwise conv1d + bias + SiLU over the xBC channels, with a per-sequence
// conv-state cache: the stage in front of the SSD scan in a Mamba-2 block
// (RL-Kernel issue page, Figure 2, and §1 item 2 on the per-sequence conv cache; the
// JAX Nemotron 3 Nano page's model configuration sets the kernel width to 4).
//
// Channel c of token t of a sequence, with width K and the sequence's previous K-1
// inputs (the conv state; zeros if none) in front of its first token:
//   out[t][c] = silu(bias[c] + sum_{k<K} w[c][k] * in[t - (K-1) + k][c]).
// The outputs are split into the scan's inputs: channels [0, H*P) -> x [T,H,P],
// [H*P, H*P+G*N) -> B [T,G,N], the rest -> C [T,G,N]. The final conv state of a
// sequence is its last K-1 inputs (oldest first), taking them from the incoming state
// when the sequence is shorter than K-1.
//
// HBM-bound: every input is read once and every output written once. A thread owns 8
// consecutive channels (one 16-byte bf16 vector) over a run of tokens and keeps the
// sliding window in registers; the taps run as paired FP32 FMAs (two channels per
// instruction) and SiLU costs one special-function operation per bf16 output.
#pragma once

#include "ssd_common.cuh"
#include "ssd_tc_ptx.cuh"

namespace ssd {

constexpr int kConvTokens = 64;      // tokens per block of the prefill kernel
constexpr int kConvThreads = 256;    // 8 channels each

__device__ __forceinline__ void load8(const float* p, float (&o)[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&o)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = __uint_as_float(w[i] << 16);
        o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// silu(v) = v * sigmoid(v). For float outputs: v * 1 / (1 + 2^(-v log2 e)) with the
// hardware base-2 exponential and reciprocal (a few ulp). For bf16 outputs: sigmoid(v) =
// (1 + tanh(v / 2)) / 2 with the hardware tanh (relative error about 2^-11, below the
// bf16 rounding of the result), one special-function operation instead of two. The
// prefill and decode kernels use the same operations in the same order, paired or not,
// so a decode step and a one-token prefill give the same bits.
__device__ __forceinline__ float conv_ex2(float v) {
    float e;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(v));
    return e;
}
__device__ __forceinline__ float conv_rcp(float v) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}
__device__ __forceinline__ float conv_tanh(float v) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(v));
    return t;
}
constexpr float kNegLog2e = -1.4426950408889634f;

template <typename T>
__device__ __forceinline__ float silu(float v);
template <>
__device__ __forceinline__ float silu<float>(float v) {
    const float e = conv_ex2(__fmul_rn(v, kNegLog2e));
    return __fmul_rn(v, conv_rcp(__fadd_rn(e, 1.f)));
}
template <>
__device__ __forceinline__ float silu<__nv_bfloat16>(float v) {
    const float t = conv_tanh(__fmul_rn(v, 0.5f));
    return __fmul_rn(v, __fmaf_rn(t, 0.5f, 0.5f));
}
// The same for a pair of channels with paired FP32 instructions.
template <typename T>
__device__ __forceinline__ float2 silu2(float2 v);
template <>
__device__ __forceinline__ float2 silu2<float>(float2 v) {
    const float2 a = tc::fmul2(v, make_float2(kNegLog2e, kNegLog2e));
    const float2 d = tc::ffma2(make_float2(conv_ex2(a.x), conv_ex2(a.y)), make_float2(1.f, 1.f),
                               make_float2(1.f, 1.f));
    return tc::fmul2(v, make_float2(conv_rcp(d.x), conv_rcp(d.y)));
}
template <>
__device__ __forceinline__ float2 silu2<__nv_bfloat16>(float2 v) {
    const float2 a = tc::fmul2(v, make_float2(0.5f, 0.5f));
    const float2 sg = tc::ffma2(make_float2(conv_tanh(a.x), conv_tanh(a.y)), make_float2(0.5f, 0.5f),
                                make_float2(0.5f, 0.5f));
    return tc::fmul2(v, sg);
}

// Weights of channels c0..c0+7 of thread `tid` (w [D][K]). A lane's 8 rows are 32*K
// bytes away from its neighbour's, so direct loads would touch one cache line per lane;
// the block first copies its channels' taps to shared memory with coalesced 16-byte
// loads, into rows of 8*K floats padded to 8*K+4 (conflict-free 16-byte reads), then
// every thread reads its own row. cbase = first channel of the block; nch = channels of
// the block that exist.
constexpr int kTapRow(int K) { return 8 * K + 4; }

template <int K>
__device__ __forceinline__ void load_taps(const float* __restrict__ w, int cbase, int nch, float* sw,
                                          float (&wk)[K][8]) {
    const int tid = threadIdx.x;
    const int nvec = nch * K / 4;                // float4s of the block's taps (nch multiple of 8)
    const float4* src = reinterpret_cast<const float4*>(w + (int64_t)cbase * K);
    for (int i = tid; i < nvec; i += kConvThreads) {
        const int f = 4 * i;                     // first float of this vector within the block
        const int row = f / (8 * K), col = f % (8 * K);
        *reinterpret_cast<float4*>(sw + row * kTapRow(K) + col) = __ldg(src + i);
    }
    __syncthreads();
    const float* r = sw + tid * kTapRow(K);
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int k = 0; k < K; ++k) wk[k][j] = r[j * K + k];
}

// Token ring of the prefill kernel. Once the taps are in registers, the tap staging
// buffer holds, per thread, the next R token vectors of its 8 channels (slot k of thread
// tid at element (k * kConvThreads + tid) * 8), filled by 16-byte asynchronous copies
// (cp.async), so R tokens per thread are in flight without holding registers. R is the
// largest power of two (at most 8) whose slots fit the thread's tap row.
template <typename T, int K>
constexpr int conv_ring() {
    constexpr int cap = kTapRow(K) * 4 / (8 * (int)sizeof(T));
    return cap >= 8 ? 8 : (cap >= 4 ? 4 : (cap >= 2 ? 2 : 1));
}

// Destination of channel vector c0 (8 channels) of one token row: x, B or C.
template <typename T>
__device__ __forceinline__ T* conv_dst(int64_t row, int c0, int HP, int GN, T* x, T* B, T* C) {
    if (c0 < HP) return x + row * HP + c0;
    if (c0 < HP + GN) return B + row * GN + (c0 - HP);
    return C + row * GN + (c0 - HP - GN);
}

// Prefill: block (token tile of kConvTokens, channel tile). seq_begin(s) gives packed
// token offsets (cu_seqlens, or s * seqlen for a dense batch).
template <typename T, int K>
__global__ void __launch_bounds__(kConvThreads, 2)
k_conv1d_fwd(const T* __restrict__ in, const float* __restrict__ w, const float* __restrict__ bias,
             const T* __restrict__ st_in, const int32_t* __restrict__ cu, int32_t nseq, int64_t T_,
             int64_t seqlen, int Dc, int HP, int GN, T* __restrict__ x, T* __restrict__ B,
             T* __restrict__ C, T* __restrict__ st_out) {
    __shared__ __align__(16) float sw[kConvThreads * kTapRow(K)];
    const int cbase = blockIdx.y * kConvThreads * 8;
    const int c0 = cbase + threadIdx.x * 8;
    const int64_t t0 = (int64_t)blockIdx.x * kConvTokens;
    float wk[K][8];
    load_taps<K>(w, cbase, min(kConvThreads * 8, Dc - cbase), sw, wk);
    __syncthreads();                             // taps are in registers: sw becomes the token ring
    if (c0 >= Dc || t0 >= T_) return;
    const int64_t t1 = t0 + kConvTokens < T_ ? t0 + kConvTokens : T_;
    T* const dst = conv_dst((int64_t)0, c0, HP, GN, x, B, C);   // row 0 of this thread's output
    const int64_t dstride = c0 < HP ? HP : GN;                   // elements per token row
    auto seq_begin = [&](int s) -> int64_t { return cu ? (int64_t)cu[s] : (int64_t)s * seqlen; };
    // Sequence of token t0: the last s with seq_begin(s) <= t0 and a non-empty range.
    int lo = 0, hi = nseq;                      // invariant: seq_begin(lo) <= t0 < seq_begin(hi)
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (seq_begin(mid) <= t0) lo = mid; else hi = mid;
    }
    int s = lo;
    int64_t sb = seq_begin(s), se = seq_begin(s + 1);
    float bv[8];
    if (bias) load8(bias + c0, bv);
    else
#pragma unroll
        for (int j = 0; j < 8; ++j) bv[j] = 0.f;
    // History of the last K inputs as a circular buffer: the input of token t0 + i sits in
    // hist[i % K], so the input k positions before it is hist[(i - k) % K]. The token loop
    // runs in groups of K with the position in the group a compile-time constant, so every
    // index is fixed and the window slides without register moves.
    float hist[K][8];
    auto state_in = [&](int seq, int k, float (&dst)[8]) {   // input k positions before seq's start
#pragma unroll
        for (int j = 0; j < 8; ++j)
            dst[j] = st_in ? to_f32(st_in[((int64_t)seq * Dc + c0 + j) * (K - 1) + (K - 1 - k)]) : 0.f;
    };
    // Initial window for t0: inputs t0-1 .. t0-K+1, from the sequence, or from its
    // incoming state for positions before the sequence start.
#pragma unroll
    for (int k = 1; k < K; ++k) {
        const int64_t tp = t0 - k;
        if (tp >= sb) load8(in + tp * Dc + c0, hist[(K - k) % K]);
        else state_in(s, (int)(sb - tp), hist[(K - k) % K]);
    }
    constexpr int R = conv_ring<T, K>();
    T* const ring = reinterpret_cast<T*>(sw);
    auto slot = [&](int k) { return ring + ((int64_t)k * kConvThreads + threadIdx.x) * 8; };
    auto issue = [&](int64_t t, int k) {         // token t's 8 channels into slot k
        const char* src = reinterpret_cast<const char*>(in + t * Dc + c0);
        char* d = reinterpret_cast<char*>(slot(k));
#pragma unroll
        for (int q = 0; q < (int)(8 * sizeof(T) / 16); ++q) cp_async16(d + 16 * q, src + 16 * q);
    };
#pragma unroll
    for (int k = 0; k < R; ++k) {                // one commit group per token, in token order
        if (t0 + k < t1) issue(t0 + k, k);
        cp_async_commit();
    }
    for (int64_t tg = t0; tg < t1; tg += K) {
#pragma unroll
        for (int u = 0; u < K; ++u) {
            const int64_t t = tg + u;
            if (t >= t1) break;
            const int kr = (int)(t - t0) & (R - 1);
            cp_async_wait<R - 1>();              // token t's group (the oldest pending) is done
            load8(slot(kr), hist[u]);
            while (t >= se) {                    // next sequence (skipping empty ones)
                ++s;
                sb = seq_begin(s);
                se = seq_begin(s + 1);
#pragma unroll
                for (int k = 1; k < K; ++k) state_in(s, k, hist[(u - k + K) % K]);
            }
            // Output: bias + taps over the inputs t-K+1 .. t, then SiLU; the final conv state
            // (the last K-1 inputs) at a sequence's last token.
            float o[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int j = 2 * i;
                float2 acc = tc::ffma2(make_float2(wk[K - 1][j], wk[K - 1][j + 1]),
                                       make_float2(hist[u][j], hist[u][j + 1]), make_float2(bv[j], bv[j + 1]));
#pragma unroll
                for (int k = 1; k < K; ++k)
                    acc = tc::ffma2(make_float2(wk[K - 1 - k][j], wk[K - 1 - k][j + 1]),
                                    make_float2(hist[(u - k + K) % K][j], hist[(u - k + K) % K][j + 1]), acc);
                const float2 v = silu2<T>(acc);
                o[j] = v.x;
                o[j + 1] = v.y;
            }
            store8(dst + t * dstride, o);
            if (t == se - 1 && st_out) {
#pragma unroll
                for (int k = 1; k < K; ++k)
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        st_out[((int64_t)s * Dc + c0 + j) * (K - 1) + (K - 1 - k)] =
                            from_f32<T>(hist[(u - (k - 1) + K) % K][j]);
            }
            if (t + R < t1) issue(t + R, kr);   // slot kr was consumed above
            cp_async_commit();
        }
    }
}

// Final conv state of empty sequences (no token writes it): the incoming state, or 0.
template <typename T, int K>
__global__ void k_conv1d_empty(const T* __restrict__ st_in, const int32_t* __restrict__ cu, int32_t nseq,
                               int64_t seqlen, int Dc, T* __restrict__ st_out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)nseq * Dc) return;
    const int s = (int)(i / Dc);
    const int64_t len = cu ? (int64_t)cu[s + 1] - cu[s] : seqlen;
    if (len != 0) return;
#pragma unroll
    for (int k = 0; k < K - 1; ++k) st_out[i * (K - 1) + k] = st_in ? st_in[i * (K - 1) + k] : from_f32<T>(0.f);
}

// Decode: one new token per sequence. state [nseq][Dc][K-1] (oldest first) is updated
// in place; out goes to x/B/C rows of the sequence.
constexpr int kConvSeqs = 8;         // sequences per block of the decode kernel

template <typename T, int K>
__global__ void __launch_bounds__(kConvThreads)
k_conv1d_update(T* __restrict__ state, const T* __restrict__ in, const float* __restrict__ w,
                const float* __restrict__ bias, int32_t nseq, int Dc, int HP, int GN, T* __restrict__ x,
                T* __restrict__ B, T* __restrict__ C) {
    __shared__ __align__(16) float sw[kConvThreads * kTapRow(K)];
    const int cbase = blockIdx.x * kConvThreads * 8;
    const int c0 = cbase + threadIdx.x * 8;
    float wk[K][8];
    load_taps<K>(w, cbase, min(kConvThreads * 8, Dc - cbase), sw, wk);
    if (c0 >= Dc) return;
    float bv[8];
    if (bias) load8(bias + c0, bv);
    else
#pragma unroll
        for (int j = 0; j < 8; ++j) bv[j] = 0.f;
    const int s1 = min(nseq, (int)(blockIdx.y + 1) * kConvSeqs);
    for (int s = blockIdx.y * kConvSeqs; s < s1; ++s) {
    float cur[8];
    load8(in + (int64_t)s * Dc + c0, cur);
    // The 8 channels' states are 8*(K-1) consecutive elements: read them as whole vectors.
    constexpr int E = 8 * (K - 1);
    float sv[E];
    T* sp = state + ((int64_t)s * Dc + c0) * (K - 1);
    if constexpr (sizeof(T) == 2 && E % 8 == 0) {
#pragma unroll
        for (int v = 0; v < E / 8; ++v) {
            float t8[8];
            load8(sp + 8 * v, t8);
#pragma unroll
            for (int i = 0; i < 8; ++i) sv[8 * v + i] = t8[i];
        }
    } else {
#pragma unroll
        for (int i = 0; i < E; ++i) sv[i] = to_f32(sp[i]);
    }
    float o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float acc = __fmaf_rn(wk[K - 1][j], cur[j], bv[j]);
        // newest previous input first: the prefill kernel's order, so a decode step and
        // a one-token prefill give the same bits
#pragma unroll
        for (int k = K - 2; k >= 0; --k) acc = __fmaf_rn(wk[k][j], sv[j * (K - 1) + k], acc);
        o[j] = silu<T>(acc);
    }
    store8(conv_dst((int64_t)s, c0, HP, GN, x, B, C), o);
    // shift: drop the oldest input of each channel, append the new one
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
        for (int k = 0; k < K - 2; ++k) sv[j * (K - 1) + k] = sv[j * (K - 1) + k + 1];
        sv[j * (K - 1) + K - 2] = cur[j];
    }
    if constexpr (sizeof(T) == 2 && E % 8 == 0) {
#pragma unroll
        for (int v = 0; v < E / 8; ++v) {
            float t8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) t8[i] = sv[8 * v + i];
            store8(sp + 8 * v, t8);
        }
    } else {
#pragma unroll
        for (int i = 0; i < E; ++i) sp[i] = from_f32<T>(sv[i]);
    }
    }
}

}  // namespace ssd
