/*
 * libssd: the Mamba-2 SSD selective scan (chunked prefill) and its per-token decode
 * step, for NVIDIA B200 (sm_100a).
 *
 * The operation. For every sequence and head h (group g = h / (H/G), heads share B
 * and C within a group, as keys/values are shared in grouped-query attention: JAX
 * Nemotron 3 Nano page, NemotronConfig `mamba_ngroups`), token by token:
 *
 *     dt_t   = softplus(dt_raw[t,h] + dt_bias[h])          RL-Kernel issue page, Figure 2
 *     h_t    = exp(dt_t * A[h]) * h_{t-1} + dt_t * x_t B_t^T      (FP32 state, ibid. §1)
 *     y_t[p] = sum_n C_t[n] * h_t[p][n] + D[h] * x_t[p]           (D skip: JAX page,
 *                                                                  "Key Components")
 *
 * starting from the caller's initial state (or zero). Prefill evaluates this with
 * the chunked SSD algorithm, whose memory stays bounded by the chunk size (JAX page,
 * "Key Components" 1; RL-Kernel issue page, Figure 2, the chunked SSD scan box),
 * decode with the per-token recurrent update (RL-Kernel issue page, §1 and §2: the
 * conv-state update followed by the selective state update). The state is stored
 * [P][N] with N contiguous (the transpose of B x^T).
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library never
 *     frees or retains them. Layouts are row-major and contiguous:
 *         x, y        [T, H, P]           (dtype: float32 or bf16)
 *         B, C        [T, G, N]           (same dtype as x)
 *         dt_raw      [T, H]              float32
 *         dt_bias, A, D [H]               float32 (A must be <= 0 and finite)
 *         states      [nseq, H, P, N]     float32
 *     where T is the number of tokens in the call (dense: batch*seqlen).
 *   - Work is enqueued on `stream` and the call returns without waiting for it.
 *     Errors found on the host are returned at once; errors found by a kernel
 *     (bad cu_seqlens, A > 0, a bounded wait that ran out) are latched in a device
 *     error word that ssd_get_device_status() reads and clears.
 *   - Fail closed: geometry outside the supported set returns SSD_ERR_UNSUPPORTED
 *     and nothing is launched; there is no CPU or other fallback (RL-Kernel issue
 *     page, §4.1 and §7: unsupported geometry is refused rather than approximated).
 *   - Functions are thread-safe; ssd_last_error() is per host thread.
 */
#ifndef SSD_H
#define SSD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* ssd_stream_t;

typedef enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, negative size, inconsistent dims */
    SSD_ERR_UNSUPPORTED = 2,   /* valid but outside the supported geometry (fail closed) */
    SSD_ERR_CUDA = 3,          /* a CUDA runtime call failed (message in ssd_last_error) */
    SSD_ERR_TIMEOUT = 4        /* a device-side bounded wait expired */
} ssd_status;

typedef enum {
    SSD_DTYPE_F32 = 0,         /* x, B, C, y are float32 */
    SSD_DTYPE_BF16 = 1         /* x, B, C, y are bf16; dt, A, D and states stay float32 */
} ssd_dtype;

/*
 * Problem description.
 *   Dense mode (cu_seqlens == NULL): nseq = batch sequences of seqlen tokens each,
 *     T = batch * seqlen; token t of sequence b is packed row b*seqlen + t.
 *   Packed varlen mode (cu_seqlens != NULL): nseq sequences, T = total_tokens, which
 *     must equal cu_seqlens[nseq]; sequence s owns rows [cu_seqlens[s], cu_seqlens[s+1]).
 *     batch and seqlen are ignored.
 *   nheads H, headdim P, ngroups G (H % G == 0), dstate N.
 *   workspace / workspace_bytes: optional device scratch of at least the size
 *     ssd_scan_fwd_workspace_size() reports (256-byte aligned). When workspace is
 *     NULL the call allocates and frees scratch itself with cudaMallocAsync /
 *     cudaFreeAsync on `stream`. The decode step needs no workspace.
 */
typedef struct {
    int64_t batch;
    int64_t seqlen;
    int32_t nseq;
    int64_t total_tokens;
    int32_t nheads;
    int32_t headdim;
    int32_t ngroups;
    int32_t dstate;
    ssd_dtype dtype;
    void* workspace;
    size_t workspace_bytes;
} ssd_dims;

/*
 * Bytes of device scratch ssd_scan_fwd needs for `dims` and `chunk`, written to
 * *bytes. Returns SSD_OK, or the status ssd_scan_fwd would return for these dims.
 */
ssd_status ssd_scan_fwd_workspace_size(const ssd_dims* dims, int chunk, size_t* bytes);

/*
 * Chunked SSD prefill (the operation above) over every sequence of the call.
 *   x, dt_raw, dt_bias, A, B, C, D: inputs (layouts above).
 *   init_state: [nseq,H,P,N] float32, or NULL for zero initial states.
 *   cu_seqlens: [nseq+1] int32 device array, or NULL for dense mode. Chunks are
 *     anchored at each sequence start and the state never crosses a sequence
 *     boundary (RL-Kernel issue page, §7: chunks start where sequences start; §8 Q4:
 *     chunking follows cu_seqlens); a sequence's last chunk may be partial.
 *   y: [T,H,P] output, same dtype as x (bf16 rounded to nearest even).
 *   final_state: [nseq,H,P,N] float32 output (the state after each sequence's last
 *     token; the initial state for an empty sequence), or NULL.
 *   chunk: 64, 128 or 256 tokens per chunk. The result does not depend on it
 *     beyond rounding.
 * Supported: P and N in {16, 32, 64, 128}; x/B/C/y 16-byte aligned; other arrays
 * 4-byte aligned. x, B, C and y must not overlap each other or the states.
 */
ssd_status ssd_scan_fwd(const void* x, const float* dt_raw, const float* dt_bias, const float* A,
                        const void* B, const void* C, const float* D, const float* init_state,
                        const int32_t* cu_seqlens, void* y, float* final_state,
                        const ssd_dims* dims, int chunk, ssd_stream_t stream);

/*
 * ssd_scan_fwd that also returns the state at fixed token intervals of every
 * sequence: state snapshots for prefix-cache reuse and chunked prefill (RL-Kernel
 * issue page: §1 names Mamba prefix-cache reuse as a serving feature, §7 and §8 Q4
 * tie it to sequence-anchored chunk boundaries). Snapshot k (k = 1, 2, ...) of a sequence is its state after its first
 * k * snapshot_tokens tokens, for every k with k * snapshot_tokens <= its length
 * (the last one equals final_state when the length is a multiple).
 *   snapshots: [n_snap,H,P,N] float32 output, 16-byte aligned, where n_snap is the
 *     sum over sequences of floor(length / snapshot_tokens) (ssd_snapshot_count),
 *     ordered by sequence, then by k.
 *   snapshot_tokens: > 0; a multiple of 128 on the tensor-core pipeline (which then
 *     uses segments that divide it), a multiple of `chunk` on the CUDA-core pipeline;
 *     otherwise SSD_ERR_UNSUPPORTED.
 *   dims->workspace, if given, must hold ssd_scan_fwd_snapshots_workspace_size bytes.
 * Everything else is as in ssd_scan_fwd; y and final_state are the same.
 */
ssd_status ssd_scan_fwd_snapshots(const void* x, const float* dt_raw, const float* dt_bias, const float* A,
                                  const void* B, const void* C, const float* D, const float* init_state,
                                  const int32_t* cu_seqlens, void* y, float* final_state, float* snapshots,
                                  int64_t snapshot_tokens, const ssd_dims* dims, int chunk,
                                  ssd_stream_t stream);

/* Workspace bytes for ssd_scan_fwd_snapshots (as ssd_scan_fwd_workspace_size). */
ssd_status ssd_scan_fwd_snapshots_workspace_size(const ssd_dims* dims, int chunk, int64_t snapshot_tokens,
                                                 size_t* bytes);

/*
 * Number of snapshots ssd_scan_fwd_snapshots writes, into *count. cu_seqlens_host is
 * a HOST copy of cu_seqlens ([dims->nseq + 1]) for a varlen call, or NULL for a
 * dense call (dims->batch sequences of dims->seqlen tokens).
 */
ssd_status ssd_snapshot_count(const ssd_dims* dims, const int32_t* cu_seqlens_host, int64_t snapshot_tokens,
                              int64_t* count);

/*
 * One decode step for nseq = dims->batch sequences (dims->seqlen must be 1; varlen
 * fields are ignored): per sequence and head, dt = softplus(dt_raw + dt_bias),
 * state <- exp(dt*A) * state + dt * x B^T in place, y = state . C + D * x.
 *   state: [nseq,H,P,N] float32, read and overwritten.
 *   x [nseq,H,P], B/C [nseq,G,N] (dims->dtype), dt_raw [nseq,H] float32.
 *   y: [nseq,H,P] output, dims->dtype.
 * Same support set as ssd_scan_fwd; no workspace.
 */
ssd_status ssd_state_update(float* state, const void* x, const float* dt_raw, const float* dt_bias,
                            const float* A, const void* B, const void* C, const float* D, void* y,
                            const ssd_dims* dims, ssd_stream_t stream);

/*
 * Causal depthwise conv1d + bias + SiLU over the xBC channels, the stage that feeds the
 * scan in a Mamba-2 block (RL-Kernel issue page, Figure 2, and §1 item 2: a conv state
 * per sequence; width 4 in the JAX Nemotron 3 Nano page's configuration). With
 * D = H*P + 2*G*N channels, width K and each sequence's previous K-1 inputs in front of
 * its first token (conv_state_in, or zeros):
 *   out[t][c] = silu(bias[c] + sum_{k<K} weight[c][k] * in[t-(K-1)+k][c]),
 * written split into the scan's inputs: channels [0,H*P) -> x [T,H,P], [H*P,H*P+G*N)
 * -> B [T,G,N], the rest -> C [T,G,N].
 *   xbc: [T,D] (dims->dtype), packed like the scan's inputs (dense batch or cu_seqlens).
 *   weight: [D,K] float32; bias: [D] float32 or NULL (both 16-byte aligned).
 *   conv_state_in: [nseq,D,K-1] (dims->dtype, oldest input first) or NULL for zeros.
 *   conv_state_out: [nseq,D,K-1] output or NULL: each sequence's last K-1 inputs
 *     (taken from conv_state_in where the sequence is shorter than K-1).
 *   width: K in {2,3,4}. The convolution never crosses a sequence boundary.
 * Supported: the scan's head/group geometry; xbc/x/B/C 16-byte aligned. The states may
 * not overlap each other or xbc.
 */
ssd_status ssd_conv1d_fwd(const void* xbc, const float* weight, const float* bias, const void* conv_state_in,
                          const int32_t* cu_seqlens, void* x, void* B, void* C, void* conv_state_out,
                          const ssd_dims* dims, int width, ssd_stream_t stream);

/*
 * One decode step of the conv1d above for nseq = dims->batch sequences (seqlen 1):
 * conv_state [nseq,D,K-1] (16-byte aligned) is read and shifted in place (the new
 * input appended), xbc [nseq,D] in, x [nseq,H,P], B/C [nseq,G,N] out (dims->dtype).
 * A step gives the same bits as ssd_conv1d_fwd on one token from the same state.
 */
ssd_status ssd_conv1d_update(void* conv_state, const void* xbc, const float* weight, const float* bias, void* x,
                             void* B, void* C, const ssd_dims* dims, int width, ssd_stream_t stream);

/*
 * Gated group RMSNorm, the stage after the scan in a Mamba-2 block (RL-Kernel issue page,
 * Figure 2: y gated by SiLU of the z branch, normalised over groups of 512 channels; the
 * JAX Nemotron 3 Nano page's configuration gives the RMSNorm epsilon, 1e-6). Per token t
 * and channel c of its group:
 *   g = y[t][c] * silu(z[t][c]);  out[t][c] = g * rsqrt(mean over the group of g^2 + eps) * weight[c]
 * in FP32, rounded to `dtype`.
 *   y, z, out: [ntok, channels] (dtype; y is the scan's output viewed as [T, H*P]).
 *   weight: [channels] float32. All four 16-byte aligned; out may alias y.
 *   group_size: 256, 512 or 1024, dividing channels; eps >= 0.
 */
ssd_status ssd_gated_rmsnorm(const void* y, const void* z, const float* weight, void* out, int64_t ntok,
                             int channels, int group_size, float eps, ssd_dtype dtype, ssd_stream_t stream);

/*
 * ssd_scan_fwd without any device allocation (the pages have no counterpart; this is a
 * deployment convenience). Some callers cannot allocate device memory while they run:
 * serving engines that reserve their whole memory budget at start-up and forbid later
 * allocations, and latency-critical loops where a cudaMalloc/cudaFree (or a caching
 * allocator's slow path) mid-step is unacceptable. This variant computes exactly what
 * ssd_scan_fwd computes, with the same arguments, but takes its scratch from a 32 MiB
 * array compiled into the library instead of dims->workspace (which must be NULL) or
 * cudaMallocAsync. It calls no cudaMalloc, cudaFree or other allocating routine.
 *   - Size limit: if the problem needs more scratch than 32 MiB (see
 *     ssd_scan_fwd_workspace_size) it returns SSD_ERR_UNSUPPORTED and launches nothing.
 *     Of the named workloads the tiny, batched (4 x 4096) and long-context (1 x 65536)
 *     prefills fit; the 16-sequence packed prefill (about 48 MiB: a segment state per
 *     sequence and segment) is refused.
 *   - Every GPU that loads the library holds those 32 MiB until the process exits.
 *   - Each call made outside stream capture looks up the array's device address (with
 *     the device current); a call during capture reuses the device's last lookup, so
 *     make the first call on each device before any stream capture (a first call during
 *     capture returns SSD_ERR_UNSUPPORTED).
 *   - All calls share the one array and it keeps the last call's contents: calls whose
 *     work can overlap on the GPU (different streams, or different host threads on one
 *     device) race on it and must be serialised by the caller. Nothing in it needs
 *     clearing between calls: every slot a kernel reads is written earlier in the call.
 */
ssd_status ssd_scan_fwd_noalloc(const void* x, const float* dt_raw, const float* dt_bias, const float* A,
                                const void* B, const void* C, const float* D, const float* init_state,
                                const int32_t* cu_seqlens, void* y, float* final_state,
                                const ssd_dims* dims, int chunk, ssd_stream_t stream);

/*
 * Strict mode: bitwise split invariance (RL-Kernel issue page, §4.1: a token's output is
 * bitwise the same whether it came from a full-sequence pass, a prefill of any length or a
 * decode at any step after any chunk-aligned prefill split; §7: prefill and decode share
 * device functions, the decode emulates the chunked arithmetic, and strict mode fails
 * closed where chunks cannot stay sequence-anchored).
 *
 * Both entry points below evaluate the chunked algorithm (chunks of `chunk` tokens
 * anchored at each sequence start) with one set of FP32 device functions, every sum and
 * dot product taken left to right over its index and every operation correctly rounded
 * (no contraction, no reassociation):
 *   dt_s = softplus(dt_raw_s + dt_bias);  Acum_s = Acum_{s-1} + dt_s A  (in-chunk, from 0)
 *   y_t  = D x_t + exp(Acum_t) (C_t . h_in) + sum_{s<=t} (C_t . B_s) exp(Acum_t - Acum_s) dt_s x_s
 *   h_in(next chunk) = exp(Acum_last) h_in + sum_s exp(Acum_last - Acum_s) dt_s x_s B_s^T
 * The decode keeps each sequence's open (partial) chunk in a chunk cache and computes a
 * new token's y as the prefill computes that chunk position; when the chunk fills, it
 * folds the chunk into the cached state as the prefill does. So for any split of a
 * sequence into a strict prefill followed by strict decode steps, or into strict prefills
 * at chunk boundaries, every y and every cached state is bit-identical to a single strict
 * prefill over the whole sequence, and no result depends on batch size or position.
 * Strict results agree with ssd_scan_fwd to within rounding but not bitwise.
 *
 * The chunk cache, per sequence (Q = chunk; all arrays device memory owned by the caller):
 *   state [nseq,H,P,N] float32: the state entering the sequence's open chunk (16-byte aligned)
 *   x     [nseq,H,Q,P] dtype:   x of the open chunk's tokens, rows 0..len-1 (16-byte aligned)
 *   B     [nseq,G,Q,N] dtype:   B of the open chunk's tokens (16-byte aligned)
 *   dt    [nseq,H,Q]   float32: their dt;  acum [nseq,H,Q] float32: their Acum
 *   len   [nseq,H]     int32:   tokens in the open chunk, 0..Q-1 (equal across a sequence's heads)
 * Rows at or past len are never read. Only these entry points should write a cache.
 */
typedef struct {
    float* state;
    void* x;
    void* B;
    float* dt;
    float* acum;
    int32_t* len;
} ssd_chunk_cache;

/* Workspace bytes for ssd_strict_scan_fwd (as ssd_scan_fwd_workspace_size). */
ssd_status ssd_strict_scan_fwd_workspace_size(const ssd_dims* dims, int chunk, size_t* bytes);

/*
 * Strict chunked prefill. Arguments as ssd_scan_fwd, except:
 *   cache: required; written on return with each sequence's open chunk (the tokens of a
 *     partial last chunk, len = length mod chunk) and the state entering it.
 *   resume: 0 starts every sequence from a zero state; 1 starts from cache->state, which
 *     must have an empty open chunk (len == 0 for every sequence and head: the previous
 *     strict call ended on a chunk boundary). Otherwise the kernel latches
 *     SSD_ERR_UNSUPPORTED (fail closed) and the results are not valid.
 *   final_state: optional, the state after each sequence's last token.
 * Supported: fp32 or bf16 x/B/C, P and N in {16, 32, 64, 128}, chunk in {64, 128, 256};
 * the CUDA-core kernels are used for every geometry (no tensor cores: their summation
 * order is not the decode's).
 */
ssd_status ssd_strict_scan_fwd(const void* x, const float* dt_raw, const float* dt_bias, const float* A,
                               const void* B, const void* C, const float* D, const int32_t* cu_seqlens,
                               void* y, float* final_state, const ssd_chunk_cache* cache, int resume,
                               const ssd_dims* dims, int chunk, ssd_stream_t stream);

/*
 * Chunk-emulating decode step for nseq = dims->batch sequences (dims->seqlen must be 1),
 * continuing the caches that ssd_strict_scan_fwd or earlier steps wrote with the same
 * dims and chunk. Per sequence and head the token becomes position len of the open
 * chunk: y is that position's strict prefill output, the token is appended, and when the
 * chunk is full it is folded into cache->state (len back to 0). A len outside [0, chunk)
 * latches SSD_ERR_INVALID_ARG. x [nseq,H,P], B/C [nseq,G,N], dt_raw [nseq,H], y out
 * [nseq,H,P], as ssd_state_update.
 */
ssd_status ssd_strict_state_update(const ssd_chunk_cache* cache, const void* x, const float* dt_raw,
                                   const float* dt_bias, const float* A, const void* B, const void* C,
                                   const float* D, void* y, const ssd_dims* dims, int chunk, ssd_stream_t stream);

/*
 * Waits for `stream`, then reads and clears the device error word: SSD_OK, or the
 * first error a kernel latched since the last read (SSD_ERR_INVALID_ARG for bad
 * cu_seqlens or A > 0, SSD_ERR_TIMEOUT for an expired bounded wait). SSD_ERR_CUDA
 * if the wait itself failed.
 */
ssd_status ssd_get_device_status(ssd_stream_t stream);

/* Message for the last non-OK status returned on this host thread ("" if none). */
const char* ssd_last_error(void);

/*
 * Name of the kernel pipeline ssd_scan_fwd uses for these dims and chunk
 * ("tc": tcgen05 tensor-core kernels; "simt": CUDA-core FP32 kernels), or "" when
 * the dims are rejected.
 */
const char* ssd_scan_fwd_variant(const ssd_dims* dims, int chunk);

/*
 * Tokens per segment of the tensor-core pipeline for these dims (the unit whose
 * state is materialised between its kernels), or 0 for the CUDA-core pipeline or
 * rejected dims.
 */
int ssd_scan_fwd_segment_tokens(const ssd_dims* dims, int chunk);

/*
 * Tuning and testing knob (process-wide): force the tensor-core pipeline's segment
 * length to `tokens` (a multiple of 128, at most 2^20) for every later call; 0 or any
 * other value restores the planner's choice. Results do not depend on it beyond
 * rounding; the workspace size does (query it after setting).
 */
void ssd_set_segment_tokens(int tokens);

/*
 * Test hook for the fail-closed path (RL-Kernel issue page, §4.1 and §7: fail closed),
 * process-wide, for later calls. The tensor-core prefill's warps hand work to each other
 * through shared-memory barriers, and every wait on one is bounded (about 2 s): a wait
 * that runs out latches SSD_ERR_TIMEOUT (read with ssd_get_device_status), the CTA's TMA
 * and UMMA warps issue nothing more and wait (bounded) for the copies and MMAs already in
 * flight, and the CTA exits, so the context stays usable; y and the states of that call
 * are undefined. pass = 1 or 2 makes the UMMA warp of every CTA of the segment-state (1)
 * or chunk-scan (2) pass first wait on a barrier that nothing arrives at, so that this
 * wait runs out (each such call takes a few seconds); 0 (or any other value): off.
 */
void ssd_test_stall(int pass);


/* Number of kernels the last successful call on this host thread enqueued. */
int ssd_last_launch_count(void);

/*
 * Per-kernel timing (tracing). While enabled, every kernel the library enqueues is
 * bracketed by a pair of CUDA events on its stream; ssd_profile_read() waits for
 * the recorded events and reports, per kernel name, the launches and the summed
 * device time since profiling was enabled (or last read). Enabling resets the
 * totals. At most 65536 launches are kept between reads; later ones are counted
 * in `dropped`. Device time only: the events add no host synchronisation.
 */
typedef struct {
    const char* name;      /* kernel name (static string) */
    int launches;
    double total_ms;
} ssd_kernel_time;

void ssd_profile_enable(int on);

/*
 * Diagnostic for the tensor-core path's operand formats: multiplies two 128x128
 * row-major bf16 device matrices X1, X2 five ways on the tcgen05 tensor cores (each
 * with a different pairing of TMA-written / thread-written, K-major / MN-major shared
 * memory operands, or an A operand held in tensor memory) and writes
 * out[5][128][128] float32:
 *   out[0] = X1 X2^T, out[1] = out[3] = out[4] = X1 X2[:, :64], out[2] = X1^T X2[:, :64]
 * (columns >= 64 of out[1..4] are zero). Enqueued on `stream`; no workspace.
 */
ssd_status ssd_selftest_umma(const void* X1, const void* X2, float* out, ssd_stream_t stream);
/* Fills up to `max` entries, returns how many kernel names had launches, or -1 if
 * waiting on an event failed. *dropped (nullable) receives the unrecorded count. */
int ssd_profile_read(ssd_kernel_time* out, int max, int* dropped);

#ifdef __cplusplus
}
#endif

#endif /* SSD_H */
