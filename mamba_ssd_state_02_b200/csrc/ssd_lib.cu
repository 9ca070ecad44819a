// libssd C ABI: argument validation (fail closed), workspace planning and kernel
// dispatch for the chunked SSD prefill and the decode step. All kernels of the
// library live in this translation unit (the .cuh files), so they share the device
// error word without relocatable device code.
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdarg>
#include <cstdio>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <cstdlib>

#include "ssd.h"
#include "ssd_common.cuh"
#include "ssd_conv.cuh"
#include "ssd_norm.cuh"
#include "ssd_decode.cuh"
#include "ssd_scan_simt.cuh"
#include "ssd_strict.cuh"
#include "ssd_scan_tc.cuh"
#include "ssd_tc_selftest.cuh"

namespace ssd {
namespace {

thread_local std::string t_last_error;
thread_local int t_launches = 0;

ssd_status fail(ssd_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return st;
}

ssd_status cuda_fail(cudaError_t e, const char* what) {
    return fail(SSD_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ---------------------------------------------------------------------------------
// Per-kernel event timing (ssd_profile_enable / ssd_profile_read).
enum Stage { ST_TABLE, ST_CUMSUM, ST_CHUNK_STATE, ST_STATE_PASSING, ST_CHUNK_SCAN, ST_STATE_UPDATE,
             ST_CONV, ST_CONV_UPDATE, ST_NORM, ST_STRICT_CUMSUM, ST_STRICT_STATE, ST_STRICT_PASSING,
             ST_STRICT_SCAN, ST_STRICT_CACHE, ST_STRICT_UPDATE, ST_STRICT_FOLD, ST_COUNT };
const char* const kStageName[ST_COUNT] = {"ssd_chunk_table", "ssd_chunk_cumsum", "ssd_chunk_state",
                                          "ssd_state_passing", "ssd_chunk_scan", "ssd_state_update", "ssd_conv1d", "ssd_conv1d_update",
                                          "ssd_gated_rmsnorm", "ssd_strict_cumsum", "ssd_strict_chunk_state",
                                          "ssd_strict_state_passing", "ssd_strict_chunk_scan",
                                          "ssd_strict_cache_fill", "ssd_strict_state_update",
                                          "ssd_strict_fold"};
constexpr size_t kMaxRecords = 65536;

struct Profiler {
    std::mutex mu;
    bool on = false;
    struct Rec { int stage; cudaEvent_t a, b; };
    std::vector<Rec> recs;
    std::vector<cudaEvent_t> pool;
    int dropped = 0;
    cudaEvent_t get() {
        if (!pool.empty()) {
            cudaEvent_t e = pool.back();
            pool.pop_back();
            return e;
        }
        cudaEvent_t e = nullptr;
        if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
        return e;
    }
};
Profiler g_prof;

// Brackets one kernel launch: an NVTX range named after the stage on the host timeline
// (a no-op unless a tool such as Nsight Systems or Nsight Compute has attached), and CUDA
// events on the stream when profiling is on.
struct StageScope {
    int stage;
    cudaStream_t st;
    cudaEvent_t a = nullptr;
    StageScope(int s, cudaStream_t stream) : stage(s), st(stream) {
        nvtxRangePushA(kStageName[s]);
        std::lock_guard<std::mutex> lk(g_prof.mu);
        if (!g_prof.on) return;
        if (g_prof.recs.size() >= kMaxRecords) {
            ++g_prof.dropped;
            return;
        }
        a = g_prof.get();
        if (a) cudaEventRecord(a, st);
    }
    ~StageScope() {
        if (a) {
            std::lock_guard<std::mutex> lk(g_prof.mu);
            cudaEvent_t b = g_prof.get();
            if (b) {
                cudaEventRecord(b, st);
                g_prof.recs.push_back({stage, a, b});
            } else {
                g_prof.pool.push_back(a);
            }
        }
        nvtxRangePop();
    }
};

// ---------------------------------------------------------------------------------
// TMA descriptors (driver entry point, resolved once).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// 3-D bf16 tensor map: dims {d0 (contiguous), d1, d2}, byte strides s1, s2, box
// {64, 1, 128} (or {64, 128, 1} for 2-D data), 128-byte swizzle, zero fill.
bool make_map3(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
               uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {s1, s2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool pow2_in(int v, int lo, int hi) { return v >= lo && v <= hi && (v & (v - 1)) == 0; }

// Streaming multiprocessors of the current device (148 on B200 when no device answers).
int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return 148;
    }
    return n;
}

// Segment length forced by ssd_set_segment_tokens (0: the planner chooses).
std::atomic<int> g_segment_override{0};
// Test hook set by ssd_test_stall: the tensor-core pass whose UMMA warp stalls (0: none).
std::atomic<int> g_test_stall{0};

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Validate dims/chunk and fill the plan (no pointers looked at here).
ssd_status make_plan(const ssd_dims* d, int chunk, bool varlen, Plan* pl, int64_t snap = 0, bool strict = false) {
    if (!d) return fail(SSD_ERR_INVALID_ARG, "dims is NULL");
    if (d->nheads <= 0 || d->headdim <= 0 || d->ngroups <= 0 || d->dstate <= 0)
        return fail(SSD_ERR_INVALID_ARG, "nheads, headdim, ngroups and dstate must be positive");
    if (d->nheads % d->ngroups != 0)
        return fail(SSD_ERR_UNSUPPORTED, "nheads (%d) must be a multiple of ngroups (%d)", d->nheads,
                    d->ngroups);
    if (!pow2_in(d->headdim, 16, 128))
        return fail(SSD_ERR_UNSUPPORTED, "headdim %d not in {16,32,64,128}", d->headdim);
    if (!pow2_in(d->dstate, 16, 128))
        return fail(SSD_ERR_UNSUPPORTED, "dstate %d not in {16,32,64,128}", d->dstate);
    if (chunk != 64 && chunk != 128 && chunk != 256)
        return fail(SSD_ERR_UNSUPPORTED, "chunk %d not in {64,128,256}", chunk);
    if (d->dtype != SSD_DTYPE_F32 && d->dtype != SSD_DTYPE_BF16)
        return fail(SSD_ERR_INVALID_ARG, "unknown dtype %d", (int)d->dtype);
    Plan p;
    p.H = d->nheads;
    p.P = d->headdim;
    p.G = d->ngroups;
    p.N = d->dstate;
    p.Q = chunk;
    p.bf16 = d->dtype == SSD_DTYPE_BF16;
    p.varlen = varlen;
    if (varlen) {
        if (d->nseq < 0 || d->total_tokens < 0)
            return fail(SSD_ERR_INVALID_ARG, "nseq and total_tokens must be >= 0");
        p.nseq = d->nseq;
        p.T = d->total_tokens;
        p.max_chunks = p.T / chunk + p.nseq;
    } else {
        if (d->batch < 0 || d->seqlen < 0) return fail(SSD_ERR_INVALID_ARG, "batch and seqlen must be >= 0");
        if (d->batch > INT32_MAX) return fail(SSD_ERR_UNSUPPORTED, "batch too large");
        p.nseq = (int32_t)d->batch;
        p.seqlen = d->seqlen;
        if (d->seqlen > 0 && d->batch > INT64_MAX / d->seqlen)
            return fail(SSD_ERR_INVALID_ARG, "batch*seqlen overflows");
        p.T = d->batch * d->seqlen;
        p.max_chunks = d->batch * ((d->seqlen + chunk - 1) / chunk);
    }
    // Packed token rows and chunk indices are int32 on the device.
    if (p.T >= INT32_MAX || p.max_chunks >= INT32_MAX / 2)
        return fail(SSD_ERR_UNSUPPORTED, "more than 2^31-1 tokens in one call");
    if (p.T * (int64_t)p.H * p.P >= (int64_t)1 << 40)
        return fail(SSD_ERR_UNSUPPORTED, "x has more than 2^40 elements");
    // Tensor-core pipeline: bf16, headdim 64, dstate 128, heads per group a multiple of 4.
    p.tc = !strict && p.bf16 && p.P == tc::kP && p.N == tc::kN && (p.H / p.G) % tc::kHeads == 0;
    auto segs_for = [&](int64_t Ls) -> int64_t {
        return varlen ? p.T / Ls + p.nseq : (int64_t)p.nseq * ((p.seqlen + Ls - 1) / Ls);
    };
    if (p.tc) {
        int Ls = 256;
        if (!varlen) {
            // Dense batch: the segment length, any multiple of 128 tokens up to 16384, that
            // minimises the estimated time of the two tensor-core passes. Each pass runs its
            // CTAs (segment x 2 heads for the chunk scan, segment x 4 heads for the segment
            // states) in waves of one CTA per SM; a CTA costs (chunks per segment + 2) chunk
            // steps, the 2 standing for its prologue and epilogue; a segment-state chunk step
            // costs about 0.76 of a chunk-scan one. Ties go to the longer segment (fewer states).
            const int64_t nsm = sm_count();
            const int64_t nch = (p.seqlen + tc::kTile - 1) / tc::kTile;
            const int64_t mmax = nch < 2 ? 2 : (nch < 128 ? nch : 128);
            double best = 0.0;
            for (int64_t m = 2; m <= mmax; ++m) {
                const int64_t segs = (int64_t)p.nseq * ((nch + m - 1) / m);
                const int64_t wB = (segs * (p.H / tc::kHeadsB) + nsm - 1) / nsm;
                const int64_t wA = (segs * (p.H / tc::kHeads) + nsm - 1) / nsm;
                const double cost = ((double)wB + 0.76 * (double)wA) * (double)(m + 2);
                if (m == 2 || cost <= best) {
                    best = cost;
                    Ls = (int)(m * tc::kTile);
                }
            }
        } else {
            // Packed varlen (segment counts known only as an upper bound): the longest of
            // 8192/.../512/256 tokens whose chunk-scan grid still fills one wave.
            const int64_t nsm = sm_count();
            for (int cand : {8192, 4096, 2048, 1024, 512}) {
                if (segs_for(cand) * (p.H / tc::kHeadsB) >= nsm) {
                    Ls = cand;
                    break;
                }
            }
        }
        if (const int v = g_segment_override.load()) Ls = v;
        // Snapshots cut the segments' states at multiples of snap (sub-segments), which
        // must fall on 128-token chunk boundaries; the segment length stays as chosen.
        if (snap > 0 && snap % tc::kTile != 0)
            return fail(SSD_ERR_UNSUPPORTED, "snapshot_tokens (%lld) must be a multiple of %d here",
                        (long long)snap, tc::kTile);
        p.Ls = Ls;
        p.max_segs = segs_for(Ls);
        p.max_subs = p.max_segs + (snap > 0 ? p.T / snap : 0);
    }
    if (snap < 0) return fail(SSD_ERR_INVALID_ARG, "snapshot_tokens must be >= 0");
    if (snap > 0 && !p.tc && snap % chunk != 0)
        return fail(SSD_ERR_UNSUPPORTED, "snapshot_tokens (%lld) must be a multiple of chunk (%d) here",
                    (long long)snap, chunk);
    p.snap = snap;
    // Workspace carving (256-byte aligned pieces).
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    if (p.tc) {
        const size_t ms = (size_t)p.max_segs, mu = (size_t)p.max_subs;
        p.off_table = take(sizeof(ChunkEntry) * (ms > 0 ? ms : 1));
        p.off_first = take(sizeof(int32_t) * ((size_t)p.nseq + 1));
        p.off_count = take(sizeof(int32_t));
        p.off_states = take(sizeof(float) * mu * p.H * p.P * p.N);
        p.off_seg_acum = take(sizeof(float) * mu * p.H);
        p.off_order = take(sizeof(int32_t) * (ms > 0 ? ms : 1));
        if (snap > 0) {
            p.off_sub_first = take(sizeof(int32_t) * ((size_t)p.nseq + 1));
            p.off_sub_end = take(sizeof(int32_t) * (mu > 0 ? mu : 1));
        }
    } else {
        const size_t mc = (size_t)p.max_chunks;
        p.off_table = take(sizeof(ChunkEntry) * (mc > 0 ? mc : 1));
        p.off_first = take(sizeof(int32_t) * ((size_t)p.nseq + 1));
        p.off_count = take(sizeof(int32_t));
        p.off_dt = take(sizeof(float) * mc * p.H * p.Q);
        p.off_acum = take(sizeof(float) * mc * p.H * p.Q);
        p.off_states = take(sizeof(float) * mc * p.H * p.P * p.N);
    }
    if (snap > 0) p.off_snap_first = take(sizeof(int32_t) * ((size_t)p.nseq + 1));
    p.bytes = off;
    *pl = p;
    return SSD_OK;
}

// ---------------------------------------------------------------------------------
// SIMT pipeline launch, templated on the geometry.
template <typename T, int Q, int P, int N>
ssd_status launch_simt(const Plan& pl, char* ws, const T* x, const float* dt_raw,
                       const float* dt_bias, const float* A, const T* B, const T* C,
                       const float* D, const float* init, const int32_t* cu, T* y, float* fin,
                       cudaStream_t st) {
    auto* table = reinterpret_cast<ChunkEntry*>(ws + pl.off_table);
    auto* first = reinterpret_cast<int32_t*>(ws + pl.off_first);
    auto* count = reinterpret_cast<int32_t*>(ws + pl.off_count);
    auto* dtc = reinterpret_cast<float*>(ws + pl.off_dt);
    auto* acum = reinterpret_cast<float*>(ws + pl.off_acum);
    auto* states = reinterpret_cast<float*>(ws + pl.off_states);
    const int H = pl.H, G = pl.G;
    int n = 0;
    {
        StageScope sc(ST_TABLE, st);
        k_chunk_table<<<1, kTableThreads, 0, st>>>(cu, pl.nseq, pl.T, pl.seqlen, Q, table, first, count, pl.snap,
                                                   reinterpret_cast<int32_t*>(ws + pl.off_snap_first));
    }
    ++n;
    if (pl.max_chunks > 0) {
        const unsigned mc = (unsigned)pl.max_chunks;
        {
            StageScope sc(ST_CUMSUM, st);
            k_chunk_cumsum<Q><<<dim3(mc, (H + 31) / 32), 256, 0, st>>>(dt_raw, dt_bias, A, table,
                                                                        count, H, dtc, acum);
        }
        {
            StageScope sc(ST_CHUNK_STATE, st);
            k_chunk_state_simt<T, Q, P, N><<<dim3(mc, H), 256, 0, st>>>(x, B, dtc, acum, table,
                                                                         count, H, G, states);
        }
        n += 2;
    }
    if (pl.nseq > 0) {
        StageScope sc(ST_STATE_PASSING, st);
        k_state_passing<Q><<<dim3(pl.nseq, H, (P * N + 255) / 256), 256, 0, st>>>(
            states, acum, table, first, init, fin, H, P * N, pl.snap,
            reinterpret_cast<const int32_t*>(ws + pl.off_snap_first), pl.snap_out);
        ++n;
    }
    if (pl.max_chunks > 0) {
        constexpr size_t smem = chunk_scan_simt_smem<Q, P, N>();
        cudaError_t e = cudaFuncSetAttribute(k_chunk_scan_simt<T, Q, P, N>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(chunk_scan)");
        StageScope sc(ST_CHUNK_SCAN, st);
        k_chunk_scan_simt<T, Q, P, N><<<dim3((unsigned)pl.max_chunks, H, Q / 32), 256, smem, st>>>(
            x, B, C, D, dtc, acum, states, table, count, H, G, y);
        ++n;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch (simt scan)");
    t_launches = n;
    return SSD_OK;
}

// ---------------------------------------------------------------------------------
// Tensor-core pipeline launch (bf16, P = 64, N = 128).
ssd_status launch_tc(const Plan& pl, char* ws, const void* x, const float* dt_raw, const float* dt_bias,
                     const float* A, const void* B, const void* C, const float* D, const float* init,
                     const int32_t* cu, void* y, float* fin, cudaStream_t st) {
    auto* table = reinterpret_cast<ChunkEntry*>(ws + pl.off_table);
    auto* first = reinterpret_cast<int32_t*>(ws + pl.off_first);
    auto* count = reinterpret_cast<int32_t*>(ws + pl.off_count);
    auto* seg_state = reinterpret_cast<float*>(ws + pl.off_states);
    auto* seg_acum = reinterpret_cast<float*>(ws + pl.off_seg_acum);
    int32_t* order = pl.varlen ? reinterpret_cast<int32_t*>(ws + pl.off_order) : nullptr;
    // with snapshots the chain walks sub-segments (slot ranges sub_first), else segments
    int32_t* sub_first = pl.snap > 0 ? reinterpret_cast<int32_t*>(ws + pl.off_sub_first) : nullptr;
    int32_t* sub_end = pl.snap > 0 ? reinterpret_cast<int32_t*>(ws + pl.off_sub_end) : nullptr;
    const int32_t* slot_first = sub_first ? sub_first : first;
    const int H = pl.H, G = pl.G;
    int n = 0;
    // A dense batch without snapshots: the segment-state pass writes the table itself.
    const bool dense_table = !pl.varlen && pl.snap <= 0 && pl.max_segs > 0 && pl.T > 0;
    if (!dense_table) {
        StageScope sc(ST_TABLE, st);
        k_chunk_table<<<1, kTableThreads, 0, st>>>(cu, pl.nseq, pl.T, pl.seqlen, pl.Ls, table, first, count,
                                                   pl.snap, reinterpret_cast<int32_t*>(ws + pl.off_snap_first),
                                                   order, sub_first, sub_end);
        ++n;
    }
    if (pl.max_segs > 0 && pl.T > 0) {
        CUtensorMap mx, mxa, mb, mc, my;
        const uint64_t T = (uint64_t)pl.T;
        if (!make_map3(&mx, x, tc::kP, H, T, (uint64_t)tc::kP * 2, (uint64_t)H * tc::kP * 2, 64, 1, tc::kTile) ||
            !make_map3(&mxa, x, tc::kP, H, T, (uint64_t)tc::kP * 2, (uint64_t)H * tc::kP * 2, 64, 1, tc::kXRows) ||
            !make_map3(&mb, B, tc::kN, G, T, (uint64_t)tc::kN * 2, (uint64_t)G * tc::kN * 2, 64, 1, tc::kTile) ||
            !make_map3(&mc, C, tc::kN, G, T, (uint64_t)tc::kN * 2, (uint64_t)G * tc::kN * 2, 64, 1, tc::kTile) ||
            !make_map3(&my, y, tc::kP, H, T, (uint64_t)tc::kP * 2, (uint64_t)H * tc::kP * 2, 64, 1, tc::kTile))
            return fail(SSD_ERR_CUDA, "cuTensorMapEncodeTiled failed (x/B/C/y tensor maps)");
        cudaError_t e = cudaFuncSetAttribute(tc::k_tc_segment_state, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             tc::kSmemA);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(tc::k_tc_chunk_scan, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::kSmemB);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(tc kernels)");
        {
            StageScope sc(ST_CHUNK_STATE, st);
            tc::k_tc_segment_state<<<(unsigned)(pl.max_segs * (H / tc::kHeads)), tc::kThreadsA, tc::kSmemA,
                                     st>>>(mxa, mb, dt_raw, dt_bias, A, table, count, H, G,
                                                                  seg_state, seg_acum, order, first, pl.snap,
                                                                  g_test_stall.load() == 1, pl.nseq,
                                                                  dense_table ? pl.seqlen : 0, pl.Ls);
        }
        ++n;
        {
            StageScope sc(ST_STATE_PASSING, st);
            tc::k_tc_segment_passing<<<dim3(pl.nseq, H, tc::kP * tc::kN / tc::kPassElems), 256, 0, st>>>(
                seg_state, seg_acum, slot_first, init, fin, H, pl.Ls, pl.snap, sub_end,
                reinterpret_cast<const int32_t*>(ws + pl.off_snap_first), pl.snap_out);
        }
        ++n;
        {
            StageScope sc(ST_CHUNK_SCAN, st);
            tc::k_tc_chunk_scan<<<(unsigned)(pl.max_segs * (H / tc::kHeadsB)), tc::kThreadsB, tc::kSmemB, st>>>(mx, mb, mc, my, dt_raw, dt_bias, A, D, table, count, H,
                                                               G, seg_state, (__nv_bfloat16*)y, order,
                                                               g_test_stall.load() == 2);
        }
        ++n;
    } else {
        StageScope sc(ST_STATE_PASSING, st);
        tc::k_tc_segment_passing<<<dim3(pl.nseq, H, tc::kP * tc::kN / tc::kPassElems), 256, 0, st>>>(
            seg_state, seg_acum, slot_first, init, fin, H, pl.Ls, pl.snap, sub_end,
            reinterpret_cast<const int32_t*>(ws + pl.off_snap_first), pl.snap_out);
        ++n;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch (tc scan)");
    t_launches = n;
    return SSD_OK;
}

template <typename T, int Q>
ssd_status dispatch_PN(const Plan& pl, char* ws, const void* x, const float* dt_raw,
                       const float* dt_bias, const float* A, const void* B, const void* C,
                       const float* D, const float* init, const int32_t* cu, void* y, float* fin,
                       cudaStream_t st) {
#define SSD_CASE(PP, NN)                                                                       \
    if (pl.P == PP && pl.N == NN)                                                              \
        return launch_simt<T, Q, PP, NN>(pl, ws, (const T*)x, dt_raw, dt_bias, A, (const T*)B, \
                                         (const T*)C, D, init, cu, (T*)y, fin, st);
#define SSD_CASES_N(PP) SSD_CASE(PP, 16) SSD_CASE(PP, 32) SSD_CASE(PP, 64) SSD_CASE(PP, 128)
    SSD_CASES_N(16) SSD_CASES_N(32) SSD_CASES_N(64) SSD_CASES_N(128)
#undef SSD_CASES_N
#undef SSD_CASE
    return fail(SSD_ERR_UNSUPPORTED, "headdim/dstate combination");
}

template <typename T>
ssd_status dispatch_Q(const Plan& pl, char* ws, const void* x, const float* dt_raw,
                      const float* dt_bias, const float* A, const void* B, const void* C,
                      const float* D, const float* init, const int32_t* cu, void* y, float* fin,
                      cudaStream_t st) {
    switch (pl.Q) {
        case 64: return dispatch_PN<T, 64>(pl, ws, x, dt_raw, dt_bias, A, B, C, D, init, cu, y, fin, st);
        case 128: return dispatch_PN<T, 128>(pl, ws, x, dt_raw, dt_bias, A, B, C, D, init, cu, y, fin, st);
        case 256: return dispatch_PN<T, 256>(pl, ws, x, dt_raw, dt_bias, A, B, C, D, init, cu, y, fin, st);
    }
    return fail(SSD_ERR_UNSUPPORTED, "chunk");
}

template <typename T, int P, int N>
void launch_decode(float* state, const void* x, const float* dt_raw, const float* dt_bias,
                   const float* A, const void* B, const void* C, const float* D, void* y,
                   int64_t nseq, int H, int G, cudaStream_t st) {
    StageScope sc(ST_STATE_UPDATE, st);
    k_state_update<T, P, N><<<(unsigned)(nseq * H), kDecodeThreads, 0, st>>>(
        state, (const T*)x, dt_raw, dt_bias, A, (const T*)B, (const T*)C, D, (T*)y, H, G);
}

template <typename T>
ssd_status dispatch_decode(int P, int N, float* state, const void* x, const float* dt_raw,
                           const float* dt_bias, const float* A, const void* B, const void* C,
                           const float* D, void* y, int64_t nseq, int H, int G, cudaStream_t st) {
#define SSD_CASE(PP, NN)                                                                \
    if (P == PP && N == NN) {                                                           \
        launch_decode<T, PP, NN>(state, x, dt_raw, dt_bias, A, B, C, D, y, nseq, H, G, st); \
        return SSD_OK;                                                                  \
    }
#define SSD_CASES_N(PP) SSD_CASE(PP, 16) SSD_CASE(PP, 32) SSD_CASE(PP, 64) SSD_CASE(PP, 128)
    SSD_CASES_N(16) SSD_CASES_N(32) SSD_CASES_N(64) SSD_CASES_N(128)
#undef SSD_CASES_N
#undef SSD_CASE
    return fail(SSD_ERR_UNSUPPORTED, "headdim/dstate combination");
}

}  // namespace
}  // namespace ssd

using namespace ssd;

extern "C" {

ssd_status ssd_scan_fwd_workspace_size(const ssd_dims* dims, int chunk, size_t* bytes) {
    if (!bytes) return fail(SSD_ERR_INVALID_ARG, "bytes is NULL");
    // Covers both modes for the fields given: the dense reading (batch, seqlen) and
    // the packed reading (nseq, total_tokens); the larger of the valid ones wins.
    Plan dense, packed;
    const ssd_status sd = make_plan(dims, chunk, false, &dense);
    const ssd_status sp = make_plan(dims, chunk, true, &packed);
    if (sd != SSD_OK && sp != SSD_OK) return sd;
    size_t b = 0;
    if (sd == SSD_OK) b = dense.bytes;
    if (sp == SSD_OK && packed.bytes > b) b = packed.bytes;
    t_last_error.clear();
    *bytes = b;
    return SSD_OK;
}

}  // extern "C"

namespace ssd {
namespace {

// ssd_scan_fwd and ssd_scan_fwd_snapshots: validate, find scratch, launch.
ssd_status scan_fwd_impl(const void* x, const float* dt_raw, const float* dt_bias, const float* A, const void* B,
                         const void* C, const float* D, const float* init_state, const int32_t* cu_seqlens,
                         void* y, float* final_state, float* snapshots, int64_t snapshot_tokens,
                         const ssd_dims* dims, int chunk, ssd_stream_t stream) {
    Plan pl;
    ssd_status s = make_plan(dims, chunk, cu_seqlens != nullptr, &pl, snapshot_tokens);
    if (s != SSD_OK) return s;
    if (!dt_bias || !A || !D) return fail(SSD_ERR_INVALID_ARG, "dt_bias, A and D must be non-NULL");
    if (pl.T > 0 && (!x || !dt_raw || !B || !C || !y))
        return fail(SSD_ERR_INVALID_ARG, "x, dt_raw, B, C and y must be non-NULL");
    if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(y, 16))
        return fail(SSD_ERR_INVALID_ARG, "x, B, C and y must be 16-byte aligned");
    if (!aligned(dt_raw, 4) || !aligned(dt_bias, 4) || !aligned(A, 4) || !aligned(D, 4) ||
        !aligned(init_state, 16) || !aligned(final_state, 16) || !aligned(cu_seqlens, 4))
        return fail(SSD_ERR_INVALID_ARG, "float/int arrays must be 4-byte aligned, states 16-byte");
    if (snapshot_tokens > 0 && (!snapshots || !aligned(snapshots, 16)))
        return fail(SSD_ERR_INVALID_ARG, "snapshots must be a non-NULL 16-byte aligned array");
    pl.snap_out = snapshots;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (pl.nseq == 0) {
        t_launches = 0;
        t_last_error.clear();
        return SSD_OK;
    }
    char* ws = static_cast<char*>(dims->workspace);
    bool owned = false;
    if (ws) {
        if (dims->workspace_bytes < pl.bytes)
            return fail(SSD_ERR_INVALID_ARG, "workspace_bytes %zu < required %zu", dims->workspace_bytes,
                        pl.bytes);
        if (!aligned(ws, 256)) return fail(SSD_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    } else {
        cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(&ws), pl.bytes, st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(workspace)");
        owned = true;
    }
    if (pl.tc)
        s = launch_tc(pl, ws, x, dt_raw, dt_bias, A, B, C, D, init_state, cu_seqlens, y, final_state, st);
    else if (pl.bf16)
        s = dispatch_Q<__nv_bfloat16>(pl, ws, x, dt_raw, dt_bias, A, B, C, D, init_state, cu_seqlens, y,
                                      final_state, st);
    else
        s = dispatch_Q<float>(pl, ws, x, dt_raw, dt_bias, A, B, C, D, init_state, cu_seqlens, y,
                              final_state, st);
    if (owned) {
        cudaError_t e = cudaFreeAsync(ws, st);
        if (e != cudaSuccess && s == SSD_OK) return cuda_fail(e, "cudaFreeAsync(workspace)");
    }
    if (s == SSD_OK) t_last_error.clear();
    return s;
}

}  // namespace
}  // namespace ssd

extern "C" {

ssd_status ssd_scan_fwd(const void* x, const float* dt_raw, const float* dt_bias, const float* A,
                        const void* B, const void* C, const float* D, const float* init_state,
                        const int32_t* cu_seqlens, void* y, float* final_state,
                        const ssd_dims* dims, int chunk, ssd_stream_t stream) {
    return scan_fwd_impl(x, dt_raw, dt_bias, A, B, C, D, init_state, cu_seqlens, y, final_state, nullptr, 0,
                         dims, chunk, stream);
}

ssd_status ssd_scan_fwd_snapshots(const void* x, const float* dt_raw, const float* dt_bias, const float* A,
                                  const void* B, const void* C, const float* D, const float* init_state,
                                  const int32_t* cu_seqlens, void* y, float* final_state, float* snapshots,
                                  int64_t snapshot_tokens, const ssd_dims* dims, int chunk,
                                  ssd_stream_t stream) {
    if (snapshot_tokens <= 0) return fail(SSD_ERR_INVALID_ARG, "snapshot_tokens must be > 0");
    return scan_fwd_impl(x, dt_raw, dt_bias, A, B, C, D, init_state, cu_seqlens, y, final_state, snapshots,
                         snapshot_tokens, dims, chunk, stream);
}

ssd_status ssd_scan_fwd_snapshots_workspace_size(const ssd_dims* dims, int chunk, int64_t snapshot_tokens,
                                                 size_t* bytes) {
    if (!bytes) return fail(SSD_ERR_INVALID_ARG, "bytes is NULL");
    if (snapshot_tokens <= 0) return fail(SSD_ERR_INVALID_ARG, "snapshot_tokens must be > 0");
    Plan dense, packed;
    const ssd_status sd = make_plan(dims, chunk, false, &dense, snapshot_tokens);
    const ssd_status sp = make_plan(dims, chunk, true, &packed, snapshot_tokens);
    if (sd != SSD_OK && sp != SSD_OK) return sd;
    size_t b = 0;
    if (sd == SSD_OK) b = dense.bytes;
    if (sp == SSD_OK && packed.bytes > b) b = packed.bytes;
    t_last_error.clear();
    *bytes = b;
    return SSD_OK;
}

ssd_status ssd_snapshot_count(const ssd_dims* dims, const int32_t* cu_seqlens_host, int64_t snapshot_tokens,
                              int64_t* count) {
    if (!dims || !count) return fail(SSD_ERR_INVALID_ARG, "dims and count must be non-NULL");
    if (snapshot_tokens <= 0) return fail(SSD_ERR_INVALID_ARG, "snapshot_tokens must be > 0");
    int64_t n = 0;
    if (cu_seqlens_host) {
        if (dims->nseq < 0) return fail(SSD_ERR_INVALID_ARG, "nseq must be >= 0");
        for (int32_t s = 0; s < dims->nseq; ++s) {
            const int64_t len = (int64_t)cu_seqlens_host[s + 1] - cu_seqlens_host[s];
            if (len < 0) return fail(SSD_ERR_INVALID_ARG, "cu_seqlens must be non-decreasing");
            n += len / snapshot_tokens;
        }
    } else {
        if (dims->batch < 0 || dims->seqlen < 0) return fail(SSD_ERR_INVALID_ARG, "batch and seqlen must be >= 0");
        n = dims->batch * (dims->seqlen / snapshot_tokens);
    }
    t_last_error.clear();
    *count = n;
    return SSD_OK;
}

ssd_status ssd_state_update(float* state, const void* x, const float* dt_raw, const float* dt_bias,
                            const float* A, const void* B, const void* C, const float* D, void* y,
                            const ssd_dims* dims, ssd_stream_t stream) {
    if (!dims) return fail(SSD_ERR_INVALID_ARG, "dims is NULL");
    Plan pl;
    ssd_dims d = *dims;
    if (d.seqlen != 1) return fail(SSD_ERR_INVALID_ARG, "decode takes seqlen == 1 (got %lld)",
                                   (long long)d.seqlen);
    ssd_status s = make_plan(&d, 64, false, &pl);
    if (s != SSD_OK) return s;
    if (pl.nseq == 0) {
        t_launches = 0;
        t_last_error.clear();
        return SSD_OK;
    }
    if (!state || !x || !dt_raw || !dt_bias || !A || !B || !C || !D || !y)
        return fail(SSD_ERR_INVALID_ARG, "all decode pointers must be non-NULL");
    if (!aligned(state, 16) || !aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(y, 16))
        return fail(SSD_ERR_INVALID_ARG, "state, x, B, C and y must be 16-byte aligned");
    if (!aligned(dt_raw, 4) || !aligned(dt_bias, 4) || !aligned(A, 4) || !aligned(D, 4))
        return fail(SSD_ERR_INVALID_ARG, "float arrays must be 4-byte aligned");
    if ((int64_t)pl.nseq * pl.H >= INT32_MAX) return fail(SSD_ERR_UNSUPPORTED, "nseq*nheads too large");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (pl.bf16)
        s = dispatch_decode<__nv_bfloat16>(pl.P, pl.N, state, x, dt_raw, dt_bias, A, B, C, D, y,
                                           pl.nseq, pl.H, pl.G, st);
    else
        s = dispatch_decode<float>(pl.P, pl.N, state, x, dt_raw, dt_bias, A, B, C, D, y, pl.nseq,
                                   pl.H, pl.G, st);
    if (s != SSD_OK) return s;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch (state update)");
    t_launches = 1;
    t_last_error.clear();
    return SSD_OK;
}

ssd_status ssd_get_device_status(ssd_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int code = 0;
    e = cudaMemcpyFromSymbol(&code, g_device_error, sizeof code);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol(error word)");
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyToSymbol(error word)");
    if (code == 0) {
        t_last_error.clear();
        return SSD_OK;
    }
    if (code == SSD_ERR_TIMEOUT) return fail(SSD_ERR_TIMEOUT, "a device-side bounded wait expired");
    return fail((ssd_status)code, "a kernel rejected its data (bad cu_seqlens, or A > 0 / not finite)");
}

const char* ssd_last_error(void) { return t_last_error.c_str(); }

const char* ssd_scan_fwd_variant(const ssd_dims* dims, int chunk) {
    Plan pl;
    if (make_plan(dims, chunk, false, &pl) != SSD_OK) return "";
    return pl.tc ? "tc" : "simt";
}

int ssd_last_launch_count(void) { return t_launches; }

void ssd_set_segment_tokens(int tokens) {
    g_segment_override.store(tokens >= tc::kTile && tokens % tc::kTile == 0 && tokens <= (1 << 20) ? tokens : 0);
}

void ssd_test_stall(int pass) { g_test_stall.store(pass == 1 || pass == 2 ? pass : 0); }

int ssd_scan_fwd_segment_tokens(const ssd_dims* dims, int chunk) {
    Plan pl;
    if (make_plan(dims, chunk, dims && dims->batch == 0 && dims->nseq > 0, &pl) != SSD_OK) return 0;
    return pl.tc ? pl.Ls : 0;
}

ssd_status ssd_selftest_umma(const void* X1, const void* X2, float* out, ssd_stream_t stream) {
    if (!X1 || !X2 || !out) return fail(SSD_ERR_INVALID_ARG, "selftest pointers must be non-NULL");
    if (!aligned(X1, 16) || !aligned(X2, 16) || !aligned(out, 16))
        return fail(SSD_ERR_INVALID_ARG, "selftest pointers must be 16-byte aligned");
    CUtensorMap m1, m2;
    if (!make_map3(&m1, X1, 128, 128, 1, 256, 256 * 128, 64, 128, 1) ||
        !make_map3(&m2, X2, 128, 128, 1, 256, 256 * 128, 64, 128, 1))
        return fail(SSD_ERR_CUDA, "cuTensorMapEncodeTiled failed (selftest)");
    cudaError_t e = cudaFuncSetAttribute(tc::k_umma_selftest, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         tc::kSelftestSmem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(selftest)");
    tc::k_umma_selftest<<<1, 128, tc::kSelftestSmem, reinterpret_cast<cudaStream_t>(stream)>>>(
        m1, m2, (const __nv_bfloat16*)X1, (const __nv_bfloat16*)X2, out);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch (selftest)");
    t_launches = 1;
    t_last_error.clear();
    return SSD_OK;
}

void ssd_profile_enable(int on) {
    std::lock_guard<std::mutex> lk(g_prof.mu);
    g_prof.on = on != 0;
    if (g_prof.on) {
        for (auto& r : g_prof.recs) {
            g_prof.pool.push_back(r.a);
            g_prof.pool.push_back(r.b);
        }
        g_prof.recs.clear();
        g_prof.dropped = 0;
    }
}

int ssd_profile_read(ssd_kernel_time* out, int max, int* dropped) {
    std::lock_guard<std::mutex> lk(g_prof.mu);
    double ms[ST_COUNT] = {0};
    int cnt[ST_COUNT] = {0};
    int rc = 0;
    for (auto& r : g_prof.recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
            rc = -1;
        ms[r.stage] += t;
        cnt[r.stage] += 1;
        g_prof.pool.push_back(r.a);
        g_prof.pool.push_back(r.b);
    }
    g_prof.recs.clear();
    if (dropped) *dropped = g_prof.dropped;
    g_prof.dropped = 0;
    if (rc) return fail(SSD_ERR_CUDA, "waiting on a profiling event failed"), -1;
    int k = 0;
    for (int i = 0; i < ST_COUNT; ++i)
        if (cnt[i] > 0) {
            if (out && k < max) out[k] = {kStageName[i], cnt[i], ms[i]};
            ++k;
        }
    return k;
}

}  // extern "C"

// ---------------------------------------------------------------------------------
// Prefill without any allocation. Some callers cannot allocate device memory at call
// time: serving engines that reserve their whole memory budget up front and forbid
// later allocations, and latency-critical callers for which a cudaMalloc/cudaFree (or
// a trip into a caching allocator) in the middle of a step is not acceptable. This
// entry point takes its scratch from one array compiled into the library instead.
namespace ssd {
namespace {

// Scratch compiled into the library: every GPU that loads libssd holds these 32 MiB
// until the process exits. Host code must not pass the symbol itself to a kernel (on
// the host it is only a stand-in); the device address is looked up with the device
// current.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device. It is looked up on every
// call made outside stream capture (cheap), so a context that was reset and re-created
// since an earlier call gets the address in its own module; during capture the address
// of the device's last lookup is used (so the first call on a device must come before
// any capture).
ssd_status noalloc_scratch(cudaStream_t st, char** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(SSD_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(st, &cap);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (cap == cudaStreamCaptureStatusNone) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
        g_noalloc_addr[dev] = p;
    } else if (!g_noalloc_addr[dev]) {
        return fail(SSD_ERR_UNSUPPORTED, "first ssd_scan_fwd_noalloc call on device %d made during stream capture", dev);
    }
    *out = static_cast<char*>(g_noalloc_addr[dev]);
    return SSD_OK;
}

}  // namespace
}  // namespace ssd

extern "C" ssd_status ssd_scan_fwd_noalloc(const void* x, const float* dt_raw, const float* dt_bias,
                                           const float* A, const void* B, const void* C, const float* D,
                                           const float* init_state, const int32_t* cu_seqlens, void* y,
                                           float* final_state, const ssd_dims* dims, int chunk,
                                           ssd_stream_t stream) {
    Plan pl;
    ssd_status s = make_plan(dims, chunk, cu_seqlens != nullptr, &pl);
    if (s != SSD_OK) return s;
    if (dims->workspace)
        return fail(SSD_ERR_INVALID_ARG, "ssd_scan_fwd_noalloc uses its own scratch: dims->workspace must be NULL");
    if (!dt_bias || !A || !D) return fail(SSD_ERR_INVALID_ARG, "dt_bias, A and D must be non-NULL");
    if (pl.T > 0 && (!x || !dt_raw || !B || !C || !y))
        return fail(SSD_ERR_INVALID_ARG, "x, dt_raw, B, C and y must be non-NULL");
    if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(y, 16))
        return fail(SSD_ERR_INVALID_ARG, "x, B, C and y must be 16-byte aligned");
    if (!aligned(dt_raw, 4) || !aligned(dt_bias, 4) || !aligned(A, 4) || !aligned(D, 4) ||
        !aligned(init_state, 16) || !aligned(final_state, 16) || !aligned(cu_seqlens, 4))
        return fail(SSD_ERR_INVALID_ARG, "float/int arrays must be 4-byte aligned, states 16-byte");
    if (pl.bytes > kNoAllocScratchBytes)
        return fail(SSD_ERR_UNSUPPORTED,
                    "problem needs %zu bytes of scratch; ssd_scan_fwd_noalloc has %zu (use ssd_scan_fwd)",
                    pl.bytes, kNoAllocScratchBytes);
    if (pl.nseq == 0) {
        t_launches = 0;
        t_last_error.clear();
        return SSD_OK;
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* ws = nullptr;
    s = noalloc_scratch(st, &ws);
    if (s != SSD_OK) return s;
    // Every slot of the scratch that a kernel reads is written earlier in the same call
    // (chunk/segment table, then states), so nothing needs clearing between calls.
    if (pl.tc)
        s = launch_tc(pl, ws, x, dt_raw, dt_bias, A, B, C, D, init_state, cu_seqlens, y, final_state, st);
    else if (pl.bf16)
        s = dispatch_Q<__nv_bfloat16>(pl, ws, x, dt_raw, dt_bias, A, B, C, D, init_state, cu_seqlens, y,
                                      final_state, st);
    else
        s = dispatch_Q<float>(pl, ws, x, dt_raw, dt_bias, A, B, C, D, init_state, cu_seqlens, y, final_state,
                              st);
    if (s == SSD_OK) t_last_error.clear();
    return s;
}

// ---------------------------------------------------------------------------------
// Causal conv1d prologue (prefill and decode).
namespace ssd {
namespace {

struct ConvShape {
    int64_t T = 0, seqlen = 0;
    int32_t nseq = 0;
    int Dc = 0, HP = 0, GN = 0;
    bool bf16 = false;
};

ssd_status conv_shape(const ssd_dims* d, bool varlen, int width, ConvShape* cs) {
    if (!d) return fail(SSD_ERR_INVALID_ARG, "dims is NULL");
    if (d->nheads <= 0 || d->headdim <= 0 || d->ngroups <= 0 || d->dstate <= 0)
        return fail(SSD_ERR_INVALID_ARG, "nheads, headdim, ngroups and dstate must be positive");
    if (d->nheads % d->ngroups != 0) return fail(SSD_ERR_UNSUPPORTED, "nheads must be a multiple of ngroups");
    if (!pow2_in(d->headdim, 16, 128) || !pow2_in(d->dstate, 16, 128))
        return fail(SSD_ERR_UNSUPPORTED, "headdim and dstate must be in {16,32,64,128}");
    if (width < 2 || width > 4) return fail(SSD_ERR_UNSUPPORTED, "conv width %d not in {2,3,4}", width);
    if (d->dtype != SSD_DTYPE_F32 && d->dtype != SSD_DTYPE_BF16)
        return fail(SSD_ERR_INVALID_ARG, "unknown dtype %d", (int)d->dtype);
    ConvShape c;
    c.HP = d->nheads * d->headdim;
    c.GN = d->ngroups * d->dstate;
    c.Dc = c.HP + 2 * c.GN;
    c.bf16 = d->dtype == SSD_DTYPE_BF16;
    if (varlen) {
        if (d->nseq < 0 || d->total_tokens < 0) return fail(SSD_ERR_INVALID_ARG, "nseq and total_tokens must be >= 0");
        c.nseq = d->nseq;
        c.T = d->total_tokens;
    } else {
        if (d->batch < 0 || d->seqlen < 0) return fail(SSD_ERR_INVALID_ARG, "batch and seqlen must be >= 0");
        if (d->batch > INT32_MAX) return fail(SSD_ERR_UNSUPPORTED, "batch too large");
        if (d->seqlen > 0 && d->batch > INT64_MAX / d->seqlen) return fail(SSD_ERR_INVALID_ARG, "batch*seqlen overflows");
        c.nseq = (int32_t)d->batch;
        c.seqlen = d->seqlen;
        c.T = d->batch * d->seqlen;
    }
    if (c.T >= INT32_MAX) return fail(SSD_ERR_UNSUPPORTED, "more than 2^31-1 tokens in one call");
    *cs = c;
    return SSD_OK;
}

template <typename T, int K>
void launch_conv(const ConvShape& c, const void* in, const float* w, const float* bias, const void* st_in,
                 const int32_t* cu, void* x, void* B, void* C, void* st_out, cudaStream_t st) {
    const unsigned cx = (unsigned)((c.Dc / 8 + kConvThreads - 1) / kConvThreads);
    if (c.T > 0) {
        StageScope sc(ST_CONV, st);
        k_conv1d_fwd<T, K><<<dim3((unsigned)((c.T + kConvTokens - 1) / kConvTokens), cx), kConvThreads, 0, st>>>(
            (const T*)in, w, bias, (const T*)st_in, cu, c.nseq, c.T, c.seqlen, c.Dc, c.HP, c.GN, (T*)x, (T*)B, (T*)C,
            (T*)st_out);
    }
    if (st_out && c.nseq > 0) {
        const int64_t n = (int64_t)c.nseq * c.Dc;
        k_conv1d_empty<T, K><<<(unsigned)((n + 255) / 256), 256, 0, st>>>((const T*)st_in, cu, c.nseq, c.seqlen, c.Dc,
                                                                          (T*)st_out);
    }
}

template <typename T, int K>
void launch_conv_update(const ConvShape& c, void* state, const void* in, const float* w, const float* bias, void* x,
                        void* B, void* C, cudaStream_t st) {
    StageScope sc(ST_CONV_UPDATE, st);
    const unsigned cx = (unsigned)((c.Dc / 8 + kConvThreads - 1) / kConvThreads);
    k_conv1d_update<T, K><<<dim3(cx, (unsigned)((c.nseq + kConvSeqs - 1) / kConvSeqs)), kConvThreads, 0, st>>>(
        (T*)state, (const T*)in, w, bias, c.nseq, c.Dc, c.HP, c.GN, (T*)x, (T*)B, (T*)C);
}

}  // namespace
}  // namespace ssd

extern "C" ssd_status ssd_conv1d_fwd(const void* xbc, const float* weight, const float* bias,
                                     const void* conv_state_in, const int32_t* cu_seqlens, void* x, void* B,
                                     void* C, void* conv_state_out, const ssd_dims* dims, int width,
                                     ssd_stream_t stream) {
    ConvShape c;
    ssd_status s = conv_shape(dims, cu_seqlens != nullptr, width, &c);
    if (s != SSD_OK) return s;
    if (c.T > 0 && (!xbc || !weight || !x || !B || !C))
        return fail(SSD_ERR_INVALID_ARG, "xbc, weight, x, B and C must be non-NULL");
    if (!aligned(xbc, 16) || !aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16))
        return fail(SSD_ERR_INVALID_ARG, "xbc, x, B and C must be 16-byte aligned");
    if (!aligned(weight, 16) || !aligned(bias, 16) || !aligned(cu_seqlens, 4) || !aligned(conv_state_in, 4) ||
        !aligned(conv_state_out, 4))
        return fail(SSD_ERR_INVALID_ARG, "weight and bias must be 16-byte aligned, cu_seqlens and conv states 4-byte");
    if (c.nseq == 0) {
        t_launches = 0;
        t_last_error.clear();
        return SSD_OK;
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define SSD_CONV_CASE(TT, KK)                                                                          \
    if (width == KK) launch_conv<TT, KK>(c, xbc, weight, bias, conv_state_in, cu_seqlens, x, B, C, conv_state_out, st);
    if (c.bf16) {
        SSD_CONV_CASE(__nv_bfloat16, 2) SSD_CONV_CASE(__nv_bfloat16, 3) SSD_CONV_CASE(__nv_bfloat16, 4)
    } else {
        SSD_CONV_CASE(float, 2) SSD_CONV_CASE(float, 3) SSD_CONV_CASE(float, 4)
    }
#undef SSD_CONV_CASE
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch (conv1d)");
    t_launches = (c.T > 0 ? 1 : 0) + (conv_state_out ? 1 : 0);
    t_last_error.clear();
    return SSD_OK;
}

extern "C" ssd_status ssd_conv1d_update(void* conv_state, const void* xbc, const float* weight, const float* bias,
                                        void* x, void* B, void* C, const ssd_dims* dims, int width,
                                        ssd_stream_t stream) {
    if (!dims) return fail(SSD_ERR_INVALID_ARG, "dims is NULL");
    if (dims->seqlen != 1) return fail(SSD_ERR_INVALID_ARG, "decode takes seqlen == 1 (got %lld)", (long long)dims->seqlen);
    ConvShape c;
    ssd_status s = conv_shape(dims, false, width, &c);
    if (s != SSD_OK) return s;
    if (c.nseq == 0) {
        t_launches = 0;
        t_last_error.clear();
        return SSD_OK;
    }
    if (c.nseq > 65535LL * kConvSeqs) return fail(SSD_ERR_UNSUPPORTED, "too many sequences in one decode call");
    if (!conv_state || !xbc || !weight || !x || !B || !C)
        return fail(SSD_ERR_INVALID_ARG, "conv_state, xbc, weight, x, B and C must be non-NULL");
    if (!aligned(xbc, 16) || !aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16))
        return fail(SSD_ERR_INVALID_ARG, "xbc, x, B and C must be 16-byte aligned");
    if (!aligned(weight, 16) || !aligned(bias, 16) || !aligned(conv_state, 16))
        return fail(SSD_ERR_INVALID_ARG, "weight, bias and conv_state must be 16-byte aligned");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define SSD_CONV_CASE(TT, KK) \
    if (width == KK) launch_conv_update<TT, KK>(c, conv_state, xbc, weight, bias, x, B, C, st);
    if (c.bf16) {
        SSD_CONV_CASE(__nv_bfloat16, 2) SSD_CONV_CASE(__nv_bfloat16, 3) SSD_CONV_CASE(__nv_bfloat16, 4)
    } else {
        SSD_CONV_CASE(float, 2) SSD_CONV_CASE(float, 3) SSD_CONV_CASE(float, 4)
    }
#undef SSD_CONV_CASE
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch (conv1d update)");
    t_launches = 1;
    t_last_error.clear();
    return SSD_OK;
}

// ---------------------------------------------------------------------------------
// Gated group RMSNorm (epilogue stage).
extern "C" ssd_status ssd_gated_rmsnorm(const void* y, const void* z, const float* weight, void* out, int64_t ntok,
                                        int channels, int group_size, float eps, ssd_dtype dtype,
                                        ssd_stream_t stream) {
    if (ntok < 0 || channels <= 0) return fail(SSD_ERR_INVALID_ARG, "ntok must be >= 0 and channels > 0");
    if (group_size != 256 && group_size != 512 && group_size != 1024)
        return fail(SSD_ERR_UNSUPPORTED, "group_size %d not in {256,512,1024}", group_size);
    if (channels % group_size != 0)
        return fail(SSD_ERR_UNSUPPORTED, "channels (%d) must be a multiple of group_size (%d)", channels, group_size);
    if (dtype != SSD_DTYPE_F32 && dtype != SSD_DTYPE_BF16) return fail(SSD_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (!(eps >= 0.f)) return fail(SSD_ERR_INVALID_ARG, "eps must be >= 0");
    if (ntok > 0 && (!y || !z || !weight || !out)) return fail(SSD_ERR_INVALID_ARG, "y, z, weight and out must be non-NULL");
    if (!aligned(y, 16) || !aligned(z, 16) || !aligned(weight, 16) || !aligned(out, 16))
        return fail(SSD_ERR_INVALID_ARG, "y, z, weight and out must be 16-byte aligned");
    if (ntok == 0) {
        t_launches = 0;
        t_last_error.clear();
        return SSD_OK;
    }
    const int64_t warps = (ntok + kNormTokens - 1) / kNormTokens * (channels / group_size);
    const int64_t blocks = (warps + kNormWarps - 1) / kNormWarps;
    if (blocks > INT32_MAX) return fail(SSD_ERR_UNSUPPORTED, "too many tokens in one call");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    {
        StageScope sc(ST_NORM, st);
#define SSD_NORM_CASE(TT, VV)                                                                              \
    if (group_size == 256 * VV)                                                                            \
        k_gated_rmsnorm<TT, VV><<<(unsigned)blocks, 32 * kNormWarps, 0, st>>>((const TT*)y, (const TT*)z, weight, \
                                                                           (TT*)out, ntok, channels, eps);
        if (dtype == SSD_DTYPE_BF16) {
            SSD_NORM_CASE(__nv_bfloat16, 1) SSD_NORM_CASE(__nv_bfloat16, 2) SSD_NORM_CASE(__nv_bfloat16, 4)
        } else {
            SSD_NORM_CASE(float, 1) SSD_NORM_CASE(float, 2) SSD_NORM_CASE(float, 4)
        }
#undef SSD_NORM_CASE
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch (gated rmsnorm)");
    t_launches = 1;
    t_last_error.clear();
    return SSD_OK;
}

// ---------------------------------------------------------------------------------
// Strict mode: bitwise split-invariant prefill and the chunk-emulating decode step.
namespace ssd {
namespace {

ssd_status check_cache(const ssd_chunk_cache* cc) {
    if (!cc) return fail(SSD_ERR_INVALID_ARG, "cache is NULL");
    if (!cc->state || !cc->x || !cc->B || !cc->dt || !cc->acum || !cc->len)
        return fail(SSD_ERR_INVALID_ARG, "every cache array must be non-NULL");
    if (!aligned(cc->state, 16) || !aligned(cc->x, 16) || !aligned(cc->B, 16) || !aligned(cc->dt, 4) ||
        !aligned(cc->acum, 4) || !aligned(cc->len, 4))
        return fail(SSD_ERR_INVALID_ARG, "cache state/x/B must be 16-byte aligned, dt/acum/len 4-byte");
    return SSD_OK;
}

template <typename T>
ssd_status launch_strict(const Plan& pl, char* ws, const T* x, const float* dt_raw, const float* dt_bias,
                         const float* A, const T* B, const T* C, const float* D, const int32_t* cu, T* y,
                         float* fin, const ssd_chunk_cache& cc, int resume, cudaStream_t st) {
    using namespace strict;
    auto* table = reinterpret_cast<ChunkEntry*>(ws + pl.off_table);
    auto* first = reinterpret_cast<int32_t*>(ws + pl.off_first);
    auto* count = reinterpret_cast<int32_t*>(ws + pl.off_count);
    auto* dtc = reinterpret_cast<float*>(ws + pl.off_dt);
    auto* acum = reinterpret_cast<float*>(ws + pl.off_acum);
    auto* states = reinterpret_cast<float*>(ws + pl.off_states);
    const int H = pl.H, G = pl.G, P = pl.P, N = pl.N, Q = pl.Q;
    // Headdim 64 with heads per group a multiple of 4 (the Nemotron shape) takes the
    // wide-tile chunk scan; both kernels give the same bits.
    const bool wide = P == 64 && (H / G) % 4 == 0;
    const size_t scan_smem = wide ? chunk_scan_wide_smem<T>(N, Q) : chunk_scan_smem(P, N, Q);
    void (*scan_kernel)(const T*, const T*, const T*, const float*, const float*, const float*, const float*,
                        const ChunkEntry*, const int32_t*, int, int, int, int, T*) = nullptr;
    switch (wide ? 0 : P) {
        case 0: scan_kernel = k_strict_chunk_scan_wide<T>; break;
        case 16: scan_kernel = k_strict_chunk_scan<T, 16>; break;
        case 32: scan_kernel = k_strict_chunk_scan<T, 32>; break;
        case 64: scan_kernel = k_strict_chunk_scan<T, 64>; break;
        case 128: scan_kernel = k_strict_chunk_scan<T, 128>; break;
        default: return fail(SSD_ERR_UNSUPPORTED, "headdim %d", P);
    }
    cudaError_t e = cudaFuncSetAttribute(scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)scan_smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(strict chunk scan)");
    int n = 0;
    {
        StageScope sc(ST_TABLE, st);
        k_chunk_table<<<1, kTableThreads, 0, st>>>(cu, pl.nseq, pl.T, pl.seqlen, Q, table, first, count, 0,
                                                   nullptr);
    }
    ++n;
    const unsigned mc = (unsigned)pl.max_chunks;
    if ((int64_t)mc * std::max<int64_t>(H, (int64_t)G * (Q / 32)) >= INT32_MAX)
        return fail(SSD_ERR_UNSUPPORTED, "too many chunks for one strict call (%u chunks x %d heads)", mc, H);
    if (mc > 0) {
        {
            StageScope sc(ST_STRICT_CUMSUM, st);
            k_strict_cumsum<<<dim3(mc, (H + 127) / 128), 128, 0, st>>>(dt_raw, dt_bias, A, table, count, H, Q,
                                                                       dtc, acum);
        }
        {
            StageScope sc(ST_STRICT_STATE, st);
            const unsigned grid = (unsigned)((int64_t)mc * H);
            const size_t sm = chunk_state_smem<T>(P, N, Q);
            switch (P * N / kThreads) {
#define SSD_NOUT(V)                                                                                        \
                case V: if (cudaFuncSetAttribute(k_strict_chunk_state<T, V>,                                  \
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess) \
                        return fail(SSD_ERR_CUDA, "cudaFuncSetAttribute(strict chunk state)");               \
                    k_strict_chunk_state<T, V><<<grid, kThreads, sm, st>>>(x, B, dtc, acum, table, count,     \
                                                                          H, G, P, N, Q, states);            \
                    break;
                SSD_NOUT(1) SSD_NOUT(2) SSD_NOUT(4) SSD_NOUT(8) SSD_NOUT(16) SSD_NOUT(32) SSD_NOUT(64)
#undef SSD_NOUT
                default: return fail(SSD_ERR_UNSUPPORTED, "headdim*dstate");
            }
        }
        n += 2;
    }
    {
        StageScope sc(ST_STRICT_PASSING, st);
        k_strict_passing<<<dim3(pl.nseq, H, (P * N / 4 + kThreads - 1) / kThreads), kThreads, 0, st>>>(
            states, acum, table, first, resume, cc.state, cc.len, fin, H, P * N, Q);
    }
    ++n;
    if (mc > 0) {
        StageScope sc(ST_STRICT_SCAN, st);
        scan_kernel<<<(unsigned)((int64_t)mc * G * (Q / 32)), kThreads, scan_smem, st>>>(
            x, B, C, D, dtc, acum, states, table, count, H, G, N, Q, y);
        ++n;
    }
    {
        StageScope sc(ST_STRICT_CACHE, st);
        k_strict_cache_fill<T><<<dim3(pl.nseq, H), kThreads, 0, st>>>(
            x, B, dtc, acum, table, first, H, G, P, N, Q, static_cast<T*>(cc.x), static_cast<T*>(cc.B), cc.dt,
            cc.acum, cc.len);
    }
    ++n;
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch (strict scan)");
    t_launches = n;
    return SSD_OK;
}

// Chunk-emulating decode: the step kernel, then the fold of chunks it filled.
template <typename T>
ssd_status launch_strict_decode(const Plan& pl, const ssd_chunk_cache& cc, const void* x, const float* dt_raw,
                                const float* dt_bias, const float* A, const void* B, const void* C, const float* D,
                                void* y, cudaStream_t st) {
    using namespace strict;
    const unsigned grid = (unsigned)(pl.nseq * pl.H);
    const int H = pl.H, G = pl.G, P = pl.P, N = pl.N, Q = pl.Q;
    const size_t dsm = decode_smem(H, G, N, Q);
    if (dsm > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_strict_decode<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsm);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(strict decode)");
    }
    {
        StageScope sc(ST_STRICT_UPDATE, st);
        k_strict_decode<T><<<(unsigned)(pl.nseq * pl.G), kDecThreads, dsm, st>>>(
            cc.state, static_cast<T*>(cc.x), static_cast<T*>(cc.B), cc.dt, cc.acum, cc.len, static_cast<const T*>(x),
            dt_raw, dt_bias, A, static_cast<const T*>(B), static_cast<const T*>(C), D, static_cast<T*>(y), H, G, P,
            N, Q);
    }
    {
        StageScope sc(ST_STRICT_FOLD, st);
        const size_t sm = fold_smem<T>(P, N, Q);
        // a few blocks per SM, each over a stretch of at most 32 pairs
        const int per_block = (int)std::min<int64_t>(32, std::max<int64_t>(1, ((int64_t)grid + 4 * sm_count() - 1) /
                                                                               (4 * sm_count())));
        const unsigned fold_grid = (unsigned)(((int64_t)grid + per_block - 1) / per_block);
        switch (P * N / kThreads) {
#define SSD_NOUT(V)                                                                                              \
            case V: if (cudaFuncSetAttribute(k_strict_fold<T, V>, cudaFuncAttributeMaxDynamicSharedMemorySize,   \
                                             (int)sm) != cudaSuccess)                                           \
                    return fail(SSD_ERR_CUDA, "cudaFuncSetAttribute(strict fold)");                            \
                k_strict_fold<T, V><<<fold_grid, kThreads, sm, st>>>(                                           \
                        cc.state, static_cast<const T*>(cc.x), static_cast<const T*>(cc.B), cc.dt, cc.acum, cc.len, \
                        H, G, P, N, Q, (int)grid, per_block);                                                   \
                break;
            SSD_NOUT(1) SSD_NOUT(2) SSD_NOUT(4) SSD_NOUT(8) SSD_NOUT(16) SSD_NOUT(32) SSD_NOUT(64)
#undef SSD_NOUT
            default: return fail(SSD_ERR_UNSUPPORTED, "headdim*dstate");
        }
    }
    return SSD_OK;
}

}  // namespace
}  // namespace ssd

extern "C" ssd_status ssd_strict_scan_fwd_workspace_size(const ssd_dims* dims, int chunk, size_t* bytes) {
    if (!bytes) return fail(SSD_ERR_INVALID_ARG, "bytes is NULL");
    Plan dense, packed;
    const ssd_status sd = make_plan(dims, chunk, false, &dense, 0, true);
    const ssd_status sp = make_plan(dims, chunk, true, &packed, 0, true);
    if (sd != SSD_OK && sp != SSD_OK) return sd;
    size_t b = 0;
    if (sd == SSD_OK) b = dense.bytes;
    if (sp == SSD_OK && packed.bytes > b) b = packed.bytes;
    t_last_error.clear();
    *bytes = b;
    return SSD_OK;
}

extern "C" ssd_status ssd_strict_scan_fwd(const void* x, const float* dt_raw, const float* dt_bias, const float* A,
                                          const void* B, const void* C, const float* D, const int32_t* cu_seqlens,
                                          void* y, float* final_state, const ssd_chunk_cache* cache, int resume,
                                          const ssd_dims* dims, int chunk, ssd_stream_t stream) {
    Plan pl;
    ssd_status s = make_plan(dims, chunk, cu_seqlens != nullptr, &pl, 0, true);
    if (s != SSD_OK) return s;
    s = check_cache(cache);
    if (s != SSD_OK) return s;
    if (!dt_bias || !A || !D) return fail(SSD_ERR_INVALID_ARG, "dt_bias, A and D must be non-NULL");
    if (pl.T > 0 && (!x || !dt_raw || !B || !C || !y))
        return fail(SSD_ERR_INVALID_ARG, "x, dt_raw, B, C and y must be non-NULL");
    if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(y, 16))
        return fail(SSD_ERR_INVALID_ARG, "x, B, C and y must be 16-byte aligned");
    if (!aligned(dt_raw, 4) || !aligned(dt_bias, 4) || !aligned(A, 4) || !aligned(D, 4) ||
        !aligned(final_state, 16) || !aligned(cu_seqlens, 4))
        return fail(SSD_ERR_INVALID_ARG, "float/int arrays must be 4-byte aligned, states 16-byte");
    if (resume != 0 && resume != 1) return fail(SSD_ERR_INVALID_ARG, "resume must be 0 or 1");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (pl.nseq == 0) {
        t_launches = 0;
        t_last_error.clear();
        return SSD_OK;
    }
    char* ws = static_cast<char*>(dims->workspace);
    bool owned = false;
    if (ws) {
        if (dims->workspace_bytes < pl.bytes)
            return fail(SSD_ERR_INVALID_ARG, "workspace_bytes %zu < required %zu", dims->workspace_bytes,
                        pl.bytes);
        if (!aligned(ws, 256)) return fail(SSD_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    } else {
        cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(&ws), pl.bytes, st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(workspace)");
        owned = true;
    }
    if (pl.bf16)
        s = launch_strict<__nv_bfloat16>(pl, ws, static_cast<const __nv_bfloat16*>(x), dt_raw, dt_bias, A,
                                         static_cast<const __nv_bfloat16*>(B), static_cast<const __nv_bfloat16*>(C),
                                         D, cu_seqlens, static_cast<__nv_bfloat16*>(y), final_state, *cache,
                                         resume, st);
    else
        s = launch_strict<float>(pl, ws, static_cast<const float*>(x), dt_raw, dt_bias, A,
                                 static_cast<const float*>(B), static_cast<const float*>(C), D, cu_seqlens,
                                 static_cast<float*>(y), final_state, *cache, resume, st);
    if (owned) {
        cudaError_t e = cudaFreeAsync(ws, st);
        if (e != cudaSuccess && s == SSD_OK) return cuda_fail(e, "cudaFreeAsync(workspace)");
    }
    if (s == SSD_OK) t_last_error.clear();
    return s;
}

extern "C" ssd_status ssd_strict_state_update(const ssd_chunk_cache* cache, const void* x, const float* dt_raw,
                                              const float* dt_bias, const float* A, const void* B, const void* C,
                                              const float* D, void* y, const ssd_dims* dims, int chunk,
                                              ssd_stream_t stream) {
    if (!dims) return fail(SSD_ERR_INVALID_ARG, "dims is NULL");
    ssd_dims d = *dims;
    if (d.seqlen != 1) return fail(SSD_ERR_INVALID_ARG, "decode takes seqlen == 1 (got %lld)", (long long)d.seqlen);
    Plan pl;
    ssd_status s = make_plan(&d, chunk, false, &pl, 0, true);
    if (s != SSD_OK) return s;
    if (pl.nseq == 0) {
        t_launches = 0;
        t_last_error.clear();
        return SSD_OK;
    }
    s = check_cache(cache);
    if (s != SSD_OK) return s;
    if (!x || !dt_raw || !dt_bias || !A || !B || !C || !D || !y)
        return fail(SSD_ERR_INVALID_ARG, "all decode pointers must be non-NULL");
    if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(y, 16))
        return fail(SSD_ERR_INVALID_ARG, "x, B, C and y must be 16-byte aligned");
    if (!aligned(dt_raw, 4) || !aligned(dt_bias, 4) || !aligned(A, 4) || !aligned(D, 4))
        return fail(SSD_ERR_INVALID_ARG, "float arrays must be 4-byte aligned");
    if ((int64_t)pl.nseq * pl.H >= INT32_MAX) return fail(SSD_ERR_UNSUPPORTED, "nseq*nheads too large");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (pl.bf16)
        s = launch_strict_decode<__nv_bfloat16>(pl, *cache, x, dt_raw, dt_bias, A, B, C, D, y, st);
    else
        s = launch_strict_decode<float>(pl, *cache, x, dt_raw, dt_bias, A, B, C, D, y, st);
    if (s != SSD_OK) return s;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch (strict state update)");
    t_launches = 2;
    t_last_error.clear();
    return SSD_OK;
}
