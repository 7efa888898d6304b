// spec_verify.cu -- sm_100a kernels and C ABI of libspecverify (see include/spec_verify.h).
//
// Data path (one call = one verify round over B sequences):
//
//   k_stats     streams every logit row once.  The (sequence, row, chunk) work
//               items -- a chunk is 128 threads x 8 x 16-byte vectors = 16 KB
//               (8192 bf16 or 4096 f32 elements) -- are split into contiguous
//               per-CTA ranges.  Each warp reduces its 4 KB of a chunk to one
//               statistic: online softmax (max m, sum 2^(x - m), x = l*log2e/T)
//               for the sampling entry points, (max value, lowest index) for
//               greedy.  No atomics, no fences: the next kernel in stream order
//               (a programmatic dependent) reads the statistics.
//
//   finalisation, one dependent launch per call:
//     k_chain_final_pair  chain, a cluster of two CTAs per sequence: both take
//               the decision, each stages half of the rejected row pair with
//               bulk copies and scans its residual mass; the halves meet
//               through distributed shared memory and one CTA draws.
//     k_chain_final       chain, one CTA per (sequence, slice of chunks); the
//               last to arrive (atomicAdd after __threadfence, no spin-wait)
//               draws and resets its counter.
//     k_tree_final        trees: greedy walk, target-only sibling walk, or
//               multi-step speculative sampling with draft distributions.
//   The last token is drawn by inverse CDF: the chunk holding u*S is located
//   from chunk masses, then rescanned with coalesced 8-element groups and a
//   block-wide fp64 prefix scan.
//
//   Variants on the same statistics:
//     k_filter + k_chain_final_filt     top-k / top-p filtered chain verify.
//     k_lz_*                            row-on-demand (lazy) level walk.
//     k_vp_*                            vocabulary-parallel chain verify: the
//               per-shard device steps between the callers' collectives.
//
// Nothing here is a dense contraction, so no tensor cores: the path is a
// streaming reduction bounded by HBM bandwidth, with the exp2 unit (MUFU, 16
// per clock per SM) as the secondary ceiling.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <limits.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "spec_verify.h"

namespace sv {

constexpr int NT = 128;               // threads per CTA
constexpr int NWARP = NT / 32;
constexpr int VPT = 8;                // 16-byte vectors per thread per 16 KB chunk
constexpr int SPC = NWARP;            // statistics per chunk (one per warp)
constexpr int STATS_CTAS_PER_SM = 10; // occupancy target of the statistics kernel
constexpr int SEQ_BT = 512;           // threads of the one-CTA-per-sequence finalize kernels
constexpr unsigned FULL = 0xffffffffu;
constexpr int MAXR = 256;             // max statistic rows per sequence (2*16+1 or N)
constexpr int MAXCH = SPEC_MAX_V / (NT * VPT * 4);   // max chunks per row (f32 rows)
constexpr double LOG2E = 1.4426950408889634073599246810019;

enum { MODE_CHAIN = 0, MODE_GREEDY = 1, MODE_SAMPLE = 2, MODE_MSS = 3, MODE_SAMPLE_FILT = 4,
       MODE_SAMPLE_FILT_OD = 5 };
enum { DK_NONE = 0, DK_LOGITS = 1, DK_PROBS = 2 };

template <int DT> struct Tr;
template <> struct Tr<SPEC_BF16> { static constexpr int EPV = 8; static constexpr int ESZ = 2; };
template <> struct Tr<SPEC_F32> { static constexpr int EPV = 4; static constexpr int ESZ = 4; };
template <int DT> __host__ __device__ constexpr int chunk_elems() { return NT * VPT * Tr<DT>::EPV; }

// Per-sequence state of lazy (row-on-demand) verification.
struct LazySeq {
    int cur;       // chain: last position decided; trees: current node
    int k;         // accepted draft tokens so far
    int state;     // LZ_ACTIVE, LZ_DRAW (last token still to draw), LZ_DONE, LZ_INVALID
    int nrej;      // trees: rejected children of cur
    float s;       // log2(e) / T
    float m, mq;   // combined statistics of the last decided row (chain: target, draft)
    float th;      // filtered trees: threshold of cur's row (z is then its kept mass)
    double z, zq;
};
enum { LZ_ACTIVE = 0, LZ_DRAW = 1, LZ_DONE = 2, LZ_INVALID = 3 };
constexpr int LZ_MAX_LEVELS = SPEC_MAX_DEPTH + 1;

struct Params {
    int B, V, R, nch, gamma, N, max_depth;
    int rows_tgt;                  // target rows per sequence
    int nsl;                       // chain finalisation: CTAs (slices of chunks) per sequence
    int stage_cap;                 // finalize kernels: shared bytes for a sequence's statistics
    int stage_off;                 // pair-staged chain finalisation / MSS walk: offset of the area after the stage
    const char* tgt;
    int64_t tstride;               // bytes between consecutive target rows
    const char* drf;
    int64_t dstride;               // bytes between consecutive draft rows
    const int32_t* draft_tokens;
    const int32_t* tokens;
    const int32_t* parents;
    const float* temperature;
    const float* coins;
    const float* final_u;
    const float* draft_probs;      // tree sample, nullable
    int64_t dpstride;              // bytes
    float th_single, th_acc;
    int32_t* out_tokens;
    int32_t* out_accept_index;
    int32_t* out_num_accepted;
    float* diag;
    float2* stats;                 // [B][R][nch][SPC]
    float2* stats2;                // [B][nch][NWARP]   (chain residual chunk sums)
    unsigned* cnt2;                // [B]               (chain residual arrivals)
    unsigned* status;
    unsigned wait_tries;           // polls of the first wait for a CTA's own bulk copy (0: give up at once)
    unsigned filt_mode;            // bit 0: no candidate pass in the filters; bit 1: count filtered rows by path
    // lazy (row-on-demand) verification
    struct LazySeq* lz_seq;        // [B]
    int* lz_rej;                   // [B][rej_cap]      (trees: rejected children tokens)
    int rej_cap;
    int* lz_list;                  // [2][B]            (active sequences of a level, ping-pong)
    unsigned* lz_count;            // [LZ_MAX_LEVELS + 1] (active count of each level; zero at rest)
    int level;
    // top-k / top-p filtering (chain)
    const int32_t* top_k;          // [B], nullable (0 = off)
    const float* top_p;            // [B], nullable (1 = off)
    struct FiltRec* filt;          // [B][R]            (per-row threshold and kept mass)
    double* vp_cm;                 // [B][nch]          (vocabulary-parallel: chunk masses of the shard's residual)
};

// Top-k / top-p filter of one row: keep logits >= theta; Z = the kept mass in
// units of 2^(x - m) (the row's statistics units).  on = 0: no filter (theta
// -inf, the statistics' Z applies); on = -1: invalid filter parameters.
struct FiltRec {
    float theta;
    int on;
    double Z;
};

// ----------------------------------------------------------------------------- small helpers

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Bounds checks of data-driven indices (token ids, parents, chunk indices),
// compiled in with -DSPEC_DEBUG_BOUNDS: a failed check is counted in a device
// counter (spec_debug_bounds_hits) and the access is skipped.  Without the
// flag every check is the constant true.
#ifdef SPEC_DEBUG_BOUNDS
__device__ unsigned long long g_bounds_hits;
__device__ __forceinline__ bool bounds_ok(bool c) {
    if (!c) atomicAdd(&g_bounds_hits, 1ull);
    return c;
}
#else
__device__ __forceinline__ constexpr bool bounds_ok(bool) { return true; }
#endif

// Element j of a row of V elements (a NaN, counted, when a bounds-checked
// build finds j outside [0, V)).
template <int DT> __device__ __forceinline__ float ld_elem(const char* row, int64_t j, int64_t V) {
    if (!bounds_ok(j >= 0 && j < V)) return __int_as_float(0x7fffffff);
    if constexpr (DT == SPEC_BF16) {
        unsigned short h = __ldg(reinterpret_cast<const unsigned short*>(row) + j);
        return __uint_as_float((uint32_t)h << 16);
    } else {
        return __ldg(reinterpret_cast<const float*>(row) + j);
    }
}

// One 16-byte vector starting at element e0; elements at or past V read as -inf.
template <int DT> __device__ __forceinline__ uint4 ld_vec(const char* row, int64_t e0, int V) {
    constexpr int EPV = Tr<DT>::EPV;
    if (e0 + EPV <= V) return ld_stream(row + e0 * Tr<DT>::ESZ);
    uint32_t w[4];
    if constexpr (DT == SPEC_BF16) {
        const unsigned short* h = reinterpret_cast<const unsigned short*>(row);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t lo = (e0 + 2 * i < V) ? (uint32_t)__ldg(h + e0 + 2 * i) : 0xFF80u;
            uint32_t hi = (e0 + 2 * i + 1 < V) ? (uint32_t)__ldg(h + e0 + 2 * i + 1) : 0xFF80u;
            w[i] = lo | (hi << 16);
        }
    } else {
        const uint32_t* f = reinterpret_cast<const uint32_t*>(row);
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = (e0 + i < V) ? __ldg(f + e0 + i) : 0xFF800000u;
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

template <int DT> __device__ __forceinline__ float vec_elem(const uint4& v, int i) {
    uint32_t w = (i >> (DT == SPEC_BF16 ? 1 : 0)) == 0 ? v.x
               : (i >> (DT == SPEC_BF16 ? 1 : 0)) == 1 ? v.y
               : (i >> (DT == SPEC_BF16 ? 1 : 0)) == 2 ? v.z : v.w;
    if constexpr (DT == SPEC_BF16) return __uint_as_float((i & 1) ? (w & 0xFFFF0000u) : (w << 16));
    else return __uint_as_float(w);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    return v;
}
__device__ __forceinline__ float nanf_() { return __int_as_float(0x7fffffff); }

__host__ __device__ __forceinline__ bool temperature_ok(float T) {
    return T >= 1.17549435e-38f && T <= 3.40282347e38f;   // false for NaN
}
__device__ __forceinline__ float scale_of(float T) { return (float)(LOG2E / (double)T); }

__device__ __forceinline__ float2 ldcg2(const float2* p) { return __ldcg(p); }

// Programmatic dependent launch: the statistics kernel lets the finalize
// kernel be scheduled early; the finalize kernel waits for the statistics
// kernel's completion (and memory) before reading anything it wrote.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// mbarrier and 1-D bulk copy (TMA) helpers, used to stage a row pair in
// shared memory.  Waits are bounded: WAIT_LIMIT tries and WAIT_NS.
constexpr unsigned WAIT_LIMIT = 1u << 24;
constexpr unsigned long long WAIT_NS = 1000000000ull;
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(uint32_t a, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(a), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t a, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}" : "=r"(ok) : "r"(a), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// At most `tries` polls (0: give up at once, without polling) and WAIT_NS.
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity, unsigned tries = WAIT_LIMIT) {
    if (tries == 0) return false;
    if (mbar_try(a, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (unsigned i = 0; i < tries; ++i) {
        if (mbar_try(a, parity)) return true;
        if (global_ns() - t0 > WAIT_NS) break;
    }
    return false;
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t a, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(a), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t mbar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(dst), "l"(src), "r"(bytes), "r"(mbar) : "memory");
}

// A first bounded wait for a CTA's own bulk copy gave up: record it; if the
// second (full-budget) wait that lets the copy land gave up too, record that
// the copy may still have been writing this CTA's shared memory when the CTA
// went on.
__device__ __forceinline__ void copy_timed_out(const Params& P, bool landed) {
    atomicOr(P.status, (1u << SPEC_ERR_TIMEOUT) | (landed ? 0u : (1u << SPEC_ERR_COPY_IN_FLIGHT)));
}

// Stage sequence b's statistics block (R rows of nch*SPC float2, contiguous)
// in shared memory with one bulk copy when it fits in `cap` bytes; returns
// where to read it (shared memory, or global memory when it does not fit or
// the bounded wait ran out).  All threads of the CTA must call it.
__device__ const float2* stage_stats(const Params& P, int b, int R, unsigned char* buf, size_t cap,
                                     uint64_t* bar) {
    const size_t bytes = (size_t)R * P.nch * SPC * sizeof(float2);
    const float2* src = P.stats + (size_t)b * P.R * P.nch * SPC;
    if (bytes > cap || buf == nullptr) return src;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(bar), 1);
        mbar_expect_tx(smem_u32(bar), (uint32_t)bytes);
        bulk_g2s(smem_u32(buf), src, (uint32_t)bytes, smem_u32(bar));
    }
    __syncthreads();
    if (__syncthreads_and(mbar_wait(smem_u32(bar), 0, P.wait_tries)))
        return reinterpret_cast<const float2*>(buf);
    // the copy did not land in time (for some thread): report, let it land
    // (bounded), read global memory
    const bool landed = __syncthreads_and(mbar_wait(smem_u32(bar), 0)) != 0;
    if (threadIdx.x == 0) copy_timed_out(P, landed);
    return src;
}

__device__ __forceinline__ void flag_input_error(const Params& P) {
    atomicOr(P.status, 1u << SPEC_ERR_DEVICE_INPUT);
}

// Block-wide exclusive scan of one double per thread (BT threads); *total
// receives the sum.
template <int BT>
__device__ double block_excl_scan(double v, double* total) {
    constexpr int BW = BT / 32;
    __shared__ double wsum[BW];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    double inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        double n = __shfl_up_sync(FULL, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    double before = 0.0, tot = 0.0;
#pragma unroll
    for (int w = 0; w < BW; ++w) {
        if (w < warp) before += wsum[w];
        tot += wsum[w];
    }
    __syncthreads();
    *total = tot;
    return before + inc - v;
}

// ----------------------------------------------------------------------------- row-chunk statistics

// Sum of N values as a balanced binary tree (fully unrolled).
template <int N>
__device__ __forceinline__ float tree_sum(const float* a) {
    if constexpr (N == 1) return a[0];
    else return tree_sum<N / 2>(a) + tree_sum<N - N / 2>(a + N / 2);
}

// 2^(a - b) in fp64 (the rescaling of a statistic to another maximum).  Not
// inlined: the fp64 exp2 needs many registers, and the callers (one call per
// statistic) are kernels that run at high occupancy.
__device__ __noinline__ double ex2d(float a, float b) { return exp2((double)a - (double)b); }

// Per-thread online-softmax partial of NV 16-byte vectors held in registers:
// (max x, sum 2^(x - max)), x = l * s.  `bad` is set by a NaN or +inf.
template <int DT, int NV>
__device__ __forceinline__ void thread_softmax_regs(const uint4 (&v)[NV], float s, float& mt, float& st,
                                                    bool& bad) {
    constexpr int EPV = Tr<DT>::EPV;
    float lmax;
    bool b = false;
    if constexpr (DT == SPEC_BF16) {
        __nv_bfloat162 mx = *reinterpret_cast<const __nv_bfloat162*>(&v[0].x);
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[k]);
#pragma unroll
            for (int i = 0; i < 4; ++i) mx = __hmax2_nan(mx, h[i]);
        }
        float a = __low2float(mx), c = __high2float(mx);
        b = (a != a) || (c != c);
        lmax = fmaxf(a, c);
    } else {
        lmax = -INFINITY;
#pragma unroll
        for (int k = 0; k < NV; ++k)
#pragma unroll
            for (int i = 0; i < EPV; ++i) {
                float x = vec_elem<DT>(v[k], i);
                b |= (x != x);
                lmax = fmaxf(lmax, x);
            }
    }
    b |= (lmax == INFINITY);
    mt = -INFINITY;
    st = 0.f;
    if (!b && lmax != -INFINITY) {
        mt = lmax * s;
        const float nm = -mt;
        // pairwise: each vector's terms, then the vectors' sums, as balanced
        // trees (at most log2(NV * EPV) roundings on any term)
        float vs[NV];
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            float e[EPV];
#pragma unroll
            for (int i = 0; i < EPV; ++i) e[i] = ex2(fmaf(vec_elem<DT>(v[k], i), s, nm));
            vs[k] = tree_sum<EPV>(e);
        }
        st = tree_sum<NV>(vs);
    }
    bad |= b;
}

// NV 16-byte vectors of a row starting at element e_base (thread tid takes
// vectors k*NT + tid); elements at or past V read as -inf.
template <int DT, int NV>
__device__ __forceinline__ void load_vecs(const char* row, int V, int64_t e_base, uint4 (&v)[NV]) {
    constexpr int EPV = Tr<DT>::EPV;
#pragma unroll
    for (int k = 0; k < NV; ++k) v[k] = ld_vec<DT>(row, e_base + (int64_t)(k * NT + threadIdx.x) * EPV, V);
}

template <int DT, int NV>
__device__ __forceinline__ void thread_softmax(const char* row, int V, int64_t e_base, float s,
                                               float& mt, float& st, bool& bad) {
    uint4 v[NV];
    load_vecs<DT, NV>(row, V, e_base, v);
    thread_softmax_regs<DT, NV>(v, s, mt, st, bad);
}

// Warp combination of per-thread softmax partials into the warp's statistic.
__device__ __forceinline__ float2 warp_softmax_stat(float mt, float st, bool bad) {
    const float mw = warp_max(mt);
    const bool anybad = __any_sync(FULL, bad);
    const double contrib = (mt == -INFINITY) ? 0.0 : (double)(st * ex2(mt - mw));
    float sw = (float)warp_sum_d(contrib);
    if (anybad) sw = nanf_();
    return make_float2(mw, sw);
}

// Online-softmax statistic of chunk c of a row, CH elements per chunk (the
// target's chunking; rows of another dtype are split into as many 16-byte
// vectors as that takes).  Per warp: (max x, sum 2^(x - max)); NaN sum for a
// row holding a NaN or +inf.
template <int DT, int CH>
__device__ __forceinline__ float2 chunk_softmax(const char* row, int V, int c, float s) {
    constexpr int EPV = Tr<DT>::EPV;
    constexpr int NVT = CH / (NT * EPV);          // vectors per thread for this dtype
    constexpr int NV = NVT < VPT ? NVT : VPT;
    constexpr int NSUB = NVT / NV;
    static_assert(NV * NSUB * NT * EPV == CH, "chunk geometry");
    float mt, st;
    bool bad = false;
    thread_softmax<DT, NV>(row, V, (int64_t)c * CH, s, mt, st, bad);
#pragma unroll
    for (int sub = 1; sub < NSUB; ++sub) {
        float m2, s2;
        thread_softmax<DT, NV>(row, V, (int64_t)c * CH + (int64_t)sub * NV * NT * EPV, s, m2, s2, bad);
        const float m = fmaxf(mt, m2);
        if (m > -INFINITY)
            st = (float)((mt > -INFINITY ? (double)st * ex2d(mt, m) : 0.0) +
                         (m2 > -INFINITY ? (double)s2 * ex2d(m2, m) : 0.0));
        mt = m;
    }
    return warp_softmax_stat(mt, st, bad);
}

// (max value, lowest index) per warp of one chunk held in registers (vector
// k of thread tid starts at element c*CH + (k*NT + tid)*EPV); value NaN if any
// NaN was seen.
template <int DT>
__device__ __forceinline__ float2 argmax_regs(const uint4 (&v)[VPT], int c) {
    constexpr int EPV = Tr<DT>::EPV, CH = chunk_elems<DT>();
    const int tid = threadIdx.x;
    float best = -INFINITY;
    int bestk = 0;
    uint4 bw = v[0];
    bool bad = false;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        float mk;
        if constexpr (DT == SPEC_BF16) {
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[k]);
            __nv_bfloat162 m2 = __hmax2_nan(__hmax2_nan(h[0], h[1]), __hmax2_nan(h[2], h[3]));
            float a = __low2float(m2), b = __high2float(m2);
            bad |= (a != a) || (b != b);
            mk = fmaxf(a, b);
        } else {
            mk = -INFINITY;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float x = vec_elem<DT>(v[k], i);
                bad |= (x != x);
                mk = fmaxf(mk, x);
            }
        }
        if (mk > best) { best = mk; bestk = k; bw = v[k]; }
    }
    int j = EPV - 1;
#pragma unroll
    for (int i = EPV - 1; i >= 0; --i)
        if (vec_elem<DT>(bw, i) == best) j = i;
    int idx = c * CH + (bestk * NT + tid) * EPV + j;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        float ov = __shfl_xor_sync(FULL, best, o);
        int oi = __shfl_xor_sync(FULL, idx, o);
        if (ov > best || (ov == best && oi < idx)) { best = ov; idx = oi; }
    }
    if (__any_sync(FULL, bad)) best = nanf_();
    return make_float2(best, __int_as_float(idx));
}

template <int DT>
__device__ __forceinline__ float2 chunk_argmax(const char* row, int V, int c) {
    uint4 v[VPT];
    load_vecs<DT, VPT>(row, V, (int64_t)c * chunk_elems<DT>(), v);
    return argmax_regs<DT>(v, c);
}

// ============================================================================= top-k / top-p filtering
//
// The filtered target distribution keeps the logits >= theta: theta_k = the
// top_k-th largest logit (ties kept), then, within that set, theta_p = the
// largest logit whose set {l >= theta_p} carries a top_p share of the set's
// mass; p'(v) = 2^(x_v - m) / Z' on the kept set.  Thresholds are found over
// order-preserving keys of the logits (-0 folded onto +0).  bf16 rows: the
// candidates near the row's maximum first (cfilter_row), else the whole row's
// value histogram (vh_build / vh_select, 1024 threads) or windowed histogram
// (wfilter_row); f32 rows (and a bf16 row whose histogram counter would wrap):
// a radix descent of 12 + 12 + 8 bit digits (filter_row).  Counts decide
// top-k; masses are fixed point (2^-40 units, integer sums, so they do not
// depend on the order of the additions) and decide top-p and Z'.

constexpr int FILT_BT = 1024;
constexpr int FILT_BT_BF16 = 256;                 // filter CTAs of launches whose filtered rows are all bf16
constexpr double FIX_ONE = 1099511627776.0;      // 2^40

template <int DT> __device__ __forceinline__ uint32_t order_key(float v) {
    uint32_t b = __float_as_uint(v);
    if (b == 0x80000000u) b = 0u;                                   // -0 sorts with +0
    const uint32_t k = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return DT == SPEC_BF16 ? (k >> 16) : k;
}
template <int DT> __device__ __forceinline__ float key_value(uint32_t k) {
    if constexpr (DT == SPEC_BF16) {
        const uint32_t b = (k & 0x8000u) ? (k & 0x7FFFu) : (~k & 0xFFFFu);
        return __uint_as_float(b << 16);
    } else {
        return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
    }
}

// Digits of the order keys, most significant first: 12 + 4 bits for bf16,
// 12 + 12 + 8 for f32.  The wide first digit (sign, exponent and the top
// mantissa bits) spreads a row's values over many buckets, so the shared
// histogram updates rarely collide.
template <int DT> struct FiltDigits;
template <> struct FiltDigits<SPEC_BF16> {
    static constexpr int NL = 2;
    __host__ __device__ static constexpr int width(int l) { return l == 0 ? 12 : 4; }
    __host__ __device__ static constexpr int shift(int l) { return l == 0 ? 4 : 0; }
};
template <> struct FiltDigits<SPEC_F32> {
    static constexpr int NL = 3;
    __host__ __device__ static constexpr int width(int l) { return l == 2 ? 8 : 12; }
    __host__ __device__ static constexpr int shift(int l) { return l == 0 ? 20 : (l == 1 ? 8 : 0); }
};
// Shared bytes of the per-level histograms (counts u32 + masses u64 per bucket).
template <int DT> __host__ __device__ constexpr size_t filt_hist_bytes() {
    size_t n = 0;
    for (int l = 0; l < FiltDigits<DT>::NL; ++l) n += ((size_t)1 << FiltDigits<DT>::width(l)) * 12;
    return n;
}

struct FiltShared {
    unsigned long long red[FILT_BT / 32];
    unsigned redc[FILT_BT / 32];
    unsigned long long at, above, tm;
    unsigned tc;
    int sel;
};

// Level l's histograms inside the dynamic area.
template <int DT> struct FiltHist {
    unsigned char* base;
    __device__ unsigned long long* mass(int l) const {
        size_t off = 0;
        for (int k = 0; k < l; ++k) off += ((size_t)1 << FiltDigits<DT>::width(k)) * 12;
        return reinterpret_cast<unsigned long long*>(base + off);
    }
    __device__ unsigned* cnt(int l) const {
        return reinterpret_cast<unsigned*>(mass(l) + ((size_t)1 << FiltDigits<DT>::width(l)));
    }
};

// One pass over a row: histograms of digit `level` (counts and fixed-point
// masses of 2^(x s - m)) of the keys whose higher digits equal `prefix` (all
// keys at level 0).  Integer atomics: the sums do not depend on their order.
template <int DT>
__device__ void filt_pass(const char* row, int V, float s, float m, int level, uint32_t prefix, const FiltHist<DT>& h) {
    using D = FiltDigits<DT>;
    constexpr int EPV = Tr<DT>::EPV;
    const int nb = 1 << D::width(level), sh = D::shift(level);
    const int psh = sh + D::width(level);
    unsigned* cnt = h.cnt(level);
    unsigned long long* mass = h.mass(level);
    for (int d = threadIdx.x; d < nb; d += FILT_BT) { cnt[d] = 0u; mass[d] = 0ull; }
    __syncthreads();
    const int nv = (V + EPV - 1) / EPV;
    for (int vi = threadIdx.x; vi < nv; vi += FILT_BT) {
        const uint4 v = ld_vec<DT>(row, (int64_t)vi * EPV, V);
#pragma unroll
        for (int i = 0; i < EPV; ++i) {
            if (vi * EPV + i >= V) break;
            const float x = vec_elem<DT>(v, i);
            const uint32_t key = order_key<DT>(x);
            if (level > 0 && (key >> psh) != prefix) continue;
            const uint32_t d = (key >> sh) & (uint32_t)(nb - 1);
            atomicAdd(&cnt[d], 1u);
            atomicAdd(&mass[d], (unsigned long long)(ex2(fmaf(x, s, -m)) * (float)FIX_ONE));
        }
    }
    __syncthreads();
}

// Scan buckets [dlo, nb) from the top for the first bucket d whose running
// total base + (buckets above d) + w[d] reaches target; every thread owns a
// run of buckets, a block-wide u64 scan gives each run its start.  Returns d,
// or -1 when the range never reaches the target.  fs.above = base + the
// buckets of the range strictly above d (the whole range when -1), fs.at =
// fs.above + w[d].  All threads call it.
template <class T>
__device__ int filt_scan(const T* w, int nb, int dlo, unsigned long long base, double target, FiltShared& fs) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = nb - dlo;
    const int per = (n + FILT_BT - 1) / FILT_BT;
    const int hi = nb - tid * per, lo = max(dlo, hi - per);     // buckets [lo, hi), this thread's run
    unsigned long long own = 0ull;
    for (int d = hi - 1; d >= lo; --d) own += (unsigned long long)w[d];
    unsigned long long inc = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long v = __shfl_up_sync(FULL, inc, o);
        if (lane >= o) inc += v;
    }
    if (lane == 31) fs.red[warp] = inc;
    if (tid == 0) fs.sel = -1;
    __syncthreads();
    unsigned long long excl = base;
    for (int k = 0; k < warp; ++k) excl += fs.red[k];
    excl += inc - own;
    if (hi > lo && (double)excl < target && (double)(excl + own) >= target) {
        unsigned long long cum = excl;
        for (int d = hi - 1; d >= lo; --d) {
            if ((double)(cum + (unsigned long long)w[d]) >= target) {
                fs.sel = d;
                fs.above = cum;
                fs.at = cum + (unsigned long long)w[d];
                break;
            }
            cum += (unsigned long long)w[d];
        }
    }
    __syncthreads();
    const int d = fs.sel;
    if (d < 0 && tid == 0) {
        unsigned long long t = base;
        for (int k = 0; k < FILT_BT / 32; ++k) t += fs.red[k];
        fs.above = t;
        fs.at = t;
    }
    __syncthreads();
    return d;
}

// The mass the top-p share is taken of, in fixed-point units: the kept mass
// of top-k (exact), or with top-k off the row's mass from its statistics
// (zrow, fp64 across chunks, ~2e-7 relative) -- with top_p capped below
// 1 - 2^-20 so that the target stays under the exact total; both differences
// lie inside the oracle's 1e-6 flag on top-p decisions.
__device__ __forceinline__ double top_p_target(bool use_k, float Pp, unsigned long long zk, double zrow) {
    return use_k ? (double)Pp * (double)zk : fmin((double)Pp, 1.0 - 9.5367431640625e-07) * zrow * FIX_ONE;
}

// Threshold and kept mass of one row (one CTA).
//  top-k: walk the digits of the top_k-th largest key (filt_scan over the
//    counts, one pass per digit); every pass keeps the masses, so the mass of
//    the kept set {key >= path} is the masses strictly above the path at
//    each level plus the path's key.
//  top-p: within the kept set, scan from the top -- the buckets strictly
//    above the path at each level, then the path's key -- for the bucket
//    where the mass reaches top_p * (kept mass); a whole key ends the search,
//    another bucket is refined digit by digit with more passes (every key in
//    it lies above the top-k key).
//  top-p alone: one pass of the first digit over every key; the crossing
//    bucket is refined the same way.
template <int DT>
__device__ FiltRec filter_row(const char* row, int V, float s, float m, double zrow, int K, float Pp, FiltShared& fs,
                              const FiltHist<DT>& h) {
    using D = FiltDigits<DT>;
    constexpr int NL = D::NL;
    FiltRec r{-INFINITY, 0, 0.0};
    const bool use_k = K > 0 && K < V, use_p = Pp < 1.f;
    if (!use_k && !use_p) return r;
    int path[NL];
    uint32_t prefix = 0;
    unsigned long long cabove = 0ull, mabove = 0ull;           // counts / masses strictly above the path
    const int nl = use_k ? NL : 1;
    for (int level = 0; level < nl; ++level) {
        filt_pass<DT>(row, V, s, m, level, prefix, h);
        const int nb = 1 << D::width(level);
        if (use_k) {
            path[level] = filt_scan(h.cnt(level), nb, 0, cabove, (double)K, fs);
            cabove = fs.above;
        } else {
            path[level] = 0;                                   // top-p alone: every key is kept
        }
        filt_scan(h.mass(level), nb, path[level] + 1, 0ull, INFINITY, fs);   // masses above the path digit
        mabove += fs.above;
        prefix = (prefix << D::width(level)) | (uint32_t)path[level];
    }
    const unsigned long long mk = mabove + h.mass(nl - 1)[path[nl - 1]];
    uint32_t key = prefix;
    unsigned long long z = mk;
    if (use_p) {
        const double target = top_p_target(use_k, Pp, mk, zrow);
        unsigned long long base = 0ull;
        int cl = -1, cd = 0;
        for (int l = 0; l < nl && cl < 0; ++l) {                // buckets strictly above the path digit
            const int d = filt_scan(h.mass(l), 1 << D::width(l), path[l] + 1, base, target, fs);
            if (d >= 0) { cl = l; cd = d; z = fs.at; }
            base = fs.above;
        }
        if (cl < 0) {                                          // the path's own bucket
            cl = nl - 1;
            cd = path[nl - 1];
            z = base + h.mass(cl)[cd];
        }
        uint32_t pre = 0;
        for (int l = 0; l < cl; ++l) pre = (pre << D::width(l)) | (uint32_t)path[l];
        pre = (pre << D::width(cl)) | (uint32_t)cd;
        if (!(use_k && cl == NL - 1)) {                        // not a whole key: refine
            for (int level = cl + 1; level < NL; ++level) {
                filt_pass<DT>(row, V, s, m, level, pre, h);
                int d = filt_scan(h.mass(level), 1 << D::width(level), 0, base, target, fs);
                if (d < 0) d = 0;                              // rounding only
                base = fs.above;
                z = fs.at;
                pre = (pre << D::width(level)) | (uint32_t)d;
            }
        }
        key = pre;
    }
    r.theta = key_value<DT>(key);
    r.on = 1;
    r.Z = (double)z / FIX_ONE;
    return r;
}

// Order keys of the two bf16 values packed in x (low half = lower index), as
// order_key does for one value: -0 folded onto +0, negative values
// complemented, the sign bit of the others set.
__device__ __forceinline__ uint32_t vh_keys2(uint32_t x) {
    x &= ~__vcmpeq2(x, 0x80008000u);
    return x ^ ((((x >> 15) & 0x00010001u) * 0xFFFFu) | 0x80008000u);
}


// bf16 rows: an exact histogram of the row's values (65536 order keys, two
// 16-bit counters per 32-bit word, 128 KB of shared memory) from one pass;
// every mass then follows exactly as count * fixed(2^(v s - m)) per value,
// the same fixed-point numbers the radix path adds element by element.
// (The windowed filter below forms the same numbers in 52 KB for callers
// that cannot hold 192 KB.)
//
// A row has at most V distinct values, so most of the 32768 words are empty.
// Thread t reads the 32 words of key block 1023 - t (16-byte loads, the four
// quads of a block stored XOR-swizzled by the block index so that eight
// consecutive threads hit eight distinct bank groups), and a block-wide scan
// packs the indices of the non-empty words into a list in descending key
// order.  The counts and masses are then summed over equal slices of that
// list, so the exp2 work is spread evenly whatever the values' spread, and
// one more scan orders the slices: the top-k key is where the running count
// reaches top_k, the top-p key where the running mass reaches top_p times the
// mass kept by top-k.
constexpr int VH_WORDS = 32768;
constexpr size_t VH_BYTES = (size_t)VH_WORDS * 4 + (size_t)VH_WORDS * 2;   // counters + word list

// Physical word of logical word i (= key >> 1): block i >> 5, quad
// ((i >> 2) & 7) ^ (block & 7), lane i & 3.
__device__ __forceinline__ uint32_t vh_phys(uint32_t i) { return i ^ ((i >> 3) & 0x1Cu); }

__device__ __forceinline__ void vh_count1(uint32_t* w, uint32_t k) {
    atomicAdd(&w[vh_phys(k >> 1)], (k & 1u) ? 0x10000u : 1u);
}
__device__ __forceinline__ unsigned long long vh_mass(unsigned c, uint32_t k, float s, float m) {
    if (c == 0u) return 0ull;
    return (unsigned long long)c *
           (unsigned long long)(ex2(fmaf(key_value<SPEC_BF16>(k), s, -m)) * (float)FIX_ONE);
}

// Exclusive block-wide scan, in thread order, of a u32 and a u64; the totals
// go to *ta / *tb.  All threads call it.
__device__ void vh_scan2(unsigned a, unsigned long long b, unsigned* ea, unsigned long long* eb, unsigned* ta,
                         unsigned long long* tb, FiltShared& fs) {
    static_assert(FILT_BT == 1024, "one warp scans the 32 warp totals");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned ia = a;
    unsigned long long ib = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned va = __shfl_up_sync(FULL, ia, o);
        const unsigned long long vb = __shfl_up_sync(FULL, ib, o);
        if (lane >= o) { ia += va; ib += vb; }
    }
    if (lane == 31) { fs.redc[warp] = ia; fs.red[warp] = ib; }
    __syncthreads();
    if (warp == 0) {
        const unsigned xa = fs.redc[lane];
        const unsigned long long xb = fs.red[lane];
        unsigned sa = xa;
        unsigned long long sb = xb;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned va = __shfl_up_sync(FULL, sa, o);
            const unsigned long long vb = __shfl_up_sync(FULL, sb, o);
            if (lane >= o) { sa += va; sb += vb; }
        }
        fs.redc[lane] = sa - xa;
        fs.red[lane] = sb - xb;
        if (lane == 31) { fs.tc = sa; fs.tm = sb; }
    }
    __syncthreads();
    *ea = fs.redc[warp] + ia - a;
    *eb = fs.red[warp] + ib - b;
    *ta = fs.tc;
    *tb = fs.tm;
    __syncthreads();                                   // fs is free again
}

// The value histogram of a bf16 row and its list of non-empty words (from the
// logits alone, before the statistics are needed).  Returns the list length.
// All threads call it.
__device__ int vh_build(const char* row, int V, FiltShared& fs, uint32_t* w) {
    const int tid = threadIdx.x;
    uint4* w4 = reinterpret_cast<uint4*>(w);
    unsigned short* list = reinterpret_cast<unsigned short*>(w + VH_WORDS);
    // histogram: four 16-byte loads per thread in flight (the first four
    // while the counters are cleared), then the updates
    const int nv = (V + 7) / 8;
    uint4 v[4];
    auto load4 = [&](int v0) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int vi = v0 + q * FILT_BT;
            v[q] = vi < nv ? ld_vec<SPEC_BF16>(row, (int64_t)vi * 8, V) : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    load4(tid);
    for (int i = tid; i < VH_WORDS / 4; i += FILT_BT) w4[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    for (int v0 = tid;;) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int vi = v0 + q * FILT_BT;
            if (vi >= nv) break;
            const uint32_t xs[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
            const int lim = V - vi * 8;                   // elements of this vector inside the row
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t k2 = vh_keys2(xs[c]);
                if (2 * c < lim) vh_count1(w, k2 & 0xFFFFu);
                if (2 * c + 1 < lim) vh_count1(w, k2 >> 16);
            }
        }
        v0 += 4 * FILT_BT;
        if (v0 >= nv) break;
        load4(v0);
    }
    __syncthreads();
    // non-empty words of this thread's block, highest first
    const uint32_t blk = (uint32_t)(VH_WORDS / 32 - 1 - tid);
    uint32_t mask = 0u;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint4 x = w4[blk * 8 + (q ^ (blk & 7u))];
        mask |= (x.x ? 1u : 0u) << (4 * q) | (x.y ? 1u : 0u) << (4 * q + 1) | (x.z ? 1u : 0u) << (4 * q + 2) |
                (x.w ? 1u : 0u) << (4 * q + 3);
    }
    unsigned off, n;
    unsigned long long d0, d1;
    vh_scan2((unsigned)__popc(mask), 0ull, &off, &d0, &n, &d1, fs);
    while (mask) {
        const int j = 31 - __clz(mask);
        list[off++] = (unsigned short)(blk * 32 + j);
        mask &= ~(1u << j);
    }
    __syncthreads();
    return (int)n;
}

// Threshold and kept mass of a bf16 row from its value histogram and word
// list (vh_build).  Returns false when a value occurs 65536 times or more (a
// 16-bit counter wrapped: possible only for V > 65535); the caller then takes
// the radix path.  All threads call it.
__device__ bool vh_select(int V, int n, float s, float m, double zrow, int K, float Pp, FiltShared& fs,
                          const uint32_t* w, FiltRec* out) {
    const int tid = threadIdx.x;
    const unsigned short* list = reinterpret_cast<const unsigned short*>(w + VH_WORDS);
    // counts and masses of this thread's slice of the list
    const int e0 = (int)((long long)n * tid / FILT_BT), e1 = (int)((long long)n * (tid + 1) / FILT_BT);
    unsigned cs = 0u;
    unsigned long long ms = 0ull;
    for (int e = e0; e < e1; ++e) {
        const uint32_t i = list[e];
        const uint32_t x = w[vh_phys(i)];
        cs += (x >> 16) + (x & 0xFFFFu);
        ms += vh_mass(x >> 16, 2 * i + 1, s, m) + vh_mass(x & 0xFFFFu, 2 * i, s, m);
    }
    unsigned c0, ctot;
    unsigned long long m0, mtot;
    vh_scan2(cs, ms, &c0, &m0, &ctot, &mtot, fs);
    if (V > 65535 && ctot != (unsigned)V) return false;   // a counter wrapped (the same in every thread)
    const bool use_k = K > 0 && K < V, use_p = Pp < 1.f;
    // top-k: the first key (from the top) where the running count reaches K
    if (tid == 0) { fs.sel = 0; fs.at = mtot; }          // top-p alone: every key is kept
    __syncthreads();
    if (use_k && c0 < (unsigned)K && c0 + cs >= (unsigned)K) {
        unsigned c = c0;
        unsigned long long mm = m0;
        for (int e = e0; e < e1; ++e) {
            const uint32_t i = list[e];
            const uint32_t x = w[vh_phys(i)];
            const unsigned ch = x >> 16, cl = x & 0xFFFFu;
            c += ch;
            mm += vh_mass(ch, 2 * i + 1, s, m);
            if (c >= (unsigned)K) { fs.sel = (int)(2 * i + 1); fs.at = mm; break; }
            c += cl;
            mm += vh_mass(cl, 2 * i, s, m);
            if (c >= (unsigned)K) { fs.sel = (int)(2 * i); fs.at = mm; break; }
        }
    }
    __syncthreads();
    uint32_t t = (uint32_t)fs.sel;
    const unsigned long long zk = fs.at;
    unsigned long long z = zk;
    if (use_p) {
        // the first key where the running mass reaches top_p of the kept mass
        // (a key >= the top-k key, since the running mass there is zk); with
        // top-k off the kept mass is the row's, as wfilter_row takes it
        const double target = top_p_target(use_k, Pp, zk, zrow);
        __syncthreads();
        if (tid == 0) fs.sel = -1;
        __syncthreads();
        if ((double)m0 < target && (double)(m0 + ms) >= target) {
            unsigned long long mm = m0;
            for (int e = e0; e < e1; ++e) {
                const uint32_t i = list[e];
                const uint32_t x = w[vh_phys(i)];
                mm += vh_mass(x >> 16, 2 * i + 1, s, m);
                if ((double)mm >= target) { fs.sel = (int)(2 * i + 1); fs.at = mm; break; }
                mm += vh_mass(x & 0xFFFFu, 2 * i, s, m);
                if ((double)mm >= target) { fs.sel = (int)(2 * i); fs.at = mm; break; }
            }
        }
        __syncthreads();
        if (fs.sel >= 0) {
            t = (uint32_t)fs.sel;
            z = fs.at;
        }
    }
    out->theta = key_value<SPEC_BF16>(t);
    out->on = 1;
    out->Z = (double)z / FIX_ONE;
    return true;
}

// bf16 rows, two passes and a sparse window.
//  1. a count histogram of the order keys' top 12 bits (4096 buckets of 16
//     keys) over the whole row;
//  2. from it, per bucket, bounds on its mass (count times the fixed-point
//     mass of its lowest and highest key, with a relative slack far above
//     the exp2 unit's ulp); scanned from the top, the bounds give a bucket at
//     or below both thresholds: the top-k bucket (counts are exact) and the
//     first bucket whose lower-bound running mass reaches top_p times the
//     upper bound of the kept mass;
//  3. a second pass counts, per key, only the elements of the non-empty
//     buckets from the top down to that bucket (16 counters per non-empty
//     bucket, in descending key order).
// Every key's mass is count * fixed(2^(v s - m)), so the running counts and
// masses from the top, the top-k key and the kept mass are exact integers,
// independent of the order of the additions.  With top-k off the mass the
// top-p share is taken of is the whole row's, zrow (the row statistics' sum,
// fp64 across chunks, relative error ~2e-7): top-p decisions that close to a
// boundary are the near-ties the oracle flags.  A window needing more than
// WF_SLOTS counters is counted in segments, one more pass each.
constexpr int WF_NB = 4096;                       // coarse buckets (key >> 4)
constexpr int WF_SLOTS = 7168;                    // per-key counters of the window (a segment)
constexpr size_t WF_BYTES = (size_t)WF_NB * 4 + (size_t)WF_NB * 2 + (size_t)WF_SLOTS * 4;   // 52 KB

struct WinShared {
    unsigned long long red[32];
    double rlo[32], rhi[32];
    unsigned redc[32];
    unsigned long long tm, acc;
    double tlo, thi, dv;
    unsigned tc;
    int pos_k, pos_p, nord, sel;
    unsigned long long at;
};

__device__ __forceinline__ unsigned long long fix_mass(float x, float s, float m) {
    return (unsigned long long)(ex2(fmaf(x, s, -m)) * (float)FIX_ONE);
}
// The same mass as a double, for bounds only (exponent clamped: a bucket's
// top key may lie above the row's maximum).
__device__ __forceinline__ double bound_mass(float x, float s, float m) {
    return (double)ex2(fminf(fmaf(x, s, -m), 60.f)) * FIX_ONE;
}

// Block-wide exclusive scan, in thread order, of a u32 and a u64 (BT / 32 <=
// 32 warps); totals to *ta / *tb.  All threads call it.
template <int BT>
__device__ void wf_scan2(unsigned a, unsigned long long b, unsigned* ea, unsigned long long* eb, unsigned* ta,
                         unsigned long long* tb, WinShared& ws) {
    constexpr int NW = BT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned ia = a;
    unsigned long long ib = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned va = __shfl_up_sync(FULL, ia, o);
        const unsigned long long vb = __shfl_up_sync(FULL, ib, o);
        if (lane >= o) { ia += va; ib += vb; }
    }
    if (lane == 31) { ws.redc[warp] = ia; ws.red[warp] = ib; }
    __syncthreads();
    if (warp == 0) {
        const unsigned xa = lane < NW ? ws.redc[lane] : 0u;
        const unsigned long long xb = lane < NW ? ws.red[lane] : 0ull;
        unsigned sa = xa;
        unsigned long long sb = xb;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned va = __shfl_up_sync(FULL, sa, o);
            const unsigned long long vb = __shfl_up_sync(FULL, sb, o);
            if (lane >= o) { sa += va; sb += vb; }
        }
        if (lane < NW) { ws.redc[lane] = sa - xa; ws.red[lane] = sb - xb; }
        if (lane == 31) { ws.tc = sa; ws.tm = sb; }
    }
    __syncthreads();
    *ea = ws.redc[warp] + ia - a;
    *eb = ws.red[warp] + ib - b;
    *ta = ws.tc;
    *tb = ws.tm;
    __syncthreads();
}

// Block-wide exclusive scan, in thread order, of a u32 and two doubles (the
// bucket counts and mass bounds); totals to *tc, *tl, *th.
template <int BT>
__device__ void wf_scan3(unsigned c, double l, double h, unsigned* ec, double* el, double* eh, unsigned* tc,
                         double* tl, double* th, WinShared& ws) {
    constexpr int NW = BT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned ic = c;
    double il = l, ih = h;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned vc = __shfl_up_sync(FULL, ic, o);
        const double vl = __shfl_up_sync(FULL, il, o), vh = __shfl_up_sync(FULL, ih, o);
        if (lane >= o) { ic += vc; il += vl; ih += vh; }
    }
    if (lane == 31) { ws.redc[warp] = ic; ws.rlo[warp] = il; ws.rhi[warp] = ih; }
    __syncthreads();
    if (warp == 0) {
        const unsigned xc = lane < NW ? ws.redc[lane] : 0u;
        const double xl = lane < NW ? ws.rlo[lane] : 0.0, xh = lane < NW ? ws.rhi[lane] : 0.0;
        unsigned sc = xc;
        double sl = xl, sh = xh;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned vc = __shfl_up_sync(FULL, sc, o);
            const double vl = __shfl_up_sync(FULL, sl, o), vh = __shfl_up_sync(FULL, sh, o);
            if (lane >= o) { sc += vc; sl += vl; sh += vh; }
        }
        if (lane < NW) { ws.redc[lane] = sc - xc; ws.rlo[lane] = sl - xl; ws.rhi[lane] = sh - xh; }
        if (lane == 31) { ws.tc = sc; ws.tlo = sl; ws.thi = sh; }
    }
    __syncthreads();
    *ec = ws.redc[warp] + ic - c;
    *el = ws.rlo[warp] + il - l;
    *eh = ws.rhi[warp] + ih - h;
    *tc = ws.tc;
    *tl = ws.tlo;
    *th = ws.thi;
    __syncthreads();
}

// Calls f(key) for every element of a bf16 row (BT threads, WF_NV 16-byte
// loads in flight per thread: one CTA per row streams it alone).
constexpr int WF_NV = 8;
template <int BT, class F>
__device__ __forceinline__ void wf_each_key(const char* row, int V, F f) {
    const int nv = (V + 7) / 8;
    for (int v0 = threadIdx.x; v0 < nv; v0 += WF_NV * BT) {
        uint4 v[WF_NV];
#pragma unroll
        for (int q = 0; q < WF_NV; ++q) {
            const int vi = v0 + q * BT;
            v[q] = vi < nv ? ld_vec<SPEC_BF16>(row, (int64_t)vi * 8, V) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int q = 0; q < WF_NV; ++q) {
            const int vi = v0 + q * BT;
            if (vi >= nv) break;
            const uint32_t xs[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
            const int lim = V - vi * 8;
            if (lim >= 8) {                               // a whole vector inside the row
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t k2 = vh_keys2(xs[c]);
                    f(k2 & 0xFFFFu);
                    f(k2 >> 16);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t k2 = vh_keys2(xs[c]);
                    if (2 * c < lim) f(k2 & 0xFFFFu);
                    if (2 * c + 1 < lim) f(k2 >> 16);
                }
            }
        }
    }
}

// Threshold and kept mass of one bf16 row (the record filter_row gives).
// smem: WF_BYTES of shared memory.  All threads call it.
template <int BT>
__device__ FiltRec wfilter_row(const char* row, int V, float s, float m, double zrow, int K, float Pp,
                               unsigned char* smem, WinShared& ws) {
    constexpr int RB = WF_NB / BT;                    // coarse buckets per thread (descending positions)
    constexpr int RS = WF_SLOTS / BT;                 // window counters per thread
    static_assert(RB * BT == WF_NB && RS * BT == WF_SLOTS, "split");
    const int tid = threadIdx.x;
    FiltRec r{-INFINITY, 0, 0.0};
    const bool use_k = K > 0 && K < V, use_p = Pp < 1.f;
    if (!use_k && !use_p) return r;
    uint32_t* coarse = reinterpret_cast<uint32_t*>(smem);                        // pass 1 counts
    int32_t* sbase = reinterpret_cast<int32_t*>(smem);                           // bucket -> its keys' first counter
                                                                                 // + 15 (reuses coarse)
    unsigned short* bucket_of = reinterpret_cast<unsigned short*>(smem + (size_t)WF_NB * 4);  // ordinal -> bucket
    uint32_t* slots = reinterpret_cast<uint32_t*>(smem + (size_t)WF_NB * 6);
    // ---- pass 1: coarse counts
    for (int i = tid; i < WF_NB / 4; i += BT) reinterpret_cast<uint4*>(coarse)[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    wf_each_key<BT>(row, V, [&](uint32_t k) { atomicAdd(&coarse[k >> 4], 1u); });
    __syncthreads();
    // ---- choose the window: positions p = 0.. from the top bucket down
    const int p0 = tid * RB;
    unsigned cnt[RB];
    unsigned rc = 0u;
    double rl = 0.0, rh = 0.0;
    constexpr double LO = 1.0 - 1e-5, HI = 1.0 + 1e-5;      // slack over the exp2 unit's rounding
#pragma unroll
    for (int j = 0; j < RB; ++j) {
        const uint32_t b = (uint32_t)(WF_NB - 1 - (p0 + j));
        cnt[j] = coarse[b];
        if (cnt[j]) {
            rc += cnt[j];
            rl += (double)cnt[j] * bound_mass(key_value<SPEC_BF16>(b << 4), s, m) * LO;
            rh += (double)cnt[j] * bound_mass(key_value<SPEC_BF16>((b << 4) | 15u), s, m) * HI;
        }
    }
    unsigned c0, ctot;
    double l0, h0, ltot, htot;
    wf_scan3<BT>(rc, rl, rh, &c0, &l0, &h0, &ctot, &ltot, &htot, ws);
    const double zfix = zrow * FIX_ONE;                 // the row's mass in fixed-point units
    if (tid == 0) { ws.pos_k = -1; ws.pos_p = WF_NB - 1; ws.dv = zfix; }
    __syncthreads();
    if (use_k && c0 < (unsigned)K && c0 + rc >= (unsigned)K) {     // the top-k bucket (exact counts)
        unsigned c = c0;
        double h = h0;
#pragma unroll
        for (int j = 0; j < RB; ++j) {
            c += cnt[j];
            if (cnt[j]) {
                const uint32_t b = (uint32_t)(WF_NB - 1 - (p0 + j));
                h += (double)cnt[j] * bound_mass(key_value<SPEC_BF16>((b << 4) | 15u), s, m) * HI;
            }
            if (c >= (unsigned)K) { ws.pos_k = p0 + j; ws.dv = h; break; }
        }
    }
    __syncthreads();
    const int pos_k = ws.pos_k;
    // top_p of an upper bound of the kept mass (only used with top-k off)
    const double target_hi = top_p_target(false, Pp, 0ull, zrow) * HI;
    __syncthreads();
    if (use_p && l0 < target_hi && l0 + rl >= target_hi) {
        double l = l0;
#pragma unroll
        for (int j = 0; j < RB; ++j) {
            if (cnt[j]) {
                const uint32_t b = (uint32_t)(WF_NB - 1 - (p0 + j));
                l += (double)cnt[j] * bound_mass(key_value<SPEC_BF16>(b << 4), s, m) * LO;
            }
            if (l >= target_hi) { ws.pos_p = p0 + j; break; }
        }
    }
    __syncthreads();
    // window: positions [0, nb) -- down to the top-k bucket (the top-p key lies
    // at or above the top-k key), else down to the top-p bound
    const int nb = use_k ? pos_k + 1 : ws.pos_p + 1;
    // ---- ordinals of the window's non-empty buckets, in descending order
    unsigned ne = 0u;
#pragma unroll
    for (int j = 0; j < RB; ++j) ne += (p0 + j < nb && cnt[j]) ? 1u : 0u;
    unsigned o0, otot;
    unsigned long long d0, d1;
    wf_scan2<BT>(ne, 0ull, &o0, &d0, &otot, &d1, ws);      // (after its barriers nobody reads coarse)
    {
        unsigned o = o0;
#pragma unroll
        for (int j = 0; j < RB; ++j) {
            const uint32_t b = (uint32_t)(WF_NB - 1 - (p0 + j));
            if (p0 + j < nb && cnt[j]) {
                sbase[b] = (int32_t)(o * 16u + 15u);     // key k of b counts at sbase[b] - (k & 15)
                bucket_of[o] = (unsigned short)b;
                ++o;
            } else {
                sbase[b] = INT_MIN / 2;                  // outside the window: never a valid counter
            }
        }
    }
    __syncthreads();
    const int nslot = (int)otot * 16;
    // ---- pass 2, per segment of WF_SLOTS counters: per-key counts, exact totals
    bool rk = !use_k, rp = !use_p;
    uint32_t tk = 0x007Fu, tp = 0x007Fu;             // -inf: keep everything (never left so)
    unsigned cb = 0u;                                  // count of the keys above this segment
    unsigned long long mb = 0ull, zk = 0ull, z = 0ull;
    for (int seg = 0; seg * WF_SLOTS < max(nslot, 1) && !(rk && rp); ++seg) {
        const int slo = seg * WF_SLOTS, used = min(WF_SLOTS, nslot - slo);
        for (int i = tid; i < (used + 3) / 4; i += BT) reinterpret_cast<uint4*>(slots)[i] = make_uint4(0u, 0u, 0u, 0u);
        __syncthreads();
        wf_each_key<BT>(row, V, [&](uint32_t k) {
            const int sl = sbase[k >> 4] - (int)(k & 15u) - slo;
            if ((unsigned)sl < (unsigned)used) atomicAdd(&slots[sl], 1u);
        });
        __syncthreads();
        // this segment's keys in descending order: thread runs of RS counters
        const int s0 = tid * RS;
        unsigned sc = 0u;
        unsigned long long sm = 0ull;
        for (int j = 0; j < RS && s0 + j < used; ++j) {
            const unsigned c = slots[s0 + j];
            if (c) {
                const int g = slo + s0 + j;
                const uint32_t key = ((uint32_t)bucket_of[g >> 4] << 4) | (uint32_t)(15 - (g & 15));
                sc += c;
                sm += (unsigned long long)c * fix_mass(key_value<SPEC_BF16>(key), s, m);
            }
        }
        unsigned e0, etot;
        unsigned long long f0, ftot;
        wf_scan2<BT>(sc, sm, &e0, &f0, &etot, &ftot, ws);
        e0 += cb;
        f0 += mb;
        auto find = [&](bool by_count, double target) {   // the thread whose run crosses the target
            if (tid == 0) ws.sel = -1;
            __syncthreads();
            const bool cross = by_count ? (e0 < (unsigned)K && e0 + sc >= (unsigned)K)
                                        : ((double)f0 < target && (double)(f0 + sm) >= target);
            if (cross) {
                unsigned c = e0;
                unsigned long long mm = f0;
                for (int j = 0; j < RS && s0 + j < used; ++j) {
                    const unsigned cj = slots[s0 + j];
                    if (!cj) continue;
                    const int g = slo + s0 + j;
                    const uint32_t key = ((uint32_t)bucket_of[g >> 4] << 4) | (uint32_t)(15 - (g & 15));
                    c += cj;
                    mm += (unsigned long long)cj * fix_mass(key_value<SPEC_BF16>(key), s, m);
                    if (by_count ? c >= (unsigned)K : (double)mm >= target) {
                        ws.sel = (int)key;
                        ws.at = mm;
                        break;
                    }
                }
            }
            __syncthreads();
        };
        if (!rk && cb + etot >= (unsigned)K) {               // the top-k key lies in this segment
            find(true, 0.0);
            tk = (uint32_t)ws.sel;
            zk = ws.at;
            rk = true;
            __syncthreads();
        }
        if (rk && !rp) {
            const double target = top_p_target(use_k, Pp, zk, zrow);
            if (seg > 0 && (double)mb >= target) {
                // the top-p key lies above this segment (the top-k key, which
                // sets the target, was found only here): count the segments
                // again from the top for it
                cb = 0u;
                mb = 0ull;
                seg = -1;
                continue;
            }
            if ((double)(mb + ftot) >= target) {            // the top-p key lies in this segment
                find(false, target);
                tp = (uint32_t)ws.sel;
                z = ws.at;
                rp = true;
                __syncthreads();
            }
        }
        cb += etot;
        mb += ftot;
    }
    if (!use_p) { tp = tk; z = zk; }
    r.theta = key_value<SPEC_BF16>(tp);
    r.on = 1;
    r.Z = (double)z / FIX_ONE;
    return r;
}

// bf16 rows, candidates first.  A cut x_c = (m - D) / s, D log2 units below
// the row's maximum (see CfCut; with top-p alone, never more than when the whole row's mass
// bound V * 2^(x s - m) already proves the top-p key lies above it), rounded
// down to a bf16 value.  The candidates' order keys lie in [key(x_c),
// key(max)], both known from the statistics before the row is read: that
// window of per-key counters -- without the keys of the tiny values |v| <
// 2^-10 inside it, which a cut below zero would otherwise bring in by the
// tens of thousands of (mostly absent) keys; those few values are counted
// together, with their exact fixed-point mass -- is cleared, and one pass
// over the row counts every value >= x_c into it (bf16 pair compares make a
// survivor mask per 16-byte vector; a warp stages the survivors of a pass
// step and counts them with whole-warp 32-bit shared atomics, at the position
// a 512-entry table of key groups gives).  The window is then scanned from its top as the
// value histogram scans its keys -- count and fixed-point mass count *
// fixed(2^(v s - m)) per key, a block scan, the thread whose run crosses
// top_k or the top-p target walks it -- so the record is the same integers
// and the same keys.  The window holds every value >= x_c, so the record is
// exact unless the crossing falls among the tiny values: with top-k, the
// top-p key lies at or above the top-k key; with top-p alone, the window's
// mass must reach the top-p target.  A cut that holds fewer than top_k values
// or too little mass is deepened by 6 log2 units, twice (the row is read again,
// mostly from L2); otherwise, or when the window would outgrow the shared
// memory, the function returns false and the caller takes a whole-row path.
// First cut, log2 units below the maximum: 12 where many rows share the SMs
// (fewer candidates, more rows deepened), 14 where one row's latency is the
// walk's.  (Scaling the top-k cut as 1 / T was measured: fewer rows deepened
// on workload 6, but many more candidates on workload 8's T = 0.8 rows.)
struct CfCut { float d; };
constexpr CfCut CF_MANY{12.f}, CF_ONE{14.f};
constexpr float CF_DEEPER = 6.f;                  // a cut too shallow goes 6 log2 units deeper, twice
constexpr float CF_TINY = 9.765625e-04f;          // 2^-10 (a whole number of key groups either side of 0)
constexpr int CF_TINY_G = INT_MIN / 2;            // group table: a group of tiny values
struct CfShared {
    WinShared ws;                                 // block scans
    unsigned tiny, over;
    int sel, tz;
    unsigned long long at, tinym;
    int gbase[512];                               // key group (key >> 7) -> window position of its key 0
};
constexpr size_t CF_HEAD = ((sizeof(CfShared) + 127) / 128) * 128;
constexpr int CF_STG = 256;                       // staged survivors per warp and pass step
enum { CF_OK = 0, CF_SHORT = 1, CF_FAIL = 2 };

// 16-byte loads in flight per thread and step: 64 KB per SM (four 256-thread
// CTAs, or one CTA of 512 or 1024 threads).
template <int BT> __host__ __device__ constexpr int cf_nv() { return BT == 512 ? 8 : 4; }
// A row's first step of loads, issued before the statistics are waited for
// (the logits do not depend on them); have: this thread's step lies inside
// the row's whole vectors.
template <int BT> struct CfPre {
    uint4 v[cf_nv<BT>()];
    bool have;
};
template <int BT> __device__ __forceinline__ void cf_prefetch(const char* row, int V, CfPre<BT>& pre) {
    constexpr int NV = cf_nv<BT>();
    pre.have = (int)threadIdx.x + (NV - 1) * BT < V / 8;
    if (pre.have) {
#pragma unroll
        for (int q = 0; q < NV; ++q) pre.v[q] = ld_stream(row + (size_t)(threadIdx.x + q * BT) * 16);
    }
}

// One cut at D log2 units: CF_OK (record in *out), CF_SHORT (the cut holds
// too few values or too little mass: a deeper cut may hold the answer) or
// CF_FAIL.  All threads call it.
template <int BT>
__device__ __forceinline__ int cf_attempt(const char* row, int V, float s, float m, double zrow, int K, float Pp,
                                          float D, unsigned char* smem, size_t bytes, FiltRec* out,
                                          const CfPre<BT>* pre) {
    CfShared& cs = *reinterpret_cast<CfShared*>(smem);
    unsigned* win = reinterpret_cast<unsigned*>(smem + CF_HEAD);
    // the end of the shared memory: each warp's survivor staging (CF_STG values)
    const size_t stg_off = (bytes - (size_t)(BT / 32) * CF_STG * sizeof(unsigned short)) & ~(size_t)15;
    unsigned short* stg = reinterpret_cast<unsigned short*>(smem + stg_off) + (threadIdx.x >> 5) * CF_STG;
    const unsigned wmax = (unsigned)min((size_t)16384, ((stg_off - CF_HEAD) / 4) & ~(size_t)3);
    const int tid = threadIdx.x, lane = tid & 31;
    const bool use_k = K > 0 && K < V, use_p = Pp < 1.f;
    const __nv_bfloat16 tb = __float2bfloat16_rd((m - D) / s);
    const float xc = __bfloat162float(tb);
    if (!(xc > -INFINITY)) return CF_FAIL;            // (a cut at -inf would count the row's padding)
    const __nv_bfloat162 t2 = __halves2bfloat162(tb, tb);
    // the window: keys [klo, khi] less the tiny keys [g0, g1] inside it
    const uint32_t klo = order_key<SPEC_BF16>(xc);
    const uint32_t khi = order_key<SPEC_BF16>(__bfloat162float(__float2bfloat16_ru(m / s))) + 1u;
    const uint32_t g0 = max(order_key<SPEC_BF16>(-CF_TINY) + 1u, klo);
    const uint32_t g1 = min(order_key<SPEC_BF16>(CF_TINY) - 1u, khi);
    const uint32_t glen = g0 <= g1 ? g1 - g0 + 1u : 0u;
    if (khi < klo || khi - klo + 1u - glen > wmax) return CF_FAIL;
    const unsigned W = khi - klo + 1u - glen;
    for (unsigned i = tid; i < (W + 3u) / 4u; i += BT) reinterpret_cast<uint4*>(win)[i] = make_uint4(0u, 0u, 0u, 0u);
    // window position of key k = gbase[k >> 7] + (k & 127); outside [0, W):
    // not in the window (a tiny group is marked)
    for (int g = tid; g < 512; g += BT) {
        const uint32_t k0 = (uint32_t)g << 7;
        cs.gbase[g] = (glen && k0 >= g0 && k0 <= g1) ? CF_TINY_G
                                                     : (int)k0 - (int)klo - ((glen && k0 > g1) ? (int)glen : 0);
    }
    if (tid == 0) { cs.tiny = 0u; cs.over = 0u; cs.tinym = 0ull; cs.tz = 0; }
    __syncthreads();
    auto count = [&](uint32_t u) {                  // one bf16 value (raw bits) >= x_c
        u = u == 0x8000u ? 0u : u;                    // -0 counts as +0
        const uint32_t k = u ^ (((u >> 15) * 0x7FFFu) | 0x8000u);
        const int b = cs.gbase[k >> 7];
        const int sl = b + (int)(k & 127u);
        if ((unsigned)sl < W) {
            atomicAdd(&win[sl], 1u);
        } else if (b == CF_TINY_G) {
            atomicAdd(&cs.tiny, 1u);
            atomicAdd(&cs.tinym, fix_mass(key_value<SPEC_BF16>(k), s, m));
        } else {
            cs.over = 1u;
        }
    };
    // survivor mask of one 16-byte vector: bit c for the low value of pair c,
    // bit 16 + c for the high one
    auto smask = [&](const uint4& vq) {
        const uint32_t xs[4] = {vq.x, vq.y, vq.z, vq.w};
        unsigned bits = 0u;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            __nv_bfloat162 h;
            memcpy(&h, &xs[c], 4);
            bits |= (__hge2_mask(h, t2) & 0x10001u) << c;
        }
        return bits;
    };
    auto svalue = [](const uint4& vq, int p) {       // the raw bits of survivor p of vq
        const int c = p & 3;
        const uint32_t w = c < 2 ? (c == 0 ? vq.x : vq.y) : (c == 2 ? vq.z : vq.w);
        return p >= 16 ? (w >> 16) : (w & 0xFFFFu);
    };
    auto survivors = [&](const uint4& vq) {
        unsigned bits = smask(vq);
        while (bits) {
            const int p = __ffs(bits) - 1;
            bits &= bits - 1u;
            count(svalue(vq, p));
        }
    };
    // One step's vectors of a converged warp: the lanes' survivors are staged
    // in the warp's slice (a warp prefix sum of their counts gives each lane
    // its place) and counted by the whole warp, so a step costs about one
    // shared atomic instruction per 32 survivors instead of one per vector.
    // A step with more than CF_STG survivors counts vector by vector.
    auto step_survivors = [&](const uint4 (&vs)[cf_nv<BT>()]) {
        constexpr int NV = cf_nv<BT>();
        if (__activemask() != FULL) {
#pragma unroll
            for (int q = 0; q < NV; ++q) survivors(vs[q]);
            return;
        }
        int c = 0;
#pragma unroll
        for (int q = 0; q < NV; ++q) c += __popc(smask(vs[q]));
        if (!__any_sync(FULL, c > 0)) return;
        int inc = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(FULL, inc, o);
            if (lane >= o) inc += n;
        }
        const int total = __shfl_sync(FULL, inc, 31);
        if (total > CF_STG) {
#pragma unroll
            for (int q = 0; q < NV; ++q) survivors(vs[q]);
            return;
        }
        int at = inc - c;
#pragma unroll
        for (int q = 0; q < NV; ++q) {
            unsigned bits = smask(vs[q]);
            while (bits) {
                const int p = __ffs(bits) - 1;
                bits &= bits - 1u;
                stg[at++] = (unsigned short)svalue(vs[q], p);
            }
        }
        __syncwarp();
        for (int j = lane; j < total; j += 32) count(stg[j]);
        __syncwarp();                                 // the slice is read before the next step writes it
    };
    // ---- one pass: the values >= x_c.  Per 16-byte vector the four pair
    // compares make a survivor mask (bit c: the low value of pair c, bit
    // 16 + c: the high one); each lane then counts only its own survivors.
    // The next step's loads are issued before this step's vectors are
    // examined, so the examination hides under the memory latency.
    constexpr int CF_NV = cf_nv<BT>();
    const int nfull = V / 8, nv = (V + 7) / 8;      // whole vectors; with the ragged tail
    int v0 = tid;
    if (v0 + (CF_NV - 1) * BT < nfull) {
        uint4 a[CF_NV], b[CF_NV];
        if (pre && pre->have) {
#pragma unroll
            for (int q = 0; q < CF_NV; ++q) a[q] = pre->v[q];
        } else {
#pragma unroll
            for (int q = 0; q < CF_NV; ++q) a[q] = ld_stream(row + (size_t)(v0 + q * BT) * 16);
        }
        for (;;) {
            const int v1 = v0 + CF_NV * BT;
            const bool more = v1 + (CF_NV - 1) * BT < nfull;
            if (more) {
#pragma unroll
                for (int q = 0; q < CF_NV; ++q) b[q] = ld_stream(row + (size_t)(v1 + q * BT) * 16);
            }
            step_survivors(a);
            v0 = v1;
            if (!more) break;
#pragma unroll
            for (int q = 0; q < CF_NV; ++q) a[q] = b[q];
        }
    }
    for (; v0 < nv; v0 += BT) survivors(ld_vec<SPEC_BF16>(row, (int64_t)v0 * 8, V));   // (past V: -inf)
    __syncthreads();
    if (cs.over) {                                    // (the statistics' maximum disagrees with the row)
        __syncthreads();
        return CF_FAIL;
    }
    const unsigned tinyc = cs.tiny;
    const unsigned long long tinym = cs.tinym;
    // ---- the window from its top: thread t takes positions [t * per, (t + 1) * per);
    // the tiny values come just before position pl (the first key below them)
    auto key_at = [&](unsigned p) -> uint32_t {      // key of position p from the top
        const uint32_t w = W - 1u - p;
        return (glen && klo + w >= g0) ? klo + w + glen : klo + w;
    };
    const unsigned pl = glen ? W - (g0 - klo) : W;
    const unsigned per = (W + BT - 1) / BT;
    const unsigned p0 = min(W, tid * per), p1 = min(W, p0 + per);
    const bool own_tiny = tinyc && p0 < p1 && ((pl >= p0 && pl < p1) || (pl == W && p1 == W));
    unsigned sc = own_tiny ? tinyc : 0u;
    unsigned long long sm = own_tiny ? tinym : 0ull;
    {
        unsigned p = p0;
        for (; p + 4u <= p1; p += 4u) {                // four counters read before any is used
            unsigned c4[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) c4[j] = win[W - 1u - (p + j)];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (c4[j]) {
                    sc += c4[j];
                    sm += (unsigned long long)c4[j] * fix_mass(key_value<SPEC_BF16>(key_at(p + j)), s, m);
                }
        }
        for (; p < p1; ++p) {
            const unsigned c = win[W - 1u - p];
            if (c) {
                sc += c;
                sm += (unsigned long long)c * fix_mass(key_value<SPEC_BF16>(key_at(p)), s, m);
            }
        }
    }
    unsigned c0, ctot;
    unsigned long long m0, mtot;
    wf_scan2<BT>(sc, sm, &c0, &m0, &ctot, &mtot, cs.ws);
    // the thread whose run crosses the count K (by_count) or the mass target;
    // a crossing inside the tiny values sets cs.tz.  The first barrier keeps
    // thread 0 from resetting cs.sel before every thread has read the
    // previous search's result: the outcome must be the same in every thread
    // (it decides which barriers they reach next).
    auto find = [&](bool by_count, double target) {
        __syncthreads();
        if (tid == 0) cs.sel = -1;
        __syncthreads();
        const bool cross = by_count ? (c0 < (unsigned)K && c0 + sc >= (unsigned)K)
                                    : ((double)m0 < target && (double)(m0 + sm) >= target);
        if (cross) {
            unsigned c = c0;
            unsigned long long mm = m0;
            auto hit = [&]() { return by_count ? c >= (unsigned)K : (double)mm >= target; };
            bool done = false;
            for (unsigned p = p0; p < p1 && !done; ++p) {
                if (own_tiny && p == pl) {
                    c += tinyc;
                    mm += tinym;
                    if (hit()) { cs.tz = 1; done = true; break; }
                }
                const unsigned cj = win[W - 1u - p];
                if (!cj) continue;
                const uint32_t k = key_at(p);
                c += cj;
                mm += (unsigned long long)cj * fix_mass(key_value<SPEC_BF16>(k), s, m);
                if (hit()) {
                    cs.sel = (int)k;
                    cs.at = mm;
                    done = true;
                }
            }
            if (!done && own_tiny && pl == W) cs.tz = 1;   // the tiny values close the window
        }
        __syncthreads();
    };
    int key = -1, st = CF_OK;
    unsigned long long z = 0ull;
    if (use_k) {
        find(true, 0.0);
        key = cs.sel;
        z = cs.at;
        st = cs.tz ? CF_FAIL : key < 0 ? CF_SHORT : CF_OK;
    }
    if (use_p && st == CF_OK) {
        // with top-k the top-p key lies at or above the top-k key (the running
        // mass there is the kept mass)
        find(false, top_p_target(use_k, Pp, z, zrow));
        key = cs.sel;
        z = cs.at;
        st = cs.tz ? CF_FAIL : key < 0 ? CF_SHORT : CF_OK;
    }
    __syncthreads();                                  // cs is read; the shared memory is free again
    if (st == CF_OK) {
        out->theta = key_value<SPEC_BF16>((uint32_t)key);
        out->on = 1;
        out->Z = (double)z / FIX_ONE;
    }
    return st;
}

// Rows with at most this many statistics entries get the top-k cut below.
constexpr int CF_SEG_MAX = 256;

// A cut that holds the top-k crossing, from the row's statistics: entry e is
// fl(x_max * s) over the elements of one warp of one chunk, so the K-th
// largest entry m_K belongs to K distinct elements, each >= m_K / s up to the
// rounding of the product, and at least K values lie at or above a cut just
// below m_K / s.  Returns that cut in log2 units below m (the margin covers
// the product's rounding and the cut's own arithmetic), or +inf when m_K is
// -inf.  E <= CF_SEG_MAX entries at st; smem: the candidate filter's shared
// memory, whose window is not in use yet.  All threads call it.
template <int BT>
__device__ float cf_topk_cut(const float2* st, int E, int K, float m, unsigned char* smem) {
    float* v = reinterpret_cast<float*>(smem + CF_HEAD);
    float* res = v + CF_SEG_MAX;
    for (int i = threadIdx.x; i < E; i += BT) v[i] = st[i].x;
    if (threadIdx.x == 0) *res = -INFINITY;
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += BT) {       // rank of entry i, ties by index
        const float x = v[i];
        int rank = 0;
        for (int j = 0; j < E; ++j) {
            const float y = v[j];
            rank += (y > x || (y == x && j < i)) ? 1 : 0;
        }
        if (rank == K - 1) *res = x;
    }
    __syncthreads();
    const float mk = *res;
    __syncthreads();                                  // the window's memory is free again
    if (!(mk > -INFINITY)) return INFINITY;
    return (m - mk) + 0.015625f + fabsf(mk) * 1.52587890625e-05f;
}

// Threshold and kept mass of one bf16 row from its candidates (see above):
// 1 (first cut) or 2 (deeper cut) with the record in *out; 0: the caller
// takes a whole-row path.  sts: the row's E statistics entries.  smem: `bytes`
// of shared memory (up to 16384 window counters).  All threads call it.
template <int BT>
__device__ int cfilter_row(const char* row, int V, float s, float m, double zrow, int K, float Pp,
                            const float2* sts, int E, unsigned char* smem, size_t bytes, FiltRec* out,
                            const CfPre<BT>* pre, CfCut cut) {
    float D = cut.d, Dsure = INFINITY;
    if (!(K > 0 && K < V)) {                          // top-p alone: the row's mass bound, factor-2 slack
        const double rest = zrow - top_p_target(false, Pp, 0ull, zrow) / FIX_ONE;
        if (rest > 0.0) D = fminf(D, log2f((float)(2.0 * V / rest)));
    } else if (K <= E && E <= CF_SEG_MAX) {           // top-k: a cut that surely holds K values
        Dsure = cf_topk_cut<BT>(sts, E, K, m, smem);
        D = fminf(D, Dsure);
    }
    int st = cf_attempt<BT>(row, V, s, m, zrow, K, Pp, D, smem, bytes, out, pre);
    if (st != CF_SHORT) return st == CF_OK ? 1 : 0;
    for (int i = 0; i < 2 && st == CF_SHORT; ++i) {
        D = fminf(Dsure, D + CF_DEEPER);
        st = cf_attempt<BT>(row, V, s, m, zrow, K, Pp, D, smem, bytes, out, (const CfPre<BT>*)nullptr);
    }
    return st == CF_OK ? 2 : 0;
}

// Rows the candidates resolved at the first cut ([0]) or at the deeper one
// ([2]) and rows left to a whole-row path ([1]), counted only when the caller
// asks (spec_debug_filter_path).
__device__ unsigned long long g_filter_rows[3];

// cfilter_row unless the caller switched the candidate pass off; counts the
// outcome when asked.  st: the row's statistics (P.nch * SPC entries).
template <int BT>
__device__ __forceinline__ bool cand_filter(const Params& P, const char* row, const float2* st, float s, float m,
                                            double z, int K, float Pp, unsigned char* smem, size_t bytes,
                                            FiltRec* out, const CfPre<BT>* pre = nullptr, CfCut cut = CF_ONE) {
    const int how = (P.filt_mode & 1u)
                        ? 0
                        : cfilter_row<BT>(row, P.V, s, m, z, K, Pp, st, P.nch * SPC, smem, bytes, out, pre, cut);
    if ((P.filt_mode & 2u) && threadIdx.x == 0) atomicAdd(&g_filter_rows[how == 0 ? 1 : how == 1 ? 0 : 2], 1ull);
    return how != 0;
}

// ----------------------------------------------------------------------------- finaliser pieces

struct FinShared {
    float m[MAXR];
    double z[MAXR];
    int bad[MAXR];
    int par[SPEC_MAX_NODES];
    int tok[SPEC_MAX_NODES];
    double pch[SPEC_MAX_NODES];
    int rej[SPEC_MAX_NODES];
    double M[MAXCH];
    float wp[MAXCH][NWARP];
    uint32_t bitmap[(NT * VPT * 8) / 32];
    float th[MAXR];
    int ivals[8];
    double dvals[4];
};

// Combine the per-warp softmax statistics of rows [0, R) into (m, Z, bad).
// `blk` is sequence b's statistics block ([R][nch][SPC]), in shared memory
// when staged, else in global memory (written by the previous kernel).
// One row's statistics (E entries at st) combined by one warp: max m and sum
// Z (fp64) in every lane; returns whether the row is unusable (NaN/+inf
// logit, all -inf, Z not positive and finite).
__device__ __forceinline__ bool warp_combine(const float2* st, int E, float& m_out, double& z_out) {
    const int lane = threadIdx.x & 31;
    {
        // one pass: each lane keeps an online (max, sum) over its entries
        float m = -INFINITY;
        double z = 0.0;
        bool bad = false;
#pragma unroll 4
        for (int e = lane; e < E; e += 32) {
            const float2 x = st[e];
            bad |= (x.y != x.y);
            if (x.x > m) {
                z = (m > -INFINITY ? z * ex2d(m, x.x) : 0.0) + (double)x.y;
                m = x.x;
            } else if (x.x > -INFINITY) {
                z += (double)x.y * ex2d(x.x, m);
            }
        }
        const float mw = warp_max(m);
        bad = __any_sync(FULL, bad);
        double zw = (m > -INFINITY && mw < INFINITY) ? z * ex2d(m, mw) : 0.0;
        zw = warp_sum_d(zw);
        m_out = mw;
        z_out = zw;
        return bad || !(mw > -INFINITY) || !(mw < INFINITY) || !(zw > 0.0) || !(zw < 1e300);
    }
}

// warp_combine of one row into sh slot `slot` (written by lane 0).
__device__ __forceinline__ void combine_row(const float2* st, int E, FinShared& sh, int slot) {
    float m;
    double z;
    const bool bad = warp_combine(st, E, m, z);
    if ((threadIdx.x & 31) == 0) {
        sh.m[slot] = m;
        sh.z[slot] = z;
        sh.bad[slot] = bad;
    }
}

template <int BT>
__device__ void combine_softmax_rows(const Params& P, const float2* blk, int R, FinShared& sh) {
    const int warp = threadIdx.x >> 5;
    const int E = P.nch * SPC;
    for (int r = warp; r < R; r += BT / 32) combine_row(blk + (size_t)r * E, E, sh, r);
}

// p(x) of one element, fp64 exp2, in the units of the row statistics.
__device__ __forceinline__ double prob_d(float l, float s, float m, double z) {
    return exp2((double)l * (double)s - (double)m) / z;
}

// Eight consecutive elements e0..e0+7 of a row (e0 a multiple of 8) as f32;
// elements at or past V read as `fill`.
template <int DT> __device__ __forceinline__ void ld8(const char* row, int64_t e0, int V, float fill,
                                                      float (&x)[8]) {
    if constexpr (DT == SPEC_BF16) {
        if (e0 + 8 <= V) {
            uint4 v = ld_stream(row + e0 * 2);
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = vec_elem<DT>(v, i);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = (e0 + i < V) ? ld_elem<DT>(row, e0 + i, V) : fill;
        }
    } else {
        if (e0 + 8 <= V) {
            uint4 a = ld_stream(row + e0 * 4), b = ld_stream(row + e0 * 4 + 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) { x[i] = vec_elem<DT>(a, i); x[4 + i] = vec_elem<DT>(b, i); }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = (e0 + i < V) ? ld_elem<DT>(row, e0 + i, V) : fill;
        }
    }
}

// Eight consecutive elements of a row held as raw 16-byte vectors (one for
// bf16, two for f32): loaded without bounds checks when the whole group lies
// inside the row, so that several groups' loads can be in flight at once.
template <int DT> struct Raw8 {
    uint4 v[DT == SPEC_BF16 ? 1 : 2];
};
template <int DT> __device__ __forceinline__ void load_raw8(const char* row, int64_t e0, Raw8<DT>& r) {
    if constexpr (DT == SPEC_BF16) {
        r.v[0] = ld_stream(row + e0 * 2);
    } else {
        r.v[0] = ld_stream(row + e0 * 4);
        r.v[1] = ld_stream(row + e0 * 4 + 16);
    }
}
template <int DT> __device__ __forceinline__ void raw8_f32(const Raw8<DT>& r, float (&x)[8]) {
    if constexpr (DT == SPEC_BF16) {
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = vec_elem<DT>(r.v[0], i);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) { x[i] = vec_elem<DT>(r.v[0], i); x[4 + i] = vec_elem<DT>(r.v[1], i); }
    }
}

__device__ __forceinline__ bool excluded(const uint32_t* bitmap, int base, int64_t j) {
    const int o = (int)(j - base);
    return (bitmap[o >> 5] >> (o & 31)) & 1u;
}

// Weight functors of the inverse-CDF draws.  group(e0, w) gives the (f32)
// weights of elements e0..e0+7 (0 past V); for groups wholly inside the row
// the same weights come from load(e0, raw) followed by weights(e0, raw, w).
// Chunk sums and rescans both use them, so the arithmetic is identical.
template <int TDT> struct WTarget {          // 2^(x_j - m), excluded tokens 0
    const char* row; float s, m; const uint32_t* bitmap; int base; int V;
    struct Raw { Raw8<TDT> t; };
    __device__ __forceinline__ void load(int64_t e0, Raw& r) const { load_raw8<TDT>(row, e0, r.t); }
    __device__ __forceinline__ void finish(int64_t e0, const float (&x)[8], float (&w)[8]) const {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            w[i] = ex2(fmaf(x[i], s, -m));
            if (bitmap && e0 + i < V && excluded(bitmap, base, e0 + i)) w[i] = 0.f;
        }
    }
    __device__ __forceinline__ void weights(int64_t e0, const Raw& r, float (&w)[8]) const {
        float x[8];
        raw8_f32<TDT>(r.t, x);
        finish(e0, x, w);
    }
    __device__ __forceinline__ void group(int64_t e0, float (&w)[8]) const {
        float x[8];
        ld8<TDT>(row, e0, V, -INFINITY, x);
        finish(e0, x, w);
    }
};
template <int TDT, int DDT, int DK> struct WChainRes {   // max(0, p_j - q_j)
    static constexpr int QDT = DK == DK_PROBS ? SPEC_F32 : DDT;
    const char* trow; const char* drow; float s, mp, izp, mq, izq; int V;
    struct Raw { Raw8<TDT> t; Raw8<QDT> d; };
    __device__ __forceinline__ void load(int64_t e0, Raw& r) const {
        load_raw8<TDT>(trow, e0, r.t);
        load_raw8<QDT>(drow, e0, r.d);
    }
    __device__ __forceinline__ void finish(const float (&x)[8], const float (&d)[8], float (&w)[8]) const {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float p = ex2(fmaf(x[i], s, -mp)) * izp;
            const float q = (DK == DK_PROBS) ? d[i] : ex2(fmaf(d[i], s, -mq)) * izq;
            w[i] = fmaxf(0.f, p - q);
        }
    }
    __device__ __forceinline__ void weights(int64_t, const Raw& r, float (&w)[8]) const {
        float x[8], d[8];
        raw8_f32<TDT>(r.t, x);
        raw8_f32<QDT>(r.d, d);
        finish(x, d, w);
    }
    __device__ __forceinline__ void group(int64_t e0, float (&w)[8]) const {
        float x[8], d[8];
        ld8<TDT>(trow, e0, V, -INFINITY, x);
        if constexpr (DK == DK_PROBS) ld8<SPEC_F32>(drow, e0, V, 0.f, d);
        else ld8<DDT>(drow, e0, V, -INFINITY, d);
        finish(x, d, w);
    }
};
template <int TDT> struct WTreeRes {         // relu(p_j - d_j), excluded tokens 0
    const char* row; const char* drow; float s, m, iz; const uint32_t* bitmap; int base; int V;
    struct Raw { Raw8<TDT> t; Raw8<SPEC_F32> d; };
    __device__ __forceinline__ void load(int64_t e0, Raw& r) const {
        load_raw8<TDT>(row, e0, r.t);
        load_raw8<SPEC_F32>(drow, e0, r.d);
    }
    __device__ __forceinline__ void finish(int64_t e0, const float (&x)[8], const float (&d)[8],
                                           float (&w)[8]) const {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            w[i] = fmaxf(0.f, ex2(fmaf(x[i], s, -m)) * iz - d[i]);
            if (bitmap && e0 + i < V && excluded(bitmap, base, e0 + i)) w[i] = 0.f;
        }
    }
    __device__ __forceinline__ void weights(int64_t e0, const Raw& r, float (&w)[8]) const {
        float x[8], d[8];
        raw8_f32<TDT>(r.t, x);
        raw8_f32<SPEC_F32>(r.d, d);
        finish(e0, x, d, w);
    }
    __device__ __forceinline__ void group(int64_t e0, float (&w)[8]) const {
        float x[8], d[8];
        ld8<TDT>(row, e0, V, -INFINITY, x);
        ld8<SPEC_F32>(drow, e0, V, 0.f, d);
        finish(e0, x, d, w);
    }
};

// relu(p'_j - d_j) of a filtered tree row: p' = [x >= th] 2^(x s - m) / Z'
// (iz = 1 / Z'), d = the draft-probability row (HD) or zeros; excluded tokens
// (the rejected children) 0.
template <int TDT, bool HD> struct WTreeFilt {
    const char* row; const char* drow; float s, m, iz, th; const uint32_t* bitmap; int base; int V;
    struct Raw { Raw8<TDT> t; Raw8<SPEC_F32> d; };
    __device__ __forceinline__ void load(int64_t e0, Raw& r) const {
        load_raw8<TDT>(row, e0, r.t);
        if constexpr (HD) load_raw8<SPEC_F32>(drow, e0, r.d);
    }
    __device__ __forceinline__ void finish(int64_t e0, const float (&x)[8], const float (&d)[8],
                                           float (&w)[8]) const {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float p = x[i] >= th ? ex2(fmaf(x[i], s, -m)) * iz : 0.f;
            w[i] = fmaxf(0.f, p - d[i]);
            if (bitmap && e0 + i < V && excluded(bitmap, base, e0 + i)) w[i] = 0.f;
        }
    }
    __device__ __forceinline__ void weights(int64_t e0, const Raw& r, float (&w)[8]) const {
        float x[8], d[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        raw8_f32<TDT>(r.t, x);
        if constexpr (HD) raw8_f32<SPEC_F32>(r.d, d);
        finish(e0, x, d, w);
    }
    __device__ __forceinline__ void group(int64_t e0, float (&w)[8]) const {
        float x[8], d[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        ld8<TDT>(row, e0, V, -INFINITY, x);
        if constexpr (HD) ld8<SPEC_F32>(drow, e0, V, 0.f, d);
        finish(e0, x, d, w);
    }
};

// Multi-step residual weights at one tree node.  After j rejections the
// target distribution is p_j = max(0, p_0 - c_j q) / F(c_j), where
// F(c) = sum_v max(0, p_0(v) - c q(v)), c_0 = 0 and c_{j+1} = c_j + F(c_j):
// the residual of max(0, p_0 - c q) / F(c) against q is max(0, p_0 - (c +
// F(c)) q) / F(c) wherever it is positive, and 0 where p_0 <= c q.  The
// weight here is max(0, p_0 - c q) with p_0 = 2^(x s - m) / Z; its sum is
// F(c).
template <int TDT> struct WMss {
    const char* row; const char* drow; float s, m, iz, c; int V;
    struct Raw { Raw8<TDT> t; Raw8<SPEC_F32> d; };
    __device__ __forceinline__ void load(int64_t e0, Raw& r) const {
        load_raw8<TDT>(row, e0, r.t);
        load_raw8<SPEC_F32>(drow, e0, r.d);
    }
    __device__ __forceinline__ void finish(const float (&x)[8], const float (&d)[8], float (&w)[8]) const {
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = fmaxf(0.f, fmaf(-c, d[i], ex2(fmaf(x[i], s, -m)) * iz));
    }
    __device__ __forceinline__ void weights(int64_t, const Raw& r, float (&w)[8]) const {
        float x[8], d[8];
        raw8_f32<TDT>(r.t, x);
        raw8_f32<SPEC_F32>(r.d, d);
        finish(x, d, w);
    }
    __device__ __forceinline__ void group(int64_t e0, float (&w)[8]) const {
        float x[8], d[8];
        ld8<TDT>(row, e0, V, -INFINITY, x);
        ld8<SPEC_F32>(drow, e0, V, 0.f, d);
        finish(x, d, w);
    }
};

// Group sums of the GPT groups this thread owns in chunk c (groups
// g = k*NT + tid, coalesced).  For a chunk wholly inside the row, four groups'
// loads are issued before any of them is used.
template <int CH, int BT, class WF>
__device__ __forceinline__ void chunk_group_sums(const WF& wf, int c, float (&gs)[CH / 8 / BT]) {
    constexpr int GPT = CH / 8 / BT;
    constexpr int BATCH = GPT < 4 ? GPT : 4;
    const int64_t c0 = (int64_t)c * CH;
    if (c0 + CH <= wf.V) {
#pragma unroll
        for (int k0 = 0; k0 < GPT; k0 += BATCH) {
            typename WF::Raw raw[BATCH];
#pragma unroll
            for (int i = 0; i < BATCH; ++i) wf.load(c0 + (int64_t)((k0 + i) * BT + threadIdx.x) * 8, raw[i]);
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
                float w[8];
                wf.weights(c0 + (int64_t)((k0 + i) * BT + threadIdx.x) * 8, raw[i], w);
                gs[k0 + i] = ((w[0] + w[1]) + (w[2] + w[3])) + ((w[4] + w[5]) + (w[6] + w[7]));
            }
        }
    } else {
        // the row's last chunk: whole groups two at a time, the one group
        // that straddles V (and the groups past it) bounds-checked
        constexpr int PB = GPT < 2 ? GPT : 2;
#pragma unroll
        for (int k0 = 0; k0 < GPT; k0 += PB) {
            typename WF::Raw raw[PB];
#pragma unroll
            for (int i = 0; i < PB; ++i) {
                const int64_t e0 = c0 + (int64_t)((k0 + i) * BT + threadIdx.x) * 8;
                if (e0 + 8 <= wf.V) wf.load(e0, raw[i]);
            }
#pragma unroll
            for (int i = 0; i < PB; ++i) {
                const int64_t e0 = c0 + (int64_t)((k0 + i) * BT + threadIdx.x) * 8;
                float w[8];
                gs[k0 + i] = 0.f;
                if (e0 + 8 <= wf.V) {
                    wf.weights(e0, raw[i], w);
                    gs[k0 + i] = ((w[0] + w[1]) + (w[2] + w[3])) + ((w[4] + w[5]) + (w[6] + w[7]));
                } else if (e0 < wf.V) {
                    wf.group(e0, w);
                    gs[k0 + i] = ((w[0] + w[1]) + (w[2] + w[3])) + ((w[4] + w[5]) + (w[6] + w[7]));
                }
            }
        }
    }
}

// Sum of the weights of chunk c over this thread's groups.
template <int CH, int BT, class WF>
__device__ __forceinline__ float chunk_weight_partial(const WF& wf, int c) {
    constexpr int GPT = CH / 8 / BT;
    float gs[GPT];
    chunk_group_sums<CH, BT>(wf, c, gs);
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < GPT; ++k) acc += gs[k];
    return acc;
}

// Per-warp sums of the weights of every chunk of a row: wpw[c * BT/32 + warp]
// (f32).  Whole chunks inside the row go three at a time, the loads of all
// three issued before any weight is formed; no block-wide barrier per chunk.
template <int CH, int BT, class WF>
__device__ void row_warp_sums(const WF& wf, int nch, float* wpw) {
    constexpr int GPT = CH / 8 / BT, NWB = BT / 32, CB = 3;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int c = 0;
    for (; c + CB <= nch && (int64_t)(c + CB) * CH <= wf.V; c += CB) {
        typename WF::Raw raw[CB][GPT];
#pragma unroll
        for (int j = 0; j < CB; ++j)
#pragma unroll
            for (int k = 0; k < GPT; ++k)
                wf.load((int64_t)(c + j) * CH + (int64_t)(k * BT + threadIdx.x) * 8, raw[j][k]);
#pragma unroll
        for (int j = 0; j < CB; ++j) {
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < GPT; ++k) {
                float w[8];
                wf.weights((int64_t)(c + j) * CH + (int64_t)(k * BT + threadIdx.x) * 8, raw[j][k], w);
                acc += ((w[0] + w[1]) + (w[2] + w[3])) + ((w[4] + w[5]) + (w[6] + w[7]));
            }
            acc = warp_sum(acc);
            if (lane == 0) wpw[(c + j) * NWB + warp] = acc;
        }
    }
    for (; c < nch; ++c) {
        const float acc = warp_sum(chunk_weight_partial<CH, BT>(wf, c));
        if (lane == 0) wpw[c * NWB + warp] = acc;
    }
}

// Inverse-CDF rescan of chunk c: the chunk is read as coalesced 8-element
// groups (group g covers elements c*CH + 8g .. +7, thread tid owns groups
// g = k*NT + tid), group sums are scanned block-wide in fp64 in index order,
// and the thread owning t_loc recomputes its group and walks its 8 weights.
// If t_loc < 0, t_loc = u * (chunk total) (single-chunk rows).  Returns the
// drawn index, or -1 when the chunk has no positive weight; *chunk_total gets
// the chunk's sum.
template <int CH, int BT, class WF>
__device__ int rescan_chunk(const WF& wf, int c, int V, double t_loc, float u, double* chunk_total) {
    constexpr int GPT = CH / 8 / BT;
    constexpr int BW = BT / 32;
    __shared__ double wt[GPT][BW];
    __shared__ int owner, found;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (!bounds_ok(c >= 0 && (int64_t)c * CH < V)) c = 0;
    float gs[GPT];
    chunk_group_sums<CH, BT>(wf, c, gs);
    double inc[GPT];
#pragma unroll
    for (int k = 0; k < GPT; ++k) {
        inc[k] = (double)gs[k];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            double n = __shfl_up_sync(FULL, inc[k], o);
            if (lane >= o) inc[k] += n;
        }
        if (lane == 31) wt[k][warp] = inc[k];
    }
    if (tid == 0) { owner = -1; found = -1; }
    __syncthreads();
    double total = 0.0;
#pragma unroll
    for (int k = 0; k < GPT; ++k)
#pragma unroll
        for (int w = 0; w < BW; ++w) total += wt[k][w];
    if (chunk_total) *chunk_total = total;
    if (t_loc < 0.0) t_loc = (double)u * total;
    double base = 0.0;
#pragma unroll
    for (int k = 0; k < GPT; ++k) {
        double before = base;
#pragma unroll
        for (int w = 0; w < BW; ++w) if (w < warp) before += wt[k][w];
        const double excl = before + inc[k] - (double)gs[k];
        if (gs[k] > 0.f && excl <= t_loc) atomicMax(&owner, k * BT + tid);
#pragma unroll
        for (int w = 0; w < BW; ++w) base += wt[k][w];
    }
    __syncthreads();
    const int og = owner;
    if (og >= 0 && (og % BT) == tid) {
        const int k = og / BT;
        double before = 0.0;
        for (int kk = 0; kk < k; ++kk)
            for (int w = 0; w < BW; ++w) before += wt[kk][w];
        for (int w = 0; w < warp; ++w) before += wt[k][w];
        double excl = 0.0;
#pragma unroll
        for (int kk = 0; kk < GPT; ++kk)
            if (kk == k) excl = before + inc[kk] - (double)gs[kk];
        const int64_t e0 = (int64_t)c * CH + (int64_t)og * 8;
        float w[8];
        wf.group(e0, w);
        const double loc = t_loc - excl;
        double acc = 0.0;
        int pick = -1, last = -1;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            acc += (double)w[i];
            if (w[i] > 0.f) {
                last = (int)(e0 + i);
                if (pick < 0 && loc < acc) pick = (int)(e0 + i);
            }
        }
        found = pick >= 0 ? pick : last;
    }
    __syncthreads();
    const int r = found;
    __syncthreads();
    return r;
}

// Inverse-CDF draw from the target row `row` (statistics st: nch*SPC entries)
// with the tokens in excl[0..nexcl) removed.  Chunk masses come from the
// statistics (fp64), excluded tokens are subtracted from their chunk, the
// chunk holding u*S is rescanned.  *S_unnorm = remaining mass in units of
// 2^(x - m).  Returns the token (or -1 if nothing is left).
template <int TDT, int BT>
__device__ int sample_target_row(const char* row, int V, int nch, const float2* st, float s, float m,
                                 float u, const int* excl, int nexcl, FinShared& sh, double* S_unnorm) {
    constexpr int CH = chunk_elems<TDT>();
    const int tid = threadIdx.x;
    for (int c = tid; c < nch; c += BT) {
        double M = 0.0;
#pragma unroll
        for (int w = 0; w < SPC; ++w) {
            float2 x = ldcg2(st + c * SPC + w);
            if (x.x > -INFINITY) M += (double)x.y * ex2d(x.x, m);
        }
        sh.M[c] = M;
    }
    __syncthreads();
    if (tid == 0) {
        for (int i = 0; i < nexcl; ++i) {
            int t = excl[i];
            bool dup = false;
            for (int j = 0; j < i; ++j) dup |= (excl[j] == t);
            if (dup) continue;
            if (!bounds_ok(t >= 0 && t < V)) continue;
            double e = exp2((double)ld_elem<TDT>(row, t, V) * (double)s - (double)m);
            double& M = sh.M[t / CH];
            M = fmax(0.0, M - e);
        }
        double S = 0.0;
        for (int c = 0; c < nch; ++c) S += sh.M[c];
        sh.dvals[0] = S;
    }
    __syncthreads();
    const double S = sh.dvals[0];
    *S_unnorm = S;
    const double t = (double)u * S;
    int result = -1;
    for (int attempt = 0; attempt < nch; ++attempt) {
        if (tid == 0) {
            double C = 0.0;
            int cs = -1;
            double before = 0.0;
            for (int c = 0; c < nch; ++c) {
                if (sh.M[c] <= 0.0) continue;
                if (t < C + sh.M[c]) { cs = c; before = C; break; }
                C += sh.M[c];
            }
            if (cs < 0) {                       // rounding past the end: last chunk with mass
                for (int c = nch - 1; c >= 0; --c)
                    if (sh.M[c] > 0.0) { cs = c; break; }
                before = C - (cs >= 0 ? sh.M[cs] : 0.0);
            }
            sh.ivals[0] = cs;
            sh.dvals[1] = before;
        }
        __syncthreads();
        const int cs = sh.ivals[0];
        if (cs < 0) break;
        for (int w = tid; w < CH / 32; w += BT) sh.bitmap[w] = 0u;
        __syncthreads();
        for (int i = tid; i < nexcl; i += BT) {
            int o = excl[i] - cs * CH;
            if (o >= 0 && o < CH) atomicOr(&sh.bitmap[o >> 5], 1u << (o & 31));
        }
        __syncthreads();
        WTarget<TDT> wf{row, s, m, nexcl ? sh.bitmap : nullptr, cs * CH, V};
        double tot;
        result = rescan_chunk<CH, BT>(wf, cs, V, fmax(0.0, t - sh.dvals[1]), u, &tot);
        if (result >= 0) break;
        if (tid == 0) sh.M[cs] = 0.0;         // nothing positive there after all: skip it
        __syncthreads();
    }
    return result;
}

// Validate a tree held in sh.par / sh.tok (N nodes); returns 1 if well formed.
template <int BT>
__device__ int tree_valid(const Params& P, int N, int V, int max_depth, FinShared& sh) {
    __shared__ int ok;
    if (threadIdx.x == 0) ok = 1;
    __syncthreads();
    for (int n = threadIdx.x; n < N; n += BT) {
        int pa = sh.par[n];
        bool good = (n == 0) ? (pa == -1) : (pa >= 0 && pa < n && sh.tok[n] >= 0 && sh.tok[n] < V);
        if (!good) ok = 0;
    }
    __syncthreads();
    if (ok) {
        for (int n = threadIdx.x; n < N; n += BT) {
            int d = 0, a = n;
            while (a > 0 && d <= max_depth) { a = bounds_ok(a < N) ? sh.par[a] : 0; ++d; }
            if (d > max_depth) ok = 0;
        }
    }
    __syncthreads();
    int r = ok;
    __syncthreads();
    return r;
}

// ----------------------------------------------------------------------------- finalisers

// Inputs of the chain decision that the statistics kernel does not write:
// loaded by threads 0..gamma-1 before waiting for that kernel (programmatic
// dependent launch), so their latency hides under its tail.
struct ChainPrefetch {
    int x;          // draft token of position tid
    float l;        // target logit at x
    float d;        // draft logit (or probability) at x
    float coin;     // coins[b, tid]
    bool ok;        // x in [0, V)
};

template <int TDT, int DDT, int DK>
__device__ __forceinline__ ChainPrefetch chain_prefetch(const Params& P, int b) {
    ChainPrefetch f{0, 0.f, 0.f, 0.f, false};
    const int tid = threadIdx.x, gamma = P.gamma, i = tid & 31;
    if (tid < 64 && i < gamma) {                      // warp 0: p side, warp 1: q side of position i
        f.x = P.draft_tokens[(size_t)b * gamma + i];
        f.ok = f.x >= 0 && f.x < P.V;
        if (tid < 32) {
            f.coin = P.coins[(size_t)b * gamma + i];
            if (f.ok) f.l = ld_elem<TDT>(P.tgt + ((size_t)b * (gamma + 1) + i) * P.tstride, f.x, P.V);
        } else if (f.ok) {
            const char* drow = P.drf + ((size_t)b * gamma + i) * P.dstride;
            if constexpr (DK == DK_PROBS) f.d = __ldg(reinterpret_cast<const float*>(drow) + f.x);
            else f.d = ld_elem<DDT>(drow, f.x, P.V);
        }
    }
    return f;
}

// Chain decision for sequence b (rule 1), after the row statistics were
// combined into sh.m / sh.z / sh.bad.  Threads i of warps 0 and 1 turn their
// prefetched logits into p_i(x_i) and q_i(x_i) (fp64 exp2 in the units of the
// row statistics), thread i tests position i's coin, and thread 0 takes the
// first rejection.  Leaves sh.ivals[0] =
// valid, sh.ivals[1] = k, sh.dvals[0] = s.  When `write` is set it also writes
// the accepted tokens, the -1 tail (position k excluded), num_accepted and
// the p/q diagnostics, and flags invalid sequences.  Ends with __syncthreads.
template <int TDT, int DDT, int DK, bool FILT = false>
__device__ void chain_decide(const Params& P, int b, FinShared& sh, bool write, const ChainPrefetch& f) {
    const int tid = threadIdx.x;
    const int gamma = P.gamma, W = gamma + 1;
    int32_t* toks = P.out_tokens + (size_t)b * W;
    float* dg = P.diag ? P.diag + (size_t)b * (2 * gamma + 1) : nullptr;
    const float T = P.temperature[b];
    const bool tok = temperature_ok(T);
    const float s = tok ? scale_of(T) : 0.f;
    // p(x_i) in warp 0 and q(x_i) in warp 1 (thread i of each), then each
    // position's coin test in thread i; thread 0 finds the first rejection
    const int wi = tid & 31;
    if (tid < 64 && wi < gamma) {
        const bool q_side = tid >= 32;
        bool ok = f.ok;
        double v = 0.0;
        if (ok && tok) {
            if (!q_side) {
                v = prob_d(f.l, s, sh.m[wi], sh.z[wi]);
                if (FILT && f.l < sh.th[wi]) v = 0.0;             // filtered out
            } else if constexpr (DK == DK_PROBS) {
                v = (double)f.d;
                ok &= (v >= 0.0 && v <= 3.0e38);
            } else {
                v = prob_d(f.d, s, sh.m[gamma + 1 + wi], sh.z[gamma + 1 + wi]);
                if (FILT && f.d < sh.th[gamma + 1 + wi]) v = 0.0;
            }
        }
        sh.pch[(q_side ? SPEC_MAX_GAMMA : 0) + wi] = v;
        if (q_side) {
            sh.rej[wi] = ok;
        } else {
            sh.pch[2 * SPEC_MAX_GAMMA + wi] = (double)f.coin;
            sh.tok[wi] = f.x;
        }
    }
    __syncthreads();
    if (tid < gamma) {                                // accept position tid?
        const double pi = sh.pch[tid], qi = sh.pch[SPEC_MAX_GAMMA + tid];
        const double ratio = (qi > 0.0) ? pi / qi : INFINITY;
        sh.par[tid] = (sh.pch[2 * SPEC_MAX_GAMMA + tid] <= ratio) ? 1 : 0;
    }
    __syncthreads();
    if (tid == 0) {
        bool ok = tok;
        for (int r = 0; r < P.R; ++r) ok &= !sh.bad[r];
        for (int i = 0; i < gamma; ++i) ok &= (sh.rej[i] != 0);
        int k = gamma;
        if (ok)
            for (int i = 0; i < gamma; ++i)
                if (!sh.par[i]) { k = i; break; }
        sh.ivals[0] = ok;
        sh.ivals[1] = k;
        sh.dvals[0] = (double)s;
        if (write) {
            if (!ok) {
                for (int i = 0; i < W; ++i) toks[i] = -1;
                P.out_num_accepted[b] = -1;
                if (dg) for (int i = 0; i < 2 * gamma + 1; ++i) dg[i] = nanf_();
                flag_input_error(P);
            } else {
                for (int i = 0; i < k; ++i) toks[i] = sh.tok[i];
                for (int i = k + 1; i < W; ++i) toks[i] = -1;
                P.out_num_accepted[b] = k;
                if (dg)
                    for (int i = 0; i < gamma; ++i) {
                        dg[i] = (float)sh.pch[i];
                        dg[gamma + i] = (float)sh.pch[SPEC_MAX_GAMMA + i];
                    }
            }
        }
    }
    __syncthreads();
}

// Start of the lazy chain finalisation for sequence b: the decision comes from
// the level walk.  A sequence still active after position gamma - 1 takes the
// bonus draw from row gamma, whose statistics are combined here.  Leaves the
// same shared state as chain_decide (sh.ivals[0] = valid, sh.ivals[1] = k,
// sh.dvals[0] = s, the statistics of rows k and gamma + 1 + k); when `write`
// is set also writes the accepted tokens, the -1 tail, num_accepted, NaN for
// the diagnostics of positions never evaluated, and flags invalid sequences.
// Ends with __syncthreads.
__device__ void chain_lazy_state(const Params& P, int b, FinShared& sh, bool write) {
    const int tid = threadIdx.x, gamma = P.gamma, W = gamma + 1;
    if (tid < 32) {
        const LazySeq L = P.lz_seq[b];
        int ok = L.state == LZ_DRAW || (L.state == LZ_ACTIVE && L.k == gamma);
        float m = L.m;
        double z = L.z;
        if (ok && L.state == LZ_ACTIVE) {
            const int E = P.nch * SPC;
            ok = !warp_combine(P.stats + ((size_t)b * P.R + gamma) * E, E, m, z);
            if (!ok && tid == 0) flag_input_error(P);
        }
        if (tid == 0) {
            const int k = ok ? L.k : 0;
            sh.ivals[0] = ok;
            sh.ivals[1] = k;
            sh.dvals[0] = (double)L.s;
            sh.m[k] = m;
            sh.z[k] = z;
            if (k < gamma) {
                sh.m[gamma + 1 + k] = L.mq;
                sh.z[gamma + 1 + k] = L.zq;
            }
            if (write) {
                int32_t* toks = P.out_tokens + (size_t)b * W;
                float* dg = P.diag ? P.diag + (size_t)b * (2 * gamma + 1) : nullptr;
                if (!ok) {
                    for (int i = 0; i < W; ++i) toks[i] = -1;
                    P.out_num_accepted[b] = -1;
                    if (dg) for (int i = 0; i < 2 * gamma + 1; ++i) dg[i] = nanf_();
                } else {
                    for (int i = 0; i < k; ++i) toks[i] = P.draft_tokens[(size_t)b * gamma + i];
                    for (int i = k + 1; i < W; ++i) toks[i] = -1;
                    P.out_num_accepted[b] = k;
                    if (dg)
                        for (int i = k + 1; i < gamma; ++i) { dg[i] = nanf_(); dg[gamma + i] = nanf_(); }
                }
            }
        }
    }
    __syncthreads();
}

// One row's argmax statistics (E entries at st) combined by one warp: the
// maximum's lowest index in every lane; returns whether a NaN was seen.
__device__ __forceinline__ bool warp_argmax(const float2* st, int E, int& idx_out) {
    const int lane = threadIdx.x & 31;
    float best = -INFINITY;
    int idx = 0x7fffffff;
    bool bad = false;
    for (int e = lane; e < E; e += 32) {
        const float2 x = st[e];
        int xi = __float_as_int(x.y);
        if (x.x != x.x) bad = true;
        else if (x.x > best || (x.x == best && xi < idx)) { best = x.x; idx = xi; }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        float ov = __shfl_xor_sync(FULL, best, o);
        int oi = __shfl_xor_sync(FULL, idx, o);
        if (ov > best || (ov == best && oi < idx)) { best = ov; idx = oi; }
    }
    idx_out = idx;
    return __any_sync(FULL, bad);
}

// warp_argmax of one row: index to sh.rej[slot], NaN flag to sh.bad[slot].
__device__ __forceinline__ void argmax_row(const float2* st, int E, FinShared& sh, int slot) {
    int idx;
    const bool bad = warp_argmax(st, E, idx);
    if ((threadIdx.x & 31) == 0) { sh.rej[slot] = idx; sh.bad[slot] = bad; }
}

template <int TDT, int BT>
__device__ void finalize_greedy(const Params& P, int b, FinShared& sh, const float2* blk) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = P.N, V = P.V, W = P.max_depth + 1;
    const int E = P.nch * SPC;
    // per-node argmax (lowest index among equal maxima)
    for (int r = warp; r < N; r += BT / 32) argmax_row(blk + (size_t)r * E, E, sh, r);
    for (int n = tid; n < N; n += BT) {
        sh.par[n] = P.parents[(size_t)b * N + n];
        sh.tok[n] = P.tokens[(size_t)b * N + n];
    }
    __syncthreads();
    int ok = tree_valid<BT>(P, N, V, P.max_depth, sh);
    if (tid == 0) {
        for (int r = 0; r < N; ++r) ok &= !sh.bad[r];
        sh.ivals[0] = ok;
    }
    __syncthreads();
    ok = sh.ivals[0];
    int32_t* ai = P.out_accept_index + (size_t)b * W;
    int32_t* ot = P.out_tokens + (size_t)b * W;
    if (!ok) {
        for (int i = tid; i < W; i += BT) { ai[i] = -1; ot[i] = -1; }
        if (tid == 0) { P.out_num_accepted[b] = -1; flag_input_error(P); }
        return;
    }
    if (warp == 0) {
        const int* g = sh.rej;
        int cur = 0, k = 0;
        if (lane == 0) ai[0] = 0;
        for (;;) {
            int next = -1;
            for (int base = cur + 1; base < N && next < 0; base += 32) {
                int c = base + lane;
                bool hit = c < N && sh.par[c] == cur && sh.tok[c] == g[cur];
                unsigned m = __ballot_sync(FULL, hit);
                if (m) next = base + __ffs(m) - 1;
            }
            if (next < 0) break;
            if (lane == 0) { ot[k] = sh.tok[next]; ai[k + 1] = next; }
            ++k;
            cur = next;
        }
        if (lane == 0) {
            ot[k] = g[cur];
            for (int i = k + 1; i < W; ++i) { ot[i] = -1; ai[i] = -1; }
            P.out_num_accepted[b] = k;
        }
    }
}

// Last token of a target-only tree walk ending at node `cur`: drawn with
// final_u[b] from relu(p_cur - d_cur), d_cur = the draft_probs row of cur
// (zeros when draft_probs is NULL) with the rejected children's tokens
// rej[0..nrej) overwritten by their target probabilities.  (mc, zc) are the
// statistics of row cur.  *S_out receives the mass of relu(p_cur - d_cur).
template <int TDT, int BT>
__device__ int tree_final_draw(const Params& P, int b, int cur, const int* rej, int nrej, float s, float mc,
                               double zc, FinShared& sh, double* S_out) {
    const int tid = threadIdx.x, N = P.N, V = P.V;
    const char* row = P.tgt + ((size_t)b * N + cur) * P.tstride;
    const float u = P.final_u[b];
    int y;
    double S;
    if (!P.draft_probs) {
        const float2* st = P.stats + ((size_t)b * P.R + cur) * P.nch * SPC;
        double Su;
        y = sample_target_row<TDT, BT>(row, V, P.nch, st, s, mc, u, rej, nrej, sh, &Su);
        S = Su / zc;
    } else {
        // relu(p_cur - d_cur) over the whole row: chunk sums, then one rescan.
        constexpr int CH = chunk_elems<TDT>();
        const char* drow = reinterpret_cast<const char*>(P.draft_probs) + ((size_t)b * N + cur) * P.dpstride;
        const float m = mc, iz = (float)(1.0 / zc);
        for (int c = 0; c < P.nch; ++c) {
            for (int w = tid; w < CH / 32; w += BT) sh.bitmap[w] = 0u;
            __syncthreads();
            for (int i = tid; i < nrej; i += BT) {
                int o = rej[i] - c * CH;
                if (o >= 0 && o < CH) atomicOr(&sh.bitmap[o >> 5], 1u << (o & 31));
            }
            __syncthreads();
            WTreeRes<TDT> wf{row, drow, s, m, iz, sh.bitmap, c * CH, V};
            double tot;
            block_excl_scan<BT>((double)chunk_weight_partial<CH, BT>(wf, c), &tot);
            if (tid == 0) sh.M[c] = tot;
            __syncthreads();
        }
        if (tid == 0) {
            double tot = 0.0;
            for (int c = 0; c < P.nch; ++c) tot += sh.M[c];
            sh.dvals[0] = tot;
        }
        __syncthreads();
        S = sh.dvals[0];
        y = -1;
        if (S > 0.0) {
            const double t = (double)u * S;
            for (int attempt = 0; attempt < P.nch && y < 0; ++attempt) {
                if (tid == 0) {
                    double C = 0.0, before = 0.0;
                    int cs = -1;
                    for (int c = 0; c < P.nch; ++c) {
                        if (sh.M[c] <= 0.0) continue;
                        if (t < C + sh.M[c]) { cs = c; before = C; break; }
                        C += sh.M[c];
                    }
                    if (cs < 0)
                        for (int c = P.nch - 1; c >= 0; --c)
                            if (sh.M[c] > 0.0) { cs = c; before = C - sh.M[c]; break; }
                    sh.ivals[4] = cs;
                    sh.dvals[1] = before;
                }
                __syncthreads();
                const int cs = sh.ivals[4];
                if (cs < 0) break;
                for (int w = tid; w < CH / 32; w += BT) sh.bitmap[w] = 0u;
                __syncthreads();
                for (int i = tid; i < nrej; i += BT) {
                    int o = rej[i] - cs * CH;
                    if (o >= 0 && o < CH) atomicOr(&sh.bitmap[o >> 5], 1u << (o & 31));
                }
                __syncthreads();
                WTreeRes<TDT> wf{row, drow, s, m, iz, sh.bitmap, cs * CH, V};
                double tot;
                y = rescan_chunk<CH, BT>(wf, cs, V, fmax(0.0, t - sh.dvals[1]), u, &tot);
                if (y < 0 && tid == 0) sh.M[cs] = 0.0;
                __syncthreads();
            }
        }
        if (y < 0) {
            // empty residual (rounding only): draw from p_cur itself
            const float2* st = P.stats + ((size_t)b * P.R + cur) * P.nch * SPC;
            double Su;
            y = sample_target_row<TDT, BT>(row, V, P.nch, st, s, m, u, nullptr, 0, sh, &Su);
        }
    }
    *S_out = S;
    return y;
}

// Chunk masses sh.M[0..nch) of the weights wf over a row (per-warp sums in
// wpw, then fp64 per chunk in warp order); returns their total (fp64, chunk
// order).  All threads of the CTA call it.
template <int CH, int BT, class WF>
__device__ double row_chunk_masses(const WF& wf, int nch, float* wpw, FinShared& sh) {
    constexpr int NWB = BT / 32;
    row_warp_sums<CH, BT>(wf, nch, wpw);
    __syncthreads();
    for (int c = threadIdx.x; c < nch; c += BT) {
        double M = 0.0;
#pragma unroll
        for (int w = 0; w < NWB; ++w) M += (double)wpw[c * NWB + w];
        sh.M[c] = M;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double S = 0.0;
        for (int c = 0; c < nch; ++c) S += sh.M[c];
        sh.dvals[0] = S;
    }
    __syncthreads();
    const double S = sh.dvals[0];
    __syncthreads();
    return S;
}

// Bitmap (sh.bitmap) of the excluded tokens rej[0..nrej) that fall in chunk c.
template <int CH, int BT>
__device__ void excl_bitmap(const int* rej, int nrej, int c, FinShared& sh) {
    for (int w = threadIdx.x; w < CH / 32; w += BT) sh.bitmap[w] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < nrej; i += BT) {
        const int o = rej[i] - c * CH;
        if (o >= 0 && o < CH) atomicOr(&sh.bitmap[o >> 5], 1u << (o & 31));
    }
    __syncthreads();
}

// Inverse-CDF draw over a whole row with the weights wf (whose bitmap is
// sh.bitmap) and the tokens rej[0..nrej) excluded.  The chunk masses come
// from one pass over the row without exclusions (row_chunk_masses; wpw holds
// nch * BT/32 floats); the few chunks that hold an excluded token are summed
// again with their exclusions (block sums in fp64), so no mass is subtracted.
// Then the chunk holding u*S and one rescan.  *S_out = the total; -1 when it
// is not positive.  All threads call it.
template <int CH, int BT, class WF>
__device__ int draw_excluding(WF wf, const int* rej, int nrej, int nch, int V, float u, float* wpw, FinShared& sh,
                              double* S_out) {
    const int tid = threadIdx.x;
    wf.bitmap = nullptr;
    row_chunk_masses<CH, BT>(wf, nch, wpw, sh);
    wf.bitmap = sh.bitmap;
    for (int i = 0; i < nrej; ++i) {                  // rej is uniform across the CTA
        const int e = rej[i];
        if (e < 0 || e >= V) continue;
        bool seen = false;
        for (int j = 0; j < i; ++j) seen |= rej[j] >= 0 && rej[j] < V && rej[j] / CH == e / CH;
        if (seen) continue;
        const int c = e / CH;
        excl_bitmap<CH, BT>(rej, nrej, c, sh);
        wf.base = c * CH;
        double tot;
        block_excl_scan<BT>((double)chunk_weight_partial<CH, BT>(wf, c), &tot);
        if (tid == 0) sh.M[c] = tot;
        __syncthreads();
    }
    if (tid == 0) {
        double tot = 0.0;
        for (int c = 0; c < nch; ++c) tot += sh.M[c];
        sh.dvals[0] = tot;
    }
    __syncthreads();
    const double S = sh.dvals[0];
    *S_out = S;
    int y = -1;
    if (S > 0.0) {
        const double t = (double)u * S;
        for (int attempt = 0; attempt < nch && y < 0; ++attempt) {
            if (tid == 0) {
                double C = 0.0, before = 0.0;
                int cs = -1;
                for (int c = 0; c < nch; ++c) {
                    if (sh.M[c] <= 0.0) continue;
                    if (t < C + sh.M[c]) { cs = c; before = C; break; }
                    C += sh.M[c];
                }
                if (cs < 0)
                    for (int c = nch - 1; c >= 0; --c)
                        if (sh.M[c] > 0.0) { cs = c; before = C - sh.M[c]; break; }
                sh.ivals[4] = cs;
                sh.dvals[1] = before;
            }
            __syncthreads();
            const int cs = sh.ivals[4];
            if (cs < 0) break;
            excl_bitmap<CH, BT>(rej, nrej, cs, sh);
            wf.base = cs * CH;
            double tot;
            y = rescan_chunk<CH, BT>(wf, cs, V, fmax(0.0, t - sh.dvals[1]), u, &tot);
            if (y < 0 && tid == 0) sh.M[cs] = 0.0;
            __syncthreads();
        }
    }
    return y;
}

// The last token of a filtered target-only walk that stopped at node cur:
// drawn from relu(p'_cur - d_cur) with the rejected children removed
// (d = draft_probs row, or zeros); an empty residual (rounding only) draws
// from p'_cur itself.  *S_out = the residual's mass.
template <int TDT, int BT, bool HD>
__device__ int tree_filt_draw(const Params& P, int b, int cur, const int* rej, int nrej, float s, float m,
                              double zc, float th, float* wpw, FinShared& sh, double* S_out) {
    constexpr int CH = chunk_elems<TDT>();
    const char* row = P.tgt + ((size_t)b * P.N + cur) * P.tstride;
    const char* drow = HD ? reinterpret_cast<const char*>(P.draft_probs) + ((size_t)b * P.N + cur) * P.dpstride
                          : nullptr;
    const float u = P.final_u[b], iz = (float)(1.0 / zc);
    WTreeFilt<TDT, HD> wr{row, drow, s, m, iz, th, sh.bitmap, 0, P.V};
    int y = draw_excluding<CH, BT>(wr, rej, nrej, P.nch, P.V, u, wpw, sh, S_out);
    if (y < 0) {
        WTreeFilt<TDT, false> wp{row, nullptr, s, m, iz, th, sh.bitmap, 0, P.V};
        double S1;
        y = draw_excluding<CH, BT>(wp, rej, 0, P.nch, P.V, u, wpw, sh, &S1);
    }
    return y;
}

// Target-only tree sampling, one CTA per sequence (FILT: on the top-k /
// top-p filtered rows, from the records of k_filter).
// Target-only tree sampling for sequence b, one CTA.  FILT: under top-k /
// top-p filtering, with each row's threshold and kept mass read from the
// filter records (k_filter) -- or, OD (on demand, bf16 rows, no diagnostics),
// computed here for the rows of the nodes the walk visits, one window
// histogram each (win: WF_BYTES of shared memory).  FILT: win also holds the
// final draw's per-warp chunk sums (P.nch * BT/32 floats).
template <int TDT, int BT, bool FILT = false, bool OD = false>
__device__ void finalize_sample(const Params& P, int b, FinShared& sh, const float2* blk, unsigned char* win = nullptr,
                                WinShared* ws = nullptr) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = P.N, V = P.V, W = P.max_depth + 1;
    combine_softmax_rows<BT>(P, blk, N, sh);
    for (int n = tid; n < N; n += BT) {
        sh.par[n] = P.parents[(size_t)b * N + n];
        sh.tok[n] = P.tokens[(size_t)b * N + n];
    }
    __syncthreads();
    const int K = (FILT && OD && P.top_k) ? P.top_k[b] : 0;
    const float Pp = (FILT && OD && P.top_p) ? P.top_p[b] : 1.f;
    if constexpr (FILT && !OD) {
        // each row's threshold and kept mass (same 2^(x s - m) units as z)
        for (int n = tid; n < N; n += BT) {
            const FiltRec f = P.filt[(size_t)b * P.R + n];
            sh.th[n] = f.theta;
            if (f.on > 0) sh.z[n] = f.Z;
            if (f.on < 0) sh.bad[n] = 1;             // invalid top_k / top_p
        }
        __syncthreads();
    }
    int ok = tree_valid<BT>(P, N, V, P.max_depth, sh);
    const float T = P.temperature[b];
    if (tid == 0) {
        ok &= temperature_ok(T);
        for (int r = 0; r < N; ++r) ok &= !sh.bad[r];
        if (FILT && OD) ok &= (K >= 0 && Pp > 0.f && Pp <= 1.f);        // invalid top_k / top_p
        sh.ivals[0] = ok;
    }
    __syncthreads();
    ok = sh.ivals[0];
    int32_t* ai = P.out_accept_index + (size_t)b * W;
    int32_t* ot = P.out_tokens + (size_t)b * W;
    float* dg = P.diag ? P.diag + (size_t)b * (N + 1) : nullptr;
    if (!ok) {
        for (int i = tid; i < W; i += BT) { ai[i] = -1; ot[i] = -1; }
        if (dg) for (int i = tid; i < N + 1; i += BT) dg[i] = nanf_();
        if (tid == 0) { P.out_num_accepted[b] = -1; flag_input_error(P); }
        return;
    }
    const float s = scale_of(T);
    if constexpr (FILT && OD) {
        // the walk, filtering the row of each node it visits
        const double ths = (double)P.th_single, tha = (double)P.th_acc;
        int cur = 0, k = 0, nrej = 0;
        float thc;
        double zc;
        if (tid == 0) ai[0] = 0;
        for (;;) {
            const char* row = P.tgt + ((size_t)b * N + cur) * P.tstride;
            FiltRec f{-INFINITY, 0, 0.0};
            const float2* st = P.stats + ((size_t)b * P.R + cur) * P.nch * SPC;
            if (((K > 0 && K < V) || Pp < 1.f) &&
                !cand_filter<BT>(P, row, st, s, sh.m[cur], sh.z[cur], K, Pp, win, WF_BYTES, &f))
                f = wfilter_row<BT>(row, V, s, sh.m[cur], sh.z[cur], K, Pp, win, *ws);
            thc = f.theta;
            zc = f.on > 0 ? f.Z : sh.z[cur];
            for (int n = cur + 1 + tid; n < N; n += BT)
                if (sh.par[n] == cur) {
                    const float l = ld_elem<TDT>(row, sh.tok[n], V);
                    sh.pch[n] = l >= thc ? prob_d(l, s, sh.m[cur], zc) : 0.0;
                }
            __syncthreads();
            if (warp == 0) {
                const double coin = (double)P.coins[(size_t)b * N + cur];
                double acc = 0.0;
                int next = -1;
                nrej = 0;
                for (int base = cur + 1; base < N && next < 0; base += 32) {
                    const int c = base + lane;
                    unsigned m = __ballot_sync(FULL, c < N && sh.par[c] == cur);
                    if (lane == 0) {
                        while (m && next < 0) {
                            const int cc = base + __ffs(m) - 1;
                            m &= m - 1;
                            const double pc = sh.pch[cc];
                            acc += pc;
                            if (coin <= acc / tha || pc >= ths) next = cc;
                            else sh.rej[nrej++] = sh.tok[cc];
                        }
                    }
                    next = __shfl_sync(FULL, next, 0);
                }
                if (lane == 0) { sh.ivals[1] = next; sh.ivals[3] = nrej; }
            }
            __syncthreads();
            const int next = sh.ivals[1];
            nrej = sh.ivals[3];
            __syncthreads();
            if (next < 0) break;
            if (tid == 0) { ot[k] = sh.tok[next]; ai[k + 1] = next; }
            ++k;
            cur = next;
        }
        double S;
        float* wpw = reinterpret_cast<float*>(win);    // (the window's shared memory is free now)
        const int y = P.draft_probs ? tree_filt_draw<TDT, BT, true>(P, b, cur, sh.rej, nrej, s, sh.m[cur], zc, thc,
                                                                    wpw, sh, &S)
                                    : tree_filt_draw<TDT, BT, false>(P, b, cur, sh.rej, nrej, s, sh.m[cur], zc, thc,
                                                                     wpw, sh, &S);
        if (tid == 0) {
            ot[k] = y;
            for (int i = k + 1; i < W; ++i) { ot[i] = -1; ai[i] = -1; }
            P.out_num_accepted[b] = k;
        }
        return;
    }
    // p_parent(n)(tokens[n]) for every non-root node (0 below the row's threshold)
    for (int n = tid; n < N; n += BT) {
        double pc = 0.0;
        if (n > 0) {
            int pa = sh.par[n];
            const char* row = P.tgt + ((size_t)b * N + pa) * P.tstride;
            const float l = ld_elem<TDT>(row, sh.tok[n], P.V);
            if (!FILT || l >= sh.th[pa]) pc = prob_d(l, s, sh.m[pa], sh.z[pa]);
        }
        sh.pch[n] = pc;
        if (dg) dg[n] = (float)pc;
    }
    __syncthreads();
    // sibling walk with prob_acc
    if (warp == 0) {
        const double ths = (double)P.th_single, tha = (double)P.th_acc;
        int cur = 0, k = 0, nrej = 0;
        if (lane == 0) ai[0] = 0;
        for (;;) {
            const double coin = (double)P.coins[(size_t)b * N + cur];
            double acc = 0.0;
            int next = -1;
            nrej = 0;
            for (int base = cur + 1; base < N && next < 0; base += 32) {
                int c = base + lane;
                unsigned m = __ballot_sync(FULL, c < N && sh.par[c] == cur);
                if (lane == 0) {
                    while (m && next < 0) {
                        int cc = base + __ffs(m) - 1;
                        m &= m - 1;
                        double pc = sh.pch[cc];
                        acc += pc;
                        if (coin <= acc / tha || pc >= ths) next = cc;
                        else sh.rej[nrej++] = sh.tok[cc];
                    }
                }
                next = __shfl_sync(FULL, next, 0);
            }
            if (next < 0) break;
            if (lane == 0) { ot[k] = sh.tok[next]; ai[k + 1] = next; }
            ++k;
            cur = next;
        }
        if (lane == 0) { sh.ivals[1] = cur; sh.ivals[2] = k; sh.ivals[3] = nrej; }
    }
    __syncthreads();
    const int cur = sh.ivals[1], k = sh.ivals[2], nrej = sh.ivals[3];
    double S;
    int y;
    if constexpr (FILT) {
        float* wpw = reinterpret_cast<float*>(win);
        y = P.draft_probs ? tree_filt_draw<TDT, BT, true>(P, b, cur, sh.rej, nrej, s, sh.m[cur], sh.z[cur],
                                                          sh.th[cur], wpw, sh, &S)
                          : tree_filt_draw<TDT, BT, false>(P, b, cur, sh.rej, nrej, s, sh.m[cur], sh.z[cur],
                                                           sh.th[cur], wpw, sh, &S);
    } else {
        y = tree_final_draw<TDT, BT>(P, b, cur, sh.rej, nrej, s, sh.m[cur], sh.z[cur], sh, &S);
    }
    if (tid == 0) {
        ot[k] = y;
        for (int i = k + 1; i < W; ++i) { ot[i] = -1; ai[i] = -1; }
        P.out_num_accepted[b] = k;
        if (dg) dg[N] = (float)S;
    }
}

// Locate the chunk holding t among the chunk masses sh.M[0..nch) (skipping
// empty chunks) and rescan it; retries past chunks whose rescan finds no
// positive weight (possible only through rounding).  Returns -1 if none.
template <int CH, int BT, class WF>
__device__ int draw_from_chunks(const WF& wf, int nch, int V, double t, float u, FinShared& sh) {
    const int tid = threadIdx.x;
    int y = -1;
    for (int attempt = 0; attempt < nch && y < 0; ++attempt) {
        if (tid == 0) {
            double C = 0.0, before = 0.0;
            int cs = -1;
            for (int cc = 0; cc < nch; ++cc) {
                if (sh.M[cc] <= 0.0) continue;
                if (t < C + sh.M[cc]) { cs = cc; before = C; break; }
                C += sh.M[cc];
            }
            if (cs < 0)
                for (int cc = nch - 1; cc >= 0; --cc)
                    if (sh.M[cc] > 0.0) { cs = cc; before = C - sh.M[cc]; break; }
            sh.ivals[2] = cs;
            sh.dvals[1] = before;
        }
        __syncthreads();
        const int cs = sh.ivals[2];
        if (cs < 0) break;
        double tot;
        y = rescan_chunk<CH, BT>(wf, cs, V, fmax(0.0, t - sh.dvals[1]), u, &tot);
        if (y < 0 && tid == 0) sh.M[cs] = 0.0;
        __syncthreads();
    }
    return y;
}

// State of the multi-step sampling walk at one node: p_j = max(0, p_0 - c q)
// / D, D = F(c) (see WMss), after `steps` residual steps; `have_M` when sh.M
// holds the chunk masses of max(0, p_0 - c q); S = the last residual mass
// S_j = D_j / D_{j-1} (1 before any).  Uniform across the CTA.
struct MssState {
    double c, D, S;
    int steps;
    bool have_M;
};

// Multi-step speculative sampling at node cur of sequence b ([origins]
// "SpecInfer", MSS bullet), all threads of the CTA: the children of cur
// (sh.par / sh.tok) are tested in node order, child c with coins[b, c]
// against p_j(x) / q(x), p_j(x) = max(0, p_0(x) - c q(x)) / D in fp64 from the
// gathered logit; a rejection costs one pass over the (target, q) row pair
// for the next F.  Returns the accepted child, -1 when none is (st then
// describes the p of the final draw), -2 for an invalid drafted q(x) or a
// non-finite residual mass.  Writes p_j(x) of each test to dg[c].
template <int TDT, int BT>
__device__ int mss_node(const Params& P, int b, int cur, float s, float m, double z, float* dg, float* wpw,
                        FinShared& sh, MssState& st) {
    constexpr int CH = chunk_elems<TDT>();
    const int tid = threadIdx.x, N = P.N;
    const char* row = P.tgt + ((size_t)b * N + cur) * P.tstride;
    const char* drow = reinterpret_cast<const char*>(P.draft_probs) + ((size_t)b * N + cur) * P.dpstride;
    st = MssState{0.0, 1.0, 1.0, 0, false};
    for (int c = cur + 1; c < N; ++c) {
        if (sh.par[c] != cur) continue;
        if (tid == 0) {
            const int x = sh.tok[c];
            const double qx = (double)__ldg(reinterpret_cast<const float*>(drow) + x);
            int verdict = -1;                         // -1 invalid, 0 reject, 1 accept
            if (qx >= 0.0 && qx <= 3.4028234663852886e38) {
                const double p = fmax(0.0, prob_d(ld_elem<TDT>(row, x, P.V), s, m, z) - st.c * qx) / st.D;
                if (dg) dg[c] = (float)p;
                const double ratio = qx > 0.0 ? p / qx : INFINITY;
                verdict = ((double)P.coins[(size_t)b * N + c] <= ratio) ? 1 : 0;
            }
            sh.ivals[1] = verdict;
        }
        __syncthreads();
        const int verdict = sh.ivals[1];
        __syncthreads();
        if (verdict < 0) return -2;
        if (verdict > 0) return c;
        const double cn = st.c + st.D;
        WMss<TDT> wf{row, drow, s, m, (float)(1.0 / z), (float)cn, P.V};
        const double F = row_chunk_masses<CH, BT>(wf, P.nch, wpw, sh);
        if (!(F <= 1.7976931348623157e308)) return -2;          // inf or NaN
        st.have_M = F > 0.0;
        if (st.have_M) {                                        // else p stays (rounding only)
            st.S = F / st.D;
            st.c = cn;
            st.D = F;
            ++st.steps;
        }
    }
    return -1;
}

// The last token of a multi-step sampling walk that stopped at node cur: drawn
// with final_u from the current p (the row statistics when no residual step
// was taken, else the chunk masses of max(0, p_0 - c q) and one chunk rescan).
template <int TDT, int BT>
__device__ int mss_draw(const Params& P, int b, int cur, float s, float m, double z, float* wpw, FinShared& sh,
                        const MssState& st) {
    constexpr int CH = chunk_elems<TDT>();
    const int nch = P.nch;
    const char* row = P.tgt + ((size_t)b * P.N + cur) * P.tstride;
    const float u = P.final_u[b];
    int y = -1;
    if (st.steps > 0) {
        const char* drow = reinterpret_cast<const char*>(P.draft_probs) + ((size_t)b * P.N + cur) * P.dpstride;
        WMss<TDT> wf{row, drow, s, m, (float)(1.0 / z), (float)st.c, P.V};
        if (!st.have_M) row_chunk_masses<CH, BT>(wf, nch, wpw, sh);
        double tot = 0.0;
        for (int c = 0; c < nch; ++c) tot += sh.M[c];
        if (tot > 0.0) y = draw_from_chunks<CH, BT>(wf, nch, P.V, (double)u * tot, u, sh);
    }
    if (y < 0) {
        const float2* stt = P.stats + ((size_t)b * P.R + cur) * nch * SPC;
        double Su;
        y = sample_target_row<TDT, BT>(row, P.V, nch, stt, s, m, u, nullptr, 0, sh, &Su);
    }
    return y;
}

// Tree verification with a draft distribution, one CTA per sequence: combine
// every node's statistics, validate, then walk with mss_node and draw with
// mss_draw.
template <int TDT, int BT>
__device__ void finalize_mss(const Params& P, int b, FinShared& sh, const float2* blk, float* wpw) {
    const int tid = threadIdx.x;
    const int N = P.N, V = P.V, W = P.max_depth + 1;
    combine_softmax_rows<BT>(P, blk, N, sh);
    for (int n = tid; n < N; n += BT) {
        sh.par[n] = P.parents[(size_t)b * N + n];
        sh.tok[n] = P.tokens[(size_t)b * N + n];
    }
    __syncthreads();
    int ok = tree_valid<BT>(P, N, V, P.max_depth, sh);
    const float T = P.temperature[b];
    if (tid == 0) {
        ok &= temperature_ok(T);
        for (int r = 0; r < N; ++r) ok &= !sh.bad[r];
        sh.ivals[0] = ok;
    }
    __syncthreads();
    ok = sh.ivals[0];
    int32_t* ai = P.out_accept_index + (size_t)b * W;
    int32_t* ot = P.out_tokens + (size_t)b * W;
    float* dg = P.diag ? P.diag + (size_t)b * (N + 1) : nullptr;
    if (dg) for (int i = tid; i <= N; i += BT) dg[i] = nanf_();
    __syncthreads();
    const float s = ok ? scale_of(T) : 0.f;
    int cur = 0, k = 0;
    MssState st{0.0, 1.0, 1.0, 0, false};
    if (ok) {
        if (tid == 0) ai[0] = 0;
        for (;;) {
            const int next = mss_node<TDT, BT>(P, b, cur, s, sh.m[cur], sh.z[cur], dg, wpw, sh, st);
            if (next == -2) ok = 0;
            if (next < 0) break;
            if (tid == 0) {
                ot[k] = sh.tok[next];
                ai[k + 1] = next;
            }
            ++k;
            cur = next;
        }
    }
    if (!ok) {
        for (int i = tid; i < W; i += BT) { ai[i] = -1; ot[i] = -1; }
        __syncthreads();
        if (dg) for (int i = tid; i <= N; i += BT) dg[i] = nanf_();
        if (tid == 0) { P.out_num_accepted[b] = -1; flag_input_error(P); }
        return;
    }
    const int y = mss_draw<TDT, BT>(P, b, cur, s, sh.m[cur], sh.z[cur], wpw, sh, st);
    if (tid == 0) {
        ot[k] = y;
        for (int i = k + 1; i < W; ++i) { ot[i] = -1; ai[i] = -1; }
        P.out_num_accepted[b] = k;
        if (dg) dg[N] = (float)st.S;
    }
}

// ----------------------------------------------------------------------------- kernels

// Row statistics (the streaming kernel).  The B*R*nch work items (sequence-
// major, then row, then chunk; a chunk is 16 KB of one row) are split into
// gridDim.x contiguous ranges of equal length (within one), one per CTA;
// (b, r, c) advance incrementally.  Each thread loads its eight 16-byte
// vectors of a chunk at once; each warp reduces its quarter to one statistic
// -- online softmax (max x, sum 2^(x - max)) or (max, lowest index) -- and
// writes it.  Nothing else is shared: no atomics, no fences; the finalize
// kernel that follows in stream order reads the statistics.  Ten CTAs of four
// warps per SM (at most 51 registers) keep enough loads in flight and enough
// warps to hide the exp2 and ALU latency.
template <int MODE, int TDT, int DDT>
__global__ void __launch_bounds__(NT, STATS_CTAS_PER_SM) k_stats(const Params P) {
    constexpr int CH = chunk_elems<TDT>();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    pdl_trigger();
    const int per_seq = P.R * P.nch;
    const long long total = (long long)P.B * per_seq;
    const long long lo = total * blockIdx.x / gridDim.x;
    const long long n = total * (blockIdx.x + 1) / gridDim.x - lo;
    int b = (int)(lo / per_seq);
    int r, c;
    {
        const int rem = (int)(lo - (long long)b * per_seq);
        r = rem / P.nch;
        c = rem - r * P.nch;
    }
    int sb = -1;
    float s = 0.f;
    for (long long j = 0; j < n; ++j) {
        float2 stat;
        if constexpr (MODE == MODE_GREEDY) {
            const char* row = P.tgt + ((size_t)b * P.R + r) * P.tstride;
            stat = chunk_argmax<TDT>(row, P.V, c);
        } else {
            if (b != sb) { sb = b; s = scale_of(__ldg(P.temperature + b)); }
            if (r < P.rows_tgt) {
                const char* row = P.tgt + ((size_t)b * P.rows_tgt + r) * P.tstride;
                stat = chunk_softmax<TDT, CH>(row, P.V, c, s);
            } else {
                const char* row = P.drf + ((size_t)b * (P.R - P.rows_tgt) + (r - P.rows_tgt)) * P.dstride;
                stat = chunk_softmax<DDT, CH>(row, P.V, c, s);
            }
        }
        if (lane == 0) P.stats[(((size_t)b * P.R + r) * P.nch + c) * SPC + warp] = stat;
        if (++c == P.nch) {
            c = 0;
            if (++r == P.R) { r = 0; ++b; }
        }
    }
}

// Chain finalisation, grid = B * nsl: CTA (b, slice) recomputes sequence b's
// decision from the row statistics (cheap, identical in every CTA of b), then
//  - k = gamma: slice 0 draws the bonus token from p_gamma (rule 3);
//  - k < gamma: every slice sums max(0, p_k - q_k) over its chunks of row k;
//    with one slice the CTA draws directly, otherwise the last CTA of the
//    sequence to arrive locates the chunk holding u*S and rescans it (rule 2).
template <int TDT, int DDT, int DK, bool LZ>
__global__ void __launch_bounds__(NT) k_chain_final(const Params P) {
    __shared__ FinShared sh;
    __shared__ int is_last;
    __shared__ __align__(8) uint64_t sbar;
    extern __shared__ __align__(128) unsigned char dyn[];
    constexpr int CH = chunk_elems<TDT>();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nsl = P.nsl, nch = P.nch;
    const int b = blockIdx.x / nsl, sl = blockIdx.x - b * nsl;
    const int c0 = (int)((long long)nch * sl / nsl), c1 = (int)((long long)nch * (sl + 1) / nsl);
    const int gamma = P.gamma, V = P.V;
    if constexpr (LZ) {
        pdl_wait();
        chain_lazy_state(P, b, sh, sl == 0);
    } else {
        const ChainPrefetch pf = chain_prefetch<TDT, DDT, DK>(P, b);
        pdl_wait();
        const float2* blk = stage_stats(P, b, P.R, dyn, P.stage_cap, &sbar);
        combine_softmax_rows<NT>(P, blk, P.R, sh);
        __syncthreads();
        chain_decide<TDT, DDT, DK>(P, b, sh, sl == 0, pf);
    }
    const int ok = sh.ivals[0], k = sh.ivals[1];
    const float s = (float)sh.dvals[0];
    if (!ok) return;
    const float u = P.final_u[b];
    int32_t* toks = P.out_tokens + (size_t)b * (gamma + 1);
    float* dg = P.diag ? P.diag + (size_t)b * (2 * gamma + 1) : nullptr;
    const char* trow = P.tgt + ((size_t)b * (gamma + 1) + k) * P.tstride;
    if (k == gamma) {
        if (sl != 0) return;
        const float2* st = P.stats + ((size_t)b * P.R + gamma) * nch * SPC;
        double S;
        int y = sample_target_row<TDT, NT>(trow, V, nch, st, s, sh.m[gamma], u, nullptr, 0, sh, &S);
        if (tid == 0) {
            toks[k] = y;
            if (dg) dg[2 * gamma] = 1.0f;
        }
        return;
    }
    const char* drow = P.drf + ((size_t)b * gamma + k) * P.dstride;
    const float mp = sh.m[k], izp = (float)(1.0 / sh.z[k]);
    const float mq = (DK == DK_PROBS) ? 0.f : sh.m[gamma + 1 + k];
    const float izq = (DK == DK_PROBS) ? 0.f : (float)(1.0 / sh.z[gamma + 1 + k]);
    WChainRes<TDT, DDT, DK> wf{trow, drow, s, mp, izp, mq, izq, V};
    // chunk sums of max(0, p_k - q_k) for this slice's chunks
    for (int c = c0; c < c1; ++c) {
        const float ws = warp_sum(chunk_weight_partial<CH, NT>(wf, c));
        if (lane == 0) {
            if (nsl == 1) sh.wp[c][warp] = ws;
            else P.stats2[((size_t)b * nch + c) * NWARP + warp] = make_float2(ws, 0.f);
        }
    }
    if (nsl == 1) {
        __syncthreads();
        for (int c = tid; c < nch; c += NT) {
            double M = 0.0;
#pragma unroll
            for (int w = 0; w < NWARP; ++w) M += (double)sh.wp[c][w];
            sh.M[c] = M;
        }
    } else {
        if (lane == 0) __threadfence();
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            const unsigned prev = atomicAdd(P.cnt2 + b, 1u);
            is_last = (prev == (unsigned)nsl - 1u);
        }
        __syncthreads();
        if (!is_last) return;
        __threadfence();
        for (int c = tid; c < nch; c += NT) {
            double M = 0.0;
#pragma unroll
            for (int w = 0; w < NWARP; ++w) M += (double)ldcg2(P.stats2 + ((size_t)b * nch + c) * NWARP + w).x;
            sh.M[c] = M;
        }
    }
    __syncthreads();
    if (tid == 0) {
        double S = 0.0;
        for (int c = 0; c < nch; ++c) S += sh.M[c];
        sh.dvals[0] = S;
    }
    __syncthreads();
    const double S = sh.dvals[0];
    int y = (S > 0.0) ? draw_from_chunks<CH, NT>(wf, nch, V, (double)u * S, u, sh) : -1;
    if (y < 0) {
        // empty residual (rounding only): draw from p_k
        const float2* stk = P.stats + ((size_t)b * P.R + k) * nch * SPC;
        double Su;
        y = sample_target_row<TDT, NT>(trow, V, nch, stk, s, mp, u, nullptr, 0, sh, &Su);
    }
    if (tid == 0) {
        toks[k] = y;
        if (dg) dg[2 * gamma] = (float)S;
        if (nsl > 1) {
            __threadfence();
            P.cnt2[b] = 0u;
        }
    }
}

// Eight elements e0..e0+7 of a row staged in shared memory: elements below
// `nstaged` come from the stage, the rest below V from global memory, the
// rest are `fill`.
template <int DT>
__device__ __forceinline__ void ld8_staged(const unsigned char* stage, const char* row, int64_t e0, int nstaged,
                                           int V, float fill, float (&x)[8]) {
    if (e0 + 8 <= nstaged) {
        if constexpr (DT == SPEC_BF16) {
            const uint4 v = *reinterpret_cast<const uint4*>(stage + e0 * 2);
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = vec_elem<DT>(v, i);
        } else {
            const uint4 a = *reinterpret_cast<const uint4*>(stage + e0 * 4);
            const uint4 b = *reinterpret_cast<const uint4*>(stage + e0 * 4 + 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) { x[i] = vec_elem<DT>(a, i); x[4 + i] = vec_elem<DT>(b, i); }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int64_t e = e0 + i;
            if (e < nstaged) {
                if constexpr (DT == SPEC_BF16)
                    x[i] = __uint_as_float((uint32_t)reinterpret_cast<const unsigned short*>(stage)[e] << 16);
                else
                    x[i] = reinterpret_cast<const float*>(stage)[e];
            } else {
                x[i] = e < V ? ld_elem<DT>(row, e, V) : fill;
            }
        }
    }
}

// max(0, p_j - q_j) read from a staged row pair.
template <int TDT, int DDT, int DK> struct WChainResStaged {
    const unsigned char* ts; const unsigned char* ds; const char* trow; const char* drow;
    int nt, nd; float s, mp, izp, mq, izq; int V;
    __device__ __forceinline__ void group(int64_t e0, float (&w)[8]) const {
        float x[8], d[8];
        ld8_staged<TDT>(ts, trow, e0, nt, V, -INFINITY, x);
        if constexpr (DK == DK_PROBS) ld8_staged<SPEC_F32>(ds, drow, e0, nd, V, 0.f, d);
        else ld8_staged<DDT>(ds, drow, e0, nd, V, -INFINITY, d);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float p = ex2(fmaf(x[i], s, -mp)) * izp;
            const float q = (DK == DK_PROBS) ? d[i] : ex2(fmaf(d[i], s, -mq)) * izq;
            w[i] = fmaxf(0.f, p - q);
        }
    }
};

// Shared-memory bytes of one CTA's part of a staged row pair (target part,
// draft part, its group sums), rounded up to 16 bytes; the statistics area
// follows.
__host__ __device__ inline size_t staged_bytes(int V, int tesz, int desz) {
    const size_t bt = ((size_t)V * tesz) & ~(size_t)15, bd = ((size_t)V * desz) & ~(size_t)15;
    return (bt + bd + (size_t)((V + 7) / 8) * 4 + 15) & ~(size_t)15;
}

// Thread-block cluster helpers (a pair of CTAs per sequence).
__device__ __forceinline__ unsigned cluster_rank() {
    unsigned r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ double peer_ld_f64(const double* p, unsigned peer) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(p)), "r"(peer));
    double v;
    asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(remote) : "memory");
    return v;
}
__device__ __forceinline__ int peer_ld_s32(const int* p, unsigned peer) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(p)), "r"(peer));
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
    return v;
}

// Chain finalisation by a cluster of two CTAs per sequence: both take the
// decision (identical); the rejected row pair is split at a group boundary,
// each CTA stages its half with two bulk copies, forms the 8-element group
// sums of max(0, p_k - q_k) and scans them; the two half masses meet through
// distributed shared memory (two cluster barriers, which every CTA of the pair
// reaches on every path: the decision is the same in both); the CTA whose
// half holds u*S draws inside it.  The bonus token is drawn by the first CTA
// as in the one-CTA kernel.
template <int TDT, int DDT, int DK, bool LZ>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(SEQ_BT) k_chain_final_pair(const Params P) {
    __shared__ FinShared sh;
    __shared__ __align__(8) uint64_t bar, sbar;
    __shared__ int owner, found_g, s_fail;
    __shared__ double s_half;
    extern __shared__ __align__(128) unsigned char stage[];
    constexpr int TESZ = Tr<TDT>::ESZ;
    constexpr int DESZ = DK == DK_PROBS ? 4 : Tr<DDT>::ESZ;
    const unsigned rank = cluster_rank();
    const int tid = threadIdx.x, b = blockIdx.x >> 1;
    const int gamma = P.gamma, V = P.V;
    if constexpr (LZ) {
        pdl_wait();
        if (tid == 0) mbar_init(smem_u32(&bar), 1);
        chain_lazy_state(P, b, sh, rank == 0);
    } else {
        const ChainPrefetch pf = chain_prefetch<TDT, DDT, DK>(P, b);
        pdl_wait();
        const float2* blk = stage_stats(P, b, P.R, stage + P.stage_off, P.stage_cap, &sbar);
        if (tid == 0) mbar_init(smem_u32(&bar), 1);
        combine_softmax_rows<SEQ_BT>(P, blk, P.R, sh);
        __syncthreads();
        chain_decide<TDT, DDT, DK>(P, b, sh, rank == 0, pf);
    }
    const int ok = sh.ivals[0], k = sh.ivals[1];
    const float s = (float)sh.dvals[0];
    if (!ok) return;                                  // the same in both CTAs of the pair
    const float u = P.final_u[b];
    int32_t* toks = P.out_tokens + (size_t)b * (gamma + 1);
    float* dg = P.diag ? P.diag + (size_t)b * (2 * gamma + 1) : nullptr;
    const char* trow = P.tgt + ((size_t)b * (gamma + 1) + k) * P.tstride;
    if (k == gamma) {                                 // the same in both CTAs of the pair
        if (rank != 0) return;
        const float2* st = P.stats + ((size_t)b * P.R + gamma) * P.nch * SPC;
        double S;
        const int y = sample_target_row<TDT, SEQ_BT>(trow, V, P.nch, st, s, sh.m[gamma], u, nullptr, 0, sh, &S);
        if (tid == 0) {
            toks[k] = y;
            if (dg) dg[2 * gamma] = 1.0f;
        }
        return;
    }
    const char* drow = P.drf + ((size_t)b * gamma + k) * P.dstride;
    // this CTA's half: groups [0, G0) or [G0, G), G0 = ceil(G / 2)
    const int G = (V + 7) / 8, G0 = (G + 1) / 2;
    const int lo = rank == 0 ? 0 : 8 * G0;
    const int Vh = rank == 0 ? min(V, 8 * G0) : max(0, V - 8 * G0);
    const char* th = trow + (size_t)lo * TESZ;
    const char* dh = drow + (size_t)lo * DESZ;
    const uint32_t bt = ((uint32_t)Vh * TESZ) & ~15u, bd = ((uint32_t)Vh * DESZ) & ~15u;
    unsigned char* ts = stage;
    unsigned char* ds = stage + bt;
    float* gs = reinterpret_cast<float*>(stage + bt + bd);
    if (tid == 0) {
        mbar_expect_tx(smem_u32(&bar), bt + bd);
        if (bt) bulk_g2s(smem_u32(ts), th, bt, smem_u32(&bar));
        if (bd) bulk_g2s(smem_u32(ds), dh, bd, smem_u32(&bar));
    }
    const float mp = sh.m[k], izp = (float)(1.0 / sh.z[k]);
    const float mq = (DK == DK_PROBS) ? 0.f : sh.m[gamma + 1 + k];
    const float izq = (DK == DK_PROBS) ? 0.f : (float)(1.0 / sh.z[gamma + 1 + k]);
    WChainResStaged<TDT, DDT, DK> wf{ts, ds, th, dh, (int)(bt / TESZ), (int)(bd / DESZ), s, mp, izp, mq, izq, Vh};
    // the same verdict in every thread: a wait that gave up in any thread fails the copy
    const bool copied = __syncthreads_and(mbar_wait(smem_u32(&bar), 0, P.wait_tries)) != 0;
    if (!copied && tid == 0) copy_timed_out(P, mbar_wait(smem_u32(&bar), 0));   // let the copy land (bounded)
    const int Gh = (Vh + 7) / 8;
    if (copied)
        for (int g = tid; g < Gh; g += SEQ_BT) {
            float w[8];
            wf.group((int64_t)g * 8, w);
            gs[g] = ((w[0] + w[1]) + (w[2] + w[3])) + ((w[4] + w[5]) + (w[6] + w[7]));
        }
    __syncthreads();
    const int g0 = (int)((long long)Gh * tid / SEQ_BT), g1 = (int)((long long)Gh * (tid + 1) / SEQ_BT);
    double seg = 0.0;
    if (copied)
        for (int g = g0; g < g1; ++g) seg += (double)gs[g];
    if (tid == 0) { owner = -1; found_g = -1; }
    double Sh;
    const double excl = block_excl_scan<SEQ_BT>(seg, &Sh);
    if (tid == 0) { s_half = Sh; s_fail = copied ? 0 : 1; }
    cluster_sync_all();                               // both halves' masses are written
    const double Sp = peer_ld_f64(&s_half, rank ^ 1u);
    const int fail = (copied ? 0 : 1) | peer_ld_s32(&s_fail, rank ^ 1u);
    cluster_sync_all();                               // nothing reads the peer's shared memory after this
    if (fail) {
        if (rank == 0 && tid == 0) {
            for (int i = 0; i <= gamma; ++i) toks[i] = -1;
            P.out_num_accepted[b] = -1;
        }
        return;
    }
    const double S0 = rank == 0 ? Sh : Sp, S1 = rank == 0 ? Sp : Sh;
    const double S = S0 + S1;                         // the same sum in both CTAs
    const double t = (double)u * S;
    if (!(S > 0.0)) {                                 // empty residual (rounding only): draw from p_k
        if (rank != 0) return;
        const float2* stk = P.stats + ((size_t)b * P.R + k) * P.nch * SPC;
        double Su;
        const int y = sample_target_row<TDT, SEQ_BT>(trow, V, P.nch, stk, s, mp, u, nullptr, 0, sh, &Su);
        if (tid == 0) {
            toks[k] = y;
            if (dg) dg[2 * gamma] = (float)S;
        }
        return;
    }
    // the half holding t (rounding past the end goes to the last half with mass)
    const unsigned own = (S0 > 0.0 && (t < S0 || !(S1 > 0.0))) ? 0u : 1u;
    if (rank != own) return;
    const double tl = own == 0 ? t : t - S0;
    if (seg > 0.0 && excl <= tl) atomicMax(&owner, tid);
    __syncthreads();
    if (tid == owner) {
        double acc = excl;
        int gsel = -1, glast = -1;
        double before = excl;
        for (int g = g0; g < g1; ++g) {
            const double v = (double)gs[g];
            if (v > 0.0) {
                glast = g;
                before = acc;
                if (tl < acc + v) { gsel = g; break; }
            }
            acc += v;
        }
        if (gsel < 0) gsel = glast;
        float w[8];
        wf.group((int64_t)gsel * 8, w);
        const double loc = tl - before;
        double a = 0.0;
        int pick = -1, last = -1;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            a += (double)w[i];
            if (w[i] > 0.f) {
                last = gsel * 8 + i;
                if (pick < 0 && loc < a) pick = gsel * 8 + i;
            }
        }
        found_g = pick >= 0 ? pick : last;
    }
    __syncthreads();
    int y = found_g >= 0 ? lo + found_g : -1;
    if (y < 0) {                                      // nothing positive found (rounding only): draw from p_k
        const float2* stk = P.stats + ((size_t)b * P.R + k) * P.nch * SPC;
        double Su;
        y = sample_target_row<TDT, SEQ_BT>(trow, V, P.nch, stk, s, mp, u, nullptr, 0, sh, &Su);
    }
    if (tid == 0) {
        toks[k] = y;
        if (dg) dg[2 * gamma] = (float)S;
    }
}

// Tree finalisation, one CTA per sequence.
template <int MODE, int TDT>
__global__ void __launch_bounds__(SEQ_BT) k_tree_final(const Params P) {
    __shared__ FinShared sh;
    __shared__ __align__(8) uint64_t sbar;
    extern __shared__ __align__(128) unsigned char dyn[];
    pdl_wait();
    const float2* blk = stage_stats(P, blockIdx.x, P.N, dyn, P.stage_cap, &sbar);
    if constexpr (MODE == MODE_GREEDY) finalize_greedy<TDT, SEQ_BT>(P, blockIdx.x, sh, blk);
    else if constexpr (MODE == MODE_SAMPLE) finalize_sample<TDT, SEQ_BT>(P, blockIdx.x, sh, blk);
    else if constexpr (MODE == MODE_SAMPLE_FILT)
        finalize_sample<TDT, SEQ_BT, true>(P, blockIdx.x, sh, blk, dyn + P.stage_off);
    else if constexpr (MODE == MODE_SAMPLE_FILT_OD) {
        __shared__ WinShared ws;
        finalize_sample<TDT, SEQ_BT, true, true>(P, blockIdx.x, sh, blk,
                                                 dyn + P.stage_off, &ws);
    }
    else finalize_mss<TDT, SEQ_BT>(P, blockIdx.x, sh, blk, reinterpret_cast<float*>(dyn + P.stage_off));
}

// The filter record of one row of sequence b (statistics row r, logits at
// `row`, element type DT): invalid top_k / top_p give on = -1; filters off, a
// bad temperature or an unusable row (the decision marks the sequence
// invalid) give on = 0.  bf16 rows try their candidates first (cfilter_row);
// the whole-row path is, with FILT_BT threads, the value histogram (the radix
// descent when a counter wraps), else the windowed filter; f32 rows take the
// radix descent.  All threads of the CTA call it; thread 0 writes.
template <int DT, int BT>
__device__ void filter_one_row(const Params& P, int b, int r, const char* row, FiltShared& fs, WinShared& ws,
                               unsigned char* dyn) {
    __shared__ float msh;
    __shared__ double zsh_;
    __shared__ int bad;
    FiltRec* out = P.filt + (size_t)b * P.R + r;
    const int K = P.top_k ? P.top_k[b] : 0;
    const float Pp = P.top_p ? P.top_p[b] : 1.f;
    const float T = P.temperature[b];
    if (K < 0 || !(Pp > 0.f && Pp <= 1.f)) {
        if (threadIdx.x == 0) *out = FiltRec{-INFINITY, -1, 0.0};
        return;
    }
    if (!temperature_ok(T) || ((K <= 0 || K >= P.V) && Pp >= 1.f)) {
        if (threadIdx.x == 0) *out = FiltRec{-INFINITY, 0, 0.0};
        return;
    }
    const int E = P.nch * SPC;
    if (threadIdx.x < 32) {
        float m;
        double z;
        const bool bd = warp_combine(P.stats + ((size_t)b * P.R + r) * E, E, m, z);
        if (threadIdx.x == 0) { msh = m; zsh_ = z; bad = bd; }
    }
    __syncthreads();
    const bool unusable = bad;
    const float s = scale_of(T), m = msh;
    const double zsh = zsh_;
    __syncthreads();
    if (unusable) {
        if (threadIdx.x == 0) *out = FiltRec{-INFINITY, 0, 0.0};
        return;
    }
    FiltRec rec{-INFINITY, 0, 0.0};
    bool done = false;
    if constexpr (DT == SPEC_BF16)
        done = cand_filter<BT>(P, row, P.stats + ((size_t)b * P.R + r) * E, s, m, zsh, K, Pp, dyn,
                               BT == FILT_BT ? VH_BYTES : WF_BYTES, &rec);
    if constexpr (BT == FILT_BT) {
        uint32_t* w = reinterpret_cast<uint32_t*>(dyn);
        if (!done && (DT != SPEC_BF16 || !vh_select(P.V, vh_build(row, P.V, fs, w), s, m, zsh, K, Pp, fs, w, &rec)))
            rec = filter_row<DT>(row, P.V, s, m, zsh, K, Pp, fs, FiltHist<DT>{dyn});
    } else if constexpr (DT == SPEC_BF16) {
        if (!done) rec = wfilter_row<BT>(row, P.V, s, m, zsh, K, Pp, dyn, ws);
    }
    if (threadIdx.x == 0) *out = rec;
}

// Filter thresholds of every row of a round, one CTA per (sequence, row):
// target rows 0..gamma, then the draft-logit rows (TREE: the N node rows of
// every tree).  A bf16 row's first step of loads is issued before the wait
// for the statistics.  Every CTA waits for the statistics before it exits,
// so the finalize kernel that follows (and reads the records and the
// statistics) waits for them through this kernel.
template <int TDT, int DDT, int DK, bool TREE, int BT>
__global__ void __launch_bounds__(BT, BT == FILT_BT ? 1 : 4) k_filter(const Params P) {
    // FILT_BT threads: the value histogram and the radix descent (any row);
    // fewer: bf16 rows only, the windowed filter as the whole-row path
    static_assert(BT == FILT_BT || (TDT == SPEC_BF16 && (DK != DK_LOGITS || DDT == SPEC_BF16)), "bf16 rows only");
    __shared__ FiltShared fs;
    __shared__ WinShared ws;
    __shared__ float msh;
    __shared__ double zsh;
    __shared__ int bad;
    extern __shared__ __align__(128) unsigned char dyn[];
    pdl_trigger();
    const int rows = TREE ? P.N : ((DK == DK_LOGITS) ? 2 * P.gamma + 1 : P.gamma + 1);
    const int b = blockIdx.x / rows, r = blockIdx.x - b * rows;
    FiltRec* out = P.filt + (size_t)b * P.R + r;
    const int K = P.top_k ? P.top_k[b] : 0;
    const float Pp = P.top_p ? P.top_p[b] : 1.f;
    const float T = P.temperature[b];
    if (K < 0 || !(Pp > 0.f && Pp <= 1.f)) {
        pdl_wait();
        if (threadIdx.x == 0) *out = FiltRec{-INFINITY, -1, 0.0};
        return;
    }
    if (!temperature_ok(T) || ((K <= 0 || K >= P.V) && Pp >= 1.f)) {
        pdl_wait();
        if (threadIdx.x == 0) *out = FiltRec{-INFINITY, 0, 0.0};
        return;
    }
    const bool tgt = TREE || r <= P.gamma;
    const char* row = TREE  ? P.tgt + ((size_t)b * P.N + r) * P.tstride
                      : tgt ? P.tgt + ((size_t)b * (P.gamma + 1) + r) * P.tstride
                            : P.drf + ((size_t)b * P.gamma + (r - P.gamma - 1)) * P.dstride;
    const bool vh = tgt ? TDT == SPEC_BF16 : DDT == SPEC_BF16;
    uint32_t* w = reinterpret_cast<uint32_t*>(dyn);
    CfPre<BT> pre;
    pre.have = false;
    if (vh && !(P.filt_mode & 1u)) cf_prefetch<BT>(row, P.V, pre);
    pdl_wait();
    const int E = P.nch * SPC;
    if (threadIdx.x < 32) {
        float m;
        double z;
        const bool bd = warp_combine(P.stats + ((size_t)b * P.R + r) * E, E, m, z);
        if (threadIdx.x == 0) { msh = m; zsh = z; bad = bd; }
    }
    __syncthreads();
    if (bad) {                                   // the decision marks the sequence invalid
        if (threadIdx.x == 0) *out = FiltRec{-INFINITY, 0, 0.0};
        return;
    }
    const float s = scale_of(T), m = msh;
    const double z = zsh;
    FiltRec rec;
    if constexpr (BT != FILT_BT) {
        if (!cand_filter<BT>(P, row, P.stats + ((size_t)b * P.R + r) * E, s, m, z, K, Pp, dyn, WF_BYTES, &rec, &pre,
                             CF_MANY))
            rec = wfilter_row<BT>(row, P.V, s, m, z, K, Pp, dyn, ws);
    } else if (!vh || !(cand_filter<BT>(P, row, P.stats + ((size_t)b * P.R + r) * E, s, m, z, K, Pp, dyn, VH_BYTES,
                                        &rec, &pre, CF_MANY) ||
                        vh_select(P.V, vh_build(row, P.V, fs, w), s, m, z, K, Pp, fs, w, &rec))) {
        if (tgt) rec = filter_row<TDT>(row, P.V, s, m, z, K, Pp, fs, FiltHist<TDT>{dyn});
        else rec = filter_row<DDT>(row, P.V, s, m, z, K, Pp, fs, FiltHist<DDT>{dyn});
    }
    if (threadIdx.x == 0) *out = rec;
}


// max(0, p' - q') of a filtered target row and a filtered draft row (QK =
// DK_LOGITS), a draft probability row (DK_PROBS), or no draft (DK_NONE: p').
template <int TDT, int QDT, int QK> struct WFilt {
    const char* trow; const char* drow; float s, mp, izp, thp, mq, izq, thq; int V;
    struct Raw { Raw8<TDT> t; Raw8<QDT> d; };
    __device__ __forceinline__ void load(int64_t e0, Raw& r) const {
        load_raw8<TDT>(trow, e0, r.t);
        if constexpr (QK != DK_NONE) load_raw8<QDT>(drow, e0, r.d);
    }
    __device__ __forceinline__ void finish(const float (&x)[8], const float (&d)[8], float (&w)[8]) const {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float p = x[i] >= thp ? ex2(fmaf(x[i], s, -mp)) * izp : 0.f;
            float q = 0.f;
            if constexpr (QK == DK_PROBS) q = d[i];
            if constexpr (QK == DK_LOGITS) q = d[i] >= thq ? ex2(fmaf(d[i], s, -mq)) * izq : 0.f;
            w[i] = fmaxf(0.f, p - q);
        }
    }
    __device__ __forceinline__ void weights(int64_t, const Raw& r, float (&w)[8]) const {
        float x[8], d[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        raw8_f32<TDT>(r.t, x);
        if constexpr (QK != DK_NONE) raw8_f32<QDT>(r.d, d);
        finish(x, d, w);
    }
    __device__ __forceinline__ void group(int64_t e0, float (&w)[8]) const {
        float x[8], d[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        ld8<TDT>(trow, e0, V, -INFINITY, x);
        if constexpr (QK == DK_PROBS) ld8<SPEC_F32>(drow, e0, V, 0.f, d);
        if constexpr (QK == DK_LOGITS) ld8<QDT>(drow, e0, V, -INFINITY, d);
        finish(x, d, w);
    }
};

// Inverse-CDF draw over a whole row with the weights wf (chunk masses, one
// chunk rescanned); *S receives the total.  -1 when the total is not positive.
template <int CH, int BT, class WF>
__device__ int draw_row(const WF& wf, int nch, float u, float* wpw, FinShared& sh, double* S) {
    *S = row_chunk_masses<CH, BT>(wf, nch, wpw, sh);
    return *S > 0.0 ? draw_from_chunks<CH, BT>(wf, nch, wf.V, (double)u * *S, u, sh) : -1;
}

// The last token of a filtered chain round for sequence b with k accepted:
// the correction from max(0, p'_k - q'_k) or, for k = gamma (or an empty
// residual), from p'_k, over the whole row (chunk masses, one chunk
// rescanned), with sh.m / sh.z / sh.th holding rows k and gamma + 1 + k.
// Writes out_tokens[b, k] and the S diagnostic.  All threads call it.
template <int TDT, int DDT, int DK>
__device__ void chain_filt_draw(const Params& P, int b, int k, float s, FinShared& sh, float* wpw) {
    constexpr int CH = chunk_elems<TDT>();
    constexpr int QDT = DK == DK_PROBS ? SPEC_F32 : DDT;
    const int gamma = P.gamma, V = P.V;
    const float u = P.final_u[b];
    const char* trow = P.tgt + ((size_t)b * (gamma + 1) + k) * P.tstride;
    const float mp = sh.m[k], izp = (float)(1.0 / sh.z[k]), thp = sh.th[k];
    double S;
    int y = -1;
    if (k < gamma) {
        const char* drow = P.drf + ((size_t)b * gamma + k) * P.dstride;
        const int rq = gamma + 1 + k;
        WFilt<TDT, QDT, DK> wf{trow, drow, s, mp, izp, thp, DK == DK_LOGITS ? sh.m[rq] : 0.f,
                               DK == DK_LOGITS ? (float)(1.0 / sh.z[rq]) : 0.f,
                               DK == DK_LOGITS ? sh.th[rq] : -INFINITY, V};
        y = draw_row<CH, SEQ_BT>(wf, P.nch, u, wpw, sh, &S);
    }
    if (y < 0) {                                     // bonus, or an empty residual (rounding only)
        WFilt<TDT, QDT, DK_NONE> wp{trow, nullptr, s, mp, izp, thp, 0.f, 0.f, -INFINITY, V};
        double S0;
        y = draw_row<CH, SEQ_BT>(wp, P.nch, u, wpw, sh, &S0);
        if (k == gamma) S = 1.0;
    }
    if (threadIdx.x == 0) {
        P.out_tokens[(size_t)b * (gamma + 1) + k] = y;
        if (P.diag) P.diag[(size_t)b * (2 * gamma + 1) + 2 * gamma] = (float)S;
    }
}

// Filtered chain finalisation, one CTA per sequence: the decision of
// chain_decide on the filtered distributions (p' and q' from each row's
// statistics, threshold and kept mass), then the correction from
// max(0, p'_k - q'_k) or the bonus from p'_gamma over the whole row.
template <int TDT, int DDT, int DK>
__global__ void __launch_bounds__(SEQ_BT) k_chain_final_filt(const Params P) {
    __shared__ FinShared sh;
    extern __shared__ __align__(128) unsigned char dyn[];
    const int tid = threadIdx.x, b = blockIdx.x;
    const int gamma = P.gamma;
    float* wpw = reinterpret_cast<float*>(dyn);
    const ChainPrefetch pf = chain_prefetch<TDT, DDT, DK>(P, b);
    pdl_wait();
    combine_softmax_rows<SEQ_BT>(P, P.stats + (size_t)b * P.R * P.nch * SPC, P.R, sh);
    __syncthreads();
    const int rows = (DK == DK_LOGITS) ? 2 * gamma + 1 : gamma + 1;
    for (int r = tid; r < rows; r += SEQ_BT) {
        const FiltRec f = P.filt[(size_t)b * P.R + r];
        sh.th[r] = f.theta;
        if (f.on > 0) sh.z[r] = f.Z;
        if (f.on < 0) sh.bad[r] = 1;                 // invalid top_k / top_p
    }
    __syncthreads();
    chain_decide<TDT, DDT, DK, true>(P, b, sh, true, pf);
    const int ok = sh.ivals[0], k = sh.ivals[1];
    if (!ok) return;
    chain_filt_draw<TDT, DDT, DK>(P, b, k, (float)sh.dvals[0], sh, wpw);
}

// Lazy filtered chain: the last token after the level walk, drawn as the
// dense filtered finalisation draws it, from the filter records the walk
// computed for the rows it reached.
template <int TDT, int DDT, int DK>
__global__ void __launch_bounds__(SEQ_BT) k_lz_chain_final_filt(const Params P) {
    __shared__ FinShared sh;
    extern __shared__ __align__(128) unsigned char dyn[];
    const int b = blockIdx.x, gamma = P.gamma;
    pdl_wait();
    chain_lazy_state(P, b, sh, true);
    const int ok = sh.ivals[0], k = sh.ivals[1];
    if (!ok) return;
    if (threadIdx.x == 0) {
        const FiltRec fp = P.filt[(size_t)b * P.R + k];
        sh.th[k] = fp.theta;
        if (fp.on > 0) sh.z[k] = fp.Z;
        if (DK == DK_LOGITS && k < gamma) {
            const FiltRec fq = P.filt[(size_t)b * P.R + gamma + 1 + k];
            sh.th[gamma + 1 + k] = fq.theta;
            if (fq.on > 0) sh.z[gamma + 1 + k] = fq.Z;
        }
    }
    __syncthreads();
    chain_filt_draw<TDT, DDT, DK>(P, b, k, (float)sh.dvals[0], sh, reinterpret_cast<float*>(dyn));
}

// ============================================================================= vocabulary-parallel chain verify
//
// The target (and draft) logits are sharded along the vocabulary over the
// ranks of a tensor-parallel group; rank r holds columns [off_r, off_r + Vs)
// of every row.  A round takes three small exchanges between four kernel
// steps (the collectives themselves are the caller's, e.g. NCCL):
//   stats    per row and shard: (m_r, Z_r) in the base-2 units of the
//            statistics, and the drafted token's logit (or draft
//            probability) when the token falls in the shard  -> all-gather
//   decide   every rank combines the shards' rows in rank order (m = max m_r,
//            Z = sum Z_r 2^(m_r - m), fp64) and takes the same decisions
//   residual the shard's mass of max(0, p_k - q_k) (or of p_gamma for the
//            bonus, from the statistics alone)                  -> all-gather
//   sample   every rank locates the shard holding u * S; that shard draws
//            inside itself, the others give -1                  -> all-reduce max
//   finish   the token goes to position k.

struct ShardRec {
    float m;          // max x of the shard's row (base-2 units), -inf if none
    float val;        // logit (or draft probability) at the drafted token, if in this shard
    double Z;         // sum 2^(x - m) over the shard's row
    int has;          // the drafted token lies in this shard
    int bad;          // NaN / +inf in the shard's row
};

// Per-sequence result of the decision, kept in the workspace for the
// residual and sample steps.
struct VpState {
    int k;            // accepted drafts; -1 invalid
    float s;          // log2(e) / T
    float mp, mq;     // global maxima of target row k and draft row k
    double zp, zq;    // global sums of target row k and draft row k
};

// stats: one warp per (sequence, row) of the shard, from k_stats' chunk
// statistics; rows 0..gamma target, gamma+1.. draft logits; with draft
// probabilities the draft "rows" only carry q(x).
template <int TDT, int DDT, int DK>
__global__ void __launch_bounds__(NT) k_vp_rows(const Params P, ShardRec* out, int off) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * NWARP + (threadIdx.x >> 5);
    const int R2 = 2 * P.gamma + 1;
    if (gw >= P.B * R2) return;
    const int b = gw / R2, r = gw - b * R2, gamma = P.gamma;
    ShardRec rec{-INFINITY, 0.f, 0.0, 0, 0};
    const int E = P.nch * SPC;
    if (r <= gamma || DK == DK_LOGITS) {
        const bool bd = warp_combine(P.stats + ((size_t)b * P.R + r) * E, E, rec.m, rec.Z);
        // an all -inf shard row is legal (the other shards hold the mass); NaN / +inf is not
        const float2* st = P.stats + ((size_t)b * P.R + r) * E;
        bool nan = false;
        for (int e = lane; e < E; e += 32) nan |= (st[e].y != st[e].y);
        rec.bad = __any_sync(FULL, nan) ? 1 : 0;
        if (!(rec.m > -INFINITY)) { rec.m = -INFINITY; rec.Z = 0.0; }
        (void)bd;
    }
    if (lane == 0) {
        const int i = r <= gamma ? r : r - gamma - 1;
        if (i < gamma) {
            const int x = P.draft_tokens[(size_t)b * gamma + i] - off;
            if (x >= 0 && x < P.V) {
                rec.has = 1;
                if (r <= gamma) {
                    rec.val = ld_elem<TDT>(P.tgt + ((size_t)b * (gamma + 1) + i) * P.tstride, x, P.V);
                } else {
                    const char* drow = P.drf + ((size_t)b * gamma + i) * P.dstride;
                    rec.val = (DK == DK_PROBS) ? __ldg(reinterpret_cast<const float*>(drow) + x) : ld_elem<DDT>(drow, x, P.V);
                }
            }
        }
        out[(size_t)b * R2 + r] = rec;
    }
}

// Shards' records are read VP_WB at a time into registers, so that their
// loads are in flight together rather than one per loop iteration.
constexpr int VP_WB = 8;

// Threads of the per-sequence residual and sampling kernels (the residual
// kernel four CTAs per SM; the sampling kernel, where only the owner shard's
// CTAs draw, two with more registers).
constexpr int VP_BT = 256;

// Global (m, Z) of row r of sequence b from all shards, in rank order, and
// how many shards hold the drafted token (with its value).  `softmax` false
// (a draft probability row): only the owners.
__device__ __forceinline__ void vp_combine(const ShardRec* all, int world, int B, int R2, int b, int r, bool softmax,
                                           float* m, double* Z, bool* bad, int* owners, float* val) {
    const size_t stride = (size_t)B * R2;
    const ShardRec* base = all + (size_t)b * R2 + r;
    float mm = -INFINITY, v = 0.f;
    bool bd = false;
    int own = 0;
    for (int w0 = 0; w0 < world; w0 += VP_WB) {
        float xm[VP_WB], xv[VP_WB];
        int xb[VP_WB], xh[VP_WB];
#pragma unroll
        for (int j = 0; j < VP_WB; ++j)
            if (w0 + j < world) {
                const ShardRec* x = base + (size_t)(w0 + j) * stride;
                xm[j] = x->m;
                xv[j] = x->val;
                xb[j] = x->bad;
                xh[j] = x->has;
            }
#pragma unroll
        for (int j = 0; j < VP_WB; ++j)
            if (w0 + j < world) {
                mm = fmaxf(mm, xm[j]);
                bd |= xb[j] != 0;
                if (xh[j]) { ++own; v = xv[j]; }
            }
    }
    *owners = own;
    *val = v;
    if (!softmax) {
        *m = 0.f;
        *Z = 1.0;
        *bad = false;
        return;
    }
    double z = 0.0;
    for (int w0 = 0; w0 < world; w0 += VP_WB) {
        float xm[VP_WB];
        double xz[VP_WB];
#pragma unroll
        for (int j = 0; j < VP_WB; ++j)
            if (w0 + j < world) {
                const ShardRec* x = base + (size_t)(w0 + j) * stride;
                xm[j] = x->m;
                xz[j] = x->Z;
            }
#pragma unroll
        for (int j = 0; j < VP_WB; ++j)
            if (w0 + j < world && xm[j] > -INFINITY) z += xz[j] * exp2((double)xm[j] - (double)mm);
    }
    *m = mm;
    *Z = z;
    *bad = bd || !(mm > -INFINITY) || !(mm < INFINITY) || !(z > 0.0) || !(z < 1e300);
}

// decide: one warp per sequence, identical on every rank (rule 1).  Lanes
// combine the rows over the shards (one row each, ranks in order) into
// shared memory; lane 0 then takes the decisions.
template <int DK>
__global__ void __launch_bounds__(NT) k_vp_decide(const Params P, const ShardRec* all, int world, VpState* vs) {
    constexpr int MR = 2 * SPEC_MAX_GAMMA + 1;
    __shared__ float sm_m[NWARP][MR], sm_v[NWARP][MR];
    __shared__ double sm_z[NWARP][MR];
    __shared__ int sm_ok[NWARP][MR];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int b = blockIdx.x * NWARP + warp;
    if (b >= P.B) return;
    const int gamma = P.gamma, R2 = 2 * gamma + 1;
    for (int r = lane; r < R2; r += 32) {
        float m, v;
        double Z;
        bool bad;
        int owners;
        vp_combine(all, world, P.B, R2, b, r, !(DK == DK_PROBS && r > gamma), &m, &Z, &bad, &owners, &v);
        const int i = r <= gamma ? r : r - gamma - 1;
        sm_m[warp][r] = m;
        sm_z[warp][r] = Z;
        sm_v[warp][r] = v;
        sm_ok[warp][r] = !bad && (i >= gamma || owners == 1);
    }
    __syncwarp();
    if (lane != 0) return;
    const float T = P.temperature[b];
    bool ok = temperature_ok(T);
    const float s = ok ? scale_of(T) : 0.f;
    int32_t* toks = P.out_tokens + (size_t)b * (gamma + 1);
    float* dg = P.diag ? P.diag + (size_t)b * (2 * gamma + 1) : nullptr;
    double px[SPEC_MAX_GAMMA], qx[SPEC_MAX_GAMMA];
    for (int r = 0; r < R2 && ok; ++r) ok &= sm_ok[warp][r] != 0;
    for (int i = 0; i < gamma && ok; ++i) {
        const int x = P.draft_tokens[(size_t)b * gamma + i];
        ok &= (x >= 0 && x < P.V);
        px[i] = exp2((double)sm_v[warp][i] * (double)s - (double)sm_m[warp][i]) / sm_z[warp][i];
        if constexpr (DK == DK_PROBS) {
            qx[i] = (double)sm_v[warp][gamma + 1 + i];
            ok &= (qx[i] >= 0.0 && qx[i] <= 3.0e38);
        } else {
            qx[i] = exp2((double)sm_v[warp][gamma + 1 + i] * (double)s - (double)sm_m[warp][gamma + 1 + i]) /
                    sm_z[warp][gamma + 1 + i];
        }
    }
    VpState st{-1, s, 0.f, 0.f, 0.0, 0.0};
    if (!ok) {
        for (int i = 0; i <= gamma; ++i) toks[i] = -1;
        P.out_num_accepted[b] = -1;
        if (dg) for (int i = 0; i < 2 * gamma + 1; ++i) dg[i] = nanf_();
        flag_input_error(P);
        vs[b] = st;
        return;
    }
    int k = gamma;
    for (int i = 0; i < gamma; ++i) {
        const double ratio = qx[i] > 0.0 ? px[i] / qx[i] : INFINITY;
        if (!((double)P.coins[(size_t)b * gamma + i] <= ratio)) { k = i; break; }
    }
    for (int i = 0; i < k; ++i) toks[i] = P.draft_tokens[(size_t)b * gamma + i];
    for (int i = k; i <= gamma; ++i) toks[i] = -1;
    P.out_num_accepted[b] = k;
    if (dg)
        for (int i = 0; i < gamma; ++i) { dg[i] = (float)px[i]; dg[gamma + i] = (float)qx[i]; }
    st.k = k;
    st.mp = sm_m[warp][k];
    st.zp = sm_z[warp][k];
    if (DK == DK_LOGITS && k < gamma) {
        st.mq = sm_m[warp][gamma + 1 + k];
        st.zq = sm_z[warp][gamma + 1 + k];
    }
    vs[b] = st;
}

// residual: the shard's part of the mass the last token is drawn from, one
// CTA per sequence -- sum over the shard of max(0, p_k - q_k) (k < gamma), or
// Z_r 2^(m_r - m) of row gamma (the bonus; no pass over the row).
template <int TDT, int DDT, int DK>
__global__ void __launch_bounds__(VP_BT, 4) k_vp_residual(const Params P, const ShardRec* all, int rank,
                                                         const VpState* vs, double* mass) {
    __shared__ FinShared sh;
    extern __shared__ __align__(128) unsigned char dyn[];
    constexpr int CH = chunk_elems<TDT>();
    const int b = blockIdx.x, gamma = P.gamma, R2 = 2 * gamma + 1;
    const VpState st = vs[b];
    double M = 0.0;
    if (st.k >= 0 && st.k < gamma) {
        const char* trow = P.tgt + ((size_t)b * (gamma + 1) + st.k) * P.tstride;
        const char* drow = P.drf + ((size_t)b * gamma + st.k) * P.dstride;
        WChainRes<TDT, DDT, DK> wf{trow, drow, st.s, st.mp, (float)(1.0 / st.zp), st.mq,
                                   DK == DK_PROBS ? 0.f : (float)(1.0 / st.zq), P.V};
        M = row_chunk_masses<CH, VP_BT>(wf, P.nch, reinterpret_cast<float*>(dyn), sh);
        for (int c = threadIdx.x; c < P.nch; c += VP_BT) P.vp_cm[(size_t)b * P.nch + c] = sh.M[c];
    } else if (st.k == gamma) {
        const ShardRec& x = all[((size_t)rank * P.B + b) * R2 + gamma];
        M = x.m > -INFINITY ? x.Z * exp2((double)x.m - (double)st.mp) : 0.0;
    }
    if (threadIdx.x == 0) mass[b] = M;
}

// The shard holding u * S among per-shard masses (smallest r with u*S below
// the running total, skipping empty shards; rounding past the end goes to
// the last non-empty one), or -1 when the total is not positive.
__device__ __forceinline__ int vp_owner(const double* ms, int world, int B, int b, double u, double* t_local,
                                        double* S) {
    double tot = 0.0;
    for (int w0 = 0; w0 < world; w0 += VP_WB) {
        double x[VP_WB];
#pragma unroll
        for (int j = 0; j < VP_WB; ++j)
            if (w0 + j < world) x[j] = ms[(size_t)(w0 + j) * B + b];
#pragma unroll
        for (int j = 0; j < VP_WB; ++j)
            if (w0 + j < world) tot += x[j];
    }
    *S = tot;
    if (!(tot > 0.0)) return -1;
    const double t = u * tot;
    double c = 0.0;
    int last = -1;
    double before_last = 0.0;
    for (int w0 = 0; w0 < world; w0 += VP_WB) {
        double x[VP_WB];
#pragma unroll
        for (int j = 0; j < VP_WB; ++j)
            if (w0 + j < world) x[j] = ms[(size_t)(w0 + j) * B + b];
#pragma unroll
        for (int j = 0; j < VP_WB; ++j)
            if (w0 + j < world) {
                if (x[j] > 0.0) {
                    if (t < c + x[j]) { *t_local = t - c; return w0 + j; }
                    last = w0 + j;
                    before_last = c;
                }
                c += x[j];
            }
    }
    *t_local = t - before_last;
    return last;
}

// sample: one CTA per sequence; every rank finds the owner shard from the
// gathered masses, the owner draws inside its shard (chunk masses of the same
// weights, one chunk rescanned) and writes the global token id, the others
// write -1.  An empty residual (rounding only) draws from p_k instead, with
// the shards' masses of p_k taken from the statistics.
template <int TDT, int DDT, int DK>
__global__ void __launch_bounds__(VP_BT, 2) k_vp_sample(const Params P, const ShardRec* all, int world, int rank,
                                                       int off, const VpState* vs, const double* mass_all,
                                                       int32_t* tok) {
    __shared__ FinShared sh;
    __shared__ double pk[64];
    extern __shared__ __align__(128) unsigned char dyn[];
    constexpr int CH = chunk_elems<TDT>();
    const int b = blockIdx.x, gamma = P.gamma, R2 = 2 * gamma + 1;
    const VpState st = vs[b];
    if (st.k < 0) {
        if (threadIdx.x == 0) tok[b] = -1;
        return;
    }
    const double u = (double)P.final_u[b];
    double tl = 0.0, S = 0.0;
    int owner = vp_owner(mass_all, world, P.B, b, u, &tl, &S);
    bool from_p = st.k == gamma;
    if (owner < 0 && st.k < gamma) {                 // empty residual: draw from p_k
        for (int w = threadIdx.x; w < world; w += VP_BT) {
            const ShardRec& x = all[((size_t)w * P.B + b) * R2 + st.k];
            pk[w] = x.m > -INFINITY ? x.Z * exp2((double)x.m - (double)st.mp) : 0.0;
        }
        __syncthreads();
        double Sp;
        owner = vp_owner(pk, world, 1, 0, u, &tl, &Sp);
        from_p = true;
    }
    int y = -1;
    if (owner == rank) {
        const char* trow = P.tgt + ((size_t)b * (gamma + 1) + st.k) * P.tstride;
        float* wpw = reinterpret_cast<float*>(dyn);
        if (from_p) {
            WTarget<TDT> wf{trow, st.s, st.mp, nullptr, 0, P.V};
            row_chunk_masses<CH, VP_BT>(wf, P.nch, wpw, sh);
            y = draw_from_chunks<CH, VP_BT>(wf, P.nch, P.V, tl, (float)u, sh);
        } else {
            const char* drow = P.drf + ((size_t)b * gamma + st.k) * P.dstride;
            WChainRes<TDT, DDT, DK> wf{trow, drow, st.s, st.mp, (float)(1.0 / st.zp), st.mq,
                                       DK == DK_PROBS ? 0.f : (float)(1.0 / st.zq), P.V};
            // the chunk masses k_vp_residual computed over the same weights
            for (int c = threadIdx.x; c < P.nch; c += VP_BT) sh.M[c] = P.vp_cm[(size_t)b * P.nch + c];
            __syncthreads();
            y = draw_from_chunks<CH, VP_BT>(wf, P.nch, P.V, tl, (float)u, sh);
        }
        if (y >= 0) y += off;
    }
    if (threadIdx.x == 0) {
        tok[b] = y;
        if (P.diag) P.diag[(size_t)b * (2 * gamma + 1) + 2 * gamma] = st.k == gamma ? 1.f : (float)S;
    }
}

// finish: the reduced token goes to position k.
__global__ void k_vp_finish(const Params P, const VpState* vs, const int32_t* tok) {
    const int b = blockIdx.x * NT + threadIdx.x;
    if (b >= P.B) return;
    const int k = vs[b].k;
    if (k >= 0) P.out_tokens[(size_t)b * (P.gamma + 1) + k] = tok[b];
}

// ============================================================================= lazy (row-on-demand) verification
//
// The verify rules need only some rows: the chain reads the target row (and
// draft row) of position i only if positions 0..i-1 were all accepted, and a
// tree walk reads the row of each node it visits.  The lazy entry points walk
// level by level -- statistics of the rows the active sequences need, then
// one decision per active sequence -- so a round reads about (accepted + 1)
// rows per sequence instead of all of them.  Each level is two programmatic
// dependent launches; the list of sequences still active at a level lives in
// the workspace, so the host never synchronises.  The row statistics have the
// dense path's layout and arithmetic, so every decision and draw is bit-for-
// bit the dense one; rows that are never read are not validated either.

// Sequence j of the current level's active list (level 0: every sequence).
__device__ __forceinline__ int lz_count_of(const Params& P) {
    return P.level == 0 ? P.B : (int)__ldcg(P.lz_count + P.level);
}
__device__ __forceinline__ int lz_seq_of(const Params& P, int j) {
    return P.level == 0 ? j : __ldcg(P.lz_list + (P.level & 1) * P.B + j);
}
// Append sequence b to the next level's active list.
__device__ __forceinline__ void lz_push(const Params& P, int b) {
    const unsigned j = atomicAdd(P.lz_count + P.level + 1, 1u);
    P.lz_list[((P.level + 1) & 1) * P.B + j] = b;
}

// Row statistics of the rows the active sequences need at this level: chain
// position `level` (target row, and the draft row when the draft is given as
// logits and level < gamma), or the current node of a tree walk.  Work items
// are (active sequence, row, chunk), split into contiguous ranges as in
// k_stats; the statistics land where the dense path puts them.  Level 0 also
// clears the per-level active counts.
template <int MODE, int TDT, int DDT>
__global__ void __launch_bounds__(NT, STATS_CTAS_PER_SM) k_lz_stats(const Params P) {
    constexpr int CH = chunk_elems<TDT>();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    pdl_trigger();
    pdl_wait();
    const int level = P.level;
    if (level == 0 && blockIdx.x == 0 && threadIdx.x <= LZ_MAX_LEVELS) P.lz_count[threadIdx.x] = 0u;
    const int nact = lz_count_of(P);
    const int rpl = (MODE == MODE_CHAIN && P.R > P.rows_tgt && level < P.gamma) ? 2 : 1;
    const int per_seq = rpl * P.nch;
    const long long total = (long long)nact * per_seq;
    const long long lo = total * blockIdx.x / gridDim.x;
    const long long n = total * (blockIdx.x + 1) / gridDim.x - lo;
    if (n <= 0) return;
    int j = (int)(lo / per_seq);
    int r, c;
    {
        const int rem = (int)(lo - (long long)j * per_seq);
        r = rem / P.nch;
        c = rem - r * P.nch;
    }
    int jb = -1, b = 0, node = 0;
    float s = 0.f;
    for (long long i = 0; i < n; ++i) {
        if (j != jb) {
            jb = j;
            b = lz_seq_of(P, j);
            if constexpr (MODE != MODE_GREEDY) s = scale_of(__ldg(P.temperature + b));
            if constexpr (MODE != MODE_CHAIN) node = level == 0 ? 0 : __ldcg(&P.lz_seq[b].cur);
        }
        float2 stat;
        int srow;
        if constexpr (MODE == MODE_GREEDY) {
            srow = node;
            stat = chunk_argmax<TDT>(P.tgt + ((size_t)b * P.R + node) * P.tstride, P.V, c);
        } else if constexpr (MODE == MODE_SAMPLE) {
            srow = node;
            stat = chunk_softmax<TDT, CH>(P.tgt + ((size_t)b * P.R + node) * P.tstride, P.V, c, s);
        } else {
            if (r == 0) {
                srow = level;
                stat = chunk_softmax<TDT, CH>(P.tgt + ((size_t)b * P.rows_tgt + level) * P.tstride, P.V, c, s);
            } else {
                srow = P.rows_tgt + level;
                stat = chunk_softmax<DDT, CH>(P.drf + ((size_t)b * P.gamma + level) * P.dstride, P.V, c, s);
            }
        }
        if (lane == 0) P.stats[(((size_t)b * P.R + srow) * P.nch + c) * SPC + warp] = stat;
        if (++c == P.nch) {
            c = 0;
            if (++r == rpl) { r = 0; ++j; }
        }
    }
}

// Chain decision at position `level` < gamma, one warp per active sequence:
// combine the row statistics, gather p(x) and q(x) at the drafted token, test
// coin <= p/q.  Accepted sequences move to the next level; a rejection leaves
// the sequence for the final kernel (residual at this position).  The
// temperature is checked at level 0; a bad row or token marks the sequence
// invalid.  Writes the p/q diagnostics of this position.
template <int TDT, int DDT, int DK, bool FILT = false>
__global__ void __launch_bounds__(NT) k_lz_decide_chain(const Params P) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int j = blockIdx.x * NWARP + (threadIdx.x >> 5);
    if (j >= lz_count_of(P)) return;
    const int b = lz_seq_of(P, j);
    const int level = P.level, gamma = P.gamma, E = P.nch * SPC;
    bool ok = true;
    float s;
    if (level == 0) {
        const float T = P.temperature[b];
        ok = temperature_ok(T);
        s = ok ? scale_of(T) : 0.f;
    } else {
        s = __ldcg(&P.lz_seq[b].s);
    }
    float m, mq = 0.f;
    double z, zq = 0.0;
    ok &= !warp_combine(P.stats + ((size_t)b * P.R + level) * E, E, m, z);
    if constexpr (DK != DK_PROBS) ok &= !warp_combine(P.stats + ((size_t)b * P.R + gamma + 1 + level) * E, E, mq, zq);
    if (lane != 0) return;
    const int x = P.draft_tokens[(size_t)b * gamma + level];
    ok &= (x >= 0 && x < P.V);
    float th = -INFINITY, thq = -INFINITY;
    if constexpr (FILT) {                       // the rows' filter records (this level's filter kernel)
        const FiltRec fp = P.filt[(size_t)b * P.R + level];
        ok &= fp.on >= 0;
        th = fp.theta;
        if (fp.on > 0) z = fp.Z;
        if constexpr (DK == DK_LOGITS) {
            const FiltRec fq = P.filt[(size_t)b * P.R + gamma + 1 + level];
            ok &= fq.on >= 0;
            thq = fq.theta;
            if (fq.on > 0) zq = fq.Z;
        }
    }
    double p = 0.0, q = 0.0;
    if (ok) {
        const float l = ld_elem<TDT>(P.tgt + ((size_t)b * (gamma + 1) + level) * P.tstride, x, P.V);
        p = (l >= th) ? prob_d(l, s, m, z) : 0.0;
        const char* drow = P.drf + ((size_t)b * gamma + level) * P.dstride;
        if constexpr (DK == DK_PROBS) {
            q = (double)__ldg(reinterpret_cast<const float*>(drow) + x);
            ok &= (q >= 0.0 && q <= 3.0e38);
        } else {
            const float d = ld_elem<DDT>(drow, x, P.V);
            q = (d >= thq) ? prob_d(d, s, mq, zq) : 0.0;
        }
    }
    LazySeq L;
    L.cur = level; L.nrej = 0; L.th = -INFINITY;
    L.s = s; L.m = m; L.mq = mq; L.z = z; L.zq = zq;
    if (!ok) {
        L.state = LZ_INVALID;
        L.k = -1;
        flag_input_error(P);
    } else {
        if (P.diag) {
            float* dg = P.diag + (size_t)b * (2 * gamma + 1);
            dg[level] = (float)p;
            dg[gamma + level] = (float)q;
        }
        const double ratio = (q > 0.0) ? p / q : INFINITY;
        if ((double)P.coins[(size_t)b * gamma + level] <= ratio) {
            L.state = LZ_ACTIVE;
            L.k = level + 1;
            lz_push(P, b);
        } else {
            L.state = LZ_DRAW;
            L.k = level;
        }
    }
    P.lz_seq[b] = L;
}

// Is sequence b's tree well formed (parents[0] = -1, 0 <= parents[n] < n,
// tokens in [0, V), depth <= max_depth)?  One warp.
__device__ bool warp_tree_valid(const Params& P, int b) {
    const int lane = threadIdx.x & 31, N = P.N;
    const int32_t* par = P.parents + (size_t)b * N;
    const int32_t* tok = P.tokens + (size_t)b * N;
    bool good = true;
    for (int n = lane; n < N; n += 32) {
        const int pa = par[n];
        good &= (n == 0) ? (pa == -1) : (pa >= 0 && pa < n && tok[n] >= 0 && tok[n] < P.V);
    }
    good = __all_sync(FULL, good);
    if (good) {
        for (int n = lane; n < N; n += 32) {
            int d = 0, a = n;
            while (a > 0 && d <= P.max_depth) { a = bounds_ok(a < N) ? par[a] : 0; ++d; }
            good &= d <= P.max_depth;
        }
        good = __all_sync(FULL, good);
    }
    return good;
}

// Tree walk at depth `level`, one warp per active sequence at node cur.
// Greedy: the first child of cur whose token is the argmax of row cur is
// accepted, else the walk ends with that argmax as the bonus token (written
// here: greedy needs no final kernel).  Sampling: the children of cur are
// tried in node order with the coin of cur against prob_acc / threshold_acc
// or p >= threshold_single; rejected children's tokens are kept for the final
// draw.  Level 0 validates the tree (and the temperature).  Diagnostics hold
// p_cur(token) for the children of visited nodes, NaN for the other nodes.
template <int MODE, int TDT, bool FILT = false>
__global__ void __launch_bounds__(NT) k_lz_decide_tree(const Params P) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int j = blockIdx.x * NWARP + (threadIdx.x >> 5);
    if (j >= lz_count_of(P)) return;
    const int b = lz_seq_of(P, j);
    const int level = P.level, N = P.N, W = P.max_depth + 1, E = P.nch * SPC;
    int32_t* ai = P.out_accept_index + (size_t)b * W;
    int32_t* ot = P.out_tokens + (size_t)b * W;
    float* dg = (MODE == MODE_SAMPLE && P.diag) ? P.diag + (size_t)b * (N + 1) : nullptr;
    const int32_t* par = P.parents + (size_t)b * N;
    const int32_t* tok = P.tokens + (size_t)b * N;
    LazySeq L;
    bool ok = true;
    if (level == 0) {
        ok = warp_tree_valid(P, b);
        L.cur = 0; L.k = 0; L.s = 0.f;
        if constexpr (MODE == MODE_SAMPLE) {
            const float T = P.temperature[b];
            ok &= temperature_ok(T);
            L.s = ok ? scale_of(T) : 0.f;
        }
        if (ok) {
            if (lane == 0) ai[0] = 0;
            if (dg) for (int n = lane; n < N; n += 32) dg[n] = n == 0 ? 0.f : nanf_();
            __syncwarp();
        }
    } else {
        L = P.lz_seq[b];
    }
    const int cur = L.cur, k = L.k;
    const float2* st = P.stats + ((size_t)b * P.R + cur) * E;
    int next = -1, nrej = 0;
    int g = 0;
    float m = 0.f;
    double z = 0.0;
    if (ok) {
        if constexpr (MODE == MODE_GREEDY) {
            ok = !warp_argmax(st, E, g);
            if (ok)
                for (int base = cur + 1; base < N && next < 0; base += 32) {
                    const int c = base + lane;
                    const unsigned hit = __ballot_sync(FULL, c < N && par[c] == cur && tok[c] == g);
                    if (hit) next = base + __ffs(hit) - 1;
                }
        } else {
            ok = !warp_combine(st, E, m, z);
            float th = -INFINITY;
            if constexpr (FILT) {                      // cur's filter record (k_lz_filter_tree)
                const FiltRec f = P.filt[(size_t)b * P.R + cur];
                if (f.on < 0) ok = false;
                if (f.on > 0) z = f.Z;
                th = f.theta;
                L.th = th;
            }
            if (ok) {
                const char* trow = P.tgt + ((size_t)b * N + cur) * P.tstride;
                const double coin = (double)P.coins[(size_t)b * N + cur];
                const double ths = (double)P.th_single, tha = (double)P.th_acc;
                int* rej = P.lz_rej + (size_t)b * P.rej_cap;
                double acc = 0.0;
                for (int base = cur + 1; base < N; base += 32) {
                    const int c = base + lane;
                    const bool child = c < N && par[c] == cur;
                    double pc = 0.0;
                    int t = 0;
                    if (child) {
                        t = tok[c];
                        const float l = ld_elem<TDT>(trow, t, P.V);
                        if (!FILT || l >= th) pc = prob_d(l, L.s, m, z);
                        if (dg) dg[c] = (float)pc;
                    }
                    unsigned msk = __ballot_sync(FULL, child);
                    while (msk && next < 0) {
                        const int l = __ffs(msk) - 1;
                        msk &= msk - 1;
                        const double p = __shfl_sync(FULL, pc, l);
                        const int tl = __shfl_sync(FULL, t, l);
                        acc += p;
                        if (coin <= acc / tha || p >= ths) next = base + l;
                        else {
                            if (lane == 0) rej[nrej] = tl;
                            ++nrej;
                        }
                    }
                }
            }
        }
    }
    if (lane != 0) return;
    if (!ok) {
        for (int i = 0; i < W; ++i) { ai[i] = -1; ot[i] = -1; }
        P.out_num_accepted[b] = -1;
        if (dg) for (int i = 0; i <= N; ++i) dg[i] = nanf_();
        flag_input_error(P);
        L.state = LZ_INVALID;
    } else if (next >= 0) {
        ot[k] = tok[next];
        ai[k + 1] = next;
        L.cur = next;
        L.k = k + 1;
        L.state = LZ_ACTIVE;
        lz_push(P, b);
    } else if constexpr (MODE == MODE_GREEDY) {
        ot[k] = g;
        for (int i = k + 1; i < W; ++i) { ot[i] = -1; ai[i] = -1; }
        P.out_num_accepted[b] = k;
        L.state = LZ_DONE;
    } else {
        L.state = LZ_DRAW;
        L.nrej = nrej;
        L.m = m;
        L.z = z;
    }
    P.lz_seq[b] = L;
}

// Lazy filtered tree walk: the filter record of the current node's row of
// every active sequence at this level (one CTA each, as k_filter), between
// the level's statistics and its decisions.
template <int TDT, int BT>
__global__ void __launch_bounds__(BT, BT == FILT_BT ? 1 : 3) k_lz_filter_tree(const Params P) {
    __shared__ FiltShared fs;
    __shared__ WinShared ws;
    extern __shared__ __align__(128) unsigned char dyn[];
    pdl_trigger();
    pdl_wait();
    if ((int)blockIdx.x >= lz_count_of(P)) return;
    const int b = lz_seq_of(P, blockIdx.x);
    const int cur = P.level == 0 ? 0 : P.lz_seq[b].cur;
    filter_one_row<TDT, BT>(P, b, cur, P.tgt + ((size_t)b * P.N + cur) * P.tstride, fs, ws, dyn);
}

// Lazy filtered chain, one CTA per still-active sequence: the filter records
// of target row `level` and, for draft logits below gamma, draft row `level`.
template <int TDT, int DDT, int DK, int BT>
__global__ void __launch_bounds__(BT, BT == FILT_BT ? 1 : 3) k_lz_filter_chain(const Params P) {
    __shared__ FiltShared fs;
    __shared__ WinShared ws;
    extern __shared__ __align__(128) unsigned char dyn[];
    pdl_trigger();
    pdl_wait();
    if ((int)blockIdx.x >= lz_count_of(P)) return;
    const int b = lz_seq_of(P, blockIdx.x);
    const int level = P.level, gamma = P.gamma;
    filter_one_row<TDT, BT>(P, b, level, P.tgt + ((size_t)b * (gamma + 1) + level) * P.tstride, fs, ws, dyn);
    if (DK == DK_LOGITS && level < gamma) {
        __syncthreads();
        filter_one_row<DDT, BT>(P, b, gamma + 1 + level, P.drf + ((size_t)b * gamma + level) * P.dstride, fs, ws,
                                dyn);
    }
}

// Lazy multi-step sampling walk, one CTA per active sequence at this level:
// level 0 validates the tree and the temperature; the current node's row is
// combined from its statistics; mss_node tests its children.  An accepted
// child moves the sequence to the next level; otherwise the last token is
// drawn here (mss_draw) and the sequence is done.
template <int TDT>
__global__ void __launch_bounds__(SEQ_BT) k_lz_decide_mss(const Params P) {
    __shared__ FinShared sh;
    extern __shared__ __align__(128) unsigned char dyn[];
    pdl_trigger();
    pdl_wait();
    if ((int)blockIdx.x >= lz_count_of(P)) return;
    const int b = lz_seq_of(P, blockIdx.x);
    const int tid = threadIdx.x, N = P.N, W = P.max_depth + 1, level = P.level;
    int32_t* ai = P.out_accept_index + (size_t)b * W;
    int32_t* ot = P.out_tokens + (size_t)b * W;
    float* dg = P.diag ? P.diag + (size_t)b * (N + 1) : nullptr;
    float* wpw = reinterpret_cast<float*>(dyn);
    for (int n = tid; n < N; n += SEQ_BT) {
        sh.par[n] = P.parents[(size_t)b * N + n];
        sh.tok[n] = P.tokens[(size_t)b * N + n];
    }
    __syncthreads();
    LazySeq L;
    int ok = 1;
    if (level == 0) {
        ok = tree_valid<SEQ_BT>(P, N, P.V, P.max_depth, sh);
        const float T = P.temperature[b];
        ok &= temperature_ok(T);
        L.cur = 0; L.k = 0; L.nrej = 0; L.th = -INFINITY;
        L.s = ok ? scale_of(T) : 0.f;
        L.mq = 0.f; L.zq = 0.0;
        if (ok) {
            if (tid == 0) ai[0] = 0;
            if (dg) for (int i = tid; i <= N; i += SEQ_BT) dg[i] = nanf_();
            __syncthreads();
        }
    } else {
        L = P.lz_seq[b];
    }
    if (ok) {
        if (tid < 32) {
            const int E = P.nch * SPC;
            float m;
            double z;
            const bool bad = warp_combine(P.stats + ((size_t)b * P.R + L.cur) * E, E, m, z);
            if (tid == 0) { sh.m[0] = m; sh.z[0] = z; sh.ivals[0] = !bad; }
        }
        __syncthreads();
        ok = sh.ivals[0];
        __syncthreads();
    }
    if (ok) {
        L.m = sh.m[0];
        L.z = sh.z[0];
        MssState st;
        const int next = mss_node<TDT, SEQ_BT>(P, b, L.cur, L.s, L.m, L.z, dg, wpw, sh, st);
        if (next == -2) {
            ok = 0;
        } else if (next >= 0) {
            if (tid == 0) {
                ot[L.k] = sh.tok[next];
                ai[L.k + 1] = next;
                L.cur = next;
                L.k += 1;
                L.state = LZ_ACTIVE;
                lz_push(P, b);
                P.lz_seq[b] = L;
            }
        } else {
            const int y = mss_draw<TDT, SEQ_BT>(P, b, L.cur, L.s, L.m, L.z, wpw, sh, st);
            if (tid == 0) {
                ot[L.k] = y;
                for (int i = L.k + 1; i < W; ++i) { ot[i] = -1; ai[i] = -1; }
                P.out_num_accepted[b] = L.k;
                if (dg) dg[N] = (float)st.S;
                L.state = LZ_DONE;
                P.lz_seq[b] = L;
            }
        }
    }
    if (!ok) {
        for (int i = tid; i < W; i += SEQ_BT) { ai[i] = -1; ot[i] = -1; }
        __syncthreads();
        if (dg) for (int i = tid; i <= N; i += SEQ_BT) dg[i] = nanf_();
        if (tid == 0) {
            P.out_num_accepted[b] = -1;
            flag_input_error(P);
            L.state = LZ_INVALID;
            P.lz_seq[b] = L;
        }
    }
}

// Last token of a lazy target-only tree walk, one CTA per sequence (those
// left in LZ_DRAW): tree_final_draw at the node where the walk stopped, with
// the rejected children's tokens it kept.  FILT: the dynamic shared memory
// holds the draw's per-warp chunk sums (P.nch * SEQ_BT/32 floats).
template <int TDT, bool FILT = false>
__global__ void __launch_bounds__(SEQ_BT) k_lz_tree_final(const Params P) {
    __shared__ FinShared sh;
    extern __shared__ __align__(128) unsigned char dyn[];
    pdl_wait();
    const int b = blockIdx.x, tid = threadIdx.x;
    const LazySeq L = P.lz_seq[b];
    if (L.state != LZ_DRAW) return;
    const int W = P.max_depth + 1;
    for (int i = tid; i < L.nrej; i += SEQ_BT) sh.rej[i] = P.lz_rej[(size_t)b * P.rej_cap + i];
    __syncthreads();
    double S;
    int y;
    if constexpr (FILT) {
        float* wpw = reinterpret_cast<float*>(dyn);
        y = P.draft_probs
                ? tree_filt_draw<TDT, SEQ_BT, true>(P, b, L.cur, sh.rej, L.nrej, L.s, L.m, L.z, L.th, wpw, sh, &S)
                : tree_filt_draw<TDT, SEQ_BT, false>(P, b, L.cur, sh.rej, L.nrej, L.s, L.m, L.z, L.th, wpw, sh, &S);
    } else {
        y = tree_final_draw<TDT, SEQ_BT>(P, b, L.cur, sh.rej, L.nrej, L.s, L.m, L.z, sh, &S);
    }
    if (tid == 0) {
        int32_t* ai = P.out_accept_index + (size_t)b * W;
        int32_t* ot = P.out_tokens + (size_t)b * W;
        ot[L.k] = y;
        for (int i = L.k + 1; i < W; ++i) { ot[i] = -1; ai[i] = -1; }
        P.out_num_accepted[b] = L.k;
        if (P.diag) P.diag[(size_t)b * (P.N + 1) + P.N] = (float)S;
    }
}

}  // namespace sv

// ============================================================================= host side

using namespace sv;

namespace {

thread_local char g_detail[512];

// An NVTX range around one C-ABI call (visible in Nsight Systems timelines;
// a no-op without a tool attached).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
thread_local cudaEvent_t g_prof_start = nullptr, g_prof_stop = nullptr;
thread_local unsigned g_wait_tries = WAIT_LIMIT;
thread_local unsigned g_filt_mode = 0u;
thread_local unsigned long long g_launches = 0;   // kernel launches issued by this host thread

cudaError_t record(cudaEvent_t ev, cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(st, &cs);
    if (e != cudaSuccess) return e;
    return cs == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal)
                                               : cudaEventRecord(ev, st);
}

spec_status fail(spec_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof g_detail, fmt, ap);
    va_end(ap);
    return st;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Layout {
    size_t status, cnt2, stats, stats2, lz_seq, lz_rej, lz_list, lz_count, filt, vp, vpcm, total;
    int rej_cap;
    int R, nch_max;
};

// Chunks are sized for the widest element (f32: 4096 per chunk) so that one
// workspace size serves both input dtypes.
Layout make_layout(int entry, int B, int rows, int V) {
    Layout L{};
    const int nch = (V + chunk_elems<SPEC_F32>() - 1) / chunk_elems<SPEC_F32>();
    L.nch_max = nch;
    L.R = (entry == SPEC_ENTRY_CHAIN) ? 2 * rows + 1 : rows;
    size_t off = 0;
    L.status = off; off = align256(off + 16);
    L.cnt2 = off; off = align256(off + sizeof(unsigned) * (size_t)B);
    L.stats = off; off = align256(off + sizeof(float2) * (size_t)B * L.R * nch * SPC);
    L.stats2 = off;
    if (entry == SPEC_ENTRY_CHAIN) off = align256(off + sizeof(float2) * (size_t)B * nch * NWARP);
    // lazy (row-on-demand) verification state
    L.lz_seq = off; off = align256(off + sizeof(LazySeq) * (size_t)B);
    L.rej_cap = (entry == SPEC_ENTRY_CHAIN) ? 1 : rows;
    L.lz_rej = off; off = align256(off + sizeof(int) * (size_t)B * L.rej_cap);
    L.lz_list = off; off = align256(off + sizeof(int) * 2 * (size_t)B);
    L.lz_count = off; off = align256(off + sizeof(unsigned) * (LZ_MAX_LEVELS + 1));
    // top-k / top-p filter records of the chain's rows (or of every tree node's row)
    L.filt = off;
    if (entry == SPEC_ENTRY_CHAIN || entry == SPEC_ENTRY_TREE_SAMPLE)
        off = align256(off + sizeof(FiltRec) * (size_t)B * L.R);
    // vocabulary-parallel chain: the decision's per-sequence state
    L.vp = off;
    if (entry == SPEC_ENTRY_CHAIN) off = align256(off + sizeof(VpState) * (size_t)B);
    // ... and the chunk masses of the shard's residual (reused by the draw)
    L.vpcm = off;
    if (entry == SPEC_ENTRY_CHAIN) off = align256(off + sizeof(double) * (size_t)B * nch);
    L.total = off;
    return L;
}

constexpr int MAX_DEVICES = 64;

// A value computed once per device ordinal (with that device current): kernel
// attributes set with cudaFuncSetAttribute and occupancy queries apply to the
// current device only, so a process that drives several GPUs needs each one's.
template <class T>
class PerDevice {
  public:
    template <class F>
    T get(F make) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return make();
        std::lock_guard<std::mutex> lock(mu_);
        if (!set_[dev]) {
            val_[dev] = make();
            set_[dev] = true;
        }
        return val_[dev];
    }

  private:
    std::mutex mu_;
    bool set_[MAX_DEVICES] = {};
    T val_[MAX_DEVICES] = {};
};

int num_sms() {
    static PerDevice<int> cache;
    return cache.get([] {
        int dev = 0, n = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        return n;
    });
}

template <class K>
int blocks_per_sm(K kernel) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, NT, 0) != cudaSuccess || n <= 0) n = 1;
    return n;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

spec_status check_rows(const char* what, const void* p, spec_dtype dt, int64_t stride, int V) {
    if (!p) return fail(SPEC_ERR_INVALID_ARG, "%s is NULL", what);
    if (dt != SPEC_F32 && dt != SPEC_BF16) return fail(SPEC_ERR_INVALID_ARG, "%s: unknown dtype %d", what, (int)dt);
    if (stride < V) return fail(SPEC_ERR_INVALID_ARG, "%s: row stride %lld < V %d", what, (long long)stride, V);
    const int esz = dt == SPEC_F32 ? 4 : 2;
    if (!aligned16(p)) return fail(SPEC_ERR_INVALID_ARG, "%s: base pointer not 16-byte aligned", what);
    if ((stride * esz) % 16 != 0)
        return fail(SPEC_ERR_INVALID_ARG, "%s: row stride * element size (%lld bytes) not a multiple of 16",
                    what, (long long)(stride * esz));
    return SPEC_OK;
}

spec_status check_ws(void* ws, size_t bytes, const Layout& L) {
    if (!ws) return fail(SPEC_ERR_WORKSPACE, "workspace is NULL");
    if (((uintptr_t)ws & 255u) != 0) return fail(SPEC_ERR_WORKSPACE, "workspace not 256-byte aligned");
    if (bytes < L.total)
        return fail(SPEC_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", bytes, L.total);
    return SPEC_OK;
}

void bind_ws(Params& P, void* ws, const Layout& L) {
    char* w = static_cast<char*>(ws);
    P.wait_tries = g_wait_tries;
    P.filt_mode = g_filt_mode;
    P.status = reinterpret_cast<unsigned*>(w + L.status);
    P.cnt2 = reinterpret_cast<unsigned*>(w + L.cnt2);
    P.stats = reinterpret_cast<float2*>(w + L.stats);
    P.stats2 = reinterpret_cast<float2*>(w + L.stats2);
    P.lz_seq = reinterpret_cast<LazySeq*>(w + L.lz_seq);
    P.lz_rej = reinterpret_cast<int*>(w + L.lz_rej);
    P.rej_cap = L.rej_cap;
    P.lz_list = reinterpret_cast<int*>(w + L.lz_list);
    P.lz_count = reinterpret_cast<unsigned*>(w + L.lz_count);
    P.filt = reinterpret_cast<FiltRec*>(w + L.filt);
    P.vp_cm = reinterpret_cast<double*>(w + L.vpcm);
}

spec_status launched(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(SPEC_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(e));
    ++g_launches;
    return SPEC_OK;
}

// Grid of a statistics kernel over `items` chunks with `occ` resident CTAs
// per SM.  Up to 4 CTAs per resident slot when every CTA would own many
// chunks (the extra CTAs start as others retire, which keeps the CTAs out of
// lockstep); then as few CTAs as give every CTA the same number of chunks
// (within one), so that no CTA trails the rest by a whole chunk.
unsigned stats_grid(long long items, int occ) {
    const long long resident = (long long)num_sms() * occ;
    long long mult = items / (8 * resident);
    mult = mult < 1 ? 1 : (mult > 4 ? 4 : mult);
    const long long slots = resident * mult;
    const long long per_cta = (items + slots - 1) / slots;
    return (unsigned)((items + per_cta - 1) / per_cta);
}

// Launch a kernel as a programmatic dependent of the kernel enqueued before it
// on `st` (the statistics kernel, a filter or level kernel): it may start
// while that kernel drains and waits for it (griddepcontrol.wait) before
// reading what that kernel writes.
template <class K>
spec_status launch_dependent(K kernel, unsigned grid, unsigned block, size_t smem, const Params& P,
                             cudaStream_t st, const char* what) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, P);
    if (e != cudaSuccess) return fail(SPEC_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(e));
    return launched(what);
}

template <int MODE, int TDT, int DDT>
spec_status launch_stats(const Params& P, cudaStream_t st) {
    auto kern = k_stats<MODE, TDT, DDT>;
    static PerDevice<int> occ_c;
    const int occ = occ_c.get([&] { return blocks_per_sm(kern); });
    const unsigned grid = stats_grid((long long)P.B * P.R * P.nch, occ);
    if (g_prof_start && record(g_prof_start, st) != cudaSuccess) return fail(SPEC_ERR_CUDA, "profile event");
    kern<<<grid, NT, 0, st>>>(P);
    spec_status s = launched("k_stats");
    if (s == SPEC_OK && g_prof_stop && record(g_prof_stop, st) != cudaSuccess)
        return fail(SPEC_ERR_CUDA, "profile event");
    return s;
}

// Shared memory for staging a sequence's statistics in the finalize kernels.
constexpr int STAGE_STATS_MAX = 96 * 1024;

// Allow a kernel `bytes` of dynamic shared memory on the current device.
template <class K>
bool allow_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) == cudaSuccess;
}

// Allow a finalize kernel STAGE_STATS_MAX bytes of dynamic shared memory.
template <class K>
bool allow_stage(K kernel) {
    return allow_smem(kernel, STAGE_STATS_MAX);
}


// Bytes of one sequence's statistics block, or 0 when it is not staged.
inline int stats_stage_bytes(const Params& P, int rows, size_t limit) {
    const size_t bytes = (size_t)rows * P.nch * SPC * sizeof(float2);
    return bytes <= limit ? (int)bytes : 0;
}

// Dynamic shared memory available to a pair-staged chain finalisation kernel
// (0 if it cannot be configured).
template <class K>
size_t stage_capacity(K kern) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return 0;
    int dev = 0, optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return 0;
    const long long cap = (long long)optin - (long long)fa.sharedSizeBytes - 1024;
    if (cap <= 0) return 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cap) != cudaSuccess) return 0;
    return (size_t)cap;
}

// Chain finalisation after the statistics (dense, LZ = false) or after the
// lazy level walk (LZ = true, which stages no statistics).
template <int TDT, int DDT, int DK, bool LZ>
spec_status launch_chain_final(Params P, cudaStream_t st) {
    constexpr int DESZ = DK == DK_PROBS ? 4 : Tr<DDT>::ESZ;
    // A pair of CTAs per sequence (a cluster) when each half of the rejected
    // row pair fits in shared memory and the pairs fit in a single wave; else
    // the sliced kernel.
    static PerDevice<size_t> cap2_c;
    const size_t cap2 = cap2_c.get([] { return stage_capacity(k_chain_final_pair<TDT, DDT, DK, LZ>); });
    const int G = (P.V + 7) / 8;
    const size_t half = staged_bytes(min(P.V, 8 * ((G + 1) / 2)), Tr<TDT>::ESZ, DESZ);
    if (P.nch > 1 && half <= cap2 && P.B <= num_sms()) {
        P.stage_off = (int)half;
        P.stage_cap = LZ ? 0 : stats_stage_bytes(P, P.R, cap2 - half);
        return launch_dependent(k_chain_final_pair<TDT, DDT, DK, LZ>, (unsigned)(2 * P.B), SEQ_BT,
                                half + P.stage_cap, P, st, "k_chain_final_pair");
    }
    static PerDevice<bool> big_c;
    const bool big = big_c.get([] { return allow_stage(k_chain_final<TDT, DDT, DK, LZ>); });
    P.stage_cap = LZ ? 0 : stats_stage_bytes(P, P.R, big ? STAGE_STATS_MAX : 48 * 1024 - 1024);
    // enough CTAs to cover the SMs twice, at most one per chunk
    int nsl = (2 * num_sms() + P.B - 1) / P.B;
    P.nsl = nsl < 1 ? 1 : (nsl > P.nch ? P.nch : nsl);
    return launch_dependent(k_chain_final<TDT, DDT, DK, LZ>, (unsigned)(P.B * P.nsl), NT, P.stage_cap, P, st,
                            "k_chain_final");
}

// Filtered chain: statistics, per-row filter thresholds, filtered finalisation.
template <int TDT, int DDT, int DK>
spec_status launch_chain_filtered(Params P, cudaStream_t st) {
    spec_status s = launch_stats<MODE_CHAIN, TDT, DK == DK_PROBS ? TDT : DDT>(P, st);
    if (s != SPEC_OK) return s;
    const int rows = (DK == DK_LOGITS) ? 2 * P.gamma + 1 : P.gamma + 1;
    // bf16 rows only: FILT_BT_BF16 threads, four rows per SM, the windowed
    // filter's 52 KB; else FILT_BT threads, a bf16 row's value histogram
    // (VH_BYTES), an f32 row's radix histograms
    constexpr bool any_bf16 = TDT == SPEC_BF16 || (DK == DK_LOGITS && DDT == SPEC_BF16);
    constexpr bool all_bf16 = TDT == SPEC_BF16 && (DK != DK_LOGITS || DDT == SPEC_BF16);
    constexpr int bt = all_bf16 ? FILT_BT_BF16 : FILT_BT;
    constexpr size_t hist = all_bf16 ? WF_BYTES : any_bf16 ? VH_BYTES : filt_hist_bytes<SPEC_F32>();
    auto kf = k_filter<TDT, DDT, DK, false, bt>;
    static PerDevice<bool> attr_c;
    const bool attr = attr_c.get([&] { return allow_smem(kf, hist); });
    if (!attr) return fail(SPEC_ERR_CUDA, "k_filter shared memory attribute");
    const size_t wpw = (size_t)P.nch * (SEQ_BT / 32) * sizeof(float);
    s = launch_dependent(kf, (unsigned)(P.B * rows), bt, hist, P, st, "k_filter");
    if (s != SPEC_OK) return s;
    return launch_dependent(k_chain_final_filt<TDT, DDT, DK>, (unsigned)P.B, SEQ_BT, wpw, P, st,
                            "k_chain_final_filt");
}

template <int TDT, int DDT, int DK>
spec_status launch_chain(Params P, cudaStream_t st) {
    // draft probabilities are read only by the finalize kernel
    spec_status s = launch_stats<MODE_CHAIN, TDT, DK == DK_PROBS ? TDT : DDT>(P, st);
    if (s != SPEC_OK) return s;
    return launch_chain_final<TDT, DDT, DK, false>(P, st);
}

template <int MODE, int TDT>
spec_status launch_tree(Params P, cudaStream_t st) {
    // the multi-step sampling walk uses the same softmax statistics as target-only sampling
    spec_status s = launch_stats<MODE == MODE_MSS ? MODE_SAMPLE : MODE, TDT, TDT>(P, st);
    if (s != SPEC_OK) return s;
    static PerDevice<bool> big_c;
    const bool big = big_c.get([] { return allow_stage(k_tree_final<MODE, TDT>); });
    P.stage_cap = stats_stage_bytes(P, P.N, big ? STAGE_STATS_MAX : 48 * 1024 - 1024);
    size_t smem = P.stage_cap;
    if (MODE == MODE_MSS) {
        // per-warp chunk sums of the residual passes after the statistics stage
        const size_t wpw = (size_t)P.nch * (SEQ_BT / 32) * sizeof(float);
        P.stage_cap = stats_stage_bytes(P, P.N, (big ? STAGE_STATS_MAX : 48 * 1024 - 1024) - wpw);
        P.stage_off = (P.stage_cap + 15) & ~15;
        smem = P.stage_off + wpw;
    }
    return launch_dependent(k_tree_final<MODE, TDT>, (unsigned)P.B, SEQ_BT, smem, P, st, "k_tree_final");
}

// Filtered target-only tree sampling: statistics, per-node-row filter
// thresholds, the filtered walk.
template <int TDT>
spec_status launch_tree_filtered(Params P, cudaStream_t st) {
    spec_status s = launch_stats<MODE_SAMPLE, TDT, TDT>(P, st);
    if (s != SPEC_OK) return s;
    if constexpr (TDT == SPEC_BF16) {
        // No diagnostics to fill: the walk filters only the rows it visits.
        if (P.diag == nullptr) {
            static PerDevice<bool> od_c;
            const bool od = od_c.get([] { return allow_stage(k_tree_final<MODE_SAMPLE_FILT_OD, TDT>); });
            P.stage_cap = stats_stage_bytes(P, P.N, (od ? STAGE_STATS_MAX : 48 * 1024 - 1024) - WF_BYTES);
            P.stage_off = (P.stage_cap + 15) & ~15;
            return launch_dependent(k_tree_final<MODE_SAMPLE_FILT_OD, TDT>, (unsigned)P.B, SEQ_BT,
                                    (size_t)P.stage_off + WF_BYTES, P, st, "k_tree_final");
        }
    }
    constexpr int bt = TDT == SPEC_BF16 ? FILT_BT_BF16 : FILT_BT;
    constexpr size_t hist = TDT == SPEC_BF16 ? WF_BYTES : filt_hist_bytes<SPEC_F32>();
    auto kf = k_filter<TDT, TDT, DK_NONE, true, bt>;
    static PerDevice<bool> attr_c;
    const bool attr = attr_c.get([&] { return allow_smem(kf, hist); });
    if (!attr) return fail(SPEC_ERR_CUDA, "k_filter shared memory attribute");
    s = launch_dependent(kf, (unsigned)(P.B * P.N), bt, hist, P, st, "k_filter");
    if (s != SPEC_OK) return s;
    static PerDevice<bool> big_c;
    const bool big = big_c.get([] { return allow_stage(k_tree_final<MODE_SAMPLE_FILT, TDT>); });
    // per-warp chunk sums of the final draw after the statistics stage
    const size_t wpw = (size_t)P.nch * (SEQ_BT / 32) * sizeof(float);
    P.stage_cap = stats_stage_bytes(P, P.N, (big ? STAGE_STATS_MAX : 48 * 1024 - 1024) - wpw);
    P.stage_off = (P.stage_cap + 15) & ~15;
    return launch_dependent(k_tree_final<MODE_SAMPLE_FILT, TDT>, (unsigned)P.B, SEQ_BT, (size_t)P.stage_off + wpw, P,
                            st, "k_tree_final");
}

// One level of the lazy walk: the statistics kernel (the first one as an
// ordinary launch, so the walk starts after all earlier work on the stream),
// then the decision kernel (none after the chain's bonus row).
template <class KS, class KD>
spec_status launch_level(KS ks, unsigned sgrid, KD kd, unsigned dgrid, Params& P, int level, cudaStream_t st,
                         unsigned dblock = NT, size_t dsmem = 0) {
    P.level = level;
    spec_status s;
    if (level == 0) {
        ks<<<sgrid, NT, 0, st>>>(P);
        s = launched("k_lz_stats");
    } else {
        s = launch_dependent(ks, sgrid, NT, 0, P, st, "k_lz_stats");
    }
    if (s != SPEC_OK || kd == nullptr) return s;
    return launch_dependent(kd, dgrid, dblock, dsmem, P, st, "k_lz_decide");
}

template <int TDT, int DDT, int DK>
spec_status launch_chain_lazy(Params P, cudaStream_t st) {
    auto ks = k_lz_stats<MODE_CHAIN, TDT, DK == DK_PROBS ? TDT : DDT>;
    auto kd = k_lz_decide_chain<TDT, DDT, DK>;
    static PerDevice<int> occ_c;
    const int occ = occ_c.get([&] { return blocks_per_sm(ks); });
    const int rpl = P.R > P.rows_tgt ? 2 : 1;
    const unsigned sgrid = stats_grid((long long)P.B * rpl * P.nch, occ);
    const unsigned dgrid = (unsigned)((P.B + NWARP - 1) / NWARP);
    if (g_prof_start && record(g_prof_start, st) != cudaSuccess) return fail(SPEC_ERR_CUDA, "profile event");
    for (int level = 0; level <= P.gamma; ++level) {
        spec_status s = launch_level(ks, sgrid, level < P.gamma ? kd : nullptr, dgrid, P, level, st);
        if (s != SPEC_OK) return s;
    }
    spec_status s = launch_chain_final<TDT, DDT, DK, true>(P, st);
    if (s == SPEC_OK && g_prof_stop && record(g_prof_stop, st) != cudaSuccess)
        return fail(SPEC_ERR_CUDA, "profile event");
    return s;
}

// Lazy filtered chain: per level the statistics of the rows the still-active
// sequences reach, their filter records, the decisions; then the draw.
template <int TDT, int DDT, int DK>
spec_status launch_chain_filtered_lazy(Params P, cudaStream_t st) {
    auto ks = k_lz_stats<MODE_CHAIN, TDT, DK == DK_PROBS ? TDT : DDT>;
    auto kd = k_lz_decide_chain<TDT, DDT, DK, true>;
    constexpr bool any_bf16 = TDT == SPEC_BF16 || (DK == DK_LOGITS && DDT == SPEC_BF16);
    constexpr int fbt = FILT_BT;
    constexpr size_t hist = any_bf16 ? VH_BYTES : filt_hist_bytes<SPEC_F32>();
    auto kf = k_lz_filter_chain<TDT, DDT, DK, fbt>;
    static PerDevice<bool> attr_c;
    const bool attr = attr_c.get([&] { return allow_smem(kf, hist); });
    if (!attr) return fail(SPEC_ERR_CUDA, "k_lz_filter_chain shared memory attribute");
    static PerDevice<int> occ_c;
    const int occ = occ_c.get([&] { return blocks_per_sm(ks); });
    const int rpl = P.R > P.rows_tgt ? 2 : 1;
    const unsigned sgrid = stats_grid((long long)P.B * rpl * P.nch, occ);
    const unsigned dgrid = (unsigned)((P.B + NWARP - 1) / NWARP);
    if (g_prof_start && record(g_prof_start, st) != cudaSuccess) return fail(SPEC_ERR_CUDA, "profile event");
    for (int level = 0; level <= P.gamma; ++level) {
        spec_status s = launch_level(ks, sgrid, (void (*)(Params))nullptr, 0, P, level, st);
        if (s != SPEC_OK) return s;
        s = launch_dependent(kf, (unsigned)P.B, fbt, hist, P, st, "k_lz_filter_chain");
        if (s != SPEC_OK) return s;
        if (level < P.gamma) {
            s = launch_dependent(kd, dgrid, NT, 0, P, st, "k_lz_decide");
            if (s != SPEC_OK) return s;
        }
    }
    const size_t wpw = (size_t)P.nch * (SEQ_BT / 32) * sizeof(float);
    spec_status s = launch_dependent(k_lz_chain_final_filt<TDT, DDT, DK>, (unsigned)P.B, SEQ_BT, wpw, P, st,
                                     "k_lz_chain_final_filt");
    if (s == SPEC_OK && g_prof_stop && record(g_prof_stop, st) != cudaSuccess)
        return fail(SPEC_ERR_CUDA, "profile event");
    return s;
}

template <int TDT>
spec_status launch_mss_lazy(Params P, cudaStream_t st) {
    auto ks = k_lz_stats<MODE_SAMPLE, TDT, TDT>;
    auto kd = k_lz_decide_mss<TDT>;
    static PerDevice<int> occ_c;
    const int occ = occ_c.get([&] { return blocks_per_sm(ks); });
    const unsigned sgrid = stats_grid((long long)P.B * P.nch, occ);
    const size_t wpw = (size_t)P.nch * (SEQ_BT / 32) * sizeof(float);
    if (g_prof_start && record(g_prof_start, st) != cudaSuccess) return fail(SPEC_ERR_CUDA, "profile event");
    for (int level = 0; level <= P.max_depth; ++level) {
        spec_status s = launch_level(ks, sgrid, kd, (unsigned)P.B, P, level, st, SEQ_BT, wpw);
        if (s != SPEC_OK) return s;
    }
    if (g_prof_stop && record(g_prof_stop, st) != cudaSuccess) return fail(SPEC_ERR_CUDA, "profile event");
    return SPEC_OK;
}

template <int MODE, int TDT>
spec_status launch_tree_lazy(Params P, cudaStream_t st) {
    auto ks = k_lz_stats<MODE, TDT, TDT>;
    auto kd = k_lz_decide_tree<MODE, TDT>;
    static PerDevice<int> occ_c;
    const int occ = occ_c.get([&] { return blocks_per_sm(ks); });
    const unsigned sgrid = stats_grid((long long)P.B * P.nch, occ);
    const unsigned dgrid = (unsigned)((P.B + NWARP - 1) / NWARP);
    if (g_prof_start && record(g_prof_start, st) != cudaSuccess) return fail(SPEC_ERR_CUDA, "profile event");
    for (int level = 0; level <= P.max_depth; ++level) {
        spec_status s = launch_level(ks, sgrid, kd, dgrid, P, level, st);
        if (s != SPEC_OK) return s;
    }
    spec_status s = SPEC_OK;
    if constexpr (MODE == MODE_SAMPLE)
        s = launch_dependent(k_lz_tree_final<TDT>, (unsigned)P.B, SEQ_BT, 0, P, st, "k_lz_tree_final");
    if (s == SPEC_OK && g_prof_stop && record(g_prof_stop, st) != cudaSuccess)
        return fail(SPEC_ERR_CUDA, "profile event");
    return s;
}

// Lazy filtered target-only tree sampling: per level the statistics of the
// current nodes' rows, their filter records, the decisions; then the draw.
template <int TDT>
spec_status launch_tree_filtered_lazy(Params P, cudaStream_t st) {
    auto ks = k_lz_stats<MODE_SAMPLE, TDT, TDT>;
    constexpr int fbt = FILT_BT;
    auto kf = k_lz_filter_tree<TDT, fbt>;
    auto kd = k_lz_decide_tree<MODE_SAMPLE, TDT, true>;
    static PerDevice<int> occ_c;
    const int occ = occ_c.get([&] { return blocks_per_sm(ks); });
    const unsigned sgrid = stats_grid((long long)P.B * P.nch, occ);
    const unsigned dgrid = (unsigned)((P.B + NWARP - 1) / NWARP);
    constexpr size_t hist = TDT == SPEC_BF16 ? VH_BYTES : filt_hist_bytes<SPEC_F32>();
    static PerDevice<bool> attr_c;
    const bool attr = attr_c.get([&] { return allow_smem(kf, hist); });
    if (!attr) return fail(SPEC_ERR_CUDA, "k_lz_filter_tree shared memory attribute");
    if (g_prof_start && record(g_prof_start, st) != cudaSuccess) return fail(SPEC_ERR_CUDA, "profile event");
    for (int level = 0; level <= P.max_depth; ++level) {
        spec_status s = launch_level(ks, sgrid, (void (*)(Params))nullptr, 0, P, level, st);
        if (s != SPEC_OK) return s;
        s = launch_dependent(kf, (unsigned)P.B, fbt, hist, P, st, "k_lz_filter_tree");
        if (s != SPEC_OK) return s;
        s = launch_dependent(kd, dgrid, NT, 0, P, st, "k_lz_decide");
        if (s != SPEC_OK) return s;
    }
    const size_t wpw = (size_t)P.nch * (SEQ_BT / 32) * sizeof(float);
    spec_status s = launch_dependent(k_lz_tree_final<TDT, true>, (unsigned)P.B, SEQ_BT, wpw, P, st, "k_lz_tree_final");
    if (s == SPEC_OK && g_prof_stop && record(g_prof_stop, st) != cudaSuccess)
        return fail(SPEC_ERR_CUDA, "profile event");
    return s;
}

}  // namespace

extern "C" {

size_t spec_workspace_bytes(int entry, int B, int rows, int V) {
    if (B < 0 || V < 1 || V > SPEC_MAX_V) return 0;
    if (entry == SPEC_ENTRY_CHAIN) {
        if (rows < 1 || rows > SPEC_MAX_GAMMA) return 0;
    } else if (entry == SPEC_ENTRY_TREE_GREEDY || entry == SPEC_ENTRY_TREE_SAMPLE || entry == SPEC_ENTRY_TREE_MSS) {
        if (rows < 1 || rows > SPEC_MAX_NODES) return 0;
    } else {
        return 0;
    }
    return make_layout(entry, B, rows, V).total;
}

spec_status spec_workspace_init(void* workspace, size_t bytes, void* stream) {
    if (!workspace) return fail(SPEC_ERR_WORKSPACE, "workspace is NULL");
    cudaError_t e = cudaMemsetAsync(workspace, 0, bytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(SPEC_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
    return SPEC_OK;
}

spec_status spec_read_device_status(void* workspace, int* status_out, void* stream) {
    if (!workspace || !status_out) return fail(SPEC_ERR_INVALID_ARG, "NULL workspace or status_out");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof v, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof v, st);
    if (e != cudaSuccess) return fail(SPEC_ERR_CUDA, "reading status: %s", cudaGetErrorString(e));
    *status_out = (int)v;
    return SPEC_OK;
}

const char* spec_status_string(spec_status s) {
    switch (s) {
        case SPEC_OK: return "ok";
        case SPEC_ERR_INVALID_ARG: return "invalid argument";
        case SPEC_ERR_UNSUPPORTED: return "unsupported";
        case SPEC_ERR_CUDA: return "CUDA error";
        case SPEC_ERR_DEVICE_INPUT: return "invalid device-side input in a sequence";
        case SPEC_ERR_TIMEOUT: return "device-side wait timed out";
        case SPEC_ERR_WORKSPACE: return "workspace too small or misaligned";
        case SPEC_ERR_COPY_IN_FLIGHT: return "a timed-out bulk copy may still have been in flight when its CTA went on";
    }
    return "unknown status";
}

const char* spec_last_error_detail(void) { return g_detail; }

unsigned long long spec_launch_count(void) { return g_launches; }

spec_status spec_debug_bounds_hits(unsigned long long* hits) {
    if (!hits) return fail(SPEC_ERR_INVALID_ARG, "hits is NULL");
#ifdef SPEC_DEBUG_BOUNDS
    unsigned long long zero = 0ull;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(hits, g_bounds_hits, sizeof *hits);
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_bounds_hits, &zero, sizeof zero);
    if (e != cudaSuccess) return fail(SPEC_ERR_CUDA, "bounds counter: %s", cudaGetErrorString(e));
    return SPEC_OK;
#else
    *hits = 0ull;
    return fail(SPEC_ERR_UNSUPPORTED, "this build has no bounds checks (compile with -DSPEC_DEBUG_BOUNDS)");
#endif
}

spec_status spec_debug_wait_budget(long long tries) {
    g_wait_tries = tries < 0 ? WAIT_LIMIT : (tries > (long long)WAIT_LIMIT ? WAIT_LIMIT : (unsigned)tries);
    return SPEC_OK;
}

spec_status spec_debug_filter_path(int mode, unsigned long long* rows) {
    if (mode < -1 || mode > 1) return fail(SPEC_ERR_INVALID_ARG, "mode = %d outside [-1, 1]", mode);
    if (rows) {
        unsigned long long zero[3] = {0ull, 0ull, 0ull};
        cudaError_t e = cudaMemcpyFromSymbol(rows, g_filter_rows, sizeof zero);
        if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_filter_rows, zero, sizeof zero);
        if (e != cudaSuccess) return fail(SPEC_ERR_CUDA, "filter row counters: %s", cudaGetErrorString(e));
    }
    if (mode >= 0) g_filt_mode = (mode == 1 ? 1u : 0u) | 2u;
    else g_filt_mode = 0u;
    return SPEC_OK;
}

spec_status spec_profile_events(void* start_event, void* stop_event) {
    g_prof_start = static_cast<cudaEvent_t>(start_event);
    g_prof_stop = static_cast<cudaEvent_t>(stop_event);
    return SPEC_OK;
}

}  // extern "C"

// Host-side argument checks of the chain entry points (everything except the
// workspace); B == 0 passes.
static spec_status chain_args(int B, int gamma, int V, const void* target_logits, spec_dtype tdt,
                              int64_t t_row_stride, const void* draft, spec_dtype ddt, int draft_is_probs,
                              int64_t d_row_stride, const int32_t* draft_tokens, const float* temperature,
                              const float* coins, const float* final_u, const int32_t* out_tokens,
                              const int32_t* out_num_accepted) {
    if (B < 0) return fail(SPEC_ERR_INVALID_ARG, "B = %d < 0", B);
    if (gamma < 1 || gamma > SPEC_MAX_GAMMA) return fail(SPEC_ERR_INVALID_ARG, "gamma = %d outside [1, %d]", gamma, SPEC_MAX_GAMMA);
    if (V < 1 || V > SPEC_MAX_V) return fail(SPEC_ERR_INVALID_ARG, "V = %d outside [1, %d]", V, SPEC_MAX_V);
    if (B == 0) return SPEC_OK;
    spec_status s = check_rows("target_logits", target_logits, tdt, t_row_stride, V);
    if (s != SPEC_OK) return s;
    if (draft_is_probs && ddt != SPEC_F32) return fail(SPEC_ERR_INVALID_ARG, "draft probabilities must be SPEC_F32");
    s = check_rows("draft", draft, ddt, d_row_stride, V);
    if (s != SPEC_OK) return s;
    if (!draft_tokens || !temperature || !coins || !final_u || !out_tokens || !out_num_accepted)
        return fail(SPEC_ERR_INVALID_ARG, "a required pointer is NULL");
    return SPEC_OK;
}

static spec_status chain_entry(int mode, int B, int gamma, int V,
                               const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                               const void* draft, spec_dtype ddt, int draft_is_probs,
                               int64_t d_row_stride,
                               const int32_t* draft_tokens, const float* temperature,
                               const float* coins, const float* final_u,
                               int32_t* out_tokens, int32_t* out_num_accepted, float* diag,
                               void* workspace, size_t workspace_bytes, void* stream,
                               const int32_t* top_k = nullptr, const float* top_p = nullptr) {
    g_detail[0] = 0;
    spec_status s = chain_args(B, gamma, V, target_logits, tdt, t_row_stride, draft, ddt, draft_is_probs,
                               d_row_stride, draft_tokens, temperature, coins, final_u, out_tokens,
                               out_num_accepted);
    if (s != SPEC_OK || B == 0) return s;
    const Layout L = make_layout(SPEC_ENTRY_CHAIN, B, gamma, V);
    s = check_ws(workspace, workspace_bytes, L);
    if (s != SPEC_OK) return s;
    Params P{};
    P.B = B; P.V = V; P.gamma = gamma;
    P.rows_tgt = gamma + 1;
    P.R = draft_is_probs ? gamma + 1 : 2 * gamma + 1;
    P.nch = (V + (tdt == SPEC_BF16 ? chunk_elems<SPEC_BF16>() : chunk_elems<SPEC_F32>()) - 1) /
            (tdt == SPEC_BF16 ? chunk_elems<SPEC_BF16>() : chunk_elems<SPEC_F32>());
    P.tgt = static_cast<const char*>(target_logits);
    P.tstride = t_row_stride * (tdt == SPEC_F32 ? 4 : 2);
    P.drf = static_cast<const char*>(draft);
    P.dstride = d_row_stride * (ddt == SPEC_F32 ? 4 : 2);
    P.draft_tokens = draft_tokens; P.temperature = temperature; P.coins = coins; P.final_u = final_u;
    P.out_tokens = out_tokens; P.out_num_accepted = out_num_accepted; P.diag = diag;
    P.top_k = top_k; P.top_p = top_p;
    bind_ws(P, workspace, L);
    // The statistics of a row are laid out with the chain's full row count so
    // that draft rows keep their offsets for either draft kind.
    cudaStream_t st = static_cast<cudaStream_t>(stream);
#define SPEC_CHAIN(T, D, K)                                                                          \
    return mode == 1   ? launch_chain_lazy<T, D, K>(P, st)                                           \
           : mode == 2 ? launch_chain_filtered<T, D, K>(P, st)                                       \
           : mode == 3 ? launch_chain_filtered_lazy<T, D, K>(P, st)                                  \
                       : launch_chain<T, D, K>(P, st)
    if (draft_is_probs) {
        if (tdt == SPEC_BF16) SPEC_CHAIN(SPEC_BF16, SPEC_F32, DK_PROBS);
        SPEC_CHAIN(SPEC_F32, SPEC_F32, DK_PROBS);
    }
    if (tdt == SPEC_BF16 && ddt == SPEC_BF16) SPEC_CHAIN(SPEC_BF16, SPEC_BF16, DK_LOGITS);
    if (tdt == SPEC_BF16 && ddt == SPEC_F32) SPEC_CHAIN(SPEC_BF16, SPEC_F32, DK_LOGITS);
    if (tdt == SPEC_F32 && ddt == SPEC_BF16) SPEC_CHAIN(SPEC_F32, SPEC_BF16, DK_LOGITS);
    SPEC_CHAIN(SPEC_F32, SPEC_F32, DK_LOGITS);
#undef SPEC_CHAIN
}

static spec_status tree_common(Params& P, int B, int N, int V, int max_depth,
                               const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                               const int32_t* tokens, const int32_t* parents,
                               int32_t* out_accept_index, int32_t* out_tokens, int32_t* out_num_accepted) {
    if (B < 0) return fail(SPEC_ERR_INVALID_ARG, "B = %d < 0", B);
    if (N < 1 || N > SPEC_MAX_NODES) return fail(SPEC_ERR_INVALID_ARG, "N = %d outside [1, %d]", N, SPEC_MAX_NODES);
    if (V < 1 || V > SPEC_MAX_V) return fail(SPEC_ERR_INVALID_ARG, "V = %d outside [1, %d]", V, SPEC_MAX_V);
    if (max_depth < 0 || max_depth > SPEC_MAX_DEPTH)
        return fail(SPEC_ERR_INVALID_ARG, "max_depth = %d outside [0, %d]", max_depth, SPEC_MAX_DEPTH);
    if (B == 0) return SPEC_OK;
    spec_status s = check_rows("target_logits", target_logits, tdt, t_row_stride, V);
    if (s != SPEC_OK) return s;
    if (!tokens || !parents || !out_accept_index || !out_tokens || !out_num_accepted)
        return fail(SPEC_ERR_INVALID_ARG, "a required pointer is NULL");
    P.B = B; P.N = N; P.V = V; P.max_depth = max_depth;
    P.R = N; P.rows_tgt = N;
    const int CH = tdt == SPEC_BF16 ? chunk_elems<SPEC_BF16>() : chunk_elems<SPEC_F32>();
    P.nch = (V + CH - 1) / CH;
    P.tgt = static_cast<const char*>(target_logits);
    P.tstride = t_row_stride * (tdt == SPEC_F32 ? 4 : 2);
    P.tokens = tokens; P.parents = parents;
    P.out_accept_index = out_accept_index; P.out_tokens = out_tokens; P.out_num_accepted = out_num_accepted;
    return SPEC_OK;
}

static spec_status greedy_entry(bool lazy, int B, int N, int V, int max_depth,
                                const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                                const int32_t* tokens, const int32_t* parents,
                                int32_t* out_accept_index, int32_t* out_tokens,
                                int32_t* out_num_accepted,
                                void* workspace, size_t workspace_bytes, void* stream) {
    g_detail[0] = 0;
    Params P{};
    spec_status s = tree_common(P, B, N, V, max_depth, target_logits, tdt, t_row_stride, tokens, parents,
                                out_accept_index, out_tokens, out_num_accepted);
    if (s != SPEC_OK || B == 0) return s;
    const Layout L = make_layout(SPEC_ENTRY_TREE_GREEDY, B, N, V);
    s = check_ws(workspace, workspace_bytes, L);
    if (s != SPEC_OK) return s;
    bind_ws(P, workspace, L);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (lazy) {
        if (tdt == SPEC_BF16) return launch_tree_lazy<MODE_GREEDY, SPEC_BF16>(P, st);
        return launch_tree_lazy<MODE_GREEDY, SPEC_F32>(P, st);
    }
    if (tdt == SPEC_BF16) return launch_tree<MODE_GREEDY, SPEC_BF16>(P, st);
    return launch_tree<MODE_GREEDY, SPEC_F32>(P, st);
}

static spec_status sample_entry(bool lazy, int B, int N, int V, int max_depth,
                                const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                                const int32_t* tokens, const int32_t* parents,
                                const float* temperature, const float* coins, const float* final_u,
                                const float* draft_probs, int64_t dp_row_stride,
                                float threshold_single, float threshold_acc,
                                int32_t* out_accept_index, int32_t* out_tokens,
                                int32_t* out_num_accepted, float* diag,
                                void* workspace, size_t workspace_bytes, void* stream,
                                const int32_t* top_k = nullptr, const float* top_p = nullptr) {
    g_detail[0] = 0;
    Params P{};
    spec_status s = tree_common(P, B, N, V, max_depth, target_logits, tdt, t_row_stride, tokens, parents,
                                out_accept_index, out_tokens, out_num_accepted);
    if (s != SPEC_OK || B == 0) return s;
    if (!temperature || !coins || !final_u) return fail(SPEC_ERR_INVALID_ARG, "a required pointer is NULL");
    if (!(threshold_single > 0.f) || !(threshold_acc > 0.f))
        return fail(SPEC_ERR_INVALID_ARG, "thresholds must be > 0");
    if (draft_probs) {
        s = check_rows("draft_probs", draft_probs, SPEC_F32, dp_row_stride, V);
        if (s != SPEC_OK) return s;
    }
    const Layout L = make_layout(SPEC_ENTRY_TREE_SAMPLE, B, N, V);
    s = check_ws(workspace, workspace_bytes, L);
    if (s != SPEC_OK) return s;
    bind_ws(P, workspace, L);
    P.temperature = temperature; P.coins = coins; P.final_u = final_u;
    P.draft_probs = draft_probs; P.dpstride = dp_row_stride * 4;
    P.th_single = threshold_single; P.th_acc = threshold_acc;
    P.diag = diag;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (top_k || top_p) {
        P.top_k = top_k; P.top_p = top_p;
        if (lazy) {
            if (tdt == SPEC_BF16) return launch_tree_filtered_lazy<SPEC_BF16>(P, st);
            return launch_tree_filtered_lazy<SPEC_F32>(P, st);
        }
        if (tdt == SPEC_BF16) return launch_tree_filtered<SPEC_BF16>(P, st);
        return launch_tree_filtered<SPEC_F32>(P, st);
    }
    if (lazy) {
        if (tdt == SPEC_BF16) return launch_tree_lazy<MODE_SAMPLE, SPEC_BF16>(P, st);
        return launch_tree_lazy<MODE_SAMPLE, SPEC_F32>(P, st);
    }
    if (tdt == SPEC_BF16) return launch_tree<MODE_SAMPLE, SPEC_BF16>(P, st);
    return launch_tree<MODE_SAMPLE, SPEC_F32>(P, st);
}

static spec_status mss_entry(bool lazy, int B, int N, int V, int max_depth,
                             const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                             const int32_t* tokens, const int32_t* parents,
                             const float* temperature, const float* coins, const float* final_u,
                             const float* draft_probs, int64_t dp_row_stride,
                             int32_t* out_accept_index, int32_t* out_tokens,
                             int32_t* out_num_accepted, float* diag,
                             void* workspace, size_t workspace_bytes, void* stream) {
    g_detail[0] = 0;
    Params P{};
    spec_status s = tree_common(P, B, N, V, max_depth, target_logits, tdt, t_row_stride, tokens, parents,
                                out_accept_index, out_tokens, out_num_accepted);
    if (s != SPEC_OK || B == 0) return s;
    if (!temperature || !coins || !final_u) return fail(SPEC_ERR_INVALID_ARG, "a required pointer is NULL");
    s = check_rows("draft_probs", draft_probs, SPEC_F32, dp_row_stride, V);
    if (s != SPEC_OK) return s;
    const Layout L = make_layout(SPEC_ENTRY_TREE_MSS, B, N, V);
    s = check_ws(workspace, workspace_bytes, L);
    if (s != SPEC_OK) return s;
    bind_ws(P, workspace, L);
    P.temperature = temperature; P.coins = coins; P.final_u = final_u;
    P.draft_probs = draft_probs; P.dpstride = dp_row_stride * 4;
    P.diag = diag;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (lazy) {
        if (tdt == SPEC_BF16) return launch_mss_lazy<SPEC_BF16>(P, st);
        return launch_mss_lazy<SPEC_F32>(P, st);
    }
    if (tdt == SPEC_BF16) return launch_tree<MODE_MSS, SPEC_BF16>(P, st);
    return launch_tree<MODE_MSS, SPEC_F32>(P, st);
}

#define SPEC_CHAIN_ARGS_DECL                                                                         \
    int B, int gamma, int V, const void* target_logits, spec_dtype tdt, int64_t t_row_stride,      \
        const void* draft, spec_dtype ddt, int draft_is_probs, int64_t d_row_stride,               \
        const int32_t* draft_tokens, const float* temperature, const float* coins,                 \
        const float* final_u, int32_t* out_tokens, int32_t* out_num_accepted, float* diag,         \
        void* workspace, size_t workspace_bytes, void* stream
#define SPEC_CHAIN_ARGS                                                                              \
    B, gamma, V, target_logits, tdt, t_row_stride, draft, ddt, draft_is_probs, d_row_stride,        \
        draft_tokens, temperature, coins, final_u, out_tokens, out_num_accepted, diag, workspace,   \
        workspace_bytes, stream
#define SPEC_GREEDY_ARGS_DECL                                                                        \
    int B, int N, int V, int max_depth, const void* target_logits, spec_dtype tdt,                 \
        int64_t t_row_stride, const int32_t* tokens, const int32_t* parents,                       \
        int32_t* out_accept_index, int32_t* out_tokens, int32_t* out_num_accepted,                 \
        void* workspace, size_t workspace_bytes, void* stream
#define SPEC_GREEDY_ARGS                                                                             \
    B, N, V, max_depth, target_logits, tdt, t_row_stride, tokens, parents, out_accept_index,        \
        out_tokens, out_num_accepted, workspace, workspace_bytes, stream
#define SPEC_SAMPLE_ARGS_DECL                                                                        \
    int B, int N, int V, int max_depth, const void* target_logits, spec_dtype tdt,                 \
        int64_t t_row_stride, const int32_t* tokens, const int32_t* parents,                       \
        const float* temperature, const float* coins, const float* final_u,                        \
        const float* draft_probs, int64_t dp_row_stride, float threshold_single,                   \
        float threshold_acc, int32_t* out_accept_index, int32_t* out_tokens,                       \
        int32_t* out_num_accepted, float* diag, void* workspace, size_t workspace_bytes, void* stream
#define SPEC_SAMPLE_ARGS                                                                             \
    B, N, V, max_depth, target_logits, tdt, t_row_stride, tokens, parents, temperature, coins,      \
        final_u, draft_probs, dp_row_stride, threshold_single, threshold_acc, out_accept_index,     \
        out_tokens, out_num_accepted, diag, workspace, workspace_bytes, stream

extern "C" {

spec_status spec_verify_chain(SPEC_CHAIN_ARGS_DECL) {
    NvtxRange nvtx("spec_verify_chain");
    return chain_entry(0, SPEC_CHAIN_ARGS);
}
spec_status spec_verify_chain_lazy(SPEC_CHAIN_ARGS_DECL) {
    NvtxRange nvtx("spec_verify_chain_lazy");
    return chain_entry(1, SPEC_CHAIN_ARGS);
}

spec_status spec_verify_chain_filtered(int B, int gamma, int V,
                                       const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                                       const void* draft, spec_dtype ddt, int draft_is_probs,
                                       int64_t d_row_stride,
                                       const int32_t* draft_tokens, const float* temperature,
                                       const float* coins, const float* final_u,
                                       const int32_t* top_k, const float* top_p,
                                       int32_t* out_tokens, int32_t* out_num_accepted, float* diag,
                                       void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx("spec_verify_chain_filtered");
    if (!top_k && !top_p) return fail(SPEC_ERR_INVALID_ARG, "top_k and top_p are both NULL");
    return chain_entry(2, B, gamma, V, target_logits, tdt, t_row_stride, draft, ddt, draft_is_probs,
                       d_row_stride, draft_tokens, temperature, coins, final_u, out_tokens, out_num_accepted,
                       diag, workspace, workspace_bytes, stream, top_k, top_p);
}
spec_status spec_verify_chain_filtered_lazy(int B, int gamma, int V,
                                            const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                                            const void* draft, spec_dtype ddt, int draft_is_probs,
                                            int64_t d_row_stride,
                                            const int32_t* draft_tokens, const float* temperature,
                                            const float* coins, const float* final_u,
                                            const int32_t* top_k, const float* top_p,
                                            int32_t* out_tokens, int32_t* out_num_accepted, float* diag,
                                            void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx("spec_verify_chain_filtered_lazy");
    if (!top_k && !top_p) return fail(SPEC_ERR_INVALID_ARG, "top_k and top_p are both NULL");
    return chain_entry(3, B, gamma, V, target_logits, tdt, t_row_stride, draft, ddt, draft_is_probs,
                       d_row_stride, draft_tokens, temperature, coins, final_u, out_tokens, out_num_accepted,
                       diag, workspace, workspace_bytes, stream, top_k, top_p);
}

spec_status spec_verify_tree_greedy(SPEC_GREEDY_ARGS_DECL) {
    NvtxRange nvtx("spec_verify_tree_greedy");
    return greedy_entry(false, SPEC_GREEDY_ARGS);
}
spec_status spec_verify_tree_greedy_lazy(SPEC_GREEDY_ARGS_DECL) {
    NvtxRange nvtx("spec_verify_tree_greedy_lazy");
    return greedy_entry(true, SPEC_GREEDY_ARGS);
}
spec_status spec_verify_tree_sample(SPEC_SAMPLE_ARGS_DECL) {
    NvtxRange nvtx("spec_verify_tree_sample");
    return sample_entry(false, SPEC_SAMPLE_ARGS);
}
spec_status spec_verify_tree_sample_lazy(SPEC_SAMPLE_ARGS_DECL) {
    NvtxRange nvtx("spec_verify_tree_sample_lazy");
    return sample_entry(true, SPEC_SAMPLE_ARGS);
}

spec_status spec_verify_tree_sample_filtered(int B, int N, int V, int max_depth, const void* target_logits,
                                             spec_dtype tdt, int64_t t_row_stride, const int32_t* tokens,
                                             const int32_t* parents, const float* temperature, const float* coins,
                                             const float* final_u, const float* draft_probs,
                                             int64_t dp_row_stride, float threshold_single, float threshold_acc,
                                             const int32_t* top_k, const float* top_p, int32_t* out_accept_index,
                                             int32_t* out_tokens, int32_t* out_num_accepted, float* diag,
                                             void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx("spec_verify_tree_sample_filtered");
    if (!top_k && !top_p) return fail(SPEC_ERR_INVALID_ARG, "top_k and top_p are both NULL");
    return sample_entry(false, B, N, V, max_depth, target_logits, tdt, t_row_stride, tokens, parents, temperature,
                        coins, final_u, draft_probs, dp_row_stride, threshold_single, threshold_acc,
                        out_accept_index, out_tokens, out_num_accepted, diag, workspace, workspace_bytes, stream,
                        top_k, top_p);
}

spec_status spec_verify_tree_sample_filtered_lazy(int B, int N, int V, int max_depth, const void* target_logits,
                                                  spec_dtype tdt, int64_t t_row_stride, const int32_t* tokens,
                                                  const int32_t* parents, const float* temperature,
                                                  const float* coins, const float* final_u, const float* draft_probs,
                                                  int64_t dp_row_stride, float threshold_single,
                                                  float threshold_acc, const int32_t* top_k, const float* top_p,
                                                  int32_t* out_accept_index, int32_t* out_tokens,
                                                  int32_t* out_num_accepted, float* diag, void* workspace,
                                                  size_t workspace_bytes, void* stream) {
    NvtxRange nvtx("spec_verify_tree_sample_filtered_lazy");
    if (!top_k && !top_p) return fail(SPEC_ERR_INVALID_ARG, "top_k and top_p are both NULL");
    return sample_entry(true, B, N, V, max_depth, target_logits, tdt, t_row_stride, tokens, parents, temperature,
                        coins, final_u, draft_probs, dp_row_stride, threshold_single, threshold_acc,
                        out_accept_index, out_tokens, out_num_accepted, diag, workspace, workspace_bytes, stream,
                        top_k, top_p);
}

#define SPEC_MSS_ARGS_DECL                                                                           \
    int B, int N, int V, int max_depth, const void* target_logits, spec_dtype tdt,                 \
        int64_t t_row_stride, const int32_t* tokens, const int32_t* parents,                       \
        const float* temperature, const float* coins, const float* final_u,                        \
        const float* draft_probs, int64_t dp_row_stride, int32_t* out_accept_index,                \
        int32_t* out_tokens, int32_t* out_num_accepted, float* diag, void* workspace,              \
        size_t workspace_bytes, void* stream
#define SPEC_MSS_ARGS                                                                                \
    B, N, V, max_depth, target_logits, tdt, t_row_stride, tokens, parents, temperature, coins,      \
        final_u, draft_probs, dp_row_stride, out_accept_index, out_tokens, out_num_accepted, diag,  \
        workspace, workspace_bytes, stream

spec_status spec_verify_tree_mss(SPEC_MSS_ARGS_DECL) {
    NvtxRange nvtx("spec_verify_tree_mss");
    return mss_entry(false, SPEC_MSS_ARGS);
}
spec_status spec_verify_tree_mss_lazy(SPEC_MSS_ARGS_DECL) {
    NvtxRange nvtx("spec_verify_tree_mss_lazy");
    return mss_entry(true, SPEC_MSS_ARGS);
}

}  // extern "C"

// ============================================================================= vocabulary-parallel chain entries

namespace {

// Common checks and Params of a shard step (V = the shard's width, or the full
// vocabulary for the decision).  target == NULL skips the row checks.
spec_status vp_params(Params& P, int B, int gamma, int V, const void* target, spec_dtype tdt, int64_t ts,
                      const void* draft, spec_dtype ddt, int draft_is_probs, int64_t ds, void* workspace,
                      size_t wsb, VpState** vs) {
    if (B < 1) return fail(SPEC_ERR_INVALID_ARG, "B = %d < 1", B);
    if (gamma < 1 || gamma > SPEC_MAX_GAMMA) return fail(SPEC_ERR_INVALID_ARG, "gamma = %d outside [1, %d]", gamma, SPEC_MAX_GAMMA);
    if (V < 1 || V > SPEC_MAX_V) return fail(SPEC_ERR_INVALID_ARG, "V = %d outside [1, %d]", V, SPEC_MAX_V);
    spec_status s = SPEC_OK;
    if (target) {
        s = check_rows("target_logits", target, tdt, ts, V);
        if (s != SPEC_OK) return s;
        if (draft_is_probs && ddt != SPEC_F32) return fail(SPEC_ERR_INVALID_ARG, "draft probabilities must be SPEC_F32");
        s = check_rows("draft", draft, ddt, ds, V);
        if (s != SPEC_OK) return s;
    }
    const Layout L = make_layout(SPEC_ENTRY_CHAIN, B, gamma, V);
    s = check_ws(workspace, wsb, L);
    if (s != SPEC_OK) return s;
    P.B = B; P.V = V; P.gamma = gamma;
    P.rows_tgt = gamma + 1;
    P.R = draft_is_probs ? gamma + 1 : 2 * gamma + 1;
    const int CH = tdt == SPEC_BF16 ? chunk_elems<SPEC_BF16>() : chunk_elems<SPEC_F32>();
    P.nch = (V + CH - 1) / CH;
    P.tgt = static_cast<const char*>(target);
    P.tstride = ts * (tdt == SPEC_F32 ? 4 : 2);
    P.drf = static_cast<const char*>(draft);
    P.dstride = ds * (ddt == SPEC_F32 ? 4 : 2);
    bind_ws(P, workspace, L);
    *vs = reinterpret_cast<VpState*>(static_cast<char*>(workspace) + L.vp);
    return SPEC_OK;
}

template <int TDT, int DDT, int DK>
spec_status vp_stats_launch(Params P, ShardRec* rec, int off, cudaStream_t st) {
    spec_status s = launch_stats<MODE_CHAIN, TDT, DK == DK_PROBS ? TDT : DDT>(P, st);
    if (s != SPEC_OK) return s;
    const unsigned grid = (unsigned)(((long long)P.B * (2 * P.gamma + 1) + NWARP - 1) / NWARP);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NT);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_vp_rows<TDT, DDT, DK>, P, rec, off);
    if (e != cudaSuccess) return fail(SPEC_ERR_CUDA, "k_vp_rows launch: %s", cudaGetErrorString(e));
    return launched("k_vp_rows");
}

template <int TDT, int DDT, int DK>
spec_status vp_residual_launch(Params P, const ShardRec* all, int rank, const VpState* vs, double* mass,
                               cudaStream_t st) {
    const size_t wpw = (size_t)P.nch * (VP_BT / 32) * sizeof(float);
    k_vp_residual<TDT, DDT, DK><<<(unsigned)P.B, VP_BT, wpw, st>>>(P, all, rank, vs, mass);
    return launched("k_vp_residual");
}

template <int TDT, int DDT, int DK>
spec_status vp_sample_launch(Params P, const ShardRec* all, int world, int rank, int off, const VpState* vs,
                             const double* mass_all, int32_t* tok, cudaStream_t st) {
    const size_t wpw = (size_t)P.nch * (VP_BT / 32) * sizeof(float);
    k_vp_sample<TDT, DDT, DK><<<(unsigned)P.B, VP_BT, wpw, st>>>(P, all, world, rank, off, vs, mass_all, tok);
    return launched("k_vp_sample");
}

#define SPEC_VP_DISPATCH(CALL)                                                                       \
    do {                                                                                             \
        if (draft_is_probs) {                                                                        \
            if (tdt == SPEC_BF16) return CALL(SPEC_BF16, SPEC_F32, DK_PROBS);                        \
            return CALL(SPEC_F32, SPEC_F32, DK_PROBS);                                               \
        }                                                                                            \
        if (tdt == SPEC_BF16 && ddt == SPEC_BF16) return CALL(SPEC_BF16, SPEC_BF16, DK_LOGITS);      \
        if (tdt == SPEC_BF16 && ddt == SPEC_F32) return CALL(SPEC_BF16, SPEC_F32, DK_LOGITS);        \
        if (tdt == SPEC_F32 && ddt == SPEC_BF16) return CALL(SPEC_F32, SPEC_BF16, DK_LOGITS);        \
        return CALL(SPEC_F32, SPEC_F32, DK_LOGITS);                                                  \
    } while (0)

}  // namespace

extern "C" {

size_t spec_vp_record_bytes(void) { return sizeof(ShardRec); }

spec_status spec_vp_chain_stats(int B, int gamma, int V_shard, int vocab_offset,
                                const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                                const void* draft, spec_dtype ddt, int draft_is_probs, int64_t d_row_stride,
                                const int32_t* draft_tokens, const float* temperature, void* rec_out,
                                void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx("spec_vp_chain_stats");
    g_detail[0] = 0;
    if (!target_logits || !draft_tokens || !temperature || !rec_out)
        return fail(SPEC_ERR_INVALID_ARG, "a required pointer is NULL");
    if (vocab_offset < 0) return fail(SPEC_ERR_INVALID_ARG, "vocab_offset < 0");
    Params P{};
    VpState* vs;
    spec_status s = vp_params(P, B, gamma, V_shard, target_logits, tdt, t_row_stride, draft, ddt, draft_is_probs,
                              d_row_stride, workspace, workspace_bytes, &vs);
    if (s != SPEC_OK) return s;
    P.draft_tokens = draft_tokens;
    P.temperature = temperature;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    ShardRec* rec = static_cast<ShardRec*>(rec_out);
#define SPEC_VP_STATS(T, D, K) vp_stats_launch<T, D, K>(P, rec, vocab_offset, st)
    SPEC_VP_DISPATCH(SPEC_VP_STATS);
#undef SPEC_VP_STATS
}

spec_status spec_vp_chain_decide(int B, int gamma, int V, int V_shard, int world, const void* rec_all,
                                 int draft_is_probs,
                                 const int32_t* draft_tokens, const float* temperature, const float* coins,
                                 int32_t* out_tokens, int32_t* out_num_accepted, float* diag,
                                 void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx("spec_vp_chain_decide");
    g_detail[0] = 0;
    if (world < 1 || world > 64) return fail(SPEC_ERR_INVALID_ARG, "world = %d outside [1, 64]", world);
    if (!rec_all || !draft_tokens || !temperature || !coins || !out_tokens || !out_num_accepted)
        return fail(SPEC_ERR_INVALID_ARG, "a required pointer is NULL");
    if (V < 1 || V > SPEC_MAX_V) return fail(SPEC_ERR_INVALID_ARG, "V = %d outside [1, %d]", V, SPEC_MAX_V);
    Params P{};
    VpState* vs;
    spec_status s = vp_params(P, B, gamma, V_shard, nullptr, SPEC_BF16, 0, nullptr, SPEC_BF16, draft_is_probs, 0,
                              workspace, workspace_bytes, &vs);
    if (s != SPEC_OK) return s;
    P.V = V;                                     // drafted tokens range over the whole vocabulary
    P.draft_tokens = draft_tokens; P.temperature = temperature; P.coins = coins;
    P.out_tokens = out_tokens; P.out_num_accepted = out_num_accepted; P.diag = diag;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const unsigned grid = (unsigned)((B + NWARP - 1) / NWARP);
    if (draft_is_probs) k_vp_decide<DK_PROBS><<<grid, NT, 0, st>>>(P, static_cast<const ShardRec*>(rec_all), world, vs);
    else k_vp_decide<DK_LOGITS><<<grid, NT, 0, st>>>(P, static_cast<const ShardRec*>(rec_all), world, vs);
    return launched("k_vp_decide");
}

spec_status spec_vp_chain_residual(int B, int gamma, int V_shard, int world, int rank,
                                   const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                                   const void* draft, spec_dtype ddt, int draft_is_probs, int64_t d_row_stride,
                                   const void* rec_all, double* mass_out,
                                   void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx("spec_vp_chain_residual");
    g_detail[0] = 0;
    if (world < 1 || world > 64 || rank < 0 || rank >= world)
        return fail(SPEC_ERR_INVALID_ARG, "rank %d / world %d", rank, world);
    if (!target_logits || !rec_all || !mass_out) return fail(SPEC_ERR_INVALID_ARG, "a required pointer is NULL");
    Params P{};
    VpState* vs;
    spec_status s = vp_params(P, B, gamma, V_shard, target_logits, tdt, t_row_stride, draft, ddt, draft_is_probs,
                              d_row_stride, workspace, workspace_bytes, &vs);
    if (s != SPEC_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const ShardRec* all = static_cast<const ShardRec*>(rec_all);
#define SPEC_VP_RES(T, D, K) vp_residual_launch<T, D, K>(P, all, rank, vs, mass_out, st)
    SPEC_VP_DISPATCH(SPEC_VP_RES);
#undef SPEC_VP_RES
}

spec_status spec_vp_chain_sample(int B, int gamma, int V_shard, int vocab_offset, int world, int rank,
                                 const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                                 const void* draft, spec_dtype ddt, int draft_is_probs, int64_t d_row_stride,
                                 const float* final_u, const void* rec_all, const double* mass_all,
                                 int32_t* tok_out, float* diag,
                                 void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx("spec_vp_chain_sample");
    g_detail[0] = 0;
    if (world < 1 || world > 64 || rank < 0 || rank >= world)
        return fail(SPEC_ERR_INVALID_ARG, "rank %d / world %d", rank, world);
    if (!target_logits || !final_u || !rec_all || !mass_all || !tok_out)
        return fail(SPEC_ERR_INVALID_ARG, "a required pointer is NULL");
    Params P{};
    VpState* vs;
    spec_status s = vp_params(P, B, gamma, V_shard, target_logits, tdt, t_row_stride, draft, ddt, draft_is_probs,
                              d_row_stride, workspace, workspace_bytes, &vs);
    if (s != SPEC_OK) return s;
    P.final_u = final_u;
    P.diag = diag;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const ShardRec* all = static_cast<const ShardRec*>(rec_all);
#define SPEC_VP_SAMPLE(T, D, K) vp_sample_launch<T, D, K>(P, all, world, rank, vocab_offset, vs, mass_all, tok_out, st)
    SPEC_VP_DISPATCH(SPEC_VP_SAMPLE);
#undef SPEC_VP_SAMPLE
}

spec_status spec_vp_chain_finish(int B, int gamma, int V_shard, const int32_t* tok, int32_t* out_tokens,
                                 void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx("spec_vp_chain_finish");
    g_detail[0] = 0;
    if (!tok || !out_tokens) return fail(SPEC_ERR_INVALID_ARG, "a required pointer is NULL");
    Params P{};
    VpState* vs;
    spec_status s = vp_params(P, B, gamma, V_shard, nullptr, SPEC_BF16, 0, nullptr, SPEC_BF16, 0, 0, workspace,
                              workspace_bytes, &vs);
    if (s != SPEC_OK) return s;
    P.out_tokens = out_tokens;
    k_vp_finish<<<(unsigned)((B + NT - 1) / NT), NT, 0, static_cast<cudaStream_t>(stream)>>>(P, vs, tok);
    return launched("k_vp_finish");
}

}  // extern "C"

// ============================================================================= no-allocation variant
//
// Some callers cannot allocate device memory at the point where they verify:
// a plugin inside a serving engine whose own allocator owns every byte of the
// GPU, code that must not pay the implicit device-wide synchronisation that
// cudaMalloc/cudaFree can cause in a latency-critical decode loop, or a host
// thread that holds no allocator at all.  For them spec_verify_chain_noalloc
// runs the same kernels on a scratch area compiled into the library.

// The scratch area: SPEC_NOALLOC_SCRATCH_BYTES on every GPU that loads this
// library, held until the process exits.  In host code this name is only a
// host-side stand-in; the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SPEC_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[256] = {};

// Device address of the scratch area on the current device, looked up once per
// device (with that device current) and cached.
spec_status noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(SPEC_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= 256) return fail(SPEC_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return fail(SPEC_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return SPEC_OK;
}

}  // namespace

extern "C" spec_status spec_verify_chain_noalloc(int B, int gamma, int V,
                                                 const void* target_logits, spec_dtype tdt,
                                                 int64_t t_row_stride,
                                                 const void* draft, spec_dtype ddt, int draft_is_probs,
                                                 int64_t d_row_stride,
                                                 const int32_t* draft_tokens, const float* temperature,
                                                 const float* coins, const float* final_u,
                                                 int32_t* out_tokens, int32_t* out_num_accepted,
                                                 float* diag, void* stream) {
    NvtxRange nvtx("spec_verify_chain_noalloc");
    g_detail[0] = 0;
    if (B < 0) return fail(SPEC_ERR_INVALID_ARG, "B = %d < 0", B);
    if (gamma < 1 || gamma > SPEC_MAX_GAMMA) return fail(SPEC_ERR_INVALID_ARG, "gamma = %d outside [1, %d]", gamma, SPEC_MAX_GAMMA);
    if (V < 1 || V > SPEC_MAX_V) return fail(SPEC_ERR_INVALID_ARG, "V = %d outside [1, %d]", V, SPEC_MAX_V);
    if (B == 0) return SPEC_OK;
    const Layout L = make_layout(SPEC_ENTRY_CHAIN, B, gamma, V);
    if (L.total > (size_t)SPEC_NOALLOC_SCRATCH_BYTES)
        return fail(SPEC_ERR_WORKSPACE,
                    "B=%d gamma=%d V=%d needs %zu bytes of scratch; the built-in scratch holds %zu "
                    "(use spec_verify_chain with a caller workspace)",
                    B, gamma, V, L.total, (size_t)SPEC_NOALLOC_SCRATCH_BYTES);
    // every other argument check runs before anything is enqueued on the
    // shared array
    spec_status s = chain_args(B, gamma, V, target_logits, tdt, t_row_stride, draft, ddt, draft_is_probs,
                               d_row_stride, draft_tokens, temperature, coins, final_u, out_tokens,
                               out_num_accepted);
    if (s != SPEC_OK) return s;
    void* scratch = nullptr;
    s = noalloc_scratch(&scratch);
    if (s != SPEC_OK) return s;
    // The area keeps whatever the previous call left there: clear the status
    // word and the arrival counters (everything before the statistics), the
    // only parts that must start at zero.
    cudaError_t e = cudaMemsetAsync(scratch, 0, L.stats, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(SPEC_ERR_CUDA, "cudaMemsetAsync(scratch): %s", cudaGetErrorString(e));
    return spec_verify_chain(B, gamma, V, target_logits, tdt, t_row_stride, draft, ddt, draft_is_probs,
                             d_row_stride, draft_tokens, temperature, coins, final_u, out_tokens,
                             out_num_accepted, diag, scratch, (size_t)SPEC_NOALLOC_SCRATCH_BYTES, stream);
}

