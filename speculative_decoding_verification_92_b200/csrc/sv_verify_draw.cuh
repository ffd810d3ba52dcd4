// sv_verify_draw.cuh -- K2, acceptance scan and the final draw.
//
// One thread-block cluster per request, of C2 = ceil(C / R) CTAs; CTA c of
// the cluster owns the R consecutive vocabulary chunks c*R .. c*R+R-1 of the
// row that the final draw uses.
//
//  1. validate draft_lens[b] and the first L drafted ids (bad values never
//     cause an access: the request is reported with out_accept_len = -1);
//  2. merge the C row-statistics partials of every used row into lse (log2
//     domain) -- or into the row argmax for greedy verification;
//  3. p_i = 2^(z_i(x_i)/T*log2e - lse_i), q_i likewise or 1 for one-hot q,
//     a_i = min(1, p_i/q_i), reject when !(u_i < a_i); j = first rejection
//     ("AI 开始抄自己的作业——而且抄得理直气壮", section "⚡ 投机解码：让草稿先跑，
//     考官殿后"; stop at the first rejection: "今热点：让AI草稿模型学会"照镜子"",
//     section "先搞懂投机解码在干什么");
//  4. final draw on row j with uniforms[b][k_max]:
//       bonus (j == L):     w = p_L, chunk sums straight from the K1 partials;
//       one-hot rejection:  w = p_j with the drafted id removed, same;
//       draft rejection:    w = max(0, p_j - q_j); every CTA runs the draw
//                           pass over its chunks and the chunk sums are
//                           exchanged through distributed shared memory and
//                           a cluster barrier;
//     every CTA locates the chunk k* holding u*W, and only its owner goes on.
//  5. inverse CDF inside chunk k*.  The draw pass streams a chunk through a
//     small shared-memory ring filled by 16-byte cp.async copies (each thread
//     reads back only what it copied, so the ring needs no block barrier) and
//     keeps one weight sum per segment of 32 vectors.  A warp then picks the
//     segment (scan over lanes), re-reads that one segment (one vector per
//     lane) to pick the vector, and the element from the lane's registers.
//     For a draft rejection the pass of step 4 already holds chunk k*'s
//     segment sums; a bonus or one-hot draw runs the pass over chunk k*
//     alone.  Rows that do not start on a 16-byte boundary (or very long
//     chunks) use contiguous per-thread segments, a block scan and one walk.
//
// R is the fewest chunks per CTA that fit the batch in about two waves of the
// resident CTAs.  The kernel is a programmatic dependent of the
// row-statistics kernel (which signals at the end of each CTA): its
// input-only prologue overlaps that kernel's last CTAs, and it waits for the
// kernel's completion (griddepcontrol.wait) before reading the partials.
#pragma once

#include <cooperative_groups.h>

#include "spec_verify.h"
#include "sv_common.cuh"

// Draw-kernel geometry (compile time; defaults tuned on B200).
#ifndef SV_DRAW_CTAS_PER_SM
#define SV_DRAW_CTAS_PER_SM 3
#endif
#ifndef SV_DRAW_PIECE_VECS
#define SV_DRAW_PIECE_VECS 512
#endif
#ifndef SV_DRAW_STAGES
#define SV_DRAW_STAGES 3
#endif

namespace sv {

namespace cg = cooperative_groups;

struct DrawParams {
    const unsigned char* target;
    const unsigned char* draft;  // null -> one-hot q
    const int32_t* tokens;
    const int32_t* lens;         // null -> k_max
    const float* uniforms;       // null allowed when greedy
    const float2* partials;
    int32_t* out_len;
    int32_t* out_tokens;
    float* out_lse_t;            // stats mode outputs (natural log), may be null
    float* out_lse_d;
    float* out_p;
    float* out_q;
    float* out_accept_prob;      // acceptance simulation outputs (stats mode), may be null
    float* out_expected_len;
    int32_t* out_first_reject;
    float* out_weights;
    float decay;
    int32_t b0;
    int32_t k_max;
    int32_t V;
    int64_t row_stride;
    int32_t C;                   // row-statistics chunks per row (partials per row)
    int32_t CE;                  // elements per chunk
    int32_t R;                   // chunks per draw CTA; a request's cluster has ceil(C / R) CTAs
    float scale;                 // log2(e) / T
    int32_t greedy;
    int32_t stats_only;
    int32_t rows_aligned;        // every row starts on a 16-byte boundary
    int32_t fast_draw;           // ring-based draw pass (aligned rows, chunks of at most
                                 // kMaxChunkBytesFast); the launch provides the ring
};

constexpr int kDrawThreads = 256;
constexpr int kDrawWarps = kDrawThreads / 32;
constexpr int kDrawCtasPerSm = SV_DRAW_CTAS_PER_SM;  // resident draw CTAs per SM the kernel is built for
constexpr int kBatchVecs = 4;        // 16-byte vectors (per row) per thread in flight in the segment passes
constexpr int kMaxDraftsPerThread = (SV_MAX_K + kDrawThreads - 1) / kDrawThreads;

// Ring of the fast draw pass: kDrawStages stages, each holding kPieceVecs
// 16-byte vectors of the target row and as many of the draft row.
constexpr int kPieceVecs = SV_DRAW_PIECE_VECS;
constexpr int kDrawStages = SV_DRAW_STAGES;
constexpr int kPieceVecsPerThread = kPieceVecs / kDrawThreads;
constexpr int kStageRowBytes = kPieceVecs * 16;
static_assert(kPieceVecs % kDrawThreads == 0 && 1024 % kPieceVecs == 0, "a piece must divide a 16 KiB stage");
constexpr size_t kDrawRingBytes = size_t(kDrawStages) * 2 * kStageRowBytes;
constexpr int kSegVecs = 32;  // vectors per segment: one warp-wide 16-byte load
// The fast path takes chunks of at most kMaxChunkBytesFast, i.e.
// kMaxSegsPerChunk segments.
constexpr int kMaxChunkBytesFast = 8 * 16384;
constexpr int kMaxSegsPerChunk = kMaxChunkBytesFast / 16 / kSegVecs;

// Dynamic shared memory: lse_t[k+1] | lse_d[k] | p[k] | q[k] | ring (fast draw only)
__host__ __device__ inline size_t draw_scalar_bytes(int k_max) {
    return (4 * (size_t(k_max + 1) + 3 * size_t(k_max)) + 127) & ~size_t(127);
}
__host__ __device__ inline size_t draw_smem_bytes(int k_max, bool ring) {
    return draw_scalar_bytes(k_max) + (ring ? kDrawRingBytes : 0);
}

// Block-wide inclusive scan of one float per thread; returns the thread's
// inclusive value and, through *excl, the previous thread's inclusive value
// (0 for thread 0) so that segment bounds meet exactly.  s_incl[kDrawThreads-1]
// holds the total afterwards.
__device__ __forceinline__ float block_scan_incl(float v, float* s_warp, float* s_incl, float* excl) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        float w = lane < kDrawWarps ? s_warp[lane] : 0.f;
        float wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        if (lane < kDrawWarps) s_warp[lane] = wi - w;
    }
    __syncthreads();
    incl += s_warp[warp];
    s_incl[threadIdx.x] = incl;
    __syncthreads();
    *excl = threadIdx.x ? s_incl[threadIdx.x - 1] : 0.f;
    return incl;
}

enum DrawMode { kBonus = 0, kOneHot = 1, kResidual = 2 };

// Acceptance probability min(1, p/q); NaN stays NaN (and then rejects).
__device__ __forceinline__ float accept_prob(float p, float q) {
    const float a = p / q;
    return a > 1.f ? 1.f : a;
}

// Everything a segment pass needs to turn logits of row j into draw weights.
struct WeightRow {
    const unsigned char* trow;   // target row j
    const unsigned char* drow;   // draft row j (residual only)
    float scale, lse_p, lse_q;   // log2 domain
    int zero_at;                 // row index whose weight is 0 (one-hot), or -1
};

// Draw weight of one element: residual max(0, p - q) or p.
template <bool kResid>
__device__ __forceinline__ float draw_weight(const WeightRow& r, float z, float y) {
    float w = ex2_approx(fmaf(z, r.scale, -r.lse_p));
    if constexpr (kResid) w = fmaxf(0.f, w - ex2_approx(fmaf(y, r.scale, -r.lse_q)));
    return w;
}

// The contiguous segment [lo, hi) (row element indices) of the chunk owned by
// this thread; segment starts are vector-aligned.
template <typename T>
__device__ __forceinline__ void thread_segment(int e0, int n, int* lo, int* hi) {
    constexpr int PV = Logit<T>::kPerVec;
    const int seg = (((n + kDrawThreads - 1) / kDrawThreads) + PV - 1) / PV * PV;
    *lo = e0 + min(n, int(threadIdx.x) * seg);
    *hi = e0 + min(n, int(threadIdx.x) * seg + seg);
}

// Visit the weights of row elements [lo, hi) in order, batch by batch with
// all loads of a batch in flight; `f(index, weight)` returns true to stop.
template <typename T, bool kResid, typename F>
__device__ __forceinline__ void visit_weights(const WeightRow& r, int lo, int hi, bool vec_ok, F&& f) {
    constexpr int PV = Logit<T>::kPerVec;
    constexpr int ES = Logit<T>::kSize;
    int e = lo;
    if (vec_ok) {
        const int vend = lo + (hi - lo) / PV * PV;  // lo is vector-aligned
        for (; e < vend; e += kBatchVecs * PV) {
            uint4 a[kBatchVecs], d[kBatchVecs];
#pragma unroll
            for (int k = 0; k < kBatchVecs; ++k) {
                if (e + k * PV < vend) {
                    a[k] = ld_global_stream_v4(r.trow + int64_t(e + k * PV) * ES);
                    if constexpr (kResid) d[k] = ld_global_stream_v4(r.drow + int64_t(e + k * PV) * ES);
                }
            }
#pragma unroll
            for (int k = 0; k < kBatchVecs; ++k) {
                if (e + k * PV < vend) {
                    float zf[PV], yf[PV];
                    Logit<T>::unpack(a[k], zf);
                    if constexpr (kResid) Logit<T>::unpack(d[k], yf);
#pragma unroll
                    for (int i = 0; i < PV; ++i) {
                        const int idx = e + k * PV + i;
                        float w = draw_weight<kResid>(r, zf[i], kResid ? yf[i] : 0.f);
                        if (!kResid && idx == r.zero_at) w = 0.f;  // max(0, p - 1) = 0 at the drafted id
                        if (f(idx, w)) return;
                    }
                }
            }
        }
        e = vend;
    }
    for (; e < hi; e += kBatchVecs) {
        float z[kBatchVecs], y[kBatchVecs];
#pragma unroll
        for (int k = 0; k < kBatchVecs; ++k) {
            if (e + k < hi) {
                z[k] = Logit<T>::load(r.trow, e + k);
                if constexpr (kResid) y[k] = Logit<T>::load(r.drow, e + k);
            }
        }
#pragma unroll
        for (int k = 0; k < kBatchVecs; ++k) {
            if (e + k < hi) {
                float w = draw_weight<kResid>(r, z[k], kResid ? y[k] : 0.f);
                if (!kResid && e + k == r.zero_at) w = 0.f;
                if (f(e + k, w)) return;
            }
        }
    }
}

template <typename T>
__device__ __forceinline__ float segment_sum(const WeightRow& r, bool resid, int lo, int hi, bool vec_ok) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int i = 0;
    auto add = [&](int, float w) { acc[i++ & 3] += w; return false; };
    if (resid) visit_weights<T, true>(r, lo, hi, vec_ok, add);
    else visit_weights<T, false>(r, lo, hi, vec_ok, add);
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// First index in [lo, hi) with positive weight at which the running sum
// (starting at acc0) exceeds target; the last positive-weight index if
// rounding leaves none; -1 if the segment has no positive weight.
template <typename T>
__device__ __noinline__ int segment_walk(const WeightRow& r, bool resid, int lo, int hi, bool vec_ok, float acc0,
                            float target) {
    float acc = acc0;
    int found = -1, last = -1;
    auto step = [&](int idx, float w) {
        if (w > 0.f) {
            last = idx;
            acc += w;
            if (acc > target) { found = idx; return true; }
        }
        return false;
    };
    if (resid) visit_weights<T, true>(r, lo, hi, vec_ok, step);
    else visit_weights<T, false>(r, lo, hi, vec_ok, step);
    return found >= 0 ? found : last;
}

// Weights of the PV elements of one 16-byte vector (tz from the target row,
// ty from the draft row), the element at row index zero_at (one-hot draw)
// set to 0; returns their sum, added in element order.
template <typename T, bool kResid>
__device__ __forceinline__ float vector_weights(const WeightRow& r, const uint4& tz, const uint4& ty, int idx0,
                                                float (&w)[Logit<T>::kPerVec]) {
    constexpr int PV = Logit<T>::kPerVec;
    float z[PV], y[PV];
    Logit<T>::unpack(tz, z);
    if constexpr (kResid) Logit<T>::unpack(ty, y);
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < PV; ++i) {
        float wi = draw_weight<kResid>(r, z[i], kResid ? y[i] : 0.f);
        if (!kResid && idx0 + i == r.zero_at) wi = 0.f;
        w[i] = wi;
        sum += wi;
    }
    return sum;
}

// The same for the partial vector at the end of a row (count < PV
// elements), read element-wise; absent elements get weight 0.
template <typename T, bool kResid>
__device__ __forceinline__ float tail_weights(const WeightRow& r, int idx0, int count,
                                              float (&w)[Logit<T>::kPerVec]) {
    constexpr int PV = Logit<T>::kPerVec;
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < PV; ++i) {
        w[i] = 0.f;
        if (i < count) {
            const int idx = idx0 + i;
            float wi = draw_weight<kResid>(r, Logit<T>::load(r.trow, idx), kResid ? Logit<T>::load(r.drow, idx) : 0.f);
            if (!kResid && idx == r.zero_at) wi = 0.f;
            w[i] = wi;
            sum += wi;
        }
    }
    return sum;
}

// Fast draw pass over the nch consecutive chunks k0 .. k0+nch-1 of row j
// (and of the draft row j for the residual).  The chunks stream through a
// ring of kDrawStages shared-memory stages filled by 16-byte cp.async copies
// (every thread copies the vectors it will read, so no register holds data
// in flight and no barrier is needed); the weight sum of each segment of
// kSegVecs vectors goes to s_seg[(k - k0) * kMaxSegsPerChunk + segment].
// Chunks are whole multiples of 16 KiB, so every stage but the last of the
// row is full.
template <typename T, bool kResid>
__device__ __noinline__ void draw_pass(const WeightRow r, int k0, int nch, int CE, int V, unsigned char* ring,
                                       float* s_seg) {
    constexpr int PV = Logit<T>::kPerVec;
    constexpr int ES = Logit<T>::kSize;
    const int tid = threadIdx.x, lane = tid & 31;
    const int spst = CE / PV / kPieceVecs;  // stages per full chunk
    const int n_last = min(V - (k0 + nch - 1) * CE, CE);
    const int G = (nch - 1) * spst + ((n_last + PV - 1) / PV + kPieceVecs - 1) / kPieceVecs;
    auto issue = [&](int g) {
        if (g < G) {
            const int slot = g / spst, piece = g - slot * spst;
            const int e0 = (k0 + slot) * CE;
            const int nfull = min(V - e0, CE) / PV;
            unsigned char* buf = ring + size_t(g % kDrawStages) * 2 * kStageRowBytes;
#pragma unroll
            for (int i = 0; i < kPieceVecsPerThread; ++i) {
                const int lv = tid + i * kDrawThreads;  // vector within the piece
                const int v = piece * kPieceVecs + lv;  // vector within the chunk
                if (v < nfull) {
                    cp_async_16(buf + lv * 16, r.trow + int64_t(e0 + v * PV) * ES);
                    if constexpr (kResid) cp_async_16(buf + kStageRowBytes + lv * 16, r.drow + int64_t(e0 + v * PV) * ES);
                }
            }
        }
        cp_async_commit();  // possibly empty: keeps the group count per iteration fixed
    };
#pragma unroll
    for (int g = 0; g < kDrawStages - 1; ++g) issue(g);
#pragma unroll 1
    for (int g = 0; g < G; ++g) {
        // Each thread copies exactly the vectors it reads back (vector
        // tid + i * kDrawThreads of every piece), so its own wait_group makes
        // stage g visible to it, and program order keeps the refill below of
        // the stage it consumed in iteration g - 1 behind its reads: the
        // ring needs no block barrier.
        issue(g + kDrawStages - 1);
        cp_async_wait<kDrawStages - 1>();
        const int slot = g / spst, piece = g - slot * spst;
        const int e0 = (k0 + slot) * CE;
        const int n = min(V - e0, CE);
        const int nfull = n / PV, nvec = (n + PV - 1) / PV;
        const unsigned char* buf = ring + size_t(g % kDrawStages) * 2 * kStageRowBytes;
#pragma unroll
        for (int i = 0; i < kPieceVecsPerThread; ++i) {
            const int lv = tid + i * kDrawThreads;
            const int v = piece * kPieceVecs + lv;
            float w[Logit<T>::kPerVec];
            float sum = 0.f;
            if (v < nfull) {
                const uint4 tz = ld_shared_v4(buf + lv * 16);
                const uint4 ty = kResid ? ld_shared_v4(buf + kStageRowBytes + lv * 16) : tz;
                sum = vector_weights<T, kResid>(r, tz, ty, e0 + v * PV, w);
            } else if (v < nvec) {
                sum = tail_weights<T, kResid>(r, e0 + v * PV, n - v * PV, w);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            // lane 0 holds the first vector of its warp's segment
            if (lane == 0) s_seg[slot * kMaxSegsPerChunk + v / kSegVecs] = sum;
        }
    }
    __syncthreads();  // s_seg complete
}

// Inclusive warp scan of v over lanes.
__device__ __forceinline__ float warp_scan_incl(float v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Final step of the fast draw, run by one warp: inside chunk [e0, e0+n)
// whose segment sums are segs[0 .. nseg), find the element at which the
// running weight first exceeds `target` -- segment (a scan over lanes, each
// lane holding consecutive segments), then vector (one warp-wide re-read of
// the segment, one vector per lane, and a scan over lanes), then element.
// Rounding that leaves the target past every block takes the last block with
// positive weight instead.  Returns the row index (same in every lane), or -1
// when the chunk has no positive weight.
template <typename T>
__device__ __noinline__ int draw_select(const WeightRow r, bool resid, int e0, int n, const float* segs,
                                        float target) {
    constexpr int PV = Logit<T>::kPerVec;
    constexpr int ES = Logit<T>::kSize;
    const int lane = threadIdx.x & 31;
    const int nfull = n / PV, nvec = (n + PV - 1) / PV;
    const int nseg = (nvec + kSegVecs - 1) / kSegVecs;
    // segment
    const int cps = (nseg + 31) / 32;
    const int s0 = lane * cps;
    const int ns = min(cps, max(0, nseg - s0));
    float mine = 0.f;
    for (int i = 0; i < ns; ++i) mine += segs[s0 + i];
    const float li = warp_scan_incl(mine);
    unsigned cross = __ballot_sync(0xffffffffu, mine > 0.f && li > target);
    unsigned pos = __ballot_sync(0xffffffffu, mine > 0.f);
    int lsel = cross ? __ffs(cross) - 1 : (pos ? 31 - __clz(pos) : -1);
    if (lsel < 0) return -1;
    int seg = 0;
    float t_seg = INFINITY;
    if (lane == lsel) {
        const float t1 = cross ? target : INFINITY;
        float run = li - mine, before = 0.f, last_before = 0.f;
        int isel = -1, ilast = -1;
        for (int i = 0; i < ns; ++i) {
            const float w = segs[s0 + i];
            if (w > 0.f) {
                ilast = i;
                last_before = run;
                if (run + w > t1) { isel = i; before = run; break; }
            }
            run += w;
        }
        const bool hit = isel >= 0;
        if (!hit) { isel = ilast; before = last_before; }
        seg = s0 + isel;
        t_seg = hit ? t1 - before : INFINITY;
    }
    seg = __shfl_sync(0xffffffffu, seg, lsel);
    t_seg = __shfl_sync(0xffffffffu, t_seg, lsel);
    // vector: lane l re-reads vector seg * kSegVecs + l of the chunk
    const int v = seg * kSegVecs + lane;
    float w[PV];
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < PV; ++i) w[i] = 0.f;
    if (v < nfull) {
        const uint4 tz = ld_global_stream_v4(r.trow + int64_t(e0 + v * PV) * ES);
        if (resid) {
            const uint4 ty = ld_global_stream_v4(r.drow + int64_t(e0 + v * PV) * ES);
            sum = vector_weights<T, true>(r, tz, ty, e0 + v * PV, w);
        } else {
            sum = vector_weights<T, false>(r, tz, tz, e0 + v * PV, w);
        }
    } else if (v < nvec) {
        sum = resid ? tail_weights<T, true>(r, e0 + v * PV, n - v * PV, w)
                    : tail_weights<T, false>(r, e0 + v * PV, n - v * PV, w);
    }
    const float lv = warp_scan_incl(sum);
    cross = __ballot_sync(0xffffffffu, sum > 0.f && lv > t_seg);
    pos = __ballot_sync(0xffffffffu, sum > 0.f);
    lsel = cross ? __ffs(cross) - 1 : (pos ? 31 - __clz(pos) : -1);
    if (lsel < 0) return -1;
    // element, in the selected lane's registers
    int found = -1, last = -1;
    if (lane == lsel) {
        const float t2 = cross ? t_seg : INFINITY;
        float run = lv - sum;
#pragma unroll
        for (int i = 0; i < PV; ++i) {
            if (w[i] > 0.f && found < 0) {
                last = i;
                run += w[i];
                if (run > t2) found = i;
            }
        }
        found = e0 + v * PV + (found >= 0 ? found : last);
    }
    return __shfl_sync(0xffffffffu, found, lsel);
}

template <typename T>
__global__ void __launch_bounds__(kDrawThreads, kDrawCtasPerSm)
verify_draw_kernel(const DrawParams p) {
    extern __shared__ __align__(128) unsigned char draw_dsm[];
    __shared__ float s_Wc[kMaxChunks];
    __shared__ float s_warp[kDrawWarps];
    __shared__ float s_incl[kDrawThreads];
    __shared__ float s_seg[kMaxChunks * kMaxSegsPerChunk];  // segment sums of the fast draw pass
    __shared__ int s_first, s_fail, s_cstar, s_mode, s_found, s_segsel, s_lastseg;
    __shared__ float s_local_target;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = blockIdx.x;
    const int b = p.b0 + blockIdx.y;
    const int K = p.k_max;
    const int nslots = 2 * K + 1;  // partial rows per request
    const int C = p.C;
    const int64_t esz = Logit<T>::kSize;
    float* s_lse_t = reinterpret_cast<float*>(draw_dsm);
    float* s_lse_d = s_lse_t + (K + 1);
    float* s_p = s_lse_d + K;   // gathered z(x_i), then p_i
    float* s_q = s_p + K;       // gathered y(x_i), then q_i
    int* s_arg_t = reinterpret_cast<int*>(s_lse_t);  // greedy: argmax per target row
    unsigned char* ring = draw_dsm + draw_scalar_bytes(K);
    const int32_t* x = p.tokens + int64_t(b) * K;
    int32_t* out_tok = p.out_tokens ? p.out_tokens + int64_t(b) * (K + 1) : nullptr;
    const bool has_draft = p.draft != nullptr && !p.greedy;
    const float* u = p.uniforms ? p.uniforms + int64_t(b) * (K + 1) : nullptr;
    auto trow_of = [&](int i) { return p.target + (int64_t(b) * (K + 1) + i) * p.row_stride * esz; };
    auto drow_of = [&](int i) { return p.draft + (int64_t(b) * K + i) * p.row_stride * esz; };

    auto write_failed = [&](int code) {
        if (c != 0) return;
        const float nan = __int_as_float(0x7fc00000);
        if (p.stats_only) {
            for (int i = tid; i <= K; i += kDrawThreads)
                if (p.out_lse_t) p.out_lse_t[int64_t(b) * (K + 1) + i] = nan;
            for (int i = tid; i < K; i += kDrawThreads) {
                if (p.out_lse_d) p.out_lse_d[int64_t(b) * K + i] = nan;
                if (p.out_p) p.out_p[int64_t(b) * K + i] = nan;
                if (p.out_q) p.out_q[int64_t(b) * K + i] = nan;
                if (p.out_accept_prob) p.out_accept_prob[int64_t(b) * K + i] = nan;
                if (p.out_weights) p.out_weights[int64_t(b) * K + i] = nan;
            }
            if (tid == 0) {
                if (p.out_expected_len) p.out_expected_len[b] = nan;
                if (p.out_first_reject) p.out_first_reject[b] = code;
            }
        } else {
            for (int i = tid; i <= K; i += kDrawThreads) out_tok[i] = -1;
            if (tid == 0) p.out_len[b] = code;
        }
    };

    // 1. inputs only: validation, gathered logits at the drafted ids, uniforms
    const int L = p.lens ? __ldg(p.lens + b) : K;
    bool ok = L >= 0 && L <= K;
    int xr[kMaxDraftsPerThread];
#pragma unroll
    for (int k = 0; k < kMaxDraftsPerThread; ++k) {
        const int i = tid + k * kDrawThreads;
        xr[k] = 0;
        if (ok && i < L) {
            xr[k] = __ldg(x + i);
            if (xr[k] < 0 || xr[k] >= p.V) ok = false;
        }
    }
    ok = __syncthreads_and(ok);
    float ur[kMaxDraftsPerThread];
    if (ok && !p.greedy) {
#pragma unroll
        for (int k = 0; k < kMaxDraftsPerThread; ++k) {
            const int i = tid + k * kDrawThreads;
            ur[k] = 0.f;
            if (i < L) {
                s_p[i] = Logit<T>::load(trow_of(i), xr[k]);
                if (has_draft) s_q[i] = Logit<T>::load(drow_of(i), xr[k]);
                if (u) ur[k] = __ldg(u + i);
            }
        }
    }

    // 2. the row-statistics kernel's partials (this kernel is a programmatic
    // dependent of it: wait for its completion before reading them), merged
    // straight from global memory: G lanes per row, 32/G rows per warp at once
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (!ok) {
        write_failed(-1);
        return;
    }
    if (tid == 0) { s_fail = 0; s_first = L; }
    const int n_t = L + 1;
    const int n_d = has_draft ? L : 0;
    const int nrows = n_t + n_d;
    {
        const int G = C <= 1 ? 1 : (C <= 2 ? 2 : (C <= 4 ? 4 : 8));
        const int sub = lane / G, gl = lane - sub * G;
        const float2* part_b = p.partials + int64_t(b) * nslots * C;
        for (int r0 = warp * (32 / G); r0 < nrows; r0 += kDrawWarps * (32 / G)) {
            const int row = r0 + sub;
            const bool act = row < nrows && gl < C;
            const int slot = row < n_t ? row : K + 1 + (row - n_t);
            const float2 v = act ? part_b[int64_t(slot) * C + gl] : make_float2(-INFINITY, 0.f);
            bool bad;
            if (p.greedy) {
                const int idx = act ? __float_as_int(v.y) : 0x7fffffff;
                bad = act && (idx < 0 || idx >= p.V);
                VI r{v.x, idx};
                for (int o = G >> 1; o > 0; o >>= 1)
                    r = vi_better(r, VI{__shfl_xor_sync(0xffffffffu, r.v, o), __shfl_xor_sync(0xffffffffu, r.i, o)});
                if (row < nrows && gl == 0) s_arg_t[row] = r.i;
            } else {
                bad = act && (isnan(v.x) || isnan(v.y));
                float m = v.x;
                for (int o = G >> 1; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                float sum = m == -INFINITY ? 0.f : v.y * ex2_approx(v.x - m);
                for (int o = G >> 1; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                if (row < nrows && gl == 0) {
                    const float lse2 = m + log2f(sum);
                    if (row < n_t) s_lse_t[row] = lse2; else s_lse_d[row - n_t] = lse2;
                }
            }
            if (__any_sync(0xffffffffu, bad) && lane == 0) s_fail = 1;
        }
    }
    __syncthreads();
    if (s_fail) {
        write_failed(-2);
        return;
    }

    // 3. p, q at the drafted ids; acceptance scan ----------------------------------
#pragma unroll
    for (int k = 0; k < kMaxDraftsPerThread; ++k) {
        const int i = tid + k * kDrawThreads;
        if (i >= L) continue;
        bool rej;
        if (p.greedy) {
            rej = xr[k] != s_arg_t[i];
        } else {
            const float pi = exp2f(s_p[i] * p.scale - s_lse_t[i]);
            const float qi = has_draft ? exp2f(s_q[i] * p.scale - s_lse_d[i]) : 1.f;
            s_p[i] = pi;
            s_q[i] = qi;
            const float a = accept_prob(pi, qi);
            rej = u ? !(ur[k] < a) : false;  // no uniforms (statistics only): no scan
        }
        if (rej) atomicMin(&s_first, i);
    }
    __syncthreads();

    if (p.stats_only) {
        if (c == 0) {
            const float nan = __int_as_float(0x7fc00000);
            const int j = s_first;  // L when no uniforms were given
            for (int i = tid; i <= K; i += kDrawThreads)
                if (p.out_lse_t) p.out_lse_t[int64_t(b) * (K + 1) + i] = i <= L ? s_lse_t[i] * kLn2 : nan;
            for (int i = tid; i < K; i += kDrawThreads) {
                if (p.out_lse_d) p.out_lse_d[int64_t(b) * K + i] = (has_draft && i < L) ? s_lse_d[i] * kLn2 : nan;
                if (p.out_p) p.out_p[int64_t(b) * K + i] = i < L ? s_p[i] : nan;
                if (p.out_q) p.out_q[int64_t(b) * K + i] = i < L ? s_q[i] : nan;
                if (p.out_accept_prob) p.out_accept_prob[int64_t(b) * K + i] = i < L ? accept_prob(s_p[i], s_q[i]) : nan;
                if (p.out_weights)  // full weight up to the first rejection, the decay curve from there
                    p.out_weights[int64_t(b) * K + i] = i >= L ? 0.f : (i <= j ? 1.f : powf(p.decay, float(i - j)));
            }
            if (tid == 0) {
                if (p.out_first_reject) p.out_first_reject[b] = j;
                if (p.out_expected_len) {
                    // E[j] = sum_{m=1..L} P(j >= m), P(j >= m) = prod_{l<m} a_l
                    float prod = 1.f, e = 0.f;
                    for (int i = 0; i < L; ++i) {
                        prod *= accept_prob(s_p[i], s_q[i]);
                        e += prod;
                    }
                    p.out_expected_len[b] = e;
                }
            }
        }
        return;
    }

    const int j = s_first;
    if (c == 0) {
        for (int i = tid; i <= K; i += kDrawThreads) {
            if (i < j) out_tok[i] = __ldg(x + i);
            else if (i > j) out_tok[i] = -1;
            else if (p.greedy) out_tok[i] = s_arg_t[j];
        }
        if (tid == 0) p.out_len[b] = j;
    }
    if (p.greedy) return;

    // 4. final draw on row j: chunk weights and the chunk that holds u*W ---------------
    WeightRow wr;
    wr.trow = trow_of(j);
    wr.drow = (has_draft && j < L) ? drow_of(j) : nullptr;
    wr.scale = p.scale;
    wr.lse_p = s_lse_t[j];
    wr.lse_q = (has_draft && j < L) ? s_lse_d[j] : 0.f;
    wr.zero_at = -1;
    const float ustar = __ldg(u + K);
    const bool vec_ok = p.rows_aligned != 0;
    const bool fast = p.fast_draw != 0;
    const int mode = j == L ? kBonus : (has_draft ? kResidual : kOneHot);
    const int k_lo = c * p.R, k_hi = min(C, k_lo + p.R);  // this CTA's chunks
    const float2* part_j = p.partials + (int64_t(b) * nslots + j) * C;  // row j's chunk partials
    float ssum = 0.f, excl = 0.f, incl = 0.f;
    auto chunk_bounds = [&](int k, int* e0, int* n) {
        *e0 = k * p.CE;
        *n = min(p.V - *e0, p.CE);
    };
    // Slow path: sum of the draw weights over chunk k from contiguous
    // per-thread segments (block-wide; all threads get it).
    auto chunk_total_slow = [&](int k, bool resid) {
        int e0, n;
        chunk_bounds(k, &e0, &n);
        int lo, hi;
        thread_segment<T>(e0, n, &lo, &hi);
        ssum = segment_sum<T>(wr, resid, lo, hi, vec_ok);
        incl = block_scan_incl(ssum, s_warp, s_incl, &excl);
        return s_incl[kDrawThreads - 1];
    };

    bool have_segs = false;  // s_seg holds this CTA's chunks for the residual weights
    if (mode == kResidual) {
        // every CTA sums its chunks; the sums are exchanged across the cluster
        cg::cluster_group cluster = cg::this_cluster();
        const int C2 = (C + p.R - 1) / p.R;
        if (fast) {
            draw_pass<T, true>(wr, k_lo, k_hi - k_lo, p.CE, p.V, ring, s_seg);
            have_segs = true;
            if (warp < k_hi - k_lo) {  // warp w totals chunk k_lo + w (R <= 8 warps)
                int e0, n;
                chunk_bounds(k_lo + warp, &e0, &n);
                const int nseg = ((n + Logit<T>::kPerVec - 1) / Logit<T>::kPerVec + kSegVecs - 1) / kSegVecs;
                float t = 0.f;
                for (int s = lane; s < nseg; s += 32) t += s_seg[warp * kMaxSegsPerChunk + s];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
                if (lane < C2) cluster.map_shared_rank(&s_Wc[0], lane)[k_lo + warp] = t;
            }
        } else {
            for (int k = k_lo; k < k_hi; ++k) {
                const float Wk = chunk_total_slow(k, true);
                if (tid < C2) cluster.map_shared_rank(&s_Wc[0], tid)[k] = Wk;
            }
        }
        cluster.sync();
    }

    if (warp == 0) {
        // lane cc holds chunk cc's weight
        float W = 0.f;
        int m2 = mode;
        if (lane < C) {
            if (mode == kResidual) {
                W = s_Wc[lane];
            } else {
                const float2 pp = part_j[lane];
                W = pp.y * exp2f(pp.x - wr.lse_p);
                if (mode == kOneHot && lane == __ldg(x + j) / p.CE) W = fmaxf(0.f, W - s_p[j]);
            }
        }
        float total = W;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
        if (!(total > 0.f)) {
            // zero residual mass (p == q numerically): draw from p_j
            m2 = kBonus;
            W = 0.f;
            if (lane < C) {
                const float2 pp = part_j[lane];
                W = pp.y * exp2f(pp.x - wr.lse_p);
            }
            total = W;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
        }
        const float target = ustar * total;
        const float wi = warp_scan_incl(W);
        const unsigned cross = __ballot_sync(0xffffffffu, W > 0.f && wi > target);
        const unsigned pos = __ballot_sync(0xffffffffu, W > 0.f);
        const int cstar = cross ? __ffs(cross) - 1 : (pos ? 31 - __clz(pos) : 0);
        const float before = __shfl_sync(0xffffffffu, wi - W, cstar);
        if (lane == 0) {
            s_cstar = cstar;
            s_mode = m2;
            s_local_target = cross ? fmaxf(0.f, target - before) : INFINITY;
            s_found = -1;
            s_segsel = 0x7fffffff;
            s_lastseg = -1;
        }
    }
    __syncthreads();
    const int kstar = s_cstar;
    if (kstar < k_lo || kstar >= k_hi) return;

    // 5. inverse CDF inside chunk k* ---------------------------------------------------
    const bool resid = s_mode == kResidual;
    const float target = s_local_target;
    wr.zero_at = s_mode == kOneHot ? __ldg(x + j) : -1;
    int e0, n;
    chunk_bounds(kstar, &e0, &n);
    if (fast) {
        const float* segs = s_seg + (kstar - k_lo) * kMaxSegsPerChunk;
        if (!(resid && have_segs)) {
            // bonus or one-hot draw: one pass over chunk k* alone
            draw_pass<T, false>(wr, kstar, 1, p.CE, p.V, ring, s_seg);
            segs = s_seg;
        }
        if (warp == 0) {
            const int t = draw_select<T>(wr, resid, e0, n, segs, target);
            if (lane == 0) out_tok[j] = t >= 0 ? t : e0;
        }
        return;
    }

    // slow path: contiguous per-thread segments, one block scan, one walk
    (void)chunk_total_slow(kstar, resid);
    int lo, hi;
    thread_segment<T>(e0, n, &lo, &hi);
    if (ssum > 0.f) {
        if (incl > target) atomicMin(&s_segsel, tid);
        atomicMax(&s_lastseg, tid);
    }
    __syncthreads();
    if (tid == s_segsel) s_found = segment_walk<T>(wr, resid, lo, hi, vec_ok, excl, target);
    else if (s_segsel == 0x7fffffff && tid == s_lastseg)  // rounding left u*W past the last step
        s_found = segment_walk<T>(wr, resid, lo, hi, vec_ok, 0.f, INFINITY);
    __syncthreads();
    if (tid == 0) out_tok[j] = s_found >= 0 ? s_found : e0;
}

}  // namespace sv
