// sv_verify_draw.cuh -- K2, acceptance scan and the final draw.
//
// One thread-block cluster of C CTAs per request; CTA c of the cluster owns
// vocabulary chunk c of the row that the final draw uses.
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
//       draft rejection:    w = max(0, p_j - q_j); every CTA computes its
//                           chunk's sum, the sums are exchanged through
//                           distributed shared memory and a cluster barrier;
//     every CTA locates the chunk holding u*W.  In that CTA the chunk is read
//     once with coalesced 16-byte loads (warp w owns a contiguous run of
//     vectors, lane l the vectors w*WV + 32*it + l); each lane keeps the
//     weight sum of each of its vectors in registers, so the crossing is
//     found by narrowing down warp -> iteration -> lane (block scan of warp
//     totals, a running sum over iterations, a warp scan over lanes), and only
//     the one vector holding C_t > u*W is read again to pick the element.  In
//     the residual case the same pass also yields the chunk sum that is
//     exchanged, so the chosen CTA does not read its chunk twice.  Rows that
//     do not start on a 16-byte boundary (or very long chunks) use a slower
//     pass over contiguous per-thread segments instead.
//
// Shared memory stays small (the row partials and per-draft scalars), so
// many clusters are resident at once.  A request's cluster has ceil(C / R)
// CTAs, each owning R consecutive chunks, with R chosen so that the whole
// batch fits in about one wave.  The kernel is a programmatic dependent of the
// row-statistics kernel (which signals at the end of each CTA): its
// input-only prologue overlaps that kernel's last CTAs, and it waits for the
// kernel's completion (griddepcontrol.wait) before reading the partials.
#pragma once

#include <cooperative_groups.h>

#include "spec_verify.h"
#include "sv_common.cuh"

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
};

constexpr int kDrawThreads = 256;
constexpr int kDrawWarps = kDrawThreads / 32;
constexpr int kBatchVecs = 4;        // 16-byte vectors (per row) per thread in flight in the segment passes
constexpr int kMaxDraftsPerThread = (SV_MAX_K + kDrawThreads - 1) / kDrawThreads;

// Dynamic shared memory: partials[(2k+1) * C] float2 | lse_t[k+1] | lse_d[k] | p[k] | q[k]
__host__ __device__ inline size_t draw_smem_bytes(int C, int k_max) {
    return 8 * size_t(2 * k_max + 1) * size_t(C) + 4 * (size_t(k_max + 1) + 3 * size_t(k_max)) + 16;
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

constexpr int kWarpIters = 16;  // 32-vector iterations per warp run in the coalesced draw pass

// Coalesced pass over the chunk [e0, e0+n) of row j: warp w owns vectors
// [w*WV, (w+1)*WV) of the chunk (the last, partial vector at the row end is
// read element-wise); vs[it] = weight sum of vector w*WV + 32*it + lane.
// Returns this warp's total (same value in every lane).
template <typename T, bool kResid>
__device__ __forceinline__ float chunk_vector_sums(const WeightRow& r, int e0, int n, int WV,
                                                   float (&vs)[kWarpIters]) {
    constexpr int PV = Logit<T>::kPerVec;
    constexpr int ES = Logit<T>::kSize;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nfull = n / PV;                 // complete vectors
    const int nvec = (n + PV - 1) / PV;       // including a partial last one
    constexpr int kBatch = kResid ? 4 : 8;  // iterations whose loads are in flight together
    float tot = 0.f;
#pragma unroll
    for (int half = 0; half < kWarpIters; half += kBatch) {
        if (half * 32 >= WV) {  // uniform: nothing left for any lane
#pragma unroll
            for (int k = 0; k < kBatch; ++k) vs[half + k] = 0.f;
            continue;
        }
        uint4 a[kBatch], d[kBatch];
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const int it = half + k;
            const int v = warp * WV + it * 32 + lane;
            if (it * 32 + lane < WV && v < nfull) {
                a[k] = ld_global_stream_v4(r.trow + int64_t(e0 + v * PV) * ES);
                if constexpr (kResid) d[k] = ld_global_stream_v4(r.drow + int64_t(e0 + v * PV) * ES);
            }
        }
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const int it = half + k;
            const int v = warp * WV + it * 32 + lane;
            float sum = 0.f;
            if (it * 32 + lane < WV && v < nfull) {
                float zf[PV], yf[PV];
                Logit<T>::unpack(a[k], zf);
                if constexpr (kResid) Logit<T>::unpack(d[k], yf);
#pragma unroll
                for (int i = 0; i < PV; ++i) {
                    float w = draw_weight<kResid>(r, zf[i], kResid ? yf[i] : 0.f);
                    if (!kResid && e0 + v * PV + i == r.zero_at) w = 0.f;
                    sum += w;
                }
            } else if (it * 32 + lane < WV && v < nvec) {  // partial vector at the row end
                for (int i = 0; v * PV + i < n; ++i) {
                    const int idx = e0 + v * PV + i;
                    float w = draw_weight<kResid>(r, Logit<T>::load(r.trow, idx),
                                                  kResid ? Logit<T>::load(r.drow, idx) : 0.f);
                    if (!kResid && idx == r.zero_at) w = 0.f;
                    sum += w;
                }
            }
            vs[it] = sum;
            tot += sum;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    return tot;
}

// Within one vector (row elements first .. first+count-1, count <= PV): the
// first element with positive weight at which acc0 + running weight exceeds
// target, else the last positive-weight element, else -1.  A full aligned
// vector is read with one 16-byte load per row.
template <typename T>
__device__ __noinline__ int vector_walk(const WeightRow& r, bool resid, int first, int count, bool vec_ok,
                                        float acc0, float target) {
    constexpr int PV = Logit<T>::kPerVec;
    float z[PV], y[PV];
    if (vec_ok && count == PV) {
        Logit<T>::unpack(ld_global_stream_v4(r.trow + int64_t(first) * Logit<T>::kSize), z);
        if (resid) Logit<T>::unpack(ld_global_stream_v4(r.drow + int64_t(first) * Logit<T>::kSize), y);
    } else {
#pragma unroll
        for (int i = 0; i < PV; ++i) {
            z[i] = i < count ? Logit<T>::load(r.trow, first + i) : -INFINITY;
            y[i] = (resid && i < count) ? Logit<T>::load(r.drow, first + i) : 0.f;
        }
    }
    float acc = acc0;
    int found = -1, last = -1;
#pragma unroll
    for (int i = 0; i < PV; ++i) {
        if (i >= count || found >= 0) continue;
        const int idx = first + i;
        const float w = resid ? draw_weight<true>(r, z[i], y[i])
                              : (idx == r.zero_at ? 0.f : draw_weight<false>(r, z[i], 0.f));
        if (w > 0.f) {
            last = idx;
            acc += w;
            if (acc > target) found = idx;
        }
    }
    return found >= 0 ? found : last;
}

template <typename T>
__global__ void __launch_bounds__(kDrawThreads, 2)
verify_draw_kernel(const DrawParams p) {
    extern __shared__ __align__(16) unsigned char draw_dsm[];
    __shared__ float s_Wc[kMaxChunks];
    __shared__ float s_warp[kDrawWarps];
    __shared__ float s_incl[kDrawThreads];
    __shared__ int s_first, s_fail, s_cstar, s_mode, s_found, s_seg, s_lastseg;
    __shared__ float s_local_target;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = blockIdx.x;
    const int b = p.b0 + blockIdx.y;
    const int K = p.k_max;
    const int R = 2 * K + 1;
    const int C = p.C;
    const int64_t esz = Logit<T>::kSize;
    float2* s_part = reinterpret_cast<float2*>(draw_dsm);   // used rows, compact: row r at r*C
    float* s_lse_t = reinterpret_cast<float*>(s_part + size_t(R) * C);
    float* s_lse_d = s_lse_t + (K + 1);
    float* s_p = s_lse_d + K;   // gathered z(x_i), then p_i
    float* s_q = s_p + K;       // gathered y(x_i), then q_i
    int* s_arg_t = reinterpret_cast<int*>(s_lse_t);  // greedy: argmax per target row
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
            for (int i = tid; i <= K; i += kDrawThreads) p.out_lse_t[int64_t(b) * (K + 1) + i] = nan;
            for (int i = tid; i < K; i += kDrawThreads) {
                if (p.out_lse_d) p.out_lse_d[int64_t(b) * K + i] = nan;
                if (p.out_p) p.out_p[int64_t(b) * K + i] = nan;
                if (p.out_q) p.out_q[int64_t(b) * K + i] = nan;
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
                if (!p.stats_only) ur[k] = __ldg(u + i);
            }
        }
    }

    // 2. the row-statistics kernel's partials (this kernel is a programmatic
    // dependent of it: wait for its completion before reading them) --------------
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (!ok) {
        write_failed(-1);
        return;
    }
    if (tid == 0) { s_fail = 0; s_first = L; }
    const int n_t = L + 1;
    const int n_d = has_draft ? L : 0;
    const int nrows = n_t + n_d;
    for (int idx = tid; idx < nrows * C; idx += kDrawThreads) {
        const int row = idx / C, cc = idx - row * C;
        const int slot = row < n_t ? row : K + 1 + (row - n_t);
        s_part[idx] = p.partials[(int64_t(b) * R + slot) * C + cc];
    }
    __syncthreads();

    // 3. merge the partials: G lanes per row, 32/G rows per warp at once -----------
    {
        const int G = C <= 1 ? 1 : (C <= 2 ? 2 : (C <= 4 ? 4 : 8));
        const int sub = lane / G, gl = lane - sub * G;
        for (int r0 = warp * (32 / G); r0 < nrows; r0 += kDrawWarps * (32 / G)) {
            const int row = r0 + sub;
            const bool act = row < nrows && gl < C;
            const float2 v = act ? s_part[row * C + gl] : make_float2(-INFINITY, 0.f);
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

    // 4. p, q at the drafted ids; acceptance scan ----------------------------------
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
            float a = pi / qi;
            a = a > 1.f ? 1.f : a;  // min(1, p/q); NaN stays NaN (rejects)
            rej = p.stats_only ? false : !(ur[k] < a);
        }
        if (rej) atomicMin(&s_first, i);
    }
    __syncthreads();

    if (p.stats_only) {
        if (c == 0) {
            const float nan = __int_as_float(0x7fc00000);
            for (int i = tid; i <= K; i += kDrawThreads)
                p.out_lse_t[int64_t(b) * (K + 1) + i] = i <= L ? s_lse_t[i] * kLn2 : nan;
            for (int i = tid; i < K; i += kDrawThreads) {
                if (p.out_lse_d) p.out_lse_d[int64_t(b) * K + i] = (has_draft && i < L) ? s_lse_d[i] * kLn2 : nan;
                if (p.out_p) p.out_p[int64_t(b) * K + i] = i < L ? s_p[i] : nan;
                if (p.out_q) p.out_q[int64_t(b) * K + i] = i < L ? s_q[i] : nan;
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

    // 5. final draw on row j: chunk weights and the chunk that holds u*W ---------------
    WeightRow wr;
    wr.trow = trow_of(j);
    wr.drow = (has_draft && j < L) ? drow_of(j) : nullptr;
    wr.scale = p.scale;
    wr.lse_p = s_lse_t[j];
    wr.lse_q = (has_draft && j < L) ? s_lse_d[j] : 0.f;
    const float ustar = __ldg(u + K);
    const bool vec_ok = p.rows_aligned != 0;
    int mode = j == L ? kBonus : (has_draft ? kResidual : kOneHot);
    constexpr int PV = Logit<T>::kPerVec;
    const int WV_full = ((p.CE + PV - 1) / PV + kDrawWarps - 1) / kDrawWarps;  // vectors per warp run
    const bool fast = vec_ok && WV_full <= 32 * kWarpIters;
    const int k_lo = c * p.R, k_hi = min(C, k_lo + p.R);  // this CTA's chunks
    float vs[kWarpIters];
    float wtot = 0.f;          // this warp's total of the last chunk summed (fast path)
    float ssum = 0.f, excl = 0.f, incl = 0.f;
    auto chunk_bounds = [&](int k, int* e0, int* n) {
        *e0 = k * p.CE;
        *n = min(p.V - *e0, p.CE);
    };
    // Sum of the draw weights over chunk k (block-wide; all threads get it).
    auto chunk_total = [&](int k, bool resid) {
        int e0, n;
        chunk_bounds(k, &e0, &n);
        if (fast) {
            const int WV = ((n + PV - 1) / PV + kDrawWarps - 1) / kDrawWarps;
            wtot = resid ? chunk_vector_sums<T, true>(wr, e0, n, WV, vs) : chunk_vector_sums<T, false>(wr, e0, n, WV, vs);
            __syncthreads();  // previous readers of s_warp are done
            if (lane == 0) s_warp[warp] = wtot;
            __syncthreads();
            float t = 0.f;
#pragma unroll
            for (int w = 0; w < kDrawWarps; ++w) t += s_warp[w];
            return t;
        }
        int lo, hi;
        thread_segment<T>(e0, n, &lo, &hi);
        ssum = segment_sum<T>(wr, resid, lo, hi, vec_ok);
        incl = block_scan_incl(ssum, s_warp, s_incl, &excl);
        return s_incl[kDrawThreads - 1];
    };

    if (mode == kResidual) {
        // every CTA sums its chunks; the sums are exchanged across the cluster
        wr.zero_at = -1;
        cg::cluster_group cluster = cg::this_cluster();
        const int C2 = (C + p.R - 1) / p.R;
        for (int k = k_lo; k < k_hi; ++k) {
            const float Wk = chunk_total(k, true);
            if (tid < C2) {
                float* remote = cluster.map_shared_rank(&s_Wc[0], tid);
                remote[k] = Wk;
            }
        }
        cluster.sync();
    }

    if (tid == 0) {
        float W[kMaxChunks];
        float total = 0.f;
        for (int cc = 0; cc < C; ++cc) {
            if (mode == kResidual) {
                W[cc] = s_Wc[cc];
            } else {
                const float2 pp = s_part[j * C + cc];
                W[cc] = pp.y * exp2f(pp.x - wr.lse_p);
            }
        }
        if (mode == kOneHot) {
            const int cx = __ldg(x + j) / p.CE;
            W[cx] = fmaxf(0.f, W[cx] - s_p[j]);
        }
        for (int cc = 0; cc < C; ++cc) total += W[cc];
        if (!(total > 0.f)) {
            // zero residual mass (p == q numerically): draw from p_j
            mode = kBonus;
            total = 0.f;
            for (int cc = 0; cc < C; ++cc) {
                const float2 pp = s_part[j * C + cc];
                W[cc] = pp.y * exp2f(pp.x - wr.lse_p);
                total += W[cc];
            }
        }
        const float target = ustar * total;
        int cstar = -1, last_pos = 0;
        float before = 0.f, run = 0.f;
        for (int cc = 0; cc < C; ++cc) {
            if (W[cc] > 0.f) last_pos = cc;
            if (cstar < 0 && run + W[cc] > target) { cstar = cc; before = run; }
            run += W[cc];
        }
        if (cstar < 0) {
            cstar = last_pos;
            before = 0.f;
            for (int cc = 0; cc < cstar; ++cc) before += W[cc];
        }
        s_cstar = cstar;
        s_mode = mode;
        s_local_target = fmaxf(0.f, target - before);
        s_found = -1;
        s_seg = 0x7fffffff;
        s_lastseg = -1;
    }
    __syncthreads();
    const int kstar = s_cstar;
    if (kstar < k_lo || kstar >= k_hi) return;

    // 6. inverse CDF inside chunk k* ---------------------------------------------------
    const bool resid = s_mode == kResidual;
    // the residual pass already left chunk k*'s sums in registers when it was
    // this CTA's only (hence last) chunk
    const bool recompute = mode != s_mode || !resid || k_hi - k_lo != 1;
    const float target = s_local_target;
    wr.zero_at = s_mode == kOneHot ? __ldg(x + j) : -1;
    int e0, n;
    chunk_bounds(kstar, &e0, &n);
    if (recompute) (void)chunk_total(kstar, resid);
    if (fast) {
        const int WV = ((n + PV - 1) / PV + kDrawWarps - 1) / kDrawWarps;
        __syncthreads();
        if (tid == 0) {
            // warp whose run holds the target (first with positive total), or
            // the last positive warp when rounding leaves the target past it
            float run = 0.f;
            int ws = -1, wl = -1;
            float wb = 0.f;
            for (int w = 0; w < kDrawWarps; ++w) {
                const float t = s_warp[w];
                if (t > 0.f) {
                    wl = w;
                    if (ws < 0 && run + t > target) { ws = w; wb = run; }
                }
                run += t;
            }
            s_seg = ws >= 0 ? ws : wl;
            s_incl[0] = ws >= 0 ? target - wb : INFINITY;
        }
        __syncthreads();
        if (warp == s_seg) {
            const float t1 = s_incl[0];
            // iteration holding the target within this warp's run
            float run = 0.f;
            int its = -1, itl = -1;
            float itb = 0.f;
#pragma unroll
            for (int it = 0; it < kWarpIters; ++it) {
                float tsum = vs[it];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) tsum += __shfl_xor_sync(0xffffffffu, tsum, o);
                if (tsum > 0.f) {
                    itl = it;
                    if (its < 0 && run + tsum > t1) { its = it; itb = run; }
                }
                run += tsum;
            }
            const int it_sel = its >= 0 ? its : itl;
            const float t2 = its >= 0 ? t1 - itb : INFINITY;
            float mine = 0.f;
#pragma unroll
            for (int it = 0; it < kWarpIters; ++it)
                if (it == it_sel) mine = vs[it];
            // lane holding the target: inclusive scan over lanes
            float li = mine;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, li, o);
                if (lane >= o) li += v;
            }
            const unsigned cross = __ballot_sync(0xffffffffu, mine > 0.f && li > t2);
            const unsigned pos = __ballot_sync(0xffffffffu, mine > 0.f);
            const int lsel = cross ? __ffs(cross) - 1 : (pos ? 31 - __clz(pos) : -1);
            if (lsel >= 0 && lane == lsel) {
                const int v = warp * WV + it_sel * 32 + lane;
                const int first = e0 + v * PV;
                const int count = min(PV, e0 + n - first);
                s_found = vector_walk<T>(wr, resid, first, count, vec_ok, li - mine, cross ? t2 : INFINITY);
            }
        }
        __syncthreads();
        if (tid == 0) out_tok[j] = s_found >= 0 ? s_found : e0;
        return;
    }

    // slow path: contiguous per-thread segments, one block scan, one walk
    int lo, hi;
    thread_segment<T>(e0, n, &lo, &hi);
    if (ssum > 0.f) {
        if (incl > target) atomicMin(&s_seg, tid);
        atomicMax(&s_lastseg, tid);
    }
    __syncthreads();
    if (tid == s_seg) s_found = segment_walk<T>(wr, resid, lo, hi, vec_ok, excl, target);
    else if (s_seg == 0x7fffffff && tid == s_lastseg)  // rounding left u*W past the last step
        s_found = segment_walk<T>(wr, resid, lo, hi, vec_ok, 0.f, INFINITY);
    __syncthreads();
    if (tid == 0) out_tok[j] = s_found >= 0 ? s_found : e0;
}

}  // namespace sv
