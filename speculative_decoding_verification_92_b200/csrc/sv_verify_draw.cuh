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
//     every CTA locates the chunk holding u*W; that CTA stages its chunk's
//     weights in shared memory and finds the smallest t with C_t > u*W.
#pragma once

#include <cooperative_groups.h>

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
    int32_t C;
    int32_t CE;
    float scale;                 // log2(e) / T
    int32_t greedy;
    int32_t stats_only;
    int32_t rows_aligned;        // every row starts on a 16-byte boundary
};

constexpr int kDrawThreads = 256;

// Dynamic shared memory: w[CE] | lse_t[k+1] | lse_d[k] | p[k] | q[k]
__host__ __device__ inline size_t draw_smem_bytes(int CE, int k_max) {
    return 4 * (size_t(CE) + size_t(k_max + 1) + 3 * size_t(k_max)) + 16;
}

// Block-wide inclusive scan of one float per thread (256 threads); returns
// the thread's inclusive value and, through *excl, the previous thread's
// inclusive value (0 for thread 0) so that segment bounds meet exactly.
__device__ __forceinline__ float block_scan_incl(float v, float* s_warp /*[8]*/, float* s_incl /*[256]*/,
                                                 float* excl) {
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
        float w = lane < kDrawThreads / 32 ? s_warp[lane] : 0.f;
        float wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        if (lane < kDrawThreads / 32) s_warp[lane] = wi - w;
    }
    __syncthreads();
    incl += s_warp[warp];
    s_incl[threadIdx.x] = incl;
    __syncthreads();
    *excl = threadIdx.x ? s_incl[threadIdx.x - 1] : 0.f;
    return incl;
}

__device__ __forceinline__ float block_sum(float v, float* s_warp /*[8]*/) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) s_warp[warp] = v;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kDrawThreads / 32; ++w) t += s_warp[w];
    return t;
}

enum DrawMode { kBonus = 0, kOneHot = 1, kResidual = 2 };

// Stage the draw weights of elements [e0, e0+n) of row j into w_stage[0..n)
// and return this thread's share of their sum:
//   residual:  w = max(0, 2^(z*s - lse_p) - 2^(y*s - lse_q))
//   otherwise: w = 2^(z*s - lse_p), with w = 0 at element `zero_at`
// Aligned rows use 16-byte loads, kUnroll of them (per row) in flight per
// thread; the ragged end and unaligned rows use element loads.
template <typename T, bool kResid>
__device__ __forceinline__ float stage_weights(const unsigned char* trow, const unsigned char* drow, int e0, int n,
                                               float scale, float lse_p, float lse_q, int zero_at, bool vec_ok,
                                               float* w_stage) {
    constexpr int PV = Logit<T>::kPerVec;
    constexpr int kUnroll = 4;
    const int tid = threadIdx.x;
    float acc = 0.f;
    int done = 0;
    if (vec_ok) {
        const int nvec = static_cast<int>((int64_t(n) * Logit<T>::kSize) >> 4);
        const unsigned char* tsrc = trow + int64_t(e0) * Logit<T>::kSize;
        const unsigned char* dsrc = kResid ? drow + int64_t(e0) * Logit<T>::kSize : nullptr;
        for (int v0 = tid; v0 < nvec; v0 += kDrawThreads * kUnroll) {
            uint4 a[kUnroll], d[kUnroll];
#pragma unroll
            for (int k = 0; k < kUnroll; ++k) {
                const int v = v0 + k * kDrawThreads;
                if (v < nvec) {
                    a[k] = ld_global_stream_v4(tsrc + 16 * int64_t(v));
                    if constexpr (kResid) d[k] = ld_global_stream_v4(dsrc + 16 * int64_t(v));
                }
            }
#pragma unroll
            for (int k = 0; k < kUnroll; ++k) {
                const int v = v0 + k * kDrawThreads;
                if (v < nvec) {
                    float f[PV];
                    Logit<T>::unpack(a[k], f);
                    float g[PV];
                    if constexpr (kResid) Logit<T>::unpack(d[k], g);
#pragma unroll
                    for (int e = 0; e < PV; ++e) {
                        float w = ex2_approx(fmaf(f[e], scale, -lse_p));
                        if constexpr (kResid) w = fmaxf(0.f, w - ex2_approx(fmaf(g[e], scale, -lse_q)));
                        else if (v * PV + e == zero_at) w = 0.f;
                        f[e] = w;
                        acc += w;
                    }
                    float4* dst = reinterpret_cast<float4*>(w_stage + v * PV);
#pragma unroll
                    for (int e = 0; e < PV; e += 4) dst[e / 4] = make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
                }
            }
        }
        done = nvec * PV;
    }
    for (int e = done + tid; e < n; e += kDrawThreads) {
        float w = ex2_approx(fmaf(Logit<T>::load(trow, e0 + e), scale, -lse_p));
        if constexpr (kResid) w = fmaxf(0.f, w - ex2_approx(fmaf(Logit<T>::load(drow, e0 + e), scale, -lse_q)));
        else if (e == zero_at) w = 0.f;
        w_stage[e] = w;
        acc += w;
    }
    return acc;
}

template <typename T>
__global__ void __launch_bounds__(kDrawThreads)
verify_draw_kernel(const DrawParams p) {
    extern __shared__ __align__(16) float dsm[];
    __shared__ float s_Wc[kMaxChunks];
    __shared__ float s_warp[kDrawThreads / 32];
    __shared__ float s_incl[kDrawThreads];
    __shared__ int s_first, s_fail, s_cstar, s_mode, s_found, s_lastpos, s_seg;
    __shared__ float s_local_target;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = blockIdx.x;
    const int b = p.b0 + blockIdx.y;
    const int K = p.k_max;
    const int R = 2 * K + 1;
    const int64_t esz = Logit<T>::kSize;
    float* w_stage = dsm;
    float* s_lse_t = dsm + p.CE;
    float* s_lse_d = s_lse_t + (K + 1);
    float* s_p = s_lse_d + K;
    float* s_q = s_p + K;
    int* s_arg_t = reinterpret_cast<int*>(s_lse_t);  // greedy: argmax per target row
    const int32_t* x = p.tokens + int64_t(b) * K;
    int32_t* out_tok = p.out_tokens ? p.out_tokens + int64_t(b) * (K + 1) : nullptr;
    const bool has_draft = p.draft != nullptr && !p.greedy;

    auto write_failed = [&](int code) {
        if (c != 0) return;
        if (p.stats_only) {
            for (int i = tid; i <= K; i += kDrawThreads) p.out_lse_t[int64_t(b) * (K + 1) + i] = __int_as_float(0x7fc00000);
            for (int i = tid; i < K; i += kDrawThreads) {
                if (p.out_lse_d) p.out_lse_d[int64_t(b) * K + i] = __int_as_float(0x7fc00000);
                if (p.out_p) p.out_p[int64_t(b) * K + i] = __int_as_float(0x7fc00000);
                if (p.out_q) p.out_q[int64_t(b) * K + i] = __int_as_float(0x7fc00000);
            }
        } else {
            for (int i = tid; i <= K; i += kDrawThreads) out_tok[i] = -1;
            if (tid == 0) p.out_len[b] = code;
        }
    };

    // 1. validation --------------------------------------------------------------
    const int L = p.lens ? __ldg(p.lens + b) : K;
    bool ok = L >= 0 && L <= K;
    if (ok)
        for (int i = tid; i < L; i += kDrawThreads) {
            const int xi = __ldg(x + i);
            if (xi < 0 || xi >= p.V) ok = false;
        }
    if (!__syncthreads_and(ok)) {
        write_failed(-1);
        return;
    }

    // 2. merge row partials -----------------------------------------------------
    if (tid == 0) { s_fail = 0; s_first = L; }
    const int n_t = L + 1;
    const int n_d = has_draft ? L : 0;
    __syncthreads();
    for (int row = warp; row < n_t + n_d; row += kDrawThreads / 32) {
        const int slot = row < n_t ? row : K + 1 + (row - n_t);
        const float2* pp = p.partials + (int64_t(b) * R + slot) * p.C;
        const float2 v = lane < p.C ? pp[lane] : make_float2(-INFINITY, 0.f);
        if (p.greedy) {
            const int idx = __float_as_int(v.y);
            const bool bad = lane < p.C && (idx < 0 || idx >= p.V);
            VI r = warp_merge_vi(lane < p.C ? VI{v.x, idx} : VI{-INFINITY, 0x7fffffff});
            if (__any_sync(0xffffffffu, bad) && lane == 0) s_fail = 1;
            if (lane == 0) s_arg_t[row] = r.i;
        } else {
            const bool bad = lane < p.C && (isnan(v.x) || isnan(v.y));
            MS r = warp_merge_ms(MS{v.x, v.y});
            if (__any_sync(0xffffffffu, bad) && lane == 0) s_fail = 1;
            if (lane == 0) {
                const float lse2 = r.m + log2f(r.s);
                if (row < n_t) s_lse_t[row] = lse2; else s_lse_d[row - n_t] = lse2;
            }
        }
    }
    __syncthreads();
    if (s_fail) {
        write_failed(-2);
        return;
    }

    // 3. p, q at the drafted ids; acceptance scan --------------------------------
    const float* u = p.uniforms ? p.uniforms + int64_t(b) * (K + 1) : nullptr;
    for (int i = tid; i < L; i += kDrawThreads) {
        const int xi = __ldg(x + i);
        bool rej;
        if (p.greedy) {
            rej = xi != s_arg_t[i];
        } else {
            const unsigned char* trow = p.target + (int64_t(b) * (K + 1) + i) * p.row_stride * esz;
            const float pi = exp2f(Logit<T>::load(trow, xi) * p.scale - s_lse_t[i]);
            float qi = 1.f;
            if (has_draft) {
                const unsigned char* drow = p.draft + (int64_t(b) * K + i) * p.row_stride * esz;
                qi = exp2f(Logit<T>::load(drow, xi) * p.scale - s_lse_d[i]);
            }
            s_p[i] = pi;
            s_q[i] = qi;
            float a = pi / qi;
            a = a > 1.f ? 1.f : a;  // min(1, p/q); NaN stays NaN (rejects)
            rej = p.stats_only ? false : !(__ldg(u + i) < a);
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

    // 4. final draw on row j -----------------------------------------------------
    const float lse_p = s_lse_t[j];
    const float ustar = __ldg(u + K);
    const unsigned char* trow = p.target + (int64_t(b) * (K + 1) + j) * p.row_stride * esz;
    const int e0 = c * p.CE;
    const int n = min(p.V - e0, p.CE);
    int mode = j == L ? kBonus : (has_draft ? kResidual : kOneHot);

    if (mode == kResidual) {
        const float lse_q = s_lse_d[j];
        const unsigned char* drow = p.draft + (int64_t(b) * K + j) * p.row_stride * esz;
        const float acc = stage_weights<T, true>(trow, drow, e0, n, p.scale, lse_p, lse_q, -1, p.rows_aligned != 0,
                                                 w_stage);
        const float Wc = block_sum(acc, s_warp);
        cg::cluster_group cluster = cg::this_cluster();
        if (tid < p.C) {
            float* remote = cluster.map_shared_rank(&s_Wc[0], tid);
            remote[c] = Wc;
        }
        cluster.sync();
    }

    if (tid == 0) {
        float W[kMaxChunks];
        float total = 0.f;
        for (int cc = 0; cc < p.C; ++cc) {
            if (mode == kResidual) {
                W[cc] = s_Wc[cc];
            } else {
                const float2 pp = p.partials[(int64_t(b) * R + j) * p.C + cc];
                W[cc] = pp.y * exp2f(pp.x - lse_p);
            }
        }
        if (mode == kOneHot) {
            const int xj = __ldg(x + j);
            const int cx = xj / p.CE;
            W[cx] = fmaxf(0.f, W[cx] - s_p[j]);
        }
        for (int cc = 0; cc < p.C; ++cc) total += W[cc];
        if (!(total > 0.f)) {
            // zero residual mass (p == q numerically): draw from p_j
            mode = kBonus;
            total = 0.f;
            for (int cc = 0; cc < p.C; ++cc) {
                const float2 pp = p.partials[(int64_t(b) * R + j) * p.C + cc];
                W[cc] = pp.y * exp2f(pp.x - lse_p);
                total += W[cc];
            }
        }
        const float target = ustar * total;
        int cstar = -1, last_pos = 0;
        float before = 0.f, run = 0.f;
        for (int cc = 0; cc < p.C; ++cc) {
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
    }
    __syncthreads();
    if (c != s_cstar) return;
    const bool restage = s_mode != kResidual;
    if (restage) {
        // w = p_j, and max(0, p - 1) = 0 at the drafted id for one-hot q
        const int zero_at = s_mode == kOneHot ? __ldg(x + j) - e0 : -1;
        (void)stage_weights<T, false>(trow, nullptr, e0, n, p.scale, lse_p, 0.f, zero_at, p.rows_aligned != 0,
                                      w_stage);
    }
    if (tid == 0) { s_found = 0x7fffffff; s_lastpos = -1; s_seg = 0x7fffffff; }
    __syncthreads();

    // Inverse CDF inside the chunk: contiguous segments per thread (odd length
    // to keep shared-memory banks apart), a block scan of the segment sums,
    // then a walk of the first segment with positive weight whose running
    // sum passes the target.  Only a segment holding positive weight can be
    // chosen, so rounding in the scan can never select a zero-weight token;
    // when rounding leaves the target past the last step, the chunk's last
    // positive-weight token is taken.
    const float target = s_local_target;
    const int seg = ((n + kDrawThreads - 1) / kDrawThreads) | 1;
    const int lo = min(n, tid * seg), hi = min(n, lo + seg);
    float ssum = 0.f;
    int lastpos = -1;
    for (int e = lo; e < hi; ++e) {
        const float w = w_stage[e];
        ssum += w;
        if (w > 0.f) lastpos = e;
    }
    float excl;
    const float incl = block_scan_incl(ssum, s_warp, s_incl, &excl);
    if (lastpos >= 0) atomicMax(&s_lastpos, lastpos);
    if (lastpos >= 0 && incl > target) atomicMin(&s_seg, tid);
    __syncthreads();
    if (tid == s_seg) {
        float acc = excl;
        int f = lastpos;
        for (int e = lo; e < hi; ++e) {
            acc += w_stage[e];
            if (acc > target && w_stage[e] > 0.f) { f = e; break; }
        }
        s_found = f;
    }
    __syncthreads();
    if (tid == 0) {
        int t = s_found != 0x7fffffff ? s_found : s_lastpos;
        if (t < 0) t = 0;
        out_tok[j] = e0 + t;
    }
}

}  // namespace sv
