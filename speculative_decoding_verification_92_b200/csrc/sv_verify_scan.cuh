// sv_verify_scan.cuh -- K2a, the acceptance scan (one CTA per request).
//
//  1. validate draft_lens[b] and the first L drafted ids (bad values never
//     cause an access: the request is reported with out_accept_len = -1);
//     gather the logits at the drafted ids and the uniforms (inputs only, so
//     this overlaps the tail of the row-statistics kernel);
//  2. merge the P row-statistics partials of every used row into lse (log2
//     domain) -- or into the row argmax for greedy verification;
//  3. p_i = 2^(z_i(x_i)/T*log2e - lse_i), q_i likewise or 1 for one-hot q,
//     a_i = min(1, p_i/q_i), reject when !(u_i < a_i); j = first rejection
//     ("AI 开始抄自己的作业——而且抄得理直气壮", section "⚡ 投机解码：让草稿先跑，
//     考官殿后"; stop at the first rejection: "今热点：让AI草稿模型学会"照镜子"",
//     section "先搞懂投机解码在干什么");
//  4. write out_accept_len = j, the accepted ids and -1 after position j
//     (greedy: the argmax of row j at position j);
//  5. sampling: queue the final draw on row j for the draw kernel --
//       bonus (j == L):        w = p_L; the piece holding u*W is chosen here
//                              from row L's partials (one piece to load);
//       one-hot rejection:     w = p_j with the drafted id removed (one task:
//                              it loads the drafted id's piece first);
//       draft rejection:       w = max(0, p_j - q_j) (P tasks, one per piece).
// Statistics-only calls (spec_verify_stats, spec_verify_accept_sim) stop after
// step 3 and write their per-row outputs instead.
#pragma once

#include "spec_verify.h"
#include "sv_common.cuh"

namespace sv {

enum DrawMode { kBonus = 0, kOneHot = 1, kResidual = 2 };

// One final draw queued for the draw kernel.
struct alignas(16) DrawReq {
    int32_t b;          // request
    int32_t j;          // row of the draw (accepted drafts)
    int32_t mode;       // DrawMode
    int32_t x;          // drafted id at position j (one-hot), else -1
    int32_t piece;      // bonus: the piece that holds u*W; else -1
    float lse_p;        // log2-domain lse of target row j
    float lse_q;        // log2-domain lse of draft row j (residual)
    float ustar;        // uniforms[b][k_max]
    float target;       // bonus: u*W minus the weight of the pieces before `piece`
                        // (+inf: rounding left u*W past the last step)
    int32_t pad[3];
};
static_assert(sizeof(DrawReq) == 48, "DrawReq layout");

struct ScanParams {
    const unsigned char* target;
    const unsigned char* draft;  // null -> one-hot q
    const int32_t* tokens;
    const int32_t* lens;         // null -> k_max
    const float* uniforms;       // null allowed when greedy / statistics only
    const float2* partials;      // [B][2k+1][P]
    int32_t* out_len;
    int32_t* out_tokens;
    float* out_lse_t;            // statistics outputs (natural log), may be null
    float* out_lse_d;
    float* out_p;
    float* out_q;
    float* out_accept_prob;      // acceptance simulation outputs, may be null
    float* out_expected_len;
    int32_t* out_first_reject;
    float* out_weights;
    float decay;
    int32_t* ctrl;               // [0] residual draws queued, [1] single-piece draws queued
    DrawReq* res_req;            // [B] residual draws
    DrawReq* one_req;            // [B] bonus / one-hot draws
    int32_t* res_lost;           // [B] residual draws lost by the draw kernel (cleared here)
    int32_t k_max;
    int32_t V;
    int64_t row_stride;
    int32_t P;                   // pieces per row (partials per row)
    int32_t PE;                  // elements per piece
    float scale;                 // log2(e) / T
    int32_t greedy;
    int32_t stats_only;
};

constexpr int kScanThreads = 256;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kMaxDraftsPerThread = (SV_MAX_K + kScanThreads - 1) / kScanThreads;

// Dynamic shared memory: lse_t[k+1] | lse_d[k] | p[k] | q[k] | x[k] | the target
// rows' partials [k+1][P] (kept for the bonus draw's piece choice when they
// fit in kScanPartBytes; otherwise that choice reads them again).
constexpr size_t kScanPartBytes = 24 * 1024;
__host__ __device__ inline size_t scan_scalar_bytes(int k_max) {
    return (4 * (size_t(k_max + 1) + 4 * size_t(k_max)) + 127) & ~size_t(127);
}
__host__ __device__ inline bool scan_keeps_partials(int k_max, int P) {
    return size_t(k_max + 1) * size_t(P) * 8 <= kScanPartBytes;
}
__host__ __device__ inline size_t scan_smem_bytes(int k_max, int P) {
    return scan_scalar_bytes(k_max) + (scan_keeps_partials(k_max, P) ? size_t(k_max + 1) * size_t(P) * 8 : 0);
}

// Acceptance probability min(1, p/q); NaN stays NaN (and then rejects).
__device__ __forceinline__ float accept_prob(float p, float q) {
    const float a = p / q;
    return a > 1.f ? 1.f : a;
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

// Warp-wide pick of the block holding `target` among n consecutive blocks of
// weights, lane l holding blocks [l*cps, l*cps + cps) in w_l (cps = ceil(n/32),
// at most kMaxPer): the first block with positive weight at which the running
// sum exceeds target, else (rounding) the last block with positive weight.
// Returns the block (-1 when no block has positive weight) and, through
// *local, target minus the weight before it (+inf for the fallback).
template <int kMaxPer>
__device__ __forceinline__ int warp_pick(const float (&w)[kMaxPer], int n, float target, float* local) {
    const int lane = threadIdx.x & 31;
    const int cps = (n + 31) / 32;
    const int s0 = lane * cps;
    const int ns = min(cps, max(0, n - s0));
    float mine = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i)
        if (i < ns) mine += w[i];
    const float li = warp_scan_incl(mine);
    const unsigned cross = __ballot_sync(0xffffffffu, mine > 0.f && li > target);
    const unsigned pos = __ballot_sync(0xffffffffu, mine > 0.f);
    const int lsel = cross ? __ffs(cross) - 1 : (pos ? 31 - __clz(pos) : -1);
    if (lsel < 0) {
        *local = INFINITY;
        return -1;
    }
    int blk = 0;
    float t_loc = INFINITY;
    if (lane == lsel) {
        const float t1 = cross ? target : INFINITY;
        float run = li - mine, before = 0.f, last_before = 0.f;
        int isel = -1, ilast = -1;
#pragma unroll
        for (int i = 0; i < kMaxPer; ++i) {
            if (i < ns && isel < 0) {
                const float wi = w[i];
                if (wi > 0.f) {
                    ilast = i;
                    last_before = run;
                    if (run + wi > t1) { isel = i; before = run; }
                }
                run += wi;
            }
        }
        const bool hit = isel >= 0;
        if (!hit) { isel = ilast; before = last_before; }
        blk = s0 + isel;
        t_loc = hit ? t1 - before : INFINITY;
    }
    *local = __shfl_sync(0xffffffffu, t_loc, lsel);
    return __shfl_sync(0xffffffffu, blk, lsel);
}

constexpr int kMaxPieces = (SV_MAX_V * 4 + kPieceBytes - 1) / kPieceBytes;
constexpr int kMaxPiecesPerLane = (kMaxPieces + 31) / 32;

// The shared-memory scalars of one request's scan.
struct ScanShared {
    int first, fail;
    float ustar;
    DrawReq draw;
};

// Steps 1-5 for request b, by one CTA of kScanThreads threads (all of them
// call it; scan_dsm holds scan_smem_bytes(k_max, P) bytes).  `outputs`: this
// CTA writes the request's outputs (step 4); `queue`: the scan kernel's
// form -- it lets the next grid launch before step 4 and queues the final
// draw for the draw kernel itself.  Otherwise returns true when a final draw
// follows (sampling, valid request), with the draw in ss->draw (visible to
// every thread: the function ends with __syncthreads() then).
template <typename T>
__device__ __forceinline__ bool scan_request(const ScanParams& p, int b, unsigned char* scan_dsm, ScanShared* ss,
                                             bool outputs, bool queue) {
    int& s_first = ss->first;
    int& s_fail = ss->fail;
    float& s_ustar = ss->ustar;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = p.k_max;
    const int nslots = 2 * K + 1;  // partial rows per request
    const int P = p.P;
    const int64_t esz = Logit<T>::kSize;
    float* s_lse_t = reinterpret_cast<float*>(scan_dsm);
    float* s_lse_d = s_lse_t + (K + 1);
    float* s_p = s_lse_d + K;   // gathered z(x_i), then p_i
    float* s_q = s_p + K;       // gathered y(x_i), then q_i
    int* s_x = reinterpret_cast<int*>(s_q + K);  // the drafted ids (valid ones only)
    int* s_arg_t = reinterpret_cast<int*>(s_lse_t);  // greedy: argmax per target row
    const bool keep_parts = !p.greedy && !p.stats_only && scan_keeps_partials(K, P);
    float2* s_part_t = reinterpret_cast<float2*>(scan_dsm + scan_scalar_bytes(K));  // [L+1][P] when kept
    const int32_t* x = p.tokens + int64_t(b) * K;
    int32_t* out_tok = p.out_tokens ? p.out_tokens + int64_t(b) * (K + 1) : nullptr;
    const bool has_draft = p.draft != nullptr && !p.greedy;
    const float* u = p.uniforms ? p.uniforms + int64_t(b) * (K + 1) : nullptr;
    auto trow_of = [&](int i) { return p.target + (int64_t(b) * (K + 1) + i) * p.row_stride * esz; };
    auto drow_of = [&](int i) { return p.draft + (int64_t(b) * K + i) * p.row_stride * esz; };

    auto write_failed = [&](int code) {
        const float nan = __int_as_float(0x7fc00000);
        if (p.stats_only) {
            for (int i = tid; i <= K; i += kScanThreads)
                if (p.out_lse_t) p.out_lse_t[int64_t(b) * (K + 1) + i] = nan;
            for (int i = tid; i < K; i += kScanThreads) {
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
            for (int i = tid; i <= K; i += kScanThreads) out_tok[i] = -1;
            if (tid == 0) p.out_len[b] = code;
        }
    };

    // 1. inputs only: validation, gathered logits at the drafted ids, uniforms
    const int L = p.lens ? __ldg(p.lens + b) : K;
    bool ok = L >= 0 && L <= K;
    int xr[kMaxDraftsPerThread];
#pragma unroll
    for (int k = 0; k < kMaxDraftsPerThread; ++k) {
        const int i = tid + k * kScanThreads;
        xr[k] = 0;
        if (ok && i < L) {
            xr[k] = __ldg(x + i);
            if (xr[k] < 0 || xr[k] >= p.V) ok = false;
            s_x[i] = xr[k];
        }
    }
    // the final draw's uniform, read now so that step 5 waits on no load
    if (tid == 0 && u && !p.greedy && !p.stats_only) s_ustar = __ldg(u + K);
    ok = __syncthreads_and(ok);
    float ur[kMaxDraftsPerThread];
    if (ok && !p.greedy) {
#pragma unroll
        for (int k = 0; k < kMaxDraftsPerThread; ++k) {
            const int i = tid + k * kScanThreads;
            ur[k] = 0.f;
            if (i < L) {
                s_p[i] = Logit<T>::load(trow_of(i), xr[k]);
                if (has_draft) s_q[i] = Logit<T>::load(drow_of(i), xr[k]);
                if (u) ur[k] = __ldg(u + i);
            }
        }
    }

    // 2. the row-statistics kernel's partials (this kernel is a programmatic
    // dependent of it: wait for its completion before reading them).  Four
    // lanes merge one row, 64 rows at a time: lane q of a row's group folds
    // the row's partials q, q + 4, ... (maximum first, then the rescaled
    // sums), and two shuffles combine the four.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (!ok) {
        if (outputs) write_failed(-1);
        return false;
    }
    if (tid == 0) { s_fail = 0; s_first = L; }
    const int n_t = L + 1;
    const int n_d = has_draft ? L : 0;
    const int nrows = n_t + n_d;
    {
        constexpr int kLanesPerRow = 4;
        constexpr int kRowsPerPass = kScanThreads / kLanesPerRow;
        constexpr int kMaxPerLane = (kMaxPieces + kLanesPerRow - 1) / kLanesPerRow;
        const float2* part_b = p.partials + int64_t(b) * nslots * P;
        const int q = tid & (kLanesPerRow - 1);
        bool bad = false;
        for (int r0 = 0; r0 < nrows; r0 += kRowsPerPass) {
            const int row = r0 + tid / kLanesPerRow;
            const bool act = row < nrows;
            const int slot = row < n_t ? row : K + 1 + (row - n_t);
            const float2* pr = part_b + int64_t(slot) * P;
            float2 v[kMaxPerLane];
#pragma unroll
            for (int k = 0; k < kMaxPerLane; ++k) {
                const int c = q + kLanesPerRow * k;
                v[k] = (act && c < P) ? pr[c] : make_float2(-INFINITY, p.greedy ? __int_as_float(0x7fffffff) : 0.f);
                if (keep_parts && act && row < n_t && c < P) s_part_t[row * P + c] = v[k];
            }
            if (p.greedy) {
                VI r{v[0].x, __float_as_int(v[0].y)};
#pragma unroll
                for (int k = 0; k < kMaxPerLane; ++k) {
                    if (act && q + kLanesPerRow * k < P) {
                        const int idx = __float_as_int(v[k].y);
                        bad |= idx < 0 || idx >= p.V;
                    }
                    if (k > 0) r = vi_better(r, VI{v[k].x, __float_as_int(v[k].y)});
                }
#pragma unroll
                for (int o = 1; o < kLanesPerRow; o <<= 1)
                    r = vi_better(r, VI{__shfl_xor_sync(0xffffffffu, r.v, o), __shfl_xor_sync(0xffffffffu, r.i, o)});
                if (act && q == 0) s_arg_t[row] = r.i;
            } else {
                float m = -INFINITY;
#pragma unroll
                for (int k = 0; k < kMaxPerLane; ++k) {
                    bad |= isnan(v[k].x) || isnan(v[k].y);
                    m = fmaxf(m, v[k].x);
                }
#pragma unroll
                for (int o = 1; o < kLanesPerRow; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                float sum = 0.f;
                if (m != -INFINITY) {
#pragma unroll
                    for (int k = 0; k < kMaxPerLane; ++k)
                        if (v[k].x != -INFINITY) sum = fmaf(v[k].y, ex2_approx(v[k].x - m), sum);
                }
#pragma unroll
                for (int o = 1; o < kLanesPerRow; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                if (act && q == 0) {
                    const float lse2 = m + log2f(sum);
                    if (row < n_t) s_lse_t[row] = lse2; else s_lse_d[row - n_t] = lse2;
                }
            }
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0) s_fail = 1;
    }
    __syncthreads();
    if (s_fail) {
        if (outputs) write_failed(-2);
        return false;
    }

    // 3. p, q at the drafted ids; acceptance scan ----------------------------------
#pragma unroll
    for (int k = 0; k < kMaxDraftsPerThread; ++k) {
        const int i = tid + k * kScanThreads;
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
        const float nan = __int_as_float(0x7fc00000);
        const int j = s_first;  // L when no uniforms were given
        for (int i = tid; i <= K; i += kScanThreads)
            if (p.out_lse_t) p.out_lse_t[int64_t(b) * (K + 1) + i] = i <= L ? s_lse_t[i] * kLn2 : nan;
        for (int i = tid; i < K; i += kScanThreads) {
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
        return false;
    }

    // 4. outputs of the scan -----------------------------------------------------------
    // The draw kernel may be launched now (its CTAs then wait for this grid);
    // launching it earlier would let its waiting CTAs slow this grid down.
    if (queue && tid == 0) asm volatile("griddepcontrol.launch_dependents;");
    const int j = s_first;
    if (outputs) {
        for (int i = tid; i <= K; i += kScanThreads) {
            if (i < j) out_tok[i] = s_x[i];
            else if (i > j) out_tok[i] = -1;
            else if (p.greedy) out_tok[i] = s_arg_t[j];
        }
        if (tid == 0) p.out_len[b] = j;
    }
    if (p.greedy) return false;

    // 5. the final draw on row j ----------------------------------------------------------
    if (warp == 0) {
        DrawReq r;
        r.b = b;
        r.j = j;
        r.mode = j == L ? kBonus : (has_draft ? kResidual : kOneHot);
        r.x = j < L ? s_x[j] : -1;
        r.piece = -1;
        r.lse_p = s_lse_t[j];
        r.lse_q = r.mode == kResidual ? s_lse_d[j] : 0.f;
        r.ustar = s_ustar;
        r.target = INFINITY;
        r.pad[0] = r.pad[1] = r.pad[2] = 0;
        if (r.mode == kBonus) {
            // piece weights of p_L from the partials: s * 2^(m - lse); lane l
            // holds pieces [l*cps, l*cps + cps)
            const float2* part_j = keep_parts ? s_part_t + j * P : p.partials + (int64_t(b) * nslots + j) * P;
            const int cps = (P + 31) / 32;
            float w[kMaxPiecesPerLane];
#pragma unroll
            for (int i = 0; i < kMaxPiecesPerLane; ++i) {
                const int c = lane * cps + i;
                w[i] = 0.f;
                if (i < cps && c < P) {
                    const float2 pp = part_j[c];
                    w[i] = pp.y * exp2f(pp.x - r.lse_p);
                }
            }
            float tot = 0.f;
#pragma unroll
            for (int i = 0; i < kMaxPiecesPerLane; ++i) tot += w[i];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
            float local;
            const int pc = warp_pick<kMaxPiecesPerLane>(w, P, r.ustar * tot, &local);
            r.piece = pc < 0 ? 0 : pc;
            r.target = pc < 0 ? INFINITY : local;
        }
        if (lane == 0) {
            if (!queue) {
                ss->draw = r;
            } else if (r.mode == kResidual) {
                const int slot = atomicAdd(p.ctrl + 0, 1);
                p.res_lost[slot] = 0;
                p.res_req[slot] = r;
            } else {
                const int slot = atomicAdd(p.ctrl + 1, 1);
                p.one_req[slot] = r;
            }
        }
    }
    if (queue) return false;
    __syncthreads();
    return true;
}

template <typename T>
__global__ void __launch_bounds__(kScanThreads)
verify_scan_kernel(const ScanParams p) {
    extern __shared__ __align__(128) unsigned char scan_dsm[];
    __shared__ ScanShared ss;
    (void)scan_request<T>(p, blockIdx.x, scan_dsm, &ss, true, true);
}

}  // namespace sv
