// sv_row_stats.cuh -- K1, the row-statistics pass.
//
// Every row a request uses (target rows 0..L_b, draft rows 0..L_b-1) is cut
// into C vocabulary chunks of CE elements.  One work item = one (row, chunk);
// items are dealt round-robin over a persistent grid.  Each item is reduced
// to one partial:
//   sampling: (m, s) with m = max_v t_v, s = sum_v 2^(t_v - m), t_v = z_v * log2(e)/T
//             (the temperature softmax statistics of step 1 of the rule,
//             "AI 开始抄自己的作业——而且抄得理直气壮", section "⚡ 投机解码：让草稿先跑，考官殿后")
//   greedy:   (max z_v, lowest index attaining it)
// written to partials[(b * (2*k_max+1) + slot) * C + c], slot = i for target
// row i and k_max+1+i for draft row i.  K2 merges the C partials of a row.
//
// Variants:
//   row_stats_tma_kernel  one producer warp streams each item through a ring
//                         of shared-memory stages with 1-D cp.async.bulk
//                         copies completing on mbarriers; consumer warps
//                         reduce from shared memory.  Needs 16-byte aligned
//                         rows.  Waits are bounded; a timed-out CTA marks its
//                         remaining items with NaN partials.
//   row_stats_ldg_kernel  the same item schedule with 16-byte vector loads
//                         (aligned rows) or element loads (any alignment).
#pragma once

#include "sv_common.cuh"

// Ring geometry of the bulk-copy variant (compile-time; defaults tuned on B200).
#ifndef SV_STAGE_BYTES
#define SV_STAGE_BYTES 16384
#endif
#ifndef SV_TMA_CONSUMER_WARPS
#define SV_TMA_CONSUMER_WARPS 4
#endif
#ifndef SV_TMA_STAGES
#define SV_TMA_STAGES 2
#endif
// Resident CTAs per SM the bulk-copy variant is built for, per logit type:
// bf16 spends twice the exps per byte of fp32, so it wants more consumer warps
// in flight (6 x 4 on B200); fp32 does best at 5 x 4.
#ifndef SV_TMA_CTAS_PER_SM_BF16
#define SV_TMA_CTAS_PER_SM_BF16 6
#endif
#ifndef SV_TMA_CTAS_PER_SM_F32
#define SV_TMA_CTAS_PER_SM_F32 5
#endif
// 16-byte vectors per thread in flight in the vector-load variant.
#ifndef SV_LDG_UNROLL
#define SV_LDG_UNROLL 4
#endif

namespace sv {

struct StatsParams {
    const unsigned char* target;  // [B][k_max+1][row_stride]
    const unsigned char* draft;   // [B][k_max][row_stride] or null
    const int32_t* lens;          // [B] or null (all k_max)
    float2* partials;             // [B][2*k_max+1][C]
    int32_t b0;                   // first request handled by this launch
    int32_t nB;                   // requests handled by this launch (<= kMaxRequestsPerLaunch)
    int32_t k_max;
    int32_t V;
    int64_t row_stride;           // elements
    int32_t C;                    // chunks per row
    int32_t CE;                   // elements per chunk, multiple of 8
    float scale;                  // log2(e) / T
    int32_t use_draft;            // draft rows are part of the work
    uint64_t timeout_ns;          // bound on each barrier wait (TMA variant)
    int64_t lost_copy_partial;    // test fault injection: this item's first stage is never copied; -1 = off
};

struct ItemDesc {
    const unsigned char* row;     // first byte of the row
    int64_t partial_idx;
    int32_t e0, e1;               // element range of the chunk
};

__device__ __forceinline__ int clamp_len(const StatsParams& p, int b) {
    int L = p.lens ? __ldg(p.lens + b) : p.k_max;
    return L < 0 ? 0 : (L > p.k_max ? p.k_max : L);
}

__device__ __forceinline__ int rows_of(const StatsParams& p, int L) {
    return p.use_draft ? 2 * L + 1 : L + 1;
}

// row_start[i] = number of rows of requests b0 .. b0+i-1, for i in [0, nB].
// Uses a block-wide exclusive scan; ends with __syncthreads().
template <int kThreads>
__device__ void build_row_prefix(const StatsParams& p, int* row_start, int* scratch /*[32]*/) {
    const int tid = threadIdx.x;
    if (p.lens == nullptr) {
        const int r = rows_of(p, p.k_max);
        for (int i = tid; i <= p.nB; i += kThreads) row_start[i] = i * r;
        __syncthreads();
        return;
    }
    const int per = (p.nB + kThreads - 1) / kThreads;
    const int lo = tid * per;
    const int hi = min(p.nB, lo + per);
    int local = 0;
    for (int i = lo; i < hi; ++i) local += rows_of(p, clamp_len(p, p.b0 + i));
    // block exclusive scan of `local`
    const int lane = tid & 31, warp = tid >> 5;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        constexpr int kWarps = kThreads / 32;
        int w = lane < kWarps ? scratch[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        if (lane < kWarps) scratch[lane] = wi - w;
    }
    __syncthreads();
    int run = scratch[warp] + incl - local;
    for (int i = lo; i < hi; ++i) {
        row_start[i] = run;
        run += rows_of(p, clamp_len(p, p.b0 + i));
    }
    if (hi == p.nB && lo < hi) row_start[p.nB] = run;
    if (p.nB == 0 && tid == 0) row_start[0] = 0;
    __syncthreads();
}

template <typename T>
__device__ __forceinline__ ItemDesc decode_item(const StatsParams& p, const int* row_start, int64_t item) {
    const int64_t g = item / p.C;
    const int c = static_cast<int>(item - g * p.C);
    int lo = 0, hi = p.nB;  // row_start[lo] <= g < row_start[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (row_start[mid] <= g) lo = mid; else hi = mid;
    }
    const int bl = lo;
    const int b = p.b0 + bl;
    const int r = static_cast<int>(g - row_start[bl]);
    const int nrows = row_start[bl + 1] - row_start[bl];
    const int L = p.use_draft ? (nrows - 1) / 2 : nrows - 1;
    ItemDesc d;
    int slot;
    if (r <= L) {
        slot = r;
        d.row = p.target + ((int64_t)b * (p.k_max + 1) + r) * p.row_stride * Logit<T>::kSize;
    } else {
        const int i = r - L - 1;
        slot = p.k_max + 1 + i;
        d.row = p.draft + ((int64_t)b * p.k_max + i) * p.row_stride * Logit<T>::kSize;
    }
    d.partial_idx = ((int64_t)b * (2 * p.k_max + 1) + slot) * p.C + c;
    d.e0 = c * p.CE;
    d.e1 = min(p.V, d.e0 + p.CE);
    return d;
}

// Per-thread accumulators -----------------------------------------------------

template <bool kGreedy> struct Acc;

template <> struct Acc<false> {
    MS ms;
    __device__ __forceinline__ void reset() { ms = MS{-INFINITY, 0.f}; }
    // Fold N raw logits z (-inf for absent lanes) with t = z * scale: tree max,
    // one ex2 per element of fma(z, scale, -M), tree sum -- short dependency
    // chains so few warps keep the FMA and MUFU pipes busy.
    template <int N>
    __device__ __forceinline__ void fold_raw(const float (&z)[N], float scale) {
        float m[N];
#pragma unroll
        for (int i = 0; i < N; ++i) m[i] = z[i];
#pragma unroll
        for (int w = 1; w < N; w <<= 1)
#pragma unroll
            for (int i = 0; i + w < N; i += 2 * w) m[i] = fmaxf(m[i], m[i + w]);
        const float M = fmaxf(ms.m, m[0] * scale);
        if (M == -INFINITY) return;
        float e[N];
#pragma unroll
        for (int i = 0; i < N; ++i) e[i] = ex2_approx(fmaf(z[i], scale, -M));
#pragma unroll
        for (int w = 1; w < N; w <<= 1)
#pragma unroll
            for (int i = 0; i + w < N; i += 2 * w) e[i] += e[i + w];
        ms = MS{M, fmaf(ms.s, ex2_approx(ms.m - M), e[0])};
    }
    __device__ __forceinline__ void fold1(float t) {
        const float m = fmaxf(ms.m, t);
        if (m == -INFINITY) return;
        ms = MS{m, ms.s * ex2_approx(ms.m - m) + ex2_approx(t - m)};
    }
};

template <> struct Acc<true> {
    VI vi;
    __device__ __forceinline__ void reset() { vi = VI{-INFINITY, 0x7fffffff}; }
    __device__ __forceinline__ void take(float z, int idx) {
        if (z > vi.v || (z == vi.v && idx < vi.i)) vi = VI{z, idx};
    }
};

// Fold K 16-byte vectors of raw logits into a sampling accumulator.  The
// row maximum of bf16 data comes from max.bf16x2 on the stored words (half an
// instruction per element, no unpacking); then each element costs one
// integer unpack (bf16), one FFMA for z * scale - M, one ex2 and one FADD into
// one of four independent partial sums.  Absent vectors must be passed as
// -inf (bf16 words 0xff80ff80, fp32 0xff800000).
constexpr uint32_t kBf16NegInfPair = 0xff80ff80u;
constexpr uint32_t kF32NegInfBits = 0xff800000u;

template <typename T, int K>
__device__ __forceinline__ void fold_vectors(Acc<false>& acc, const uint4 (&v)[K], float scale) {
    constexpr int NW = 4 * K;
    uint32_t w[NW];
#pragma unroll
    for (int k = 0; k < K; ++k) {
        w[4 * k] = v[k].x; w[4 * k + 1] = v[k].y; w[4 * k + 2] = v[k].z; w[4 * k + 3] = v[k].w;
    }
    float zmax;
    if constexpr (Logit<T>::kSize == 2) {
        uint32_t m[NW];
#pragma unroll
        for (int i = 0; i < NW; ++i) m[i] = w[i];
#pragma unroll
        for (int d = 1; d < NW; d <<= 1)
#pragma unroll
            for (int i = 0; i + d < NW; i += 2 * d) m[i] = bf16x2_max(m[i], m[i + d]);
        zmax = fmaxf(bf16_lo(m[0]), bf16_hi(m[0]));
    } else {
        float m[NW];
#pragma unroll
        for (int i = 0; i < NW; ++i) m[i] = __uint_as_float(w[i]);
#pragma unroll
        for (int d = 1; d < NW; d <<= 1)
#pragma unroll
            for (int i = 0; i + d < NW; i += 2 * d) m[i] = fmaxf(m[i], m[i + d]);
        zmax = m[0];
    }
    const float M = fmaxf(acc.ms.m, zmax * scale);
    if (M == -INFINITY) return;
    const float negM = -M;
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < NW; ++i) {
        if constexpr (Logit<T>::kSize == 2) {
            s[(2 * i) & 3] += ex2_approx(fmaf(bf16_lo(w[i]), scale, negM));
            s[(2 * i + 1) & 3] += ex2_approx(fmaf(bf16_hi(w[i]), scale, negM));
        } else {
            s[i & 3] += ex2_approx(fmaf(__uint_as_float(w[i]), scale, negM));
        }
    }
    acc.ms = MS{M, fmaf(acc.ms.s, ex2_approx(acc.ms.m - M), (s[0] + s[1]) + (s[2] + s[3]))};
}

// Fold only the first `nv` (0 <= nv <= K) of K vectors: one fold with a
// compile-time count per possible nv, so no ex2 is spent on absent elements
// (the partial stage or batch at the end of each item).
template <typename T, int K, int N>
__device__ __forceinline__ void fold_prefix(Acc<false>& acc, const uint4 (&v)[K], float scale) {
    uint4 part[N];
#pragma unroll
    for (int k = 0; k < N; ++k) part[k] = v[k];
    fold_vectors<T, N>(acc, part, scale);
}

template <typename T, int K, int N>
__device__ __forceinline__ void fold_prefix_select(Acc<false>& acc, const uint4 (&v)[K], int nv, float scale) {
    if constexpr (N >= 1) {
        if (nv == N) {
            fold_prefix<T, K, N>(acc, v, scale);
            return;
        }
        fold_prefix_select<T, K, N - 1>(acc, v, nv, scale);
    }
}

template <typename T, int K>
__device__ __forceinline__ void fold_vectors_count(Acc<false>& acc, const uint4 (&v)[K], int nv, float scale) {
    if (nv >= K) fold_vectors<T, K>(acc, v, scale);
    else fold_prefix_select<T, K, K - 1>(acc, v, nv, scale);
}

template <typename T>
__device__ __forceinline__ uint4 neg_inf_vector() {
    const uint32_t x = Logit<T>::kSize == 2 ? kBf16NegInfPair : kF32NegInfBits;
    return make_uint4(x, x, x, x);
}

// Reduce the reducing threads' accumulators and let thread 0 write the
// partial (a NaN pair when any thread lost its data to a wait timeout).
// `red` holds 3 * kWarps floats for this item (double-buffered by the
// caller); `bar_id`/`nthreads` name the barrier of the reducing threads.
template <bool kGreedy, int kWarps>
__device__ __forceinline__ void reduce_and_store(Acc<kGreedy>& acc, float* red, int bar_id, int nthreads,
                                                 float2* out, bool failed) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool warp_failed = __any_sync(0xffffffffu, failed);
    float a, b;
    if constexpr (kGreedy) {
        VI v = warp_merge_vi(acc.vi);
        a = v.v;
        b = __int_as_float(v.i);
    } else {
        MS v = warp_merge_ms_maxfirst(acc.ms);
        a = v.m;
        b = v.s;
    }
    if (lane == 0) {
        red[3 * warp] = a;
        red[3 * warp + 1] = b;
        red[3 * warp + 2] = warp_failed ? 1.f : 0.f;
    }
    named_barrier_sync(bar_id, nthreads);
    if (threadIdx.x == 0) {
        bool any_failed = false;
        for (int w = 0; w < kWarps; ++w) any_failed |= red[3 * w + 2] != 0.f;
        float2 r;
        if constexpr (kGreedy) {
            VI t{red[0], __float_as_int(red[1])};
            for (int w = 1; w < kWarps; ++w) t = vi_better(t, VI{red[3 * w], __float_as_int(red[3 * w + 1])});
            r = make_float2(t.v, __int_as_float(t.i));
        } else {
            MS t{red[0], red[1]};
            for (int w = 1; w < kWarps; ++w) t = ms_merge(t, MS{red[3 * w], red[3 * w + 1]});
            r = make_float2(t.m, t.s);
        }
        if (any_failed) r = make_float2(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
        *out = r;
    }
}

// Fold the elements of one 16-byte vector whose first element has row index
// `idx0`.
template <typename T, bool kGreedy>
__device__ __forceinline__ void fold_vector(Acc<kGreedy>& acc, const uint4& w, int idx0, float scale) {
    float f[Logit<T>::kPerVec];
    Logit<T>::unpack(w, f);
    if constexpr (kGreedy) {
#pragma unroll
        for (int e = 0; e < Logit<T>::kPerVec; ++e) acc.take(f[e], idx0 + e);
    } else {
        acc.fold_raw(f, scale);
    }
}

// ============================================================================
// TMA bulk-copy variant.

constexpr int kStageBytes = SV_STAGE_BYTES;

template <typename T>
struct TmaCtasPerSm {
    static constexpr int value = Logit<T>::kSize == 2 ? SV_TMA_CTAS_PER_SM_BF16 : SV_TMA_CTAS_PER_SM_F32;
};

struct StageMeta {
    const unsigned char* tail;  // first ragged-tail element (row's last chunk), or null
    int64_t partial_idx;
    int32_t elem0;              // row index of the stage's first element
    int32_t n_bytes;            // bytes delivered by the bulk copy (multiple of 16)
    int32_t tail_n;             // ragged-tail elements (< 16 / sizeof element)
    int32_t flags;              // 1: first stage of the item, 2: last stage of the item
};

template <int kConsumerWarps, int kStages>
struct TmaSmem {
    static constexpr size_t kMetaOff = size_t(kStages) * kStageBytes;
    static constexpr size_t kBarOff = kMetaOff + sizeof(StageMeta) * kStages;
    static constexpr size_t kMiscOff = kBarOff + 16 * kStages;          // full[], empty[]
    static constexpr size_t kRedOff = kMiscOff + 4 * 64;                // misc ints
    static constexpr size_t kRowOff = kRedOff + 4 * 6 * kConsumerWarps;  // red[2][3*warps]
    static size_t bytes(int nB) { return kRowOff + 4 * size_t(nB + 1); }
};

template <typename T, bool kGreedy, int kConsumerWarps, int kStages>
__global__ void __launch_bounds__((kConsumerWarps + 1) * 32, TmaCtasPerSm<T>::value)
row_stats_tma_kernel(const StatsParams p) {
    constexpr int kConsumers = kConsumerWarps * 32;
    constexpr int kThreads = kConsumers + 32;
    constexpr int kVecPerThread = (kStageBytes / 16 + kConsumers - 1) / kConsumers;
    using L = TmaSmem<kConsumerWarps, kStages>;
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char* stage_buf = smem;
    StageMeta* meta = reinterpret_cast<StageMeta*>(smem + L::kMetaOff);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* empty = full + kStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff);
    int* scan_scratch = reinterpret_cast<int*>(smem + L::kMiscOff) + 8;
    float* red = reinterpret_cast<float*>(smem + L::kRedOff);
    int* row_start = reinterpret_cast<int*>(smem + L::kRowOff);

    const int tid = threadIdx.x;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, kConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    build_row_prefix<kThreads>(p, row_start, scan_scratch);  // ends with __syncthreads
    const int64_t total_items = (int64_t)row_start[p.nB] * p.C;

    if (tid >= kConsumers) {
        // ----------------------------- producer warp -----------------------------
        const int lane = tid - kConsumers;
        int slot = 0;               // ring position of the next stage
        uint32_t phase = 0;         // parity of the ring round in progress
        bool wrapped = false;       // the ring has been filled once
        uint32_t last_phase[kStages];
#pragma unroll
        for (int s = 0; s < kStages; ++s) last_phase[s] = 0xffffffffu;
        bool stop = false;
        for (int64_t item = blockIdx.x; item < total_items && !stop; item += gridDim.x) {
            const ItemDesc d = decode_item<T>(p, row_start, item);
            const int64_t bytes_all = int64_t(d.e1 - d.e0) * Logit<T>::kSize;
            const int64_t tma_bytes = bytes_all & ~int64_t(15);
            const int tail_n = static_cast<int>((bytes_all - tma_bytes) / Logit<T>::kSize);
            const int nsub = tma_bytes == 0 ? 1 : static_cast<int>((tma_bytes + kStageBytes - 1) / kStageBytes);
            const unsigned char* src0 = d.row + int64_t(d.e0) * Logit<T>::kSize;
            for (int sub = 0; sub < nsub; ++sub) {
                if (lane == 0) {
                    bool ok = true;
                    if (wrapped) ok = mbar_wait_bounded(empty + slot, phase ^ 1u, p.timeout_ns);
                    if (!ok) *abort_flag = 1;
                    if (*abort_flag) {
                        stop = true;
                    } else if (sub == 0 && d.partial_idx == p.lost_copy_partial) {
                        // injected fault: the stage is neither armed nor copied, so
                        // the consumers' bounded wait on it runs out; last_phase[slot]
                        // keeps the previous (completed) phase for the drain below
                    } else {
                        const int64_t off = int64_t(sub) * kStageBytes;
                        const int64_t left = tma_bytes - off;
                        const int n = static_cast<int>(left < kStageBytes ? left : int64_t(kStageBytes));
                        StageMeta m;
                        m.tail = tail_n ? src0 + tma_bytes : nullptr;
                        m.partial_idx = d.partial_idx;
                        m.elem0 = d.e0 + static_cast<int>(off / Logit<T>::kSize);
                        m.n_bytes = n > 0 ? n : 0;
                        m.tail_n = tail_n;
                        m.flags = (sub == 0 ? 1 : 0) | (sub == nsub - 1 ? 2 : 0);
                        meta[slot] = m;
                        last_phase[slot] = phase;
                        if (n > 0) {
                            mbar_arrive_expect_tx(full + slot, static_cast<uint32_t>(n));
                            bulk_copy_g2s(stage_buf + size_t(slot) * kStageBytes, src0 + off,
                                          static_cast<uint32_t>(n), full + slot);
                        } else {
                            mbar_arrive(full + slot);
                        }
                    }
                }
                stop = __shfl_sync(0xffffffffu, stop, 0);
                if (stop) break;
                if (++slot == kStages) {
                    slot = 0;
                    phase ^= 1u;
                    wrapped = true;
                }
            }
        }
        // Wait until the consumers are done, then (only after a timeout) make
        // sure no copy issued by this CTA is still in flight before exiting.
        named_barrier_sync(2, kThreads);
        if (lane == 0 && *abort_flag) {
            for (int s = 0; s < kStages; ++s)
                if (last_phase[s] != 0xffffffffu) (void)mbar_wait_bounded(full + s, last_phase[s], p.timeout_ns);
        }
        return;
    }

    // ------------------------------- consumer warps -------------------------------
    // Every consumer thread runs the reduction of every item exactly once, so
    // the named barrier 1 stays in step even after a timeout; wait outcomes are
    // made warp-uniform with __all_sync before anyone acts on them.
    Acc<kGreedy> acc;
    int slot = 0;          // ring position of the next stage
    uint32_t phase = 0;    // parity of the ring round in progress
    int parity_item = 0;
    for (int64_t item = blockIdx.x; item < total_items; item += gridDim.x, parity_item ^= 1) {
        acc.reset();
        bool failed = __any_sync(0xffffffffu, *abort_flag != 0);  // warp-uniform
        int64_t partial_idx = -1;
        while (!failed) {
            bool ok = !*abort_flag && mbar_wait_bounded(full + slot, phase, p.timeout_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) {
                *abort_flag = 1;
                failed = true;
                break;
            }
            const StageMeta m = meta[slot];
            partial_idx = m.partial_idx;
            const unsigned char* buf = stage_buf + size_t(slot) * kStageBytes;
            const int nvec = m.n_bytes >> 4;
            if constexpr (kGreedy) {
#pragma unroll
                for (int k = 0; k < kVecPerThread; ++k) {
                    const int v = tid + k * kConsumers;
                    if (v < nvec) fold_vector<T, true>(acc, ld_shared_v4(buf + 16 * v), m.elem0 + v * Logit<T>::kPerVec, 0.f);
                }
            } else {
                uint4 vv[kVecPerThread];
                if (nvec == kVecPerThread * kConsumers) {  // full stage: no guards
#pragma unroll
                    for (int k = 0; k < kVecPerThread; ++k) vv[k] = ld_shared_v4(buf + 16 * (tid + k * kConsumers));
                    fold_vectors<T, kVecPerThread>(acc, vv, p.scale);
                } else {
#pragma unroll
                    for (int k = 0; k < kVecPerThread; ++k) {
                        const int v = tid + k * kConsumers;
                        vv[k] = v < nvec ? ld_shared_v4(buf + 16 * v) : make_uint4(0, 0, 0, 0);
                    }
                    const int nv = nvec > tid ? (nvec - tid + kConsumers - 1) / kConsumers : 0;
                    fold_vectors_count<T, kVecPerThread>(acc, vv, nv, p.scale);
                }
            }
            __syncwarp();
            if ((tid & 31) == 0) mbar_arrive(empty + slot);
            if (++slot == kStages) {
                slot = 0;
                phase ^= 1u;
            }
            if (m.flags & 2) {
                if (m.tail && tid < m.tail_n) {
                    const float z = Logit<T>::load(m.tail, tid);
                    const int idx = m.elem0 + (m.n_bytes / Logit<T>::kSize) + tid;
                    if constexpr (kGreedy) acc.take(z, idx);
                    else acc.fold1(z * p.scale);
                }
                break;
            }
        }
        if (failed) partial_idx = decode_item<T>(p, row_start, item).partial_idx;
        reduce_and_store<kGreedy, kConsumerWarps>(acc, red + parity_item * 3 * kConsumerWarps, 1, kConsumers,
                                                 p.partials + partial_idx, failed);
    }
    named_barrier_sync(2, kThreads);
    // this CTA is done: the dependent draw kernel may start its prologue here
    if (tid == 0) asm volatile("griddepcontrol.launch_dependents;");
}

// ============================================================================
// Load-instruction variant (16-byte vectors or single elements).

template <typename T, bool kGreedy, bool kVec, int kThreads>
__global__ void __launch_bounds__(kThreads)
row_stats_ldg_kernel(const StatsParams p) {
    constexpr int kWarps = kThreads / 32;
    constexpr int kUnroll = SV_LDG_UNROLL;
    extern __shared__ __align__(16) int ldg_row_start[];
    __shared__ int scan_scratch[32];
    __shared__ float red[2][3 * kWarps];
    build_row_prefix<kThreads>(p, ldg_row_start, scan_scratch);
    const int64_t total_items = (int64_t)ldg_row_start[p.nB] * p.C;
    const int tid = threadIdx.x;
    int parity_item = 0;
    for (int64_t item = blockIdx.x; item < total_items; item += gridDim.x, parity_item ^= 1) {
        const ItemDesc d = decode_item<T>(p, ldg_row_start, item);
        Acc<kGreedy> acc;
        acc.reset();
        if constexpr (kVec) {
            // Software-pipelined: the next batch of kUnroll vectors is in
            // flight while the current one is folded.
            const int64_t bytes_all = int64_t(d.e1 - d.e0) * Logit<T>::kSize;
            const int nvec = static_cast<int>(bytes_all >> 4);
            const unsigned char* src = d.row + int64_t(d.e0) * Logit<T>::kSize;
            constexpr int kStride = kThreads * kUnroll;
            uint4 cur[kUnroll];
#pragma unroll
            for (int k = 0; k < kUnroll; ++k) {
                const int v = tid + k * kThreads;
                cur[k] = v < nvec ? ld_global_stream_v4(src + 16 * int64_t(v)) : neg_inf_vector<T>();
            }
            for (int v0 = tid; v0 < nvec; v0 += kStride) {
                uint4 nxt[kUnroll];
#pragma unroll
                for (int k = 0; k < kUnroll; ++k) {
                    const int v = v0 + kStride + k * kThreads;
                    nxt[k] = v < nvec ? ld_global_stream_v4(src + 16 * int64_t(v)) : neg_inf_vector<T>();
                }
                if constexpr (kGreedy) {
#pragma unroll
                    for (int k = 0; k < kUnroll; ++k) {
                        const int v = v0 + k * kThreads;
                        if (v < nvec) fold_vector<T, true>(acc, cur[k], d.e0 + v * Logit<T>::kPerVec, 0.f);
                    }
                } else {
                    const int nv = (nvec - v0 + kThreads - 1) / kThreads;
                    fold_vectors_count<T, kUnroll>(acc, cur, nv, p.scale);
                }
#pragma unroll
                for (int k = 0; k < kUnroll; ++k) cur[k] = nxt[k];
            }
            const int tail0 = d.e0 + nvec * Logit<T>::kPerVec;
            if (tail0 + tid < d.e1) {
                const float z = Logit<T>::load(d.row, tail0 + tid);
                if constexpr (kGreedy) acc.take(z, tail0 + tid);
                else acc.fold1(z * p.scale);
            }
        } else {
            for (int e = d.e0 + tid; e < d.e1; e += kThreads) {
                const float z = Logit<T>::load(d.row, e);
                if constexpr (kGreedy) acc.take(z, e);
                else acc.fold1(z * p.scale);
            }
        }
        reduce_and_store<kGreedy, kWarps>(acc, red[parity_item], 1, kThreads, p.partials + d.partial_idx, false);
    }
    __syncthreads();
    if (tid == 0) asm volatile("griddepcontrol.launch_dependents;");
}

}  // namespace sv
