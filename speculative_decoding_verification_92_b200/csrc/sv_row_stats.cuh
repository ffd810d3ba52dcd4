// sv_row_stats.cuh -- K1, the row-statistics pass.
//
// Every row a request uses (target rows 0..L_b, draft rows 0..L_b-1) is cut
// into P pieces of PE elements (16 KiB each, the last one ragged).  The
// pieces of all used rows, in request order, form one list of N pieces.
// Bulk-copy variant: CTA x of a grid of G first takes the contiguous range
// [x*S, (x+1)*S) with S = floor(N * static_pct / 100 / G), then pieces
// G*S, G*S + 1, ... one at a time from a shared counter, so CTAs that stream
// faster (SMs do not all get the same share of HBM bandwidth) take more
// pieces and all CTAs finish within about one piece of each other.  The
// element-load variant takes the contiguous range [x*N/G, (x+1)*N/G).  Each
// piece is reduced to one partial:
//   sampling: (m, s) with m = max_v t_v, s = sum_v 2^(t_v - m), t_v = z_v * log2(e)/T
//             (the temperature softmax statistics of step 1 of the rule,
//             "AI 开始抄自己的作业——而且抄得理直气壮", section "⚡ 投机解码：让草稿先跑，考官殿后")
//   greedy:   (max z_v, lowest index attaining it)
// written to partials[(b * (2*k_max+1) + slot) * P + piece], slot = i for
// target row i and k_max+1+i for draft row i.  The scan kernel merges the P
// partials of a row; the draw kernel uses the pieces as its units of work.
//
// Variants:
//   row_stats_tma_kernel  one producer warp streams the pieces through a ring
//                         of shared-memory stages (one piece per stage) with
//                         1-D cp.async.bulk copies completing on mbarriers;
//                         consumer warps fold the stage and leave one
//                         (m, s) per thread in shared memory, which the
//                         producer warp merges into the piece's partial before
//                         it refills the stage.  Needs 16-byte aligned rows.
//                         Waits are bounded; after a timeout the CTA writes
//                         NaN partials for the rest of its range.
//   row_stats_ldg_kernel  the same piece ranges with 16-byte vector loads
//                         (aligned rows) or element loads (any alignment) and
//                         a block reduction per piece.
#pragma once

#include "sv_common.cuh"

// Ring geometry of the bulk-copy variant (compile-time; defaults tuned on B200;
// the stage size is SV_STAGE_BYTES of sv_common.cuh).
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

// One piece = one ring stage of the bulk-copy variant.
constexpr int kStageBytes = kPieceBytes;

struct StatsParams {
    const unsigned char* target;  // [B][k_max+1][row_stride]
    const unsigned char* draft;   // [B][k_max][row_stride] or null
    const int32_t* lens;          // [B] or null (all k_max)
    float2* partials;             // [B][2*k_max+1][P]
    int32_t* dyn_ticket;          // this launch's counter of handed-out pieces (zero at launch; the
                                  // bulk-copy variant only)
    int32_t b0;                   // first request handled by this launch
    int32_t nB;                   // requests handled by this launch (<= kMaxRequestsPerLaunch)
    int32_t k_max;
    int32_t V;
    int64_t row_stride;           // elements
    int32_t P;                    // pieces per row
    int32_t PE;                   // elements per piece (kPieceBytes / element size)
    float scale;                  // log2(e) / T
    int32_t use_draft;            // draft rows are part of the work
    uint64_t timeout_ns;          // bound on each barrier wait (TMA variant)
    int64_t lost_copy_partial;    // test fault injection: this piece is never copied; -1 = off
    int32_t static_pct;           // bulk-copy variant: percent of the pieces split statically
};

struct ItemDesc {
    const unsigned char* row;     // first byte of the row
    int64_t partial_idx;
    int32_t e0, e1;               // element range of the piece
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

// Piece `item` of the list: row g = item / P of the used rows, piece item % P.
template <typename T>
__device__ __forceinline__ ItemDesc decode_item(const StatsParams& p, const int* row_start, int64_t item) {
    const int64_t g = item / p.P;
    const int c = static_cast<int>(item - g * p.P);
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
    d.partial_idx = ((int64_t)b * (2 * p.k_max + 1) + slot) * p.P + c;
    d.e0 = c * p.PE;
    d.e1 = min(p.V, d.e0 + p.PE);
    return d;
}

// This CTA's contiguous range [*lo, *hi) of the piece list.
__device__ __forceinline__ void piece_range(int64_t total, int64_t* lo, int64_t* hi) {
    *lo = total * blockIdx.x / gridDim.x;
    *hi = total * (blockIdx.x + 1) / gridDim.x;
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
    __device__ __forceinline__ float2 as_float2() const { return make_float2(ms.m, ms.s); }
};

template <> struct Acc<true> {
    VI vi;
    __device__ __forceinline__ void reset() { vi = VI{-INFINITY, 0x7fffffff}; }
    __device__ __forceinline__ void take(float z, int idx) {
        if (z > vi.v || (z == vi.v && idx < vi.i)) vi = VI{z, idx};
    }
    __device__ __forceinline__ float2 as_float2() const { return make_float2(vi.v, __int_as_float(vi.i)); }
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
    if constexpr (Logit<T>::kSize == 2) {
        // Packed pairs: word i's two elements share one FFMA2 and one FADD2
        // (into {s0, s1} for even i, {s2, s3} for odd i), each lane rounded
        // as the scalar FFMA and FADD would be.
        const uint64_t sc2 = f2_pack(scale, scale), nm2 = f2_pack(negM, negM);
        uint64_t acc2[2] = {0ull, 0ull};
#pragma unroll
        for (int i = 0; i < NW; ++i) {
            float xl, xh;
            f2_unpack(f2_fma(bf16x2_to_f2(w[i]), sc2, nm2), xl, xh);
            acc2[i & 1] = f2_add(acc2[i & 1], f2_pack(ex2_approx(xl), ex2_approx(xh)));
        }
        f2_unpack(acc2[0], s[0], s[1]);
        f2_unpack(acc2[1], s[2], s[3]);
    } else {
#pragma unroll
        for (int i = 0; i < NW; ++i) s[i & 3] += ex2_approx(fmaf(__uint_as_float(w[i]), scale, negM));
    }
    acc.ms = MS{M, fmaf(acc.ms.s, ex2_approx(acc.ms.m - M), (s[0] + s[1]) + (s[2] + s[3]))};
}

// Fold only the first `nv` (0 <= nv <= K) of K vectors: one fold with a
// compile-time count per possible nv, so no ex2 is spent on absent elements
// (the partial stage at the end of each row).
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

// Merge 32 x kPer per-thread partials (one warp, lane l holding parts[l + 32 k])
// into one; lane 0 gets the result.  Sampling: max first, then every sum
// rescaled once; greedy: larger value, then lower index.
template <bool kGreedy, int kPer>
__device__ __forceinline__ float2 warp_merge_parts(const float2 (&v)[kPer]) {
    if constexpr (kGreedy) {
        VI best{v[0].x, __float_as_int(v[0].y)};
#pragma unroll
        for (int k = 1; k < kPer; ++k) best = vi_better(best, VI{v[k].x, __float_as_int(v[k].y)});
        best = warp_merge_vi(best);
        return make_float2(best.v, __int_as_float(best.i));
    } else {
        float m = v[0].x;
#pragma unroll
        for (int k = 1; k < kPer; ++k) m = fmaxf(m, v[k].x);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float s = 0.f;
        if (m != -INFINITY) {
#pragma unroll
            for (int k = 0; k < kPer; ++k)
                if (v[k].x != -INFINITY) s = fmaf(v[k].y, ex2_approx(v[k].x - m), s);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        return m == -INFINITY ? make_float2(-INFINITY, 0.f) : make_float2(m, s);
    }
}

// Block reduction of the reducing threads' accumulators for the element-load
// variant; thread 0 writes the partial.  `red` holds 2 * kWarps floats for
// this item (double-buffered by the caller); `bar_id`/`nthreads` name the
// barrier of the reducing threads.
template <bool kGreedy, int kWarps>
__device__ __forceinline__ void reduce_and_store(Acc<kGreedy>& acc, float* red, int bar_id, int nthreads,
                                                 float2* out) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
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
        red[2 * warp] = a;
        red[2 * warp + 1] = b;
    }
    named_barrier_sync(bar_id, nthreads);
    if (threadIdx.x == 0) {
        float2 r;
        if constexpr (kGreedy) {
            VI t{red[0], __float_as_int(red[1])};
            for (int w = 1; w < kWarps; ++w) t = vi_better(t, VI{red[2 * w], __float_as_int(red[2 * w + 1])});
            r = make_float2(t.v, __int_as_float(t.i));
        } else {
            MS t{red[0], red[1]};
            for (int w = 1; w < kWarps; ++w) t = ms_merge(t, MS{red[2 * w], red[2 * w + 1]});
            r = make_float2(t.m, t.s);
        }
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

template <typename T>
struct TmaCtasPerSm {
    static constexpr int value = Logit<T>::kSize == 2 ? SV_TMA_CTAS_PER_SM_BF16 : SV_TMA_CTAS_PER_SM_F32;
};

struct StageMeta {
    const unsigned char* tail;  // first ragged-tail element (row's last piece), or null
    int64_t partial_idx;
    int32_t elem0;              // row index of the stage's first element
    int32_t n_bytes;            // bytes delivered by the bulk copy (multiple of 16); -1: no more pieces
    int32_t tail_n;             // ragged-tail elements (< 16 / sizeof element)
    int32_t pad;
};

template <int kConsumerWarps, int kStages>
struct TmaSmem {
    static constexpr size_t kMetaOff = size_t(kStages) * kStageBytes;
    static constexpr size_t kBarOff = kMetaOff + sizeof(StageMeta) * kStages;
    static constexpr size_t kMiscOff = kBarOff + 16 * kStages;                         // full[], empty[]
    static constexpr size_t kPartOff = kMiscOff + 4 * 64;                              // misc ints
    static constexpr size_t kRowOff = kPartOff + 8 * size_t(2 * kStages) * kConsumerWarps * 32;  // part[round&1][stage][thread]
    static size_t bytes(int nB) { return kRowOff + 4 * size_t(nB + 1); }
};

// Bounded wait that also gives up as soon as *abort_flag is set.
__device__ __forceinline__ bool mbar_wait_or_abort(uint64_t* bar, uint32_t parity, uint64_t timeout_ns,
                                                   const volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        if (mbar_try_wait_suspend(bar, parity, 20000u)) return true;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > timeout_ns) return false;
    }
}

template <typename T, bool kGreedy, int kConsumerWarps, int kStages>
__global__ void __launch_bounds__((kConsumerWarps + 1) * 32, TmaCtasPerSm<T>::value)
row_stats_tma_kernel(const StatsParams p) {
    constexpr int kConsumers = kConsumerWarps * 32;
    constexpr int kThreads = kConsumers + 32;
    constexpr int kVecPerThread = kStageBytes / 16 / kConsumers;
    static_assert(kStageBytes % (16 * kConsumers) == 0, "a stage must split evenly over the consumers");
    constexpr int kPartsPerLane = kConsumers / 32;
    using L = TmaSmem<kConsumerWarps, kStages>;
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char* stage_buf = smem;
    StageMeta* meta = reinterpret_cast<StageMeta*>(smem + L::kMetaOff);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* empty = full + kStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff);
    int* scan_scratch = reinterpret_cast<int*>(smem + L::kMiscOff) + 8;
    float2* part = reinterpret_cast<float2*>(smem + L::kPartOff);   // [2][kStages][kConsumers]
    int* row_start = reinterpret_cast<int*>(smem + L::kRowOff);

    const int tid = threadIdx.x;
    // The scan kernel may be launched now: its CTAs take the places of this
    // grid's CTAs as they exit (this grid is one resident wave) and run their
    // input-only prologue, then wait for this grid to complete.
    if (tid == 0) asm volatile("griddepcontrol.launch_dependents;");
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, kConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    build_row_prefix<kThreads>(p, row_start, scan_scratch);  // ends with __syncthreads
    const int64_t total = (int64_t)row_start[p.nB] * p.P;

    if (tid >= kConsumers) {
        // ----------------------------- producer warp -----------------------------
        // The i-th item issued goes to stage i % kStages in round i / kStages:
        // the copy's arrival is that round's completion of full[stage], the
        // consumers' release of it the same round's completion of empty[stage]
        // (parity round & 1).  After the last piece the producer posts an end
        // marker (no copy) that stops the consumers.  While the ring is full
        // it waits for the oldest piece's release, refills that stage at once
        // and only then merges the consumers' per-thread partials of the
        // released piece (they live in part[round & 1][stage], so the
        // consumers of the next round never overwrite them before the merge).
        const int lane = tid - kConsumers;
        const uint64_t stream_policy = l2_evict_first_policy();  // logits are read once
        const int64_t S = total * p.static_pct / 100 / gridDim.x;  // static pieces per CTA
        const int64_t dyn_base = S * gridDim.x;
        const int64_t dyn_n = total - dyn_base;
        int64_t stat_next = S * blockIdx.x;
        const int64_t stat_end = stat_next + S;
        // lane 0: the next dynamic ticket, fetched one piece ahead (-1: none yet)
        int64_t ticket = -1;
        bool tickets_done = false;
        bool ctrl_ready = false;
        auto take_ticket = [&]() {
            // the ticket counter is zeroed by the grid this one is a
            // programmatic dependent of: wait for it before the first ticket
            if (!ctrl_ready) {
                asm volatile("griddepcontrol.wait;" ::: "memory");
                ctrl_ready = true;
            }
            ticket = dyn_n > 0 ? int64_t(atomicAdd(p.dyn_ticket, 1)) : dyn_n;
        };
        // lane 0: the next piece to issue, or -1 when there is none
        auto next_piece = [&]() -> int64_t {
            if (stat_next < stat_end) {
                const int64_t pc = stat_next++;
                if (stat_next == stat_end && !tickets_done && ticket < 0) take_ticket();
                return pc;
            }
            if (tickets_done) return -1;
            if (ticket < 0) take_ticket();
            if (ticket >= dyn_n) {
                tickets_done = true;
                return -1;
            }
            const int64_t pc = dyn_base + ticket;
            take_ticket();
            return pc;
        };
        int64_t cur = lane == 0 ? next_piece() : -1;
        int issued = 0, merged = 0;
        bool end_sent = false, stop = false;
        int last_round[kStages];    // round of the last copy issued into each stage, -1 = none
#pragma unroll
        for (int s = 0; s < kStages; ++s) last_round[s] = -1;
        // lane 0: issue the next item (piece `cur`, or the end marker) into its stage
        auto issue_next = [&]() {
            const int slot = issued % kStages;
            const int round = issued / kStages;
            if (lane == 0) {
                StageMeta m;
                if (cur >= 0) {
                    const ItemDesc d = decode_item<T>(p, row_start, cur);
                    const int64_t bytes_all = int64_t(d.e1 - d.e0) * Logit<T>::kSize;
                    const int n = static_cast<int>(bytes_all & ~int64_t(15));
                    const int tail_n = static_cast<int>((bytes_all - n) / Logit<T>::kSize);
                    const unsigned char* src = d.row + int64_t(d.e0) * Logit<T>::kSize;
                    m.tail = tail_n ? src + n : nullptr;
                    m.partial_idx = d.partial_idx;
                    m.elem0 = d.e0;
                    m.n_bytes = n;
                    m.tail_n = tail_n;
                    m.pad = 0;
                    meta[slot] = m;
                    if (d.partial_idx == p.lost_copy_partial) {
                        // injected fault: the stage is neither armed nor copied, so
                        // the consumers' bounded wait on it runs out
                    } else {
#pragma unroll
                        for (int s = 0; s < kStages; ++s)
                            if (s == slot) last_round[s] = round;
                        if (n > 0) {
                            mbar_arrive_expect_tx(full + slot, static_cast<uint32_t>(n));
                            bulk_copy_g2s_hint(stage_buf + size_t(slot) * kStageBytes, src, static_cast<uint32_t>(n),
                                               full + slot, stream_policy);
                        } else {
                            mbar_arrive(full + slot);
                        }
                    }
                    cur = next_piece();
                } else {
                    m.tail = nullptr;
                    m.partial_idx = -1;
                    m.elem0 = 0;
                    m.n_bytes = -1;
                    m.tail_n = 0;
                    m.pad = 0;
                    meta[slot] = m;
                    mbar_arrive(full + slot);
                }
            }
        };
        for (;;) {
            if (!end_sent && issued - merged < kStages) {
                const bool has_piece = __shfl_sync(0xffffffffu, cur >= 0, 0);
                issue_next();
                if (!has_piece) end_sent = true;
                ++issued;
                continue;
            }
            const int n_real = issued - (end_sent ? 1 : 0);
            if (merged == n_real) break;
            const int slot = merged % kStages;
            const int round = merged / kStages;
            bool ok = true;
            if (lane == 0) ok = mbar_wait_or_abort(empty + slot, static_cast<uint32_t>(round & 1), p.timeout_ns,
                                                   abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                if (lane == 0) *abort_flag = 1;
                stop = true;
                break;
            }
            // the piece's partial index, read before the refill rewrites meta[slot]
            const int64_t pidx = meta[slot].partial_idx;
            __syncwarp();
            ++merged;
            if (!end_sent && issued - merged < kStages) {
                const bool has_piece = __shfl_sync(0xffffffffu, cur >= 0, 0);
                issue_next();
                if (!has_piece) end_sent = true;
                ++issued;
            }
            float2 v[kPartsPerLane];
            const float2* ps = part + ((round & 1) * kStages + slot) * kConsumers;
#pragma unroll
            for (int i = 0; i < kPartsPerLane; ++i) v[i] = ps[lane + 32 * i];
            const float2 r = warp_merge_parts<kGreedy, kPartsPerLane>(v);
            if (lane == 0) p.partials[pidx] = r;
        }
        if (stop && lane == 0) {
            // every piece this CTA took and did not finish gets a NaN partial
            // (the scan kernel reports its request with out_accept_len = -2):
            // the pieces in the ring, the rest of the static range, the piece
            // about to be issued and the ticket fetched ahead
            const float nan = __int_as_float(0x7fc00000);
            const float2 bad = make_float2(nan, nan);
            const int n_real = issued - (end_sent ? 1 : 0);
            for (int i = merged; i < n_real; ++i) p.partials[meta[i % kStages].partial_idx] = bad;
            for (int64_t it = stat_next; it < stat_end; ++it)
                p.partials[decode_item<T>(p, row_start, it).partial_idx] = bad;
            if (cur >= 0) p.partials[decode_item<T>(p, row_start, cur).partial_idx] = bad;
            if (!tickets_done && ticket >= 0 && ticket < dyn_n)
                p.partials[decode_item<T>(p, row_start, dyn_base + ticket).partial_idx] = bad;
        }
        // This grid completes only after the grid that zeroed the control
        // words (the kernels after it rely on that); a no-op once waited for.
        if (lane == 0 && !ctrl_ready) asm volatile("griddepcontrol.wait;" ::: "memory");
        // Wait until the consumers are done, then make sure no copy issued by
        // this CTA is still in flight before exiting (after a timeout).
        named_barrier_sync(2, kThreads);
        if (lane == 0 && stop) {
#pragma unroll
            for (int s = 0; s < kStages; ++s)
                if (last_round[s] >= 0)
                    (void)mbar_wait_bounded(full + s, static_cast<uint32_t>(last_round[s] & 1), p.timeout_ns);
        }
        return;
    }

    // ------------------------------- consumer warps -------------------------------
    // Item i: wait for its stage, stop at the end marker, else fold the piece
    // (plus the row's ragged tail on the row's last piece), leave this
    // thread's partial in part[round & 1][stage][tid] and release the stage.
    // A failed wait is made warp-uniform; the warp then leaves the loop (the
    // producer writes the NaN partials).
    const int lane = tid & 31;
    for (int i = 0;; ++i) {
        const int slot = i % kStages;
        const int round = i / kStages;
        bool ok = !*abort_flag && mbar_wait_or_abort(full + slot, static_cast<uint32_t>(round & 1), p.timeout_ns,
                                                     abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
            if (lane == 0) *abort_flag = 1;
            break;
        }
        const StageMeta m = meta[slot];
        if (m.n_bytes < 0) break;  // end marker: no more pieces
        const unsigned char* buf = stage_buf + size_t(slot) * kStageBytes;
        const int nvec = m.n_bytes >> 4;
        Acc<kGreedy> acc;
        acc.reset();
        if constexpr (kGreedy) {
#pragma unroll
            for (int kk = 0; kk < kVecPerThread; ++kk) {
                const int v = tid + kk * kConsumers;
                if (v < nvec)
                    fold_vector<T, true>(acc, ld_shared_v4(buf + 16 * v), m.elem0 + v * Logit<T>::kPerVec, 0.f);
            }
        } else {
            uint4 vv[kVecPerThread];
            if (nvec == kVecPerThread * kConsumers) {  // full stage: no guards
#pragma unroll
                for (int kk = 0; kk < kVecPerThread; ++kk) vv[kk] = ld_shared_v4(buf + 16 * (tid + kk * kConsumers));
                fold_vectors<T, kVecPerThread>(acc, vv, p.scale);
            } else {
#pragma unroll
                for (int kk = 0; kk < kVecPerThread; ++kk) {
                    const int v = tid + kk * kConsumers;
                    vv[kk] = v < nvec ? ld_shared_v4(buf + 16 * v) : make_uint4(0, 0, 0, 0);
                }
                const int nv = nvec > tid ? (nvec - tid + kConsumers - 1) / kConsumers : 0;
                fold_vectors_count<T, kVecPerThread>(acc, vv, nv, p.scale);
            }
        }
        if (m.tail && tid < m.tail_n) {
            const float z = Logit<T>::load(m.tail, tid);
            const int idx = m.elem0 + (m.n_bytes / Logit<T>::kSize) + tid;
            if constexpr (kGreedy) acc.take(z, idx);
            else acc.fold1(z * p.scale);
        }
        part[((round & 1) * kStages + slot) * kConsumers + tid] = acc.as_float2();
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + slot);  // release: the partials above are visible to the producer
    }
    named_barrier_sync(2, kThreads);
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
    __shared__ float red[2][2 * kWarps];
    if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;");  // see the bulk-copy variant
    // this grid completes only after the grid that zeroed the control words
    if (threadIdx.x == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
    build_row_prefix<kThreads>(p, ldg_row_start, scan_scratch);
    int64_t lo, hi;
    piece_range((int64_t)ldg_row_start[p.nB] * p.P, &lo, &hi);
    const int tid = threadIdx.x;
    int parity_item = 0;
    for (int64_t item = lo; item < hi; ++item, parity_item ^= 1) {
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
        reduce_and_store<kGreedy, kWarps>(acc, red[parity_item], 1, kThreads, p.partials + d.partial_idx);
    }
}

}  // namespace sv
