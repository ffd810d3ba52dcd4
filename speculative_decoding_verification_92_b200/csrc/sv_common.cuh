// sv_common.cuh -- device helpers shared by the verification kernels:
// inline-PTX wrappers (mbarrier, 1-D bulk copy, ex2, global timer), logit
// dtype traits and (m, s) / (value, index) reduction helpers.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace sv {

// A row is cut into pieces of this many bytes: one bulk-copy stage of the
// row-statistics kernel, and the unit of work of the draw kernel.
#ifndef SV_STAGE_BYTES
#define SV_STAGE_BYTES 16384
#endif

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kPieceBytes = SV_STAGE_BYTES;
constexpr int kMaxRequestsPerLaunch = 4096;  // K1 keeps a per-CTA row prefix of this many requests

// ---------------------------------------------------------------------------
// Logit storage types.  bf16 is kept as raw 16-bit patterns; widening to fp32
// is a shift (exact).

struct bf16_bits { uint16_t v; };

template <typename T> struct Logit;

template <> struct Logit<float> {
    static constexpr int kSize = 4;
    static constexpr int kPerVec = 4;   // per 16-byte vector
    __device__ __forceinline__ static float load(const void* base, int64_t i) {
        return __ldg(reinterpret_cast<const float*>(base) + i);
    }
    __device__ __forceinline__ static void unpack(const uint4& w, float (&f)[4]) {
        f[0] = __uint_as_float(w.x); f[1] = __uint_as_float(w.y);
        f[2] = __uint_as_float(w.z); f[3] = __uint_as_float(w.w);
    }
};

template <> struct Logit<bf16_bits> {
    static constexpr int kSize = 2;
    static constexpr int kPerVec = 8;
    __device__ __forceinline__ static float load(const void* base, int64_t i) {
        const unsigned short h = __ldg(reinterpret_cast<const unsigned short*>(base) + i);
        return __uint_as_float(static_cast<uint32_t>(h) << 16);
    }
    __device__ __forceinline__ static void unpack(const uint4& w, float (&f)[8]) {
        f[0] = __uint_as_float(w.x << 16); f[1] = __uint_as_float(w.x & 0xffff0000u);
        f[2] = __uint_as_float(w.y << 16); f[3] = __uint_as_float(w.y & 0xffff0000u);
        f[4] = __uint_as_float(w.z << 16); f[5] = __uint_as_float(w.z & 0xffff0000u);
        f[6] = __uint_as_float(w.w << 16); f[7] = __uint_as_float(w.w & 0xffff0000u);
    }
};

// ---------------------------------------------------------------------------
// Small PTX wrappers.

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed bf16x2 maximum of two words (two elements per instruction).
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Packed FP32 pairs for the sm_100 f32x2 instructions: one issue slot does
// two round-to-nearest fp32 operations, each lane rounded exactly as the
// scalar instruction would.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// The bf16 pair of a word, widened to fp32 (low element in the low lane).
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w) { return f2_pack(bf16_lo(w), bf16_hi(w)); }

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait that may suspend the thread for up to hint_ns (it resumes as soon
// as the phase completes), so waiting threads do not spin on the issue slots.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete, giving up after
// timeout_ns of global time.  Returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        if (mbar_try_wait_suspend(bar, parity, 20000u)) return true;
        if (global_timer_ns() - t0 > timeout_ns) return false;
    }
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`
// (no multicast).  dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// L2 policy for data read once: its lines are the first to be evicted, so a
// stream of logits does not push out what later kernels read again (their
// code, the row-statistics partials, the draw queue).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// bulk_copy_g2s with an L2 cache policy (l2_evict_first_policy).
__device__ __forceinline__ void bulk_copy_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                                   uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// 16-byte asynchronous copy global -> shared memory (L2 only), grouped with
// cp_async_commit and awaited with cp_async_wait<N> (at most N newest groups
// still pending).  Both addresses must be 16-byte aligned.
__device__ __forceinline__ void cp_async_16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(const void* p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

// Streaming 16-byte global load (read once: no L1 allocation).
__device__ __forceinline__ uint4 ld_global_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ---------------------------------------------------------------------------
// Online log-sum-exp partials in the log2 domain: a set of values t_v is
// summarised by (m, s) with m = max t_v and s = sum 2^(t_v - m).

struct MS { float m; float s; };

__device__ __forceinline__ MS ms_merge(MS a, MS b) {
    const float m = fmaxf(a.m, b.m);
    if (m == -INFINITY) return MS{-INFINITY, 0.f};
    return MS{m, a.s * ex2_approx(a.m - m) + b.s * ex2_approx(b.m - m)};
}

// Warp reduction of (m, s) pairs with one ex2 per lane: the warp maximum
// first, then every lane rescales its own sum to it and the sums are added.
__device__ __forceinline__ MS warp_merge_ms_maxfirst(MS v) {
    float m = v.m;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (m == -INFINITY) return MS{-INFINITY, 0.f};
    float s = v.s * ex2_approx(v.m - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return MS{m, s};
}

__device__ __forceinline__ MS warp_merge_ms(MS v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        MS w{__shfl_xor_sync(0xffffffffu, v.m, o), __shfl_xor_sync(0xffffffffu, v.s, o)};
        v = ms_merge(v, w);
    }
    return v;
}

// Greedy partials: (value, index) with larger value winning and the lower
// index winning among equal values.
struct VI { float v; int i; };

__device__ __forceinline__ VI vi_better(VI a, VI b) {
    if (b.v > a.v || (b.v == a.v && b.i < a.i)) return b;
    return a;
}

__device__ __forceinline__ VI warp_merge_vi(VI a) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        VI b{__shfl_xor_sync(0xffffffffu, a.v, o), __shfl_xor_sync(0xffffffffu, a.i, o)};
        a = vi_better(a, b);
    }
    return a;
}

}  // namespace sv
