// Device helpers of libtreedec: inline-PTX wrappers for the sm_100a
// asynchronous copy engine and mbarriers, element decoding, and the log-depth
// merge of partial softmax states used by both the fused ticket combine and
// the standalone combine kernel.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace td {
namespace dev {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.69314718055994531f;
constexpr float kNegInf = -__builtin_huge_valf();
// A pipeline wait that has not completed after this long is treated as a
// failure: the kernel records it in the error word and winds down.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make barrier initialisation visible to the asynchronous (copy-engine) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase of `bar` with the given parity to complete.  Gives up
// (returns false, sets `code` in *err and raises *abort) after limit_ns
// nanoseconds, or at once when another thread of the CTA has raised *abort.
// With abort == nullptr only the time limit ends the wait.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile int* abort, int* err, int code,
                                                  unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 0u) {
            if (abort != nullptr && *abort) return false;
            if (global_timer_ns() - t0 > limit_ns) {
                atomicOr(err, code);
                if (abort != nullptr) *abort = 1;
                return false;
            }
        }
    }
}

// L2 policy for data read exactly once.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// One contiguous global -> shared copy on the bulk-copy engine, completing
// `bytes` transactions on mbarrier `bar`.  Not multicast.  dst and src must be
// 16-byte aligned and bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                              uint32_t bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(pol)
        : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// 2^x on the special-function unit (PTX ex2.approx; ex2(-inf) = +0).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Weight of a state with running max m (log2 units) under a larger max M.
__device__ __forceinline__ float rescale(float m, float M) {
    return m == kNegInf ? 0.f : ex2(m - M);
}

// ---------------------------------------------------------------- elements

template <typename T>
struct Elem;

template <>
struct Elem<float> {
    static constexpr int kVec = 4;  // elements per 16-byte vector
    __device__ __forceinline__ static void to_f32(const uint4& r, float* f) {
        f[0] = __uint_as_float(r.x);
        f[1] = __uint_as_float(r.y);
        f[2] = __uint_as_float(r.z);
        f[3] = __uint_as_float(r.w);
    }
};

// bfloat16 is the upper half of an fp32: the low element of each 32-bit word
// moves up 16 bits, the high element is masked in place.
template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kVec = 8;
    __device__ __forceinline__ static void pair(uint32_t w, float* f) {
        f[0] = __uint_as_float(w << 16);
        f[1] = __uint_as_float(w & 0xffff0000u);
    }
    __device__ __forceinline__ static void to_f32(const uint4& r, float* f) {
        pair(r.x, f);
        pair(r.y, f + 2);
        pair(r.z, f + 4);
        pair(r.w, f + 6);
    }
};

// FP8 E4M3 storage element (K/V caches only): one byte; the kernels convert
// pairs with cvt.rn.f16x2.e4m3x2 and multiply-add them in half precision.
struct E4M3 {
    unsigned char bits;
};
template <>
struct Elem<E4M3> {
    static constexpr int kVec = 16;  // elements per 16 B
};

// two E4M3 values (low byte -> low half) as an f16x2 word
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(r)
        : "r"(two));
    return r;
}

template <>
struct Elem<__half> {
    static constexpr int kVec = 8;
    __device__ __forceinline__ static void pair(uint32_t w, float* f) {
        __half2 h = *reinterpret_cast<__half2*>(&w);
        float2 x = __half22float2(h);
        f[0] = x.x;
        f[1] = x.y;
    }
    __device__ __forceinline__ static void to_f32(const uint4& r, float* f) {
        pair(r.x, f);
        pair(r.y, f + 2);
        pair(r.z, f + 4);
        pair(r.w, f + 6);
    }
};

__device__ __forceinline__ uint4 lds128(const void* p) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(smem_addr(p)));
    return r;
}

// ------------------------------------------------------- block reductions

// Reductions over `nthreads` threads (a multiple of 32, <= 1024) that meet at
// named barrier `bar`; `scratch` holds >= nthreads/32 floats.  The order of
// the operations is fixed (xor butterfly in each warp, then a pairwise tree
// over the warp results), so the result does not depend on timing.
__device__ __forceinline__ float block_max(float x, int t, int nthreads, float* scratch, int bar) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    const int nw = nthreads >> 5;
    if ((t & 31) == 0) scratch[t >> 5] = x;
    named_bar_sync(bar, nthreads);
    float r = scratch[0];
    for (int w = 1; w < nw; ++w) r = fmaxf(r, scratch[w]);
    named_bar_sync(bar, nthreads);
    return r;
}

__device__ __forceinline__ float block_sum(float x, int t, int nthreads, float* scratch, int bar) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    const int nw = nthreads >> 5;
    if ((t & 31) == 0) scratch[t >> 5] = x;
    named_bar_sync(bar, nthreads);
    // pairwise tree over the warp partials, identical in every thread
    float v[32];
    for (int w = 0; w < nw; ++w) v[w] = scratch[w];
    for (int span = 1; span < nw; span <<= 1)
        for (int w = 0; w + span < nw; w += 2 * span) v[w] += v[w + span];
    named_bar_sync(bar, nthreads);
    return v[0];
}

// ------------------------------------------------------------ tree merge

// Merge n partial states (max m in log2 units, denominator l, numerator
// num[D]) into out[D] = sum_i e^(m_i - M) num_i / sum_i e^(m_i - M) l_i and
// lse = (M + log2 L) ln 2, with M = max_i m_i: the gist's global max,
// renormalisation and sums.  Parts with m = -inf contribute nothing; if all do,
// out = 0 and lse = -inf.
// The parts are taken in chunks: the weights e^(m_i - M) of a chunk are
// computed once into shared memory, then every thread streams its column
// slice of the chunk's records with independent loads.  The sum over parts is
// split across SL thread lanes per column and finished by a pairwise tree, so
// the order of operations is fixed.  `scratch` holds `scratch_floats` >=
// nthreads floats.
template <class Acc>
__device__ void tree_merge(const Acc& acc, int n, int D, int t, int nthreads, float* scratch,
                           int scratch_floats, int bar, float* out_row, float* lse_ptr) {
    float mx = kNegInf;
    for (int i = t; i < n; i += nthreads) mx = fmaxf(mx, acc.m2(i));
    const float M = block_max(mx, t, nthreads, scratch, bar);

    const int DL = D < nthreads ? D : nthreads;  // columns handled at once
    int SL = 1;                                   // part lanes per column
    while (SL * 2 * DL <= nthreads) SL *= 2;
    const int sl = t / DL, dd = t - sl * DL;
    const int passes = (D + DL - 1) / DL;         // 1 or 2 (D <= 2 * nthreads)
    float a0 = 0.f, a1 = 0.f, ls = 0.f;
    if (M != kNegInf) {
        for (int i0 = 0; i0 < n; i0 += scratch_floats) {
            const int cnt = n - i0 < scratch_floats ? n - i0 : scratch_floats;
            for (int i = t; i < cnt; i += nthreads) {
                const float r = rescale(acc.m2(i0 + i), M);
                scratch[i] = r;
                ls += r * acc.l(i0 + i);
            }
            named_bar_sync(bar, nthreads);
            if (sl < SL) {
                const int d0 = dd, d1 = DL + dd;
                const bool two = passes > 1 && d1 < D;
                constexpr int kBatch = 16;  // independent record loads in flight per thread
                int i = sl;
#pragma unroll 1
                for (; i + (kBatch - 1) * SL < cnt; i += kBatch * SL) {
                    float x0[kBatch], x1[kBatch];
#pragma unroll
                    for (int j = 0; j < kBatch; ++j) x0[j] = acc.num(i0 + i + j * SL, d0);
                    if (two) {
#pragma unroll
                        for (int j = 0; j < kBatch; ++j) x1[j] = acc.num(i0 + i + j * SL, d1);
                    }
#pragma unroll
                    for (int j = 0; j < kBatch; ++j) a0 = fmaf(scratch[i + j * SL], x0[j], a0);
                    if (two) {
#pragma unroll
                        for (int j = 0; j < kBatch; ++j) a1 = fmaf(scratch[i + j * SL], x1[j], a1);
                    }
                }
                for (; i < cnt; i += SL) {
                    const float r = scratch[i];
                    if (d0 < D) a0 = fmaf(r, acc.num(i0 + i, d0), a0);
                    if (two) a1 = fmaf(r, acc.num(i0 + i, d1), a1);
                }
            }
            named_bar_sync(bar, nthreads);
        }
    }
    const float L = block_sum(ls, t, nthreads, scratch, bar);
    // parts may carry a second denominator for the lse (sum of unrounded p when
    // the numerator was formed with rounded p)
    float Lx = L;
    if constexpr (Acc::kSplitL) {
        float lx = 0.f;
        if (M != kNegInf)
            for (int i = t; i < n; i += nthreads) lx += rescale(acc.m2(i), M) * acc.lx(i);
        Lx = block_sum(lx, t, nthreads, scratch, bar);
    }
    for (int ps = 0; ps < passes; ++ps) {
        const float a = ps == 0 ? a0 : a1;
        const int d = ps * DL + dd;
        if (sl < SL) scratch[sl * DL + dd] = a;
        named_bar_sync(bar, nthreads);
        for (int w = SL >> 1; w > 0; w >>= 1) {
            if (sl < w) scratch[sl * DL + dd] += scratch[(sl + w) * DL + dd];
            named_bar_sync(bar, nthreads);
        }
        if (sl == 0 && d < D) out_row[d] = M == kNegInf ? 0.f : scratch[dd] / L;
        named_bar_sync(bar, nthreads);
    }
    if (t == 0 && lse_ptr) *lse_ptr = M == kNegInf ? kNegInf : (M + log2f(Lx)) * kLn2;
}

}  // namespace dev
}  // namespace td
