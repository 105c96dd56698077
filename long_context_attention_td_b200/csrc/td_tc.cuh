// td_tc.cuh -- sm_100a tensor-core, TMA and partition helpers shared by the
// tensor-core kernels (td_gqa_keys.cu: grouped-query decode with the keys on
// the MMA M axis; td_gqa_combine.cu: its merge; td_prefill.cu).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "td_device.cuh"
#include "td_internal.cuh"
#include "treedec.h"

namespace td {
namespace {

using namespace dev;

struct GCtl {
    long long T, x0, x1, b0, pre0;
    int abort;
    int last;
    uint32_t tmem;
};
// ------------------------------------------------------------ tcgen05 PTX

__device__ __forceinline__ void fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// non-blocking test of the phase with the given parity
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16, one CTA
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// arrive on `bar` when every tcgen05 op issued so far by this thread is done
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
          "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
          "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
          "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
          "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 2-D tiled TMA load (no multicast) of box {64 columns, 64 rows}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(pol)
        : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 format (version 1).
// lbo/sbo in bytes.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= uint64_t((addr >> 4) & 0x3FFFu);
    d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
    d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
    d |= uint64_t(1) << 46;  // descriptor version for sm_100
    d |= uint64_t(2) << 61;  // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::f16, fp32 accumulate.  ab: 0 = f16, 1 = bf16.
__host__ __device__ constexpr uint32_t instr_desc_f16(int ab, int m, int n, int a_mn, int b_mn) {
    return (1u << 4) | (uint32_t(ab) << 7) | (uint32_t(ab) << 10) | (uint32_t(a_mn) << 15) |
           (uint32_t(b_mn) << 16) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}

// offset of 16-byte chunk c of row r inside a 128-byte-swizzled block
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return uint32_t(r) * 128u + (uint32_t(c ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint32_t pack_round(float a, float b, bool bf16, float& ra, float& rb) {
    uint32_t w;
    if (bf16) {
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(b), "f"(a));
        ra = __uint_as_float(w << 16);
        rb = __uint_as_float(w & 0xffff0000u);
    } else {
        asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(b), "f"(a));
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
        ra = f.x;
        rb = f.y;
    }
    return w;
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// ------------------------------------------------------ records and walk

// Part record of one query head: num[D], m (log2 units), l of the rounded p
// (normalises num), l of the unrounded p (for lse).
struct GSlotAcc {
    static constexpr bool kSplitL = true;
    const float* part;
    long long c_lo;
    int first_slot, G, g, D;
    __device__ __forceinline__ const float* rec(int i) const {
        const long long c = c_lo + i;
        const int slot = i == 0 ? first_slot : 0;
        return part + ((c * 2 + slot) * G + g) * (D + 3);
    }
    __device__ __forceinline__ float m2(int i) const { return __ldcg(rec(i) + D); }
    __device__ __forceinline__ float l(int i) const { return __ldcg(rec(i) + D + 1); }
    __device__ __forceinline__ float lx(int i) const { return __ldcg(rec(i) + D + 2); }
    __device__ __forceinline__ float num(int i, int d) const { return __ldcg(rec(i) + d); }
};

__device__ __forceinline__ long long gseq_len(const GqaParams& p, int b) {
    int n = __ldg(p.seqlens + b);
    if (n < 0 || n > p.N) {
        atomicOr(p.err, TD_DEVERR_BAD_SEQLEN);
        n = n < 0 ? 0 : static_cast<int>(p.N);
    }
    return n;
}

struct GWalk {
    long long start, len, pre;
    int b, h;  // h: kv head
};

__device__ __forceinline__ bool gwalk_first(const GqaParams& p, const GCtl& ctl, GWalk& w) {
    if (ctl.x0 >= ctl.x1) return false;
    if (p.seqlens == nullptr) {
        const long long g = ctl.x0 / p.N;
        w.b = static_cast<int>(g / p.Hkv);
        w.h = static_cast<int>(g % p.Hkv);
        w.start = g * p.N;
        w.len = p.N;
        w.pre = 0;
    } else {
        w.b = static_cast<int>(ctl.b0);
        w.pre = ctl.pre0;
        w.len = gseq_len(p, w.b);
        w.h = static_cast<int>((ctl.x0 - p.Hkv * w.pre) / w.len);
        w.start = p.Hkv * w.pre + w.h * w.len;
    }
    return true;
}

__device__ __forceinline__ bool gwalk_next(const GqaParams& p, const GCtl& ctl, GWalk& w) {
    if (p.seqlens == nullptr) {
        if (++w.h == p.Hkv) {
            w.h = 0;
            ++w.b;
        }
        w.start += p.N;
    } else {
        if (++w.h == p.Hkv) {
            w.h = 0;
            w.pre += w.len;
            do {
                ++w.b;
            } while (w.b < p.B && (w.len = gseq_len(p, w.b)) == 0);
            if (w.b >= p.B) return false;
        }
        w.start = p.Hkv * w.pre + w.h * w.len;
    }
    return w.start < ctl.x1;
}

__device__ __forceinline__ long long gpart_start(long long c, long long T, long long P) {
    return c * T / P;
}
__device__ __forceinline__ long long gpart_of(long long x, long long T, long long P) {
    return ((x + 1) * P - 1) / T;
}

// Part boundaries of CTA c over the flattened keys (ctl.T, x0, x1 and, for
// ragged batches, the first sequence b0 with its key offset pre0), found by
// warp 0; CTAs also zero the outputs of empty sequences.  Every thread calls
// it; ctl is read after the caller's __syncthreads.
__device__ __forceinline__ void gqa_partition(const GqaParams& p, GCtl& ctl, long long c, int tid,
                                              int warp, int lane, int nthreads, int D) {
    const long long P = p.P;
    if (p.seqlens == nullptr) {
        if (tid == 0) {
            ctl.T = p.T;
            ctl.x0 = gpart_start(c, p.T, P);
            ctl.x1 = gpart_start(c + 1, p.T, P);
            ctl.b0 = 0;
            ctl.pre0 = 0;
        }
    } else {
        if (warp == 0) {
            long long sum = 0;
            for (int b = lane; b < p.B; b += 32) sum += gseq_len(p, b);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            const long long T = sum * p.Hkv;
            const long long x0 = T > 0 ? gpart_start(c, T, P) : 0;
            const long long x1 = T > 0 ? gpart_start(c + 1, T, P) : 0;
            long long b0 = p.B, pre0 = sum;
            if (x0 < x1) {
                long long run = 0;
                for (int base = 0; base < p.B; base += 32) {
                    const int b = base + lane;
                    const long long n = b < p.B ? gseq_len(p, b) : 0;
                    long long incl = n;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const long long y = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += y;
                    }
                    const bool hit = b < p.B && p.Hkv * (run + incl) > x0;
                    const unsigned m = __ballot_sync(0xffffffffu, hit);
                    if (m) {
                        const int L = __ffs(m) - 1;
                        const long long inclL = __shfl_sync(0xffffffffu, incl, L);
                        const long long nL = __shfl_sync(0xffffffffu, n, L);
                        b0 = base + L;
                        pre0 = run + inclL - nL;
                        break;
                    }
                    run += __shfl_sync(0xffffffffu, incl, 31);
                }
            }
            if (lane == 0) {
                ctl.T = T;
                ctl.x0 = x0;
                ctl.x1 = x1;
                ctl.b0 = b0;
                ctl.pre0 = pre0;
            }
        }
        for (long long b = c; b < p.B; b += P) {
            if (gseq_len(p, static_cast<int>(b)) != 0) continue;
            for (int i = tid; i < p.Hq * D; i += nthreads) p.out[b * p.Hq * D + i] = 0.f;
            if (p.lse)
                for (int h = tid; h < p.Hq; h += nthreads) p.lse[b * p.Hq + h] = kNegInf;
            if (!p.fused_merge)
                for (int h = tid; h < p.Hkv; h += nthreads) p.seg_desc[(b * p.Hkv + h) * 3 + 1] = 0;
        }
    }
}

}  // namespace
}  // namespace td
