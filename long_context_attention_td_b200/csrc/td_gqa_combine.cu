// td_gqa_combine -- the merge kernel of the grouped-query decode (sm_100a).
//
// When many CTAs share a (b, kv head) sequence and many query heads share it,
// merging the part records in the last CTA of the sequence would serialise
// G x parts records on one SM; this kernel spreads the merge over one CTA per
// (sequence, query head, 32 columns of D) instead.  What it computes is the
// gist's global max, renormalisation and sums ("Tree Attention Decoding",
// tree_attn_decode) over the records the grouped-query decode kernel wrote.
#include <cuda.h>

#include "td_device.cuh"
#include "td_internal.cuh"
#include "td_tc.cuh"
#include "treedec.h"

namespace td {

using namespace dev;

// The merge of the split sequences' part records: the gist's global max,
// renormalisation and sums, for one (sequence, query head, 32 columns of D) per
// CTA, so that a few sequences with many query heads still spread over the SMs.
// The part statistics (m, l, lx) are read once into shared memory (in chunks of
// kCombChunk parts) with independent loads; each column's parts are split over
// SL lanes that issue their record loads together, and the lanes' partial sums
// finish in a fixed pairwise tree, so the result does not depend on timing.
// Launched as a programmatic dependent of the decode kernel: its CTAs may start
// while that kernel drains and wait (griddepcontrol.wait) until its records are
// complete and visible.
constexpr int kCombChunk = 1024;
constexpr int kCombCols = 32;

template <int kThreads>
__global__ void __launch_bounds__(kThreads) td_gqa_combine_kernel(const GqaParams p, int D) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    constexpr int SL = kThreads / kCombCols;  // part lanes per column
    __shared__ float m_s[kCombChunk], l_s[kCombChunk], lx_s[kCombChunk];
    __shared__ float red[kThreads];
    const int t = static_cast<int>(threadIdx.x);
    const long long seg = blockIdx.x;
    const int g = blockIdx.y;
    const int n = p.seg_desc[seg * 3 + 1];
    if (n <= 1) return;
    const long long c_lo = p.seg_desc[seg * 3 + 0];
    const int first_slot = p.seg_desc[seg * 3 + 2];
    const long long b = seg / p.Hkv, h = seg % p.Hkv;
    const long long orow = b * p.Hq + h * p.G + g;
    const GSlotAcc acc{p.part, c_lo, first_slot, p.G, g, D};
    const int col = t % kCombCols, sl = t / kCombCols;
    const int d = blockIdx.z * kCombCols + col;

    // the maximum over the parts; the first chunk's statistics stay in
    // shared memory (one round of independent loads)
    float mx = kNegInf;
    for (int i = t; i < n; i += kThreads) {
        const float m = acc.m2(i);
        if (i < kCombChunk) {
            m_s[i] = m;
            l_s[i] = acc.l(i);
            lx_s[i] = acc.lx(i);
        }
        mx = fmaxf(mx, m);
    }
    const float M = block_max(mx, t, kThreads, red, 1);

    float a = 0.f, ls = 0.f, lxs = 0.f;
    if (M != kNegInf) {
        for (int i0 = 0; i0 < n; i0 += kCombChunk) {
            const int cnt = n - i0 < kCombChunk ? n - i0 : kCombChunk;
            if (i0 > 0) {
                named_bar_sync(1, kThreads);
                for (int i = t; i < cnt; i += kThreads) {
                    m_s[i] = acc.m2(i0 + i);
                    l_s[i] = acc.l(i0 + i);
                    lx_s[i] = acc.lx(i0 + i);
                }
            }
            named_bar_sync(1, kThreads);
            // weights e^(m_i - M), in place of m
            for (int i = t; i < cnt; i += kThreads) {
                const float w = rescale(m_s[i], M);
                m_s[i] = w;
                ls += w * l_s[i];
                lxs += w * lx_s[i];
            }
            named_bar_sync(1, kThreads);
            constexpr int kBatch = 16;  // independent record loads in flight per thread
            int i = sl;
#pragma unroll 1
            for (; i + (kBatch - 1) * SL < cnt; i += kBatch * SL) {
                float x[kBatch];
#pragma unroll
                for (int j = 0; j < kBatch; ++j) x[j] = acc.num(i0 + i + j * SL, d);
#pragma unroll
                for (int j = 0; j < kBatch; ++j) a = fmaf(m_s[i + j * SL], x[j], a);
            }
            {
                // the rest: at most kBatch - 1 parts per lane, loads first
                float x[kBatch - 1];
                const int left = (cnt - i + SL - 1) / SL;  // <= kBatch - 1
#pragma unroll
                for (int j = 0; j < kBatch - 1; ++j)
                    x[j] = j < left ? acc.num(i0 + i + j * SL, d) : 0.f;
#pragma unroll
                for (int j = 0; j < kBatch - 1; ++j)
                    if (j < left) a = fmaf(m_s[i + j * SL], x[j], a);
            }
        }
    }
    const float L = block_sum(ls, t, kThreads, red, 1);
    const float Lx = block_sum(lxs, t, kThreads, red, 1);
    // the SL partial sums of each column, pairwise
    red[sl * kCombCols + col] = a;
    named_bar_sync(1, kThreads);
#pragma unroll
    for (int w = SL >> 1; w > 0; w >>= 1) {
        if (sl < w) red[sl * kCombCols + col] += red[(sl + w) * kCombCols + col];
        named_bar_sync(1, kThreads);
    }
    if (sl == 0) p.out[orow * D + d] = M == kNegInf ? 0.f : red[col] / L;
    if (t == 0 && blockIdx.z == 0 && p.lse)
        p.lse[orow] = M == kNegInf ? kNegInf : (M + log2f(Lx)) * kLn2;
}

template <int kThreads>
cudaError_t launch_comb_t(dim3 grid, int D, const GqaParams& p, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, td_gqa_combine_kernel<kThreads>, p, D);
}

cudaError_t launch_gqa_combine(int D, const GqaParams& p, cudaStream_t s) {
    const long long segs = static_cast<long long>(p.B) * p.Hkv;
    if (segs > 0x7fffffffLL || p.G > 65535 || D % kCombCols != 0) return cudaErrorInvalidValue;
    dim3 grid(static_cast<unsigned>(segs), static_cast<unsigned>(p.G),
              static_cast<unsigned>(D / kCombCols));
    // parts that touch one sequence, at most
    const long long per_seg = (p.P + segs - 1) / segs + 1;
    if (per_seg >= 64) return launch_comb_t<512>(grid, D, p, s);
    return per_seg >= 16 ? launch_comb_t<256>(grid, D, p, s) : launch_comb_t<128>(grid, D, p, s);
}

}  // namespace td
