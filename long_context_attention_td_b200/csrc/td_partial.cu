// td_partial -- the split-KV decode kernel of libtreedec (sm_100a).
//
// What it computes ("Tree Attention Decoding" gist, tree_attn_decode): the
// keys of all (b,h) sequences, laid end to end, form one flattened key space
// of T keys; CTA c owns keys [floor(cT/P), floor((c+1)T/P)).  For every piece
// of a sequence inside that range it computes the piece's local max m,
// denominator l = sum e^(s-m) and numerator num = sum e^(s-m) v (the gist's
// per-rank local_max, den and num) with an online max-rescaled update per
// tile ("Flash Aandacht", softmax decomposition and fusion).  A piece that is a
// whole sequence is normalised and written out directly.  A sequence cut
// across CTAs leaves one part record per CTA; the last CTA to finish it (an
// atomic ticket, no waiting) merges the records with the gist's global max,
// renormalisation and sums, writes out and lse, and resets the ticket.
//
// Scores: s_j = q.k_j D^-1/2 + slope (j - n + 1) (ALiBi broadcast row, "ALiBi
// with causal=True unexpected bias?"), carried in log2 units (q pre-scaled by
// D^-1/2 log2 e) so every exponential is one ex2.
//
// Structure of a CTA: warp 8 is the producer -- one lane streams K and V tiles
// of the CTA's range into a kStages-deep ring in shared memory with
// cp.async.bulk (the bulk-copy engine; K and V of a sequence are contiguous
// rows, so each tile is one contiguous copy) and mbarrier transaction counts.
// Warps 0-7 consume: a group of kG lanes owns one key row per step, each lane
// holding 16 bytes of q, k, v and its slice of the fp32 accumulator; the dot
// product is finished with xor shuffles inside the group.
#include <atomic>
#include <type_traits>

#include "td_device.cuh"
#include "td_internal.cuh"
#include "treedec.h"

namespace td {
namespace {

using namespace dev;

template <typename T, int D>
struct Cfg {
    static constexpr int kElt = sizeof(T);
    static constexpr int kRowBytes = D * kElt;
    static constexpr int kVec = Elem<T>::kVec;                  // elements per 16 B
    static constexpr int kG = (D / kVec) < 32 ? (D / kVec) : 32;  // lanes per key row
    static constexpr int kNV = D / (kVec * kG);                 // 16-B vectors per lane
    static constexpr int kGPW = 32 / kG;                        // row groups per warp
    static constexpr int kNG = kConsumerWarps * kGPW;           // row groups per CTA
    static constexpr int kRPGraw = (kStageBytes / 2) / (kNG * kRowBytes);
    static constexpr int kRPG = kRPGraw < 1 ? 1 : (kRPGraw > 8 ? 8 : kRPGraw);
    static constexpr int kTile = kRPG * kNG;                    // key rows per stage
    static constexpr int kTileBytes = kTile * kRowBytes;        // K (or V) bytes per stage
    static constexpr int kStage = 2 * kTileBytes;
    static constexpr size_t kSmem =
        size_t(kStages) * kStage + size_t(kConsumerWarps) * (D + 2) * sizeof(float);
    static_assert(kG * kNV * kVec == D, "a key row must split evenly over a lane group");
    static_assert(kRowBytes % 16 == 0, "bulk copies move whole 16-byte units");
    static_assert(kTileBytes % 128 == 0, "stage buffers stay 128-byte aligned");
    static_assert(kConsumerWarps * (D + 2) >= kConsumerThreads, "merge scratch");
};

struct Ctl {
    long long T, x0, x1;  // attended keys, this CTA's flattened range
    long long b0, pre0;   // ragged: batch holding key x0, keys of batches before it
    int abort;            // raised by a failed bounded wait
    int last;             // this CTA took the last ticket of the current sequence
};

__device__ __forceinline__ long long seq_len(const PartialParams& p, int b) {
    int n = __ldg(p.seqlens + b);
    if (n < 0 || n > p.N) {
        atomicOr(p.err, TD_DEVERR_BAD_SEQLEN);
        n = n < 0 ? 0 : static_cast<int>(p.N);
    }
    return n;
}

// First key of part c, and the part holding flattened key x.
__device__ __forceinline__ long long part_start(long long c, long long T, long long P) {
    return c * T / P;
}
__device__ __forceinline__ long long part_of(long long x, long long T, long long P) {
    return ((x + 1) * P - 1) / T;
}

// Walk over the sequences that intersect [x0, x1), in flattened order.
struct Walk {
    long long start, len, pre;
    int b, h;
};

__device__ __forceinline__ bool walk_first(const PartialParams& p, const Ctl& ctl, Walk& w) {
    if (ctl.x0 >= ctl.x1) return false;
    if (p.seqlens == nullptr) {
        const long long g = ctl.x0 / p.N;
        w.b = static_cast<int>(g / p.H);
        w.h = static_cast<int>(g % p.H);
        w.start = g * p.N;
        w.len = p.N;
        w.pre = 0;
    } else {
        w.b = static_cast<int>(ctl.b0);
        w.pre = ctl.pre0;
        w.len = seq_len(p, w.b);
        w.h = static_cast<int>((ctl.x0 - p.H * w.pre) / w.len);
        w.start = p.H * w.pre + w.h * w.len;
    }
    return true;
}

__device__ __forceinline__ bool walk_next(const PartialParams& p, const Ctl& ctl, Walk& w) {
    if (p.seqlens == nullptr) {
        if (++w.h == p.H) {
            w.h = 0;
            ++w.b;
        }
        w.start += p.N;
    } else {
        if (++w.h == p.H) {
            w.h = 0;
            w.pre += w.len;
            do {
                ++w.b;
            } while (w.b < p.B && (w.len = seq_len(p, w.b)) == 0);
            if (w.b >= p.B) return false;
        }
        w.start = p.H * w.pre + w.h * w.len;
    }
    return w.start < ctl.x1;
}

// Part records written by the CTAs that share one sequence, for tree_merge.
struct SlotAcc {
    static constexpr bool kSplitL = false;
    const float* part;
    long long c_lo;
    int first_slot;
    int D;
    __device__ __forceinline__ const float* rec(int i) const {
        const long long c = c_lo + i;
        const int slot = i == 0 ? first_slot : 0;
        return part + (c * 2 + slot) * (D + 2);
    }
    __device__ __forceinline__ float m2(int i) const { return __ldcg(rec(i) + D); }
    __device__ __forceinline__ float l(int i) const { return __ldcg(rec(i) + D + 1); }
    __device__ __forceinline__ float num(int i, int d) const { return __ldcg(rec(i) + d); }
};

constexpr int kBarConsumers = 1;

// 16 E4M3 keys of a lane's slice (one 16-byte word) dotted with its q slice in
// half precision: 8 chained f16x2 fused multiply-adds (q pre-scaled by a power
// of two so every partial stays below 2^15).
__device__ __forceinline__ float dot16_e4m3(const __half2 (&qh)[8], const uint4 w) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    __half2 acc = __float2half2_rn(0.f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = e4m3x2_to_f16x2(ws[i] & 0xffffu);
        const uint32_t hi = e4m3x2_to_f16x2(ws[i] >> 16);
        acc = __hfma2(qh[2 * i], *reinterpret_cast<const __half2*>(&lo), acc);
        acc = __hfma2(qh[2 * i + 1], *reinterpret_cast<const __half2*>(&hi), acc);
    }
    return __low2float(acc) + __high2float(acc);
}

// EQ: type of q; E: type of the K/V rows (EQ, or E4M3 for an FP8 cache).
template <typename EQ, typename E, int D>
__global__ void __launch_bounds__(kPartialThreads, kCtasPerSm) td_partial_kernel(const PartialParams p) {
    using C = Cfg<E, D>;
    constexpr bool kFp8 = std::is_same<E, E4M3>::value;
    static_assert(kFp8 || std::is_same<E, EQ>::value, "q and K/V share a type unless K/V is FP8");
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ __align__(8) uint64_t full_bar[kStages];
    __shared__ __align__(8) uint64_t empty_bar[kStages];
    __shared__ Ctl ctl;
    float* red = reinterpret_cast<float*>(smem + size_t(kStages) * C::kStage);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const long long c = blockIdx.x;
    const long long P = p.P;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_addr(&full_bar[s]), 1);
            mbar_init(smem_addr(&empty_bar[s]), kConsumerWarps);
        }
        fence_barrier_init();
        ctl.abort = 0;
        ctl.last = 0;
    }
    if (p.seqlens == nullptr) {
        if (tid == 0) {
            ctl.T = p.T;
            ctl.x0 = part_start(c, p.T, P);
            ctl.x1 = part_start(c + 1, p.T, P);
            ctl.b0 = 0;
            ctl.pre0 = 0;
        }
    } else {
        if (warp == 0) {
            // total attended keys, then the batch that holds key x0
            long long sum = 0;
            for (int b = lane; b < p.B; b += 32) sum += seq_len(p, b);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            const long long T = sum * p.H;
            const long long x0 = T > 0 ? part_start(c, T, P) : 0;
            const long long x1 = T > 0 ? part_start(c + 1, T, P) : 0;
            long long b0 = p.B, pre0 = sum;
            if (x0 < x1) {
                long long run = 0;
                for (int base = 0; base < p.B; base += 32) {
                    const int b = base + lane;
                    const long long n = b < p.B ? seq_len(p, b) : 0;
                    long long incl = n;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const long long y = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += y;
                    }
                    const bool hit = b < p.B && p.H * (run + incl) > x0;
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
        // sequences of length 0 own no key: part (b mod P) writes their result
        for (long long b = c; b < p.B; b += P) {
            if (seq_len(p, static_cast<int>(b)) != 0) continue;
            for (int i = tid; i < p.H * D; i += kPartialThreads) p.out[b * p.H * D + i] = 0.f;
            if (p.lse)
                for (int h = tid; h < p.H; h += kPartialThreads) p.lse[b * p.H + h] = kNegInf;
        }
    }
    __syncthreads();

    const long long T = ctl.T, x0 = ctl.x0, x1 = ctl.x1;
    volatile int* abort_flag = &ctl.abort;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        if (lane != 0) return;
        const uint64_t pol = l2_policy_evict_first();
        const char* kbase = static_cast<const char*>(p.k);
        const char* vbase = static_cast<const char*>(p.v);
        int stage = 0;
        uint32_t phase = 0;
        long long issued = 0;
        bool aborted = false;
        // the failure-path test: CTA 0 stops arming stages at this tile, so
        // the consumers' next wait can only end by its time limit
        const long long stop_at = c == 0 ? p.withhold_tile : -1;
        Walk w;
        if (walk_first(p, ctl, w)) {
            do {
                const long long j0 = (x0 > w.start ? x0 : w.start) - w.start;
                const long long e = w.start + w.len;
                const long long j1 = (x1 < e ? x1 : e) - w.start;
                const long long rowbase = (static_cast<long long>(w.b) * p.H + w.h) * p.N;
                for (long long t0 = j0; t0 < j1; t0 += C::kTile) {
                    const long long left = j1 - t0;
                    const int rows = left < C::kTile ? static_cast<int>(left) : C::kTile;
                    if (issued == stop_at) aborted = true;
                    if (!aborted && !mbar_wait_bounded(smem_addr(&empty_bar[stage]), phase ^ 1u,
                                                       abort_flag, p.err, TD_DEVERR_WAIT_TIMEOUT,
                                                       p.wait_ns))
                        aborted = true;
                    if (!aborted) {
                        const uint32_t bytes = static_cast<uint32_t>(rows) * C::kRowBytes;
                        const uint32_t fb = smem_addr(&full_bar[stage]);
                        const size_t off = static_cast<size_t>(rowbase + t0) * C::kRowBytes;
                        const uint32_t dst = smem_addr(smem + size_t(stage) * C::kStage);
                        mbar_arrive_expect_tx(fb, 2u * bytes);
                        bulk_copy_g2s(dst, kbase + off, bytes, fb, pol);
                        bulk_copy_g2s(dst + C::kTileBytes, vbase + off, bytes, fb, pol);
                        ++issued;
                    }
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            } while (walk_next(p, ctl, w));
        }
        // No copy may still be landing in shared memory when the CTA exits:
        // wait (bounded, ignoring the abort flag) for the last phase issued
        // on every stage.
        for (int s = 0; s < kStages && s < issued; ++s) {
            const long long lastTile = s + ((issued - 1 - s) / kStages) * kStages;
            const uint32_t par = static_cast<uint32_t>((lastTile / kStages) & 1);
            mbar_wait_bounded(smem_addr(&full_bar[s]), par, nullptr, p.err,
                              TD_DEVERR_WAIT_TIMEOUT, p.wait_ns);
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    const int lig = lane % C::kG;             // lane within its row group
    const int gi = warp * C::kGPW + lane / C::kG;  // row group index in the CTA
    int stage = 0;
    uint32_t phase = 0;
    bool aborted = false;
    int piece = 0;
    Walk w;
    if (!walk_first(p, ctl, w)) return;
    do {
        const long long j0 = (x0 > w.start ? x0 : w.start) - w.start;
        const long long e = w.start + w.len;
        const long long j1 = (x1 < e ? x1 : e) - w.start;
        const bool whole = (j0 == 0 && j1 == w.len);
        const long long bh = static_cast<long long>(w.b) * p.H + w.h;

        // q widened to fp32 once per piece; the D^-1/2 log2(e) scale is applied
        // to the finished dot product
        float qf[C::kNV][C::kVec];
        {
            const EQ* qrow = static_cast<const EQ*>(p.q) + bh * D;
            constexpr int kQV = Elem<EQ>::kVec;  // q elements per 16-byte load
#pragma unroll
            for (int u = 0; u < C::kNV; ++u)
#pragma unroll
                for (int part = 0; part < C::kVec / kQV; ++part)
                    Elem<EQ>::to_f32(__ldg(reinterpret_cast<const uint4*>(
                                         qrow + (u * C::kG + lig) * C::kVec + part * kQV)),
                                     qf[u] + part * kQV);
        }
        float qscale2 = p.qscale2;
        // FP8 cache: q in half precision, scaled by 2^e so that |q| 2^e < 8 and
        // each 8-term partial of q . k (|k| <= 448) stays below 2^15; the dot
        // product is taken back by 2^-e, and the per-head key scale joins the
        // score scale
        __half2 qh[C::kNV][C::kVec / 2];
        float qinv = 1.f;
        if constexpr (kFp8) {
            float amax = 0.f;
#pragma unroll
            for (int u = 0; u < C::kNV; ++u)
#pragma unroll
                for (int x = 0; x < C::kVec; ++x) amax = fmaxf(amax, fabsf(qf[u][x]));
            int ex = 0;
            frexpf(amax, &ex);                       // amax < 2^ex
            const int e = amax > 0.f ? max(-24, min(24, 3 - ex)) : 0;
            const float up = ldexpf(1.f, e);
            qinv = ldexpf(1.f, -e);
#pragma unroll
            for (int u = 0; u < C::kNV; ++u)
#pragma unroll
                for (int x = 0; x < C::kVec / 2; ++x)
                    qh[u][x] = __floats2half2_rn(qf[u][2 * x] * up, qf[u][2 * x + 1] * up);
            qscale2 *= __ldg(p.k_scale + w.h);
        }
        const bool has_bias = p.slopes != nullptr;
        const float slope2 = has_bias ? __ldg(p.slopes + w.h) * kLog2e : 0.f;
        const long long pos0 = 1 - w.len + p.alibi_off;   // ALiBi position of key 0

        float m = kNegInf, l = 0.f;
        float acc[C::kNV][C::kVec];
#pragma unroll
        for (int u = 0; u < C::kNV; ++u)
#pragma unroll
            for (int x = 0; x < C::kVec; ++x) acc[u][x] = 0.f;

        for (long long t0 = j0; t0 < j1; t0 += C::kTile) {
            const long long left = j1 - t0;
            const int rows = left < C::kTile ? static_cast<int>(left) : C::kTile;
            if (!aborted && !mbar_wait_bounded(smem_addr(&full_bar[stage]), phase, abort_flag,
                                               p.err, TD_DEVERR_WAIT_TIMEOUT, p.wait_ns))
                aborted = true;
            const unsigned char* sk = smem + size_t(stage) * C::kStage;
            const unsigned char* sv = sk + C::kTileBytes;

            float s[C::kRPG];
#pragma unroll
            for (int i = 0; i < C::kRPG; ++i) {
                const int row = gi + i * C::kNG;
                float a = 0.f;
                if (row < rows) {
#pragma unroll
                    for (int u = 0; u < C::kNV; ++u) {
                        if constexpr (kFp8) {
                            a = fmaf(dot16_e4m3(qh[u], lds128(sk + row * C::kRowBytes +
                                                              (u * C::kG + lig) * 16)),
                                     qinv, a);
                        } else {
                            float kf[C::kVec];
                            Elem<E>::to_f32(
                                lds128(sk + row * C::kRowBytes + (u * C::kG + lig) * 16), kf);
#pragma unroll
                            for (int x = 0; x < C::kVec; ++x) a = fmaf(qf[u][x], kf[x], a);
                        }
                    }
                }
                s[i] = a;
            }
#pragma unroll
            for (int i = 0; i < C::kRPG; ++i)
#pragma unroll
                for (int o = C::kG / 2; o > 0; o >>= 1) s[i] += __shfl_xor_sync(0xffffffffu, s[i], o);

            float tmax = kNegInf;
#pragma unroll
            for (int i = 0; i < C::kRPG; ++i) {
                const int row = gi + i * C::kNG;
                if (row < rows) {
                    s[i] = has_bias
                               ? fmaf(s[i], qscale2, slope2 * static_cast<float>(t0 + row + pos0))
                               : s[i] * qscale2;
                    tmax = fmaxf(tmax, s[i]);
                } else {
                    s[i] = kNegInf;
                }
            }
            if (tmax != kNegInf) {
                const float mn = fmaxf(m, tmax);
                const float alpha = rescale(m, mn);
                l *= alpha;
#pragma unroll
                for (int u = 0; u < C::kNV; ++u)
#pragma unroll
                    for (int x = 0; x < C::kVec; ++x) acc[u][x] *= alpha;
                if constexpr (kFp8) {
                    // the tile's p v products in half precision (at most kRPG
                    // terms per value), then added to the fp32 accumulators
                    __half2 acch[C::kNV][C::kVec / 2];
#pragma unroll
                    for (int u = 0; u < C::kNV; ++u)
#pragma unroll
                        for (int x = 0; x < C::kVec / 2; ++x) acch[u][x] = __float2half2_rn(0.f);
#pragma unroll
                    for (int i = 0; i < C::kRPG; ++i) {
                        const int row = gi + i * C::kNG;
                        if (row < rows) {
                            const float pr = ex2(s[i] - mn);
                            l += pr;
                            const __half2 ph = __float2half2_rn(pr);
#pragma unroll
                            for (int u = 0; u < C::kNV; ++u) {
                                const uint4 wv =
                                    lds128(sv + row * C::kRowBytes + (u * C::kG + lig) * 16);
                                const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                                for (int y = 0; y < 4; ++y) {
                                    const uint32_t lo = e4m3x2_to_f16x2(ws[y] & 0xffffu);
                                    const uint32_t hi = e4m3x2_to_f16x2(ws[y] >> 16);
                                    acch[u][2 * y] = __hfma2(
                                        ph, *reinterpret_cast<const __half2*>(&lo), acch[u][2 * y]);
                                    acch[u][2 * y + 1] =
                                        __hfma2(ph, *reinterpret_cast<const __half2*>(&hi),
                                                acch[u][2 * y + 1]);
                                }
                            }
                        }
                    }
#pragma unroll
                    for (int u = 0; u < C::kNV; ++u)
#pragma unroll
                        for (int x = 0; x < C::kVec / 2; ++x) {
                            acc[u][2 * x] += __low2float(acch[u][x]);
                            acc[u][2 * x + 1] += __high2float(acch[u][x]);
                        }
                } else {
#pragma unroll
                    for (int i = 0; i < C::kRPG; ++i) {
                        const int row = gi + i * C::kNG;
                        if (row < rows) {
                            const float pr = ex2(s[i] - mn);
                            l += pr;
#pragma unroll
                            for (int u = 0; u < C::kNV; ++u) {
                                float vf[C::kVec];
                                Elem<E>::to_f32(
                                    lds128(sv + row * C::kRowBytes + (u * C::kG + lig) * 16), vf);
#pragma unroll
                                for (int x = 0; x < C::kVec; ++x)
                                    acc[u][x] = fmaf(pr, vf[x], acc[u][x]);
                            }
                        }
                    }
                }
                m = mn;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&empty_bar[stage]));
            if (++stage == kStages) {
                stage = 0;
                phase ^= 1u;
            }
        }

        if constexpr (kFp8) {
            // the per-head value scale of the FP8 cache
            const float vs = __ldg(p.v_scale + w.h);
#pragma unroll
            for (int u = 0; u < C::kNV; ++u)
#pragma unroll
                for (int x = 0; x < C::kVec; ++x) acc[u][x] *= vs;
        }

        // ---- end of piece: merge the row groups of the warp (xor butterfly)
#pragma unroll
        for (int o = C::kG; o < 32; o <<= 1) {
            const float mo = __shfl_xor_sync(0xffffffffu, m, o);
            const float lo = __shfl_xor_sync(0xffffffffu, l, o);
            const float M = fmaxf(m, mo);
            const float a = rescale(m, M), b = rescale(mo, M);
            l = l * a + lo * b;
#pragma unroll
            for (int u = 0; u < C::kNV; ++u)
#pragma unroll
                for (int x = 0; x < C::kVec; ++x) {
                    const float ao = __shfl_xor_sync(0xffffffffu, acc[u][x], o);
                    acc[u][x] = acc[u][x] * a + ao * b;
                }
            m = M;
        }
        float* rw = red + warp * (D + 2);
        if (lane < C::kG) {
#pragma unroll
            for (int u = 0; u < C::kNV; ++u)
#pragma unroll
                for (int x = 0; x < C::kVec; ++x) rw[(u * C::kG + lig) * C::kVec + x] = acc[u][x];
            if (lane == 0) {
                rw[D] = m;
                rw[D + 1] = l;
            }
        }
        named_bar_sync(kBarConsumers, kConsumerThreads);

        // ---- then across the consumer warps (fixed order)
        float M = kNegInf;
#pragma unroll
        for (int q = 0; q < kConsumerWarps; ++q) M = fmaxf(M, red[q * (D + 2) + D]);
        float sc[kConsumerWarps];
        float L = 0.f;
#pragma unroll
        for (int q = 0; q < kConsumerWarps; ++q) {
            sc[q] = rescale(red[q * (D + 2) + D], M);
            L += sc[q] * red[q * (D + 2) + D + 1];
        }
        if (whole) {
            for (int d = tid; d < D; d += kConsumerThreads) {
                float A = 0.f;
#pragma unroll
                for (int q = 0; q < kConsumerWarps; ++q) A += sc[q] * red[q * (D + 2) + d];
                p.out[bh * D + d] = A / L;
            }
            if (tid == 0 && p.lse) p.lse[bh] = (M + log2f(L)) * kLn2;
            named_bar_sync(kBarConsumers, kConsumerThreads);
        } else {
            const int slot = piece == 0 ? 0 : 1;
            float* rec = p.part + (c * 2 + slot) * (D + 2);
            for (int d = tid; d < D; d += kConsumerThreads) {
                float A = 0.f;
#pragma unroll
                for (int q = 0; q < kConsumerWarps; ++q) A += sc[q] * red[q * (D + 2) + d];
                rec[d] = A;
            }
            if (tid == 0) {
                rec[D] = M;
                rec[D + 1] = L;
            }
            __threadfence();
            named_bar_sync(kBarConsumers, kConsumerThreads);
            const long long c_lo = part_of(w.start, T, P);
            const long long c_hi = part_of(w.start + w.len - 1, T, P);
            const int n = static_cast<int>(c_hi - c_lo + 1);
            if (tid == 0) {
                const int prev = atomicAdd(p.tickets + bh, 1);
                const int last = prev == n - 1;
                if (last) atomicExch(p.tickets + bh, 0);
                ctl.last = last;
            }
            named_bar_sync(kBarConsumers, kConsumerThreads);
            if (ctl.last) {
                __threadfence();
                const SlotAcc sa{p.part, c_lo, part_start(c_lo, T, P) < w.start ? 1 : 0, D};
                tree_merge(sa, n, D, tid, kConsumerThreads, red, kConsumerWarps * (D + 2),
                           kBarConsumers, p.out + bh * D, p.lse ? p.lse + bh : nullptr);
            }
            named_bar_sync(kBarConsumers, kConsumerThreads);
        }
        ++piece;
    } while (walk_next(p, ctl, w));
}

template <typename TQ, typename T, int D>
cudaError_t launch_t(int device, const PartialParams& p, cudaStream_t s) {
    using C = Cfg<T, D>;
    auto kern = td_partial_kernel<TQ, T, D>;
    // the dynamic shared-memory opt-in is per device: set it once on each
    static std::atomic<unsigned long long> configured{0};
    const unsigned long long bit = device < 64 ? (1ull << device) : 0ull;
    if (!bit || !(configured.load(std::memory_order_acquire) & bit)) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::kSmem));
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    kern<<<static_cast<unsigned>(p.P), kPartialThreads, C::kSmem, s>>>(p);
    return cudaGetLastError();
}

template <typename TQ, typename T = TQ>
cudaError_t launch_d(int device, int D, const PartialParams& p, cudaStream_t s) {
    switch (D) {
        case 64: return launch_t<TQ, T, 64>(device, p, s);
        case 128: return launch_t<TQ, T, 128>(device, p, s);
        case 256: return launch_t<TQ, T, 256>(device, p, s);
        case 512: return launch_t<TQ, T, 512>(device, p, s);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
size_t smem_d(int D) {
    switch (D) {
        case 64: return Cfg<T, 64>::kSmem;
        case 128: return Cfg<T, 128>::kSmem;
        case 256: return Cfg<T, 256>::kSmem;
        case 512: return Cfg<T, 512>::kSmem;
        default: return 0;
    }
}

}  // namespace

cudaError_t launch_partial(int device, int dtype, int D, const PartialParams& p, cudaStream_t s) {
    switch (dtype) {
        case kF32: return launch_d<float>(device, D, p, s);
        case kBF16: return launch_d<__nv_bfloat16>(device, D, p, s);
        case kF16: return launch_d<__half>(device, D, p, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_partial_fp8(int device, int q_dtype, int D, const PartialParams& p,
                               cudaStream_t s) {
    if (!p.k_scale || !p.v_scale) return cudaErrorInvalidValue;
    switch (q_dtype) {
        case kBF16: return launch_d<__nv_bfloat16, E4M3>(device, D, p, s);
        case kF16: return launch_d<__half, E4M3>(device, D, p, s);
        default: return cudaErrorInvalidValue;
    }
}

size_t partial_smem_bytes(int dtype, int D) {
    switch (dtype) {
        case kF32: return smem_d<float>(D);
        case kBF16: return smem_d<__nv_bfloat16>(D);
        case kF16: return smem_d<__half>(D);
        case kE4M3: return smem_d<E4M3>(D);
        default: return 0;
    }
}

int partial_ctas_per_sm(int dtype, int D) {
    // 228 KiB of shared memory per SM, 1 KiB reserved per CTA, plus the static
    // barriers/control block; the launch bounds ask for one CTA's registers.
    const size_t smem = partial_smem_bytes(dtype, D);
    if (smem == 0) return 0;
    const size_t per_cta = smem + 1024 + 256;
    int by_smem = static_cast<int>((228u * 1024u) / per_cta);
    const int by_threads = 2048 / kPartialThreads;
    int n = by_smem < by_threads ? by_smem : by_threads;
    if (n > kCtasPerSm) n = kCtasPerSm;
    return n < 1 ? 1 : n;
}

}  // namespace td
