// td_gqa -- grouped-query / multi-query split-KV decode on the sm_100a
// tensor cores (tcgen05 + TMEM).
//
// What it computes: as td_partial ("Tree Attention Decoding" gist, Algorithm
// 3), but G = Hq / Hkv query heads share each key/value head, so one pass over
// a K/V tile serves G queries.  The tile work is then a small dense
// contraction: S = Q K^T with Q [G x D] and P V with P [G x keys], which this
// kernel issues to the 5th-generation tensor cores with the query heads on
// the MMA's M axis (M = 128, rows >= G are zero).
//
// The keys of all (b, kv-head) sequences form one flattened space split evenly
// over the CTAs, exactly as in td_partial; pieces of a sequence cut across CTAs
// are merged by the last CTA to finish (atomic ticket), per query head.
//
// One CTA per SM, 10 warps:
//   warp 0      TMA producer: K and V tiles of 64 keys, 2-D tensor-map loads
//               with 128-byte swizzle (one box per 64 columns of D), 4 stages;
//   warp 1      allocates 512 TMEM columns and issues the MMAs from one lane:
//               S(t) = Q K(t)^T into S buffer t%2, O(t%2) += P(t) V(t), with
//               completion signalled by tcgen05.commit;
//   warps 2-5   softmax warpgroup 0 (even tiles), warps 6-9 warpgroup 1 (odd
//               tiles); warp w reads TMEM lanes 32*(w%4)..+31.  Each group keeps
//               its own running max and O accumulator, so one group's latency
//               chain (read S, exponentials, write P) overlaps the other's.  The
//               query rows are replicated across the lane quarters (see
//               softmax_role) and every (group, replica) is merged at the end of
//               a piece, which then gives the output or a part record.
// The running max m of a row is only moved when a tile's max exceeds it by
// more than 8 (log2 units); O in TMEM is rescaled then, and p <= 2^8 otherwise.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <type_traits>

#include "td_device.cuh"
#include "td_internal.cuh"
#include "td_tc.cuh"
#include "treedec.h"

namespace td {
namespace {

using namespace dev;

constexpr int kTK = 64;            // keys per tile
constexpr int kM = 128;            // MMA rows (query heads, padded)
constexpr int kGqaStages = 4;      // K/V pipeline depth
constexpr int kGqaThreads = 320;   // 10 warps
constexpr int kSoftmaxThreads = 128;  // one softmax warpgroup
constexpr int kTmemCols = 512;     // S0 [0,64) S1 [64,128) O0 [128,256) O1 [256,384)
constexpr int kScratchFloats = 1024;
constexpr float kRescaleThreshold = 8.f;  // log2 units

template <int D>
struct GCfg {
    static constexpr int kAtoms = D / 64;                    // 64-column swizzle atoms
    static constexpr int kQBytes = kAtoms * kM * 128;        // Q, K-major SW128
    static constexpr int kPBytes = kM * 128;                 // one P buffer (64 keys)
    static constexpr int kKVAtomBytes = kTK * 128;           // 64 keys x 64 columns
    static constexpr int kStageBytes = 2 * kAtoms * kKVAtomBytes;  // K atoms, then V atoms
    static constexpr int kOffQ = 0;
    static constexpr int kOffP = kOffQ + kQBytes;
    static constexpr int kOffKV = kOffP + 2 * kPBytes;
    static constexpr int kOffScratch = kOffKV + kGqaStages * kStageBytes;
    // end-of-piece staging of the replicas' O rows: 128 rows x 32 columns, row stride 33
    static constexpr int kOffStage = kOffScratch + kScratchFloats * 4;
    static constexpr int kStageFloats = kM * 33;
    static constexpr size_t kSmem = size_t(kOffStage) + kStageFloats * 4 + 1024;  // +align
    static_assert(D == 64 || D == 128, "D");
};

constexpr int kBarSoftmax = 1;  // named barrier of softmax warpgroup 0
constexpr int kBarGroups = 2;   // named barrier of both softmax warpgroups

struct SmCtx {
    unsigned char* smem;
    float* scratch;
    uint64_t* s_full;
    uint64_t* s_empty;
    uint64_t* p_full;
    uint64_t* pv_done;
    uint64_t* q_ready;
    GCtl* ctl;
    volatile int* abort_flag;
    uint32_t tmem;
    long long T, x0, x1, P, c;
    int warp, lane, tid;
};

// The softmax warpgroup.  The G query rows are replicated R = 64 / CW times
// across the TMEM lane quarters (rows rep*RR + g, RR = 128 / R); replica rep
// handles key columns [rep*CW, rep*CW + CW) of every tile as an independent
// split with its own running max, so all four warps share the exponentials.
// At the end of a piece the replicas are merged in shared memory.
template <typename E, int D, int CW>
__device__ __forceinline__ void softmax_role(const GqaParams& p, const SmCtx& x) {
    using C = GCfg<D>;
    constexpr bool kBF16 = std::is_same<E, __nv_bfloat16>::value;
    constexpr int R = kTK / CW;   // replicas
    constexpr int RR = kM / R;    // MMA rows per replica
    const int G = p.G;
    const int grp = (x.warp - 2) >> 2;    // 0: even tiles, 1: odd tiles
    const int quarter = x.warp & 3;
    const int r = quarter * 32 + x.lane;  // MMA row (TMEM lane)
    const int rep = r / RR;               // replica: key-column slice of each tile
    const int g = r - rep * RR;           // query head within the group
    const bool warp_active = ((quarter * 32) % RR) < G;
    const bool active = g < G;
    const int st = (x.tid - 64) & (kSoftmaxThreads - 1);  // 0..127 within the warpgroup
    const int lane = x.lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t o_col = 128u + 128u * static_cast<uint32_t>(grp);  // this group's O
    const int cb = rep * CW;              // first key column of this replica
    const float qscale2 = p.qscale2;
    unsigned char* smem = x.smem;
    float* stage = reinterpret_cast<float*>(smem + C::kOffStage);
    float* stats = x.scratch;             // group 0: merged (m, l, lx) per row
    float* stats1 = x.scratch + 3 * kM;   // group 1's (m, l, lx) per row
    long long t = 0;
    long long pc = 0;
    bool aborted = false;
    auto wait = [&](uint64_t* bar, uint32_t par) {
        if (!aborted && !mbar_wait_bounded(smem_addr(bar), par, x.abort_flag, p.err,
                                           TD_DEVERR_WAIT_TIMEOUT))
            aborted = true;
    };
    GWalk w;
    if (!gwalk_first(p, *x.ctl, w)) return;
    do {
        const long long j0 = (x.x0 > w.start ? x.x0 : w.start) - w.start;
        const long long e = w.start + w.len;
        const long long j1 = (x.x1 < e ? x.x1 : e) - w.start;
        const long long nt = (j1 - j0 + kTK - 1) / kTK;
        const bool whole = (j0 == 0 && j1 == w.len);
        const long long hq = static_cast<long long>(w.h) * G + g;          // query head
        const long long qrow = static_cast<long long>(w.b) * p.Hq + hq;   // b*Hq + hq
        // Q rows of this kv head's group (each replica a copy), K-major SW128
        if (grp == 0) {
            if (active) {
                const uint4* qg =
                    reinterpret_cast<const uint4*>(static_cast<const E*>(p.q) + qrow * D);
#pragma unroll
                for (int a = 0; a < C::kAtoms; ++a)
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc)
                        *reinterpret_cast<uint4*>(smem + C::kOffQ + a * (kM * 128) + swz(r, cc)) =
                            __ldg(qg + a * 8 + cc);
            }
            fence_proxy_async_smem();
        }
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(x.q_ready));

        const float slope2 = (active && p.slopes) ? __ldg(p.slopes + hq) * kLog2e : 0.f;
        // l: sum of p as rounded for the P V product (normalises O);
        // lx: sum of the unrounded p (for lse)
        float m_ref = kNegInf, l = 0.f, lx = 0.f;
        long long last_own = -1;
        for (long long i = 0; i < nt; ++i, ++t) {
            if (static_cast<int>(t & 1) != grp) continue;
            last_own = t;
            const long long t0 = j0 + i * kTK;
            const int rows = static_cast<int>((j1 - t0) < kTK ? (j1 - t0) : kTK);
            wait(&x.s_full[grp], static_cast<uint32_t>((t >> 1) & 1));
            fence_after();
            uint32_t sr[CW];
            if (warp_active) {
                const uint32_t sa = x.tmem + lane_addr + static_cast<uint32_t>(grp * kTK + cb);
                if constexpr (CW == 16) {
                    tmem_ld16(sa, sr);
                } else {
#pragma unroll
                    for (int h = 0; h < CW / 32; ++h)
                        tmem_ld32(sa + 32 * h, *reinterpret_cast<uint32_t(*)[32]>(sr + 32 * h));
                }
                tmem_wait_ld();
            }
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&x.s_empty[grp]));

            if (rows < kTK) {
                // keys past the piece end: the tile holds other rows (or padding
                // that may not be finite); p is 0 there, and 0 * NaN would poison
                // O, so zero those V rows before the P V product reads them
                const int stg = static_cast<int>(t % kGqaStages);
                unsigned char* vb =
                    smem + C::kOffKV + stg * C::kStageBytes + C::kAtoms * C::kKVAtomBytes;
                const int per_atom = (kTK - rows) * 8;  // 16-B units per atom
                for (int u = st; u < per_atom * C::kAtoms; u += kSoftmaxThreads) {
                    const int a = u / per_atom;
                    const int rem = u - a * per_atom;
                    *reinterpret_cast<uint4*>(vb + a * C::kKVAtomBytes +
                                              swz(rows + rem / 8, rem % 8)) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
            // the group's previous P V product (tile t - 2) read this P buffer
            // and wrote this O accumulator
            if (t >= 2) wait(&x.pv_done[grp], static_cast<uint32_t>(((t >> 1) - 1) & 1));
            fence_after();
            if (warp_active) {
                float sv[CW];
                float mt = kNegInf;
#pragma unroll
                for (int k = 0; k < CW; ++k) {
                    const int col = cb + k;
                    const float raw = __uint_as_float(sr[k]);
                    float v = p.slopes
                                  ? fmaf(raw, qscale2, slope2 * static_cast<float>(t0 + col - w.len + 1))
                                  : raw * qscale2;
                    v = (col < rows && active) ? v : kNegInf;
                    sv[k] = v;
                    mt = fmaxf(mt, v);
                }
                const bool need = active && (m_ref == kNegInf ? mt != kNegInf
                                                               : mt > m_ref + kRescaleThreshold);
                const float m_new = need ? fmaxf(m_ref, mt) : m_ref;
                const float factor = need ? rescale(m_ref, m_new) : 1.f;
                if (__any_sync(0xffffffffu, need && m_ref != kNegInf)) {
                    // O already holds earlier tiles of this piece: scale it
#pragma unroll 1
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t o[32];
                        const uint32_t oa = x.tmem + lane_addr + o_col + cc * 32;
                        tmem_ld32(oa, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int y = 0; y < 32; ++y)
                            o[y] = __float_as_uint(__uint_as_float(o[y]) * factor);
                        tmem_st32(oa, o);
                    }
                    tmem_wait_st();
                }
                l *= factor;
                lx *= factor;
                m_ref = m_new;
                if (active) {
                    unsigned char* prow = smem + C::kOffP + grp * C::kPBytes;
#pragma unroll
                    for (int cc = 0; cc < CW / 8; ++cc) {
                        float ev[8];
                        uint32_t w4[4];
                        float lsum = 0.f, xsum = 0.f;
#pragma unroll
                        for (int y = 0; y < 8; ++y) {
                            // masked keys give 0, also while the row has no finite max yet
                            const float sk = sv[cc * 8 + y];
                            ev[y] = sk == kNegInf ? 0.f : ex2(sk - m_ref);
                            xsum += ev[y];
                        }
#pragma unroll
                        for (int y = 0; y < 4; ++y) {
                            float ra, rb;
                            w4[y] = pack_round(ev[2 * y], ev[2 * y + 1], kBF16, ra, rb);
                            lsum += ra + rb;
                        }
                        l += lsum;
                        lx += xsum;
                        *reinterpret_cast<uint4*>(prow + swz(r, cb / 8 + cc)) =
                            make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                }
                fence_proxy_async_smem();
            }
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&x.p_full[grp]));
        }

        // ---- end of piece: the group's last P V product must be complete
        if (last_own >= 0 && warp_active) {
            wait(&x.pv_done[grp], static_cast<uint32_t>((last_own >> 1) & 1));
            fence_after();
        }
        if (grp == 1) {
            // hand this group's row state to group 0, which merges and writes
            if (active) {
                stats1[r * 3 + 0] = m_ref;
                stats1[r * 3 + 1] = l;
                stats1[r * 3 + 2] = lx;
            }
            fence_before();
            named_bar_sync(kBarGroups, 2 * kSoftmaxThreads);
        } else {
            named_bar_sync(kBarGroups, 2 * kSoftmaxThreads);
            fence_after();
            // this row's state over both groups
            float m1 = kNegInf, l1 = 0.f, lx1 = 0.f;
            if (active) {
                m1 = stats1[r * 3 + 0];
                l1 = stats1[r * 3 + 1];
                lx1 = stats1[r * 3 + 2];
            }
            const float Mr = fmaxf(m_ref, m1);
            const float w0 = rescale(m_ref, Mr), w1 = rescale(m1, Mr);
            const bool use1 = m1 != kNegInf;  // group 1's O holds this piece's tiles
            const bool any1 = __any_sync(0xffffffffu, active && use1);
            float M = Mr, L = w0 * l + w1 * l1, LX = w0 * lx + w1 * lx1, wgt = 1.f;
            if constexpr (R > 1) {
                named_bar_sync(kBarSoftmax, kSoftmaxThreads);
                if (active) {
                    stats[r * 3 + 0] = M;
                    stats[r * 3 + 1] = L;
                    stats[r * 3 + 2] = LX;
                }
                named_bar_sync(kBarSoftmax, kSoftmaxThreads);
                if (active) {
                    M = kNegInf;
#pragma unroll
                    for (int j = 0; j < R; ++j) M = fmaxf(M, stats[(j * RR + g) * 3]);
                    L = 0.f;
                    LX = 0.f;
#pragma unroll
                    for (int j = 0; j < R; ++j) {
                        const float wj = rescale(stats[(j * RR + g) * 3], M);
                        L += wj * stats[(j * RR + g) * 3 + 1];
                        LX += wj * stats[(j * RR + g) * 3 + 2];
                    }
                    wgt = rescale(Mr, M);
                }
            }
            const int slot = pc == 0 ? 0 : 1;  // the CTA's first piece uses slot 0
            const bool writer = active && rep == 0;
            float* rec =
                (!whole && writer) ? p.part + ((x.c * 2 + slot) * G + g) * (D + 3) : nullptr;
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                if (warp_active) {
                    uint32_t o1[32];
                    tmem_ld32(x.tmem + lane_addr + 128 + cc * 32, o);
                    if (any1) tmem_ld32(x.tmem + lane_addr + 256 + cc * 32, o1);
                    tmem_wait_ld();
#pragma unroll
                    for (int y = 0; y < 32; ++y) {
                        float v = __uint_as_float(o[y]) * w0;
                        if (any1 && use1) v = fmaf(w1, __uint_as_float(o1[y]), v);
                        o[y] = __float_as_uint(v);
                    }
                }
                if constexpr (R > 1) {
                    if (active)
#pragma unroll
                        for (int y = 0; y < 32; ++y) stage[r * 33 + y] = __uint_as_float(o[y]) * wgt;
                    named_bar_sync(kBarSoftmax, kSoftmaxThreads);
                    if (writer)
#pragma unroll
                        for (int y = 0; y < 32; ++y) {
                            float a = 0.f;
#pragma unroll
                            for (int j = 0; j < R; ++j) a += stage[(j * RR + g) * 33 + y];
                            o[y] = __float_as_uint(a);
                        }
                    named_bar_sync(kBarSoftmax, kSoftmaxThreads);
                }
                if (writer) {
                    if (whole) {
                        float* dst = p.out + qrow * D + cc * 32;
#pragma unroll
                        for (int y = 0; y < 32; ++y) dst[y] = __uint_as_float(o[y]) / L;
                    } else {
#pragma unroll
                        for (int y = 0; y < 32; ++y) rec[cc * 32 + y] = __uint_as_float(o[y]);
                    }
                }
            }
            if (writer) {
                if (whole) {
                    if (p.lse) p.lse[qrow] = (M + log2f(LX)) * kLn2;
                } else {
                    rec[D] = M;
                    rec[D + 1] = L;
                    rec[D + 2] = LX;
                }
            }
            fence_before();
            if (!p.fused_merge) {
                // the CTA holding the sequence's first key describes its parts for
                // the combine kernel (one part: already written, nothing to merge)
                if (j0 == 0 && st == 0) {
                    const long long seg = static_cast<long long>(w.b) * p.Hkv + w.h;
                    const long long c_lo = gpart_of(w.start, x.T, x.P);
                    const long long c_hi = gpart_of(w.start + w.len - 1, x.T, x.P);
                    p.seg_desc[seg * 3 + 0] = static_cast<int>(c_lo);
                    p.seg_desc[seg * 3 + 1] = static_cast<int>(c_hi - c_lo + 1);
                    p.seg_desc[seg * 3 + 2] = gpart_start(c_lo, x.T, x.P) < w.start ? 1 : 0;
                }
            } else if (!whole) {
                __threadfence();
                named_bar_sync(kBarSoftmax, kSoftmaxThreads);
                const long long c_lo = gpart_of(w.start, x.T, x.P);
                const long long c_hi = gpart_of(w.start + w.len - 1, x.T, x.P);
                const int n = static_cast<int>(c_hi - c_lo + 1);
                const long long seg = static_cast<long long>(w.b) * p.Hkv + w.h;
                if (st == 0) {
                    const int prev = atomicAdd(p.tickets + seg, 1);
                    const int last = prev == n - 1;
                    if (last) atomicExch(p.tickets + seg, 0);
                    x.ctl->last = last;
                }
                named_bar_sync(kBarSoftmax, kSoftmaxThreads);
                if (x.ctl->last) {
                    __threadfence();
                    const int first_slot = gpart_start(c_lo, x.T, x.P) < w.start ? 1 : 0;
                    for (int gg = 0; gg < G; ++gg) {
                        const long long orow = static_cast<long long>(w.b) * p.Hq +
                                               static_cast<long long>(w.h) * G + gg;
                        const GSlotAcc acc{p.part, c_lo, first_slot, G, gg, D};
                        tree_merge(acc, n, D, st, kSoftmaxThreads, x.scratch, kScratchFloats,
                                   kBarSoftmax, p.out + orow * D, p.lse ? p.lse + orow : nullptr);
                    }
                }
            }
            named_bar_sync(kBarSoftmax, kSoftmaxThreads);
        }
        ++pc;
    } while (gwalk_next(p, *x.ctl, w));
}

template <typename E, int D, int CW>
__global__ void __launch_bounds__(kGqaThreads, 1)
    td_gqa_kernel(const GqaParams p, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV) {
    using C = GCfg<D>;
    constexpr bool kBF16 = std::is_same<E, __nv_bfloat16>::value;
    extern __shared__ unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled operand blocks
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* scratch = reinterpret_cast<float*>(smem + C::kOffScratch);

    __shared__ __align__(8) uint64_t kv_full[kGqaStages], kv_empty[kGqaStages];
    __shared__ __align__(8) uint64_t s_full[2], s_empty[2], p_full[2], pv_done[2], q_ready;
    __shared__ GCtl ctl;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long c = blockIdx.x;
    const long long P = p.P;

    if (tid == 0) {
        for (int s = 0; s < kGqaStages; ++s) {
            mbar_init(smem_addr(&kv_full[s]), 1);
            mbar_init(smem_addr(&kv_empty[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&s_full[s]), 1);
            mbar_init(smem_addr(&s_empty[s]), 4);
            mbar_init(smem_addr(&p_full[s]), 4);
            mbar_init(smem_addr(&pv_done[s]), 1);
        }
        mbar_init(smem_addr(&q_ready), 8);
        fence_barrier_init();
        ctl.abort = 0;
        ctl.last = 0;
    }
    if (warp == 1) {
        // TMEM: 256 columns, address written to ctl.tmem
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_addr(&ctl.tmem)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (warp >= 2) {
        // Q and both P buffers start at zero (rows >= G stay zero)
        uint4* z = reinterpret_cast<uint4*>(smem + C::kOffQ);
        const int n16 = (C::kQBytes + 2 * C::kPBytes) / 16;
        for (int i = tid - 64; i < n16; i += kGqaThreads - 64) z[i] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
    }
    gqa_partition(p, ctl, c, tid, warp, lane, kGqaThreads, D);
    fence_before();
    __syncthreads();
    fence_after();

    const long long T = ctl.T, x0 = ctl.x0, x1 = ctl.x1;
    const uint32_t tmem = ctl.tmem;
    volatile int* abort_flag = &ctl.abort;
    const uint32_t sQ = smem_addr(smem + C::kOffQ);
    const uint32_t sP = smem_addr(smem + C::kOffP);
    const uint32_t sKV = smem_addr(smem + C::kOffKV);

    if (warp == 0) {
        // -------------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool aborted = false;
            GWalk w;
            if (gwalk_first(p, ctl, w)) {
                do {
                    const long long j0 = (x0 > w.start ? x0 : w.start) - w.start;
                    const long long e = w.start + w.len;
                    const long long j1 = (x1 < e ? x1 : e) - w.start;
                    const long long rowbase = (static_cast<long long>(w.b) * p.Hkv + w.h) * p.N;
                    for (long long t0 = j0; t0 < j1; t0 += kTK) {
                        if (!aborted &&
                            !mbar_wait_bounded(smem_addr(&kv_empty[stage]), phase ^ 1u, abort_flag,
                                               p.err, TD_DEVERR_WAIT_TIMEOUT))
                            aborted = true;
                        if (!aborted) {
                            const uint32_t fb = smem_addr(&kv_full[stage]);
                            const uint32_t base = sKV + stage * C::kStageBytes;
                            const int y = static_cast<int>(rowbase + t0);
                            mbar_arrive_expect_tx(fb, C::kStageBytes);
#pragma unroll
                            for (int a = 0; a < C::kAtoms; ++a) {
                                tma_load_2d(base + a * C::kKVAtomBytes, &tmK, 64 * a, y, fb, pol);
                                tma_load_2d(base + (C::kAtoms + a) * C::kKVAtomBytes, &tmV, 64 * a,
                                            y, fb, pol);
                            }
                            ++issued;
                        }
                        if (++stage == kGqaStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                } while (gwalk_next(p, ctl, w));
            }
            for (int s = 0; s < kGqaStages && s < issued; ++s) {
                const long long lastTile = s + ((issued - 1 - s) / kGqaStages) * kGqaStages;
                mbar_wait_bounded(smem_addr(&kv_full[s]),
                                  static_cast<uint32_t>((lastTile / kGqaStages) & 1), nullptr,
                                  p.err, TD_DEVERR_WAIT_TIMEOUT);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idS = instr_desc_f16(kBF16 ? 1 : 0, kM, kTK, 0, 0);
            constexpr uint32_t idO = instr_desc_f16(kBF16 ? 1 : 0, kM, D, 0, 1);
            long long t = 0;    // tiles issued so far (global)
            long long pc = 0;   // pieces so far
            bool aborted = false;
            long long last_pv = -1;
            auto wait = [&](uint64_t* bar, uint32_t par) {
                if (!aborted && !mbar_wait_bounded(smem_addr(bar), par, abort_flag, p.err,
                                                   TD_DEVERR_WAIT_TIMEOUT))
                    aborted = true;
            };
            auto issue_S = [&](long long tt) {
                const int stage = static_cast<int>(tt % kGqaStages);
                wait(&kv_full[stage], static_cast<uint32_t>((tt / kGqaStages) & 1));
                if (tt >= 2) wait(&s_empty[tt & 1], static_cast<uint32_t>(((tt >> 1) - 1) & 1));
                fence_after();
                const uint32_t kb = sKV + stage * C::kStageBytes;
                const uint32_t dS = tmem + static_cast<uint32_t>((tt & 1) * kTK);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = static_cast<uint32_t>((kk & 3) * 32);  // 16 cols in the atom
                    const uint64_t a = smem_desc_sw128(sQ + (kk >> 2) * (kM * 128) + off, 16, 1024);
                    const uint64_t b = smem_desc_sw128(kb + (kk >> 2) * C::kKVAtomBytes + off, 16, 1024);
                    umma_f16(dS, a, b, idS, kk > 0 ? 1u : 0u);
                }
                umma_commit(smem_addr(&s_full[tt & 1]));
            };
            GWalk w;
            if (gwalk_first(p, ctl, w)) {
                do {
                    const long long j0 = (x0 > w.start ? x0 : w.start) - w.start;
                    const long long e = w.start + w.len;
                    const long long j1 = (x1 < e ? x1 : e) - w.start;
                    const long long nt = (j1 - j0 + kTK - 1) / kTK;
                    wait(&q_ready, static_cast<uint32_t>(pc & 1));
                    fence_after();
                    // Event loop over this piece's tiles: S products are issued in
                    // order as soon as their K tile has landed and their S buffer is
                    // free; P V products in order as soon as their P is written.  The
                    // two streams interleave, so neither softmax group waits for the
                    // other's P before its next S is issued.
                    const long long t_end = t + nt;
                    long long ts = t;   // next S to issue
                    long long tp = t;   // next P V to issue
                    uint64_t t_stall = 0;   // when the current stall began (0: none)
                    uint32_t spins = 0;
                    while (tp < t_end && !aborted) {
                        bool progressed = false;
                        if (ts < t_end &&
                            mbar_test(smem_addr(&kv_full[ts % kGqaStages]),
                                      static_cast<uint32_t>((ts / kGqaStages) & 1)) &&
                            (ts < 2 || mbar_test(smem_addr(&s_empty[ts & 1]),
                                                 static_cast<uint32_t>(((ts >> 1) - 1) & 1)))) {
                            issue_S(ts);
                            ++ts;
                            progressed = true;
                        }
                        if (tp < ts && mbar_test(smem_addr(&p_full[tp & 1]),
                                                 static_cast<uint32_t>((tp >> 1) & 1))) {
                            fence_after();
                            const long long i = tp - t;
                            const int stage = static_cast<int>(tp % kGqaStages);
                            const uint32_t vb =
                                sKV + stage * C::kStageBytes + C::kAtoms * C::kKVAtomBytes;
                            const uint32_t pb = sP + static_cast<uint32_t>((tp & 1) * C::kPBytes);
                            const uint32_t dO = tmem + 128 + static_cast<uint32_t>((tp & 1) * 128);
#pragma unroll
                            for (int kk = 0; kk < kTK / 16; ++kk) {
                                const uint64_t a = smem_desc_sw128(pb + kk * 32, 16, 1024);
                                const uint64_t b =
                                    smem_desc_sw128(vb + kk * 2048, C::kKVAtomBytes, 1024);
                                // each group's first tile of the piece starts its accumulator
                                umma_f16(dO, a, b, idO, (i > 1 || kk > 0) ? 1u : 0u);
                            }
                            umma_commit(smem_addr(&pv_done[tp & 1]));
                            umma_commit(smem_addr(&kv_empty[stage]));
                            last_pv = tp;
                            ++tp;
                            progressed = true;
                        }
                        if (progressed) {
                            spins = 0;
                            t_stall = 0;
                        } else if ((++spins & 255u) == 0u) {
                            const uint64_t now = global_timer_ns();
                            if (t_stall == 0) t_stall = now;
                            if (*abort_flag) aborted = true;
                            else if (now - t_stall > kWaitLimitNs) {
                                atomicOr(p.err, TD_DEVERR_WAIT_TIMEOUT);
                                *abort_flag = 1;
                                aborted = true;
                            }
                        }
                    }
                    t = t_end;
                    ++pc;
                } while (gwalk_next(p, ctl, w));
            }
            // every MMA must be complete before the CTA frees TMEM
            for (long long tl = last_pv - 1; tl <= last_pv; ++tl)
                if (tl >= 0)
                    mbar_wait_bounded(smem_addr(&pv_done[tl & 1]),
                                      static_cast<uint32_t>((tl >> 1) & 1), nullptr, p.err,
                                      TD_DEVERR_WAIT_TIMEOUT);
        }
        __syncwarp();
    } else {
        // --------------------------------------------------------- softmax
        const SmCtx sx{smem, scratch, s_full, s_empty, p_full, pv_done, &q_ready, &ctl, abort_flag,
                       tmem, T, x0, x1, P, c, warp, lane, tid};
        softmax_role<E, D, CW>(p, sx);
    }

    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols) : "memory");
    }
}

template <typename E, int D, int CW>
cudaError_t launch_gqa_t(int device, const GqaParams& p, const CUtensorMap& mk,
                         const CUtensorMap& mv, cudaStream_t s) {
    using C = GCfg<D>;
    auto kern = td_gqa_kernel<E, D, CW>;
    static std::atomic<unsigned long long> configured{0};
    const unsigned long long bit = device < 64 ? (1ull << device) : 0ull;
    if (!bit || !(configured.load(std::memory_order_acquire) & bit)) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::kSmem));
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    kern<<<static_cast<unsigned>(p.P), kGqaThreads, C::kSmem, s>>>(p, mk, mv);
    return cudaGetLastError();
}


template <typename E, int D>
cudaError_t launch_gqa_g(int device, const GqaParams& p, const CUtensorMap& mk,
                         const CUtensorMap& mv, cudaStream_t s) {
    // key columns per replica of the query rows: 4 replicas while G fits a
    // TMEM lane quarter, 2 while it fits half, else 1
    if (p.G <= 32) return launch_gqa_t<E, D, 16>(device, p, mk, mv, s);
    if (p.G <= 64) return launch_gqa_t<E, D, 32>(device, p, mk, mv, s);
    return launch_gqa_t<E, D, 64>(device, p, mk, mv, s);
}

}  // namespace

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

size_t gqa_smem_bytes(int D) {
    return D == 64 ? GCfg<64>::kSmem : D == 128 ? GCfg<128>::kSmem : 0;
}

cudaError_t launch_gqa(int device, int dtype, int D, const GqaParams& p, const CUtensorMap& mk,
                       const CUtensorMap& mv, cudaStream_t s) {
    if (dtype == kBF16) {
        if (D == 64) return launch_gqa_g<__nv_bfloat16, 64>(device, p, mk, mv, s);
        if (D == 128) return launch_gqa_g<__nv_bfloat16, 128>(device, p, mk, mv, s);
    } else if (dtype == kF16) {
        if (D == 64) return launch_gqa_g<__half, 64>(device, p, mk, mv, s);
        if (D == 128) return launch_gqa_g<__half, 128>(device, p, mk, mv, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace td
