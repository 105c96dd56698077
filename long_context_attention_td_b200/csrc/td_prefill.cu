// td_prefill -- causal (or full) prefill attention on the sm_100a tensor cores.
//
// What it computes (every query row i of every (b, h) sequence of S tokens):
//     s_ij  = q_i . k_j D^-1/2 + slope_h (j - S + 1)     for j in J(i),
//     out_i = sum_j e^(s_ij - m_i) v_j / sum_j e^(s_ij - m_i),  lse_i = m_i + ln sum,
// with J(i) = {0..i} when causal, else every key: the ALiBi broadcast row and
// causal mask of "ALiBi with causal=True unexpected bias?", computed blockwise
// as "Flash Aandacht" describes it -- running max m, running sum l and output O
// per query row over key blocks, the normalised O rescaled by its old sum
// before each update (the listing as printed leaves that factor out).
//
// One CTA per (b, h, pair of adjacent 128-row query tiles); the heaviest causal
// pairs are scheduled first.  Every K and V tile of 128 keys that the CTA loads
// serves both query tiles g = 0, 1:
//     S_g [128 q x 128 k] = Q_g [128 x D] . K^T       (D/16 tcgen05.mma, N = 128)
//     O_g [128 q x D]    += P_g [128 x 128] . V       (8 tcgen05.mma, N = D)
// S_g and O_g are fp32 in TMEM.  P_g, rounded to the input type, is written
// back over the first 64 columns of S_g (two 16-bit values per column, key k in
// column k/2) and read from there as the A operand of P V, so the shared memory
// holds only Q, K and V.  The MMAs of one CTA run in the order they are issued,
// so S_g of the next tile, issued after P_g V, cannot overwrite P_g before that
// product has read it; and the completion of S_g (its commit) means every
// earlier product of group g, P_g V of the previous tile included, is done.
// Each softmax thread owns one query row (its TMEM lane): its running max and
// sums need no cross-thread reduction; its O row is rescaled in TMEM when the
// row's max grows by more than 8 (log2 units).
//
// 12 warps in three warpgroups: warpgroup 0 -- warp 0 loads Q and K, warp 2
// loads V (3-D boxes of {64 columns, 128 rows, 1 sequence}; 2 K and 3 V
// stages), warp 1 owns TMEM and issues the MMAs as their inputs become
// ready, warp 3 idles; warpgroup 1 is
// the softmax of query tile 0, warpgroup 2 that of query tile 1 (warp w reads
// TMEM lanes 32 (w % 4) .. + 31).
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

constexpr int kPQ = 128;             // query rows per tile (MMA M)
constexpr int kPK = 128;             // keys per tile (MMA N of S)
constexpr int kPThreads = 384;       // 12 warps (two softmax warpgroups)
// register split (setmaxnreg): warpgroup 0 (loads, MMA, one idle warp) drops
// to kRegLow, the softmax warpgroups rise to kRegHigh; 4*32*kRegLow +
// 8*32*kRegHigh must not exceed the 384 x 168 registers the block is launched
// with, or the increase would wait for ever
constexpr int kRegLow = 64;
constexpr int kRegHigh = 216;
static_assert(4 * 32 * kRegLow + 8 * 32 * kRegHigh <= kPThreads * 168, "register split");
constexpr int kKStages = 2;          // K ring depth
constexpr int kVStages = 3;          // V ring depth (its stage is held until P V is done)
constexpr int kPTmemCols = 512;      // S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D)
constexpr float kPRescale = 8.f;     // log2 units

template <int D>
struct PCfg {
    static constexpr int kAtoms = D / 64;                 // 64-column swizzle atoms of D
    static constexpr int kRowAtom = 128 * 128;            // 128 rows x 64 columns, 16 KB
    static constexpr int kTileBytes = kAtoms * kRowAtom;  // one 128-row tile of Q, K or V
    static constexpr int kOffQ = 0;                       // Q_0, Q_1
    static constexpr int kOffK = 2 * kTileBytes;
    static constexpr int kOffV = kOffK + kKStages * kTileBytes;
    static constexpr int kOffRamp = kOffV + kVStages * kTileBytes;  // ALiBi slope * c, 128 floats
    static constexpr size_t kSmem = size_t(kOffRamp) + kPK * 4 + 1024;  // +align
    static_assert(D == 64 || D == 128, "D");
    static_assert(kSmem <= 232448 - 256, "shared memory");
};

// 3-D tiled TMA load of a box {64 columns, 128 rows, 1 sequence} (no multicast)
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            int z, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16, one CTA: A is M = 128 lanes
// by K = 16 elements held as 8 columns of two 16-bit values (element k in
// column k / 2, the even element in the low half)
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// mbarrier phase test that may suspend the thread for up to `ns` nanoseconds
// while the phase is incomplete (frees the issue slots a polling thread takes)
__device__ __forceinline__ bool mbar_try_wait_ns(uint32_t bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// max of three (one instruction on sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

struct PCtl {
    int abort;
    uint32_t tmem;
};

// ---------------------------------------------- packed fp32 pairs (f32x2)

__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}


template <typename E, int D>
__global__ void __launch_bounds__(kPThreads, 1)
    td_prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV) {
    using C = PCfg<D>;
    constexpr bool kBF16 = std::is_same<E, __nv_bfloat16>::value;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    __shared__ __align__(8) uint64_t k_full[kKStages], k_empty[kKStages];
    __shared__ __align__(8) uint64_t v_full[kVStages], v_empty[kVStages];
    __shared__ __align__(8) uint64_t q_full, s_full[2], p_full[2], o_done[2], mma_done;
    __shared__ PCtl ctl;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Sequences are taken in groups of hg whose K and V together fill about
    // 32 MB, so the query tiles in flight share key tiles in L2; inside a
    // group the heaviest causal pairs go first (the group's last pair of query
    // tiles of every sequence, then the one before, ...), which keeps the tail
    // short.
    const long long BH = static_cast<long long>(p.B) * p.H;
    const long long nqt = (p.S + kPQ - 1) / kPQ;
    const long long npair = (nqt + 1) / 2;
    const long long kv_bytes = static_cast<long long>(p.S) * D * 2 * static_cast<long long>(sizeof(E));
    long long hg = (32ll << 20) / kv_bytes;
    hg = hg < 1 ? 1 : (hg > BH ? BH : hg);
    const long long grp0 = (static_cast<long long>(blockIdx.x) / (hg * npair)) * hg;
    const long long hcnt = BH - grp0 < hg ? BH - grp0 : hg;
    const long long idx = static_cast<long long>(blockIdx.x) - grp0 * npair;
    const long long bh = grp0 + idx % hcnt;
    const long long pair = npair - 1 - idx / hcnt;
    const long long nkt_all = (p.S + kPK - 1) / kPK;
    static_assert(kPQ == kPK, "causal tile count assumes square tiles");
    // query tile of each group, and the key tiles it reads (0: no such tile)
    const long long qt0 = 2 * pair, qt1 = 2 * pair + 1;
    const long long n0 = p.causal ? (qt0 + 1 < nkt_all ? qt0 + 1 : nkt_all) : nkt_all;
    const long long n1 = qt1 >= nqt ? 0 : (p.causal ? (qt1 + 1 < nkt_all ? qt1 + 1 : nkt_all)
                                                    : nkt_all);
    const long long nt = n0 > n1 ? n0 : n1;

    if (tid == 0) {
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(smem_addr(&k_full[s]), 1);
            mbar_init(smem_addr(&k_empty[s]), 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(smem_addr(&v_full[s]), 1);
            mbar_init(smem_addr(&v_empty[s]), 1);
        }
        mbar_init(smem_addr(&q_full), 1);
        for (int g = 0; g < 2; ++g) {
            mbar_init(smem_addr(&s_full[g]), 1);
            mbar_init(smem_addr(&p_full[g]), 4);   // one arrival per softmax warp
            mbar_init(smem_addr(&o_done[g]), 1);
        }
        mbar_init(smem_addr(&mma_done), 1);
        fence_barrier_init();
        ctl.abort = 0;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_addr(&ctl.tmem)), "r"(kPTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid >= 128 && tid < 128 + kPK) {
        // the ALiBi ramp slope_h c (log2 units) of key c of a tile, zero without
        // a bias; the tile's offset slope_h (j0 - S + 1) is added to the row's
        // running max instead
        reinterpret_cast<float*>(smem + C::kOffRamp)[tid - 128] =
            p.slopes ? __ldg(p.slopes + (bh % p.H)) * kLog2e * static_cast<float>(tid - 128)
                     : 0.f;
    }
    fence_before();
    __syncthreads();
    fence_after();

    const uint32_t tmem = ctl.tmem;
    volatile int* abort_flag = &ctl.abort;
    constexpr int kSoft0 = 4;  // first softmax warp
    const uint32_t sQ = smem_addr(smem + C::kOffQ);
    const uint32_t sK = smem_addr(smem + C::kOffK);
    const uint32_t sV = smem_addr(smem + C::kOffV);
    const int z = static_cast<int>(bh);

    if (warp < kSoft0) {
    // each warpgroup's register change heads its branch, so the code of the
    // branch is compiled for that register count
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegLow));
    if (warp == 0 || warp == 2) {
        // -------------------------------------------------------- loaders
        // warp 0: Q and K; warp 2: V -- a K load never waits behind a V stage
        // still held by a P V product
        if (lane == 0) {
            const bool doK = warp == 0;
            const int nst = doK ? kKStages : kVStages;
            uint64_t* full = doK ? k_full : v_full;
            uint64_t* empty = doK ? k_empty : v_empty;
            const CUtensorMap* map = doK ? &tmK : &tmV;
            const uint32_t ring = doK ? sK : sV;
            bool aborted = false;
            if (doK) {
                const uint32_t qb = smem_addr(&q_full);
                mbar_arrive_expect_tx(qb, (n1 > 0 ? 2 : 1) * C::kTileBytes);
#pragma unroll
                for (int a = 0; a < C::kAtoms; ++a) {
                    tma_load_3d(sQ + a * C::kRowAtom, &tmQ, 64 * a, static_cast<int>(qt0 * kPQ), z,
                                qb);
                    if (n1 > 0)
                        tma_load_3d(sQ + C::kTileBytes + a * C::kRowAtom, &tmQ, 64 * a,
                                    static_cast<int>(qt1 * kPQ), z, qb);
                }
            }
            long long issued = 0;
            for (long long t = 0; t < nt; ++t) {
                const int stage = static_cast<int>(t % nst);
                const uint32_t par = static_cast<uint32_t>((t / nst) & 1);
                if (!aborted && !mbar_wait_bounded(smem_addr(&empty[stage]), par ^ 1u, abort_flag,
                                                   p.err, TD_DEVERR_WAIT_TIMEOUT))
                    aborted = true;
                if (aborted) break;
                const uint32_t fb = smem_addr(&full[stage]);
                mbar_arrive_expect_tx(fb, C::kTileBytes);
#pragma unroll
                for (int a = 0; a < C::kAtoms; ++a)
                    tma_load_3d(ring + stage * C::kTileBytes + a * C::kRowAtom, map, 64 * a,
                                static_cast<int>(t * kPK), z, fb);
                ++issued;
            }
            // the CTA must not exit with copies into its shared memory in
            // flight: wait (bounded) for the last load issued on every stage
            if (doK)
                mbar_wait_bounded(smem_addr(&q_full), 0, nullptr, p.err, TD_DEVERR_WAIT_TIMEOUT);
            for (int s = 0; s < nst; ++s) {
                if (s >= issued) break;
                const long long lt = s + ((issued - 1 - s) / nst) * nst;
                mbar_wait_bounded(smem_addr(&full[s]), static_cast<uint32_t>((lt / nst) & 1),
                                  nullptr, p.err, TD_DEVERR_WAIT_TIMEOUT);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idS = instr_desc_f16(kBF16 ? 1 : 0, kPQ, kPK, 0, 0);
            constexpr uint32_t idO = instr_desc_f16(kBF16 ? 1 : 0, kPQ, D, 0, 1);
            bool aborted = false;
            // S_g of key tile t into TMEM columns [128 g, 128 g + 128)
            auto issue_s = [&](int g, int t) {
                const int stage = static_cast<int>(t % kKStages);
                const uint32_t kb = sK + stage * C::kTileBytes;
                const uint32_t qb = sQ + g * C::kTileBytes;
                const uint32_t dS = tmem + static_cast<uint32_t>(g * kPK);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = static_cast<uint32_t>((kk & 3) * 32);
                    const uint64_t a = smem_desc_sw128(qb + (kk >> 2) * C::kRowAtom + off, 16, 1024);
                    const uint64_t b = smem_desc_sw128(kb + (kk >> 2) * C::kRowAtom + off, 16, 1024);
                    umma_f16(dS, a, b, idS, kk > 0 ? 1u : 0u);
                }
                umma_commit(smem_addr(&s_full[g]));
            };
            // O_g += P_g V of key tile t, P_g from TMEM columns [128 g, 128 g + 64)
            auto issue_pv = [&](int g, int t) {
                const int stage = static_cast<int>(t % kVStages);
                const uint32_t vb = sV + stage * C::kTileBytes;
                const uint32_t pa = tmem + static_cast<uint32_t>(g * kPK);
                const uint32_t dO = tmem + static_cast<uint32_t>(2 * kPK + g * D);
#pragma unroll
                for (int kk = 0; kk < kPK / 16; ++kk) {
                    // V: 16 keys, all D columns (two 64-column halves kRowAtom apart)
                    const uint64_t b = smem_desc_sw128(vb + kk * 2048, C::kRowAtom, 1024);
                    umma_f16_tmem_a(dO, pa + static_cast<uint32_t>(kk * 8), b, idO,
                                    (t > 0 || kk > 0) ? 1u : 0u);
                }
                if (t == static_cast<int>(g == 0 ? n0 : n1) - 1) umma_commit(smem_addr(&o_done[g]));
            };
            // Event loop: each group's products go out as soon as their inputs
            // are ready, so neither softmax group waits behind the other's.
            // S_g(t) follows P_g V(t - 1) (it overwrites P_g); P_g V(t) needs
            // P_g(t) written and V(t) landed.  A K (V) stage is released after
            // its last user: (t < n0) + (t < n1) products read tile t.
            if (mbar_wait_bounded(smem_addr(&q_full), 0, abort_flag, p.err,
                                  TD_DEVERR_WAIT_TIMEOUT)) {
                fence_after();
                // tile counters fit 32 bits (S < 2^31 keys)
                const int ngr[2] = {static_cast<int>(n0), static_cast<int>(n1)};
                int ts[2] = {0, 0}, tp[2] = {0, 0};
                // products issued so far on each stage's current tile, 2 bits a stage
                uint32_t kuse = 0, vuse = 0;
                static_assert(kKStages <= 16 && kVStages <= 16, "stage use counters");
                uint64_t t_stall = 0;
                uint32_t spins = 0;
                while (!aborted && (tp[0] < ngr[0] || tp[1] < ngr[1])) {
                    bool progressed = false;
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        if (tp[g] < ts[g]) {
                            const int t = tp[g];
                            const int vst = static_cast<int>(t % kVStages);
                            if (mbar_test(smem_addr(&p_full[g]), static_cast<uint32_t>(t & 1)) &&
                                mbar_test(smem_addr(&v_full[vst]),
                                          static_cast<uint32_t>((t / kVStages) & 1))) {
                                fence_after();
                                issue_pv(g, t);
                                const uint32_t sh = 2u * static_cast<uint32_t>(vst);
                                const uint32_t u = ((vuse >> sh) & 3u) + 1u;
                                if (u == static_cast<uint32_t>((t < ngr[0]) + (t < ngr[1]))) {
                                    vuse &= ~(3u << sh);
                                    umma_commit(smem_addr(&v_empty[vst]));
                                } else {
                                    vuse = (vuse & ~(3u << sh)) | (u << sh);
                                }
                                ++tp[g];
                                progressed = true;
                            }
                        }
                        if (ts[g] < ngr[g] && ts[g] == tp[g]) {
                            const int t = ts[g];
                            const int kst = static_cast<int>(t % kKStages);
                            if (mbar_test(smem_addr(&k_full[kst]),
                                          static_cast<uint32_t>((t / kKStages) & 1))) {
                                fence_after();
                                issue_s(g, t);
                                const uint32_t sh = 2u * static_cast<uint32_t>(kst);
                                const uint32_t u = ((kuse >> sh) & 3u) + 1u;
                                if (u == static_cast<uint32_t>((t < ngr[0]) + (t < ngr[1]))) {
                                    kuse &= ~(3u << sh);
                                    umma_commit(smem_addr(&k_empty[kst]));
                                } else {
                                    kuse = (kuse & ~(3u << sh)) | (u << sh);
                                }
                                ++ts[g];
                                progressed = true;
                            }
                        }
                    }
                    if (progressed) {
                        spins = 0;
                        t_stall = 0;
                        continue;
                    }
                    // nothing ready: suspend briefly on the P of the group whose
                    // product is oldest (or on the next K tile), then check the
                    // time limit and the abort flag
                    const bool w0 = tp[0] < ts[0], w1 = tp[1] < ts[1];
                    if (w0 || w1) {
                        const bool first0 = w0 && (!w1 || tp[0] <= tp[1]);
                        const int tw = first0 ? tp[0] : tp[1];
                        mbar_try_wait_ns(smem_addr(first0 ? &p_full[0] : &p_full[1]),
                                         static_cast<uint32_t>(tw & 1), 100);
                    }
                    if ((++spins & 31u) == 0u) {
                        const uint64_t now = global_timer_ns();
                        if (t_stall == 0) t_stall = now;
                        if (*abort_flag) {
                            aborted = true;
                        } else if (now - t_stall > kWaitLimitNs) {
                            atomicOr(p.err, TD_DEVERR_WAIT_TIMEOUT);
                            *abort_flag = 1;
                            aborted = true;
                        }
                    }
                }
            }
            // every MMA issued must be complete before the CTA frees TMEM
            umma_commit(smem_addr(&mma_done));
            mbar_wait_bounded(smem_addr(&mma_done), 0, nullptr, p.err, TD_DEVERR_WAIT_TIMEOUT);
        }
        __syncwarp();
    }
    } else {
        // --------------------------------------------------------- softmax
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegHigh));
        const int g = (warp - kSoft0) >> 2;           // query tile of this group
        const long long ng = g == 0 ? n0 : n1;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;            // query row of the tile (TMEM lane)
        const long long i = (g == 0 ? qt0 : qt1) * kPQ + r;  // query index in the sequence
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t s_col = static_cast<uint32_t>(g * kPK);
        const uint32_t o_col = static_cast<uint32_t>(2 * kPK + g * D);
        const float qscale2 = p.qscale2;
        const float slope2 = p.slopes ? __ldg(p.slopes + (bh % p.H)) * kLog2e : 0.f;
        bool aborted = false;
        auto wait = [&](uint64_t* bar, uint32_t par) {
            if (!aborted && !mbar_wait_bounded(smem_addr(bar), par, abort_flag, p.err,
                                               TD_DEVERR_WAIT_TIMEOUT))
                aborted = true;
        };
        float m = kNegInf, thr = kNegInf, lx = 0.f;
        // key indices fit 32 bits (the host keeps S + 256 < 2^31)
        const int jmax = static_cast<int>(p.causal ? (i < p.S - 1 ? i : p.S - 1) : p.S - 1);
        const int S1 = static_cast<int>(p.S - 1);
        for (long long t = 0; t < ng; ++t) {
            wait(&s_full[g], static_cast<uint32_t>(t & 1));
            fence_after();
            uint32_t sr[kPK];
#pragma unroll
            for (int c = 0; c < kPK / 32; ++c)
                tmem_ld32(tmem + lane_addr + s_col + static_cast<uint32_t>(32 * c),
                          *reinterpret_cast<uint32_t(*)[32]>(sr + 32 * c));
            tmem_wait_ld();

            // scores in log2 units: x_c = raw_c qscale2 + slope2 (j0 + c - S + 1);
            // keys past the row's last visible key (causal) or past the
            // sequence end are -inf (every row sees key j0, so its max is
            // finite).  One code path serves every tile (a compact loop body
            // keeps the instruction stream in cache): a tile with every key
            // visible and no bias keeps the raw products in sr, takes the row
            // max on them (qscale2 > 0 keeps the order) and forms x_c - m with
            // one fma in the exponent loop; any other tile first rewrites sr as
            // x'_c = raw_c qscale2 + slope2 c (the ramp in shared memory, -inf
            // where masked), and the tile's offset ofs = slope2 (j0 - S + 1)
            // joins the max: x_c - m = x'_c - (m - ofs).  The max runs as 8
            // independent chains of three-input maxima.
            const int j0 = static_cast<int>(t) * kPK;
            const int cmax = jmax - j0 < kPK - 1 ? jmax - j0 : kPK - 1;
            const bool plain = p.slopes == nullptr && __all_sync(0xffffffffu, cmax == kPK - 1);
            const float ofs = slope2 * static_cast<float>(j0 - S1);
            if (!plain) {
                const float* ramp = reinterpret_cast<const float*>(smem + C::kOffRamp);
                const uint64_t sc2 = pk2(qscale2, qscale2);
#pragma unroll
                for (int c4 = 0; c4 < kPK; c4 += 4) {
                    const float4 b4 = *reinterpret_cast<const float4*>(ramp + c4);
                    float x[4];
                    upk2(fma2(pk2(__uint_as_float(sr[c4]), __uint_as_float(sr[c4 + 1])), sc2,
                              pk2(b4.x, b4.y)),
                         x[0], x[1]);
                    upk2(fma2(pk2(__uint_as_float(sr[c4 + 2]), __uint_as_float(sr[c4 + 3])), sc2,
                              pk2(b4.z, b4.w)),
                         x[2], x[3]);
#pragma unroll
                    for (int u = 0; u < 4; ++u) sr[c4 + u] = __float_as_uint(x[u]);
                }
                if (__any_sync(0xffffffffu, cmax < kPK - 1)) {
#pragma unroll
                    for (int c = 0; c < kPK; ++c)
                        if (c > cmax) sr[c] = __float_as_uint(kNegInf);
                }
            }
            float mx8[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) mx8[c] = __uint_as_float(sr[c]);
#pragma unroll
            for (int k = 1; k < 15; k += 2)
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    mx8[c] = fmax3(mx8[c], __uint_as_float(sr[c + 8 * k]),
                                   __uint_as_float(sr[c + 8 * (k + 1)]));
            // columns 120..127 join the final combination
            float mt = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                             fmax3(mx8[6], mx8[7],
                                   fmax3(__uint_as_float(sr[120]), __uint_as_float(sr[121]),
                                         __uint_as_float(sr[122]))));
            mt = fmax3(mt, fmax3(__uint_as_float(sr[123]), __uint_as_float(sr[124]),
                                 __uint_as_float(sr[125])),
                       fmaxf(__uint_as_float(sr[126]), __uint_as_float(sr[127])));
            mt = plain ? mt * qscale2 : mt + ofs;
            // move this row's max when the tile exceeds it by more than the
            // threshold (always on the first tile)
            const bool need = mt > thr;
            if (__any_sync(0xffffffffu, need && t >= 1)) {
                // O holds this group's earlier tiles, all complete (the commit
                // of S_g of this tile follows them): rescale this warp's rows
                const float f = need ? rescale(m, mt) : 1.f;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    const uint32_t oa = tmem + lane_addr + o_col + static_cast<uint32_t>(32 * c);
                    tmem_ld32(oa, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int y = 0; y < 32; ++y) o[y] = __float_as_uint(__uint_as_float(o[y]) * f);
                    tmem_st32(oa, o);
                }
            }
            if (need) {
                lx *= rescale(m, mt);
                m = mt;
                thr = mt + kPRescale;
            }
            // p rounded to the input type, two keys per 32-bit column, over the
            // first 64 columns of S_g, and the row sum over independent partials
            // (masked keys give ex2(-inf) = 0)
            uint64_t ls2[2] = {pk2(0.f, 0.f), pk2(0.f, 0.f)};
            {
                const float a = plain ? qscale2 : 1.f;
                const float b = plain ? -m : -(m - ofs);
                const uint64_t a2 = pk2(a, a), b2 = pk2(b, b);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t w[32];
#pragma unroll
                    for (int y = 0; y < 32; ++y) {
                        const uint64_t x = fma2(pk2(__uint_as_float(sr[64 * h + 2 * y]),
                                                    __uint_as_float(sr[64 * h + 2 * y + 1])),
                                                a2, b2);
                        float x0, x1;
                        upk2(x, x0, x1);
                        const float e0 = ex2(x0), e1 = ex2(x1);
                        ls2[y & 1] = add2(ls2[y & 1], pk2(e0, e1));
                        if (kBF16)
                            asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w[y]) : "f"(e1), "f"(e0));
                        else
                            asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(w[y]) : "f"(e1), "f"(e0));
                    }
                    tmem_st32(tmem + lane_addr + s_col + static_cast<uint32_t>(32 * h), w);
                }
            }
            {
                float a0, a1, b0, b1;
                upk2(ls2[0], a0, a1);
                upk2(ls2[1], b0, b1);
                lx += (a0 + a1) + (b0 + b1);
            }
            tmem_wait_st();
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&p_full[g]));
        }
        // ---- this group's last P V product must be complete before O is read
        if (ng > 0) wait(&o_done[g], 0);
        fence_after();
        // P is normalised by its unrounded sum (the rounded sum would carry
        // the same error bound)
        if (ng > 0) {
            const float inv = 1.f / lx;
            float* orow = p.out + (bh * p.S + i) * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_addr + o_col + static_cast<uint32_t>(32 * c), o);
                tmem_wait_ld();
                if (i < p.S) {
#pragma unroll
                    for (int y = 0; y < 32; y += 4) {
                        float4 v;
                        v.x = __uint_as_float(o[y]) * inv;
                        v.y = __uint_as_float(o[y + 1]) * inv;
                        v.z = __uint_as_float(o[y + 2]) * inv;
                        v.w = __uint_as_float(o[y + 3]) * inv;
                        *reinterpret_cast<float4*>(orow + 32 * c + y) = v;
                    }
                }
            }
            if (i < p.S && p.lse) p.lse[bh * p.S + i] = (m + log2f(lx)) * kLn2;
        }
    }

    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kPTmemCols) : "memory");
    }
}

template <typename E, int D>
cudaError_t launch_prefill_t(int device, const PrefillParams& p, const CUtensorMap& mq,
                             const CUtensorMap& mk, const CUtensorMap& mv, cudaStream_t s) {
    using C = PCfg<D>;
    auto kern = td_prefill_kernel<E, D>;
    static std::atomic<unsigned long long> configured{0};
    const unsigned long long bit = device < 64 ? (1ull << device) : 0ull;
    if (!bit || !(configured.load(std::memory_order_acquire) & bit)) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::kSmem));
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    const long long BH = static_cast<long long>(p.B) * p.H;
    const long long nqt = (p.S + kPQ - 1) / kPQ;
    const long long npair = (nqt + 1) / 2;
    if (BH * npair > 0x7fffffffLL) return cudaErrorInvalidValue;
    kern<<<static_cast<unsigned>(BH * npair), kPThreads, C::kSmem, s>>>(p, mq, mk, mv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(int device, int dtype, int D, const PrefillParams& p,
                           const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                           cudaStream_t s) {
    if (dtype == kBF16) {
        if (D == 64) return launch_prefill_t<__nv_bfloat16, 64>(device, p, mq, mk, mv, s);
        if (D == 128) return launch_prefill_t<__nv_bfloat16, 128>(device, p, mq, mk, mv, s);
    } else if (dtype == kF16) {
        if (D == 64) return launch_prefill_t<__half, 64>(device, p, mq, mk, mv, s);
        if (D == 128) return launch_prefill_t<__half, 128>(device, p, mq, mk, mv, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace td
