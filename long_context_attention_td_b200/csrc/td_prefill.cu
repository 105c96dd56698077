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
// One CTA per (b, h, tile of 128 query rows); the heaviest causal tiles are
// scheduled first.  Per key tile of 128 keys:
//     S [128 q x 128 k] = Q [128 x D] . K^T       (D/16 tcgen05.mma, N = 128)
//     O [128 q x D]    += P [128 x 128] . V       (8 tcgen05.mma, N = D)
// with S and O as fp32 in TMEM and P rounded to the input type in shared
// memory (the A operand of P V).  Two softmax groups take alternate key tiles,
// each with its own S buffer, P buffer, running max and sum and O accumulator;
// their rows are merged at the end.  Each softmax thread owns one query row
// (its TMEM lane), so its running max and sums need no cross-thread
// reduction; O is rescaled row by row in TMEM when a row's max grows by more
// than 8 (log2 units).
//
// 12 warps in three warpgroups: warpgroup 0 -- warp 0 Q and K producer, warp 2
// V producer (3-D boxes of {64 columns, 128 rows, 1 sequence}, 2 stages),
// warp 1 TMEM owner and MMA issuer, warp 3 idle; warpgroups 1 and 2 -- the
// softmax groups (warp w reads TMEM lanes 32 (w % 4) .. + 31).
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

constexpr int kPQ = 128;             // query rows per CTA (MMA M)
constexpr int kPK = 128;             // keys per tile (MMA N of S)
constexpr int kPThreads = 384;       // 12 warps (two softmax warpgroups)
// register split (setmaxnreg): warpgroup 0 (TMA, MMA,
// two idle warps) drops to kRegLow, the softmax warpgroups rise to kRegHigh;
// 4*32*kRegLow + 8*32*kRegHigh must not exceed the 384 x 168 registers the
// block is launched with, or the increase would wait for ever
constexpr int kRegLow = 56;
constexpr int kRegHigh = 224;
static_assert(4 * 32 * kRegLow + 8 * 32 * kRegHigh <= kPThreads * 168, "register split");
constexpr int kPStages = 2;          // K/V pipeline depth
constexpr int kPTmemCols = 512;      // S0 [0,128) S1 [128,256) O [256, 256 + D)
constexpr float kPRescale = 8.f;     // log2 units

template <int D>
struct PCfg {
    static constexpr int kAtoms = D / 64;                 // 64-column swizzle atoms of D
    static constexpr int kRowAtom = 128 * 128;            // 128 rows x 64 columns, 16 KB
    static constexpr int kQBytes = kAtoms * kRowAtom;
    static constexpr int kStageBytes = 2 * kAtoms * kRowAtom;  // K atoms, then V atoms
    static constexpr int kPBytes = (kPK / 64) * kRowAtom;     // 128 rows x 128 keys
    static constexpr int kOffQ = 0;
    static constexpr int kOffKV = kOffQ + kQBytes;
    static constexpr int kOffP = kOffKV + kPStages * kStageBytes;
    static constexpr int kOffBias = kOffP + 2 * kPBytes;       // ALiBi row of a tile, x2
    static constexpr size_t kSmem = size_t(kOffBias) + 2 * kPK * 4 + 1024;  // +align
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

struct PCtl {
    int abort;
    uint32_t tmem;
};

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

    // K and V of a stage have their own barriers: K is free once its S
    // product is done, V once its P V product is
    __shared__ __align__(8) uint64_t k_full[kPStages], k_empty[kPStages];
    __shared__ __align__(8) uint64_t v_full[kPStages], v_empty[kPStages];
    __shared__ __align__(8) uint64_t q_full, s_full[2], s_empty[2], p_full[2], pv_done[2];
    __shared__ PCtl ctl;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Sequences are taken in groups of hg whose K and V together fill about
    // 32 MB, so the query tiles in flight share key tiles in L2; inside a
    // group the heaviest causal tiles go first (the group's last query tile
    // of every sequence, then the one before, ...), which keeps the tail short.
    const long long BH = static_cast<long long>(p.B) * p.H;
    const long long nqt = (p.S + kPQ - 1) / kPQ;
    const long long kv_bytes = static_cast<long long>(p.S) * D * 2 * static_cast<long long>(sizeof(E));
    long long hg = (32ll << 20) / kv_bytes;
    hg = hg < 1 ? 1 : (hg > BH ? BH : hg);
    const long long grp0 = (static_cast<long long>(blockIdx.x) / (hg * nqt)) * hg;  // first sequence
    const long long hcnt = BH - grp0 < hg ? BH - grp0 : hg;                           // its size
    const long long idx = static_cast<long long>(blockIdx.x) - grp0 * nqt;
    const long long bh = grp0 + idx % hcnt;
    const long long qt = nqt - 1 - idx / hcnt;
    const long long nkt_all = (p.S + kPK - 1) / kPK;
    // key tiles this query tile reads
    const long long nt = p.causal ? (qt + 1 < nkt_all ? qt + 1 : nkt_all) : nkt_all;
    static_assert(kPQ == kPK, "causal tile count assumes square tiles");

    if (tid == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(smem_addr(&k_full[s]), 1);
            mbar_init(smem_addr(&k_empty[s]), 1);
            mbar_init(smem_addr(&v_full[s]), 1);
            mbar_init(smem_addr(&v_empty[s]), 1);
        }
        mbar_init(smem_addr(&q_full), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&s_full[s]), 1);
            mbar_init(smem_addr(&s_empty[s]), 4);
            mbar_init(smem_addr(&p_full[s]), 4);
            mbar_init(smem_addr(&pv_done[s]), 1);
        }
        fence_barrier_init();
        ctl.abort = 0;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_addr(&ctl.tmem)), "r"(kPTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_before();
    __syncthreads();
    fence_after();

    const uint32_t tmem = ctl.tmem;
    volatile int* abort_flag = &ctl.abort;
    constexpr int kSoft0 = 4;  // first softmax warp
    const uint32_t sQ = smem_addr(smem + C::kOffQ);
    const uint32_t sKV = smem_addr(smem + C::kOffKV);
    const uint32_t sP = smem_addr(smem + C::kOffP);
    const int z = static_cast<int>(bh);

    if (warp < kSoft0) {
    // each warpgroup's register change heads its branch, so the code of the
    // branch is compiled for that register count
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegLow));
    if (warp == 0 || warp == 2) {
        // -------------------------------------------------------- producer
        // one warp for Q and K and another for V, so that a K load never
        // waits behind a V stage still held by a P V product
        const bool doK = warp == 0;
        const bool doV = warp == 2;
        if (lane == 0) {
            bool aborted = false;
            if (doK) {
                mbar_arrive_expect_tx(smem_addr(&q_full), C::kQBytes);
#pragma unroll
                for (int a = 0; a < C::kAtoms; ++a)
                    tma_load_3d(sQ + a * C::kRowAtom, &tmQ, 64 * a, static_cast<int>(qt * kPQ), z,
                                smem_addr(&q_full));
            }
            int stage = 0;
            uint32_t phase = 0;
            long long k_issued = 0, v_issued = 0;   // K / V tiles whose loads were issued
            for (long long t = 0; t < nt; ++t) {
                const uint32_t base = sKV + stage * C::kStageBytes;
                const int y = static_cast<int>(t * kPK);
                if (doK) {
                    if (!aborted && !mbar_wait_bounded(smem_addr(&k_empty[stage]), phase ^ 1u,
                                                       abort_flag, p.err, TD_DEVERR_WAIT_TIMEOUT))
                        aborted = true;
                    if (!aborted) {
                        const uint32_t fb = smem_addr(&k_full[stage]);
                        mbar_arrive_expect_tx(fb, C::kStageBytes / 2);
#pragma unroll
                        for (int a = 0; a < C::kAtoms; ++a)
                            tma_load_3d(base + a * C::kRowAtom, &tmK, 64 * a, y, z, fb);
                        ++k_issued;
                    }
                }
                if (doV) {
                    if (!aborted && !mbar_wait_bounded(smem_addr(&v_empty[stage]), phase ^ 1u,
                                                       abort_flag, p.err, TD_DEVERR_WAIT_TIMEOUT))
                        aborted = true;
                    if (!aborted) {
                        const uint32_t fb = smem_addr(&v_full[stage]);
                        mbar_arrive_expect_tx(fb, C::kStageBytes / 2);
#pragma unroll
                        for (int a = 0; a < C::kAtoms; ++a)
                            tma_load_3d(base + (C::kAtoms + a) * C::kRowAtom, &tmV, 64 * a, y, z,
                                        fb);
                        ++v_issued;
                    }
                }
                if (++stage == kPStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            // the CTA must not exit with copies into its shared memory in flight
            if (doK)
                mbar_wait_bounded(smem_addr(&q_full), 0, nullptr, p.err, TD_DEVERR_WAIT_TIMEOUT);
            // tiles are issued in order, so the last K (V) load on stage s is
            // tile s + kPStages * floor((issued - 1 - s) / kPStages)
            for (int s = 0; s < kPStages; ++s) {
                if (s < k_issued) {
                    const long long lt = s + ((k_issued - 1 - s) / kPStages) * kPStages;
                    mbar_wait_bounded(smem_addr(&k_full[s]),
                                      static_cast<uint32_t>((lt / kPStages) & 1), nullptr, p.err,
                                      TD_DEVERR_WAIT_TIMEOUT);
                }
                if (s < v_issued) {
                    const long long lt = s + ((v_issued - 1 - s) / kPStages) * kPStages;
                    mbar_wait_bounded(smem_addr(&v_full[s]),
                                      static_cast<uint32_t>((lt / kPStages) & 1), nullptr, p.err,
                                      TD_DEVERR_WAIT_TIMEOUT);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idS = instr_desc_f16(kBF16 ? 1 : 0, kPQ, kPK, 0, 0);
            constexpr uint32_t idO = instr_desc_f16(kBF16 ? 1 : 0, kPQ, D, 0, 1);
            bool aborted = false;
            long long last_pv = -1;
            if (!mbar_wait_bounded(smem_addr(&q_full), 0, abort_flag, p.err,
                                   TD_DEVERR_WAIT_TIMEOUT))
                aborted = true;
            fence_after();
            long long ts = 0, tp = 0;
            uint64_t t_stall = 0;
            uint32_t spins = 0;
            while (tp < nt && !aborted) {
                bool progressed = false;
                if (ts < nt &&
                    mbar_test(smem_addr(&k_full[ts % kPStages]),
                              static_cast<uint32_t>((ts / kPStages) & 1)) &&
                    (ts < 2 || mbar_test(smem_addr(&s_empty[ts & 1]),
                                         static_cast<uint32_t>(((ts >> 1) - 1) & 1)))) {
                    fence_after();
                    const uint32_t kb = sKV + static_cast<uint32_t>(ts % kPStages) * C::kStageBytes;
                    const uint32_t dS = tmem + static_cast<uint32_t>((ts & 1) * kPK);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = static_cast<uint32_t>((kk & 3) * 32);
                        const uint64_t a =
                            smem_desc_sw128(sQ + (kk >> 2) * C::kRowAtom + off, 16, 1024);
                        const uint64_t b =
                            smem_desc_sw128(kb + (kk >> 2) * C::kRowAtom + off, 16, 1024);
                        umma_f16(dS, a, b, idS, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(smem_addr(&s_full[ts & 1]));
                    umma_commit(smem_addr(&k_empty[ts % kPStages]));
                    ++ts;
                    progressed = true;
                }
                if (tp < ts &&
                    mbar_test(smem_addr(&p_full[tp & 1]), static_cast<uint32_t>((tp >> 1) & 1)) &&
                    mbar_test(smem_addr(&v_full[tp % kPStages]),
                              static_cast<uint32_t>((tp / kPStages) & 1))) {
                    fence_after();
                    const int stage = static_cast<int>(tp % kPStages);
                    const uint32_t vb = sKV + stage * C::kStageBytes + C::kAtoms * C::kRowAtom;
                    const uint32_t pb = sP + static_cast<uint32_t>((tp & 1) * C::kPBytes);
                    // one O accumulator per softmax group (tiles alternate)
                    const uint32_t dO = tmem + 2 * kPK + static_cast<uint32_t>((tp & 1) * D);
#pragma unroll
                    for (int kk = 0; kk < kPK / 16; ++kk) {
                        // P: 16 keys of every query row; V: the same 16 keys,
                        // all D columns (two 64-column halves kRowAtom apart)
                        const uint64_t a = smem_desc_sw128(
                            pb + (kk >> 2) * C::kRowAtom + (kk & 3) * 32, 16, 1024);
                        const uint64_t b = smem_desc_sw128(vb + kk * 2048, C::kRowAtom, 1024);
                        umma_f16(dO, a, b, idO, (tp >= 2 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(smem_addr(&pv_done[tp & 1]));
                    umma_commit(smem_addr(&v_empty[stage]));
                    last_pv = tp;
                    ++tp;
                    progressed = true;
                }
                if (progressed) {
                    spins = 0;
                    t_stall = 0;
                    continue;
                }
                if ((++spins & 63u) == 0u) {
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
            // every MMA must be complete before the CTA frees TMEM
            for (long long tl = last_pv - 1; tl <= last_pv; ++tl)
                if (tl >= 0)
                    mbar_wait_bounded(smem_addr(&pv_done[tl & 1]),
                                      static_cast<uint32_t>((tl >> 1) & 1), nullptr, p.err,
                                      TD_DEVERR_WAIT_TIMEOUT);
            if (last_pv < 0 && ts > 0)
                // S products issued without a P V: wait for the last one
                mbar_wait_bounded(smem_addr(&s_full[(ts - 1) & 1]),
                                  static_cast<uint32_t>(((ts - 1) >> 1) & 1), nullptr, p.err,
                                  TD_DEVERR_WAIT_TIMEOUT);
        }
        __syncwarp();
    }
    } else {
        // --------------------------------------------------------- softmax
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegHigh));
        const int g = (warp - kSoft0) >> 2;           // softmax group: tiles t % 2 == g
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;            // query row of the tile (TMEM lane)
        const long long i = qt * kPQ + r;             // query index in the sequence
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const float qscale2 = p.qscale2;
        const float slope2 = p.slopes ? __ldg(p.slopes + (bh % p.H)) * kLog2e : 0.f;
        bool aborted = false;
        auto wait = [&](uint64_t* bar, uint32_t par) {
            if (!aborted && !mbar_wait_bounded(smem_addr(bar), par, abort_flag, p.err,
                                               TD_DEVERR_WAIT_TIMEOUT))
                aborted = true;
        };
        float m = kNegInf, thr = kNegInf, lx = 0.f;
        unsigned char* prow0 = smem + C::kOffP;
        const uint32_t o_col = static_cast<uint32_t>(2 * kPK + g * D);
        for (long long t = g; t < nt; t += 2) {
            const int buf = static_cast<int>(t & 1);
            wait(&s_full[buf], static_cast<uint32_t>((t >> 1) & 1));
            fence_after();
            uint32_t sr[kPK];
#pragma unroll
            for (int c = 0; c < kPK / 32; ++c)
                tmem_ld32(tmem + lane_addr + static_cast<uint32_t>(buf * kPK + 32 * c),
                          *reinterpret_cast<uint32_t(*)[32]>(sr + 32 * c));
            tmem_wait_ld();
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&s_empty[buf]));

            // scores in log2 units: x_c = raw_c qscale2 + slope2 (j0 + c - S + 1);
            // keys past the row's last visible key (causal) or past the
            // sequence end are -inf.  A tile with every key visible and no bias
            // (all but the diagonal and last tiles) takes the row max on the raw
            // products (qscale2 > 0 keeps the order) and forms x_c - m with one
            // fma in the exponential loop; the others build x_c first.  Maxima
            // run as 8 independent chains (max is exact, so any order gives the
            // same value).
            const long long j0 = t * kPK;
            const long long jmax = p.causal ? (i < p.S - 1 ? i : p.S - 1) : p.S - 1;
            const int cmax = static_cast<int>(jmax - j0 < kPK - 1 ? jmax - j0 : kPK - 1);
            const bool plain = p.slopes == nullptr && __all_sync(0xffffffffu, cmax == kPK - 1);
            float mx8[8];
            if (plain) {
#pragma unroll
                for (int c = 0; c < 8; ++c) mx8[c] = __uint_as_float(sr[c]);
#pragma unroll
                for (int c = 8; c < kPK; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], __uint_as_float(sr[c]));
            } else {
                // the ALiBi row of this key tile, slope2 (j - S + 1), is the same
                // for every query row: each thread writes one key's value
                // (one buffer per group, so the group first waits until all its
                // warps are done with its previous tile's row)
                const float* bias = reinterpret_cast<const float*>(smem + C::kOffBias) + buf * kPK;
                if (p.slopes) {
                    named_bar_sync(1 + g, 4 * 32);
                    const_cast<float*>(bias)[r] = slope2 * static_cast<float>(j0 - p.S + 1 + r);
                    named_bar_sync(1 + g, 4 * 32);
                }
#pragma unroll
                for (int c = 0; c < 8; ++c) mx8[c] = kNegInf;
                auto build = [&](auto masked_c) {
                    constexpr bool kMasked = decltype(masked_c)::value;
#pragma unroll
                    for (int c4 = 0; c4 < kPK; c4 += 4) {
                        const float4 b4 = p.slopes ? *reinterpret_cast<const float4*>(bias + c4)
                                                   : make_float4(0.f, 0.f, 0.f, 0.f);
                        const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int c = c4 + u;
                            float x = fmaf(__uint_as_float(sr[c]), qscale2, bb[u]);
                            if (kMasked) x = c <= cmax ? x : kNegInf;
                            sr[c] = __float_as_uint(x);
                            mx8[c & 7] = fmaxf(mx8[c & 7], x);
                        }
                    }
                };
                if (__any_sync(0xffffffffu, cmax < kPK - 1))
                    build(std::true_type{});
                else
                    build(std::false_type{});
            }
            float mt = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            if (plain) mt *= qscale2;
            // move this row's max when the tile exceeds it by more than the
            // threshold (always on the first tile)
            const bool need = mt > thr;
            if (__any_sync(0xffffffffu, need && t >= 2)) {
                // O holds this group's earlier tiles (the last one t - 2):
                // rescale this warp's rows in TMEM
                wait(&pv_done[(t - 2) & 1], static_cast<uint32_t>(((t - 2) >> 1) & 1));
                fence_after();
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
                tmem_wait_st();
            }
            if (need) {
                lx *= rescale(m, mt);
                m = mt;
                thr = mt + kPRescale;
            }
            // the P V product of tile t - 2 read this P buffer
            if (t >= 2) wait(&pv_done[buf], static_cast<uint32_t>(((t >> 1) - 1) & 1));
            fence_after();
            unsigned char* prow = prow0 + buf * C::kPBytes;
            // the row sum over 4 independent partials (no 128-long dependent chain)
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
            auto exps = [&](auto plain_c) {
                constexpr bool kPlain = decltype(plain_c)::value;
#pragma unroll
                for (int cc = 0; cc < kPK / 8; ++cc) {
                    uint32_t w4[4];
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        // masked keys give ex2(-inf) = 0
                        const float a0 = __uint_as_float(sr[cc * 8 + 2 * y]);
                        const float a1 = __uint_as_float(sr[cc * 8 + 2 * y + 1]);
                        const float e0 = ex2(kPlain ? fmaf(a0, qscale2, -m) : a0 - m);
                        const float e1 = ex2(kPlain ? fmaf(a1, qscale2, -m) : a1 - m);
                        ls[y] += e0 + e1;
                        if (kBF16)
                            asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w4[y]) : "f"(e1), "f"(e0));
                        else
                            asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(w4[y]) : "f"(e1), "f"(e0));
                    }
                    *reinterpret_cast<uint4*>(prow + (cc >> 3) * C::kRowAtom + swz(r, cc & 7)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            };
            if (plain)
                exps(std::true_type{});
            else
                exps(std::false_type{});
            lx += (ls[0] + ls[1]) + (ls[2] + ls[3]);
            fence_proxy_async_smem();
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&p_full[buf]));
        }
        // ---- this group's last P V product must be complete before O is read
        const long long last = nt > g ? g + 2 * ((nt - 1 - g) / 2) : -1;
        if (last >= 0) wait(&pv_done[last & 1], static_cast<uint32_t>((last >> 1) & 1));
        fence_after();
        // P is normalised by its unrounded sum (the rounded sum would carry
        // the same error bound)
        float* orow = p.out + (bh * p.S + i) * D;
        {
            // the two groups' (m, l) per row meet in shared memory (each group's
            // P buffer is free once its last product is complete); the merged
            // row is sum_g e^(m_g - M) O_g / sum_g e^(m_g - M) l_g, group g
            // writing columns [g D/2, (g+1) D/2)
            float* xg = reinterpret_cast<float*>(smem + C::kOffP + g * C::kPBytes);
            xg[r] = m;
            xg[kPQ + r] = lx;
            fence_before();
            named_bar_sync(3, 2 * 4 * 32);
            fence_after();
            const float* xa = reinterpret_cast<const float*>(smem + C::kOffP);
            const float* xb = reinterpret_cast<const float*>(smem + C::kOffP + C::kPBytes);
            const bool hasB = nt > 1;  // group 0 always has tile 0
            const float mA = xa[r], mB = hasB ? xb[r] : kNegInf;
            const float M = fmaxf(mA, mB);
            const float wA = rescale(mA, M), wB = hasB ? rescale(mB, M) : 0.f;
            const float L = wA * xa[kPQ + r] + (hasB ? wB * xb[kPQ + r] : 0.f);
            const float fa = wA / L, fb = wB / L;
#pragma unroll 1
            for (int c = g * (D / 64); c < (g + 1) * (D / 64); ++c) {
                uint32_t oa[32], ob[32];
                tmem_ld32(tmem + lane_addr + static_cast<uint32_t>(2 * kPK + 32 * c), oa);
                if (hasB) tmem_ld32(tmem + lane_addr + static_cast<uint32_t>(2 * kPK + D + 32 * c), ob);
                tmem_wait_ld();
                if (i < p.S) {
#pragma unroll
                    for (int y = 0; y < 32; y += 4) {
                        float4 v;
                        v.x = __uint_as_float(oa[y]) * fa;
                        v.y = __uint_as_float(oa[y + 1]) * fa;
                        v.z = __uint_as_float(oa[y + 2]) * fa;
                        v.w = __uint_as_float(oa[y + 3]) * fa;
                        if (hasB) {
                            v.x = fmaf(__uint_as_float(ob[y]), fb, v.x);
                            v.y = fmaf(__uint_as_float(ob[y + 1]), fb, v.y);
                            v.z = fmaf(__uint_as_float(ob[y + 2]), fb, v.z);
                            v.w = fmaf(__uint_as_float(ob[y + 3]), fb, v.w);
                        }
                        *reinterpret_cast<float4*>(orow + 32 * c + y) = v;
                    }
                }
            }
            if (g == 0 && i < p.S && p.lse) p.lse[bh * p.S + i] = (M + log2f(L)) * kLn2;
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
    if (BH * nqt > 0x7fffffffLL) return cudaErrorInvalidValue;
    kern<<<static_cast<unsigned>(BH * nqt), kPThreads, C::kSmem, s>>>(p, mq, mk, mv);
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
