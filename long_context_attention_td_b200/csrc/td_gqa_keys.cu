// td_gqa_keys -- grouped-query split-KV decode on the sm_100a tensor cores with
// the KEYS on the MMA M axis.
//
// What it computes: exactly what td_gqa computes ("Tree Attention Decoding"
// gist, Algorithm 3, with G = Hq / Hkv query heads reading each key/value
// head), and it writes the same part records.  The contraction is arranged
// transposed: per tile of 128 keys of one (b, kv head) sequence
//     S^T [128 keys x NQ]  = K [128 x D] . Q^T [D x NQ]
//     O^T [D x NQ]        += V^T [D x 128] . P^T [128 x NQ]
// where the NQ columns are the group's query heads (G padded to 16 or 32).
// One tcgen05.mma (K = 16) covers 16 columns of D in the first product and 16
// keys in the second, so a tile takes D/16 + 8 instructions, and the operands
// the tensor core reads from shared memory are the K and V tiles once plus a
// small Q or P block.  With the query heads on M instead, the same 128 keys
// take 24 instructions and re-read the 128-row Q block for every one of them.
//
// Each softmax thread owns one key of the tile (its TMEM lane) and the G
// scores of that key, so no lane idles for small groups.  The running max of
// each head is shared by a softmax warpgroup; it moves only when a score
// exceeds it by more than 8 (log2 units), which one barrier-reduction per
// tile decides, and O^T in TMEM is rescaled then.
//
// For D = 64 the P V product still runs with M = 128: the second 64-row half
// of its A operand is the stage's K tile, so rows 64-127 of O^T hold values
// that are never read, and the TMEM layout of O^T (row r in lane r) is the one
// the D = 128 kernel uses.
//
// One CTA per SM, 10 warps:
//   warp 0      TMA producer: K and V tiles of 128 keys as 2-D boxes of
//               {64 columns, 128 rows} with 128-byte swizzle, 3 stages of
//               64 KB (D = 128) or 6 stages of 32 KB (D = 64);
//   warp 1      owns TMEM (S0, S1, O0, O1: NQ columns each) and issues the
//               MMAs from one lane, signalling completion with tcgen05.commit;
//   warps 2-5   softmax group 0 (even tiles), warps 6-9 group 1 (odd tiles);
//               warp w reads TMEM lanes 32 (w % 4) .. + 31.
// Used for every grouped-query shape (D = 64 or 128, G <= 128): a group of
// more than 32 heads is cut into chunks of at most 32 heads, one CTA per
// (part, chunk) over the part's keys; the chunks of a part have adjacent block
// indices, so they run at the same time and the later ones read the K/V tiles
// from L2.
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

constexpr int kKT = 128;              // keys per tile (MMA M of S^T)
constexpr int kKMO = 128;             // MMA M of O^T (D rows, padded to 128 for D = 64)
constexpr int kKThreads = 320;        // 10 warps
constexpr int kKGroup = 128;          // threads of one softmax warpgroup
constexpr int kKScratch = 512;        // floats of tree_merge scratch (>= 128)
constexpr float kKRescale = 8.f;      // log2 units
constexpr int kBarG0 = 1;             // named barrier: softmax group 0
constexpr int kBarBoth = 2;           // named barrier: both softmax groups
constexpr int kBarG1 = 3;             // named barrier: softmax group 1

template <int GP, int D>
struct KCfg {
    static constexpr int NQ = GP < 16 ? 16 : GP;      // MMA N
    static constexpr int kAtoms = D / 64;              // 64-column swizzle atoms of D
    // CTAs per SM: two for D = 64 up to 16 heads per group (their 32 KB tiles
    // leave room for two CTAs of 3 stages each), else one
    static constexpr int kCtasPerSm = (D == 64 && GP <= 16) ? 2 : 1;
    static constexpr int kStages = D == 128 ? 3 : (kCtasPerSm == 2 ? 3 : 6);  // K/V depth
    static constexpr int kQAtom = NQ * 128;            // NQ rows x 64 columns
    static constexpr int kQBytes = kAtoms * kQAtom;
    static constexpr int kPAtom = NQ * 128;            // NQ rows x 64 keys
    static constexpr int kPBytes = (kKT / 64) * kPAtom;  // one P^T buffer
    static constexpr int kKVAtom = kKT * 128;          // 128 keys x 64 columns
    static constexpr int kStageBytes = 2 * kAtoms * kKVAtom;
    // inside a stage: D = 128, the K atoms then the V atoms; D = 64, the V atom
    // then the K atom, so the P V product's rows 64-127 (its A operand's second
    // 64-row half, kKVAtom past the V atom) read this stage's K tile
    static constexpr int kOffKAtoms = D == 128 ? 0 : kKVAtom;
    static constexpr int kOffVAtoms = D == 128 ? kAtoms * kKVAtom : 0;
    static constexpr int kOffQ = 0;
    static constexpr int kOffP = kOffQ + kQBytes;
    static constexpr int kOffKV = ((kOffP + 2 * kPBytes) + 1023) / 1024 * 1024;
    static constexpr int kOffScratch = kOffKV + kStages * kStageBytes;
    // per piece parity: [group][head] sums of p, [head][2] output weights,
    // [group][head] maxima
    static constexpr int kStatsFloats = 2 * (2 * 4 * GP * 2 + 2 * GP);
    static constexpr int kOffStats = kOffScratch + kKScratch * 4;
    // per group: [warp quarter][head] tile maxima
    static constexpr int kOffRed = kOffStats + kStatsFloats * 4;
    static constexpr int kRedFloats = 2 * 4 * GP;
    // per group: ALiBi slopes of the piece's heads (log2 units)
    static constexpr int kOffSlopes = kOffRed + kRedFloats * 4;
    static constexpr size_t kSmem = size_t(kOffSlopes) + 2 * GP * 4 + 1024;  // +align
    static constexpr int kTmemCols = 4 * NQ < 32 ? 32 : 4 * NQ;
    static_assert(GP == 4 || GP == 8 || GP == 16 || GP == 32, "GP");
    static_assert(D == 64 || D == 128, "D");
    static_assert(kSmem <= 232448 - 512, "shared memory");
    static_assert(kCtasPerSm * (kSmem + 1024) <= 233472, "shared memory of the CTAs of an SM");
};

// ----------------------------------------------------------- TMEM access

template <int X>
__device__ __forceinline__ void tmem_ld_x(uint32_t taddr, uint32_t (&r)[X]);
template <>
__device__ __forceinline__ void tmem_ld_x<4>(uint32_t taddr, uint32_t (&r)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_x<8>(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_x<16>(uint32_t taddr, uint32_t (&r)[16]) {
    tmem_ld16(taddr, r);
}

template <int X>
__device__ __forceinline__ void tmem_st_x(uint32_t taddr, const uint32_t (&r)[X]);
template <>
__device__ __forceinline__ void tmem_st_x<4>(uint32_t taddr, const uint32_t (&r)[4]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};"
                 ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
                 : "memory");
}
template <>
__device__ __forceinline__ void tmem_st_x<8>(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]),
                 "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}
template <>
__device__ __forceinline__ void tmem_st_x<16>(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
        "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// bar.red.or over `threads` threads of named barrier `id`: true when any
// participating thread passed true.
__device__ __forceinline__ bool bar_any(int id, int threads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(threads)
        : "memory");
    return r != 0;
}

// p rounded to the element type of the P V product
template <typename E>
__device__ __forceinline__ void round_store(float e, unsigned char* dst);
template <>
__device__ __forceinline__ void round_store<__nv_bfloat16>(float e, unsigned char* dst) {
    *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(e);
}
template <>
__device__ __forceinline__ void round_store<__half>(float e, unsigned char* dst) {
    *reinterpret_cast<__half*>(dst) = __float2half_rn(e);
}

// mbarrier phase test that may suspend the thread for up to `ns` nanoseconds
// while the phase is incomplete (frees issue slots of a polling thread)
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

struct KCtx {
    int g_eff, h_off;        // heads of this CTA's chunk and the first of them
    unsigned char* smem;
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

// ------------------------------------------------------------ softmax role

// The softmax warpgroups.  kSplit == false: group g takes the tiles with
// t % 2 == g and every head, with its own O^T accumulator; kSplit == true:
// both groups take every tile, group g the heads [g HG, (g+1) HG), and they
// share one O^T accumulator (its columns are disjoint by head).
template <typename E, int GP, bool kSplit, int D>
__device__ __forceinline__ void keys_softmax(const GqaParams& p, const KCtx& x) {
    using C = KCfg<GP, D>;
    constexpr int NQ = C::NQ;
    constexpr int HG = kSplit ? GP / 2 : GP;    // heads of one group
    const int G = x.g_eff;                      // heads of this CTA (its chunk)
    const int Gall = p.G;                       // heads of the kv head's group
    const int h_off = x.h_off;                  // first head of the chunk
    const int grp = (x.warp - 2) >> 2;
    const int hb = kSplit ? grp * HG : 0;       // first head of this group
    const int quarter = x.warp & 3;             // TMEM lane quarter of this warp
    const int lane = x.lane;
    const int key = quarter * 32 + lane;        // key of the tile (S^T row); D row of O^T
    const int st = (x.tid - 64) & (kKGroup - 1);  // thread within the group
    const int bar_grp = grp == 0 ? kBarG0 : kBarG1;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t o_col = static_cast<uint32_t>(2 * NQ + (kSplit ? hb : grp * NQ));
    const float qscale2 = p.qscale2;
    unsigned char* smem = x.smem;
    float* stats_all = reinterpret_cast<float*>(smem + C::kOffStats);
    float* red = reinterpret_cast<float*>(smem + C::kOffRed) + grp * 4 * GP;
    float* scratch = reinterpret_cast<float*>(smem + C::kOffScratch);
    long long t = 0;
    long long pc = 0;
    bool aborted = false;
    auto wait = [&](uint64_t* bar, uint32_t par) {
        if (!aborted && !mbar_wait_bounded(smem_addr(bar), par, x.abort_flag, p.err,
                                           TD_DEVERR_WAIT_TIMEOUT))
            aborted = true;
    };
    // wait for the P V product of tile tt (tt >= 0)
    auto wait_pv = [&](long long tt) {
        wait(&x.pv_done[tt & 1], static_cast<uint32_t>((tt >> 1) & 1));
    };
    GWalk w;
    if (!gwalk_first(p, *x.ctl, w)) return;
    do {
        const long long j0 = (x.x0 > w.start ? x.x0 : w.start) - w.start;
        const long long e = w.start + w.len;
        const long long j1 = (x.x1 < e ? x.x1 : e) - w.start;
        const long long nt = (j1 - j0 + kKT - 1) / kKT;
        const bool whole = (j0 == 0 && j1 == w.len);
        const long long qrow0 = static_cast<long long>(w.b) * p.Hq +
                                static_cast<long long>(w.h) * Gall;  // group's first query row
        const long long qrow = qrow0 + h_off;                         // this chunk's first
        float* stats = stats_all + (pc & 1) * (2 * 4 * GP * 2 + 2 * GP);
        float* st_l = stats;                      // [grp][head]
        float* st_m = stats + 2 * 4 * GP * 2;     // [grp][head]

        // Q rows of this kv head's group, K-major SW128 (rows >= G stay zero)
        if (grp == 0) {
            const uint4* qg = reinterpret_cast<const uint4*>(static_cast<const E*>(p.q) +
                                                             qrow * D);
            for (int u = st; u < G * (D / 8); u += kKGroup) {
                const int g = u / (D / 8);
                const int cc = u - g * (D / 8);
                *reinterpret_cast<uint4*>(smem + C::kOffQ + (cc >> 3) * C::kQAtom +
                                          swz(g, cc & 7)) = __ldg(qg + u);
            }
            fence_proxy_async_smem();
        }
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(x.q_ready));

        float* slope2 = reinterpret_cast<float*>(smem + C::kOffSlopes) + grp * GP;
        if (p.slopes) {
            if (st < HG)
                slope2[st] = hb + st < G
                                 ? __ldg(p.slopes + w.h * Gall + h_off + hb + st) * kLog2e
                                 : 0.f;
            named_bar_sync(bar_grp, kKGroup);
        }
        // per head: running max m (uniform in the group; moved when a score
        // exceeds m + 8) and this thread's sum of p over its keys.  Heads past G
        // (padding of the MMA's N) keep m = 0: their scores are 0 (zero Q rows),
        // so they never move it, and their p is finite and never read.
        float m_ref[HG], lx[HG];
#pragma unroll
        for (int h = 0; h < HG; ++h) {
            m_ref[h] = hb + h < G ? kNegInf : 0.f;
            lx[h] = 0.f;
        }
        // this thread's P^T element of head h: row hb + h, K column = key; with
        // hb a multiple of HG (a power of two), (hb + h) % 8 == (hb % 8) ^ (h % 8)
        const int kc2 = ((key & 63) >> 3) ^ (hb & 7);
        const int p_off = (key >> 6) * C::kPAtom + (key & 7) * 2 + hb * 128;
        long long last_own = -1;
        for (long long i = 0; i < nt; ++i, ++t) {
            if (!kSplit && static_cast<int>(t & 1) != grp) continue;
            const long long t0 = j0 + i * kKT;
            const int rows = static_cast<int>((j1 - t0) < kKT ? (j1 - t0) : kKT);
            const int buf = static_cast<int>(t & 1);
            wait(&x.s_full[buf], static_cast<uint32_t>((t >> 1) & 1));
            fence_after();
            uint32_t sr[HG];
            tmem_ld_x<HG>(x.tmem + lane_addr + static_cast<uint32_t>(buf * NQ + hb), sr);
            tmem_wait_ld();

            if (rows < kKT && (!kSplit || grp == 0)) {
                // keys past the piece end: p is 0 there, and 0 * NaN would poison
                // O^T, so zero those V rows before the P V product reads them
                const int stg = static_cast<int>(t % C::kStages);
                unsigned char* vb = smem + C::kOffKV + stg * C::kStageBytes + C::kOffVAtoms;
                // 16-byte unit u: row rows + u / (8 kAtoms), atom (u / 8) % kAtoms, chunk u % 8
#pragma unroll 1
                for (int u = st; u < (kKT - rows) * 8 * C::kAtoms; u += kKGroup)
                    *reinterpret_cast<uint4*>(vb + ((u >> 3) % C::kAtoms) * C::kKVAtom +
                                              swz(rows + u / (8 * C::kAtoms), u & 7)) =
                        make_uint4(0, 0, 0, 0);
                fence_proxy_async_smem();
            }

            // e = score - running max, in log2 units (one fma; the first tile of
            // a piece, with m = -inf, gives +inf and always moves the max); keys
            // past the piece end are -inf (the select also drops whatever those
            // K rows hold)
            float e[HG];
            bool need = false;
            const bool kvalid = key < rows;
            const float jpos = static_cast<float>(t0 + key - w.len + 1);
            auto scores = [&](bool masked, bool absolute) {
#pragma unroll
                for (int h = 0; h < HG; ++h) {
                    const float raw = __uint_as_float(sr[h]);
                    const float base = absolute ? 0.f : -m_ref[h];
                    float v = p.slopes ? fmaf(raw, qscale2, fmaf(slope2[h], jpos, base))
                                       : fmaf(raw, qscale2, base);
                    if (masked) v = kvalid ? v : kNegInf;
                    e[h] = v;
                    need |= v > kKRescale;
                }
            };
            if (rows == kKT)
                scores(false, false);
            else
                scores(true, false);
            if (bar_any(bar_grp, kKGroup, need)) {
                // move the group's max to the tile max of every head: the
                // absolute scores again from TMEM (the S buffer is released below)
                tmem_ld_x<HG>(x.tmem + lane_addr + static_cast<uint32_t>(buf * NQ + hb), sr);
                tmem_wait_ld();
                if (rows == kKT)
                    scores(false, true);
                else
                    scores(true, true);
#pragma unroll
                for (int h = 0; h < HG; ++h) {
                    float mx = e[h];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    if (lane == 0) red[quarter * GP + h] = mx;
                }
                named_bar_sync(bar_grp, kKGroup);
                // O^T holds earlier tiles of the piece once a P V product of this
                // group's columns was issued: tile t - 2 (own tiles alternate) or
                // t - 1 (every tile)
                const long long prev = kSplit ? (i > 0 ? t - 1 : -1) : last_own;
                uint32_t o[HG];
                if (prev >= 0) {
                    wait_pv(prev);
                    fence_after();
                    tmem_ld_x<HG>(x.tmem + lane_addr + o_col, o);
                    tmem_wait_ld();
                }
#pragma unroll
                for (int h = 0; h < HG; ++h) {
                    const float tm = fmaxf(fmaxf(red[h], red[GP + h]),
                                           fmaxf(red[2 * GP + h], red[3 * GP + h]));
                    const float mn = fmaxf(m_ref[h], tm);
                    const float f = rescale(m_ref[h], mn);
                    if (hb + h < G) {
                        m_ref[h] = mn;
                        lx[h] *= f;
                        if (prev >= 0) o[h] = __float_as_uint(__uint_as_float(o[h]) * f);
                    }
                    e[h] -= m_ref[h];
                }
                if (prev >= 0) {
                    tmem_st_x<HG>(x.tmem + lane_addr + o_col, o);
                    tmem_wait_st();
                }
                // the maxima are read before any thread of the group can pass
                // the next tile's reduction and overwrite them
            }
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&x.s_empty[buf]));
            // the P V product of tile t - 2 read this P^T buffer
            if (t >= 2) wait_pv(t - 2);
            fence_after();
            unsigned char* pb = smem + C::kOffP + buf * C::kPBytes + p_off;
#pragma unroll
            for (int h = 0; h < HG; ++h) {
                // masked keys give ex2(-inf) = 0
                const float ev = ex2(e[h]);
                round_store<E>(ev, pb + h * 128 + ((kc2 ^ (h & 7)) << 4));
                lx[h] += ev;
            }
            fence_proxy_async_smem();
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&x.p_full[buf]));
            last_own = t;
        }

        // ---- end of piece: the last P V product into this group's O^T columns
        // must be complete
        if (last_own >= 0) {
            wait_pv(last_own);
            fence_after();
        }
        // The epilogue runs once per piece, so its code is kept compact (head
        // loops are not unrolled): it would otherwise be fetched cold into the
        // instruction cache while the other SMs saturate L2 with K/V traffic.
        // The group's sums of p per head, reduced through shared memory in a
        // fixed order: [head][thread] -> kKGroup / HG partials per head -> one
        // sum per head.  Group g uses P^T buffer g, which no P V product reads
        // any more: in alternate mode it is the group's own buffer and its last
        // product is complete; in split mode every product of the piece is.
        // p is normalised by its unrounded sum (l = lx): sum_k r_k v_k / sum_k
        // p_k differs from the exact average by at most the relative rounding of
        // r times max |v|, as the rounded sum would.
        constexpr int TPH = kKGroup / HG;  // partials per head
        static_assert(kKGroup * HG * 4 <= C::kPBytes, "sum scratch");
        float* lsum = reinterpret_cast<float*>(smem + C::kOffP + grp * C::kPBytes);
#pragma unroll
        for (int u = 0; u < HG; ++u) lsum[u * kKGroup + st] = lx[u];
        if (st == 0) {
#pragma unroll
            for (int u = 0; u < HG; ++u) st_m[grp * GP + hb + u] = m_ref[u];
        }
        named_bar_sync(bar_grp, kKGroup);
        {
            const int u = st / TPH;
            float b = 0.f;
#pragma unroll 1
            for (int r = st % TPH; r < kKGroup; r += TPH) b += lsum[u * kKGroup + r];
            named_bar_sync(bar_grp, kKGroup);
            lsum[st] = b;  // [head][partial]
        }
        named_bar_sync(bar_grp, kKGroup);
        if (st < HG) {
            float b = 0.f;
#pragma unroll 1
            for (int r = 0; r < TPH; ++r) b += lsum[st * TPH + r];
            st_l[grp * GP + hb + st] = hb + st < G ? b : 0.f;
            if (kSplit) {
                // the other group's heads: nothing from this group
                const int ob = grp == 0 ? HG : 0;
                st_l[grp * GP + ob + st] = 0.f;
                st_m[grp * GP + ob + st] = kNegInf;
            }
        }
        fence_before();
        named_bar_sync(kBarBoth, 2 * kKGroup);
        fence_after();
        // a group's O^T is stale when it had no tile of this piece
        const long long t_first = t - nt;
        const bool has0 = kSplit || nt >= 2 || (t_first & 1) == 0;
        const bool has1 = !kSplit && (nt >= 2 || (t_first & 1) == 1);
        const int slot = pc == 0 ? 0 : 1;  // the CTA's first piece uses slot 0
        float* const part0 = p.part + ((x.c * 2 + slot) * Gall + h_off) * (D + 3);
        // per head, once: the merged max M and sum L of both groups, and the
        // weights of the two O^T accumulators in the output (split mode: one
        // accumulator, already relative to the owning group's max)
        float* hs = stats + 8 * GP;  // [head][2]
        if (grp == 0 && st < G) {
            const int h = st;
            const float m0 = st_m[h], m1 = st_m[GP + h];
            const float M = fmaxf(m0, m1);
            const float w0 = rescale(m0, M), w1 = rescale(m1, M);
            const float L = w0 * st_l[h] + w1 * st_l[GP + h];
            float a0 = kSplit ? 1.f : w0, a1 = kSplit ? 0.f : w1;
            if (whole) {
                a0 /= L;
                a1 /= L;
                if (p.lse) p.lse[qrow + h] = (M + log2f(L)) * kLn2;
            } else {
                float* rec = part0 + h * (D + 3);
                rec[D] = M;
                rec[D + 1] = L;
                rec[D + 2] = L;
            }
            hs[2 * h] = has0 ? a0 : 0.f;
            hs[2 * h + 1] = has1 ? a1 : 0.f;
        }
        named_bar_sync(kBarBoth, 2 * kKGroup);
        // row `key` of O^T for every head, four heads per TMEM load, the two
        // groups taking alternate blocks of four
#pragma unroll 1
        for (int h0 = grp * 4; h0 < G; h0 += 8) {
            uint32_t o0[4], o1[4];
            if (has0) tmem_ld_x<4>(x.tmem + lane_addr + static_cast<uint32_t>(2 * NQ + h0), o0);
            if (has1) tmem_ld_x<4>(x.tmem + lane_addr + static_cast<uint32_t>(3 * NQ + h0), o1);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int h = h0 + j;
                // O^T rows >= D (D = 64) are not part of the result
                if (h < G && key < D) {
                    float v = has0 ? __uint_as_float(o0[j]) * hs[2 * h] : 0.f;
                    if (has1) v = fmaf(hs[2 * h + 1], __uint_as_float(o1[j]), v);
                    if (whole)
                        p.out[(qrow + h) * D + key] = v;
                    else
                        part0[h * (D + 3) + key] = v;
                }
            }
        }
        fence_before();
        if (!p.fused_merge) {
            // the CTA holding the sequence's first key describes its parts for
            // the combine kernel (one part: already written, nothing to merge)
            if (grp == 0 && j0 == 0 && st == 0 && h_off == 0) {
                const long long seg = static_cast<long long>(w.b) * p.Hkv + w.h;
                const long long c_lo = gpart_of(w.start, x.T, x.P);
                const long long c_hi = gpart_of(w.start + w.len - 1, x.T, x.P);
                p.seg_desc[seg * 3 + 0] = static_cast<int>(c_lo);
                p.seg_desc[seg * 3 + 1] = static_cast<int>(c_hi - c_lo + 1);
                p.seg_desc[seg * 3 + 2] = gpart_start(c_lo, x.T, x.P) < w.start ? 1 : 0;
            }
        } else if (!whole) {
            // both groups wrote records: make them visible, then take the ticket
            __threadfence();
            named_bar_sync(kBarBoth, 2 * kKGroup);
            if (grp == 0) {
                const long long c_lo = gpart_of(w.start, x.T, x.P);
                const long long c_hi = gpart_of(w.start + w.len - 1, x.T, x.P);
                // every chunk CTA of every part of the sequence takes a ticket
                const int n = static_cast<int>(c_hi - c_lo + 1) * p.chunks;
                const long long seg = static_cast<long long>(w.b) * p.Hkv + w.h;
                if (st == 0) {
                    const int prev = atomicAdd(p.tickets + seg, 1);
                    const int last = prev == n - 1;
                    if (last) atomicExch(p.tickets + seg, 0);
                    x.ctl->last = last;
                }
                named_bar_sync(kBarG0, kKGroup);
                if (x.ctl->last) {
                    __threadfence();
                    const int first_slot = gpart_start(c_lo, x.T, x.P) < w.start ? 1 : 0;
                    const int nparts = n / p.chunks;
                    for (int gg = 0; gg < Gall; ++gg) {
                        const GSlotAcc acc{p.part, c_lo, first_slot, Gall, gg, D};
                        tree_merge(acc, nparts, D, st, kKGroup, scratch, kKScratch, kBarG0,
                                   p.out + (qrow0 + gg) * D, p.lse ? p.lse + qrow0 + gg : nullptr);
                    }
                }
                named_bar_sync(kBarG0, kKGroup);
            }
        }
        ++pc;
    } while (gwalk_next(p, *x.ctl, w));
}

// ------------------------------------------------------------------ kernel

template <typename E, int GP, bool kSplit, int D>
__global__ void __launch_bounds__(kKThreads, KCfg<GP, D>::kCtasPerSm)
    td_gqa_keys_kernel(const GqaParams p, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV) {
    using C = KCfg<GP, D>;
    constexpr int NQ = C::NQ;
    constexpr int kKStages = C::kStages;
    constexpr bool kBF16 = std::is_same<E, __nv_bfloat16>::value;
    extern __shared__ unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled operand blocks
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    __shared__ __align__(8) uint64_t kv_full[kKStages], kv_empty[kKStages];
    __shared__ __align__(8) uint64_t s_full[2], s_empty[2], p_full[2], pv_done[2], q_ready;
    __shared__ GCtl ctl;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // part c and head chunk of this CTA (chunks of a part are adjacent)
    const long long c = blockIdx.x / p.chunks;
    const int chunk = static_cast<int>(blockIdx.x % p.chunks);
    const int h_off = chunk * p.gc;
    const int g_eff = p.G - h_off < p.gc ? p.G - h_off : p.gc;
    const long long P = p.P;

    if (tid == 0) {
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(smem_addr(&kv_full[s]), 1);
            mbar_init(smem_addr(&kv_empty[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&s_full[s]), 1);
            // one arrival per softmax warp that reads S / writes P of the tile
            mbar_init(smem_addr(&s_empty[s]), kSplit ? 8 : 4);
            mbar_init(smem_addr(&p_full[s]), kSplit ? 8 : 4);
            mbar_init(smem_addr(&pv_done[s]), 1);
        }
        mbar_init(smem_addr(&q_ready), 8);
        fence_barrier_init();
        ctl.abort = 0;
        ctl.last = 0;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_addr(&ctl.tmem)), "r"(C::kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (warp >= 2) {
        // Q and both P^T buffers start at zero (rows >= G stay zero)
        uint4* z = reinterpret_cast<uint4*>(smem + C::kOffQ);
        const int n16 = (C::kQBytes + 2 * C::kPBytes) / 16;
        for (int i = tid - 64; i < n16; i += kKThreads - 64) z[i] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
    }
    gqa_partition(p, ctl, c, tid, warp, lane, kKThreads, D);
    fence_before();
    __syncthreads();
    fence_after();
    // the merge kernel that follows may be scheduled now; it waits for this
    // grid's completion before it reads any record
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

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
                    for (long long t0 = j0; t0 < j1; t0 += kKT) {
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
                                tma_load_2d(base + C::kOffKAtoms + a * C::kKVAtom, &tmK, 64 * a,
                                            y, fb, pol);
                                tma_load_2d(base + C::kOffVAtoms + a * C::kKVAtom, &tmV, 64 * a,
                                            y, fb, pol);
                            }
                            ++issued;
                        }
                        if (++stage == kKStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                } while (gwalk_next(p, ctl, w));
            }
            // the CTA must not exit with copies into its shared memory in flight
            for (int s = 0; s < kKStages && s < issued; ++s) {
                const long long lastTile = s + ((issued - 1 - s) / kKStages) * kKStages;
                mbar_wait_bounded(smem_addr(&kv_full[s]),
                                  static_cast<uint32_t>((lastTile / kKStages) & 1), nullptr,
                                  p.err, TD_DEVERR_WAIT_TIMEOUT);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA
        if (lane == 0) {
            // S^T: A = K tile (K-major), B = Q (K-major); O^T: A = V^T (V tile,
            // D contiguous: MN-major), B = P^T (K-major)
            constexpr uint32_t idS = instr_desc_f16(kBF16 ? 1 : 0, kKT, NQ, 0, 0);
            constexpr uint32_t idO = instr_desc_f16(kBF16 ? 1 : 0, kKMO, NQ, 1, 0);
            long long t = 0;    // tiles so far (global)
            long long pc = 0;   // pieces so far
            bool aborted = false;
            long long last_pv = -1;
            GWalk w;
            if (gwalk_first(p, ctl, w)) {
                do {
                    const long long j0 = (x0 > w.start ? x0 : w.start) - w.start;
                    const long long e = w.start + w.len;
                    const long long j1 = (x1 < e ? x1 : e) - w.start;
                    const long long nt = (j1 - j0 + kKT - 1) / kKT;
                    if (!aborted &&
                        !mbar_wait_bounded(smem_addr(&q_ready), static_cast<uint32_t>(pc & 1),
                                           abort_flag, p.err, TD_DEVERR_WAIT_TIMEOUT))
                        aborted = true;
                    fence_after();
                    // S products are issued in order as soon as their K tile has
                    // landed and their S buffer is free; P V products in order as
                    // soon as their P^T is written
                    const long long t_end = t + nt;
                    long long ts = t;
                    long long tp = t;
                    uint64_t t_stall = 0;
                    uint32_t spins = 0;
                    while (tp < t_end && !aborted) {
                        bool progressed = false;
                        if (ts < t_end &&
                            mbar_test(smem_addr(&kv_full[ts % kKStages]),
                                      static_cast<uint32_t>((ts / kKStages) & 1)) &&
                            (ts < 2 || mbar_test(smem_addr(&s_empty[ts & 1]),
                                                 static_cast<uint32_t>(((ts >> 1) - 1) & 1)))) {
                            fence_after();
                            const uint32_t kb = sKV + static_cast<uint32_t>(ts % kKStages) *
                                                          C::kStageBytes;
                            const uint32_t dS = tmem + static_cast<uint32_t>((ts & 1) * NQ);
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint32_t off = static_cast<uint32_t>((kk & 3) * 32);
                                const uint64_t a = smem_desc_sw128(
                                    kb + C::kOffKAtoms + (kk >> 2) * C::kKVAtom + off, 16, 1024);
                                const uint64_t b =
                                    smem_desc_sw128(sQ + (kk >> 2) * C::kQAtom + off, 16, 1024);
                                umma_f16(dS, a, b, idS, kk > 0 ? 1u : 0u);
                            }
                            umma_commit(smem_addr(&s_full[ts & 1]));
                            ++ts;
                            progressed = true;
                        }
                        if (tp < ts && mbar_test(smem_addr(&p_full[tp & 1]),
                                                 static_cast<uint32_t>((tp >> 1) & 1))) {
                            fence_after();
                            const long long i = tp - t;
                            const int stage = static_cast<int>(tp % kKStages);
                            const uint32_t vb = sKV + stage * C::kStageBytes + C::kOffVAtoms;
                            const uint32_t pb = sP + static_cast<uint32_t>((tp & 1) * C::kPBytes);
                            // one O^T per group (tiles alternate), or one shared
                            const uint32_t dO = tmem + static_cast<uint32_t>(
                                                           2 * NQ + (kSplit ? 0 : (tp & 1) * NQ));
#pragma unroll
                            for (int kk = 0; kk < kKT / 16; ++kk) {
                                // 16 keys: rows 16 kk.. of the V tile; the two
                                // 64-row halves of M are kKVAtom apart (D = 64:
                                // the second is the K tile, rows never read)
                                const uint64_t a =
                                    smem_desc_sw128(vb + kk * 2048, C::kKVAtom, 1024);
                                const uint64_t b = smem_desc_sw128(
                                    pb + (kk >> 2) * C::kPAtom + (kk & 3) * 32, 16, 1024);
                                // the first tile of the piece into an accumulator starts it
                                const bool acc = (kSplit ? i > 0 : i > 1) || kk > 0;
                                umma_f16(dO, a, b, idO, acc ? 1u : 0u);
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
                            continue;
                        }
                        // nothing ready: sleep briefly on the barrier the next
                        // product is most likely waiting for
                        if (tp < ts)
                            mbar_try_wait_ns(smem_addr(&p_full[tp & 1]),
                                             static_cast<uint32_t>((tp >> 1) & 1), 64);
                        else if (ts < t_end)
                            mbar_try_wait_ns(smem_addr(&kv_full[ts % kKStages]),
                                             static_cast<uint32_t>((ts / kKStages) & 1), 64);
                        if ((++spins & 15u) == 0u) {
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
        const KCtx kx{g_eff, h_off, smem, s_full, s_empty, p_full, pv_done, &q_ready, &ctl,
                      abort_flag, tmem, T, x0, x1, P, c, warp, lane, tid};
        keys_softmax<E, GP, kSplit, D>(p, kx);
    }

    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(C::kTmemCols) : "memory");
    }
}

template <typename E, int GP, bool kSplit, int D>
cudaError_t launch_keys_t(int device, const GqaParams& p, const CUtensorMap& mk,
                          const CUtensorMap& mv, cudaStream_t s) {
    using C = KCfg<GP, D>;
    auto kern = td_gqa_keys_kernel<E, GP, kSplit, D>;
    static std::atomic<unsigned long long> configured{0};
    const unsigned long long bit = device < 64 ? (1ull << device) : 0ull;
    if (!bit || !(configured.load(std::memory_order_acquire) & bit)) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::kSmem));
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    kern<<<static_cast<unsigned>(p.P * p.chunks), kKThreads, C::kSmem, s>>>(p, mk, mv);
    return cudaGetLastError();
}

template <typename E, int D>
cudaError_t launch_keys_g(int device, const GqaParams& p, const CUtensorMap& mk,
                          const CUtensorMap& mv, cudaStream_t s) {
    // up to 8 heads a thread keeps every head and the groups alternate tiles;
    // beyond, both groups take every tile with half the heads each
    if (p.gc <= 4) return launch_keys_t<E, 4, false, D>(device, p, mk, mv, s);
    if (p.gc <= 8) return launch_keys_t<E, 8, false, D>(device, p, mk, mv, s);
    if (p.gc <= 16) return launch_keys_t<E, 16, true, D>(device, p, mk, mv, s);
    return launch_keys_t<E, 32, true, D>(device, p, mk, mv, s);
}

template <int D>
size_t keys_smem(int G) {
    return G <= 4 ? KCfg<4, D>::kSmem : G <= 8 ? KCfg<8, D>::kSmem
                                               : G <= 16 ? KCfg<16, D>::kSmem
                                                         : KCfg<32, D>::kSmem;
}

}  // namespace

bool gqa_keys_path(int D, int G) { return (D == 64 || D == 128) && G >= 1 && G <= 128; }

int gqa_keys_chunks(int G) { return (G + 31) / 32; }

int gqa_keys_ctas_per_sm(int D, int gc) {
    if (D == 64)
        return gc <= 4 ? KCfg<4, 64>::kCtasPerSm : gc <= 8 ? KCfg<8, 64>::kCtasPerSm
               : gc <= 16 ? KCfg<16, 64>::kCtasPerSm : KCfg<32, 64>::kCtasPerSm;
    return 1;
}

size_t gqa_keys_smem_bytes(int D, int G) {
    return D == 64 ? keys_smem<64>(G) : D == 128 ? keys_smem<128>(G) : 0;
}

cudaError_t launch_gqa_keys(int device, int dtype, int D, const GqaParams& p,
                            const CUtensorMap& mk, const CUtensorMap& mv, cudaStream_t s) {
    if (D == 128) {
        if (dtype == kBF16) return launch_keys_g<__nv_bfloat16, 128>(device, p, mk, mv, s);
        if (dtype == kF16) return launch_keys_g<__half, 128>(device, p, mk, mv, s);
    } else if (D == 64) {
        if (dtype == kBF16) return launch_keys_g<__nv_bfloat16, 64>(device, p, mk, mv, s);
        if (dtype == kF16) return launch_keys_g<__half, 64>(device, p, mk, mv, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace td
