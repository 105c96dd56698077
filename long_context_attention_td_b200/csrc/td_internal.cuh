// Internal declarations shared by the kernels and the host entry points of
// libtreedec.  Not part of the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace td {

// Element types (same numbering as td_dtype).
enum : int { kF32 = 0, kBF16 = 1, kF16 = 2, kE4M3 = 3 };  // kE4M3: K/V storage only

// Shape of the split-KV kernel's pipeline (compile-time; the defaults are the
// tuned values, the macros exist for tuning sweeps).
#ifndef TD_CONSUMER_WARPS
#define TD_CONSUMER_WARPS 8
#endif
#ifndef TD_STAGES
#define TD_STAGES 2
#endif
#ifndef TD_STAGE_BYTES
#define TD_STAGE_BYTES 32768
#endif
#ifndef TD_CTAS_PER_SM
#define TD_CTAS_PER_SM 3
#endif

// Consumer warps per CTA of the split-KV kernel, plus one producer warp.
constexpr int kConsumerWarps = TD_CONSUMER_WARPS;
constexpr int kConsumerThreads = 32 * kConsumerWarps;
constexpr int kPartialThreads = kConsumerThreads + 32;
// Pipeline depth of the split-KV kernel (stages of K+V tiles in shared memory).
constexpr int kStages = TD_STAGES;
// Bytes of K+V rows one pipeline stage holds (the tile is sized to this).
constexpr int kStageBytes = TD_STAGE_BYTES;
// CTAs of the split-KV kernel meant to share one SM (launch bounds).
constexpr int kCtasPerSm = TD_CTAS_PER_SM;
// Smallest part the heuristic creates (bytes of K+V).
constexpr int64_t kMinPartBytes = 65536;

// Workspace layout: [error word | pad to 256 B][tickets: B*H int32, padded to
// 256 B][part records: parts * 2 * (D + 2) fp32].
constexpr size_t kErrRegion = 256;

struct PartialParams {
    const void* q;
    const void* k;
    const void* v;
    float* out;
    float* lse;              // may be null
    const float* slopes;     // may be null
    const int32_t* seqlens;  // null: every sequence has N keys
    int B, H;
    int64_t N;               // keys per sequence, or the padded Nmax when ragged
    int64_t T;               // total attended keys when known (uniform), else -1
    int64_t P;               // parts == grid size
    float qscale2;           // D^-1/2 * log2(e)
    float* part;             // part records
    int* tickets;            // [B*H]
    int* err;                // error word
    int64_t alibi_off;       // ALiBi position of key j is j - n + 1 + alibi_off (0: the
                             // sequence is whole; a shard adds its place in the full one)
    const float* k_scale;    // FP8 K/V: per-head dequantisation scales [H] (else null)
    const float* v_scale;
    unsigned long long wait_ns;  // limit of every pipeline wait (ns)
    long long withhold_tile;     // >= 0: CTA 0's producer arms no stage from this tile on
                                 // (tests the bounded-wait failure path); -1: off
};

// Grouped-query decode (td_gqa_keys.cu, merge in td_gqa_combine.cu): Hq = G * Hkv
// query heads over Hkv kv heads.
struct GqaParams {
    const void* q;           // [B, Hq, 1, D]
    float* out;              // [B, Hq, 1, D]
    float* lse;              // [B, Hq, 1] or null
    const float* slopes;     // [Hq] or null
    const int32_t* seqlens;  // [B] or null
    int B, Hq, Hkv, G;
    int64_t N;               // keys per sequence, or the padded Nmax
    int64_t T;               // attended keys over all (b, kv head) when uniform, else -1
    int64_t P;               // parts == grid size
    float qscale2;           // D^-1/2 * log2(e)
    float* part;             // part records [P][2][G][D + 3]
    int* tickets;            // [B * Hkv]
    int* seg_desc;           // [B * Hkv][3]: first part, parts, slot of the first part
    int fused_merge;         // 1: last CTA merges (ticket); 0: td_gqa_combine merges
    int* err;
    int chunks;              // keys-on-M kernel: the group's heads in this many chunks,
    int gc;                  // of gc heads (the last may be shorter), one CTA per (part,
                             // chunk); 1 and G otherwise
};
// Merge the part records of every split sequence (p.fused_merge == 0).
cudaError_t launch_gqa_combine(int D, const GqaParams& p, cudaStream_t s);
// The grouped-query kernel, keys on the MMA M axis (td_gqa_keys.cu), for D == 64
// or 128 and G <= 128 (groups of more than 32 heads in chunks of at most 32,
// one CTA per part and chunk); its K and V tensor maps are 2-D [B*Hkv*N rows,
// D columns] with boxes of {64 columns, 128 rows} and 128-byte swizzle.
bool gqa_keys_path(int D, int G);
// head chunks of a group of G and heads per chunk on that kernel
int gqa_keys_chunks(int G);
// CTAs of that kernel that share one SM (its launch bounds) for chunks of gc heads
int gqa_keys_ctas_per_sm(int D, int gc);
size_t gqa_keys_smem_bytes(int D, int G);
cudaError_t launch_gqa_keys(int device, int dtype, int D, const GqaParams& p,
                            const CUtensorMap& mk, const CUtensorMap& mv, cudaStream_t s);

// The split-KV kernel over an FP8 E4M3 K/V cache, q of type q_dtype (kBF16, kF16).
cudaError_t launch_partial_fp8(int device, int q_dtype, int D, const PartialParams& p,
                               cudaStream_t s);

// Dynamic shared memory of the split-KV kernel for (K/V dtype, D).
size_t partial_smem_bytes(int dtype, int D);
// CTAs of the split-KV kernel that fit on one SM (static estimate from shared
// memory and threads; matches the kernel's launch bounds).
int partial_ctas_per_sm(int dtype, int D);
// Prefill kernel (td_prefill.cu): every query row of B*H sequences of S tokens.
struct PrefillParams {
    float* out;              // [B, H, S, D]
    float* lse;              // [B, H, S] or null
    const float* slopes;     // [H] or null
    int B, H;
    int64_t S;
    int causal;
    float qscale2;           // D^-1/2 * log2(e)
    int* err;
};
// Q, K, V tensor maps: 3-D [B*H, S, D], box {64, 128, 1}, 128-byte swizzle.
cudaError_t launch_prefill(int device, int dtype, int D, const PrefillParams& p,
                           const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                           cudaStream_t s);

// Empty partial state (out 0, lse -inf) of `rows` (b,h) rows: a shard with no keys.
cudaError_t launch_empty_state(float* out, float* lse, long long rows, int D, cudaStream_t s);
// Merge W gathered shard states [W][rows*D | rows] into out[rows][D], lse[rows].
cudaError_t launch_merge_shards(const float* states, int W, long long rows, int D, float* out,
                                float* lse, cudaStream_t s);

// Launch the split-KV kernel (grid = p.P) with its fused combine on `device`
// (the current device).
cudaError_t launch_partial(int device, int dtype, int D, const PartialParams& p, cudaStream_t s);
// Launch the standalone tree combine over dense partials.
cudaError_t launch_combine(const float* num, const float* m, const float* l, float* out,
                           float* lse, int64_t rows, int S, int D, cudaStream_t s);

}  // namespace td
