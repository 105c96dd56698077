/*
 * treedec.h -- C ABI of libtreedec: exact single-query (decode-step) softmax
 * attention over a long KV sequence on one NVIDIA B200 (sm_100a).
 *
 * The computation is the decode scheme of the "Tree Attention Decoding" gist
 * (tree_attn_decode.py, function tree_attn_decode, "Algorithm 3 proposed in
 * Tree Attention"): the key/value sequence is cut into parts, each part yields
 * a numerator num = sum_j e^(s_j - m) v_j, its local max m and denominator
 * l = sum_j e^(s_j - m), and the parts are merged by rescaling with
 * e^(m - max m) and summing (the gist's all-reduce MAX and two all-reduce
 * SUMs; the softmax decomposition and fusion formulas of "Flash Aandacht",
 * section "De Wiskunde Achter Flash Aandacht").  Here the parts are CTAs of
 * one GPU and the merge runs on the GPU.  The result equals plain attention
 * (the gist's regular_decode):
 *
 *   s_j  = (q . k_j) * D^-1/2 + slope_h * (j - n + 1)
 *   out  = sum_j softmax(s)_j v_j        lse = ln sum_j e^(s_j)
 *
 * where the optional ALiBi term is the broadcast bias row arange(1-n, 1)
 * times the head slope ("ALiBi with causal=True unexpected bias?",
 * llm-foundry issue #186), computed in registers: no bias tensor is read.
 *
 * Conventions shared by every entry point
 *   - Layout (row-major, contiguous): q [B,H,1,D], k and v [B,H,N,D],
 *     out [B,H,1,D] fp32, lse [B,H,1] fp32.  Element type of q, k, v: dtype.
 *   - Pointers named "device" must be CUDA device (or managed) memory on the
 *     current device; the caller owns all of them.  q, k, v must be 16-byte
 *     aligned; out, lse, slopes, seqlens 4-byte aligned.
 *   - D must be 64, 128, 256 or 512.
 *   - All work is enqueued on `stream`; no call synchronises the device
 *     except td_check_device_error, td_release_workspace and td_decode_host
 *     (which only waits on its own stream when asked to).
 *   - Errors are returned as td_status; arguments are validated on the host
 *     before anything is launched, and a rejected call launches nothing.
 *   - The library-owned workspace is per device and grows on demand (a
 *     cudaMalloc on growth: make the first call of a given size outside
 *     stream capture).  Calls that share it must be ordered on one stream;
 *     for concurrent streams give each its own workspace (td_decode_ws).
 */
#ifndef TREEDEC_H
#define TREEDEC_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TD_API __attribute__((visibility("default")))
#else
#define TD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA stream type (identical to cudaStream_t / CUstream). */
struct CUstream_st;
typedef struct CUstream_st *td_stream;

typedef enum { TD_F32 = 0, TD_BF16 = 1, TD_F16 = 2 } td_dtype;

typedef enum {
    TD_OK = 0,
    TD_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, overflow   */
    TD_ERR_UNSUPPORTED = 2, /* D or dtype outside the compiled set           */
    TD_ERR_CUDA = 3,        /* a CUDA runtime call failed: td_last_cuda_error */
    TD_ERR_NO_MEMORY = 4,   /* workspace allocation failed                   */
    TD_ERR_DEVICE = 5,      /* a kernel reported an error word (see below)    */
    TD_ERR_WORKSPACE = 6    /* caller workspace too small                     */
} td_status;

/* Device error word bits reported through td_check_device_error. */
#define TD_DEVERR_WAIT_TIMEOUT 0x1 /* a bounded pipeline wait ran out        */
#define TD_DEVERR_BAD_SEQLEN 0x2   /* a seqlens[b] outside [0, Nmax], clamped */

/*
 * td_decode -- decode attention for every (b,h): q[b,h] against the N keys of
 * k[b,h] and values of v[b,h]  (gist: tree_attn_decode / regular_decode).
 *   q, k, v   device, dtype, layouts above.
 *   out       device fp32 [B,H,1,D]; lse device fp32 [B,H,1] or NULL.
 *   N >= 1    keys per sequence.
 *   n_split   0: the library's split heuristic (td_auto_split) over the whole
 *             flattened key space; > 0: each (b,h) is cut into
 *             min(n_split, N) parts of balanced length (the gist's one chunk
 *             per rank).  The result is the same to rounding either way.
 *   alibi_slopes  device fp32 [H] (per-head slope) or NULL for no bias.
 * Uses the library-owned per-device workspace.
 */
TD_API td_status td_decode(const void *q, const void *k, const void *v, float *out, float *lse,
                    int B, int H, int64_t N, int D, int n_split,
                    const float *alibi_slopes, td_dtype dtype, td_stream stream);

/*
 * td_decode_fp8 -- td_decode / td_decode_varlen over an FP8 K/V cache: k8, v8
 * device [B,H,Nmax,D] bytes holding OCP FP8 E4M3 codes (1 sign, 4 exponent
 * bits with bias 7, 3 fraction bits; no infinities), dequantised per head as
 * K = e4m3(k8) * k_scale[h], V = e4m3(v8) * v_scale[h] (k_scale, v_scale
 * device fp32 [H]).  The result is the attention of q (q_dtype TD_BF16 or
 * TD_F16) over those dequantised K, V.  seqlens/seqlens_host as
 * td_decode_varlen (NULL: every sequence has Nmax keys); other arguments and
 * errors as td_decode.  Arithmetic: q.k and p v are multiply-added in half
 * precision (8-term chains for q.k with q pre-scaled by a power of two; at most
 * a tile's rows for p v, then fp32), softmax and sums in fp32.
 */
TD_API td_status td_decode_fp8(const void *q, const void *k8, const void *v8, const float *k_scale,
                               const float *v_scale, float *out, float *lse, int B, int H,
                               int64_t Nmax, int D, const int32_t *seqlens,
                               const int32_t *seqlens_host, int n_split,
                               const float *alibi_slopes, td_dtype q_dtype, td_stream stream);

/*
 * td_decode_varlen -- as td_decode for a batch of sequences of different
 * lengths stored padded: k, v [B,H,Nmax,D]; sequence b attends to its first
 * seqlens[b] keys and the ALiBi term uses n = seqlens[b].
 *   seqlens       device int32 [B], 0 <= seqlens[b] <= Nmax (a value outside
 *                 is clamped and flagged with TD_DEVERR_BAD_SEQLEN).  A length
 *                 of 0 gives out = 0 and lse = -inf.
 *   seqlens_host  optional host copy of the same lengths (or NULL); when given
 *                 the heuristic sizes the split from the true key count.
 *   n_split       0: heuristic; > 0: B*H*n_split parts over the flattened
 *                 (b, h, key) space of attended keys.
 * Keys at positions >= seqlens[b] are never read.
 */
TD_API td_status td_decode_varlen(const void *q, const void *k, const void *v, float *out,
                           float *lse, int B, int H, int64_t Nmax, int D,
                           const int32_t *seqlens, const int32_t *seqlens_host, int n_split,
                           const float *alibi_slopes, td_dtype dtype, td_stream stream);

/*
 * td_decode_ws -- the general form with a caller-owned workspace and an
 * explicit part count.
 *   seqlens / seqlens_host  as td_decode_varlen, or both NULL (every sequence
 *                 has N keys).
 *   parts         total number of parts over the flattened (b, h, key) space
 *                 (one CTA each): 0 = heuristic.  Part c covers the flattened
 *                 keys [floor(c*T/parts), floor((c+1)*T/parts)) where T is the
 *                 number of attended keys; parts = B*H*n gives exactly n
 *                 balanced parts per (b,h) when all lengths are equal.
 *   workspace     device, at least td_workspace_bytes(B, H, D, parts_used)
 *                 bytes (parts_used = the heuristic's value when parts = 0:
 *                 ask td_plan_parts), zero-filled before its first use; the
 *                 kernels leave it ready for the next call (a call with a
 *                 larger B*H than the workspace has served re-zeroes its
 *                 ticket region on `stream` first).  Calls sharing one
 *                 workspace must be ordered on one stream.
 */
TD_API td_status td_decode_ws(const void *q, const void *k, const void *v, float *out, float *lse,
                       int B, int H, int64_t N, int D, const int32_t *seqlens,
                       const int32_t *seqlens_host, int64_t parts,
                       const float *alibi_slopes, td_dtype dtype, void *workspace,
                       size_t workspace_bytes, td_stream stream);

/*
 * td_decode_gqa -- grouped-query (and multi-query) decode: Hq query heads
 * share Hkv key/value heads, query head h attending to kv head h / (Hq/Hkv)
 * (the pages' per-head decode with the key/value tile shared by the G =
 * Hq/Hkv queries of a group; Hkv = 1 is multi-query attention).  Each K/V
 * tile is read once for its G queries and the two products S = Q K^T and
 * P V run on the tensor cores (tcgen05), with fp32 accumulation; p is rounded
 * to the input element type before P V (error ~2^-9 relative for bf16).
 *   q        device [B,Hq,1,D]; k, v device [B,Hkv,N,D] (padded Nmax when
 *            seqlens is given); dtype TD_BF16 or TD_F16; D 64 or 128;
 *            1 <= Hq/Hkv <= 128; B*Hkv*N < 2^31.
 *   out      device fp32 [B,Hq,1,D]; lse device fp32 [B,Hq,1] or NULL.
 *   seqlens / seqlens_host  as td_decode_varlen, or both NULL.
 *   n_split  0: heuristic; > 0: parts per (b, kv head) (equal lengths), or
 *            B*Hkv*n_split parts over the flattened keys (ragged).
 *   alibi_slopes  device fp32 [Hq] (per query head) or NULL.
 */
TD_API td_status td_decode_gqa(const void *q, const void *k, const void *v, float *out, float *lse,
                               int B, int Hq, int Hkv, int64_t N, int D, const int32_t *seqlens,
                               const int32_t *seqlens_host, int n_split,
                               const float *alibi_slopes, td_dtype dtype, td_stream stream);

/* td_decode_gqa with a caller-owned workspace (td_gqa_workspace_bytes) and an
 * explicit part count over the flattened (b, kv head, key) space (0 =
 * heuristic: td_plan_parts_gqa); same workspace rules as td_decode_ws. */
TD_API td_status td_decode_gqa_ws(const void *q, const void *k, const void *v, float *out,
                                  float *lse, int B, int Hq, int Hkv, int64_t N, int D,
                                  const int32_t *seqlens, const int32_t *seqlens_host,
                                  int64_t parts, const float *alibi_slopes, td_dtype dtype,
                                  void *workspace, size_t workspace_bytes, td_stream stream);

/* Part count td_decode_gqa would use on the current device (total_keys as in
 * td_plan_parts: < 0 for equal lengths Nmax); -1 on invalid arguments. */
TD_API int64_t td_plan_parts_gqa(int B, int Hq, int Hkv, int64_t Nmax, int D, td_dtype dtype,
                                 int n_split, int64_t total_keys);

/* Bytes of workspace td_decode_gqa_ws needs for `parts` parts. */
TD_API size_t td_gqa_workspace_bytes(int B, int Hq, int Hkv, int D, int64_t parts);

/*
 * td_combine -- merge caller-provided partials into the final output: the
 * gist's global max, renormalisation and two sums (tree_attn_decode after
 * "first get global max"), done per (b,h) as a log-depth tree on the GPU.
 *   num   device fp32 [B,H,S,D]: sum_j e^(s_j - m_s) v_j of part s;
 *   m     device fp32 [B,H,S]: the part's max score (natural-log units);
 *   l     device fp32 [B,H,S]: sum_j e^(s_j - m_s).
 *   An empty part is (num = 0, m = -inf, l = 0) and contributes nothing; if
 *   every part of a (b,h) is empty its out is 0 and lse is -inf.
 *   out   device fp32 [B,H,1,D]; lse device fp32 [B,H,1] or NULL.
 *   1 <= D <= 512, S >= 1.
 */
TD_API td_status td_combine(const float *num, const float *m, const float *l, float *out, float *lse,
                     int B, int H, int S, int D, td_stream stream);

/*
 * Sequence-sharded decode over several GPUs ("Tree Attention Decoding" gist,
 * tree_attn_decode: each rank holds one chunk of the keys, computes its local
 * partial attention, and the ranks exchange partial states to finish).  Here
 * the exchange is ONE all-gather of a packed state per rank, done by the
 * caller (e.g. NCCL through torch.distributed), instead of the gist's three
 * all-reduces:
 *   1. every rank: td_decode_shard on its keys -> its state buffer;
 *   2. all-gather the states of the W ranks into one [W][state] buffer;
 *   3. every rank: td_merge_shards -> out, lse of the whole sequence.
 *
 * td_decode_shard -- decode keys [key_offset, key_offset + N_shard) of every
 * (b,h) sequence of N_total keys, held in k, v device [B,H,N_shard,D]; q as for
 * td_decode.  ALiBi (alibi_slopes != NULL) uses each key's position in the
 * full sequence: slope_h (key_offset + j - N_total + 1) for key j of the shard.
 *   state  device fp32, B*H*(D+1) floats: the shard's normalised partial
 *          outputs [B*H][D], then their natural-log log-sum-exps [B*H].
 *   N_shard = 0 (a rank past the end of a short sequence, as torch.chunk can
 *   leave) writes the empty state: outputs 0, log-sum-exps -inf; k and v may
 *   then be NULL.
 *   n_split, dtype, D, stream: as td_decode.  Requires 0 <= key_offset,
 *   key_offset + N_shard <= N_total.  Errors as td_decode.
 *
 * td_merge_shards -- merge W gathered states (device fp32 [W][B*H*(D+1)], the
 * layout td_decode_shard writes, in any rank order) into out [B,H,1,D] and
 * lse [B,H,1] (may be NULL): the gist's global max, renormalisation and sums
 * with (num, m, l) = (out_r, lse_r, 1).  Empty states contribute nothing.
 * 1 <= D <= 512, W >= 1.
 */
TD_API td_status td_decode_shard(const void *q, const void *k, const void *v, float *state, int B,
                                 int H, int64_t N_shard, int D, int64_t key_offset,
                                 int64_t N_total, int n_split, const float *alibi_slopes,
                                 td_dtype dtype, td_stream stream);
TD_API td_status td_merge_shards(const float *states, int W, int B, int H, int D, float *out,
                                 float *lse, td_stream stream);

/*
 * td_prefill -- attention of every query row of B*H sequences of S tokens
 * (the step before decoding): for query i of head h,
 *   s_ij = q_i . k_j D^-1/2 + slope_h (j - S + 1)  over keys j <= i (causal != 0)
 *   or all keys (causal == 0); out_i = softmax_j(s_ij) . v, lse_i = ln sum_j e^s_ij.
 * The bias is the ALiBi broadcast row of "ALiBi with causal=True unexpected
 * bias?" over the whole sequence; the computation is the blockwise forward of
 * "Flash Aandacht" (running max and sum per query row over key blocks, the
 * running output rescaled by its old sum), on the tensor cores.
 *   q, k, v  device [B,H,S,D] bf16 or fp16 (dtype), row-major, 16-byte aligned;
 *   out      device fp32 [B,H,S,D], 16-byte aligned; lse device fp32 [B,H,S] or NULL;
 *   alibi_slopes device fp32 [H] or NULL.
 *   D in {64, 128}; 1 <= S <= 2^31 - 257; B*H*ceil(S/128) < 2^31.
 * Errors: TD_ERR_INVALID_ARG / TD_ERR_UNSUPPORTED before any launch; a bounded
 * wait that ran out sets TD_DEVERR_WAIT_TIMEOUT (td_check_device_error).
 */
TD_API td_status td_prefill(const void *q, const void *k, const void *v, float *out, float *lse,
                            int B, int H, int64_t S, int D, int causal,
                            const float *alibi_slopes, td_dtype dtype, td_stream stream);

/*
 * td_auto_split -- the split heuristic: the number of parts (CTAs) for T =
 * B*H*N attended keys on a GPU with num_sms SMs: enough to fill every SM with
 * as many CTAs as fit at once, but no part smaller than 64 KiB of K+V, no more
 * than floor(sqrt(0.62 * N * element bytes)) parts per sequence (beyond that
 * the merge of a sequence's parts by its last CTA costs more than the shorter
 * parts save: about 100 parts for N = 4096 fp32 keys), and never more parts
 * than keys.  Pure host arithmetic (no GPU needed).  Returns -1 on invalid
 * arguments.
 */
TD_API int64_t td_auto_split(int B, int H, int64_t N, int D, td_dtype dtype, int num_sms);

/*
 * td_plan_parts -- the part count the decode entry points use on the current
 * device.  total_keys < 0: equal lengths Nmax, td_decode's rule (n_split > 0
 * gives B*H*min(n_split, Nmax) parts).  total_keys >= 0: ragged lengths
 * summing to total_keys over all (b,h), td_decode_varlen's rule with
 * seqlens_host given (n_split > 0 gives B*H*n_split parts).  Either way
 * n_split = 0 means the heuristic, and the count is capped at the number of
 * keys.  Returns -1 on invalid arguments or when no device is available.
 */
TD_API int64_t td_plan_parts(int B, int H, int64_t Nmax, int D, td_dtype dtype, int n_split,
                      int64_t total_keys);

/*
 * td_decode_static -- td_decode that allocates nothing.  (The pages have no
 * counterpart: this entry point exists for callers of the library, not for
 * the method.)  Some callers cannot allocate device memory: serving engines
 * that reserve nearly all HBM for their KV-cache pool up front (a cudaMalloc
 * would fail or fragment the pool), host applications that own every device
 * allocation of a plug-in, and latency-critical decode loops that cannot
 * absorb the device-wide synchronisation of cudaMalloc/cudaFree.
 *   Arguments, layouts, results and error returns are those of td_decode; the
 *   caller still provides q, k, v, out and lse.  The workspace is a fixed
 *   array of TD_STATIC_SCRATCH_BYTES inside the library's device image (every
 *   GPU that loads the library holds it until the process exits); no
 *   cudaMalloc, cudaFree or other allocating routine is called.
 *   - A problem whose workspace (td_workspace_bytes for the part count
 *     td_plan_parts gives) exceeds TD_STATIC_SCRATCH_BYTES is rejected with
 *     TD_ERR_WORKSPACE before anything is launched (with the heuristic split
 *     on a B200 every D fits for B*H up to about 60,000, and D=128 up to about
 *     400,000; very large explicit n_split values may not).
 *   - The first call on a device sets up that device (looks up the array's
 *     address, zero-fills it and synchronises the device); make that first
 *     call before any stream capture.
 *   - Every call on a device shares the one array and it keeps the last call's
 *     contents (tickets are left at zero by each call).  Calls that overlap on
 *     the GPU -- on different streams, or from different threads without
 *     ordering -- race on it and give wrong results: order them on one stream.
 *   - Device error bits of these calls are kept in the array: read and clear
 *     them with td_check_static_error (td_check_device_error looks at the
 *     library-owned workspace instead).
 */
#define TD_STATIC_SCRATCH_BYTES (2u << 20)
TD_API td_status td_decode_static(const void *q, const void *k, const void *v, float *out,
                                  float *lse, int B, int H, int64_t N, int D, int n_split,
                                  const float *alibi_slopes, td_dtype dtype, td_stream stream);

/*
 * td_check_static_error -- td_check_device_error for the fixed array of
 * td_decode_static on the current device: waits for `stream`, reads and
 * clears the array's error word, and returns TD_OK or TD_ERR_DEVICE with the
 * TD_DEVERR_* bits in *bits (bits may be NULL).  After an error the whole
 * array is zero-filled (synchronously), so the next static call starts clean.
 * Before the first td_decode_static call on the device it only waits for
 * `stream`.  Allocates nothing.
 */
TD_API td_status td_check_static_error(int *bits, td_stream stream);

/* Bytes of workspace td_decode_ws needs for `parts` parts. */
TD_API size_t td_workspace_bytes(int B, int H, int D, int64_t parts);

/*
 * td_decode_host -- td_decode / td_decode_varlen with HOST buffers: copies
 * q, k, v (and slopes, seqlens) to device staging owned by the library, runs
 * the decode, and copies out and lse back, all on `stream`.  Host buffers
 * should be pinned for the copies to be asynchronous.  seqlens (host int32
 * [B]) may be NULL for equal lengths N.  If sync != 0 the call waits for the
 * stream before returning (out/lse are then valid); otherwise the caller
 * must synchronise `stream` before reading them.  Ragged batches (seqlens
 * given) copy only the first seqlens[b] key and value rows of each (b,h),
 * since the rows past them are never read.  The staging buffer is one per
 * device and shared by every td_decode_host call on it: calls on different
 * streams, or from threads without ordering, race on it -- order them on one
 * stream.
 */
TD_API td_status td_decode_host(const void *q, const void *k, const void *v, float *out, float *lse,
                         int B, int H, int64_t N, int D, const int32_t *seqlens,
                         int n_split, const float *alibi_slopes, td_dtype dtype,
                         td_stream stream, int sync);

/*
 * td_check_device_error -- wait for `stream`, then read and clear the device
 * error word of the library-owned workspace on the current device (or of
 * `workspace` when it is not NULL).  Returns TD_OK, or TD_ERR_DEVICE with the
 * TD_DEVERR_* bits stored in *bits (if bits is not NULL).  After a device
 * error the workspace's tickets are re-zeroed so the next call starts clean.
 */
TD_API td_status td_check_device_error(void *workspace, size_t workspace_bytes, int *bits,
                                td_stream stream);

/* Human-readable name of a status. */
TD_API const char *td_status_string(td_status s);

/* The last CUDA runtime error seen by this thread's calls (as an int
 * cudaError_t), and clears it. */
TD_API int td_last_cuda_error(void);

/* Frees the library-owned workspaces and host-call staging on every device
 * (waits for the device first). */
TD_API void td_release_workspace(void);

/*
 * Measurement hooks (no counterpart in the method; they report what the
 * library launched, for benchmarks and tests).
 *
 * td_launch_count -- number of kernels launched so far by this thread's
 * calls: the main attention kernel of every decode call (split-KV, or
 * grouped-query), the grouped-query merge kernel when a call runs it, and
 * td_combine's kernel.  Copies and memsets are not counted.
 *
 * td_set_kernel_events -- `before` and `after` are cudaEvent_t handles
 * (created by the caller on the device of the later calls) or both NULL.
 * While set, every decode call of this thread records `before` on its stream
 * immediately before launching its main attention kernel and `after`
 * immediately after, so the events' elapsed time is that kernel's duration
 * (the grouped-query merge kernel, when it runs, comes after `after`).
 * Errors: TD_ERR_INVALID_ARG when exactly one is NULL; a failed record is
 * reported by the decode call as TD_ERR_CUDA.
 *
 * td_last_kernel -- name of the main kernel this thread's last successful
 * launch used ("td_partial_kernel", "td_gqa_keys_kernel",
 * "td_tree_combine_kernel", "td_merge_shards_kernel", "td_empty_state_kernel",
 * "td_prefill_kernel", "td_partial_kernel (fp8 kv)";
 * "" before the first).  Static storage.
 */
TD_API uint64_t td_launch_count(void);
TD_API td_status td_set_kernel_events(void *before, void *after);
TD_API const char *td_last_kernel(void);

/*
 * td_set_wait_test -- settings of this thread's later split-KV decode calls
 * (td_decode, td_decode_varlen, td_decode_ws, td_decode_fp8, td_decode_shard,
 * td_decode_static, td_decode_host) for testing the kernel's failure path.
 * (No counterpart in the method.)  Every pipeline wait of the kernel is
 * bounded: when a wait has not completed after wait_limit_ns nanoseconds the
 * kernel sets TD_DEVERR_WAIT_TIMEOUT, winds down without waiting further and
 * returns, so the context stays usable and the error is read with
 * td_check_device_error / td_check_static_error.
 *   wait_limit_ns   0: the default limit of 2 s; else 1000 .. 10^10.
 *   withhold_tile   -1 (normal operation), or >= 0: the first CTA's loader
 *                   issues its first withhold_tile tiles and then no more, so
 *                   that CTA's next wait can only end by its limit.  The
 *                   results of such a call are not valid.
 * Returns TD_ERR_INVALID_ARG for values outside these ranges.
 */
TD_API td_status td_set_wait_test(uint64_t wait_limit_ns, int64_t withhold_tile);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
TD_API int td_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TREEDEC_H */
