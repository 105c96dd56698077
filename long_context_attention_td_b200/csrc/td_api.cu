// Host side of libtreedec: argument validation, the split heuristic, the
// per-device workspace and staging buffers, and the extern "C" entry points
// declared in treedec.h.  Nothing here computes attention: every step of the
// decode runs in the kernels of td_partial.cu and td_combine.cu.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "td_internal.cuh"
#include "treedec.h"

namespace {

thread_local int g_last_cuda = 0;
// kernels launched by this thread's calls; events recorded around the main
// attention kernel when set (td_set_kernel_events); name of that kernel
thread_local unsigned long long g_launches = 0;
thread_local cudaEvent_t g_ev_before = nullptr;
thread_local cudaEvent_t g_ev_after = nullptr;
thread_local const char* g_last_kernel = "";
// limit of the split-KV kernel's pipeline waits, and the failure-path test's
// withheld tile (td_set_wait_test)
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;
thread_local unsigned long long g_wait_ns = kDefaultWaitNs;
thread_local long long g_withhold_tile = -1;
std::mutex g_mu;

struct DevState {
    void* ws = nullptr;
    size_t ws_bytes = 0;
    void* stage = nullptr;  // device staging of td_decode_host
    size_t stage_bytes = 0;
    int num_sms = 0;
};
constexpr int kMaxDevices = 64;
DevState g_dev[kMaxDevices];

constexpr long long kLimit = 1LL << 62;

// Per workspace (library- or caller-owned): how many leading tickets are
// known to be zero.  The kernels return every ticket they use to zero, but the
// part records start right after the B*H tickets, so a later call with a
// larger B*H finds part-record bytes where its new tickets go; those calls
// zero the ticket region on the stream first.
struct KnownZero {
    const void* ws;
    long long tickets;
};
constexpr int kMaxKnown = 256;
KnownZero g_known[kMaxKnown];
int g_known_n = 0;

KnownZero* known_entry(const void* ws) {
    for (int i = 0; i < g_known_n; ++i)
        if (g_known[i].ws == ws) return &g_known[i];
    return nullptr;
}

void forget_workspace(const void* ws) {
    for (int i = 0; i < g_known_n; ++i)
        if (g_known[i].ws == ws) {
            g_known[i] = g_known[--g_known_n];
            return;
        }
}

void remember_workspace(const void* ws, long long tickets) {
    KnownZero* e = known_entry(ws);
    if (!e) {
        if (g_known_n == kMaxKnown) g_known_n = kMaxKnown - 1;  // drop one: it gets re-zeroed
        e = &g_known[g_known_n++];
        e->ws = ws;
    }
    e->tickets = tickets;
}

// Launch the main attention kernel of a call through `launch`, counting it and
// recording the timing events around it when they are set.
template <class F>
cudaError_t launch_main(cudaStream_t s, const char* name, F&& launch) {
    if (g_ev_before) {
        const cudaError_t e = cudaEventRecord(g_ev_before, s);
        if (e != cudaSuccess) return e;
    }
    const cudaError_t e = launch();
    if (e != cudaSuccess) return e;
    ++g_launches;
    g_last_kernel = name;
    if (g_ev_after) return cudaEventRecord(g_ev_after, s);
    return cudaSuccess;
}

// Launch a secondary (merge) kernel through `launch`, counting it.
template <class F>
cudaError_t launch_aux(F&& launch) {
    const cudaError_t e = launch();
    if (e == cudaSuccess) ++g_launches;
    return e;
}

td_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return TD_OK;
    g_last_cuda = static_cast<int>(e);
    return e == cudaErrorMemoryAllocation ? TD_ERR_NO_MEMORY : TD_ERR_CUDA;
}

bool dtype_ok(int t) { return t == TD_F32 || t == TD_BF16 || t == TD_F16; }
int elt_size(int t) { return t == TD_F32 ? 4 : (t == td::kE4M3 ? 1 : 2); }
bool d_ok(int D) { return D == 64 || D == 128 || D == 256 || D == 512; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
// a * b <= kLimit for non-negative a, b
bool mul_fits(long long a, long long b) { return a >= 0 && b >= 0 && (b == 0 || a <= kLimit / b); }

size_t ticket_region(long long BH) { return align_up(static_cast<size_t>(BH) * 4, 256); }

size_t ws_bytes_for(long long BH, int D, long long parts) {
    return td::kErrRegion + ticket_region(BH) +
           static_cast<size_t>(parts) * 2 * static_cast<size_t>(D + 2) * sizeof(float);
}

// The split heuristic over T attended keys of BH sequences: fill every SM with
// as many CTAs as fit at once, no part below kMinPartBytes of K+V, and no more
// parts per sequence than keep the merge cheap.  The last CTA of a sequence
// reads all of its n part records ((D+2) floats each) at about the rate one
// CTA streams K/V (measured ~62 vs ~50 GB/s on B200), so a part count n per
// sequence of average length L costs ~ 2 L D elt / n + 4 D n / 1.24 bytes of
// one CTA's time, smallest at n = sqrt(0.62 L elt): ~100 for 4096 fp32 keys,
// ~400 for 128K bf16 keys -- a cap that only shows when few, short sequences
// would otherwise be cut into hundreds of parts.
long long auto_parts(long long T, long long BH, int D, int dtype, int num_sms) {
    if (T <= 0) return 1;
    const long long fill = static_cast<long long>(num_sms) * td::partial_ctas_per_sm(dtype, D);
    const long long bytes_per_key = 2LL * D * elt_size(dtype);
    long long by_size = T / (td::kMinPartBytes / bytes_per_key > 0
                                 ? td::kMinPartBytes / bytes_per_key
                                 : 1);
    if (by_size < 1) by_size = 1;
    long long P = fill < by_size ? fill : by_size;
    if (BH > 0) {
        const double L = static_cast<double>(T) / static_cast<double>(BH);
        long long per_seq = static_cast<long long>(std::sqrt(0.62 * L * elt_size(dtype)));
        if (per_seq < 1) per_seq = 1;
        if (mul_fits(BH, per_seq) && P > BH * per_seq) P = BH * per_seq;
    }
    if (P > T) P = T;
    return P < 1 ? 1 : P;
}

td_status current_device(int* dev, int* num_sms) {
    td_status st = cuda_status(cudaGetDevice(dev));
    if (st != TD_OK) return st;
    if (*dev < 0 || *dev >= kMaxDevices) return TD_ERR_UNSUPPORTED;
    DevState& d = g_dev[*dev];
    if (d.num_sms == 0) {
        int n = 0;
        st = cuda_status(cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, *dev));
        if (st != TD_OK) return st;
        d.num_sms = n;
    }
    *num_sms = d.num_sms;
    return TD_OK;
}

// Grow the library-owned workspace of `dev` to at least `need` bytes.  A new
// buffer is zero-filled on `stream` (the tickets must start at zero).
td_status library_ws(int dev, size_t need, cudaStream_t stream, void** ws, size_t* bytes) {
    std::lock_guard<std::mutex> lk(g_mu);
    DevState& d = g_dev[dev];
    if (d.ws_bytes < need) {
        size_t nb = need < (size_t(1) << 20) ? (size_t(1) << 20) : need;
        if (nb < 2 * d.ws_bytes) nb = 2 * d.ws_bytes;
        if (d.ws) {
            // cudaFree waits for outstanding work on the device first
            cudaFree(d.ws);
            forget_workspace(d.ws);
            d.ws = nullptr;
            d.ws_bytes = 0;
        }
        void* p = nullptr;
        td_status st = cuda_status(cudaMalloc(&p, nb));
        if (st != TD_OK) return st;
        st = cuda_status(cudaMemsetAsync(p, 0, nb, stream));
        if (st != TD_OK) {
            cudaFree(p);
            return st;
        }
        d.ws = p;
        d.ws_bytes = nb;
        remember_workspace(p, static_cast<long long>((nb - td::kErrRegion) / 4));
    }
    *ws = d.ws;
    *bytes = d.ws_bytes;
    return TD_OK;
}

// The workspace a call runs on: the caller's (checked) or the library's
// (grown), with its first `tickets` tickets known to be zero.
td_status prepare_ws(int dev, void* user_ws, size_t user_bytes, long long tickets, size_t need,
                     cudaStream_t stream, char** base_out) {
    void* ws = user_ws;
    size_t wsb = user_bytes;
    td_status st = TD_OK;
    if (ws) {
        if (!aligned(ws, 256)) return TD_ERR_INVALID_ARG;
        if (wsb < need) return TD_ERR_WORKSPACE;
    } else {
        st = library_ws(dev, need, stream, &ws, &wsb);
        if (st != TD_OK) return st;
    }
    char* base = static_cast<char*>(ws);
    {
        std::lock_guard<std::mutex> lk(g_mu);
        const KnownZero* e = known_entry(ws);
        if (!e || e->tickets < tickets) {
            st = cuda_status(
                cudaMemsetAsync(base + td::kErrRegion, 0, ticket_region(tickets), stream));
            if (st != TD_OK) return st;
        }
        remember_workspace(ws, tickets);
    }
    *base_out = base;
    return TD_OK;
}

struct Req {
    const void *q, *k, *v;
    float *out, *lse;
    int B, H;
    long long N;
    int D;
    const int32_t* seqlens;
    const int32_t* seqlens_host;
    long long parts;  // 0 = heuristic
    const float* slopes;
    int dtype;
    void* ws;  // null = library-owned
    size_t ws_bytes;
    cudaStream_t stream;
    long long alibi_off = 0;  // ALiBi position shift of a shard (see td_decode_shard)
    // FP8 K/V cache: kv_dtype = td::kE4M3 with per-head scales; -1: K/V of type dtype
    int kv_dtype = -1;
    const float* k_scale = nullptr;
    const float* v_scale = nullptr;
    int kv() const { return kv_dtype < 0 ? dtype : kv_dtype; }
};

td_status validate(const Req& r) {
    if (!r.q || !r.k || !r.v || !r.out) return TD_ERR_INVALID_ARG;
    if (!dtype_ok(r.dtype)) return TD_ERR_UNSUPPORTED;
    if (r.B < 1 || r.H < 1 || r.N < 1 || r.D < 1 || r.parts < 0) return TD_ERR_INVALID_ARG;
    if (!d_ok(r.D)) return TD_ERR_UNSUPPORTED;
    if (!aligned(r.q, 16) || !aligned(r.k, 16) || !aligned(r.v, 16)) return TD_ERR_INVALID_ARG;
    if (!aligned(r.out, 4) || (r.lse && !aligned(r.lse, 4)) ||
        (r.slopes && !aligned(r.slopes, 4)) || (r.seqlens && !aligned(r.seqlens, 4)))
        return TD_ERR_INVALID_ARG;
    if (r.seqlens_host && !r.seqlens) return TD_ERR_INVALID_ARG;
    const long long BH = static_cast<long long>(r.B) * r.H;
    if (BH > 0x7fffffffLL) return TD_ERR_INVALID_ARG;
    if (!mul_fits(BH, r.N) || !mul_fits(BH * r.N, static_cast<long long>(r.D) * 4))
        return TD_ERR_INVALID_ARG;
    if (r.seqlens_host)
        for (int b = 0; b < r.B; ++b)
            if (r.seqlens_host[b] < 0 || r.seqlens_host[b] > r.N) return TD_ERR_INVALID_ARG;
    if (r.kv_dtype == td::kE4M3) {
        // FP8 cache: q in half precision, both scales given
        if (r.dtype != TD_BF16 && r.dtype != TD_F16) return TD_ERR_UNSUPPORTED;
        if (!r.k_scale || !r.v_scale || !aligned(r.k_scale, 4) || !aligned(r.v_scale, 4))
            return TD_ERR_INVALID_ARG;
    } else if (r.kv_dtype >= 0 && r.kv_dtype != r.dtype) {
        return TD_ERR_UNSUPPORTED;
    }
    return TD_OK;
}

// Attended keys when known on the host, else -1.
long long known_keys(const Req& r) {
    if (!r.seqlens) return static_cast<long long>(r.B) * r.H * r.N;
    if (!r.seqlens_host) return -1;
    long long s = 0;
    for (int b = 0; b < r.B; ++b) s += r.seqlens_host[b];
    return s * r.H;
}

long long plan_parts(const Req& r, int num_sms) {
    const long long bound = static_cast<long long>(r.B) * r.H * r.N;
    const long long known = known_keys(r);
    const long long T = known >= 0 ? known : bound;
    long long P = r.parts > 0 ? r.parts
                              : auto_parts(T, static_cast<long long>(r.B) * r.H, r.D, r.kv(),
                                           num_sms);
    const long long cap = T > 0 ? T : 1;
    if (P > cap) P = cap;
    if (P > 0x7fffffffLL) P = 0x7fffffffLL;
    return P < 1 ? 1 : P;
}

td_status decode_impl(const Req& r) {
    td_status st = validate(r);
    if (st != TD_OK) return st;
    int dev = 0, sms = 0;
    st = current_device(&dev, &sms);
    if (st != TD_OK) return st;
    const long long P = plan_parts(r, sms);
    const long long BH = static_cast<long long>(r.B) * r.H;
    if (!mul_fits(P + 1, BH * r.N)) return TD_ERR_INVALID_ARG;
    const size_t need = ws_bytes_for(BH, r.D, P);
    char* base = nullptr;
    st = prepare_ws(dev, r.ws, r.ws_bytes, BH, need, r.stream, &base);
    if (st != TD_OK) return st;
    td::PartialParams p;
    p.q = r.q;
    p.k = r.k;
    p.v = r.v;
    p.out = r.out;
    p.lse = r.lse;
    p.slopes = r.slopes;
    p.seqlens = r.seqlens;
    p.B = r.B;
    p.H = r.H;
    p.N = r.N;
    p.T = r.seqlens ? -1 : BH * r.N;
    p.P = P;
    p.qscale2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(r.D)));
    p.err = reinterpret_cast<int*>(base);
    p.tickets = reinterpret_cast<int*>(base + td::kErrRegion);
    p.part = reinterpret_cast<float*>(base + td::kErrRegion + ticket_region(BH));
    p.alibi_off = r.alibi_off;
    p.k_scale = r.k_scale;
    p.v_scale = r.v_scale;
    p.wait_ns = g_wait_ns;
    p.withhold_tile = g_withhold_tile;
    if (r.kv() == td::kE4M3)
        return cuda_status(launch_main(r.stream, "td_partial_kernel (fp8 kv)", [&] {
            return td::launch_partial_fp8(dev, r.dtype, r.D, p, r.stream);
        }));
    return cuda_status(launch_main(r.stream, "td_partial_kernel", [&] {
        return td::launch_partial(dev, r.dtype, r.D, p, r.stream);
    }));
}

// ------------------------------------------------------------- grouped-query

// parts-per-sequence x group size from which the merge runs as its own kernel
// (the last CTA of a sequence would merge its query heads one after another; the
// combine kernel spreads them over the SMs)
constexpr long long kGqaSeparateMerge = 16;

// [error word][tickets][segment descriptors: 3 int32 each][part records]
size_t gqa_desc_region(long long BHkv) { return align_up(static_cast<size_t>(BHkv) * 12, 256); }

size_t gqa_ws_bytes_for(long long BHkv, int G, int D, long long parts) {
    return td::kErrRegion + ticket_region(BHkv) + gqa_desc_region(BHkv) +
           static_cast<size_t>(parts) * 2 * static_cast<size_t>(G) *
               static_cast<size_t>(D + 3) * sizeof(float);
}

// Head chunks of a group on the grouped-query kernel and the heads per chunk.
void gqa_chunking(int G, int* chunks, int* gc) {
    *chunks = td::gqa_keys_chunks(G);
    *gc = (G + *chunks - 1) / *chunks;
}

long long gqa_auto_parts(long long T, int D, int G, int num_sms) {
    if (T <= 0) return 1;
    int chunks = 1, gc = G;
    gqa_chunking(G, &chunks, &gc);
    const int per_sm = td::gqa_keys_ctas_per_sm(D, gc);
    // each part runs as `chunks` CTAs: fill the SMs with parts x chunks CTAs
    long long fill = static_cast<long long>(num_sms) * per_sm / chunks;
    if (fill < 1) fill = 1;
    const long long bytes_per_key = 2LL * D * 2;
    long long by_size = T / (td::kMinPartBytes / bytes_per_key);
    if (by_size < 1) by_size = 1;
    long long P = fill < by_size ? fill : by_size;
    if (P > T) P = T;
    return P < 1 ? 1 : P;
}

struct GqaReq {
    const void *q, *k, *v;
    float *out, *lse;
    int B, Hq, Hkv;
    long long N;
    int D;
    const int32_t* seqlens;
    const int32_t* seqlens_host;
    long long parts;  // 0 = heuristic
    int n_split;      // used when parts == 0 and n_split > 0
    const float* slopes;
    int dtype;
    void* ws;
    size_t ws_bytes;
    cudaStream_t stream;
};

td_status gqa_validate(const GqaReq& r) {
    if (!r.q || !r.k || !r.v || !r.out) return TD_ERR_INVALID_ARG;
    if (r.dtype != TD_BF16 && r.dtype != TD_F16) return TD_ERR_UNSUPPORTED;
    if (r.D != 64 && r.D != 128) return TD_ERR_UNSUPPORTED;
    if (r.B < 1 || r.Hq < 1 || r.Hkv < 1 || r.N < 1 || r.parts < 0 || r.n_split < 0)
        return TD_ERR_INVALID_ARG;
    if (r.Hq % r.Hkv != 0) return TD_ERR_INVALID_ARG;
    if (r.Hq / r.Hkv > 128) return TD_ERR_UNSUPPORTED;
    if (!aligned(r.q, 16) || !aligned(r.k, 16) || !aligned(r.v, 16)) return TD_ERR_INVALID_ARG;
    if (!aligned(r.out, 4) || (r.lse && !aligned(r.lse, 4)) ||
        (r.slopes && !aligned(r.slopes, 4)) || (r.seqlens && !aligned(r.seqlens, 4)))
        return TD_ERR_INVALID_ARG;
    if (r.seqlens_host && !r.seqlens) return TD_ERR_INVALID_ARG;
    const long long BHkv = static_cast<long long>(r.B) * r.Hkv;
    if (static_cast<long long>(r.B) * r.Hq > 0x7fffffffLL) return TD_ERR_INVALID_ARG;
    // the tensor-map row coordinate is a 32-bit integer
    if (!mul_fits(BHkv, r.N) || BHkv * r.N > 0x7fffffffLL) return TD_ERR_INVALID_ARG;
    if (r.seqlens_host)
        for (int b = 0; b < r.B; ++b)
            if (r.seqlens_host[b] < 0 || r.seqlens_host[b] > r.N) return TD_ERR_INVALID_ARG;
    return TD_OK;
}

long long gqa_plan(const GqaReq& r, int num_sms) {
    const long long BHkv = static_cast<long long>(r.B) * r.Hkv;
    const long long bound = BHkv * r.N;
    long long known = -1;
    if (!r.seqlens) {
        known = bound;
    } else if (r.seqlens_host) {
        long long s = 0;
        for (int b = 0; b < r.B; ++b) s += r.seqlens_host[b];
        known = s * r.Hkv;
    }
    const long long T = known >= 0 ? known : bound;
    long long P = r.parts;
    if (P == 0 && r.n_split > 0) {
        const long long per = (!r.seqlens && r.n_split > r.N) ? r.N : r.n_split;
        P = BHkv * per;
    }
    if (P == 0) P = gqa_auto_parts(T, r.D, r.Hq / r.Hkv, num_sms);
    const long long cap = T > 0 ? T : 1;
    if (P > cap) P = cap;
    if (P > 0x7fffffffLL) P = 0x7fffffffLL;
    return P < 1 ? 1 : P;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D map over [rows, D] elements, box {64 columns, box_rows rows}, 128-byte
// swizzle, out-of-range rows read as zero.
td_status make_kv_map(CUtensorMap* map, const void* base, long long rows, int D, int dtype,
                      int box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return TD_ERR_CUDA;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    const CUresult rc = enc(map,
                            dtype == TD_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                             : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                            2, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return rc == CUDA_SUCCESS ? TD_OK : TD_ERR_INVALID_ARG;
}

td_status gqa_impl(const GqaReq& r) {
    td_status st = gqa_validate(r);
    if (st != TD_OK) return st;
    int dev = 0, sms = 0;
    st = current_device(&dev, &sms);
    if (st != TD_OK) return st;
    const long long P = gqa_plan(r, sms);
    const long long BHkv = static_cast<long long>(r.B) * r.Hkv;
    if (!mul_fits(P + 1, BHkv * r.N)) return TD_ERR_INVALID_ARG;
    const int G = r.Hq / r.Hkv;
    const size_t need = gqa_ws_bytes_for(BHkv, G, r.D, P);
    // the keys go on the MMA M axis in tiles of 128: boxes of 128 rows
    if (!td::gqa_keys_path(r.D, G)) return TD_ERR_UNSUPPORTED;
    const int box_rows = 128;
    CUtensorMap mk, mv;
    st = make_kv_map(&mk, r.k, BHkv * r.N, r.D, r.dtype, box_rows);
    if (st != TD_OK) return st;
    st = make_kv_map(&mv, r.v, BHkv * r.N, r.D, r.dtype, box_rows);
    if (st != TD_OK) return st;
    char* base = nullptr;
    st = prepare_ws(dev, r.ws, r.ws_bytes, BHkv, need, r.stream, &base);
    if (st != TD_OK) return st;
    td::GqaParams p;
    p.q = r.q;
    p.out = r.out;
    p.lse = r.lse;
    p.slopes = r.slopes;
    p.seqlens = r.seqlens;
    p.B = r.B;
    p.Hq = r.Hq;
    p.Hkv = r.Hkv;
    p.G = G;
    p.N = r.N;
    p.T = r.seqlens ? -1 : BHkv * r.N;
    p.P = P;
    p.qscale2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(r.D)));
    p.err = reinterpret_cast<int*>(base);
    p.tickets = reinterpret_cast<int*>(base + td::kErrRegion);
    p.seg_desc = reinterpret_cast<int*>(base + td::kErrRegion + ticket_region(BHkv));
    p.part = reinterpret_cast<float*>(base + td::kErrRegion + ticket_region(BHkv) +
                                      gqa_desc_region(BHkv));
    // The last CTA of a sequence merges its parts itself when that is a small
    // job; when many CTAs share a sequence and many query heads share it, a
    // second kernel spreads the merge over one CTA per (sequence, query head).
    const long long per_seg = (P + BHkv - 1) / BHkv + 1;  // parts touching a sequence
    p.fused_merge = per_seg * G < kGqaSeparateMerge ? 1 : 0;
    gqa_chunking(G, &p.chunks, &p.gc);
    if (!mul_fits(P, p.chunks) || P * p.chunks > 0x7fffffffLL) return TD_ERR_INVALID_ARG;
    st = cuda_status(launch_main(r.stream, "td_gqa_keys_kernel", [&] {
        return td::launch_gqa_keys(dev, r.dtype, r.D, p, mk, mv, r.stream);
    }));
    if (st != TD_OK || p.fused_merge) return st;
    return cuda_status(launch_aux([&] { return td::launch_gqa_combine(r.D, p, r.stream); }));
}

// ------------------------------------------------------------------ prefill

// 3-D map over [BH, S, D] elements, box {64 columns, 128 rows, 1}, 128-byte
// swizzle; rows past S read as zero.
td_status make_seq_map(CUtensorMap* map, const void* base, long long BH, long long S, int D,
                       int dtype) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return TD_ERR_CUDA;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(S) * D * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult rc = enc(map,
                            dtype == TD_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                             : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                            3, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return rc == CUDA_SUCCESS ? TD_OK : TD_ERR_INVALID_ARG;
}

td_status prefill_validate(const void* q, const void* k, const void* v, const float* out,
                           const float* lse, int B, int H, int64_t S, int D,
                           const float* slopes, int dtype) {
    if (!q || !k || !v || !out) return TD_ERR_INVALID_ARG;
    if (dtype != TD_BF16 && dtype != TD_F16) return TD_ERR_UNSUPPORTED;
    if (D != 64 && D != 128) return TD_ERR_UNSUPPORTED;
    if (B < 1 || H < 1 || S < 1) return TD_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        (lse && !aligned(lse, 4)) || (slopes && !aligned(slopes, 4)))
        return TD_ERR_INVALID_ARG;
    const long long BH = static_cast<long long>(B) * H;
    // tensor-map coordinates and the kernel's key indices are 32-bit (a tile
    // index times 128 stays below 2^31); the grid is B*H*ceil(S/128) CTAs
    if (S > 0x7fffffffLL - 256 || BH > 0x7fffffffLL || !mul_fits(BH, S) ||
        BH * ((S + 127) / 128) > 0x7fffffffLL || !mul_fits(BH * S, static_cast<long long>(D) * 4))
        return TD_ERR_INVALID_ARG;
    return TD_OK;
}

}  // namespace

extern "C" {

td_status td_prefill(const void* q, const void* k, const void* v, float* out, float* lse, int B,
                     int H, int64_t S, int D, int causal, const float* alibi_slopes,
                     td_dtype dtype, td_stream stream) {
    td_status st = prefill_validate(q, k, v, out, lse, B, H, S, D, alibi_slopes,
                                    static_cast<int>(dtype));
    if (st != TD_OK) return st;
    int dev = 0, sms = 0;
    st = current_device(&dev, &sms);
    if (st != TD_OK) return st;
    const long long BH = static_cast<long long>(B) * H;
    CUtensorMap mq, mk, mv;
    st = make_seq_map(&mq, q, BH, S, D, dtype);
    if (st == TD_OK) st = make_seq_map(&mk, k, BH, S, D, dtype);
    if (st == TD_OK) st = make_seq_map(&mv, v, BH, S, D, dtype);
    if (st != TD_OK) return st;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* base = nullptr;
    st = prepare_ws(dev, nullptr, 0, 0, td::kErrRegion, s, &base);
    if (st != TD_OK) return st;
    td::PrefillParams p;
    p.out = out;
    p.lse = lse;
    p.slopes = alibi_slopes;
    p.B = B;
    p.H = H;
    p.S = S;
    p.causal = causal ? 1 : 0;
    p.qscale2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
    p.err = reinterpret_cast<int*>(base);
    return cuda_status(launch_main(s, "td_prefill_kernel", [&] {
        return td::launch_prefill(dev, static_cast<int>(dtype), D, p, mq, mk, mv, s);
    }));
}


td_status td_decode_gqa(const void* q, const void* k, const void* v, float* out, float* lse, int B,
                        int Hq, int Hkv, int64_t N, int D, const int32_t* seqlens,
                        const int32_t* seqlens_host, int n_split, const float* alibi_slopes,
                        td_dtype dtype, td_stream stream) {
    GqaReq r{q, k, v, out, lse, B, Hq, Hkv, N, D, seqlens, seqlens_host, 0, n_split,
             alibi_slopes, static_cast<int>(dtype), nullptr, 0,
             reinterpret_cast<cudaStream_t>(stream)};
    return gqa_impl(r);
}

td_status td_decode_gqa_ws(const void* q, const void* k, const void* v, float* out, float* lse,
                           int B, int Hq, int Hkv, int64_t N, int D, const int32_t* seqlens,
                           const int32_t* seqlens_host, int64_t parts, const float* alibi_slopes,
                           td_dtype dtype, void* workspace, size_t workspace_bytes,
                           td_stream stream) {
    if (!workspace || parts < 0) return TD_ERR_INVALID_ARG;
    GqaReq r{q, k, v, out, lse, B, Hq, Hkv, N, D, seqlens, seqlens_host, parts, 0,
             alibi_slopes, static_cast<int>(dtype), workspace, workspace_bytes,
             reinterpret_cast<cudaStream_t>(stream)};
    return gqa_impl(r);
}

int64_t td_plan_parts_gqa(int B, int Hq, int Hkv, int64_t Nmax, int D, td_dtype dtype,
                          int n_split, int64_t total_keys) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Nmax < 1 || n_split < 0 || Hq % Hkv != 0) return -1;
    if ((dtype != TD_BF16 && dtype != TD_F16) || (D != 64 && D != 128)) return -1;
    const long long BHkv = static_cast<long long>(B) * Hkv;
    if (!mul_fits(BHkv, Nmax) || (total_keys >= 0 && total_keys > BHkv * Nmax)) return -1;
    int dev = 0, sms = 0;
    if (current_device(&dev, &sms) != TD_OK) return -1;
    GqaReq r{nullptr, nullptr, nullptr, nullptr, nullptr, B, Hq, Hkv, Nmax, D, nullptr, nullptr,
             0, n_split, nullptr, static_cast<int>(dtype), nullptr, 0, nullptr};
    if (total_keys >= 0) {
        // ragged: size from the given key count
        long long T = total_keys;
        long long P = n_split > 0 ? BHkv * n_split : gqa_auto_parts(T, D, Hq / Hkv, sms);
        const long long cap = T > 0 ? T : 1;
        if (P > cap) P = cap;
        return P < 1 ? 1 : P;
    }
    return gqa_plan(r, sms);
}

size_t td_gqa_workspace_bytes(int B, int Hq, int Hkv, int D, int64_t parts) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || D < 1 || parts < 1) return 0;
    return gqa_ws_bytes_for(static_cast<long long>(B) * Hkv, Hq / Hkv, D, parts);
}


td_status td_decode(const void* q, const void* k, const void* v, float* out, float* lse, int B,
                    int H, int64_t N, int D, int n_split, const float* alibi_slopes,
                    td_dtype dtype, td_stream stream) {
    if (n_split < 0) return TD_ERR_INVALID_ARG;
    long long parts = 0;
    if (n_split > 0) {
        const long long per = n_split < N ? n_split : N;
        parts = static_cast<long long>(B) * H * (per > 0 ? per : 1);
    }
    Req r{q, k, v, out, lse, B, H, N, D, nullptr, nullptr, parts, alibi_slopes,
          static_cast<int>(dtype), nullptr, 0, reinterpret_cast<cudaStream_t>(stream)};
    return decode_impl(r);
}

td_status td_decode_varlen(const void* q, const void* k, const void* v, float* out, float* lse,
                           int B, int H, int64_t Nmax, int D, const int32_t* seqlens,
                           const int32_t* seqlens_host, int n_split, const float* alibi_slopes,
                           td_dtype dtype, td_stream stream) {
    if (n_split < 0 || !seqlens) return TD_ERR_INVALID_ARG;
    const long long parts = n_split > 0 ? static_cast<long long>(B) * H * n_split : 0;
    Req r{q, k, v, out, lse, B, H, Nmax, D, seqlens, seqlens_host, parts, alibi_slopes,
          static_cast<int>(dtype), nullptr, 0, reinterpret_cast<cudaStream_t>(stream)};
    return decode_impl(r);
}

td_status td_decode_ws(const void* q, const void* k, const void* v, float* out, float* lse, int B,
                       int H, int64_t N, int D, const int32_t* seqlens,
                       const int32_t* seqlens_host, int64_t parts, const float* alibi_slopes,
                       td_dtype dtype, void* workspace, size_t workspace_bytes,
                       td_stream stream) {
    if (!workspace || parts < 0) return TD_ERR_INVALID_ARG;
    Req r{q, k, v, out, lse, B, H, N, D, seqlens, seqlens_host, parts, alibi_slopes,
          static_cast<int>(dtype), workspace, workspace_bytes,
          reinterpret_cast<cudaStream_t>(stream)};
    return decode_impl(r);
}

td_status td_decode_fp8(const void* q, const void* k8, const void* v8, const float* k_scale,
                        const float* v_scale, float* out, float* lse, int B, int H, int64_t Nmax,
                        int D, const int32_t* seqlens, const int32_t* seqlens_host, int n_split,
                        const float* alibi_slopes, td_dtype q_dtype, td_stream stream) {
    if (n_split < 0) return TD_ERR_INVALID_ARG;
    long long parts = 0;
    if (n_split > 0) {
        const long long per = (!seqlens && n_split > Nmax) ? Nmax : n_split;
        parts = static_cast<long long>(B) * H * (per > 0 ? per : 1);
    }
    Req r{q, k8, v8, out, lse, B, H, Nmax, D, seqlens, seqlens_host, parts, alibi_slopes,
          static_cast<int>(q_dtype), nullptr, 0, reinterpret_cast<cudaStream_t>(stream)};
    r.kv_dtype = td::kE4M3;
    r.k_scale = k_scale;
    r.v_scale = v_scale;
    return decode_impl(r);
}

td_status td_decode_shard(const void* q, const void* k, const void* v, float* state, int B, int H,
                          int64_t N_shard, int D, int64_t key_offset, int64_t N_total,
                          int n_split, const float* alibi_slopes, td_dtype dtype,
                          td_stream stream) {
    if (!q || !state || n_split < 0 || (N_shard > 0 && (!k || !v))) return TD_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || D < 1 || N_shard < 0 || key_offset < 0 || N_total < 1)
        return TD_ERR_INVALID_ARG;
    if (key_offset > N_total || N_shard > N_total - key_offset) return TD_ERR_INVALID_ARG;
    if (!aligned(state, 4)) return TD_ERR_INVALID_ARG;
    const long long rows = static_cast<long long>(B) * H;
    if (!mul_fits(rows, static_cast<long long>(D) + 1)) return TD_ERR_INVALID_ARG;
    float* out = state;
    float* lse = state + rows * D;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (N_shard == 0) {
        // no keys here (a rank past the end of a short sequence): the empty state
        if (!dtype_ok(static_cast<int>(dtype))) return TD_ERR_UNSUPPORTED;
        if (!d_ok(D)) return TD_ERR_UNSUPPORTED;
        return cuda_status(launch_main(s, "td_empty_state_kernel", [&] {
            return td::launch_empty_state(out, lse, rows, D, s);
        }));
    }
    long long parts = 0;
    if (n_split > 0) {
        const long long per = n_split < N_shard ? n_split : N_shard;
        parts = rows * per;
    }
    Req r{q, k, v, out, lse, B, H, N_shard, D, nullptr, nullptr, parts, alibi_slopes,
          static_cast<int>(dtype), nullptr, 0, s};
    // key j of the shard sits at key_offset + j of the N_total keys
    r.alibi_off = key_offset + N_shard - N_total;
    return decode_impl(r);
}

td_status td_merge_shards(const float* states, int W, int B, int H, int D, float* out,
                          float* lse, td_stream stream) {
    if (!states || !out || W < 1 || B < 1 || H < 1 || D < 1 || D > 512) return TD_ERR_INVALID_ARG;
    const long long rows = static_cast<long long>(B) * H;
    if (rows > 0x7fffffffLL || !mul_fits(rows * (D + 1), static_cast<long long>(W) * 4))
        return TD_ERR_INVALID_ARG;
    if (!aligned(states, 4) || !aligned(out, 4) || (lse && !aligned(lse, 4)))
        return TD_ERR_INVALID_ARG;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return cuda_status(launch_main(s, "td_merge_shards_kernel", [&] {
        return td::launch_merge_shards(states, W, rows, D, out, lse, s);
    }));
}

td_status td_combine(const float* num, const float* m, const float* l, float* out, float* lse,
                     int B, int H, int S, int D, td_stream stream) {
    if (!num || !m || !l || !out) return TD_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || S < 1 || D < 1 || D > 512) return TD_ERR_INVALID_ARG;
    const long long rows = static_cast<long long>(B) * H;
    if (rows > 0x7fffffffLL || !mul_fits(rows * S, static_cast<long long>(D) * 4))
        return TD_ERR_INVALID_ARG;
    if (!aligned(num, 4) || !aligned(m, 4) || !aligned(l, 4) || !aligned(out, 4) ||
        (lse && !aligned(lse, 4)))
        return TD_ERR_INVALID_ARG;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return cuda_status(launch_main(s, "td_tree_combine_kernel", [&] {
        return td::launch_combine(num, m, l, out, lse, rows, S, D, s);
    }));
}

int64_t td_auto_split(int B, int H, int64_t N, int D, td_dtype dtype, int num_sms) {
    if (B < 1 || H < 1 || N < 1 || num_sms < 1 || !dtype_ok(dtype) || !d_ok(D)) return -1;
    const long long BH = static_cast<long long>(B) * H;
    if (!mul_fits(BH, N)) return -1;
    return auto_parts(BH * N, BH, D, dtype, num_sms);
}

int64_t td_plan_parts(int B, int H, int64_t Nmax, int D, td_dtype dtype, int n_split,
                      int64_t total_keys) {
    if (B < 1 || H < 1 || Nmax < 1 || n_split < 0 || !dtype_ok(dtype) || !d_ok(D)) return -1;
    const long long BH = static_cast<long long>(B) * H;
    if (!mul_fits(BH, Nmax)) return -1;
    int dev = 0, sms = 0;
    if (current_device(&dev, &sms) != TD_OK) return -1;
    const long long bound = BH * Nmax;
    long long T = total_keys >= 0 ? total_keys : bound;
    if (T > bound) return -1;
    long long parts = 0;
    if (n_split > 0) {
        const long long per = n_split < Nmax ? n_split : Nmax;
        parts = total_keys < 0 ? BH * per : BH * n_split;
    }
    long long P = parts > 0 ? parts : auto_parts(T, BH, D, dtype, sms);
    const long long cap = T > 0 ? T : 1;
    if (P > cap) P = cap;
    return P < 1 ? 1 : P;
}

size_t td_workspace_bytes(int B, int H, int D, int64_t parts) {
    if (B < 1 || H < 1 || D < 1 || parts < 1) return 0;
    return ws_bytes_for(static_cast<long long>(B) * H, D, parts);
}

td_status td_decode_host(const void* q, const void* k, const void* v, float* out, float* lse,
                         int B, int H, int64_t N, int D, const int32_t* seqlens, int n_split,
                         const float* alibi_slopes, td_dtype dtype, td_stream stream, int sync) {
    if (!q || !k || !v || !out || n_split < 0) return TD_ERR_INVALID_ARG;
    if (!dtype_ok(dtype)) return TD_ERR_UNSUPPORTED;
    if (B < 1 || H < 1 || N < 1) return TD_ERR_INVALID_ARG;
    if (!d_ok(D)) return TD_ERR_UNSUPPORTED;
    const long long BH = static_cast<long long>(B) * H;
    if (!mul_fits(BH, N) || !mul_fits(BH * N, static_cast<long long>(D) * 4))
        return TD_ERR_INVALID_ARG;
    if (seqlens)
        for (int b = 0; b < B; ++b)
            if (seqlens[b] < 0 || seqlens[b] > N) return TD_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t es = static_cast<size_t>(elt_size(dtype));
    const size_t qb = static_cast<size_t>(BH) * D * es;
    const size_t kvb = static_cast<size_t>(BH) * static_cast<size_t>(N) * D * es;
    const size_t ob = static_cast<size_t>(BH) * D * sizeof(float);
    const size_t lb = static_cast<size_t>(BH) * sizeof(float);
    const size_t sb = alibi_slopes ? static_cast<size_t>(H) * sizeof(float) : 0;
    const size_t nb = seqlens ? static_cast<size_t>(B) * sizeof(int32_t) : 0;
    size_t off[7];
    size_t total = 0;
    const size_t sizes[7] = {qb, kvb, kvb, ob, lb, sb, nb};
    for (int i = 0; i < 7; ++i) {
        off[i] = total;
        total += align_up(sizes[i] ? sizes[i] : 1, 256);
    }
    int dev = 0, sms = 0;
    td_status st = current_device(&dev, &sms);
    if (st != TD_OK) return st;
    char* base = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        DevState& d = g_dev[dev];
        if (d.stage_bytes < total) {
            if (d.stage) cudaFree(d.stage);
            d.stage = nullptr;
            d.stage_bytes = 0;
            void* p = nullptr;
            st = cuda_status(cudaMalloc(&p, total));
            if (st != TD_OK) return st;
            d.stage = p;
            d.stage_bytes = total;
        }
        base = static_cast<char*>(d.stage);
    }
    const cudaMemcpyKind h2d = cudaMemcpyHostToDevice;
    st = cuda_status(cudaMemcpyAsync(base + off[0], q, qb, h2d, s));
    if (!seqlens) {
        if (st == TD_OK) st = cuda_status(cudaMemcpyAsync(base + off[1], k, kvb, h2d, s));
        if (st == TD_OK) st = cuda_status(cudaMemcpyAsync(base + off[2], v, kvb, h2d, s));
    } else {
        // only the attended rows: for batch b, H row blocks of seqlens[b] keys
        // at a pitch of N keys
        const size_t row = static_cast<size_t>(D) * es;
        const size_t pitch = static_cast<size_t>(N) * row;
        for (int b = 0; st == TD_OK && b < B; ++b) {
            if (seqlens[b] == 0) continue;
            const size_t at = static_cast<size_t>(b) * H * pitch;
            const size_t width = static_cast<size_t>(seqlens[b]) * row;
            st = cuda_status(cudaMemcpy2DAsync(base + off[1] + at, pitch,
                                               static_cast<const char*>(k) + at, pitch, width,
                                               static_cast<size_t>(H), h2d, s));
            if (st == TD_OK)
                st = cuda_status(cudaMemcpy2DAsync(base + off[2] + at, pitch,
                                                   static_cast<const char*>(v) + at, pitch, width,
                                                   static_cast<size_t>(H), h2d, s));
        }
    }
    if (st == TD_OK && sb) st = cuda_status(cudaMemcpyAsync(base + off[5], alibi_slopes, sb, h2d, s));
    if (st == TD_OK && nb) st = cuda_status(cudaMemcpyAsync(base + off[6], seqlens, nb, h2d, s));
    if (st != TD_OK) return st;
    float* dout = reinterpret_cast<float*>(base + off[3]);
    float* dlse = reinterpret_cast<float*>(base + off[4]);
    const float* dsl = sb ? reinterpret_cast<const float*>(base + off[5]) : nullptr;
    const int32_t* dsq = nb ? reinterpret_cast<const int32_t*>(base + off[6]) : nullptr;
    if (dsq)
        st = td_decode_varlen(base + off[0], base + off[1], base + off[2], dout, dlse, B, H, N, D,
                              dsq, seqlens, n_split, dsl, dtype, stream);
    else
        st = td_decode(base + off[0], base + off[1], base + off[2], dout, dlse, B, H, N, D,
                       n_split, dsl, dtype, stream);
    if (st != TD_OK) return st;
    st = cuda_status(cudaMemcpyAsync(out, dout, ob, cudaMemcpyDeviceToHost, s));
    if (st == TD_OK && lse) st = cuda_status(cudaMemcpyAsync(lse, dlse, lb, cudaMemcpyDeviceToHost, s));
    if (st == TD_OK && sync) st = cuda_status(cudaStreamSynchronize(s));
    return st;
}

td_status td_check_device_error(void* workspace, size_t workspace_bytes, int* bits,
                                td_stream stream) {
    if (bits) *bits = 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    td_status st = cuda_status(cudaStreamSynchronize(s));
    if (st != TD_OK) return st;
    void* ws = workspace;
    size_t wsb = workspace_bytes;
    if (!ws) {
        int dev = 0, sms = 0;
        st = current_device(&dev, &sms);
        if (st != TD_OK) return st;
        std::lock_guard<std::mutex> lk(g_mu);
        ws = g_dev[dev].ws;
        wsb = g_dev[dev].ws_bytes;
    }
    if (!ws) return TD_OK;
    if (wsb < td::kErrRegion) return TD_ERR_INVALID_ARG;
    int h = 0;
    st = cuda_status(cudaMemcpy(&h, ws, sizeof(int), cudaMemcpyDeviceToHost));
    if (st != TD_OK) return st;
    if (h == 0) return TD_OK;
    if (bits) *bits = h;
    st = cuda_status(cudaMemset(ws, 0, wsb));
    if (st != TD_OK) return st;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        remember_workspace(ws, static_cast<long long>((wsb - td::kErrRegion) / 4));
    }
    return TD_ERR_DEVICE;
}

const char* td_status_string(td_status s) {
    switch (s) {
        case TD_OK: return "ok";
        case TD_ERR_INVALID_ARG: return "invalid argument";
        case TD_ERR_UNSUPPORTED: return "unsupported head size or element type";
        case TD_ERR_CUDA: return "CUDA runtime error";
        case TD_ERR_NO_MEMORY: return "out of device memory";
        case TD_ERR_DEVICE: return "kernel reported an error";
        case TD_ERR_WORKSPACE: return "workspace too small";
        default: return "unknown status";
    }
}

int td_last_cuda_error(void) {
    const int e = g_last_cuda;
    g_last_cuda = 0;
    return e;
}

void td_release_workspace(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return;
    for (int d = 0; d < kMaxDevices; ++d) {
        DevState& s = g_dev[d];
        if (!s.ws && !s.stage) continue;
        if (cudaSetDevice(d) != cudaSuccess) continue;
        cudaDeviceSynchronize();
        if (s.ws) {
            cudaFree(s.ws);
            forget_workspace(s.ws);
        }
        if (s.stage) cudaFree(s.stage);
        s.ws = s.stage = nullptr;
        s.ws_bytes = s.stage_bytes = 0;
    }
    cudaSetDevice(cur);
}

td_status td_set_wait_test(uint64_t wait_limit_ns, int64_t withhold_tile) {
    if (wait_limit_ns != 0 && (wait_limit_ns < 1000ull || wait_limit_ns > 10000000000ull))
        return TD_ERR_INVALID_ARG;
    if (withhold_tile < -1) return TD_ERR_INVALID_ARG;
    g_wait_ns = wait_limit_ns == 0 ? kDefaultWaitNs : wait_limit_ns;
    g_withhold_tile = withhold_tile;
    return TD_OK;
}

uint64_t td_launch_count(void) { return g_launches; }

td_status td_set_kernel_events(void* before, void* after) {
    if ((before == nullptr) != (after == nullptr)) return TD_ERR_INVALID_ARG;
    g_ev_before = static_cast<cudaEvent_t>(before);
    g_ev_after = static_cast<cudaEvent_t>(after);
    return TD_OK;
}

const char* td_last_kernel(void) { return g_last_kernel; }

int td_version(void) { return 100; }

}  // extern "C"
