// td_decode_static -- td_decode for callers that cannot allocate device
// memory.
//
// Some callers of a decode kernel are not allowed to allocate: a serving
// engine that reserves nearly all HBM for its KV-cache pool up front leaves a
// cudaMalloc nothing to take (or lets it fragment the pool), a host
// application that loads this library as a plug-in may own every device
// allocation itself, and a latency-critical decode loop cannot absorb the
// device-wide synchronisation a cudaMalloc/cudaFree may cause.  td_decode
// lazily allocates its workspace (error word, tickets, part records) on first
// use; this entry point instead takes that scratch from a fixed array in the
// library's own device image, so it never allocates.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds TD_STATIC_SCRATCH_BYTES of it until the process exits.  Host
// code only sees a host-side stand-in under the array's name, so its device
// address is fetched once per device with cudaGetSymbolAddress (with that
// device current) and passed to the kernels as a plain pointer.
#include <cuda_runtime.h>

#include <mutex>

#include "treedec.h"

namespace {

constexpr size_t kScratchBytes = TD_STATIC_SCRATCH_BYTES;
static_assert(kScratchBytes % 256 == 0, "scratch keeps 256-byte alignment");

// Shared by every td_decode_static call on a device; keeps the last call's
// contents between calls.
static __device__ __align__(256) unsigned char g_static_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_ptr[kMaxDevices] = {};

// Device address of the scratch on device `dev` (the current device).  The
// first call on a device fetches it and zero-fills the array (the error word
// and the tickets must start at zero).  cudaMemset is ordered only on the
// legacy default stream, which a caller's non-blocking stream does not wait
// for, so the device is synchronised before the address is handed out.
td_status static_scratch(int dev, void** out) {
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (g_static_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
            return TD_ERR_CUDA;
        if (cudaMemset(p, 0, kScratchBytes) != cudaSuccess) return TD_ERR_CUDA;
        if (cudaDeviceSynchronize() != cudaSuccess) return TD_ERR_CUDA;
        g_static_ptr[dev] = p;
    }
    *out = g_static_ptr[dev];
    return TD_OK;
}

// The scratch address of the current device if a static call has set it up,
// else nullptr.
td_status static_scratch_if_set(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return TD_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return TD_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_static_mu);
    *out = g_static_ptr[dev];
    return TD_OK;
}

}  // namespace

extern "C" td_status td_decode_static(const void* q, const void* k, const void* v, float* out,
                                      float* lse, int B, int H, int64_t N, int D, int n_split,
                                      const float* alibi_slopes, td_dtype dtype,
                                      td_stream stream) {
    if (dtype != TD_F32 && dtype != TD_BF16 && dtype != TD_F16) return TD_ERR_UNSUPPORTED;
    if (D != 64 && D != 128 && D != 256 && D != 512) return TD_ERR_UNSUPPORTED;
    if (n_split < 0 || B < 1 || H < 1 || N < 1) return TD_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return TD_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return TD_ERR_UNSUPPORTED;
    // the same part count td_decode would use, and the scratch it needs
    const int64_t parts = td_plan_parts(B, H, N, D, dtype, n_split, -1);
    if (parts < 1) return TD_ERR_INVALID_ARG;
    const size_t need = td_workspace_bytes(B, H, D, parts);
    if (need == 0 || need > kScratchBytes) return TD_ERR_WORKSPACE;
    void* scratch = nullptr;
    const td_status st = static_scratch(dev, &scratch);
    if (st != TD_OK) return st;
    return td_decode_ws(q, k, v, out, lse, B, H, N, D, nullptr, nullptr, parts, alibi_slopes,
                        dtype, scratch, kScratchBytes, stream);
}

extern "C" td_status td_check_static_error(int* bits, td_stream stream) {
    if (bits) *bits = 0;
    void* scratch = nullptr;
    const td_status st = static_scratch_if_set(&scratch);
    if (st != TD_OK) return st;
    if (scratch == nullptr) {
        // no static call has run on this device: nothing can have failed,
        // but the caller still gets the stream's own errors
        return cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
                   ? TD_OK
                   : TD_ERR_CUDA;
    }
    // the error word and the ticket/record layout of the array are those of a
    // caller workspace of kScratchBytes
    return td_check_device_error(scratch, kScratchBytes, bits, stream);
}
