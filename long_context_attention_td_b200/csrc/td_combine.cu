// td_tree_combine -- merge caller-provided partial softmax states per (b,h)
// (td_combine), and the gathered states of a sequence-sharded decode
// (td_merge_shards)
// ("Tree Attention Decoding" gist, tree_attn_decode after "first get global
// max": all-reduce MAX of the local maxima, renormalise by e^(m - M), two
// all-reduce SUMs, divide).  One CTA per (b,h); the max and the sums run as
// log-depth trees over the parts (dev::tree_merge), the same routine the
// fused ticket combine of td_partial uses.
#include "td_device.cuh"
#include "td_internal.cuh"

namespace td {
namespace {

using namespace dev;

constexpr int kCombineThreads = 256;
constexpr int kCombineScratch = 2048;  // weights of up to 2048 parts per chunk

// Dense caller layout: num [rows, S, D], m and l [rows, S], m in natural-log
// units (converted to the log2 units of tree_merge).
struct DenseAcc {
    static constexpr bool kSplitL = false;
    const float* pn;
    const float* pm;
    const float* pl;
    long long row;
    int S, D;
    __device__ __forceinline__ float m2(int i) const { return __ldg(pm + row * S + i) * kLog2e; }
    __device__ __forceinline__ float l(int i) const { return __ldg(pl + row * S + i); }
    __device__ __forceinline__ float num(int i, int d) const {
        return __ldg(pn + (row * S + i) * D + d);
    }
};

__global__ void __launch_bounds__(kCombineThreads) td_tree_combine_kernel(
    const float* __restrict__ num, const float* __restrict__ m, const float* __restrict__ l,
    float* __restrict__ out, float* __restrict__ lse, int S, int D) {
    __shared__ float scratch[kCombineScratch];
    const long long row = blockIdx.x;
    const DenseAcc acc{num, m, l, row, S, D};
    tree_merge(acc, S, D, static_cast<int>(threadIdx.x), kCombineThreads, scratch,
               kCombineScratch, 1, out + row * D, lse ? lse + row : nullptr);
}

// Gathered shard states ("Tree Attention Decoding" gist: every rank's
// normalised partial output and its log-sum-exp, gathered over the ranks):
// shard i holds out [rows][D] then lse [rows] (natural log), rows*(D+1) floats.
// As partial states (num, m, l) = (out, lse, 1): e^(lse_i - M) out_i summed
// over shards and divided by the summed e^(lse_i - M) is the whole sequence's
// softmax average, and M + ln of that sum its log-sum-exp.
struct ShardAcc {
    static constexpr bool kSplitL = false;
    const float* st;
    long long rows, row;
    int D;
    __device__ __forceinline__ long long stride() const { return rows * (D + 1); }
    __device__ __forceinline__ float m2(int i) const {
        return __ldg(st + i * stride() + rows * D + row) * kLog2e;
    }
    __device__ __forceinline__ float l(int) const { return 1.f; }
    __device__ __forceinline__ float num(int i, int d) const {
        return __ldg(st + i * stride() + row * D + d);
    }
};

__global__ void __launch_bounds__(kCombineThreads) td_merge_shards_kernel(
    const float* __restrict__ states, int W, long long rows, int D, float* __restrict__ out,
    float* __restrict__ lse) {
    __shared__ float scratch[kCombineScratch];
    const long long row = blockIdx.x;
    const ShardAcc acc{states, rows, row, D};
    tree_merge(acc, W, D, static_cast<int>(threadIdx.x), kCombineThreads, scratch,
               kCombineScratch, 1, out + row * D, lse ? lse + row : nullptr);
}

// A shard with no keys: its partial output is 0 and its log-sum-exp -inf.
__global__ void td_empty_state_kernel(float* __restrict__ out, float* __restrict__ lse,
                                      long long rows, int D) {
    const long long n = rows * D;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n + rows;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        if (i < n)
            out[i] = 0.f;
        else if (lse)
            lse[i - n] = kNegInf;
    }
}

}  // namespace

cudaError_t launch_merge_shards(const float* states, int W, long long rows, int D, float* out,
                                float* lse, cudaStream_t s) {
    if (rows <= 0 || rows > 0x7fffffffLL || W < 1) return cudaErrorInvalidValue;
    td_merge_shards_kernel<<<static_cast<unsigned>(rows), kCombineThreads, 0, s>>>(states, W, rows,
                                                                                  D, out, lse);
    return cudaGetLastError();
}

cudaError_t launch_empty_state(float* out, float* lse, long long rows, int D, cudaStream_t s) {
    if (rows <= 0) return cudaErrorInvalidValue;
    const long long n = rows * (D + 1);
    long long blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    td_empty_state_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(out, lse, rows, D);
    return cudaGetLastError();
}

cudaError_t launch_combine(const float* num, const float* m, const float* l, float* out,
                           float* lse, int64_t rows, int S, int D, cudaStream_t s) {
    if (rows <= 0 || rows > 0x7fffffffLL) return cudaErrorInvalidValue;
    td_tree_combine_kernel<<<static_cast<unsigned>(rows), kCombineThreads, 0, s>>>(num, m, l, out,
                                                                                 lse, S, D);
    return cudaGetLastError();
}

}  // namespace td
