// td_tree_combine -- merge caller-provided partial softmax states per (b,h)
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

}  // namespace

cudaError_t launch_combine(const float* num, const float* m, const float* l, float* out,
                           float* lse, int64_t rows, int S, int D, cudaStream_t s) {
    if (rows <= 0 || rows > 0x7fffffffLL) return cudaErrorInvalidValue;
    td_tree_combine_kernel<<<static_cast<unsigned>(rows), kCombineThreads, 0, s>>>(num, m, l, out,
                                                                                 lse, S, D);
    return cudaGetLastError();
}

}  // namespace td
