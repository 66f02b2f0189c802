// Relative L1 error of an attention output against a reference, the
// quantity the per-layer calibration of the SpargeAttention notes bounds
// ([P3] 2.4: L1 = sum |O - O'| / sum |O|).
//
// One pass over both tensors: each thread accumulates |ref - x| and |ref| of
// 16-byte vectors in fp64 (long sums of positive terms), a warp reduces with
// shuffles, and one lane per warp adds its pair to the two output sums with
// fp64 atomics.  Memory-bound: 2 x n x element size bytes read.
#include "sa_internal.cuh"

namespace sa {
namespace {

template <typename T>
__global__ void __launch_bounds__(256) l1_kernel(const uint4* __restrict__ ref, const uint4* __restrict__ x,
                                                 int64_t nvec, double* __restrict__ sums) {
  constexpr int EPL = 16 / sizeof(T);
  double dsum = 0.0, rsum = 0.0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nvec; i += stride) {
    float a[EPL], b[EPL];
    unpack16(__ldg(ref + i), T(), a);
    unpack16(__ldg(x + i), T(), b);
    float ds = 0.f, rs = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      ds += fabsf(a[e] - b[e]);
      rs += fabsf(a[e]);
    }
    dsum += ds;
    rsum += rs;
  }
  for (int off = 16; off > 0; off >>= 1) {
    dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
    rsum += __shfl_xor_sync(0xffffffffu, rsum, off);
  }
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(&sums[0], dsum);
    atomicAdd(&sums[1], rsum);
  }
}

}  // namespace

sa_status launch_l1(const void* ref, const void* x, int64_t n, int32_t dtype, double* sums, cudaStream_t st) {
  if (cudaMemsetAsync(sums, 0, 2 * sizeof(double), st) != cudaSuccess)
    return set_error(SA_ERR_CUDA, "cudaMemsetAsync(sums) failed");
  const int64_t esz = dtype == SA_BF16 ? 2 : 4;
  const int64_t nvec = n * esz / 16;
  if (nvec == 0) return SA_OK;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = ceil_div(nvec, 256);
  const int grid = (int)min64(want, (int64_t)sms * 8);
  if (dtype == SA_BF16)
    l1_kernel<uint16_t><<<grid, 256, 0, st>>>(static_cast<const uint4*>(ref), static_cast<const uint4*>(x), nvec,
                                              sums);
  else
    l1_kernel<float><<<grid, 256, 0, st>>>(static_cast<const uint4*>(ref), static_cast<const uint4*>(x), nvec,
                                           sums);
  return check_launch("l1_kernel");
}

}  // namespace sa
