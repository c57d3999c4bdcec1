// Read-bandwidth probe: the denominator for kernels whose bytes come from L2
// (the loop block's weights, re-read every iteration) rather than HBM.
//
// A grid of CTAs sized to the SMs reads a buffer with 16-byte loads, each
// thread keeping 8 loads in flight, `reps` times over; every CTA folds what it
// read into one word of the sink so the loads cannot be dropped.  A buffer well
// under the L2 capacity stays resident after the first pass (the L2 figure); a
// buffer many times the L2 capacity measures HBM reads.
#include "common.cuh"
#include "host_util.h"

namespace tl {

__global__ void __launch_bounds__(512) read_probe_kernel(const uint4* __restrict__ src, int64_t n16, int reps,
                                                         uint32_t* __restrict__ sink) {
  constexpr int U = 8;
  uint32_t acc = 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int r = 0; r < reps; ++r) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; i + (U - 1) * stride < n16; i += U * stride) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) v[u] = __ldcg(src + i + u * stride);
#pragma unroll
      for (int u = 0; u < U; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
    }
    for (; i < n16; i += stride) {
      const uint4 v = __ldcg(src + i);
      acc ^= v.x ^ v.y ^ v.z ^ v.w;
    }
  }
  acc = __reduce_xor_sync(0xffffffffu, acc);
  __shared__ uint32_t red[16];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t a = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) a ^= red[w];
    sink[blockIdx.x] = a;
  }
}

}  // namespace tl

using namespace tl;

extern "C" int tl_read_probe(const void* dev_src, size_t bytes, int32_t reps, uint32_t* dev_sink, int32_t n_sink,
                             void* cuda_stream) {
  if (!dev_src || !dev_sink || bytes < 16 || bytes % 16 || ((uintptr_t)dev_src & 15) || reps < 1 ||
      ((uintptr_t)dev_sink & 3))
    return TL_EINVAL;
  int dev = 0, sms = 0;
  TL_CUDA(cudaGetDevice(&dev));
  TL_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const int grid = 4 * sms;  // four 512-thread CTAs per SM
  if (n_sink < grid) return TL_EINVAL;
  read_probe_kernel<<<grid, 512, 0, (cudaStream_t)cuda_stream>>>(static_cast<const uint4*>(dev_src),
                                                                  (int64_t)(bytes / 16), reps, dev_sink);
  return check_cuda(cudaGetLastError());
}
