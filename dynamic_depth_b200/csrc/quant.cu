// Weight preparation on the device: symmetric per-group INT4 quantisation
// ("Benchmark Comparison" (measured benchmarks), section 7: per-group min-max,
// no calibration; section 5: the symmetric (q - 8) * scale convention), the
// exact INT4 dequant, and float64 -> bfloat16 rounding.
#include "common.cuh"
#include "host_util.h"

namespace tl {

// One warp per (row, group): scale = fp16_rne(max|w| / 7).
__global__ void int4_scales_kernel(const double* __restrict__ w, int64_t N, int64_t K, int group,
                                   __half* __restrict__ scales) {
  const int64_t gpr = K / group;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= N * gpr) return;
  const int64_t n = warp / gpr, j = warp % gpr;
  const double* p = w + n * K + j * group;
  double m = 0.0;
  for (int i = lane; i < group; i += 32) m = fmax(m, fabs(p[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) scales[warp] = __double2half(m / 7.0);
}

// One thread per output byte: two codes, rint(w / s) (ties to even) clamped to
// [-7, 7], stored as nibbles code + 8, element 2i in the low nibble.
__global__ void int4_pack_kernel(const double* __restrict__ w, int64_t N, int64_t K, int group,
                                 const __half* __restrict__ scales, uint8_t* __restrict__ packed) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N * K / 2) return;
  const int64_t n = (2 * i) / K, k = (2 * i) % K;
  const double s = (double)__half2float(scales[n * (K / group) + k / group]);
  uint32_t u[2];
  for (int e = 0; e < 2; ++e) {
    double q = 0.0;
    if (s > 0.0) q = fmin(7.0, fmax(-7.0, rint(w[n * K + k + e] / s)));
    u[e] = (uint32_t)((int)q + 8);
  }
  packed[i] = (uint8_t)(u[0] | (u[1] << 4));
}

__global__ void int4_dequant_kernel(const uint8_t* __restrict__ packed, const __half* __restrict__ scales,
                                    int64_t N, int64_t K, int group, float* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N * K / 2) return;
  const int64_t n = (2 * i) / K, k = (2 * i) % K;
  const float s = __half2float(scales[n * (K / group) + k / group]);
  const uint32_t b = packed[i];
  out[n * K + k] = nib_to_f(b, 0) * s;
  out[n * K + k + 1] = nib_to_f(b, 4) * s;
}

// float64 -> nearest bfloat16 (ties to even), by rounding the float64 bit
// pattern to 8 significant bits; below 2^-126 (bfloat16 subnormals) the grid is
// the fixed spacing 2^-133.
__device__ __forceinline__ uint16_t f64_to_bf16_bits(double x) {
  double r;
  if (fabs(x) < 0x1p-126) {
    r = rint(x * 0x1p133) * 0x1p-133;
  } else {
    unsigned long long b = (unsigned long long)__double_as_longlong(x);
    const unsigned long long lsb = (b >> 45) & 1ull;
    b += (1ull << 44) - 1ull + lsb;
    b &= ~((1ull << 45) - 1ull);
    r = __longlong_as_double((long long)b);
  }
  const float f = (float)r;  // exact: r has at most 8 significant bits and fits float's range (or is inf)
  return (uint16_t)(__float_as_uint(f) >> 16);
}

__global__ void round_bf16_kernel(const double* __restrict__ w, int64_t n, uint16_t* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = f64_to_bf16_bits(w[i]);
}

}  // namespace tl

using namespace tl;

static unsigned blocks_for(int64_t n, int t) { return (unsigned)((n + t - 1) / t); }

extern "C" int tl_quantize_int4(const double* dev_w, int64_t N, int64_t K, int32_t group,
                                uint8_t* dev_packed, uint16_t* dev_scales, void* stream) {
  if (!dev_w || !dev_packed || !dev_scales || N <= 0 || K <= 0 || group <= 0 || group % 32 ||
      K % group)
    return TL_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  const int64_t groups = N * (K / group);
  int4_scales_kernel<<<blocks_for(groups * 32, 256), 256, 0, s>>>(dev_w, N, K, group,
                                                                  (__half*)dev_scales);
  int4_pack_kernel<<<blocks_for(N * K / 2, 256), 256, 0, s>>>(dev_w, N, K, group,
                                                             (const __half*)dev_scales, dev_packed);
  return check_cuda(cudaGetLastError());
}

extern "C" int tl_dequant_int4(const uint8_t* dev_packed, const uint16_t* dev_scales, int64_t N,
                               int64_t K, int32_t group, float* dev_out, void* stream) {
  if (!dev_packed || !dev_scales || !dev_out || N <= 0 || K <= 0 || group <= 0 || group % 2 ||
      K % group)
    return TL_EINVAL;
  int4_dequant_kernel<<<blocks_for(N * K / 2, 256), 256, 0, (cudaStream_t)stream>>>(
      dev_packed, (const __half*)dev_scales, N, K, group, dev_out);
  return check_cuda(cudaGetLastError());
}

extern "C" int tl_round_bf16(const double* dev_w, int64_t n, uint16_t* dev_out, void* stream) {
  if (!dev_w || !dev_out || n <= 0) return TL_EINVAL;
  round_bf16_kernel<<<blocks_for(n, 256), 256, 0, (cudaStream_t)stream>>>(dev_w, n, dev_out);
  return check_cuda(cudaGetLastError());
}
