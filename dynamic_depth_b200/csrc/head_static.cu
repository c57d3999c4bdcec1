// Greedy LM head that allocates nothing: RMSNorm of caller-given hidden rows,
// INT4 head projection, and argmax (lowest id on ties), with every
// intermediate in one fixed-size array in device global memory that this
// library defines at file scope.
//
// Why it exists: some callers cannot allocate device memory when they want
// the head.  A serving loop that reserved all of its device memory at start-up
// and forbids allocation afterwards, an allocator-managed host framework that
// owns every cudaMalloc, or code running while a stream is being captured
// (where cudaMalloc is not allowed) can still pass its inputs and outputs, but
// cannot supply the scratch space the workspace-based path (tl_head_logits)
// takes from tl_create's workspace.  This entry point keeps that scratch in a
// static array instead.
//
// The static array and its limits: kMaxRows rows of kMaxD normalised
// activations plus kMaxRows x kMaxParts (value, index) partial maxima, about
// 1.5 MB, held by every GPU that loads the library until the process exits.
// Every call on a device uses the same array, which keeps the previous call's
// contents; each call writes every element it later reads, so nothing needs
// clearing, but two calls whose kernels overlap on the GPU (different streams,
// no ordering between them) race on it.  The first call on a device looks up
// the array's device address (cudaGetSymbolAddress with that device current);
// make that first call before any stream capture begins.
#include <mutex>

#include "common.cuh"
#include "host_util.h"

namespace tl {

namespace head_static {

constexpr int kMaxRows = 64;
constexpr int kMaxD = 4096;
constexpr int kRowsPerCta = 256;   // vocabulary rows per CTA (8 warps x 32)
constexpr int kMaxParts = 1024;    // so V <= 262144
constexpr size_t kXnBytes = (size_t)kMaxRows * kMaxD * 4;
constexpr size_t kPartBytes = (size_t)kMaxRows * kMaxParts * 4;
constexpr size_t kBytes = kXnBytes + 2 * kPartBytes;

// The whole scratch space of this entry point.  In host code this name is a
// host-side stand-in, not a device address: the device address comes from
// cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_scratch[kBytes];

__global__ void norm_kernel(const float* __restrict__ h, int d, const float* __restrict__ g, float eps,
                            float* __restrict__ xn) {
  __shared__ float red[32];
  const int r = blockIdx.x;
  const float* x = h + (int64_t)r * d;
  float ss = 0.f;
  for (int k = threadIdx.x; k < d; k += blockDim.x) ss += x[k] * x[k];
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / (float)d + eps);
  for (int k = threadIdx.x; k < d; k += blockDim.x) xn[(int64_t)r * d + k] = x[k] * inv * g[k];
}

// Weights in the blob's packing: byte k/2 holds element k (low nibble, k even)
// and k+1 (high nibble); value (u - 8) * scale.  Each warp takes 32
// consecutive vocabulary rows; a lane takes 32-element chunks of a row.
__global__ void __launch_bounds__(256) proj_argmax_kernel(const float* __restrict__ xn, int rows, int d,
                                                          const uint8_t* __restrict__ q,
                                                          const __half* __restrict__ s, int V, int group,
                                                          float* __restrict__ logits, float* __restrict__ part_v,
                                                          int32_t* __restrict__ part_i, int n_parts) {
  __shared__ float bv_s[8][kMaxRows];
  __shared__ int bi_s[8][kMaxRows];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float bv[kMaxRows / 32];
  int bi[kMaxRows / 32];  // lane l tracks rows l and l + 32
#pragma unroll
  for (int j = 0; j < kMaxRows / 32; ++j) { bv[j] = -INFINITY; bi[j] = 0x7fffffff; }
  const int v0 = blockIdx.x * kRowsPerCta + warp * 32;
  for (int vv = 0; vv < 32; ++vv) {
    const int v = v0 + vv;
    if (v >= V) break;
    for (int r = 0; r < rows; ++r) {
      float acc = 0.f;
      for (int c = lane; c < d / 32; c += 32) {
        const uint4 w = *reinterpret_cast<const uint4*>(q + (int64_t)v * (d / 2) + c * 16);
        const float sc = __half2float(s[(int64_t)v * (d / group) + (c * 32) / group]);
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
        const float* xr = xn + (int64_t)r * d + c * 32;
        float p = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int e = 0; e < 8; ++e) p = fmaf((float)(int)((u[j] >> (4 * e)) & 0xFu) - 8.f, xr[8 * j + e], p);
        acc = fmaf(p, sc, acc);
      }
      acc = warp_sum(acc);
      if (logits && lane == 0) logits[(int64_t)r * V + v] = acc;
      if (lane == (r & 31)) {
        const int j = r >> 5;
        if (acc > bv[j] || (acc == bv[j] && v < bi[j])) { bv[j] = acc; bi[j] = v; }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kMaxRows / 32; ++j) {
    bv_s[warp][lane + 32 * j] = bv[j];
    bi_s[warp][lane + 32 * j] = bi[j];
  }
  __syncthreads();
  for (int r = threadIdx.x; r < rows; r += blockDim.x) {
    float b = bv_s[0][r];
    int i = bi_s[0][r];
    for (int w = 1; w < 8; ++w)
      if (bv_s[w][r] > b || (bv_s[w][r] == b && bi_s[w][r] < i)) { b = bv_s[w][r]; i = bi_s[w][r]; }
    part_v[(int64_t)r * n_parts + blockIdx.x] = b;
    part_i[(int64_t)r * n_parts + blockIdx.x] = i;
  }
}

__global__ void finalize_kernel(const float* __restrict__ part_v, const int32_t* __restrict__ part_i, int n_parts,
                                int32_t* __restrict__ argmax) {
  const int r = blockIdx.x;
  if (threadIdx.x != 0) return;
  float b = -INFINITY;
  int i = 0x7fffffff;
  for (int p = 0; p < n_parts; ++p) {
    const float v = part_v[(int64_t)r * n_parts + p];
    const int ix = part_i[(int64_t)r * n_parts + p];
    if (v > b || (v == b && ix < i)) { b = v; i = ix; }
  }
  argmax[r] = i;
}

// Device address of g_scratch on each device, looked up once per device.
static std::mutex g_mu;
static void* g_addr[64];

static int scratch_for_current_device(unsigned char** out) {
  int dev = 0;
  TL_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return TL_EINVAL;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    TL_CUDA(cudaGetSymbolAddress(&p, g_scratch));
    g_addr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_addr[dev]);
  return TL_OK;
}

}  // namespace head_static
}  // namespace tl

using namespace tl;

extern "C" int tl_head_argmax_static(const float* dev_h, int32_t rows, const float* dev_g_final, float rms_eps,
                                     const uint8_t* dev_head_packed, const uint16_t* dev_head_scales, int32_t V,
                                     int32_t d, int32_t group, float* dev_logits, int32_t* dev_argmax,
                                     void* cuda_stream) {
  namespace hs = head_static;
  if (!dev_h || !dev_g_final || !dev_head_packed || !dev_head_scales || !dev_argmax) return TL_EINVAL;
  if (rows < 1 || d < 32 || d % 32 || group < 32 || group % 32 || d % group || V < 1) return TL_EINVAL;
  // the head rows are read as 16-byte words; everything else by its element size
  if (((uintptr_t)dev_head_packed & 15) || ((uintptr_t)dev_head_scales & 1) || ((uintptr_t)dev_h & 3) ||
      ((uintptr_t)dev_g_final & 3) || ((uintptr_t)dev_logits & 3) || ((uintptr_t)dev_argmax & 3))
    return TL_EINVAL;
  const int n_parts = (V + hs::kRowsPerCta - 1) / hs::kRowsPerCta;
  // sizes beyond the static array's capacity
  if (rows > hs::kMaxRows || d > hs::kMaxD || n_parts > hs::kMaxParts) return TL_ENOMEM;
  unsigned char* base = nullptr;
  TL_TRY(hs::scratch_for_current_device(&base));
  float* xn = reinterpret_cast<float*>(base);
  float* pv = reinterpret_cast<float*>(base + hs::kXnBytes);
  int32_t* pi = reinterpret_cast<int32_t*>(base + hs::kXnBytes + hs::kPartBytes);
  cudaStream_t s = (cudaStream_t)cuda_stream;
  hs::norm_kernel<<<rows, 256, 0, s>>>(dev_h, d, dev_g_final, rms_eps, xn);
  hs::proj_argmax_kernel<<<n_parts, 256, 0, s>>>(xn, rows, d, dev_head_packed,
                                                 reinterpret_cast<const __half*>(dev_head_scales), V, group,
                                                 dev_logits, pv, pi, n_parts);
  hs::finalize_kernel<<<rows, 32, 0, s>>>(pv, pi, n_parts, dev_argmax);
  return check_cuda(cudaGetLastError());
}
