// Glue kernels of a linear whose sides are mixed-radix butterflies (harp_create_layer_mr):
// the int16 GEMV operand of an fp32 transformed input, and the fixed-order sum of the
// tensor-core path's split partials. The transforms themselves are the mixed-radix
// kernel's (mixed_radix.cu); the GEMV and the tcgen05 contraction are the radix-2 layers'.
#include "common.cuh"

namespace harp {
namespace {

// one warp per group of 64: blockIdx.y = row, 8 groups per CTA
__global__ void __launch_bounds__(256) operand_prep_kernel(const float* __restrict__ x, int64_t n, int bits,
                                                           int32_t* xq, int64_t xq_stride, float* xs, float* xsum,
                                                           int64_t g_stride) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row = blockIdx.y, g = (int64_t)blockIdx.x * 8 + warp;
  if (g >= n / 64) return;
  int16_t* q16 = reinterpret_cast<int16_t*>(xq + row * xq_stride);
  prep_group(x + row * n + g * 64, bits, q16 + g * 64, q16 + n + g * 64, xs + row * g_stride + g,
             xsum + row * g_stride + g, lane);
}

__global__ void sum_splits_kernel(const float* __restrict__ part, int splits, int64_t count, float* __restrict__ z) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x) {
    float t = part[i];
    for (int s = 1; s < splits; ++s) t += part[(int64_t)s * count + i];
    z[i] = t;
  }
}

}  // namespace

cudaError_t launch_operand_prep(const float* x, int64_t n, int bits, int batch, int32_t* xq, int64_t xq_stride,
                                float* xs, float* xsum, int64_t g_stride, cudaStream_t st) {
  if (batch <= 0) return cudaSuccess;
  const dim3 grid((unsigned)((n / 64 + 7) / 8), (unsigned)batch);
  operand_prep_kernel<<<grid, 256, 0, st>>>(x, n, bits, xq, xq_stride, xs, xsum, g_stride);
  return cudaGetLastError();
}

cudaError_t launch_sum_splits(const float* part, int splits, int64_t count, float* z, cudaStream_t st) {
  if (count <= 0) return cudaSuccess;
  int64_t blocks = (count + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  sum_splits_kernel<<<(unsigned)blocks, 256, 0, st>>>(part, splits, count, z);
  return cudaGetLastError();
}

}  // namespace harp
