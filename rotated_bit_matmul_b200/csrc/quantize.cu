// Group-wise uniform quantizer (the library's stand-in codebook; the HARP pages leave
// the codebook to the backend, Sec. 2.4 "Compatibilidade") and code packing.
//
// One warp per (output row, group of 64 columns); lane l holds columns 2l, 2l+1.
//   zero16 = fp16(min), scale16 = fp16((max - min) / (2^b - 1)), 1 if that is 0,
//   q = clamp(round_half_even((w - zero16) / scale16), 0, 2^b - 1).
// The rule is evaluated in fp64 (the inputs are fp32, so min, max and every
// difference are exact), which gives the codes an fp64 evaluation would give.
#include "common.cuh"

namespace harp {

__global__ void __launch_bounds__(256) quantize_kernel(int64_t n_out, int64_t n_in, int bits,
                                                       const float* __restrict__ W, uint32_t* codes,
                                                       uint32_t* sz) {
  const int lane = threadIdx.x & 31;
  const int64_t ng = n_in / 64;
  const int64_t total = n_out * ng;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); gw < total; gw += nwarps) {
    const int64_t r = gw / ng, g = gw % ng;
    const float2 v = *reinterpret_cast<const float2*>(W + r * n_in + g * 64 + 2 * lane);
    float mn = fminf(v.x, v.y), mx = fmaxf(v.x, v.y);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const double L = (double)((1 << bits) - 1);
    const __half zh = __double2half((double)mn);
    __half sh = __double2half(((double)mx - (double)mn) / L);
    if (__half2float(sh) == 0.f) sh = __ushort_as_half((unsigned short)0x3C00u);
    const double zd = (double)__half2float(zh), sd = (double)__half2float(sh);
    unsigned q[2];
    const float vv[2] = {v.x, v.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      double t = rint(((double)vv[i] - zd) / sd);
      if (!(t >= 0.0)) t = 0.0;
      if (t > L) t = L;
      q[i] = (unsigned)t;
    }
    if (lane == 0)
      sz[gw] = (uint32_t)__half_as_ushort(sh) | ((uint32_t)__half_as_ushort(zh) << 16);

    // pack: every lane contributes its two codes to one word, OR-reduced over the
    // lanes that share that word
    if (bits == 2 || bits == 3) {
      const uint32_t part = ((q[0] & 3u) | ((q[1] & 3u) << 2)) << (4 * (lane & 7));
      uint32_t word = part;
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) word |= __shfl_xor_sync(0xffffffffu, word, o);
      if ((lane & 7) == 0) codes[(r * n_in + g * 64) / 16 + (lane >> 3)] = word;
      if (bits == 3) {
        // 1-bit plane after the n_out*n_in/4 bytes of the 2-bit plane
        const uint32_t hb = ((q[0] >> 2) & 1u) << ((2 * lane) & 31) | ((q[1] >> 2) & 1u) << ((2 * lane + 1) & 31);
        uint32_t hw = hb;
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) hw |= __shfl_xor_sync(0xffffffffu, hw, o);
        if ((lane & 15) == 0) codes[(n_out * n_in) / 16 + (r * n_in + g * 64) / 32 + (lane >> 4)] = hw;
      }
    } else {  // 4 bits: lanes 4k..4k+3 fill word k
      const uint32_t part = ((q[0] & 15u) | ((q[1] & 15u) << 4)) << (8 * (lane & 3));
      uint32_t word = part;
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) word |= __shfl_xor_sync(0xffffffffu, word, o);
      if ((lane & 3) == 0) codes[(r * n_in + g * 64) / 8 + (lane >> 2)] = word;
    }
  }
}

cudaError_t launch_quantize(int64_t n_out, int64_t n_in, int bits, const float* W, void* codes,
                            void* scale_zero, cudaStream_t st) {
  const int64_t total = n_out * (n_in / 64);
  if (total <= 0) return cudaSuccess;
  int64_t blocks = (total + 7) / 8;
  if (blocks > 148 * 64) blocks = 148 * 64;
  quantize_kernel<<<(unsigned)blocks, 256, 0, st>>>(n_out, n_in, bits, W, static_cast<uint32_t*>(codes),
                                                    static_cast<uint32_t*>(scale_zero));
  return cudaGetLastError();
}

}  // namespace harp
