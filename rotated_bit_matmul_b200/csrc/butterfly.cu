// Butterfly transform F(theta, s, w) and its transpose on sm_100a.
//
// "HARP: Hadamard-Preconditioned Adaptive Rotation Processor for Extreme LLM
// Quantization", Sec. 2.1-2.2: a product of stride stages, each a block-diagonal
// orthogonal matrix of 2x2 blocks B = Q(theta) G_2 (Givens times the normalised
// Sylvester H_2), i.e. [[cos p, sin p], [sin p, -cos p]] with p = pi/4 + theta.
// Forward: signs, then stages of stride 1, 2, ..., w/2. Transpose: stages in
// reverse, then signs (each 2x2 block is symmetric).
//
// One CTA owns one w-wide block (w <= 8192, 32 KB of fp32 in shared memory) of one
// row and runs all log2(w) stages there; the optional epilogue turns the result
// into the operand the dequant-GEMV reads (int16 values in dp2a pair order, one
// power-of-two scale and one fp32 sum per group of 64).
#include "common.cuh"

namespace harp {

// Position (int16 index inside the group's 32-word block) of column j (0..63) of a
// group in the dp2a pair order the GEMV expects for its code format.
__device__ __forceinline__ int xq_pos_lo(int bits, int j) {
  if (bits == 4) {
    const int c = j >> 3, r = j & 7;
    return (c * 4 + (r & 1) * 2 + (r >> 2)) * 2 + ((r >> 1) & 1);
  }
  const int c = j >> 4, r = j & 15, m = r & 3, q = r >> 2;  // 2-bit codes / 2-bit plane
  return (c * 8 + 2 * m + (q >> 1)) * 2 + (q & 1);
}
__device__ __forceinline__ int xq_pos_hi(int j) {  // 1-bit plane of 3-bit codes
  const int c = j >> 5, r = j & 31, m = r & 7, q = r >> 3;
  return (c * 16 + 2 * m + (q >> 1)) * 2 + (q & 1);
}

__global__ void __launch_bounds__(512) bfly_kernel(BflyParams p) {
  extern __shared__ float sx[];
  const int w = p.w, m = p.m;
  const int64_t k = blockIdx.x, row = blockIdx.y;
  const int64_t base = k * w;
  const int nthr = blockDim.x, tid = threadIdx.x;
  const int64_t half_n = p.n >> 1;
  const float kQuarterPi = 0.785398163397448309616f;

  for (int i = tid; i < w; i += nthr) {
    float v = load_act(p.x, row * p.x_stride + base + i, p.xt);
    if (!p.inverse) v *= (float)p.sign[base + i];
    sx[i] = v;
  }
  __syncthreads();

  for (int s = 0; s < m; ++s) {
    const int t = p.inverse ? (m - 1 - s) : s;
    const int h = 1 << t;
    const int64_t off = (int64_t)t * half_n + k * (w >> 1);
    for (int q = tid; q < (w >> 1); q += nthr) {
      const int i = ((q >> t) << (t + 1)) | (q & (h - 1));
      float c, sn;
      if (p.cs) {
        const float2 v = p.cs[off + q];
        c = v.x;
        sn = v.y;
      } else {
        sincosf(kQuarterPi + p.theta[off + q], &sn, &c);
      }
      const float a = sx[i], b = sx[i + h];
      sx[i] = fmaf(c, a, sn * b);
      sx[i + h] = fmaf(sn, a, -c * b);
    }
    __syncthreads();
  }

  if (p.inverse)
    for (int i = tid; i < w; i += nthr) sx[i] *= (float)p.sign[base + i];
  if (p.inverse) __syncthreads();

  if (p.y)
    for (int i = tid; i < w; i += nthr) store_act(p.y, row * p.y_stride + base + i, p.yt, sx[i]);

  if (p.xq) {
    // Per group of 64: e = 15 - E with max|v| = f 2^E, f in [0.5, 1), so that
    // max|v| 2^e < 2^15; int16 value = rint(v 2^e) (clamped to +-32767).
    const int lane = tid & 31, warp = tid >> 5, nwarps = nthr >> 5;
    int16_t* xq16 = reinterpret_cast<int16_t*>(p.xq + row * p.xq_stride);
    for (int g = warp; g < (w >> 6); g += nwarps) {
      const float v0 = sx[g * 64 + 2 * lane], v1 = sx[g * 64 + 2 * lane + 1];
      float amax = fmaxf(fabsf(v0), fabsf(v1));
      float sum = v0 + v1;
      const bool bad = __any_sync(0xffffffffu, !(isfinite(v0) && isfinite(v1)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
      }
      int e = 0;
      if (amax > 0.f && !bad) {
        int E;
        frexpf(amax, &E);
        e = min(max(15 - E, -126), 126);
      }
      const float sc = ldexpf(1.f, e);
      const int q0 = max(-32767, min(32767, __float2int_rn(v0 * sc)));
      const int q1 = max(-32767, min(32767, __float2int_rn(v1 * sc)));
      const int64_t gg = k * (w >> 6) + g;
      int16_t* grp = xq16 + gg * 64;
      grp[xq_pos_lo(p.bits, 2 * lane)] = (int16_t)q0;
      grp[xq_pos_lo(p.bits, 2 * lane + 1)] = (int16_t)q1;
      if (p.bits == 3) {
        int16_t* hi = xq16 + p.n + gg * 64;  // hi-plane order starts after n int16 values
        hi[xq_pos_hi(2 * lane)] = (int16_t)q0;
        hi[xq_pos_hi(2 * lane + 1)] = (int16_t)q1;
      }
      if (lane == 0) {
        p.xs[row * p.g_stride + gg] = bad ? __int_as_float(0x7fc00000) : ldexpf(1.f, -e);
        p.xsum[row * p.g_stride + gg] = bad ? __int_as_float(0x7fc00000) : sum;
      }
    }
  }
}

cudaError_t launch_butterfly(const BflyParams& p, int batch, cudaStream_t st) {
  if (batch <= 0) return cudaSuccess;
  const int threads = p.w >= 1024 ? 512 : (p.w >= 64 ? p.w / 2 : 32);
  const size_t smem = sizeof(float) * (size_t)p.w;
  // at most 32 KB of dynamic shared memory: below the default 48 KB limit
  dim3 grid((unsigned)(p.n / p.w), (unsigned)batch);
  bfly_kernel<<<grid, threads, smem, st>>>(p);
  return cudaGetLastError();
}

// cos/sin tables of pi/4 + theta, computed once per layer in fp32.
__global__ void cs_table_kernel(const float* theta, int64_t count, float2* cs) {
  const float kQuarterPi = 0.785398163397448309616f;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x) {
    float s, c;
    sincosf(kQuarterPi + theta[i], &s, &c);
    cs[i] = make_float2(c, s);
  }
}

cudaError_t launch_cs_table(const float* theta, int64_t count, float2* cs, cudaStream_t st) {
  if (count <= 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (count + threads - 1) / threads;
  cs_table_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), threads, 0, st>>>(theta, count, cs);
  return cudaGetLastError();
}

}  // namespace harp
