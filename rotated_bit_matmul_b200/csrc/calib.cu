// Calibration objective of the rotated low-bit linear, on the device: the per-layer
// fitting loss of "HARP: Hadamard-Preconditioned Adaptive Rotation Processor for Extreme
// LLM Quantization", Sec. 2.3 (Objetivo de Otimizacao), and its gradient in the angles.
//
//   W' = U W V^T,  T = deq(Q(W')),  H' = V H V^T,  d = diag(H')
//   L_diag = sum_{r,j} d_j (W' - T)_rj^2
//   R_bd   = sum of H'_ij^2 over i, j in different 64-column quantizer groups
//   L_fit  = L_diag + lambda_bd R_bd
//
// The gradient holds T constant (the page stops gradients through the code assignment)
// and flows into theta_U through W' and into theta_V through W', d and R_bd.
//
// The pieces:
//   - rotations use the library's butterfly kernels; a tiled transpose turns columns
//     into rows;
//   - the codes and their scale/zero words come from the quantizer the linear uses;
//   - bfly_back_kernel runs a butterfly backwards from its outputs. Every 2x2 block
//     B(p) = [[c, s], [s, -c]], p = pi/4 + theta, is its own inverse, so each stage's
//     inputs are the block applied to its outputs. The block's derivative in p maps
//     (a, b) to (-v, u), so dL/dtheta = g_v u - g_u v needs only the outputs (u, v) and
//     their gradients (g_u, g_v);
//   - every sum is fp64 or ends in fp64, in a fixed order, so results repeat exactly
//     run to run.
#include "common.cuh"

namespace harp {
namespace {

constexpr int kTile = 32;
constexpr float kQuarterPiF = 0.78539816339744830962f;
constexpr float kRsqrt2F = 0.70710678118654752440f;
constexpr int kBackThreads = 512;
constexpr int kBackSmem = 128 * 1024;  // R rows x w x (value, gradient) fp32
constexpr int kColChunks = 16;
constexpr int kSumThreads = 256;

// out[c][r] = in[r][c] for an R x C fp32 matrix, through 32 x 33 shared tiles.
__global__ void __launch_bounds__(256) transpose_kernel(const float* __restrict__ in, float* __restrict__ out,
                                                        int64_t R, int64_t C) {
  __shared__ float tile[kTile][kTile + 1];
  const int64_t c0 = (int64_t)blockIdx.x * kTile, r0 = (int64_t)blockIdx.y * kTile;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8 threads
  for (int k = ty; k < kTile; k += 8) {
    const int64_t r = r0 + k, c = c0 + tx;
    if (r < R && c < C) tile[k][tx] = in[r * C + c];
  }
  __syncthreads();
  for (int k = ty; k < kTile; k += 8) {
    const int64_t c = c0 + k, r = r0 + tx;
    if (r < R && c < C) out[c * R + r] = tile[tx][k];
  }
}

// E = W' - (scale16 * q + zero16), the codes read from the canonical packed layout.
__global__ void __launch_bounds__(256) residual_kernel(const float* __restrict__ Wr, const uint32_t* __restrict__ codes,
                                                       const uint32_t* __restrict__ sz, int64_t n_out, int64_t n_in,
                                                       int bits, float* __restrict__ E) {
  const int64_t n = n_out * n_in;
  const int pb = bits == 4 ? 4 : 2;  // bits of the first plane
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t bit = e * pb;
    unsigned q = (codes[bit >> 5] >> (bit & 31)) & ((1u << pb) - 1u);
    if (bits == 3) {
      const uint32_t* hi = codes + (n >> 4);  // the 1-bit plane follows n/4 bytes of 2-bit codes
      q |= ((hi[e >> 5] >> (e & 31)) & 1u) << 2;
    }
    const int64_t r = e / n_in, j = e - r * n_in;
    const uint32_t w = sz[r * (n_in / 64) + j / 64];
    const float s = __half2float(__ushort_as_half((unsigned short)(w & 0xffffu)));
    const float z = __half2float(__ushort_as_half((unsigned short)(w >> 16)));
    E[e] = Wr[e] - fmaf(s, (float)q, z);
  }
}

// d_j = H'_jj (1 without a Hessian proxy).
__global__ void diag_kernel(const float* __restrict__ Hq, int64_t n, float* __restrict__ d) {
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n; j += (int64_t)gridDim.x * blockDim.x)
    d[j] = Hq ? Hq[j * n + j] : 1.f;
}

// Fixed-order CTA reduction of one fp64 value per thread (kSumThreads threads); the
// total is valid in thread 0.
__device__ double cta_sum(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0)
    for (int k = 0; k < kSumThreads / 32; ++k) t += red[k];
  return t;
}

// rowsum[i] = sum of H'_ij^2 over j outside row i's group (one CTA per row).
__global__ void __launch_bounds__(kSumThreads) offgroup_kernel(const float* __restrict__ Hq, int64_t n,
                                                               double* __restrict__ rowsum) {
  __shared__ double red[kSumThreads / 32];
  const int64_t i = blockIdx.x, gi = i / 64;
  double acc = 0.0;
  for (int64_t j = threadIdx.x; j < n; j += kSumThreads)
    if (j / 64 != gi) {
      const double v = Hq[i * n + j];
      acc += v * v;
    }
  const double t = cta_sum(acc, red);
  if (threadIdx.x == 0) rowsum[i] = t;
}

// part[chunk][j] = sum of E_rj^2 over the chunk's rows (32 columns x 8 row lanes per CTA).
__global__ void __launch_bounds__(256) colsq_kernel(const float* __restrict__ E, int64_t n_out, int64_t n_in,
                                                    int64_t rows_per_chunk, double* __restrict__ part) {
  __shared__ double red[8][kTile];
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int64_t j = (int64_t)blockIdx.x * kTile + tx;
  const int64_t r0 = (int64_t)blockIdx.y * rows_per_chunk;
  const int64_t r1 = min(n_out, r0 + rows_per_chunk);
  double acc = 0.0;
  if (j < n_in)
    for (int64_t r = r0 + ty; r < r1; r += 8) {
      const double v = E[r * n_in + j];
      acc += v * v;
    }
  red[ty][tx] = acc;
  __syncthreads();
  if (ty == 0 && j < n_in) {
    double t = 0.0;
    for (int k = 0; k < 8; ++k) t += red[k][tx];
    part[(int64_t)blockIdx.y * n_in + j] = t;
  }
}

// out[i] = sum_c part[c][i] over nch slices of n (fixed order), into fp64.
__global__ void chunk_sum_kernel(const double* __restrict__ part, int nch, int64_t n, double* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    double t = 0.0;
    for (int c = 0; c < nch; ++c) t += part[(int64_t)c * n + i];
    out[i] = t;
  }
}

// *out = sum_i a_i (times b_i when b is set): each thread a contiguous run, then a fixed tree.
__global__ void __launch_bounds__(kSumThreads) dot_kernel(const double* __restrict__ a, const float* __restrict__ b,
                                                          int64_t n, double* __restrict__ out) {
  __shared__ double red[kSumThreads / 32];
  const int64_t per = (n + kSumThreads - 1) / kSumThreads;
  const int64_t i0 = threadIdx.x * per, i1 = min(n, i0 + per);
  double t = 0.0;
  for (int64_t i = i0; i < i1; ++i) t += b ? a[i] * (double)b[i] : a[i];
  const double s = cta_sum(t, red);
  if (threadIdx.x == 0) *out = s;
}

__global__ void finish_loss_kernel(const double* __restrict__ Ld, const double* __restrict__ Rb, double lambda,
                                   double* __restrict__ loss) {
  const double l = *Ld, r = Rb ? *Rb : 0.0;
  loss[0] = l + lambda * r;
  loss[1] = l;
  loss[2] = r;
}

// G' = 2 d_j E_rj, in place.
__global__ void scale_cols_kernel(float* __restrict__ E, const float* __restrict__ d, int64_t n_out, int64_t n_in) {
  const int64_t n = n_out * n_in;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x)
    E[e] *= 2.f * d[e % n_in];
}

// K = dL/dH' = 2 lambda_bd H' on off-group entries, plus diag(e), e_j = sum_r E_rj^2.
__global__ void kmat_kernel(const float* __restrict__ Hq, const double* __restrict__ e, float lam2, int64_t n,
                            float* __restrict__ K) {
  const int64_t nn = n * n;
  for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < nn; x += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = x / n, j = x - i * n;
    float k = i / 64 != j / 64 ? lam2 * Hq[x] : 0.f;
    if (i == j) k += (float)e[i];
    K[x] = k;
  }
}

struct BackParams {
  int64_t n;            // row length
  int w, m, inverse;    // block width, log2 w, 1 when the rows went through F^T
  const float* theta;   // [m][n/2] or null (Theta = 0)
  const int8_t* sign;   // [n]
  float* y;             // [batch][n] outputs, replaced by the inputs
  float* g;             // [batch][n] dL/d outputs, replaced by dL/d inputs
  int64_t batch, rows_per_chunk;
  int R;                // rows held in shared memory at once
  float* part;          // [chunks][m][n/2] this launch's angle-gradient partials (zeroed)
};

// Grid (n / w blocks, chunks of rows). Each CTA owns block `blockIdx.x` of the rows in its
// chunk and the partials part[chunk][.][block's pairs], so no two CTAs write one word.
__global__ void __launch_bounds__(kBackThreads) bfly_back_kernel(BackParams p) {
  extern __shared__ float sm[];
  const int w = p.w, hw = w >> 1, tid = threadIdx.x;
  const int64_t blk = blockIdx.x, half_n = p.n >> 1;
  const int64_t r_begin = (int64_t)blockIdx.y * p.rows_per_chunk;
  const int64_t r_end = min(p.batch, r_begin + p.rows_per_chunk);
  float* ys = sm;
  float* gs = sm + (size_t)p.R * w;
  const int64_t col0 = blk * w;
  const int8_t* sg = p.sign + col0;
  float* part = p.part + (int64_t)blockIdx.y * p.m * half_n + blk * hw;
  for (int64_t r0 = r_begin; r0 < r_end; r0 += p.R) {
    const int rc = (int)min((int64_t)p.R, r_end - r0);
    for (int idx = tid; idx < rc * w; idx += kBackThreads) {
      const int k = idx >> p.m, i = idx & (w - 1);
      const int64_t off = (r0 + k) * p.n + col0 + i;
      float yv = p.y[off], gv = p.g[off];
      if (p.inverse) {  // F^T = D S_0 ... S_{m-1}: D was applied last
        const float sv = (float)sg[i];
        yv *= sv;
        gv *= sv;
      }
      ys[idx] = yv;
      gs[idx] = gv;
    }
    __syncthreads();
    for (int step = 0; step < p.m; ++step) {
      const int t = p.inverse ? step : p.m - 1 - step;
      const int h = 1 << t;
      for (int q = tid; q < hw; q += kBackThreads) {
        const int i = ((q >> t) << (t + 1)) + (q & (h - 1));
        float c, s;
        if (p.theta)
          sincosf(kQuarterPiF + p.theta[(int64_t)t * half_n + blk * hw + q], &s, &c);
        else
          c = s = kRsqrt2F;
        float acc = 0.f;
        for (int k = 0; k < rc; ++k) {
          float* yk = ys + k * w;
          float* gk = gs + k * w;
          const float u = yk[i], v = yk[i + h], gu = gk[i], gv = gk[i + h];
          acc = fmaf(gv, u, fmaf(-gu, v, acc));
          yk[i] = fmaf(c, u, s * v);
          yk[i + h] = fmaf(s, u, -c * v);
          gk[i] = fmaf(c, gu, s * gv);
          gk[i + h] = fmaf(s, gu, -c * gv);
        }
        part[(int64_t)t * half_n + q] += acc;
      }
      __syncthreads();
    }
    for (int idx = tid; idx < rc * w; idx += kBackThreads) {
      const int k = idx >> p.m, i = idx & (w - 1);
      const int64_t off = (r0 + k) * p.n + col0 + i;
      float yv = ys[idx], gv = gs[idx];
      if (!p.inverse) {  // F = S_{m-1} ... S_0 D: D was applied first
        const float sv = (float)sg[i];
        yv *= sv;
        gv *= sv;
      }
      p.y[off] = yv;
      p.g[off] = gv;
    }
    __syncthreads();
  }
}

// acc[i] += sum over chunks of part[c][i] (fixed order), fp64.
__global__ void grad_accum_kernel(const float* __restrict__ part, int nch, int64_t n, double* __restrict__ acc) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    double t = 0.0;
    for (int c = 0; c < nch; ++c) t += (double)part[(int64_t)c * n + i];
    acc[i] += t;
  }
}

__global__ void to_f32_kernel(const double* __restrict__ a, int64_t n, float* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = (float)a[i];
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

int log2_pow2(int64_t w) {
  if (w < 2 || (w & (w - 1))) return -1;
  int m = 0;
  while ((int64_t(1) << m) < w) ++m;
  return m;
}

// Chunks of rows per butterfly block: about one CTA per SM over all blocks.
int back_chunks(int64_t n, int w) {
  const int64_t nb = n / w;
  return (int)std::max<int64_t>(1, (148 + nb - 1) / nb);
}

int back_rows(int w) { return std::max(1, std::min(32, kBackSmem / (8 * w))); }

struct CalibWs {
  float *Wr, *S, *X;
  void* codes;
  void* sz;
  float* d;
  double *e, *colpart, *rowsum, *scal;
  float *Hp, *Hq, *K;
  float* part;
  double *gaccV, *gaccU;
  size_t bytes;
};

CalibWs calib_layout(int64_t n_out, int64_t n_in, int bits, int w_in, int w_out, bool hess, bool grad, void* base) {
  CalibWs w{};
  char* b = static_cast<char*>(base);
  size_t off = 0;
  auto carve = [&](size_t bytes) -> void* {
    const size_t o = off;
    off = align256(off + bytes);
    return b ? b + o : nullptr;
  };
  const size_t nw = (size_t)n_out * (size_t)n_in, nh = (size_t)n_in * (size_t)n_in;
  w.Wr = static_cast<float*>(carve(4 * nw));
  w.S = static_cast<float*>(carve(4 * nw));
  w.X = grad ? static_cast<float*>(carve(4 * nw)) : nullptr;
  w.codes = carve(nw * (size_t)bits / 8);
  w.sz = carve((size_t)n_out * (size_t)(n_in / 64) * 4);
  w.d = static_cast<float*>(carve(4 * (size_t)n_in));
  w.e = static_cast<double*>(carve(8 * (size_t)n_in));
  w.colpart = static_cast<double*>(carve(8 * (size_t)kColChunks * (size_t)n_in));
  w.rowsum = static_cast<double*>(carve(8 * (size_t)n_in));
  w.scal = static_cast<double*>(carve(8 * 4));
  if (hess) {
    w.Hp = static_cast<float*>(carve(4 * nh));
    w.Hq = static_cast<float*>(carve(4 * nh));
    w.K = grad ? static_cast<float*>(carve(4 * nh)) : nullptr;
  }
  if (grad) {
    const int mi = log2_pow2(w_in), mo = log2_pow2(w_out);
    const size_t pv = (size_t)back_chunks(n_in, w_in) * mi * (size_t)(n_in / 2);
    const size_t pu = (size_t)back_chunks(n_out, w_out) * mo * (size_t)(n_out / 2);
    w.part = static_cast<float*>(carve(4 * std::max(pv, pu)));
    w.gaccV = static_cast<double*>(carve(8 * (size_t)mi * (size_t)(n_in / 2)));
    w.gaccU = static_cast<double*>(carve(8 * (size_t)mo * (size_t)(n_out / 2)));
  }
  w.bytes = off;
  return w;
}

harp_status check(int64_t n_out, int64_t n_in, int bits, int group, int w_in, int w_out) {
  if (bits < 2 || bits > 4) return set_error(HARP_ERR_INVALID_ARG, "calib: bits=%d not in {2,3,4}", bits);
  if (group != kGroup) return set_error(HARP_ERR_UNSUPPORTED, "calib: group=%d (only 64 is supported)", group);
  // each side is also the other's butterfly batch, so both stay below 65536
  if (n_in <= 0 || n_in % 256 || n_in > 65535 || n_out <= 0 || n_out > 65535 || n_out % 32)
    return set_error(HARP_ERR_INVALID_ARG, "calib: n_in must be a multiple of 256 and n_out of 32, both < 65536");
  const int mi = log2_pow2(w_in), mo = log2_pow2(w_out);
  if (mi < 1 || w_in > kMaxW || n_in % w_in || mo < 1 || w_out > kMaxW || n_out % w_out)
    return set_error(HARP_ERR_INVALID_ARG, "calib: butterfly widths must be powers of two in [2, 8192] dividing n");
  return HARP_OK;
}

unsigned ew_blocks(int64_t n) { return (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 148 * 16)); }

cudaError_t transpose(const float* in, float* out, int64_t R, int64_t C, cudaStream_t st) {
  const dim3 grid((unsigned)((C + kTile - 1) / kTile), (unsigned)((R + kTile - 1) / kTile));
  transpose_kernel<<<grid, dim3(kTile, 8), 0, st>>>(in, out, R, C);
  return cudaGetLastError();
}

cudaError_t rows(const float* x, float* y, int64_t n, int w, int64_t batch, const float* theta, const int8_t* sign,
                 int inverse, int* status, cudaStream_t st) {
  BflyParams p{};
  p.n = n;
  p.w = w;
  p.m = log2_pow2(w);
  p.inverse = inverse;
  p.theta = theta;  // null: the fixed randomized Hadamard transform
  p.sign = sign;
  p.x = x;
  p.xt = DT_F32;
  p.x_stride = n;
  p.y = y;
  p.yt = DT_F32;
  p.y_stride = n;
  p.status = status;
  return launch_butterfly(p, (int)batch, st);
}

// Backward through `batch` rows of a butterfly, adding dL/dtheta into gacc (fp64).
cudaError_t rows_back(float* y, float* g, int64_t n, int w, int64_t batch, const float* theta, const int8_t* sign,
                      int inverse, float* part, double* gacc, cudaStream_t st) {
  // the opt-in is per device and cheap to repeat, so it is set on every call
  cudaError_t e = cudaFuncSetAttribute(bfly_back_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kBackSmem);
  if (e != cudaSuccess) return e;
  BackParams p{};
  p.n = n;
  p.w = w;
  p.m = log2_pow2(w);
  p.inverse = inverse;
  p.theta = theta;
  p.sign = sign;
  p.y = y;
  p.g = g;
  p.batch = batch;
  const int nch = back_chunks(n, w);
  p.rows_per_chunk = (batch + nch - 1) / nch;
  p.R = back_rows(w);
  p.part = part;
  const int64_t np = (int64_t)p.m * (n / 2);
  e = cudaMemsetAsync(part, 0, sizeof(float) * (size_t)nch * (size_t)np, st);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(float) * 2 * (size_t)p.R * (size_t)w;
  bfly_back_kernel<<<dim3((unsigned)(n / w), (unsigned)nch), kBackThreads, smem, st>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  grad_accum_kernel<<<ew_blocks(np), 256, 0, st>>>(part, nch, np, gacc);
  return cudaGetLastError();
}

}  // namespace
}  // namespace harp

using namespace harp;

extern "C" {

harp_status harp_calib_workspace_size(int64_t n_out, int64_t n_in, int bits, int w_in, int w_out, int with_hessian,
                                      int with_grad, size_t* bytes) {
  if (!bytes) return set_error(HARP_ERR_INVALID_ARG, "calib_workspace_size: null pointer");
  harp_status s = check(n_out, n_in, bits, kGroup, w_in, w_out);
  if (s != HARP_OK) return s;
  *bytes = calib_layout(n_out, n_in, bits, w_in, w_out, with_hessian != 0, with_grad != 0, nullptr).bytes;
  return HARP_OK;
}

harp_status harp_calib_fit(int64_t n_out, int64_t n_in, int bits, int group, int w_in, int w_out, const float* W,
                           const float* theta_V, const int8_t* sign_V, const float* theta_U, const int8_t* sign_U,
                           const float* H, double lambda_bd, double* loss, float* grad_theta_V, float* grad_theta_U,
                           void* workspace, size_t ws_bytes, void* stream) {
  harp_status s = check(n_out, n_in, bits, group, w_in, w_out);
  if (s != HARP_OK) return s;
  if (!W || !sign_V || !sign_U || !loss || !workspace) return set_error(HARP_ERR_INVALID_ARG, "calib: null pointer");
  auto a16 = [](const void* q) { return q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  if (!a16(W) || !a16(sign_V) || !a16(sign_U) || !a16(theta_V) || !a16(theta_U) || !a16(H) || !a16(grad_theta_V) ||
      !a16(grad_theta_U) || (reinterpret_cast<uintptr_t>(loss) & 7u) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return set_error(HARP_ERR_INVALID_ARG, "calib: pointers must be 16-byte aligned (workspace 256, loss 8)");
  if (!(lambda_bd >= 0.0)) return set_error(HARP_ERR_INVALID_ARG, "calib: lambda_bd must be >= 0");
  const bool hess = H != nullptr, grad = grad_theta_V || grad_theta_U;
  const CalibWs w = calib_layout(n_out, n_in, bits, w_in, w_out, hess, grad, workspace);
  if (ws_bytes < w.bytes)
    return set_error(HARP_ERR_WORKSPACE, "calib: workspace of %zu bytes, %zu needed", ws_bytes, w.bytes);
  int* status = nullptr;
  if ((s = device_status_for_kernels(&status)) != HARP_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t nw = n_out * n_in;
  cudaError_t e = cudaSuccess;
  auto ok = [&](cudaError_t r) { return (e = r) == cudaSuccess; };
  auto fail = [&](const char* what) {
    return set_error(HARP_ERR_CUDA, "calib: %s: %s", what, cudaGetErrorString(e));
  };

  // W' = U W V^T (rows through F_V, columns through F_U^T), its codes and E = W' - T
  if (!ok(rows(W, w.Wr, n_in, w_in, n_out, theta_V, sign_V, 0, status, st)) ||
      !ok(transpose(w.Wr, w.S, n_out, n_in, st)) ||
      !ok(rows(w.S, w.S, n_out, w_out, n_in, theta_U, sign_U, 1, status, st)) ||
      !ok(transpose(w.S, w.Wr, n_in, n_out, st)) ||
      !ok(launch_quantize(n_out, n_in, bits, w.Wr, w.codes, w.sz, st)))
    return fail("rotation or quantization");
  residual_kernel<<<ew_blocks(nw), 256, 0, st>>>(w.Wr, static_cast<const uint32_t*>(w.codes),
                                                  static_cast<const uint32_t*>(w.sz), n_out, n_in, bits, w.S);
  if (!ok(cudaGetLastError())) return fail("residual");

  // H' = V H V^T (rows of H through F_V, then rows of the transpose), d and R_bd
  if (hess) {
    if (!ok(rows(H, w.Hp, n_in, w_in, n_in, theta_V, sign_V, 0, status, st)) ||
        !ok(transpose(w.Hp, w.Hq, n_in, n_in, st)) ||
        !ok(rows(w.Hq, w.Hq, n_in, w_in, n_in, theta_V, sign_V, 0, status, st)))
      return fail("Hessian rotation");
    offgroup_kernel<<<(unsigned)n_in, kSumThreads, 0, st>>>(w.Hq, n_in, w.rowsum);
    dot_kernel<<<1, kSumThreads, 0, st>>>(w.rowsum, nullptr, n_in, w.scal + 1);
  }
  diag_kernel<<<ew_blocks(n_in), 256, 0, st>>>(hess ? w.Hq : nullptr, n_in, w.d);

  // e_j = sum_r E_rj^2, L_diag = sum_j d_j e_j, the loss
  const int64_t rpc = (n_out + kColChunks - 1) / kColChunks;
  colsq_kernel<<<dim3((unsigned)((n_in + kTile - 1) / kTile), kColChunks), dim3(kTile, 8), 0, st>>>(w.S, n_out, n_in,
                                                                                                 rpc, w.colpart);
  chunk_sum_kernel<<<ew_blocks(n_in), 256, 0, st>>>(w.colpart, kColChunks, n_in, w.e);
  dot_kernel<<<1, kSumThreads, 0, st>>>(w.e, w.d, n_in, w.scal);
  finish_loss_kernel<<<1, 1, 0, st>>>(w.scal, hess ? w.scal + 1 : nullptr, lambda_bd, loss);
  if (!ok(cudaGetLastError())) return fail("loss reduction");
  if (!grad) return HARP_OK;

  const int mi = log2_pow2(w_in), mo = log2_pow2(w_out);
  const int64_t nV = (int64_t)mi * (n_in / 2), nU = (int64_t)mo * (n_out / 2);
  if (!ok(cudaMemsetAsync(w.gaccV, 0, sizeof(double) * (size_t)nV, st)) ||
      !ok(cudaMemsetAsync(w.gaccU, 0, sizeof(double) * (size_t)nU, st)))
    return fail("gradient accumulators");
  // dL/dW' = 2 d_j E_rj; back through the columns (F_U^T) with W' and G' transposed
  scale_cols_kernel<<<ew_blocks(nw), 256, 0, st>>>(w.S, w.d, n_out, n_in);
  if (!ok(cudaGetLastError()) || !ok(transpose(w.Wr, w.X, n_out, n_in, st)) ||
      !ok(transpose(w.S, w.Wr, n_out, n_in, st)) ||
      !ok(rows_back(w.X, w.Wr, n_out, w_out, n_in, theta_U, sign_U, 1, w.part, w.gaccU, st)) ||
      // then back through the rows (F_V), their outputs recomputed from W
      !ok(transpose(w.Wr, w.S, n_in, n_out, st)) ||
      !ok(rows(W, w.X, n_in, w_in, n_out, theta_V, sign_V, 0, status, st)) ||
      !ok(rows_back(w.X, w.S, n_in, w_in, n_out, theta_V, sign_V, 0, w.part, w.gaccV, st)))
    return fail("weight-side backward");
  if (hess) {
    // dL/dH' = 2 lambda_bd H' off the groups + diag(e); back through both passes of V
    kmat_kernel<<<ew_blocks(n_in * n_in), 256, 0, st>>>(w.Hq, w.e, (float)(2.0 * lambda_bd), n_in, w.K);
    if (!ok(cudaGetLastError()) ||
        !ok(rows_back(w.Hq, w.K, n_in, w_in, n_in, theta_V, sign_V, 0, w.part, w.gaccV, st)) ||
        !ok(transpose(w.Hq, w.Hp, n_in, n_in, st)) || !ok(transpose(w.K, w.Hq, n_in, n_in, st)) ||
        !ok(rows_back(w.Hp, w.Hq, n_in, w_in, n_in, theta_V, sign_V, 0, w.part, w.gaccV, st)))
      return fail("Hessian-side backward");
  }
  if (grad_theta_V) to_f32_kernel<<<ew_blocks(nV), 256, 0, st>>>(w.gaccV, nV, grad_theta_V);
  if (grad_theta_U) to_f32_kernel<<<ew_blocks(nU), 256, 0, st>>>(w.gaccU, nU, grad_theta_U);
  if (!ok(cudaGetLastError())) return fail("gradient output");
  return HARP_OK;
}

}  // extern "C"
