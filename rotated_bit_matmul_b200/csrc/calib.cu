// Calibration-time forward of the rotated low-bit linear: the weighted reconstruction
// error that adapting the angles reduces ("HARP: Hadamard-Preconditioned Adaptive
// Rotation Processor for Extreme LLM Quantization", Sec. 2.2 and 3: each layer's rotation
// is adapted to its quantizer).
//
//   W' = U W V^T,   W^ = U^T deq(Q(W')) V,   L = sum_{r,j} h_j (W_rj - W^_rj)^2
//
// Everything runs on the device with the inference kernels:
//   - the butterflies rotate rows;
//   - a tiled transpose turns columns into rows;
//   - the quantizer is the codes' own;
//   - a dequantize kernel reads the canonical packed layout;
//   - a two-pass reduction forms the sum in fp64, in a fixed order.
#include "common.cuh"

namespace harp {
namespace {

constexpr int kTile = 32;

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

// W^'_rj = scale16 * q + zero16 from the canonical packed codes (one element per thread).
__global__ void __launch_bounds__(256) dequant_kernel(const uint32_t* __restrict__ codes, const uint32_t* __restrict__ sz,
                                                      int64_t n_out, int64_t n_in, int bits, float* __restrict__ out) {
  const int64_t n = n_out * n_in;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int pb = bits == 4 ? 4 : 2;  // bits of the (first) plane
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
    out[e] = fmaf(s, (float)q, z);
  }
}

// rowsum[r] = sum_j h_j (W_rj - A_rj)^2 in fp64 (one CTA per row, fixed reduction tree).
__global__ void __launch_bounds__(256) row_error_kernel(const float* __restrict__ W, const float* __restrict__ A,
                                                        const float* __restrict__ h, int64_t n_in,
                                                        double* __restrict__ rowsum) {
  __shared__ double red[8];
  const int64_t r = blockIdx.x;
  const int tid = threadIdx.x;
  double acc = 0.0;
  for (int64_t j = tid; j < n_in; j += 256) {
    const double d = (double)W[r * n_in + j] - (double)A[r * n_in + j];
    acc += (h ? (double)h[j] : 1.0) * d * d;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((tid & 31) == 0) red[tid >> 5] = acc;
  __syncthreads();
  if (tid == 0) {
    double t = 0.0;
    for (int w = 0; w < 8; ++w) t += red[w];
    rowsum[r] = t;
  }
}

// out = sum_r rowsum[r]: each thread a contiguous run, then a fixed tree.
__global__ void __launch_bounds__(256) total_kernel(const double* __restrict__ rowsum, int64_t n, double* out) {
  __shared__ double red[256];
  const int tid = threadIdx.x;
  const int64_t per = (n + 255) / 256;
  double t = 0.0;
  for (int64_t i = tid * per; i < (tid + 1) * per && i < n; ++i) t += rowsum[i];
  red[tid] = t;
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if (tid < s) red[tid] += red[tid + s];
    __syncthreads();
  }
  if (tid == 0) *out = red[0];
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct CalibWs {
  float* A;
  float* B;
  void* codes;
  void* sz;
  double* rowsum;
  size_t bytes;
};

CalibWs calib_layout(int64_t n_out, int64_t n_in, int bits, void* base) {
  CalibWs w{};
  char* b = static_cast<char*>(base);
  size_t off = 0;
  auto carve = [&](size_t bytes) -> void* {
    const size_t o = off;
    off = align256(off + bytes);
    return b ? b + o : nullptr;
  };
  const size_t nw = (size_t)n_out * (size_t)n_in;
  w.A = static_cast<float*>(carve(4 * nw));
  w.B = static_cast<float*>(carve(4 * nw));
  w.codes = carve(nw * (size_t)bits / 8);
  w.sz = carve((size_t)n_out * (size_t)(n_in / 64) * 4);
  w.rowsum = static_cast<double*>(carve(8 * (size_t)n_out));
  w.bytes = off;
  return w;
}

int log2_pow2(int64_t w) {
  if (w < 2 || (w & (w - 1))) return -1;
  int m = 0;
  while ((int64_t(1) << m) < w) ++m;
  return m;
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

cudaError_t transpose(const float* in, float* out, int64_t R, int64_t C, cudaStream_t st) {
  const dim3 grid((unsigned)((C + kTile - 1) / kTile), (unsigned)((R + kTile - 1) / kTile));
  transpose_kernel<<<grid, dim3(kTile, 8), 0, st>>>(in, out, R, C);
  return cudaGetLastError();
}

cudaError_t rows(const float* x, float* y, int64_t n, int w, int batch, const float* theta, const int8_t* sign,
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
  return launch_butterfly(p, batch, st);
}

}  // namespace
}  // namespace harp

using namespace harp;

extern "C" {

harp_status harp_calib_workspace_size(int64_t n_out, int64_t n_in, int bits, size_t* bytes) {
  if (!bytes) return set_error(HARP_ERR_INVALID_ARG, "calib_workspace_size: null pointer");
  harp_status s = check(n_out, n_in, bits, kGroup, 2, 2);
  if (s != HARP_OK) return s;
  *bytes = calib_layout(n_out, n_in, bits, nullptr).bytes;
  return HARP_OK;
}

harp_status harp_calib_error(int64_t n_out, int64_t n_in, int bits, int group, int w_in, int w_out, const float* W,
                             const float* theta_V, const int8_t* sign_V, const float* theta_U,
                             const int8_t* sign_U, const float* h, double* err, void* workspace, size_t ws_bytes,
                             void* stream) {
  harp_status s = check(n_out, n_in, bits, group, w_in, w_out);
  if (s != HARP_OK) return s;
  if (!W || !sign_V || !sign_U || !err || !workspace) return set_error(HARP_ERR_INVALID_ARG, "calib: null pointer");
  auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  if (!a16(W) || !a16(sign_V) || !a16(sign_U) || (theta_V && !a16(theta_V)) || (theta_U && !a16(theta_U)) ||
      (h && !a16(h)) || (reinterpret_cast<uintptr_t>(err) & 7u) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return set_error(HARP_ERR_INVALID_ARG, "calib: pointers must be 16-byte aligned (workspace 256, err 8)");
  const CalibWs w = calib_layout(n_out, n_in, bits, workspace);
  if (ws_bytes < w.bytes)
    return set_error(HARP_ERR_WORKSPACE, "calib: workspace of %zu bytes, %zu needed", ws_bytes, w.bytes);
  int* status = nullptr;
  if ((s = device_status_for_kernels(&status)) != HARP_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t nw = n_out * n_in;
  const unsigned eblocks = (unsigned)std::min<int64_t>((nw + 255) / 256, 148 * 16);
  cudaError_t e = cudaSuccess;
  auto ok = [&](cudaError_t r) { return (e = r) == cudaSuccess; };
  // W' = U W V^T: rows through F_V, columns through F_U^T
  if (!ok(rows(W, w.A, n_in, w_in, (int)n_out, theta_V, sign_V, 0, status, st)) ||
      !ok(transpose(w.A, w.B, n_out, n_in, st)) ||
      !ok(rows(w.B, w.B, n_out, w_out, (int)n_in, theta_U, sign_U, 1, status, st)) ||
      !ok(transpose(w.B, w.A, n_in, n_out, st)) ||
      // codes and their dequantized values
      !ok(launch_quantize(n_out, n_in, bits, w.A, w.codes, w.sz, st)))
    return set_error(HARP_ERR_CUDA, "calib: rotation or quantization launch: %s", cudaGetErrorString(e));
  dequant_kernel<<<eblocks, 256, 0, st>>>(static_cast<const uint32_t*>(w.codes), static_cast<const uint32_t*>(w.sz),
                                          n_out, n_in, bits, w.A);
  // W^ = U^T W^' V: columns through F_U, rows through F_V^T
  if (!ok(cudaGetLastError()) || !ok(transpose(w.A, w.B, n_out, n_in, st)) ||
      !ok(rows(w.B, w.B, n_out, w_out, (int)n_in, theta_U, sign_U, 0, status, st)) ||
      !ok(transpose(w.B, w.A, n_in, n_out, st)) ||
      !ok(rows(w.A, w.A, n_in, w_in, (int)n_out, theta_V, sign_V, 1, status, st)))
    return set_error(HARP_ERR_CUDA, "calib: dequantize or back-rotation launch: %s", cudaGetErrorString(e));
  row_error_kernel<<<(unsigned)n_out, 256, 0, st>>>(W, w.A, h, n_in, w.rowsum);
  total_kernel<<<1, 256, 0, st>>>(w.rowsum, n_out, err);
  if (!ok(cudaGetLastError())) return set_error(HARP_ERR_CUDA, "calib: error reduction launch: %s", cudaGetErrorString(e));
  return HARP_OK;
}

}  // extern "C"
