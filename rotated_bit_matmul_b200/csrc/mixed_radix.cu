// Mixed-radix butterfly schedules on sm_100a ("HARP: Hadamard-Preconditioned Adaptive
// Rotation Processor for Extreme LLM Quantization", Sec. 2.1, Suporte a Misto-Raiz, and
// Sec. 2.2): for d = b_0 b_1 ... b_{m-1}, stage t mixes the b_t coordinates that differ
// only in mixed-radix digit t (stride s_t = b_0 ... b_{t-1}) with a block
// B_{t,c} = Q_{t,c}(theta) G_{b_t}:
//   b = 2: the Givens block [[cos p, sin p], [sin p, -cos p]], p = pi/4 + theta;
//   b > 2: Q = (I - A)(I + A)^-1 (Cayley) of the skew-symmetric A holding the b(b-1)/2
//          parameters of the group (strict upper triangle, row by row), and G_b the
//          normalised Sylvester Hadamard for powers of two, else the orthogonal factor of a
//          fixed Gaussian matrix with R's diagonal made positive.
// Group c of stage t starts at base_c = (c mod s_t) + (c div s_t) s_t b_t.
//
// A plan builds every stage's blocks once (fp64 arithmetic, stored fp32):
//   mixer_kernel   one thread per stage: Sylvester entries, or modified Gram-Schmidt run
//                  twice over the Gaussian's columns;
//   blocks_kernel  one thread per group: the Cayley map by Gauss-Jordan elimination with
//                  partial pivoting, then B = Q G.
// The transform keeps a whole row (d <= 16384) in shared memory. A stage computes every
// output i of group c as sum_j B_{t,c}[i][j] v[base_c + j s_t] (B^T for the transpose)
// into a second buffer, and the two buffers swap after each stage.
#include <algorithm>
#include <new>

#include "common.cuh"

namespace harp {
namespace {

constexpr int kMrMaxStages = 32;
constexpr int kMrMaxRadix = 64;
constexpr int64_t kMrMaxD = 16384;
constexpr int kMrThreads = 512;

struct MrParams {
  int64_t d;
  int m, inverse;
  int radix[kMrMaxStages];
  int64_t stride[kMrMaxStages];
  int64_t block_off[kMrMaxStages];  // floats before stage t's blocks [d / b_t][b_t][b_t]
  const float* blocks;
  const int8_t* sign;
  const void* x;
  int xt;
  void* y;
  int yt;
};

__global__ void __launch_bounds__(kMrThreads) mr_kernel(MrParams p) {
  extern __shared__ __align__(16) float mr_sm[];
  const int64_t d = p.d, row = blockIdx.x;
  float* a = mr_sm;
  float* b2 = mr_sm + d;
  for (int64_t i = threadIdx.x; i < d; i += blockDim.x) {
    const float v = load_act(p.x, row * d + i, p.xt);
    a[i] = p.inverse ? v : v * (float)p.sign[i];
  }
  __syncthreads();
  for (int step = 0; step < p.m; ++step) {
    const int t = p.inverse ? p.m - 1 - step : step;
    const int b = p.radix[t];
    const int64_t st = p.stride[t];
    const float* B = p.blocks + p.block_off[t];
    for (int64_t o = threadIdx.x; o < d; o += blockDim.x) {
      const int64_t digit = (o / st) % b, base = o - digit * st;
      const int64_t c = (base % st) + (base / (st * b)) * st;
      const float* Bc = B + c * b * b;
      float acc = 0.f;
      if (p.inverse)
        for (int j = 0; j < b; ++j) acc = fmaf(Bc[(int64_t)j * b + digit], a[base + j * st], acc);
      else
        for (int j = 0; j < b; ++j) acc = fmaf(Bc[digit * b + j], a[base + j * st], acc);
      b2[o] = acc;
    }
    __syncthreads();
    float* tmp = a;
    a = b2;
    b2 = tmp;
  }
  for (int64_t i = threadIdx.x; i < d; i += blockDim.x)
    store_act(p.y, row * d + i, p.yt, p.inverse ? a[i] * (float)p.sign[i] : a[i]);
}

// G_b [b][b] in fp64: Sylvester H_b / sqrt(b), or the Q factor of M by modified
// Gram-Schmidt on its columns (each column orthogonalised twice); q is b doubles of scratch.
__global__ void mixer_kernel(int b, const float* M, double* G, double* q, int* bad) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  if ((b & (b - 1)) == 0) {
    const double sc = 1.0 / sqrt((double)b);
    for (int i = 0; i < b; ++i)
      for (int j = 0; j < b; ++j) G[i * b + j] = (__popc((unsigned)(i & j)) & 1) ? -sc : sc;
    return;
  }
  for (int j = 0; j < b; ++j) {
    for (int i = 0; i < b; ++i) q[i] = (double)M[i * b + j];
    for (int pass = 0; pass < 2; ++pass)
      for (int k = 0; k < j; ++k) {
        double dot = 0.0;
        for (int i = 0; i < b; ++i) dot += G[i * b + k] * q[i];
        for (int i = 0; i < b; ++i) q[i] -= dot * G[i * b + k];
      }
    double nrm = 0.0;
    for (int i = 0; i < b; ++i) nrm += q[i] * q[i];
    nrm = sqrt(nrm);
    if (!(nrm > 0.0)) {
      *bad = 1;
      return;
    }
    for (int i = 0; i < b; ++i) G[i * b + j] = q[i] / nrm;
  }
}

// One thread per group c of a stage: B_c = Q(theta_c) G, stored fp32 row-major.
// scratch: 3 b x b doubles per group (I + A reduced in place, its inverse, A).
__global__ void blocks_kernel(int b, int64_t groups, const float* theta, const double* G, double* scratch,
                              float* Bout) {
  const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= groups) return;
  float* B = Bout + c * b * b;
  if (b == 2) {
    double s, co;
    sincos(0.78539816339744830962 + (double)theta[c], &s, &co);
    B[0] = (float)co;
    B[1] = (float)s;
    B[2] = (float)s;
    B[3] = (float)-co;
    return;
  }
  const int64_t bb = (int64_t)b * b;
  double* P = scratch + c * 3 * bb;
  double* X = P + bb;
  double* A = X + bb;
  const float* th = theta + c * (int64_t)(b * (b - 1) / 2);
  for (int64_t e = 0; e < bb; ++e) A[e] = 0.0;
  int k = 0;
  for (int i = 0; i < b; ++i)
    for (int j = i + 1; j < b; ++j, ++k) {
      A[i * b + j] = (double)th[k];
      A[j * b + i] = -(double)th[k];
    }
  for (int i = 0; i < b; ++i)
    for (int j = 0; j < b; ++j) {
      P[i * b + j] = (i == j ? 1.0 : 0.0) + A[i * b + j];
      X[i * b + j] = i == j ? 1.0 : 0.0;
    }
  for (int col = 0; col < b; ++col) {
    int piv = col;
    for (int r = col + 1; r < b; ++r)
      if (fabs(P[r * b + col]) > fabs(P[piv * b + col])) piv = r;
    if (piv != col)
      for (int j = 0; j < b; ++j) {
        double tv = P[col * b + j];
        P[col * b + j] = P[piv * b + j];
        P[piv * b + j] = tv;
        tv = X[col * b + j];
        X[col * b + j] = X[piv * b + j];
        X[piv * b + j] = tv;
      }
    const double dv = P[col * b + col];
    for (int j = 0; j < b; ++j) {
      P[col * b + j] /= dv;
      X[col * b + j] /= dv;
    }
    for (int r = 0; r < b; ++r) {
      if (r == col) continue;
      const double f = P[r * b + col];
      if (f == 0.0) continue;
      for (int j = 0; j < b; ++j) {
        P[r * b + j] -= f * P[col * b + j];
        X[r * b + j] -= f * X[col * b + j];
      }
    }
  }
  // Q = (I - A) X, then B = Q G (Q kept row by row in P, which is free now)
  for (int i = 0; i < b; ++i) {
    for (int j = 0; j < b; ++j) {
      double acc = 0.0;
      for (int l = 0; l < b; ++l) acc += ((i == l ? 1.0 : 0.0) - A[i * b + l]) * X[l * b + j];
      P[j] = acc;
    }
    for (int j = 0; j < b; ++j) {
      double acc = 0.0;
      for (int l = 0; l < b; ++l) acc += P[l] * G[l * b + j];
      B[i * b + j] = (float)acc;
    }
  }
}

int mr_params_of(int b) { return b == 2 ? 1 : b * (b - 1) / 2; }

}  // namespace
}  // namespace harp

using namespace harp;

struct harp_mr_plan_s {
  MrParams p{};
  float* blocks = nullptr;
  int8_t* sign = nullptr;
  int device = 0;
};

extern "C" {

harp_status harp_mr_plan_create(harp_mr_plan* out, int64_t d, int m, const int* radix, const float* theta,
                                const int8_t* sign, const float* gauss, void* stream) {
  if (!out) return set_error(HARP_ERR_INVALID_ARG, "mr_plan_create: null output handle");
  *out = nullptr;
  if (!radix || !theta || !sign) return set_error(HARP_ERR_INVALID_ARG, "mr_plan_create: null pointer");
  if (m < 1 || m > kMrMaxStages) return set_error(HARP_ERR_INVALID_ARG, "mr_plan_create: m=%d not in [1, 32]", m);
  if (d < 2 || d > kMrMaxD) return set_error(HARP_ERR_INVALID_ARG, "mr_plan_create: d=%lld not in [2, 16384]", (long long)d);
  int64_t prod = 1;
  bool any_odd = false;
  for (int t = 0; t < m; ++t) {
    if (radix[t] < 2 || radix[t] > kMrMaxRadix)
      return set_error(HARP_ERR_INVALID_ARG, "mr_plan_create: radix %d not in [2, 64]", radix[t]);
    prod *= radix[t];
    if (prod > kMrMaxD) break;
    any_odd |= (radix[t] & (radix[t] - 1)) != 0;
  }
  if (prod != d) return set_error(HARP_ERR_INVALID_ARG, "mr_plan_create: the radices do not multiply to d");
  if (any_odd && !gauss)
    return set_error(HARP_ERR_INVALID_ARG, "mr_plan_create: a radix that is not a power of two needs its Gaussian");
  auto al = [](const void* q) { return q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  if (!al(theta) || !al(sign) || !al(gauss))
    return set_error(HARP_ERR_INVALID_ARG, "mr_plan_create: device pointers must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  harp_mr_plan_s* h = new (std::nothrow) harp_mr_plan_s();
  if (!h) return set_error(HARP_ERR_INVALID_ARG, "mr_plan_create: out of host memory");
  cudaGetDevice(&h->device);
  MrParams& p = h->p;
  p.d = d;
  p.m = m;
  int64_t total = 0, s_t = 1, scratch = 0;
  for (int t = 0; t < m; ++t) {
    p.radix[t] = radix[t];
    p.stride[t] = s_t;
    p.block_off[t] = total;
    total += d * radix[t];  // (d / b) groups of b x b
    s_t *= radix[t];
    scratch = std::max<int64_t>(scratch, (d / radix[t]) * 3 * (int64_t)radix[t] * radix[t]);
  }
  double* G = nullptr;
  double* work = nullptr;
  int* bad = nullptr;
  auto done = [&](harp_status s) {
    cudaFree(G);
    cudaFree(work);
    cudaFree(bad);
    if (s != HARP_OK) {
      cudaFree(h->blocks);
      cudaFree(h->sign);
      delete h;
    }
    return s;
  };
  cudaError_t e;
  if ((e = cudaMalloc(&h->blocks, sizeof(float) * (size_t)total)) != cudaSuccess ||
      (e = cudaMalloc(&h->sign, (size_t)d)) != cudaSuccess ||
      (e = cudaMalloc(&G, sizeof(double) * kMrMaxRadix * (kMrMaxRadix + 1))) != cudaSuccess ||
      (e = cudaMalloc(&work, sizeof(double) * (size_t)std::max<int64_t>(scratch, 1))) != cudaSuccess ||
      (e = cudaMalloc(&bad, sizeof(int))) != cudaSuccess)
    return done(set_error(HARP_ERR_CUDA, "mr_plan_create: cudaMalloc: %s", cudaGetErrorString(e)));
  if ((e = cudaMemsetAsync(bad, 0, sizeof(int), st)) != cudaSuccess ||
      (e = cudaMemcpyAsync(h->sign, sign, (size_t)d, cudaMemcpyDeviceToDevice, st)) != cudaSuccess)
    return done(set_error(HARP_ERR_CUDA, "mr_plan_create: copies: %s", cudaGetErrorString(e)));
  int64_t toff = 0, goff = 0;
  for (int t = 0; t < m; ++t) {
    const int b = radix[t];
    const int64_t groups = d / b;
    if (b > 2) mixer_kernel<<<1, 32, 0, st>>>(b, gauss ? gauss + goff : nullptr, G, G + kMrMaxRadix * kMrMaxRadix, bad);
    blocks_kernel<<<(unsigned)((groups + 127) / 128), 128, 0, st>>>(b, groups, theta + toff, G, work,
                                                                    h->blocks + p.block_off[t]);
    if ((e = cudaGetLastError()) != cudaSuccess)
      return done(set_error(HARP_ERR_CUDA, "mr_plan_create: block set-up launch: %s", cudaGetErrorString(e)));
    toff += groups * mr_params_of(b);
    goff += (int64_t)b * b;
  }
  int hbad = 0;
  if ((e = cudaMemcpyAsync(&hbad, bad, sizeof(int), cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
      (e = cudaStreamSynchronize(st)) != cudaSuccess)
    return done(set_error(HARP_ERR_CUDA, "mr_plan_create: block set-up: %s", cudaGetErrorString(e)));
  if (hbad) return done(set_error(HARP_ERR_INVALID_ARG, "mr_plan_create: a Gaussian mixer matrix is singular"));
  p.blocks = h->blocks;
  p.sign = h->sign;
  *out = h;
  return done(HARP_OK);
}

harp_status harp_mr_plan_destroy(harp_mr_plan plan) {
  if (!plan) return HARP_OK;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(plan->device);
  cudaDeviceSynchronize();
  cudaFree(plan->blocks);
  cudaFree(plan->sign);
  cudaSetDevice(prev);
  delete plan;
  return HARP_OK;
}

}  // extern "C"

namespace harp {

cudaError_t launch_mr(const harp_mr_plan_s* plan, int inverse, int batch, const void* x, int xt, void* y, int yt,
                      cudaStream_t st) {
  if (batch <= 0) return cudaSuccess;
  MrParams p = plan->p;
  p.inverse = inverse;
  p.x = x;
  p.xt = xt;
  p.y = y;
  p.yt = yt;
  const size_t smem = sizeof(float) * 2 * (size_t)p.d;
  cudaError_t e = cudaFuncSetAttribute(mr_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  mr_kernel<<<(unsigned)batch, kMrThreads, smem, st>>>(p);
  return cudaGetLastError();
}

int64_t mr_plan_d(const harp_mr_plan_s* plan) { return plan->p.d; }
int mr_plan_device(const harp_mr_plan_s* plan) { return plan->device; }

}  // namespace harp

extern "C" {

static harp_status mr_apply(harp_mr_plan plan, int batch, const void* x, harp_dtype xt, void* y, harp_dtype yt,
                            void* stream, int inverse) {
  if (!plan || !x || !y) return set_error(HARP_ERR_INVALID_ARG, "mr_butterfly: null pointer");
  if (batch < 0) return set_error(HARP_ERR_INVALID_ARG, "mr_butterfly: batch=%d out of range", batch);
  if (xt < HARP_F32 || xt > HARP_F16 || yt < HARP_F32 || yt > HARP_F16)
    return set_error(HARP_ERR_INVALID_ARG, "mr_butterfly: unknown dtype");
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(y) & 15u))
    return set_error(HARP_ERR_INVALID_ARG, "mr_butterfly: device pointers must be 16-byte aligned");
  if (x == y && xt != yt) return set_error(HARP_ERR_INVALID_ARG, "mr_butterfly: in-place needs equal dtypes");
  if (batch == 0) return HARP_OK;
  const cudaError_t e = launch_mr(plan, inverse, batch, x, xt, y, yt, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return set_error(HARP_ERR_CUDA, "mr_butterfly launch: %s", cudaGetErrorString(e));
  return HARP_OK;
}

harp_status harp_mr_butterfly_fwd(harp_mr_plan plan, int batch, const void* x, harp_dtype xt, void* y, harp_dtype yt,
                                  void* stream) {
  return mr_apply(plan, batch, x, xt, y, yt, stream, 0);
}

harp_status harp_mr_butterfly_inv(harp_mr_plan plan, int batch, const void* x, harp_dtype xt, void* y, harp_dtype yt,
                                  void* stream) {
  return mr_apply(plan, batch, x, xt, y, yt, stream, 1);
}

}  // extern "C"
