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
// A plan whose radices are all 2 (64 <= d <= 8192) is the radix-2 butterfly of width d: it
// runs on the butterfly kernels, with a (cos, sin) table taken from its blocks.
// Otherwise, for many rows the transform keeps a whole row (d <= 16384) in shared memory,
// one CTA per row. A stage computes every output i of group c as
// sum_j B_{t,c}[i][j] v[base_c + j s_t] (B^T for the transpose) into a second buffer, and
// the two buffers swap after each stage.
// For a few rows (one CTA per row would leave the GPU idle) the stages are cut into runs of
// consecutive stages whose radices multiply to at most 256: within a run the row falls into
// d / (b_t0 ... b_t1-1) independent sub-problems (the indices that share every digit outside
// the run), and one launch per run spreads them over many CTAs, each keeping a few
// sub-problems and all the blocks the run applies to them in shared memory; fp32 results
// pass between runs through global memory.
#include <algorithm>
#include <cstdlib>
#include <new>

#include "common.cuh"

namespace harp {
namespace {

constexpr int kMrMaxStages = 32;
constexpr int kMrMaxRadix = 64;
constexpr int64_t kMrMaxD = 16384;
constexpr int kMrThreads = 512;
// Below kMrSegRows rows the transform runs run by run: runs of at most kMrSegRun
// coordinates, at most kMrSegElems coordinates and kMrSegSmem bytes of shared memory per CTA.
constexpr int kMrSegRows = 8;
constexpr int kMrSegRun = 256;
constexpr int kMrSegElems = 1024;
constexpr int kMrSegSmem = 96 * 1024;
constexpr int kMrSegThreads = 512;
static_assert(kMrSegRun <= 256, "a run holds at most 8 stages");

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

struct SegParams {
  MrParams mp;
  int t0, t1;       // the run: stages t0 .. t1-1
  int K;            // sub-problems per CTA
  int first, last;  // reads x (and applies the forward signs) / writes y (and the transpose's signs)
  int s0, br;       // stride of the run's first digit, product of the run's radices
  int sumb;         // sum of the run's radices
  const float* src; // fp32 input of a run that is not the first
  float* dst;       // fp32 output of a run that is not the last
};

// Integer quotient a / d for 0 <= a < 2^20 and d >= 1 from d's fp32 reciprocal: the
// product is within 0.25 of a / d, so the truncated estimate is off by at most one, and
// the remainder's sign and size correct it. (Every index here is below 2^17.)
struct Div {
  int d;
  float r;
};
__device__ __forceinline__ Div mkdiv(int d) { return Div{d, 1.0f / (float)d}; }
__device__ __forceinline__ int qdiv(int a, Div v) {
  int q = __float2int_rz(__int2float_rn(a) * v.r);
  const int r = a - q * v.d;
  q += (r >= v.d) - (r < 0);
  return q;
}

// One run of stages over K sub-problems per CTA (blockIdx.x: row, then sub-problem block).
// Shared memory: the sub-problems' coordinates twice (the stage buffers), every block the
// run applies to them, gathered before the first stage so that their loads overlap (stage
// t's block of sub-problem qi, group gl, at off_t + (qi (br / b_t) + gl) b_t^2), and the
// global group number of each of those blocks (at goff_t + qi (br / b_t) + gl).
__global__ void __launch_bounds__(kMrSegThreads) mr_seg_kernel(SegParams sp) {
  extern __shared__ __align__(16) float mr_sm[];
  const MrParams& p = sp.mp;
  const int d = (int)p.d, s0 = sp.s0, br = sp.br, nsub = d / br;
  const int nblk = (nsub + sp.K - 1) / sp.K;
  const int64_t row = blockIdx.x / nblk;
  const int q0 = (int)(blockIdx.x % nblk) * sp.K;
  const int K = nsub - q0 < sp.K ? nsub - q0 : sp.K;
  const int n = K * br;
  const Div dbr = mkdiv(br), dK = mkdiv(K), ds0 = mkdiv(s0);
  float* a = mr_sm;
  float* b2 = mr_sm + n;
  float* bs = mr_sm + 2 * n;
  int* gidx = reinterpret_cast<int*>(bs + n * sp.sumb);
  // element lam of sub-problem q: the lower digits q mod s0, the run's digits lam, the
  // higher digits q div s0
  auto goff = [&](int qi, int lam) {
    const int q = q0 + qi, hi = qdiv(q, ds0);
    return (q - hi * s0) + s0 * lam + hi * s0 * br;
  };
  // load and store order: along the row when the run starts at stride 1, else across the
  // sub-problems (neighbouring lower digits sit next to each other)
  auto split = [&](int o, int& qi, int& lam) {
    if (s0 == 1) {
      qi = qdiv(o, dbr);
      lam = o - qi * br;
    } else {
      lam = qdiv(o, dK);
      qi = o - lam * K;
    }
  };
  // the run's stage parameters (at most 8 stages: a run holds at most 256 coordinates):
  // radix, global and local stride, offsets of the stage's blocks and group numbers
  __shared__ int s_b[8], s_st[8], s_ls[8], s_off[8], s_go[8];
  __shared__ const float* s_blk[8];
  const int ns = sp.t1 - sp.t0;
  if (threadIdx.x == 0) {
    int off = 0, go = 0;
    for (int i = 0; i < ns; ++i) {
      const int t = sp.t0 + i, b = p.radix[t];
      s_b[i] = b;
      s_st[i] = (int)p.stride[t];
      s_ls[i] = (int)p.stride[t] / s0;
      s_off[i] = off;
      s_go[i] = go;
      s_blk[i] = p.blocks + p.block_off[t];
      off += n * b;
      go += n / b;
    }
  }
  __syncthreads();
  // group numbers: group gl of stage i in sub-problem qi starts at local coordinate
  // (gl mod ls) + (gl div ls) ls b; the global group of coordinate gb at stride st is
  // (gb mod st) + (gb div (st b)) st
  for (int i = 0; i < ns; ++i) {
    const int b = s_b[i], st = s_st[i], ls = s_ls[i], ng = br / b, go = s_go[i];
    const Div dng = mkdiv(ng), dls = mkdiv(ls), dst = mkdiv(st), db = mkdiv(b);
    for (int gq = threadIdx.x; gq < n / b; gq += blockDim.x) {  // gq = qi (br / b) + gl
      const int qi = qdiv(gq, dng), gl = gq - qi * ng;
      const int gb = goff(qi, gl + qdiv(gl, dls) * ls * (b - 1));
      const int u = qdiv(gb, dst), w = qdiv(u, db);
      gidx[go + gq] = (gb - u * st) + w * st;
    }
  }
  // the x (or previous run's) values: at most kX per thread, loaded into registers first so
  // that their latency overlaps the gather's
  constexpr int kX = kMrSegElems / kMrSegThreads;
  float xv[kX];
#pragma unroll
  for (int k = 0; k < kX; ++k) {
    const int o = threadIdx.x + k * kMrSegThreads;
    xv[k] = 0.f;
    if (o < n) {
      int qi, lam;
      split(o, qi, lam);
      const int g = goff(qi, lam);
      if (sp.first) {
        xv[k] = load_act(p.x, row * d + g, p.xt);
        if (!p.inverse) xv[k] *= (float)p.sign[g];
      } else {
        xv[k] = sp.src[row * d + g];
      }
    }
  }
  __syncthreads();
  // the gather over every stage of the run at once, kG independent loads per thread in
  // flight: a thread issues them all before it stores any
  constexpr int kG = 8;
  const int total = n * sp.sumb;
  for (int o0 = threadIdx.x; o0 < total; o0 += kMrSegThreads * kG) {
    float v[kG];
#pragma unroll
    for (int k = 0; k < kG; ++k) {
      const int o = o0 + k * kMrSegThreads;
      v[k] = 0.f;
      if (o < total) {
        int i = 0;
        while (i + 1 < ns && o >= s_off[i + 1]) ++i;
        const int bb = s_b[i] * s_b[i], r = o - s_off[i], gq = qdiv(r, mkdiv(bb));
        v[k] = __ldg(s_blk[i] + (int64_t)gidx[s_go[i] + gq] * bb + (r - gq * bb));
      }
    }
#pragma unroll
    for (int k = 0; k < kG; ++k)
      if (o0 + k * kMrSegThreads < total) bs[o0 + k * kMrSegThreads] = v[k];
  }
#pragma unroll
  for (int k = 0; k < kX; ++k) {
    const int o = threadIdx.x + k * kMrSegThreads;
    if (o < n) {
      int qi, lam;
      split(o, qi, lam);
      a[qi * br + lam] = xv[k];
    }
  }
  __syncthreads();
  // the stages: the thread's elements o = qi br + lam stay the same through the run
  int eq[kX], el[kX];
#pragma unroll
  for (int k = 0; k < kX; ++k) {
    const int o = threadIdx.x + k * kMrSegThreads;
    eq[k] = qdiv(o, dbr);
    el[k] = o - eq[k] * br;
  }
  for (int step = 0; step < ns; ++step) {
    const int i = p.inverse ? ns - 1 - step : step;
    const int off = s_off[i], b = s_b[i], ls = s_ls[i], ng = br / b;
    const Div dls = mkdiv(ls), db = mkdiv(b);
#pragma unroll
    for (int k = 0; k < kX; ++k) {
      const int o = threadIdx.x + k * kMrSegThreads;
      if (o < n) {
        const int lam = el[k], t1 = qdiv(lam, dls), hi = qdiv(t1, db), digit = t1 - hi * b;
        const int gl = (lam - t1 * ls) + hi * ls;  // lam's group: its digit i taken out
        const float* Bc = bs + off + (eq[k] * ng + gl) * b * b;
        const float* av = a + eq[k] * br + (lam - digit * ls);
        float acc = 0.f;
        if (p.inverse)
          for (int j = 0; j < b; ++j) acc = fmaf(Bc[j * b + digit], av[j * ls], acc);
        else
          for (int j = 0; j < b; ++j) acc = fmaf(Bc[digit * b + j], av[j * ls], acc);
        b2[o] = acc;
      }
    }
    __syncthreads();
    float* tmp = a;
    a = b2;
    b2 = tmp;
  }
  for (int k = 0; k < kX; ++k) {
    const int o = threadIdx.x + k * kMrSegThreads;
    if (o < n) {
      int qi, lam;
      split(o, qi, lam);
      const int g = goff(qi, lam);
      const float v = a[qi * br + lam];
      if (sp.last) store_act(p.y, row * d + g, p.yt, p.inverse ? v * (float)p.sign[g] : v);
      else sp.dst[row * d + g] = v;
    }
  }
}

// all-radix-2 plans: (cos, sin) of stage t, pair c from the block's first row (stage t's
// blocks start at t 2d, four floats per group)
__global__ void cs_of_blocks_kernel(const float* blocks, int64_t d, int m, float2* cs) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)m * (d / 2)) return;
  const int64_t t = i / (d / 2), c = i - t * (d / 2);
  const float* B = blocks + t * 2 * d + 4 * c;
  cs[i] = make_float2(B[0], B[1]);
}

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
  // the first P stages of radix 2 with 64 <= 2^P <= 8192: they are the block-diagonal
  // radix-2 butterfly of width 2^P over the row, whose (cos, sin) table [P][d/2] is taken
  // from the blocks, so that they run on the butterfly kernels (P = m: the whole plan)
  float2* cs2 = nullptr;
  int P = 0;
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
      cudaFree(h->cs2);
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
  int P = 0;  // leading stages of radix 2
  while (P < m && radix[P] == 2) ++P;
  if (P >= 6 && P <= 13) {
    // stage t < P: group c is the butterfly's pair c of stage t (both number a pair by its
    // lower index with bit t removed, block after block), and its block's first row is
    // (cos p, sin p)
    h->P = P;
    if ((e = cudaMalloc(&h->cs2, sizeof(float2) * (size_t)P * (d / 2))) != cudaSuccess)
      return done(set_error(HARP_ERR_CUDA, "mr_plan_create: cudaMalloc: %s", cudaGetErrorString(e)));
    const int64_t n = (int64_t)P * (d / 2);
    cs_of_blocks_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(h->blocks, d, P, h->cs2);
    if ((e = cudaGetLastError()) != cudaSuccess)
      return done(set_error(HARP_ERR_CUDA, "mr_plan_create: table launch: %s", cudaGetErrorString(e)));
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
  cudaFree(plan->cs2);
  cudaSetDevice(prev);
  delete plan;
  return HARP_OK;
}

}  // extern "C"

namespace harp {

cudaError_t launch_mr(const harp_mr_plan_s* plan, int inverse, int batch, const void* x, int xt, void* y, int yt,
                      cudaStream_t st, float* scratch) {
  if (batch <= 0) return cudaSuccess;
  if (plan->cs2 && plan->P == plan->p.m) {  // all radices 2: the radix-2 butterfly of width d
    BflyParams bp{};
    bp.n = plan->p.d;
    bp.w = (int)plan->p.d;
    bp.m = plan->p.m;
    bp.inverse = inverse;
    bp.cs = plan->cs2;
    bp.sign = plan->sign;
    bp.x = x;
    bp.xt = xt;
    bp.x_stride = plan->p.d;
    bp.y = y;
    bp.yt = yt;
    bp.y_stride = plan->p.d;
    bp.nsum = 1;
    return launch_butterfly(bp, batch, st);
  }
  MrParams p = plan->p;
  p.inverse = inverse;
  p.x = x;
  p.xt = xt;
  p.y = y;
  p.yt = yt;
  // few rows: runs of stages over many CTAs, fp32 between runs in y (when fp32) or scratch
  float* buf = yt == DT_F32 ? static_cast<float*>(y) : scratch;
  if (batch < kMrSegRows && buf) {
    // forward with leading radix-2 stages: those first, on the butterfly kernels (signs
    // included), into buf; the runs then start at stage P
    // (in place only up to width 512, where one CTA reads its whole block before writing)
    const bool pre2 = plan->cs2 && !inverse && (x != buf || plan->P <= 9);
    if (pre2) {
      BflyParams bp{};
      bp.n = p.d;
      bp.w = 1 << plan->P;
      bp.m = plan->P;
      bp.cs = plan->cs2;
      bp.sign = plan->sign;
      bp.x = x;
      bp.xt = xt;
      bp.x_stride = p.d;
      bp.y = buf;
      bp.yt = DT_F32;
      bp.y_stride = p.d;
      bp.nsum = 1;
      const cudaError_t e = launch_butterfly(bp, batch, st);
      if (e != cudaSuccess) return e;
    }
    static const int run_cap = [] {
      const char* e = getenv("HARP_MR_RUN");
      return e ? std::max(2, std::min(kMrSegRun, atoi(e))) : kMrSegRun;
    }();
    int runs[kMrMaxStages + 1], nr = 0;  // run boundaries in stage order
    runs[nr++] = pre2 ? plan->P : 0;
    int64_t prod = 1;
    for (int t = runs[0]; t < p.m; ++t) {
      if (prod * p.radix[t] > run_cap && prod > 1) {
        runs[nr++] = t;
        prod = 1;
      }
      prod *= p.radix[t];
    }
    runs[nr] = p.m;
    for (int k = 0; k < nr; ++k) {
      const int r = inverse ? nr - 1 - k : k;  // the transpose runs the stages backwards
      SegParams sp;
      sp.mp = p;
      sp.t0 = runs[r];
      sp.t1 = runs[r + 1];
      if (sp.t1 - sp.t0 > 8) return cudaErrorInvalidValue;
      sp.s0 = (int)p.stride[sp.t0];
      sp.br = 1;
      sp.sumb = 0;
      for (int t = sp.t0; t < sp.t1; ++t) {
        sp.br *= p.radix[t];
        sp.sumb += p.radix[t];
      }
      const int nsub = (int)(p.d / sp.br);
      // enough sub-problems per CTA to fill about one CTA per SM, within the caps
      int K = (nsub * batch + 147) / 148;
      K = std::min(K, std::max(1, kMrSegElems / sp.br));
      int ngrp = 0;  // blocks per sub-problem over the run
      for (int t = sp.t0; t < sp.t1; ++t) ngrp += sp.br / p.radix[t];
      const int per = (sp.br * (2 + sp.sumb) + ngrp) * (int)sizeof(float);  // shared bytes per sub-problem
      K = std::max(1, std::min(K, kMrSegSmem / per));
      sp.K = K;
      sp.first = k == 0 && !pre2;
      sp.last = k == nr - 1;
      sp.src = buf;
      sp.dst = buf;
      const int nblk = (nsub + K - 1) / K;
      const size_t smem = (size_t)K * per;
      if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(mr_seg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
      }
      mr_seg_kernel<<<(unsigned)(nblk * batch), kMrSegThreads, smem, st>>>(sp);
      const cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
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
