// Butterfly transform F(theta, s, w) and its transpose on sm_100a.
//
// "HARP: Hadamard-Preconditioned Adaptive Rotation Processor for Extreme LLM
// Quantization", Sec. 2.1-2.2: a product of stride stages, each a block-diagonal
// orthogonal matrix of 2x2 blocks B = Q(theta) G_2 (Givens times the normalised
// Sylvester H_2), i.e. [[cos p, sin p], [sin p, -cos p]] with p = pi/4 + theta.
// Forward: signs, then stages of stride 1, 2, ..., w/2. Transpose: stages in
// reverse, then signs (each 2x2 block is symmetric).
//
// Work split. A w-wide block is held by a thread-block cluster of C CTAs (C = 8 for
// w >= 4096, 4 for 2048, 2 for 1024, else 1), E = w / C elements each:
//   layout A: CTA r holds the contiguous chunk [r E, (r+1) E) -> stages 0 .. e-1
//             (e = log2 E) are local;
//   layout B: CTA r holds, for every chunk j, the run [j E + r E/C, j E + (r+1) E/C)
//             -> the remaining log2 C stages (which pair chunk j with j + 2^d) are local.
// Switching layouts is one gather through distributed shared memory between two
// cluster barriers. Each CTA first prefetches exactly its slice of the per-stage
// parameters with bulk copies into shared memory, so no stage waits on global memory.
// The parameters come in one of three forms (TM): raw theta (the stand-alone API),
// the layer's cos/sin pairs, or the layer's int8 angles, whose (cos, sin) of
// pi/4 + delta_t q are evaluated as each rotation needs them.
// The forward epilogue can also emit the GEMV operand: per group of 64 outputs an
// int16 copy in dp2a pair order, the power-of-two scale and the fp32 group sum.
#include "bfly_engine.cuh"
#include "common.cuh"

namespace harp {

namespace {

constexpr int kBflyThreads = 256;
// the engine-based forward path (fast_bfly_kernel) serves the forward calls it covers
constexpr bool kDisableFastButterfly = false;
constexpr float kRsqrt2 = 0.70710678118654752440f;  // cos(pi/4) = sin(pi/4)

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float ld_dsmem(const float* local, uint32_t cta) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(cta));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
  return v;
}

struct Geom {
  int C, lc, E, e, run;  // cluster size, log2 C, elements per CTA, log2 E, E / C
};

__device__ __forceinline__ Geom geom(int w, int m, int C) {
  Geom g;
  g.C = C;
  g.lc = 31 - __clz(C);
  g.E = w / C;
  g.e = m - g.lc;
  g.run = g.E / C;
  return g;
}

enum { kTabTheta = 0, kTabCS = 1, kTabQ8 = 2 };

// (cos, sin) of pi/4 + theta for parameter slot q of a stage's table (sc: the int8 step)
template <int TM>
__device__ __forceinline__ void coef(const void* tab, int q, float sc, float& c, float& s) {
  const float kQuarterPi = 0.785398163397448309616f;
  if (!tab) {
    c = s = kRsqrt2;  // Theta == 0: the randomized Hadamard transform
  } else if (TM == kTabCS) {
    const float2 v = static_cast<const float2*>(tab)[q];
    c = v.x;
    s = v.y;
  } else if (TM == kTabQ8) {
    sincosf(fmaf(sc, (float)static_cast<const int8_t*>(tab)[q], kQuarterPi), &s, &c);
  } else {
    sincosf(kQuarterPi + static_cast<const float*>(tab)[q], &s, &c);
  }
}

// one stage on the layout-A buffer: local pairs (i, i + 2^t), parameter slot q
template <int TM>
__device__ __forceinline__ void stage_a(float* x, const void* tab, float sc, int t, int E, int tid, int nthr) {
  const int h = 1 << t;
  for (int q = tid; q < (E >> 1); q += nthr) {
    const int i = ((q >> t) << (t + 1)) | (q & (h - 1));
    float c, s;
    coef<TM>(tab, q, sc, c, s);
    const float a = x[i], b = x[i + h];
    x[i] = fmaf(c, a, s * b);
    x[i + h] = fmaf(s, a, -c * b);
  }
}

// one stage on the layout-B buffer: runs j and j + 2^d (bit d of j clear), same offset
template <int TM>
__device__ __forceinline__ void stage_b(float* x, const void* tab, float sc, int d, int run, int E, int tid, int nthr) {
  for (int q = tid; q < (E >> 1); q += nthr) {
    const int jj = q / run, ii = q - jj * run;
    const int j = ((jj >> d) << (d + 1)) | (jj & ((1 << d) - 1));
    float c, s;
    coef<TM>(tab, q, sc, c, s);
    float* pa = x + j * run + ii;
    float* pb = pa + (run << d);
    const float a = *pa, b = *pb;
    *pa = fmaf(c, a, s * b);
    *pb = fmaf(s, a, -c * b);
  }
}

template <int TM>
__global__ void __launch_bounds__(kBflyThreads) bfly_kernel(BflyParams p, int C) {
  extern __shared__ __align__(16) uint8_t sm[];
  const Geom g = geom(p.w, p.m, C);
  const int w = p.w, m = p.m, E = g.E, run = g.run;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const uint32_t r = C > 1 ? cluster_rank() : 0;
  const int64_t blk = blockIdx.x / C, row = blockIdx.y;
  const int64_t base = blk * w;
  const int64_t half_n = p.n >> 1;
  constexpr int esz = TM == kTabCS ? 8 : (TM == kTabQ8 ? 1 : 4);

  float* xa = reinterpret_cast<float*>(sm);
  float* xb = xa + E;
  uint8_t* tab = reinterpret_cast<uint8_t*>(xb + E);
  uint64_t* bar = reinterpret_cast<uint64_t*>(tab + (((size_t)m * (E >> 1) * esz + 7) & ~size_t(7)));
  const void* gtab = TM == kTabCS   ? static_cast<const void*>(p.cs)
                     : TM == kTabQ8 ? static_cast<const void*>(p.q8 ? p.q8 + kQ8Head : nullptr)
                                    : static_cast<const void*>(p.theta);
  const bool rht = gtab == nullptr;  // Theta == 0: no per-stage parameters to load
  const uint8_t* stab = rht ? nullptr : tab;
  // int8 angles: stage t's step, read where the stage starts (uniform, cached)
  const float* steps = TM == kTabQ8 && !rht ? reinterpret_cast<const float*>(p.q8) : nullptr;
  auto step_of = [&](int t) -> float { return steps ? __ldg(steps + t) : 0.f; };

  // ---- prefetch this CTA's parameter slice: stage t occupies E/2 entries. Bulk copies
  // need 16-byte aligned sources, destinations and sizes; tiny widths use plain loads.
  const bool use_bulk = !rht && (((E >> 1) * esz) % 16 == 0) && ((half_n * esz) % 16 == 0) &&
                        (((w >> 1) * esz) % 16 == 0) && (C == 1 || (run * esz) % 16 == 0);
  bool ok = true;  // false once a bounded wait has run out
  if (rht) {
    // nothing to prefetch
  } else if (!use_bulk) {
    for (int t = 0; t < m; ++t) {
      const uint8_t* src_stage = static_cast<const uint8_t*>(gtab) + ((int64_t)t * half_n + blk * (w >> 1)) * esz;
      uint8_t* dst = tab + (size_t)t * (E >> 1) * esz;
      for (int q = tid; q < (E >> 1); q += nthr) {
        int64_t src_q;
        if (t < g.e) {
          src_q = (int64_t)r * (E >> 1) + q;
        } else {
          const int d = t - g.e, jj = q / run, ii = q - jj * run;
          const int j = ((jj >> d) << (d + 1)) | (jj & ((1 << d) - 1));
          src_q = (int64_t)(j >> (d + 1)) * (1 << t) + (int64_t)E * (j & ((1 << d) - 1)) + (int64_t)r * run + ii;
        }
        if (esz == 1)
          dst[q] = src_stage[src_q];
        else
          for (int b = 0; b < esz; b += 4)
            *reinterpret_cast<uint32_t*>(dst + (size_t)q * esz + b) =
                *reinterpret_cast<const uint32_t*>(src_stage + src_q * esz + b);
      }
    }
  } else if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, (uint32_t)(m * (E >> 1) * esz));
    for (int t = 0; t < m; ++t) {
      const uint8_t* src_stage = static_cast<const uint8_t*>(gtab) + ((int64_t)t * half_n + blk * (w >> 1)) * esz;
      uint8_t* dst = tab + (size_t)t * (E >> 1) * esz;
      if (t < g.e) {
        bulk_g2s(dst, src_stage + (int64_t)r * (E >> 1) * esz, (uint32_t)((E >> 1) * esz), bar);
      } else {
        const int d = t - g.e;
        for (int jj = 0; jj < (C >> 1); ++jj) {
          const int j = ((jj >> d) << (d + 1)) | (jj & ((1 << d) - 1));
          const int64_t pbase = (int64_t)(j >> (d + 1)) * (1 << t) + (int64_t)E * (j & ((1 << d) - 1)) + (int64_t)r * run;
          bulk_g2s(dst + (size_t)jj * run * esz, src_stage + pbase * esz, (uint32_t)(run * esz), bar);
        }
      }
    }
  }

  if (!p.inverse) {
    // ---- load chunk r (layout A), signs first
    for (int i = tid; i < E; i += nthr) {
      const int64_t gi = base + (int64_t)r * E + i;
      float v = load_act(p.x, row * p.x_stride + gi, p.xt);
      for (int k = 1; k < p.nsum; ++k) v += load_act(p.x, k * p.sum_stride + row * p.x_stride + gi, p.xt);
      xa[i] = v * (float)p.sign[gi];
    }
    __syncthreads();
    // a parameter copy that never lands ends this CTA's work (the status word says where);
    // the cluster barriers the peers expect are still taken
    if (use_bulk) ok = __syncthreads_and(mbar_wait(bar, 0, p.status, 10)) != 0;
    if (ok)
      for (int t = 0; t < g.e; ++t) {
        stage_a<TM>(xa, stab ? stab + (size_t)t * (E >> 1) * esz : nullptr, step_of(t), t, E, tid, nthr);
        __syncthreads();
      }
    float* out = xa;
    if (C > 1) {
      cluster_sync();
      if (ok)
        for (int L = tid; L < E; L += nthr) {
          const int j = L / run, ii = L - j * run;
          xb[L] = ld_dsmem(xa + r * run + ii, (uint32_t)j);
        }
      cluster_sync();  // every peer has finished reading this CTA's chunk
      if (ok)
        for (int d = 0; d < g.lc; ++d) {
          stage_b<TM>(xb, stab ? stab + (size_t)(g.e + d) * (E >> 1) * esz : nullptr, step_of(g.e + d), d, run, E,
                      tid, nthr);
          __syncthreads();
        }
      out = xb;
    }
    // local index L <-> global element: layout A: r E + L; layout B: j E + r run + ii
    auto gidx = [&](int L) -> int64_t {
      if (C == 1) return base + L;
      const int j = L / run, ii = L - j * run;
      return base + (int64_t)j * E + (int64_t)r * run + ii;
    };
    if (ok && p.y)
      for (int L = tid; L < E; L += nthr) store_act(p.y, row * p.y_stride + gidx(L), p.yt, out[L]);
    if (ok && p.xq) {
      // groups of 64 consecutive outputs (runs are >= 64 long): int16 at scale 2^e with
      // max|v| 2^e < 2^15 (e = 15 - E', max|v| = f 2^E', f in [0.5, 1))
      const int lane = tid & 31, warp = tid >> 5, nwarps = nthr >> 5;
      int16_t* xq16 = reinterpret_cast<int16_t*>(p.xq + row * p.xq_stride);
      for (int gl = warp; gl < (E >> 6); gl += nwarps) {
        const float v0 = out[gl * 64 + 2 * lane], v1 = out[gl * 64 + 2 * lane + 1];
        float amax = fmaxf(fabsf(v0), fabsf(v1));
        float sum = v0 + v1;
        const bool bad = __any_sync(0xffffffffu, !(isfinite(v0) && isfinite(v1)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
          sum += __shfl_xor_sync(0xffffffffu, sum, o);
        }
        int ex = 0;
        if (amax > 0.f && !bad) ex = group_exponent(amax);
        const float sc = pow2f(ex);
        const int q0 = max(-32767, min(32767, __float2int_rn(v0 * sc)));
        const int q1 = max(-32767, min(32767, __float2int_rn(v1 * sc)));
        const int64_t gg = gidx(gl * 64) >> 6;  // global group index
        int16_t* grp = xq16 + gg * 64;
        grp[xq_pos_lo(p.bits, 2 * lane)] = (int16_t)q0;
        grp[xq_pos_lo(p.bits, 2 * lane + 1)] = (int16_t)q1;
        if (p.bits == 3) {
          int16_t* hi = xq16 + p.n + gg * 64;  // the 1-bit-plane order follows n int16 values
          hi[xq_pos_hi(2 * lane)] = (int16_t)q0;
          hi[xq_pos_hi(2 * lane + 1)] = (int16_t)q1;
        }
        if (lane == 0) {
          p.xs[row * p.g_stride + gg] = bad ? __int_as_float(0x7fc00000) : pow2f(-ex);
          p.xsum[row * p.g_stride + gg] = bad ? __int_as_float(0x7fc00000) : sum;
        }
      }
    }
  } else {
    // ---- transpose: high stages first (layout B), then the local ones (layout A)
    float* cur = xa;
    if (C > 1) {
      for (int L = tid; L < E; L += nthr) {
        const int j = L / run, ii = L - j * run;
        xb[L] = load_act(p.x, row * p.x_stride + base + (int64_t)j * E + (int64_t)r * run + ii, p.xt);
      }
      __syncthreads();
      if (use_bulk) ok = __syncthreads_and(mbar_wait(bar, 0, p.status, 11)) != 0;
      if (ok)
        for (int d = g.lc - 1; d >= 0; --d) {
          stage_b<TM>(xb, stab ? stab + (size_t)(g.e + d) * (E >> 1) * esz : nullptr, step_of(g.e + d), d, run, E,
                      tid, nthr);
          __syncthreads();
        }
      cluster_sync();
      if (ok)
        for (int u = tid; u < E; u += nthr) {
          const int q = u / run;  // owner CTA of chunk-r element u in layout B
          xa[u] = ld_dsmem(xb + r * run + (u - q * run), (uint32_t)q);
        }
      cluster_sync();
    } else {
      for (int i = tid; i < E; i += nthr) xa[i] = load_act(p.x, row * p.x_stride + base + i, p.xt);
      __syncthreads();
      if (use_bulk) ok = __syncthreads_and(mbar_wait(bar, 0, p.status, 11)) != 0;
    }
    if (ok) {
      for (int t = g.e - 1; t >= 0; --t) {
        stage_a<TM>(cur, stab ? stab + (size_t)t * (E >> 1) * esz : nullptr, step_of(t), t, E, tid, nthr);
        __syncthreads();
      }
      for (int i = tid; i < E; i += nthr) {
        const int64_t gi = base + (int64_t)r * E + i;
        store_act(p.y, row * p.y_stride + gi, p.yt, cur[i] * (float)p.sign[gi]);
      }
    }
  }
  // after a time-out the parameter copy may still be writing into this CTA's shared
  // memory: give it one more bounded wait before the CTA exits
  if (!ok && tid == 0) mbar_wait(bar, 0, nullptr, 12);
}

int cluster_for(int w) { return w >= 4096 ? 8 : (w == 2048 ? 4 : (w == 1024 ? 2 : 1)); }

// ------------------------------------------------------------------ fast forward path
// The forward transform with the layer's tables (or Theta == 0) on the butterfly engines:
// one CTA per (row, block) up to 512 wide, one cluster of 8 per (row, block) from 1024 to
// 8192. 512 threads, one element each (two at 8192); coefficients straight from the tables.
template <int EB, int TM, bool CLUSTER>
__global__ void __launch_bounds__(dec::kNT) fast_bfly_kernel(BflyParams p) {
  using namespace dec;
  __shared__ __align__(16) float sm_T[kRxFloats];
  __shared__ __align__(16) float sm_rx[2][CLUSTER ? kRxFloats : 1];
  __shared__ uint64_t sm_bar[2];
  EngCtx ctx;
  ctx.T = sm_T;
  ctx.rx[0] = sm_rx[0];
  ctx.rx[1] = sm_rx[1];
  ctx.xbar = sm_bar;
  const int ct = threadIdx.x, warp = ct >> 5, lane = ct & 31;
  const int64_t row = blockIdx.y;
  if (ct == 0) {
    s_wait_cycles = p.wait_cycles > 0 ? p.wait_cycles : 4000000000ll;
    mbar_init(&sm_bar[0], 1);
    mbar_init(&sm_bar[1], 1);
    fence_mbar_init();
  }
  if (CLUSTER) cluster_sync_all();
  else __syncthreads();
  const uint8_t* tab = TM == kTmCS ? reinterpret_cast<const uint8_t*>(p.cs) : (TM == kTmQ8 ? p.q8 : nullptr);
  using M = Map<CLUSTER ? EB : EB>;
  const int64_t w = CLUSTER ? (int64_t)kC * M::E : (int64_t)M::E;
  const int64_t blk = CLUSTER ? blockIdx.x / kC : blockIdx.x;
  auto in = [&](int64_t g) {
    float v = load_act(p.x, row * p.x_stride + g, p.xt);
    for (int k = 1; k < p.nsum; ++k) v += load_act(p.x, k * p.sum_stride + row * p.x_stride + g, p.xt);
    return v * (float)__ldg(p.sign + g);
  };
  int16_t* xq16 = p.xq ? reinterpret_cast<int16_t*>(p.xq + row * p.xq_stride) : nullptr;
  if constexpr (CLUSTER) {
    using BF = ClusterBfly<EB, TM>;
    const uint32_t r = cta_rank();
    BF bf;
    bf.fetch(tab, p.n >> 1, blk, r, ct);
    float v[2] = {0.f, 0.f};
    if (ct < M::NT)
#pragma unroll
      for (int s = 0; s < M::P; ++s) v[s] = in(blk * w + BF::ga(r, ct, s));
    Xch x;
    const bool ok = bf.run(v, ctx, x, r, ct, p.status, 20);
    if (ok && p.y && ct < M::NT)
#pragma unroll
      for (int s = 0; s < M::P; ++s) store_act(p.y, row * p.y_stride + blk * w + BF::gb(r, ct, s), p.yt, v[s]);
    if constexpr (M::RUN >= 64) {
      if (ok && xq16) {  // groups of 64 lie inside the layout-B runs
        constexpr int GPR = M::RUN / 64, NGL = M::E / 64;
        if (ct < M::NT)
#pragma unroll
          for (int s = 0; s < M::P; ++s) sm_T[M::idx_b(M::bj(ct), M::bii(ct, s))] = v[s];
        cbar();
        if (warp < NGL) {
          const int j = warp / GPR, kk = warp - j * GPR;
          const int64_t G = (blk * w + j * M::E + (int)r * M::RUN + 64 * kk) >> 6;
          prep_group(sm_T + j * M::PAD + 64 * kk, p.bits, xq16 + G * 64, xq16 + p.n + G * 64,
                     p.xs + row * p.g_stride + G, p.xsum + row * p.g_stride + G, lane);
        }
      }
    }
    cluster_sync_all();  // no CTA leaves while a peer may still store into it
  } else {
    LocalBfly<EB, TM> lb;
    lb.fetch(tab, p.n >> 1, blk, ct);
    float v = ct < M::NT ? in(blk * w + M::e1(ct, 0)) : 0.f;
    lb.run(v, ctx, ct);
    if (ct < M::NT) {
      if (p.y) store_act(p.y, row * p.y_stride + blk * w + M::e2(ct, 0), p.yt, v);
      if (xq16) sm_T[M::e2(ct, 0)] = v;  // natural order for the groups
    }
    if (xq16) {
      cbar();
      if (warp < (M::E >> 6)) {
        const int64_t G = ((blk * w) >> 6) + warp;
        prep_group(sm_T + 64 * warp, p.bits, xq16 + G * 64, xq16 + p.n + G * 64, p.xs + row * p.g_stride + G,
                   p.xsum + row * p.g_stride + G, lane);
      }
    }
  }
}

template <int TM, bool CLUSTER>
const void* fast_kernel_for(int eb) {
  if (CLUSTER) {
    switch (eb) {
      case 7: return reinterpret_cast<const void*>(fast_bfly_kernel<7, TM, true>);
      case 8: return reinterpret_cast<const void*>(fast_bfly_kernel<8, TM, true>);
      case 9: return reinterpret_cast<const void*>(fast_bfly_kernel<9, TM, true>);
      case 10: return reinterpret_cast<const void*>(fast_bfly_kernel<10, TM, true>);
    }
  } else {
    switch (eb) {
      case 6: return reinterpret_cast<const void*>(fast_bfly_kernel<6, TM, false>);
      case 7: return reinterpret_cast<const void*>(fast_bfly_kernel<7, TM, false>);
      case 8: return reinterpret_cast<const void*>(fast_bfly_kernel<8, TM, false>);
      case 9: return reinterpret_cast<const void*>(fast_bfly_kernel<9, TM, false>);
    }
  }
  return nullptr;
}

// true (and *e set) when the fast path took the call
bool launch_fast(const BflyParams& p, int batch, cudaStream_t st, cudaError_t* e) {
  if (p.inverse || (!p.cs && !p.q8 && p.theta)) return false;  // transposes and raw angles: the general kernel
  const int w = p.w;
  const bool local = w >= 64 && w <= 512, cluster = w >= 1024 && w <= 8192;
  if (!local && !cluster) return false;
  if (cluster && p.xq && w < 4096) return false;  // operand groups would straddle CTAs
  int eb = 0;
  while ((1 << eb) < (cluster ? w / dec::kC : w)) ++eb;
  const int tm = p.q8 ? dec::kTmQ8 : (p.cs ? dec::kTmCS : dec::kTmHad);
  const void* fn = nullptr;
  if (tm == dec::kTmCS) fn = cluster ? fast_kernel_for<dec::kTmCS, true>(eb) : fast_kernel_for<dec::kTmCS, false>(eb);
  else if (tm == dec::kTmQ8) fn = cluster ? fast_kernel_for<dec::kTmQ8, true>(eb) : fast_kernel_for<dec::kTmQ8, false>(eb);
  else fn = cluster ? fast_kernel_for<dec::kTmHad, true>(eb) : fast_kernel_for<dec::kTmHad, false>(eb);
  if (!fn) return false;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((p.n / w) * (cluster ? dec::kC : 1)), (unsigned)batch, 1);
  cfg.blockDim = dim3(dec::kNT, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster ? dec::kC : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {const_cast<BflyParams*>(&p)};
  *e = cudaLaunchKernelExC(&cfg, fn, args);
  return true;
}

}  // namespace

cudaError_t launch_butterfly(const BflyParams& p, int batch, cudaStream_t st) {
  if (batch <= 0) return cudaSuccess;
  if (!kDisableFastButterfly) {
    cudaError_t e = cudaSuccess;
    if (launch_fast(p, batch, st, &e)) return e;
  }
  const int C = cluster_for(p.w);
  const int E = p.w / C;
  const int tm = p.q8 ? kTabQ8 : (p.cs ? kTabCS : kTabTheta);
  const int esz = tm == kTabCS ? 8 : (tm == kTabQ8 ? 1 : 4);
  // the parameter table is followed by the mbarrier, which wants 8-byte alignment
  const size_t tab_bytes = ((size_t)p.m * (E / 2) * esz + 7) & ~size_t(7);
  const size_t smem = sizeof(float) * 2 * (size_t)E + tab_bytes + 16;
  int threads = E / 2 < kBflyThreads ? E / 2 : kBflyThreads;
  if (threads < 32) threads = 32;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((p.n / p.w) * C), (unsigned)batch, 1);
  cfg.blockDim = dim3((unsigned)threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const void* fn = tm == kTabQ8   ? reinterpret_cast<const void*>(bfly_kernel<kTabQ8>)
                   : tm == kTabCS ? reinterpret_cast<const void*>(bfly_kernel<kTabCS>)
                                  : reinterpret_cast<const void*>(bfly_kernel<kTabTheta>);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  if (tm == kTabQ8) return cudaLaunchKernelEx(&cfg, bfly_kernel<kTabQ8>, p, C);
  if (tm == kTabCS) return cudaLaunchKernelEx(&cfg, bfly_kernel<kTabCS>, p, C);
  return cudaLaunchKernelEx(&cfg, bfly_kernel<kTabTheta>, p, C);
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

// int8 angle storage, one CTA per stage: delta_t = fp32(max |theta_t| / 127) and
// q = round-half-even(theta / delta_t) evaluated in fp64 (the inputs are fp32, so the
// quotient is exact before rounding), clamped to +-127; q = 0 when delta_t = 0.
__global__ void __launch_bounds__(256) quantize_angles_kernel(const float* __restrict__ theta, int64_t half_n,
                                                              int8_t* __restrict__ q, float* __restrict__ delta) {
  __shared__ float red[8];
  __shared__ float dsh;
  const int t = blockIdx.x, tid = threadIdx.x;
  const float* th = theta + (int64_t)t * half_n;
  float mx = 0.f;
  for (int64_t i = tid; i < half_n; i += 256) mx = fmaxf(mx, fabsf(th[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) red[tid >> 5] = mx;
  __syncthreads();
  if (tid == 0) {
    float m = 0.f;
    for (int k = 0; k < 8; ++k) m = fmaxf(m, red[k]);
    dsh = (float)((double)m / 127.0);
    delta[t] = dsh;
  }
  __syncthreads();
  const double d = (double)dsh;
  for (int64_t i = tid; i < half_n; i += 256) {
    double v = d > 0.0 ? rint((double)th[i] / d) : 0.0;
    v = fmin(fmax(v, -127.0), 127.0);
    q[(int64_t)t * half_n + i] = (int8_t)(int)v;
  }
}

cudaError_t launch_quantize_angles(int m, int64_t half_n, const float* theta, int8_t* q, float* delta,
                                   cudaStream_t st) {
  if (m <= 0 || half_n <= 0) return cudaSuccess;
  quantize_angles_kernel<<<(unsigned)m, 256, 0, st>>>(theta, half_n, q, delta);
  return cudaGetLastError();
}

}  // namespace harp
