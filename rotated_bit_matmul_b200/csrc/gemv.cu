// Fused dequant-GEMV for decode batches (1..8 rows) on sm_100a CUDA cores.
//
// z[b][r] = sum_g ( scale16[r][g] * sum_{j in g} q[r][j] x~[b][j] + zero16[r][g] * X[b][g] )
// with x~ = F_V(x) and X[b][g] the fp32 group sums of x~ (the stand-in quantizer's
// dequant scale16*q + zero16, regrouped so the zero term is one FMA per group).
//
// Inner product: x~ arrives as int16 with one power-of-two scale per group, so
// sum_j q_j x~_j is an exact int32 dot product evaluated with dp2a (two int16 x
// uint8 products per instruction); the 2-bit codes are masked in place (no shifts)
// and the mask's power-of-four weight is removed by an exact arithmetic shift.
//
// Data movement: one producer warp streams the CTA's rows of packed codes and
// scale_zero from HBM with 2-D TMA tile loads (128-byte swizzle, no multicast) into
// a ring of shared-memory stages guarded by mbarriers; consumer warps own one output
// row per lane and split each stage's groups between them. Every CTA gets a
// contiguous, balanced range of output rows; the grid is one CTA per SM.
#include "gemv_core.cuh"

namespace harp {

namespace {

using namespace gemv_core;

constexpr int kConsumerWarps = 8;
constexpr int kThreads = 32 * (1 + kConsumerWarps);
template <int BITS, bool XS>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_hi,
                const __grid_constant__ CUtensorMap tm_sz, GemvParams p) {
  using G = Geo<BITS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + G::kStages * G::kStageBytes);
  uint64_t* empty = full + G::kStages;
  uint64_t* xbar = empty + G::kStages;
  float* red = reinterpret_cast<float*>(xbar + 2);  // [kConsumerWarps][kMaxBatchGemv][32]
  // staged activation operand (XS): per batch row xq (xq_stride words), xs and xsum (g_stride each)
  uint8_t* xstage = reinterpret_cast<uint8_t*>(red + kConsumerWarps * kMaxBatchGemv * 32);
  const int64_t xrow_bytes = 4 * (p.xq_stride + 2 * p.g_stride);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = (int)(((int64_t)p.n_out * blockIdx.x) / gridDim.x);
  const int r1 = (int)(((int64_t)p.n_out * (blockIdx.x + 1)) / gridDim.x);
  const int nrows = r1 - r0;
  const int nsub = (nrows + 31) / 32;
  const int ngroups = p.n_in / 64;
  const int nchunks = (ngroups + G::kChunkGroups - 1) / G::kChunkGroups;
  const int nstages = nsub * nchunks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < G::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    mbar_init(xbar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (nrows <= 0) return;

  if (warp == 0) {
    // ---------------- producer: weights never depend on activations, so it runs ahead
    if (lane == 0) {
      tma_prefetch_desc(&tm_codes);
      tma_prefetch_desc(&tm_sz);
      if (BITS == 3) tma_prefetch_desc(&tm_hi);
      if constexpr (XS) {
        mbar_arrive_expect_tx(xbar, (uint32_t)(xrow_bytes * p.batch));
        for (int b = 0; b < p.batch; ++b) {
          uint8_t* dst = xstage + b * xrow_bytes;
          bulk_g2s(dst, p.xq + b * p.xq_stride, (uint32_t)(4 * p.xq_stride), xbar);
          bulk_g2s(dst + 4 * p.xq_stride, p.xs + b * p.g_stride, (uint32_t)(4 * p.g_stride), xbar);
          bulk_g2s(dst + 4 * (p.xq_stride + p.g_stride), p.xsum + b * p.g_stride, (uint32_t)(4 * p.g_stride), xbar);
        }
      }
      int k = 0;
      for (; k < nstages; ++k) {
        const int slot = k % G::kStages;
        if (k >= G::kStages && !mbar_wait(&empty[slot], ((k / G::kStages) - 1) & 1, p.status, 1, p.wait_ns)) break;
        if (k == p.skip_stage && blockIdx.x == 0) continue;  // testing hook: this stage never lands
        const int sub = k / nchunks, ch = k % nchunks;
        const int row0 = r0 + (int)(((int64_t)nrows * sub) / nsub);
        const int g0 = ch * G::kChunkGroups;
        const int gc = min(G::kChunkGroups, ngroups - g0);
        const int cslabs = (gc + G::kGroupsPerSlab - 1) / G::kGroupsPerSlab;
        const int hslabs = BITS == 3 ? (gc + 15) / 16 : 0;
        uint8_t* st = ring + slot * G::kStageBytes;
        mbar_arrive_expect_tx(&full[slot], (uint32_t)((cslabs + hslabs + (gc + 31) / 32) * kSlab));
        // x coordinates are in 8-byte units; every one is a multiple of 16 (128-byte slabs)
        const int code_x0 = g0 * (BITS == 4 ? 32 : 16) / 8;  // 16 or 32 code bytes per group
        for (int s = 0; s < cslabs; ++s) tma_load_2d(st + s * kSlab, &tm_codes, &full[slot], code_x0 + s * 16, row0);
        if (BITS == 3)
          for (int s = 0; s < hslabs; ++s)
            tma_load_2d(st + (G::kCodeSlabs + s) * kSlab, &tm_hi, &full[slot], g0 + s * 16, row0);
        for (int s = 0; s < (gc + 31) / 32; ++s)
          tma_load_2d(st + (G::kCodeSlabs + G::kHiSlabs + s) * kSlab, &tm_sz, &full[slot], g0 + s * 32, row0);
      }
      // the CTA must not exit while copies are still writing into its shared memory: wait
      // (bounded) for the stages issued last, which the consumers may have left behind
      const int nlast = k < G::kStages ? k : G::kStages;
      for (int q = k - nlast; q < k; ++q)
        if (!(q == p.skip_stage && blockIdx.x == 0))
          mbar_wait(&full[q % G::kStages], (q / G::kStages) & 1, nullptr, 4, p.wait_ns);
    }
    return;
  }

  // ---------------- consumers
  const int cw = warp - 1;
  float zacc[kMaxBatchGemv];
#pragma unroll
  for (int b = 0; b < kMaxBatchGemv; ++b) zacc[b] = 0.f;
  bool ok = true;
  if constexpr (XS) ok = mbar_wait(xbar, 0, p.status, 3, p.wait_ns);

  for (int k = 0; k < nstages && ok; ++k) {
    const int slot = k % G::kStages;
    if (!mbar_wait(&full[slot], (k / G::kStages) & 1, p.status, 2, p.wait_ns)) {
      ok = false;
      break;
    }
    const int sub = k / nchunks, ch = k % nchunks;
    const int row0 = r0 + (int)(((int64_t)nrows * sub) / nsub);
    const int row1 = r0 + (int)(((int64_t)nrows * (sub + 1)) / nsub);
    const int g0 = ch * G::kChunkGroups;
    const int gc = min(G::kChunkGroups, ngroups - g0);
    const uint8_t* st = ring + slot * G::kStageBytes;
    const uint8_t* szs = st + (G::kCodeSlabs + G::kHiSlabs) * kSlab;

    for (int gl = cw; gl < gc; gl += kConsumerWarps) {
      const int g = g0 + gl;
      const uint32_t szw = sz_word(szs, lane, gl);
      const float s16 = __half2float(__ushort_as_half((unsigned short)(szw & 0xffffu)));
      const float z16 = __half2float(__ushort_as_half((unsigned short)(szw >> 16)));
#pragma unroll
      for (int b = 0; b < kMaxBatchGemv; ++b) {
        if (b < p.batch) {
          const int32_t* xqb;
          float xs, xsum;
          if constexpr (XS) {
            const uint8_t* row = xstage + b * xrow_bytes;
            xqb = reinterpret_cast<const int32_t*>(row);
            xs = reinterpret_cast<const float*>(row + 4 * p.xq_stride)[g];
            xsum = reinterpret_cast<const float*>(row + 4 * (p.xq_stride + p.g_stride))[g];
          } else {
            xqb = p.xq + b * p.xq_stride;
            xs = p.xs[b * p.g_stride + g];
            xsum = p.xsum[b * p.g_stride + g];
          }
          const int4* xg = reinterpret_cast<const int4*>(xqb + (int64_t)g * 32);
          const int4* xgh = reinterpret_cast<const int4*>(xqb + p.n_in / 2 + (int64_t)g * 32);
          const int acc = group_dot<BITS, XS>(st, st + G::kCodeSlabs * kSlab, lane, gl, xg, xgh);
          zacc[b] = fmaf(s16, (float)acc * xs, fmaf(z16, xsum, zacc[b]));
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);

    if (ch == nchunks - 1) {
      // reduce the consumer warps' partial sums of this sub-tile's rows, fixed order
#pragma unroll
      for (int b = 0; b < kMaxBatchGemv; ++b)
        if (b < p.batch) red[(cw * kMaxBatchGemv + b) * 32 + lane] = zacc[b];
      asm volatile("bar.sync 1, %0;" ::"r"(kConsumerWarps * 32) : "memory");
      for (int b = cw; b < p.batch; b += kConsumerWarps) {
        float s = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < kConsumerWarps; ++w2) s += red[(w2 * kMaxBatchGemv + b) * 32 + lane];
        if (row0 + lane < row1) p.z[b * p.z_stride + row0 + lane] = s;
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kConsumerWarps * 32) : "memory");
#pragma unroll
      for (int b = 0; b < kMaxBatchGemv; ++b) zacc[b] = 0.f;
    }
  }
}

template <int BITS, bool XS>
cudaError_t launch_bits(const Layer& L, const GemvParams& p, cudaStream_t st, int dev, int nsm) {
  using G = Geo<BITS>;
  const size_t xbytes = XS ? (size_t)4 * (p.xq_stride + 2 * p.g_stride) * p.batch : 0;
  const size_t base = 1024 + (size_t)G::kStages * G::kStageBytes + (2 * G::kStages + 2) * sizeof(uint64_t) +
                      sizeof(float) * kConsumerWarps * kMaxBatchGemv * 32;
  const size_t smem = base + xbytes;
  const size_t smem_max = base + (XS ? kXStageMax : 0);
  static bool attr_done[64] = {false};  // the attribute is per device; set it once each
  if (!attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<BITS, XS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_max);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  // one CTA per SM, but never fewer than ~8 rows per CTA
  int grid = nsm;
  if (p.n_out < 8 * grid) grid = (p.n_out + 7) / 8;
  gemv_kernel<BITS, XS><<<grid, kThreads, smem, st>>>(L.tm_codes, L.tm_hi, L.tm_sz, p);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_bits(const Layer& L, const GemvParams& p, cudaStream_t st) {
  int dev = 0, nsm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t xbytes = 4 * (p.xq_stride + 2 * p.g_stride) * (int64_t)p.batch;
  // bulk copies need 16-byte multiples: xq rows are n_in/2 or n_in words, xs/xsum rows n_in/64 floats
  const bool aligned = (p.g_stride % 4 == 0) && (p.xq_stride % 4 == 0);
  if (xbytes <= kXStageMax && aligned) return launch_bits<BITS, true>(L, p, st, dev, nsm);
  return launch_bits<BITS, false>(L, p, st, dev, nsm);
}

}  // namespace

cudaError_t launch_gemv(const Layer& L, const GemvParams& p, cudaStream_t st) {
  if (p.batch <= 0) return cudaSuccess;
  switch (p.bits) {
    case 2: return launch_bits<2>(L, p, st);
    case 3: return launch_bits<3>(L, p, st);
    case 4: return launch_bits<4>(L, p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace harp
