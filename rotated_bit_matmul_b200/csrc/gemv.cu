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
#include "common.cuh"

namespace harp {

namespace {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = 32 * (1 + kConsumerWarps);
constexpr int kStages = 6;
constexpr int kSlab = 32 * 128;  // one TMA box: 32 rows x 128 bytes

template <int BITS>
struct Geo {
  static constexpr int kChunkCols = BITS == 4 ? 1024 : 2048;  // columns per stage
  static constexpr int kChunkGroups = kChunkCols / 64;
  static constexpr int kGroupsPerSlab = BITS == 4 ? 4 : 8;       // codes (or 2-bit plane)
  static constexpr int kCodeSlabs = kChunkGroups / kGroupsPerSlab;
  static constexpr int kHiSlabs = BITS == 3 ? kChunkGroups / 16 : 0;  // 1-bit plane
  static constexpr int kStageBytes = (kCodeSlabs + kHiSlabs + 1) * kSlab;
};

// Address of the 16-byte chunk `c` (0..7) of `row` inside a 128B-swizzled box.
__device__ __forceinline__ const uint8_t* swz(const uint8_t* slab, int row, int c) {
  return slab + row * 128 + ((c ^ (row & 7)) << 4);
}

template <int BITS>
__device__ __forceinline__ int group_dot(const uint8_t* codes_slabs, const uint8_t* hi_slabs, int lane,
                                         int gl, const int4* __restrict__ xg, const int4* __restrict__ xgh) {
  if constexpr (BITS == 2 || BITS == 3) {
    const uint4 cw = *reinterpret_cast<const uint4*>(swz(codes_slabs + (gl >> 3) * kSlab, lane, gl & 7));
    const uint32_t wv[4] = {cw.x, cw.y, cw.z, cw.w};
    int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int4 xa = ldg_nc_v4(xg + 2 * k), xb = ldg_nc_v4(xg + 2 * k + 1);
      const uint32_t w = wv[k];
      const uint32_t m0 = w & 0x03030303u, m1 = w & 0x0C0C0C0Cu, m2 = w & 0x30303030u, m3 = w & 0xC0C0C0C0u;
      a0 = dp2a_lo(xa.x, m0, a0);
      a0 = dp2a_hi(xa.y, m0, a0);
      a1 = dp2a_lo(xa.z, m1, a1);
      a1 = dp2a_hi(xa.w, m1, a1);
      a2 = dp2a_lo(xb.x, m2, a2);
      a2 = dp2a_hi(xb.y, m2, a2);
      a3 = dp2a_lo(xb.z, m3, a3);
      a3 = dp2a_hi(xb.w, m3, a3);
    }
    int acc = a0 + (a1 >> 2) + (a2 >> 4) + (a3 >> 6);
    if constexpr (BITS == 3) {
      const int gh = gl & 15;
      const uint2 hw = *reinterpret_cast<const uint2*>(swz(hi_slabs + (gl >> 4) * kSlab, lane, gh >> 1) + (gh & 1) * 8);
      const uint32_t hv[2] = {hw.x, hw.y};
      int h = 0;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
#pragma unroll
        for (int mm = 0; mm < 8; mm += 2) {
          const int4 xa = ldg_nc_v4(xgh + 4 * k + mm / 2);
          const uint32_t ma = hv[k] & (0x01010101u << mm), mb = hv[k] & (0x01010101u << (mm + 1));
          int ha = 0, hb = 0;
          ha = dp2a_lo(xa.x, ma, ha);
          ha = dp2a_hi(xa.y, ma, ha);
          hb = dp2a_lo(xa.z, mb, hb);
          hb = dp2a_hi(xa.w, mb, hb);
          h += (ha >> mm) + (hb >> (mm + 1));
        }
      }
      acc += 4 * h;
    }
    return acc;
  } else {  // 4-bit: two 16-byte chunks per group, 8 codes per word
    const uint8_t* slab = codes_slabs + (gl >> 2) * kSlab;
    const int c0 = (gl & 3) * 2;
    const uint4 ca = *reinterpret_cast<const uint4*>(swz(slab, lane, c0));
    const uint4 cb = *reinterpret_cast<const uint4*>(swz(slab, lane, c0 + 1));
    const uint32_t wv[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
    int lo = 0, hi = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int4 xa = ldg_nc_v4(xg + k);
      const uint32_t ml = wv[k] & 0x0F0F0F0Fu, mh = wv[k] & 0xF0F0F0F0u;
      lo = dp2a_lo(xa.x, ml, lo);
      lo = dp2a_hi(xa.y, ml, lo);
      hi = dp2a_lo(xa.z, mh, hi);
      hi = dp2a_hi(xa.w, mh, hi);
    }
    return lo + (hi >> 4);
  }
}

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_hi,
                const __grid_constant__ CUtensorMap tm_sz, GemvParams p) {
  using G = Geo<BITS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + kStages * G::kStageBytes);
  uint64_t* empty = full + kStages;
  float* red = reinterpret_cast<float*>(empty + kStages);  // [kConsumerWarps][kMaxBatchGemv][32]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = (int)(((int64_t)p.n_out * blockIdx.x) / gridDim.x);
  const int r1 = (int)(((int64_t)p.n_out * (blockIdx.x + 1)) / gridDim.x);
  const int nrows = r1 - r0;
  const int nsub = (nrows + 31) / 32;
  const int ngroups = p.n_in / 64;
  const int nchunks = (ngroups + G::kChunkGroups - 1) / G::kChunkGroups;
  const int nstages = nsub * nchunks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
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
      for (int k = 0; k < nstages; ++k) {
        const int slot = k % kStages;
        if (k >= kStages && !mbar_wait(&empty[slot], ((k / kStages) - 1) & 1, p.status, 1)) break;
        const int sub = k / nchunks, ch = k % nchunks;
        const int row0 = r0 + (int)(((int64_t)nrows * sub) / nsub);
        const int g0 = ch * G::kChunkGroups;
        const int gc = min(G::kChunkGroups, ngroups - g0);
        const int cslabs = (gc + G::kGroupsPerSlab - 1) / G::kGroupsPerSlab;
        const int hslabs = BITS == 3 ? (gc + 15) / 16 : 0;
        uint8_t* st = ring + slot * G::kStageBytes;
        mbar_arrive_expect_tx(&full[slot], (uint32_t)((cslabs + hslabs + 1) * kSlab));
        // x coordinates are in 8-byte units; every one is a multiple of 16 (128-byte slabs)
        const int code_x0 = g0 * (BITS == 4 ? 32 : 16) / 8;  // 16 or 32 code bytes per group
        for (int s = 0; s < cslabs; ++s) tma_load_2d(st + s * kSlab, &tm_codes, &full[slot], code_x0 + s * 16, row0);
        if (BITS == 3)
          for (int s = 0; s < hslabs; ++s)
            tma_load_2d(st + (G::kCodeSlabs + s) * kSlab, &tm_hi, &full[slot], g0 + s * 16, row0);
        tma_load_2d(st + (G::kCodeSlabs + G::kHiSlabs) * kSlab, &tm_sz, &full[slot], g0, row0);
      }
    }
    return;
  }

  // ---------------- consumers
  const int cw = warp - 1;
  float zacc[kMaxBatchGemv];
#pragma unroll
  for (int b = 0; b < kMaxBatchGemv; ++b) zacc[b] = 0.f;
  bool ok = true;

  for (int k = 0; k < nstages && ok; ++k) {
    const int slot = k % kStages;
    if (!mbar_wait(&full[slot], (k / kStages) & 1, p.status, 2)) {
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
      const uint32_t szw = *reinterpret_cast<const uint32_t*>(swz(szs, lane, gl >> 2) + (gl & 3) * 4);
      const float s16 = __half2float(__ushort_as_half((unsigned short)(szw & 0xffffu)));
      const float z16 = __half2float(__ushort_as_half((unsigned short)(szw >> 16)));
#pragma unroll
      for (int b = 0; b < kMaxBatchGemv; ++b) {
        if (b < p.batch) {
          const int4* xg = reinterpret_cast<const int4*>(p.xq + b * p.xq_stride + (int64_t)g * 32);
          const int4* xgh = reinterpret_cast<const int4*>(p.xq + b * p.xq_stride + p.n_in / 2 + (int64_t)g * 32);
          const int acc = group_dot<BITS>(st, st + G::kCodeSlabs * kSlab, lane, gl, xg, xgh);
          const float xs = p.xs[b * p.g_stride + g], xsum = p.xsum[b * p.g_stride + g];
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

template <int BITS>
cudaError_t launch_bits(const Layer& L, const GemvParams& p, cudaStream_t st) {
  using G = Geo<BITS>;
  const size_t smem = 1024 + (size_t)kStages * G::kStageBytes + 2 * kStages * sizeof(uint64_t) +
                      sizeof(float) * kConsumerWarps * kMaxBatchGemv * 32;
  int dev = 0, nsm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  static bool attr_done[64] = {false};  // the attribute is per device; set it once each
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {
    e = cudaFuncSetAttribute(gemv_kernel<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  // one CTA per SM, but never fewer than ~8 rows per CTA
  int grid = nsm;
  if (p.n_out < 8 * grid) grid = (p.n_out + 7) / 8;
  gemv_kernel<BITS><<<grid, kThreads, smem, st>>>(L.tm_codes, L.tm_hi, L.tm_sz, p);
  return cudaGetLastError();
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
