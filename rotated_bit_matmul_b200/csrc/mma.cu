// Dequant -> tcgen05 tensor-core contraction of the rotated low-bit linear for token
// batches of 16 and more (HARP: "rotated, quantized linear y = U^T deq(Q(U W V^T)) V x").
//
// One CTA owns a tile of 128 weight rows, up to 256 tokens and one split of the input
// groups:
// * warp 0 streams, with TMA and no multicast, into a shared-memory ring:
//   * the packed codes of one 64-column group per stage;
//   * the matching 64 columns of the fp16 token operand.
// * warps 2..9 expand the codes to fp16 s*q in the 128-byte-swizzled K-major layout
//   that the tensor core reads.
// * one lane of warp 1 issues tcgen05.mma kind::f16 (M = 128, N = tokens, K = 16) into a
//   tensor-memory accumulator. It commits each stage back to the ring.
// * warps 2..9 then read the accumulator with tcgen05.ld and store the split's fp32
//   partial sums. The output butterfly adds the splits in a fixed order.
//
// Fused epilogue (output blocks of w_out = 128 or 256 rows, HARP Sec. 2.4: the stride
// stages fused with the contraction). The H = w_out / 128 tiles of one output block and
// all S splits run as one thread-block cluster of H S CTAs. Each CTA writes its scaled
// partial tile into its own (by then idle) ring, token-major. After a cluster barrier each
// CTA takes a share of the token columns, one warp per column: it reads the block's H S
// partial tiles through distributed shared memory, adds the splits in split order, applies
// the signs and the block's stride stages (the layer's cos/sin pairs, int8 angles, or
// Theta = 0) in registers and warp shuffles, and writes y. A second cluster barrier keeps every tile alive until its last
// reader is done. No partial array and no output-butterfly launch remain.
//
// Zero term. deq(q) = s q + m for each (row, group), so
//   z = sum_j (s q_j) x_j + sum_g m_g X_g,
// where X_g is a group sum of the operand. The second sum runs on the tensor core as one
// extra K block per split, the first stage of the ring:
// * the weight side holds the split's m values (fp16, exactly as stored);
// * the token side holds the group sums, which the operand prep appends after the n_in
//   columns.
// Hoisting m leaves one packed FMA per pair of weights: fma(1024 + q, s, -1024 s) rounds
// q s once.
#include "common.cuh"
#include "mma.h"

#include <algorithm>
#include <cstdlib>

namespace harp {
namespace mma {
namespace {

// ------------------------------------------------------------------ tcgen05 / proxy helpers
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of 128 bytes,
// 8-row groups 1024 bytes apart (start address 16-byte units, version 1, layout 2).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3fffu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator, A = B = fp16, both K-major,
// N >> 3 in bits 17..22, M >> 4 in bits 24..28.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
      : "memory");
}

// Arrives on `bar` once every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 8 consecutive accumulator columns of this thread's lane (whole warp).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r0, r1, r2, r3, r4, r5, r6, r7;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3), "=r"(r4), "=r"(r5), "=r"(r6), "=r"(r7)
               : "r"(taddr)
               : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  v[0] = __uint_as_float(r0); v[1] = __uint_as_float(r1); v[2] = __uint_as_float(r2); v[3] = __uint_as_float(r3);
  v[4] = __uint_as_float(r4); v[5] = __uint_as_float(r5); v[6] = __uint_as_float(r6); v[7] = __uint_as_float(r7);
}

__device__ __forceinline__ void st_shared_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(smem_u32(p)), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// fp16 (q_lo, q_hi) * s, rounded once, from t = (1024 + q_lo, 1024 + q_hi) as fp16 bits.
// The fast form needs -1024 s finite in fp16 (|s| < 64); larger scales take two steps.
__device__ __forceinline__ uint32_t scale_pair(uint32_t t, __half2 s2, __half2 c2, bool fast) {
  if (fast) return h2u(__hfma2(u2h(t), s2, c2));
  return h2u(__hmul2(__hsub2(u2h(t), __half2half2(__float2half(1024.f))), s2));
}

constexpr int kMaxStages = 8;

struct Params {
  CUtensorMap tm_codes;  // codes (2-bit plane of 3-bit codes) as bytes, box {cb, 128}
  CUtensorMap tm_sz;     // scale_zero as uint32, box {gs, 128}
  CUtensorMap tm_hi;     // 1-bit plane of 3-bit codes as bytes, box {8 gs, 128}
  CUtensorMap tm_x;      // fp16 operand [batch][ld], box {64, N}, 128-byte swizzle
  int n_out, n_in, G, gs, N, stages, batch, ncols;
  const float* rowscale;
  float* zpart;
  int* status;
  // fused epilogue (fuse != 0): cluster of H tiles x all splits per w_out-row block
  int fuse, H, w_out, m_out;
  const int8_t* sign;  // [n_out] output-side signs
  const float2* cs;    // [m_out][n_out/2] (cos, sin), or null
  const uint8_t* q8;   // int8 angles (fp32 steps head, then [m_out][n_out/2]), or null
  void* y;
  int yt;
  int64_t y_stride;
};


template <int BITS>
struct Geo {
  static constexpr int kCodeBytes = BITS == 4 ? 32 : 16;  // bytes of one row's group in the code tile
  static constexpr int kA = kBM * 128;                     // dequantized weight tile (16 KB)
};

// Dynamic shared memory: [ring: stages x (A 16 KB | X N*128 | codes 128*cb)] [sz 128*gs*4]
// [hi 128*gs*8] [barriers, 256 B] [fused epilogue: the output block's (cos, sin) pairs];
// the ring starts 1024-byte aligned (swizzle atoms).
constexpr int kCfBytes = 8 * 128 * 8;  // log2 256 stages x 128 pairs x (cos, sin)
template <int BITS>
__host__ __device__ inline int stage_bytes(int N) {
  return Geo<BITS>::kA + N * 128 + kBM * Geo<BITS>::kCodeBytes;
}
template <int BITS>
__host__ __device__ inline int fixed_bytes(int gs, bool fuse) {
  // + barriers + alignment slack (+ the fused epilogue's coefficients)
  return kBM * gs * 4 + (BITS == 3 ? kBM * gs * 8 : 0) + 256 + 1024 + (fuse ? kCfBytes : 0);
}

// (cos, sin) of pi/4 + theta_t for pair q of the output side's stage t (global slot)
__device__ __forceinline__ void out_coef(const Params& p, int t, int64_t slot, float& c, float& s) {
  if (p.q8) {
    const float step = __ldg(reinterpret_cast<const float*>(p.q8) + t);
    const int8_t a = reinterpret_cast<const int8_t*>(p.q8 + kQ8Head)[(int64_t)t * (p.n_out >> 1) + slot];
    sincosf(fmaf(step, (float)a, 0.785398163397448309616f), &s, &c);
  } else if (p.cs) {
    const float2 v = __ldg(p.cs + (int64_t)t * (p.n_out >> 1) + slot);
    c = v.x;
    s = v.y;
  } else {
    c = s = 0.70710678118654752440f;  // Theta = 0
  }
}

// the output block's (cos, sin) pairs into cf, stage-major, by the 256 dequant threads (t);
// out of line, so that the int8 angles' sincosf does not weigh on the main loop's registers
__device__ __noinline__ void stage_out_coefs(const Params& p, float2* cf, int blk, int t) {
  const int hw = p.w_out >> 1;
  for (int k = t; k < p.m_out * hw; k += 32 * kDqWarps) {
    float c, s;
    out_coef(p, k / hw, (int64_t)blk * hw + (k % hw), c, s);
    cf[k] = make_float2(c, s);
  }
}

// four fp32 at `local` (16-byte aligned, this CTA's shared memory) in cluster CTA `cta`'s copy
__device__ __forceinline__ float4 ld_peer4(const float* local, uint32_t cta) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(cta));
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(ra)
               : "memory");
  return v;
}

// The cluster's output block of W rows: split sums, signs, stride stages and the store of y
// for this CTA's share of the token columns. Every CTA of the cluster takes both cluster
// barriers. One warp per token column, W / 32 consecutive rows per lane: stages of stride
// below W / 32 stay inside a lane, the wider ones pair lanes through shuffles. `tile` is
// this CTA's partial tile; `cf` holds the block's log2 W x W/2 (cos, sin) pairs, stage-major.
template <int W>
__device__ __noinline__ void fused_epilogue(const Params& p, const float* tile, const float2* cf, int tile_idx, int b0) {
  constexpr int EPL = W / 32, LE = EPL == 8 ? 3 : 2, LW = W == 256 ? 8 : 7, HW = W / 2;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H, S = (int)gridDim.y, R = H * S;
  const int blk = tile_idx / H;
  const uint32_t rank = cluster_rank();
  cluster_sync_all();  // every partial tile of the cluster written
  const int nval = min(p.N, p.batch - b0);
  const int per = (nval + R - 1) / R;
  const int c_lo = min(nval, (int)rank * per), c_hi = min(nval, c_lo + per);
  const int e0 = lane * EPL, h0 = e0 >> 7;
  const int8_t* sg = p.sign + (int64_t)blk * W + e0;
  float sgn[EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) sgn[j] = (float)__ldg(sg + j);
  for (int col = c_lo + warp; col < c_hi; col += kThreads / 32) {
    const float* src = tile + col * kBM + (e0 & (kBM - 1));
    float v[EPL];
#pragma unroll
    for (int k = 0; k < EPL / 4; ++k) {
      const float4 a = ld_peer4(src + 4 * k, (uint32_t)h0);  // split 0 of tile h0: cluster rank h0
      v[4 * k] = a.x;
      v[4 * k + 1] = a.y;
      v[4 * k + 2] = a.z;
      v[4 * k + 3] = a.w;
    }
    for (int sp = 1; sp < S; ++sp) {
#pragma unroll
      for (int k = 0; k < EPL / 4; ++k) {
        const float4 a = ld_peer4(src + 4 * k, (uint32_t)(h0 + sp * H));
        v[4 * k] += a.x;
        v[4 * k + 1] += a.y;
        v[4 * k + 2] += a.z;
        v[4 * k + 3] += a.w;
      }
    }
#pragma unroll
    for (int j = 0; j < EPL; ++j) v[j] *= sgn[j];
    // stages inside the lane: pairs (j, j + 2^t)
#pragma unroll
    for (int t = 0; t < LE; ++t) {
      const int hs = 1 << t;
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        if (j & hs) continue;
        const int i = e0 + j, q = ((i >> (t + 1)) << t) | (i & (hs - 1));
        const float2 k2 = cf[t * HW + q];
        const float a = v[j], b = v[j + hs];
        v[j] = fmaf(k2.x, a, k2.y * b);
        v[j + hs] = fmaf(k2.y, a, -k2.x * b);
      }
    }
    // stages across lanes: lane bit t - LE pairs row i (bit clear) with i + 2^t
#pragma unroll
    for (int t = LE; t < LW; ++t) {
      const int lb = 1 << (t - LE), hs = 1 << t;
      const bool upper = (lane & lb) != 0;
      const int il = (lane & ~lb) * EPL;  // the lower lane's first row
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        const float o = __shfl_xor_sync(0xffffffffu, v[j], lb);
        const int i = il + j, q = ((i >> (t + 1)) << t) | (i & (hs - 1));
        const float2 k2 = cf[t * HW + q];
        v[j] = upper ? fmaf(k2.y, o, -k2.x * v[j]) : fmaf(k2.x, v[j], k2.y * o);
      }
    }
    const int64_t yo = (int64_t)(b0 + col) * p.y_stride + (int64_t)blk * W + e0;
#pragma unroll
    for (int j = 0; j < EPL; ++j) store_act(p.y, yo + j, p.yt, v[j]);
  }
  cluster_sync_all();  // no tile leaves while a peer may still read it
}

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) mma_kernel(const __grid_constant__ Params p) {
  using Gm = Geo<BITS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int SB = stage_bytes<BITS>(p.N);
  const int ST = p.stages;
  uint8_t* ring = base;
  uint32_t* sz_s = reinterpret_cast<uint32_t*>(ring + (size_t)ST * SB);
  uint8_t* hi_s = reinterpret_cast<uint8_t*>(sz_s + kBM * p.gs);
  uint64_t* bars = reinterpret_cast<uint64_t*>(hi_s + (BITS == 3 ? kBM * p.gs * 8 : 0));
  uint64_t* full = bars;                    // [ST] TMA landed (codes + operand)
  uint64_t* afull = bars + kMaxStages;      // [ST] dequantized tile written
  uint64_t* empty = bars + 2 * kMaxStages;  // [ST] MMAs of the stage completed
  uint64_t* pre = bars + 3 * kMaxStages;    // scale/zero (and hi plane) of the split landed
  uint64_t* accb = pre + 1;                 // accumulator complete
  uint32_t* tslot = reinterpret_cast<uint32_t*>(accb + 1);
  float2* cf_s = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(bars) + 256);  // fused epilogue only

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, split = blockIdx.y, b0 = blockIdx.z * kMaxN;
  const int g0 = split * p.gs;
  const int ngs = min(p.gs, p.G - g0);  // groups of this split
  const int nst = 1 + ngs;              // the zero block, then one stage per group
  const int row0 = tile * kBM;

  if (tid == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&afull[i], kDqWarps);
      mbar_init(&empty[i], 1);
    }
    mbar_init(pre, 1);
    mbar_init(accb, 1);
    fence_mbar_init();
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tslot, (uint32_t)p.ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    // ---------------- producer (lane 0 issues; the warp stays converged around it)
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_codes);
      tma_prefetch_desc(&p.tm_x);
      mbar_arrive_expect_tx(pre, (uint32_t)(kBM * p.gs * 4 + (BITS == 3 ? kBM * p.gs * 8 : 0)));
      tma_load_2d(sz_s, &p.tm_sz, pre, g0, row0);
      if (BITS == 3) tma_load_2d(hi_s, &p.tm_hi, pre, g0 * 8, row0);
      int k = 0;
      for (; k < nst; ++k) {
        const int slot = k % ST;
        if (k >= ST && !mbar_wait_sleep(&empty[slot], ((k / ST) - 1) & 1, p.status, 80)) break;
        uint8_t* st = ring + (size_t)slot * SB;
        uint8_t* X = st + Gm::kA;
        uint8_t* C = X + p.N * 128;
        if (k == 0) {
          mbar_arrive_expect_tx(&full[slot], (uint32_t)(p.N * 128));
          tma_load_2d(X, &p.tm_x, &full[slot], p.n_in + g0, b0);
        } else {
          const int g = g0 + k - 1;
          mbar_arrive_expect_tx(&full[slot], (uint32_t)(p.N * 128 + kBM * Gm::kCodeBytes));
          tma_load_2d(C, &p.tm_codes, &full[slot], g * Gm::kCodeBytes, row0);
          tma_load_2d(X, &p.tm_x, &full[slot], g * 64, b0);
        }
      }
      // copies still in flight land before the CTA may leave
      mbar_wait(pre, 0, p.status, 81);
      for (int q = max(0, k - ST); q < k; ++q) mbar_wait(&full[q % ST], (q / ST) & 1, p.status, 82);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(kBM, p.N);
      for (int k = 0; k < nst; ++k) {
        const int slot = k % ST, ph = (k / ST) & 1;
        if (!mbar_wait_sleep(&full[slot], ph, p.status, 83) || !mbar_wait_sleep(&afull[slot], ph, p.status, 84)) break;
        tc_fence_after();
        const uint32_t a = smem_u32(ring + (size_t)slot * SB);
        const uint32_t x = a + Gm::kA;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(tmem, sw128_desc(a + 32 * kk), sw128_desc(x + 32 * kk), idesc, (k | kk) != 0);
        mma_commit(&empty[slot]);
      }
      mma_commit(accb);  // also when stopped early: arrives once the issued MMAs are done
      mbar_wait(accb, 0, p.status, 85);
    }
    __syncwarp();
  } else {
    // ---------------- dequant, then epilogue (256 threads: row m, half h of each group)
    const int t = tid - 64, m = t & (kBM - 1), h = t >> 7;
    const int sw = m & 7;
    // lane 0 of each warp waits and the warp meets it at __syncwarp, which orders the
    // landed tile before the other lanes' reads (a few pollers, not 256, on each barrier)
    auto warp_wait = [&](uint64_t* bar, uint32_t ph, int where) -> bool {
      int w = 1;
      if (lane == 0) w = mbar_wait_sleep(bar, ph, p.status, where);
      return __shfl_sync(0xffffffffu, w, 0) != 0;
    };
    // the output block's coefficients, for the fused epilogue: loaded now, so that their
    // latency hides under the ring's first copies
    if (p.fuse) stage_out_coefs(p, cf_s, tile / p.H, t);
    bool ok = warp_wait(pre, 0, 86);
    for (int k = 0; ok && k < nst; ++k) {
      const int slot = k % ST, ph = (k / ST) & 1;
      if (!warp_wait(&full[slot], ph, 87)) {
        ok = false;
        break;
      }
      uint8_t* st = ring + (size_t)slot * SB;
      uint8_t* arow = st + (m >> 3) * 1024 + sw * 128;
      if (k == 0) {
        // zero block: column j < ngs holds m of group g0 + j, the rest 0
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j0 = 32 * h + 8 * c + 2 * e;
            const uint32_t lo = j0 < ngs ? (sz_s[m * p.gs + j0] >> 16) : 0u;
            const uint32_t hi = j0 + 1 < ngs ? (sz_s[m * p.gs + j0 + 1] >> 16) : 0u;
            o[e] = lo | (hi << 16);
          }
          st_shared_v4(arow + (((4 * h + c) ^ sw) << 4), o[0], o[1], o[2], o[3]);
        }
      } else {
        const int gl = k - 1;
        const uint32_t szw = sz_s[m * p.gs + gl];
        const __half s = __ushort_as_half((unsigned short)(szw & 0xffffu));
        const __half2 s2 = __half2half2(s);
        const bool fast = fabsf(__half2float(s)) < 32.f;
        const __half2 c2 = __half2half2(fast ? __hmul(s, __float2half(-1024.f)) : __float2half(0.f));
        const uint8_t* C = st + Gm::kA + p.N * 128;
        if (BITS == 4) {
          const uint4 cw = *reinterpret_cast<const uint4*>(C + m * 32 + 16 * h);
          const uint32_t wv[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              o[i] = scale_pair(((wv[u] >> (4 * i)) & 0x000F000Fu) | 0x64006400u, s2, c2, fast);
            st_shared_v4(arow + (((4 * h + u) ^ sw) << 4), o[0], o[1], o[2], o[3]);
          }
        } else {
          const uint2 cw = *reinterpret_cast<const uint2*>(C + m * 16 + 8 * h);
          uint32_t hw = 0;
          if (BITS == 3) hw = reinterpret_cast<const uint32_t*>(hi_s + (m * p.gs + gl) * 8)[h];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const uint32_t w = u ? cw.y : cw.x;
            // hi bits of codes 16u+i and 16u+8+i moved to bits i and 16+i, then up by 2
            const uint32_t y2 = BITS == 3 ? (__byte_perm(hw, 0u, u ? 0x4342u : 0x4140u) << 2) : 0u;
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              uint32_t tq = ((w >> (2 * i)) & 0x00030003u) | 0x64006400u;
              if (BITS == 3) tq |= (y2 >> i) & 0x00040004u;
              o[i] = scale_pair(tq, s2, c2, fast);
            }
            st_shared_v4(arow + (((4 * h + 2 * u) ^ sw) << 4), o[0], o[1], o[2], o[3]);
            st_shared_v4(arow + (((4 * h + 2 * u + 1) ^ sw) << 4), o[4], o[5], o[6], o[7]);
          }
        }
      }
      fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[slot]);
    }
    // ---------------- epilogue: accumulator lanes 32 (warp % 4) .. +31, half of the columns
    if (ok && warp_wait(accb, 0, 88)) {
      tc_fence_after();
      const int q = warp & 3, ch = (warp - 2) >> 2;
      const int r = row0 + 32 * q + lane;
      const int half = p.N >> 1;
      float* zp = p.zpart + (int64_t)split * p.batch * p.n_out;
      float* ptile = reinterpret_cast<float*>(ring);  // fused: [N][128] in the idle ring
      for (int c0 = ch * half; c0 < (ch + 1) * half; c0 += 8) {
        float v[8];
        tmem_ld8(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int b = b0 + c0 + j;
          if (p.fuse)
            ptile[(c0 + j) * kBM + 32 * q + lane] = b < p.batch ? v[j] * p.rowscale[b] : 0.f;
          else if (b < p.batch && r < p.n_out)
            zp[(int64_t)b * p.n_out + r] = v[j] * p.rowscale[b];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, (uint32_t)p.ncols);
  }
  if (p.fuse) {
    if (p.w_out == 256) fused_epilogue<256>(p, reinterpret_cast<const float*>(ring), cf_s, tile, b0);
    else fused_epilogue<128>(p, reinterpret_cast<const float*>(ring), cf_s, tile, b0);
  }
}

// ------------------------------------------------------------------ fp16 operand prep
// One CTA of 1024 threads per token row: max |v| -> scale 2^e with max |v| 2^e in
// [256, 512) (so the group sums stay below 2^15), then the scaled values in pair order and
// the group sums. Each warp owns whole groups of 64 and keeps them in registers between
// the two passes (16 groups per warp, 32768 inputs; wider rows re-read the rest).
constexpr int kPrepThreads = 1024;
constexpr int kPrepGroupsPerWarp = 16;

template <int BITS>
__global__ void __launch_bounds__(kPrepThreads) x16_prep_kernel(const float* __restrict__ xt, int n_in, int64_t ld,
                                                                __half* __restrict__ x16, float* __restrict__ rowscale) {
  __shared__ float red[kPrepThreads / 32];
  __shared__ int bad_s;
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = kPrepThreads / 32;
  const float* x = xt + (int64_t)b * n_in;
  const int G = n_in / 64;
  float2 v[kPrepGroupsPerWarp];
  float amax = 0.f;
  int bad = 0;
#pragma unroll
  for (int i = 0; i < kPrepGroupsPerWarp; ++i) {
    const int g = warp + i * NW;
    v[i] = g < G ? *reinterpret_cast<const float2*>(x + g * 64 + 2 * lane) : make_float2(0.f, 0.f);
    bad |= !(isfinite(v[i].x) && isfinite(v[i].y));
    amax = fmaxf(amax, fmaxf(fabsf(v[i].x), fabsf(v[i].y)));
  }
  for (int g = warp + kPrepGroupsPerWarp * NW; g < G; g += NW) {  // rows wider than the cache
    const float2 t = *reinterpret_cast<const float2*>(x + g * 64 + 2 * lane);
    bad |= !(isfinite(t.x) && isfinite(t.y));
    amax = fmaxf(amax, fmaxf(fabsf(t.x), fabsf(t.y)));
  }
  bad = __any_sync(0xffffffffu, bad);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (tid == 0) bad_s = 0;
  __syncthreads();
  if (lane == 0) {
    red[warp] = amax;
    if (bad) bad_s = 1;
  }
  __syncthreads();
  amax = red[0];
  for (int i = 1; i < NW; ++i) amax = fmaxf(amax, red[i]);
  int e = 0;
  if (amax > 0.f) {
    const int field = (int)((__float_as_uint(amax) >> 23) & 0xffu);
    const int E = field == 0 ? -127 : field - 127;  // amax in [2^E, 2^(E+1))
    e = min(max(8 - E, -126), 126);
  }
  const float sc = pow2f(e);
  __half* out = x16 + (int64_t)b * ld;
  for (int i = 0;; ++i) {
    const int g = warp + i * NW;
    if (g >= G) break;
    float2 t;
    if (i < kPrepGroupsPerWarp) {
#pragma unroll
      for (int k = 0; k < kPrepGroupsPerWarp; ++k)
        if (k == i) t = v[k];
    } else {
      t = *reinterpret_cast<const float2*>(x + g * 64 + 2 * lane);
    }
    const float v0 = t.x * sc, v1 = t.y * sc;
    float s = v0 + v1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const int jj[2] = {2 * lane, 2 * lane + 1};
    const float vv[2] = {v0, v1};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int j = jj[k];
      int pos;
      if (BITS == 4) {
        const int c = j >> 3, q = j & 7;
        pos = 8 * c + (q < 4 ? 2 * q : 2 * (q - 4) + 1);
      } else {
        const int c = j >> 4, q = j & 15;
        pos = 16 * c + (q < 8 ? 2 * q : 2 * (q - 8) + 1);
      }
      out[g * 64 + pos] = __float2half_rn(vv[k]);
    }
    if (lane == 0) out[n_in + g] = __float2half_rn(s);
  }
  for (int64_t j = n_in + G + tid; j < ld; j += kPrepThreads) out[j] = __float2half_rn(0.f);
  if (tid == 0) rowscale[b] = bad_s ? __int_as_float(0x7fc00000) : pow2f(-e);
}

}  // namespace

int64_t x16_ld(int64_t n_in) { return n_in + ((n_in / 64 + 63) / 64) * 64; }

Split choose_split(int64_t n_out, int64_t n_in, int bits) {
  const int tiles = (int)((n_out + kBM - 1) / kBM);
  const int G = (int)(n_in / 64);
  const int gmax = bits == 3 ? 32 : kMaxGs;  // the 1-bit plane box holds 8 bytes per group
  // gs is a multiple of 8 so that every split's first group sum (fp16 column n_in + g0)
  // starts a TMA box on a 16-byte boundary
  auto fit = [&](int s) {
    int gs = (G + s - 1) / s;
    gs = std::min(gmax, std::max(8, (gs + 7) / 8 * 8));
    return Split{(G + gs - 1) / gs, gs};
  };
  if (const char* e = getenv("HARP_MMA_SPLITS")) return fit(std::max(1, atoi(e)));  // tuning: a fixed request
  // About one CTA per SM, and no split of 32 or 64 groups, which measured slow on B200:
  // 7B gate/up ran 3 splits of 24 groups in 50.9 us per call at 16 tokens against 66.5 us
  // with 2 of 32, and down (4096 x 11008) 5 of 40 in 47.0 us against 69.2 us with 6 of 32.
  // The cause is not known: the scale/zero reads' bank conflicts at those widths were
  // ruled out (a tile transposed to group-major changed nothing).
  const int s0 = std::max(1, (148 + tiles - 1) / tiles);
  const char* m = getenv("HARP_MMA_SPLIT_MODEL");
  const Split base = fit(s0);
  if ((m && atoi(m) == 0) || base.gs % 32 != 0) return base;
  for (int s = s0 + 1; s <= G / 8; ++s) {  // at most one more wave of CTAs
    const Split c = fit(s);
    if ((int64_t)tiles * c.splits > (int64_t)tiles * base.splits + 148) break;
    if (c.gs % 32 != 0) return c;
  }
  return base;
}

cudaError_t launch_x16_prep(const float* xt, int64_t n_in, int bits, int batch, __half* x16, float* rowscale,
                            int* status, cudaStream_t st) {
  (void)status;
  const int64_t ld = x16_ld(n_in);
  if (bits == 4)
    x16_prep_kernel<4><<<batch, kPrepThreads, 0, st>>>(xt, (int)n_in, ld, x16, rowscale);
  else
    x16_prep_kernel<2><<<batch, kPrepThreads, 0, st>>>(xt, (int)n_in, ld, x16, rowscale);
  return cudaGetLastError();
}

// ring stages for N tokens within the opt-in shared memory (0: does not fit)
template <int BITS>
static int ring_stages(int N, int gs, bool fuse, int optin) {
  return std::min(kMaxStages, (optin - fixed_bytes<BITS>(gs, fuse)) / stage_bytes<BITS>(N));
}

static int optin_smem() {
  int dev = 0, optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  return optin;
}

template <int BITS>
static bool fuses_t(const Layer& L, int batch) {
  // opt-in (HARP_MMA_FUSE=1): measured slower than the separate output butterfly so far
  const char* e = getenv("HARP_MMA_FUSE");
  const bool on = e && atoi(e) != 0;
  if (!on || (L.w_out != 128 && L.w_out != 256) || (1 << L.m_out) != L.w_out || L.n_out % L.w_out != 0) return false;
  if ((L.w_out / kBM) * L.msplits > 8) return false;  // portable cluster size
  const int N = (std::min(batch, kMaxN) + 15) / 16 * 16;
  const int stages = ring_stages<BITS>(N, L.mgs, true, optin_smem());
  // the idle ring holds the N x 128 partial tile
  return stages >= 2 && (int64_t)stages * stage_bytes<BITS>(N) >= (int64_t)N * kBM * 4;
}

template <int BITS>
static cudaError_t launch_t(const Layer& L, const Call& c, cudaStream_t st) {
  Params p{};
  p.tm_codes = L.tm_mcodes;
  p.tm_sz = L.tm_msz;
  p.tm_hi = L.tm_mhi;
  p.n_out = (int)L.n_out;
  p.n_in = (int)L.n_in;
  p.G = (int)(L.n_in / 64);
  p.gs = L.mgs;
  p.batch = c.batch;
  const int n16 = (std::min(c.batch, kMaxN) + 15) / 16 * 16;
  p.N = n16;
  p.ncols = 32;
  while (p.ncols < p.N) p.ncols <<= 1;
  p.rowscale = c.rowscale;
  p.zpart = c.zpart;
  p.status = c.status;
  p.fuse = c.y && fuses_t<BITS>(L, c.batch);
  if (c.y && !p.fuse) return cudaErrorInvalidValue;  // the caller asked without checking fuses()
  p.H = L.w_out / kBM;
  p.w_out = L.w_out;
  p.m_out = L.m_out;
  p.sign = L.sU;
  p.cs = L.q8U ? nullptr : L.csU;
  p.q8 = L.q8U;
  p.y = c.y;
  p.yt = c.yt;
  p.y_stride = c.y_stride;

  int dev = 0, optin = 0, sm_smem = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  cudaDeviceGetAttribute(&sm_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  const int SB = stage_bytes<BITS>(p.N), FB = fixed_bytes<BITS>(p.gs, p.fuse);
  p.stages = ring_stages<BITS>(p.N, p.gs, p.fuse, optin);
  if (p.stages < 2) return cudaErrorInvalidConfiguration;
  int smem = FB + p.stages * SB;
  // tensor memory: CTAs resident on one SM must fit in its 512 columns
  const int max_ctas = 512 / p.ncols;
  const int per_cta_floor = sm_smem / (max_ctas + 1) + 1;  // more than this keeps <= max_ctas per SM
  if ((sm_smem / (smem + 1024)) > max_ctas) smem = std::max(smem, per_cta_floor);
  static bool attr_done[64] = {false};  // the attribute is per device; set it once each
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(mma_kernel<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }

  // operand tensor map: fp16 [batch][ld], box {64, N}, 128-byte swizzle
  if (!encode_map_2d(&p.tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, c.x16, (uint64_t)c.ld, (uint64_t)c.batch,
                     (uint64_t)c.ld * 2, 64, (uint32_t)p.N, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int tiles = (p.n_out + kBM - 1) / kBM;
  const int splits = (p.G + p.gs - 1) / p.gs;
  const int chunks = (c.batch + kMaxN - 1) / kMaxN;
  if (!p.fuse) {
    mma_kernel<BITS><<<dim3(tiles, splits, chunks), kThreads, smem, st>>>(p);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)tiles, (unsigned)splits, (unsigned)chunks);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.H;
  attr[0].val.clusterDim.y = (unsigned)splits;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mma_kernel<BITS>, p);
}

bool fuses(const Layer& L, int batch) {
  if (L.bits == 2) return fuses_t<2>(L, batch);
  if (L.bits == 3) return fuses_t<3>(L, batch);
  return fuses_t<4>(L, batch);
}

cudaError_t launch(const Layer& L, const Call& c, cudaStream_t st) {
  if (L.bits == 2) return launch_t<2>(L, c, st);
  if (L.bits == 3) return launch_t<3>(L, c, st);
  return launch_t<4>(L, c, st);
}

}  // namespace mma
}  // namespace harp
