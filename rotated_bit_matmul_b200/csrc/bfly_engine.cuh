// Butterfly engines of the sm_100a kernels: one w-wide block of the HARP butterfly
// ("HARP: Hadamard-Preconditioned Adaptive Rotation Processor for Extreme LLM
// Quantization", Sec. 2.1-2.2: signs, then stages of stride 1, 2, ..., w/2 of the 2x2 blocks
// [[cos p, sin p], [sin p, -cos p]], p = pi/4 + theta), on 512 cooperating threads of a CTA
// (LocalBfly, w <= 512) or of each CTA of a cluster of 8 (ClusterBfly, w = 8 E).
//
// Every thread holds one element (two when E = 1024). Stages of stride below 32 are warp
// shuffles; one transpose through shared memory makes the next five stride bits lane bits;
// in a cluster the last three stages (the CTA bits) follow one exchange in which every CTA
// stores its elements straight into the owners' shared memory with st.async, each store
// counting its bytes on the receiver's mbarrier. Each thread fetches the coefficients of
// its own rotations from the layer's tables (L2) before it starts.
//
// Used by the fused decode step (decode.cu) and the stand-alone forward butterfly
// (butterfly.cu). The 512 participating threads meet at named barrier 1.
#pragma once

#include "common.cuh"
#include "decode.h"

namespace harp {
namespace dec {

// ------------------------------------------------------------------ small device helpers
__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
// not the .aligned form: the producer warp reaches the final barrier at another time
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ uint32_t peer_addr(const void* local, uint32_t cta) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(cta));
  return ra;
}
// stores into CTA `cta`'s copy of `local_dst`; the receiver's copy of `local_bar` counts the bytes
__device__ __forceinline__ void st_async_f32(float* local_dst, uint64_t* local_bar, uint32_t cta, float v) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(
                   peer_addr(local_dst, cta)),
               "r"(__float_as_uint(v)), "r"(peer_addr(local_bar, cta))
               : "memory");
}
__device__ __forceinline__ void st_async_v4(void* local_dst, uint64_t* local_bar, uint32_t cta, int4 v) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   peer_addr(local_dst, cta)),
               "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(peer_addr(local_bar, cta))
               : "memory");
}
__device__ __forceinline__ bool try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool aborted(const int* status) { return *(volatile const int*)status != 0; }

// Wait bounds are counted in SM clock cycles (clock64 is cheap to read, the global
// timer is not): by default 4e9 cycles, about 2 s at the B200's top clock, longer when
// slower. The launch sets it (Params::wait_cycles) into this CTA-wide copy.
__shared__ long long s_wait_cycles;
constexpr long long kAbortCheckCycles = 40000;  // start reading the shared abort word after ~20 us

// bounded wait on a local mbarrier phase; false on time-out, or on abort when ABORT.
// SLEEP (the producer warp) backs off between polls so that a waiting producer leaves
// its issue slots to the consumer warps sharing its scheduler.
template <bool CLUSTER, bool SLEEP = false, bool ABORT = true>
__device__ __noinline__ bool wait_phase(uint64_t* bar, uint32_t parity, int* status, int where) {
  if (CLUSTER ? try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    for (int i = 0; i < (SLEEP ? 4 : 64); ++i) {
      if (CLUSTER ? try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
      if (SLEEP) __nanosleep(128);
    }
    const long long dt = clock64() - t0;
    if (ABORT && dt > kAbortCheckCycles && aborted(status)) return false;
    if (dt > s_wait_cycles) {
      report(status, 5, where);
      return false;
    }
  }
}

__device__ __forceinline__ void cbar() { asm volatile("bar.sync 1, %0;" ::"r"(kNT) : "memory"); }

// barrier of the consumer threads that also ANDs a predicate across them: every wait
// that decides control flow is polled by one thread and its outcome made uniform here,
// so a time-out can never leave some consumer threads at a barrier the others have left
__device__ __forceinline__ bool cbar_and(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred q, p;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.and.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)v), "r"(kNT)
      : "memory");
  return out != 0;
}
// sum of an int over the consumer threads
__device__ __forceinline__ int cbar_sum(int v, int* scratch, int ct) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((ct & 31) == 0) scratch[ct >> 5] = v;
  cbar();
  int t = 0;
#pragma unroll
  for (int w = 0; w < kCW; ++w) t += scratch[w];
  cbar();
  return t;
}

// ------------------------------------------------------------------ engine context
constexpr int kRxFloats = 8 * (128 + 4);  // a layout-B vector of the widest chunk (runs of 128, padded)

// the shared-memory buffers and barriers the engines use (kRxFloats floats each; the two
// mbarriers initialised with count 1)
struct EngCtx {
  float* T;        // local transposes and operand staging
  float* rx[2];    // receive buffers of alternate exchanges
  uint64_t* xbar;  // [2]
};

// ------------------------------------------------------------------ cluster exchanges
// Exchange k (the same sequence in every CTA of the cluster) lands in rx[k & 1] and is
// counted on xbar[k & 1]. A CTA pushes exchange k + 1 only after it has read what
// exchange k delivered (xch_begin starts with a consumer barrier), and it can run at most
// one exchange ahead of any peer (completing exchange k needs every peer's exchange-k
// data), so exchange k + 2 never overwrites data a peer has not read.
struct Xch {
  uint32_t k = 0;
};

__device__ __forceinline__ uint32_t xb_of(const Xch& x) { return x.k & 1; }

// opens exchange x.k: this CTA will receive rx_bytes from its peers
__device__ __forceinline__ void xch_begin(EngCtx& s, const Xch& x, uint32_t rx_bytes, int ct) {
  cbar();
  if (ct == 0) mbar_arrive_expect_tx(&s.xbar[xb_of(x)], rx_bytes);
}

__device__ __forceinline__ bool xch_end(EngCtx& s, Xch& x, int* status, int where, int ct) {
  bool mine = true;
  if (ct == 0) mine = wait_phase<true>(&s.xbar[xb_of(x)], (x.k >> 1) & 1, status, where);
  ++x.k;
  return cbar_and(mine);
}

// a float for element slot `idx` of CTA `dst`'s receive buffer of this exchange
__device__ __forceinline__ void put(EngCtx& s, const Xch& x, uint32_t me, uint32_t dst, int idx, float v) {
  float* buf = s.rx[xb_of(x)] + idx;
  if (dst == me) *buf = v;
  else st_async_f32(buf, &s.xbar[xb_of(x)], dst, v);
}

// ------------------------------------------------------------------ element maps
// A butterfly whose CTA share is E = 2^EB elements (a w = 8E wide block spread over the
// cluster, or a whole block of w = E in one CTA):
//   phase 1: thread ct holds e = s * 512 + ct: stages 0..4 pair lanes (shuffles);
//   phase 2: after a transpose, lane bits 0..L2-1 hold e bits 5..5+L2-1, so stages 5..EB-1
//            pair lanes again; e bits 0..4 come from the remaining lane bits, the warp
//            and the slot s;
//   layout B (cluster butterflies): CTA r holds, for every CTA index j, the run
//            [j E + r run, +run), run = E/8: thread ct holds j = lane & 7 and the offset
//            ii = (lane >> 3) | (warp << 2) | (s << 6), so the three cross-CTA stages pair
//            lanes 1, 2 and 4 apart.
// s < P = max(1, E / 512) slots per thread; threads from min(E, 512) on hold nothing.
template <int EB>
struct Map {
  static constexpr int E = 1 << EB;
  static constexpr int P = E > kNT ? E / kNT : 1;
  static constexpr int NT = E < kNT ? E : kNT;
  static constexpr int L2 = EB - 5 < 5 ? EB - 5 : 5;
  static constexpr int RUN = E / kC;
  static constexpr int RB = EB - 3;
  static constexpr int PAD = RUN + 4;  // run stride in the layout-B buffer: a warp's reads hit 32 banks
  __device__ static int e1(int ct, int s) { return s * kNT + ct; }
  __device__ static int e2(int ct, int s) {
    if constexpr (EB <= 5) {
      return e1(ct, s);
    } else {
      const int lane = ct & 31, warp = ct >> 5;
      return ((lane & ((1 << L2) - 1)) << 5) | (((lane >> L2) | (warp << (5 - L2)) | (s << (9 - L2))) & 31);
    }
  }
  __device__ static int bj(int ct) { return ct & 7; }
  __device__ static int bii(int ct, int s) { return ((ct & 31) >> 3) | ((ct >> 5) << 2) | (s << 6); }
  __device__ static int idx_b(int j, int ii) { return j * PAD + ii; }
};

// the lane bit a stage pairs on: t in phase 1, t - 5 in phase 2, t - EB across the cluster
__device__ __forceinline__ int stage_lane_bit(int EB, int t) { return t < (EB < 5 ? EB : 5) ? t : (t < EB ? t - 5 : t - EB); }
// the lane with bit b removed (4 bits) / a 4-bit value with a zero inserted at bit b
__device__ __forceinline__ int rm_bit(int x, int b) { return ((x >> (b + 1)) << b) | (x & ((1 << b) - 1)); }
__device__ __forceinline__ int ins0(int x, int b) { return ((x >> b) << (b + 1)) | (x & ((1 << b) - 1)); }
// Thread-order coefficient tables: for every stage the two lanes of a pair share one slot,
// (warp << 4) | (lane without the stage's lane bit), so a warp reads 16 consecutive entries.
// Layout [block][cta r][stage t][slot s][NT/2 slots]; entries are (cos, sin) float2, or the
// angle pi/4 + delta_t q as a float for int8 layers.
__device__ __forceinline__ int stage_slot(int EB, int t, int ct) {
  return ((ct >> 5) << 4) | rm_bit(ct & 31, stage_lane_bit(EB, t));
}

// layout-A buffer index: xor swizzle keeps a warp's phase-1 and phase-2 accesses on
// (nearly) distinct banks
__device__ __forceinline__ int idx_a(int e) { return e ^ ((e >> 5) & 31); }

// pair number of element g in stage t (pairs numbered by their first index)
__device__ __forceinline__ int64_t pair_of(int64_t g, int t) {
  return ((g >> (t + 1)) << t) | (g & ((int64_t(1) << t) - 1));
}

// ------------------------------------------------------------------ rotation coefficients
// What a thread keeps in registers per rotation: the (cos, sin) pair, the angle pi/4 +
// delta_t q of an int8 layer (decoded by the fast sine/cosine unit when the stage runs),
// or nothing for Theta == 0.
template <int TM>
struct Cf {
  float2 v;
};
template <>
struct Cf<kTmQ8> {
  float psi;
};
template <>
struct Cf<kTmHad> {};

constexpr float kQuarterPi = 0.785398163397448309616f;
constexpr float kRsqrt2 = 0.70710678118654752440f;  // cos(pi/4) = sin(pi/4): the Theta == 0 block

// tab: the side's angle storage (float2 [m][n/2], or int8 after a 64-byte head of steps)
template <int TM>
__device__ __forceinline__ Cf<TM> fetch_cf(const uint8_t* tab, int64_t half_n, int t, int64_t q) {
  Cf<TM> c;
  if constexpr (TM == kTmCS) {
    c.v = __ldg(reinterpret_cast<const float2*>(tab) + (int64_t)t * half_n + q);
  } else if constexpr (TM == kTmQ8) {
    const float step = __ldg(reinterpret_cast<const float*>(tab) + t);
    const int8_t code = __ldg(reinterpret_cast<const int8_t*>(tab + kQ8Head) + (int64_t)t * half_n + q);
    c.psi = fmaf(step, (float)code, kQuarterPi);
  }
  return c;
}

// one entry of a thread-order table (see stage_slot)
template <int TM>
__device__ __forceinline__ Cf<TM> fetch_rt(const uint8_t* rt, int64_t idx) {
  Cf<TM> c;
  if constexpr (TM == kTmCS) c.v = __ldg(reinterpret_cast<const float2*>(rt) + idx);
  else if constexpr (TM == kTmQ8) c.psi = __ldg(reinterpret_cast<const float*>(rt) + idx);
  return c;
}

template <int TM>
__device__ __forceinline__ float2 cs_of(const Cf<TM>& c) {
  if constexpr (TM == kTmCS) {
    return c.v;
  } else if constexpr (TM == kTmQ8) {
    float sn, co;
    __sincosf(c.psi, &sn, &co);
    return make_float2(co, sn);
  } else {
    return make_float2(kRsqrt2, kRsqrt2);
  }
}

// one 2x2 block [[c, s], [s, -c]] applied to the pair (a, b) held by two lanes: the lane
// holding a (upper = false) gets c a + s b, the lane holding b gets s a - c b
template <int TM>
__device__ __forceinline__ float rot_lane(float v, int lanes, bool upper, const Cf<TM>& cf) {
  const float p = __shfl_xor_sync(0xffffffffu, v, lanes);
  const float2 cs = cs_of<TM>(cf);
  return fmaf(upper ? -cs.x : cs.x, v, cs.y * p);
}

// ------------------------------------------------------------------ butterfly engines
// Cluster-distributed F(theta, s, w) over one w = 8E wide block (block `blk` of the side's
// n-vector). fetch() loads the thread's coefficients; run() takes the signed input in
// phase-1 order and leaves the output in layout B.
template <int EB, int TM>
struct ClusterBfly {
  using M = Map<EB>;
  static constexpr int NS = EB + 3;
  Cf<TM> cf[NS][M::P];

  __device__ __forceinline__ void fetch(const uint8_t* tab, int64_t half_n, int64_t blk, uint32_t r, int ct) {
    if constexpr (TM != kTmHad) {
      if (ct >= M::NT) return;
      const int64_t base = blk * (int64_t)(kC * M::E);
#pragma unroll
      for (int s = 0; s < M::P; ++s) {
        const int64_t g1 = base + (int64_t)r * M::E + M::e1(ct, s);
        const int64_t g2 = base + (int64_t)r * M::E + M::e2(ct, s);
        const int64_t gb = base + (int64_t)M::bj(ct) * M::E + (int64_t)r * M::RUN + M::bii(ct, s);
#pragma unroll
        for (int t = 0; t < NS; ++t)
          cf[t][s] = fetch_cf<TM>(tab, half_n, t, pair_of(t < 5 ? g1 : (t < EB ? g2 : gb), t));
      }
    }
  }

  // the same coefficients from a thread-order table (block blk of the side)
  __device__ __forceinline__ void fetch_rt(const uint8_t* rt, int64_t blk, uint32_t r, int ct) {
    if constexpr (TM != kTmHad) {
      if (ct >= M::NT) return;
      const int64_t base = (blk * kC + r) * (int64_t)NS;
#pragma unroll
      for (int t = 0; t < NS; ++t)
#pragma unroll
        for (int s = 0; s < M::P; ++s)
          cf[t][s] = dec::fetch_rt<TM>(rt, ((base + t) * M::P + s) * (M::NT / 2) + stage_slot(EB, t, ct));
    }
  }

  // v: this CTA's chunk in phase-1 order, signs applied. Returns with v in layout B.
  __device__ __forceinline__ bool run(float (&v)[2], EngCtx& sm, Xch& x, uint32_t r, int ct, int* status,
                                      int where) {
    const bool act = ct < M::NT;
    if (act) {
#pragma unroll
      for (int t = 0; t < (EB < 5 ? EB : 5); ++t)
#pragma unroll
        for (int s = 0; s < M::P; ++s) v[s] = rot_lane<TM>(v[s], 1 << t, (M::e1(ct, s) >> t) & 1, cf[t][s]);
    }
    if constexpr (EB > 5) {
      cbar();  // earlier readers of T are done
      if (act)
#pragma unroll
        for (int s = 0; s < M::P; ++s) sm.T[idx_a(M::e1(ct, s))] = v[s];
      cbar();
      if (act) {
#pragma unroll
        for (int s = 0; s < M::P; ++s) v[s] = sm.T[idx_a(M::e2(ct, s))];
#pragma unroll
        for (int t = 5; t < EB; ++t)
#pragma unroll
          for (int s = 0; s < M::P; ++s)
            v[s] = rot_lane<TM>(v[s], 1 << (t - 5), (M::e2(ct, s) >> t) & 1, cf[t][s]);
      }
    }
    // layout A -> B: element e goes to CTA e / run, slot (j = r, ii = e mod run)
    xch_begin(sm, x, 4u * M::RUN * (kC - 1), ct);
    if (act)
#pragma unroll
      for (int s = 0; s < M::P; ++s) {
        const int e = M::e2(ct, s);
        put(sm, x, r, (uint32_t)(e >> M::RB), M::idx_b((int)r, e & (M::RUN - 1)), v[s]);
      }
    const float* rx = sm.rx[xb_of(x)];
    const bool ok = xch_end(sm, x, status, where, ct);
    if (act) {
#pragma unroll
      for (int s = 0; s < M::P; ++s) v[s] = rx[M::idx_b(M::bj(ct), M::bii(ct, s))];
#pragma unroll
      for (int d = 0; d < 3; ++d)
#pragma unroll
        for (int s = 0; s < M::P; ++s) v[s] = rot_lane<TM>(v[s], 1 << d, (M::bj(ct) >> d) & 1, cf[EB + d][s]);
    }
    return ok;
  }

  // global (within the block) element index of slot s in layout B
  __device__ __forceinline__ static int gb(uint32_t r, int ct, int s) {
    return M::bj(ct) * M::E + (int)r * M::RUN + M::bii(ct, s);
  }
  __device__ __forceinline__ static int ga(uint32_t r, int ct, int s) { return (int)r * M::E + M::e1(ct, s); }
};

// A whole w = 2^EB block (EB <= 9) in one CTA: phase-1 input, phase-2 output.
template <int EB, int TM>
struct LocalBfly {
  using M = Map<EB>;
  Cf<TM> cf[EB];

  __device__ __forceinline__ void fetch(const uint8_t* tab, int64_t half_n, int64_t blk, int ct) {
    if constexpr (TM != kTmHad) {
      if (ct >= M::NT) return;
      const int64_t base = blk * (int64_t)M::E;
#pragma unroll
      for (int t = 0; t < EB; ++t)
        cf[t] = fetch_cf<TM>(tab, half_n, t, pair_of(base + (t < 5 ? M::e1(ct, 0) : M::e2(ct, 0)), t));
    }
  }

  __device__ __forceinline__ void fetch_rt(const uint8_t* rt, int64_t blk, int ct) {
    if constexpr (TM != kTmHad) {
      if (ct >= M::NT) return;
#pragma unroll
      for (int t = 0; t < EB; ++t)
        cf[t] = dec::fetch_rt<TM>(rt, (blk * EB + t) * (int64_t)(M::NT / 2) + stage_slot(EB, t, ct));
    }
  }

  __device__ __forceinline__ void run(float& v, EngCtx& sm, int ct) {
    const bool act = ct < M::NT;
    if (act)
#pragma unroll
      for (int t = 0; t < (EB < 5 ? EB : 5); ++t) v = rot_lane<TM>(v, 1 << t, (M::e1(ct, 0) >> t) & 1, cf[t]);
    if constexpr (EB > 5) {
      cbar();
      if (act) sm.T[idx_a(M::e1(ct, 0))] = v;
      cbar();
      if (act) {
        v = sm.T[idx_a(M::e2(ct, 0))];
#pragma unroll
        for (int t = 5; t < EB; ++t) v = rot_lane<TM>(v, 1 << (t - 5), (M::e2(ct, 0) >> t) & 1, cf[t]);
      }
    }
  }
};

// Builds a thread-order table for nblk blocks of a side (block width w = 8 * 2^EB spread
// over a cluster when cluster, else w = 2^EB in one CTA) from the layer's storage (tab:
// float2 (cos, sin) [m][n/2], or int8 after a 64-byte head of steps). One thread per entry.
template <int EB, int TM, bool CLUSTER>
__global__ void repack_kernel(const uint8_t* tab, int64_t half_n, int nblk, uint8_t* rt) {
  using M = Map<EB>;
  constexpr int NS = CLUSTER ? EB + 3 : EB, P = CLUSTER ? M::P : 1, NR = CLUSTER ? kC : 1, H = M::NT / 2;
  const int64_t total = (int64_t)nblk * NR * NS * P * H;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    int64_t k = i;
    const int slot = (int)(k % H);
    k /= H;
    const int s = (int)(k % P);
    k /= P;
    const int t = (int)(k % NS);
    k /= NS;
    const int r = (int)(k % NR);
    const int64_t blk = k / NR;
    const int b = stage_lane_bit(EB, t);
    const int ct = ((slot >> 4) << 5) | ins0(slot & 15, b);  // the lane of the pair with the bit clear
    int64_t g;
    if (t < (EB < 5 ? EB : 5)) g = (int64_t)r * M::E + M::e1(ct, s);
    else if (t < EB) g = (int64_t)r * M::E + M::e2(ct, s);
    else g = (int64_t)M::bj(ct) * M::E + (int64_t)r * M::RUN + M::bii(ct, s);
    const int64_t w = (int64_t)NR * M::E;
    const int64_t q = blk * (w >> 1) + pair_of(g, t);
    if constexpr (TM == kTmCS) {
      reinterpret_cast<float2*>(rt)[i] = reinterpret_cast<const float2*>(tab)[(int64_t)t * half_n + q];
    } else {
      const float step = reinterpret_cast<const float*>(tab)[t];
      const int8_t code = reinterpret_cast<const int8_t*>(tab + kQ8Head)[(int64_t)t * half_n + q];
      reinterpret_cast<float*>(rt)[i] = fmaf(step, (float)code, kQuarterPi);
    }
  }
}

}  // namespace dec
}  // namespace harp
