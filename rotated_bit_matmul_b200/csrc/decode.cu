// One batch-1 decode step through a whole Llama-shaped stack of rotated low-bit
// linears, in a single persistent kernel on sm_100a.
//
// The per-linear path launches three kernels per linear (input butterfly, GEMV,
// output butterfly) plus the glue; at batch 1 every launch is short and the
// launch/ramp/drain overheads dominate. Here one kernel does the whole step:
//
//  * Weights never depend on activations, so a producer warp per CTA streams that
//    CTA's share of every GEMV of the step, in order, with 2-D TMA tile loads (no
//    multicast) into a ring of shared-memory stages, while the activation chain runs.
//    A GEMV is cut into units of 32 output rows x one column chunk (split-K); each
//    unit's partial sums go to a buffer the next chain adds up in a fixed order. The
//    16 consumer warps form two halves that take alternate units, without any
//    CTA-wide barrier: the last warp of a half to finish a unit reduces it.
//  * CTAs form clusters of 8. Each cluster computes the activation chain between two
//    GEMVs itself (redundantly with the other clusters): a w-wide butterfly spread
//    over its 8 CTAs (w/8 elements each), local stages register-blocked (8 values per
//    thread, three stages per shared-memory round trip), the cross-CTA stages reached
//    by pushing data into the peers' shared memory and one cluster barrier (8
//    parallel release-arrives, acquire on the own barrier). A second producer warp
//    prefetches every chain's angle tables with bulk copies. The kernel is instantiated
//    per form of the angles (TM): (cos, sin) fp32 pairs, 8 bytes per rotation; int8
//    angles, 1 byte per rotation plus one step per stage, whose cos/sin are evaluated as
//    the rotation runs; or Theta == 0 everywhere (the fixed randomized Hadamard
//    transform), where the constant 1/sqrt 2 blocks need no table at all.
//  * Grid-wide barriers (release/acquire counters) only where a whole output vector
//    is needed: after q/k/v, o, gate/up, the MLP blocks, and down.
//
// Per block l (Sec. 2.1-2.2 and 5 of the HARP page for the butterflies; the glue is the
// stack definition of include/harp.h):
//   P1 chain: x_l = h_{l-1} + F_U_down(z_down)  (x_0 = input), rms, F_V of the cluster's
//             share of q/k/v, int16 GEMV operand, broadcast within the cluster
//   P2 GEMV q, k or v                           -> grid barrier
//   P3 chain: F_U_v(z_v), broadcast per KV group, F_V_o, operand
//   P4 GEMV o                                   -> grid barrier
//   P5 chain: h_l = x_l + F_U_o(z_o), rms, F_V of gate or up, operand
//   P6 GEMV gate or up                          -> grid barrier
//   P7 per MLP block (one CTA each): F_U_gate, F_U_up, silu*up, F_V_down, operand to
//      global; two otherwise idle clusters apply F_U_q and F_U_k of this block
//                                               -> grid barrier
//   P8 GEMV down                                -> grid barrier
// and after the last block: out = h_{L-1} + F_U_down(z_down).
//
// Every wait is bounded (about 2 s of SM clock) and checks a shared abort word, and every
// outcome that decides control flow is made uniform across the consumer threads, so a
// failure anywhere ends the kernel with HARP_ERR_TIMEOUT instead of a hang.
#include "decode.h"
#include "gemv_core.cuh"

namespace harp {
namespace dec {

using namespace gemv_core;

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
// not the .aligned form: the producer warps reach the final barrier at other times
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ uint32_t peer_addr(const void* local, uint32_t cta) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(cta));
  return ra;
}
__device__ __forceinline__ void st_peer4(void* local, uint32_t cta, float4 v) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(peer_addr(local, cta)), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_peer(void* local, uint32_t cta, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(peer_addr(local, cta)), "f"(v) : "memory");
}
__device__ __forceinline__ void arrive_remote(uint64_t* bar, uint32_t cta) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(peer_addr(bar, cta)) : "memory");
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

// bounded wait on a local mbarrier phase; false on time-out or abort. SLEEP (the
// producer warps) backs off between polls so that a waiting producer leaves its issue
// slots to the consumer warps sharing its scheduler.
template <bool CLUSTER, bool SLEEP = false>
__device__ __noinline__ bool wait_phase(uint64_t* bar, uint32_t parity, int* status, int where) {
  if (CLUSTER ? try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    for (int i = 0; i < (SLEEP ? 4 : 64); ++i) {
      if (CLUSTER ? try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
      if (SLEEP) __nanosleep(128);
    }
    const long long dt = clock64() - t0;
    if (dt > kAbortCheckCycles && aborted(status)) return false;
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

template <bool CLUSTER>
__device__ __forceinline__ bool wait_uniform(uint64_t* bar, uint32_t parity, int* status, int where, int ct) {
  bool mine = true;
  if (ct == 0) mine = wait_phase<CLUSTER>(bar, parity, status, where);
  return cbar_and(mine);
}

// ------------------------------------------------------------------ shared memory carve-up
constexpr int kSgnSlot = 1024;  // bytes per prefetched sign slice (>= the widest per-CTA chunk)

struct Smem {
  uint8_t* ring;
  uint8_t* tab;
  int8_t* sgn;  // 4 slots of kSgnSlot: the sign slices of the current chain's butterflies
  float *xa, *xb, *res, *ss, *red;
  int* ucnt;
  int32_t* xq;  // local GEMV operand: xq words, then xs [ng], then xsum [ng]
  uint64_t *full, *empty, *tab_full, *tab_empty, *xchg;
};

__device__ __forceinline__ Smem carve(const Params& p, int stage_bytes) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* b = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem s;
  s.ring = b;
  b += (size_t)p.ring_stages * stage_bytes;
  s.tab = b;
  b += p.tab_bytes;
  s.sgn = reinterpret_cast<int8_t*>(b);
  b += 4 * kSgnSlot;
  s.xa = reinterpret_cast<float*>(b);
  b += 4 * p.E;
  s.xb = reinterpret_cast<float*>(b);
  b += 4 * p.E;
  s.res = reinterpret_cast<float*>(b);
  b += 4 * p.E;
  s.ss = reinterpret_cast<float*>(b);
  b += 4 * 16;
  s.red = reinterpret_cast<float*>(b);
  b += (size_t)4 * kCW * 32 * p.ring_stages;
  s.ucnt = reinterpret_cast<int*>(b);
  b += 4 * ((p.ring_stages + 3) & ~3);
  s.xq = reinterpret_cast<int32_t*>(b);
  b += p.xq_bytes;
  s.full = reinterpret_cast<uint64_t*>(b);
  s.empty = s.full + p.ring_stages;
  s.tab_full = s.empty + p.ring_stages;
  s.tab_empty = s.tab_full + 1;
  s.xchg = s.tab_empty + 1;
  return s;
}

// ------------------------------------------------------------------ GEMV work units
// A unit is 32 output rows x one column chunk of one linear: exactly one ring stage.
struct Range {
  const Lin* L;
  float* zp;  // partial sums [nk][n_out]
  int nk, u0, u1;
};

__device__ __forceinline__ int split(int n, int i, int parts) { return (int)(((int64_t)n * i) / parts); }

// units of phase ph (0: q/k/v, 1: o, 2: gate/up, 3: down) of block l for CTA (c, r)
template <int BITS>
__device__ __forceinline__ Range units(const Params& p, int l, int ph, int c, int r) {
  const Lin* lin = p.lin + 7 * l;
  Range g;
  int i, parts;
  if (ph == 0 || ph == 2) {
    const int which = ph == 0 ? p.asg_qkv[c] : p.asg_gu[c];
    const int ci = ph == 0 ? p.idx_qkv[c] : p.idx_gu[c];
    const int nc = ph == 0 ? p.cnt_qkv[which] : p.cnt_gu[which];
    g.L = lin + (ph == 0 ? which : 4 + which);
    i = ci * kC + r;
    parts = nc * kC;
    if (ph == 0) {
      const int nk = p.nk_h;
      g.zp = which == 0 ? p.zpq + (int64_t)l * nk * g.L->n_out
                        : (which == 1 ? p.zpk + (int64_t)l * nk * g.L->n_out : p.zpv);
    } else {
      g.zp = which == 0 ? p.zpg : p.zpu;
    }
  } else {
    g.L = lin + (ph == 1 ? 3 : 6);
    i = c * kC + r;
    parts = p.G * kC;
    g.zp = ph == 1 ? p.zpo : p.zpd;
  }
  g.nk = (g.L->n_in + Geo<BITS>::kChunkCols - 1) / Geo<BITS>::kChunkCols;
  const int U = ((g.L->n_out + 31) / 32) * g.nk;
  g.u0 = split(U, i, parts);
  g.u1 = split(U, i + 1, parts);
  return g;
}

// Cursor over a CTA's units in consumer order (block, phase, unit), used to run the L2
// prefetch ahead of the ring.
struct UnitCursor {
  int l, ph, u;
  Range g;
  template <int BITS>
  __device__ __forceinline__ void normalize(const Params& p, int c, int r) {
    while (l < p.L && u >= g.u1) {
      if (++ph == 4) {
        ph = 0;
        ++l;
      }
      if (l >= p.L) return;
      g = units<BITS>(p, l, ph, c, r);
      u = g.u0;
    }
  }
  template <int BITS>
  __device__ __forceinline__ void next(const Params& p, int c, int r) {
    ++u;
    normalize<BITS>(p, c, r);
  }
};

// the boxes of one unit, as the ring loads them, requested into L2
template <int BITS>
__device__ __forceinline__ void prefetch_unit(const Range& g, int u) {
  using Gm = Geo<BITS>;
  const int ngroups = g.L->n_in / 64;
  const int tile = u / g.nk, kc = u - tile * g.nk;
  const int g0 = kc * Gm::kChunkGroups, gc = min(Gm::kChunkGroups, ngroups - g0);
  const int cslabs = (gc + Gm::kGroupsPerSlab - 1) / Gm::kGroupsPerSlab;
  const int code_x0 = g0 * (BITS == 4 ? 32 : 16) / 8;
  for (int q = 0; q < cslabs; ++q) tma_prefetch_l2_2d(&g.L->tm_codes, code_x0 + q * 16, tile * 32);
  if (BITS == 3)
    for (int q = 0; q < (gc + 15) / 16; ++q) tma_prefetch_l2_2d(&g.L->tm_hi, g0 + q * 16, tile * 32);
  for (int q = 0; q < (gc + 31) / 32; ++q) tma_prefetch_l2_2d(&g.L->tm_sz, g0 + q * 32, tile * 32);
}

// ------------------------------------------------------------------ table loads (producer warp 1)
// Table of one butterfly in shared memory: stage t holds the (cos, sin) pairs of the
// CTA's rotations in stage order, E/2 entries of 8 bytes. fp32 tables are copied as they
// are; int8 angles are expanded into pairs by the producer warp as it stages them, so the
// activation chains read the same table format whatever the layer keeps in memory.
template <int TM>
__device__ __forceinline__ constexpr int tab_esz() { return 8; }
template <int TM>
__device__ __forceinline__ constexpr int tab_head() { return 0; }

template <int TM>
__device__ __forceinline__ uint32_t table_bytes_cluster(int w, int m) {
  return (uint32_t)(tab_head<TM>() + tab_esz<TM>() * m * (w / kC / 2));
}
template <int TM>
__device__ __forceinline__ uint32_t table_bytes_local(int w, int m) {
  return (uint32_t)(tab_head<TM>() + tab_esz<TM>() * m * (w / 2));
}
// bytes a table load transfers by bulk copy (fp32 tables only: none for Theta == 0, and
// int8 angles are expanded by the warp's own loads)
template <int TM>
__device__ __forceinline__ uint32_t copied_bytes_cluster(const uint8_t* src, int w, int m) {
  return TM != kTmCS || !src ? 0u : table_bytes_cluster<TM>(w, m);
}
template <int TM>
__device__ __forceinline__ uint32_t copied_bytes_local(const uint8_t* src, int w, int m) {
  return TM != kTmCS || !src ? 0u : table_bytes_local<TM>(w, m);
}

// pair index, in the stage's full row, of entry q of the CTA's slice of a
// cluster-distributed stage t (the order load_table_cluster copies them in)
__device__ __forceinline__ int64_t slice_pair(int t, int q, int E, int e, int r) {
  if (t < e) return (int64_t)r * (E >> 1) + q;
  const int run = E / kC, dd = t - e, jj = q / run, ii = q - jj * run;
  const int j = ((jj >> dd) << (dd + 1)) | (jj & ((1 << dd) - 1));
  return (int64_t)(j >> (dd + 1)) * (1 << t) + (int64_t)E * (j & ((1 << dd) - 1)) + (int64_t)r * run + ii;
}

// int8 angles -> (cos, sin) of pi/4 + delta_t q for the CTA's slice (all 32 lanes of the
// producer warp; the fast sine/cosine unit, about 5e-7 absolute error near pi/4)
__device__ __noinline__ void expand_cluster(uint8_t* dst, const uint8_t* q8, int64_t n, int w, int m, int r,
                                            int lane) {
  if (!q8) return;
  const int E = w / kC, e = m - 3;
  const int64_t half_n = n >> 1;
  const float* steps = reinterpret_cast<const float*>(q8);
  const int8_t* codes = reinterpret_cast<const int8_t*>(q8 + kQ8Head);
  float2* out = reinterpret_cast<float2*>(dst);
  for (int t = 0; t < m; ++t) {
    const float st = __ldg(steps + t);
    for (int q = lane; q < (E >> 1); q += 32) {
      float sn, cs;
      __sincosf(fmaf(st, (float)__ldg(codes + (int64_t)t * half_n + slice_pair(t, q, E, e, r)),
                     0.785398163397448309616f),
                &sn, &cs);
      out[(size_t)t * (E >> 1) + q] = make_float2(cs, sn);
    }
  }
}

// the same for block `blk` of width w held whole by one CTA
__device__ __noinline__ void expand_local(uint8_t* dst, const uint8_t* q8, int64_t n, int w, int m, int blk,
                                          int lane) {
  if (!q8) return;
  const float* steps = reinterpret_cast<const float*>(q8);
  const int8_t* codes = reinterpret_cast<const int8_t*>(q8 + kQ8Head);
  float2* out = reinterpret_cast<float2*>(dst);
  for (int t = 0; t < m; ++t) {
    const float st = __ldg(steps + t);
    for (int q = lane; q < (w >> 1); q += 32) {
      float sn, cs;
      __sincosf(fmaf(st, (float)__ldg(codes + (int64_t)t * (n >> 1) + (int64_t)blk * (w >> 1) + q),
                     0.785398163397448309616f),
                &sn, &cs);
      out[(size_t)t * (w >> 1) + q] = make_float2(cs, sn);
    }
  }
}

// Per-CTA slice of a cluster-distributed butterfly (width w, C = 8): stage t < e is the
// contiguous run of the CTA's chunk; stage t >= e is C/2 runs of `run` pairs.
template <int TM>
__device__ __forceinline__ uint32_t load_table_cluster(uint8_t* dst, const uint8_t* src, int64_t n, int w, int m,
                                                       int blk, int r, uint64_t* bar) {
  constexpr int esz = tab_esz<TM>(), head = tab_head<TM>();
  const int E = w / kC, e = m - 3, run = E / kC;
  const int64_t half_n = n >> 1;
  if (TM != kTmCS || !src) return table_bytes_cluster<TM>(w, m);  // nothing to copy, same layout
  if (head) bulk_g2s(dst, src, (uint32_t)head, bar);
  for (int t = 0; t < m; ++t) {
    const uint8_t* st = src + head + ((int64_t)t * half_n + (int64_t)blk * (w >> 1)) * esz;
    uint8_t* d = dst + head + (size_t)t * (E >> 1) * esz;
    if (t < e) {
      bulk_g2s(d, st + (int64_t)r * (E >> 1) * esz, (uint32_t)(esz * (E >> 1)), bar);
    } else {
      const int dd = t - e;
      for (int jj = 0; jj < (kC >> 1); ++jj) {
        const int j = ((jj >> dd) << (dd + 1)) | (jj & ((1 << dd) - 1));
        const int64_t pb = (int64_t)(j >> (dd + 1)) * (1 << t) + (int64_t)E * (j & ((1 << dd) - 1)) + (int64_t)r * run;
        bulk_g2s(d + (size_t)jj * run * esz, st + pb * esz, (uint32_t)(esz * run), bar);
      }
    }
  }
  return table_bytes_cluster<TM>(w, m);
}

// the whole block `blk` of width w held by one CTA: one run of w/2 pairs per stage
template <int TM>
__device__ __forceinline__ uint32_t load_table_local(uint8_t* dst, const uint8_t* src, int64_t n, int w, int m, int blk,
                                                     uint64_t* bar) {
  constexpr int esz = tab_esz<TM>(), head = tab_head<TM>();
  if (TM != kTmCS || !src) return table_bytes_local<TM>(w, m);
  if (head) bulk_g2s(dst, src, (uint32_t)head, bar);
  for (int t = 0; t < m; ++t)
    bulk_g2s(dst + head + (size_t)t * (w >> 1) * esz, src + head + ((int64_t)t * (n >> 1) + (int64_t)blk * (w >> 1)) * esz,
             (uint32_t)(esz * (w >> 1)), bar);
  return table_bytes_local<TM>(w, m);
}

// P7 roles: block CTAs, and the clusters applying F_U_q / F_U_k
__device__ __forceinline__ int qk_cluster(const Params& p, int which) { return p.G - 1 - which; }

// ------------------------------------------------------------------ butterfly stages
constexpr float kRsqrt2 = 0.70710678118654752440f;  // cos(pi/4) = sin(pi/4): the Theta == 0 block

// One stage's row of a table of E/2 entries per stage: (cos, sin) pairs, or int8 angles
// with the stage's step.
struct StageTab {
  const float2* cs;
  const int8_t* q8;
  float step;
};

template <int TM>
__device__ __forceinline__ StageTab stage_tab(const uint8_t* tab, int ts, int E) {
  StageTab r;
  r.cs = reinterpret_cast<const float2*>(tab) + (size_t)ts * (E >> 1);
  r.q8 = reinterpret_cast<const int8_t*>(tab + kQ8Head) + (size_t)ts * (E >> 1);
  r.step = TM == kTmQ8 ? reinterpret_cast<const float*>(tab)[ts] : 0.f;
  return r;
}

// (cos, sin) of rotation q of a stage. int8 angles take the fast sine/cosine unit:
// pi/4 + delta_t q lies within a few tenths of pi/4.
template <int TM>
__device__ __forceinline__ float2 coef(const StageTab& st, int q) {
  if (TM == kTmHad) return make_float2(kRsqrt2, kRsqrt2);
  if (TM == kTmCS) return st.cs[q];
  float s, c;
  __sincosf(fmaf(st.step, (float)st.q8[q], 0.785398163397448309616f), &s, &c);
  return make_float2(c, s);
}

__device__ __forceinline__ void rot(float& a, float& b, float2 cs) {
  const float x = a, y = b;
  a = fmaf(cs.x, x, cs.y * y);
  b = fmaf(cs.y, x, -cs.x * y);
}

// NS stages t .. t+NS-1 (pairs (i, i + 2^s)) on a buffer of E elements, 2^NS values per
// thread held in registers; table row s (E/2 pairs, pair numbered by first index).
// TM == kTmHad: every block is the Theta == 0 block [[1, 1], [1, -1]] / sqrt 2 (no table read).
template <int NS, int TM>
__device__ __forceinline__ void round_a(float* x, const uint8_t* tab, int t, int E, int ct) {
  constexpr int P = 1 << NS;
  const int nthr = E / P, h = 1 << t;
  if (ct < nthr) {
    const int base = ((ct >> t) << (t + NS)) | (ct & (h - 1));
    float v[P];
#pragma unroll
    for (int k = 0; k < P; ++k) v[k] = x[base + k * h];
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      const int ts = t + s, hs = 1 << ts;
      const StageTab st = stage_tab<TM>(tab, ts, E);
#pragma unroll
      for (int k = 0; k < P; ++k) {
        if (k & (1 << s)) continue;
        const int i = base + k * h;
        const int q = ((i >> (ts + 1)) << ts) | (i & (hs - 1));
        rot(v[k], v[k + (1 << s)], coef<TM>(st, q));
      }
    }
#pragma unroll
    for (int k = 0; k < P; ++k) x[base + k * h] = v[k];
  }
  cbar();
}

// layout-A stages t0 .. t1-1, three per shared-memory round
template <int TM>
__device__ __forceinline__ void stages_a(float* x, const uint8_t* tab, int t0, int t1, int E, int ct) {
  int t = t0;
  while (t1 - t >= 3) {
    round_a<3, TM>(x, tab, t, E, ct);
    t += 3;
  }
  if (t1 - t == 2) round_a<2, TM>(x, tab, t, E, ct);
  if (t1 - t == 1) round_a<1, TM>(x, tab, t, E, ct);
}

// the three layout-B stages (runs j and j + 2^d, same offset), one round: thread T holds
// the 8 values {j run + T}; table rows e, e+1, e+2 numbered jj run + T
template <int TM>
__device__ __forceinline__ void stages_b(float* x, const uint8_t* tab, int e, int E, int ct) {
  const int run = E / kC;
  if (ct < run) {
    float v[kC];
#pragma unroll
    for (int j = 0; j < kC; ++j) v[j] = x[j * run + ct];
#pragma unroll
    for (int d = 0; d < 3; ++d) {
      const StageTab st = stage_tab<TM>(tab, e + d, E);
#pragma unroll
      for (int j = 0; j < kC; ++j) {
        if (j & (1 << d)) continue;
        const int jj = ((j >> (d + 1)) << d) | (j & ((1 << d) - 1));
        rot(v[j], v[j + (1 << d)], coef<TM>(st, jj * run + ct));
      }
    }
#pragma unroll
    for (int j = 0; j < kC; ++j) x[j * run + ct] = v[j];
  }
  cbar();
}

// ------------------------------------------------------------------ cluster data movement
struct Xchg {
  uint32_t phase = 0;
};

// Cluster-wide exchange point among the consumer threads of the 8 CTAs: everything this
// CTA pushed into its peers before it is visible to them after it.
__device__ __forceinline__ bool exchange(Smem& s, Xchg& x, int ct, int* status, int where) {
  cbar();
  if (ct < kC) arrive_remote(s.xchg, (uint32_t)ct);
  bool mine = true;
  if (ct == 0) mine = wait_phase<true>(s.xchg, x.phase, status, where);
  x.phase ^= 1;
  return cbar_and(mine);
}

// layout A (own chunk) -> layout B: run q of my chunk goes to CTA q at offset r*run
__device__ void push_a_to_b(const float* src, float* dst, int E, uint32_t r, int ct) {
  const int run = E / kC;
  for (int v = ct; v < (E >> 2); v += kNT) {
    const int i = v * 4, q = i / run, ii = i - q * run;
    st_peer4(dst + r * run + ii, (uint32_t)q, *reinterpret_cast<const float4*>(src + i));
  }
}

// layout B -> layout A: my run j goes to CTA j at offset r*run
__device__ void push_b_to_a(const float* src, float* dst, int E, uint32_t r, int ct) {
  const int run = E / kC;
  for (int v = ct; v < (E >> 2); v += kNT) {
    const int L = v * 4, j = L / run, ii = L - j * run;
    st_peer4(dst + r * run + ii, (uint32_t)j, *reinterpret_cast<const float4*>(src + L));
  }
}

// global element index of local position L in layout B (width kC*E, CTA rank r)
__device__ __forceinline__ int gidx_b(int L, int E, uint32_t r) {
  const int run = E / kC, j = L / run, ii = L - j * run;
  return j * E + (int)r * run + ii;
}

// int16 GEMV operand of one group of 64 values (one warp); lane 0 writes xs and xsum
__device__ __forceinline__ void prep_group(const float* v, int bits, int16_t* grp, int16_t* grp_hi, float* xs,
                                           float* xsum, int lane) {
  const float v0 = v[2 * lane], v1 = v[2 * lane + 1];
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
  grp[xq_pos_lo(bits, 2 * lane)] = (int16_t)q0;
  grp[xq_pos_lo(bits, 2 * lane + 1)] = (int16_t)q1;
  if (bits == 3) {
    grp_hi[xq_pos_hi(2 * lane)] = (int16_t)q0;
    grp_hi[xq_pos_hi(2 * lane + 1)] = (int16_t)q1;
  }
  if (lane == 0) {
    *xs = bad ? __int_as_float(0x7fc00000) : pow2f(-ex);
    *xsum = bad ? __int_as_float(0x7fc00000) : sum;
  }
}

// operand of a hidden-wide input held in layout B: prep the CTA's own groups into its
// local operand buffer and push them into every peer's buffer, then exchange
__device__ __forceinline__ bool prep_and_broadcast(Smem& s, Xchg& X, const float* xb, int n_in, int bits, int E, uint32_t r, int ct,
                                   int* status) {
  const int ng = n_in / 64;
  int16_t* xq16 = reinterpret_cast<int16_t*>(s.xq);
  const int words = bits == 3 ? n_in : n_in / 2;
  float* xsA = reinterpret_cast<float*>(s.xq + words);
  float* xsumA = xsA + ng;
  const int warp = ct >> 5, lane = ct & 31, ngl = E >> 6;
  for (int gl = warp; gl < ngl; gl += kCW) {
    const int g = gidx_b(gl * 64, E, r) >> 6;
    prep_group(xb + gl * 64, bits, xq16 + (int64_t)g * 64, xq16 + n_in + (int64_t)g * 64, xsA + g, xsumA + g, lane);
  }
  cbar();
  // 8 float4 per group (16 with the 1-bit-plane order), to the 7 peers
  const int per = bits == 3 ? 16 : 8;
  for (int it = ct; it < ngl * per * kC; it += kNT) {
    const int q = it % kC, rest = it / kC, part = rest % per, gl = rest / per;
    if (q == (int)r) continue;
    const int g = gidx_b(gl * 64, E, r) >> 6;
    const int word = part < 8 ? g * 32 + part * 4 : n_in / 2 + g * 32 + (part - 8) * 4;
    st_peer4(s.xq + word, (uint32_t)q, *reinterpret_cast<const float4*>(s.xq + word));
  }
  for (int it = ct; it < ngl * kC; it += kNT) {
    const int q = it % kC, gl = it / kC;
    if (q == (int)r) continue;
    const int g = gidx_b(gl * 64, E, r) >> 6;
    st_peer(xsA + g, (uint32_t)q, xsA[g]);
    st_peer(xsumA + g, (uint32_t)q, xsumA[g]);
  }
  return exchange(s, X, ct, status, 40);
}

// sum of the split-K partials of element i (fixed order)
__device__ __forceinline__ float zsum(const float* zp, int nk, int n, int i) {
  float t = __ldcg(zp + i);
  for (int k = 1; k < nk; ++k) t += __ldcg(zp + (int64_t)k * n + i);
  return t;
}

// ------------------------------------------------------------------ chains (cluster-collective)
// residual chain: [res += F_U(z)] ; n = rms(res) ; x~ = F_V(n) ; operand
template <int TM>
__device__ __forceinline__ bool chain_residual(const Params& p, Smem& s, Xchg& X, const Lin* U, const float* zp, int nk,
                               const Lin* V, bool first, uint32_t r, int ct, const uint8_t* tabU,
                               const uint8_t* tabV) {
  const int W = p.hidden, E = p.E, e = p.m_hidden - 3;
  if (first) {
    for (int L = ct; L < E; L += kNT) s.res[L] = load_act(p.x_in, gidx_b(L, E, r), p.xt);
  } else {
    for (int i = ct; i < E; i += kNT) {
      const int gi = (int)r * E + i;
      s.xa[i] = zsum(zp, nk, W, gi) * (float)s.sgn[i];
    }
    cbar();
    stages_a<TM>(s.xa, tabU, 0, e, E, ct);
    push_a_to_b(s.xa, s.xb, E, r, ct);
    if (!exchange(s, X, ct, p.status, 41)) return false;
    stages_b<TM>(s.xb, tabU, e, E, ct);
    for (int L = ct; L < E; L += kNT) s.res[L] += s.xb[L];
  }
  if (!V) {
    cbar();
    return true;  // final step: no input butterfly
  }
  // sum of squares of this CTA's share (fixed-order tree) pushed to every peer's slot r,
  // together with the residual values each peer needs for its layout-A chunk
  float acc = 0.f;
  for (int L = ct; L < E; L += kNT) acc = fmaf(s.res[L], s.res[L], acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((ct & 31) == 0) s.red[ct >> 5] = acc;
  cbar();
  if (ct < kC) {
    float t = 0.f;
    for (int w = 0; w < kCW; ++w) t += s.red[w];
    st_peer(s.ss + r, (uint32_t)ct, t);
  }
  push_b_to_a(s.res, s.xa, E, r, ct);
  if (!exchange(s, X, ct, p.status, 42)) return false;
  float t = 0.f;
  for (int q = 0; q < kC; ++q) t += s.ss[q];
  const float inv = 1.0f / sqrtf(t / (float)W + p.eps);
  for (int i = ct; i < E; i += kNT) s.xa[i] *= inv * (float)s.sgn[kSgnSlot + i];
  cbar();
  stages_a<TM>(s.xa, tabV, 0, e, E, ct);
  push_a_to_b(s.xa, s.xb, E, r, ct);
  if (!exchange(s, X, ct, p.status, 43)) return false;
  stages_b<TM>(s.xb, tabV, e, E, ct);
  return prep_and_broadcast(s, X, s.xb, V->n_in, p.bits, E, r, ct, p.status);
}

// attention chain: v = F_U_v(z_v); a = v broadcast per KV group; x~ = F_V_o(a); operand
template <int TM>
__device__ __forceinline__ bool chain_attn(const Params& p, Smem& s, Xchg& X, const Lin* Lv, const Lin* Lo, uint32_t r, int ct,
                           const uint8_t* tabU, const uint8_t* tabV) {
  const int Wu = Lv->w_out, Eu = Wu / kC, eu = Lv->m_out - 3;

  for (int i = ct; i < Eu; i += kNT) {
    const int gi = (int)r * Eu + i;
    s.xa[i] = zsum(p.zpv, p.nk_h, Wu, gi) * (float)s.sgn[i];
  }
  cbar();
  stages_a<TM>(s.xa, tabU, 0, eu, Eu, ct);
  push_a_to_b(s.xa, s.xb, Eu, r, ct);
  if (!exchange(s, X, ct, p.status, 44)) return false;
  stages_b<TM>(s.xb, tabU, eu, Eu, ct);
  // push every v value to the layout-A owners of the query-head elements that copy it
  const int Eo = p.E, eo = p.m_hidden - 3, hd = p.head_dim, rep = p.rep;
  for (int L = ct; L < Eu; L += kNT) {
    const int gv = gidx_b(L, Eu, r), kvh = gv / hd, d = gv - kvh * hd;
    for (int h = kvh * rep; h < (kvh + 1) * rep; ++h) {
      const int ga = h * hd + d;
      st_peer(s.xa + (ga % Eo), (uint32_t)(ga / Eo), s.xb[L]);
    }
  }
  if (!exchange(s, X, ct, p.status, 45)) return false;
  for (int i = ct; i < Eo; i += kNT) s.xa[i] *= (float)s.sgn[kSgnSlot + i];
  cbar();
  stages_a<TM>(s.xa, tabV, 0, eo, Eo, ct);
  push_a_to_b(s.xa, s.xb, Eo, r, ct);
  if (!exchange(s, X, ct, p.status, 46)) return false;
  stages_b<TM>(s.xb, tabV, eo, Eo, ct);
  return prep_and_broadcast(s, X, s.xb, Lo->n_in, p.bits, Eo, r, ct, p.status);
}

// F_U of a q or k GEMV output (cluster-distributed), written to out[gidx]
template <int TM>
__device__ __forceinline__ bool chain_out_only(const Params& p, Smem& s, Xchg& X, const Lin* Lq, const float* zp, float* out,
                               uint32_t r, int ct, const uint8_t* tab) {
  const int W = Lq->w_out, E = W / kC, e = Lq->m_out - 3;

  for (int i = ct; i < E; i += kNT) {
    const int gi = (int)r * E + i;
    s.xa[i] = zsum(zp, p.nk_h, W, gi) * (float)s.sgn[i];
  }
  cbar();
  stages_a<TM>(s.xa, tab, 0, e, E, ct);
  push_a_to_b(s.xa, s.xb, E, r, ct);
  if (!exchange(s, X, ct, p.status, 47)) return false;
  stages_b<TM>(s.xb, tab, e, E, ct);
  for (int L = ct; L < E; L += kNT) out[gidx_b(L, E, r)] = s.xb[L];
  cbar();
  return true;
}

// one whole MLP block (width <= 512) in one CTA: F_U_gate, F_U_up, silu*up, F_V_down,
// operand of the down projection for this block (to global)
template <int TM>
__device__ __forceinline__ void block_chain(const Params& p, Smem& s, const Lin* Lg, const Lin* Lu, const Lin* Ld, int blk, int ct,
                            const uint8_t* tab) {
  const int wb = Lg->w_out, mb = Lg->m_out, F = p.ffn;
  const int base = blk * wb;
  for (int i = ct; i < wb; i += kNT) {
    s.xa[i] = zsum(p.zpg, p.nk_h, F, base + i) * (float)s.sgn[i];
    s.xb[i] = zsum(p.zpu, p.nk_h, F, base + i) * (float)s.sgn[kSgnSlot + i];
  }
  cbar();
  stages_a<TM>(s.xa, tab, 0, mb, wb, ct);
  stages_a<TM>(s.xb, tab + table_bytes_local<TM>(wb, mb), 0, mb, wb, ct);
  for (int i = ct; i < wb; i += kNT) {
    const float g = s.xa[i];
    s.xa[i] = g / (1.0f + expf(-g)) * s.xb[i] * (float)s.sgn[2 * kSgnSlot + i];
  }
  cbar();
  stages_a<TM>(s.xa, tab + 2 * table_bytes_local<TM>(wb, mb), 0, mb, wb, ct);
  const int n_in = Ld->n_in;
  int16_t* xq16 = reinterpret_cast<int16_t*>(p.xq_down);
  const int warp = ct >> 5, lane = ct & 31;
  for (int gl = warp; gl < (wb >> 6); gl += kCW) {
    const int g = (base >> 6) + gl;
    prep_group(s.xa + gl * 64, p.bits, xq16 + (int64_t)g * 64, xq16 + n_in + (int64_t)g * 64, p.xs_down + g,
               p.xsum_down + g, lane);
  }
  cbar();
}

// ------------------------------------------------------------------ GEMV (consumer side)
// The 16 consumer warps form two halves that take alternate units of the CTA's range,
// so two units are in flight and each warp covers 8 groups of a unit; the last warp of a
// half to finish a unit reduces its 8 per-warp partial rows and writes the unit's sums.
constexpr int kHalf = kCW / 2;

template <int BITS>
__device__ __forceinline__ bool run_units(const Params& p, Smem& s, const Range& g, uint32_t& kring, int ct) {
  using Gm = Geo<BITS>;
  const int warp = ct >> 5, lane = ct & 31;
  const int hv = warp / kHalf, hw = warp - hv * kHalf;  // half, warp within the half
  const int n_out = g.L->n_out, n_in = g.L->n_in, ngroups = n_in / 64;
  const int words = BITS == 3 ? n_in : n_in / 2;
  const float* xsA = reinterpret_cast<const float*>(s.xq + words);
  const float* xsumA = xsA + ngroups;
  const int nu = g.u1 - g.u0;
  bool ok = true;
  for (int i = hv; i < nu; i += 2) {
    const uint32_t kr = kring + (uint32_t)i;
    const int slot = kr % p.ring_stages;
    const int u = g.u0 + i;
    if (ok) {
      int w = 1;
      if (lane == 0) w = wait_phase<false>(&s.full[slot], (kr / p.ring_stages) & 1, p.status, 50);
      ok = __shfl_sync(0xffffffffu, w, 0) != 0;
    }
    const int tile = u / g.nk, kc = u - tile * g.nk, row0 = tile * 32;
    const int g0 = kc * Gm::kChunkGroups, gc = min(Gm::kChunkGroups, ngroups - g0);
    float zacc = 0.f;
    if (ok) {
      const uint8_t* st = s.ring + (size_t)slot * Gm::kStageBytes;
      const uint8_t* szs = st + (Gm::kCodeSlabs + Gm::kHiSlabs) * kSlab;
      for (int gl = hw; gl < gc; gl += kHalf) {
        const int gg = g0 + gl;
        const uint32_t szw = sz_word(szs, lane, gl);
        const float s16 = __half2float(__ushort_as_half((unsigned short)(szw & 0xffffu)));
        const float z16 = __half2float(__ushort_as_half((unsigned short)(szw >> 16)));
        const int4* xg = reinterpret_cast<const int4*>(s.xq + (int64_t)gg * 32);
        const int4* xgh = reinterpret_cast<const int4*>(s.xq + n_in / 2 + (int64_t)gg * 32);
        const int acc = group_dot<BITS, true>(st, st + Gm::kCodeSlabs * kSlab, lane, gl, xg, xgh);
        zacc = fmaf(s16, (float)acc * xsA[gg], fmaf(z16, xsumA[gg], zacc));
      }
    }
    float* red = s.red + (size_t)slot * kCW * 32;
    red[hw * 32 + lane] = zacc;
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      __threadfence_block();
      last = atomicAdd(&s.ucnt[slot], 1) == kHalf - 1;
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      __threadfence_block();
      float t = 0.f;
#pragma unroll
      for (int w = 0; w < kHalf; ++w) t += red[w * 32 + lane];
      if (ok && row0 + lane < n_out) g.zp[(int64_t)kc * n_out + row0 + lane] = t;
      __syncwarp();
      if (lane == 0) s.ucnt[slot] = 0;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[slot]);
  }
  kring += (uint32_t)nu;
  return cbar_and(ok);
}

// ------------------------------------------------------------------ grid barrier
__device__ __noinline__ bool grid_barrier(const Params& p, int idx, int ct) {
  cbar();
  bool mine = true;
  if (ct == 0) {
    unsigned* c = p.counters + idx;
    __threadfence();
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(c) : "memory");
    const unsigned target = (unsigned)(p.G * kC) + (idx == p.barrier_extra ? 1u : 0u);  // + testing hook
    const long long t0 = clock64();
    for (uint32_t it = 0;; ++it) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(c) : "memory");
      if (v >= target) break;
      if ((it & 15) == 15) {
        const long long dt = clock64() - t0;
        if (dt > kAbortCheckCycles && aborted(p.status)) {
          mine = false;
          break;
        }
        if (dt > s_wait_cycles) {
          report(p.status, 5, 60 + (idx % 5));
          mine = false;
          break;
        }
      }
    }
  }
  return cbar_and(mine);
}

// ------------------------------------------------------------------ the kernel
// TM: how every butterfly of the stack keeps its angles (kTmCS, kTmHad, kTmQ8); each form
// has its own instantiation, so no rotation round branches on it.
template <int BITS, int TM>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ Params p) {
  using Gm = Geo<BITS>;
  // the form the consumers read the staged tables in: int8 angles arrive expanded
  constexpr int TC = TM == kTmQ8 ? kTmCS : TM;
  Smem s = carve(p, Gm::kStageBytes);
  const uint32_t r = cta_rank();
  const int c = (int)cluster_id_x();
  const int tid = threadIdx.x;
  const int t_cta = c * kC + (int)r;

  if (tid == 0) {
    s_wait_cycles = p.wait_cycles;
    for (int i = 0; i < p.ring_stages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], kHalf);  // the 8 warps of the half that consumed the unit
      s.ucnt[i] = 0;
    }
    mbar_init(s.tab_full, 1);
    mbar_init(s.tab_empty, 1);
    mbar_init(s.xchg, kC);
    fence_mbar_init();
  }
  cluster_sync_all();  // every CTA's barriers exist before any remote arrive

  const int L = p.L;
  const int nblocks = p.ffn / p.lin[4].w_out;  // MLP blocks of the gate/up output side

  if (tid >= kNT) {
    // Two producer warps. Every lane of a producer warp runs the same loop (so the warp
    // never diverges around a blocking wait); lane 0 waits and issues, the others follow.
    const int pw = (tid - kNT) >> 5, lane = tid & 31;
    if (pw == 0) {
      // ---------------- weight ring: every unit of the step, in consumer order. A second
      // cursor runs p.pf_dist units ahead and asks for those units' boxes to be brought
      // into L2, so HBM keeps streaming while the activation chains run and the ring's
      // copies are served from L2.
      UnitCursor pf;
      pf.l = 0;
      pf.ph = 0;
      pf.g = units<BITS>(p, 0, 0, c, (int)r);
      pf.u = pf.g.u0;
      pf.normalize<BITS>(p, c, (int)r);
      if (lane == 0)
        for (int d = 0; d < p.pf_dist && pf.l < L; ++d) {
          prefetch_unit<BITS>(pf.g, pf.u);
          pf.next<BITS>(p, c, (int)r);
        }
      uint32_t k = 0;
      bool ok = true;
      for (int l = 0; l < L && ok; ++l)
        for (int ph = 0; ph < 4 && ok; ++ph) {
          const Range g = units<BITS>(p, l, ph, c, (int)r);
          const int ngroups = g.L->n_in / 64;
          for (int u = g.u0; u < g.u1; ++u) {
            const int slot = k % p.ring_stages;
            int go = 1;
            if (lane == 0 && pf.l < L) {
              prefetch_unit<BITS>(pf.g, pf.u);
              pf.next<BITS>(p, c, (int)r);
            }
            if (lane == 0) {
              if (k >= (uint32_t)p.ring_stages &&
                  !wait_phase<false, true>(&s.empty[slot], ((k / p.ring_stages) - 1) & 1, p.status, 51)) {
                go = 0;
              } else {
                const int tile = u / g.nk, kc = u - tile * g.nk;
                const int g0 = kc * Gm::kChunkGroups, gc = min(Gm::kChunkGroups, ngroups - g0);
                const int cslabs = (gc + Gm::kGroupsPerSlab - 1) / Gm::kGroupsPerSlab;
                const int hslabs = BITS == 3 ? (gc + 15) / 16 : 0;
                uint8_t* st = s.ring + (size_t)slot * Gm::kStageBytes;
                mbar_arrive_expect_tx(&s.full[slot], (uint32_t)((cslabs + hslabs + (gc + 31) / 32) * kSlab));
                const int code_x0 = g0 * (BITS == 4 ? 32 : 16) / 8;
                for (int q = 0; q < cslabs; ++q)
                  tma_load_2d(st + q * kSlab, &g.L->tm_codes, &s.full[slot], code_x0 + q * 16, tile * 32);
                if (BITS == 3)
                  for (int q = 0; q < hslabs; ++q)
                    tma_load_2d(st + (Gm::kCodeSlabs + q) * kSlab, &g.L->tm_hi, &s.full[slot], g0 + q * 16,
                                tile * 32);
                for (int q = 0; q < (gc + 31) / 32; ++q)
                  tma_load_2d(st + (Gm::kCodeSlabs + Gm::kHiSlabs + q) * kSlab, &g.L->tm_sz, &s.full[slot],
                              g0 + q * 32, tile * 32);
              }
            }
            ok = __shfl_sync(0xffffffffu, go, 0) != 0;
            if (!ok) break;
            ++k;  // k counts the stages issued so far
          }
        }
      // drain: wait for the copies still in flight before the CTA may exit
      if (lane == 0) {
        const uint32_t nwait = k < (uint32_t)p.ring_stages ? k : (uint32_t)p.ring_stages;
        for (uint32_t q = k - nwait; q < k; ++q)
          wait_phase<false, true>(&s.full[q % p.ring_stages], (q / p.ring_stages) & 1, p.status, 52);
      }
      __syncwarp();
    } else {
      // ---------------- tables: one set per chain slot, in consumer order
      uint32_t slot = 0;
      bool ok = true;
      // fp32 tables: the bulk copies' bytes complete the slot. int8 angles: the bytes
      // announced are the signs'; the warp expands the angles into (cos, sin) pairs, then
      // lane 0's arrival completes the slot together with those copies.
      auto announce = [&](uint32_t bytes) {
        if (TM == kTmQ8) mbar_expect_tx(s.tab_full, bytes);
        else mbar_arrive_expect_tx(s.tab_full, bytes);
      };
      auto finish = [&]() {
        if (TM == kTmQ8) {
          __syncwarp();
          if (lane == 0) mbar_arrive(s.tab_full);
        }
      };
      auto begin = [&]() -> bool {
        int go = 1;
        if (lane == 0 && slot > 0 && !wait_phase<false, true>(s.tab_empty, (slot - 1) & 1, p.status, 53)) go = 0;
        return __shfl_sync(0xffffffffu, go, 0) != 0;
      };
      for (int l = 0; l <= L && ok; ++l) {
        const Lin* lin = p.lin + 7 * l;
        const Lin* prev = l > 0 ? p.lin + 7 * (l - 1) : nullptr;
        // P1 (or the final step when l == L)
        if (!(ok = begin())) break;
        if (lane == 0) {
          uint32_t bytes = 0;
          if (prev) bytes += copied_bytes_cluster<TM>(prev[6].tU, prev[6].w_out, prev[6].m_out);
          const Lin* V = l < L ? lin + p.asg_qkv[c] : nullptr;
          if (V) bytes += copied_bytes_cluster<TM>(V->tV, V->w_in, V->m_in);
          const int Eh = p.E;
          if (prev) bytes += Eh;
          if (V) bytes += Eh;
          announce(bytes);
          uint32_t off = 0;
          if (prev)
            off += load_table_cluster<TM>(s.tab, prev[6].tU, prev[6].n_out, prev[6].w_out, prev[6].m_out, 0, (int)r,
                                      s.tab_full);
          if (V) load_table_cluster<TM>(s.tab + off, V->tV, V->n_in, V->w_in, V->m_in, 0, (int)r, s.tab_full);
          if (prev) bulk_g2s(s.sgn, prev[6].sU + (int64_t)r * Eh, (uint32_t)Eh, s.tab_full);
          if (V) bulk_g2s(s.sgn + kSgnSlot, V->sV + (int64_t)r * Eh, (uint32_t)Eh, s.tab_full);
        }
        if (TM == kTmQ8) {
          const Lin* V = l < L ? lin + p.asg_qkv[c] : nullptr;
          uint32_t off = 0;
          if (prev) {
            expand_cluster(s.tab, prev[6].tU, prev[6].n_out, prev[6].w_out, prev[6].m_out, (int)r, lane);
            off = table_bytes_cluster<TM>(prev[6].w_out, prev[6].m_out);
          }
          if (V) expand_cluster(s.tab + off, V->tV, V->n_in, V->w_in, V->m_in, (int)r, lane);
        }
        finish();
        ++slot;
        if (l == L) break;
        // P3
        if (!(ok = begin())) break;
        if (lane == 0) {
          const uint32_t b0 = table_bytes_cluster<TM>(lin[2].w_out, lin[2].m_out);
          const int Eu = lin[2].w_out / kC, Eo = lin[3].w_in / kC;
          announce(copied_bytes_cluster<TM>(lin[2].tU, lin[2].w_out, lin[2].m_out) +
                   copied_bytes_cluster<TM>(lin[3].tV, lin[3].w_in, lin[3].m_in) + Eu + Eo);
          load_table_cluster<TM>(s.tab, lin[2].tU, lin[2].n_out, lin[2].w_out, lin[2].m_out, 0, (int)r, s.tab_full);
          load_table_cluster<TM>(s.tab + b0, lin[3].tV, lin[3].n_in, lin[3].w_in, lin[3].m_in, 0, (int)r, s.tab_full);
          bulk_g2s(s.sgn, lin[2].sU + (int64_t)r * Eu, (uint32_t)Eu, s.tab_full);
          bulk_g2s(s.sgn + kSgnSlot, lin[3].sV + (int64_t)r * Eo, (uint32_t)Eo, s.tab_full);
        }
        if (TM == kTmQ8) {
          expand_cluster(s.tab, lin[2].tU, lin[2].n_out, lin[2].w_out, lin[2].m_out, (int)r, lane);
          expand_cluster(s.tab + table_bytes_cluster<TM>(lin[2].w_out, lin[2].m_out), lin[3].tV, lin[3].n_in,
                         lin[3].w_in, lin[3].m_in, (int)r, lane);
        }
        finish();
        ++slot;
        // P5
        if (!(ok = begin())) break;
        if (lane == 0) {
          const Lin* V = lin + 4 + p.asg_gu[c];
          const uint32_t b0 = table_bytes_cluster<TM>(lin[3].w_out, lin[3].m_out);
          const int Eh = p.E;
          announce(copied_bytes_cluster<TM>(lin[3].tU, lin[3].w_out, lin[3].m_out) +
                   copied_bytes_cluster<TM>(V->tV, V->w_in, V->m_in) + 2 * Eh);
          load_table_cluster<TM>(s.tab, lin[3].tU, lin[3].n_out, lin[3].w_out, lin[3].m_out, 0, (int)r, s.tab_full);
          load_table_cluster<TM>(s.tab + b0, V->tV, V->n_in, V->w_in, V->m_in, 0, (int)r, s.tab_full);
          bulk_g2s(s.sgn, lin[3].sU + (int64_t)r * Eh, (uint32_t)Eh, s.tab_full);
          bulk_g2s(s.sgn + kSgnSlot, V->sV + (int64_t)r * Eh, (uint32_t)Eh, s.tab_full);
        }
        if (TM == kTmQ8) {
          const Lin* V = lin + 4 + p.asg_gu[c];
          expand_cluster(s.tab, lin[3].tU, lin[3].n_out, lin[3].w_out, lin[3].m_out, (int)r, lane);
          expand_cluster(s.tab + table_bytes_cluster<TM>(lin[3].w_out, lin[3].m_out), V->tV, V->n_in, V->w_in,
                         V->m_in, (int)r, lane);
        }
        finish();
        ++slot;
        // P7: this CTA's MLP blocks, or F_U_q / F_U_k for the two q/k clusters
        if (!(ok = begin())) break;
        if (lane == 0) {
          uint32_t bytes = 0;
          const int wb = lin[4].w_out, mb = lin[4].m_out;
          const int blk = t_cta;  // at most one MLP block per CTA (checked at set-up)
          if (blk < nblocks)
            bytes += copied_bytes_local<TM>(lin[4].tU, wb, mb) + copied_bytes_local<TM>(lin[5].tU, wb, mb) +
                     copied_bytes_local<TM>(lin[6].tV, wb, mb) + 3 * wb;
          const int qk = c == qk_cluster(p, 0) ? 0 : (c == qk_cluster(p, 1) ? 1 : -1);
          const int Eq = qk >= 0 ? lin[qk].w_out / kC : 0;
          if (qk >= 0) bytes += copied_bytes_cluster<TM>(lin[qk].tU, lin[qk].w_out, lin[qk].m_out) + Eq;
          announce(bytes);
          if (blk < nblocks) {
            uint32_t off = 0;
            off += load_table_local<TM>(s.tab + off, lin[4].tU, lin[4].n_out, wb, mb, blk, s.tab_full);
            off += load_table_local<TM>(s.tab + off, lin[5].tU, lin[5].n_out, wb, mb, blk, s.tab_full);
            load_table_local<TM>(s.tab + off, lin[6].tV, lin[6].n_in, wb, mb, blk, s.tab_full);
            bulk_g2s(s.sgn, lin[4].sU + (int64_t)blk * wb, (uint32_t)wb, s.tab_full);
            bulk_g2s(s.sgn + kSgnSlot, lin[5].sU + (int64_t)blk * wb, (uint32_t)wb, s.tab_full);
            bulk_g2s(s.sgn + 2 * kSgnSlot, lin[6].sV + (int64_t)blk * wb, (uint32_t)wb, s.tab_full);
          }
          if (qk >= 0) {
            load_table_cluster<TM>(s.tab, lin[qk].tU, lin[qk].n_out, lin[qk].w_out, lin[qk].m_out, 0, (int)r, s.tab_full);
            bulk_g2s(s.sgn, lin[qk].sU + (int64_t)r * Eq, (uint32_t)Eq, s.tab_full);
          }
        }
        if (TM == kTmQ8) {
          const int wb = lin[4].w_out, mb = lin[4].m_out, blk = t_cta;
          if (blk < nblocks) {
            const uint32_t tb = table_bytes_local<TM>(wb, mb);
            expand_local(s.tab, lin[4].tU, lin[4].n_out, wb, mb, blk, lane);
            expand_local(s.tab + tb, lin[5].tU, lin[5].n_out, wb, mb, blk, lane);
            expand_local(s.tab + 2 * tb, lin[6].tV, lin[6].n_in, wb, mb, blk, lane);
          }
          const int qk = c == qk_cluster(p, 0) ? 0 : (c == qk_cluster(p, 1) ? 1 : -1);
          if (qk >= 0) expand_cluster(s.tab, lin[qk].tU, lin[qk].n_out, lin[qk].w_out, lin[qk].m_out, (int)r, lane);
        }
        finish();
        ++slot;
      }
      if (lane == 0 && slot > 0) wait_phase<false, true>(s.tab_full, (slot - 1) & 1, p.status, 54);
      __syncwarp();
    }
    cluster_sync_all();
    return;
  }

  // ---------------- consumers
  const int ct = tid;
  uint32_t kring = 0, tslot = 0;
  Xchg X;
  bool ok = true;
  auto tab_acquire = [&]() -> bool { return wait_uniform<false>(s.tab_full, tslot & 1, p.status, 55, ct); };
  auto tab_release = [&]() {
    cbar();
    if (ct == 0) mbar_arrive(s.tab_empty);
    ++tslot;
  };

  for (int l = 0; l < L && ok; ++l) {
    const Lin* lin = p.lin + 7 * l;
    const Lin* prev = l > 0 ? p.lin + 7 * (l - 1) : nullptr;
    // P1
    if (!(ok = tab_acquire())) break;
    {
      const uint8_t* tU = s.tab;
      const uint8_t* tV = prev ? s.tab + table_bytes_cluster<TC>(prev[6].w_out, prev[6].m_out) : s.tab;
      ok = chain_residual<TC>(p, s, X, prev ? prev + 6 : nullptr, p.zpd, p.nk_f, lin + p.asg_qkv[c], l == 0, r, ct, tU,
                          tV);
    }
    tab_release();
    if (!ok) break;
    // P2
    if (!(ok = run_units<BITS>(p, s, units<BITS>(p, l, 0, c, (int)r), kring, ct))) break;
    if (!(ok = grid_barrier(p, l * 5 + 0, ct))) break;
    // P3
    if (!(ok = tab_acquire())) break;
    ok = chain_attn<TC>(p, s, X, lin + 2, lin + 3, r, ct, s.tab,
                    s.tab + table_bytes_cluster<TC>(lin[2].w_out, lin[2].m_out));
    tab_release();
    if (!ok) break;
    // P4
    if (!(ok = run_units<BITS>(p, s, units<BITS>(p, l, 1, c, (int)r), kring, ct))) break;
    if (!(ok = grid_barrier(p, l * 5 + 1, ct))) break;
    // P5
    if (!(ok = tab_acquire())) break;
    ok = chain_residual<TC>(p, s, X, lin + 3, p.zpo, p.nk_h, lin + 4 + p.asg_gu[c], false, r, ct, s.tab,
                        s.tab + table_bytes_cluster<TC>(lin[3].w_out, lin[3].m_out));
    tab_release();
    if (!ok) break;
    // P6
    if (!(ok = run_units<BITS>(p, s, units<BITS>(p, l, 2, c, (int)r), kring, ct))) break;
    if (!(ok = grid_barrier(p, l * 5 + 2, ct))) break;
    // P7
    if (!(ok = tab_acquire())) break;
    {
      if (t_cta < nblocks) block_chain<TC>(p, s, lin + 4, lin + 5, lin + 6, t_cta, ct, s.tab);
      const int qk = c == qk_cluster(p, 0) ? 0 : (c == qk_cluster(p, 1) ? 1 : -1);
      if (qk >= 0) {
        float* out = qk == 0 ? p.qout + (int64_t)l * lin[0].n_out : p.kout + (int64_t)l * lin[1].n_out;
        const float* zp = qk == 0 ? p.zpq + (int64_t)l * p.nk_h * lin[0].n_out
                                  : p.zpk + (int64_t)l * p.nk_h * lin[1].n_out;
        ok = chain_out_only<TC>(p, s, X, lin + qk, zp, out, r, ct, s.tab);
      }
    }
    tab_release();
    if (!ok) break;
    if (!(ok = grid_barrier(p, l * 5 + 3, ct))) break;
    // P8: the down projection's operand from global
    {
      const int n_in = lin[6].n_in, ng = n_in / 64;
      const int words = BITS == 3 ? n_in : n_in / 2;
      const int4* src = reinterpret_cast<const int4*>(p.xq_down);
      int4* dst = reinterpret_cast<int4*>(s.xq);
      for (int i = ct; i < words / 4; i += kNT) dst[i] = __ldcg(src + i);
      float* xsA = reinterpret_cast<float*>(s.xq + words);
      for (int g = ct; g < ng; g += kNT) {
        xsA[g] = __ldcg(p.xs_down + g);
        xsA[ng + g] = __ldcg(p.xsum_down + g);
      }
      cbar();
      if (!(ok = run_units<BITS>(p, s, units<BITS>(p, l, 3, c, (int)r), kring, ct))) break;
    }
    if (!(ok = grid_barrier(p, l * 5 + 4, ct))) break;
  }
  // final: out = h_{L-1} + F_U_down(z_down)
  if (ok && (ok = tab_acquire())) {
    const Lin* last = p.lin + 7 * (L - 1);
    ok = chain_residual<TC>(p, s, X, last + 6, p.zpd, p.nk_f, nullptr, false, r, ct, s.tab, s.tab);
    if (ok && c == 0)
      for (int L2 = ct; L2 < p.E; L2 += kNT) store_act(p.y_out, gidx_b(L2, p.E, r), p.yt, s.res[L2]);
    tab_release();
  }
  cluster_sync_all();
}

// ------------------------------------------------------------------ host side
template <int BITS>
size_t smem_bytes(const Params& p) {
  return 1024 + (size_t)p.ring_stages * Geo<BITS>::kStageBytes + p.tab_bytes + 4 * kSgnSlot + 12 * (size_t)p.E + 64 +
         (size_t)4 * kCW * 32 * p.ring_stages + 4 * ((p.ring_stages + 3) & ~3) + p.xq_bytes +
         8 * (2 * (size_t)p.ring_stages + 3);
}

template <int BITS>
const void* kernel_ptr(int tm) {
  return tm == kTmHad  ? reinterpret_cast<const void*>(decode_kernel<BITS, kTmHad>)
         : tm == kTmQ8 ? reinterpret_cast<const void*>(decode_kernel<BITS, kTmQ8>)
                       : reinterpret_cast<const void*>(decode_kernel<BITS, kTmCS>);
}

template <int BITS>
cudaError_t launch_bits(const Params& p, cudaStream_t st) {
  const size_t smem = smem_bytes<BITS>(p);
  cudaError_t e = cudaFuncSetAttribute(kernel_ptr<BITS>(p.tm), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.G * kC), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kC;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (p.tm == kTmHad) return cudaLaunchKernelEx(&cfg, decode_kernel<BITS, kTmHad>, p);
  if (p.tm == kTmQ8) return cudaLaunchKernelEx(&cfg, decode_kernel<BITS, kTmQ8>, p);
  return cudaLaunchKernelEx(&cfg, decode_kernel<BITS, kTmCS>, p);
}

cudaError_t launch(const Params& p, cudaStream_t st) {
  switch (p.bits) {
    case 2: return launch_bits<2>(p, st);
    case 3: return launch_bits<3>(p, st);
    case 4: return launch_bits<4>(p, st);
  }
  return cudaErrorInvalidValue;
}

size_t smem_for(const Params& p) {
  switch (p.bits) {
    case 2: return smem_bytes<2>(p);
    case 3: return smem_bytes<3>(p);
    default: return smem_bytes<4>(p);
  }
}

int chunk_cols_for(int bits) {
  return bits == 2 ? Geo<2>::kChunkCols : (bits == 3 ? Geo<3>::kChunkCols : Geo<4>::kChunkCols);
}

cudaError_t max_clusters(const Params& p, int* out) {
  const void* fn = p.bits == 2 ? kernel_ptr<2>(p.tm) : (p.bits == 3 ? kernel_ptr<3>(p.tm) : kernel_ptr<4>(p.tm));
  const size_t smem = smem_for(p);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kC * 16, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kC;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaOccupancyMaxActiveClusters(out, fn, &cfg);
}

}  // namespace dec
}  // namespace harp
