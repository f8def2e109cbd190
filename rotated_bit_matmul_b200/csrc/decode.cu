// One batch-1 decode step through a whole Llama-shaped stack of rotated low-bit
// linears, in a single persistent kernel on sm_100a.
//
// The per-linear path launches three kernels per linear (input butterfly, GEMV,
// output butterfly) plus the glue, ~26 launches per block; at batch 1 every one of
// them is short and the launch/ramp/drain overheads dominate. Here one kernel does
// the whole step:
//
//  * Weights never depend on activations, so one producer lane per CTA streams that
//    CTA's rows of every GEMV of the step, in order, with 2-D TMA tile loads (no
//    multicast) into a ring of shared-memory stages. HBM keeps streaming while the
//    activation chain is busy elsewhere.
//  * The CTAs form clusters of 8. Each cluster computes the activation chain between
//    two GEMVs itself (redundantly with the other clusters), a w-wide butterfly
//    spread over its 8 CTAs (w/8 elements each) with the cross-CTA stages exchanged
//    through distributed shared memory (layouts A/B as in butterfly.cu). A second
//    producer lane prefetches each chain's cos/sin tables into shared memory.
//  * Grid-wide barriers (release/acquire counters) only where a whole output vector
//    is needed: after q/k/v, o, gate/up, the 256-wide down-input blocks, and down.
//
// Per block l (Sec. 2.1-2.2 and 5 of the HARP page for the butterflies; the glue is the
// stack definition of include/harp.h):
//   P1 chain: x_l = h_{l-1} + F_U_down(z_down)  (x_0 = input), rms, F_V of the cluster's
//             share of q/k/v, int16 GEMV operand, gathered across the cluster
//   P2 GEMV q, k or v rows                      -> grid barrier
//   P3 chain: F_U_v(z_v), broadcast per KV group, F_V_o, operand
//   P4 GEMV o rows                              -> grid barrier
//   P5 chain: h_l = x_l + F_U_o(z_o), rms, F_V of gate or up, operand
//   P6 GEMV gate or up rows                     -> grid barrier
//   P7 per 256-wide block (one CTA each): F_U_gate, F_U_up, silu*up, F_V_down, operand
//      to global; two idle clusters apply F_U_q and F_U_k to this block's q/k rows
//                                               -> grid barrier
//   P8 GEMV down rows                           -> grid barrier
// and after the last block: out = h_{L-1} + F_U_down(z_down).
//
// Every wait is bounded (%globaltimer, 1 s) and checks a shared abort word, so a
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
// not the .aligned form: the producer warp's lanes reach the final barrier at different times
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ uint32_t peer_addr(const void* local, uint32_t cta) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(cta));
  return ra;
}
__device__ __forceinline__ float4 ld_peer4(const void* local, uint32_t cta) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(peer_addr(local, cta))
               : "memory");
  return v;
}
__device__ __forceinline__ float ld_peer(const void* local, uint32_t cta) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(peer_addr(local, cta)) : "memory");
  return v;
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

constexpr uint64_t kWaitNs = 1000000000ull;

// bounded wait on a local mbarrier phase; false on time-out or abort
template <bool CLUSTER>
__device__ bool wait_phase(uint64_t* bar, uint32_t parity, int* status, int where) {
  if (CLUSTER ? try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 32; ++i)
      if (CLUSTER ? try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
    if (aborted(status)) return false;
    if (globaltimer_ns() - t0 > kWaitNs) {
      report(status, 5, where);
      return false;
    }
  }
}

__device__ __forceinline__ void cbar() { asm volatile("bar.sync 1, %0;" ::"r"(kNT) : "memory"); }

// barrier of the consumer threads that also ANDs a predicate across them: every wait
// below is polled by one thread and its outcome made uniform here, so a time-out can
// never leave some consumer threads waiting at a barrier the others have left
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
struct Smem {
  uint8_t* ring;
  float2* tab;
  float *xa, *xb, *res, *red, *ss;
  int32_t* xq;  // local GEMV operand: xq words, then xs [ng], then xsum [ng]
  uint64_t *full, *empty, *tab_full, *tab_empty, *xchg;
};

__device__ __forceinline__ Smem carve(const Params& p, int stage_bytes) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* b = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem s;
  s.ring = b;
  b += (size_t)p.ring_stages * stage_bytes;
  s.tab = reinterpret_cast<float2*>(b);
  b += p.tab_bytes;
  s.xa = reinterpret_cast<float*>(b);
  b += 4 * p.E;
  s.xb = reinterpret_cast<float*>(b);
  b += 4 * p.E;
  s.res = reinterpret_cast<float*>(b);
  b += 4 * p.E;
  s.red = reinterpret_cast<float*>(b);
  b += 4 * kCW * 32;
  s.ss = reinterpret_cast<float*>(b);
  b += 4 * 16;
  s.xq = reinterpret_cast<int32_t*>(b);
  b += p.xq_bytes;
  s.full = reinterpret_cast<uint64_t*>(b);
  s.empty = s.full + p.ring_stages;
  s.tab_full = s.empty + p.ring_stages;
  s.tab_empty = s.tab_full + 1;
  s.xchg = s.tab_empty + 1;
  return s;
}

// ------------------------------------------------------------------ static work assignment
struct Job {
  const Lin* L;
  int row0, row1;
  float* z;
};

__device__ __forceinline__ int split(int n, int i, int parts) { return (int)(((int64_t)n * i) / parts); }

// GEMV job of phase `ph` (0: q/k/v, 1: o, 2: gate/up, 3: down) of block l for CTA (c, r)
__device__ Job gemv_job(const Params& p, int l, int ph, int c, int r) {
  const Lin* lin = p.lin + 7 * l;
  Job j;
  if (ph == 0 || ph == 2) {
    const int which = ph == 0 ? p.asg_qkv[c] : p.asg_gu[c];
    const int ci = ph == 0 ? p.idx_qkv[c] : p.idx_gu[c];
    const int nc = ph == 0 ? p.cnt_qkv[which] : p.cnt_gu[which];
    j.L = lin + (ph == 0 ? which : 4 + which);
    const int n = j.L->n_out, i = ci * kC + r, parts = nc * kC;
    j.row0 = split(n, i, parts);
    j.row1 = split(n, i + 1, parts);
    if (ph == 0) j.z = which == 0 ? p.zq + (int64_t)l * j.L->n_out : (which == 1 ? p.zk + (int64_t)l * j.L->n_out : p.zv);
    else j.z = which == 0 ? p.zg : p.zu;
  } else {
    j.L = lin + (ph == 1 ? 3 : 6);
    const int n = j.L->n_out, t = c * kC + r, parts = p.G * kC;
    j.row0 = split(n, t, parts);
    j.row1 = split(n, t + 1, parts);
    j.z = ph == 1 ? p.zo : p.zd;
  }
  return j;
}

// ------------------------------------------------------------------ table loads (producer lane 1)
// Per-CTA slice of a cluster-distributed butterfly (width w, C = 8): stage t < e is the
// contiguous run of the CTA's chunk; stage t >= e is C/2 runs of `run` pairs.
__device__ uint32_t load_table_cluster(float2* dst, const float2* cs, int64_t n, int w, int m, int blk, int r,
                                       uint64_t* bar) {
  const int E = w / kC, e = m - 3, run = E / kC;
  const int64_t half_n = n >> 1;
  for (int t = 0; t < m; ++t) {
    const float2* src = cs + (int64_t)t * half_n + (int64_t)blk * (w >> 1);
    float2* d = dst + (size_t)t * (E >> 1);
    if (t < e) {
      bulk_g2s(d, src + (int64_t)r * (E >> 1), (uint32_t)(8 * (E >> 1)), bar);
    } else {
      const int dd = t - e;
      for (int jj = 0; jj < (kC >> 1); ++jj) {
        const int j = ((jj >> dd) << (dd + 1)) | (jj & ((1 << dd) - 1));
        const int64_t pb = (int64_t)(j >> (dd + 1)) * (1 << t) + (int64_t)E * (j & ((1 << dd) - 1)) + (int64_t)r * run;
        bulk_g2s(d + jj * run, src + pb, (uint32_t)(8 * run), bar);
      }
    }
  }
  return (uint32_t)(8 * m * (E >> 1));
}

// the whole block `blk` of width w held by one CTA: one run of w/2 pairs per stage
__device__ uint32_t load_table_local(float2* dst, const float2* cs, int64_t n, int w, int m, int blk, uint64_t* bar) {
  for (int t = 0; t < m; ++t)
    bulk_g2s(dst + (size_t)t * (w >> 1), cs + (int64_t)t * (n >> 1) + (int64_t)blk * (w >> 1), (uint32_t)(4 * w), bar);
  return (uint32_t)(4 * w * m);
}

__device__ __forceinline__ uint32_t table_bytes_cluster(int w, int m) { return (uint32_t)(8 * m * (w / kC / 2)); }

// P7 roles: block CTAs, and the clusters applying F_U_q / F_U_k
__device__ __forceinline__ int qk_cluster(const Params& p, int which) { return p.G - 1 - which; }

// ------------------------------------------------------------------ butterfly stages (consumer threads)
__device__ __forceinline__ void rot(float* a, float* b, float2 cs) {
  const float x = *a, y = *b;
  *a = fmaf(cs.x, x, cs.y * y);
  *b = fmaf(cs.y, x, -cs.x * y);
}

// layout-A stages 0..e-1 on a buffer of E elements (table: e rows of E/2 pairs)
__device__ void stages_a(float* x, const float2* tab, int e, int E, int ct) {
  for (int t = 0; t < e; ++t) {
    const int h = 1 << t;
    const float2* tt = tab + (size_t)t * (E >> 1);
    for (int q = ct; q < (E >> 1); q += kNT) {
      const int i = ((q >> t) << (t + 1)) | (q & (h - 1));
      rot(x + i, x + i + h, tt[q]);
    }
    cbar();
  }
}

// layout-B stages (pairing run j with j + 2^d) on E elements; table rows follow the e A-rows
__device__ void stages_b(float* x, const float2* tab, int e, int E, int ct) {
  const int run = E / kC;
  for (int d = 0; d < 3; ++d) {
    const float2* tt = tab + (size_t)(e + d) * (E >> 1);
    for (int q = ct; q < (E >> 1); q += kNT) {
      const int jj = q / run, ii = q - jj * run;
      const int j = ((jj >> d) << (d + 1)) | (jj & ((1 << d) - 1));
      float* pa = x + j * run + ii;
      rot(pa, pa + (run << d), tt[q]);
    }
    cbar();
  }
}

// cluster-wide exchange point among the consumer threads of the 8 CTAs
struct Xchg {
  uint32_t phase = 0;
};
__device__ bool exchange(Smem& s, Xchg& x, int ct, int* status, int where) {
  cbar();
  bool mine = true;
  if (ct == 0) {
    for (uint32_t q = 0; q < kC; ++q) arrive_remote(s.xchg, q);
    mine = wait_phase<true>(s.xchg, x.phase, status, where);
  }
  x.phase ^= 1;
  return cbar_and(mine);
}

// gather layout A (peer j's chunk, local offset r*run + ii) into layout B
__device__ void gather_a_to_b(float* dst_b, const float* src_a, int E, uint32_t r, int ct) {
  const int run = E / kC;
  for (int L4 = ct; L4 < (E >> 2); L4 += kNT) {
    const int L = L4 * 4, j = L / run, ii = L - j * run;
    const float4 v = ld_peer4(src_a + r * run + ii, (uint32_t)j);
    *reinterpret_cast<float4*>(dst_b + L) = v;
  }
}

// global element index of local position L in layout B (width w, CTA rank r)
__device__ __forceinline__ int gidx_b(int L, int E, uint32_t r) {
  const int run = E / kC, j = L / run, ii = L - j * run;
  return j * E + (int)r * run + ii;
}

// int16 GEMV operand of one group of 64 values (one warp): returns (xs, xsum) via lane 0
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
  if (amax > 0.f && !bad) {
    int E2;
    frexpf(amax, &E2);
    ex = min(max(15 - E2, -126), 126);
  }
  const float sc = ldexpf(1.f, ex);
  const int q0 = max(-32767, min(32767, __float2int_rn(v0 * sc)));
  const int q1 = max(-32767, min(32767, __float2int_rn(v1 * sc)));
  grp[xq_pos_lo(bits, 2 * lane)] = (int16_t)q0;
  grp[xq_pos_lo(bits, 2 * lane + 1)] = (int16_t)q1;
  if (bits == 3) {
    grp_hi[xq_pos_hi(2 * lane)] = (int16_t)q0;
    grp_hi[xq_pos_hi(2 * lane + 1)] = (int16_t)q1;
  }
  if (lane == 0) {
    *xs = bad ? __int_as_float(0x7fc00000) : ldexpf(1.f, -ex);
    *xsum = bad ? __int_as_float(0x7fc00000) : sum;
  }
}

// operand of a w-wide (w >= 4096) input in layout B: prep the CTA's own groups into its
// local operand buffer, exchange, then copy every other group from its owner
__device__ bool prep_and_gather(Smem& s, Xchg& X, const float* xb, int n_in, int bits, int E, uint32_t r, int ct,
                                int* status) {
  const int ng = n_in / 64, run = E / kC;
  int16_t* xq16 = reinterpret_cast<int16_t*>(s.xq);
  const int words = bits == 3 ? n_in : n_in / 2;
  float* xsA = reinterpret_cast<float*>(s.xq + words);
  float* xsumA = xsA + ng;
  const int warp = ct >> 5, lane = ct & 31;
  for (int gl = warp; gl < (E >> 6); gl += kCW) {
    const int g = gidx_b(gl * 64, E, r) >> 6;
    prep_group(xb + gl * 64, bits, xq16 + (int64_t)g * 64, xq16 + n_in + (int64_t)g * 64, xsA + g, xsumA + g, lane);
  }
  if (!exchange(s, X, ct, status, 40)) return false;
  // copy foreign groups: 8 int4 per group (lo plane), 8 more for the 1-bit plane order
  const int per = bits == 3 ? 16 : 8;
  for (int it = ct; it < ng * per; it += kNT) {
    const int g = it / per, part = it - g * per;
    const uint32_t owner = (uint32_t)(((g * 64) % E) / run);
    if (owner == r) continue;
    const int word = part < 8 ? g * 32 + part * 4 : n_in / 2 + g * 32 + (part - 8) * 4;
    *reinterpret_cast<float4*>(s.xq + word) = ld_peer4(s.xq + word, owner);
  }
  for (int g = ct; g < ng; g += kNT) {
    const uint32_t owner = (uint32_t)(((g * 64) % E) / run);
    if (owner == r) continue;
    xsA[g] = ld_peer(xsA + g, owner);
    xsumA[g] = ld_peer(xsumA + g, owner);
  }
  cbar();
  return true;
}

// ------------------------------------------------------------------ chains (cluster-collective)
// residual chain: [res += F_U(z)] ; n = rms(res) ; x~ = F_V(n) ; operand
__device__ bool chain_residual(const Params& p, Smem& s, Xchg& X, const Lin* U, const float* z, const Lin* V,
                               bool first, uint32_t r, int ct, const float2* tabU, const float2* tabV) {
  const int W = p.hidden, E = p.E, e = p.m_hidden - 3;
  if (first) {
    for (int L = ct; L < E; L += kNT) s.res[L] = load_act(p.x_in, gidx_b(L, E, r), p.xt);
  } else {
    for (int i = ct; i < E; i += kNT) {
      const int gi = (int)r * E + i;
      s.xa[i] = __ldcg(z + gi) * (float)U->sU[gi];
    }
    cbar();
    stages_a(s.xa, tabU, e, E, ct);
    if (!exchange(s, X, ct, p.status, 41)) return false;
    gather_a_to_b(s.xb, s.xa, E, r, ct);
    cbar();
    stages_b(s.xb, tabU, e, E, ct);
    for (int L = ct; L < E; L += kNT) s.res[L] += s.xb[L];
  }
  if (!V) return true;  // final step: no input butterfly
  // sum of squares of this CTA's share, fixed-order tree
  float acc = 0.f;
  for (int L = ct; L < E; L += kNT) acc = fmaf(s.res[L], s.res[L], acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((ct & 31) == 0) s.red[ct >> 5] = acc;
  cbar();
  if (ct == 0) {
    float t = 0.f;
    for (int w = 0; w < kCW; ++w) t += s.red[w];
    s.ss[0] = t;
  }
  if (!exchange(s, X, ct, p.status, 42)) return false;
  __shared__ float inv_rms;
  if (ct == 0) {
    float t = 0.f;
    for (uint32_t q = 0; q < kC; ++q) t += ld_peer(s.ss, q);
    inv_rms = 1.0f / sqrtf(t / (float)W + p.eps);
  }
  cbar();
  const float inv = inv_rms;
  const int run = E / kC;
  for (int i4 = ct; i4 < (E >> 2); i4 += kNT) {
    const int i = i4 * 4, q = i / run;  // chunk-r element i sits in CTA q at r*run + i%run
    const float4 v = ld_peer4(s.res + (int)r * run + (i - q * run), (uint32_t)q);
    const int gi = (int)r * E + i;
    s.xa[i + 0] = v.x * inv * (float)V->sV[gi + 0];
    s.xa[i + 1] = v.y * inv * (float)V->sV[gi + 1];
    s.xa[i + 2] = v.z * inv * (float)V->sV[gi + 2];
    s.xa[i + 3] = v.w * inv * (float)V->sV[gi + 3];
  }
  cbar();
  stages_a(s.xa, tabV, e, E, ct);
  if (!exchange(s, X, ct, p.status, 43)) return false;
  gather_a_to_b(s.xb, s.xa, E, r, ct);
  cbar();
  stages_b(s.xb, tabV, e, E, ct);
  return prep_and_gather(s, X, s.xb, V->n_in, p.bits, E, r, ct, p.status);
}

// attention chain: v = F_U_v(z_v); a = v broadcast per KV group; x~ = F_V_o(a); operand
__device__ bool chain_attn(const Params& p, Smem& s, Xchg& X, const Lin* Lv, const Lin* Lo, uint32_t r, int ct,
                           const float2* tabU, const float2* tabV) {
  const int Wu = Lv->w_out, Eu = Wu / kC, eu = Lv->m_out - 3;
  for (int i = ct; i < Eu; i += kNT) {
    const int gi = (int)r * Eu + i;
    s.xa[i] = __ldcg(p.zv + gi) * (float)Lv->sU[gi];
  }
  cbar();
  stages_a(s.xa, tabU, eu, Eu, ct);
  if (!exchange(s, X, ct, p.status, 44)) return false;
  gather_a_to_b(s.xb, s.xa, Eu, r, ct);
  cbar();
  stages_b(s.xb, tabU, eu, Eu, ct);
  if (!exchange(s, X, ct, p.status, 45)) return false;
  const int Eo = p.E, eo = p.m_hidden - 3, hd = p.head_dim, rep = p.rep, runu = Eu / kC;
  for (int i = ct; i < Eo; i += kNT) {
    const int ga = (int)r * Eo + i;                         // element of a (query-head space)
    const int gv = ((ga / hd) / rep) * hd + (ga % hd);       // element of v it copies
    const int j = gv / Eu, rem = gv - j * Eu, q = rem / runu; // owner of gv in v's layout B
    s.xa[i] = ld_peer(s.xb + j * runu + (rem - q * runu), (uint32_t)q) * (float)Lo->sV[ga];
  }
  cbar();
  stages_a(s.xa, tabV, eo, Eo, ct);
  if (!exchange(s, X, ct, p.status, 46)) return false;
  gather_a_to_b(s.xb, s.xa, Eo, r, ct);
  cbar();
  stages_b(s.xb, tabV, eo, Eo, ct);
  return prep_and_gather(s, X, s.xb, Lo->n_in, p.bits, Eo, r, ct, p.status);
}

// F_U of a q or k GEMV output (cluster-distributed), written to out[gidx]
__device__ bool chain_out_only(const Params& p, Smem& s, Xchg& X, const Lin* Lq, const float* z, float* out,
                               uint32_t r, int ct, const float2* tab) {
  const int W = Lq->w_out, E = W / kC, e = Lq->m_out - 3;
  for (int i = ct; i < E; i += kNT) {
    const int gi = (int)r * E + i;
    s.xa[i] = __ldcg(z + gi) * (float)Lq->sU[gi];
  }
  cbar();
  stages_a(s.xa, tab, e, E, ct);
  if (!exchange(s, X, ct, p.status, 47)) return false;
  gather_a_to_b(s.xb, s.xa, E, r, ct);
  cbar();
  stages_b(s.xb, tab, e, E, ct);
  for (int L = ct; L < E; L += kNT) out[gidx_b(L, E, r)] = s.xb[L];
  return true;
}

// one whole 256-wide (<= 512) block of the MLP in one CTA: F_U_gate, F_U_up, silu*up,
// F_V_down, operand rows of the down projection (to global)
__device__ void block_chain(const Params& p, Smem& s, const Lin* Lg, const Lin* Lu, const Lin* Ld, int blk, int ct,
                            const float2* tab) {
  const int wb = Lg->w_out, mb = Lg->m_out;
  const int64_t base = (int64_t)blk * wb;
  for (int i = ct; i < wb; i += kNT) {
    s.xa[i] = __ldcg(p.zg + base + i) * (float)Lg->sU[base + i];
    s.xb[i] = __ldcg(p.zu + base + i) * (float)Lu->sU[base + i];
  }
  cbar();
  stages_a(s.xa, tab, mb, wb, ct);
  stages_a(s.xb, tab + (size_t)mb * (wb >> 1), mb, wb, ct);
  for (int i = ct; i < wb; i += kNT) {
    const float g = s.xa[i];
    s.xa[i] = g / (1.0f + expf(-g)) * s.xb[i] * (float)Ld->sV[base + i];
  }
  cbar();
  stages_a(s.xa, tab + (size_t)2 * mb * (wb >> 1), mb, wb, ct);
  const int n_in = Ld->n_in, ng = n_in / 64;
  int16_t* xq16 = reinterpret_cast<int16_t*>(p.xq_down);
  const int warp = ct >> 5, lane = ct & 31;
  for (int gl = warp; gl < (wb >> 6); gl += kCW) {
    const int g = (int)(base >> 6) + gl;
    prep_group(s.xa + gl * 64, p.bits, xq16 + (int64_t)g * 64, xq16 + n_in + (int64_t)g * 64, p.xs_down + g,
               p.xsum_down + g, lane);
  }
  (void)ng;
  cbar();
}

// ------------------------------------------------------------------ GEMV job (consumer side)
template <int BITS>
__device__ bool run_gemv(const Params& p, Smem& s, const Job& j, uint32_t& kring, int ct) {
  using Gm = Geo<BITS>;
  const int warp = ct >> 5, lane = ct & 31;
  const int nrows = j.row1 - j.row0;
  if (nrows <= 0) return true;
  const int nsub = (nrows + 31) / 32, ngroups = j.L->n_in / 64;
  const int nchunks = (ngroups + Gm::kChunkGroups - 1) / Gm::kChunkGroups;
  const int words = BITS == 3 ? j.L->n_in : j.L->n_in / 2;
  const float* xsA = reinterpret_cast<const float*>(s.xq + words);
  const float* xsumA = xsA + ngroups;
  float zacc = 0.f;
  for (int sub = 0; sub < nsub; ++sub) {
    const int row0 = j.row0 + split(nrows, sub, nsub), row1 = j.row0 + split(nrows, sub + 1, nsub);
    for (int ch = 0; ch < nchunks; ++ch, ++kring) {
      const int slot = kring % p.ring_stages;
      if (!wait_uniform<false>(&s.full[slot], (kring / p.ring_stages) & 1, p.status, 50, ct)) return false;
      const uint8_t* st = s.ring + (size_t)slot * Gm::kStageBytes;
      const uint8_t* szs = st + (Gm::kCodeSlabs + Gm::kHiSlabs) * kSlab;
      const int g0 = ch * Gm::kChunkGroups, gc = min(Gm::kChunkGroups, ngroups - g0);
      for (int gl = warp; gl < gc; gl += kCW) {
        const int g = g0 + gl;
        const uint32_t szw = *reinterpret_cast<const uint32_t*>(swz(szs, lane, gl >> 2) + (gl & 3) * 4);
        const float s16 = __half2float(__ushort_as_half((unsigned short)(szw & 0xffffu)));
        const float z16 = __half2float(__ushort_as_half((unsigned short)(szw >> 16)));
        const int4* xg = reinterpret_cast<const int4*>(s.xq + (int64_t)g * 32);
        const int4* xgh = reinterpret_cast<const int4*>(s.xq + j.L->n_in / 2 + (int64_t)g * 32);
        const int acc = group_dot<BITS, true>(st, st + Gm::kCodeSlabs * kSlab, lane, gl, xg, xgh);
        zacc = fmaf(s16, (float)acc * xsA[g], fmaf(z16, xsumA[g], zacc));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.empty[slot]);
      if (ch == nchunks - 1) {
        s.red[warp * 32 + lane] = zacc;
        cbar();
        if (warp == 0) {
          float t = 0.f;
#pragma unroll
          for (int w = 0; w < kCW; ++w) t += s.red[w * 32 + lane];
          if (row0 + lane < row1) j.z[row0 + lane] = t;
        }
        cbar();
        zacc = 0.f;
      }
    }
  }
  return true;
}

// ------------------------------------------------------------------ grid barrier
__device__ bool grid_barrier(const Params& p, int idx, int ct) {
  cbar();
  bool mine = true;
  if (ct == 0) {
    unsigned* c = p.counters + idx;
    __threadfence();
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(c) : "memory");
    const unsigned target = (unsigned)(p.G * kC);
    const uint64_t t0 = globaltimer_ns();
    while (true) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(c) : "memory");
      if (v >= target) break;
      if (aborted(p.status)) {
        mine = false;
        break;
      }
      if (globaltimer_ns() - t0 > kWaitNs) {
        report(p.status, 5, 60 + (idx % 5));
        mine = false;
        break;
      }
    }
  }
  return cbar_and(mine);
}

// ------------------------------------------------------------------ the kernel
template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ Params p) {
  using Gm = Geo<BITS>;
  Smem s = carve(p, Gm::kStageBytes);
  const uint32_t r = cta_rank();
  const int c = (int)cluster_id_x();
  const int tid = threadIdx.x;
  const int t_cta = c * kC + (int)r;

  if (tid == 0) {
    for (int i = 0; i < p.ring_stages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], kCW);
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
    const int lane = tid - kNT;
    if (lane == 0) {
      // ---------------- ring producer: every GEMV job of the step, in consumer order
      uint32_t k = 0;
      bool ok = true;
      for (int l = 0; l < L && ok; ++l)
        for (int ph = 0; ph < 4 && ok; ++ph) {
          const Job j = gemv_job(p, l, ph, c, (int)r);
          const int nrows = j.row1 - j.row0;
          if (nrows <= 0) continue;
          const int nsub = (nrows + 31) / 32, ngroups = j.L->n_in / 64;
          const int nchunks = (ngroups + Gm::kChunkGroups - 1) / Gm::kChunkGroups;
          for (int sub = 0; sub < nsub && ok; ++sub) {
            const int row0 = j.row0 + split(nrows, sub, nsub);
            for (int ch = 0; ch < nchunks; ++ch, ++k) {
              const int slot = k % p.ring_stages;
              if (k >= (uint32_t)p.ring_stages &&
                  !wait_phase<false>(&s.empty[slot], ((k / p.ring_stages) - 1) & 1, p.status, 51)) {
                ok = false;
                break;
              }
              const int g0 = ch * Gm::kChunkGroups, gc = min(Gm::kChunkGroups, ngroups - g0);
              const int cslabs = (gc + Gm::kGroupsPerSlab - 1) / Gm::kGroupsPerSlab;
              const int hslabs = BITS == 3 ? (gc + 15) / 16 : 0;
              uint8_t* st = s.ring + (size_t)slot * Gm::kStageBytes;
              mbar_arrive_expect_tx(&s.full[slot], (uint32_t)((cslabs + hslabs + 1) * kSlab));
              const int code_x0 = g0 * (BITS == 4 ? 32 : 16) / 8;
              for (int q = 0; q < cslabs; ++q)
                tma_load_2d(st + q * kSlab, &j.L->tm_codes, &s.full[slot], code_x0 + q * 16, row0);
              if (BITS == 3)
                for (int q = 0; q < hslabs; ++q)
                  tma_load_2d(st + (Gm::kCodeSlabs + q) * kSlab, &j.L->tm_hi, &s.full[slot], g0 + q * 16, row0);
              tma_load_2d(st + (Gm::kCodeSlabs + Gm::kHiSlabs) * kSlab, &j.L->tm_sz, &s.full[slot], g0, row0);
            }
          }
        }
      // drain: wait for the copies still in flight before the CTA may exit
      const uint32_t nwait = k < (uint32_t)p.ring_stages ? k : (uint32_t)p.ring_stages;
      for (uint32_t q = k - nwait; q < k; ++q) wait_phase<false>(&s.full[q % p.ring_stages], (q / p.ring_stages) & 1, p.status, 52);
    } else if (lane == 1) {
      // ---------------- table producer: one table set per chain slot, in consumer order
      uint32_t slot = 0;
      bool ok = true;
      auto begin = [&]() -> bool {
        if (slot > 0 && !wait_phase<false>(s.tab_empty, (slot - 1) & 1, p.status, 53)) return false;
        return true;
      };
      for (int l = 0; l <= L && ok; ++l) {
        const Lin* lin = p.lin + 7 * l;
        const Lin* prev = l > 0 ? p.lin + 7 * (l - 1) : nullptr;
        // P1 (or the final step when l == L)
        if (!(ok = begin())) break;
        {
          uint32_t bytes = 0;
          if (prev) bytes += table_bytes_cluster(prev[6].w_out, prev[6].m_out);
          const Lin* V = l < L ? lin + p.asg_qkv[c] : nullptr;
          if (V) bytes += table_bytes_cluster(V->w_in, V->m_in);
          mbar_arrive_expect_tx(s.tab_full, bytes);
          uint32_t off = 0;
          if (prev) off += load_table_cluster(s.tab, prev[6].csU, prev[6].n_out, prev[6].w_out, prev[6].m_out, 0, (int)r, s.tab_full);
          if (V) load_table_cluster(s.tab + off / 8, V->csV, V->n_in, V->w_in, V->m_in, 0, (int)r, s.tab_full);
        }
        ++slot;
        if (l == L) break;
        // P3
        if (!(ok = begin())) break;
        {
          const uint32_t b0 = table_bytes_cluster(lin[2].w_out, lin[2].m_out);
          mbar_arrive_expect_tx(s.tab_full, b0 + table_bytes_cluster(lin[3].w_in, lin[3].m_in));
          load_table_cluster(s.tab, lin[2].csU, lin[2].n_out, lin[2].w_out, lin[2].m_out, 0, (int)r, s.tab_full);
          load_table_cluster(s.tab + b0 / 8, lin[3].csV, lin[3].n_in, lin[3].w_in, lin[3].m_in, 0, (int)r, s.tab_full);
        }
        ++slot;
        // P5
        if (!(ok = begin())) break;
        {
          const Lin* V = lin + 4 + p.asg_gu[c];
          const uint32_t b0 = table_bytes_cluster(lin[3].w_out, lin[3].m_out);
          mbar_arrive_expect_tx(s.tab_full, b0 + table_bytes_cluster(V->w_in, V->m_in));
          load_table_cluster(s.tab, lin[3].csU, lin[3].n_out, lin[3].w_out, lin[3].m_out, 0, (int)r, s.tab_full);
          load_table_cluster(s.tab + b0 / 8, V->csV, V->n_in, V->w_in, V->m_in, 0, (int)r, s.tab_full);
        }
        ++slot;
        // P7: this CTA's MLP blocks, or F_U_q / F_U_k for the two q/k clusters
        if (!(ok = begin())) break;
        {
          uint32_t bytes = 0;
          const int wb = lin[4].w_out, mb = lin[4].m_out;
          for (int blk = t_cta; blk < nblocks; blk += p.G * kC) bytes += 3 * 4 * wb * mb;
          const int qk = c == qk_cluster(p, 0) ? 0 : (c == qk_cluster(p, 1) ? 1 : -1);
          if (qk >= 0) bytes += table_bytes_cluster(lin[qk].w_out, lin[qk].m_out);
          mbar_arrive_expect_tx(s.tab_full, bytes);
          uint32_t off = 0;
          for (int blk = t_cta; blk < nblocks; blk += p.G * kC) {
            off += load_table_local(s.tab + off / 8, lin[4].csU, lin[4].n_out, wb, mb, blk, s.tab_full);
            off += load_table_local(s.tab + off / 8, lin[5].csU, lin[5].n_out, wb, mb, blk, s.tab_full);
            off += load_table_local(s.tab + off / 8, lin[6].csV, lin[6].n_in, wb, mb, blk, s.tab_full);
          }
          if (qk >= 0)
            load_table_cluster(s.tab + off / 8, lin[qk].csU, lin[qk].n_out, lin[qk].w_out, lin[qk].m_out, 0, (int)r,
                               s.tab_full);
        }
        ++slot;
      }
      if (slot > 0) wait_phase<false>(s.tab_full, (slot - 1) & 1, p.status, 54);
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
      const float2* tU = s.tab;
      const float2* tV = prev ? s.tab + table_bytes_cluster(prev[6].w_out, prev[6].m_out) / 8 : s.tab;
      ok = chain_residual(p, s, X, prev ? prev + 6 : nullptr, p.zd, lin + p.asg_qkv[c], l == 0, r, ct, tU, tV);
    }
    tab_release();
    if (!ok) break;
    // P2
    {
      const Job j = gemv_job(p, l, 0, c, (int)r);
      if (!(ok = run_gemv<BITS>(p, s, j, kring, ct))) break;
    }
    if (!(ok = grid_barrier(p, l * 5 + 0, ct))) break;
    // P3
    if (!(ok = tab_acquire())) break;
    ok = chain_attn(p, s, X, lin + 2, lin + 3, r, ct, s.tab,
                    s.tab + table_bytes_cluster(lin[2].w_out, lin[2].m_out) / 8);
    tab_release();
    if (!ok) break;
    // P4
    {
      const Job j = gemv_job(p, l, 1, c, (int)r);
      if (!(ok = run_gemv<BITS>(p, s, j, kring, ct))) break;
    }
    if (!(ok = grid_barrier(p, l * 5 + 1, ct))) break;
    // P5
    if (!(ok = tab_acquire())) break;
    ok = chain_residual(p, s, X, lin + 3, p.zo, lin + 4 + p.asg_gu[c], false, r, ct, s.tab,
                        s.tab + table_bytes_cluster(lin[3].w_out, lin[3].m_out) / 8);
    tab_release();
    if (!ok) break;
    // P6
    {
      const Job j = gemv_job(p, l, 2, c, (int)r);
      if (!(ok = run_gemv<BITS>(p, s, j, kring, ct))) break;
    }
    if (!(ok = grid_barrier(p, l * 5 + 2, ct))) break;
    // P7
    if (!(ok = tab_acquire())) break;
    {
      const int wb = lin[4].w_out, mb = lin[4].m_out;
      size_t off = 0;
      for (int blk = t_cta; blk < nblocks; blk += p.G * kC) {
        block_chain(p, s, lin + 4, lin + 5, lin + 6, blk, ct, s.tab + off);
        off += (size_t)3 * mb * (wb >> 1);
      }
      const int qk = c == qk_cluster(p, 0) ? 0 : (c == qk_cluster(p, 1) ? 1 : -1);
      if (qk >= 0) {
        float* out = qk == 0 ? p.qout + (int64_t)l * lin[0].n_out : p.kout + (int64_t)l * lin[1].n_out;
        const float* z = qk == 0 ? p.zq + (int64_t)l * lin[0].n_out : p.zk + (int64_t)l * lin[1].n_out;
        ok = chain_out_only(p, s, X, lin + qk, z, out, r, ct, s.tab + off);
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
      const Job j = gemv_job(p, l, 3, c, (int)r);
      if (!(ok = run_gemv<BITS>(p, s, j, kring, ct))) break;
    }
    if (!(ok = grid_barrier(p, l * 5 + 4, ct))) break;
  }
  // final: out = h_{L-1} + F_U_down(z_down)
  if (ok && (ok = tab_acquire())) {
    const Lin* last = p.lin + 7 * (L - 1);
    ok = chain_residual(p, s, X, last + 6, p.zd, nullptr, false, r, ct, s.tab, s.tab);
    if (ok && c == 0)
      for (int L2 = ct; L2 < p.E; L2 += kNT) store_act(p.y_out, gidx_b(L2, p.E, r), p.yt, s.res[L2]);
    tab_release();
  }
  cluster_sync_all();
}

// ------------------------------------------------------------------ host side
int xq_words(int n_in, int bits) { return bits == 3 ? n_in : n_in / 2; }

template <int BITS>
size_t smem_bytes(const Params& p) {
  return 1024 + (size_t)p.ring_stages * Geo<BITS>::kStageBytes + p.tab_bytes + 12 * (size_t)p.E + 4 * kCW * 32 +
         64 + p.xq_bytes + 8 * (2 * (size_t)p.ring_stages + 3);
}

template <int BITS>
const void* kernel_ptr() {
  return reinterpret_cast<const void*>(decode_kernel<BITS>);
}

template <int BITS>
cudaError_t launch_bits(const Params& p, cudaStream_t st) {
  const size_t smem = smem_bytes<BITS>(p);
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
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
  return cudaLaunchKernelEx(&cfg, decode_kernel<BITS>, p);
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

int stage_bytes_for(int bits) {
  return bits == 2 ? Geo<2>::kStageBytes : (bits == 3 ? Geo<3>::kStageBytes : Geo<4>::kStageBytes);
}

cudaError_t max_clusters(const Params& p, int* out) {
  const void* fn = p.bits == 2 ? kernel_ptr<2>() : (p.bits == 3 ? kernel_ptr<3>() : kernel_ptr<4>());
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
