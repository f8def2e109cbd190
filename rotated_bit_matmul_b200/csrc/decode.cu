// One batch-1 decode step through a whole Llama-shaped stack of rotated low-bit
// linears, in a single persistent kernel on sm_100a.
//
// The per-linear path launches three kernels per linear (input butterfly, GEMV,
// output butterfly) plus the glue; at batch 1 every launch is short and the
// launch/ramp/drain overheads dominate. Here one kernel does the whole step:
//
//  * Weights never depend on activations, so as each GEMV phase starts, every warp asks
//    for its rows of the next phase's weights in L2 (plain per-lane line prefetches), and
//    HBM streams them while the chains run. A GEMV is cut into units of 32 output rows x
//    2048 input columns (split-K); each unit's partial sums go to a buffer the next chain
//    adds up in a fixed order. Each of the 16 warps takes two rows of every unit; a
//    lane holds one group of 64 input columns, with its operand words in registers, and
//    loads that group's codes and scale/zero words of its rows straight from L2 (a warp
//    reads each row's chunk as one contiguous span).
//  * CTAs form clusters of 8. Each cluster computes the activation chain between two
//    GEMVs itself (redundantly with the other clusters): a w-wide butterfly is spread
//    over the 8 CTAs, w/8 elements each. Every consumer thread holds one (two when
//    w = 8192) elements. Stages of stride below 32 are warp shuffles; one transpose
//    through shared memory turns the next five stride bits into lane bits; the last
//    three stages (the CTA bits) follow one exchange: every CTA stores its elements
//    straight into the owners' shared memory with st.async, whose completion is
//    counted in bytes on the receiver's mbarrier (data and signal in one). Exchanges
//    alternate between two receive buffers and two mbarriers, so a CTA that runs one
//    exchange ahead never writes into data a peer is still reading.
//  * Every thread fetches the (cos, sin) pairs of its own rotations from the layer's
//    tables in L2 (int8 angles: the code, decoded as it rotates) when the chain starts,
//    together with the GEMV outputs it needs; no table is staged in shared memory, which
//    leaves it to the weight ring. Theta == 0 (the fixed randomized Hadamard transform)
//    needs no fetch at all.
//  * The residual stream lives in registers, in the layout the last butterfly stage
//    leaves it in.
//  * Grid-wide barriers (release/acquire counters) only where a whole output vector is
//    needed: after q/k/v, o, gate/up, the MLP blocks, and down.
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
//   P7 MLP blocks (one CTA each up to 512 wide, one cluster each from 2048): F_U_gate,
//      F_U_up, silu*up, F_V_down, operand to global; the two last clusters apply F_U_q
//      and F_U_k of this block                  -> grid barrier
//   P8 GEMV down                                -> grid barrier
// and after the last block: out = h_{L-1} + F_U_down(z_down).
//
// Every wait is bounded (about 2 s of SM clock unless the testing hook shortens it) and
// checks a shared abort word, and every outcome that decides control flow is made
// uniform across the consumer threads, so a failure anywhere ends the kernel with
// HARP_ERR_TIMEOUT instead of a hang.
#include "bfly_engine.cuh"
#include "decode.h"
#include "gemv_core.cuh"

namespace harp {
namespace dec {

using namespace gemv_core;

// ------------------------------------------------------------------ GEMV unit geometry
// 32 output rows x 2048 input columns (one group of 64 columns per lane) per unit.
template <int BITS>
struct FGeo {
  static constexpr int kChunkCols = 2048;
  static constexpr int kChunkGroups = kChunkCols / 64;
  static constexpr int kGroupBytes = BITS == 4 ? 32 : 16;  // a group's codes (first plane)
  static constexpr int kRowBatch = 4;  // rows whose loads are in flight at once
};

// ------------------------------------------------------------------ shared memory carve-up

struct Smem : EngCtx {
  float* misc;     // [0, 8) rms partials by source CTA, [8, 24) per-warp scratch
  int32_t* xq;     // GEMV operand: xq words, then xs [ng], then xsum [ng]
  float* red;      // GEMV row partials: 16 warps x 8 rows x 33 (32 lanes, padded)
  struct Plan* plan;
};

__device__ __forceinline__ Smem carve(const Params& p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* b = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~uintptr_t(15));
  Smem s;
  s.T = reinterpret_cast<float*>(b);
  b += 4 * kRxFloats;
  s.rx[0] = reinterpret_cast<float*>(b);
  b += 4 * kRxFloats;
  s.rx[1] = reinterpret_cast<float*>(b);
  b += 4 * kRxFloats;
  s.misc = reinterpret_cast<float*>(b);
  b += 4 * 32;
  s.xq = reinterpret_cast<int32_t*>(b);
  b += p.xq_bytes;
  s.red = reinterpret_cast<float*>(b);
  b += 4 * kCW * 8 * 33;
  s.plan = reinterpret_cast<struct Plan*>(b);
  b += 512;
  s.xbar = reinterpret_cast<uint64_t*>(b);
  return s;
}

// a butterfly's coefficients: from the side's thread-order table when the stack built one
template <int EB, int TM>
__device__ __forceinline__ void fetch_side(ClusterBfly<EB, TM>& bf, const uint8_t* rt, const uint8_t* tab,
                                           int64_t half_n, int64_t blk, uint32_t r, int ct) {
  if (rt) bf.fetch_rt(rt, blk, r, ct);
  else bf.fetch(tab, half_n, blk, r, ct);
}
template <int EB, int TM>
__device__ __forceinline__ void fetch_side(LocalBfly<EB, TM>& bf, const uint8_t* rt, const uint8_t* tab,
                                           int64_t half_n, int64_t blk, int ct) {
  if (rt) bf.fetch_rt(rt, blk, ct);
  else bf.fetch(tab, half_n, blk, ct);
}

// ------------------------------------------------------------------ GEMV operand
// x~ of a hidden-wide input in layout B (runs of >= 64): the CTA's groups into its own
// operand buffer, then to every peer's (one exchange)
template <int EB>
__device__ bool prep_broadcast(const float (&v)[2], int n_in, int bits, Smem& sm, Xch& x, uint32_t r, int ct,
                               int* status) {
  using M = Map<EB>;
  static_assert(M::RUN >= 64, "operand groups must lie inside one run");
  constexpr int GPR = M::RUN / 64, NGL = M::E / 64;  // groups per run, groups of this CTA
  const int warp = ct >> 5, lane = ct & 31;
  const int words = bits == 3 ? n_in : n_in / 2, ng = n_in / 64;
  int16_t* xq16 = reinterpret_cast<int16_t*>(sm.xq);
  float* xsA = reinterpret_cast<float*>(sm.xq + words);
  float* xsumA = xsA + ng;
  cbar();
  if (ct < M::NT)
#pragma unroll
    for (int s = 0; s < M::P; ++s) sm.T[M::idx_b(M::bj(ct), M::bii(ct, s))] = v[s];
  cbar();
  if (warp < NGL) {
    const int j = warp / GPR, kk = warp - j * GPR;
    const int G = (j * M::E + (int)r * M::RUN + 64 * kk) >> 6;
    prep_group(sm.T + j * M::PAD + 64 * kk, bits, xq16 + (int64_t)G * 64, xq16 + n_in + (int64_t)G * 64, xsA + G,
               xsumA + G, lane, G & 7);
  }
  const int planes = bits == 3 ? 2 : 1;
  xch_begin(sm, x, (uint32_t)((kC - 1) * NGL * (128 * planes + 8)), ct);  // starts with a barrier: prep is done
  uint64_t* bar = &sm.xbar[xb_of(x)];
  // 8 int4 per group and plane, to the 7 peers
  for (int it = ct; it < NGL * planes * 8 * (kC - 1); it += kNT) {
    const int qi = it % (kC - 1), rest = it / (kC - 1);
    const int part = rest & 7, pl = (rest >> 3) % planes, lg = (rest >> 3) / planes;
    const uint32_t q = (uint32_t)(qi < (int)r ? qi : qi + 1);
    const int j = lg / GPR, kk = lg - j * GPR;
    const int G = (j * M::E + (int)r * M::RUN + 64 * kk) >> 6;
    const int word = pl * (n_in / 2) + G * 32 + part * 4;
    st_async_v4(sm.xq + word, bar, q, *reinterpret_cast<const int4*>(sm.xq + word));
  }
  for (int it = ct; it < NGL * (kC - 1); it += kNT) {
    const int qi = it % (kC - 1), lg = it / (kC - 1);
    const uint32_t q = (uint32_t)(qi < (int)r ? qi : qi + 1);
    const int j = lg / GPR, kk = lg - j * GPR;
    const int G = (j * M::E + (int)r * M::RUN + 64 * kk) >> 6;
    st_async_f32(xsA + G, bar, q, xsA[G]);
    st_async_f32(xsumA + G, bar, q, xsumA[G]);
  }
  return xch_end(sm, x, status, 40, ct);
}

// sum of the split-K partials of element i (fixed order); the loads are independent and
// go out together (one L2 round trip for up to 16 partials)
__device__ __forceinline__ float zsum(const float* zp, int nk, int64_t n, int64_t i) {
  constexpr int kMaxK = 16;
  float v[kMaxK];
#pragma unroll
  for (int k = 0; k < kMaxK; ++k) v[k] = k < nk ? __ldcg(zp + (int64_t)k * n + i) : 0.f;
  float t = v[0];
#pragma unroll
  for (int k = 1; k < kMaxK; ++k)
    if (k < nk) t += v[k];
  for (int k = kMaxK; k < nk; ++k) t += __ldcg(zp + (int64_t)k * n + i);
  return t;
}

// ------------------------------------------------------------------ chains (cluster-collective)
// Residual chain: [res += F_U(z)] ; n = rms(res) ; x~ = F_V(n) ; operand. EB: log2 of the
// hidden-wide chunk (hidden / 8). U null: res is the step's input; V null: the final step.
template <int EB, int TM>
__device__ __noinline__ bool chain_residual(const Params& p, Smem& sm, Xch& x, float (&res)[2], const Lin* U,
                                            const float* zp, int nk, const Lin* V, uint32_t r, int ct) {
  using M = Map<EB>;
  using BF = ClusterBfly<EB, TM>;
  const bool act = ct < M::NT;
  bool ok = true;
  if (!U) {
    if (act)
#pragma unroll
      for (int s = 0; s < M::P; ++s) res[s] = load_act(p.x_in, BF::gb(r, ct, s), p.xt);
  } else {
    BF fu;
    fetch_side(fu, U->rU, U->tU, (int64_t)U->n_out / 2, 0, r, ct);
    float v[2] = {0.f, 0.f};
    if (act)
#pragma unroll
      for (int s = 0; s < M::P; ++s) {
        const int g = BF::ga(r, ct, s);
        v[s] = zsum(zp, nk, U->n_out, g) * (float)__ldg(U->sU + g);
      }
    ok = fu.run(v, sm, x, r, ct, p.status, 41);
    if (act)
#pragma unroll
      for (int s = 0; s < M::P; ++s) res[s] += v[s];
  }
  if (!V || !ok) return ok;
  BF fv;
  fetch_side(fv, V->rV, V->tV, (int64_t)V->n_in / 2, 0, r, ct);
  float sgn[2] = {0.f, 0.f};  // F_V's signs, read before the exchange (its wait orders memory)
  if (act)
#pragma unroll
    for (int s = 0; s < M::P; ++s) sgn[s] = (float)__ldg(V->sV + (int)r * M::E + M::e1(ct, s));
  // sum of squares: warps, then the CTA (fixed order), then to every peer's slot r along
  // with the residual values each peer holds in layout A for F_V
  float acc = 0.f;
  if (act)
#pragma unroll
    for (int s = 0; s < M::P; ++s) acc = fmaf(res[s], res[s], acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((ct & 31) == 0) sm.misc[8 + (ct >> 5)] = acc;
  xch_begin(sm, x, 4u * M::RUN * (kC - 1) + 4u * (kC - 1), ct);
  if (ct == 0) {
    float t = 0.f;
    for (int w = 0; w < kCW; ++w) t += sm.misc[8 + w];
    for (uint32_t q = 0; q < kC; ++q)
      if (q == r) sm.misc[r] = t;
      else st_async_f32(sm.misc + r, &sm.xbar[xb_of(x)], q, t);
  }
  if (act)
#pragma unroll
    for (int s = 0; s < M::P; ++s) {
      const int j = M::bj(ct), ii = M::bii(ct, s);
      put(sm, x, r, (uint32_t)j, idx_a((int)r * M::RUN + ii), res[s]);
    }
  const float* rx = sm.rx[xb_of(x)];
  if (!(ok = xch_end(sm, x, p.status, 42, ct))) return false;
  float tot = 0.f;
  for (int q = 0; q < kC; ++q) tot += sm.misc[q];
  const float inv = 1.0f / sqrtf(tot / (float)p.hidden + p.eps);
  float v[2] = {0.f, 0.f};
  if (act)
#pragma unroll
    for (int s = 0; s < M::P; ++s) {
      const int e = M::e1(ct, s);
      v[s] = rx[idx_a(e)] * inv * sgn[s];
    }
  if (!(ok = fv.run(v, sm, x, r, ct, p.status, 43))) return false;
  return prep_broadcast<EB>(v, V->n_in, p.bits, sm, x, r, ct, p.status);
}

// attention chain: v = F_U_v(z_v); a = v repeated per KV group; x~ = F_V_o(a); operand.
// EBU: log2 of the v chunk (dkv / 8), EB: of the hidden chunk.
template <int EBU, int EB, int TM>
__device__ __noinline__ bool chain_attn(const Params& p, Smem& sm, Xch& x, const Lin* Lv, const Lin* Lo, uint32_t r,
                                        int ct) {
  using MU = Map<EBU>;
  using M = Map<EB>;
  ClusterBfly<EBU, TM> fu;
  fetch_side(fu, Lv->rU, Lv->tU, (int64_t)Lv->n_out / 2, 0, r, ct);
  float v[2] = {0.f, 0.f};
  if (ct < MU::NT)
#pragma unroll
    for (int s = 0; s < MU::P; ++s) {
      const int g = ClusterBfly<EBU, TM>::ga(r, ct, s);
      v[s] = zsum(p.zpv, p.nk_h, Lv->n_out, g) * (float)__ldg(Lv->sU + g);
    }
  if (!fu.run(v, sm, x, r, ct, p.status, 44)) return false;
  ClusterBfly<EB, TM> fv;
  fetch_side(fv, Lo->rV, Lo->tV, (int64_t)Lo->n_in / 2, 0, r, ct);
  float sgn[2] = {0.f, 0.f};  // F_V's signs, read before the exchange
  if (ct < M::NT)
#pragma unroll
    for (int s = 0; s < M::P; ++s) sgn[s] = (float)__ldg(Lo->sV + (int)r * M::E + M::e1(ct, s));
  // every v value to the layout-A owners of the query-head elements that copy it
  const int hd = p.head_dim, rep = p.rep;
  int self = 0;
  if (ct < MU::NT)
#pragma unroll
    for (int s = 0; s < MU::P; ++s) {
      const int gv = ClusterBfly<EBU, TM>::gb(r, ct, s), kvh = gv / hd, d = gv - kvh * hd;
      for (int h = kvh * rep; h < (kvh + 1) * rep; ++h) self += ((h * hd + d) >> EB) == (int)r;
    }
  self = cbar_sum(self, reinterpret_cast<int*>(sm.misc + 8), ct);
  xch_begin(sm, x, 4u * (uint32_t)(M::E - self), ct);
  if (ct < MU::NT)
#pragma unroll
    for (int s = 0; s < MU::P; ++s) {
      const int gv = ClusterBfly<EBU, TM>::gb(r, ct, s), kvh = gv / hd, d = gv - kvh * hd;
      for (int h = kvh * rep; h < (kvh + 1) * rep; ++h) {
        const int ga = h * hd + d;
        put(sm, x, r, (uint32_t)(ga >> EB), idx_a(ga & (M::E - 1)), v[s]);
      }
    }
  const float* rx = sm.rx[xb_of(x)];
  if (!xch_end(sm, x, p.status, 45, ct)) return false;
  float w[2] = {0.f, 0.f};
  if (ct < M::NT)
#pragma unroll
    for (int s = 0; s < M::P; ++s) {
      const int e = M::e1(ct, s);
      w[s] = rx[idx_a(e)] * sgn[s];
    }
  if (!fv.run(w, sm, x, r, ct, p.status, 46)) return false;
  return prep_broadcast<EB>(w, Lo->n_in, p.bits, sm, x, r, ct, p.status);
}

// F_U of a q or k GEMV output (cluster-distributed), written to out[g]
template <int EB, int TM>
__device__ __noinline__ bool chain_out_only(const Params& p, Smem& sm, Xch& x, const Lin* Lq, const float* zp,
                                            float* out, uint32_t r, int ct) {
  using M = Map<EB>;
  using BF = ClusterBfly<EB, TM>;
  BF fu;
  fetch_side(fu, Lq->rU, Lq->tU, (int64_t)Lq->n_out / 2, 0, r, ct);
  float v[2] = {0.f, 0.f};
  if (ct < M::NT)
#pragma unroll
    for (int s = 0; s < M::P; ++s) {
      const int g = BF::ga(r, ct, s);
      v[s] = zsum(zp, p.nk_h, Lq->n_out, g) * (float)__ldg(Lq->sU + g);
    }
  const bool ok = fu.run(v, sm, x, r, ct, p.status, 47);
  if (ok && ct < M::NT)
#pragma unroll
    for (int s = 0; s < M::P; ++s) out[BF::gb(r, ct, s)] = v[s];
  return ok;
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

// One MLP block of width 2^EB <= 512 in one CTA: F_U_gate, F_U_up, silu * up, F_V_down,
// operand of the down projection for this block (to global)
template <int EB, int TM>
__device__ __noinline__ void mlp_block_local(const Params& p, Smem& sm, const Lin* Lg, const Lin* Lu, const Lin* Ld,
                                             int blk, int ct) {
  using M = Map<EB>;
  if constexpr (2 * M::E <= kNT) {
    // blocks up to 256 wide: F_U(gate) on threads [0, E) and F_U(up) on [E, 2E) at once,
    // each half with its own transpose buffer; the up half then hands its values over
    const bool up = ct >= M::E;
    const int cl = up ? ct - M::E : ct;  // the thread within its half (>= E: idle)
    const Lin* Lx = up ? Lu : Lg;
    LocalBfly<EB, TM> fx, fd;
    fetch_side(fx, Lx->rU, Lx->tU, (int64_t)Lx->n_out / 2, blk, cl);
    if (!up) fetch_side(fd, Ld->rV, Ld->tV, (int64_t)Ld->n_in / 2, blk, cl);
    const bool act = cl < M::NT;
    const int64_t base = (int64_t)blk * M::E;
    float v = 0.f, sd = 0.f;
    if (act) {
      const int64_t g = base + M::e1(cl, 0);
      v = zsum(up ? p.zpu : p.zpg, p.nk_h, Lx->n_out, g) * (float)__ldg(Lx->sU + g);
      if (!up) sd = (float)__ldg(Ld->sV + base + M::e2(cl, 0));  // F_V_down's sign, read up front
    }
    EngCtx half = sm;
    if (up) half.T += 512;
    fx.run(v, half, cl);
    cbar();  // the gate half has read its transpose buffer
    if (act && up) sm.T[idx_a(M::e2(cl, 0))] = v;  // both halves hold phase-2 order
    cbar();
    float h = 0.f;
    if (act && !up) h = silu(v) * sm.T[idx_a(M::e2(cl, 0))] * sd;
    cbar();
    if (act && !up) sm.T[idx_a(M::e2(cl, 0))] = h;
    cbar();
    if (act && !up) h = sm.T[idx_a(M::e1(cl, 0))];
    fd.run(h, sm, up ? M::NT : cl);  // F_V_down from phase-1 order, on the gate half
    cbar();
    if (act && !up) sm.T[M::e2(cl, 0)] = h;  // natural order for the groups
    cbar();
    const int warp = ct >> 5, lane = ct & 31, n_in = Ld->n_in;
    int16_t* xq16 = reinterpret_cast<int16_t*>(p.xq_down);
    if (warp < (M::E >> 6)) {
      const int G = (int)(base >> 6) + warp;
      prep_group(sm.T + 64 * warp, p.bits, xq16 + (int64_t)G * 64, xq16 + n_in + (int64_t)G * 64, p.xs_down + G,
                 p.xsum_down + G, lane, G & 7);
    }
    return;
  }
  LocalBfly<EB, TM> fg, fu, fd;
  fetch_side(fg, Lg->rU, Lg->tU, (int64_t)Lg->n_out / 2, blk, ct);
  fetch_side(fu, Lu->rU, Lu->tU, (int64_t)Lu->n_out / 2, blk, ct);
  fetch_side(fd, Ld->rV, Ld->tV, (int64_t)Ld->n_in / 2, blk, ct);
  const bool act = ct < M::NT;
  const int64_t base = (int64_t)blk * M::E;
  float vg = 0.f, vu = 0.f, sd = 0.f;
  if (act) {
    const int64_t g = base + M::e1(ct, 0);
    vg = zsum(p.zpg, p.nk_h, Lg->n_out, g) * (float)__ldg(Lg->sU + g);
    vu = zsum(p.zpu, p.nk_h, Lu->n_out, g) * (float)__ldg(Lu->sU + g);
    sd = (float)__ldg(Ld->sV + base + M::e2(ct, 0));  // F_V_down's sign, read up front
  }
  fg.run(vg, sm, ct);
  fu.run(vu, sm, ct);
  // both in phase-2 order; F_V_down starts from phase-1 order
  float h = 0.f;
  if (act) h = silu(vg) * vu * sd;
  cbar();
  if (act) sm.T[idx_a(M::e2(ct, 0))] = h;
  cbar();
  if (act) h = sm.T[idx_a(M::e1(ct, 0))];
  fd.run(h, sm, ct);
  cbar();
  if (act) sm.T[M::e2(ct, 0)] = h;  // natural order for the groups
  cbar();
  const int warp = ct >> 5, lane = ct & 31, n_in = Ld->n_in;
  int16_t* xq16 = reinterpret_cast<int16_t*>(p.xq_down);
  if (warp < (M::E >> 6)) {
    const int G = (int)(base >> 6) + warp;
    prep_group(sm.T + 64 * warp, p.bits, xq16 + (int64_t)G * 64, xq16 + n_in + (int64_t)G * 64, p.xs_down + G,
               p.xsum_down + G, lane, G & 7);
  }
}

// One MLP block of width 8 * 2^EB (>= 2048) on one cluster: the same steps, each
// butterfly spread over the cluster; the operand groups go to global from layout B.
template <int EB, int TM>
__device__ __noinline__ bool mlp_block_cluster(const Params& p, Smem& sm, Xch& x, const Lin* Lg, const Lin* Lu,
                                               const Lin* Ld, int blk, uint32_t r, int ct) {
  using M = Map<EB>;
  using BF = ClusterBfly<EB, TM>;
  static_assert(M::RUN >= 64, "operand groups must lie inside one run");
  constexpr int W = kC * M::E;
  const bool act = ct < M::NT;
  const int64_t base = (int64_t)blk * W;
  float vg[2] = {0.f, 0.f}, vu[2] = {0.f, 0.f};
  {
    BF fg;
    fetch_side(fg, Lg->rU, Lg->tU, (int64_t)Lg->n_out / 2, blk, r, ct);
    if (act)
#pragma unroll
      for (int s = 0; s < M::P; ++s) {
        const int64_t g = base + BF::ga(r, ct, s);
        vg[s] = zsum(p.zpg, p.nk_h, Lg->n_out, g) * (float)__ldg(Lg->sU + g);
      }
    if (!fg.run(vg, sm, x, r, ct, p.status, 48)) return false;
  }
  {
    BF fu;
    fetch_side(fu, Lu->rU, Lu->tU, (int64_t)Lu->n_out / 2, blk, r, ct);
    if (act)
#pragma unroll
      for (int s = 0; s < M::P; ++s) {
        const int64_t g = base + BF::ga(r, ct, s);
        vu[s] = zsum(p.zpu, p.nk_h, Lu->n_out, g) * (float)__ldg(Lu->sU + g);
      }
    if (!fu.run(vu, sm, x, r, ct, p.status, 49)) return false;
  }
  BF fd;
  fetch_side(fd, Ld->rV, Ld->tV, (int64_t)Ld->n_in / 2, blk, r, ct);
  float sgn[2] = {0.f, 0.f};  // F_V_down's signs, read before the exchange
  if (act)
#pragma unroll
    for (int s = 0; s < M::P; ++s) sgn[s] = (float)__ldg(Ld->sV + base + (int)r * M::E + M::e1(ct, s));
  // h = silu(gate) * up in layout B, to the layout-A owners
  xch_begin(sm, x, 4u * M::RUN * (kC - 1), ct);
  if (act)
#pragma unroll
    for (int s = 0; s < M::P; ++s)
      put(sm, x, r, (uint32_t)M::bj(ct), idx_a((int)r * M::RUN + M::bii(ct, s)), silu(vg[s]) * vu[s]);
  const float* rx = sm.rx[xb_of(x)];
  if (!xch_end(sm, x, p.status, 50, ct)) return false;
  float v[2] = {0.f, 0.f};
  if (act)
#pragma unroll
    for (int s = 0; s < M::P; ++s) {
      const int e = M::e1(ct, s);
      v[s] = rx[idx_a(e)] * sgn[s];
    }
  if (!fd.run(v, sm, x, r, ct, p.status, 51)) return false;
  // groups of 64 inside the runs, to the global down operand
  constexpr int GPR = M::RUN / 64, NGL = M::E / 64;
  cbar();
  if (act)
#pragma unroll
    for (int s = 0; s < M::P; ++s) sm.T[M::idx_b(M::bj(ct), M::bii(ct, s))] = v[s];
  cbar();
  const int warp = ct >> 5, lane = ct & 31, n_in = Ld->n_in;
  int16_t* xq16 = reinterpret_cast<int16_t*>(p.xq_down);
  if (warp < NGL) {
    const int j = warp / GPR, kk = warp - j * GPR;
    const int G = (int)((base + j * M::E + (int)r * M::RUN + 64 * kk) >> 6);
    prep_group(sm.T + j * M::PAD + 64 * kk, p.bits, xq16 + (int64_t)G * 64, xq16 + n_in + (int64_t)G * 64,
               p.xs_down + G, p.xsum_down + G, lane, G & 7);
  }
  return true;
}

// ------------------------------------------------------------------ GEMV work units
// A unit is 32 output rows x one 2048-column chunk of one linear.
// Units are numbered chunk-major (u = kc * tiles + tile), so the consecutive units a CTA
// takes mostly share their chunk of the operand.
struct Range {
  const Lin* L;
  float* zp;  // partial sums [nk][n_out]
  int n_in, n_out;
  int nk, nt, u0, u1;  // chunks, 32-row tiles, the CTA's units [u0, u1)
  __device__ __forceinline__ void tk(int u, int& tile, int& kc) const {
    kc = u / nt;
    tile = u - kc * nt;
  }
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
  g.n_in = g.L->n_in;
  g.n_out = g.L->n_out;
  g.nk = (g.n_in + FGeo<BITS>::kChunkCols - 1) / FGeo<BITS>::kChunkCols;
  g.nt = (g.n_out + 31) / 32;
  const int U = g.nt * g.nk;
  g.u0 = split(U, i, parts);
  g.u1 = split(U, i + 1, parts);
  return g;
}

__device__ __forceinline__ void prefetch_line_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// L2 requests for this warp's rows of range g, the same rows run_units will take (rows
// rw and rw + 16 of every unit, rw turned by the phase's first unit index k0): lanes 0..7
// (0..15 at 4 bits) ask for the 128-byte lines of the two rows' codes in the chunk, lanes
// 16, 17 for their scale/zero words, lanes 18..21 for their 1-bit plane (3 bits). Plain
// prefetches from every lane: nothing queues behind the TMA unit.
template <int BITS>
__device__ __forceinline__ void prefetch_rows(const Range& g, uint32_t k0, int warp, int lane) {
  using Gm = FGeo<BITS>;
  const int ngroups = g.n_in / 64, row_bytes = ngroups * Gm::kGroupBytes;
  const int rw = (warp - (int)(k0 & 15)) & 15;
  constexpr int LPR = 2048 * (BITS == 4 ? 4 : 2) / 8 / 128;  // code lines per row of a chunk
  for (int i = 0; i < g.u1 - g.u0; ++i) {
    int tile, kc;
    g.tk(g.u0 + i, tile, kc);
    const int g0 = kc * Gm::kChunkGroups, gc = min(Gm::kChunkGroups, ngroups - g0);
    int row, bytes = 0;
    const uint8_t* src = nullptr;
    if (lane < 2 * LPR) {
      row = tile * 32 + rw + 16 * (lane / LPR);
      const int o = (lane % LPR) * 128;
      if (o < gc * Gm::kGroupBytes) {
        src = g.L->codes + (size_t)row * row_bytes + (size_t)g0 * Gm::kGroupBytes + o;
        bytes = 1;
      }
    } else if (lane == 16 || lane == 17) {
      row = tile * 32 + rw + 16 * (lane - 16);
      src = reinterpret_cast<const uint8_t*>(g.L->sz + (size_t)row * ngroups + g0);
      bytes = 1;
    } else if (BITS == 3 && lane >= 18 && lane < 22) {
      row = tile * 32 + rw + 16 * ((lane - 18) >> 1);
      const int o = ((lane - 18) & 1) * 128;
      if (o < gc * 8) {
        src = g.L->hi + (size_t)row * (ngroups * 8) + (size_t)g0 * 8 + o;
        bytes = 1;
      }
    }
    if (bytes && row < g.n_out) prefetch_line_l2(src);
  }
}

// The CTA's ranges of block 0 by phase, and how they move per block (the next block's
// linears are 7 Lin further; q and k partials have a buffer per block): worked out once and
// kept in shared memory, so finding a unit chases no pointer in global memory.
struct Plan {
  Range r0[4];
  long long zstride[4];  // partial-sum offset per block
  int nb;                // the CTA's units per block
};

template <int BITS>
__device__ __forceinline__ void make_plan(const Params& p, int c, int r, Plan& q) {
  q.nb = 0;
  for (int ph = 0; ph < 4; ++ph) {
    q.r0[ph] = units<BITS>(p, 0, ph, c, r);
    q.zstride[ph] = p.L > 1 ? units<BITS>(p, 1, ph, c, r).zp - q.r0[ph].zp : 0;
    q.nb += q.r0[ph].u1 - q.r0[ph].u0;
  }
}

__device__ __forceinline__ Range range_of(const Plan& q, int l, int ph) {
  Range g = q.r0[ph];
  g.L += 7 * l;
  g.zp += (long long)l * q.zstride[ph];
  return g;
}

// ------------------------------------------------------------------ GEMV
// Every warp takes two rows of every unit of the CTA's range (rows rw and rw + 16, rw
// turned by the CTA's unit count from phase to phase), and lane l the unit's group l (64
// input columns). The lane loads its own bytes of each row straight from global memory (a
// warp reads each row's chunk as one contiguous, coalesced span; the phase's weights were
// requested into L2 a phase earlier), two units' rows in flight at once when they share a
// chunk, and keeps its operand words in registers while the chunk stays the same. No data
// passes between warps but the row sums: a warp's per-lane partials go through its own
// scratch in shared memory, and eight lanes add up each row, in a fixed order.
constexpr int kRowsW = 8;  // rows of scratch per warp (four are used)
constexpr int kRedRow = 33;  // scratch row stride: the adders' reads hit 32 distinct banks

// 16-byte chunk k of operand group G in shared memory (and in the down operand in global):
// swizzled by G, so that lanes holding consecutive groups read distinct banks
__device__ __forceinline__ int xq_chunk(int G, int k) { return (G << 3) | (k ^ (G & 7)); }

// one row's data for one lane: the group's codes (first plane), its 1-bit plane (3-bit)
// and its scale/zero word
template <int BITS>
struct RowW {
  uint4 c[BITS == 4 ? 2 : 1];
  uint2 h;
  uint32_t sz;
};

template <int BITS>
__device__ __forceinline__ void load_row(RowW<BITS>& w, const Range& g, int row, int G, int ngroups) {
  using Gm = FGeo<BITS>;
  const uint4* cp = reinterpret_cast<const uint4*>(g.L->codes + ((size_t)row * ngroups + G) * Gm::kGroupBytes);
  w.c[0] = ldg_nc_u4(cp);
  if constexpr (BITS == 4) w.c[1] = ldg_nc_u4(cp + 1);
  if constexpr (BITS == 3) w.h = ldg_nc_u2(reinterpret_cast<const uint2*>(g.L->hi + ((size_t)row * ngroups + G) * 8));
  w.sz = ldg_nc_u32(g.L->sz + (size_t)row * ngroups + G);
}

// exact integer dot product of one row's group with the operand words x of that group;
// xh: the 1-bit plane's operand (3-bit)
template <int BITS>
__device__ __forceinline__ int row_dot(const RowW<BITS>& rw, const int4 (&x)[8], const int4* xh, int G) {
  if constexpr (BITS == 2 || BITS == 3) {
    const uint32_t wv[4] = {rw.c[0].x, rw.c[0].y, rw.c[0].z, rw.c[0].w};
    int a0 = 0, a1 = 0, a2 = 0, a3 = 0, b0 = 0, b1 = 0, b2 = 0, b3 = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int4 xa = x[2 * k], xb = x[2 * k + 1];
      const uint32_t w = wv[k];
      const uint32_t m0 = w & 0x03030303u, m1 = w & 0x0C0C0C0Cu, m2 = w & 0x30303030u, m3 = w & 0xC0C0C0C0u;
      a0 = dp2a_lo(xa.x, m0, a0);
      b0 = dp2a_hi(xa.y, m0, b0);
      a1 = dp2a_lo(xa.z, m1, a1);
      b1 = dp2a_hi(xa.w, m1, b1);
      a2 = dp2a_lo(xb.x, m2, a2);
      b2 = dp2a_hi(xb.y, m2, b2);
      a3 = dp2a_lo(xb.z, m3, a3);
      b3 = dp2a_hi(xb.w, m3, b3);
    }
    int acc = (a0 + b0) + ((a1 + b1) >> 2) + ((a2 + b2) >> 4) + ((a3 + b3) >> 6);  // exact shifts
    if constexpr (BITS == 3) {
      const uint32_t hv[2] = {rw.h.x, rw.h.y};
      int h = 0;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
#pragma unroll
        for (int mm = 0; mm < 8; mm += 2) {
          const int4 xa = xh[xq_chunk(G, 4 * k + mm / 2)];
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
    const uint32_t wv[8] = {rw.c[0].x, rw.c[0].y, rw.c[0].z, rw.c[0].w, rw.c[1].x, rw.c[1].y, rw.c[1].z, rw.c[1].w};
    int lo = 0, hi = 0, lo2 = 0, hi2 = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int4 xa = x[k];
      const uint32_t ml = wv[k] & 0x0F0F0F0Fu, mh = wv[k] & 0xF0F0F0F0u;
      lo = dp2a_lo(xa.x, ml, lo);
      lo2 = dp2a_hi(xa.y, ml, lo2);
      hi = dp2a_lo(xa.z, mh, hi);
      hi2 = dp2a_hi(xa.w, mh, hi2);
    }
    return (lo + lo2) + ((hi + hi2) >> 4);
  }
}

template <int BITS>
__device__ __noinline__ bool run_units(const Params& p, Smem& s, const Range& g, uint32_t& kring, int ct) {
  using Gm = FGeo<BITS>;
  const int warp = ct >> 5, lane = ct & 31;
  const int n_out = g.n_out, n_in = g.n_in, ngroups = n_in / 64;
  const int words = BITS == 3 ? n_in : n_in / 2;
  const float* xsA = reinterpret_cast<const float*>(s.xq + words);
  const float* xsumA = xsA + ngroups;
  const int4* xlo = reinterpret_cast<const int4*>(s.xq);
  const int4* xhi = reinterpret_cast<const int4*>(s.xq + n_in / 2);
  const int nu = g.u1 - g.u0;
  // rows rw and rw + 16 of every unit; the mapping turns with the CTA's unit count so that
  // no warp keeps the same rows phase after phase
  const int rw = (warp - (int)(kring & 15)) & 15;
  int4 xr[8];
  float xs = 0.f, xsum = 0.f;
  int kc_have = -1;
  float* red = s.red + warp * (kRowsW * kRedRow);
  for (int i = 0; i < nu;) {
    // this unit and, when it has the same chunk, the next: up to four rows in flight
    int tile[2], kc;
    g.tk(g.u0 + i, tile[0], kc);
    tile[1] = tile[0];
    int nb = 1;
    if (i + 1 < nu) {
      int t1, k1;
      g.tk(g.u0 + i + 1, t1, k1);
      if (k1 == kc) {
        tile[1] = t1;
        nb = 2;
      }
    }
    const int g0 = kc * Gm::kChunkGroups, gc = min(Gm::kChunkGroups, ngroups - g0);
    const bool act = lane < gc;
    const int G = g0 + lane;
    if (kc != kc_have) {
      kc_have = kc;
      if (act) {
#pragma unroll
        for (int k = 0; k < 8; ++k) xr[k] = xlo[xq_chunk(G, k)];
        xs = xsA[G];
        xsum = xsumA[G];
      }
    }
    RowW<BITS> w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int row = tile[j >> 1] * 32 + rw + 16 * (j & 1);
      if ((j >> 1) < nb && act && row < n_out) load_row<BITS>(w[j], g, row, G, ngroups);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int row = tile[j >> 1] * 32 + rw + 16 * (j & 1);
      float z = 0.f;
      if ((j >> 1) < nb && act && row < n_out) {
        const float s16 = __half2float(__ushort_as_half((unsigned short)(w[j].sz & 0xffffu)));
        const float z16 = __half2float(__ushort_as_half((unsigned short)(w[j].sz >> 16)));
        const int acc = row_dot<BITS>(w[j], xr, xhi, G);
        z = fmaf(s16, (float)acc * xs, z16 * xsum);
      }
      red[j * kRedRow + lane] = z;
    }
    __syncwarp();
    // row j = lane / 8: lane % 8 adds lanes 4 (lane % 8) .. + 3, then the eight
    float t = 0.f;
    {
      const float* rp = red + (lane >> 3) * kRedRow + (lane & 7) * 4;
#pragma unroll
      for (int k = 0; k < 4; ++k) t += rp[k];
    }
    t += __shfl_xor_sync(0xffffffffu, t, 1);
    t += __shfl_xor_sync(0xffffffffu, t, 2);
    t += __shfl_xor_sync(0xffffffffu, t, 4);
    __syncwarp();  // the scratch is free for the next rows
    {
      const int j = lane >> 3, row = tile[j >> 1] * 32 + rw + 16 * (j & 1);
      if ((lane & 7) == 0 && (j >> 1) < nb && row < n_out) g.zp[(int64_t)kc * n_out + row] = t;
    }
    i += nb;
  }
  kring += (uint32_t)nu;
  return cbar_and(true);
}

// as GEMV phase ph of block l starts (its first unit is the CTA's kring-th): this
// warp's rows of the following phase into L2
template <int BITS>
__device__ __forceinline__ void prefetch_next(const Params& p, Smem& s, int l, int ph, uint32_t kring, int ct) {
  if (p.pf_dist == 0) return;
  const Plan& q = *s.plan;
  const uint32_t k0 = kring + (uint32_t)(q.r0[ph].u1 - q.r0[ph].u0);
  if (++ph == 4) {
    ph = 0;
    if (++l >= p.L) return;
  }
  prefetch_rows<BITS>(range_of(q, l, ph), k0, ct >> 5, ct & 31);
}

// This CTA's rows of GEMV phase (l, ph) into L2, spread over the lanes of warps 1..15 while
// thread 0 polls a grid barrier (those warps would only wait): line by line, codes and
// 1-bit plane of each row's chunk, then its scale/zero words.
template <int BITS>
__device__ __forceinline__ void prefetch_phase_l2(const Params& p, const Smem& s, int l, int ph, int ct) {
  using Gm = FGeo<BITS>;
  if (l >= p.L) return;
  const Range g = range_of(*s.plan, l, ph);
  const int ngroups = g.n_in / 64, row_bytes = ngroups * Gm::kGroupBytes;
  constexpr int kLines = 2048 * (BITS == 4 ? 4 : 2) / 8 / 128 + (BITS == 3 ? 2 : 0) + 1;  // per row of a chunk
  const int per_unit = 32 * kLines;
  for (int it = ct - 32; it < (g.u1 - g.u0) * per_unit; it += kNT - 32) {
    const int i = it / per_unit, rest = it - i * per_unit, row_in = rest / kLines, ln = rest - row_in * kLines;
    int tile, kc;
    g.tk(g.u0 + i, tile, kc);
    const int row = tile * 32 + row_in;
    if (row >= g.n_out) continue;
    const int g0 = kc * Gm::kChunkGroups, gc = min(Gm::kChunkGroups, ngroups - g0);
    constexpr int kCodeLines = 2048 * (BITS == 4 ? 4 : 2) / 8 / 128;
    if (ln < kCodeLines) {
      if (ln * 128 < gc * Gm::kGroupBytes)
        prefetch_line_l2(g.L->codes + (size_t)row * row_bytes + (size_t)g0 * Gm::kGroupBytes + ln * 128);
    } else if (BITS == 3 && ln < kCodeLines + 2) {
      if ((ln - kCodeLines) * 128 < gc * 8)
        prefetch_line_l2(g.L->hi + (size_t)row * (ngroups * 8) + (size_t)g0 * 8 + (ln - kCodeLines) * 128);
    } else {
      prefetch_line_l2(g.L->sz + (size_t)row * ngroups + g0);
    }
  }
}

// ------------------------------------------------------------------ waits on global counters
// CTA-wide: thread 0 polls until *c >= target (acquire), bounded like every wait here
__device__ __noinline__ bool wait_count(const Params& p, const unsigned* c, unsigned target, int where, int ct) {
  bool mine = true;
  if (ct == 0) {
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
          report(p.status, 5, where);
          mine = false;
          break;
        }
      }
    }
  }
  return cbar_and(mine);
}

// ------------------------------------------------------------------ grid barrier
// pf_l, pf_ph: a GEMV phase whose rows warps 1..15 ask for in L2 meanwhile (pf_l < 0: none);
// synced: the caller has just passed a CTA barrier (a GEMV phase's end), so every thread's
// writes are already ordered before thread 0's release
template <int BITS>
__device__ __noinline__ bool grid_barrier(const Params& p, const Smem& s, int idx, int ct, int pf_l = -1,
                                          int pf_ph = 0, bool synced = false) {
  if (!synced) cbar();
  if (ct >= 32 && pf_l >= 0 && p.bar_pf) prefetch_phase_l2<BITS>(p, s, pf_l, pf_ph, ct);
  bool mine = true;
  if (ct == 0) {
    // the CTA barrier above orders every thread's writes before this release, which makes
    // them visible with the count at gpu scope (no separate fence)
    unsigned* c = p.counters + idx;
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

// ------------------------------------------------------------------ chain dispatch
// the widths come from the stack's shapes at run time; each width has its instantiation
template <int TM>
__device__ __forceinline__ bool residual_any(const Params& p, Smem& sm, Xch& x, float (&res)[2], const Lin* U,
                                             const float* zp, int nk, const Lin* V, uint32_t r, int ct) {
  return p.eb_h == 10 ? chain_residual<10, TM>(p, sm, x, res, U, zp, nk, V, r, ct)
                      : chain_residual<9, TM>(p, sm, x, res, U, zp, nk, V, r, ct);
}

template <int TM, int EB>
__device__ __forceinline__ bool attn_eb(const Params& p, Smem& sm, Xch& x, const Lin* Lv, const Lin* Lo, uint32_t r,
                                        int ct) {
  switch (p.eb_kv) {
    case 5: return chain_attn<5, EB, TM>(p, sm, x, Lv, Lo, r, ct);
    case 6: return chain_attn<6, EB, TM>(p, sm, x, Lv, Lo, r, ct);
    case 7: return chain_attn<7, EB, TM>(p, sm, x, Lv, Lo, r, ct);
    case 8: return chain_attn<8, EB, TM>(p, sm, x, Lv, Lo, r, ct);
    case 9: return chain_attn<9, EB, TM>(p, sm, x, Lv, Lo, r, ct);
    default: return chain_attn<10, EB, TM>(p, sm, x, Lv, Lo, r, ct);
  }
}

template <int TM>
__device__ __forceinline__ bool out_only_any(const Params& p, Smem& sm, Xch& x, int eb, const Lin* Lq,
                                             const float* zp, float* out, uint32_t r, int ct) {
  switch (eb) {
    case 5: return chain_out_only<5, TM>(p, sm, x, Lq, zp, out, r, ct);
    case 6: return chain_out_only<6, TM>(p, sm, x, Lq, zp, out, r, ct);
    case 7: return chain_out_only<7, TM>(p, sm, x, Lq, zp, out, r, ct);
    case 8: return chain_out_only<8, TM>(p, sm, x, Lq, zp, out, r, ct);
    case 9: return chain_out_only<9, TM>(p, sm, x, Lq, zp, out, r, ct);
    default: return chain_out_only<10, TM>(p, sm, x, Lq, zp, out, r, ct);
  }
}

// MLP blocks of phase P7: eb_blk = log2(block width); <= 9: one CTA per block, else one
// cluster per block (4096 or 8192 wide: log2 of the per-CTA share = eb_blk - 3)
template <int TM>
__device__ __forceinline__ bool mlp_any(const Params& p, Smem& sm, Xch& x, const Lin* lin, int c, uint32_t r,
                                        int ct) {
  const int t_cta = c * kC + (int)r;
  switch (p.eb_blk) {
    case 6:
      if (t_cta < p.nblocks) mlp_block_local<6, TM>(p, sm, lin + 4, lin + 5, lin + 6, t_cta, ct);
      return true;
    case 7:
      if (t_cta < p.nblocks) mlp_block_local<7, TM>(p, sm, lin + 4, lin + 5, lin + 6, t_cta, ct);
      return true;
    case 8:
      if (t_cta < p.nblocks) mlp_block_local<8, TM>(p, sm, lin + 4, lin + 5, lin + 6, t_cta, ct);
      return true;
    case 9:
      if (t_cta < p.nblocks) mlp_block_local<9, TM>(p, sm, lin + 4, lin + 5, lin + 6, t_cta, ct);
      return true;
    case 12: return c < p.nblocks ? mlp_block_cluster<9, TM>(p, sm, x, lin + 4, lin + 5, lin + 6, c, r, ct) : true;
    default: return c < p.nblocks ? mlp_block_cluster<10, TM>(p, sm, x, lin + 4, lin + 5, lin + 6, c, r, ct) : true;
  }
}

// one local MLP block (width <= 512) by index
template <int TM>
__device__ __forceinline__ void mlp_local_blk(const Params& p, Smem& sm, const Lin* lin, int blk, int ct) {
  switch (p.eb_blk) {
    case 6: mlp_block_local<6, TM>(p, sm, lin + 4, lin + 5, lin + 6, blk, ct); break;
    case 7: mlp_block_local<7, TM>(p, sm, lin + 4, lin + 5, lin + 6, blk, ct); break;
    case 8: mlp_block_local<8, TM>(p, sm, lin + 4, lin + 5, lin + 6, blk, ct); break;
    default: mlp_block_local<9, TM>(p, sm, lin + 4, lin + 5, lin + 6, blk, ct); break;
  }
}

// P7 roles: MLP-block CTAs or clusters first, the last two clusters apply F_U_q / F_U_k
__device__ __forceinline__ int qk_cluster(const Params& p, int which) { return p.G - 1 - which; }

// L2 hint for this CTA's slice of a side's thread-order table (cluster layout: CTA r's
// entries are contiguous) and of its sign vector
__device__ __forceinline__ void prefetch_side(const uint8_t* rt, const int8_t* sign, int eb, int tm, uint32_t r) {
  if (!rt) return;
  const int E = 1 << eb, nt = E < kNT ? E : kNT, P = E > kNT ? E / kNT : 1;
  const uint32_t bytes = (uint32_t)((eb + 3) * P * (nt / 2) * (tm == kTmCS ? 8 : 4));
  bulk_prefetch_l2(rt + (size_t)r * bytes, bytes);
  if (E % 16 == 0) bulk_prefetch_l2(sign + (size_t)r * E, (uint32_t)E);
}

// L2 hint for one block of a side kept in the local (one CTA per block) thread order, and
// for that block's signs
__device__ __forceinline__ void prefetch_block(const uint8_t* rt, const int8_t* sign, int eb, int tm, int blk) {
  if (!rt) return;
  const int E = 1 << eb, nt = E < kNT ? E : kNT;
  const uint32_t bytes = (uint32_t)(eb * (nt / 2) * (tm == kTmCS ? 8 : 4));
  bulk_prefetch_l2(rt + (size_t)blk * bytes, bytes);
  if (E % 16 == 0) bulk_prefetch_l2(sign + (size_t)blk * E, (uint32_t)E);
}

// the tables of the chain that follows GEMV phase ph of block l (one thread, as the phase
// starts)
__device__ __forceinline__ void prefetch_chain(const Params& p, int l, int ph, int c, uint32_t r) {
  const Lin* lin = p.lin + 7 * l;
  if (ph == 0) {  // P3: F_U of v, F_V of o
    prefetch_side(lin[2].rU, lin[2].sU, p.eb_kv, p.tm, r);
    prefetch_side(lin[3].rV, lin[3].sV, p.eb_h, p.tm, r);
  } else if (ph == 1) {  // P5: F_U of o, F_V of the cluster's gate or up
    prefetch_side(lin[3].rU, lin[3].sU, p.eb_h, p.tm, r);
    prefetch_side(lin[4 + p.asg_gu[c]].rV, lin[4 + p.asg_gu[c]].sV, p.eb_h, p.tm, r);
  } else if (ph == 2) {  // P7: the MLP block this CTA runs (up to 512 wide), F_U of q or k
    const int t_cta = c * kC + (int)r;
    if (p.eb_blk <= 9 && t_cta < p.nblocks) {
      prefetch_block(lin[4].rU, lin[4].sU, p.eb_blk, p.tm, t_cta);
      prefetch_block(lin[5].rU, lin[5].sU, p.eb_blk, p.tm, t_cta);
      prefetch_block(lin[6].rV, lin[6].sV, p.eb_blk, p.tm, t_cta);
    }
    if (c == qk_cluster(p, 0)) prefetch_side(lin[0].rU, lin[0].sU, p.eb_h, p.tm, r);
    if (c == qk_cluster(p, 1)) prefetch_side(lin[1].rU, lin[1].sU, p.eb_kv, p.tm, r);
  } else if (ph == 3) {  // next P1: F_U of down, F_V of the cluster's q, k or v in block l + 1
    prefetch_side(lin[6].rU, lin[6].sU, p.eb_h, p.tm, r);
    if (l + 1 < p.L) {
      const Lin* nx = lin + 7 + p.asg_qkv[c];
      prefetch_side(nx->rV, nx->sV, p.eb_h, p.tm, r);
    }
  }
}

// ------------------------------------------------------------------ the kernel
// TM: how every butterfly of the stack keeps its angles (kTmCS, kTmHad, kTmQ8); each form
// has its own instantiation, so no rotation branches on it.
template <int BITS, int TM>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ Params p) {
  using Gm = FGeo<BITS>;
  Smem s = carve(p);
  const uint32_t r = cta_rank();
  const int c = (int)cluster_id_x();
  const int tid = threadIdx.x;

  if (tid == 0) {
    make_plan<BITS>(p, c, (int)r, *s.plan);
    s_wait_cycles = p.wait_cycles;
    mbar_init(&s.xbar[0], 1);
    mbar_init(&s.xbar[1], 1);
    fence_mbar_init();
  }
  cluster_sync_all();  // every CTA's barriers exist before any remote store signals one

  const int L = p.L;
  const int ct = tid;
  // the first GEMV phase's weights into L2 while the first chain runs
  if (p.pf_dist > 0)
    prefetch_rows<BITS>(range_of(*s.plan, 0, 0), 0, ct >> 5, ct & 31);
  uint32_t kring = 0;
  Xch X;
  float res[2] = {0.f, 0.f};  // the residual stream, this CTA's layout-B share
  bool ok = true;

  for (int l = 0; l < L && ok; ++l) {
    const Lin* lin = p.lin + 7 * l;
    const Lin* prev = l > 0 ? p.lin + 7 * (l - 1) : nullptr;
    // P1
    if (!(ok = residual_any<TM>(p, s, X, res, prev ? prev + 6 : nullptr, p.zpd, p.nk_f, lin + p.asg_qkv[c], r,
                                ct)))
      break;
    // P2 (L2 requests for the tables of the chain that follows, as every GEMV phase)
    if (ct == 0 && p.table_pf && p.tm != kTmHad) prefetch_chain(p, l, 0, c, r);
    prefetch_next<BITS>(p, s, l, 0, kring, ct);
    if (!(ok = run_units<BITS>(p, s, range_of(*s.plan, l, 0), kring, ct))) break;
    if (!(ok = grid_barrier<BITS>(p, s, l * 5 + 0, ct, l, 1, true))) break;
    // P3
    if (!(ok = p.eb_h == 10 ? attn_eb<TM, 10>(p, s, X, lin + 2, lin + 3, r, ct)
                            : attn_eb<TM, 9>(p, s, X, lin + 2, lin + 3, r, ct)))
      break;
    // P4
    if (ct == 0 && p.table_pf && p.tm != kTmHad) prefetch_chain(p, l, 1, c, r);
    prefetch_next<BITS>(p, s, l, 1, kring, ct);
    if (!(ok = run_units<BITS>(p, s, range_of(*s.plan, l, 1), kring, ct))) break;
    if (!(ok = grid_barrier<BITS>(p, s, l * 5 + 1, ct, l, 2, true))) break;
    // P5
    if (!(ok = residual_any<TM>(p, s, X, res, lin + 3, p.zpo, p.nk_h, lin + 4 + p.asg_gu[c], r, ct))) break;
    // P6
    if (ct == 0 && p.table_pf && p.tm != kTmHad) prefetch_chain(p, l, 2, c, r);
    prefetch_next<BITS>(p, s, l, 2, kring, ct);
    if (p.mlp_ready) {
      // no grid barrier: each CTA adds its gate/up units, once they are all written, to the
      // counters of the MLP blocks they belong to (one fence for the lot), and CTA b runs
      // MLP block b as soon as its count reaches the block's 2 x wb/32 x nk units
      const Range g6 = range_of(*s.plan, l, 2);
      if (!(ok = run_units<BITS>(p, s, g6, kring, ct))) break;
      const int wb = lin[4].w_out;
      unsigned* ready = p.counters + 5 * L + (size_t)l * p.nblocks;
      if (ct == 0) {
        __threadfence();
        int cur = -1;
        unsigned cnt = 0;
        for (int u = g6.u0; u <= g6.u1; ++u) {
          int b = -2;
          if (u < g6.u1) {
            int tile, kc;
            g6.tk(u, tile, kc);
            b = tile * 32 / wb;
          }
          if (b != cur) {
            if (cnt) asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(ready + cur), "r"(cnt) : "memory");
            cur = b;
            cnt = 0;
          }
          ++cnt;
        }
      }
      const int t_cta = c * kC + (int)r;
      if (t_cta < p.nblocks) {
        if (!(ok = wait_count(p, ready + t_cta, (unsigned)(2 * (wb / 32) * p.nk_h), 70, ct))) break;
        mlp_local_blk<TM>(p, s, lin, t_cta, ct);
      } else if (ct >= 32 && p.bar_pf) {
        prefetch_phase_l2<BITS>(p, s, l, 3, ct);  // idle until the MLP blocks are done
      }
    } else {
      if (!(ok = run_units<BITS>(p, s, range_of(*s.plan, l, 2), kring, ct))) break;
      if (!(ok = grid_barrier<BITS>(p, s, l * 5 + 2, ct, l, 3, true))) break;
      // P7
      if (!(ok = mlp_any<TM>(p, s, X, lin, c, r, ct))) break;
    }
    {
      const int qk = c == qk_cluster(p, 0) ? 0 : (c == qk_cluster(p, 1) ? 1 : -1);
      if (qk >= 0) {
        float* out = qk == 0 ? p.qout + (int64_t)l * lin[0].n_out : p.kout + (int64_t)l * lin[1].n_out;
        const float* zp = qk == 0 ? p.zpq + (int64_t)l * p.nk_h * lin[0].n_out
                                  : p.zpk + (int64_t)l * p.nk_h * lin[1].n_out;
        if (!(ok = out_only_any<TM>(p, s, X, qk == 0 ? p.eb_h : p.eb_kv, lin + qk, zp, out, r, ct))) break;
      }
    }
    if (!(ok = grid_barrier<BITS>(p, s, l * 5 + 3, ct))) break;
    // P8: the down projection's operand from global into shared memory, then the GEMV
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
      if (ct == 0 && p.table_pf && p.tm != kTmHad) prefetch_chain(p, l, 3, c, r);
      prefetch_next<BITS>(p, s, l, 3, kring, ct);
      if (!(ok = run_units<BITS>(p, s, range_of(*s.plan, l, 3), kring, ct))) break;
    }
    if (!(ok = grid_barrier<BITS>(p, s, l * 5 + 4, ct, l + 1, 0, true))) break;
  }
  // final: out = h_{L-1} + F_U_down(z_down)
  if (ok) {
    const Lin* last = p.lin + 7 * (L - 1);
    ok = residual_any<TM>(p, s, X, res, last + 6, p.zpd, p.nk_f, nullptr, r, ct);
    if (ok && c == 0) {
      const int E = p.hidden / kC;
      for (int sl = 0; sl < 2; ++sl) {
        if (sl * kNT >= E || ct >= (E < kNT ? E : kNT)) continue;
        const int run = E / kC;
        const int g = (ct & 7) * E + (int)r * run + (((ct & 31) >> 3) | ((ct >> 5) << 2) | (sl << 6));
        store_act(p.y_out, g, p.yt, res[sl]);
      }
    }
  }
  cluster_sync_all();
}

// ------------------------------------------------------------------ thread-order tables
size_t repack_bytes(int tm, int eb, bool cluster, int nblk) {
  if (tm == kTmHad) return 0;
  const int E = 1 << eb, nt = E < kNT ? E : kNT, P = cluster && E > kNT ? E / kNT : 1;
  const int ns = cluster ? eb + 3 : eb, nr = cluster ? kC : 1;
  return (size_t)nblk * nr * ns * P * (nt / 2) * (tm == kTmCS ? 8 : 4);
}

template <int TM, bool CLUSTER>
static cudaError_t repack_t(int eb, int nblk, const uint8_t* tab, int64_t half_n, uint8_t* rt, cudaStream_t st) {
  const int grid = 296, thr = 256;
  switch (eb) {
    case 5: if (CLUSTER) repack_kernel<5, TM, CLUSTER><<<grid, thr, 0, st>>>(tab, half_n, nblk, rt); else return cudaErrorInvalidValue; break;
    case 6: repack_kernel<6, TM, CLUSTER><<<grid, thr, 0, st>>>(tab, half_n, nblk, rt); break;
    case 7: repack_kernel<7, TM, CLUSTER><<<grid, thr, 0, st>>>(tab, half_n, nblk, rt); break;
    case 8: repack_kernel<8, TM, CLUSTER><<<grid, thr, 0, st>>>(tab, half_n, nblk, rt); break;
    case 9: repack_kernel<9, TM, CLUSTER><<<grid, thr, 0, st>>>(tab, half_n, nblk, rt); break;
    case 10: if (CLUSTER) repack_kernel<10, TM, CLUSTER><<<grid, thr, 0, st>>>(tab, half_n, nblk, rt); else return cudaErrorInvalidValue; break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t repack_side(int tm, int eb, bool cluster, int nblk, const uint8_t* tab, int64_t half_n, uint8_t* rt,
                        cudaStream_t st) {
  if (tm == kTmCS) return cluster ? repack_t<kTmCS, true>(eb, nblk, tab, half_n, rt, st)
                                  : repack_t<kTmCS, false>(eb, nblk, tab, half_n, rt, st);
  if (tm == kTmQ8) return cluster ? repack_t<kTmQ8, true>(eb, nblk, tab, half_n, rt, st)
                                  : repack_t<kTmQ8, false>(eb, nblk, tab, half_n, rt, st);
  return cudaSuccess;
}

// ------------------------------------------------------------------ host side
template <int BITS>
size_t smem_bytes(const Params& p) {
  return 16 + 3 * 4 * (size_t)kRxFloats + 4 * 32 + p.xq_bytes + 4 * kCW * 8 * 33 + 512 + 8 * 2;
}

template <int BITS>
const void* kernel_ptr(int tm) {
  return tm == kTmHad  ? reinterpret_cast<const void*>(decode_kernel<BITS, kTmHad>)
         : tm == kTmQ8 ? reinterpret_cast<const void*>(decode_kernel<BITS, kTmQ8>)
                       : reinterpret_cast<const void*>(decode_kernel<BITS, kTmCS>);
}

// The grid barriers need every CTA resident at once. The launch asks for that explicitly
// (cooperative), so a grid that cannot be co-resident -- because other work holds SMs --
// is refused at launch instead of timing out in its first barrier.
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
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kC;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  // A driver that does not take the cooperative attribute together with cluster dimensions
  // gets the plain cluster launch (co-residency then rests on the occupancy query made at
  // set-up); a grid too large to be co-resident is refused either way.
  static int coop_ok[64] = {0};  // 0 unknown, 1 accepted, -1 not accepted (per device)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  const bool coop = p.cooperative && coop_ok[dev] >= 0;
  cfg.numAttrs = coop ? 2 : 1;
  auto go = [&]() -> cudaError_t {
    if (p.tm == kTmHad) return cudaLaunchKernelEx(&cfg, decode_kernel<BITS, kTmHad>, p);
    if (p.tm == kTmQ8) return cudaLaunchKernelEx(&cfg, decode_kernel<BITS, kTmQ8>, p);
    return cudaLaunchKernelEx(&cfg, decode_kernel<BITS, kTmCS>, p);
  };
  e = go();
  if (coop && coop_ok[dev] == 0) {
    if (e == cudaSuccess) {
      coop_ok[dev] = 1;
    } else if (e != cudaErrorCooperativeLaunchTooLarge) {
      cudaGetLastError();
      coop_ok[dev] = -1;
      cfg.numAttrs = 1;
      e = go();
    }
  }
  return e;
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
  return bits == 2 ? FGeo<2>::kChunkCols : (bits == 3 ? FGeo<3>::kChunkCols : FGeo<4>::kChunkCols);
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
