// Inner pieces of the dequant-GEMV shared by the stand-alone GEMV kernel and the fused
// decode-step kernel: TMA box geometry, swizzled shared-memory addressing and the
// exact int16 x u2/u3/u4 group dot product built on dp2a.
#pragma once

#include "common.cuh"

namespace harp {
namespace gemv_core {

constexpr int kSlab = 32 * 128;  // one TMA box: 32 rows x 128 bytes
constexpr int kXStageMax = 64 * 1024;  // activation operand staged in shared memory up to this size

// One ring stage holds one unit of work: 32 rows x one chunk of input columns. Chunks of
// 4096 columns (2048 for 4-bit codes) make stages of 36-56 KB, which keeps the number of
// per-unit hand-offs low; TMA rings sustain only a few million stages per second per SM.
template <int BITS>
struct Geo {
  static constexpr int kChunkCols = BITS == 4 ? 2048 : 4096;  // columns per stage
  static constexpr int kChunkGroups = kChunkCols / 64;
  static constexpr int kGroupsPerSlab = BITS == 4 ? 4 : 8;       // codes (or 2-bit plane)
  static constexpr int kCodeSlabs = kChunkGroups / kGroupsPerSlab;
  static constexpr int kHiSlabs = BITS == 3 ? kChunkGroups / 16 : 0;  // 1-bit plane
  static constexpr int kSzSlabs = kChunkGroups / 32;                  // scale/zero, 32 groups per box
  static constexpr int kStageBytes = (kCodeSlabs + kHiSlabs + kSzSlabs) * kSlab;
  static constexpr int kStages = BITS == 3 ? 2 : (BITS == 2 ? 3 : 4);  // stand-alone GEMV ring (<= 160 KB)
};


// Address of the 16-byte chunk `c` (0..7) of `row` inside a 128B-swizzled box.
__device__ __forceinline__ const uint8_t* swz(const uint8_t* slab, int row, int c) {
  return slab + row * 128 + ((c ^ (row & 7)) << 4);
}

// scale_zero word of group gl (of the chunk) for `row`, from the stage's scale/zero boxes
__device__ __forceinline__ uint32_t sz_word(const uint8_t* szs, int row, int gl) {
  return *reinterpret_cast<const uint32_t*>(swz(szs + (gl >> 5) * kSlab, row, (gl >> 2) & 7) + (gl & 3) * 4);
}

template <bool XS>
__device__ __forceinline__ int4 ldx(const int4* p) {
  if constexpr (XS) return *p;  // shared memory, same address in every lane: a broadcast
  else return ldg_nc_v4(p);
}

template <int BITS, bool XS>
__device__ __forceinline__ int group_dot(const uint8_t* codes_slabs, const uint8_t* hi_slabs, int lane,
                                         int gl, const int4* __restrict__ xg, const int4* __restrict__ xgh) {
  if constexpr (BITS == 2 || BITS == 3) {
    const uint4 cw = *reinterpret_cast<const uint4*>(swz(codes_slabs + (gl >> 3) * kSlab, lane, gl & 7));
    const uint32_t wv[4] = {cw.x, cw.y, cw.z, cw.w};
    // eight independent accumulator chains (lo/hi byte pairs of each mask) for ILP
    int a0 = 0, a1 = 0, a2 = 0, a3 = 0, b0 = 0, b1 = 0, b2 = 0, b3 = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int4 xa = ldx<XS>(xg + 2 * k), xb = ldx<XS>(xg + 2 * k + 1);
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
    // each (a_m + b_m) is an exact multiple of 4^m: the shifts are exact
    int acc = (a0 + b0) + ((a1 + b1) >> 2) + ((a2 + b2) >> 4) + ((a3 + b3) >> 6);
    if constexpr (BITS == 3) {
      const int gh = gl & 15;
      const uint2 hw = *reinterpret_cast<const uint2*>(swz(hi_slabs + (gl >> 4) * kSlab, lane, gh >> 1) + (gh & 1) * 8);
      const uint32_t hv[2] = {hw.x, hw.y};
      int h = 0;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
#pragma unroll
        for (int mm = 0; mm < 8; mm += 2) {
          const int4 xa = ldx<XS>(xgh + 4 * k + mm / 2);
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
    int lo = 0, hi = 0, lo2 = 0, hi2 = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int4 xa = ldx<XS>(xg + k);
      const uint32_t ml = wv[k] & 0x0F0F0F0Fu, mh = wv[k] & 0xF0F0F0F0u;
      lo = dp2a_lo(xa.x, ml, lo);
      lo2 = dp2a_hi(xa.y, ml, lo2);
      hi = dp2a_lo(xa.z, mh, hi);
      hi2 = dp2a_hi(xa.w, mh, hi2);
    }
    return (lo + lo2) + ((hi + hi2) >> 4);
  }
}


}  // namespace gemv_core
}  // namespace harp
