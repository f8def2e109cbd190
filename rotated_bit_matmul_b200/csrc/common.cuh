// Device helpers shared by the sm_100a kernels of the rotated low-bit linear.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "harp_internal.h"

namespace harp {

// ------------------------------------------------------------------ dtypes
__device__ __forceinline__ float load_act(const void* p, int64_t i, int dt) {
  if (dt == DT_F32) return static_cast<const float*>(p)[i];
  if (dt == DT_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
  return __half2float(static_cast<const __half*>(p)[i]);
}

__device__ __forceinline__ void store_act(void* p, int64_t i, int dt, float v) {
  if (dt == DT_F32) static_cast<float*>(p)[i] = v;
  else if (dt == DT_BF16) static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else static_cast<__half*>(p)[i] = __float2half_rn(v);
}

// ------------------------------------------------------------------ status word
// Records the first device-side failure (code, where) for the host to read.
__device__ __forceinline__ void report(int* status, int code, int where) {
  if (status && atomicCAS(status, 0, code) == 0) atomicExch(status + 1, where);
}

// ------------------------------------------------------------------ shared-memory barriers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// raises the barrier's expected transaction bytes without arriving
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, but a thread that finds the phase incomplete may sleep up to
// `hint_ns` (it wakes when the phase completes) instead of returning at once.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait: gives up (after reporting HARP_ERR_TIMEOUT with `where`) once
// `limit_ns` of wall time (read from %globaltimer) has passed without the phase
// completing. The caller then skips its remaining work and exits.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status, int where,
                                          uint64_t limit_ns = 1000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) break;
  }
  report(status, 5 /* HARP_ERR_TIMEOUT */, where);
  return false;
}

// Bounded wait for one thread of a warp (the others meet it at __syncwarp): sleeps in
// slices of up to 0.2 ms, gives up after `limit_ns` like mbar_wait.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, int* status, int where,
                                                uint64_t limit_ns = 1000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait_sleep(bar, parity, 200000u))
    if (globaltimer_ns() - t0 > limit_ns) {
      report(status, 5 /* HARP_ERR_TIMEOUT */, where);
      return false;
    }
  return true;
}

// ------------------------------------------------------------------ TMA (no multicast)
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 1-D bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16)
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// hint: bring `bytes` (a multiple of 16, 16-byte aligned) of global memory into L2
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// hint: bring one box of a 2-D tensor map into L2 (no shared memory, no completion)
__device__ __forceinline__ void tma_prefetch_l2_2d(const void* tmap, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(tmap), "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ------------------------------------------------------------------ integer dot products
// acc + a.lo16 * b.byte0 + a.hi16 * b.byte1 (a: two signed int16, b: unsigned bytes)
__device__ __forceinline__ int dp2a_lo(int a, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// acc + a.lo16 * b.byte2 + a.hi16 * b.byte3
__device__ __forceinline__ int dp2a_hi(int a, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// read-only global loads of streamed weights (no L1 allocation: each byte is read once)
__device__ __forceinline__ uint4 ldg_nc_u4(const uint4* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ldg_nc_u2(const uint2* p) {
  uint2 v;
  asm("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ldg_nc_u32(const uint32_t* p) {
  uint32_t v;
  asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ int4 ldg_nc_v4(const int4* p) {
  int4 v;
  asm("ld.global.nc.v4.s32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Position (int16 index inside the group's 32-word block) of column j (0..63) of a
// group in the dp2a pair order the GEMV expects for its code format.
__device__ __forceinline__ int xq_pos_lo(int bits, int j) {
  if (bits == 4) {
    const int c = j >> 3, r = j & 7;
    return (c * 4 + (r & 1) * 2 + (r >> 2)) * 2 + ((r >> 1) & 1);
  }
  const int c = j >> 4, r = j & 15, m = r & 3, q = r >> 2;  // 2-bit codes / 2-bit plane
  return (c * 8 + 2 * m + (q >> 1)) * 2 + (q & 1);
}
__device__ __forceinline__ int xq_pos_hi(int j) {  // 1-bit plane of 3-bit codes
  const int c = j >> 5, r = j & 31, m = r & 7, q = r >> 3;
  return (c * 16 + 2 * m + (q >> 1)) * 2 + (q & 1);
}

// Scale exponent of a group of the GEMV operand: the e in [-126, 126] with
// max|v| * 2^e in [2^14, 2^15), i.e. 15 - E for max|v| = f 2^E, f in [0.5, 1), read straight
// from the exponent field (a denormal maximum takes the largest scale, 126).
__device__ __forceinline__ int group_exponent(float amax) {
  const int field = (int)((__float_as_uint(amax) >> 23) & 0xffu);
  const int E = field == 0 ? -126 : field - 126;
  return min(max(15 - E, -126), 126);
}
// 2^e for e in [-126, 127], exact
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((e + 127) << 23); }

// int16 GEMV operand of one group of 64 values v[0..63] (one warp): the values at scale
// 2^e with max |v| 2^e in [2^14, 2^15), in dp2a pair order (and the 1-bit-plane order for
// 3-bit codes); lane 0 writes the scale 2^-e and the fp32 group sum. A non-finite value
// makes the group's scale and sum NaN.
// key: the group's 16-byte chunks are stored at chunk ^ key (0: in order; a consumer that
// keeps one group per lane swizzles them to spread its reads over the banks)
__device__ __forceinline__ void prep_group(const float* v, int bits, int16_t* grp, int16_t* grp_hi, float* xs,
                                           float* xsum, int lane, int key = 0) {
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
  const int kx = key << 3;  // 8 int16 per chunk
  grp[xq_pos_lo(bits, 2 * lane) ^ kx] = (int16_t)q0;
  grp[xq_pos_lo(bits, 2 * lane + 1) ^ kx] = (int16_t)q1;
  if (bits == 3) {
    grp_hi[xq_pos_hi(2 * lane) ^ kx] = (int16_t)q0;
    grp_hi[xq_pos_hi(2 * lane + 1) ^ kx] = (int16_t)q1;
  }
  if (lane == 0) {
    *xs = bad ? __int_as_float(0x7fc00000) : pow2f(-ex);
    *xsum = bad ? __int_as_float(0x7fc00000) : sum;
  }
}

}  // namespace harp
