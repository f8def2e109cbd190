// C ABI of the rotated low-bit linear library: argument checks, layer handles,
// workspace layout and kernel dispatch. Declarations and contracts: include/harp.h.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>

#include "harp_internal.h"
#include "mma.h"

using namespace harp;

namespace {

thread_local std::string g_last_error;

harp_status fail(harp_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

harp_status cuda_fail(cudaError_t e, const char* what) {
  return fail(HARP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define HARP_CUDA(call, what)                       \
  do {                                              \
    cudaError_t e_ = (call);                        \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int log2_exact(int64_t w) {
  if (w < 1) return -1;
  int m = 0;
  while ((int64_t(1) << m) < w) ++m;
  return (int64_t(1) << m) == w ? m : -1;
}

bool valid_dtype(int dt) { return dt == HARP_F32 || dt == HARP_BF16 || dt == HARP_F16; }

// ------------------------------------------------------------------ device status words
std::mutex g_status_mu;
int* g_status[64] = {nullptr};

harp_status device_status_ptr(int** out) {
  int dev = 0;
  HARP_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(HARP_ERR_UNSUPPORTED, "device index %d >= 64", dev);
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status[dev]) {
    int* p = nullptr;
    HARP_CUDA(cudaMalloc(&p, 4 * sizeof(int)), "cudaMalloc(status)");
    HARP_CUDA(cudaMemset(p, 0, 4 * sizeof(int)), "cudaMemset(status)");
    HARP_CUDA(cudaDeviceSynchronize(), "cudaDeviceSynchronize");
    g_status[dev] = p;
  }
  *out = g_status[dev];
  return HARP_OK;
}

// ------------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D row-major tensor [rows][inner] of `esize`-byte elements, box 32 rows x 128 bytes,
// 128-byte swizzle, zero fill out of bounds.
harp_status make_tmap(CUtensorMap* tm, const void* base, CUtensorMapDataType dt, int esize, uint64_t inner,
                      uint64_t rows, uint64_t row_bytes) {
  if (!encode_fn()) return fail(HARP_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (!harp::encode_map_2d(tm, dt, base, inner, rows, row_bytes, (uint32_t)(128 / esize), 32,
                           CU_TENSOR_MAP_SWIZZLE_128B))
    return fail(HARP_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  return HARP_OK;
}

harp_status check_bfly_args(int64_t n, int w, int batch, const float* theta, const int8_t* sign, const void* x,
                            int xt, const void* y, int yt) {
  if (n <= 0 || n > (int64_t(1) << 30)) return fail(HARP_ERR_INVALID_ARG, "butterfly: n=%lld out of range", (long long)n);
  if (log2_exact(w) < 1 || w > kMaxW) return fail(HARP_ERR_INVALID_ARG, "butterfly: w=%d must be a power of two in [2, 8192]", w);
  if (n % w) return fail(HARP_ERR_INVALID_ARG, "butterfly: w=%d does not divide n=%lld", w, (long long)n);
  if (batch < 0 || batch > 65535) return fail(HARP_ERR_INVALID_ARG, "butterfly: batch=%d out of range", batch);
  if (!valid_dtype(xt) || !valid_dtype(yt)) return fail(HARP_ERR_INVALID_ARG, "butterfly: unknown dtype");
  if (!sign || !x || !y) return fail(HARP_ERR_INVALID_ARG, "butterfly: null pointer");
  if ((theta && !aligned16(theta)) || !aligned16(sign) || !aligned16(x) || !aligned16(y))
    return fail(HARP_ERR_INVALID_ARG, "butterfly: device pointers must be 16-byte aligned");
  if (x == y && xt != yt) return fail(HARP_ERR_INVALID_ARG, "butterfly: in-place needs equal dtypes");
  return HARP_OK;
}

harp_status bfly_common(int64_t n, int w, int batch, const float* theta, const int8_t* sign, const void* x,
                        harp_dtype xt, void* y, harp_dtype yt, void* stream, int inverse) {
  harp_status st = check_bfly_args(n, w, batch, theta, sign, x, xt, y, yt);
  if (st != HARP_OK) return st;
  if (batch == 0) return HARP_OK;
  int* status = nullptr;
  if ((st = device_status_ptr(&status)) != HARP_OK) return st;
  BflyParams p{};
  p.n = n;
  p.w = w;
  p.m = log2_exact(w);
  p.inverse = inverse;
  p.theta = theta;
  p.cs = nullptr;
  p.sign = sign;
  p.x = x;
  p.xt = xt;
  p.x_stride = n;
  p.y = y;
  p.yt = yt;
  p.y_stride = n;
  p.status = status;
  HARP_CUDA(launch_butterfly(p, batch, static_cast<cudaStream_t>(stream)), "butterfly launch");
  return HARP_OK;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

}  // namespace

namespace harp {

bool encode_map_2d(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(tm, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int xq_words_per_row(int64_t n_in, int bits) { return (int)(bits == 3 ? n_in : n_in / 2); }

LinearWs linear_ws_layout(const Layer& L, int batch, void* base) {
  LinearWs w{};
  const int64_t ng = L.n_in / kGroup;
  size_t off = 0;
  char* b = static_cast<char*>(base);
  auto carve = [&](size_t bytes) -> void* {
    const size_t o = off;
    off = align256(off + bytes);
    return b ? b + o : nullptr;
  };
  if (batch >= kMinBatchMma) {
    w.x16_ld = mma::x16_ld(L.n_in);
    w.xf = static_cast<float*>(carve(sizeof(float) * (size_t)batch * (size_t)L.n_in));
    w.x16 = carve(2 * (size_t)batch * (size_t)w.x16_ld);
    w.rowscale = static_cast<float*>(carve(sizeof(float) * (size_t)batch));
    w.zpart = static_cast<float*>(carve(sizeof(float) * (size_t)L.msplits * (size_t)batch * (size_t)L.n_out));
    if (L.mrU) w.zmr = static_cast<float*>(carve(sizeof(float) * (size_t)batch * (size_t)L.n_out));
  } else {
    if (L.mrV) w.xmr = static_cast<float*>(carve(sizeof(float) * (size_t)batch * (size_t)L.n_in));
    w.xq_stride = xq_words_per_row(L.n_in, L.bits);
    w.g_stride = ng;
    w.xq = static_cast<int32_t*>(carve(sizeof(int32_t) * (size_t)batch * (size_t)w.xq_stride));
    w.xs = static_cast<float*>(carve(sizeof(float) * (size_t)batch * (size_t)ng));
    w.xsum = static_cast<float*>(carve(sizeof(float) * (size_t)batch * (size_t)ng));
    w.z = static_cast<float*>(carve(sizeof(float) * (size_t)batch * (size_t)L.n_out));
  }
  w.bytes = off;
  return w;
}

// Enqueues y = F_U(dequant(codes) F_V(x)) on st; arguments already validated.
harp_status linear_forward(const Layer& L, int batch, const void* x, int xt, int64_t x_stride, void* y, int yt,
                           int64_t y_stride, void* ws, cudaStream_t st) {
  int* status = nullptr;
  harp_status s = device_status_ptr(&status);
  if (s != HARP_OK) return s;
  return linear_forward_status(L, batch, x, xt, x_stride, y, yt, y_stride, ws, st, status);
}

// y = F_U(dequant(codes) F_V(x)) with mixed-radix sides: the plans' transforms around
// the radix-2 layers' GEMV (operand prepared from the fp32 transform) or tensor-core
// contraction (split partials summed before the output transform)
static harp_status mr_linear_forward(const Layer& L, int batch, const void* x, int xt, int64_t x_stride, void* y,
                                     int yt, int64_t y_stride, void* ws, cudaStream_t st, int* status) {
  if (x_stride != L.n_in || y_stride != L.n_out)
    return fail(HARP_ERR_UNSUPPORTED, "mixed-radix linear: rows must be contiguous");
  LinearWs w = linear_ws_layout(L, batch, ws);
  const float* z = nullptr;
  if (batch >= kMinBatchMma) {
    HARP_CUDA(launch_mr(L.mrV, 0, batch, x, xt, w.xf, DT_F32, st), "input transform launch");
    HARP_CUDA(mma::launch_x16_prep(w.xf, L.n_in, L.bits, batch, static_cast<__half*>(w.x16), w.rowscale, status, st),
              "operand prep launch");
    mma::Call c{};
    c.x16 = static_cast<const __half*>(w.x16);
    c.ld = w.x16_ld;
    c.rowscale = w.rowscale;
    c.zpart = w.zpart;
    c.batch = batch;
    c.status = status;
    HARP_CUDA(mma::launch(L, c, st), "dequant-MMA launch");
    HARP_CUDA(launch_sum_splits(w.zpart, L.msplits, (int64_t)batch * L.n_out, w.zmr, st), "split sum launch");
    z = w.zmr;
  } else {
    HARP_CUDA(launch_mr(L.mrV, 0, batch, x, xt, w.xmr, DT_F32, st), "input transform launch");
    HARP_CUDA(launch_operand_prep(w.xmr, L.n_in, L.bits, batch, w.xq, w.xq_stride, w.xs, w.xsum, w.g_stride, st),
              "operand prep launch");
    for (int b0 = 0; b0 < batch; b0 += kMaxBatchGemv) {
      GemvParams gp{};
      const TestHooks th = test_hooks();
      gp.wait_ns = th.wait_ns;
      gp.skip_stage = th.gemv_skip_stage;
      gp.n_out = (int)L.n_out;
      gp.n_in = (int)L.n_in;
      gp.bits = L.bits;
      gp.batch = batch - b0 < kMaxBatchGemv ? batch - b0 : kMaxBatchGemv;
      gp.xq = w.xq + (int64_t)b0 * w.xq_stride;
      gp.xq_stride = w.xq_stride;
      gp.xs = w.xs + (int64_t)b0 * w.g_stride;
      gp.xsum = w.xsum + (int64_t)b0 * w.g_stride;
      gp.g_stride = w.g_stride;
      gp.z = w.z + (int64_t)b0 * L.n_out;
      gp.z_stride = L.n_out;
      gp.status = status;
      HARP_CUDA(launch_gemv(L, gp, st), "dequant-GEMV launch");
    }
    z = w.z;
  }
  // z is this call's own workspace: the transform may use it between its launches
  HARP_CUDA(launch_mr(L.mrU, 0, batch, z, DT_F32, y, yt, st, const_cast<float*>(z)), "output transform launch");
  return HARP_OK;
}

harp_status linear_forward_status(const Layer& L, int batch, const void* x, int xt, int64_t x_stride, void* y,
                                  int yt, int64_t y_stride, void* ws, cudaStream_t st, int* status) {
  if (L.mrV) return mr_linear_forward(L, batch, x, xt, x_stride, y, yt, y_stride, ws, st, status);
  LinearWs w = linear_ws_layout(L, batch, ws);
  const bool tc = batch >= kMinBatchMma;

  BflyParams pv{};
  pv.n = L.n_in;
  pv.w = L.w_in;
  pv.m = L.m_in;
  pv.inverse = 0;
  pv.cs = L.csV;
  pv.q8 = L.q8V;
  pv.sign = L.sV;
  pv.x = x;
  pv.xt = xt;
  pv.x_stride = x_stride;
  pv.status = status;
  if (tc) {
    // x~ in fp32, then the fp16 operand with its group sums
    pv.y = w.xf;
    pv.yt = DT_F32;
    pv.y_stride = L.n_in;
    HARP_CUDA(launch_butterfly(pv, batch, st), "input butterfly launch");
    HARP_CUDA(mma::launch_x16_prep(w.xf, L.n_in, L.bits, batch, static_cast<__half*>(w.x16), w.rowscale, status, st),
              "operand prep launch");
    mma::Call c{};
    c.x16 = static_cast<const __half*>(w.x16);
    c.ld = w.x16_ld;
    c.rowscale = w.rowscale;
    c.zpart = w.zpart;
    c.batch = batch;
    c.status = status;
    if (mma::fuses(L, batch)) {  // output butterfly inside the tensor-core kernel
      c.y = y;
      c.yt = yt;
      c.y_stride = y_stride;
      HARP_CUDA(mma::launch(L, c, st), "dequant-MMA launch");
      return HARP_OK;
    }
    HARP_CUDA(mma::launch(L, c, st), "dequant-MMA launch");
  } else {
    pv.y = nullptr;
    pv.xq = w.xq;
    pv.xs = w.xs;
    pv.xsum = w.xsum;
    pv.bits = L.bits;
    pv.xq_stride = w.xq_stride;
    pv.g_stride = w.g_stride;
    HARP_CUDA(launch_butterfly(pv, batch, st), "input butterfly launch");

    for (int b0 = 0; b0 < batch; b0 += kMaxBatchGemv) {
      GemvParams gp{};
      const TestHooks th = test_hooks();
      gp.wait_ns = th.wait_ns;
      gp.skip_stage = th.gemv_skip_stage;
      gp.n_out = (int)L.n_out;
      gp.n_in = (int)L.n_in;
      gp.bits = L.bits;
      gp.batch = batch - b0 < kMaxBatchGemv ? batch - b0 : kMaxBatchGemv;
      gp.xq = w.xq + (int64_t)b0 * w.xq_stride;
      gp.xq_stride = w.xq_stride;
      gp.xs = w.xs + (int64_t)b0 * w.g_stride;
      gp.xsum = w.xsum + (int64_t)b0 * w.g_stride;
      gp.g_stride = w.g_stride;
      gp.z = w.z + (int64_t)b0 * L.n_out;
      gp.z_stride = L.n_out;
      gp.status = status;
      HARP_CUDA(launch_gemv(L, gp, st), "dequant-GEMV launch");
    }
  }

  BflyParams pu{};
  pu.n = L.n_out;
  pu.w = L.w_out;
  pu.m = L.m_out;
  pu.inverse = 0;
  pu.cs = L.csU;
  pu.q8 = L.q8U;
  pu.sign = L.sU;
  pu.x = tc ? w.zpart : w.z;
  pu.xt = DT_F32;
  pu.x_stride = L.n_out;
  pu.nsum = tc ? L.msplits : 1;
  pu.sum_stride = (int64_t)batch * L.n_out;
  pu.y = y;
  pu.yt = yt;
  pu.y_stride = y_stride;
  pu.status = status;
  HARP_CUDA(launch_butterfly(pu, batch, st), "output butterfly launch");
  return HARP_OK;
}

harp_status device_status_for_kernels(int** out) { return device_status_ptr(out); }

namespace {
std::atomic<uint64_t> g_hook_wait_ns{0};
std::atomic<long long> g_hook_wait_cycles{0};
std::atomic<int> g_hook_gemv_skip{-1};
std::atomic<int> g_hook_barrier_extra{-1};
}  // namespace

TestHooks test_hooks() {
  TestHooks h;
  const uint64_t ns = g_hook_wait_ns.load();
  const long long cyc = g_hook_wait_cycles.load();
  h.wait_ns = ns ? ns : 1000000000ull;         // 1 s of wall time
  h.wait_cycles = cyc ? cyc : 4000000000ll;    // about 2 s of SM clock at 1.97 GHz
  h.gemv_skip_stage = g_hook_gemv_skip.load();
  h.decode_barrier_extra = g_hook_barrier_extra.load();
  return h;
}

harp_status set_error(harp_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

}  // namespace harp

extern "C" {

const char* harp_last_error(void) { return g_last_error.c_str(); }

harp_status harp_test_set_faults(int wait_limit_us, int gemv_skip_stage, int decode_barrier) {
  if (wait_limit_us < 0 || gemv_skip_stage < -1 || decode_barrier < -1)
    return fail(HARP_ERR_INVALID_ARG, "test_set_faults: negative limit or index");
  g_hook_wait_ns.store((uint64_t)wait_limit_us * 1000ull);
  // the fused step counts SM clock cycles: 2 per nanosecond covers clocks up to 2 GHz
  g_hook_wait_cycles.store((long long)wait_limit_us * 2000ll);
  g_hook_gemv_skip.store(gemv_skip_stage);
  g_hook_barrier_extra.store(decode_barrier);
  return HARP_OK;
}

harp_status harp_device_status(void* stream) {
  int* status = nullptr;
  harp_status st = device_status_ptr(&status);
  if (st != HARP_OK) return st;
  int host[2] = {0, 0};
  HARP_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "cudaStreamSynchronize");
  HARP_CUDA(cudaMemcpy(host, status, sizeof host, cudaMemcpyDeviceToHost), "cudaMemcpy(status)");
  if (host[0] == 0) return HARP_OK;
  HARP_CUDA(cudaMemset(status, 0, 4 * sizeof(int)), "cudaMemset(status)");
  HARP_CUDA(cudaDeviceSynchronize(), "cudaDeviceSynchronize");
  return fail((harp_status)host[0], "device reported status %d at site %d", host[0], host[1]);
}

harp_status harp_butterfly_fwd(int64_t n, int w, int batch, const float* theta, const int8_t* sign, const void* x,
                               harp_dtype xt, void* y, harp_dtype yt, void* stream) {
  return bfly_common(n, w, batch, theta, sign, x, xt, y, yt, stream, 0);
}

harp_status harp_butterfly_inv(int64_t n, int w, int batch, const float* theta, const int8_t* sign, const void* x,
                               harp_dtype xt, void* y, harp_dtype yt, void* stream) {
  return bfly_common(n, w, batch, theta, sign, x, xt, y, yt, stream, 1);
}

harp_status harp_quantize_weights(int64_t n_out, int64_t n_in, int bits, int group, const float* W_rot, void* codes,
                                  void* scale_zero, void* stream) {
  if (bits < 2 || bits > 4) return fail(HARP_ERR_INVALID_ARG, "quantize: bits=%d not in {2,3,4}", bits);
  if (group != kGroup) return fail(HARP_ERR_UNSUPPORTED, "quantize: group=%d (only 64 is supported)", group);
  if (n_out <= 0 || n_in <= 0 || n_in % 64 || n_out > (int64_t(1) << 24) || n_in > (int64_t(1) << 24))
    return fail(HARP_ERR_INVALID_ARG, "quantize: n_out=%lld n_in=%lld (need n_in %% 64 == 0)", (long long)n_out,
                (long long)n_in);
  if (!W_rot || !codes || !scale_zero) return fail(HARP_ERR_INVALID_ARG, "quantize: null pointer");
  if (!aligned16(W_rot) || !aligned16(codes) || !aligned16(scale_zero))
    return fail(HARP_ERR_INVALID_ARG, "quantize: device pointers must be 16-byte aligned");
  HARP_CUDA(launch_quantize(n_out, n_in, bits, W_rot, codes, scale_zero, static_cast<cudaStream_t>(stream)),
            "quantize launch");
  return HARP_OK;
}

namespace {

harp_status layer_maps(Layer& L);

// One side's angles: raw theta (cos/sin tables are built), int8 codes with their steps
// (copied into the layer's int8 storage), or neither (Theta = 0).
struct SideAngles {
  const float* theta;
  const int8_t* q8;
  const float* delta;
};

harp_status create_layer_impl(harp_layer* out, int64_t n_in, int64_t n_out, int bits, int group, int w_in, int w_out,
                              SideAngles av, const int8_t* sign_V, SideAngles au, const int8_t* sign_U,
                              const void* codes, const void* scale_zero, void* stream) {
  if (!out) return fail(HARP_ERR_INVALID_ARG, "create_layer: null output handle");
  *out = nullptr;
  if (bits < 2 || bits > 4) return fail(HARP_ERR_INVALID_ARG, "create_layer: bits=%d not in {2,3,4}", bits);
  if (group != kGroup) return fail(HARP_ERR_UNSUPPORTED, "create_layer: group=%d (only 64 is supported)", group);
  if (n_in <= 0 || n_in % 256 || n_in > 65536)
    return fail(HARP_ERR_INVALID_ARG, "create_layer: n_in=%lld must be a positive multiple of 256, <= 65536",
                (long long)n_in);
  if (n_out <= 0 || n_out > 65536) return fail(HARP_ERR_INVALID_ARG, "create_layer: n_out=%lld out of range", (long long)n_out);
  const int m_in = log2_exact(w_in), m_out = log2_exact(w_out);
  if (m_in < 6 || w_in > kMaxW || n_in % w_in)
    return fail(HARP_ERR_INVALID_ARG, "create_layer: w_in=%d must be a power of two in [64, 8192] dividing n_in", w_in);
  if (m_out < 1 || w_out > kMaxW || n_out % w_out)
    return fail(HARP_ERR_INVALID_ARG, "create_layer: w_out=%d must be a power of two in [2, 8192] dividing n_out", w_out);
  if (!sign_V || !sign_U || !codes || !scale_zero) return fail(HARP_ERR_INVALID_ARG, "create_layer: null pointer");
  const float* theta_V = av.theta;
  const float* theta_U = au.theta;
  if ((av.q8 && !av.delta) || (au.q8 && !au.delta))
    return fail(HARP_ERR_INVALID_ARG, "create_layer_q8: int8 angles need their per-stage steps");
  if ((theta_V && !aligned16(theta_V)) || !aligned16(sign_V) || (theta_U && !aligned16(theta_U)) ||
      !aligned16(sign_U) || !aligned16(codes) || !aligned16(scale_zero) || (av.q8 && !aligned16(av.q8)) ||
      (au.q8 && !aligned16(au.q8)) || (av.delta && !aligned16(av.delta)) || (au.delta && !aligned16(au.delta)))
    return fail(HARP_ERR_INVALID_ARG, "create_layer: device pointers must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  harp_layer_s* h = new (std::nothrow) harp_layer_s();
  if (!h) return fail(HARP_ERR_INVALID_ARG, "create_layer: out of host memory");
  Layer& L = h->L;
  L.n_in = n_in;
  L.n_out = n_out;
  L.bits = bits;
  L.group = group;
  L.w_in = w_in;
  L.w_out = w_out;
  L.m_in = m_in;
  L.m_out = m_out;
  L.codes = codes;
  L.scale_zero = scale_zero;
  cudaGetDevice(&L.device);
  const int64_t cnt_v = (int64_t)m_in * (n_in / 2), cnt_u = (int64_t)m_out * (n_out / 2);
  auto cleanup = [&](harp_status s) {
    cudaFree(L.csV);
    cudaFree(L.csU);
    cudaFree(L.q8V);
    cudaFree(L.q8U);
    cudaFree(L.sV);
    cudaFree(L.sU);
    delete h;
    return s;
  };
  cudaError_t e;
  // a side with a null theta is the fixed randomized Hadamard transform: no table
  if ((theta_V && (e = cudaMalloc(&L.csV, sizeof(float2) * cnt_v)) != cudaSuccess) ||
      (theta_U && (e = cudaMalloc(&L.csU, sizeof(float2) * cnt_u)) != cudaSuccess) ||
      (e = cudaMalloc(&L.sV, (size_t)n_in)) != cudaSuccess || (e = cudaMalloc(&L.sU, (size_t)n_out)) != cudaSuccess)
    return cleanup(cuda_fail(e, "create_layer: cudaMalloc"));
  if ((theta_V && (e = launch_cs_table(theta_V, cnt_v, L.csV, st)) != cudaSuccess) ||
      (theta_U && (e = launch_cs_table(theta_U, cnt_u, L.csU, st)) != cudaSuccess) ||
      (e = cudaMemcpyAsync(L.sV, sign_V, (size_t)n_in, cudaMemcpyDeviceToDevice, st)) != cudaSuccess ||
      (e = cudaMemcpyAsync(L.sU, sign_U, (size_t)n_out, cudaMemcpyDeviceToDevice, st)) != cudaSuccess)
    return cleanup(cuda_fail(e, "create_layer: copies"));
  // int8 angles: a zeroed 64-byte head with the m fp32 steps, then the codes
  auto q8_side = [&](const SideAngles& a, int m, int64_t cnt, uint8_t** dst) -> cudaError_t {
    if (!a.q8) return cudaSuccess;
    cudaError_t r = cudaMalloc(dst, (size_t)kQ8Head + (size_t)cnt);
    if (r == cudaSuccess) r = cudaMemsetAsync(*dst, 0, kQ8Head, st);
    if (r == cudaSuccess) r = cudaMemcpyAsync(*dst, a.delta, sizeof(float) * (size_t)m, cudaMemcpyDeviceToDevice, st);
    if (r == cudaSuccess) r = cudaMemcpyAsync(*dst + kQ8Head, a.q8, (size_t)cnt, cudaMemcpyDeviceToDevice, st);
    return r;
  };
  if ((e = q8_side(av, m_in, cnt_v, &L.q8V)) != cudaSuccess || (e = q8_side(au, m_out, cnt_u, &L.q8U)) != cudaSuccess)
    return cleanup(cuda_fail(e, "create_layer_q8: int8 angle storage"));
  harp_status s = layer_maps(L);
  if (s != HARP_OK) return cleanup(s);
  *out = h;
  return HARP_OK;
}

}  // namespace

namespace {
// TMA descriptors of a layer's codes and scale/zero (GEMV and tensor-core boxes) and the
// tensor-core split of its input groups
harp_status layer_maps(Layer& L) {
  const int64_t n_in = L.n_in, n_out = L.n_out;
  const int bits = L.bits;
  const void* codes = L.codes;
  const void* scale_zero = L.scale_zero;
  const int pb = bits == 4 ? 4 : 2;  // bits of the (first) code plane
  harp_status s =
      make_tmap(&L.tm_codes, codes, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, (uint64_t)n_in * pb / 64, (uint64_t)n_out,
                (uint64_t)n_in * pb / 8);
  if (s == HARP_OK && bits == 3)
    s = make_tmap(&L.tm_hi, static_cast<const char*>(codes) + n_out * n_in / 4, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8,
                  (uint64_t)n_in / 64, (uint64_t)n_out, (uint64_t)n_in / 8);
  if (s == HARP_OK && bits != 3) L.tm_hi = L.tm_codes;
  if (s == HARP_OK)
    s = make_tmap(&L.tm_sz, scale_zero, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, (uint64_t)n_in / 64, (uint64_t)n_out,
                  (uint64_t)n_in / 16);
  if (s != HARP_OK) return s;
  // tensor-core path: one group of codes, a split's scale_zero / 1-bit plane per 128 rows
  const mma::Split sp = mma::choose_split(n_out, n_in, bits);
  L.msplits = sp.splits;
  L.mgs = sp.gs;
  const uint64_t rb = (uint64_t)n_in * pb / 8;  // bytes per row of the (first) code plane
  bool mok = encode_map_2d(&L.tm_mcodes, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, rb, (uint64_t)n_out, rb,
                           (uint32_t)(64 * pb / 8), mma::kBM, CU_TENSOR_MAP_SWIZZLE_NONE) &&
             encode_map_2d(&L.tm_msz, CU_TENSOR_MAP_DATA_TYPE_UINT32, scale_zero, (uint64_t)n_in / 64,
                           (uint64_t)n_out, (uint64_t)n_in / 16, (uint32_t)sp.gs, mma::kBM,
                           CU_TENSOR_MAP_SWIZZLE_NONE);
  if (mok && bits == 3)
    mok = encode_map_2d(&L.tm_mhi, CU_TENSOR_MAP_DATA_TYPE_UINT8, static_cast<const char*>(codes) + n_out * n_in / 4,
                        (uint64_t)n_in / 8, (uint64_t)n_out, (uint64_t)n_in / 8, (uint32_t)(8 * sp.gs), mma::kBM,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
  if (mok && bits != 3) L.tm_mhi = L.tm_msz;
  if (!mok) return fail(HARP_ERR_CUDA, "create_layer: tensor maps of the tensor-core path");
  return HARP_OK;
}

}  // namespace

harp_status harp_create_layer(harp_layer* out, int64_t n_in, int64_t n_out, int bits, int group, int w_in,
                              int w_out, const float* theta_V, const int8_t* sign_V, const float* theta_U,
                              const int8_t* sign_U, const void* codes, const void* scale_zero, void* stream) {
  return create_layer_impl(out, n_in, n_out, bits, group, w_in, w_out, SideAngles{theta_V, nullptr, nullptr}, sign_V,
                           SideAngles{theta_U, nullptr, nullptr}, sign_U, codes, scale_zero, stream);
}

harp_status harp_create_layer_q8(harp_layer* out, int64_t n_in, int64_t n_out, int bits, int group, int w_in,
                                 int w_out, const int8_t* q_V, const float* delta_V, const int8_t* sign_V,
                                 const int8_t* q_U, const float* delta_U, const int8_t* sign_U, const void* codes,
                                 const void* scale_zero, void* stream) {
  return create_layer_impl(out, n_in, n_out, bits, group, w_in, w_out, SideAngles{nullptr, q_V, delta_V}, sign_V,
                           SideAngles{nullptr, q_U, delta_U}, sign_U, codes, scale_zero, stream);
}

harp_status harp_create_layer_mr(harp_layer* out, int64_t n_in, int64_t n_out, int bits, int group, harp_mr_plan V,
                                 harp_mr_plan U, const void* codes, const void* scale_zero, void* stream) {
  (void)stream;
  if (!out) return fail(HARP_ERR_INVALID_ARG, "create_layer_mr: null output handle");
  *out = nullptr;
  if (bits < 2 || bits > 4) return fail(HARP_ERR_INVALID_ARG, "create_layer_mr: bits=%d not in {2,3,4}", bits);
  if (group != kGroup) return fail(HARP_ERR_UNSUPPORTED, "create_layer_mr: group=%d (only 64 is supported)", group);
  if (!V || !U || !codes || !scale_zero) return fail(HARP_ERR_INVALID_ARG, "create_layer_mr: null pointer");
  if (n_in <= 0 || n_in % 256 || n_in > 16384)
    return fail(HARP_ERR_INVALID_ARG, "create_layer_mr: n_in=%lld must be a positive multiple of 256, <= 16384",
                (long long)n_in);
  if (n_out <= 0 || n_out > 16384)
    return fail(HARP_ERR_INVALID_ARG, "create_layer_mr: n_out=%lld not in [1, 16384]", (long long)n_out);
  if (mr_plan_d(V) != n_in || mr_plan_d(U) != n_out)
    return fail(HARP_ERR_INVALID_ARG, "create_layer_mr: the plans' lengths must be n_in and n_out");
  if (!aligned16(codes) || !aligned16(scale_zero))
    return fail(HARP_ERR_INVALID_ARG, "create_layer_mr: device pointers must be 16-byte aligned");
  int dev = 0;
  HARP_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (mr_plan_device(V) != dev || mr_plan_device(U) != dev)
    return fail(HARP_ERR_INVALID_ARG, "create_layer_mr: the plans live on another device");
  harp_layer_s* h = new (std::nothrow) harp_layer_s();
  if (!h) return fail(HARP_ERR_INVALID_ARG, "create_layer_mr: out of host memory");
  Layer& L = h->L;
  L.n_in = n_in;
  L.n_out = n_out;
  L.bits = bits;
  L.group = group;
  L.mrV = V;
  L.mrU = U;
  L.codes = codes;
  L.scale_zero = scale_zero;
  L.device = dev;
  // no radix-2 butterfly: the fused decode step and the radix-2 kernels never take this layer
  L.w_in = L.w_out = 0;
  const harp_status s = layer_maps(L);
  if (s != HARP_OK) {
    delete h;
    return s;
  }
  *out = h;
  return HARP_OK;
}

harp_status harp_quantize_angles(int m, int64_t half_n, const float* theta, int8_t* q, float* delta, void* stream) {
  if (m < 1 || m > 16 || half_n < 1 || half_n > (int64_t(1) << 29))
    return fail(HARP_ERR_INVALID_ARG, "quantize_angles: m=%d or half_n=%lld out of range", m, (long long)half_n);
  if (!theta || !q || !delta) return fail(HARP_ERR_INVALID_ARG, "quantize_angles: null pointer");
  if (!aligned16(theta) || !aligned16(q) || !aligned16(delta))
    return fail(HARP_ERR_INVALID_ARG, "quantize_angles: device pointers must be 16-byte aligned");
  HARP_CUDA(launch_quantize_angles(m, half_n, theta, q, delta, static_cast<cudaStream_t>(stream)),
            "quantize_angles launch");
  return HARP_OK;
}

harp_status harp_destroy_layer(harp_layer layer) {
  if (!layer) return HARP_OK;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(layer->L.device);
  cudaDeviceSynchronize();
  cudaFree(layer->L.csV);
  cudaFree(layer->L.csU);
  cudaFree(layer->L.q8V);
  cudaFree(layer->L.q8U);
  cudaFree(layer->L.sV);
  cudaFree(layer->L.sU);
  cudaSetDevice(prev);
  delete layer;
  return HARP_OK;
}

harp_status harp_linear_workspace_size(harp_layer layer, int batch, size_t* bytes) {
  if (!layer || !bytes) return fail(HARP_ERR_INVALID_ARG, "linear_workspace_size: null pointer");
  if (batch < 1 || batch > kMaxBatch)
    return fail(HARP_ERR_INVALID_ARG, "linear_workspace_size: batch=%d not in [1,%d]", batch, kMaxBatch);
  *bytes = linear_ws_layout(layer->L, batch, nullptr).bytes;
  return HARP_OK;
}

harp_status harp_linear_fwd(harp_layer layer, int batch, const void* x, harp_dtype xt, void* y, harp_dtype yt,
                            void* workspace, size_t ws_bytes, void* stream) {
  if (!layer) return fail(HARP_ERR_INVALID_ARG, "linear_fwd: null layer");
  if (batch < 1 || batch > kMaxBatch)
    return fail(HARP_ERR_INVALID_ARG, "linear_fwd: batch=%d not in [1,%d]", batch, kMaxBatch);
  if (!valid_dtype(xt) || !valid_dtype(yt)) return fail(HARP_ERR_INVALID_ARG, "linear_fwd: unknown dtype");
  if (!x || !y) return fail(HARP_ERR_INVALID_ARG, "linear_fwd: null pointer");
  if (!aligned16(x) || !aligned16(y)) return fail(HARP_ERR_INVALID_ARG, "linear_fwd: pointers must be 16-byte aligned");
  if (x == y) return fail(HARP_ERR_INVALID_ARG, "linear_fwd: y must not alias x");
  const size_t need = linear_ws_layout(layer->L, batch, nullptr).bytes;
  if (!workspace || ws_bytes < need)
    return fail(HARP_ERR_WORKSPACE, "linear_fwd: workspace of %zu bytes needed, %zu given", need, ws_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(HARP_ERR_INVALID_ARG, "linear_fwd: workspace must be 256-byte aligned");
  int dev = 0;
  HARP_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev != layer->L.device) return fail(HARP_ERR_INVALID_ARG, "linear_fwd: layer lives on device %d, current is %d", layer->L.device, dev);
  return linear_forward(layer->L, batch, x, xt, layer->L.n_in, y, yt, layer->L.n_out, workspace,
                        static_cast<cudaStream_t>(stream));
}

}  // extern "C"
