// Internal declarations of the rotated low-bit linear library (host + device).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "harp.h"

struct harp_mr_plan_s;

namespace harp {

enum { DT_F32 = 0, DT_BF16 = 1, DT_F16 = 2 };

constexpr int kGroup = 64;       // quantization group (columns)
constexpr int kMaxBatchGemv = 8; // batch rows the CUDA-core GEMV handles per launch
constexpr int kMaxW = 8192;      // widest butterfly block held by one CTA
constexpr int kMinBatchMma = 16; // token batches from here on take the tensor-core path
constexpr int kMaxBatch = 65535; // token rows per harp_linear_fwd call (a grid dimension)
// int8 angle storage of one butterfly: a 64-byte head holding the fp32 step delta_t of
// every stage (up to 16; log2 8192 = 13), then the codes int8 [m][n/2].
constexpr int kQ8Head = 64;

// Butterfly launch description. One CTA transforms one w-wide block of one row.
struct BflyParams {
  int64_t n;
  int w, m, inverse;
  const float* theta;  // [m][n/2] angle offsets (pi/4 added in-kernel) or null when cs is set
  const float2* cs;    // [m][n/2] (cos, sin) of pi/4 + theta, or null
  const uint8_t* q8;   // int8 angles (kQ8Head bytes of fp32 steps, then int8 [m][n/2]), or null
  const int8_t* sign;  // [n]
  const void* x;
  int xt;
  int64_t x_stride;    // elements between rows
  void* y;             // may be null when only the prep outputs are wanted
  int yt;
  int64_t y_stride;
  // Optional epilogue producing the GEMV operand (null xq disables it):
  int32_t* xq;         // int16 pairs in dp2a order, xq_stride words per row
  float* xs;           // per group 2^-e (the int16 scale), g_stride per row
  float* xsum;         // per group fp32 sum of the transformed values
  int bits;
  int64_t xq_stride, g_stride;
  int nsum;            // forward input: sum of nsum fp32 partial arrays sum_stride apart (<= 1: one)
  int64_t sum_stride;
  int* status;
  long long wait_cycles;  // bound of the fast kernel's exchange waits (SM cycles; 0: the default)
};

// Testing hooks (harp_test_set_faults): off by default. wait_ns bounds every mbarrier
// wait of the stand-alone kernels, wait_cycles every wait of the fused decode step
// (SM clock cycles); gemv_skip_stage >= 0 makes the stand-alone GEMV's producer in CTA 0
// skip that ring stage; decode_barrier_extra raises the target of one grid barrier of the
// fused step (its index, or -1) by one, so that barrier can never complete.
struct TestHooks {
  uint64_t wait_ns;
  long long wait_cycles;
  int gemv_skip_stage;
  int decode_barrier_extra;
};
TestHooks test_hooks();

// Dequant-GEMV launch description (codes come through the layer's tensor maps).
struct GemvParams {
  uint64_t wait_ns;     // bound of every mbarrier wait
  int skip_stage;       // testing hook: ring stage CTA 0's producer does not issue (-1: none)
  int n_out, n_in, bits, batch;
  const int32_t* xq;
  int64_t xq_stride;
  const float* xs;
  const float* xsum;
  int64_t g_stride;
  float* z;
  int64_t z_stride;
  int* status;
};

struct Layer {
  int64_t n_in, n_out;
  int bits, group, w_in, w_out, m_in, m_out;
  // mixed-radix sides (harp_create_layer_mr): borrowed plans, or null for radix-2 sides
  const harp_mr_plan_s* mrV;
  const harp_mr_plan_s* mrU;
  float2* csV;   // [m_in][n_in/2]
  float2* csU;   // [m_out][n_out/2]
  uint8_t* q8V;  // int8 angle storage of the input side (kQ8Head + m_in * n_in/2 bytes), or null
  uint8_t* q8U;  // int8 angle storage of the output side, or null
  int8_t* sV;
  int8_t* sU;
  const void* codes;
  const void* scale_zero;
  CUtensorMap tm_codes;  // 2-bit/4-bit codes, or the 2-bit plane of 3-bit codes
  CUtensorMap tm_hi;     // 1-bit plane of 3-bit codes (unused otherwise)
  CUtensorMap tm_sz;     // scale_zero as uint32 [n_out][n_in/64]
  // tensor-core path (token batches >= kMinBatchMma): 128-row boxes of one group's codes,
  // of a split's scale_zero and of a split's 1-bit plane (3-bit codes)
  CUtensorMap tm_mcodes, tm_msz, tm_mhi;
  int msplits, mgs;      // input-group splits per 128-row tile and groups per split
  int device;
};

// Workspace carve-up for a linear forward with `batch` rows. Below kMinBatchMma rows
// (GEMV): xq, xs, xsum, z. From kMinBatchMma rows (tensor cores): xf, x16, rowscale, zpart.
struct LinearWs {
  float* xmr;         // mixed-radix layers: [batch][n_in] transformed input (GEMV path)
  float* zmr;         // mixed-radix layers: [batch][n_out] sum of the split partials (tensor-core path)
  int32_t* xq;
  float* xs;
  float* xsum;
  float* z;
  int64_t xq_stride, g_stride;
  float* xf;          // [batch][n_in] transformed input
  void* x16;          // [batch][x16_ld] fp16 operand + group sums
  float* rowscale;    // [batch]
  float* zpart;       // [msplits][batch][n_out]
  int64_t x16_ld;
  size_t bytes;
};

LinearWs linear_ws_layout(const Layer& L, int batch, void* base);
int xq_words_per_row(int64_t n_in, int bits);

cudaError_t launch_butterfly(const BflyParams& p, int batch, cudaStream_t st);
// mixed-radix transform of `batch` contiguous rows (plan forward, or its transpose).
// For fewer than 8 rows the stages run in several launches with fp32 rows in between,
// held in y when y is fp32, else in `scratch` (batch x d floats, may be x); with neither,
// one CTA per row runs every stage.
cudaError_t launch_mr(const harp_mr_plan_s* plan, int inverse, int batch, const void* x, int xt, void* y, int yt,
                      cudaStream_t st, float* scratch = nullptr);
int64_t mr_plan_d(const harp_mr_plan_s* plan);
int mr_plan_device(const harp_mr_plan_s* plan);
// int16 GEMV operand of `batch` fp32 rows of n (groups of 64): xq words, xs, xsum
cudaError_t launch_operand_prep(const float* x, int64_t n, int bits, int batch, int32_t* xq, int64_t xq_stride,
                                float* xs, float* xsum, int64_t g_stride, cudaStream_t st);
// z[i] = sum over s of part[s][i], s in fixed order (count elements per split)
cudaError_t launch_sum_splits(const float* part, int splits, int64_t count, float* z, cudaStream_t st);
cudaError_t launch_gemv(const Layer& L, const GemvParams& p, cudaStream_t st);
cudaError_t launch_quantize(int64_t n_out, int64_t n_in, int bits, const float* W, void* codes,
                            void* scale_zero, cudaStream_t st);
cudaError_t launch_cs_table(const float* theta, int64_t count, float2* cs, cudaStream_t st);
cudaError_t launch_quantize_angles(int m, int64_t half_n, const float* theta, int8_t* q, float* delta,
                                   cudaStream_t st);

// 2-D tiled tensor map over a row-major [rows][inner] array; false if the driver
// entry point is missing or rejects the arguments.
bool encode_map_2d(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw);

// Records a printf-style message as the thread's last error and returns `st`.
harp_status set_error(harp_status st, const char* fmt, ...);
// Per-device status word the kernels report failures into (allocated on first use,
// which therefore must not happen inside a stream capture).
harp_status device_status_for_kernels(int** out);
// Enqueues y = F_U(dequant(codes) F_V(x)) for validated arguments.
harp_status linear_forward(const Layer& L, int batch, const void* x, int xt, int64_t x_stride, void* y, int yt,
                           int64_t y_stride, void* ws, cudaStream_t st);
// The same with an explicit status word (null: device-side failures are not recorded).
harp_status linear_forward_status(const Layer& L, int batch, const void* x, int xt, int64_t x_stride, void* y,
                                  int yt, int64_t y_stride, void* ws, cudaStream_t st, int* status);

}  // namespace harp

struct harp_layer_s {
  harp::Layer L;
};
