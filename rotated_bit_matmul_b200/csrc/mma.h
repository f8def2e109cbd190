// Tensor-core path of the rotated low-bit linear for token batches of 16 and more.
#pragma once

#include <cuda_fp16.h>

#include "harp_internal.h"

namespace harp {
namespace mma {

constexpr int kBM = 128;     // weight rows per tile (the MMA's M)
constexpr int kMaxN = 256;   // tokens per launch (the MMA's N)
constexpr int kMaxGs = 64;   // input groups per split: the zero term is one 64-wide K block
constexpr int kDqWarps = 8;  // dequant + epilogue warps
constexpr int kThreads = 64 + 32 * kDqWarps;

// Split of the input groups for a layer: `splits` CTAs share one 128-row tile, each
// over `gs` consecutive groups (a multiple of 8; the last split may hold fewer).
struct Split {
  int splits, gs;
};
Split choose_split(int64_t n_out, int64_t n_in, int bits);

// fp16 operand: per token row, the n_in transformed values at scale 2^e (max |v| 2^e
// in [256, 512)), permuted within blocks so that one mask extracts a pair of codes,
// then the G group sums at the same scale, zero padded to `ld` columns.
int64_t x16_ld(int64_t n_in);

struct Call {
  const __half* x16;     // [batch][ld]
  int64_t ld;
  const float* rowscale; // [batch] 2^-e
  float* zpart;          // [splits][batch][n_out] (unused when y is set)
  int batch;
  int* status;
  // set only when fuses(L, batch): the kernel adds the splits and applies the output
  // side's butterfly itself, writing y ([batch] rows of n_out, y_stride apart, dtype yt)
  void* y = nullptr;
  int yt = 0;
  int64_t y_stride = 0;
};

// true when the fused epilogue is switched on (HARP_MMA_FUSE=1, read at each call; off by
// default) and the layer's output blocks (w_out = 128 or 256 rows) can be finished inside
// the tensor-core kernel at this batch: a cluster of (w_out / 128) x splits <= 8 CTAs, and
// the ring holds the partial tile.
bool fuses(const Layer& L, int batch);

cudaError_t launch_x16_prep(const float* xt, int64_t n_in, int bits, int batch, __half* x16, float* rowscale,
                            int* status, cudaStream_t st);
cudaError_t launch(const Layer& L, const Call& c, cudaStream_t st);

}  // namespace mma
}  // namespace harp
