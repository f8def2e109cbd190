// Fused batch-1 decode step: shared host/device declarations.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace harp {
namespace dec {

constexpr int kC = 8;                // CTAs per cluster
constexpr int kCW = 16;              // consumer warps per CTA
constexpr int kNT = 32 * kCW;        // consumer threads
constexpr int kThreads = kNT;        // every warp consumes; the ring is refilled by them
constexpr int kMaxClusters = 64;

// How the butterflies of a fused stack keep their angles (one kernel instantiation each):
// kTmCS (cos, sin) fp32 pairs per rotation; kTmHad every butterfly Theta == 0 (no
// parameters); kTmQ8 int8 angles with a per-stage step (a 64-byte head, then the codes).
enum { kTmCS = 0, kTmHad = 1, kTmQ8 = 2 };

// One linear as the fused kernel sees it (device array, 64-byte aligned for the maps).
struct alignas(64) Lin {
  const uint8_t* codes;  // [n_out][n_in/64] groups of 16 bytes (2-bit) or 32 (4-bit); 3-bit: the 2-bit plane
  const uint8_t* hi;     // 3-bit: the 1-bit plane, [n_out][n_in/64] x 8 bytes; else null
  const uint32_t* sz;    // scale/zero words [n_out][n_in/64]
  const uint8_t* tV;  // input-side angle storage in the stack's form (see kTm*), or null
  const uint8_t* tU;  // output-side angle storage
  const int8_t* sV;
  const int8_t* sU;
  const uint8_t* rV;  // thread-order copies of the angle storage (see repack_side), or null
  const uint8_t* rU;
  int n_in, n_out, w_in, w_out, m_in, m_out, pad0, pad1;
};

struct Params {
  const Lin* lin;  // [L][7]: q, k, v, o, gate, up, down
  int L, hidden, ffn, n_heads, n_kv, head_dim, rep, bits;
  float eps;
  int G;           // clusters in the grid
  // log2 of the per-CTA share of a hidden-wide (eb_h) and a kv-wide (eb_kv) butterfly,
  // log2 of the MLP block width (eb_blk; <= 9: one CTA per block, else one cluster)
  int eb_h, eb_kv, eb_blk, nblocks;
  const void* x_in;
  int xt;
  void* y_out;
  int yt;
  // split-K partial sums of every GEMV, [nk][n_out] (q and k kept per block: [L][nk][n])
  float *zpq, *zpk, *zpv, *zpo, *zpg, *zpu, *zpd;
  int nk_h, nk_f;      // column chunks of a hidden-wide / ffn-wide input
  float *qout, *kout;  // F_U of q and k per block, [L][dq], [L][dkv]
  int32_t* xq_down;
  float* xs_down;
  float* xsum_down;
  unsigned* counters;  // [L][5] grid barriers, then [L][nblocks] MLP-block tickets; zero at launch
  int mlp_ready;       // 1: CTA b runs MLP block b once its counter says the block's gate/up rows are in (no grid barrier)
  int* status;
  long long wait_cycles;  // bound of every wait, in SM clock cycles
  int barrier_extra;      // testing hook: grid barrier whose target is raised by one (-1: none)
  int tm;   // kTmCS, kTmHad or kTmQ8: how every butterfly of the stack keeps its angles
  int xq_bytes;
  int pf_dist;      // nonzero: each GEMV phase asks for the next phase's weights in L2
  int table_pf;     // nonzero: each GEMV phase asks for the next chain's tables in L2
  int bar_pf;       // nonzero: while a grid barrier polls, the idle warps ask for the next GEMV phase's rows in L2
  int cooperative;  // launch with the cooperative attribute (all CTAs co-resident or refused)
  int asg_qkv[kMaxClusters], idx_qkv[kMaxClusters], cnt_qkv[3];
  int asg_gu[kMaxClusters], idx_gu[kMaxClusters], cnt_gu[2];
};

cudaError_t launch(const Params& p, cudaStream_t st);
// Thread-order copy of one side's angles for the fused step: nblk blocks, each spread over a
// cluster (per-CTA share 2^eb) or held by one CTA (width 2^eb). Bytes of the copy, and the
// kernel that builds it from the layer's storage (tab) on `st`.
size_t repack_bytes(int tm, int eb, bool cluster, int nblk);
cudaError_t repack_side(int tm, int eb, bool cluster, int nblk, const uint8_t* tab, int64_t half_n, uint8_t* rt,
                        cudaStream_t st);
size_t smem_for(const Params& p);
int chunk_cols_for(int bits);
cudaError_t max_clusters(const Params& p, int* out);

}  // namespace dec
}  // namespace harp
