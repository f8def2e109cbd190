// Llama-shaped decoder stack whose seven linears per block are rotated low-bit
// layers: RMSNorm, residual adds, SiLU * up, and the key/value-group broadcast of a
// one-key attention (its output is the value), around harp linear forwards.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "common.cuh"
#include "decode.h"

using namespace harp;

struct harp_stack_s {
  int n_layers, hidden, ffn, n_heads, n_kv_heads, head_dim;
  float eps;
  std::vector<harp_layer> layers;
  int device;
  // fused batch-1 decode step (null when this stack's shapes are outside its domain)
  bool fused = false;
  dec::Lin* d_lin = nullptr;
  uint8_t* d_rt = nullptr;  // thread-order angle tables of every butterfly (one allocation)
  dec::Params fp{};
  std::string fused_why;
};

namespace {

__global__ void convert_kernel(const void* x, int xt, float* y, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    y[i] = load_act(x, i, xt);
}

__global__ void store_kernel(const float* x, void* y, int yt, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    store_act(y, i, yt, x[i]);
}

// out[b] = in[b] / sqrt(mean(in[b]^2) + eps); one CTA (512 threads) per row, fixed-order reduction
__global__ void __launch_bounds__(512) rmsnorm_kernel(const float* in, float* out, int n, float eps) {
  __shared__ float red[512];
  const float* x = in + (int64_t)blockIdx.x * n;
  float s = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s = fmaf(x[i], x[i], s);
  red[threadIdx.x] = s;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  const float inv = 1.0f / sqrtf(red[0] / (float)n + eps);
  float* y = out + (int64_t)blockIdx.x * n;
  for (int i = threadIdx.x; i < n; i += blockDim.x) y[i] = x[i] * inv;
}

__global__ void add_kernel(float* acc, const float* v, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    acc[i] += v[i];
}

__global__ void silu_mul_kernel(float* g, const float* u, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float a = g[i];
    g[i] = a / (1.0f + expf(-a)) * u[i];
  }
}

// a[b][h*hd + d] = v[b][(h / rep)*hd + d]
__global__ void repeat_kv_kernel(const float* v, float* a, int batch, int n_heads, int rep, int hd) {
  const int64_t dq = (int64_t)n_heads * hd, dkv = dq / rep, n = (int64_t)batch * dq;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t b = i / dq, r = i % dq, h = r / hd, d = r % hd;
    a[i] = v[b * dkv + (h / rep) * hd + d];
  }
}

unsigned eltwise_blocks(int64_t n) {
  int64_t b = (n + 255) / 256;
  return (unsigned)(b > 4096 ? 4096 : (b < 1 ? 1 : b));
}

size_t a256(size_t v) { return (v + 255) & ~size_t(255); }

struct StackWs {
  float *x, *n1, *q, *k, *v, *a, *o, *g, *u;
  void* lin;
  size_t bytes;
};

StackWs stack_ws(const harp_stack_s* S, int batch, void* base) {
  const size_t B = (size_t)batch;
  const size_t dq = (size_t)S->n_heads * S->head_dim, dkv = (size_t)S->n_kv_heads * S->head_dim;
  const size_t sizes[9] = {B * S->hidden, B * S->hidden, B * dq, B * dkv, B * dkv, B * dq, B * S->hidden, B * S->ffn,
                           B * S->ffn};
  StackWs w{};
  float** ptrs[9] = {&w.x, &w.n1, &w.q, &w.k, &w.v, &w.a, &w.o, &w.g, &w.u};
  size_t off = 0;
  for (int i = 0; i < 9; ++i) {
    if (base) *ptrs[i] = reinterpret_cast<float*>(static_cast<char*>(base) + off);
    off = a256(off + sizeof(float) * sizes[i]);
  }
  size_t lin = 0;
  for (auto l : S->layers) {
    const size_t b = linear_ws_layout(l->L, batch, nullptr).bytes;
    if (b > lin) lin = b;
  }
  w.lin = base ? static_cast<char*>(base) + off : nullptr;
  w.bytes = off + lin;
  return w;
}

harp_status sfail(harp_status s, const std::string& msg) { return set_error(s, "%s", msg.c_str()); }

// ---------------------------------------------------------------- fused decode step
struct FusedWs {
  size_t bytes;
};

// carves the fused kernel's buffers out of `base` (or just sizes them when base is null)
size_t fused_ws(const harp_stack_s* S, dec::Params* p, void* base) {
  const size_t L = S->n_layers, dq = (size_t)S->n_heads * S->head_dim, dkv = (size_t)S->n_kv_heads * S->head_dim;
  const size_t H = S->hidden, F = S->ffn;
  const int bits = S->layers[0]->L.bits;
  const size_t kc = (size_t)dec::chunk_cols_for(bits);
  const size_t nkh = (H + kc - 1) / kc, nkf = (F + kc - 1) / kc;
  const size_t words = bits == 3 ? F : F / 2, ngf = F / 64;
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* r = base ? static_cast<char*>(base) + off : nullptr;
    off = a256(off + bytes);
    return r;
  };
  char* zpq = take(4 * L * nkh * dq);
  char* zpk = take(4 * L * nkh * dkv);
  char* qo = take(4 * L * dq);
  char* ko = take(4 * L * dkv);
  char* zpv = take(4 * nkh * dkv);
  char* zpo = take(4 * nkh * H);
  char* zpg = take(4 * nkh * F);
  char* zpu = take(4 * nkh * F);
  char* zpd = take(4 * nkf * H);
  char* xq = take(4 * words);
  char* xs = take(4 * ngf);
  char* xsum = take(4 * ngf);
  const size_t nblk = (size_t)(F / (size_t)S->layers[4]->L.w_out);
  char* cnt = take(4 * (5 + nblk) * L);
  if (p) {
    p->nk_h = (int)nkh;
    p->nk_f = (int)nkf;
  }
  if (p && base) {
    p->zpq = reinterpret_cast<float*>(zpq);
    p->zpk = reinterpret_cast<float*>(zpk);
    p->qout = reinterpret_cast<float*>(qo);
    p->kout = reinterpret_cast<float*>(ko);
    p->zpv = reinterpret_cast<float*>(zpv);
    p->zpo = reinterpret_cast<float*>(zpo);
    p->zpg = reinterpret_cast<float*>(zpg);
    p->zpu = reinterpret_cast<float*>(zpu);
    p->zpd = reinterpret_cast<float*>(zpd);
    p->xq_down = reinterpret_cast<int32_t*>(xq);
    p->xs_down = reinterpret_cast<float*>(xs);
    p->xsum_down = reinterpret_cast<float*>(xsum);
    p->counters = reinterpret_cast<unsigned*>(cnt);
  }
  return off;
}

int ilog2(int v) {
  int m = 0;
  while ((1 << m) < v) ++m;
  return m;
}

// proportional split of G clusters over linears of n_k rows (each >= 1), largest remainder
void assign(int G, const int* rows, int k, int* asg, int* idx, int* cnt) {
  long long tot = 0;
  for (int i = 0; i < k; ++i) tot += rows[i];
  int given = 0;
  double rem[3];
  for (int i = 0; i < k; ++i) {
    const double share = (double)G * rows[i] / (double)tot;
    cnt[i] = (int)share < 1 ? 1 : (int)share;
    rem[i] = share - cnt[i];
    given += cnt[i];
  }
  while (given < G) {
    int best = 0;
    for (int i = 1; i < k; ++i)
      if (rem[i] > rem[best]) best = i;
    cnt[best] += 1;
    rem[best] -= 1.0;
    ++given;
  }
  while (given > G) {
    int best = -1;
    for (int i = 0; i < k; ++i)
      if (cnt[i] > 1 && (best < 0 || rem[i] < rem[best])) best = i;
    cnt[best] -= 1;
    rem[best] += 1.0;
    --given;
  }
  int c = 0;
  for (int i = 0; i < k; ++i)
    for (int j = 0; j < cnt[i]; ++j, ++c) {
      asg[c] = i;
      idx[c] = j;
    }
}

// Decides whether the fused kernel covers this stack and prepares its constant state.
void setup_fused(harp_stack_s* S) {
  S->fused = false;
  auto no = [&](const std::string& why) { S->fused_why = why; };
  const int H = S->hidden, F = S->ffn, dq = S->n_heads * S->head_dim, dkv = S->n_kv_heads * S->head_dim;
  const int bits = S->layers[0]->L.bits;
  if (H < 4096 || H > kMaxW || (H & (H - 1))) return no("hidden must be a power of two in [4096, 8192]");
  if (dq != H) return no("n_heads * head_dim must equal hidden");
  if (dkv < 256 || dkv > H || (dkv & (dkv - 1))) return no("n_kv_heads * head_dim must be a power of two in [256, hidden]");
  const int wb = S->layers[4]->L.w_out;
  // MLP blocks: up to 512 wide one CTA each, 4096 or 8192 wide one cluster each
  if (!((wb >= 64 && wb <= 512) || wb == 4096 || wb == 8192))
    return no("gate/up output blocks must be 64..512, 4096 or 8192 wide");
  for (int l = 0; l < S->n_layers; ++l) {
    const Layer* L[7];
    for (int i = 0; i < 7; ++i) L[i] = &S->layers[7 * l + i]->L;
    for (int i = 0; i < 7; ++i)
      if (L[i]->bits != bits) return no("all linears must share one bit width");
    for (int i = 0; i < 3; ++i)
      if (L[i]->w_in != H) return no("q/k/v input butterflies must be hidden-wide");
    if (L[0]->w_out != dq || L[1]->w_out != dkv || L[2]->w_out != dkv) return no("q/k/v output butterflies must be single blocks");
    if (L[3]->w_in != H || L[3]->w_out != H) return no("o butterflies must be hidden-wide");
    if (L[4]->w_in != H || L[5]->w_in != H) return no("gate/up input butterflies must be hidden-wide");
    if (L[4]->w_out != wb || L[5]->w_out != wb || L[6]->w_in != wb) return no("gate/up output and down input blocks must match");
    if (L[6]->w_out != H) return no("down output butterfly must be hidden-wide");
  }
  // every butterfly in one form: fp32 angles (cos/sin tables), int8 angles, or Theta == 0.
  // One kernel instantiation per form, so none pays for another in its rotations.
  int n_cs = 0, n_q8 = 0, n_had = 0;
  for (const harp_layer l : S->layers) {
    const Layer& L = l->L;
    for (int side = 0; side < 2; ++side) {
      const bool q8 = side ? L.q8U != nullptr : L.q8V != nullptr;
      const bool cs = side ? L.csU != nullptr : L.csV != nullptr;
      n_q8 += q8;
      n_cs += cs && !q8;
      n_had += !cs && !q8;
    }
  }
  int tm = dec::kTmCS;
  if (n_had && !n_cs && !n_q8)
    tm = dec::kTmHad;
  else if (n_q8 && !n_cs && !n_had)
    tm = dec::kTmQ8;
  else if (n_q8 || n_had)
    return no("butterflies with fp32 angles, int8 angles and Theta = 0 are not fused together");
  dec::Params& p = S->fp;
  p = dec::Params{};
  p.tm = tm;
  p.L = S->n_layers;
  p.hidden = H;
  p.ffn = F;
  p.n_heads = S->n_heads;
  p.n_kv = S->n_kv_heads;
  p.head_dim = S->head_dim;
  p.rep = S->n_heads / S->n_kv_heads;
  p.bits = bits;
  p.eps = S->eps;
  p.eb_h = ilog2(H / dec::kC);
  p.eb_kv = ilog2(dkv / dec::kC);
  p.eb_blk = ilog2(wb);
  p.nblocks = F / wb;
  // shared memory: the operand of the widest input and the chain buffers
  auto xqb = [&](int n) { return 4 * ((bits == 3 ? n : n / 2) + 2 * (n / 64)); };
  p.xq_bytes = (std::max(xqb(H), xqb(F)) + 15) & ~15;  // keeps what follows it 16-byte aligned
  int optin = 0;
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, S->device);
  if (dec::smem_for(p) > (size_t)optin) return no("not enough shared memory for the operand");
  // HARP_PF_DIST=1: each GEMV phase asks for the next phase's weights in L2 (per-lane line
  // prefetches). Off by default: the burst of requests stalls the issuing warps for longer
  // than the L2 hits save (same-box A/B: 2.924 ms/step without, 3.101 ms with).
  // HARP_TABLE_PF=0: no bulk L2 requests for the next chain's tables. Cooperative launch
  // unless HARP_COOPERATIVE=0.
  p.pf_dist = 0;
  if (const char* e = getenv("HARP_PF_DIST")) p.pf_dist = std::max(0, atoi(e));
  p.table_pf = 1;
  if (const char* e = getenv("HARP_TABLE_PF")) p.table_pf = atoi(e) != 0;
  // HARP_BAR_PF=0: the warps idle at a grid barrier do not ask for the next GEMV phase's
  // rows in L2
  p.bar_pf = 1;
  if (const char* e = getenv("HARP_BAR_PF")) p.bar_pf = atoi(e) != 0;
  p.cooperative = 1;
  if (const char* e = getenv("HARP_COOPERATIVE")) p.cooperative = atoi(e) != 0;
  // MLP blocks up to 512 wide, one CTA each: CTA b starts block b's chain as soon as that
  // block's gate and up rows are in (a counter per block that each CTA adds its units to
  // once), without a grid barrier; HARP_MLP_READY=0 waits for the whole phase instead
  p.mlp_ready = wb <= 512 && F % 32 == 0;
  if (const char* e = getenv("HARP_MLP_READY")) p.mlp_ready = p.mlp_ready && atoi(e) != 0;
  int G = 0;
  cudaError_t e = dec::max_clusters(p, &G);
  if (e != cudaSuccess || G < 1)
    return no(std::string("cluster occupancy query failed: ") + cudaGetErrorString(e) + ", G=" + std::to_string(G) +
              ", smem " + std::to_string(dec::smem_for(p)));
  if (G > dec::kMaxClusters) G = dec::kMaxClusters;
  // P7: MLP-block CTAs (or clusters) come first, the last two clusters apply F_U_q / F_U_k
  const int cap = wb <= 512 ? dec::kC : 1;
  if (G < 3 || p.nblocks > (G - 2) * cap) return no("too few co-resident clusters");
  p.G = G;
  if (getenv("HARP_DEBUG"))
    fprintf(stderr, "harp fused step: G=%d smem=%zu xq_bytes=%d eb_h=%d eb_kv=%d eb_blk=%d nblocks=%d tm=%d\n", G,
            dec::smem_for(p), p.xq_bytes, p.eb_h, p.eb_kv, p.eb_blk, p.nblocks, p.tm);
  const int rq[3] = {dq, dkv, dkv}, rg[2] = {F, F};
  assign(G, rq, 3, p.asg_qkv, p.idx_qkv, p.cnt_qkv);
  assign(G, rg, 2, p.asg_gu, p.idx_gu, p.cnt_gu);
  // device copy of the per-linear descriptors
  std::vector<dec::Lin> h(7 * (size_t)S->n_layers);
  for (size_t i = 0; i < h.size(); ++i) {
    const Layer& L = S->layers[i]->L;
    dec::Lin& d = h[i];
    memset(&d, 0, sizeof d);
    d.codes = static_cast<const uint8_t*>(L.codes);
    d.hi = L.bits == 3 ? static_cast<const uint8_t*>(L.codes) + L.n_out * L.n_in / 4 : nullptr;
    d.sz = static_cast<const uint32_t*>(L.scale_zero);
    d.tV = L.q8V ? L.q8V : reinterpret_cast<const uint8_t*>(L.csV);
    d.tU = L.q8U ? L.q8U : reinterpret_cast<const uint8_t*>(L.csU);
    d.sV = L.sV;
    d.sU = L.sU;
    d.n_in = (int)L.n_in;
    d.n_out = (int)L.n_out;
    d.w_in = L.w_in;
    d.w_out = L.w_out;
    d.m_in = L.m_in;
    d.m_out = L.m_out;
  }
  // thread-order copies of the angle tables (HARP_REPACK=0 reads the layers' own tables)
  bool repack = tm != dec::kTmHad;
  if (const char* e = getenv("HARP_REPACK")) repack = repack && atoi(e) != 0;
  if (repack) {
    struct Side {
      size_t i;
      bool u, cl;
      int eb, nblk;
    };
    std::vector<Side> sides;
    auto mlp = [&](size_t i, bool u) {
      if (wb <= 512) sides.push_back({i, u, false, p.eb_blk, p.nblocks});
      else sides.push_back({i, u, true, p.eb_blk - 3, p.nblocks});
    };
    for (size_t i = 0; i < h.size(); ++i) {
      const int li = (int)(i % 7);
      if (li <= 5) sides.push_back({i, false, true, p.eb_h, 1});
      else mlp(i, false);
      if (li == 0 || li == 3 || li == 6) sides.push_back({i, true, true, p.eb_h, 1});
      else if (li == 1 || li == 2) sides.push_back({i, true, true, p.eb_kv, 1});
      else mlp(i, true);
    }
    size_t total = 0;
    for (const Side& sd : sides) total += (dec::repack_bytes(tm, sd.eb, sd.cl, sd.nblk) + 255) & ~size_t(255);
    if (cudaMalloc(&S->d_rt, total) != cudaSuccess) return no("cudaMalloc of the thread-order tables failed");
    size_t off = 0;
    for (const Side& sd : sides) {
      dec::Lin& d = h[sd.i];
      const Layer& L = S->layers[sd.i]->L;
      uint8_t* dst = S->d_rt + off;
      off += (dec::repack_bytes(tm, sd.eb, sd.cl, sd.nblk) + 255) & ~size_t(255);
      const uint8_t* src = sd.u ? d.tU : d.tV;
      if (dec::repack_side(tm, sd.eb, sd.cl, sd.nblk, src, (sd.u ? L.n_out : L.n_in) / 2, dst, 0) != cudaSuccess) {
        cudaFree(S->d_rt);
        S->d_rt = nullptr;
        return no("building the thread-order tables failed");
      }
      if (sd.u) d.rU = dst;
      else d.rV = dst;
    }
    if (cudaStreamSynchronize(0) != cudaSuccess) return no("building the thread-order tables failed");
  }
  if (cudaMalloc(&S->d_lin, sizeof(dec::Lin) * h.size()) != cudaSuccess) return no("cudaMalloc failed");
  if (cudaMemcpy(S->d_lin, h.data(), sizeof(dec::Lin) * h.size(), cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaFree(S->d_lin);
    S->d_lin = nullptr;
    return no("cudaMemcpy failed");
  }
  p.lin = S->d_lin;
  S->fused = true;
}

}  // namespace

extern "C" {

harp_status harp_stack_create(harp_stack* out, int n_layers, int hidden, int ffn, int n_heads, int n_kv_heads,
                              int head_dim, float eps, const harp_layer* layers, void* stream) {
  (void)stream;
  if (!out || !layers) return sfail(HARP_ERR_INVALID_ARG, "stack_create: null pointer");
  *out = nullptr;
  if (n_layers < 1 || hidden < 1 || ffn < 1 || n_heads < 1 || n_kv_heads < 1 || head_dim < 1 ||
      n_heads % n_kv_heads || !(eps >= 0.f))
    return sfail(HARP_ERR_INVALID_ARG, "stack_create: bad dimensions");
  const int64_t dq = (int64_t)n_heads * head_dim, dkv = (int64_t)n_kv_heads * head_dim;
  const int64_t shapes[7][2] = {{dq, hidden}, {dkv, hidden}, {dkv, hidden}, {hidden, dq},
                                {ffn, hidden}, {ffn, hidden}, {hidden, ffn}};
  for (int l = 0; l < n_layers; ++l)
    for (int i = 0; i < 7; ++i) {
      harp_layer h = layers[7 * l + i];
      if (!h) return sfail(HARP_ERR_INVALID_ARG, "stack_create: null layer handle");
      if (h->L.n_out != shapes[i][0] || h->L.n_in != shapes[i][1])
        return sfail(HARP_ERR_INVALID_ARG, "stack_create: layer " + std::to_string(l) + " linear " +
                                               std::to_string(i) + " has the wrong shape");
    }
  harp_stack_s* S = new (std::nothrow) harp_stack_s();
  if (!S) return sfail(HARP_ERR_INVALID_ARG, "stack_create: out of host memory");
  S->n_layers = n_layers;
  S->hidden = hidden;
  S->ffn = ffn;
  S->n_heads = n_heads;
  S->n_kv_heads = n_kv_heads;
  S->head_dim = head_dim;
  S->eps = eps;
  S->layers.assign(layers, layers + 7 * (size_t)n_layers);
  cudaGetDevice(&S->device);
  setup_fused(S);
  cudaGetLastError();  // a refused fused set-up is not an error of this call
  *out = S;
  return HARP_OK;
}

harp_status harp_stack_destroy(harp_stack stack) {
  if (!stack) return HARP_OK;
  if (stack->d_lin || stack->d_rt) {
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(stack->device);
    cudaDeviceSynchronize();
    cudaFree(stack->d_lin);
    cudaFree(stack->d_rt);
    cudaSetDevice(prev);
  }
  delete stack;
  return HARP_OK;
}

int harp_stack_uses_fused_step(harp_stack stack, int batch) {
  if (stack && !stack->fused) set_error(HARP_OK, "fused step not taken: %s", stack->fused_why.c_str());
  return stack && stack->fused && batch == 1;
}

harp_status harp_stack_workspace_size(harp_stack stack, int batch, size_t* bytes) {
  if (!stack || !bytes) return sfail(HARP_ERR_INVALID_ARG, "stack_workspace_size: null pointer");
  if (batch < 1 || batch > 256) return sfail(HARP_ERR_INVALID_ARG, "stack_workspace_size: batch out of range");
  *bytes = stack_ws(stack, batch, nullptr).bytes;
  if (stack->fused && batch == 1) *bytes = std::max(*bytes, fused_ws(stack, nullptr, nullptr));
  return HARP_OK;
}

harp_status harp_stack_step(harp_stack S, int batch, const void* x, harp_dtype xt, void* out, harp_dtype ot,
                            void* workspace, size_t ws_bytes, void* stream) {
  if (!S || !x || !out) return sfail(HARP_ERR_INVALID_ARG, "stack_step: null pointer");
  if (batch < 1 || batch > 256) return sfail(HARP_ERR_INVALID_ARG, "stack_step: batch out of range");
  if (xt < 0 || xt > 2 || ot < 0 || ot > 2) return sfail(HARP_ERR_INVALID_ARG, "stack_step: unknown dtype");
  size_t need = stack_ws(S, batch, nullptr).bytes;
  const bool fused = S->fused && batch == 1;
  if (fused) need = std::max(need, fused_ws(S, nullptr, nullptr));
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return sfail(HARP_ERR_WORKSPACE, "stack_step: workspace of " + std::to_string(need) +
                                         " bytes (256-byte aligned) needed");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (fused) {
    int* status = nullptr;
    harp_status hs = device_status_for_kernels(&status);
    if (hs != HARP_OK) return hs;
    dec::Params p = S->fp;
    fused_ws(S, &p, workspace);
    p.x_in = x;
    p.xt = xt;
    p.y_out = out;
    p.yt = ot;
    p.status = status;
    const TestHooks th = test_hooks();
    p.wait_cycles = th.wait_cycles;
    p.barrier_extra = th.decode_barrier_extra;
    cudaError_t e =
        cudaMemsetAsync(p.counters, 0, sizeof(unsigned) * (5 + (size_t)p.nblocks) * (size_t)S->n_layers, st);
    if (e == cudaSuccess) e = dec::launch(p, st);
    if (e != cudaSuccess) return sfail(HARP_ERR_CUDA, std::string("fused decode step: ") + cudaGetErrorString(e));
    return HARP_OK;
  }
  StackWs w = stack_ws(S, batch, workspace);
  const int64_t B = batch, H = S->hidden, F = S->ffn;
  const int64_t dq = (int64_t)S->n_heads * S->head_dim, dkv = (int64_t)S->n_kv_heads * S->head_dim;
  const int rep = S->n_heads / S->n_kv_heads;
  convert_kernel<<<eltwise_blocks(B * H), 256, 0, st>>>(x, xt, w.x, B * H);
  harp_status s = HARP_OK;
  for (int l = 0; l < S->n_layers && s == HARP_OK; ++l) {
    const Layer* L[7];
    for (int i = 0; i < 7; ++i) L[i] = &S->layers[7 * l + i]->L;
    rmsnorm_kernel<<<(unsigned)B, 512, 0, st>>>(w.x, w.n1, (int)H, S->eps);
    s = linear_forward(*L[0], batch, w.n1, DT_F32, H, w.q, DT_F32, dq, w.lin, st);
    if (s == HARP_OK) s = linear_forward(*L[1], batch, w.n1, DT_F32, H, w.k, DT_F32, dkv, w.lin, st);
    if (s == HARP_OK) s = linear_forward(*L[2], batch, w.n1, DT_F32, H, w.v, DT_F32, dkv, w.lin, st);
    const float* attn = w.v;
    if (rep > 1) {
      repeat_kv_kernel<<<eltwise_blocks(B * dq), 256, 0, st>>>(w.v, w.a, batch, S->n_heads, rep, S->head_dim);
      attn = w.a;
    }
    if (s == HARP_OK) s = linear_forward(*L[3], batch, attn, DT_F32, dq, w.o, DT_F32, H, w.lin, st);
    add_kernel<<<eltwise_blocks(B * H), 256, 0, st>>>(w.x, w.o, B * H);
    rmsnorm_kernel<<<(unsigned)B, 512, 0, st>>>(w.x, w.n1, (int)H, S->eps);
    if (s == HARP_OK) s = linear_forward(*L[4], batch, w.n1, DT_F32, H, w.g, DT_F32, F, w.lin, st);
    if (s == HARP_OK) s = linear_forward(*L[5], batch, w.n1, DT_F32, H, w.u, DT_F32, F, w.lin, st);
    silu_mul_kernel<<<eltwise_blocks(B * F), 256, 0, st>>>(w.g, w.u, B * F);
    if (s == HARP_OK) s = linear_forward(*L[6], batch, w.g, DT_F32, F, w.o, DT_F32, H, w.lin, st);
    add_kernel<<<eltwise_blocks(B * H), 256, 0, st>>>(w.x, w.o, B * H);
  }
  if (s != HARP_OK) return s;
  store_kernel<<<eltwise_blocks(B * H), 256, 0, st>>>(w.x, out, ot, B * H);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return sfail(HARP_ERR_CUDA, std::string("stack_step launch: ") + cudaGetErrorString(e));
  return HARP_OK;
}

}  // extern "C"
