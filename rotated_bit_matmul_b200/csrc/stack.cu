// Llama-shaped decoder stack whose seven linears per block are rotated low-bit
// layers: RMSNorm, residual adds, SiLU * up, and the key/value-group broadcast of a
// one-key attention (its output is the value), around harp linear forwards.
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "common.cuh"

using namespace harp;

struct harp_stack_s {
  int n_layers, hidden, ffn, n_heads, n_kv_heads, head_dim;
  float eps;
  std::vector<harp_layer> layers;
  int device;
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
  *out = S;
  return HARP_OK;
}

harp_status harp_stack_destroy(harp_stack stack) {
  delete stack;
  return HARP_OK;
}

harp_status harp_stack_workspace_size(harp_stack stack, int batch, size_t* bytes) {
  if (!stack || !bytes) return sfail(HARP_ERR_INVALID_ARG, "stack_workspace_size: null pointer");
  if (batch < 1 || batch > 256) return sfail(HARP_ERR_INVALID_ARG, "stack_workspace_size: batch out of range");
  *bytes = stack_ws(stack, batch, nullptr).bytes;
  return HARP_OK;
}

harp_status harp_stack_step(harp_stack S, int batch, const void* x, harp_dtype xt, void* out, harp_dtype ot,
                            void* workspace, size_t ws_bytes, void* stream) {
  if (!S || !x || !out) return sfail(HARP_ERR_INVALID_ARG, "stack_step: null pointer");
  if (batch < 1 || batch > 256) return sfail(HARP_ERR_INVALID_ARG, "stack_step: batch out of range");
  if (xt < 0 || xt > 2 || ot < 0 || ot > 2) return sfail(HARP_ERR_INVALID_ARG, "stack_step: unknown dtype");
  const size_t need = stack_ws(S, batch, nullptr).bytes;
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return sfail(HARP_ERR_WORKSPACE, "stack_step: workspace of " + std::to_string(need) +
                                         " bytes (256-byte aligned) needed");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
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
