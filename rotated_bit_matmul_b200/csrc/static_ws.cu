// harp_linear_fwd_static: the rotated linear forward for callers that cannot
// allocate device memory.
//
// Some callers may not call cudaMalloc at all: code that runs inside another
// framework's memory pool, real-time paths where an allocation may block or fail,
// and hosts that hand the library only pre-registered buffers. They still own x
// and y, but cannot provide the scratch harp_linear_fwd needs. This entry point
// takes its scratch from a fixed array in the library's device image instead:
// kStaticScratchBytes (2 MiB) of device memory that every GPU which loads the
// library keeps until the process exits.
//
// Properties the caller must know:
//   - The first call on a device looks up the array's device address
//     (cudaGetSymbolAddress) with that device current. With CUDA's lazy module
//     loading that lookup is also what loads the part of the library image holding
//     the array, so the array's 2 MiB are taken from the device at that first call
//     (by the driver, not by an allocation call of this library). Make that first call
//     before any stream capture, and at a point where taking 2 MiB is acceptable.
//     Later calls on the device do no set-up and take no device memory.
//   - Requests whose scratch would exceed 2 MiB are rejected (HARP_ERR_WORKSPACE).
//   - All calls on a device share the one array, which keeps what the last call
//     wrote. Nothing in it has to start at zero (every byte is written before it is
//     read), but calls whose work overlaps on the GPU -- different streams, or
//     different host threads -- race on it: serialise them.
//   - No cudaMalloc, cudaFree or allocating library routine is called. For the same
//     reason this path has no device status word: a bounded device-side wait that
//     runs out ends the kernel without a report (harp_device_status does not see it).
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(2) << 20;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_addr[64] = {nullptr};

harp_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return harp::set_error(HARP_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return harp::set_error(HARP_ERR_UNSUPPORTED, "device index %d >= 64", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p)
      return harp::set_error(HARP_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return HARP_OK;
}

}  // namespace

using namespace harp;

extern "C" harp_status harp_linear_fwd_static(harp_layer layer, int batch, const void* x, harp_dtype xt, void* y,
                                              harp_dtype yt, void* stream) {
  if (!layer) return set_error(HARP_ERR_INVALID_ARG, "linear_fwd_static: null layer");
  if (batch < 1 || batch > kMaxBatch)
    return set_error(HARP_ERR_INVALID_ARG, "linear_fwd_static: batch=%d not in [1,%d]", batch, kMaxBatch);
  if (xt < HARP_F32 || xt > HARP_F16 || yt < HARP_F32 || yt > HARP_F16)
    return set_error(HARP_ERR_INVALID_ARG, "linear_fwd_static: unknown dtype");
  if (!x || !y) return set_error(HARP_ERR_INVALID_ARG, "linear_fwd_static: null pointer");
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(y) & 15u))
    return set_error(HARP_ERR_INVALID_ARG, "linear_fwd_static: pointers must be 16-byte aligned");
  if (x == y) return set_error(HARP_ERR_INVALID_ARG, "linear_fwd_static: y must not alias x");
  const Layer& L = layer->L;
  const size_t need = linear_ws_layout(L, batch, nullptr).bytes;
  if (need > kStaticScratchBytes)
    return set_error(HARP_ERR_WORKSPACE,
                     "linear_fwd_static: this layer needs %zu bytes of scratch for batch %d; the static scratch "
                     "holds %zu bytes (use harp_linear_fwd with a caller workspace)",
                     need, batch, kStaticScratchBytes);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(HARP_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev != L.device) return set_error(HARP_ERR_INVALID_ARG, "linear_fwd_static: layer lives on device %d, current is %d", L.device, dev);
  void* base = nullptr;
  harp_status s = scratch_address(&base);
  if (s != HARP_OK) return s;
  int* status = nullptr;  // see the note on device status above
  harp_status r = linear_forward_status(L, batch, x, xt, L.n_in, y, yt, L.n_out, base,
                                        static_cast<cudaStream_t>(stream), status);
  if (r != HARP_OK) return set_error(r, "linear_fwd_static: %s", harp_last_error());
  return HARP_OK;
}
