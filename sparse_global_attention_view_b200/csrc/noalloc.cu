// gsa_forward_noalloc: the whole GSA layer for callers that cannot allocate
// device memory.  Its intermediates live in one fixed device array defined in
// this file instead of a caller-supplied workspace; everything else is
// gsa_forward, unchanged.
#include <mutex>

#include "internal.h"

namespace {

// The fixed scratch.  Every GPU that loads libgsa holds these bytes until the
// process exits.  In host code `g_noalloc_scratch` is only a host-side stand-in
// for the symbol, never a device address: its device address is obtained with
// cudaGetSymbolAddress on each device below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};  // device address of the array, per device

// Once per device, with that device current: look up the array's address.
gsa_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return GSA_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return GSA_OK;
}

}  // namespace

extern "C" gsa_status gsa_forward_noalloc(const gsa_shape* shape, const gsa_bf16* q,
                                          const gsa_bf16* k, const gsa_bf16* v, const float* w,
                                          gsa_bf16* out, void* stream) {
  size_t need = 0;
  gsa_status st = gsa_workspace_size(shape, &need);
  if (st != GSA_OK) return st;
  if (need > (size_t)GSA_NOALLOC_SCRATCH_BYTES) return GSA_ERR_SCRATCH_LIMIT;
  void* ws = nullptr;
  st = scratch_for_current_device(&ws);
  if (st != GSA_OK) return st;
  // the header holds the device error word, which must start at zero
  if (cudaMemsetAsync(ws, 0, GSA_WS_HEADER_BYTES, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return GSA_ERR_CUDA;
  return gsa_forward(shape, q, k, v, w, out, ws, (size_t)GSA_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" gsa_status gsa_noalloc_check_device_error(void* stream) {
  // the fixed array's first word is the error word of the last no-alloc call
  // on the current device (its header was zeroed when that call began)
  void* ws = nullptr;
  gsa_status st = scratch_for_current_device(&ws);
  if (st != GSA_OK) return st;
  return gsa_check_device_error(ws, stream);
}
