// Decode anchor selection without a caller-provided workspace.
//
// Some callers cannot hand this library any device scratch and must not
// allocate: for example an operator plugged into a host runtime that owns and
// pre-plans all device memory and offers its kernels no workspace argument.
// For them this entry point runs the same decode selection as
// kascade_select, with its scratch in a fixed array that lives in the
// library's own device image.
//
// The array (kStaticBytes) is a file-scope __device__ variable: every GPU
// that loads the library holds it until the process exits.  In host code its
// name is only a host-side stand-in, so the device address is looked up with
// cudaGetSymbolAddress once per device, with that device current, on the
// first call that runs on it.  That first call should therefore come before
// any stream capture.  Every call shares the array and it keeps the last
// call's contents; nothing in it has to start at zero for the decode
// selection.  Calls that may overlap on the GPU (on different streams, or on
// different host threads) race on the array and must be serialised by the
// caller.
#include <mutex>

#include "../../include/kascade.h"
#include "common.cuh"

namespace {

constexpr size_t kStaticBytes = (size_t)8 << 20;   // 8 MiB

__device__ __align__(256) unsigned char g_select_scratch[kStaticBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// device address of the scratch array on the current device (set-up on first use)
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KASCADE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || p == nullptr) return KASCADE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KASCADE_OK;
}

}  // namespace

extern "C" {

size_t kascade_select_decode_static_max_bytes(void) { return kStaticBytes; }

int kascade_select_decode_static(const kascade_shape* shape, const void* q, const void* k, int32_t* idx,
                                 void* stream) {
  if (!shape) return KASCADE_ERR_INVALID_ARG;
  if (shape->q_len != 1) return KASCADE_ERR_UNSUPPORTED;
  const size_t need = kascade_workspace_bytes(shape, KASCADE_OP_SELECT);
  if (need == 0) return KASCADE_ERR_INVALID_ARG;   // invalid shape
  if (need > kStaticBytes) return KASCADE_ERR_TOO_LARGE;
  if (!q || !k || !idx) return KASCADE_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc) return rc;
  return kascade_select(shape, q, k, idx, scratch, kStaticBytes, stream);
}

}  // extern "C"
