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
// cudaGetSymbolAddress once per device context, with that device current, on
// the first call that runs in it.  That first call should therefore come
// before any stream capture.  The lookup is keyed on the current CUDA
// context as well as the device ordinal, so a context created after
// cudaDeviceReset gets its own lookup instead of a stale address.  Every call
// shares the array and it keeps the last call's contents; nothing in it has
// to start at zero for the decode selection, except the error word (its
// first int), which only kascade_select_decode_static_error clears.  Calls
// that may overlap on the GPU (on different streams, or on different host
// threads) race on the array and must be serialised by the caller.
#include <mutex>

#include "../../include/kascade.h"
#include "common.cuh"

namespace {

constexpr size_t kStaticBytes = (size_t)8 << 20;   // 8 MiB

__device__ __align__(256) unsigned char g_select_scratch[kStaticBytes];

constexpr int kMaxDevices = 64;
struct Cached {
  void* ctx;    // CUDA context the address was looked up in
  void* ptr;    // device address of g_select_scratch in that context
};
Cached g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mu;

// cuCtxGetCurrent through the runtime's driver entry point (the library
// links no driver stub); NULL context when it cannot be had
using CtxGetCurrentFn = int (*)(void**);

void* current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
    tried = true;
  }
  void* ctx = nullptr;
  if (fn && fn(&ctx) != 0) ctx = nullptr;
  return ctx;
}

// device address of the scratch array in the current device's context
// (looked up on first use in that context)
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KASCADE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  void* ctx = current_context();
  Cached& c = g_scratch[dev];
  if (!ctx || !c.ptr || c.ctx != ctx) {
    // the lookup also makes the device's primary context current on this
    // thread if no runtime call has yet
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || p == nullptr) return KASCADE_ERR_CUDA;
    c.ptr = p;
    c.ctx = ctx ? ctx : current_context();
  }
  *out = c.ptr;
  return KASCADE_OK;
}

}  // namespace

extern "C" {

size_t kascade_select_decode_static_max_bytes(void) { return kStaticBytes; }

int kascade_select_decode_static(const kascade_shape* shape, const void* q, const void* k, int32_t* idx,
                                 void* stream) {
  if (!shape) return KASCADE_ERR_INVALID_ARG;
  const size_t need = kascade_workspace_bytes(shape, KASCADE_OP_SELECT);
  // an invalid shape: kascade_select reports the shape check's own status
  // (invalid or unsupported) before it launches anything
  if (need == 0) return kascade_select(shape, q, k, idx, nullptr, 0, stream);
  if (shape->q_len != 1) return KASCADE_ERR_UNSUPPORTED;
  if (need > kStaticBytes) return KASCADE_ERR_TOO_LARGE;
  if (!q || !k || !idx) return KASCADE_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc) return rc;
  return kascade_select(shape, q, k, idx, scratch, kStaticBytes, stream);
}

int kascade_select_decode_static_error(int* error_out, int clear, void* stream) {
  if (!error_out) return KASCADE_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc) return rc;
  return kascade_workspace_error(scratch, error_out, clear, stream);
}

}  // extern "C"
