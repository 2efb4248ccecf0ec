// Allocation-free variant of shampoo_inv_root.
//
// Some callers cannot allocate device memory when they need a root: code
// running while a CUDA graph is being captured (a cudaMalloc there breaks or
// invalidates the capture), allocator callbacks and memory-pool hooks that
// must not re-enter the allocator, and programs with a fixed, preallocated
// memory budget.  They call shampoo_inv_root_static, which takes its scratch
// space from a fixed-size array in device global memory that this file
// defines instead of from a caller-provided workspace.
#include <cstdio>
#include <mutex>
#include <string>

#include "../../include/shampoo.h"
#include "internal.h"

namespace {

// Scratch shared by every call on a device.  In host code the symbol is only
// a stand-in for the device array; its device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char shp_static_scratch[SHP_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch[kMaxDevices] = {nullptr};

shp_status fail(shp_status code, const char* msg) {
  shp::set_last_error(msg);
  return code;
}

}  // namespace

extern "C" {

SHP_API shp_status shampoo_inv_root_static(const float* A, int32_t count, int32_t n, float eps, int32_t p,
                                           int32_t method, int32_t iters, int32_t dtype, int32_t scaling,
                                           int32_t pi_vectors, int32_t pi_iters, const float* pi_starts,
                                           float* X_out, float* scale_out, int32_t* status_out, void* stream) {
  const size_t need = shampoo_inv_root_workspace_bytes(count, n, method, dtype, scaling, pi_vectors);
  if (need == 0)  // invalid sizes or enums: let the checked call report them
    return shampoo_inv_root(A, count, n, eps, p, method, iters, dtype, scaling, pi_vectors, pi_iters, pi_starts,
                            X_out, scale_out, status_out, nullptr, 0, stream);
  if (need > (size_t)SHP_STATIC_SCRATCH_BYTES) {
    char buf[256];
    snprintf(buf, sizeof(buf),
             "shampoo_inv_root_static: this stack needs %zu bytes of scratch; the static scratch holds %zu "
             "(SHP_STATIC_SCRATCH_BYTES); use shampoo_inv_root with a workspace",
             need, (size_t)SHP_STATIC_SCRATCH_BYTES);
    return fail(SHP_ERR_WORKSPACE, buf);
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SHP_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(SHP_ERR_UNSUPPORTED, "device ordinal above 63");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch[dev]) {  // once per device, with that device current
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, shp_static_scratch);
      if (e != cudaSuccess) return fail(SHP_ERR_CUDA, cudaGetErrorString(e));
      g_scratch[dev] = ptr;
    }
    scratch = g_scratch[dev];
  }
  return shampoo_inv_root(A, count, n, eps, p, method, iters, dtype, scaling, pi_vectors, pi_iters, pi_starts,
                          X_out, scale_out, status_out, scratch, (size_t)SHP_STATIC_SCRATCH_BYTES, stream);
}

}  // extern "C"
