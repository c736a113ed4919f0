// rglru_fwd_noalloc: the generic forward with its scratch in a static device
// array instead of a caller-provided workspace, for callers that cannot
// allocate device memory (see include/rglru.h).
#include <mutex>

#include "common.cuh"
#include "kernels.h"

// The fixed scratch. Every device that loads the library holds one copy until
// the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[RGLRU_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices];  // device address of g_noalloc_scratch, per device

// Looks up, once per device and with that device current, the device address
// of the static array. In host code the array's name is only a host-side
// stand-in, never a device address.
int scratch_for_current_device(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return RGLRU_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RGLRU_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return RGLRU_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return RGLRU_OK;
}

}  // namespace

extern "C" int rglru_fwd_noalloc(const void *x, const void *conv_w, const void *W_a,
                                 const void *b_a, const void *W_x, const void *b_x,
                                 const float *Lambda, const float *h0,
                                 const void *conv_state_in, void *y, float *h_T,
                                 void *conv_state_out, int B, int T, int D, int H, int io,
                                 void *stream) {
  const size_t need = rglru_fwd_workspace_bytes(B, T, D, H, io);
  if (need == 0) return RGLRU_ERR_INVALID_ARG;
  if (need > RGLRU_NOALLOC_SCRATCH_BYTES) return RGLRU_ERR_WORKSPACE;
  void *scratch = nullptr;
  const int st = scratch_for_current_device(&scratch);
  if (st != RGLRU_OK) return st;
  return rglru_fwd_algo(x, conv_w, W_a, b_a, W_x, b_x, Lambda, h0, conv_state_in, y, h_T,
                        conv_state_out, B, T, D, H, io, scratch, RGLRU_NOALLOC_SCRATCH_BYTES,
                        nullptr, stream, RGLRU_ALGO_GENERIC);
}
