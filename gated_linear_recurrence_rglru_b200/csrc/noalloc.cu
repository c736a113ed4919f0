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

// The device address of the static array on the current device. In host code
// the array's name is only a host-side stand-in, never a device address, so
// the address is looked up with cudaGetSymbolAddress, with the device current.
// The lookup is repeated on every call made while `stream` is not capturing
// (after a device reset the module is loaded again and the array may move);
// while it is capturing, the address found by the last such call is used, and
// a device with none yet is refused.
int scratch_for_current_device(cudaStream_t stream, void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return RGLRU_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RGLRU_ERR_UNSUPPORTED;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return RGLRU_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return RGLRU_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  if (g_scratch_ptr[dev] == nullptr) return RGLRU_ERR_CUDA;
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
  // the shape checks of rglru_fwd first (the same status for the same sizes),
  // then the scratch of the generic algorithm, the one this entry point runs
  int st = rglru::check_shape(B, T, D, H, io);
  if (st != RGLRU_OK) return st;
  const size_t need = rglru::generic_workspace_bytes(B, T, D, H);
  if (need > RGLRU_NOALLOC_SCRATCH_BYTES) return RGLRU_ERR_WORKSPACE;
  void *scratch = nullptr;
  st = scratch_for_current_device(static_cast<cudaStream_t>(stream), &scratch);
  if (st != RGLRU_OK) return st;
  return rglru_fwd_algo(x, conv_w, W_a, b_a, W_x, b_x, Lambda, h0, conv_state_in, y, h_T,
                        conv_state_out, B, T, D, H, io, scratch, RGLRU_NOALLOC_SCRATCH_BYTES,
                        nullptr, stream, RGLRU_ALGO_GENERIC);
}
