// Internal interface between the C ABI layer and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace rglru {

struct FwdArgs {
  const void *x, *conv_w, *W_a, *b_a, *W_x, *b_x;
  const float *Lambda, *h0;
  const void *conv_state_in;
  void *y;
  float *h_T;
  void *conv_state_out;
  int B, T, D, H;
  int *dev_status;
  unsigned long long wait_ns;  // 0: default bound of device-side waits
  int fault_tile;              // testing only: tile of unit 0 that never publishes (-1: off)
  cudaEvent_t ev_begin, ev_end;  // recorded around the compute kernels when set
};

struct BwdArgs {
  const void *x, *conv_w, *W_a, *b_a, *W_x, *b_x;
  const float *Lambda, *h0;
  const void *conv_state_in, *dy;
  const float *dh_T;
  void *dx;
  float *dconv_w, *dW_a, *db_a, *dW_x, *db_x, *dLambda, *dh0, *dconv_state_in;
  int B, T, D, H;
};

struct DecArgs {
  const void *x_t;
  void *conv_state;
  int pos;
  float *h;
  void *y_t;
  const void *conv_w, *W_a, *b_a, *W_x, *b_x;
  const float *Lambda;
  int B, D, H;
};

// Shape checks shared by every entry point: an rglru_status (RGLRU_OK when the
// sizes and the I/O type are well formed and supported).
int check_shape(int B, int T, int D, int H, int io);

struct GenericPlan {
  int nseg;  // time segments
  int L;     // tokens per segment (the last may be shorter)
};

GenericPlan generic_plan(int B, int T, int H);
size_t generic_workspace_bytes(int B, int T, int D, int H);
int generic_kernel_launches(int B, int T, int H);
size_t bwd_workspace_bytes(int B, int T, int D, int H);
int bwd_launches();
cudaError_t launch_bwd(const BwdArgs &p, int io, void *ws, cudaStream_t st);

// Recurrent block around the layer (block.cu): workspace offsets of x W_in,
// x W_gate, the layer output y and the layer's own forward workspace.
struct BlockLayout {
  size_t off_xr, off_g, off_y, off_fwd, total;
};
BlockLayout block_layout(int B, int T, int D, int io, size_t fwd_ws);
// Row-major C[M x N] = A[M x K] B[K x N] in the I/O type (cuBLAS); an RGLRU_* status.
int launch_block_gemm(int io, int M, int N, int K, const void *A, const void *B, void *C,
                      cudaStream_t st);
cudaError_t launch_gelu_gate(int io, void *y, const void *g, size_t n, cudaStream_t st);
// Row-major bf16 C[M x N] = A[M x K] B[K x N] on the tensor core (gemm_tc.cu);
// with Y (M x N bf16, may alias C) non-null, C = Y * GeLU(A B). An RGLRU_* status.
bool gemm_tc_supported(int M, int N, int K);
int launch_gemm_tc(int M, int N, int K, const void *A, const void *B, const void *Y, void *C,
                   int *dev_status, cudaStream_t st);
cudaError_t launch_fwd_generic(const FwdArgs &p, int io, void *ws, cudaStream_t st);
cudaError_t launch_decode_generic(const DecArgs &p, int io, cudaStream_t st);

// Tensor-core (tcgen05) fused forward, bf16 I/O.
bool tc_supported(int B, int T, int D, int H, int io);
size_t tc_workspace_bytes(int B, int T, int D, int H);
cudaError_t launch_fwd_tc(const FwdArgs &p, void *ws, cudaStream_t st);

// Tensor-core decode step, bf16 I/O (same shape rules as the forward).
bool tc_decode_supported(int B, int D, int H, int io);
int tc_decode_launches(int D, int H);
cudaError_t launch_decode_tc(const DecArgs &p, cudaStream_t st);

}  // namespace rglru
