// The extern "C" boundary of the library: argument checks, algorithm choice
// and launches on the caller's stream. See include/rglru.h for the contract.
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

using namespace rglru;

namespace rglru {

int check_shape(int B, int T, int D, int H, int io) {
  if (B < 1 || T < 1 || D < 1 || H < 1) return RGLRU_ERR_INVALID_ARG;
  if (io != RGLRU_IO_F32 && io != RGLRU_IO_BF16) return RGLRU_ERR_INVALID_ARG;
  if (D % H != 0 || D % 8 != 0) return RGLRU_ERR_INVALID_ARG;
  if (D / H > 1024) return RGLRU_ERR_UNSUPPORTED;
  if ((long long)B * D > (1ll << 31) - 1) return RGLRU_ERR_UNSUPPORTED;
  if ((long long)B * T > (1ll << 31) - 1) return RGLRU_ERR_UNSUPPORTED;
  return RGLRU_OK;
}

}  // namespace rglru

namespace {

constexpr int kVersion = 100;  // 0.1.0

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool opt_ok(const void *p) { return p == nullptr || aligned16(p); }

bool overlap(const void *a, size_t na, const void *b, size_t nb) {
  if (a == nullptr || b == nullptr || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

size_t io_bytes(int io) { return io == RGLRU_IO_F32 ? 4 : 2; }

}  // namespace

extern "C" {

const char *rglru_status_str(int status) {
  switch (status) {
    case RGLRU_OK: return "ok";
    case RGLRU_ERR_INVALID_ARG: return "invalid argument";
    case RGLRU_ERR_UNSUPPORTED: return "unsupported shape, type or algorithm";
    case RGLRU_ERR_CUDA: return "CUDA error";
    case RGLRU_ERR_TIMEOUT: return "device-side wait timed out";
    case RGLRU_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    default: return "unknown status";
  }
}

int rglru_version(void) { return kVersion; }

size_t rglru_fwd_workspace_bytes(int B, int T, int D, int H, int io) {
  if (check_shape(B, T, D, H, io) != RGLRU_OK) return 0;
  size_t need = generic_workspace_bytes(B, T, D, H);
  if (tc_supported(B, T, D, H, io)) {
    const size_t tc = tc_workspace_bytes(B, T, D, H);
    if (tc > need) need = tc;
  }
  return need < 256 ? 256 : need;
}

int rglru_fwd_launches(int B, int T, int D, int H, int io, int algo) {
  if (check_shape(B, T, D, H, io) != RGLRU_OK) return 0;
  if (algo != RGLRU_ALGO_AUTO && algo != RGLRU_ALGO_GENERIC && algo != RGLRU_ALGO_TENSOR)
    return 0;
  const bool tc = tc_supported(B, T, D, H, io);
  if (algo == RGLRU_ALGO_TENSOR && !tc) return 0;
  if (algo == RGLRU_ALGO_GENERIC || !tc) return generic_kernel_launches(B, T, H);
  return 1;
}

int rglru_decode_launches(int B, int D, int H, int io, int algo) {
  if (check_shape(B, 1, D, H, io) != RGLRU_OK) return 0;
  if (algo != RGLRU_ALGO_AUTO && algo != RGLRU_ALGO_GENERIC && algo != RGLRU_ALGO_TENSOR)
    return 0;
  const bool tc = tc_decode_supported(B, D, H, io);
  if (algo == RGLRU_ALGO_TENSOR && !tc) return 0;
  if (algo == RGLRU_ALGO_GENERIC || !tc) return 1;
  return tc_decode_launches(D, H);
}

int rglru_fwd_ex(const void *x, const void *conv_w, const void *W_a, const void *b_a,
                 const void *W_x, const void *b_x, const float *Lambda, const float *h0,
                 const void *conv_state_in, void *y, float *h_T, void *conv_state_out, int B,
                 int T, int D, int H, int io, void *workspace, size_t workspace_bytes,
                 int *dev_status, void *stream, int algo, const rglru_fwd_options *opts) {
  int st = check_shape(B, T, D, H, io);
  if (st != RGLRU_OK) return st;
  if (!x || !conv_w || !W_a || !b_a || !W_x || !b_x || !Lambda || !y)
    return RGLRU_ERR_INVALID_ARG;
  const void *req[] = {x, conv_w, W_a, b_a, W_x, b_x, Lambda, y};
  for (const void *p : req)
    if (!aligned16(p)) return RGLRU_ERR_INVALID_ARG;
  if (!opt_ok(h0) || !opt_ok(conv_state_in) || !opt_ok(h_T) || !opt_ok(conv_state_out) ||
      !opt_ok(dev_status))
    return RGLRU_ERR_INVALID_ARG;
  const size_t eb = io_bytes(io);
  const size_t seq_bytes = (size_t)B * T * D * eb;
  const size_t cs_bytes = (size_t)B * 3 * D * eb;
  if (overlap(y, seq_bytes, x, seq_bytes)) return RGLRU_ERR_INVALID_ARG;
  if (overlap(conv_state_out, cs_bytes, conv_state_in, cs_bytes)) return RGLRU_ERR_INVALID_ARG;
  if (overlap(conv_state_out, cs_bytes, x, seq_bytes)) return RGLRU_ERR_INVALID_ARG;
  if (algo != RGLRU_ALGO_AUTO && algo != RGLRU_ALGO_GENERIC && algo != RGLRU_ALGO_TENSOR)
    return RGLRU_ERR_INVALID_ARG;
  const bool tc = tc_supported(B, T, D, H, io);
  if (algo == RGLRU_ALGO_TENSOR && !tc) return RGLRU_ERR_UNSUPPORTED;
  const bool use_tc = tc && algo != RGLRU_ALGO_GENERIC;

  const size_t need =
      use_tc ? tc_workspace_bytes(B, T, D, H) : generic_workspace_bytes(B, T, D, H);
  if (need > 0 && (workspace == nullptr || !aligned16(workspace) || workspace_bytes < need))
    return RGLRU_ERR_WORKSPACE;

  if (opts != nullptr && opts->wait_limit_ns > 0 && opts->wait_limit_ns < 1000000ull)
    return RGLRU_ERR_INVALID_ARG;                // below 1 ms a healthy wait could expire
  if (opts != nullptr && opts->fault_unpublished_tile < 0) return RGLRU_ERR_INVALID_ARG;
  FwdArgs p{x, conv_w, W_a, b_a, W_x, b_x, Lambda, h0, conv_state_in, y, h_T, conv_state_out,
            B, T, D, H, dev_status,
            opts ? opts->wait_limit_ns : 0ull, opts ? opts->fault_unpublished_tile - 1 : -1,
            opts ? static_cast<cudaEvent_t>(opts->kernel_begin_event) : nullptr,
            opts ? static_cast<cudaEvent_t>(opts->kernel_end_event) : nullptr};
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = use_tc ? launch_fwd_tc(p, workspace, s) : launch_fwd_generic(p, io, workspace, s);
  return e == cudaSuccess ? RGLRU_OK : RGLRU_ERR_CUDA;
}

int rglru_fwd_algo(const void *x, const void *conv_w, const void *W_a, const void *b_a,
                   const void *W_x, const void *b_x, const float *Lambda, const float *h0,
                   const void *conv_state_in, void *y, float *h_T, void *conv_state_out,
                   int B, int T, int D, int H, int io, void *workspace,
                   size_t workspace_bytes, int *dev_status, void *stream, int algo) {
  return rglru_fwd_ex(x, conv_w, W_a, b_a, W_x, b_x, Lambda, h0, conv_state_in, y, h_T,
                      conv_state_out, B, T, D, H, io, workspace, workspace_bytes, dev_status,
                      stream, algo, nullptr);
}

int rglru_fwd(const void *x, const void *conv_w, const void *W_a, const void *b_a,
              const void *W_x, const void *b_x, const float *Lambda, const float *h0,
              const void *conv_state_in, void *y, float *h_T, void *conv_state_out, int B,
              int T, int D, int H, int io, void *workspace, size_t workspace_bytes,
              int *dev_status, void *stream) {
  return rglru_fwd_algo(x, conv_w, W_a, b_a, W_x, b_x, Lambda, h0, conv_state_in, y, h_T,
                        conv_state_out, B, T, D, H, io, workspace, workspace_bytes, dev_status,
                        stream, RGLRU_ALGO_AUTO);
}

int rglru_decode_step_algo(const void *x_t, void *conv_state, int pos, float *h, void *y_t,
                           const void *conv_w, const void *W_a, const void *b_a,
                           const void *W_x, const void *b_x, const float *Lambda, int B,
                           int D, int H, int io, void *stream, int algo) {
  int st = check_shape(B, 1, D, H, io);
  if (st != RGLRU_OK) return st;
  if (pos < 0) return RGLRU_ERR_INVALID_ARG;
  if (!x_t || !conv_state || !h || !y_t || !conv_w || !W_a || !b_a || !W_x || !b_x || !Lambda)
    return RGLRU_ERR_INVALID_ARG;
  const void *req[] = {x_t, conv_state, h, y_t, conv_w, W_a, b_a, W_x, b_x, Lambda};
  for (const void *p : req)
    if (!aligned16(p)) return RGLRU_ERR_INVALID_ARG;
  const size_t eb = io_bytes(io);
  const size_t row_bytes = (size_t)B * D * eb;
  if (overlap(y_t, row_bytes, x_t, row_bytes)) return RGLRU_ERR_INVALID_ARG;
  if (overlap(y_t, row_bytes, conv_state, 3 * row_bytes)) return RGLRU_ERR_INVALID_ARG;
  if (overlap(h, (size_t)B * D * 4, conv_state, 3 * row_bytes)) return RGLRU_ERR_INVALID_ARG;
  if (algo != RGLRU_ALGO_AUTO && algo != RGLRU_ALGO_GENERIC && algo != RGLRU_ALGO_TENSOR)
    return RGLRU_ERR_INVALID_ARG;
  const bool tc = tc_decode_supported(B, D, H, io);
  if (algo == RGLRU_ALGO_TENSOR && !tc) return RGLRU_ERR_UNSUPPORTED;
  DecArgs p{x_t, conv_state, pos, h, y_t, conv_w, W_a, b_a, W_x, b_x, Lambda, B, D, H};
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = (tc && algo != RGLRU_ALGO_GENERIC) ? launch_decode_tc(p, s)
                                                     : launch_decode_generic(p, io, s);
  return e == cudaSuccess ? RGLRU_OK : RGLRU_ERR_CUDA;
}

int rglru_decode_step(const void *x_t, void *conv_state, int pos, float *h, void *y_t,
                      const void *conv_w, const void *W_a, const void *b_a, const void *W_x,
                      const void *b_x, const float *Lambda, int B, int D, int H, int io,
                      void *stream) {
  return rglru_decode_step_algo(x_t, conv_state, pos, h, y_t, conv_w, W_a, b_a, W_x, b_x,
                                Lambda, B, D, H, io, stream, RGLRU_ALGO_AUTO);
}

}  // extern "C"

extern "C" {

size_t rglru_bwd_workspace_bytes(int B, int T, int D, int H, int io) {
  if (check_shape(B, T, D, H, io) != RGLRU_OK) return 0;
  return bwd_workspace_bytes(B, T, D, H);
}

int rglru_bwd_launches(int B, int T, int D, int H, int io) {
  if (check_shape(B, T, D, H, io) != RGLRU_OK) return 0;
  return bwd_launches();
}

int rglru_bwd(const void *x, const void *conv_w, const void *W_a, const void *b_a,
              const void *W_x, const void *b_x, const float *Lambda, const float *h0,
              const void *conv_state_in, const void *dy, const float *dh_T, void *dx,
              float *dconv_w, float *dW_a, float *db_a, float *dW_x, float *db_x,
              float *dLambda, float *dh0, float *dconv_state_in, int B, int T, int D, int H,
              int io, void *workspace, size_t workspace_bytes, void *stream) {
  int st = check_shape(B, T, D, H, io);
  if (st != RGLRU_OK) return st;
  const void *req[] = {x, conv_w, W_a, b_a, W_x, b_x, Lambda, dy, dx,
                       dconv_w, dW_a, db_a, dW_x, db_x, dLambda};
  for (const void *p : req)
    if (p == nullptr || !aligned16(p)) return RGLRU_ERR_INVALID_ARG;
  if (!opt_ok(h0) || !opt_ok(conv_state_in) || !opt_ok(dh_T) || !opt_ok(dh0) ||
      !opt_ok(dconv_state_in))
    return RGLRU_ERR_INVALID_ARG;
  const size_t eb = io_bytes(io);
  const size_t seq = (size_t)B * T * D * eb;
  const size_t bw = (size_t)D / H;
  // outputs must not overlap the inputs they are computed from
  const void *ins[] = {x, dy, conv_w, W_a, W_x};
  const size_t in_n[] = {seq, seq, 4 * (size_t)D * eb, (size_t)D * bw * eb, (size_t)D * bw * eb};
  const void *outs[] = {dx, dconv_w, dW_a, dW_x, db_a, db_x, dLambda, dh0, dconv_state_in};
  const size_t out_n[] = {seq, 16 * (size_t)D, 4 * (size_t)D * bw, 4 * (size_t)D * bw,
                          4 * (size_t)D, 4 * (size_t)D, 4 * (size_t)D, 4 * (size_t)B * D,
                          12 * (size_t)B * D};
  for (int i = 0; i < 5; ++i)
    for (int o = 0; o < 9; ++o)
      if (overlap(ins[i], in_n[i], outs[o], out_n[o])) return RGLRU_ERR_INVALID_ARG;
  const size_t need = bwd_workspace_bytes(B, T, D, H);
  if (workspace == nullptr || !aligned16(workspace) || workspace_bytes < need)
    return RGLRU_ERR_WORKSPACE;
  BwdArgs p{x, conv_w, W_a, b_a, W_x, b_x, Lambda, h0, conv_state_in, dy, dh_T, dx,
            dconv_w, dW_a, db_a, dW_x, db_x, dLambda, dh0, dconv_state_in, B, T, D, H};
  const cudaError_t e = launch_bwd(p, io, workspace, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RGLRU_OK : RGLRU_ERR_CUDA;
}

}  // extern "C"

extern "C" {

size_t rglru_block_fwd_workspace_bytes(int B, int T, int Dm, int D, int H, int io) {
  if (check_shape(B, T, D, H, io) != RGLRU_OK || Dm < 8 || Dm % 8 != 0) return 0;
  return block_layout(B, T, D, io, rglru_fwd_workspace_bytes(B, T, D, H, io)).total;
}

int rglru_block_fwd(const void *x, const void *W_in, const void *W_gate, const void *W_out,
                    const void *conv_w, const void *W_a, const void *b_a, const void *W_x,
                    const void *b_x, const float *Lambda, const float *h0,
                    const void *conv_state_in, void *out, float *h_T, void *conv_state_out,
                    int B, int T, int Dm, int D, int H, int io, void *workspace,
                    size_t workspace_bytes, int *dev_status, void *stream) {
  int st = check_shape(B, T, D, H, io);
  if (st != RGLRU_OK) return st;
  if (Dm < 8 || Dm % 8 != 0) return RGLRU_ERR_INVALID_ARG;
  const void *req[] = {x, W_in, W_gate, W_out, out};
  for (const void *p : req)
    if (p == nullptr || !aligned16(p)) return RGLRU_ERR_INVALID_ARG;
  const size_t eb = io_bytes(io);
  if (overlap(out, (size_t)B * T * Dm * eb, x, (size_t)B * T * Dm * eb))
    return RGLRU_ERR_INVALID_ARG;
  const size_t fwd_ws = rglru_fwd_workspace_bytes(B, T, D, H, io);
  const BlockLayout L = block_layout(B, T, D, io, fwd_ws);
  if (workspace == nullptr || !aligned16(workspace) || workspace_bytes < L.total)
    return RGLRU_ERR_WORKSPACE;
  unsigned char *w = static_cast<unsigned char *>(workspace);
  void *xr = w + L.off_xr, *g = w + L.off_g, *y = w + L.off_y, *fw = w + L.off_fwd;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int M = B * T;
  if (io == RGLRU_IO_BF16) {
    // tensor-core GEMMs; the gating runs in the gate projection's epilogue, over y
    if ((st = launch_gemm_tc(M, D, Dm, x, W_in, nullptr, xr, dev_status, s)) != RGLRU_OK)
      return st;
    st = rglru_fwd(xr, conv_w, W_a, b_a, W_x, b_x, Lambda, h0, conv_state_in, y, h_T,
                   conv_state_out, B, T, D, H, io, fw, workspace_bytes - L.off_fwd, dev_status,
                   stream);
    if (st != RGLRU_OK) return st;
    if ((st = launch_gemm_tc(M, D, Dm, x, W_gate, y, y, dev_status, s)) != RGLRU_OK) return st;
    return launch_gemm_tc(M, Dm, D, y, W_out, nullptr, out, dev_status, s);
  }
  if ((st = launch_block_gemm(io, M, D, Dm, x, W_in, xr, s)) != RGLRU_OK) return st;
  if ((st = launch_block_gemm(io, M, D, Dm, x, W_gate, g, s)) != RGLRU_OK) return st;
  st = rglru_fwd(xr, conv_w, W_a, b_a, W_x, b_x, Lambda, h0, conv_state_in, y, h_T,
                 conv_state_out, B, T, D, H, io, fw, workspace_bytes - L.off_fwd, dev_status,
                 stream);
  if (st != RGLRU_OK) return st;
  if (launch_gelu_gate(io, y, g, (size_t)M * D, s) != cudaSuccess) return RGLRU_ERR_CUDA;
  return launch_block_gemm(io, M, Dm, D, y, W_out, out, s);
}

}  // extern "C"

