// The recurrent block around the RG-LRU layer (S. De's thread on Griffin: a
// simple recurrent block with a temporal Conv1D and the RG-LRU, and gated MLP
// blocks; "Beyond Transformer Architecture: Griffin and Google RecurrentGemma",
// "Core Components of Griffin", 3. Architecture Design: a GeGeLU-like gated
// MLP). The pages print no equation for it. Read as two branches from the
// block input x (B, T, Dm):
//   gate branch       g = GeLU(x W_gate)                      (B, T, D)
//   recurrent branch  y = RG-LRU layer (Conv1D, gates, scan) of x W_in
//   output            out = (y * g) W_out                      (B, T, Dm)
// with GeLU(v) = v Phi(v) = v (1 + erf(v / sqrt 2)) / 2 (the exact form).
//
// bf16 I/O: the three projections run on the library's tcgen05 GEMM
// (gemm_tc.cu), and the gating is fused into the gate projection's epilogue:
// y * GeLU(x W_gate) is formed where x W_gate leaves the accumulator, written
// over y. fp32 I/O: the projections run on cuBLAS with the pedantic fp32
// compute type (no TF32: the exact fp32 reference of the block), and
// y * GeLU(g) is one elementwise kernel over 16-byte vectors. Intermediates
// are in the I/O type in the caller's workspace.
#include <cublas_v2.h>

#include "common.cuh"
#include "kernels.h"

namespace rglru {

namespace {

// One cuBLAS handle per (host thread, device): a handle is bound to the
// device that was current at its creation and must not be shared by threads
// that set different streams on it.
cublasHandle_t block_handle(int dev) {
  constexpr int kMaxDev = 64;
  thread_local cublasHandle_t handles[kMaxDev] = {};
  if (dev < 0 || dev >= kMaxDev) return nullptr;
  if (handles[dev] == nullptr) {
    cublasHandle_t h = nullptr;
    if (cublasCreate(&h) != CUBLAS_STATUS_SUCCESS) return nullptr;
    handles[dev] = h;
  }
  return handles[dev];
}

// Row-major C[M x N] = A[M x K] B[K x N]: column-major C^T = B^T A^T.
cublasStatus_t gemm_rm(cublasHandle_t h, int io, int M, int N, int K, const void *A,
                       const void *B, void *C) {
  const float one = 1.0f, zero = 0.0f;
  const cudaDataType_t t = io == RGLRU_IO_F32 ? CUDA_R_32F : CUDA_R_16BF;
  const cublasComputeType_t ct =
      io == RGLRU_IO_F32 ? CUBLAS_COMPUTE_32F_PEDANTIC : CUBLAS_COMPUTE_32F;
  return cublasGemmEx(h, CUBLAS_OP_N, CUBLAS_OP_N, N, M, K, &one, B, t, N, A, t, K, &zero, C, t,
                      N, ct, CUBLAS_GEMM_DEFAULT);
}

// y[i] *= GeLU(g[i]) over n elements, 16 bytes per thread per step.
template <typename T>
__global__ void __launch_bounds__(256) gelu_gate_kernel(T *__restrict__ y,
                                                        const T *__restrict__ g, size_t n) {
  constexpr int kV = 16 / sizeof(T);
  const size_t nv = n / kV;
  for (size_t v = blockIdx.x * (size_t)blockDim.x + threadIdx.x; v < nv;
       v += (size_t)gridDim.x * blockDim.x) {
    uint4 yv = reinterpret_cast<const uint4 *>(y)[v];
    const uint4 gv = __ldg(reinterpret_cast<const uint4 *>(g) + v);
    T *ye = reinterpret_cast<T *>(&yv);
    const T *ge = reinterpret_cast<const T *>(&gv);
#pragma unroll
    for (int e = 0; e < kV; ++e) ye[e] = from_f32<T>(to_f32<T>(ye[e]) * gelu_exact(to_f32<T>(ge[e])));
    reinterpret_cast<uint4 *>(y)[v] = yv;
  }
  // the tail (n not a multiple of kV)
  const size_t i = nv * kV + blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (i < n) y[i] = from_f32<T>(to_f32<T>(y[i]) * gelu_exact(to_f32<T>(g[i])));
}

}  // namespace

BlockLayout block_layout(int B, int T, int D, int io, size_t fwd_ws) {
  const size_t eb = io == RGLRU_IO_F32 ? 4 : 2;
  const size_t seq = align_up((size_t)B * T * D * eb, 256);
  BlockLayout L;
  L.off_xr = 0;
  L.off_g = seq;
  L.off_y = 2 * seq;
  L.off_fwd = 3 * seq;
  L.total = 3 * seq + align_up(fwd_ws, 256);
  return L;
}

int launch_block_gemm(int io, int M, int N, int K, const void *A, const void *B, void *C,
                      cudaStream_t st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RGLRU_ERR_CUDA;
  cublasHandle_t h = block_handle(dev);
  if (h == nullptr) return RGLRU_ERR_CUDA;
  if (cublasSetStream(h, st) != CUBLAS_STATUS_SUCCESS) return RGLRU_ERR_CUDA;
  return gemm_rm(h, io, M, N, K, A, B, C) == CUBLAS_STATUS_SUCCESS ? RGLRU_OK : RGLRU_ERR_CUDA;
}

cudaError_t launch_gelu_gate(int io, void *y, const void *g, size_t n, cudaStream_t st) {
  const int threads = 256;
  const size_t per = (io == RGLRU_IO_F32 ? 4 : 8) * (size_t)threads;
  size_t blocks = (n + per - 1) / per;
  if (blocks < 1) blocks = 1;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (io == RGLRU_IO_F32)
    gelu_gate_kernel<float><<<(unsigned)blocks, threads, 0, st>>>(
        static_cast<float *>(y), static_cast<const float *>(g), n);
  else
    gelu_gate_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, st>>>(
        static_cast<__nv_bfloat16 *>(y), static_cast<const __nv_bfloat16 *>(g), n);
  return cudaGetLastError();
}

}  // namespace rglru
