/*
 * rglru.h -- C ABI of the B200 (sm_100a) RG-LRU library.
 *
 * The RG-LRU layer, the recurrent core of Griffin / Hawk. The source pages
 * describe its parts but print no formula for it; the equations below are the
 * layer's definition as this library states it, and every page passage cited
 * in this header supports only what it says:
 *   - S. De's thread on Griffin ("how we got there"): the RG-LRU is the LRU, a
 *     diagonal recurrence, with a recurrent gate added; the simple recurrent
 *     block carries a temporal Conv1D; the layer is memory-bound, its kernel
 *     optimises HBM accesses and runs a linear scan rather than a parallel one;
 *   - "Beyond Transformer Architecture: Griffin and Google RecurrentGemma",
 *     "Core Components of Griffin", 1. RG-LRU: the gates do not depend on the
 *     recurrent state; "Key Strengths of RecurrentGemma", 1. Reduced Memory
 *     Usage: the state has a fixed size, whatever the sequence length.
 *
 *   u_t     = sum_{k=0..3} conv_w[k] * x_{t-3+k}          causal depthwise Conv1D, width 4
 *   r_t     = sigmoid(u_t W_a + b_a)                       block-diagonal per head
 *   i_t     = sigmoid(u_t W_x + b_x)                       block-diagonal per head
 *   log a_t = -8 * r_t * softplus(-Lambda)                 a_t = sigmoid(Lambda)^(8 r_t)
 *   h_t     = a_t * h_{t-1} + sqrt(1 - a_t^2) * (i_t * u_t)
 *   y_t     = h_t
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     allocates no memory and keeps no state between calls. Every pointer must
 *     be 16-byte aligned. Tensors are dense and row-major in the shapes given.
 *   - io selects the storage type of x, conv_w, W_a, W_x, b_a, b_x, y and the
 *     conv state: RGLRU_IO_F32 (float) or RGLRU_IO_BF16 (bfloat16). Lambda and
 *     every recurrent state (h0, h_T, h) are always float. Arithmetic is fp32.
 *   - D = H * bw. Weights W_a, W_x have shape (H, bw, bw) with
 *     z[h*bw + j] = sum_i u[h*bw + i] * W[h, i, j]. conv_w has shape (4, D);
 *     tap k multiplies x_{t-3+k} (tap 3 is the current input).
 *   - A conv state is (B, 3, D) in the I/O type. In rglru_fwd it is
 *     chronological: slot 0 holds x_{t-3}, slot 2 holds x_{t-1}. In
 *     rglru_decode_step it is a ring: at step pos, slot pos%3 holds x_{pos-3},
 *     slot (pos+1)%3 holds x_{pos-2} and slot (pos+2)%3 holds x_{pos-1}; a
 *     chronological state is the ring at pos = 0.
 *   - stream is a cudaStream_t (NULL = the legacy default stream). Calls are
 *     asynchronous: the return value reports argument checks and launch
 *     errors only.
 *   - Return values are rglru_status codes. On any nonzero return nothing was
 *     launched (argument errors) or the launch failed (RGLRU_ERR_CUDA).
 */
#ifndef RGLRU_B200_H
#define RGLRU_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RGLRU_OK = 0,
  RGLRU_ERR_INVALID_ARG = 1,   /* NULL or misaligned pointer, non-positive or inconsistent size */
  RGLRU_ERR_UNSUPPORTED = 2,   /* well-formed request outside what the kernels implement */
  RGLRU_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed */
  RGLRU_ERR_TIMEOUT = 4,       /* device side: a bounded wait expired (reported via dev_status) */
  RGLRU_ERR_WORKSPACE = 5      /* workspace NULL, misaligned or smaller than required */
} rglru_status;

typedef enum { RGLRU_IO_F32 = 0, RGLRU_IO_BF16 = 1 } rglru_io;

typedef enum {
  RGLRU_ALGO_AUTO = 0,         /* tensor-core path when supported, else the generic path */
  RGLRU_ALGO_GENERIC = 1,      /* CUDA-core gates, three passes over time segments */
  RGLRU_ALGO_TENSOR = 2        /* tcgen05 gate contraction, single fused pass */
} rglru_algo;

/* Human-readable name of a status code. Never NULL. */
const char *rglru_status_str(int status);

/* Library version, major*10000 + minor*100 + patch. */
int rglru_version(void);

/*
 * Bytes of device workspace that rglru_fwd / rglru_fwd_algo need for this
 * shape, for any algorithm. Returns 0 on invalid sizes. The workspace holds
 * the per-segment carries of the time-split scan and the scheduling counters;
 * it needs no initialisation by the caller and may be reused across calls
 * issued to the same stream (calls that overlap on the GPU need separate
 * workspaces).
 */
size_t rglru_fwd_workspace_bytes(int B, int T, int D, int H, int io);

/*
 * Number of kernel launches one rglru_fwd_algo call with these arguments
 * issues on its stream (0 on invalid or unsupported arguments).
 */
int rglru_fwd_launches(int B, int T, int D, int H, int io, int algo);

/*
 * Full-sequence forward of the layer: every equation above over t = 0..T-1,
 * the scan carried across time by a linear scan (S. De's thread: linear scans
 * rather than parallel ones), split across thread blocks by tiles of time.
 *   x              (B, T, D)  io     input of the Conv1D
 *   conv_w         (4, D)     io
 *   W_a, W_x       (H, bw, bw) io    gate weights
 *   b_a, b_x       (D)        io     gate biases
 *   Lambda         (D)        float  a = sigmoid(Lambda)
 *   h0             (B, D)     float  initial state, or NULL for zeros
 *   conv_state_in  (B, 3, D)  io     chronological history, or NULL for zeros
 *   y              (B, T, D)  io     output h_t (written)
 *   h_T            (B, D)     float  final state (written), or NULL
 *   conv_state_out (B, 3, D)  io     last three inputs, chronological (written), or NULL;
 *                                    must not alias conv_state_in
 *   workspace      device scratch of at least rglru_fwd_workspace_bytes(...)
 *   dev_status     device int, or NULL. On a device-side failure a kernel
 *                  stores a nonzero word there (the first failure only): bits
 *                  0-7 hold the rglru_status (RGLRU_ERR_TIMEOUT when a bounded
 *                  wait expired; y is then incomplete); for a timeout of the
 *                  tensor-core forward bits 8-15 name the wait that gave up
 *                  (1 tile claims and input copies, 2 MMA issue, 3 Conv1D,
 *                  4 epilogue, 5 a predecessor tile's carry) and bits 16-31
 *                  the index of the thread block. The library never clears it.
 * Requirements: B, T >= 1; H >= 1; D % H == 0; D % 8 == 0; bw = D / H <= 1024.
 */
int rglru_fwd(const void *x, const void *conv_w, const void *W_a, const void *b_a,
              const void *W_x, const void *b_x, const float *Lambda, const float *h0,
              const void *conv_state_in, void *y, float *h_T, void *conv_state_out,
              int B, int T, int D, int H, int io, void *workspace, size_t workspace_bytes,
              int *dev_status, void *stream);

/*
 * rglru_fwd with an explicit algorithm (rglru_algo). RGLRU_ALGO_TENSOR needs
 * io = RGLRU_IO_BF16, D % 128 == 0 and bw in {64, 128, 256}; otherwise
 * it returns RGLRU_ERR_UNSUPPORTED. Both algorithms compute the same layer.
 */
int rglru_fwd_algo(const void *x, const void *conv_w, const void *W_a, const void *b_a,
                   const void *W_x, const void *b_x, const float *Lambda, const float *h0,
                   const void *conv_state_in, void *y, float *h_T, void *conv_state_out,
                   int B, int T, int D, int H, int io, void *workspace,
                   size_t workspace_bytes, int *dev_status, void *stream, int algo);

/*
 * Options of rglru_fwd_ex. Zero-initialise, then set what is needed.
 *   wait_limit_ns           bound of every device-side wait of the tensor-core
 *                           forward (a CTA waiting for its predecessor's carry, or
 *                           one of its pipeline stages); 0 = the default of 2 s.
 *                           Values from 1 ns to 1 ms are refused (INVALID_ARG):
 *                           healthy waits could expire.
 *   fault_unpublished_tile  testing of the failure path: 0 = off (the default,
 *                           and that of rglru_fwd and rglru_fwd_algo); n > 0: the
 *                           tile of index n - 1 in the first (batch row 0,
 *                           channels 0..127) group never publishes its carry, so
 *                           the waits of its successors run out: the call then
 *                           reports RGLRU_ERR_TIMEOUT through dev_status and
 *                           returns with y incomplete; the context stays usable.
 *                           Negative values are refused (INVALID_ARG).
 *   kernel_begin_event,     cudaEvent_t handles, or NULL: when set, recorded on the
 *   kernel_end_event        stream right before the first and right after the last
 *                           compute kernel of the call (after the reset of the
 *                           workspace), so that a caller can time the kernels alone.
 *                           The events must belong to the stream's device; the call
 *                           neither creates nor destroys them.
 */
typedef struct {
  unsigned long long wait_limit_ns;
  int fault_unpublished_tile;
  void *kernel_begin_event;
  void *kernel_end_event;
} rglru_fwd_options;

/* rglru_fwd_algo with options (NULL = defaults). */
int rglru_fwd_ex(const void *x, const void *conv_w, const void *W_a, const void *b_a,
                 const void *W_x, const void *b_x, const float *Lambda, const float *h0,
                 const void *conv_state_in, void *y, float *h_T, void *conv_state_out, int B,
                 int T, int D, int H, int io, void *workspace, size_t workspace_bytes,
                 int *dev_status, void *stream, int algo, const rglru_fwd_options *opts);

/*
 * Size of the library's fixed device scratch used by rglru_fwd_noalloc.
 * Every GPU that loads the library holds this much device memory until the
 * process exits.
 */
#define RGLRU_NOALLOC_SCRATCH_BYTES (2u << 20)

/*
 * rglru_fwd_noalloc: the forward of the layer (the generic algorithm, as
 * rglru_fwd_algo with RGLRU_ALGO_GENERIC) for callers that cannot allocate
 * device memory. The paper has no counterpart to this entry point: it exists
 * for deployment only.
 *
 * Who needs it: code that must not call cudaMalloc once it is running, such
 * as a serving loop that reserves all device memory for its own pool at
 * start-up, or a plugin hosted by a framework that owns the allocator and
 * gives the plugin no way to ask for scratch. rglru_fwd needs a workspace
 * from its caller; this variant takes none. Its scratch (the per-segment
 * carries of the time split) lives in a static device array of
 * RGLRU_NOALLOC_SCRATCH_BYTES inside the library, and the call allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *
 * Arguments, layouts and results are those of rglru_fwd without the
 * workspace and dev_status arguments; invalid sizes get the status that
 * rglru_fwd gives them. The stream must belong to the current device. Each
 * call made while the stream is not capturing looks up the current device's
 * copy of the static array (cudaGetSymbolAddress, with that device current),
 * so the address stays right after a device reset; a call made while the
 * stream is capturing uses the address found by the last such call, so make
 * a first call on each device before any stream capture. A problem whose
 * scratch would exceed RGLRU_NOALLOC_SCRATCH_BYTES is rejected with
 * RGLRU_ERR_WORKSPACE before anything is launched: the generic algorithm
 * needs 12 bytes per (batch row, time segment, channel) when it splits time
 * into segments (about 296 / (B * H) segments, each of at least 16 tokens),
 * and none when it does not. The forward shapes measured by this library need
 * well under 1 MiB (B=8 T=2048 D=1024 H=16: 0.29 MB; B=16 T=4096 D=2560
 * H=10: 0.98 MB; B=1 T=131072 D=4096 H=16: 0.93 MB). All calls on a device
 * share the one array, which keeps the last call's contents (nothing in it
 * needs to start at zero): calls that can overlap on the GPU, from different
 * streams or threads, race on it and must be serialised by the caller.
 */
int rglru_fwd_noalloc(const void *x, const void *conv_w, const void *W_a, const void *b_a,
                      const void *W_x, const void *b_x, const float *Lambda, const float *h0,
                      const void *conv_state_in, void *y, float *h_T, void *conv_state_out,
                      int B, int T, int D, int H, int io, void *stream);

/*
 * One decode step for B independent sequences, state updated in place: the
 * equations above for one t, from the fixed-size state (h and the last three
 * inputs) rather than the sequence ("Beyond Transformer Architecture: Griffin
 * and Google RecurrentGemma", "Key Strengths of RecurrentGemma", 1. Reduced
 * Memory Usage: the memory needed stays constant whatever the length).
 *   x_t        (B, D)     io     this step's input
 *   conv_state (B, 3, D)  io     ring at step pos (read); slot pos%3 is overwritten with x_t
 *   pos        >= 0              step index that places the ring (see above)
 *   h          (B, D)     float  state h_{t-1} (read), h_t (written)
 *   y_t        (B, D)     io     output h_t (written); must not alias x_t
 *   conv_w, W_a, b_a, W_x, b_x, Lambda as in rglru_fwd.
 * Requirements: B >= 1; D % H == 0; D % 8 == 0; bw <= 1024.
 */
int rglru_decode_step(const void *x_t, void *conv_state, int pos, float *h, void *y_t,
                      const void *conv_w, const void *W_a, const void *b_a, const void *W_x,
                      const void *b_x, const float *Lambda, int B, int D, int H, int io,
                      void *stream);

/*
 * Number of kernel launches one rglru_decode_step_algo call with these
 * arguments issues on its stream (0 on invalid or unsupported arguments).
 */
int rglru_decode_launches(int B, int D, int H, int io, int algo);

/* rglru_decode_step with an explicit algorithm (same rules as rglru_fwd_algo). */
int rglru_decode_step_algo(const void *x_t, void *conv_state, int pos, float *h, void *y_t,
                           const void *conv_w, const void *W_a, const void *b_a,
                           const void *W_x, const void *b_x, const float *Lambda, int B,
                           int D, int H, int io, void *stream, int algo);

/*
 * Backward of the layer (the gradient of a scalar loss through one forward
 * call), the training side of the layer whose kernel S. De's thread reports a
 * 3x training speed-up for. The backward is the chain rule through the
 * equations above: with
 * dy = dL/dy (B, T, D) and dh_T = dL/dh_T (B, D, or NULL for zeros) it returns
 * the gradients of L with respect to every forward input, recomputing the
 * forward from its inputs (nothing is saved between the calls). Time is cut
 * into segments of at most 512 tokens whose carries run in both time
 * directions, so the result does not depend on the batch or sequence size
 * beyond fp32 rounding.
 *
 * Inputs (as for rglru_fwd, same dtypes, layouts and alignment): x, conv_w,
 * W_a, b_a, W_x, b_x, Lambda, h0 (or NULL), conv_state_in (or NULL), and dy
 * (B, T, D) in the I/O dtype, dh_T fp32 (B, D) or NULL.
 * Outputs (device memory, caller-owned, not aliasing any input):
 *   dx              (B, T, D), the I/O dtype
 *   dconv_w         (4, D) fp32
 *   dW_a, dW_x      (H, bw, bw) fp32
 *   db_a, db_x      (D) fp32
 *   dLambda         (D) fp32
 *   dh0             (B, D) fp32, or NULL (not computed)
 *   dconv_state_in  (B, 3, D) fp32 (gradient with respect to the chronological
 *                   conv history, zeros if conv_state_in is NULL), or NULL
 * The library zeroes and accumulates the fp32 parameter gradients itself
 * (the call overwrites them; it does not add to their contents).
 * workspace: device memory of rglru_bwd_workspace_bytes(B, T, D, H, io) bytes,
 * 16-byte aligned, not shared with a concurrent call.
 * Arithmetic is fp32, except that for bf16 I/O with heads 32, 64 or 128 wide
 * and B * T >= 8 the gate contractions z = u W and d z W^T (and U^T dZ for
 * heads 64 or 128 wide) run on the tensor cores with bf16 operands and fp32
 * accumulation (below 8 tokens over all rows the operands stay fp32); any
 * head width up to 1024 that divides D. Returns RGLRU_OK, INVALID_ARG (shapes, NULL required
 * pointers, alignment, overlaps), WORKSPACE or CUDA. Nothing in the backward
 * waits on another block, so it has no device-side status.
 */
size_t rglru_bwd_workspace_bytes(int B, int T, int D, int H, int io);

int rglru_bwd(const void *x, const void *conv_w, const void *W_a, const void *b_a,
              const void *W_x, const void *b_x, const float *Lambda, const float *h0,
              const void *conv_state_in, const void *dy, const float *dh_T, void *dx,
              float *dconv_w, float *dW_a, float *db_a, float *dW_x, float *db_x,
              float *dLambda, float *dh0, float *dconv_state_in, int B, int T, int D, int H,
              int io, void *workspace, size_t workspace_bytes, void *stream);

/* Number of kernel launches of one rglru_bwd call (0 on invalid arguments). */
int rglru_bwd_launches(int B, int T, int D, int H, int io);

/*
 * Recurrent block around the layer (S. De's thread: a simple recurrent block
 * with a temporal Conv1D and the RG-LRU, and gated MLP blocks; "Beyond
 * Transformer Architecture: Griffin and Google RecurrentGemma", "Core
 * Components of Griffin", 3. Architecture Design: the gated MLP is GeGLU-like).
 * The pages print no equation for it; it is read as two branches of the block
 * input x (B, T, Dm):
 *   g   = GeLU(x W_gate)              GeLU(v) = v (1 + erf(v / sqrt 2)) / 2
 *   y   = rglru_fwd(x W_in)           the layer above, with h0 / conv_state_in
 *   out = (y * g) W_out               (B, T, Dm)
 * Shapes (row-major, the I/O dtype): x (B, T, Dm), W_in and W_gate (Dm, D),
 * W_out (D, Dm), out (B, T, Dm); the layer's parameters, h0, conv_state_in,
 * h_T and conv_state_out as for rglru_fwd (the state and conv history are the
 * layer's, over D channels). Dm >= 8 and a multiple of 8.
 * bf16 I/O: the three projections run on the library's tcgen05 GEMM (bf16
 * operands, fp32 accumulation in TMEM; CTA pairs on 256 x 256 tiles when B*T,
 * D and Dm are multiples of 256), and GeLU and the product are fused into the
 * gate projection's epilogue (y * GeLU(x W_gate) is formed where x W_gate
 * leaves the accumulator and written over y; erf there is Abramowitz and
 * Stegun's formula 7.1.26, |error| <= 1.5e-7, below the bf16 rounding of the
 * result). fp32 I/O: the
 * projections run on cuBLAS with the pedantic fp32 compute type (no TF32),
 * and GeLU and the product are one memory-bound kernel of this library.
 * x W_in and y are kept in the I/O dtype in the workspace (and x W_gate for
 * fp32 I/O).
 * workspace: rglru_block_fwd_workspace_bytes(...) bytes of device memory,
 * 16-byte aligned. out must not overlap x. dev_status as for rglru_fwd.
 * Returns RGLRU_OK, INVALID_ARG, UNSUPPORTED, WORKSPACE or CUDA (including a
 * cuBLAS failure).
 */
size_t rglru_block_fwd_workspace_bytes(int B, int T, int Dm, int D, int H, int io);

int rglru_block_fwd(const void *x, const void *W_in, const void *W_gate, const void *W_out,
                    const void *conv_w, const void *W_a, const void *b_a, const void *W_x,
                    const void *b_x, const float *Lambda, const float *h0,
                    const void *conv_state_in, void *out, float *h_T, void *conv_state_out,
                    int B, int T, int Dm, int D, int H, int io, void *workspace,
                    size_t workspace_bytes, int *dev_status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* RGLRU_B200_H */
