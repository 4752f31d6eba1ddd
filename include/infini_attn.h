/*
 * infini_attn.h -- C ABI of the Infini-attention forward for NVIDIA B200 (sm_100a).
 *
 * The operation is the Infini-attention layer of "Leave No Context Behind:
 * Efficient Infinite Context Transformers with Infini-attention" (arXiv
 * 2404.07143), as laid out on the explainer page of that title
 * (paper-graph-ui.vercel.app), section 3 "Technical Approach":
 *
 *   per (batch b, head h), the sequence of L tokens is cut into S = ceil(L/N)
 *   segments of N tokens (the last one may be shorter; section 3, "Training
 *   infrastructure: segment chunking at each layer").  For segment s with
 *   rows Q, K, V:
 *     A_dot = softmax_causal(scale * Q K^T) V                       (Eq. 6)
 *     A_mem = sigma(Q) M_{s-1} / (sigma(Q) z_{s-1}),  sigma = ELU+1  (Eq. 7)
 *     A     = sigmoid(beta_h) A_mem + (1 - sigmoid(beta_h)) A_dot  (Eq. 10)
 *   then the memory is updated, linear rule (Eq. 8):
 *     M_s = M_{s-1} + sigma(K)^T V,          z_s = z_{s-1} + sum_t sigma(K_t)
 *   or delta rule (Eq. 9):
 *     M_s = M_{s-1} + sigma(K)^T (V - sigma(K) M_{s-1} / (sigma(K) z_{s-1})),
 *     z_s as in the linear rule.
 *
 * Conventions where the pages leave a step open:
 *   - scale defaults to 1/sqrt(dk);
 *   - a retrieval row whose denominator sigma(q) z is exactly 0 (empty
 *     memory, M_0 = 0 and z_0 = 0) is the zero row, for A_mem and for the
 *     delta rule's retrieval term alike;
 *   - ELU uses alpha = 1; the causal mask includes the diagonal; A_dot never
 *     looks across a segment boundary;
 *   - M and z are fp32 throughout; products run with fp32 accumulation.
 *
 * Layouts (row-major, element strides; "contiguous" = the default):
 *   q, k   [B, H, L, dk]   v, out [B, H, L, dv]    element type bf16, or fp32
 *                                                  when mode has INFINI_F32
 *   beta   [H]        fp32, shared by every batch row
 *   M      [B, H, dk, dv] fp32, z [B, H, dk] fp32: on entry M_0, z_0; on
 *          return M_S, z_S (updated in place)
 *
 * Ownership: every pointer is caller-owned DEVICE memory on the current
 * device.  q, k, v and beta are read only; M and z are read and written;
 * out is written and must not alias any input.  The library keeps no state
 * between calls apart from a per-device error word (see
 * infini_attn_device_status).  Temporary workspace is taken with
 * cudaMallocAsync on `stream` and released on `stream` before the call
 * returns, unless infini_attn_forward_ex is handed a caller workspace.
 *
 * Errors: every call returns INFINI_OK (0) or a negative INFINI_ERR_* code
 * after validating its arguments on the host; nothing is launched when
 * validation fails.  Work is asynchronous on `stream`: faults of the
 * launched kernels surface on the caller's next synchronisation, and a
 * bounded device-side wait that ran out is reported by
 * infini_attn_device_status.  No kernel traps.
 */
#ifndef INFINI_ATTN_H
#define INFINI_ATTN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define INFINI_API __attribute__((visibility("default")))
#else
#define INFINI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* update rule, low bits of `mode` */
#define INFINI_LINEAR 0x0 /* Eq. 8 */
#define INFINI_DELTA 0x1  /* Eq. 9 */
/* element type of q, k, v and out: bf16 unless this bit is set */
#define INFINI_F32 0x10
/* infini_attn_params.flags: run the CUDA-core (SIMT) kernels even where the
 * tensor-core kernels apply -- a second GPU implementation, for testing */
#define INFINI_FLAG_FORCE_SIMT 0x1
/* tensor-core attention schedule: pairs of query tiles per CTA (the default
 * for grids that fill the GPU), one query tile per CTA with its key tiles
 * split between the CTA's two softmax warpgroups (the default for grids that
 * would otherwise leave SMs idle, e.g. one segment), or one query tile per
 * CTA on one warpgroup; these force one of them, for testing */
#define INFINI_FLAG_ATTN_SINGLE 0x2
#define INFINI_FLAG_ATTN_PAIRS 0x4
#define INFINI_FLAG_ATTN_SPLIT 0x8

enum {
  INFINI_OK = 0,
  INFINI_ERR_INVALID_ARG = -1, /* null pointer, size <= 0, n > N, aliasing */
  INFINI_ERR_UNSUPPORTED = -2, /* head size, mode bits, stride or alignment not handled */
  INFINI_ERR_WORKSPACE = -3,   /* workspace too small, or cudaMallocAsync failed */
  INFINI_ERR_LAUNCH = -4,      /* a CUDA launch or runtime call failed */
  INFINI_ERR_TIMEOUT = -5,     /* a bounded device-side wait ran out */
  INFINI_ERR_DEVICE = -6,      /* no CUDA device, or not sm_100 */
  INFINI_ERR_SCRATCH_LIMIT = -7 /* shape needs more than infini_attn_forward_noalloc's fixed scratch */
};

/*
 * Whole-sequence forward over L tokens in segments of N (Eq. 4 applied
 * S = ceil(L/N) times per (b, h)).  q, k, v, out contiguous [B, H, L, d].
 * mode = INFINI_LINEAR or INFINI_DELTA, optionally | INFINI_F32.
 * Supported: 1 <= dk, dv <= 128 (bf16 with dk = dv = 128 runs on the
 * tensor cores, everything else on CUDA cores); B, H, N >= 1; L >= 1.
 */
INFINI_API int infini_attn_forward(const void* q, const void* k, const void* v, const float* beta, float* M, float* z,
                        void* out, int B, int H, long L, int N, int dk, int dv, int mode, cudaStream_t stream);

/*
 * One streaming step (Eq. 4 once): every (b, h) consumes one segment of
 * n tokens, 1 <= n.  q, k, v, out contiguous [B, H, n, d].  Reads the live
 * M, z as M_{s-1}, z_{s-1} and leaves M_s, z_s in them.  S calls of this
 * function give the same result as one infini_attn_forward over S*n tokens
 * with N = n.
 */
INFINI_API int infini_attn_segment_step(const void* q, const void* k, const void* v, const float* beta, float* M, float* z,
                             void* out, int B, int H, int n, int dk, int dv, int mode, cudaStream_t stream);

/*
 * infini_attn_forward without any device allocation.  The paper has no
 * counterpart: this exists for callers that must not allocate device memory
 * while they run -- for example a serving loop that forbids allocation after
 * start-up, or code under a memory budget fixed in advance -- and so can
 * neither let the call take its workspace with cudaMallocAsync nor hand it a
 * buffer of their own.  Same arguments, layouts, results and errors as
 * infini_attn_forward; the workspace instead comes from one fixed 32 MiB
 * buffer in device memory that belongs to this library (every GPU that
 * loads the library holds it until the process exits).
 *   - Shapes whose workspace (infini_attn_workspace_size) exceeds 32 MiB are
 *     rejected with INFINI_ERR_SCRATCH_LIMIT before anything is launched.
 *   - The first call on a device looks up that device's address of the
 *     buffer (with the device current), and so does the first call after the
 *     device's context was reset; make that first call before any stream
 *     capture.  Nothing else is set up, and no call allocates.
 *   - All calls on a device share the one buffer and it keeps the previous
 *     call's contents; nothing in it has to start at zero, since a call reads
 *     only what it wrote earlier in the same call.  Calls whose work overlaps
 *     on the GPU (different streams without ordering between them) race on
 *     the buffer and give wrong results: order them on one stream.
 */
INFINI_API int infini_attn_forward_noalloc(const void* q, const void* k, const void* v, const float* beta, float* M,
                                           float* z, void* out, int B, int H, long L, int N, int dk, int dv,
                                           int mode, cudaStream_t stream);

/* Extended call: explicit scale, strides, workspace and flags. */
typedef struct infini_attn_params {
  const void* q;
  const void* k;
  const void* v;
  const float* beta;
  float* M;
  float* z;
  void* out;
  int B, H;
  long long L; /* tokens per (b, h) */
  int N;       /* segment length */
  int dk, dv;
  int mode;    /* INFINI_LINEAR | INFINI_DELTA, optionally | INFINI_F32 */
  float scale; /* softmax scale; 0 selects 1/sqrt(dk) */
  /* element strides of the (B, H, L) dimensions of q, k, v, out; the last
   * dimension is always contiguous.  All zero selects the contiguous
   * [B, H, L, d] layout.  A layout such as [B, L, H, d] is
   * {L*H*d, d, H*d}.  Tensor-core kernels need every stride times the
   * element size to be a multiple of 16 bytes and 16-byte aligned bases. */
  long long q_stride[3], k_stride[3], v_stride[3], o_stride[3];
  /* caller workspace of at least infini_attn_workspace_size(...) bytes,
   * 256-byte aligned; NULL lets the call allocate and free its own on
   * `stream` (cudaMallocAsync / cudaFreeAsync). */
  void* workspace;
  size_t workspace_bytes;
  int flags; /* INFINI_FLAG_* */
  cudaStream_t stream;
  /* Rotary position embeddings on the local attention only (section 4.1 of
   * the paper, quoted on the explainer page: position embeddings act on the
   * Q, K of the dot-product attention and not on the compressive memory's).
   * rope_base > 0 turns them on: A_dot (Eq. 6) is computed from rotated
   * Q, K, where the pair (x_2i, x_2i+1) of a row at position p is rotated by
   * the angle p * rope_base^(-2i/dk), and p = rope_offset + t for token t of
   * the call (0 <= t < L).  sigma(Q) of the memory read (Eq. 7) and the
   * update (Eq. 8 / 9) use the un-rotated q, k.  dk must be even.  The
   * rotated copies of q and k live in the workspace
   * (infini_attn_workspace_size_ex).  rope_base = 0: no position embedding. */
  double rope_base;
  long long rope_offset;
} infini_attn_params;

INFINI_API int infini_attn_forward_ex(const infini_attn_params* p);

/* Bytes of workspace a forward of this shape needs (0 if the shape is invalid). */
INFINI_API size_t infini_attn_workspace_size(int B, int H, long L, int N, int dk, int dv, int mode);

/* Bytes of workspace infini_attn_forward_ex(p) needs (0 if p is invalid):
 * infini_attn_workspace_size of the shape, plus the rotated q and k when
 * p->rope_base > 0.  Only the shape, mode and rope_base fields are read. */
INFINI_API size_t infini_attn_workspace_size_ex(const infini_attn_params* p);

/*
 * Token-level streaming decode (the "fast streaming inference" of the
 * abstract, taken one token at a time): every (b, h) appends one token at
 * position pos (0 <= pos < N, the same for all (b, h)) of its current
 * segment of N tokens.  The call
 *   1. writes k_t, v_t into row pos of the caller-owned caches,
 *   2. computes the token's output: causal softmax attention over the
 *      segment's keys 0..pos (Eq. 6 for one query row), the memory read with
 *      the live M, z = M_{s-1}, z_{s-1} (Eq. 7, 0 when the denominator is 0)
 *      and the gate (Eq. 10), into out,
 *   3. when pos == N - 1 or fold != 0, folds the segment's pos + 1 keys and
 *      values into M, z with the linear (Eq. 8) or delta (Eq. 9) rule.
 * Feeding a sequence token by token with pos = t mod N, and fold on its last
 * token, gives the outputs and final state of infini_attn_forward.
 *   q_t, k_t, out: [B, H, dk] / [B, H, dv]; v_t [B, H, dv]; contiguous, bf16 or
 *   fp32 (mode | INFINI_F32); k_cache [B, H, N, dk], v_cache [B, H, N, dv] in
 *   the same type, contiguous, caller-owned, rows > pos not read.
 * Steps 1 and 2 are one launch with the keys split over enough CTAs to fill
 * the GPU, plus a merge launch (a small scratch buffer of partial softmax
 * states is taken and released on `stream`); the fold runs the forward's
 * memory-update kernels alone on the cached segment.  Errors as
 * infini_attn_forward; pos outside [0, N) is INFINI_ERR_INVALID_ARG.
 */
INFINI_API int infini_attn_decode_step(const void* q_t, const void* k_t, const void* v_t, void* k_cache,
                                       void* v_cache, const float* beta, float* M, float* z, void* out, int B,
                                       int H, int N, int pos, int dk, int dv, int mode, int fold,
                                       cudaStream_t stream);

/*
 * Full multi-head layer around the Infini-attention step (multi-head
 * formulation, Eq. 5 and Eq. 11 of "Leave No Context Behind"):
 * Q = X W_Q, K = X W_K, V = X W_V per head, the forward of
 * infini_attn_forward on them, and Y = [A_1 ... A_H] W_O.  bf16 only,
 * head size 128 (dk = dv = 128, tensor-core path), d_model = D >= 1.
 *   x      [B, L, D] bf16, contiguous
 *   w_qkv  [D, 3*H*128] bf16, row-major: columns [0, H*128) give Q (head h
 *          in columns h*128 .. h*128 + 127), then K, then V
 *   w_o    [H*128, D] bf16, row-major (row h*128 + j multiplies value
 *          column j of head h)
 *   y      [B, L, D] bf16, written
 *   beta, M, z, N, mode as in infini_attn_forward (mode without INFINI_F32).
 * The projections run on this library's tensor-core GEMM
 * (infini_attn_gemm_bf16: bf16 operands, fp32 accumulation, bf16 results);
 * Q, K, V and the attention output are stored in bf16 between the steps, in
 * a workspace of infini_attn_layer_workspace_size(...) bytes (256-byte
 * aligned) that the call allocates and frees on `stream` when `workspace` is
 * NULL.  d_model must be a multiple of 8 and x, w_qkv, w_o, y 16-byte
 * aligned (rows of the GEMM operands are loaded by TMA), else
 * INFINI_ERR_UNSUPPORTED.  Errors otherwise as infini_attn_forward.
 */
INFINI_API int infini_attn_layer_forward(const void* x, const void* w_qkv, const void* w_o, const float* beta,
                                         float* M, float* z, void* y, int B, int H, long L, int N, int d_model,
                                         int mode, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Bytes of workspace infini_attn_layer_forward needs (0 if the shape is invalid). */
INFINI_API size_t infini_attn_layer_workspace_size(int B, int H, long L, int N, int d_model, int mode);

/*
 * The projection product of the full layer (Eq. 5, Q K V = X W; Eq. 11,
 * Y = [A_1 ... A_H] W_O) on its own: C[M, N] = A[M, K] B[K, N] for row-major
 * contiguous bf16 matrices, fp32 accumulation, C rounded to bf16 (nearest
 * even).  A tcgen05 kernel: 128 x 256 output tiles over a persistent grid,
 * operands staged by TMA, accumulators in tensor memory.  N and K must be
 * multiples of 8 and the pointers 16-byte aligned (INFINI_ERR_UNSUPPORTED
 * otherwise); C must not overlap A or B.  Device pointers, asynchronous on
 * `stream`; no workspace.
 */
INFINI_API int infini_attn_gemm_bf16(const void* A, const void* B, void* C, long M, int N, int K,
                                     cudaStream_t stream);

/*
 * Backward pass: gradients of a scalar loss through infini_attn_forward, by
 * back-propagation through time over the compressive memory (explainer page
 * "Leave No Context Behind", section 3, "Training infrastructure"; the chain
 * rule through Eq. 6-10 segment by segment in reverse, the forward's
 * conventions kept: zero retrieval rows where a denominator is 0, sigma'(x) =
 * 1 above zero and e^x at or below).  Given dLoss/d out and, optionally,
 * dLoss/d M_S and dLoss/d z_S, returns dLoss/d q, k, v, beta and, optionally,
 * dLoss/d M_0 and dLoss/d z_0.  The forward quantities it needs (the memory
 * entering every segment, the local attention's output and row
 * log-sum-exp) are recomputed from q, k, v, beta, M_0, z_0 inside the call.
 *
 * Layouts: q, k, dq, dk [B, H, L, dk]; v, d_out, dv [B, H, L, dv], all
 * contiguous, bf16 or fp32 (mode | INFINI_F32, one type for all); beta,
 * dbeta [H] fp32 (dbeta sums over the batch); M0, dM_S, dM0 [B, H, dk, dv]
 * and z0, dz_S, dz0 [B, H, dk] fp32.  M0 / z0 NULL: the empty memory;
 * dM_S / dz_S NULL: zero; dM0 / dz0 NULL: not returned.  Every pointer is
 * caller-owned device memory; the inputs are read only, the outputs written.
 * bf16 with dk = dv = 128 (16-byte aligned tensors): the local attention's
 * gradients run on the tensor cores (tcgen05; P and dS rounded to bf16 as
 * operands, fp32 accumulation), everything else in fp32 on CUDA cores;
 * other shapes, fp32 tensors and INFINI_FLAG_FORCE_SIMT: all in fp32 on CUDA
 * cores.  No position embeddings.  Workspace as for the forward: taken on
 * `stream` unless given (infini_attn_backward_workspace_size bytes, 256-byte
 * aligned).  Errors as infini_attn_forward.
 */
typedef struct infini_attn_bwd_params {
  const void* q;
  const void* k;
  const void* v;
  const float* beta;
  const float* M0;
  const float* z0;
  const void* d_out;
  const float* dM_S;
  const float* dz_S;
  void* dq;
  void* dk;
  void* dv;
  float* dbeta;
  float* dM0;
  float* dz0;
  int B, H;
  long long L;
  int N;
  int d_k, d_v;
  int mode;    /* INFINI_LINEAR | INFINI_DELTA, optionally | INFINI_F32 */
  float scale; /* softmax scale; 0 selects 1/sqrt(dk) */
  void* workspace;
  size_t workspace_bytes;
  cudaStream_t stream;
  int flags; /* INFINI_FLAG_FORCE_SIMT: CUDA-core kernels even where the tensor-core ones apply */
} infini_attn_bwd_params;

INFINI_API int infini_attn_backward(const infini_attn_bwd_params* p);

/* Bytes of workspace infini_attn_backward needs for p's shape and mode (0 if invalid). */
INFINI_API size_t infini_attn_backward_workspace_size(const infini_attn_bwd_params* p);

/*
 * Workspace that the library allocates itself (calls given no workspace)
 * comes from a stream-ordered pool of its own, one per CUDA context, that
 * keeps freed blocks for the next call.  This returns the pool's unused
 * device memory (of the current context) to the driver; blocks still in use
 * by queued work stay.  INFINI_OK, or INFINI_ERR_DEVICE if the trim failed.
 */
INFINI_API int infini_attn_trim_workspace(void);

/* Static English text for a return code; never NULL. */
INFINI_API const char* infini_attn_error_string(int code);

/*
 * Synchronises the current device and returns INFINI_ERR_TIMEOUT if any
 * kernel of this library gave up a bounded wait since the last reset,
 * else INFINI_OK (or INFINI_ERR_LAUNCH if the synchronisation failed).
 * reset != 0 clears the error word.
 */
INFINI_API int infini_attn_device_status(int reset);

/*
 * Self-test of the bounded-wait machinery: launches one block that waits on
 * an mbarrier nothing will ever complete, with a limit of `limit_us`
 * microseconds (1 .. 1000000).  The kernel must give up, record
 * INFINI_ERR_TIMEOUT in the error word and return; the call synchronises
 * and returns what infini_attn_device_status(0) then reports.
 */
INFINI_API int infini_attn_selftest_timeout(unsigned limit_us, cudaStream_t stream);

/*
 * Kernel timing for benchmarks.  phase_mask selects phases (bit 0 = memory
 * update kernels, bit 1 = state/snapshot kernels, bit 2 = attention
 * kernel, bit 3 = position-embedding pre-pass, bit 4 = projection GEMMs of
 * the full layer, bit 5 = backward kernels on CUDA cores, bit 6 = the
 * local attention's backward kernels on the tensor cores, bit 7 = the
 * memory branch's backward kernels on the tensor cores); while a bit is set, every
 * launch of that phase is bracketed by two CUDA events recorded on the
 * launch's stream.  0 turns timing off.
 */
INFINI_API int infini_attn_profile_enable(int phase_mask);
/*
 * Synchronises the recorded events and adds, per phase p in 0..7, the
 * elapsed milliseconds to ms[p] and the number of timed launches to
 * launches[p], for everything recorded since the last reset; reset != 0
 * then drops the records.  Either array may be NULL.
 */
INFINI_API int infini_attn_profile_read(double* ms, long long* launches, int reset);
/* Number of kernels this library has launched in this process (all phases). */
INFINI_API long long infini_attn_launch_count(void);
/*
 * The cudaError_t value behind the most recent INFINI_ERR_LAUNCH returned by
 * any call of this library in this process (0 if there was none), for
 * diagnostics; its name (cudaGetErrorName) is copied into name[0..n-1],
 * NUL-terminated, when name != NULL and n > 0.
 */
INFINI_API int infini_attn_last_cuda_error(char* name, int n);

/* sizeof(infini_attn_params), for bindings that build the struct themselves. */
INFINI_API size_t infini_attn_params_size(void);

/* Which kernels the given arguments would run: 1 tensor-core, 0 CUDA-core, <0 error code. */
INFINI_API int infini_attn_path(int dk, int dv, int mode, int flags);

#ifdef __cplusplus
}
#endif

#endif /* INFINI_ATTN_H */
