/*
 * tpblock — the Megatron tensor-parallel Transformer sublayer on one B200.
 *
 *   MLP sublayer:        Y = LN( X + sum_i Act(X A_i) B_i )
 *   attention sublayer:  Y = LN( X + sum_s O_s Wo_s ),
 *                        O_s = concat_{h in shard s} softmax(Q_h K_h^T / sqrt d) V_h
 *
 * The t tensor-parallel shards are logical partitions held in one GPU's HBM:
 * the column split's concatenation is a memory layout and the row split's
 * reduction happens in the tensor-core accumulator or in the fused
 * reduce + residual + LayerNorm kernel.  No second device, no collective.
 *
 * Pages that define the operations (cited by title and section):
 *   [TYPC] "张量并行：千亿大模型突破单卡显存限制的底层技术" (typc.net)
 *   [0539] "1. 张量并行：Tensor Parallelism" (0539edu.com news 288531)
 *   [PWWT] "TP到底在切什么——从一次矩阵乘法说起" (pwwt.cn news 5934571)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  Layout     Row-major everywhere.  Weights use the pages' [in, out] layout
 *             (Y = X W with X [seq, H], W [H, N]; [PWWT] §1.1); the `_ex`
 *             entry points also take nn.Linear's [out, in] (TP_W_OUT_IN).
 *  Shards     Each shard is its own contiguous device buffer, as the pages'
 *             weight chunking makes one ([PWWT] §3.1).  `*_shards` arguments
 *             are HOST arrays of t DEVICE pointers.  1 <= t <= TP_MAX_SHARDS.
 *  Ownership  Every pointer is owned by the caller.  The library allocates
 *             no device memory: scratch comes from the caller's `workspace`,
 *             sized by the matching *_workspace_bytes() query.
 *  Alignment  Every device pointer must be 16-byte aligned.
 *  Ordering   Work is enqueued on `stream` (a cudaStream_t; NULL = legacy
 *             default stream).  No call synchronises; results are valid once
 *             the caller has synchronised the stream.
 *  Graphs     Calls may be captured into a CUDA graph (they allocate nothing
 *             and never synchronise; make one uncaptured call per device
 *             first) and the graph replayed, on the default schedules.  The
 *             forced stream-K schedule (tp_set_gemm_stream_k(1 or 2)) is not
 *             replay-safe: its flags carry an epoch taken on the host at each
 *             call, which a replay repeats; so is tp_peer_barrier, whose
 *             epoch is an argument.  The attention key split clears its flags
 *             after use, so it is replay-safe.
 *  Errors     Arguments are checked before anything is launched; a failed
 *             check returns its status and enqueues nothing.  A CUDA launch
 *             error returns TP_ERR_CUDA.  Every device-side wait is bounded:
 *             if one gives up, the kernel returns early and tp_device_error()
 *             reports TP_ERR_TIMEOUT after the stream is synchronised.  No C++
 *             exception crosses this interface.
 *  Types      dtype TP_DTYPE_BF16: bf16 storage, f32 accumulation on the
 *             tensor cores (tcgen05).  dtype TP_DTYPE_F32: f32 storage and
 *             f32 CUDA-core arithmetic.  gamma/beta are always f32 (NULL means
 *             gamma = 1, beta = 0).
 */
#ifndef TPBLOCK_H_
#define TPBLOCK_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TP_MAX_SHARDS 8
#define TP_API_VERSION 1

typedef enum {
  TP_OK = 0,
  TP_ERR_INVALID_ARG = 1,        /* null pointer, t out of range, bad enum, misaligned pointer */
  TP_ERR_UNSUPPORTED_SHAPE = 2,  /* shape outside the supported set (see each entry point) */
  TP_ERR_WORKSPACE_TOO_SMALL = 3,
  TP_ERR_CUDA = 4,               /* a CUDA runtime/driver call failed */
  TP_ERR_TIMEOUT = 5,            /* a bounded device-side wait gave up (tp_device_error) */
  TP_ERR_NO_DEVICE = 6           /* no sm_100 device current */
} tp_status;

typedef enum { TP_DTYPE_F32 = 0, TP_DTYPE_BF16 = 1 } tp_dtype;

/* Elementwise activation between the two MLP products ([0539] §1.2.1: "ReLU 或
 * GeLU").  GELU_TANH: 0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3)));
 * GELU_ERF: 0.5 u (1 + erf(u / sqrt 2)); RELU: max(u, 0). */
typedef enum { TP_ACT_NONE = 0, TP_ACT_GELU_TANH = 1, TP_ACT_GELU_ERF = 2, TP_ACT_RELU = 3 } tp_act;

/* Weight layouts.  TP_W_IN_OUT: the pages' [in, out] (Y = X W, [PWWT] §1.1),
 * the layout every entry point without `_ex` takes.  TP_W_OUT_IN: nn.Linear's
 * [out, in] (`x @ W.T`, [PWWT] §3.2-§3.3): each shard is the transpose of the
 * [in, out] shard, read K-major by the tensor cores (no transpose pass). */
#define TP_W_IN_OUT 0
#define TP_W_OUT_IN 1

/* Library version (TP_API_VERSION) and a static string for a status code. */
int tp_version(void);
const char* tp_status_string(int status);

/* Reads and clears the device-side error word of the current device (0 when no
 * bounded wait gave up).  Call after synchronising the streams that ran the
 * library's kernels.  Returns TP_OK or TP_ERR_TIMEOUT (or TP_ERR_CUDA).  While
 * the word is set, the library's kernels give up any wait that does not
 * complete at once (their outputs are then unspecified), so a failure is not
 * silently followed by more work: read the word to re-arm the library. */
int tp_device_error(void);

/* ------------------------------------------------------------------ MLP ----
 * Y = LN(X + sum_i Act(X A_i) B_i), post-LN, no biases, no dropout.
 * [0539] §1.2.1 eqs (1.2)-(1.5) (Act(X A) B with A column-split and B
 * row-split, one reduction); [TYPC] §3 (MLP: column split then row split);
 * [PWWT] §2.3 (the reduction fused with the residual add and the next
 * LayerNorm's statistics).
 *
 *   S, H, F   sequence rows, hidden size, FFN size; F % t == 0.
 *   X         [S, H] dtype.
 *   A_shards  t pointers, A_i = columns [i F/t, (i+1) F/t) of A [H, F]: [H, F/t].
 *   B_shards  t pointers, B_i = rows    [i F/t, (i+1) F/t) of B [F, H]: [F/t, H].
 *   gamma, beta  [H] f32 or NULL.  eps > 0.
 *   Y         [S, H] out_dtype (bf16 or f32 for dtype bf16; f32 for dtype f32).
 *   workspace caller-owned device scratch of >= tp_mlp_workspace_bytes():
 *             the [S, F] activation buffer plus (bf16) up to 4 f32 [S, H]
 *             partial-sum slots; its contents on return are unspecified.
 * Supported: S >= 1; H % 8 == 0 and 8 <= H <= 16384; (F/t) % 8 == 0.
 * Kernels (bf16): column-split GEMM with the activation in its epilogue
 * (writes Act(X A_i) into its column slice of a [S, F] bf16 buffer), row-split
 * GEMM summing every shard in the TMEM accumulator ([S, H] f32; its K loop
 * is cut into up to 4 ranges with one f32 partial slot each when that fills
 * the GPU's last wave better), then the reduce + residual + LayerNorm kernel
 * that adds the slots. */
size_t tp_mlp_workspace_bytes(int S, int H, int F, int t, int dtype);
int tp_mlp_forward(int S, int H, int F, int t, int dtype, int out_dtype,
                   const void* X, const void* const* A_shards, const void* const* B_shards,
                   const float* gamma, const float* beta, float eps, int act,
                   void* Y, void* workspace, size_t workspace_bytes, void* stream);

/* tp_mlp_forward with a weight layout: for TP_W_OUT_IN, A_shards[i] is
 * [F/t, H] (rows i F/t .. of the [F, H] expansion weight) and B_shards[i] is
 * [H, F/t] (columns i F/t .. of the [H, F] compression weight). */
int tp_mlp_forward_ex(int S, int H, int F, int t, int dtype, int out_dtype, int w_layout,
                      const void* X, const void* const* A_shards, const void* const* B_shards,
                      const float* gamma, const float* beta, float eps, int act,
                      void* Y, void* workspace, size_t workspace_bytes, void* stream);

/* -------------------------------------------------- MLP training step ----
 * Backward pass of the MLP sublayer (post-LN, [in, out] weights, bf16).  The
 * pages give no backward formulas, only that each shard computes the gradient
 * of its own weight block ([PWWT] §4) and that the two split directions differ
 * in backward ([TYPC] §2.2); what is computed is the chain rule through
 *   U = X A, G = Act(U), V = G B, Z = X + V, Y = LN(Z):
 *   dZ = LayerNorm backward of dY;  dU_i = (dZ B_i^T) * Act'(U_i);
 *   dX = dZ + sum_i dU_i A_i^T;  dA_i = X^T dU_i;  dB_i = G_i^T dZ;
 *   dgamma = sum_rows dY * (Z - mean) / sqrt(var + eps);  dbeta = sum_rows dY.
 *
 * tp_mlp_forward_train: tp_mlp_forward (dtype bf16 only) that also keeps, in
 * the caller's `state` (>= tp_mlp_train_state_bytes()), what the backward
 * reads: U [S, F] bf16 (pre-activation), G [S, F] bf16, V [S, H] f32 and the
 * LayerNorm's row statistics ([S][2] f32: each row's mean and
 * 1/sqrt(var + eps), so the backward normalises with the forward's values).
 * Y is the same as tp_mlp_forward's up to rounding.
 *
 * tp_mlp_backward: from the same X, shards, gamma, eps, act and the state of
 * one tp_mlp_forward_train call, and the upstream gradient dY [S, H] bf16,
 * writes dX [S, H] bf16, dA_shards[i] [H, F/t] f32 and dB_shards[i] [F/t, H]
 * f32 (the gradients of shard i's weights, same layout as the weights),
 * dgamma and dbeta [H] f32 (either may be NULL).  workspace >=
 * tp_mlp_backward_workspace_bytes().  S == 0 writes nothing.  Shapes as
 * tp_mlp_forward. */
size_t tp_mlp_train_state_bytes(int S, int H, int F, int t, int dtype);
int tp_mlp_forward_train(int S, int H, int F, int t, int dtype, int out_dtype, const void* X,
                         const void* const* A_shards, const void* const* B_shards,
                         const float* gamma, const float* beta, float eps, int act,
                         void* Y, void* state, size_t state_bytes, void* stream);
size_t tp_mlp_backward_workspace_bytes(int S, int H, int F, int t, int dtype);
int tp_mlp_backward(int S, int H, int F, int t, int dtype, const void* X,
                    const void* const* A_shards, const void* const* B_shards,
                    const float* gamma, float eps, int act, const void* state, size_t state_bytes,
                    const void* dY, void* dX, void* const* dA_shards, void* const* dB_shards,
                    float* dgamma, float* dbeta, void* workspace, size_t workspace_bytes, void* stream);
/* The same with a weight layout.  For TP_W_OUT_IN the weight shards are
 * [out, in] (A_shards[i] [F/t, H], B_shards[i] [H, F/t]) and so are their
 * gradients (dA_shards[i] [F/t, H], dB_shards[i] [H, F/t]); the state of a
 * tp_mlp_forward_train_ex call with the same layout. */
int tp_mlp_forward_train_ex(int S, int H, int F, int t, int dtype, int out_dtype, int w_layout, const void* X,
                            const void* const* A_shards, const void* const* B_shards,
                            const float* gamma, const float* beta, float eps, int act,
                            void* Y, void* state, size_t state_bytes, void* stream);
int tp_mlp_backward_ex(int S, int H, int F, int t, int dtype, int w_layout, const void* X,
                       const void* const* A_shards, const void* const* B_shards,
                       const float* gamma, float eps, int act, const void* state, size_t state_bytes,
                       const void* dY, void* dX, void* const* dA_shards, void* const* dB_shards,
                       float* dgamma, float* dbeta, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------- MLP without allocation ----
 * The pages have no counterpart to this entry point: it exists for callers
 * that cannot allocate device memory (plugin hosts that forbid allocation in
 * their execute hook, latency-critical loops that cannot afford cudaMalloc's
 * implicit synchronisation, programs whose own allocator holds the device
 * memory).  Same arguments and result as tp_mlp_forward, minus the workspace:
 * the scratch is a fixed device array inside the library, of
 * tp_noalloc_scratch_bytes() bytes (32 MiB), held on every GPU that loads the
 * library until the process exits.
 *  - Arguments are checked first, exactly as tp_mlp_forward checks them
 *    (same statuses).  Then sizes whose tp_mlp_workspace_bytes() exceeds the
 *    maximum are rejected with TP_ERR_WORKSPACE_TOO_SMALL before anything is
 *    launched.
 *  - The call allocates nothing.  Its first call on a device whose arguments
 *    pass the checks looks up the array's device address (with that device
 *    current); an empty call (S == 0, X and Y may be NULL) is enough.  Make
 *    that first call before any stream capture.
 *  - Every call on a device shares the array: calls whose kernels may overlap
 *    on the GPU race on it; order them on one stream.  Nothing in it needs to
 *    start at zero. */
size_t tp_noalloc_scratch_bytes(void);
int tp_mlp_forward_noalloc(int S, int H, int F, int t, int dtype, int out_dtype,
                           const void* X, const void* const* A_shards, const void* const* B_shards,
                           const float* gamma, const float* beta, float eps, int act,
                           void* Y, void* stream);

/* ------------------------------------------------------------ attention ----
 * Y = LN(X + concat_h(softmax(Q_h K_h^T / sqrt d) V_h) Wo), non-causal, no
 * mask, heads split over t shards of nh/t heads.  [0539] §1.2.2 (every head
 * is independent; W_O row-split by head; one reduction); [TYPC] §3 (64 heads
 * on 4 shards, 16 per shard); [PWWT] §2.1-§2.2 (QKV column-split, O row-split).
 *
 *   Full weights: Wqkv = [W_Q | W_K | W_V], [H, 3H], head j in columns
 *   j d .. j d + d - 1 of each block; Wo [H, H], rows in the same head order.
 *   Wqkv_shards[s]: [H, 3 (nh/t) d] = [Q cols of shard s's heads | K cols | V cols].
 *   Wo_shards[s]:   [(nh/t) d, H] = rows s (nh/t) d .. of Wo.
 *   X [S, H] bf16; Y [S, H] out_dtype; gamma, beta [H] f32 or NULL.
 * Supported: dtype bf16; d == 128; H == nh * d; nh % t == 0; S % 128 == 0;
 * H <= 16384. */
size_t tp_attn_workspace_bytes(int S, int H, int nh, int d, int t, int dtype);
int tp_qkv_attn_oproj_forward(int S, int H, int nh, int d, int t, int dtype, int out_dtype,
                              const void* X, const void* const* Wqkv_shards, const void* const* Wo_shards,
                              const float* gamma, const float* beta, float eps,
                              void* Y, void* workspace, size_t workspace_bytes, void* stream);

/* tp_qkv_attn_oproj_forward with a weight layout: for TP_W_OUT_IN,
 * Wqkv_shards[s] is [3 (nh/t) d, H] and Wo_shards[s] is [H, (nh/t) d]. */
int tp_qkv_attn_oproj_forward_ex(int S, int H, int nh, int d, int t, int dtype, int out_dtype, int w_layout,
                                 const void* X, const void* const* Wqkv_shards, const void* const* Wo_shards,
                                 const float* gamma, const float* beta, float eps,
                                 void* Y, void* workspace, size_t workspace_bytes, void* stream);

/* -------------------------------------------- attention training step ----
 * Backward pass of the attention sublayer (post-LN, [in, out] weights, bf16),
 * the chain rule through QKV = X Wqkv, S_h = Q_h K_h^T / sqrt d,
 * P_h = softmax(S_h), O_h = P_h V_h, Z = X + O Wo, Y = LN(Z):
 *   dZ = LayerNorm backward of dY;  dO = dZ Wo^T;  dWo = O^T dZ;
 *   per head: dV_h = P_h^T dO_h, dS_h = P_h * (dO_h V_h^T - rowsum(dO_h * O_h)) / sqrt d,
 *             dQ_h = dS_h K_h, dK_h = dS_h^T Q_h;
 *   dX = dZ + dQKV Wqkv^T;  dWqkv = X^T dQKV.
 * Each shard's weight gradients stay with the shard ([PWWT] §4).
 *
 * tp_attn_forward_train: tp_qkv_attn_oproj_forward that also keeps, in the
 * caller's `state` (>= tp_attn_train_state_bytes()), QKV [S, 3H] bf16, O
 * [S, H] bf16, O Wo [S, H] f32, each row's log2 softmax denominator per
 * head [nh, S] f32 (P is rebuilt from it in the backward) and the
 * LayerNorm's row statistics ([S][2] f32, as tp_mlp_forward_train).
 *
 * tp_attn_backward: from the same X, shards, gamma, eps and the state of one
 * tp_attn_forward_train call, and dY [S, H] bf16, writes dX [S, H] bf16,
 * dWqkv_shards[s] [H, 3 (nh/t) d] and dWo_shards[s] [(nh/t) d, H] f32 (the
 * shards' layout), dgamma and dbeta [H] f32 (either may be NULL).
 * workspace >= tp_attn_backward_workspace_bytes(): dZ, dO, dQKV, the
 * f32 partial of dX, the row dots D and the LayerNorm backward's partial
 * rows.  The per-head products run in two fused kernels that keep the score,
 * P, dP and dS tiles on chip (TMEM), so no [S, S] matrix is held.  Shapes as
 * tp_qkv_attn_oproj_forward. */
size_t tp_attn_train_state_bytes(int S, int H, int nh, int d, int t, int dtype);
int tp_attn_forward_train(int S, int H, int nh, int d, int t, int dtype, int out_dtype, const void* X,
                          const void* const* Wqkv_shards, const void* const* Wo_shards,
                          const float* gamma, const float* beta, float eps,
                          void* Y, void* state, size_t state_bytes, void* stream);
size_t tp_attn_backward_workspace_bytes(int S, int H, int nh, int d, int t, int dtype);
int tp_attn_backward(int S, int H, int nh, int d, int t, int dtype, const void* X,
                     const void* const* Wqkv_shards, const void* const* Wo_shards,
                     const float* gamma, float eps, const void* state, size_t state_bytes,
                     const void* dY, void* dX, void* const* dWqkv_shards, void* const* dWo_shards,
                     float* dgamma, float* dbeta, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------- Transformer block ----
 * The attention sublayer followed by the MLP sublayer, the two TP pairs of one
 * Transformer block ([PWWT] §2.1 figure 3: QKV/O one pair, the two MLP
 * layers the other, two reductions per block).
 *   pre_ln = 0 (post-LN):  Y1 = LN1(X + Attn(X));  Y = LN2(Y1 + MLP(Y1))
 *   pre_ln = 1 (pre-LN, the order [PWWT] §2.1 lists):
 *                          Z1 = X + Attn(LN1(X)); Y = Z1 + MLP(LN2(Z1))
 * Attn and MLP are the sublayers above without their residual and LayerNorm;
 * the intermediate Y1 / Z1 / LN outputs are bf16.  Weights as in
 * tp_qkv_attn_oproj_forward and tp_mlp_forward; ln*_gamma/beta [H] f32 or
 * NULL.  dtype bf16; out_dtype bf16 or f32.  Shapes: the union of both
 * sublayers' limits (d == 128, H == nh d, nh % t == 0, S % 128 == 0,
 * (F/t) % 8 == 0, H <= 16384).  workspace >= tp_block_workspace_bytes(). */
size_t tp_block_workspace_bytes(int S, int H, int F, int nh, int d, int t, int dtype);
int tp_transformer_block_forward(int S, int H, int F, int nh, int d, int t, int dtype, int out_dtype, int pre_ln,
                                 const void* X, const void* const* Wqkv_shards, const void* const* Wo_shards,
                                 const void* const* A_shards, const void* const* B_shards,
                                 const float* ln1_gamma, const float* ln1_beta,
                                 const float* ln2_gamma, const float* ln2_beta, float eps, int act,
                                 void* Y, void* workspace, size_t workspace_bytes, void* stream);
/* The same with a weight layout (TP_W_OUT_IN: every shard [out, in], as in
 * tp_qkv_attn_oproj_forward_ex and tp_mlp_forward_ex). */
int tp_transformer_block_forward_ex(int S, int H, int F, int nh, int d, int t, int dtype, int out_dtype, int pre_ln,
                                    int w_layout, const void* X, const void* const* Wqkv_shards,
                                    const void* const* Wo_shards, const void* const* A_shards,
                                    const void* const* B_shards, const float* ln1_gamma, const float* ln1_beta,
                                    const float* ln2_gamma, const float* ln2_beta, float eps, int act, void* Y,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------ single linears ----
 * Column-split linear ([TYPC] §2.1; [PWWT] §1.1 figure 1; [0539] §1.1 列切分):
 *   Y[:, i N/t : (i+1) N/t] = Act(X W_i),  X [M, K], W_i [K, N/t]  (concat in place).
 * Row-split linear ([TYPC] §2.2; [PWWT] §1.2 figure 2; [0539] eq. (1.1)):
 *   Y = sum_i X[:, i K/t : (i+1) K/t] W_i,  X [M, K] (full), W_i [K/t, N].
 * Y is [M, N] out_dtype (bf16 or f32; f32 only for dtype f32).
 * Supported: M >= 1; K % 8 == 0, N % 8 == 0, (N/t) % 8 (column) or (K/t) % 8
 * (row) == 0.  The row-split linear accumulates every shard in the tensor-core
 * accumulator and needs no workspace (workspace may be NULL). */
int tp_linear_column_forward(int M, int K, int N, int t, int dtype, int out_dtype,
                             const void* X, const void* const* W_shards, int act,
                             void* Y, void* stream);
int tp_linear_row_forward(int M, int K, int N, int t, int dtype, int out_dtype,
                          const void* X, const void* const* W_shards,
                          void* Y, void* workspace, size_t workspace_bytes, void* stream);
/* The same with a weight layout: for TP_W_OUT_IN the column-split shard i is
 * [N/t, K] and the row-split shard i is [N, K/t]. */
int tp_linear_column_forward_ex(int M, int K, int N, int t, int dtype, int out_dtype, int w_layout,
                                const void* X, const void* const* W_shards, int act, void* Y, void* stream);
int tp_linear_row_forward_ex(int M, int K, int N, int t, int dtype, int out_dtype, int w_layout,
                             const void* X, const void* const* W_shards,
                             void* Y, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------- reduce + residual + LayerNorm ----
 * Y = LN(X + sum_{p < nparts} P_p) per row over H ([PWWT] §2.3, §5.3): mean,
 * then the biased variance (divide by H), eps inside the square root.
 *   parts  nparts f32 buffers [S, H] laid out back to back (may be NULL if
 *          nparts == 0).  X [S, H] x_dtype; Y [S, H] out_dtype.
 * Supported: H % 8 == 0, 8 <= H <= 16384. */
int tp_reduce_residual_layernorm(int S, int H, int nparts, const float* parts,
                                 const void* X, int x_dtype, const float* gamma, const float* beta,
                                 float eps, void* Y, int out_dtype, void* stream);

/* ------------------------------------ tensor parallelism across GPUs ----
 * The multi-GPU form of the sublayers: each rank (GPU) holds its own weight
 * shards, computes its partial sum of the row-split product, and the partial
 * sums of all ranks are reduced before the residual add and the LayerNorm
 * ([TYPC] §2.2 and §3; [PWWT] §3.3 RowParallelLinear's all_reduce, and §5.1:
 * an AllReduce is a ReduceScatter followed by an AllGather, and the
 * ReduceScatter's output can be used as it is, split by rows, which is what
 * sequence parallelism does).  The exchange itself is either a collective
 * library call made by the caller between these entry points, or the pointer
 * lists of tp_reduce_residual_layernorm_multi below, which read other GPUs'
 * partials and write other GPUs' outputs directly (peer access).
 *
 * tp_mlp_partial_forward: P = sum_{i < t} Act(X A_i) B_i over the t shards
 *   this rank holds (F = the FFN width they cover; A_i [H, F/t], B_i [F/t, H]),
 *   f32 [S, H], no residual and no LayerNorm.  dtype bf16 (tensor cores) or
 *   f32 (CUDA cores).  workspace >= tp_mlp_partial_workspace_bytes(): the
 *   [S, F] activation buffer.  Supported: H % 8 == 0, (F/t) % 8 == 0.
 * tp_attn_partial_forward: P = sum_{s < t} O_s Wo_s for the nh heads this
 *   rank holds (t shards of nh/t heads; X [S, H] with H the model's hidden
 *   size, nh d <= H; Wqkv_shards[s] [H, 3 (nh/t) d] = [Q | K | V] columns of
 *   shard s's heads; Wo_shards[s] [(nh/t) d, H]), f32 [S, H].  dtype bf16;
 *   d == 128; nh % t == 0; S % 128 == 0; H % 8 == 0.  workspace >=
 *   tp_attn_partial_workspace_bytes(): QKV [S, 3 nh d] and O [S, nh d] bf16.
 * tp_reduce_residual_layernorm_multi: for `rows` rows,
 *   Y = LN(X + sum_{q < nparts} parts[q]) (mean, biased variance, eps inside
 *   the square root, gamma/beta [H] f32 or NULL), written to every one of the
 *   nout outputs Y_outs[0..nout).  parts (nparts f32 buffers), X (x_dtype) and
 *   each Y_outs[o] (out_dtype) are host arrays of device pointers to the first
 *   of the `rows` rows, rows of H contiguous elements.  A pointer may address
 *   another GPU's memory that this device can reach (peer access, CUDA IPC):
 *   rank r then reduces its 1/N slice of the rows from every rank's partial
 *   and stores the normalised rows into every rank's output, the
 *   ReduceScatter -> LayerNorm on S/N rows -> AllGather of [PWWT] §5.1 in one
 *   kernel.  The caller orders it after the partials are complete on every
 *   rank and before the outputs are read.  0 <= nparts <= 8; 1 <= nout <= 8;
 *   H % 8 == 0, 8 <= H <= 16384. */
/* Peer access for the fused form, between the ranks' processes (CUDA IPC).
 * tp_ipc_export writes a TP_IPC_HANDLE_BYTES-byte handle (host memory) for a
 * device address of this process (the allocation containing it, and the
 * address's offset in it); tp_ipc_import maps that allocation in another
 * process on its current device and returns the same address's counterpart
 * there (peer access is enabled as needed); tp_ipc_close unmaps an address
 * tp_ipc_import returned.  TP_ERR_CUDA when the
 * runtime refuses (for example an import in the exporting process itself).
 * tp_peer_barrier: rank `rank` of `nranks` (<= 8) stores `epoch` into its
 * slot of every rank's flag array, then waits (bounded; TP_ERR_TIMEOUT
 * through tp_device_error() if it gives up) until its own array holds `epoch`
 * in every rank's slot.  flags[q] is rank q's array of nranks unsigned 64-bit
 * words (this device's own array at flags[rank], the peers' through
 * tp_ipc_import), zero when first used; every rank passes the same epoch,
 * which must grow from call to call.  Enqueued on `stream` between the
 * partial sums and tp_reduce_residual_layernorm_multi (every partial is
 * complete before any rank reads it), and after it (every rank's rows have
 * landed before any output is read). */
#define TP_IPC_HANDLE_BYTES 72
int tp_ipc_export(const void* dev_ptr, void* handle);
int tp_ipc_import(const void* handle, void** dev_ptr);
int tp_ipc_close(void* dev_ptr);
int tp_peer_barrier(int nranks, int rank, unsigned long long* const* flags, unsigned long long epoch, void* stream);

size_t tp_mlp_partial_workspace_bytes(int S, int H, int F, int t, int dtype);
int tp_mlp_partial_forward(int S, int H, int F, int t, int dtype, const void* X, const void* const* A_shards,
                           const void* const* B_shards, int act, float* P, void* workspace, size_t workspace_bytes,
                           void* stream);
size_t tp_attn_partial_workspace_bytes(int S, int H, int nh, int d, int t, int dtype);
int tp_attn_partial_forward(int S, int H, int nh, int d, int t, int dtype, const void* X,
                            const void* const* Wqkv_shards, const void* const* Wo_shards, float* P, void* workspace,
                            size_t workspace_bytes, void* stream);
int tp_reduce_residual_layernorm_multi(int rows, int H, int nparts, const float* const* parts, const void* X,
                                       int x_dtype, const float* gamma, const float* beta, float eps, int nout,
                                       void* const* Y_outs, int out_dtype, void* stream);

/* -------------------------------------------------------- GEMM tiling ----
 * Tuning override for the tensor-core GEMMs (every sublayer and linear here).
 * tile_n == 0 (the default): a cost model picks, per launch, 256-column tiles
 * (with an optional K split for f32 partial sums) or wide tiles of up to 512
 * columns (two MMAs per K step filling TMEM) where they give fuller waves on
 * the SM pairs, or 128-column tiles with an N = 128 MMA where a shard has at
 * most 128 columns and B is N-major.  tile_n in [256, 512], a multiple of 32:
 * every GEMM of at least 129 rows uses that tile width (rounded up to a
 * multiple of 64 for bf16 output) and no K split.  tile_n = 128: every GEMM
 * uses 128-column tiles (an N = 128 MMA where B is N-major) and no K split.
 * Results are the same to rounding either way.
 * Process-wide, not thread-safe against concurrent launches.  Returns
 * TP_ERR_INVALID_ARG for other values. */
int tp_set_gemm_tile_n(int tile_n);

/* The tile plan the next tensor-core GEMM launch of this shape would get (the
 * cost model above, or the tp_set_gemm_tile_n override): host logic only, no
 * device is touched.  M output rows; t shards, each shard_n columns of B
 * (column mode, row_mode = 0) or shard_k rows of K (row mode, the shards
 * summed); K = shard_k in column mode.  out_f32: f32 output (only then may the
 * K loop be split, into at most max_splits ranges).  b_kmajor: B stored
 * [n, k].  heavy_epilogue: the epilogue also stores the pre-activation or
 * reads a second operand (the training step's GEMMs).  slots: co-resident
 * CTA pairs (74 on a 148-SM B200), or SMs where M < 129 (single CTAs).
 * Writes *tile_n (128, 256 or a wide width up to 512) and *splits.  Returns
 * TP_ERR_INVALID_ARG for non-positive sizes, t outside [1, TP_MAX_SHARDS] or
 * NULL outputs. */
int tp_gemm_plan(int M, int t, int row_mode, int shard_k, int shard_n, int out_f32, int b_kmajor,
                 int heavy_epilogue, int slots, int max_splits, int* tile_n, int* splits);

/* Stream-K scheduling of the tensor-core GEMMs.  Where a sublayer has
 * scratch to spare for it (the partial-sum slots past the first of the MLP
 * and attention workspaces) and the epilogue is the plain one, a GEMM whose
 * tiles leave a partly filled last wave may keep its whole waves of tiles and
 * cut only the remainder tiles along K: each remainder tile's first k-blocks
 * run on the pair that finishes it, the tails of all remainder tiles are
 * spread over the pairs the last wave would leave idle.  The finishing pair
 * adds the tails' f32 partials after a bounded wait for their flags
 * (TP_ERR_TIMEOUT through tp_device_error() if it gives up), in a fixed
 * order, so results are run-to-run repeatable.
 * mode 0 (the default): whole tiles only (stream-K measured slower on B200
 * for the MLP sublayer's GEMMs); 1: every GEMM that has the scratch and a
 * partial last wave uses stream-K; 2: the tile cost model chooses per launch.
 * Process-wide, not thread-safe against concurrent launches.  Returns
 * TP_ERR_INVALID_ARG for other values. */
int tp_set_gemm_stream_k(int mode);

/* tp_gemm_plan with the stream-K option: sk_area_bytes of scratch available
 * to the launch (0: none).  Also writes *stream_k (1 if the launch would use
 * stream-K) and *sk_clusters (the CTA pairs, or single CTAs, it would run
 * on); either may be NULL. */
int tp_gemm_plan_sk(int M, int t, int row_mode, int shard_k, int shard_n, int out_f32, int b_kmajor,
                    int heavy_epilogue, int slots, int max_splits, size_t sk_area_bytes, int* tile_n, int* splits,
                    int* stream_k, int* sk_clusters);
/* tp_gemm_plan_sk for a GEMM whose A operand is read M-major (a_mnmajor = 1:
 * A stored [K, M], the weight-gradient GEMMs X^T dU, G^T dZ, O^T dZ and
 * X^T dQKV of the backward passes), for which the 256-column tiles cost
 * more per k-block than with a K-major A. */
int tp_gemm_plan_ex(int M, int t, int row_mode, int shard_k, int shard_n, int out_f32, int a_mnmajor, int b_kmajor,
                    int heavy_epilogue, int slots, int max_splits, size_t sk_area_bytes, int* tile_n, int* splits,
                    int* stream_k, int* sk_clusters);

/* Last-wave key split of the attention kernel (tp_qkv_attn_oproj_forward,
 * tp_attn_forward_train, tp_attn_partial_forward).  The attention kernel runs
 * one CTA per (head, 256 query rows) unit; U units on the GPU's SMs end with
 * a partial wave of U mod SMs units.  mode 1 (the default): when twice that
 * remainder fits in one wave, each of those last units runs as two CTAs over
 * the two halves of the keys, whose softmax-weighted partial sums the second
 * to finish merges with the first's (flash attention's combination of key
 * ranges; a bounded wait, TP_ERR_TIMEOUT through tp_device_error() if it
 * gives up); 0: never; 2: every unit is split (for tests).  The scratch is
 * the workspace's partial-sum area, which the O projection overwrites
 * afterwards.  Process-wide.  Returns TP_ERR_INVALID_ARG for other values. */
int tp_set_attn_kv_split(int mode);

/* The attention key-split plan for S query rows and nh heads on `slots`
 * resident CTAs (148 on a B200) under `mode` (as tp_set_attn_kv_split) with
 * scratch_bytes of scratch: writes *whole (units run over all keys), *split
 * (units run as two half-key CTAs) and *kv_half (128-key blocks of a split
 * unit's first half).  Host-only.  Returns TP_ERR_INVALID_ARG for S < 0,
 * nh < 1, slots < 1, a mode outside [0, 2] or NULL outputs. */
int tp_attn_split_plan(int S, int nh, int slots, int mode, size_t scratch_bytes, int* whole, int* split,
                       int* kv_half);

/* ------------------------------------------------------------ self-test ----
 * Diagnostic for the bounded-wait path every kernel here takes when one of its
 * device-side waits gives up: launches one CTA whose mbarrier wait nothing can
 * complete, so the wait ends after `limit_cycles` SM cycles (> 0), raises the
 * device error word and returns.  After the caller synchronises `stream`,
 * tp_device_error() returns TP_ERR_TIMEOUT (and clears the word); the context
 * stays usable.  Returns TP_ERR_INVALID_ARG for limit_cycles < 1. */
int tp_selftest_wait_timeout(long long limit_cycles, void* stream);
/* The same for the other kind of bounded wait the kernels make: one thread
 * waits for a flag in global memory that nothing sets (what a stream-K GEMM's
 * finishing CTA pair does for the pairs whose partial sums it adds), so the
 * wait ends after `limit_cycles` SM cycles and raises the device error word;
 * tp_device_error() then returns TP_ERR_TIMEOUT and clears it. */
int tp_selftest_flag_wait_timeout(long long limit_cycles, void* stream);

/* Diagnostic for the attention kernel's exponentials: part of the softmax's
 * 2^x terms are evaluated on the FMA pipe by a polynomial instead of the MUFU
 * unit.  Writes, for the n f32 inputs x (device), that evaluation into y_poly
 * and CUDA's exp2f(x) into y_exp2f (device, n each). */
int tp_selftest_exp2(const float* x, float* y_poly, float* y_exp2f, int n, void* stream);
/* The same with a choice of the polynomial: form 0 the degree-4 single-value
 * evaluation (as tp_selftest_exp2), form 1 the degree-3 evaluation of two
 * values at once with packed f32x2 arithmetic (inputs 2i and 2i + 1 share
 * one evaluation), which is the form the attention kernel's softmax uses.
 * Returns TP_ERR_INVALID_ARG for another form. */
int tp_selftest_exp2_form(const float* x, float* y_poly, float* y_exp2f, int n, int form, void* stream);

/* ----------------------------------------------------- kernel timing ----
 * When enabled, every kernel the library launches is counted, and the first
 * 16384 launches between two collects are bracketed by CUDA events recorded on
 * the launch's stream.  tp_profile_collect synchronises those events and
 * writes per kernel kind (0 tensor-core GEMM, 1 reduce+residual+LayerNorm,
 * 2 f32 CUDA-core GEMM, 3 attention, 4 LayerNorm backward, 5 the attention
 * backward's elementwise row-dot kernel, 6 the LayerNorm backward's sum of
 * the per-CTA dgamma/dbeta rows): `launches` = all launches, `timed` = the
 * launches with events, `ms` = their summed device milliseconds; then it
 * clears the record.  Any output array may be NULL.  Returns the number of
 * kinds written (<= max_kinds), or -TP_ERR_CUDA.  Not thread-safe: enable,
 * launch and collect from one host thread. */
int tp_profile_enable(int on);
int tp_profile_collect(int* launches, int* timed, double* ms, int max_kinds);
/* While profiling is enabled: on = 0 stops recording events for the
 * following launches (they are still counted), on = 1 resumes.  Events sit in
 * the stream between launches, so sampling a subset of launches leaves the
 * others running back to back (programmatic dependent launch).  Enabling
 * profiling resumes recording. */
int tp_profile_sample(int on);
const char* tp_kernel_kind_name(int kind);

#ifdef __cplusplus
}
#endif

#endif /* TPBLOCK_H_ */
