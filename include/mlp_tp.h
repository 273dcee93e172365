/*
 * mlp_tp.h — C-ABI of the B200 (sm_100a) tensor-parallel Transformer MLP block
 * with biases, all t shards on one GPU.
 *
 *   forward   Y = sum_{i<t} GeLU(X·A_i + a_i)·B_i + b
 *   backward  dX, dA, da, dB, db given dY
 *
 * The block is Megatron's Column->Row parallel MLP: the first linear layer's
 * weight A[h,f] is split by columns into A_i (ColumnParallelLinear, output not
 * gathered), the second layer's weight B[f,h] by rows into B_i
 * (RowParallelLinear, input already parallel), and the t partial outputs are
 * summed once ("Megatron-LM — 架构与原理", §4 巧妙之处, item "Column→Row 配对让
 * MLP 只做一次通信"; "Megatron-LM（英伟达超大模型训练框架）完整介绍", §二.2 MLP层).
 * The all-reduce of the forward ("reduce" operator) and of the backward
 * ("copy" operator's backward, same §4, item "通信原语的「前向/反向对偶」") become
 * on-device shard reductions: Y = P_0 + P_1 + ... + P_{t-1} + b and
 * dX = Q_0 + ... + Q_{t-1}, summed in fp32 in ascending shard order and
 * rounded once to bf16.  GeLU is the tanh form
 * g(x) = x/2·(1 + tanh(sqrt(2/pi)·(x + 0.044715·x^3))).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All matrices are row-major and contiguous in device memory owned by the
 *    caller.  bf16 (IEEE bfloat16): X[T,h], A[h,f], a[f], B[f,h], b[h],
 *    Y[T,h], dY[T,h], dX[T,h], dA[h,f], da[f], dB[f,h], db[h], and the
 *    pairs H, H_lo[T,f] and dH, dH_lo[T,f].  fp32: Z[T,f].  Shard i owns
 *    columns [i·f/t, (i+1)·f/t) of A, a, Z, H, dH, dA, da and rows
 *    [i·f/t, (i+1)·f/t) of B and dB.
 *  - Saved activations.  The forward saves the pre-activation Z = X·A + a in
 *    fp32 and the activation H = g(Z) as a bf16 pair (H, H_lo) with
 *    H = bf16(g(Z)) and H_lo = bf16(g(Z) − H), about 16 significant bits.
 *    The backward forms dH = (dY·Bᵀ) ⊙ g'(Z) in fp32 and keeps it as the
 *    same kind of pair.  The weight gradients dA = Xᵀ·dH and dB = Hᵀ·dY
 *    always use both halves of the pair (two bf16 tensor-core products);
 *    Y and dX use both halves in the default mode (MLP_TP_ACCURATE) and the
 *    high half only in the fast modes below.  da is summed from the fp32 dH
 *    before rounding.  With bf16-rounded intermediates alone, the gradients
 *    of a unit-scale batch of a few thousand tokens already differ from the
 *    exact block by more than 1e-2·(|exact| + 1); the pairs keep them well
 *    inside it.
 *  - Every device pointer must be 16-byte aligned.  Inputs are only read;
 *    outputs are overwritten (never accumulated into).  Outputs must not
 *    alias inputs or each other.
 *  - Shapes: T >= 0, h >= 64 and h % 64 == 0, t >= 1, f % t == 0,
 *    fs = f/t >= 64 and fs % 64 == 0, and T, h, f < 2^31.
 *  - `ws` is a caller-owned device workspace of at least
 *    mlp_tp_workspace_bytes(T, h, f, t) bytes, 256-byte aligned and
 *    zero-filled once before its first use; the library keeps a device
 *    status word in its first bytes and scratch after it.  Calls that share
 *    a workspace must be ordered on one stream.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *    enqueued on it; no entry point except mlp_tp_check synchronises, and
 *    none allocates or frees memory.  The enqueued work is kernel launches
 *    and asynchronous memsets; in addition, mlp_tp_forward / mlp_tp_backward
 *    (and the recomputing pair) in MLP_TP_FP8 run the mode's operand copies
 *    on a second stream the library owns (one per device and host thread,
 *    created on first use), forked from and joined back into `stream` with
 *    events, so stream order holds for the caller.  A sequence of calls can
 *    be captured into a CUDA graph and replayed (after one uncaptured call
 *    per shape, which sets the kernels' shared-memory limits and creates that
 *    stream); a replay reads the buffers' current contents.
 *  - Results are reproducible bit for bit for a given GPU model, shape and
 *    t: every reduction runs in a fixed order.
 *  - Arguments are validated on the host before anything is launched; on any
 *    error nothing is enqueued.  Errors raised by the CUDA runtime when
 *    launching map to MLP_ERR_CUDA.  Faults found by the kernels themselves
 *    (a bounded wait that ran out) are reported by mlp_tp_check.
 *  - The current CUDA device must be an sm_100 part (B200); there is no other
 *    code path and no CPU fallback.
 */
#ifndef MLP_TP_H_
#define MLP_TP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLP_OK = 0,
  MLP_ERR_INVALID_ARG = 1,         /* null pointer, negative size, t < 1 */
  MLP_ERR_UNSUPPORTED_SHAPE = 2,   /* divisibility / range rules above violated */
  MLP_ERR_MISALIGNED = 3,          /* a pointer is not 16-byte aligned */
  MLP_ERR_WORKSPACE_TOO_SMALL = 4, /* ws_bytes < mlp_tp_workspace_bytes(...) */
  MLP_ERR_UNSUPPORTED_DEVICE = 5,  /* current device is not sm_100, or none */
  MLP_ERR_CUDA = 6,                /* the CUDA runtime reported an error */
  MLP_ERR_TIMEOUT = 7,             /* a kernel's bounded wait ran out (mlp_tp_check) */
  MLP_ERR_BOUNDS = 8,              /* bounds-checking build only: an index fell outside its
                                      buffer; the access was skipped (mlp_tp_check) */
  MLP_ERR_RANGE = 9                /* MLP_TP_FP8 only: a value the mode's formats cannot hold
                                      (|H| or |dH·sH| >= 2^13, or a weight beyond the fp16
                                      range); the outputs are not valid (mlp_tp_check) */
} mlp_status_t;

/* Bytes of workspace needed by every entry point below for this shape
 * (the maximum over all of them): a 256-byte status header, the dH pair
 * used by mlp_tp_backward, fp32 column-sum partials, and fp32 scratch for
 * output tiles whose K loop is split into pieces (the shard sums of a
 * partial last wave, or the weight gradients when they have fewer tiles
 * than the GPU has CTA pairs).  Returns 0 for an invalid shape. */
size_t mlp_tp_workspace_bytes(int64_t T, int64_t h, int64_t f, int32_t t);

/* Precision mode of the composite calls: which second-layer products also
 * use the low half of the activation pair.  The weight gradients always do.
 *
 * 0 (MLP_TP_ACCURATE) is the default: Y = Σ_i (H_i + H_lo_i)·B_i + b and
 * dX = Σ_i (dH_i + dH_lo_i)·A_iᵀ, which meets
 * max|result − exact| <= 1e-2·(|exact| + 1) on every workload the tests run.
 *
 * The fast flags drop the low half from one or both of those products (half
 * their tensor-core work).  The error they add grows like
 * 2^-9·sqrt(f)·rms(B)·rms(H) for Y (and the same with A, dH for dX), so it
 * depends on the data, not on the shape alone.  Known cases:
 *   - meets the bar: the tiny (T=64, h=256, f=1024), GPT-2-medium (T=8192,
 *     h=1024, f=4096), h=4096 (T=4096, h=4096, f=16384, weights
 *     ~N(0, 0.0025)) and 175B-class (T=8192, h=12288, f=49152, weights
 *     ~N(0, 0.006)) workloads;
 *   - exceeds it: the 8.3B-class workload (T=16384, h=3072, f=12288,
 *     weights ~N(0, 0.02)), Y by 1.08x and dX by 1.14x of the tolerance. */
typedef enum {
  MLP_TP_ACCURATE = 0,
  MLP_TP_FAST_FC2_FORWARD = 1,       /* Y  = Σ_i H_i·B_i + b       (high half only) */
  MLP_TP_FAST_FC1_BACKWARD_DATA = 2, /* dX = Σ_i dH_i·A_iᵀ         (high half only) */
  MLP_TP_FAST = 3,                   /* both */
  MLP_TP_FP8 = 4                     /* fp16 operands with e4m3 residual products, below */
} mlp_tp_mode_t;

/* MLP_TP_FP8: FP8 tensor-core products ("NVIDIA Megatron-LM：大规模Transformer
 * 模型分布式训练框架", tech-stack item 混合精度: FP8 training on the newer
 * tensor cores) where they keep the block inside the parity bar.  Operands
 * enter 8-bit products only as the residual of a 16-bit one:
 *  - the forward saves Z (fp32), H as fp16 in `H` and the e4m3 residual
 *    e4m3((g(Z) − H)·2^7) in `H_lo` (T·f bytes of the caller's buffer);
 *  - Y = Σ_i H_i·fp16(B_i) + b and dX = Σ_i dH16_i·fp16(A_i)ᵀ / sH, one
 *    fp16 tensor-core product each (11 significant bits);
 *  - dH16 = fp16(dH·sH) and dH8 = e4m3((dH·sH − dH16)·2^7);
 *  - dB = (Hᵀ·dY16 + H_loᵀ·dY8) / sY and dA = (X16ᵀ·dH16 + X8ᵀ·dH8)/(sX·sH),
 *    where X16 = fp16(X·sX), X8 = e4m3(X·sX·2^-7) and the same for dY: an
 *    fp16 product plus an e4m3 (kind::f8f6f4) product into one fp32
 *    accumulator, about 15 significant bits for 1.5 bf16-products of tensor
 *    time instead of the pair's 2.
 * sX, sY are the largest powers of two with max|X|·sX, max|dY|·sY <= 2^15;
 * sH the largest with 1.212·max_t‖dY_t‖·max_k‖B_k‖·sH <= 2^12, which bounds
 * |dH·sH| (Cauchy–Schwarz, max|g'| < 1.2).  The statistics are reduced on
 * the device each backward; nothing is read back to the host.  Values the
 * formats cannot hold (|H| >= 2^13; a weight beyond 65504) are reported as
 * MLP_ERR_RANGE by mlp_tp_check.  Every output stays within
 * 1e-2·(|exact| + 1) of the exact block on all five workloads the tests run,
 * the 8.3B-class one included.  Y and dX carry 11 bits of H and dH: with
 * pre-activations near 40 and weights ~N(0, 0.3) (a stress case, not a
 * workload) Y reaches 1.96x the tolerance, where MLP_TP_ACCURATE keeps 16
 * bits.  This mode needs
 * mlp_tp_workspace_bytes_mode(..., MLP_TP_FP8) bytes of workspace (the
 * copies X16, X8, dY16, dY8 and fp16 B or A: 6·T·h + 2·h·f more bytes). */
size_t mlp_tp_workspace_bytes_mode(int64_t T, int64_t h, int64_t f, int32_t t, int32_t mode);

/* ---------------------------------------------------------------- forward */

/* Whole forward: mlp_tp_fc1_forward then mlp_tp_fc2_forward (the latter
 * given H_lo unless `mode` has MLP_TP_FAST_FC2_FORWARD; with MLP_TP_FP8 the
 * fp8 calls below).  Writes Y[T,h] and saves Z[T,f] (fp32), H[T,f] and
 * H_lo[T,f] for the backward. */
mlp_status_t mlp_tp_forward(const void* X, const void* A, const void* a,
                            const void* B, const void* b,
                            int64_t T, int64_t h, int64_t f, int32_t t, int32_t mode,
                            void* Y, void* Z, void* H, void* H_lo,
                            void* ws, size_t ws_bytes, void* stream);

/* ColumnParallelLinear of every shard plus the activation, one launch:
 * Z_i = X·A_i + a_i (fp32) and H_i = g(Z_i) as the pair (H_i, H_lo_i)
 * (shard i is column block i of Z, H and H_lo).  No reduction: the column
 * split needs none. */
mlp_status_t mlp_tp_fc1_forward(const void* X, const void* A, const void* a,
                                int64_t T, int64_t h, int64_t f, int32_t t,
                                void* Z, void* H, void* H_lo,
                                void* ws, size_t ws_bytes, void* stream);

/* RowParallelLinear of every shard plus the reduce that stands in for the
 * forward all-reduce: P_i = H_i·B_i (+ H_lo_i·B_i when H_lo is not NULL) in
 * fp32, Y = (((P_0 + P_1) + ...) + P_{t-1}) + b, rounded once to bf16.
 * `b` may be NULL (no bias); `H_lo` may be NULL (high half only). */
mlp_status_t mlp_tp_fc2_forward(const void* H, const void* H_lo, const void* B, const void* b,
                                int64_t T, int64_t h, int64_t f, int32_t t,
                                void* Y,
                                void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------- backward */

/* Whole backward, given dY and Z, H, H_lo saved by the forward:
 * mlp_tp_fc2_backward_data (dH pair into the workspace),
 * mlp_tp_fc2_backward_weight, mlp_tp_fc1_backward_data (given dH_lo unless
 * `mode` has MLP_TP_FAST_FC1_BACKWARD_DATA) and mlp_tp_fc1_backward_weight;
 * with MLP_TP_FP8 the fp8 calls below.  `da` and `db` may be NULL (bias
 * gradients not wanted). */
mlp_status_t mlp_tp_backward(const void* dY, const void* X, const void* A,
                             const void* B, const void* Z, const void* H, const void* H_lo,
                             int64_t T, int64_t h, int64_t f, int32_t t, int32_t mode,
                             void* dX, void* dA, void* da, void* dB, void* db,
                             void* ws, size_t ws_bytes, void* stream);

/* Backward of the row-parallel layer through the activation, per shard:
 * dH_i = (dY·B_iᵀ) ⊙ g'(Z_i) in fp32, written as the pair (dH, dH_lo), and
 * da = sum over rows of the fp32 dH (NULL: skip).  dY reaches every shard
 * unchanged (the reduce's backward is the identity). */
mlp_status_t mlp_tp_fc2_backward_data(const void* dY, const void* B, const void* Z,
                                      int64_t T, int64_t h, int64_t f, int32_t t,
                                      void* dH, void* dH_lo, void* da,
                                      void* ws, size_t ws_bytes, void* stream);

/* Weight gradients of the row-parallel layer: dB_i = (H_i + H_lo_i)ᵀ·dY
 * (each shard's own rows of dB, no reduction) and db = sum over rows of dY
 * (NULL: skip). */
mlp_status_t mlp_tp_fc2_backward_weight(const void* H, const void* H_lo, const void* dY,
                                        int64_t T, int64_t h, int64_t f, int32_t t,
                                        void* dB, void* db,
                                        void* ws, size_t ws_bytes, void* stream);

/* Input gradient of the column-parallel layer plus the reduce that stands in
 * for the copy operator's backward all-reduce: Q_i = dH_i·A_iᵀ (+ dH_lo_i·A_iᵀ
 * when dH_lo is not NULL) in fp32, dX = ((Q_0 + Q_1) + ...) + Q_{t-1},
 * rounded once to bf16. */
mlp_status_t mlp_tp_fc1_backward_data(const void* dH, const void* dH_lo, const void* A,
                                      int64_t T, int64_t h, int64_t f, int32_t t,
                                      void* dX,
                                      void* ws, size_t ws_bytes, void* stream);

/* Weight gradient of the column-parallel layer: dA_i = Xᵀ·(dH_i + dH_lo_i)
 * (each shard's own columns of dA, no reduction). */
mlp_status_t mlp_tp_fc1_backward_weight(const void* X, const void* dH, const void* dH_lo,
                                        int64_t T, int64_t h, int64_t f, int32_t t,
                                        void* dA,
                                        void* ws, size_t ws_bytes, void* stream);

/* ----------------------------------------------------- recomputation */

/* Activation recomputation ("Megatron-LM（英伟达超大模型训练框架）完整介绍", §三
 * 显存优化关键技术, item 2 激活重计算: drop the intermediate activations and
 * recompute them in the backward; "Megatron-LM 深度解读报告" §二 2.7 table).
 * mlp_tp_forward_recompute keeps Z, H and H_lo only in the workspace, where
 * the next call may overwrite them, so nothing of size T·f outlives the
 * forward; mlp_tp_backward_recompute reruns the column-parallel GEMM from X
 * (one extra 2·T·h·f product, bit-identical Z, H, H_lo) and then runs the
 * backward of mlp_tp_backward.  Both need
 * mlp_tp_recompute_workspace_bytes(T, h, f, t) bytes of workspace (the
 * ordinary workspace plus T·f·8 bytes for Z, H, H_lo).  Same conventions
 * and modes as mlp_tp_forward / mlp_tp_backward; with MLP_TP_FP8 the
 * workspace is mlp_tp_recompute_workspace_bytes_mode(..., MLP_TP_FP8)
 * bytes (the mode's operand copies after the recomputed activations). */
size_t mlp_tp_recompute_workspace_bytes(int64_t T, int64_t h, int64_t f, int32_t t);
size_t mlp_tp_recompute_workspace_bytes_mode(int64_t T, int64_t h, int64_t f, int32_t t, int32_t mode);

mlp_status_t mlp_tp_forward_recompute(const void* X, const void* A, const void* a,
                                      const void* B, const void* b,
                                      int64_t T, int64_t h, int64_t f, int32_t t, int32_t mode,
                                      void* Y,
                                      void* ws, size_t ws_bytes, void* stream);

mlp_status_t mlp_tp_backward_recompute(const void* dY, const void* X, const void* A,
                                       const void* a, const void* B,
                                       int64_t T, int64_t h, int64_t f, int32_t t, int32_t mode,
                                       void* dX, void* dA, void* da, void* dB, void* db,
                                       void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------- the fp16 + e4m3 mode by stage */

/* The stages of MLP_TP_FP8 (see the mode's description above), for callers
 * that interleave other work; mlp_tp_forward / mlp_tp_backward with
 * MLP_TP_FP8 run the same kernels in this order and give the same bits (they
 * only move the casts of the prepare calls onto their side stream, beside
 * the GEMMs).  All of them take a
 * workspace of mlp_tp_workspace_bytes_mode(..., MLP_TP_FP8) bytes, and the
 * same workspace from the prepare call on:
 *   forward:  mlp_tp_fp8_prepare_forward (fp16 copy of B into the workspace),
 *             mlp_tp_fc1_forward_fp8, mlp_tp_fc2_forward_fp8;
 *   backward: mlp_tp_fp8_prepare_backward (statistics, scales, the fp16 and
 *             e4m3 copies of X and dY and the fp16 copy of A), then
 *             mlp_tp_fc2_backward_data_fp8, mlp_tp_fc2_backward_weight_fp8,
 *             mlp_tp_fc1_backward_data_fp8, mlp_tp_fc1_backward_weight_fp8.
 * H and dH are fp16 [T,f]; H_lo and dH_lo hold the e4m3 residuals, T·f
 * bytes.  A stage given the outputs of another mode's stage computes
 * garbage: the formats differ. */
mlp_status_t mlp_tp_fp8_prepare_forward(const void* B, int64_t T, int64_t h, int64_t f, int32_t t,
                                        void* ws, size_t ws_bytes, void* stream);
mlp_status_t mlp_tp_fp8_prepare_backward(const void* dY, const void* X, const void* A, const void* B,
                                         int64_t T, int64_t h, int64_t f, int32_t t,
                                         void* ws, size_t ws_bytes, void* stream);
mlp_status_t mlp_tp_fc1_forward_fp8(const void* X, const void* A, const void* a,
                                    int64_t T, int64_t h, int64_t f, int32_t t,
                                    void* Z, void* H, void* H_lo,
                                    void* ws, size_t ws_bytes, void* stream);
/* `b` may be NULL (no bias). */
mlp_status_t mlp_tp_fc2_forward_fp8(const void* H, const void* b,
                                    int64_t T, int64_t h, int64_t f, int32_t t,
                                    void* Y, void* ws, size_t ws_bytes, void* stream);
/* `da` may be NULL; da is summed from the fp32 dH before any rounding. */
mlp_status_t mlp_tp_fc2_backward_data_fp8(const void* dY, const void* B, const void* Z,
                                          int64_t T, int64_t h, int64_t f, int32_t t,
                                          void* dH, void* dH_lo, void* da,
                                          void* ws, size_t ws_bytes, void* stream);
/* `db` may be NULL; db is summed from the bf16 dY. */
mlp_status_t mlp_tp_fc2_backward_weight_fp8(const void* H, const void* H_lo, const void* dY,
                                            int64_t T, int64_t h, int64_t f, int32_t t,
                                            void* dB, void* db,
                                            void* ws, size_t ws_bytes, void* stream);
mlp_status_t mlp_tp_fc1_backward_data_fp8(const void* dH,
                                          int64_t T, int64_t h, int64_t f, int32_t t,
                                          void* dX, void* ws, size_t ws_bytes, void* stream);
mlp_status_t mlp_tp_fc1_backward_weight_fp8(const void* dH, const void* dH_lo,
                                            int64_t T, int64_t h, int64_t f, int32_t t,
                                            void* dA, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------- across GPUs */

/* The block sharded over `world` GPUs, one shard per GPU (rank r holds
 * columns [r·f/world, (r+1)·f/world) of A and a and those rows of B; each
 * rank calls the stage entry points above with t = 1 on its shard, fs =
 * f/world).  The two sums of the tensor-parallel pair ("Megatron-LM — 架构与
 * 原理", §4 巧妙之处: Y = Σ_r P_r + b after the row-parallel layer, the
 * reduce operator's forward all-reduce, and dX = Σ_r Q_r, the copy
 * operator's backward all-reduce) are fused into the row-parallel GEMMs:
 *
 *  - mlp_tp_fc2_forward_peer / mlp_tp_fc1_backward_data_peer compute this
 *    rank's partial P_r = (H_r + H_lo_r)·B_r (or Q_r = (dH_r + dH_lo_r)·A_rᵀ)
 *    in fp32 and, from the GEMM epilogue, store each 128-row block of it into
 *    the receive buffer of the rank that owns those tokens (rank o owns rows
 *    [o·T/world, (o+1)·T/world)), slot r, with plain stores through the peer
 *    mapping (NVLink), then raise that block's arrival count on the owner;
 *  - mlp_tp_peer_reduce, on the owner, waits for the `world` partials of each
 *    block, sums them in fp32 in rank order, adds `bias` once (NULL: none),
 *    rounds once to bf16 into out[T/world, h] (this rank's token rows) and
 *    marks the block consumed, so the next exchange may overwrite it.
 *
 * That is the reduce-scatter of the sequence-parallel form; the plain
 * tensor-parallel form follows it with an all-gather of the bf16 rows.  The
 * partials stay fp32 and are rounded once: summing per-rank bf16 outputs,
 * as a 16-bit all-reduce does, exceeds 1e-2·(|exact| + 1) on the 8.3B-class
 * workload at 2, 4 and 8 ranks.
 *
 * Buffers.  Each rank allocates (device memory, zero-filled once) a receive
 * buffer of mlp_tp_peer_recv_bytes(T, h, world) bytes ([world][T/world][h]
 * fp32) and a flag block of mlp_tp_peer_flag_bytes(T, h, world) bytes, and
 * every rank's descriptor lists all ranks' buffers as addressed from its own
 * GPU (its own pointers for itself; mappings of the others', for example
 * from mlp_tp_ipc_import).  Shapes: T % world == 0, and with world > 1 the
 * T/world rows of a rank a multiple of 128; h as elsewhere.
 *
 * Ordering.  `epoch` numbers the exchanges on these buffers: 1 for the first,
 * then +1 per exchange, the same on every rank.  Each wait is bounded by the
 * wait budget (mlp_tp_set_wait_budget_ns); one that runs out records
 * MLP_ERR_TIMEOUT in the caller's workspace (mlp_tp_check), and the flag
 * blocks must then be zero-filled again and `epoch` restarted at 1.  With
 * epoch == 0 no flag is read or written (flags may be NULL): the caller
 * orders the GEMM and the reduce itself, e.g. on one stream with a
 * collective on the fp32 buffer in between (world = 1 then describes this
 * rank's own buffer: the GEMM writes its whole [T, h] partial to slot 0). */
#define MLP_TP_MAX_WORLD 8
#define MLP_TP_IPC_HANDLE_BYTES 64

typedef struct {
  int32_t rank;                   /* this GPU's rank, 0 <= rank < world */
  int32_t world;                  /* GPUs in the group, 1..MLP_TP_MAX_WORLD */
  uint32_t epoch;                 /* exchange number (1, 2, ...), or 0: no flags */
  uint32_t reserved;              /* 0 */
  void* recv[MLP_TP_MAX_WORLD];   /* rank o's receive buffer as addressed from this GPU */
  void* flags[MLP_TP_MAX_WORLD];  /* rank o's flag block as addressed from this GPU */
} mlp_tp_peer_t;

/* Bytes of one rank's receive buffer and flag block (multiples of 256);
 * 0 for an invalid shape. */
size_t mlp_tp_peer_recv_bytes(int64_t T, int64_t h, int32_t world);
size_t mlp_tp_peer_flag_bytes(int64_t T, int64_t h, int32_t world);

/* This rank's row-parallel partial P_r = (H + H_lo)·B (H_lo NULL: H only),
 * H[T, fs], B[fs, h], sent to the owners as described above.  `ws` as for
 * mlp_tp_fc2_forward with f = fs, t = 1. */
mlp_status_t mlp_tp_fc2_forward_peer(const void* H, const void* H_lo, const void* B,
                                     int64_t T, int64_t h, int64_t fs, const mlp_tp_peer_t* peer,
                                     void* ws, size_t ws_bytes, void* stream);

/* This rank's partial input gradient Q_r = (dH + dH_lo)·Aᵀ (dH_lo NULL: dH
 * only), dH[T, fs], A[h, fs], sent to the owners likewise. */
mlp_status_t mlp_tp_fc1_backward_data_peer(const void* dH, const void* dH_lo, const void* A,
                                           int64_t T, int64_t h, int64_t fs, const mlp_tp_peer_t* peer,
                                           void* ws, size_t ws_bytes, void* stream);

/* The same two GEMMs in MLP_TP_FP8 form, after mlp_tp_fp8_prepare_forward /
 * mlp_tp_fp8_prepare_backward on this rank's shard (t = 1, f = fs) and
 * workspace (mlp_tp_workspace_bytes_mode(T, h, fs, 1, MLP_TP_FP8) bytes):
 * P_r = H16·fp16(B_r) and Q_r = dH16·fp16(A_r)ᵀ / sH with H, dH fp16 [T, fs].
 * Each rank's sH follows from its own shard of B; the fp32 partials carry no
 * scale, so the owner's sum is the same call as in the other modes. */
mlp_status_t mlp_tp_fc2_forward_peer_fp8(const void* H, int64_t T, int64_t h, int64_t fs,
                                         const mlp_tp_peer_t* peer, void* ws, size_t ws_bytes, void* stream);
mlp_status_t mlp_tp_fc1_backward_data_peer_fp8(const void* dH, int64_t T, int64_t h, int64_t fs,
                                               const mlp_tp_peer_t* peer, void* ws, size_t ws_bytes,
                                               void* stream);

/* The owner's sum: out[T/world, h] = bf16(Σ_r slot r + bias), rank order.
 * `ws` needs only its 256-byte status header here. */
mlp_status_t mlp_tp_peer_reduce(const mlp_tp_peer_t* peer, const void* bias, int64_t T, int64_t h,
                                void* out, void* ws, size_t ws_bytes, void* stream);

/* Mapping a buffer of another process on another GPU (CUDA IPC).
 * mlp_tp_ipc_export writes the MLP_TP_IPC_HANDLE_BYTES-byte handle of the
 * allocation that holds `ptr` and ptr's offset in it; mlp_tp_ipc_import, in
 * another process, maps that allocation (peer access enabled) and returns
 * the address of the same byte; mlp_tp_ipc_close unmaps it.  A process does
 * not import its own handles. */
mlp_status_t mlp_tp_ipc_export(const void* ptr, void* handle, uint64_t* offset);
mlp_status_t mlp_tp_ipc_import(const void* handle, uint64_t offset, void** ptr);
mlp_status_t mlp_tp_ipc_close(void* ptr, uint64_t offset);

/* ----------------------------------------------------- allocation-free */

/* db = sum over rows of dY (the row-parallel layer's bias gradient, as
 * mlp_tp_fc2_backward_weight computes it) without a workspace.
 *
 * The pages describe nothing like this; it exists for callers that cannot
 * allocate device memory: code that must run from a fixed, pre-planned
 * memory budget (a serving process whose pool already owns every byte of
 * HBM), or a host framework whose plugin interface hands over only the
 * input and output pointers, with no scratch and no allocator.  The fp32
 * partial sums go to a static device array of 2^20 floats (4 MiB) inside the
 * library, which every GPU that loads the library holds until the process
 * exits.  Shapes with ceil(T/256)·h > 2^20 are rejected with
 * MLP_ERR_UNSUPPORTED_SHAPE (use mlp_tp_fc2_backward_weight then).
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls share the one array: calls whose
 * work overlaps on the GPU (different streams, or several host threads
 * without ordering) race on it; calls ordered on one stream do not.  No
 * call allocates or frees memory.  Same pointer, alignment and device rules
 * as the other entry points; dY may be NULL when T == 0 (db is zero-filled).
 * The path keeps its own device status word beside the array;
 * mlp_tp_check(NULL, stream) reads it. */
mlp_status_t mlp_tp_fc2_bias_grad_noalloc(const void* dY, int64_t T, int64_t h, void* db, void* stream);

/* ------------------------------------------------------------ diagnostics */

/* Synchronises `stream`, then reads and clears the device status word in
 * `ws` (ws == NULL: the status word of mlp_tp_fc2_bias_grad_noalloc on the
 * current device).  Returns MLP_OK, MLP_ERR_TIMEOUT (a kernel's bounded wait
 * ran out; that launch's outputs, and anything later on the context, are not
 * to be trusted: a copy the kernel could not wait for may still have landed
 * after it returned), MLP_ERR_BOUNDS (only from a library built with
 * -DMLPTP_BOUNDS_CHECK: a plain global access outside its buffer was found
 * and skipped) or MLP_ERR_CUDA (the stream reported an error). */
mlp_status_t mlp_tp_check(void* ws, void* stream);

/* Static, NUL-terminated name of a status code. */
const char* mlp_tp_status_string(mlp_status_t status);

/* Thread-local, NUL-terminated description of the last error returned to
 * this thread (which argument, which CUDA call).  Valid until the next call
 * from the same thread. */
const char* mlp_tp_last_error(void);

/* Number of kernels the library enqueued from this process so far (all
 * threads).  Used to count launches inside a timed region. */
uint64_t mlp_tp_launch_count(void);

/* Upper bound, in nanoseconds, on any single wait inside a kernel (default
 * 1e9).  Past it the kernel records MLP_ERR_TIMEOUT and returns.  Applies to
 * later launches; values below 1e6 are raised to 1e6. */
void mlp_tp_set_wait_budget_ns(uint64_t ns);

/* Test hook: when `flags` & 1, the next launches' operand-loading warp
 * stops after its first tile stage, so the tensor-core warp's wait for the
 * second stage can only end by running out of its budget.  Takes effect on
 * launches enqueued after the call; 0 restores normal operation. */
void mlp_tp_set_debug_flags(uint32_t flags);

#ifdef __cplusplus
}
#endif

#endif /* MLP_TP_H_ */
