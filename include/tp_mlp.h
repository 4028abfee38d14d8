/*
 * tp_mlp.h -- C ABI of the tensor-parallel two-projection MLP on one B200.
 *
 * The operation (sources by page title and section):
 *   "LLM 推理并行化：先找瓶颈，再决定怎么切", §三 2) 张量并行（TP）: the first
 *   weight is split by columns and the second by rows; rank i computes
 *   hidden_i = act(x @ A_i) and partial_i = hidden_i @ B_i, and the layer
 *   output is the sum of the partials (an all-reduce across ranks).  The
 *   default activation is tanh.
 *   "大模型推理系统揭秘（07）：Multi-GPU：一张卡不够时如何扩展？", §1.2.2 (column-
 *   and row-parallel linears), §1.2.3 (Z = [Y_0|..|Y_P-1][W_20;..] = sum_i
 *   Y_i W_2i), §1.2.4 (gate/up column-parallel, activation local, down
 *   row-parallel) and §1.4.3 (SwiGLU: W_2[SiLU(W_1 x) ⊙ (W_3 x)]).
 *
 * Here every rank's shards live in the memory of ONE GPU, so the all-reduce
 * is a sum on the device, fused into the second projection's accumulation.
 *
 * Two more operators from the same pages take no handle but follow the same
 * conventions: tp_mlp_allreduce_residual_rmsnorm (the all-reduce of the
 * ranks' partials fused with the residual add and RMSNorm that follow it) and
 * tp_mlp_merge_attention_partials (decode context parallelism's merge of the
 * KV shards' partial attention results).  Their declarations are at the end.
 *
 * Conventions for every entry point
 *   - Matrices are row-major and densely packed (row stride = row length).
 *   - "device pointer" = memory of the current CUDA device; "host" = CPU memory.
 *   - Every pointer argument must be 16-byte aligned (TP_MLP_ERR_ALIGNMENT).
 *   - All calls that take a stream are asynchronous on it; arguments are
 *     checked on the host first and, on any error, nothing is launched and no
 *     output is written.  Errors of earlier asynchronous work surface as
 *     TP_MLP_ERR_CUDA on a later call or at the caller's synchronisation.
 *   - The library never allocates device memory.  The caller owns x, the
 *     shards, out, partials, the packed buffer and the workspace; the handle
 *     owns host metadata only.
 *   - A handle must not be used from two host threads or two streams at once:
 *     its workspace is shared by the calls made on it.
 *   - Accumulation is always fp32.  x, the weights and out share the handle's
 *     dtype; partials are fp32.
 */
#ifndef TP_MLP_H
#define TP_MLP_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque handle (host memory, owned by the library). */
typedef struct tp_mlp_s *tp_mlp_t;

/* A CUDA stream; the same type as cudaStream_t.  NULL = the legacy default stream. */
typedef struct CUstream_st *tp_mlp_stream_t;

/* Activation applied to the first projection.
 *   TANH:     H = tanh(X A)                 (the pages' default activation)
 *   SWIGLU:   H = SiLU(X gate) * (X up), SiLU(g) = g / (1 + e^{-g})
 *   IDENTITY: H = X A                       (no activation; exact-integer tests) */
typedef enum { TP_MLP_ACT_TANH = 0, TP_MLP_ACT_SWIGLU = 1, TP_MLP_ACT_IDENTITY = 2 } tp_mlp_act;

/* Element type of x, the weights and out. */
typedef enum { TP_MLP_F32 = 0, TP_MLP_BF16 = 1 } tp_mlp_dtype;

typedef enum {
    TP_MLP_OK = 0,
    TP_MLP_ERR_INVALID_ARG = 1,  /* NULL handle/pointer, unknown enum value            */
    TP_MLP_ERR_SHAPE = 2,        /* sizes, shard count, d_ff % tp, tokens > max_tokens */
    TP_MLP_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned                   */
    TP_MLP_ERR_UNSUPPORTED = 4,  /* valid request the library cannot serve            */
    TP_MLP_ERR_CUDA = 5,         /* a CUDA runtime call failed (launch or earlier work) */
    TP_MLP_ERR_TIMEOUT = 6,      /* a bounded device-side wait ran out (status calls)  */
    TP_MLP_ERR_WORKSPACE = 7     /* no workspace set, or smaller than required         */
} tp_mlp_status;

/* Kernel family used for a forward (for tests and measurements). */
typedef enum {
    TP_MLP_PLAN_AUTO = 0,   /* let the library choose (default)                      */
    TP_MLP_PLAN_SIMT = 1,   /* tiled CUDA-core kernels, any shape and layout          */
    TP_MLP_PLAN_GEMV = 2,   /* packed bf16, 1-4 tokens: streaming split-K GEMV        */
    TP_MLP_PLAN_TC = 3,     /* packed bf16: tcgen05 tensor-core GEMMs (TMA + TMEM);
                               the library picks the tiling from the token count      */
    TP_MLP_PLAN_TC_WIDE = 4,   /* tcgen05, tiles of 128 tokens x 256 weight rows      */
    TP_MLP_PLAN_TC_SKINNY = 5, /* tcgen05, weights as the MMA's M (tiles of 128 or 256
                                  rows), 1..128 tokens as N; the weight stream split
                                  evenly over the SMs, or whole CTAs per tile when
                                  tiles are few                                       */
    TP_MLP_PLAN_TC_WIDE256 = 6, /* tcgen05, tiles of 256 tokens x 256 weight rows     */
    TP_MLP_PLAN_TC_PAIR = 7,    /* packed bf16: tcgen05 on pairs of CTAs (cta_group::2),
                                   256 tokens x 256 weight rows per pair, two TMEM
                                   accumulators per CTA                               */
    TP_MLP_PLAN_TC_PAIR2 = 8,   /* packed bf16: pairs of CTAs, 256 tokens x 512 weight
                                   rows per pair (two weight tiles share each X stage) */
    TP_MLP_PLAN_TC_FUSED = 9    /* bf16, 1..128 tokens: the skinny tiling with both
                                   projections in one persistent launch (the
                                   second projection's weights stream in while the
                                   first finishes; its H loads wait on a device
                                   counter).  Needs every CTA of the grid (one per
                                   SM) resident at once: a GPU shared with other work
                                   can make the bounded wait run out, reported as
                                   TP_MLP_ERR_TIMEOUT by tp_mlp_get_device_status.
                                   Auto takes it for packed weights; the shard form
                                   (tp_mlp_forward) runs it when chosen.       */
} tp_mlp_plan;

/*
 * Create a handle for one MLP shape: the shapes of the pages' call
 * tensor_parallel_output(x, a_shards, b_shards, activation) ("LLM 推理并行化"
 * §三 2)), fixed once.
 *   d_model    input width (columns of x, rows of every A_i), >= 1
 *   d_ff       intermediate width summed over ranks; d_ff % tp_degree == 0
 *   d_out      output width (columns of every B_i); pass d_model for the usual
 *              square layer (the §1.2.3 example maps 8 -> 8 -> 4)
 *   tp_degree  number of ranks (shards), 1..8
 *   act, dtype see the enums above
 *   max_tokens largest token count a call will pass, >= 1
 * Allocates host memory only.  Returns TP_MLP_OK and sets *handle, or an
 * error and leaves *handle untouched.
 */
int tp_mlp_create(tp_mlp_t *handle, int d_model, int d_ff, int d_out, int tp_degree,
                  int act, int dtype, int max_tokens);

/* Free the handle (host memory).  NULL is accepted.  The pages' function holds
 * no state; the handle only caches the shape of one tensor_parallel_output. */
int tp_mlp_destroy(tp_mlp_t handle);

/*
 * Device workspace (bytes) the forward / partials / packed calls need for
 * `tokens` tokens (0 <= tokens <= max_tokens).  It holds the intermediate
 * activation H (tokens x d_ff, dtype) -- the per-rank hidden_i = act(x @ A_i)
 * of "LLM 推理并行化" §三 2), stored for all ranks side by side -- and split-K
 * scratch.  The first tp_mlp_workspace_bytes(handle, 0) bytes are the split-
 * tile counters and the device status word.  Returns 0 for an invalid handle
 * or token count.
 */
size_t tp_mlp_workspace_bytes(tp_mlp_t handle, int tokens);

/*
 * Give the handle a device workspace of `bytes` bytes (owned by the caller,
 * kept until replaced or the handle is destroyed; the pages leave memory to
 * the caller, who here is PyTorch).  Zeroes the split-K counters inside it and
 * waits for that to finish.  bytes must be at least
 * tp_mlp_workspace_bytes(handle, max_tokens) -- or pass the size for the
 * largest token count you will use: each call checks its own need.
 */
int tp_mlp_set_workspace(tp_mlp_t handle, void *dev_ptr, size_t bytes);

/*
 * Forward pass on per-rank shards, the pages' interface
 * tensor_parallel_output(x, a_shards, b_shards, activation):
 *   out = sum_{i<tp} act(x @ A_i) @ B_i
 *   x          device, tokens x d_model
 *   A_shards   host array of tp_degree device pointers.
 *              tanh / identity: A_i is d_model x f_s (columns i*f_s.. of A);
 *              SwiGLU: A_i is d_model x 2*f_s laid out [gate_i | up_i]
 *              (gate and up columns of the same intermediate features).
 *   B_shards   host array of tp_degree device pointers; B_i is f_s x d_out
 *              (rows i*f_s.. of B).           f_s = d_ff / tp_degree.
 *   tp_degree  must equal the handle's (the shard arrays are paired strictly)
 *   act        must equal the handle's
 *   out        device, tokens x d_out
 *   stream     CUDA stream
 * tokens == 0 is a no-op.  Uses the workspace.  For bf16 with f_s a multiple
 * of 64 (and d_model, d_ff, d_out multiples of 8) the tcgen05 kernels read the
 * shards directly, as MN-major operands; otherwise CUDA-core kernels run.
 */
int tp_mlp_forward(tp_mlp_t handle, const void *x, int tokens, const void *const *A_shards,
                   const void *const *B_shards, int tp_degree, int act, void *out,
                   tp_mlp_stream_t stream);

/*
 * Per-rank partials without the final sum ("大模型推理系统揭秘（07）" §1.2.2,
 * row-parallel linear: each rank's Z_i = Y_i W_2i, still to be all-reduced;
 * "LLM 推理并行化" §三 2): partial_i = hidden_i @ B_i):
 *   partials[i] = act(x @ A_i) @ B_i, fp32, laid out tp_degree x tokens x d_out
 * (device).  Other arguments as tp_mlp_forward.  Summing them over i gives the
 * forward's result (before rounding to the output dtype).  For bf16 with f_s
 * a multiple of 64 the tcgen05 kernels run, with each rank's K loop kept
 * apart; otherwise CUDA-core kernels.
 */
int tp_mlp_partials(tp_mlp_t handle, const void *x, int tokens, const void *const *A_shards,
                    const void *const *B_shards, int tp_degree, int act, float *partials,
                    tp_mlp_stream_t stream);

/*
 * Size in bytes of the packed weight buffer (the shard-layout packer's output).
 * The packer holds the column shards A_i and row shards B_i of
 * "大模型推理系统揭秘（07）" §1.2.2-§1.2.3 (A split along columns, B along
 * rows, each rank taking f_s = d_ff / tp of them, "LLM 推理并行化" §三 2)).
 * The buffer has two parts, each a matrix of R "rows" by K, one row per output
 * of its projection (element = the handle's dtype):
 *   part 1, first projection, K = d_model: tanh / identity: row n holds column
 *     n of A (n = i*f_s + j over ranks i in order), R = d_ff.  SwiGLU: row
 *     256*b + r holds the gate column of feature 128*b + r and row 256*b + 128
 *     + r its up column (r < 128), R = 256 * ceil(d_ff / 128).
 *   part 2, second projection, K = d_ff: row c holds column c of B, i.e.
 *     B[k][c] with k over rank 0's rows, then rank 1's, ... (R = d_out), so one
 *     K loop along a row sums the ranks.
 * Each part is stored tile-blocked: rows in tiles of 256, K in blocks of 64;
 * element (row, k) is at ((row/256 * ceil(K/64) + k/64) * 256 + row%256) * 64
 * + k%64, so every 256 x 64 block is contiguous and the blocks of a tile follow
 * each other.  Unused rows and k positions are zero.  Part 2 starts at the
 * first 256-byte boundary after part 1.
 */
size_t tp_mlp_packed_bytes(tp_mlp_t handle);

/* Pack the shards (same arrays as tp_mlp_forward) into `packed` (device,
 * tp_mlp_packed_bytes bytes).  A bit-exact copy in a new order: concatenating
 * the column shards gives A and stacking the row shards gives B
 * ("大模型推理系统揭秘（07）" §1.2.3), and that is the order stored.  The
 * handle's tp_degree fixes how many pointers each array holds. */
int tp_mlp_pack(tp_mlp_t handle, const void *const *A_shards, const void *const *B_shards,
                void *packed, tp_mlp_stream_t stream);

/* Inverse of tp_mlp_pack: cut A and B back into the per-rank shards of
 * "大模型推理系统揭秘（07）" §1.2.2 and write them from `packed` (bit-exact). */
int tp_mlp_unpack(tp_mlp_t handle, const void *packed, void *const *A_shards,
                  void *const *B_shards, tp_mlp_stream_t stream);

/*
 * Forward pass on packed weights (the fast path; weights are packed once):
 * the same out = sum_i act(x @ A_i) @ B_i as tp_mlp_forward ("LLM 推理并行化"
 * §三 2); "大模型推理系统揭秘（07）" §1.2.3), with the sum over ranks done
 * inside the second projection's accumulation.
 *   x device tokens x d_model, out device tokens x d_out, packed from
 *   tp_mlp_pack.  Same result as tp_mlp_forward up to fp32 summation order.
 */
int tp_mlp_forward_packed(tp_mlp_t handle, const void *x, int tokens, const void *packed,
                          void *out, tp_mlp_stream_t stream);

/* Force a kernel family (tp_mlp_plan) for later forwards; AUTO restores the
 * library's choice (decode is weight-read-bound, prefill compute-bound,
 * "7.4 推理侧并行" §7.4.1, so the choice follows the token count).  A forced plan that cannot serve a call returns
 * TP_MLP_ERR_UNSUPPORTED from that call. */
int tp_mlp_set_plan(tp_mlp_t handle, int plan);

/*
 * How the skinny tensor-core tiling (TP_MLP_PLAN_TC_SKINNY) finishes a weight
 * tile whose K loop is split between CTAs.  Both add the fp32 partial slots in
 * the same fixed order, so they give identical results; they differ in speed.
 */
typedef enum {
    TP_MLP_SPLITK_AUTO = 0,      /* default: SEPARATE (measured fastest on B200)       */
    TP_MLP_SPLITK_IN_KERNEL = 1, /* the last CTA to finish its share adds the slots   */
    TP_MLP_SPLITK_SEPARATE = 2,  /* a reduction kernel behind each GEMM adds them,
                                    spread over the whole GPU                        */
    TP_MLP_SPLITK_CLUSTER = 3    /* where a whole number (2..8) of CTAs share each
                                    tile and all fit at once, those CTAs form a
                                    thread-block cluster and add their slots through
                                    distributed shared memory at the end of the GEMM;
                                    otherwise as SEPARATE                            */
} tp_mlp_splitk;

/* Choose the split-tile finish (tp_mlp_splitk) for later forwards.  Returns
 * TP_MLP_ERR_INVALID_ARG for another value.  Other plans ignore it.  (No
 * counterpart in the pages: how one GPU adds the pieces of one tile.) */
int tp_mlp_set_splitk(tp_mlp_t handle, int mode);

/*
 * Timing hook (measurement only; no counterpart in the pages): with n > 0, later forward / forward_packed / partials calls
 * record events[0] on their stream before their first kernel, events[1] after
 * the first projection's kernels and events[2] after the second projection's
 * (events beyond events[2] are not recorded).  The events are caller-owned cudaEvent_t handles (created with
 * timing enabled) and must stay valid while calls use them; n = 0 (or
 * events = NULL) turns the hook off.  At most 8 events.
 */
int tp_mlp_set_profile_events(tp_mlp_t handle, void *const *events, int n);

/*
 * Device-side status of the work issued so far on this handle's workspace
 * (the pages describe no failure detection; this is the library's own):
 * synchronises the device, returns TP_MLP_ERR_TIMEOUT if a kernel gave up a
 * bounded internal wait (its results are then invalid), TP_MLP_OK otherwise.
 * On a timeout it also zeroes the split-tile counters, which the CTAs that
 * left early may have left part-way, and the flag: calls made after a timeout
 * and before this call may give wrong results.  Needs a workspace.
 */
int tp_mlp_get_device_status(tp_mlp_t handle);

/*
 * Self-test of failure detection (the pages describe none): launches one
 * small kernel that waits, through the same bounded mbarrier wait every
 * pipelined kernel here uses, on a barrier nothing will complete.  The wait
 * gives up after wait_us microseconds (1..100000), the kernel records the
 * timeout in the handle's status word and returns; nothing traps.  A later
 * tp_mlp_get_device_status then returns TP_MLP_ERR_TIMEOUT (and clears it),
 * and the context stays usable.  Needs a workspace.
 */
int tp_mlp_selftest_bounded_wait(tp_mlp_t handle, unsigned wait_us, tp_mlp_stream_t stream);

/* Plan (tp_mlp_plan) and number of kernel launches of the last successful
 * forward / partials call on this handle; -1 before the first.  (Measurement
 * hooks; the pages put each launch at 5-10 us of a decode step, "7.4 推理侧并行"
 * §7.4.2.) */
int tp_mlp_last_plan(tp_mlp_t handle);
int tp_mlp_last_launches(tp_mlp_t handle);

/*
 * Decode forward that allocates nothing and needs no workspace.
 *
 * The pages have no counterpart of this call; it exists for callers that
 * cannot allocate device memory (code inside host callbacks or allocator
 * hooks, plugins whose host owns every allocation, sandboxes that forbid
 * cudaMalloc), so they cannot provide the workspace the other calls need.
 * It computes what tp_mlp_forward_packed computes with the GEMV kernels --
 * bf16 only, 1..4 tokens -- but keeps the intermediate activation and the
 * split-K scratch in one fixed 8 MiB array of device memory built into the
 * library, which every GPU that loads the library holds until the process
 * exits.
 *   d_model, d_ff, d_out, tp_degree, act   describe the MLP as for tp_mlp_create
 *   x       device, tokens x d_model bf16
 *   packed  device, the buffer tp_mlp_pack wrote for this shape (bf16)
 *   out     device, tokens x d_out bf16
 * The caller still owns x, packed and out.  The first call on each device
 * looks up that device's copy of the array (with the device current); make
 * that first call before capturing a stream.  Every call shares the array and
 * leaves its contents behind; each call clears, on its stream, the parts that
 * must start at zero.  Calls whose kernels overlap on the GPU race on the
 * array: order them on one stream or with events.  A kernel that gives up a
 * bounded internal wait records it in the array's status word, which no call
 * clears; tp_mlp_decode_static_status reports it.
 * Errors: TP_MLP_ERR_WORKSPACE if this shape needs more scratch than the
 * 8 MiB array holds (nothing is launched); TP_MLP_ERR_UNSUPPORTED for shapes
 * the GEMV kernels do not take (d_model or d_ff not a multiple of 8);
 * otherwise as tp_mlp_forward_packed.  tokens == 0 is a no-op.
 */
int tp_mlp_decode_forward_static(int d_model, int d_ff, int d_out, int tp_degree, int act,
                                 const void *x, int tokens, const void *packed, void *out,
                                 tp_mlp_stream_t stream);

/*
 * Status of the tp_mlp_decode_forward_static calls issued so far on the
 * current device (no counterpart in the pages): synchronises the device and
 * returns TP_MLP_ERR_TIMEOUT if one of their kernels gave up a bounded
 * internal wait -- the results of that call are invalid -- and clears the
 * record; TP_MLP_OK otherwise (also when no call has run on this device).
 * Allocates nothing.
 */
int tp_mlp_decode_static_status(void);

/*
 * The all-reduce of the ranks' partial outputs fused with the residual add and
 * RMSNorm that follow it ("7.4 推理侧并行", §7.4.2, optimisation 2: done in
 * one kernel, the summed activations are not stored and reloaded).  With
 * every rank on one GPU the all-reduce is the sum of the fp32 partials that
 * tp_mlp_partials returns.  For every token row t (ranks added in order,
 * fp32 arithmetic):
 *     h               = residual[t] + sum_i partials[i][t]
 *     residual_out[t] = h
 *     y[t]            = h / sqrt(mean_j h_j^2 + eps) * gamma
 * The pages do not define RMSNorm; this is the textbook form (no mean
 * subtraction, no bias).  Needs no handle and no workspace.
 *
 *   partials      device fp32, tp_degree x tokens x d, row-major (rank-major)
 *   residual      device, tokens x d, element type `dtype` (tp_mlp_dtype)
 *   gamma         device, d elements of `dtype`
 *   y             device, tokens x d of `dtype`
 *   residual_out  device, tokens x d of `dtype`; may be `residual` itself
 *                 (updated in place).  Other overlaps between the buffers are
 *                 not allowed.
 * Requirements: 1 <= tp_degree <= 8, tokens >= 0 (0 is a no-op),
 * 4 <= d <= 49152 with d % 4 == 0 (TP_MLP_ERR_SHAPE otherwise), eps >= 0 and
 * finite (TP_MLP_ERR_INVALID_ARG), every pointer 16-byte aligned
 * (TP_MLP_ERR_ALIGNMENT) and inside a device allocation of the stated size
 * (TP_MLP_ERR_SHAPE / TP_MLP_ERR_INVALID_ARG).  Asynchronous on `stream`;
 * the caller owns every buffer.
 */
int tp_mlp_allreduce_residual_rmsnorm(const float *partials, int tp_degree, int tokens, int d,
                                      const void *residual, const void *gamma, float eps, int dtype,
                                      void *y, void *residual_out, tp_mlp_stream_t stream);

/*
 * Merge of partial attention results across KV shards (decode context
 * parallelism; "LLM 推理并行化：先找瓶颈，再决定怎么切", §三 4) 上下文并行（CP））.
 * Each of the tp_degree ranks attended over its own part of the KV history
 * and reports, for every query row (one token and head): its maximum score,
 * the sum of exp(score - maximum) and the exp-weighted sum of the values.
 * The merge takes the global maximum M of a row, rescales every rank by
 * exp(maximum_i - M), adds, and divides the merged weighted sum by the merged
 * exponential sum -- attention over the whole history.  A rank with no keys
 * for a row reports maximum -inf (and 0, 0) and contributes nothing; a row
 * with every rank empty is written as zeros.  Needs no handle and no workspace.
 *
 *   maximum, exp_sum  device fp32, tp_degree x rows (rank-major)
 *   weighted          device, tp_degree x rows x head_dim, element type `dtype`
 *   out               device, rows x head_dim of `dtype`; must not overlap
 *                     the inputs
 * Requirements: 1 <= tp_degree <= 8, rows >= 0 (0 is a no-op), 4 <= head_dim
 * <= 4096 with head_dim % 4 == 0 (TP_MLP_ERR_SHAPE otherwise), a valid dtype
 * (TP_MLP_ERR_INVALID_ARG), every pointer 16-byte aligned
 * (TP_MLP_ERR_ALIGNMENT) and inside a device allocation of the stated size
 * (TP_MLP_ERR_SHAPE / TP_MLP_ERR_INVALID_ARG).  fp32 arithmetic; asynchronous
 * on `stream`; the caller owns every buffer.
 */
int tp_mlp_merge_attention_partials(int tp_degree, int rows, int head_dim, const float *maximum,
                                    const float *exp_sum, const void *weighted, int dtype, void *out,
                                    tp_mlp_stream_t stream);

/*
 * Tensor parallelism across GPUs: rank i holds only A_i and B_i, and the sum of
 * the partials is an all-reduce between GPUs ("大模型推理系统揭秘（07）" §1.2.3:
 * Z = sum_i Y_i W_2i takes one all-reduce per MLP).  Here that all-reduce is
 * the one-shot kind of "7.4 推理侧并行" §7.4.2, optimisation 2 -- every rank
 * sends its whole partial to every other rank, and every rank adds them up
 * itself -- and it is fused into the second projection: as soon as the CTAs
 * of an output tile have added their split-K pieces (a thread-block cluster,
 * through distributed shared memory), they store the tile's bf16 partial
 * straight into every rank's exchange buffer (plain stores; over NVLink for a
 * peer), publish it with a flag, wait for the same tile from every rank and
 * add the ranks in rank order.  No library collective runs.
 *
 * Size of one rank's exchange buffer, for the handle's tp_degree, max_tokens
 * and d_out.  Each rank allocates one on its own GPU, zeroes it once before
 * the first call, and makes it reachable from every other rank (for example
 * with tp_mlp_ipc_get_handle / tp_mlp_ipc_open_handle).
 */
size_t tp_mlp_xgpu_comm_bytes(tp_mlp_t handle);

/*
 * One forward of ranks rank0 .. rank0 + nranks - 1 of the handle's tp_degree:
 *   outs[i] = sum_{r < tp_degree} act(x @ A_r) @ B_r        (for every local i)
 *   handle     the whole MLP (d_model, d_ff, d_out, tp_degree, act; bf16),
 *              with a workspace; f_s = d_ff / tp_degree must be a multiple of 64
 *   rank0, nranks  the ranks this call runs: one per process and GPU
 *              (nranks = 1), or every rank at once on one GPU (rank0 = 0,
 *              nranks = tp_degree; a single launch then runs all ranks, which
 *              is how one GPU checks the exchange)
 *   x          device, tokens x d_model (the same on every rank)
 *   A_local, B_local  host arrays of nranks device pointers: the local ranks'
 *              shards, laid out as for tp_mlp_forward
 *   comm       host array of tp_degree pointers: comm[r] is rank r's exchange
 *              buffer as this process sees it (its own, or a peer's mapping)
 *   outs       host array of nranks device pointers, tokens x d_out each
 * Every rank must make the same calls with the same token counts, in the same
 * order, on one stream each.  The call count is kept in the exchange buffers
 * (zeroed once before the first call), so the calls may be captured in a CUDA
 * graph and replayed -- the pages ask this of a custom all-reduce ("7.4 推理侧
 * 并行" §7.4.2).  1 <= tokens <= min(max_tokens, 128) (TP_MLP_ERR_SHAPE);
 * tokens == 0 launches nothing.  TP_MLP_ERR_UNSUPPORTED if
 * the GPU cannot hold every CTA of the exchange at once.  A rank that waits
 * too long for another gives up (bounded wait), and tp_mlp_get_device_status
 * then reports TP_MLP_ERR_TIMEOUT.
 */
int tp_mlp_xgpu_forward(tp_mlp_t handle, int rank0, int nranks, const void *x, int tokens,
                        const void *const *A_local, const void *const *B_local, void *const *comm,
                        void *const *outs, tp_mlp_stream_t stream);

/*
 * The sequence-parallel form of the same step ("7.4 推理侧并行" §7.4.2,
 * optimisation 3): outside the MLP the activations are split by token rows,
 * so the all-reduce becomes an all-gather before the first projection and a
 * reduce-scatter after the second, and each is overlapped with its GEMM.
 *   x_local  host array of nranks device pointers: local rank i's own token
 *            rows, tokens / tp_degree of them (rank r owns rows
 *            [r * tokens / tp_degree, (r + 1) * tokens / tp_degree))
 *   tokens   the total number of token rows, a multiple of tp_degree
 *   outs     host array of nranks device pointers: local rank i's rows of the
 *            output, tokens / tp_degree x d_out each
 * A small kernel first stores each rank's rows into every rank's exchange
 * buffer and counts itself in there; the first projection streams its
 * weights at once and reads X only when every rank's rows have arrived.  The
 * second projection's exchange sends each output row only to the rank that
 * owns it, which adds the ranks' rows (in rank order) and writes its own.
 * Other arguments, requirements and errors as tp_mlp_xgpu_forward; the two
 * calls may be mixed on the same exchange buffers.
 */
int tp_mlp_xgpu_sp_forward(tp_mlp_t handle, int rank0, int nranks, const void *const *x_local, int tokens,
                           const void *const *A_local, const void *const *B_local, void *const *comm,
                           void *const *outs, tp_mlp_stream_t stream);

/*
 * CUDA IPC helpers for the exchange buffers (no counterpart in the pages).
 * get_handle: a 64-byte handle for the device allocation holding dev_ptr, and
 * dev_ptr's offset inside it.  open_handle (in another process): map that
 * allocation and return the same address there.  close_handle: unmap it.
 * TP_MLP_ERR_CUDA if the runtime refuses (for example memory not from
 * cudaMalloc, or a handle opened in the process that made it).
 */
int tp_mlp_ipc_get_handle(const void *dev_ptr, void *handle, size_t *offset);
int tp_mlp_ipc_open_handle(const void *handle, size_t offset, void **dev_ptr);
int tp_mlp_ipc_close_handle(void *dev_ptr, size_t offset);

/*
 * Copy `bytes` bytes from src to dst on `stream`, for a step's host<->device
 * transfers (no counterpart in the pages, which count a decode step's fixed
 * costs per launch, "7.4 推理侧并行" §7.4.2: a decode step's input and output
 * are a few kilobytes, so the transfer's setup, not its bytes, is what costs).
 * Up to 1 MiB the copy is a library kernel that reads or writes the host side
 * directly over the bus, so it needs no copy-engine setup, can be captured in
 * a CUDA graph with the forward, and hands over to the next library kernel by
 * programmatic dependent launch; larger copies go to the copy engine
 * (cudaMemcpyAsync).
 *
 *   dst, src  each either device memory of the current device or page-locked
 *             host memory mapped into its address space (cudaHostAlloc /
 *             cudaMallocHost, or cudaHostRegister with mapping, under unified
 *             addressing); 16-byte aligned; each inside one allocation of at
 *             least `bytes` from the pointer on.  The two ranges must not
 *             overlap.
 *   bytes     any count; 0 is a no-op.
 * Errors (nothing is launched): TP_MLP_ERR_INVALID_ARG for a null pointer,
 * memory CUDA does not know (pageable host memory), host memory not mapped
 * for this device, device memory of another device or context, or
 * overlapping ranges; TP_MLP_ERR_ALIGNMENT; TP_MLP_ERR_SHAPE if `bytes` runs
 * past the allocation.
 * Asynchronous on `stream`: a host destination holds the data once the
 * stream's work up to this call has completed.
 */
int tp_mlp_copy_async(void *dst, const void *src, size_t bytes, tp_mlp_stream_t stream);

/* Human-readable name of a status code (static string; no counterpart in the pages). */
const char *tp_mlp_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* TP_MLP_H */
