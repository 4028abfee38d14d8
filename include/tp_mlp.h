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
    TP_MLP_ERR_TIMEOUT = 6,      /* reserved: a bounded device-side wait ran out       */
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
    TP_MLP_PLAN_TC_WIDE256 = 6 /* tcgen05, tiles of 256 tokens x 256 weight rows      */
} tp_mlp_plan;

/*
 * Create a handle for one MLP shape.
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

/* Free the handle (host memory).  NULL is accepted. */
int tp_mlp_destroy(tp_mlp_t handle);

/*
 * Device workspace (bytes) the forward / partials / packed calls need for
 * `tokens` tokens (0 <= tokens <= max_tokens).  It holds the intermediate
 * activation H (tokens x d_ff, dtype) and split-K scratch.  Returns 0 for an
 * invalid handle or token count.
 */
size_t tp_mlp_workspace_bytes(tp_mlp_t handle, int tokens);

/*
 * Give the handle a device workspace of `bytes` bytes (owned by the caller,
 * kept until replaced or the handle is destroyed).  Zeroes the split-K
 * counters inside it synchronously (cudaMemset).  bytes must be at least
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
 * Per-rank partials without the final sum: partials[i] = act(x @ A_i) @ B_i,
 * fp32, laid out tp_degree x tokens x d_out (device).  Other arguments as
 * tp_mlp_forward.  Summing them over i gives the forward's result (before
 * rounding to the output dtype).
 */
int tp_mlp_partials(tp_mlp_t handle, const void *x, int tokens, const void *const *A_shards,
                    const void *const *B_shards, int tp_degree, int act, float *partials,
                    tp_mlp_stream_t stream);

/*
 * Size in bytes of the packed weight buffer (the shard-layout packer's output).
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
 * tp_mlp_packed_bytes bytes).  A bit-exact copy in a new order.  The handle's
 * tp_degree fixes how many pointers each array holds. */
int tp_mlp_pack(tp_mlp_t handle, const void *const *A_shards, const void *const *B_shards,
                void *packed, tp_mlp_stream_t stream);

/* Inverse of tp_mlp_pack: write the shards back from `packed` (bit-exact). */
int tp_mlp_unpack(tp_mlp_t handle, const void *packed, void *const *A_shards,
                  void *const *B_shards, tp_mlp_stream_t stream);

/*
 * Forward pass on packed weights (the fast path; weights are packed once).
 *   x device tokens x d_model, out device tokens x d_out, packed from
 *   tp_mlp_pack.  Same result as tp_mlp_forward up to fp32 summation order.
 */
int tp_mlp_forward_packed(tp_mlp_t handle, const void *x, int tokens, const void *packed,
                          void *out, tp_mlp_stream_t stream);

/* Force a kernel family (tp_mlp_plan) for later forwards; AUTO restores the
 * library's choice.  A forced plan that cannot serve a call returns
 * TP_MLP_ERR_UNSUPPORTED from that call. */
int tp_mlp_set_plan(tp_mlp_t handle, int plan);

/*
 * How the skinny tensor-core tiling (TP_MLP_PLAN_TC_SKINNY) finishes a weight
 * tile whose K loop is split between CTAs.  Both add the fp32 partial slots in
 * the same fixed order, so they give identical results; they differ in speed.
 */
typedef enum {
    TP_MLP_SPLITK_AUTO = 0,      /* by the size of the partials (default)            */
    TP_MLP_SPLITK_IN_KERNEL = 1, /* the last CTA to finish its share adds the slots   */
    TP_MLP_SPLITK_SEPARATE = 2   /* a reduction kernel behind each GEMM adds them,
                                    spread over the whole GPU                        */
} tp_mlp_splitk;

/* Choose the split-tile finish (tp_mlp_splitk) for later forwards.  Returns
 * TP_MLP_ERR_INVALID_ARG for another value.  Other plans ignore it. */
int tp_mlp_set_splitk(tp_mlp_t handle, int mode);

/*
 * Timing hook: with n > 0, later forward / forward_packed / partials calls
 * record events[0] on their stream before their first kernel, events[1] after
 * the first projection's kernels and events[2] after the second projection's
 * (events beyond events[2] are not recorded).  The events are caller-owned cudaEvent_t handles (created with
 * timing enabled) and must stay valid while calls use them; n = 0 (or
 * events = NULL) turns the hook off.  At most 8 events.
 */
int tp_mlp_set_profile_events(tp_mlp_t handle, void *const *events, int n);

/*
 * Device-side status of the work issued so far on this handle's workspace:
 * synchronises the device, returns TP_MLP_ERR_TIMEOUT if a kernel gave up a
 * bounded internal wait (its results are then invalid) and clears the flag,
 * TP_MLP_OK otherwise.  Needs a workspace.
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
 * forward / partials call on this handle; -1 before the first. */
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
 * array: order them on one stream or with events.
 * Errors: TP_MLP_ERR_WORKSPACE if this shape needs more scratch than the
 * 8 MiB array holds (nothing is launched); TP_MLP_ERR_UNSUPPORTED for shapes
 * the GEMV kernels do not take (d_model or d_ff not a multiple of 8);
 * otherwise as tp_mlp_forward_packed.  tokens == 0 is a no-op.
 */
int tp_mlp_decode_forward_static(int d_model, int d_ff, int d_out, int tp_degree, int act,
                                 const void *x, int tokens, const void *packed, void *out,
                                 tp_mlp_stream_t stream);

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

/* Human-readable name of a status code (static string). */
const char *tp_mlp_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* TP_MLP_H */
