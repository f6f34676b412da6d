/*
 * tspmlp.h -- C ABI of libtspmlp: the column-then-row sharded transformer MLP
 * on one NVIDIA B200 (sm_100a).
 *
 * The operation.  For token rows X[n][d_model]:
 *
 *   plain  (TSP_ACT_GELU):   Y = GeLU(X.A).B                     GeLU(z) = z Phi(z)
 *   gated  (TSP_ACT_SWIGLU): Y = (SiLU(X.W_gate) (*) (X.W_up)).W_down
 *
 * "Tensor Parallelism: Splitting the Math" (section "Why the column-then-row
 * split -- and what happens in attention") defines the plain block and shows
 * that splitting A by columns and B by rows lets every shard apply the
 * nonlinearity to values it fully owns; steps 2-6 of its two-GPU walk-through
 * ("One transformer MLP, split across two GPUs") define the shards and the sum
 * of their partial outputs.  "Folding Tensor and Sequence Parallelism for
 * Memory-Efficient Transformer Training & Inference" (Abstract) gives the
 * gated form and the folded schedule in which weight shards circulate in a
 * ring while each sequence shard accumulates its partial outputs locally.
 *
 * Here the P shards are logical: shard w owns hidden columns
 * [w d_ff/P, (w+1) d_ff/P) of A (= W_gate) and W_up and the same rows of
 * B (= W_down).  All shards run on the calling GPU; each shard's partial output
 * is added into an fp32 accumulator in place, in shard order (no collective).
 *
 * Layout and types.  Every matrix is dense and row-major, as in the pages'
 * product X.A:
 *   X[n][d_model], A = W_gate[d_model][d_ff], W_up[d_model][d_ff],
 *   B = W_down[d_ff][d_model], Y[n][d_model], dY[n][d_model].
 * (torch.nn.Linear stores the transpose of each weight.)
 * TSP_DT_BF16: X, weights, dY, Y and dX are bfloat16; every product
 *   accumulates in fp32; the hidden activation is rounded to bf16 once before
 *   the down projection; in the backward, the activation's derivative factors
 *   and dG (dU) are rounded to bf16 before their products; weight gradients
 *   are fp32.
 * TSP_DT_F32: everything fp32 (no TF32), plain or gated.
 *
 * Ownership.  The caller owns every buffer.  Pointers are device pointers on
 * the current device unless a function says otherwise.  The library keeps no
 * state between calls apart from per-device kernel attributes set once and a
 * device-side error word.  Calls that take no workspace allocate their scratch
 * with cudaMallocAsync on `stream` and free it on the same stream.
 *
 * Errors.  Arguments are validated before anything is launched; a bad call
 * returns a status and touches nothing.  Kernels bound every wait on the GPU
 * (about two seconds); a wait that runs out sets the device error word and the
 * kernel returns early, so a later tsp_poll_device_error() reports
 * TSP_ERR_TIMEOUT instead of hanging (TSP_ERR_RANGE: see TSP attention).  All
 * calls are asynchronous on `stream`.
 */
#ifndef TSPMLP_H
#define TSPMLP_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TSP_API __attribute__((visibility("default")))
#else
#define TSP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (layout-compatible with cudaStream_t); NULL is the legacy
 * default stream. */
typedef struct CUstream_st* tsp_stream_t;

typedef enum {
    TSP_OK = 0,
    TSP_ERR_INVALID_ARG = 1,       /* NULL pointer, non-positive size, bad enum, aliasing */
    TSP_ERR_UNSUPPORTED_SHAPE = 2, /* d_ff % P, alignment or size limits (see each call) */
    TSP_ERR_ARCH = 3,              /* current device is not compute capability 10.0 */
    TSP_ERR_CUDA = 4,              /* a CUDA runtime call or launch failed */
    TSP_ERR_TIMEOUT = 5,           /* a bounded device-side wait ran out */
    TSP_ERR_WORKSPACE = 6,         /* workspace NULL or smaller than tsp_mlp_workspace_size */
    TSP_ERR_SCRATCH_LIMIT = 7,     /* needs more scratch than tsp_mlp_forward_noalloc holds */
    TSP_ERR_RANGE = 8              /* reported by tsp_poll_device_error: an fp16 intermediate
                                    * (tsp_attn_forward's Q or K) exceeded 65504 in magnitude
                                    * and was saturated */
} tsp_status_t;

typedef enum {
    TSP_ACT_GELU = 0,  /* exact erf GeLU: z * (1 + erf(z / sqrt 2)) / 2 */
    TSP_ACT_SWIGLU = 1 /* SiLU(g) * u with SiLU(g) = g / (1 + exp(-g)) */
} tsp_act_t;

typedef enum { TSP_DT_BF16 = 0, TSP_DT_F32 = 1 } tsp_dtype_t;

typedef enum {
    /* Weight-shard schedule: every token meets shard 0, 1, ..., P-1 in order
     * and the partial outputs accumulate in that order (the library picks its
     * fastest measured implementation: TSP_SCHED_SHARD_PASSES for bf16). */
    TSP_SCHED_WEIGHT_SHARDS = 0,
    /* Folded tensor-and-sequence ring: tokens form P equal sequence shards;
     * at ring step t sequence shard s meets weight shard (s + t) mod P, and
     * each sequence shard sums its partial outputs in that ring order.  Needs
     * n % P == 0.  bf16 with (d_ff / P) % 128 == 0: per group of sequence
     * shards (as many as fit 512 MB of hidden activations) one gate/up launch
     * over all d_ff columns and one down projection whose K loop runs over
     * the weight shards in each sequence shard's ring order, summing in
     * tensor memory.  Otherwise: per ring step one gate/up and one down
     * launch, the partial outputs added into an fp32 accumulator in place. */
    TSP_SCHED_TSP_RING = 1,
    /* Weight-shard schedule as separate passes: per chunk of whole shards
     * (as many as fit a 512 MB hidden buffer) one gate/up launch and one
     * down-projection launch.  With several chunks each partial output is
     * added into an fp32 [n][d_model] accumulator in place; with one chunk
     * the down projection's tensor-memory accumulator sums the shards in
     * order and writes Y directly. */
    TSP_SCHED_SHARD_PASSES = 2,
    /* Weight-shard schedule as one persistent launch (bf16): per block of 128
     * tokens the hidden activations go to a ring of row-block slots and the
     * down projection's fp32 tensor-memory accumulator takes the shards'
     * partial outputs in shard order.  Needs no [n][d_model] accumulator. */
    TSP_SCHED_FUSED = 3,
    /* The TSP ring as one persistent launch (bf16): as TSP_SCHED_FUSED, each
     * sequence shard's K loop over the hidden units starting at its own weight
     * shard.  Needs n % P == 0 and (d_ff / P) % 64 == 0. */
    TSP_SCHED_TSP_RING_FUSED = 4,
    /* TSP_SCHED_SHARD_PASSES with all passes in one persistent launch on CTA
     * pairs (bf16): chunk c's down-projection tiles run alongside chunk c+1's
     * gate/up tiles, ordered by per-row-block counters.  Needs
     * (d_ff / P) % 64 == 0 and at most 32 chunks. */
    TSP_SCHED_SHARD_PASSES_FUSED = 5
} tsp_sched_t;

/* Forward pass, bf16, weight-shard schedule.
 * Defined by "Tensor Parallelism: Splitting the Math", walk-through "One
 * transformer MLP, split across two GPUs", steps 2-6 (A split by columns, the
 * nonlinearity on each shard's own hidden columns, B split by rows to match,
 * the shards' partial outputs summed into the exact unsharded Y), and by
 * "Folding Tensor and Sequence Parallelism ...", Abstract (the gated form;
 * partial outputs accumulate locally instead of through a collective).
 *   X        [n_tokens][d_model] bf16
 *   W_gate   [d_model][d_ff] bf16 -- A for TSP_ACT_GELU
 *   W_up     [d_model][d_ff] bf16 -- must be NULL for TSP_ACT_GELU
 *   W_down   [d_ff][d_model] bf16 -- B for TSP_ACT_GELU
 *   Y        [n_tokens][d_model] bf16, written (must not overlap any input)
 * Requirements: n_tokens, d_model, d_ff > 0; 1 <= P <= 4096; d_ff % P == 0;
 * d_model % 8 == 0 and (d_ff / P) % 8 == 0 (16-byte rows for TMA);
 * every pointer 16-byte aligned.  Scratch: cudaMallocAsync on `stream`. */
TSP_API tsp_status_t tsp_mlp_forward(const void* X, const void* W_gate, const void* W_up,
                             const void* W_down, int64_t n_tokens, int64_t d_model,
                             int64_t d_ff, int P, tsp_act_t act, void* Y, tsp_stream_t stream);

/* Forward pass with every option and a caller workspace.
 * Defined as tsp_mlp_forward ("Tensor Parallelism: Splitting the Math",
 * walk-through steps 2-6); the TSP_SCHED_TSP_RING schedules follow "Folding
 * Tensor and Sequence Parallelism ...", Abstract (weight shards circulate in
 * a ring while each sequence shard accumulates its partial outputs locally).
 *   dtype      TSP_DT_BF16 (tensor cores) or TSP_DT_F32 (fp32 FMA; any sizes)
 *   sched      a tsp_sched_t (the ring schedules need n % P == 0; the fused
 *              ones bf16; TSP_SCHED_TSP_RING_FUSED also (d_ff / P) % 64 == 0)
 *   workspace  256-byte aligned device buffer, not overlapping any argument.
 *              tsp_mlp_workspace_size() gives the preferred size.  For bf16 a
 *              smaller workspace is accepted: the schedule then runs fewer
 *              token rows (or sequence shards) a launch while 256 rows of all
 *              d_ff hidden units still fit, and below that narrower hidden
 *              chunks whose partial outputs go through an [n][d_model] fp32
 *              accumulator, down to one 128-column chunk (one sequence shard)
 *              plus that accumulator; below that the call returns
 *              TSP_ERR_WORKSPACE.  fp32 needs the preferred size.
 * Other arguments as tsp_mlp_forward. */
TSP_API tsp_status_t tsp_mlp_forward_ex(const void* X, const void* W_gate, const void* W_up,
                                const void* W_down, int64_t n_tokens, int64_t d_model,
                                int64_t d_ff, int P, tsp_act_t act, tsp_dtype_t dtype,
                                tsp_sched_t sched, void* Y, void* workspace,
                                size_t workspace_bytes, tsp_stream_t stream);

/* Forward pass that allocates nothing (bf16, TSP_SCHED_FUSED).  The
 * pages have no counterpart: this entry point exists for callers that cannot
 * call cudaMalloc or cudaMallocAsync -- code running inside a host engine or
 * plugin whose device memory is planned up front and must not grow, and code
 * for which an allocation is unacceptable because it may synchronise the
 * device and stall other streams.
 * The scratch it needs (the ring of hidden-activation slots, 128 x d_ff bf16
 * each, and the per-row-block counters of the fused schedule) lives in a
 * static device array of TSP_NOALLOC_SCRATCH_BYTES inside the library; every
 * GPU that loads the library holds that array until the process exits.  The
 * ring is sized to fit the array; problems whose narrowest ring (three slots,
 * or one per block of 128 tokens when there are fewer) does not fit -- d_ff
 * above about 43,000 -- return TSP_ERR_SCRATCH_LIMIT before anything is
 * launched.
 * Arguments, requirements and results are those of tsp_mlp_forward.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  If it is also the first call into this library on that device,
 * CUDA's lazy module loading may load the library's device code there at that
 * moment -- the static array, the other device globals and the kernels --
 * which allocates device memory and can synchronise.  Callers with a fixed
 * memory plan should therefore make one call (any problem size) during their
 * set-up; later calls allocate nothing.  All calls on a device share the one array and it keeps the last
 * call's contents; calls whose executions overlap on the GPU (different
 * streams, or other threads) race on it and must be serialised by the caller. */
#define TSP_NOALLOC_SCRATCH_BYTES (32u << 20)
TSP_API tsp_status_t tsp_mlp_forward_noalloc(const void* X, const void* W_gate, const void* W_up,
                                             const void* W_down, int64_t n_tokens,
                                             int64_t d_model, int64_t d_ff, int P, tsp_act_t act,
                                             void* Y, tsp_stream_t stream);

/* Backward pass, bf16, weight-shard schedule, for upstream gradient dY.
 * "Tensor Parallelism: Splitting the Math", its paragraph counting the
 * communication (the forward's pattern happens again in the backward pass):
 * the gradients are the exact derivatives of the forward of tsp_mlp_forward,
 * computed shard by shard with the input gradient's partials summed locally
 * like Y's.  With G = X.W_gate, U = X.W_up, dH = dY.W_down^T:
 *   SwiGLU: dU = dH SiLU(G), dG = dH U SiLU'(G);  GeLU: dG = dH GeLU'(G);
 *   dX = dG.W_gate^T (+ dU.W_up^T), dW_gate = X^T.dG, dW_up = X^T.dU,
 *   dW_down = H^T.dY.
 *   dY        [n_tokens][d_model] bf16
 *   dX        [n_tokens][d_model] bf16, written
 *   dW_gate   [d_model][d_ff] fp32, written (dA for TSP_ACT_GELU)
 *   dW_up     [d_model][d_ff] fp32, written; NULL for TSP_ACT_GELU
 *   dW_down   [d_ff][d_model] fp32, written (dB for TSP_ACT_GELU)
 * The hidden activations are recomputed from X (no forward state is kept).
 * Requirements as tsp_mlp_forward; outputs must not overlap inputs or each
 * other.  Scratch: cudaMallocAsync on `stream`. */
TSP_API tsp_status_t tsp_mlp_backward(const void* X, const void* W_gate, const void* W_up,
                              const void* W_down, const void* dY, int64_t n_tokens,
                              int64_t d_model, int64_t d_ff, int P, tsp_act_t act, void* dX,
                              float* dW_gate, float* dW_up, float* dW_down,
                              tsp_stream_t stream);

/* Backward with a caller workspace (bf16 only; weight-shard schedule).
 * Defined as tsp_mlp_backward ("Tensor Parallelism: Splitting the Math",
 * paragraph counting the communication: the same pattern in the backward
 * pass).  As for
 * tsp_mlp_forward_ex, a workspace smaller than the preferred size is accepted
 * down to one 128-column chunk of the hidden buffers plus the fp32 dX
 * accumulator. */
TSP_API tsp_status_t tsp_mlp_backward_ex(const void* X, const void* W_gate, const void* W_up,
                                 const void* W_down, const void* dY, int64_t n_tokens,
                                 int64_t d_model, int64_t d_ff, int P, tsp_act_t act, void* dX,
                                 float* dW_gate, float* dW_up, float* dW_down, void* workspace,
                                 size_t workspace_bytes, tsp_stream_t stream);

/* Preferred bytes of workspace of the _ex calls for these arguments (backward
 * != 0 for tsp_mlp_backward_ex): hidden chunks sized to stay resident in L2.
 * Writes *bytes; no device is touched. */
TSP_API tsp_status_t tsp_mlp_workspace_size(int64_t n_tokens, int64_t d_model, int64_t d_ff, int P,
                                    tsp_act_t act, tsp_dtype_t dtype, tsp_sched_t sched,
                                    int backward, size_t* bytes);

/* Training: a forward that keeps its activations, and a backward that uses
 * them instead of recomputing the gate/up projection from X.
 *
 * The backward of the block needs, at every hidden unit, dH = dY.W_down^T
 * times the derivative of the activation ("Folding Tensor and Sequence
 * Parallelism ...", Abstract: the gated form; "Tensor Parallelism: Splitting
 * the Math": the plain block).  tsp_mlp_forward_train writes, besides Y, the
 * activations and the activation's derivative factors at every hidden unit:
 *   H  = h(X)                    bf16 [n_tokens][d_ff]  (as the forward's)
 *   S1 = SiLU(G)  (SwiGLU)  or  GeLU'(Z) (GeLU)          bf16 [n_tokens][d_ff]
 *   S2 = U SiLU'(G)  (SwiGLU only)                       bf16 [n_tokens][d_ff]
 * with G = X.W_gate, U = X.W_up, Z = X.A (fp32 accumulations), SiLU'(g) =
 * s (1 + g (1 - s)), s = sigmoid(g), GeLU'(z) = Phi(z) + z phi(z), each factor
 * evaluated in fp32 and rounded to bf16; and tsp_mlp_backward_saved forms
 * dU = dH S1 and dG = dH S2 (GeLU: dG = dH S1) in the epilogue of the dH
 * product, so dH is never stored.  tsp_mlp_backward_ex evaluates and rounds
 * the factors the same way from its recomputed G and U, so dX, dW_gate and
 * dW_up are bit-identical to its results; dW_down uses the forward's H.
 *
 * The saved buffer is opaque to the caller: H (row-major), then S1, then S2
 * (each over whole 32-row blocks, in the layout the two epilogues access
 * fastest), then 16 MB of scratch the training forward's down projection uses
 * as the forward's uses its workspace, every region 256-byte aligned;
 * tsp_mlp_saved_size gives its size.  It must be 256-byte
 * aligned and overlap no other argument; the backward only reads it. */
TSP_API tsp_status_t tsp_mlp_saved_size(int64_t n_tokens, int64_t d_model, int64_t d_ff, int P,
                                        tsp_act_t act, size_t* bytes);

/* Forward pass (bf16, weight-shard schedule) that also fills `saved`.  Y as
 * tsp_mlp_forward (bit-identical to it); requirements as tsp_mlp_forward.  H
 * lives in `saved`, so no workspace is needed: token rows run in groups of
 * at most 128 MB of H (as the pass schedule's row groups), each one gate/up
 * launch writing H, S1 (S2) and one down projection reading H. */
TSP_API tsp_status_t tsp_mlp_forward_train(const void* X, const void* W_gate, const void* W_up,
                                           const void* W_down, int64_t n_tokens, int64_t d_model,
                                           int64_t d_ff, int P, tsp_act_t act, void* Y,
                                           void* saved, size_t saved_bytes, tsp_stream_t stream);

/* Preferred workspace bytes of tsp_mlp_backward_saved: the dG (dU) chunk
 * buffers and, with more than one chunk, the fp32 dX accumulator. */
TSP_API tsp_status_t tsp_mlp_backward_saved_workspace_size(int64_t n_tokens, int64_t d_model,
                                                           int64_t d_ff, int P, tsp_act_t act,
                                                           size_t* bytes);

/* Backward pass from the activations tsp_mlp_forward_train saved for the
 * same X and weights.  Outputs, requirements and the smaller-workspace rule
 * as tsp_mlp_backward_ex.  Per hidden chunk: the dH product with the factors
 * applied (dG, dU to the workspace), dW_down = H^T.dY from the saved H,
 * dW_gate (dW_up) = X^T.dG (dU), and dX (+)= dG.W_gate^T (+ dU.W_up^T). */
TSP_API tsp_status_t tsp_mlp_backward_saved(const void* X, const void* W_gate, const void* W_up,
                                            const void* W_down, const void* dY, const void* saved,
                                            size_t saved_bytes, int64_t n_tokens, int64_t d_model,
                                            int64_t d_ff, int P, tsp_act_t act, void* dX,
                                            float* dW_gate, float* dW_up, float* dW_down,
                                            void* workspace, size_t workspace_bytes,
                                            tsp_stream_t stream);

/* ---------------------------------------------------------------------------
 * TSP attention: multi-head self-attention under the attention schedule of
 * "Folding Tensor and Sequence Parallelism for Memory-Efficient Transformer
 * Training & Inference", Abstract -- every rank holds one sequence shard of
 * tokens, the ranks iterate over the broadcast parameter shards (groups of
 * heads), and each reconstructs the whole context through a sequence-wise
 * key/value exchange.  The head split itself is "Tensor Parallelism:
 * Splitting the Math", section "Why the column-then-row split -- and what
 * happens in attention": heads are independent, so W_q, W_k, W_v split by
 * columns and W_o by rows, with one sum of the partial outputs.
 *
 *   Q = X.W_q, K = X.W_k, V = X.W_v                 (head h: columns [128 h, 128 h + 128))
 *   O_h = softmax(Q_h K_h^T / sqrt(128) + M) V_h    (M = -inf above the diagonal when causal)
 *   Y = [O_0 | O_1 | ...] . W_o
 *
 * Here the P sequence shards (tokens [s n/P, (s+1) n/P)) and the P parameter
 * shards (heads [w H/P, (w+1) H/P)) are logical.  The queries of sequence
 * shard s visit the key/value shards in ring order s, s+1, ..., s-1 (mod P),
 * 128 keys a block, each block merged into a running row maximum, row sum and
 * weighted value sum in fp32 (tensor memory), so the result is the exact
 * softmax up to rounding for every P.  With the causal mask the shards after
 * s hold only future keys and are skipped.  Y_s accumulates the parameter
 * shards' partial outputs O_{s,w} . W_o[rows of w] in shard order, in fp32
 * tensor memory, rounded to bf16 once.
 *
 * Layout and types: X, Y, Q, K, V, O are [n_tokens][d_model] row-major,
 * W_q, W_k, W_v, W_o are [d_model][d_model] bf16 row-major (torch.nn.Linear
 * stores the transposes).  Head dimension 128: d_model = 128 n_heads.
 * X, Y, V, O and the weights are bf16.  tsp_attn_core takes bf16 Q and K;
 * tsp_attn_forward keeps its own Q and K in fp16 (three more mantissa bits
 * where the scores' rounding matters most): a projected value above 65504 in
 * magnitude saturates and the next tsp_poll_device_error() returns
 * TSP_ERR_RANGE.  The probabilities are rounded to bf16 before P.V; all
 * products accumulate in fp32.
 *
 * Requirements: n_tokens > 0, n_tokens % P == 0, n_tokens <= 2^28,
 * d_model == 128 n_heads, every pointer 16-byte aligned, outputs overlapping
 * no input.  Errors as for the MLP calls. */

/* The attention core alone: O from Q, K, V (all [n_tokens][d_model] bf16),
 * sequence shard s's queries over the key/value shards in ring order.
 * causal != 0 applies the causal mask.  Allocates nothing. */
TSP_API tsp_status_t tsp_attn_core(const void* Q, const void* K, const void* V, int64_t n_tokens,
                                   int64_t d_model, int n_heads, int P, int causal, void* O,
                                   tsp_stream_t stream);

/* Workspace bytes of tsp_attn_forward: Q, K (fp16), V and O (bf16),
 * [n_tokens][d_model] each, 256-byte aligned.  Needs n_heads % P == 0.  No device is
 * touched. */
TSP_API tsp_status_t tsp_attn_workspace_size(int64_t n_tokens, int64_t d_model, int n_heads, int P,
                                             size_t* bytes);

/* The attention block, Y = attention(X) . W_o, under the TSP schedule: the
 * three projections (every parameter shard's columns for every sequence
 * shard's tokens, one launch each), the attention core as tsp_attn_core, and
 * the output projection summing the parameter shards' partial outputs in
 * order.  Needs n_heads % P == 0 and a workspace of tsp_attn_workspace_size
 * bytes (256-byte aligned, overlapping no argument). */
TSP_API tsp_status_t tsp_attn_forward(const void* X, const void* W_q, const void* W_k,
                                      const void* W_v, const void* W_o, int64_t n_tokens,
                                      int64_t d_model, int n_heads, int P, int causal, void* Y,
                                      void* workspace, size_t workspace_bytes,
                                      tsp_stream_t stream);

/* A static, human-readable name for a status. */
TSP_API const char* tsp_status_string(tsp_status_t status);

/* Per-kernel tracing.  While enabled, every kernel the library launches is
 * bracketed by two CUDA events recorded on the stream it is launched on; the
 * events are kept until tsp_trace_collect().  Process-wide; off by default. */
typedef struct {
    const char* name;  /* static string, e.g. "fwd_hidden_swiglu" */
    int64_t launches;  /* launches since the last reset */
    double total_ms;   /* sum of their event-timed durations */
} tsp_kernel_stat_t;

TSP_API tsp_status_t tsp_trace_enable(int enable);

/* Waits for every traced launch to finish, folds them into per-kernel totals
 * and copies up to `capacity` entries to `stats` (`*count` = entries filled).
 * Totals accumulate until tsp_trace_reset(). */
TSP_API tsp_status_t tsp_trace_collect(tsp_kernel_stat_t* stats, int capacity, int* count);

/* Drops all totals and pending events. */
TSP_API tsp_status_t tsp_trace_reset(void);

/* Failure-detection self-test; nothing faults, traps or hangs.
 *   mode 0: a one-thread kernel waits on an mbarrier that nothing arrives on,
 *           through the bounded wait every kernel of the library uses.
 *   mode 1: one tile of the gate/up kernel whose producer arms its first stage
 *           but leaves out that stage's loads, so the tensor-core pipeline
 *           itself must give up: every role leaves through the abort path,
 *           loads in flight are waited for, tensor memory is freed.
 * Either kernel returns after about two seconds; the call returns TSP_OK once
 * it is launched, and the following tsp_poll_device_error() reports
 * TSP_ERR_TIMEOUT (and clears it).  Mode 1 allocates and frees its small
 * buffers with cudaMallocAsync / cudaFreeAsync on `stream`. */
TSP_API tsp_status_t tsp_selftest_timeout(int mode, tsp_stream_t stream);

/* Synchronises `stream`, then reads and clears the current device's error
 * word: TSP_OK, TSP_ERR_TIMEOUT if a kernel gave up waiting, TSP_ERR_RANGE if
 * an fp16 intermediate saturated (and no wait ran out), TSP_ERR_CUDA if the
 * stream reported an error. */
TSP_API tsp_status_t tsp_poll_device_error(tsp_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TSPMLP_H */
