/*
 * zero.h -- C ABI of libzero: the ZeRO stage 1/2/3 partitioned mixed-precision
 * Adam step on one B200, with Nd data-parallel ranks emulated as virtual ranks.
 *
 * The operation (pages cited by title and section):
 *   [P1] "Your 7.5B model's weights fit in 15 GB. Training state was 120 GB per
 *        GPU" (blog.teqners.com) -- "Where 16 bytes per parameter comes from",
 *        "Why you can't just delete the fp32 copies", "The replication nobody
 *        questioned" (stage table), "The part that sounds too good:
 *        communication".
 *   [P2] "Engine Room" ch. 10, "ZeRO and the Memory Tricks" -- "The Mathematics"
 *        (M_states(p, Nd)), "What It Enabled" (stage table).
 *   [P3] "DeepSpeed ZeRO: account for every training state" -- "What each ZeRO
 *        stage partitions", "Partitioned parameters still have to participate
 *        in computation", "Check your understanding".
 *
 * One step, for every element i owned by rank r ([P1] "communication": each
 * rank reduce-scatters the gradients, updates only its slice, and the ranks
 * all-gather the updated fp16 parameters):
 *   s   = fp32(g_0[i]) + fp32(g_1[i]) + ... + fp32(g_{Nd-1}[i])  (rank order, fp32)
 *   g   = s * inv_scale,  inv_scale = (float)(1.0 / (double)loss_scale)
 *   skip the whole step if any g over all partitions is inf or NaN
 *   m   = b1*m + (1-b1)*g ;  v = b2*v + (1-b2)*(g*g)
 *   u   = (m / bc1) / (sqrt(v / bc2) + eps),  bc_k = (float)(1 - beta_k^t)
 *   w   = w - lr*(u + wd*w)                              (fp32 master;
 *         wd = 0 on tensors flagged ZERO_TENSOR_NO_DECAY)
 *   p16 = fp16(w), round to nearest even, written to every rank's replica
 *         (stage 1/2) or to rank r's fp16 shard (stage 3).
 * Each binary32 operation is one IEEE-rounded operation in that order (no FMA
 * contraction, no flush to zero). Stage 3 adds zero_gather_layer, the
 * on-demand gather of one layer's full fp16 weights ([P1] "communication",
 * stage 3; [P3] "Partitioned parameters still have to participate").
 *
 * A handle with rank_view = r acts as rank r alone. With one process per GPU
 * it is rank r of a real job: on stage 1/2 with view_outputs = Nd its step
 * reads partition r of every rank's gradient and writes partition r into
 * every rank's parameter buffer; on stage 3 it keeps shard r and
 * zero_gather_layer_ranks gathers layers from every rank's shard; in both
 * cases the ranks agree on overflow through zero_flag_words. The other
 * ranks' buffers are mapped with zero_peer.h.
 *
 * Conventions for every call:
 *   - fp16 values are IEEE binary16 bit patterns (uint16_t).
 *   - "device" pointers are CUDA global-memory addresses on the current device;
 *     every device pointer passed in must be 16-byte aligned (ZERO_ERR_ALIGN).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). All device
 *     work of a call is ordered on it.
 *   - The caller owns and allocates all device memory (workspace, gradients,
 *     parameter buffers, gather output). The library never allocates device
 *     memory; a handle is a small host object freed by zero_destroy.
 *   - Handles are not thread-safe; one handle serves one caller thread.
 */
#ifndef ZERO_H
#define ZERO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes ---- */
#define ZERO_OK 0
#define ZERO_SKIPPED 1          /* informational: overflow, step skipped, state untouched */
#define ZERO_ERR_ARG (-1)       /* invalid argument or configuration */
#define ZERO_ERR_ALIGN (-2)     /* a device pointer is not 16-byte aligned */
#define ZERO_ERR_STAGE (-3)     /* call not valid for this stage (gather on stage 1/2) */
#define ZERO_ERR_WORKSPACE (-4) /* workspace smaller than zero_state_bytes says */
#define ZERO_ERR_CUDA (-5)      /* a CUDA call failed; see zero_last_cuda_error */
#define ZERO_ERR_INTERNAL (-6)  /* internal consistency check failed, or a bounded
                                   wait inside a kernel gave up; the step is then
                                   rolled back like a skipped one */
#define ZERO_ERR_PARTIAL (-7)   /* a bounded wait of the in-place update pass of
                                   ZERO_VARIANT_TWO_PASS_TMA gave up: some elements
                                   of the master (without one: the 16-bit weights),
                                   m, v and the parameters hold this step's values,
                                   the others the previous step's; t did not
                                   advance. Nothing can be rolled back: restore a
                                   saved state with zero_set_state, which rewrites
                                   the parameters too */

/* ---- step variants ---- */
/* One pass: reads the gradients and the current master/m/v, writes the next
 * master/m/v into a second state buffer and the fp16 parameters in place.
 * Commits by switching buffers; on overflow the buffers stay and the fp16
 * parameters are rewritten from the unchanged master (a pure function of it).
 * Moves the minimum (24 + 4 Nd) bytes per element (stage 1/2). */
#define ZERO_VARIANT_FUSED 0
/* Two passes: the reduce pass writes the unscaled fp32 reduced gradient of
 * every partition and the overflow flag; the update pass checks the flag and
 * runs Adam in place. One state buffer; 8 more bytes per element. */
#define ZERO_VARIANT_TWO_PASS 1
/* The fused pass with its loads and stores done by the Tensor Memory
 * Accelerator: tiles of the Nd gradient slices and of master/m/v are staged
 * into shared memory by bulk asynchronous copies while earlier tiles are
 * computed, and results leave by bulk stores. Same arithmetic, bytes and
 * workspace as ZERO_VARIANT_FUSED. Used when Nd <= 16 and every run's state
 * and output indices are in 16-byte phase with its gradient index; otherwise
 * the handle runs the ZERO_VARIANT_FUSED kernel. */
#define ZERO_VARIANT_FUSED_TMA 2
/* The two passes of ZERO_VARIANT_TWO_PASS with their loads done by the Tensor
 * Memory Accelerator (bulk copies of gradient, reduced-gradient, moment and
 * weight tiles into shared memory, as in ZERO_VARIANT_FUSED_TMA); same
 * arithmetic, bytes and workspace as ZERO_VARIANT_TWO_PASS, under the same
 * eligibility rule as ZERO_VARIANT_FUSED_TMA (otherwise the plain two-pass
 * kernels run). Valid with both precisions. The update pass writes in place:
 * should one of its bounded waits give up, the step returns ZERO_ERR_PARTIAL
 * (part of the state is already updated; restore it with zero_set_state). A
 * wait of the reduce pass that gives up is rolled back (ZERO_ERR_INTERNAL):
 * the update pass then writes nothing. */
#define ZERO_VARIANT_TWO_PASS_TMA 3

#define ZERO_MAX_ND 1024

/* ---- precision of the parameters and gradients ---- */
/* fp16 gradients and parameters, fp32 master weights and Adam moments:
 * K = 12 bytes of optimizer state per parameter ([P1] "Where 16 bytes per
 * parameter comes from"). */
#define ZERO_PRECISION_FP16 0
/* bfloat16 gradients and parameters and NO fp32 master ([P3] "Why parameter
 * count is not training memory": not every BF16 setup keeps master weights):
 * fp32 m and v only, K = 8. Each step reads the weight from the bfloat16
 * parameter, runs the same binary32 Adam element and rounds the result back
 * to bfloat16 (nearest even) into every replica / the shard. Updates smaller
 * than half a bfloat16 spacing are lost ([P1] "Why you can't just delete the
 * fp32 copies" describes the same loss for fp16). Without a master a
 * speculative write could destroy the only copy of the weights, so the fused
 * variants (ZERO_VARIANT_FUSED, ZERO_VARIANT_FUSED_TMA) exist only where a
 * second copy does: stage 1/2 with all Nd >= 2 ranks emulated (rank_view =
 * -1). Their step reads the weight from the last replica and writes the new
 * one into the other Nd - 1; a replica pass, enqueued by the commit (or by
 * zero_step_async), then copies replica 0 into the last one, or on overflow
 * (or a kernel's failed wait) copies the last one's unchanged values back
 * over the others. Per element that is 4 B more than the floor instead of the
 * two-pass variants' 8 B of reduced gradient. Every other configuration needs
 * ZERO_VARIANT_TWO_PASS or ZERO_VARIANT_TWO_PASS_TMA (ZERO_ERR_ARG otherwise).
 * master_init of zero_init is rounded to bfloat16; the ledger's master
 * offsets are -1 and zero_current_state returns master = NULL; for
 * zero_set_state master may be NULL (the parameters stay as they are) or
 * fp32 values in state order to round into the parameters. */
#define ZERO_PRECISION_BF16 1

/* Tensor flag: exclude the tensor from weight decay (it takes the Adam update
 * with wd = 0). Decoupled weight decay (Loshchilov and Hutter) is commonly not
 * applied to biases and normalisation gains; the pages do not discuss it.
 * Numerics are unchanged for tensors without the flag. */
#define ZERO_TENSOR_NO_DECAY 1

/* One tensor of the flat parameter vector, in flat order. `unit` is the layer
 * unit a stage-3 gather rebuilds (units are numbered 0, 1, ... and appear in
 * non-decreasing order along the tensor list). */
typedef struct zero_tensor {
    int64_t numel;
    int32_t unit;
    int32_t flags; /* 0 or ZERO_TENSOR_NO_DECAY; other bits: ZERO_ERR_ARG */
} zero_tensor;

typedef struct zero_config {
    int64_t psi;       /* number of parameters of the flat vector */
    int32_t nd;        /* virtual data-parallel ranks, 1 .. ZERO_MAX_ND */
    int32_t stage;     /* ZeRO stage 1, 2 or 3 */
    int32_t rank_view; /* -1: emulate all Nd ranks; r >= 0: act as rank r
                          alone, owning partition r (stage 1/2) or shard r
                          (stage 3: rank r of a real job; grads are the Nd
                          ranks' full-length gradients, master_init the full
                          flat master, the fp16 shard stays in the workspace
                          at zero_ledger.off_shard16, and layer units are
                          gathered with zero_gather_layer_ranks) */
    int32_t variant;   /* ZERO_VARIANT_FUSED, _TWO_PASS, _FUSED_TMA or _TWO_PASS_TMA */
    int32_t n_tensors; /* 0 allowed for stage 1/2 (one flat tensor) */
    int32_t precision; /* ZERO_PRECISION_FP16 (0) or ZERO_PRECISION_BF16 */
    const zero_tensor* tensors; /* host array of n_tensors; sum of numel == psi;
                                   required for stage 3 */
    int32_t view_outputs; /* single-rank view only (else 0): parameter buffers
                             written, 0 or 1 = one buffer, nd = every rank's
                             replica (rank r of a real Nd-rank job: param_bufs
                             are all ranks' replicas, e.g. peer-mapped; see
                             zero_flag_words); stage 3: 0 or 1, the
                             output is the rank's own shard */
    int32_t reserved;     /* must be 0 */
} zero_config;

typedef struct zero_hyper {
    float lr;
    float beta1;
    float beta2;
    float eps;
    float weight_decay; /* decoupled, scaled by lr; 0 = plain Adam */
} zero_hyper;

/* Memory ledger and layout ([P1] "Where 16 bytes per parameter comes from":
 * 2 + 2 + K bytes, K = 12; [P1] stage table and [P2] "The Mathematics"). */
typedef struct zero_ledger {
    /* per-rank model-state bytes from the pages' formulas:
       [0] 16 psi, [1] 4 psi + 12 psi/Nd, [2] 2 psi + 14 psi/Nd, [3] 16 psi/Nd */
    double formula_bytes[4];
    /* the same for the rank holding the most under the ceil split, exact */
    int64_t exact_bytes[4];
    /* elements sent per step summed over ranks, ring collectives:
       [0] reduce-scatter, [1] all-gather, [2] DP all-reduce, [3..5] stage 1..3
       ([P1] "communication": 2 psi for DP and stages 1/2, 3 psi for stage 3,
       reached as Nd grows) */
    int64_t comm_elements[6];
    int64_t allreduce_buffer_bytes; /* flat fp32 buffer of the model, 4 psi
                                       ([P1] "What the 16 Psi formula doesn't cover") */
    int64_t transient_bytes;   /* stage 3: largest layer unit gathered (fp16), else 0 */
    int64_t peak_stage3_bytes; /* exact_bytes[3] + transient_bytes: the persistent
                                  estimate is not the peak ([P3] "Check your
                                  understanding") */
    int64_t workspace_bytes;   /* bytes zero_init needs */
    int64_t partition_len;     /* P = ceil(psi / Nd) */
    int64_t state_elems;       /* elements of each state array (master, m, v) */
    int64_t grad_len;          /* elements each grads[k] must hold */
    int64_t off_master[2];     /* byte offsets in the workspace of state buffer 0 and */
    int64_t off_m[2];          /*   1 (fused variant; -1 for two-pass)               */
    int64_t off_v[2];
    int64_t off_shard16;       /* stage 3: fp16 shard array (state order), else -1 */
    int64_t off_reduced;       /* two-pass: fp32 reduced gradients (state order), else -1 */
    int32_t n_units;           /* stage 3 layer units, else 0 */
    int32_t n_out;             /* parameter buffers zero_init takes (stage 1/2) */
} zero_ledger;

typedef struct zero_handle zero_handle;

/* Ledger, layout and workspace size for `cfg`. Host only: no device work, no
 * allocation. Returns ZERO_OK or ZERO_ERR_ARG. */
int zero_state_bytes(const zero_config* cfg, zero_ledger* out);

/* Where rank `rank`'s shard sits in the state arrays: elements
 * [*state_begin, *state_begin + *len) of master/m/v (and of the stage-3 fp16
 * shard array). Stage 1/2 with all ranks: the flat partition [r*P, ...).
 * Stage 3: rank r's chunk of every tensor, in tensor order, ranks back to back
 * ([P3] "What each ZeRO stage partitions"). Single-rank view: the viewed
 * rank's partition starts at 0, other ranks hold nothing here. Host only. */
int zero_rank_shard(const zero_config* cfg, int32_t rank, int64_t* state_begin, int64_t* len);

/* Flat range [*flat_begin, *flat_begin + *numel) of stage-3 layer unit
 * `unit`; zero_gather_layer writes *numel fp16 values. Host only. */
int zero_unit_range(const zero_config* cfg, int32_t unit, int64_t* flat_begin, int64_t* numel);

/* Bind a workspace and initialise the optimizer state.
 *   workspace     device, >= ledger.workspace_bytes, owned by the caller and
 *                 used by the handle until zero_destroy.
 *   master_init   device fp32: the initial master weights of the elements this
 *                 handle owns, in flat order (psi values; the stage 1/2
 *                 single-rank view takes the P_r values of partition r, NULL
 *                 if that is empty; a stage-3 rank view takes all psi values
 *                 and keeps its chunks).
 *   param_bufs    host array of device fp16 buffers that receive the all-
 *                 gathered parameters: stage 1/2 with all ranks: Nd replicas
 *                 of psi values each; single-rank view: one full psi-value
 *                 buffer of which partition r is written; stage 3: NULL (the
 *                 fp16 parameters live in the workspace shards).
 * Sets m = v = 0, master = master_init, t = 0, and writes fp16(master) to the
 * parameter buffers (or shards). Synchronises `stream` before returning. */
int zero_init(const zero_config* cfg, void* workspace, size_t workspace_bytes,
              const float* master_init, uint16_t* const* param_bufs, void* stream,
              zero_handle** out);

/* One optimizer step.
 *   grads       host array of Nd device fp16 gradient buffers, rank order.
 *               All ranks: each holds psi values (the rank's full gradient).
 *               Stage 1/2 single-rank view: each holds rank k's P_r
 *               gradients of the viewed partition r. Stage-3 rank view: each
 *               holds rank k's full gradient (psi values).
 *   loss_scale  > 0 and finite; gradients are multiplied by 1/loss_scale.
 *   skipped     optional out: 1 if the step was skipped for overflow.
 * Returns ZERO_OK, or ZERO_SKIPPED when some unscaled reduced gradient is inf
 * or NaN: then master/m/v, t and the fp16 parameters are as before the call.
 * Reads one 4-byte flag back and synchronises `stream` once. */
int zero_step(zero_handle* h, const uint16_t* const* grads, float loss_scale,
              const zero_hyper* hp, void* stream, int* skipped);

/* zero_step in two halves, for callers that overlap host work with the step
 * or time its kernels on the stream. zero_step_launch validates and enqueues
 * the step's kernels on `stream` and returns without waiting. zero_step_commit
 * waits for `stream` to reach the end of the step, reads the overflow flag and
 * commits (ZERO_OK) or rolls back (ZERO_SKIPPED) exactly as zero_step. Every
 * launch must be followed by its commit before the next launch or gather on
 * the handle (ZERO_ERR_ARG otherwise). */
int zero_step_launch(zero_handle* h, const uint16_t* const* grads, float loss_scale,
                     const zero_hyper* hp, void* stream);
int zero_step_commit(zero_handle* h, void* stream, int* skipped);

/* The handle's overflow word and kernel-error word: two consecutive uint32 in
 * the workspace (device memory). A step of ZeRO stage 1/2 is skipped if ANY
 * rank's reduced gradient overflows ([P1] "The part that sounds too good:
 * communication": the ranks reduce-scatter, update their slices, all-gather;
 * one overflow decision for the step). When each rank of a real Nd-rank job
 * runs its own single-rank-view handle (view_outputs = nd on stage 1/2; any
 * stage-3 rank view), the ranks agree by
 * reducing these two words with MAX across ranks on `stream` between
 * zero_step_launch and zero_step_commit (for instance ncclAllReduce with
 * ncclMax on ncclUint32, count 2); the words hold the handle's step call id on
 * overflow, which advances identically on every rank. With a two-pass variant
 * such a handle's zero_step_launch enqueues only the reduce pass and its
 * zero_step_commit enqueues the in-place update pass after the agreement (the
 * pass returns at once if the agreed words say overflow); the fused variants
 * write speculatively and roll back on an agreed overflow. Such handles take
 * no asynchronous steps (zero_async_begin: ZERO_ERR_ARG). Host only (returns
 * the address). ZERO_OK or ZERO_ERR_ARG. */
int zero_flag_words(zero_handle* h, uint32_t** words);

/* ---- asynchronous steps ([P1]-[P3] do not cover loss scaling; the usual
 * dynamic loss scaling is the reading) ----
 * Between zero_async_begin and zero_async_end the step count, the bias-
 * correction products, the live state buffer and a dynamic loss scale live on
 * the device, and zero_step_async only enqueues work: it reads nothing back
 * and calls nothing that synchronises, so a caller can issue steps back to
 * back or capture one in a CUDA graph and replay it. Each step computes what
 * zero_step computes with the current loss scale; then, on the device, an
 * overflowing step is rolled back (as with ZERO_SKIPPED) and the scale is
 * multiplied by backoff_factor, while a good step commits and, after
 * growth_interval good steps in a row, multiplies the scale by growth_factor
 * (kept if that would overflow binary32). */
typedef struct zero_scaler {
    float init_scale;        /* > 0 and finite */
    float growth_factor;     /* >= 1 */
    float backoff_factor;    /* in (0, 1] */
    int32_t growth_interval; /* >= 1 */
} zero_scaler;

typedef struct zero_async_state {
    int64_t t;          /* steps committed (all time) */
    int64_t skipped;    /* steps skipped during this run */
    float loss_scale;   /* the scale the next step would use */
    int32_t good_steps; /* good steps since the last growth or back-off */
} zero_async_state;

/* Open an asynchronous run: grads (host array of Nd device pointers, as for
 * zero_step) are bound for the whole run -- refill the same buffers between
 * steps -- and beta1/beta2 are fixed. Synchronises `stream` once. Every later
 * zero_step_async must pass the same betas. zero_step, zero_step_launch and
 * zero_current_state return ZERO_ERR_ARG until zero_async_end. */
int zero_async_begin(zero_handle* h, const uint16_t* const* grads, const zero_scaler* sc,
                     float beta1, float beta2, void* stream);
/* Enqueue one step (no host synchronisation, no host-side reads). */
int zero_step_async(zero_handle* h, const zero_hyper* hp, void* stream);
/* Close the run: synchronise `stream`, return the device-side counters and
 * hand t and the live buffer back to the host. Returns ZERO_ERR_INTERNAL if a
 * kernel gave up a bounded wait during the run (those steps, and every later
 * one of the run, were skipped), or ZERO_ERR_PARTIAL if that kernel was the
 * in-place update pass of ZERO_VARIANT_TWO_PASS_TMA (part of the state holds
 * that step's values: restore a saved state with zero_set_state). */
int zero_async_end(zero_handle* h, void* stream, zero_async_state* out);

/* Stage 3: write layer unit `unit`'s full fp16 weights into `out` (device,
 * >= the numel zero_unit_range reports): its tensors in tensor order, each whole
 * and contiguous, back to back. Call it per unit in forward order and again in
 * reverse for backward ([P1] "communication": parameters are gathered on demand
 * in the forward and backward passes, then discarded). ZERO_ERR_STAGE on 1/2.
 * Every variant gathers with the same copy kernel as zero_gather_layer_ranks
 * (16-byte loads and stores, each block copying 16 KB tiles of one rank's
 * chunk in turn), launched as a programmatic dependent of the previous kernel
 * on `stream`: its blocks may be scheduled while that kernel finishes, but it
 * touches no memory before that kernel has completed. */
int zero_gather_layer(zero_handle* h, int32_t unit, uint16_t* out, void* stream);

/* Stage-3 layer gather of rank r of a real Nd-rank job (a handle with
 * rank_view = r): the fp16 values of layer unit `unit` in flat order, copied
 * from the Nd ranks' fp16 shards ([P1] "The part that sounds too good:
 * communication": stage 3 all-gathers each layer's parameters when the
 * forward or the backward pass needs them). shards[k]: device address of
 * rank k's shard (the region at zero_ledger.off_shard16 of rank k's
 * workspace, shard_len(k) elements; peer-mapped for k != r, see zero_peer.h;
 * may be NULL for an empty shard); out: device buffer of the unit's numel
 * elements (zero_unit_range). Every rank's step must have finished before the
 * gather reads its shard (the caller's barrier). Returns ZERO_ERR_STAGE on
 * stage 1/2, ZERO_ERR_ARG for a handle that emulates all ranks (use
 * zero_gather_layer) or a bad unit, ZERO_ERR_ALIGN for unaligned buffers. */
int zero_gather_layer_ranks(zero_handle* h, int32_t unit, const uint16_t* const* shards, uint16_t* out,
                            void* stream);

/* One copy of a stage-3 layer gather: `len` fp16 elements from offset
 * src_begin of rank src_rank's shard to offset out_begin of the unit. */
typedef struct zero_gather_run {
    int64_t src_begin;
    int64_t out_begin;
    int64_t len;      /* > 0 */
    int32_t src_rank;
    int32_t reserved; /* 0 */
} zero_gather_run;

/* The copies that gather layer unit `unit` of a stage-3 configuration (any
 * rank_view): one per non-empty chunk, tensor by tensor in the unit, ranks in
 * order within a tensor, so out_begin increases and the runs tile the unit.
 * What zero_gather_layer_ranks executes, for callers that move the chunks
 * with a transport of their own. *n_runs receives the count; runs may be NULL
 * to ask for it, else it must hold cap >= *n_runs entries. Host only.
 * ZERO_ERR_STAGE on stage 1/2, ZERO_ERR_ARG for a bad unit or a short cap. */
int zero_gather_plan(const zero_config* cfg, int32_t unit, zero_gather_run* runs, int64_t cap,
                     int64_t* n_runs);

/* Current state: device pointers to the live master/m/v arrays (the fused
 * variant alternates between two buffers) and the step count t. Any output
 * pointer may be NULL. ZERO_ERR_ARG while an asynchronous run is open. */
int zero_current_state(const zero_handle* h, float** master, float** m, float** v, int64_t* t);

/* Checkpoint / resume: restore a saved state into the handle. master, m, v
 * are device fp32 arrays in state order (ledger.state_elems values each, as
 * zero_current_state exposes them; they may be the live arrays themselves),
 * t the step count they belong to. The fp16 parameters (replicas or stage-3
 * shards) are rewritten from master. To save, copy the three arrays
 * zero_current_state points to, and t. Synchronises `stream`. */
int zero_set_state(zero_handle* h, const float* master, const float* m, const float* v, int64_t t,
                   void* stream);

/* Memory bandwidth reference: copy `bytes` (a multiple of 16, both pointers
 * 16-byte aligned) from src to dst with 16-byte streaming loads and stores. */
int zero_stream_copy(void* dst, const void* src, size_t bytes, void* stream);

/* ---- allocation-free step (no counterpart on the pages) ----
 *
 * Some callers cannot allocate device memory for a workspace: code whose
 * device memory belongs to another allocator it cannot reach from plain C (an
 * embedding framework's caching allocator, say), or code that must not pay
 * cudaMalloc's cost and its implicit device synchronisation in the middle of
 * a training step. zero_step_static serves them: one two-pass stage 1/2 step
 * (all Nd ranks emulated, flat parameter vector) whose scratch -- the fp32
 * reduced gradients, the overflow word and the pointer and run tables -- lives
 * in a fixed array inside the library, so the call allocates nothing. The
 * caller still owns and passes every input and output:
 *   grads      host array of nd device fp16 gradient buffers, psi values each
 *   master, m, v  device fp32, psi values each, updated in place (the caller
 *              initialises them: m = v = 0 before the first step)
 *   replicas   host array of nd device fp16 parameter buffers, psi values each
 *   t          host in/out step count, 0 <= t < INT64_MAX (the bias
 *              corrections use the (t+1)-fold products of the betas; it
 *              advances by one on a step that is not skipped). The library
 *              keeps the last products and continues from them while the
 *              betas stay the same and t does not go backwards, so a run
 *              pays one multiplication per step; a large first t costs at
 *              most a few million (the products stop changing at 0 or the
 *              smallest subnormal).
 * The arithmetic and the result are those of zero_step with
 * ZERO_VARIANT_TWO_PASS on the same state. Returns ZERO_OK or ZERO_SKIPPED
 * (nothing changed), ZERO_ERR_ARG when psi > ZERO_STATIC_MAX_PSI or
 * nd > ZERO_STATIC_MAX_ND (or for any other invalid argument), ZERO_ERR_ALIGN
 * for a device pointer that is not 16-byte aligned, ZERO_ERR_CUDA otherwise.
 *
 * The scratch is one array of 8 KiB + 4 * ZERO_STATIC_MAX_PSI bytes (4 MiB +
 * 8 KiB); every device that loads it holds it until the process exits. The
 * first call on a device, with that device current, looks up the array's
 * device address; make that first call before any stream capture. All calls
 * on a device share the array and it keeps the last call's contents (the
 * overflow word is cleared by each call): calls that overlap on the GPU, for
 * example on two streams, race with each other and must not be issued. Calls
 * from two host threads at the same time race as well, even on one stream,
 * because one call's table uploads can land between the other call's uploads
 * and its kernels: serialise them. The call synchronises `stream` once to
 * read the overflow word. */
#define ZERO_STATIC_MAX_PSI 1048576
#define ZERO_STATIC_MAX_ND 64
int zero_step_static(int64_t psi, int32_t nd, const uint16_t* const* grads, float* master,
                     float* m, float* v, uint16_t* const* replicas, float loss_scale,
                     const zero_hyper* hp, int64_t* t, void* stream, int* skipped);

/* 1 if the handle's steps run the TMA-staged kernel (ZERO_VARIANT_FUSED_TMA
 * on an eligible configuration), 0 if not, ZERO_ERR_ARG for a NULL handle. */
int zero_uses_tma(const zero_handle* h);

/* Test hook for the bounded waits of the TMA kernels, which fail without any
 * GPU fault: the next TMA step on this handle leaves its tile number `tile`
 * unarmed, so the waits on it give up after `wait_rounds` try_wait rounds
 * (each suspends about a microsecond). The kernel sets its error word and
 * drains its own copies; the step is rolled back like a skipped one and
 * returns ZERO_ERR_INTERNAL. The hook applies once.
 * Has no effect on handles that do not run the TMA kernels. For
 * ZERO_VARIANT_TWO_PASS_TMA the tile is one of the reduce pass. */
int zero_test_hold_tile(zero_handle* h, int64_t tile, uint32_t wait_rounds);

/* The same test hook for the update pass of ZERO_VARIANT_TWO_PASS_TMA: the
 * next step's update pass leaves its tile number `tile` unarmed, its waits on
 * it give up after `wait_rounds` rounds, the other tiles are updated in place,
 * and the step returns ZERO_ERR_PARTIAL. Applies once; ZERO_ERR_ARG on a
 * handle of another variant, or one that does not run the TMA kernels. */
int zero_test_hold_update_tile(zero_handle* h, int64_t tile, uint32_t wait_rounds);

/* The cudaError_t of the last failed CUDA call made through `h` (0 if none). */
int zero_last_cuda_error(const zero_handle* h);

/* Static text for a return code. */
const char* zero_error_string(int code);

/* Release the handle (host memory only; the caller frees the workspace). */
void zero_destroy(zero_handle* h);

#ifdef __cplusplus
}
#endif
#endif
