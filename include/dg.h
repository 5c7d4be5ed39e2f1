/*
 * dg.h -- C ABI of the B200 denoising-step library (libdg.so).
 *
 * One denoising step of block discrete-diffusion text generation over
 * canvases of L = 256 token slots: the tied LM head z = h . E^T fused with
 * the sampler (temperature-scaled softmax entropy, Gumbel-max draw),
 * entropy-bounded acceptance, full renoise of the unaccepted slots and the
 * adaptive-stop test.  Sources, by page title and section:
 *
 *   [Docs]   "DiffusionGemma" (Google AI for Developers model docs), table
 *            "Recommended serving configuration": max 48 denoising steps,
 *            temperature linear 0.8 -> 0.4, adaptive stop at mean entropy
 *            0.005 with two identical consecutive predictions, token
 *            selection with entropy bound 0.1 and full renoise of the rest.
 *   [Report] "DiffusionGemma Technical Report" (arXiv:2608.00146), Table 1
 *            (262k vocabulary, 740M embedder => d = 2816), Figure 3 (uniform
 *            noise), Figure 4 (denoising loop over a 256-token canvas).
 *   [Press]  "Google DiffusionGemma generates 256 tokens in parallel and
 *            self-corrects", section "What DiffusionGemma does" (every
 *            position re-evaluated each step; low-confidence positions are
 *            randomised; once the block settles its open positions are fixed).
 *
 * Conventions for every entry point:
 *   - Tensors are DEVICE pointers owned by the caller unless marked "host".
 *     The library allocates no device memory; scratch lives in a caller
 *     workspace of dg_workspace_size() bytes, zeroed once by
 *     dg_workspace_init() before its first use.
 *   - Row r = b*L + s of a [B*L, ...] tensor is slot s of canvas b.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t, NULL =
 *     legacy default stream).  Argument errors are detected on the host
 *     before anything is launched.  Faults detected on the device (a
 *     bounded wait that ran out) are latched in the workspace and reported
 *     by dg_device_status().
 *   - Errors are returned, never raised: no exit(), no abort().
 *   - Calls that share a workspace must not overlap on the device.
 */
#ifndef DG_H
#define DG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DG_OK = 0,
  DG_ERR_INVALID_ARG = 1,      /* null pointer, misalignment, bad parameter */
  DG_ERR_UNSUPPORTED_SHAPE = 2,/* L != 256, d % 64, V % 256, B out of range */
  DG_ERR_WORKSPACE = 3,        /* workspace smaller than dg_workspace_size() */
  DG_ERR_RANGE = 4,            /* a step index k outside [0, max_steps) */
  DG_ERR_CUDA = 5,             /* a CUDA runtime call failed */
  DG_ERR_TIMEOUT = 6,          /* a device-side bounded wait ran out */
  DG_ERR_CALLBACK = 7,         /* the hidden-state callback returned non-zero */
  DG_ERR_NO_DEVICE = 8,        /* no sm_100 device current */
  DG_ERR_VALUE = 9             /* FP8 head: a hidden-state value is not finite
                                  (found on the device) */
} dg_status;

typedef enum { DG_E_BF16 = 0, DG_E_FP8_E4M3 = 1 } dg_edtype;

/* Problem shape.  L must be 256 ([Report] Figure 4: 256-token canvas);
 * d a multiple of 64 and >= 64; V a multiple of 256 and >= 256;
 * 1 <= B <= DG_MAX_B. */
typedef struct {
  int32_t B;        /* canvases per step */
  int32_t L;        /* slots per canvas (256) */
  int32_t d;        /* hidden size */
  int32_t V;        /* vocabulary size */
  int32_t e_dtype;  /* dg_edtype of the embedder */
} dg_shape;

#define DG_MAX_B 256

/* Selection rule: which prefix of the slots ordered by (entropy, slot) is
 * accepted each step.  Every rule accepts at least one slot.
 *   DG_SELECT_CUMSUM  the longest prefix whose entropy sum is <= entropy_bound
 *                     (default; this library's reading of the [Docs]
 *                     token-selection row, which bounds a mutual-information
 *                     estimate by 0.1 and gives no formula).
 *   DG_SELECT_MI      the longest prefix whose entropy sum minus its largest
 *                     entropy is <= entropy_bound (the usual form of such a
 *                     bound in the literature; not stated on the pages).
 *   DG_SELECT_TOPK    the top_k lowest-entropy slots (1 <= top_k <= L). */
typedef enum { DG_SELECT_CUMSUM = 0, DG_SELECT_MI = 1, DG_SELECT_TOPK = 2 } dg_selection;

/* Sampler parameters; dg_default_params() gives the [Docs] serving
 * defaults (tau0 0.8, tau1 0.4, 48 steps, bound 0.1, stop 0.005,
 * DG_SELECT_CUMSUM, seed 1234, block 0). */
typedef struct {
  double tau0;             /* temperature at step 0 */
  double tau1;             /* temperature at step max_steps-1 */
  int32_t max_steps;       /* N, at most this many steps per canvas */
  double entropy_bound;    /* selection bound on the entropies (see dg_selection) */
  double stop_entropy;     /* adaptive stop: canvas-mean entropy threshold */
  uint64_t seed;           /* Philox4x32-10 key (low word, high word) */
  int32_t selection_rule;  /* a dg_selection */
  int32_t top_k;           /* slots accepted by DG_SELECT_TOPK */
  int32_t block;           /* index of the canvas block in a block-by-block
                              generation (0 for a single block): every
                              block draws its own random streams, the
                              Philox counter's step word being
                              k | block << 16 (0 <= block < 65536;
                              max_steps <= 65536) */
} dg_params;

dg_params dg_default_params(void);

/* Human-readable name of a status code (static storage). */
const char* dg_error_string(dg_status s);

/* Bytes of device workspace one step of this shape needs on the current
 * device (it depends on the device's SM count).  Returns 0 for an invalid
 * shape. */
size_t dg_workspace_size(const dg_shape* shape);

/* Zero a workspace (enqueued on `stream`).  Needed once per workspace. */
dg_status dg_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/* dg_denoise_step -- one denoising step of B canvases.
 *
 * Inputs
 *   h         bf16 [B*L, d] row-major: canvas hidden states.
 *   E         embedder [V, d] row-major: bf16, or FP8-E4M3 codes (uint8)
 *             when shape->e_dtype == DG_E_FP8_E4M3.  The tied LM head
 *             ([Report] Table 1) is z = h . E^T (times e_scale[v] for FP8).
 *   e_scale   float [V] per-row dequantisation scale, 16-byte aligned:
 *             required for FP8, must be NULL for bf16 (DG_ERR_INVALID_ARG).
 *             The FP8 head computes z[r, v] = e_scale[v] * sum_k h[r,k] q[v,k]
 *             on E4M3 tensor-core operands: q as given, and h split per row
 *             into two E4M3 terms with a power-of-two scale 2^k_r
 *             (h * 2^k_r = h1 + h2), exact for every |h[r,k]| >= 2^-9 *
 *             max_k |h[r,k]| and within 2^-10 * 2^-k_r below that.  A
 *             non-finite h latches DG_ERR_VALUE (see dg_device_status) and
 *             leaves the step's results undefined.
 *   step_idx  HOST int32 [B]: step k of each canvas, 0 <= k < max_steps.
 *             tau_k = tau0 - (tau0 - tau1) * k / (max_steps - 1)
 *             ([Docs] temperature schedule), tau0 for max_steps == 1.
 *   has_prev  HOST uint8 [B]: 1 if prev_argmax holds the previous step's
 *             prediction for that canvas (0 on a canvas's first step).
 *   active    HOST uint8 [B] or NULL (= all 1): canvases with 0 are frozen:
 *             they cost no head or merge work and none of their outputs
 *             (canvas, prev_argmax, accept, entropy, sampled, argmax, stop)
 *             is written.  With every canvas frozen nothing is launched.
 * In/out
 *   canvas      int32 [B*L]: overwritten with the new canvas (accepted slots
 *               take the sampled token, the rest a uniform random token).
 *   prev_argmax int32 [B*L]: read as the previous prediction, then
 *               overwritten with this step's argmax prediction.
 * Outputs
 *   accept   uint8 [B*L]   entropy-bounded acceptance mask.
 *   entropy  float [B*L]   entropy (nats) of softmax(z / tau_k).
 *   sampled  int32 [B*L]   Gumbel-max draw from softmax(z / tau_k).
 *   argmax   int32 [B*L]   argmax_v z (ties to the lower v).
 *   stop     int32 [B]     adaptive-stop flag of each canvas.
 * Scratch
 *   workspace, ws_bytes >= dg_workspace_size(shape), zeroed once.
 * h and E must be 16-byte aligned.  Asynchronous on `stream`.
 */
dg_status dg_denoise_step(const dg_shape* shape, const dg_params* params,
                          const void* h, const void* E, const float* e_scale,
                          const int32_t* step_idx, const uint8_t* has_prev,
                          const uint8_t* active,
                          int32_t* canvas, int32_t* prev_argmax,
                          uint8_t* accept, float* entropy, int32_t* sampled,
                          int32_t* argmax, int32_t* stop,
                          void* workspace, size_t ws_bytes, void* stream);

/* dg_debug_logits -- the same step as dg_denoise_step (same kernels, same
 * outputs) that also writes the raw float32 logits z [B*L, V] the fused
 * sampler consumed.  For parity checks only: it writes B*L*V*4 bytes. */
dg_status dg_debug_logits(const dg_shape* shape, const dg_params* params,
                          const void* h, const void* E, const float* e_scale,
                          const int32_t* step_idx, const uint8_t* has_prev,
                          const uint8_t* active,
                          int32_t* canvas, int32_t* prev_argmax,
                          uint8_t* accept, float* entropy, int32_t* sampled,
                          int32_t* argmax, int32_t* stop, float* logits,
                          void* workspace, size_t ws_bytes, void* stream);

/* Synchronise `stream`, then read and clear the device fault latch of the
 * workspace.  Returns DG_OK, DG_ERR_TIMEOUT (a bounded wait ran out),
 * DG_ERR_VALUE (FP8 head: a non-finite h; self-conditioning: logits beyond
 * the probability encoding's range) or DG_ERR_CUDA. */
dg_status dg_device_status(void* workspace, size_t ws_bytes, void* stream);

/* Hidden-state producer for the loop: writes the bf16 [B*L, d] hidden
 * states of step k for the current canvas into h_out (device), enqueued on
 * `stream`.  Returns 0 on success; anything else stops the loop with
 * DG_ERR_CALLBACK.  It stands in for the denoiser's forward pass. */
typedef int (*dg_hidden_fn)(int32_t k, const int32_t* canvas, void* h_out,
                            void* user, void* stream);

/* dg_denoise_loop -- the adaptive loop ([Docs] max steps and adaptive stop;
 * [Report] Figure 4).  For k = k_start, k_start+1, ...: hidden_fn writes h,
 * one dg_denoise_step runs on every still-active canvas, the B stop flags
 * are read back (one device->host copy per step).  A canvas that stops, or
 * reaches k = max_steps-1, commits: every slot takes that step's sampled
 * token ([Press]: the settled block's open positions are fixed) and the
 * canvas is frozen.
 *
 *   h_buf        bf16 [B*L, d] device buffer handed to hidden_fn.
 *   canvas       int32 [B*L] in/out: the committed canvas on return.
 *   prev_argmax  int32 [B*L] in/out: prediction state (see has_prev).
 *   has_prev     HOST uint8 [B] in/out: resume state; all 0 for a fresh start.
 *   steps_taken  HOST int32 [B] out: steps run for each canvas.
 *   accept, entropy, sampled, argmax, stop: device outputs of each canvas's
 *                last step (a frozen canvas is skipped by the later steps:
 *                it costs no head work and its outputs are left as they were).
 * Resuming with the state of an interrupted loop at k_start gives the same
 * result as the uninterrupted run (the random streams are counter-based).
 */
dg_status dg_denoise_loop(const dg_shape* shape, const dg_params* params,
                          const void* E, const float* e_scale,
                          dg_hidden_fn hidden_fn, void* user, int32_t k_start,
                          void* h_buf, int32_t* canvas, int32_t* prev_argmax,
                          uint8_t* has_prev, int32_t* steps_taken,
                          uint8_t* accept, float* entropy, int32_t* sampled,
                          int32_t* argmax, int32_t* stop,
                          void* workspace, size_t ws_bytes, void* stream);

/* ---- self-conditioning signal ([Report] Table 1: the model carries a
 * 7.8M-parameter self-conditioning MLP; the pages define neither the signal
 * nor the MLP).  Reading: the signal of slot r is the embedding expected under the
 * step's tempered distribution, s[r] = sum_v softmax(z[r] / tau_k)_v E[v]
 * (a d-vector per slot), the input such an MLP would project.  The MLP has
 * trained weights and is out of scope.
 *
 * The head writes block-scaled bf16 probabilities while it samples; a
 * pass normalises them with the merged softmax statistics, a split-K
 * tcgen05 GEMM against E^T (both operands K-major) multiplies, and a
 * fixed-order reduction forms s.  P is rounded to bf16 twice (block-scaled, then normalised):
 * |s_gpu - s| <= 2^-8 sum_v p_v |E[v]| per element, plus float32 sums. */

/* E_t = E^T as bf16 [d, V] row-major (device, d * V * 2 bytes, caller-
 * owned): E's bf16 values, or for the FP8 embedder its E4M3 codes widened
 * to bf16 exactly (the row scales are applied to the probabilities).  Made
 * once per embedder. */
dg_status dg_embedder_transpose(const dg_shape* shape, const void* E, void* E_t, void* stream);

/* Workspace bytes of dg_denoise_step_selfcond on the current device: the
 * step's workspace, P (B*L*V bf16), the block references, the row
 * statistics and the split-K partial sums.  0 for an invalid shape. */
size_t dg_selfcond_workspace_size(const dg_shape* shape);

/* dg_denoise_step_selfcond -- dg_denoise_step (every canvas updated; no
 * `active`) that also writes the self-conditioning signal
 *   signal  float [B*L, d] (device, 16-byte aligned).
 * E_t from dg_embedder_transpose of the same E; workspace of
 * dg_selfcond_workspace_size() bytes (zeroed once, like a step's).  A
 * block of logits spanning more than the bf16 probability encoding can hold
 * (2^126) latches DG_ERR_VALUE (see dg_device_status). */
dg_status dg_denoise_step_selfcond(const dg_shape* shape, const dg_params* params,
                                   const void* h, const void* E, const float* e_scale, const void* E_t,
                                   const int32_t* step_idx, const uint8_t* has_prev,
                                   int32_t* canvas, int32_t* prev_argmax,
                                   uint8_t* accept, float* entropy, int32_t* sampled,
                                   int32_t* argmax, int32_t* stop, float* signal,
                                   void* workspace, size_t ws_bytes, void* stream);

/* ---- the adaptive loop on the device -------------------------------------
 * dg_denoise_loop reads the stop flags back to the host after every step.
 * dg_denoise_loop_graph runs the same loop as one CUDA graph: a conditional
 * (while) node whose body is [hidden_graph] -> step -> loop control, where a
 * control kernel commits and freezes the canvases that stopped (or reached
 * k = max_steps-1), advances k, prepares the next step's temperatures and
 * the list of canvases still running, and ends the loop when none is left;
 * nothing returns to the host until the loop is over.  Results equal
 * dg_denoise_loop's for the same hidden states. */

/* Bytes of device loop state for B canvases (256-byte aligned buffer,
 * owned by the caller); 0 for B outside [1, DG_MAX_B].  Its first int32 is
 * the step index k the graph body is about to run: the hidden-state graph
 * reads it there to produce step k's hidden states. */
size_t dg_loop_state_bytes(int32_t B);

/* hidden_graph  a cudaGraph_t (or NULL) embedded at the head of the loop
 *               body: it must write the bf16 [B*L, d] hidden states of step
 *               k (k = the first int32 of loop_state) into h_buf, using only
 *               node kinds a conditional body accepts (kernels, memcpy,
 *               memset).  NULL: h_buf is used as it stands every step.
 * has_prev      HOST uint8 [B] in/out, as for dg_denoise_loop.
 * steps_taken   HOST int32 [B] out.
 * loop_state    device buffer of dg_loop_state_bytes(B) bytes.
 * Other arguments as for dg_denoise_loop.  The graph is built, run and
 * destroyed inside the call, which returns after synchronising `stream`; a
 * device-side fault ends the loop and is returned (DG_ERR_TIMEOUT or
 * DG_ERR_VALUE). */
dg_status dg_denoise_loop_graph(const dg_shape* shape, const dg_params* params,
                                const void* E, const float* e_scale, void* hidden_graph,
                                int32_t k_start, void* h_buf, int32_t* canvas, int32_t* prev_argmax,
                                uint8_t* has_prev, int32_t* steps_taken,
                                uint8_t* accept, float* entropy, int32_t* sampled,
                                int32_t* argmax, int32_t* stop,
                                void* loop_state, size_t state_bytes,
                                void* workspace, size_t ws_bytes, void* stream);

/* The same loop built once and run many times: dg_denoise_loop_graph
 * builds (by stream capture), instantiates and destroys its graph in every
 * call; a dg_loop_graph keeps it.
 *
 * dg_loop_graph_create -- build and instantiate the loop graph on the current
 * device for fixed buffers.  Arguments as for dg_denoise_loop_graph, less
 * the per-call ones (k_start, has_prev, steps_taken, stream); every buffer
 * must stay allocated, and hold its role, until the handle is destroyed.
 * The hidden-state graph is copied into the loop when the handle is built:
 * later changes to hidden_graph do not reach it.  On success *out holds the
 * handle; on failure *out is NULL.
 *
 * dg_loop_graph_run -- one adaptive loop from step k_start with the given
 * has_prev (HOST uint8 [B], in/out) and steps_taken (HOST int32 [B], out),
 * enqueued on `stream` and synchronised, exactly as dg_denoise_loop_graph
 * (whose results it equals).  The canvas and prev_argmax buffers given at
 * create time are the loop's input and output.  Must be called on the
 * device the handle was built on (else DG_ERR_INVALID_ARG); runs of one
 * handle must not overlap (they share the loop state and workspace).
 *
 * dg_loop_graph_destroy -- release the graph (NULL is a no-op). */
typedef struct dg_loop_graph_s* dg_loop_graph;
dg_status dg_loop_graph_create(const dg_shape* shape, const dg_params* params,
                               const void* E, const float* e_scale, void* hidden_graph,
                               void* h_buf, int32_t* canvas, int32_t* prev_argmax,
                               uint8_t* accept, float* entropy, int32_t* sampled,
                               int32_t* argmax, int32_t* stop,
                               void* loop_state, size_t state_bytes,
                               void* workspace, size_t ws_bytes, dg_loop_graph* out);
dg_status dg_loop_graph_run(dg_loop_graph graph, int32_t k_start, uint8_t* has_prev,
                            int32_t* steps_taken, void* stream);
void dg_loop_graph_destroy(dg_loop_graph graph);

/* ---- block-by-block generation ([Report] Figure 4: encode & append) ----
 * Generation runs block after block: each block of B canvases starts from
 * uniform noise, the adaptive loop denoises it until it settles, and the
 * committed block is appended to the context the next block is conditioned
 * on.  The model that encodes the committed blocks and produces the hidden
 * states is the caller's (hidden_fn); this library runs the blocks' steps. */

/* Fill canvas (int32 [B*L], device) with the uniform noise block
 * params->block starts from ([Report] Figure 3: uniform noise): token
 * (r V) >> 32 of Philox counter (0, slot | 3 << 16, block << 16, b), lane 0. */
dg_status dg_init_canvas(const dg_shape* shape, const dg_params* params, int32_t* canvas, void* stream);

/* Hidden-state producer of block j: writes the bf16 [B*L, d] hidden states
 * of step k of block j into h_out (device) given the block's current canvas
 * (device int32 [B*L]) and the blocks committed before it (device int32
 * [j][B*L], the first j rows of dg_generate_blocks' `blocks`; NULL for
 * j = 0), enqueued on `stream`.  Returns 0 on success; anything else stops
 * the generation with DG_ERR_CALLBACK. */
typedef int (*dg_block_hidden_fn)(int32_t block, int32_t k, const int32_t* canvas,
                                  const int32_t* committed, void* h_out, void* user, void* stream);

/* dg_generate_blocks -- n_blocks blocks, one after another.  Block j
 * (numbered params->block + j in the random streams) starts from
 * dg_init_canvas' noise and runs dg_denoise_loop from k = 0; its committed
 * canvas is written to blocks[j] before block j + 1 starts.
 *   blocks       int32 [n_blocks][B*L] device out: the committed blocks.
 *   steps_taken  HOST int32 [n_blocks][B] out: steps each canvas ran.
 *   canvas, prev_argmax  int32 [B*L] device scratch (the current block).
 *   h_buf, accept, entropy, sampled, argmax, stop, workspace: as for
 *   dg_denoise_loop (the outputs hold the last block's last steps).
 * Synchronises `stream` once per step (the loop's stop-flag read). */
dg_status dg_generate_blocks(const dg_shape* shape, const dg_params* params,
                             const void* E, const float* e_scale, int32_t n_blocks,
                             dg_block_hidden_fn hidden_fn, void* user, void* h_buf,
                             int32_t* blocks, int32_t* steps_taken,
                             int32_t* canvas, int32_t* prev_argmax,
                             uint8_t* accept, float* entropy, int32_t* sampled,
                             int32_t* argmax, int32_t* stop,
                             void* workspace, size_t ws_bytes, void* stream);

/* dg_denoise_step_noalloc -- dg_denoise_step for callers that cannot
 * allocate device memory for a workspace: a serving runtime that has carved
 * up the whole GPU for its own pools, or code that must not call the CUDA
 * allocator (which can synchronise the device) where it runs steps.  The
 * pages have no counterpart; this is an interface convenience.
 *
 * Same arguments and results as dg_denoise_step, without workspace and
 * ws_bytes.  The scratch lives in a fixed 8 MiB array of the library's own
 * device memory, held on every GPU that loads the library until the process
 * exits.  Shapes needing more (dg_workspace_size() > 8 MiB) return
 * DG_ERR_WORKSPACE before anything is launched, with the sizes in
 * dg_last_error_message(); on a 148-SM B200 at d = 2816, V = 262,144 that
 * is B > 18 canvases with the bf16 embedder and B > 2 with the FP8 embedder
 * (whose scratch also holds the two E4M3 terms of h).  All argument checks
 * run before the array is touched.  The first call on a device looks the
 * array's device address up once (the runtime may initialise the context
 * then), so make it before any stream capture.  Every call uses the same
 * array: calls that overlap on the GPU (other streams, other threads) race
 * and must be serialised by the caller.  Each call clears, on `stream`, the
 * parts that must start at zero (tickets, key records).  A device-side
 * fault (a bounded wait that ran out, or for the FP8 head a non-finite h)
 * latches in the array and leaves that call's results undefined; the latch
 * is kept across calls until dg_noalloc_status() reads and clears it. */
dg_status dg_denoise_step_noalloc(const dg_shape* shape, const dg_params* params,
                                  const void* h, const void* E, const float* e_scale,
                                  const int32_t* step_idx, const uint8_t* has_prev,
                                  const uint8_t* active,
                                  int32_t* canvas, int32_t* prev_argmax,
                                  uint8_t* accept, float* entropy, int32_t* sampled,
                                  int32_t* argmax, int32_t* stop, void* stream);

/* Synchronise `stream`, then read and clear the fault latch of
 * dg_denoise_step_noalloc's array on the current device: DG_OK (no fault
 * since the last read), DG_ERR_TIMEOUT, DG_ERR_VALUE or DG_ERR_CUDA, as
 * dg_device_status() does for a workspace.  Call it after the steps whose
 * results are to be trusted. */
dg_status dg_noalloc_status(void* stream);

/* ---- vocabulary-sharded step ---------------------------------------------
 * For an embedder split over G GPUs by vocabulary rows (equal shards of
 * V / G rows, each a multiple of 256): every rank runs dg_head_partials on
 * its shard, the caller gathers the G record blocks (for example an NCCL
 * all-gather into a [G][...] buffer), and every rank (or one) runs
 * dg_merge_partials on all of them.  The result equals dg_denoise_step over
 * the whole vocabulary: the Philox counters and token indices use the
 * global vocabulary index; only the float32 merge order of the softmax
 * partials differs (entropies agree to rounding).  The pages do not describe
 * a sharded step; this is the data-parallel layout of the same method. */

/* Records per canvas row that dg_head_partials writes for a shard of this
 * shape on the current device (shape->V = the shard's rows); the records
 * occupy 7 * B * L * count floats.  0 for an invalid shape. */
int32_t dg_partials_count(const dg_shape* shard_shape);

/* The fused head and sampler over one shard: E_shard holds vocabulary rows
 * v_offset .. v_offset + shard_shape->V - 1 (v_offset a multiple of 256),
 * e_scale_shard their scales (FP8 only).  Writes the per-row partial records
 * (online softmax, argmax, best Gumbel key) to `partials` (device, 16-byte
 * aligned, 7 * B * L * dg_partials_count(shard_shape) floats).  step_idx is
 * a host array as for dg_denoise_step; the workspace is one of
 * dg_workspace_size(shard_shape) bytes. */
dg_status dg_head_partials(const dg_shape* shard_shape, const dg_params* params, int32_t v_offset,
                           const void* h, const void* E_shard, const float* e_scale_shard,
                           const int32_t* step_idx, float* partials,
                           void* workspace, size_t ws_bytes, void* stream);

/* Merge `shards` record blocks of `count` records per row each (laid out
 * [shards][7][B*L][count] as written by dg_head_partials), then selection,
 * renoise and the stop test as dg_denoise_step does.  shape->V is the whole
 * vocabulary (the renoise draws from all of it).  The workspace may be the
 * one the head used (any workspace for the same B). */
dg_status dg_merge_partials(const dg_shape* shape, const dg_params* params, const float* partials,
                            int32_t shards, int32_t count, const int32_t* step_idx,
                            const uint8_t* has_prev, const uint8_t* active,
                            int32_t* canvas, int32_t* prev_argmax,
                            uint8_t* accept, float* entropy, int32_t* sampled,
                            int32_t* argmax, int32_t* stop,
                            void* workspace, size_t ws_bytes, void* stream);

/* ---- diagnostics (no counterpart on the pages; used by the tests) ---- */

/* Text of the last CUDA runtime error met by a call on this host thread
 * ("" if none); static thread-local storage, valid until the next call. */
const char* dg_last_error_message(void);

/* Profiling hook: while set (per host thread), every step records
 * ev_start / ev_stop (cudaEvent_t handles, created by the caller) on its
 * stream immediately before and after the fused head kernel, so its device
 * time can be measured inside a running workload.  NULL, NULL clears it. */
dg_status dg_set_head_events(void* ev_start, void* ev_stop);

/* Self test of the device-side bounded wait: launches one kernel that waits
 * on a barrier nothing ever arrives at, gives up after limit_ns
 * nanoseconds, latches the fault in the workspace and returns normally.
 * The call synchronises `stream` and returns DG_ERR_TIMEOUT when the wait
 * ran out as designed (the context stays usable), DG_OK otherwise. */
dg_status dg_selftest_bounded_wait(uint64_t limit_ns, void* workspace, size_t ws_bytes,
                                   void* stream);

/* The same self test against the fault latch of dg_denoise_step_noalloc's
 * array; returns what dg_noalloc_status() then reports (DG_ERR_TIMEOUT when
 * the wait ran out as designed; the latch is cleared). */
dg_status dg_noalloc_selftest_bounded_wait(uint64_t limit_ns, void* stream);

/* For n Philox words (device uint32 [n]) write the specified float32
 * Gumbel noise g32 = -L(-L(u)) (device float [n]) and the approximate
 * lg2(E / ln 2), E = -ln u, that the sampler's screening pass uses (device
 * float [n]; its noise is -ln(ln 2) - ln 2 * lg2(E / ln 2)), so tests can
 * compare both with the oracle and bound the approximation over every
 * possible input. */
dg_status dg_debug_gumbel(const uint32_t* words, int32_t n, float* g_exact, float* lg2e_approx,
                          void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DG_H */
