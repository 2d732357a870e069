/*
 * l4moe.h -- C ABI of a B200 (sm_100a) implementation of the Llama-4 style
 * mixture-of-experts feed-forward layer: top-1 routing with a sigmoid gate on
 * the routed expert's input, a SwiGLU routed expert and an always-on SwiGLU
 * shared expert whose outputs are summed.
 *
 * What the layer computes (per token t, input row x_t of width d):
 *   - router logits l_e = x_t . W_router[:, e] (+ optional bias b_e), fp32;
 *     superteams.ai "Llama 4" glossary, section "Mixture of Experts: Why
 *     Total and Active Parameters Diverge" (routing sketch: one logit per
 *     expert);
 *   - the single expert e* with the largest logit (lowest index on ties),
 *     same section (top-1 routing) and KerasFormers "Llama 4" API table
 *     (num_experts_per_tok = 1);
 *   - gate g = sigmoid(l_{e*}) applied to the routed expert's INPUT:
 *     KerasFormers "Llama 4", section "What is unusual about the block";
 *   - routed output  y_r = SwiGLU_{e*}(g * x_t), shared output
 *     y_s = SwiGLU_shared(x_t), out_t = y_s + y_r: glossary routing sketch
 *     (shared plus routed) and llm-architectures-explained "Llama 4
 *     Maverick" field table (ffns.moe.* rows: gated experts of width 8192,
 *     one shared expert of width 8192).
 *   SwiGLU_W(u) = (silu(u . Wg) * (u . Wu)) . Wd with silu(z) = z/(1+e^-z).
 * l4moe_set_top_k selects k > 1 experts per token instead (the k largest
 * logits, each expert gated by the sigmoid of its own logit, the k routed
 * outputs added to the shared one).
 * With E = 0 the layer is the dense SwiGLU feed-forward of the layers
 * without experts (the Maverick field table's dense width 16384 as Fs):
 * W_router, W_gate_up and W_down are unused (may be NULL) and F may be 0.
 *
 * Layouts (all row-major, "x @ W" orientation, element = the dtype below):
 *   x          [T, d]        W_router  [d, E]
 *   W_gate_up  [d, 2F] per expert: gate columns [0, F), up columns [F, 2F)
 *   W_down     [F, d]  per expert
 *   Ws_gate_up [d, 2Fs], Ws_down [Fs, d]  (shared expert)
 *   out        [T, d]
 * Dtypes (l4moe_dtype):
 *   L4MOE_F32       every tensor fp32 (tensor-core math in TF32, fp32 accumulate)
 *   L4MOE_BF16      every tensor bf16 (bf16 MMA, fp32 accumulate)
 *   L4MOE_FP8_E4M3  expert and shared weights OCP E4M3 with one fp32 scale per
 *                   output column (l4moe_set_weight_scales); x, W_router, out bf16.
 *                   The expert contractions run in f16 (kind::f16 MMA, fp32
 *                   accumulate): weights widened exactly, x and the hidden
 *                   rows held in f16, the column scale applied in fp32.  Each
 *                   token row of x is divided by a power of two that brings
 *                   its largest value within f16's 65504 (1 for rows already
 *                   inside), which the fp32 accumulators get back, so every
 *                   bf16 value of magnitude >= 2^-14 times that scale is
 *                   exact; a hidden value that f16 cannot hold (|h| >= 65520)
 *                   sets L4MOE_ERR_RANGE in the device status.
 *   L4MOE_INT8      expert and shared weights int8 (two's complement, symmetric:
 *                   no zero point) with one fp32 scale per output column, the
 *                   weight-only int8 of KerasFormers "Llama 4", "Lower memory";
 *                   otherwise as L4MOE_FP8_E4M3 (every int8 value is exact in f16).
 *   L4MOE_INT4      expert and shared weights int4 (two's-complement nibbles,
 *                   symmetric) with one fp32 scale per output column, the
 *                   int4 the glossary's "The Llama 4 Herd" and the aibase
 *                   card's "Quantization" name for Scout; packed two per byte
 *                   along the output columns, the even column in the low
 *                   nibble: W_gate_up is [d, F] bytes, W_down [F, d/2] (same
 *                   for the shared expert); otherwise as L4MOE_INT8.
 *
 * Ownership: the caller owns every tensor, the scale vectors, the bias and
 * the stream.  The handle owns only its workspace (unless the caller supplies
 * one) and a cache of TMA descriptors keyed by the weight pointer values.
 * Pointers passed to l4moe_forward must stay valid until the work enqueued on
 * the stream has finished.
 *
 * Errors: every entry point returns a status; argument errors are reported
 * synchronously and launch nothing.  l4moe_forward never synchronises the
 * stream; device-side faults of the kernels' own bounded waits are recorded
 * in a device word that l4moe_check_device_status reads (it synchronises).
 * l4moe_last_error gives a message for the last non-OK status of a handle.
 *
 * Requirements: d, F, Fs multiples of 64; 0 <= E <= 256 (F > 0 when E > 0); all tensor pointers
 * 16-byte aligned.  One handle serves one stream at a time (the workspace is
 * shared by the calls made with it).  The library sees raw pointers, not
 * buffer sizes: every tensor must hold at least the elements its layout above
 * states, or the kernels read or write past it (the Python binding checks
 * shapes and dtypes before it calls in).
 */
#ifndef L4MOE_H
#define L4MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define L4MOE_API __attribute__((visibility("default")))
#else
#define L4MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    L4MOE_OK = 0,
    L4MOE_ERR_ARG = 1,          /* null / out-of-range argument                */
    L4MOE_ERR_DTYPE = 2,        /* unknown dtype or missing 8-bit weight scales */
    L4MOE_ERR_ALIGN = 3,        /* pointer not 16-byte aligned / bad multiple  */
    L4MOE_ERR_CUDA = 4,         /* a CUDA runtime or driver call failed        */
    L4MOE_ERR_WORKSPACE = 5,    /* workspace too small / allocation failed     */
    L4MOE_ERR_TIMEOUT = 6,      /* a kernel's bounded wait ran out             */
    L4MOE_ERR_UNSUPPORTED = 7,  /* device is not sm_100 or feature unavailable */
    L4MOE_ERR_RANGE = 8         /* E4M3 / int8 layers: a hidden value left f16's range */
} l4moe_status;

typedef enum {
    L4MOE_F32 = 0,
    L4MOE_BF16 = 1,
    L4MOE_FP8_E4M3 = 2,
    L4MOE_INT8 = 3,
    L4MOE_INT4 = 4
} l4moe_dtype;

typedef struct {
    int d_model;      /* d  : model width (KerasFormers "Llama 4": embed_dim)       */
    int expert_ffn;   /* F  : routed expert width (Maverick table: d_expert)       */
    int shared_ffn;   /* Fs : shared expert width (Maverick table: d_shared)       */
    int num_experts;  /* E  : routed experts (16 Scout, 128 Maverick); 0 = a dense
                         feed-forward layer: out = SwiGLU_shared(x) alone          */
    l4moe_dtype dtype;
} l4moe_params;

typedef struct l4moe_handle l4moe_handle;

/* Validate the shapes and dtype and create a handle.  Host only; no device
 * work and no allocation on the device.  *out receives the handle.  The
 * handle belongs to the CUDA device current at this call: its forwards must
 * run with that device current (L4MOE_ERR_ARG otherwise). */
L4MOE_API l4moe_status l4moe_create(const l4moe_params *params, l4moe_handle **out);

/* Free the handle, its own workspace and descriptor cache.  Waits for
 * nothing: the caller must ensure no enqueued work still uses it. */
L4MOE_API void l4moe_destroy(l4moe_handle *h);

/* Bytes of device workspace l4moe_forward needs for up to max_tokens tokens
 * with the handle's current experts per token (l4moe_set_top_k) and FP8
 * activation mode (l4moe_set_act_fp8): routing
 * vectors, permutation, group tables, gated expert-ordered input, both
 * hidden activations, fp32 partials, host-path staging.  0 on a bad
 * argument. */
L4MOE_API size_t l4moe_workspace_size(const l4moe_handle *h, int max_tokens);

/* Give the handle a caller-owned device workspace of `bytes` bytes (256-byte
 * aligned) sized for max_tokens tokens.  Without this call, l4moe_forward
 * allocates one itself (cudaMalloc) on first use or when T grows. */
L4MOE_API l4moe_status l4moe_set_workspace(l4moe_handle *h, void *dev_ptr, size_t bytes, int max_tokens);

/* Optional fp32 router bias b[E] (device pointer, NULL = none) added to the
 * logits before the arg-max and the gate.  The pages' router has no bias;
 * this exists to draw skewed expert loads. */
L4MOE_API l4moe_status l4moe_set_router_bias(l4moe_handle *h, const float *bias_dev);

/* Experts per token (default 1, the Llama-4 layer).  k > 1: each token runs
 * its k highest-scoring experts (descending fp32 logit, lower index first on
 * equal values, NaN never selected), each on the input gated by the sigmoid
 * of its own logit, and their outputs add to the shared expert's (the
 * "experts per token" of a token-choice router, torchtune MoE
 * documentation).  1 <= k <= min(4, E), any dtype and expert count.  The
 * routing arrays of l4moe_get_routing then hold T * k entries (entry t * k + j: token t's j-th
 * expert; margin stays [T]: the k-th logit minus the next one).  Changing k
 * frees a workspace the handle allocated (it synchronises the device) and
 * fails with L4MOE_ERR_WORKSPACE when a caller's workspace is too small; the
 * routing arrays then describe the next forward, not the earlier ones. */
L4MOE_API l4moe_status l4moe_set_top_k(l4moe_handle *h, int k);

/* E4M3, int8 or int4 weights only: per-output-column fp32 scales (device
 * pointers).  s_gate_up / s_down are HOST arrays of E device pointers to
 * [2F] / [d] vectors; ss_gate_up [2Fs] and ss_down [d] are the shared
 * expert's.  The dequantised weight is e4m3(q) * scale[column] or
 * q * scale[column].  The pointers are kept, not copied: the vectors must
 * stay valid while the handle runs forwards.  L4MOE_ERR_DTYPE for other
 * dtypes, L4MOE_ERR_ARG for a NULL pointer. */
L4MOE_API l4moe_status l4moe_set_weight_scales(l4moe_handle *h, const float *const *s_gate_up,
                                     const float *const *s_down, const float *ss_gate_up,
                                     const float *ss_down);
/* The same call under its E4M3-era name. */
L4MOE_API l4moe_status l4moe_set_fp8_scales(l4moe_handle *h, const float *const *s_gate_up,
                                  const float *const *s_down, const float *ss_gate_up,
                                  const float *ss_down);

/* FP8 activation mode (on = 1; off = 0, the default), E4M3 weights only.
 * superteams.ai "Llama 4" glossary, "Running Llama 4 Yourself": Maverick is
 * served with FP8 quantisation; the pages fix no activation scaling, so this
 * is an opt-in reading.  Every contraction input row is quantised to E4M3
 * with one fp32 scale for the row: a token's x (before the router's gate,
 * which still scales the routed expert's dequantised input), and each
 * hidden row an expert produces, held in bf16 first:
 *   s = fp32(max|v| / 448) (1 for a row of zeros),
 *   code = E4M3 round-to-nearest-even, saturating, of fp32(v / s),
 * and every tensor-core contraction multiplies E4M3 codes by E4M3 codes
 * (tcgen05 kind::f8f6f4), the weight column scale and the row scale applied
 * to the fp32 accumulator.  The router still reads the bf16 x.  The layer
 * then differs from the bf16-activation one by the quantisation (a few
 * percent of rms(out)).  Changing the mode frees a workspace the handle
 * allocated (it synchronises the device; the mode needs room for the hidden
 * rows' codes) and fails with L4MOE_ERR_WORKSPACE when a caller's workspace
 * is too small.  L4MOE_ERR_DTYPE for other weight types, L4MOE_ERR_ARG for
 * `on` other than 0 or 1. */
L4MOE_API l4moe_status l4moe_set_act_fp8(l4moe_handle *h, int on);

/* Enqueue one forward pass of the layer for T tokens on `stream` (a
 * cudaStream_t, NULL = legacy default stream).  x, W_router, Ws_gate_up,
 * Ws_down, out are device pointers; W_gate_up and W_down are HOST arrays of E
 * device pointers (one weight matrix per expert).  out is fully written.  T = 0
 * enqueues nothing and returns L4MOE_OK.  Asynchronous: no host sync. */
L4MOE_API l4moe_status l4moe_forward(l4moe_handle *h, int T, const void *x, const void *W_router,
                           const void *const *W_gate_up, const void *const *W_down,
                           const void *Ws_gate_up, const void *Ws_down, void *out,
                           void *stream);

/* As l4moe_forward, but x_host and out_host are HOST buffers (pinned memory
 * recommended).  The input copy runs on a copy-in stream of the handle into
 * one of two staging slots of the workspace, the layer runs on `stream`, and
 * the output copy runs on a copy-out stream; events order them, so the
 * copies of consecutive calls overlap each other's layer computation.  Weights
 * stay device pointers.  Asynchronous: x_host must not change and out_host is
 * not complete until the call's output copy has finished -- make a stream
 * wait for it with l4moe_join_host, or call l4moe_check_device_status (which
 * synchronises).  The input copy does not wait for earlier work on `stream`. */
L4MOE_API l4moe_status l4moe_forward_host(l4moe_handle *h, int T, const void *x_host, const void *W_router,
                                const void *const *W_gate_up, const void *const *W_down,
                                const void *Ws_gate_up, const void *Ws_down, void *out_host,
                                void *stream);

/* Allocation-free forward (no counterpart in the pages; an interface for
 * callers that cannot allocate device memory).  Some callers may not call
 * cudaMalloc at all: code running while a CUDA graph is being captured,
 * inside another framework's allocator or memory-pool callbacks, or under a
 * hard memory budget where every byte is pre-reserved.  l4moe_forward
 * allocates its workspace (and a descriptor table) on first use; this entry
 * point instead uses one fixed scratch area compiled into the library, a
 * file-scope device array of L4MOE_STATIC_WORKSPACE_BYTES bytes that every
 * GPU loading the library holds until the process exits.  It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *
 * Arguments and results are those of l4moe_forward (the caller still owns
 * x, the weights and out).  The first call on each device resolves the
 * scratch array's device address (cudaGetSymbolAddress, with that device
 * current) and caches it; make that first call before any stream capture.
 * Fails with L4MOE_ERR_WORKSPACE, launching nothing, when T tokens of this
 * layer do not fit in the scratch area: it holds the device part of the
 * workspace (l4moe_workspace_size without the host-path staging slots,
 * rounded up to 256 bytes) plus 2(E+1) TMA descriptors of 128 bytes (and,
 * for 8-bit weights, the 2(E+1) scale-vector pointers), e.g.
 * about 390 tokens at d_model 5120 and F = Fs = 8192 in bf16 (E4M3 layers
 * also keep x in f16 there: about 350 tokens).  Every call, from any
 * handle, shares the one array: calls
 * whose work overlaps on the GPU (other streams, other threads) race and
 * corrupt each other; serialise them.  The array keeps the last call's
 * contents; the call clears the device error word itself.  Each call copies
 * the handle's weight descriptors (and, for 8-bit weights, its scale-pointer
 * table) from host tables the handle owns into the array; those tables sit at
 * fixed addresses for the handle's life and always describe the weights of
 * the handle's latest call (and scales of its latest l4moe_set_weight_scales).
 * Copies recorded under stream capture read them again at every replay, so
 * such a graph needs its handle alive and still keyed to the graph's weights
 * and scales.  Per-kernel
 * timing is not recorded for these calls, and l4moe_get_routing /
 * l4moe_check_device_status keep referring to the handle's own workspace. */
#define L4MOE_STATIC_WORKSPACE_BYTES (32u << 20)
L4MOE_API l4moe_status l4moe_forward_static(l4moe_handle *h, int T, const void *x, const void *W_router,
                                  const void *const *W_gate_up, const void *const *W_down,
                                  const void *Ws_gate_up, const void *Ws_down, void *out,
                                  void *stream);

/* Make `stream` wait (on the device, no host sync) until the output copies of
 * every l4moe_forward_host call enqueued so far have completed. */
L4MOE_API l4moe_status l4moe_join_host(l4moe_handle *h, void *stream);

/* Device pointers (inside the workspace) to the routing of the last forward
 * enqueued with this handle; valid once that work has run and until the next
 * forward.  Any output pointer may be NULL.
 *   idx[T] int32 expert per token; gate[T] fp32 sigmoid gate; lmax[T] fp32
 *   winning logit; margin[T] fp32 winning minus runner-up logit;
 *   counts[E] int32; offsets[E+1] int32 exclusive prefix of counts;
 *   perm[T] int32 expert-ordered slot -> token (stable by token).
 * With top_k = k > 1, idx, gate, lmax and perm hold T * k entries (entry
 * t * k + j is token t's j-th expert; perm maps a slot to its entry). */
L4MOE_API l4moe_status l4moe_get_routing(const l4moe_handle *h, const int32_t **idx, const float **gate,
                               const float **lmax, const float **margin, const int32_t **counts,
                               const int32_t **offsets, const int32_t **perm);

/* Synchronise `stream` (and the handle's copy-out stream) and read the device
 * error word of the handle's workspace: L4MOE_OK, L4MOE_ERR_TIMEOUT (a
 * bounded wait ran out), L4MOE_ERR_RANGE (an E4M3 / int8 layer met a hidden
 * value beyond f16's range: that forward's output is not valid), L4MOE_ERR_ARG
 * (an expert index out of range reached the permutation) or L4MOE_ERR_CUDA.
 * Clears the word. */
L4MOE_API l4moe_status l4moe_check_device_status(l4moe_handle *h, void *stream);

/* Self-test of the device failure path (no counterpart in the pages): enqueue
 * on `stream` one small kernel that waits, with a limit of limit_ms
 * milliseconds (0 < limit_ms <= 1000), for an mbarrier phase that nothing
 * completes.  The wait gives up as every bounded wait of the layer's kernels
 * does -- it records a timeout bit in the handle's device error word and the
 * kernel returns -- so the next l4moe_check_device_status returns
 * L4MOE_ERR_TIMEOUT and clears the word.  Nothing faults or hangs; the
 * context stays usable.  Allocates the handle's workspace if it has none. */
L4MOE_API l4moe_status l4moe_selftest_wait(l4moe_handle *h, double limit_ms, void *stream);

/* How the last forward on this handle was launched (all zero before the
 * first): split_gate_up / split_down, the split-K ranges of the two GEMMs
 * (1 = none); small_routing, routing, top-k, permutation and row copy in one
 * launch (batches of up to 16 tokens with experts); early_shared, the
 * gate/up launch began with the shared expert's tiles while that routing
 * launch was still running; fused, gate/up and down ran as one launch (the
 * kernel-timing slot of gate/up then covers both, the down slot only its
 * finish); small_tiles, the GEMMs used the configuration for groups of at
 * most 64 rows.  L4MOE_ERR_ARG for a null pointer. */
typedef struct {
    int split_gate_up, split_down, small_routing, early_shared, fused, small_tiles;
} l4moe_plan;
L4MOE_API l4moe_status l4moe_get_plan(const l4moe_handle *h, l4moe_plan *plan);

/* Per-kernel timing.  `mask` selects kernel slots (bit i = slot i; 0 turns
 * timing off; L4MOE_TIME_ALL every slot; anything else: L4MOE_ERR_ARG).
 * For each selected slot l4moe_forward records a CUDA event before and
 * after the kernel(s) of that slot, on the caller's stream, so the durations
 * are those of the real launches in place (every event pair adds a little
 * to the step, so time only what is needed).  Kernel slots: 0 router
 * (with the dispatch when a top-1 tensor-core router finishes it; the
 * whole routing for batches of up to 16 tokens), 1 permute (a separate
 * dispatch launch, when there is one), 2 row copy, 3 gate/up GEMM (+ its
 * split-K finish), 4 down GEMM + finish, 5 hidden-row quantisation of the
 * FP8 activation mode (L4MOE_NUM_KERNELS); a slot with no launch in a
 * forward records nothing.  l4moe_read_timing synchronises on the last recorded
 * event, adds every recorded pair to ms[slot] and launches[slot] (arrays of
 * at least L4MOE_NUM_KERNELS entries, accumulated into), and recycles the
 * events.  Returns L4MOE_ERR_CUDA if an event call fails. */
#define L4MOE_NUM_KERNELS 6
#define L4MOE_TIME_ALL ((1 << L4MOE_NUM_KERNELS) - 1)
L4MOE_API l4moe_status l4moe_set_timing(l4moe_handle *h, int mask);
L4MOE_API l4moe_status l4moe_read_timing(l4moe_handle *h, double *ms, uint64_t *launches);
L4MOE_API const char *l4moe_kernel_name(int slot);

/* Number of kernels this handle has launched so far. */
L4MOE_API uint64_t l4moe_launch_count(const l4moe_handle *h);

/* Message for the handle's last non-OK status ("" if none); h may be NULL
 * for errors of l4moe_create. */
L4MOE_API const char *l4moe_last_error(const l4moe_handle *h);

/* Static name of a status code. */
L4MOE_API const char *l4moe_status_string(l4moe_status s);

/* ABI version (major * 100 + minor). */
L4MOE_API int l4moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* L4MOE_H */
