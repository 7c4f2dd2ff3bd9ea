/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse Mixture-of-Experts layer forward.
 *
 * The layer (token-choice routing, dropless unless a capacity is set):
 *   router logits   l = x W_r^T                                   [T, E]
 *   selection key   kappa = l + b        (b: optional per-expert bias)
 *   top-k           the k largest kappa per token, descending, ties -> lower index
 *   gate weights    one of four rules (moe_gating), fp32
 *   dispatch        rows grouped by expert (ascending), tokens ascending inside;
 *                   with a capacity C each expert keeps its first C rows
 *   expert FFN      h = SiLU(x_e Wg^T) * (x_e Wu^T),  o = h Wd^T   (SwiGLU)
 *                   or h = GELU(x_e Wu^T), o = h Wd^T               (moe_expert_act)
 *   combine         y[t] = sum_s w[t,s] o_{t,s} + sum_shared FFN_shared(x[t])
 *                   (a dropped slot adds nothing)
 *
 * Sources (page title, section):
 *   "Mixture of Experts (MoE): routing, expert parallelism, and memory"
 *       -- "How does MoE routing work" (score, softmax, top-k, combine),
 *          "Shared experts" (always-on experts).
 *   "Mixture of Experts: why a model with 671 billion parameters uses only 37"
 *       -- "The router: how a token chooses experts" (a bias-free linear
 *          router, top-k then softmax over the kept scores, per-expert loop),
 *          "How many experts to pick and how to score them: top-k, softmax,
 *          sigmoid" (sigmoid scores normalised over the selected set),
 *          "Capacity factor: when tokens don't fit" (dropless grouping),
 *          "How data centres handle it" (tokens grouped by expert, all expert
 *          multiplies in one launch over a stacked weight matrix).
 *   "Mixture of experts: how MoE works and what it costs"
 *       -- "What mixture of experts means in an LLM" (Mixtral top-2 softmax,
 *          DeepSeek-V3 shared + routed), "Why load balancing is the hard part
 *          of MoE" (bias steers routing, not the gate values).
 *   "Mixture of Experts Explained: Routers, Active Parameters and VRAM"
 *       -- the five router steps (Score, Normalise, Keep the top k,
 *          Renormalise, Run and combine); "a gated feed-forward block with
 *          three matrices".
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or retains them.  Layouts are row-major; weights
 *    are "out x in" (as nn.Linear), so every GEMM is A * B^T with both
 *    operands contiguous along the reduction dimension.
 *  - dtype MOE_BF16: x, weights, x_perm, h, y_perm, y are bfloat16, all
 *    accumulation is fp32.  dtype MOE_F32: every tensor is fp32 and all math is
 *    fp32 on CUDA cores (no TF32).  Routing weights are always fp32, expert ids,
 *    counts, offsets and permutations always int32.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  Argument checks happen on the host before anything is
 *    launched: a failed check returns MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED /
 *    MOE_ERR_WORKSPACE and launches nothing.  A failed launch returns MOE_ERR_CUDA.
 *  - Pointers must be 16-byte aligned.  d_model, d_ff and d_ff_shared must be
 *    multiples of 8.  Limits: 1 <= n_experts <= 1024, 1 <= top_k <= min(16, E),
 *    T * top_k < 2^31, n_shared in {0, 1}.
 *  - `ws` is caller-owned device scratch of at least moe_workspace_bytes(cfg)
 *    bytes, 256-byte aligned.  Its first 16 bytes hold the device status word
 *    that kernels set on a bounded-wait expiry or an out-of-range expert id
 *    (a bounded-wait expiry overrides any other code; otherwise the first
 *    code set stays);
 *    moe_forward clears it on entry; a caller chaining the single-stage entry
 *    points zeroes those 16 bytes before the first of them.  moe_device_status()
 *    reads it.
 *  - Device-side waits (pipeline barriers of the tensor-core GEMMs) are bounded
 *    by cfg->wait_limit_ns (0 = 2 s).  On expiry the kernel drains its own
 *    copies, frees its tensor memory, records MOE_ERR_TIMEOUT in the status
 *    word and returns; it never traps.
 *  - Calls that share a workspace must not overlap on the GPU.
 *  - Device: a call runs on the device that owns its workspace (moe_combine:
 *    y; moe_quantize_e4m3: blob; moe_permute_noalloc: counts), making it
 *    current for the duration of the call and restoring the caller's current
 *    device before returning.  x (moe_forward) must live on that device, and
 *    a stream created on another device is rejected (MOE_ERR_INVALID_ARG);
 *    NULL and the legacy / per-thread default streams are the bound device's.
 *  - Failure injection (tests): with the environment variable MOE_FAULT set to
 *    "launch", every entry point that would launch work returns MOE_ERR_CUDA
 *    after its host-side checks and before any CUDA call, so nothing runs.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* identical to cudaStream_t */
typedef struct CUevent_st* moe_event_t;   /* identical to cudaEvent_t  */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad shape, k > E, ... */
  MOE_ERR_UNSUPPORTED = 2,  /* valid request outside this build's limits      */
  MOE_ERR_WORKSPACE = 3,    /* ws smaller than moe_workspace_bytes(cfg)       */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed              */
  MOE_ERR_TIMEOUT = 5,      /* a bounded device wait expired (status word)    */
  MOE_ERR_BAD_EXPERT_ID = 6 /* moe_permute saw an id outside [0, E) (status)  */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

typedef enum {
  /* softmax over all E kappas, keep the top k, divide by their sum
     ("Mixture of Experts Explained...", router steps 2-4)                    */
  MOE_SOFTMAX_ALL_RENORM = 0,
  /* top-k kappas, softmax over those k
     ("...671 billion parameters uses only 37", "The router"; Mixtral)        */
  MOE_SOFTMAX_TOPK = 1,
  /* sigmoid score per expert, top-k, divide by the sum of the k
     ("...671 billion parameters uses only 37", sigmoid gating; DeepSeek-V3)  */
  MOE_SIGMOID_TOPK_RENORM = 2,
  /* softmax over all E kappas, the k kept probabilities used as they are
     ("Mixture of Experts (MoE): routing...", "How does MoE routing work";
     with k = 1 the raw router probability of top-1 routing, "Mixture of
     Experts Explained...", "Why top-1 routing cannot renormalise")          */
  MOE_SOFTMAX_ALL_NO_RENORM = 3
} moe_gating;

typedef enum {
  /* gated expert, three matrices: h = SiLU(x Wg^T) * (x Wu^T), o = h Wd^T;
     w_gate_up [E, 2f, d] (rows 0..f-1 Wg, f..2f-1 Wu)                       */
  MOE_ACT_SWIGLU = 0,
  /* plain expert, two matrices: h = GELU(x Wu^T) (exact erf form), o = h Wd^T;
     the w_gate_up argument holds W_up [E, f, d]
     ("Mixture of Experts Explained...", the runnable top-k MoE build)       */
  MOE_ACT_GELU = 1
} moe_expert_act;

typedef enum {
  /* expert weights in dtype (bf16 or fp32) */
  MOE_W_NATIVE = 0,
  /* 8-bit experts: every expert weight tensor (w_gate_up, w_down, ws_gate_up,
     ws_down) is an E4M3 blob made by moe_quantize_e4m3: FP8 E4M3 codes of the
     [rows, cols] matrix (rows = E*2f or E*f, resp. E*d; cols = d, resp. f),
     then at byte offset align256(rows*cols) one fp32 scale per row.  The
     expert inputs (x_perm, the shared expert's x) and h are quantised per
     token row the same way inside the call; accumulation is fp32, h and the
     outputs stay bf16.  Requires dtype MOE_BF16 and d_model, d_ff, d_ff_shared
     multiples of 16.  The pages name 8-bit experts ("Mixture of Experts: why
     a model...", "How data centres handle it") without fixing a scheme; per-
     row absolute-max scaling to E4M3 is the one used here.                 */
  MOE_W_E4M3 = 1
} moe_weight_format;

typedef struct {
  int64_t T;                /* tokens                                          */
  int32_t d_model;          /* d                                               */
  int32_t n_experts;        /* E routed experts                                */
  int32_t top_k;            /* k                                               */
  int32_t d_ff;             /* f, routed expert hidden width                   */
  int32_t n_shared;         /* S always-on shared experts (0 or 1)             */
  int32_t d_ff_shared;      /* f_s                                             */
  int32_t dtype;            /* moe_dtype                                       */
  int32_t gating;           /* moe_gating                                      */
  int32_t bias_select_only; /* sigmoid rule: bias steers selection only        */
  int32_t expert_act;       /* moe_expert_act (routed and shared experts)      */
  int64_t wait_limit_ns;    /* bound on any single device wait; 0 = 2 s        */
  float capacity_factor;    /* 0: dropless.  > 0: every expert keeps only its
                               first C = ceil(T*k/E * capacity_factor)
                               assignments in token order; the rest skip it
                               ("Mixture of Experts: why a model...",
                               "Capacity factor: when tokens don't fit";
                               "Mixture of Experts Explained...", expert
                               capacity).  A dropped slot adds nothing to its
                               token's output; the other slots keep their
                               weights.                                        */
  int32_t weight_format;    /* moe_weight_format of the expert weights         */
} moe_config;

/* Bytes of scratch every entry point below accepts for this config
   (x_perm, h, y_perm, shared-expert buffers, routing and dispatch metadata,
   status word).  0 on an invalid config. */
size_t moe_workspace_bytes(const moe_config* cfg);

/* Static, NUL-terminated description of a status code. */
const char* moe_status_string(moe_status s);

/* Bytes of an E4M3 weight blob for a [rows, cols] matrix: align256(rows*cols)
   code bytes, then rows fp32 scales; 0 when cols is not a positive multiple
   of 16. */
size_t moe_e4m3_weight_bytes(int64_t rows, int64_t cols);

/* Quantise a bf16 [rows, cols] row-major matrix into an E4M3 blob (see
   MOE_W_E4M3): per row s = max|w| / 448 (1 for a zero row), codes =
   E4M3(w / s) rounded to nearest even with saturation.  blob: device,
   256-byte aligned, moe_e4m3_weight_bytes(rows, cols) bytes.  Asynchronous
   on stream; allocates nothing. */
moe_status moe_quantize_e4m3(const void* src, int64_t rows, int32_t cols, void* blob, moe_stream_t stream);

/* Rows each expert keeps: ceil(T*k/E * capacity_factor) evaluated in double
   (capped at T, which no expert can exceed) when capacity_factor > 0, T*k
   when it is 0 (dropless); -1 for an invalid config.  Host only.  With a
   capacity C, the dropped slot count of a call is sum_e max(counts[e] - C, 0)
   ("Mixture of Experts Explained...": dropped slots per capacity factor). */
int64_t moe_expert_capacity(const moe_config* cfg);

/* Router + top-k + gate weights, one fused pass.
   Defined by: "Mixture of Experts Explained: Routers, Active Parameters and
   VRAM", the router steps Score, Normalise, Keep the top k and Renormalise;
   "Mixture of Experts: why a model with 671 billion parameters uses only 37",
   "The router: how a token chooses experts" and "How many experts to pick and
   how to score them: top-k, softmax, sigmoid".
   x [T, d] (dtype), w_router [E, d] (dtype), logit_bias [E] fp32 or NULL
   -> topk_ids [T, k] int32 (slots in descending kappa), topk_w [T, k] fp32. */
moe_status moe_router_topk(const moe_config* cfg, const void* x, const void* w_router,
                           const float* logit_bias, int32_t* topk_ids, float* topk_w,
                           void* ws, size_t ws_bytes, moe_stream_t stream);

/* Router penalties of a batch, forward values only (training-side
   quantities; the caller applies their loss weights):
     out[0]  balance loss without alpha: E * sum_e f_e * P_e, with f_e =
             counts[e] / sum(counts) the share of routed slots and P_e the mean
             over tokens of the softmax probability of expert e
             ("Mixture of Experts Explained...", the load-balancing loss of the
             top-1 routing paper, counted over routing slots for top-k);
     out[1]  router z-loss without its weight: the mean over tokens of
             (log sum_e exp l[t,e])^2 ("Mixture of Experts: why a model...",
             "Router z-loss").
   Both use the bias-free router logits l = x W_r^T.  x [T, d], w_router
   [E, d] (dtype), counts [E] int32 (routed slots per expert, as moe_permute
   or moe_forward return them), out [2] fp32 device.  The logits are
   recomputed on the CUDA cores; sums run in a fixed order (deterministic),
   in fp32.  T = 0 writes zeros. */
moe_status moe_router_aux_losses(const moe_config* cfg, const void* x, const void* w_router,
                                 const int32_t* counts, float* out, void* ws, size_t ws_bytes,
                                 moe_stream_t stream);

/* Dispatch: a stable counting sort of the T*k assignments by expert, then
   the row gather.
   Defined by: "Mixture of Experts: why a model with 671 billion parameters
   uses only 37", "How data centres handle it" (tokens grouped by their
   assigned expert) and "Capacity factor: when tokens don't fit" (dropless
   grouping; a capacity drops the overflow).
   topk_ids [T, k] int32, x [T, d]
   -> counts [E] (assignments routed to each expert, before any capacity cut),
      offsets [E+1] (exclusive scan of the rows each expert keeps:
      min(counts[e], C) with a capacity C, counts[e] when dropless;
      offsets[E] = rows kept, T*k when dropless),
      perm [offsets[E]] (perm[row] = t*k + s),
      row_of [T*k] (inverse of perm; -1 for a dropped assignment),
      x_perm [offsets[E], d] (x_perm[row] = x[perm[row] / k]).
   Rows inside an expert follow ascending token order, so with a capacity an
   expert keeps its first C assignments in token order.
   Ids outside [0, E) are skipped and flag MOE_ERR_BAD_EXPERT_ID in the status
   word (read it with moe_device_status). */
moe_status moe_permute(const moe_config* cfg, const int32_t* topk_ids, const void* x,
                       int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* row_of,
                       void* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_permute without a workspace.  No counterpart on the pages: this is a
   calling convention for callers that cannot provide device scratch when they
   dispatch -- e.g. a plug-in whose host framework owns every device
   allocation and passes it only tensors, or a serving loop whose memory policy
   forbids allocating once it runs (an allocation there may stall the device,
   or fail with out-of-memory in the middle of a step).
   Same arguments and results as moe_permute, minus ws/ws_bytes.  The
   per-(expert, chunk) histogram lives in a 256 KiB array compiled into the
   library (held on every GPU that loads it until the process exits):
   n_experts * ceil(T*k / 2048) must be <= 65536, else MOE_ERR_UNSUPPORTED and
   nothing runs; a config moe_permute rejects gets the same status here.  It
   runs on the device that owns `counts` and restores the caller's current
   device before returning (as every entry point does).  The call
   allocates nothing.  The first call on a device looks up the array's device
   address (with that device current) and keeps it for the rest of the process;
   make that first call before any stream capture, and do not reset the device
   afterwards.  All calls share the one array: calls that overlap on the GPU
   (different streams, or several host threads) race and must be serialised by
   the caller.  Every call rewrites the part of the array it reads, so nothing
   has to be cleared between calls.  There is no status word: an id outside
   [0, E) is skipped (its row_of is -1) and is not reported. */
moe_status moe_permute_noalloc(const moe_config* cfg, const int32_t* topk_ids, const void* x,
                               int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* row_of,
                               void* x_perm, moe_stream_t stream);

/* Grouped SwiGLU experts over the dispatched rows.
   Defined by: "Mixture of Experts: why a model with 671 billion parameters
   uses only 37", "How data centres handle it" (every expert multiply in one
   launch over a stacked weight matrix); the expert is the "gated feed-forward
   block with three matrices" of "Mixture of Experts Explained: Routers,
   Active Parameters and VRAM", read as SwiGLU (or its two-matrix GELU
   expert with MOE_ACT_GELU).
   x_perm [T*k, d], offsets [E+1] (device), w_gate_up [E, 2f, d] (rows 0..f-1
   gate, f..2f-1 up), w_down [E, d, f] -> y_perm [T*k, d].
   Rows [offsets[e], offsets[e+1]) use expert e; h [T*k, f] lives in ws. */
moe_status moe_grouped_ffn(const moe_config* cfg, const void* x_perm, const int32_t* offsets,
                           const void* w_gate_up, const void* w_down, void* y_perm,
                           void* ws, size_t ws_bytes, moe_stream_t stream);

/* Weighted un-permute: y[t] = sum_s topk_w[t,s] * y_perm[row_of[t*k+s]] (+ y_shared[t]).
   Defined by: "Mixture of Experts Explained: Routers, Active Parameters and
   VRAM", router step "Run and combine"; "Mixture of Experts (MoE): routing,
   expert parallelism, and memory", "Shared experts" (the always-on add).
   y_shared [T, d] or NULL.  fp32 accumulation, y in dtype. */
moe_status moe_combine(const moe_config* cfg, const void* y_perm, const int32_t* row_of,
                       const float* topk_w, const void* y_shared, void* y, moe_stream_t stream);

/* The whole layer: router_topk -> permute -> grouped_ffn (+ shared expert) -> combine.
   Defined by: "Mixture of Experts: why a model with 671 billion parameters
   uses only 37", "The router: how a token chooses experts" (the layer's
   forward pass as a per-expert loop), computed here with grouped launches;
   "Mixture of experts: how MoE works and what it costs", "What mixture of
   experts means in an LLM" (routed plus shared experts).
   ws_gate_up [S, 2f_s, d] and ws_down [S, d, f_s] when n_shared = 1, else NULL.
   opt_topk_ids [T,k], opt_topk_w [T,k], opt_counts [E]: optional outputs (NULL = none).
   Clears the status word first; no host synchronisation inside.  The kernels
   after the router are launched with programmatic stream serialisation: each
   may be scheduled while its predecessor finishes and waits on the device
   before reading its predecessor's output, so stream order is kept as with
   plain launches.  With 8-bit experts the dispatched rows are quantised while
   they are gathered (no bf16 copy is made). */
moe_status moe_forward(const moe_config* cfg, const void* x, const void* w_router,
                       const float* logit_bias, const void* w_gate_up, const void* w_down,
                       const void* ws_gate_up, const void* ws_down, void* y,
                       int32_t* opt_topk_ids, float* opt_topk_w, int32_t* opt_counts,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_forward with stage markers, for per-stage timing of the layer step as
   it runs (the pages have no counterpart; it is a tracing aid).  Same
   arguments, checks, launches and results as moe_forward, plus
   stage_events[6] (caller-created CUDA events; any entry, or the whole
   array, may be NULL), each recorded on `stream` at a stage boundary:
     [0] before the first operation of the step (the status-word clear),
     [1] after the router, [2] after the dispatch (and the 8-bit gather),
     [3] after the routed experts' GEMMs, [4] after the shared expert's
     GEMMs (equal to [3] without one), [5] after the combine.
   Elapsed time between consecutive events is that stage's device time.  A
   recorded event separates two launches, so the next kernel of the chain
   starts after the marker instead of overlapping its predecessor's tail. */
moe_status moe_forward_traced(const moe_config* cfg, const void* x, const void* w_router,
                              const float* logit_bias, const void* w_gate_up, const void* w_down,
                              const void* ws_gate_up, const void* ws_down, void* y,
                              int32_t* opt_topk_ids, float* opt_topk_w, int32_t* opt_counts,
                              void* ws, size_t ws_bytes, moe_stream_t stream,
                              const moe_event_t* stage_events);

/* Synchronises `stream` and returns the status word of `ws`: MOE_OK,
   MOE_ERR_TIMEOUT or MOE_ERR_BAD_EXPERT_ID (or MOE_ERR_CUDA). */
moe_status moe_device_status(const void* ws, size_t ws_bytes, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
