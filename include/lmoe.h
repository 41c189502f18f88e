/*
 * lmoe.h - C ABI of a B200 (sm_100a) LatentMoE expert layer, forward pass.
 *
 * The layer (LatentMoE, "Nemotron 3 Super" notes on guokunwang.com, section 3.2; shapes from the
 * section 3.1 architecture table), per token x in R^d:
 *   logits = W_r x (+ b)                       gating network, full dimension d
 *   S, g   = top-K of the logits (value desc, lower expert index first on ties);
 *            g = softmax over the K selected logits
 *   h      = W_down x                          W_down in R^{l x d}
 *   z      = sum_k g_k * W2_{S_k} sqrelu(W1_{S_k} h)   routed experts in the latent space l -> m -> l
 *   y      = W_up z + W_s2 sqrelu(W_s1 x)      W_up in R^{d x l}; shared expert d -> m_s -> d
 * where sqrelu(v) = max(v, 0)^2 elementwise.  The pages leave the expert nonlinearity, the router
 * normalisation and the NVFP4 block size open; this library fixes them to squared ReLU (non-gated,
 * no biases), softmax over the selected K, and 16-element E2M1 blocks with E4M3 block scales and an
 * fp32 per-tensor scale.
 *
 * Conventions
 *   - Every call returns lmoe_status; nothing throws across the ABI.
 *   - Matrices are row-major [out, in] (the pages' W_down in R^{l x d}, W_up in R^{d x l}).
 *   - bf16 means IEEE bfloat16 bit patterns (uint16).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Device calls are asynchronous on
 *     it; no call below synchronises the host unless it says so.
 *   - Device pointers must be 16-byte aligned; a misaligned pointer returns LMOE_ERR_INVALID_ARG.
 *   - Thread safety: one handle must not be used by two host threads at once; forward calls on one
 *     handle share its workspace, so two forward calls on different streams must not overlap.
 */
#ifndef LMOE_H
#define LMOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct lmoe_ctx* lmoe_handle;

typedef enum {
  LMOE_OK = 0,
  LMOE_ERR_INVALID_ARG = 1,    /* null/misaligned pointer, bad enum value */
  LMOE_ERR_SHAPE = 2,          /* T > max_tokens, T < 0 */
  LMOE_ERR_UNSUPPORTED = 3,    /* a config this build does not implement (see lmoe_create) */
  LMOE_ERR_OOM = 4,            /* device allocation failed */
  LMOE_ERR_CUDA = 5,           /* a CUDA runtime/driver call failed */
  LMOE_ERR_NOT_LOADED = 6,     /* forward before lmoe_load_weights */
  LMOE_ERR_DEVICE_TIMEOUT = 7, /* a kernel's bounded wait gave up (see lmoe_get_device_status) */
  LMOE_ERR_DEVICE_INDEX = 8,   /* a kernel found an out-of-range index and skipped the access */
  LMOE_ERR_NO_DEVICE = 9       /* no sm_100 device, or the device index is invalid */
} lmoe_status;

typedef enum { LMOE_PREC_BF16 = 0, LMOE_PREC_NVFP4 = 1 } lmoe_precision;
typedef enum { LMOE_DTYPE_BF16 = 0, LMOE_DTYPE_F32 = 1 } lmoe_dtype;

typedef struct {
  int32_t d;           /* model dimension (multiple of 64) */
  int32_t latent;      /* latent dimension l (multiple of 64), or 0 for the standard MoE that LatentMoE
                          replaces ("Nemotron 3 Super" notes, section 3.2): experts d -> m -> d on x
                          itself, no W_down / W_up, y = sum_k g_k W2 sqrelu(W1 x) + shared expert
                          (bf16 precision only) */
  int32_t n_experts;   /* N, a multiple of 16, at most 1024 */
  int32_t top_k;       /* K, 1..min(32, N) */
  int32_t expert_ffn;  /* m, routed expert hidden (multiple of 64) */
  int32_t shared_ffn;  /* m_s, shared expert hidden (multiple of 64) */
  int32_t max_tokens;  /* largest T a forward call may pass; sizes the workspace */
  int32_t precision;   /* lmoe_precision: NVFP4 quantises routed+shared experts (weights and inputs);
                          NVFP4 needs d, latent, expert_ffn and shared_ffn to be multiples of 128 */
  int32_t has_router_bias; /* 1: a per-expert fp32 bias is added to the router logits */
  int32_t weight_scale;    /* NVFP4 weight block scales (lmoe_weight_scale); ignored for bf16 */
  int32_t ep_world;        /* expert parallelism: 0 or 1 = this layer holds every expert; G in 2..8 = this
                              layer is rank ep_rank of G ranks and holds only experts [ep_rank * N / G,
                              (ep_rank + 1) * N / G) (bf16 LatentMoE only; N a multiple of 16 * G).  Such a
                              layer runs through lmoe_ep_dispatch / lmoe_ep_experts / lmoe_ep_combine, and
                              lmoe_forward returns LMOE_ERR_UNSUPPORTED */
  int32_t ep_rank;         /* 0 .. ep_world - 1 */
} lmoe_config;

/* How the NVFP4 quantiser picks a weight block's E4M3 scale.  AMAX: s = E4M3(amax_block / (6 g)).
 * MSE: the per-block MSE weight quantiser that the "Nemotron 3 Super" notes (section 4.2, the NVFP4
 * quantisation ablation) name but do not define, read here as: among the AMAX scale (code c0), the
 * next larger E4M3 value and the six next smaller ones (codes c0, c0+1, c0-1 .. c0-6, kept in
 * 1..0x7E), the first, in that order, with the strictly smallest fp32 sum of squared block
 * reconstruction errors.  Activations always use AMAX. */
typedef enum { LMOE_WSCALE_AMAX = 0, LMOE_WSCALE_MSE = 1 } lmoe_weight_scale;

/* Device pointers to the caller's weights, all of element type `dtype`, row-major [out, in].
 * With LMOE_DTYPE_F32 the router stays fp32 (scored with fp32 FMAs) and every other matrix is
 * converted to bf16 (round to nearest even) at load.  The library copies everything into its own
 * memory; the caller may free these buffers once `stream` has passed the load. */
typedef struct {
  const void* w_router;  /* [N, d] */
  const float* b_router; /* [N] fp32, or NULL (required iff has_router_bias) */
  const void* w_down;    /* [l, d]   (W_down); NULL for a standard MoE (latent == 0), else required */
  const void* w_up;      /* [d, l]   (W_up); NULL for a standard MoE, else required */
  const void* w1;        /* [N, m, l] expert up matrices ([N, m, d] for a standard MoE; [N / G, m, l], the
                            owned experts in order, for an expert-parallel layer) */
  const void* w2;        /* [N, l, m] expert down matrices (likewise) */
  const void* ws1;       /* [m_s, d] shared expert */
  const void* ws2;       /* [d, m_s] shared expert */
  int32_t dtype;         /* lmoe_dtype */
} lmoe_weights;

/* Create a layer on CUDA device `device` and allocate its workspace for cfg->max_tokens tokens.
 * Errors: INVALID_ARG (null), UNSUPPORTED (a dimension not a multiple of 64, N not a multiple of 16
 * or above 1024, K > 32, K > N), NO_DEVICE (device missing or not compute capability 10.0), OOM. */
lmoe_status lmoe_create(const lmoe_config* cfg, int device, lmoe_handle* out);

/* Copy (and, for NVFP4, quantise) the weights into library-owned device memory, enqueued on
 * `stream`.  May be called again to replace the weights. */
lmoe_status lmoe_load_weights(lmoe_handle h, const lmoe_weights* w, void* stream);

/* y = LatentMoE(x) for T tokens, all pointers on the device:
 *   x         [T, d]  bf16, read only
 *   y         [T, d]  bf16, written
 *   topk_idx  [T, K]  int32 expert ids per token in slot order, written; may be NULL
 *   topk_gate [T, K]  fp32 softmax gates, written; may be NULL
 * T = 0 returns LMOE_OK and enqueues nothing.  T > max_tokens: LMOE_ERR_SHAPE.
 * Enqueued on `stream`; device-side faults are reported by lmoe_get_device_status. */
lmoe_status lmoe_forward(lmoe_handle h, const void* x, int32_t T, void* y, int32_t* topk_idx, float* topk_gate,
                         void* stream);

/* Same as lmoe_forward, with x/y/topk_idx/topk_gate in HOST memory (pinned memory gives
 * asynchronous copies).  The host-to-device copy of x, the layer and the device-to-host copies of
 * the outputs are all ordered after earlier work on `stream`, and later work on `stream` is ordered
 * after them; the caller synchronises before reading the outputs.  BF16 layers with T >= 8192 run
 * the batch in chunks of 4096 tokens: each chunk's input copy and output copies run on two streams
 * the handle creates on first use, overlapping the layer's work on the neighbouring chunks.  Every
 * token's routing is the one-call forward's; y can differ from it in rounding only (the chunks'
 * expert-up GEMM may take another tile shape).  Staging buffers for max_tokens are allocated on the
 * first call. */
lmoe_status lmoe_forward_host(lmoe_handle h, const void* x_host, int32_t T, void* y_host, int32_t* topk_idx_host,
                              float* topk_gate_host, void* stream);

/* Copy one NVFP4-quantised weight matrix back to the host in plain row-major form (synchronous).
 *   which  0: W1 of expert `index` [m, l]   1: W2 of expert `index` [l, m]
 *          2: W_s1 [m_s, d]                 3: W_s2 [d, m_s]
 *   codes_host  [rows, K/2] bytes, element 2i in the low nibble (E2M1: bit 3 sign, bits 0-2
 *               magnitude index into {0, 0.5, 1, 1.5, 2, 3, 4, 6})
 *   scales_host [rows, K/16] E4M3 block scales, one per 16 consecutive K elements
 *   gscale_host fp32 tensor scale; a weight element is code * scale * gscale.
 * Errors: UNSUPPORTED unless the handle was created with LMOE_PREC_NVFP4; NOT_LOADED; SHAPE for a
 * bad `which` / `index`. */
lmoe_status lmoe_export_nvfp4(lmoe_handle h, int32_t which, int32_t index, uint8_t* codes_host,
                              uint8_t* scales_host, float* gscale_host);

/* Synchronise the handle's device and return the sticky device status raised by any kernel since
 * the last call (DEVICE_TIMEOUT or DEVICE_INDEX), then clear it.  LMOE_OK if none. */
lmoe_status lmoe_get_device_status(lmoe_handle h);

/* Intermediate buffers of the last forward call, for inspection and tests (device pointers owned by
 * the handle, valid until the next forward / destroy).  `count` receives the element count. */
typedef enum {
  LMOE_BUF_LOGITS = 0,     /* fp32 [T, N]   router logits (bias not included) */
  LMOE_BUF_COUNTS = 1,     /* int32 [N]     assignments per expert */
  LMOE_BUF_OFFSETS = 2,    /* int32 [N+1]   exclusive prefix sum of counts */
  LMOE_BUF_ROW_OF = 3,     /* int32 [T*K]   grouped row of assignment (t, k) */
  LMOE_BUF_TOK_OF_ROW = 4, /* int32 [T*K]   token of grouped row r */
  LMOE_BUF_H = 5,          /* bf16 [T, l]   latent h = W_down x (UNSUPPORTED for a standard MoE) */
  LMOE_BUF_Z = 6,          /* bf16 [T, l + m_s] columns 0..l-1: latent sum z; the rest: sqrelu(W_s1 x) */
  LMOE_BUF_U = 7,          /* bf16 [T*K, m] expert hidden activations, grouped rows (bf16 precision) */
  /* NVFP4 precision only: packed E2M1 codes [rows, K/2] (element 2i in the low nibble) and the E4M3
   * block scales of the quantised activations, and the fp32 shared-expert output.  Scales are in
   * tile-local 512-byte atoms, the layout the block-scaled GEMM reads: with the forward's token tile
   * of R rows (64 when T*K <= 48*N, else 192), nra = ceil(R / 128), S = ceil(K / 256), the scale of
   * row j of tile tile (grouped tensors: tiles restart at each expert's first row) and 16-element
   * block b is at byte (((tile*S + b/16)*4 + (b/4)%4)*nra + j/128)*512 + (j%32)*16 + ((j%128)/32)*4
   * + b%4; with 192-row tiles every atom is stored four times in a row (multiply the atom index, the
   * part before *512, by 4 and add 512 per copy).  The count covers the allocation for max_tokens. */
  LMOE_BUF_XQ = 8,         /* x codes [T, d/2] */
  LMOE_BUF_X_SF = 9,       /* x scales */
  LMOE_BUF_HQ = 10,        /* h codes, grouped rows [T*K, l/2] */
  LMOE_BUF_H_SF = 11,      /* h scales, grouped rows */
  LMOE_BUF_UQ = 12,        /* u codes, grouped rows [T*K, m/2] */
  LMOE_BUF_U_SF = 13,      /* u scales */
  LMOE_BUF_USQ = 14,       /* u_s codes [T, m_s/2] */
  LMOE_BUF_US_SF = 15,     /* u_s scales */
  LMOE_BUF_Y_S = 16,       /* fp32 [T, d]: W_s2 u_s */
  LMOE_BUF_ACT_SCALE = 17  /* fp32 [2]: tensor scales of x and h in the last forward */
} lmoe_buffer;
lmoe_status lmoe_inspect(lmoe_handle h, int32_t which, void** dev_ptr, int64_t* count);

/* Per-stage device timing of forward calls (CUDA events recorded on the forward's own stream
 * between consecutive kernels).  lmoe_profile(h, 1) clears the record and starts recording the next
 * forward calls (at most 1024); lmoe_profile(h, 0) stops.  lmoe_profile_read synchronises on the
 * recorded events and returns, per stage, the summed milliseconds over the recorded calls, the
 * number of recorded calls, and the number of kernel launches one forward call makes. */
typedef enum {
  LMOE_STAGE_ROUTER = 0,      /* router logits + W_down (one fused GEMM when the router is bf16) */
  LMOE_STAGE_SHARED_UP = 1,   /* sqrelu(W_s1 x) */
  LMOE_STAGE_TOPK = 2,        /* top-K, softmax gates, per-chunk expert histogram */
  LMOE_STAGE_GROUPING = 3,    /* expert offsets and grouped-GEMM work lists */
  LMOE_STAGE_SCATTER = 4,     /* stable row assignment + gather of latent rows */
  LMOE_STAGE_EXPERT_UP = 5,   /* u = sqrelu(W1_e h), grouped */
  LMOE_STAGE_EXPERT_DOWN = 6, /* o = g * W2_e u, grouped */
  LMOE_STAGE_COMBINE = 7,     /* z = sum_k o */
  LMOE_STAGE_OUTPUT = 8,      /* y = W_up z + W_s2 u_s */
  LMOE_NUM_STAGES = 9
} lmoe_stage;
lmoe_status lmoe_profile(lmoe_handle h, int32_t enable);
lmoe_status lmoe_profile_read(lmoe_handle h, double* stage_ms /* [LMOE_NUM_STAGES] */, int32_t* forwards,
                              int32_t* launches_per_forward);

/* Routing of T tokens from precomputed router logits WITHOUT allocating device memory.
 *
 * The paper has no counterpart; this entry point exists for callers that cannot allocate on their
 * call path: cudaMalloc may synchronise the device (stalling the caller's other streams), and a
 * process whose device memory is fully reserved by its own allocator (for example a serving engine
 * that pre-reserves HBM for its caches) would get an out-of-memory error from it.
 *
 * Computes exactly what lmoe_forward's routing stage computes: top-K of (logits + bias) per token
 * (value desc, lower index first on ties), softmax over the K selected values, and the stable
 * expert grouping.  All pointers are device pointers owned by the caller, 16-byte aligned:
 *   logits    [T, N] fp32, read       bias [N] fp32 or NULL, read
 *   topk_idx  [T, K] int32, written   topk_gate [T, K] fp32, written
 *   counts    [N] int32, written      offsets [N + 1] int32 (exclusive prefix sum), written
 *   row_of    [T * K] int32 grouped row of assignment (t, k), written
 *   status    one uint32 word (4-byte aligned), or NULL: the call sets it to 0 on `stream`, and the
 *             kernels OR into it the device status bits that lmoe_get_device_status reports for a
 *             layer (1: a bounded wait gave up; 2: an out-of-range expert id or row was skipped, and
 *             row_of holds -1 for that assignment).  Read it after synchronising `stream`.  With
 *             NULL such events are not reported.
 * Logits (plus bias) must be finite; NaN logits give in-range but unspecified expert ids.
 * Limits: 1 <= N <= 1024, 1 <= K <= min(32, N), T * K <= 131072; beyond them the call returns
 * LMOE_ERR_UNSUPPORTED (N, K) or LMOE_ERR_SHAPE (T), and enqueues nothing.  T = 0 returns LMOE_OK.
 * Intermediate results live in one 2 MiB array in the library's static device memory, which every
 * GPU that loads the library holds until the process exits.  That array is shared by every call:
 * calls that overlap on the GPU (on different streams, or from different host threads) race on it
 * and must be serialised by the caller.  The first call on a device looks up the array's device
 * address (once per device, with that device current); make that first call before any stream
 * capture.  Enqueued on `stream` (the current device's); returns LMOE_ERR_CUDA if a launch fails. */
lmoe_status lmoe_route_noalloc(const float* logits, const float* bias, int32_t T, int32_t n_experts, int32_t top_k,
                               int32_t* topk_idx, float* topk_gate, int32_t* counts, int32_t* offsets,
                               int32_t* row_of, uint32_t* status, void* stream);

/* ------------------------------------------------------------------------------------------------
 * Expert parallelism ("Nemotron 3 Super" notes, section 3.2: the routing traffic of distributed MoE
 * grows with the dispatched vectors' width times K; LatentMoE dispatches the l-wide latent h = W_down x
 * instead of x).  G ranks (one layer handle each, created with ep_world = G) each own N / G
 * consecutive experts and replicate the router, W_down, W_up and the shared expert.  A forward of a
 * rank's T tokens is three calls with two exchanges between them, done by the caller (for example an
 * all-to-all over NCCL):
 *
 *   1. lmoe_ep_dispatch  (every rank, its own tokens)  routing and the send plan: one latent row per
 *      (token, owner rank) pair, pairs in (destination, token) order, and per assignment in
 *      (destination, token, slot) order its pair index within the destination and its expert id local
 *      to the destination, with the gate.
 *      exchange: rows, assignments and gates to their destinations (sizes from `counts`);
 *   2. lmoe_ep_experts   (every rank, the rows it received)  the owned experts, gate folded in, and
 *      the sum of each pair's gated outputs in slot order: one fp32 partial latent sum per pair.
 *      exchange: partial sums back to their sources, in the order the rows came;
 *   3. lmoe_ep_combine   (every rank, its own tokens)  z[t] = the token's partial sums in ascending
 *      owner-rank order, then y = W_up z + W_s2 sqrelu(W_s1 x).
 *
 * z is the single-GPU layer's K gated expert outputs grouped by owner rank; the two differ only in
 * rounding.  At most min(K, G) latent rows of l per token cross in each direction instead of K rows of
 * d.  All pointers are device pointers, 16-byte aligned; calls are enqueued on `stream`; the handle's
 * workspace is shared by the three calls, so one rank's calls must not overlap each other.
 * ------------------------------------------------------------------------------------------------ */

/* Step 1.  x [T, d] bf16 in.  Out, with P = pairs and A = T * K assignments:
 *   topk_idx [T, K] int32 (global expert ids), topk_gate [T, K] fp32
 *   send_rows [T * min(K, G), l] bf16: rows 0 .. P-1 are the latent rows of the pairs in send order
 *   send_meta [T * K, 2] int32: per assignment in send order, (pair index within its destination,
 *             expert id local to the destination)
 *   send_gate [T * K] fp32: per assignment in send order
 *   counts    [G, 2] int32: pairs and assignments sent to each destination (destinations in order)
 *   tok_pairs [T, min(K, G)] int32: the send-order indices of token t's pairs, ascending destination,
 *             then -1
 * Errors: UNSUPPORTED unless the handle is expert-parallel; SHAPE for T outside 0 .. max_tokens. */
lmoe_status lmoe_ep_dispatch(lmoe_handle h, const void* x, int32_t T, int32_t* topk_idx, float* topk_gate,
                             void* send_rows, int32_t* send_meta, float* send_gate, int32_t* counts,
                             int32_t* tok_pairs, void* stream);

/* Step 2.  recv_rows [R, l] bf16: the latent rows received (any order of sources); recv_meta [A, 2]
 * int32: per received assignment, (row of recv_rows, expert id local to this rank), with the rows
 * nondecreasing (each source's assignments arrive in its send order, sources one after another);
 * recv_gate [A] fp32.  Out: partial [R, l] fp32, row r = sum over the assignments of row r, in arrival
 * order, of gate * W2_e sqrelu(W1_e recv_rows[r]).  R <= ep_world * max_tokens * min(K, G) and
 * A <= ep_world * max_tokens * K, else SHAPE.  A row with no assignment gets zeros. */
lmoe_status lmoe_ep_experts(lmoe_handle h, const void* recv_rows, int32_t R, const int32_t* recv_meta,
                            const float* recv_gate, int32_t A, float* partial, void* stream);

/* Step 3.  x [T, d] bf16 (the tokens of step 1); back [P, l] fp32: the partial sums returned for this
 * rank's pairs, in send order; tok_pairs from step 1.  Out: y [T, d] bf16. */
lmoe_status lmoe_ep_combine(lmoe_handle h, const void* x, int32_t T, const float* back, const int32_t* tok_pairs,
                            void* y, void* stream);

/* Failure-detection self-test.  Enqueues on `stream` one kernel that waits, with the bounded
 * mbarrier wait that every pipelined kernel of the library uses, on a barrier that nothing ever
 * arrives on.  After `limit_ns` nanoseconds (clamped to 1 us .. 2 s) the wait gives up, the kernel
 * records a timeout in the handle's device status word and returns, leaving the context usable; the
 * next lmoe_get_device_status then returns LMOE_ERR_DEVICE_TIMEOUT (and clears the word).
 * Returns LMOE_ERR_CUDA if the launch fails. */
lmoe_status lmoe_selftest_wait_timeout(lmoe_handle h, uint64_t limit_ns, void* stream);

/* Human-readable name of a status code (static string). */
const char* lmoe_status_string(lmoe_status s);

/* Free everything the handle owns (synchronises its device first).  NULL is ignored. */
void lmoe_destroy(lmoe_handle h);

#ifdef __cplusplus
}
#endif
#endif /* LMOE_H */
