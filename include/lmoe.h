/*
 * lmoe.h -- C ABI of a B200 (sm_100a) LatentMoE layer forward.
 *
 * The layer (Nemotron 3 whitepaper, as summarised on the greeksharifa page,
 * section 2.2 "LatentMoE"; notes.yuuk.io page, section 2 "LatentMoE"):
 *
 *   logits = x W_r^T (+ b)                      router on the d-dim hidden state
 *   (idx, g) = top-K(logits), softmax renormalised over the K chosen
 *   z = x W_dn^T                                 d -> l latent down-projection
 *   a = relu(z W1_e^T)^2, y = g * (a W2_e^T)     routed experts in l, per expert e
 *   c_t = sum_k y(t, k)                          gate-weighted combine
 *   out = c W_up^T + sum_s Ws2_s relu(Ws1_s x)^2 l -> d up-projection + shared experts
 *
 * NVFP4 (same page, section 2.4 "NVFP4 Training"): E2M1 elements, 16-element
 * micro-blocks with an E4M3 scale, and an FP32 per-tensor global scale.
 *
 * Conventions for every entry point:
 *  - Pointers named x, w*, out, ... are DEVICE pointers unless the comment says
 *    host. The caller owns and allocates every buffer; the library never
 *    allocates or frees memory. Scratch memory is the caller's workspace,
 *    sized by lmoe_workspace_size().
 *  - Matrices are row-major. Weights use the [out][in] layout, so every
 *    contraction is "row-major activations x K-major weights".
 *  - BF16 tensors are 2-byte bfloat16; F32 tensors are 4-byte IEEE floats.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream). No call synchronises the host except
 *    lmoe_read_device_error().
 *  - Errors a host can see (NULL pointer, unsupported shape, misalignment,
 *    workspace too small) are returned before anything is launched. Errors
 *    found on the device (a pipeline wait that timed out, an index out of
 *    range) are written to an error word in the first 8 bytes of the
 *    workspace and read with lmoe_read_device_error(). A new workspace must
 *    have its first 256 bytes zeroed once before its first use; the library
 *    only ever writes the word on an error, and reading it clears it.
 *    Kernels never trap.
 *  - Inputs are assumed finite. Results are deterministic run to run (no
 *    floating-point atomics).
 *  - Device pointers must be 16-byte aligned; row pitches must be multiples
 *    of 16 bytes (for BF16: dimensions that are multiples of 8).
 */
#ifndef LMOE_H_
#define LMOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LMOE_OK = 0,
  LMOE_ERR_INVALID_ARG = 1,    /* NULL pointer, bad size, K > N, misalignment */
  LMOE_ERR_UNSUPPORTED = 2,    /* valid but not implemented (e.g. a dtype mix) */
  LMOE_ERR_WORKSPACE = 3,      /* workspace NULL or smaller than required */
  LMOE_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed */
  LMOE_ERR_DEVICE_TIMEOUT = 5, /* a device pipeline wait exceeded its limit */
  LMOE_ERR_DEVICE_BOUNDS = 6   /* a device index check failed */
} lmoe_status;

typedef enum { LMOE_F32 = 0, LMOE_BF16 = 1, LMOE_NVFP4 = 2 } lmoe_dtype;

/* Scale-factor layouts of an NVFP4 tensor [rows][cols]:
 * ROWMAJOR: byte (r, j) at r * (cols/16) + j, j = block index along the row.
 * MMA_TILED: the layout the block-scaled tensor-core MMA reads. Rows are
 *   grouped in blocks of 128 and columns in groups of 64 (4 scales); each
 *   (row block rb, column group cg) is a 512-byte atom at
 *   (rb * ceil(cols/64) + cg) * 512, and inside it scale (r, j) sits at
 *   (r % 32) * 16 + ((r % 128) / 32) * 4 + (j % 4). rows are padded to a
 *   multiple of 128 and cols to a multiple of 64 (padding bytes are written 0). */
typedef enum { LMOE_SF_ROWMAJOR = 0, LMOE_SF_MMA_TILED = 1 } lmoe_sf_layout;

/* OR-ed into lmoe_nvfp4_quantize's sf_layout: two-dimensional scale blocks of
 * 16 rows x 16 columns (the greeksharifa page on the Nemotron 3 whitepaper,
 * section 2.4 "NVFP4 Training": the recipe scales weights in 2-D blocks, so a
 * matrix and its transpose quantise alike). Each block's scale is the E4M3
 * rounding of its 256-element amax / (6 s_g) and is stored in every one of its
 * rows' 1 x 16 entries, so GEMMs and decoders read the result unchanged. */
#define LMOE_SF_BLOCK_16X16 0x10

/* Flag: l == d and there is no down/up projection (the standard-MoE limit). */
#define LMOE_FLAG_IDENTITY_PROJ 1u

/* Flag: the shared experts run in FP8 (E4M3), as in the Ultra checkpoint
 * recipe (chathome page on Nemotron 3 Ultra, quantisation paragraph: NVFP4
 * routed experts with FP8 shared experts). ws1 / ws2 then hold E4M3 codes
 * (lmoe_fp8_quantize of each weight tensor, one scale per tensor: all S
 * experts' Ws1 as one [S*m_s][d] tensor, all their Ws2 as one [S*d][m_s]
 * tensor) with their scales in ws1_scale / ws2_scale; x is quantised with the
 * static scale shared_x_scale, the hidden layer relu(x Ws1^T)^2 is stored as
 * E4M3 with the static scale shared_h_scale, and the output layer's sum (in
 * BF16) is added to the layer output. Needs act BF16 and n_shared > 0. */
#define LMOE_FLAG_SHARED_FP8 2u

/* Supported configurations (every entry point that takes a config checks
 * them before launching anything):
 *  LMOE_ERR_INVALID_ARG: T < 0 or T > 2^25; d, l, N, K or m not positive;
 *    K > N; n_shared < 0, or n_shared > 0 with m_shared <= 0; d, l, m or
 *    m_shared not a multiple of 8; LMOE_FLAG_IDENTITY_PROJ with l != d.
 *  LMOE_ERR_UNSUPPORTED: K > 32 or N > 1024; act F32 with expert other than
 *    F32; act BF16 with expert F32; act BF16 with shared experts and m_shared
 *    not a multiple of 64; expert NVFP4 with l or m not a multiple of 256;
 *    LMOE_FLAG_SHARED_FP8 with act F32, d not a multiple of 16 or m_shared
 *    not a multiple of 128 (LMOE_ERR_INVALID_ARG without shared experts);
 *    N not a multiple of 8 where the logits are computed (lmoe_forward,
 *    lmoe_route without logits_in). */

typedef struct {
  int64_t T;        /* tokens */
  int32_t d;        /* hidden size */
  int32_t l;        /* latent size (== d with LMOE_FLAG_IDENTITY_PROJ) */
  int32_t N;        /* routed experts */
  int32_t K;        /* experts per token, 1 <= K <= N */
  int32_t m;        /* routed expert hidden size */
  int32_t n_shared; /* always-on shared experts (0 = none) */
  int32_t m_shared; /* shared expert hidden size */
  int32_t act;      /* lmoe_dtype of x, router, projections and the stored
                       intermediates z, a, y, c, out: LMOE_F32 or LMOE_BF16 */
  int32_t expert;   /* lmoe_dtype of the routed expert weights and the latent
                       activations fed to them: LMOE_F32 (with act F32),
                       LMOE_BF16 or LMOE_NVFP4 (with act BF16) */
  uint32_t flags;   /* LMOE_FLAG_* */
} lmoe_config;

/* Layer weights (device pointers, `act` dtype unless stated).
 *  w_router [N][d]; router_bias [N] F32 or NULL;
 *  w_down [l][d], w_up [d][l] (NULL with LMOE_FLAG_IDENTITY_PROJ);
 *  w1 [N][m][l], w2 [N][l][m]: routed experts. For expert == LMOE_NVFP4 these
 *    are packed E2M1 codes ([N][m][l/2], [N][l][m/2] bytes; element 2j in the
 *    low nibble), w1_sf / w2_sf their E4M3 block scales in LMOE_SF_MMA_TILED
 *    layout per expert matrix (as written by lmoe_nvfp4_quantize), and
 *    w1_gs / w2_gs [N] F32 the per-matrix global scales;
 *  a_global_scale: NVFP4 only, device pointer to one F32: the static scale of
 *    the expert hidden activation a, as a checkpoint carries it;
 *  ws1 [S][m_s][d], ws2 [S][d][m_s]: shared experts (NULL when n_shared == 0);
 *    E4M3 codes (1 byte each) with LMOE_FLAG_SHARED_FP8;
 *  ws1_scale, ws2_scale, shared_x_scale, shared_h_scale: LMOE_FLAG_SHARED_FP8
 *    only, device pointers to one F32 each (the two weight tensors' scales and
 *    the static scales of the shared experts' input and hidden layer). */
typedef struct {
  const void* w_router;
  const float* router_bias;
  const void* w_down;
  const void* w_up;
  const void* w1;
  const void* w2;
  const uint8_t* w1_sf;
  const uint8_t* w2_sf;
  const float* w1_gs;
  const float* w2_gs;
  const float* a_global_scale;
  const void* ws1;
  const void* ws2;
  const float* ws1_scale;
  const float* ws2_scale;
  const float* shared_x_scale;
  const float* shared_h_scale;
} lmoe_weights;

/* Workspace size queries, one per entry point. */
typedef enum {
  LMOE_OP_ROUTE = 0,
  LMOE_OP_PERMUTE = 1,
  LMOE_OP_EXPERT_FFN = 2,
  LMOE_OP_COMBINE = 3,
  LMOE_OP_FORWARD = 4,
  LMOE_OP_NVFP4_QUANTIZE = 5,
  LMOE_OP_FP8_QUANTIZE = 6
} lmoe_op;

/* Bytes of workspace `op` needs for `cfg` (for LMOE_OP_NVFP4_QUANTIZE and
 * LMOE_OP_FP8_QUANTIZE the tensor is taken as [cfg->T][cfg->l]). Returns 0 for an invalid config or
 * an unknown op, and for LMOE_OP_COMBINE (which needs none). */
size_t lmoe_workspace_size(const lmoe_config* cfg, int op);

/* Rows of the expert-grouped (padded) buffers: each expert's rows start at a
 * multiple of 128, so the buffers hold at most T*K + N*127 rows, rounded up
 * to a multiple of 128. Returns 0 for an invalid config. */
int64_t lmoe_padded_rows(const lmoe_config* cfg);

/* Router (greeksharifa page, section 2.2 "LatentMoE": the routing gate reads
 * the d-dim hidden state, outside the latent compression; the Nemotron 3 Nano
 * blog's architecture section: a learned router over the routed experts).
 * The score function, tie rule and renormalisation are not on the pages; the
 * reading taken: logits = x W_r^T + b, then per token the K experts with the largest
 * logits (ties to the lower index), in that order, and their gates
 * g_k = exp(l_k - l_max) / sum_j exp(l_j - l_max) over the chosen K (the
 * softmax over all N restricted to the K and renormalised).
 *  x [T][d] (act), w_router [N][d] (act), bias [N] F32 or NULL.
 *  logits_in: NULL to compute the logits; else [T][N] F32 logits to route
 *    (x, w_router, bias are then ignored and may be NULL).
 *  topk_idx [T][K] int32, topk_w [T][K] F32: outputs.
 *  logits_out [T][N] F32 or NULL: the computed logits (bias included).
 *  Errors: the config checks above; LMOE_ERR_INVALID_ARG for NULL outputs,
 *  NULL x or w_router when logits are computed, or x / w_router not 16-byte
 *  aligned; LMOE_ERR_UNSUPPORTED for N % 8 when logits are computed;
 *  LMOE_ERR_WORKSPACE; on the device, LMOE_ERR_DEVICE_TIMEOUT. */
lmoe_status lmoe_route(const lmoe_config* cfg, const void* x, const void* w_router,
                       const float* bias, const float* logits_in, int32_t* topk_idx,
                       float* topk_w, float* logits_out, void* ws, size_t ws_bytes,
                       void* stream);

/* Dispatch grouped by expert (greeksharifa page, section 2.2 "LatentMoE": the
 * routed experts run on the latent z, so the rows sent to each expert are
 * l-dim; the pages give no dispatch layout). A stable counting sort of the slots
 * f = t*K + k by expert (expert ascending, then f ascending).
 *  topk_idx [T][K] int32 (each in [0, N); out-of-range -> device bounds error).
 *    A slot with an out-of-range expert is left out: offsets[N] counts only
 *    the in-range slots, its inv_perm entry is not written, and it is neither
 *    gathered nor given a gate.
 *  offsets [N+1] int32: expert e owns sorted positions [offsets[e], offsets[e+1]).
 *  perm_src [T*K] int32: sorted position r holds slot perm_src[r].
 *  inv_perm [T*K] int32: slot f sits at sorted position inv_perm[f].
 *  padded_offsets [N+1] int32: expert e's rows in the padded buffers start at
 *    padded_offsets[e] (a multiple of 128); sorted position r of expert e is
 *    padded row r - offsets[e] + padded_offsets[e].
 *  rows / row_bytes / permuted_rows (all optional, NULL/0 to skip): gather the
 *    token rows rows[t] (row_bytes each, a multiple of 16) to padded rows.
 *  rows_sf / permuted_sf (optional): NVFP4 row-major scales [T][row_cols/16]
 *    of `rows`, re-laid to LMOE_SF_MMA_TILED at the padded rows; row_cols is
 *    2*row_bytes (the rows then hold packed E2M1 codes).
 *  topk_w / perm_gate (optional): the gate of each padded row ([padded] F32).
 *  With T = 0 only offsets and padded_offsets are needed (written as zeros);
 *  the other buffers may be NULL.
 *  Errors: the config checks above; LMOE_ERR_INVALID_ARG for a NULL index
 *  buffer, rows without permuted_rows (or scales, gates without their
 *  destination), row_bytes not a positive multiple of 16, unaligned rows,
 *  scales whose row width 2*row_bytes is not a multiple of 64;
 *  LMOE_ERR_WORKSPACE; on the device, LMOE_ERR_DEVICE_BOUNDS (info = the
 *  first out-of-range slot f seen). */
lmoe_status lmoe_permute(const lmoe_config* cfg, const int32_t* topk_idx, int32_t* offsets,
                         int32_t* perm_src, int32_t* inv_perm, int32_t* padded_offsets,
                         const void* rows, int64_t row_bytes, void* permuted_rows,
                         const uint8_t* rows_sf, uint8_t* permuted_sf, const float* topk_w,
                         float* perm_gate, void* ws, size_t ws_bytes, void* stream);

/* lmoe_permute without a workspace: the same permutation, offsets, padded
 * offsets and optional row/scale/gate gathers, bit for bit, for callers that
 * cannot allocate device memory -- e.g. a plugin that an inference runtime
 * hands only its input and output buffers, or a latency-critical loop that
 * must not call cudaMalloc (an allocation can synchronise the device).
 * The pages have no counterpart to this entry point; it is a deployment aid.
 *  - Scratch: a fixed 512 KiB array in device memory defined by the library
 *    (every GPU that loads the library holds it until the process exits).
 *    It holds (ceil(T*K / 8192) + 1) * N counters at most 131072, e.g.
 *    T*K up to about 2 million slots with N = 512; larger problems return
 *    LMOE_ERR_WORKSPACE before anything is launched.
 *  - The first call on each device looks up the array's device address (with
 *    that device current); make that first call before any stream capture.
 *    The address is cached per device together with the id of the context it
 *    was looked up in; a call in a new context (after cudaDeviceReset, for
 *    instance) looks it up again, so make the first call after such a reset
 *    before any stream capture too.
 *  - All calls share the one array: calls that overlap on the GPU (two
 *    streams, or two host threads) race and must be serialised by the caller.
 *  - There is no error word: an out-of-range expert index is skipped without
 *    a report (lmoe_permute reports it). Allocates nothing. */
lmoe_status lmoe_permute_noalloc(const lmoe_config* cfg, const int32_t* topk_idx, int32_t* offsets,
                                 int32_t* perm_src, int32_t* inv_perm, int32_t* padded_offsets,
                                 const void* rows, int64_t row_bytes, void* permuted_rows,
                                 const uint8_t* rows_sf, uint8_t* permuted_sf, const float* topk_w,
                                 float* perm_gate, void* stream);

/* Routed expert FFNs in the latent dimension (greeksharifa page, section 2.2
 * "LatentMoE": every routed expert maps l -> m -> l; section 2.4 "NVFP4
 * Training" for the NVFP4 operands; the activation is not on the pages and is
 * read as squared ReLU), on the padded expert-grouped rows:
 *  y = g * (relu(z_e W1_e^T)^2 W2_e^T) for the rows of each expert e.
 *  permuted_in [padded][l]: `act` rows, or for expert == NVFP4 packed E2M1
 *    codes [padded][l/2] with permuted_sf (MMA_TILED) and in_global_scale
 *    (device pointer to one F32).
 *  offsets, padded_offsets [N+1]: from lmoe_permute.
 *  perm_gate [padded] F32 or NULL (gates of 1).
 *  y_perm [padded][l] (act): output; padding rows are left unspecified.
 *  Errors: the config checks above; LMOE_ERR_INVALID_ARG for NULL or
 *  unaligned buffers or weights (NVFP4: also missing scales or global
 *  scales); LMOE_ERR_WORKSPACE; on the device, LMOE_ERR_DEVICE_TIMEOUT. */
lmoe_status lmoe_expert_ffn(const lmoe_config* cfg, const lmoe_weights* w,
                            const void* permuted_in, const uint8_t* permuted_sf,
                            const float* in_global_scale, const int32_t* offsets,
                            const int32_t* padded_offsets, const float* perm_gate,
                            void* y_perm, void* ws, size_t ws_bytes, void* stream);

/* Combine (greeksharifa page, section 2.2 "LatentMoE": the experts' outputs
 * are summed in l and then projected back to d):
 * c_t = sum_{k=0..K-1} w[t][k] * y_perm[row(t*K+k)], summed in fp32
 * in k order, stored as `act`; row(f) = inv_perm[f] - offsets[e] +
 * padded_offsets[e] with e = topk_idx[f]. topk_w NULL means the gates were
 * already applied (w = 1). c [T][l]. No workspace. A slot whose expert index
 * is out of range (left out by lmoe_permute) contributes nothing.
 * Errors: the config checks above; LMOE_ERR_INVALID_ARG for NULL buffers or
 * unaligned y_perm / c. There is no error word (no device errors). */
lmoe_status lmoe_combine(const lmoe_config* cfg, const void* y_perm, const int32_t* topk_idx,
                         const int32_t* inv_perm, const int32_t* offsets,
                         const int32_t* padded_offsets, const float* topk_w, void* c,
                         void* stream);

/* The whole layer (greeksharifa page, section 2.2 "LatentMoE"; notes.yuuk.io
 * page, section 2 "LatentMoE"; the two always-on shared experts of the
 * Nemotron 3 Nano blog's architecture section): route, down-project (NVFP4: quantise z with its current
 * amax), permute, expert FFNs, combine, up-project and add the shared
 * experts. x [T][d] (act) -> out [T][d] (act). N must be a multiple of 8
 * (the router GEMM stores logit rows in 16-byte vectors; LMOE_ERR_UNSUPPORTED
 * otherwise, also from lmoe_route when it computes the logits).
 * Errors: the config checks above; LMOE_ERR_INVALID_ARG for NULL w,
 * w_router, w1 or w2, w_down / w_up given with LMOE_FLAG_IDENTITY_PROJ or
 * missing without it, missing shared-expert weights, missing NVFP4 scales,
 * NULL or unaligned x / out (not checked when T == 0, which launches
 * nothing), or a weight a TMA descriptor cannot address (not 16-byte
 * aligned); LMOE_ERR_WORKSPACE; on the device, LMOE_ERR_DEVICE_TIMEOUT.
 * Ordering: every launch is ordered after earlier work on `stream`, and
 * later work on `stream` sees the result. With latent projections (BF16
 * with T > 64, or NVFP4) the top-K and permutation run beside the
 * down-projection on a library-owned stream of the same device, forked from
 * and joined back to `stream` with events; the call can be captured in a
 * CUDA graph. */
lmoe_status lmoe_forward(const lmoe_config* cfg, const lmoe_weights* w, const void* x,
                         void* out, void* ws, size_t ws_bytes, void* stream);

/* lmoe_forward with stage tracing: when `events` is not NULL it holds
 * LMOE_TRACE_EVENTS cudaEvent_t handles (created by the caller) that are
 * recorded on `stream` at the stage boundaries, in order:
 *   0 start, 1 after routing, 2 after the down-projection (and NVFP4
 *   quantisation of z), 3 after the permutation and gather, 4 after expert
 *   GEMM 1, 5 after expert GEMM 2, 6 after the combine, 7 after the shared
 *   experts and up-projection (end).
 * Stages that do not run for a configuration record their event at the same
 * point as the previous one. Costs one event record per stage. */
#define LMOE_TRACE_EVENTS 8
lmoe_status lmoe_forward_traced(const lmoe_config* cfg, const lmoe_weights* w, const void* x,
                                void* out, void* ws, size_t ws_bytes, void* stream,
                                void* const* events);

/* NVFP4 quantiser (greeksharifa page, section 2.4 "NVFP4 Training": E2M1
 * elements, 16-element micro-blocks with an E4M3 scale and an FP32 per-tensor
 * global scale; the scale formulas are not on the pages and are read as the
 * standard two-level recipe below). Two-level quantisation of in [rows][cols] (F32 or BF16, cols a
 * multiple of 16) along its rows:
 *  s_g = global_in ? *global_in : fp32(amax / 2688) (1 when amax == 0);
 *  per 16-block: s_b = E4M3_satfinite_rn(amax_b / (s_g * 6));
 *  q_i = E2M1_satfinite_rn(x_i / (dec(s_b) * s_g)) (all codes +0 if dec(s_b) == 0).
 *  codes [rows][cols/2] (low nibble first), sf per sf_layout, global_out
 *  (device F32, may be NULL) receives s_g. global_in: device pointer or NULL.
 *  sf_layout | LMOE_SF_BLOCK_16X16: amax_b over 16 x 16 blocks instead (rows
 *  need not be a multiple of 16: the last block has the remaining rows).
 *  Errors: LMOE_ERR_INVALID_ARG for null pointers, cols % 16, an unknown
 *  layout, an unaligned input (16 B) or code buffer (8 B). */
lmoe_status lmoe_nvfp4_quantize(const void* in, int in_dtype, int64_t rows, int64_t cols,
                                const float* global_in, uint8_t* codes, uint8_t* sf,
                                float* global_out, int sf_layout, void* ws, size_t ws_bytes,
                                void* stream);

/* FP8 quantiser (the format of the shared experts in the Ultra checkpoint
 * recipe: chathome page on Nemotron 3 Ultra, quantisation paragraph; one FP32
 * scale per tensor is the reading taken, the pages give only the format):
 *  s = scale_in ? *scale_in : fp32(amax / 448) (1 when amax == 0);
 *  q = E4M3_satfinite_rn(fp32(x / s)) for every element of in [rows][cols]
 *  (F32 or BF16, cols a multiple of 16), codes [rows][cols] (1 byte each);
 *  scale_out (device F32, may be NULL) receives s. scale_in: device pointer
 *  or NULL (a static scale, as for activations).
 *  Errors: LMOE_ERR_INVALID_ARG for null pointers, cols % 16, an unaligned
 *  input or code buffer (16 B); LMOE_ERR_WORKSPACE (scale_in NULL and the
 *  workspace smaller than lmoe_workspace_size(LMOE_OP_FP8_QUANTIZE)). */
lmoe_status lmoe_fp8_quantize(const void* in, int in_dtype, int64_t rows, int64_t cols,
                              const float* scale_in, uint8_t* codes, float* scale_out, void* ws,
                              size_t ws_bytes, void* stream);

/* NVFP4 quantiser of the training recipe's GEMM operands (greeksharifa page,
 * section 2.4 "NVFP4 Training"; notes.yuuk.io page, section 4: gradients are
 * rounded stochastically, the wgrad inputs get a random Hadamard transform,
 * weights use 2-D scale blocks; the transform and rounding details are
 * readings, the pages name only the techniques). Quantises out = in
 * [rows][cols], or in^T with LMOE_QX_TRANSPOSE ([cols][rows]: the blocks then
 * run along the input's rows, e.g. along the tokens of an activation or
 * gradient), along out's rows with lmoe_nvfp4_quantize's two-level scales:
 *  - LMOE_QX_RHT: every 16-block v of out's rows becomes H16 diag(s) v / 4
 *    first (H16 the Sylvester Hadamard matrix, s_i = -1 where bit i of
 *    rht_signs is set), formed in fp64;
 *  - LMOE_QX_SR: elements round stochastically: between grid neighbours
 *    lo <= |v| < hi to hi when u * (hi - lo) < |v| - lo, u = (w >> 8) * 2^-24
 *    with w word i % 4 of Philox-4x32-10 (Salmon et al., SC11) at counter
 *    (i / 4 low, i / 4 high, sr_stream, 0) under key (seed low, seed high),
 *    i = r * out_cols + c the element's index in out; |v| >= 6 saturates;
 *    the block scales still round to nearest even;
 *  - sf_layout | LMOE_SF_BLOCK_16X16: 16 x 16 scale blocks (not with RHT or SR).
 *  Every step after the transform is an fp32 operation on its exact inputs
 *  (fp64 division rounded once to fp32), so results equal those of the
 *  definition taken in exact arithmetic and rounded step by step.
 *  codes [out_rows][out_cols/2], sf per sf_layout, global_in / global_out as
 *  lmoe_nvfp4_quantize. out_cols must be a multiple of 16.
 *  Errors: LMOE_ERR_INVALID_ARG for null pointers, out_cols % 16, an unknown
 *  flag or layout, 2-D blocks with RHT or SR, an unaligned input (16 B) or
 *  code buffer (8 B); LMOE_ERR_WORKSPACE (global_in NULL and the workspace
 *  smaller than lmoe_nvfp4_quantize_ex_workspace(rows, cols)). */
#define LMOE_QX_TRANSPOSE 1u
#define LMOE_QX_RHT 2u
#define LMOE_QX_SR 4u
size_t lmoe_nvfp4_quantize_ex_workspace(int64_t rows, int64_t cols);
lmoe_status lmoe_nvfp4_quantize_ex(const void* in, int in_dtype, int64_t rows, int64_t cols, uint32_t flags,
                                   uint32_t rht_signs, uint64_t seed, uint32_t sr_stream,
                                   const float* global_in, uint8_t* codes, uint8_t* sf, float* global_out,
                                   int sf_layout, void* ws, size_t ws_bytes, void* stream);

/* Transpose of NVFP4 weights quantised with 16 x 16 scale blocks (the
 * training recipe's 2-D weight blocks: greeksharifa page, section 2.4 "NVFP4
 * Training"; the dgrads read W^T). With square blocks W^T quantises to W's
 * codes and scales transposed: every element keeps its block's scale and the
 * global scale is W's, so this replaces quantising the transpose.
 *  codes: `groups` matrices [rows][cols/2] back to back (element 2k in the
 *  low nibble), sf: their MMA-tiled scales (rows * cols / 16 bytes each), as
 *  lmoe_nvfp4_quantize_ex writes with LMOE_SF_MMA_TILED | LMOE_SF_BLOCK_16X16;
 *  codes_t [groups][cols][rows/2] and sf_t (same sizes) receive W^T's; the
 *  global scales are unchanged. Device pointers, 16-byte aligned, no overlap.
 *  Errors: LMOE_ERR_INVALID_ARG for null or unaligned pointers or negative
 *  sizes; LMOE_ERR_UNSUPPORTED unless rows and cols are multiples of 128
 *  (whole scale atoms) and groups <= 65535. Nothing to do for zero sizes. */
lmoe_status lmoe_nvfp4_transpose_2d(const uint8_t* codes, const uint8_t* sf, int64_t groups, int64_t rows,
                                    int64_t cols, uint8_t* codes_t, uint8_t* sf_t, void* stream);

/* Grouped block-scaled NVFP4 GEMM (the kernel of the routed experts, exposed
 * for the training recipe's dgrad and wgrad; greeksharifa page, section 2.4
 * "NVFP4 Training": fprop, dgrad and wgrad run as NVFP4 GEMMs):
 *   out[r][c] = BF16( g_a * g_b[e] * sum_k qa[r][k] sa[r][k/16] qb[e][c][k] sb[e][c][k/16] )
 *   (times row_scale[r] when given), for rows r of group e: rows
 *   padded_offsets[e] .. padded_offsets[e] + offsets[e+1] - offsets[e].
 *  a_codes [a_rows][k/2] with a_sf in LMOE_SF_MMA_TILED layout over a_rows
 *    (a multiple of 128; each group's padded range a multiple of 128);
 *  a_global: device F32, one value, or [groups] with a_global_per_group;
 *  b_codes [groups][cols][k/2], b_sf [groups] MMA-tiled blocks of cols x k/16,
 *    b_global [groups] device F32;
 *  k and cols multiples of 256; out [a_rows][ld_out] BF16 (padding rows
 *  unspecified). ws: at least 256 bytes, its first 256 zeroed before first
 *  use (the error word). One group with offsets {0, a_rows} is a plain GEMM.
 *  Errors: LMOE_ERR_INVALID_ARG for null or unaligned buffers, sizes out of
 *  range; LMOE_ERR_UNSUPPORTED for k or cols not multiples of 256 or more
 *  than 1024 groups; LMOE_ERR_WORKSPACE; on the device, LMOE_ERR_DEVICE_TIMEOUT. */
lmoe_status lmoe_nvfp4_gemm(int groups, const int32_t* offsets, const int32_t* padded_offsets, int64_t a_rows,
                            const uint8_t* a_codes, const uint8_t* a_sf, const float* a_global,
                            int a_global_per_group, const uint8_t* b_codes, const uint8_t* b_sf,
                            const float* b_global, int cols, int64_t k, const float* row_scale, void* out,
                            int64_t ld_out, void* ws, size_t ws_bytes, void* stream);

/* Backward of the routed experts under the NVFP4 training recipe
 * (greeksharifa page on the Nemotron 3 whitepaper, section 2.4 "NVFP4
 * Training"; notes.yuuk.io page, section 4: fprop, dgrad and wgrad as NVFP4
 * GEMMs, 16 x 16 weight blocks, stochastic rounding of gradients, a random
 * Hadamard transform on the wgrad inputs; the details are readings). Slots
 * are in lmoe_permute's padded layout: expert e owns rows
 * padded_offsets[e] .. padded_offsets[e] + counts[e] - 1, padded_offsets[e]
 * = sum over e' < e of counts[e'] rounded up to 128. Per expert, over its n
 * rows (zero rows up to R = n rounded up to 16 wherever a quantiser runs
 * along the rows):
 *   W1q, W2q = the BF16 masters w1[e] [m][l], w2[e] [l][m] quantised with
 *     16 x 16 blocks (current amax); h = zq W1q^T (fp32), aq = NVFP4(relu(h)^2)
 *     with the static global scale a_global, o = aq W2q^T (fp32);
 *   dgate[r] = dy[r] . o[r];  do = gate[r] dy[r]  (fp32);
 *   dA = SR(do) W2q;  dh = dA * 2 max(h, 0);  dz = SR(dh) W1q;
 *   dW2 = SR(RHT(do)^T) RN(RHT(aq)^T)^T;  dW1 = SR(RHT(dh)^T) RN(RHT(zq)^T)^T;
 *   SR: lmoe_nvfp4_quantize_ex's stochastic rounding with sr_stream
 *   4 e + 2 g + j (g: 0 first GEMM, 1 second; j: 0 dgrad, 1 wgrad) and
 *   `seed`; RHT with rht_signs; every quantiser takes its tensor's current
 *   amax (per expert).
 *  counts [N]: HOST array of rows per expert. offsets, padded_offsets [N+1]:
 *    DEVICE arrays as lmoe_permute writes them.
 *  z_codes [P][l/2], z_sf (MMA-tiled over the P padded rows), z_global
 *    (device F32): the NVFP4 latent rows as lmoe_permute moves them.
 *  w1, w2: BF16 masters [N][m][l], [N][l][m]. a_global: device F32.
 *  gate [P] F32, dy [P][l] F32: each slot row's gate and upstream gradient
 *    (fp32: the stochastic quantiser of do = gate * dy must see it unrounded).
 *  Outputs (device): dz [P][l] BF16 (padding rows unspecified), dgate [P] F32
 *    (set for real rows only), dw1 [N][m][l] and dw2 [N][l][m] BF16.
 *  l and m multiples of 256; 16-byte aligned buffers; ws of at least
 *  lmoe_expert_backward_nvfp4_workspace(cfg, counts) bytes, its first 256
 *  zeroed before first use (the error word).
 *  Errors: LMOE_ERR_INVALID_ARG for null or unaligned pointers, negative
 *  counts, N outside 1..1024; LMOE_ERR_UNSUPPORTED for l or m not multiples
 *  of 256; LMOE_ERR_WORKSPACE; on the device, LMOE_ERR_DEVICE_TIMEOUT. */
size_t lmoe_expert_backward_nvfp4_workspace(const lmoe_config* cfg, const int32_t* counts);
lmoe_status lmoe_expert_backward_nvfp4(const lmoe_config* cfg, const int32_t* counts, const int32_t* offsets,
                                       const int32_t* padded_offsets, const uint8_t* z_codes, const uint8_t* z_sf,
                                       const float* z_global, const void* w1, const void* w2,
                                       const float* a_global, const float* gate, const float* dy, uint64_t seed,
                                       uint32_t rht_signs, void* dz, float* dgate, void* dw1, void* dw2, void* ws,
                                       size_t ws_bytes, void* stream);

/* Gradients of the layer, written by lmoe_backward_nvfp4 (device buffers,
 * BF16 unless noted; the ones a configuration does not have may be NULL). */
typedef struct {
  void* dx;             /* [T][d] */
  void* dw_router;      /* [N][d] */
  float* drouter_bias;  /* [N] F32; needed with a router bias */
  void* dw_down;        /* [l][d]; latent projections only */
  void* dw_up;          /* [d][l]; latent projections only */
  void* dw1;            /* [N][m][l] */
  void* dw2;            /* [N][l][m] */
  void* dws1;           /* [S][m_shared][d]; with shared experts */
  void* dws2;           /* [S][d][m_shared] */
} lmoe_grads;

/* The layer's backward pass with its routed experts trained under the NVFP4
 * recipe (greeksharifa page, sections 2.2 "LatentMoE" and 2.4 "NVFP4
 * Training"; notes.yuuk.io page, section 4). The forward pieces the gradients
 * need are recomputed from x: router logits (+ bias) and the top-K gates, z
 * (down-projection), z quantised to NVFP4 with its current amax, the slots
 * permuted by expert. Then, for the upstream gradient dout [T][d]:
 *   dc = dout W_up (identity projections: dout);
 *   the routed experts: lmoe_expert_backward_nvfp4 on the slot rows (BF16
 *     masters w1, w2; a_global, seed and rht_signs as there), giving dz per
 *     slot, dgate, dW1, dW2 and the experts' outputs o;
 *   c = sum_k g_k o_k;  dW_up = dout^T c;
 *   dsel_k = g_k (dgate_k - sum_j g_j dgate_j) at the K chosen experts (top-K
 *     selection passes no gradient), dW_router = dsel^T x, drouter_bias =
 *     sum over tokens of dsel;
 *   dz_t = sum_k dz(t, k);  dW_down = dz^T x;
 *   each shared expert s: pre = x Ws1_s^T, dWs2_s = dout^T relu(pre)^2,
 *     dpre = (dout Ws2_s) 2 max(pre, 0), dWs1_s = dpre^T x;
 *   dx = dsel W_router + dz W_down + sum_s dpre_s Ws1_s (dz W_down -> dz with
 *     identity projections).
 * The router, the projections and the shared experts (kept in higher
 * precision by the recipe) are BF16 tensor-core GEMMs with fp32 accumulation.
 *  cfg: act and expert BF16 (w->w1, w->w2 are the BF16 masters), no
 *    LMOE_FLAG_SHARED_FP8; d % 64, l and m multiples of 256, N % 8,
 *    m_shared % 64. w: the forward's weights. x, dout [T][d] BF16.
 *  The call synchronises its stream once (the experts' row counts are read
 *  on the host). ws: lmoe_backward_nvfp4_workspace(cfg) bytes, the first 256
 *  zeroed before first use (the error word).
 *  Errors: LMOE_ERR_INVALID_ARG for null or unaligned pointers and missing
 *  weights or gradients; LMOE_ERR_UNSUPPORTED for the dtype, flag and size
 *  conditions above; LMOE_ERR_WORKSPACE; LMOE_ERR_CUDA. */
size_t lmoe_backward_nvfp4_workspace(const lmoe_config* cfg);
lmoe_status lmoe_backward_nvfp4(const lmoe_config* cfg, const lmoe_weights* w, const void* x, const void* dout,
                                const float* a_global, uint64_t seed, uint32_t rht_signs, const lmoe_grads* g,
                                void* ws, size_t ws_bytes, void* stream);

/* Expert parallelism in the latent dimension (greeksharifa page on the
 * Nemotron 3 whitepaper, section 2.2 "LatentMoE": the rows that cross GPUs
 * between the projections are l-dim, so the all-to-all volume falls by d/l).
 * G ranks each route and permute their own tokens; rank h owns the experts
 * [first(h), first(h) + n(h)), n(h) = N/G (one more for the first N%G ranks).
 *
 * lmoe_ep_plan (HOST arrays, no device work): from counts [G][N] (counts[g][e]
 * = slots rank g routes to expert e, known to every rank after a count
 * exchange) computes, for `rank`:
 *  send_counts/send_offsets [G]: the rows of this rank's sorted (expert-major)
 *    permuted buffer that go to each rank, one contiguous block per rank;
 *  recv_counts/recv_offsets [G]: the blocks an all-to-all delivers, in source
 *    rank order (each sorted by expert);
 *  first_expert, local_experts (NL); local_offsets/local_padded_offsets
 *    [NL+1]: the expert-grouped layout of the received rows (sources in rank
 *    order inside an expert; each expert's range padded to a multiple of 128,
 *    as the expert GEMMs read it);
 *  block_src/block_dst/block_rows [G*NL] (source-major, block (g, el) at
 *    g*NL + el): where each (source, local expert) block sits in the received
 *    buffer and where it goes in the expert-grouped buffer.
 * Errors: LMOE_ERR_INVALID_ARG for null pointers, G, rank or N out of range,
 * negative counts; LMOE_ERR_UNSUPPORTED for N > 1024, G > N or more than
 * 2^31 rows. */
lmoe_status lmoe_ep_plan(int G, int rank, int N, const int32_t* counts, int32_t* send_counts,
                         int32_t* send_offsets, int32_t* recv_counts, int32_t* recv_offsets, int32_t* first_expert,
                         int32_t* local_experts, int32_t* local_offsets, int32_t* local_padded_offsets,
                         int32_t* block_src, int32_t* block_dst, int32_t* block_rows);

/* Row-block copy between the all-to-all's source-major order and the
 * expert-grouped padded order (either direction: swap src_rows and dst_rows):
 * block b moves its rows from row src_rows[b] of `in` to row dst_rows[b] of
 * `out`; row_prefix [nblocks] (DEVICE, int64) is the inclusive prefix of the
 * blocks' row counts and total_rows its last value. in, out, src_rows,
 * dst_rows, row_prefix are device pointers; rows are row_bytes each (a
 * multiple of 16, 16-byte aligned). Asynchronous on `stream`.
 * Errors: LMOE_ERR_INVALID_ARG for null or unaligned buffers, bad sizes. */
lmoe_status lmoe_ep_reorder(const void* in, void* out, int64_t row_bytes, int nblocks, const int32_t* src_rows,
                            const int32_t* dst_rows, const int64_t* row_prefix, int64_t total_rows, void* stream);

/* The expert-parallel data plane over peer memory (greeksharifa page,
 * section 2.2 "LatentMoE": the rows that cross GPUs are the l-dim latent
 * rows). Instead of an all-to-all into a staging buffer and a reorder, each
 * rank's dispatch kernel stores its token rows straight into the owner
 * ranks' expert-grouped buffers through peer pointers, and its combine kernel
 * reads the owners' expert outputs back the same way; the owners run
 * lmoe_expert_ffn on their received rows between the two. Plain loads and
 * stores only (no TMA, no multicast). Between the phases the caller
 * separates the ranks with a barrier of its own (every rank's dispatch done
 * before any owner's expert FFN; every expert FFN done before any combine):
 * the kernels do not wait on other GPUs.
 *
 * lmoe_ep_slot_bases (HOST arrays, no device work): from counts [G][N] (after
 * the count exchange) gives, for this rank, expert_owner [N] (the rank that
 * owns each expert, ownership as lmoe_ep_plan) and dst_base [N]: the owner's
 * padded row of this rank's first row for the expert in the owner's
 * expert-grouped buffer (sources in rank order inside an expert, each expert's
 * range padded to 128 rows: lmoe_ep_plan's local_padded_offsets and
 * block_dst). Errors as lmoe_ep_plan. */
lmoe_status lmoe_ep_slot_bases(int G, int rank, int N, const int32_t* counts, int32_t* expert_owner,
                               int32_t* dst_base);

/* Dispatch: slot f = t*K + k (expert e = topk_idx[f]; slots with e outside
 * [0, N) are skipped, as lmoe_permute leaves them out) goes to rank
 * h = expert_owner[e], row dst_base[e] + inv_perm[f] - offsets[e] of that
 * rank's buffer: the token's row rows[t] (row_bytes, a multiple of 16) is
 * copied there, and with topk_w its gate to the same row of the rank's gate
 * buffer (F32, the perm_gate of its lmoe_expert_ffn call).
 *  topk_idx, inv_perm, offsets: this rank's lmoe_permute results ([T][K],
 *  [T*K], [N+1]); expert_owner, dst_base [N]: DEVICE copies of
 *  lmoe_ep_slot_bases's arrays; peer_rows [G], peer_gates [G] (or NULL with
 *  topk_w NULL): DEVICE arrays of device pointers, rank h's buffers (another
 *  GPU's memory mapped into this process, or this GPU's own for h = rank),
 *  each 16-byte aligned and holding peer_rows_cap rows. err_word (device, may be NULL): a row or
 *  owner out of range is skipped and recorded there (LMOE_ERR_DEVICE_BOUNDS,
 *  info the slot) as in a workspace's error word. Asynchronous on `stream`.
 *  Errors: LMOE_ERR_INVALID_ARG for null pointers, K outside [1, 32], sizes,
 *  unaligned rows, topk_w without peer_gates or the reverse. */
lmoe_status lmoe_ep_dispatch(int64_t T, int K, int N, int G, const void* rows, int64_t row_bytes,
                             const int32_t* topk_idx, const int32_t* inv_perm, const int32_t* offsets,
                             const int32_t* expert_owner, const int32_t* dst_base, void* const* peer_rows,
                             int64_t peer_rows_cap, const float* topk_w, float* const* peer_gates, uint32_t* err_word,
                             void* stream);

/* Combine: c[t] = sum over the token's in-range slots, in k order, in fp32,
 * of the owner's expert-output row (BF16 [*][l], gates applied by the owner's
 * lmoe_expert_ffn from the dispatched gates) at the slot's row, stored BF16
 * -- lmoe_combine's arithmetic with topk_w NULL. peer_y [G]: DEVICE array of
 * the ranks' y buffers (16-byte aligned, peer_rows_cap rows each); the
 * other arguments as
 * lmoe_ep_dispatch; c [T][l] (16-byte aligned), l a multiple of 8.
 *  Errors: LMOE_ERR_INVALID_ARG for null pointers, K outside [1, 32], sizes,
 *  an unaligned c; LMOE_ERR_UNSUPPORTED for T >= 2^31. */
lmoe_status lmoe_ep_combine(int64_t T, int K, int N, int G, int l, const void* const* peer_y, int64_t peer_rows_cap,
                            const int32_t* topk_idx, const int32_t* inv_perm, const int32_t* offsets,
                            const int32_t* expert_owner, const int32_t* dst_base, void* c, uint32_t* err_word,
                            void* stream);

/* Synchronises `stream`, returns the device error status recorded in the
 * workspace `ws` (LMOE_OK if none) and clears it (the read and the clear run
 * on `stream`). `info` (host, may be NULL) receives a kernel-specific detail
 * word. Errors: LMOE_ERR_INVALID_ARG for a NULL ws; LMOE_ERR_CUDA when the
 * synchronisation, the read or the clear fails. */
lmoe_status lmoe_read_device_error(void* ws, void* stream, uint32_t* info);

/* Static description of a status code. */
const char* lmoe_status_string(lmoe_status s);

/* Self test of the device failure path (no counterpart on the pages): one
 * thread waits on an mbarrier that nothing arrives on, through the same
 * bounded wait every pipeline uses, shortened to limit_cycles (1 ..
 * 4e9 SM clock cycles). The wait gives up, records LMOE_ERR_DEVICE_TIMEOUT
 * with info 0x7001 in the workspace error word (first 256 bytes of `ws`,
 * zeroed before first use) and the kernel returns; lmoe_read_device_error
 * reports it and the context stays usable. Asynchronous on `stream`.
 * Errors: LMOE_ERR_WORKSPACE (ws NULL or < 256 bytes), LMOE_ERR_INVALID_ARG
 * (limit out of range). */
lmoe_status lmoe_selftest_wait_timeout(void* ws, size_t ws_bytes, uint64_t limit_cycles, void* stream);

/* Number of kernels launched by this library since load (host counter; used
 * by harnesses to report how many of the library's kernels a region ran). */
uint64_t lmoe_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* LMOE_H_ */
