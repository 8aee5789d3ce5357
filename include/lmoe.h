/*
 * lmoe.h -- C ABI of the B200 (sm_100a) LatentMoE layer: forward pass, its
 * backward pass (lmoe_backward) with the aux-loss-free router-bias update,
 * and the NVFP4 gradient-path pieces (lmoe_rht16, lmoe_nvfp4_quantize_sr).
 *
 * The layer ("NVIDIA Nemotron 3: Efficient and Open Intelligence", xllm-io
 * paper review, section 三 "LatentMoE 架构" with eq.(1); "Nemotron-3 Super
 * 精读报告", section 3.3 and table 2.2):
 *   router at hidden width d: z = W_r x, s = sigmoid(z), key = s + b
 *     ("Nemotron-3 Super 精读报告", table 6.3: Sigmoid + Expert Biasing);
 *   the top-K experts by key, weights w = s_sel / sum(s_sel);
 *   u = W_dn x (d -> l, BF16: the latent projections stay BF16 under the
 *     pages' NVFP4 recipe, "Nemotron-3 Super 精读报告" table 5.2);
 *   every selected expert in latent space: o_k = W2[e] sqrelu(W1[e] u);
 *   v = sum_k w_k o_k; r = W_upl v (l -> d);
 *   shared expert at width d: sh = W_s2 sqrelu(W_s1 x);  y = r + sh.
 * sqrelu(a) = max(a, 0)^2 is a convention: the pages name no activation.
 *
 * Conventions of every entry point:
 *   - matrices are row-major [out][in] (K-major), bf16 unless stated;
 *   - "device" pointers are CUDA device memory of the current device;
 *   - a `stream` argument is a cudaStream_t (NULL = legacy default stream);
 *   - calls return LMOE_OK (0) or a negative LMOE_ERR_* code and never throw,
 *     abort or print; lmoe_strerror() names a code;
 *   - kernels never trap: a bounded device-side wait that runs out records
 *     LMOE_ERR_TIMEOUT, read back by lmoe_sync_status().
 */
#ifndef LMOE_H_
#define LMOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LMOE_OK 0
#define LMOE_ERR_INVALID_ARG (-1) /* null pointer, bad size, T > max_tokens */
#define LMOE_ERR_UNSUPPORTED (-2) /* dims outside what the kernels handle   */
#define LMOE_ERR_OOM (-3)         /* device allocation failed (create only) */
#define LMOE_ERR_CUDA (-4)        /* a CUDA runtime/driver call failed      */
#define LMOE_ERR_TIMEOUT (-5)     /* a bounded device wait ran out          */
#define LMOE_ERR_DEVICE (-6)      /* a kernel flagged bad data (e.g. index) */

/* Standard MoE (lmoe_config.flags): no latent projections.  The experts
 * work at the hidden width (latent must equal d) on x itself, u = x and
 * r = v; w_dn and w_upl are ignored (may be NULL).  This is the layer the
 * pages compare LatentMoE against at equal active and total parameters
 * ("NVIDIA Nemotron 3: Efficient and Open Intelligence", section 三 eq.(1):
 * N = 128, K = 6 at d = 4096 against N' = 512, K' = 22 at l = 1024; section
 * 六 Table 1).  BF16 experts only. */
#define LMOE_FLAG_NO_PROJECTION 1

/* NVFP4 expert weights (lmoe_config.flags, LMOE_FMT_NVFP4 only), following
 * the pages' other weight recipes ("Nemotron-3 Super 精读报告", section 5.3:
 * 2D block scaling of weights in training; section 9.2: weight block scales
 * chosen by minimum weight MSE in post-training quantisation).  Activations
 * keep 1D max-based blocks.
 *   LMOE_FLAG_NVFP4_WEIGHT_2D: one E4M3 scale per 16 x 16 block of W1[e] and
 *     W2[e] (16 output rows by 16 reduction elements), from the block's amax.
 *   LMOE_FLAG_NVFP4_WEIGHT_MSE: each block's scale is the E4M3 code, from 8
 *     below to 2 above the max-based one, with the smallest squared error
 *     (float32, summed in row-major element order; ties to the higher code).
 * Both may be set (MSE search over 2D blocks).  Quantisation runs once, in
 * lmoe_create. */
#define LMOE_FLAG_NVFP4_WEIGHT_2D 2
#define LMOE_FLAG_NVFP4_WEIGHT_MSE 4
/* LMOE_FLAG_BACKWARD: also reserve the workspace of lmoe_backward (BF16
 * experts, or NVFP4 experts with LMOE_FLAG_NVFP4_WEIGHT_2D, with latent
 * projections; UNSUPPORTED otherwise). */
#define LMOE_FLAG_BACKWARD 8
/* LMOE_FLAG_EP_DENSE: a handle for expert parallelism that holds the router,
 * the latent projections and the shared expert but no expert weights (w1, w2
 * may be NULL): lmoe_forward_dispatch and lmoe_forward_combine apply, the
 * experts run in expert shards (lmoe_experts_create), lmoe_forward returns
 * UNSUPPORTED.  BF16 experts with latent projections only. */
#define LMOE_FLAG_EP_DENSE 16

#define LMOE_FMT_BF16 0  /* experts in BF16                                   */
#define LMOE_FMT_NVFP4 1 /* experts in NVFP4: W1, W2 and the expert inputs u
                            and H as E2M1 codes with E4M3 scales per 16
                            elements along the reduction axis and an FP32
                            global scale; latent projections, router and
                            shared expert stay BF16 ("Nemotron-3 Super 精读报告",
                            table 5.2).  Needs l and h multiples of 128.      */
#define LMOE_FMT_W4A16 3 /* experts with NVFP4 weights (as LMOE_FMT_NVFP4,
                            LMOE_FLAG_NVFP4_WEIGHT_* apply) and 16-bit
                            activations ("Nemotron 3 Ultra 解读", W4A16):
                            u and H stay unquantised, in FP16; the GEMMs
                            expand each weight tile to f16 in shared memory
                            (code value x block scale, exact) and apply the
                            global scale in the epilogue.  Needs l and h
                            multiples of 128; act_gscale_* unused.          */
#define LMOE_FMT_FP8 2   /* experts in FP8 W8A8 ("Nemotron-3 Super 精读报告",
                            section 9.1): W1, W2, u and H as E4M3 codes with
                            one FP32 scale per tensor (s_W = amax / 448 per
                            expert matrix, static scales for u and H from
                            act_gscale_*), value = code * s; router, latent
                            projections and shared expert stay BF16.  Needs
                            l and h multiples of 128.                        */

/* Layer shape.  d, latent, expert_hidden, shared_hidden: multiples of 64
 * (latent and expert_hidden multiples of 128 for LMOE_FMT_NVFP4 and _FP8).
 * n_experts: multiple of 32, at most 1024.  top_k: 1..min(32, n_experts).
 * max_tokens: the largest T a forward call accepts (sizes the workspace). */
typedef struct lmoe_config {
  int32_t d;             /* hidden width                                  */
  int32_t latent;        /* latent width l                                */
  int32_t n_experts;     /* N                                             */
  int32_t top_k;         /* K                                             */
  int32_t expert_hidden; /* h: expert FFN hidden width                    */
  int32_t shared_hidden; /* h_s: shared-expert hidden width               */
  int32_t expert_format; /* LMOE_FMT_*                                     */
  int32_t flags;         /* 0, or LMOE_FLAG_* bits (see above)            */
  int64_t max_tokens;    /* >= 1                                          */
} lmoe_config;

/* Layer weights, all device pointers, copied by lmoe_create (the caller may
 * free them afterwards). */
typedef struct lmoe_weights {
  const void* w_router;    /* [N][d]      bf16                              */
  const float* router_bias;/* [N]         fp32, or NULL for zeros           */
  const void* w_dn;        /* [l][d]      bf16 (unused without projections) */
  const void* w1;          /* [N][h][l]   bf16                              */
  const void* w2;          /* [N][l][h]   bf16                              */
  const void* w_upl;       /* [d][l]      bf16 (unused without projections) */
  const void* w_s1;        /* [h_s][d]    bf16                              */
  const void* w_s2;        /* [d][h_s]    bf16                              */
  float act_gscale_latent; /* NVFP4 and FP8 only (> 0): static scale of u --
                              NVFP4: global scale under the E4M3 block
                              scales E4M3(amax16/(6 g)); FP8: the per-tensor
                              scale, u = code * s                            */
  float act_gscale_hidden; /* NVFP4 and FP8 only (> 0): the same for the
                              expert hidden activation sqrelu(W1 u)         */
} lmoe_weights;

typedef struct lmoe_handle lmoe_handle;

/* Build a layer on the current device: validates cfg, allocates the weights'
 * copies (re-laid out: [W_r; W_dn; W_s1] as one [N+l+h_s][d] matrix and
 * [W_upl | W_s2] as one [d][l+h_s] matrix; for NVFP4 experts W1 and W2 are
 * quantised on the device instead, per expert matrix with global scale
 * amax/(6*448)) and a workspace for max_tokens, and synchronizes the device
 * once.  *out receives the handle, owned by the
 * caller until lmoe_destroy.  Errors: INVALID_ARG, UNSUPPORTED, OOM, CUDA. */
int lmoe_create(const lmoe_config* cfg, const lmoe_weights* w, lmoe_handle** out);

/* y = layer(x) for T tokens.  x: [T][d] bf16 device, y: [T][d] bf16 device,
 * both caller-owned, y must not overlap x.  Asynchronous on `stream`: no host
 * synchronisation, no allocation, no host<->device copy.  T == 0 is a no-op.
 * One forward may be in flight per handle (the workspace is shared); a handle
 * is not thread-safe.  Errors: INVALID_ARG (null, T < 0, T > max_tokens),
 * CUDA (a launch failed).  Device-side faults surface in lmoe_sync_status. */
int lmoe_forward(lmoe_handle* h, const void* x, int64_t T, void* y, void* stream);

/* Same as lmoe_forward with HOST buffers: copies x [T][d] bf16 to the device,
 * runs the layer and copies y [T][d] bf16 back on `stream`, then waits for the
 * stream.  Page-locked host buffers make the copies asynchronous.  Returns the
 * lmoe_sync_status() of the call. */
int lmoe_forward_host(lmoe_handle* h, const void* x_host, int64_t T, void* y_host, void* stream);

/* Waits for `stream`, then returns TIMEOUT or DEVICE if a kernel of this
 * handle raised its error word since the last call (and clears it), CUDA if
 * the stream reports an error, else OK. */
int lmoe_sync_status(lmoe_handle* h, void* stream);

/* Gradients of the weights, fp32 device buffers in the layouts of
 * lmoe_weights, written (not accumulated) by lmoe_backward. */
typedef struct lmoe_grads {
  float* d_router;  /* [N][d]     dL/dW_r                                   */
  float* d_dn;      /* [l][d]     dL/dW_dn                                  */
  float* d_w1;      /* [N][h][l]  dL/dW1 (zero for experts no token chose)  */
  float* d_w2;      /* [N][l][h]  dL/dW2                                    */
  float* d_upl;     /* [d][l]     dL/dW_upl                                 */
  float* d_s1;      /* [h_s][d]   dL/dW_s1                                  */
  float* d_s2;      /* [d][h_s]   dL/dW_s2                                  */
} lmoe_grads;

/* Backward pass of the last lmoe_forward on this handle: given dy = dL/dy
 * [T][d] bf16 (device), writes dx = dL/dx [T][d] bf16 (device) and the weight
 * gradients into *g.  x must be the forward's input (same pointer contents
 * and the same T); no other forward may run on the handle in between, since
 * the backward reads the forward's routing and saved activations (expert
 * inputs u, expert hidden sqrelu(W1 u), v and the shared hidden) from the
 * workspace.  The derivative is the exact one of the forward: the top-K
 * selection is piecewise constant, so the router receives gradient through
 * the renormalised weights w = s_S / sum s_S only, and the expert bias none
 * (see lmoe_bias_update).  The activation derivative 2 max(a, 0) is taken
 * as 2 sqrt(sqrelu(a)) from the saved bf16 hidden activations.  Products in
 * bf16 with fp32 accumulation; dx and the intermediate gradients rounded to
 * bf16.  Asynchronous on `stream`, no allocation.  dx must not overlap x or
 * dy; every pointer 16-byte aligned.  T == 0 is a no-op.
 * NVFP4 experts (LMOE_FMT_NVFP4 with LMOE_FLAG_NVFP4_WEIGHT_2D): the routed
 * experts follow the NVFP4 training recipe of lmoe_experts_backward_nvfp4
 * (their forward recomputed from the saved u), with the random bits of seed
 * 8 c, c the number of earlier lmoe_backward calls on the handle; the router,
 * the latent projections and the shared expert stay BF16.
 * Errors: INVALID_ARG (null, T differs from the last forward's, overlap,
 * misalignment), UNSUPPORTED (handle without LMOE_FLAG_BACKWARD, or not
 * BF16 or 2D-block NVFP4 experts with projections), CUDA. */
int lmoe_backward(lmoe_handle* h, const void* x, const void* dy, int64_t T, void* dx,
                  const lmoe_grads* g, void* stream);

/* Aux-loss-free load balancing ("Nemotron-3 Super 精读报告", table 6.3:
 * update rate 1e-3): after a forward, every expert bias moves by
 * rate * sign(mean - c_e), c_e the rows routed to expert e by that forward
 * and mean = T K / N (an expert exactly at the mean keeps its bias); float32
 * arithmetic on the handle's router bias, which the next forward uses.
 * Asynchronous on `stream`.  Errors: INVALID_ARG (no forward yet, rate not
 * finite), CUDA. */
int lmoe_bias_update(lmoe_handle* h, float rate, void* stream);

/* Debug/test readout of the last forward's intermediates into HOST memory
 * (synchronizes the device first).  `bytes` must equal the item's size for
 * the last T:
 *   LMOE_DBG_TOPK_IDX  int32 [T][K]   selected experts, key-descending
 *   LMOE_DBG_TOPK_W    fp32  [T][K]   renormalised router weights
 *   LMOE_DBG_COUNTS    int32 [N]      routed rows per expert
 *   LMOE_DBG_OFFSETS   int32 [N+1]    exclusive scan of counts
 *   LMOE_DBG_PERM      int32 [T*K]    row -> t*K + k (expert, then token order)
 *   LMOE_DBG_INV       int32 [T][K]   slot -> row
 *   LMOE_DBG_LOGITS    fp32  [T][N]   router logits z
 *   LMOE_DBG_U         bf16  [T][l]   latent u
 *   LMOE_DBG_V         bf16  [T][l]   latent combine v
 *   LMOE_DBG_HS        bf16  [T][h_s] shared hidden sqrelu(W_s1 x)
 *   LMOE_DBG_BIAS      fp32  [N]      the router bias (after lmoe_bias_update)
 * and, for NVFP4 experts (lp, hp = l, h rounded up to 256):
 *   LMOE_DBG_W1Q_CODES u8   [N*h][lp/2]  E2M1 codes, lower index in the low nibble
 *   LMOE_DBG_W1Q_SF    u8   [N*h/128][lp/64][512] E4M3 scales; row m, 16-block
 *                           k1 of a 64-chunk at byte (m%32)*16+((m/32)%4)*4+k1
 *   LMOE_DBG_W1Q_G     fp32 [N]          global scales
 *   LMOE_DBG_W2Q_CODES / _SF / _G   the same for W2 ([N*l][hp/2], ...)
 * Errors: INVALID_ARG (unknown item, wrong size), CUDA. */
#define LMOE_DBG_TOPK_IDX 1
#define LMOE_DBG_TOPK_W 2
#define LMOE_DBG_COUNTS 3
#define LMOE_DBG_OFFSETS 4
#define LMOE_DBG_PERM 5
#define LMOE_DBG_INV 6
#define LMOE_DBG_LOGITS 7
#define LMOE_DBG_U 8
#define LMOE_DBG_V 9
#define LMOE_DBG_HS 10
#define LMOE_DBG_W1Q_CODES 11
#define LMOE_DBG_W1Q_SF 12
#define LMOE_DBG_W1Q_G 13
#define LMOE_DBG_W2Q_CODES 14
#define LMOE_DBG_W2Q_SF 15
#define LMOE_DBG_W2Q_G 16
#define LMOE_DBG_BIAS 17
/* and of the last lmoe_experts_backward_nvfp4 (R = T K routed rows in expert
 * order, C = columns of the transposed operands, lmoe_nvfp4_bw_columns):
 *   LMOE_DBG_BW4_DO_CODES u8  [R][l/2]   NVFP4 codes of w dv (stochastic)
 *   LMOE_DBG_BW4_DO_SF    u8  [R][l/16]  their E4M3 scales
 *   LMOE_DBG_BW4_DOT_CODES u8 [l][C/2]   codes of the transformed (w dv)^T
 *   LMOE_DBG_BW4_DOT_SF   u8  [l][C/16]
 *   LMOE_DBG_BW4_UT_CODES u8  [l][C/2]   codes of the transformed u^T
 *   LMOE_DBG_BW4_UT_SF    u8  [l][C/16]
 *   LMOE_DBG_BW4_SCALES   fp32 [16]      amax of w dv, da, (w dv)^T, g^T,
 *                                        da^T, u^T, two unused, then their
 *                                        global scales in the same order
 *   LMOE_DBG_BW4_SEG      int32 [2][N+1] column offsets of the experts in the
 *                                        transposed operands, segments
 *                                        padded to 16, then to 256
 *   LMOE_DBG_BW4_DA       fp32 [R][h]    da = (W2q^T Q(w dv)) 2 max(a, 0) */
#define LMOE_DBG_BW4_DO_CODES 18
#define LMOE_DBG_BW4_DO_SF 19
#define LMOE_DBG_BW4_DOT_CODES 20
#define LMOE_DBG_BW4_DOT_SF 21
#define LMOE_DBG_BW4_UT_CODES 22
#define LMOE_DBG_BW4_UT_SF 23
#define LMOE_DBG_BW4_SCALES 24
#define LMOE_DBG_BW4_SEG 25
#define LMOE_DBG_BW4_DA 26
/* NVFP4 experts: the scale tables of the static scales g_u then g_h, fp32
 * [2][256]: [k] for k = 1..126 the smallest block amax whose scale code
 * E4M3(f32(amax / f32(6 g))) is at least k ([0] = 0, [127] = infinity),
 * [128 + k] = f32(1 / f32(E4M3value(k) g)) (0 when that product is 0),
 * [255] = f32(1 / f32(6 g)); the activation quantisers use them instead of
 * dividing. */
#define LMOE_DBG_SCALE_TABLES 27
/* Handles with LMOE_FLAG_BACKWARD: dL/dv of the last lmoe_backward, bf16
 * [T][l] (the experts' output gradient before the router weights). */
#define LMOE_DBG_DV 28
int lmoe_get_debug(lmoe_handle* h, int what, void* dst_host, size_t bytes);

/* Kernel launches one lmoe_forward of T tokens issues, or a negative error
 * code: 10, plus the y-GEMM's split-K reduction when T is small, minus 2
 * up to 256 tokens (the per-expert segments from one kernel instead of
 * histogram, scan and scatter), plus 2 for the opt-in overlapped forward
 * (the shared expert's GEMMs apart).  When the x-GEMM ([W_r; W_dn; W_s1] x)
 * splits K, its reduction also runs the router (sigmoid, bias, top-K,
 * renormalised weights) and replaces the router kernel, so the count stays
 * the same. */
int lmoe_launches_per_forward(const lmoe_handle* h, int64_t T);

/* Per-kernel timing: when enabled, every forward records CUDA events around
 * each of its kernels on the forward's stream and accumulates their elapsed
 * times (read at lmoe_profile_read, which synchronizes the device).
 * lmoe_profile_read fills up to `max` entries: name (static string), total
 * milliseconds and launch count, and returns the number of entries; `reset`
 * != 0 clears the accumulators.  Errors: INVALID_ARG, CUDA. */
int lmoe_profile_enable(lmoe_handle* h, int on);
int lmoe_profile_read(lmoe_handle* h, const char** names, double* total_ms, int64_t* launches,
                      int max, int reset);

/* Standalone routing and segment build (the router's top-K, weights and the
 * per-expert row order) from precomputed fp32 logits [T][N] (device):
 * outputs (device, caller-owned) topk_idx [T][K] int32, topk_w [T][K] fp32,
 * counts [N] int32, offsets [N+1] int32, perm [T*K] int32, inv [T][K] int32.
 * bias: [N] fp32 device or NULL.  workspace: device scratch of at least
 * lmoe_route_workspace_size(T, N) bytes, 256-byte aligned, caller-owned.
 * Asynchronous on `stream`.  Errors: INVALID_ARG, UNSUPPORTED, CUDA; a
 * selected expert index outside [0, N) found by the segment kernels is
 * recorded in the workspace (cleared at the start of each call) and read by
 * lmoe_route_status. */
size_t lmoe_route_workspace_size(int64_t T, int32_t N);
int lmoe_route(const float* logits, const float* bias, int64_t T, int32_t N, int32_t K,
               int32_t* topk_idx, float* topk_w, int32_t* counts, int32_t* offsets,
               int32_t* perm, int32_t* inv, void* workspace, size_t workspace_bytes,
               void* stream);

/* Device status of the last lmoe_route call that used `workspace` with the
 * same T and N: waits for `stream`, then returns DEVICE if that call's
 * kernels flagged an expert index outside [0, N), else OK.  Reading does not
 * clear the record (the next lmoe_route call on the workspace does).
 * Errors: INVALID_ARG (null or misaligned workspace, T < 0, N <= 0), CUDA. */
int lmoe_route_status(const void* workspace, int64_t T, int32_t N, void* stream);

/* Allocation-free variant of lmoe_route (no counterpart on the pages: it is a
 * deployment convenience).  For callers that cannot give this library device
 * memory -- e.g. a serving engine that reserves all of HBM for its own pool at
 * start-up, or a host path where cudaMalloc (which may synchronize the device)
 * is not allowed -- the scratch lives in a static device array of about 2 MiB
 * that every GPU loading the library holds until the process exits.  Same
 * arguments and outputs as lmoe_route minus the workspace; it allocates
 * nothing (no cudaMalloc/cudaFree, no allocating library call).
 * Limits: T <= LMOE_NOALLOC_MAX_TOKENS, T*K <= LMOE_NOALLOC_MAX_ROUTED,
 * N <= 1024; larger sizes return LMOE_ERR_UNSUPPORTED.
 * The first call on a device looks up the array's device address once (with
 * that device current); make that first call before any stream capture.
 * All calls share the one array, so calls whose work overlaps on the GPU
 * (other streams, other host threads) race: serialize them.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA; a flagged expert index is recorded
 * in the shared array and read by lmoe_route_noalloc_status. */
#define LMOE_NOALLOC_MAX_TOKENS 8192
#define LMOE_NOALLOC_MAX_ROUTED 262144
int lmoe_route_noalloc(const float* logits, const float* bias, int64_t T, int32_t N, int32_t K,
                       int32_t* topk_idx, float* topk_w, int32_t* counts, int32_t* offsets,
                       int32_t* perm, int32_t* inv, void* stream);

/* Device status of the last lmoe_route_noalloc call on the current device:
 * waits for `stream`, then returns DEVICE if that call's kernels flagged an
 * expert index outside [0, N), else OK.  The next lmoe_route_noalloc call
 * clears the record, so read it before making another call.  Allocates
 * nothing.  Errors: UNSUPPORTED (device ordinal >= 256), CUDA. */
int lmoe_route_noalloc_status(void* stream);

/* NVFP4 quantisation of fp32 rows x [rows][cols] (device, 16-byte aligned,
 * cols a multiple of 16) with global scale g >= 0, exactly as the layer
 * quantises its activations: per 16 consecutive elements s = E4M3(amax /
 * (6 g)) and q = E2M1(x * r) with r = 1 / (s g) rounded once per block
 * (round to nearest even, saturating; all float32).  Outputs (device): codes [rows][cols/2] (lower index in the low
 * nibble), scales [rows][cols/16] E4M3 codes.  Asynchronous on `stream`.
 * Errors: INVALID_ARG, CUDA. */
int lmoe_nvfp4_quantize(const float* x, int64_t rows, int32_t cols, float g, uint8_t* codes,
                        uint8_t* scales, void* stream);

/* Gradient-path pieces of the NVFP4 training recipe ("Nemotron-3 Super
 * 精读报告", section 5.3: a random Hadamard transform on the weight-gradient
 * GEMMs' inputs, stochastic rounding of gradients).  Random bits come from
 * SplitMix64 (Steele, Lea, Flood, OOPSLA 2014) as a counter-based generator:
 * counter i of `seed` gives mix(seed + (i + 1) * 0x9E3779B97F4A7C15).
 *
 * lmoe_rht16: y = (1/4) H16 diag(s) x on every 16 consecutive elements of
 * the fp32 rows x [rows][cols] (cols a multiple of 16), H16 the 16 x 16
 * Sylvester Hadamard matrix and s the 16 signs of counters 0..15 (-1 where
 * bit 63 is set), shared by all blocks; float32 butterflies (stages 1, 2, 4,
 * 8: (a, b) -> (a + b, a - b)), then x 0.25.  Orthonormal and its own inverse
 * up to the signs.  x and y device, 16-byte aligned; y may equal x.
 *
 * lmoe_nvfp4_quantize_sr: as lmoe_nvfp4_quantize (same block scales), but
 * each element v = f32(x * r) rounds to the upper of its two E2M1 grid
 * neighbours with probability (|v| - lo) / (hi - lo), decided by the
 * uniform (top 24 bits x 2^-24) of counter row * cols + col: unbiased in
 * expectation.  Asynchronous on `stream`.  Errors: INVALID_ARG, CUDA. */
int lmoe_rht16(const float* x, int64_t rows, int32_t cols, uint64_t seed, float* y,
               void* stream);
int lmoe_nvfp4_quantize_sr(const float* x, int64_t rows, int32_t cols, float g, uint64_t seed,
                           uint8_t* codes, uint8_t* scales, void* stream);

/* Runs a one-CTA kernel that waits on an mbarrier nothing arrives on, with a
 * wait limit of limit_ns nanoseconds (1e3..1e10), and returns the status the
 * host reads afterwards: LMOE_ERR_TIMEOUT when the bounded wait gave up as
 * designed.  Checks the device-side failure path without a fault. */
int lmoe_check_bounded_wait(int64_t limit_ns);

/* Expert parallelism ("NVIDIA Nemotron 3: Efficient and Open Intelligence",
 * section 三: the routed experts work on l-wide latent rows, so an expert-
 * parallel exchange moves l values per routed row instead of d;
 * "Nemotron-3 Super 精读报告", section 6.5: 64-way expert parallelism).  The
 * experts are split into contiguous ranges, one per rank; a rank's forward is
 *   lmoe_forward_dispatch   (router, projections, shared expert, segments and
 *                            the latent rows of every routed (token, expert)
 *                            pair in expert order: the send buffer);
 *   exchange                (the caller: all-to-all of row slices by expert
 *                            range, re-sort into local expert order with
 *                            lmoe_permute_rows);
 *   lmoe_experts_forward    (the grouped expert GEMMs of a shard);
 *   exchange back           (lmoe_permute_rows, reverse all-to-all);
 *   lmoe_forward_combine    (weighted sum per token, up-projection + shared).
 * BF16 experts with latent projections only; asynchronous on `stream`.
 *
 * lmoe_forward_dispatch: x [T][d] bf16 (device) -> rows_out [T*K][l] bf16
 * (device, caller-owned, 16-byte aligned): u = W_dn x of the token of each
 * routed row, rows in expert order (expert, then token, then slot; the
 * order of LMOE_DBG_PERM), and counts_out [N] int32 (device): rows per
 * expert.  A layer handle (with or without LMOE_FLAG_EP_DENSE).  Keeps the
 * routing for lmoe_forward_combine.  Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
int lmoe_forward_dispatch(lmoe_handle* h, const void* x, int64_t T, void* rows_out,
                          int32_t* counts_out, void* stream);

/* lmoe_forward_combine: rows_in [T*K][l] bf16 (device) -- the expert outputs
 * W2[e] sqrelu(W1[e] u), unweighted, in the order of the last dispatch's
 * rows_out -- -> y [T][d] bf16 (device): v = sum_k w_k o_k per token (fp32,
 * slot order), y = W_upl v + W_s2 sqrelu(W_s1 x).  T must be the last
 * dispatch's.  Errors: INVALID_ARG (T differs, null, misaligned),
 * UNSUPPORTED, CUDA. */
int lmoe_forward_combine(lmoe_handle* h, const void* rows_in, int64_t T, void* y, void* stream);

/* An expert shard: experts [first_expert, first_expert + n_local) of the layer
 * described by cfg (n_experts is the layer's N; BF16 experts; flags 0 or
 * LMOE_FLAG_EP_DENSE).  w1 [n_local][h][l] and w2 [n_local][l][h] bf16
 * (device) are the shard's experts, copied.  max_rows: the most rows one
 * lmoe_experts_forward accepts.  The handle takes lmoe_experts_forward,
 * lmoe_sync_status and lmoe_destroy; the layer calls return UNSUPPORTED or
 * INVALID_ARG on it.  Errors: INVALID_ARG, UNSUPPORTED, OOM, CUDA. */
int lmoe_experts_create(const lmoe_config* cfg, int32_t first_expert, int32_t n_local,
                        const void* w1, const void* w2, int64_t max_rows, lmoe_handle** out);

/* out[r] = W2[e] sqrelu(W1[e] rows[r]) for the R rows [R][l] bf16 (device) in
 * local expert order, counts [n_local] int32 (device) rows per local expert;
 * out [R][l] bf16 (device, must not overlap rows).  The counts are checked on
 * the device: a negative count or a sum other than R computes nothing and
 * records DEVICE (read by lmoe_sync_status).  Errors: INVALID_ARG (null, R <
 * 0, R > max_rows, overlap, misalignment), CUDA. */
int lmoe_experts_forward(lmoe_handle* h, const void* rows, const int32_t* counts, int64_t R,
                         void* out, void* stream);

/* Row permutation of an exchange: rows of row_bytes (a multiple of 16),
 * gather (scatter = 0) dst[r] = src[idx[r]] or scatter (scatter = 1)
 * dst[idx[r]] = src[r], for r < n; idx int32 (device).  An index outside
 * [0, n_other) -- the row count of the indexed side -- skips its row.
 * src, dst 16-byte aligned, not overlapping.  Errors: INVALID_ARG, CUDA. */
int lmoe_permute_rows(const void* src, const int32_t* idx, int64_t n, int64_t n_other,
                      int32_t row_bytes, void* dst, int scatter, void* stream);

/* The routed experts' forward and backward under the NVFP4 training recipe
 * ("Nemotron-3 Super 精读报告", section 5.3: fprop, dgrad and wgrad GEMMs in
 * NVFP4; weights in 2D 16 x 16 blocks, whose one scale serves W and W^T;
 * activations and gradients in 1D blocks along each GEMM's reduction axis; a
 * random Hadamard transform on the weight-gradient GEMMs' inputs; stochastic
 * rounding of the gradients).  A handle with LMOE_FMT_NVFP4,
 * LMOE_FLAG_NVFP4_WEIGHT_2D and LMOE_FLAG_BACKWARD (else UNSUPPORTED).
 * Inputs (device): u [T][l] bf16 latent rows, topk_idx [T][K] int32 selected
 * experts (distinct per token), topk_w [T][K] fp32 router weights, dv [T][l]
 * bf16 = dL/dv.  The forward: u and sqrelu(W1q u) quantised with the
 * handle's static scales (act_gscale_*), o = W2q g per routed row.  The
 * backward, rows in expert order (expert, token, slot):
 *   dw[t][k] = o . dv[t];  do = w dv, stochastically rounded with global
 *   scale amax / (6 * 448) and the counters of seed + 0;  da = (W2q^T Q(do))
 *   2 max(a, 0), a = W1q u, stochastically rounded (seed + 1);
 *   du[t] = sum over t's rows of W1q^T Q(da);
 *   dW2[e] = Q_sr(R(do_e^T)) Q(R(g_e^T))^T, dW1[e] = Q_sr(R(da_e^T))
 *   Q(R(u_e^T))^T over expert e's rows, R the transform on 16-row blocks
 *   (signs of seed + 2 for dW2, seed + 4 for dW1), stochastic rounding with
 *   seed + 3 (do^T) and seed + 5 (da^T), element (f, j) of an operand taking
 *   the counter of its place in the layout whose expert segments are padded
 *   to 16 rows; every tensor's global scale is its amax / (6 * 448).
 * Outputs (device): du [T][l] bf16, dw [T][K] fp32, d_w1 [N][h][l] and d_w2
 * [N][l][h] fp32 (zero for experts without rows).  Asynchronous on `stream`;
 * 16-byte aligned pointers.  Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
int lmoe_experts_backward_nvfp4(lmoe_handle* h, const void* u, const int32_t* topk_idx,
                                const float* topk_w, const void* dv, int64_t T, uint64_t seed,
                                void* du, float* dw, float* d_w1, float* d_w2, void* stream);

/* Columns C of the transposed weight-gradient operands of an NVFP4 training
 * handle (the row pitch of LMOE_DBG_BW4_*T_*), or a negative error code. */
int64_t lmoe_nvfp4_bw_columns(const lmoe_handle* h);

/* Frees everything the handle owns (synchronizes the device first). */
void lmoe_destroy(lmoe_handle* h);

/* Static description of an error code. */
const char* lmoe_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* LMOE_H_ */
