/*
 * libqlora: QLoRA projection through a frozen NF4 base weight plus a rank-r
 * LoRA adapter, forward and hand-derived backward, and the gated MLP built
 * from three such projections.  Hand-written CUDA for sm_100a (B200).
 *
 * Sources (web pages on Unsloth's QLoRA kernels, cited by title + section):
 *  - Mistral blog "用 Unsloth 微调 Mistral，速度提升 14 倍": benchmark
 *    configuration (QLoRA nf4 on q/k/v/o/gate/up/down, rank 16, alpha 16,
 *    dropout 0); per-optimisation table items "2. Bitsandbytes bfloat16"
 *    (dequantise straight to bf16) and "10、11. 手动 Autograd" (hand-derived
 *    backward, rank-r factor bracketed first).
 *  - Gemma blog "使用 Unsloth 微调 Gemma：速度提升 2.4 倍，显存占用降低 58%",
 *    section "GeGLU 与 Swiglu 激活函数" (gated MLP activations and their
 *    derivatives).
 *  - Show HN "80% faster, 50% less memory, 0% loss of accuracy Llama
 *    finetuning": highlight 1 (manual autograd), highlight 4 (exact), and the
 *    link to the QLoRA paper for the NF4 format.
 *
 * Conventions for every call
 *  - All tensors are row-major and contiguous, in device memory owned by the
 *    caller; every pointer must be 16-byte aligned.  bf16 values are passed as
 *    `qlora_bf16` (their 16-bit pattern).
 *  - Shapes follow nn.Linear: base weight W [n_out, k_in], LoRA A [k_in, r],
 *    LoRA B [r, n_out], activations X [M, k_in], output Y [M, n_out].
 *    The LoRA scale is s = alpha / r (passed as `scale`).
 *  - Every call enqueues work on the caller's stream and returns without
 *    synchronising.  The library never allocates device memory: the caller
 *    passes a workspace of at least the size the matching *_workspace_bytes
 *    query returns; its first 256 bytes hold the device status word and must
 *    be zeroed by the caller once before first use.
 *  - Invalid arguments are rejected on the host before anything is enqueued
 *    (QLORA_ERR_INVALID_ARG, _UNSUPPORTED_SHAPE, _MISALIGNED,
 *    _WORKSPACE_TOO_SMALL).  A failed launch returns QLORA_ERR_CUDA.  Errors
 *    found on the device (a pipeline wait that exceeded its time limit) are
 *    recorded in the status word and reported by qlora_last_device_status.
 *  - M = 0 is valid.  A forward then enqueues nothing; a backward sets its
 *    adapter gradients dA, dB to zero (sums over no tokens) with memsets on
 *    the stream and reads or writes nothing else.
 *  - M, k_in, n_out (and nq + nk + nv of the fused Q/K/V calls) are at most
 *    2^23 = 8,388,608; larger values return QLORA_ERR_UNSUPPORTED_SHAPE (the
 *    kernels index rank-side partials and output tiles with 32-bit integers).
 */
#ifndef QLORA_H_
#define QLORA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* qlora_stream_t; /* a cudaStream_t; NULL = legacy default stream */
typedef struct CUevent_st* qlora_event_t;   /* a cudaEvent_t */
typedef uint16_t qlora_bf16;                /* bf16 bit pattern */

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad enum */
  QLORA_ERR_UNSUPPORTED_SHAPE = 2,  /* k_in % 64 != 0, n_out % 8 != 0, unsupported rank ... */
  QLORA_ERR_MISALIGNED = 3,         /* a pointer is not 16-byte aligned */
  QLORA_ERR_WORKSPACE_TOO_SMALL = 4,
  QLORA_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed */
  QLORA_ERR_TIMEOUT = 6,            /* a device pipeline wait exceeded its limit */
  QLORA_ERR_DEVICE = 7              /* other device-side error flag */
} qlora_status;

typedef enum { QLORA_ACT_SWIGLU = 0, QLORA_ACT_GEGLU_TANH = 1 } qlora_act;

/* NF4 weight: codes uint8 [n_out * k_in / 2] (two 4-bit level indices per
 * byte, even element in the high nibble), absmax fp32 [n_out * k_in / 64]
 * (one per block of 64 consecutive elements along k_in). */
typedef struct {
  const uint8_t* codes;
  const float* absmax;
  int64_t n_out;
  int64_t k_in;
} qlora_nf4;

/* One QLoRA projection: frozen NF4 base W plus LoRA A [k_in, r], B [r, n_out]. */
typedef struct {
  qlora_nf4 w;
  const qlora_bf16* A;
  const qlora_bf16* B;
  int32_t r;   /* 16, 32 or 64 (tile configuration 4); 16 (configurations 1-3) */
  float scale; /* s = alpha / r (or any scale, e.g. alpha / sqrt(r)) */
} qlora_lora_linear;

/* One projection with a frozen bf16 base W [n_out, k_in] (row-major) instead
 * of NF4: plain LoRA rather than QLoRA (Mistral blog FAQ, "load_in_4bit set
 * to False"; Show HN highlight 7, 4-bit and 16-bit LoRA).  Same LoRA factors
 * and scale as qlora_lora_linear. */
typedef struct {
  const qlora_bf16* w;
  int64_t n_out;
  int64_t k_in;
  const qlora_bf16* A;
  const qlora_bf16* B;
  int32_t r;   /* 16, 32 or 64 */
  float scale; /* s = alpha / r (or any scale) */
} qlora_lora_linear16;

/* Tensors the MLP forward saves for its backward (caller-allocated):
 * E, G, H [M, h] (e = gate projection, g = up projection, h = act(e) * g),
 * XA_g, XA_u [M, r] (X A_g, X A_u) and HA_d [M, r] (H A_d). */
typedef struct {
  qlora_bf16* E;
  qlora_bf16* G;
  qlora_bf16* H;
  qlora_bf16* XA_g;
  qlora_bf16* XA_u;
  qlora_bf16* HA_d;
} qlora_mlp_saved;

/* The 16 NF4 levels this library uses, as binary32, ascending.  Host only;
 * needs no GPU.  Levels: QLoRA NormalFloat construction (Show HN thread's
 * QLoRA link), normalised to [-1, 1] with an exact 0 at index 7. */
QLORA_API qlora_status qlora_nf4_codebook(float out[16]);

/* NF4 block quantisation of a bf16 weight [n_out, k_in] (k_in % 64 == 0).
 * absmax = max |w| per 64-block; v = w / absmax rounded to binary32; level =
 * number of level midpoints strictly below v (ties to the lower level);
 * all-zero blocks store level 7.  Writes codes [n_out*k_in/2] and
 * absmax [n_out*k_in/64].  (Mistral blog benchmark configuration, QLoRA nf4.) */
QLORA_API qlora_status nf4_quantize(const qlora_bf16* w, int64_t n_out, int64_t k_in, uint8_t* codes, float* absmax,
                          qlora_stream_t stream);

/* NF4 dequantisation straight to bf16 (Mistral blog item "2. Bitsandbytes
 * bfloat16"): out[n, k] = RNE_bf16(level[q] * absmax) with the product in
 * binary32.  Bit-exact.  out is [n_out, k_in]. */
QLORA_API qlora_status nf4_dequantize(const uint8_t* codes, const float* absmax, int64_t n_out, int64_t k_in, qlora_bf16* out,
                            qlora_stream_t stream);

/* Workspace bytes needed by qlora_linear_fwd and qlora_linear_bwd under the
 * current tile configuration (the staged configuration 4 adds room for the
 * dequantised bf16 weight, n_out * k_in * 2 bytes). */
QLORA_API size_t qlora_linear_workspace_bytes(int64_t M, int64_t k_in, int64_t n_out, int32_t r);

/* Forward of one QLoRA projection (Mistral blog "10、11. 手动 Autograd"):
 *   XA = X A                      -> XA_saved [M, r]  (kept for the backward)
 *   Y  = X dequant(W)^T + s XA B  -> Y [M, n_out]
 * X [M, k_in].  Requires k_in % 64 == 0 (one NF4 block), n_out % 8 == 0, and
 * r = 16, 32 or 64 under tile configuration 4 (what the default, automatic
 * setting uses here).  Tile configurations 1-3 further require k_in % 256 ==
 * 0 (their GEMM loads each weight row's absmax values by TMA, in 16-byte
 * pieces) and r = 16. */
QLORA_API qlora_status qlora_linear_fwd(const qlora_lora_linear* lin, const qlora_bf16* X, int64_t M, qlora_bf16* Y,
                              qlora_bf16* XA_saved, void* workspace, size_t workspace_bytes, qlora_stream_t stream);

/* Hand-derived backward (Mistral blog "10、11. 手动 Autograd"; Show HN
 * highlight 1), rank-r factor bracketed first, no gradient for the frozen W:
 *   G  = dY B^T                    [M, r]
 *   dX = dY dequant(W) + s G A^T   -> dX [M, k_in]
 *   dA = s X^T G                   -> dA [k_in, r]
 *   dB = s (XA)^T dY               -> dB [r, n_out]
 * dY [M, n_out]; XA_saved from qlora_linear_fwd. */
QLORA_API qlora_status qlora_linear_bwd(const qlora_lora_linear* lin, const qlora_bf16* X, const qlora_bf16* XA_saved,
                              const qlora_bf16* dY, int64_t M, qlora_bf16* dX, qlora_bf16* dA, qlora_bf16* dB,
                              void* workspace, size_t workspace_bytes, qlora_stream_t stream);

/* Workspace bytes needed by qlora_mlp_fwd and qlora_mlp_bwd (d = model
 * width, h = MLP width) under the current tile configuration (configuration 4
 * adds room for two dequantised bf16 weights, 2 * h * d * 2 bytes). */
QLORA_API size_t qlora_mlp_workspace_bytes(int64_t M, int64_t d, int64_t h, int32_t r);

/* Gated MLP forward (Gemma blog "GeGLU 与 Swiglu 激活函数"):
 *   e = X Wg^T + s_g (X A_g) B_g,  g = X Wu^T + s_u (X A_u) B_u,
 *   h = act(e) * g,  Y = h Wd^T + s_d (h A_d) B_d,
 * act = SiLU (QLORA_ACT_SWIGLU) or tanh-approximate GELU
 * (QLORA_ACT_GEGLU_TANH).  gate/up: n_out = h, k_in = d; down: n_out = d,
 * k_in = h.  X [M, d], Y [M, d]; `saved` receives E, G, H, XA_g, XA_u, HA_d.
 * Requires d % 64 == 0, h % 256 == 0, the same r for the three projections,
 * and r = 16, 32 or 64 under tile configuration 4; tile configurations 1-3
 * require d % 256 == 0 and r = 16 (the automatic setting picks 2 only when
 * they hold; see qlora_set_tile_config). */
QLORA_API qlora_status qlora_mlp_fwd(qlora_act act, const qlora_lora_linear* gate, const qlora_lora_linear* up,
                           const qlora_lora_linear* down, const qlora_bf16* X, int64_t M, qlora_bf16* Y,
                           const qlora_mlp_saved* saved, void* workspace, size_t workspace_bytes,
                           qlora_stream_t stream);

/* Gated MLP backward by the chain rule with closed-form act':
 *   dH = dY Wd + s_d (dY B_d^T) A_d^T,  dE = dH * g * act'(e),  dG = dH * act(e),
 *   dX = dE Wg + dG Wu + s_g (dE B_g^T) A_g^T + s_u (dG B_u^T) A_u^T,
 * and the six adapter gradients dA_* [k_in, r], dB_* [r, n_out] of the three
 * projections as in qlora_linear_bwd.  dY [M, d] -> dX [M, d]. */
QLORA_API qlora_status qlora_mlp_bwd(qlora_act act, const qlora_lora_linear* gate, const qlora_lora_linear* up,
                           const qlora_lora_linear* down, const qlora_bf16* X, const qlora_mlp_saved* saved,
                           const qlora_bf16* dY, int64_t M, qlora_bf16* dX, qlora_bf16* dA_g, qlora_bf16* dB_g,
                           qlora_bf16* dA_u, qlora_bf16* dB_u, qlora_bf16* dA_d, qlora_bf16* dB_d, void* workspace,
                           size_t workspace_bytes, qlora_stream_t stream);

/* qlora_mlp_bwd that also records `early_grads` (a cudaEvent_t created by the
 * caller; NULL = none) on `stream` as soon as dA_d, dB_d, dB_g and dB_u are
 * final, before the gate/up dX GEMM is enqueued (for M = 0, after their
 * memsets).  A data-parallel caller can make a second stream wait for that
 * event and start summing those four gradients across ranks while the rest of
 * the backward runs (the pages' DDP gradient sync; Mistral blog, 2 x T4 DDP
 * tables).  Everything else is exactly qlora_mlp_bwd. */
QLORA_API qlora_status qlora_mlp_bwd_ev(qlora_act act, const qlora_lora_linear* gate, const qlora_lora_linear* up,
                                        const qlora_lora_linear* down, const qlora_bf16* X,
                                        const qlora_mlp_saved* saved, const qlora_bf16* dY, int64_t M, qlora_bf16* dX,
                                        qlora_bf16* dA_g, qlora_bf16* dB_g, qlora_bf16* dA_u, qlora_bf16* dB_u,
                                        qlora_bf16* dA_d, qlora_bf16* dB_d, void* workspace, size_t workspace_bytes,
                                        qlora_stream_t stream, qlora_event_t early_grads);

/* The same four computations with bf16 base weights (qlora_lora_linear16):
 * outputs, saved tensors, shapes, workspace rules and errors as the NF4 calls
 * above, with dequant(W) replaced by W itself.  They always run the CTA-pair
 * GEMM that streams the weight by TMA (tile configuration 4), whatever
 * qlora_set_tile_config selected, and need no room for a staged weight: the
 * *16_workspace_bytes queries give their sizes.  The three weights of an MLP
 * call must all be bf16. */
QLORA_API size_t qlora_linear16_workspace_bytes(int64_t M, int64_t k_in, int64_t n_out, int32_t r);
QLORA_API size_t qlora_mlp16_workspace_bytes(int64_t M, int64_t d, int64_t h, int32_t r);
QLORA_API qlora_status qlora_linear16_fwd(const qlora_lora_linear16* lin, const qlora_bf16* X, int64_t M,
                                          qlora_bf16* Y, qlora_bf16* XA_saved, void* workspace, size_t workspace_bytes,
                                          qlora_stream_t stream);
QLORA_API qlora_status qlora_linear16_bwd(const qlora_lora_linear16* lin, const qlora_bf16* X,
                                          const qlora_bf16* XA_saved, const qlora_bf16* dY, int64_t M, qlora_bf16* dX,
                                          qlora_bf16* dA, qlora_bf16* dB, void* workspace, size_t workspace_bytes,
                                          qlora_stream_t stream);
QLORA_API qlora_status qlora_mlp16_fwd(qlora_act act, const qlora_lora_linear16* gate,
                                       const qlora_lora_linear16* up, const qlora_lora_linear16* down,
                                       const qlora_bf16* X, int64_t M, qlora_bf16* Y, const qlora_mlp_saved* saved,
                                       void* workspace, size_t workspace_bytes, qlora_stream_t stream);
QLORA_API qlora_status qlora_mlp16_bwd(qlora_act act, const qlora_lora_linear16* gate,
                                       const qlora_lora_linear16* up, const qlora_lora_linear16* down,
                                       const qlora_bf16* X, const qlora_mlp_saved* saved, const qlora_bf16* dY,
                                       int64_t M, qlora_bf16* dX, qlora_bf16* dA_g, qlora_bf16* dB_g,
                                       qlora_bf16* dA_u, qlora_bf16* dB_u, qlora_bf16* dA_d, qlora_bf16* dB_d,
                                       void* workspace, size_t workspace_bytes, qlora_stream_t stream);
/* qlora_mlp16_bwd with the `early_grads` event of qlora_mlp_bwd_ev. */
QLORA_API qlora_status qlora_mlp16_bwd_ev(qlora_act act, const qlora_lora_linear16* gate,
                                          const qlora_lora_linear16* up, const qlora_lora_linear16* down,
                                          const qlora_bf16* X, const qlora_mlp_saved* saved, const qlora_bf16* dY,
                                          int64_t M, qlora_bf16* dX, qlora_bf16* dA_g, qlora_bf16* dB_g,
                                          qlora_bf16* dA_u, qlora_bf16* dB_u, qlora_bf16* dA_d, qlora_bf16* dB_d,
                                          void* workspace, size_t workspace_bytes, qlora_stream_t stream,
                                          qlora_event_t early_grads);

/* Fused Q/K/V projection (the pages' manual-autograd QKV, with grouped-query
 * K/V widths, e.g. Mistral's 4096 / 1024 / 1024): three NF4 projections q, k,
 * v of one input X [M, k_in] with the same k_in and rank, computed as one GEMM
 * over the three dequantised weights stacked by rows.
 *   XA = X [A_q | A_k | A_v]                        -> XA_saved [M, 3r]
 *   Y  = [Y_q | Y_k | Y_v], Y_p = X dequant(W_p)^T + s_p XA_p B_p
 *                                                   -> Y [M, nq + nk + nv]
 * Backward from dY = [dY_q | dY_k | dY_v] (same layout as Y):
 *   dX = sum_p dY_p dequant(W_p) + s_p (dY_p B_p^T) A_p^T   (one GEMM over the
 *   concatenated reduction, three LoRA steps), dA_p, dB_p as qlora_linear_bwd.
 * Requires nq % 256 == 0 and nk % 256 == 0 (an output tile never spans two
 * projections), k_in % 64 == 0, r in {16, 32, 64}.  Always runs the staged
 * feed (tile configuration 4); the workspace also holds the stacked bf16
 * weight ((nq + nk + nv) * k_in * 2 bytes). */
QLORA_API size_t qlora_qkv_workspace_bytes(int64_t M, int64_t k_in, int64_t nq, int64_t nk, int64_t nv, int32_t r);
QLORA_API qlora_status qlora_qkv_fwd(const qlora_lora_linear* q, const qlora_lora_linear* k,
                                     const qlora_lora_linear* v, const qlora_bf16* X, int64_t M, qlora_bf16* Y,
                                     qlora_bf16* XA_saved, void* workspace, size_t workspace_bytes,
                                     qlora_stream_t stream);
QLORA_API qlora_status qlora_qkv_bwd(const qlora_lora_linear* q, const qlora_lora_linear* k,
                                     const qlora_lora_linear* v, const qlora_bf16* X, const qlora_bf16* XA_saved,
                                     const qlora_bf16* dY, int64_t M, qlora_bf16* dX, qlora_bf16* dA_q,
                                     qlora_bf16* dB_q, qlora_bf16* dA_k, qlora_bf16* dB_k, qlora_bf16* dA_v,
                                     qlora_bf16* dB_v, void* workspace, size_t workspace_bytes, qlora_stream_t stream);

/* RMS layer norm of X [M, d] (the step before the MLP; Mistral blog item
 * "8. 快速 RMS Layernorm", Gemma blog "+1 to RMS LayerNorm"):
 *   rstd = 1 / sqrt(mean_j x_j^2 + eps),  Y = X * rstd * g,
 *   g = w (plus_one = 0: Llama, Mistral) or 1 + w (plus_one = 1: Gemma).
 * Y [M, d] bf16; rstd [M] fp32 is kept for the backward.  Statistics in fp32.
 * Requires d % 8 == 0 and 16-byte aligned pointers. */
QLORA_API qlora_status qlora_rmsnorm_fwd(const qlora_bf16* X, const qlora_bf16* w, int64_t M, int64_t d, float eps,
                                         int32_t plus_one, qlora_bf16* Y, float* rstd, qlora_stream_t stream);
/* Its backward with the norm weight frozen: from dY [M, d] (the gradient of Y),
 *   dX = rstd * (g * dY - n * mean_j(n_j g_j dY_j)),  n = X * rstd. */
QLORA_API qlora_status qlora_rmsnorm_bwd(const qlora_bf16* X, const qlora_bf16* w, const float* rstd,
                                         const qlora_bf16* dY, int64_t M, int64_t d, int32_t plus_one,
                                         qlora_bf16* dX, qlora_stream_t stream);

/* Reads the device status word in `workspace` (synchronising `stream`),
 * clears it, and maps it to a status: QLORA_OK, QLORA_ERR_TIMEOUT or
 * QLORA_ERR_DEVICE. */
QLORA_API qlora_status qlora_last_device_status(void* workspace, qlora_stream_t stream);

/* Test hook for the timeout path (synchronous; not needed in normal use).
 * Arms a one-shot fault: the first CTA of the next skinny pass (the rank-side
 * products X A, dY B^T, ...) leaves one of its tiles unloaded, so that CTA's
 * consumers reach their bounded wait (about 4 s), record QLORA_ERR_TIMEOUT in
 * the status word and return; the kernels after it in the same call see the
 * status and return early too.  Nothing traps or hangs: every wait is bounded
 * and every copy already issued lands before its CTA exits.  The call's
 * results are then meaningless; qlora_last_device_status reports and clears
 * the timeout, and the next call computes normally. */
QLORA_API qlora_status qlora_test_inject_timeout(void);

/* Test hook (not needed in normal use; host side, not thread-safe): caps the
 * number of CTAs of every persistent launch -- the GEMMs (rounded down to
 * whole CTA pairs), the rank-side passes and the weight dequantisation -- at
 * `max_ctas` (0 = no cap, the default; negative values are ignored).  With a
 * small cap every CTA or CTA pair walks many output tiles and work units on
 * small problems, so tests reach the persistent scheduling paths (accumulator
 * ping-pong, ring phases across tiles, tile-group wrap, multi-unit ranges)
 * without full-size inputs.  Results stay within the same tolerance; the
 * rank-side sums may change in their last bits because their split changes.
 * Workspace queries follow the cap current when they are called.  Returns the
 * previous cap. */
QLORA_API int32_t qlora_test_set_grid_cap(int32_t max_ctas);

/* Checked debug build.  lib/libqlora_check.so is the same library compiled
 * with QLORA_CHECK: its kernels check the indices they derive from their
 * arguments (partial-sum slots and groups of the rank-side passes and their
 * reduction, the GEMMs' tile-walk arguments) and, on a failed check, record
 * QL_DEV_BAD_CONFIG in the workspace status word and skip the access instead
 * of touching memory out of range; nothing traps.  qlora_last_device_status
 * then returns QLORA_ERR_DEVICE.  In the normal build the checks compile away.
 * qlora_checked_build returns 1 in the checked build, 0 otherwise. */
QLORA_API int32_t qlora_checked_build(void);

/* Test hook for the checked build (host side, one shot): the next rank-side
 * pass whose plan gives some output group more than one partial slot tells
 * its kernels one slot fewer than planned.  The partial buffer keeps the
 * planned size, so every access stays inside the workspace; the checked build
 * reports the mismatch (QLORA_ERR_DEVICE), the normal build silently computes
 * wrong adapter values for that call. */
QLORA_API qlora_status qlora_test_shrink_next_slot_cap(void);

/* Human-readable name of a status code (static string). */
QLORA_API const char* qlora_status_string(qlora_status status);

/* Selects how the NF4 GEMMs are tiled and fed (all give the same results).
 * Configurations 1-3 dequantise the weight tile by tile in shared memory
 * inside the GEMM mainloop: 1 = one CTA per 128 x 256 tile, 2 = a CTA pair
 * (cta_group::2) per 256 x 256 tile, 3 = a CTA pair per 512 x 128 tile whose
 * dequantised weight tile feeds two M = 256 MMAs.  Configuration 4 = a CTA
 * pair per 256 x 256 tile whose weight is first dequantised once per call
 * into the workspace (the nf4_dequantize kernel) and then streamed by TMA:
 * each weight element is decoded once instead of once per 256-row tile, at
 * the price of that bf16 copy in the workspace.  0 (the default) = automatic:
 * the NF4 gated-MLP calls use configuration 2 for at most 512 tokens (rank
 * 16, d % 256 == 0), where decoding in the mainloop is faster than staging
 * the three weights, and configuration 4 otherwise; the projection and Q/K/V
 * calls use 4.  The workspace size queries follow the configuration current
 * when they are called.  Invalid values are ignored.  Returns the previous
 * value.  Not thread-safe. */
QLORA_API int32_t qlora_set_tile_config(int32_t tiles);
/* The tile configuration (1-4) that qlora_mlp_fwd / qlora_mlp_bwd use for M
 * tokens, width d, MLP width h and rank r under the current setting.  Host
 * only. */
QLORA_API int32_t qlora_mlp_tile_config(int64_t M, int64_t d, int64_t h, int32_t r);

/* Kernel tracing (host side, not thread-safe).  While enabled, every kernel
 * launch of the library is bracketed by CUDA events on its stream. */
typedef struct {
  const char* name; /* static kernel name */
  int64_t launches;
  double total_ms;  /* summed device time between the bracketing events */
} qlora_trace_entry;
QLORA_API qlora_status qlora_trace_begin(void);
/* As qlora_trace_begin, but only launches of the kernel named `kernel_name`
 * (one of the names qlora_trace_end reports, e.g. "gemm_nf4_gateup_glu_fwd")
 * are bracketed; every other launch keeps its programmatic overlap with its
 * neighbours.  QLORA_ERR_INVALID_ARG for an unknown name. */
QLORA_API qlora_status qlora_trace_begin_only(const char* kernel_name);
/* Stops tracing, waits for the recorded events and fills up to `max_entries`
 * per-kernel totals; returns the number of distinct kernels (or -1). */
QLORA_API int32_t qlora_trace_end(qlora_trace_entry* out, int32_t max_entries);
/* Number of kernels this library has launched since it was loaded. */
QLORA_API uint64_t qlora_launch_count(void);

/* Same computation and outputs as qlora_linear_fwd, for callers that cannot
 * allocate device memory and so cannot pass a workspace: for example a plugin
 * that only receives the device pointers of its tensors from a host framework
 * that owns all device memory, or a path where allocating is not permitted.
 * (The pages describe no such call; it has no counterpart there.)
 * Its scratch is a fixed 4 MiB array inside the library that every GPU which
 * loads the library keeps until the process exits.  A call uses at most
 * 256 + 32 M + 4096 ceil(M / 64) bytes of it (each term rounded up to a
 * multiple of 256): the status word, the s-scaled X A and the partial sums of
 * the X A pass.  So M <= 43,648 rows is accepted for any k_in, and larger M
 * returns QLORA_ERR_WORKSPACE_TOO_SMALL before anything is enqueued.  It
 * allocates nothing and frees nothing.
 * The fixed array has no room for a staged weight, so this call always runs a
 * GEMM that dequantises the weight in its mainloop: tile configuration 2 under
 * the automatic setting (the default) or when configuration 4 is selected,
 * else the selected 1-3.  Those
 * take rank-16 adapters only; other ranks return QLORA_ERR_UNSUPPORTED_SHAPE
 * before anything is enqueued.
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it by device ordinal for the life of the
 * process; make that first call before any stream capture.  The cached
 * address does not survive cudaDeviceReset: do not use this call on a device
 * after resetting it.  All calls share the one array: calls whose GPU work
 * overlaps (on different streams, or from different threads) race and must
 * not be issued.  Each call zeroes the status word it uses; device-side
 * timeouts are recorded there and are not reported back through this call. */
QLORA_API qlora_status qlora_linear_fwd_noalloc(const qlora_lora_linear* lin, const qlora_bf16* X, int64_t M,
                                                qlora_bf16* Y, qlora_bf16* XA_saved, qlora_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H_ */
