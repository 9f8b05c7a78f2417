/*
 * dg_canvas.h -- C ABI of libdgcanvas.so: the per-step denoise of a token
 * canvas (DiffusionGemma-style block diffusion decoding) on one NVIDIA B200.
 *
 * What one denoise step computes, and where the method is described
 * ("DiffusionGemma解析：扩散模型如何让LLM快5倍" = [P1],
 *  "DiffusionGemma深度拆解：从逐字蹦到整块喷，LLM生成范式的结构性跃迁" = [P3],
 *  "谷歌DiffusionGemma：并行生成与自纠的新突破" = [P4]):
 *   1. embed the canvas tokens (a block of up to 256 positions; [P1] 整片并行去噪,
 *      [P3] 架构解剖 diagram, [P4] 工作原理);
 *   2. project Q and the canvas's own K/V, recomputed every step ([P3] 架构解剖 2);
 *   3. bidirectional GQA attention of every canvas query over the cached prompt
 *      K/V prefix plus the canvas K/V, no mask ([P1] 整片并行去噪 last paragraph,
 *      [P3] 架构解剖 2 and diagram);
 *   4. output projection with residual; optionally an MoE FFN with 128 experts,
 *      top-8 routing and one shared expert ([P3] 架构解剖 3);
 *   5. the LM head over the vocabulary fused with a per-position softmax
 *      entropy and argmax; logits are never written to memory ([P1]
 *      整片并行去噪: one distribution per position, lower entropy = more sure);
 *   6. entropy-ordered freezing of the most certain unfrozen positions, each
 *      taking its argmax token ([P1] 整片并行去噪, [P4] 工作原理);
 *   7. re-noising every other unfrozen position with a fresh uniform token id
 *      (unified-state noise, not [MASK]: [P3] 架构解剖 4, [P4] 工作原理), and an
 *      adaptive stop within the step cap ([P1] 自适应停步机制: at most 48 steps).
 *
 * Conventions (apply to every entry point):
 *   - All matrices are row-major; weights are stored [out][in], so both GEMM
 *     operands are contiguous along the contraction dimension.
 *   - "device" pointers are CUDA device memory on the current device; "host"
 *     pointers are ordinary CPU memory. Caller-owned buffers are never freed by
 *     the library. The library owns its workspace and the canvas state and
 *     releases them in dg_canvas_destroy.
 *   - Work is queued on the CUDA stream given to dg_canvas_init (NULL = the
 *     legacy default stream) and is stream-ordered. Calls marked "synchronous"
 *     wait for the stream.
 *   - Errors are reported by status code only; nothing is thrown across the
 *     ABI. Arguments are validated before any launch. Device-side checks
 *     (token id out of range, NaN entropy, a bounded wait that gave up) set an
 *     error word that the next synchronous call reports as
 *     DG_ERR_DEVICE_CHECK / DG_ERR_TIMEOUT; kernels never trap.
 *   - A context must not be used from two host threads at once.
 *   - Shapes supported: canvas_len 1..1024; storage dtype f32 (CUDA-core
 *     kernels, head_dim 32..128 multiple of 32) or bf16 (tensor-core kernels,
 *     head_dim 128, d_model a multiple of 64, vocab a multiple of 256,
 *     n_q_heads a multiple of n_kv_heads).
 */
#ifndef DG_CANVAS_H
#define DG_CANVAS_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DG_ABI_VERSION 2

typedef enum dg_status {
  DG_OK = 0,
  DG_ERR_INVALID_ARG = 1,   /* null pointer, bad size, inconsistent shapes */
  DG_ERR_UNSUPPORTED = 2,   /* valid but outside the supported shapes/dtypes */
  DG_ERR_OOM = 3,           /* workspace allocation failed (or over DG_WORKSPACE_LIMIT_MB) */
  DG_ERR_CUDA = 4,          /* a CUDA runtime call failed; see dg_last_error() */
  DG_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up */
  DG_ERR_DEVICE_CHECK = 6   /* a device-side argument/data check failed */
} dg_status;

typedef enum dg_dtype { DG_F32 = 0, DG_BF16 = 1 } dg_dtype;

/* Weights of the single-layer canvas denoiser. All pointers are device,
 * caller-owned, in the storage dtype `dtype`, and must stay valid until
 * dg_canvas_destroy. */
typedef struct dg_model_desc {
  int32_t d_model, n_q_heads, n_kv_heads, head_dim, vocab, dtype;
  const void *embed;    /* [vocab][d_model]                       */
  const void *wq;       /* [n_q_heads*head_dim][d_model]          */
  const void *wk;       /* [n_kv_heads*head_dim][d_model]         */
  const void *wv;       /* [n_kv_heads*head_dim][d_model]         */
  const void *wo;       /* [d_model][n_q_heads*head_dim]          */
  const void *lm_head;  /* [vocab][d_model]                       */
  /* MoE FFN after attention ([P3] 架构解剖 3); n_experts = 0 disables it.
   * r = Hs W_router^T; p = softmax(r); the top_k experts by p (lower expert id
   * on ties) with gates g = p / sum of the chosen p; for each chosen and each
   * shared expert e: FFN_e(x) = W_down[e] (GELU(W_gate[e] x) * (W_up[e] x))
   * (exact-erf GELU, the product rounded to the storage dtype); Hs becomes
   * Hs + sum g_e FFN_e(Hs) + sum_shared FFN_e(Hs), rounded to the storage
   * dtype. Shared experts are stored after the routed ones. Supported (else
   * DG_ERR_UNSUPPORTED): bf16 only, n_experts a multiple of 32 and <= 256,
   * top_k <= 8, n_shared <= 2, moe_inter a multiple of 64, batch * canvas_len
   * <= 256. */
  int32_t n_experts, top_k, moe_inter, n_shared;
  const void *w_router; /* [n_experts][d_model]                   */
  const void *w_gate;   /* [n_experts+n_shared][moe_inter][d_model] */
  const void *w_up;     /* [n_experts+n_shared][moe_inter][d_model] */
  const void *w_down;   /* [n_experts+n_shared][d_model][moe_inter] */
  /* Storage of lm_head (the FP8 deployment of [P3] 性能数据 and [P4]
   * 引入扩散机制): DG_LM_STORAGE (0) = the storage dtype; DG_LM_E4M3 (1) =
   * e4m3 byte codes [vocab][d_model] with lm_head_scale[v] (device, [vocab]
   * f32, a power of two) the scale of row v. With DG_LM_E4M3 each row r of
   * the residual stream is quantized to e4m3 with the smallest power-of-two
   * scale s_r that fits its largest magnitude (round to nearest, ties to
   * even) and the logits are s_r lm_head_scale[v] (q_r . q_v), f32
   * accumulate. Needs the bf16 dtype and d_model % 128 == 0. */
  int32_t lm_head_format;
  const float *lm_head_scale;
  /* Attention layers ([P3] 局限 2 raises deeper and longer variants): 0 or 1
   * = the single layer above; L > 1 = L layers in sequence, each the single
   * layer (Q/K/V of its input, bidirectional attention over its own prompt
   * K/V and the canvas, Wo + residual) fed the previous layer's output, the
   * LM head reading the last. wq, wk, wv, wo then hold the L layers stacked
   * layer-major ([L][out][in]) and each request's prompt K/V cache is
   * [L][S_b][n_kv_heads][head_dim]. L <= 64; not with the MoE block. */
  int32_t n_layers;
  /* Storage of the expert weights: DG_LM_STORAGE (0) = the storage dtype;
   * DG_LM_E4M3 (1) = w_gate, w_up, w_down hold e4m3 byte codes and
   * w_gate_scale / w_up_scale ([n_experts+n_shared][moe_inter] f32) and
   * w_down_scale ([n_experts+n_shared][d_model] f32) their per-row scales
   * (powers of two). The token rows are then quantized per row (as for the
   * e4m3 LM head) for the gate and up projections, and the GeGLU product,
   * after its rounding to the storage dtype, per row for the down
   * projection; f32 accumulate. Needs d_model % 128 == 0. */
  int32_t expert_format;
  const float *w_gate_scale, *w_up_scale, *w_down_scale;
} dg_model_desc;
#define DG_LM_STORAGE 0
#define DG_LM_E4M3 1

/* Freeze schedule and stop rule ([P1] 整片并行去噪, 自适应停步机制).
 * At step t of a canvas with U unfrozen positions, k = ceil(U / (max_steps - t))
 * positions freeze (all of them when max_steps - t <= 1). With adaptive_stop,
 * the canvas stops once the smallest entropy among positions still unfrozen
 * after freezing is below stop_entropy (nats); the rest then take their argmax. */
typedef struct dg_schedule {
  int32_t max_steps;     /* 1..1024; the pages' cap is 48 */
  float stop_entropy;    /* nats; 0.05 in the reference configuration */
  int32_t adaptive_stop; /* 0 = run every canvas to full freeze */
  int32_t kind;          /* DG_SCHED_CEIL (only value) */
} dg_schedule;
#define DG_SCHED_CEIL 0

/* Optional per-step outputs of dg_denoise_step (each device, may be NULL). */
typedef struct dg_step_out {
  float *ent;           /* [B*C] entropy of softmax(logits * inv_temp), nats   */
  int32_t *argmax;      /* [B*C] argmax of the unscaled logits, lowest id on ties */
  uint8_t *freeze_mask; /* [B*C] 1 where the position froze at this step        */
  void *attn_out;       /* [B*C][n_q_heads*head_dim] attention output O (dtype) */
  void *hidden;         /* [B*C][d_model] residual stream fed to the LM head   */
  void *hidden_attn;    /* [B*C][d_model] residual stream after attention and Wo,
                           before the MoE block (equals `hidden` without MoE)  */
  void *q;              /* [B*C][n_q_heads*head_dim] queries (dtype)           */
  void *k_canvas;       /* [B*C][n_kv_heads*head_dim] canvas keys (dtype)      */
  void *v_canvas;       /* [B*C][n_kv_heads*head_dim] canvas values (dtype)    */
  void *layer_out;      /* [L][B*C][d_model] residual stream after each layer;
                           q, k_canvas, v_canvas, attn_out are the last layer's */
} dg_step_out;

/* Host-side copy of the decode state (all host arrays). */
typedef struct dg_state {
  int32_t *tokens;  /* [B*C] current canvas token ids                      */
  uint8_t *frozen;  /* [B*C] 1 = frozen (never changes again)              */
  int32_t *step;    /* [B]   steps completed by each canvas               */
  uint64_t *seed;   /* [B]   Philox seed of each canvas                   */
  uint8_t *done;    /* [B]   1 = canvas finished (stopped)                */
} dg_state;

typedef struct dg_ctx dg_ctx;

/* Create a decode context and draw the initial canvases.
 *   model       weights (see dg_model_desc); copied by value.
 *   batch       B >= 1 independent canvases (requests).
 *   canvas_len  C, 1..1024 positions per canvas (the pages use 256; longer
 *               canvases are an open question there: [P3] 局限).
 *   prefix_len  host [B]: cached prompt length S_b >= 0 of each request.
 *   prefix_k/v  host arrays of B device pointers, each [S_b][n_kv_heads][head_dim]
 *               in the storage dtype ([L][S_b][...] with n_layers = L > 1; NULL
 *               allowed when S_b = 0).
 *   inv_temp    device [B*C] f32 per-position inverse temperature (>= 0) applied
 *               to the logits before the entropy, or NULL for 1; a negative
 *               value gives an undefined entropy.
 *   seeds       host [B] Philox seeds; canvas b position p starts at
 *               draw(seeds[b], step 0, p, b).
 *   cuda_stream cudaStream_t to queue all work on (NULL = default stream).
 * Allocates the workspace (DG_ERR_OOM on failure). Returns DG_OK and *out. */
dg_status dg_canvas_init(dg_ctx **out, const dg_model_desc *model, int32_t batch,
                         int32_t canvas_len, const int32_t *prefix_len,
                         const void *const *prefix_k, const void *const *prefix_v,
                         const float *inv_temp, const uint64_t *seeds, void *cuda_stream);

/* One denoise step of every canvas that is not done: steps 1-7 above. Canvases
 * that are done are left unchanged. Asynchronous. dbg may be NULL; without it
 * the step runs as one CUDA graph launch (captured on the first call with a
 * given schedule, so that first call must not happen inside a stream capture). */
dg_status dg_denoise_step(dg_ctx *ctx, const dg_schedule *sched, const dg_step_out *dbg);

/* Start a new block: redraw every canvas at step 0 from `seeds` (host [B]; NULL
 * keeps the current seeds), clear the frozen and done flags. Asynchronous. */
dg_status dg_canvas_reset(dg_ctx *ctx, const uint64_t *seeds);

/* Start a new block with some positions given in advance: infilling between a
 * given prefix and suffix, or a puzzle's given cells ([P3] 为什么值得重视 2:
 * fill-in-the-middle, constraints propagating from every direction; [P4]
 * 工作原理: constrained generation). As dg_canvas_reset, then every position
 * with fixed_mask[i] != 0 takes fixed_tokens[i] and starts frozen: it keeps
 * its token, keeps contributing K/V, and the freeze schedule counts only the
 * open positions (k_t = ceil(U_t / (T - t)) over the unfrozen ones).
 *   seeds         host [B] or NULL (keep the current seeds).
 *   fixed_mask    host [B*C] uint8 (canvas-major), nonzero = given.
 *   fixed_tokens  host [B*C] int32; read only where fixed_mask is set, each
 *                 in [0, vocab) (else DG_ERR_INVALID_ARG before any work).
 * Synchronous. A canvas whose positions are all given stops after one step. */
dg_status dg_canvas_reset_fixed(dg_ctx *ctx, const uint64_t *seeds, const uint8_t *fixed_mask,
                                const int32_t *fixed_tokens);

/* Block-autoregressive decoding: after a canvas is committed, its tokens'
 * K/V join the request's cached prompt and the next canvas attends to both
 * ([P3] 架构解剖 1: blocks in sequence, parallel within a block; the committed
 * block's K/V come from the causal encoder pass). With one layer and no
 * positional encoding a token's K/V depend only on its embedding, so the
 * encoder pass is the K/V projection of the committed tokens.
 *
 * dg_canvas_block_kv writes the K/V of the current canvas tokens:
 *   k_out, v_out  device [B*C][n_kv_heads*head_dim] in the storage dtype,
 *                 canvas-major (rows b*C .. b*C+C-1 belong to request b), the
 *                 same per-token layout as the prompt cache, so appending a
 *                 request's rows to its cache is a plain copy.
 * Asynchronous; overwrites the context's step scratch (call between steps). */
dg_status dg_canvas_block_kv(dg_ctx *ctx, void *k_out, void *v_out);

/* Point the context at new prompt K/V caches (e.g. the old prefix followed by
 * a committed block): arguments as in dg_canvas_init (host [B] lengths,
 * host arrays of device pointers, 16-byte aligned, caller-owned). Waits for the
 * queued work; the next step re-captures its graph. The canvas state is not
 * touched (use dg_canvas_reset to start the next block). */
dg_status dg_canvas_set_prefix(dg_ctx *ctx, const int32_t *prefix_len, const void *const *prefix_k,
                               const void *const *prefix_v);

/* Denoise until every canvas is done (at most sched->max_steps steps each).
 *   tokens_out  [B*C] int32, device or host memory (copied with UVA), or NULL.
 *   steps_out   host [B] steps taken per canvas, or NULL.
 * Synchronous. The loop runs on the device: one CUDA graph launch, whose
 * conditional while node repeats the step until the step's selection kernel
 * finds every canvas done (no step runs after that); the host waits once.
 * The first call with a given schedule builds that graph, so it must not
 * happen inside a stream capture. A canvas still open after max_steps steps
 * (impossible under DG_SCHED_CEIL) ends the loop with DG_ERR_DEVICE_CHECK. */
dg_status dg_decode_block(dg_ctx *ctx, const dg_schedule *sched, int32_t *tokens_out,
                          int32_t *steps_out);

/* Copy the decode state to / from host arrays (synchronous). set_state
 * validates token ids (< vocab) and steps (>= 0). Together with the counter-based
 * RNG this resumes a decode bit-exactly at any step. */
dg_status dg_canvas_get_state(dg_ctx *ctx, dg_state *host_out);
dg_status dg_canvas_set_state(dg_ctx *ctx, const dg_state *host_in);

/* Timing support: with n > 0 pairs of CUDA events (cudaEvent_t, created by the
 * caller with timing enabled), step number i (counted from this call) of
 * dg_denoise_step without debug outputs records starts[i % n] just before and
 * stops[i % n] just after the kernel named by `kernel`: DG_KERNEL_LMHEAD (the
 * LM head with its entropy/argmax epilogue) or DG_KERNEL_ATTENTION (the
 * attention kernel, with its merge kernel when CTAs share units). n = 0 turns it
 * off for that kernel; the settings are independent. DG_KERNEL_DECODE takes
 * one pair (n <= 1), recorded by dg_decode_block's graph just before its loop
 * starts and just after it ends (the device time of the loop alone); the
 * kernel pairs are not recorded inside that loop.
 * Synchronous (drops the captured graphs). */
#define DG_KERNEL_LMHEAD 0
#define DG_KERNEL_ATTENTION 1
#define DG_KERNEL_DECODE 2
dg_status dg_canvas_set_kernel_timing(dg_ctx *ctx, int32_t kernel, int32_t n, void *const *starts,
                                      void *const *stops);
/* dg_canvas_set_kernel_timing(ctx, DG_KERNEL_LMHEAD, n, starts, stops). */
dg_status dg_canvas_set_timing_events(dg_ctx *ctx, int32_t n, void *const *starts, void *const *stops);

/* Steps run by the device-side loop of the most recent dg_decode_block (0
 * before the first), into host *steps_out. Synchronous. */
dg_status dg_canvas_loop_steps(dg_ctx *ctx, int32_t *steps_out);

/* Wait for the context's stream and report device-side errors (synchronous). */
dg_status dg_canvas_sync(dg_ctx *ctx);

/* Release the workspace and the context (synchronous). NULL is a no-op. */
void dg_canvas_destroy(dg_ctx *ctx);

/* Static description of a status code. */
const char *dg_status_string(dg_status s);

/* Last error message of the calling thread (empty string if none). */
const char *dg_last_error(void);

/* ABI version of the loaded library (DG_ABI_VERSION). */
int32_t dg_abi_version(void);

/* Number of GPU kernel launches queued by the most recent dg_denoise_step
 * (for launch accounting). */
int32_t dg_launches_per_step(const dg_ctx *ctx);

#ifdef __cplusplus
}
#endif
#endif /* DG_CANVAS_H */
