/*
 * dg_ops.h -- single operations of the canvas denoise step on caller buffers,
 * for kernel-level testing and for callers that compose their own step. Each
 * runs the same kernels dg_denoise_step uses. Page references as in
 * dg_canvas.h ([P1] "DiffusionGemma解析：扩散模型如何让LLM快5倍", [P3]
 * "DiffusionGemma深度拆解：从逐字蹦到整块喷，LLM生成范式的结构性跃迁").
 *
 * All pointers are device memory unless marked host; all matrices row-major;
 * dtype is DG_F32 or DG_BF16 (the storage type of every non-f32 buffer).
 * Each call queues work on `stream` (cudaStream_t, NULL = default), allocates
 * and frees its own temporary buffers (stream-ordered; except
 * dg_lmhead_entropy_noalloc), and returns DG_OK or an error status (see
 * dg_canvas.h); dg_last_error() has the detail. The calls do not synchronize;
 * dg_ops_check reports what went wrong on the device.
 */
#ifndef DG_OPS_H
#define DG_OPS_H

#include <stddef.h>
#include <stdint.h>

#include "dg_canvas.h"

#ifdef __cplusplus
extern "C" {
#endif

/* LM head fused with the per-row softmax entropy and argmax ([P1] 整片并行去噪):
 *   x[r][v] = hs[r] . lm_head[v]          (f32 accumulate)
 *   ent[r]  = H(softmax(x[r] * inv_temp[r])) in nats
 *   argmax[r] = argmax_v x[r][v] (lowest v on ties)
 * hs [M][d], lm_head [V][d] (dtype); inv_temp [M] f32 >= 0 or NULL (= 1; a
 * negative inverse temperature gives an undefined entropy);
 * ent [M] f32, argmax [M] int32 (outputs). The logits are never stored.
 * bf16 needs d % 64 == 0 and V % 256 == 0; f32 any d % 8 == 0. */
dg_status dg_lmhead_entropy(int32_t dtype, const void *hs, const void *lm_head, const float *inv_temp,
                            int32_t M, int32_t d, int32_t V, float *ent, int32_t *argmax, void *stream);

/* The LM head with e4m3 weights (the FP8 deployment of [P3] 性能数据):
 * each row of hs (bf16 [M][d]) is quantized to e4m3 with the smallest
 * power-of-two scale s_r that fits its largest magnitude (round to nearest,
 * ties to even), and
 *   x[r][v] = s_r lm_scale[v] (q_r . q_v)   (f32 accumulate)
 * with lm_head e4m3 byte codes [V][d] and lm_scale [V] f32 row scales
 * (powers of two); then ent and argmax as in dg_lmhead_entropy.
 * Needs d % 128 == 0 and V % 256 == 0. */
dg_status dg_lmhead_entropy_e4m3(const void *hs, const void *lm_head, const float *lm_scale, const float *inv_temp,
                                 int32_t M, int32_t d, int32_t V, float *ent, int32_t *argmax, void *stream);

/* The quantization step of dg_lmhead_entropy_e4m3 alone: each row r of x
 * (bf16 [M][d]) becomes e4m3 codes [M][d] (bytes) and scales[r] (f32, the
 * smallest power of two s with 448 s >= max |x[r]|), codes = x[r] / s
 * rounded to the nearest e4m3 value, ties to even. d % 8 == 0. */
dg_status dg_quantize_rows_e4m3(const void *x, uint8_t *codes, float *scales, int32_t M, int32_t d, void *stream);

/* Allocation-free variant of dg_lmhead_entropy. The pages have no counterpart
 * to this call: it exists for callers of this library that cannot allocate
 * device memory where they run the LM head -- an application whose device
 * memory is reserved up front by its own allocator (a driver allocation in
 * the middle of a step would fail or fragment what is left), or a host that
 * gives a plug-in only the buffers it passes and forbids it to allocate.
 * Same arguments and results as dg_lmhead_entropy (the same kernels with the
 * same vocab partitions, so the same bits). Its temporary per-row partial
 * results go to a fixed device array inside the library (2 MiB, held on
 * every GPU that loads the library until the process exits) instead of a
 * fresh buffer; the call makes no cudaMalloc, cudaFree or other allocation.
 * Limit: M times the number of vocab partitions (at most the GPU's SM count,
 * fewer for M > 256) must not exceed dg_lmhead_entropy_noalloc_max_records()
 * (65,536); larger problems return DG_ERR_UNSUPPORTED before any work.
 * The first call on each device (and CUDA context) looks up the array's
 * device address; make that first call before any stream capture. All calls
 * on a device share the array: two calls whose work can overlap on the GPU
 * (e.g. on different streams without ordering between them) race. Nothing in
 * the array needs to start at zero: each call writes every entry it reads.
 * Device-side failures are reported by dg_ops_check. */
dg_status dg_lmhead_entropy_noalloc(int32_t dtype, const void *hs, const void *lm_head,
                                    const float *inv_temp, int32_t M, int32_t d, int32_t V,
                                    float *ent, int32_t *argmax, void *stream);

/* Capacity of the fixed array used by dg_lmhead_entropy_noalloc, in partial
 * records (one per row and vocab partition). */
size_t dg_lmhead_entropy_noalloc_max_records(void);

/* Bidirectional GQA attention of B*C canvas queries over each request's
 * cached prompt K/V followed by the canvas K/V, no mask, scale 1/sqrt(h),
 * query head q reading KV head q / (Hq/Hk) ([P1] 整片并行去噪 last paragraph;
 * [P3] 架构解剖 2 and diagram).
 *   q [B*C][Hq*h]; kc, vc [B*C][Hk*h]; prefix_len host [B];
 *   prefix_k / prefix_v host arrays of B device pointers, each [S_b][Hk][h];
 *   o [B*C][Hq*h] (output, dtype). bf16 needs h == 128. */
dg_status dg_attention(int32_t dtype, const void *q, const void *kc, const void *vc, int32_t B, int32_t C,
                       int32_t Hq, int32_t Hk, int32_t h, const int32_t *prefix_len,
                       const void *const *prefix_k, const void *const *prefix_v, void *o, void *stream);

/* out[M][N] = a[M][K] . w[N][K]^T (+ residual[M][N] if not NULL), f32
 * accumulate, one rounding to dtype ([P3] 架构解剖 2: the canvas's K/V are
 * re-projected every step). bf16 needs K % 64 == 0 and N % 64 == 0. */
dg_status dg_linear(int32_t dtype, const void *a, const void *w, const void *residual, void *out,
                    int32_t M, int32_t N, int32_t K, void *stream);

/* Device-side status of the calls above: waits for `stream` and reports the
 * first device-side failure any of their kernels recorded since the last
 * dg_ops_check -- DG_ERR_TIMEOUT when a bounded wait inside a kernel gave up
 * (its outputs are then not valid), DG_ERR_DEVICE_CHECK for a failed data
 * check (a NaN entropy) -- and clears it. DG_OK when none failed.
 * Synchronous. The calls above only validate their arguments and queue work;
 * their return status cannot include what happens on the device. */
dg_status dg_ops_check(void* stream);

/* Failure-detection self-test (no counterpart in the pages): one CTA waits on
 * a barrier that nothing completes, through the same bounded wait every kernel
 * of the step uses. The wait gives up after its limit (2 s), records a timeout
 * in a device error word and the kernel returns; the call then returns
 * DG_ERR_TIMEOUT, leaving the CUDA context usable. Synchronous. Anything else
 * (DG_OK included) means the bounded-wait path is broken. */
dg_status dg_selftest_wait_timeout(void *stream);

#ifdef __cplusplus
}
#endif
#endif /* DG_OPS_H */
