// Single-operation entry points (include/dg_ops.h): the step's kernels on
// caller buffers, each with its own stream-ordered temporaries.
#include <string>
#include <vector>

#include "dg_internal.cuh"
#include "dg_ops.h"

using dg::set_last_error;

namespace {

#define OP_ARG(cond, msg)                                          \
  do {                                                             \
    if (!(cond)) {                                                 \
      set_last_error(std::string("invalid argument: ") + (msg));   \
      return DG_ERR_INVALID_ARG;                                   \
    }                                                              \
  } while (0)
#define OP_UNSUP(cond, msg)                                        \
  do {                                                             \
    if (!(cond)) {                                                 \
      set_last_error(std::string("unsupported: ") + (msg));        \
      return DG_ERR_UNSUPPORTED;                                   \
    }                                                              \
  } while (0)

dg_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return DG_OK;
  set_last_error(std::string(what) + ": " + cudaGetErrorString(e));
  return e == cudaErrorMemoryAllocation ? DG_ERR_OOM : DG_ERR_CUDA;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device error word of these entry points: their kernels record the first
// device-side failure here (a bounded wait that gave up, a NaN entropy) and
// dg_ops_check reads and clears it.
static __device__ int g_ops_err;
dg::SymbolAddressCache g_ops_err_addr;

dg_status make_exec(void* stream, dg::Exec* ex) {
  ex->stream = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&ex->sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    set_last_error("no usable CUDA device");
    return DG_ERR_CUDA;
  }
  return dg::ops_error_word(&ex->err);
}

}  // namespace

namespace dg {
dg_status ops_error_word(int** out) {
  void* p = nullptr;
  const dg_status st = g_ops_err_addr.get(g_ops_err, &p);
  *out = static_cast<int*>(p);
  return st;
}
}  // namespace dg

extern "C" {

dg_status dg_lmhead_entropy(int32_t dtype, const void* hs, const void* lm_head, const float* inv_temp, int32_t M,
                            int32_t d, int32_t V, float* ent, int32_t* argmax, void* stream) {
  OP_ARG(dtype == DG_F32 || dtype == DG_BF16, "dtype");
  OP_ARG(hs && lm_head && ent && argmax, "NULL buffer");
  OP_ARG(M >= 1 && d >= 1 && V >= 2, "sizes");
  OP_ARG(al16(hs) && al16(lm_head), "hs / lm_head must be 16-byte aligned");
  OP_UNSUP(d % 8 == 0, "d % 8 != 0");
  if (dtype == DG_BF16) OP_UNSUP(d % 64 == 0 && V % 256 == 0, "bf16 needs d % 64 == 0 and V % 256 == 0");
  dg::Exec ex;
  if (dg_status est = make_exec(stream, &ex)) return est;
  dg::LmPartials part;
  part.P = dtype == DG_BF16 ? dg::lmhead_tc_partitions(M, V, ex.sm_count) : std::max(1, std::min(128, V / 1024));
  part.rec = nullptr;
  dg_status st = cuda_status(cudaMallocAsync((void**)&part.rec, sizeof(dg::LmRec) * (size_t)M * part.P, ex.stream),
                             "cudaMallocAsync");
  if (st != DG_OK) return st;
  if (dtype == DG_BF16) {
    CUtensorMap a, b;
    if (!dg::lmhead_tc_prepare(hs, lm_head, M, d, V, &a, &b)) {
      cudaFreeAsync(part.rec, ex.stream);
      return DG_ERR_CUDA;
    }
    dg::launch_lmhead_tc(ex, a, b, part, inv_temp, M, d, V);
  } else {
    dg::launch_lmhead_simple(ex, dtype, hs, lm_head, inv_temp, part, M, d, V);
  }
  dg::launch_merge_select(ex, part, ent, argmax, nullptr, nullptr, nullptr, 1, M, V);
  st = cuda_status(cudaGetLastError(), "launch");
  cudaFreeAsync(part.rec, ex.stream);
  return st;
}

dg_status dg_lmhead_entropy_e4m3(const void* hs, const void* lm_head, const float* lm_scale, const float* inv_temp,
                                 int32_t M, int32_t d, int32_t V, float* ent, int32_t* argmax, void* stream) {
  OP_ARG(hs && lm_head && lm_scale && ent && argmax, "NULL buffer");
  OP_ARG(M >= 1 && d >= 1 && V >= 2, "sizes");
  OP_ARG(al16(hs) && al16(lm_head), "hs / lm_head must be 16-byte aligned");
  OP_UNSUP(d % 128 == 0 && V % 256 == 0, "the e4m3 LM head needs d % 128 == 0 and V % 256 == 0");
  dg::Exec ex;
  if (dg_status est = make_exec(stream, &ex)) return est;
  dg::LmPartials part;
  part.P = dg::lmhead_tc_partitions(M, V, ex.sm_count);
  uint8_t* q = nullptr;
  float* sa = nullptr;
  dg_status st = cuda_status(cudaMallocAsync((void**)&part.rec, sizeof(dg::LmRec) * (size_t)M * part.P, ex.stream),
                             "cudaMallocAsync");
  if (st == DG_OK) st = cuda_status(cudaMallocAsync((void**)&q, (size_t)M * d, ex.stream), "cudaMallocAsync");
  if (st == DG_OK) st = cuda_status(cudaMallocAsync((void**)&sa, sizeof(float) * M, ex.stream), "cudaMallocAsync");
  CUtensorMap a, b;
  if (st == DG_OK && !dg::lmhead_tc_prepare(q, lm_head, M, d, V, &a, &b, true)) st = DG_ERR_CUDA;
  if (st == DG_OK) {
    dg::launch_quantize_rows_e4m3(ex, hs, q, sa, M, d);
    dg::launch_lmhead_tc(ex, a, b, part, inv_temp, M, d, V, sa, lm_scale);
    dg::launch_merge_select(ex, part, ent, argmax, nullptr, nullptr, nullptr, 1, M, V);
    st = cuda_status(cudaGetLastError(), "launch");
  }
  if (sa) cudaFreeAsync(sa, ex.stream);
  if (q) cudaFreeAsync(q, ex.stream);
  if (part.rec) cudaFreeAsync(part.rec, ex.stream);
  return st;
}

dg_status dg_quantize_rows_e4m3(const void* x, uint8_t* codes, float* scales, int32_t M, int32_t d, void* stream) {
  OP_ARG(x && codes && scales, "NULL buffer");
  OP_ARG(M >= 1 && d >= 1, "sizes");
  OP_ARG(al16(x) && (reinterpret_cast<uintptr_t>(codes) & 7u) == 0, "x must be 16-byte and codes 8-byte aligned");
  OP_UNSUP(d % 8 == 0, "d % 8 != 0");
  dg::Exec ex;
  if (dg_status est = make_exec(stream, &ex)) return est;
  dg::launch_quantize_rows_e4m3(ex, x, codes, scales, M, d);
  return cuda_status(cudaGetLastError(), "launch");
}

dg_status dg_attention(int32_t dtype, const void* q, const void* kc, const void* vc, int32_t B, int32_t C,
                       int32_t Hq, int32_t Hk, int32_t h, const int32_t* prefix_len, const void* const* prefix_k,
                       const void* const* prefix_v, void* o, void* stream) {
  OP_ARG(dtype == DG_F32 || dtype == DG_BF16, "dtype");
  OP_ARG(q && kc && vc && o && prefix_len, "NULL buffer");
  OP_ARG(B >= 1 && C >= 1 && Hq >= 1 && Hk >= 1 && Hq % Hk == 0, "sizes");
  if (dtype == DG_BF16) OP_UNSUP(h == 128, "bf16 needs h == 128");
  else OP_UNSUP(h % 32 == 0 && h <= 128, "f32 needs h in {32, 64, 96, 128}");
  std::vector<dg::PrefixDesc> pd(B);
  for (int b = 0; b < B; ++b) {
    OP_ARG(prefix_len[b] >= 0, "negative prefix length");
    if (prefix_len[b] > 0) OP_ARG(prefix_k && prefix_v && prefix_k[b] && prefix_v[b], "NULL prefix pointer");
    pd[b] = {prefix_len[b] ? prefix_k[b] : nullptr, prefix_len[b] ? prefix_v[b] : nullptr, prefix_len[b], 0};
  }
  dg::Exec ex;
  if (dg_status est = make_exec(stream, &ex)) return est;
  if (dtype == DG_BF16) {
    OP_ARG(al16(q) && al16(kc) && al16(vc) && al16(o), "buffers must be 16-byte aligned");
    dg::AttnShape sh{B, C, Hq, Hk, h};
    const int slots = dg::attn_tc_slots(B, C, Hq, Hk, prefix_len, ex.sm_count);
    float* part = nullptr;
    const size_t rows = (size_t)B * C * Hq;
    if (slots > 1) {
      dg_status st = cuda_status(cudaMallocAsync((void**)&part, slots * rows * 130 * sizeof(float), ex.stream),
                                 "cudaMallocAsync");
      if (st != DG_OK) return st;
    }
    dg::AttnTc at;
    dg_status st = DG_OK;
    if (!dg::attn_tc_prepare(&at, sh, q, kc, vc, prefix_len, prefix_k, prefix_v, o, part,
                             part ? part + slots * rows * 128 : nullptr, slots, ex.sm_count))
      st = DG_ERR_CUDA;
    else {
      dg::launch_attn_tc(ex, at);
      st = cuda_status(cudaGetLastError(), "launch");
    }
    if (part) cudaFreeAsync(part, ex.stream);
    return st;
  }
  dg::PrefixDesc* dpd = nullptr;
  dg_status st = cuda_status(cudaMallocAsync((void**)&dpd, sizeof(dg::PrefixDesc) * B, ex.stream), "cudaMallocAsync");
  if (st != DG_OK) return st;
  st = cuda_status(cudaMemcpyAsync(dpd, pd.data(), sizeof(dg::PrefixDesc) * B, cudaMemcpyHostToDevice, ex.stream),
                   "cudaMemcpyAsync");
  if (st == DG_OK) {
    dg::AttnShape sh{B, C, Hq, Hk, h};
    dg::launch_attention_simple(ex, dtype, q, dpd, kc, vc, o, sh);
    st = cuda_status(cudaGetLastError(), "launch");
  }
  cudaFreeAsync(dpd, ex.stream);
  return st;
}

dg_status dg_ops_check(void* stream) {
  int* words[2] = {nullptr, nullptr};
  dg_status st = dg::ops_error_word(&words[0]);
  if (st == DG_OK) st = dg::noalloc_error_word(&words[1]);
  if (st != DG_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int h[2] = {0, 0};
  for (int i = 0; i < 2; ++i) {
    st = cuda_status(cudaMemcpyAsync(&h[i], words[i], sizeof(int), cudaMemcpyDeviceToHost, s), "cudaMemcpyAsync");
    if (st == DG_OK) st = cuda_status(cudaMemsetAsync(words[i], 0, sizeof(int), s), "cudaMemsetAsync");
    if (st != DG_OK) return st;
  }
  st = cuda_status(cudaStreamSynchronize(s), "cudaStreamSynchronize");
  if (st != DG_OK) return st;
  const int code = h[0] ? h[0] : h[1];
  if (code == 0) return DG_OK;
  set_last_error("device-side check failed in a single-operation call (code " + std::to_string(code) + ")");
  return code == dg::kDevWaitTimeout ? DG_ERR_TIMEOUT : DG_ERR_DEVICE_CHECK;
}

dg_status dg_linear(int32_t dtype, const void* a, const void* w, const void* residual, void* out, int32_t M,
                    int32_t N, int32_t K, void* stream) {
  OP_ARG(dtype == DG_F32 || dtype == DG_BF16, "dtype");
  OP_ARG(a && w && out, "NULL buffer");
  OP_ARG(M >= 1 && N >= 1 && K >= 1, "sizes");
  dg::Exec ex;
  if (dg_status est = make_exec(stream, &ex)) return est;
  if (dtype == DG_BF16) {
    OP_UNSUP(K % 64 == 0 && N % 64 == 0, "bf16 needs K % 64 == 0 and N % 64 == 0");
    OP_ARG(al16(a) && al16(w) && al16(out) && (!residual || al16(residual)), "buffers must be 16-byte aligned");
    dg::GemmTc g;
    const void* ws[1] = {w};
    void* os[1] = {out};
    const int ns[1] = {N};
    if (!dg::gemm_tc_prepare(&g, a, M, K, 1, ws, os, ns, ex.sm_count)) return DG_ERR_CUDA;
    void* tmp = nullptr;
    const size_t pf = dg::gemm_tc_partial_floats(g);
    if (g.splits > 1) {
      dg_status st = cuda_status(cudaMallocAsync(&tmp, pf * sizeof(float), ex.stream), "cudaMallocAsync");
      if (st != DG_OK) return st;
      g.part = static_cast<float*>(tmp);
    }
    dg::launch_gemm_tc(ex, g, residual);
    if (tmp) cudaFreeAsync(tmp, ex.stream);
  } else {
    dg::launch_linear_simple(ex, dtype, a, w, residual, out, M, N, K);
  }
  return cuda_status(cudaGetLastError(), "launch");
}

}  // extern "C"
