// C ABI of libdgcanvas: argument validation, workspace, the per-step launch
// sequence, the device-side decode loop and state transfer. The operations
// themselves are described in include/dg_canvas.h.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include "dg_internal.cuh"

namespace dg {

static thread_local std::string g_last_error;
void set_last_error(const std::string& msg) { g_last_error = msg; }

}  // namespace dg

using dg::set_last_error;

#define DG_CUDA_RET(expr)                                                              \
  do {                                                                                 \
    cudaError_t e__ = (expr);                                                          \
    if (e__ != cudaSuccess) {                                                          \
      set_last_error(std::string(#expr) + ": " + cudaGetErrorString(e__));             \
      return DG_ERR_CUDA;                                                              \
    }                                                                                  \
  } while (0)

#define DG_ARG(cond, msg)                          \
  do {                                             \
    if (!(cond)) {                                 \
      set_last_error(std::string("invalid argument: ") + (msg)); \
      return DG_ERR_INVALID_ARG;                   \
    }                                              \
  } while (0)

#define DG_UNSUP(cond, msg)                        \
  do {                                             \
    if (!(cond)) {                                 \
      set_last_error(std::string("unsupported: ") + (msg)); \
      return DG_ERR_UNSUPPORTED;                   \
    }                                              \
  } while (0)

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Bump allocator over one cudaMalloc'd block; every buffer 256-byte aligned.
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <typename T> T* take(size_t count) {
    off = (off + 255) & ~size_t(255);
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off += count * sizeof(T);
    return p;
  }
};

void layout_workspace(dg_ctx* c, void* base, size_t* total) {
  Carver w(base);
  const size_t M = c->M, d = c->m.d_model;
  const size_t qd = (size_t)c->m.n_q_heads * c->m.head_dim, kd = (size_t)c->m.n_kv_heads * c->m.head_dim;
  c->cs.tok = w.take<int32_t>(M);
  c->cs.frozen = w.take<uint8_t>(M);
  c->cs.step = w.take<int32_t>(c->B);
  c->cs.seed = w.take<uint64_t>(c->B);
  c->cs.done = w.take<uint8_t>(c->B);
  c->cs.all_done = w.take<int32_t>(1);
  c->cs.counters = w.take<uint32_t>(c->B + 1);
  c->cs.loop_iter = w.take<int32_t>(1);
  c->err = w.take<int32_t>(1);
  c->d_prefix = w.take<dg::PrefixDesc>((size_t)c->L * c->B);  // [L][B]
  c->xres.assign(c->L + 1, nullptr);
  for (int l = 0; l <= c->L; ++l) c->xres[l] = w.take<char>(M * d * c->es);
  c->X = c->xres[0];
  c->Q = w.take<char>(M * qd * c->es);
  c->Kc = w.take<char>(M * kd * c->es);
  c->Vc = w.take<char>(M * kd * c->es);
  c->O = w.take<char>(M * qd * c->es);
  c->Hs = c->xres[c->L];
  c->Hs2 = c->m.n_experts ? w.take<char>(M * d * c->es) : nullptr;
  c->lm.rec = w.take<dg::LmRec>(M * (size_t)c->lm.P);
  if (c->m.lm_head_format == DG_LM_E4M3) {
    c->hs8 = w.take<uint8_t>(M * d);
    c->hs8_scale = w.take<float>(M);
  }
  c->ent = w.take<float>(M);
  c->am = w.take<int32_t>(M);
  if (c->m.n_experts) {
    dg::MoeShape ms{c->M, c->m.d_model, c->m.n_experts, c->m.top_k, c->m.n_shared, c->m.moe_inter,
                    c->m.expert_format == DG_LM_E4M3};
    c->moe_ws = w.take<char>(dg::moe_workspace_bytes(ms));
  }
  if (c->m.dtype == DG_BF16) {  // split-K partials, shared by the layers (same shapes)
    float* pq = w.take<float>(dg::gemm_tc_partial_floats(c->g_qkv[0]));
    float* po = w.take<float>(dg::gemm_tc_partial_floats(c->g_wo[0]));
    for (int l = 0; l < c->L; ++l) {
      c->g_qkv[l].part = pq;
      c->g_wo[l].part = po;
    }
  }
  if (c->m.dtype == DG_BF16 && c->attn_slots > 1) {
    const size_t rows = M * (size_t)c->m.n_q_heads;
    c->attn_part_o = w.take<float>((size_t)c->attn_slots * rows * 128);
    c->attn_part_ml = w.take<float>((size_t)c->attn_slots * rows * 2);
  }
  *total = w.off + 256;
}

dg_status validate_model(const dg_model_desc* m) {
  DG_ARG(m != nullptr, "model is NULL");
  DG_ARG(m->dtype == DG_F32 || m->dtype == DG_BF16, "dtype must be DG_F32 or DG_BF16");
  DG_ARG(m->d_model > 0 && m->n_q_heads > 0 && m->n_kv_heads > 0 && m->head_dim > 0 && m->vocab > 1,
         "dimensions must be positive (vocab >= 2)");
  DG_ARG(m->n_q_heads % m->n_kv_heads == 0, "n_q_heads must be a multiple of n_kv_heads");
  DG_ARG(m->embed && m->wq && m->wk && m->wv && m->wo && m->lm_head, "a weight pointer is NULL");
  DG_ARG(aligned16(m->embed) && aligned16(m->wq) && aligned16(m->wk) && aligned16(m->wv) &&
             aligned16(m->wo) && aligned16(m->lm_head),
         "weight pointers must be 16-byte aligned");
  DG_UNSUP(m->d_model % 8 == 0, "d_model must be a multiple of 8");
  if (m->dtype == DG_F32) {
    DG_UNSUP(m->head_dim % 32 == 0 && m->head_dim <= 128, "f32 head_dim must be 32, 64, 96 or 128");
  } else {
    DG_UNSUP(m->head_dim == 128, "bf16 head_dim must be 128");
    DG_UNSUP(m->d_model % 64 == 0, "bf16 d_model must be a multiple of 64");
    DG_UNSUP(m->vocab % 256 == 0, "bf16 vocab must be a multiple of 256");
  }
  DG_ARG(m->lm_head_format == DG_LM_STORAGE || m->lm_head_format == DG_LM_E4M3, "unknown lm_head_format");
  DG_ARG(m->n_layers >= 0 && m->n_layers <= 64, "n_layers must be in [0, 64]");
  if (m->n_layers > 1) DG_UNSUP(m->n_experts == 0, "the MoE block needs the single-layer model");
  if (m->lm_head_format == DG_LM_E4M3) {
    DG_ARG(m->lm_head_scale != nullptr, "lm_head_scale is NULL");
    DG_UNSUP(m->dtype == DG_BF16 && m->d_model % 128 == 0, "an e4m3 LM head needs bf16 and d_model % 128 == 0");
  }
  DG_ARG(m->expert_format == DG_LM_STORAGE || m->expert_format == DG_LM_E4M3, "unknown expert_format");
  if (m->expert_format == DG_LM_E4M3)
    DG_ARG(m->n_experts > 0 && m->w_gate_scale && m->w_up_scale && m->w_down_scale,
           "e4m3 experts need n_experts > 0 and the three row-scale arrays");
  if (m->n_experts != 0) {
    DG_ARG(m->n_experts > 0 && m->top_k > 0 && m->top_k <= m->n_experts && m->moe_inter > 0 &&
               m->n_shared >= 0,
           "MoE sizes");
    DG_ARG(m->w_router && m->w_gate && m->w_up && m->w_down, "an MoE weight pointer is NULL");
    DG_UNSUP(m->dtype == DG_BF16, "the MoE FFN needs the bf16 storage dtype");
    DG_UNSUP(m->n_experts <= 256 && m->n_experts % 32 == 0 && m->top_k <= 8 && m->n_shared <= 2 &&
                 m->moe_inter % 64 == 0,
             "MoE needs n_experts <= 256 and a multiple of 32, top_k <= 8, n_shared <= 2, moe_inter % 64 == 0");
  }
  return DG_OK;
}

dg_status validate_sched(const dg_schedule* s) {
  DG_ARG(s != nullptr, "schedule is NULL");
  DG_ARG(s->max_steps >= 1 && s->max_steps <= 1024, "max_steps must be in [1, 1024]");
  DG_ARG(s->kind == DG_SCHED_CEIL, "unknown schedule kind");
  DG_ARG(s->stop_entropy == s->stop_entropy, "stop_entropy is NaN");
  return DG_OK;
}

dg_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error(std::string(what) + ": " + cudaGetErrorString(e));
    return DG_ERR_CUDA;
  }
  return DG_OK;
}

// Layer l's slice of a stacked weight of `count` elements per layer.
const void* layer_w(const dg_ctx* c, const void* base, int l, size_t count) {
  return static_cast<const char*>(base) + (size_t)l * count * c->es;
}

// Request b's prompt K (or V) cache of layer l: [L][S_b][Hk][h] per request.
const void* layer_prefix(const dg_ctx* c, const void* base, int b, int l) {
  if (!base) return nullptr;
  return static_cast<const char*>(base) + (size_t)l * c->S[b] * c->m.n_kv_heads * c->m.head_dim * c->es;
}

// Binds each layer's projection GEMMs (bf16) to the context's buffers and
// that layer's weights: Q/K/V from xres[l], Wo + residual into xres[l + 1].
bool prepare_layer_gemms(dg_ctx* c) {
  const int d = c->m.d_model, qd = c->m.n_q_heads * c->m.head_dim, kd = c->m.n_kv_heads * c->m.head_dim;
  for (int l = 0; l < c->L; ++l) {
    const void* wqkv[3] = {layer_w(c, c->m.wq, l, (size_t)qd * d), layer_w(c, c->m.wk, l, (size_t)kd * d),
                           layer_w(c, c->m.wv, l, (size_t)kd * d)};
    void* oqkv[3] = {c->Q, c->Kc, c->Vc};
    const int nqkv[3] = {qd, kd, kd};
    const void* wo[1] = {layer_w(c, c->m.wo, l, (size_t)d * qd)};
    void* oo[1] = {c->xres[l + 1]};
    const int no[1] = {d};
    float *pq = c->g_qkv[l].part, *po = c->g_wo[l].part;  // keep the bound partial buffers
    if (!dg::gemm_tc_prepare(&c->g_qkv[l], c->xres[l], c->M, d, 3, wqkv, oqkv, nqkv, c->ex.sm_count) ||
        !dg::gemm_tc_prepare(&c->g_wo[l], c->O, c->M, qd, 1, wo, oo, no, c->ex.sm_count))
      return false;
    c->g_qkv[l].part = pq;
    c->g_wo[l].part = po;
  }
  return true;
}

// Each layer's attention (bf16) over that layer's prompt caches; the device
// prompt descriptors [L][B] for the f32 path.
dg_status prepare_layer_attention(dg_ctx* c) {
  std::vector<dg::PrefixDesc> pd((size_t)c->L * c->B);
  for (int l = 0; l < c->L; ++l) {
    std::vector<const void*> pk(c->B), pv(c->B);
    for (int b = 0; b < c->B; ++b) {
      pk[b] = layer_prefix(c, c->pk[b], b, l);
      pv[b] = layer_prefix(c, c->pv[b], b, l);
      pd[(size_t)l * c->B + b] = {pk[b], pv[b], c->S[b], 0};
    }
    if (c->m.dtype == DG_BF16) {
      dg::AttnShape sh{c->B, c->C, c->m.n_q_heads, c->m.n_kv_heads, c->m.head_dim};
      if (!dg::attn_tc_prepare(&c->attn[l], sh, c->Q, c->Kc, c->Vc, c->S.data(), pk.data(), pv.data(), c->O,
                               c->attn_part_o, c->attn_part_ml, c->attn_slots, c->ex.sm_count))
        return DG_ERR_CUDA;
    }
  }
  DG_CUDA_RET(cudaMemcpyAsync(c->d_prefix, pd.data(), pd.size() * sizeof(dg::PrefixDesc), cudaMemcpyHostToDevice,
                              c->ex.stream));
  return DG_OK;
}

// The launch sequence of one denoise step (steps 1-7 of the header).
dg_status enqueue_step(dg_ctx* c, const dg_schedule& s, const dg_step_out* dbg) {
  const int M = c->M, d = c->m.d_model, V = c->m.vocab;
  const int qd = c->m.n_q_heads * c->m.head_dim, kd = c->m.n_kv_heads * c->m.head_dim;
  const int dt = c->m.dtype;
  dg::Exec& ex = c->ex;
  ex.launches = 0;
  dg::launch_embed(ex, dt, c->m.embed, c->cs.tok, c->X, M, d, V);
  dg::AttnShape sh{c->B, c->C, c->m.n_q_heads, c->m.n_kv_heads, c->m.head_dim};
  for (int l = 0; l < c->L; ++l) {  // layer l: xres[l] -> xres[l + 1]
    if (dt == DG_BF16) {
      dg::launch_gemm_tc(ex, c->g_qkv[l], nullptr);
    } else {
      dg::launch_linear_simple(ex, dt, c->xres[l], layer_w(c, c->m.wq, l, (size_t)qd * d), nullptr, c->Q, M, qd, d);
      dg::launch_linear_simple(ex, dt, c->xres[l], layer_w(c, c->m.wk, l, (size_t)kd * d), nullptr, c->Kc, M, kd, d);
      dg::launch_linear_simple(ex, dt, c->xres[l], layer_w(c, c->m.wv, l, (size_t)kd * d), nullptr, c->Vc, M, kd, d);
    }
    // inside a stream capture, only an "external" record becomes an event node
    // (timed: the last layer's attention)
    const bool timed = l == c->L - 1;
    if (timed && c->cur_ev_start[DG_KERNEL_ATTENTION])
      DG_CUDA_RET(cudaEventRecordWithFlags(c->cur_ev_start[DG_KERNEL_ATTENTION], ex.stream, cudaEventRecordExternal));
    if (dt == DG_BF16)
      dg::launch_attn_tc(ex, c->attn[l]);
    else
      dg::launch_attention_simple(ex, dt, c->Q, c->d_prefix + (size_t)l * c->B, c->Kc, c->Vc, c->O, sh);
    if (timed && c->cur_ev_stop[DG_KERNEL_ATTENTION])
      DG_CUDA_RET(cudaEventRecordWithFlags(c->cur_ev_stop[DG_KERNEL_ATTENTION], ex.stream, cudaEventRecordExternal));
    if (dt == DG_BF16)
      dg::launch_gemm_tc(ex, c->g_wo[l], c->xres[l]);
    else
      dg::launch_linear_simple(ex, dt, c->O, layer_w(c, c->m.wo, l, (size_t)d * qd), c->xres[l], c->xres[l + 1],
                               M, d, qd);
  }
  const void* hs = c->Hs;
  if (c->m.n_experts) {
    dg::launch_moe(ex, c->moe);
    hs = c->Hs2;
  }
  // e4m3 LM head: the residual stream is quantized first (outside the LM-head timing)
  const bool fp8 = c->m.lm_head_format == DG_LM_E4M3;
  if (fp8) dg::launch_quantize_rows_e4m3(ex, hs, c->hs8, c->hs8_scale, M, d);
  if (c->cur_ev_start[DG_KERNEL_LMHEAD])
    DG_CUDA_RET(cudaEventRecordWithFlags(c->cur_ev_start[DG_KERNEL_LMHEAD], ex.stream, cudaEventRecordExternal));
  if (fp8)
    dg::launch_lmhead_tc(ex, c->tm_lm_a, c->tm_lm_b, c->lm, c->inv_temp, M, d, V, c->hs8_scale,
                         c->m.lm_head_scale);
  else if (dt == DG_BF16)
    dg::launch_lmhead_tc(ex, c->tm_lm_a, c->tm_lm_b, c->lm, c->inv_temp, M, d, V);
  else
    dg::launch_lmhead_simple(ex, dt, hs, c->m.lm_head, c->inv_temp, c->lm, M, d, V);
  if (c->cur_ev_stop[DG_KERNEL_LMHEAD])
    DG_CUDA_RET(cudaEventRecordWithFlags(c->cur_ev_stop[DG_KERNEL_LMHEAD], ex.stream, cudaEventRecordExternal));
  dg::launch_merge_select(ex, c->lm, c->ent, c->am, dbg ? dbg->freeze_mask : nullptr, &c->cs, &s, c->B, c->C, V,
                          c->cur_loop);
  c->launches = ex.launches;
  dg_status st = check_launch("denoise step launch");
  if (st != DG_OK) return st;
  if (dbg) {
    if (dbg->ent) DG_CUDA_RET(cudaMemcpyAsync(dbg->ent, c->ent, M * sizeof(float), cudaMemcpyDeviceToDevice, ex.stream));
    if (dbg->argmax) DG_CUDA_RET(cudaMemcpyAsync(dbg->argmax, c->am, M * sizeof(int32_t), cudaMemcpyDeviceToDevice, ex.stream));
    if (dbg->attn_out) DG_CUDA_RET(cudaMemcpyAsync(dbg->attn_out, c->O, (size_t)M * qd * c->es, cudaMemcpyDeviceToDevice, ex.stream));
    if (dbg->hidden) DG_CUDA_RET(cudaMemcpyAsync(dbg->hidden, hs, (size_t)M * d * c->es, cudaMemcpyDeviceToDevice, ex.stream));
    if (dbg->hidden_attn)
      DG_CUDA_RET(cudaMemcpyAsync(dbg->hidden_attn, c->Hs, (size_t)M * d * c->es, cudaMemcpyDeviceToDevice, ex.stream));
    if (dbg->q) DG_CUDA_RET(cudaMemcpyAsync(dbg->q, c->Q, (size_t)M * qd * c->es, cudaMemcpyDeviceToDevice, ex.stream));
    if (dbg->k_canvas)
      DG_CUDA_RET(cudaMemcpyAsync(dbg->k_canvas, c->Kc, (size_t)M * kd * c->es, cudaMemcpyDeviceToDevice, ex.stream));
    if (dbg->v_canvas)
      DG_CUDA_RET(cudaMemcpyAsync(dbg->v_canvas, c->Vc, (size_t)M * kd * c->es, cudaMemcpyDeviceToDevice, ex.stream));
    if (dbg->layer_out)
      for (int l = 0; l < c->L; ++l)
        DG_CUDA_RET(cudaMemcpyAsync(static_cast<char*>(dbg->layer_out) + (size_t)l * M * d * c->es, c->xres[l + 1],
                                    (size_t)M * d * c->es, cudaMemcpyDeviceToDevice, ex.stream));
  }
  return DG_OK;
}

bool same_sched(const dg_schedule& a, const dg_schedule& b) {
  return a.max_steps == b.max_steps && a.stop_entropy == b.stop_entropy && a.adaptive_stop == b.adaptive_stop &&
         a.kind == b.kind;
}

void drop_graphs(dg_ctx* c) {
  for (auto g : c->graphs)
    if (g) cudaGraphExecDestroy(g);
  c->graphs.clear();
  if (c->decode_graph) cudaGraphExecDestroy(c->decode_graph);
  c->decode_graph = nullptr;
}

// dg_decode_block's graph: a memset node clears the loop's step counter, then
// a conditional while node runs the step (the same launch sequence as a graph
// step, captured into the node's body) until the selection kernel of the step
// that leaves every canvas done sets the condition to 0. The loop never runs
// more than max_steps steps: every canvas stops by then (the freeze count
// takes all remaining positions at its last step), and the kernel also ends
// the loop at the cap (recording kDevLoopCap if a canvas is still open).
// The body is captured with programmatic launches first, and without them if
// the conditional body does not take them.
dg_status build_decode_graph(dg_ctx* c, const dg_schedule& s) {
  if (c->decode_graph && same_sched(c->decode_sched, s)) return DG_OK;
  if (c->decode_graph) cudaGraphExecDestroy(c->decode_graph);
  c->decode_graph = nullptr;
  if (!c->capture_stream) DG_CUDA_RET(cudaStreamCreateWithFlags(&c->capture_stream, cudaStreamNonBlocking));
  std::string why;
  for (int attempt = 0; attempt < 2 && !c->decode_graph; ++attempt) {
    cudaGraph_t g = nullptr;
    cudaGraphExec_t exec = nullptr;
    cudaError_t e = cudaGraphCreate(&g, 0);
    cudaGraphConditionalHandle h = 0;
    if (e == cudaSuccess) e = cudaGraphConditionalHandleCreate(&h, g, 1, cudaGraphCondAssignDefault);
    cudaGraphNode_t reset = nullptr, loop = nullptr, ev0 = nullptr, ev1 = nullptr;
    const cudaEvent_t t_start = c->ev_start[DG_KERNEL_DECODE].empty() ? nullptr : c->ev_start[DG_KERNEL_DECODE][0];
    const cudaEvent_t t_stop = c->ev_stop[DG_KERNEL_DECODE].empty() ? nullptr : c->ev_stop[DG_KERNEL_DECODE][0];
    if (e == cudaSuccess && t_start) e = cudaGraphAddEventRecordNode(&ev0, g, nullptr, 0, t_start);
    if (e == cudaSuccess) {
      cudaMemsetParams mp = {};
      mp.dst = c->cs.loop_iter;
      mp.value = 0;
      mp.elementSize = 4;
      mp.width = 1;
      mp.height = 1;
      mp.pitch = 4;
      e = cudaGraphAddMemsetNode(&reset, g, ev0 ? &ev0 : nullptr, ev0 ? 1 : 0, &mp);
    }
    cudaGraphNodeParams cp = {};
    if (e == cudaSuccess) {
      cp.type = cudaGraphNodeTypeConditional;
      cp.conditional.handle = h;
      cp.conditional.type = cudaGraphCondTypeWhile;
      cp.conditional.size = 1;
      e = cudaGraphAddNode(&loop, g, &reset, 1, &cp);
    }
    if (e == cudaSuccess && t_stop) e = cudaGraphAddEventRecordNode(&ev1, g, &loop, 1, t_stop);
    dg_status st = DG_OK;
    if (e == cudaSuccess) {
      cudaGraph_t body = cp.conditional.phGraph_out[0];
      cudaStream_t user = c->ex.stream;
      c->ex.stream = c->capture_stream;
      c->loop.handle = h;
      c->loop.cap = s.max_steps;
      c->cur_loop = &c->loop;
      dg::t_pdl_off = attempt == 1;
      e = cudaStreamBeginCaptureToGraph(c->capture_stream, body, nullptr, nullptr, 0,
                                        cudaStreamCaptureModeThreadLocal);
      if (e == cudaSuccess) {
        st = enqueue_step(c, s, nullptr);
        cudaGraph_t out = nullptr;
        const cudaError_t e2 = cudaStreamEndCapture(c->capture_stream, &out);
        if (e2 != cudaSuccess) e = e2;
      }
      dg::t_pdl_off = false;
      c->cur_loop = nullptr;
      c->ex.stream = user;
    }
    if (e == cudaSuccess && st == DG_OK) e = cudaGraphInstantiate(&exec, g, 0);
    if (g) cudaGraphDestroy(g);
    cudaGetLastError();
    if (st != DG_OK) return st;
    if (e == cudaSuccess) {
      c->decode_graph = exec;
      c->decode_sched = s;
    } else {
      why += std::string(attempt ? "; without programmatic launch: " : "") + cudaGetErrorString(e);
    }
  }
  if (!c->decode_graph) {
    set_last_error("building the device-side decode loop failed: " + why);
    return DG_ERR_CUDA;
  }
  return DG_OK;
}

// One step without debug outputs: a CUDA graph of the whole launch sequence,
// captured on a private stream the first time (and again when the schedule
// changes), then launched on the caller's stream. With timing events set,
// graph variant i records, for each timed kernel k, event pair i mod n_k
// around that kernel, and step n uses variant n mod (largest n_k).
dg_status launch_step_graph(dg_ctx* c, const dg_schedule& s) {
  const size_t nvar = std::max<size_t>(1, std::max(c->ev_start[0].size(), c->ev_start[1].size()));
  if (c->graphs.size() != nvar || !same_sched(c->graph_sched, s)) {
    drop_graphs(c);
    c->graphs.assign(nvar, nullptr);
    c->graph_sched = s;
  }
  const size_t v = (size_t)(c->step_launch_count % (long long)nvar);
  if (!c->graphs[v]) {
    if (!c->capture_stream) DG_CUDA_RET(cudaStreamCreateWithFlags(&c->capture_stream, cudaStreamNonBlocking));
    cudaStream_t user = c->ex.stream;
    c->ex.stream = c->capture_stream;
    for (int k = 0; k < 2; ++k) {
      const size_t nk = c->ev_start[k].size();
      c->cur_ev_start[k] = nk ? c->ev_start[k][v % nk] : nullptr;
      c->cur_ev_stop[k] = nk ? c->ev_stop[k][v % nk] : nullptr;
    }
    cudaGraph_t g = nullptr;
    cudaError_t e = cudaStreamBeginCapture(c->capture_stream, cudaStreamCaptureModeThreadLocal);
    dg_status st = DG_OK;
    if (e == cudaSuccess) {
      st = enqueue_step(c, s, nullptr);
      e = cudaStreamEndCapture(c->capture_stream, &g);
    }
    c->ex.stream = user;
    for (int k = 0; k < 2; ++k) c->cur_ev_start[k] = c->cur_ev_stop[k] = nullptr;
    if (st != DG_OK) {
      if (g) cudaGraphDestroy(g);
      return st;
    }
    DG_CUDA_RET(e);
    e = cudaGraphInstantiate(&c->graphs[v], g, 0);
    cudaGraphDestroy(g);
    DG_CUDA_RET(e);
    c->graph_launches = c->launches;
  }
  DG_CUDA_RET(cudaGraphLaunch(c->graphs[v], c->ex.stream));
  c->step_launch_count++;
  c->launches = c->graph_launches;
  return DG_OK;
}

dg_status read_device_error(dg_ctx* c) {
  int32_t e = 0;
  DG_CUDA_RET(cudaMemcpyAsync(&e, c->err, sizeof(e), cudaMemcpyDeviceToHost, c->ex.stream));
  DG_CUDA_RET(cudaStreamSynchronize(c->ex.stream));
  if (e == 0) return DG_OK;
  char buf[96];
  snprintf(buf, sizeof buf, "device-side check failed (code %d)", e);
  set_last_error(buf);
  return e == dg::kDevWaitTimeout ? DG_ERR_TIMEOUT : DG_ERR_DEVICE_CHECK;
}

}  // namespace

extern "C" {

int32_t dg_abi_version(void) { return DG_ABI_VERSION; }

const char* dg_last_error(void) { return dg::g_last_error.c_str(); }

const char* dg_status_string(dg_status s) {
  switch (s) {
    case DG_OK: return "ok";
    case DG_ERR_INVALID_ARG: return "invalid argument";
    case DG_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case DG_ERR_OOM: return "out of device memory";
    case DG_ERR_CUDA: return "CUDA error";
    case DG_ERR_TIMEOUT: return "device wait timed out";
    case DG_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

int32_t dg_launches_per_step(const dg_ctx* ctx) { return ctx ? ctx->launches : 0; }

dg_status dg_canvas_init(dg_ctx** out, const dg_model_desc* model, int32_t batch, int32_t canvas_len,
                         const int32_t* prefix_len, const void* const* prefix_k,
                         const void* const* prefix_v, const float* inv_temp, const uint64_t* seeds,
                         void* cuda_stream) {
  DG_ARG(out != nullptr, "out is NULL");
  *out = nullptr;
  dg_status st = validate_model(model);
  if (st != DG_OK) return st;
  DG_ARG(batch >= 1 && batch <= 4096, "batch must be in [1, 4096]");
  DG_ARG(canvas_len >= 1 && canvas_len <= 1024, "canvas_len must be in [1, 1024]");
  if (model->n_experts) DG_UNSUP(batch * canvas_len <= 256, "the MoE FFN needs batch * canvas_len <= 256");
  DG_ARG(prefix_len && seeds, "prefix_len / seeds is NULL");
  for (int b = 0; b < batch; ++b) {
    DG_ARG(prefix_len[b] >= 0 && prefix_len[b] <= (1 << 24), "prefix_len out of range");
    if (prefix_len[b] > 0) {
      DG_ARG(prefix_k && prefix_v && prefix_k[b] && prefix_v[b], "prefix K/V pointer is NULL");
      DG_ARG(aligned16(prefix_k[b]) && aligned16(prefix_v[b]), "prefix K/V must be 16-byte aligned");
    }
  }
  if (inv_temp) DG_ARG(aligned16(inv_temp), "inv_temp must be 16-byte aligned");

  dg_ctx* c = new dg_ctx();
  c->m = *model;
  c->B = batch;
  c->C = canvas_len;
  c->M = batch * canvas_len;
  c->es = model->dtype == DG_F32 ? 4 : 2;
  c->L = std::max(1, (int)model->n_layers);
  c->g_qkv.resize(c->L);
  c->g_wo.resize(c->L);
  c->attn.resize(c->L);
  c->inv_temp = inv_temp;
  c->ex.stream = static_cast<cudaStream_t>(cuda_stream);
  for (int b = 0; b < batch; ++b) {
    c->S.push_back(prefix_len[b]);
    c->pk.push_back(prefix_len[b] ? prefix_k[b] : nullptr);
    c->pv.push_back(prefix_len[b] ? prefix_v[b] : nullptr);
    c->max_S = std::max(c->max_S, (int)prefix_len[b]);
  }
  auto fail = [&](dg_status s) { dg_canvas_destroy(c); return s; };
  if (cudaGetDevice(&c->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&c->ex.sm_count, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess) {
    cudaGetLastError();
    set_last_error("no usable CUDA device");
    return fail(DG_ERR_CUDA);
  }
  if (model->dtype == DG_BF16) {
    c->lm.P = dg::lmhead_tc_partitions(c->M, model->vocab, c->ex.sm_count);
    c->attn_slots = dg::attn_tc_slots(batch, canvas_len, model->n_q_heads, model->n_kv_heads, c->S.data(),
                                      c->ex.sm_count);
    // tile / split choice only (buffers are bound after the workspace exists)
    const int qd = model->n_q_heads * model->head_dim, kd = model->n_kv_heads * model->head_dim;
    const void* wqkv[3] = {model->wq, model->wk, model->wv};
    void* none[3] = {nullptr, nullptr, nullptr};
    const int nqkv[3] = {qd, kd, kd};
    const void* wo[1] = {model->wo};
    const int no[1] = {model->d_model};
    if (!dg::gemm_tc_prepare(&c->g_qkv[0], model->embed, c->M, model->d_model, 3, wqkv, none, nqkv, c->ex.sm_count) ||
        !dg::gemm_tc_prepare(&c->g_wo[0], model->embed, c->M, qd, 1, wo, none, no, c->ex.sm_count))
      return fail(DG_ERR_CUDA);
  }
  else
    c->lm.P = std::max(1, std::min(128, model->vocab / 1024));

  size_t total = 0;
  layout_workspace(c, nullptr, &total);
  const char* lim = std::getenv("DG_WORKSPACE_LIMIT_MB");
  if (lim && (double)total > std::atof(lim) * 1048576.0) {
    set_last_error("workspace exceeds DG_WORKSPACE_LIMIT_MB");
    return fail(DG_ERR_OOM);
  }
  if (cudaMalloc(&c->ws, total) != cudaSuccess) {
    cudaGetLastError();
    set_last_error("cudaMalloc of the workspace failed");
    return fail(DG_ERR_OOM);
  }
  c->ws_bytes = total;
  layout_workspace(c, c->ws, &total);
  c->ex.err = c->err;
  if (model->dtype == DG_BF16) {
    const bool fp8 = model->lm_head_format == DG_LM_E4M3;
    const void* lm_in = fp8 ? (const void*)c->hs8 : model->n_experts ? c->Hs2 : c->Hs;
    if (!dg::lmhead_tc_prepare(lm_in, model->lm_head, c->M, model->d_model, model->vocab, &c->tm_lm_a,
                               &c->tm_lm_b, fp8) ||
        !prepare_layer_gemms(c))
      return fail(DG_ERR_CUDA);
    if (model->n_experts) {
      dg::MoeShape ms{c->M, model->d_model, model->n_experts, model->top_k, model->n_shared, model->moe_inter,
                      model->expert_format == DG_LM_E4M3};
      const float* scales[3] = {model->w_gate_scale, model->w_up_scale, model->w_down_scale};
      if (!dg::moe_prepare(&c->moe, ms, c->Hs, c->Hs2, model->w_router, model->w_gate, model->w_up, model->w_down,
                           c->moe_ws, c->ex.sm_count, scales))
        return fail(DG_ERR_UNSUPPORTED);
    }
  }

  st = prepare_layer_attention(c);
  if (st != DG_OK) return fail(st);
  cudaStream_t sm = c->ex.stream;
  if (cudaMemcpyAsync(c->cs.seed, seeds, batch * sizeof(uint64_t), cudaMemcpyHostToDevice, sm) != cudaSuccess ||
      cudaMemsetAsync(c->cs.counters, 0, (batch + 1) * sizeof(uint32_t), sm) != cudaSuccess ||
      cudaMemsetAsync(c->cs.loop_iter, 0, sizeof(int32_t), sm) != cudaSuccess ||
      cudaMemsetAsync(c->err, 0, sizeof(int32_t), sm) != cudaSuccess) {
    set_last_error("initial copies failed");
    return fail(DG_ERR_CUDA);
  }
  dg::launch_init_canvas(c->ex, c->cs, c->B, c->C, model->vocab);
  st = check_launch("init canvas");
  if (st != DG_OK) return fail(st);
  if (cudaStreamSynchronize(sm) != cudaSuccess) {
    set_last_error("init synchronize failed");
    return fail(DG_ERR_CUDA);
  }
  *out = c;
  return DG_OK;
}

dg_status dg_denoise_step(dg_ctx* ctx, const dg_schedule* sched, const dg_step_out* dbg) {
  DG_ARG(ctx != nullptr, "ctx is NULL");
  dg_status st = validate_sched(sched);
  if (st != DG_OK) return st;
  if (dbg) return enqueue_step(ctx, *sched, dbg);
  return launch_step_graph(ctx, *sched);
}

dg_status dg_canvas_reset(dg_ctx* ctx, const uint64_t* seeds) {
  DG_ARG(ctx != nullptr, "ctx is NULL");
  if (seeds)
    DG_CUDA_RET(cudaMemcpyAsync(ctx->cs.seed, seeds, ctx->B * sizeof(uint64_t), cudaMemcpyHostToDevice,
                                ctx->ex.stream));
  dg::launch_init_canvas(ctx->ex, ctx->cs, ctx->B, ctx->C, ctx->m.vocab);
  return check_launch("reset canvas");
}

dg_status dg_canvas_reset_fixed(dg_ctx* ctx, const uint64_t* seeds, const uint8_t* fixed_mask,
                                const int32_t* fixed_tokens) {
  DG_ARG(ctx != nullptr, "ctx is NULL");
  DG_ARG(fixed_mask && fixed_tokens, "fixed_mask / fixed_tokens is NULL");
  for (int i = 0; i < ctx->M; ++i)
    if (fixed_mask[i]) DG_ARG(fixed_tokens[i] >= 0 && fixed_tokens[i] < ctx->m.vocab, "fixed token id out of range");
  dg_status st = dg_canvas_reset(ctx, seeds);
  if (st != DG_OK) return st;
  // the step-0 draws of the open positions stay; the given ones overwrite theirs
  std::vector<int32_t> tok(ctx->M);
  std::vector<uint8_t> frozen(ctx->M);
  DG_CUDA_RET(cudaMemcpyAsync(tok.data(), ctx->cs.tok, ctx->M * sizeof(int32_t), cudaMemcpyDeviceToHost, ctx->ex.stream));
  DG_CUDA_RET(cudaStreamSynchronize(ctx->ex.stream));
  for (int i = 0; i < ctx->M; ++i) {
    frozen[i] = fixed_mask[i] ? 1 : 0;
    if (fixed_mask[i]) tok[i] = fixed_tokens[i];
  }
  DG_CUDA_RET(cudaMemcpyAsync(ctx->cs.tok, tok.data(), ctx->M * sizeof(int32_t), cudaMemcpyHostToDevice, ctx->ex.stream));
  DG_CUDA_RET(cudaMemcpyAsync(ctx->cs.frozen, frozen.data(), ctx->M, cudaMemcpyHostToDevice, ctx->ex.stream));
  DG_CUDA_RET(cudaStreamSynchronize(ctx->ex.stream));
  return read_device_error(ctx);
}

dg_status dg_canvas_block_kv(dg_ctx* c, void* k_out, void* v_out) {
  DG_ARG(c != nullptr, "ctx is NULL");
  DG_ARG(k_out && v_out, "k_out / v_out is NULL");
  DG_UNSUP(c->L == 1, "block K/V need the single-layer model (deeper stacks need a causal encoder pass)");
  const int M = c->M, d = c->m.d_model, V = c->m.vocab;
  const int qd = c->m.n_q_heads * c->m.head_dim, kd = c->m.n_kv_heads * c->m.head_dim;
  dg::Exec& ex = c->ex;
  ex.launches = 0;
  dg::launch_embed(ex, c->m.dtype, c->m.embed, c->cs.tok, c->X, M, d, V);
  if (c->m.dtype == DG_BF16) {
    dg::launch_gemm_tc(ex, c->g_qkv[0], nullptr);
  } else {
    dg::launch_linear_simple(ex, c->m.dtype, c->X, c->m.wk, nullptr, c->Kc, M, kd, d);
    dg::launch_linear_simple(ex, c->m.dtype, c->X, c->m.wv, nullptr, c->Vc, M, kd, d);
  }
  (void)qd;
  dg_status st = check_launch("block K/V");
  if (st != DG_OK) return st;
  DG_CUDA_RET(cudaMemcpyAsync(k_out, c->Kc, (size_t)M * kd * c->es, cudaMemcpyDeviceToDevice, ex.stream));
  DG_CUDA_RET(cudaMemcpyAsync(v_out, c->Vc, (size_t)M * kd * c->es, cudaMemcpyDeviceToDevice, ex.stream));
  return DG_OK;
}

dg_status dg_canvas_set_prefix(dg_ctx* c, const int32_t* prefix_len, const void* const* prefix_k,
                               const void* const* prefix_v) {
  DG_ARG(c != nullptr, "ctx is NULL");
  DG_ARG(prefix_len != nullptr, "prefix_len is NULL");
  for (int b = 0; b < c->B; ++b) {
    DG_ARG(prefix_len[b] >= 0 && prefix_len[b] <= (1 << 24), "prefix_len out of range");
    if (prefix_len[b] > 0) {
      DG_ARG(prefix_k && prefix_v && prefix_k[b] && prefix_v[b], "prefix K/V pointer is NULL");
      DG_ARG(aligned16(prefix_k[b]) && aligned16(prefix_v[b]), "prefix K/V must be 16-byte aligned");
    }
  }
  DG_CUDA_RET(cudaStreamSynchronize(c->ex.stream));  // queued steps read the old prefix
  drop_graphs(c);
  c->max_S = 0;
  for (int b = 0; b < c->B; ++b) {
    c->S[b] = prefix_len[b];
    c->pk[b] = prefix_len[b] ? prefix_k[b] : nullptr;
    c->pv[b] = prefix_len[b] ? prefix_v[b] : nullptr;
    c->max_S = std::max(c->max_S, (int)prefix_len[b]);
  }
  // the attention's partial buffers were sized at init: its schedule for the
  // new lengths shares no unit among more CTAs than they hold
  dg_status st = prepare_layer_attention(c);
  if (st != DG_OK) return st;
  DG_CUDA_RET(cudaStreamSynchronize(c->ex.stream));
  return DG_OK;
}

dg_status dg_decode_block(dg_ctx* ctx, const dg_schedule* sched, int32_t* tokens_out, int32_t* steps_out) {
  DG_ARG(ctx != nullptr, "ctx is NULL");
  dg_status st = validate_sched(sched);
  if (st != DG_OK) return st;
  // One launch of the decode graph: the loop over steps and its end run on
  // the device. The host only looks at the done flag first (a block that is
  // already finished launches nothing).
  int32_t all = 0;
  DG_CUDA_RET(cudaMemcpyAsync(&all, ctx->cs.all_done, sizeof(all), cudaMemcpyDeviceToHost, ctx->ex.stream));
  DG_CUDA_RET(cudaStreamSynchronize(ctx->ex.stream));
  if (!all) {
    st = build_decode_graph(ctx, *sched);
    if (st != DG_OK) return st;
    DG_CUDA_RET(cudaGraphLaunch(ctx->decode_graph, ctx->ex.stream));
  }
  // results and the device error word come back together: one wait
  if (tokens_out)
    DG_CUDA_RET(cudaMemcpyAsync(tokens_out, ctx->cs.tok, ctx->M * sizeof(int32_t), cudaMemcpyDefault, ctx->ex.stream));
  if (steps_out)
    DG_CUDA_RET(cudaMemcpyAsync(steps_out, ctx->cs.step, ctx->B * sizeof(int32_t), cudaMemcpyDeviceToHost, ctx->ex.stream));
  return read_device_error(ctx);
}

dg_status dg_canvas_get_state(dg_ctx* ctx, dg_state* h) {
  DG_ARG(ctx && h, "NULL argument");
  DG_ARG(h->tokens && h->frozen && h->step && h->seed && h->done, "a state array is NULL");
  DG_CUDA_RET(cudaMemcpyAsync(h->tokens, ctx->cs.tok, ctx->M * sizeof(int32_t), cudaMemcpyDeviceToHost, ctx->ex.stream));
  DG_CUDA_RET(cudaMemcpyAsync(h->frozen, ctx->cs.frozen, ctx->M, cudaMemcpyDeviceToHost, ctx->ex.stream));
  DG_CUDA_RET(cudaMemcpyAsync(h->step, ctx->cs.step, ctx->B * sizeof(int32_t), cudaMemcpyDeviceToHost, ctx->ex.stream));
  DG_CUDA_RET(cudaMemcpyAsync(h->seed, ctx->cs.seed, ctx->B * sizeof(uint64_t), cudaMemcpyDeviceToHost, ctx->ex.stream));
  DG_CUDA_RET(cudaMemcpyAsync(h->done, ctx->cs.done, ctx->B, cudaMemcpyDeviceToHost, ctx->ex.stream));
  DG_CUDA_RET(cudaStreamSynchronize(ctx->ex.stream));
  return read_device_error(ctx);
}

dg_status dg_canvas_set_state(dg_ctx* ctx, const dg_state* h) {
  DG_ARG(ctx && h, "NULL argument");
  DG_ARG(h->tokens && h->frozen && h->step && h->seed && h->done, "a state array is NULL");
  int all = 1;
  for (int i = 0; i < ctx->M; ++i) DG_ARG(h->tokens[i] >= 0 && h->tokens[i] < ctx->m.vocab, "token id out of range");
  for (int b = 0; b < ctx->B; ++b) {
    DG_ARG(h->step[b] >= 0, "negative step");
    all &= h->done[b] ? 1 : 0;
  }
  DG_CUDA_RET(cudaStreamSynchronize(ctx->ex.stream));
  DG_CUDA_RET(cudaMemcpyAsync(ctx->cs.tok, h->tokens, ctx->M * sizeof(int32_t), cudaMemcpyHostToDevice, ctx->ex.stream));
  DG_CUDA_RET(cudaMemcpyAsync(ctx->cs.frozen, h->frozen, ctx->M, cudaMemcpyHostToDevice, ctx->ex.stream));
  DG_CUDA_RET(cudaMemcpyAsync(ctx->cs.step, h->step, ctx->B * sizeof(int32_t), cudaMemcpyHostToDevice, ctx->ex.stream));
  DG_CUDA_RET(cudaMemcpyAsync(ctx->cs.seed, h->seed, ctx->B * sizeof(uint64_t), cudaMemcpyHostToDevice, ctx->ex.stream));
  DG_CUDA_RET(cudaMemcpyAsync(ctx->cs.done, h->done, ctx->B, cudaMemcpyHostToDevice, ctx->ex.stream));
  DG_CUDA_RET(cudaMemcpyAsync(ctx->cs.all_done, &all, sizeof(int32_t), cudaMemcpyHostToDevice, ctx->ex.stream));
  DG_CUDA_RET(cudaStreamSynchronize(ctx->ex.stream));
  return DG_OK;
}

dg_status dg_canvas_set_kernel_timing(dg_ctx* ctx, int32_t kernel, int32_t n, void* const* starts,
                                      void* const* stops) {
  DG_ARG(ctx != nullptr, "ctx is NULL");
  DG_ARG(kernel == DG_KERNEL_LMHEAD || kernel == DG_KERNEL_ATTENTION || kernel == DG_KERNEL_DECODE,
         "unknown kernel id");
  DG_ARG(n >= 0 && n <= 64, "n must be in [0, 64]");
  DG_ARG(kernel != DG_KERNEL_DECODE || n <= 1, "the decode loop takes one event pair");
  if (n > 0) DG_ARG(starts && stops, "event arrays are NULL");
  for (int i = 0; i < n; ++i) DG_ARG(starts[i] && stops[i], "NULL event");
  DG_CUDA_RET(cudaStreamSynchronize(ctx->ex.stream));
  drop_graphs(ctx);
  ctx->ev_start[kernel].clear();
  ctx->ev_stop[kernel].clear();
  for (int i = 0; i < n; ++i) {
    ctx->ev_start[kernel].push_back(static_cast<cudaEvent_t>(starts[i]));
    ctx->ev_stop[kernel].push_back(static_cast<cudaEvent_t>(stops[i]));
  }
  ctx->step_launch_count = 0;
  return DG_OK;
}

dg_status dg_canvas_set_timing_events(dg_ctx* ctx, int32_t n, void* const* starts, void* const* stops) {
  return dg_canvas_set_kernel_timing(ctx, DG_KERNEL_LMHEAD, n, starts, stops);
}

dg_status dg_canvas_loop_steps(dg_ctx* ctx, int32_t* steps_out) {
  DG_ARG(ctx != nullptr && steps_out != nullptr, "NULL argument");
  DG_CUDA_RET(cudaMemcpyAsync(steps_out, ctx->cs.loop_iter, sizeof(int32_t), cudaMemcpyDeviceToHost, ctx->ex.stream));
  DG_CUDA_RET(cudaStreamSynchronize(ctx->ex.stream));
  return DG_OK;
}

dg_status dg_canvas_sync(dg_ctx* ctx) {
  DG_ARG(ctx != nullptr, "ctx is NULL");
  return read_device_error(ctx);
}

void dg_canvas_destroy(dg_ctx* ctx) {
  if (!ctx) return;
  if (ctx->ws) {
    cudaStreamSynchronize(ctx->ex.stream);
    cudaFree(ctx->ws);
  }
  drop_graphs(ctx);
  if (ctx->capture_stream) cudaStreamDestroy(ctx->capture_stream);
  delete ctx;
}

}  // extern "C"
