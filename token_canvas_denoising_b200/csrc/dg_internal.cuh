// Internal declarations of libdgcanvas: the context, its workspace layout and
// the kernel launchers. Not part of the C ABI.
#pragma once
#include <cuda.h>

#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "dg_canvas.h"
#include "dg_common.cuh"

namespace dg {

struct PrefixDesc {  // one request's cached prompt K/V, device pointers
  const void* k;     // [len][Hk][h]
  const void* v;
  int32_t len;
  int32_t pad;
};

// Per-row partial of the fused LM-head epilogue over one vocab range. Stored
// row-major by row ([M][P] records) so that one warp reads a row's P partials
// with contiguous 32-byte loads.
struct alignas(32) LmRec {
  float m;      // running max of the scaled logits
  float z;      // sum exp(l - m)
  float s;      // sum (l - m) exp(l - m)
  float best;   // max unscaled logit
  int32_t idx;  // its vocab id (lowest on ties)
  int32_t pad0, pad1, pad2;
};
struct LmPartials {
  LmRec* rec;   // [M][P]
  int P;
};

// Where and how kernels are launched.
struct Exec {
  cudaStream_t stream = nullptr;
  int* err = nullptr;   // device error word
  int launches = 0;     // kernels queued (for launch accounting)
  int sm_count = 148;
};

// Shapes of one attention call.
struct AttnShape {
  int B, C, Hq, Hk, h;
};

void set_last_error(const std::string& msg);

// The calling thread's current CUDA context (dg_tmap.cu).
bool current_context(void** ctx);

// Device addresses of one file-scope __device__ variable, one per (device,
// context). In host code the variable's name is only a host-side stand-in,
// so its address on the current device is looked up with
// cudaGetSymbolAddress the first time a context uses it, and kept. Keying on
// the context makes an address looked up before a device reset (which ends
// that context) unreachable afterwards. get() must be instantiated in the
// translation unit that defines the variable.
struct SymbolAddressCache {
  struct Entry {
    int device;
    void* ctx;
    void* addr;
  };
  std::mutex mu;
  std::vector<Entry> entries;

  template <typename T> dg_status get(const T& symbol, void** out) {
    int dev = -1;
    void* ctx = nullptr;
    if (cudaGetDevice(&dev) != cudaSuccess) {
      cudaGetLastError();
      set_last_error("no usable CUDA device");
      return DG_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (current_context(&ctx))
      for (const Entry& e : entries)
        if (e.device == dev && e.ctx == ctx) {
          *out = e.addr;
          return DG_OK;
        }
    // not seen in this context (the lookup also makes the device's primary
    // context current if no context was yet)
    void* p = nullptr;
    const cudaError_t err = cudaGetSymbolAddress(&p, symbol);
    if (err != cudaSuccess || !p || !current_context(&ctx)) {
      cudaGetLastError();
      set_last_error(std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(err));
      return DG_ERR_CUDA;
    }
    entries.push_back({dev, ctx, p});
    *out = p;
    return DG_OK;
  }
};

// Device error word of the single-operation entry points (dg_ops.cu); the
// allocation-free LM head has its own beside its scratch (dg_noalloc.cu).
dg_status ops_error_word(int** out);
dg_status noalloc_error_word(int** out);

// Launch with programmatic stream serialization (see griddep_wait in
// dg_common.cuh); the kernel must call griddep_wait() before using its
// predecessors' outputs.
// Programmatic launch is dropped (plain stream order) while this is set on
// the launching thread: for graphs whose bodies take no programmatic edges.
inline thread_local bool t_pdl_off = false;

template <typename... KArgs, typename... Args>
inline void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = t_pdl_off ? 0 : 1;
  cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// launch_pdl for kernels whose CTAs run in pairs (thread-block clusters of 2
// along x, for tcgen05 .cta_group::2): grid.x must be even.
template <typename... KArgs, typename... Args>
inline void launch_pdl_pairs(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = t_pdl_off ? 1 : 2;
  cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---- embed / linear / attention / LM head (dtype-dispatched)
void launch_embed(Exec& ex, int dtype, const void* E, const int32_t* tok, void* X, int M, int d, int V);
void launch_linear_simple(Exec& ex, int dtype, const void* A, const void* W, const void* R, void* out,
                          int M, int N, int K);
void launch_attention_simple(Exec& ex, int dtype, const void* Q, const PrefixDesc* d_prefix, const void* Kc,
                             const void* Vc, void* O, const AttnShape& s);
void launch_lmhead_simple(Exec& ex, int dtype, const void* hs, const void* W, const float* invT,
                          LmPartials part, int M, int d, int V);

// tcgen05 LM head (bf16): vocab partitions for M rows, tensor maps, launch
int lmhead_tc_partitions(int M, int V, int sm_count);
// With fp8, hs and lm_head are e4m3 codes ([M][d] and [V][d] bytes) and the
// launch takes their power-of-two row scales sa [M] and sw [V] (sa == null:
// bf16 operands).
bool lmhead_tc_prepare(const void* hs, const void* lm_head, int M, int d, int V, CUtensorMap* tmA,
                       CUtensorMap* tmB, bool fp8 = false);
void launch_lmhead_tc(Exec& ex, const CUtensorMap& tmA, const CUtensorMap& tmB, LmPartials part,
                      const float* invT, int M, int d, int V, const float* sa = nullptr,
                      const float* sw = nullptr);
// Quantize rows of a bf16 matrix to e4m3 with the smallest power-of-two scale
// per row that fits the row's largest magnitude: codes [M][d], scales [M].
void launch_quantize_rows_e4m3(Exec& ex, const void* x, uint8_t* codes, float* scales, int M, int d);

// tcgen05 projection GEMM (bf16): out_i = A W_i^T (+ R) for up to 3 output
// segments sharing A; prepared once (tensor maps), launched many times.
struct alignas(64) GemmTc {
  unsigned char maps[4 * 128];  // CUtensorMap for A and each W_i
  int M = 0, K = 0, nseg = 0, tiles = 0, bn = 64, splits = 1, ncols = 0;
  int out_f32 = 0;               // f32 outputs (set after prepare; requires splits == 1)
  void* out[3] = {nullptr, nullptr, nullptr};
  int N[3] = {0, 0, 0};
  float* part = nullptr;         // split-K partials [splits][M][ncols]
};
// Chooses the tile width and the K splits (for sm_count SMs) and encodes the
// tensor maps; the caller then provides `part` of the size below when
// splits > 1.
bool gemm_tc_prepare(GemmTc* g, const void* A, int M, int K, int nseg, const void* const* W, void* const* out,
                     const int* N, int sm_count);
bool gemm_tc_prepare_with(GemmTc* g, const void* A, int M, int K, int nseg, const void* const* W,
                          void* const* out, const int* N, int bn, int splits);
size_t gemm_tc_partial_floats(const GemmTc& g);
void launch_gemm_tc(Exec& ex, const GemmTc& g, const void* residual);

// tcgen05 attention (bf16, head_dim 128): tensor maps and the stream-K
// schedule per group of up to 8 requests; partial buffers for the units that
// several CTAs share.
struct AttnTc {
  // stream-K schedule of one launch: the units' T key tiles over G CTAs, at
  // most `parts` CTAs per unit (the partial slots it needs)
  struct Sched {
    int G = 1, T = 0, Tp = 0, parts = 1;
    int nt[8] = {0}, reqoff[8] = {0};
  };
  struct Group {
    alignas(64) unsigned char maps[19 * 128];
    int b0 = 0, nreq = 0;
    int S[8] = {0};
    Sched sched;
  };
  AttnShape sh{};
  void* O = nullptr;
  float* part_o = nullptr;
  float* part_ml = nullptr;
  std::vector<Group> groups;
};
// Partial slots (parts per row) the attention needs for these prefix lengths
// on sm_count SMs; 1 = none.
int attn_tc_slots(int B, int C, int Hq, int Hk, const int* S, int sm_count);
// Tensor maps and schedules; the schedules share no unit among more than
// `slots` CTAs (the partial buffers hold [slots][B*C*Hq] rows; with part_o
// NULL every unit runs in one CTA).
bool attn_tc_prepare(AttnTc* at, const AttnShape& sh, const void* Q, const void* Kc, const void* Vc,
                     const int32_t* S, const void* const* pk, const void* const* pv, void* O, float* part_o,
                     float* part_ml, int slots, int sm_count);
void launch_attn_tc(Exec& ex, const AttnTc& at);

// MoE FFN (bf16): router GEMM, routing, gather, expert gate/up and down GEMMs,
// combine; all buffers in one workspace region of moe_workspace_bytes().
struct MoeShape {
  int M, d, E, topk, nsh, I;
  bool fp8 = false;  // e4m3 expert weights
};
struct MoeTc {
  MoeShape s{};
  const void* hs = nullptr;  // residual stream in [M][d]
  void* hs_out = nullptr;    // residual stream out [M][d]
  float* logits = nullptr;   // [M][E]
  float* gate = nullptr;     // [M][topk]
  int* sel = nullptr;        // [M][topk] chosen experts
  int* pos = nullptr;        // [M][topk + nsh]
  int* off = nullptr;        // [E + nsh + 1]
  int* pair_tok = nullptr;   // [R]
  void* xg = nullptr;        // [R][d] bf16
  void* act = nullptr;       // [R][I] bf16
  float* y = nullptr;        // [R][d]
  uint8_t* xg8 = nullptr;    // e4m3: quantized token rows [R][d] and their scales sx [R]
  uint8_t* act8 = nullptr;   // e4m3: quantized intermediate [R][I] and its scales sa [R]
  float* sx = nullptr;
  float* sa = nullptr;
  const float* w_scale[3] = {nullptr, nullptr, nullptr};  // e4m3: row scales of W_gate, W_up, W_down
  GemmTc router;
  alignas(64) unsigned char maps_gateup[3 * 128];
  alignas(64) unsigned char maps_down[3 * 128];
};
size_t moe_workspace_bytes(const MoeShape& s);
// With s.fp8 the expert weights are e4m3 codes and w_scales their row scales
// (W_gate, W_up, W_down; [E+nsh][rows] f32 each).
bool moe_prepare(MoeTc* mt, const MoeShape& s, const void* hs, void* hs_out, const void* w_router,
                 const void* w_gate, const void* w_up, const void* w_down, void* ws, int sm_count,
                 const float* const* w_scales = nullptr);
void launch_moe(Exec& ex, const MoeTc& mt);

// ---- canvas bookkeeping
struct CanvasState {
  int32_t* tok;
  uint8_t* frozen;
  int32_t* step;
  uint64_t* seed;
  uint8_t* done;
  int32_t* all_done;
  uint32_t* counters;  // [B + 1], zero between launches
  int32_t* loop_iter;  // steps run by the current device-side decode loop
};
// A device-side decode loop: the conditional node that repeats the step, and
// the most steps it may take (the loop ends once every canvas is done).
struct DecodeLoop {
  cudaGraphConditionalHandle handle = 0;
  int cap = 0;
};
void launch_init_canvas(Exec& ex, const CanvasState& cs, int B, int C, int V);
// Merge the LM-head partials into ent/am; with `sched` non-null also run the
// freeze / stop / re-noise selection on every canvas.
// With `loop` set, the step is the body of a device-side decode loop: the
// kernel that finds every canvas done (or the cap reached) ends the loop.
void launch_merge_select(Exec& ex, LmPartials part, float* ent, int32_t* am, uint8_t* fmask,
                         const CanvasState* cs, const dg_schedule* sched, int B, int C, int V,
                         const DecodeLoop* loop = nullptr);

}  // namespace dg

struct dg_ctx {
  dg_model_desc m;
  int B = 0, C = 0, M = 0;
  int es = 0;  // storage element size (4 f32, 2 bf16)
  std::vector<int32_t> S;
  std::vector<const void*> pk, pv;
  int max_S = 0;
  const float* inv_temp = nullptr;
  int device = 0;
  dg::Exec ex;

  void* ws = nullptr;
  size_t ws_bytes = 0;

  dg::CanvasState cs{};
  int32_t* err = nullptr;

  // activations, storage dtype
  void *X = nullptr, *Q = nullptr, *Kc = nullptr, *Vc = nullptr, *O = nullptr;
  void *Hs = nullptr, *Hs2 = nullptr;
  uint8_t* hs8 = nullptr;      // e4m3 LM head: the quantized residual stream [M][d]
  float* hs8_scale = nullptr;  // and its row scales [M]
  dg::PrefixDesc* d_prefix = nullptr;

  dg::LmPartials lm{};
  float* ent = nullptr;
  int32_t* am = nullptr;

  // attention layers: per layer the projection GEMMs and the attention
  // (bf16 path); the residual stream after layer l is xres[l + 1] (xres[0] =
  // X, the embedding; xres[L] = Hs, the input of the MoE block / LM head)
  int L = 1;
  std::vector<void*> xres;
  CUtensorMap tm_lm_a, tm_lm_b;
  std::vector<dg::GemmTc> g_qkv, g_wo;
  std::vector<dg::AttnTc> attn;
  float* attn_part_o = nullptr;   // attention partials (units shared by CTAs), shared by the layers
  float* attn_part_ml = nullptr;
  int attn_slots = 1;             // partial slots per row the workspace holds
  dg::MoeTc moe;
  void* moe_ws = nullptr;

  int launches = 0;  // kernels queued by the last denoise step

  // the step captured as CUDA graphs (per schedule), launched on ex.stream;
  // with timing events there is one graph variant per event pair, used in turn
  cudaStream_t capture_stream = nullptr;
  std::vector<cudaGraphExec_t> graphs;
  dg_schedule graph_sched{};
  int graph_launches = 0;
  // timing event pairs per timed kernel (DG_KERNEL_LMHEAD, DG_KERNEL_ATTENTION)
  // and around the device-side decode loop (DG_KERNEL_DECODE)
  std::vector<cudaEvent_t> ev_start[3], ev_stop[3];
  cudaEvent_t cur_ev_start[2] = {nullptr, nullptr}, cur_ev_stop[2] = {nullptr, nullptr};  // set while capturing
  // dg_decode_block's graph: the step as the body of a conditional while node
  cudaGraphExec_t decode_graph = nullptr;
  dg_schedule decode_sched{};
  dg::DecodeLoop loop{};
  const dg::DecodeLoop* cur_loop = nullptr;  // set while capturing the loop body
  long long step_launch_count = 0;
};
