// Internal declarations of libdgcanvas: the context, its workspace layout and
// the kernel launchers. Not part of the C ABI.
#pragma once
#include <string>
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

// Split-KV attention partials: unnormalised O plus (max, sum) per query row.
struct AttnPartials {
  float* o;      // [splits][M*Hq][h]
  float* ml;     // [splits][M*Hq][2]
  int splits;
};

}  // namespace dg

struct dg_ctx {
  dg_model_desc m;
  int B = 0, C = 0, M = 0;
  int es = 0;  // storage element size (4 f32, 2 bf16)
  std::vector<int32_t> S;
  std::vector<const void*> pk, pv;
  int max_S = 0;
  const float* inv_temp = nullptr;
  cudaStream_t stream = nullptr;
  int device = 0, sm_count = 0;

  void* ws = nullptr;
  size_t ws_bytes = 0;

  // decode state
  int32_t* tok = nullptr;
  uint8_t* frozen = nullptr;
  int32_t* step = nullptr;
  uint64_t* seed = nullptr;
  uint8_t* done = nullptr;
  int32_t* err = nullptr;        // device error word
  int32_t* all_done = nullptr;   // 1 when every canvas is done
  uint32_t* counters = nullptr;  // scratch arrival counters (zero between launches)

  // activations, storage dtype
  void *X = nullptr, *Q = nullptr, *Kc = nullptr, *Vc = nullptr, *O = nullptr;
  void *Hs = nullptr, *Hs2 = nullptr;
  dg::PrefixDesc* d_prefix = nullptr;

  dg::LmPartials lm{};
  dg::AttnPartials attn{};
  float* ent = nullptr;
  int32_t* am = nullptr;
  uint8_t* fmask = nullptr;

  int launches = 0;  // kernels queued by the last denoise step

  // captured step graph
  cudaGraphExec_t graph_exec = nullptr;
  dg_schedule graph_sched{};
  bool graph_valid = false;
};

namespace dg {

// error reporting (thread-local message)
void set_last_error(const std::string& msg);

// simple CUDA-core kernels (f32 storage)
void launch_embed(dg_ctx* c);
void launch_linear_simple(dg_ctx* c, const void* A, const void* W, const void* R, void* out,
                          int M, int N, int K);
void launch_attention_simple(dg_ctx* c);
void launch_lmhead_simple(dg_ctx* c, const void* hs);

// canvas bookkeeping
void launch_init_canvas(dg_ctx* c);
void launch_merge_select(dg_ctx* c, const dg_schedule& s, uint8_t* fmask_out);

}  // namespace dg
