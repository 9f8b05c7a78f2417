// MoE FFN of the canvas step: a router over E experts, softmax top-k with
// renormalised gates, GeGLU experts and always-on shared experts, output added
// to the residual stream ("DiffusionGemma深度拆解：从逐字蹦到整块喷，LLM生成范式的结构性跃迁",
// 架构解剖 3: 128 fine-grained experts plus one shared expert, top-8 routing).
//
//   router   r = Hs Wr^T (f32)                      projection GEMM, f32 output
//   top-k    p = softmax(r); top-k by p (lower expert id on ties); gates
//            g = p_sel / sum p_sel (one warp per token)
//   group    rows of each expert listed in token order (one block)
//   gather   Xg[row] = Hs[token(row)]  (rows grouped by expert; shared experts
//            take every token)
//   gate/up  a = GELU(Xg W_gate^T) * (Xg W_up^T), rounded to bf16
//   down     y = a W_down^T (f32)
//   combine  Hs2 = bf16(Hs + sum_k g_k y_k + sum_shared y_shared), summed in
//            slot order so the result does not depend on scheduling
//
// With e4m3 expert weights (the FP8 deployment of "DiffusionGemma深度拆解",
// 性能数据) the weights are e4m3 codes with power-of-two scales per output row,
// the gathered token rows and the GeGLU intermediate are quantized per row
// (dg_fp8.cu) ahead of the gate/up and the down GEMMs, the MMAs are
// kind::f8f6f4 over 128-byte K blocks (a K tail past moe_inter is zero-filled
// by the tensor map), and the epilogues multiply by the weight row's and the
// token row's scales.
//
// The expert GEMMs put the weights on the 128-row MMA side (M = 128 rows of
// W) and an expert's tokens (a few dozen) on the N side, so a CTA streams one
// 128-row weight tile of one expert through a TMA ring while its tokens' rows
// ride along; the work is bound by the 1.5 GB of expert weights.
#include "dg_internal.cuh"
#include "dg_sm100.cuh"
#include "dg_tmap.cuh"

namespace dg {
namespace moe {

using namespace sm100;

constexpr int kMaxE = 256;       // routed experts
constexpr int kMaxTopK = 8;
constexpr int kMaxPairs = 8192;  // M * top_k held in shared memory by the router

// ---------------------------------------------------------------- routing
struct RouteParams {
  const float* logits;  // [M][E]
  int M, E, topk, nsh;
  float* gate;          // [M][topk]
  int* sel;             // [M][topk] chosen expert per (token, slot)
  int* pos;             // [M][topk + nsh] row of each (token, slot) in the grouped buffers
  int* off;             // [E + nsh + 1] first row of each expert (shared experts last)
  int* pair_tok;        // [M * (topk + nsh)] token of each grouped row
};

// One warp per token: softmax over the E <= 256 router logits (8 per lane),
// then top_k rounds of a warp argmax on (probability, -expert id); round k's
// winner is kept by lane k, so the selection stays in registers.
__global__ void __launch_bounds__(256) moe_topk_kernel(RouteParams p) {
  griddep_launch();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= p.M) return;  // whole warp
  float lv[8];
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    lv[j] = e < p.E ? p.logits[(size_t)t * p.E + e] : -INFINITY;
    m = fmaxf(m, lv[j]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float ev[8], sum = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    ev[j] = (lane + 32 * j < p.E) ? expf(lv[j] - m) : 0.f;
    sum += ev[j];
  }
  sum = warp_sum(sum);
  const float inv = 1.f / sum;
  unsigned taken = 0u;
  float my_p = 0.f;
  int my_e = 0;
#pragma unroll
  for (int k = 0; k < kMaxTopK; ++k) {
    if (k >= p.topk) break;  // uniform
    float bv = -1.f;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      const float pv = ev[j] * inv;
      if (!(taken >> j & 1u) && e < p.E && (pv > bv || (pv == bv && e < bi))) {
        bv = pv;
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == k) {
      my_p = bv;
      my_e = bi;
    }
  }
  const float psum = warp_sum(lane < p.topk ? my_p : 0.f);
  if (lane < p.topk) {
    p.gate[(size_t)t * p.topk + lane] = my_p / psum;
    p.sel[(size_t)t * p.topk + lane] = my_e;
  }
}

// One block of 1024 threads: per-expert counts, row offsets (shared experts
// last), and for each expert its (token, slot) pairs in token order, one warp
// per expert (ballot + popc over 32-token chunks).
__global__ void __launch_bounds__(1024) moe_group_kernel(RouteParams p) {
  griddep_launch();
  griddep_wait();
  __shared__ int s_cnt[kMaxE];
  __shared__ int s_off[kMaxE + 3];
  __shared__ unsigned char s_sel[kMaxPairs];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int npairs = p.M * p.topk;
  for (int i = threadIdx.x; i < p.E; i += blockDim.x) s_cnt[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < npairs; i += blockDim.x) {
    const int e = p.sel[i];
    s_sel[i] = (unsigned char)e;
    atomicAdd(&s_cnt[e], 1);
  }
  __syncthreads();
  if (warp == 0) {  // exclusive prefix over the experts, 32 at a time
    int base = 0;
    for (int e0 = 0; e0 < p.E; e0 += 32) {
      const int c = (e0 + lane < p.E) ? s_cnt[e0 + lane] : 0;
      int x = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (e0 + lane < p.E) s_off[e0 + lane] = base + x - c;
      base += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) {
      for (int sh = 0; sh < p.nsh; ++sh) s_off[p.E + sh] = base + sh * p.M;
      s_off[p.E + p.nsh] = base + p.nsh * p.M;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i <= p.E + p.nsh; i += blockDim.x) p.off[i] = s_off[i];
  const int width = p.topk + p.nsh;
  for (int e = warp; e < p.E; e += nw) {
    int base = s_off[e];
    for (int t0 = 0; t0 < p.M; t0 += 32) {
      const int t = t0 + lane;
      int slot = -1;
      if (t < p.M)
        for (int k = 0; k < p.topk; ++k)
          if (s_sel[t * p.topk + k] == e) slot = k;
      const unsigned bal = __ballot_sync(0xffffffffu, slot >= 0);
      if (slot >= 0) {
        const int r = base + __popc(bal & ((1u << lane) - 1u));
        p.pos[(size_t)t * width + slot] = r;
        p.pair_tok[r] = t;
      }
      base += __popc(bal);
    }
  }
  for (int i = threadIdx.x; i < p.M * p.nsh; i += blockDim.x) {
    const int sh = i / p.M, t = i % p.M;
    const int r = s_off[p.E + sh] + t;
    p.pos[(size_t)t * width + p.topk + sh] = r;
    p.pair_tok[r] = t;
  }
}

// Xg[row] = Hs[pair_tok[row]] (16-byte vector copies).
__global__ void moe_gather_kernel(const __nv_bfloat16* __restrict__ Hs, const int* __restrict__ pair_tok,
                                  __nv_bfloat16* __restrict__ Xg, int d) {
  griddep_launch();
  griddep_wait();
  const int r = blockIdx.x;
  const uint4* src = reinterpret_cast<const uint4*>(Hs + (size_t)pair_tok[r] * d);
  uint4* dst = reinterpret_cast<uint4*>(Xg + (size_t)r * d);
  for (int i = threadIdx.x; i < d / 8; i += blockDim.x) dst[i] = src[i];
}

// ---------------------------------------------------------------- expert GEMMs
constexpr int kThreads = 192;  // TMA warp, MMA warp, 4 epilogue warps
constexpr int kATile = 128 * 128;  // 128 weight rows x 64 K (bf16) = 16 KB
constexpr int kBox = 32;           // token rows per B box
constexpr int kBBytes = 256 * 128; // up to 256 token rows x 64 K
constexpr int kStageBytes = 2 * kATile + kBBytes;  // 64 KB
constexpr int kStages = 3;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 256;

struct FfnMaps {
  CUtensorMap a0;  // gate/up: W_gate [E+nsh][I][d] (box 128 rows); down: W_down [E+nsh][d][I] (box 256 rows)
  CUtensorMap a1;  // gate/up: W_up (box 128 rows); unused by down
  CUtensorMap b;   // gate/up: Xg [R][d]; down: act [R][I]                          (2D, box 32 rows)
};

struct FfnParams {
  const int* off;      // [E + nsh + 1]
  int K;               // contraction: d (gate/up) or I (down)
  int rows;            // weight rows: I (gate/up) or d (down)
  __nv_bfloat16* act;  // gate/up output [R][I]
  float* y;            // down output [R][d]
  const float* sw0;    // e4m3: row scales of W_gate (gate/up) or W_down (down), [E+nsh][rows]
  const float* sw1;    // e4m3: row scales of W_up (gate/up)
  const float* sx;     // e4m3: token row scales, [R]
  int* err;
};

__device__ __forceinline__ float gelu_erf(float x) { return 0.5f * x * (1.f + erff(x * 0.70710678118654752f)); }

// CTA (weight tile rt, expert e); two 128 x N accumulators in TMEM, fed per
// K block by the same B (the expert's token rows). MODE 0: a 128-row tile of
// W_gate and of W_up, GeGLU epilogue to act. MODE 1: a 256-row tile of W_down
// (one box) as two 128-row halves, f32 y.
template <int MODE, bool FP8>
__global__ void __launch_bounds__(kThreads, 1) moe_ffn_kernel(const __grid_constant__ FfnMaps maps, FfnParams p) {
  constexpr int kBK = FP8 ? 128 : 64;  // K elements per 128-byte block
  griddep_launch();
  griddep_wait();  // the routing offsets and the B rows come from the previous kernels
  const int e = blockIdx.y, rt = blockIdx.x;
  const int r0 = p.off[e];
  const int n = p.off[e + 1] - r0;
  if (n <= 0) return;  // expert without tokens (uniform over the CTA)
  const int N = (n + 15) & ~15;
  const int nbox = (n + kBox - 1) / kBox;
  const int nk = (p.K + kBK - 1) / kBK;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t kCols = 512;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t polW = policy_evict_first();
      const uint64_t polX = policy_evict_last();
      const uint32_t bytes = 2 * kATile + nbox * kBox * 128;
      int s = 0;
      uint32_t ph = 0;
      bool issued[kStages] = {false, false, false};
      uint32_t iph[kStages] = {0, 0, 0};
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(&empty[s], ph ^ 1u, p.err, abort_flag)) break;
        uint8_t* st = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&full[s], bytes);
        if (MODE == 0) {
          tma_load_3d(st, &maps.a0, &full[s], kb * kBK, rt * 128, e, polW);
          tma_load_3d(st + kATile, &maps.a1, &full[s], kb * kBK, rt * 128, e, polW);
        } else {
          tma_load_3d(st, &maps.a0, &full[s], kb * kBK, rt * 256, e, polW);  // 256 rows = both halves
        }
        for (int bx = 0; bx < nbox; ++bx)
          tma_load_2d(st + 2 * kATile + bx * kBox * 128, &maps.b, &full[s], kb * kBK, r0 + bx * kBox, polX);
        issued[s] = true;
        iph[s] = ph;
        if (++s == kStages) { s = 0; ph ^= 1u; }
      }
      if (*abort_flag)
        for (int i = 0; i < kStages; ++i)
          if (issued[i]) mbar_wait(&full[i], iph[i], p.err, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = FP8 ? idesc_e4m3_f32(128, N) : idesc_bf16_f32(128, N);
      int s = 0;
      uint32_t ph = 0;
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(&full[s], ph, p.err, abort_flag)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + s * kStageBytes);
        const uint32_t b0 = a0 + 2 * kATile;
#pragma unroll
        for (int k = 0; k < 4; ++k) {  // 32 bytes of K per instruction
          const uint64_t bd = umma_desc_sw128(b0 + k * 32, 16, 1024);
          if constexpr (FP8) {
            mma_f8_ss(tmem, umma_desc_sw128(a0 + k * 32, 16, 1024), bd, idesc, (kb | k) != 0);
            mma_f8_ss(tmem + 256, umma_desc_sw128(a0 + kATile + k * 32, 16, 1024), bd, idesc, (kb | k) != 0);
          } else {
            mma_bf16_ss(tmem, umma_desc_sw128(a0 + k * 32, 16, 1024), bd, idesc, (kb | k) != 0);
            mma_bf16_ss(tmem + 256, umma_desc_sw128(a0 + kATile + k * 32, 16, 1024), bd, idesc, (kb | k) != 0);
          }
        }
        mma_commit(&empty[s]);
        if (++s == kStages) { s = 0; ph ^= 1u; }
      }
      mma_commit(tfull);
    }
  } else {
    const int quad = warp & 3;
    // weight row: I index (MODE 0) or d index of the first half (MODE 1)
    const int row = rt * (MODE == 0 ? 128 : 256) + quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const bool ok = mbar_wait_warp(tfull, 0, p.err, abort_flag);
    tc_fence_after();
    // e4m3: this thread's weight-row scales (both halves of a down tile)
    float ws0 = 1.f, ws1 = 1.f;
    if (FP8 && ok) {
      const size_t base = (size_t)e * p.rows;
      if (row < p.rows) ws0 = p.sw0[base + row];
      if (MODE == 0 && row < p.rows) ws1 = p.sw1[base + row];
      if (MODE == 1 && row + 128 < p.rows) ws1 = p.sw0[base + row + 128];
    }
    if (ok) {
      for (int c = 0; c < (n + 31) / 32; ++c) {
        uint32_t g[32];
        tmem_ld32_sync(tmem + lane_off + c * 32, g);
        if (MODE == 0) {
          uint32_t u[32];
          tmem_ld32_sync(tmem + lane_off + 256 + c * 32, u);
          if (row < p.rows) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int tok = c * 32 + j;
              if (tok < n) {
                float gv = __uint_as_float(g[j]), uv = __uint_as_float(u[j]);
                if constexpr (FP8) {
                  const float sx = __ldg(p.sx + r0 + tok);
                  gv *= ws0 * sx;
                  uv *= ws1 * sx;
                }
                const float a = gelu_erf(gv) * uv;
                p.act[(size_t)(r0 + tok) * p.rows + row] = __float2bfloat16_rn(a);
              }
            }
          }
        } else {
          uint32_t g1[32];
          tmem_ld32_sync(tmem + lane_off + 256 + c * 32, g1);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int tok = c * 32 + j;
            const float sx = (FP8 && tok < n) ? __ldg(p.sx + r0 + tok) : 1.f;
            if (tok < n && row < p.rows) p.y[(size_t)(r0 + tok) * p.rows + row] = __uint_as_float(g[j]) * (ws0 * sx);
            if (tok < n && row + 128 < p.rows)
              p.y[(size_t)(r0 + tok) * p.rows + row + 128] = __uint_as_float(g1[j]) * (ws1 * sx);
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

// Hs2[t] = bf16(Hs[t] + sum_k gate[t][k] y[pos[t][k]] + sum_sh y[pos[t][topk+sh]]),
// accumulated in f32 in slot order. One block per token, 8 columns per thread.
__global__ void moe_combine_kernel(const __nv_bfloat16* __restrict__ Hs, const float* __restrict__ y,
                                   const int* __restrict__ pos, const float* __restrict__ gate,
                                   __nv_bfloat16* __restrict__ out, int d, int topk, int nsh) {
  griddep_launch();
  griddep_wait();
  const int t = blockIdx.x;
  __shared__ int s_pos[kMaxTopK + 4];
  __shared__ float s_g[kMaxTopK];
  const int width = topk + nsh;
  if (threadIdx.x < width) s_pos[threadIdx.x] = pos[(size_t)t * width + threadIdx.x];
  if (threadIdx.x < topk) s_g[threadIdx.x] = gate[(size_t)t * topk + threadIdx.x];
  __syncthreads();
  for (int c = threadIdx.x; c < d / 8; c += blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int k = 0; k < width; ++k) {
      const float gk = k < topk ? s_g[k] : 1.f;
      const float4* yr = reinterpret_cast<const float4*>(y + (size_t)s_pos[k] * d + c * 8);
      const float4 a = yr[0], b = yr[1];
      acc[0] = fmaf(gk, a.x, acc[0]); acc[1] = fmaf(gk, a.y, acc[1]);
      acc[2] = fmaf(gk, a.z, acc[2]); acc[3] = fmaf(gk, a.w, acc[3]);
      acc[4] = fmaf(gk, b.x, acc[4]); acc[5] = fmaf(gk, b.y, acc[5]);
      acc[6] = fmaf(gk, b.z, acc[6]); acc[7] = fmaf(gk, b.w, acc[7]);
    }
    const uint4 hu = reinterpret_cast<const uint4*>(Hs + (size_t)t * d)[c];
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hu);
    uint4 w;
    __nv_bfloat162* w2 = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 h = __bfloat1622float2(h2[j]);
      w2[j] = __floats2bfloat162_rn(h.x + acc[2 * j], h.y + acc[2 * j + 1]);
    }
    reinterpret_cast<uint4*>(out + (size_t)t * d)[c] = w;
  }
}

}  // namespace moe

// ---------------------------------------------------------------- host side
size_t moe_workspace_bytes(const MoeShape& s) {
  const size_t R = (size_t)s.M * (s.topk + s.nsh);
  auto al = [](size_t b) { return (b + 255) & ~size_t(255); };
  return al(sizeof(float) * s.M * s.E) + al(sizeof(float) * s.M * s.topk) + al(sizeof(int) * s.M * s.topk) +
         al(sizeof(int) * s.M * (s.topk + s.nsh)) +
         al(sizeof(int) * (s.E + s.nsh + 1)) + al(sizeof(int) * R) + al(2 * R * s.d) + al(2 * R * s.I) +
         al(4 * R * s.d) + (s.fp8 ? al(R * s.d) + al(R * s.I) + 2 * al(4 * R) : 0) + 12 * 256;
}

bool moe_prepare(MoeTc* mt, const MoeShape& s, const void* hs, void* hs_out, const void* w_router, const void* w_gate,
                 const void* w_up, const void* w_down, void* ws, int sm_count, const float* const* w_scales) {
  if (s.E > moe::kMaxE || s.topk > moe::kMaxTopK || s.M * s.topk > moe::kMaxPairs || s.nsh < 0 || s.nsh > 2 ||
      s.I % 64 != 0 || s.d % 64 != 0 || (s.fp8 && s.d % 128 != 0)) {
    set_last_error("MoE: unsupported sizes (E <= 256, top_k <= 8, M*top_k <= 8192, n_shared <= 2, "
                   "moe_inter and d_model multiples of 64, d_model a multiple of 128 with e4m3 experts)");
    return false;
  }
  for (auto f : {(const void*)moe::moe_ffn_kernel<0, false>, (const void*)moe::moe_ffn_kernel<1, false>,
                 (const void*)moe::moe_ffn_kernel<0, true>, (const void*)moe::moe_ffn_kernel<1, true>})
    if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, moe::kSmemBytes) != cudaSuccess) {
      set_last_error("cudaFuncSetAttribute(moe_ffn_kernel) failed");
      return false;
    }
  mt->s = s;
  mt->hs = hs;
  mt->hs_out = hs_out;
  const size_t R = (size_t)s.M * (s.topk + s.nsh);
  char* w = static_cast<char*>(ws);
  auto take = [&](size_t b) {
    char* q = w;
    w += (b + 255) & ~size_t(255);
    return q;
  };
  mt->logits = reinterpret_cast<float*>(take(sizeof(float) * s.M * s.E));
  mt->gate = reinterpret_cast<float*>(take(sizeof(float) * s.M * s.topk));
  mt->sel = reinterpret_cast<int*>(take(sizeof(int) * s.M * s.topk));
  mt->pos = reinterpret_cast<int*>(take(sizeof(int) * s.M * (s.topk + s.nsh)));
  mt->off = reinterpret_cast<int*>(take(sizeof(int) * (s.E + s.nsh + 1)));
  mt->pair_tok = reinterpret_cast<int*>(take(sizeof(int) * R));
  mt->xg = take(2 * R * s.d);
  mt->act = take(2 * R * s.I);
  mt->y = reinterpret_cast<float*>(take(4 * R * s.d));
  if (s.fp8) {
    mt->xg8 = reinterpret_cast<uint8_t*>(take(R * s.d));
    mt->act8 = reinterpret_cast<uint8_t*>(take(R * s.I));
    mt->sx = reinterpret_cast<float*>(take(4 * R));
    mt->sa = reinterpret_cast<float*>(take(4 * R));
    for (int i = 0; i < 3; ++i) mt->w_scale[i] = w_scales[i];
  }
  // router: f32 logits, one K split (no partial buffer needed)
  const void* wr[1] = {w_router};
  void* lo[1] = {mt->logits};
  const int ne[1] = {s.E};
  if (!gemm_tc_prepare_with(&mt->router, hs, s.M, s.d, 1, wr, lo, ne, 32, 1)) return false;
  mt->router.out_f32 = 1;
  (void)sm_count;
  // expert tensor maps
  moe::FfnMaps* gu = reinterpret_cast<moe::FfnMaps*>(mt->maps_gateup);
  moe::FfnMaps* dn = reinterpret_cast<moe::FfnMaps*>(mt->maps_down);
  static_assert(sizeof(moe::FfnMaps) <= sizeof(mt->maps_gateup), "MoeTc map storage too small");
  const uint64_t ne_tot = (uint64_t)s.E + s.nsh;
  const uint64_t dgu[3] = {(uint64_t)s.d, (uint64_t)s.I, ne_tot};
  const uint64_t sgu[2] = {(uint64_t)s.d * 2, (uint64_t)s.I * s.d * 2};
  const uint64_t ddn[3] = {(uint64_t)s.I, (uint64_t)s.d, ne_tot};
  const uint64_t sdn[2] = {(uint64_t)s.I * 2, (uint64_t)s.d * s.I * 2};
  const uint32_t bw[3] = {64, 128, 1};
  const uint32_t bw_dn[3] = {64, 256, 1};
  const uint64_t dx[2] = {(uint64_t)s.d, R}, sx[1] = {(uint64_t)s.d * 2};
  const uint64_t da[2] = {(uint64_t)s.I, R}, sa[1] = {(uint64_t)s.I * 2};
  const uint32_t bb[2] = {64, (uint32_t)moe::kBox};
  if (s.fp8) {  // e4m3 codes: one byte per element, 128-byte K boxes
    const uint64_t sgu8[2] = {(uint64_t)s.d, (uint64_t)s.I * s.d};
    const uint64_t sdn8[2] = {(uint64_t)s.I, (uint64_t)s.d * s.I};
    const uint32_t bw8[3] = {128, 128, 1};
    const uint32_t bw_dn8[3] = {128, 256, 1};
    const uint64_t sx8[1] = {(uint64_t)s.d}, sa8[1] = {(uint64_t)s.I};
    const uint32_t bb8[2] = {128, (uint32_t)moe::kBox};
    return encode_tmap_u8(&gu->a0, w_gate, 3, dgu, sgu8, bw8, true) &&
           encode_tmap_u8(&gu->a1, w_up, 3, dgu, sgu8, bw8, true) &&
           encode_tmap_u8(&gu->b, mt->xg8, 2, dx, sx8, bb8, true) &&
           encode_tmap_u8(&dn->a0, w_down, 3, ddn, sdn8, bw_dn8, true) &&
           encode_tmap_u8(&dn->a1, w_down, 3, ddn, sdn8, bw_dn8, true) &&
           encode_tmap_u8(&dn->b, mt->act8, 2, da, sa8, bb8, true);
  }
  if (!encode_tmap_bf16(&gu->a0, w_gate, 3, dgu, sgu, bw, true) || !encode_tmap_bf16(&gu->a1, w_up, 3, dgu, sgu, bw, true) ||
      !encode_tmap_bf16(&gu->b, mt->xg, 2, dx, sx, bb, true) || !encode_tmap_bf16(&dn->a0, w_down, 3, ddn, sdn, bw_dn, true) ||
      !encode_tmap_bf16(&dn->a1, w_down, 3, ddn, sdn, bw_dn, true) || !encode_tmap_bf16(&dn->b, mt->act, 2, da, sa, bb, true))
    return false;
  return true;
}

void launch_moe(Exec& ex, const MoeTc& mt) {
  const MoeShape& s = mt.s;
  launch_gemm_tc(ex, mt.router, nullptr);
  moe::RouteParams rp;
  rp.logits = mt.logits;
  rp.M = s.M;
  rp.E = s.E;
  rp.topk = s.topk;
  rp.nsh = s.nsh;
  rp.gate = mt.gate;
  rp.sel = mt.sel;
  rp.pos = mt.pos;
  rp.off = mt.off;
  rp.pair_tok = mt.pair_tok;
  launch_pdl(moe::moe_topk_kernel, dim3(ceil_div(s.M, 8)), dim3(256), 0, ex.stream, rp);
  launch_pdl(moe::moe_group_kernel, dim3(1), dim3(1024), 0, ex.stream, rp);
  const int R = s.M * (s.topk + s.nsh);
  launch_pdl(moe::moe_gather_kernel, dim3(R), dim3(128), 0, ex.stream, static_cast<const __nv_bfloat16*>(mt.hs),
             (const int*)mt.pair_tok, static_cast<__nv_bfloat16*>(mt.xg), s.d);
  moe::FfnParams fp;
  fp.off = mt.off;
  fp.err = ex.err;
  fp.act = static_cast<__nv_bfloat16*>(mt.act);
  fp.y = mt.y;
  fp.K = s.d;
  fp.rows = s.I;
  fp.sw0 = mt.w_scale[0];
  fp.sw1 = mt.w_scale[1];
  fp.sx = mt.sx;
  const dim3 g_gu(ceil_div(s.I, 128), s.E + s.nsh), g_dn(ceil_div(s.d, 256), s.E + s.nsh);
  const moe::FfnMaps& m_gu = *reinterpret_cast<const moe::FfnMaps*>(mt.maps_gateup);
  const moe::FfnMaps& m_dn = *reinterpret_cast<const moe::FfnMaps*>(mt.maps_down);
  if (s.fp8) {
    launch_quantize_rows_e4m3(ex, mt.xg, mt.xg8, mt.sx, R, s.d);
    launch_pdl(moe::moe_ffn_kernel<0, true>, g_gu, dim3(moe::kThreads), moe::kSmemBytes, ex.stream, m_gu, fp);
    launch_quantize_rows_e4m3(ex, mt.act, mt.act8, mt.sa, R, s.I);
  } else {
    launch_pdl(moe::moe_ffn_kernel<0, false>, g_gu, dim3(moe::kThreads), moe::kSmemBytes, ex.stream, m_gu, fp);
  }
  fp.K = s.I;
  fp.rows = s.d;
  fp.sw0 = mt.w_scale[2];
  fp.sw1 = nullptr;
  fp.sx = mt.sa;
  if (s.fp8)
    launch_pdl(moe::moe_ffn_kernel<1, true>, g_dn, dim3(moe::kThreads), moe::kSmemBytes, ex.stream, m_dn, fp);
  else
    launch_pdl(moe::moe_ffn_kernel<1, false>, g_dn, dim3(moe::kThreads), moe::kSmemBytes, ex.stream, m_dn, fp);
  launch_pdl(moe::moe_combine_kernel, dim3(s.M), dim3(256), 0, ex.stream, static_cast<const __nv_bfloat16*>(mt.hs),
             (const float*)mt.y, (const int*)mt.pos, (const float*)mt.gate, static_cast<__nv_bfloat16*>(mt.hs_out), s.d,
             s.topk, s.nsh);
  ex.launches += 6;
}

}  // namespace dg
