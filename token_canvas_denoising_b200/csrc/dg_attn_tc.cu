// Bidirectional GQA canvas attention on the 5th-generation tensor cores.
//
// Method: every canvas position attends to every other canvas position (no
// triangular mask) and to the prompt's cached K/V ("DiffusionGemma解析：扩散模型如何
// 让LLM快5倍", 整片并行去噪, last paragraph; "DiffusionGemma深度拆解：从逐字蹦到整块喷，
// LLM生成范式的结构性跃迁", 架构解剖 2 and the encoder/decoder diagram); the canvas's
// own K/V are recomputed every step (架构解剖 2). Per query head q (KV head
// g = q / (Hq/Hk)): O = softmax(Q K^T / sqrt(h)) V over [prefix keys; canvas keys].
//
// CTA work item: (request b, query head q, 128-query tile, KV split). The KV
// sequence is walked in 128-key tiles (prefix tiles from the request's own
// tensor map, then canvas tiles) through 3-slot TMA rings for K and for V.
//   warp 0   : TMA producer: Q once; K tiles one ahead of V tiles (a K slot
//              frees when its QK completes, a V slot when its PV does);
//              prompt-prefix tiles a few tiles ahead are prefetched into L2
//   warp 1   : TMEM allocator and MMA issuer: S_j = Q K_j^T (M=N=128, K=128)
//              into one of two TMEM score buffers, then O += P_j V_j (V as an
//              MN-major operand) into the TMEM output accumulator. Q and P are
//              A operands read from TMEM, so shared memory only feeds K and V
//              (the tile's operand traffic through shared memory halves).
//   warps 2-5: softmax, one query row per thread: copy the Q row from shared
//              memory into TMEM once; per tile read S_j from TMEM, mask the
//              keys past the tile's end, exponentiate in base 2 against a
//              running maximum, write P_j (bf16 pairs) into TMEM. The running
//              maximum is only raised when the tile's maximum exceeds it by
//              more than 8 (a factor 256), and then O and the running sum are
//              rescaled in place; otherwise the stale maximum is kept (the
//              result is the same ratio). The decision is per warp, since the
//              TMEM accesses are collective.
// TMEM columns: S0 [0,128) | S1 [128,256) | O [256,384) | Q [384,448) | P [448,512).
// With one split the rows are normalised and stored as bf16; with several,
// unnormalised O and (max, sum) go to a partial buffer for attn_merge_kernel.
#include <cstring>

#include "dg_internal.cuh"
#include "dg_sm100.cuh"
#include "dg_tmap.cuh"

namespace dg {
namespace attntc {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kTile = 128;
constexpr int kAtom = 128 * 128;       // 128 rows x 128 B = 16 KB
constexpr int kMatBytes = 2 * kAtom;   // a 128 x 128 bf16 tile = 32 KB
constexpr int kSlots = 3;              // K ring and V ring depth
// smem: Q | K0 K1 K2 | V0 V1 V2 | barriers. The dynamic shared window starts
// 1024-aligned (after the CTA's reserved 1 KB); the kernel checks this
// instead of reserving alignment slack.
constexpr int kOffQ = 0;
constexpr int kOffK = kMatBytes;
constexpr int kOffV = kOffK + kSlots * kMatBytes;
constexpr int kOffBar = kOffV + kSlots * kMatBytes;
constexpr int kSmemBytes = kOffBar + 256;
static_assert(kSmemBytes <= 232448, "attention tile exceeds the opt-in shared memory of a CTA");
constexpr int kMaxReq = 8;
constexpr float kRescaleThreshold = 8.f;  // log2 units
constexpr int kAhead = 4;                 // prompt-prefix tiles prefetched into L2 ahead of their load
constexpr uint32_t kColO = 256, kColQ = 384, kColP = 448;

struct Maps {
  CUtensorMap q;    // [B*C][Hq*h]
  CUtensorMap kc;   // [B*C][Hk*h]
  CUtensorMap vc;
  CUtensorMap pk[kMaxReq];  // [S_b][Hk*h] per request of this launch
  CUtensorMap pv[kMaxReq];
};

struct Params {
  int b0, nreq;  // requests [b0, b0 + nreq) in this launch
  int C, Hq, Hk;
  int S[kMaxReq];
  int q_tiles, splits;
  int rows_total;    // B_total * C * Hq (partial buffer row count)
  float scale_log2;  // log2(e) / sqrt(h)
  __nv_bfloat16* O;  // [B*C][Hq*h]
  float* part_o;     // [splits][rows_total][128]
  float* part_ml;    // [splits][rows_total][2]
  int* err;
};

__device__ __forceinline__ uint64_t kdesc(uint32_t base, int kk) {
  // K-major 128-row operand with 128 columns of K split into two 64-wide atoms
  return umma_desc_sw128(base + (kk >> 2) * kAtom + (kk & 3) * 32, 16, 1024);
}

__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ Maps maps, Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {  // SW128 tiles need 1024-byte alignment (uniform: no TMEM held yet)
    if (threadIdx.x == 0) set_error(p.err, kDevBadAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bar + 0;      // Q tile landed in shared memory
  uint64_t* q_tmem = bar + 1;      // Q copied into TMEM (4 softmax warps)
  uint64_t* k_full = bar + 2;      // [3]
  uint64_t* v_full = bar + 5;      // [3]
  uint64_t* k_empty = bar + 8;     // [3] QK_i done: K slot i % 3 free
  uint64_t* v_empty = bar + 11;    // [3] PV_i done: V slot i % 3 free
  uint64_t* s_full = bar + 14;     // [2] S_i in TMEM buffer i & 1
  uint64_t* s_free = bar + 16;     // [2] S buffer read by the softmax (4 warps)
  uint64_t* p_full = bar + 18;     // P_i in TMEM (4 warps)
  uint64_t* pv_done = bar + 19;    // PV_i complete: O stable, P columns free
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar + 20);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x % p.q_tiles;
  const int qh = blockIdx.x / p.q_tiles;
  const int lb = blockIdx.y;            // request within this launch
  const int b = p.b0 + lb;              // request index
  const int z = blockIdx.z;             // KV split
  const int g = qh / (p.Hq / p.Hk);
  const int S = p.S[lb];
  const int nps = (S + kTile - 1) / kTile;
  const int nct = (p.C + kTile - 1) / kTile;
  const int nt = nps + nct;
  const int t0 = (int)(((long long)z * nt) / p.splits);
  const int t1 = (int)(((long long)(z + 1) * nt) / p.splits);
  const int n = t1 - t0;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_tmem, 4);
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  griddep_launch();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      // tile i: K and V rows [y, y + 128) of the prompt prefix or of the canvas
      auto tile_src = [&](int i, const CUtensorMap*& mk, const CUtensorMap*& mv, int& y) {
        const int j = t0 + i;
        if (j < nps) {
          mk = &maps.pk[lb];
          mv = &maps.pv[lb];
          y = j * kTile;
        } else {
          mk = &maps.kc;
          mv = &maps.vc;
          y = b * p.C + (j - nps) * kTile;
        }
      };
      auto load_k = [&](int i) {
        const CUtensorMap *mk, *mv;
        int y;
        tile_src(i, mk, mv, y);
        uint8_t* kb = smem + kOffK + (i % kSlots) * kMatBytes;
        mbar_arrive_expect_tx(&k_full[i % kSlots], kMatBytes);
        tma_load_3d(kb, mk, &k_full[i % kSlots], 0, y, g * 2, pol);
      };
      auto load_v = [&](int i) {
        const CUtensorMap *mk, *mv;
        int y;
        tile_src(i, mk, mv, y);
        uint8_t* vb = smem + kOffV + (i % kSlots) * kMatBytes;
        mbar_arrive_expect_tx(&v_full[i % kSlots], kMatBytes);
        tma_load_3d(vb, mv, &v_full[i % kSlots], 0, y, g * 2, pol);
      };
      // prompt-prefix tiles further ahead are pulled into L2 early
      auto prefetch = [&](int i) {
        if (i < n && t0 + i < nps) {
          tma_prefetch_3d(&maps.pk[lb], 0, (t0 + i) * kTile, g * 2);
          tma_prefetch_3d(&maps.pv[lb], 0, (t0 + i) * kTile, g * 2);
        }
      };
      int nk = 0, nv = 0;  // next K tile and next V tile to load
      // the prompt prefix is an input of the step: its first tiles may be
      // fetched before the predecessor kernels are done
      while (nk < kSlots && nk < n && t0 + nk < nps) {
        load_k(nk);
        load_v(nk);
        ++nk;
        ++nv;
      }
      for (int i = nk; i < nk + kAhead; ++i) prefetch(i);
      griddep_wait();
      mbar_arrive_expect_tx(q_full, kMatBytes);
      tma_load_3d(smem + kOffQ, &maps.q, q_full, 0, b * p.C + qt * kTile, qh * 2, pol);
      // K runs one tile ahead of V
      while (nv < n && !*abort_flag) {
        if (nk < n && nk <= nv + 1) {
          if (nk >= kSlots && !mbar_wait(&k_empty[nk % kSlots], ((nk / kSlots) - 1) & 1, p.err, abort_flag)) break;
          load_k(nk);
          prefetch(nk + kAhead);
          ++nk;
        } else {
          if (nv >= kSlots && !mbar_wait(&v_empty[nv % kSlots], ((nv / kSlots) - 1) & 1, p.err, abort_flag)) break;
          load_v(nv);
          ++nv;
        }
      }
      if (*abort_flag) {  // drain this CTA's own copies: the last load of each slot
        mbar_wait(q_full, 0, p.err, nullptr);
        for (int i = nk - kSlots; i < nk; ++i)
          if (i >= 0) mbar_wait(&k_full[i % kSlots], (i / kSlots) & 1, p.err, nullptr);
        for (int i = nv - kSlots; i < nv; ++i)
          if (i >= 0) mbar_wait(&v_full[i % kSlots], (i / kSlots) & 1, p.err, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    griddep_wait();
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16_f32(128, 128, false);
      const uint32_t id_pv = idesc_bf16_f32(128, 128, true);
      bool ok = mbar_wait(q_tmem, 0, p.err, abort_flag);
      auto issue_qk = [&](int i) -> bool {
        const int s = i & 1, slot = i % kSlots;
        if (!mbar_wait(&k_full[slot], (i / kSlots) & 1, p.err, abort_flag)) return false;
        if (i >= 2 && !mbar_wait(&s_free[s], ((i >> 1) - 1) & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t kbase = smem_u32(smem + kOffK + slot * kMatBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + s * 128, tmem + kColQ + kk * 8, kdesc(kbase, kk), id_qk, kk != 0);
        mma_commit(&s_full[s]);
        mma_commit(&k_empty[slot]);
        return true;
      };
      if (ok && n > 0) ok = issue_qk(0);
      for (int i = 0; ok && i < n; ++i) {
        if (i + 1 < n && !(ok = issue_qk(i + 1))) break;
        const int slot = i % kSlots;
        if (!mbar_wait(p_full, i & 1, p.err, abort_flag)) break;
        if (!mbar_wait(&v_full[slot], (i / kSlots) & 1, p.err, abort_flag)) break;
        tc_fence_after();
        const uint32_t vbase = smem_u32(smem + kOffV + slot * kMatBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + kColO, tmem + kColP + kk * 8, umma_desc_sw128(vbase + kk * 2048, kAtom, 1024), id_pv,
                      (i | kk) != 0);
        mma_commit(pv_done);
        mma_commit(&v_empty[slot]);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    griddep_wait();
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // query row within the tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    float m_run = -INFINITY, l = 0.f;
    // Q row into TMEM columns [384, 448): 16-byte chunk c of swizzle atom a
    // holds head dims a*64 + c*8 .. +7, i.e. columns a*32 + c*4 .. +3
    bool ok = mbar_wait_warp(q_full, 0, p.err, abort_flag);
    if (ok) {
      const uint8_t* qrow = smem + kOffQ + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        uint32_t u[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(qrow + a * kAtom + ((c ^ (r & 7)) << 4));
          u[c * 4 + 0] = v.x;
          u[c * 4 + 1] = v.y;
          u[c * 4 + 2] = v.z;
          u[c * 4 + 3] = v.w;
        }
        tmem_st32(tmem + lane_off + kColQ + a * 32, u);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_tmem);
    }
    for (int i = 0; ok && i < n; ++i) {
      const int s = i & 1;
      if (!(ok = mbar_wait_warp(&s_full[s], (i >> 1) & 1, p.err, abort_flag))) break;
      tc_fence_after();
      float x[128];
      {
        uint32_t u[128];
        tmem_ld128_sync(tmem + lane_off + s * 128, u);
#pragma unroll
        for (int e = 0; e < 128; ++e) x[e] = __uint_as_float(u[e]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[s]);
      // keys of this tile that exist
      const int j = t0 + i;
      const int valid = (j < nps) ? min(kTile, S - j * kTile) : min(kTile, p.C - (j - nps) * kTile);
      if (valid < kTile) {  // ragged last tile (uniform over the CTA)
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) x[c] = -INFINITY;
      }
      // row maximum over 8 independent chains (short dependency chains)
      float mx[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) mx[c] = x[c];
#pragma unroll
      for (int c = 8; c < 128; ++c) mx[c & 7] = fmaxf(mx[c & 7], x[c]);
#pragma unroll
      for (int w = 4; w > 0; w >>= 1)
#pragma unroll
        for (int c = 0; c < w; ++c) mx[c] = fmaxf(mx[c], mx[c + w]);
      const float mt = mx[0] * p.scale_log2;  // the scale is positive: maximum of the scaled scores
      // The O rows live in TMEM and are rescaled with warp-collective
      // tcgen05.ld/st, so the decision is taken per warp: when any row of the
      // warp has outgrown its maximum by the threshold, every row of the warp
      // moves its maximum up to its tile maximum (alpha = 1 where it stays).
      const bool rescale = __any_sync(0xffffffffu, mt > m_run + kRescaleThreshold);
      float alpha = 1.f;
      if (rescale) {
        const float m_new = fmaxf(m_run, mt);
        alpha = ex2_approx(m_run - m_new);
        m_run = m_new;
      }
      // P = 2^(x scale - m_run) as bf16 pairs, row sum over 8 chains
      uint32_t pk[64];
      float ls[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const float neg_m = -m_run;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ex2_approx(fmaf(x[2 * c], p.scale_log2, neg_m));
        const float p1 = ex2_approx(fmaf(x[2 * c + 1], p.scale_log2, neg_m));
        ls[(2 * c) & 7] += p0;
        ls[(2 * c + 1) & 7] += p1;
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        pk[c] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      // PV_{i-1} complete: O holds it (for the rescale) and the P columns are free
      if (i > 0) {
        if (!(ok = mbar_wait_warp(pv_done, (i - 1) & 1, p.err, abort_flag))) break;
        tc_fence_after();
      }
      if (rescale && i > 0) {
        l *= alpha;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t u[32];
          tmem_ld32_sync(tmem + lane_off + kColO + c * 32, u);
#pragma unroll
          for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
          tmem_st32(tmem + lane_off + kColO + c * 32, u);
        }
      }
      l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      {
        uint32_t u[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) u[e] = pk[e];
        tmem_st32(tmem + lane_off + kColP, u);
#pragma unroll
        for (int e = 0; e < 32; ++e) u[e] = pk[32 + e];
        tmem_st32(tmem + lane_off + kColP + 32, u);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // ------------------------------------------------------------ epilogue
    if (ok && n > 0 && mbar_wait_warp(pv_done, (n - 1) & 1, p.err, abort_flag)) {
      tc_fence_after();
      const int qrow = qt * kTile + r;
      const bool has_row = qrow < p.C;
      const size_t grow = (size_t)(b * p.C + qrow);
      const float inv = 1.f / l;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t u[32];
        tmem_ld32_sync(tmem + lane_off + kColO + c * 32, u);
        if (!has_row) continue;
        if (p.splits == 1) {
          uint4* dst = reinterpret_cast<uint4*>(p.O + grow * p.Hq * 128 + qh * 128 + c * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w;
            __nv_bfloat162* w2 = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w2[e] = __floats2bfloat162_rn(__uint_as_float(u[v4 * 8 + 2 * e]) * inv,
                                            __uint_as_float(u[v4 * 8 + 2 * e + 1]) * inv);
            dst[v4] = w;
          }
        } else {
          const size_t prow_i = (size_t)z * p.rows_total + grow * p.Hq + qh;
          float4* dst = reinterpret_cast<float4*>(p.part_o + prow_i * 128 + c * 32);
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            dst[v4] = make_float4(__uint_as_float(u[4 * v4]), __uint_as_float(u[4 * v4 + 1]),
                                  __uint_as_float(u[4 * v4 + 2]), __uint_as_float(u[4 * v4 + 3]));
          if (c == 0) {
            p.part_ml[prow_i * 2] = m_run;
            p.part_ml[prow_i * 2 + 1] = l;
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Combine split partials: m = max m_z, w_z = 2^(m_z - m),
// O = sum_z w_z O_z / sum_z w_z l_z. One warp per (row, head), 4 dims per lane.
__global__ void attn_merge_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                                  __nv_bfloat16* __restrict__ O, int rows_total, int splits) {
  griddep_launch();
  griddep_wait();
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= rows_total) return;
  float m = -INFINITY;
  for (int z = 0; z < splits; ++z) m = fmaxf(m, part_ml[((size_t)z * rows_total + w) * 2]);
  float l = 0.f, o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
  for (int z = 0; z < splits; ++z) {
    const size_t rz = (size_t)z * rows_total + w;
    const float wz = ex2_approx(part_ml[rz * 2] - m);
    l += wz * part_ml[rz * 2 + 1];
    const float4 v = reinterpret_cast<const float4*>(part_o + rz * 128)[lane];
    o0 += wz * v.x;
    o1 += wz * v.y;
    o2 += wz * v.z;
    o3 += wz * v.w;
  }
  const float inv = 1.f / l;
  __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(O + (size_t)w * 128 + lane * 4);
  dst[0] = __floats2bfloat162_rn(o0 * inv, o1 * inv);
  dst[1] = __floats2bfloat162_rn(o2 * inv, o3 * inv);
}

}  // namespace attntc

// ---------------------------------------------------------------- host side
int attn_tc_splits(int B, int C, int Hq, const int* S, int sm_count) {
  const int q_tiles = ceil_div(C, 128);
  int min_tiles = 1 << 30;
  for (int b = 0; b < B; ++b) min_tiles = std::min(min_tiles, ceil_div(S[b], 128) + q_tiles);
  int splits = sm_count / std::max(1, B * Hq * q_tiles);
  splits = std::max(1, std::min(splits, std::min(min_tiles, 16)));
  return splits;
}

bool attn_tc_prepare(AttnTc* at, const AttnShape& sh, const void* Q, const void* Kc, const void* Vc,
                     const int32_t* S, const void* const* pk, const void* const* pv, void* O, float* part_o,
                     float* part_ml, int splits) {
  if (cudaFuncSetAttribute(attntc::attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           attntc::kSmemBytes) != cudaSuccess) {
    set_last_error("cudaFuncSetAttribute(attn_tc_kernel) failed");
    return false;
  }
  if (sh.h != 128) {
    set_last_error("attn_tc: head_dim must be 128");
    return false;
  }
  at->sh = sh;
  at->O = O;
  at->part_o = part_o;
  at->part_ml = part_ml;
  at->splits = splits;
  at->groups.clear();
  // [rows][heads * 128] bf16 as 3D (64 elements, rows, heads * 2): one box
  // (64, 128, 2) is a head's 128 x 128 tile as two 128-byte-swizzled halves
  const uint64_t rows = (uint64_t)sh.B * sh.C;
  const uint64_t dq[3] = {64, rows, (uint64_t)sh.Hq * 2}, sq[2] = {(uint64_t)sh.Hq * 256, 128};
  const uint64_t dk[3] = {64, rows, (uint64_t)sh.Hk * 2}, sk[2] = {(uint64_t)sh.Hk * 256, 128};
  const uint32_t box[3] = {64, 128, 2};
  for (int b0 = 0; b0 < sh.B; b0 += attntc::kMaxReq) {
    AttnTc::Group grp;
    grp.b0 = b0;
    grp.nreq = std::min(attntc::kMaxReq, sh.B - b0);
    static_assert(sizeof(attntc::Maps) <= sizeof(grp.maps), "AttnTc map storage too small");
    attntc::Maps* m = reinterpret_cast<attntc::Maps*>(grp.maps);
    memset(grp.maps, 0, sizeof(grp.maps));
    if (!encode_tmap_bf16(&m->q, Q, 3, dq, sq, box, true) || !encode_tmap_bf16(&m->kc, Kc, 3, dk, sk, box, true) ||
        !encode_tmap_bf16(&m->vc, Vc, 3, dk, sk, box, true))
      return false;
    for (int i = 0; i < grp.nreq; ++i) {
      const int b = b0 + i;
      grp.S[i] = S[b];
      if (S[b] > 0) {
        const uint64_t dp[3] = {64, (uint64_t)S[b], (uint64_t)sh.Hk * 2};
        if (!encode_tmap_bf16(&m->pk[i], pk[b], 3, dp, sk, box, true) ||
            !encode_tmap_bf16(&m->pv[i], pv[b], 3, dp, sk, box, true))
          return false;
      }
    }
    at->groups.push_back(grp);
  }
  return true;
}

void launch_attn_tc(Exec& ex, const AttnTc& at) {
  const AttnShape& sh = at.sh;
  const int q_tiles = ceil_div(sh.C, 128);
  const int rows_total = sh.B * sh.C * sh.Hq;
  for (const auto& grp : at.groups) {
    attntc::Params p;
    p.b0 = grp.b0;
    p.nreq = grp.nreq;
    p.C = sh.C;
    p.Hq = sh.Hq;
    p.Hk = sh.Hk;
    for (int i = 0; i < attntc::kMaxReq; ++i) p.S[i] = i < grp.nreq ? grp.S[i] : 0;
    p.q_tiles = q_tiles;
    p.splits = at.splits;
    p.rows_total = rows_total;
    p.scale_log2 = 1.4426950408889634f / sqrtf(128.f);
    p.O = static_cast<__nv_bfloat16*>(at.O);
    p.part_o = at.part_o;
    p.part_ml = at.part_ml;
    p.err = ex.err;
    dim3 grid(q_tiles * sh.Hq, grp.nreq, at.splits);
    launch_pdl(attntc::attn_tc_kernel, grid, dim3(attntc::kThreads), attntc::kSmemBytes, ex.stream,
               *reinterpret_cast<const attntc::Maps*>(grp.maps), p);
    ex.launches++;
  }
  if (at.splits > 1) {
    launch_pdl(attntc::attn_merge_kernel, dim3(ceil_div(rows_total, 8)), dim3(256), 0, ex.stream,
               (const float*)at.part_o, (const float*)at.part_ml, static_cast<__nv_bfloat16*>(at.O), rows_total,
               at.splits);
    ex.launches++;
  }
}

}  // namespace dg
