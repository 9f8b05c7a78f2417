// Projection GEMM on the 5th-generation tensor cores: out = A W^T (+ R), bf16
// in, f32 accumulate in TMEM, one rounding to bf16. Used for the Q / canvas K
// / canvas V projections (one launch, three output segments: the canvas's own
// K/V are recomputed every step, "DiffusionGemma深度拆解：从逐字蹦到整块喷，LLM生成范式
// 的结构性跃迁", 架构解剖 2) and for the output projection with the residual.
//
// CTA tile: up to 256 rows (two 128-row halves) x 64 output columns, full K.
// K-loop of 64-wide blocks through a 5-stage TMA pipeline (A 32 KB + B 8 KB per
// stage). Warp 0 issues TMA, warp 1 allocates TMEM and issues the MMAs
// (M=128, N=64, K=16) into two accumulators, warps 2..9 drain TMEM (warp w reads
// lanes 32*(w%4) of half (w-2)/4), add the residual, round and store.
#include "dg_internal.cuh"
#include "dg_sm100.cuh"
#include "dg_tmap.cuh"

namespace dg {
namespace gemmtc {

using namespace sm100;

constexpr int kStages = 5;
constexpr int kBK = 64;
constexpr int kBN = 64;
constexpr int kHalfBytes = 128 * 128;           // 128 rows x 128 B
constexpr int kABytes = 2 * kHalfBytes;         // 32 KB
constexpr int kBBytes = kBN * 128;              // 8 KB
constexpr int kStageBytes = kABytes + kBBytes;  // 40 KB
constexpr int kThreads = 320;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 256;

struct Seg {
  __nv_bfloat16* out;  // [M][ldo]
  int ldo;             // row stride of out (elements) = N of this segment
  int tiles;           // number of 64-column tiles in this segment
};

struct Params {
  int M, K;
  int nseg;
  Seg seg[3];
  const __nv_bfloat16* R;  // residual [M][ldo of segment 0] or null (single-segment use)
  int* err;
};

struct Maps {
  CUtensorMap a;
  CUtensorMap b[3];
};

__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ Maps maps, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * 256;
  const int halves = (p.M - m0 > 128) ? 2 : 1;
  // output segment of this column tile
  int seg = 0, t = blockIdx.x;
  while (seg + 1 < p.nseg && t >= p.seg[seg].tiles) t -= p.seg[seg++].tiles;
  const int n0 = t * kBN;
  const CUtensorMap* mapB = &maps.b[seg];
  const int nk = p.K / kBK;

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
    tmem_alloc(tmem_holder, 128);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.a);
    tma_prefetch_desc(mapB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t polA = policy_evict_last();
      const uint64_t polB = policy_evict_first();
      const uint32_t bytes = halves * kHalfBytes + kBBytes;
      int s = 0;
      uint32_t ph = 0;
      bool issued[kStages];
      uint32_t issued_ph[kStages];
      for (int i = 0; i < kStages; ++i) issued[i] = false, issued_ph[i] = 0;
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(&empty[s], ph ^ 1u, p.err, abort_flag)) break;
        uint8_t* st = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&full[s], bytes);
        for (int h = 0; h < halves; ++h) tma_load_2d(st + h * kHalfBytes, &maps.a, &full[s], kb * kBK, m0 + h * 128, polA);
        tma_load_2d(st + kABytes, mapB, &full[s], kb * kBK, n0, polB);
        issued[s] = true;
        issued_ph[s] = ph;
        if (++s == kStages) { s = 0; ph ^= 1u; }
      }
      if (*abort_flag)
        for (int i = 0; i < kStages; ++i)
          if (issued[i]) mbar_wait(&full[i], issued_ph[i], p.err, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, kBN);
      int s = 0;
      uint32_t ph = 0;
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(&full[s], ph, p.err, abort_flag)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + s * kStageBytes);
        const uint32_t b0 = a0 + kABytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h < halves) {
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
              mma_bf16_ss(tmem + h * kBN, umma_desc_sw128(a0 + h * kHalfBytes + k * 32, 16, 1024),
                          umma_desc_sw128(b0 + k * 32, 16, 1024), idesc, (kb | k) != 0);
          }
        }
        mma_commit(&empty[s]);
        if (++s == kStages) { s = 0; ph ^= 1u; }
      }
      mma_commit(tfull);  // also covers every MMA above before TMEM is read or freed
    }
  } else {
    const int ew = warp - 2;
    const int half = ew >> 2;
    const int quad = warp & 3;
    const int row = m0 + half * 128 + quad * 32 + lane;
    const bool ok = mbar_wait(tfull, 0, p.err, abort_flag);
    tc_fence_after();
    if (ok && half < halves) {
      const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(half * kBN);
      uint32_t r0[32], r1[32];
      tmem_ld32_sync(tbase, r0);
      tmem_ld32_sync(tbase + 32, r1);
      if (row < p.M) {
        const Seg sg = p.seg[seg];
        __nv_bfloat16* dst = sg.out + (size_t)row * sg.ldo + n0;
        float v[64];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          v[i] = __uint_as_float(r0[i]);
          v[32 + i] = __uint_as_float(r1[i]);
        }
        if (p.R) {
          const uint4* rs = reinterpret_cast<const uint4*>(p.R + (size_t)row * sg.ldo + n0);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4 u = rs[c];
            const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 f = __bfloat1622float2(b2[j]);
              v[c * 8 + 2 * j] += f.x;
              v[c * 8 + 2 * j + 1] += f.y;
            }
          }
        }
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 u;
          __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
          for (int j = 0; j < 4; ++j) b2[j] = __floats2bfloat162_rn(v[c * 8 + 2 * j], v[c * 8 + 2 * j + 1]);
          d4[c] = u;
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace gemmtc

// ---------------------------------------------------------------- host side
bool gemm_tc_prepare(GemmTc* g, const void* A, int M, int K, int nseg, const void* const* W, void* const* out,
                     const int* N) {
  if (cudaFuncSetAttribute(gemmtc::gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gemmtc::kSmemBytes) != cudaSuccess) {
    set_last_error("cudaFuncSetAttribute(gemm_tc_kernel) failed");
    return false;
  }
  if (nseg < 1 || nseg > 3 || K % 64 != 0) {
    set_last_error("gemm_tc: unsupported shape");
    return false;
  }
  static_assert(sizeof(gemmtc::Maps) <= sizeof(g->maps), "GemmTc map storage too small");
  gemmtc::Maps* maps = reinterpret_cast<gemmtc::Maps*>(g->maps);
  const uint64_t dA[2] = {(uint64_t)K, (uint64_t)M};
  const uint64_t sA[1] = {(uint64_t)K * 2};
  const uint32_t bA[2] = {64, 128};
  if (!encode_tmap_bf16(&maps->a, A, 2, dA, sA, bA, true)) return false;
  g->M = M;
  g->K = K;
  g->nseg = nseg;
  g->tiles = 0;
  for (int i = 0; i < nseg; ++i) {
    if (N[i] % gemmtc::kBN != 0) {
      set_last_error("gemm_tc: N must be a multiple of 64");
      return false;
    }
    const uint64_t dB[2] = {(uint64_t)K, (uint64_t)N[i]};
    const uint32_t bB[2] = {64, (uint32_t)gemmtc::kBN};
    if (!encode_tmap_bf16(&maps->b[i], W[i], 2, dB, sA, bB, true)) return false;
    g->out[i] = out[i];
    g->N[i] = N[i];
    g->tiles += N[i] / gemmtc::kBN;
  }
  return true;
}

void launch_gemm_tc(Exec& ex, const GemmTc& g, const void* residual) {
  gemmtc::Params p;
  p.M = g.M;
  p.K = g.K;
  p.nseg = g.nseg;
  for (int i = 0; i < 3; ++i) {
    p.seg[i].out = i < g.nseg ? static_cast<__nv_bfloat16*>(g.out[i]) : nullptr;
    p.seg[i].ldo = i < g.nseg ? g.N[i] : 0;
    p.seg[i].tiles = i < g.nseg ? g.N[i] / gemmtc::kBN : 0;
  }
  p.R = static_cast<const __nv_bfloat16*>(residual);
  p.err = ex.err;
  dim3 grid(g.tiles, ceil_div(g.M, 256));
  gemmtc::gemm_tc_kernel<<<grid, gemmtc::kThreads, gemmtc::kSmemBytes, ex.stream>>>(
      *reinterpret_cast<const gemmtc::Maps*>(g.maps), p);
  ex.launches++;
}

}  // namespace dg
