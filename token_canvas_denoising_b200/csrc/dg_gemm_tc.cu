// Projection GEMM on the 5th-generation tensor cores: out = A W^T (+ R), bf16
// in, f32 accumulate in TMEM, one rounding to bf16. Used for the Q / canvas K
// / canvas V projections (one launch, three output segments: the canvas's own
// K/V are recomputed every step, "DiffusionGemma深度拆解：从逐字蹦到整块喷，LLM生成范式
// 的结构性跃迁", 架构解剖 2) and for the output projection with the residual.
//
// CTA: 128 rows x BN (32..256) output columns x one K split. The canvas has
// only B*C rows and the activation block A is re-read by every column tile, so
// a 128-row tile keeps the bytes per K block small (16 KB of A + BN*128 B of W)
// while giving 2 CTAs per column tile for a 256-row canvas. The column tile is
// chosen so that about one CTA per SM is launched; K is split only when even
// 32-column tiles leave SMs idle. K-loop of 64-wide blocks through a TMA ring
// of ~200 KB; a stage holds KB consecutive K blocks of A and of W, each
// fetched by one 3D box (64 elements, rows, K blocks): a TMA stream is bounded
// by its per-box cost, so boxes are as large as the ring allows (KB = 4 for
// BN <= 64, 2 for 128, 1 for 256). Warp 0 issues TMA, warp 1 allocates TMEM and issues the MMAs
// (M=128, N=BN, K=16), warps 2..5 drain TMEM (warp w reads lanes 32*(w%4)).
// With one split they add the residual, round and store; with several, every
// CTA writes its f32 partial and a reduction kernel sums the partials in split
// order (the result does not depend on which CTA finishes first), adds the
// residual and stores.
#include "dg_internal.cuh"
#include "dg_sm100.cuh"
#include "dg_tmap.cuh"

namespace dg {
namespace gemmtc {

using namespace sm100;

constexpr int kBK = 64;
constexpr int kBM = 128;                        // rows per CTA
constexpr int kABytes = kBM * 128;              // 16 KB per 64-wide K block
constexpr int kThreads = 192;                   // TMA warp, MMA warp, 4 epilogue warps

__host__ __device__ constexpr int kblocks_per_stage(int bn) { return bn <= 64 ? 4 : (bn == 128 ? 2 : 1); }

template <int BN> struct Cfg {
  static constexpr int kKB = kblocks_per_stage(BN);   // K blocks per stage (one box each for A and W)
  static constexpr int kBBytes = BN * 128;            // W bytes per K block
  static constexpr int kStageABytes = kKB * kABytes;
  static constexpr int kStageBytes = kKB * (kABytes + kBBytes);
  static constexpr int kStages = (200 * 1024) / kStageBytes > 12 ? 12 : (200 * 1024) / kStageBytes;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 256;
  static_assert(kStages >= 2, "GEMM ring needs two stages");
};

struct Seg {
  __nv_bfloat16* out;  // [M][ldo]
  int ldo;             // row stride of out (elements) = N of this segment
  int tiles;           // number of BN-column tiles in this segment
  int col0;            // first column of this segment in the split-K partial buffer
};

struct Params {
  int M, K;
  int nseg;
  Seg seg[3];
  const __nv_bfloat16* R;  // residual [M][ldo of segment 0] or null (single-segment use)
  int out_f32;             // 1: outputs are f32 (no rounding; one split, no residual)
  int splits;              // K splits (gridDim.z)
  int ncols;               // total columns over the segments (partial buffer row length)
  float* part;             // [splits][M][ncols] f32 (splits > 1)
  int* err;
};

// Sum of the K-split partials in split order, plus the residual, rounded to
// bf16 and scattered to the output segments. 8 columns per thread; every
// split's loads are issued before the sum.
struct ReduceParams {
  const float* part;
  int splits, M, ncols;
  int nseg;
  __nv_bfloat16* out[3];
  int col0[4];  // segment column starts (col0[nseg] = ncols)
  const __nv_bfloat16* R;
};

template <int MAXS>
__global__ void __launch_bounds__(256) gemm_reduce_kernel(ReduceParams p) {
  griddep_launch();
  griddep_wait();
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;  // 8-column group
  const int groups = p.ncols / 8;
  if (idx >= (long long)p.M * groups) return;
  const int row = (int)(idx / groups);
  const int col = (int)(idx % groups) * 8;
  float4 a[MAXS][2];
#pragma unroll
  for (int z = 0; z < MAXS; ++z) {
    if (z < p.splits) {
      const float4* src = reinterpret_cast<const float4*>(p.part + ((size_t)z * p.M + row) * p.ncols + col);
      a[z][0] = __ldcg(src);
      a[z][1] = __ldcg(src + 1);
    }
  }
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int z = 0; z < MAXS; ++z) {
    if (z < p.splits) {
      acc[0] += a[z][0].x; acc[1] += a[z][0].y; acc[2] += a[z][0].z; acc[3] += a[z][0].w;
      acc[4] += a[z][1].x; acc[5] += a[z][1].y; acc[6] += a[z][1].z; acc[7] += a[z][1].w;
    }
  }
  int seg = 0;
  while (seg + 1 < p.nseg && col >= p.col0[seg + 1]) ++seg;
  const int ldo = p.col0[seg + 1] - p.col0[seg];
  const size_t o = (size_t)row * ldo + (col - p.col0[seg]);
  if (p.R) {
    const uint4 u = *reinterpret_cast<const uint4*>(p.R + o);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(b2[j]);
      acc[2 * j] += f.x;
      acc[2 * j + 1] += f.y;
    }
  }
  uint4 w;
  __nv_bfloat162* w2 = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
  for (int j = 0; j < 4; ++j) w2[j] = __floats2bfloat162_rn(acc[2 * j], acc[2 * j + 1]);
  *reinterpret_cast<uint4*>(p.out[seg] + o) = w;
}

struct Maps {
  CUtensorMap a;
  CUtensorMap b[3];
};

// Rounds 32 f32 values to bf16 (+ residual) and stores them at dst.
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const __nv_bfloat16* res, const float* v) {
  float w[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) w[i] = v[i];
  if (res) {
    const uint4* rs = reinterpret_cast<const uint4*>(res);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint4 u = rs[c];
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(b2[j]);
        w[c * 8 + 2 * j] += f.x;
        w[c * 8 + 2 * j + 1] += f.y;
      }
    }
  }
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 u;
    __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int j = 0; j < 4; ++j) b2[j] = __floats2bfloat162_rn(w[c * 8 + 2 * j], w[c * 8 + 2 * j + 1]);
    d4[c] = u;
  }
}

// CTA (column tile, 128-row block, K split). With one split the epilogue adds
// the residual, rounds to bf16 and stores; with several it writes the f32
// partial of its K range for gemm_reduce_kernel.
template <int BN>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ Maps maps, Params p) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * kBM;
  int seg = 0, t = blockIdx.x;
  while (seg + 1 < p.nseg && t >= p.seg[seg].tiles) t -= p.seg[seg++].tiles;
  const int n0 = t * BN;
  const CUtensorMap* mapB = &maps.b[seg];
  const int nk_all = p.K / kBK;
  const int z = blockIdx.z;
  const int kb0 = (int)(((long long)z * nk_all) / p.splits);
  const int kb1 = (int)(((long long)(z + 1) * nk_all) / p.splits);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, BN < 32 ? 32 : BN);
    tmem_relinquish();
  }
  griddep_launch();
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
      const uint32_t bytes = C::kStageBytes;  // rows past M / N and K blocks past K are zero-filled
      int s = 0;
      uint32_t ph = 0;
      bool issued[C::kStages];
      uint32_t issued_ph[C::kStages];
      for (int i = 0; i < C::kStages; ++i) issued[i] = false, issued_ph[i] = 0;
      // Stage u covers K blocks [kb0 + u KB, kb0 + (u + 1) KB) of this split.
      // Every CTA walks K in the same order: the CTAs that share an A tile
      // then request the same lines at about the same time, which L2 serves
      // far faster than as many distinct lines.
      const int nst = (kb1 - kb0 + C::kKB - 1) / C::kKB;
      auto kstart = [&](int u) { return kb0 + u * C::kKB; };
      // weights are read-only inputs: the first stages' W boxes are fetched
      // before waiting for the kernel that produces A
      const int pre = min(C::kStages, nst);
      for (int i = 0; i < pre; ++i) {
        uint8_t* st = smem + i * C::kStageBytes;
        mbar_arrive_expect_tx(&full[i], bytes);
        tma_load_3d(st + C::kStageABytes, mapB, &full[i], 0, n0, kstart(i), polB);
        issued[i] = true;
        issued_ph[i] = 0;
      }
      griddep_wait();
      for (int i = 0; i < pre; ++i) tma_load_3d(smem + i * C::kStageBytes, &maps.a, &full[i], 0, m0, kstart(i), polA);
      s = pre % C::kStages;
      ph = (pre == C::kStages) ? 1u : 0u;
      for (int u = pre; u < nst; ++u) {
        if (!mbar_wait(&empty[s], ph ^ 1u, p.err, abort_flag)) break;
        uint8_t* st = smem + s * C::kStageBytes;
        mbar_arrive_expect_tx(&full[s], bytes);
        tma_load_3d(st, &maps.a, &full[s], 0, m0, kstart(u), polA);
        tma_load_3d(st + C::kStageABytes, mapB, &full[s], 0, n0, kstart(u), polB);
        issued[s] = true;
        issued_ph[s] = ph;
        if (++s == C::kStages) { s = 0; ph ^= 1u; }
      }
      if (*abort_flag)
        for (int i = 0; i < C::kStages; ++i)
          if (issued[i]) mbar_wait(&full[i], issued_ph[i], p.err, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, BN);
      const int nst = (kb1 - kb0 + C::kKB - 1) / C::kKB;
      int s = 0;
      uint32_t ph = 0;
      for (int u = 0; u < nst; ++u) {
        // the same stage order as the producer; only the split's K blocks count
        const int ks = kb0 + u * C::kKB;
        const int nvalid = min(C::kKB, kb1 - ks);
        if (!mbar_wait(&full[s], ph, p.err, abort_flag)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + s * C::kStageBytes);
        const uint32_t b0 = a0 + C::kStageABytes;
        for (int j = 0; j < nvalid; ++j) {
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            mma_bf16_ss(tmem, umma_desc_sw128(a0 + j * kABytes + k * 32, 16, 1024),
                        umma_desc_sw128(b0 + j * C::kBBytes + k * 32, 16, 1024), idesc,
                        (u > 0 || j > 0 || k != 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
        if (++s == C::kStages) { s = 0; ph ^= 1u; }
      }
      mma_commit(tfull);  // also covers every MMA above before TMEM is read or freed
    }
  }
  // ---------------------------------------------------------------- epilogue
  if (warp >= 2) {
    griddep_wait();  // the residual and the outputs belong to earlier kernels
    const int quad = warp & 3;
    const int row = m0 + quad * 32 + lane;
    const Seg sg = p.seg[seg];
    const bool ok = mbar_wait_warp(tfull, 0, p.err, abort_flag);
    tc_fence_after();
    if (ok) {
      const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {  // 32 columns at a time
        float v[32];
        uint32_t r[32];
        tmem_ld32_sync(tbase + c * 32, r);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
        if (row < p.M) {
          if (p.out_f32) {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(sg.out) + (size_t)row * sg.ldo + n0 + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          } else if (p.splits == 1) {
            store_row32(sg.out + (size_t)row * sg.ldo + n0 + c * 32,
                        p.R ? p.R + (size_t)row * sg.ldo + n0 + c * 32 : nullptr, v);
          } else {  // this split's f32 partial; gemm_reduce_kernel sums the splits in order
            float4* dst =
                reinterpret_cast<float4*>(p.part + ((size_t)z * p.M + row) * p.ncols + sg.col0 + n0 + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN < 32 ? 32 : BN);
  }
}

}  // namespace gemmtc

// ---------------------------------------------------------------- host side
constexpr int kMaxSplits = 16;

bool gemm_tc_prepare_with(GemmTc* g, const void* A, int M, int K, int nseg, const void* const* W,
                          void* const* out, const int* N, int bn, int splits) {
  if (cudaFuncSetAttribute(gemmtc::gemm_tc_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gemmtc::Cfg<32>::kSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(gemmtc::gemm_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gemmtc::Cfg<64>::kSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(gemmtc::gemm_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gemmtc::Cfg<128>::kSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(gemmtc::gemm_tc_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gemmtc::Cfg<256>::kSmemBytes) != cudaSuccess) {
    set_last_error("cudaFuncSetAttribute(gemm_tc_kernel) failed");
    return false;
  }
  if (nseg < 1 || nseg > 3 || K % 64 != 0) {
    set_last_error("gemm_tc: unsupported shape");
    return false;
  }
  static_assert(sizeof(gemmtc::Maps) <= sizeof(g->maps), "GemmTc map storage too small");
  gemmtc::Maps* maps = reinterpret_cast<gemmtc::Maps*>(g->maps);
  int ncols = 0, gcd = 256;
  for (int i = 0; i < nseg; ++i) {
    if (N[i] % 32 != 0) {
      set_last_error("gemm_tc: N must be a multiple of 32");
      return false;
    }
    while (N[i] % gcd) gcd >>= 1;
    ncols += N[i];
  }
  if (bn != 32 && bn != 64 && bn != 128 && bn != 256) bn = 64;
  if (gcd < bn) {
    set_last_error("gemm_tc: column tile wider than a segment allows");
    return false;
  }
  g->bn = bn;
  // K-major operands as 3D (64 elements, rows, K / 64) so that one box holds
  // KB consecutive 128-byte-swizzled K blocks
  const uint32_t kb = (uint32_t)gemmtc::kblocks_per_stage(bn);
  const uint64_t dA[3] = {64, (uint64_t)M, (uint64_t)K / 64};
  const uint64_t sA[2] = {(uint64_t)K * 2, 128};
  const uint32_t bA[3] = {64, (uint32_t)gemmtc::kBM, kb};
  if (!encode_tmap_bf16(&maps->a, A, 3, dA, sA, bA, true)) return false;
  g->M = M;
  g->K = K;
  g->nseg = nseg;
  g->tiles = 0;
  g->ncols = ncols;
  for (int i = 0; i < nseg; ++i) {
    const uint64_t dB[3] = {64, (uint64_t)N[i], (uint64_t)K / 64};
    const uint32_t bB[3] = {64, (uint32_t)g->bn, kb};
    if (!encode_tmap_bf16(&maps->b[i], W[i], 3, dB, sA, bB, true)) return false;
    g->out[i] = out[i];
    g->N[i] = N[i];
    g->tiles += N[i] / g->bn;
  }
  g->splits = std::max(1, std::min(std::min(splits, kMaxSplits), K / 64));
  return true;
}

bool gemm_tc_prepare(GemmTc* g, const void* A, int M, int K, int nseg, const void* const* W, void* const* out,
                     const int* N, int sm_count) {
  int gcd = 256;
  for (int i = 0; i < nseg; ++i)
    while (gcd > 32 && N[i] % gcd) gcd >>= 1;
  // Column tile by a cost model: waves of CTAs x bytes each CTA moves per K
  // block (16 KB of A + bn * 128 B of W); ties go to the wider tile. K is
  // split only when the best choice still leaves most SMs idle.
  const int mblocks = ceil_div(M, gemmtc::kBM);
  auto ctas = [&](int w) {
    int tiles = 0;
    for (int i = 0; i < nseg; ++i) tiles += N[i] / w;
    return tiles * mblocks;
  };
  int bn = gcd;
  long long best = -1;
  for (int w = gcd; w >= 32; w >>= 1) {
    const long long cost = (long long)ceil_div(ctas(w), sm_count) * (gemmtc::kABytes + w * 128);
    if (best < 0 || cost < best) {
      best = cost;
      bn = w;
    }
  }
  int splits = 1;
  if (ctas(bn) * 2 <= sm_count) splits = std::max(1, std::min(sm_count / ctas(bn), (K / 64) / 4));
  return gemm_tc_prepare_with(g, A, M, K, nseg, W, out, N, bn, splits);
}

size_t gemm_tc_partial_floats(const GemmTc& g) {
  return g.splits > 1 ? (size_t)g.splits * g.M * g.ncols : 0;
}

void launch_gemm_tc(Exec& ex, const GemmTc& g, const void* residual) {
  gemmtc::Params p;
  p.M = g.M;
  p.K = g.K;
  p.nseg = g.nseg;
  int col0 = 0;
  for (int i = 0; i < 3; ++i) {
    p.seg[i].out = i < g.nseg ? static_cast<__nv_bfloat16*>(g.out[i]) : nullptr;
    p.seg[i].ldo = i < g.nseg ? g.N[i] : 0;
    p.seg[i].tiles = i < g.nseg ? g.N[i] / g.bn : 0;
    p.seg[i].col0 = col0;
    if (i < g.nseg) col0 += g.N[i];
  }
  p.R = static_cast<const __nv_bfloat16*>(residual);
  p.out_f32 = g.out_f32;
  p.splits = g.splits;
  p.ncols = g.ncols;
  p.part = g.part;
  p.err = ex.err;
  dim3 grid(g.tiles, ceil_div(g.M, gemmtc::kBM), g.splits);
  const gemmtc::Maps& maps = *reinterpret_cast<const gemmtc::Maps*>(g.maps);
  const dim3 block(gemmtc::kThreads);
  if (g.bn == 32)
    launch_pdl(gemmtc::gemm_tc_kernel<32>, grid, block, gemmtc::Cfg<32>::kSmemBytes, ex.stream, maps, p);
  else if (g.bn == 256)
    launch_pdl(gemmtc::gemm_tc_kernel<256>, grid, block, gemmtc::Cfg<256>::kSmemBytes, ex.stream, maps, p);
  else if (g.bn == 128)
    launch_pdl(gemmtc::gemm_tc_kernel<128>, grid, block, gemmtc::Cfg<128>::kSmemBytes, ex.stream, maps, p);
  else
    launch_pdl(gemmtc::gemm_tc_kernel<64>, grid, block, gemmtc::Cfg<64>::kSmemBytes, ex.stream, maps, p);
  ex.launches++;
  if (g.splits > 1) {
    gemmtc::ReduceParams r;
    r.part = g.part;
    r.splits = g.splits;
    r.M = g.M;
    r.ncols = g.ncols;
    r.nseg = g.nseg;
    int c = 0;
    for (int i = 0; i < 3; ++i) {
      r.out[i] = i < g.nseg ? static_cast<__nv_bfloat16*>(g.out[i]) : nullptr;
      r.col0[i] = c;
      if (i < g.nseg) c += g.N[i];
    }
    r.col0[3] = c;
    for (int i = g.nseg; i < 3; ++i) r.col0[i + 1] = c;
    r.R = static_cast<const __nv_bfloat16*>(residual);
    const long long threads = (long long)g.M * (g.ncols / 8);
    launch_pdl(gemmtc::gemm_reduce_kernel<kMaxSplits>, dim3((unsigned)ceil_div((int)threads, 256)), dim3(256), 0,
               ex.stream, r);
    ex.launches++;
  }
}

}  // namespace dg
