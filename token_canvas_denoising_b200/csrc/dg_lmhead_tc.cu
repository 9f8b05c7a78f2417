// LM head over the vocabulary fused with the per-position softmax entropy and
// argmax, on the 5th-generation tensor cores (tcgen05, TMEM accumulators,
// TMA-fed shared memory). The [rows x vocab] logits never reach HBM.
//
// Method: the model gives one distribution over the ~250K-entry vocabulary per
// canvas position and lower entropy marks a more certain position
// ("DiffusionGemma解析：扩散模型如何让LLM快5倍", 整片并行去噪; vocabulary size in
// 自回归的瓶颈). Logit x_v = Hs[r] . W[v]; the entropy uses l_v = x_v * invT[r],
// the argmax uses x_v (lowest id on ties).
//
// Two kernels share the epilogue arithmetic (RowState): for up to 128 rows a
// single-CTA kernel (below), for more the CTA-pair kernel further down, whose
// double-buffered accumulator lets the epilogue overlap the next tile's MMAs.
//
// Single CTAs: CTA (p, mb) owns rows [256 mb, 256 mb + 256) and a contiguous run
// of 32-column vocab granules; it walks that run in tiles of up to 256 columns.
// Per tile: K-loop of 64-wide blocks, each two 256-row TMA boxes (the rows' A
// block and 256 W rows from the tile's first granule; per-box cost, not bytes,
// bounds a TMA stream, so boxes are as large as they go), then 2 x 4 MMAs
// (M=128, N<=256, K=16)
// into two TMEM accumulators (columns [0,256) and [256,512)). Eight epilogue
// warps then stream the accumulators out of TMEM and fold them into each row's
// online (max, Z, S, best, id) state in base 2 (exp2 on the MUFU). One
// partial record per (row, CTA) is written at the end; a merge kernel folds
// the CTAs' records.
//
// Warp roles: warp 0 = TMA producer, warp 1 = TMEM allocator + MMA issuer,
// warps 2..9 = epilogue (warp w reads TMEM lanes 32*(w%4)..+31 of half (w-2)/4).
// The epilogue and the MMAs alternate: both accumulators hold the one tile.
//
// FP8 variant (the FP8 deployment of "DiffusionGemma深度拆解", 性能数据): the
// rows' activations and the vocab weights are e4m3 codes with power-of-two
// scales (one per row of Hs, one per vocab row); the MMAs are kind::f8f6f4
// (K = 32 per instruction, twice the K per 128-byte row), and the epilogue
// multiplies each accumulated logit by its row's and its column's scale
// before the online entropy/argmax (the product is exact for powers of two).
#include "dg_internal.cuh"
#include "dg_sm100.cuh"
#include "dg_tmap.cuh"

namespace dg {
namespace lmtc {

using namespace sm100;

constexpr int kStages = 3;
constexpr int kRowBytes = 128;                 // one K block: 64 bf16 or 128 e4m3 per row
constexpr int kHalfBytes = 128 * 128;          // 128 rows x 128 B
constexpr int kABytes = 2 * kHalfBytes;        // 32 KB
constexpr int kGranule = 32;                   // vocab columns per work granule
constexpr int kGranBytes = kGranule * 128;     // 4 KB
constexpr int kMaxGran = 8;                    // 256-column tile
constexpr int kBBytes = kMaxGran * kGranBytes; // 32 KB
constexpr int kStageBytes = kABytes + kBBytes; // 64 KB
constexpr int kThreads = 320;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;

struct Params {
  int M, d, V;
  const float* invT;  // [M] or null
  const float* sa;    // FP8: [M] row scales of the activations
  const float* sw;    // FP8: [V] row scales of the vocab weights
  LmRec* rec;         // [M][gridDim.x]
  int* err;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One row's online state over the vocabulary columns a thread folds, in
// base 2: m = max of x * it2 (it2 = inverse temperature / ln 2), z0 + z1 =
// sum of 2^(l - m), s0 + s1 = sum of (l - m) 2^(l - m) (two chains each, for
// instruction-level parallelism), and the argmax (best x, lowest id on ties).
template <bool kFp8>
struct RowState {
  float m = -INFINITY, z0 = 0.f, z1 = 0.f, s0 = 0.f, s1 = 0.f, best = -INFINITY;
  int idx = 0x7fffffff;

  // Folds 32 columns (one TMEM load; column vbase + i in r[i]). Per logit:
  // half a three-input max, the scaled logit l = x * it2 rounded on its own
  // (so that l - m is exactly 0 at the maximum and a one-hot row has entropy
  // exactly 0), the difference, the exponential and two accumulations. The
  // argmax needs only the chunk's maximum, compared with the best so far; the
  // chunk is searched for its first (lowest-id) maximal column only when that
  // maximum improves on it. FP8: lane i loads the scale of column vbase + i
  // and hands it to the other lanes; each thread applies it with its own
  // row's scale sa.
  __device__ __forceinline__ void fold(uint32_t (&r)[32], int vbase, float it2, const float* sw, float sa,
                                       int lane) {
    if constexpr (kFp8) {
      const float swl = __ldg(sw + vbase + lane);
#pragma unroll
      for (int i = 0; i < 32; ++i)
        r[i] = __float_as_uint(__uint_as_float(r[i]) * (__shfl_sync(0xffffffffu, swl, i) * sa));
    }
    float mk[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {  // four independent chains of 8 columns
      const float* x = reinterpret_cast<const float*>(r) + 8 * k;
      mk[k] = fmaxf(fmax3(fmax3(fmax3(x[0], x[1], x[2]), x[3], x[4]), x[5], x[6]), x[7]);
    }
    const float bx = fmax3(mk[0], mk[1], fmaxf(mk[2], mk[3]));
    if (bx > best) {
      best = bx;
      int j = 0;
#pragma unroll
      for (int i = 31; i >= 0; --i)
        if (__uint_as_float(r[i]) == bx) j = i;
      idx = vbase + j;
    }
    const float bm = __fmul_rn(bx, it2);  // = the largest x * it2 (rounding is monotone)
    if (bm > m) {
      if (m != -INFINITY) {
        const float c = ex2(m - bm);
        const float dm = m - bm;
        s0 = c * fmaf(dm, z0, s0);
        s1 = c * fmaf(dm, z1, s1);
        z0 *= c;
        z1 *= c;
      }
      m = bm;
    }
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float d0 = __fmul_rn(__uint_as_float(r[i]), it2) - m;
      const float d1 = __fmul_rn(__uint_as_float(r[i + 1]), it2) - m;
      const float e0 = ex2(d0), e1 = ex2(d1);
      z0 += e0;
      z1 += e1;
      s0 = fmaf(d0, e0, s0);
      s1 = fmaf(d1, e1, s1);
    }
  }

  // Folds another state of the same row (other columns) into this one.
  __device__ __forceinline__ void merge(float mo, float zo, float so, float besto, int idxo) {
    if (mo != -INFINITY) {
      float z = z0 + z1, s = s0 + s1;
      if (m == -INFINITY) {
        z = zo;
        s = so;
        m = mo;
      } else {
        const float mm = fmaxf(m, mo);
        const float ca = ex2(m - mm), cb = ex2(mo - mm);
        s = ca * fmaf(m - mm, z, s) + cb * fmaf(mo - mm, zo, so);
        z = ca * z + cb * zo;
        m = mm;
      }
      z0 = z;
      z1 = 0.f;
      s0 = s;
      s1 = 0.f;
    }
    if (besto > best || (besto == best && idxo < idx)) {
      best = besto;
      idx = idxo;
    }
  }

  // The partial record in natural-log units.
  __device__ __forceinline__ LmRec record() const {
    const float kLn2 = 0.6931471805599453f;
    LmRec rec;
    rec.m = m * kLn2;
    rec.z = z0 + z1;
    rec.s = (s0 + s1) * kLn2;
    rec.best = best;
    rec.idx = idx;
    rec.pad0 = rec.pad1 = rec.pad2 = 0;
    return rec;
  }
};

// Folds TMEM columns [32 c_beg, 32 c_end) of this warp's 32 lanes at taddr
// (column 32 c holds vocab ids vbase0 + 32 c ..) into st: two register
// buffers, so the next 32 columns load from TMEM while the current ones are
// folded. Warp-collective; c_beg and c_end are the same in every lane.
template <bool kFp8>
__device__ __forceinline__ void fold_columns(RowState<kFp8>& st, uint32_t taddr, int c_beg, int c_end, int vbase0,
                                             float it2, const float* sw, float sa, int lane) {
  if (c_beg >= c_end) return;
  uint32_t ra[32], rb[32];
  tmem_ld32(taddr + c_beg * 32, ra);
  tmem_ld_wait_regs(ra);
  for (int c = c_beg; c < c_end; c += 2) {
    const bool has_b = c + 1 < c_end;
    if (has_b) tmem_ld32(taddr + (c + 1) * 32, rb);
    st.fold(ra, vbase0 + c * 32, it2, sw, sa, lane);
    if (has_b) {
      tmem_ld_wait_regs(rb);
      const bool has_a = c + 2 < c_end;
      if (has_a) tmem_ld32(taddr + (c + 2) * 32, ra);
      st.fold(rb, vbase0 + (c + 1) * 32, it2, sw, sa, lane);
      if (has_a) tmem_ld_wait_regs(ra);
    }
  }
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
lmhead_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, Params p) {
  constexpr int kBK = kFp8 ? kRowBytes : kRowBytes / 2;  // K elements per block
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 1;
  uint64_t* mdone = tempty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mdone + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * 256;
  const int halves = (p.M - m0 > 128) ? 2 : 1;
  const int G = p.V / kGranule;
  const int g0 = (int)(((long long)blockIdx.x * G) / gridDim.x);
  const int g1 = (int)(((long long)(blockIdx.x + 1) * G) / gridDim.x);
  const int n_tiles = (g1 - g0 + kMaxGran - 1) / kMaxGran;
  const int nk = p.d / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 8);
    mbar_init(mdone, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  griddep_launch();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t polA = policy_evict_last();   // rows' activations: re-read every tile
      const uint64_t polB = policy_evict_first();  // vocab weights: streamed once
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued_ph[kStages];
      bool issued[kStages];
      for (int i = 0; i < kStages; ++i) issued[i] = false, issued_ph[i] = 0;
      // vocab weights are read-only inputs: the first stages' W tiles are
      // fetched before waiting for the kernel that produces Hs
      int pre = 0;
      // every stage is one 256-row A box and one 256-row W box (rows past M
      // or V are zero-filled and still counted; unused rows are never read)
      const uint32_t bytes = kStageBytes;
      if (n_tiles > 0) {
        pre = min(kStages, nk);
        for (int i = 0; i < pre; ++i) {
          uint8_t* st = smem + i * kStageBytes;
          mbar_arrive_expect_tx(&full[i], bytes);
          tma_load_2d(st + kABytes, &tmB, &full[i], i * kBK, g0 * kGranule, polB);
          issued[i] = true;
          issued_ph[i] = 0;
        }
        griddep_wait();
        for (int i = 0; i < pre; ++i) tma_load_2d(smem + i * kStageBytes, &tmA, &full[i], i * kBK, m0, polA);
        s = pre % kStages;
        ph = (pre == kStages) ? 1u : 0u;
      }
      for (int t = 0; t < n_tiles && !*abort_flag; ++t) {
        const int gt = g0 + t * kMaxGran;
        for (int kb = (t == 0 ? pre : 0); kb < nk; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, p.err, abort_flag)) break;
          uint8_t* st = smem + s * kStageBytes;
          mbar_arrive_expect_tx(&full[s], bytes);
          tma_load_2d(st, &tmA, &full[s], kb * kBK, m0, polA);
          tma_load_2d(st + kABytes, &tmB, &full[s], kb * kBK, gt * kGranule, polB);
          issued[s] = true;
          issued_ph[s] = ph;
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
      }
      if (*abort_flag) {  // drain this CTA's own copies before it exits
        for (int i = 0; i < kStages; ++i)
          if (issued[i]) mbar_wait(&full[i], issued_ph[i], p.err, nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, tph = 0;
      bool any = false;
      for (int t = 0; t < n_tiles && !*abort_flag; ++t) {
        const int gt = g0 + t * kMaxGran;
        const int ng = min(kMaxGran, g1 - gt);
        const uint32_t idesc = kFp8 ? idesc_e4m3_f32(128, ng * kGranule) : idesc_bf16_f32(128, ng * kGranule);
        if (!mbar_wait(tempty, tph ^ 1u, p.err, abort_flag)) break;
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[s], ph, p.err, abort_flag)) break;
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * kStageBytes);
          const uint32_t b0 = a0 + kABytes;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (h < halves) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {  // 32 bytes of K per instruction
                const uint64_t ad = umma_desc_sw128(a0 + h * kHalfBytes + k * 32, 16, 1024);
                const uint64_t bd = umma_desc_sw128(b0 + k * 32, 16, 1024);
                if constexpr (kFp8)
                  mma_f8_ss(tmem + h * 256, ad, bd, idesc, (kb | k) != 0);
                else
                  mma_bf16_ss(tmem + h * 256, ad, bd, idesc, (kb | k) != 0);
              }
            }
          }
          any = true;
          mma_commit(&empty[s]);
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
        mma_commit(tfull);
        tph ^= 1u;
      }
      if (any) {  // every MMA of this CTA has landed before TMEM is released
        mma_commit(mdone);
        mbar_wait(mdone, 0, p.err, nullptr);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    griddep_wait();  // invT and the partial records belong to earlier kernels
    const int ew = warp - 2;
    const int half = ew >> 2;
    const int quad = warp & 3;
    const int row = m0 + half * 128 + quad * 32 + lane;
    const bool has_row = half < halves && row < p.M;
    const float kLog2e = 1.4426950408889634f;
    const float it2 = (has_row && p.invT ? p.invT[row] : 1.f) * kLog2e;  // logit -> scaled base-2
    const float sa = kFp8 && has_row ? p.sa[row] : 1.f;
    RowState<kFp8> st;
    uint32_t tph = 0;
    const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(half * 256);
    for (int t = 0; t < n_tiles; ++t) {
      const int gt = g0 + t * kMaxGran;
      const int ng = min(kMaxGran, g1 - gt);
      if (!mbar_wait_warp(tfull, tph, p.err, abort_flag)) break;
      tc_fence_after();
      if (half < halves) fold_columns(st, tbase, 0, ng, gt * kGranule, it2, p.sw, sa, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty);
      tph ^= 1u;
    }
    if (has_row && !*abort_flag) p.rec[(size_t)row * gridDim.x + blockIdx.x] = st.record();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- CTA pairs
// For more than 128 rows the LM head runs on CTA pairs (clusters of 2, tcgen05
// .cta_group::2). Pair (p, mb) owns rows [256 mb, 256 mb + 256) -- the even
// CTA rows 0..127 of them, the odd CTA rows 128..255 -- and a contiguous run
// of 32-column vocab granules, walked in tiles of up to 256 columns. Per K
// block each CTA fetches one 128-row box of its own rows' activations and one
// 128-row box of vocab weights (the tile's first N/2 columns in the even CTA,
// the other N/2 in the odd one), 32 KB; the even CTA issues M = 256 MMAs that
// read both CTAs' boxes and leave each CTA's 128 rows x N logits in its own
// tensor memory. Per CTA a tile is half the MMA work of a 256 x 256 tile on one
// SM for half the bytes, so the per-SM ingest rate is the same, but only 256 of
// the 512 TMEM columns hold a tile: the accumulator is double-buffered and the
// epilogue of tile t runs while the tensor cores compute tile t + 1.
//
// Warp roles (in both CTAs): warp 0 = TMA producer; warp 1 = TMEM allocator
// (both CTAs) and MMA issuer (even CTA only); warps 2..9 = epilogue, warp w
// reading lanes 32*(w%4)..+31 and half (w-2)/4 of each tile's 32-column
// chunks; the two halves of a row merge in shared memory at the end. The
// producers count their bytes on the even CTA's stage barrier; the MMA
// completions arrive on both CTAs' stage-free and accumulator-full barriers;
// all 16 epilogue warps of the pair arrive on the even CTA's accumulator-free
// barrier.
constexpr int kPairStages = 7;
constexpr int kPairABytes = 128 * kRowBytes;                // 16 KB: this CTA's 128 rows
constexpr int kPairBBytes = 128 * kRowBytes;                // 16 KB: up to 128 vocab rows
constexpr int kPairStageBytes = kPairABytes + kPairBBytes;  // 32 KB
// the dynamic shared window starts 1024-aligned (checked at entry): seven
// 32 KB stages and the barriers fill it; the epilogue's merge area (one row
// state per TMEM lane, 4 KB) reuses stage 0 once every MMA has completed
constexpr int kPairSmemBytes = kPairStages * kPairStageBytes + 256;

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
lmhead_tc_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, Params p) {
  constexpr int kBK = kFp8 ? kRowBytes : kRowBytes / 2;  // K elements per block
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // SW128 tiles need 1024-byte alignment; the window's start is the same in
  // both CTAs of the pair, so both return here (before any pair operation)
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) set_error(p.err, kDevBadAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPairStages * kPairStageBytes);
  uint64_t* empty = full + kPairStages;
  uint64_t* tfull = empty + kPairStages;  // [2]
  uint64_t* tempty = tfull + 2;           // [2]
  uint64_t* mdone = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mdone + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* merge_area = reinterpret_cast<float*>(smem);  // [128][8], stage 0 after the last tile

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the pair's MMA issuer
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int m0 = blockIdx.y * 256;
  const int G = p.V / kGranule;
  const int g0 = (int)(((long long)pair * G) / npairs);
  const int g1 = (int)(((long long)(pair + 1) * G) / npairs);
  const int n_tiles = (g1 - g0 + kMaxGran - 1) / kMaxGran;
  const int nk = p.d / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 16);  // 8 epilogue warps in each CTA of the pair
    }
    mbar_init(mdone, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, 512);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  griddep_launch();
  tc_fence_before();
  __syncwarp();
  cluster_sync();  // both CTAs' barriers exist and both hold their TMEM
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t polA = policy_evict_last();   // rows' activations: re-read every tile
      const uint64_t polB = policy_evict_first();  // vocab weights: streamed
      const uint32_t full_even = mapa_shared(full, 0);
      const uint32_t tx = 2 * kPairStageBytes;  // both CTAs' boxes (rows past M or V are zero-filled, counted)
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued_ph[kPairStages];
      bool issued[kPairStages];
      for (int i = 0; i < kPairStages; ++i) issued[i] = false, issued_ph[i] = 0;
      const int yA = m0 + (int)rank * 128;
      // vocab weights are read-only inputs: the first stages' W boxes are
      // fetched before waiting for the kernel that produces Hs
      int pre = 0;
      if (n_tiles > 0) {
        pre = min(kPairStages, nk);
        const int ng = min(kMaxGran, g1 - g0);
        const int yB = g0 * kGranule + (int)rank * ng * (kGranule / 2);
        for (int i = 0; i < pre; ++i) {
          if (rank == 0) mbar_arrive_expect_tx(&full[i], tx);
          tma_load_2d_pair(smem + i * kPairStageBytes + kPairABytes, &tmB, full_even + 8u * i, i * kBK, yB, polB);
          issued[i] = true;
        }
        griddep_wait();
        for (int i = 0; i < pre; ++i)
          tma_load_2d_pair(smem + i * kPairStageBytes, &tmA, full_even + 8u * i, i * kBK, yA, polA);
        s = pre % kPairStages;
        ph = (pre == kPairStages) ? 1u : 0u;
      }
      for (int t = 0; t < n_tiles && !*abort_flag; ++t) {
        const int gt = g0 + t * kMaxGran;
        const int ng = min(kMaxGran, g1 - gt);
        const int yB = gt * kGranule + (int)rank * ng * (kGranule / 2);
        for (int kb = (t == 0 ? pre : 0); kb < nk; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, p.err, abort_flag)) break;
          uint8_t* st = smem + s * kPairStageBytes;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], tx);
          tma_load_2d_pair(st, &tmA, full_even + 8u * s, kb * kBK, yA, polA);
          tma_load_2d_pair(st + kPairABytes, &tmB, full_even + 8u * s, kb * kBK, yB, polB);
          issued[s] = true;
          issued_ph[s] = ph;
          if (++s == kPairStages) { s = 0; ph ^= 1u; }
        }
      }
      if (*abort_flag) {
        // drain the copies in flight before the CTA exits: the even CTA waits
        // for its stage barriers (which count both CTAs' bytes); the odd CTA
        // cannot observe them and gives its copies a bounded grace period
        if (rank == 0) {
          for (int i = 0; i < kPairStages; ++i)
            if (issued[i]) mbar_wait(&full[i], issued_ph[i], p.err, nullptr);
        } else {
          const uint64_t t0 = globaltimer();
          while (globaltimer() - t0 < 200000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (rank == 0 && lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool any = false;
      for (int t = 0; t < n_tiles && !*abort_flag; ++t) {
        const int b = t & 1;
        const uint32_t use = (uint32_t)(t >> 1);
        const int gt = g0 + t * kMaxGran;
        const int ng = min(kMaxGran, g1 - gt);
        const uint32_t idesc = kFp8 ? idesc_e4m3_f32(256, ng * kGranule) : idesc_bf16_f32(256, ng * kGranule);
        if (!mbar_wait_cluster(&tempty[b], (use & 1u) ^ 1u, p.err, abort_flag)) break;
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[s], ph, p.err, abort_flag)) break;
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * kPairStageBytes);
          const uint32_t b0 = a0 + kPairABytes;
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 32 bytes of K per instruction
            const uint64_t ad = umma_desc_sw128(a0 + k * 32, 16, 1024);
            const uint64_t bd = umma_desc_sw128(b0 + k * 32, 16, 1024);
            if constexpr (kFp8)
              mma_f8_ss_pair(tmem + b * 256, ad, bd, idesc, (kb | k) != 0);
            else
              mma_bf16_ss_pair(tmem + b * 256, ad, bd, idesc, (kb | k) != 0);
          }
          any = true;
          mma_commit_pair_mc(&empty[s], 3);
          if (++s == kPairStages) { s = 0; ph ^= 1u; }
        }
        mma_commit_pair_mc(&tfull[b], 3);
      }
      if (any) {  // every MMA of the pair has landed before TMEM is released
        mma_commit_pair(mdone);
        mbar_wait(mdone, 0, p.err, nullptr);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    griddep_wait();  // invT and the partial records belong to earlier kernels
    const int chalf = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int rloc = quad * 32 + lane;
    const int row = m0 + (int)rank * 128 + rloc;
    const bool has_row = row < p.M;
    const float kLog2e = 1.4426950408889634f;
    const float it2 = (has_row && p.invT ? p.invT[row] : 1.f) * kLog2e;  // logit -> scaled base-2
    const float sa = kFp8 && has_row ? p.sa[row] : 1.f;
    const uint32_t tempty_even = mapa_shared(tempty, 0);
    const uint32_t tlane = tmem + ((uint32_t)(quad * 32) << 16);
    RowState<kFp8> st;
    for (int t = 0; t < n_tiles; ++t) {
      const int b = t & 1;
      const uint32_t use = (uint32_t)(t >> 1);
      const int gt = g0 + t * kMaxGran;
      const int ng = min(kMaxGran, g1 - gt);
      const int nh = (ng + 1) >> 1;  // 32-column chunks of column half 0
      if (!mbar_wait_warp(&tfull[b], use & 1u, p.err, abort_flag)) break;
      tc_fence_after();
      fold_columns(st, tlane + (uint32_t)(b * 256), chalf ? nh : 0, chalf ? ng : nh, gt * kGranule, it2, p.sw, sa,
                   lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_even + 8u * b);
    }
    // the two column halves of each row: half 1 hands its state to half 0
    float* ms = merge_area + rloc * 8;
    if (chalf == 1) {
      const LmRec r = st.record();
      ms[0] = st.m;
      ms[1] = st.z0 + st.z1;
      ms[2] = st.s0 + st.s1;
      ms[3] = r.best;
      ms[4] = __int_as_float(r.idx);
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (chalf == 0) {
      st.merge(ms[0], ms[1], ms[2], ms[3], __float_as_int(ms[4]));
      if (has_row && !*abort_flag) p.rec[(size_t)row * npairs + pair] = st.record();
    }
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();  // the pair's MMAs have landed and neither CTA touches the other's memory any more
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace lmtc

// More than 128 rows run on CTA pairs (each pair owns 256 rows); up to 128 on
// single CTAs, which then need only one 128-row accumulator.
static bool lmhead_tc_pairs(int M) { return M > 128; }

// Number of vocab partitions (CTAs, or CTA pairs, along the vocabulary) for M
// rows: one CTA per SM.
int lmhead_tc_partitions(int M, int V, int sm_count) {
  const int mb = ceil_div(M, 256);
  int P = (lmhead_tc_pairs(M) ? sm_count / 2 : sm_count) / mb;
  if (P < 1) P = 1;
  const int G = V / lmtc::kGranule;
  return P > G ? G : P;
}

bool lmhead_tc_prepare(const void* hs, const void* lm_head, int M, int d, int V, CUtensorMap* tmA,
                       CUtensorMap* tmB, bool fp8) {
  // kernel attributes are set here, on the host path that precedes any launch
  // (and never inside a stream capture)
  const bool pairs = lmhead_tc_pairs(M);
  cudaError_t e;
  if (pairs)
    e = cudaFuncSetAttribute(fp8 ? lmtc::lmhead_tc_pair_kernel<true> : lmtc::lmhead_tc_pair_kernel<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, lmtc::kPairSmemBytes);
  else
    e = cudaFuncSetAttribute(fp8 ? lmtc::lmhead_tc_kernel<true> : lmtc::lmhead_tc_kernel<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, lmtc::kSmemBytes);
  if (e != cudaSuccess) {
    set_last_error("cudaFuncSetAttribute(lmhead_tc kernel) failed");
    return false;
  }
  // one box = 128 bytes of K (64 bf16 or 128 e4m3) x 256 rows (single CTAs)
  // or 128 rows (pairs: each CTA fetches its half of the rows and of the tile)
  const uint32_t box_rows = pairs ? 128 : 256;
  const uint64_t es = fp8 ? 1 : 2;
  const uint64_t dA[2] = {(uint64_t)d, (uint64_t)M};
  const uint64_t sA[1] = {(uint64_t)d * es};
  const uint32_t bA[2] = {(uint32_t)(lmtc::kRowBytes / es), box_rows};
  const uint64_t dB[2] = {(uint64_t)d, (uint64_t)V};
  const uint32_t bB[2] = {(uint32_t)(lmtc::kRowBytes / es), box_rows};
  if (fp8)
    return encode_tmap_u8(tmA, hs, 2, dA, sA, bA, true) && encode_tmap_u8(tmB, lm_head, 2, dB, sA, bB, true);
  return encode_tmap_bf16(tmA, hs, 2, dA, sA, bA, true) && encode_tmap_bf16(tmB, lm_head, 2, dB, sA, bB, true);
}

void launch_lmhead_tc(Exec& ex, const CUtensorMap& tmA, const CUtensorMap& tmB, LmPartials part,
                      const float* invT, int M, int d, int V, const float* sa, const float* sw) {
  lmtc::Params p;
  p.M = M;
  p.d = d;
  p.V = V;
  p.invT = invT;
  p.sa = sa;
  p.sw = sw;
  p.rec = part.rec;
  p.err = ex.err;
  if (lmhead_tc_pairs(M)) {
    dim3 grid(2 * part.P, ceil_div(M, 256));
    if (sa)
      launch_pdl_pairs(lmtc::lmhead_tc_pair_kernel<true>, grid, dim3(lmtc::kThreads), lmtc::kPairSmemBytes,
                       ex.stream, tmA, tmB, p);
    else
      launch_pdl_pairs(lmtc::lmhead_tc_pair_kernel<false>, grid, dim3(lmtc::kThreads), lmtc::kPairSmemBytes,
                       ex.stream, tmA, tmB, p);
  } else {
    dim3 grid(part.P, ceil_div(M, 256));
    if (sa)
      launch_pdl(lmtc::lmhead_tc_kernel<true>, grid, dim3(lmtc::kThreads), lmtc::kSmemBytes, ex.stream, tmA, tmB, p);
    else
      launch_pdl(lmtc::lmhead_tc_kernel<false>, grid, dim3(lmtc::kThreads), lmtc::kSmemBytes, ex.stream, tmA, tmB,
                 p);
  }
  ex.launches++;
}

}  // namespace dg
