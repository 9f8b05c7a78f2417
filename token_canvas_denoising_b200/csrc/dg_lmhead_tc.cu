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
// Work split: CTA (p, mb) owns rows [256 mb, 256 mb + 256) and a contiguous run
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
    float m2 = -INFINITY, z0 = 0.f, z1 = 0.f, s0 = 0.f, s1 = 0.f, best = -INFINITY;
    int idx = 0x7fffffff;
    uint32_t tph = 0;
    const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(half * 256);
    for (int t = 0; t < n_tiles; ++t) {
      const int gt = g0 + t * kMaxGran;
      const int ncol = min(kMaxGran, g1 - gt) * kGranule;
      if (!mbar_wait_warp(tfull, tph, p.err, abort_flag)) break;
      tc_fence_after();
      if (half < halves) {
        for (int c0 = 0; c0 < ncol; c0 += 32) {
          uint32_t r[32];
          tmem_ld32_sync(tbase + c0, r);
          const int vbase = gt * kGranule + c0;
          // FP8: lane i loads the scale of column vbase + i and hands it to
          // the other lanes; each thread applies it with its own row's scale
          const float swl = kFp8 ? __ldg(p.sw + vbase + lane) : 1.f;
          float l[32];
          float bm = -INFINITY;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float x = __uint_as_float(r[i]);
            if constexpr (kFp8) x *= __shfl_sync(0xffffffffu, swl, i) * sa;
            if (x > best) { best = x; idx = vbase + i; }
            l[i] = x * it2;
            bm = fmaxf(bm, l[i]);
          }
          if (bm > m2) {
            if (m2 != -INFINITY) {
              const float c = ex2(m2 - bm);
              const float dm = m2 - bm;
              s0 = c * fmaf(dm, z0, s0);
              s1 = c * fmaf(dm, z1, s1);
              z0 *= c;
              z1 *= c;
            }
            m2 = bm;
          }
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float d0 = l[i] - m2, d1 = l[i + 1] - m2;
            const float e0 = ex2(d0), e1 = ex2(d1);
            z0 += e0;
            z1 += e1;
            s0 = fmaf(d0, e0, s0);
            s1 = fmaf(d1, e1, s1);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty);
      tph ^= 1u;
    }
    if (has_row && !*abort_flag) {
      const float kLn2 = 0.6931471805599453f;
      LmRec rec;
      rec.m = m2 * kLn2;
      rec.z = z0 + z1;
      rec.s = (s0 + s1) * kLn2;
      rec.best = best;
      rec.idx = idx;
      rec.pad0 = rec.pad1 = rec.pad2 = 0;
      p.rec[(size_t)row * gridDim.x + blockIdx.x] = rec;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace lmtc

// Number of vocab partitions (CTAs along the vocabulary) for M rows.
int lmhead_tc_partitions(int M, int V, int sm_count) {
  const int mb = ceil_div(M, 256);
  int P = sm_count / mb;
  if (P < 1) P = 1;
  const int G = V / lmtc::kGranule;
  return P > G ? G : P;
}

bool lmhead_tc_prepare(const void* hs, const void* lm_head, int M, int d, int V, CUtensorMap* tmA,
                       CUtensorMap* tmB, bool fp8) {
  // kernel attributes are set here, on the host path that precedes any launch
  // (and never inside a stream capture)
  if (cudaFuncSetAttribute(fp8 ? lmtc::lmhead_tc_kernel<true> : lmtc::lmhead_tc_kernel<false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, lmtc::kSmemBytes) != cudaSuccess) {
    set_last_error("cudaFuncSetAttribute(lmhead_tc_kernel) failed");
    return false;
  }
  // one box = 128 bytes of K (64 bf16 or 128 e4m3) x 256 rows
  const uint64_t es = fp8 ? 1 : 2;
  const uint64_t dA[2] = {(uint64_t)d, (uint64_t)M};
  const uint64_t sA[1] = {(uint64_t)d * es};
  const uint32_t bA[2] = {(uint32_t)(lmtc::kRowBytes / es), 256};
  const uint64_t dB[2] = {(uint64_t)d, (uint64_t)V};
  const uint32_t bB[2] = {(uint32_t)(lmtc::kRowBytes / es), (uint32_t)(lmtc::kMaxGran * lmtc::kGranule)};
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
  dim3 grid(part.P, ceil_div(M, 256));
  if (sa)
    launch_pdl(lmtc::lmhead_tc_kernel<true>, grid, dim3(lmtc::kThreads), lmtc::kSmemBytes, ex.stream, tmA, tmB, p);
  else
    launch_pdl(lmtc::lmhead_tc_kernel<false>, grid, dim3(lmtc::kThreads), lmtc::kSmemBytes, ex.stream, tmA, tmB, p);
  ex.launches++;
}

}  // namespace dg
