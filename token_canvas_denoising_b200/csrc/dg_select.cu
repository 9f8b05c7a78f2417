// Canvas bookkeeping kernels: the initial random canvas, and the fused
// "merge LM-head partials -> entropy/argmax -> freeze -> stop test ->
// re-noise" tail of every denoise step.
//
// Method ("DiffusionGemma解析：扩散模型如何让LLM快5倍", 整片并行去噪 and
// 自适应停步机制; "谷歌DiffusionGemma：并行生成与自纠的新突破", 工作原理):
// positions are ordered by entropy, the most certain ones are locked to the
// model's most likely token, every other position is re-randomised, and the
// block stops once enough positions are settled (at most 48 steps).
#include "dg_internal.cuh"

namespace dg {

// ------------------------------------------------------------------ init
// tok[b][p] = draw(seed_b, step 0, p, b); nothing frozen; step 0; not done.
__global__ void init_canvas_kernel(int32_t* tok, uint8_t* frozen, int32_t* step, const uint64_t* seed,
                                   uint8_t* done, int32_t* all_done, int C, int V) {
  const int b = blockIdx.x;
  for (int p = threadIdx.x; p < C; p += blockDim.x) {
    tok[b * C + p] = canvas_draw(seed[b], 0u, (uint32_t)p, (uint32_t)b, (uint32_t)V);
    frozen[b * C + p] = 0;
  }
  if (threadIdx.x == 0) {
    step[b] = 0;
    done[b] = 0;
    if (b == 0) *all_done = 0;
  }
}

void launch_init_canvas(Exec& ex, const CanvasState& cs, int B, int C, int V) {
  init_canvas_kernel<<<B, 256, 0, ex.stream>>>(cs.tok, cs.frozen, cs.step, cs.seed, cs.done, cs.all_done, C, V);
  ex.launches++;
}

// ------------------------------------------------------------------ merge + select
struct SelectArgs {
  LmPartials part;
  float* ent;           // [M]
  int32_t* am;          // [M]
  uint8_t* fmask;       // [M] or null
  int32_t* tok;
  uint8_t* frozen;
  int32_t* step;
  const uint64_t* seed;
  uint8_t* done;
  int32_t* all_done;
  uint32_t* counters;   // [B + 1], zero on entry, left zero
  int32_t* loop_iter;   // steps of the device-side decode loop (with cond)
  cudaGraphConditionalHandle cond;  // 0, or the decode loop's condition
  int loop_cap;
  int32_t* err;
  int B, C, V, max_steps, adaptive;
  float stop_entropy;
  int select;           // 0: only merge the partials into ent / am
};

__device__ __forceinline__ EntStats load_rec(const LmRec* r) {
  const float4 a = __ldcg(reinterpret_cast<const float4*>(r));
  const int4 b = __ldcg(reinterpret_cast<const int4*>(r) + 1);
  return {a.x, a.y, a.z, a.w, b.x};
}

// Orderable 32-bit image of a float (total order, negatives below positives).
__device__ __forceinline__ uint32_t float_order(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kMaxRecPerLane = 8;  // partials preloaded per lane (P <= 256 in one pass)
constexpr int kMaxSelect = 1024;   // positions per canvas the selection sorts (one per thread)

// Ascending bitonic sort of one 64-bit key per thread across the block
// (blockDim.x a power of two, at most kMaxSelect): compare-exchange stages
// with partner distances below 32 run inside a warp through shuffles, the
// others through shared memory. Afterwards thread t holds the t-th smallest.
__device__ __forceinline__ unsigned long long block_bitonic_sort(unsigned long long key,
                                                                 unsigned long long* s_x) {
  const int t = threadIdx.x, n = blockDim.x;
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      unsigned long long other;
      if (stride >= 32) {
        s_x[t] = key;
        __syncthreads();
        other = s_x[t ^ stride];
        __syncthreads();
      } else {
        other = __shfl_xor_sync(0xffffffffu, key, stride);
      }
      const bool up = (t & size) == 0;      // this run is sorted ascending
      const bool lower = (t & stride) == 0;  // lower element of the pair
      key = (lower == up) ? (other < key ? other : key) : (other > key ? other : key);
    }
  }
  return key;
}

// Grid (ceil(C / (blockDim/32)), B), blockDim the power of two >= C between
// 256 and 1024. Phase 1: one warp per canvas row folds the row's P partials
// (lane j takes partials j, j+32, ..., all loaded before the fold; then a
// fixed xor butterfly), giving ent = ln Z - S/Z and the argmax. Phase 2 runs
// in the last block of each canvas to arrive: the unfrozen positions' keys
// (entropy, position) are sorted across the block (frozen and padding slots
// sort last); the first k freeze to their argmax; stop test; re-noise. The
// last canvas to finish sets the all-done flag (and ends a device-side decode
// loop).
// kLoop: the step is the body of a device-side decode loop (a.cond set); only
// that instantiation contains the call that sets the loop's condition.
template <bool kLoop>
__global__ void __launch_bounds__(kMaxSelect) merge_select_kernel(SelectArgs a) {
  griddep_launch();
  griddep_wait();
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p_row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (p_row < a.C) {
    const int r = b * a.C + p_row;
    const LmRec* rec = a.part.rec + (size_t)r * a.part.P;
    EntStats st = ent_empty();
    for (int j0 = 0; j0 < a.part.P; j0 += 32 * kMaxRecPerLane) {
      EntStats buf[kMaxRecPerLane];
#pragma unroll
      for (int u = 0; u < kMaxRecPerLane; ++u) {
        const int j = j0 + lane + 32 * u;
        buf[u] = (j < a.part.P) ? load_rec(rec + j) : ent_empty();
      }
#pragma unroll
      for (int u = 0; u < kMaxRecPerLane; ++u) st = ent_merge(st, buf[u]);
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      EntStats ot;
      ot.m = __shfl_xor_sync(0xffffffffu, st.m, o);
      ot.z = __shfl_xor_sync(0xffffffffu, st.z, o);
      ot.s = __shfl_xor_sync(0xffffffffu, st.s, o);
      ot.best = __shfl_xor_sync(0xffffffffu, st.best, o);
      ot.idx = __shfl_xor_sync(0xffffffffu, st.idx, o);
      st = (lane & o) ? ent_merge(ot, st) : ent_merge(st, ot);
    }
    if (lane == 0) {
      float e = logf(st.z) - st.s / st.z;
      if (!isfinite(e)) set_error(a.err, kDevNanEntropy);
      a.ent[r] = e;
      a.am[r] = st.idx;
    }
  }
  if (!a.select) return;
  // ---- arrival: the last block of canvas b runs the selection
  __shared__ int s_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(&a.counters[b], 1u);
    s_last = (prev == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  __shared__ unsigned long long s_x[kMaxSelect];
  __shared__ uint8_t s_freeze[kMaxSelect];
  __shared__ float s_min[kMaxSelect / 32];
  const int p = threadIdx.x;
  const bool valid = p < a.C;
  const int r = b * a.C + p;
  // this block runs alone on the step's critical path: every load it needs
  // is issued here together, and the re-noise draw (which depends only on
  // the seed, the step and the position) is computed before the sort
  const bool canvas_done = __ldcg(&a.done[b]) != 0;
  float e = valid ? __ldcg(&a.ent[r]) : INFINITY;
  const bool unf = valid && __ldcg(&a.frozen[r]) == 0;
  const int amv = valid ? __ldcg(&a.am[r]) : 0;
  const int t = __ldcg(&a.step[b]);
  const uint64_t seed = __ldcg(&a.seed[b]);
  if (canvas_done) {
    if (valid && a.fmask) a.fmask[r] = 0;
  } else {
    const int32_t draw = unf ? canvas_draw(seed, (uint32_t)(t + 1), (uint32_t)p, (uint32_t)b, (uint32_t)a.V) : 0;
    if (!(e == e)) e = INFINITY;  // NaN (already flagged) orders last
    // key = (entropy, position); frozen and padding slots sort after every unfrozen one
    const unsigned long long key =
        unf ? (((unsigned long long)float_order(e) << 32) | (unsigned)p) : ~0ull;
    const int U = __syncthreads_count(unf);
    const int left = a.max_steps - t;
    const int k = (left <= 1) ? U : (U + left - 1) / left;
    const unsigned long long sorted = block_bitonic_sort(key, s_x);
    s_freeze[p] = 0;
    __syncthreads();
    if (p < k) s_freeze[(unsigned)(sorted & 0xffffffffu)] = 1;  // k <= U: an unfrozen position
    __syncthreads();
    const bool F = unf && s_freeze[p];
    if (F) {
      a.tok[r] = amv;
      a.frozen[r] = 1;
    }
    const bool rest = unf && !F;
    // smallest entropy among positions still unfrozen after this freeze
    float mr = rest ? e : INFINITY;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mr = fminf(mr, __shfl_xor_sync(0xffffffffu, mr, o));
    if (lane == 0) s_min[warp] = mr;
    const int R = __syncthreads_count(rest);
    float min_rest = s_min[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) min_rest = fminf(min_rest, s_min[w]);
    const bool stop = (R == 0) || (a.adaptive && min_rest < a.stop_entropy);
    if (stop) {
      if (rest) a.tok[r] = amv;
      if (valid) a.frozen[r] = 1;
    } else if (rest) {
      a.tok[r] = draw;
    }
    if (valid && a.fmask) a.fmask[r] = F ? 1 : 0;
    if (threadIdx.x == 0) {
      a.step[b] = t + 1;
      if (stop) a.done[b] = 1;
    }
  }
  // ---- canvas finished: reset its counter; the last canvas sets all_done
  if (threadIdx.x == 0) {
    a.counters[b] = 0;
    __threadfence();
    const unsigned prev = atomicAdd(&a.counters[a.B], 1u);
    if (prev == (unsigned)a.B - 1) {
      __threadfence();
      int all = 1;
      for (int i = 0; i < a.B; ++i) all &= (__ldcg(&a.done[i]) != 0) ? 1 : 0;
      *a.all_done = all;
      a.counters[a.B] = 0;
      if constexpr (kLoop) {  // the step is the body of a device-side decode loop
        const int it = *a.loop_iter + 1;
        *a.loop_iter = it;
        if (!all && it >= a.loop_cap) set_error(a.err, kDevLoopCap);
        cudaGraphSetConditional(a.cond, (!all && it < a.loop_cap) ? 1u : 0u);
      }
    }
  }
}

void launch_merge_select(Exec& ex, LmPartials part, float* ent, int32_t* am, uint8_t* fmask,
                         const CanvasState* cs, const dg_schedule* sched, int B, int C, int V,
                         const DecodeLoop* loop) {
  SelectArgs a{};
  a.part = part;
  a.ent = ent;
  a.am = am;
  a.fmask = fmask;
  a.err = ex.err;
  a.B = B;
  a.C = C;
  a.V = V;
  a.select = (cs && sched) ? 1 : 0;
  if (a.select) {
    a.tok = cs->tok;
    a.frozen = cs->frozen;
    a.step = cs->step;
    a.seed = cs->seed;
    a.done = cs->done;
    a.all_done = cs->all_done;
    a.counters = cs->counters;
    a.max_steps = sched->max_steps;
    a.adaptive = sched->adaptive_stop;
    a.stop_entropy = sched->stop_entropy;
    a.loop_iter = cs->loop_iter;
    if (loop) {
      a.cond = loop->handle;
      a.loop_cap = loop->cap;
    }
  }
  // one thread per position in the selection: the power of two >= C, at
  // least 256 (phase 1 then folds blockDim/32 rows per block)
  int threads = 256;
  while (threads < C && threads < kMaxSelect) threads <<= 1;
  dim3 grid(ceil_div(C, threads / 32), B);
  if (a.cond)
    launch_pdl(merge_select_kernel<true>, grid, dim3(threads), 0, ex.stream, a);
  else
    launch_pdl(merge_select_kernel<false>, grid, dim3(threads), 0, ex.stream, a);
  ex.launches++;
}

}  // namespace dg
