// Device-side helpers shared by the canvas-denoise kernels: storage-type
// conversion, the Philox-4x64-10 generator, the device error word.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dg {

// ---------------------------------------------------------------- error word
// Device code records the first failure here (atomicCAS from 0) and carries on
// without trapping; the host reads it at the next synchronous call.
enum DeviceError : int {
  kDevOk = 0,
  kDevBadToken = 1,      // a canvas token id outside [0, vocab)
  kDevNanEntropy = 2,    // entropy not finite
  kDevWaitTimeout = 3,   // a bounded mbarrier wait gave up
  kDevBadShape = 4,      // a kernel was launched on shapes it does not support
  kDevBadAlign = 5,      // shared memory not aligned as a kernel's tile layout needs
  kDevLoopCap = 6,       // a device-side decode loop reached its step cap with a canvas not done
};

__device__ __forceinline__ void set_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// ---------------------------------------------------------------- storage types
template <typename T> struct Storage;
template <> struct Storage<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Storage<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// ---------------------------------------------------------------- Philox-4x64-10
// Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3"
// (SC'11): per round, two 64x64->128 multiplies; the high halves are XORed
// with the other two counter words and the key; the key advances by the Weyl
// constants between rounds.
struct Philox4x64Out { uint64_t x0, x1, x2, x3; };

__host__ __device__ __forceinline__ void mulhilo64(uint64_t a, uint64_t b, uint64_t& hi, uint64_t& lo) {
#ifdef __CUDA_ARCH__
  lo = a * b;
  hi = __umul64hi(a, b);
#else
  unsigned __int128 p = (unsigned __int128)a * b;
  lo = (uint64_t)p;
  hi = (uint64_t)(p >> 64);
#endif
}

__host__ __device__ __forceinline__ Philox4x64Out philox4x64_10(uint64_t c0, uint64_t c1, uint64_t c2,
                                                                uint64_t c3, uint64_t k0, uint64_t k1) {
  const uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
  const uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) { k0 += W0; k1 += W1; }
    uint64_t hi0, lo0, hi1, lo1;
    mulhilo64(M0, c0, hi0, lo0);
    mulhilo64(M1, c2, hi1, lo1);
    uint64_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
  }
  return {c0, c1, c2, c3};
}

// Token id of canvas `canvas`, position `pos` at noise step `step`:
// key (seed, 0), counter (pos, step, canvas, 0), word 0, top 32 bits scaled
// to the vocabulary by multiply-shift (exactly uniform for power-of-two V).
__host__ __device__ __forceinline__ int32_t canvas_draw(uint64_t seed, uint32_t step, uint32_t pos,
                                                        uint32_t canvas, uint32_t vocab) {
  Philox4x64Out o = philox4x64_10(pos, step, canvas, 0, seed, 0);
  return (int32_t)(((o.x0 >> 32) * (uint64_t)vocab) >> 32);
}

// ---------------------------------------------------------------- launch order
// Programmatic dependent launch: a kernel may start while its predecessor in
// the stream is still running. Each kernel calls griddep_launch() early (its
// dependents may then be scheduled) and griddep_wait() before it touches any
// memory a predecessor writes (or reads); work before the wait is limited to
// set-up and loads of read-only weights.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- misc
__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Online (max, Z, S) entropy accumulator for one row: after folding the
// scaled logits l_j, with m = max l_j:  Z = sum exp(l_j - m),
// S = sum (l_j - m) exp(l_j - m), and the entropy is ln Z - S / Z.
// Argmax is tracked separately on the unscaled logits (lowest id on ties).
struct EntStats {
  float m, z, s, best;
  int32_t idx;
};

__device__ __forceinline__ EntStats ent_empty() { return {-INFINITY, 0.f, 0.f, -INFINITY, 0x7fffffff}; }

// Merge two partial states; argmax ties resolve to the lower vocab id.
__device__ __forceinline__ EntStats ent_merge(EntStats a, EntStats b) {
  EntStats r;
  float m = fmaxf(a.m, b.m);
  if (m == -INFINITY) {
    r.m = m; r.z = 0.f; r.s = 0.f;
  } else {
    float ea = (a.m == -INFINITY) ? 0.f : __expf(a.m - m);
    float eb = (b.m == -INFINITY) ? 0.f : __expf(b.m - m);
    // S relative to the new maximum: e^(m_i - m) * (S_i + (m_i - m) Z_i)
    float sa = (a.m == -INFINITY) ? 0.f : ea * (a.s + (a.m - m) * a.z);
    float sb = (b.m == -INFINITY) ? 0.f : eb * (b.s + (b.m - m) * b.z);
    r.m = m;
    r.z = ea * a.z + eb * b.z;
    r.s = sa + sb;
  }
  if (b.best > a.best || (b.best == a.best && b.idx < a.idx)) {
    r.best = b.best; r.idx = b.idx;
  } else {
    r.best = a.best; r.idx = a.idx;
  }
  return r;
}

}  // namespace dg
