// e4m3 quantization of the residual stream ahead of the FP8 LM head (the FP8
// deployment of "DiffusionGemma深度拆解：从逐字蹦到整块喷，LLM生成范式的结构性跃迁",
// 性能数据; "谷歌DiffusionGemma：并行生成与自纠的新突破", 引入扩散机制).
//
// Each row r of Hs gets the smallest power-of-two scale 2^e_r with
// 448 * 2^e_r >= max |Hs[r]| (448 is the largest finite e4m3 value): with
// max |Hs[r]| = f 2^k, f in [0.5, 1) (frexp), e_r = k - 9 when f <= 0.875,
// else k - 8. The row is divided by 2^e_r (exact) and each value rounded to
// the nearest e4m3 value, ties to even; no value exceeds 448, so saturation
// never applies. One warp per row, 8 bf16 per lane per pass.
#include <cuda_fp8.h>

#include "dg_internal.cuh"

namespace dg {

__global__ void __launch_bounds__(256) quantize_rows_e4m3_kernel(const __nv_bfloat16* __restrict__ x,
                                                                 uint8_t* __restrict__ q,
                                                                 float* __restrict__ scales, int M, int d) {
  griddep_launch();
  griddep_wait();
  const int row = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const __nv_bfloat16* xr = x + (size_t)row * d;
  float amax = 0.f;
  for (int c = lane * 8; c < d; c += 256) {
    const uint4 u = *reinterpret_cast<const uint4*>(xr + c);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(h[j]);
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  int k = 0;
  const float f = frexpf(amax, &k);
  const int e = amax > 0.f ? (f <= 0.875f ? k - 9 : k - 8) : 0;
  const float inv = ldexpf(1.f, -e);
  if (lane == 0) scales[row] = ldexpf(1.f, e);
  uint8_t* qr = q + (size_t)row * d;
  for (int c = lane * 8; c < d; c += 256) {
    const uint4 u = *reinterpret_cast<const uint4*>(xr + c);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 fv = __bfloat1622float2(h[j]);
      const uint32_t b0 = __nv_cvt_float_to_fp8(fv.x * inv, __NV_SATFINITE, __NV_E4M3);
      const uint32_t b1 = __nv_cvt_float_to_fp8(fv.y * inv, __NV_SATFINITE, __NV_E4M3);
      w[j >> 1] |= (b0 | (b1 << 8)) << ((j & 1) * 16);
    }
    *reinterpret_cast<uint2*>(qr + c) = make_uint2(w[0], w[1]);
  }
}

void launch_quantize_rows_e4m3(Exec& ex, const void* x, uint8_t* codes, float* scales, int M, int d) {
  launch_pdl(quantize_rows_e4m3_kernel, dim3(ceil_div(M, 8)), dim3(256), 0, ex.stream,
             static_cast<const __nv_bfloat16*>(x), codes, scales, M, d);
  ex.launches++;
}

}  // namespace dg
