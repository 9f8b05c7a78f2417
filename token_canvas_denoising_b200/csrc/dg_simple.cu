// CUDA-core kernels for the f32 storage dtype (the tiny configuration), where
// the tensor-core formats would round operands: embedding gather, projection
// GEMM with optional residual, bidirectional GQA attention, and the LM head
// with the online entropy/argmax fold.
#include "dg_internal.cuh"

namespace dg {

// ------------------------------------------------------------------ embed
// X[r, :] = E[tok[r], :]  (a row gather; 16-byte vector copies).
template <typename T>
__global__ void embed_kernel(const T* __restrict__ E, const int32_t* __restrict__ tok,
                             T* __restrict__ X, int d, int V, int* err) {
  griddep_launch();
  griddep_wait();
  const int r = blockIdx.x;
  int t = tok[r];
  if (t < 0 || t >= V) {
    if (threadIdx.x == 0) set_error(err, kDevBadToken);
    t = 0;
  }
  const uint4* src = reinterpret_cast<const uint4*>(E + (size_t)t * d);
  uint4* dst = reinterpret_cast<uint4*>(X + (size_t)r * d);
  const int n = d * (int)sizeof(T) / 16;
  for (int i = threadIdx.x; i < n; i += blockDim.x) dst[i] = src[i];
}

void launch_embed(Exec& ex, int dtype, const void* E, const int32_t* tok, void* X, int M, int d, int V) {
  if (dtype == DG_F32)
    embed_kernel<float><<<M, 128, 0, ex.stream>>>((const float*)E, tok, (float*)X, d, V, ex.err);
  else
    launch_pdl(embed_kernel<__nv_bfloat16>, dim3(M), dim3(128), 0, ex.stream, (const __nv_bfloat16*)E, tok,
               (__nv_bfloat16*)X, d, V, ex.err);
  ex.launches++;
}

// ------------------------------------------------------------------ linear
// out[M][N] = A[M][K] W[N][K]^T (+ R[M][N]); fp32 accumulate, one rounding to
// the storage type at the end. 32x32 output tile, 256 threads.
template <typename T>
__global__ void linear_simple_kernel(const T* __restrict__ A, const T* __restrict__ W,
                                     const T* __restrict__ R, T* __restrict__ out, int M, int N, int K) {
  __shared__ float As[32][33];
  __shared__ float Ws[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int row0 = blockIdx.y * 32, col0 = blockIdx.x * 32;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < K; k0 += 32) {
    for (int i = ty; i < 32; i += 8) {
      const int k = k0 + tx;
      const int r = row0 + i, n = col0 + i;
      As[i][tx] = (r < M && k < K) ? Storage<T>::to_f(A[(size_t)r * K + k]) : 0.f;
      Ws[i][tx] = (n < N && k < K) ? Storage<T>::to_f(W[(size_t)n * K + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      const float w = Ws[tx][kk];
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j] = fmaf(As[ty + 8 * j][kk], w, acc[j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int r = row0 + ty + 8 * j, n = col0 + tx;
    if (r < M && n < N) {
      float v = acc[j];
      if (R) v += Storage<T>::to_f(R[(size_t)r * N + n]);
      out[(size_t)r * N + n] = Storage<T>::from_f(v);
    }
  }
}

void launch_linear_simple(Exec& ex, int dtype, const void* A, const void* W, const void* R, void* out,
                          int M, int N, int K) {
  dim3 grid(ceil_div(N, 32), ceil_div(M, 32));
  if (dtype == DG_F32)
    linear_simple_kernel<float><<<grid, 256, 0, ex.stream>>>((const float*)A, (const float*)W,
                                                             (const float*)R, (float*)out, M, N, K);
  else
    linear_simple_kernel<__nv_bfloat16><<<grid, 256, 0, ex.stream>>>(
        (const __nv_bfloat16*)A, (const __nv_bfloat16*)W, (const __nv_bfloat16*)R,
        (__nv_bfloat16*)out, M, N, K);
  ex.launches++;
}

// ------------------------------------------------------------------ attention
// One warp per (request b, query head q, canvas position p): online softmax
// over the S_b prefix keys then the C canvas keys of KV head g = q / (Hq/Hk);
// no mask. Each lane owns HPL consecutive head dimensions.
template <typename T, int HPL>
__global__ void attn_simple_kernel(const T* __restrict__ Q, const PrefixDesc* __restrict__ pre,
                                   const T* __restrict__ Kc, const T* __restrict__ Vc, T* __restrict__ O,
                                   int B, int C, int Hq, int Hk, float scale) {
  const int h = HPL * 32;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= B * C * Hq) return;
  const int q = warp % Hq, row = warp / Hq, b = row / C;
  const int g = q / (Hq / Hk);
  float qv[HPL], o[HPL];
#pragma unroll
  for (int i = 0; i < HPL; ++i) {
    qv[i] = Storage<T>::to_f(Q[((size_t)row * Hq + q) * h + lane * HPL + i]);
    o[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  auto fold = [&](const T* kp, const T* vp) {
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < HPL; ++i) dot = fmaf(qv[i], Storage<T>::to_f(kp[lane * HPL + i]), dot);
    dot = warp_sum(dot) * scale;
    const float mn = fmaxf(m, dot);
    const float corr = expf(m - mn);
    const float p = expf(dot - mn);
    l = l * corr + p;
#pragma unroll
    for (int i = 0; i < HPL; ++i) o[i] = fmaf(o[i], corr, p * Storage<T>::to_f(vp[lane * HPL + i]));
    m = mn;
  };
  const T* pk = static_cast<const T*>(pre[b].k);
  const T* pv = static_cast<const T*>(pre[b].v);
  const int S = pre[b].len;
  for (int j = 0; j < S; ++j) fold(pk + ((size_t)j * Hk + g) * h, pv + ((size_t)j * Hk + g) * h);
  for (int j = 0; j < C; ++j) {
    const size_t off = ((size_t)(b * C + j) * Hk + g) * h;
    fold(Kc + off, Vc + off);
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int i = 0; i < HPL; ++i) O[((size_t)row * Hq + q) * h + lane * HPL + i] = Storage<T>::from_f(o[i] * inv);
}

template <typename T>
static void attn_simple_dispatch(Exec& ex, const void* Qv, const PrefixDesc* pre, const void* Kcv,
                                 const void* Vcv, void* Ov, const AttnShape& sh) {
  const int warps = sh.B * sh.C * sh.Hq;
  const int blocks = ceil_div(warps, 8);
  const float scale = 1.f / sqrtf((float)sh.h);
  const T* Q = (const T*)Qv;
  const T* Kc = (const T*)Kcv;
  const T* Vc = (const T*)Vcv;
  T* O = (T*)Ov;
  switch (sh.h / 32) {
    case 1: attn_simple_kernel<T, 1><<<blocks, 256, 0, ex.stream>>>(Q, pre, Kc, Vc, O, sh.B, sh.C, sh.Hq, sh.Hk, scale); break;
    case 2: attn_simple_kernel<T, 2><<<blocks, 256, 0, ex.stream>>>(Q, pre, Kc, Vc, O, sh.B, sh.C, sh.Hq, sh.Hk, scale); break;
    case 3: attn_simple_kernel<T, 3><<<blocks, 256, 0, ex.stream>>>(Q, pre, Kc, Vc, O, sh.B, sh.C, sh.Hq, sh.Hk, scale); break;
    default: attn_simple_kernel<T, 4><<<blocks, 256, 0, ex.stream>>>(Q, pre, Kc, Vc, O, sh.B, sh.C, sh.Hq, sh.Hk, scale); break;
  }
}

void launch_attention_simple(Exec& ex, int dtype, const void* Q, const PrefixDesc* d_prefix, const void* Kc,
                             const void* Vc, void* O, const AttnShape& s) {
  if (dtype == DG_F32) attn_simple_dispatch<float>(ex, Q, d_prefix, Kc, Vc, O, s);
  else attn_simple_dispatch<__nv_bfloat16>(ex, Q, d_prefix, Kc, Vc, O, s);
  ex.launches++;
}

// ------------------------------------------------------------------ LM head
// One warp per row and vocab range: logit x_v = Hs[r] . W[v] (fp32), folded
// into the row's online entropy state with l_v = x_v * invT[r]; the argmax
// runs on x_v. Vocab ids are visited in increasing order, so a strict '>'
// keeps the lowest id among equal maxima. Writes one partial per (range, row).
template <typename T>
__global__ void lmhead_simple_kernel(const T* __restrict__ Hs, const T* __restrict__ W,
                                     const float* __restrict__ invT, LmPartials part, int M, int d,
                                     int V, int chunk) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y * 8 + warp;
  if (r >= M) return;
  const int v0 = blockIdx.x * chunk, v1 = min(V, v0 + chunk);
  const float it = invT ? invT[r] : 1.f;
  const T* hrow = Hs + (size_t)r * d;
  float m = -INFINITY, z = 0.f, s = 0.f, best = -INFINITY;
  int idx = 0x7fffffff;
  for (int v = v0; v < v1; ++v) {
    const T* wrow = W + (size_t)v * d;
    float dot = 0.f;
    for (int k = lane; k < d; k += 32) dot = fmaf(Storage<T>::to_f(hrow[k]), Storage<T>::to_f(wrow[k]), dot);
    dot = warp_sum(dot);
    if (dot > best) { best = dot; idx = v; }
    const float l = dot * it;
    if (l > m) {
      if (z > 0.f) {
        const float cr = expf(m - l);
        s = cr * (s + (m - l) * z);
        z = cr * z;
      }
      m = l;
    }
    const float e = expf(l - m);
    z += e;
    s = fmaf(l - m, e, s);
  }
  if (lane == 0) {
    LmRec rec;
    rec.m = m; rec.z = z; rec.s = s; rec.best = best; rec.idx = idx;
    rec.pad0 = rec.pad1 = rec.pad2 = 0;
    part.rec[(size_t)r * part.P + blockIdx.x] = rec;
  }
}

void launch_lmhead_simple(Exec& ex, int dtype, const void* hs, const void* W, const float* invT,
                          LmPartials part, int M, int d, int V) {
  const int chunk = ceil_div(V, part.P);
  dim3 grid(part.P, ceil_div(M, 8));
  if (dtype == DG_F32)
    lmhead_simple_kernel<float><<<grid, 256, 0, ex.stream>>>((const float*)hs, (const float*)W, invT, part, M,
                                                             d, V, chunk);
  else
    lmhead_simple_kernel<__nv_bfloat16><<<grid, 256, 0, ex.stream>>>(
        (const __nv_bfloat16*)hs, (const __nv_bfloat16*)W, invT, part, M, d, V, chunk);
  ex.launches++;
}

}  // namespace dg
