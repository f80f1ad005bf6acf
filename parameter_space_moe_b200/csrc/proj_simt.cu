// Grouped expert projection with the parameter-space mix in its epilogue, CUDA-core (SIMT) version.
// It serves the fp32 layer (whose 1e-5 accuracy rules out tensor-core rounding) and is the
// reference-grade kernel the tensor-core version is checked against.
//
// Paper: Swimba notes, key design 1: every active expert e projects X_t into its candidate streams
// (x^(e), B^(e), C^(e)), which are mixed in parameter space with the router weights:
//   Xs[m][j] = x^(j),   Bpi[m][j] = pi_mj B^(j),   Cpi[m][j] = pi_mj C^(j)   (C~_m = sum_j Cpi[m][j])
// Rows are (token, slot) pairs in expert-major order (see dispatch.cu); each CTA computes a
// kRowTile x 64 tile of one expert's output and writes every element straight to its stream.
#include "common.cuh"

namespace swimba {

constexpr int kSBM = kRowTile, kSBN = 64, kSBK = 16;

// Route one projected value to its stream.  c is the column of the expert output z = [x | B | C].
template <class S>
__device__ __forceinline__ void emit(const Dims& d, int mode, int p, int c, float v, float pi, S* bpi, S* xs, S* cpi,
                                     float* Z, unsigned* st) {
  if (mode == 2) { Z[(size_t)p * d.We + c] = v; return; }
  float o;
  S* dst;
  if (c < d.HP) { o = v; dst = xs + (size_t)p * d.HP + c; }
  else if (c < d.HP + d.GN) { o = mode == 1 ? v : pi * v; dst = bpi + (size_t)p * d.GN + (c - d.HP); }
  else { o = pi * v; dst = cpi + (size_t)p * d.GN + (c - d.HP - d.GN); }
  if (out_of_range<S>(o)) atomicOr(st, ST_RANGE);
  *dst = from_f32<S>(o);
}

template <class T, class S>
__global__ void __launch_bounds__(256)
proj_simt_kernel(Dims d, const T* __restrict__ X, const T* __restrict__ W, const int32_t* __restrict__ perm,
                 const int32_t* __restrict__ tiles, const int32_t* __restrict__ ntiles,
                 const int32_t* __restrict__ offsets, const float* __restrict__ topk_w, int mode, S* __restrict__ bpi,
                 S* __restrict__ xs, S* __restrict__ cpi, float* __restrict__ Z, unsigned* st) {
  __shared__ float As[kSBK][kSBM + 4];
  __shared__ float Bs[kSBK][kSBN + 4];
  __shared__ int tok_s[kSBM];
  if ((int)blockIdx.x >= *ntiles) return;
  const int e = tiles[2 * blockIdx.x], row0 = tiles[2 * blockIdx.x + 1];
  const int rows = min(kSBM, offsets[e + 1] - row0);
  const int n0 = blockIdx.y * kSBN;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  for (int r = tid; r < kSBM; r += 256) tok_s[r] = r < rows ? perm[row0 + r] / d.k : -1;
  __syncthreads();
  const T* We = W + (size_t)e * d.We * d.D;
  float acc[8][4] = {};
  for (int k0 = 0; k0 < d.D; k0 += kSBK) {
    for (int i = tid; i < kSBK * kSBM; i += 256) {
      int r = i / kSBK, kk = i % kSBK, t = tok_s[r];
      As[kk][r] = (t >= 0 && k0 + kk < d.D) ? to_f32(X[(size_t)t * d.D + k0 + kk]) : 0.f;
    }
    for (int i = tid; i < kSBK * kSBN; i += 256) {
      int c = i / kSBK, kk = i % kSBK;
      Bs[kk][c] = (n0 + c < d.We && k0 + kk < d.D) ? to_f32(We[(size_t)(n0 + c) * d.D + k0 + kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSBK; ++kk) {
      float a[8], b[4];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = ty + 16 * i;
    if (r >= rows) continue;
    const int p = perm[row0 + r];
    const float pi = mode == 2 ? 0.f : topk_w[p];  // raw mode has no router weights
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tx + 16 * j;
      if (c < d.We) emit<S>(d, mode, p, c, acc[i][j], pi, bpi, xs, cpi, Z, st);
    }
  }
}

template <class S>
__global__ void mix_kernel(Dims d, const float* __restrict__ Z, const float* __restrict__ topk_w, int flags,
                           S* __restrict__ bpi, S* __restrict__ xs, S* __restrict__ cpi, unsigned* st) {
  const size_t total = (size_t)d.M * d.k * d.We;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int p = (int)(i / d.We), c = (int)(i % d.We);
    emit<S>(d, (flags & SWIMBA_MIX_UNSCALED_B) ? 1 : 0, p, c, Z[i], topk_w[p], bpi, xs, cpi, nullptr, st);
  }
}

cudaError_t launch_proj_simt(const Dims& d, const void* X, const void* w_exp, const int32_t* perm,
                             const int32_t* tiles, const int32_t* ntiles, const int32_t* offsets,
                             const float* topk_w, int mode, void* bpi, void* xs, void* cpi, float* Z, unsigned* st,
                             cudaStream_t s) {
  dim3 grid(max_row_tiles(d), ceil_div(d.We, kSBN));
  if (d.dtype == SWIMBA_BF16)
    proj_simt_kernel<__nv_bfloat16, __half><<<grid, 256, 0, s>>>(
        d, (const __nv_bfloat16*)X, (const __nv_bfloat16*)w_exp, perm, tiles, ntiles, offsets, topk_w, mode,
        (__half*)bpi, (__half*)xs, (__half*)cpi, Z, st);
  else
    proj_simt_kernel<float, float><<<grid, 256, 0, s>>>(d, (const float*)X, (const float*)w_exp, perm, tiles,
                                                          ntiles, offsets, topk_w, mode, (float*)bpi, (float*)xs,
                                                          (float*)cpi, Z, st);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_mix(const Dims& d, const float* Z, const float* topk_w, int flags, void* bpi, void* xs, void* cpi,
                       unsigned* st, cudaStream_t s) {
  const int blocks = 148 * 8;
  if (d.dtype == SWIMBA_BF16)
    mix_kernel<__half><<<blocks, 256, 0, s>>>(d, Z, topk_w, flags, (__half*)bpi, (__half*)xs, (__half*)cpi, st);
  else
    mix_kernel<float><<<blocks, 256, 0, s>>>(d, Z, topk_w, flags, (float*)bpi, (float*)xs, (float*)cpi, st);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace swimba
