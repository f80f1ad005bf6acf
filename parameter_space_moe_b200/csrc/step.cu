// Recurrent decode step: one new token per sequence advances the cached state in place.
//
// Paper: Swimba notes, key design 1, second display equation, for a single token:
//   h <- a h + sum_j Bpi_j Xs_j^T,   y = C~^T h,   a = exp(dt A_h),   C~ = sum_j Cpi_j
// One CTA per (sequence, head) streams the N x P fp32 state once (read + write, 16-byte vectors);
// the readout reduces over n in registers and then across the CTA in shared memory.
#include "common.cuh"

namespace swimba {

constexpr int kStepThreads = 256;

template <class S, class T>
__global__ void __launch_bounds__(kStepThreads)
step_update_kernel(Dims d, const S* __restrict__ bpi, const S* __restrict__ xs, const S* __restrict__ cpi,
                   const float* __restrict__ dt, const float* __restrict__ A, float* __restrict__ state,
                   T* __restrict__ y) {
  extern __shared__ float sm[];
  const int P4 = d.P / 4;
  float* Bs = sm;                     // [k][N]
  float* Xv = Bs + d.k * d.N;         // [k][P]
  float* Cs = Xv + d.k * d.P;         // [N]
  float* red = Cs + d.N;              // [kStepThreads / P4][P]
  const int bh = blockIdx.x, b = bh / d.H, h = bh % d.H, g = h / d.hpg;
  for (int x = threadIdx.x; x < d.k * d.N; x += blockDim.x) {
    const int j = x / d.N, n = x % d.N;
    Bs[x] = to_f32(bpi[((size_t)b * d.k + j) * d.GN + (size_t)g * d.N + n]);
  }
  for (int x = threadIdx.x; x < d.k * d.P; x += blockDim.x) {
    const int j = x / d.P, p = x % d.P;
    Xv[x] = to_f32(xs[((size_t)b * d.k + j) * d.HP + (size_t)h * d.P + p]);
  }
  for (int n = threadIdx.x; n < d.N; n += blockDim.x) {
    float v = 0.f;
    for (int j = 0; j < d.k; ++j) v += to_f32(cpi[((size_t)b * d.k + j) * d.GN + (size_t)g * d.N + n]);
    Cs[n] = v;
  }
  __syncthreads();
  const float a = expf(dt[(size_t)b * d.H + h] * A[h]);
  float4* st = reinterpret_cast<float4*>(state + (size_t)bh * d.N * d.P);
  const int q = threadIdx.x % P4, ng = threadIdx.x / P4, nstride = kStepThreads / P4;
  float4 yacc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int n = ng; n < d.N; n += nstride) {
    float4 hv = st[n * P4 + q];
    float u0 = 0.f, u1 = 0.f, u2 = 0.f, u3 = 0.f;
    for (int j = 0; j < d.k; ++j) {
      const float bn = Bs[j * d.N + n];
      const float* xv = Xv + j * d.P + 4 * q;
      u0 = fmaf(bn, xv[0], u0); u1 = fmaf(bn, xv[1], u1); u2 = fmaf(bn, xv[2], u2); u3 = fmaf(bn, xv[3], u3);
    }
    hv.x = fmaf(a, hv.x, u0); hv.y = fmaf(a, hv.y, u1); hv.z = fmaf(a, hv.z, u2); hv.w = fmaf(a, hv.w, u3);
    st[n * P4 + q] = hv;
    const float cn = Cs[n];
    yacc.x = fmaf(cn, hv.x, yacc.x); yacc.y = fmaf(cn, hv.y, yacc.y);
    yacc.z = fmaf(cn, hv.z, yacc.z); yacc.w = fmaf(cn, hv.w, yacc.w);
  }
  if (ng < nstride) {
    float* r = red + ng * d.P + 4 * q;
    r[0] = yacc.x; r[1] = yacc.y; r[2] = yacc.z; r[3] = yacc.w;
  }
  __syncthreads();
  for (int p = threadIdx.x; p < d.P; p += blockDim.x) {
    float v = 0.f;
    for (int w = 0; w < nstride; ++w) v += red[w * d.P + p];
    y[(size_t)bh * d.P + p] = from_f32<T>(v);
  }
}

cudaError_t launch_step_update(const Dims& d, const void* bpi, const void* xs, const void* cpi, const float* dt,
                               const float* A, float* state, void* y, cudaStream_t s) {
  const int P4 = d.P / 4, nstride = kStepThreads / P4;
  size_t smem = sizeof(float) * ((size_t)d.k * d.N + (size_t)d.k * d.P + d.N + (size_t)nstride * d.P);
  if (d.dtype == SWIMBA_BF16)
    step_update_kernel<__half, __nv_bfloat16><<<d.Bsz * d.H, kStepThreads, smem, s>>>(
        d, (const __half*)bpi, (const __half*)xs, (const __half*)cpi, dt, A, state, (__nv_bfloat16*)y);
  else
    step_update_kernel<float, float><<<d.Bsz * d.H, kStepThreads, smem, s>>>(
        d, (const float*)bpi, (const float*)xs, (const float*)cpi, dt, A, state, (float*)y);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace swimba
