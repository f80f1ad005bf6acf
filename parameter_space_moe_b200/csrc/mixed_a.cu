// Expert-mixed diagonal transition: the parameter-space mixing carried over from (B, C, x) to the
// diagonal of A.
//
// Paper: Swimba notes, limitations and outlook -- the mixing is proposed for the diagonal components of
// the transition matrix, with Lyapunov stability kept.  Here every expert e has its own A_exp[e][h] per
// head, mixed with the router weights of the token's active set:
//   A~_t,h = sum_j pi_tj A_exp[K_tj][h],      a_t,h = exp(dt_t,h A~_t,h).
// A~ is a convex combination, so negative expert values give a negative A~ and 0 < a < 1: the layer still
// has one contracting trajectory, and the scan and decode kernels run unchanged on dA = dt A~ with A = 1.
// One thread per (token, head); the k (index, weight) pairs of a token are read once per head from L1.
#include "common.cuh"

namespace swimba {

namespace {
__global__ void mixed_a_kernel(Dims d, const int32_t* __restrict__ idx, const float* __restrict__ wts,
                               const float* __restrict__ A_exp, const float* __restrict__ dt, float* __restrict__ dA,
                               float* __restrict__ ones, unsigned* st) {
  const size_t total = (size_t)d.M * d.H;
  bool bad_index = false, unstable = false;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const size_t m = i / d.H;
    const int h = (int)(i % d.H);
    float a = 0.f;
    for (int j = 0; j < d.k; ++j) {
      const int e = idx[m * d.k + j];
      if (e < 0 || e >= d.E) { bad_index = true; continue; }
      a = fmaf(wts[m * d.k + j], A_exp[(size_t)e * d.H + h], a);
    }
    unstable |= !(a < 0.f);
    dA[i] = dt[i] * a;
    if (i < (size_t)d.H) ones[i] = 1.f;
  }
  if (bad_index) atomicOr(st, ST_INDEX);
  if (unstable) atomicOr(st, ST_UNSTABLE);
}
}  // namespace

cudaError_t launch_mixed_a(const Dims& d, const int32_t* idx, const float* wts, const float* A_exp, const float* dt,
                           float* dA, float* ones, unsigned* st, cudaStream_t s) {
  const long long total = (long long)d.M * d.H;
  const int blocks = (int)std::min<long long>((total + 255) / 256, 148LL * 8);
  mixed_a_kernel<<<blocks, 256, 0, s>>>(d, idx, wts, A_exp, dt, dA, ones, st);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace swimba
